// Stage 1 (query-cluster summaries, selection) and stage 2 (far field +
// exact retrieval, one softmax) of MuSe, plus the causal local block and the
// merge of the hierarchical levels.
//
// Sources: the gist.science page "Multipole Semantic Attention: A Fast
// Approximation of Softmax Attention for Pretraining", Technical Summary,
// Core Mechanisms (residual decomposition; Stage 1 (Coarse); Stage 2
// (Refinement); Exponential Tilting; Cluster Selection; Exact Attention), and
// the newx.sg page of the same title, Abstract (monopole + dipole;
// hierarchical block decomposition).
//
// With nu_i the query-cluster centroid, mu_j the key-cluster centroid and
// k~ = k - mu_j, the kept terms of exp(s (nu_i + q~).(mu_j + k~)) give per key
// cluster j, as seen from query cluster i:
//   MONOPOLE  W_ij = n_j,                     u_ij = S_j / n_j
//   DIPOLE    W_ij = n_j,                     u_ij = sum_t v_t (1 + s nu_i.k~_t) / n_j
//             (= (S_j + s M_j nu_i) / n_j, the dipole moment contracted with
//             nu_i, evaluated without forming M_j)
//   TILTED    w_t = exp(s nu_i.k~_t), W_ij = sum w_t, u_ij = sum w_t v_t / W_ij,
//             k_hat_ij = sum w_t k_t / W_ij
// and the far-field logit of a query q of cluster i is
//   s q.mu_j + log W_ij                                   (MONOPOLE, DIPOLE)
//   s q.k_hat_ij + s nu_i.(mu_j - k_hat_ij) + log W_ij    (TILTED)
#include <cuda_fp16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace muse {

// ----------------------------------------------------------------------------
// stage 1: one CTA per (query problem, key cluster j).  The cluster's members
// (k - mu_j and v) are staged in shared memory once; query centroids come in
// chunks of 32.  For each chunk the CTA forms a_ti = s nu_i.k~_t, the weights
// (1 + a for DIPOLE, exp(a - max) for TILTED) and the weighted sums over the
// members, giving u_ij, log W_ij, the far-field key row and logit offset.
// ----------------------------------------------------------------------------
// Stage-1 table stores in the form the stage-2 kernel of the input dtype reads.
__device__ inline void put_u(const Stage1& s1, size_t i, float v) {
  if (s1.Uh) {
    const __half hi = __float2half_rn(v);
    s1.Uh[i] = hi;
    s1.Ul[i] = __float2half_rn(v - __half2float(hi));
  } else {
    s1.U[i] = v;
  }
}
__device__ inline void put_kf(const Stage1& s1, size_t i, float v) {
  if (s1.Kfh) {
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    s1.Kfh[i] = hi;
    s1.Kfl[i] = __float2bfloat16_rn(v - __bfloat162float(hi));
  } else {
    s1.Kf[i] = v;
  }
}

constexpr int kS1T = 256;  // threads
constexpr int kS1M = 128;  // members per staged chunk
constexpr int kS1I = 32;   // query clusters per pass

template <int D>
constexpr size_t stage1_smem() {
  return sizeof(float) * ((size_t)2 * kS1M * (D + 1) + (size_t)kS1I * (D + 1) +
                          (size_t)kS1M * (kS1I + 1) + (size_t)kS1I * D + D + 3 * kS1I);
}

template <typename T, int D>
__global__ void __launch_bounds__(kS1T) stage1_kernel(AttnArgs a, Stage1 s1, int qp0) {
  constexpr int GROUPS = kS1T / D;      // query-cluster lanes per pass
  constexpr int R = kS1I / GROUPS;      // outputs (i, e) per thread
  extern __shared__ float sm1[];
  float(*kt)[D + 1] = reinterpret_cast<float(*)[D + 1]>(sm1);
  float(*vt)[D + 1] = reinterpret_cast<float(*)[D + 1]>(sm1 + kS1M * (D + 1));
  float(*nu)[D + 1] = reinterpret_cast<float(*)[D + 1]>(sm1 + 2 * kS1M * (D + 1));
  float(*ws)[kS1I + 1] = reinterpret_cast<float(*)[kS1I + 1]>(sm1 + 2 * kS1M * (D + 1) + kS1I * (D + 1));
  float(*red)[D] = reinterpret_cast<float(*)[D]>(sm1 + 2 * kS1M * (D + 1) + kS1I * (D + 1) +
                                                 kS1M * (kS1I + 1));
  float* mu = reinterpret_cast<float*>(red) + kS1I * D;
  float* mrun = mu + D;
  float* zrun = mrun + kS1I;
  float* rsc = zrun + kS1I;

  const int lq = blockIdx.x, qpid = qp0 + lq, j = blockIdx.y;
  const Prob pq = prob_of(a.qg, qpid);
  const int kpid = kv_problem(a, qpid);
  const Prob pk = prob_of(a.kg, kpid);
  if (j >= pk.C) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Cq = a.Cq, Ck = a.Ck;
  const int nj = a.ks.counts[(size_t)kpid * Ck + j];
  const size_t ij0 = ((size_t)lq * Cq) * Ck + j;  // + i * Ck
  if (nj == 0) {
    for (int i = tid; i < pq.C; i += kS1T) {
      s1.logW[ij0 + (size_t)i * Ck] = -INFINITY;
      s1.fbias[ij0 + (size_t)i * Ck] = -INFINITY;
    }
    return;
  }
  const int off = a.ks.off[(size_t)kpid * (Ck + 1) + j];
  const int* perm = a.ks.perm + pk.slot0;
  const T* K = static_cast<const T*>(a.kg.X);
  const T* V = static_cast<const T*>(a.V);
  for (int d = tid; d < D; d += kS1T) mu[d] = a.ks.cent32[((size_t)kpid * Ck + j) * D + d];
  __syncthreads();
  const float s = a.scale;
  const int mode = a.mode;
  const float lognj = logf((float)nj);

  auto load_chunk = [&](int c0, int cnt) {
    for (int e = tid; e < cnt * D; e += kS1T) {
      const int r = e / D, d = e - r * D;
      const long long row = pk.row0 + perm[off + c0 + r];
      kt[r][d] = ld<T>(K + row * D + d) - mu[d];
      vt[r][d] = ld<T>(V + row * D + d);
    }
  };

  const int e = tid % D, g0 = tid / D;
  if (mode == 0) {  // MONOPOLE: u_ij = S_j / n_j for every i
    float acc = 0.f;
    for (int c0 = 0; c0 < nj; c0 += kS1M) {
      const int cnt = imin(kS1M, nj - c0);
      __syncthreads();
      load_chunk(c0, cnt);
      __syncthreads();
      if (tid < D)
        for (int t = 0; t < cnt; ++t) acc += vt[t][tid];
    }
    if (tid < D) red[0][tid] = acc / (float)nj;
    __syncthreads();
    for (int idx = tid; idx < pq.C * D; idx += kS1T) {
      const int i = idx / D, d = idx - i * D;
      put_u(s1, (ij0 + (size_t)i * Ck) * D + d, red[0][d]);
    }
    for (int i = tid; i < pq.C; i += kS1T) {
      s1.logW[ij0 + (size_t)i * Ck] = lognj;
      s1.fbias[ij0 + (size_t)i * Ck] = lognj;
    }
    return;
  }

  const bool one_chunk = nj <= kS1M;
  if (one_chunk) load_chunk(0, nj);
  for (int i0 = 0; i0 < pq.C; i0 += kS1I) {
    const int ic = imin(kS1I, pq.C - i0);
    __syncthreads();
    for (int idx = tid; idx < ic * D; idx += kS1T) {
      const int ii = idx / D, d = idx - ii * D;
      nu[ii][d] = a.qs.cent32[((size_t)qpid * Cq + i0 + ii) * D + d];
    }
    if (tid < kS1I) {
      mrun[tid] = -INFINITY;
      zrun[tid] = 0.f;
    }
    float accU[R], accK[R];
#pragma unroll
    for (int r = 0; r < R; ++r) accU[r] = accK[r] = 0.f;
    for (int c0 = 0; c0 < nj; c0 += kS1M) {
      const int cnt = imin(kS1M, nj - c0);
      if (!one_chunk) {
        __syncthreads();
        load_chunk(c0, cnt);
      }
      __syncthreads();
      // a_ti = s nu_i . k~_t
      for (int idx = tid; idx < kS1M * kS1I; idx += kS1T) {
        const int tt = idx >> 5, ii = idx & 31;
        if (tt < cnt && ii < ic) {
          float g = 0.f;
#pragma unroll 16
          for (int d = 0; d < D; ++d) g = fmaf(nu[ii][d], kt[tt][d], g);
          ws[tt][ii] = s * g;
        }
      }
      __syncthreads();
      if (mode == 1) {
        for (int idx = tid; idx < cnt * kS1I; idx += kS1T) {
          const int tt = idx >> 5, ii = idx & 31;
          ws[tt][ii] = 1.f + ws[tt][ii];  // first-order term of exp(s nu.k~)
        }
      } else {
        // per query cluster: running max-shifted exponential weights
        for (int ii = warp; ii < ic; ii += kS1T / 32) {
          float mx = -INFINITY;
          for (int tt = lane; tt < cnt; tt += 32) mx = fmaxf(mx, ws[tt][ii]);
          for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          const float mo = mrun[ii], mn = fmaxf(mo, mx);
          float zs = 0.f;
          for (int tt = lane; tt < cnt; tt += 32) {
            const float wv = expf(ws[tt][ii] - mn);
            ws[tt][ii] = wv;
            zs += wv;
          }
          for (int o = 16; o; o >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, o);
          if (lane == 0) {
            const float rs = (mo == -INFINITY) ? 0.f : expf(mo - mn);
            rsc[ii] = rs;
            zrun[ii] = zrun[ii] * rs + zs;
            mrun[ii] = mn;
          }
        }
      }
      __syncthreads();
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int ii = g0 + GROUPS * r;
        if (ii >= ic) continue;
        float su = 0.f, sk = 0.f;
        for (int tt = 0; tt < cnt; ++tt) {
          const float wv = ws[tt][ii];
          su = fmaf(wv, vt[tt][e], su);
          if (mode == 2) sk = fmaf(wv, kt[tt][e], sk);
        }
        if (mode == 2) {
          const float rs = rsc[ii];
          accU[r] = fmaf(accU[r], rs, su);
          accK[r] = fmaf(accK[r], rs, sk);
        } else {
          accU[r] += su;
        }
      }
    }
    // outputs of this chunk of query clusters
    if (mode == 1) {
      const float inv = 1.f / (float)nj;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int ii = g0 + GROUPS * r;
        if (ii < ic) put_u(s1, (ij0 + (size_t)(i0 + ii) * Ck) * D + e, accU[r] * inv);
      }
      for (int ii = tid; ii < ic; ii += kS1T) {
        s1.logW[ij0 + (size_t)(i0 + ii) * Ck] = lognj;
        s1.fbias[ij0 + (size_t)(i0 + ii) * Ck] = lognj;
      }
    } else {
      // k_hat = mu + sum w k~ / W;  offset = log W - s nu.(k_hat - mu)
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int ii = g0 + GROUPS * r;
        if (ii >= ic) continue;
        const float inv = 1.f / zrun[ii];
        const float kh = accK[r] * inv;
        const size_t ij = ij0 + (size_t)(i0 + ii) * Ck;
        put_u(s1, ij * D + e, accU[r] * inv);
        put_kf(s1, ij * D + e, mu[e] + kh);
        red[ii][e] = nu[ii][e] * kh;
      }
      __syncthreads();
      for (int ii = warp; ii < ic; ii += kS1T / 32) {
        float part = 0.f;
        for (int d = lane; d < D; d += 32) part += red[ii][d];
        for (int o = 16; o; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (lane == 0) {
          const float lw = mrun[ii] + logf(zrun[ii]);
          const size_t ij = ij0 + (size_t)(i0 + ii) * Ck;
          s1.logW[ij] = lw;
          s1.fbias[ij] = lw - s * part;
        }
      }
    }
  }
}

// ----------------------------------------------------------------------------
// stage 2: far field + exact retrieval in one online softmax
// ----------------------------------------------------------------------------
constexpr int kQ = 64;     // queries per pass
constexpr int kRows = 32;  // key rows staged per step

template <int D>
struct TPQ {
  static constexpr int v = D / 64;  // threads per query, 64 dims each
};

struct Online {
  float m, l;
};

template <typename T, typename TO, int D>
__global__ void __launch_bounds__(kQ * (D / 64)) stage2_kernel(AttnArgs a, Stage1 s1, int qp0) {
  constexpr int P = D / 64;
  __shared__ float ks_[kRows][D];
  __shared__ float vs_[kRows][D];
  __shared__ float bs_[kRows];
  __shared__ unsigned char inR[kMaxC];
  __shared__ int sel[kMaxC];

  const int lq = blockIdx.x, qpid = qp0 + lq, i = blockIdx.y;
  const Prob pq = prob_of(a.qg, qpid);
  if (i >= pq.C) return;
  const int Cq = a.Cq, Ck = a.Ck;
  const int nqi = a.qs.counts[(size_t)qpid * Cq + i];
  if (nqi == 0) return;
  const int kpid = kv_problem(a, qpid);
  const Prob pk = prob_of(a.kg, kpid);
  const int tid = threadIdx.x, part = tid % P, qq = tid / P;
  const int nsel = a.topk > 0 ? s1.nsel[(size_t)qpid * Cq + i] : 0;
  for (int j = tid; j < pk.C; j += blockDim.x) inR[j] = 0;
  __syncthreads();
  for (int r = tid; r < nsel; r += blockDim.x) {
    const int j = s1.sel[((size_t)qpid * Cq + i) * a.topk + r];
    sel[r] = j;
    inR[j] = 1;
  }
  __syncthreads();
  const int* kc = a.ks.counts + (size_t)kpid * Ck;
  const int* koff = a.ks.off + (size_t)kpid * (Ck + 1);
  long long nexact = 0;
  for (int r = 0; r < nsel; ++r) nexact += kc[sel[r]];

  const T* Q = static_cast<const T*>(a.qg.X);
  const T* K = static_cast<const T*>(a.kg.X);
  const T* V = static_cast<const T*>(a.V);
  const int qo = a.qs.off[(size_t)qpid * (Cq + 1) + i];
  const int* qperm = a.qs.perm + pq.slot0;
  const int* kperm = a.ks.perm + pk.slot0;
  const size_t ij0 = ((size_t)lq * Cq + i) * Ck;
  const bool tilted = a.mode == 2;
  const float s = a.scale;

  for (int c0 = 0; c0 < nqi; c0 += kQ) {
    const bool valid = c0 + qq < nqi;
    const int tq = valid ? qperm[qo + c0 + qq] : 0;
    float q[64];
    float acc[64];
#pragma unroll
    for (int d = 0; d < 64; ++d) {
      q[d] = valid ? ld<T>(Q + (pq.row0 + tq) * D + part * 64 + d) : 0.f;
      acc[d] = 0.f;
    }
    float m = -INFINITY, l = 0.f;

    auto consume = [&](int nrows) {
      for (int r = 0; r < nrows; ++r) {
        float dt = 0.f;
#pragma unroll
        for (int d = 0; d < 64; ++d) dt = fmaf(q[d], ks_[r][part * 64 + d], dt);
        if (P == 2) dt += __shfl_xor_sync(0xffffffffu, dt, 1);
        const float lg = fmaf(s, dt, bs_[r]);
        if (lg == -INFINITY) continue;
        if (lg > m) {
          const float sc = (m == -INFINITY) ? 0.f : expf(m - lg);
          l = l * sc + 1.f;
#pragma unroll
          for (int d = 0; d < 64; ++d) acc[d] = fmaf(acc[d], sc, vs_[r][part * 64 + d]);
          m = lg;
        } else {
          const float wt = expf(lg - m);
          l += wt;
#pragma unroll
          for (int d = 0; d < 64; ++d) acc[d] = fmaf(wt, vs_[r][part * 64 + d], acc[d]);
        }
      }
    };

    // far field
    for (int j0 = 0; j0 < pk.C; j0 += kRows) {
      const int nr = imin(kRows, pk.C - j0);
      __syncthreads();
      for (int e = tid; e < nr * D; e += blockDim.x) {
        const int r = e / D, d = e - r * D, j = j0 + r;
        const size_t ij = ij0 + j;
        ks_[r][d] = tilted ? s1.Kf[ij * D + d] : a.ks.cent32[((size_t)kpid * Ck + j) * D + d];
        vs_[r][d] = s1.U[ij * D + d];
      }
      for (int r = tid; r < nr; r += blockDim.x) {
        const int j = j0 + r;
        bs_[r] = (kc[j] == 0 || inR[j]) ? -INFINITY : s1.fbias[ij0 + j];
      }
      __syncthreads();
      consume(nr);
    }
    // exact retrieval
    for (int rr = 0; rr < nsel; ++rr) {
      const int j = sel[rr], b = koff[j], n = kc[j];
      for (int t0 = 0; t0 < n; t0 += kRows) {
        const int nr = imin(kRows, n - t0);
        __syncthreads();
        for (int e = tid; e < nr * D; e += blockDim.x) {
          const int r = e / D, d = e - r * D;
          const long long row = pk.row0 + kperm[b + t0 + r];
          ks_[r][d] = ld<T>(K + row * D + d);
          vs_[r][d] = ld<T>(V + row * D + d);
        }
        for (int r = tid; r < nr; r += blockDim.x) bs_[r] = 0.f;
        __syncthreads();
        consume(nr);
      }
    }
    if (valid) {
      const long long row = pq.row0 + tq;
      const float inv = 1.f / l;
      if (a.O != nullptr) {
        TO* O = static_cast<TO*>(a.O);
#pragma unroll
        for (int d = 0; d < 64; ++d) st<TO>(O + row * D + part * 64 + d, acc[d] * inv);
      } else {
        float* pp = a.part + (size_t)(pq.slot0 + tq) * (D + 1);
#pragma unroll
        for (int d = 0; d < 64; ++d) pp[part * 64 + d] = acc[d] * inv;
        if (part == 0) pp[D] = m + logf(l);
      }
      if (a.n_exact != nullptr && part == 0) {
        if (a.O != nullptr)
          a.n_exact[row] = nexact;
        else
          atomicAdd(reinterpret_cast<unsigned long long*>(a.n_exact + row),
                    (unsigned long long)nexact);
      }
    }
  }
}

// ----------------------------------------------------------------------------
// causal: exact local block, then merge the level partials (each partial is
// the softmax of its terms, entering as one term with logit lse and value o)
// ----------------------------------------------------------------------------
template <typename T, typename TO, int D>
__global__ void __launch_bounds__(kQ * (D / 64)) local_merge_kernel(AttnArgs a, int L) {
  constexpr int P = D / 64;
  __shared__ float ks_[kRows][D];
  __shared__ float vs_[kRows][D];
  const int bhq = blockIdx.x;
  const int N = a.qg.lv.N;
  const int tid = threadIdx.x, part = tid % P, qq = tid / P;
  const int q0 = blockIdx.y * kQ;
  const int qpos = q0 + qq;
  const bool valid = qpos < N;
  const int Hq = a.qg.BH / a.B, Hkv = a.kg.BH / a.B;
  const int b = bhq / Hq, hq = bhq - b * Hq;
  const int bhk = b * Hkv + hq / a.G;
  const T* Q = static_cast<const T*>(a.qg.X);
  const T* K = static_cast<const T*>(a.kg.X);
  const T* V = static_cast<const T*>(a.V);
  const long long qrow = (long long)bhq * N + qpos;
  const long long krow0 = (long long)bhk * N;
  float q[64], acc[64];
#pragma unroll
  for (int d = 0; d < 64; ++d) {
    q[d] = valid ? ld<T>(Q + qrow * D + part * 64 + d) : 0.f;
    acc[d] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const float s = a.scale;
  const int blk = qpos / L;
  const int kbeg = (q0 / L) * L;
  const int kend = imin(q0 + kQ, N);  // exclusive
  for (int t0 = kbeg; t0 < kend; t0 += kRows) {
    const int nr = imin(kRows, kend - t0);
    __syncthreads();
    for (int e = tid; e < nr * D; e += blockDim.x) {
      const int r = e / D, d = e - r * D;
      ks_[r][d] = ld<T>(K + (krow0 + t0 + r) * D + d);
      vs_[r][d] = ld<T>(V + (krow0 + t0 + r) * D + d);
    }
    __syncthreads();
    for (int r = 0; r < nr; ++r) {
      const int t = t0 + r;
      float dt = 0.f;
#pragma unroll
      for (int d = 0; d < 64; ++d) dt = fmaf(q[d], ks_[r][part * 64 + d], dt);
      if (P == 2) dt += __shfl_xor_sync(0xffffffffu, dt, 1);
      if (!valid || t > qpos || t < blk * L) continue;
      const float lg = s * dt;
      if (lg > m) {
        const float sc = (m == -INFINITY) ? 0.f : expf(m - lg);
        l = l * sc + 1.f;
#pragma unroll
        for (int d = 0; d < 64; ++d) acc[d] = fmaf(acc[d], sc, vs_[r][part * 64 + d]);
        m = lg;
      } else {
        const float wt = expf(lg - m);
        l += wt;
#pragma unroll
        for (int d = 0; d < 64; ++d) acc[d] = fmaf(wt, vs_[r][part * 64 + d], acc[d]);
      }
    }
  }
  if (!valid) return;
  const int levels = a.accum ? (blk > 0 ? 1 : 0) : a.qg.lv.nlev;
  for (int lv = 0; lv < levels; ++lv) {
    if (!a.accum && !((blk >> lv) & 1)) continue;
    const int sz = L << lv, p = blk >> (lv + 1);
    const long long slot = a.accum ? qrow
                                   : (long long)bhq * a.qg.lv.toks_per_bh + a.qg.lv.tok_base[lv] +
                                         (long long)p * sz + (qpos - (2 * p + 1) * sz);
    const float* pp = a.part + slot * (D + 1);
    const float lg = pp[D];
    if (lg > m) {
      const float sc = (m == -INFINITY) ? 0.f : expf(m - lg);
      l = l * sc + 1.f;
#pragma unroll
      for (int d = 0; d < 64; ++d) acc[d] = fmaf(acc[d], sc, pp[part * 64 + d]);
      m = lg;
    } else {
      const float wt = expf(lg - m);
      l += wt;
#pragma unroll
      for (int d = 0; d < 64; ++d) acc[d] = fmaf(wt, pp[part * 64 + d], acc[d]);
    }
  }
  TO* O = static_cast<TO*>(a.O);
  const float inv = 1.f / l;
#pragma unroll
  for (int d = 0; d < 64; ++d) st<TO>(O + qrow * D + part * 64 + d, acc[d] * inv);
  if (a.n_exact != nullptr && part == 0)
    atomicAdd(reinterpret_cast<unsigned long long*>(a.n_exact + qrow),
              (unsigned long long)(qpos - blk * L + 1));
}

// ----------------------------------------------------------------------------
// launchers
// ----------------------------------------------------------------------------
template <typename T, int D>
static void blocks_t(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st) {
  // set on every launch: the attribute is per device, and the call is cheap
  cudaFuncSetAttribute(stage1_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)stage1_smem<D>());
  // the fine-query dipole needs no per-cluster-pair summaries: selection reads
  // the centroids and counts, and stage 2 runs per key token at every level
  const bool fq = a.mode == 3;
  if (!fq) {
    ProfScope ps(st, "stage1_summaries");
    if (sizeof(T) == 2 && a.mode == 1)
      run_stage1_dipole_tc(a, s1, qp0, nqp, st);
    else
      stage1_kernel<T, D><<<dim3(nqp, a.Ck), kS1T, stage1_smem<D>(), st>>>(a, s1, qp0);
  }
  if (a.topk > 0) {
    ProfScope ps(st, "stage1_select");
    run_select(a, s1, qp0, nqp, st);
  }
  if (a.tdip) {  // the tilted per-pair dipole: its own per-key-token stage 2
    run_stage2_tdip(a, s1, qp0, nqp, st);
  } else if (sizeof(T) == 2) {
    if (!fq) {
      ProfScope ps(st, "stage2_attn");
      run_stage2_tc(a, s1, qp0, nqp, st);
      if (!run_stage2_warp(a, s1, qp0, nqp, st)) run_stage2_mma(a, s1, qp0, nqp, st);
    }
    if (a.dense_lv) run_stage2_dense(a, s1, qp0, nqp, st);
  } else {
    ProfScope ps(st, "stage2_attn");
    if (a.out_f32)
      stage2_kernel<T, float, D><<<dim3(nqp, a.Cq), kQ * (D / 64), 0, st>>>(a, s1, qp0);
    else
      stage2_kernel<T, T, D><<<dim3(nqp, a.Cq), kQ * (D / 64), 0, st>>>(a, s1, qp0);
  }
}

void run_blocks(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st) {
  const int D = a.qg.D;
  if (a.qg.dtype == 0) {
    if (D == 64) blocks_t<__nv_bfloat16, 64>(a, s1, qp0, nqp, st);
    else blocks_t<__nv_bfloat16, 128>(a, s1, qp0, nqp, st);
  } else {
    if (D == 64) blocks_t<float, 64>(a, s1, qp0, nqp, st);
    else blocks_t<float, 128>(a, s1, qp0, nqp, st);
  }
}

void run_local_merge(const AttnArgs& a, int L, cudaStream_t st) {
  ProfScope ps(st, "causal_local_merge");
  if (run_local_mma(a, L, st)) return;  // bf16, L a multiple of 128: tensor-core tiles
  const int D = a.qg.D, N = a.qg.lv.N;
  dim3 grid(a.qg.BH, cdiv(N, kQ));
  const int thr = kQ * (D / 64);
  using bf = __nv_bfloat16;
  if (a.qg.dtype == 0) {
    if (a.out_f32) {
      if (D == 64) local_merge_kernel<bf, float, 64><<<grid, thr, 0, st>>>(a, L);
      else local_merge_kernel<bf, float, 128><<<grid, thr, 0, st>>>(a, L);
    } else {
      if (D == 64) local_merge_kernel<bf, bf, 64><<<grid, thr, 0, st>>>(a, L);
      else local_merge_kernel<bf, bf, 128><<<grid, thr, 0, st>>>(a, L);
    }
  } else {
    if (D == 64) local_merge_kernel<float, float, 64><<<grid, thr, 0, st>>>(a, L);
    else local_merge_kernel<float, float, 128><<<grid, thr, 0, st>>>(a, L);
  }
}

}  // namespace muse
