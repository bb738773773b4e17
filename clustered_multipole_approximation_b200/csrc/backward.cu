// Gradients of the operator with respect to Q, K and V, acausal and causal.
//
// The pages train models with MuSe as the attention layer (gist.science page
// "Multipole Semantic Attention: A Fast Approximation of Softmax Attention
// for Pretraining", Experimental Results), so the layer has a backward pass.
// The clusterings and the retrieval sets are piecewise constant in the inputs
// and are held at the forward pass's values; everything else is
// differentiated as the function of Q, K and V it is:
//   mu_j = (1/n_j) sum_{a(t)=j} k_t,  S_j = sum v_t,  M_j = sum v_t (k_t - mu_j)^T,
//   nu_i = (1/m_i) sum_{b(q)=i} q,
//   u_ij = S_j / n_j (MONOPOLE)   or   (S_j + s M_j nu_i) / n_j (DIPOLE),
// and the output of query q (cluster i) is one softmax over the far terms
// (j outside R_i, n_j > 0: logit s q.mu_j + log n_j, value u_ij) and the
// exact terms (keys of the clusters in R_i: logit s q.k_t, value v_t).
//
// With lse_q the log-sum-exp of the query's logits, per term p = exp(l -
// lse_q) and g = dO_q . x (x the term's value), D_q = sum p g (= dO_q . O_q,
// formed here from the same fp32 terms rather than read from the forward's
// rounded output) and dl = p (g - D_q):
//   exact t:  dq += s dl k_t,  dk_t += s dl q,  dv_t += p dO_q
//   far j:    dq += s dl mu_j, dmu_j += s dl q, du_ij += p dO_q
// and through the summaries (sums over the query clusters i of every q-head
// that reads key set j):
//   dS_j = sum_i du_ij / n_j
//   dM_j = (s / n_j) sum_i du_ij nu_i^T,   dnu_i += (s / n_j) M_j^T du_ij
//   dmu_j -= dM_j^T S_j                     (M_j's own dependence on mu_j)
//   dv_t += dS_j + dM_j (k_t - mu_j),  dk_t += dmu_j / n_j + dM_j^T v_t
//   dq   += dnu_i / m_i.
//
// Kernels (fp32 arithmetic throughout, gradients in fp32):
//   bwd_key_stats   one CTA per (key set, cluster): S_j and M_j from the
//                   cluster-sorted members;
//   bwd_u_table     (DIPOLE) one CTA per (query set, key cluster): u_ij for
//                   every query cluster i;
//   bwd_query       one CTA per (query set, query cluster i), chunks of 32
//                   member queries: log-sum-exp and D_q (the exact tiles'
//                   terms online, the far terms' g kept per (query, cluster)),
//                   the far terms (du_ij owned by the CTA, dmu_j by
//                   atomics), then the exact tiles of R_i's clusters (dk, dv
//                   by atomics);
//   bwd_cluster     one CTA per (key set, cluster): dS_j, dM_j, dnu, and the
//                   chain to the members' dk and dv;
//   bwd_query_nu    dq += dnu_i / m_i.
// Causal (the hierarchical levels and the local blocks of L keys, one softmax
// per query): bwd_query first writes each level problem's (max, sum, sum of
// p g) per query and bwd_local the local block's, bwd_combine merges them
// into every query's log-sum-exp and D_q, then bwd_query and bwd_local take
// the gradients of every term with those; a query's and a key's gradients
// are summed over its levels by fp32 atomics.
#include "common.cuh"
#include "kernels.h"

namespace muse {

namespace {

constexpr int kBT = 256;  // threads per CTA
constexpr int kBW = kBT / 32;
constexpr int kQC = 32;   // queries per chunk
constexpr int kKC = 32;   // keys per exact tile

template <typename T>
__device__ inline float ldg_(const T* p) {
  return ld<T>(p);
}

// ---------------------------------------------------------------------------
// S_j and M_j[e][d] = sum_t v_t[e] (k_t[d] - mu_j[d])
// ---------------------------------------------------------------------------
template <typename T, int D, bool DIP>
__global__ void __launch_bounds__(kBT) bwd_key_stats_kernel(AttnArgs a, BwdArgs b) {
  __shared__ float kt[kKC][D + 1];
  __shared__ float vt[kKC][D + 1];
  __shared__ float mu[D];
  const int kpid = blockIdx.x, j = blockIdx.y, tid = threadIdx.x;
  const int Ck = a.Ck;
  const Prob pk = prob_of(a.kg, kpid);
  const size_t cj = (size_t)kpid * Ck + j;
  const int n = j < pk.C ? a.ks.counts[cj] : 0;
  const int off = n > 0 ? a.ks.off[(size_t)kpid * (Ck + 1) + j] : 0;
  const int* perm = a.ks.perm + pk.slot0;
  const T* K = static_cast<const T*>(a.kg.X);
  const T* V = static_cast<const T*>(a.V);
  for (int d = tid; d < D; d += kBT) mu[d] = a.ks.cent32[cj * D + d];
  constexpr int MR = DIP ? D * D / kBT : 0;
  float m[MR > 0 ? MR : 1];
#pragma unroll
  for (int r = 0; r < (MR > 0 ? MR : 1); ++r) m[r] = 0.f;
  float sacc = 0.f;
  for (int c0 = 0; c0 < n; c0 += kKC) {
    const int cnt = imin(kKC, n - c0);
    __syncthreads();
    for (int e = tid; e < cnt * D; e += kBT) {
      const int r = e / D, d = e - r * D;
      const long long row = pk.row0 + perm[off + c0 + r];
      kt[r][d] = ldg_<T>(K + row * D + d) - mu[d];
      vt[r][d] = ldg_<T>(V + row * D + d);
    }
    __syncthreads();
    if (tid < D)
      for (int t = 0; t < cnt; ++t) sacc += vt[t][tid];
    if (DIP) {
#pragma unroll
      for (int r = 0; r < MR; ++r) {
        const int idx = tid + kBT * r, e = idx / D, d = idx - e * D;
        float x = m[r];
        for (int t = 0; t < cnt; ++t) x = fmaf(vt[t][e], kt[t][d], x);
        m[r] = x;
      }
    }
  }
  if (tid < D) b.Sst[cj * D + tid] = sacc;
  if (DIP) {
#pragma unroll
    for (int r = 0; r < MR; ++r) b.Mst[cj * D * D + tid + kBT * r] = m[r];
  }
}

// ---------------------------------------------------------------------------
// u_ij = (S_j + s M_j nu_i) / n_j for every query cluster i (DIPOLE)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kBT) bwd_u_table_kernel(AttnArgs a, BwdArgs b) {
  extern __shared__ __align__(16) float ut_raw[];
  float* M = ut_raw;                   // [D][D + 1]
  float* nu = M + D * (D + 1);         // [kBT / D][D]
  const int qpid = blockIdx.x, j = blockIdx.y, tid = threadIdx.x;
  const int Cq = a.Cq, Ck = a.Ck;
  const int kpid = kv_problem(a, qpid);
  const Prob pq = prob_of(a.qg, qpid);
  const Prob pk = prob_of(a.kg, kpid);
  const size_t cj = (size_t)kpid * Ck + j;
  const int n = j < pk.C ? a.ks.counts[cj] : 0;
  float* U = b.U + ((size_t)qpid * Cq * Ck + j) * D;  // row (i, j) at U + i * Ck * D
  if (n == 0) {
    for (int e = tid; e < pq.C * D; e += kBT) U[(size_t)(e / D) * Ck * D + e % D] = 0.f;
    return;
  }
  for (int e = tid; e < D * D; e += kBT) M[(e / D) * (D + 1) + e % D] = b.Mst[cj * D * D + e];
  constexpr int RI = kBT / D;  // query clusters per pass
  const int e = tid % D, ri = tid / D;
  const float s = a.scale, inv = 1.f / (float)n, Se = b.Sst[cj * D + e];
  const float* cent = a.qs.cent32 + (size_t)qpid * Cq * D;
  for (int i0 = 0; i0 < pq.C; i0 += RI) {
    __syncthreads();
    if (i0 + ri < pq.C) nu[ri * D + e] = cent[(size_t)(i0 + ri) * D + e];
    __syncthreads();
    if (i0 + ri < pq.C) {
      float x = 0.f;
#pragma unroll 8
      for (int d = 0; d < D; ++d) x = fmaf(M[e * (D + 1) + d], nu[ri * D + d], x);
      U[(size_t)(i0 + ri) * Ck * D + e] = fmaf(s, x, Se) * inv;
    }
  }
}

// ---------------------------------------------------------------------------
// per (query set, query cluster): the softmax's own gradient
//
// The exact tiles (32 queries x 32 keys) are register-blocked: for S = Q K^T
// and G = dO V^T every thread owns a 2 x 2 block (queries 2tq, 2tq+1; keys
// tk, tk+16, so a quarter warp's 16-byte row reads hit distinct banks); for
// dQ += dS K, dK = dS^T Q and dV = P^T dO every thread owns 2 rows x D/16
// columns.
// ---------------------------------------------------------------------------
template <int D>
struct QuerySmem {
  float q[kQC][D + 4];
  float go[kQC][D + 4];  // dO
  float kt[kKC][D + 4];
  float vt[kKC][D + 4];
  float pt[kQC][kKC + 1];
  float dst[kQC][kKC + 1];
  float lse[kQC];
  float dq_[kQC];  // D_q
  float ml[kQC][2];  // running max and sum of the far terms, per query
  float dex[kQC];  // exact terms' sum of exp(l - m) g at the running max m
  float mq[kQC];   // running max after the exact terms
  float lsum[kQC]; // running sum after the exact terms
  int row[kQC];
  unsigned rmask[kMaxC / 32];
};

// s * q.k and dO.v for the thread's 2 x 2 block of the staged tile
template <int D>
__device__ inline void tile_sg(const QuerySmem<D>& sm, int tq, int tk, float sx[2][2], float gx[2][2]) {
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int c = 0; c < 2; ++c) sx[a][c] = gx[a][c] = 0.f;
#pragma unroll 4
  for (int d = 0; d < D; d += 4) {
    float4 qv[2], gv[2], kv[2], vv[2];
#pragma unroll
    for (int a = 0; a < 2; ++a) {
      qv[a] = *reinterpret_cast<const float4*>(&sm.q[2 * tq + a][d]);
      gv[a] = *reinterpret_cast<const float4*>(&sm.go[2 * tq + a][d]);
      kv[a] = *reinterpret_cast<const float4*>(&sm.kt[tk + 16 * a][d]);
      vv[a] = *reinterpret_cast<const float4*>(&sm.vt[tk + 16 * a][d]);
    }
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        sx[a][c] = fmaf(qv[a].x, kv[c].x, fmaf(qv[a].y, kv[c].y, fmaf(qv[a].z, kv[c].z, fmaf(qv[a].w, kv[c].w, sx[a][c]))));
        gx[a][c] = fmaf(gv[a].x, vv[c].x, fmaf(gv[a].y, vv[c].y, fmaf(gv[a].z, vv[c].z, fmaf(gv[a].w, vv[c].w, gx[a][c]))));
      }
  }
}

// MODE 0: one acausal problem per query (log-sum-exp and D_q formed here);
// MODE 1: causal, write each query's (max, sum, sum of p g) over this level's
//         terms and stop; MODE 2: causal gradients with the combined
//         log-sum-exp and D_q of every query (dQ by atomics: a query sits in
//         several level problems).
template <typename T, typename TO, int D, bool DIP, int MODE>
__global__ void __launch_bounds__(kBT) bwd_query_kernel(AttnArgs a, Stage1 s1, BwdArgs b) {
  extern __shared__ __align__(16) unsigned char bq_raw[];
  QuerySmem<D>& sm = *reinterpret_cast<QuerySmem<D>*>(bq_raw);
  const int Cq = a.Cq, Ck = a.Ck;
  float* mu_s = reinterpret_cast<float*>(bq_raw + sizeof(QuerySmem<D>));  // [Ck][D + 1]
  float* lf = mu_s + (size_t)Ck * (D + 1);                               // [kQC][Ck]
  float* gf = lf + (size_t)kQC * Ck;                                      // [kQC][Ck] dO.u
  int* fl = reinterpret_cast<int*>(gf + (size_t)kQC * Ck);               // far clusters
  int* xl = fl + Ck;                                                      // exact clusters
  __shared__ int nfar, nex;
  const int qpid = blockIdx.x, i = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const Prob pq = prob_of(a.qg, qpid);
  if (i >= pq.C) return;
  const int mi = a.qs.counts[(size_t)qpid * Cq + i];
  if (mi == 0) return;
  const int kpid = kv_problem(a, qpid);
  const Prob pk = prob_of(a.kg, kpid);
  const int ck = pk.C;
  const int* kcnt = a.ks.counts + (size_t)kpid * Ck;
  const int* koff = a.ks.off + (size_t)kpid * (Ck + 1);
  const int* kperm = a.ks.perm + pk.slot0;
  const int qoff = a.qs.off[(size_t)qpid * (Cq + 1) + i];
  const int* qperm = a.qs.perm + pq.slot0;
  const T* Q = static_cast<const T*>(a.qg.X);
  const T* K = static_cast<const T*>(a.kg.X);
  const T* V = static_cast<const T*>(a.V);
  const TO* GO = static_cast<const TO*>(b.dO);
  const float s = a.scale;
  constexpr int DV = D / 16;  // columns per thread in the dQ / dK / dV blocks
  const int tq = tid >> 4, tk = tid & 15;  // 2 x 2 blocks of S and G; 2 rows x DV columns

  // retrieval set, far / exact cluster lists, centroid table
  for (int w = tid; w < kMaxC / 32; w += kBT) sm.rmask[w] = 0u;
  __syncthreads();
  if (a.topk > 0) {
    const int ns = s1.nsel[(size_t)qpid * Cq + i];
    for (int r = tid; r < ns; r += kBT) {
      const int j = s1.sel[((size_t)qpid * Cq + i) * a.topk + r];
      if (j >= 0 && j < ck) atomicOr(&sm.rmask[j >> 5], 1u << (j & 31));
    }
  }
  for (int e = tid; e < ck * D; e += kBT) {
    const int j = e / D, d = e - j * D;
    mu_s[j * (D + 1) + d] = a.ks.cent32[((size_t)kpid * Ck + j) * D + d];
  }
  __syncthreads();
  if (tid == 0) {
    int nf = 0, nx = 0;
    for (int j = 0; j < ck; ++j) {
      if (kcnt[j] == 0) continue;
      if ((sm.rmask[j >> 5] >> (j & 31)) & 1u) xl[nx++] = j;
      else fl[nf++] = j;
    }
    nfar = nf;
    nex = nx;
  }
  __syncthreads();
  const int nf = nfar, nx = nex;

  // stage one tile of retrieved keys (and values) into shared memory
  auto load_tile = [&](int o0, int kc, bool with_v) {
    for (int e = tid; e < kKC * D; e += kBT) {
      const int r = e / D, d = e - r * D;
      float kx = 0.f, vx = 0.f;
      if (r < kc) {
        const long long row = pk.row0 + kperm[o0 + r];
        kx = ldg_<T>(K + row * D + d);
        if (with_v) vx = ldg_<T>(V + row * D + d);
      }
      sm.kt[r][d] = kx;
      sm.vt[r][d] = vx;
    }
  };

  for (int c0 = 0; c0 < mi; c0 += kQC) {
    const int qc = imin(kQC, mi - c0);
    // ---- chunk rows: q, dO (rows past qc are zero) --------------------------
    __syncthreads();
    if (tid < kQC) sm.row[tid] = tid < qc ? (int)(pq.row0 + qperm[qoff + c0 + tid]) : -1;
    __syncthreads();
    for (int e = tid; e < kQC * D; e += kBT) {
      const int r = e / D, d = e - r * D;
      const long long row = sm.row[r];
      sm.q[r][d] = row >= 0 ? ldg_<T>(Q + row * D + d) : 0.f;
      sm.go[r][d] = row >= 0 ? ldg_<TO>(GO + row * D + d) : 0.f;
    }
    if (tid >= qc && tid < kQC) {  // rows past the chunk: no far terms
      sm.ml[tid][0] = -INFINITY;
      sm.ml[tid][1] = 0.f;
    }
    __syncthreads();
    // ---- far logits and their running max / sum (one warp per query) ------
    for (int r = warp; r < qc; r += kBW) {
      float mx = -INFINITY;
      for (int jj = lane; jj < nf; jj += 32) {
        const int j = fl[jj];
        float x = 0.f;
#pragma unroll 8
        for (int d = 0; d < D; ++d) x = fmaf(sm.q[r][d], mu_s[j * (D + 1) + d], x);
        const float l = fmaf(s, x, __logf((float)kcnt[j]));
        lf[r * Ck + jj] = l;
        mx = fmaxf(mx, l);
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float sum = 0.f;
      for (int jj = lane; jj < nf; jj += 32) sum += __expf(lf[r * Ck + jj] - mx);
#pragma unroll
      for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) {
        sm.ml[r][0] = mx;
        sm.ml[r][1] = nf > 0 ? sum : 0.f;
      }
    }
    __syncthreads();
    // ---- exact terms: finish the running max / sum, and their sum of p g ---
    // (the 16 threads of a query pair hold identical running values)
    float mrun[2], lrun[2], arun[2];
    const int nx1 = MODE == 2 ? 0 : nx;  // MODE 2 reads the combined values
#pragma unroll
    for (int a2 = 0; a2 < 2; ++a2) {
      mrun[a2] = sm.ml[2 * tq + a2][0];
      lrun[a2] = sm.ml[2 * tq + a2][1];
      arun[a2] = 0.f;
    }
    for (int xi = 0; xi < nx1; ++xi) {
      const int j = xl[xi], nj = kcnt[j], o0 = koff[j];
      for (int t0 = 0; t0 < nj; t0 += kKC) {
        const int kc = imin(kKC, nj - t0);
        __syncthreads();
        load_tile(o0 + t0, kc, true);
        __syncthreads();
        float sx[2][2], gx[2][2];
        tile_sg<D>(sm, tq, tk, sx, gx);
#pragma unroll
        for (int a2 = 0; a2 < 2; ++a2) {
          float l0 = tk < kc ? s * sx[a2][0] : -INFINITY;
          float l1 = tk + 16 < kc ? s * sx[a2][1] : -INFINITY;
          float mx = fmaxf(l0, l1);
#pragma unroll
          for (int o = 8; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          const float mn = fmaxf(mrun[a2], mx);
          const float p0 = __expf(l0 - mn), p1 = __expf(l1 - mn);
          float p = p0 + p1, pg = p0 * gx[a2][0] + p1 * gx[a2][1];
#pragma unroll
          for (int o = 8; o; o >>= 1) {
            p += __shfl_xor_sync(0xffffffffu, p, o);
            pg += __shfl_xor_sync(0xffffffffu, pg, o);
          }
          const float sc = __expf(mrun[a2] - mn);
          lrun[a2] = lrun[a2] * sc + p;
          arun[a2] = arun[a2] * sc + pg;
          mrun[a2] = mn;
        }
      }
    }
    if (tk == 0) {
#pragma unroll
      for (int a2 = 0; a2 < 2; ++a2) {
        const int r = 2 * tq + a2;
        sm.lse[r] = mrun[a2] + __logf(lrun[a2]);
        sm.mq[r] = mrun[a2];
        sm.lsum[r] = lrun[a2];
        sm.dex[r] = arun[a2];
        if (MODE == 2 && r < qc) {  // the combined values of all the query's terms
          sm.lse[r] = b.lse_all[sm.row[r]];
          sm.dq_[r] = b.d_all[sm.row[r]];
        }
      }
    }
    // ---- far terms' g = dO_q . u_ij: one warp per far cluster -------------
    for (int jj = warp; jj < nf; jj += kBW) {
      const int j = fl[jj];
      float ux[D / 32];
      const float invn = 1.f / (float)kcnt[j];
#pragma unroll
      for (int u = 0; u < D / 32; ++u) {
        const int d = lane + 32 * u;
        ux[u] = DIP ? b.U[(((size_t)qpid * Cq + i) * Ck + j) * D + d]
                    : b.Sst[((size_t)kpid * Ck + j) * D + d] * invn;
      }
      for (int r = 0; r < qc; ++r) {
        float g = 0.f;
#pragma unroll
        for (int u = 0; u < D / 32; ++u) g = fmaf(sm.go[r][lane + 32 * u], ux[u], g);
#pragma unroll
        for (int o = 16; o; o >>= 1) g += __shfl_xor_sync(0xffffffffu, g, o);
        if (lane == 0) gf[r * Ck + jj] = g;
      }
    }
    __syncthreads();
    // D_q = sum over the terms of p g (MODE 1: this level's share, unnormalised)
    if (MODE != 2) {
      for (int r = warp; r < qc; r += kBW) {
        const float m = sm.mq[r];
        float acc = 0.f;
        for (int jj = lane; jj < nf; jj += 32) acc = fmaf(__expf(lf[r * Ck + jj] - m), gf[r * Ck + jj], acc);
#pragma unroll
        for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) {
          if (MODE == 1) {
            const long long slot = pq.slot0 + (sm.row[r] - pq.row0);
            b.pm[slot] = m;
            b.pl[slot] = sm.lsum[r];
            b.pa[slot] = acc + sm.dex[r];
          } else {
            sm.dq_[r] = (acc + sm.dex[r]) * __expf(m - sm.lse[r]);
          }
        }
      }
    }
    if (MODE == 1) continue;  // the partials are all this pass writes
    __syncthreads();

    // ---- far terms: one warp per far cluster ------------------------------
    for (int jj = warp; jj < nf; jj += kBW) {
      const int j = fl[jj];
      float gu[D / 32], gm[D / 32];
#pragma unroll
      for (int u = 0; u < D / 32; ++u) gu[u] = gm[u] = 0.f;
      for (int r = 0; r < qc; ++r) {
        const float p = __expf(lf[r * Ck + jj] - sm.lse[r]);
        const float dl = p * (gf[r * Ck + jj] - sm.dq_[r]);
#pragma unroll
        for (int u = 0; u < D / 32; ++u) {
          gu[u] = fmaf(p, sm.go[r][lane + 32 * u], gu[u]);
          gm[u] = fmaf(s * dl, sm.q[r][lane + 32 * u], gm[u]);
        }
        __syncwarp();
        if (lane == 0) lf[r * Ck + jj] = s * dl;  // now the coefficient of mu_j in dq
      }
      float* du = b.dU + (((size_t)qpid * Cq + i) * Ck + j) * D;
      float* dm = b.dmu + ((size_t)kpid * Ck + j) * D;
#pragma unroll
      for (int u = 0; u < D / 32; ++u) {
        const int d = lane + 32 * u;
        du[d] += gu[u];  // this CTA owns the row (query set, i, j)
        atomicAdd(dm + d, gm[u]);
      }
    }
    __syncthreads();
    // dq = sum_j (s dl_qj) mu_j: the thread's 2 rows x DV columns
    float dq[2][DV];
#pragma unroll
    for (int a2 = 0; a2 < 2; ++a2)
#pragma unroll
      for (int v = 0; v < DV; ++v) dq[a2][v] = 0.f;
    {
      const int r0 = 2 * tq;
      for (int jj = 0; jj < nf; ++jj) {
        const float c0_ = r0 < qc ? lf[r0 * Ck + jj] : 0.f;
        const float c1_ = r0 + 1 < qc ? lf[(r0 + 1) * Ck + jj] : 0.f;
        const float* m = mu_s + fl[jj] * (D + 1) + tk * DV;
#pragma unroll
        for (int v = 0; v < DV; ++v) {
          dq[0][v] = fmaf(c0_, m[v], dq[0][v]);
          dq[1][v] = fmaf(c1_, m[v], dq[1][v]);
        }
      }
    }
    // ---- exact tiles --------------------------------------------------------
    for (int xi = 0; xi < nx; ++xi) {
      const int j = xl[xi], nj = kcnt[j], o0 = koff[j];
      for (int t0 = 0; t0 < nj; t0 += kKC) {
        const int kc = imin(kKC, nj - t0);
        __syncthreads();
        load_tile(o0 + t0, kc, true);
        __syncthreads();
        {
          float sx[2][2], gx[2][2];
          tile_sg<D>(sm, tq, tk, sx, gx);
#pragma unroll
          for (int a2 = 0; a2 < 2; ++a2) {
            const int r = 2 * tq + a2;
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
              const int t = tk + 16 * c2;
              float p = 0.f, ds = 0.f;
              if (r < qc && t < kc) {
                p = __expf(s * sx[a2][c2] - sm.lse[r]);
                ds = p * (gx[a2][c2] - sm.dq_[r]);
              }
              sm.pt[r][t] = p;
              sm.dst[r][t] = s * ds;
            }
          }
        }
        __syncthreads();
        // dq += (s dS) K over the tile's keys
#pragma unroll 4
        for (int t = 0; t < kKC; ++t) {
          const float c0_ = sm.dst[2 * tq][t], c1_ = sm.dst[2 * tq + 1][t];
#pragma unroll
          for (int v = 0; v < DV; v += 4) {
            const float4 k4 = *reinterpret_cast<const float4*>(&sm.kt[t][tk * DV + v]);
            dq[0][v] = fmaf(c0_, k4.x, dq[0][v]);
            dq[0][v + 1] = fmaf(c0_, k4.y, dq[0][v + 1]);
            dq[0][v + 2] = fmaf(c0_, k4.z, dq[0][v + 2]);
            dq[0][v + 3] = fmaf(c0_, k4.w, dq[0][v + 3]);
            dq[1][v] = fmaf(c1_, k4.x, dq[1][v]);
            dq[1][v + 1] = fmaf(c1_, k4.y, dq[1][v + 1]);
            dq[1][v + 2] = fmaf(c1_, k4.z, dq[1][v + 2]);
            dq[1][v + 3] = fmaf(c1_, k4.w, dq[1][v + 3]);
          }
        }
        // dK = (s dS)^T Q and dV = P^T dO for the thread's 2 keys x DV columns
        {
          float gk[2][DV], gv[2][DV];
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
            for (int v = 0; v < DV; ++v) gk[c2][v] = gv[c2][v] = 0.f;
#pragma unroll 4
          for (int r = 0; r < kQC; ++r) {
            const float d0 = sm.dst[r][2 * tq], d1 = sm.dst[r][2 * tq + 1];
            const float p0 = sm.pt[r][2 * tq], p1 = sm.pt[r][2 * tq + 1];
#pragma unroll
            for (int v = 0; v < DV; v += 4) {
              const float4 q4 = *reinterpret_cast<const float4*>(&sm.q[r][tk * DV + v]);
              const float4 g4 = *reinterpret_cast<const float4*>(&sm.go[r][tk * DV + v]);
              gk[0][v] = fmaf(d0, q4.x, gk[0][v]);
              gk[0][v + 1] = fmaf(d0, q4.y, gk[0][v + 1]);
              gk[0][v + 2] = fmaf(d0, q4.z, gk[0][v + 2]);
              gk[0][v + 3] = fmaf(d0, q4.w, gk[0][v + 3]);
              gk[1][v] = fmaf(d1, q4.x, gk[1][v]);
              gk[1][v + 1] = fmaf(d1, q4.y, gk[1][v + 1]);
              gk[1][v + 2] = fmaf(d1, q4.z, gk[1][v + 2]);
              gk[1][v + 3] = fmaf(d1, q4.w, gk[1][v + 3]);
              gv[0][v] = fmaf(p0, g4.x, gv[0][v]);
              gv[0][v + 1] = fmaf(p0, g4.y, gv[0][v + 1]);
              gv[0][v + 2] = fmaf(p0, g4.z, gv[0][v + 2]);
              gv[0][v + 3] = fmaf(p0, g4.w, gv[0][v + 3]);
              gv[1][v] = fmaf(p1, g4.x, gv[1][v]);
              gv[1][v + 1] = fmaf(p1, g4.y, gv[1][v + 1]);
              gv[1][v + 2] = fmaf(p1, g4.z, gv[1][v + 2]);
              gv[1][v + 3] = fmaf(p1, g4.w, gv[1][v + 3]);
            }
          }
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
            const int t = 2 * tq + c2;
            if (t >= kc) continue;
            const long long row = pk.row0 + kperm[o0 + t0 + t];
#pragma unroll
            for (int v = 0; v < DV; ++v) {
              atomicAdd(b.dK + row * D + tk * DV + v, gk[c2][v]);
              atomicAdd(b.dV + row * D + tk * DV + v, gv[c2][v]);
            }
          }
        }
      }
    }
    // ---- this chunk's dq (the centroid term is added later) ---------------
#pragma unroll
    for (int a2 = 0; a2 < 2; ++a2) {
      const int r = 2 * tq + a2;
      if (r >= qc) continue;
#pragma unroll
      for (int v = 0; v < DV; ++v) {
        float* dst = b.dQ + (long long)sm.row[r] * D + tk * DV + v;
        if (MODE == 2) atomicAdd(dst, dq[a2][v]);
        else *dst = dq[a2][v];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// causal: the local blocks (exact attention to the keys [bL, q] of the
// query's own block), 32 queries per CTA, key tiles of 32 up to the chunk's
// last query.  MODE 1: each query's (max, sum, sum of p g); MODE 2: the
// gradients with the combined log-sum-exp and D_q.
// ---------------------------------------------------------------------------
template <typename T, typename TO, int D, int MODE>
__global__ void __launch_bounds__(kBT) bwd_local_kernel(AttnArgs a, BwdArgs b, int L) {
  extern __shared__ __align__(16) unsigned char bl_raw[];
  QuerySmem<D>& sm = *reinterpret_cast<QuerySmem<D>*>(bl_raw);
  const int bhq = blockIdx.x, c0 = blockIdx.y * kQC;
  const int N = a.qg.lv.N, tid = threadIdx.x;
  const int Hq = a.qg.BH / a.B, Hkv = a.kg.BH / a.B;
  const int bb = bhq / Hq, hq = bhq - bb * Hq;
  const long long qrow0 = (long long)bhq * N, krow0 = (long long)(bb * Hkv + hq / a.G) * N;
  const T* Q = static_cast<const T*>(a.qg.X);
  const T* K = static_cast<const T*>(a.kg.X);
  const T* V = static_cast<const T*>(a.V);
  const TO* GO = static_cast<const TO*>(b.dO);
  const float s = a.scale;
  constexpr int DV = D / 16;
  const int tq = tid >> 4, tk = tid & 15;
  const int qc = imin(kQC, N - c0);
  for (int e = tid; e < kQC * D; e += kBT) {
    const int r = e / D, d = e - r * D;
    sm.q[r][d] = r < qc ? ld<T>(Q + (qrow0 + c0 + r) * D + d) : 0.f;
    sm.go[r][d] = r < qc ? ld<TO>(GO + (qrow0 + c0 + r) * D + d) : 0.f;
  }
  if (MODE == 2 && tid < kQC) {
    sm.lse[tid] = tid < qc ? b.lse_all[qrow0 + c0 + tid] : 0.f;
    sm.dq_[tid] = tid < qc ? b.d_all[qrow0 + c0 + tid] : 0.f;
  }
  float mrun[2] = {-INFINITY, -INFINITY}, lrun[2] = {0.f, 0.f}, arun[2] = {0.f, 0.f};
  float dq[2][DV];
#pragma unroll
  for (int a2 = 0; a2 < 2; ++a2)
#pragma unroll
    for (int v = 0; v < DV; ++v) dq[a2][v] = 0.f;
  const int kbeg = (c0 / L) * L, kend = c0 + qc;  // keys [kbeg, kend)
  for (int t0 = kbeg; t0 < kend; t0 += kKC) {
    const int kc = imin(kKC, kend - t0);
    __syncthreads();
    for (int e = tid; e < kKC * D; e += kBT) {
      const int r = e / D, d = e - r * D;
      sm.kt[r][d] = r < kc ? ld<T>(K + (krow0 + t0 + r) * D + d) : 0.f;
      sm.vt[r][d] = r < kc ? ld<T>(V + (krow0 + t0 + r) * D + d) : 0.f;
    }
    __syncthreads();
    float sx[2][2], gx[2][2];
    tile_sg<D>(sm, tq, tk, sx, gx);
    if (MODE == 1) {
#pragma unroll
      for (int a2 = 0; a2 < 2; ++a2) {
        const int qpos = c0 + 2 * tq + a2;
        const int k0 = t0 + tk, k1 = t0 + tk + 16;
        float l0 = (tk < kc && k0 <= qpos) ? s * sx[a2][0] : -INFINITY;
        float l1 = (tk + 16 < kc && k1 <= qpos) ? s * sx[a2][1] : -INFINITY;
        float mx = fmaxf(l0, l1);
#pragma unroll
        for (int o = 8; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const bool any = mx != -INFINITY;  // no key of this tile for these rows: no change
        const float mn = any ? fmaxf(mrun[a2], mx) : mrun[a2];
        const float p0 = any ? __expf(l0 - mn) : 0.f, p1 = any ? __expf(l1 - mn) : 0.f;
        float p = p0 + p1, pg = p0 * gx[a2][0] + p1 * gx[a2][1];
#pragma unroll
        for (int o = 8; o; o >>= 1) {
          p += __shfl_xor_sync(0xffffffffu, p, o);
          pg += __shfl_xor_sync(0xffffffffu, pg, o);
        }
        const float sc = any ? __expf(mrun[a2] - mn) : 1.f;
        lrun[a2] = lrun[a2] * sc + p;
        arun[a2] = arun[a2] * sc + pg;
        mrun[a2] = mn;
      }
      continue;
    }
    // MODE 2: P and s dS of the tile, then dq, dK, dV
#pragma unroll
    for (int a2 = 0; a2 < 2; ++a2) {
      const int r = 2 * tq + a2;
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        const int t = tk + 16 * c2;
        float p = 0.f, ds = 0.f;
        if (r < qc && t < kc && t0 + t <= c0 + r) {
          p = __expf(s * sx[a2][c2] - sm.lse[r]);
          ds = p * (gx[a2][c2] - sm.dq_[r]);
        }
        sm.pt[r][t] = p;
        sm.dst[r][t] = s * ds;
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int t = 0; t < kKC; ++t) {
      const float d0 = sm.dst[2 * tq][t], d1 = sm.dst[2 * tq + 1][t];
#pragma unroll
      for (int v = 0; v < DV; v += 4) {
        const float4 k4 = *reinterpret_cast<const float4*>(&sm.kt[t][tk * DV + v]);
        dq[0][v] = fmaf(d0, k4.x, dq[0][v]);
        dq[0][v + 1] = fmaf(d0, k4.y, dq[0][v + 1]);
        dq[0][v + 2] = fmaf(d0, k4.z, dq[0][v + 2]);
        dq[0][v + 3] = fmaf(d0, k4.w, dq[0][v + 3]);
        dq[1][v] = fmaf(d1, k4.x, dq[1][v]);
        dq[1][v + 1] = fmaf(d1, k4.y, dq[1][v + 1]);
        dq[1][v + 2] = fmaf(d1, k4.z, dq[1][v + 2]);
        dq[1][v + 3] = fmaf(d1, k4.w, dq[1][v + 3]);
      }
    }
    float gk[2][DV], gv[2][DV];
#pragma unroll
    for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
      for (int v = 0; v < DV; ++v) gk[c2][v] = gv[c2][v] = 0.f;
#pragma unroll 4
    for (int r = 0; r < kQC; ++r) {
      const float d0 = sm.dst[r][2 * tq], d1 = sm.dst[r][2 * tq + 1];
      const float p0 = sm.pt[r][2 * tq], p1 = sm.pt[r][2 * tq + 1];
#pragma unroll
      for (int v = 0; v < DV; v += 4) {
        const float4 q4 = *reinterpret_cast<const float4*>(&sm.q[r][tk * DV + v]);
        const float4 g4 = *reinterpret_cast<const float4*>(&sm.go[r][tk * DV + v]);
        gk[0][v] = fmaf(d0, q4.x, gk[0][v]);
        gk[0][v + 1] = fmaf(d0, q4.y, gk[0][v + 1]);
        gk[0][v + 2] = fmaf(d0, q4.z, gk[0][v + 2]);
        gk[0][v + 3] = fmaf(d0, q4.w, gk[0][v + 3]);
        gk[1][v] = fmaf(d1, q4.x, gk[1][v]);
        gk[1][v + 1] = fmaf(d1, q4.y, gk[1][v + 1]);
        gk[1][v + 2] = fmaf(d1, q4.z, gk[1][v + 2]);
        gk[1][v + 3] = fmaf(d1, q4.w, gk[1][v + 3]);
        gv[0][v] = fmaf(p0, g4.x, gv[0][v]);
        gv[0][v + 1] = fmaf(p0, g4.y, gv[0][v + 1]);
        gv[0][v + 2] = fmaf(p0, g4.z, gv[0][v + 2]);
        gv[0][v + 3] = fmaf(p0, g4.w, gv[0][v + 3]);
        gv[1][v] = fmaf(p1, g4.x, gv[1][v]);
        gv[1][v + 1] = fmaf(p1, g4.y, gv[1][v + 1]);
        gv[1][v + 2] = fmaf(p1, g4.z, gv[1][v + 2]);
        gv[1][v + 3] = fmaf(p1, g4.w, gv[1][v + 3]);
      }
    }
#pragma unroll
    for (int c2 = 0; c2 < 2; ++c2) {
      const int t = 2 * tq + c2;
      if (t >= kc) continue;
      const long long row = krow0 + t0 + t;
#pragma unroll
      for (int v = 0; v < DV; ++v) {
        atomicAdd(b.dK + row * D + tk * DV + v, gk[c2][v]);
        atomicAdd(b.dV + row * D + tk * DV + v, gv[c2][v]);
      }
    }
  }
  if (MODE == 1) {
    if (tk == 0) {
#pragma unroll
      for (int a2 = 0; a2 < 2; ++a2) {
        const int r = 2 * tq + a2;
        if (r >= qc) continue;
        b.lm[qrow0 + c0 + r] = mrun[a2];
        b.ll[qrow0 + c0 + r] = lrun[a2];
        b.la[qrow0 + c0 + r] = arun[a2];
      }
    }
    return;
  }
#pragma unroll
  for (int a2 = 0; a2 < 2; ++a2) {
    const int r = 2 * tq + a2;
    if (r >= qc) continue;
#pragma unroll
    for (int v = 0; v < DV; ++v) atomicAdd(b.dQ + (qrow0 + c0 + r) * D + tk * DV + v, dq[a2][v]);
  }
}

// causal: every query's log-sum-exp and D_q over its local block and the level
// problems it is a query of (the forward's merge: level l when bit l of its
// block index is set)
__global__ void bwd_combine_kernel(AttnArgs a, BwdArgs b, int L) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int N = a.qg.lv.N;
  if (e >= (long long)a.qg.BH * N) return;
  const int bhq = (int)(e / N), qpos = (int)(e - (long long)bhq * N);
  const Levels& lv = a.qg.lv;
  const int blk = qpos / L;
  float m = b.lm[e];
  for (int l = 0; l < lv.nlev; ++l)
    if ((blk >> l) & 1) {
      const int sz = L << l, p = blk >> (l + 1);
      const long long slot = (long long)bhq * lv.toks_per_bh + lv.tok_base[l] + (long long)p * sz +
                             (qpos - (2 * p + 1) * sz);
      m = fmaxf(m, b.pm[slot]);
    }
  float sum = b.ll[e] * __expf(b.lm[e] - m), acc = b.la[e] * __expf(b.lm[e] - m);
  for (int l = 0; l < lv.nlev; ++l)
    if ((blk >> l) & 1) {
      const int sz = L << l, p = blk >> (l + 1);
      const long long slot = (long long)bhq * lv.toks_per_bh + lv.tok_base[l] + (long long)p * sz +
                             (qpos - (2 * p + 1) * sz);
      const float w = __expf(b.pm[slot] - m);
      sum = fmaf(b.pl[slot], w, sum);
      acc = fmaf(b.pa[slot], w, acc);
    }
  b.lse_all[e] = m + __logf(sum);
  b.d_all[e] = acc / sum;
}

// ---------------------------------------------------------------------------
// per (key set, cluster): the summaries' gradients and the chain to k and v
// ---------------------------------------------------------------------------
template <typename T, int D, bool DIP>
__global__ void __launch_bounds__(kBT) bwd_cluster_kernel(AttnArgs a, BwdArgs b) {
  extern __shared__ __align__(16) float bc_raw[];
  float* M = bc_raw;                 // [D][D + 1]   M_j (DIPOLE)
  float* dM = M + D * (D + 1);       // [D][D + 1]   dM_j (DIPOLE)
  float* rows = dM + D * (D + 1);    // [32][D]      du rows, then k - mu rows
  float* nus = rows + 32 * D;        // [32][D]      nu rows, then v rows
  float* dS = nus + 32 * D;          // [D]
  float* dmt = dS + D;               // [D]          dmu_j total / n_j
  float* Sj = dmt + D;               // [D]
  float* mu = Sj + D;                // [D]
  const int kpid = blockIdx.x, j = blockIdx.y, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int Cq = a.Cq, Ck = a.Ck;
  const Prob pk = prob_of(a.kg, kpid);
  if (j >= pk.C) return;
  const size_t cj = (size_t)kpid * Ck + j;
  const int n = a.ks.counts[cj];
  if (n == 0) return;
  const float s = a.scale, invn = 1.f / (float)n;
  for (int d = tid; d < D; d += kBT) {
    Sj[d] = b.Sst[cj * D + d];
    mu[d] = a.ks.cent32[cj * D + d];
  }
  if (DIP)
    for (int e = tid; e < D * D; e += kBT) M[(e / D) * (D + 1) + e % D] = b.Mst[cj * D * D + e];
  // query sets reading key set kpid: the G q-heads of its kv-head
  const int ppb = a.kg.lv.pairs_per_bh;
  const int bhk = kpid / ppb, pi = kpid - bhk * ppb;
  const int Hq = a.qg.BH / a.B, Hkv = a.kg.BH / a.B;
  const int bb = bhk / Hkv, hk = bhk - bb * Hkv;
  constexpr int MR = DIP ? D * D / kBT : 1;
  float dm[MR];
#pragma unroll
  for (int r = 0; r < MR; ++r) dm[r] = 0.f;
  float dsacc = 0.f;
  for (int g = 0; g < a.G; ++g) {
    const int qpid = (bb * Hq + hk * a.G + g) * a.qg.lv.pairs_per_bh + pi;
    const Prob pq = prob_of(a.qg, qpid);
    for (int i0 = 0; i0 < pq.C; i0 += 32) {
      const int ic = imin(32, pq.C - i0);
      __syncthreads();
      for (int e = tid; e < ic * D; e += kBT) {
        const int r = e / D, d = e - r * D;
        rows[r * D + d] = b.dU[(((size_t)qpid * Cq + i0 + r) * Ck + j) * D + d];
        if (DIP) nus[r * D + d] = a.qs.cent32[((size_t)qpid * Cq + i0 + r) * D + d];
      }
      __syncthreads();
      if (tid < D)
        for (int r = 0; r < ic; ++r) dsacc += rows[r * D + tid];
      if (DIP) {
#pragma unroll
        for (int r = 0; r < MR; ++r) {
          const int idx = tid + kBT * r, e = idx / D, d = idx - e * D;
          float x = dm[r];
          for (int q = 0; q < ic; ++q) x = fmaf(rows[q * D + e], nus[q * D + d], x);
          dm[r] = x;
        }
        // dnu_i += (s / n) M^T du_ij
        for (int e = tid; e < ic * D; e += kBT) {
          const int r = e / D, d = e - r * D;
          float x = 0.f;
#pragma unroll 8
          for (int f = 0; f < D; ++f) x = fmaf(M[f * (D + 1) + d], rows[r * D + f], x);
          atomicAdd(b.dnu + ((size_t)qpid * Cq + i0 + r) * D + d, s * invn * x);
        }
      }
    }
  }
  __syncthreads();
  if (tid < D) dS[tid] = dsacc * invn;
  if (DIP) {
#pragma unroll
    for (int r = 0; r < MR; ++r) {
      const int idx = tid + kBT * r, e = idx / D, d = idx - e * D;
      dM[e * (D + 1) + d] = s * invn * dm[r];
    }
  }
  __syncthreads();
  // dmu_j total: the logits' part minus dM_j^T S_j, divided by n_j
  for (int d = tid; d < D; d += kBT) {
    float x = b.dmu[cj * D + d];
    if (DIP)
      for (int e = 0; e < D; ++e) x = fmaf(-dM[e * (D + 1) + d], Sj[e], x);
    dmt[d] = x * invn;
  }
  __syncthreads();
  // members: dv_t += dS + dM (k_t - mu), dk_t += dmu / n + dM^T v_t
  const int off = a.ks.off[(size_t)kpid * (Ck + 1) + j];
  const int* perm = a.ks.perm + pk.slot0;
  const T* K = static_cast<const T*>(a.kg.X);
  const T* V = static_cast<const T*>(a.V);
  constexpr int DL = D / 32;
  for (int c0 = 0; c0 < n; c0 += 32) {
    const int cnt = imin(32, n - c0);
    __syncthreads();
    for (int e = tid; e < cnt * D; e += kBT) {
      const int r = e / D, d = e - r * D;
      const long long row = pk.row0 + perm[off + c0 + r];
      rows[r * D + d] = ldg_<T>(K + row * D + d) - mu[d];
      nus[r * D + d] = ldg_<T>(V + row * D + d);
    }
    __syncthreads();
    for (int r = warp; r < cnt; r += kBW) {
      const long long row = pk.row0 + perm[off + c0 + r];
#pragma unroll
      for (int u = 0; u < DL; ++u) {
        const int e = lane + 32 * u;
        float gv = dS[e], gk = dmt[e];
        if (DIP)
          for (int f = 0; f < D; ++f) {
            gv = fmaf(dM[e * (D + 1) + f], rows[r * D + f], gv);
            gk = fmaf(dM[f * (D + 1) + e], nus[r * D + f], gk);
          }
        if (a.qg.lv.causal) {  // a key sits in one key set per level
          atomicAdd(b.dV + row * D + e, gv);
          atomicAdd(b.dK + row * D + e, gk);
        } else {  // the member's only writer in this launch
          b.dV[row * D + e] += gv;
          b.dK[row * D + e] += gk;
        }
      }
    }
  }
}

// dq += dnu_i / m_i for the members of every query cluster (DIPOLE)
template <int D>
__global__ void __launch_bounds__(kBT) bwd_query_nu_kernel(AttnArgs a, BwdArgs b) {
  const int qpid = blockIdx.x, i = blockIdx.y, tid = threadIdx.x;
  const int Cq = a.Cq;
  const Prob pq = prob_of(a.qg, qpid);
  if (i >= pq.C) return;
  const int m = a.qs.counts[(size_t)qpid * Cq + i];
  if (m == 0) return;
  const int off = a.qs.off[(size_t)qpid * (Cq + 1) + i];
  const int* perm = a.qs.perm + pq.slot0;
  const float* dn = b.dnu + ((size_t)qpid * Cq + i) * D;
  const float inv = 1.f / (float)m;
  for (int e = tid; e < m * D; e += kBT) {
    const int r = e / D, d = e - r * D;
    const long long row = pq.row0 + perm[off + r];
    if (a.qg.lv.causal) atomicAdd(b.dQ + row * D + d, dn[d] * inv);  // one query set per level
    else b.dQ[row * D + d] += dn[d] * inv;
  }
}

template <typename T, int D, bool DIP>
size_t query_smem(int Ck) {
  return sizeof(QuerySmem<D>) + (size_t)Ck * (D + 1) * 4 + (size_t)2 * kQC * Ck * 4 + (size_t)2 * Ck * 4;
}

template <typename T, typename TO, int D, bool DIP>
void launch_bwd(const AttnArgs& a, const Stage1& s1, const BwdArgs& b, int L, cudaStream_t st) {
  const int nk = a.ks.nprob, nq = a.qs.nprob;
  if (nk > 0) {
    ProfScope ps(st, "bwd_key_stats");
    bwd_key_stats_kernel<T, D, DIP><<<dim3(nk, a.Ck), kBT, 0, st>>>(a, b);
  }
  if (DIP && nq > 0) {
    ProfScope ps(st, "bwd_u_table");
    const size_t sm = (size_t)(D * (D + 1) + kBT) * 4;
    cudaFuncSetAttribute(bwd_u_table_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    bwd_u_table_kernel<D><<<dim3(nq, a.Ck), kBT, sm, st>>>(a, b);
  }
  if (L == 0) {
    ProfScope ps(st, "bwd_query");
    const size_t sm = query_smem<T, D, DIP>(a.Ck);
    cudaFuncSetAttribute(bwd_query_kernel<T, TO, D, DIP, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)sm);
    bwd_query_kernel<T, TO, D, DIP, 0><<<dim3(nq, a.Cq), kBT, sm, st>>>(a, s1, b);
  } else {
    const size_t sm = query_smem<T, D, DIP>(a.Ck);
    const size_t sl = sizeof(QuerySmem<D>);
    const long long rows = (long long)a.qg.BH * a.qg.lv.N;
    const dim3 lgrid(a.qg.BH, cdiv(a.qg.lv.N, kQC));
    cudaFuncSetAttribute(bwd_query_kernel<T, TO, D, DIP, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)sm);
    cudaFuncSetAttribute(bwd_query_kernel<T, TO, D, DIP, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)sm);
    cudaFuncSetAttribute(bwd_local_kernel<T, TO, D, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sl);
    cudaFuncSetAttribute(bwd_local_kernel<T, TO, D, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sl);
    {
      ProfScope ps(st, "bwd_lse");
      if (nq > 0) bwd_query_kernel<T, TO, D, DIP, 1><<<dim3(nq, a.Cq), kBT, sm, st>>>(a, s1, b);
      bwd_local_kernel<T, TO, D, 1><<<lgrid, kBT, sl, st>>>(a, b, L);
      bwd_combine_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(a, b, L);
    }
    {
      ProfScope ps(st, "bwd_query");
      if (nq > 0) bwd_query_kernel<T, TO, D, DIP, 2><<<dim3(nq, a.Cq), kBT, sm, st>>>(a, s1, b);
    }
    {
      ProfScope ps(st, "bwd_local");
      bwd_local_kernel<T, TO, D, 2><<<lgrid, kBT, sl, st>>>(a, b, L);
    }
  }
  if (nk > 0) {
    ProfScope ps(st, "bwd_cluster");
    const size_t sm = (size_t)(2 * D * (D + 1) + 64 * D + 4 * D) * 4;
    cudaFuncSetAttribute(bwd_cluster_kernel<T, D, DIP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)sm);
    bwd_cluster_kernel<T, D, DIP><<<dim3(nk, a.Ck), kBT, sm, st>>>(a, b);
  }
  if (DIP && nq > 0) {
    ProfScope ps(st, "bwd_query_nu");
    bwd_query_nu_kernel<D><<<dim3(nq, a.Cq), kBT, 0, st>>>(a, b);
  }
}

template <typename T, typename TO>
void dispatch_d(const AttnArgs& a, const Stage1& s1, const BwdArgs& b, int L, cudaStream_t st) {
  const bool dip = a.mode == 1;
  if (a.qg.D == 64) {
    if (dip) launch_bwd<T, TO, 64, true>(a, s1, b, L, st);
    else launch_bwd<T, TO, 64, false>(a, s1, b, L, st);
  } else {
    if (dip) launch_bwd<T, TO, 128, true>(a, s1, b, L, st);
    else launch_bwd<T, TO, 128, false>(a, s1, b, L, st);
  }
}

}  // namespace

bool backward_supported(int D, int Ck, int mode) {
  return (mode == 0 || mode == 1) && (D == 64 || D == 128) && Ck * D <= 16384;
}

static void run_bwd(const AttnArgs& a, const Stage1& s1, const BwdArgs& b, int L, cudaStream_t st) {
  using bf = __nv_bfloat16;
  if (a.qg.dtype == 0) {
    if (b.o_f32) dispatch_d<bf, float>(a, s1, b, L, st);
    else dispatch_d<bf, bf>(a, s1, b, L, st);
  } else {
    dispatch_d<float, float>(a, s1, b, L, st);
  }
}

void run_attn_bwd(const AttnArgs& a, const Stage1& s1, const BwdArgs& b, cudaStream_t st) {
  run_bwd(a, s1, b, 0, st);
}

void run_attn_bwd_causal(const AttnArgs& a, const Stage1& s1, const BwdArgs& b, int L,
                         cudaStream_t st) {
  run_bwd(a, s1, b, L, st);
}

}  // namespace muse
