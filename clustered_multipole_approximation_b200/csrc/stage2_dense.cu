// Stage 2 of the low causal levels, one term per key token, on mma.sync
// tensor-core tiles (bf16 inputs, DIPOLE summaries).
//
// For a query q of query cluster i, the DIPOLE far-field term of a key cluster
// j outside R_i (gist.science page "Multipole Semantic Attention: A Fast
// Approximation of Softmax Attention for Pretraining", Technical Summary, Core
// Mechanisms: the monopole and dipole summaries and Stage 2) has weight
// exp(s q.mu_j + log n_j) and value u_ij = (1/n_j) sum_{t in j} v_t (1 + s nu_i.(k_t - mu_j)).
// Weight times value, and the weight itself, are sums over the cluster's
// tokens:
//     exp(s q.mu_j + log n_j) u_ij = sum_{t in j} exp(s q.mu_j) (1 + s nu_i.(k_t - mu_j)) v_t,
//     exp(s q.mu_j + log n_j)      = sum_{t in j} exp(s q.mu_j).
// So the far field is one softmax term per key token t, with logit
// s q.mu_a(t) and value factor f = 1 + s nu_i.(k_t - mu_a(t)) (the factor is
// left out of the denominator).  A key of a retrieved cluster takes the exact
// term instead: logit s q.k_t, factor 1.  One online softmax over every key of
// the pair's key block then equals the per-cluster form up to rounding.
//
// Where a block holds few tokens per cluster (s <= 8 C) this costs less than
// the per-cluster tables: those hold C_q x C_k x D summaries for only s
// queries, and a query cluster of about four tokens fills a 16-row
// tensor-core tile a quarter full.  Here every tile is full: 8 warps x 16
// consecutive queries of the query block against 32-key blocks.  Per block:
//   S_ex  = Q K^T                                  bf16 q and k, exact
//   S_far = Q (mu_hi + mu_lo)^T                    centroid row of each key's cluster
//   F     = (nu_hi + nu_lo) K^T - (nu_hi + nu_lo)(mu_hi + mu_lo)^T   (lo x lo left out)
// all m16n8k16 MMAs with fp32 accumulation (hi + lo: the bf16 split of the
// fp32 centroid, residual 2^-17 relative).  The negative part of F enters
// through sign-flipped nu fragments in the same accumulator, k-step by
// k-step, so the cancellation of nu.k against nu.mu happens in fp32.  The
// weights p f enter P V as an fp16 hi + lo pair, V in fp16.
//
// The fine-query dipole (mode DIPOLE_Q, an accuracy variant: u_qj = (S_j +
// s M_j q) / n_j) is the same per-token sum with the query in place of its
// cluster centroid: f = 1 + s q.(k_t - mu_a(t)) = 1 + s (S_ex - S_far), from
// the two score tiles the kernel forms anyway.  It has no per-cluster form
// short of q-dependent M_j products, so in that mode every level (and the
// acausal layer, one block of N keys) runs here; the key clusters are then
// read per block from global memory instead of a block table.
#include <cuda_fp16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"

namespace muse {

namespace {

constexpr int kDQ = 128;            // queries per CTA (8 warps x 16 rows)
constexpr int kDK = 32;             // key rows per block
constexpr int kDThreads = 256;
constexpr int kDMaxC = 256;         // clusters per problem (retrieval bit table)
constexpr int kDMaxS = 2048;        // block size (key cluster table)
constexpr int kDTokPerCluster = 8;  // per key token where s <= 8 C

template <int D>
struct DenseBuf {
  int kcl[kDK];                  // cluster of each key of the block
  __nv_bfloat16 k[kDK][D + 8];   // k_t
  __nv_bfloat16 mh[kDK][D + 8];  // hi part of mu_a(t)
  __nv_bfloat16 ml[kDK][D + 8];  // lo part of mu_a(t)
  __half v[kDK][D + 8];          // v_t in fp16
};

template <int D>
struct DenseSmem {
  __nv_bfloat16 q[kDQ][D + 8];
  __nv_bfloat16 nh[kDQ][D + 8];  // hi part of nu_i(q)
  __nv_bfloat16 nl[kDQ][D + 8];  // lo part of nu_i(q)
  DenseBuf<D> buf[2];
  unsigned rmask[kDMaxC][kDMaxC / 32];  // bit j of row i: key cluster j is in R_i
  int qcl[kDQ];                         // cluster of each query row
  int nex[kDMaxC];                      // keys of the retrieved clusters, per query cluster
};

}  // namespace

template <int D, bool FQ>
__global__ void __launch_bounds__(kDThreads, D == 64 ? 2 : 1)
    stage2_dense_kernel(AttnArgs a, Stage1 s1, int qp0) {
  extern __shared__ __align__(16) unsigned char dn_raw[];
  DenseSmem<D>& sm = *reinterpret_cast<DenseSmem<D>*>(dn_raw);
  constexpr int KD = D / 16, ND = D / 8, CH = D / 8;
  const int qpid = qp0 + blockIdx.x;
  const Prob pq = prob_of(a.qg, qpid);
  if (!((a.dense_lv >> pq.level) & 1)) return;  // a level with per-cluster tables
  const int q0 = blockIdx.y * kDQ;
  if (q0 >= pq.s) return;
  const int kpid = kv_problem(a, qpid);
  const Prob pk = prob_of(a.kg, kpid);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int Cq = a.Cq, Ck = a.Ck, cq = pq.C, ck = pk.C, S = pk.s;

  // ---- per-CTA tables ------------------------------------------------------
  const int* kas = a.ks.assign + pk.slot0;
  const int* qas = a.qs.assign + pq.slot0 + q0;
  for (int r = tid; r < kDQ; r += kDThreads) sm.qcl[r] = min(max(qas[r], 0), cq - 1);
  for (int e = tid; e < cq * (kDMaxC / 32); e += kDThreads) (&sm.rmask[0][0])[e] = 0u;
  for (int i = tid; i < cq; i += kDThreads) sm.nex[i] = 0;
  __syncthreads();
  const int* kc = a.ks.counts + (size_t)kpid * Ck;
  if (a.topk > 0) {
    const int K1 = a.topk;
    for (int e = tid; e < cq * K1; e += kDThreads) {
      const int i = e / K1, r = e - i * K1;
      if (r < s1.nsel[(size_t)qpid * Cq + i]) {
        const int j = s1.sel[((size_t)qpid * Cq + i) * K1 + r];
        if (j >= 0 && j < ck) {
          atomicOr(&sm.rmask[i][j >> 5], 1u << (j & 31));
          if (a.n_exact != nullptr) atomicAdd(&sm.nex[i], kc[j]);
        }
      }
    }
  }

  // ---- operands: query rows, their clusters' centroids, key blocks ----------
  const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(a.qg.X);
  const __nv_bfloat16* K = static_cast<const __nv_bfloat16*>(a.kg.X);
  const __half* V16 = a.V16;
  const __nv_bfloat16* nuh = a.qs.cbf_hi + (size_t)qpid * Cq * D;
  const __nv_bfloat16* nul = a.qs.cbf_lo + (size_t)qpid * Cq * D;
  const __nv_bfloat16* muh = a.ks.cbf_hi + (size_t)kpid * Ck * D;
  const __nv_bfloat16* mul = a.ks.cbf_lo + (size_t)kpid * Ck * D;
  for (int e = tid; e < kDQ * CH; e += kDThreads) {
    const int r = e / CH, c = (e % CH) * 8;
    const size_t qo = (size_t)(pq.row0 + q0 + r) * D + c;
    const size_t no = (size_t)sm.qcl[r] * D + c;
    cp16(&sm.q[r][c], Q + qo, 16);
    cp16(&sm.nh[r][c], nuh + no, 16);
    cp16(&sm.nl[r][c], nul + no, 16);
  }
  auto issue = [&](int b, DenseBuf<D>& B) {
    const int t0 = b * kDK;
    for (int r = tid; r < kDK; r += kDThreads) B.kcl[r] = min(max(kas[t0 + r], 0), ck - 1);
    for (int e = tid; e < kDK * CH; e += kDThreads) {
      const int r = e / CH, c = (e % CH) * 8, t = t0 + r;
      const size_t ko = (size_t)(pk.row0 + t) * D + c;
      const size_t mo = (size_t)min(max(kas[t], 0), ck - 1) * D + c;
      cp16(&B.k[r][c], K + ko, 16);
      cp16(&B.mh[r][c], muh + mo, 16);
      cp16(&B.ml[r][c], mul + mo, 16);
      cp16(&B.v[r][c], V16 + ko, 16);
    }
    cp_commit();
  };
  issue(0, sm.buf[0]);  // commits the query rows with block 0

  const int nkb = S / kDK;
  const float s = a.scale, sl2 = a.scale * 1.4426950408889634f;  // logits in base-2 units
  const int r0 = warp * 16 + g;                                    // rows r0 and r0 + 8
  const unsigned* mrow_bits[2] = {sm.rmask[sm.qcl[r0]], sm.rmask[sm.qcl[r0 + 8]]};
  float o[ND][4];
#pragma unroll
  for (int n = 0; n < ND; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float mrow[2] = {kMaxFloor, kMaxFloor}, lrow[2] = {0.f, 0.f};

  for (int b = 0; b < nkb; ++b) {
    if (b + 1 < nkb) {
      issue(b + 1, sm.buf[(b + 1) & 1]);
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    const DenseBuf<D>& B = sm.buf[b & 1];
    float sx[kDK / 8][4], sf[kDK / 8][4], fd[kDK / 8][4];
#pragma unroll
    for (int n = 0; n < kDK / 8; ++n)
#pragma unroll
      for (int h = 0; h < 4; ++h) sx[n][h] = sf[n][h] = fd[n][h] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KD; ++kk) {
      const int row = warp * 16 + (lane & 15), col = kk * 16 + (lane >> 4) * 8;
      uint32_t qa[4], ha[4] = {0, 0, 0, 0}, la[4] = {0, 0, 0, 0}, hn[4], ln[4];
      ldsm_x4(smem_u32(&sm.q[row][col]), qa[0], qa[1], qa[2], qa[3]);
      if (!FQ) {
        ldsm_x4(smem_u32(&sm.nh[row][col]), ha[0], ha[1], ha[2], ha[3]);
        ldsm_x4(smem_u32(&sm.nl[row][col]), la[0], la[1], la[2], la[3]);
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        hn[x] = ha[x] ^ 0x80008000u;  // -nu_hi (sign bit of both bf16 halves)
        ln[x] = la[x] ^ 0x80008000u;  // -nu_lo
      }
#pragma unroll
      for (int np = 0; np < kDK / 16; ++np) {
        const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int kc_ = kk * 16 + ((lane >> 3) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_u32(&B.k[key][kc_]), b0, b1, b2, b3);
        mma_bf16(sx[2 * np], qa, b0, b1);
        mma_bf16(sx[2 * np + 1], qa, b2, b3);
        if (!FQ) {
          mma_bf16(fd[2 * np], ha, b0, b1);
          mma_bf16(fd[2 * np + 1], ha, b2, b3);
          mma_bf16(fd[2 * np], la, b0, b1);
          mma_bf16(fd[2 * np + 1], la, b2, b3);
        }
        ldsm_x4(smem_u32(&B.mh[key][kc_]), b0, b1, b2, b3);
        mma_bf16(sf[2 * np], qa, b0, b1);
        mma_bf16(sf[2 * np + 1], qa, b2, b3);
        if (!FQ) {
          mma_bf16(fd[2 * np], hn, b0, b1);
          mma_bf16(fd[2 * np + 1], hn, b2, b3);
          mma_bf16(fd[2 * np], ln, b0, b1);
          mma_bf16(fd[2 * np + 1], ln, b2, b3);
        }
        ldsm_x4(smem_u32(&B.ml[key][kc_]), b0, b1, b2, b3);
        mma_bf16(sf[2 * np], qa, b0, b1);
        mma_bf16(sf[2 * np + 1], qa, b2, b3);
        if (!FQ) {
          mma_bf16(fd[2 * np], hn, b0, b1);
          mma_bf16(fd[2 * np + 1], hn, b2, b3);
        }
      }
    }
    if (FQ) {  // q.(k_t - mu_a(t)) from the exact and far scores
#pragma unroll
      for (int n = 0; n < kDK / 8; ++n)
#pragma unroll
        for (int h = 0; h < 4; ++h) fd[n][h] = sx[n][h] - sf[n][h];
    }
    // exact or far term per (row, key); running maximum of the chosen logits
    const int t0 = b * kDK;
    float mx[2] = {kMaxFloor, kMaxFloor};
#pragma unroll
    for (int n = 0; n < kDK / 8; ++n) {
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const int j = B.kcl[n * 8 + 2 * t4 + (h & 1)];
        const bool ex = (mrow_bits[h >> 1][j >> 5] >> (j & 31)) & 1u;
        const float lg = sl2 * (ex ? sx[n][h] : sf[n][h]);
        fd[n][h] = ex ? 1.f : fmaf(s, fd[n][h], 1.f);
        sx[n][h] = lg;
        mx[h >> 1] = fmaxf(mx[h >> 1], lg);
      }
    }
    float scale[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      const float mn = fmaxf(mrow[r], mx[r]);
      scale[r] = fast_exp2(mrow[r] - mn);
      mrow[r] = mn;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int n = 0; n < kDK / 8; ++n) {
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float p = fast_exp2(sx[n][h] - mrow[h >> 1]);
        rs[h >> 1] += p;          // the denominator takes the weight alone
        sx[n][h] = p * fd[n][h];  // the numerator weight carries the dipole factor
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      rs[r] += __shfl_xor_sync(0xffffffffu, rs[r], 1);
      rs[r] += __shfl_xor_sync(0xffffffffu, rs[r], 2);
      lrow[r] = lrow[r] * scale[r] + rs[r];
    }
#pragma unroll
    for (int n = 0; n < ND; ++n) {
      o[n][0] *= scale[0];
      o[n][1] *= scale[0];
      o[n][2] *= scale[1];
      o[n][3] *= scale[1];
    }
    // the weights p f take either sign and can exceed the denominator's
    // terms, so they enter P V as an fp16 hi + lo pair (residual 2^-22)
#pragma unroll
    for (int kk = 0; kk < kDK / 16; ++kk) {
      uint32_t pa[4], pl[4];
      split_h2(sx[2 * kk][0], sx[2 * kk][1], pa[0], pl[0]);
      split_h2(sx[2 * kk][2], sx[2 * kk][3], pa[1], pl[1]);
      split_h2(sx[2 * kk + 1][0], sx[2 * kk + 1][1], pa[2], pl[2]);
      split_h2(sx[2 * kk + 1][2], sx[2 * kk + 1][3], pa[3], pl[3]);
#pragma unroll
      for (int np = 0; np < ND / 2; ++np) {
        const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int col = np * 16 + (lane >> 4) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32(&B.v[key][col]), b0, b1, b2, b3);
        mma_f16(o[2 * np], pa, b0, b1);
        mma_f16(o[2 * np + 1], pa, b2, b3);
        mma_f16(o[2 * np], pl, b0, b1);
        mma_f16(o[2 * np + 1], pl, b2, b3);
      }
    }
    __syncthreads();
  }
  // ---- each row: the normalised output (acausal), or the level partial:
  // normalised output and log-sum-exp (causal) -------------------------------
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int tq = q0 + r0 + 8 * r;  // problem-local query index
    const float inv = 1.f / lrow[r];
    if (FQ && a.O != nullptr) {  // only the fine-query dipole runs acausal layers here
      const long long orow = pq.row0 + tq;
#pragma unroll
      for (int n = 0; n < ND; ++n) {
        const float x0 = o[n][2 * r] * inv, x1 = o[n][2 * r + 1] * inv;
        if (a.out_f32) {
          *reinterpret_cast<float2*>(static_cast<float*>(a.O) + orow * D + n * 8 + 2 * t4) = make_float2(x0, x1);
        } else {
          *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(a.O) + orow * D + n * 8 + 2 * t4) =
              __floats2bfloat162_rn(x0, x1);
        }
      }
      if (t4 == 0 && a.n_exact != nullptr) a.n_exact[orow] = sm.nex[sm.qcl[r0 + 8 * r]];
      continue;
    }
    float* pp = a.part + (size_t)(pq.slot0 + tq) * (D + 1);
#pragma unroll
    for (int n = 0; n < ND; ++n) {
      pp[n * 8 + 2 * t4] = o[n][2 * r] * inv;
      pp[n * 8 + 2 * t4 + 1] = o[n][2 * r + 1] * inv;
    }
    if (t4 == 0) {
      pp[D] = (mrow[r] + log2f(lrow[r])) * 0.6931471805599453f;
      if (a.n_exact != nullptr)
        atomicAdd(reinterpret_cast<unsigned long long*>(a.n_exact + pq.row0 + tq),
                  (unsigned long long)sm.nex[sm.qcl[r0 + 8 * r]]);
    }
  }
}

template <int D, bool FQ>
static void launch_dense(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, int smax,
                         cudaStream_t st) {
  // set on every launch: the attribute is per device, and the call is cheap
  cudaFuncSetAttribute(stage2_dense_kernel<D, FQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)sizeof(DenseSmem<D>));
  const dim3 grid(nqp, smax / kDQ);
  stage2_dense_kernel<D, FQ><<<grid, kDThreads, sizeof(DenseSmem<D>), st>>>(a, s1, qp0);
}

int dense_levels(const Levels& lv, int D, int Cq, int Ck) {
  if (!lv.causal || (D != 64 && D != 128) || Cq > kDMaxC || Ck > kDMaxC) return 0;
  int m = 0;
  for (int l = 0; l < lv.nlev; ++l) {
    const int s = lv.s[l], ce = imin(Ck, s);
    if (s % kDQ == 0 && s <= kDMaxS && s <= kDTokPerCluster * ce) m |= 1 << l;
  }
  return m;
}

int fine_query_dense_levels(const Levels& lv, int D, int Cq, int Ck) {
  if ((D != 64 && D != 128) || Cq > kDMaxC || Ck > kDMaxC) return -1;
  int m = 0;
  for (int l = 0; l < lv.nlev; ++l) {
    if (lv.s[l] % kDQ != 0) return -1;
    m |= 1 << l;
  }
  return m;
}

void run_stage2_dense(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st) {
  int smax = 0;
  for (int l = 0; l < a.qg.lv.nlev; ++l)
    if ((a.dense_lv >> l) & 1) smax = smax > a.qg.lv.s[l] ? smax : a.qg.lv.s[l];
  if (smax == 0) return;
  ProfScope ps(st, "stage2_dense");
  const bool fq = a.mode == 3;
  if (a.qg.D == 64) {
    if (fq) launch_dense<64, true>(a, s1, qp0, nqp, smax, st);
    else launch_dense<64, false>(a, s1, qp0, nqp, smax, st);
  } else {
    if (fq) launch_dense<128, true>(a, s1, qp0, nqp, smax, st);
    else launch_dense<128, false>(a, s1, qp0, nqp, smax, st);
  }
}

}  // namespace muse
