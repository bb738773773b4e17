// Stage 1 of MuSe for DIPOLE summaries on tensor cores (bf16 inputs).
//
// For key cluster j of a key block and every query cluster i of the paired
// query block, the dipole-corrected summary value is
//   u_ij = (1/n_j) sum_{t in j} v_t (1 + s nu_i . (k_t - mu_j))
// (newx.sg page "Multipole Semantic Attention: A Fast Approximation of Softmax
// Attention for Pretraining", Abstract: monopole plus dipole corrections; the
// first-order term of the kept cross term, gist.science page, Technical
// Summary, Core Mechanisms, residual decomposition).  Per CTA (one query
// problem, one key cluster) this is two small GEMMs over the cluster's members:
//   G[t][i] = k_t . nu_i           (bf16 keys x bf16 hi + lo split of nu)
//   W[t][i] = 1 + s (G[t][i] - nu_i . mu_j)
//   U^T[e][i] = sum_t v_t[e] W[t][i]   (fp16 V x fp16 W, fp32 accumulation)
// with mma.sync m16n8k16 tiles; u_ij is written in fp16, the operand form of
// stage 2.
#include <cuda_fp16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace muse {

namespace {

constexpr int kT = 64;     // members per chunk
constexpr int kI = 128;    // query clusters per pass
constexpr int kThr = 128;  // 4 warps

__device__ inline uint32_t su32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ inline void cp16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(su32(dst)), "l"(src),
               "r"(src_bytes));
}
__device__ inline void cp_commit_wait() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
}
__device__ inline void ldsm4(uint32_t a, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
__device__ inline void ldsm4t(uint32_t a, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
__device__ inline void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ inline void mma_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D>
struct S1Smem {
  __nv_bfloat16 nh[kI][D + 8];  // query centroids, bf16 hi part
  __nv_bfloat16 nl[kI][D + 8];  // and lo part
  __nv_bfloat16 k[kT][D + 8];   // member keys (exact)
  __half v[kT][D + 8];          // member values (fp16 copy)
  __half w[kI][kT + 8];         // weights, [i][t]
  float nm[kI];                 // nu_i . mu_j
  float mu[D];
};

__device__ inline int kvp1(const AttnArgs& a, int qpid) {
  const int ppb = a.qg.lv.pairs_per_bh;
  const int bhq = qpid / ppb, pi = qpid - bhq * ppb;
  const int Hq = a.qg.BH / a.B, Hkv = a.kg.BH / a.B;
  const int b = bhq / Hq, hq = bhq - b * Hq;
  return (b * Hkv + hq / a.G) * a.kg.lv.pairs_per_bh + pi;
}

}  // namespace

template <int D>
size_t stage1_mma_smem() {
  return sizeof(S1Smem<D>);
}

template <int D>
__global__ void __launch_bounds__(kThr) stage1_dipole_mma_kernel(AttnArgs a, Stage1 s1, int qp0) {
  extern __shared__ __align__(16) unsigned char s1raw[];
  S1Smem<D>& sm = *reinterpret_cast<S1Smem<D>*>(s1raw);
  constexpr int KD = D / 16;      // k-steps of the first GEMM
  constexpr int MT = D / 64;      // row tiles of 16 (per warp) of the second GEMM
  constexpr int CH = D / 8;       // 16-byte chunks per row
  const int lq = blockIdx.x, qpid = qp0 + lq, j = blockIdx.y;
  const Prob pq = prob_of(a.qg, qpid);
  const int kpid = kvp1(a, qpid);
  const Prob pk = prob_of(a.kg, kpid);
  if (j >= pk.C) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int Cq = a.Cq, Ck = a.Ck;
  const int nj = a.ks.counts[(size_t)kpid * Ck + j];
  const size_t ij0 = ((size_t)lq * Cq) * Ck + j;  // + i * Ck
  if (nj == 0) {
    for (int i = tid; i < pq.C; i += kThr) {
      s1.logW[ij0 + (size_t)i * Ck] = -INFINITY;
      s1.fbias[ij0 + (size_t)i * Ck] = -INFINITY;
    }
    return;
  }
  const float lognj = logf((float)nj);
  for (int i = tid; i < pq.C; i += kThr) {
    s1.logW[ij0 + (size_t)i * Ck] = lognj;
    s1.fbias[ij0 + (size_t)i * Ck] = lognj;
  }
  const int off = a.ks.off[(size_t)kpid * (Ck + 1) + j];
  const int* perm = a.ks.perm + pk.slot0;
  const __nv_bfloat16* K = static_cast<const __nv_bfloat16*>(a.kg.X);
  const float* mug = a.ks.cent32 + ((size_t)kpid * Ck + j) * D;
  for (int d = tid; d < D; d += kThr) sm.mu[d] = mug[d];
  const float s = a.scale;
  const float inv_n = 1.f / (float)nj;

  for (int i0 = 0; i0 < pq.C; i0 += kI) {
    const int ic = imin(kI, pq.C - i0);
    // query centroids (bf16 split) of this pass; rows past ic are zero
    for (int e = tid; e < kI * CH; e += kThr) {
      const int r = e / CH, c = (e % CH) * 8;
      const bool live = r < ic;
      const size_t o = ((size_t)qpid * Cq + i0 + (live ? r : 0)) * D + c;
      cp16(&sm.nh[r][c], a.qs.cbf_hi + o, live ? 16 : 0);
      cp16(&sm.nl[r][c], a.qs.cbf_lo + o, live ? 16 : 0);
    }
    __syncthreads();
    for (int r = tid; r < kI; r += kThr) {
      float dt = 0.f;
      if (r < ic) {
        const float* nu = a.qs.cent32 + ((size_t)qpid * Cq + i0 + r) * D;
        for (int d = 0; d < D; ++d) dt = fmaf(nu[d], sm.mu[d], dt);
      }
      sm.nm[r] = dt;
    }
    float u[MT][kI / 8][4];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
      for (int n = 0; n < kI / 8; ++n) u[m][n][0] = u[m][n][1] = u[m][n][2] = u[m][n][3] = 0.f;

    for (int t0 = 0; t0 < nj; t0 += kT) {
      const int nt = imin(kT, nj - t0);
      __syncthreads();
      for (int e = tid; e < kT * CH; e += kThr) {
        const int r = e / CH, c = (e % CH) * 8;
        const bool live = r < nt;
        const long long row = pk.row0 + (live ? perm[off + t0 + r] : 0);
        cp16(&sm.k[r][c], K + row * D + c, live ? 16 : 0);
        cp16(&sm.v[r][c], a.V16 + row * D + c, live ? 16 : 0);
      }
      cp_commit_wait();
      __syncthreads();
      // ---- G = K nu^T: warp w owns members 16w..16w+15 ----------------------
      {
        float gacc[kI / 8][4];
#pragma unroll
        for (int n = 0; n < kI / 8; ++n) gacc[n][0] = gacc[n][1] = gacc[n][2] = gacc[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KD; ++kk) {
          uint32_t af[4];
          ldsm4(su32(&sm.k[warp * 16 + (lane & 15)][kk * 16 + (lane >> 4) * 8]), af);
#pragma unroll
          for (int np = 0; np < kI / 16; ++np) {
            const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
            const int col = kk * 16 + ((lane >> 3) & 1) * 8;
            uint32_t bh[4], bl[4];
            ldsm4(su32(&sm.nh[key][col]), bh);
            ldsm4(su32(&sm.nl[key][col]), bl);
            mma_bf16(gacc[2 * np], af, bh[0], bh[1]);
            mma_bf16(gacc[2 * np + 1], af, bh[2], bh[3]);
            mma_bf16(gacc[2 * np], af, bl[0], bl[1]);
            mma_bf16(gacc[2 * np + 1], af, bl[2], bl[3]);
          }
        }
        // W[t][i] = 1 + s (G - nu_i . mu_j), stored [i][t]; members past nt get 0
#pragma unroll
        for (int n = 0; n < kI / 8; ++n) {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int t = warp * 16 + g + 8 * (h >> 1);
            const int i = n * 8 + 2 * t4 + (h & 1);
            const float wv = t < nt ? fmaf(s, gacc[n][h] - sm.nm[i], 1.f) : 0.f;
            sm.w[i][t] = __float2half_rn(wv);
          }
        }
      }
      __syncthreads();
      // ---- U^T[e][i] += V^T W: warp w owns value rows 16(w + 4m)... ------------
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const int e0 = (warp + 4 * m) * 16;
#pragma unroll
        for (int kk = 0; kk < kT / 16; ++kk) {
          uint32_t af[4];
          const int tr = kk * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int ec = e0 + ((lane >> 3) & 1) * 8;
          ldsm4t(su32(&sm.v[tr][ec]), af);
          // ldmatrix.trans of the [t][e] tile gives A = V^T with (e, t) fragments
          const uint32_t a4[4] = {af[0], af[1], af[2], af[3]};
#pragma unroll
          for (int np = 0; np < kI / 16; ++np) {
            const int ir = np * 16 + (lane & 7) + ((lane >> 4) << 3);
            const int tc = kk * 16 + ((lane >> 3) & 1) * 8;
            uint32_t bw[4];
            ldsm4(su32(&sm.w[ir][tc]), bw);
            mma_f16(u[m][2 * np], a4, bw[0], bw[1]);
            mma_f16(u[m][2 * np + 1], a4, bw[2], bw[3]);
          }
        }
      }
    }
    // ---- u_ij = U^T[e][i] / n_j, in fp16 -------------------------------------
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const int e0 = (warp + 4 * m) * 16;
#pragma unroll
      for (int n = 0; n < kI / 8; ++n) {
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int e = e0 + g + 8 * (h >> 1);
          const int i = n * 8 + 2 * t4 + (h & 1);
          if (i < ic) s1.Uh[(ij0 + (size_t)(i0 + i) * Ck) * D + e] = __float2half_rn(u[m][n][h] * inv_n);
        }
      }
    }
  }
}

template <int D>
static void launch_t(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(stage1_dipole_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)stage1_mma_smem<D>());
    attr = true;
  }
  stage1_dipole_mma_kernel<D><<<dim3(nqp, a.Ck), kThr, stage1_mma_smem<D>(), st>>>(a, s1, qp0);
}

void run_stage1_dipole_mma(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st) {
  if (a.qg.D == 64)
    launch_t<64>(a, s1, qp0, nqp, st);
  else
    launch_t<128>(a, s1, qp0, nqp, st);
}

}  // namespace muse
