// Stage 2 of MuSe on tensor cores for bf16 inputs: for the queries of one
// query cluster i, one online softmax over
//   - the far field: one row per non-retrieved non-empty key cluster j, key
//     row mu_j (or the tilted centroid k_hat_ij), logit offset fbias_ij and
//     value u_ij (gist.science page "Multipole Semantic Attention: A Fast
//     Approximation of Softmax Attention for Pretraining", Technical Summary,
//     Core Mechanisms: Stage 2 (Refinement));
//   - exact attention over every key of the retrieved clusters (same page,
//     Exact Attention).
// Each warp owns 16 query rows; S = Q K^T runs as bf16 m16n8k16 MMAs with fp32
// accumulation.  bf16 query and key rows are exact; a far-field key row (fp32)
// is split into hi + lo bf16 parts and contracted twice, leaving a residual of
// 2^-18 relative.  P and V enter the PV product as fp16 (V bf16 -> fp16 is
// exact in fp16's normal range; u_ij rounds to 11 bits), accumulating in fp32.
#include <cuda_fp16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace muse {

namespace {

constexpr int kMQ = 64;      // queries per pass (4 warps x 16 rows)
constexpr int kMK = 64;      // key rows per block
constexpr int kThreads = 128;

__device__ inline int kvp(const AttnArgs& a, int qpid) {
  const int ppb = a.qg.lv.pairs_per_bh;
  const int bhq = qpid / ppb, pi = qpid - bhq * ppb;
  const int Hq = a.qg.BH / a.B, Hkv = a.kg.BH / a.B;
  const int b = bhq / Hq, hq = bhq - b * Hq;
  return (b * Hkv + hq / a.G) * a.kg.lv.pairs_per_bh + pi;
}

__device__ inline uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ inline void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ inline void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
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

__device__ inline uint32_t pack_h2(float x, float y) {
  __half2 h = __floats2half2_rn(x, y);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int D>
struct Smem2 {
  __nv_bfloat16 q[kMQ][D + 8];
  __nv_bfloat16 k[kMK][D + 8];    // exact keys, or the hi part of far keys
  __nv_bfloat16 k2[kMK][D + 8];   // lo part of far keys
  __half v[kMK][D + 8];
  float bias[kMK];
  unsigned char inR[kMaxC];
  int sel[kMaxC];
};

}  // namespace

template <int D>
size_t stage2_mma_smem() {
  return sizeof(Smem2<D>);
}

template <typename TO, int D>
__global__ void __launch_bounds__(kThreads) stage2_mma_kernel(AttnArgs a, Stage1 s1, int qp0) {
  extern __shared__ __align__(16) unsigned char sm2_raw[];
  Smem2<D>& sm = *reinterpret_cast<Smem2<D>*>(sm2_raw);
  constexpr int KD = D / 16;   // k-steps over the head dimension
  constexpr int ND = D / 8;    // n-tiles over the head dimension
  const int lq = blockIdx.x, qpid = qp0 + lq, i = blockIdx.y;
  const Prob pq = prob_of(a.qg, qpid);
  if (i >= pq.C) return;
  const int Cq = a.Cq, Ck = a.Ck;
  const int nqi = a.qs.counts[(size_t)qpid * Cq + i];
  if (nqi == 0) return;
  const int kpid = kvp(a, qpid);
  const Prob pk = prob_of(a.kg, kpid);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int nsel = a.topk > 0 ? s1.nsel[(size_t)qpid * Cq + i] : 0;
  for (int j = tid; j < pk.C; j += kThreads) sm.inR[j] = 0;
  __syncthreads();
  for (int r = tid; r < nsel; r += kThreads) {
    const int j = s1.sel[((size_t)qpid * Cq + i) * a.topk + r];
    sm.sel[r] = j;
    sm.inR[j] = 1;
  }
  __syncthreads();
  const int* kc = a.ks.counts + (size_t)kpid * Ck;
  const int* koff = a.ks.off + (size_t)kpid * (Ck + 1);
  long long nexact = 0;
  for (int r = 0; r < nsel; ++r) nexact += kc[sm.sel[r]];

  const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(a.qg.X);
  const __nv_bfloat16* K = static_cast<const __nv_bfloat16*>(a.kg.X);
  const __nv_bfloat16* V = static_cast<const __nv_bfloat16*>(a.V);
  const int qo = a.qs.off[(size_t)qpid * (Cq + 1) + i];
  const int* qperm = a.qs.perm + pq.slot0;
  const int* kperm = a.ks.perm + pk.slot0;
  const size_t ij0 = ((size_t)lq * Cq + i) * Ck;
  const bool tilted = a.mode == 2;
  const float sl2 = a.scale * 1.4426950408889634f;  // logits in base-2 units

  for (int c0 = 0; c0 < nqi; c0 += kMQ) {
    const int nq = imin(kMQ, nqi - c0);
    __syncthreads();
    // gather the chunk's query rows (16-byte pieces), zero rows past the end
    for (int e = tid; e < kMQ * (D / 8); e += kThreads) {
      const int r = e / (D / 8), c = (e % (D / 8)) * 8;
      uint4 val = make_uint4(0, 0, 0, 0);
      if (r < nq) {
        const long long row = pq.row0 + qperm[qo + c0 + r];
        val = *reinterpret_cast<const uint4*>(Q + row * D + c);
      }
      *reinterpret_cast<uint4*>(&sm.q[r][c]) = val;
    }
    __syncthreads();
    uint32_t qa[KD][4];
#pragma unroll
    for (int kk = 0; kk < KD; ++kk) {
      const int row = warp * 16 + (lane & 15), col = kk * 16 + (lane >> 4) * 8;
      ldsm_x4(smem_u32(&sm.q[row][col]), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
    }
    float o[ND][4];
#pragma unroll
    for (int n = 0; n < ND; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};

    // one block of up to 64 staged key rows
    auto consume = [&](bool two_part) {
      float sc[kMK / 8][4];
#pragma unroll
      for (int n = 0; n < kMK / 8; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < KD; ++kk) {
#pragma unroll
        for (int np = 0; np < kMK / 16; ++np) {
          const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int col = kk * 16 + ((lane >> 3) & 1) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4(smem_u32(&sm.k[key][col]), b0, b1, b2, b3);
          mma_bf16(sc[2 * np], qa[kk], b0, b1);
          mma_bf16(sc[2 * np + 1], qa[kk], b2, b3);
          if (two_part) {
            ldsm_x4(smem_u32(&sm.k2[key][col]), b0, b1, b2, b3);
            mma_bf16(sc[2 * np], qa[kk], b0, b1);
            mma_bf16(sc[2 * np + 1], qa[kk], b2, b3);
          }
        }
      }
      // logits (base 2), row maxima over this block
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int n = 0; n < kMK / 8; ++n) {
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int col = n * 8 + 2 * t4 + (h & 1);
          const float lg = fmaf(sl2, sc[n][h], sm.bias[col]);
          sc[n][h] = lg;
          mx[h >> 1] = fmaxf(mx[h >> 1], lg);
        }
      }
      float scale[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
        const float mn = fmaxf(mrow[r], mx[r]);
        scale[r] = (mrow[r] == -INFINITY) ? 0.f : exp2f(mrow[r] - mn);
        mrow[r] = mn;
      }
      float rs[2] = {0.f, 0.f};
#pragma unroll
      for (int n = 0; n < kMK / 8; ++n) {
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float m = mrow[h >> 1];
          const float p = (m == -INFINITY) ? 0.f : exp2f(sc[n][h] - m);
          sc[n][h] = p;
          rs[h >> 1] += p;
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
      // O += P V  (P as fp16 A fragments straight from the S accumulators)
#pragma unroll
      for (int kk = 0; kk < kMK / 16; ++kk) {
        uint32_t pa[4];
        pa[0] = pack_h2(sc[2 * kk][0], sc[2 * kk][1]);
        pa[1] = pack_h2(sc[2 * kk][2], sc[2 * kk][3]);
        pa[2] = pack_h2(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
        pa[3] = pack_h2(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
#pragma unroll
        for (int np = 0; np < ND / 2; ++np) {
          const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int col = np * 16 + (lane >> 4) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_u32(&sm.v[key][col]), b0, b1, b2, b3);
          mma_f16(o[2 * np], pa, b0, b1);
          mma_f16(o[2 * np + 1], pa, b2, b3);
        }
      }
    };

    // far field
    for (int j0 = 0; j0 < pk.C; j0 += kMK) {
      __syncthreads();
      for (int e = tid; e < kMK * (D / 4); e += kThreads) {
        const int r = e / (D / 4), c = (e % (D / 4)) * 4, j = j0 + r;
        const bool live = j < pk.C && kc[j] > 0 && !sm.inR[j];
        float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), uv = kv;
        if (live) {
          const size_t ij = ij0 + j;
          kv = tilted ? *reinterpret_cast<const float4*>(s1.Kf + ij * D + c)
                      : *reinterpret_cast<const float4*>(a.ks.cent32 + ((size_t)kpid * Ck + j) * D + c);
          uv = *reinterpret_cast<const float4*>(s1.U + ij * D + c);
        }
        const float kx[4] = {kv.x, kv.y, kv.z, kv.w};
        const float ux[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const __nv_bfloat16 hi = __float2bfloat16_rn(kx[u]);
          sm.k[r][c + u] = hi;
          sm.k2[r][c + u] = __float2bfloat16_rn(kx[u] - __bfloat162float(hi));
          sm.v[r][c + u] = __float2half_rn(ux[u]);
        }
      }
      for (int r = tid; r < kMK; r += kThreads) {
        const int j = j0 + r;
        const bool live = j < pk.C && kc[j] > 0 && !sm.inR[j];
        sm.bias[r] = live ? s1.fbias[ij0 + j] * 1.4426950408889634f : -INFINITY;
      }
      __syncthreads();
      consume(true);
    }
    // exact retrieval
    for (int rr = 0; rr < nsel; ++rr) {
      const int j = sm.sel[rr], b = koff[j], n = kc[j];
      for (int t0 = 0; t0 < n; t0 += kMK) {
        const int nr = imin(kMK, n - t0);
        __syncthreads();
        for (int e = tid; e < kMK * (D / 8); e += kThreads) {
          const int r = e / (D / 8), c = (e % (D / 8)) * 8;
          uint4 kv = make_uint4(0, 0, 0, 0), vv = kv;
          if (r < nr) {
            const long long row = pk.row0 + kperm[b + t0 + r];
            kv = *reinterpret_cast<const uint4*>(K + row * D + c);
            vv = *reinterpret_cast<const uint4*>(V + row * D + c);
          }
          *reinterpret_cast<uint4*>(&sm.k[r][c]) = kv;
          const __nv_bfloat16* vb = reinterpret_cast<const __nv_bfloat16*>(&vv);
#pragma unroll
          for (int u = 0; u < 8; ++u) sm.v[r][c + u] = __float2half_rn(__bfloat162float(vb[u]));
        }
        for (int r = tid; r < kMK; r += kThreads) sm.bias[r] = r < nr ? 0.f : -INFINITY;
        __syncthreads();
        consume(false);
      }
    }
    // write the chunk's rows
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int qr = warp * 16 + g + 8 * r;
      if (qr >= nq) continue;
      const int tq = qperm[qo + c0 + qr];
      const long long row = pq.row0 + tq;
      const float inv = 1.f / lrow[r];
      if (a.O != nullptr) {
        TO* O = static_cast<TO*>(a.O);
#pragma unroll
        for (int n = 0; n < ND; ++n) {
          st<TO>(O + row * D + n * 8 + 2 * t4, o[n][2 * r] * inv);
          st<TO>(O + row * D + n * 8 + 2 * t4 + 1, o[n][2 * r + 1] * inv);
        }
      } else {
        float* pp = a.part + (size_t)(pq.slot0 + tq) * (D + 1);
#pragma unroll
        for (int n = 0; n < ND; ++n) {
          pp[n * 8 + 2 * t4] = o[n][2 * r] * inv;
          pp[n * 8 + 2 * t4 + 1] = o[n][2 * r + 1] * inv;
        }
        if (t4 == 0) pp[D] = (mrow[r] + log2f(lrow[r])) * 0.6931471805599453f;
      }
      if (a.n_exact != nullptr && t4 == 0) {
        if (a.O != nullptr)
          a.n_exact[row] = nexact;
        else
          atomicAdd(reinterpret_cast<unsigned long long*>(a.n_exact + row),
                    (unsigned long long)nexact);
      }
    }
  }
}

template <int D>
static void launch_t(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(stage2_mma_kernel<float, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)stage2_mma_smem<D>());
    cudaFuncSetAttribute(stage2_mma_kernel<__nv_bfloat16, D>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)stage2_mma_smem<D>());
    attr = true;
  }
  dim3 grid(nqp, a.Cq);
  if (a.out_f32)
    stage2_mma_kernel<float, D><<<grid, kThreads, stage2_mma_smem<D>(), st>>>(a, s1, qp0);
  else
    stage2_mma_kernel<__nv_bfloat16, D><<<grid, kThreads, stage2_mma_smem<D>(), st>>>(a, s1, qp0);
}

void run_stage2_mma(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st) {
  if (a.qg.D == 64)
    launch_t<64>(a, s1, qp0, nqp, st);
  else
    launch_t<128>(a, s1, qp0, nqp, st);
}

}  // namespace muse
