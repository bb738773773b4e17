// k-means assignment screen on the 5th-generation tensor cores (bf16 inputs).
//
// The clustering step of MuSe (gist.science page "Multipole Semantic
// Attention: A Fast Approximation of Softmax Attention for Pretraining",
// Technical Summary, Core Mechanisms, "Bidirectional Semantic Clustering")
// needs, for every token x of a 128-token tile, argmin_c ||x - c||^2 =
// argmin_c (||c||^2 - 2 x.c).  The tile's x.c products are one GEMM:
// A = the 128 x D token tile (bf16, exact), B = the centroids split into
// c_hi + c_lo bf16 parts (residual 2^-18 relative), D = 128 x N fp32 in
// tensor memory.  One elected thread issues tcgen05.mma (kind::f16, M = 128,
// N <= 256, K = 16 per instruction) over 128-byte-swizzled shared-memory
// operands and commits to an mbarrier; the four warps then read their 32 TMEM
// lanes (one token row per thread) with tcgen05.ld and keep the best and
// runner-up screen distances.  A token whose gap is inside the certified
// error bound of the screen is re-decided in fp64 (kmeans_tail.cuh), so the
// final assignment equals the plain fp64 argmin with ties to the lowest
// index.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "kmeans_tail.cuh"

namespace muse {

namespace {

constexpr int kNCMax = 256;  // centroids per MMA pass (TMEM fp32 columns)

__device__ inline uint32_t saddr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory matrix descriptor of a K-major operand stored as rows of 128
// bytes with the 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ inline uint64_t desc_sw128(uint32_t a) {
  return (uint64_t)((a >> 4) & 0x3FFF) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}

// byte offset of 16-byte chunk q of row r in a 128-byte-swizzled K-block
__device__ inline uint32_t sw128_chunk(int r, int q) { return r * 128 + (((q ^ (r & 7))) << 4); }

__device__ inline void mma_bf16_ss(uint32_t tmem, uint64_t ad, uint64_t bd, uint32_t idesc,
                                   uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem),
      "l"(ad), "l"(bd), "r"(idesc), "r"(acc));
}

__device__ inline void mma_commit(uint32_t mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(mbar)
               : "memory");
}

// Bounded wait on an mbarrier phase; false if it did not complete in time.
__device__ inline bool mbar_wait(uint32_t mbar, uint32_t parity) {
  for (int it = 0; it < (1 << 20); ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(mbar), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

__device__ inline void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int u = 0; u < 16; ++u) v[u] = __uint_as_float(r[u]);
}

__device__ inline void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ inline void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ inline void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

}  // namespace

size_t assign_tc_smem(int D, int NC) {
  const int KB = D / 64;
  return 1024 + (size_t)KB * kTile * 128 + 2 * (size_t)KB * NC * 128 + (size_t)NC * 4 +
         (size_t)kMaxC * 4;
}

template <int D>
__global__ void __launch_bounds__(kTile) kmeans_assign_tc_kernel(RoleGeo g, KState ks, int NC,
                                                                 int tcols) {
  constexpr int KB = D / 64;
  extern __shared__ __align__(1024) unsigned char tc_dyn[];
  unsigned char* base = tc_dyn + ((1024 - (saddr(tc_dyn) & 1023)) & 1023);
  unsigned char* A = base;
  unsigned char* BH = A + KB * kTile * 128;
  unsigned char* BL = BH + KB * NC * 128;
  float* cn2s = reinterpret_cast<float*>(BL + KB * NC * 128);
  int* hist = reinterpret_cast<int*>(cn2s + NC);
  __shared__ __align__(8) uint64_t mbar;
  __shared__ uint32_t tmem_slot;
  __shared__ int flagged[kTile];
  __shared__ int decision[kTile];
  __shared__ int nflag;
  __shared__ int is_last;
  __shared__ float cmax_s;

  int pid, tin;
  tile_of(g, blockIdx.x, &pid, &tin);
  const Prob p = prob_of(g, pid);
  const int C = p.C;
  const int t0 = tin * kTile;
  const int nt = imin(kTile, p.s - t0);
  const __nv_bfloat16* X = static_cast<const __nv_bfloat16*>(g.X);
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t mb = saddr(&mbar);

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     saddr(&tmem_slot)),
                 "r"(tcols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
  }
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(mb));
    asm volatile("fence.mbarrier_init.release.cluster;\n");
    nflag = 0;
    cmax_s = 0.f;
  }
  for (int i = tid; i < C; i += kTile) hist[i] = 0;
  // token tile, 16-byte chunks into the swizzled K-blocks; rows past the end are zero
  for (int e = tid; e < kTile * KB * 8; e += kTile) {
    const int r = e / (KB * 8), q = e - r * (KB * 8), kb = q >> 3, cq = q & 7;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < nt) v = *reinterpret_cast<const uint4*>(X + (p.row0 + t0 + r) * D + kb * 64 + cq * 8);
    *reinterpret_cast<uint4*>(A + kb * kTile * 128 + sw128_chunk(r, cq)) = v;
  }
  // largest centroid norm of the problem (for the error bound)
  {
    float m = 0.f;
    for (int c = tid; c < C; c += kTile) m = fmaxf(m, ks.cn2[(size_t)pid * g.C + c]);
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __syncthreads();
    if ((tid & 31) == 0) atomicMax(reinterpret_cast<int*>(&cmax_s), __float_as_int(m));
  }
  fence_async_smem();
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t taddr = tmem_slot;

  auto xrow = [&](int r, int d) -> float {
    const int kb = d >> 6, k = d & 63;
    const unsigned char* pz = A + kb * kTile * 128 + sw128_chunk(r, k >> 3) + ((k & 7) << 1);
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(pz));
  };
  float xn2 = 0.f;
  for (int d = 0; d < D; ++d) {
    const float v = xrow(tid, d);
    xn2 = fmaf(v, v, xn2);
  }
  const float xn = sqrtf(xn2) * 1.0001f;

  float b1 = INFINITY, b2 = INFINITY;
  int bi = 0;
  uint32_t phase = 0;
  bool ok = true;
  const __nv_bfloat16* ch = ks.cbf_hi + (size_t)pid * g.C * D;
  const __nv_bfloat16* cl = ks.cbf_lo + (size_t)pid * g.C * D;
  for (int c0 = 0; c0 < C; c0 += NC) {
    const int nc = imin(NC, C - c0);
    const int ncp = (nc + 15) & ~15;
    for (int e = tid; e < ncp * KB * 8; e += kTile) {
      const int r = e / (KB * 8), q = e - r * (KB * 8), kb = q >> 3, cq = q & 7;
      uint4 vh = make_uint4(0, 0, 0, 0), vl = vh;
      if (r < nc) {
        const size_t off = (size_t)(c0 + r) * D + kb * 64 + cq * 8;
        vh = *reinterpret_cast<const uint4*>(ch + off);
        vl = *reinterpret_cast<const uint4*>(cl + off);
      }
      *reinterpret_cast<uint4*>(BH + kb * NC * 128 + sw128_chunk(r, cq)) = vh;
      *reinterpret_cast<uint4*>(BL + kb * NC * 128 + sw128_chunk(r, cq)) = vl;
    }
    for (int c = tid; c < nc; c += kTile) cn2s[c] = ks.cn2[(size_t)pid * g.C + c0 + c];
    fence_async_smem();
    fence_before();
    __syncthreads();
    fence_after();
    if (tid == 0) {
      // D (f32) | A bf16 | B bf16 | K-major A and B | N | M = 128
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(ncp >> 3) << 17) |
                             ((uint32_t)(128 >> 4) << 24);
      for (int kb = 0; kb < KB; ++kb) {
        const uint64_t ad = desc_sw128(saddr(A + kb * kTile * 128));
        const uint64_t bh = desc_sw128(saddr(BH + kb * NC * 128));
        const uint64_t bl = desc_sw128(saddr(BL + kb * NC * 128));
#pragma unroll
        for (int k = 0; k < 4; ++k) {  // K = 16 bf16 = 32 bytes per instruction
          mma_bf16_ss(taddr, ad + 2 * k, bh + 2 * k, idesc, (kb | k) ? 1u : 0u);
          mma_bf16_ss(taddr, ad + 2 * k, bl + 2 * k, idesc, 1u);
        }
      }
      mma_commit(mb);
    }
    __syncwarp();
    const bool done = mbar_wait(mb, phase);
    if (!__syncthreads_and(done)) {
      ok = false;  // CTA-uniform: skip the TMEM reads, re-decide every token in fp64
      if (tid == 0) atomicOr(ks.err, kErrMmaWait);
    }
    phase ^= 1u;
    fence_after();
    if (ok) {
      for (int cc = 0; cc < ncp; cc += 16) {
        float acc[16];
        tmem_ld16(taddr + ((uint32_t)(warp * 32) << 16) + (uint32_t)cc, acc);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int c = cc + u;
          if (c < nc) {
            const float dd = fmaf(-2.f, acc[u], cn2s[c]);
            if (dd < b1) {
              b2 = b1;
              b1 = dd;
              bi = c0 + c;
            } else if (dd < b2) {
              b2 = dd;
            }
          }
        }
      }
    }
    fence_before();
    __syncthreads();
    fence_after();
  }
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(tcols));
  // |screen - exact| <= 2 eta |x| |c| + 2^-22 (|c|^2 + 2 |x| |c|), eta = 2^-14 (bf16 split
  // residual plus fp32 accumulation of 2D exact products, with margin)
  const float cm = sqrtf(cmax_s) * 1.0001f;
  const float E = 2.f * 6.1035156e-05f * xn * cm + 2.3841858e-07f * (cm * cm + 2.f * xn * cm);
  const bool flag = !ok || (b2 - b1) <= 2.f * E;
  assign_tail<D>(g, ks, p, pid, t0, nt, bi, flag, xrow, hist, flagged, decision, &nflag, &is_last);
}

template <int D>
static void launch(const RoleGeo& g, const KState& ks, cudaStream_t st) {
  const int NC = imin(kNCMax, (g.C + 15) & ~15);
  int tcols = 32;
  while (tcols < NC) tcols <<= 1;
  const size_t smem = assign_tc_smem(D, NC);
  // set on every launch: the attribute is per device, and the call is cheap
  cudaFuncSetAttribute(kmeans_assign_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)assign_tc_smem(D, kNCMax));
  kmeans_assign_tc_kernel<D><<<(unsigned)ks.ntiles, kTile, smem, st>>>(g, ks, NC, tcols);
}

void launch_assign_tc(const RoleGeo& g, const KState& ks, cudaStream_t st) {
  if (g.D == 64)
    launch<64>(g, ks, st);
  else
    launch<128>(g, ks, st);
}

}  // namespace muse
