// Persistent Lloyd k-means for bf16 inputs: one thread-block cluster of NCT
// CTAs per problem runs every round in a single launch.
//
// The clustering step of MuSe (gist.science page "Multipole Semantic
// Attention: A Fast Approximation of Softmax Attention for Pretraining",
// Technical Summary, Core Mechanisms, "Bidirectional Semantic Clustering").
// Round structure inside the kernel:
//   1. every CTA screens its 128-token tiles against the centroids with
//      tcgen05.mma (bf16 hi/lo split of the centroids, fp32 TMEM accumulator),
//      keeps best/runner-up per token and re-decides uncertain tokens in fp64;
//   2. every CTA sorts its tokens by cluster (stable counting sort in shared
//      memory) and publishes its per-cluster counts and member lists;
//   3. cluster barrier; cluster c is owned by CTA rank c % NCT, which reads all
//      CTAs' counts and member lists through distributed shared memory and sums
//      the member rows in ascending token order in fp64 (the same order as a
//      plain sequential evaluation), then writes the new centroid (fp64, fp32,
//      bf16 hi/lo, norms) to global memory;
//   4. cluster barrier, next round.
// After the last round the owners also write the counts, segment offsets and
// the cluster-sorted permutation that the summaries and stage 2 read.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace muse {

namespace {

constexpr int kNCF = 256;  // centroids handled by the fused path (one MMA pass)

__device__ inline uint32_t saddr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ inline uint64_t desc_sw128(uint32_t a) {
  return (uint64_t)((a >> 4) & 0x3FFF) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}
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
// 16 columns without waiting; pair with tmem_wait() before using the values
__device__ inline void tmem_ld16_nw(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ inline void tmem_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
__device__ inline void cp16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(saddr(dst)), "l"(src),
               "r"(src_bytes));
}
__device__ inline void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ inline void cp_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }
__device__ inline void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ inline void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ inline void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

struct FusedLayout {
  int KB, NC, tpc;  // K-blocks, centroid columns (multiple of 32), tiles per CTA
  size_t a, bh, bl, cn2, acc, asg, list, lcnt, loff, total;
};

__host__ __device__ inline FusedLayout fused_layout(int D, int NC, int tpc) {
  FusedLayout L;
  L.KB = D / 64;
  L.NC = NC;
  L.tpc = tpc;
  size_t o = 0;
  L.a = o;    o += (size_t)3 * L.KB * kTile * 128;   // in use, under MMA, loading
  L.bh = o;   o += (size_t)L.KB * NC * 128;
  L.bl = o;   o += (size_t)L.KB * NC * 128;
  L.cn2 = o;  o += (size_t)NC * 4;
  o = (o + 15) & ~(size_t)15;
  L.acc = o;  o += (size_t)NC * D * 8;   // per-cluster fp64 partial sums of this CTA
  L.lcnt = o; o += (size_t)kNCF * 4;
  L.loff = o; o += (size_t)(kNCF + 1) * 4;
  L.asg = o;  o += (size_t)tpc * kTile * 2;
  L.list = o; o += (size_t)tpc * kTile * 2;
  L.total = o + 1024;
  return L;
}

}  // namespace

// Up to two independent problem sets (the key and the query clusterings)
// share one launch: CTAs [0, nblk0) serve set 0, the rest set 1.
struct FusedSets {
  RoleGeo g[2];
  KState ks[2];
  int nblk0;
};

// Exclusive scan of n <= 2 * blockDim.x ints in shared memory, called by
// every thread of the CTA; returns the total.  `tmp` holds one int per warp.
__device__ inline int block_scan_excl(int* a, int n, int* tmp) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  const int i0 = 2 * tid, i1 = 2 * tid + 1;
  const int v0 = i0 < n ? a[i0] : 0, v1 = i1 < n ? a[i1] : 0;
  int x = v0 + v1;
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  int wbase = 0, total = 0;
  for (int w = 0; w < nw; ++w) {
    if (w < warp) wbase += tmp[w];
    total += tmp[w];
  }
  const int excl = wbase + x - (v0 + v1);
  if (i0 < n) a[i0] = excl;
  if (i1 < n) a[i1] = excl + v0;
  __syncthreads();
  return total;
}

constexpr int kFT = 256;  // threads of the fused kernel (8 warps)

// acc[k][.] += x for the warp-uniform k (registers stay registers).
template <int KA, int R>
__device__ inline void acc_add(double (&acc)[KA > 0 ? KA : 1][R], int k, const double (&x)[R]) {
#define MUSE_ACC_CASE(K)                                                     \
  case K:                                                                    \
    if (K < (KA > 0 ? KA : 1)) {                                             \
      _Pragma("unroll") for (int q = 0; q < R; ++q)                          \
          acc[K < (KA > 0 ? KA : 1) ? K : 0][q] =                            \
              __dadd_rn(acc[K < (KA > 0 ? KA : 1) ? K : 0][q], x[q]);        \
    }                                                                        \
    break;
  switch (k) {
    MUSE_ACC_CASE(0) MUSE_ACC_CASE(1) MUSE_ACC_CASE(2) MUSE_ACC_CASE(3)
    MUSE_ACC_CASE(4) MUSE_ACC_CASE(5) MUSE_ACC_CASE(6) MUSE_ACC_CASE(7)
    MUSE_ACC_CASE(8) MUSE_ACC_CASE(9) MUSE_ACC_CASE(10) MUSE_ACC_CASE(11)
    MUSE_ACC_CASE(12) MUSE_ACC_CASE(13) MUSE_ACC_CASE(14) MUSE_ACC_CASE(15)
    default: break;
  }
#undef MUSE_ACC_CASE
}

// KA > 0: each warp keeps the fp64 sums of its clusters (c = w mod 8, at most
// 8 KA of them) in registers and the fp64 centroids are staged in shared
// memory for the re-decision; KA == 0: sums in shared memory, centroids read
// from L2.
template <int D, int KA>
__global__ void __launch_bounds__(kFT, 1) kmeans_fused_kernel(FusedSets fs, int iters, int NCT,
                                                             int NC, int tpc_max, int tcols) {
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(1024) unsigned char fz_dyn[];
  unsigned char* base = fz_dyn + ((1024 - (saddr(fz_dyn) & 1023)) & 1023);
  const FusedLayout Lo = fused_layout(D, NC, tpc_max);
  const int set = (int)blockIdx.x < fs.nblk0 ? 0 : 1;
  const RoleGeo& g = fs.g[set];
  const KState& ks = fs.ks[set];
  const int blk = (int)blockIdx.x - (set ? fs.nblk0 : 0);
  constexpr int KB = D / 64;
  constexpr int R = D / 32;
  constexpr int ATILE = KB * kTile * 128;  // bytes of one swizzled token tile
  unsigned char* A0 = base + Lo.a;
  unsigned char* BH = base + Lo.bh;
  unsigned char* BL = base + Lo.bl;
  float* cn2s = reinterpret_cast<float*>(base + Lo.cn2);
  double* sacc = reinterpret_cast<double*>(base + Lo.acc);  // KA > 0: staged centroids first
  int* lcnt = reinterpret_cast<int*>(base + Lo.lcnt);
  int* loff = reinterpret_cast<int*>(base + Lo.loff);
  unsigned short* asg = reinterpret_cast<unsigned short*>(base + Lo.asg);
  unsigned short* list = reinterpret_cast<unsigned short*>(base + Lo.list);
  __shared__ __align__(8) uint64_t mbar[2];
  __shared__ uint32_t tmem_slot;
  __shared__ float hb1[kTile], hb2[kTile];   // upper column half: best, runner-up
  __shared__ int hbi[kTile];
  __shared__ int tasg[kTile];                // assignment of the tile's tokens
  __shared__ int scan_tmp[32];
  __shared__ float cmax_s;
  __shared__ int gcnt[kNCF];
  __shared__ int goff[kNCF + 1];

  const int rank = (int)cluster.block_rank();
  const int pid = blk / NCT;
  const Prob p = prob_of(g, pid);
  const int C = p.C;
  const int ntp = cdiv(p.s, kTile);
  const int tpc = cdiv(ntp, NCT);
  const int tile0 = rank * tpc, tile1 = imin(ntp, tile0 + tpc);
  const int ntl = tile1 > tile0 ? tile1 - tile0 : 0;
  const int tok0 = tile0 * kTile, tok1 = imin(p.s, tile1 * kTile);
  const int ntok = tok1 > tok0 ? tok1 - tok0 : 0;
  const __nv_bfloat16* X = static_cast<const __nv_bfloat16*>(g.X);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = tid & (kTile - 1);      // TMEM lane / token row of this thread
  const int half = warp >> 2;             // column half of this thread's epilogue
  const size_t cbase = (size_t)pid * g.C;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     saddr(&tmem_slot)),
                 "r"(tcols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
  }
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(saddr(&mbar[0])));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(saddr(&mbar[1])));
    asm volatile("fence.mbarrier_init.release.cluster;\n");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tbase = tmem_slot;
  uint32_t phase[2] = {0u, 0u};
  const int ncp = (C + 31) & ~31;          // columns, a multiple of 32 (two halves of 16k)
  const int hw = ncp / 2;                  // columns per half
  const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(ncp >> 3) << 17) |
                         ((uint32_t)(128 >> 4) << 24);
  const double* c64g = ks.cent64 + cbase * D;

  auto xrow = [&](const unsigned char* A, int r, int d) -> float {
    const int kb = d >> 6, k = d & 63;
    const unsigned char* pz = A + kb * kTile * 128 + sw128_chunk(r, k >> 3) + ((k & 7) << 1);
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(pz));
  };
  auto load_tile = [&](int tl, unsigned char* A) {  // cp.async; caller commits
    const int t0 = tl * kTile, nt = imin(kTile, p.s - t0);
    for (int e = tid; e < kTile * KB * 8; e += kFT) {
      const int r = e / (KB * 8), q = e - r * (KB * 8), kb = q >> 3, cq = q & 7;
      const bool live = r < nt;
      cp16(A + kb * kTile * 128 + sw128_chunk(r, cq),
           X + (p.row0 + t0 + (live ? r : 0)) * D + kb * 64 + cq * 8, live ? 16 : 0);
    }
  };
  auto issue_mma = [&](const unsigned char* A, int buf) {
    const uint32_t tm = tbase + (uint32_t)(buf * ncp);
    for (int kb = 0; kb < KB; ++kb) {
      const uint64_t ad = desc_sw128(saddr(A + kb * kTile * 128));
      const uint64_t bh = desc_sw128(saddr(BH + kb * NC * 128));
      const uint64_t bl = desc_sw128(saddr(BL + kb * NC * 128));
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        mma_bf16_ss(tm, ad + 2 * k, bh + 2 * k, idesc, (kb | k) ? 1u : 0u);
        mma_bf16_ss(tm, ad + 2 * k, bl + 2 * k, idesc, 1u);
      }
    }
    mma_commit(saddr(&mbar[buf]));
  };
  auto tile_buf = [&](int k) { return A0 + (k % 3) * ATILE; };

  for (int it = 0; it < iters; ++it) {
    const bool last = it + 1 == iters;
    // ---- centroids of this round (bf16 split; KA > 0: fp64 copy too) ----------
    for (int e = tid; e < ncp * KB * 8; e += kFT) {
      const int r = e / (KB * 8), q = e - r * (KB * 8), kb = q >> 3, cq = q & 7;
      const bool live = r < C;
      const size_t off = (cbase + (live ? r : 0)) * D + kb * 64 + cq * 8;
      cp16(BH + kb * NC * 128 + sw128_chunk(r, cq), ks.cbf_hi + off, live ? 16 : 0);
      cp16(BL + kb * NC * 128 + sw128_chunk(r, cq), ks.cbf_lo + off, live ? 16 : 0);
    }
    if (KA > 0)
      for (int e = tid; e < C * D / 2; e += kFT) cp16(sacc + 2 * e, c64g + 2 * e, 16);
    if (KA == 0)
      for (int e = tid; e < C * D; e += kFT) sacc[e] = 0.0;
    for (int c = tid; c < C; c += kFT) lcnt[c] = 0;
    if (tid == 0) cmax_s = 0.f;
    if (ntl > 0) load_tile(tile0, tile_buf(0));
    cp_commit();
    if (ntl > 1) load_tile(tile0 + 1, tile_buf(1));
    cp_commit();
    {
      float m = 0.f;
      for (int c = tid; c < C; c += kFT) {
        const float v = __ldcg(ks.cn2 + cbase + c);
        cn2s[c] = v;
        m = fmaxf(m, v);
      }
      for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      __syncthreads();
      if (lane == 0) atomicMax(reinterpret_cast<int*>(&cmax_s), __float_as_int(m));
    }
    asm volatile("cp.async.wait_group 1;\n" ::: "memory");  // centroids and tile 0
    fence_async_smem();
    fence_before();
    __syncthreads();
    fence_after();
    const float cm = sqrtf(cmax_s) * 1.0001f;
    if (ntl > 0 && tid == 0) issue_mma(tile_buf(0), 0);
    double racc[KA > 0 ? KA : 1][R];
#pragma unroll
    for (int kk = 0; kk < (KA > 0 ? KA : 1); ++kk)
#pragma unroll
      for (int q = 0; q < R; ++q) racc[kk][q] = 0.0;

    for (int k = 0; k < ntl; ++k) {
      const int tl = tile0 + k, buf = k & 1;
      const int t0 = tl * kTile, nt = imin(kTile, p.s - t0);
      const unsigned char* A = tile_buf(k);
      // ---- tile k+1 goes to the tensor cores, tile k+2 starts loading ---------
      if (k + 1 < ntl) {
        cp_wait_all();
        fence_async_smem();
        fence_before();
        __syncthreads();
        fence_after();
        if (tid == 0) issue_mma(tile_buf(k + 1), buf ^ 1);
        if (k + 2 < ntl) load_tile(tl + 2, tile_buf(k + 2));
        cp_commit();
      }
      // token norm for the screen bound (own row, 16-byte loads)
      float xn = 0.f;
      if (tid < nt) {
        const uint4* xr = reinterpret_cast<const uint4*>(X + (p.row0 + t0 + tid) * D);
        float q2 = 0.f;
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          const uint4 v = xr[c];
          const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 f = __bfloat1622float2(b[u]);
            q2 = fmaf(f.x, f.x, fmaf(f.y, f.y, q2));
          }
        }
        xn = sqrtf(q2) * 1.0001f;
      }
      __syncwarp();
      const bool done = mbar_wait(saddr(&mbar[buf]), phase[buf]);
      phase[buf] ^= 1u;
      const bool ok = __syncthreads_and(done);
      if (!ok && tid == 0) atomicExch(ks.err, 1);
      fence_after();
      const uint32_t tm = tbase + (uint32_t)(buf * ncp) + ((uint32_t)((warp & 3) * 32) << 16);
      // ---- epilogue: each half of the warps scans half of the columns ---------
      // four independent best / runner-up trackers (columns c = 4m + u) keep
      // the compare chain short; merged by (value, index) so ties keep the
      // lowest index
      float b1 = INFINITY, b2 = INFINITY;
      int bi = 0;
      if (ok) {
        float t1[4], t2[4];
        int ti[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          t1[u] = INFINITY;
          t2[u] = INFINITY;
          ti[u] = 0;
        }
        for (int c0 = half * hw; c0 < (half + 1) * hw; c0 += 64) {
          uint32_t rv[4][16];
          const int nb = imin(4, ((half + 1) * hw - c0) / 16);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (u < nb) tmem_ld16_nw(tm + (uint32_t)(c0 + 16 * u), rv[u]);
          tmem_wait();
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (u >= nb) break;
#pragma unroll
            for (int v = 0; v < 16; ++v) {
              const int c = c0 + 16 * u + v;
              const int tk = v & 3;
              const float dd = c < C ? fmaf(-2.f, __uint_as_float(rv[u][v]), cn2s[c]) : INFINITY;
              if (dd < t1[tk]) {
                t2[tk] = t1[tk];
                t1[tk] = dd;
                ti[tk] = c;
              } else if (dd < t2[tk]) {
                t2[tk] = dd;
              }
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (t1[u] < b1 || (t1[u] == b1 && ti[u] < bi)) {
            b2 = fminf(b1, t2[u]);
            b1 = t1[u];
            bi = ti[u];
          } else {
            b2 = fminf(b2, t1[u]);
          }
        }
      }
      if (half == 1) {
        hb1[row] = b1;
        hb2[row] = b2;
        hbi[row] = bi;
      }
      __syncthreads();
      if (half == 0) {
        // merge the upper half (higher indices lose ties)
        const float u1 = hb1[row], u2 = hb2[row];
        if (u1 < b1) {
          b2 = fminf(b1, u2);
          b1 = u1;
          bi = hbi[row];
        } else {
          b2 = fminf(b2, u1);
        }
        // |screen - exact| <= 2 eta |x| |c| + 2^-22 (|c|^2 + 2 |x| |c|), eta = 2^-15:
        // bf16 split residual (2^-18) plus fp32 accumulation of 2D exact products
        const float E = 2.f * 3.0517578e-05f * xn * cm + 2.3841858e-07f * (cm * cm + 2.f * xn * cm);
        const bool flag = tid < nt && (!ok || (b2 - b1) <= 2.f * E);
        // exact re-decision: only clusters inside the certified band can win
        int bx = bi;
        if (__any_sync(0xffffffffu, flag)) {
          double best = 0.0;
          int bc = -1;
          const float lim = b1 + 2.f * E;
          for (int cc = 0; cc < ncp; cc += 16) {
            uint32_t rv[16];
            if (ok) {
              tmem_ld16_nw(tm + (uint32_t)cc, rv);
              tmem_wait();
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const int c = cc + u;
              const bool cand =
                  flag && c < C && (!ok || fmaf(-2.f, __uint_as_float(rv[u]), cn2s[c]) <= lim);
              if (cand) {
                const double* ccen = (KA > 0 ? (const double*)sacc : c64g) + (size_t)c * D;
                double sd = 0.0;
                for (int d0 = 0; d0 < D; d0 += 16) {
                  double cv[16];
#pragma unroll
                  for (int kk = 0; kk < 16; ++kk) cv[kk] = KA > 0 ? ccen[d0 + kk] : __ldcg(ccen + d0 + kk);
#pragma unroll
                  for (int kk = 0; kk < 16; ++kk) {
                    const double t = __dsub_rn((double)xrow(A, row, d0 + kk), cv[kk]);
                    sd = __dadd_rn(sd, __dmul_rn(t, t));
                  }
                }
                if (bc < 0 || sd < best) {
                  best = sd;
                  bc = c;
                }
              }
            }
          }
          if (flag) bx = bc;
        }
        const int a = tid < nt ? bx : -1;
        tasg[row] = a;
        if (a >= 0) {
          asg[t0 - tok0 + row] = (unsigned short)a;
          atomicAdd(&lcnt[a], 1);
          if (last) ks.assign[p.slot0 + t0 + row] = a;
        }
      }
      fence_before();
      __syncthreads();
      // ---- fp64 partial sums: warp w owns the clusters c = w (mod 8) and walks
      // their tokens in tile order (lanes over dimensions), so every sum sees
      // its members in ascending token order --------------------------------------
      for (int r0 = 0; r0 < nt; r0 += 32) {
        const int ra = r0 + lane < nt ? tasg[r0 + lane] : -1;
        unsigned mine = __ballot_sync(0xffffffffu, ra >= 0 && (ra & 7) == warp);
        while (mine) {
          const int bit = __ffs(mine) - 1;
          mine &= mine - 1;
          const int r = r0 + bit;
          const int a = __shfl_sync(0xffffffffu, ra, bit);
          double x[R];
#pragma unroll
          for (int q = 0; q < R; ++q) x[q] = (double)xrow(A, r, lane + 32 * q);
          if (KA > 0) {
            acc_add<KA, R>(racc, a >> 3, x);
          } else {
            double* sp = sacc + (size_t)a * D;
#pragma unroll
            for (int q = 0; q < R; ++q) sp[lane + 32 * q] = __dadd_rn(sp[lane + 32 * q], x[q]);
          }
        }
      }
      __syncthreads();
    }
    if (KA > 0) {
      // the staged centroids are no longer read: publish the sums there
#pragma unroll
      for (int kk = 0; kk < (KA > 0 ? KA : 1); ++kk) {
        const int c = kk * 8 + warp;
        if (c < C)
#pragma unroll
          for (int q = 0; q < R; ++q) sacc[(size_t)c * D + lane + 32 * q] = racc[kk][q];
      }
    }
    // ---- last round: this CTA's tokens grouped by cluster (stable) ----------
    if (last) {
      for (int c = tid; c < C; c += kFT) loff[c] = lcnt[c];
      __syncthreads();
      block_scan_excl(loff, C, scan_tmp);
      if (warp == 0) {
        for (int b0 = 0; b0 < ntok; b0 += 32) {
          const int t = b0 + lane;
          const int aa = t < ntok ? (int)asg[t] : -1 - lane;
          const unsigned same = __match_any_sync(0xffffffffu, aa);
          const int rnk = __popc(same & ((1u << lane) - 1u));
          int pos = 0;
          if (t < ntok) pos = loff[aa] + rnk;
          __syncwarp();
          if (t < ntok) list[pos] = (unsigned short)t;
          if (t < ntok && rnk == 0) loff[aa] += __popc(same);
          __syncwarp();
        }
      }
      __syncthreads();
      for (int c = tid; c < C; c += kFT) loff[c] -= lcnt[c];  // back to segment starts
    }
    __threadfence();
    cluster.sync();
    // ---- owners: counts, offsets, means from the CTAs' partial sums ----------
    for (int c = tid; c < C; c += kFT) {
      int tot = 0;
      for (int r = 0; r < NCT; ++r) tot += *cluster.map_shared_rank(lcnt + c, r);
      gcnt[c] = tot;
    }
    __syncthreads();
    if (last) {
      for (int c = tid; c < C; c += kFT) goff[c] = gcnt[c];
      __syncthreads();
      const int tot = block_scan_excl(goff, C, scan_tmp);
      if (tid == 0) goff[C] = tot;
      __syncthreads();
    }
    for (int c = rank + NCT * warp; c < C; c += NCT * (kFT / 32)) {
      const int n = gcnt[c];
      if (last && lane == 0) {
        ks.counts[cbase + c] = n;
        ks.off[(size_t)pid * (g.C + 1) + c] = goff[c];
        if (c == C - 1) ks.off[(size_t)pid * (g.C + 1) + C] = goff[C];
      }
      if (n == 0) continue;  // an empty cluster keeps its centroid
      double sm[R];
#pragma unroll
      for (int q = 0; q < R; ++q) sm[q] = 0.0;
      for (int rr = 0; rr < NCT; ++rr) {
        const double* ra = cluster.map_shared_rank(sacc, rr) + (size_t)c * D;
#pragma unroll
        for (int q = 0; q < R; ++q) sm[q] = __dadd_rn(sm[q], ra[lane + 32 * q]);
      }
      if (last) {
        int pos = goff[c];
        for (int rr = 0; rr < NCT; ++rr) {
          const int m0 = *cluster.map_shared_rank(loff + c, rr);
          const int mc = *cluster.map_shared_rank(lcnt + c, rr);
          const unsigned short* rl = cluster.map_shared_rank(list, rr);
          const int rtok0 = rr * tpc * kTile;
          for (int m = lane; m < mc; m += 32) ks.perm[p.slot0 + pos + m] = rtok0 + rl[m0 + m];
          pos += mc;
        }
      }
      const double nn = (double)n;
      double q2 = 0.0;
      float qf = 0.f;
#pragma unroll
      for (int q = 0; q < R; ++q) {
        const double v = __ddiv_rn(sm[q], nn);
        const float v32 = (float)v;
        const size_t i = (cbase + c) * D + lane + 32 * q;
        ks.cent64[i] = v;
        ks.cent32[i] = v32;
        const __nv_bfloat16 hi = __float2bfloat16_rn(v32);
        ks.cbf_hi[i] = hi;
        ks.cbf_lo[i] = __float2bfloat16_rn(v32 - __bfloat162float(hi));
        q2 += v * v;
        qf = fmaf(v32, v32, qf);
      }
      for (int o = 16; o; o >>= 1) {
        qf += __shfl_xor_sync(0xffffffffu, qf, o);
        q2 += __shfl_xor_sync(0xffffffffu, q2, o);
      }
      if (lane == 0) {
        ks.cnorm[cbase + c] = sqrtf(qf) * 1.0001f;
        ks.cn2[cbase + c] = (float)q2;
      }
    }
    __threadfence();
    cluster.sync();
  }
  fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tbase), "r"(tcols));
}

// Returns false (nothing launched) when the fused path does not cover these
// problem sets: more than 256 clusters, or more than 65535 tokens per CTA.
template <int D, int KA>
static bool launch_fused_t(const RoleGeo* gs, const KState* kss, int nsets, int iters,
                           cudaStream_t st) {
  int cmax = 0;
  for (int k = 0; k < nsets; ++k) {
    if (gs[k].dtype != 0 || gs[k].C > kNCF || gs[k].D != D) return false;
    cmax = cmax > gs[k].C ? cmax : gs[k].C;
  }
  const int NC = (cmax + 31) & ~31;
  int tcols = 32;
  while (tcols < 2 * NC) tcols <<= 1;  // two accumulators (tiles in flight)
  const int nprob = kss[0].nprob + (nsets > 1 ? kss[1].nprob : 0);
  // largest cluster size (up to 16, beyond the portable 8 where the GPU
  // allows it) whose clusters are all resident at once
  int NCT = 0;
  FusedLayout L{};
  const bool big_ok =
      cudaFuncSetAttribute(kmeans_fused_kernel<D, KA>,
                           cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
  if (!big_ok) cudaGetLastError();
  for (int nct = big_ok ? 16 : 8; nct >= 1; --nct) {
    int tpc_max = 1;
    for (int k = 0; k < nsets; ++k)
      for (int l = 0; l < gs[k].lv.nlev; ++l) {
        const int tpc = cdiv(cdiv(gs[k].lv.s[l], kTile), nct);
        tpc_max = tpc_max > tpc ? tpc_max : tpc;
      }
    if (tpc_max * kTile > 65535) break;
    const FusedLayout Lc = fused_layout(D, NC, tpc_max);
    if (Lc.total > 218 * 1024) continue;  // leaves room for the static shared arrays
    cudaFuncSetAttribute(kmeans_fused_kernel<D, KA>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)Lc.total);
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3((unsigned)(nprob * nct));
    q.blockDim = dim3(kFT);
    q.dynamicSmemBytes = Lc.total;
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = nct;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    q.attrs = qa;
    q.numAttrs = 1;
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, kmeans_fused_kernel<D, KA>, &q) != cudaSuccess) {
      cudaGetLastError();
      active = 0;
    }
    if (nct <= 8 && NCT == 0) {  // fallback: the largest portable size that fits at all
      NCT = nct;
      L = Lc;
    }
    if (active >= nprob) {
      NCT = nct;
      L = Lc;
      break;
    }
  }
  if (NCT == 0) return false;
  FusedSets fs{};
  for (int k = 0; k < nsets; ++k) {
    fs.g[k] = gs[k];
    fs.ks[k] = kss[k];
  }
  fs.nblk0 = kss[0].nprob * NCT;
  const int nblk = fs.nblk0 + (nsets > 1 ? kss[1].nprob * NCT : 0);
  cudaFuncSetAttribute(kmeans_fused_kernel<D, KA>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)L.total);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)nblk);
  cfg.blockDim = dim3(kFT);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = NCT;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kmeans_fused_kernel<D, KA>, fs, iters, NCT, NC, L.tpc, tcols);
  return true;
}

bool launch_kmeans_fused(const RoleGeo* gs, const KState* kss, int nsets, int iters,
                         cudaStream_t st) {
  int cmax = 0;
  for (int k = 0; k < nsets; ++k) cmax = cmax > gs[k].C ? cmax : gs[k].C;
  // register sums when a warp's clusters (C / 8) x its dimensions (D / 32) fit in 32 doubles
  if (gs[0].D == 64)
    return cmax <= 128 ? launch_fused_t<64, 16>(gs, kss, nsets, iters, st)
                       : launch_fused_t<64, 0>(gs, kss, nsets, iters, st);
  return cmax <= 64 ? launch_fused_t<128, 8>(gs, kss, nsets, iters, st)
                    : launch_fused_t<128, 0>(gs, kss, nsets, iters, st);
}

}  // namespace muse
