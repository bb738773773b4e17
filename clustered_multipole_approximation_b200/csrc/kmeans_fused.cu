// Persistent Lloyd k-means for bf16 inputs: NCT CTAs per problem run every
// round in a single launch -- a cooperative launch when all problems fit on
// the GPU at once with more CTAs each than a thread-block cluster allows,
// else one thread-block cluster per problem.
//
// The clustering step of MuSe (gist.science page "Multipole Semantic
// Attention: A Fast Approximation of Softmax Attention for Pretraining",
// Technical Summary, Core Mechanisms, "Bidirectional Semantic Clustering").
// Round structure inside the kernel:
//   1. every CTA streams its 128-token tiles through shared memory (a cp.async
//      ring of three) and screens them against the centroids with
//      tcgen05.mma (bf16 hi/lo split of the centroids, fp32 TMEM accumulator;
//      two accumulators, so the tensor cores run one tile ahead of the
//      epilogue).  The epilogue keeps the best and runner-up screened distance
//      of every token; a token whose gap lies inside the certified error of
//      the screen goes to a queue;
//   2. the CTA's warps drain the queue: a queued token gets the exact fp64
//      argmin over all clusters, each distance summed in dimension order with
//      no fused operations (a plain sequential fp64 evaluation, bit for bit);
//   3. the CTA groups its tokens by cluster (stable counting sort) and
//      publishes the grouped list and its per-cluster offsets in global memory;
//   4. barrier; cluster c is owned by CTA rank c % NCT, where one warp
//      (clusters taken largest first) walks the members of c over all CTAs in
//      ascending token order and sums their rows in fp64 -- the order of a
//      plain sequential evaluation -- lanes over dimensions, with the next
//      batch of rows in flight, then writes the new centroid (fp64, fp32,
//      bf16 hi/lo, norms) to global memory;
//   5. barrier, next round.
// After the last round every CTA writes its tokens' assignments and the
// owners write the counts, segment offsets and the cluster-sorted permutation
// that the summaries and stage 2 read.
#include <cooperative_groups.h>
#include <stdio.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace muse {

namespace {

constexpr int kNCF = 256;          // centroids handled by the fused path (one MMA pass)
constexpr int kFT = 256;           // threads of the fused kernel
constexpr int kWarps = kFT / 32;
constexpr int kMaxNCT = 32;        // CTAs per problem
constexpr int kSpinLimit = 1 << 24;  // team barrier polls (64 ns apart) before giving up

// Failure-path testing: a CTA rank that skips its first barrier arrival and
// the poll bound of the barrier waits (muse_debug_inject_barrier_fault).
int g_fault_rank = -1;
int g_spin_limit = kSpinLimit;
// Testing: route every problem through the sequential-order kernel.
int g_no_resident = 0;
constexpr int kOT = kNCF + kMaxNCT;  // (owned cluster, rank) pairs per CTA, at most
constexpr int kTilesPerCta = 16;     // cluster launches: target tiles per CTA
constexpr int kFCandCap = 128;       // queued tokens per round with a candidate list
constexpr int kFMaxCand = 8;         // candidates kept per queued token
constexpr size_t kSmemLimit = 218 * 1024;  // dynamic shared memory (static arrays come on top)

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

// flags: bit 0 stages the fp64 centroids for the exact re-decisions; bit 1
// keeps two token tiles in shared memory instead of three (large C and D).
struct FusedLayout {
  int KB, NC, tpc, flags;  // K-blocks, centroid columns (multiple of 32), tiles per CTA
  size_t a, bh, bl, cn2, xs, whist, loff, gtab, xn, asg, queue, cand, ccnt, cst, total;
};

__host__ __device__ inline FusedLayout fused_layout(int D, int NC, int tpc, int flags) {
  FusedLayout L;
  L.KB = D / 64;
  L.NC = NC;
  L.tpc = tpc;
  L.flags = flags;
  const int ring = (flags & 2) ? 2 : 3;
  size_t o = 0;
  L.a = o;     o += (size_t)ring * L.KB * kTile * 128;  // in use, under MMA, loading
  // the queued rows and the per-warp counts are used only after a round's
  // tiles are done: they share the tile slots
  L.xs = L.a;                                          // queued token rows in fp64
  L.whist = L.a + (size_t)kWarps * D * 8;              // per-warp counts, then bases
  L.bh = o;    o += (size_t)L.KB * NC * 128;
  L.bl = o;    o += (size_t)L.KB * NC * 128;
  L.cn2 = o;   o += (size_t)NC * 4;
  o = (o + 15) & ~(size_t)15;
  L.loff = o;  o += (size_t)(NC + 1) * 4;
  L.gtab = o;  o += (size_t)kWarps * (2 * kMaxNCT + 1) * 4;   // owner warps' rank tables
  L.xn = o;    o += (size_t)tpc * kTile * 4;          // token norms (screen bound)
  L.asg = o;   o += (size_t)tpc * kTile * 2;
  L.queue = o; o += (size_t)tpc * kTile * 2;
  L.cand = o;  o += (size_t)kFCandCap * kFMaxCand * 2;  // candidate clusters of queued tokens
  o = (o + 15) & ~(size_t)15;
  L.ccnt = o;  o += (size_t)kFCandCap * 4;              // their counts (> kFMaxCand: every cluster)
  o = (o + 15) & ~(size_t)15;
  L.cst = o;                                          // fp64 centroids, row stride D + 1
  if (flags & 1) o += (size_t)NC * (D + 1) * 8;
  L.total = o + 1024;
  return L;
}

// A lane's share of one bf16 row in the owner sums: D / 32 consecutive values.
template <int D>
struct LaneRow;
template <>
struct LaneRow<64> {
  using T = uint32_t;
};
template <>
struct LaneRow<128> {
  using T = uint2;
};
__device__ inline void add_row(double (&acc)[2], uint32_t w) {
  const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
  acc[0] = __dadd_rn(acc[0], (double)f.x);
  acc[1] = __dadd_rn(acc[1], (double)f.y);
}
__device__ inline void add_row(double (&acc)[4], uint2 w) {
  const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
  const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
  acc[0] = __dadd_rn(acc[0], (double)f0.x);
  acc[1] = __dadd_rn(acc[1], (double)f0.y);
  acc[2] = __dadd_rn(acc[2], (double)f1.x);
  acc[3] = __dadd_rn(acc[3], (double)f1.y);
}

// Exact fp64 argmin over the C centroids for one token (x in fp64, shared
// memory, broadcast), lanes over clusters; ties go to the lowest index.
template <int D, bool STAGED>
__device__ inline int exact_argmin(const double* x, const double* cst, const double* c64, int C,
                                   int lane) {
  constexpr int MM = kNCF / 32;
  double sd[MM];
#pragma unroll
  for (int m = 0; m < MM; ++m) sd[m] = 0.0;
  for (int d = 0; d < D; ++d) {
    const double xd = x[d];
#pragma unroll
    for (int m = 0; m < MM; ++m) {
      const int c = lane + 32 * m;
      if (c < C) {
        const double cv = STAGED ? cst[c * (D + 1) + d] : __ldcg(c64 + (size_t)c * D + d);
        const double t = __dsub_rn(xd, cv);
        sd[m] = __dadd_rn(sd[m], __dmul_rn(t, t));
      }
    }
  }
  double bd = 0.0;
  int bc = -1;
#pragma unroll
  for (int m = 0; m < MM; ++m) {
    const int c = lane + 32 * m;
    if (c < C && (bc < 0 || sd[m] < bd)) {
      bd = sd[m];
      bc = c;
    }
  }
  for (int o = 16; o; o >>= 1) {
    const double od = __shfl_xor_sync(0xffffffffu, bd, o);
    const int oc = __shfl_xor_sync(0xffffffffu, bc, o);
    if (oc >= 0 && (bc < 0 || od < bd || (od == bd && oc < bc))) {
      bd = od;
      bc = oc;
    }
  }
  return bc;
}

}  // namespace

// Up to two independent problem sets (the key and the query clusterings)
// share one launch: CTAs [0, nblk0) serve set 0, the rest set 1.  lvl >= 0
// restricts a launch to the problems of one causal level (all (b, head) pairs
// of that level), so each level gets its own CTAs per problem.
struct FusedSets {
  RoleGeo g[2];
  KState ks[2];
  int nblk0;
  int lvl;
  int fault_rank;  // cooperative launches: this CTA rank skips its first arrival
  int spin_limit;  // polls of a barrier wait before it gives up
  int skip_certified;  // leave problems with certified-exact sums (the resident kernel's)
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

// COOP: a cooperative launch of NCT CTAs per problem (all resident at once;
// a problem's CTAs meet at a barrier on a workspace counter); otherwise one
// thread-block cluster of NCT CTAs per problem (hardware cluster barrier).
template <int D, bool COOP>
__global__ void __launch_bounds__(kFT, 1) kmeans_fused_kernel(FusedSets fs, int iters, int NCT,
                                                             int NC, int tpc_max, int tcols,
                                                             int stage) {
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(1024) unsigned char fz_dyn[];
  unsigned char* base = fz_dyn + ((1024 - (saddr(fz_dyn) & 1023)) & 1023);
  const FusedLayout Lo = fused_layout(D, NC, tpc_max, stage);
  const int ring = (stage & 2) ? 2 : 3;  // token tile slots
  const int set = (int)blockIdx.x < fs.nblk0 ? 0 : 1;
  const RoleGeo& g = fs.g[set];
  const KState& ks = fs.ks[set];
  const int blk = (int)blockIdx.x - (set ? fs.nblk0 : 0);
  constexpr int KB = D / 64;
  constexpr int VPL = D / 32;                // owner sums: dimensions per lane
  constexpr int kOB = D == 64 ? 32 : 16;     // owner sums: member rows per batch
  using RowT = typename LaneRow<D>::T;
  constexpr int ATILE = KB * kTile * 128;    // bytes of one swizzled token tile
  unsigned char* A0 = base + Lo.a;
  unsigned char* BH = base + Lo.bh;
  unsigned char* BL = base + Lo.bl;
  float* cn2s = reinterpret_cast<float*>(base + Lo.cn2);
  double* xs = reinterpret_cast<double*>(base + Lo.xs);
  int* whist = reinterpret_cast<int*>(base + Lo.whist);
  int* loff = reinterpret_cast<int*>(base + Lo.loff);
  int* gtab = reinterpret_cast<int*>(base + Lo.gtab);
  float* xns = reinterpret_cast<float*>(base + Lo.xn);
  unsigned short* asg = reinterpret_cast<unsigned short*>(base + Lo.asg);
  unsigned short* queue = reinterpret_cast<unsigned short*>(base + Lo.queue);
  unsigned short* cand = reinterpret_cast<unsigned short*>(base + Lo.cand);
  int* ccnt = reinterpret_cast<int*>(base + Lo.ccnt);
  double* cst = reinterpret_cast<double*>(base + Lo.cst);
  __shared__ __align__(8) uint64_t mbar[2];
  __shared__ uint32_t tmem_slot;
  __shared__ float hb1[kTile], hb2[kTile];   // upper column half: best, runner-up
  __shared__ int hbi[kTile];
  __shared__ int scan_tmp[32];
  __shared__ float cmax_s;
  __shared__ int qcount;
  __shared__ int goff[kNCF + 1];
  __shared__ int own_n[kNCF], own_ord[kNCF];  // owned clusters: sizes, largest-first order
  __shared__ int otab[2 * kOT];               // owned clusters x ranks: list start, count
  __shared__ int own_ctr;
  __shared__ int bar_fail;

  const int rank = COOP ? (int)blockIdx.x % NCT : (int)cluster.block_rank();
  int pid = blk / NCT;
  if (fs.lvl >= 0) {  // j-th problem of the level -> problem id
    const int np = g.lv.npairs[fs.lvl];
    pid = (pid / np) * g.lv.pairs_per_bh + g.lv.pair_base[fs.lvl] + pid % np;
  }
  const Prob p = prob_of(g, pid);
  // every CTA of the problem takes the same decision
  if (fs.skip_certified && sums_exact(ks, pid, p.s)) return;
  const int C = p.C;
  const int ntp = cdiv(p.s, kTile);
  const int tpc = cdiv(ntp, NCT);
  const int nra = cdiv(ntp, tpc);          // ranks that hold tokens
  const int tile0 = rank * tpc, tile1 = imin(ntp, tile0 + tpc);
  const int ntl = tile1 > tile0 ? tile1 - tile0 : 0;
  const int tok0 = tile0 * kTile, tok1 = imin(p.s, tile1 * kTile);
  const int ntok = tok1 > tok0 ? tok1 - tok0 : 0;
  const __nv_bfloat16* X = static_cast<const __nv_bfloat16*>(g.X);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = tid & (kTile - 1);      // TMEM lane / token row of this thread
  const int half = warp >> 2;             // column half of this thread's epilogue
  const size_t cbase = (size_t)pid * g.C;
  int* xoff = ks.hist + (size_t)p.tile0 * (g.C + 1);  // row r: rank r's list offsets
  // team barrier (COOP): arrival counter of this problem, monotonic over the launch
  int* bar_ctr = ks.arrive + pid;
  int nbar = 0;
  // A wait that gives up (a CTA of the problem never arrived) records
  // kErrTeamBarrier and sets bar_fail; the caller then leaves the round loop
  // at once, so no CTA reads lists or centroids that were never published.
  auto team_sync = [&]() {
    if (COOP) {
      __syncthreads();
      if (tid == 0) {
        ++nbar;
        __threadfence();
        if (!(nbar == 1 && rank == fs.fault_rank)) atomicAdd(bar_ctr, 1);
        for (int it = 0;; ++it) {
          int v;
          asm volatile("ld.acquire.gpu.global.s32 %0, [%1];\n" : "=r"(v) : "l"(bar_ctr) : "memory");
          if (v >= nbar * NCT) break;
          if (it >= fs.spin_limit) {
            bar_fail = 1;
            atomicOr(ks.err, kErrTeamBarrier);
            break;
          }
          __nanosleep(64);
        }
        __threadfence();
      }
      __syncthreads();
    } else {
      __threadfence();
      cluster.sync();
    }
  };
  unsigned short* tl = ks.tlist + p.slot0;           // rank r's list at r * tpc * kTile

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     saddr(&tmem_slot)),
                 "r"(tcols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
  }
  if (tid == 0) {
    bar_fail = 0;
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

  auto load_tile = [&](int tl_, unsigned char* A) {  // cp.async; caller commits
    const int t0 = tl_ * kTile, nt = imin(kTile, p.s - t0);
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
  auto tile_buf = [&](int k) { return A0 + (k % ring) * ATILE; };
  // new centroid c = acc / n (lane l: dimensions l VPL ..): fp64, fp32, bf16
  // hi / lo split and norms
  auto write_centroid = [&](int c, int n, const double (&acc)[VPL]) {
    const double nn = (double)n;
    double q2 = 0.0;
    float qf = 0.f;
    double v64[VPL];
    float v32[VPL];
    uint32_t wh[VPL / 2], wl[VPL / 2];
#pragma unroll
    for (int e = 0; e < VPL; ++e) {
      v64[e] = __ddiv_rn(acc[e], nn);
      v32[e] = (float)v64[e];
      q2 += v64[e] * v64[e];
      qf = fmaf(v32[e], v32[e], qf);
    }
#pragma unroll
    for (int e = 0; e < VPL / 2; ++e) {
      const __nv_bfloat16 h0 = __float2bfloat16_rn(v32[2 * e]);
      const __nv_bfloat16 h1 = __float2bfloat16_rn(v32[2 * e + 1]);
      const __nv_bfloat16 l0 = __float2bfloat16_rn(v32[2 * e] - __bfloat162float(h0));
      const __nv_bfloat16 l1 = __float2bfloat16_rn(v32[2 * e + 1] - __bfloat162float(h1));
      wh[e] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
      wl[e] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
    }
    const size_t i0 = (cbase + c) * D + (size_t)lane * VPL;
#pragma unroll
    for (int e = 0; e < VPL / 2; ++e) {
      reinterpret_cast<double2*>(ks.cent64 + i0)[e] = make_double2(v64[2 * e], v64[2 * e + 1]);
      reinterpret_cast<float2*>(ks.cent32 + i0)[e] = make_float2(v32[2 * e], v32[2 * e + 1]);
      reinterpret_cast<uint32_t*>(ks.cbf_hi + i0)[e] = wh[e];
      reinterpret_cast<uint32_t*>(ks.cbf_lo + i0)[e] = wl[e];
    }
    for (int o = 16; o; o >>= 1) {
      qf += __shfl_xor_sync(0xffffffffu, qf, o);
      q2 += __shfl_xor_sync(0xffffffffu, q2, o);
    }
    if (lane == 0) {
      ks.cnorm[cbase + c] = sqrtf(qf) * 1.0001f;
      ks.cn2[cbase + c] = (float)q2;
    }
  };
  // Problems whose sums are certified exact in any order keep a running
  // state after the first round (sum64 = exact member sums, counts, dirty =
  // last round that changed the members, chg = tokens that moved): later
  // rounds move only the changed tokens' rows, and a round without moves
  // ends the problem (every later round would repeat it exactly).
  const bool cert = ks.sum64 != nullptr && sums_exact(ks, pid, p.s);
  double* sumg = cert ? ks.sum64 + cbase * D : nullptr;
  int* cntg = ks.counts + cbase;
  int* dirt = cert ? ks.dirty + cbase : nullptr;
  int* chgp = cert ? ks.chg + (size_t)pid * 2 : nullptr;
  __shared__ int nmv_s;

  for (int it = 0; it < iters; ++it) {
    const bool last = it + 1 == iters;
    bool fin = last;  // the problem's final round
    // ---- centroids of this round (bf16 split, tensor-core operand) ----------
    for (int e = tid; e < ncp * KB * 8; e += kFT) {
      const int r = e / (KB * 8), q = e - r * (KB * 8), kb = q >> 3, cq = q & 7;
      const bool live = r < C;
      const size_t off = (cbase + (live ? r : 0)) * D + kb * 64 + cq * 8;
      cp16(BH + kb * NC * 128 + sw128_chunk(r, cq), ks.cbf_hi + off, live ? 16 : 0);
      cp16(BL + kb * NC * 128 + sw128_chunk(r, cq), ks.cbf_lo + off, live ? 16 : 0);
    }
    if (tid == 0) {
      cmax_s = 0.f;
      qcount = 0;
    }
    if (ntl > 0) load_tile(tile0, tile_buf(0));
    cp_commit();
    if (ntl > 1) load_tile(tile0 + 1, tile_buf(1));
    cp_commit();
    {
      // padding columns get +inf so they never win
      float m = 0.f;
      for (int c = tid; c < ncp; c += kFT) {
        const float v = c < C ? __ldcg(ks.cn2 + cbase + c) : INFINITY;
        cn2s[c] = v;
        if (c < C) m = fmaxf(m, v);
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

    for (int k = 0; k < ntl; ++k) {
      const int tl_ = tile0 + k, buf = k & 1;
      const int t0 = tl_ * kTile, nt = imin(kTile, p.s - t0);
      const int u = t0 - tok0 + row;         // CTA-local token index of this row
      const unsigned char* A = tile_buf(k);
      // ---- tile k+1 goes to the tensor cores, tile k+2 starts loading ---------
      if (k + 1 < ntl) {
        cp_wait_all();
        fence_async_smem();
        fence_before();
        __syncthreads();
        fence_after();
        if (tid == 0) issue_mma(tile_buf(k + 1), buf ^ 1);
        if (ring == 3 && k + 2 < ntl) load_tile(tl_ + 2, tile_buf(k + 2));
        cp_commit();
      }
      // token norms for the screen bound, from the staged tile, first round only
      if (it == 0 && half == 0 && row < nt) {
        float q2 = 0.f;
#pragma unroll
        for (int kb = 0; kb < KB; ++kb)
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint4 v = *reinterpret_cast<const uint4*>(A + kb * kTile * 128 + sw128_chunk(row, q));
            const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(b[e]);
              q2 = fmaf(f.x, f.x, fmaf(f.y, f.y, q2));
            }
          }
        xns[u] = sqrtf(q2) * 1.0001f;
      }
      const bool done = mbar_wait(saddr(&mbar[buf]), phase[buf]);
      phase[buf] ^= 1u;
      const bool ok = __syncthreads_and(done);
      if (!ok && tid == 0) atomicOr(ks.err, kErrMmaWait);
      if (ring == 2 && k + 2 < ntl) {  // tile k's slot is free once its MMA is done
        load_tile(tl_ + 2, tile_buf(k + 2));
        cp_commit();
      }
      fence_after();
      const uint32_t tm = tbase + (uint32_t)(buf * ncp) + ((uint32_t)((warp & 3) * 32) << 16);
      // ---- epilogue: each half of the warps scans half of the columns ---------
      // four independent best / runner-up trackers (columns c = 4m + e) keep
      // the compare chains short; merged by (value, index)
      float b1 = INFINITY, b2 = INFINITY;
      int bi = 0;
      if (ok) {
        float t1[4], t2[4];
        int ti[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          t1[e] = INFINITY;
          t2[e] = INFINITY;
          ti[e] = 0;
        }
        for (int c0 = half * hw; c0 < (half + 1) * hw; c0 += 64) {
          uint32_t rv[4][16];
          const int nb = imin(4, ((half + 1) * hw - c0) / 16);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (q < nb) tmem_ld16_nw(tm + (uint32_t)(c0 + 16 * q), rv[q]);
          tmem_wait();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (q >= nb) break;
            const float4* cq4 = reinterpret_cast<const float4*>(cn2s + c0 + 16 * q);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              const float4 cc = cq4[v4];
              const float cn[4] = {cc.x, cc.y, cc.z, cc.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int c = c0 + 16 * q + 4 * v4 + e;
                const float dd = fmaf(-2.f, __uint_as_float(rv[q][4 * v4 + e]), cn[e]);
                const bool lt = dd < t1[e];
                t2[e] = lt ? t1[e] : fminf(t2[e], dd);
                ti[e] = lt ? c : ti[e];
                t1[e] = lt ? dd : t1[e];
              }
            }
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (t1[e] < b1 || (t1[e] == b1 && ti[e] < bi)) {
            b2 = fminf(b1, t2[e]);
            b1 = t1[e];
            bi = ti[e];
          } else {
            b2 = fminf(b2, t1[e]);
          }
        }
      }
      if (half == 1) {
        hb1[row] = b1;
        hb2[row] = b2;
        hbi[row] = bi;
      }
      __syncthreads();
      if (half == 0 && row < nt) {
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
        const float xn = xns[u];
        const float E = 2.f * 3.0517578e-05f * xn * cm + 2.3841858e-07f * (cm * cm + 2.f * xn * cm);
        asg[u] = (unsigned short)bi;
        const bool queued = !ok || (b2 - b1) <= 2.f * E;
        int qi = -1;
        if (queued) {
          qi = atomicAdd(&qcount, 1);
          queue[qi] = (unsigned short)u;
          if (qi < kFCandCap) ccnt[qi] = ok ? 0 : kFMaxCand + 1;  // unusable screen: every cluster
        }
        // the band of a queued row for the candidate scan below (the merged
        // best and runner-up are read; hb2 / hbi now carry the band and slot)
        hb2[row] = (queued && ok && qi < kFCandCap) ? b1 + 2.f * E : -INFINITY;
        hbi[row] = qi;
      } else if (half == 0) {
        hb2[row] = -INFINITY;
      }
      __syncthreads();
      // ---- candidates of the queued rows: every column inside the band, both
      // column halves, while the tile's accumulator is still in TMEM (the next
      // MMA into this buffer is issued after the next loop-top barrier) --------
      {
        const float lim = hb2[row];
        const bool rec = lim > -INFINITY;
        if (__any_sync(0xffffffffu, rec)) {
          const int qi = hbi[row];
          for (int c0 = half * hw; c0 < (half + 1) * hw; c0 += 16) {  // hw: a multiple of 16
            uint32_t rv[16];
            tmem_ld16_nw(tm + (uint32_t)c0, rv);
            tmem_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int c = c0 + e;
              const float dd = fmaf(-2.f, __uint_as_float(rv[e]), cn2s[c]);
              if (rec && dd <= lim) {
                const int k = atomicAdd(&ccnt[qi], 1);
                if (k < kFMaxCand) cand[qi * kFMaxCand + k] = (unsigned short)c;
              }
            }
          }
        }
      }
    }
    __syncthreads();
    // ---- exact fp64 decision of the queued tokens, one warp per token --------
    const int qn = qcount;
    // tokens without a usable candidate list: an exact argmin over every cluster
    bool any_full = qn > kFCandCap;
    for (int e = tid; e < qn && e < kFCandCap; e += kFT)
      if (ccnt[e] < 1 || ccnt[e] > kFMaxCand) any_full = true;
    any_full = __syncthreads_or(any_full);
    if (qn > 0) {
      if ((stage & 1) && any_full) {
        const int tot = C * D;
        for (int e0 = tid; e0 < tot; e0 += 16 * kFT) {  // 16 loads in flight per thread
          double v[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) v[u] = e0 + u * kFT < tot ? __ldcg(c64g + e0 + u * kFT) : 0.0;
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const int e = e0 + u * kFT;
            if (e < tot) {
              const int c = e / D, d = e - c * D;
              cst[c * (D + 1) + d] = v[u];
            }
          }
        }
        __syncthreads();
      }
      double* xw = xs + warp * D;
      for (int e = warp; e < qn; e += kWarps) {
        const int uq = queue[e];
        const __nv_bfloat16* xr = X + (p.row0 + tok0 + uq) * D;
        for (int d = lane; d < D; d += 32) xw[d] = (double)__bfloat162float(xr[d]);
        __syncwarp();
        const int nc = e < kFCandCap ? ccnt[e] : kFMaxCand + 1;
        int bc;
        if (nc >= 1 && nc <= kFMaxCand) {
          // the exact winner lies in the band: one candidate per lane, each a
          // plain sequential fp64 distance in dimension order
          double bd = 0.0;
          bc = -1;
          if (lane < nc) {
            const int c = cand[e * kFMaxCand + lane];
            const double* cr = c64g + (size_t)c * D;
            double sd = 0.0;
#pragma unroll 16
            for (int d = 0; d < D; ++d) {
              const double t = __dsub_rn(xw[d], __ldcg(cr + d));
              sd = __dadd_rn(sd, __dmul_rn(t, t));
            }
            bd = sd;
            bc = c;
          }
          for (int o = 16; o; o >>= 1) {
            const double od = __shfl_xor_sync(0xffffffffu, bd, o);
            const int oc = __shfl_xor_sync(0xffffffffu, bc, o);
            if (oc >= 0 && (bc < 0 || od < bd || (od == bd && oc < bc))) {
              bd = od;
              bc = oc;
            }
          }
        } else {
          bc = ((stage & 1) && any_full) ? exact_argmin<D, true>(xw, cst, c64g, C, lane)
                                         : exact_argmin<D, false>(xw, cst, c64g, C, lane);
        }
        if (lane == 0) asg[uq] = (unsigned short)bc;
        __syncwarp();
      }
      __syncthreads();
    }
    if (cert && it > 0) {
      // ---- the tokens that changed cluster move the running sums ---------------
      // (ks.assign holds every token's cluster of the previous round)
      if (tid == 0) nmv_s = 0;
      __syncthreads();
      int* asg_g = ks.assign + p.slot0 + tok0;
      for (int u0 = 0; u0 < ntok; u0 += kFT) {
        const int u = u0 + tid;
        const bool moved = u < ntok && (int)asg[u] != __ldcg(asg_g + u);
        const unsigned bal = __ballot_sync(0xffffffffu, moved);
        int slot = 0;
        if (lane == 0 && bal) slot = atomicAdd(&nmv_s, __popc(bal));
        slot = __shfl_sync(0xffffffffu, slot, 0);
        if (moved) queue[slot + __popc(bal & ((1u << lane) - 1u))] = (unsigned short)u;
      }
      __syncthreads();
      const int nmv = nmv_s;
      for (int e = warp; e < nmv; e += kWarps) {
        const int u = queue[e];
        const int a = asg[u], b = __ldcg(asg_g + u);
        const __nv_bfloat16* xr = X + (p.row0 + tok0 + u) * D;
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
          const int d = lane + 32 * j;
          const double x = (double)__bfloat162float(xr[d]);
          atomicAdd(sumg + (size_t)a * D + d, x);
          atomicAdd(sumg + (size_t)b * D + d, -x);
        }
        if (lane == 0) {
          atomicAdd(cntg + a, 1);
          atomicAdd(cntg + b, -1);
          dirt[a] = it;
          dirt[b] = it;
        }
      }
      __syncthreads();
      for (int e = tid; e < nmv; e += kFT) {
        const int u = queue[e];
        asg_g[u] = asg[u];
      }
      if (tid == 0 && nmv > 0) atomicAdd(chgp + (it & 1), nmv);
      team_sync();
      if (bar_fail) break;
      // every CTA of the problem reads the same total after the barrier
      const int moved_all = __ldcg(chgp + (it & 1));
      fin = last || moved_all == 0;
      if (rank == 0 && tid == 0) chgp[(it + 1) & 1] = 0;
      if (!fin) {
        // owners: new centroids of the clusters whose members changed
        for (int c = rank + NCT * warp; c < C; c += NCT * kWarps) {
          const int n = __ldcg(dirt + c) == it ? __ldcg(cntg + c) : 0;
          if (n == 0) continue;  // unchanged members, or an empty cluster: the centroid stays
          double acc[VPL];
          const double* sr = sumg + (size_t)c * D + (size_t)lane * VPL;
#pragma unroll
          for (int e = 0; e < VPL; ++e) acc[e] = __ldcg(sr + e);
          write_centroid(c, n, acc);
        }
        team_sync();
        if (bar_fail) break;
        continue;
      }
    }
    // ---- group this CTA's tokens by cluster (stable) and publish the list ----
    {
      const int per = cdiv(cdiv(ntok, kWarps), 32) * 32;
      const int lo = imin(ntok, warp * per), hi = imin(ntok, lo + per);
      int* wh = whist + warp * NC;
      for (int c = lane; c < C; c += 32) wh[c] = 0;
      __syncwarp();
      for (int b0 = lo; b0 < hi; b0 += 32) {
        const int t = b0 + lane;
        const int a = t < hi ? (int)asg[t] : -1 - lane;
        const unsigned same = __match_any_sync(0xffffffffu, a);
        if (a >= 0 && __ffs(same) - 1 == lane) wh[a] += __popc(same);
        __syncwarp();
      }
      __syncthreads();
      for (int c = tid; c < C; c += kFT) {
        int run = 0;
        for (int w = 0; w < kWarps; ++w) {
          const int h = whist[w * NC + c];
          whist[w * NC + c] = run;
          run += h;
        }
        loff[c] = run;
      }
      __syncthreads();
      block_scan_excl(loff, C, scan_tmp);
      int* xr = xoff + (size_t)rank * (g.C + 1);
      for (int c = tid; c < C; c += kFT) {
        const int s0 = loff[c];
        for (int w = 0; w < kWarps; ++w) whist[w * NC + c] += s0;
        if (ntok > 0) xr[c] = s0;
      }
      if (tid == 0 && ntok > 0) xr[C] = ntok;
      __syncthreads();
      unsigned short* myl = tl + (size_t)rank * tpc * kTile;
      for (int b0 = lo; b0 < hi; b0 += 32) {
        const int t = b0 + lane;
        const int a = t < hi ? (int)asg[t] : -1 - lane;
        const unsigned same = __match_any_sync(0xffffffffu, a);
        if (a >= 0) myl[wh[a] + __popc(same & ((1u << lane) - 1u))] = (unsigned short)t;
        __syncwarp();
        if (a >= 0 && __ffs(same) - 1 == lane) wh[a] += __popc(same);
        __syncwarp();
      }
      if (fin || cert)
        for (int t = tid; t < ntok; t += kFT) ks.assign[p.slot0 + tok0 + t] = asg[t];
    }
    team_sync();
    if (bar_fail) break;
    // ---- owners: counts, offsets, means over all CTAs' members ----------------
    if (fin) {
      for (int c = tid; c < C; c += kFT) goff[c] = 0;
      __syncthreads();
      for (int k = tid; k < C * nra; k += kFT) {  // (cluster, rank) pairs
        const int c = k / nra, r = k - c * nra;
        const int* xr = xoff + (size_t)r * (g.C + 1) + c;
        atomicAdd(&goff[c], __ldcg(xr + 1) - __ldcg(xr));
      }
      __syncthreads();
      const int tot = block_scan_excl(goff, C, scan_tmp);
      if (tid == 0) goff[C] = tot;
      __syncthreads();
    }
    // ---- owners: this CTA's clusters, largest first, one warp per cluster ----
    {
      const int nown = C > rank ? cdiv(C - rank, NCT) : 0;  // clusters rank + NCT i
      // (owned cluster, rank) pairs, one thread each: list start and count
      // (nown * nra < C + NCT <= kOT pairs)
      for (int k = tid; k < nown * nra; k += kFT) {
        const int i = k / nra, r = k - i * nra;
        const int* xr = xoff + (size_t)r * (g.C + 1) + rank + NCT * i;
        const int m0 = __ldcg(xr), m1 = __ldcg(xr + 1);
        otab[2 * k] = m0;
        otab[2 * k + 1] = m1 - m0;
      }
      if (tid == 0) own_ctr = 0;
      __syncthreads();
      for (int i = tid; i < nown; i += kFT) {
        int n = 0;
        for (int r = 0; r < nra; ++r) n += otab[2 * (i * nra + r) + 1];
        own_n[i] = n;
      }
      __syncthreads();
      for (int i = tid; i < nown; i += kFT) {  // sizes descending: largest clusters first
        const int ni = own_n[i];
        int rk = 0;
        for (int k = 0; k < nown; ++k) {
          const int nk = own_n[k];
          rk += (nk > ni || (nk == ni && k < i)) ? 1 : 0;
        }
        own_ord[rk] = i;
      }
      __syncthreads();
      int* gP = gtab + warp * (2 * kMaxNCT + 1);  // [0, nra]: members before rank r
      int* gB = gP + kMaxNCT + 1;                 // [r]: list index of rank r's first member
      const RowT* Xl = reinterpret_cast<const RowT*>(X + p.row0 * D) + lane;
      for (;;) {
        int k = 0;
        if (lane == 0) k = atomicAdd(&own_ctr, 1);
        k = __shfl_sync(0xffffffffu, k, 0);
        if (k >= nown) break;
        const int io = own_ord[k];
        const int c = rank + NCT * io;
        const int n = own_n[io];
        int cnt = 0, m0 = 0;
        if (lane < nra) {
          m0 = otab[2 * (io * nra + lane)];
          cnt = otab[2 * (io * nra + lane) + 1];
        }
        int incl = cnt;
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        if (lane < nra) {
          gP[lane] = incl - cnt;
          gB[lane] = lane * tpc * kTile + m0;
        }
        if (lane == 0) gP[nra] = n;
        __syncwarp();
        // member j (concatenated over ranks, ascending token order) -> its
        // problem-local token; lanes fetch the entries of a batch in parallel
        int cur = 0;
        auto entry = [&](int j) -> int {
          if (j >= n || lane >= kOB) return 0;
          while (gP[cur + 1] <= j) ++cur;
          return cur * tpc * kTile + (int)__ldcg(tl + gB[cur] + (j - gP[cur]));
        };
        const size_t pbase = (size_t)p.slot0 + (fin ? goff[c] : 0);
        double acc[VPL];
#pragma unroll
        for (int e = 0; e < VPL; ++e) acc[e] = 0.0;
        // three batches in flight: rows of batches b+1 and b+2 load while
        // batch b is summed
        auto rows = [&](int e, int jb, RowT (&v)[kOB]) {
#pragma unroll
          for (int q = 0; q < kOB; ++q) {
            const int t = __shfl_sync(0xffffffffu, e, q);
            v[q] = jb + q < n ? __ldg(Xl + (size_t)t * (D / VPL)) : RowT{};
          }
        };
        RowT va[kOB], vb[kOB], vc[kOB];
        int ea = entry(lane);
        rows(ea, 0, va);
        int eb = entry(kOB + lane);
        rows(eb, kOB, vb);
        int ec = entry(2 * kOB + lane);
        for (int j0 = 0; j0 < n; j0 += kOB) {
          rows(ec, j0 + 2 * kOB, vc);
          const int ed = j0 + 3 * kOB < n ? entry(j0 + 3 * kOB + lane) : 0;
          if (fin && lane < kOB && j0 + lane < n) ks.perm[pbase + j0 + lane] = ea;
#pragma unroll
          for (int q = 0; q < kOB; ++q)
            if (j0 + q < n) add_row(acc, va[q]);
#pragma unroll
          for (int q = 0; q < kOB; ++q) {
            va[q] = vb[q];
            vb[q] = vc[q];
          }
          ea = eb;
          eb = ec;
          ec = ed;
        }
        if (fin && lane == 0) {
          ks.counts[cbase + c] = n;
          ks.off[(size_t)pid * (g.C + 1) + c] = goff[c];
          if (c == C - 1) ks.off[(size_t)pid * (g.C + 1) + C] = goff[C];
        }
        if (cert) {  // the running state of the later rounds
          double* sr = sumg + (size_t)c * D + (size_t)lane * VPL;
#pragma unroll
          for (int e = 0; e < VPL; ++e) sr[e] = acc[e];
          if (lane == 0) {
            cntg[c] = n;
            dirt[c] = 0;
          }
        }
        if (n > 0) write_centroid(c, n, acc);  // an empty cluster keeps its centroid
        __syncwarp();  // the warp's tables are rewritten for its next cluster
      }
    }
    // the change counter of round 1 starts from zero
    if (cert && it == 0 && rank == 0 && tid == 0) chgp[1] = 0;
    team_sync();
    if (bar_fail) break;
    if (fin) break;
  }
  fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tbase), "r"(tcols));
}

// CTAs per problem and launch form for the problems of one level (lvl >= 0)
// or of all levels (lvl < 0, the acausal single level).
struct FusedPlan {
  bool coop;
  int NCT;
  FusedLayout L;
};

template <int D>
static bool plan_fused(const RoleGeo* gs, const KState* kss, int nsets, int lvl, int NC,
                       FusedPlan& plan) {
  int ntp_max = 1, nprob = 0;
  for (int k = 0; k < nsets; ++k) {
    const int l0 = lvl < 0 ? 0 : lvl, l1 = lvl < 0 ? gs[k].lv.nlev : lvl + 1;
    for (int l = l0; l < l1; ++l) {
      const int ntp = cdiv(gs[k].lv.s[l], kTile);
      ntp_max = ntp_max > ntp ? ntp_max : ntp;
    }
    nprob += lvl < 0 ? kss[k].nprob : gs[k].BH * gs[k].lv.npairs[lvl];
  }
  auto layout_for = [&](int nct, FusedLayout& Lc) {
    const int tpc_max = cdiv(ntp_max, nct);
    if (tpc_max * kTile > 65535) return false;
    for (int flags : {1, 0, 3, 2}) {  // three tile slots first, staging first
      Lc = fused_layout(D, NC, tpc_max, flags);
      if (Lc.total <= kSmemLimit) return true;
    }
    return false;
  };
  int dev = 0, nsm = 0, coop_ok = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&coop_ok, cudaDevAttrCooperativeLaunch, dev);
  // cooperative launch: every problem's CTAs resident at once, as many per
  // problem as the GPU allows (at most one per tile)
  int nctc = nsm / (nprob > 0 ? nprob : 1);
  nctc = nctc < kMaxNCT ? nctc : kMaxNCT;
  nctc = nctc < ntp_max ? nctc : ntp_max;
  if (coop_ok && nctc >= 2 && layout_for(nctc, plan.L)) {
    cudaFuncSetAttribute(kmeans_fused_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)plan.L.total);
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kmeans_fused_kernel<D, true>, kFT,
                                                      plan.L.total) == cudaSuccess &&
        (long long)per_sm * nsm >= (long long)nprob * nctc) {
      plan.coop = true;
      plan.NCT = nctc;
      return true;
    }
    cudaGetLastError();
  }
  // thread-block clusters, in waves when the problems do not all fit: about
  // sixteen tiles per CTA (the per-round fixed costs -- set-up, drain, sort,
  // owner sums, barriers -- stay small against the tiles), at least enough
  // CTAs to fill the GPU, at most one per tile; when that layout does not fit
  // in shared memory, more CTAs (fewer tiles each), else fewer
  const bool big_ok =
      cudaFuncSetAttribute(kmeans_fused_kernel<D, false>,
                           cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
  if (!big_ok) cudaGetLastError();
  const int cmax = big_ok ? 16 : 8;
  int nct0 = cdiv(ntp_max, kTilesPerCta);
  const int fill = nsm / (nprob > 0 ? nprob : 1);
  nct0 = nct0 > fill ? nct0 : fill;
  nct0 = nct0 < ntp_max ? nct0 : ntp_max;
  nct0 = nct0 < cmax ? nct0 : cmax;
  nct0 = nct0 > 1 ? nct0 : 1;
  auto try_nct = [&](int nct) {
    FusedLayout Lc;
    if (!layout_for(nct, Lc)) return false;
    cudaFuncSetAttribute(kmeans_fused_kernel<D, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lc.total);
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
    if (cudaOccupancyMaxActiveClusters(&active, kmeans_fused_kernel<D, false>, &q) != cudaSuccess) {
      cudaGetLastError();
      active = 0;
    }
    if (active < 1) return false;
    plan.coop = false;
    plan.NCT = nct;
    plan.L = Lc;
    return true;
  };
  for (int nct = nct0; nct <= cmax && nct <= ntp_max; ++nct)
    if (try_nct(nct)) return true;
  for (int nct = nct0 - 1; nct >= 1; --nct)
    if (try_nct(nct)) return true;
  return false;
}

template <int D>
static void launch_plan(const RoleGeo* gs, const KState* kss, int nsets, int lvl, int iters,
                        int NC, int tcols, const FusedPlan& plan, bool skip_certified,
                        cudaStream_t st) {
  FusedSets fs{};
  int np[2] = {0, 0};
  for (int k = 0; k < nsets; ++k) {
    fs.g[k] = gs[k];
    fs.ks[k] = kss[k];
    np[k] = lvl < 0 ? kss[k].nprob : gs[k].BH * gs[k].lv.npairs[lvl];
  }
  fs.lvl = lvl;
  fs.fault_rank = plan.coop ? g_fault_rank : -1;
  fs.spin_limit = g_spin_limit;
  fs.skip_certified = skip_certified ? 1 : 0;
  fs.nblk0 = np[0] * plan.NCT;
  const int nblk = (np[0] + np[1]) * plan.NCT;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)nblk);
  cfg.blockDim = dim3(kFT);
  cfg.dynamicSmemBytes = plan.L.total;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  if (plan.coop) {
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
  } else {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = plan.NCT;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (plan.coop) {
    cudaFuncSetAttribute(kmeans_fused_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)plan.L.total);
    cudaLaunchKernelEx(&cfg, kmeans_fused_kernel<D, true>, fs, iters, plan.NCT, NC, plan.L.tpc,
                       tcols, plan.L.flags);
  } else {
    cudaFuncSetAttribute(kmeans_fused_kernel<D, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.L.total);
    cudaLaunchKernelEx(&cfg, kmeans_fused_kernel<D, false>, fs, iters, plan.NCT, NC, plan.L.tpc,
                       tcols, plan.L.flags);
  }
}

// Returns false (nothing launched) when the fused path does not cover these
// problem sets: more than 256 clusters, or no layout fits in shared memory.
// A causal problem set (several levels) gets one launch per level, each with
// its own CTAs per problem.
template <int D>
static bool launch_fused_t(const RoleGeo* gs, const KState* kss, int nsets, int iters,
                           cudaStream_t st) {
  int cmax = 0;
  for (int k = 0; k < nsets; ++k) {
    if (gs[k].dtype != 0 || gs[k].C > kNCF || gs[k].D != D) return false;
    if (k > 0 && gs[k].lv.nlev != gs[0].lv.nlev) return false;
    cmax = cmax > gs[k].C ? cmax : gs[k].C;
  }
  const int NC = (cmax + 31) & ~31;
  int tcols = 32;
  while (tcols < 2 * NC) tcols <<= 1;  // two accumulators (tiles in flight)
  // per level: the resident-tile kernel where it covers the sizes, followed
  // by this kernel for the problems whose sums it cannot certify exact
  const int nlev = gs[0].lv.nlev;
  FusedPlan plans[kMaxLevels];
  auto level = [&](int l, const FusedPlan& plan) {
    bool res;
    {
      ProfScope ps(st, "kmeans_resident");
      res = !g_no_resident && launch_kmeans_resident(gs, kss, nsets, l, iters, st);
    }
#ifdef MUSE_PHASE_CLOCKS
    {
      const cudaError_t e = cudaStreamSynchronize(st);
      fprintf(stderr, "after resident lvl %d (launched %d): %s\n", l, (int)res, cudaGetErrorString(e));
    }
#endif
    ProfScope ps(st, "kmeans_ordered");
    launch_plan<D>(gs, kss, nsets, l, iters, NC, tcols, plan, res, st);
#ifdef MUSE_PHASE_CLOCKS
    {
      const cudaError_t e = cudaStreamSynchronize(st);
      fprintf(stderr, "after ordered lvl %d (coop %d nct %d): %s\n", l, (int)plan.coop, plan.NCT,
              cudaGetErrorString(e));
    }
#endif
  };
  if (nlev == 1) {
    if (!plan_fused<D>(gs, kss, nsets, -1, NC, plans[0])) return false;
    level(-1, plans[0]);
    return true;
  }
  for (int l = 0; l < nlev; ++l)
    if (!plan_fused<D>(gs, kss, nsets, l, NC, plans[l])) return false;
  for (int l = 0; l < nlev; ++l) level(l, plans[l]);
  return true;
}

void set_barrier_fault(int rank, int spin_limit) {
  g_fault_rank = rank;
  g_spin_limit = rank >= 0 && spin_limit > 0 ? spin_limit : kSpinLimit;
  // the fault hook targets this kernel's cooperative barrier
  g_no_resident = rank >= 0 ? 1 : 0;
}

bool launch_kmeans_fused(const RoleGeo* gs, const KState* kss, int nsets, int iters,
                         cudaStream_t st) {
  return gs[0].D == 64 ? launch_fused_t<64>(gs, kss, nsets, iters, st)
                       : launch_fused_t<128>(gs, kss, nsets, iters, st);
}

}  // namespace muse
