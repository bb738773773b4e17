// Persistent Lloyd k-means for bf16 inputs with every token tile resident in
// shared memory for the whole launch, and centroid sums taken in any order.
//
// The clustering step of MuSe (gist.science page "Multipole Semantic
// Attention: A Fast Approximation of Softmax Attention for Pretraining",
// Technical Summary, Core Mechanisms, "Bidirectional Semantic Clustering");
// Lloyd's algorithm with squared Euclidean distance, ties to the lowest
// cluster index, empty clusters keeping their centroid.
//
// NCT CTAs serve one problem (one thread-block cluster, or one CTA when the
// problem's tiles fit in one), each holding its share of the problem's
// 128-token tiles in shared memory from the first round on.  Per round:
//   1. the centroids' bf16 hi + lo split (the tensor-core B operand) and
//      their squared norms are loaded;
//   2. screen: one warp issues tcgen05.mma for every tile into a ring of TMEM
//      accumulators; two warpgroups of epilogue warps take alternate tiles,
//      one thread per token row scanning every centroid column for the best
//      and runner-up screened distance.  A token whose gap lies inside the
//      certified error of the screen is queued, with the clusters inside
//      that band (the only possible exact winners) as its candidates;
//   3. the queued tokens get the exact argmin among their candidates, each
//      distance a plain sequential fp64 sum in dimension order (so ties
//      resolve exactly as a sequential evaluation does);
//   4. first round: the CTA groups its tokens by cluster (stable counting
//      sort) and sums each cluster's rows from shared memory in fp64, in any
//      order: the exponent range of the problem's values, measured by the
//      seeded-start kernel, certifies that every partial sum is exact
//      (sums_exact), so the result equals a sequential fp64 sum bit for bit.
//      A problem that fails the certificate is left to the sequential-order
//      kernel.  The CTAs' partial sums meet in global memory (L2); after a
//      team barrier the owner CTA of each centroid (c % NCT) adds them, keeps
//      the exact total and the count as the problem's running state, and
//      writes the new centroid;
//   5. later rounds: only the tokens whose cluster changed move the running
//      sums (fp64 atomic adds of +x and -x, exact in any order since every
//      value passed through is the sum of a subset of the problem's tokens)
//      and counts; after the barrier the owners recompute just the clusters
//      whose members changed.  A round in which no token of the problem moved
//      repeats the previous one exactly, and so would every later round: the
//      problem ends there with the same result as running all rounds.
// After the last round every CTA writes its tokens' assignments and its
// members' places in the cluster-sorted permutation; the owners write the
// counts and segment offsets.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <stdio.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace muse {

namespace {

constexpr int kEW = 16;                // epilogue warps: four warpgroups of kWGW
constexpr int kWGW = 4;                // warps per warpgroup (one per TMEM lane quadrant)
constexpr int kRW = kEW + 1;           // + the MMA warp
constexpr int kRT = kRW * 32;          // threads
constexpr int kRMaxNCT = 16;           // CTAs per problem (one thread-block cluster)
constexpr int kMaxCand = 8;            // candidates kept per queued token
constexpr int kCandCap = 128;          // queued tokens with a candidate list per round
constexpr unsigned kFull = 0xFFu;      // candidate count meaning "every cluster"
constexpr size_t kRSmemMax = 222 * 1024;  // dynamic shared memory (static arrays come on top)
constexpr int kNCFR = 256;             // clusters (one MMA pass of N <= 256)
constexpr int kRMaxTPC = 16;           // tiles per CTA
constexpr int kPartSMs = 160;          // CTA bound behind the partial-sum tables' size

__device__ inline uint32_t sa(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ inline uint64_t desc128(uint32_t a) {  // K-major, 128-byte swizzle, 8-row groups 1 KB apart
  return (uint64_t)((a >> 4) & 0x3FFF) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}
__device__ inline uint32_t swz(int r, int q) { return r * 128 + ((q ^ (r & 7)) << 4); }
__device__ inline void umma(uint32_t tmem, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem),
      "l"(ad), "l"(bd), "r"(idesc), "r"(acc));
}
__device__ inline void umma_commit(uint32_t mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(mbar)
               : "memory");
}
__device__ inline void mbar_init(uint32_t mbar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(mbar), "r"(count));
}
__device__ inline void mbar_arrive(uint32_t mbar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}\n" ::"r"(mbar)
               : "memory");
}
// Bounded wait for the completion of the phase with this parity.
__device__ inline bool mbar_wait(uint32_t mbar, uint32_t parity) {
  for (int it = 0; it < (1 << 22); ++it) {
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
__device__ inline void tld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ inline void tld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
__device__ inline void tc_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ inline void tc_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ inline void fence_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
__device__ inline void cp16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(sa(dst)), "l"(src),
               "r"(src_bytes));
}
__device__ inline void cp_commit_wait() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
}

// Exclusive scan of n <= 2 * blockDim.x ints in shared memory by the whole
// CTA; returns the total.  `tmp` holds one int per warp.
__device__ inline int scan_excl(int* a, int n, int* tmp) {
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

// Shared-memory plan of one CTA: TPC resident tiles and the per-round tables.
struct RLayout {
  int KB, NC, TPC;
  size_t tiles, bh, bl, stage, cn2, xn, asg, lst, queue, cand, ccnt, whist, loff, xs, total;
};

__host__ __device__ inline RLayout rlayout(int D, int NC, int TPC) {
  RLayout L;
  L.KB = D / 64;
  L.NC = NC;
  L.TPC = TPC;
  size_t o = 0;
  L.tiles = o;  o += (size_t)TPC * L.KB * kTile * 128;
  // centroid hi / lo operands; after each round's screen the same bytes stage
  // the drain's fp64 candidate rows: at least one row of D + 1 doubles per warp
  L.bh = o;
  L.bl = o + (size_t)L.KB * NC * 128;
  L.stage = 2 * (size_t)L.KB * NC * 128;
  if (L.stage < (size_t)kRW * (D + 1) * 8) L.stage = (size_t)kRW * (D + 1) * 8;
  o += (L.stage + 15) & ~(size_t)15;
  L.cn2 = o;    o += (size_t)NC * 4;
  L.xn = o;     o += (size_t)TPC * kTile * 4;
  L.asg = o;    o += (size_t)TPC * kTile * 2;
  L.lst = o;    o += (size_t)TPC * kTile * 2;
  L.queue = o;  o += (size_t)TPC * kTile * 2;
  L.cand = o;   o += (size_t)kCandCap * kMaxCand * 2;
  L.ccnt = o;   o += (size_t)kCandCap;
  o = (o + 15) & ~(size_t)15;
  L.whist = o;  o += (size_t)kRW * NC * 4;
  L.loff = o;   o += (size_t)(NC + 1) * 4;
  o = (o + 15) & ~(size_t)15;
  L.xs = o;     o += (size_t)kRW * D * 8;
  L.total = o + 1024;  // alignment slack of the dynamic base
  return L;
}

// A lane's D/32 consecutive dimensions of token row r of a resident tile.
template <int D>
__device__ inline void row_part(const unsigned char* tile, int r, int lane, float (&v)[D / 32]) {
  if (D == 64) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(tile + swz(r, lane >> 2) + (lane & 3) * 4);
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
    v[0] = f.x;
    v[1] = f.y;
  } else {
    const int kb = lane >> 4, l = lane & 15;
    const uint2 w = *reinterpret_cast<const uint2*>(tile + kb * kTile * 128 + swz(r, l >> 1) + (l & 1) * 8);
    const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
    const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
    v[0] = f0.x;
    v[1] = f0.y;
    v[D / 32 - 2] = f1.x;
    v[D / 32 - 1] = f1.y;
  }
}

}  // namespace

// Phase clocks for tuning (compiled only with -DMUSE_PHASE_CLOCKS): thread 0
// of every CTA adds the clock64 cycles of each phase to a shared row, written
// to a per-CTA global row when the CTA ends (slots 10..: event counts).
#ifdef MUSE_PHASE_CLOCKS
constexpr int kPhaseSlots = 16;
__device__ long long g_phase_clk[8192][kPhaseSlots];
#define PHASE_INIT                                            \
  __shared__ long long ph_acc[kPhaseSlots];                   \
  if (threadIdx.x < kPhaseSlots) ph_acc[threadIdx.x] = 0;     \
  __syncthreads();                                            \
  long long ph_t = clock64()
#define PHASE(i)                                        \
  do {                                                  \
    if (threadIdx.x == 0) {                             \
      const long long t_ = clock64();                   \
      ph_acc[i] += t_ - ph_t;                           \
      ph_t = t_;                                        \
    }                                                   \
  } while (0)
#define PHASE_COUNT(i, v)                               \
  do {                                                  \
    if (threadIdx.x == 0) ph_acc[i] += (v);             \
  } while (0)
#define PHASE_FLUSH                                                          \
  do {                                                                       \
    __syncthreads();                                                         \
    if (threadIdx.x < kPhaseSlots)                                           \
      g_phase_clk[blockIdx.x & 8191][threadIdx.x] += ph_acc[threadIdx.x];    \
  } while (0)
__device__ int g_bad[16];
#define BADCHK(cond, code)                       \
  do {                                           \
    if (!(cond)) atomicExch(&g_bad[code], 1 + (int)blockIdx.x); \
  } while (0)
#else
#define BADCHK(cond, code) \
  do {                     \
  } while (0)
#define PHASE_INIT
#define PHASE(i) \
  do {           \
  } while (0)
#define PHASE_COUNT(i, v) \
  do {                    \
  } while (0)
#define PHASE_FLUSH \
  do {              \
  } while (0)
#endif

struct ResidentSets {
  RoleGeo g[2];
  KState ks[2];
  double* part[2];   // [problem][NCT][C][D] per-CTA partial sums (NCT > 1)
  int* pcnt[2];      // [problem][NCT][C]    per-CTA member counts (NCT > 1)
  int nblk0;
  int lvl;
};

// MODE 0: one CTA per problem; 1: the NCT CTAs of a problem form one
// thread-block cluster (hardware barrier); 2: cooperative launch, the NCT CTAs
// of a problem meet at a bounded barrier on a global counter.  tcols: TMEM
// columns (NACC accumulators of NC columns).
template <int D, int MODE>
__global__ void __launch_bounds__(kRT, 1) kmeans_resident_kernel(ResidentSets rs, int iters, int NCT,
                                                                int NC, int TPC, int NACC,
                                                                int tcols) {
  constexpr bool CLUSTER = MODE == 1;
  extern __shared__ __align__(1024) unsigned char rz_dyn[];
  unsigned char* base = rz_dyn + ((1024 - (sa(rz_dyn) & 1023)) & 1023);
  const RLayout Lo = rlayout(D, NC, TPC);
  constexpr int KB = D / 64;
  constexpr int VPL = D / 32;
  constexpr int TILEB = KB * kTile * 128;
  const int set = (int)blockIdx.x < rs.nblk0 ? 0 : 1;
  const RoleGeo& g = rs.g[set];
  const KState& ks = rs.ks[set];
  const int blk = (int)blockIdx.x - (set ? rs.nblk0 : 0);
  const int rank = CLUSTER ? (int)cg::this_cluster().block_rank()
                            : (MODE == 2 ? (int)(blockIdx.x - (set ? rs.nblk0 : 0)) % NCT : 0);
  int pid = blk / NCT;
  if (rs.lvl >= 0) {  // j-th problem of the level -> problem id
    const int np = g.lv.npairs[rs.lvl];
    pid = (pid / np) * g.lv.pairs_per_bh + g.lv.pair_base[rs.lvl] + pid % np;
  }
  const Prob p = prob_of(g, pid);
  // every CTA of the problem takes the same decision: the sequential-order
  // kernel runs the problems whose sums are not certified exact
  if (!sums_exact(ks, pid, p.s)) return;
  PHASE_INIT;
  const int C = p.C;
  const int ntp = cdiv(p.s, kTile);
  const int tpc = cdiv(ntp, NCT);
  const int tile0 = rank * tpc, tile1 = imin(ntp, tile0 + tpc);
  const int ntl = tile1 > tile0 ? tile1 - tile0 : 0;
  const int tok0 = tile0 * kTile, tok1 = imin(p.s, tile1 * kTile);
  const int ntok = tok1 > tok0 ? tok1 - tok0 : 0;
  const __nv_bfloat16* X = static_cast<const __nv_bfloat16*>(g.X);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t cbase = (size_t)pid * g.C;
  const double* c64g = ks.cent64 + cbase * D;

  unsigned char* T = base + Lo.tiles;
  unsigned char* BH = base + Lo.bh;
  unsigned char* BL = base + Lo.bl;
  float* cn2s = reinterpret_cast<float*>(base + Lo.cn2);
  float* xns = reinterpret_cast<float*>(base + Lo.xn);
  unsigned short* asg = reinterpret_cast<unsigned short*>(base + Lo.asg);
  unsigned short* lst = reinterpret_cast<unsigned short*>(base + Lo.lst);
  unsigned short* queue = reinterpret_cast<unsigned short*>(base + Lo.queue);
  unsigned short* cand = reinterpret_cast<unsigned short*>(base + Lo.cand);
  unsigned char* ccnt = base + Lo.ccnt;
  int* whist = reinterpret_cast<int*>(base + Lo.whist);
  int* loff = reinterpret_cast<int*>(base + Lo.loff);
  double* xsw = reinterpret_cast<double*>(base + Lo.xs) + warp * D;
  __shared__ __align__(8) uint64_t mma_done[4], acc_free[4];
  __shared__ uint32_t tmem_slot;
  __shared__ int scan_tmp[32];
  __shared__ float cmax_s;
  __shared__ int qcount, nchg_s;
  __shared__ int gtot[kNCFR], gbefore[kNCFR];

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     sa(&tmem_slot)),
                 "r"(tcols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
  }
  if (tid == 0) {
    for (int s = 0; s < NACC; ++s) {
      mbar_init(sa(&mma_done[s]), 1);
      mbar_init(sa(&acc_free[s]), kWGW);  // one arrival per warp of the consuming warpgroup
    }
    asm volatile("fence.mbarrier_init.release.cluster;\n");
  }
  // the resident tiles (rows past the problem's end are zero)
  for (int e = tid; e < ntl * kTile * KB * 8; e += kRT) {
    const int t = e / (KB * 8), q = e - t * (KB * 8), kb = q >> 3, cq = q & 7;
    const int k = t >> 7, r = t & (kTile - 1);
    const bool live = t < ntok;
    cp16(T + k * TILEB + kb * kTile * 128 + swz(r, cq),
         X + (p.row0 + tok0 + (live ? t : 0)) * D + kb * 64 + cq * 8, live ? 16 : 0);
  }
  cp_commit_wait();
  tc_before();
  __syncthreads();
  tc_after();
  const uint32_t tbase = tmem_slot;
  // token norms (the screen's error bound), from the resident rows
  for (int u = tid; u < ntok; u += kRT) {
    const unsigned char* tile = T + (u >> 7) * TILEB;
    const int r = u & (kTile - 1);
    float q2 = 0.f;
#pragma unroll
    for (int kb = 0; kb < KB; ++kb)
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint4 v = *reinterpret_cast<const uint4*>(tile + kb * kTile * 128 + swz(r, q));
        const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(b[e]);
          q2 = fmaf(f.x, f.x, fmaf(f.y, f.y, q2));
        }
      }
    xns[u] = sqrtf(q2) * 1.0001f;
  }
  PHASE(0);
  const int ncp = (C + 31) & ~31;  // accumulator columns in use
  const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(ncp >> 3) << 17) |
                         ((uint32_t)(128 >> 4) << 24);
  // cooperative mode: arrivals counted on the problem's counter (zeroed by
  // the caller); a wait that gives up records kErrTeamBarrier and the CTA
  // leaves the round loop at once (bar_fail), reading nothing unpublished
  __shared__ int bar_fail;
  int nbar = 0;
  int* bar_ctr = ks.arrive + pid;
  if (tid == 0) bar_fail = 0;
  auto team_sync = [&]() {
    if (MODE == 1) {
      __threadfence();
      cg::this_cluster().sync();
    } else if (MODE == 2) {
      __syncthreads();
      if (tid == 0) {
        ++nbar;
        __threadfence();
        atomicAdd(bar_ctr, 1);
        for (int it = 0;; ++it) {
          int v;
          asm volatile("ld.acquire.gpu.global.s32 %0, [%1];\n" : "=r"(v) : "l"(bar_ctr) : "memory");
          if (v >= nbar * NCT) break;
          if (it >= (1 << 24)) {
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
      __syncthreads();
    }
  };
  bool mma_ok = true;
  int issued = 0;  // tiles the MMA warp has issued (its lane 0)

  for (int it = 0; it < iters; ++it) {
    const bool last = it + 1 == iters;
    // ---- 1. centroid operands of this round ---------------------------------
    for (int e = tid; e < ncp * KB * 8; e += kRT) {
      const int r = e / (KB * 8), q = e - r * (KB * 8), kb = q >> 3, cq = q & 7;
      const bool live = r < C;
      const size_t off = (cbase + (live ? r : 0)) * D + kb * 64 + cq * 8;
      cp16(BH + kb * NC * 128 + swz(r, cq), ks.cbf_hi + off, live ? 16 : 0);
      cp16(BL + kb * NC * 128 + swz(r, cq), ks.cbf_lo + off, live ? 16 : 0);
    }
    if (tid == 0) {
      cmax_s = 0.f;
      qcount = 0;
    }
    __syncthreads();
    {
      float m = 0.f;
      for (int c = tid; c < ncp; c += kRT) {
        const float v = c < C ? __ldcg(ks.cn2 + cbase + c) : INFINITY;  // padding never wins
        cn2s[c] = v;
        if (c < C) m = fmaxf(m, v);
      }
      for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) atomicMax(reinterpret_cast<int*>(&cmax_s), __float_as_int(m));
    }
    cp_commit_wait();
    fence_async();
    tc_before();
    __syncthreads();
    tc_after();
    const float cm = sqrtf(cmax_s) * 1.0001f;
    PHASE(1);

    // ---- 2. screen ------------------------------------------------------------
    if (warp == kEW) {
      if (lane == 0) {
        for (int k = 0; k < ntl; ++k) {
          const int kg = it * ntl + k, s = kg % NACC, use = kg / NACC;
          if (use > 0 && !mbar_wait(sa(&acc_free[s]), (uint32_t)((use - 1) & 1))) mma_ok = false;
          tc_after();
          const uint32_t tm = tbase + (uint32_t)(s * NC);
          const unsigned char* A = T + k * TILEB;
          for (int kb = 0; kb < KB; ++kb) {
            const uint64_t ad = desc128(sa(A + kb * kTile * 128));
            const uint64_t bh = desc128(sa(BH + kb * NC * 128));
            const uint64_t bl = desc128(sa(BL + kb * NC * 128));
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              umma(tm, ad + 2 * q, bh + 2 * q, idesc, (kb | q) ? 1u : 0u);
              umma(tm, ad + 2 * q, bl + 2 * q, idesc, 1u);
            }
          }
          umma_commit(sa(&mma_done[s]));
          ++issued;
          BADCHK(s * NC + ncp <= tcols, 6);
        }
      }
      __syncwarp();
    } else if (warp / kWGW < NACC) {
      // warpgroup wg takes the tiles k = wg (mod NACC): within a round each
      // accumulator slot belongs to one warpgroup, which waits for its uses
      // in order (a wait for a later phase parity must never be posted while
      // an earlier phase of the same barrier is still pending)
      const int wg = warp / kWGW, q4 = warp % kWGW, row = q4 * 32 + lane;
      for (int k = wg; k < ntl; k += NACC) {
        const int kg = it * ntl + k, s = kg % NACC, use = kg / NACC;
        BADCHK(k < TPC && s < NACC, 8);
#ifdef MUSE_PHASE_CLOCKS
        const long long sw0 = clock64();
#endif
        const bool ok = __all_sync(0xffffffffu, mbar_wait(sa(&mma_done[s]), (uint32_t)(use & 1)));
        tc_after();
#ifdef MUSE_PHASE_CLOCKS
        const long long sw1 = clock64();
        PHASE_COUNT(14, sw1 - sw0);
#endif
        const int u = k * kTile + row;  // CTA-local token of this thread's row
        const bool live = u < ntok;
        const uint32_t tm = tbase + (uint32_t)(s * NC) + ((uint32_t)(q4 * 32) << 16);
        float b1 = INFINITY, b2 = INFINITY;
        int bi = 0;
        if (ok) {
          // four best / runner-up trackers (columns c = 4 m + e) keep the
          // dependent chains short; merged by (value, index) below
          float t1[4], t2[4];
          int ti[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            t1[e] = INFINITY;
            t2[e] = INFINITY;
            ti[e] = 0;
          }
          for (int c0 = 0; c0 < ncp; c0 += 32) {  // ncp is a multiple of 32
            uint32_t rv[2][16];
#pragma unroll
            for (int q = 0; q < 2; ++q) tld16(tm + (uint32_t)(c0 + 16 * q), rv[q]);
            tld_wait();
#pragma unroll
            for (int q = 0; q < 2; ++q) {
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
        // |screen - exact| <= 2 |x| |c - hi - lo| + 2^-22 (|c|^2 + 2 |x| |c|): the
        // bf16 hi + lo split of the fp32 centroid leaves 2^-18 |c| and the fp32
        // rounding of the fp64 centroid 2^-24 |c| (2^-17 |x| |c| taken, twice
        // the sum), plus the fp32 rounding of |c|^2 and the fp32 accumulation
        // of 2D exact products
        const float xn = live ? xns[u] : 0.f;
        const float E = 1.5258789e-05f * xn * cm + 2.3841858e-07f * (cm * cm + 2.f * xn * cm);
        const bool queued = live && (!ok || (b2 - b1) <= 2.f * E);
        if (live) asg[u] = (unsigned short)bi;
        int qi = -1;
        if (queued) {
          qi = atomicAdd(&qcount, 1);
          queue[qi] = (unsigned short)u;
        }
        // candidates of the queued rows: every column within the band
        if (__any_sync(0xffffffffu, queued && ok && qi < kCandCap)) {
          const bool rec = queued && ok && qi < kCandCap;
          int nc = 0;
          const float lim = b1 + 2.f * E;
          for (int c0 = 0; c0 < ncp; c0 += 16) {
            uint32_t rv[16];
            tld16(tm + (uint32_t)c0, rv);
            tld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int c = c0 + e;
              const float dd = fmaf(-2.f, __uint_as_float(rv[e]), cn2s[c]);
              if (rec && dd <= lim) {
                if (nc < kMaxCand) cand[qi * kMaxCand + nc] = (unsigned short)c;
                ++nc;
              }
            }
          }
          if (rec) ccnt[qi] = (unsigned char)(nc <= kMaxCand ? nc : kFull);
          BADCHK(!rec || nc >= 1, 2);
        } else if (queued && qi < kCandCap) {
          ccnt[qi] = (unsigned char)kFull;  // the screen is unusable: every cluster
        }
        tc_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sa(&acc_free[s]));
#ifdef MUSE_PHASE_CLOCKS
        PHASE_COUNT(15, clock64() - sw1);
#endif
      }
    }
    __syncthreads();
    PHASE(2);
    if (warp == kEW && !mma_ok && lane == 0) atomicOr(ks.err, kErrMmaWait);

    // ---- 3. exact fp64 decision of the queued tokens, one warp per token -----
    // The candidates' fp64 centroid rows are staged in the warp's share of the
    // centroid-operand buffers (free until the next round reloads them), RB
    // rows at a time with a row stride of D + 1 doubles (distinct banks); each
    // lane then sums one candidate's distance in dimension order.
    {
      const int RB = (int)((Lo.stage / kRW) / ((D + 1) * 8));  // >= 1 by the layout
      double* crow = reinterpret_cast<double*>(BH + (size_t)warp * RB * (D + 1) * 8);
      const int qn = qcount;
      for (int e = warp; e < qn; e += kRW) {
        const int uq = queue[e];
        {  // x in fp64 (bf16 values are exact), lane l holds dimensions l VPL ..
          float v[VPL];
          row_part<D>(T + (uq >> 7) * TILEB, uq & (kTile - 1), lane, v);
#pragma unroll
          for (int j = 0; j < VPL; ++j) xsw[lane * VPL + j] = (double)v[j];
        }
        const unsigned ncc = e < kCandCap ? ccnt[e] : kFull;
        const bool full = ncc == kFull;
#ifdef MUSE_PHASE_CLOCKS
        if (lane == 0) atomicAdd(reinterpret_cast<unsigned long long*>(&ph_acc[10]),
                                 full ? 1000ull : (unsigned long long)ncc);
#endif
        const int nc = full ? C : (int)ncc;  // every cluster when the band was not recorded
        double bd = 0.0;
        int bc = -1;
        for (int j0 = 0; j0 < nc; j0 += RB) {
          const int nb = imin(RB, nc - j0);
          __syncwarp();
          for (int q = lane; q < nb * (D / 2); q += 32) {  // 16-byte pieces of the rows
            const int r = q / (D / 2), h = q - r * (D / 2);
            const int c = full ? j0 + r : (int)cand[e * kMaxCand + j0 + r];
            BADCHK(c >= 0 && c < C && (r * (D + 1) + 2 * h + 1) * 8 < (int)(Lo.stage / kRW) , 7);
            const double2 v = __ldcg(reinterpret_cast<const double2*>(c64g + (size_t)c * D) + h);
            crow[r * (D + 1) + 2 * h] = v.x;
            crow[r * (D + 1) + 2 * h + 1] = v.y;
          }
          __syncwarp();
          if (lane < nb) {
            const int c = full ? j0 + lane : (int)cand[e * kMaxCand + j0 + lane];
            const double* cr = crow + lane * (D + 1);
            double sd = 0.0;
#pragma unroll 16
            for (int d = 0; d < D; ++d) {
              const double t = __dsub_rn(xsw[d], cr[d]);
              sd = __dadd_rn(sd, __dmul_rn(t, t));
            }
            if (bc < 0 || sd < bd || (sd == bd && c < bc)) {
              bd = sd;
              bc = c;
            }
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
        BADCHK(bc >= 0 && bc < C, 3);
        if (lane == 0) asg[uq] = (unsigned short)bc;
        __syncwarp();
      }
    }
    __syncthreads();
    PHASE(3);
    PHASE_COUNT(11, qcount);

    // ---- 4. group this CTA's tokens by cluster (stable): lst, loff ------------
    auto group = [&]() {
      const int per = cdiv(cdiv(ntok > 0 ? ntok : 1, kRW), 32) * 32;
      const int lo = imin(ntok, warp * per), hi = imin(ntok, lo + per);
      int* wh = whist + warp * NC;
      for (int c = lane; c < C; c += 32) wh[c] = 0;
      __syncwarp();
      for (int b0 = lo; b0 < hi; b0 += 32) {
        const int t = b0 + lane;
        const int a = t < hi ? (int)asg[t] : -1 - lane;
        const unsigned same = __match_any_sync(0xffffffffu, a);
        BADCHK(a < C, 1);
        if (a >= 0 && a < C && __ffs(same) - 1 == lane) wh[a] += __popc(same);
        __syncwarp();
      }
      __syncthreads();
      for (int c = tid; c < C; c += kRT) {
        int run = 0;
        for (int w = 0; w < kRW; ++w) {
          const int h = whist[w * NC + c];
          whist[w * NC + c] = run;
          run += h;
        }
        loff[c] = run;
      }
      __syncthreads();
      scan_excl(loff, C, scan_tmp);
      if (tid == 0) loff[C] = ntok;
      for (int c = tid; c < C; c += kRT) {
        const int s0 = loff[c];
        for (int w = 0; w < kRW; ++w) whist[w * NC + c] += s0;
      }
      __syncthreads();
      for (int b0 = lo; b0 < hi; b0 += 32) {
        const int t = b0 + lane;
        const int a = t < hi ? (int)asg[t] : -1 - lane;
        const unsigned same = __match_any_sync(0xffffffffu, a);
        BADCHK(a < C, 0);
        if (a >= 0 && a < C) lst[wh[a] + __popc(same & ((1u << lane) - 1u))] = (unsigned short)t;
        __syncwarp();
        if (a >= 0 && __ffs(same) - 1 == lane) wh[a] += __popc(same);
        __syncwarp();
      }
      __syncthreads();
    };

    // ---- 5. the problem's exact cluster sums ----------------------------------
    // (exact in any order: sums_exact holds for this problem, and every value
    // a sum passes through below is the sum of a subset of its tokens)
    auto write_centroid = [&](int c, int n, const double (&acc)[VPL]) {
      const double nn = (double)n;
      double q2 = 0.0;
      float qf = 0.f;
      double v64[VPL];
      float v32[VPL];
#pragma unroll
      for (int e = 0; e < VPL; ++e) {
        v64[e] = __ddiv_rn(acc[e], nn);
        v32[e] = (float)v64[e];
        q2 += v64[e] * v64[e];
        qf = fmaf(v32[e], v32[e], qf);
      }
      const size_t i0 = (cbase + c) * D + (size_t)lane * VPL;
#pragma unroll
      for (int e = 0; e < VPL / 2; ++e) {
        const __nv_bfloat16 h0 = __float2bfloat16_rn(v32[2 * e]);
        const __nv_bfloat16 h1 = __float2bfloat16_rn(v32[2 * e + 1]);
        const __nv_bfloat16 l0 = __float2bfloat16_rn(v32[2 * e] - __bfloat162float(h0));
        const __nv_bfloat16 l1 = __float2bfloat16_rn(v32[2 * e + 1] - __bfloat162float(h1));
        reinterpret_cast<double2*>(ks.cent64 + i0)[e] = make_double2(v64[2 * e], v64[2 * e + 1]);
        reinterpret_cast<float2*>(ks.cent32 + i0)[e] = make_float2(v32[2 * e], v32[2 * e + 1]);
        reinterpret_cast<uint32_t*>(ks.cbf_hi + i0)[e] =
            (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
        reinterpret_cast<uint32_t*>(ks.cbf_lo + i0)[e] =
            (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
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
    // The running state of the problem in global memory: sum64[c] = the exact
    // sum of cluster c's members, counts[c] their number, dirty[c] = the last
    // round whose membership changes touched c, chg[round & 1] the tokens
    // that changed cluster in that round.
    double* sumg = ks.sum64 + cbase * D;
    int* cntg = ks.counts + cbase;
    int* dirt = ks.dirty + cbase;
    int* chgp = ks.chg + (size_t)pid * 2;
    bool fin = last;
    if (it == 0) {
      // first round: every member summed, from the grouped rows
      group();
      PHASE(4);
      // lane l holds dimensions l * VPL .. l * VPL + VPL - 1 of every sum
      const size_t pslot = ((size_t)(blk / NCT) * NCT + rank) * g.C;  // this CTA's partial row block
      for (int c = warp; c < C; c += kRW) {
        const int m0 = loff[c], n = loff[c + 1] - m0;
        double acc[VPL], acc2[VPL];
#pragma unroll
        for (int e = 0; e < VPL; ++e) acc[e] = acc2[e] = 0.0;
        // four members per step, every row load issued before the first add
        constexpr int MB = 4;
        for (int j0 = 0; j0 < n; j0 += MB) {
          float a[MB][VPL];
#pragma unroll
          for (int m = 0; m < MB; ++m) {
            if (j0 + m < n) {
              const int u = lst[m0 + j0 + m];
              row_part<D>(T + (u >> 7) * TILEB, u & (kTile - 1), lane, a[m]);
            } else {
#pragma unroll
              for (int e = 0; e < VPL; ++e) a[m][e] = 0.f;
            }
          }
#pragma unroll
          for (int m = 0; m < MB; m += 2)
#pragma unroll
            for (int e = 0; e < VPL; ++e) {
              acc[e] = __dadd_rn(acc[e], (double)a[m][e]);
              acc2[e] = __dadd_rn(acc2[e], (double)a[m + 1][e]);
            }
        }
#pragma unroll
        for (int e = 0; e < VPL; ++e) acc[e] = __dadd_rn(acc[e], acc2[e]);
        if (NCT == 1) {
          double* sr = sumg + (size_t)c * D + (size_t)lane * VPL;
#pragma unroll
          for (int e = 0; e < VPL / 2; ++e)
            reinterpret_cast<double2*>(sr)[e] = make_double2(acc[2 * e], acc[2 * e + 1]);
          if (lane == 0) {
            cntg[c] = n;
            dirt[c] = 0;
          }
          if (n > 0) write_centroid(c, n, acc);  // an empty cluster keeps its centroid
        } else {
          BADCHK(pslot / g.C < (size_t)ks.part_blocks, 5);
          if (lane == 0) rs.pcnt[set][pslot + c] = n;
          if (n > 0) {
            double* pr = rs.part[set] + (pslot + c) * D + (size_t)lane * VPL;
#pragma unroll
            for (int e = 0; e < VPL / 2; ++e)
              reinterpret_cast<double2*>(pr)[e] = make_double2(acc[2 * e], acc[2 * e + 1]);
          }
        }
      }
      __syncthreads();
      PHASE(5);
      if (NCT > 1) {
        team_sync();
        if (MODE == 2 && bar_fail) break;
        PHASE(6);
        // owners: add the problem's partial sums (exact), write centroids
        const size_t pbase = (size_t)(blk / NCT) * NCT * g.C;
        for (int c = rank + NCT * warp; c < C; c += NCT * kRW) {
          const int cnt = lane < NCT ? __ldcg(rs.pcnt[set] + pbase + (size_t)lane * g.C + c) : 0;
          double acc[VPL];
#pragma unroll
          for (int e = 0; e < VPL; ++e) acc[e] = 0.0;
          // eight ranks' rows in flight; a rank without members left no row
          for (int r0 = 0; r0 < NCT; r0 += 8) {
            double2 v[8][VPL / 2];
#pragma unroll
            for (int m = 0; m < 8; ++m) {
              const int rr = r0 + m < NCT ? r0 + m : NCT - 1;  // never past the problem's blocks
              const double* pr = rs.part[set] + (pbase + (size_t)rr * g.C + c) * D + (size_t)lane * VPL;
#pragma unroll
              for (int e = 0; e < VPL / 2; ++e)
                v[m][e] = r0 + m < NCT ? __ldcg(reinterpret_cast<const double2*>(pr) + e) : make_double2(0.0, 0.0);
            }
#pragma unroll
            for (int m = 0; m < 8; ++m) {
              const int cm = __shfl_sync(0xffffffffu, cnt, (r0 + m) & 31);
              if (r0 + m < NCT && cm > 0) {
#pragma unroll
                for (int e = 0; e < VPL / 2; ++e) {
                  acc[2 * e] = __dadd_rn(acc[2 * e], v[m][e].x);
                  acc[2 * e + 1] = __dadd_rn(acc[2 * e + 1], v[m][e].y);
                }
              }
            }
          }
          int n = cnt;
          for (int o = 16; o; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
          double* sr = sumg + (size_t)c * D + (size_t)lane * VPL;
#pragma unroll
          for (int e = 0; e < VPL / 2; ++e)
            reinterpret_cast<double2*>(sr)[e] = make_double2(acc[2 * e], acc[2 * e + 1]);
          if (lane == 0) {
            cntg[c] = n;
            dirt[c] = 0;
          }
          if (n > 0) write_centroid(c, n, acc);
        }
      }
      // the change counter of the next round starts from zero (its slot was
      // last read before the previous round's closing barrier)
      if (rank == 0 && tid == 0) chgp[1] = 0;
    } else {
      // later rounds: only the tokens that changed cluster move the sums; a
      // warp takes one such token, lane l dimensions l, l + 32, ...
      if (tid == 0) nchg_s = 0;
      __syncthreads();
      for (int u0 = 0; u0 < ntok; u0 += kRT) {
        const int u = u0 + tid;
        const bool moved = u < ntok && asg[u] != lst[u];  // lst holds the previous round's clusters
        const unsigned bal = __ballot_sync(0xffffffffu, moved);
        int slot = 0;
        if (lane == 0 && bal) slot = atomicAdd(&nchg_s, __popc(bal));
        slot = __shfl_sync(0xffffffffu, slot, 0);
        if (moved) queue[slot + __popc(bal & ((1u << lane) - 1u))] = (unsigned short)u;
      }
      __syncthreads();
      const int nmv = nchg_s;
      for (int e = warp; e < nmv; e += kRW) {
        const int u = queue[e];
        const int a = asg[u], b = lst[u];
        const unsigned char* tile = T + (u >> 7) * TILEB;
        const int r = u & (kTile - 1);
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
          const int d = lane + 32 * j, kb = d >> 6, dd = d & 63;
          const unsigned short h =
              *reinterpret_cast<const unsigned short*>(tile + kb * kTile * 128 + swz(r, dd >> 3) + (dd & 7) * 2);
          const double x = (double)__uint_as_float((uint32_t)h << 16);
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
      for (int e = tid; e < nmv; e += kRT) {
        const int u = queue[e];
        lst[u] = asg[u];
      }
      if (tid == 0 && nmv > 0) atomicAdd(chgp + (it & 1), nmv);
      PHASE_COUNT(12, nmv);
      PHASE(5);
      if (MODE == 0) {
        __threadfence();
        __syncthreads();
      } else {
        team_sync();
        if (MODE == 2 && bar_fail) break;
      }
      PHASE(6);
      // every CTA of the problem reads the same total after the barrier: no
      // token moved means the centroids are those of the previous round, and
      // every later round would repeat this one exactly
      const int moved_all = __ldcg(chgp + (it & 1));
      fin = last || moved_all == 0;
      if (rank == 0 && tid == 0) chgp[(it + 1) & 1] = 0;
      if (moved_all > 0) {
        // owners: new centroids of the clusters whose membership changed
        for (int c = rank + NCT * warp; c < C; c += NCT * kRW) {
          if (__ldcg(dirt + c) != it) continue;
          const int n = __ldcg(cntg + c);
          if (n == 0) continue;  // an empty cluster keeps its centroid
          double acc[VPL];
          const double* sr = sumg + (size_t)c * D + (size_t)lane * VPL;
#pragma unroll
          for (int e = 0; e < VPL / 2; ++e) {
            const double2 v = __ldcg(reinterpret_cast<const double2*>(sr) + e);
            acc[2 * e] = v.x;
            acc[2 * e + 1] = v.y;
          }
          write_centroid(c, n, acc);
        }
      }
    }
    __syncthreads();
    PHASE(7);
    // ---- last round: counts, offsets, the cluster-sorted permutation -----------
    if (fin) {
      PHASE_COUNT(13, it + 1);
      if (it > 0) {
        group();
        if (NCT > 1) {
          const size_t pslot = ((size_t)(blk / NCT) * NCT + rank) * g.C;
          for (int c = tid; c < C; c += kRT) rs.pcnt[set][pslot + c] = loff[c + 1] - loff[c];
          __syncthreads();
          team_sync();
          if (MODE == 2 && bar_fail) break;
        }
      }
      for (int t = tid; t < ntok; t += kRT) ks.assign[p.slot0 + tok0 + t] = asg[t];
      // members of every cluster in the problem, and in the CTAs before this one
      const size_t pbase = (size_t)(blk / NCT) * NCT * g.C;
      for (int c = tid; c < C; c += kRT) {
        int tot = 0, before = 0;
        if (NCT == 1) {
          tot = loff[c + 1] - loff[c];
        } else {
          for (int r = 0; r < NCT; ++r) {
            const int v = __ldcg(rs.pcnt[set] + pbase + (size_t)r * g.C + c);
            before += r < rank ? v : 0;
            tot += v;
          }
        }
        gtot[c] = tot;
        gbefore[c] = before;
      }
      __syncthreads();
      const int total = scan_excl(gtot, C, scan_tmp);  // gtot -> offsets
      int* offg = ks.off + (size_t)pid * (g.C + 1);
      for (int c = tid; c < C; c += kRT) {
        if (c % NCT == rank) {
          const int nxt = c + 1 < C ? gtot[c + 1] : total;
          ks.counts[cbase + c] = nxt - gtot[c];
          offg[c] = gtot[c];
        }
      }
      if (tid == 0 && rank == 0) offg[C] = total;
      // this CTA's members, in ascending token order within each cluster
      for (int c = warp; c < C; c += kRW) {
        const int m0 = loff[c], n = loff[c + 1] - m0;
        const size_t at = (size_t)p.slot0 + gtot[c] + gbefore[c];
        BADCHK(gtot[c] + gbefore[c] + n <= p.s, 4);
        for (int j = lane; j < n; j += 32) ks.perm[at + j] = tok0 + lst[m0 + j];
      }
      PHASE(8);
      break;
    }
    if (it == 0) {  // lst keeps each token's cluster of the previous round from here on
      for (int t = tid; t < ntok; t += kRT) lst[t] = asg[t];
    }
    __syncthreads();
    PHASE(8);
    team_sync();
    if (MODE == 2 && bar_fail) break;
    PHASE(9);
  }
  PHASE_FLUSH;
  // no MMA may still write the accumulators when they are freed: the MMA warp
  // waits (bounded) for the last commit of every slot of the last round
  if (warp == kEW && lane == 0 && issued > 0) {
    const int kg1 = issued;
    for (int s2 = 0; s2 < NACC && s2 < kg1; ++s2) {
      const int last_use = (kg1 - 1 - s2) / NACC;  // uses of slot s2: kg = s2 + NACC u < kg1
      mbar_wait(sa(&mma_done[s2]), (uint32_t)(last_use & 1));
    }
  }
  tc_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tbase), "r"(tcols));
}

// ----------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------
// Most tiles one CTA can hold for these sizes (0: not even one).
int resident_tpc_max(int D, int C) {
  if (C > kNCFR || (D != 64 && D != 128)) return 0;
  const int NC = (C + 31) & ~31;
  int t = 0;
  while (t < kRMaxTPC && rlayout(D, NC, t + 1).total <= kRSmemMax) ++t;
  return t;
}

// Partial-sum blocks (CTA x problem) the workspace holds for one role: per
// level, its problems times the most CTAs per problem the planner may choose
// there (enough to fill kPartSMs SMs, at least as many as the tiles need, at
// most kRMaxNCT and one per tile).
static int nct_cap(int ntp, int nprob, int tpc_max) {
  if (tpc_max < 1 || ntp < 2) return 1;
  int need = cdiv(ntp, tpc_max);
  int fill = cdiv(kPartSMs, nprob > 0 ? nprob : 1);
  int cap = need > fill ? need : fill;
  cap = cap < kRMaxNCT ? cap : kRMaxNCT;
  return cap < ntp ? cap : ntp;
}

size_t resident_partial_blocks(const Levels& lv, int BH, int D, int C) {
  const int tmax = resident_tpc_max(D, C);
  if (tmax < 4) return 0;  // the resident kernel does not serve these sizes
  size_t best = 0;
  for (int l = 0; l < lv.nlev; ++l) {
    const int nprob = BH * lv.npairs[l];
    const int cap = nct_cap(cdiv(lv.s[l], kTile), nprob, tmax);
    if (cap > 1 && (size_t)nprob * cap > best) best = (size_t)nprob * cap;
  }
  return best;
}

struct PlanEntry {
  long long key[8];
  int nct, tpc, mode;
};
std::mutex g_plan_mu;
std::vector<PlanEntry> g_plans;

template <int D>
static bool launch_resident(const RoleGeo* gs, const KState* kss, int nsets, int lvl, int iters,
                            const int* np, int nprob, int NC, int nct, int tpc, int mode,
                            int nacc, int tcols, size_t smem, cudaStream_t st);

template <int D>
static bool resident_t(const RoleGeo* gs, const KState* kss, int nsets, int lvl, int iters,
                       cudaStream_t st) {
  int cmax = 0, ntp = 1, nprob = 0, np[2] = {0, 0};
  for (int k = 0; k < nsets; ++k) {
    if (gs[k].dtype != 0 || gs[k].C > kNCFR || gs[k].D != D || kss[k].sum64 == nullptr) return false;
    const int l0 = lvl < 0 ? 0 : lvl;
    const int ce = imin(gs[k].C, gs[k].lv.s[l0]);
    cmax = cmax > ce ? cmax : ce;
    const int t = cdiv(gs[k].lv.s[l0], kTile);
    ntp = ntp > t ? ntp : t;
    np[k] = lvl < 0 ? kss[k].nprob : gs[k].BH * gs[k].lv.npairs[lvl];
    nprob += np[k];
  }
  const int NC = (cmax + 31) & ~31;
  // with fewer than four resident tiles per CTA (D = 128 with C > 128) the
  // per-round fixed costs outweigh what residency saves: the streaming kernel
  // serves those sizes
  const int tmax = resident_tpc_max(D, cmax);
  if (tmax < 4) return false;
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int nacc = NC <= 128 ? 4 : 2;
  int tcols = 32;
  while (tcols < nacc * NC) tcols <<= 1;
  const size_t per_sm = 227 * 1024;
  // shared memory of a CTA holding tpc tiles; a CTA that would share its SM
  // with others whose TMEM does not fit asks for more, one CTA per SM
  auto smem_for = [&](int tpc) {
    size_t sm = rlayout(D, NC, tpc).total;
    if ((per_sm / (sm + 4096)) * (size_t)tcols > 512) sm = per_sm / 2 + 1024;
    return sm;
  };
  // plans are cached per device and sizes: the occupancy queries cost host time
  const long long key[8] = {dev, D, NC, ntp, np[0], np[1], (long long)kss[0].part_blocks,
                            nsets > 1 ? (long long)kss[1].part_blocks : -1};
  {
    std::lock_guard<std::mutex> lock(g_plan_mu);
    for (const auto& e : g_plans)
      if (std::equal(key, key + 8, e.key)) {
        if (e.nct == 0) return false;
        return launch_resident<D>(gs, kss, nsets, lvl, iters, np, nprob, NC, e.nct, e.tpc, e.mode,
                                  nacc, tcols, smem_for(e.tpc), st);
      }
  }
  // Candidates: every CTA count per problem from what the tiles need up to
  // kRMaxNCT (none idle, within the workspace's partial-sum blocks), as one
  // thread-block cluster per problem or as one cooperative launch (every CTA
  // resident at once).  Cost: the waves of problems the GPU runs at once
  // times the tiles per CTA plus a per-round fixed cost of about four tiles
  // (five with the slower global-memory barrier).
  int best_nct = 0, best_tpc = 0, best_mode = 0;
  long long best_cost = 0;
  auto consider = [&](int nct, int tpc, int mode, long long cost) {
    if (best_nct == 0 || cost < best_cost) {
      best_nct = nct;
      best_tpc = tpc;
      best_mode = mode;
      best_cost = cost;
    }
  };
  for (int cand = cdiv(ntp, tmax); cand <= kRMaxNCT && cand <= ntp; ++cand) {
    const int tpc = cdiv(ntp, cand), nct = cdiv(ntp, tpc);
    if (nct != cand) continue;  // the same split as a smaller count
    bool fits = true;
    for (int k = 0; k < nsets; ++k)
      if (nct > 1 && (size_t)np[k] * nct > kss[k].part_blocks) fits = false;
    if (!fits) continue;
    const size_t sm = smem_for(tpc);
    if (nct == 1) {
      auto kfn = kmeans_resident_kernel<D, 0>;
      cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      int per = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, kfn, kRT, sm) == cudaSuccess && per > 0)
        consider(1, tpc, 0, (long long)cdiv(nprob, per * nsm) * (tpc + 4));
      cudaGetLastError();
      continue;
    }
    {  // thread-block clusters
      auto kfn = kmeans_resident_kernel<D, 1>;
      cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      bool ok = nct <= 8 ||
                cudaFuncSetAttribute(kfn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3((unsigned)(nprob * nct));
      q.blockDim = dim3(kRT);
      q.dynamicSmemBytes = sm;
      cudaLaunchAttribute qa[1];
      qa[0].id = cudaLaunchAttributeClusterDimension;
      qa[0].val.clusterDim.x = nct;
      qa[0].val.clusterDim.y = 1;
      qa[0].val.clusterDim.z = 1;
      q.attrs = qa;
      q.numAttrs = 1;
      int active = 0;
      if (ok && cudaOccupancyMaxActiveClusters(&active, kfn, &q) == cudaSuccess && active > 0)
        consider(nct, tpc, 1, (long long)cdiv(nprob, active) * (tpc + 4));
      cudaGetLastError();
    }
    {  // cooperative: only when every CTA of the launch is resident at once
      auto kfn = kmeans_resident_kernel<D, 2>;
      cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      int per = 0, coop = 0;
      cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
      if (coop && cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, kfn, kRT, sm) == cudaSuccess &&
          (long long)per * nsm >= (long long)nprob * nct)
        consider(nct, tpc, 2, tpc + 5);
      cudaGetLastError();
    }
  }
  {
    std::lock_guard<std::mutex> lock(g_plan_mu);
    if (g_plans.size() > 256) g_plans.clear();
    PlanEntry pe;
    std::copy(key, key + 8, pe.key);
    pe.nct = best_nct;
    pe.tpc = best_tpc;
    pe.mode = best_mode;
    g_plans.push_back(pe);
  }
  if (best_nct == 0) return false;
#ifdef MUSE_PHASE_CLOCKS
  fprintf(stderr, "resident plan: lvl %d nprob %d nct %d tpc %d mode %d nacc %d tcols %d cost %lld\n",
          lvl, nprob, best_nct, best_tpc, best_mode, nacc, tcols, best_cost);
#endif
  return launch_resident<D>(gs, kss, nsets, lvl, iters, np, nprob, NC, best_nct, best_tpc,
                            best_mode, nacc, tcols, smem_for(best_tpc), st);
}

template <int D>
static bool launch_resident(const RoleGeo* gs, const KState* kss, int nsets, int lvl, int iters,
                            const int* np, int nprob, int NC, int nct, int tpc, int mode,
                            int nacc, int tcols, size_t smem, cudaStream_t st) {
  ResidentSets rs{};
  for (int k = 0; k < nsets; ++k) {
    rs.g[k] = gs[k];
    rs.ks[k] = kss[k];
    rs.part[k] = kss[k].part;
    rs.pcnt[k] = kss[k].pcnt;
  }
  rs.lvl = lvl;
  rs.nblk0 = np[0] * nct;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(nprob * nct));
  cfg.blockDim = dim3(kRT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  if (mode == 1) {
    auto kfn = kmeans_resident_kernel<D, 1>;
    cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (nct > 8) cudaFuncSetAttribute(kfn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = nct;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kfn, rs, iters, nct, NC, tpc, nacc, tcols);
  } else if (mode == 2) {
    auto kfn = kmeans_resident_kernel<D, 2>;
    cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kfn, rs, iters, nct, NC, tpc, nacc, tcols);
  } else {
    auto kfn = kmeans_resident_kernel<D, 0>;
    cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaLaunchKernelEx(&cfg, kfn, rs, iters, nct, NC, tpc, nacc, tcols);
  }
  return true;
}

#ifdef MUSE_PHASE_CLOCKS
extern "C" void muse_phase_read(long long* out, int rows) {
  cudaMemcpyFromSymbol(out, g_phase_clk, (size_t)rows * kPhaseSlots * sizeof(long long));
}
extern "C" void muse_bad_read(int* out) { cudaMemcpyFromSymbol(out, g_bad, sizeof(g_bad)); }
extern "C" void muse_phase_clear(void) {
  static long long zero[8192][kPhaseSlots];
  cudaMemcpyToSymbol(g_phase_clk, zero, sizeof(zero));
}
#endif

bool launch_kmeans_resident(const RoleGeo* gs, const KState* kss, int nsets, int lvl, int iters,
                            cudaStream_t st) {
  return gs[0].D == 64 ? resident_t<64>(gs, kss, nsets, lvl, iters, st)
                       : resident_t<128>(gs, kss, nsets, lvl, iters, st);
}

}  // namespace muse
