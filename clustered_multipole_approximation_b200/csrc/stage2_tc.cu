// Stage 2 of MuSe on the fifth-generation tensor cores (tcgen05, TMEM) for
// bf16 inputs, at the levels whose query clusters hold many queries.
//
// For the queries of query cluster i (gist.science page "Multipole Semantic
// Attention: A Fast Approximation of Softmax Attention for Pretraining",
// Technical Summary, Core Mechanisms: Stage 2 (Refinement), Exact Attention)
// one online softmax runs over the far field -- one row per non-retrieved
// non-empty key cluster j: key row mu_j (TILTED: k_hat_ij) as a bf16 hi + lo
// pair, logit offset fbias_ij, value u_ij as an fp16 hi + lo pair -- and over
// every key of the retrieved clusters, exactly (bf16 k, fp16 v).
//
// One CTA of 128 threads takes a tile of up to 128 queries of one cluster;
// thread t owns query row t, which is TMEM lane t.  Per block of 64 key rows:
//   S = Q K^T        tcgen05.mma M=128, N=64, bf16, fp32 accumulator in TMEM
//                    (two S buffers: S of block b+1 runs during the softmax of b);
//   P = 2^(s log2e S + bias - m)   thread t, from its TMEM lane; written to
//                    shared memory as the fp16 A operand (far rows: hi + lo);
//   O += P V         tcgen05.mma M=128, N=D, fp16, V MN-major, O in TMEM for
//                    the whole tile.
// The row maximum m is a reference that moves only when a block's logits
// exceed it by more than 8 (base 2): P stays below 2^8, and O is rescaled in
// TMEM on those rare moves only.
//
// The retrieved keys arrive without a gather: permute_keys_kernel writes, per
// key problem, K and V (fp16) in cluster-sorted order with every cluster
// padded to whole groups of 8 rows, each group stored in the 128-byte-swizzled
// form of the MMA operand ([64-dimension chunk][8 rows][128 B] per cluster).
// A key block is then 8 groups from the query cluster's retrieved clusters,
// each run of groups one bulk copy (cp.async.bulk, completion counted on an
// mbarrier) per chunk, three blocks in flight.  The far-field tables are read
// with cp.async (two blocks of 64 at 128 or 256 clusters).
#include <cuda_fp16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"

namespace muse {

namespace {

constexpr int kTQ = 128;      // query rows per CTA (TMEM lanes, one thread each)
constexpr int kTK = 64;       // key rows per block
constexpr int kTC = 256;      // softmax threads: two per query row, each half the columns
constexpr int kTT = kTC + 64;  // threads: + an MMA warp and a load warp
constexpr int kTMaxSel = 64;  // retrieved clusters per query cluster
constexpr int kTStages = 3;   // key blocks in flight
constexpr float kLazy = 8.f;  // headroom (base 2) of the reference maximum

__device__ inline uint32_t s32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ inline uint32_t swz(int r, int q) { return r * 128 + ((q ^ (r & 7)) << 4); }
// K-major operand, 128-byte swizzle, 8-row groups 1 KB apart
__device__ inline uint64_t desc_k(uint32_t a) {
  return (uint64_t)((a >> 4) & 0x3FFF) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}
// MN-major operand, 128-byte swizzle: lbo = bytes between 64-element column chunks
__device__ inline uint64_t desc_mn(uint32_t a, uint32_t lbo) {
  return (uint64_t)((a >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}
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
__device__ inline void mbar_expect_tx(uint32_t mbar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}\n" ::"r"(
                   mbar),
               "r"(bytes)
               : "memory");
}
// Bounded wait for the phase of this parity; false when it gave up.
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
// Contiguous bytes global -> shared (16-byte aligned, a multiple of 16 bytes).
__device__ inline void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(mbar)
      : "memory");
}
__device__ inline void tld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ inline void tst16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
// The wait for this thread's TMEM loads, tied to their registers so that no
// use of them moves above it.
__device__ inline void tld_wait(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
                 "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}
__device__ inline void tld_wait2(uint32_t (&r)[2][16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n"
               : "+r"(r[0][0]), "+r"(r[0][1]), "+r"(r[0][2]), "+r"(r[0][3]), "+r"(r[0][4]), "+r"(r[0][5]),
                 "+r"(r[0][6]), "+r"(r[0][7]), "+r"(r[0][8]), "+r"(r[0][9]), "+r"(r[0][10]),
                 "+r"(r[0][11]), "+r"(r[0][12]), "+r"(r[0][13]), "+r"(r[0][14]), "+r"(r[0][15]),
                 "+r"(r[1][0]), "+r"(r[1][1]), "+r"(r[1][2]), "+r"(r[1][3]), "+r"(r[1][4]), "+r"(r[1][5]),
                 "+r"(r[1][6]), "+r"(r[1][7]), "+r"(r[1][8]), "+r"(r[1][9]), "+r"(r[1][10]),
                 "+r"(r[1][11]), "+r"(r[1][12]), "+r"(r[1][13]), "+r"(r[1][14]), "+r"(r[1][15])
               :
               : "memory");
}
__device__ inline void tst_wait() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }
__device__ inline void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ inline void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ inline void fence_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
__device__ inline void cp16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes));
}
__device__ inline void cp_commit_wait() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
}
__device__ inline uint32_t h2bits(float x, float y) {
  const __half2 h = __floats2half2_rn(x, y);
  return *reinterpret_cast<const uint32_t*>(&h);
}
// fp16 pair (x, y) = hi + lo
__device__ inline void split_h2bits(float x, float y, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(x, y);
  const float2 f = __half22float2(h);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = h2bits(x - f.x, y - f.y);
}

// Shared-memory plan of one CTA (bytes from a 1 KB-aligned base).
template <int D>
struct TcL {
  static constexpr int KB = D / 64;
  static constexpr int QC = kTQ * 128;          // one 64-dimension chunk of Q (or P)
  static constexpr int KC = kTK * 128;          // one 64-dimension chunk of a key block
  static constexpr int Q = 0;                   // [KB][128 rows][128 B], K-major
  static constexpr int STG = Q + KB * QC;       // stage s: K at STG + s SS, V after it
  static constexpr int SS = 2 * KB * KC;
  static constexpr int P = STG + kTStages * SS;  // P hi: [128 rows][64 fp16], K-major
  static constexpr int PL = P + QC;             // P lo (far rows)
  static constexpr int MAXB = 256;              // exact blocks with a precomputed key-slot mask
  static constexpr int BM = PL + QC;
  static constexpr int TOTAL = BM + MAXB * 8 + 1024;
};

// Exclusive scan of n <= 2 * kTT ints in shared memory by the whole CTA;
// returns the total.
__device__ inline int cta_scan(int* a, int n, int* tmp) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
  for (int w = 0; w < kTT / 32; ++w) {
    if (w < warp) wbase += tmp[w];
    total += tmp[w];
  }
  const int excl = wbase + x - (v0 + v1);
  if (i0 < n) a[i0] = excl;
  if (i1 < n) a[i1] = excl + v0;
  __syncthreads();
  return total;
}

}  // namespace

// First group (of 8 rows, KB x 1 KB each) of key problem kpid in the sorted
// copies: its token slots plus up to one padding group per cluster before it.
__device__ inline long long key_group_base(const AttnArgs& a, const Prob& pk, int kpid) {
  return pk.slot0 / 8 + (long long)a.Ck * kpid;
}

// Cluster-sorted, group-padded, pre-swizzled copies of K (bf16) and V (fp16)
// of the key problems at the levels in a.tc_lv; CTA (x, y) copies groups
// [y kPermGroups, (y + 1) kPermGroups) of key problem x.
constexpr int kPermGroups = 32;

template <int D>
__global__ void __launch_bounds__(256) permute_keys_kernel(AttnArgs a) {
  constexpr int KB = D / 64;
  const int kpid = blockIdx.x;
  const Prob pk = prob_of(a.kg, kpid);
  if (!((a.tc_lv >> pk.level) & 1)) return;
  const int C = pk.C, Ck = a.Ck, tid = threadIdx.x;
  const int* kc = a.ks.counts + (size_t)kpid * Ck;
  const int* koff = a.ks.off + (size_t)kpid * (Ck + 1);
  const int* kperm = a.ks.perm + pk.slot0;
  if ((long long)blockIdx.y * kPermGroups >= (long long)pk.s / 8 + C) return;  // past any group
  __shared__ int sg[257];
  __shared__ int tmp[8];
  for (int j = tid; j <= C; j += 256) sg[j] = j < C ? (kc[j] + 7) / 8 : 0;
  __syncthreads();
  // exclusive scan of the groups per cluster (C + 1 <= 257 entries)
  {
    const int lane = tid & 31, warp = tid >> 5;
    const int i0 = 2 * tid, i1 = 2 * tid + 1;
    const int v0 = i0 <= C ? sg[i0] : 0, v1 = i1 <= C ? sg[i1] : 0;
    int x = v0 + v1;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) tmp[warp] = x;
    __syncthreads();
    int wbase = 0;
    for (int w = 0; w < warp; ++w) wbase += tmp[w];
    const int excl = wbase + x - (v0 + v1);
    __syncthreads();
    if (i0 <= C) sg[i0] = excl;
    if (i1 <= C) sg[i1] = excl + v0;
    __syncthreads();
  }
  if (blockIdx.y == 0) {
    int* gofs = a.gofs + (size_t)kpid * (Ck + 1);
    for (int j = tid; j <= C; j += 256) gofs[j] = sg[j];
  }
  const long long pb = key_group_base(a, pk, kpid);
  const int TG = sg[C];
  const int gbeg = blockIdx.y * kPermGroups, gend = imin(TG, gbeg + kPermGroups);
  const __nv_bfloat16* K = static_cast<const __nv_bfloat16*>(a.kg.X);
  uint4* kd = reinterpret_cast<uint4*>(a.kpad);
  uint4* vd = reinterpret_cast<uint4*>(a.vpad);
  // one 16-byte piece per step: (group, row, chunk)
  for (int e = tid; e < (gend - gbeg) * 8 * KB * 8; e += 256) {
    const int c = e & 7, kb = (e >> 3) % KB;
    const int gr = (e >> 3) / KB;  // group * 8 + row, from gbeg
    const int gi = gbeg + (gr >> 3), r = gr & 7;
    int lo = 0, hi = C - 1;  // the cluster of group gi
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sg[mid] <= gi) lo = mid;
      else hi = mid - 1;
    }
    const int j = lo, g = gi - sg[j], ng = sg[j + 1] - sg[j];
    const int row = 8 * g + r;
    const bool live = row < kc[j];
    const long long dst = (((pb + sg[j]) * KB + (long long)kb * ng + g) * 1024 + swz(r, c)) / 16;
    uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
    if (live) {
      const long long src = (pk.row0 + kperm[koff[j] + row]) * D + kb * 64 + c * 8;
      kv = __ldg(reinterpret_cast<const uint4*>(K + src));
      vv = __ldg(reinterpret_cast<const uint4*>(a.V16 + src));
    }
    kd[dst] = kv;
    vd[dst] = vv;
  }
}

template <typename TO, int D>
__global__ void __launch_bounds__(kTT, D == 64 ? 2 : 1) stage2_tc_kernel(AttnArgs a, Stage1 s1, int qp0) {
  constexpr int HK = kTK / 2;  // columns of a block per softmax thread
  constexpr int HD = D / 2;    // O columns per softmax thread
  using Lt = TcL<D>;
  constexpr int KB = Lt::KB;
  extern __shared__ __align__(1024) unsigned char tc_raw[];
  unsigned char* sm = tc_raw + ((1024 - (s32(tc_raw) & 1023)) & 1023);
  const uint32_t sb = s32(sm);
  unsigned long long* bmask = reinterpret_cast<unsigned long long*>(sm + Lt::BM);
  // exact blocks: loads done (tx bytes), S done, S read, P written, P V done
  __shared__ __align__(8) uint64_t mLd[kTStages], mEmpty[kTStages], mS[2], mSfree[2], mP, mPV;
  __shared__ uint32_t tslot;
  __shared__ int tpre[257];
  __shared__ int stmp[kTT / 32];
  __shared__ int jsel[kTMaxSel], jng[kTMaxSel], jgof[kTMaxSel], jn[kTMaxSel];
  __shared__ int gpre[kTMaxSel + 1];
  __shared__ float fbs[kTK];
  // the two halves of a row exchange partial maxima (then sums) here, in a
  // buffer that alternates between steps: a half writes step n + 2's value
  // only after both passed step n + 1's barrier, so after the read of step n
  __shared__ float xch[2][2][kTQ];

  const int lq = blockIdx.x, qpid = qp0 + lq;
  const Prob pq = prob_of(a.qg, qpid);
  if (!((a.tc_lv >> pq.level) & 1)) return;
  const int Cq = a.Cq, Ck = a.Ck, cq = pq.C;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // warps 0-7 softmax: row (warp % 4) 32 + lane (its TMEM lane), column half
  // warp / 4; warp 8 issues the MMAs, warp 9 the loads
  const bool consumer = warp < kTC / 32;
  const int row = tid & (kTQ - 1), hc = (warp >> 2) & 1;
  const int kIssue = kTC;  // the MMA warp's lane 0

  // ---- this CTA's tile: cluster i, queries [r0, r0 + nq) of it ----------------
  const int* qcnt = a.qs.counts + (size_t)qpid * Cq;
  for (int c = tid; c < cq; c += kTT) tpre[c] = (qcnt[c] + kTQ - 1) / kTQ;
  __syncthreads();
  const int ntile = cta_scan(tpre, cq, stmp);
  const int tile = blockIdx.y;
  if (tile >= ntile) return;
  int lo = 0, hi = cq - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tpre[mid] <= tile) lo = mid;
    else hi = mid - 1;
  }
  const int i = lo;
  const int r0 = (tile - tpre[i]) * kTQ;
  const int nq = imin(kTQ, qcnt[i] - r0);

  const int kpid = kv_problem(a, qpid);
  const Prob pk = prob_of(a.kg, kpid);
  const int* kc = a.ks.counts + (size_t)kpid * Ck;
  const int nsel = a.topk > 0 ? s1.nsel[(size_t)qpid * Cq + i] : 0;
  const int* gofs = a.gofs + (size_t)kpid * (Ck + 1);
  for (int r = tid; r < nsel; r += kTT) {
    const int j = s1.sel[((size_t)qpid * Cq + i) * a.topk + r];
    jsel[r] = j;
    jn[r] = kc[j];
    jgof[r] = gofs[j];
    jng[r] = gofs[j + 1] - gofs[j];
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int r = 0; r < nsel; ++r) {
      gpre[r] = run;
      run += jng[r];
    }
    gpre[nsel] = run;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 256;\n" ::"r"(s32(&tslot)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
  }
  if (tid == kIssue) {
    for (int s = 0; s < kTStages; ++s) {
      mbar_init(s32(&mLd[s]), 1);
      mbar_init(s32(&mEmpty[s]), 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(s32(&mS[k]), 1);
      mbar_init(s32(&mSfree[k]), kTC / 32);
    }
    mbar_init(s32(&mP), kTC / 32);
    mbar_init(s32(&mPV), 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n");
  }
  // the query rows (rows past nq zero); the third key stage zero (the far
  // field fills the first two): a block's unused slots then hold finite rows
  const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(a.qg.X);
  const int qo = a.qs.off[(size_t)qpid * (Cq + 1) + i];
  const int* qperm = a.qs.perm + pq.slot0;
  for (int e = tid; e < kTQ * KB * 8; e += kTT) {
    const int r = e / (KB * 8), q = e - r * (KB * 8), kb = q >> 3, c = q & 7;
    const bool live = r < nq;
    const long long row = pq.row0 + (live ? qperm[qo + r0 + r] : 0);
    cp16(sb + Lt::Q + kb * Lt::QC + swz(r, c), Q + row * D + kb * 64 + c * 8, live ? 16 : 0);
  }
  for (int e = tid; e < Lt::SS / 16; e += kTT)
    *reinterpret_cast<uint4*>(sm + Lt::STG + 2 * Lt::SS + 16 * e) = make_uint4(0, 0, 0, 0);
  cp_commit_wait();
  fence_async();
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tbase = tslot;
  const uint32_t tS[2] = {tbase, tbase + (uint32_t)kTK};
  const uint32_t tO = tbase + 2u * kTK;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  // S: f32 accumulator, bf16 A (queries) and B (keys), both K-major, N = 64
  const uint32_t id_s = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kTK >> 3) << 17) |
                        ((uint32_t)(kTQ >> 4) << 24);
  // P V: f32 accumulator, f16 A = P (K-major) and B = V (MN-major), N = D
  const uint32_t id_pv = (1u << 4) | (1u << 16) | ((uint32_t)(D >> 3) << 17) |
                         ((uint32_t)(kTQ >> 4) << 24);
  const float sl2 = a.scale * 1.4426950408889634f;  // logits in base-2 units
  const int TG = gpre[nsel];  // groups of 8 rows of the retrieved clusters
  const int nblk = (TG + 7) / 8;
  // key slot 8 q + r of exact block b is row r of group 8 b + q of the
  // concatenated retrieved clusters: live when the cluster has that row
  auto block_mask = [&](int b, int& rc) {
    unsigned long long m = 0;
    for (int q = 0; q < 8; ++q) {
      const int G = 8 * b + q;
      if (G >= TG) break;
      while (gpre[rc + 1] <= G) ++rc;
      const int rows = jn[rc] - 8 * (G - gpre[rc]);
      m |= (rows >= 8 ? 0xFFull : ((1ull << rows) - 1ull)) << (8 * q);
    }
    return m;
  };
  for (int b = tid; b < nblk && b < Lt::MAXB; b += kTT) {
    int rc = 0;
    bmask[b] = block_mask(b, rc);
  }
  __syncthreads();
  bool ok = true;
  int uS[2] = {0, 0}, uSf[2] = {0, 0}, uP = 0, uPV = 0, uLd[kTStages] = {0, 0, 0};
  bool o_init = false;  // some P V has written O
  float mref = kMaxFloor, lsum = 0.f;
  int xstep = 0;  // exchanges made (the same count in both halves of a row)

  auto wait_on = [&](uint64_t& bar, int& use) {
    ok = mbar_wait(s32(&bar), (uint32_t)(use & 1)) && ok;
    ++use;
  };
  auto issue_S = [&](int k, uint32_t kaddr, uint32_t kloaddr) {  // one thread
    for (int kb = 0; kb < KB; ++kb) {
      const uint64_t ad = desc_k(sb + Lt::Q + kb * Lt::QC);
      const uint64_t bd = desc_k(kaddr + kb * Lt::KC);
#pragma unroll
      for (int q = 0; q < 4; ++q) umma(tS[k], ad + 2 * q, bd + 2 * q, id_s, (kb | q) ? 1u : 0u);
      if (kloaddr) {
        const uint64_t bl = desc_k(kloaddr + kb * Lt::KC);
#pragma unroll
        for (int q = 0; q < 4; ++q) umma(tS[k], ad + 2 * q, bl + 2 * q, id_s, 1u);
      }
    }
    umma_commit(s32(&mS[k]));
  };
  auto issue_PV = [&](uint32_t vaddr, uint32_t vloaddr, bool plo) {  // one thread
#pragma unroll
    for (int q = 0; q < kTK / 16; ++q) {
      const uint64_t pd = desc_k(sb + Lt::P) + 2 * q;
      const uint64_t vd = desc_mn(vaddr + 2048 * q, Lt::KC);
      umma(tO, pd, vd, id_pv, (o_init || q > 0) ? 1u : 0u);
      if (plo) umma(tO, desc_k(sb + Lt::PL) + 2 * q, vd, id_pv, 1u);
      if (vloaddr) umma(tO, pd, desc_mn(vloaddr + 2048 * q, Lt::KC), id_pv, 1u);
    }
    umma_commit(s32(&mPV));
  };
  // Consumer step on S buffer k: logits (base 2, bias per column from
  // `biasf`), the reference-maximum step, O rescale when it moves, P (hi, and
  // lo when far) into shared memory.  `wait_pv`: a P V is still running (P and
  // O are touched only after it).  `sfree`: report the S buffer read.
  // Exact blocks with a positive scale keep the raw scores (masked slots
  // -inf, applied per 8-slot group only where a group is partial) and fold
  // the scale into the exponent; far blocks and other scales form the
  // logits with their bias first.
  auto softmax = [&](int k, auto biasf, unsigned long long emask, bool far, bool wait_pv, bool sfree) {
    const bool raw = !far && sl2 > 0.f;
    float p[HK];
    float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    {  // this thread's 32 scores of the row: two loads in flight, one wait
      uint32_t r[2][16];
#pragma unroll
      for (int q = 0; q < 2; ++q) tld16(tS[k] + lane_off + (uint32_t)(HK * hc + 16 * q), r[q]);
      tld_wait2(r);
      if (raw) {
#pragma unroll
        for (int c = 0; c < HK; ++c) p[c] = __uint_as_float(r[c >> 4][c & 15]);
        const unsigned hm = (unsigned)(emask >> (HK * hc));
#pragma unroll
        for (int q = 0; q < HK / 8; ++q) {
          const unsigned g = (hm >> (8 * q)) & 0xFFu;
          if (g != 0xFFu) {
#pragma unroll
            for (int e = 0; e < 8; ++e)
              if (!((g >> e) & 1u)) p[8 * q + e] = -INFINITY;
          }
        }
#pragma unroll
        for (int c = 0; c < HK; ++c) mx4[c & 3] = fmaxf(mx4[c & 3], p[c]);
      } else {
#pragma unroll
        for (int c = 0; c < HK; ++c) {
          const float lg = fmaf(sl2, __uint_as_float(r[c >> 4][c & 15]), biasf(HK * hc + c));
          p[c] = lg;
          mx4[c & 3] = fmaxf(mx4[c & 3], lg);
        }
      }
    }
    if (sfree) {
      fence_before();
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(s32(&mSfree[k])) : "memory");
    }
    // the row's maximum over both halves (the two threads of a row meet at a
    // named barrier of their 64 threads)
    float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
    xch[xstep & 1][hc][row] = mx;
    asm volatile("bar.sync %0, 64;\n" ::"r"(1 + (warp & 3)) : "memory");
    mx = fmaxf(mx, xch[xstep & 1][hc ^ 1][row]);
    ++xstep;
    if (raw) mx *= sl2;
    const bool move = mx > mref + kLazy;
    const float mnew = move ? mx : mref;
    const float scale = move ? fast_exp2(mref - mnew) : 1.f;
    float rs4[4] = {0.f, 0.f, 0.f, 0.f};
    if (raw) {
#pragma unroll
      for (int c = 0; c < HK; ++c) {
        const float v = fast_exp2(fmaf(sl2, p[c], -mnew));
        p[c] = v;
        rs4[c & 3] += v;
      }
    } else {
#pragma unroll
      for (int c = 0; c < HK; ++c) {
        const float v = fast_exp2(p[c] - mnew);
        p[c] = v;
        rs4[c & 3] += v;
      }
    }
    lsum = lsum * scale + ((rs4[0] + rs4[1]) + (rs4[2] + rs4[3]));  // this half's share
    mref = mnew;
    if (wait_pv) {  // P and O are free once the previous P V is done
      wait_on(mPV, uPV);
      fence_after();
    }
    if (o_init && __any_sync(0xffffffffu, move)) {  // each half rescales half of O's columns
#pragma unroll
      for (int d0 = 0; d0 < HD; d0 += 16) {
        uint32_t r[16];
        tld16(tO + lane_off + (uint32_t)(HD * hc + d0), r);
        tld_wait(r);
#pragma unroll
        for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * scale);
        tst16(tO + lane_off + (uint32_t)(HD * hc + d0), r);
      }
      tst_wait();
    }
#pragma unroll
    for (int c = 0; c < HK / 8; ++c) {  // 16-byte pieces 4 hc + c of the row
      uint32_t hv[4], lv[4];
      if (far) {
#pragma unroll
        for (int u = 0; u < 4; ++u) split_h2bits(p[8 * c + 2 * u], p[8 * c + 2 * u + 1], hv[u], lv[u]);
        *reinterpret_cast<uint4*>(sm + Lt::PL + swz(row, 4 * hc + c)) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) hv[u] = h2bits(p[8 * c + 2 * u], p[8 * c + 2 * u + 1]);
      }
      *reinterpret_cast<uint4*>(sm + Lt::P + swz(row, 4 * hc + c)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
    }
    fence_async();
    fence_before();
  };

  // ---- far field: blocks of 64 key clusters, retrieved / empty ones masked ----
  // (every thread; the tables are plain rows, staged with cp.async)
  const size_t ij0 = ((size_t)lq * Cq + i) * Ck;
  const bool tilted = a.mode == 2;
  const __nv_bfloat16* khi = tilted ? s1.Kfh + ij0 * D : a.ks.cbf_hi + (size_t)kpid * Ck * D;
  const __nv_bfloat16* klo = tilted ? s1.Kfl + ij0 * D : a.ks.cbf_lo + (size_t)kpid * Ck * D;
  const __half* uh = s1.Uh + ij0 * D;
  const __half* ul = s1.Ul + ij0 * D;
  const uint32_t st0K = sb + Lt::STG, st0V = st0K + KB * Lt::KC;
  const uint32_t st1K = sb + Lt::STG + Lt::SS, st1V = st1K + KB * Lt::KC;
  for (int j0 = 0; j0 < pk.C; j0 += kTK) {
    // far row j0 + r: a non-empty cluster outside R_i; other rows are zero
    // (an empty or retrieved cluster's table rows need not hold numbers)
    if (tid < kTK) {
      const int j = j0 + tid;
      bool fl = j < pk.C && kc[j] > 0;
      for (int r = 0; r < nsel && fl; ++r) fl = jsel[r] != j;
      fbs[tid] = fl ? s1.fbias[ij0 + j] * 1.4426950408889634f : -INFINITY;
    }
    __syncthreads();
    for (int e = tid; e < kTK * KB * 8; e += kTT) {
      const int r = e / (KB * 8), q = e - r * (KB * 8), kb = q >> 3, c = q & 7;
      const bool live = fbs[r] != -INFINITY;
      const size_t off = (size_t)(live ? j0 + r : 0) * D + kb * 64 + c * 8;
      const uint32_t so = kb * Lt::KC + swz(r, c);
      const int nb = live ? 16 : 0;
      cp16(st0K + so, khi + off, nb);
      cp16(st1K + so, klo + off, nb);
      cp16(st0V + so, uh + off, nb);
      cp16(st1V + so, ul + off, nb);
    }
    cp_commit_wait();
    fence_async();
    fence_before();
    __syncthreads();
    fence_after();
    if (tid == kIssue) issue_S(0, st0K, st1K);
    if (consumer) {
      wait_on(mS[0], uS[0]);
      fence_after();
      softmax(0, [&](int c) { return fbs[c]; }, 0ull, true, false, false);
    }
    __syncthreads();
    fence_after();
    if (tid == kIssue) issue_PV(st0V, st1V, true);
    o_init = true;
    wait_on(mPV, uPV);  // the stages and P are reloaded next
    fence_after();
  }

  // ---- exact retrieval: blocks of 8 groups of the retrieved clusters ----------
  const long long pb = key_group_base(a, pk, kpid);
  const unsigned char* kpad = static_cast<const unsigned char*>(a.kpad);
  const unsigned char* vpad = static_cast<const unsigned char*>(a.vpad);
  auto stage_K = [&](int b) { return sb + Lt::STG + (b % kTStages) * Lt::SS; };
  if (!consumer) {
    if (lane == 0) {
      // block b's groups into stage b % 3: a run of one cluster's groups is one
      // copy per 64-dimension chunk and tensor
      auto issue_load = [&](int b) {
        const int s = b % kTStages;
        const uint32_t dK = stage_K(b), dV = dK + KB * Lt::KC;
        const int g0 = 8 * b, g1 = imin(TG, g0 + 8);
        mbar_expect_tx(s32(&mLd[s]), (uint32_t)(g1 - g0) * 2048u * KB);
        int r = 0;
        for (int gs = g0; gs < g1;) {
          while (gpre[r + 1] <= gs) ++r;
          const int gl = gs - gpre[r];
          const int cnt = imin(g1, gpre[r + 1]) - gs;
          const int slot = gs - g0;
          for (int kb = 0; kb < KB; ++kb) {
            const long long src = ((pb + jgof[r]) * KB + (long long)kb * jng[r] + gl) * 1024;
            bulk_g2s(dK + kb * Lt::KC + slot * 1024, kpad + src, (uint32_t)cnt * 1024u, s32(&mLd[s]));
            bulk_g2s(dV + kb * Lt::KC + slot * 1024, vpad + src, (uint32_t)cnt * 1024u, s32(&mLd[s]));
          }
          gs += cnt;
        }
      };
      if (warp == kTC / 32 + 1) {
        // the load warp: a stage is refilled once the P V of its block is done
        int uE[kTStages] = {0, 0, 0};
        for (int b = 0; b < nblk; ++b) {
          const int s = b % kTStages;
          if (b >= kTStages) wait_on(mEmpty[s], uE[s]);
          issue_load(b);
        }
      } else {
        // the MMA warp: S of block b as soon as its keys and an S buffer are
        // there, then P V of block b - 1 once the consumers wrote P
        for (int b = 0; b < nblk; ++b) {
          wait_on(mLd[b % kTStages], uLd[b % kTStages]);
          if (b >= 2) wait_on(mSfree[b & 1], uSf[b & 1]);  // consumers are done with S(b - 2)
          fence_after();
          issue_S(b & 1, stage_K(b), 0);
          if (b >= 1) {
            wait_on(mP, uP);  // P(b - 1) written
            fence_after();
            issue_PV(stage_K(b - 1) + KB * Lt::KC, 0, false);
            umma_commit(s32(&mEmpty[(b - 1) % kTStages]));
            o_init = true;
          }
        }
        if (nblk > 0) {
          wait_on(mP, uP);
          fence_after();
          issue_PV(stage_K(nblk - 1) + KB * Lt::KC, 0, false);
          umma_commit(s32(&mEmpty[(nblk - 1) % kTStages]));
        }
      }
    }
  } else {
    int rc = 0;  // the retrieved cluster of the current group (blocks past the table)
    for (int b = 0; b < nblk; ++b) {
      const unsigned long long m = b < Lt::MAXB ? bmask[b] : block_mask(b, rc);
      wait_on(mS[b & 1], uS[b & 1]);
      fence_after();
      softmax(b & 1, [&](int c) { return (m >> c) & 1ull ? 0.f : -INFINITY; }, m, false, b > 0, true);
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(s32(&mP)) : "memory");
    }
    if (nblk > 0) {
      wait_on(mPV, uPV);
      fence_after();
    }
  }

  // ---- the tile's rows: normalised output (or level partial), exact counts ----
  if (consumer) {
    int nexact = 0;
    for (int r = 0; r < nsel; ++r) nexact += jn[r];
    xch[xstep & 1][hc][row] = lsum;  // the row's sum over both halves
    asm volatile("bar.sync %0, 64;\n" ::"r"(1 + (warp & 3)) : "memory");
    const float ltot = lsum + xch[xstep & 1][hc ^ 1][row];
    const bool live = row < nq;
    const int tq = live ? qperm[qo + r0 + row] : 0;
    const long long orow = pq.row0 + tq;
    const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
#pragma unroll
    for (int d0 = 0; d0 < HD; d0 += 16) {
      uint32_t r[16];
      tld16(tO + lane_off + (uint32_t)(HD * hc + d0), r);
      tld_wait(r);
      if (!live) continue;
      if (a.O != nullptr) {
        TO* O = static_cast<TO*>(a.O) + orow * D + HD * hc + d0;
        if (sizeof(TO) == 2) {
          uint32_t w[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[2 * e]) * inv,
                                                           __uint_as_float(r[2 * e + 1]) * inv);
            w[e] = *reinterpret_cast<const uint32_t*>(&h);
          }
          reinterpret_cast<uint4*>(O)[0] = make_uint4(w[0], w[1], w[2], w[3]);
          reinterpret_cast<uint4*>(O)[1] = make_uint4(w[4], w[5], w[6], w[7]);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            reinterpret_cast<float4*>(O)[e] =
                make_float4(__uint_as_float(r[4 * e]) * inv, __uint_as_float(r[4 * e + 1]) * inv,
                            __uint_as_float(r[4 * e + 2]) * inv, __uint_as_float(r[4 * e + 3]) * inv);
        }
      } else {
        float* pp = a.part + (size_t)(pq.slot0 + tq) * (D + 1) + HD * hc + d0;
#pragma unroll
        for (int e = 0; e < 16; ++e) pp[e] = __uint_as_float(r[e]) * inv;
      }
    }
    if (live && hc == 0 && a.O == nullptr)
      a.part[(size_t)(pq.slot0 + tq) * (D + 1) + D] = (mref + log2f(ltot)) * 0.6931471805599453f;
    if (live && hc == 0 && a.n_exact != nullptr) {
      if (a.O != nullptr)
        a.n_exact[orow] = nexact;
      else
        atomicAdd(reinterpret_cast<unsigned long long*>(a.n_exact + orow), (unsigned long long)nexact);
    }
  }
  if (!ok) atomicOr(a.qs.err, kErrMmaWait);
  fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;\n" ::"r"(tbase));
}

// Levels whose query clusters average at least this many queries, and that
// retrieve, take the tensor-core kernel (far-field-only tiles and small
// clusters run better as 16-query warp slices; at D = 128 the warp slices are
// register-bound, so smaller clusters already pay on the tensor cores).
int stage2_tc_levels(const Levels& lv, int D, int Cq, int Ck, int topk, int dense_lv) {
  if (topk < 1 || topk > kTMaxSel || Cq > 256 || Ck > 256) return 0;
  const int min_q = D == 128 ? 32 : 64;
  int m = 0;
  for (int l = 0; l < lv.nlev; ++l)
    if (!((dense_lv >> l) & 1) && lv.s[l] >= min_q * imin(Cq, lv.s[l]) && lv.s[l] >= kTQ)
      m |= 1 << l;
  return m;
}

void run_permute_keys(const AttnArgs& a, cudaStream_t st) {
  if (a.tc_lv == 0) return;
  ProfScope ps(st, "stage2_permute");
  int gmax = 0;  // groups of a key problem at those levels, at most
  for (int l = 0; l < a.kg.lv.nlev; ++l)
    if ((a.tc_lv >> l) & 1) {
      const int gl = a.kg.lv.s[l] / 8 + imin(a.Ck, a.kg.lv.s[l]);
      gmax = gmax > gl ? gmax : gl;
    }
  const dim3 grid(a.ks.nprob, cdiv(gmax, kPermGroups));
  if (a.kg.D == 64)
    permute_keys_kernel<64><<<grid, 256, 0, st>>>(a);
  else
    permute_keys_kernel<128><<<grid, 256, 0, st>>>(a);
}

template <int D>
static void launch_tc(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, int ty, cudaStream_t st) {
  const size_t smem = TcL<D>::TOTAL;
  const dim3 grid(nqp, ty);
  if (a.out_f32) {
    cudaFuncSetAttribute(stage2_tc_kernel<float, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    stage2_tc_kernel<float, D><<<grid, kTT, smem, st>>>(a, s1, qp0);
  } else {
    cudaFuncSetAttribute(stage2_tc_kernel<__nv_bfloat16, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    stage2_tc_kernel<__nv_bfloat16, D><<<grid, kTT, smem, st>>>(a, s1, qp0);
  }
}

void run_stage2_tc(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st) {
  if (a.tc_lv == 0) return;
  int ty = 0;  // tiles of a query problem, at most: one per 128 queries plus one per cluster
  for (int l = 0; l < a.qg.lv.nlev; ++l)
    if ((a.tc_lv >> l) & 1) {
      const int t = cdiv(a.qg.lv.s[l], kTQ) + imin(a.Cq, a.qg.lv.s[l]);
      ty = ty > t ? ty : t;
    }
  if (a.qg.D == 64)
    launch_tc<64>(a, s1, qp0, nqp, ty, st);
  else
    launch_tc<128>(a, s1, qp0, nqp, ty, st);
}

}  // namespace muse
