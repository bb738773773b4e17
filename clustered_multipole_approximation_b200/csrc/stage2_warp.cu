// Stage 2 of MuSe for bf16 inputs with one warp per 16-query slice.
//
// For the queries of query cluster i (gist.science page "Multipole Semantic
// Attention: A Fast Approximation of Softmax Attention for Pretraining",
// Technical Summary, Core Mechanisms: Stage 2 (Refinement), Exact Attention)
// one online softmax runs over
//   - the far field: one row per non-retrieved non-empty key cluster j, key
//     row mu_j (TILTED: k_hat_ij) as a bf16 hi + lo pair, logit offset
//     fbias_ij, value u_ij as an fp16 hi + lo pair;
//   - every key of the retrieved clusters, exactly (bf16 k, fp16 v).
// Query clusters hold few queries where a block holds few tokens per cluster
// (16 at 4096 tokens and 256 clusters), so the work unit is a slice of at most
// 16 queries of one cluster, and each warp streams its own slice's keys: the
// eight warps of a CTA take eight slices of one query problem.  S = Q K^T and
// P V run as m16n8k16 MMAs with fp32 accumulation, in blocks of 16 keys.
//   - K rows go straight from global memory into B fragments: the dot product
//     does not depend on the order of the dimensions, so thread t of a
//     fragment quad takes dimensions [t D/4, (t+1) D/4) of its rows for Q and
//     K alike, and loads them with 16-byte vectors;
//   - V rows (and u_ij) pass through a per-warp shared buffer for the
//     transposed ldmatrix of the P V operand, copied with cp.async one block
//     ahead (exact keys) in a ping-pong of two blocks.
#include <cuda_fp16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"

namespace muse {

namespace {

constexpr int kWW = 8;        // warps (slices) per CTA
constexpr int kWK = 16;       // keys per block
constexpr int kWMaxSel = 64;  // retrieved clusters per query cluster this kernel takes

template <int D>
struct __align__(16) WarpBuf {  // 16-byte aligned rows for cp.async and ldmatrix
  __half v[2][kWK][D + 8];  // exact: ping-pong of value blocks; far: u hi, u lo
                            // (rows of (D + 8) halves: multiples of 16 bytes)
  int sel[kWMaxSel];        // the query cluster's retrieved clusters
  int start[kWMaxSel + 1];  // their first position in the concatenated key list
  int base[kWMaxSel];       // their first position in the key problem's sorted order
};

static_assert(sizeof(WarpBuf<64>) % 16 == 0 && sizeof(WarpBuf<128>) % 16 == 0, "warp buffers");

template <int D>
constexpr size_t warp_smem(int Cq) {
  return (((size_t)(Cq + 1) * 4 + 15) & ~(size_t)15) + (size_t)kWW * sizeof(WarpBuf<D>);
}

// The thread's D/4 dimensions of a bf16 row as 16-byte pieces (zero past nq).
template <int D>
__device__ inline void load_chunk(const __nv_bfloat16* row, int t, bool live, uint4 (&c)[D / 32]) {
#pragma unroll
  for (int q = 0; q < D / 32; ++q)
    c[q] = live ? __ldg(reinterpret_cast<const uint4*>(row + t * (D / 4)) + q) : make_uint4(0, 0, 0, 0);
}
// 32-bit word m of a chunk (dimensions t D/4 + 2m, + 1)
template <int D>
__device__ inline uint32_t cw(const uint4 (&c)[D / 32], int m) {
  const uint4 v = c[m >> 2];
  return (m & 3) == 0 ? v.x : (m & 3) == 1 ? v.y : (m & 3) == 2 ? v.z : v.w;
}

}  // namespace

template <int D>
size_t stage2_warp_smem(int Cq) {
  return warp_smem<D>(Cq);
}

template <typename TO, int D>
__global__ void __launch_bounds__(kWW * 32) stage2_warp_kernel(AttnArgs a, Stage1 s1, int qp0) {
  extern __shared__ __align__(16) unsigned char sw_raw[];
  constexpr int KD = D / 16;  // k-steps over the head dimension
  constexpr int ND = D / 8;   // n-tiles over the head dimension
  constexpr int CH = D / 8;   // 16-byte pieces per row
  const int lq = blockIdx.x, qpid = qp0 + lq;
  const Prob pq = prob_of(a.qg, qpid);
  if ((a.dense_lv >> pq.level) & 1) return;  // that level runs one key token at a time
  if ((a.tc_lv >> pq.level) & 1) return;     // that level runs on the tensor-core kernel
  const int Cq = a.Cq, Ck = a.Ck, cq = pq.C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  int* spre = reinterpret_cast<int*>(sw_raw);  // [cq + 1] slices before each cluster
  WarpBuf<D>& wb = reinterpret_cast<WarpBuf<D>*>(sw_raw + (((size_t)(Cq + 1) * 4 + 15) & ~(size_t)15))[warp];
  __shared__ int wtot[kWW];

  // ---- slices of 16 queries: prefix over the query problem's clusters --------
  const int* qcnt = a.qs.counts + (size_t)qpid * Cq;
  {
    const int per = cdiv(cq, kWW * 32);  // clusters per thread, in order
    const int c0 = imin(cq, tid * per), c1 = imin(cq, c0 + per);
    int sum = 0;
    for (int c = c0; c < c1; ++c) sum += cdiv(qcnt[c], 16);
    int x = sum;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wtot[warp] = x;
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < kWW; ++w) {
      before += w < warp ? wtot[w] : 0;
      total += wtot[w];
    }
    int run = before + x - sum;
    for (int c = c0; c < c1; ++c) {
      spre[c] = run;
      run += cdiv(qcnt[c], 16);
    }
    if (tid == 0) spre[cq] = total;
    __syncthreads();
  }
  const int sl = blockIdx.y * kWW + warp;
  if (sl >= spre[cq]) return;  // no slice for this warp (no CTA-wide sync below)
  int lo = 0, hi = cq - 1;  // the cluster whose slices contain sl
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (spre[mid] <= sl) lo = mid;
    else hi = mid - 1;
  }
  const int i = lo;
  const int r0 = (sl - spre[i]) * 16;
  const int nq = imin(16, qcnt[i] - r0);

  const int kpid = kv_problem(a, qpid);
  const Prob pk = prob_of(a.kg, kpid);
  const int* kc = a.ks.counts + (size_t)kpid * Ck;
  const int* koff = a.ks.off + (size_t)kpid * (Ck + 1);
  const int* kperm = a.ks.perm + pk.slot0;
  const int nsel = a.topk > 0 ? s1.nsel[(size_t)qpid * Cq + i] : 0;
  // the retrieved clusters and their runs in the concatenated key list
  for (int r = lane; r < nsel; r += 32) {
    const int j = s1.sel[((size_t)qpid * Cq + i) * a.topk + r];
    wb.sel[r] = j;
    wb.base[r] = koff[j];
  }
  __syncwarp();
  if (lane == 0) {
    int run = 0;
    for (int r = 0; r < nsel; ++r) {
      wb.start[r] = run;
      run += kc[wb.sel[r]];
    }
    wb.start[nsel] = run;
  }
  __syncwarp();
  const int nexact = wb.start[nsel];

  const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(a.qg.X);
  const __nv_bfloat16* K = static_cast<const __nv_bfloat16*>(a.kg.X);
  const __half* V16 = a.V16;
  const int qo = a.qs.off[(size_t)qpid * (Cq + 1) + i];
  const int* qperm = a.qs.perm + pq.slot0;
  const size_t ij0 = ((size_t)lq * Cq + i) * Ck;
  const bool tilted = a.mode == 2;
  const float sl2 = a.scale * 1.4426950408889634f;  // logits in base-2 units
  const __nv_bfloat16* khi = tilted ? s1.Kfh + ij0 * D : a.ks.cbf_hi + (size_t)kpid * Ck * D;
  const __nv_bfloat16* klo = tilted ? s1.Kfl + ij0 * D : a.ks.cbf_lo + (size_t)kpid * Ck * D;
  const __half* uh = s1.Uh + ij0 * D;
  const __half* ul = s1.Ul + ij0 * D;

  // ---- the slice's query rows: A fragments ------------------------------------
  const int tq = lane < nq ? qperm[qo + r0 + lane] : 0;
  const int tqa = __shfl_sync(0xffffffffu, tq, g), tqb = __shfl_sync(0xffffffffu, tq, g + 8);
  uint32_t qa[KD][4];
  {
    uint4 ca[D / 32], cb[D / 32];
    load_chunk<D>(Q + (pq.row0 + tqa) * D, t4, g < nq, ca);
    load_chunk<D>(Q + (pq.row0 + tqb) * D, t4, g + 8 < nq, cb);
#pragma unroll
    for (int kk = 0; kk < KD; ++kk) {
      qa[kk][0] = cw<D>(ca, 2 * kk);
      qa[kk][1] = cw<D>(cb, 2 * kk);
      qa[kk][2] = cw<D>(ca, 2 * kk + 1);
      qa[kk][3] = cw<D>(cb, 2 * kk + 1);
    }
  }
  float o[ND][4];
#pragma unroll
  for (int n = 0; n < ND; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float mrow[2] = {kMaxFloor, kMaxFloor}, lrow[2] = {0.f, 0.f};

  // one block: logits from the B fragments (and lo parts when far), then the
  // online softmax step and P V from the value buffers (hi, lo when far)
  auto block = [&](const uint4 (&k0)[D / 32], const uint4 (&k1)[D / 32], const uint4* l0,
                   const uint4* l1, const float (&bias)[4], const __half (*vb)[D + 8],
                   const __half (*vl)[D + 8]) {
    float sc[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KD; ++kk) {
      mma_bf16(sc[0], qa[kk], cw<D>(k0, 2 * kk), cw<D>(k0, 2 * kk + 1));
      mma_bf16(sc[1], qa[kk], cw<D>(k1, 2 * kk), cw<D>(k1, 2 * kk + 1));
    }
    if (l0 != nullptr) {
      const uint4(&m0)[D / 32] = *reinterpret_cast<const uint4(*)[D / 32]>(l0);
      const uint4(&m1)[D / 32] = *reinterpret_cast<const uint4(*)[D / 32]>(l1);
#pragma unroll
      for (int kk = 0; kk < KD; ++kk) {
        mma_bf16(sc[0], qa[kk], cw<D>(m0, 2 * kk), cw<D>(m0, 2 * kk + 1));
        mma_bf16(sc[1], qa[kk], cw<D>(m1, 2 * kk), cw<D>(m1, 2 * kk + 1));
      }
    }
    float mx[2] = {kMaxFloor, kMaxFloor};
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float lg = fmaf(sl2, sc[n][h], bias[2 * n + (h & 1)]);
        sc[n][h] = lg;
        mx[h >> 1] = fmaxf(mx[h >> 1], lg);
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
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float p = fast_exp2(sc[n][h] - mrow[h >> 1]);
        sc[n][h] = p;
        rs[h >> 1] += p;
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
    uint32_t pa[4], pl[4];
    if (vl == nullptr) {
      pa[0] = pack_h2(sc[0][0], sc[0][1]);
      pa[1] = pack_h2(sc[0][2], sc[0][3]);
      pa[2] = pack_h2(sc[1][0], sc[1][1]);
      pa[3] = pack_h2(sc[1][2], sc[1][3]);
    } else {  // far rows: P and u_ij as fp16 hi + lo pairs
      split_h2(sc[0][0], sc[0][1], pa[0], pl[0]);
      split_h2(sc[0][2], sc[0][3], pa[1], pl[1]);
      split_h2(sc[1][0], sc[1][1], pa[2], pl[2]);
      split_h2(sc[1][2], sc[1][3], pa[3], pl[3]);
    }
    const int key = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
    for (int np = 0; np < ND / 2; ++np) {
      const int col = np * 16 + (lane >> 4) * 8;
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(smem_u32(&vb[key][col]), b0, b1, b2, b3);
      mma_f16(o[2 * np], pa, b0, b1);
      mma_f16(o[2 * np + 1], pa, b2, b3);
      if (vl != nullptr) {
        mma_f16(o[2 * np], pl, b0, b1);
        mma_f16(o[2 * np + 1], pl, b2, b3);
        ldsm_x4_t(smem_u32(&vl[key][col]), b0, b1, b2, b3);
        mma_f16(o[2 * np], pa, b0, b1);
        mma_f16(o[2 * np + 1], pa, b2, b3);
      }
    }
  };

  // ---- far field: the key clusters in blocks of 16, retrieved / empty masked --
  for (int j0 = 0; j0 < pk.C; j0 += kWK) {
    // far row j0 + r (lane r < 16): a non-empty cluster outside R_i; the rows
    // of other clusters are zero (an empty or retrieved cluster's table rows
    // need not hold numbers) and get a -inf logit
    bool fl = false;
    if (lane < kWK) {
      const int j = j0 + lane;
      fl = j < pk.C && kc[j] > 0;
      for (int r = 0; r < nsel && fl; ++r) fl = wb.sel[r] != j;
    }
    __syncwarp();  // the previous block's value reads are done
#pragma unroll
    for (int q = 0; q < kWK * CH / 32; ++q) {
      const int e = lane + 32 * q, r = e / CH, c = (e % CH) * 8;
      const bool live = __shfl_sync(0xffffffffu, fl, r);
      const size_t off = (size_t)(live ? j0 + r : 0) * D + c;
      cp16(&wb.v[0][r][c], uh + off, live ? 16 : 0);
      cp16(&wb.v[1][r][c], ul + off, live ? 16 : 0);
    }
    cp_commit();
    float bias[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int r = 8 * (x >> 1) + 2 * t4 + (x & 1);
      const bool live = __shfl_sync(0xffffffffu, fl, r);
      bias[x] = live ? s1.fbias[ij0 + j0 + r] * 1.4426950408889634f : -INFINITY;
    }
    const bool la = __shfl_sync(0xffffffffu, fl, g), lb = __shfl_sync(0xffffffffu, fl, g + 8);
    const int ja = la ? j0 + g : 0, jb = lb ? j0 + g + 8 : 0;
    uint4 h0[D / 32], h1[D / 32], m0[D / 32], m1[D / 32];
    load_chunk<D>(khi + (size_t)ja * D, t4, la, h0);
    load_chunk<D>(khi + (size_t)jb * D, t4, lb, h1);
    load_chunk<D>(klo + (size_t)ja * D, t4, la, m0);
    load_chunk<D>(klo + (size_t)jb * D, t4, lb, m1);
    cp_wait<0>();
    __syncwarp();
    block(h0, h1, m0, m1, bias, wb.v[0], wb.v[1]);
  }

  // ---- exact retrieval: the retrieved clusters' keys, 16 at a time -------------
  // (the row of key p of the concatenated list, resolved by its lane)
  auto key_row = [&](int p) -> int {
    if (p >= nexact) return -1;
    int r = 0;
    while (r + 1 < nsel && wb.start[r + 1] <= p) ++r;
    return kperm[wb.base[r] + p - wb.start[r]];
  };
  const int nblk = cdiv(nexact, kWK);
  int rowv = key_row(lane < kWK ? lane : nexact);  // block 0's rows on lanes 0-15
  __syncwarp();
  auto copy_v = [&](int rv, int buf) {
    // lane l copies pieces l, l + 32, ... of the 16 x CH grid (row r = piece / CH)
#pragma unroll
    for (int q = 0; q < kWK * CH / 32; ++q) {
      const int e = lane + 32 * q, r = e / CH, c = (e % CH) * 8;
      const int rr = __shfl_sync(0xffffffffu, rv, r);
      cp16(&wb.v[buf][r][c], V16 + (pk.row0 + (rr >= 0 ? rr : 0)) * D + c, rr >= 0 ? 16 : 0);
    }
    cp_commit();
  };
  if (nblk > 0) copy_v(rowv, 0);
  for (int b = 0; b < nblk; ++b) {
    const int p0 = b * kWK;
    const int ra = __shfl_sync(0xffffffffu, rowv, g), rb = __shfl_sync(0xffffffffu, rowv, g + 8);
    uint4 k0[D / 32], k1[D / 32];
    load_chunk<D>(K + (pk.row0 + (ra >= 0 ? ra : 0)) * D, t4, ra >= 0, k0);
    load_chunk<D>(K + (pk.row0 + (rb >= 0 ? rb : 0)) * D, t4, rb >= 0, k1);
    int rown = -1;
    if (b + 1 < nblk) {  // the next block's rows and values start loading now
      rown = key_row(lane < kWK ? p0 + kWK + lane : nexact);
      __syncwarp();  // block b - 1's value reads of the other buffer are done
      copy_v(rown, (b + 1) & 1);
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncwarp();
    float bias[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int p = p0 + 8 * (x >> 1) + 2 * t4 + (x & 1);
      bias[x] = p < nexact ? 0.f : -INFINITY;
    }
    block(k0, k1, nullptr, nullptr, bias, wb.v[b & 1], nullptr);
    rowv = rown;
  }

  // ---- the slice's rows: normalised output (or level partial), exact counts ----
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int qr = g + 8 * r;
    const int tqr = r ? tqb : tqa;
    if (qr >= nq) continue;
    const long long row = pq.row0 + tqr;
    const float inv = 1.f / lrow[r];
    if (a.O != nullptr) {
      TO* O = static_cast<TO*>(a.O);
#pragma unroll
      for (int n = 0; n < ND; ++n) {
        st<TO>(O + row * D + n * 8 + 2 * t4, o[n][2 * r] * inv);
        st<TO>(O + row * D + n * 8 + 2 * t4 + 1, o[n][2 * r + 1] * inv);
      }
    } else {
      float* pp = a.part + (size_t)(pq.slot0 + tqr) * (D + 1);
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

template <int D>
static void launch_w(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, int nslice,
                     cudaStream_t st) {
  const size_t smem = warp_smem<D>(a.Cq);
  const dim3 grid(nqp, cdiv(nslice, kWW));
  if (a.out_f32) {
    cudaFuncSetAttribute(stage2_warp_kernel<float, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    stage2_warp_kernel<float, D><<<grid, kWW * 32, smem, st>>>(a, s1, qp0);
  } else {
    cudaFuncSetAttribute(stage2_warp_kernel<__nv_bfloat16, D>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    stage2_warp_kernel<__nv_bfloat16, D><<<grid, kWW * 32, smem, st>>>(a, s1, qp0);
  }
}

bool run_stage2_warp(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st) {
  if (a.qg.dtype != 0 || a.V16 == nullptr || a.topk > kWMaxSel) return false;
  // slices of a query problem: at most one per 16 queries plus one per cluster
  int smax = 0;
  for (int l = 0; l < a.qg.lv.nlev; ++l)
    if (!(((a.dense_lv | a.tc_lv) >> l) & 1)) smax = smax > a.qg.lv.s[l] ? smax : a.qg.lv.s[l];
  if (smax == 0) return true;  // every level runs elsewhere
  const int nslice = cdiv(smax, 16) + imin(a.Cq, smax);
  if (a.qg.D == 64)
    launch_w<64>(a, s1, qp0, nqp, nslice, st);
  else
    launch_w<128>(a, s1, qp0, nqp, nslice, st);
  return true;
}

}  // namespace muse
