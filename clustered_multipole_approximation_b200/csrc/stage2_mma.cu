// Stage 2 of MuSe on tensor cores for bf16 inputs: for the queries of one
// query cluster i, one online softmax over
//   - the far field: one row per non-retrieved non-empty key cluster j, key
//     row mu_j (or the tilted centroid k_hat_ij), logit offset fbias_ij and
//     value u_ij (gist.science page "Multipole Semantic Attention: A Fast
//     Approximation of Softmax Attention for Pretraining", Technical Summary,
//     Core Mechanisms: Stage 2 (Refinement));
//   - exact attention over every key of the retrieved clusters (same page,
//     Exact Attention).
// Eight warps own 16 query rows each (128 queries per pass).  S = Q K^T runs
// as bf16 m16n8k16 MMAs with fp32 accumulation: bf16 query and key rows are
// exact, a far-field key row (fp32) enters as its bf16 hi + lo split (two
// MMAs, residual 2^-18 relative).  P and V enter the PV product as fp16 (the
// fp16 copy of V is exact in fp16's normal range); for far rows P and u_ij
// each enter as an fp16 hi + lo pair, accumulating in fp32.  Key blocks of 64 rows stream through shared memory
// with cp.async, two blocks in flight.
#include <cuda_fp16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"

namespace muse {

namespace {

constexpr int kMQ = 128;     // queries per pass (8 warps x 16 rows)
constexpr int kMK = 64;      // key rows per block
constexpr int kThreads = 256;
constexpr int kXRows = 2048;  // exact rows resolved once per CTA

template <int D>
struct KBuf {
  __nv_bfloat16 k[kMK][D + 8];    // exact keys, or the hi part of far keys
  __nv_bfloat16 k2[kMK][D + 8];   // lo part of far keys
  __half v[kMK][D + 8];           // exact values, or the hi part of u_ij
  __half v2[kMK][D + 8];          // lo part of u_ij (far blocks)
  float bias[kMK];
};

template <int D>
struct Smem2 {
  __nv_bfloat16 q[kMQ][D + 8];
  KBuf<D> buf[2];
  float fb[kMaxC];      // far-field logit offset (base 2) per key cluster, -inf if not far
  unsigned short sel[kMaxC];
  int selstart[kMaxC];  // start of each retrieved cluster in the concatenated list
  int selbase[kMaxC];   // its first position in the key problem's sorted order
  int xrow[kXRows];     // the concatenated list's rows, when it has at most kXRows
};
// two CTAs per SM at D = 64 (228 KB per SM, 1 KB reserved per CTA)
static_assert(2 * (sizeof(Smem2<64>) + 1024) <= 228 * 1024, "stage-2 tables too large");

}  // namespace

template <int D>
size_t stage2_mma_smem() {
  return sizeof(Smem2<D>);
}

// fp16 copy of bf16 V (the PV operand).  A finite value that overflows fp16
// (|v| >= 65520) is flagged in the device error word.
__global__ void bf16_to_half_kernel(const __nv_bfloat16* __restrict__ src, __half* __restrict__ dst,
                                    size_t n8, int* err) {
  bool over = false;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8;
       i += (size_t)gridDim.x * blockDim.x) {
    const uint4 v = reinterpret_cast<const uint4*>(src)[i];
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
    uint4 o;
    __half2* h = reinterpret_cast<__half2*>(&o);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = __bfloat1622float2(b[u]);
      h[u] = __float22half2_rn(f);
      // finite and |v| >= 65520 (the fp16 overflow threshold)
      over |= fabsf(f.x) >= 65520.f && fabsf(f.x) < INFINITY;
      over |= fabsf(f.y) >= 65520.f && fabsf(f.y) < INFINITY;
    }
    reinterpret_cast<uint4*>(dst)[i] = o;
  }
  if (over) atomicOr(err, kErrVRange);
}

void run_bf16_to_half(const void* src, __half* dst, size_t n, int* err, cudaStream_t st) {
  ProfScope ps(st, "v_to_half");
  const size_t n8 = n / 8;
  const int blocks = (int)((n8 + 255) / 256 < 148 * 8 ? (n8 + 255) / 256 : 148 * 8);
  bf16_to_half_kernel<<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(src), dst, n8,
                                              err);
}

template <typename TO, int D>
__global__ void __launch_bounds__(kThreads, D == 64 ? 2 : 1) stage2_mma_kernel(AttnArgs a, Stage1 s1,
                                                                               int qp0) {
  extern __shared__ __align__(16) unsigned char sm2_raw[];
  Smem2<D>& sm = *reinterpret_cast<Smem2<D>*>(sm2_raw);
  constexpr int KD = D / 16;   // k-steps over the head dimension
  constexpr int ND = D / 8;    // n-tiles over the head dimension
  constexpr int CH = D / 8;    // 16-byte chunks per row
  const int lq = blockIdx.x, qpid = qp0 + lq, i = blockIdx.y;
  const Prob pq = prob_of(a.qg, qpid);
  if (i >= pq.C || (((a.dense_lv | a.tc_lv) >> pq.level) & 1)) return;
  const int Cq = a.Cq, Ck = a.Ck;
  const int nqi = a.qs.counts[(size_t)qpid * Cq + i];
  if (nqi == 0) return;
  const int kpid = kv_problem(a, qpid);
  const Prob pk = prob_of(a.kg, kpid);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int nsel = a.topk > 0 ? s1.nsel[(size_t)qpid * Cq + i] : 0;
  const int* kc = a.ks.counts + (size_t)kpid * Ck;
  // far-field offsets of the non-empty clusters; the retrieved ones are then
  // taken out of the far field (their keys enter exactly)
  for (int r = tid; r < nsel; r += kThreads)
    sm.sel[r] = (unsigned short)s1.sel[((size_t)qpid * Cq + i) * a.topk + r];
  for (int j = tid; j < pk.C; j += kThreads)
    sm.fb[j] = kc[j] > 0 ? s1.fbias[((size_t)lq * Cq + i) * Ck + j] * 1.4426950408889634f : -INFINITY;
  __syncthreads();
  for (int r = tid; r < nsel; r += kThreads) sm.fb[sm.sel[r]] = -INFINITY;
  const int* koff = a.ks.off + (size_t)kpid * (Ck + 1);
  const int* kperm = a.ks.perm + pk.slot0;
  // the retrieved clusters' members, concatenated in selection order, are one
  // list of exact keys cut into blocks of 64 (a block may span two clusters)
  long long nexact = 0;
  for (int r = 0; r < nsel; ++r) {
    sm.selstart[r] = (int)nexact;
    nexact += kc[sm.sel[r]];
  }
  // per-CTA tables: the retrieved clusters' first sorted positions and, when
  // it fits, the row of every exact key
  for (int r = tid; r < nsel; r += kThreads) sm.selbase[r] = koff[sm.sel[r]];
  __syncthreads();
  const bool prerow = nexact <= kXRows;
  if (prerow) {
    constexpr int U = 2;
    for (int q0 = tid; q0 < (int)nexact; q0 += U * kThreads) {
      int v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int pos = q0 + u * kThreads;
        v[u] = 0;
        if (pos < (int)nexact) {
          int rr = 0;
          while (rr + 1 < nsel && sm.selstart[rr + 1] <= pos) ++rr;
          v[u] = kperm[sm.selbase[rr] + pos - sm.selstart[rr]];
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (q0 + u * kThreads < (int)nexact) sm.xrow[q0 + u * kThreads] = v[u];
    }
  }
  __syncthreads();
  const int nblk_exact = cdiv((int)nexact, kMK);
  const int nblk_far = cdiv(pk.C, kMK);
  const int nblk = nblk_far + nblk_exact;

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

  // block b (far blocks first, then the retrieved clusters' keys) into buf
  auto issue = [&](int b, KBuf<D>& B) {
    if (b < nblk_far) {
      const int j0 = b * kMK;
      for (int e = tid; e < kMK * CH; e += kThreads) {
        const int r = e / CH, c = (e % CH) * 8, j = j0 + r;
        const bool live = j < pk.C && sm.fb[j] > -INFINITY;
        const size_t o = (size_t)(live ? j : 0) * D + c;
        cp16(&B.k[r][c], khi + o, live ? 16 : 0);
        cp16(&B.k2[r][c], klo + o, live ? 16 : 0);
        cp16(&B.v[r][c], uh + o, live ? 16 : 0);
        cp16(&B.v2[r][c], ul + o, live ? 16 : 0);
      }
      for (int r = tid; r < kMK; r += kThreads) {
        const int j = j0 + r;
        B.bias[r] = j < pk.C ? sm.fb[j] : -INFINITY;
      }
    } else {
      // rows p0 .. p0+63 of the concatenated member list
      const int p0 = (b - nblk_far) * kMK;
      const int nr = imin(kMK, (int)nexact - p0);
      for (int e = tid; e < kMK * CH; e += kThreads) {
        const int r = e / CH, c = (e % CH) * 8;
        const bool live = r < nr;
        long long row = pk.row0;
        if (live) {
          const int pos = p0 + r;
          if (prerow) {
            row += sm.xrow[pos];
          } else {
            int rr = 0;
            while (rr + 1 < nsel && sm.selstart[rr + 1] <= pos) ++rr;
            row += kperm[sm.selbase[rr] + pos - sm.selstart[rr]];
          }
        }
        cp16(&B.k[r][c], K + row * D + c, live ? 16 : 0);
        cp16(&B.v[r][c], V16 + row * D + c, live ? 16 : 0);
      }
      for (int r = tid; r < kMK; r += kThreads) B.bias[r] = r < nr ? 0.f : -INFINITY;
    }
    cp_commit();
  };

  for (int c0 = 0; c0 < nqi; c0 += kMQ) {
    const int nq = imin(kMQ, nqi - c0);
    const bool wact = warp * 16 < nq;  // warps with no query rows skip the math
    __syncthreads();
    for (int e = tid; e < kMQ * CH; e += kThreads) {
      const int r = e / CH, c = (e % CH) * 8;
      const bool live = r < nq;
      const long long row = pq.row0 + (live ? qperm[qo + c0 + r] : 0);
      cp16(&sm.q[r][c], Q + row * D + c, live ? 16 : 0);
    }
    issue(0, sm.buf[0]);  // commits the query rows with block 0
    uint32_t qa[KD][4];
    float o[ND][4];
#pragma unroll
    for (int n = 0; n < ND; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float mrow[2] = {kMaxFloor, kMaxFloor}, lrow[2] = {0.f, 0.f};

    for (int b = 0; b < nblk; ++b) {
      if (b + 1 < nblk) {
        issue(b + 1, sm.buf[(b + 1) & 1]);
        cp_wait<1>();
      } else {
        cp_wait<0>();
      }
      __syncthreads();
      if (b == 0 && wact) {
#pragma unroll
        for (int kk = 0; kk < KD; ++kk) {
          const int row = warp * 16 + (lane & 15), col = kk * 16 + (lane >> 4) * 8;
          ldsm_x4(smem_u32(&sm.q[row][col]), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
        }
      }
      const KBuf<D>& B = sm.buf[b & 1];
      const bool two = b < nblk_far;
      if (wact) {
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
            ldsm_x4(smem_u32(&B.k[key][col]), b0, b1, b2, b3);
            mma_bf16(sc[2 * np], qa[kk], b0, b1);
            mma_bf16(sc[2 * np + 1], qa[kk], b2, b3);
            if (two) {
              ldsm_x4(smem_u32(&B.k2[key][col]), b0, b1, b2, b3);
              mma_bf16(sc[2 * np], qa[kk], b0, b1);
              mma_bf16(sc[2 * np + 1], qa[kk], b2, b3);
            }
          }
        }
        float mx[2] = {kMaxFloor, kMaxFloor};
#pragma unroll
        for (int n = 0; n < kMK / 8; ++n) {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int col = n * 8 + 2 * t4 + (h & 1);
            const float lg = fmaf(sl2, sc[n][h], B.bias[col]);
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
          scale[r] = fast_exp2(mrow[r] - mn);
          mrow[r] = mn;
        }
        float rs[2] = {0.f, 0.f};
#pragma unroll
        for (int n = 0; n < kMK / 8; ++n) {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float p = fast_exp2(sc[n][h] - mrow[h >> 1]);
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
        // far rows: P and u_ij each as an fp16 hi + lo pair (P_hi u_hi +
        // P_lo u_hi + P_hi u_lo), since a dipole summary can be far larger
        // than the values it averages; exact rows: P and v in fp16
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
            ldsm_x4_t(smem_u32(&B.v[key][col]), b0, b1, b2, b3);
            mma_f16(o[2 * np], pa, b0, b1);
            mma_f16(o[2 * np + 1], pa, b2, b3);
          }
        }
        if (two) {
#pragma unroll
          for (int kk = 0; kk < kMK / 16; ++kk) {
            uint32_t pa[4], pl[4];
            split_h2(sc[2 * kk][0], sc[2 * kk][1], pa[0], pl[0]);
            split_h2(sc[2 * kk][2], sc[2 * kk][3], pa[1], pl[1]);
            split_h2(sc[2 * kk + 1][0], sc[2 * kk + 1][1], pa[2], pl[2]);
            split_h2(sc[2 * kk + 1][2], sc[2 * kk + 1][3], pa[3], pl[3]);
#pragma unroll
            for (int np = 0; np < ND / 2; ++np) {
              const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
              const int col = np * 16 + (lane >> 4) * 8;
              uint32_t b0, b1, b2, b3;
              ldsm_x4_t(smem_u32(&B.v[key][col]), b0, b1, b2, b3);
              mma_f16(o[2 * np], pl, b0, b1);
              mma_f16(o[2 * np + 1], pl, b2, b3);
              ldsm_x4_t(smem_u32(&B.v2[key][col]), b0, b1, b2, b3);
              mma_f16(o[2 * np], pa, b0, b1);
              mma_f16(o[2 * np + 1], pa, b2, b3);
            }
          }
        }
      }
      __syncthreads();
    }
    // write the pass's rows
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

// Causal exact local block + merge of the level partials, on mma.sync tiles
// (bf16 inputs; gist.science page "Multipole Semantic Attention: A Fast
// Approximation of Softmax Attention for Pretraining", Technical Summary,
// hierarchical causal decomposition: exact attention inside each local
// block, approximated levels beyond it).  One CTA of 8 warps per 128
// consecutive queries of one (b, q-head); the local block length L is a
// multiple of 128, so the tile lies inside one block and its keys are the
// contiguous run [block start, last query], streamed in 64-row blocks with
// cp.async, two in flight.  S = Q K^T in bf16 with fp32 accumulation, the
// causal mask on the diagonal blocks, one online softmax in base 2, P and V in
// fp16; then every level partial of the row (normalised output, log-sum-exp)
// enters the same softmax as one term.
template <int D>
struct LocSmem {
  __nv_bfloat16 q[kMQ][D + 8];
  __nv_bfloat16 k[2][kMK][D + 8];
  __half v[2][kMK][D + 8];
};

template <typename TO, int D>
__global__ void __launch_bounds__(kThreads, D == 64 ? 2 : 1) local_mma_kernel(AttnArgs a, int L) {
  extern __shared__ __align__(16) unsigned char loc_raw[];
  LocSmem<D>& sm = *reinterpret_cast<LocSmem<D>*>(loc_raw);
  constexpr int KD = D / 16, ND = D / 8, CH = D / 8;
  const int bhq = blockIdx.x, N = a.qg.lv.N;
  const int q0 = blockIdx.y * kMQ;
  const int nq = imin(kMQ, N - q0);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const bool wact = warp * 16 < nq;
  const int Hq = a.qg.BH / a.B, Hkv = a.kg.BH / a.B;
  const int bhk = (bhq / Hq) * Hkv + (bhq % Hq) / a.G;
  const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(a.qg.X) + (size_t)bhq * N * D;
  const __nv_bfloat16* K = static_cast<const __nv_bfloat16*>(a.kg.X) + (size_t)bhk * N * D;
  const __half* V16 = a.V16 + (size_t)bhk * N * D;
  const int blk = q0 / L, kbeg = blk * L, kend = q0 + nq;  // keys [kbeg, kend)
  const int nkb = cdiv(kend - kbeg, kMK);
  const float sl2 = a.scale * 1.4426950408889634f;
  auto issue = [&](int b) {
    const int t0 = kbeg + b * kMK, nr = imin(kMK, kend - t0), st = b & 1;
    for (int e = tid; e < kMK * CH; e += kThreads) {
      const int r = e / CH, c = (e % CH) * 8;
      const bool live = r < nr;
      const size_t o = (size_t)(live ? t0 + r : 0) * D + c;
      cp16(&sm.k[st][r][c], K + o, live ? 16 : 0);
      cp16(&sm.v[st][r][c], V16 + o, live ? 16 : 0);
    }
    cp_commit();
  };
  for (int e = tid; e < kMQ * CH; e += kThreads) {
    const int r = e / CH, c = (e % CH) * 8;
    const bool live = r < nq;
    cp16(&sm.q[r][c], Q + (size_t)(live ? q0 + r : 0) * D + c, live ? 16 : 0);
  }
  issue(0);  // commits the query rows with block 0
  uint32_t qa[KD][4];
  float o[ND][4];
#pragma unroll
  for (int n = 0; n < ND; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float mrow[2] = {kMaxFloor, kMaxFloor}, lrow[2] = {0.f, 0.f};
  const int qpos[2] = {q0 + warp * 16 + g, q0 + warp * 16 + g + 8};

  for (int b = 0; b < nkb; ++b) {
    if (b + 1 < nkb) {
      issue(b + 1);
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    if (b == 0 && wact) {
#pragma unroll
      for (int kk = 0; kk < KD; ++kk) {
        const int row = warp * 16 + (lane & 15), col = kk * 16 + (lane >> 4) * 8;
        ldsm_x4(smem_u32(&sm.q[row][col]), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
      }
    }
    const int st = b & 1, t0 = kbeg + b * kMK;
    // blocks wholly after this warp's last row contribute nothing
    if (wact && t0 <= q0 + warp * 16 + 15) {
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
          ldsm_x4(smem_u32(&sm.k[st][key][col]), b0, b1, b2, b3);
          mma_bf16(sc[2 * np], qa[kk], b0, b1);
          mma_bf16(sc[2 * np + 1], qa[kk], b2, b3);
        }
      }
      float mx[2] = {kMaxFloor, kMaxFloor};
#pragma unroll
      for (int n = 0; n < kMK / 8; ++n) {
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int t = t0 + n * 8 + 2 * t4 + (h & 1);
          const float lg = (t < kend && t <= qpos[h >> 1]) ? sl2 * sc[n][h] : -INFINITY;
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
        scale[r] = fast_exp2(mrow[r] - mn);
        mrow[r] = mn;
      }
      float rs[2] = {0.f, 0.f};
#pragma unroll
      for (int n = 0; n < kMK / 8; ++n) {
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float pv = fast_exp2(sc[n][h] - mrow[h >> 1]);
          sc[n][h] = pv;
          rs[h >> 1] += pv;
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
          ldsm_x4_t(smem_u32(&sm.v[st][key][col]), b0, b1, b2, b3);
          mma_f16(o[2 * np], pa, b0, b1);
          mma_f16(o[2 * np + 1], pa, b2, b3);
        }
      }
    }
    __syncthreads();
  }
  if (!wact) return;
  // ---- the level partials of each row, one softmax term each -----------------
  const int levels = a.accum ? (blk > 0 ? 1 : 0) : a.qg.lv.nlev;
  const float* part = a.part;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int qp = qpos[r];
    if (qp >= kend) continue;
    for (int lv = 0; lv < levels; ++lv) {
      if (!a.accum && !((blk >> lv) & 1)) continue;
      const int sz = L << lv, pp_ = blk >> (lv + 1);
      const long long slot = a.accum ? (long long)bhq * N + qp
                                     : (long long)bhq * a.qg.lv.toks_per_bh + a.qg.lv.tok_base[lv] +
                                           (long long)pp_ * sz + (qp - (2 * pp_ + 1) * sz);
      const float* pp = part + slot * (D + 1);
      const float lg = pp[D] * 1.4426950408889634f;  // natural log -> base 2
      const float mn = fmaxf(mrow[r], lg);
      const float sc = fast_exp2(mrow[r] - mn), wt = fast_exp2(lg - mn);
      lrow[r] = lrow[r] * sc + wt;
#pragma unroll
      for (int n = 0; n < ND; ++n) {
        const int c = n * 8 + 2 * t4;
        o[n][2 * r] = fmaf(o[n][2 * r], sc, wt * pp[c]);
        o[n][2 * r + 1] = fmaf(o[n][2 * r + 1], sc, wt * pp[c + 1]);
      }
      mrow[r] = mn;
    }
    TO* O = static_cast<TO*>(a.O) + ((size_t)bhq * N + qp) * D;
    const float inv = 1.f / lrow[r];
#pragma unroll
    for (int n = 0; n < ND; ++n) {
      st<TO>(O + n * 8 + 2 * t4, o[n][2 * r] * inv);
      st<TO>(O + n * 8 + 2 * t4 + 1, o[n][2 * r + 1] * inv);
    }
    if (a.n_exact != nullptr && t4 == 0)
      atomicAdd(reinterpret_cast<unsigned long long*>(a.n_exact + (size_t)bhq * N + qp),
                (unsigned long long)(qp - kbeg + 1));
  }
}

template <int D>
static void launch_local(const AttnArgs& a, int L, cudaStream_t st) {
  // set on every launch: the attribute is per device, and the call is cheap
  cudaFuncSetAttribute(local_mma_kernel<float, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)sizeof(LocSmem<D>));
  cudaFuncSetAttribute(local_mma_kernel<__nv_bfloat16, D>,
                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(LocSmem<D>));
  dim3 grid(a.qg.BH, cdiv(a.qg.lv.N, kMQ));
  if (a.out_f32)
    local_mma_kernel<float, D><<<grid, kThreads, sizeof(LocSmem<D>), st>>>(a, L);
  else
    local_mma_kernel<__nv_bfloat16, D><<<grid, kThreads, sizeof(LocSmem<D>), st>>>(a, L);
}

bool run_local_mma(const AttnArgs& a, int L, cudaStream_t st) {
  if (a.qg.dtype != 0 || L % kMQ != 0 || a.V16 == nullptr) return false;
  if (a.qg.D == 64)
    launch_local<64>(a, L, st);
  else
    launch_local<128>(a, L, st);
  return true;
}

template <int D>
static void launch_t(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st) {
  // set on every launch: the attribute is per device, and the call is cheap
  cudaFuncSetAttribute(stage2_mma_kernel<float, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)stage2_mma_smem<D>());
  cudaFuncSetAttribute(stage2_mma_kernel<__nv_bfloat16, D>,
                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)stage2_mma_smem<D>());
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
