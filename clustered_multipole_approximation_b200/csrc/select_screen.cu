// Cluster selection of MuSe (gist.science page "Multipole Semantic Attention:
// A Fast Approximation of Softmax Attention for Pretraining", Technical
// Summary, Core Mechanisms, "Cluster Selection"): for every query cluster i
// the top-k1 key clusters j by the summary score
//     s_ij = s nu_i . mu_j + log W_ij      (log W_ij = log n_j, or the tilted
//                                            log-weight of stage 1)
// in rank order, ties to the lowest j, empty clusters never.
//
// The decision is taken on exact fp64 scores -- each dot product a plain
// sequential sum in dimension order, as a sequential evaluation forms it --
// but only for the clusters that can reach the top k1:
//   1. screen: every score in fp32 from the fp32 centroids (FMA chains), with
//      a certified bound E_i on its distance from the exact score;
//   2. T = the k1-th largest screened score; a cluster whose screened score is
//      below T - 2 E_i has k1 clusters certainly ahead of it and is dropped;
//   3. the remaining candidates get their exact fp64 scores and the top k1 of
//      those, ties to the lowest index, is the selection.
// One warp per query cluster; the CTA stages the key problem's fp32 centroids
// once and serves a block of query clusters of one query problem.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace muse {

namespace {

constexpr int kSW = 8;  // warps per CTA

struct SelLayout {
  int ld;  // staged centroid row stride (floats, a multiple of 4)
  size_t mu, lw, nu32, nu64, sc, cand, total;
};

__host__ __device__ inline SelLayout sel_layout(int D, int Ck, bool staged) {
  SelLayout L;
  L.ld = D + 4;
  size_t o = 0;
  L.mu = o;    o += staged ? (size_t)Ck * L.ld * 4 : 0;
  L.lw = o;    o += (size_t)Ck * 8;
  o = (o + 15) & ~(size_t)15;  // float4 reads of nu
  L.nu32 = o;  o += (size_t)kSW * D * 4;
  L.nu64 = o;  o += (size_t)kSW * D * 8;
  L.sc = o;    o += (size_t)kSW * Ck * 8;
  L.cand = o;  o += (size_t)kSW * Ck * 4;
  L.total = o;
  return L;
}

constexpr size_t kSelSmemMax = 200 * 1024;

// (v, j) ranks before (w, k): larger score, ties to the lower index.
__device__ inline bool ahead(double v, int j, double w, int k) { return v > w || (v == w && j < k); }

// Sorts one (score, index) pair per lane across the warp, best first.
__device__ inline void warp_sort(double& v, int& j) {
  const int lane = threadIdx.x & 31;
  for (int k = 2; k <= 32; k <<= 1)
    for (int h = k >> 1; h > 0; h >>= 1) {
      const double w = __shfl_xor_sync(0xffffffffu, v, h);
      const int q = __shfl_xor_sync(0xffffffffu, j, h);
      const bool first = ((lane & h) == 0) == ((lane & k) == 0);  // keeps the better one
      if (first == ahead(w, q, v, j)) {
        v = w;
        j = q;
      }
    }
}

// Given two best-first sorted warp lists (a, b), leaves the best 32 of their
// union in (a), best first.
__device__ inline void warp_merge(double& av, int& aj, double bv, int bj) {
  const int lane = threadIdx.x & 31;
  // a followed by b reversed is bitonic; keep the better of each mirrored pair
  const double rv = __shfl_sync(0xffffffffu, bv, 31 - lane);
  const int rj = __shfl_sync(0xffffffffu, bj, 31 - lane);
  if (ahead(rv, rj, av, aj)) {
    av = rv;
    aj = rj;
  }
  // the 32 kept form a bitonic sequence: half-cleaners sort it, best first
  for (int h = 16; h > 0; h >>= 1) {
    const double w = __shfl_xor_sync(0xffffffffu, av, h);
    const int q = __shfl_xor_sync(0xffffffffu, aj, h);
    const bool first = (lane & h) == 0;
    if (first == ahead(w, q, av, aj)) {
      av = w;
      aj = q;
    }
  }
}

}  // namespace

template <int D, bool STAGED>
__global__ void __launch_bounds__(kSW * 32) select_screen_kernel(AttnArgs a, Stage1 s1, int qp0,
                                                                int qpb) {
  extern __shared__ __align__(16) unsigned char ss_raw[];
  const int lq = blockIdx.x, qpid = qp0 + lq;
  const Prob pq = prob_of(a.qg, qpid);
  const int kpid = kv_problem(a, qpid);
  const Prob pk = prob_of(a.kg, kpid);
  const int Cq = a.Cq, Ck = a.Ck, K1 = a.topk, ck = pk.C;
  const SelLayout L = sel_layout(D, Ck, STAGED);
  float* mu = reinterpret_cast<float*>(ss_raw + L.mu);
  double* lw = reinterpret_cast<double*>(ss_raw + L.lw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* nu32 = reinterpret_cast<float*>(ss_raw + L.nu32) + warp * D;
  double* nu64 = reinterpret_cast<double*>(ss_raw + L.nu64) + warp * D;
  double* sc = reinterpret_cast<double*>(ss_raw + L.sc) + (size_t)warp * Ck;
  int* cand = reinterpret_cast<int*>(ss_raw + L.cand) + (size_t)warp * Ck;
  __shared__ float mumax_s;
  const float* mu32g = a.ks.cent32 + (size_t)kpid * Ck * D;
  const double* mu64g = a.ks.cent64 + (size_t)kpid * Ck * D;
  const int* kc = a.ks.counts + (size_t)kpid * Ck;
  const bool tilted = a.mode == 2;
  const double s = (double)a.scale;
  const float sf = a.scale;

  // ---- the key problem's centroids (fp32), their largest norm, log n_j -----
  if (tid == 0) mumax_s = 0.f;
  if (STAGED) {
    for (int e = tid; e < ck * (D / 4); e += kSW * 32) {
      const int j = e / (D / 4), q = e - j * (D / 4);
      reinterpret_cast<float4*>(mu + (size_t)j * L.ld)[q] =
          reinterpret_cast<const float4*>(mu32g + (size_t)j * D)[q];
    }
  }
  __syncthreads();
  for (int j = tid; j < ck; j += kSW * 32) {
    const float* r = STAGED ? mu + (size_t)j * L.ld : mu32g + (size_t)j * D;
    float q2 = 0.f;
    for (int d = 0; d < D; ++d) q2 = fmaf(r[d], r[d], q2);
    const float n = sqrtf(q2) * 1.0001f;
    atomicMax(reinterpret_cast<int*>(&mumax_s), __float_as_int(n));
    lw[j] = kc[j] > 0 ? log((double)kc[j]) : -INFINITY;
  }
  __syncthreads();
  const float mumax = mumax_s;
  const int nm = (ck + 31) >> 5;  // clusters per lane

  const int i0 = blockIdx.y * qpb, i1 = imin(pq.C, i0 + qpb);
  for (int i = i0 + warp; i < i1; i += kSW) {  // warp-uniform
    const size_t row = (size_t)qpid * Cq + i;
    for (int d = lane; d < D; d += 32) {
      nu32[d] = a.qs.cent32[row * D + d];
      nu64[d] = a.qs.cent64[row * D + d];
    }
    __syncwarp();
    float nn = 0.f;
    for (int d = lane; d < D; d += 32) nn = fmaf(nu32[d], nu32[d], nn);
    for (int o = 16; o; o >>= 1) nn += __shfl_xor_sync(0xffffffffu, nn, o);
    nn = sqrtf(nn) * 1.0001f;
    const float* lwt = tilted ? s1.logW + ((size_t)lq * Cq + i) * Ck : nullptr;
    // ---- 1. screened scores (fp32), and the largest |log-weight| ----------
    float lwmax = 0.f;
    int nonempty = 0;
    for (int m = 0; m < nm; ++m) {
      const int j = lane + 32 * m;
      float v = -INFINITY;
      if (j < ck && kc[j] > 0) {
        const float* r = STAGED ? mu + (size_t)j * L.ld : mu32g + (size_t)j * D;
        float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll 8
        for (int d = 0; d < D; d += 4) {
          const float4 x = *reinterpret_cast<const float4*>(nu32 + d);
          const float4 y = *reinterpret_cast<const float4*>(r + d);
          p0 = fmaf(x.x, y.x, p0);
          p1 = fmaf(x.y, y.y, p1);
          p2 = fmaf(x.z, y.z, p2);
          p3 = fmaf(x.w, y.w, p3);
        }
        const float l = tilted ? lwt[j] : (float)lw[j];
        v = fmaf(sf, (p0 + p1) + (p2 + p3), l);
        lwmax = fmaxf(lwmax, fabsf(l));
        ++nonempty;
      }
      if (j < ck) sc[j] = (double)v;
    }
    for (int o = 16; o; o >>= 1) {
      lwmax = fmaxf(lwmax, __shfl_xor_sync(0xffffffffu, lwmax, o));
      nonempty += __shfl_xor_sync(0xffffffffu, nonempty, o);
    }
    __syncwarp();
    // ---- 2. the band: T - 2 E below the k1-th screened score ----------------
    // |screen - exact| <= |s| (D + 10) 2^-24 |nu| |mu|max (fp32 centroids and
    // FMA accumulation) + 2^-22 (|s| |nu| |mu|max + |log W|max) (roundings of
    // the product, the log-weight and the sum)
    const float E = fabsf(sf) * (float)(D + 10) * 5.9604645e-08f * nn * mumax +
                    2.3841858e-07f * (fabsf(sf) * nn * mumax + lwmax);
    float lim = -INFINITY;  // every non-empty cluster is a candidate
    if (nonempty > K1 && nm <= 8) {
      // the exact K1-th largest screened score: each lane sorts its (at most
      // eight) scores, then K1 rounds take the warp's best head and advance
      // the winning lane's list
      float v[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int j = lane + 32 * m;
        v[m] = (m < nm && j < ck) ? (float)sc[j] : -INFINITY;
      }
#pragma unroll
      for (int a0 = 0; a0 < 8; ++a0)  // odd-even transposition sort, best first
#pragma unroll
        for (int m = a0 & 1; m + 1 < 8; m += 2)
          if (v[m + 1] > v[m]) {
            const float t = v[m];
            v[m] = v[m + 1];
            v[m + 1] = t;
          }
      float kth = -INFINITY;
      for (int r = 0; r < K1; ++r) {
        float wv = v[0];
        for (int o = 16; o; o >>= 1) wv = fmaxf(wv, __shfl_xor_sync(0xffffffffu, wv, o));
        const unsigned who = __ballot_sync(0xffffffffu, v[0] == wv);
        if (lane == __ffs(who) - 1) {
#pragma unroll
          for (int m = 0; m < 7; ++m) v[m] = v[m + 1];
          v[7] = -INFINITY;
        }
        kth = wv;
      }
      lim = kth - 2.f * E;
    } else if (nonempty > K1 && K1 <= 32) {
      // the K1-th largest of the 32 lane maxima: at least K1 screened scores
      // reach it, so it is no more than the K1-th largest screened score
      double lmax = -INFINITY;
      for (int m = 0; m < nm; ++m) {
        const int j = lane + 32 * m;
        if (j < ck) lmax = fmax(lmax, sc[j]);
      }
      int dummy = lane;
      warp_sort(lmax, dummy);
      lim = (float)__shfl_sync(0xffffffffu, lmax, K1 - 1) - 2.f * E;
    } else if (nonempty > K1) {
      uint32_t taken = 0u;
      float kth = INFINITY;
      for (int r = 0; r < K1; ++r) {
        float bv = -INFINITY;
        int bm = -1;
        for (int m = 0; m < nm; ++m) {
          const int j = lane + 32 * m;
          if (j < ck && !((taken >> m) & 1u)) {
            const float v = (float)sc[j];
            if (v > -INFINITY && (bm < 0 || v > bv)) {
              bv = v;
              bm = m;
            }
          }
        }
        float wv = bv;
        for (int o = 16; o; o >>= 1) wv = fmaxf(wv, __shfl_xor_sync(0xffffffffu, wv, o));
        const unsigned who = __ballot_sync(0xffffffffu, bm >= 0 && bv == wv);
        if (lane == __ffs(who) - 1) taken |= 1u << bm;
        kth = wv;
      }
      lim = kth - 2.f * E;
    }
    // ---- 3. exact scores of the candidates, then the top k1 ---------------
    int nc = 0;
    for (int m = 0; m < nm; ++m) {
      const int j = lane + 32 * m;
      const bool in = j < ck && sc[j] > -INFINITY && (float)sc[j] >= lim;
      const unsigned bal = __ballot_sync(0xffffffffu, in);
      if (in) cand[nc + __popc(bal & ((1u << lane) - 1u))] = j;
      nc += __popc(bal);
      if (j < ck) sc[j] = -INFINITY;  // non-candidates never win
    }
    __syncwarp();
    for (int b = 0; b < nc; b += 32) {
      if (b + lane < nc) {
        const int j = cand[b + lane];
        const double* mr = mu64g + (size_t)j * D;
        double dt = 0.0;
#pragma unroll 16
        for (int d = 0; d < D; ++d) dt = __dadd_rn(dt, __dmul_rn(nu64[d], __ldg(mr + d)));
        const double l = tilted ? (double)lwt[j] : lw[j];
        sc[j] = __dadd_rn(__dmul_rn(s, dt), l);
      }
    }
    __syncwarp();
    int taken = 0;
    int* out = s1.sel + row * (K1 > 0 ? K1 : 1);
    if (K1 <= 32) {
      // best 32 candidates, best first: sorted chunks of 32 merged in turn
      double tv = -INFINITY;
      int tj = 0x7fffffff;
      for (int b = 0; b < nc; b += 32) {
        double v = -INFINITY;
        int j = 0x7fffffff;
        if (b + lane < nc) {
          j = cand[b + lane];
          v = sc[j];
        }
        warp_sort(v, j);
        if (b == 0) {
          tv = v;
          tj = j;
        } else {
          warp_merge(tv, tj, v, j);
        }
      }
      const unsigned ok = __ballot_sync(0xffffffffu, tv > -INFINITY);
      taken = imin(K1, __popc(ok));  // the valid entries lead the list
      if (lane < taken) out[lane] = tj;
    }
    for (int r = 0; K1 > 32 && r < K1; ++r) {
      double bv = -INFINITY;
      int bj = -1;
      for (int q = lane; q < nc; q += 32) {  // candidates are in ascending j
        const int j = cand[q];
        const double v = sc[j];
        if (v > -INFINITY && (bj < 0 || v > bv)) {
          bv = v;
          bj = j;
        }
      }
      for (int o = 16; o; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
        if (oj >= 0 && (bj < 0 || ov > bv || (ov == bv && oj < bj))) {
          bv = ov;
          bj = oj;
        }
      }
      if (bj < 0) break;
      if (lane == 0) out[r] = bj;
      if (lane == 0) sc[bj] = -INFINITY;  // out of the later rounds
      __syncwarp();
      ++taken;
    }
    if (lane == 0) {
      for (int r = taken; r < K1; ++r) out[r] = -1;
      s1.nsel[row] = taken;
    }
    __syncwarp();
  }
}

template <int D>
static void launch_sel(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st) {
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  // query clusters per CTA: enough CTAs to fill the GPU twice, at least one
  // cluster per warp, the whole query problem at most
  long long want = (long long)a.Cq * nqp / (2LL * (nsm > 0 ? nsm : 148));
  int qpb = (int)(want < kSW ? kSW : want);
  qpb = ((qpb + kSW - 1) / kSW) * kSW;
  if (qpb > a.Cq) qpb = a.Cq;
  const dim3 grid(nqp, cdiv(a.Cq, qpb));
  const SelLayout Ls = sel_layout(D, a.Ck, true);
  if (Ls.total <= kSelSmemMax) {
    cudaFuncSetAttribute(select_screen_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)Ls.total);
    select_screen_kernel<D, true><<<grid, kSW * 32, Ls.total, st>>>(a, s1, qp0, qpb);
  } else {
    const SelLayout Lg = sel_layout(D, a.Ck, false);
    cudaFuncSetAttribute(select_screen_kernel<D, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lg.total);
    select_screen_kernel<D, false><<<grid, kSW * 32, Lg.total, st>>>(a, s1, qp0, qpb);
  }
}

void run_select(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st) {
  if (a.qg.D == 64)
    launch_sel<64>(a, s1, qp0, nqp, st);
  else
    launch_sel<128>(a, s1, qp0, nqp, st);
}

}  // namespace muse
