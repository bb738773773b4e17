// Stage 2 of the tilted per-pair dipole (an accuracy variant of TILTED).
//
// TILTED (gist.science page "Multipole Semantic Attention: A Fast
// Approximation of Softmax Attention for Pretraining", Core Mechanisms,
// "Exponential Tilting") summarises key cluster j for query cluster i with
// the weights w_t proportional to exp(s nu_i . k_t): the tilted centroid k^_ij
// and value u^_ij, so the far term reproduces exp(s nu_i . k_t) exactly and
// approximates exp(s (q - nu_i) . k_t) by its value at k^_ij.  The per-pair
// dipole keeps the next term of that expansion about k^_ij:
//     exp(s (q - nu_i) . k_t) ~ exp(s (q - nu_i) . k^_ij) (1 + s (q - nu_i) . (k_t - k^_ij)),
// which adds s M^_ij (q - nu_i) to the value (M^_ij the tilted value-key
// moment about k^_ij) and leaves the weight unchanged (the tilted mean of
// k_t - k^_ij is zero).  Token by token, the far term of (q, j) is the sum
// over t in j of one softmax term with
//     logit   s (q . k^_ij + nu_i . (k_t - k^_ij))   (the denominator's weight),
//     factor  1 + s ((q . k_t - q . k^_ij) - (nu_i . k_t - nu_i . k^_ij)),
// the factor applied to v_t in the numerator only.  A key of a retrieved
// cluster takes the exact term (logit s q . k_t, factor 1).
//
// One CTA per (query set, query cluster i), 32 queries of the cluster per
// pass, the key clusters one after another in 32-key tiles (fp32 SIMT: this
// variant has exact attention's O(N^2 D) cost; it is an accuracy reference).
// Each thread owns a 2 x 2 block of the score tile and 2 rows x D/16 columns
// of the output.
#include "common.cuh"
#include "kernels.h"

namespace muse {

namespace {

constexpr int kTT = 256;  // threads
constexpr int kTW = kTT / 32;
constexpr int kTQr = 32;  // queries per pass
constexpr int kTKr = 32;  // keys per tile

template <int D>
struct TdipSmem {
  float q[kTQr][D + 4];
  float kt[kTKr][D + 4];
  float vt[kTKr][D + 4];
  float wt[kTQr][kTKr + 1];  // p f of the tile
  float kh[D];               // k^_ij
  float nu[D];
  float c[kTQr];             // q . k^_ij
  float bt[kTKr];            // nu . k_t
  float e;                   // nu . k^_ij
  int row[kTQr];
  unsigned rmask[kMaxC / 32];
};

template <typename T, typename TO, int D>
__global__ void __launch_bounds__(kTT) stage2_tdip_kernel(AttnArgs a, Stage1 s1, int qp0) {
  extern __shared__ __align__(16) unsigned char td_raw[];
  TdipSmem<D>& sm = *reinterpret_cast<TdipSmem<D>*>(td_raw);
  const int lq = blockIdx.x, qpid = qp0 + lq, i = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Cq = a.Cq, Ck = a.Ck;
  const Prob pq = prob_of(a.qg, qpid);
  if (i >= pq.C) return;
  const int mi = a.qs.counts[(size_t)qpid * Cq + i];
  if (mi == 0) return;
  const int kpid = kv_problem(a, qpid);
  const Prob pk = prob_of(a.kg, kpid);
  const int ck = pk.C;
  const int* kcnt = a.ks.counts + (size_t)kpid * Ck;
  const int* koff = a.ks.off + (size_t)kpid * (Ck + 1);
  const int* kperm = a.ks.perm + pk.slot0;
  const int qoff = a.qs.off[(size_t)qpid * (Cq + 1) + i];
  const int* qperm = a.qs.perm + pq.slot0;
  const T* Q = static_cast<const T*>(a.qg.X);
  const T* K = static_cast<const T*>(a.kg.X);
  const T* V = static_cast<const T*>(a.V);
  const float s = a.scale;
  constexpr int DV = D / 16;
  const int tq = tid >> 4, tk = tid & 15;
  const size_t ij0 = ((size_t)lq * Cq + i) * Ck;  // this pair row of the stage-1 tables

  for (int w = tid; w < kMaxC / 32; w += kTT) sm.rmask[w] = 0u;
  for (int d = tid; d < D; d += kTT) sm.nu[d] = a.qs.cent32[((size_t)qpid * Cq + i) * D + d];
  __syncthreads();
  int nret = 0;  // keys of the retrieved clusters (the same for every query of i)
  if (a.topk > 0) {
    const int ns = s1.nsel[(size_t)qpid * Cq + i];
    for (int r = tid; r < ns; r += kTT) {
      const int j = s1.sel[((size_t)qpid * Cq + i) * a.topk + r];
      if (j >= 0 && j < ck) atomicOr(&sm.rmask[j >> 5], 1u << (j & 31));
    }
    for (int r = 0; r < ns; ++r) {
      const int j = s1.sel[((size_t)qpid * Cq + i) * a.topk + r];
      if (j >= 0 && j < ck) nret += kcnt[j];
    }
  }
  __syncthreads();

  for (int c0 = 0; c0 < mi; c0 += kTQr) {
    const int qc = imin(kTQr, mi - c0);
    __syncthreads();
    if (tid < kTQr) sm.row[tid] = tid < qc ? qperm[qoff + c0 + tid] : -1;  // problem-local token
    __syncthreads();
    for (int e = tid; e < kTQr * D; e += kTT) {
      const int r = e / D, d = e - r * D;
      sm.q[r][d] = sm.row[r] >= 0 ? ld<T>(Q + (pq.row0 + sm.row[r]) * D + d) : 0.f;
    }
    float o[2][DV], mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
#pragma unroll
    for (int a2 = 0; a2 < 2; ++a2)
#pragma unroll
      for (int v = 0; v < DV; ++v) o[a2][v] = 0.f;
    for (int j = 0; j < ck; ++j) {
      const int nj = kcnt[j];
      if (nj == 0) continue;
      const bool ex = (sm.rmask[j >> 5] >> (j & 31)) & 1u;
      __syncthreads();  // the previous cluster's readers are done
      if (!ex) {
        for (int d = tid; d < D; d += kTT) {
          const size_t o2 = (ij0 + j) * D + d;
          sm.kh[d] = s1.Kfh ? __bfloat162float(s1.Kfh[o2]) + __bfloat162float(s1.Kfl[o2]) : s1.Kf[o2];
        }
        __syncthreads();
        for (int r = warp; r < kTQr; r += kTW) {  // q . k^ per query row, and nu . k^
          float x = 0.f;
          for (int d = lane; d < D; d += 32) x = fmaf(sm.q[r][d], sm.kh[d], x);
#pragma unroll
          for (int o2 = 16; o2; o2 >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o2);
          if (lane == 0) sm.c[r] = x;
        }
        if (warp == 0) {
          float x = 0.f;
          for (int d = lane; d < D; d += 32) x = fmaf(sm.nu[d], sm.kh[d], x);
#pragma unroll
          for (int o2 = 16; o2; o2 >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o2);
          if (lane == 0) sm.e = x;
        }
      }
      for (int t0 = 0; t0 < nj; t0 += kTKr) {
        const int kc = imin(kTKr, nj - t0);
        __syncthreads();
        for (int e2 = tid; e2 < kTKr * D; e2 += kTT) {
          const int r = e2 / D, d = e2 - r * D;
          float kx = 0.f, vx = 0.f;
          if (r < kc) {
            const long long row = pk.row0 + kperm[koff[j] + t0 + r];
            kx = ld<T>(K + row * D + d);
            vx = ld<T>(V + row * D + d);
          }
          sm.kt[r][d] = kx;
          sm.vt[r][d] = vx;
        }
        __syncthreads();
        if (!ex)
          for (int r = warp; r < kTKr; r += kTW) {  // nu . k_t per key
            float x = 0.f;
            for (int d = lane; d < D; d += 32) x = fmaf(sm.nu[d], sm.kt[r][d], x);
#pragma unroll
            for (int o2 = 16; o2; o2 >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o2);
            if (lane == 0) sm.bt[r] = x;
          }
        __syncthreads();
        // the 2 x 2 block of q . k_t (queries 2tq, 2tq+1; keys tk, tk+16)
        float sx[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll 4
        for (int d = 0; d < D; d += 4) {
          float4 qv[2], kv[2];
#pragma unroll
          for (int a2 = 0; a2 < 2; ++a2) {
            qv[a2] = *reinterpret_cast<const float4*>(&sm.q[2 * tq + a2][d]);
            kv[a2] = *reinterpret_cast<const float4*>(&sm.kt[tk + 16 * a2][d]);
          }
#pragma unroll
          for (int a2 = 0; a2 < 2; ++a2)
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2)
              sx[a2][c2] = fmaf(qv[a2].x, kv[c2].x, fmaf(qv[a2].y, kv[c2].y,
                            fmaf(qv[a2].z, kv[c2].z, fmaf(qv[a2].w, kv[c2].w, sx[a2][c2]))));
        }
#pragma unroll
        for (int a2 = 0; a2 < 2; ++a2) {
          const int r = 2 * tq + a2;
          float lg[2], f[2];
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
            const int t = tk + 16 * c2;
            lg[c2] = -INFINITY;
            f[c2] = 0.f;
            if (t < kc) {
              if (ex) {
                lg[c2] = s * sx[a2][c2];
                f[c2] = 1.f;
              } else {
                const float cq = sm.c[r], bt = sm.bt[t], e = sm.e;
                lg[c2] = s * (cq + (bt - e));
                f[c2] = fmaf(s, (sx[a2][c2] - cq) - (bt - e), 1.f);
              }
            }
          }
          float mx = fmaxf(lg[0], lg[1]);
#pragma unroll
          for (int o2 = 8; o2; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
          const float mn = fmaxf(mrow[a2], mx);  // the tile has a live key: mn is finite
          const float sc = __expf(mrow[a2] - mn);
          const float p0 = __expf(lg[0] - mn), p1 = __expf(lg[1] - mn);
          float ps = p0 + p1;
#pragma unroll
          for (int o2 = 8; o2; o2 >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o2);
          lrow[a2] = lrow[a2] * sc + ps;
#pragma unroll
          for (int v = 0; v < DV; ++v) o[a2][v] *= sc;
          mrow[a2] = mn;
          sm.wt[r][tk] = p0 * f[0];
          sm.wt[r][tk + 16] = p1 * f[1];
        }
        __syncthreads();
        // o += (p f) V over the tile's keys
#pragma unroll 4
        for (int t = 0; t < kTKr; ++t) {
          const float w0 = sm.wt[2 * tq][t], w1 = sm.wt[2 * tq + 1][t];
#pragma unroll
          for (int v = 0; v < DV; v += 4) {
            const float4 v4 = *reinterpret_cast<const float4*>(&sm.vt[t][tk * DV + v]);
            o[0][v] = fmaf(w0, v4.x, o[0][v]);
            o[0][v + 1] = fmaf(w0, v4.y, o[0][v + 1]);
            o[0][v + 2] = fmaf(w0, v4.z, o[0][v + 2]);
            o[0][v + 3] = fmaf(w0, v4.w, o[0][v + 3]);
            o[1][v] = fmaf(w1, v4.x, o[1][v]);
            o[1][v + 1] = fmaf(w1, v4.y, o[1][v + 1]);
            o[1][v + 2] = fmaf(w1, v4.z, o[1][v + 2]);
            o[1][v + 3] = fmaf(w1, v4.w, o[1][v + 3]);
          }
        }
      }
    }
    // ---- the rows: the output (acausal) or the level partial (causal) -------
#pragma unroll
    for (int a2 = 0; a2 < 2; ++a2) {
      const int r = 2 * tq + a2;
      if (r >= qc) continue;
      const int tq_ = sm.row[r];
      const float inv = 1.f / lrow[a2];
      if (a.O != nullptr) {
        TO* Ot = static_cast<TO*>(a.O) + (pq.row0 + tq_) * D + tk * DV;
#pragma unroll
        for (int v = 0; v < DV; ++v) st<TO>(Ot + v, o[a2][v] * inv);
        if (tk == 0 && a.n_exact != nullptr) a.n_exact[pq.row0 + tq_] = nret;
      } else {
        float* pp = a.part + (size_t)(pq.slot0 + tq_) * (D + 1);
#pragma unroll
        for (int v = 0; v < DV; ++v) pp[tk * DV + v] = o[a2][v] * inv;
        if (tk == 0) {
          pp[D] = mrow[a2] + __logf(lrow[a2]);
          if (a.n_exact != nullptr)
            atomicAdd(reinterpret_cast<unsigned long long*>(a.n_exact + pq.row0 + tq_),
                      (unsigned long long)nret);
        }
      }
    }
  }
}

template <typename T, typename TO, int D>
void launch_tdip(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st) {
  const size_t sm = sizeof(TdipSmem<D>);
  cudaFuncSetAttribute(stage2_tdip_kernel<T, TO, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)sm);
  stage2_tdip_kernel<T, TO, D><<<dim3(nqp, a.Cq), kTT, sm, st>>>(a, s1, qp0);
}

template <typename T, typename TO>
void dispatch_tdip(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st) {
  if (a.qg.D == 64) launch_tdip<T, TO, 64>(a, s1, qp0, nqp, st);
  else launch_tdip<T, TO, 128>(a, s1, qp0, nqp, st);
}

}  // namespace

void run_stage2_tdip(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st) {
  ProfScope ps(st, "stage2_tdip");
  using bf = __nv_bfloat16;
  if (a.qg.dtype == 0) {
    if (a.out_f32) dispatch_tdip<bf, float>(a, s1, qp0, nqp, st);
    else dispatch_tdip<bf, bf>(a, s1, qp0, nqp, st);
  } else {
    dispatch_tdip<float, float>(a, s1, qp0, nqp, st);
  }
}

}  // namespace muse
