// Key-cluster summaries for a given assignment: count n_j, centroid mu_j,
// monopole sum S_j and dipole moment M_j[e][d] = sum_{t in j} v_t[e] (k_t[d] -
// mu_j[d]) (newx.sg page "Multipole Semantic Attention: A Fast Approximation
// of Softmax Attention for Pretraining", Abstract: monopole plus dipole
// corrections).  One CTA per (b, h, cluster); members are visited in
// ascending token order, so the sums are reproducible.  The attention entry
// points do not call this: they contract the dipole with the query centroid
// directly (stage 1); this is the standalone summary operator.
#include "common.cuh"
#include "kernels.h"

namespace muse {

constexpr int kSm = 256;

template <typename T, int D>
__global__ void __launch_bounds__(kSm) summarize_kernel(const T* K, const T* V, int N, int C,
                                                        const int* assign, int* counts, float* mu_out,
                                                        float* S_out, float* M_out) {
  __shared__ int mem[kSm];
  __shared__ int nmem;
  __shared__ int wcnt[kSm / 32];
  __shared__ float mus[D];
  __shared__ float kt[32][D + 1];
  __shared__ float vt[32][D + 1];
  const int bh = blockIdx.x, c = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int* a = assign + (size_t)bh * N;
  const T* Kb = K + (size_t)bh * N * D;
  const T* Vb = V + (size_t)bh * N * D;
  double sk = 0.0, sv = 0.0;  // thread d < D
  int total = 0;
  // pass 1: count, sum k, sum v
  for (int t0 = 0; t0 < N; t0 += kSm) {
    const int t = t0 + tid;
    const bool in = t < N && a[t] == c;
    const unsigned bal = __ballot_sync(0xffffffffu, in);
    if (lane == 0) wcnt[warp] = __popc(bal);
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += wcnt[w];
    if (in) mem[base + __popc(bal & ((1u << lane) - 1u))] = t;
    if (tid == 0) {
      int n = 0;
      for (int w = 0; w < kSm / 32; ++w) n += wcnt[w];
      nmem = n;
    }
    __syncthreads();
    const int n = nmem;
    if (tid < D)
      for (int m = 0; m < n; ++m) {
        sk += (double)ld<T>(Kb + (size_t)mem[m] * D + tid);
        sv += (double)ld<T>(Vb + (size_t)mem[m] * D + tid);
      }
    total += n;
    __syncthreads();
  }
  if (tid < D) {
    const float m = total > 0 ? (float)(sk / (double)total) : 0.f;
    mus[tid] = m;
    if (mu_out) mu_out[((size_t)bh * C + c) * D + tid] = m;
    if (S_out) S_out[((size_t)bh * C + c) * D + tid] = (float)sv;
  }
  if (tid == 0 && counts) counts[(size_t)bh * C + c] = total;
  if (M_out == nullptr) return;
  __syncthreads();
  // pass 2: M[e][d] = sum v[e] (k[d] - mu[d]); thread owns entries tid, tid + kSm, ...
  constexpr int E = D * D / kSm;
  float acc[E];
#pragma unroll
  for (int r = 0; r < E; ++r) acc[r] = 0.f;
  for (int t0 = 0; t0 < N; t0 += kSm) {
    const int t = t0 + tid;
    const bool in = t < N && a[t] == c;
    const unsigned bal = __ballot_sync(0xffffffffu, in);
    if (lane == 0) wcnt[warp] = __popc(bal);
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += wcnt[w];
    if (in) mem[base + __popc(bal & ((1u << lane) - 1u))] = t;
    if (tid == 0) {
      int n = 0;
      for (int w = 0; w < kSm / 32; ++w) n += wcnt[w];
      nmem = n;
    }
    __syncthreads();
    const int n = nmem;
    for (int m0 = 0; m0 < n; m0 += 32) {
      const int cnt = imin(32, n - m0);
      for (int e = tid; e < cnt * D; e += kSm) {
        const int r = e / D, d = e - r * D;
        kt[r][d] = ld<T>(Kb + (size_t)mem[m0 + r] * D + d) - mus[d];
        vt[r][d] = ld<T>(Vb + (size_t)mem[m0 + r] * D + d);
      }
      __syncthreads();
#pragma unroll
      for (int r = 0; r < E; ++r) {
        const int idx = tid + r * kSm, e = idx / D, d = idx - e * D;
        float s = acc[r];
        for (int m = 0; m < cnt; ++m) s = fmaf(vt[m][e], kt[m][d], s);
        acc[r] = s;
      }
      __syncthreads();
    }
  }
  float* Mo = M_out + ((size_t)bh * C + c) * D * D;
#pragma unroll
  for (int r = 0; r < E; ++r) Mo[tid + r * kSm] = acc[r];
}

void run_summarize(const void* K, const void* V, int dtype, int BH, int N, int D, int C,
                   const int* assign, int* counts, float* mu, float* S, float* M, int*, int*,
                   cudaStream_t st) {
  dim3 grid(BH, C);
  ProfScope ps(st, "summarize");
  if (dtype == 0) {
    auto k = static_cast<const __nv_bfloat16*>(K);
    auto v = static_cast<const __nv_bfloat16*>(V);
    if (D == 64) summarize_kernel<__nv_bfloat16, 64><<<grid, kSm, 0, st>>>(k, v, N, C, assign, counts, mu, S, M);
    else summarize_kernel<__nv_bfloat16, 128><<<grid, kSm, 0, st>>>(k, v, N, C, assign, counts, mu, S, M);
  } else {
    auto k = static_cast<const float*>(K);
    auto v = static_cast<const float*>(V);
    if (D == 64) summarize_kernel<float, 64><<<grid, kSm, 0, st>>>(k, v, N, C, assign, counts, mu, S, M);
    else summarize_kernel<float, 128><<<grid, kSm, 0, st>>>(k, v, N, C, assign, counts, mu, S, M);
  }
}

}  // namespace muse
