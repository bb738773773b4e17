// Shared end of the k-means assignment kernels: fp64 re-decision of the
// tokens whose screen could not certify the nearest centroid, the write of
// the assignment, the tile histogram, and -- by the last tile of the problem
// to finish -- the cluster offsets and per-tile scatter bases.
#pragma once

#include "common.cuh"

namespace muse {

// flagged/decision: smem [kTile]; hist: smem [C] zeroed; nflag: smem, 0.
template <int D, typename XRow>
__device__ inline void assign_tail(const RoleGeo& g, const KState& ks, const Prob& p, int pid,
                                   int t0, int nt, int best, bool flag, XRow xrow, int* hist,
                                   int* flagged, int* decision, int* nflag, int* is_last) {
  const int tid = threadIdx.x;
  const int C = p.C;
  const bool valid = tid < nt;
  const double* c64 = ks.cent64 + (size_t)pid * g.C * D;
  if (valid && flag) {
    int slot = atomicAdd(nflag, 1);
    flagged[slot] = tid;
  }
  __syncthreads();
  // fp64 re-decision, one warp per flagged token, lanes over clusters; the
  // distance is accumulated in dimension order without fused operations so
  // it equals a plain sequential fp64 evaluation bit for bit.
  const int warp = tid >> 5, lane = tid & 31;
  const int nf = *nflag;
  for (int f = warp; f < nf; f += kTile / 32) {
    const int r = flagged[f];
    double bdd = 0.0;
    int bc = -1;
    for (int c = lane; c < C; c += 32) {
      const double* cc = c64 + (size_t)c * D;
      double s = 0.0;
      for (int d = 0; d < D; ++d) {
        double t = __dsub_rn((double)xrow(r, d), cc[d]);
        s = __dadd_rn(s, __dmul_rn(t, t));
      }
      if (bc < 0 || s < bdd) {
        bdd = s;
        bc = c;
      }
    }
    for (int o = 16; o; o >>= 1) {
      double od = __shfl_xor_sync(0xffffffffu, bdd, o);
      int oc = __shfl_xor_sync(0xffffffffu, bc, o);
      if (oc >= 0 && (bc < 0 || od < bdd || (od == bdd && oc < bc))) {
        bdd = od;
        bc = oc;
      }
    }
    if (lane == 0) decision[r] = bc;
  }
  __syncthreads();
  if (valid) {
    if (flag) best = decision[tid];
    ks.assign[p.slot0 + t0 + tid] = best;
    atomicAdd(&hist[best], 1);
  }
  __syncthreads();
  int* th = ks.hist + (size_t)blockIdx.x * g.C;
  for (int i = tid; i < C; i += blockDim.x) th[i] = hist[i];
  // the last tile of the problem turns histograms into offsets and bases
  __threadfence();
  __syncthreads();
  const int ntp = cdiv(p.s, kTile);
  if (tid == 0) *is_last = (atomicAdd(&ks.arrive[pid], 1) == ntp - 1);
  __syncthreads();
  if (!*is_last) return;
  __threadfence();
  int* ph = ks.hist + (size_t)p.tile0 * g.C;
  int* cnt = ks.counts + (size_t)pid * g.C;
  int* off = ks.off + (size_t)pid * (g.C + 1);
  constexpr int U = 16;  // tile counts fetched per round trip
  for (int c = tid; c < C; c += blockDim.x) {
    int tot = 0;
    for (int t0 = 0; t0 < ntp; t0 += U) {
      int v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) v[u] = (t0 + u < ntp) ? __ldcg(ph + (size_t)(t0 + u) * g.C + c) : 0;
#pragma unroll
      for (int u = 0; u < U; ++u) tot += v[u];
    }
    hist[c] = tot;
    cnt[c] = tot;
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int c = 0; c < C; ++c) {
      off[c] = run;
      int v = hist[c];
      hist[c] = run;
      run += v;
    }
    off[C] = run;
    ks.arrive[pid] = 0;
  }
  __syncthreads();
  for (int c = tid; c < C; c += blockDim.x) {
    int run = hist[c];
    for (int t0 = 0; t0 < ntp; t0 += U) {
      int v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) v[u] = (t0 + u < ntp) ? __ldcg(ph + (size_t)(t0 + u) * g.C + c) : 0;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (t0 + u < ntp) ph[(size_t)(t0 + u) * g.C + c] = run;
        run += v[u];
      }
    }
  }
}

}  // namespace muse
