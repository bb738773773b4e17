// Lloyd k-means over many token blocks at once (the clustering step of
// MuSe: queries and keys are clustered separately, each in its own space --
// "Multipole Semantic Attention" gist.science page, Technical Summary, Core
// Mechanisms, "Bidirectional Semantic Clustering").
//
// One round = assign -> scatter -> reduce:
//   assign   128 tokens per CTA.  An fp32 screen computes every squared
//            distance together with a certified error bound; a token whose
//            best and runner-up bounds overlap is re-decided in fp64 with the
//            same operation order as a plain sequential evaluation, ties to
//            the lowest index.  The CTA writes its per-cluster histogram; the
//            last CTA of each problem to finish turns the histograms into
//            cluster offsets and per-tile scatter bases.
//   scatter  stable counting-sort scatter: perm lists each problem's tokens
//            grouped by cluster, ascending token order inside a cluster.
//   reduce   one warp per (problem, cluster): fp64 sum of the members in
//            ascending token order, divided by the count; an empty cluster
//            keeps its centroid.
// Every reduction has a fixed order, so results are bitwise reproducible and
// the centroids equal a sequential fp64 evaluation of the same means.
#include "common.cuh"
#include "kernels.h"
#include "kmeans_tail.cuh"

namespace muse {

// ----------------------------------------------------------------------------
// seeded start: splitmix64-driven partial Fisher-Yates over the block rows
// ----------------------------------------------------------------------------
__device__ inline uint64_t splitmix64_next(uint64_t& state) {
  uint64_t z = (state += 0x9E3779B97F4A7C15ULL);
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

// r mod m for a 32-bit m, exactly: reduce the high word first, then the
// remaining < m * 2^32 by a double-precision quotient estimate and an exact
// integer correction (the generic 64-bit remainder is a long software loop).
__device__ inline uint32_t mod_u64_u32(uint64_t r, uint32_t m) {
  if (m < (1u << 16)) return (uint32_t)(r % m);
  const uint64_t t = ((uint64_t)((uint32_t)(r >> 32) % m) << 32) | (uint32_t)r;
  uint64_t q = (uint64_t)((double)t / (double)m);
  long long rem = (long long)(t - q * (uint64_t)m);
  while (rem < 0) rem += m;
  while (rem >= (long long)m) rem -= m;
  return (uint32_t)rem;
}

// Both roles' problems in one launch: CTAs [0, nblk0) serve set 0.  Each
// problem is split over `nsplit` CTAs, each writing a slice of the rows.
struct InitSets {
  RoleGeo g[2];
  KState ks[2];
  int nblk0;
  int nsplit;
};

template <typename T>
__global__ void __launch_bounds__(256) kmeans_init_kernel(InitSets is, const float* init) {
  __shared__ int jd[kMaxC];
  __shared__ int pick[kMaxC];
  const int set = (int)blockIdx.x < is.nblk0 ? 0 : 1;
  const RoleGeo& g = is.g[set];
  const KState& ks = is.ks[set];
  const int blk = (int)blockIdx.x - (set ? is.nblk0 : 0);
  const int pid = blk / is.nsplit, part = blk - pid * is.nsplit;
  const Prob p = prob_of(g, pid);
  const int D = g.D, C = p.C;
  const int rows = cdiv(C, is.nsplit);
  const int cb = part * rows, ce = imin(C, cb + rows);  // this CTA's rows
  const T* X = static_cast<const T*>(g.X);
  double* c64 = ks.cent64 + (size_t)pid * g.C * D;
  float* c32 = ks.cent32 + (size_t)pid * g.C * D;
  if (init == nullptr) {
    // Partial Fisher-Yates: step c swaps positions c and j_c = c + (r_c mod
    // (n - c)) of the identity and picks the new value at c.  splitmix64 is
    // counter based (draw c uses state0 + (c + 1) * gamma), so every j_c is
    // drawn in parallel.  The swaps are resolved without replaying them: the
    // value at a position pos >= s before step s is the value that stood at
    // position c' before step c', for the latest c' < s with j_c' = pos (step
    // c' moved it there), else pos itself; the recursion ends because c' < pos.
    const uint64_t st0 = g.seed + 0x9E3779B97F4A7C15ULL * (2ULL * p.sid + (uint64_t)g.role + 1ULL);
    const int n = p.s;
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
      uint64_t st = st0 + 0x9E3779B97F4A7C15ULL * (uint64_t)c;
      const uint64_t r = splitmix64_next(st);
      jd[c] = c + (int)mod_u64_u32(r, (uint32_t)(n - c));
    }
    __syncthreads();
    for (int c = cb + (int)threadIdx.x; c < ce; c += blockDim.x) {
      int pos = jd[c], s = c;
      for (;;) {
        int f = s - 1;
        while (f >= 0 && jd[f] != pos) --f;
        if (f < 0) break;
        pos = f;
        s = f;
      }
      pick[c] = pos;
    }
    __syncthreads();
  }
  if (sizeof(T) == 2) {
    // exponent range of the problem's values: the exactness certificate of
    // the order-free centroid sums (sums_exact); this CTA scans its share of
    // the problem's rows, 8 bf16 values per 16-byte load
    const int per = cdiv(p.s, is.nsplit);
    const int t0 = part * per, t1 = imin(p.s, t0 + per);
    int lo = 1 << 30, hi = -1;
    if (t1 > t0) {
      const uint4* xv = reinterpret_cast<const uint4*>(X + (p.row0 + t0) * D);
      const int nv = (t1 - t0) * D / 8;
      for (int i0 = threadIdx.x; i0 < nv; i0 += 4 * blockDim.x) {
        uint4 v[4];  // four loads in flight; zero words count for nothing
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + u * (int)blockDim.x;
          v[u] = i < nv ? xv[i] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t b = (w[k >> 1] >> (16 * (k & 1))) & 0xFFFFu;
            if (b & 0x7FFFu) {
              const int e = (int)((b >> 7) & 0xFFu);
              lo = min(lo, e > 0 ? e : 1);
              hi = max(hi, e);
            }
          }
        }
      }
    }
    for (int o = 16; o; o >>= 1) {
      lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if ((threadIdx.x & 31) == 0 && hi >= 0) {
      atomicMin(ks.emin + pid, lo);
      atomicMax(ks.emax + pid, hi);
    }
  }
  // one warp per centroid row, four rows per step (loads issued together):
  // fp64/fp32 copies, the bf16 split for the tensor cores, and the norms
  const float* src = init ? init + (size_t)p.bh * g.C * D : nullptr;  // muse_cluster: one problem per bh
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  constexpr int RR = 4;
  for (int c0 = cb + warp * RR; c0 < ce; c0 += nw * RR) {
    float v[RR][4];
#pragma unroll
    for (int u = 0; u < RR; ++u)
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int c = c0 + u, d = lane + 32 * r;
        v[u][r] = 0.f;
        if (c < ce && d < D)
          v[u][r] = src ? src[(size_t)c * D + d] : ld<T>(X + (p.row0 + pick[c]) * D + d);
      }
#pragma unroll
    for (int u = 0; u < RR; ++u) {
      const int c = c0 + u;
      if (c >= ce) break;
      float s = 0.f;
      double s2 = 0.0;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int d = lane + 32 * r;
        if (d >= D) break;
        const size_t i = (size_t)c * D + d;
        const float x = v[u][r];
        c64[i] = (double)x;
        c32[i] = x;
        s = fmaf(x, x, s);
        s2 += (double)x * (double)x;
        const __nv_bfloat16 hi = __float2bfloat16_rn(x);
        ks.cbf_hi[(size_t)pid * g.C * D + i] = hi;
        ks.cbf_lo[(size_t)pid * g.C * D + i] = __float2bfloat16_rn(x - __bfloat162float(hi));
      }
      for (int o = 16; o; o >>= 1) {
        s += __shfl_xor_sync(0xffffffffu, s, o);
        s2 += __shfl_xor_sync(0xffffffffu, s2, o);
      }
      if (lane == 0) {
        ks.cnorm[(size_t)pid * g.C + c] = sqrtf(s) * 1.0001f;
        ks.cn2[(size_t)pid * g.C + c] = (float)s2;
      }
    }
  }
}

// ----------------------------------------------------------------------------
// assign: fp32 screen with a certified bound, fp64 re-decision of near ties
// ----------------------------------------------------------------------------
constexpr int kChunk = 32;

template <int D>
constexpr size_t assign_smem() {
  return ((size_t)kTile * (D + 1) + (size_t)kChunk * D + kMaxC) * sizeof(float) +
         kMaxC * sizeof(int);
}

template <typename T, int D>
__global__ void __launch_bounds__(kTile) kmeans_assign_kernel(RoleGeo g, KState ks) {
  extern __shared__ float as_dyn[];
  float(*xs)[D + 1] = reinterpret_cast<float(*)[D + 1]>(as_dyn);
  float(*cs)[D] = reinterpret_cast<float(*)[D]>(as_dyn + kTile * (D + 1));
  float* cn = as_dyn + kTile * (D + 1) + kChunk * D;
  int* hist = reinterpret_cast<int*>(cn + kMaxC);
  __shared__ int flagged[kTile];
  __shared__ int decision[kTile];
  __shared__ int nflag;
  __shared__ int is_last;

  int pid, tin;
  tile_of(g, blockIdx.x, &pid, &tin);
  const Prob p = prob_of(g, pid);
  const int C = p.C;
  const int t0 = tin * kTile;
  const int nt = imin(kTile, p.s - t0);
  const T* X = static_cast<const T*>(g.X);
  const float* c32 = ks.cent32 + (size_t)pid * g.C * D;
  const int tid = threadIdx.x;

  for (int i = tid; i < C; i += kTile) {
    cn[i] = ks.cnorm[(size_t)pid * g.C + i];
    hist[i] = 0;
  }
  if (tid == 0) nflag = 0;
  for (int i = tid; i < nt * D; i += kTile) {
    int r = i / D, d = i - r * D;
    xs[r][d] = ld<T>(X + (p.row0 + t0 + r) * D + d);
  }
  __syncthreads();

  const bool valid = tid < nt;
  float xn = 0.f;
  for (int d = 0; d < D; ++d) xn = fmaf(xs[tid][d], xs[tid][d], xn);
  xn = sqrtf(xn) * 1.0001f;
  // |d~ - d| <= u (D+4) d~ + 2.01 u (|x| + |c|) |c|   (u = 2^-24), see the
  // derivation in the design notes: fp32 rounding of the centroid, of each
  // difference and of each fused square-accumulate.
  const float u = 5.9604645e-08f;
  const float ea = u * (float)(D + 4), eb = 2.01f * u;
  float bd = INFINITY, be = 0.f, blb = INFINITY, olb = INFINITY;
  int best = 0;
  for (int c0 = 0; c0 < C; c0 += kChunk) {
    const int cc = imin(kChunk, C - c0);
    __syncthreads();
    for (int i = tid; i < cc * D; i += kTile) cs[i / D][i % D] = c32[(size_t)c0 * D + i];
    __syncthreads();
    if (valid) {
      for (int k = 0; k < cc; ++k) {
        float dd = 0.f;
#pragma unroll 16
        for (int d = 0; d < D; ++d) {
          float t = xs[tid][d] - cs[k][d];
          dd = fmaf(t, t, dd);
        }
        const float cnk = cn[c0 + k];
        const float e = fmaf(ea, dd, eb * (xn + cnk) * cnk);
        const float lb = dd - e;
        if (dd < bd) {
          olb = fminf(olb, blb);
          bd = dd;
          be = e;
          blb = lb;
          best = c0 + k;
        } else {
          olb = fminf(olb, lb);
        }
      }
    }
  }
  auto xrow = [&](int r, int d) { return xs[r][d]; };
  assign_tail<D>(g, ks, p, pid, t0, nt, best, valid && olb <= bd + be, xrow, hist, flagged,
                 decision, &nflag, &is_last);
}

// ----------------------------------------------------------------------------
// scatter: stable counting sort of each problem's tokens by cluster
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(kTile) kmeans_scatter_kernel(RoleGeo g, KState ks) {
  __shared__ int cnt[kMaxC];
  int pid, tin;
  tile_of(g, blockIdx.x, &pid, &tin);
  const Prob p = prob_of(g, pid);
  const int t0 = tin * kTile;
  const int nt = imin(kTile, p.s - t0);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < p.C; i += kTile) cnt[i] = 0;
  __syncthreads();
  const int* base = ks.hist + (size_t)blockIdx.x * g.C;
  const bool valid = tid < nt;
  const int a = valid ? ks.assign[p.slot0 + t0 + tid] : -1 - tid;
  const unsigned same = __match_any_sync(0xffffffffu, a);
  const int rank = __popc(same & ((1u << lane) - 1u));
  for (int w = 0; w < kTile / 32; ++w) {
    if (warp == w && valid) {
      ks.perm[p.slot0 + base[a] + cnt[a] + rank] = t0 + tid;
    }
    __syncthreads();
    if (warp == w && valid && rank == 0) cnt[a] += __popc(same);
    __syncthreads();
  }
}

// ----------------------------------------------------------------------------
// reduce: centroid = fp64 mean of the members in ascending token order
// ----------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256) kmeans_reduce_kernel(RoleGeo g, KState ks) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long gw = (long long)blockIdx.x * 8 + warp;
  const int pid = (int)(gw / g.C), c = (int)(gw - (long long)pid * g.C);
  if (pid >= ks.nprob) return;
  const Prob p = prob_of(g, pid);
  if (c >= p.C) return;
  const int* off = ks.off + (size_t)pid * (g.C + 1);
  const int b = off[c], e = off[c + 1];
  double* c64 = ks.cent64 + ((size_t)pid * g.C + c) * D;
  float* c32 = ks.cent32 + ((size_t)pid * g.C + c) * D;
  constexpr int R = D / 32;
  if (e > b) {
    const T* X = static_cast<const T*>(g.X);
    const int* perm = ks.perm + p.slot0;
    double s[R];
#pragma unroll
    for (int r = 0; r < R; ++r) s[r] = 0.0;
    constexpr int U = 8;  // members loaded ahead; the adds stay in token order
    int m = b;
    for (; m + U <= e; m += U) {
      float v[U][R];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const T* row = X + (p.row0 + perm[m + u]) * D;
#pragma unroll
        for (int r = 0; r < R; ++r) v[u][r] = ld<T>(row + lane + 32 * r);
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int r = 0; r < R; ++r) s[r] = __dadd_rn(s[r], (double)v[u][r]);
    }
    for (; m < e; ++m) {
      const T* row = X + (p.row0 + perm[m]) * D;
#pragma unroll
      for (int r = 0; r < R; ++r) s[r] = __dadd_rn(s[r], (double)ld<T>(row + lane + 32 * r));
    }
    const double n = (double)(e - b);
    double q2 = 0.0;
    float q = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const double v = __ddiv_rn(s[r], n);
      const float v32 = (float)v;
      const size_t i = ((size_t)pid * g.C + c) * D + lane + 32 * r;
      c64[lane + 32 * r] = v;
      c32[lane + 32 * r] = v32;
      const __nv_bfloat16 hi = __float2bfloat16_rn(v32);
      ks.cbf_hi[i] = hi;
      ks.cbf_lo[i] = __float2bfloat16_rn(v32 - __bfloat162float(hi));
      q2 += v * v;
      q = fmaf(v32, v32, q);
    }
    for (int o = 16; o; o >>= 1) {
      q += __shfl_xor_sync(0xffffffffu, q, o);
      q2 += __shfl_xor_sync(0xffffffffu, q2, o);
    }
    if (lane == 0) {
      ks.cnorm[(size_t)pid * g.C + c] = sqrtf(q) * 1.0001f;
      ks.cn2[(size_t)pid * g.C + c] = (float)q2;
    }
  }
}

// ----------------------------------------------------------------------------
// host-side launchers
// ----------------------------------------------------------------------------
template <typename T, int D>
static void launch_round(const RoleGeo& g, const KState& ks, cudaStream_t st) {
  // set on every launch: the attribute is per device, and the call is cheap
  cudaFuncSetAttribute(kmeans_assign_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)assign_smem<D>());
  {
    ProfScope ps(st, "kmeans_assign");
    if (sizeof(T) == 2)
      launch_assign_tc(g, ks, st);
    else
      kmeans_assign_kernel<T, D><<<(unsigned)ks.ntiles, kTile, assign_smem<D>(), st>>>(g, ks);
  }
  {
    ProfScope ps(st, "kmeans_scatter");
    kmeans_scatter_kernel<<<(unsigned)ks.ntiles, kTile, 0, st>>>(g, ks);
  }
  const long long warps = (long long)ks.nprob * g.C;
  {
    ProfScope ps(st, "kmeans_reduce");
    kmeans_reduce_kernel<T, D><<<(unsigned)cdiv((int)warps, 8), 256, 0, st>>>(g, ks);
  }
}

template <typename T>
static void init_t(const RoleGeo* gs, const KState* kss, int nsets, const float* init,
                   cudaStream_t st) {
  ProfScope ps(st, "kmeans_init");
  InitSets is{};
  for (int k = 0; k < nsets; ++k) {
    is.g[k] = gs[k];
    is.ks[k] = kss[k];
  }
  const int nprob = kss[0].nprob + (nsets > 1 ? kss[1].nprob : 0);
  if (sizeof(T) == 2)
    for (int k = 0; k < nsets; ++k) {  // empty ranges: emin = 0x7F7F7F7F > emax = 0x80808080
      cudaMemsetAsync(kss[k].emin, 0x7F, (size_t)kss[k].nprob * 4, st);
      cudaMemsetAsync(kss[k].emax, 0x80, (size_t)kss[k].nprob * 4, st);
    }
  is.nsplit = nprob >= 148 ? 1 : 8;  // spread few problems over more SMs
  is.nblk0 = kss[0].nprob * is.nsplit;
  const int nblk = nprob * is.nsplit;
  kmeans_init_kernel<T><<<(unsigned)nblk, 256, 0, st>>>(is, init);
}

void run_kmeans_init(const RoleGeo* gs, const KState* kss, int nsets, const float* init,
                     cudaStream_t st) {
  if (gs[0].dtype == 0)
    init_t<__nv_bfloat16>(gs, kss, nsets, init, st);
  else
    init_t<float>(gs, kss, nsets, init, st);
}

template <typename T>
static void rounds_t(const RoleGeo& g, const KState& ks, int iters, cudaStream_t st) {
  for (int it = 0; it < iters; ++it) {
    if (g.D == 64)
      launch_round<T, 64>(g, ks, st);
    else
      launch_round<T, 128>(g, ks, st);
  }
}

void run_kmeans_rounds(const RoleGeo& g, const KState& ks, int iters, cudaStream_t st) {
  if (g.dtype == 0)
    rounds_t<__nv_bfloat16>(g, ks, iters, st);
  else
    rounds_t<float>(g, ks, iters, st);
}

void run_kmeans(const RoleGeo& g, const KState& ks, int iters, const float* init, cudaStream_t st) {
  run_kmeans_init(&g, &ks, 1, init, st);
  run_kmeans_rounds(g, ks, iters, st);
}

}  // namespace muse
