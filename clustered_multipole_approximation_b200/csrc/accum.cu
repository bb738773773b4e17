// Causal operator with causal accumulation of block summaries and two-level
// retrieval (gist.science page "Multipole Semantic Attention: A Fast
// Approximation of Softmax Attention for Pretraining", Technical Summary,
// Core Mechanisms: "Causal Accumulation" and "Retrieval-Augmented
// Approximation").
//
// Both roles are clustered over the whole sequence of a (b, head) (the
// acausal clustering).  The sequence is cut into blocks of L tokens.  Per
// (key cluster j, block b): n_jb, the key sum (fp64) and the value sum, and for
// DIPOLE, per query cluster i, A_ijb = sum_{t in (j, b)} v_t (k_t . nu_i)
// (so that M nu_i = A - S (mu . nu_i) over any union of blocks).  The
// summaries a query block b reads are the exclusive prefix over blocks
// 0 .. b-1, accumulated in block order.  Per (query cluster i, block b):
//   1. top-k1 key clusters by s nu_i . mu_j^{<b} + log n_j^{<b} (fp64, the
//      dot product in dimension order, ties to the lowest j);
//   2. per selected j, top-k2 blocks b' < b by s nu_i . mu_jb' + log n_jb';
//   3. one online softmax over the keys of the retrieved (j, b') pairs
//      (exact) and, per key cluster, the summary of its prefix members outside
//      the retrieved blocks (far: logit s q.mu + log n, value S / n or
//      (S + s M nu_i) / n); the result enters the local block's softmax as one
//      term (normalised output, log-sum-exp), merged by the causal local
//      kernels.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace muse {

namespace {

constexpr int kAT = 256;
constexpr int kAW = kAT / 32;

// ---------------------------------------------------------------------------
// per (set, cluster): members per block (counts, first member of each block)
// and, for keys, the block key sums (fp64, token order) and value sums
// ---------------------------------------------------------------------------
template <typename T, int D, bool KEYS>
__global__ void __launch_bounds__(kAT) acc_block_stats_kernel(AttnArgs a, AccArgs c) {
  const int pid = blockIdx.x, j = blockIdx.y, tid = threadIdx.x;
  const RoleGeo& g = KEYS ? a.kg : a.qg;
  const KState& ks = KEYS ? a.ks : a.qs;
  const int C = KEYS ? a.Ck : a.Cq, NB = c.NB, L = c.L;
  const Prob p = prob_of(g, pid);
  const size_t cj = (size_t)pid * C + j;
  const int n = ks.counts[cj];
  const int off = ks.off[(size_t)pid * (C + 1) + j];
  const int* perm = ks.perm + p.slot0 + off;
  int* boff = (KEYS ? c.kboff : c.qboff) + cj * (NB + 1);
  // first member of each block: members are in token order within a cluster
  for (int b = tid; b <= NB; b += kAT) {
    int lo = 0, hi = n;
    const int t = b * L;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (perm[mid] < t) lo = mid + 1;
      else hi = mid;
    }
    boff[b] = lo;
  }
  if (!KEYS) return;
  const T* K = static_cast<const T*>(a.kg.X);
  const T* V = static_cast<const T*>(a.V);
  for (int d = tid; d < D; d += kAT) {
    double sk = 0.0;
    float sv = 0.f;
    int cur = n > 0 ? perm[0] / L : 0, cnt = 0;
    for (int m = 0; m < n; ++m) {
      const int t = perm[m], b = t / L;
      if (b != cur) {
        const size_t o = ((size_t)pid * NB + cur) * C + j;
        c.bk[o * D + d] = sk;
        c.bs[o * D + d] = sv;
        if (d == 0) c.bn[o] = cnt;
        sk = 0.0;
        sv = 0.f;
        cnt = 0;
        cur = b;
      }
      const long long row = p.row0 + t;
      sk += (double)ld<T>(K + row * D + d);
      sv += ld<T>(V + row * D + d);
      ++cnt;
    }
    if (n > 0) {
      const size_t o = ((size_t)pid * NB + cur) * C + j;
      c.bk[o * D + d] = sk;
      c.bs[o * D + d] = sv;
      if (d == 0) c.bn[o] = cnt;
    }
  }
}

// exclusive prefix over blocks, in block order: one thread per (set, j, d)
template <int D>
__global__ void acc_prefix_kernel(AttnArgs a, AccArgs c) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int Ck = a.Ck, NB = c.NB;
  const long long total = (long long)a.ks.nprob * Ck * D;
  if (e >= total) return;
  const int d = (int)(e % D);
  const long long pj = e / D;  // pid * Ck + j
  const int pid = (int)(pj / Ck), j = (int)(pj - (long long)pid * Ck);
  double pk = 0.0;
  float ps = 0.f;
  int pn = 0;
  for (int b = 0; b < NB; ++b) {
    const size_t o = ((size_t)pid * NB + b) * Ck + j;
    const int bn = c.bn[o];
    const double bk = c.bk[o * D + d];
    c.pk[o * D + d] = pk;
    c.ps[o * D + d] = ps;
    // centroids of the prefix and of the block, for the selection scores
    // prefix centroids [set][b][d][j] (a warp reads consecutive j), block
    // centroids [set][j][d][b] (a warp reads consecutive b)
    c.pmu[(((size_t)pid * NB + b) * D + d) * Ck + j] = pn > 0 ? __ddiv_rn(pk, (double)pn) : 0.0;
    c.bmu[(((size_t)pid * Ck + j) * D + d) * NB + b] = bn > 0 ? __ddiv_rn(bk, (double)bn) : 0.0;
    if (d == 0) c.pn[o] = pn;
    pk += bk;
    ps += c.bs[o * D + d];
    pn += bn;
  }
}

// ---------------------------------------------------------------------------
// DIPOLE: A_ijb = sum_{t in (j, b)} v_t (k_t . nu_i) for every query cluster i
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(kAT) acc_block_a_kernel(AttnArgs a, AccArgs c) {
  extern __shared__ __align__(16) float aa_raw[];
  const int Cq = a.Cq, Ck = a.Ck, NB = c.NB, L = c.L;
  float* nu = aa_raw;                     // [Cq][D + 1]
  float* kt = nu + Cq * (D + 1);          // [32][D + 1]
  float* vt = kt + 32 * (D + 1);          // [32][D]
  float* gt = vt + 32 * D;                // [32][Cq]
  int* tb = reinterpret_cast<int*>(gt + 32 * Cq);  // [32] block of each member
  const int qpid = blockIdx.x, j = blockIdx.y, tid = threadIdx.x;
  const int kpid = kv_problem(a, qpid);
  const Prob pk = prob_of(a.kg, kpid);
  const size_t cj = (size_t)kpid * Ck + j;
  const int n = a.ks.counts[cj];
  const int off = a.ks.off[(size_t)kpid * (Ck + 1) + j];
  const int* perm = a.ks.perm + pk.slot0 + off;
  const T* K = static_cast<const T*>(a.kg.X);
  const T* V = static_cast<const T*>(a.V);
  for (int e = tid; e < Cq * D; e += kAT) {
    const int i = e / D, d = e - i * D;
    nu[i * (D + 1) + d] = a.qs.cent32[((size_t)qpid * Cq + i) * D + d];
  }
  constexpr int R = 32;  // outputs (i, e) per thread: Cq * D <= kAT * R
  float acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.f;
  const int nout = Cq * D;
  int cur = -1;
  auto flush = [&](int b) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int o = tid + kAT * r;
      if (o < nout) {
        const int i = o / D, e = o - i * D;
        c.ba[((((size_t)qpid * NB + b) * Cq + i) * Ck + j) * D + e] = acc[r];
      }
      acc[r] = 0.f;
    }
  };
  for (int m0 = 0; m0 < n; m0 += 32) {
    const int cnt = imin(32, n - m0);
    __syncthreads();
    for (int e = tid; e < cnt * D; e += kAT) {
      const int r = e / D, d = e - r * D;
      const long long row = pk.row0 + perm[m0 + r];
      kt[r * (D + 1) + d] = ld<T>(K + row * D + d);
      vt[r * D + d] = ld<T>(V + row * D + d);
    }
    if (tid < cnt) tb[tid] = perm[m0 + tid] / L;
    __syncthreads();
    for (int e = tid; e < cnt * Cq; e += kAT) {
      const int r = e / Cq, i = e - r * Cq;
      float x = 0.f;
#pragma unroll 8
      for (int d = 0; d < D; ++d) x = fmaf(kt[r * (D + 1) + d], nu[i * (D + 1) + d], x);
      gt[r * Cq + i] = x;
    }
    __syncthreads();
    for (int r = 0; r < cnt; ++r) {
      const int b = tb[r];
      if (b != cur) {
        if (cur >= 0) flush(cur);
        cur = b;
      }
#pragma unroll
      for (int q = 0; q < R; ++q) {
        const int o = tid + kAT * q;
        if (o < nout) {
          const int i = o / D, e = o - i * D;
          acc[q] = fmaf(vt[r * D + e], gt[r * Cq + i], acc[q]);
        }
      }
    }
  }
  if (cur >= 0) flush(cur);
}

// exclusive prefix of A over blocks: one thread per (q-set, i, j, e)
template <int D>
__global__ void acc_prefix_a_kernel(AttnArgs a, AccArgs c) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int Cq = a.Cq, Ck = a.Ck, NB = c.NB;
  const long long per = (long long)Cq * Ck * D;  // one block of one q-set
  const long long total = (long long)a.qs.nprob * per;
  if (e >= total) return;
  const long long qp = e / per, r = e - qp * per;
  float s = 0.f;
  for (int b = 0; b < NB; ++b) {
    const size_t o = (size_t)(qp * NB + b) * per + r;
    const float x = c.ba[o];
    c.pa[o] = s;
    s += x;
  }
}

// ---------------------------------------------------------------------------
// selection: per (q-set, block b), warps over the query clusters present in b
// ---------------------------------------------------------------------------
// x . y in dimension order (no fused multiply-add); y strided by `ys`
__device__ inline double dot_ordered(const double* x, const double* y, size_t ys, int D) {
  double s = 0.0;
  for (int d = 0; d < D; ++d) s = __dadd_rn(s, __dmul_rn(x[d], y[(size_t)d * ys]));
  return s;
}

__global__ void __launch_bounds__(kAT) acc_select_kernel(AttnArgs a, AccArgs c) {
  extern __shared__ __align__(16) double sel_raw[];
  const int Cq = a.Cq, Ck = a.Ck, NB = c.NB, k1 = a.topk, k2 = c.k2, D = a.qg.D;
  const int qpid = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int smax = Ck > NB ? Ck : NB;
  double* sc = sel_raw + (size_t)warp * smax;
  double* nu = sel_raw + (size_t)kAW * smax + (size_t)warp * D;
  const int kpid = kv_problem(a, qpid);
  const double s = (double)a.scale;
  for (int i = warp; i < Cq; i += kAW) {
    int* s1 = c.sel1 + (((size_t)qpid * NB + b) * Cq + i) * k1;
    int* s2 = c.sel2 + ((((size_t)qpid * NB + b) * Cq + i) * k1) * k2;
    for (int r = lane; r < k1; r += 32) s1[r] = -1;
    for (int r = lane; r < k1 * k2; r += 32) s2[r] = -1;
    const int* qb = c.qboff + ((size_t)qpid * Cq + i) * (NB + 1);
    if (b == 0 || qb[b + 1] == qb[b]) continue;  // no query of cluster i in block b
    for (int d = lane; d < D; d += 32) nu[d] = a.qs.cent64[((size_t)qpid * Cq + i) * D + d];
    __syncwarp();
    // 1. key clusters by their prefix summaries
    for (int j = lane; j < Ck; j += 32) {
      const size_t o = ((size_t)kpid * NB + b) * Ck + j;
      const int n = c.pn[o];
      const double* mu = c.pmu + ((size_t)kpid * NB + b) * D * Ck + j;  // lanes: consecutive j
      sc[j] = n > 0 ? __dadd_rn(__dmul_rn(s, dot_ordered(nu, mu, Ck, D)), log((double)n))
                    : -INFINITY;
    }
    __syncwarp();
    for (int r = 0; r < k1; ++r) {
      double bv = -INFINITY;
      int bj = -1;
      for (int j = lane; j < Ck; j += 32)
        if (sc[j] > bv) {  // the lowest j wins ties within a lane (ascending j)
          bv = sc[j];
          bj = j;
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
      if (lane == 0) {
        s1[r] = bj;
        sc[bj] = -INFINITY;
      }
      __syncwarp();
    }
    __syncwarp();
    // 2. blocks within each selected cluster, by their block summaries
    for (int r = 0; r < k1; ++r) {
      const int j = s1[r];
      if (j < 0) break;
      __syncwarp();
      for (int bb = lane; bb < b; bb += 32) {
        const size_t o = ((size_t)kpid * NB + bb) * Ck + j;
        const int n = c.bn[o];
        const double* mu = c.bmu + ((size_t)kpid * Ck + j) * D * NB + bb;  // lanes: consecutive bb
        sc[bb] = n > 0 ? __dadd_rn(__dmul_rn(s, dot_ordered(nu, mu, NB, D)), log((double)n))
                       : -INFINITY;
      }
      __syncwarp();
      for (int r2 = 0; r2 < k2; ++r2) {
        double bv = -INFINITY;
        int bj = -1;
        for (int bb = lane; bb < b; bb += 32)
          if (sc[bb] > bv) {
            bv = sc[bb];
            bj = bb;
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
        if (lane == 0) {
          s2[r * k2 + r2] = bj;
          sc[bj] = -INFINITY;
        }
        __syncwarp();
      }
      __syncwarp();
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// far summaries + retrieved keys: one CTA per (q-set, block b, kCI query
// clusters).  The prefix table of the block (centroids, log-counts and, for
// MONOPOLE, the values) is built once per CTA; per query cluster i the CTA
// adds the remainders of its selected clusters (prefix minus the retrieved
// blocks) and, for DIPOLE, its values u_ij.  One warp per query; the far
// terms one key cluster per lane.
// ---------------------------------------------------------------------------
constexpr int kCI = 16;   // query clusters per CTA
constexpr int kST = 512;  // threads of the stage-2 CTA (one CTA per SM fits its tables)
constexpr int kSW = kST / 32;
constexpr int kXL = 1024; // retrieved keys listed in shared memory per pass

template <int D>
size_t stage2_smem(int Ck, int k1) {
  return ((size_t)Ck * (D + 1) + (size_t)Ck * D + Ck + (size_t)k1 * (D + 1) + (size_t)k1 * D + k1 +
          (size_t)kSW * D + D) * 4 + (size_t)Ck * 4 + 8 + (size_t)kXL * 8 + (size_t)kSW * 32 * 4 +
         (size_t)kSW * 32 * 8;
}

template <typename T, int D, bool DIP>
__global__ void __launch_bounds__(kST) acc_stage2_kernel(AttnArgs a, AccArgs c) {
  extern __shared__ __align__(16) float s2_raw[];
  const int Cq = a.Cq, Ck = a.Ck, NB = c.NB, k1 = a.topk, k2 = c.k2;
  float* mu_s = s2_raw;                         // [Ck][D + 1] prefix centroids
  float* u_s = mu_s + (size_t)Ck * (D + 1);     // [Ck][D] values (DIPOLE: of cluster i)
  float* ln_s = u_s + (size_t)Ck * D;           // [Ck] log n, -inf if empty
  float* rm_s = ln_s + Ck;                      // [k1][D + 1] remainder centroids
  float* ru_s = rm_s + (size_t)k1 * (D + 1);    // [k1][D] remainder values
  float* rl_s = ru_s + (size_t)k1 * D;          // [k1] remainder log n
  float* q_s = rl_s + k1;                       // [kSW][D] each warp's query
  float* nu = q_s + kSW * D;                    // [D]
  int* rsel = reinterpret_cast<int*>(nu + D);   // [Ck] rank among the selected, or -1
  long long* xrow = reinterpret_cast<long long*>(  // [kXL] rows of the retrieved keys
      reinterpret_cast<uintptr_t>(rsel + Ck + 1) & ~(uintptr_t)7);
  float* pw_s = reinterpret_cast<float*>(xrow + kXL);             // [kSW][32] far weights
  const float** uw_s = reinterpret_cast<const float**>(pw_s + kSW * 32);  // [kSW][32] their rows
  __shared__ int nretr;
  const int qpid = blockIdx.x, b = blockIdx.y, i0 = blockIdx.z * kCI;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (b == 0) return;
  const Prob pq = prob_of(a.qg, qpid);
  const int kpid = kv_problem(a, qpid);
  const Prob pk = prob_of(a.kg, kpid);
  const float s = a.scale;
  constexpr int DL = D / 32;
  // ---- the block's prefix table --------------------------------------------
  for (int j = warp; j < Ck; j += kSW) {
    const size_t o = ((size_t)kpid * NB + b) * Ck + j;
    const int n = c.pn[o];
    if (lane == 0) ln_s[j] = n > 0 ? logf((float)n) : -INFINITY;
    if (n == 0) {  // no prefix member: a zero row, never weighted
#pragma unroll
      for (int u = 0; u < DL; ++u) {
        mu_s[j * (D + 1) + lane + 32 * u] = 0.f;
        u_s[j * D + lane + 32 * u] = 0.f;
      }
      continue;
    }
#pragma unroll
    for (int u = 0; u < DL; ++u) {
      const int d = lane + 32 * u;
      mu_s[j * (D + 1) + d] = (float)(c.pk[o * D + d] / (double)n);
      if (!DIP) u_s[j * D + d] = c.ps[o * D + d] / (float)n;
    }
  }
  const T* Q = static_cast<const T*>(a.qg.X);
  const T* K = static_cast<const T*>(a.kg.X);
  const T* V = static_cast<const T*>(a.V);
  const int* kperm = a.ks.perm + pk.slot0;
  const int* koff = a.ks.off + (size_t)kpid * (Ck + 1);
  for (int i = i0; i < imin(i0 + kCI, Cq); ++i) {
    const int* qb = c.qboff + ((size_t)qpid * Cq + i) * (NB + 1);
    const int m0 = qb[b], m1 = qb[b + 1];
    if (m1 == m0) continue;  // no query of cluster i in block b (CTA-uniform)
    const int* s1 = c.sel1 + (((size_t)qpid * NB + b) * Cq + i) * k1;
    const int* s2 = c.sel2 + ((((size_t)qpid * NB + b) * Cq + i) * k1) * k2;
    __syncthreads();  // the previous cluster's readers are done
    for (int d = tid; d < D; d += kST) nu[d] = a.qs.cent32[((size_t)qpid * Cq + i) * D + d];
    for (int j = tid; j < Ck; j += kST) rsel[j] = -1;
    __syncthreads();
    if (tid < k1 && s1[tid] >= 0) rsel[s1[tid]] = tid;
    if (tid == 0) {
      int cnt = 0;
      for (int r = 0; r < k1; ++r) {
        const int j = s1[r];
        if (j < 0) break;
        for (int r2 = 0; r2 < k2; ++r2) {
          const int bb = s2[r * k2 + r2];
          if (bb < 0) break;
          cnt += c.bn[((size_t)kpid * NB + bb) * Ck + j];
        }
      }
      nretr = cnt;
    }
    __syncthreads();  // rsel and nretr complete
    // the rows of the first kXL retrieved keys (the rest are read in place)
    const int nx = imin(nretr, kXL);
    if (warp == 0) {
      int base = 0;
      for (int r = 0; r < k1 && base < nx; ++r) {
        const int j = s1[r];
        if (j < 0) break;
        const int* kb = c.kboff + ((size_t)kpid * Ck + j) * (NB + 1);
        for (int r2 = 0; r2 < k2 && base < nx; ++r2) {
          const int bb = s2[r * k2 + r2];
          if (bb < 0) break;
          const int cnt = kb[bb + 1] - kb[bb];
          for (int mm = lane; mm < cnt && base + mm < nx; mm += 32)
            xrow[base + mm] = pk.row0 + kperm[koff[j] + kb[bb] + mm];
          base += cnt;
        }
      }
    }
    // remainders of the selected clusters: prefix minus the retrieved blocks
    for (int r = warp; r < k1; r += kSW) {
      const int j = s1[r];
      if (j < 0) {
        if (lane == 0) rl_s[r] = -INFINITY;
        continue;
      }
      const size_t o = ((size_t)kpid * NB + b) * Ck + j;
      int n = c.pn[o];
      double ksum[DL];
      float ss[DL], aa[DL];
#pragma unroll
      for (int u = 0; u < DL; ++u) {
        const int d = lane + 32 * u;
        ksum[u] = c.pk[o * D + d];
        ss[u] = c.ps[o * D + d];
        aa[u] = DIP ? c.pa[((((size_t)qpid * NB + b) * Cq + i) * Ck + j) * D + d] : 0.f;
      }
      for (int r2 = 0; r2 < k2; ++r2) {
        const int bb = s2[r * k2 + r2];
        if (bb < 0) break;
        const size_t ob = ((size_t)kpid * NB + bb) * Ck + j;
        n -= c.bn[ob];
#pragma unroll
        for (int u = 0; u < DL; ++u) {
          const int d = lane + 32 * u;
          ksum[u] -= c.bk[ob * D + d];
          ss[u] -= c.bs[ob * D + d];
          if (DIP) aa[u] -= c.ba[((((size_t)qpid * NB + bb) * Cq + i) * Ck + j) * D + d];
        }
      }
      if (n <= 0) {
        if (lane == 0) rl_s[r] = -INFINITY;
        continue;
      }
      const float inv = 1.f / (float)n;
      float mn = 0.f;
#pragma unroll
      for (int u = 0; u < DL; ++u) {
        const int d = lane + 32 * u;
        const float mu = (float)(ksum[u] / (double)n);
        rm_s[r * (D + 1) + d] = mu;
        mn = fmaf(mu, nu[d], mn);
      }
#pragma unroll
      for (int o2 = 16; o2; o2 >>= 1) mn += __shfl_xor_sync(0xffffffffu, mn, o2);
#pragma unroll
      for (int u = 0; u < DL; ++u) {
        const int d = lane + 32 * u;
        // M nu = A - S (mu . nu) over the remainder
        ru_s[r * D + d] = DIP ? fmaf(s, fmaf(-ss[u], mn, aa[u]), ss[u]) * inv : ss[u] * inv;
      }
      if (lane == 0) rl_s[r] = logf((float)n);
    }
    if (DIP) {  // u_ij of the unselected clusters: (S + s (A - S (mu . nu_i))) / n
      for (int j = warp; j < Ck; j += kSW) {
        const size_t o = ((size_t)kpid * NB + b) * Ck + j;
        const int n = c.pn[o];
        if (n == 0 || rsel[j] >= 0) continue;
        float mn = 0.f;
#pragma unroll
        for (int u = 0; u < DL; ++u) mn = fmaf(mu_s[j * (D + 1) + lane + 32 * u], nu[lane + 32 * u], mn);
#pragma unroll
        for (int o2 = 16; o2; o2 >>= 1) mn += __shfl_xor_sync(0xffffffffu, mn, o2);
        const float inv = 1.f / (float)n;
#pragma unroll
        for (int u = 0; u < DL; ++u) {
          const int d = lane + 32 * u;
          const float S = c.ps[o * D + d];
          const float A = c.pa[((((size_t)qpid * NB + b) * Cq + i) * Ck + j) * D + d];
          u_s[j * D + d] = fmaf(s, fmaf(-S, mn, A), S) * inv;
        }
      }
    }
    __syncthreads();
    // ---- one warp per query of cluster i in block b ----------------------
    const int* qperm = a.qs.perm + pq.slot0 + a.qs.off[(size_t)qpid * (Cq + 1) + i];
    float* qw = q_s + warp * D;
    for (int m = m0 + warp; m < m1; m += kSW) {
      const long long qrow = pq.row0 + qperm[m];
      float o[DL];
#pragma unroll
      for (int u = 0; u < DL; ++u) {
        qw[lane + 32 * u] = ld<T>(Q + qrow * D + lane + 32 * u);
        o[u] = 0.f;
      }
      __syncwarp();
      float mx = -INFINITY, l = 0.f;
      // far terms, 32 key clusters at a time (one per lane); the weights go
      // through the warp's shared-memory row so the value loop has no shuffles
      float* pw = pw_s + warp * 32;
      const float** uw = uw_s + warp * 32;
      for (int j0 = 0; j0 < Ck; j0 += 32) {
        const int j = j0 + lane;
        float lg = -INFINITY;
        const float* urow = u_s;
        if (j < Ck) {
          const int r = rsel[j];
          const float lnj = r >= 0 ? rl_s[r] : ln_s[j];
          if (lnj != -INFINITY) {
            const float* mrow = r >= 0 ? rm_s + r * (D + 1) : mu_s + j * (D + 1);
            float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;  // four chains for latency
#pragma unroll 4
            for (int d = 0; d < D; d += 4) {
              x0 = fmaf(qw[d], mrow[d], x0);
              x1 = fmaf(qw[d + 1], mrow[d + 1], x1);
              x2 = fmaf(qw[d + 2], mrow[d + 2], x2);
              x3 = fmaf(qw[d + 3], mrow[d + 3], x3);
            }
            lg = fmaf(s, (x0 + x1) + (x2 + x3), lnj);
            urow = r >= 0 ? ru_s + r * D : u_s + j * D;
          }
        }
        float bm = lg;
#pragma unroll
        for (int o2 = 16; o2; o2 >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o2));
        if (bm == -INFINITY) continue;
        const float mn = fmaxf(mx, bm);
        const float sc = __expf(mx - mn);
        const float p = __expf(lg - mn);
        pw[lane] = p;
        uw[lane] = urow;
        float ps = p;
#pragma unroll
        for (int o2 = 16; o2; o2 >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o2);
        l = l * sc + ps;
#pragma unroll
        for (int u = 0; u < DL; ++u) o[u] *= sc;
        mx = mn;
        __syncwarp();
#pragma unroll 8
        for (int jj = 0; jj < 32; ++jj) {
          const float pj = pw[jj];
          if (pj == 0.f) continue;  // an empty or absent cluster: its row is not read
          const float* ur = uw[jj];
#pragma unroll
          for (int u = 0; u < DL; ++u) o[u] = fmaf(pj, ur[lane + 32 * u], o[u]);
        }
        __syncwarp();
      }
      // exact terms: the keys of the retrieved (cluster, block) pairs, 32 at
      // a time (one per lane for the logits, then the warp over the values)
      for (int x0 = 0; x0 < nx; x0 += 32) {
        const int t = x0 + lane;
        float lg = -INFINITY;
        long long krow = 0;
        if (t < nx) {
          krow = xrow[t];
          const uint4* kp = reinterpret_cast<const uint4*>(K + krow * D);
          float x = 0.f;
          if (sizeof(T) == 2) {
#pragma unroll
            for (int c8 = 0; c8 < D / 8; ++c8) {
              const uint4 w = __ldg(kp + c8);
              const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h[e]);
                x = fmaf(qw[c8 * 8 + 2 * e], f.x, x);
                x = fmaf(qw[c8 * 8 + 2 * e + 1], f.y, x);
              }
            }
          } else {
#pragma unroll 16
            for (int d = 0; d < D; ++d) x = fmaf(qw[d], ld<T>(K + krow * D + d), x);
          }
          lg = s * x;
        }
        float bm = lg;
#pragma unroll
        for (int o2 = 16; o2; o2 >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o2));
        const float mn = fmaxf(mx, bm);
        const float sc = __expf(mx - mn);
        const float p = __expf(lg - mn);
        float ps = p;
#pragma unroll
        for (int o2 = 16; o2; o2 >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o2);
        l = l * sc + ps;
#pragma unroll
        for (int u = 0; u < DL; ++u) o[u] *= sc;
        mx = mn;
        const int nt = imin(32, nx - x0);
        for (int jj = 0; jj < nt; ++jj) {
          const float pj = __shfl_sync(0xffffffffu, p, jj);
          const long long vr = xrow[x0 + jj];
#pragma unroll
          for (int u = 0; u < DL; ++u) o[u] = fmaf(pj, ld<T>(V + vr * D + lane + 32 * u), o[u]);
        }
      }
      if (nretr > kXL) {  // retrieved keys past the list, one at a time
        int idx = 0;
        for (int r = 0; r < k1; ++r) {
          const int j = s1[r];
          if (j < 0) break;
          const int* kb = c.kboff + ((size_t)kpid * Ck + j) * (NB + 1);
          for (int r2 = 0; r2 < k2; ++r2) {
            const int bb = s2[r * k2 + r2];
            if (bb < 0) break;
            for (int mm = kb[bb]; mm < kb[bb + 1]; ++mm, ++idx) {
              if (idx < kXL) continue;
              const long long krow = pk.row0 + kperm[koff[j] + mm];
              float x = 0.f;
#pragma unroll
              for (int u = 0; u < DL; ++u)
                x = fmaf(qw[lane + 32 * u], ld<T>(K + krow * D + lane + 32 * u), x);
#pragma unroll
              for (int o2 = 16; o2; o2 >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o2);
              const float lg = s * x;
              const float mn = fmaxf(mx, lg);
              const float sc = __expf(mx - mn), w = __expf(lg - mn);
              l = l * sc + w;
#pragma unroll
              for (int u = 0; u < DL; ++u)
                o[u] = fmaf(o[u], sc, w * ld<T>(V + krow * D + lane + 32 * u));
              mx = mn;
            }
          }
        }
      }
      float* pp = a.part + (size_t)qrow * (D + 1);
      const float inv = 1.f / l;
#pragma unroll
      for (int u = 0; u < DL; ++u) pp[lane + 32 * u] = o[u] * inv;
      if (lane == 0) {
        pp[D] = mx + logf(l);
        if (a.n_exact != nullptr) a.n_exact[qrow] = nretr;
      }
      __syncwarp();
    }
  }
}

// ---------------------------------------------------------------------------
// The same terms with every query of the CTA's clusters in flight at once.
// The unselected clusters' centroids and log-counts are shared by all query
// clusters; so are their MONOPOLE values S / n.  A DIPOLE value adds
// s (A_ij / n_j - (S_j / n_j)(mu_j . nu_i)), formed per query from the prefix
// table A and the per-cluster dots mu_j . nu_i.  Only the selected clusters'
// remainders are per query cluster (kCM * k1 rows).
// ---------------------------------------------------------------------------
constexpr int kCM = 16;    // query clusters per CTA
constexpr int kRM = 64;    // remainder rows per CTA: kCM clusters x k1, or fewer clusters for k1 > 4

template <int D>
size_t stage2_mono_smem(int Ck, bool dip) {
  return ((size_t)Ck * (D + 1) + (size_t)Ck * D + Ck + (size_t)kRM * (D + 1) + (size_t)kRM * D + kRM +
          (size_t)kSW * D) * 4 + (size_t)2 * kCM * Ck + (size_t)kSW * 32 * 4 + (size_t)kSW * 32 * 8 * 3 +
         64 + (dip ? ((size_t)kCM * Ck + Ck + (size_t)kSW * 32 * 2 + (size_t)kCM * D) * 4 : 0);
}

template <typename T, int D, bool DIP>
__global__ void __launch_bounds__(kST) acc_stage2_mono_kernel(AttnArgs a, AccArgs c, int nci) {
  extern __shared__ __align__(16) float sm_raw[];
  const int Cq = a.Cq, Ck = a.Ck, NB = c.NB, k1 = a.topk, k2 = c.k2;
  float* mu_s = sm_raw;                         // [Ck][D + 1] prefix centroids
  float* u_s = mu_s + (size_t)Ck * (D + 1);     // [Ck][D] prefix values S / n
  float* ln_s = u_s + (size_t)Ck * D;           // [Ck]
  float* rm_s = ln_s + Ck;                      // [kRM][D + 1] remainder centroids
  float* ru_s = rm_s + (size_t)kRM * (D + 1);   // [kRM][D] remainder values
  float* rl_s = ru_s + (size_t)kRM * D;         // [kRM]
  float* q_s = rl_s + kRM;                      // [kSW][D]
  float* pw_s = q_s + kSW * D;                  // [kSW][32]
  const float** uw_s = reinterpret_cast<const float**>(  // [kSW][32]
      (reinterpret_cast<uintptr_t>(pw_s + kSW * 32) + 7) & ~(uintptr_t)7);
  long long* xb_s = reinterpret_cast<long long*>(uw_s + kSW * 32);   // [kSW][32] retrieved rows
  const float** aw_s = reinterpret_cast<const float**>(xb_s + kSW * 32);  // [kSW][32] DIPOLE A rows
  // DIPOLE only (the MONOPOLE allocation ends before them): mu_j . nu_i per
  // (query cluster, key cluster), 1 / n_j, each warp's copies of both, nu_i
  float* dip0 = reinterpret_cast<float*>(aw_s + kSW * 32);
  float* mn_s = dip0;                                                  // [kCM][Ck]
  float* inv_s = mn_s + (size_t)kCM * Ck;                              // [Ck]
  float* cw_s = inv_s + Ck;                                            // [kSW][32]
  float* iw_s = cw_s + kSW * 32;                                       // [kSW][32]
  float* nu_s = iw_s + kSW * 32;                                       // [kCM][D]
  signed char* rsel = reinterpret_cast<signed char*>(DIP ? nu_s + (size_t)kCM * D : dip0);  // [nci][Ck]
  __shared__ int qcum[kCM + 1];
  __shared__ int nretr[kCM];
  const int qpid = blockIdx.x, b = blockIdx.y, i0 = blockIdx.z * nci;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (b == 0) return;
  const int ncl = imin(nci, Cq - i0);
  const Prob pq = prob_of(a.qg, qpid);
  const int kpid = kv_problem(a, qpid);
  const Prob pk = prob_of(a.kg, kpid);
  const float s = a.scale;
  constexpr int DL = D / 32;
  // ---- the block's prefix table --------------------------------------------
  for (int j = warp; j < Ck; j += kSW) {
    const size_t o = ((size_t)kpid * NB + b) * Ck + j;
    const int n = c.pn[o];
    if (lane == 0) {
      ln_s[j] = n > 0 ? logf((float)n) : -INFINITY;
      if (DIP) inv_s[j] = n > 0 ? 1.f / (float)n : 0.f;
    }
#pragma unroll
    for (int u = 0; u < DL; ++u) {
      const int d = lane + 32 * u;
      mu_s[j * (D + 1) + d] = n > 0 ? (float)(c.pk[o * D + d] / (double)n) : 0.f;
      u_s[j * D + d] = n > 0 ? c.ps[o * D + d] / (float)n : 0.f;
    }
  }
  if (DIP)
    for (int e = tid; e < ncl * D; e += kST) {
      const int cc = e / D, d = e - cc * D;
      nu_s[cc * D + d] = a.qs.cent32[((size_t)qpid * Cq + i0 + cc) * D + d];
    }
  // ---- per cluster: its query range, its selected clusters, their remainders
  for (int e = tid; e < ncl * Ck; e += kST) rsel[e] = -1;
  if (tid == 0) {
    int acc = 0;
    for (int cc = 0; cc < ncl; ++cc) {
      const int* qb = c.qboff + ((size_t)qpid * Cq + i0 + cc) * (NB + 1);
      qcum[cc] = acc;
      acc += qb[b + 1] - qb[b];
    }
    qcum[ncl] = acc;
  }
  __syncthreads();
  for (int e = tid; e < ncl * k1; e += kST) {
    const int cc = e / k1, r = e - cc * k1;
    const int j = c.sel1[(((size_t)qpid * NB + b) * Cq + i0 + cc) * k1 + r];
    if (j >= 0) rsel[cc * Ck + j] = (signed char)r;
  }
  if (tid < ncl) {
    const int* s1 = c.sel1 + (((size_t)qpid * NB + b) * Cq + i0 + tid) * k1;
    const int* s2 = c.sel2 + ((((size_t)qpid * NB + b) * Cq + i0 + tid) * k1) * k2;
    int cnt = 0;
    for (int r = 0; r < k1; ++r) {
      const int j = s1[r];
      if (j < 0) break;
      for (int r2 = 0; r2 < k2; ++r2) {
        const int bb = s2[r * k2 + r2];
        if (bb < 0) break;
        cnt += c.bn[((size_t)kpid * NB + bb) * Ck + j];
      }
    }
    nretr[tid] = cnt;
  }
  if (DIP)  // mu_j . nu_i of every (query cluster, key cluster) of the CTA
    for (int e = warp; e < ncl * Ck; e += kSW) {
      const int cc = e / Ck, j = e - cc * Ck;
      float x = 0.f;
#pragma unroll
      for (int u = 0; u < DL; ++u) x = fmaf(mu_s[j * (D + 1) + lane + 32 * u], nu_s[cc * D + lane + 32 * u], x);
#pragma unroll
      for (int o2 = 16; o2; o2 >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o2);
      if (lane == 0) mn_s[cc * Ck + j] = x;
    }
  for (int e = warp; e < ncl * k1; e += kSW) {
    const int cc = e / k1, r = e - cc * k1, row = cc * k1 + r;
    const int* s1 = c.sel1 + (((size_t)qpid * NB + b) * Cq + i0 + cc) * k1;
    const int* s2 = c.sel2 + ((((size_t)qpid * NB + b) * Cq + i0 + cc) * k1) * k2;
    const int j = s1[r];
    if (j < 0) {
      if (lane == 0) rl_s[row] = -INFINITY;
      continue;
    }
    const size_t o = ((size_t)kpid * NB + b) * Ck + j;
    const size_t oa = (((size_t)qpid * NB + b) * Cq + i0 + cc) * Ck + j;  // the A table row
    int n = c.pn[o];
    double ksum[DL];
    float ss[DL], aa[DL];
#pragma unroll
    for (int u = 0; u < DL; ++u) {
      ksum[u] = c.pk[o * D + lane + 32 * u];
      ss[u] = c.ps[o * D + lane + 32 * u];
      aa[u] = DIP ? c.pa[oa * D + lane + 32 * u] : 0.f;
    }
    for (int r2 = 0; r2 < k2; ++r2) {
      const int bb = s2[r * k2 + r2];
      if (bb < 0) break;
      const size_t ob = ((size_t)kpid * NB + bb) * Ck + j;
      n -= c.bn[ob];
#pragma unroll
      for (int u = 0; u < DL; ++u) {
        ksum[u] -= c.bk[ob * D + lane + 32 * u];
        ss[u] -= c.bs[ob * D + lane + 32 * u];
        if (DIP)
          aa[u] -= c.ba[((((size_t)qpid * NB + bb) * Cq + i0 + cc) * Ck + j) * D + lane + 32 * u];
      }
    }
    float mn = 0.f;
#pragma unroll
    for (int u = 0; u < DL; ++u) {
      const int d = lane + 32 * u;
      const float mu = n > 0 ? (float)(ksum[u] / (double)n) : 0.f;
      rm_s[row * (D + 1) + d] = mu;
      if (DIP) mn = fmaf(mu, a.qs.cent32[((size_t)qpid * Cq + i0 + cc) * D + d], mn);
    }
    if (DIP) {
#pragma unroll
      for (int o2 = 16; o2; o2 >>= 1) mn += __shfl_xor_sync(0xffffffffu, mn, o2);
    }
#pragma unroll
    for (int u = 0; u < DL; ++u) {
      const int d = lane + 32 * u;
      // M nu = A - S (mu . nu) over the remainder
      ru_s[row * D + d] = n <= 0 ? 0.f
                          : DIP ? fmaf(a.scale, fmaf(-ss[u], mn, aa[u]), ss[u]) / (float)n
                                : ss[u] / (float)n;
    }
    if (lane == 0) rl_s[row] = n > 0 ? logf((float)n) : -INFINITY;
  }
  __syncthreads();
  // ---- one warp per query, across all of the CTA's clusters ----------------
  const T* Q = static_cast<const T*>(a.qg.X);
  const T* K = static_cast<const T*>(a.kg.X);
  const T* V = static_cast<const T*>(a.V);
  const int* kperm = a.ks.perm + pk.slot0;
  const int* koff = a.ks.off + (size_t)kpid * (Ck + 1);
  float* qw = q_s + warp * D;
  float* pw = pw_s + warp * 32;
  const float** uw = uw_s + warp * 32;
  const float** aw = aw_s + warp * 32;
  float* cw = cw_s + warp * 32;
  float* iw = iw_s + warp * 32;
  for (int m = warp; m < qcum[ncl]; m += kSW) {
    int cc = 0;
    while (qcum[cc + 1] <= m) ++cc;
    const int i = i0 + cc;
    const int* qb = c.qboff + ((size_t)qpid * Cq + i) * (NB + 1);
    const int* qperm = a.qs.perm + pq.slot0 + a.qs.off[(size_t)qpid * (Cq + 1) + i];
    const long long qrow = pq.row0 + qperm[qb[b] + (m - qcum[cc])];
    const signed char* rs = rsel + cc * Ck;
    const int* s1 = c.sel1 + (((size_t)qpid * NB + b) * Cq + i) * k1;
    const int* s2 = c.sel2 + ((((size_t)qpid * NB + b) * Cq + i) * k1) * k2;
    float o[DL];
#pragma unroll
    for (int u = 0; u < DL; ++u) {
      qw[lane + 32 * u] = ld<T>(Q + qrow * D + lane + 32 * u);
      o[u] = 0.f;
    }
    __syncwarp();
    float mx = -INFINITY, l = 0.f;
    const float* arow0 = DIP ? c.pa + (((size_t)qpid * NB + b) * Cq + i) * Ck * D : nullptr;
    for (int j0 = 0; j0 < Ck; j0 += 32) {
      const int j = j0 + lane;
      float lg = -INFINITY;
      const float* urow = u_s;
      const float* arow = nullptr;  // DIPOLE: the unselected cluster's A row (the value's dipole part)
      if (j < Ck) {
        const int r = rs[j];
        const int row = cc * k1 + r;
        const float lnj = r >= 0 ? rl_s[row] : ln_s[j];
        if (lnj != -INFINITY) {
          const float* mrow = r >= 0 ? rm_s + row * (D + 1) : mu_s + j * (D + 1);
          float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;
#pragma unroll 4
          for (int d = 0; d < D; d += 4) {
            x0 = fmaf(qw[d], mrow[d], x0);
            x1 = fmaf(qw[d + 1], mrow[d + 1], x1);
            x2 = fmaf(qw[d + 2], mrow[d + 2], x2);
            x3 = fmaf(qw[d + 3], mrow[d + 3], x3);
          }
          lg = fmaf(s, (x0 + x1) + (x2 + x3), lnj);
          urow = r >= 0 ? ru_s + row * D : u_s + j * D;
          if (DIP && r < 0) arow = arow0 + (size_t)j * D;
        }
      }
      if (DIP) {
        aw[lane] = arow;
        cw[lane] = j < Ck ? mn_s[cc * Ck + j] : 0.f;
        iw[lane] = j < Ck ? inv_s[j] : 0.f;
      }
      float bm = lg;
#pragma unroll
      for (int o2 = 16; o2; o2 >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o2));
      if (bm == -INFINITY) continue;
      const float mn = fmaxf(mx, bm);
      const float sc = __expf(mx - mn);
      const float p = __expf(lg - mn);
      pw[lane] = p;
      uw[lane] = urow;
      float ps = p;
#pragma unroll
      for (int o2 = 16; o2; o2 >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o2);
      l = l * sc + ps;
#pragma unroll
      for (int u = 0; u < DL; ++u) o[u] *= sc;
      mx = mn;
      __syncwarp();
#pragma unroll 8
      for (int jj = 0; jj < 32; ++jj) {
        const float pj = pw[jj];
        if (pj == 0.f) continue;
        const float* ur = uw[jj];
        const float* ar = DIP ? aw[jj] : nullptr;
        if (DIP && ar != nullptr) {  // u = S/n + s (A/n - (S/n)(mu . nu))
          const float cj = cw[jj], ij = iw[jj];
#pragma unroll
          for (int u = 0; u < DL; ++u) {
            const float u0 = ur[lane + 32 * u];
            o[u] = fmaf(pj, fmaf(s, fmaf(ar[lane + 32 * u], ij, -u0 * cj), u0), o[u]);
          }
        } else {
#pragma unroll
          for (int u = 0; u < DL; ++u) o[u] = fmaf(pj, ur[lane + 32 * u], o[u]);
        }
      }
      __syncwarp();
    }
    // retrieved keys: their rows gathered 32 at a time into the warp's buffer,
    // then one key per lane for the logits and the warp over the values
    long long* xb = xb_s + warp * 32;
    int nb = 0;
    auto flush = [&]() {
      float lg = -INFINITY;
      if (lane < nb) {
        const long long krow = xb[lane];
        float x = 0.f;
        if (sizeof(T) == 2) {
          const uint4* kp = reinterpret_cast<const uint4*>(K + krow * D);
#pragma unroll
          for (int c8 = 0; c8 < D / 8; ++c8) {
            const uint4 w = __ldg(kp + c8);
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(h[e]);
              x = fmaf(qw[c8 * 8 + 2 * e], f.x, x);
              x = fmaf(qw[c8 * 8 + 2 * e + 1], f.y, x);
            }
          }
        } else {
#pragma unroll 16
          for (int d = 0; d < D; ++d) x = fmaf(qw[d], ld<T>(K + krow * D + d), x);
        }
        lg = s * x;
      }
      float bm = lg;
#pragma unroll
      for (int o2 = 16; o2; o2 >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o2));
      const float mn = fmaxf(mx, bm);
      const float sc = __expf(mx - mn);
      const float p = __expf(lg - mn);
      float ps = p;
#pragma unroll
      for (int o2 = 16; o2; o2 >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o2);
      l = l * sc + ps;
#pragma unroll
      for (int u = 0; u < DL; ++u) o[u] *= sc;
      mx = mn;
      for (int jj = 0; jj < nb; ++jj) {
        const float pj = __shfl_sync(0xffffffffu, p, jj);
        const long long vr = xb[jj];
#pragma unroll
        for (int u = 0; u < DL; ++u) o[u] = fmaf(pj, ld<T>(V + vr * D + lane + 32 * u), o[u]);
      }
      __syncwarp();
      nb = 0;
    };
    for (int r = 0; r < k1; ++r) {
      const int j = s1[r];
      if (j < 0) break;
      const int* kb = c.kboff + ((size_t)kpid * Ck + j) * (NB + 1);
      for (int r2 = 0; r2 < k2; ++r2) {
        const int bb = s2[r * k2 + r2];
        if (bb < 0) break;
        const int m0 = kb[bb], cnt = kb[bb + 1] - m0;
        for (int x0 = 0; x0 < cnt;) {
          const int take = imin(32 - nb, cnt - x0);
          if (lane < take) xb[nb + lane] = pk.row0 + kperm[koff[j] + m0 + x0 + lane];
          __syncwarp();
          nb += take;
          x0 += take;
          if (nb == 32) flush();
        }
      }
    }
    if (nb > 0) flush();
    float* pp = a.part + (size_t)qrow * (D + 1);
    const float inv = 1.f / l;
#pragma unroll
    for (int u = 0; u < DL; ++u) pp[lane + 32 * u] = o[u] * inv;
    if (lane == 0) {
      pp[D] = mx + logf(l);
      if (a.n_exact != nullptr) a.n_exact[qrow] = nretr[cc];
    }
    __syncwarp();
  }
}

template <typename T, int D>
void launch_accum(const AttnArgs& a, const AccArgs& c, cudaStream_t st) {
  const int nk = a.ks.nprob, nq = a.qs.nprob;
  const bool dip = a.mode == 1;
  {
    ProfScope ps(st, "accum_block_stats");
    acc_block_stats_kernel<T, D, true><<<dim3(nk, a.Ck), kAT, 0, st>>>(a, c);
    acc_block_stats_kernel<T, D, false><<<dim3(nq, a.Cq), kAT, 0, st>>>(a, c);
    const long long tot = (long long)nk * a.Ck * D;
    acc_prefix_kernel<D><<<(unsigned)((tot + 255) / 256), 256, 0, st>>>(a, c);
  }
  if (dip) {
    ProfScope ps(st, "accum_block_a");
    const size_t sm = ((size_t)a.Cq * (D + 1) + 32 * (D + 1) + 32 * D + 32 * a.Cq) * 4 + 32 * 4;
    cudaFuncSetAttribute(acc_block_a_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    acc_block_a_kernel<T, D><<<dim3(nq, a.Ck), kAT, sm, st>>>(a, c);
    const long long tot = (long long)nq * a.Cq * a.Ck * D;
    acc_prefix_a_kernel<D><<<(unsigned)((tot + 255) / 256), 256, 0, st>>>(a, c);
  }
  if (a.topk > 0 && c.k2 > 0) {
    ProfScope ps(st, "accum_select");
    const int smax = a.Ck > c.NB ? a.Ck : c.NB;
    const size_t sm = ((size_t)kAW * smax + (size_t)kAW * D) * 8;
    cudaFuncSetAttribute(acc_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    acc_select_kernel<<<dim3(nq, c.NB), kAT, sm, st>>>(a, c);
  }
  {
    ProfScope ps(st, "accum_stage2");
    const size_t smf = stage2_mono_smem<D>(a.Ck, dip);
    if (!dip || smf <= 227 * 1024) {  // DIPOLE: where its per-query tables fit, else per cluster
      // query clusters per CTA: the remainder rows of all of them must fit
      const int nci = a.topk > 0 ? imin(kCM, kRM / a.topk) : kCM;
      const size_t sm = smf;
      auto kern = dip ? acc_stage2_mono_kernel<T, D, true> : acc_stage2_mono_kernel<T, D, false>;
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      kern<<<dim3(nq, c.NB, cdiv(a.Cq, nci)), kST, sm, st>>>(a, c, nci);
    } else {
      const size_t sm = stage2_smem<D>(a.Ck, a.topk);
      cudaFuncSetAttribute(acc_stage2_kernel<T, D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)sm);
      acc_stage2_kernel<T, D, true><<<dim3(nq, c.NB, cdiv(a.Cq, kCI)), kST, sm, st>>>(a, c);
    }
  }
}

}  // namespace

bool accum_supported(int D, int Cq, int Ck, int NB, int k1, int k2, int mode) {
  if (mode != 0 && mode != 1) return false;
  if (D != 64 && D != 128) return false;
  if (Cq > 256 || Ck > 256 || Ck * D > 16384 || k1 > 32) return false;
  if ((D == 64 ? stage2_smem<64>(Ck, k1) : stage2_smem<128>(Ck, k1)) > 227 * 1024) return false;
  if (mode == 0 && (D == 64 ? stage2_mono_smem<64>(Ck, false) : stage2_mono_smem<128>(Ck, false)) >
                       227 * 1024)
    return false;
  if (mode == 1 && Cq * D > kAT * 32) return false;  // acc_block_a: 32 outputs per thread
  if (NB < 1 || NB > 1024 || k2 < 0 || k2 > NB) return false;
  return true;
}

void run_accum(const AttnArgs& a, const AccArgs& c, cudaStream_t st) {
  using bf = __nv_bfloat16;
  if (a.qg.dtype == 0) {
    if (a.qg.D == 64) launch_accum<bf, 64>(a, c, st);
    else launch_accum<bf, 128>(a, c, st);
  } else {
    if (a.qg.D == 64) launch_accum<float, 64>(a, c, st);
    else launch_accum<float, 128>(a, c, st);
  }
}

}  // namespace muse
