// Shared device-side definitions of libmuse: problem geometry, element
// loads, and the workspace-resident per-problem state.
//
// A "problem" is one clustering of one token block: acausal -> the whole
// sequence of one (b, head); causal -> the key block or the query block of
// one (level, pair) of the hierarchical decomposition of one (b, head).  Both
// cases are one level table: acausal has a single level with one pair whose
// block is the whole sequence.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace muse {

constexpr int kMaxLevels = 24;
constexpr int kTile = 128;  // tokens per assignment tile
constexpr int kMaxC = 1024;

// Bits of the device error word (the public MUSE_DEVERR_* values).
constexpr int kErrMmaWait = 1;      // a tensor-core completion wait gave up
constexpr int kErrTeamBarrier = 2;  // a k-means team barrier gave up
constexpr int kErrVRange = 4;       // a finite bf16 value of V overflowed fp16

struct Levels {
  int nlev;                 // number of levels (acausal: 1)
  int causal;
  int N;                    // sequence length
  int s[kMaxLevels];        // block size of each level
  int npairs[kMaxLevels];   // pairs at each level
  int pair_base[kMaxLevels];   // first pair index of the level (per bh)
  int tile_base[kMaxLevels];   // first tile index of the level (per bh)
  int tiles_per_pair[kMaxLevels];
  int tok_base[kMaxLevels];    // first token slot of the level (per bh)
  int pairs_per_bh;
  int tiles_per_bh;
  int toks_per_bh;
  int pmax;                 // pairs at level 0 (stream-id stride)
};

// Geometry of one role (keys or queries) over one tensor.
struct RoleGeo {
  Levels lv;
  int BH;      // B * heads of this tensor
  int D;
  int C;       // requested clusters (effective: min(C, s))
  int role;    // 0 keys, 1 queries
  int dtype;   // 0 bf16, 1 f32
  const void* X;
  uint64_t seed;
  uint64_t sid0;  // stream id of row set (b, h) = (0, 0): row set bh draws stream sid0 + bh
};

struct Prob {
  int bh, level, pair, s, C;
  long long row0;   // first row of the block in X (rows of D elements)
  long long slot0;  // first token slot of the problem (assign / perm arrays)
  long long tile0;  // first global tile of the problem
  uint64_t sid;
};

__host__ __device__ inline int imin(int a, int b) { return a < b ? a : b; }
__host__ __device__ inline int cdiv(int a, int b) { return (a + b - 1) / b; }

__device__ inline Prob prob_of(const RoleGeo& g, int pid) {
  Prob p;
  const Levels& L = g.lv;
  p.bh = pid / L.pairs_per_bh;
  int pi = pid - p.bh * L.pairs_per_bh;
  int l = 0;
  while (l + 1 < L.nlev && pi >= L.pair_base[l + 1]) ++l;
  p.level = l;
  p.pair = pi - L.pair_base[l];
  p.s = L.s[l];
  p.C = imin(g.C, p.s);
  long long seq0 = (long long)p.bh * L.N;
  p.row0 = seq0 + (L.causal ? (long long)(2 * p.pair + g.role) * p.s : 0);
  p.slot0 = (long long)p.bh * L.toks_per_bh + L.tok_base[l] + (long long)p.pair * p.s;
  p.tile0 = (long long)p.bh * L.tiles_per_bh + L.tile_base[l] +
            (long long)p.pair * L.tiles_per_pair[l];
  p.sid = L.causal ? ((g.sid0 + (uint64_t)p.bh) * L.nlev + l) * (uint64_t)L.pmax + p.pair
                   : g.sid0 + (uint64_t)p.bh;
  return p;
}

// Global tile -> (problem id, tile within problem).
__device__ inline void tile_of(const RoleGeo& g, long long t, int* pid, int* tin) {
  const Levels& L = g.lv;
  int bh = (int)(t / L.tiles_per_bh);
  int r = (int)(t - (long long)bh * L.tiles_per_bh);
  int l = 0;
  while (l + 1 < L.nlev && r >= L.tile_base[l + 1]) ++l;
  r -= L.tile_base[l];
  int pair = r / L.tiles_per_pair[l];
  *tin = r - pair * L.tiles_per_pair[l];
  *pid = bh * L.pairs_per_bh + L.pair_base[l] + pair;
}

template <typename T>
__device__ inline float ld(const T* p);
template <>
__device__ inline float ld<float>(const float* p) { return *p; }
template <>
__device__ inline float ld<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

template <typename T>
__device__ inline void st(T* p, float v);
template <>
__device__ inline void st<float>(float* p, float v) { *p = v; }
template <>
__device__ inline void st<__nv_bfloat16>(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// Per-role k-means state in the workspace.
struct KState {
  double* cent64;   // [nprob][C][D] current centroids (fp64 master copy)
  float* cent32;    // [nprob][C][D] fp32 rounding of cent64
  float* cnorm;     // [nprob][C]    ||cent32|| (slightly enlarged)
  int* counts;      // [nprob][C]
  int* off;         // [nprob][C+1]  segment offsets of the sorted order
  int* assign;      // [tokens]      cluster of each token (problem-local index)
  int* perm;        // [tokens]      problem-local token index in cluster-sorted order
  int* hist;        // [tiles][C+1]  per-tile histogram, then scatter bases; the
                    //               persistent k-means: per-CTA list offsets
  unsigned short* tlist;  // [tokens]  persistent k-means: each CTA's tokens grouped
                          //           by cluster (CTA-local token index)
  int* arrive;      // [nprob]       tile arrival counters (self-resetting)
  __nv_bfloat16* cbf_hi;  // [nprob][C][D] bf16 rounding of cent32
  __nv_bfloat16* cbf_lo;  // [nprob][C][D] bf16 rounding of cent32 - cbf_hi
  float* cn2;       // [nprob][C]    ||c||^2 (fp64 sum rounded to fp32)
  int* emin;        // [nprob]       smallest biased exponent of a nonzero value (bf16)
  int* emax;        // [nprob]       largest biased exponent of a value (bf16)
  double* part;     // [part_blocks][C][D] per-CTA partial centroid sums (resident k-means)
  int* pcnt;        // [part_blocks][C]    per-CTA member counts (resident k-means)
  double* sum64;    // [nprob][C][D] resident k-means: exact running sums of the members
  int* dirty;       // [nprob][C]    resident k-means: last round that changed the members
  int* chg;         // [nprob][2]    resident k-means: tokens that changed cluster (round & 1)
  size_t part_blocks;
  int* err;         // device error word (0 = ok)
  int nprob;
  long long ntiles;
  long long ntok;
};

// The centroid sums of a problem are exact in fp64 in any order -- and so
// equal to a plain sequential fp64 sum bit for bit -- when every partial sum
// is a representable multiple of the smallest value's ulp: with bf16 values
// of biased exponents in [emin, emax] (ulp 2^(emin - 134) for emin >= 1, the
// subnormals counted as emin = 1) and at most s members,
// |partial| < s 2^(emax - 126) <= 2^53 ulp  <=  (emax - emin) + ceil(log2 s) <= 45.
__device__ inline bool sums_exact(const KState& ks, int pid, int s) {
  const int lo = ks.emin[pid], hi = ks.emax[pid];
  if (hi < lo) return true;  // no nonzero value
  int lg = 0;
  while ((1 << lg) < s) ++lg;
  return (hi - lo) + lg <= 45;
}

}  // namespace muse
