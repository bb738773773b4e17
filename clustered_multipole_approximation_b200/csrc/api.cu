// C ABI of libmuse: argument checks, workspace plan, and the launch sequence
// of each entry point.  Everything runs on the caller's stream; nothing here
// allocates, frees or synchronises.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdio.h>

#include <string>

#include "../../include/muse.h"
#include "common.cuh"
#include "kernels.h"

using namespace muse;

namespace {

thread_local std::string g_last_error;

muse_status fail(muse_status s, const char* msg) {
  g_last_error = msg;
  return s;
}

muse_status check_launch() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    g_last_error = std::string("CUDA launch failed: ") + cudaGetErrorString(e);
    return MUSE_ERR_CUDA;
  }
  return MUSE_OK;
}

// A pointer argument that violates its alignment (NULL passes: the caller
// checks required pointers separately).
bool misaligned(const void* p, size_t a) { return p && (reinterpret_cast<uintptr_t>(p) % a) != 0; }

int ilog2_exact(int x) {  // -1 unless x is a power of two
  if (x <= 0 || (x & (x - 1))) return -1;
  int l = 0;
  while ((1 << l) < x) ++l;
  return l;
}

Levels make_levels(int N, int L, bool causal) {
  Levels lv{};
  lv.N = N;
  lv.causal = causal ? 1 : 0;
  if (!causal) {
    lv.nlev = 1;
    lv.s[0] = N;
    lv.npairs[0] = 1;
    lv.tiles_per_pair[0] = cdiv(N, kTile);
    lv.pairs_per_bh = 1;
    lv.tiles_per_bh = lv.tiles_per_pair[0];
    lv.toks_per_bh = N;
    lv.pmax = 1;
    return lv;
  }
  const int nblk = N / L;
  lv.nlev = ilog2_exact(nblk);
  lv.pmax = nblk / 2 > 0 ? nblk / 2 : 1;
  int pb = 0, tb = 0;
  for (int l = 0; l < lv.nlev; ++l) {
    lv.s[l] = L << l;
    lv.npairs[l] = nblk >> (l + 1);
    lv.tiles_per_pair[l] = cdiv(lv.s[l], kTile);
    lv.pair_base[l] = pb;
    lv.tile_base[l] = tb;
    lv.tok_base[l] = l * (N / 2);
    pb += lv.npairs[l];
    tb += lv.npairs[l] * lv.tiles_per_pair[l];
  }
  lv.pairs_per_bh = pb;
  lv.tiles_per_bh = tb;
  lv.toks_per_bh = lv.nlev * (N / 2);
  return lv;
}

// Bump allocator over the caller's workspace (256-byte aligned pieces).
struct Carver {
  char* base;
  size_t used = 0;
  template <typename P>
  P* take(size_t bytes) {
    size_t at = (used + 255) & ~(size_t)255;
    used = at + bytes;
    return base ? reinterpret_cast<P*>(base + at) : nullptr;
  }
};

void carve_kstate(Carver& cv, KState& ks, const RoleGeo& g) {
  const long long BH = g.BH;
  ks.nprob = (int)(BH * g.lv.pairs_per_bh);
  ks.ntiles = BH * g.lv.tiles_per_bh;
  ks.ntok = BH * g.lv.toks_per_bh;
  const size_t np = ks.nprob, C = g.C, D = g.D;
  ks.cent64 = cv.take<double>(np * C * D * 8);
  ks.cent32 = cv.take<float>(np * C * D * 4);
  ks.cnorm = cv.take<float>(np * C * 4);
  ks.counts = cv.take<int>(np * C * 4);
  ks.off = cv.take<int>(np * (C + 1) * 4);
  ks.assign = cv.take<int>((size_t)ks.ntok * 4);
  ks.perm = cv.take<int>((size_t)ks.ntok * 4);
  ks.hist = cv.take<int>((size_t)ks.ntiles * (C + 1) * 4);
  ks.tlist = cv.take<unsigned short>((size_t)ks.ntok * 2);
  ks.arrive = cv.take<int>(np * 4);
  ks.cbf_hi = cv.take<__nv_bfloat16>(np * C * D * 2);
  ks.cbf_lo = cv.take<__nv_bfloat16>(np * C * D * 2);
  ks.cn2 = cv.take<float>(np * C * 4);
  ks.emin = cv.take<int>(np * 4);
  ks.emax = cv.take<int>(np * 4);
  ks.part_blocks = g.dtype == 0 ? resident_partial_blocks(g.lv, g.BH, g.D, g.C) : 0;
  ks.part = cv.take<double>(ks.part_blocks * C * D * 8);
  ks.pcnt = cv.take<int>(ks.part_blocks * C * 4);
  // running-sum tables of the persistent k-means kernels (bf16, C <= 256)
  const bool res = g.dtype == 0 && g.C <= 256;
  ks.sum64 = res ? cv.take<double>(np * C * D * 8) : nullptr;
  ks.dirty = res ? cv.take<int>(np * C * 4) : nullptr;
  ks.chg = res ? cv.take<int>(np * 2 * 4) : nullptr;
}

RoleGeo make_geo(const void* X, int BH, int D, int C, int role, int dtype, uint64_t seed,
                 const Levels& lv) {
  RoleGeo g{};
  g.lv = lv;
  g.BH = BH;
  g.D = D;
  g.C = C;
  g.role = role;
  g.dtype = dtype;
  g.X = X;
  g.seed = seed;
  return g;
}

constexpr size_t kStage1Budget = (size_t)2 << 30;  // bytes of stage-1 tables per wave

struct AttnPlan {
  size_t bytes;
  int wave;  // query problems per stage-1 wave
};

struct AttnLayout {
  int* err;
  __half* V16;
  RoleGeo qg, kg;
  KState qs, ks;
  Stage1 s1;
  float* part;
  void* kpad;  // sorted key copies of the tensor-core stage 2 (bf16 K, fp16 V)
  void* vpad;
  int* gofs;
  int nq;
  int wave;
  size_t bytes;
};

muse_status validate(const muse_shape* sh, const muse_params* pr, bool causal) {
  if (!sh || !pr) return fail(MUSE_ERR_INVALID_ARG, "shape and params must not be NULL");
  if (sh->B < 1 || sh->Hq < 1 || sh->Hkv < 1 || sh->N < 1)
    return fail(MUSE_ERR_INVALID_ARG, "B, Hq, Hkv and N must be >= 1");
  if (sh->Hq % sh->Hkv) return fail(MUSE_ERR_INVALID_ARG, "Hq must be a multiple of Hkv");
  if (sh->D != 64 && sh->D != 128) return fail(MUSE_ERR_UNSUPPORTED, "D must be 64 or 128");
  if (sh->dtype != MUSE_BF16 && sh->dtype != MUSE_F32)
    return fail(MUSE_ERR_INVALID_ARG, "dtype must be MUSE_BF16 or MUSE_F32");
  if (sh->out_f32 != 0 && sh->out_f32 != 1) return fail(MUSE_ERR_INVALID_ARG, "out_f32 must be 0 or 1");
  if (pr->iters < 1) return fail(MUSE_ERR_INVALID_ARG, "iters must be >= 1");
  if (pr->mode < MUSE_MONOPOLE || pr->mode > MUSE_TILTED_DIPOLE)
    return fail(MUSE_ERR_INVALID_ARG, "unknown mode");
  if (pr->Cq < 1 || pr->Ck < 1) return fail(MUSE_ERR_INVALID_ARG, "Cq and Ck must be >= 1");
  if (pr->Cq > kMaxC || pr->Ck > kMaxC)
    return fail(MUSE_ERR_UNSUPPORTED, "Cq and Ck must be <= 1024");
  if (pr->topk < 0 || pr->topk > pr->Ck)
    return fail(MUSE_ERR_INVALID_ARG, "topk must be in [0, Ck]");
  if (!(pr->scale == pr->scale)) return fail(MUSE_ERR_INVALID_ARG, "scale is NaN");
  const long long elems = (long long)sh->B * (sh->Hq > sh->Hkv ? sh->Hq : sh->Hkv) * sh->N;
  if (elems > (1LL << 31) - 1) return fail(MUSE_ERR_UNSUPPORTED, "B*H*N must be < 2^31");
  if (!causal) {
    if (pr->Cq > sh->N || pr->Ck > sh->N)
      return fail(MUSE_ERR_INVALID_ARG, "Cq and Ck must be <= N");
  } else {
    if (pr->Cq != pr->Ck) return fail(MUSE_ERR_INVALID_ARG, "causal needs Cq == Ck");
    if (pr->block < 1 || sh->N % pr->block)
      return fail(MUSE_ERR_INVALID_ARG, "block must divide N");
    if (ilog2_exact(sh->N / pr->block) < 0)
      return fail(MUSE_ERR_INVALID_ARG, "N / block must be a power of two");
    if (ilog2_exact(sh->N / pr->block) >= kMaxLevels)
      return fail(MUSE_ERR_UNSUPPORTED, "too many levels");
  }
  return MUSE_OK;
}

AttnLayout layout(const muse_shape* sh, const muse_params* pr, bool causal, const void* Q,
                  const void* K, void* ws) {
  AttnLayout L{};
  const Levels lv = make_levels(sh->N, causal ? pr->block : sh->N, causal);
  const int dt = sh->dtype == MUSE_BF16 ? 0 : 1;
  L.kg = make_geo(K, sh->B * sh->Hkv, sh->D, pr->Ck, 0, dt, pr->seed, lv);
  L.qg = make_geo(Q, sh->B * sh->Hq, sh->D, pr->Cq, 1, dt, pr->seed, lv);
  L.kg.sid0 = pr->key_stream0;
  L.qg.sid0 = pr->query_stream0;
  Carver cv{static_cast<char*>(ws)};
  L.err = cv.take<int>(4);
  carve_kstate(cv, L.ks, L.kg);
  carve_kstate(cv, L.qs, L.qg);
  L.ks.err = L.qs.err = L.err;
  L.nq = L.qs.nprob;
  const size_t cc = (size_t)pr->Cq * pr->Ck;
  const bool tilt = pr->mode == MUSE_TILTED || pr->mode == MUSE_TILTED_DIPOLE;
  const size_t per = cc * 4 * 2 + cc * sh->D * 4 * (tilt ? 2 : 1);  // upper bound
  size_t wave = L.nq;
  if (causal && per * wave > kStage1Budget) wave = kStage1Budget / per;
  if (wave < 1) wave = 1;
  L.wave = (int)wave;
  L.s1.logW = cv.take<float>(wave * cc * 4);
  L.s1.fbias = cv.take<float>(wave * cc * 4);
  const bool tilted = tilt;  // the tilted centroids are carved for both tilted modes
  if (dt == 0) {
    L.s1.Uh = cv.take<__half>(wave * cc * sh->D * 2);
    L.s1.Ul = cv.take<__half>(wave * cc * sh->D * 2);
    L.s1.Kfh = tilted ? cv.take<__nv_bfloat16>(wave * cc * sh->D * 2) : nullptr;
    L.s1.Kfl = tilted ? cv.take<__nv_bfloat16>(wave * cc * sh->D * 2) : nullptr;
    L.V16 = cv.take<__half>((size_t)sh->B * sh->Hkv * sh->N * sh->D * 2);
  } else {
    L.s1.U = cv.take<float>(wave * cc * sh->D * 4);
    L.s1.Kf = tilted ? cv.take<float>(wave * cc * sh->D * 4) : nullptr;
  }
  const int k1 = pr->topk > 0 ? pr->topk : 1;
  L.s1.sel = cv.take<int>((size_t)L.nq * pr->Cq * k1 * 4);
  L.s1.nsel = cv.take<int>((size_t)L.nq * pr->Cq * 4);
  L.part = causal ? cv.take<float>((size_t)L.qs.ntok * (sh->D + 1) * 4) : nullptr;
  if (dt == 0 && pr->Ck <= 256) {
    // every key problem's tokens plus up to one padding group of 8 rows per cluster
    const size_t rows = (size_t)L.ks.ntok + (size_t)8 * pr->Ck * L.ks.nprob;
    L.kpad = cv.take<__nv_bfloat16>(rows * sh->D * 2);
    L.vpad = cv.take<__half>(rows * sh->D * 2);
    L.gofs = cv.take<int>((size_t)L.ks.nprob * (pr->Ck + 1) * 4);
  } else {
    L.kpad = L.vpad = nullptr;
    L.gofs = nullptr;
  }
  L.bytes = cv.used + 256;
  return L;
}

muse_status attn(const void* Q, const void* K, const void* V, void* O, const muse_shape* sh,
                 const muse_params* pr, muse_debug* dbg, void* ws, size_t ws_bytes,
                 cudaStream_t st, bool causal) {
  muse_status s = validate(sh, pr, causal);
  if (s != MUSE_OK) return s;
  if (!Q || !K || !V || !O) return fail(MUSE_ERR_INVALID_ARG, "Q, K, V and O must not be NULL");
  if (misaligned(Q, 16) || misaligned(K, 16) || misaligned(V, 16) || misaligned(O, 16))
    return fail(MUSE_ERR_INVALID_ARG, "Q, K, V and O must be 16-byte aligned");
  if (misaligned(ws, 256)) return fail(MUSE_ERR_INVALID_ARG, "the workspace must be 256-byte aligned");
  if (dbg && (misaligned(dbg->q_assign, 4) || misaligned(dbg->k_assign, 4) ||
              misaligned(dbg->selected, 4) || misaligned(dbg->k_counts, 4) ||
              misaligned(dbg->q_centroids, 4) || misaligned(dbg->k_centroids, 4) ||
              misaligned(dbg->n_exact, 8) || misaligned(dbg->device_error, 4)))
    return fail(MUSE_ERR_INVALID_ARG, "debug outputs must be aligned to their element size");
  const AttnLayout need = layout(sh, pr, causal, Q, K, nullptr);
  if (!ws || ws_bytes < need.bytes) return fail(MUSE_ERR_WORKSPACE, "workspace too small");
  AttnLayout L = layout(sh, pr, causal, Q, K, ws);
  AttnArgs a{};
  a.qg = L.qg;
  a.kg = L.kg;
  a.qs = L.qs;
  a.ks = L.ks;
  a.V = V;
  a.V16 = L.V16;
  a.O = causal ? nullptr : O;
  a.out_f32 = sh->out_f32 ? 1 : 0;
  a.part = L.part;
  a.n_exact = dbg ? reinterpret_cast<long long*>(dbg->n_exact) : nullptr;
  a.B = sh->B;
  a.G = sh->Hq / sh->Hkv;
  a.mode = (int)pr->mode;
  if (pr->mode == MUSE_TILTED_DIPOLE) {  // stage 1 and selection are TILTED's
    a.mode = MUSE_TILTED;
    a.tdip = 1;
  }
  a.topk = pr->topk;
  a.scale = pr->scale;
  a.Cq = pr->Cq;
  a.Ck = pr->Ck;
  // bf16 DIPOLE causal levels with few tokens per cluster: per key token;
  // the fine-query dipole: per key token at every level
  if (pr->mode == MUSE_DIPOLE_Q) {
    const int m = L.V16 ? fine_query_dense_levels(L.qg.lv, sh->D, pr->Cq, pr->Ck) : -1;
    if (m < 0)
      return fail(MUSE_ERR_UNSUPPORTED,
                  "DIPOLE_Q needs bf16, Cq and Ck <= 256 and block sizes that are multiples of 128");
    a.dense_lv = m;
  } else {
    a.dense_lv = (causal && sh->dtype == MUSE_BF16 && pr->mode == MUSE_DIPOLE && L.V16)
                     ? dense_levels(L.qg.lv, sh->D, pr->Cq, pr->Ck)
                     : 0;
  }
  a.tc_lv = (sh->dtype == MUSE_BF16 && L.V16 && L.kpad && !a.tdip)
                ? stage2_tc_levels(L.qg.lv, sh->D, pr->Cq, pr->Ck, pr->topk, a.dense_lv)
                : 0;
  a.kpad = L.kpad;
  a.vpad = L.vpad;
  a.gofs = L.gofs;
  const size_t elt = sh->dtype == MUSE_BF16 ? 2 : 4;
  if (a.n_exact && causal)
    cudaMemsetAsync(a.n_exact, 0, (size_t)sh->B * sh->Hq * sh->N * 8, st);
  cudaMemsetAsync(L.err, 0, 4, st);
  // rows of small causal levels (C_eff < Cq) are never selected into: -1
  if (dbg && dbg->selected && causal && pr->topk > 0)
    cudaMemsetAsync(L.s1.sel, 0xFF, (size_t)L.nq * pr->Cq * pr->topk * 4, st);
  if (L.nq > 0 && L.V16)
    run_bf16_to_half(V, L.V16, (size_t)sh->B * sh->Hkv * sh->N * sh->D, L.err, st);
  if (L.nq > 0) {
    cudaMemsetAsync(L.ks.arrive, 0, (size_t)L.ks.nprob * 4, st);
    cudaMemsetAsync(L.qs.arrive, 0, (size_t)L.qs.nprob * 4, st);
    const RoleGeo gs[2] = {L.kg, L.qg};
    const KState kss[2] = {L.ks, L.qs};
    run_kmeans_init(gs, kss, 2, nullptr, st);
#ifdef MUSE_PHASE_CLOCKS
    {
      const cudaError_t e = cudaStreamSynchronize(st);
      fprintf(stderr, "after v_to_half + kmeans_init: %s\n", cudaGetErrorString(e));
    }
#endif
    const bool fused = launch_kmeans_fused(gs, kss, 2, pr->iters, st);
    if (!fused) {
      run_kmeans_rounds(L.kg, L.ks, pr->iters, st);
      run_kmeans_rounds(L.qg, L.qs, pr->iters, st);
    }
    run_permute_keys(a, st);
    for (int q0 = 0; q0 < L.nq; q0 += L.wave) {
      const int n = L.nq - q0 < L.wave ? L.nq - q0 : L.wave;
      run_blocks(a, L.s1, q0, n, st);
    }
  }
  if (causal) {
    a.O = O;
    run_local_merge(a, pr->block, st);
  }
  if (dbg) {
    const size_t D = sh->D;
    if (dbg->device_error) cudaMemcpyAsync(dbg->device_error, L.err, 4, cudaMemcpyDeviceToDevice, st);
    if (dbg->q_assign) cudaMemcpyAsync(dbg->q_assign, L.qs.assign, (size_t)L.qs.ntok * 4, cudaMemcpyDeviceToDevice, st);
    if (dbg->k_assign) cudaMemcpyAsync(dbg->k_assign, L.ks.assign, (size_t)L.ks.ntok * 4, cudaMemcpyDeviceToDevice, st);
    // acausal [B,Hq,Cq,topk]; causal [B,Hq,P,Cq,topk] (the same table: one
    // row block per query problem, problems numbered (b, q-head, pair))
    if (dbg->selected && pr->topk > 0)
      cudaMemcpyAsync(dbg->selected, L.s1.sel, (size_t)L.nq * pr->Cq * pr->topk * 4, cudaMemcpyDeviceToDevice, st);
    if (!causal) {
      if (dbg->k_counts) cudaMemcpyAsync(dbg->k_counts, L.ks.counts, (size_t)L.ks.nprob * pr->Ck * 4, cudaMemcpyDeviceToDevice, st);
      if (dbg->q_centroids) cudaMemcpyAsync(dbg->q_centroids, L.qs.cent32, (size_t)L.qs.nprob * pr->Cq * D * 4, cudaMemcpyDeviceToDevice, st);
      if (dbg->k_centroids) cudaMemcpyAsync(dbg->k_centroids, L.ks.cent32, (size_t)L.ks.nprob * pr->Ck * D * 4, cudaMemcpyDeviceToDevice, st);
    }
  }
  (void)elt;
  return check_launch();
}

// The backward pass's scratch, carved after the forward's part of the
// workspace (base == nullptr: sizes only).
struct BwdLayout {
  BwdArgs b;
  size_t bytes;
};

BwdLayout bwd_layout(const muse_shape* sh, const muse_params* pr, const AttnLayout& L, void* ws,
                     bool causal = false) {
  BwdLayout r{};
  Carver cv{static_cast<char*>(ws)};
  cv.used = L.bytes;
  const size_t nk = L.ks.nprob, nq = L.qs.nprob, D = sh->D, Cq = pr->Cq, Ck = pr->Ck;
  const bool dip = pr->mode == MUSE_DIPOLE;
  r.b.Sst = cv.take<float>(nk * Ck * D * 4);
  r.b.Mst = dip ? cv.take<float>(nk * Ck * D * D * 4) : nullptr;
  r.b.U = dip ? cv.take<float>(nq * Cq * Ck * D * 4) : nullptr;
  r.b.dU = cv.take<float>(nq * Cq * Ck * D * 4);
  r.b.dmu = cv.take<float>(nk * Ck * D * 4);
  r.b.dnu = cv.take<float>(nq * Cq * D * 4);
  if (causal) {
    const size_t toks = L.qs.ntok, rows = (size_t)sh->B * sh->Hq * sh->N;
    r.b.pm = cv.take<float>(toks * 4);
    r.b.pl = cv.take<float>(toks * 4);
    r.b.pa = cv.take<float>(toks * 4);
    r.b.lm = cv.take<float>(rows * 4);
    r.b.ll = cv.take<float>(rows * 4);
    r.b.la = cv.take<float>(rows * 4);
    r.b.lse_all = cv.take<float>(rows * 4);
    r.b.d_all = cv.take<float>(rows * 4);
  }
  r.bytes = cv.used + 256;
  return r;
}

// Workspace of the block-accumulation causal operator: the acausal
// clusterings' state, the fp16 copy of V, one partial per query, the block
// tables and the selections.
struct AccLayout {
  int* err;
  __half* V16;
  RoleGeo qg, kg;
  KState qs, ks;
  float* part;
  AccArgs c;
  size_t bytes;
};

AccLayout accum_layout(const muse_shape* sh, const muse_params* pr, int k2, const void* Q,
                       const void* K, void* ws) {
  AccLayout L{};
  const Levels lv = make_levels(sh->N, sh->N, false);
  const int dt = sh->dtype == MUSE_BF16 ? 0 : 1;
  L.kg = make_geo(K, sh->B * sh->Hkv, sh->D, pr->Ck, 0, dt, pr->seed, lv);
  L.qg = make_geo(Q, sh->B * sh->Hq, sh->D, pr->Cq, 1, dt, pr->seed, lv);
  L.kg.sid0 = pr->key_stream0;
  L.qg.sid0 = pr->query_stream0;
  Carver cv{static_cast<char*>(ws)};
  L.err = cv.take<int>(4);
  carve_kstate(cv, L.ks, L.kg);
  carve_kstate(cv, L.qs, L.qg);
  L.ks.err = L.qs.err = L.err;
  const size_t BHq = (size_t)sh->B * sh->Hq, BHk = (size_t)sh->B * sh->Hkv, N = sh->N, D = sh->D;
  L.V16 = dt == 0 ? cv.take<__half>(BHk * N * D * 2) : nullptr;
  L.part = cv.take<float>(BHq * N * (D + 1) * 4);
  AccArgs& c = L.c;
  c.L = pr->block;
  c.NB = pr->block > 0 ? (int)(N / pr->block) : 1;
  c.k2 = k2;
  const size_t nk = L.ks.nprob, nq = L.qs.nprob, NB = c.NB, Cq = pr->Cq, Ck = pr->Ck;
  const size_t k1 = pr->topk > 0 ? pr->topk : 1, kk2 = k2 > 0 ? k2 : 1;
  c.kboff = cv.take<int>(nk * Ck * (NB + 1) * 4);
  c.qboff = cv.take<int>(nq * Cq * (NB + 1) * 4);
  c.bn = cv.take<int>(nk * NB * Ck * 4);
  c.pn = cv.take<int>(nk * NB * Ck * 4);
  c.bk = cv.take<double>(nk * NB * Ck * D * 8);
  c.pk = cv.take<double>(nk * NB * Ck * D * 8);
  c.bmu = cv.take<double>(nk * NB * Ck * D * 8);
  c.pmu = cv.take<double>(nk * NB * Ck * D * 8);
  c.bs = cv.take<float>(nk * NB * Ck * D * 4);
  c.ps = cv.take<float>(nk * NB * Ck * D * 4);
  const bool dip = pr->mode == MUSE_DIPOLE;
  c.ba = dip ? cv.take<float>(nq * NB * Cq * Ck * D * 4) : nullptr;
  c.pa = dip ? cv.take<float>(nq * NB * Cq * Ck * D * 4) : nullptr;
  c.sel1 = cv.take<int>(nq * NB * Cq * k1 * 4);
  c.sel2 = cv.take<int>(nq * NB * Cq * k1 * kk2 * 4);
  L.bytes = cv.used + 256;
  return L;
}

muse_status validate_accum(const muse_shape* sh, const muse_params* pr, int k2) {
  muse_status s = validate(sh, pr, false);
  if (s != MUSE_OK) return s;
  if (pr->block < 1 || sh->N % pr->block) return fail(MUSE_ERR_INVALID_ARG, "block must divide N");
  if (k2 < 0 || k2 > sh->N / pr->block)
    return fail(MUSE_ERR_INVALID_ARG, "topk2 must be in [0, N / block]");
  if (!accum_supported(sh->D, pr->Cq, pr->Ck, sh->N / pr->block, pr->topk, k2, (int)pr->mode))
    return fail(MUSE_ERR_UNSUPPORTED,
                "block accumulation needs MONOPOLE or DIPOLE, Cq, Ck <= 256, Ck * D <= 16384, "
                "topk <= 32, N / block <= 1024 (DIPOLE: Cq * D <= 8192)");
  return MUSE_OK;
}

muse_status attn_bwd(const void* Q, const void* K, const void* V, const void* dO, float* dQ,
                     float* dK, float* dV, const muse_shape* sh, const muse_params* pr, void* ws,
                     size_t ws_bytes, cudaStream_t st, bool causal);

muse_status validate_bwd(const muse_shape* sh, const muse_params* pr, bool causal = false) {
  muse_status s = validate(sh, pr, causal);
  if (s != MUSE_OK) return s;
  if (causal && pr->block % 32)
    return fail(MUSE_ERR_UNSUPPORTED, "the causal backward pass needs block % 32 == 0");
  if (!backward_supported(sh->D, pr->Ck, (int)pr->mode))
    return fail(MUSE_ERR_UNSUPPORTED, "the backward pass needs mode MONOPOLE or DIPOLE and Ck * D <= 16384");
  return MUSE_OK;
}

}  // namespace

namespace muse {
void set_last_error(const char* msg) { g_last_error = msg; }
}  // namespace muse

extern "C" {

size_t muse_workspace_size(const muse_shape* shape, const muse_params* params, int causal) {
  if (validate(shape, params, causal != 0) != MUSE_OK) return 0;
  return layout(shape, params, causal != 0, nullptr, nullptr, nullptr).bytes;
}

size_t muse_attn_bwd_workspace_size(const muse_shape* shape, const muse_params* params) {
  if (validate_bwd(shape, params) != MUSE_OK) return 0;
  const AttnLayout L = layout(shape, params, false, nullptr, nullptr, nullptr);
  return bwd_layout(shape, params, L, nullptr).bytes;
}

size_t muse_attn_bwd_causal_workspace_size(const muse_shape* shape, const muse_params* params) {
  if (validate_bwd(shape, params, true) != MUSE_OK) return 0;
  const AttnLayout L = layout(shape, params, true, nullptr, nullptr, nullptr);
  return bwd_layout(shape, params, L, nullptr, true).bytes;
}

muse_status muse_attn_bwd(const void* Q, const void* K, const void* V, const void* dO, float* dQ,
                          float* dK, float* dV, const muse_shape* sh, const muse_params* pr,
                          void* ws, size_t ws_bytes, cudaStream_t st) {
  return attn_bwd(Q, K, V, dO, dQ, dK, dV, sh, pr, ws, ws_bytes, st, false);
}

muse_status muse_attn_bwd_causal(const void* Q, const void* K, const void* V, const void* dO,
                                 float* dQ, float* dK, float* dV, const muse_shape* sh,
                                 const muse_params* pr, void* ws, size_t ws_bytes,
                                 cudaStream_t st) {
  return attn_bwd(Q, K, V, dO, dQ, dK, dV, sh, pr, ws, ws_bytes, st, true);
}

}  // extern "C"

namespace {

muse_status attn_bwd(const void* Q, const void* K, const void* V, const void* dO, float* dQ,
                     float* dK, float* dV, const muse_shape* sh, const muse_params* pr, void* ws,
                     size_t ws_bytes, cudaStream_t st, bool causal) {
  muse_status s = validate_bwd(sh, pr, causal);
  if (s != MUSE_OK) return s;
  if (!Q || !K || !V || !dO || !dQ || !dK || !dV)
    return fail(MUSE_ERR_INVALID_ARG, "Q, K, V, dO, dQ, dK and dV must not be NULL");
  if (misaligned(Q, 16) || misaligned(K, 16) || misaligned(V, 16) || misaligned(dO, 16) ||
      misaligned(dQ, 16) || misaligned(dK, 16) || misaligned(dV, 16))
    return fail(MUSE_ERR_INVALID_ARG, "all tensors must be 16-byte aligned");
  if (misaligned(ws, 256)) return fail(MUSE_ERR_INVALID_ARG, "the workspace must be 256-byte aligned");
  const AttnLayout need = layout(sh, pr, causal, Q, K, nullptr);
  if (!ws || ws_bytes < bwd_layout(sh, pr, need, nullptr, causal).bytes)
    return fail(MUSE_ERR_WORKSPACE, "workspace too small for the backward pass");
  AttnLayout L = layout(sh, pr, causal, Q, K, ws);
  AttnArgs a{};
  a.qg = L.qg;
  a.kg = L.kg;
  a.qs = L.qs;
  a.ks = L.ks;
  a.V = V;
  a.B = sh->B;
  a.G = sh->Hq / sh->Hkv;
  a.mode = (int)pr->mode;
  a.topk = pr->topk;
  a.scale = pr->scale;
  a.Cq = pr->Cq;
  a.Ck = pr->Ck;
  BwdLayout bl = bwd_layout(sh, pr, L, ws, causal);
  BwdArgs& b = bl.b;
  b.dO = dO;
  b.o_f32 = (sh->out_f32 || sh->dtype == MUSE_F32) ? 1 : 0;
  b.dQ = dQ;
  b.dK = dK;
  b.dV = dV;
  const size_t kv = (size_t)sh->B * sh->Hkv * sh->N * sh->D * 4;
  cudaMemsetAsync(dK, 0, kv, st);
  cudaMemsetAsync(dV, 0, kv, st);
  const size_t nq = L.qs.nprob, nk = L.ks.nprob;
  cudaMemsetAsync(b.dU, 0, nq * pr->Cq * pr->Ck * sh->D * 4, st);
  cudaMemsetAsync(b.dmu, 0, nk * pr->Ck * sh->D * 4, st);
  cudaMemsetAsync(b.dnu, 0, nq * pr->Cq * sh->D * 4, st);
  if (causal) {
    cudaMemsetAsync(dQ, 0, (size_t)sh->B * sh->Hq * sh->N * sh->D * 4, st);  // sums over levels
    run_attn_bwd_causal(a, L.s1, b, pr->block, st);
  } else {
    run_attn_bwd(a, L.s1, b, st);
  }
  return check_launch();
}

}  // namespace

extern "C" {

size_t muse_accum_workspace_size(const muse_shape* shape, const muse_params* params, int topk2) {
  if (validate_accum(shape, params, topk2) != MUSE_OK) return 0;
  return accum_layout(shape, params, topk2, nullptr, nullptr, nullptr).bytes;
}

muse_status muse_attn_fwd_causal_accum(const void* Q, const void* K, const void* V, void* O,
                                       const muse_shape* sh, const muse_params* pr, int topk2,
                                       muse_accum_debug* dbg, void* ws, size_t ws_bytes,
                                       cudaStream_t st) {
  muse_status s = validate_accum(sh, pr, topk2);
  if (s != MUSE_OK) return s;
  if (!Q || !K || !V || !O) return fail(MUSE_ERR_INVALID_ARG, "Q, K, V and O must not be NULL");
  if (misaligned(Q, 16) || misaligned(K, 16) || misaligned(V, 16) || misaligned(O, 16))
    return fail(MUSE_ERR_INVALID_ARG, "Q, K, V and O must be 16-byte aligned");
  if (misaligned(ws, 256)) return fail(MUSE_ERR_INVALID_ARG, "the workspace must be 256-byte aligned");
  if (dbg && (misaligned(dbg->q_assign, 4) || misaligned(dbg->k_assign, 4) ||
              misaligned(dbg->sel1, 4) || misaligned(dbg->sel2, 4) ||
              misaligned(dbg->n_exact, 8) || misaligned(dbg->device_error, 4)))
    return fail(MUSE_ERR_INVALID_ARG, "debug outputs must be aligned to their element size");
  if (!ws || ws_bytes < accum_layout(sh, pr, topk2, Q, K, nullptr).bytes)
    return fail(MUSE_ERR_WORKSPACE, "workspace too small");
  AccLayout L = accum_layout(sh, pr, topk2, Q, K, ws);
  AttnArgs a{};
  a.qg = L.qg;
  a.kg = L.kg;
  a.qs = L.qs;
  a.ks = L.ks;
  a.V = V;
  a.V16 = L.V16;
  a.out_f32 = sh->out_f32 ? 1 : 0;
  a.part = L.part;
  a.n_exact = dbg ? reinterpret_cast<long long*>(dbg->n_exact) : nullptr;
  a.B = sh->B;
  a.G = sh->Hq / sh->Hkv;
  a.mode = (int)pr->mode;
  a.topk = topk2 > 0 ? pr->topk : 0;  // no block retrieved: no cluster retrieval either
  a.scale = pr->scale;
  a.Cq = pr->Cq;
  a.Ck = pr->Ck;
  a.accum = 1;
  const AccArgs& c = L.c;
  const size_t N = sh->N, D = sh->D, nk = L.ks.nprob, nq = L.qs.nprob, NB = c.NB;
  cudaMemsetAsync(L.err, 0, 4, st);
  if (a.n_exact) cudaMemsetAsync(a.n_exact, 0, (size_t)sh->B * sh->Hq * N * 8, st);
  cudaMemsetAsync(c.bn, 0, nk * NB * pr->Ck * 4, st);
  cudaMemsetAsync(c.bk, 0, nk * NB * pr->Ck * D * 8, st);
  cudaMemsetAsync(c.bs, 0, nk * NB * pr->Ck * D * 4, st);
  if (c.ba) cudaMemsetAsync(c.ba, 0, nq * NB * pr->Cq * pr->Ck * D * 4, st);
  if (L.V16) run_bf16_to_half(V, L.V16, (size_t)sh->B * sh->Hkv * N * D, L.err, st);
  cudaMemsetAsync(L.ks.arrive, 0, nk * 4, st);
  cudaMemsetAsync(L.qs.arrive, 0, nq * 4, st);
  const RoleGeo gs[2] = {L.kg, L.qg};
  const KState kss[2] = {L.ks, L.qs};
  run_kmeans_init(gs, kss, 2, nullptr, st);
  if (!launch_kmeans_fused(gs, kss, 2, pr->iters, st)) {
    run_kmeans_rounds(L.kg, L.ks, pr->iters, st);
    run_kmeans_rounds(L.qg, L.qs, pr->iters, st);
  }
  run_accum(a, c, st);
  a.O = O;
  run_local_merge(a, pr->block, st);
  if (dbg) {
    if (dbg->device_error) cudaMemcpyAsync(dbg->device_error, L.err, 4, cudaMemcpyDeviceToDevice, st);
    if (dbg->q_assign) cudaMemcpyAsync(dbg->q_assign, L.qs.assign, (size_t)L.qs.ntok * 4, cudaMemcpyDeviceToDevice, st);
    if (dbg->k_assign) cudaMemcpyAsync(dbg->k_assign, L.ks.assign, (size_t)L.ks.ntok * 4, cudaMemcpyDeviceToDevice, st);
    if (a.topk > 0) {
      const size_t rows = nq * NB * pr->Cq * pr->topk;
      if (dbg->sel1) cudaMemcpyAsync(dbg->sel1, c.sel1, rows * 4, cudaMemcpyDeviceToDevice, st);
      if (dbg->sel2) cudaMemcpyAsync(dbg->sel2, c.sel2, rows * topk2 * 4, cudaMemcpyDeviceToDevice, st);
    }
  }
  return check_launch();
}

size_t muse_cluster_workspace_size(int B, int H, int N, int D, int C) {
  if (B < 1 || H < 1 || N < 1 || C < 1 || (D != 64 && D != 128)) return 0;
  const Levels lv = make_levels(N, N, false);
  RoleGeo g = make_geo(nullptr, B * H, D, C, 0, 0, 0, lv);
  Carver cv{nullptr};
  KState ks{};
  cv.take<int>(4);
  carve_kstate(cv, ks, g);
  return cv.used + 256;
}

muse_status muse_cluster(const void* X, muse_dtype dtype, int B, int H, int N, int D, int C,
                         int iters, uint64_t seed, int role, const float* init, int32_t* assign,
                         float* centroids, int32_t* counts, int32_t* device_error, void* ws,
                         size_t ws_bytes, cudaStream_t stream) {
  if (!X || !assign || !centroids) return fail(MUSE_ERR_INVALID_ARG, "X, assign and centroids must not be NULL");
  if (misaligned(X, 16) || misaligned(init, 16) || misaligned(assign, 4) ||
      misaligned(centroids, 4) || misaligned(counts, 4) || misaligned(device_error, 4))
    return fail(MUSE_ERR_INVALID_ARG, "X and init must be 16-byte aligned, the outputs 4-byte");
  if (misaligned(ws, 256)) return fail(MUSE_ERR_INVALID_ARG, "the workspace must be 256-byte aligned");
  if (B < 1 || H < 1 || N < 1) return fail(MUSE_ERR_INVALID_ARG, "B, H and N must be >= 1");
  if (D != 64 && D != 128) return fail(MUSE_ERR_UNSUPPORTED, "D must be 64 or 128");
  if (dtype != MUSE_BF16 && dtype != MUSE_F32) return fail(MUSE_ERR_INVALID_ARG, "bad dtype");
  if (C < 1 || C > N) return fail(MUSE_ERR_INVALID_ARG, "C must be in [1, N]");
  if (C > kMaxC) return fail(MUSE_ERR_UNSUPPORTED, "C must be <= 1024");
  if (iters < 1) return fail(MUSE_ERR_INVALID_ARG, "iters must be >= 1");
  if (role != 0 && role != 1) return fail(MUSE_ERR_INVALID_ARG, "role must be 0 or 1");
  if ((long long)B * H * N > (1LL << 31) - 1) return fail(MUSE_ERR_UNSUPPORTED, "B*H*N must be < 2^31");
  const size_t need = muse_cluster_workspace_size(B, H, N, D, C);
  if (!ws || ws_bytes < need) return fail(MUSE_ERR_WORKSPACE, "workspace too small");
  const Levels lv = make_levels(N, N, false);
  RoleGeo g = make_geo(X, B * H, D, C, role, dtype == MUSE_BF16 ? 0 : 1, seed, lv);
  Carver cv{static_cast<char*>(ws)};
  KState ks{};
  int* err = cv.take<int>(4);
  carve_kstate(cv, ks, g);
  ks.err = err;
  cudaMemsetAsync(err, 0, 4, stream);
  cudaMemsetAsync(ks.arrive, 0, (size_t)ks.nprob * 4, stream);
  run_kmeans_init(&g, &ks, 1, init, stream);
  const bool fused = launch_kmeans_fused(&g, &ks, 1, iters, stream);
  if (!fused) run_kmeans_rounds(g, ks, iters, stream);
  cudaMemcpyAsync(assign, ks.assign, (size_t)ks.ntok * 4, cudaMemcpyDeviceToDevice, stream);
  cudaMemcpyAsync(centroids, ks.cent32, (size_t)ks.nprob * C * D * 4, cudaMemcpyDeviceToDevice, stream);
  if (counts) cudaMemcpyAsync(counts, ks.counts, (size_t)ks.nprob * C * 4, cudaMemcpyDeviceToDevice, stream);
  if (device_error) cudaMemcpyAsync(device_error, err, 4, cudaMemcpyDeviceToDevice, stream);
  return check_launch();
}

muse_status muse_summarize(const void* K, const void* V, muse_dtype dtype, int B, int H, int N,
                           int D, int C, const int32_t* assign, int32_t* counts, float* mu,
                           float* S, float* M, void* ws, size_t ws_bytes, cudaStream_t stream) {
  (void)ws;
  (void)ws_bytes;
  if (!K || !V || !assign || !counts || !mu || !S)
    return fail(MUSE_ERR_INVALID_ARG, "K, V, assign, counts, mu and S must not be NULL");
  if (B < 1 || H < 1 || N < 1) return fail(MUSE_ERR_INVALID_ARG, "B, H and N must be >= 1");
  if (D != 64 && D != 128) return fail(MUSE_ERR_UNSUPPORTED, "D must be 64 or 128");
  if (dtype != MUSE_BF16 && dtype != MUSE_F32) return fail(MUSE_ERR_INVALID_ARG, "bad dtype");
  if (C < 1) return fail(MUSE_ERR_INVALID_ARG, "C must be >= 1");
  if (C > 65535) return fail(MUSE_ERR_UNSUPPORTED, "C must be < 65536");
  if (misaligned(K, 16) || misaligned(V, 16) || misaligned(assign, 4) || misaligned(counts, 4) ||
      misaligned(mu, 16) || misaligned(S, 16) || misaligned(M, 16))
    return fail(MUSE_ERR_INVALID_ARG, "K, V, mu, S and M must be 16-byte aligned, assign and counts 4-byte");
  run_summarize(K, V, dtype == MUSE_BF16 ? 0 : 1, B * H, N, D, C, assign, counts, mu, S, M,
                nullptr, nullptr, stream);
  return check_launch();
}

muse_status muse_attn_fwd(const void* Q, const void* K, const void* V, void* O,
                          const muse_shape* shape, const muse_params* params, muse_debug* debug,
                          void* ws, size_t ws_bytes, cudaStream_t stream) {
  return attn(Q, K, V, O, shape, params, debug, ws, ws_bytes, stream, false);
}

muse_status muse_attn_fwd_causal(const void* Q, const void* K, const void* V, void* O,
                                 const muse_shape* shape, const muse_params* params,
                                 muse_debug* debug, void* ws, size_t ws_bytes,
                                 cudaStream_t stream) {
  return attn(Q, K, V, O, shape, params, debug, ws, ws_bytes, stream, true);
}

muse_status muse_device_status(const int32_t* device_error, cudaStream_t stream) {
  if (!device_error) return fail(MUSE_ERR_INVALID_ARG, "device_error must not be NULL");
  if (misaligned(device_error, 4)) return fail(MUSE_ERR_INVALID_ARG, "device_error must be 4-byte aligned");
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, device_error, 4, cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    g_last_error = std::string("reading the device error word failed: ") + cudaGetErrorString(e);
    return MUSE_ERR_CUDA;
  }
  if (v == 0) return MUSE_OK;
  std::string msg = "device error word " + std::to_string(v) + ":";
  if (v & MUSE_DEVERR_MMA_WAIT) msg += " a tensor-core completion wait gave up;";
  if (v & MUSE_DEVERR_TEAM_BARRIER) msg += " a k-means team barrier gave up (outputs invalid);";
  if (v & MUSE_DEVERR_V_RANGE) msg += " V holds a finite value outside the fp16 range (output invalid);";
  g_last_error = msg;
  return MUSE_ERR_DEVICE_CHECK;
}

void muse_debug_inject_barrier_fault(int rank, int spin_limit) { set_barrier_fault(rank, spin_limit); }

const char* muse_status_string(muse_status s) {
  switch (s) {
    case MUSE_OK: return "ok";
    case MUSE_ERR_INVALID_ARG: return "invalid argument";
    case MUSE_ERR_UNSUPPORTED: return "unsupported shape or parameter";
    case MUSE_ERR_WORKSPACE: return "workspace too small";
    case MUSE_ERR_CUDA: return "CUDA error";
    case MUSE_ERR_DEVICE_CHECK: return "device-side check failed";
  }
  return "unknown status";
}

const char* muse_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
