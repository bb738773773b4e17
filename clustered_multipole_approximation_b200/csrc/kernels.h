// Host-side launchers shared between the translation units of libmuse.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace muse {

// Brackets one kernel launch with profiling events when profiling is on.
struct ProfScope {
  ProfScope(cudaStream_t st, const char* name);
  ~ProfScope();
  cudaStream_t st;
  int slot;
};

// Per-(query problem) stage-1 tables in the workspace.
struct Stage1 {
  float* logW;    // [nq][Cq][Ck]  log W_ij, -inf for empty key clusters
  float* fbias;   // [nq][Cq][Ck]  far-field logit offset (log W, plus the tilt term)
  // fp32 inputs: fp32 tables; bf16 inputs: the tensor-core operand forms
  float* U;       // [nq][Cq][Ck][D] summary values u_ij (fp32 path)
  float* Kf;      // [nq][Cq][Ck][D] far-field key rows, TILTED only: k_hat_ij (fp32 path)
  __half* Uh;     // [nq][Cq][Ck][D] u_ij in fp16 (bf16 path)
  __half* Ul;     // [nq][Cq][Ck][D] u_ij - Uh in fp16 (bf16 path)
  __nv_bfloat16* Kfh;  // [nq][Cq][Ck][D] bf16 hi / lo split of k_hat_ij (bf16 path, TILTED)
  __nv_bfloat16* Kfl;
  int* sel;       // [nq_total][Cq][topk]
  int* nsel;      // [nq_total][Cq]
};

struct AttnArgs {
  RoleGeo qg, kg;     // query and key geometry
  KState qs, ks;      // their k-means state
  const void* V;
  const __half* V16;  // fp16 copy of V (bf16 inputs; the PV operand)
  void* O;            // acausal: final output
  int out_f32;        // O is fp32 (else the input dtype)
  float* part;        // causal: [nq_total tokens][D + 1] partial (o, lse)
  long long* n_exact; // optional [B,Hq,N]
  int B;              // batch
  int G;              // q-heads per kv-head
  int mode, topk;
  float scale;
  int Cq, Ck;
  int dense_lv;       // causal levels (bit l) whose far field runs per key token
  int tc_lv;          // levels (bit l) whose stage 2 runs on the tensor-core kernel
  void* kpad;         // those levels' keys, cluster-sorted, group-padded, pre-swizzled (bf16)
  void* vpad;         // the same for V (fp16)
  int* gofs;          // [key problems][Ck + 1] first group of each cluster in kpad / vpad
  int tdip;           // stage 2 of the tilted per-pair dipole (stage 1 and selection: TILTED)
  int accum;          // causal local merge: one partial per query of blocks >= 1 at row
                      // b H N + q (block-summary accumulation), else the level partials
};

// Key problem that a query problem attends: the same (b, level, pair) of the
// kv-head its q-head shares.
__device__ inline int kv_problem(const AttnArgs& a, int qpid) {
  const int ppb = a.qg.lv.pairs_per_bh;
  const int bhq = qpid / ppb, pi = qpid - bhq * ppb;
  const int Hq = a.qg.BH / a.B, Hkv = a.kg.BH / a.B;
  const int b = bhq / Hq, hq = bhq - b * Hq;
  const int bhk = b * Hkv + hq / a.G;
  return bhk * a.kg.lv.pairs_per_bh + pi;
}

void run_kmeans(const RoleGeo& g, const KState& ks, int iters, const float* init,
                cudaStream_t st);

// Seeded (or given) start centroids for up to two problem sets, one launch.
void run_kmeans_init(const RoleGeo* gs, const KState* kss, int nsets, const float* init,
                     cudaStream_t st);

// All Lloyd rounds of up to two problem sets in one persistent launch
// (thread-block clusters, bf16 inputs); false if these sets are not covered.
bool launch_kmeans_fused(const RoleGeo* gs, const KState* kss, int nsets, int iters,
                         cudaStream_t st);

// Failure-path testing of the persistent k-means' team barrier.
void set_barrier_fault(int rank, int spin_limit);

// The resident-tile k-means for the problems of one level (lvl < 0: the
// acausal single level) whose centroid sums are certified exact; false when
// these sizes are not covered (nothing launched).
bool launch_kmeans_resident(const RoleGeo* gs, const KState* kss, int nsets, int lvl, int iters,
                            cudaStream_t st);
// Partial-sum blocks the resident k-means may need for one role's levels.
size_t resident_partial_blocks(const Levels& lv, int BH, int D, int C);

// Lloyd rounds one launch sequence at a time (any dtype / size).
void run_kmeans_rounds(const RoleGeo& g, const KState& ks, int iters, cudaStream_t st);

// Tensor-core (tcgen05) assignment screen for bf16 inputs.
void launch_assign_tc(const RoleGeo& g, const KState& ks, cudaStream_t st);

// Stage 1 + selection + stage 2 for query problems [qp0, qp0 + nqp).
void run_blocks(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st);

// fp16 copy of a bf16 tensor (n elements, n % 8 == 0); a finite value that
// overflows fp16 sets kErrVRange in *err.
void run_bf16_to_half(const void* src, __half* dst, size_t n, int* err, cudaStream_t st);

// Top-k1 key clusters of every query cluster (certified fp32 screen, exact
// fp64 scores for the candidates).
void run_select(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st);

// Stage 2 with one warp per 16-query slice (bf16 inputs, topk <= 64); false
// (nothing launched) when these arguments are not covered.
bool run_stage2_warp(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st);
// Tensor-core stage 2 (stage2_tc.cu): the levels it takes, the sorted key
// copies it reads (once per call, after the k-means) and the launch for the
// query problems [qp0, qp0 + nqp) at those levels.
int stage2_tc_levels(const Levels& lv, int D, int Cq, int Ck, int topk, int dense_lv);
void run_permute_keys(const AttnArgs& a, cudaStream_t st);
void run_stage2_tc(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st);

// Stage 2 on mma.sync tensor-core tiles (bf16 inputs).
void run_stage2_mma(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st);
// Stage 1 (DIPOLE) on tcgen05 tensor cores (bf16 inputs).
void run_stage1_dipole_tc(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st);

// The levels in a.dense_lv (bf16 DIPOLE, causal): far field and retrieved
// keys per key token on mma.sync tiles, no stage-1 tables.
void run_stage2_dense(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st);
// Levels the dense form covers for these sizes (bit l set), 0 if none.
int dense_levels(const Levels& lv, int D, int Cq, int Ck);
// Levels of the fine-query dipole (every level, acausal included), or -1 when
// the shape is outside the per-key-token kernel's limits.
int fine_query_dense_levels(const Levels& lv, int D, int Cq, int Ck);

// Backward pass of the acausal operator (backward.cu).
struct BwdArgs {
  const void* dO;  // gradient of the output [B,Hq,N,D]
  int o_f32;       // dO is fp32 (else the input dtype)
  float* dQ;       // [B,Hq,N,D]
  float* dK;       // [B,Hkv,N,D], zeroed by the caller
  float* dV;       // [B,Hkv,N,D], zeroed by the caller
  float* Sst;      // [key sets][Ck][D]    S_j
  float* Mst;      // [key sets][Ck][D][D] M_j (DIPOLE)
  float* U;        // [query sets][Cq][Ck][D] u_ij (DIPOLE)
  float* dU;       // [query sets][Cq][Ck][D], zeroed by the caller
  float* dmu;      // [key sets][Ck][D], zeroed by the caller
  float* dnu;      // [query sets][Cq][D], zeroed by the caller
  // causal only: per level-problem slot and per query row, (max, sum, sum of
  // p g) over that set of terms; then the combined log-sum-exp and D_q
  float* pm;       // [query tokens of all levels]
  float* pl;
  float* pa;
  float* lm;       // [B Hq N] the local block's
  float* ll;
  float* la;
  float* lse_all;  // [B Hq N]
  float* d_all;    // [B Hq N]
};
bool backward_supported(int D, int Ck, int mode);
// Causal backward (the hierarchical levels plus the local blocks of L keys).
void run_attn_bwd_causal(const AttnArgs& a, const Stage1& s1, const BwdArgs& b, int L,
                         cudaStream_t st);
void run_attn_bwd(const AttnArgs& a, const Stage1& s1, const BwdArgs& b, cudaStream_t st);

// Causal operator with block-summary accumulation (accum.cu).
struct AccArgs {
  int L, NB, k2;   // block size, blocks, blocks retrieved per selected cluster
  int* kboff;      // [key sets][Ck][NB + 1] first member of each block in a cluster's list
  int* qboff;      // [query sets][Cq][NB + 1]
  int* bn;         // [key sets][NB][Ck] members of (block, cluster)
  int* pn;         // [key sets][NB][Ck] exclusive prefix over blocks
  double* bk;      // [key sets][NB][Ck][D] key sums (token order)
  double* pk;      // prefix of bk (block order)
  double* bmu;     // [key sets][Ck][D][NB] bk / bn (fp64 division), block index fastest
  double* pmu;     // [key sets][NB][D][Ck] pk / pn, dimension-major
  float* bs;       // [key sets][NB][Ck][D] value sums
  float* ps;       // prefix of bs
  float* ba;       // [query sets][NB][Cq][Ck][D] sum v (k . nu_i) (DIPOLE)
  float* pa;       // prefix of ba
  int* sel1;       // [query sets][NB][Cq][k1] selected key clusters, -1 padded
  int* sel2;       // [query sets][NB][Cq][k1][k2] selected blocks, -1 padded
};
bool accum_supported(int D, int Cq, int Ck, int NB, int k1, int k2, int mode);
void run_accum(const AttnArgs& a, const AccArgs& c, cudaStream_t st);

// Stage 2 of the tilted per-pair dipole (stage2_tdip.cu): per key token, SIMT.
void run_stage2_tdip(const AttnArgs& a, const Stage1& s1, int qp0, int nqp, cudaStream_t st);

// Causal: exact local block + merge of the level partials into O.
void run_local_merge(const AttnArgs& a, int L, cudaStream_t st);
// The same on mma.sync tiles (bf16, L a multiple of 128); false if not covered.
bool run_local_mma(const AttnArgs& a, int L, cudaStream_t st);

// Summaries (n, mu, S, M) of given assignments; used by muse_summarize.
void run_summarize(const void* K, const void* V, int dtype, int BH, int N, int D, int C,
                   const int* assign, int* counts, float* mu, float* S, float* M,
                   int* perm, int* off, cudaStream_t st);

}  // namespace muse
