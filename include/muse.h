/*
 * libmuse -- B200 (sm_100a) implementation of the forward operator of
 * Multipole Semantic Attention (MuSe).
 *
 * Sources.  All cited pages carry the title "Multipole Semantic Attention:
 * A Fast Approximation of Softmax Attention for Pretraining":
 *   [G]  the gist.science page, section "Technical Summary" -> "Methodology"
 *        -> "Core Mechanisms" (bidirectional clustering, residual
 *        decomposition, stage 1 / stage 2, exponential tilting, retrieval);
 *   [A1] the newx.sg page, section "Abstract" (monopole + dipole
 *        corrections, hierarchical block decomposition for causal attention,
 *        O(NCD) acausal and O(NCD log N) causal cost).
 *
 * Conventions shared by every entry point.
 *   - All tensor arguments are DEVICE pointers to contiguous row-major data;
 *     the caller owns every buffer, including the workspace.  The library
 *     never allocates, frees or synchronises: all work is enqueued on the
 *     given stream and the call returns before it finishes.
 *   - Q is [B,Hq,N,D]; K and V are [B,Hkv,N,D]; O has Q's shape, and Q's
 *     dtype unless muse_shape.out_f32 asks for fp32.
 *     q-head h reads kv-head h / (Hq/Hkv) (grouped-query attention).
 *   - Arguments are validated before anything is launched; a failing check
 *     returns MUSE_ERR_INVALID_ARG (or MUSE_ERR_UNSUPPORTED for shapes the
 *     kernels do not cover, or MUSE_ERR_WORKSPACE for a short workspace) and
 *     leaves every output untouched.  A launch error reported by the CUDA
 *     runtime returns MUSE_ERR_CUDA.  muse_last_error() then gives a message
 *     (per host thread).
 *   - Alignment: every tensor pointer (Q, K, V, O, X, init, the summary
 *     outputs) must be 16-byte aligned, the workspace 256-byte aligned, and
 *     the optional int32 / int64 debug outputs aligned to their element
 *     size; a misaligned pointer returns MUSE_ERR_INVALID_ARG before any
 *     launch.
 *   - Device-side status: a few conditions can only be seen on the GPU (a
 *     bounded wait that gave up, a value the kernels cannot represent).  The
 *     kernels then record a non-zero MUSE_DEVERR_* bit set in a device error
 *     word instead of faulting; entry points that take a `device_error`
 *     pointer copy that word there on the stream, and muse_device_status()
 *     turns it into MUSE_OK or MUSE_ERR_DEVICE_CHECK.
 *   - Calls with distinct workspaces and outputs may run concurrently.
 */
#ifndef MUSE_H_
#define MUSE_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MUSE_OK = 0,
  MUSE_ERR_INVALID_ARG = 1,
  MUSE_ERR_UNSUPPORTED = 2,
  MUSE_ERR_WORKSPACE = 3,
  MUSE_ERR_CUDA = 4,
  MUSE_ERR_DEVICE_CHECK = 5
} muse_status;

/* Bits of the device error word (0 = every kernel finished normally). */
enum {
  /* A wait for tensor-core (tcgen05) completion gave up after its bound.  The
   * k-means re-decides the affected tokens on its fp64 path; other kernels'
   * outputs are unreliable. */
  MUSE_DEVERR_MMA_WAIT = 1,
  /* A barrier between the CTAs of one k-means problem (cooperative launch)
   * gave up after its bound, because a CTA never arrived; every CTA of the
   * problem then stops, and the clustering outputs are invalid. */
  MUSE_DEVERR_TEAM_BARRIER = 2,
  /* A finite bf16 value of V lies outside the fp16 range (|v| >= 65520), so
   * its fp16 tensor-core operand became infinite; the output is invalid. */
  MUSE_DEVERR_V_RANGE = 4
};

typedef enum { MUSE_BF16 = 0, MUSE_F32 = 1 } muse_dtype;

/* Far-field summary of a key cluster j as seen from query cluster i:
 *   MONOPOLE  count, centroid and summed values ([A1] Abstract; [G] Core
 *             Mechanisms, "Retrieval-Augmented Approximation");
 *   DIPOLE    MONOPOLE plus the first-order correction (s/n_j) M_j nu_i with
 *             M_j = sum_{t in j} v_t (k_t - mu_j)^T ([A1] Abstract);
 *   TILTED    exponentially tilted summaries weighted by exp(s nu_i . k_t)
 *             ([G] Core Mechanisms, "Exponential Tilting");
 *   DIPOLE_Q  an accuracy variant of DIPOLE: the first-order correction is
 *             taken at each query, (s/n_j) M_j q, instead of at its cluster
 *             centroid nu_i ([A1] Abstract: the dipole expands exp(s q.k)
 *             around the centroid of the keys, and q is the expansion's own
 *             variable).  Selection is the same as DIPOLE's.  The far field
 *             is evaluated as one softmax term per key token (weight
 *             exp(s q.mu_a(t)), value factor 1 + s q.(k_t - mu_a(t))),
 *             O(N^2 D) work like exact attention, so it serves as an
 *             accuracy reference rather than a fast path.  Supported for
 *             dtype MUSE_BF16 with Cq, Ck <= 256 and every block size (N for
 *             muse_attn_fwd, L 2^l for muse_causal_fwd) a multiple of 128;
 *             other shapes return MUSE_ERR_UNSUPPORTED.
 *   TILTED_DIPOLE  an accuracy variant of TILTED: the tilt exp(s nu_i . k_t)
 *             is kept exactly and exp(s (q - nu_i) . k_t) is expanded to
 *             first order about the tilted centroid k^_ij, so the value gains
 *             s M^_ij (q - nu_i) (M^_ij: the tilted value-key moment about
 *             k^_ij) and the weight is TILTED's.  Stage 1 and the selection
 *             are TILTED's; the far field is evaluated per key token (fp32,
 *             O(N^2 D) like exact attention), an accuracy reference.  Both
 *             dtypes, acausal and causal.
 */
typedef enum {
  MUSE_MONOPOLE = 0,
  MUSE_DIPOLE = 1,
  MUSE_TILTED = 2,
  MUSE_DIPOLE_Q = 3,
  MUSE_TILTED_DIPOLE = 4
} muse_mode;

typedef struct {
  int B, Hq, Hkv, N, D; /* D in {64, 128}; Hq % Hkv == 0 */
  muse_dtype dtype;     /* of Q, K and V (and of O unless out_f32) */
  int out_f32;          /* 0: O in dtype; 1: O in fp32 */
} muse_shape;

typedef struct {
  int Cq, Ck;      /* query and key clusters (causal: both = C per level) */
  int iters;       /* Lloyd iterations, >= 1 */
  uint64_t seed;   /* seeds the k-means start rows */
  int topk;        /* k1: key clusters retrieved exactly per query cluster */
  int block;       /* causal local block L (ignored by muse_attn_fwd) */
  float scale;     /* softmax scale s: logits are s q.k */
  muse_mode mode;
  /* Stream ids of the first key and query row sets, (b, h) = (0, 0): row set
   * (b, h) of this call draws its seeded k-means start from stream
   * stream0 + b H + h.  0 for a whole layer; a shard of a layer made of
   * consecutive (b, kv-head) units u0 .. u1 (each unit one batch entry with
   * Hkv = 1 and Hq = G) passes key_stream0 = u0 and query_stream0 = G u0 and
   * gets bit for bit the whole layer's rows. */
  uint64_t key_stream0, query_stream0;
} muse_params;

/* Optional device outputs for inspection; any member may be NULL.
 * Acausal layouts: q_assign [B,Hq,N], k_assign [B,Hkv,N],
 *   q_centroids [B,Hq,Cq,D], k_centroids [B,Hkv,Ck,D], k_counts [B,Hkv,Ck],
 *   selected [B,Hq,Cq,topk] (rank order, -1 padded), n_exact [B,Hq,N].
 * Causal layouts: q_assign [B,Hq,levels,N/2], k_assign [B,Hkv,levels,N/2]
 *   (entry (l, p*s + r) is token r of pair p's block at level l, s = L 2^l),
 *   selected [B,Hq,P,Cq,topk] with P = N/L - 1 block problems per head,
 *   numbered level by level (level l's pairs start at sum_{l'<l} N/(2 s_l')),
 *   rows i >= min(Cq, s) are -1; n_exact [B,Hq,N]; the centroid and count
 *   members are not written by the causal entry point. */
typedef struct {
  int32_t *q_assign, *k_assign, *selected, *k_counts;
  float *q_centroids, *k_centroids;
  int64_t *n_exact;
  int32_t *device_error; /* the device error word: 0 or MUSE_DEVERR_* bits */
} muse_debug;

/* Workspace bytes muse_attn_fwd (causal == 0) or muse_attn_fwd_causal
 * (causal != 0) needs for this shape and these parameters; 0 if the
 * arguments are invalid. */
size_t muse_workspace_size(const muse_shape *shape, const muse_params *params,
                           int causal);

/* Waits for `stream`, reads a device error word written by an entry point
 * (`device_error`, a device pointer to one int32) and returns MUSE_OK if it
 * is 0, else MUSE_ERR_DEVICE_CHECK with a message naming the MUSE_DEVERR_*
 * bits (MUSE_ERR_CUDA if the stream or the copy fails).  The one call of
 * the library that synchronises. */
muse_status muse_device_status(const int32_t *device_error, cudaStream_t stream);

/* Workspace bytes of muse_cluster / muse_summarize for these sizes. */
size_t muse_cluster_workspace_size(int B, int H, int N, int D, int C);

/*
 * Lloyd k-means of every (b, h) row set of X [B,H,N,D] into C clusters
 * ([G] Core Mechanisms, "Bidirectional Semantic Clustering"; the algorithm
 * is not named on the pages -- Lloyd with squared Euclidean distance is the
 * reading taken here).
 *   iters        >= 1 rounds of (assign, update).  Ties in the assignment
 *                go to the lowest cluster index; an empty cluster keeps its
 *                previous centroid.
 *   init         NULL: start from C distinct rows chosen by a partial
 *                Fisher-Yates shuffle driven by splitmix64 seeded with
 *                seed + 0x9E3779B97F4A7C15 * (2 (b H + h) + role + 1);
 *                else fp32 start centroids [B,H,C,D].
 *   role         0 = key stream, 1 = query stream (selects the seed stream;
 *                muse_attn_fwd clusters keys with role 0 and queries with
 *                role 1).
 *   assign       out [B,H,N] int32: cluster of each row after the last round.
 *   centroids    out [B,H,C,D] fp32: centroids after the last update.
 *   counts       out [B,H,C] int32 (may be NULL).
 *   device_error out, one int32 (may be NULL): the device error word.
 * 1 <= C <= min(N, 1024); D in {64, 128}.
 */
muse_status muse_cluster(const void *X, muse_dtype dtype, int B, int H, int N,
                         int D, int C, int iters, uint64_t seed, int role,
                         const float *init, int32_t *assign, float *centroids,
                         int32_t *counts, int32_t *device_error, void *ws,
                         size_t ws_bytes, cudaStream_t stream);

/*
 * Key-cluster summaries for a given assignment ([A1] Abstract: monopole and
 * dipole): counts n_j, centroid mu_j (mean of members; zero when empty),
 * S_j = sum_{t in j} v_t and M_j[e][d] = sum_{t in j} v_t[e] (k_t[d] - mu_j[d]).
 *   assign  [B,H,N] int32 in [0, C).
 *   counts [B,H,C] int32, mu [B,H,C,D] f32, S [B,H,C,D] f32,
 *   M [B,H,C,D,D] f32 (M may be NULL).
 */
muse_status muse_summarize(const void *K, const void *V, muse_dtype dtype,
                           int B, int H, int N, int D, int C,
                           const int32_t *assign, int32_t *counts, float *mu,
                           float *S, float *M, void *ws, size_t ws_bytes,
                           cudaStream_t stream);

/*
 * Acausal MuSe forward ([G] Core Mechanisms; [A1] Abstract, O(NCD) form).
 * Per (b, kv-head) the keys are clustered (Ck) and summarised; per q-head the
 * queries are clustered (Cq).  Stage 1 scores every key cluster j from every
 * query cluster i, s_ij = s nu_i.mu_j + log W_ij, and retrieves the top
 * `topk` (ties to the lowest j, empty clusters never).  Stage 2 gives each
 * query one far-field term per other non-empty cluster (logit
 * s q.mu_j + log W_ij, or for TILTED s (q - nu_i).k_hat_ij + s nu_i.mu_j +
 * log W_ij; value u_ij) plus one exact term per key of the retrieved
 * clusters, all in one softmax.  O is written in the input dtype (fp32 with
 * out_f32).  Accumulation is fp32 or wider.  For bf16 inputs the tensor-core
 * operands are 16-bit: q, k and v exactly; centroids, summary values u_ij
 * and far-field weights as bf16/fp16 hi + lo pairs; the softmax weights of
 * exact keys rounded once to fp16.
 * Requires 1 <= Cq, Ck <= min(N, 1024), 0 <= topk <= Ck, iters >= 1.
 */
muse_status muse_attn_fwd(const void *Q, const void *K, const void *V, void *O,
                          const muse_shape *shape, const muse_params *params,
                          muse_debug *debug, void *ws, size_t ws_bytes,
                          cudaStream_t stream);

/*
 * Causal MuSe forward by the hierarchical block decomposition ([A1]
 * Abstract).  With L = params->block (N % L == 0, N/L a power of two), the
 * query at position q in block b = q / L attends exactly to the keys
 * [bL, q] of its own block, and for every level l whose bit is set in b to
 * the key block [2p s, (2p+1) s) (s = L 2^l, p = b >> (l+1)) through one MuSe
 * block problem clustered inside that key block and the query block
 * [(2p+1) s, (2p+2) s) with C_eff = min(Ck, s) clusters; topk is a per-block
 * problem budget.  All terms meet in one softmax.  Requires Cq == Ck.
 * For bf16 DIPOLE, levels with s <= 8 C_eff (s a multiple of 128, Ck <= 256)
 * evaluate the far field one key token at a time (the same sums, expanded
 * over each cluster's tokens) instead of through per-cluster summaries.
 */
muse_status muse_attn_fwd_causal(const void *Q, const void *K, const void *V,
                                 void *O, const muse_shape *shape,
                                 const muse_params *params, muse_debug *debug,
                                 void *ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Causal MuSe with causal accumulation of block summaries and two-level
 * retrieval ([G] Technical Summary, Core Mechanisms: "Causal Accumulation"
 * and "Retrieval-Augmented Approximation").  Keys and queries are clustered
 * over the whole sequence (the clusterings of muse_attn_fwd).  With
 * L = params->block (N % L == 0) and NB = N / L blocks, a query q in block b
 * attends exactly to the keys [bL, q] of its own block and, for b >= 1:
 *   - selects the top params->topk key clusters j by
 *     s nu_i . mu_j^{<b} + log n_j^{<b}, the summary of j's members in blocks
 *     0 .. b-1 accumulated block by block (fp64, ties to the lowest j);
 *   - within each, the top topk2 blocks b' < b by s nu_i . mu_jb' + log n_jb'
 *     (ties to the lowest block), and attends exactly to their keys;
 *   - sees every key cluster's remaining prefix members (outside the
 *     retrieved blocks) as one far term: logit s q.mu + log n, value S / n
 *     (MONOPOLE) or (S + s M nu_i) / n (DIPOLE, M about that set's centroid).
 * All terms meet in one softmax.  topk2 == 0 retrieves nothing.  Supported:
 * MONOPOLE and DIPOLE, Cq, Ck <= 256, Ck * D <= 16384, topk <= 32,
 * N / L <= 1024, and for DIPOLE Cq * D <= 8192 (MUSE_ERR_UNSUPPORTED
 * otherwise).
 * Debug layouts: q_assign [B,Hq,N], k_assign [B,Hkv,N],
 * sel1 [B,Hq,NB,Cq,topk], sel2 [B,Hq,NB,Cq,topk,topk2] (-1 padded; rows of
 * block 0 and of clusters with no query in the block are -1),
 * n_exact [B,Hq,N] (retrieved plus local keys).
 */
typedef struct {
  int32_t *q_assign, *k_assign, *sel1, *sel2;
  int64_t *n_exact;
  int32_t *device_error;
} muse_accum_debug;

size_t muse_accum_workspace_size(const muse_shape *shape, const muse_params *params, int topk2);
muse_status muse_attn_fwd_causal_accum(const void *Q, const void *K, const void *V, void *O,
                                       const muse_shape *shape, const muse_params *params,
                                       int topk2, muse_accum_debug *debug, void *ws,
                                       size_t ws_bytes, cudaStream_t stream);

/*
 * Gradients of the acausal operator: dQ, dK, dV of <dO, O> for the O of a
 * muse_attn_fwd call ([G] Experimental Results: the layer is trained
 * through).  The clusterings and the retrieval sets are held at the forward
 * call's values (they are piecewise constant in the inputs); centroids, S_j,
 * M_j and the query centroids are differentiated through the member means and
 * sums they are.  Call order: size the workspace with
 * muse_attn_bwd_workspace_size(), pass that workspace to muse_attn_fwd (with
 * the same Q, K, V, shape and params), then to this function, unchanged in
 * between: the backward reads the forward's clusterings and selections from
 * it, and uses the space after the forward's part as scratch.  dO is
 * [B,Hq,N,D] in the output dtype (fp32 if shape->out_f32); dQ [B,Hq,N,D],
 * dK and dV [B,Hkv,N,D] are fp32, overwritten.  fp32 arithmetic; O itself is
 * not read: sum_t p_t dO.x_t (= dO.O) is formed from the backward's own
 * terms.  dK, dV and dQ are sums of fp32 atomic adds, so their last bits may
 * differ from call to call.
 * Supported: modes MONOPOLE and DIPOLE, Ck * D <= 16384; other modes and
 * sizes return MUSE_ERR_UNSUPPORTED.  (The causal operator's gradients:
 * muse_attn_bwd_causal below.)  A workspace smaller than
 * muse_attn_bwd_workspace_size() returns MUSE_ERR_WORKSPACE.
 */
size_t muse_attn_bwd_workspace_size(const muse_shape *shape, const muse_params *params);
muse_status muse_attn_bwd(const void *Q, const void *K, const void *V, const void *dO,
                          float *dQ, float *dK, float *dV, const muse_shape *shape,
                          const muse_params *params, void *ws, size_t ws_bytes,
                          cudaStream_t stream);

/*
 * Gradients of the causal operator (muse_attn_fwd_causal), with the same
 * contract as muse_attn_bwd: the workspace sized by
 * muse_attn_bwd_causal_workspace_size() goes to muse_attn_fwd_causal first
 * and then, unchanged, here.  Every query's terms -- its local block and the
 * level problems it is a query of -- meet in one softmax, so the backward
 * first forms each query's combined log-sum-exp and sum of p dO.x (per level
 * problem and per local block, then combined), then the gradients of every
 * term; a query's and a key's gradient is summed over its levels by fp32
 * atomic adds.  Modes MONOPOLE and DIPOLE, Ck * D <= 16384, block % 32 == 0
 * (MUSE_ERR_UNSUPPORTED otherwise).
 */
size_t muse_attn_bwd_causal_workspace_size(const muse_shape *shape, const muse_params *params);
muse_status muse_attn_bwd_causal(const void *Q, const void *K, const void *V, const void *dO,
                                 float *dQ, float *dK, float *dV, const muse_shape *shape,
                                 const muse_params *params, void *ws, size_t ws_bytes,
                                 cudaStream_t stream);

/*
 * muse_cluster without a workspace argument, for callers that cannot
 * allocate device memory (no counterpart on the pages: this is a packaging
 * choice of this library).  The scratch comes from a fixed array compiled
 * into the library (muse_cluster_static_capacity() bytes, 16 MiB, held on
 * every GPU that loads the library until the process exits); sizes whose
 * muse_cluster_workspace_size() exceeds it return MUSE_ERR_WORKSPACE with a
 * message and launch nothing.  The first call on each device looks up the
 * array's device address (cudaGetSymbolAddress, with that device current):
 * make that first call before any stream capture.  The looked-up address is
 * kept for the life of the process: after cudaDeviceReset() on a device the
 * kept address is stale, so do not call this entry point on that device
 * again in the same process.  All calls share the one array and it keeps the
 * last call's contents -- the parts that must start at zero are cleared by
 * each call -- so calls whose work overlaps on the GPU (other streams, other
 * host threads) race.  Arguments and outputs are those of muse_cluster.
 */
muse_status muse_cluster_static(const void *X, muse_dtype dtype, int B, int H,
                                int N, int D, int C, int iters, uint64_t seed,
                                int role, const float *init, int32_t *assign,
                                float *centroids, int32_t *counts,
                                int32_t *device_error, cudaStream_t stream);

/* Bytes of the scratch array built into the library for muse_cluster_static. */
size_t muse_cluster_static_capacity(void);

const char *muse_status_string(muse_status status);

/* Per-kernel timing, for benchmarks (instrumentation only; no paper
 * counterpart).  While enabled, every kernel launched by the library is
 * bracketed by two CUDA events recorded on its launch stream.
 * muse_profile_read() waits for the recorded events, writes up to `cap`
 * entries -- kernel name (NUL-terminated, at most name_stride bytes, into
 * names + i * name_stride), launch count and summed milliseconds -- returns
 * the number of distinct kernels, and clears the record.  Not thread-safe. */
void muse_profile_enable(int on);
int muse_profile_read(char *names, int name_stride, int *launches, double *ms,
                      int cap);

/* Failure-path testing (no paper counterpart).  While rank >= 0, the
 * persistent k-means of this process runs every problem on its
 * sequential-order kernel, and each of that kernel's cooperative launches
 * lets CTA `rank` of each problem skip its arrival at the first barrier;
 * every barrier wait gives up after `spin_limit` polls (about 64 ns apart):
 * the kernel then records MUSE_DEVERR_TEAM_BARRIER and returns without
 * touching its outputs.  rank < 0 restores normal operation.  Not
 * thread-safe. */
void muse_debug_inject_barrier_fault(int rank, int spin_limit);

/* Message of the last failing call on this host thread ("" if none). */
const char *muse_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MUSE_H_ */
