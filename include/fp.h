/*
 * fp.h -- C ABI of the FlexPrefill prefill-attention hot path on B200 (sm_100a).
 *
 * The method (FlexPrefill: A Context-Aware Sparse Attention Mechanism for
 * Efficient Long-Sequence Inference; atlas.scime.ai summary, "Approach"):
 * for every attention head, estimate block-pooled attention from the last
 * query block, compare it with the true distribution by the square root of
 * the Jensen-Shannon divergence, choose query-aware block selection when the
 * estimate is accurate and a vertical-slash pattern otherwise, keep the
 * smallest set of blocks/lines whose cumulative normalised attention reaches
 * gamma (within min/max token budgets), and run causal block-sparse
 * attention over the kept blocks.  The abstract (same title; OpenReview and
 * codewithpapers pages) names the two parts "Query-Aware Sparse Pattern
 * Determination" and "Cumulative-Attention Based Index Selection".
 *
 * Conventions shared by every call
 * --------------------------------
 *  * Layouts are dense and row-major (C order):
 *      q            [Bt, Hq,  N, d]   (fp_shape.dtype: bf16 or fp32)
 *      k, v         [Bt, Hkv, N, d]
 *      out          [Bt, Hq,  N, d]   (same dtype as q)
 *    with N = seq_len, d = head_dim, B = block_size, nb = ceil(N / B),
 *    T = nb (nb + 1) / 2 and g = Hq / Hkv; query head h reads kv head h / g.
 *    When B does not divide N the last block is partial: it holds the
 *    N - (nb - 1) B tokens left, is pooled over those tokens, is the last
 *    query block of the estimate (its queries are the representative ones),
 *    and attention reads no key or query position at or past N.
 *  * Every data pointer is DEVICE memory owned by the caller, except the
 *    *_host pointers of fp_prefill_attn_host.  The library allocates no
 *    device memory; scratch space is the caller's workspace (`ws`, at least
 *    fp_workspace_size() bytes, 256-byte aligned).  A workspace must not be
 *    shared by calls that may run concurrently.
 *  * Device data pointers must be aligned: q, k, v, out, qbar and kbar to
 *    16 bytes (they are moved with 16-byte vector accesses and tensor-map
 *    copies), every other array to its element size (4 bytes; stats 8).
 *    torch allocations and views that start on such a boundary qualify; a
 *    misaligned pointer returns FP_ERR_ALIGN.
 *  * Arguments are validated on the host before anything is launched; a
 *    failed check returns an error code and launches nothing.
 *  * Kernels run asynchronously on `stream` (NULL = the legacy default
 *    stream).  A launch failure returns FP_ERR_CUDA.  Errors found on the
 *    device (an index outside the causal range, a pipeline wait that ran out
 *    of time) are recorded in a per-device status word and read with
 *    fp_last_device_status().
 *  * No C++ exception crosses this ABI.  Calls on distinct streams with
 *    distinct workspaces may run from several host threads.
 *  * The device-memory calls (all but fp_prefill_attn_host) launch only on
 *    `stream` and do not synchronise, so they may be captured into a CUDA
 *    graph; make one eager call on the device first (it caches the device's
 *    status word and properties).  A replay reads the current contents of
 *    the captured buffers.
 *  * Supported shapes: N >= 1 (any length), nb <= 4096, Hq % Hkv == 0,
 *    B in {64, 128}, d in {64, 128}.  The bf16 attention (tensor cores)
 *    needs d == 128; fp32 (the debug path, CUDA cores) takes every listed
 *    shape.
 */
#ifndef FP_H_
#define FP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t (struct CUstream_st *). */
typedef struct CUstream_st *fp_stream_t;

typedef enum {
  FP_OK = 0,
  FP_ERR_NULL = 1,          /* a required pointer is NULL                        */
  FP_ERR_SHAPE = 2,         /* unsupported or inconsistent shape                 */
  FP_ERR_DTYPE = 3,         /* unsupported dtype for this call                   */
  FP_ERR_PARAM = 4,         /* gamma / tau / budget out of range                 */
  FP_ERR_WORKSPACE = 5,     /* workspace NULL, misaligned or too small          */
  FP_ERR_CUDA = 6,          /* a CUDA runtime call or launch failed              */
  FP_ERR_TIMEOUT = 7,       /* device: a pipeline wait ran out of time           */
  FP_ERR_DEVICE_CHECK = 8,  /* device: an argument failed an on-device check     */
  FP_ERR_UNSUPPORTED = 9,   /* the current device is not sm_100                  */
  FP_ERR_ALIGN = 10         /* a data pointer is not aligned as required         */
} fp_status;

typedef enum { FP_BF16 = 0, FP_F32 = 1 } fp_dtype;

typedef struct {
  int batch;       /* Bt                                    */
  int n_q_heads;   /* Hq                                    */
  int n_kv_heads;  /* Hkv, divides Hq (grouped-query heads) */
  int seq_len;     /* N >= 1; need not be a multiple of B   */
  int head_dim;    /* d                                     */
  int block_size;  /* B                                     */
  fp_dtype dtype;  /* element type of q, k, v and out       */
} fp_shape;

typedef struct {
  float gamma;     /* cumulative-attention threshold, 0 < gamma <= 1 (>= 1 keeps all) */
  float tau;       /* JS-distance threshold, >= 0; tau == 0 disables query-aware mode   */
  int min_budget;  /* tokens per query row, >= 0 (0: no minimum)                        */
  int max_budget;  /* tokens per query row; <= 0: uncapped                              */
  int qa_mode;     /* query-aware heads: FP_QA_FLATTENED (0, the default) or
                      FP_QA_QUERYWISE (1); anything else is FP_ERR_PARAM           */
  int vs_mode;     /* vertical-slash heads: FP_VS_TOKENS (0, the default) or
                      FP_VS_BLOCKS (1); anything else is FP_ERR_PARAM              */
} fp_params;

/*
 * Selection rule for query-aware heads (atlas.scime.ai summary, "Measured
 * effects": the flattened estimated map, and query-wise index selection as the
 * alternative the ablation compares):
 *   FP_QA_FLATTENED  one rule over the whole flattened causal map of the head,
 *                    budgets nb * ceil(min/B) .. nb * floor(max/B) block pairs;
 *   FP_QA_QUERYWISE  one rule per query-block row i over A[i, 0..i] with the
 *                    row's own total, budgets min(i+1, ceil(min/B)) ..
 *                    min(i+1, floor(max/B)) blocks (i+1 when uncapped).
 * Both keep every row's diagonal block.  Vertical-slash heads are unaffected.
 */
enum { FP_QA_FLATTENED = 0, FP_QA_QUERYWISE = 1 };

/*
 * Line granularity for vertical-slash heads (atlas.scime.ai summary,
 * "Approach": the smallest set of "blocks/lines" reaching gamma):
 *   FP_VS_TOKENS  lines are tokens: columns t and offsets o are selected from
 *                 vert[N] and slash[N] with budgets min .. max lines, then
 *                 column t covers key block t/B and offset o the block
 *                 distances floor(o/B) and, if B does not divide o, +1;
 *   FP_VS_BLOCKS  lines are blocks: vert is summed per key block and slash per
 *                 block distance floor(o/B) (float64, one add at a time in
 *                 ascending order, rounded to float32 once), and the rule picks
 *                 key blocks and block distances directly with budgets
 *                 ceil(min/B) .. floor(max/B) blocks.
 * With FP_VS_BLOCKS, fp_select uses counts and indices as scratch for the
 * pooled lines before it writes the lists.
 */
enum { FP_VS_TOKENS = 0, FP_VS_BLOCKS = 1 };

enum { FP_PATTERN_QA = 0, FP_PATTERN_VS = 1 };

/* Calls that take a workspace, for fp_workspace_size(). */
enum {
  FP_CALL_ESTIMATE = 0,
  FP_CALL_SELECT = 1,
  FP_CALL_SPARSE_ATTN = 2,
  FP_CALL_PREFILL = 3,      /* fp_prefill_attn: every intermediate lives in ws     */
  FP_CALL_PREFILL_HOST = 4  /* fp_prefill_attn_host: also device copies of q,k,v,out */
};

/* Bytes of workspace `which_call` needs for `shape` (0 if the shape is invalid). */
size_t fp_workspace_size(const fp_shape *shape, int which_call);

/*
 * fp_estimate -- the pattern-determination inputs of every head.
 * Source: atlas.scime.ai summary, "Approach" (block-pooled estimate from the
 * last query block; the true distribution; vertical-slash lines).
 *   qbar      [Bt,Hq,nb,d]  fp32  mean of q over each block of B tokens
 *   kbar      [Bt,Hkv,nb,d] fp32  mean of k over each block
 *   map       [Bt,Hq,T]     fp32  estimated block map: row i (stored at
 *             i(i+1)/2 .. i(i+1)/2+i) is the softmax over key blocks j <= i of
 *             qbar[i].kbar[j] / sqrt(d)
 *   est_last  [Bt,Hq,nb]    fp32  the last row of map (the estimate a-hat)
 *   true_last [Bt,Hq,nb]    fp32  true attention of the last query block,
 *             summed over the keys of each block and averaged over its R rows
 *   vert      [Bt,Hq,N]     fp32  vert[t]  = sum over the last R queries of P[r,t]
 *   slash     [Bt,Hq,N]     fp32  slash[o] = sum over r of P[r, N-R+r-o]
 * where P is the causal softmax of q.k/sqrt(d) for the last block's R
 * queries (R = B, or the partial last block's length).
 * Arithmetic: fp32 accumulation throughout.  The map's logits are tensor-core
 * products of the fp32 pooled vectors split into tf32 halves (3 products per
 * pair), off by at most about 2^-19 of sum_k |qbar_k kbar_k| / sqrt(d); for
 * bf16 inputs the last block's scores are tensor-core products of q and k
 * (fp32 inputs: fp32 products on the CUDA cores).
 * Workspace: fp_workspace_size(shape, FP_CALL_ESTIMATE).
 */
fp_status fp_estimate(const fp_shape *shape, const void *q, const void *k,
                      float *qbar, float *kbar, float *map, float *est_last,
                      float *true_last, float *vert, float *slash,
                      void *ws, size_t ws_bytes, fp_stream_t stream);

/*
 * fp_pattern -- per-head pattern choice.
 * Source: atlas.scime.ai summary, "Approach" (square-root JS divergence of
 * the estimate against the true distribution) and its "Measured effects"
 * table (tau = 0 disables query-aware mode, so the test is strict).
 *   djs     [Bt,Hq] fp32   sqrt(JSD(est_last, true_last)), natural log, both
 *                          inputs renormalised; computed in fp64
 *   pattern [Bt,Hq] int32  FP_PATTERN_QA if djs < tau (fp64 compare), else VS
 */
fp_status fp_pattern(const fp_shape *shape, const fp_params *params,
                     const float *est_last, const float *true_last,
                     float *djs, int32_t *pattern, fp_stream_t stream);

/*
 * fp_select -- cumulative-attention index selection.
 * Source: atlas.scime.ai summary, "Approach" (smallest set of blocks/lines
 * whose cumulative normalised attention reaches gamma) and "Measured effects"
 * (min/max budgets; the flattened estimated map).
 * Rule for one list of fp32 scores: order by score descending, then index
 * ascending; masses w = ceil(score * 2^32) as integers; keep the shortest
 * prefix whose mass reaches (double)gamma * (double)sum(w); clamp its length
 * to [lo, hi].
 *   QA heads: the list is map[h] flattened (packed index), lo = min(T,
 *     nb*ceil(min_budget/B)), hi = nb*floor(max_budget/B) (or T), each kept
 *     pair (i, j) adds block j to row i.
 *   VS heads: vert[h] and slash[h] are two lists of N lines, lo =
 *     min(N, min_budget), hi = max_budget (or N); a kept column t adds key
 *     block t/B to every row; a kept offset o adds every block pair at
 *     distance o/B (and o/B + 1 when B does not divide o).
 *   Every row also keeps its diagonal block.
 *   counts  [Bt,Hq,nb]     int32  blocks kept in row i (1..i+1)
 *   indices [Bt,Hq,nb,nb]  int32  row i's blocks, ascending, in the first
 *                                 counts[i] slots (the rest is not written)
 * The result is exact (integer arithmetic on the given fp32 scores).
 * Workspace: fp_workspace_size(shape, FP_CALL_SELECT).
 */
fp_status fp_select(const fp_shape *shape, const fp_params *params,
                    const int32_t *pattern, const float *map, const float *vert,
                    const float *slash, int32_t *counts, int32_t *indices,
                    void *ws, size_t ws_bytes, fp_stream_t stream);

/*
 * fp_select_noalloc -- fp_select for callers that cannot allocate device
 * memory when they call in.  Some hosts own every byte of device memory and
 * plan it before any work starts: an engine plugin's enqueue hook, a serving
 * loop with a fixed memory budget, a framework whose caching allocator must
 * stay the only one.  For them a cudaMalloc at call time is either forbidden
 * or harmful (it can synchronise the device and fragment the plan), and they
 * may have no spare buffer to hand over as a workspace.  This entry point
 * takes no workspace: its scratch is one array of
 * FP_SELECT_NOALLOC_SCRATCH_BYTES compiled into libfp.so, which every GPU
 * that loads the library holds until the process exits.
 * The paper has no counterpart to this call; it computes exactly what
 * fp_select computes, with the same arguments minus the workspace.
 *   * The scratch needed is fp_workspace_size(shape, FP_CALL_SELECT); a
 *     problem needing more than FP_SELECT_NOALLOC_SCRATCH_BYTES is rejected
 *     with FP_ERR_WORKSPACE before anything is launched.
 *   * It allocates nothing (no cudaMalloc / cudaFree / allocating library
 *     routine).  The first call on a device looks up the array's device
 *     address for that device (cudaGetSymbolAddress) and keeps it for the
 *     life of the process; make that first call before capturing any
 *     stream.  A cudaDeviceReset() ends the context that address belongs
 *     to, so do not call this entry point on a device after resetting it.
 *   * Every call on a device uses the same array, which keeps the last
 *     call's contents; each call first clears the histograms, counters and
 *     flags it accumulates into, so no call depends on the one before it.
 *     Two calls whose work can overlap on the GPU (different streams,
 *     several host threads) race on it: the caller must order them.
 */
#define FP_SELECT_NOALLOC_SCRATCH_BYTES (4u << 20)
fp_status fp_select_noalloc(const fp_shape *shape, const fp_params *params,
                            const int32_t *pattern, const float *map,
                            const float *vert, const float *slash,
                            int32_t *counts, int32_t *indices,
                            fp_stream_t stream);

/*
 * fp_sparse_attn -- causal block-sparse attention over the given lists.
 * Source: atlas.scime.ai summary, "Approach" and "Experimental setup" (the
 * sparse kernel builds on FlashAttention).
 * Row block i of head h attends to the keys of blocks indices[b,h,i,0..
 * counts-1] (each 0 <= j <= i; inside block i only keys <= the query), with
 * softmax(q.k / sqrt(d)) V in fp32 accumulation.
 *   out [Bt,Hq,N,d] (dtype of q); lse [Bt,Hq,N] fp32, natural-log
 *   log-sum-exp of the scaled logits, or NULL.
 * A row with counts == 0 gets zeros and lse = -inf.
 * Workspace: fp_workspace_size(shape, FP_CALL_SPARSE_ATTN).
 */
fp_status fp_sparse_attn(const fp_shape *shape, const void *q, const void *k,
                         const void *v, const int32_t *counts,
                         const int32_t *indices, void *out, float *lse,
                         void *ws, size_t ws_bytes, fp_stream_t stream);

/*
 * fp_dense_attn -- dense causal attention (every block j <= i), the same
 * kernels as fp_sparse_attn; the comparison point for the speedup ("full
 * attention" in the summary's "Key results").  No workspace.
 */
fp_status fp_dense_attn(const fp_shape *shape, const void *q, const void *k,
                        const void *v, void *out, float *lse,
                        fp_stream_t stream);

/*
 * fp_prefill_attn -- the whole path for one layer: estimate, pattern,
 * select, sparse attention, with every intermediate in `ws`
 * (fp_workspace_size(shape, FP_CALL_PREFILL) bytes).  out/lse as in
 * fp_sparse_attn.  `stats` (device int64[2], or NULL) is overwritten on
 * `stream` with {kept blocks summed over every head and row, number of
 * query-aware heads}.
 */
fp_status fp_prefill_attn(const fp_shape *shape, const fp_params *params,
                          const void *q, const void *k, const void *v,
                          void *out, float *lse, int64_t *stats,
                          void *ws, size_t ws_bytes, fp_stream_t stream);

/*
 * fp_prefill_attn_varlen -- fp_prefill_attn over a batch of sequences of
 * different lengths (no counterpart in the pages: the method is defined per
 * sequence; this is the batching a serving caller needs).
 *   shape     batch must be 1 and seq_len the longest allowed length N_max;
 *             the other fields as for fp_prefill_attn
 *   n_seqs    number of sequences, >= 1
 *   seq_lens  HOST int32[n_seqs]: N_s, each in 1 .. N_max (any length)
 *   q, out    the sequences' [Hq, N_s, d] tensors back to back (sequence s
 *             starts Hq * d * (N_0 + ... + N_{s-1}) elements in);
 *   k, v      likewise [Hkv, N_s, d]
 *   lse       NULL, or [Hq, N_s] fp32 back to back
 *   stats     NULL, or device int64[n_seqs][2], per sequence as for
 *             fp_prefill_attn
 *   ws        fp_workspace_size(shape, FP_CALL_PREFILL) bytes, reused by the
 *             sequences one after another on `stream`
 * Every sequence's result is bitwise that of its own fp_prefill_attn call.
 * A bad length returns FP_ERR_SHAPE before anything is launched.
 */
fp_status fp_prefill_attn_varlen(const fp_shape *shape, const fp_params *params,
                                 int n_seqs, const int32_t *seq_lens,
                                 const void *q, const void *k, const void *v,
                                 void *out, float *lse, int64_t *stats,
                                 void *ws, size_t ws_bytes, fp_stream_t stream);

/*
 * fp_prefill_attn_host -- fp_prefill_attn on HOST buffers: copies q, k, v
 * to device memory inside `ws` (fp_workspace_size(shape,
 * FP_CALL_PREFILL_HOST) bytes), runs the path and copies the output back to
 * out_host.  Every stage is independent per query head, so the call runs as
 * units of consecutive heads of one batch entry (one query head in the first
 * and in the last unit, whose copies cannot be hidden; the rest of the first
 * and last kv heads' query heads next to them; the kv heads between in three
 * middle units): the inputs of a unit are copied in (one cudaMemcpyAsync per
 * buffer slice; a kv head's K and V with its first unit) while the previous
 * unit computes, and each unit's output is copied out while the next one
 * computes.  Units compute alternately on `stream` and on a compute stream of
 * the library's own, each with its own part of `ws`.  The copies run on two
 * more library streams; the library's streams are created once per device on
 * first use and kept until the process exits; `stream` forks to them and
 * joins them through events, so work enqueued on `stream` after this call
 * sees the finished output.
 * Page-locked host memory makes the copies asynchronous and lets them
 * overlap.  The host buffers must stay valid until `stream` reaches the end
 * of the call.  The result is bitwise that of fp_prefill_attn.
 */
fp_status fp_prefill_attn_host(const fp_shape *shape, const fp_params *params,
                               const void *q_host, const void *k_host,
                               const void *v_host, void *out_host,
                               void *ws, size_t ws_bytes, fp_stream_t stream);

/*
 * fp_last_device_status -- synchronises `stream`, returns the first error
 * the kernels recorded on the current device since the last call (FP_OK if
 * none) and clears it.
 */
fp_status fp_last_device_status(fp_stream_t stream);

/*
 * fp_selftest_watchdog -- exercises the failure detection every pipelined
 * kernel here relies on: one thread waits, with the same bounded wait the
 * kernels use, on an mbarrier that nothing ever arrives at, gives up after
 * limit_us microseconds (1 .. 1000000) and records FP_ERR_TIMEOUT in the
 * device status word, which fp_last_device_status() then returns.  The
 * device stays usable.  No counterpart in the pages (an engineering check).
 */
fp_status fp_selftest_watchdog(unsigned int limit_us, fp_stream_t stream);

/* Static, human-readable name of a status code. */
const char *fp_status_string(fp_status status);

#ifdef __cplusplus
}
#endif

#endif /* FP_H_ */
