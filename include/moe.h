/*
 * moe.h -- C ABI of libmoe.so: the forward pass of one token-choice
 * Mixture-of-Experts FFN layer on an NVIDIA B200 (sm_100a).
 *
 * The layer (pages: "How do Mixture of Expert Models Work?", section "The
 * Math Behind MoEs"; "[Paper Club] Upcycling Large Language Models into
 * Mixture of Experts", the walk-through of the MoE layer's steps):
 *
 *     logits = x . W_g (+ bias)                  router GEMM
 *     G(x)   = Softmax(TopK(logits))             k gates, summing to one
 *     permute tokens into one block per expert, keeping at most C per expert
 *     E_e(x) = (SiLU(x W1_e) * (x W3_e)) W2_e    SwiGLU expert (or GELU)
 *     y_t    = sum_j G_tj E_{idx_tj}(x_t)        un-permute + weighted sum
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every pointer argument is a DEVICE pointer unless the name says host.
 *   The caller allocates and owns every buffer; the library never allocates
 *   or frees device memory and keeps no pointer after a call returns (a
 *   moe_pipeline handle, created and destroyed by the caller, owns copy
 *   streams, events and a few bytes of pinned host memory; a moe_graph
 *   handle holds the pointers its forward was captured with).
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream).  All work is enqueued on it; calls return without waiting for
 *   the GPU, except that moe_forward(_ex) and moe_forward_expert_choice
 *   with a non-NULL `stats`, moe_forward_host and moe_pipeline_wait wait
 *   before returning.
 * - Layouts are row-major and dense: x [T, d]; W_g [d, E]; W1, W3 [E, d, H];
 *   W2 [E, H, d]; y [T, d]; idx, gate, pos [T, k].
 * - Element types: MOE_BF16 means x, W_g, W1, W3, W2, xp, h, the expert
 *   outputs o and y are bf16; MOE_FP32 means they are fp32.  Router bias,
 *   gates, margins and affinities are always fp32 (so is every accumulation);
 *   indices and counts are int32.
 * - Limits: 1 <= k <= E <= 64, k <= 8, d % 8 == 0, H % 8 == 0, T >= 0, and
 *   at most 2^31 - 1 permuted rows (int32 row indices on the device).
 *   T == 0 is valid and does nothing.  Pointers must be 16-byte aligned.
 * - Errors: arguments are checked on the host before anything is enqueued;
 *   a bad argument returns MOE_ERR_ARG and enqueues nothing.  A failed CUDA
 *   call returns MOE_ERR_CUDA.  Kernels that wait on on-chip barriers give
 *   up after a bounded time and set a device error word, reported as
 *   MOE_ERR_DEVICE by moe_forward (when it synchronises) or readable by the
 *   caller.  Nothing aborts the process or throws across the ABI.
 *
 * Permuted layout (moe_permute -> moe_grouped_ffn -> moe_unpermute_combine)
 * -------------------------------------------------------------------------
 * Expert e's kept assignments occupy rows [offsets[e], offsets[e] +
 * kept_counts[e]) of xp/h/o, in ascending token position.  Each expert's
 * block starts on a multiple of MOE_ROW_ALIGN rows:
 *     offsets[0] = 0,  offsets[e+1] = offsets[e] + roundup(kept_counts[e], 128).
 * Rows between kept_counts[e] and the next block are padding: never read
 * into y, and their contents are unspecified.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_MAX_EXPERTS 64
#define MOE_MAX_TOPK 8
#define MOE_ROW_ALIGN 128
/* 2: the expert outputs o are in the layer dtype; moe_forward_graph_*. */
#define MOE_ABI_VERSION 2

typedef enum {
  MOE_OK = 0,
  MOE_ERR_ARG = 1,          /* invalid argument; nothing was enqueued */
  MOE_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. no sm_100 GPU) */
  MOE_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
  MOE_ERR_DEVICE = 4        /* a kernel reported an error through its error word */
} moe_status;

typedef enum { MOE_BF16 = 0, MOE_FP32 = 1 } moe_dtype;
typedef enum { MOE_SWIGLU = 0, MOE_GELU = 1 } moe_act;

/* Gate formula.  TOPK_SOFTMAX: Softmax(TopK(logits)), the k gates sum to one
 * ("The Math Behind MoEs"; Mixtral).  SOFTMAX_TOPK: the softmax over all E
 * logits read at the TopK experts, the Switch order ("[Paper Club]
 * Upcycling ...": the selected gates no longer sum to one, e.g. 0.4 and 0.2).
 * Both select the same experts. */
typedef enum { MOE_GATE_TOPK_SOFTMAX = 0, MOE_GATE_SOFTMAX_TOPK = 1 } moe_gating;

/* Which assignments a full expert keeps.  POSITION: the earliest tokens
 * ("Take a Closer Look at the MoE LLM Routing", "Drop-towards-the-End").
 * GATE: Batch Priority Routing ("Scaling Vision with Sparse Mixture of
 * Experts", "Priority Routing"): tokens reach the queues in descending order
 * of their largest gate, equal gates in position order, so the least
 * important tokens are dropped. */
typedef enum { MOE_PRIORITY_POSITION = 0, MOE_PRIORITY_GATE = 1 } moe_priority;

/* Options of the *_ex entry points; NULL means all defaults. */
typedef struct {
  int32_t gating;      /* moe_gating; default MOE_GATE_TOPK_SOFTMAX                */
  float gate_scale;    /* multiplies every gate, > 0; default 1.  E/k restores the
                          dense output scale under SOFTMAX_TOPK ("[Paper Club]
                          Upcycling ...": scale the expert output by the number
                          of experts over top-k, x4 for 8 experts and top-2)   */
  int32_t priority;    /* moe_priority; default MOE_PRIORITY_POSITION; only
                          matters when a capacity is set                       */
  int32_t reserved[5]; /* must be zero                                         */
} moe_options;

/* Filled by moe_forward when `stats` is non-NULL (after the stream drains). */
typedef struct {
  int32_t counts[MOE_MAX_EXPERTS];      /* assignments routed to each expert */
  int32_t kept_counts[MOE_MAX_EXPERTS]; /* min(counts, C)                    */
  int64_t assignments;                  /* T * k                             */
  int64_t kept;                         /* sum of kept_counts                */
  int32_t capacity;                     /* C, or -1 when dropless            */
  int32_t device_error;                 /* 0 = no kernel reported an error   */
} moe_stats;

/* Byte offsets of the intermediates inside the moe_forward workspace, so a
 * caller can read them after a forward (all 256-byte aligned). */
typedef struct {
  size_t idx;          /* int32 [T, k]   selected experts, slot order       */
  size_t gate;         /* fp32  [T, k]   Softmax(TopK) gates                */
  size_t margin;       /* fp32  [T]      k-th minus (k+1)-th largest logit  */
  size_t pos;          /* int32 [T, k]   row in xp/h/o, or -1 if dropped    */
  size_t counts;       /* int32 [E]                                         */
  size_t kept_counts;  /* int32 [E]                                         */
  size_t offsets;      /* int32 [E + 1]                                     */
  size_t dev_error;    /* int32 [1]      device error word                  */
  size_t scratch;      /* permute scratch (moe_permute_workspace_bytes)     */
  size_t xp;           /* dtype [rows, d] permuted tokens                   */
  size_t h;            /* dtype [rows, H] expert hidden activations         */
  size_t o;            /* dtype [rows, d] expert outputs                    */
  size_t total;        /* == moe_workspace_bytes(...)                       */
  int64_t rows;        /* rows of xp/h/o (moe_max_permuted_rows)            */
  size_t order;        /* int32 [T] queue order (priority routing only)     */
  size_t prio_scratch; /* sort scratch (moe_priority_workspace_bytes)       */
} moe_ws_layout;

/* Human-readable name of a status code (static string, never NULL). */
const char* moe_status_string(moe_status s);

/* MOE_ABI_VERSION of the loaded library. */
int32_t moe_abi_version(void);

/* Per-expert capacity C = ceil(cf * T * k / E), evaluated in double
 * ("How do Mixture of Expert Models Work?", "Expert Capacity").  Returns -1
 * when the layer is dropless (cf <= 0, NaN or +inf). */
int32_t moe_capacity(int32_t T, int32_t E, int32_t k, double capacity_factor);

/* Rows a permuted buffer (xp, h, o) needs for any routing of T tokens:
 * min(T*k, E*C) kept assignments plus up to 127 padding rows per expert.
 * Returns -1 on invalid sizes. */
int64_t moe_max_permuted_rows(int32_t T, int32_t E, int32_t k, double capacity_factor);

/* The same bound for an explicit capacity C (C < 0: dropless), e.g. one
 * shard of a batch under the whole batch's capacity (moe_permute_ex). */
int64_t moe_rows_for_capacity(int32_t T, int32_t E, int32_t k, int32_t C);

/* Scratch bytes moe_permute needs in `ws`: the per-range expert counts,
 * 256 x E int32 whatever T is (T only has to be valid). */
size_t moe_permute_workspace_bytes(int32_t T, int32_t E);

/* Workspace bytes moe_forward needs; 0 on invalid sizes. */
size_t moe_workspace_bytes(int32_t T, int32_t d, int32_t H, int32_t E, int32_t k,
                           double capacity_factor, moe_dtype dtype, moe_act act);

/* Where each intermediate lives inside the moe_forward workspace.
 * Returns MOE_ERR_ARG on invalid sizes or a NULL `out`. */
moe_status moe_workspace_layout(int32_t T, int32_t d, int32_t H, int32_t E, int32_t k,
                                double capacity_factor, moe_dtype dtype, moe_act act,
                                moe_ws_layout* out);

/* Router GEMM + TopK + gating softmax ("The Math Behind MoEs":
 * Softmax(TopK(x . W_g)); "[Paper Club] Upcycling ...": the router is a
 * learnable matrix and the expert indices are the highest-probability
 * experts).
 *   x [T, d], Wg [d, E] (dtype); bias [E] fp32 or NULL (added to the logits
 *   before TopK and kept in the softmax).
 *   Out: idx [T, k] int32 in descending-logit order, equal logits -> lower
 *   expert first; gate [T, k] fp32 = softmax over the k selected logits;
 *   margin [T] fp32 or NULL = k-th minus (k+1)-th largest logit (+inf when
 *   k == E).  Logits are accumulated in fp32 and never stored. */
moe_status moe_route(const void* x, const void* Wg, const float* bias,
                     int32_t T, int32_t d, int32_t E, int32_t k, moe_dtype dtype,
                     int32_t* idx, float* gate, float* margin, void* stream);

/* moe_route with options (gate formula and scale); opt may be NULL. */
moe_status moe_route_ex(const void* x, const void* Wg, const float* bias,
                        int32_t T, int32_t d, int32_t E, int32_t k, moe_dtype dtype,
                        const moe_options* opt, int32_t* idx, float* gate, float* margin,
                        void* stream);

/* Permutation with optional capacity ("[Paper Club] Upcycling ...": tokens
 * that selected expert e are gathered into one matrix for e, and some are
 * dropped depending on the capacity factor; "Take a Closer Look at the MoE
 * LLM Routing", "Drop-towards-the-End": the earliest C assignments of each
 * expert, in token position, are kept).
 *   x [T, d] (dtype), idx [T, k] int32 from moe_route.
 *   capacity_factor <= 0 (or +inf) = dropless; else C = moe_capacity(...).
 *   Out: xp [xp_rows, d] (dtype) with the permuted layout above (xp_rows >=
 *   moe_max_permuted_rows); pos [T, k] int32 = row of (t, j) in xp, or -1
 *   if dropped; counts [E], kept_counts [E], offsets [E+1] int32.
 *   ws: device scratch of at least moe_permute_workspace_bytes(T, E).
 *   Deterministic: the result does not depend on scheduling.  Two kernels:
 *   per range of tokens (the streaming router's ranges), each assignment's
 *   rank among the range's earlier assignments to its expert and the
 *   range's counts; then, per range, the prefix over earlier ranges gives
 *   every assignment its place in its expert's queue, and the row copy. */
moe_status moe_permute(const void* x, const int32_t* idx, int32_t T, int32_t d,
                       int32_t E, int32_t k, double capacity_factor, moe_dtype dtype,
                       void* xp, int64_t xp_rows, int32_t* pos, int32_t* counts,
                       int32_t* kept_counts, int32_t* offsets,
                       void* ws, size_t ws_bytes, void* stream);

/* moe_permute with an explicit capacity, a queue order and earlier shards.
 *   order: queue position i is token order[i] (a permutation of 0..T-1,
 *     e.g. from moe_priority_order); NULL = token position.  Rows inside an
 *     expert block follow the queue order.
 *   prior: device int32 [E] or NULL -- assignments that earlier shards of
 *     the same batch (tokens at lower positions, held by other ranks) routed
 *     to each expert; this shard keeps at most max(0, capacity - prior[e])
 *     at expert e, so a batch split over ranks drops exactly what the whole
 *     batch would ("Drop-towards-the-End" over global position).
 *   capacity: C (e.g. moe_capacity of the whole batch), or < 0 = dropless.
 *   xp_rows >= rows for this T (moe_max_permuted_rows with the same C);
 *   ws as for moe_permute. */
moe_status moe_permute_ex(const void* x, const int32_t* idx, const int32_t* order,
                          const int32_t* prior, int32_t T, int32_t d, int32_t E, int32_t k,
                          int32_t capacity, moe_dtype dtype, void* xp, int64_t xp_rows,
                          int32_t* pos, int32_t* counts, int32_t* kept_counts, int32_t* offsets,
                          void* ws, size_t ws_bytes, void* stream);

/* Per-expert assignment counts of idx [T, k] into counts [E] (device), for
 * exchanging between ranks that hold shards of one batch (int32 sums:
 * deterministic). */
moe_status moe_expert_counts(const int32_t* idx, int32_t T, int32_t E, int32_t k, int32_t* counts,
                             void* stream);

/* prior[e] = sum of gathered[r][e] over ranks r < rank: the assignments the
 * lower-position shards routed to expert e.  gathered: device int32
 * [n_ranks][E] (the all-gathered moe_expert_counts); prior: device [E]. */
moe_status moe_rank_prefix(const int32_t* gathered, int32_t n_ranks, int32_t E, int32_t rank,
                           int32_t* prior, void* stream);

/* Batch Priority Routing order ("Scaling Vision with Sparse Mixture of
 * Experts", "Priority Routing"): order[T] = the tokens sorted by descending
 * gate[t, 0] (each token's largest gate), equal gates in ascending position
 * -- a stable, deterministic device radix sort.  gate [T, k] fp32 as from
 * moe_route.  ws: at least moe_priority_workspace_bytes(T). */
size_t moe_priority_workspace_bytes(int32_t T);
moe_status moe_priority_order(const float* gate, int32_t T, int32_t k, int32_t* order,
                              void* ws, size_t ws_bytes, void* stream);

/* moe_permute without a caller-provided scratch buffer.  The pages have no
 * counterpart to this entry point: it exists for callers that cannot
 * allocate device memory where they run the layer -- for example a serving
 * runtime that reserves all device memory for its own pool up front, or a
 * plugin that its host framework forbids from allocating inside its execute
 * call.  Arguments and results are those of moe_permute, minus ws/ws_bytes.
 *   Scratch: a fixed array of MOE_PERMUTE_STATIC_MAX_INTS int32 (1 MiB) plus
 *   512 bytes, held by every GPU that loads the library until the process
 *   exits.  A call with ceil(T / 256) * E > MOE_PERMUTE_STATIC_MAX_INTS
 *   (at E = 64: T > 1,048,576) returns MOE_ERR_ARG and enqueues nothing.
 *   Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   The first call on a device looks up the array's device address with
 *   that device current; make that first call before any stream capture.
 *   Every call uses the same array, which keeps the last call's contents
 *   (each call clears the counter that must start at zero, on its stream):
 *   calls whose work overlaps on the GPU -- different streams, or different
 *   host threads on one device -- race on it, so the caller must serialise
 *   them. */
#define MOE_PERMUTE_STATIC_MAX_INTS (1 << 18)
moe_status moe_permute_static(const void* x, const int32_t* idx, int32_t T, int32_t d,
                              int32_t E, int32_t k, double capacity_factor, moe_dtype dtype,
                              void* xp, int64_t xp_rows, int32_t* pos, int32_t* counts,
                              int32_t* kept_counts, int32_t* offsets, void* stream);

/* Grouped expert FFN over the per-expert blocks ("[Paper Club] Upcycling
 * ...": one grouped GEMM over any number of experts and tokens instead of a
 * loop over experts; Mixtral's SwiGLU expert in "The Math Behind MoEs").
 *   xp [rows, d] (dtype), offsets [E+1], kept_counts [E] as from moe_permute.
 *   W1, W3 [E, d, H] (W3 unused and may be NULL for MOE_GELU), W2 [E, H, d].
 *   Out: h [rows, H] (dtype) = SiLU(xp W1_e) * (xp W3_e)  or GELU(xp W1_e);
 *        o [rows, d] (dtype) = h W2_e.  Only kept rows are written.
 *   dev_error: int32 device word; a kernel that gives up on a bounded wait
 *   ORs a nonzero code into it (the caller zeroes it beforehand).
 *   bf16 runs on the tcgen05 tensor cores with fp32 accumulation (h is
 *   rounded to bf16 before the second GEMM, o when it is stored); fp32 runs
 *   on fp32 FMA. */
moe_status moe_grouped_ffn(const void* xp, int64_t rows, const int32_t* offsets,
                           const int32_t* kept_counts, const void* W1, const void* W3,
                           const void* W2, int32_t E, int32_t d, int32_t H, moe_act act,
                           moe_dtype dtype, void* h, void* o, int32_t* dev_error,
                           void* stream);

/* Un-permute and gate-weighted combine ("[Paper Club] Upcycling ...": the
 * tokens are put back in their original order and scaled by the router
 * probability; y = sum_i G(x)_i E_i(x)).
 *   o [rows, d] (dtype), pos [T, k], gate [T, k].
 *   Out: y [T, d] (dtype), y_t = sum over kept j, in slot order, of
 *   gate[t,j] * o[pos[t,j]], accumulated in fp32 and rounded once; a token
 *   with every slot dropped gets y_t = 0.  No atomics: deterministic. */
moe_status moe_unpermute_combine(const void* o, const int32_t* pos, const float* gate,
                                 int32_t T, int32_t d, int32_t k, moe_dtype dtype,
                                 void* y, void* stream);

/* The whole layer: moe_route -> moe_permute -> moe_grouped_ffn ->
 * moe_unpermute_combine on one stream with no host synchronisation (unless
 * `stats` is non-NULL).  ws: device workspace of at least
 * moe_workspace_bytes(...); its intermediates stay readable afterwards at
 * the offsets moe_workspace_layout reports. */
moe_status moe_forward(const void* x, const void* Wg, const float* bias,
                       const void* W1, const void* W3, const void* W2,
                       int32_t T, int32_t d, int32_t H, int32_t E, int32_t k,
                       double capacity_factor, moe_act act, moe_dtype dtype,
                       void* y, void* ws, size_t ws_bytes, moe_stats* stats,
                       void* stream);

/* moe_forward with options (gate formula and scale); opt may be NULL. */
moe_status moe_forward_ex(const void* x, const void* Wg, const float* bias,
                          const void* W1, const void* W3, const void* W2,
                          int32_t T, int32_t d, int32_t H, int32_t E, int32_t k,
                          double capacity_factor, moe_act act, moe_dtype dtype,
                          const moe_options* opt, void* y, void* ws, size_t ws_bytes,
                          moe_stats* stats, void* stream);

/* moe_forward with the tokens in HOST memory: copies x_host [T, d] to
 * x_dev, runs the layer, copies y back to y_host [T, d], and waits for the
 * stream.  x_dev and y_dev are caller-owned device buffers of T*d elements.
 * Host buffers may be pageable; pinned memory gives full PCIe bandwidth. */
moe_status moe_forward_host(const void* x_host, void* y_host, void* x_dev, void* y_dev,
                            const void* Wg, const float* bias, const void* W1,
                            const void* W3, const void* W2, int32_t T, int32_t d,
                            int32_t H, int32_t E, int32_t k, double capacity_factor,
                            moe_act act, moe_dtype dtype, void* ws, size_t ws_bytes,
                            void* stream);

/* Streaming host pipeline: consecutive batches with tokens in HOST memory,
 * each copied in, run and copied out on its own slot, so the copies of one
 * batch overlap the forward of another (copy engines in both directions run
 * beside the compute stream).  The handle owns two copy streams, events and
 * a small pinned host array for the device error words; it allocates no
 * device memory.  depth = number of slots (1 .. MOE_PIPELINE_MAX_DEPTH).
 *
 * moe_pipeline_submit enqueues, and returns without waiting:
 *   copy x_host -> x_dev (copy stream; after the slot's previous forward has
 *   finished reading x_dev), moe_forward on `stream` (after that copy and
 *   after the slot's previous copy-out has read y_dev), copy y_dev -> y_host
 *   (second copy stream); opt as moe_forward_ex (NULL = defaults).
 *   x_dev, y_dev and ws belong to the slot until
 *   moe_pipeline_wait(slot) returns; x_host must stay unchanged and y_host
 *   unread until then.  Every submit on one handle must use the same stream.
 * moe_pipeline_wait blocks the host until the slot's y_host is written and
 *   returns MOE_ERR_DEVICE if a kernel of that forward reported an error.
 * Use one handle from one host thread at a time. */
#define MOE_PIPELINE_MAX_DEPTH 4
typedef struct moe_pipeline moe_pipeline;
moe_status moe_pipeline_create(int32_t depth, moe_pipeline** out);
moe_status moe_pipeline_submit(moe_pipeline* p, int32_t slot, const void* x_host, void* y_host,
                               void* x_dev, void* y_dev, const void* Wg, const float* bias,
                               const void* W1, const void* W3, const void* W2, int32_t T,
                               int32_t d, int32_t H, int32_t E, int32_t k,
                               double capacity_factor, moe_act act, moe_dtype dtype,
                               const moe_options* opt, void* ws, size_t ws_bytes, void* stream);
moe_status moe_pipeline_wait(moe_pipeline* p, int32_t slot);
/* Waits for every slot, then releases the handle (NULL is a no-op). */
moe_status moe_pipeline_destroy(moe_pipeline* p);

/* One forward captured as a CUDA graph, for small layers whose forward is
 * shorter than the host's launch work (a handful of kernels and a memset;
 * moe_forward_graph_nodes counts them).
 * moe_forward_graph_create records moe_forward_ex with these arguments
 * (stats not available) on a private stream and instantiates it; nothing
 * runs yet.  The graph keeps the pointers it was made with: x, y, ws and the
 * weights must stay allocated while it exists, and each launch reads
 * whatever x holds when it runs.  moe_forward_graph_launch enqueues one
 * forward on `stream` (same device); moe_forward_graph_destroy releases the
 * graph (NULL is a no-op; the caller finishes its launches first).  Errors:
 * MOE_ERR_ARG for the sizes and pointers moe_forward_ex rejects, for T == 0
 * and for a NULL out; MOE_ERR_CUDA if capture or instantiation fails (the
 * stream the caller uses is not touched). */
typedef struct moe_graph moe_graph;
moe_status moe_forward_graph_create(const void* x, const void* Wg, const float* bias,
                                    const void* W1, const void* W3, const void* W2,
                                    int32_t T, int32_t d, int32_t H, int32_t E, int32_t k,
                                    double capacity_factor, moe_act act, moe_dtype dtype,
                                    const moe_options* opt, void* y, void* ws, size_t ws_bytes,
                                    moe_graph** out);
moe_status moe_forward_graph_launch(moe_graph* g, void* stream);
moe_status moe_forward_graph_destroy(moe_graph* g);
/* What one launch of the graph runs: *kernels = its kernel nodes (every one
 * a kernel of this library), *others = the rest (memsets).  Host-only, no
 * GPU work.  Errors: MOE_ERR_ARG for a NULL argument; MOE_ERR_CUDA if the
 * graph cannot be read. */
moe_status moe_forward_graph_nodes(const moe_graph* g, int32_t* kernels, int32_t* others);

/* Stage timing.  `events` points to MOE_NUM_STAGE_EVENTS cudaEvent_t
 * handles (passed as void*) created by the caller, or is NULL to stop.  The
 * next moe_forward / moe_forward_host calls on the calling host thread
 * record them on their stream: [0] before the router, [1] after the router,
 * [2] after the permutation, [3] after the up projection, [4] after the down
 * projection, [5] after the combine.  The handles are copied; the events
 * themselves stay owned by the caller and must outlive those calls. */
#define MOE_NUM_STAGE_EVENTS 6
moe_status moe_set_stage_events(void* const* events);

/* ------------------------------------------------- expert-choice routing
 * "[Paper Club] Upcycling Large Language Models into Mixture of Experts",
 * the Q&A on expert choice: the selection is reversed -- every expert takes
 * a fixed number of tokens, so a token may be processed by no expert, by
 * several, or by all.  Here the affinity of token t to expert e is the
 * router probability S[t, e] = Softmax(x_t . W_g (+ bias))_e over all E
 * experts ("How do Mixture of Expert Models Work?", "The Math Behind MoEs"),
 * stored expert-major (scores[e * T + t] = S[t, e]);
 * expert e takes the n = min(C, T) tokens with the largest S[:, e]
 * (C = moe_capacity(T, E, k, cf), k read as the average number of experts
 * per token; equal affinities -> lower position first), and
 *   y_t = sum over the experts e that took t, ascending e, of S[t, e] * E_e(x_t)
 * with no renormalisation (a token no expert took gets y_t = 0).
 * Expert e's rows in xp/h/o are [e * npad, e * npad + n), its tokens in
 * ascending position; npad = n rounded up to 128. */

/* n = min(T, moe_capacity(T, E, k, cf)); -1 when cf is not a finite
 * positive number (expert choice has no dropless form) or sizes are invalid. */
int32_t moe_expert_choice_tokens(int32_t T, int32_t E, int32_t k, double capacity_factor);

/* scores [E, T] fp32 (device, expert-major: scores[e * T + t]) = softmax
 * over all E logits of token t.  Sizes as moe_route (no k). */
moe_status moe_expert_choice_route(const void* x, const void* Wg, const float* bias, int32_t T,
                                   int32_t d, int32_t E, moe_dtype dtype, float* scores,
                                   void* stream);

/* Scratch bytes for moe_expert_choice_select (expert-major positions, T*E*4). */
size_t moe_expert_choice_select_workspace_bytes(int32_t T, int32_t E);

/* Each expert's choice of n tokens (0 <= n <= T) from scores [E, T].
 * Outputs (device):
 * tok [E, n] int32 (expert e's tokens, ascending position), pos [T, E]
 * int32 (row in xp, or -1), kept_counts [E] (= n), offsets [E + 1]
 * (= e * npad).  Deterministic: the selection and the row order follow
 * from the scores alone. */
moe_status moe_expert_choice_select(const float* scores, int32_t T, int32_t E, int32_t n,
                                    int32_t* tok, int32_t* pos, int32_t* kept_counts,
                                    int32_t* offsets, void* ws, size_t ws_bytes, void* stream);

/* xp row pos[t, e] = x[t] for every pos[t, e] >= 0 (pos from
 * moe_expert_choice_select: row e * npad + r holds expert e's r-th token;
 * padding rows untouched).  Each x row is read once and written once per
 * expert that took it.  xp_rows >= E * npad. */
moe_status moe_expert_choice_permute(const void* x, const int32_t* pos, int32_t T, int32_t d,
                                     int32_t E, int32_t n, moe_dtype dtype, void* xp,
                                     int64_t xp_rows, void* stream);

/* y [T, d] (dtype) = sum over e with pos[t, e] >= 0, ascending e, of
 * scores[e, t] * o[pos[t, e]] (o (dtype) from moe_grouped_ffn), fp32
 * accumulation, one rounding.  Every y row is written. */
moe_status moe_expert_choice_combine(const void* o, const int32_t* pos, const float* scores,
                                     int32_t T, int32_t d, int32_t E, moe_dtype dtype, void* y,
                                     void* stream);

/* Byte offsets inside the moe_forward_expert_choice workspace. */
typedef struct {
  size_t scores;       /* fp32  [E, T]  affinities (expert-major)          */
  size_t pos;          /* int32 [T, E]  row in xp/h/o, or -1               */
  size_t tok;          /* int32 [E, n]  each expert's tokens               */
  size_t kept_counts;  /* int32 [E]     (= n)                              */
  size_t offsets;      /* int32 [E + 1] (= e * npad)                       */
  size_t dev_error;    /* int32 [1]     device error word                  */
  size_t scratch;      /* select scratch                                   */
  size_t xp, h, o;     /* rows x d, rows x H, rows x d (all dtype)         */
  size_t total;
  int64_t rows;        /* E * npad                                         */
  int32_t n;           /* tokens per expert                                */
} moe_ec_ws_layout;

moe_status moe_expert_choice_layout(int32_t T, int32_t d, int32_t H, int32_t E, int32_t k,
                                    double capacity_factor, moe_dtype dtype, moe_act act,
                                    moe_ec_ws_layout* layout);
/* 0 on invalid sizes (including a capacity factor that is not finite and > 0). */
size_t moe_expert_choice_workspace_bytes(int32_t T, int32_t d, int32_t H, int32_t E, int32_t k,
                                         double capacity_factor, moe_dtype dtype, moe_act act);

/* The whole layer with expert-choice routing: route (affinities) ->
 * select -> permute -> grouped expert FFNs (as moe_grouped_ffn) -> combine,
 * on one stream.  Arguments as moe_forward; k <= E (no kMaxK limit: a token
 * may be taken by any number of experts).  stats (nullable): counts =
 * kept_counts = n per expert; when given, the call waits for the stream and
 * returns MOE_ERR_DEVICE if a kernel reported an error. */
moe_status moe_forward_expert_choice(const void* x, const void* Wg, const float* bias,
                                     const void* W1, const void* W3, const void* W2, int32_t T,
                                     int32_t d, int32_t H, int32_t E, int32_t k,
                                     double capacity_factor, moe_act act, moe_dtype dtype,
                                     void* y, void* ws, size_t ws_bytes, moe_stats* stats,
                                     void* stream);

/* ------------------------------------------------------ measurement aid
 * No counterpart on the pages: a yardstick for the HBM-bound stages.  Reads
 * `bytes` of the device buffer `buf` once with streaming 16-byte loads (two
 * 512-thread CTAs per SM, each a contiguous slice, eight loads in flight per
 * thread) and XORs one word per warp into *sink (device, 4 bytes, caller
 * owned; its value means nothing).  The router reads x once and the
 * permutation and combine copy rows, so the time this takes for the same
 * number of bytes is what "as fast as a plain read" means on this GPU at
 * that size.  bytes must be a multiple of 16 and buf 16-byte aligned
 * (MOE_ERR_ARG otherwise); bytes == 0 is a no-op.  Enqueued on `stream`. */
moe_status moe_probe_stream_read(const void* buf, size_t bytes, uint32_t* sink, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
