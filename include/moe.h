/*
 * moe.h -- C ABI of libmoe_b200.so: one Mixture-of-Experts layer on one B200.
 *
 * The layer follows the tutorial page "Expert Parallelism" (learning-materials,
 * inference engineering IX.05):
 *   §1 "What is it?"        each layer has E expert FFNs; each token is routed
 *                           to k of them; experts are placed on GPUs in
 *                           contiguous blocks (GPU 0 holds experts 0-15, ...).
 *   §4 "The All-to-All"     DISPATCH: sort tokens by destination expert (and so
 *                           by destination GPU), count per GPU, exchange, so each
 *                           GPU holds a contiguous set of tokens per expert.
 *                           COMPUTE: one grouped GEMM over all experts.
 *                           COMBINE: results back in the original order and a
 *                           weighted sum of each token's k expert outputs.
 *   §5 "Load imbalance"     the imbalance of the most loaded GPU against the
 *                           ideal (max / mean), worked example 140/64.
 * On this one GPU the "GPUs" of the page are R logical expert-parallel ranks:
 * rank r owns experts [r*E/R, (r+1)*E/R). Nothing crosses a GPU boundary; the
 * exchange becomes the rank-major row layout of the permuted buffer.
 *
 * Conventions for every entry point
 *  - All tensor pointers are DEVICE pointers, row-major and contiguous, owned
 *    by the caller. bf16 tensors are passed as uint16_t bit patterns
 *    (moe_bf16_t). bf16 tensors must be 16-byte aligned.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream). Every call
 *    is asynchronous on that stream, except moe_get_status which synchronises it.
 *  - `ws` is a caller-owned device workspace of at least moe_workspace_bytes()
 *    bytes, 256-byte aligned. Its first 256 bytes hold the device status word
 *    and the counters the kernels use across CTAs (each kernel leaves its
 *    counters at zero when it finishes); clear them once with moe_clear_status
 *    (or allocate the workspace zeroed) before first use. The library
 *    allocates nothing and keeps no per-call state outside `ws`.
 *  - Shapes are validated on the host before anything is launched; an invalid
 *    argument returns MOE_ERR_INVALID_ARG (or MOE_ERR_UNSUPPORTED for a shape
 *    the kernels do not tile) and launches nothing.
 *  - Data-dependent problems found on the device (a NaN logit, an expert index
 *    out of range, a bounded wait that ran out) never trap: they OR bits into
 *    the status word (MOE_DEV_*), read with moe_get_status.
 *  - Calls that share a workspace must be ordered on one stream.
 *
 * Supported shapes: 0 <= T, T*k <= 2^27; 1 <= E <= 256; 1 <= k <= min(E, 8);
 * 1 <= R, E % R == 0; d % 128 == 0 and f % 128 == 0 (128 <= d, f <= 65536);
 * n_shared in {0, 1}; capacity >= 0.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16_t; /* bfloat16 bit pattern */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, bad shape, misaligned buffer */
  MOE_ERR_UNSUPPORTED = 2, /* shape outside what the kernels tile (see above) */
  MOE_ERR_WORKSPACE = 3,   /* ws too small or misaligned */
  MOE_ERR_CUDA = 4         /* a CUDA runtime call or launch failed */
} moe_status_t;

/* device status bits (OR-ed by kernels into the workspace status word) */
#define MOE_DEV_NAN_LOGIT 1u      /* a NaN router logit (ordered as -inf) */
#define MOE_DEV_BOUNDS 2u         /* an expert index or row index out of range (entry skipped) */
#define MOE_DEV_TIMEOUT 4u        /* a bounded pipeline wait ran out; the kernel returned early */
#define MOE_DEV_COUNT_MISMATCH 8u /* expert_offsets inconsistent with the shape */

typedef struct moe_shape {
  int32_t T;        /* tokens in the batch */
  int32_t d;        /* model width (expert input/output size) */
  int32_t E;        /* routed experts */
  int32_t k;        /* experts per token (top-k) */
  int32_t f;        /* expert FFN width (SwiGLU hidden size) */
  int32_t R;        /* logical expert-parallel ranks */
  int32_t n_shared; /* shared experts applied to every token: 0 or 1 */
  int32_t capacity; /* per-expert limit on assignments, 0 = none (see moe_dispatch) */
} moe_shape_t;

/* Bytes of workspace the entry points need for `shape` (0 if the shape is invalid). */
size_t moe_workspace_bytes(const moe_shape_t* shape);

/* Zero the 256-byte header of `ws` (status word and internal counters),
 * asynchronously on `stream`. Call once on a new workspace before first use. */
moe_status_t moe_clear_status(void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream`, then copy the device status word (MOE_DEV_* bits) to *bits.
 * The word is left as it is (clear it with moe_clear_status). */
moe_status_t moe_get_status(const void* ws, size_t ws_bytes, uint32_t* bits, void* stream);

/* Router: top-k selection and gates.
 * Page "Expert Parallelism" §1 (each token is routed to k of E experts) and §4
 * (the router's output: the experts each token goes to).
 *   logits    [T, E] fp32 in
 *   topk_idx  [T, k] int32 out: the k experts with the largest logits, in
 *             descending logit order; equal logits go to the lower expert index
 *             (-0.0 == +0.0); a NaN logit orders as -inf and sets MOE_DEV_NAN_LOGIT.
 *   topk_gate [T, k] fp32 out: softmax over the k selected logits,
 *             g_j = exp(l_j - l_0) / sum_i exp(l_i - l_0) (1/k if l_0 = -inf). */
moe_status_t moe_route(const moe_shape_t* shape, const float* logits, int32_t* topk_idx, float* topk_gate,
                       void* ws, size_t ws_bytes, void* stream);

/* Dispatch: per-expert histogram, exclusive scan and stable permute.
 * Page "Expert Parallelism" §4 DISPATCH steps 1-4 and §5 (max/mean imbalance).
 * Assignment a = t*k + j (token t, choice j) goes to expert e = topk_idx[a].
 *   x              [T, d] bf16 in
 *   topk_idx       [T, k] int32 in (values in [0, E); others set MOE_DEV_BOUNDS and are skipped)
 *   expert_counts  [E]   int32 out: assignments per expert
 *   expert_offsets [E+1] int32 out: exclusive scan of expert_counts, [E] = total
 *   rank_counts    [R]   int32 out: assignments per logical rank
 *   rank_offsets   [R+1] int32 out: expert_offsets[r*E/R]
 *   row_src        [T*k] int32 out: permuted row p holds assignment row_src[p]
 *   assign_row     [T*k] int32 out: inverse, assignment a sits at row assign_row[a]
 *   x_perm         [T*k, d] bf16 out: x_perm[assign_row[a]] = x[a / k]; rows are
 *                  expert-contiguous (expert e at [off[e], off[e+1])), so rank-major;
 *                  inside an expert, rows keep assignment order (stable).
 *                  May be NULL (x may then be NULL too): indices only, no row copies,
 *                  for moe_expert_gate_up_gather.
 *   imbalance      [2] fp32 out: [0] = max_r rank_counts[r] / mean (= *R / total),
 *                  [1] = max_e expert_counts[e] / mean; {1, 1} when nothing is placed.
 * Capacity (page §5 "Mitigations", capacity factor): with shape->capacity = c > 0
 * an expert keeps only its first c assignments in assignment order; the others
 * are dropped: assign_row = -1, no row, nothing added by moe_combine (a dropped
 * assignment bypasses its expert, so the token keeps only its residual path
 * outside this layer). Counts, offsets, ranks and imbalance then describe the
 * kept rows; T*k - expert_offsets[E] assignments were dropped.
 * moe_capacity_for gives c for the page's capacity factor C. */
moe_status_t moe_dispatch(const moe_shape_t* shape, const moe_bf16_t* x, const int32_t* topk_idx,
                          int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_counts,
                          int32_t* rank_offsets, int32_t* row_src, int32_t* assign_row, moe_bf16_t* x_perm,
                          float* imbalance, void* ws, size_t ws_bytes, void* stream);

/* Per-expert capacity of the capacity factor C = c_num / c_den (page "Expert
 * Parallelism" §5 "Mitigations": an expert accepts at most C times the tokens an
 * even split would give it). With k choices per token the even split is T*k/E
 * assignments, so the capacity is ceil(c_num * T * k / (c_den * E)), computed in
 * exact integer arithmetic (no rounding of C). Pass the result as
 * moe_shape_t.capacity. Returns -1 for c_num < 1, c_den < 1, T < 0, k < 1,
 * E < 1, or a capacity above INT32_MAX. */
int32_t moe_capacity_for(int64_t c_num, int64_t c_den, int32_t T, int32_t k, int32_t E);

/* moe_dispatch for callers that cannot allocate device memory. The pages have
 * no counterpart to this entry point: it exists for callers such as engine
 * plugins or serving runtimes whose device memory is planned and owned by their
 * own arena, and FFI callers with no CUDA allocator, for whom a cudaMalloc on the
 * hot path is not allowed or would synchronise the device.
 * Same kernels, arguments (minus the workspace) and outputs as moe_dispatch,
 * including the index-only form (x_perm = NULL, and x may then be NULL). The
 * scratch the kernels need (status word, last-chunk ticket, per-chunk counts,
 * in-chunk ranks) is a fixed 1 MiB array inside the library, held on every GPU
 * that loads the library until the process exits. Shapes whose scratch exceeds
 * it are rejected with MOE_ERR_UNSUPPORTED before anything runs: the need is
 * 256 + (bytes of ceil(T / floor(2048 / k)) * E int32 rounded up to 256) +
 * (bytes of T*k int32 rounded up to 256), e.g. T = 16384, k = 8, E = 256 needs
 * 590,080 bytes.
 * This entry point allocates nothing (no cudaMalloc/cudaFree). The first call in
 * a device's CUDA context looks up the array's device address
 * (cudaGetSymbolAddress) with that device current, and a call after the context
 * was re-created (cudaDeviceReset) looks it up again; make the first call on
 * each device before any stream capture. Every call zeroes the array's header
 * (status word and ticket) on `stream` before its kernels run, so a call never
 * depends on what an earlier call left. Every call shares the one array, so
 * calls whose executions overlap on the GPU (other streams, other host threads)
 * race and must be serialised by the caller.
 *   status  device pointer to one uint32 (may be NULL): receives this call's
 *           MOE_DEV_* bits (asynchronously, on `stream`). */
moe_status_t moe_dispatch_static(const moe_shape_t* shape, const moe_bf16_t* x, const int32_t* topk_idx,
                                 int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_counts,
                                 int32_t* rank_offsets, int32_t* row_src, int32_t* assign_row, moe_bf16_t* x_perm,
                                 float* imbalance, uint32_t* status, void* stream);

/* Diagnostics of moe_dispatch_static: the device address and size of its fixed
 * scratch array in the current device's context (the pages have no counterpart).
 * Allocates nothing; the address is valid until the context is destroyed. */
moe_status_t moe_dispatch_static_scratch(void** scratch, size_t* bytes);

/* Expert FFN: one grouped GEMM over all experts (tcgen05 tensor cores).
 * Page "Expert Parallelism" §4 COMPUTE (every expert multiplies its own tokens;
 * the differently sized GEMMs run as one grouped launch) and §1 (E expert FFNs);
 * the FFN is SwiGLU: y = W2_e (silu(W_gate,e x) * (W_up,e x)), silu(a) = a / (1 + e^-a).
 *   x_perm         [T*k, d] bf16 in (from moe_dispatch)
 *   expert_offsets [E+1]    int32 in (from moe_dispatch)
 *   w13            [E, 2f, d] bf16 in: rows [0, f) = W_gate, [f, 2f) = W_up (K = d contiguous)
 *   w2             [E, d, f]  bf16 in (K = f contiguous)
 *   x              [T, d] bf16 in, used by the shared expert (may be NULL if n_shared = 0)
 *   w13s [2f, d], w2s [d, f] bf16 in: shared expert (NULL if n_shared = 0)
 *   y_perm         [T*k, d] bf16 out: row p = FFN of expert(p) applied to x_perm[p]
 *   y_shared       [T, d]   bf16 out: shared FFN of x (NULL if n_shared = 0)
 * fp32 accumulation; the hidden activation is rounded to bf16 between the GEMMs. */
moe_status_t moe_expert_ffn(const moe_shape_t* shape, const moe_bf16_t* x_perm, const int32_t* expert_offsets,
                            const moe_bf16_t* w13, const moe_bf16_t* w2, const moe_bf16_t* x,
                            const moe_bf16_t* w13s, const moe_bf16_t* w2s, moe_bf16_t* y_perm,
                            moe_bf16_t* y_shared, void* ws, size_t ws_bytes, void* stream);

/* The two halves of moe_expert_ffn, for callers that schedule or time them
 * separately; moe_expert_ffn is exactly gate_up followed by down.
 * moe_expert_gate_up: GEMM1 + SwiGLU, h = silu(x W_gate^T) * (x W_up^T), written
 *   to the workspace (each expert's rows padded to a multiple of 256).
 * moe_expert_down: GEMM2, y_perm (and y_shared) = h W2^T, reading the h rows that
 *   the preceding moe_expert_gate_up on the same workspace, shape and
 *   expert_offsets left there. Arguments as for moe_expert_ffn. */
moe_status_t moe_expert_gate_up(const moe_shape_t* shape, const moe_bf16_t* x_perm, const int32_t* expert_offsets,
                                const moe_bf16_t* w13, const moe_bf16_t* x, const moe_bf16_t* w13s, void* ws,
                                size_t ws_bytes, void* stream);
moe_status_t moe_expert_down(const moe_shape_t* shape, const int32_t* expert_offsets, const moe_bf16_t* w2,
                             const moe_bf16_t* w2s, moe_bf16_t* y_perm, moe_bf16_t* y_shared, void* ws,
                             size_t ws_bytes, void* stream);

/* moe_expert_gate_up without x_perm: GEMM1 gathers each row of its tiles from
 * x itself (row p of expert e is token row_src[p] / k), so the dispatched rows
 * never make a round trip through HBM. This is the single-GPU form of the
 * per-expert overlap (PEO) of the page "Balancing and Beyond: Communication-
 * Centric Optimizations in Expert Parallelism" (key idea): no exchange buffer
 * is materialised before expert compute.
 *   x [T, d] bf16 in, row_src [T*k] int32 in (from moe_dispatch, which may be
 *   called with x_perm = NULL), other arguments as moe_expert_gate_up. Follow it
 *   with moe_expert_down as usual. h is bit-identical to moe_expert_gate_up's.
 * Returns MOE_ERR_UNSUPPORTED when T * d * 2 > 2^32 - 1 (row offsets into x are
 * kept in 32 bits). The rows are copied by one warp with 16-byte cp.async
 * instead of TMA tiles, which on B200 costs more GEMM time than the x_perm
 * round trip it saves; moe_expert_gate_up stays the default. */
moe_status_t moe_expert_gate_up_gather(const moe_shape_t* shape, const moe_bf16_t* x, const int32_t* row_src,
                                       const int32_t* expert_offsets, const moe_bf16_t* w13, const moe_bf16_t* w13s,
                                       void* ws, size_t ws_bytes, void* stream);

/* moe_expert_down with the combine folded into its epilogue: the per-expert overlap
 * of the page "Balancing and Beyond: Communication-Centric Optimizations in Expert
 * Parallelism" (key idea: compute and combine pipelined along the experts), on one
 * GPU. Each output tile, once stored, counts its rows in on their tokens' counters
 * (one per token and 64 columns); the row that completes a token's count (its kept
 * assignments, plus its shared row) sums that token's rows of those 64 columns in j
 * order, as moe_combine does: out is bit for bit moe_combine's, whatever order the
 * tiles finish in. y_perm (and y_shared) are written as by moe_expert_down.
 *   row_src, assign_row [T*k] int32 in, topk_gate [T, k] fp32 in (from dispatch and
 *   route); out [T, d] bf16 out. The counters live in the workspace; this call zeroes
 *   them first (and out, when a capacity can leave a token with no row and there is
 *   no shared expert). Other arguments as moe_expert_down. */
moe_status_t moe_expert_down_combine(const moe_shape_t* shape, const int32_t* expert_offsets, const moe_bf16_t* w2,
                                     const moe_bf16_t* w2s, const int32_t* row_src, const int32_t* assign_row,
                                     const float* topk_gate, moe_bf16_t* y_perm, moe_bf16_t* y_shared,
                                     moe_bf16_t* out, void* ws, size_t ws_bytes, void* stream);

/* Combine: un-permute and gate-weighted sum, back in original token order.
 * Page "Expert Parallelism" §4 COMBINE.
 *   out[t] = sum_{j<k} topk_gate[t,j] * y_perm[assign_row[t*k+j]] (+ y_shared[t])
 *   fp32 accumulation in j order, one bf16 rounding at the end.
 *   y_perm [T*k, d] bf16 in, assign_row [T*k] int32 in, topk_gate [T, k] fp32 in,
 *   y_shared [T, d] bf16 in (NULL: no shared term), out [T, d] bf16 out. */
moe_status_t moe_combine(const moe_shape_t* shape, const moe_bf16_t* y_perm, const int32_t* assign_row,
                         const float* topk_gate, const moe_bf16_t* y_shared, moe_bf16_t* out, void* ws,
                         size_t ws_bytes, void* stream);

/* All buffers of one layer call (device pointers; see the steps above). */
typedef struct moe_layer_buffers {
  const float* logits;       /* [T, E]  in */
  const moe_bf16_t* x;       /* [T, d]  in */
  const moe_bf16_t* w13;     /* [E, 2f, d] in */
  const moe_bf16_t* w2;      /* [E, d, f]  in */
  const moe_bf16_t* w13s;    /* [2f, d] in (NULL if n_shared = 0) */
  const moe_bf16_t* w2s;     /* [d, f]  in (NULL if n_shared = 0) */
  int32_t* topk_idx;         /* [T, k]  out */
  float* topk_gate;          /* [T, k]  out */
  int32_t* expert_counts;    /* [E]     out */
  int32_t* expert_offsets;   /* [E+1]   out */
  int32_t* rank_counts;      /* [R]     out */
  int32_t* rank_offsets;     /* [R+1]   out */
  int32_t* row_src;          /* [T*k]   out */
  int32_t* assign_row;       /* [T*k]   out */
  moe_bf16_t* x_perm;        /* [T*k, d] out; NULL: not materialised, GEMM1 gathers rows of x
                                (as moe_expert_gate_up_gather, same limit) */
  float* imbalance;          /* [2]     out */
  moe_bf16_t* y_perm;        /* [T*k, d] out */
  moe_bf16_t* y_shared;      /* [T, d]  out (NULL if n_shared = 0) */
  moe_bf16_t* out;           /* [T, d]  out */
} moe_layer_buffers_t;

/* The whole layer: route -> dispatch -> expert FFN -> combine, on one stream,
 * with no host synchronisation (the grouped GEMM reads the per-expert row
 * counts on the device). Same results as the four calls in sequence. */
moe_status_t moe_layer(const moe_shape_t* shape, const moe_layer_buffers_t* buf, void* ws, size_t ws_bytes,
                       void* stream);

/* ---- Expert parallelism across GPUs ------------------------------------------
 * Page "Expert Parallelism" §1 (experts on GPUs in contiguous blocks: rank r of R
 * owns experts [r*E/R, (r+1)*E/R)) and §4 "The All-to-All": DISPATCH counts the
 * tokens per GPU, exchanges the counts, then the token rows, so that every GPU
 * holds one contiguous run of rows per expert it owns; COMPUTE runs each GPU's
 * experts as one grouped GEMM; COMBINE returns every result to the GPU its token
 * came from, in the original order, and sums it with its gate; §4 "The
 * communication volume": k * d * 2 bytes per token and direction.
 * One process (or host thread) per GPU, R ranks, each with its own batch of T
 * tokens (shape->T), all E experts' router logits, and the weights of its own
 * E/R experts. shape->R is the number of ranks; shape->capacity, if non-zero,
 * applies to every expert's rows from all ranks together.
 * The exchanges are done by the kernels themselves over peer memory (NVLink): the
 * dispatch permute stores each row into the owning rank's receive buffer, the
 * combine loads each result row from the owning rank's output buffer, and the
 * per-expert counts are stored into every rank's count table. Each rank's receive
 * buffer then holds exactly the rows that a single-GPU moe_dispatch of the R
 * batches taken as one batch (rank after rank) places in logical rank r's slice,
 * in the same order.
 * Ranks signal each step through flags in peer memory (release and acquire at
 * system scope); a wait that runs out (moe_set_wait_timeout_ns) raises
 * MOE_DEV_TIMEOUT and returns. `epoch` numbers the layer calls, 1, 2, 3, ...,
 * the same on every rank. One layer call on rank r, all on one stream:
 *   moe_route                  (local)
 *   moe_ep_exchange_counts     histogram, counts to every rank
 *   moe_ep_dispatch            wait for all counts, plan, rows to their owners
 *   moe_ep_wait(slot 1)        every rank's rows have arrived
 *   moe_expert_ffn             on the receive buffer: shape (T = rows_cap, k = 1,
 *                              E = E/R, R = 1, d, f), expert_offsets =
 *                              recv_offsets, this rank's weights, y = its output
 *                              buffer (+ a shared expert on the local x, if any)
 *   moe_ep_signal(slot 2)      this rank's expert outputs are ready
 *   moe_ep_combine             wait for every rank's outputs, gather and sum
 *   moe_ep_wait(slot 3)        every rank has read the outputs: the buffers may
 *                              be written by the next call */
typedef struct moe_ep_peers {
  int32_t* const* counts;       /* [R] device array of device pointers: rank r's count table, int32 [R][E] */
  moe_bf16_t* const* recv_rows; /* [R] ...: rank r's receive buffer, bf16 [rows_cap][d] */
  moe_bf16_t* const* y_rows;    /* [R] ...: rank r's expert-output buffer, bf16 [rows_cap][d] */
  uint64_t* const* flags;       /* [R] ...: rank r's flags, uint64 [4][R], zero before the first call */
  int64_t rows_cap;             /* rows of every receive and output buffer; R * T * k holds any routing */
} moe_ep_peers_t;

#define MOE_EP_SLOT_COUNTS 0  /* a rank's counts are in every table */
#define MOE_EP_SLOT_ROWS 1    /* a rank's rows are in their owners' receive buffers */
#define MOE_EP_SLOT_OUTPUTS 2 /* a rank's expert outputs are ready to be read */
#define MOE_EP_SLOT_DONE 3    /* a rank has read every output it needs */

/* Per-expert histogram of this rank's topk_idx (T*k assignments, no capacity):
 * expert_counts [E] out (device); stores the row into every rank's count table and
 * signals MOE_EP_SLOT_COUNTS. ws: a workspace for `shape` (moe_workspace_bytes). */
moe_status_t moe_ep_exchange_counts(const moe_shape_t* shape, int32_t rank, uint64_t epoch, const int32_t* topk_idx,
                                    int32_t* expert_counts, const moe_ep_peers_t* peers, void* ws, size_t ws_bytes,
                                    void* stream);

/* Waits for every rank's counts, computes the plan (moe_ep_plan_host is the same
 * arithmetic on the host) and stores each row of x into its owner's receive buffer;
 * signals MOE_EP_SLOT_ROWS.
 *   send_row     [T*k] int32 out: row of assignment a in its owner's buffers (-1: dropped)
 *   recv_offsets [E/R + 1] int32 out: this rank's experts' rows in its own receive
 *                buffer, [E/R] = rows received (the expert_offsets of its expert FFN)
 * ws must be the workspace of the preceding moe_ep_exchange_counts. */
moe_status_t moe_ep_dispatch(const moe_shape_t* shape, int32_t rank, uint64_t epoch, const moe_bf16_t* x,
                             const int32_t* topk_idx, int32_t* send_row, int32_t* recv_offsets,
                             const moe_ep_peers_t* peers, void* ws, size_t ws_bytes, void* stream);

/* Store epoch into flag `slot` of this rank in every rank's flags (after this
 * stream's earlier work). */
moe_status_t moe_ep_signal(int32_t R, int32_t rank, int32_t slot, uint64_t epoch, const moe_ep_peers_t* peers,
                           void* stream);

/* Wait (bounded) on the stream until every rank's flag `slot` has reached epoch;
 * on timeout raises MOE_DEV_TIMEOUT in ws's status word. */
moe_status_t moe_ep_wait(int32_t R, int32_t rank, int32_t slot, uint64_t epoch, const moe_ep_peers_t* peers, void* ws,
                         size_t ws_bytes, void* stream);

/* Waits for every rank's expert outputs, then
 *   out[t] = sum_j topk_gate[t, j] * y_rows[owner(topk_idx[t, j])][send_row[t*k + j]] (+ y_shared[t])
 * (fp32 in j order, one bf16 rounding; a dropped assignment adds nothing), and
 * signals MOE_EP_SLOT_DONE. y_shared [T, d] may be NULL. */
moe_status_t moe_ep_combine(const moe_shape_t* shape, int32_t rank, uint64_t epoch, const int32_t* send_row,
                            const int32_t* topk_idx, const float* topk_gate, const moe_bf16_t* y_shared,
                            moe_bf16_t* out, const moe_ep_peers_t* peers, void* ws, size_t ws_bytes, void* stream);

/* The exchange plan on the host, from all ranks' counts (host int32 [R][E]):
 *   row_base[e]  first row, in the owner of e's receive buffer, of `rank`'s rows of e
 *   keep[e]      how many of `rank`'s assignments to e are kept (capacity)
 *   recv_offsets [E/R + 1] this rank's experts' rows in its receive buffer
 * Returns 0, or -1 for invalid arguments. */
int32_t moe_ep_plan_host(int32_t R, int32_t E, int32_t rank, int32_t capacity, const int32_t* counts_all,
                         int32_t* row_base, int32_t* keep, int32_t* recv_offsets);

/* Human-readable name of a status code (static string). */
const char* moe_status_string(moe_status_t status);

/* Text of the last CUDA error seen by this thread in a library call ("" if none). */
const char* moe_last_cuda_error(void);

/* Diagnostic knob: the limit, in nanoseconds, of each bounded wait inside the
 * grouped-GEMM pipeline (default 2e9; 0 restores the default). A wait that runs
 * out sets MOE_DEV_TIMEOUT; the kernel then stops issuing work, waits for its
 * copies and MMAs in flight, frees its tensor memory and returns, leaving the
 * context usable. Applies to launches made after the call, process-wide.
 * Returns the previous value. */
uint64_t moe_set_wait_timeout_ns(uint64_t ns);

/* Diagnostic knob: tile shape of the grouped GEMM for launches made after the
 * call, process-wide. Two tile shapes exist: 128 x 256 tiles of one CTA, and
 * 256 x 256 tiles computed by a cluster of two CTAs on neighbouring SMs
 * (cta_group::2; the down GEMM needs d % 256 == 0 for them), where a group's last
 * block of at most 128 rows runs as a half-height tile (128 x 256, 64 rows per
 * CTA), so both shapes pad a group to a multiple of 128 rows.
 *   0 (default) = CTA-pair tiles when the routed experts average at least 1024
 *       rows (T*k >= 1024*E), single-CTA tiles otherwise;
 *   1 = single-CTA tiles only;
 *   2 = CTA-pair tiles wherever they apply.
 * Either way the CTAs claim tiles at run time from a counter in the workspace
 * header (zero between calls). Results are the same up to fp32 summation order.
 * Returns the previous value, or -1 for an unknown policy (unchanged). */
int moe_set_gemm_policy(int policy);

/* Whole-layer knob: while enabled (non-zero), moe_layer folds the combine into the
 * down GEMM's epilogue (as moe_expert_down_combine; its dispatch zeroes the counters)
 * instead of launching moe_combine's kernel. Results are bit for bit the same.
 * Process-wide, for calls made after this one; default 0. Returns the previous value. */
int moe_set_fused_combine(int enable);

/* Kernels this library has launched in this process so far, over every entry point
 * and thread (successful launches only); the difference across a region of calls is
 * the number of the library's kernels that region put on the GPU. */
uint64_t moe_kernel_launches(void);

/* Dispatch-path knob (moe_dispatch, moe_dispatch_static and the dispatch step of
 * moe_layer; results are bit for bit the same on every path):
 *   0 (default) = one pass when T*k <= 16384, the two-kernel path otherwise;
 *   1 = two kernels: a histogram kernel whose last CTA scans the per-chunk counts,
 *       then the permute kernel;
 *   2 = one pass wherever it applies: a single kernel (one CTA per SM) in which
 *       every CTA counts all T*k expert ids itself (its reads grow with T*k), ranks
 *       its own contiguous range of assignments and copies their rows; it applies
 *       while one CTA's range holds at most 1024 assignments (about T*k / SMs plus
 *       two tokens' worth), else the two-kernel path runs.
 * The one-pass kernel needs none of the workspace's scratch besides the status
 * word; moe_layer with the combine folded into the down GEMM always takes the
 * two-kernel path. Process-wide, for calls made after this one. Returns the
 * previous value, or -1 for an unknown path (unchanged). */
int moe_set_dispatch_path(int path);

/* Launch-overlap knob: while enabled (the default, non-zero), every kernel the
 * library launches carries programmatic stream serialization (programmatic
 * dependent launch): it may be scheduled while the kernel before it in the
 * stream is still running, does only work that needs none of that kernel's
 * results, and waits for it (griddepcontrol.wait) before reading its inputs or
 * writing anything. Results are identical either way; 0 launches every kernel
 * in plain stream order. Process-wide, for launches made after the call.
 * Returns the previous value. */
int moe_set_pdl(int enable);

/* Test hook for the bounded-wait path: while enabled (non-zero), every CTA of
 * the grouped-GEMM launches made after the call arms its first pipeline stage
 * but never loads it, so the MMA's wait on that stage runs out after the
 * moe_set_wait_timeout_ns limit: MOE_DEV_TIMEOUT is set, the kernel drains its
 * real copies and MMAs, frees its tensor memory and returns; outputs are
 * incomplete. Never enable it outside tests. Returns the previous value. */
int moe_set_test_stall(int enable);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
