/*
 * flide.h -- C ABI of libflide.so: the ForkAttention hot path on one B200.
 *
 * The operations follow the pages on Flide ("tree-forked decision inference"):
 *   - a decision request is a shared prefix plus option branches, all laid out
 *     in ONE flattened token stream, with the request's logical tree held as
 *     GPU-resident indices (kongchang.com article, introduction and
 *     "ForkAttention" section);
 *   - every branch query must equal an isolated forward pass over its own
 *     ancestors, for softmax attention and for Gated DeltaNet layers
 *     (kongchang.com, "ForkAttention" section and Gated DeltaNet box); branch
 *     tokens never attend to other branches (kongchang.com, attention-mask
 *     section);
 *   - the network state is cloned at the decision point instead of being
 *     recomputed (techfi24.com, "Mécanisme d'Exact State Forking"), and growing
 *     histories resume from checkpoints saved by earlier passes
 *     (kongchang.com, "ForkAttention" section).
 *
 * Conventions shared by every call
 *   - All tensor pointers are DEVICE pointers into caller-owned memory.  The
 *     library allocates nothing and keeps no state between calls except
 *     process-wide cached function pointers.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream), launches only kernels, and reads every data-dependent
 *     size (actual node/token counts, tree depth, work counts) from device
 *     memory, so a call sequence can be captured once into a CUDA graph and
 *     replayed for any tree that fits the capacities it was captured with.
 *   - The return value reports errors detected on the host (bad arguments,
 *     unsupported shapes, launch failures).  Errors that depend on device data
 *     (malformed tree, capacity overflow) are written to the index's `status`
 *     word (first error wins); kernels that find a non-zero status do nothing.
 *     Read it after synchronising the stream.  No call aborts the process.
 *   - Host threads: calls may come from several threads at once (the cached
 *     function pointers and per-device set-up flags are atomic).  Device data
 *     that calls share (an index and its scratch, the no-alloc work array) is
 *     ordered by the caller's streams and events, as for any CUDA work.  A
 *     flide_pool is host state without a lock: one thread at a time.
 *   - Stream layout: requests in order; within a request, nodes in index order
 *     with parent[i] < i; node 0 of each request is its root (the shared
 *     prefix).  Tensors are row-major [token, head, dim].
 */
#ifndef FLIDE_H
#define FLIDE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define FLIDE_OK 0
#define FLIDE_ERR_INVALID 1  /* malformed tree: parent >= self, root with parent != -1,
                                non-root seg_len < 1, req_node_ptr not monotone   */
#define FLIDE_ERR_SHAPE 2    /* unsupported head dim / dtype, Hq % Hkv != 0, NULL arg */
#define FLIDE_ERR_CAPACITY 3 /* tree or data larger than the capacities given      */
#define FLIDE_ERR_CUDA 4     /* a CUDA runtime call or kernel launch failed        */
#define FLIDE_ERR_TIMEOUT 5  /* a bounded device-side wait expired                 */
#define FLIDE_ERR_BOUNDS 6   /* bounds-checked build only: a data-dependent index left
                                its array; the access was skipped (see flide_debug_bounds) */

/* ---- element types ----------------------------------------------------- */
#define FLIDE_F32 0
#define FLIDE_BF16 1
#define FLIDE_E4M3 2 /* 8-bit e4m3 codes (flide_fork_attn_fp8, flide_quantize_e4m3) */

/* ---- flags for flide_fork_attn / flide_fork_gdn ------------------------ */
#define FLIDE_FLAG_PORTABLE 1 /* force the portable SIMT kernels (any d, any dtype) */

typedef void *flide_stream; /* cudaStream_t */

/* Number of int32 entries in flide_tree_index.counts. */
#define FLIDE_COUNTS 16
/* counts[] slots written by flide_tree_build */
#define FLIDE_CNT_N 0          /* actual nodes  = req_node_ptr[R]              */
#define FLIDE_CNT_T 1          /* actual tokens = sum(seg_len)                 */
#define FLIDE_CNT_PAST 2       /* packed past rows = sum(past_len)             */
#define FLIDE_CNT_DEPTH 3      /* deepest level present (root = 0)             */
#define FLIDE_CNT_SLOTS 4      /* node-state slots used (roots + inner nodes)  */
#define FLIDE_CNT_BRANCH_TOK 5 /* tokens of non-root nodes                     */
#define FLIDE_CNT_ROOT_TOK 6   /* tokens of root nodes                         */
#define FLIDE_CNT_CKPT_ROWS 7  /* sum over requests of past_len + root seg_len */
#define FLIDE_CNT_CHECK_SITE 12  /* first failed device check: its site number ...   */
#define FLIDE_CNT_CHECK_VALUE 13 /* ... and the offending value (0 if none failed)   */

/*
 * Tree descriptor: the request trees of one batch (kongchang.com,
 * "ForkAttention": the logical tree of each decision request, encoded as
 * indices).  R, N, T and max_depth are CAPACITIES (host integers); the actual
 * sizes are read on the device: N_actual = req_node_ptr[R],
 * T_actual = sum(seg_len[0..N_actual)).  Requests with no nodes
 * (req_node_ptr[r] == req_node_ptr[r+1]) are allowed and act as padding.
 */
typedef struct {
  int32_t R, N, T;             /* capacities: requests, nodes, stream tokens    */
  int32_t max_depth;           /* capacity: deepest level below the root        */
  const int32_t *req_node_ptr; /* [R+1] node ranges; req_node_ptr[0] == 0      */
  const int32_t *parent;       /* [N] request-local parent, -1 for the root     */
  const int32_t *seg_len;      /* [N] tokens of each node (root may be 0)       */
  const int32_t *past_len;     /* [R] checkpointed tokens before the root       */
} flide_tree_desc;

/*
 * Device-resident tree index, carved by flide_tree_index_init from ONE
 * caller-allocated device buffer of flide_tree_index_bytes() bytes.  All
 * arrays are int32 and written by flide_tree_build:
 *   node_start[N+1]  exclusive prefix sum of seg_len (stream offset of each node)
 *   node_req[N]      request of each node
 *   depth[N]         edges from the request root
 *   anc_ptr[N+1]     CSR row pointers; row n lists n's ancestors root..n
 *   anc_node[...]    CSR entries (global node ids), N*(max_depth+1) capacity
 *   ctx_len[N]       past_len + tokens of all ancestors and the node itself
 *   token_node[T]    node of each stream token
 *   token_pos[T]     position of the token in its isolated sequence
 *                    (past_len + tokens of strict ancestors + offset in node)
 *   past_start[R+1]  exclusive prefix sum of past_len (rows of the packed past)
 *   req_node[R+1]    copy of req_node_ptr (first node = root of each request)
 *   level_ptr[max_depth+2], level_node[N]  nodes grouped by depth, ascending id
 *   state_slot[N]    slot of the node's end state in a node-state buffer, for
 *                    roots and for nodes with children; -1 for leaves
 *   ckpt_start[R+1]  exclusive prefix sum of past_len + root seg_len
 *   status[1]        first device-detected error (FLIDE_* code), 0 if none
 *   counts[FLIDE_COUNTS]  actual sizes, see FLIDE_CNT_*
 *   work[...]        per-call scratch of the layer kernels
 */
typedef struct {
  int32_t R, N, T, max_depth; /* capacities the buffer was laid out for */
  int32_t *status, *counts;
  int32_t *node_start, *node_req, *depth, *anc_ptr, *anc_node, *ctx_len;
  int32_t *token_node, *token_pos, *past_start, *req_node, *level_ptr, *level_node;
  int32_t *state_slot, *ckpt_start, *work;
  int64_t work_len; /* int32 entries available in work */
} flide_tree_index;

/* Bytes of device memory a tree index with these capacities needs (256-byte
 * aligned sub-arrays).  Returns 0 for negative capacities and for capacities
 * whose arrays would pass 2^31 - 1 entries (the kernels index them with
 * int32; the ancestor lists take N * (max_depth + 1)). */
size_t flide_tree_index_bytes(int32_t R, int32_t N, int32_t T, int32_t max_depth);

/* Lays out `idx` over `dev_buf` (device memory of at least `bytes` bytes,
 * 256-byte aligned).  Host only, no device access.  Returns FLIDE_OK,
 * FLIDE_ERR_SHAPE (NULL pointer, negative capacity, misaligned buffer) or
 * FLIDE_ERR_CAPACITY (buffer too small). */
int flide_tree_index_init(flide_tree_index *idx, void *dev_buf, size_t bytes,
                          int32_t R, int32_t N, int32_t T, int32_t max_depth);

/*
 * Tree-index build (kongchang.com, "ForkAttention": topology expressed as
 * GPU metadata).  Validates the tree and fills every array of `idx` from
 * `desc` (whose capacities must not exceed idx's).  Resets idx->status first.
 * Device-detected errors: FLIDE_ERR_INVALID, FLIDE_ERR_CAPACITY (more nodes,
 * tokens or levels than the capacities).
 */
int flide_tree_build(const flide_tree_desc *desc, flide_tree_index *idx,
                     flide_stream stream);

/*
 * Fork attention (kongchang.com, "ForkAttention" and attention-mask
 * sections): every query token attends to exactly the keys of its isolated
 * sequence -- its request's past rows, every token of its ancestors, and the
 * tokens of its own node up to and including itself:
 *     o = softmax(scale * q k^T) v   over those keys, fp32 accumulation.
 * GQA: query head h reads kv head h / (Hq/Hkv).
 *   q      [T, Hq, d]    dtype            out [T, Hq, d] dtype
 *   k, v   [T, Hkv, d]   dtype            (T = idx->T, the token capacity)
 *   past_k, past_v [past_rows, Hkv, d] dtype, packed in request order
 *          (rows of request r start at idx->past_start[r]); may be NULL (with
 *          past_rows == 0) when no request has past.  A request with past rows
 *          and NULL past pointers sets FLIDE_ERR_SHAPE in the status word.
 * dtype FLIDE_F32 or FLIDE_BF16.  With bf16, d == 128, 128 % (Hq/Hkv) == 0 and
 * idx->max_depth <= 8 the tensor-core kernel runs (tcgen05 MMA, TMA, TMEM);
 * otherwise, or with FLIDE_FLAG_PORTABLE, the portable kernel (d a multiple of
 * 32, <= 256).  FLIDE_E4M3 inputs need descale factors and go through
 * flide_fork_attn_fp8 (FLIDE_ERR_SHAPE here).
 * Uses idx->work as scratch.  Host errors: FLIDE_ERR_SHAPE, FLIDE_ERR_CUDA.
 */
int flide_fork_attn(const void *q, const void *k, const void *v,
                    const void *past_k, const void *past_v, int32_t past_rows,
                    flide_tree_index *idx, int32_t Hq, int32_t Hkv, int32_t d,
                    int32_t dtype, float scale, void *out, int32_t flags,
                    flide_stream stream);

/*
 * Fork attention over e4m3 inputs (the pages run Flide in FP8 where the
 * hardware has it: techfi24.com, "Exact State Forking" and "Performances").
 * Same keys and arguments as flide_fork_attn, with
 *   q [T, Hq, 128], k, v [T, Hkv, 128], past_k, past_v [past_rows, Hkv, 128]
 *          e4m3 codes (one byte each, as written by flide_quantize_e4m3)
 *   descale  device float[3] = {sq, sk, sv}: the values are sq*q, sk*k,
 *          sv*v; past rows use sk and sv (quantise past and new rows with one
 *          shared amax, see flide_amax)
 *   out    [T, Hq, 128] bf16
 * computes o = softmax(scale * (sq q)(sk k)^T)(sv v) with fp32 accumulation.
 * Tensor-core kernel (kind::f8f6f4) only: d == 128, 128 % (Hq/Hkv) == 0 and
 * idx->max_depth <= 8, else FLIDE_ERR_SHAPE.  The softmax weights are rounded
 * to e4m3 (relative error <= 2^-4, absolute <= 2^-16 of the row's largest
 * weight) before they multiply v; one in eight comes from a polynomial exp2
 * (relative error < 1e-4); the row sums use the unrounded weights.
 * Uses idx->work as scratch.  Host errors: FLIDE_ERR_SHAPE, FLIDE_ERR_CUDA.
 */
int flide_fork_attn_fp8(const void *q, const void *k, const void *v,
                        const void *past_k, const void *past_v, int32_t past_rows,
                        flide_tree_index *idx, int32_t Hq, int32_t Hkv, int32_t d,
                        const float *descale, float scale, void *out,
                        flide_stream stream);

/*
 * Fork attention with the past rows read in place from a block-paged history
 * pool (the pool of flide_pool_* / flide_history_*), with no packed copy:
 * request r's past rows are history rows 0 .. past_len[r]-1 (past_len as
 * given to flide_tree_build) of slot req_slot[r], history row i stored at
 * pool row block_table[req_slot[r] * max_blocks + i / block_rows] *
 * block_rows + i % block_rows.  (The pages resume from a saved prefix and
 * grow it step by step -- kongchang.com closing section; techfi24.com,
 * "Exact State Forking" -- the paged layout is this library's.)
 *   pool_k, pool_v [n_blocks * block_rows, Hkv, 128] dtype
 *   block_table    device int32 [n_slots * max_blocks]
 *   req_slot       device int32 [idx->R]; a request with past rows needs
 *                  0 <= slot < n_slots and past_len <= max_blocks * block_rows
 *   block_rows     a multiple of 128 (one key tile never spans two blocks)
 * Otherwise as flide_fork_attn (dtype FLIDE_BF16) or flide_fork_attn_fp8
 * (dtype FLIDE_E4M3, with descale; the pool holds e4m3 codes); tensor-core
 * kernel only.  Device errors: FLIDE_ERR_INVALID in idx->status for a bad
 * slot, a history longer than the slot's table or a table entry outside
 * [0, n_blocks) (block 0 is read in its place).  Host errors:
 * FLIDE_ERR_SHAPE, FLIDE_ERR_CAPACITY, FLIDE_ERR_CUDA.
 */
int flide_fork_attn_paged(const void *q, const void *k, const void *v, const void *pool_k,
                          const void *pool_v, int32_t n_blocks, int32_t block_rows,
                          const int32_t *block_table, int32_t max_blocks, const int32_t *req_slot,
                          int32_t n_slots, flide_tree_index *idx, int32_t Hq, int32_t Hkv,
                          int32_t d, int32_t dtype, const float *descale, float scale, void *out,
                          flide_stream stream);

/*
 * Gated DeltaNet fork scan over e4m3 q, k, v (the pages' FP8 mode; techfi24.com,
 * "Exact State Forking" and "Performances").  Same recurrence, tree handling,
 * states and arguments as flide_fork_gdn, with
 *   q, k [T, H, 128], v [T, H, 128]   e4m3 codes (one byte each)
 *   descale  device float[3] = {sq, sk, sv}: the values are sq*q, sk*k, sv*v
 *   out      [T, H, 128] bf16
 * Tensor-core kernel only (dk = dv = 128), else FLIDE_ERR_SHAPE.  The codes
 * are converted to bf16 exactly and the descale factors fold into products
 * the scan forms anyway, so the arithmetic is that of flide_fork_gdn on the
 * decoded values.  Uses idx->work as scratch.
 */
int flide_fork_gdn_fp8(const void *q, const void *k, const void *v, const float *descale,
                       const float *g, const float *beta, const float *state_in,
                       flide_tree_index *idx, int32_t H, int32_t dk, int32_t dv, void *out,
                       float *node_state, int32_t n_state_slots, flide_stream stream);

/*
 * Absolute maximum for per-tensor e4m3 scaling.  *amax (device float) becomes
 * max(|x_i|) over the n elements of x (FLIDE_F32 or FLIDE_BF16, 16-byte
 * aligned), or max(*amax, that) when `accumulate` is non-zero, so several
 * tensors (past and new K rows, say) can share one scale.  NaN entries are
 * ignored.  Host errors: FLIDE_ERR_SHAPE, FLIDE_ERR_CUDA.
 */
int flide_amax(const void *x, int64_t n, int32_t dtype, float *amax, int32_t accumulate,
               flide_stream stream);

/*
 * Per-tensor e4m3 quantisation: with a = *amax (device float), inv = 448 / a
 * and out[i] = e4m3(x[i] * inv), both float32 operations rounded to nearest
 * and the code rounded to nearest even, magnitudes above 448 saturating to
 * 448; *descale (device float, may be NULL) = a / 448.  a == 0 gives inv =
 * descale = 1.  x: n elements of FLIDE_F32 or FLIDE_BF16, 16-byte aligned;
 * out: n bytes, 8-byte aligned.  Host errors: FLIDE_ERR_SHAPE, FLIDE_ERR_CUDA.
 */
int flide_quantize_e4m3(const void *x, int64_t n, int32_t dtype, const float *amax,
                        uint8_t *out, float *descale, flide_stream stream);

/*
 * Fork attention without caller-provided scratch.  (No counterpart in the
 * pages: this is a library convenience, not part of the method.)
 *
 * flide_fork_attn keeps a small per-call work table in idx->work, so whoever
 * lays out the index must also reserve that scratch and let every attention
 * call write into it.  Some callers cannot: the index may have been built by
 * another component into a fixed region they may only read, or the caller may
 * run inside a framework whose device memory pool is closed to new
 * allocations, so it can neither grow the index nor allocate a scratch buffer
 * of its own.  This entry point computes exactly what flide_fork_attn computes
 * (same arguments, same kernels) but never touches idx->work and allocates
 * nothing: the work table lives in a fixed 64 KB array compiled into
 * libflide.so, present on every GPU that loads the library until the process
 * exits.
 *   - At most 16384 requests (idx->R); larger indices return
 *     FLIDE_ERR_CAPACITY before any work is queued.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture that should contain it.  The address is then
 *     kept for the life of the process: a cudaDeviceReset between calls is not
 *     supported (the kept address would belong to the destroyed context).
 *   - All calls on a device share the one array.  Each call writes every entry
 *     it reads before reading it, so nothing needs clearing between calls, but
 *     calls whose executions overlap on the GPU (for example on two streams)
 *     race on it: order them on one stream or with events.
 *   - Returns as flide_fork_attn; device-detected errors go to idx->status.
 */
int flide_fork_attn_noalloc(const void *q, const void *k, const void *v,
                            const void *past_k, const void *past_v, int32_t past_rows,
                            const flide_tree_index *idx, int32_t Hq, int32_t Hkv,
                            int32_t d, int32_t dtype, float scale, void *out,
                            int32_t flags, flide_stream stream);

/*
 * Gated DeltaNet fork scan (kongchang.com, Gated DeltaNet box: each
 * branch evolves its own recurrent state in isolation order; techfi24.com:
 * the state is cloned at the decision point, not recomputed).  Per head, with
 * state S (dv x dk, fp32) and alpha = exp(g):
 *     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     o_t = S_t q_t.
 * The root of request r starts from state_in[r] (zeros if state_in is NULL);
 * every other node starts from its parent's end state.  The end state of every
 * node with a slot (roots and inner nodes) is written to
 * node_state[idx->state_slot[n]]; the root's is the request's checkpoint.
 *   q, k [T, H, dk] dtype;  v [T, H, dv] dtype;  g, beta [T, H] fp32
 *   state_in [R, H, dv, dk] fp32 or NULL
 *   out [T, H, dv] dtype
 *   node_state [n_state_slots, H, dv, dk] fp32 (required)
 * Device error FLIDE_ERR_CAPACITY if the tree needs more than n_state_slots.
 * Supported: dk in {32, 64, 128, 256}, dv a multiple of 32; bf16 with
 * dk = dv = 128 runs on the tensor cores.  FLIDE_E4M3 inputs go through
 * flide_fork_gdn_fp8 (FLIDE_ERR_SHAPE here).
 */
int flide_fork_gdn(const void *q, const void *k, const void *v,
                   const float *g, const float *beta, const float *state_in,
                   flide_tree_index *idx, int32_t H, int32_t dk, int32_t dv,
                   int32_t dtype, void *out, float *node_state,
                   int32_t n_state_slots, int32_t flags, flide_stream stream);

/*
 * Checkpoint save (kongchang.com, "ForkAttention": growing agent histories
 * resume from checkpoints saved in earlier passes).  For every request r the
 * shared prefix becomes history: rows [ckpt_start[r], ckpt_start[r+1]) of
 * ckpt_k/ckpt_v receive the request's past rows followed by its root rows, and
 * ckpt_S[r] receives the root's end state node_state[state_slot[root]] (zeros
 * for a request without nodes).  A later batch passes ckpt_k/ckpt_v as its
 * past_k/past_v and past_len[r] = ckpt_start[r+1] - ckpt_start[r].
 *   k, v   [T, Hkv, d] dtype         past_k, past_v as in flide_fork_attn
 *   node_state as written by flide_fork_gdn (may be NULL with H == 0)
 *   ckpt_k, ckpt_v [ckpt_rows, Hkv, d] dtype;  ckpt_S [R, H, dv, dk] fp32
 * Device error FLIDE_ERR_CAPACITY if the checkpoint needs more than ckpt_rows.
 */
int flide_state_save(const flide_tree_index *idx, const void *k, const void *v,
                     const void *past_k, const void *past_v, int32_t Hkv,
                     int32_t d, int32_t dtype, const float *node_state,
                     int32_t H, int32_t dk, int32_t dv, void *ckpt_k,
                     void *ckpt_v, float *ckpt_S, int32_t ckpt_rows,
                     flide_stream stream);

/*
 * Checkpoint resume: gathers saved checkpoints into the past inputs of a
 * new batch.  Request r of the new batch resumes checkpoint src_req[r] of a
 * saved set (src_req[r] < 0: a fresh request with no past).  Writes
 * past_len[r] (int32, the new tree's past lengths), the packed
 * past_k/past_v rows (request order) and state_in[r] (zeros when fresh).
 *   src_ckpt_start [src_R+1] int32 (the saved index's ckpt_start)
 *   src_k, src_v [*, Hkv, d] dtype; src_S [src_R, H, dv, dk] fp32
 *   src_req [R] int32 (device)
 *   past_k, past_v [past_rows, Hkv, d]; state_in [R, H, dv, dk] fp32
 * Writes FLIDE_ERR_CAPACITY / FLIDE_ERR_INVALID to *status (device int32) if
 * the rows exceed past_rows or src_req is out of range.  R <= 4096 (host
 * error FLIDE_ERR_CAPACITY beyond); host error FLIDE_ERR_SHAPE for NULL
 * arrays, an unsupported dtype or K/V rows not a multiple of 16 bytes.
 */
int flide_state_resume(int32_t R, const int32_t *src_req, int32_t src_R,
                       const int32_t *src_ckpt_start, const void *src_k,
                       const void *src_v, const float *src_S, int32_t Hkv,
                       int32_t d, int32_t dtype, int32_t H, int32_t dk,
                       int32_t dv, int32_t *past_len, void *past_k,
                       void *past_v, int32_t past_rows, float *state_in,
                       int32_t *status, flide_stream stream);

/* ---- decision scoring (next step after the layers) -------------------------
 * Decision models answer with probabilities over a few candidate options
 * (openai-hub.com news article on the Flide release, paragraphs on Jev-like
 * decision models); engines are compared by total variation distance to a
 * high-precision reference (kongchang.com article on Flide, "total variation
 * distance" box).  Reading used: each leaf of a request's tree is an option
 * scored by the log-likelihood of its path's branch tokens under an LM head,
 * and the decision is the softmax over the request's leaves.
 *
 * Bytes of `workspace` that flide_branch_logprob needs for a tree of up to T
 * stream tokens and a vocabulary of V (partial sums of the vocabulary split);
 * 0 when T or V is not positive. */
size_t flide_branch_logprob_workspace_bytes(int32_t T, int32_t V);

/* log p_t = h_t . w_{y_t} - logsumexp_v h_t . w_v for every branch token t
 * (tokens of non-root nodes); root tokens get NaN.
 *   h [T, D] bf16 hidden states (row t = stream token t), w_lm [V, D] bf16,
 *   targets [T] int32 in [0, V) (read for branch tokens only), logp [T] fp32 out,
 *   workspace of flide_branch_logprob_workspace_bytes(idx->T, V) bytes (device).
 * D % 64 == 0, V % 128 == 0, dtype FLIDE_BF16 (fp32 accumulation) else
 * FLIDE_ERR_SHAPE; idx built by flide_tree_build; uses idx->work.  Device errors
 * (expired waits) land in idx->status. */
int flide_branch_logprob(const void *h, const void *w_lm, const int32_t *targets,
                         const flide_tree_index *idx, int32_t D, int32_t V, int32_t dtype,
                         float *logp, void *workspace, size_t workspace_bytes,
                         flide_stream stream);

/* Per node: path_logp[n] = sum of logp over the branch tokens from the root's
 * child down to n (0 for roots); prob[n] = softmax of path_logp over the leaves
 * of n's request for leaves, 0 for other nodes.  logp [T] fp32 (from
 * flide_branch_logprob), path_logp and prob [N] fp32 out (device).  Host
 * errors: FLIDE_ERR_SHAPE for NULL arguments, FLIDE_ERR_CUDA; nothing is
 * launched for a batch without requests. */
int flide_option_probs(const flide_tree_index *idx, const float *logp, float *path_logp,
                       float *prob, flide_stream stream);

/* ---- multi-step agent history in a block-paged checkpoint pool -----------
 * (kongchang.com article on Flide, closing section: growing agent histories
 * and checkpoint reuse.)  Every request slot keeps its history's K/V rows in
 * blocks of block_rows rows drawn from a shared free list, and its latest GDN
 * state in state slot `slot` of a caller-owned state pool.  The host object
 * below only does the bookkeeping; the pool memory itself is caller-owned
 * device memory:
 *   pool_k, pool_v [n_blocks * block_rows, Hkv, d]; pool_S [max_requests, H, dv, dk] fp32.
 * The block table is [max_requests][max_blocks_per_request] int32 (-1 = none);
 * copy it (flide_pool_export) to the device before append/gather. */
typedef struct flide_pool flide_pool;

/* Host allocator; NULL on bad arguments or out of host memory. */
flide_pool *flide_pool_create(int32_t n_blocks, int32_t block_rows, int32_t max_requests,
                              int32_t max_blocks_per_request);
void flide_pool_destroy(flide_pool *pool);
/* Reserves n more rows for request `slot` (blocks are taken from the free
 * list as needed) and returns the history row where they start (its length
 * before the call); -FLIDE_ERR_CAPACITY when blocks run out or the request's
 * table is full, -FLIDE_ERR_INVALID for a bad slot.  Nothing changes on error. */
int64_t flide_pool_append(flide_pool *pool, int32_t slot, int32_t n);
/* One step's appends, all or nothing: for i < n, request slots[i] gains
 * counts[i] rows (slots[i] = -1: skipped, starts[i] = -1) and starts[i]
 * receives the history row where they start.  A request listed more than once
 * gets its appends in list order.  The whole batch is checked first, so on
 * error no request changes: FLIDE_ERR_CAPACITY when the blocks or a request's
 * table would run out (or a length would pass INT32_MAX), FLIDE_ERR_INVALID
 * for a slot >= max_requests or a negative count, FLIDE_ERR_SHAPE for NULL
 * arrays with n > 0.  Host arrays. */
int flide_pool_append_batch(flide_pool *pool, int32_t n, const int32_t *slots,
                            const int32_t *counts, int32_t *starts);
/* Returns all blocks of request `slot` to the free list; its length becomes 0.
 * FLIDE_ERR_INVALID for a bad slot. */
int flide_pool_release(flide_pool *pool, int32_t slot);
/* History rows held by `slot`; -FLIDE_ERR_INVALID for a bad slot. */
int32_t flide_pool_length(const flide_pool *pool, int32_t slot);
/* Blocks on the free list (0 for a NULL pool). */
int32_t flide_pool_free_blocks(const flide_pool *pool);
/* Copies the block table [max_requests * max_blocks_per_request] and the
 * lengths [max_requests] into caller-owned host arrays of those sizes.
 * FLIDE_ERR_SHAPE for NULL arguments. */
int flide_pool_export(const flide_pool *pool, int32_t *table, int32_t *lengths);

/* After a step: request r of the batch (req_slot[r] >= 0) writes its root's
 * tokens (stream rows of its root node, k/v [T, Hkv, d]) to history rows
 * [start[r], start[r] + root length) of its slot through the block table, and
 * its root's end state node_state[state_slot[root]] to pool_S[req_slot[r]]
 * (when node_state and pool_S are given).  start[r] is what flide_pool_append
 * returned (or flide_pool_append_batch wrote).  A row without a block sets
 * FLIDE_ERR_CAPACITY in idx->status.  Each slot at most once per call: two
 * requests of one call writing the same slot's state would race.
 * All arrays are device memory; row bytes (Hkv d element size) % 16 == 0. */
int flide_history_append(const flide_tree_index *idx, const int32_t *req_slot,
                         const int32_t *start, const int32_t *table, int32_t max_blocks,
                         int32_t block_rows, const void *k, const void *v, void *pool_k,
                         void *pool_v, int32_t Hkv, int32_t d, int32_t dtype,
                         const float *node_state, int32_t H, int32_t dk, int32_t dv,
                         float *pool_S, flide_stream stream);

/* Before a step: for the batch's R requests (req_slot[r] = pool slot, or -1 for
 * a request with no history) writes past_len[r] = hist_len[slot], the
 * histories' rows packed in request order into past_k/past_v [past_rows, Hkv, d]
 * and state_in[r] = pool_S[slot] (zeros for -1) when state_in is given.
 * With past_k = past_v = NULL and past_rows = 0 only past_len (and state_in)
 * are written: the lengths flide_tree_build needs before flide_fork_attn_paged
 * reads the rows in place.  dtype FLIDE_F32, FLIDE_BF16 or FLIDE_E4M3 (rows
 * are copied as bytes).
 * Device errors to *status: FLIDE_ERR_CAPACITY when the rows exceed
 * past_rows, FLIDE_ERR_INVALID for a slot >= max_requests or a row without a
 * block.  R <= 4096. */
int flide_history_gather(int32_t R, const int32_t *req_slot, int32_t max_requests,
                         const int32_t *hist_len, const int32_t *table, int32_t max_blocks,
                         int32_t block_rows, const void *pool_k, const void *pool_v, int32_t Hkv,
                         int32_t d, int32_t dtype, const float *pool_S, int32_t H, int32_t dk,
                         int32_t dv, int32_t *past_len, void *past_k, void *past_v,
                         int32_t past_rows, float *state_in, int32_t *status, flide_stream stream);

/* ---- memory-bounded GDN scheduling ---------------------------------------
 * Memory for cloned states is what limits how many options one call can hold
 * (techfi24.com, "Limites et perspectives").  Fork = isolation lets each
 * request's tree be cut below its root: the roots run once and keep their end
 * states, then whole level-1 subtrees run in groups, each group a batch of its
 * own whose zero-token roots resume from the kept states (the Python layer's
 * schedule.fork_gdn_bounded drives these calls).
 *
 * Host planner.  req_node_ptr [R+1], parent [N] (request-local, -1 for a
 * root) are HOST arrays.  Writes node_group[n] = -1 for roots, else the group
 * of n's level-1 ancestor's subtree; groups hold whole subtrees in stream
 * order, packed greedily so that each group's batch needs at most max_slots
 * node-state slots (one per request root in the group, plus its widest odd and
 * widest even depth's inner nodes, as flide_tree_build assigns them).  Returns
 * FLIDE_ERR_CAPACITY if one subtree alone needs more (or host memory runs
 * out), FLIDE_ERR_INVALID for a malformed tree (req_node_ptr not starting at
 * 0 or not monotone, a bad parent), FLIDE_ERR_SHAPE for bad arguments. */
int flide_plan_state_groups(int32_t R, const int32_t *req_node_ptr, const int32_t *parent,
                            int32_t max_slots, int32_t *node_group, int32_t *n_groups);

/* Host query: the node-state slots flide_tree_build will assign to this batch
 * (what it writes to counts[FLIDE_CNT_SLOTS]), for sizing the node_state
 * buffer of flide_fork_gdn before any device work.  One slot per non-empty
 * request's root (its end state is the request's checkpoint), plus the
 * largest number of inner nodes (nodes with children) at any odd depth and at
 * any even depth >= 2: depth L's inner nodes share their region with depth
 * L + 2, which the scan writes only after depth L + 1 has read them
 * (techfi24.com, "Limites et perspectives": memory for cloned states is the
 * limit).  req_node_ptr [R+1] and parent [N] are HOST arrays laid out as in
 * flide_tree_desc.  Writes *slots and returns FLIDE_OK, FLIDE_ERR_INVALID for
 * a malformed tree (req_node_ptr not starting at 0 or not monotone, a bad
 * parent), FLIDE_ERR_SHAPE for a NULL argument or R < 0, FLIDE_ERR_CAPACITY
 * if host memory runs out. */
int flide_tree_state_slots(int32_t R, const int32_t *req_node_ptr, const int32_t *parent,
                           int32_t *slots);

/* Device row copy: dst row dst_idx[i] <- src row src_idx[i] for i < n (a NULL
 * index array means i), rows of row_bytes bytes (a multiple of 4; pointers
 * 4-byte aligned, 16-byte words when rows and pointers allow).  Index arrays
 * are device int32.  Host errors: FLIDE_ERR_SHAPE, FLIDE_ERR_CUDA. */
int flide_copy_rows(void *dst, const void *src, const int32_t *dst_idx, const int32_t *src_idx,
                    int32_t n, int64_t row_bytes, flide_stream stream);

/* Diagnostic, with no counterpart in the pages: runs, in one thread on
 * `stream`, the bounded mbarrier wait that every kernel of this library uses
 * (try_wait with a suspend hint, limit checked against the global timer) on a
 * barrier in shared memory that nothing arrives at, with a limit of
 * timeout_us microseconds (1 .. 10,000,000).  On expiry it writes
 * FLIDE_ERR_TIMEOUT to *status (device int32) and returns, leaving the
 * context usable.  With arrive != 0 the thread first arrives on the barrier
 * itself, so the wait completes at once and *status is left unchanged (the
 * control case).  Returns FLIDE_ERR_SHAPE for a null status or a limit out of
 * range. */
int flide_selftest_wait_timeout(int32_t *status, int32_t timeout_us, int32_t arrive,
                                flide_stream stream);

/* Which build of the library is loaded: 1 for the bounds-checked debug build
 * (libflide_dbg.so, compiled with FLIDE_DEBUG_BOUNDS), 0 for the release build.
 * In the debug build every kernel checks the indices it takes from device data
 * (tree arrays, work tables, block tables, state slots, token rows, TMA
 * coordinates) against the array they index; a failed check skips the access
 * (a read takes entry 0 instead, a write is dropped, a tile load is moved to
 * row 0), records the check's site and value in counts[FLIDE_CNT_CHECK_SITE]
 * and counts[FLIDE_CNT_CHECK_VALUE] (first failure wins) and writes
 * FLIDE_ERR_BOUNDS to the status word -- never a trap or assert.  Both builds
 * compute the same results on valid input.  Host only, no device access. */
int32_t flide_debug_bounds(void);

/* Static message for a status code ("unknown status" for any other value);
 * never NULL, owned by the library. */
const char *flide_strerror(int32_t code);

#ifdef __cplusplus
}
#endif
#endif /* FLIDE_H */
