/*
 * moba.h -- C ABI of the MoBA (Mixture of Block Attention) causal prefill
 * forward for NVIDIA B200 (sm_100a).
 *
 * What it computes.  The pages this follows are cited by title:
 *   [W] "同一天，DeepSeek和月之暗面發表了關于改進注意力機制的論文" (MoBA write-up),
 *       section "MoBA：將 MoE 原理應用于注意力機制": the context is cut into
 *       blocks; a parameter-free top-k gate routes each query token to the
 *       most relevant KV blocks; the implementation takes five steps (assign
 *       queries to blocks under the causal mask, order queries by block,
 *       attention per block, restore the order, merge with online softmax).
 *   [E] "月球計畫 AI 研究介紹混合區塊注意力 (MoBA)：一種將混合專家 (MoE) 原則應用於
 *       注意力機制的新 AI 方法", section "技術細節與優勢": the gate scores a
 *       query against an aggregated representation of each block's keys,
 *       keeps the top-scoring blocks, always includes the query's own block,
 *       and enforces a causal mask so no future position is attended.
 *
 * Readings where the pages are silent: the aggregate is the mean of the
 * block's keys; the score is the unscaled dot product; the own block counts
 * inside top-k (k - 1 past blocks + own block); equal scores go to the lower
 * block index; each query head routes on its own against its KV head's means
 * (grouped-query attention, kv head = h / (Hq / Hkv)); softmax scale 1/sqrt(d)
 * by default; lse is the natural log of the softmax denominator; blocks
 * restart at every sequence start.
 *
 * Tensor layouts (packed variable-length, row-major, no padding):
 *   q    bf16  [T, Hq,  d]      k, v  bf16 [T, Hkv, d]
 *   out  bf16  [T, Hq,  d]      lse   fp32 [T, Hq]
 *   idx  int32 [T, Hq, topk]    block indices local to the query's sequence,
 *                               ascending, padded with -1 (a query in block j
 *                               selects min(topk, j + 1) blocks; the own block
 *                               j is always the last valid entry)
 *   cu_seqlens int32 [n_seqs + 1], device memory, cu[0] = 0, non-decreasing,
 *               cu[n_seqs] = T.
 *
 * Supported: head_dim in {64, 128}; n_heads % n_kv_heads == 0;
 * block_size a multiple of 64 and <= 65536; 1 <= topk <= 64; T * Hq < 2^31.
 * q, k, v and out must be 16-byte aligned, lse and idx 4-byte aligned, the
 * workspace 256-byte aligned (any cudaMalloc / PyTorch allocation is).
 *
 * Ownership and execution: the caller owns every buffer (all device memory,
 * including the workspace); the library allocates nothing, never
 * synchronises, and enqueues all work on `stream` (a cudaStream_t; NULL is the
 * legacy default stream).  Argument errors are returned before anything is
 * enqueued.  Errors found on the device (malformed cu_seqlens, a bounded wait
 * that gave up) are written to an error word inside the workspace; they are
 * reported by moba_check(), which synchronises the stream, or by the next
 * call that uses the same workspace (which clears the word on entry, after
 * reporting nothing: call moba_check to see it).
 */
#ifndef MOBA_H_
#define MOBA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOBA_OK = 0,
  MOBA_ERR_INVALID_ARG = 1,   /* bad pointer, size, or inconsistent arguments   */
  MOBA_ERR_UNSUPPORTED = 2,   /* valid but outside the supported shapes         */
  MOBA_ERR_WORKSPACE = 3,     /* workspace NULL, misaligned or too small        */
  MOBA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed           */
  MOBA_ERR_TIMEOUT = 5,       /* a device-side bounded wait gave up             */
  MOBA_ERR_BAD_SEQLENS = 6,   /* device check: cu_seqlens malformed             */
  MOBA_ERR_BAD_SELECTION = 7, /* device check: a backward's idx row malformed   */
  MOBA_ERR_BOUNDS = 8,        /* MOBA_DEBUG build: a gathered index out of range */
  MOBA_ERR_CANARY = 9         /* MOBA_DEBUG build: a workspace guard overwritten */
} moba_status;

/* Human-readable name of a status code.  Never NULL. */
const char* moba_status_string(moba_status s);

/*
 * Bytes of device workspace that moba_gate / moba_forward need for these
 * sizes.  chunk_tokens bounds how many query tokens are processed per pass of
 * the partial-output buffer (0 = all T at once); the buffer grows linearly
 * with it (chunk_tokens * n_heads * topk * (2 * head_dim + 4) bytes).
 * Returns 0 if the arguments are invalid or unsupported.
 */
size_t moba_workspace_size(int total_tokens, int n_seqs, int n_heads, int n_kv_heads,
                           int head_dim, int block_size, int topk, int chunk_tokens);

/*
 * The gate alone ([W] step 1, [E] 技術細節與優勢): mean keys of every full block,
 * scores q . Kbar against each past block of the query's sequence, the top
 * (topk - 1) past blocks (ties to the lower index) plus the own block.
 * Writes idx [T, Hq, topk] (device).  Uses the workspace sized with the same
 * arguments and any chunk_tokens.
 */
moba_status moba_gate(const void* q, const void* k, const int32_t* cu_seqlens, int n_seqs,
                      int total_tokens, int n_heads, int n_kv_heads, int head_dim,
                      int block_size, int topk, int32_t* idx, void* workspace,
                      size_t workspace_bytes, void* stream);

/*
 * The whole forward ([W] five steps): gate, grouping of (query, head) rows by
 * selected (block, kv head), attention of every row to each selected block
 * (the own block under the token-level causal mask), and the log-sum-exp
 * merge back into the original row order.
 *   softmax_scale <= 0 selects 1/sqrt(head_dim).
 *   out [T, Hq, d] bf16 and lse [T, Hq] fp32 (natural log) are written.
 *   idx_out, if not NULL, receives the gate's selection [T, Hq, topk].
 *   chunk_tokens must not exceed the value the workspace was sized for.
 */
moba_status moba_forward(const void* q, const void* k, const void* v,
                         const int32_t* cu_seqlens, int n_seqs, int total_tokens,
                         int n_heads, int n_kv_heads, int head_dim, int block_size, int topk,
                         float softmax_scale, void* out, float* lse, int32_t* idx_out,
                         int chunk_tokens, void* workspace, size_t workspace_bytes,
                         void* stream);

/*
 * moba_forward with stage markers, for measurement.  Same arguments, plus an
 * array of n_stage_events cudaEvent_t handles (created by the caller) that
 * are recorded on `stream` at stage boundaries, in this order:
 *   [0] before the gate prefix (plan, mean-pool, gate)   [1] after it,
 *   then for every query chunk c = 0, 1, ...:
 *   [2+3c] after the scheduler  [3+3c] after the block attention (past
 *   blocks and own block)  [4+3c] after the merge.
 * Handles beyond n_stage_events, or NULL entries, are skipped.  Recording an
 * event neither allocates nor synchronises.
 */
moba_status moba_forward_traced(const void* q, const void* k, const void* v,
                                const int32_t* cu_seqlens, int n_seqs, int total_tokens,
                                int n_heads, int n_kv_heads, int head_dim, int block_size, int topk,
                                float softmax_scale, void* out, float* lse, int32_t* idx_out,
                                int chunk_tokens, void* workspace, size_t workspace_bytes,
                                void* stream, void* const* stage_events, int n_stage_events);

/*
 * Dense causal attention through the same attention kernel: the "seamless
 * switch" between full and block-sparse attention ([W] section "將 MoBA 與
 * Full Attention 融合到一起會如何？": a model may swap MoBA and full attention
 * between training stages or per layer; [S] "MoBA: Mixture of Block Attention
 * for Long-Context LLMs", "Key contributions": seamless transition between
 * full and sparse attention).  Every query attends every key from its
 * sequence start up to itself (token-level causal mask) -- what moba_forward
 * computes when topk is at least the number of blocks of every sequence --
 * with no gate, no grouping and no merge: out and lse are written directly.
 * Same layouts, alignment and head_dim / head-count rules as moba_forward;
 * softmax_scale <= 0 selects 1/sqrt(head_dim).  The workspace (size from
 * moba_full_workspace_size, a few bytes per 256 tokens) holds the block plan
 * and the device error word; read errors with moba_check.
 */
size_t moba_full_workspace_size(int total_tokens, int n_seqs, int n_heads, int n_kv_heads,
                                int head_dim);
moba_status moba_forward_full(const void* q, const void* k, const void* v,
                              const int32_t* cu_seqlens, int n_seqs, int total_tokens,
                              int n_heads, int n_kv_heads, int head_dim, float softmax_scale,
                              void* out, float* lse, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * Decode: one new query token per sequence against a KV cache, with the
 * gate's block means kept incrementally ([W] section "MoBA：將 MoE 原理應用于
 * 注意力機制": gate over block means, attention to the chosen blocks, merge --
 * here for one query row per sequence; [S] "Limitations": generation still
 * ran full attention in the paper).
 *
 * Layouts (padded per sequence):
 *   q        bf16 [n_seqs, Hq, d]            the new token's query
 *   k_cache, v_cache
 *            bf16 [n_seqs, max_len, Hkv, d]  positions 0 .. seqlens[s]-1 valid;
 *                                            the new token's k, v already written
 *                                            at position seqlens[s] - 1
 *   seqlens  int32 [n_seqs] device            cache length INCLUDING the new token,
 *                                            1 <= seqlens[s] <= max_len
 *   kbar     fp32 [n_seqs, max_len / B, Hkv, d]  mean key of every full block;
 *                                            filled by moba_decode_init, extended
 *                                            by moba_decode (NULL if max_len < B)
 *   out      bf16 [n_seqs, Hq, d]     lse fp32 [n_seqs, Hq]
 *   idx_out  int32 [n_seqs, Hq, topk] or NULL: the selection, as in moba_gate
 *
 * moba_decode computes, for each sequence, exactly the prefill forward's
 * output row t = seqlens[s] - 1 of the sequence's first seqlens[s] tokens
 * (same gate, tie rule and causal own block).  After the gate, if the new
 * token completes block j = t / block_size, that block's mean is written to
 * kbar for later steps.  moba_decode_init computes the means of every full
 * block of every sequence (after a prefill, or to rebuild the cache).  The
 * workspace (moba_decode_workspace_size) holds the error word, the selection
 * and the per-block partial results; read device errors with moba_check
 * (malformed seqlens: MOBA_ERR_BAD_SEQLENS).  Supported: head_dim in
 * {64, 128}, n_heads % n_kv_heads == 0, block_size a multiple of 64 and
 * <= 65536, 1 <= topk <= 64; q, caches, kbar and out 16-byte aligned.
 */
size_t moba_decode_workspace_size(int n_seqs, int max_len, int n_heads, int n_kv_heads,
                                  int head_dim, int block_size, int topk);
moba_status moba_decode_init(const void* k_cache, const int32_t* seqlens, int n_seqs,
                             int max_len, int n_kv_heads, int head_dim, int block_size,
                             float* kbar, void* workspace, size_t workspace_bytes, void* stream);
moba_status moba_decode(const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* seqlens, int n_seqs, int max_len, int n_heads,
                        int n_kv_heads, int head_dim, int block_size, int topk,
                        float softmax_scale, float* kbar, void* out, float* lse,
                        int32_t* idx_out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward of moba_forward with the selection held fixed: the gradients of
 * sum(dout * out) with respect to q, k and v ([W] opening list: trainable
 * block-sparse attention; the top-k gate passes no gradient).  Inputs are
 * the forward's inputs, its out and lse, its selection idx [T, Hq, topk]
 * (moba_forward's idx_out) and dout [T, Hq, d] bf16.  Writes every element of
 * dq [T, Hq, d] and dk, dv [T, Hkv, d] as fp32 (dk and dv sum over the query
 * heads of each kv head).  cu_seqlens must be the forward's; a row whose idx
 * is not a forward selection (ascending blocks of its sequence, the own block
 * last, min(topk, j + 1) of them, -1 after) raises MOBA_ERR_BAD_SELECTION.
 *
 * On the tensor cores: dK, dV per tile of 128 keys over every row that
 * attends it (the rows routed to its block, in ascending (token, head) order,
 * and the block's own rows), written directly; the routed rows' q and dout
 * are first copied contiguously into the workspace (at most 8 GiB of them at
 * a time; more are processed in chunks whose dK, dV add up in launch order).
 * dQ per (row, selected block) goes into fp32 partial slots of a query
 * chunk of chunk_tokens tokens (0 = all; the slots take chunk * n_heads *
 * topk * head_dim * 4 bytes of the workspace), summed in ascending block
 * order.  dq, dk and dv are the same from run to run and for any
 * chunk_tokens.
 * The workspace is sized by moba_backward_workspace_size with the same
 * arguments; errors found on the device are read with moba_check on it.
 * Same shape rules as moba_forward; dq, dk, dv 16-byte aligned.
 */
size_t moba_backward_workspace_size(int total_tokens, int n_seqs, int n_heads, int n_kv_heads,
                                    int head_dim, int block_size, int topk, int chunk_tokens);
moba_status moba_backward(const void* q, const void* k, const void* v, const void* out,
                          const float* lse, const void* dout, const int32_t* idx,
                          const int32_t* cu_seqlens, int n_seqs, int total_tokens, int n_heads,
                          int n_kv_heads, int head_dim, int block_size, int topk,
                          float softmax_scale, float* dq, float* dk, float* dv, int chunk_tokens,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * moba_gate without a caller-provided workspace.  No counterpart in the paper:
 * this entry point exists for callers that cannot allocate device memory at
 * the time they run the gate -- for example a host program whose device memory
 * is entirely reserved by another allocator that this code must not call
 * into, or an integration that forbids device allocations once it has
 * started.  Such callers still own and pass q, k, cu_seqlens and idx.
 *
 * Scratch (block tables and the pooled mean keys) comes from one static
 * device array of MOBA_GATE_STATIC_SCRATCH_BYTES (32 MiB) compiled into the
 * library; every GPU that loads the library holds it until the process exits.
 * Shapes whose gate scratch (moba_workspace_size's gate part) exceeds it are
 * rejected with MOBA_ERR_WORKSPACE before anything is enqueued.  The function
 * calls no cudaMalloc, cudaFree or allocating library routine.
 *
 * The first call on a device looks up that array's device address (with the
 * device current) and caches it for the current CUDA context; make that first
 * call before any stream capture on the device.  After a cudaDeviceReset (or
 * anything else that gives the device a new context in this process) the next
 * call looks the address up again, so make that call outside a capture too.
 * A call with total_tokens == 0 only clears the error word.
 * All calls on a device share the one array, which
 * keeps the previous call's contents (the parts the gate reads are rewritten
 * or cleared on every call): calls whose work overlaps on the GPU -- on
 * different streams, or from different host threads -- race and must be
 * serialised by the caller.  Device errors are recorded in the array's error
 * word; read them with moba_gate_noalloc_check.
 */
#define MOBA_GATE_STATIC_SCRATCH_BYTES (32u << 20)
moba_status moba_gate_noalloc(const void* q, const void* k, const int32_t* cu_seqlens,
                              int n_seqs, int total_tokens, int n_heads, int n_kv_heads,
                              int head_dim, int block_size, int topk, int32_t* idx,
                              void* stream);

/* moba_check for moba_gate_noalloc: synchronise `stream`, report the static
 * scratch's error word on the current device. */
moba_status moba_gate_noalloc_check(void* stream);

/*
 * Test of the failure path (no counterpart in the pages).  With enable != 0,
 * every later launch of the block-attention kernel (moba_forward, moba_forward_full)
 * runs in a mode where its Q-gather warps publish no work unit, so the other
 * roles' first waits -- which come before any copy or tensor-core instruction
 * is issued -- run out after about a millisecond instead of two seconds; the
 * kernel then frees its tensor memory and records MOBA_ERR_TIMEOUT, which
 * moba_check reports.  enable = 0 restores normal operation.  Process-wide
 * and not synchronised with launches in flight: for tests only.
 */
moba_status moba_debug_attention_wait_test(int enable);

/*
 * The MOBA_DEBUG build (libmoba_debug.so; no counterpart in the pages) stands
 * in for a memory checker.  Every index a kernel reads from the workspace and
 * uses as an address -- a work tile's bucket and entry range, a bucket entry
 * (routed row / partial slot), a scatter position, a decode block id -- is
 * tested against the buffer it addresses first; a failed test records
 * MOBA_ERR_BOUNDS (detail: the site, see moba_debug_error_info) and the kernel
 * drops that unit, row or write instead of making the access.  Each carved
 * workspace region is followed by a 256-byte guard, filled at the start of
 * every call and checked at its end (MOBA_ERR_CANARY, detail: the guard's
 * number); the workspace size functions include the guards.  Release builds
 * (libmoba.so) compile all of it out.
 *
 * moba_debug_build: 1 in the MOBA_DEBUG build, 0 otherwise.
 *
 * moba_debug_poison: plants a slip for the tests of those checks in the
 * MOBA_DEBUG build (MOBA_ERR_UNSUPPORTED in a release build): mode 1 makes
 * the block-attention kernel read the first bucket entry of every routed
 * tile as a slot outside the query chunk (caught by the entry check, the row
 * dropped); mode 2 overwrites one word of the first workspace guard after it
 * is filled (caught by the guard check).  0 restores normal operation.
 * Process-wide, read when a call is enqueued: for tests only.
 *
 * moba_debug_error_info: synchronise `stream` and copy the detail word that
 * goes with the error moba_check reports for `workspace` (0 if none).
 */
int moba_debug_build(void);
moba_status moba_debug_poison(int mode);
moba_status moba_debug_error_info(const void* workspace, void* stream, int* info);

/*
 * Synchronise `stream` and report the device-side error word of `workspace`
 * (MOBA_OK if the last call on it ran clean).  Also reports an asynchronous
 * CUDA error as MOBA_ERR_CUDA.
 */
moba_status moba_check(void* workspace, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOBA_H_ */
