/*
 * moba.h -- C ABI of libmoba: the causal prefill forward of MoBA (Mixture of
 * Block Attention) on one NVIDIA B200 (sm_100a).
 *
 * The operation (MoBA: Mixture of Block Attention for Long-Context LLMs):
 *   - the keys of each sequence are split into contiguous blocks of B tokens,
 *     the last block possibly short (wispaper.ai blog, "The Change", block
 *     partition; sherconan.github.io step 1);
 *   - each block is represented by the mean of its keys, and every query q
 *     scores every block before its own as s_j = <q, mean(K_j)> (same
 *     section, affinity equation; sherconan.github.io step 2);
 *   - the query keeps its own block plus the k-1 past blocks of highest
 *     score; future blocks are never chosen, ties go to the lower block
 *     index, and when fewer than k blocks exist all of them are kept (same
 *     section, routing and causality rules; sherconan.github.io steps 3-4);
 *   - exact softmax attention with scale 1/sqrt(d) runs over the chosen
 *     blocks only, causal inside the own block, and the per-block partial
 *     results are combined by online softmax into O and its log-sum-exp
 *     (wispaper.ai blog, "Efficiency and Implementation";
 *     globaladvisors.biz, "Underlying computational mechanism").
 *
 * Tensor layouts (all row-major, contiguous, device memory):
 *   batch calls : q, o  [batch][seqlen][num_q_heads][head_dim]  bf16
 *                 k, v  [batch][seqlen][num_kv_heads][head_dim] bf16
 *                 lse   [batch][num_q_heads][seqlen]            fp32 (natural log)
 *                 sel   [batch][num_q_heads][seqlen][top_k]     int32
 *   varlen calls: the same with the batch and seqlen axes replaced by the
 *                 packed token axis T: q, o [T][Hq][d], k, v [T][Hkv][d],
 *                 lse [Hq][T], sel [Hq][T][top_k]; sequence s covers tokens
 *                 [cu_seqlens[s], cu_seqlens[s+1]) (int32, device, length
 *                 num_seqs + 1, cu_seqlens[0] = 0, cu_seqlens[num_seqs] = T).
 *   Query head h reads kv head h / (num_q_heads / num_kv_heads).
 *   sel lists a row's chosen blocks (block ids within the sequence),
 *   ascending, the own block last, -1 padded to top_k.
 *
 * Ownership: the caller owns every pointer, including the workspace; the
 * library allocates no device memory.  Every call is asynchronous on
 * `stream` (a cudaStream_t; NULL = legacy default stream).  The workspace
 * must not be shared by calls that can run at the same time.
 *
 * Errors: invalid arguments are reported before anything is launched.
 * Errors found on the device (a stuck pipeline wait, malformed cu_seqlens,
 * an out-of-range selection) are latched in the workspace's status word (its
 * first 4 bytes) and reported, and cleared, by moba_last_device_status().
 * The word accumulates over calls, so it must be zero when a workspace is
 * first used: zero the first 256 bytes of a new workspace (or call
 * moba_last_device_status once and discard the result).  Nothing crosses the
 * ABI as an exception.
 */
#ifndef MOBA_H
#define MOBA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moba_stream_t; /* same type as cudaStream_t */

typedef enum moba_status {
  MOBA_OK = 0,
  MOBA_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, bad size or shape */
  MOBA_ERR_UNSUPPORTED = 2,  /* head_dim not 64/128, block_size not a multiple of 128,
                                top_k beyond 65, too many blocks per sequence,
                                tokens x num_q_heads >= 2^31 (q rows take an int32
                                index) */
  MOBA_ERR_WORKSPACE = 3,    /* ws null, misaligned (256 B) or smaller than required */
  MOBA_ERR_CUDA = 4,         /* a CUDA runtime call failed (launch, attribute, device) */
  MOBA_ERR_TIMEOUT = 5,      /* device: a pipeline wait ran out of time */
  MOBA_ERR_DEVICE_CHECK = 6  /* device: malformed cu_seqlens or selection, capacity */
} moba_status;

typedef struct moba_params {
  int batch;           /* sequences in a batch call (ignored by varlen calls) */
  int seqlen;          /* tokens per sequence in a batch call (ignored by varlen calls) */
  int num_q_heads;     /* Hq */
  int num_kv_heads;    /* Hkv, divides Hq */
  int head_dim;        /* d: 64 or 128 */
  int block_size;      /* B: multiple of 128 */
  int top_k;           /* k >= 1, the own block included */
  float softmax_scale; /* <= 0 selects 1/sqrt(head_dim) */
} moba_params;

/* Workspace bytes for moba_gate / moba_forward on a batch of
 * params->batch sequences of params->seqlen tokens.  The forward processes
 * the kv heads in passes; `heads_per_pass` (1..num_kv_heads, <= 0 = all)
 * sets how many kv heads one pass holds, which is what the size grows with.
 * moba_forward picks the largest pass the given workspace holds. */
size_t moba_workspace_size(const moba_params *p, int heads_per_pass);

/* The same for varlen calls over `total_tokens` tokens in `num_seqs`
 * sequences (an upper bound covering any split of the tokens). */
size_t moba_workspace_size_varlen(const moba_params *p, int64_t total_tokens, int num_seqs,
                                  int heads_per_pass);

/* Gate only: block means, scores, top-k; writes sel.  Follows the routing
 * and causality rules cited above. */
moba_status moba_gate(const void *q, const void *k, int32_t *sel, const moba_params *p,
                      void *ws, size_t ws_bytes, moba_stream_t stream);
moba_status moba_gate_varlen(const void *q, const void *k, const int32_t *cu_seqlens,
                             int num_seqs, int64_t total_tokens, int32_t *sel,
                             const moba_params *p, void *ws, size_t ws_bytes,
                             moba_stream_t stream);

/* Allocation-free variant of moba_gate (batch layout only).  The method
 * described in the pages has no counterpart to this call: it exists for
 * callers that cannot allocate device memory or pass a workspace, such as
 * code inside a host framework that owns every device allocation, or a
 * latency-critical loop that must not call cudaMalloc.  Its scratch is one
 * fixed 16 MiB device array inside the library, so:
 *   - a shape whose gate scratch (block means: 4 * num_kv_heads *
 *     ceil(seqlen / block_size) * batch * head_dim bytes, plus a few KB)
 *     exceeds 16 MiB returns MOBA_ERR_WORKSPACE and launches nothing;
 *   - every GPU that loads the library keeps that array until exit;
 *   - all calls on a device share it and leave their data in it: calls that
 *     can overlap on the GPU race, and the caller must order them;
 *   - the first call on a device looks up the array's address with that
 *     device current; make that first call before any stream capture.
 * Results equal moba_gate's for the same inputs.  The size limit is checked
 * before the pointers, so a refused shape launches nothing whatever the
 * pointers are.  Device-side checks (a pipeline wait that ran out of time,
 * a bad index) latch bits in the array's status word, which no call clears:
 * moba_gate_noalloc_status reads them. */
moba_status moba_gate_noalloc(const void *q, const void *k, int32_t *sel, const moba_params *p,
                              moba_stream_t stream);
/* Status of the allocation-free gate's device checks on the current device:
 * synchronises `stream`, reads the status word every moba_gate_noalloc call
 * on this device latches into, clears it and returns MOBA_OK,
 * MOBA_ERR_TIMEOUT or MOBA_ERR_DEVICE_CHECK (as moba_last_device_status does
 * for a workspace).  Allocates nothing. */
moba_status moba_gate_noalloc_status(moba_stream_t stream);

/* Full MoBA prefill forward: o and lse; sel_out (nullable) receives the
 * selection. */
moba_status moba_forward(const void *q, const void *k, const void *v, void *o, float *lse,
                         int32_t *sel_out, const moba_params *p, void *ws, size_t ws_bytes,
                         moba_stream_t stream);
moba_status moba_forward_varlen(const void *q, const void *k, const void *v,
                                const int32_t *cu_seqlens, int num_seqs, int64_t total_tokens,
                                void *o, float *lse, int32_t *sel_out, const moba_params *p,
                                void *ws, size_t ws_bytes, moba_stream_t stream);

/* ------------------------------------------------- forward on host buffers
 * moba_forward with q, k, v, o, lse and sel_out (nullable) in HOST memory
 * (batch layout; page-locked memory lets the copies overlap the work).  The
 * call copies each group of kv heads' q / k / v columns in while the previous
 * group computes, and that group's o / lse / sel rows back while the next
 * computes, on two internal copy streams ordered against `stream`.  dev_buf is
 * device memory of moba_forward_host_buffer_size(p, heads_per_pass) bytes (or
 * more: the largest group of kv heads that fits is used); its first 256 bytes
 * are the status word of a workspace (zero them before first use;
 * moba_last_device_status(dev_buf) reads them).  Results equal moba_forward's.
 * Returns when the work is queued; synchronise `stream` before reading o.
 * Errors: a null q, k, v, o or lse -> MOBA_ERR_INVALID_ARG; dev_buf null, not
 * 256-byte aligned or smaller than one kv head's share -> MOBA_ERR_WORKSPACE;
 * parameters as for moba_forward. */
size_t moba_forward_host_buffer_size(const moba_params *p, int heads_per_pass);
moba_status moba_forward_host(const void *q, const void *k, const void *v, void *o, float *lse,
                              int32_t *sel_out, const moba_params *p, void *dev_buf,
                              size_t dev_bytes, moba_stream_t stream);
/* moba_forward_host for packed sequences: q, o [T][Hq][d], k, v [T][Hkv][d],
 * lse [Hq][T], sel_out [Hq][T][top_k] and cu_seqlens [num_seqs + 1] int32,
 * all in HOST memory (cu_seqlens is copied into dev_buf, sized by
 * moba_forward_host_buffer_size_varlen).  Results equal moba_forward_varlen's.
 * Errors as moba_forward_host; malformed cu_seqlens latch
 * MOBA_ERR_DEVICE_CHECK in dev_buf's status word. */
size_t moba_forward_host_buffer_size_varlen(const moba_params *p, int64_t total_tokens,
                                            int num_seqs, int heads_per_pass);
moba_status moba_forward_host_varlen(const void *q, const void *k, const void *v,
                                     const int32_t *cu_seqlens, int num_seqs,
                                     int64_t total_tokens, void *o, float *lse, int32_t *sel_out,
                                     const moba_params *p, void *dev_buf, size_t dev_bytes,
                                     moba_stream_t stream);

/* ----------------------------------------------------------------- backward
 * Gradients of the forward's attention for an output gradient dO, over the
 * selection the forward used (batch layout).  No gradient passes through the
 * hard top-k gate (wispaper.ai blog, "The Change": the gradient does not flow
 * through the discrete selection), so sel is an input: for every row and
 * head, with P the attention probabilities over the chosen keys (from q, k
 * and the forward's lse) and D = dO . o,
 *   dS_u = P_u (dO . v_u - D),  dq = scale sum_u dS_u k_u,
 *   dk_u += scale dS_u q,       dv_u += P_u dO.
 * Inputs: q, k, v, o, dO as the forward's layouts (bf16), lse [batch][Hq][seqlen]
 * fp32 and sel [batch][Hq][seqlen][top_k] exactly as moba_forward wrote them.
 * Outputs dq [batch][seqlen][Hq][d], dk / dv [batch][seqlen][Hkv][d], bf16.
 * The workspace holds the fp32 accumulators (moba_backward_workspace_size;
 * heads_per_pass as for the forward; its status word as for the forward).
 * Errors: a null pointer, a tensor not 16-byte aligned, or lse / sel not
 * 4-byte aligned -> MOBA_ERR_INVALID_ARG; parameters as for moba_forward
 * (MOBA_ERR_UNSUPPORTED for d or top_k outside what the kernels take); a
 * workspace that is null, misaligned or too small -> MOBA_ERR_WORKSPACE.  A
 * selection entry out of range (a future or missing block) is skipped and
 * latched in the status word (MOBA_ERR_DEVICE_CHECK). */
size_t moba_backward_workspace_size(const moba_params *p, int heads_per_pass);
moba_status moba_backward(const void *q, const void *k, const void *v, const void *o,
                          const float *lse, const void *dO, const int32_t *sel, void *dq,
                          void *dk, void *dv, const moba_params *p, void *ws, size_t ws_bytes,
                          moba_stream_t stream);
/* The backward for packed sequences (cu_seqlens [num_seqs + 1] int32 on the
 * device, as moba_forward_varlen): q, o, dO, dq [T][Hq][d], k, v, dk, dv
 * [T][Hkv][d], lse [Hq][T], sel [Hq][T][top_k] as moba_forward_varlen wrote
 * them; p->batch and p->seqlen are not used.  Workspace:
 * moba_backward_workspace_size_varlen.  Errors as moba_backward. */
size_t moba_backward_workspace_size_varlen(const moba_params *p, int64_t total_tokens,
                                           int num_seqs, int heads_per_pass);
moba_status moba_backward_varlen(const void *q, const void *k, const void *v, const void *o,
                                 const float *lse, const void *dO, const int32_t *sel,
                                 const int32_t *cu_seqlens, int num_seqs, int64_t total_tokens,
                                 void *dq, void *dk, void *dv, const moba_params *p, void *ws,
                                 size_t ws_bytes, moba_stream_t stream);

/* ------------------------------------------------------- routing variants
 * The pages present the gate as one member of a family: sliding-window attention is a gate that always selects the most
 * recent blocks, sink attention one that always selects the initial and the
 * most recent blocks (wispaper.ai blog, "Why the Change Is Plausible"), and
 * Quest is MoBA with smaller blocks and min/max pooling (elamur summary
 * card, "Key points").  A selection written by any of these has the gate's
 * format: for a row in block i, exactly min(top_k - 1, i) past blocks
 * ascending, then i, then -1 padding. */
typedef enum moba_route_mode {
  MOBA_ROUTE_WINDOW = 0, /* the own block and the top_k - 1 most recent past blocks */
  MOBA_ROUTE_SINK = 1    /* block 0, the top_k - 2 most recent past blocks, the own block */
} moba_route_mode;

/* Static selection (no scores) into sel [batch][num_q_heads][seqlen][top_k];
 * with fewer than top_k blocks every block is kept.  No workspace. */
moba_status moba_static_selection(int32_t *sel, int mode, const moba_params *p,
                                  moba_stream_t stream);

/* Gate with min/max-pooled blocks: the elementwise max M_j and min m_j of
 * each block's keys, score s_j = sum_c max(q_c M_jc, q_c m_jc) (Quest's bound
 * on q . k over the block), then the same top-k, causality and tie rules as
 * moba_gate.  Workspace: moba_workspace_size(p, 1). */
moba_status moba_gate_minmax(const void *q, const void *k, int32_t *sel, const moba_params *p,
                             void *ws, size_t ws_bytes, moba_stream_t stream);

/* Forward over a caller-given selection sel [batch][num_q_heads][seqlen][top_k]
 * in the gate's format (e.g. from moba_static_selection or moba_gate_minmax):
 * no scoring; the attention, merge and outputs as moba_forward.  Entries that
 * break the format (a past block >= the own block, a -1 among the first
 * min(top_k - 1, i)) latch MOBA_ERR_DEVICE_CHECK. */
moba_status moba_forward_selected(const void *q, const void *k, const void *v, void *o,
                                  float *lse, const int32_t *sel, const moba_params *p,
                                  void *ws, size_t ws_bytes, moba_stream_t stream);

/* moba_gate_minmax followed by moba_forward_selected, in one call. */
moba_status moba_forward_minmax(const void *q, const void *k, const void *v, void *o,
                                float *lse, int32_t *sel_out, const moba_params *p, void *ws,
                                size_t ws_bytes, moba_stream_t stream);

/* Packed-sequence forms of the four calls above (cu_seqlens [num_seqs + 1]
 * int32 on the device; blocks and positions counted from each sequence's
 * start, as moba_forward_varlen): q, o [T][Hq][d], k, v [T][Hkv][d], lse
 * [Hq][T], sel [Hq][T][top_k].  Workspace: moba_workspace_size_varlen(p,
 * total_tokens, num_seqs, 1) for the gate, any heads_per_pass for the
 * forwards.  Errors as the batch forms; malformed cu_seqlens latch
 * MOBA_ERR_DEVICE_CHECK. */
moba_status moba_static_selection_varlen(int32_t *sel, int mode, const int32_t *cu_seqlens,
                                         int num_seqs, int64_t total_tokens,
                                         const moba_params *p, moba_stream_t stream);
moba_status moba_gate_minmax_varlen(const void *q, const void *k, const int32_t *cu_seqlens,
                                    int num_seqs, int64_t total_tokens, int32_t *sel,
                                    const moba_params *p, void *ws, size_t ws_bytes,
                                    moba_stream_t stream);
moba_status moba_forward_selected_varlen(const void *q, const void *k, const void *v,
                                         const int32_t *cu_seqlens, int num_seqs,
                                         int64_t total_tokens, void *o, float *lse,
                                         const int32_t *sel, const moba_params *p, void *ws,
                                         size_t ws_bytes, moba_stream_t stream);
moba_status moba_forward_minmax_varlen(const void *q, const void *k, const void *v,
                                       const int32_t *cu_seqlens, int num_seqs,
                                       int64_t total_tokens, void *o, float *lse,
                                       int32_t *sel_out, const moba_params *p, void *ws,
                                       size_t ws_bytes, moba_stream_t stream);

/* Dense causal attention over every earlier token of each sequence: the
 * k = n limit of the method (wispaper.ai blog, "The Change": k = n
 * recovers full attention).  block_size and top_k are not used. */
size_t moba_full_causal_workspace_size(int64_t total_tokens, int num_seqs);
moba_status moba_full_causal(const void *q, const void *k, const void *v, void *o, float *lse,
                             const moba_params *p, void *ws, size_t ws_bytes,
                             moba_stream_t stream);
moba_status moba_full_causal_varlen(const void *q, const void *k, const void *v,
                                    const int32_t *cu_seqlens, int num_seqs,
                                    int64_t total_tokens, void *o, float *lse,
                                    const moba_params *p, void *ws, size_t ws_bytes,
                                    moba_stream_t stream);

/* ------------------------------------------------------------------ decode
 * One decode step: a single new query per sequence against its KV cache.
 * The new token of sequence b is at position t = seqlens[b] - 1 of the cache
 * (its key and value already written there), in block i = t / block_size.
 * Its selection and attention follow the same rules as the prefill (cited
 * at the top of this file): scores against the means of blocks 0..i-1, the
 * k-1 best kept (ties to the lower block), the own block i always kept,
 * attention over the kept blocks with the own block ending at t.  The pages
 * evaluate MoBA for prefill with full attention during generation
 * (wispaper.ai blog, "Real-World LLM and Benchmark Evidence") and name its
 * extension to generation as a next step ("Deep Insight and Conclusion");
 * the operation here is exactly the prefill's last row, computed against a
 * cache.
 *
 * Layouts (device memory, contiguous):
 *   q        [batch][num_q_heads][head_dim] bf16: the new token's queries
 *   k_cache, v_cache [batch][cache_len][num_kv_heads][head_dim] bf16
 *   seqlens  [batch] int32: tokens in each cache, the new one included
 *            (1 <= seqlens[b] <= cache_len; others latch MOBA_ERR_DEVICE_CHECK)
 *   kbar     [batch][num_kv_heads][ceil(cache_len / block_size)][head_dim]
 *            fp32: means of the complete blocks, kept by
 *            moba_kbar_cache_update (moba_kbar_cache_size bytes)
 *   o        [batch][num_q_heads][head_dim] bf16
 *   lse      [batch][num_q_heads] fp32 (natural log)
 *   sel_out  [batch][num_q_heads][top_k] int32, nullable: the kept blocks,
 *            ascending, own block last, -1 padded
 * Same ownership and error rules as above; top_k is at most 65. */
typedef struct moba_decode_params {
  int batch;           /* sequences */
  int cache_len;       /* capacity of each sequence's cache, in tokens */
  int num_q_heads;     /* Hq */
  int num_kv_heads;    /* Hkv, divides Hq */
  int head_dim;        /* 64 or 128 */
  int block_size;      /* multiple of 128 */
  int top_k;           /* 1 .. 65, the own block included */
  float softmax_scale; /* <= 0 selects 1/sqrt(head_dim) */
} moba_decode_params;

/* Workspace bytes for moba_decode and moba_kbar_cache_update (0 if the
 * parameters are invalid). */
size_t moba_decode_workspace_size(const moba_decode_params *p);

/* Bytes of the block-mean cache kbar. */
size_t moba_kbar_cache_size(const moba_decode_params *p);

/* Writes the mean of cache blocks into kbar.  only_last = 0: every complete
 * block of each sequence (blocks j with (j + 1) * block_size <= seqlens[b]),
 * e.g. after a prefill; only_last != 0: only the block the newest token
 * completed (when seqlens[b] is a multiple of block_size), e.g. after each
 * appended token.  Block means as defined above (wispaper.ai blog,
 * "The Change"; sherconan.github.io step 1). */
moba_status moba_kbar_cache_update(const void *k_cache, const int32_t *seqlens, float *kbar,
                                   int only_last, const moba_decode_params *p, void *ws,
                                   size_t ws_bytes, moba_stream_t stream);

/* The decode step: o, lse and (optionally) sel for every sequence's new
 * token. */
moba_status moba_decode(const void *q, const void *k_cache, const void *v_cache,
                        const int32_t *seqlens, const float *kbar, void *o, float *lse,
                        int32_t *sel_out, const moba_decode_params *p, void *ws,
                        size_t ws_bytes, moba_stream_t stream);

/* Synchronises `stream`, returns and clears the device status latched in
 * `ws` by earlier calls (MOBA_OK, MOBA_ERR_TIMEOUT or MOBA_ERR_DEVICE_CHECK). */
moba_status moba_last_device_status(void *ws, moba_stream_t stream);

/* Per-kernel timing, for benchmarks: while enabled, every kernel launch the
 * library makes is bracketed by CUDA events recorded on the launch stream.
 * moba_profile_read synchronises those events and returns, per kernel class
 * (plan, pool, gate, gate_count, bucket_scan, bucket_scatter, attn_routed,
 * attn_own, merge, attn_dense, kbar_cache, decode_gate, decode_attn,
 * decode_merge, minmax_pool, gate_minmax, static_select, bw_prep, bw_kv,
 * bw_q, bw_finish, vbound), the launch count and summed device milliseconds since the
 * last reset.  Returns the number of classes written (<= max_entries).
 * Not thread safe; meant for one benchmarking thread. */
typedef struct moba_kernel_time {
  char name[24];
  int launches;
  double total_ms;
} moba_kernel_time;
void moba_profile_enable(int on);
void moba_profile_reset(void);
int moba_profile_read(moba_kernel_time *out, int max_entries);

/* Diagnostic: launches one thread that waits, with the same bounded wait the
 * pipelines use but a limit of `limit_cycles` SM clocks (1 .. 4e9), on a
 * barrier nothing arrives on.  The wait gives up and latches the timeout bit
 * in ws's status word; moba_last_device_status(ws) then returns
 * MOBA_ERR_TIMEOUT and the context stays usable.  Shows that a stuck pipeline
 * ends in an error status instead of a hang.  ws needs 256 bytes; a null ws
 * targets the allocation-free gate's status word instead (read it back with
 * moba_gate_noalloc_status). */
moba_status moba_selftest_wait_timeout(void *ws, size_t ws_bytes, long long limit_cycles,
                                       moba_stream_t stream);

/* Static, human-readable name of a status code. */
const char *moba_status_string(moba_status s);

/* Text of the last CUDA runtime error that made a call on this thread
 * return MOBA_ERR_CUDA ("no error" if none). */
const char *moba_last_error_string(void);

/* Library version: major * 10000 + minor * 100 + patch. */
int moba_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOBA_H */
