/*
 * lvx.h — C ABI of liblvx.so: exact blockwise attention with online-softmax
 * merging on one NVIDIA B200 (sm_100a).
 *
 * What is computed.  For every batch b, query head h and query row r, with
 * key/value head g = h / (H / H_kv) and scale s (1/sqrt(d) by default):
 *     O[b,r,h,:] = sum_j softmax_j(s * q_r . k_j) v_j,
 *     LSE[b,h,r] = ln sum_j exp(s * q_r . k_j)            (natural log)
 * over the visible keys j (all keys, or j <= r when causal).  This is the
 * exact attention of "Ring Attention with Blockwise Transformers for
 * Near-Infinite Context" (citation hub page, abstract), evaluated the way
 * "LV-XAttn: Distributed Cross-Attention for Long Visual Inputs in
 * Multimodal Large Language Models" (review page, "The reading", "What
 * carries the argument", Figure 3 / Algorithm 1) evaluates it: the key/value
 * sequence is cut into n stationary blocks, each block yields a partial
 * output O_i and log-sum-exp statistic L_i, and the partials are combined by
 * FlashAttention-style rescaling.  On one GPU the n blocks are processed in
 * parallel instead of around a ring; no inter-GPU communication is involved.
 *
 * Layouts (all contiguous, row-major, element type set by lvx_dtype):
 *   q, out, dout, dq : [B, S_Q,  H,    d]
 *   k, v, dk, dv     : [B, S_KV, H_kv, d]
 *   lse              : [B, H, S_Q]  float32, natural log
 *   y                : [B, S_KV, d_embed];  w_k, w_v : [d_embed, H_kv*d]
 *
 * Ownership and ordering.  The caller owns every buffer (inputs, outputs,
 * workspace); all pointers are device pointers unless stated otherwise.  The
 * library never allocates or frees memory and never synchronises, except
 * lvx_last_device_error.  Every call is enqueued on the given stream and
 * returns before the GPU work finishes.  The library keeps no per-call state
 * and may be called from several host threads.
 *
 * Errors.  Invalid arguments are reported synchronously and nothing is
 * launched.  Launch failures return LVX_ERR_CUDA.  Kernels never trap: a
 * bounded wait that expires inside a kernel records an error word on the
 * device, the kernel returns, and lvx_last_device_error reports it as
 * LVX_ERR_DEVICE_TIMEOUT.
 */
#ifndef LVX_H_
#define LVX_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LVX_OK = 0,
  LVX_ERR_INVALID_ARG = 1,    /* null/misaligned pointer, bad size, short workspace */
  LVX_ERR_UNSUPPORTED = 2,    /* valid but not implemented (see each call)        */
  LVX_ERR_WORKSPACE = 3,      /* workspace smaller than the size query returned    */
  LVX_ERR_CUDA = 4,           /* a CUDA runtime/driver call or launch failed       */
  LVX_ERR_DEVICE_TIMEOUT = 5  /* a bounded in-kernel wait expired                  */
} lvx_status;

typedef enum { LVX_FP32 = 0, LVX_BF16 = 1 } lvx_dtype;

/* A cudaStream_t passed as an opaque pointer; NULL is the legacy default stream. */
typedef void* lvx_stream;

/* Returns a static, human-readable name for a status code. */
const char* lvx_status_string(lvx_status s);

/* Library version as 10000*major + 100*minor + patch. */
int lvx_version(void);

/*
 * Workspace bytes that lvx_attn_fwd needs for these arguments (0 when
 * n_blocks == 1).  Layout, each part starting on a 256-byte boundary:
 *   O_parts [n_blocks, B, H, S_Q, d] float32   normalised partial outputs O_i
 *   L_parts [n_blocks, B, H, S_Q]    float32   partial log-sum-exp L_i
 * For causal calls only the partials of blocks j <= (block of row r) are
 * written; the others are left untouched.  Returns 0 for invalid shapes.
 */
size_t lvx_attn_fwd_workspace(int B, int H, int H_kv, int S_Q, int S_KV, int d,
                              int n_blocks, int causal, lvx_dtype dt);

/*
 * Blockwise attention forward.
 *   LV-XAttn review page, Figure 3 / Algorithm 1: key/value block i of n
 *   (keys [i*ceil(S_KV/n), min((i+1)*ceil(S_KV/n), S_KV))) produces the
 *   partial (O_i, L_i) of attention over that block alone; "What carries the
 *   argument": the partials are combined by rescaling,
 *     L = M + ln sum_i exp(L_i - M),  M = max_i L_i;   O = sum_i exp(L_i - L) O_i.
 *   An empty block contributes the identity (O_i, L_i) = (0, -inf).
 * Causal (self-attention only, S_Q == S_KV): key j is visible to query r iff
 *   j <= r; query rows use the same n-block partition, block pairs
 *   (query block i, key block j) with j > i are skipped, and within the
 *   diagonal pair tiles entirely above the diagonal are skipped.
 * Arguments:
 *   q, k, v     inputs (device, dtype dt); out [B,S_Q,H,d] (device, dtype dt);
 *   lse         [B,H,S_Q] float32 output (device); may not be NULL.
 *   scale       softmax scale; <= 0 selects 1/sqrt(d).
 *   workspace   device buffer of at least lvx_attn_fwd_workspace(...) bytes,
 *               or NULL when that size is 0.
 * Constraints (else LVX_ERR_INVALID_ARG): all sizes >= 1, H % H_kv == 0,
 *   1 <= n_blocks <= S_KV, pointers 16-byte aligned, ws_bytes large enough.
 * LVX_ERR_UNSUPPORTED: d > 128 or d % 8 != 0; causal with S_Q != S_KV;
 *   unknown dtype.
 * bf16 with d in {64, 128} runs the tcgen05 tensor-core kernel; fp32 (and
 *   bf16 with other d) runs an fp32 CUDA-core kernel.  Accumulation and the
 *   softmax statistics are fp32 in both.
 */
lvx_status lvx_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                        int B, int H, int H_kv, int S_Q, int S_KV, int d,
                        int n_blocks, int causal, lvx_dtype dt, float scale,
                        void* workspace, size_t ws_bytes, lvx_stream stream);

/*
 * lvx_attn_fwd without a workspace, for callers that cannot allocate device
 * memory (a runtime whose device memory is fixed at start-up, a plug-in
 * inside a host program that owns all device allocations, a latency-critical
 * path that must not reach an allocator).  The pages have no counterpart to
 * this call; it computes exactly what lvx_attn_fwd computes, with the same
 * arguments minus the workspace.
 * The block partials live in one file-scope device array of 64 MiB
 * (n_blocks*B*H*S_Q*d*4 + n_blocks*B*H*S_Q*4 bytes, each part rounded up to
 * 256, must fit; otherwise LVX_ERR_WORKSPACE is returned and nothing runs).
 * Every GPU that loads the library holds that array until the process exits.
 * All calls on a device share it and it keeps the last call's contents;
 * nothing in it needs to start at zero, but calls whose kernels overlap on
 * the GPU race on it, so order them on one stream.  The first call in each
 * CUDA context (normally a device's primary context) looks up the array's
 * device address (cudaGetSymbolAddress, with that context current) and caches
 * it per context, so a context created later, after cudaDeviceReset for
 * instance, looks it up again; make the first call in a context before any
 * stream capture.  Validation, kernels and partial layout are those of
 * lvx_attn_fwd, so the results are identical.  No memory is allocated or
 * freed by this call.
 */
lvx_status lvx_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                                int B, int H, int H_kv, int S_Q, int S_KV, int d,
                                int n_blocks, int causal, lvx_dtype dt, float scale,
                                lvx_stream stream);

/*
 * Block partials without the merge: the per-block step of lvx_attn_fwd on its
 * own, for callers that merge elsewhere -- in LV-XAttn each worker keeps one
 * stationary shard of the keys and values and its partials are combined with
 * the other workers' (LV-XAttn review page, "The reading" and Figure 3 /
 * Algorithm 1; the rescaling is lvx_merge_partials); in Ring Attention each
 * worker computes the partial of its query block against the key/value block
 * it holds at each ring step (Ring Attention with Blockwise Transformers
 * page, abstract; LV-XAttn review page, "Core claim").
 *   q [B,S_Q,H,d], k, v [B,S_KV,H_kv,d] (device, dtype dt): the caller's shard
 *   of the keys and values, cut into n_blocks blocks as lvx_attn_fwd cuts them.
 *   O_parts [n_blocks, B, H, S_Q, d] float32 and L_parts [n_blocks, B, H, S_Q]
 *   float32 (device, caller-owned, 16-byte aligned): the normalised partial
 *   outputs and their natural-log log-sum-exp; an empty block writes (0, -inf).
 * causal = 1 (S_Q == S_KV, the diagonal block of a self-attention): key j is
 * visible to query row r iff j <= r.  With n_blocks > 1, the partial of block
 * i is written only for the rows that see some key of it (r >= i * block
 * length); the other rows of O_parts / L_parts are left as they were.
 * The same constraints and errors as lvx_attn_fwd without a workspace.
 */
lvx_status lvx_attn_fwd_partials(const void* q, const void* k, const void* v, float* O_parts,
                                 float* L_parts, int B, int H, int H_kv, int S_Q, int S_KV, int d,
                                 int n_blocks, int causal, lvx_dtype dt, float scale,
                                 lvx_stream stream);

/*
 * Merge of block partials on its own (the rescaling step of lvx_attn_fwd),
 * for callers that produce the partials elsewhere, e.g. one block per GPU.
 *   O_parts [n, B, H, S_Q, d] float32, L_parts [n, B, H, S_Q] float32 (device)
 *   -> out [B, S_Q, H, d] (dtype dt), lse [B, H, S_Q] float32.
 * A row whose partials are all -inf gets out = 0 and lse = -inf.
 * Same pointer/size rules as lvx_attn_fwd; d <= 128, d % 8 == 0.
 */
lvx_status lvx_merge_partials(const float* O_parts, const float* L_parts, void* out, float* lse,
                              int n, int B, int H, int S_Q, int d, lvx_dtype dt,
                              lvx_stream stream);

/*
 * Workspace bytes for lvx_attn_bwd.  Layout (256-byte aligned parts):
 *   ND     [B, H, S_Q]      float32  -rowsum(dO o O)
 *   NLSE2  [B, H, S_Q]      float32  -lse * log2(e)
 *   dQ_acc [B, S_Q, H, d]   float32  unscaled dQ accumulator
 */
size_t lvx_attn_bwd_workspace(int B, int H, int H_kv, int S_Q, int S_KV, int d,
                              int causal, lvx_dtype dt);

/*
 * Blockwise attention backward: dQ, dK, dV from the stored LSE.
 *   The pages leave the backward pass unspecified (LV-XAttn review page,
 *   referee report, major comment 1); this is the exact gradient of the
 *   forward above.  P is recomputed as exp(s * q.k - LSE) from the forward's
 *   merged lse, then
 *     dV = P^T dO,  dP = dO V^T,  D = rowsum(dO o O),  dS = P o (dP - D),
 *     dQ = s dS K,  dK = s dS^T Q,
 *   with dK, dV summed over the query heads of each key/value group.
 * Arguments: q, k, v, out, dout (dtype dt), lse (float32) are the forward's
 *   inputs/outputs and the output gradient; dq [B,S_Q,H,d] and dk, dv
 *   [B,S_KV,H_kv,d] (dtype dt) are overwritten.  Same constraints and
 *   errors as lvx_attn_fwd.
 */
lvx_status lvx_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                        const float* lse, const void* dout, void* dq, void* dk, void* dv,
                        int B, int H, int H_kv, int S_Q, int S_KV, int d, int causal,
                        lvx_dtype dt, float scale, void* workspace, size_t ws_bytes,
                        lvx_stream stream);

/*
 * The same backward, with the gradients ADDED to caller-owned float32 arrays
 * instead of written: dq [B, S_Q, H, d], dk, dv [B, S_KV, H_kv, d] float32
 * (device, 16-byte aligned) receive dq += dQ, dk += dK, dv += dV of this
 * call.  For gradients summed over several calls -- the key/value blocks of a
 * ring (Ring Attention with Blockwise Transformers page, abstract) or any
 * split of the keys -- without rounding each part to the input dtype.  The
 * caller zeroes the arrays before the first call.  Inputs, workspace, shapes
 * and errors as lvx_attn_bwd; the calls of one stream accumulate in order.
 */
lvx_status lvx_attn_bwd_accumulate(const void* q, const void* k, const void* v, const void* out,
                                   const float* lse, const void* dout, float* dq, float* dk,
                                   float* dv, int B, int H, int H_kv, int S_Q, int S_KV, int d,
                                   int causal, lvx_dtype dt, float scale, void* workspace,
                                   size_t ws_bytes, lvx_stream stream);

/*
 * Key/value recomputation from the shared visual features.
 *   LV-XAttn review page, "What carries the argument" and Figure 6: one copy
 *   of y serves every cross-attention layer, and K, V are regenerated from it
 *   when needed:  K = y W_k,  V = y W_v  (no bias).
 *   y [B, S_KV, d_embed]; w_k, w_v [d_embed, H_kv*d] row-major; k, v outputs
 *   [B, S_KV, H_kv, d] (= [B, S_KV, H_kv*d]).  fp32 accumulation; bf16 outputs
 *   are rounded to nearest even.
 * Constraints: sizes >= 1, pointers 16-byte aligned.  bf16 with
 *   d_embed % 64 == 0 and (H_kv*d) % 256 == 0 runs on the tensor cores;
 *   otherwise, and for fp32, a CUDA-core kernel runs.
 */
lvx_status lvx_kv_recompute(const void* y, const void* w_k, const void* w_v, void* k, void* v,
                            int B, int S_KV, int d_embed, int H_kv, int d, lvx_dtype dt,
                            lvx_stream stream);

/*
 * Gradients of the key/value recomputation, for training with activation
 * recomputation (LV-XAttn review page, "What carries the argument" and
 * Figure 6: the keys and values are regenerated from y in the backward pass,
 * so the gradient reaching y and the projection weights goes through the
 * linear map K = y W_k, V = y W_v).  With y, dK, dV flattened to rows
 * s = b*S_KV + t:
 *   dW_k = y^T dK,   dW_v = y^T dV              [d_embed, H_kv*d]
 *   dy   = dK W_k^T + dV W_v^T                  [B, S_KV, d_embed]
 *   y [B, S_KV, d_embed]; w_k, w_v [d_embed, H_kv*d]; dk, dv [B, S_KV, H_kv, d]
 *   (the dK, dV of lvx_attn_bwd); outputs dy, dw_k, dw_v are written (not
 *   accumulated).  All in `dt`; fp32 accumulation, bf16 results rounded to
 *   nearest even.  Buffers are owned by the caller; inputs and outputs must
 *   not overlap.
 * Constraints: sizes >= 1, pointers 16-byte aligned, B*S_KV < 2^31.  bf16 with
 *   d_embed % 256 == 0 and (H_kv*d) % 256 == 0 runs on the tensor cores (two
 *   launches); otherwise, and for fp32, CUDA-core kernels run (three
 *   launches).  Returns LVX_ERR_INVALID_ARG / LVX_ERR_UNSUPPORTED before
 *   launching anything, LVX_ERR_CUDA if a launch fails.
 */
lvx_status lvx_kv_recompute_bwd(const void* y, const void* w_k, const void* w_v, const void* dk,
                                const void* dv, void* dy, void* dw_k, void* dw_v, int B, int S_KV,
                                int d_embed, int H_kv, int d, lvx_dtype dt, lvx_stream stream);

/*
 * Attention with the keys and values regenerated from the visual features one
 * key block at a time (LV-XAttn review page, "What carries the argument" and
 * Figure 6: one shared copy of the visual features y is kept and K = y W_k,
 * V = y W_v are recomputed wherever they are needed, the backward pass
 * included).  Neither call ever holds the whole K, V (or dK, dV): only one
 * block of block_len = ceil(S_KV / n_blocks) keys, in the workspace.
 *
 * lvx_attn_fwd_recompute: out, lse of attention(q, y W_k, y W_v), as
 *   lvx_kv_recompute followed by lvx_attn_fwd with the same n_blocks
 *   computes them: for each block, K_i, V_i = y_i W_k, y_i W_v, then the
 *   block's partials; then the merge.  Workspace:
 *   lvx_attn_fwd_recompute_workspace(...) bytes = the partials of
 *   lvx_attn_fwd (same layout, same place) followed by two block-sized bf16
 *   buffers.
 * lvx_attn_bwd_recompute: the gradients of that attention with respect to q,
 *   y and the weights, from the forward's out and lse and dout:
 *     dq [B, S_Q, H, d] (bf16, written)
 *     dy [B, S_KV, d_embed] (bf16, written) = dK W_k^T + dV W_v^T
 *     dw_k, dw_v [d_embed, H_kv*d] (float32, written) = y^T dK, y^T dV
 *   where dK, dV are attention's key/value gradients (never stored whole).
 *   Per block: K_i, V_i regenerated; the fused backward on the block with the
 *   global log-sum-exp (dQ added to a float32 accumulator); dy of the block's
 *   rows written; y_i^T dK_i, y_i^T dV_i added to dw_k, dw_v.  Workspace:
 *   lvx_attn_bwd_recompute_workspace(...) bytes = the workspace of
 *   lvx_attn_bwd followed by four block-sized bf16 buffers.
 * Shapes: q, out, dout [B, S_Q, H, d]; y [B, S_KV, d_embed]; w_k, w_v
 *   [d_embed, H_kv*d] row-major; lse [B, H, S_Q] float32 (natural log).
 *   Non-causal.  Buffers are owned by the caller; inputs and outputs must not
 *   overlap.  Calls are stream-ordered; nothing is allocated.
 * Constraints (else LVX_ERR_INVALID_ARG): as lvx_attn_fwd / lvx_attn_bwd,
 *   d_embed >= 1, pointers 16-byte aligned, workspace large enough.
 *   LVX_ERR_UNSUPPORTED unless bf16, d in {64, 128}, d_embed % 256 == 0 and
 *   (H_kv*d) % 256 == 0 (the tensor-core GEMMs); the workspace queries then
 *   return 0.  Block counts leaving trailing blocks empty are allowed (their
 *   partial is the merge's identity).  LVX_ERR_CUDA if a launch fails.
 */
size_t lvx_attn_fwd_recompute_workspace(int B, int H, int H_kv, int S_Q, int S_KV, int d,
                                        int d_embed, int n_blocks, lvx_dtype dt);
lvx_status lvx_attn_fwd_recompute(const void* q, const void* y, const void* w_k, const void* w_v,
                                  void* out, float* lse, int B, int H, int H_kv, int S_Q,
                                  int S_KV, int d, int d_embed, int n_blocks, lvx_dtype dt,
                                  float scale, void* workspace, size_t ws_bytes, lvx_stream stream);
size_t lvx_attn_bwd_recompute_workspace(int B, int H, int H_kv, int S_Q, int S_KV, int d,
                                        int d_embed, int n_blocks, lvx_dtype dt);
lvx_status lvx_attn_bwd_recompute(const void* q, const void* y, const void* w_k, const void* w_v,
                                  const void* out, const float* lse, const void* dout, void* dq,
                                  void* dy, float* dw_k, float* dw_v, int B, int H, int H_kv,
                                  int S_Q, int S_KV, int d, int d_embed, int n_blocks,
                                  lvx_dtype dt, float scale, void* workspace, size_t ws_bytes,
                                  lvx_stream stream);

/*
 * Synchronises `stream`, then reads and clears the device error word of the
 * current device.  Returns LVX_ERR_DEVICE_TIMEOUT if any kernel since the last
 * call gave up on a bounded wait, LVX_ERR_CUDA if the stream reported an
 * error, LVX_OK otherwise.
 */
lvx_status lvx_last_device_error(lvx_stream stream);

/*
 * Diagnostic: launches one small kernel that waits on a barrier nothing ever
 * completes.  Its bounded wait gives up after about 2 s, records a timeout in
 * the device error word and returns, exactly as the library's tensor-core
 * kernels do when an internal wait expires; the next lvx_last_device_error
 * then returns LVX_ERR_DEVICE_TIMEOUT and the context stays usable.  (Not part
 * of the attention method; used to test the failure path without a fault.)
 */
lvx_status lvx_selftest_wait_timeout(lvx_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* LVX_H_ */
