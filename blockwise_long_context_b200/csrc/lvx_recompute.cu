// Attention with the keys and values regenerated from the visual features,
// one key/value block at a time (LV-XAttn review page, "What carries the
// argument" and Figure 6: one shared copy of the visual features y is kept,
// and K = y W_k, V = y W_v are recomputed when they are needed, in the
// backward pass too).
//
// lvx_attn_fwd_recompute: for each key block i, K_i = y_i W_k and V_i = y_i W_v
//   (tensor-core GEMM into a block-sized buffer), then the block's partials
//   (O_i, L_i) with the forward kernel; finally the merge.
// lvx_attn_bwd_recompute: D = rowsum(dO o O) and the cleared dQ accumulator
//   once, then for each key block i: K_i, V_i regenerated; the fused backward
//   on the block with the global log-sum-exp (dQ added to the float32
//   accumulator, dK_i, dV_i written to block-sized buffers); dy_i = dK_i W_k^T
//   + dV_i W_v^T written; dW_k += y_i^T dK_i and dW_v += y_i^T dV_i added in
//   float32.  Finally dQ = s dQ_acc.
// Only one block's K, V, dK, dV exist at any time: for the Llama-3-V shape
// (S_KV = 65536, 8 blocks, H_kv d = 1024) 16 MiB each instead of 128 MiB.
#include <math.h>
#include <stdint.h>

#include "lvx_common.cuh"
#include "lvx_tc.cuh"

namespace lvx {
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shapes the recomputing entry points run: bf16, the tensor-core GEMMs
// (d_embed % 256, H_kv d % 256) and the tensor-core attention kernels.
lvx_status check_recompute(int B, int H, int H_kv, int S_Q, int S_KV, int d, int d_embed,
                           int n_blocks, lvx_dtype dt) {
  lvx_status st = check_shapes(B, H, H_kv, S_Q, S_KV, d, n_blocks, 0, dt);
  if (st != LVX_OK) return st;
  if (d_embed < 1) return LVX_ERR_INVALID_ARG;
  if (dt != LVX_BF16 || (d != 64 && d != 128)) return LVX_ERR_UNSUPPORTED;
  if (d_embed % 256 != 0 || (H_kv * d) % 256 != 0) return LVX_ERR_UNSUPPORTED;
  if ((long long)B * S_KV * d_embed > (1ll << 40)) return LVX_ERR_UNSUPPORTED;
  return LVX_OK;
}

// bytes of one block's K (or V, dK, dV): block_len keys x H_kv x d bf16
size_t block_kv_bytes(int S_KV, int n_blocks, int H_kv, int d) {
  const size_t block_len = (size_t)((S_KV + n_blocks - 1) / n_blocks);
  return align256(block_len * H_kv * d * 2);
}

size_t bwd_rows_bytes(int B, int H, int S_Q) { return align256((size_t)B * H * S_Q * sizeof(float)); }

}  // namespace
}  // namespace lvx

using namespace lvx;

extern "C" {

size_t lvx_attn_fwd_recompute_workspace(int B, int H, int H_kv, int S_Q, int S_KV, int d,
                                        int d_embed, int n_blocks, lvx_dtype dt) {
  if (check_recompute(B, H, H_kv, S_Q, S_KV, d, d_embed, n_blocks, dt) != LVX_OK) return 0;
  return fwd_parts_o_bytes(B, H, S_Q, d, n_blocks) + fwd_parts_l_bytes(B, H, S_Q, n_blocks) +
         2 * block_kv_bytes(S_KV, n_blocks, H_kv, d);
}

lvx_status lvx_attn_fwd_recompute(const void* q, const void* y, const void* w_k, const void* w_v,
                                  void* out, float* lse, int B, int H, int H_kv, int S_Q,
                                  int S_KV, int d, int d_embed, int n_blocks, lvx_dtype dt,
                                  float scale, void* workspace, size_t ws_bytes,
                                  lvx_stream stream) {
  lvx_status st = check_recompute(B, H, H_kv, S_Q, S_KV, d, d_embed, n_blocks, dt);
  if (st != LVX_OK) return st;
  const void* ptrs[] = {q, y, w_k, w_v, out, lse, workspace};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return LVX_ERR_INVALID_ARG;
  if (ws_bytes < lvx_attn_fwd_recompute_workspace(B, H, H_kv, S_Q, S_KV, d, d_embed, n_blocks, dt))
    return LVX_ERR_WORKSPACE;
  if (!(scale == scale)) return LVX_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const Problem p = make_problem(B, H, H_kv, S_Q, S_KV, d, n_blocks, 0, scale);
  char* ws = reinterpret_cast<char*>(workspace);
  float* o_parts = reinterpret_cast<float*>(ws);
  float* l_parts = reinterpret_cast<float*>(ws + fwd_parts_o_bytes(B, H, S_Q, d, n_blocks));
  char* kv = ws + fwd_parts_o_bytes(B, H, S_Q, d, n_blocks) + fwd_parts_l_bytes(B, H, S_Q, n_blocks);
  void* k_blk = kv;
  void* v_blk = kv + block_kv_bytes(S_KV, n_blocks, H_kv, d);
  const int N = H_kv * d;
  const size_t q_b = (size_t)S_Q * H * d * 2, part_o = (size_t)H * S_Q * d, part_l = (size_t)H * S_Q;
  for (int i = 0; i < n_blocks; ++i) {
    const int k0 = i * p.block_len;
    const int len = k0 < S_KV ? (S_KV - k0 < p.block_len ? S_KV - k0 : p.block_len) : 0;
    for (int b = 0; b < B; ++b) {
      float* o_i = o_parts + ((size_t)i * B + b) * part_o;
      float* l_i = l_parts + ((size_t)i * B + b) * part_l;
      const void* q_bp = reinterpret_cast<const char*>(q) + b * q_b;
      cudaError_t e;
      if (len == 0) {
        // an empty block (n does not divide S_KV finely enough): the merge's identity
        e = launch_empty_partial(o_i, l_i, (size_t)H * S_Q, d, s);
      } else {
        const Problem pb = make_problem(1, H, H_kv, S_Q, len, d, 1, 0, scale);
        const void* y_b = reinterpret_cast<const char*>(y) + ((size_t)b * S_KV + k0) * d_embed * 2;
        e = launch_kv_gemm_tc(y_b, w_k, w_v, k_blk, v_blk, len, d_embed, N, s);
        if (e == cudaSuccess) e = launch_fwd_tc(pb, q_bp, k_blk, v_blk, nullptr, nullptr, o_i, l_i, s);
      }
      if (e != cudaSuccess) return LVX_ERR_CUDA;
    }
  }
  cudaError_t e = launch_merge(o_parts, l_parts, out, lse, n_blocks, B, H, S_Q, d, 0, p.block_len,
                               dt, s);
  return e == cudaSuccess ? LVX_OK : LVX_ERR_CUDA;
}

size_t lvx_attn_bwd_recompute_workspace(int B, int H, int H_kv, int S_Q, int S_KV, int d,
                                        int d_embed, int n_blocks, lvx_dtype dt) {
  if (check_recompute(B, H, H_kv, S_Q, S_KV, d, d_embed, n_blocks, dt) != LVX_OK) return 0;
  return 2 * bwd_rows_bytes(B, H, S_Q) + align256((size_t)B * S_Q * H * d * sizeof(float)) +
         4 * block_kv_bytes(S_KV, n_blocks, H_kv, d);
}

lvx_status lvx_attn_bwd_recompute(const void* q, const void* y, const void* w_k, const void* w_v,
                                  const void* out, const float* lse, const void* dout, void* dq,
                                  void* dy, float* dw_k, float* dw_v, int B, int H, int H_kv,
                                  int S_Q, int S_KV, int d, int d_embed, int n_blocks,
                                  lvx_dtype dt, float scale, void* workspace, size_t ws_bytes,
                                  lvx_stream stream) {
  lvx_status st = check_recompute(B, H, H_kv, S_Q, S_KV, d, d_embed, n_blocks, dt);
  if (st != LVX_OK) return st;
  const void* ptrs[] = {q, y, w_k, w_v, out, lse, dout, dq, dy, dw_k, dw_v, workspace};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return LVX_ERR_INVALID_ARG;
  if (ws_bytes < lvx_attn_bwd_recompute_workspace(B, H, H_kv, S_Q, S_KV, d, d_embed, n_blocks, dt))
    return LVX_ERR_WORKSPACE;
  if (!(scale == scale)) return LVX_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const Problem p = make_problem(B, H, H_kv, S_Q, S_KV, d, n_blocks, 0, scale);
  const bool tc = tc_bwd_supported(p);
  char* ws = reinterpret_cast<char*>(workspace);
  const size_t rows = bwd_rows_bytes(B, H, S_Q);
  float* ND = reinterpret_cast<float*>(ws);
  float* nlse2 = reinterpret_cast<float*>(ws + rows);
  float* dq_acc = reinterpret_cast<float*>(ws + 2 * rows);
  char* kv = ws + 2 * rows + align256((size_t)B * S_Q * H * d * sizeof(float));
  const size_t kvb = block_kv_bytes(S_KV, n_blocks, H_kv, d);
  void* k_blk = kv;
  void* v_blk = kv + kvb;
  void* dk_blk = kv + 2 * kvb;
  void* dv_blk = kv + 3 * kvb;
  const int N = H_kv * d;
  cudaError_t e = launch_bwd_pre(out, dout, lse, ND, nlse2, dq_acc, B, H, S_Q, d, dt, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(dw_k, 0, (size_t)d_embed * N * sizeof(float), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(dw_v, 0, (size_t)d_embed * N * sizeof(float), s);
  if (e != cudaSuccess) return LVX_ERR_CUDA;
  const size_t q_b = (size_t)S_Q * H * d;   // elements of one batch's q, dout, dq_acc
  for (int b = 0; b < B && e == cudaSuccess; ++b) {
    for (int i = 0; i < n_blocks && e == cudaSuccess; ++i) {
      const int k0 = i * p.block_len;
      if (k0 >= S_KV) break;   // empty trailing blocks contribute nothing
      const int len = S_KV - k0 < p.block_len ? S_KV - k0 : p.block_len;
      const void* y_b = reinterpret_cast<const char*>(y) + ((size_t)b * S_KV + k0) * d_embed * 2;
      void* dy_b = reinterpret_cast<char*>(dy) + ((size_t)b * S_KV + k0) * d_embed * 2;
      const Problem pb = make_problem(1, H, H_kv, S_Q, len, d, 1, 0, scale);
      const char* qp = reinterpret_cast<const char*>(q) + q_b * 2 * b;
      const char* dop = reinterpret_cast<const char*>(dout) + q_b * 2 * b;
      e = launch_kv_gemm_tc(y_b, w_k, w_v, k_blk, v_blk, len, d_embed, N, s);
      if (e != cudaSuccess) break;
      // the block's gradients with the global log-sum-exp (rows of batch b)
      if (tc)
        e = launch_bwd_tc(pb, qp, k_blk, v_blk, dop, nlse2 + (size_t)b * H * S_Q,
                          ND + (size_t)b * H * S_Q, dq_acc + q_b * b, dk_blk, dv_blk, false, s);
      else
        e = launch_bwd_simt(pb, dt, qp, k_blk, v_blk, dop, lse + (size_t)b * H * S_Q,
                            ND + (size_t)b * H * S_Q, dq_acc + q_b * b, dk_blk, dv_blk, false, s);
      if (e == cudaSuccess) e = launch_dy_tc(w_k, w_v, dk_blk, dv_blk, dy_b, len, d_embed, N, s);
      if (e == cudaSuccess)
        e = launch_dw_accumulate_tc(y_b, dk_blk, dv_blk, dw_k, dw_v, len, d_embed, N, s);
    }
  }
  if (e == cudaSuccess)
    e = launch_dq_finalize(dq_acc, dq, (size_t)B * S_Q * H * d, p.scale, dt, false, s);
  return e == cudaSuccess ? LVX_OK : LVX_ERR_CUDA;
}

}  // extern "C"
