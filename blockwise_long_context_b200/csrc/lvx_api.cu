// The C ABI of liblvx.so: argument validation, workspace layout and kernel
// dispatch.  No entry point allocates, frees or synchronises (except
// lvx_last_device_error); every launch goes to the caller's stream.
#include <math.h>
#include <stdint.h>

#include "lvx_common.cuh"
#include "lvx_tc.cuh"

namespace lvx {

__device__ unsigned int g_error_word = 0;

unsigned int* device_error_word() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_error_word) != cudaSuccess) return nullptr;
  return reinterpret_cast<unsigned int*>(ptr);
}

lvx_status check_shapes(int B, int H, int H_kv, int S_Q, int S_KV, int d, int n_blocks,
                        int causal, lvx_dtype dt) {
  if (B < 1 || H < 1 || H_kv < 1 || S_Q < 1 || S_KV < 1 || d < 1 || n_blocks < 1)
    return LVX_ERR_INVALID_ARG;
  if (H % H_kv != 0 || n_blocks > S_KV) return LVX_ERR_INVALID_ARG;
  if (dt != LVX_FP32 && dt != LVX_BF16) return LVX_ERR_UNSUPPORTED;
  if (d > 128 || d % 8 != 0) return LVX_ERR_UNSUPPORTED;
  if (causal && S_Q != S_KV) return LVX_ERR_UNSUPPORTED;
  if (n_blocks > 65535 || (long long)B * H > 65535) return LVX_ERR_UNSUPPORTED;
  return LVX_OK;
}

Problem make_problem(int B, int H, int H_kv, int S_Q, int S_KV, int d, int n_blocks,
                     int causal, float scale) {
  Problem p;
  p.B = B; p.H = H; p.H_kv = H_kv; p.S_Q = S_Q; p.S_KV = S_KV; p.d = d;
  p.n_blocks = n_blocks;
  p.block_len = (S_KV + n_blocks - 1) / n_blocks;
  p.causal = causal ? 1 : 0;
  p.scale = scale > 0.f ? scale : 1.0f / sqrtf((float)d);
  p.scale_log2 = p.scale * 1.4426950408889634f;
  return p;
}

size_t fwd_parts_o_bytes(int B, int H, int S_Q, int d, int n) {
  return align256((size_t)n * B * H * S_Q * d * sizeof(float));
}
size_t fwd_parts_l_bytes(int B, int H, int S_Q, int n) {
  return align256((size_t)n * B * H * S_Q * sizeof(float));
}

cudaError_t run_attn_fwd(const Problem& p, lvx_dtype dt, const void* q, const void* k,
                         const void* v, void* out, float* lse, float* o_parts, float* l_parts,
                         cudaStream_t s) {
  if (p.n_blocks == 1) o_parts = l_parts = nullptr;   // one block: the output directly
  cudaError_t e;
  if (dt == LVX_BF16 && tc_fwd_supported(p)) {
    e = launch_fwd_tc(p, q, k, v, out, lse, o_parts, l_parts, s);
  } else {
    e = launch_fwd_simt(p, dt, q, k, v, out, lse, o_parts, l_parts, s);
  }
  if (e != cudaSuccess || p.n_blocks == 1) return e;
  return launch_merge(o_parts, l_parts, out, lse, p.n_blocks, p.B, p.H, p.S_Q, p.d, p.causal,
                      p.block_len, dt, s);
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

lvx_status from_cuda(cudaError_t e) { return e == cudaSuccess ? LVX_OK : LVX_ERR_CUDA; }

}  // namespace
}  // namespace lvx

using namespace lvx;

extern "C" {

const char* lvx_status_string(lvx_status s) {
  switch (s) {
    case LVX_OK: return "LVX_OK";
    case LVX_ERR_INVALID_ARG: return "LVX_ERR_INVALID_ARG";
    case LVX_ERR_UNSUPPORTED: return "LVX_ERR_UNSUPPORTED";
    case LVX_ERR_WORKSPACE: return "LVX_ERR_WORKSPACE";
    case LVX_ERR_CUDA: return "LVX_ERR_CUDA";
    case LVX_ERR_DEVICE_TIMEOUT: return "LVX_ERR_DEVICE_TIMEOUT";
  }
  return "LVX_ERR_UNKNOWN";
}

int lvx_version(void) { return 100; }

size_t lvx_attn_fwd_workspace(int B, int H, int H_kv, int S_Q, int S_KV, int d, int n_blocks,
                              int causal, lvx_dtype dt) {
  if (check_shapes(B, H, H_kv, S_Q, S_KV, d, n_blocks, causal, dt) != LVX_OK) return 0;
  if (n_blocks == 1) return 0;
  return fwd_parts_o_bytes(B, H, S_Q, d, n_blocks) + fwd_parts_l_bytes(B, H, S_Q, n_blocks);
}

lvx_status lvx_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                        int B, int H, int H_kv, int S_Q, int S_KV, int d, int n_blocks,
                        int causal, lvx_dtype dt, float scale, void* workspace,
                        size_t ws_bytes, lvx_stream stream) {
  lvx_status st = check_shapes(B, H, H_kv, S_Q, S_KV, d, n_blocks, causal, dt);
  if (st != LVX_OK) return st;
  if (!q || !k || !v || !out || !lse) return LVX_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return LVX_ERR_INVALID_ARG;
  const size_t need = lvx_attn_fwd_workspace(B, H, H_kv, S_Q, S_KV, d, n_blocks, causal, dt);
  if (need > 0 && (!workspace || !aligned16(workspace))) return LVX_ERR_INVALID_ARG;
  if (ws_bytes < need) return LVX_ERR_WORKSPACE;
  if (!(scale == scale)) return LVX_ERR_INVALID_ARG;   // NaN scale

  const Problem p = make_problem(B, H, H_kv, S_Q, S_KV, d, n_blocks, causal, scale);
  float* o_parts = nullptr;
  float* l_parts = nullptr;
  if (n_blocks > 1) {
    o_parts = reinterpret_cast<float*>(workspace);
    l_parts = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) +
                                       fwd_parts_o_bytes(B, H, S_Q, d, n_blocks));
  }
  return from_cuda(run_attn_fwd(p, dt, q, k, v, out, lse, o_parts, l_parts,
                                reinterpret_cast<cudaStream_t>(stream)));
}

lvx_status lvx_attn_fwd_partials(const void* q, const void* k, const void* v, float* O_parts,
                                 float* L_parts, int B, int H, int H_kv, int S_Q, int S_KV, int d,
                                 int n_blocks, int causal, lvx_dtype dt, float scale,
                                 lvx_stream stream) {
  lvx_status st = check_shapes(B, H, H_kv, S_Q, S_KV, d, n_blocks, causal, dt);
  if (st != LVX_OK) return st;
  if (!q || !k || !v || !O_parts || !L_parts) return LVX_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(O_parts) || !aligned16(L_parts))
    return LVX_ERR_INVALID_ARG;
  if (!(scale == scale)) return LVX_ERR_INVALID_ARG;   // NaN scale
  const Problem p = make_problem(B, H, H_kv, S_Q, S_KV, d, n_blocks, causal ? 1 : 0, scale);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // with a partials buffer the kernels write (O_i, L_i) of every block (with a
  // mask: of every block a row sees) and never touch the final-output pointers
  cudaError_t e;
  if (dt == LVX_BF16 && tc_fwd_supported(p))
    e = launch_fwd_tc(p, q, k, v, nullptr, nullptr, O_parts, L_parts, s);
  else
    e = launch_fwd_simt(p, dt, q, k, v, nullptr, nullptr, O_parts, L_parts, s);
  return from_cuda(e);
}

lvx_status lvx_merge_partials(const float* O_parts, const float* L_parts, void* out, float* lse,
                              int n, int B, int H, int S_Q, int d, lvx_dtype dt,
                              lvx_stream stream) {
  if (n < 1 || B < 1 || H < 1 || S_Q < 1 || d < 1) return LVX_ERR_INVALID_ARG;
  if (dt != LVX_FP32 && dt != LVX_BF16) return LVX_ERR_UNSUPPORTED;
  if (d > 128 || d % 8 != 0) return LVX_ERR_UNSUPPORTED;
  if (!O_parts || !L_parts || !out || !lse) return LVX_ERR_INVALID_ARG;
  if (!aligned16(O_parts) || !aligned16(out) || !aligned16(L_parts) || !aligned16(lse))
    return LVX_ERR_INVALID_ARG;
  return from_cuda(launch_merge(O_parts, L_parts, out, lse, n, B, H, S_Q, d, 0, S_Q, dt,
                                reinterpret_cast<cudaStream_t>(stream)));
}

size_t lvx_attn_bwd_workspace(int B, int H, int H_kv, int S_Q, int S_KV, int d, int causal,
                              lvx_dtype dt) {
  if (check_shapes(B, H, H_kv, S_Q, S_KV, d, 1, causal, dt) != LVX_OK) return 0;
  return 2 * align256((size_t)B * H * S_Q * sizeof(float)) +
         align256((size_t)B * S_Q * H * d * sizeof(float));
}

namespace {

// The backward with its gradients written (accum = false: dq, dk, dv in dtype
// dt) or added to float32 arrays (accum = true).
lvx_status attn_bwd(const void* q, const void* k, const void* v, const void* out,
                    const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                    int H, int H_kv, int S_Q, int S_KV, int d, int causal, lvx_dtype dt,
                    float scale, void* workspace, size_t ws_bytes, bool accum,
                    lvx_stream stream) {
  lvx_status st = check_shapes(B, H, H_kv, S_Q, S_KV, d, 1, causal, dt);
  if (st != LVX_OK) return st;
  const void* ptrs[] = {q, k, v, out, lse, dout, dq, dk, dv, workspace};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return LVX_ERR_INVALID_ARG;
  if (ws_bytes < lvx_attn_bwd_workspace(B, H, H_kv, S_Q, S_KV, d, causal, dt))
    return LVX_ERR_WORKSPACE;
  if (!(scale == scale)) return LVX_ERR_INVALID_ARG;
  const Problem p = make_problem(B, H, H_kv, S_Q, S_KV, d, 1, causal, scale);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t row_bytes = align256((size_t)B * H * S_Q * sizeof(float));
  float* ND = reinterpret_cast<float*>(workspace);
  float* nlse2 = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + row_bytes);
  float* dq_acc = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + 2 * row_bytes);
  cudaError_t e = launch_bwd_pre(out, dout, lse, ND, nlse2, dq_acc, B, H, S_Q, d, dt, s);
  if (e != cudaSuccess) return LVX_ERR_CUDA;
  if (dt == LVX_BF16 && tc_bwd_supported(p))
    e = launch_bwd_tc(p, q, k, v, dout, nlse2, ND, dq_acc, dk, dv, accum, s);
  else
    e = launch_bwd_simt(p, dt, q, k, v, dout, lse, ND, dq_acc, dk, dv, accum, s);
  if (e != cudaSuccess) return LVX_ERR_CUDA;
  return from_cuda(
      launch_dq_finalize(dq_acc, dq, (size_t)B * S_Q * H * d, p.scale, dt, accum, s));
}

}  // namespace

lvx_status lvx_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                        const float* lse, const void* dout, void* dq, void* dk, void* dv,
                        int B, int H, int H_kv, int S_Q, int S_KV, int d, int causal,
                        lvx_dtype dt, float scale, void* workspace, size_t ws_bytes,
                        lvx_stream stream) {
  return attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, H, H_kv, S_Q, S_KV, d, causal, dt, scale,
                  workspace, ws_bytes, false, stream);
}

lvx_status lvx_attn_bwd_accumulate(const void* q, const void* k, const void* v, const void* out,
                                   const float* lse, const void* dout, float* dq, float* dk,
                                   float* dv, int B, int H, int H_kv, int S_Q, int S_KV, int d,
                                   int causal, lvx_dtype dt, float scale, void* workspace,
                                   size_t ws_bytes, lvx_stream stream) {
  return attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, H, H_kv, S_Q, S_KV, d, causal, dt, scale,
                  workspace, ws_bytes, true, stream);
}

lvx_status lvx_kv_recompute(const void* y, const void* w_k, const void* w_v, void* k, void* v,
                            int B, int S_KV, int d_embed, int H_kv, int d, lvx_dtype dt,
                            lvx_stream stream) {
  if (B < 1 || S_KV < 1 || d_embed < 1 || H_kv < 1 || d < 1) return LVX_ERR_INVALID_ARG;
  if (dt != LVX_FP32 && dt != LVX_BF16) return LVX_ERR_UNSUPPORTED;
  const void* ptrs[] = {y, w_k, w_v, k, v};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return LVX_ERR_INVALID_ARG;
  if ((long long)B * S_KV > (1ll << 31) - 1 || (long long)H_kv * d > (1 << 30))
    return LVX_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int M = B * S_KV, N = H_kv * d, K = d_embed;
  cudaError_t e;
  if (dt == LVX_BF16 && tc_gemm_supported(M, K, N)) {
    e = launch_kv_gemm_tc(y, w_k, w_v, k, v, M, K, N, s);
  } else {
    // K = y W_k, V = y W_v: A = y (row stride K), B = W (row stride N)
    SimtGemm g{{y, nullptr}, {w_k, nullptr}, k, (size_t)K, 1, (size_t)N, 1, M, N, K, 1};
    e = launch_gemm_simt(g, dt, s);
    if (e == cudaSuccess) {
      g.B[0] = w_v;
      g.C = v;
      e = launch_gemm_simt(g, dt, s);
    }
  }
  return from_cuda(e);
}

lvx_status lvx_kv_recompute_bwd(const void* y, const void* w_k, const void* w_v, const void* dk,
                                const void* dv, void* dy, void* dw_k, void* dw_v, int B, int S_KV,
                                int d_embed, int H_kv, int d, lvx_dtype dt, lvx_stream stream) {
  if (B < 1 || S_KV < 1 || d_embed < 1 || H_kv < 1 || d < 1) return LVX_ERR_INVALID_ARG;
  if (dt != LVX_FP32 && dt != LVX_BF16) return LVX_ERR_UNSUPPORTED;
  const void* ptrs[] = {y, w_k, w_v, dk, dv, dy, dw_k, dw_v};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return LVX_ERR_INVALID_ARG;
  if ((long long)B * S_KV > (1ll << 31) - 1 || (long long)H_kv * d > (1 << 30))
    return LVX_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int S = B * S_KV, E = d_embed, N = H_kv * d;
  cudaError_t e;
  if (dt == LVX_BF16 && tc_gemm_bwd_supported(S, E, N)) {
    e = launch_kv_gemm_bwd_tc(y, w_k, w_v, dk, dv, dy, dw_k, dw_v, S, E, N, s);
  } else {
    // dW_k = y^T dK: A(m=e, k=s) = y[s][e], B(k=s, n) = dK[s][n]
    SimtGemm g{{y, nullptr}, {dk, nullptr}, dw_k, 1, (size_t)E, (size_t)N, 1, E, N, S, 1};
    e = launch_gemm_simt(g, dt, s);
    if (e == cudaSuccess) {
      g.B[0] = dv;
      g.C = dw_v;
      e = launch_gemm_simt(g, dt, s);
    }
    if (e == cudaSuccess) {
      // dy = dK W_k^T + dV W_v^T: A(m=s, k=n) = dZ[s][n], B(k=n, n'=e) = W_z[e][n]
      SimtGemm h{{dk, dv}, {w_k, w_v}, dy, (size_t)N, 1, 1, (size_t)N, S, E, N, 2};
      e = launch_gemm_simt(h, dt, s);
    }
  }
  return from_cuda(e);
}

lvx_status lvx_last_device_error(lvx_stream stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return LVX_ERR_CUDA;
  unsigned int word = 0;
  e = cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word));
  if (e != cudaSuccess) return LVX_ERR_CUDA;
  if (word != 0) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return LVX_ERR_CUDA;
    return LVX_ERR_DEVICE_TIMEOUT;
  }
  return LVX_OK;
}

}  // extern "C"
