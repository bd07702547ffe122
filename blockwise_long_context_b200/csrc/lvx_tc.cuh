// Tensor-core (tcgen05 + TMA) kernels for sm_100a: entry points used by the
// C ABI layer.
#pragma once

#include "lvx_common.cuh"

namespace lvx {

// Forward partials / final output with tcgen05 MMAs (bf16 inputs, d in {64, 128}).
bool tc_fwd_supported(const Problem& p);
cudaError_t launch_fwd_tc(const Problem& p, const void* q, const void* k, const void* v,
                          void* out, float* lse, float* o_parts, float* l_parts, cudaStream_t s);

// Backward (dK, dV written in the input dtype, or with accum added to float32
// arrays; dQ accumulated unscaled into dq_acc).  nlse2 is minus the forward's
// log-sum-exp times log2(e); nd is minus rowsum(dO o O).
bool tc_bwd_supported(const Problem& p);
cudaError_t launch_bwd_tc(const Problem& p, const void* q, const void* k, const void* v,
                          const void* dout, const float* nlse2, const float* nd, float* dq_acc,
                          void* dk, void* dv, bool accum, cudaStream_t s);

// K = y W_k and V = y W_v in one launch (bf16, fp32 accumulation).
bool tc_gemm_supported(int M, int K, int N);
cudaError_t launch_kv_gemm_tc(const void* y, const void* w_k, const void* w_v, void* k, void* v,
                              int M, int K, int N, cudaStream_t s);

// Gradients of the recomputation: dW_k = y^T dK and dW_v = y^T dV in one
// launch, then dy = dK W_k^T + dV W_v^T.  y [S][E], W [E][N], dK/dV [S][N].
bool tc_gemm_bwd_supported(int S, int E, int N);
cudaError_t launch_kv_gemm_bwd_tc(const void* y, const void* w_k, const void* w_v,
                                  const void* dk, const void* dv, void* dy, void* dw_k, void* dw_v,
                                  int S, int E, int N, cudaStream_t s);

// Pieces of the key-block-at-a-time recomputation: dW_k += y^T dK and
// dW_v += y^T dV added to float32 arrays (one launch), and dy = dK W_k^T +
// dV W_v^T written in bf16.  Same shapes and support as launch_kv_gemm_bwd_tc.
cudaError_t launch_dw_accumulate_tc(const void* y, const void* dk, const void* dv, float* dw_k,
                                    float* dw_v, int S, int E, int N, cudaStream_t s);
cudaError_t launch_dy_tc(const void* w_k, const void* w_v, const void* dk, const void* dv,
                         void* dy, int S, int E, int N, cudaStream_t s);

}  // namespace lvx
