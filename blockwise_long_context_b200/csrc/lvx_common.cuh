// Shared definitions for the liblvx kernels: problem descriptor, element
// conversion, the device error word.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "lvx.h"

namespace lvx {

// One attention problem, as validated by the C ABI layer.
struct Problem {
  int B, H, H_kv, S_Q, S_KV, d;
  int n_blocks;     // key/value blocks (forward partials)
  int block_len;    // ceil(S_KV / n_blocks)
  int causal;
  float scale;      // softmax scale (natural-log domain)
  float scale_log2; // scale * log2(e): logits are exponentiated with exp2
};

// Kernels that wait on barriers receive a pointer to the library's device
// error word (defined next to lvx_last_device_error) and record the first
// expired wait there.

enum : unsigned int {
  kErrNone = 0,
  kErrTimeoutTma = 1,
  kErrTimeoutMma = 2,
  kErrTimeoutSoftmax = 3,
  kErrTimeoutEpilogue = 4,
  kErrSmemAlign = 5,
  kErrSelftestTimeout = 6,
};

__device__ __forceinline__ void record_error(unsigned int* word, unsigned int code) {
  atomicCAS(word, 0u, code);
}

// Address of the error word on the current device (host side).
unsigned int* device_error_word();

template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float x) { return x; }
  static __device__ __forceinline__ float from_f(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// Offsets of the two forward workspace parts (bytes).
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Argument checks, problem set-up and dispatch shared by the forward entry
// points (defined in lvx_api.cu).
lvx_status check_shapes(int B, int H, int H_kv, int S_Q, int S_KV, int d, int n_blocks,
                        int causal, lvx_dtype dt);
Problem make_problem(int B, int H, int H_kv, int S_Q, int S_KV, int d, int n_blocks, int causal,
                     float scale);
// Bytes of the two parts of the forward workspace: O_i [n,B,H,S_Q,d] fp32,
// then L_i [n,B,H,S_Q] fp32, each rounded up to 256 bytes.
size_t fwd_parts_o_bytes(int B, int H, int S_Q, int d, int n);
size_t fwd_parts_l_bytes(int B, int H, int S_Q, int n);
// The forward of a validated problem: block partials into o_parts / l_parts
// and their merge (with one block, the output directly; the partials are then
// unused and may be null).
cudaError_t run_attn_fwd(const Problem& p, lvx_dtype dt, const void* q, const void* k,
                         const void* v, void* out, float* lse, float* o_parts, float* l_parts,
                         cudaStream_t s);

// Launchers implemented in the kernel translation units.  Each returns the
// cudaError_t of its launch.
cudaError_t launch_fwd_simt(const Problem& p, lvx_dtype dt, const void* q, const void* k,
                            const void* v, void* out, float* lse, float* o_parts,
                            float* l_parts, cudaStream_t s);
cudaError_t launch_merge(const float* o_parts, const float* l_parts, void* out, float* lse,
                         int n, int B, int H, int S_Q, int d, int causal, int block_len,
                         lvx_dtype dt, cudaStream_t s);
cudaError_t launch_bwd_pre(const void* out, const void* dout, const float* lse, float* ND,
                           float* nlse2, float* dq_acc, int B, int H, int S_Q, int d, lvx_dtype dt,
                           cudaStream_t s);
// accum: dk, dv are float32 arrays the gradients are added to
cudaError_t launch_bwd_simt(const Problem& p, lvx_dtype dt, const void* q, const void* k,
                            const void* v, const void* dout, const float* lse, const float* ND,
                            float* dq_acc, void* dk, void* dv, bool accum, cudaStream_t s);
// The partial of an empty key block, (O, L) = (0, -inf), over `rows` rows.
cudaError_t launch_empty_partial(float* o_part, float* l_part, size_t rows, int d, cudaStream_t s);
// dq = scale * dq_acc in dtype dt, or with accum dq (float32) += scale * dq_acc
cudaError_t launch_dq_finalize(const float* dq_acc, void* dq, size_t count, float scale,
                               lvx_dtype dt, bool accum, cudaStream_t s);
// C [M][N] row-major = sum over `segments` (1 or 2) of A_g B_g, where element
// (m, k) of A_g is A[g][m*sam + k*sak] and element (k, n) of B_g is
// B[g][k*sbk + n*sbn]; every segment has the same K.
struct SimtGemm {
  const void* A[2];
  const void* B[2];
  void* C;
  size_t sam, sak, sbk, sbn;
  int M, N, K, segments;
};
cudaError_t launch_gemm_simt(const SimtGemm& g, lvx_dtype dt, cudaStream_t s);

}  // namespace lvx
