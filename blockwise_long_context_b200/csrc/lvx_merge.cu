// Memory-bound kernels: the merge of block partials, the backward
// preprocessing (D = rowsum(dO o O), dQ accumulator reset) and the dQ
// finalisation.
//
// Merge (LV-XAttn review page, "What carries the argument" and Figure 3 /
// Algorithm 1: partial outputs O_i and statistics L_i rescaled as in
// FlashAttention):  M = max_i L_i,  L = M + ln sum_i exp(L_i - M),
// O = sum_i exp(L_i - L) O_i.  Each thread owns 8 consecutive elements of one
// (row, head): two 128-bit loads per partial, one 128-bit (bf16) or two
// (fp32) stores; the per-row weights are recomputed by each of the row's
// threads from the n statistics (broadcast loads).
#include "lvx_common.cuh"

namespace lvx {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <typename T> struct Store8;
template <> struct Store8<float> {
  static __device__ __forceinline__ void run(float* dst, const float* x) {
    reinterpret_cast<float4*>(dst)[0] = make_float4(x[0], x[1], x[2], x[3]);
    reinterpret_cast<float4*>(dst)[1] = make_float4(x[4], x[5], x[6], x[7]);
  }
};
template <> struct Store8<__nv_bfloat16> {
  static __device__ __forceinline__ void run(__nv_bfloat16* dst, const float* x) {
    uint4 u;
    __nv_bfloat162 t0 = __floats2bfloat162_rn(x[0], x[1]);
    __nv_bfloat162 t1 = __floats2bfloat162_rn(x[2], x[3]);
    __nv_bfloat162 t2 = __floats2bfloat162_rn(x[4], x[5]);
    __nv_bfloat162 t3 = __floats2bfloat162_rn(x[6], x[7]);
    u.x = *reinterpret_cast<uint32_t*>(&t0);
    u.y = *reinterpret_cast<uint32_t*>(&t1);
    u.z = *reinterpret_cast<uint32_t*>(&t2);
    u.w = *reinterpret_cast<uint32_t*>(&t3);
    *reinterpret_cast<uint4*>(dst) = u;
  }
};

template <typename T> struct Load8;
template <> struct Load8<float> {
  static __device__ __forceinline__ void run(const float* src, float* x) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(src));
    const float4 b = __ldg(reinterpret_cast<const float4*>(src) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
};
template <> struct Load8<__nv_bfloat16> {
  static __device__ __forceinline__ void run(const __nv_bfloat16* src, float* x) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(src));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 t = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
      float2 f = __bfloat1622float2(t);
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
};

// Rows are enumerated in [B, H, S_Q] order, 8 elements per thread.
template <typename T>
__global__ void __launch_bounds__(256)
merge_kernel(const float* __restrict__ o_parts, const float* __restrict__ l_parts,
             T* __restrict__ out, float* __restrict__ lse, int n, int B, int H, int S_Q,
             int d, int causal, int block_len) {
  const int tpr = d / 8;
  const size_t rows = (size_t)B * H * S_Q;
  const size_t stride_part = rows * d;
  for (size_t gid = (size_t)blockIdx.x * blockDim.x + threadIdx.x; gid < rows * tpr;
       gid += (size_t)gridDim.x * blockDim.x) {
    const size_t row = gid / tpr;
    const int c0 = (int)(gid % tpr) * 8;
    const int r = (int)(row % S_Q);
    const int bh = (int)(row / S_Q);
    const int b = bh / H, h = bh % H;
    const int nb = causal ? min(n, r / block_len + 1) : n;
    float M = -INFINITY;
    for (int i = 0; i < nb; ++i) M = fmaxf(M, __ldg(l_parts + i * rows + row));
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float L = -INFINITY;
    if (M != -INFINITY) {
      const float M2 = M * kLog2e;
      float tot = 0.f;
      for (int i = 0; i < nb; ++i) tot += exp2f(__ldg(l_parts + i * rows + row) * kLog2e - M2);
      const float inv = 1.f / tot;
      for (int i = 0; i < nb; ++i) {
        const float w = exp2f(__ldg(l_parts + i * rows + row) * kLog2e - M2) * inv;
        if (w == 0.f) continue;
        float x[8];
        Load8<float>::run(o_parts + i * stride_part + row * d + c0, x);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, x[e], acc[e]);
      }
      L = M + log2f(tot) * kLn2;
    }
    Store8<T>::run(out + (((size_t)b * S_Q + r) * H + h) * d + c0, acc);
    if (c0 == 0) lse[row] = L;
  }
}

// ND[b,h,r] = -sum_c dO[b,r,h,c] * O[b,r,h,c] (minus D of the gradient) and
// NLSE2[b,h,r] = -LSE[b,h,r] * log2(e) (the tensor-core backward exponentiates with
// exp2 and adds both with packed FMAs); also clears dq_acc.  Rows are
// taken in memory order [B, S_Q, H]; a row's d/8 threads form an aligned
// power-of-two lane group of one warp and reduce with xor shuffles.
template <typename T>
__global__ void __launch_bounds__(256)
bwd_pre_kernel(const T* __restrict__ out, const T* __restrict__ dout, const float* __restrict__ lse,
               float* __restrict__ ND, float* __restrict__ nlse2, float* __restrict__ dq_acc, int B,
               int H, int S_Q, int d) {
  const int tpr = d / 8;
  int G = 1;
  while (G < tpr) G <<= 1;
  const int rows_per_warp = 32 / G;
  const size_t rows = (size_t)B * S_Q * H;
  const int lane = threadIdx.x & 31;
  const size_t warp_id = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const size_t n_warps = ((size_t)gridDim.x * blockDim.x) >> 5;
  const int sub = lane % G;
  for (size_t rbase = warp_id * rows_per_warp; rbase < rows; rbase += n_warps * rows_per_warp) {
    const size_t row = rbase + lane / G;
    float part = 0.f;
    if (row < rows && sub < tpr) {
      const int c0 = sub * 8;
      float a[8], bb[8];
      Load8<T>::run(out + row * d + c0, a);
      Load8<T>::run(dout + row * d + c0, bb);
#pragma unroll
      for (int e = 0; e < 8; ++e) part = fmaf(a[e], bb[e], part);
      const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      Store8<float>::run(dq_acc + row * d + c0, z);
    }
    for (int o = 1; o < G; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (row < rows && sub == 0) {
      const int h = (int)(row % H);
      const size_t bs = row / H;
      const int r = (int)(bs % S_Q), b = (int)(bs / S_Q);
      const size_t o = ((size_t)b * H + h) * S_Q + r;
      ND[o] = -part;
      nlse2[o] = -lse[o] * kLog2e;
    }
  }
}

// ACC: dq (float32) += scale * acc; otherwise dq = scale * acc in T.
template <typename T, bool ACC>
__global__ void __launch_bounds__(256)
dq_finalize_kernel(const float* __restrict__ acc, T* __restrict__ dq, size_t count8, float scale) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < count8;
       i += (size_t)gridDim.x * blockDim.x) {
    float x[8];
    Load8<float>::run(acc + i * 8, x);
    if constexpr (ACC) {
      float y[8];
      Load8<float>::run(reinterpret_cast<const float*>(dq) + i * 8, y);
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = fmaf(x[e], scale, y[e]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] *= scale;
    }
    Store8<T>::run(dq + i * 8, x);
  }
}

// The partial of an empty key block: O = 0, L = -inf (the merge's identity).
__global__ void __launch_bounds__(256)
empty_partial_kernel(float* __restrict__ o, float* __restrict__ l, size_t rows, int d) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows * d; i += stride)
    o[i] = 0.f;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows; i += stride)
    l[i] = -INFINITY;
}

int grid_for(size_t work, int threads) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const size_t want = (work + threads - 1) / threads;
  const size_t cap = (size_t)sms * 16;
  return (int)(want < cap ? (want ? want : 1) : cap);
}

}  // namespace

cudaError_t launch_merge(const float* o_parts, const float* l_parts, void* out, float* lse,
                         int n, int B, int H, int S_Q, int d, int causal, int block_len,
                         lvx_dtype dt, cudaStream_t s) {
  const size_t work = (size_t)B * H * S_Q * (d / 8);
  const int grid = grid_for(work, 256);
  if (dt == LVX_FP32)
    merge_kernel<float><<<grid, 256, 0, s>>>(o_parts, l_parts, (float*)out, lse, n, B, H, S_Q, d,
                                             causal, block_len);
  else
    merge_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(o_parts, l_parts, (__nv_bfloat16*)out, lse,
                                                     n, B, H, S_Q, d, causal, block_len);
  return cudaGetLastError();
}

cudaError_t launch_bwd_pre(const void* out, const void* dout, const float* lse, float* ND,
                           float* nlse2, float* dq_acc, int B, int H, int S_Q, int d, lvx_dtype dt,
                           cudaStream_t s) {
  const size_t work = (size_t)B * H * S_Q * (d / 8);
  const int grid = grid_for(work, 256);
  if (dt == LVX_FP32)
    bwd_pre_kernel<float><<<grid, 256, 0, s>>>((const float*)out, (const float*)dout, lse, ND, nlse2,
                                               dq_acc, B, H, S_Q, d);
  else
    bwd_pre_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>((const __nv_bfloat16*)out,
                                                       (const __nv_bfloat16*)dout, lse, ND, nlse2,
                                                       dq_acc, B, H, S_Q, d);
  return cudaGetLastError();
}

cudaError_t launch_empty_partial(float* o_part, float* l_part, size_t rows, int d, cudaStream_t s) {
  empty_partial_kernel<<<grid_for(rows * d, 256), 256, 0, s>>>(o_part, l_part, rows, d);
  return cudaGetLastError();
}

cudaError_t launch_dq_finalize(const float* dq_acc, void* dq, size_t count, float scale,
                               lvx_dtype dt, bool accum, cudaStream_t s) {
  const size_t count8 = count / 8;
  const int grid = grid_for(count8, 256);
  if (accum)
    dq_finalize_kernel<float, true><<<grid, 256, 0, s>>>(dq_acc, (float*)dq, count8, scale);
  else if (dt == LVX_FP32)
    dq_finalize_kernel<float, false><<<grid, 256, 0, s>>>(dq_acc, (float*)dq, count8, scale);
  else
    dq_finalize_kernel<__nv_bfloat16, false><<<grid, 256, 0, s>>>(dq_acc, (__nv_bfloat16*)dq,
                                                                 count8, scale);
  return cudaGetLastError();
}

}  // namespace lvx
