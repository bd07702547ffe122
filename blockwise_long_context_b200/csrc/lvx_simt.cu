// CUDA-core kernels: the fp32 path of the forward and backward passes (and
// the bf16 path for head widths the tensor-core kernels do not take).
//
// Forward: each CTA (8 warps) owns 8 query rows of one (batch, head) and one
// key/value block i, and produces that block's partial (O_i, L_i) with an fp32
// online softmax over 32-key tiles staged in shared memory (Ring Attention
// citation hub page, abstract: blockwise exact attention; LV-XAttn review
// page, Figure 3 / Algorithm 1: per-block partials).
//
// Backward: each CTA (2 warps, 16 keys per warp) owns 32 keys of one
// (batch, key/value head) and sweeps every query row of every query head of
// that group, recomputing P from the stored log-sum-exp; dK and dV stay in
// registers, dQ is accumulated with fp32 atomics into a workspace buffer.
#include "lvx_common.cuh"

#include <math.h>

namespace lvx {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

constexpr int kFwdRows = 8;    // query rows per CTA (one per warp)
constexpr int kFwdKeys = 32;   // keys per shared-memory tile (one per lane)
constexpr int kMaxD = 128;

template <typename T>
__global__ void __launch_bounds__(256)
fwd_simt_kernel(Problem p, const T* __restrict__ q, const T* __restrict__ k,
                const T* __restrict__ v, T* __restrict__ out, float* __restrict__ lse,
                float* __restrict__ o_parts, float* __restrict__ l_parts) {
  __shared__ float qs[kFwdRows][kMaxD];
  __shared__ float ks[kFwdKeys][kMaxD + 1];
  __shared__ float vs[kFwdKeys][kMaxD];

  const int d = p.d;
  const int blk = blockIdx.z;
  const int b = blockIdx.y / p.H, h = blockIdx.y % p.H;
  const int g = h / (p.H / p.H_kv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = blockIdx.x * kFwdRows;
  const int r = r0 + warp;

  const int kb0 = min(blk * p.block_len, p.S_KV);
  const int kb1 = min(kb0 + p.block_len, p.S_KV);
  bool row_active = r < p.S_Q;
  int kend_row = kb1;
  int kend_cta = kb1;
  if (p.causal) {
    if (r < p.S_Q && blk > r / p.block_len) row_active = false;   // block pair skipped
    kend_row = min(kb1, r + 1);
    kend_cta = min(kb1, min(r0 + kFwdRows, p.S_Q));
  }

  for (int i = threadIdx.x; i < kFwdRows * d; i += blockDim.x) {
    const int rr = r0 + i / d, c = i % d;
    qs[i / d][c] = rr < p.S_Q ? Elem<T>::to_f(q[(((size_t)b * p.S_Q + rr) * p.H + h) * d + c]) : 0.f;
  }

  float m_run = -INFINITY, l_run = 0.f;
  float o[4] = {0.f, 0.f, 0.f, 0.f};

  for (int kt = kb0; kt < kend_cta; kt += kFwdKeys) {
    __syncthreads();
    for (int i = threadIdx.x; i < kFwdKeys * d; i += blockDim.x) {
      const int jj = i / d, c = i % d, j = kt + jj;
      float kx = 0.f, vx = 0.f;
      if (j < kb1) {
        const size_t off = (((size_t)b * p.S_KV + j) * p.H_kv + g) * d + c;
        kx = Elem<T>::to_f(k[off]);
        vx = Elem<T>::to_f(v[off]);
      }
      ks[jj][c] = kx;
      vs[jj][c] = vx;
    }
    __syncthreads();
    if (!row_active) continue;
    const int j = kt + lane;
    float s = -INFINITY;
    if (j < kend_row) {
      float acc = 0.f;
      for (int c = 0; c < d; ++c) acc = fmaf(qs[warp][c], ks[lane][c], acc);
      s = acc * p.scale_log2;
    }
    const float m_new = fmaxf(m_run, warp_max(s));
    if (m_new == -INFINITY) continue;
    const float alpha = exp2f(m_run - m_new);
    const float pj = exp2f(s - m_new);
    l_run = l_run * alpha + warp_sum(pj);
#pragma unroll
    for (int t = 0; t < 4; ++t) o[t] *= alpha;
    for (int jj = 0; jj < kFwdKeys; ++jj) {
      const float pb = __shfl_sync(0xffffffffu, pj, jj);
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int c = lane + 32 * t;
        if (c < d) o[t] = fmaf(pb, vs[jj][c], o[t]);
      }
    }
    m_run = m_new;
  }

  if (!row_active) return;
  const bool seen = m_run != -INFINITY;
  const float inv_l = seen ? 1.f / l_run : 0.f;
  const float L = seen ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
  if (o_parts == nullptr) {   // the final output (one block), else the block partials
    for (int t = 0; t < 4; ++t) {
      const int c = lane + 32 * t;
      if (c < d) out[(((size_t)b * p.S_Q + r) * p.H + h) * d + c] = Elem<T>::from_f(o[t] * inv_l);
    }
    if (lane == 0) lse[((size_t)b * p.H + h) * p.S_Q + r] = L;
  } else {
    const size_t row = (((size_t)blk * p.B + b) * p.H + h) * p.S_Q + r;
    for (int t = 0; t < 4; ++t) {
      const int c = lane + 32 * t;
      if (c < d) o_parts[row * d + c] = o[t] * inv_l;
    }
    if (lane == 0) l_parts[row] = L;
  }
}

// ---------------------------------------------------------------- backward

constexpr int kBwdWarps = 2;
constexpr int kBwdKeysPerWarp = 16;
constexpr int kBwdKeys = kBwdWarps * kBwdKeysPerWarp;

// TO is the dK / dV element type: T, written; or float with ACC, added to.
template <typename T, typename TO, bool ACC>
__global__ void __launch_bounds__(128)
bwd_simt_kernel(Problem p, const T* __restrict__ q, const T* __restrict__ k,
                const T* __restrict__ v, const T* __restrict__ dout,
                const float* __restrict__ lse, const float* __restrict__ ND,
                float* __restrict__ dq_acc, TO* __restrict__ dk, TO* __restrict__ dv) {
  __shared__ float ks[kBwdKeys][kMaxD];
  __shared__ float vs[kBwdKeys][kMaxD];
  const int d = p.d;
  const int b = blockIdx.y / p.H_kv, g = blockIdx.y % p.H_kv;
  const int grp = p.H / p.H_kv;
  const int k0 = blockIdx.x * kBwdKeys;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int i = threadIdx.x; i < kBwdKeys * d; i += blockDim.x) {
    const int jj = i / d, c = i % d, j = k0 + jj;
    float kx = 0.f, vx = 0.f;
    if (j < p.S_KV) {
      const size_t off = (((size_t)b * p.S_KV + j) * p.H_kv + g) * d + c;
      kx = Elem<T>::to_f(k[off]);
      vx = Elem<T>::to_f(v[off]);
    }
    ks[jj][c] = kx;
    vs[jj][c] = vx;
  }
  __syncthreads();

  float dk_acc[kBwdKeysPerWarp][4], dv_acc[kBwdKeysPerWarp][4];
#pragma unroll
  for (int jj = 0; jj < kBwdKeysPerWarp; ++jj)
#pragma unroll
    for (int t = 0; t < 4; ++t) dk_acc[jj][t] = dv_acc[jj][t] = 0.f;

  const int jw = warp * kBwdKeysPerWarp;          // first key of this warp, tile-relative
  const int r_begin = p.causal ? min(k0 + jw, p.S_Q) : 0;
  const float lse_scale = kLog2e;

  for (int hh = 0; hh < grp; ++hh) {
    const int h = g * grp + hh;
    for (int r = r_begin; r < p.S_Q; ++r) {
      const size_t roff = (((size_t)b * p.S_Q + r) * p.H + h) * d;
      float qv[4], dov[4], dqv[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int c = lane + 32 * t;
        qv[t] = c < d ? Elem<T>::to_f(q[roff + c]) : 0.f;
        dov[t] = c < d ? Elem<T>::to_f(dout[roff + c]) : 0.f;
        dqv[t] = 0.f;
      }
      const float L2 = lse[((size_t)b * p.H + h) * p.S_Q + r] * lse_scale;
      const float NDr = ND[((size_t)b * p.H + h) * p.S_Q + r];   // minus rowsum(dO o O)
#pragma unroll
      for (int jj = 0; jj < kBwdKeysPerWarp; ++jj) {
        const int j = k0 + jw + jj;
        float sdot = 0.f, pdot = 0.f;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int c = lane + 32 * t;
          if (c < d) {
            sdot = fmaf(qv[t], ks[jw + jj][c], sdot);
            pdot = fmaf(dov[t], vs[jw + jj][c], pdot);
          }
        }
        sdot = warp_sum(sdot);
        pdot = warp_sum(pdot);
        const bool visible = j < p.S_KV && (!p.causal || j <= r);
        const float P = visible ? exp2f(sdot * p.scale_log2 - L2) : 0.f;
        const float dS = P * (pdot + NDr);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int c = lane + 32 * t;
          dv_acc[jj][t] = fmaf(P, dov[t], dv_acc[jj][t]);
          dk_acc[jj][t] = fmaf(dS, qv[t], dk_acc[jj][t]);
          if (c < d) dqv[t] = fmaf(dS, ks[jw + jj][c], dqv[t]);
        }
      }
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int c = lane + 32 * t;
        if (c < d && dqv[t] != 0.f) atomicAdd(&dq_acc[roff + c], dqv[t]);
      }
    }
  }
#pragma unroll
  for (int jj = 0; jj < kBwdKeysPerWarp; ++jj) {
    const int j = k0 + jw + jj;
    if (j >= p.S_KV) continue;
    const size_t off = (((size_t)b * p.S_KV + j) * p.H_kv + g) * d;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int c = lane + 32 * t;
      if (c < d) {
        if constexpr (ACC) {
          dk[off + c] += dk_acc[jj][t] * p.scale;
          dv[off + c] += dv_acc[jj][t];
        } else {
          dk[off + c] = Elem<T>::from_f(dk_acc[jj][t] * p.scale);
          dv[off + c] = Elem<T>::from_f(dv_acc[jj][t]);
        }
      }
    }
  }
}

// ---------------------------------------------------------------- GEMM (K/V recompute fallback)

// C[m][n] = sum over the segments g of sum_k A_g[m][k] B_g[k][n], with A_g and
// B_g addressed through element strides so that transposed operands need no
// copy.  64x64 output tile per block, 4x4 per thread, fp32 accumulation.
template <typename T>
__global__ void __launch_bounds__(256)
gemm_simt_kernel(SimtGemm g) {
  __shared__ float As[16][64 + 1];
  __shared__ float Bs[16][64];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int n_tiles = (g.N + 63) / 64;   // tiles run along N first (A-tile reuse in L2)
  const int m0 = (int)(blockIdx.x / n_tiles) * 64, n0 = (int)(blockIdx.x % n_tiles) * 64;
  float acc[4][4] = {};
  for (int seg = 0; seg < g.segments; ++seg) {
    const T* a_ptr = static_cast<const T*>(seg ? g.A[1] : g.A[0]);
    const T* b_ptr = static_cast<const T*>(seg ? g.B[1] : g.B[0]);
    for (int k0 = 0; k0 < g.K; k0 += 16) {
      for (int i = threadIdx.x; i < 64 * 16; i += 256) {
        const int mm = i / 16, kk = i % 16;
        const int gm = m0 + mm, gk = k0 + kk;
        As[kk][mm] = (gm < g.M && gk < g.K)
                         ? Elem<T>::to_f(a_ptr[(size_t)gm * g.sam + (size_t)gk * g.sak]) : 0.f;
        const int kb = i / 64, nb = i % 64;
        const int gk2 = k0 + kb, gn = n0 + nb;
        Bs[kb][nb] = (gk2 < g.K && gn < g.N)
                         ? Elem<T>::to_f(b_ptr[(size_t)gk2 * g.sbk + (size_t)gn * g.sbn]) : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) {
        float a[4], bb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) bb[j] = Bs[kk][tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
      }
      __syncthreads();
    }
  }
  T* C = reinterpret_cast<T*>(g.C);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gm = m0 + ty * 4 + i, gn = n0 + tx * 4 + j;
      if (gm < g.M && gn < g.N) C[(size_t)gm * g.N + gn] = Elem<T>::from_f(acc[i][j]);
    }
}

}  // namespace

cudaError_t launch_fwd_simt(const Problem& p, lvx_dtype dt, const void* q, const void* k,
                            const void* v, void* out, float* lse, float* o_parts,
                            float* l_parts, cudaStream_t s) {
  dim3 grid((p.S_Q + kFwdRows - 1) / kFwdRows, p.B * p.H, p.n_blocks);
  if (dt == LVX_FP32)
    fwd_simt_kernel<float><<<grid, 256, 0, s>>>(p, (const float*)q, (const float*)k,
                                                (const float*)v, (float*)out, lse, o_parts, l_parts);
  else
    fwd_simt_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        p, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
        (__nv_bfloat16*)out, lse, o_parts, l_parts);
  return cudaGetLastError();
}

cudaError_t launch_bwd_simt(const Problem& p, lvx_dtype dt, const void* q, const void* k,
                            const void* v, const void* dout, const float* lse, const float* ND,
                            float* dq_acc, void* dk, void* dv, bool accum, cudaStream_t s) {
  dim3 grid((p.S_KV + kBwdKeys - 1) / kBwdKeys, p.B * p.H_kv);
  using bf = __nv_bfloat16;
  const unsigned nt = 32 * kBwdWarps;
  if (dt == LVX_FP32) {
    const float *qq = (const float*)q, *kk = (const float*)k, *vv = (const float*)v,
                *dd = (const float*)dout;
    if (accum)
      bwd_simt_kernel<float, float, true><<<grid, nt, 0, s>>>(p, qq, kk, vv, dd, lse, ND, dq_acc,
                                                              (float*)dk, (float*)dv);
    else
      bwd_simt_kernel<float, float, false><<<grid, nt, 0, s>>>(p, qq, kk, vv, dd, lse, ND, dq_acc,
                                                               (float*)dk, (float*)dv);
  } else {
    const bf *qq = (const bf*)q, *kk = (const bf*)k, *vv = (const bf*)v, *dd = (const bf*)dout;
    if (accum)
      bwd_simt_kernel<bf, float, true><<<grid, nt, 0, s>>>(p, qq, kk, vv, dd, lse, ND, dq_acc,
                                                           (float*)dk, (float*)dv);
    else
      bwd_simt_kernel<bf, bf, false><<<grid, nt, 0, s>>>(p, qq, kk, vv, dd, lse, ND, dq_acc,
                                                         (bf*)dk, (bf*)dv);
  }
  return cudaGetLastError();
}

cudaError_t launch_gemm_simt(const SimtGemm& g, lvx_dtype dt, cudaStream_t s) {
  if (g.M < 1 || g.N < 1) return cudaSuccess;
  const long long tiles = (long long)((g.N + 63) / 64) * ((g.M + 63) / 64);
  if (tiles > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  const dim3 grid((unsigned)tiles);
  if (dt == LVX_FP32)
    gemm_simt_kernel<float><<<grid, 256, 0, s>>>(g);
  else
    gemm_simt_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(g);
  return cudaGetLastError();
}

}  // namespace lvx
