// lvx_attn_fwd_noalloc: the forward pass for callers that cannot allocate
// device memory.
//
// lvx_attn_fwd needs a caller-provided workspace for the per-block partials
// (O_i, L_i) whenever n_blocks > 1.  Some callers have no way to provide one:
// code running where cudaMalloc is forbidden or unavailable (for example a
// real-time or embedded runtime whose device memory is fixed at start-up, a
// plug-in loaded into a host program that owns every device allocation, or
// a caller that must not trigger an allocator's synchronisation in its
// latency-critical path).  This entry point takes the same inputs and
// outputs but keeps the partials in one fixed, file-scope device array
// instead, so it allocates nothing at all.
//
// Properties of the fixed array:
//   * its size is kNoAllocScratchBytes (64 MiB); a problem whose partials
//     need more is rejected with LVX_ERR_WORKSPACE before anything runs;
//   * every GPU that loads this library holds the array until the process
//     exits;
//   * all calls on a device share it and it keeps the last call's contents.
//     Nothing in it has to start at zero (every partial the merge reads is
//     written by the same call first), but two calls whose kernels overlap
//     on the GPU (different streams, no ordering between them) race on it.
// The device address of the array is looked up with cudaGetSymbolAddress on
// the first call on each device (with that device current) and cached; that
// first call should come before any stream capture.
#include <mutex>

#include "lvx_common.cuh"
#include "lvx_tc.cuh"

namespace lvx {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (host code must
// not use the symbol itself: on the host it names a stand-in, not device memory).
cudaError_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace lvx

using namespace lvx;

extern "C" lvx_status lvx_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                           float* lse, int B, int H, int H_kv, int S_Q, int S_KV,
                                           int d, int n_blocks, int causal, lvx_dtype dt,
                                           float scale, lvx_stream stream) {
  if (B < 1 || H < 1 || H_kv < 1 || S_Q < 1 || S_KV < 1 || d < 1 || n_blocks < 1)
    return LVX_ERR_INVALID_ARG;
  if (H % H_kv != 0 || n_blocks > S_KV) return LVX_ERR_INVALID_ARG;
  if (dt != LVX_FP32 && dt != LVX_BF16) return LVX_ERR_UNSUPPORTED;
  if (d > 128 || d % 8 != 0) return LVX_ERR_UNSUPPORTED;
  if (causal && S_Q != S_KV) return LVX_ERR_UNSUPPORTED;
  if (n_blocks > 65535 || (long long)B * H > 65535) return LVX_ERR_UNSUPPORTED;
  if (!q || !k || !v || !out || !lse) return LVX_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return LVX_ERR_INVALID_ARG;
  if (!(scale == scale)) return LVX_ERR_INVALID_ARG;

  // same partial layout as the lvx_attn_fwd workspace: O parts, then L parts
  const size_t o_bytes = round256((size_t)n_blocks * B * H * S_Q * d * sizeof(float));
  const size_t l_bytes = round256((size_t)n_blocks * B * H * S_Q * sizeof(float));
  if (n_blocks > 1 && o_bytes + l_bytes > kNoAllocScratchBytes) return LVX_ERR_WORKSPACE;

  Problem p;
  p.B = B; p.H = H; p.H_kv = H_kv; p.S_Q = S_Q; p.S_KV = S_KV; p.d = d;
  p.n_blocks = n_blocks;
  p.block_len = (S_KV + n_blocks - 1) / n_blocks;
  p.causal = causal ? 1 : 0;
  p.scale = scale > 0.f ? scale : 1.0f / sqrtf((float)d);
  p.scale_log2 = p.scale * 1.4426950408889634f;

  float* o_parts = nullptr;
  float* l_parts = nullptr;
  if (n_blocks > 1) {
    void* base = nullptr;
    if (scratch_address(&base) != cudaSuccess) return LVX_ERR_CUDA;
    o_parts = reinterpret_cast<float*>(base);
    l_parts = reinterpret_cast<float*>(reinterpret_cast<char*>(base) + o_bytes);
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = (dt == LVX_BF16 && tc_fwd_supported(p))
                      ? launch_fwd_tc(p, q, k, v, out, lse, o_parts, l_parts, s)
                      : launch_fwd_simt(p, dt, q, k, v, out, lse, o_parts, l_parts, s);
  if (e != cudaSuccess) return LVX_ERR_CUDA;
  if (n_blocks > 1)
    e = launch_merge(o_parts, l_parts, out, lse, n_blocks, B, H, S_Q, d, p.causal, p.block_len,
                     dt, s);
  return e == cudaSuccess ? LVX_OK : LVX_ERR_CUDA;
}
