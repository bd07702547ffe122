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
// The device address of the array is looked up with cudaGetSymbolAddress the
// first time the entry point runs in a CUDA context (the device's primary
// context, normally) with that context current, and cached per context, so
// a context created later (after cudaDeviceReset, say) looks it up afresh.
// That first call should come before any stream capture.
#include <cuda.h>

#include <mutex>

#include "lvx_common.cuh"
#include "lvx_tc.cuh"

namespace lvx {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
constexpr int kMaxContexts = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

std::mutex g_scratch_mu;
CtxGetCurrentFn g_ctx_current = nullptr;
CtxGetIdFn g_ctx_id = nullptr;
bool g_resolved = false;
// (context id, device address of g_noalloc_scratch in that context)
unsigned long long g_ctx_ids[kMaxContexts] = {};
void* g_ctx_addr[kMaxContexts] = {};
int g_n_ctx = 0;

template <typename F>
F driver_fn(const char* name) {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<F>(fn);
}

// Device address of g_noalloc_scratch in the current context (host code must
// not use the symbol itself: on the host it names a stand-in, not device memory).
cudaError_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);   // also makes the device's primary context current
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_resolved) {
    g_ctx_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    g_ctx_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    g_resolved = true;
  }
  unsigned long long id = 0;
  CUcontext ctx = nullptr;
  const bool keyed = g_ctx_current && g_ctx_id && g_ctx_current(&ctx) == CUDA_SUCCESS && ctx &&
                     g_ctx_id(ctx, &id) == CUDA_SUCCESS;
  if (keyed) {
    for (int i = 0; i < g_n_ctx; ++i) {
      if (g_ctx_ids[i] == id) {
        *out = g_ctx_addr[i];
        return cudaSuccess;
      }
    }
  }
  void* ptr = nullptr;
  e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  if (keyed && g_n_ctx < kMaxContexts) {   // else: looked up on every call
    g_ctx_ids[g_n_ctx] = id;
    g_ctx_addr[g_n_ctx] = ptr;
    ++g_n_ctx;
  }
  *out = ptr;
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace lvx

using namespace lvx;

extern "C" lvx_status lvx_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                           float* lse, int B, int H, int H_kv, int S_Q, int S_KV,
                                           int d, int n_blocks, int causal, lvx_dtype dt,
                                           float scale, lvx_stream stream) {
  // the same checks, problem and dispatch as lvx_attn_fwd; only the partials'
  // home differs
  lvx_status st = check_shapes(B, H, H_kv, S_Q, S_KV, d, n_blocks, causal, dt);
  if (st != LVX_OK) return st;
  if (!q || !k || !v || !out || !lse) return LVX_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return LVX_ERR_INVALID_ARG;
  if (!(scale == scale)) return LVX_ERR_INVALID_ARG;

  // same partial layout as the lvx_attn_fwd workspace: O parts, then L parts
  const size_t o_bytes = fwd_parts_o_bytes(B, H, S_Q, d, n_blocks);
  const size_t l_bytes = fwd_parts_l_bytes(B, H, S_Q, n_blocks);
  if (n_blocks > 1 && o_bytes + l_bytes > kNoAllocScratchBytes) return LVX_ERR_WORKSPACE;

  const Problem p = make_problem(B, H, H_kv, S_Q, S_KV, d, n_blocks, causal, scale);
  float* o_parts = nullptr;
  float* l_parts = nullptr;
  if (n_blocks > 1) {
    void* base = nullptr;
    if (scratch_address(&base) != cudaSuccess) return LVX_ERR_CUDA;
    o_parts = reinterpret_cast<float*>(base);
    l_parts = reinterpret_cast<float*>(reinterpret_cast<char*>(base) + o_bytes);
  }
  const cudaError_t e = run_attn_fwd(p, dt, q, k, v, out, lse, o_parts, l_parts,
                                     reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LVX_OK : LVX_ERR_CUDA;
}
