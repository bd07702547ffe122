#include "lvx_tc.cuh"
namespace lvx {
bool tc_fwd_supported(const Problem&) { return false; }
cudaError_t launch_fwd_tc(const Problem&, const void*, const void*, const void*, void*, float*,
                          float*, float*, cudaStream_t) { return cudaErrorNotSupported; }
bool tc_bwd_supported(const Problem&) { return false; }
cudaError_t launch_bwd_tc(const Problem&, const void*, const void*, const void*, const void*,
                          const float*, const float*, float*, void*, void*, cudaStream_t) {
  return cudaErrorNotSupported;
}
bool tc_gemm_supported(int, int, int) { return false; }
cudaError_t launch_kv_gemm_tc(const void*, const void*, const void*, void*, void*, int, int, int,
                              cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace lvx
