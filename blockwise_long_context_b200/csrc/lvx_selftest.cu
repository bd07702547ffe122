// Self-test of the bounded waits: a kernel waits on an mbarrier that nothing
// ever completes.  The wait must give up after its time limit, record the
// timeout in the library's device error word and return, leaving the CUDA
// context usable.  This is how every tensor-core kernel of the library
// behaves when one of its internal waits expires.
#include "lvx_ptx.cuh"

namespace lvx {
namespace {

__global__ void selftest_wait_kernel(unsigned int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    ptx::fence_barrier_init();
  }
  __syncthreads();
  // no thread arrives on `bar`: phase 0 never completes
  ptx::mbar_wait(&bar, 0, err, kErrSelftestTimeout, nullptr);
}

}  // namespace
}  // namespace lvx

extern "C" lvx_status lvx_selftest_wait_timeout(lvx_stream stream) {
  unsigned int* err = lvx::device_error_word();
  if (!err) return LVX_ERR_CUDA;
  lvx::selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(err);
  return cudaGetLastError() == cudaSuccess ? LVX_OK : LVX_ERR_CUDA;
}
