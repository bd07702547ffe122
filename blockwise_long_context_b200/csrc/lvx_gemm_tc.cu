// K/V recomputation from the shared visual features on the tcgen05 tensor
// cores: K = y W_k and V = y W_v in one launch (LV-XAttn review page,
// "What carries the argument" and Figure 6: one copy of y is kept and the
// keys/values are regenerated from it).
//
// Tile: 128 rows of y x 256 output columns, K step 64.  TMA brings the y tile
// (K-major, 128-byte swizzle) and four 64x64 boxes of W (N-major, 128-byte
// swizzle) into a 4-stage ring; one thread issues tcgen05.mma (M=128, N=256,
// K=16) into a 256-column fp32 TMEM accumulator; the four warps then read
// the accumulator (one 32-lane quarter each), round to bf16 and store.
#include "lvx_ptx.cuh"
#include "lvx_tc.cuh"

namespace lvx {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr uint32_t A_BYTES = BM * BK * 2;          // 16 KiB
constexpr uint32_t B_BOX_BYTES = BK * 64 * 2;      // 8 KiB: 64 K-rows x 64 N
constexpr uint32_t B_BYTES = 4 * B_BOX_BYTES;      // 32 KiB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t IDESC = ptx::idesc_bf16_f32(BM, BN, false, true);

struct GemmArgs {
  __nv_bfloat16* out_k;
  __nv_bfloat16* out_v;
  unsigned int* err;
  int M, K, N;   // N = columns of each weight
};

__global__ void __launch_bounds__(128, 1)
kv_gemm_kernel(const __grid_constant__ CUtensorMap map_y, const __grid_constant__ CUtensorMap map_wk,
               const __grid_constant__ CUtensorMap map_wv, GemmArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles_per_w = args.N / BN;
  const bool is_v = blockIdx.x >= n_tiles_per_w;
  const int n0 = (blockIdx.x % n_tiles_per_w) * BN;
  const int m0 = blockIdx.y * BM;
  const int kblocks = args.K / BK;
  const CUtensorMap* map_w = is_v ? &map_wv : &map_wk;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(acc_full, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::tma_prefetch_desc(&map_y);
    ptx::tma_prefetch_desc(map_w);
  }
  if (warp == 2) {
    ptx::tmem_alloc(tmem_slot, BN);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // producer
    int issued = 0;
    for (int kb = 0; kb < kblocks; ++kb) {
      const int s = kb % STAGES;
      const uint32_t round = kb / STAGES;
      if (!ptx::mbar_wait(&empty[s], (round & 1) ^ 1, args.err, kErrTimeoutTma, abort_flag)) break;
      uint8_t* a = smem + s * STAGE_BYTES;
      uint8_t* b = a + A_BYTES;
      ptx::mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
      ptx::tma_load_2d(a, &map_y, &full[s], kb * BK, m0);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        ptx::tma_load_2d(b + j * B_BOX_BYTES, map_w, &full[s], n0 + 64 * j, kb * BK);
      issued = kb + 1;
    }
    if (*abort_flag) {
      // let the copies already issued land before the CTA's shared memory is released
      for (int kb = issued > STAGES ? issued - STAGES : 0; kb < issued; ++kb)
        ptx::mbar_wait(&full[kb % STAGES], (kb / STAGES) & 1, args.err, kErrTimeoutTma, nullptr);
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer
    for (int kb = 0; kb < kblocks; ++kb) {
      const int s = kb % STAGES;
      const uint32_t round = kb / STAGES;
      if (!ptx::mbar_wait(&full[s], round & 1, args.err, kErrTimeoutMma, abort_flag)) break;
      ptx::tc_fence_after();
      const uint32_t a = ptx::smem_u32(smem + s * STAGE_BYTES);
      const uint32_t b = a + A_BYTES;
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk) {
        const uint64_t da = ptx::smem_desc_sw128(a + kk * 32, 16, 1024);
        const uint64_t db = ptx::smem_desc_sw128(b + kk * 16 * 128, B_BOX_BYTES, 1024);
        ptx::mma_ss(tmem, da, db, IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
      }
      ptx::mma_commit(&empty[s]);
    }
    ptx::mma_commit(acc_full);
  }
  __syncwarp();

  // epilogue: every warp reads its 32-lane quarter of the accumulator.  The
  // MMA thread always commits acc_full (also after an abort), so this wait
  // also drains the MMAs before the TMEM is released.
  const bool ok = ptx::mbar_wait(acc_full, 0, args.err, kErrTimeoutEpilogue, nullptr);
  ptx::tc_fence_after();
  if (ok && !*abort_flag) {
    const int row = m0 + warp * 32 + lane;
    __nv_bfloat16* out = is_v ? args.out_v : args.out_k;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t r[32];
      ptx::tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c * 32, r);
      ptx::tmem_wait_ld();
      if (row < args.M) {
        uint4* dst = reinterpret_cast<uint4*>(out + (size_t)row * args.N + n0 + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 u;
          u.x = ptx::pack_bf16x2(__uint_as_float(r[8 * q + 0]), __uint_as_float(r[8 * q + 1]));
          u.y = ptx::pack_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3]));
          u.z = ptx::pack_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5]));
          u.w = ptx::pack_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7]));
          dst[q] = u;
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) ptx::tmem_dealloc(tmem, BN);
}

}  // namespace

bool tc_gemm_supported(int M, int K, int N) {
  return M >= 1 && K >= BK && K % BK == 0 && N % BN == 0;
}

cudaError_t launch_kv_gemm_tc(const void* y, const void* w_k, const void* w_v, void* k, void* v,
                              int M, int K, int N, cudaStream_t s) {
  CUtensorMap my, mk, mv;
  {
    const uint64_t dims[2] = {(uint64_t)K, (uint64_t)M};
    const uint64_t strides[1] = {(uint64_t)K * 2};
    const uint32_t box[2] = {BK, BM};
    if (!encode_tensor_map(&my, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {(uint64_t)N, (uint64_t)K};
    const uint64_t strides[1] = {(uint64_t)N * 2};
    const uint32_t box[2] = {64, BK};
    if (!encode_tensor_map(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_k, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tensor_map(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_v, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(kv_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       SMEM_BYTES);
  if (e != cudaSuccess) return e;
  GemmArgs args{reinterpret_cast<__nv_bfloat16*>(k), reinterpret_cast<__nv_bfloat16*>(v),
                device_error_word(), M, K, N};
  if (!args.err) return cudaErrorInvalidValue;
  dim3 grid(2 * (N / BN), (M + BM - 1) / BM);
  kv_gemm_kernel<<<grid, 128, SMEM_BYTES, s>>>(my, mk, mv, args);
  return cudaGetLastError();
}

}  // namespace lvx
