// K/V recomputation from the shared visual features and its gradients on
// the tcgen05 tensor cores (LV-XAttn review page, "What carries the argument"
// and Figure 6: one copy of the visual features y is kept and the keys and
// values are regenerated from it; training needs the gradients of that map).
//   forward:   K = y W_k,  V = y W_v                 (A = y K-major, B = W N-major)
//   gradient:  dW_k = y^T dK,  dW_v = y^T dV          (A = y M-major, B = dK N-major)
//              dy = dK W_k^T + dV W_v^T               (A = dK K-major, B = W K-major,
//                                                      two K segments summed)
// All three share one mainloop: tile 128 x 256 outputs, K step 64, a 4-stage
// TMA ring (128-byte swizzle; K-major tiles are 64-element rows along K,
// M/N-major tiles are 64-element rows along M/N), and one thread issuing
// tcgen05.mma (M=128, N=256, K=16) into a 256-column fp32 TMEM accumulator.
// In batched mode a launch holds two independent problems (forward K and V,
// or dW_k and dW_v); in segment mode a single problem's K loop runs over two
// (A, B) pairs.  Two kernels around it:
//  - gemm_tc_persistent (bf16 outputs): one CTA per SM takes output tiles
//    round-robin, the accumulator is double-buffered in TMEM (2 x 256
//    columns), and four epilogue warps round tile i to bf16 and store it
//    while the MMAs of tile i+1 run, so neither the epilogue nor a CTA's
//    start-up sits between two tiles' MMAs;
//  - gemm_tc_kernel (float32 outputs the tile is added to, used when dW is
//    summed over the key blocks of a recomputing backward): one tile per CTA,
//    each row staged in the freed pipeline buffers and added with one bulk
//    reduce-add.
#include "lvx_ptx.cuh"
#include "lvx_tc.cuh"

namespace lvx {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr uint32_t A_BYTES = BM * BK * 2;          // 16 KiB
constexpr uint32_t B_BYTES = BN * BK * 2;          // 32 KiB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;

struct GemmArgs {
  __nv_bfloat16* out[2];   // [M][N] row-major, per problem
  float* acc[2];           // if set: float32 [M][N] the tile is added to instead
  unsigned int* err;
  int M, N;
  int kb_seg0;             // k-blocks taken from (A0, B0); the rest from (A1, B1)
  int kb_total;            // k-blocks per output tile
  int batched;             // 1: two problems (A_z, B_z) -> out[z]; 0: two K segments -> out[0]
};

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(128, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap map_a0, const __grid_constant__ CUtensorMap map_b0,
               const __grid_constant__ CUtensorMap map_a1, const __grid_constant__ CUtensorMap map_b1,
               GemmArgs args) {
  constexpr uint32_t IDESC = ptx::idesc_bf16_f32(BM, BN, A_MN, B_MN);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Tile order: N tiles fastest, then the problem, then M, so that the CTAs
  // resident together share their A tile (and, when batched, A is the same
  // matrix y for both problems) and it is read from HBM about once.
  const int n_tiles = args.N / BN;
  const int problems = args.batched ? 2 : 1;
  const int n0 = (int)(blockIdx.x % n_tiles) * BN;
  const int z = (int)(blockIdx.x / n_tiles) % problems;
  const int m0 = (int)(blockIdx.x / (n_tiles * problems)) * BM;

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
    ptx::tma_prefetch_desc(args.batched && z ? &map_a1 : &map_a0);
    ptx::tma_prefetch_desc(args.batched && z ? &map_b1 : &map_b0);
    if (!args.batched) {
      ptx::tma_prefetch_desc(&map_a1);
      ptx::tma_prefetch_desc(&map_b1);
    }
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
    // ------------------------------------------------------------------ producer
    int issued = 0;
    for (int kb = 0; kb < args.kb_total; ++kb) {
      const int s = kb % STAGES;
      const uint32_t round = kb / STAGES;
      if (!ptx::mbar_wait(&empty[s], (round & 1) ^ 1, args.err, kErrTimeoutTma, abort_flag)) break;
      const bool second = z == 1 || kb >= args.kb_seg0;
      const CUtensorMap* ma = second ? &map_a1 : &map_a0;
      const CUtensorMap* mb = second ? &map_b1 : &map_b0;
      const int k0 = (kb >= args.kb_seg0 && !args.batched ? kb - args.kb_seg0 : kb) * BK;
      uint8_t* a = smem + s * STAGE_BYTES;
      uint8_t* b = a + A_BYTES;
      ptx::mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
      if (A_MN) {   // A stored [K][M]: two 64-wide M chunks of 64 K rows
        ptx::tma_load_2d(a, ma, &full[s], m0, k0);
        ptx::tma_load_2d(a + 8192, ma, &full[s], m0 + 64, k0);
      } else {      // A stored [M][K]: 128 rows of 64 K
        ptx::tma_load_2d(a, ma, &full[s], k0, m0);
      }
      if (B_MN) {   // B stored [K][N]: four 64-wide N chunks of 64 K rows
#pragma unroll
        for (int j = 0; j < 4; ++j) ptx::tma_load_2d(b + j * 8192, mb, &full[s], n0 + 64 * j, k0);
      } else {      // B stored [N][K]: 256 rows of 64 K
        ptx::tma_load_2d(b, mb, &full[s], k0, n0);
      }
      issued = kb + 1;
    }
    if (*abort_flag) {
      // let the copies already issued land before the CTA's shared memory is released
      for (int kb = issued > STAGES ? issued - STAGES : 0; kb < issued; ++kb)
        ptx::mbar_wait(&full[kb % STAGES], (kb / STAGES) & 1, args.err, kErrTimeoutTma, nullptr);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------------ MMA issuer
    for (int kb = 0; kb < args.kb_total; ++kb) {
      const int s = kb % STAGES;
      const uint32_t round = kb / STAGES;
      if (!ptx::mbar_wait(&full[s], round & 1, args.err, kErrTimeoutMma, abort_flag)) break;
      ptx::tc_fence_after();
      const uint32_t a = ptx::smem_u32(smem + s * STAGE_BYTES);
      const uint32_t b = a + A_BYTES;
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk) {
        const uint64_t da = A_MN ? ptx::smem_desc_sw128(a + kk * 2048, 8192, 1024)
                                 : ptx::smem_desc_sw128(a + kk * 32, 16, 1024);
        const uint64_t db = B_MN ? ptx::smem_desc_sw128(b + kk * 2048, 8192, 1024)
                                 : ptx::smem_desc_sw128(b + kk * 32, 16, 1024);
        ptx::mma_ss(tmem, da, db, IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
      }
      ptx::mma_commit(&empty[s]);
    }
    ptx::mma_commit(acc_full);
  }
  __syncwarp();

  // ------------------------------------------------------------------ epilogue
  // Every warp reads its 32-lane quarter of the accumulator.  The MMA thread
  // always commits acc_full (also after an abort), so this wait also drains
  // the MMAs before the TMEM is released.
  const bool ok = ptx::mbar_wait(acc_full, 0, args.err, kErrTimeoutEpilogue, nullptr);
  ptx::tc_fence_after();
  if (ok && !*abort_flag) {
    // float32 rows added to the output: staged with a row pitch of 1040 bytes
    // (the 16-byte stores of a quarter-warp then fall in different banks) in
    // the pipeline buffers, which the MMAs no longer read, then one bulk
    // reduce-add of 1 KiB per row
    constexpr uint32_t PITCH = BN * 4 + 16;
    static_assert(BM * PITCH <= STAGES * STAGE_BYTES, "staging fits the pipeline buffers");
    const int rloc = warp * 32 + lane;
    const int row = m0 + rloc;
    uint8_t* stg = smem + rloc * PITCH;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t r[32];
      ptx::tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c * 32, r);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 8; ++q)
        *reinterpret_cast<uint4*>(stg + c * 128 + q * 16) =
            make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
    }
    ptx::fence_proxy_async_smem();
    if (row < args.M) {
      float* dst = (z ? args.acc[1] : args.acc[0]) + (size_t)row * args.N + n0;
      asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(
                       reinterpret_cast<uint64_t>(dst)),
                   "r"(ptx::smem_u32(stg)), "r"((uint32_t)(BN * 4))
                   : "memory");
      ptx::bulk_commit();
      ptx::bulk_wait_read();   // the staging must stay until the copy has read it
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) ptx::tmem_dealloc(tmem, BN);
}

// Persistent form (bf16 outputs only).  Warp roles: 0 TMA producer, 1 MMA
// issuer, 2 TMEM allocator, 4..7 epilogue (warp 4 + q reads TMEM lanes
// [32q, 32q + 32)).  The stage ring runs on across tiles; accumulator buffer
// i & 1 of the CTA's i-th tile is released by its 128 epilogue threads.
template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(256, 1)
gemm_tc_persistent(const __grid_constant__ CUtensorMap map_a0, const __grid_constant__ CUtensorMap map_b0,
                   const __grid_constant__ CUtensorMap map_a1, const __grid_constant__ CUtensorMap map_b1,
                   GemmArgs args, int n_tiles_total) {
  constexpr uint32_t IDESC = ptx::idesc_bf16_f32(BM, BN, A_MN, B_MN);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;    // [2]
  uint64_t* acc_empty = acc_full + 2;     // [2]
  uint64_t* mma_drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = args.N / BN;
  const int problems = args.batched ? 2 : 1;
  // tile t: N tiles fastest, then the problem, then M (the CTAs working at the
  // same time share their A tile, as in the one-tile-per-CTA form)
  auto decode = [&](int t, int& m0, int& n0, int& z) {
    n0 = (t % n_tiles) * BN;
    z = (t / n_tiles) % problems;
    m0 = (t / (n_tiles * problems)) * BM;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&acc_full[b], 1);
      ptx::mbar_init(&acc_empty[b], 128);
    }
    ptx::mbar_init(mma_drain, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 2) {
    ptx::tmem_alloc(tmem_slot, 2 * BN);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------------ producer
    ptx::tma_prefetch_desc(&map_a0);
    ptx::tma_prefetch_desc(&map_b0);
    ptx::tma_prefetch_desc(&map_a1);
    ptx::tma_prefetch_desc(&map_b1);
    int g = 0;   // k-blocks issued by this CTA
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles_total && ok; t += gridDim.x) {
      int m0, n0, z;
      decode(t, m0, n0, z);
      for (int kb = 0; kb < args.kb_total; ++kb, ++g) {
        const int s = g % STAGES;
        if (!ptx::mbar_wait(&empty[s], ((g / STAGES) & 1) ^ 1, args.err, kErrTimeoutTma, abort_flag)) {
          ok = false;
          break;
        }
        const bool second = z == 1 || kb >= args.kb_seg0;
        const CUtensorMap* ma = second ? &map_a1 : &map_a0;
        const CUtensorMap* mb = second ? &map_b1 : &map_b0;
        const int k0 = (kb >= args.kb_seg0 && !args.batched ? kb - args.kb_seg0 : kb) * BK;
        uint8_t* a = smem + s * STAGE_BYTES;
        uint8_t* b = a + A_BYTES;
        ptx::mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
        if (A_MN) {
          ptx::tma_load_2d(a, ma, &full[s], m0, k0);
          ptx::tma_load_2d(a + 8192, ma, &full[s], m0 + 64, k0);
        } else {
          ptx::tma_load_2d(a, ma, &full[s], k0, m0);
        }
        if (B_MN) {
#pragma unroll
          for (int j = 0; j < 4; ++j) ptx::tma_load_2d(b + j * 8192, mb, &full[s], n0 + 64 * j, k0);
        } else {
          ptx::tma_load_2d(b, mb, &full[s], k0, n0);
        }
      }
    }
    if (*abort_flag) {
      // the copies already issued must land before shared memory is released
      for (int q = g > STAGES ? g - STAGES : 0; q < g; ++q)
        ptx::mbar_wait(&full[q % STAGES], (q / STAGES) & 1, args.err, kErrTimeoutTma, nullptr);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------------ MMA issuer
    int g = 0, i = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles_total && ok; t += gridDim.x, ++i) {
      const int ab = i & 1;
      // the epilogue has read this buffer's previous tile (the CTA's tile i - 2)
      ok = ptx::mbar_wait(&acc_empty[ab], ((i >> 1) & 1) ^ 1, args.err, kErrTimeoutMma, abort_flag);
      for (int kb = 0; kb < args.kb_total && ok; ++kb, ++g) {
        const int s = g % STAGES;
        ok = ptx::mbar_wait(&full[s], (g / STAGES) & 1, args.err, kErrTimeoutMma, abort_flag);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t a = ptx::smem_u32(smem + s * STAGE_BYTES);
        const uint32_t b = a + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t da = A_MN ? ptx::smem_desc_sw128(a + kk * 2048, 8192, 1024)
                                   : ptx::smem_desc_sw128(a + kk * 32, 16, 1024);
          const uint64_t db = B_MN ? ptx::smem_desc_sw128(b + kk * 2048, 8192, 1024)
                                   : ptx::smem_desc_sw128(b + kk * 32, 16, 1024);
          ptx::mma_ss(tmem + ab * BN, da, db, IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::mma_commit(&empty[s]);
      }
      if (ok) ptx::mma_commit(&acc_full[ab]);
    }
    ptx::mma_commit(mma_drain);
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp - 4;
    int i = 0;
    for (int t = blockIdx.x; t < n_tiles_total; t += gridDim.x, ++i) {
      const int ab = i & 1;
      bool ok = ptx::mbar_wait(&acc_full[ab], (i >> 1) & 1, args.err, kErrTimeoutEpilogue, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      int m0, n0, z;
      decode(t, m0, n0, z);
      const int row = m0 + q * 32 + lane;
      __nv_bfloat16* out = z ? args.out[1] : args.out[0];
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        ptx::tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + ab * BN + c * 32, r);
        ptx::tmem_wait_ld();
        if (row < args.M) {
          uint4* dst = reinterpret_cast<uint4*>(out + (size_t)row * args.N + n0 + c * 32);
#pragma unroll
          for (int w4 = 0; w4 < 4; ++w4) {
            uint4 u;
            u.x = ptx::pack_bf16x2(__uint_as_float(r[8 * w4 + 0]), __uint_as_float(r[8 * w4 + 1]));
            u.y = ptx::pack_bf16x2(__uint_as_float(r[8 * w4 + 2]), __uint_as_float(r[8 * w4 + 3]));
            u.z = ptx::pack_bf16x2(__uint_as_float(r[8 * w4 + 4]), __uint_as_float(r[8 * w4 + 5]));
            u.w = ptx::pack_bf16x2(__uint_as_float(r[8 * w4 + 6]), __uint_as_float(r[8 * w4 + 7]));
            dst[w4] = u;
          }
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(&acc_empty[ab]);
    }
  }

  // ------------------------------------------------------------------ teardown
  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    ptx::mbar_wait(mma_drain, 0, args.err, kErrTimeoutEpilogue, nullptr);
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 2 * BN);
  }
}

// Tensor map of a row-major bf16 matrix [rows][cols] (cols contiguous) read in
// boxes of box_cols x box_rows.
bool map_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
            uint32_t box_rows) {
  const uint64_t dims[2] = {cols, rows};
  const uint64_t strides[1] = {cols * 2};
  const uint32_t box[2] = {box_cols, box_rows};
  return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B);
}

// Operand descriptions: base pointer and the row-major shape it is stored in.
struct Operand {
  const void* base;
  uint64_t rows, cols;
};

// A: K-major = stored [M][K]; M-major = stored [K][M].  B: K-major = stored
// [N][K]; N-major = stored [K][N].
template <bool A_MN, bool B_MN>
cudaError_t launch_gemm(const Operand* a, const Operand* b, __nv_bfloat16* out0,
                        __nv_bfloat16* out1, int M, int N, int kb_seg0, int kb_total, int batched,
                        cudaStream_t s, float* acc0 = nullptr, float* acc1 = nullptr) {
  CUtensorMap ma[2], mb[2];
  for (int i = 0; i < 2; ++i) {
    const bool okA = A_MN ? map_2d(&ma[i], a[i].base, a[i].rows, a[i].cols, 64, 64)
                          : map_2d(&ma[i], a[i].base, a[i].rows, a[i].cols, 64, 128);
    const bool okB = B_MN ? map_2d(&mb[i], b[i].base, b[i].rows, b[i].cols, 64, 64)
                          : map_2d(&mb[i], b[i].base, b[i].rows, b[i].cols, 64, 256);
    if (!okA || !okB) return cudaErrorInvalidValue;
  }
  GemmArgs g;
  g.out[0] = out0;
  g.out[1] = out1;
  g.acc[0] = acc0;
  g.acc[1] = acc1;
  g.err = device_error_word();
  g.M = M;
  g.N = N;
  g.kb_seg0 = kb_seg0;
  g.kb_total = kb_total;
  g.batched = batched;
  if (!g.err) return cudaErrorInvalidValue;
  const long long tiles = (long long)(N / BN) * ((M + BM - 1) / BM) * (batched ? 2 : 1);
  if (tiles > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  if (acc0 == nullptr) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_persistent<A_MN, B_MN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int dev = 0, n_sm = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int grid = (int)(tiles < n_sm ? tiles : n_sm);
    gemm_tc_persistent<A_MN, B_MN><<<grid, 256, SMEM_BYTES, s>>>(ma[0], mb[0], ma[1], mb[1], g,
                                                                 (int)tiles);
    return cudaGetLastError();
  }
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<A_MN, B_MN>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  gemm_tc_kernel<A_MN, B_MN><<<(unsigned)tiles, 128, SMEM_BYTES, s>>>(ma[0], mb[0], ma[1], mb[1], g);
  return cudaGetLastError();
}

}  // namespace

bool tc_gemm_supported(int M, int K, int N) {
  return M >= 1 && K >= BK && K % BK == 0 && N % BN == 0;
}

cudaError_t launch_kv_gemm_tc(const void* y, const void* w_k, const void* w_v, void* k, void* v,
                              int M, int K, int N, cudaStream_t s) {
  // K = y W_k, V = y W_v: A = y [M][K] (K-major), B = W [K][N] (N-major), two problems
  const Operand a[2] = {{y, (uint64_t)M, (uint64_t)K}, {y, (uint64_t)M, (uint64_t)K}};
  const Operand b[2] = {{w_k, (uint64_t)K, (uint64_t)N}, {w_v, (uint64_t)K, (uint64_t)N}};
  return launch_gemm<false, true>(a, b, reinterpret_cast<__nv_bfloat16*>(k),
                                  reinterpret_cast<__nv_bfloat16*>(v), M, N, K / BK, K / BK, 1, s);
}

bool tc_gemm_bwd_supported(int S, int E, int N) {
  // S = B*S_KV rows of y (any count: the last K step of dW reads zeros past
  // row S-1 from both operands), E = d_embed, N = H_kv*d
  return S >= 1 && E % BN == 0 && N % BN == 0;
}

cudaError_t launch_kv_gemm_bwd_tc(const void* y, const void* w_k, const void* w_v,
                                  const void* dk, const void* dv, void* dy, void* dw_k, void* dw_v,
                                  int S, int E, int N, cudaStream_t s) {
  // dW_z = y^T dZ: M = E, N = N, K = S; A = y stored [S][E] (M-major),
  // B = dZ stored [S][N] (N-major); two problems (dW_k, dW_v)
  {
    const Operand a[2] = {{y, (uint64_t)S, (uint64_t)E}, {y, (uint64_t)S, (uint64_t)E}};
    const Operand b[2] = {{dk, (uint64_t)S, (uint64_t)N}, {dv, (uint64_t)S, (uint64_t)N}};
    const int kb = (S + BK - 1) / BK;
    cudaError_t e = launch_gemm<true, true>(a, b, reinterpret_cast<__nv_bfloat16*>(dw_k),
                                            reinterpret_cast<__nv_bfloat16*>(dw_v), E, N, kb, kb,
                                            1, s);
    if (e != cudaSuccess) return e;
  }
  // dy = dK W_k^T + dV W_v^T: M = S, N = E, K = N per segment; A = dZ stored
  // [S][N] (K-major), B = W_z stored [E][N] (K-major)
  const Operand a[2] = {{dk, (uint64_t)S, (uint64_t)N}, {dv, (uint64_t)S, (uint64_t)N}};
  const Operand b[2] = {{w_k, (uint64_t)E, (uint64_t)N}, {w_v, (uint64_t)E, (uint64_t)N}};
  return launch_gemm<false, false>(a, b, reinterpret_cast<__nv_bfloat16*>(dy), nullptr, S, E,
                                   N / BK, 2 * (N / BK), 0, s);
}

cudaError_t launch_dw_accumulate_tc(const void* y, const void* dk, const void* dv, float* dw_k,
                                    float* dw_v, int S, int E, int N, cudaStream_t s) {
  // dW_z += y^T dZ: as in launch_kv_gemm_bwd_tc, the tile added to float32 outputs
  const Operand a[2] = {{y, (uint64_t)S, (uint64_t)E}, {y, (uint64_t)S, (uint64_t)E}};
  const Operand b[2] = {{dk, (uint64_t)S, (uint64_t)N}, {dv, (uint64_t)S, (uint64_t)N}};
  const int kb = (S + BK - 1) / BK;
  return launch_gemm<true, true>(a, b, nullptr, nullptr, E, N, kb, kb, 1, s, dw_k, dw_v);
}

cudaError_t launch_dy_tc(const void* w_k, const void* w_v, const void* dk, const void* dv,
                         void* dy, int S, int E, int N, cudaStream_t s) {
  // dy = dK W_k^T + dV W_v^T (two K segments), written in bf16
  const Operand a[2] = {{dk, (uint64_t)S, (uint64_t)N}, {dv, (uint64_t)S, (uint64_t)N}};
  const Operand b[2] = {{w_k, (uint64_t)E, (uint64_t)N}, {w_v, (uint64_t)E, (uint64_t)N}};
  return launch_gemm<false, false>(a, b, reinterpret_cast<__nv_bfloat16*>(dy), nullptr, S, E,
                                   N / BK, 2 * (N / BK), 0, s);
}

}  // namespace lvx
