// Backward pass on the tcgen05 tensor cores (bf16, head width 64 or 128).
//
// The pages leave the backward pass open (LV-XAttn review page, referee
// report, major comment 1: the gradient of the exact formula is the check).
// This kernel computes that exact gradient from the forward's stored
// log-sum-exp: P = exp(s q.k - LSE), dV = P^T dO, dP = dO V^T,
// dS = P o (dP - D) with D = rowsum(dO o O), dQ = s dS K, dK = s dS^T Q.
//
// A CTA works on key tiles: 128 keys of one (batch, key/value head), with K
// and V kept in shared memory, sweeping every 128-row query tile of every
// query head of the group (only tiles on or below the diagonal when causal).
// Without a mask the CTAs are persistent, one per SM, each taking a sequence
// of key tiles; with it, one CTA per key tile.  Per query tile:
//   S^T  = K Q^T        (SS)  -> TMEM [0,128)
//   dP^T = V dO^T       (SS)  -> TMEM [128,256)
//   elementwise warps: P^T = exp2(S^T * s*log2e - LSE*log2e) -> bf16 back
//       into TMEM [0,32) and [64,96); dS^T = P^T o (dP^T - D) -> bf16 into shared
//       memory, and packed over the dP^T columns already read, TMEM [128,160) and [192,224)
//   dV  += P^T dO       (TS, A = P^T from TMEM)  -> TMEM [256,256+D)
//   dK  += dS^T Q       (TS, A = dS^T from TMEM) -> TMEM [256+D,256+2D)
//   dQ_t = dS K         (SS, dS^T from shared memory read MN-major) -> TMEM [128,128+D);
//       issued after dK, so dK has read dS^T before dQ_t overwrites those columns
//   a drain warpgroup reads dQ_t out of TMEM, releases it, and adds it to the
//   fp32 dQ accumulator with TMA reduce-add, staged in the tile's dO slot
//   (idle once dV has run; the next dO load into that slot waits for the
//   reduce to have read it), so the reduction overlaps the next tile.
// dK and dV stay in TMEM for the whole sweep (the group's query heads are
// summed in place) and are written once per key tile: staged as bf16 in the
// dS buffer (free once the last dQ MMA completed) in the swizzled layout of a
// TMA box, then stored with TMA, so the global writes are whole 128-byte rows
// instead of one key row per lane.  Meanwhile the next key tile's K and V
// load into their own tiles.
#include "lvx_ptx.cuh"
#include "lvx_tc.cuh"

namespace lvx {
namespace {

using namespace ptx;

constexpr int BKEY = 128;
constexpr int BROW = 128;
constexpr int kThreads = 512;
// Register split (launched at 128 per thread): warpgroup 0 (producers, MMA
// issuer, allocator) 56, the two elementwise warpgroups 168, the dQ drain
// warpgroup 120:  128 x 56 + 256 x 168 + 128 x 120 = 65536 = 512 x 128.
constexpr uint32_t kRegsControl = 56;
constexpr uint32_t kRegsElementwise = 168;
constexpr uint32_t kRegsDrain = 120;
static_assert(128 * kRegsControl + 256 * kRegsElementwise + 128 * kRegsDrain <=
                  65536 / kThreads * kThreads,
              "register split exceeds the launch allocation");
constexpr uint32_t CHUNK = 128 * 128;   // 128 rows x 64 bf16, 128-byte swizzle

template <int D>
struct BwdLayout {
  static constexpr uint32_t TILE = 128 * D * 2;
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = OFF_K + TILE;
  static constexpr uint32_t OFF_Q = OFF_V + TILE;          // 2 stages
  static constexpr uint32_t OFF_DO = OFF_Q + 2 * TILE;     // 2 stages
  static constexpr uint32_t OFF_DS = OFF_DO + 2 * TILE;    // 128 keys x 128 rows bf16
  static constexpr uint32_t OFF_LSE = OFF_DS + 2 * CHUNK;  // 2 stages x 128 fp32
  static constexpr uint32_t OFF_DD = OFF_LSE + 2 * 512;    // 2 stages x 128 fp32
  // dQ staging, 2 stages x 32 KiB: the dO slots themselves when they are that
  // large (D = 128), otherwise a buffer of its own
  static constexpr uint32_t STAGE = 32768;
  static constexpr bool STAGE_IN_DO = TILE >= STAGE;
  static constexpr uint32_t OFF_STG = OFF_DD + 2 * 512;
  static constexpr uint32_t OFF_BAR = OFF_STG + (STAGE_IN_DO ? 0 : 2 * STAGE);
  __device__ static constexpr uint32_t stage_off(int s) {
    return STAGE_IN_DO ? OFF_DO + s * TILE : OFF_STG + s * STAGE;
  }
  static constexpr uint32_t USED = OFF_BAR + 256;
  static constexpr uint32_t SLACK = 768;                   // for aligning the base to 1 KiB
  static constexpr uint32_t BYTES = (USED + SLACK) > 118784 ? (USED + SLACK) : 118784;
  static constexpr uint32_t IDESC_SS_KK = ptx::idesc_bf16_f32(128, 128, false, false);
  static constexpr uint32_t IDESC_DP_HALF = ptx::idesc_bf16_f32(128, 64, false, false);
  static constexpr uint32_t IDESC_DV = ptx::idesc_bf16_f32(128, D, false, true);
  static constexpr uint32_t IDESC_DK = ptx::idesc_bf16_f32(128, D, false, true);
  static constexpr uint32_t IDESC_DQ = ptx::idesc_bf16_f32(128, D, true, true);
};

struct BwdArgs {
  Problem p;
  float* dq_acc;
  unsigned int* err;
  int n_kt;     // key tiles per (batch, kv head)
  int n_qt;     // query tiles per head
  int n_items;  // key tiles over all (batch, kv head)
};

// One unit of work: the 128 keys [n0, n0+128) of one (batch, key/value head)
// and the I query tiles (of the group's heads) that see them.
struct KeyTile {
  int g, b, n0, kt, m_start, per_head, I;
};

__device__ __forceinline__ KeyTile key_tile(const Problem& p, int n_kt, int n_qt, int item) {
  KeyTile w;
  w.kt = item % n_kt;
  const int bg = item / n_kt;
  w.g = bg % p.H_kv;
  w.b = bg / p.H_kv;
  w.n0 = w.kt * BKEY;
  w.m_start = p.causal ? w.kt : 0;   // query tiles below the diagonal see none of these keys
  w.per_head = n_qt - w.m_start;
  w.I = w.per_head > 0 ? (p.H / p.H_kv) * w.per_head : 0;
  return w;
}

// Key tile of CTA c in round r: c in even rounds, gridDim.x - 1 - c in odd
// ones.  With the causal mask a key tile's work falls linearly with its index,
// so each pair of rounds gives every CTA about the same number of query tiles.
__device__ __forceinline__ int serpentine(int r, int c, int step) {
  return r * step + ((r & 1) ? step - 1 - c : c);
}

// ACC: dK, dV added to float32 arrays (map_dk / map_dv are float32 32x32 pieces)
template <int D, bool ACC>
__global__ void __launch_bounds__(kThreads, 1)
bwd_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
              const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_do,
              const __grid_constant__ CUtensorMap map_lse, const __grid_constant__ CUtensorMap map_dd,
              const __grid_constant__ CUtensorMap map_dq, const __grid_constant__ CUtensorMap map_dk,
              const __grid_constant__ CUtensorMap map_dv, const BwdArgs a) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;      // [2] Q, -LSE*log2e, -D of a stage
  uint64_t* q_empty = bars + 3;     // [2]
  uint64_t* s_full = bars + 5;
  uint64_t* p_ready = bars + 7;
  uint64_t* ds_ready = bars + 8;
  uint64_t* dq_full = bars + 10;
  uint64_t* mma_drain = bars + 12;
  uint64_t* stage_free = bars + 13;   // [2] a stage's dQ staging read by the TMA
  uint64_t* do_full = bars + 15;      // [2] dO of a stage
  uint64_t* dp_full = bars + 17;      // [2] dP^T of query rows [64h, 64h+64)
  uint64_t* dq_free = bars + 19;      // [2] dQ_t columns [64h, 64h+64) read by the drain
  uint64_t* kv_free = bars + 21;      // K, V of a key tile last read (its final dQ MMA done)
  uint64_t* epi_full = bars + 22;     // a dK or dV tile staged by all 256 elementwise threads
  uint64_t* epi_free = bars + 23;     // its TMA store has read the staging buffer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 24);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if ((uint32_t)(smem - smem_raw) + L::USED > L::BYTES) {   // dynamic smem base not 1 KiB aligned
    if (threadIdx.x == 0) record_error(a.err, kErrSmemAlign);
    return;
  }
  const Problem& p = a.p;
  const int grp = p.H / p.H_kv;
  // Persistent: in round r the CTAs take key tiles r*gridDim.x .. + gridDim.x - 1,
  // in serpentine order (see serpentine()), so the CTAs resident together hold
  // consecutive key tiles of one (batch, key head), which share their query
  // rows in L2.  Every role walks the same sequence; tile counters run on
  // across key tiles, so the rings keep their phases.
  const int first = blockIdx.x, step = gridDim.x, n_items = a.n_items;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    ptx::mbar_init(kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&q_full[s], 1);
      ptx::mbar_init(&q_empty[s], 1);
      ptx::mbar_init(&stage_free[s], 4);
      ptx::mbar_init(&do_full[s], 1);
    }
    ptx::mbar_init(s_full, 1);
    ptx::mbar_init(p_ready, 256);
    ptx::mbar_init(ds_ready, 256);
    ptx::mbar_init(dq_full, 1);
    for (int h = 0; h < 2; ++h) {
      ptx::mbar_init(&dp_full[h], 1);
      ptx::mbar_init(&dq_free[h], 128);
    }
    ptx::mbar_init(mma_drain, 1);
    ptx::mbar_init(kv_free, 1);
    ptx::mbar_init(epi_full, 256);
    ptx::mbar_init(epi_free, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 2) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 256 + D;

  if (warp < 4) {
    ptx::setmaxnreg_dec<kRegsControl>();
    if (warp == 0) {
      if (lane == 0) {
        // ---------------------------------------------------------------- producer: K, V, Q, LSE, D
        // The K/V tiles of a key tile are loaded once the previous key tile's
        // last dQ MMA (their last reader) completed: kv_free completes once per
        // key tile with query tiles, and this thread waits for the phase just
        // before the one it enables, so the parity test cannot be overtaken.
        ptx::tma_prefetch_desc(&map_q);
        int gt = 0, nkv = 0;   // tiles and K/V loads issued
        bool ok = true;
        for (int r = 0; r * step < n_items && ok; ++r) {
          const int item = serpentine(r, first, step);
          if (item >= n_items) continue;
          const KeyTile w = key_tile(p, a.n_kt, a.n_qt, item);
          if (w.I == 0) continue;   // no query tile: dK, dV are zero, K and V unused
          if (nkv > 0 && !ptx::mbar_wait(kv_free, (nkv - 1) & 1, a.err, kErrTimeoutTma, abort_flag)) {
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(kv_full, 2 * L::TILE);
          for (int c = 0; c < D / 64; ++c) {
            ptx::tma_load_4d(smem + L::OFF_K + c * CHUNK, &map_k, kv_full, 64 * c, w.g, w.n0, w.b);
            ptx::tma_load_4d(smem + L::OFF_V + c * CHUNK, &map_v, kv_full, 64 * c, w.g, w.n0, w.b);
          }
          ++nkv;
          for (int i = 0; i < w.I; ++i, ++gt) {
            const int s = gt & 1;
            const int h = w.g * grp + i / w.per_head;
            const int m = w.m_start + i % w.per_head;
            if (!ptx::mbar_wait(&q_empty[s], ((gt >> 1) & 1) ^ 1, a.err, kErrTimeoutTma, abort_flag)) {
              ok = false;
              break;
            }
            ptx::mbar_arrive_expect_tx(&q_full[s], L::TILE + 2 * 512);
            for (int c = 0; c < D / 64; ++c)
              ptx::tma_load_4d(smem + L::OFF_Q + s * L::TILE + c * CHUNK, &map_q, &q_full[s], 64 * c,
                               h, BROW * m, w.b);
            ptx::tma_load_2d(smem + L::OFF_LSE + s * 512, &map_lse, &q_full[s], BROW * m, w.b * p.H + h);
            ptx::tma_load_2d(smem + L::OFF_DD + s * 512, &map_dd, &q_full[s], BROW * m, w.b * p.H + h);
          }
        }
        if (*abort_flag) {   // the copies in flight must land before shared memory is released
          if (nkv > 0) ptx::mbar_wait(kv_full, (nkv - 1) & 1, a.err, kErrTimeoutTma, nullptr);
          for (int i = gt > 2 ? gt - 2 : 0; i < gt; ++i)
            ptx::mbar_wait(&q_full[i & 1], (i >> 1) & 1, a.err, kErrTimeoutTma, nullptr);
        }
      }
    } else if (warp == 3) {
      if (lane == 0) {
        // ---------------------------------------------------------------- producer: dO
        // dO of tile gt goes into slot gt&1 once the drain's reduce has read the
        // dQ of tile gt-2 staged there (D = 128) -- that wait is what lets the
        // reduction run behind the following tile's work
        ptx::tma_prefetch_desc(&map_do);
        int gt = 0;
        bool ok = true;
        for (int r = 0; r * step < n_items && ok; ++r) {
          const int item = serpentine(r, first, step);
          if (item >= n_items) continue;
          const KeyTile w = key_tile(p, a.n_kt, a.n_qt, item);
          for (int i = 0; i < w.I; ++i, ++gt) {
            const int s = gt & 1;
            const int h = w.g * grp + i / w.per_head;
            const int m = w.m_start + i % w.per_head;
            if (!ptx::mbar_wait(&stage_free[s], ((gt >> 1) & 1) ^ 1, a.err, kErrTimeoutTma, abort_flag)) {
              ok = false;
              break;
            }
            ptx::mbar_arrive_expect_tx(&do_full[s], L::TILE);
            for (int c = 0; c < D / 64; ++c)
              ptx::tma_load_4d(smem + L::OFF_DO + s * L::TILE + c * CHUNK, &map_do, &do_full[s], 64 * c,
                               h, BROW * m, w.b);
          }
        }
        if (*abort_flag) {
          for (int i = gt > 2 ? gt - 2 : 0; i < gt; ++i)
            ptx::mbar_wait(&do_full[i & 1], (i >> 1) & 1, a.err, kErrTimeoutTma, nullptr);
        }
      }
    } else if (warp == 1) {
      if (lane == 0) {
        // ---------------------------------------------------------------- MMA issuer
        // Shared-memory descriptors (128-byte swizzle): the high word is the
        // same for every operand here (sbo 1024, version, swizzle mode), and the
        // low word is (address >> 4) | (lbo >> 4) << 16.  Only the low words of
        // the five buffers are kept (K-major form, lbo 16); a stage, K step or
        // MN-major form (lbo CHUNK) adds a compile-time constant to them.
        // Shared-memory addresses stay below 2^18, so the 14-bit address field
        // never carries into lbo.  This keeps the issuing thread, which shares
        // its sub-partition with three busy warps, at a few instructions per
        // MMA, within the registers of its warp group.  The empty asm below
        // marks the five words as changed once per query tile, so that the
        // compiler derives each descriptor where it is used instead of keeping
        // every K step's descriptor live across the loop (which spills).
        uint32_t dK = (ptx::smem_u32(smem + L::OFF_K) >> 4) | (1u << 16);
        uint32_t dV = (ptx::smem_u32(smem + L::OFF_V) >> 4) | (1u << 16);
        uint32_t dQ = (ptx::smem_u32(smem + L::OFF_Q) >> 4) | (1u << 16);
        uint32_t dDO = (ptx::smem_u32(smem + L::OFF_DO) >> 4) | (1u << 16);
        uint32_t dDS = (ptx::smem_u32(smem + L::OFF_DS) >> 4) | (1u << 16);
        constexpr uint32_t kMN = ((CHUNK >> 4) - 1u) << 16;   // lbo 16 -> lbo CHUNK
        auto desc = [](uint32_t lo) {
          return ((uint64_t)((1024u >> 4) | (1u << 14) | (2u << 29)) << 32) | lo;
        };
        constexpr uint32_t kStage16 = L::TILE >> 4;   // one Q / dO stage, in descriptor units
        // Issue order within a key tile: S_0, dP_0, dV_0, then per tile i
        //   S_{i+1}, dK_i, dQ_i, dP_{i+1}, dV_{i+1}.
        // S_{i+1} goes right after dV_i, which reads P_i from the same TMEM
        // columns: tcgen05.mma ops of one thread execute in issue order, so the
        // read completes first, and the elementwise warps can start on tile
        // i+1 while the tensor core works on dK_i and dQ_i.  dP_{i+1} reuses the
        // columns of dQ_i; it is issued as two 64-query halves, each as soon as
        // the drain warps have read the 64 dQ columns it overwrites.  The first
        // dV and dK MMAs of a key tile overwrite the accumulators: they wait
        // for P and dS of its first tile, which the elementwise warps produce
        // only after writing out the previous key tile's dK and dV.
        auto issue_s = [&](int gi) {
          const uint32_t qs = dQ + (gi & 1) * kStage16;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {   // S^T = K Q^T
            const uint32_t off = ((kk >> 2) * CHUNK + (kk & 3) * 32) >> 4;
            ptx::mma_ss(tS, desc(dK + off), desc(qs + off), L::IDESC_SS_KK, kk > 0);
          }
          ptx::mma_commit(s_full);
        };
        auto issue_dp_dv = [&](int gi, bool first_tile) -> bool {
          const uint32_t dos = dDO + (gi & 1) * kStage16;
          if (!ptx::mbar_wait(&do_full[gi & 1], (gi >> 1) & 1, a.err, kErrTimeoutMma, abort_flag))
            return false;
          ptx::tc_fence_after();
#pragma unroll
          for (int h = 0; h < 2; ++h) {   // dP^T = V dO^T, query rows [64h, 64h+64)
            if (gi > 0) {
              if (!ptx::mbar_wait(&dq_free[h], (gi - 1) & 1, a.err, kErrTimeoutMma, abort_flag))
                return false;
              ptx::tc_fence_after();
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = ((kk >> 2) * CHUNK + (kk & 3) * 32) >> 4;
              ptx::mma_ss(tdP + 64 * h, desc(dV + off), desc(dos + off + h * (8192 >> 4)),
                          L::IDESC_DP_HALF, kk > 0);
            }
            ptx::mma_commit(&dp_full[h]);
          }
          if (!ptx::mbar_wait(p_ready, gi & 1, a.err, kErrTimeoutMma, abort_flag)) return false;
          ptx::tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BROW / 16; ++kk)   // dV += P^T dO (P^T halves at columns 0 and 64)
            ptx::mma_ts(tdV, tS + (kk >> 2) * 64 + (kk & 3) * 8,
                        desc(dos + (kMN + kk * (2048 >> 4))), L::IDESC_DV,
                        (!first_tile || kk > 0) ? 1u : 0u);
          return true;
        };
        int gt = 0, nkv = 0;
        bool ok = true;
        for (int r = 0; r * step < n_items && ok; ++r) {
          const int item = serpentine(r, first, step);
          if (item >= n_items) continue;
          const KeyTile w = key_tile(p, a.n_kt, a.n_qt, item);
          if (w.I == 0) continue;
          ok = ptx::mbar_wait(kv_full, nkv & 1, a.err, kErrTimeoutMma, abort_flag);
          ++nkv;
          if (ok) ok = ptx::mbar_wait(&q_full[gt & 1], (gt >> 1) & 1, a.err, kErrTimeoutMma, abort_flag);
          if (!ok) break;
          ptx::tc_fence_after();
          issue_s(gt);
          ok = issue_dp_dv(gt, true);
          for (int i = 0; i < w.I && ok; ++i) {
            const int gi = gt + i;
            asm volatile("" : "+r"(dK), "+r"(dV), "+r"(dQ), "+r"(dDO), "+r"(dDS));
            if (i + 1 < w.I) {
              ok = ptx::mbar_wait(&q_full[(gi + 1) & 1], ((gi + 1) >> 1) & 1, a.err, kErrTimeoutMma,
                                  abort_flag);
              if (!ok) break;
              ptx::tc_fence_after();
              issue_s(gi + 1);
            }
            ok = ptx::mbar_wait(ds_ready, gi & 1, a.err, kErrTimeoutMma, abort_flag);
            if (!ok) break;
            ptx::tc_fence_after();
            const uint32_t qs = dQ + (gi & 1) * kStage16;
#pragma unroll
            for (int kk = 0; kk < BROW / 16; ++kk) {   // dK += dS^T Q (dS^T halves at columns 0 and 64)
              ptx::mma_ts(tdK, tdP + (kk >> 2) * 64 + (kk & 3) * 8, desc(qs + (kMN + kk * (2048 >> 4))),
                          L::IDESC_DK, (i > 0 || kk > 0) ? 1u : 0u);
            }
            ptx::mma_commit(&q_empty[gi & 1]);   // Q, LSE, D of this stage are no longer read
#pragma unroll
            for (int kk = 0; kk < BKEY / 16; ++kk)   // dQ_t = dS K
              ptx::mma_ss(tdP, desc(dDS + (kMN + kk * (2048 >> 4))),
                          desc(dK + (kMN + kk * (2048 >> 4))), L::IDESC_DQ, kk > 0);
            ptx::mma_commit(dq_full);
            if (i + 1 < w.I) ok = issue_dp_dv(gi + 1, false);
            else ptx::mma_commit(kv_free);   // K and V of this key tile are no longer read
          }
          gt += w.I;
        }
        ptx::mma_commit(mma_drain);
      }
    }
  } else if (warp < 12) {
    ptx::setmaxnreg_inc<kRegsElementwise>();
    // ------------------------------------------------------------------ elementwise
    const int quarter = warp & 3;
    const int hf = (warp - 4) >> 2;            // which half of the 128 query rows
    const int j = quarter * 32 + lane;         // key within the tile (TMEM lane)
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float sl2 = p.scale_log2;
    uint8_t* ds_smem = smem + L::OFF_DS + hf * CHUNK + j * 128;
    bool ok = true;
    int gt = 0, er = 0;   // tiles done, dK/dV staging rounds done
    for (int r = 0; r * step < n_items; ++r) {
      const int item = serpentine(r, first, step);
      if (item >= n_items) continue;
      const KeyTile w = key_tile(p, a.n_kt, a.n_qt, item);
      const int key = w.n0 + j;
      for (int i = 0; i < w.I && ok; ++i, ++gt) {
        const int s = gt & 1;
        const int m = w.m_start + i % w.per_head;
        const int r0 = BROW * m + 64 * hf;       // first query row handled by this thread
        // the stages hold -LSE*log2(e) and -rowsum(dO o O) (written by the preprocess kernel)
        const float* nlse_s = reinterpret_cast<const float*>(smem + L::OFF_LSE + s * 512) + 64 * hf;
        const float* nd_s = reinterpret_cast<const float*>(smem + L::OFF_DD + s * 512) + 64 * hf;
        // this stage's LSE and D rows (TMA) are read directly below; the stage is
        // only refilled after the MMAs of this tile, which wait for this thread
        ok = ptx::mbar_wait(&q_full[s], (gt >> 1) & 1, a.err, kErrTimeoutSoftmax, abort_flag);
        ok = ok && ptx::mbar_wait(s_full, gt & 1, a.err, kErrTimeoutSoftmax, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ptx::tc_fence_after();
        uint64_t P2[32];   // P^T of this thread's 64 query rows as packed fp32 pairs
        {
          uint32_t sr[64];
          ptx::tmem_ld32(tS + lane_off + 64 * hf, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
          ptx::tmem_ld32(tS + lane_off + 64 * hf + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
          ptx::tmem_wait_ld();
          // masking is needed only on the causal diagonal tile and at the ragged ends
          const bool need_mask = (p.causal && m == w.kt) || (w.n0 + BKEY > p.S_KV) ||
                                 (BROW * m + BROW > p.S_Q);
          if (need_mask) {
            const bool key_ok = key < p.S_KV;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              float e[2];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int r = r0 + 2 * c + u;
                const bool vis = key_ok && r < p.S_Q && (!p.causal || key <= r);
                e[u] = vis ? ex2(fmaf(__uint_as_float(sr[2 * c + u]), sl2, nlse_s[2 * c + u])) : 0.f;
              }
              P2[c] = pk2(e[0], e[1]);
            }
          } else {
            // x = s * scale*log2(e) - LSE*log2(e) on FFMA2; one pair in kPolyEvery of the
            // exponentials on the FMA pipe, the rest on the SFU
            const uint64_t sl2x2 = pk2(sl2, sl2);
#pragma unroll
            for (int c4 = 0; c4 < 16; ++c4) {
              const float4 l4 = *reinterpret_cast<const float4*>(nlse_s + 4 * c4);
              const uint64_t xa = ffma2(pk2(__uint_as_float(sr[4 * c4]), __uint_as_float(sr[4 * c4 + 1])),
                                        sl2x2, pk2(l4.x, l4.y));
              const uint64_t xb = ffma2(pk2(__uint_as_float(sr[4 * c4 + 2]), __uint_as_float(sr[4 * c4 + 3])),
                                        sl2x2, pk2(l4.z, l4.w));
              float a0, a1, b0, b1;
              upk2(xa, a0, a1);
              P2[2 * c4] = pk2(ex2(a0), ex2(a1));
              if ((2 * c4 + 1) % kPolyEvery == kPolyEvery - 1) {
                P2[2 * c4 + 1] = exp2_poly2(xb);
              } else {
                upk2(xb, b0, b1);
                P2[2 * c4 + 1] = pk2(ex2(b0), ex2(b1));
              }
            }
          }
        }
        {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            float lo, hi;
            upk2(P2[c], lo, hi);
            pk[c] = ptx::pack_bf16x2(lo, hi);
          }
          // P^T of rows [64hf, 64hf+64) goes to columns [64hf, 64hf+32): only over
          // S^T columns this thread has already read
          ptx::tmem_st32(tS + lane_off + 64 * hf, pk);
          ptx::tmem_wait_st();
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(p_ready);
        ok = ptx::mbar_wait(&dp_full[hf], gt & 1, a.err, kErrTimeoutSoftmax, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ptx::tc_fence_after();
        // dS^T row of key j, query rows r0 .. r0+63 (one 128-byte swizzled row),
        // dS = P o (dP - D) on FADD2/FMUL2, in two 32-column halves to bound registers
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t dr[32];
          uint32_t dsk[16];
          ptx::tmem_ld32(tdP + lane_off + 64 * hf + 32 * half, dr);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            const int c8 = 4 * half + q8;
            const float4 na = *reinterpret_cast<const float4*>(nd_s + 8 * c8);
            const float4 nb = *reinterpret_cast<const float4*>(nd_s + 8 * c8 + 4);
            const float nv[8] = {na.x, na.y, na.z, na.w, nb.x, nb.y, nb.z, nb.w};
            uint32_t wd[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const uint64_t d2 = fadd2(pk2(__uint_as_float(dr[8 * q8 + 2 * t]),
                                            __uint_as_float(dr[8 * q8 + 2 * t + 1])),
                                        pk2(nv[2 * t], nv[2 * t + 1]));
              float e0, e1;
              upk2(fmul2(P2[4 * c8 + t], d2), e0, e1);
              wd[t] = ptx::pack_bf16x2(e0, e1);
            }
            *reinterpret_cast<uint4*>(ds_smem + ((c8 ^ (j & 7)) << 4)) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
#pragma unroll
            for (int t = 0; t < 4; ++t) dsk[4 * q8 + t] = wd[t];
          }
          // dS^T of these 32 rows, packed, over dP^T columns this thread has read
          ptx::tmem_st16(tdP + lane_off + 64 * hf + 16 * half, dsk);
        }
        ptx::tmem_wait_st();
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        ptx::mbar_arrive(ds_ready);
      }
      if (!ok) break;
      // -------------------------------------------------------------- epilogue: dK, dV
      // The last dq_full of the key tile follows its last dK, dQ (and dV) MMAs,
      // so the accumulators are final and the dS buffer is free.  dV, then dK
      // (times the softmax scale) are staged there as bf16 in the swizzled
      // layout of a TMA box -- thread (hf, key j) owns head-width columns
      // [hf D/2, hf D/2 + D/2) of row j -- and stored with TMA (rows past S_KV
      // are clipped), so the global writes are whole 128-byte rows.  The
      // hand-offs use bounded mbarrier waits: a thread that gives up cannot
      // strand the others.
      if (w.I > 0) {
        ok = ptx::mbar_wait(dq_full, (gt - 1) & 1, a.err, kErrTimeoutEpilogue, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ptx::tc_fence_after();
      }
      constexpr int HALF = D / 2;
      // With ACC, dV and dK are instead added to the caller's float32
      // arrays with TMA reduce-add, 32 keys x 32 columns at a time: each warp
      // stages in the 4 KiB of the dS buffer that holds its own dS rows (its
      // keys' rows of its query half), so it waits only for its own copies, and
      // before its next dS store.  A key tile no query tile sees adds nothing.
      // (the base is made opaque here so that these addresses are not hoisted
      // into the tile loop above, where registers are short)
      uint8_t* ebase = smem;
      asm volatile("" : "+l"(ebase));
      constexpr bool acc = ACC;
      uint8_t* region = ebase + L::OFF_DS + hf * CHUNK + quarter * 4096;
#pragma unroll 1
      for (int which = 0; which < 2 && !(acc && w.I == 0); ++which) {
        const uint32_t tacc = (which == 0 ? tdV : tdK) + lane_off + HALF * hf;
        const float mul = which == 0 ? 1.f : p.scale;
        uint8_t* stg = ebase + L::OFF_DS + j * 128;
#pragma unroll 1
        for (int c = 0; c < HALF / 32; ++c) {
          uint32_t r[32];
          if (w.I > 0) {
            ptx::tmem_ld32(tacc + 32 * c, r);
            ptx::tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = 0u;
          }
          if constexpr (acc) {
            if (lane == 0 && (which | c) != 0) bulk_wait_read();   // previous piece read
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<uint4*>(region + lane * 128 + ((q ^ (lane & 7)) << 4)) =
                  make_uint4(__float_as_uint(__uint_as_float(r[4 * q]) * mul),
                             __float_as_uint(__uint_as_float(r[4 * q + 1]) * mul),
                             __float_as_uint(__uint_as_float(r[4 * q + 2]) * mul),
                             __float_as_uint(__uint_as_float(r[4 * q + 3]) * mul));
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_reduce_add_4d(which == 0 ? &map_dv : &map_dk, region, HALF * hf + 32 * c, w.g,
                                w.n0 + quarter * 32, w.b);
              bulk_commit();
            }
            continue;
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int col = HALF * hf + 32 * c + 8 * q;
            uint4 u;
            u.x = ptx::pack_bf16x2(__uint_as_float(r[8 * q + 0]) * mul, __uint_as_float(r[8 * q + 1]) * mul);
            u.y = ptx::pack_bf16x2(__uint_as_float(r[8 * q + 2]) * mul, __uint_as_float(r[8 * q + 3]) * mul);
            u.z = ptx::pack_bf16x2(__uint_as_float(r[8 * q + 4]) * mul, __uint_as_float(r[8 * q + 5]) * mul);
            u.w = ptx::pack_bf16x2(__uint_as_float(r[8 * q + 6]) * mul, __uint_as_float(r[8 * q + 7]) * mul);
            *reinterpret_cast<uint4*>(stg + (col >> 6) * CHUNK + ((((col & 63) >> 3) ^ (j & 7)) << 4)) = u;
          }
        }
        if constexpr (acc) continue;
        ++er;
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        ptx::mbar_arrive(epi_full);
        if (warp == 4 && lane == 0) {
          ok = ptx::mbar_wait(epi_full, (er - 1) & 1, a.err, kErrTimeoutEpilogue, abort_flag);
          if (ok) {
            for (int c = 0; c < D / 64; ++c)
              tma_store_4d(which == 0 ? &map_dv : &map_dk, smem + L::OFF_DS + c * CHUNK, 64 * c, w.g,
                           w.n0, w.b);
            bulk_commit();
            bulk_wait_read();
          }
          ptx::mbar_arrive(epi_free);
        }
        ok = ptx::mbar_wait(epi_free, (er - 1) & 1, a.err, kErrTimeoutEpilogue, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      if (acc && w.I > 0) {
        if (lane == 0) bulk_wait_read();   // the region takes this warp's next dS rows
        __syncwarp();
        ptx::tc_fence_before();
      }
      if (!ok) break;
    }
    if ((warp == 4 || ACC) && lane == 0) bulk_wait_all();
  } else {
    ptx::setmaxnreg_dec<kRegsDrain>();
    // ------------------------------------------------------------------ dQ drain
    // Warp 12+q reads TMEM lanes 32q..32q+31 (query rows) of dQ_t, releases the
    // columns to the MMA warp, and adds the rows to dQ_acc: 32x32 pieces are
    // staged 128-byte swizzled in its own 8 KiB of the tile's staging slot
    // (the dO slot for D = 128: its last reader, dV, completed before the dQ
    // MMA) and reduced with TMA reduce-add; the slot is handed back to the dO
    // producer once the TMA has read it.
    const int quarter = warp & 3;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    int gt = 0;
    for (int r = 0; r * step < n_items && ok; ++r) {
          const int item = serpentine(r, first, step);
          if (item >= n_items) continue;
      const KeyTile w = key_tile(p, a.n_kt, a.n_qt, item);
      for (int i = 0; i < w.I; ++i, ++gt) {
        uint8_t* stage = smem + L::stage_off(gt & 1) + quarter * 8192;
        const int h = w.g * grp + i / w.per_head;
        const int m = w.m_start + i % w.per_head;
        const int row0 = BROW * m + quarter * 32;
        ok = ptx::mbar_wait(dq_full, gt & 1, a.err, kErrTimeoutSoftmax, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int round = 0; round < D / 64; ++round) {
          uint32_t qr[64];
          ptx::tmem_ld32(tdP + lane_off + 64 * round, *reinterpret_cast<uint32_t(*)[32]>(&qr[0]));
          ptx::tmem_ld32(tdP + lane_off + 64 * round + 32, *reinterpret_cast<uint32_t(*)[32]>(&qr[32]));
          ptx::tmem_wait_ld();
          // these 64 columns may now take the next tile's dP^T half (with D = 64
          // the second half of the dP^T columns never held dQ)
          ptx::tc_fence_before();
          ptx::mbar_arrive(&dq_free[round]);
          if (D == 64) ptx::mbar_arrive(&dq_free[1]);
          if (round > 0) {   // the previous round's pieces must have been read by the TMA
            if (lane == 0) bulk_wait_read();
            __syncwarp();
          }
#pragma unroll
          for (int piece = 0; piece < 2; ++piece) {
            uint8_t* st = stage + piece * 4096;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(st + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                  make_uint4(qr[32 * piece + 4 * c], qr[32 * piece + 4 * c + 1],
                             qr[32 * piece + 4 * c + 2], qr[32 * piece + 4 * c + 3]);
          }
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_reduce_add_4d(&map_dq, stage, 64 * round, h, row0, w.b);
            tma_reduce_add_4d(&map_dq, stage + 4096, 64 * round + 32, h, row0, w.b);
            bulk_commit();
          }
        }
        if (lane == 0) {
          bulk_wait_read();
          ptx::mbar_arrive(&stage_free[gt & 1]);
        }
        __syncwarp();
      }
    }
    if (lane == 0) bulk_wait_all();
  }

  // ------------------------------------------------------------------ teardown
  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    ptx::mbar_wait(mma_drain, 0, a.err, kErrTimeoutEpilogue, nullptr);
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

template <int D>
cudaError_t launch(const Problem& p, const void* q, const void* k, const void* v,
                   const void* dout, const float* lse, const float* Dv, float* dq_acc, void* dk,
                   void* dv, bool accum, cudaStream_t s) {
  using L = BwdLayout<D>;
  CUtensorMap mq, mk, mv, mdo, mlse, mdd, mdq, mdk, mdv;
  {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)p.H, (uint64_t)p.S_Q, (uint64_t)p.B};
    const uint64_t str[3] = {(uint64_t)D * 4, (uint64_t)p.H * D * 4, (uint64_t)p.S_Q * p.H * D * 4};
    const uint32_t box4[4] = {32, 1, 32, 1};
    if (!encode_tensor_map(&mdq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dq_acc, dims, str, box4,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  const uint32_t box[4] = {64, 1, 128, 1};
  {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)p.H, (uint64_t)p.S_Q, (uint64_t)p.B};
    const uint64_t str[3] = {(uint64_t)D * 2, (uint64_t)p.H * D * 2, (uint64_t)p.S_Q * p.H * D * 2};
    if (!encode_tensor_map(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, q, dims, str, box,
                           CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tensor_map(&mdo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, dout, dims, str, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)p.H_kv, (uint64_t)p.S_KV, (uint64_t)p.B};
    const uint64_t str[3] = {(uint64_t)D * 2, (uint64_t)p.H_kv * D * 2,
                             (uint64_t)p.S_KV * p.H_kv * D * 2};
    if (!encode_tensor_map(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, k, dims, str, box,
                           CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tensor_map(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, v, dims, str, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    if (accum) {
      // float32 dK, dV, reduced 32 keys x 32 columns at a time
      const uint64_t str4[3] = {(uint64_t)D * 4, (uint64_t)p.H_kv * D * 4,
                                (uint64_t)p.S_KV * p.H_kv * D * 4};
      const uint32_t box4[4] = {32, 1, 32, 1};
      if (!encode_tensor_map(&mdk, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dk, dims, str4, box4,
                             CU_TENSOR_MAP_SWIZZLE_128B) ||
          !encode_tensor_map(&mdv, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dv, dims, str4, box4,
                             CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    } else if (!encode_tensor_map(&mdk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, dk, dims, str, box,
                                  CU_TENSOR_MAP_SWIZZLE_128B) ||
               !encode_tensor_map(&mdv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, dv, dims, str, box,
                                  CU_TENSOR_MAP_SWIZZLE_128B)) {
      return cudaErrorInvalidValue;
    }
  }
  {
    // LSE and D: [B*H, S_Q] fp32 rows; S_Q * 4 bytes must be a multiple of 16
    const uint64_t dims[2] = {(uint64_t)p.S_Q, (uint64_t)p.B * p.H};
    const uint64_t str[1] = {(uint64_t)p.S_Q * 4};
    const uint32_t box2[2] = {128, 1};
    if (!encode_tensor_map(&mlse, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, lse, dims, str, box2,
                           CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_tensor_map(&mdd, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, Dv, dims, str, box2,
                           CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  }
  BwdArgs a;
  a.p = p;
  a.dq_acc = dq_acc;
  a.err = device_error_word();
  a.n_kt = (p.S_KV + BKEY - 1) / BKEY;
  a.n_qt = (p.S_Q + BROW - 1) / BROW;
  if (!a.err) return cudaErrorInvalidValue;
  const long long items = (long long)a.n_kt * p.H_kv * p.B;
  if (items > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  a.n_items = (int)items;
  // Without a mask every key tile has the same work: one persistent CTA per SM
  // (each owns all 512 TMEM columns) saves the CTA turnaround and overlaps the
  // next key tile's K/V load with the dK/dV epilogue.  With the causal mask the
  // work per key tile falls along the diagonal, and one CTA per key tile lets
  // the hardware scheduler balance the SMs (measured faster than any static split).
  long long grid = items;
  if (!p.causal) {
    int dev = 0, n_sm = 0;
    cudaError_t ea = cudaGetDevice(&dev);
    if (ea == cudaSuccess) ea = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (ea != cudaSuccess) return ea;
    if (items > n_sm) grid = n_sm;
  }
  auto kernel = accum ? bwd_tc_kernel<D, true> : bwd_tc_kernel<D, false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
  if (e != cudaSuccess) return e;
  kernel<<<(unsigned)grid, kThreads, L::BYTES, s>>>(mq, mk, mv, mdo, mlse, mdd, mdq, mdk, mdv, a);
  return cudaGetLastError();
}

}  // namespace

// The LSE/D rows are fetched with TMA, whose row stride must be a multiple of 16 bytes.
bool tc_bwd_supported(const Problem& p) { return (p.d == 64 || p.d == 128) && p.S_Q % 4 == 0; }

cudaError_t launch_bwd_tc(const Problem& p, const void* q, const void* k, const void* v,
                          const void* dout, const float* nlse2, const float* nd, float* dq_acc,
                          void* dk, void* dv, bool accum, cudaStream_t s) {
  if (p.d == 128) return launch<128>(p, q, k, v, dout, nlse2, nd, dq_acc, dk, dv, accum, s);
  if (p.d == 64) return launch<64>(p, q, k, v, dout, nlse2, nd, dq_acc, dk, dv, accum, s);
  return cudaErrorInvalidValue;
}

}  // namespace lvx
