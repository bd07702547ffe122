// Forward block partials on the tcgen05 tensor cores (bf16 inputs, fp32
// accumulation and softmax statistics, head width 64 or 128).
//
// What one CTA computes: for 256 query rows (two 128-row tiles) of one
// (batch, head) and one stationary key/value block i, the block's partial
// output O_i and log-sum-exp L_i (LV-XAttn review page, Figure 3 /
// Algorithm 1: each KV block produces (O_i, L_i) for the queries it sees;
// Ring Attention citation hub page, abstract: exact blockwise attention).
// Inside the block the 128-key tiles are folded in with an online softmax;
// the running maximum is only moved when it grows by more than 2^8 (the
// exponentials stay below 256, so the deferred rescaling is exact).
//
// Roles (12 warps):
//   warp 0      TMA producer: Q tiles once, K (3-stage) and V (2-stage) rings
//   warp 1      MMA issuer:   S_t = Q_t K^T (SS form) and O_t += P_t V (TS form,
//                             P read from TMEM)
//   warp 2      TMEM allocator (512 columns)
//   warps 4-7   softmax for Q tile 0, warps 8-11 for Q tile 1: one thread per
//               row reads S from TMEM, writes P (bf16) back over S, rescales O
//               when needed, and finally normalises O and writes the partial.
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256,256+D), O_1 [256+D,256+2D).
// A new S_t is issued only after the P_t V MMA that reads P_t from S_t's
// columns (the MMAs of one thread execute in issue order, so that read comes
// first), and O_t is only rescaled between two P_t V MMAs.
#include "lvx_ptx.cuh"
#include "lvx_tc.cuh"

namespace lvx {
namespace {

using namespace ptx;

constexpr int BQ = 128;           // query rows per tile (MMA M)
constexpr int BKV = 128;          // keys per tile
constexpr int NQT = 2;            // query tiles per CTA
constexpr int K_STAGES = 3;   // K is needed a full softmax earlier than V: prefetch it deeper
constexpr int V_STAGES = 2;
constexpr int kThreads = 384;
// Register split: launched at 168 per thread (384 x 168 = 64512); warpgroup 0
// (producer, MMA issuer, allocator) gives up 64, the two softmax warpgroups
// take 32 each: 128 x 104 + 256 x 200 = 64512.
constexpr uint32_t kRegsControl = 104;
constexpr uint32_t kRegsSoftmax = 200;
static_assert(128 * kRegsControl + 256 * kRegsSoftmax <= 65536 / kThreads * kThreads,
              "register split exceeds the launch allocation");
constexpr uint32_t CHUNK = 128 * 128;   // one TMA box: 128 rows x 64 bf16 (128 B), swizzled
constexpr float kRescaleThreshold = 8.0f;   // log2 units
constexpr float kRescaleFactor = 256.0f;    // 2^kRescaleThreshold
constexpr float kLn2 = 0.6931471805599453f;

template <int D>
struct FwdLayout {
  static constexpr uint32_t TILE = 128 * D * 2;   // Q, K or V tile
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + NQT * TILE;
  static constexpr uint32_t OFF_V = OFF_K + K_STAGES * TILE;
  static constexpr uint32_t OFF_BAR = OFF_V + V_STAGES * TILE;
  static constexpr uint32_t USED = OFF_BAR + 256 + 1024;
  // at least ~116 KiB so that one CTA (and its 512 TMEM columns) owns the SM
  static constexpr uint32_t BYTES = USED > 118784 ? USED : 118784;
  static constexpr uint32_t IDESC_QK = ptx::idesc_bf16_f32(128, 128, false, false);
  static constexpr uint32_t IDESC_PV = ptx::idesc_bf16_f32(128, D, false, true);
};

struct FwdArgs {
  Problem p;
  __nv_bfloat16* out;   // final output (when o_parts is null)
  float* lse;
  float* o_parts;       // block partials (null: write the final output)
  float* l_parts;
  unsigned int* err;
  int n_qp;             // query tile pairs per (batch, head)
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
fwd_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
              const __grid_constant__ CUtensorMap map_v, const FwdArgs a) {
  using L = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k0_full = bars + 1;    // K_0
  uint64_t* kv_full = bars + 2;    // [2]: K_{j+1} and V_j landed (step j, slot j mod 2)
  uint64_t* k_empty = bars + 4;    // [K_STAGES]
  uint64_t* v_empty = bars + 7;    // [V_STAGES]
  uint64_t* s_full = bars + 9;
  uint64_t* p_full = bars + 11;
  uint64_t* o_done = bars + 13;
  uint64_t* mma_drain = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const Problem& p = a.p;
  int idx = blockIdx.x;
  const int qp = idx % a.n_qp;
  idx /= a.n_qp;
  const int h = idx % p.H;
  idx /= p.H;
  const int blk = idx % p.n_blocks;
  const int b = idx / p.n_blocks;
  const int g = h / (p.H / p.H_kv);
  const int m0 = qp * (NQT * BQ);
  const int kb0 = min(blk * p.block_len, p.S_KV);
  const int kb1 = min(kb0 + p.block_len, p.S_KV);
  int kend = kb1;
  if (p.causal) {
    const int last_row = min(m0 + NQT * BQ, p.S_Q) - 1;
    if (blk > last_row / p.block_len) return;   // block pair skipped: no row of this CTA needs it
    kend = min(kend, last_row + 1);
  }
  const int T = kend > kb0 ? (kend - kb0 + BKV - 1) / BKV : 0;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    ptx::mbar_init(q_full, 1);
    ptx::mbar_init(k0_full, 1);
    ptx::mbar_init(&kv_full[0], 1);
    ptx::mbar_init(&kv_full[1], 1);
    for (int s = 0; s < K_STAGES; ++s) ptx::mbar_init(&k_empty[s], 1);
    for (int s = 0; s < V_STAGES; ++s) ptx::mbar_init(&v_empty[s], 1);
    for (int t = 0; t < NQT; ++t) {
      ptx::mbar_init(&s_full[t], 1);
      ptx::mbar_init(&p_full[t], 128);
      ptx::mbar_init(&o_done[t], 1);
    }
    ptx::mbar_init(mma_drain, 1);
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
  if (warp < 4) {
    ptx::setmaxnreg_dec<kRegsControl>();
    if (warp == 0) {
      if (lane == 0 && T > 0) {
        // ---------------------------------------------------------------- producer
        ptx::tma_prefetch_desc(&map_q);
        ptx::tma_prefetch_desc(&map_k);
        ptx::tma_prefetch_desc(&map_v);
        ptx::mbar_arrive_expect_tx(q_full, NQT * L::TILE);
        for (int t = 0; t < NQT; ++t)
          for (int c = 0; c < D / 64; ++c)
            ptx::tma_load_4d(smem + L::OFF_Q + t * L::TILE + c * CHUNK, &map_q, q_full, 64 * c, h,
                             m0 + BQ * t, b);
        // K_0 on a barrier of its own, then per step j one barrier for K_{j+1} and V_j:
        // the MMA issuer waits once per step for both (a satisfied wait still keeps the
        // issuing thread, and with it the tensor pipe, idle for ~125 cycles).  Slot j mod 2
        // is re-armed only after PV1 of step j-2 has read V_{j-2}, by which time the issuer
        // has long consumed that slot's previous phase.
        ptx::mbar_arrive_expect_tx(k0_full, L::TILE);
        for (int c = 0; c < D / 64; ++c)
          ptx::tma_load_4d(smem + L::OFF_K + c * CHUNK, &map_k, k0_full, 64 * c, g, kb0, b);
        int issued = 0;   // steps whose loads were issued
        bool ok = true;
        for (int j = 0; j < T && ok; ++j) {
          const bool more = j + 1 < T;
          const int ks = (j + 1) % K_STAGES, vs = j % V_STAGES;
          if (more && !ptx::mbar_wait(&k_empty[ks], (((j + 1) / K_STAGES) & 1) ^ 1, a.err,
                                      kErrTimeoutTma, abort_flag))
            break;
          if (!ptx::mbar_wait(&v_empty[vs], ((j / V_STAGES) & 1) ^ 1, a.err, kErrTimeoutTma, abort_flag))
            break;
          uint64_t* bar = &kv_full[j & 1];
          ptx::mbar_arrive_expect_tx(bar, more ? 2 * L::TILE : L::TILE);
          if (more) {
            for (int c = 0; c < D / 64; ++c)
              ptx::tma_load_4d(smem + L::OFF_K + ks * L::TILE + c * CHUNK, &map_k, bar, 64 * c, g,
                               kb0 + BKV * (j + 1), b);
          }
          for (int c = 0; c < D / 64; ++c)
            ptx::tma_load_4d(smem + L::OFF_V + vs * L::TILE + c * CHUNK, &map_v, bar, 64 * c, g,
                             kb0 + BKV * j, b);
          issued = j + 1;
        }
        if (*abort_flag) {
          // the copies already issued must land before shared memory is released
          ptx::mbar_wait(q_full, 0, a.err, kErrTimeoutTma, nullptr);
          ptx::mbar_wait(k0_full, 0, a.err, kErrTimeoutTma, nullptr);
          for (int j = issued > 2 ? issued - 2 : 0; j < issued; ++j)
            ptx::mbar_wait(&kv_full[j & 1], (j >> 1) & 1, a.err, kErrTimeoutTma, nullptr);
        }
      }
    } else if (warp == 1) {
      if (lane == 0) {
        // ---------------------------------------------------------------- MMA issuer
        // Issue order: S0_0, S1_0, PV0_0, then per tile j >= 1
        //   S0_j, PV1_{j-1}, S1_j, PV0_j,  and finally PV1_{T-1}.
        // Softmax of Q tile 0 on S0_j overlaps PV1_{j-1} and S1_j on the tensor
        // core, softmax of tile 1 overlaps PV0_j and S0_{j+1}, so the two softmax
        // groups take turns on the exponential unit.  S_t of tile j overwrites
        // P_t of tile j-1 right after the MMA that reads it; tcgen05.mma ops of
        // one thread execute in issue order, so that read completes first.
        if (T > 0 && ptx::mbar_wait(q_full, 0, a.err, kErrTimeoutMma, abort_flag)) {
          // Shared-memory descriptors: only the low words (address >> 4 and lbo)
          // differ between operands, so the Q, K-stage and V-stage low words are
          // kept and each K step adds a compile-time offset; the high word
          // (sbo 1024, version, 128-byte swizzle) is a constant.  The issuing
          // thread shares its sub-partition with two softmax warps, so every
          // instruction saved here shortens the PV -> S hand-off on the
          // critical path.  Addresses stay below 2^18: no carry into lbo.
          constexpr uint32_t kT16 = L::TILE >> 4;
          constexpr uint32_t kMN = ((CHUNK >> 4) - 1u) << 16;   // lbo 16 -> lbo CHUNK
          const uint32_t dQ0 = (ptx::smem_u32(smem + L::OFF_Q) >> 4) | (1u << 16);
          const uint32_t dK0 = (ptx::smem_u32(smem + L::OFF_K) >> 4) | (1u << 16);
          const uint32_t dV0 = (ptx::smem_u32(smem + L::OFF_V) >> 4) | (1u << 16);
          auto desc = [](uint32_t lo) {
            return ((uint64_t)((1024u >> 4) | (1u << 14) | (2u << 29)) << 32) | lo;
          };
          uint32_t dKs = dK0, dVs = dV0;   // this tile's K and V stages
          auto issue_s = [&](int t) {
            const uint32_t dq = dQ0 + t * kT16;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = ((kk >> 2) * CHUNK + (kk & 3) * 32) >> 4;
              ptx::mma_ss(tmem + t * 128, desc(dq + off), desc(dKs + off), L::IDESC_QK,
                          kk > 0 ? 1u : 0u);
            }
            ptx::mma_commit(&s_full[t]);
          };
          auto issue_pv = [&](int t, uint32_t dv, bool first) {
#pragma unroll
            for (int kk = 0; kk < BKV / 16; ++kk)
              ptx::mma_ts(tmem + 256 + t * D, tmem + t * 128 + kk * 8,
                          desc(dv + (kMN + kk * (2048 >> 4))), L::IDESC_PV,
                          (!first || kk > 0) ? 1u : 0u);
            ptx::mma_commit(&o_done[t]);
          };
          uint32_t dVprev = dV0;   // V stage of tile j-1
          bool ok = true;
          for (int j = 0; j < T && ok; ++j) {
            // K_0 has a barrier of its own; K_j (j > 0) came with V_{j-1}, waited for below
            if (j == 0) ok = ptx::mbar_wait(k0_full, 0, a.err, kErrTimeoutMma, abort_flag);
            if (!ok) break;
            ptx::tc_fence_after();
            issue_s(0);
            if (j > 0) {
              // PV1 of the previous tile (its V stage is released afterwards)
              ok = ptx::mbar_wait(&p_full[1], (j - 1) & 1, a.err, kErrTimeoutMma, abort_flag);
              if (!ok) break;
              ptx::tc_fence_after();
              issue_pv(1, dVprev, j == 1);
              ptx::mma_commit(&v_empty[(j - 1) % V_STAGES]);
            }
            issue_s(1);
            ptx::mma_commit(&k_empty[j % K_STAGES]);
            ok = ptx::mbar_wait(&kv_full[j & 1], (j >> 1) & 1, a.err, kErrTimeoutMma, abort_flag);
            if (ok) ok = ptx::mbar_wait(&p_full[0], j & 1, a.err, kErrTimeoutMma, abort_flag);
            if (!ok) break;
            ptx::tc_fence_after();
            issue_pv(0, dVs, j == 0);
            dVprev = dVs;
            dKs = (j % K_STAGES == K_STAGES - 1) ? dK0 : dKs + kT16;
            dVs = (j % V_STAGES == V_STAGES - 1) ? dV0 : dVs + kT16;
          }
          if (ok && ptx::mbar_wait(&p_full[1], (T - 1) & 1, a.err, kErrTimeoutMma, abort_flag)) {
            ptx::tc_fence_after();
            issue_pv(1, dVprev, T == 1);
            ptx::mma_commit(&v_empty[(T - 1) % V_STAGES]);
          }
        }
        ptx::mma_commit(mma_drain);
      }
    }
  } else {
    ptx::setmaxnreg_inc<kRegsSoftmax>();
    // ------------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row_in_tile = quarter * 32 + lane;
    const int row0_tile = m0 + BQ * t;
    const int row = row0_tile + row_in_tile;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + 256 + t * D;
    const float sl2 = p.scale_log2;
    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      ok = ptx::mbar_wait(&s_full[t], j & 1, a.err, kErrTimeoutSoftmax, abort_flag);
      ok = __all_sync(0xffffffffu, ok);   // keep the warp converged for tcgen05.ld/st
      if (!ok) break;
      ptx::tc_fence_after();
      uint32_t sr[128];
      // keys 64..127 load while the exponentials of keys 0..63 are computed
      ptx::tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      ptx::tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      ptx::tmem_wait_ld();
      ptx::tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
      ptx::tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
      // the second wait, after which the compiler must treat keys 64..127 as
      // written (the load's register outputs are only valid from here on)
      auto wait_upper = [&]() {
        ptx::tmem_wait_ld();
#pragma unroll
        for (int i = 64; i < 128; i += 8)
          asm volatile("" : "+r"(sr[i]), "+r"(sr[i + 1]), "+r"(sr[i + 2]), "+r"(sr[i + 3]),
                       "+r"(sr[i + 4]), "+r"(sr[i + 5]), "+r"(sr[i + 6]), "+r"(sr[i + 7]));
      };
      const int key0 = kb0 + BKV * j;
      const bool need_mask = (key0 + BKV > kb1) || (p.causal && key0 + BKV - 1 > row0_tile);
      // Steady state (an unmasked tile once the row has a running maximum): P is
      // computed with the running maximum straight away, with no pass for the
      // tile's maximum.  Only if some exponential may exceed 2^threshold (for
      // any row of the warp) is that P discarded -- nothing has been released
      // yet -- and the tile redone below with the maximum moved, exactly as a
      // first tile is.
      bool done = false;
      if (!need_mask && m_ref != -INFINITY) {
        const uint64_t sl2x2 = pk2(sl2, sl2);
        const uint64_t negm2 = pk2(-m_ref, -m_ref);
        uint64_t acc2 = pk2(0.f, 0.f), acc2b = pk2(0.f, 0.f);
        float xp = -INFINITY;   // largest argument among the FMA-pipe exponentials
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c == 2) wait_upper();
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float s0 = __uint_as_float(sr[32 * c + 2 * i]);
            const float s1 = __uint_as_float(sr[32 * c + 2 * i + 1]);
            const uint64_t x2 = ffma2(pk2(s0, s1), sl2x2, negm2);
            uint64_t e2;
            if (i % kPolyEvery == kPolyEvery - 1) {
              float x0, x1;
              upk2(x2, x0, x1);
              xp = fmax3(xp, x0, x1);
              e2 = exp2_poly2(x2);
            } else {
              float x0, x1;
              upk2(x2, x0, x1);
              e2 = pk2(ex2(x0), ex2(x1));
            }
            if (i & 1) acc2b = fadd2(acc2b, e2); else acc2 = fadd2(acc2, e2);
            float p0, p1;
            upk2(e2, p0, p1);
            pk[i] = ptx::pack_bf16x2(p0, p1);
          }
          ptx::tmem_st16(tS + 16 * c, pk);
        }
        // Accepted only if every exponential is at most 2^threshold.  A sum of
        // positive terms bounds each of them; an SFU exponential of a larger
        // argument is large or +inf, and a NaN fails the test as well.  The
        // FMA-pipe exponential is valid only for arguments up to 127, so its
        // arguments are checked directly.
        float a0, a1;
        upk2(fadd2(acc2, acc2b), a0, a1);
        const float tile_sum = a0 + a1;
        const bool fits = tile_sum <= kRescaleFactor && xp <= kRescaleThreshold;
        if (__all_sync(0xffffffffu, fits)) {
          l_sum += tile_sum;
          done = true;
        }
      } else {
        wait_upper();
      }
      if (!done) {
        if (need_mask) {
          const int lim = p.causal ? min(kb1, row + 1) : kb1;   // keys [key0, lim) visible
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (key0 + i >= lim) sr[i] = __float_as_uint(-INFINITY);
        }
        // row max: four independent chains of 3-input maxima (a single chain is
        // latency-bound), then combined
        float m4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) m4[q] = fmaxf(__uint_as_float(sr[32 * q]), __uint_as_float(sr[32 * q + 1]));
#pragma unroll
        for (int i = 2; i < 32; i += 2)
#pragma unroll
          for (int q = 0; q < 4; ++q)
            m4[q] = fmax3(m4[q], __uint_as_float(sr[32 * q + i]), __uint_as_float(sr[32 * q + i + 1]));
        const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        const float m_tile = mx * sl2;
        const bool resc = m_tile > m_ref + kRescaleThreshold;
        float alpha = 1.f;
        if (resc) {
          alpha = ex2(m_ref - m_tile);   // 0 when m_ref is -inf
          m_ref = m_tile;
          l_sum *= alpha;
        }
        if (j > 0 && __any_sync(0xffffffffu, resc)) {
          // O_t is quiescent here: P_t V of tile j-1 finished before S_t of tile j was issued
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            ptx::tmem_ld32(tO + c * 32, o);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            ptx::tmem_st32(tO + c * 32, o);
          }
        }
        const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
        if (need_mask) {
          // masked tiles: every exponential on the special-function unit (exact 0 for -inf)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float p0 = ex2(fmaf(__uint_as_float(sr[32 * c + 2 * i]), sl2, -m_use));
              const float p1 = ex2(fmaf(__uint_as_float(sr[32 * c + 2 * i + 1]), sl2, -m_use));
              l_sum += p0 + p1;
              pk[i] = ptx::pack_bf16x2(p0, p1);
            }
            ptx::tmem_st16(tS + 16 * c, pk);
          }
        } else {
          // packed pairs: x = s*scale - m with FFMA2, one pair in kPolyEvery through the
          // FMA-pipe polynomial and the rest on the SFU, row sum with FADD2
          const uint64_t sl2x2 = pk2(sl2, sl2);
          const uint64_t negm2 = pk2(-m_use, -m_use);
          uint64_t acc2 = pk2(0.f, 0.f);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const uint64_t s2 = pk2(__uint_as_float(sr[32 * c + 2 * i]),
                                      __uint_as_float(sr[32 * c + 2 * i + 1]));
              const uint64_t x2 = ffma2(s2, sl2x2, negm2);
              uint64_t e2;
              if (i % kPolyEvery == kPolyEvery - 1) {
                e2 = exp2_poly2(x2);
              } else {
                float x0, x1;
                upk2(x2, x0, x1);
                e2 = pk2(ex2(x0), ex2(x1));
              }
              acc2 = fadd2(acc2, e2);
              float p0, p1;
              upk2(e2, p0, p1);
              pk[i] = ptx::pack_bf16x2(p0, p1);
            }
            ptx::tmem_st16(tS + 16 * c, pk);
          }
          float a0, a1;
          upk2(acc2, a0, a1);
          l_sum += a0 + a1;
        }
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&p_full[t]);
    }
    // ---------------------------------------------------------------- epilogue
    if (T > 0 && ok) ok = ptx::mbar_wait(&o_done[t], (T - 1) & 1, a.err, kErrTimeoutEpilogue, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    ptx::tc_fence_after();
    const bool seen = T > 0 && l_sum > 0.f;
    const float inv_l = seen ? 1.f / l_sum : 0.f;
    const float Lrow = seen ? (m_ref + __log2f(l_sum)) * kLn2 : -INFINITY;
    const bool write = ok && row < p.S_Q;
    const size_t prow = (((size_t)blk * p.B + b) * p.H + h) * p.S_Q + row;
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      if (T > 0 && ok) {
        ptx::tmem_ld32(tO + c * 32, o);
        ptx::tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0u;
      }
      if (!write) continue;
      if (a.o_parts == nullptr) {   // the final output (one block), else the block partials
        uint4* dst = reinterpret_cast<uint4*>(
            a.out + (((size_t)b * p.S_Q + row) * p.H + h) * D + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 u;
          u.x = ptx::pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv_l, __uint_as_float(o[8 * q + 1]) * inv_l);
          u.y = ptx::pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv_l, __uint_as_float(o[8 * q + 3]) * inv_l);
          u.z = ptx::pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv_l, __uint_as_float(o[8 * q + 5]) * inv_l);
          u.w = ptx::pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv_l, __uint_as_float(o[8 * q + 7]) * inv_l);
          dst[q] = u;
        }
      } else {
        float4* dst = reinterpret_cast<float4*>(a.o_parts + prow * D + c * 32);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          dst[q] = make_float4(__uint_as_float(o[4 * q + 0]) * inv_l, __uint_as_float(o[4 * q + 1]) * inv_l,
                               __uint_as_float(o[4 * q + 2]) * inv_l, __uint_as_float(o[4 * q + 3]) * inv_l);
      }
    }
    if (write) {
      if (a.o_parts == nullptr)
        a.lse[((size_t)b * p.H + h) * p.S_Q + row] = Lrow;
      else
        a.l_parts[prow] = Lrow;
    }
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
cudaError_t launch(const Problem& p, const void* q, const void* k, const void* v, void* out,
                   float* lse, float* o_parts, float* l_parts, cudaStream_t s) {
  using L = FwdLayout<D>;
  CUtensorMap mq, mk, mv;
  const uint32_t box[4] = {64, 1, 128, 1};
  {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)p.H, (uint64_t)p.S_Q, (uint64_t)p.B};
    const uint64_t str[3] = {(uint64_t)D * 2, (uint64_t)p.H * D * 2, (uint64_t)p.S_Q * p.H * D * 2};
    if (!encode_tensor_map(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, q, dims, str, box,
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
  }
  FwdArgs a;
  a.p = p;
  a.out = reinterpret_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.o_parts = o_parts;
  a.l_parts = l_parts;
  a.err = device_error_word();
  a.n_qp = (p.S_Q + NQT * BQ - 1) / (NQT * BQ);
  if (!a.err) return cudaErrorInvalidValue;
  const long long grid = (long long)a.n_qp * p.H * p.n_blocks * p.B;
  if (grid > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(fwd_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       L::BYTES);
  if (e != cudaSuccess) return e;
  fwd_tc_kernel<D><<<(unsigned)grid, kThreads, L::BYTES, s>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace

bool tc_fwd_supported(const Problem& p) { return p.d == 64 || p.d == 128; }

cudaError_t launch_fwd_tc(const Problem& p, const void* q, const void* k, const void* v,
                          void* out, float* lse, float* o_parts, float* l_parts, cudaStream_t s) {
  if (p.d == 128) return launch<128>(p, q, k, v, out, lse, o_parts, l_parts, s);
  if (p.d == 64) return launch<64>(p, q, k, v, out, lse, o_parts, l_parts, s);
  return cudaErrorInvalidValue;
}

}  // namespace lvx
