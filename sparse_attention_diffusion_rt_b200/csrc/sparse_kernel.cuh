// Persistent sm_100a kernel for Re-ttention's reshaped sparse step,
//   O'_i = rho_hat_i * softmax over the kept key blocks (s'_i) . v'  +  R_i
// (O'_i = R_i for a query block with no kept key block), with
// rho_hat = min(1, rho * ramp_mul + ramp_add)  ("Re-ttention", OpenReview
// replies to W1: the sparse softmax rescaled by the cached denominator ratio,
// plus the cached residual of the masked tokens; reply to Pwod's W1: ramp-up).
//
// One CTA per SM walks the (batch, head, query block) tiles tile = blockIdx.x
// + i * gridDim.x, query block fastest (see sp_decode).  Roles (320 threads):
//   warps 0-3  softmax; thread t owns tile row t (TMEM lane t).  At the end of
//              a tile it hands the row sum l to the epilogue (through a TMEM
//              column) and goes straight on to the next tile.
//   warps 4-7  epilogue; thread 128 + t owns row t.  It drains the tile's O from
//              TMEM as soon as the last PV lands (releasing the accumulator
//              for the next tile's first PV), then applies rho_hat / l, adds
//              the residual tile and stores the bf16 result through a
//              shared-memory staging tile and a TMA store, while the softmax
//              warps already work on the next tile.
//   warp 8     producer: lane 0 validates each tile's CSR row and loads Q
//              (one buffer, free again once Q is in TMEM), the K tiles of the
//              kept blocks and the residual tile; lane 1 loads the V tiles.  K
//              and V have their own NST-stage rings, released after QK^T and
//              after PV.
//   warp 9     lane 0 issues the tcgen05 MMAs: it copies each tile's Q into
//              TMEM (tcgen05.cp), then S = Q K^T into one of two TMEM logit
//              buffers with Q read from TMEM, O += P V with P read from TMEM,
//              so only K and V are read from shared memory.  The softmax
//              writes P over its own logits, so the MMA warp issues PV(j) and
//              then QK^T(j+2) into the same buffer: MMAs of one thread run in
//              issue order, so the logits are never overwritten early and the
//              tensor pipe always has the next logits queued.
// Tile metadata flows through a 2-slot ring (ti_*), the epilogue's share of it
// (kept-block count, row sums) through a second 2-slot ring (epi_*).  Every
// per-block barrier phase is indexed by a block counter that runs across
// tiles, so the MMA warp starts the next tile's QK^T while the last PV of the
// previous one runs.
//
// TMEM columns: S0/S1 [0,256) fp32 logits, each overwritten in place by its
// bf16 probabilities P (64 columns of the 128), Q [256, 256+DPAD/2) as bf16
// pairs, the row sums of the two epilogue slots at 376 and 377, O [384,
// 384+DPAD).  All waits are bounded; a timeout records RT_ERR_TIMEOUT and
// every role drains what it has in flight before TMEM is freed.
#pragma once
#include <cuda.h>
#include <cstdint>

#include "attn_kernel.cuh"
#include "ptx.cuh"
#include "softmax.cuh"

namespace rtb {

template <int DPAD>
struct SpCfg {
  static constexpr int BN = 128;
  static constexpr int C1 = DPAD - 64;
  static constexpr int C1B = C1 * 2;
  static constexpr uint32_t C1SWZ = C1 == 16 ? SWZ_32B : (C1 == 32 ? SWZ_64B : SWZ_128B);
  // Q is copied into TMEM at the start of its tile, so one shared-memory buffer
  // is enough; the rest goes to the K/V ring (4 stages at DPAD 80, 3 at 96, 2 at
  // 128) and one output staging tile.
  static constexpr int QBUF = 1;
  static constexpr int OSTG = 1;
  static constexpr int TILE_BYTES = 128 * DPAD * 2;          // one bf16 [128][DPAD] tile
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;          // K + V
  static constexpr int OFF_Q = 1024;
  static constexpr int OFF_STAGE = OFF_Q + QBUF * TILE_BYTES;
  static constexpr int NST_FIT = (232448 - 1024 - OFF_STAGE - (1 + OSTG) * TILE_BYTES) / STAGE_BYTES;
  static constexpr int NST = NST_FIT > 4 ? 4 : NST_FIT;
  static constexpr int OFF_R = OFF_STAGE + NST * STAGE_BYTES;
  static constexpr int OFF_OST = OFF_R + TILE_BYTES;
  static constexpr int SMEM = OFF_OST + OSTG * TILE_BYTES + 1024;   // + alignment slack
  static_assert(NST >= 2, "at least two K/V stages");
  static_assert(SMEM <= 232448, "shared memory per CTA");
  static constexpr uint32_t T_S = 0, T_Q = 256, T_L = 376, T_O = 384;   // S_b (P_b over it), Q, l, O
  static_assert(T_Q + DPAD / 2 <= T_L && T_L + 2 <= T_O, "Q (bf16 pairs) and the row sums fit below O");
};

// Roles of the sparse-step kernel: three warpgroups.  Each sub-partition of
// the SM holds one warp of each, so the launch gives every thread 168
// registers (3 x 32 x 168 of a sub-partition's 16384); the warpgroups then
// rebalance: the softmax holds a 128-logit row in registers, the epilogue a
// whole O row, the producer / MMA warpgroup gives back down to 80.  The split
// between the first two follows the head dimension (the epilogue's row is DPAD
// wide): 248 / 176 at DPAD 128, 256 / 168 below; either way 128 x (softmax +
// epilogue + 80) = 64512 = 384 x 168, the .inc of the first two exactly using
// what the .dec of the third returns.
constexpr int kSpThreads = 384;
constexpr int kSpEpiThread0 = 128;     // warps 4-7: epilogue
constexpr int kSpProducerWarp = 8;
constexpr int kSpMmaWarp = 9;          // warps 10-11 idle
constexpr uint32_t kSpRegsLaunch = 168, kSpRegsOther = 80;
template <int DPAD>
struct SpRegs {
  static constexpr uint32_t softmax = DPAD == 128 ? 248 : 256;
  static constexpr uint32_t epilogue = DPAD == 128 ? 176 : 168;
  static_assert(kSpRegsLaunch * kSpThreads <= 65536 && 3 * 32 * kSpRegsLaunch <= 16384,
                "launch registers fit the register file and each sub-partition");
  static_assert(32 * (softmax + epilogue + kSpRegsOther) <= 16384,
                "after the split, one warp of each warpgroup still fits a sub-partition");
  static_assert(128 * (softmax + epilogue + kSpRegsOther) <= kSpThreads * kSpRegsLaunch,
                "the warpgroups' shares fit the pool the CTA was launched with");
  static_assert(softmax % 8 == 0 && epilogue % 8 == 0 && kSpRegsOther % 8 == 0 && softmax <= 256,
                "setmaxnreg counts");
};

struct SpTile {
  int b, h, qb, n, start, bad;
  int tail_j, tail_valid;   // block index (in this row) that holds the sequence end, keys of it inside
};

struct SpCtrl {
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[4], v_full[4], k_empty[4], v_empty[4];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t o_full;
  uint64_t r_full, r_empty;
  uint64_t ti_full[2], ti_empty[2];
  uint64_t stg_ready, stg_full;
  uint64_t o_free, epi_full[2], epi_empty[2];
  uint64_t drain;
  SpTile ti[2];
  int epi_n[2], epi_bad[2];   // the epilogue's share of a tile's metadata
  uint32_t tmem_base;
  volatile int abort_flag;
};
static_assert(sizeof(SpCtrl) <= 1024, "control block");

template <typename CtrlT>
__device__ __forceinline__ bool sp_wait(uint64_t* bar, uint32_t parity, CtrlT& ctl, const AttnParams& p) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++spins & 31u) == 0) {
      if (ctl.abort_flag) return false;
      if (globaltimer_ns() - t0 > p.wait_limit_ns) {
        ctl.abort_flag = 1;
        record_status(p.status, RT_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Tile order: query block fastest within a (batch, head).  The CTAs in flight
// then cover a contiguous range of query blocks of one head, whose kept key
// blocks (local windows) overlap, so each K/V block is fetched from DRAM about
// once and re-read from L2.  (A (batch, head)-fastest order measured 8x the
// compulsory DRAM traffic on the long-video masks: reuse distance beyond L2.)
__device__ __forceinline__ void sp_decode(const AttnParams& p, int tile, int& b, int& h, int& qb) {
  qb = tile % p.nqb;
  const int bh = tile / p.nqb;
  b = bh / p.H;
  h = bh % p.H;
}

// ------------------------------------------------------------------ producer
// Lane 0: tile metadata (CSR row validation), Q, K tiles, residual tile.
// Lane 1: V tiles.  The two lanes run independent loops.
template <int DPAD>
__device__ __forceinline__ void sp_producer(const TmaSet& tm, const AttnParams& p, SpCtrl& ctl, uint8_t* base,
                                            int ntiles) {
  using C = SpCfg<DPAD>;
  const int lane = threadIdx.x & 31;
  if (lane > 1) return;
  uint8_t* sQ = base + C::OFF_Q;
  uint8_t* sStage = base + C::OFF_STAGE;
  uint8_t* sR = base + C::OFF_R;
  uint32_t g = 0, qi = 0, ri = 0;          // block, Q-load and R-load counters of this lane
  bool ok = true;
  int it = 0;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int slot = it & 1;
    int n = 0, start = 0, b = 0, h = 0, qb = 0;
    if (lane == 0) {
      if (it >= 2 && !sp_wait(&ctl.ti_empty[slot], ((it >> 1) - 1) & 1, ctl, p)) { ok = false; break; }
      sp_decode(p, tile, b, h, qb);
      const int row = (p.Hm == 1 ? 0 : h) * p.nqb + qb;
      start = __ldg(p.row_ptr + row);
      const int end = __ldg(p.row_ptr + row + 1);
      int bad = (start < 0 || end < start || static_cast<long long>(end) > p.nnz || end - start > p.nkb) ? 1 : 0;
      if (!bad) {
        int prev = -1;
        for (int i = start; i < end; ++i) {
          const int c = __ldg(p.col_idx + i);
          if (c <= prev || c >= p.nkb) { bad = 1; break; }
          prev = c;
        }
      }
      n = bad ? 0 : end - start;
      int tail_j = -1;
      const int tail_valid = p.L - (p.nkb - 1) * 128;
      if (!bad && n > 0 && tail_valid < 128 && __ldg(p.col_idx + end - 1) == p.nkb - 1) tail_j = n - 1;
      ctl.ti[slot] = SpTile{b, h, qb, n, start, bad, tail_j, tail_valid};
      if (bad) record_status(p.status, RT_ERR_BAD_INDEX);
      mbar_arrive(&ctl.ti_full[slot]);
      if (bad) continue;
      const int q_row = qb * 128;
      if (n > 0) {
        const int qs = C::QBUF == 2 ? (qi & 1) : 0;
        if (qi >= static_cast<uint32_t>(C::QBUF) &&
            !sp_wait(&ctl.q_empty[qs], ((qi / C::QBUF) - 1) & 1, ctl, p)) { ok = false; break; }
        uint8_t* q = sQ + qs * C::TILE_BYTES;
        mbar_arrive_expect_tx(&ctl.q_full[qs], C::TILE_BYTES);
        tma_load_4d(q, &tm.q[0], &ctl.q_full[qs], 0, q_row, h, b);
        if (C::C1) tma_load_4d(q + 128 * 128, &tm.q[1], &ctl.q_full[qs], 64, q_row, h, b);
        ++qi;
        for (int j = 0; j < n; ++j, ++g) {
          const int st = g % C::NST;
          if (g >= static_cast<uint32_t>(C::NST) &&
              !sp_wait(&ctl.k_empty[st], ((g / C::NST) - 1) & 1, ctl, p)) { ok = false; break; }
          const int kb = __ldg(p.col_idx + start + j);
          uint8_t* sK = sStage + st * C::STAGE_BYTES;
          mbar_arrive_expect_tx(&ctl.k_full[st], C::TILE_BYTES);
          tma_load_4d(sK, &tm.k[0], &ctl.k_full[st], 0, kb * 128, h, b);
          if (C::C1) tma_load_4d(sK + 128 * 128, &tm.k[1], &ctl.k_full[st], 64, kb * 128, h, b);
        }
        if (!ok) break;
      }
      if (!p.r_f32 && p.use_r) {
        if (ri >= 1 && !sp_wait(&ctl.r_empty, (ri - 1) & 1, ctl, p)) { ok = false; break; }
        mbar_arrive_expect_tx(&ctl.r_full, C::TILE_BYTES);
        tma_load_4d(sR, &tm.r[0], &ctl.r_full, 0, q_row, h, b);
        if (C::C1) tma_load_4d(sR + 128 * 128, &tm.r[1], &ctl.r_full, 64, q_row, h, b);
        ++ri;
      }
    } else {
      if (!sp_wait(&ctl.ti_full[slot], (it >> 1) & 1, ctl, p)) { ok = false; break; }
      const SpTile ti = ctl.ti[slot];
      mbar_arrive(&ctl.ti_empty[slot]);
      for (int j = 0; j < ti.n; ++j, ++g) {
        const int st = g % C::NST;
        if (g >= static_cast<uint32_t>(C::NST) &&
            !sp_wait(&ctl.v_empty[st], ((g / C::NST) - 1) & 1, ctl, p)) { ok = false; break; }
        const int kb = __ldg(p.col_idx + ti.start + j);
        uint8_t* sV = sStage + st * C::STAGE_BYTES + C::TILE_BYTES;
        mbar_arrive_expect_tx(&ctl.v_full[st], C::TILE_BYTES);
        tma_load_4d(sV, &tm.v[0], &ctl.v_full[st], 0, kb * 128, ti.h, ti.b);
        if (C::C1) tma_load_4d(sV + 128 * 128, &tm.v[1], &ctl.v_full[st], 64, kb * 128, ti.h, ti.b);
      }
      if (!ok) break;
    }
  }
  if (!ok) {
    // let every copy this lane started land before shared memory is released
    const uint64_t lim = p.wait_limit_ns;
    if (lane == 0) {
      for (uint32_t i = (qi > static_cast<uint32_t>(C::QBUF) ? qi - C::QBUF : 0); i < qi; ++i)
        drain_wait(&ctl.q_full[C::QBUF == 2 ? (i & 1) : 0], (i / C::QBUF) & 1, lim);
      if (ri >= 1) drain_wait(&ctl.r_full, (ri - 1) & 1, lim);
    }
    for (uint32_t i = (g > static_cast<uint32_t>(C::NST) ? g - C::NST : 0); i < g; ++i)
      drain_wait(lane == 0 ? &ctl.k_full[i % C::NST] : &ctl.v_full[i % C::NST], (i / C::NST) & 1, lim);
  }
}

// ------------------------------------------------------------------ MMA issuer
template <int DPAD>
__device__ __forceinline__ void sp_mma(const AttnParams& p, SpCtrl& ctl, uint8_t* base, uint32_t tmem, int ntiles) {
  using C = SpCfg<DPAD>;
  constexpr uint32_t IDESC_QK = make_idesc_bf16(128, 128, 0, 0);
  constexpr uint32_t IDESC_PV_FULL = make_idesc_bf16(128, DPAD == 128 ? 128 : 64, 0, 1);
  constexpr uint32_t IDESC_PV_C1 = make_idesc_bf16(128, C::C1 > 0 ? C::C1 : 16, 0, 1);
  const uint32_t q0 = smem_u32(base + C::OFF_Q);
  const uint32_t stage0 = smem_u32(base + C::OFF_STAGE);
  uint32_t g = 0, qi = 0;
  bool ok = true;

  // S_(gi&1) = Q K_gi^T.  It overwrites P(gi-2) (P is written over its own
  // logits), whose PV was issued before: MMAs of one thread run in issue order.
  // Q is read from its TMEM copy (A operand), K from shared memory.
  auto issue_qk = [&](uint32_t gi) -> bool {
    const int st = gi % C::NST;
    if (!sp_wait(&ctl.k_full[st], (gi / C::NST) & 1, ctl, p)) return false;
    tc_fence_after();
    const uint32_t k_tile = stage0 + st * C::STAGE_BYTES;
    const uint32_t dst = tmem + C::T_S + 128u * (gi & 1);
#pragma unroll
    for (int kk = 0; kk < DPAD / 16; ++kk)
      mma_ts(dst, tmem + C::T_Q + kk * 8, kmajor_desc<DPAD>(k_tile, 128, kk), IDESC_QK, kk > 0 ? 1u : 0u);
    mma_commit(&ctl.s_full[gi & 1]);
    mma_commit(&ctl.k_empty[st]);
    return true;
  };
  auto issue_pv = [&](uint32_t gi, bool first) -> bool {
    const int st = gi % C::NST;
    if (!sp_wait(&ctl.p_full[gi & 1], (gi >> 1) & 1, ctl, p)) return false;
    if (!sp_wait(&ctl.v_full[st], (gi / C::NST) & 1, ctl, p)) return false;
    tc_fence_after();
    const uint32_t v_tile = stage0 + st * C::STAGE_BYTES + C::TILE_BYTES;
    const uint32_t tp = tmem + C::T_S + 128u * (gi & 1);
    const uint32_t dst = tmem + C::T_O;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t acc = (first && kk == 0) ? 0u : 1u;
      mma_ts(dst, tp + kk * 8, v_desc_c0<DPAD, 128>(v_tile, kk), IDESC_PV_FULL, acc);
      if (C::C1 > 0 && DPAD != 128)
        mma_ts(dst + 64, tp + kk * 8, v_desc_c1<DPAD, 128>(v_tile, kk), IDESC_PV_C1, acc);
    }
    mma_commit(&ctl.v_empty[st]);
    mma_commit(&ctl.pv_done[gi & 1]);
    return true;
  };

  int it = 0;
  for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++it) {
    const int slot = it & 1;
    if (!sp_wait(&ctl.ti_full[slot], (it >> 1) & 1, ctl, p)) { ok = false; break; }
    const int n = ctl.ti[slot].n;
    if (n > 0) {
      const int qs = C::QBUF == 2 ? (qi & 1) : 0;
      if (!sp_wait(&ctl.q_full[qs], (qi / C::QBUF) & 1, ctl, p)) { ok = false; break; }
      // Q tile -> TMEM.  Every QK^T of the previous tile has completed (its last
      // PV waited for the softmax, which had read the last logits), so the one
      // TMEM copy of Q is free; the shared-memory buffer is released as soon as
      // the copy is done.
      tc_fence_after();
      const uint32_t q_addr = q0 + qs * C::TILE_BYTES;
#pragma unroll
      for (int kk = 0; kk < DPAD / 16; ++kk) tmem_cp_128x256b(tmem + C::T_Q + kk * 8, kmajor_desc<DPAD>(q_addr, 128, kk));
      mma_commit(&ctl.q_empty[qs]);
      const uint32_t g0 = g;
      for (int i = 0; ok && i < n && i < 2; ++i) ok = issue_qk(g0 + i);
      for (int j = 0; ok && j < n; ++j) {
        // the first PV restarts O: the epilogue must have drained the previous tile's O
        if (j == 0 && qi >= 1 && !sp_wait(&ctl.o_free, (qi - 1) & 1, ctl, p)) { ok = false; break; }
        ok = issue_pv(g0 + j, j == 0);
        if (ok && j + 2 < n) ok = issue_qk(g0 + j + 2);
      }
      if (!ok) break;
      mma_commit(&ctl.o_full);
      g = g0 + n;
      ++qi;
    }
    mbar_arrive(&ctl.ti_empty[slot]);
  }
  if (!ok) {
    mma_commit(&ctl.drain);
    drain_wait(&ctl.drain, 0, p.wait_limit_ns);
  }
}

// ------------------------------------------------------------------ softmax
template <int DPAD>
__device__ __forceinline__ void sp_softmax(const AttnParams& p, SpCtrl& ctl, uint32_t tmem, int ntiles) {
  using C = SpCfg<DPAD>;
  const int t = threadIdx.x;
  const int warp = t >> 5;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tS = tmem + lane_base + C::T_S;
  const uint32_t tO = tmem + lane_base + C::T_O;
  const uint32_t tL = tmem + lane_base + C::T_L;
  const float sl2 = p.scale_log2;
  uint32_t g = 0;
  bool ok = true;
  int it = 0;
  for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++it) {
    const int slot = it & 1;
    ok = __all_sync(0xffffffffu, sp_wait(&ctl.ti_full[slot], (it >> 1) & 1, ctl, p));
    if (!ok) break;
    const SpTile ti = ctl.ti[slot];
    mbar_arrive(&ctl.ti_empty[slot]);
    float m = 0.f, l = 0.f;
    for (int j = 0; !ti.bad && j < ti.n; ++j, ++g) {
      const int bf = g & 1;
      ok = __all_sync(0xffffffffu, sp_wait(&ctl.s_full[bf], (g >> 1) & 1, ctl, p));
      if (!ok) break;
      tc_fence_after();
      uint32_t s[128];
      load_scores<128>(tS + 128u * bf, s);
      tmem_wait_ld();
      mask_tail<128>(s, (j == ti.tail_j) ? ti.tail_valid : 128);
      if (j == 0) m = row_max<128>(s) * sl2;
      // P(g) over the first 64 columns of its own logits (they are in registers),
      // with the running max.  If the row sum exceeds kRescaleSum, the block's
      // largest x = s * sl2 - m tells whether that max was too small.
      float sum = exp_pack_store<128>(s, sl2, m, tS + 128u * bf);
      // chk is the same in every lane, so all lanes or none take the second vote
      const bool chk = __any_sync(0xffffffffu, sum > kRescaleSum);
      const float xmax = chk ? xmax_of<128>(s, sl2, m) : 0.f;
      if (chk && __any_sync(0xffffffffu, xmax > kRescaleLog2)) {
        // rare: the block raised the max by more than 2^8: rescale O, then redo P(g)
        tmem_wait_st();                       // the first P(g) stores land before they are redone
        const float m_new = m + fmaxf(xmax, 0.f);
        const float alpha = ex2_approx(m - m_new);
        l *= alpha;
        // O holds blocks up to g-1: wait for PV(g-1)
        ok = __all_sync(0xffffffffu, sp_wait(&ctl.pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, ctl, p));
        if (!ok) break;
        tc_fence_after();
        rescale_row<DPAD>(tO, alpha);
        m = m_new;
        sum = exp_pack_store<128>(s, sl2, m, tS + 128u * bf);
      }
      l += sum;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&ctl.p_full[bf]);
    }
    if (!ok) break;
    // hand the tile to the epilogue: slot e holds its counts and (TMEM) its row sums
    const int e = it & 1;
    if (it >= 2) {
      ok = __all_sync(0xffffffffu, sp_wait(&ctl.epi_empty[e], ((it >> 1) - 1) & 1, ctl, p));
      if (!ok) break;
    }
    if (!ti.bad && ti.n > 0) {
      tmem_st_x1(tL + e, __float_as_uint(l));
      tmem_wait_st();
    }
    if (t == 0) {
      ctl.epi_n[e] = ti.bad ? 0 : ti.n;
      ctl.epi_bad[e] = ti.bad;
    }
    tc_fence_before();
    mbar_arrive(&ctl.epi_full[e]);
  }
}

// ------------------------------------------------------------------ epilogue
template <int DPAD>
__device__ __forceinline__ void sp_epilogue(const TmaSet& tm, const AttnParams& p, SpCtrl& ctl, uint8_t* base,
                                            uint32_t tmem, int ntiles) {
  using C = SpCfg<DPAD>;
  const int t = threadIdx.x - kSpEpiThread0;          // tile row
  const int warp = threadIdx.x >> 5;
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const uint32_t tO = tmem + lane_base + C::T_O;
  const uint32_t tL = tmem + lane_base + C::T_L;
  uint8_t* sR = base + C::OFF_R;
  uint8_t* sOst = base + C::OFF_OST;
  const bool r_smem = !p.r_f32 && p.use_r;
  uint32_t oi = 0, ri = 0, si = 0;
  bool ok = true;
  int it = 0;
  for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++it) {
    const int e = it & 1;
    ok = __all_sync(0xffffffffu, sp_wait(&ctl.epi_full[e], (it >> 1) & 1, ctl, p));
    if (!ok) break;
    tc_fence_after();
    const int n = ctl.epi_n[e];
    const int bad = ctl.epi_bad[e];
    float l = 0.f;
    if (n > 0) {
      l = __uint_as_float(tmem_ld_x1(tL + e));
      tmem_wait_ld();
    }
    tc_fence_before();
    mbar_arrive(&ctl.epi_empty[e]);
    if (bad) continue;
    int b, h, qb;
    sp_decode(p, tile, b, h, qb);
    const int grow = qb * 128 + t;
    const size_t rho_idx = (static_cast<size_t>(b) * p.H + h) * p.L + grow;
    const float rho = (p.use_rho && grow < p.L) ? __ldg(p.rho_in + rho_idx) : 0.f;
    // drain O at once: the next tile's first PV waits for it
    uint32_t acc[DPAD];
    if (n > 0) {
      ok = __all_sync(0xffffffffu, sp_wait(&ctl.o_full, oi & 1, ctl, p));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c + 32 <= DPAD; c += 32) tmem_ld_x32(tO + c, *reinterpret_cast<uint32_t(*)[32]>(&acc[c]));
      if constexpr (DPAD % 32 != 0)
        tmem_ld_x16(tO + (DPAD & ~31), *reinterpret_cast<uint32_t(*)[16]>(&acc[DPAD & ~31]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&ctl.o_free);
      ++oi;
    }
    if (r_smem) {
      ok = __all_sync(0xffffffffu, sp_wait(&ctl.r_full, ri & 1, ctl, p));
      if (!ok) break;
    }
    // staging slot: thread 0 makes sure the store that last used it has read it
    if (t == 0) {
      tma_store_wait_read<0>();
      mbar_arrive(&ctl.stg_ready);
    }
    const float rho_hat = p.use_rho ? fminf(1.f, fmaf(rho, p.ramp_mul, p.ramp_add)) : 1.f;
    const float scale = n > 0 ? rho_hat / l : 0.f;
    ok = __all_sync(0xffffffffu, sp_wait(&ctl.stg_ready, si & 1, ctl, p));
    if (!ok) break;
    uint8_t* ost = sOst;
#pragma unroll
    for (int c = 0; c < DPAD; c += 16) {
      float rr[16];
      if (r_smem) {
        load_row16<DPAD>(sR, 128, t, c, false, rr);
      } else if (p.use_r && grow < p.L) {
        // fp32 residual straight from global memory
        const float4* src = reinterpret_cast<const float4*>(
            static_cast<const float*>(p.r_in) + b * p.stride_b + h * p.stride_h +
            static_cast<long long>(grow) * p.stride_l + c);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float4 v4 = (c + 4 * u < p.d) ? __ldg(src + u) : make_float4(0.f, 0.f, 0.f, 0.f);
          rr[4 * u] = v4.x; rr[4 * u + 1] = v4.y; rr[4 * u + 2] = v4.z; rr[4 * u + 3] = v4.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) rr[i] = 0.f;
      }
      uint32_t pk[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float a0 = (n > 0 ? __uint_as_float(acc[c + 2 * i]) * scale : 0.f) + rr[2 * i];
        const float a1 = (n > 0 ? __uint_as_float(acc[c + 2 * i + 1]) * scale : 0.f) + rr[2 * i + 1];
        pk[i] = pack_bf16x2(a0, a1);
      }
      const bool c1 = c >= 64;
      const uint32_t rb = c1 ? C::C1B : 128;
      const uint32_t cbase = c1 ? 128 * 128 : 0;
      const int col = c1 ? c - 64 : c;
#pragma unroll
      for (int u = 0; u < 2; ++u)
        *reinterpret_cast<uint4*>(ost + cbase + swz_off(t * rb + (col * 2 + u * 16), rb)) =
            make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
    }
    if (r_smem) {
      mbar_arrive(&ctl.r_empty);
      ++ri;
    }
    fence_proxy_async_smem();
    mbar_arrive(&ctl.stg_full);
    if (t == 0) {
      if (sp_wait(&ctl.stg_full, si & 1, ctl, p)) {
        const int q_row = qb * 128;
        tma_store_4d(&tm.o[0], ost, 0, q_row, h, b);
        if (C::C1) tma_store_4d(&tm.o[1], ost + 128 * 128, 64, q_row, h, b);
        tma_store_commit();
      }
    }
    __syncwarp();
    ++si;
  }
  if (t == 0) tma_store_wait0();
}

template <int DPAD>
__global__ void __launch_bounds__(kSpThreads, 1)
sparse_kernel(const __grid_constant__ TmaSet tm, const AttnParams p, int ntiles) {
  using C = SpCfg<DPAD>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  SpCtrl& ctl = *reinterpret_cast<SpCtrl*>(base);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl.q_full[i], 1);
      mbar_init(&ctl.q_empty[i], 1);
      mbar_init(&ctl.s_full[i], 1);
      mbar_init(&ctl.p_full[i], kSoftmaxThreads);
      mbar_init(&ctl.pv_done[i], 1);
      mbar_init(&ctl.ti_full[i], 1);
      mbar_init(&ctl.ti_empty[i], kSoftmaxThreads + 2);
      mbar_init(&ctl.epi_full[i], kSoftmaxThreads);
      mbar_init(&ctl.epi_empty[i], kSoftmaxThreads);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&ctl.k_full[i], 1);
      mbar_init(&ctl.v_full[i], 1);
      mbar_init(&ctl.k_empty[i], 1);
      mbar_init(&ctl.v_empty[i], 1);
    }
    mbar_init(&ctl.o_full, 1);
    mbar_init(&ctl.o_free, kSoftmaxThreads);
    mbar_init(&ctl.r_full, 1);
    mbar_init(&ctl.r_empty, kSoftmaxThreads);
    mbar_init(&ctl.stg_ready, 1);
    mbar_init(&ctl.stg_full, kSoftmaxThreads);
    mbar_init(&ctl.drain, 1);
    ctl.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kSpMmaWarp) {
    tmem_alloc(&ctl.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;

  if (warp < 4) {
    reg_set<kSpRegsLaunch, SpRegs<DPAD>::softmax>();
    sp_softmax<DPAD>(p, ctl, tmem, ntiles);
  } else if (warp < 8) {
    reg_set<kSpRegsLaunch, SpRegs<DPAD>::epilogue>();
    sp_epilogue<DPAD>(tm, p, ctl, base, tmem, ntiles);
  } else {
    reg_set<kSpRegsLaunch, kSpRegsOther>();
    if (warp == kSpProducerWarp) {
      sp_producer<DPAD>(tm, p, ctl, base, ntiles);
    } else if (warp == kSpMmaWarp) {
      if (lane == 0) sp_mma<DPAD>(p, ctl, base, tmem, ntiles);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kSpMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace rtb
