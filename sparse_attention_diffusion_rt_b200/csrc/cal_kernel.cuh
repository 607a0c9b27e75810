// Calibration kernel with a single TMEM accumulator (head dims 64..128,
// 128-token blocks).
//
// Computes the calibration step of "Re-ttention" (OpenReview replies to W1:
// full attention, the denominator ratio rho = Z_sparse / Z_full and the
// residual of the masked tokens, all under one shared row max):
//   O = (acc_in + acc_out) / Z,  R = acc_out / Z,  rho = l_in / Z,  Z = l_in + l_out.
// Instead of two accumulators, every CTA visits its key blocks in the order
// "masked blocks (ascending), then kept blocks (ascending)".  When the first
// kept block is reached, the accumulator (then exactly acc_out) is copied to
// spare TMEM columns and the accumulation restarts at zero; later lazy
// rescalings of the running max multiply that copy by a per-row factor.  The
// sums do not depend on the visiting order, so the result is the same
// definition.
//
// TMEM columns: S0/S1 [0,256) fp32 logits, each with its bf16 probabilities P
// written over its first 64 columns once the logits are in registers; the
// accumulator [256, 256+DPAD); then the masked-block copy.  With QT (Q in
// TMEM) the copy follows the accumulator and Q follows the copy as bf16 pairs,
// so that QK^T takes A from TMEM and shared memory carries only K and V to
// the tensor core (the operand traffic that bounds this kernel).  At DPAD = 128
// the copy then has to fit 64 columns: it is stored as f16 pairs with a
// power-of-two row scale chosen from the row's largest value (relative error
// below 2^-11 of that value); without QT it is fp32 at [384, 512).  With no P
// or copy in shared memory, the K and V rings get as many stages as fit.
//
// One CTA per (batch, head, query block), 192 threads: warps 0-3 softmax and
// epilogue (thread t owns row t), warp 4 lane 0 loads Q and the K tiles, lane 1
// the V tiles, warp 5 lane 0 issues the MMAs in the order PV(j), QK(j+2): the
// logits of block j+2 overwrite P(j), and MMAs of one thread execute in issue
// order, so the softmax never waits for a buffer, only for its logits.
#pragma once
#include <cuda.h>
#include <cstdint>

#include "attn_kernel.cuh"
#include "ptx.cuh"
#include "softmax.cuh"
#include "sparse_kernel.cuh"

namespace rtb {

template <int DPAD, bool QT>
struct CalCfg {
  static constexpr int C1 = DPAD - 64;
  static constexpr int TILE = 128 * DPAD * 2;
  static constexpr int OFF_Q = 2048;
  static constexpr int OFF_STAGE = OFF_Q + TILE;
  static constexpr int NST_FIT = (232448 - 1024 - OFF_STAGE) / (2 * TILE);
  static constexpr int NST = NST_FIT > 6 ? 6 : NST_FIT;
  static constexpr int SMEM = OFF_STAGE + NST * 2 * TILE + 1024;
  static_assert(NST >= 2, "at least two K/V stages");
  static_assert(SMEM <= 232448, "shared memory per CTA");
  static_assert(NST * 2 * TILE >= 128 * ((DPAD + 31) / 32) * 128, "residual staging fits the stages");
  static constexpr bool SNAP16 = QT && DPAD == 128;          // f16 copy with a row scale
  static constexpr uint32_t T_S = 0, T_ACC = 256;
  static constexpr uint32_t T_SNAP = QT ? 256 + DPAD : 384;
  static constexpr uint32_t SNAP_COLS = SNAP16 ? DPAD / 2 : DPAD;
  static constexpr uint32_t T_Q = T_SNAP + SNAP_COLS;          // QT: Q as bf16 pairs, DPAD / 2 columns
  static_assert(T_SNAP + SNAP_COLS <= 512 && (!QT || T_Q + DPAD / 2 <= 512), "TMEM columns");
};

struct CalCtrl {
  uint64_t q_full, q_tmem, s_full[2], p_full[2], pv_done[2], o_full, epi, drain;
  uint64_t k_full[6], v_full[6], k_empty[6], v_empty[6];
  uint32_t tmem_base;
  volatile int abort_flag;
  int bad_index;
  int n_kept;
  uint32_t kept_bits[kMaxKeyBlocks / 32];
};
static_assert(sizeof(CalCtrl) <= 2048, "control block");

// Visiting order: masked key blocks ascending, then kept key blocks ascending.
struct CalOrder {
  int cursor;      // next key block to examine
  int phase;       // 0 = masked, 1 = kept
  __device__ __forceinline__ int next(const CalCtrl& ctl, int nkb) {
    while (true) {
      if (cursor >= nkb) {
        phase = 1;
        cursor = 0;
      }
      const int kb = cursor++;
      const bool kept = (ctl.kept_bits[kb >> 5] >> (kb & 31)) & 1u;
      if (kept == (phase == 1)) return kb;
    }
  }
};

template <int DPAD, bool QT>
__device__ __forceinline__ void cal_producer(const TmaSet& tm, const AttnParams& p, CalCtrl& ctl, uint8_t* base,
                                             int b, int h, int qb) {
  using C = CalCfg<DPAD, QT>;
  const int lane = threadIdx.x & 31;
  if (lane > 1) return;
  int issued = 0;
  bool ok = true;
  // every CTA of a head streams the head's whole K and V: keep them in L2 ahead
  // of this CTA's own Q (read once)
  const uint64_t keep = l2_evict_last();
  if (lane == 0) {
    const uint64_t once = l2_evict_first();
    mbar_arrive_expect_tx(&ctl.q_full, C::TILE);
    tma_load_4d_hint(base + C::OFF_Q, &tm.q[0], &ctl.q_full, 0, qb * 128, h, b, once);
    if (C::C1) tma_load_4d_hint(base + C::OFF_Q + 128 * 128, &tm.q[1], &ctl.q_full, 64, qb * 128, h, b, once);
  }
  CalOrder order{0, ctl.n_kept == p.nkb ? 1 : 0};
  for (int j = 0; j < p.nkb; ++j) {
    const int st = j % C::NST;
    uint64_t* empty = lane == 0 ? &ctl.k_empty[st] : &ctl.v_empty[st];
    uint64_t* full = lane == 0 ? &ctl.k_full[st] : &ctl.v_full[st];
    if (j >= C::NST && !sp_wait(empty, ((j / C::NST) - 1) & 1, ctl, p)) { ok = false; break; }
    const int kb = order.next(ctl, p.nkb);
    uint8_t* dst = base + C::OFF_STAGE + st * 2 * C::TILE + lane * C::TILE;
    const CUtensorMap* m = lane == 0 ? tm.k : tm.v;
    mbar_arrive_expect_tx(full, C::TILE);
    tma_load_4d_hint(dst, &m[0], full, 0, kb * 128, h, b, keep);
    if (C::C1) tma_load_4d_hint(dst + 128 * 128, &m[1], full, 64, kb * 128, h, b, keep);
    issued = j + 1;
  }
  if (!ok) {
    const uint64_t lim = p.wait_limit_ns;
    if (lane == 0) drain_wait(&ctl.q_full, 0, lim);
    for (int j = (issued > C::NST ? issued - C::NST : 0); j < issued; ++j)
      drain_wait(lane == 0 ? &ctl.k_full[j % C::NST] : &ctl.v_full[j % C::NST], (j / C::NST) & 1, lim);
  }
}

template <int DPAD, bool QT>
__device__ __forceinline__ void cal_mma(const AttnParams& p, CalCtrl& ctl, uint8_t* base, uint32_t tmem) {
  using C = CalCfg<DPAD, QT>;
  constexpr uint32_t IDESC_QK = make_idesc_bf16(128, 128, 0, 0);
  constexpr uint32_t IDESC_PV_FULL = make_idesc_bf16(128, DPAD == 128 ? 128 : 64, 0, 1);
  constexpr uint32_t IDESC_PV_C1 = make_idesc_bf16(128, C::C1 > 0 ? C::C1 : 16, 0, 1);
  const uint32_t q_addr = smem_u32(base + C::OFF_Q);
  const uint32_t stage0 = smem_u32(base + C::OFF_STAGE);
  const int n = p.nkb;
  const int n_masked = p.nkb - ctl.n_kept;

  // S_(j&1) = Q K_j^T.  For j >= 2 it overwrites P(j-2), whose PV was issued before.
  auto issue_qk = [&](int j) -> bool {
    const int st = j % C::NST;
    if (!sp_wait(&ctl.k_full[st], (j / C::NST) & 1, ctl, p)) return false;
    tc_fence_after();
    const uint32_t k_tile = stage0 + st * 2 * C::TILE;
#pragma unroll
    for (int kk = 0; kk < DPAD / 16; ++kk) {
      if constexpr (QT)
        mma_ts(tmem + C::T_S + 128u * (j & 1), tmem + C::T_Q + kk * 8, kmajor_desc<DPAD>(k_tile, 128, kk), IDESC_QK,
               kk > 0 ? 1u : 0u);
      else
        mma_ss(tmem + C::T_S + 128u * (j & 1), kmajor_desc<DPAD>(q_addr, 128, kk),
               kmajor_desc<DPAD>(k_tile, 128, kk), IDESC_QK, kk > 0 ? 1u : 0u);
    }
    mma_commit(&ctl.s_full[j & 1]);
    mma_commit(&ctl.k_empty[st]);
    return true;
  };
  auto issue_pv = [&](int j) -> bool {
    const int st = j % C::NST;
    if (!sp_wait(&ctl.p_full[j & 1], (j >> 1) & 1, ctl, p)) return false;
    if (!sp_wait(&ctl.v_full[st], (j / C::NST) & 1, ctl, p)) return false;
    tc_fence_after();
    const uint32_t v_tile = stage0 + st * 2 * C::TILE + C::TILE;
    const uint32_t tp = tmem + C::T_S + 128u * (j & 1);
    const uint32_t dst = tmem + C::T_ACC;
    const bool first = (j == 0) || (j == n_masked);     // restart after the copy of the masked blocks
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t acc = (first && kk == 0) ? 0u : 1u;
      mma_ts(dst, tp + kk * 8, v_desc_c0<DPAD, 128>(v_tile, kk), IDESC_PV_FULL, acc);
      if (C::C1 > 0 && DPAD != 128)
        mma_ts(dst + 64, tp + kk * 8, v_desc_c1<DPAD, 128>(v_tile, kk), IDESC_PV_C1, acc);
    }
    mma_commit(&ctl.v_empty[st]);
    mma_commit(&ctl.pv_done[j & 1]);
    return true;
  };

  // Q in TMEM: the softmax warps copy it there from shared memory first
  bool ok = sp_wait(QT ? &ctl.q_tmem : &ctl.q_full, 0, ctl, p) && issue_qk(0) && (n < 2 || issue_qk(1));
  for (int j = 0; ok && j < n; ++j) {
    if (!issue_pv(j)) { ok = false; break; }
    if (j + 2 < n && !issue_qk(j + 2)) { ok = false; break; }
  }
  if (ok) {
    mma_commit(&ctl.o_full);
  } else {
    mma_commit(&ctl.drain);
    drain_wait(&ctl.drain, 0, p.wait_limit_ns);
  }
}

// Q row t (bf16, as TMA left it in the swizzled chunks) -> TMEM lane t as bf16
// pairs, the A-operand layout of QK^T.
template <int DPAD, bool QT>
__device__ __forceinline__ void cal_copy_q(const uint8_t* sQ, uint32_t tq, int t) {
  using C = CalCfg<DPAD, QT>;
#pragma unroll
  for (int u0 = 0; u0 < DPAD / 8; u0 += 2) {          // two 16-byte units (16 columns) per store
    uint32_t w[8];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int u = u0 + k;
      const bool c1 = u >= 8;
      const uint32_t rb = c1 ? C::C1 * 2 : 128;
      const uint32_t off = (c1 ? 128 * 128 : 0) + swz_off(t * rb + (c1 ? u - 8 : u) * 16, rb);
      const uint4 v = *reinterpret_cast<const uint4*>(sQ + off);
      w[4 * k] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
    }
    tmem_st_x8(tq + u0 * 4, w);
  }
}

template <int DPAD, bool QT>
__device__ __forceinline__ void cal_softmax(const TmaSet& tm, const AttnParams& p, CalCtrl& ctl, uint8_t* base,
                                            uint32_t tmem, int b, int h, int qb) {
  using C = CalCfg<DPAD, QT>;
  const int t = threadIdx.x;
  const uint32_t lane_base = static_cast<uint32_t>((t >> 5) * 32) << 16;
  const uint32_t tl = tmem + lane_base;
  const uint32_t tAcc = tl + C::T_ACC;
  const uint32_t tSnap = tl + C::T_SNAP;
  const float sl2 = p.scale_log2;
  const int n = p.nkb;
  const int n_masked = p.nkb - ctl.n_kept;
  const bool split = n_masked > 0 && ctl.n_kept > 0;    // a copy is taken between the phases
  // the last key block (the one that may run past the sequence end) is the
  // last of its phase in the visiting order
  const bool tail_kept = (ctl.kept_bits[(p.nkb - 1) >> 5] >> ((p.nkb - 1) & 31)) & 1u;
  const int tail_j = tail_kept ? n - 1 : n_masked - 1;
  const int tail_valid = p.L - (p.nkb - 1) * 128;
  float m = 0.f, l_in = 0.f, l_out = 0.f, snap_scale = 1.f;
  bool ok = true;
  if constexpr (QT) {
    ok = __all_sync(0xffffffffu, sp_wait(&ctl.q_full, 0, ctl, p));
    if (ok) {
      cal_copy_q<DPAD, QT>(base + C::OFF_Q, tl + C::T_Q, t);
      tmem_wait_st();
      tc_fence_before();
    }
    mbar_arrive(&ctl.q_tmem);
  }
  for (int j = 0; ok && j < n; ++j) {
    const int bf = j & 1;
    ok = __all_sync(0xffffffffu, sp_wait(&ctl.s_full[bf], (j >> 1) & 1, ctl, p));
    if (!ok) break;
    tc_fence_after();
    const uint32_t tS = tl + C::T_S + 128u * bf;
    uint32_t s[128];
    load_scores<128>(tS, s);
    tmem_wait_ld();
    if (j == tail_j) mask_tail<128>(s, tail_valid);
    if (j == 0) m = row_max<128>(s) * sl2;
    // P(j) over the first 64 logit columns (the logits are in registers), with
    // the running max.  If the row sum exceeds kRescaleSum, the block's largest
    // x = s * sl2 - m tells whether that max was too small.
    float sum = exp_pack_store<128>(s, sl2, m, tS);
    // chk is the same in every lane, so all lanes or none take the second vote
    const bool chk = __any_sync(0xffffffffu, sum > kRescaleSum);
    const float xmax = chk ? xmax_of<128>(s, sl2, m) : 0.f;
    if (chk && __any_sync(0xffffffffu, xmax > kRescaleLog2)) {
      // rare: the block raised the max by more than 2^8: rescale, then redo P(j)
      tmem_wait_st();                         // the first P(j) stores land before they are redone
      const float m_new = m + fmaxf(xmax, 0.f);
      const float alpha = ex2_approx(m - m_new);
      l_in *= alpha;
      l_out *= alpha;
      if (split && j >= n_masked) snap_scale *= alpha;   // the copy is relative to the old max
      // the accumulator holds blocks 0..j-1: wait until the last of them has landed
      ok = __all_sync(0xffffffffu, sp_wait(&ctl.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, ctl, p));
      if (!ok) break;
      tc_fence_after();
      // at the first kept block the accumulator is copied and restarted: nothing to rescale
      if (!(split && j == n_masked)) rescale_row<DPAD>(tAcc, alpha);
      m = m_new;
      sum = exp_pack_store<128>(s, sl2, m, tS);
    }
    if (split && j == n_masked) {
      // the accumulator now holds exactly the masked blocks: copy it to its own columns
      ok = __all_sync(0xffffffffu, sp_wait(&ctl.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, ctl, p));
      if (!ok) break;
      tc_fence_after();
      const float sc = snap_scale;            // 1, or the rescale taken at this very block
      if constexpr (C::SNAP16) {
        // f16 with a power-of-two row scale: the row's largest |value| lands in [2^14, 2^15)
        float amax = 0.f;
#pragma unroll
        for (int c = 0; c < DPAD; c += 16) {
          uint32_t a[16];
          tmem_ld_x16(tAcc + c, a);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(__uint_as_float(a[i])));
        }
        int e = 0;
        frexpf(amax * sc, &e);                // amax * sc = f * 2^e, f in [0.5, 1)
        const int k = min(15 - e, 126);
        const float f = sc * __int_as_float((127 + k) << 23);    // sc * 2^k
#pragma unroll
        for (int c = 0; c < DPAD; c += 16) {
          uint32_t a[16], w[8];
          tmem_ld_x16(tAcc + c, a);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 8; ++i)
            w[i] = pack_f16x2(__uint_as_float(a[2 * i]) * f, __uint_as_float(a[2 * i + 1]) * f);
          tmem_st_x8(tSnap + c / 2, w);
        }
        snap_scale = __int_as_float((127 - k) << 23);           // 2^-k
      } else {
#pragma unroll
        for (int c = 0; c < DPAD; c += 16) {
          uint32_t a[16];
          tmem_ld_x16(tAcc + c, a);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) a[i] = __float_as_uint(__uint_as_float(a[i]) * sc);
          tmem_st_x16(tSnap + c, a);
        }
        snap_scale = 1.f;
      }
    }
    if (j < n_masked) l_out += sum; else l_in += sum;
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&ctl.p_full[bf]);
  }
  if (ok) {
    ok = __all_sync(0xffffffffu, sp_wait(&ctl.o_full, 0, ctl, p));
    if (ok) tc_fence_after();
  }
  // ------------------------------------------------------------- epilogue
  const int grow = qb * 128 + t;
  uint8_t* sO = base + C::OFF_Q;          // all MMAs are done: Q and the stages are free
  uint8_t* sRst = base + C::OFF_STAGE;
  if (ok) {
    const float z = l_in + l_out;
    const float inv = 1.f / z;
    if (grow < p.L) p.rho_out[(static_cast<size_t>(b) * p.H + h) * p.L + grow] = l_in / z;
    const float rs = snap_scale * inv;
    const float inv_in = l_in > 0.f ? 1.f / l_in : 0.f;
#pragma unroll
    for (int c = 0; c < DPAD; c += 16) {
      uint32_t a[16], sv[16];
      tmem_ld_x16(tAcc + c, a);
      if constexpr (C::SNAP16) {
        if (split) {
          uint32_t w[8];
          tmem_ld_x8(tSnap + c / 2, w);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float lo, hi;
            unpack_f16x2(w[i], lo, hi);
            sv[2 * i] = __float_as_uint(lo);
            sv[2 * i + 1] = __float_as_uint(hi);
          }
        }
      } else {
        if (split) tmem_ld_x16(tSnap + c, sv);
      }
      tmem_wait_ld();
      float o16[16], r16[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float acc = __uint_as_float(a[i]);
        float out_masked, out_kept;
        if (split) {
          out_masked = __uint_as_float(sv[i]) * rs;
          out_kept = acc * inv;
        } else if (n_masked == 0) {
          out_masked = 0.f;
          out_kept = acc * inv;
        } else {                                 // no kept block: the accumulator is all masked
          out_masked = acc * inv;
          out_kept = 0.f;
        }
        o16[i] = out_masked + out_kept;
        // masked tokens' part, or O_full - O_sparse with O_sparse = acc_in / l_in (0 with no kept key)
        r16[i] = p.r_sub ? o16[i] - (n_masked < n ? acc * inv_in : 0.f) : out_masked;
      }
      store_row16<DPAD>(sO, 128, t, c, false, o16);
      store_row16<DPAD>(sRst, 128, t, c, p.r_f32 != 0, r16);
    }
  }
  fence_proxy_async_smem();
  mbar_arrive(&ctl.epi);
  if (t == 0) {
    if (sp_wait(&ctl.epi, 0, ctl, p) && !ctl.abort_flag) {
      const int q_row = qb * 128;
      const uint64_t once = l2_evict_first();       // outputs: written once, not re-read here
      tma_store_4d_hint(&tm.o[0], sO, 0, q_row, h, b, once);
      if (C::C1) tma_store_4d_hint(&tm.o[1], sO + 128 * 128, 64, q_row, h, b, once);
      if (p.r_f32) {
        for (int c = 0; c < (DPAD + 31) / 32; ++c)
          tma_store_4d_hint(&tm.r[c], sRst + c * 128 * 128, c * 32, q_row, h, b, once);
      } else {
        tma_store_4d_hint(&tm.r[0], sRst, 0, q_row, h, b, once);
        if (C::C1) tma_store_4d_hint(&tm.r[1], sRst + 128 * 128, 64, q_row, h, b, once);
      }
      tma_store_commit();
      tma_store_wait0();
    }
  }
}

template <int DPAD, bool QT>
__global__ void __launch_bounds__(kThreads, 1)
cal_kernel(const __grid_constant__ TmaSet tm, const AttnParams p) {
  using C = CalCfg<DPAD, QT>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  CalCtrl& ctl = *reinterpret_cast<CalCtrl*>(base);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int row = (p.Hm == 1 ? 0 : h) * p.nqb + qb;

  if (threadIdx.x == 0) {
    mbar_init(&ctl.q_full, 1);
    mbar_init(&ctl.q_tmem, kSoftmaxThreads);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl.s_full[i], 1);
      mbar_init(&ctl.p_full[i], kSoftmaxThreads);
      mbar_init(&ctl.pv_done[i], 1);
    }
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(&ctl.k_full[i], 1);
      mbar_init(&ctl.v_full[i], 1);
      mbar_init(&ctl.k_empty[i], 1);
      mbar_init(&ctl.v_empty[i], 1);
    }
    mbar_init(&ctl.o_full, 1);
    mbar_init(&ctl.epi, kSoftmaxThreads);
    mbar_init(&ctl.drain, 1);
    ctl.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp) {
    int start = 0, end = 0, bad = 0;
    if (lane == 0) {
      start = __ldg(p.row_ptr + row);
      end = __ldg(p.row_ptr + row + 1);
      if (start < 0 || end < start || static_cast<long long>(end) > p.nnz || end - start > p.nkb) bad = 1;
    }
    start = __shfl_sync(0xffffffffu, start, 0);
    end = __shfl_sync(0xffffffffu, end, 0);
    bad = __shfl_sync(0xffffffffu, bad, 0);
    for (int w = lane; w < kMaxKeyBlocks / 32; w += 32) ctl.kept_bits[w] = 0u;
    __syncwarp();
    if (!bad) {
      for (int i = lane; i < end - start; i += 32) {
        const int c = __ldg(p.col_idx + start + i);
        const int prev = i > 0 ? __ldg(p.col_idx + start + i - 1) : -1;
        if (c < 0 || c >= p.nkb || c <= prev) bad = 1;
        else atomicOr(&ctl.kept_bits[c >> 5], 1u << (c & 31));
      }
    }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      ctl.bad_index = bad;
      ctl.n_kept = end - start;
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&ctl.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;

  if (ctl.bad_index) {
    if (threadIdx.x == 0) record_status(p.status, RT_ERR_BAD_INDEX);
  } else if (warp == kProducerWarp) {
    cal_producer<DPAD, QT>(tm, p, ctl, base, b, h, qb);
  } else if (warp == kMmaWarp) {
    if (lane == 0) cal_mma<DPAD, QT>(p, ctl, base, tmem);
  } else {
    cal_softmax<DPAD, QT>(tm, p, ctl, base, tmem, b, h, qb);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace rtb
