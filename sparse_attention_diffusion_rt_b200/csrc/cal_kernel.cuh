// Calibration kernel with a single TMEM accumulator (head dims 64..128,
// 128-token blocks).
//
// Computes the calibration step of "Re-ttention" (OpenReview replies to W1:
// full attention, the denominator ratio rho = Z_sparse / Z_full and the
// residual of the masked tokens, all under one shared row max):
//   O = (acc_in + acc_out) / Z,  R = acc_out / Z,  rho = l_in / Z,  Z = l_in + l_out.
// Instead of two TMEM accumulators, every CTA visits its key blocks in the
// order "masked blocks (ascending), then kept blocks (ascending)".  When the
// first kept block is reached, the accumulator (then exactly acc_out) is copied
// to shared memory as fp32 and the accumulation restarts at zero; later lazy
// rescalings of the running max multiply that copy by a per-row factor.  The
// sums do not depend on the visiting order, so the result is the same
// definition; the freed TMEM pays for double-buffered logits and
// probabilities: S0/S1 [0,256) fp32, P0/P1 [256,384) bf16, acc [384,384+DPAD).
//
// One CTA per (batch, head, query block), 192 threads: warps 0-3 softmax and
// epilogue (thread t owns row t), warp 4 lane 0 loads Q and the K tiles, lane 1
// the V tiles (separate rings), warp 5 lane 0 issues the MMAs; the QK^T of
// block j+2 is issued as soon as the softmax has read block j's logits.
#pragma once
#include <cuda.h>
#include <cstdint>

#include "attn_kernel.cuh"
#include "ptx.cuh"
#include "softmax.cuh"
#include "sparse_kernel.cuh"

namespace rtb {

template <int DPAD>
struct CalCfg {
  static constexpr int C1 = DPAD - 64;
  static constexpr int TILE = 128 * DPAD * 2;
  static constexpr int NST = DPAD <= 96 ? 3 : 2;
  static constexpr int SNAP_ROW = DPAD * 4;                  // fp32 row of the snapshot
  static constexpr int OFF_Q = 2048;
  static constexpr int OFF_STAGE = OFF_Q + TILE;
  static constexpr int OFF_SNAP = OFF_STAGE + NST * 2 * TILE;
  static constexpr int SMEM = OFF_SNAP + 128 * SNAP_ROW + 1024;
  static_assert(SMEM <= 232448, "shared memory per CTA");
  static_assert(NST * 2 * TILE >= 128 * ((DPAD + 31) / 32) * 128, "residual staging fits the stages");
  static constexpr uint32_t T_S = 0, T_P = 256, T_ACC = 384;
};

struct CalCtrl {
  uint64_t q_full, s_full[2], s_free[2], p_full[2], pv_done[2], o_full, epi, drain;
  uint64_t k_full[3], v_full[3], k_empty[3], v_empty[3];
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

template <int DPAD>
__device__ __forceinline__ void cal_producer(const TmaSet& tm, const AttnParams& p, CalCtrl& ctl, uint8_t* base,
                                             int b, int h, int qb) {
  using C = CalCfg<DPAD>;
  const int lane = threadIdx.x & 31;
  if (lane > 1) return;
  int issued = 0;
  bool ok = true;
  if (lane == 0) {
    mbar_arrive_expect_tx(&ctl.q_full, C::TILE);
    tma_load_4d(base + C::OFF_Q, &tm.q[0], &ctl.q_full, 0, qb * 128, h, b);
    if (C::C1) tma_load_4d(base + C::OFF_Q + 128 * 128, &tm.q[1], &ctl.q_full, 64, qb * 128, h, b);
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
    tma_load_4d(dst, &m[0], full, 0, kb * 128, h, b);
    if (C::C1) tma_load_4d(dst + 128 * 128, &m[1], full, 64, kb * 128, h, b);
    issued = j + 1;
  }
  if (!ok) {
    const uint64_t lim = p.wait_limit_ns;
    if (lane == 0) drain_wait(&ctl.q_full, 0, lim);
    for (int j = (issued > C::NST ? issued - C::NST : 0); j < issued; ++j)
      drain_wait(lane == 0 ? &ctl.k_full[j % C::NST] : &ctl.v_full[j % C::NST], (j / C::NST) & 1, lim);
  }
}

template <int DPAD>
__device__ __forceinline__ void cal_mma(const AttnParams& p, CalCtrl& ctl, uint8_t* base, uint32_t tmem) {
  using C = CalCfg<DPAD>;
  constexpr uint32_t IDESC_QK = make_idesc_bf16(128, 128, 0, 0);
  constexpr uint32_t IDESC_PV_FULL = make_idesc_bf16(128, DPAD == 128 ? 128 : 64, 0, 1);
  constexpr uint32_t IDESC_PV_C1 = make_idesc_bf16(128, C::C1 > 0 ? C::C1 : 16, 0, 1);
  const uint32_t q_addr = smem_u32(base + C::OFF_Q);
  const uint32_t stage0 = smem_u32(base + C::OFF_STAGE);
  const int n = p.nkb;
  const int n_masked = p.nkb - ctl.n_kept;

  auto issue_qk = [&](int j) -> bool {
    const int st = j % C::NST;
    if (!sp_wait(&ctl.k_full[st], (j / C::NST) & 1, ctl, p)) return false;
    if (j >= 2 && !sp_wait(&ctl.s_free[j & 1], ((j >> 1) - 1) & 1, ctl, p)) return false;
    tc_fence_after();
    const uint32_t k_tile = stage0 + st * 2 * C::TILE;
#pragma unroll
    for (int kk = 0; kk < DPAD / 16; ++kk)
      mma_ss(tmem + C::T_S + 128u * (j & 1), kmajor_desc<DPAD>(q_addr, 128, kk), kmajor_desc<DPAD>(k_tile, 128, kk),
             IDESC_QK, kk > 0 ? 1u : 0u);
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
    const uint32_t tp = tmem + C::T_P + 64u * (j & 1);
    const uint32_t dst = tmem + C::T_ACC;
    const bool first = (j == 0) || (j == n_masked);     // restart after the snapshot
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

  bool ok = sp_wait(&ctl.q_full, 0, ctl, p) && issue_qk(0) && (n < 2 || issue_qk(1));
  for (int j = 0; ok && j < n; ++j) {
    if (j + 2 < n && !issue_qk(j + 2)) { ok = false; break; }
    if (!issue_pv(j)) { ok = false; break; }
  }
  if (ok) {
    mma_commit(&ctl.o_full);
  } else {
    mma_commit(&ctl.drain);
    drain_wait(&ctl.drain, 0, p.wait_limit_ns);
  }
}

template <int DPAD>
__device__ __forceinline__ void cal_softmax(const TmaSet& tm, const AttnParams& p, CalCtrl& ctl, uint8_t* base,
                                            uint32_t tmem, int b, int h, int qb) {
  using C = CalCfg<DPAD>;
  const int t = threadIdx.x;
  const uint32_t lane_base = static_cast<uint32_t>((t >> 5) * 32) << 16;
  const uint32_t tl = tmem + lane_base;
  const uint32_t tAcc = tl + C::T_ACC;
  float* snap = reinterpret_cast<float*>(base + C::OFF_SNAP);
  const float sl2 = p.scale_log2;
  const int n = p.nkb;
  const int n_masked = p.nkb - ctl.n_kept;
  const bool split = n_masked > 0 && ctl.n_kept > 0;    // a snapshot is taken between the phases
  CalOrder order{0, n_masked == 0 ? 1 : 0};
  float m = 0.f, l_in = 0.f, l_out = 0.f, snap_scale = 1.f;
  bool ok = true;
  for (int j = 0; j < n; ++j) {
    const int bf = j & 1;
    const int kb = order.next(ctl, p.nkb);
    ok = __all_sync(0xffffffffu, sp_wait(&ctl.s_full[bf], (j >> 1) & 1, ctl, p));
    if (!ok) break;
    tc_fence_after();
    uint32_t s[128];
    load_scores<128>(tl + C::T_S + 128u * bf, s);
    tmem_wait_ld();
    tc_fence_before();
    mbar_arrive(&ctl.s_free[bf]);
    mask_tail<128>(s, p.L - kb * 128);
    const float mx = row_max<128>(s) * sl2;
    bool acc_ready = false;                   // PV(j-1) known complete
    if (j == 0) {
      m = mx;
    } else if (__any_sync(0xffffffffu, mx > m + kRescaleLog2)) {
      const float m_new = fmaxf(m, mx);
      const float alpha = ex2_approx(m - m_new);
      l_in *= alpha;
      l_out *= alpha;
      if (split && j >= n_masked) snap_scale *= alpha;   // the copy is relative to the old max
      ok = __all_sync(0xffffffffu, sp_wait(&ctl.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, ctl, p));
      if (!ok) break;
      acc_ready = true;
      tc_fence_after();
      // right after the snapshot the accumulator restarts, so only rescale what it holds
      if (!(split && j == n_masked)) rescale_row<DPAD>(tAcc, alpha);
      m = m_new;
    }
    if (split && j == n_masked) {
      // the accumulator now holds exactly the masked blocks: keep it in shared memory
      if (!acc_ready) {
        ok = __all_sync(0xffffffffu, sp_wait(&ctl.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, ctl, p));
        if (!ok) break;
        tc_fence_after();
      }
#pragma unroll
      for (int c = 0; c < DPAD; c += 16) {
        uint32_t a[16];
        tmem_ld_x16(tAcc + c, a);
        tmem_wait_ld();
        const float sc = snap_scale;          // 1, or the rescale taken at this very block
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float4 v4 = make_float4(__uint_as_float(a[4 * u]) * sc, __uint_as_float(a[4 * u + 1]) * sc,
                                        __uint_as_float(a[4 * u + 2]) * sc, __uint_as_float(a[4 * u + 3]) * sc);
          const int unit = ((c >> 2) + u + t) % (DPAD / 4);   // rotate 16-byte units by row
          *reinterpret_cast<float4*>(snap + t * DPAD + unit * 4) = v4;
        }
      }
      snap_scale = 1.f;
    }
    // P buffer bf was last read by PV(j-2)
    if (j >= 2) {
      ok = __all_sync(0xffffffffu, sp_wait(&ctl.pv_done[bf], ((j >> 1) - 1) & 1, ctl, p));
      if (!ok) break;
      tc_fence_after();
    }
    const float sum = exp_pack_store<128>(s, sl2, m, tl + C::T_P + 64u * bf);
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
#pragma unroll
    for (int c = 0; c < DPAD; c += 16) {
      uint32_t a[16];
      tmem_ld_x16(tAcc + c, a);
      tmem_wait_ld();
      float o16[16], r16[16];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float4 sv = make_float4(0.f, 0.f, 0.f, 0.f);
        if (split) {
          const int unit = ((c >> 2) + u + t) % (DPAD / 4);
          sv = *reinterpret_cast<const float4*>(snap + t * DPAD + unit * 4);
        }
        const float sr[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = 4 * u + e;
          const float acc = __uint_as_float(a[i]);
          float out_masked, out_kept;
          if (split) {
            out_masked = sr[e] * rs;
            out_kept = acc * inv;
          } else if (n_masked == 0) {
            out_masked = 0.f;
            out_kept = acc * inv;
          } else {                                 // no kept block: the accumulator is all masked
            out_masked = acc * inv;
            out_kept = 0.f;
          }
          o16[i] = out_masked + out_kept;
          r16[i] = out_masked;
        }
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
      tma_store_4d(&tm.o[0], sO, 0, q_row, h, b);
      if (C::C1) tma_store_4d(&tm.o[1], sO + 128 * 128, 64, q_row, h, b);
      if (p.r_f32) {
        for (int c = 0; c < (DPAD + 31) / 32; ++c) tma_store_4d(&tm.r[c], sRst + c * 128 * 128, c * 32, q_row, h, b);
      } else {
        tma_store_4d(&tm.r[0], sRst, 0, q_row, h, b);
        if (C::C1) tma_store_4d(&tm.r[1], sRst + 128 * 128, 64, q_row, h, b);
      }
      tma_store_commit();
      tma_store_wait0();
    }
  }
}

template <int DPAD>
__global__ void __launch_bounds__(kThreads, 1)
cal_kernel(const __grid_constant__ TmaSet tm, const AttnParams p) {
  using C = CalCfg<DPAD>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  CalCtrl& ctl = *reinterpret_cast<CalCtrl*>(base);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int row = (p.Hm == 1 ? 0 : h) * p.nqb + qb;

  if (threadIdx.x == 0) {
    mbar_init(&ctl.q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl.s_full[i], 1);
      mbar_init(&ctl.s_free[i], kSoftmaxThreads);
      mbar_init(&ctl.p_full[i], kSoftmaxThreads);
      mbar_init(&ctl.pv_done[i], 1);
    }
    for (int i = 0; i < 3; ++i) {
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
    cal_producer<DPAD>(tm, p, ctl, base, b, h, qb);
  } else if (warp == kMmaWarp) {
    if (lane == 0) cal_mma<DPAD>(p, ctl, base, tmem);
  } else {
    cal_softmax<DPAD>(tm, p, ctl, base, tmem, b, h, qb);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace rtb
