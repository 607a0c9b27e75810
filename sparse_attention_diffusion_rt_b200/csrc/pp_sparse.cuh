// Ping-pong persistent sparse-step kernel for head dimensions up to 64.
//
// Same computation as sparse_kernel.cuh (the reshaped sparse step of
// "Re-ttention", OpenReview replies to W1 and to Pwod's W1):
//   O'_i = min(1, rho_i*mul + add) * softmax over kept key blocks (s'_i) . v' + R_i
// but each CTA runs two independent tile pipelines, A and B, so that one
// pipeline's softmax (bound by the MUFU exp rate) overlaps the other's max,
// barrier latency and tensor-core work.  CTA c handles tiles c + i*gridDim.x;
// even i go to pipeline A, odd i to B.
//
// Threads (384): warps 0-3 softmax + epilogue of A, warps 4-7 of B (thread t
// owns TMEM lane t % 128), lanes 0 and 1 of warp 8 are the TMA producers of A
// and B, lane 0 of warps 9 and 10 issue the MMAs of A and B, warp 11 idles.
// TMEM: pipeline p uses columns [256p, 256p+256): S logits [0,128), bf16 P
// [128,192), O [192,256).  A pipeline's next QK^T is issued as soon as its
// softmax has read the current logits (s_free), so it runs under that softmax;
// P is rewritten only after the previous PV has completed (pv_done), which also
// tells the softmax when O may be rescaled.
//
// Shared memory per pipeline: Q (one tile), a 2-stage K/V ring, the residual
// tile and an output staging tile.  All waits are bounded.
#pragma once
#include <cuda.h>
#include <cstdint>

#include "attn_kernel.cuh"
#include "ptx.cuh"
#include "softmax.cuh"
#include "sparse_kernel.cuh"

namespace rtb {

constexpr int kPpThreads = 384;
constexpr int kPpProducerWarp = 8;
constexpr int kPpMmaWarp = 9;        // warps 9 and 10: MMA issuers of pipelines A and B; warp 11 idle
// Registers: three warps per sub-partition cap the launch at 168 per thread;
// the two softmax warpgroups take 216 and the producer / MMA warpgroup gives
// back down to 56: 128 x (2 x 216 + 56) = 62464 <= 384 x 168.
constexpr uint32_t kPpRegsLaunch = 168, kPpRegsSoftmax = 216, kPpRegsOther = 56;
static_assert(kPpRegsLaunch * kPpThreads <= 65536 && 3 * 32 * kPpRegsLaunch <= 16384,
              "launch registers fit the register file and each sub-partition");
static_assert(32 * (2 * kPpRegsSoftmax + kPpRegsOther) <= 16384,
              "after the split, two softmax warps and one other warp still fit a sub-partition");
static_assert(128 * (2 * kPpRegsSoftmax + kPpRegsOther) <= kPpThreads * kPpRegsLaunch,
              "the warpgroups' shares fit the pool the CTA was launched with");

struct PpCfg {
  static constexpr int TILE = 128 * 64 * 2;                 // bf16 [128][64]
  static constexpr int NST = 2;
  static constexpr int PIPE_BYTES = TILE + NST * 2 * TILE + TILE + TILE;
  static constexpr int OFF_PIPE = 2048;
  static constexpr int SMEM = OFF_PIPE + 2 * PIPE_BYTES + 1024;
  static_assert(SMEM <= 232448, "shared memory per CTA");
  static constexpr int Q = 0, STAGE = TILE, R = TILE + NST * 2 * TILE, OST = R + TILE;
};

struct PpPipe {
  uint64_t q_full, q_empty;
  uint64_t k_full[2], v_full[2], kv_empty[2];
  uint64_t s_full, s_free, p_full, pv_done, o_full;
  uint64_t r_full, r_empty;
  uint64_t ti_full[2], ti_empty[2];
  uint64_t stg_ready, stg_full;
  SpTile ti[2];
};

struct PpCtrl {
  PpPipe pipe[2];
  uint64_t drain[2];
  uint32_t tmem_base;
  volatile int abort_flag;
};
static_assert(sizeof(PpCtrl) <= 2048, "control block");

__device__ __forceinline__ bool pp_wait(uint64_t* bar, uint32_t parity, PpCtrl& ctl, const AttnParams& p) {
  return sp_wait(bar, parity, ctl, p);
}

__device__ __forceinline__ int pp_tile(int it, int pipe) {
  return blockIdx.x + (2 * it + pipe) * gridDim.x;
}

// ------------------------------------------------------------------ producer (one lane per pipeline)
// Lane `pipe` of the producer warp serves pipeline `pipe`; the two lanes run
// independent loops (no warp collectives) and each validates its tiles' CSR
// rows serially before publishing them.
__device__ __forceinline__ void pp_producer(const TmaSet& tm, const AttnParams& p, PpCtrl& ctl, uint8_t* pbase,
                                            int pipe, int ntiles) {
  using C = PpCfg;
  PpPipe& P = ctl.pipe[pipe];
  uint8_t* sQ = pbase + C::Q;
  uint8_t* sStage = pbase + C::STAGE;
  uint8_t* sR = pbase + C::R;
  uint32_t g = 0, qi = 0, ri = 0;
  bool ok = true;
  for (int it = 0; ok; ++it) {
    const int tile = pp_tile(it, pipe);
    if (tile >= ntiles) break;
    const int slot = it & 1;
    if (it >= 2 && !pp_wait(&P.ti_empty[slot], ((it >> 1) - 1) & 1, ctl, p)) { ok = false; break; }
    int b, h, qb;
    sp_decode(p, tile, b, h, qb);
    const int row = (p.Hm == 1 ? 0 : h) * p.nqb + qb;
    const int start = __ldg(p.row_ptr + row);
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
    const int n = bad ? 0 : end - start;
    int tail_j = -1;
    const int tail_valid = p.L - (p.nkb - 1) * 128;
    if (!bad && n > 0 && tail_valid < 128 && __ldg(p.col_idx + end - 1) == p.nkb - 1) tail_j = n - 1;
    P.ti[slot] = SpTile{b, h, qb, n, start, bad, tail_j, tail_valid};
    if (bad) record_status(p.status, RT_ERR_BAD_INDEX);
    mbar_arrive(&P.ti_full[slot]);
    if (bad) continue;
    const int q_row = qb * 128;
    if (n > 0) {
      if (qi >= 1 && !pp_wait(&P.q_empty, (qi - 1) & 1, ctl, p)) { ok = false; break; }
      mbar_arrive_expect_tx(&P.q_full, C::TILE);
      tma_load_4d(sQ, &tm.q[0], &P.q_full, 0, q_row, h, b);
      ++qi;
      for (int j = 0; j < n; ++j, ++g) {
        const int st = g & 1;
        if (g >= 2 && !pp_wait(&P.kv_empty[st], ((g >> 1) - 1) & 1, ctl, p)) { ok = false; break; }
        const int kb = __ldg(p.col_idx + start + j);
        uint8_t* sK = sStage + st * 2 * C::TILE;
        mbar_arrive_expect_tx(&P.k_full[st], C::TILE);
        tma_load_4d(sK, &tm.k[0], &P.k_full[st], 0, kb * 128, h, b);
        mbar_arrive_expect_tx(&P.v_full[st], C::TILE);
        tma_load_4d(sK + C::TILE, &tm.v[0], &P.v_full[st], 0, kb * 128, h, b);
      }
      if (!ok) break;
    }
    if (!p.r_f32 && p.use_r) {
      if (ri >= 1 && !pp_wait(&P.r_empty, (ri - 1) & 1, ctl, p)) { ok = false; break; }
      mbar_arrive_expect_tx(&P.r_full, C::TILE);
      tma_load_4d(sR, &tm.r[0], &P.r_full, 0, q_row, h, b);
      ++ri;
    }
  }
  if (!ok) {
    // let every copy this lane started land before shared memory is released
    const uint64_t lim = p.wait_limit_ns;
    if (qi >= 1) drain_wait(&P.q_full, (qi - 1) & 1, lim);
    if (ri >= 1) drain_wait(&P.r_full, (ri - 1) & 1, lim);
    for (uint32_t i = (g > 2u ? g - 2u : 0u); i < g; ++i) {
      drain_wait(&P.k_full[i & 1], (i >> 1) & 1, lim);
      drain_wait(&P.v_full[i & 1], (i >> 1) & 1, lim);
    }
  }
}

// ------------------------------------------------------------------ MMA issuer (one thread per pipeline)
// Lane 0 of warp 9 + pipe issues pipeline `pipe`'s MMAs: QK^T of block j+1 as
// soon as the softmax has read block j's logits (s_free), then PV of block j
// once P is written (p_full).  tcgen05.commit tracks the issuing thread's own
// MMAs, so each pipeline's barriers see only its own work.
__device__ __forceinline__ void pp_mma(const AttnParams& p, PpCtrl& ctl, uint8_t* pbase, uint32_t tmem, int pipe,
                                       int ntiles) {
  using C = PpCfg;
  constexpr uint32_t IDESC_QK = make_idesc_bf16(128, 128, 0, 0);
  constexpr uint32_t IDESC_PV = make_idesc_bf16(128, 64, 0, 1);
  PpPipe& P = ctl.pipe[pipe];
  const uint32_t tbase = tmem + 256u * pipe;
  const uint32_t q_addr = smem_u32(pbase + C::Q);
  const uint32_t stage0 = smem_u32(pbase + C::STAGE);
  uint32_t g = 0, qi = 0;
  bool ok = true;

  auto issue_qk = [&](uint32_t gq, bool first_of_tile) -> bool {
    const int st = gq & 1;
    if (first_of_tile && !pp_wait(&P.q_full, qi & 1, ctl, p)) return false;
    if (!pp_wait(&P.k_full[st], (gq >> 1) & 1, ctl, p)) return false;
    if (gq > 0 && !pp_wait(&P.s_free, (gq - 1) & 1, ctl, p)) return false;
    tc_fence_after();
    const uint32_t k_tile = stage0 + st * 2 * C::TILE;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ss(tbase, kmajor_desc<64>(q_addr, 128, kk), kmajor_desc<64>(k_tile, 128, kk), IDESC_QK, kk > 0 ? 1u : 0u);
    mma_commit(&P.s_full);
    return true;
  };
  auto issue_pv = [&](uint32_t gp, bool first_of_tile) -> bool {
    const int st = gp & 1;
    if (!pp_wait(&P.p_full, gp & 1, ctl, p)) return false;
    if (!pp_wait(&P.v_full[st], (gp >> 1) & 1, ctl, p)) return false;
    tc_fence_after();
    const uint32_t v_tile = stage0 + st * 2 * C::TILE + C::TILE;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_ts(tbase + 192, tbase + 128 + kk * 8, v_desc_c0<64, 128>(v_tile, kk), IDESC_PV,
             (first_of_tile && kk == 0) ? 0u : 1u);
    mma_commit(&P.kv_empty[st]);
    mma_commit(&P.pv_done);
    return true;
  };

  for (int it = 0; ok; ++it) {
    if (pp_tile(it, pipe) >= ntiles) break;
    const int slot = it & 1;
    if (!pp_wait(&P.ti_full[slot], (it >> 1) & 1, ctl, p)) { ok = false; break; }
    const int n = P.ti[slot].n;
    if (n > 0) {
      if (!issue_qk(g, true)) { ok = false; break; }
      if (n == 1) mma_commit(&P.q_empty);
      for (int j = 0; j < n; ++j) {
        if (j + 1 < n) {
          if (!issue_qk(g + 1, false)) { ok = false; break; }
          if (j + 2 == n) mma_commit(&P.q_empty);
        }
        if (!issue_pv(g, j == 0)) { ok = false; break; }
        ++g;
      }
      if (!ok) break;
      mma_commit(&P.o_full);
      ++qi;
    }
    mbar_arrive(&P.ti_empty[slot]);
  }
  if (!ok) {
    mma_commit(&ctl.drain[pipe]);
    drain_wait(&ctl.drain[pipe], 0, p.wait_limit_ns);
  }
}

// ------------------------------------------------------------------ softmax + epilogue (one warpgroup per pipeline)
__device__ __forceinline__ void pp_softmax(const TmaSet& tm, const AttnParams& p, PpCtrl& ctl, uint8_t* pbase,
                                           uint32_t tmem, int pipe, int ntiles) {
  using C = PpCfg;
  PpPipe& P = ctl.pipe[pipe];
  const int t = threadIdx.x & 127;
  const int wq = (threadIdx.x >> 5) & 3;
  const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
  const uint32_t tS = tmem + 256u * pipe + lane_base;
  const uint32_t tP = tS + 128;
  const uint32_t tO = tS + 192;
  uint8_t* sR = pbase + C::R;
  uint8_t* sOst = pbase + C::OST;
  const float sl2 = p.scale_log2;
  uint32_t g = 0, oi = 0, ri = 0, si = 0;
  bool ok = true;
  for (int it = 0; ok; ++it) {
    const int tile = pp_tile(it, pipe);
    if (tile >= ntiles) break;
    const int slot = it & 1;
    ok = __all_sync(0xffffffffu, pp_wait(&P.ti_full[slot], (it >> 1) & 1, ctl, p));
    if (!ok) break;
    const SpTile ti = P.ti[slot];
    mbar_arrive(&P.ti_empty[slot]);
    if (ti.bad) continue;
    const int grow = ti.qb * 128 + t;
    const size_t rho_idx = (static_cast<size_t>(ti.b) * p.H + ti.h) * p.L + grow;
    const float rho = (p.use_rho && grow < p.L) ? __ldg(p.rho_in + rho_idx) : 0.f;
    float m = 0.f, l = 0.f;
    for (int j = 0; j < ti.n; ++j, ++g) {
      ok = __all_sync(0xffffffffu, pp_wait(&P.s_full, g & 1, ctl, p));
      if (!ok) break;
      tc_fence_after();
      const int valid = (j == ti.tail_j) ? ti.tail_valid : 128;
      const float mx = row_max_tmem<128>(tS, valid) * sl2;
      bool need_pv = g > 0;                  // P (and O) still in use by the previous PV
      if (j == 0) {
        m = mx;
      } else if (__any_sync(0xffffffffu, mx > m + kRescaleLog2)) {
        const float m_new = fmaxf(m, mx);
        const float alpha = ex2_approx(m - m_new);
        l *= alpha;
        ok = __all_sync(0xffffffffu, pp_wait(&P.pv_done, (g - 1) & 1, ctl, p));
        if (!ok) break;
        need_pv = false;
        tc_fence_after();
        rescale_row<64>(tO, alpha);
        m = m_new;
      }
      bool pv_ok = true;
      l += exp_pass_tmem_sep<128>(
          tS, tP, sl2, m, valid,
          [&] { tc_fence_before(); mbar_arrive(&P.s_free); },
          [&] {
            if (need_pv) {
              pv_ok = __all_sync(0xffffffffu, pp_wait(&P.pv_done, (g - 1) & 1, ctl, p));
              tc_fence_after();
            }
          });
      if (!pv_ok) { ok = false; break; }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&P.p_full);
    }
    if (!ok) break;
    // ------------------------------------------------------------- epilogue
    if (ti.n > 0) {
      ok = __all_sync(0xffffffffu, pp_wait(&P.o_full, oi & 1, ctl, p));
      if (!ok) break;
      tc_fence_after();
      ++oi;
    }
    if (!p.r_f32 && p.use_r) {
      ok = __all_sync(0xffffffffu, pp_wait(&P.r_full, ri & 1, ctl, p));
      if (!ok) break;
    }
    const float rho_hat = p.use_rho ? fminf(1.f, fmaf(rho, p.ramp_mul, p.ramp_add)) : 1.f;
    const float scale = ti.n > 0 ? rho_hat / l : 0.f;
    // staging tile free once this thread's previous bulk store has read it
    if (t == 0) {
      tma_store_wait_read<0>();
      mbar_arrive(&P.stg_ready);
    }
    ok = __all_sync(0xffffffffu, pp_wait(&P.stg_ready, si & 1, ctl, p));
    if (!ok) break;
#pragma unroll
    for (int h0 = 0; h0 < 64; h0 += 32) {
      uint32_t acc[32];
      if (ti.n > 0) {
        tmem_ld_x32(tO + h0, acc);
        tmem_wait_ld();
      }
#pragma unroll
      for (int c = h0; c < h0 + 32; c += 16) {
        float rr[16];
        if (!p.use_r) {
#pragma unroll
          for (int i = 0; i < 16; ++i) rr[i] = 0.f;
        } else if (p.r_f32) {
          if (grow < p.L) {
            const float4* src = reinterpret_cast<const float4*>(
                static_cast<const float*>(p.r_in) + ti.b * p.stride_b + ti.h * p.stride_h +
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
        } else {
          load_row16<64>(sR, 128, t, c, false, rr);
        }
        float o16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) o16[i] = (ti.n > 0 ? __uint_as_float(acc[c - h0 + i]) * scale : 0.f) + rr[i];
        store_row16<64>(sOst, 128, t, c, false, o16);
      }
    }
    if (!p.r_f32 && p.use_r) {
      mbar_arrive(&P.r_empty);
      ++ri;
    }
    fence_proxy_async_smem();
    mbar_arrive(&P.stg_full);
    if (t == 0) {
      if (pp_wait(&P.stg_full, si & 1, ctl, p)) {
        tma_store_4d(&tm.o[0], sOst, 0, ti.qb * 128, ti.h, ti.b);
        tma_store_commit();
      }
    }
    __syncwarp();
    ++si;
  }
  if (t == 0) tma_store_wait0();
}

template <int DPAD>
__global__ void __launch_bounds__(kPpThreads, 1)
pp_sparse_kernel(const __grid_constant__ TmaSet tm, const AttnParams p, int ntiles) {
  using C = PpCfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  PpCtrl& ctl = *reinterpret_cast<PpCtrl*>(base);
  uint8_t* pipes = base + C::OFF_PIPE;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int q = 0; q < 2; ++q) {
      PpPipe& P = ctl.pipe[q];
      mbar_init(&P.q_full, 1);
      mbar_init(&P.q_empty, 1);
      for (int i = 0; i < 2; ++i) {
        mbar_init(&P.k_full[i], 1);
        mbar_init(&P.v_full[i], 1);
        mbar_init(&P.kv_empty[i], 1);
        mbar_init(&P.ti_full[i], 1);
        mbar_init(&P.ti_empty[i], kSoftmaxThreads + 1);
      }
      mbar_init(&P.s_full, 1);
      mbar_init(&P.s_free, kSoftmaxThreads);
      mbar_init(&P.p_full, kSoftmaxThreads);
      mbar_init(&P.pv_done, 1);
      mbar_init(&P.o_full, 1);
      mbar_init(&P.r_full, 1);
      mbar_init(&P.r_empty, kSoftmaxThreads);
      mbar_init(&P.stg_ready, 1);
      mbar_init(&P.stg_full, kSoftmaxThreads);
    }
    mbar_init(&ctl.drain[0], 1);
    mbar_init(&ctl.drain[1], 1);
    ctl.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kPpMmaWarp) {
    tmem_alloc(&ctl.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;

  if (warp < 8) {
    reg_set<kPpRegsLaunch, kPpRegsSoftmax>();
    const int pipe = warp >> 2;
    pp_softmax(tm, p, ctl, pipes + pipe * C::PIPE_BYTES, tmem, pipe, ntiles);
  } else {
    reg_set<kPpRegsLaunch, kPpRegsOther>();
    if (warp == kPpProducerWarp) {
      if (lane < 2) pp_producer(tm, p, ctl, pipes + lane * C::PIPE_BYTES, lane, ntiles);
    } else if (warp < kPpMmaWarp + 2 && lane == 0) {
      const int pipe = warp - kPpMmaWarp;
      pp_mma(p, ctl, pipes + pipe * C::PIPE_BYTES, tmem, pipe, ntiles);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kPpMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace rtb
