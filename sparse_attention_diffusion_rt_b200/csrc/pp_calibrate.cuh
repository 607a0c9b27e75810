// Ping-pong calibration kernel for head dimensions up to 64.
//
// Same computation as attn_kernel<.., CAL=true> (the calibration step of
// "Re-ttention", OpenReview replies to W1: full attention plus the in-window /
// out-of-window split of the softmax denominator and of the output under one
// shared row max; rho = l_in / (l_in + l_out), R = acc_out / (l_in + l_out)).
// Each CTA computes two query tiles of one (batch, head), qb = 2x and 2x+1, in
// two pipelines that visit every key block in the same ascending order, so one
// K/V ring in shared memory feeds both.  One pipeline's exp-bound softmax
// overlaps the other's max, barrier latency and MMAs.
//
// Threads (352): warps 0-3 softmax + epilogue of tile A, warps 4-7 of tile B,
// lane 0 of warp 8 the TMA producer, lane 0 of warps 9 and 10 the MMA issuers
// of A and B.  Each 128-key block is processed as two 64-key sub-blocks so
// that a pipeline fits in 256 TMEM columns with its own P: S logits [0,64),
// bf16 P [64,96), acc_in [128,192), acc_out [192,256) (columns 256p.. for
// pipeline p).  A pipeline's next QK^T is issued as soon as its softmax has read
// the current 64 logits (s_free); P is rewritten once the previous PV is done
// (pv_done).  A K/V stage is released when both pipelines' PVs of both halves
// of that block are done.
#pragma once
#include <cuda.h>
#include <cstdint>

#include "attn_kernel.cuh"
#include "ptx.cuh"
#include "softmax.cuh"

namespace rtb {

struct PcCfg {
  static constexpr int TILE = 128 * 64 * 2;
  static constexpr int NST = 3;
  static constexpr int OFF_Q = 2048;                       // Q_A, Q_B (later O staging of A, B)
  static constexpr int OFF_STAGE = OFF_Q + 2 * TILE;
  static constexpr int OFF_R = OFF_STAGE + NST * 2 * TILE;  // R staging of A, B (fp32 size each)
  static constexpr int R_BYTES = 128 * 64 * 4;
  static constexpr int SMEM = OFF_R + 2 * R_BYTES + 1024;
  static_assert(SMEM <= 232448, "shared memory per CTA");
};

struct PcPipe {
  uint64_t q_full, s_full, s_free, p_full, pv_done, o_full, epi, drain;
};

struct PcCtrl {
  PcPipe pipe[2];
  uint64_t k_full[PcCfg::NST], v_full[PcCfg::NST], kv_empty[PcCfg::NST];
  uint32_t tmem_base;
  volatile int abort_flag;
  int bad_index[2];
  int npipes;
  uint32_t kept_bits[2][kMaxKeyBlocks / 32];
};
static_assert(sizeof(PcCtrl) <= PcCfg::OFF_Q, "control block");

__device__ __forceinline__ bool pc_kept(const PcCtrl& ctl, int pipe, int kb) {
  return (ctl.kept_bits[pipe][kb >> 5] >> (kb & 31)) & 1u;
}

__device__ __forceinline__ void pc_producer(const TmaSet& tm, const AttnParams& p, PcCtrl& ctl, uint8_t* base,
                                            int b, int h, int qb0) {
  using C = PcCfg;
  int issued = 0;
  bool ok = true;
  for (int q = 0; q < ctl.npipes; ++q) {
    mbar_arrive_expect_tx(&ctl.pipe[q].q_full, C::TILE);
    tma_load_4d(base + C::OFF_Q + q * C::TILE, &tm.q[0], &ctl.pipe[q].q_full, 0, (qb0 + q) * 128, h, b);
  }
  for (int j = 0; j < p.nkb; ++j) {
    const int st = j % C::NST;
    if (j >= C::NST && !sp_wait(&ctl.kv_empty[st], ((j / C::NST) - 1) & 1, ctl, p)) { ok = false; break; }
    uint8_t* sK = base + C::OFF_STAGE + st * 2 * C::TILE;
    mbar_arrive_expect_tx(&ctl.k_full[st], C::TILE);
    tma_load_4d(sK, &tm.k[0], &ctl.k_full[st], 0, j * 128, h, b);
    mbar_arrive_expect_tx(&ctl.v_full[st], C::TILE);
    tma_load_4d(sK + C::TILE, &tm.v[0], &ctl.v_full[st], 0, j * 128, h, b);
    issued = j + 1;
  }
  if (!ok) {
    const uint64_t lim = p.wait_limit_ns;
    for (int q = 0; q < ctl.npipes; ++q) drain_wait(&ctl.pipe[q].q_full, 0, lim);
    for (int j = (issued > C::NST ? issued - C::NST : 0); j < issued; ++j) {
      drain_wait(&ctl.k_full[j % C::NST], (j / C::NST) & 1, lim);
      drain_wait(&ctl.v_full[j % C::NST], (j / C::NST) & 1, lim);
    }
  }
}

__device__ __forceinline__ void pc_mma(const AttnParams& p, PcCtrl& ctl, uint8_t* base, uint32_t tmem, int pipe) {
  using C = PcCfg;
  constexpr uint32_t IDESC_QK = make_idesc_bf16(128, 64, 0, 0);
  constexpr uint32_t IDESC_PV = make_idesc_bf16(128, 64, 0, 1);
  PcPipe& P = ctl.pipe[pipe];
  const uint32_t tbase = tmem + 256u * pipe;
  const uint32_t q_addr = smem_u32(base + C::OFF_Q + pipe * C::TILE);
  const uint32_t stage0 = smem_u32(base + C::OFF_STAGE);
  const int nsub = 2 * p.nkb;
  bool first_in = true, first_out = true;

  // S(u) = Q K_u^T for the 64 keys of sub-block u (block u/2, half u%2)
  auto issue_qk = [&](int u) -> bool {
    const int j = u >> 1, st = j % C::NST;
    if (!(u & 1) && !sp_wait(&ctl.k_full[st], (j / C::NST) & 1, ctl, p)) return false;
    if (u > 0 && !sp_wait(&P.s_free, (u - 1) & 1, ctl, p)) return false;
    tc_fence_after();
    const uint32_t k_half = stage0 + st * 2 * C::TILE + (u & 1) * 64 * 128;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ss(tbase, kmajor_desc<64>(q_addr, 128, kk), kmajor_desc<64>(k_half, 64, kk), IDESC_QK, kk > 0 ? 1u : 0u);
    mma_commit(&P.s_full);
    return true;
  };
  auto issue_pv = [&](int u) -> bool {
    const int j = u >> 1, st = j % C::NST;
    if (!sp_wait(&P.p_full, u & 1, ctl, p)) return false;
    if (!(u & 1) && !sp_wait(&ctl.v_full[st], (j / C::NST) & 1, ctl, p)) return false;
    tc_fence_after();
    const bool kept = pc_kept(ctl, pipe, j);
    const uint32_t dst = tbase + (kept ? 128u : 192u);
    const bool first = kept ? first_in : first_out;
    if (kept) first_in = false; else first_out = false;
    const uint32_t v_tile = stage0 + st * 2 * C::TILE + C::TILE;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ts(dst, tbase + 64 + kk * 8, v_desc_c0<64, 128>(v_tile, 4 * (u & 1) + kk), IDESC_PV,
             (first && kk == 0) ? 0u : 1u);
    if (u & 1) mma_commit(&ctl.kv_empty[st]);
    mma_commit(&P.pv_done);
    return true;
  };

  bool ok = sp_wait(&P.q_full, 0, ctl, p) && issue_qk(0);
  for (int u = 0; ok && u < nsub; ++u) {
    if (u + 1 < nsub && !issue_qk(u + 1)) { ok = false; break; }
    if (!issue_pv(u)) { ok = false; break; }
  }
  if (ok) {
    mma_commit(&P.o_full);
  } else {
    mma_commit(&P.drain);
    drain_wait(&P.drain, 0, p.wait_limit_ns);
  }
}

__device__ __forceinline__ void pc_softmax(const TmaSet& tm, const AttnParams& p, PcCtrl& ctl, uint8_t* base,
                                           uint32_t tmem, int pipe, int b, int h, int qb) {
  using C = PcCfg;
  PcPipe& P = ctl.pipe[pipe];
  const int t = threadIdx.x & 127;
  const int wq = (threadIdx.x >> 5) & 3;
  const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
  const uint32_t tS = tmem + 256u * pipe + lane_base;
  const uint32_t tP = tS + 64, tIn = tS + 128, tOut = tS + 192;
  const float sl2 = p.scale_log2;
  float m = 0.f, l_in = 0.f, l_out = 0.f;
  bool any_in = false, any_out = false;
  bool ok = true;
  const int nsub = 2 * p.nkb;
  for (int u = 0; u < nsub; ++u) {
    ok = __all_sync(0xffffffffu, sp_wait(&P.s_full, u & 1, ctl, p));
    if (!ok) break;
    tc_fence_after();
    uint32_t s[64];
    tmem_ld_x32(tS, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
    tmem_ld_x32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
    tmem_wait_ld();
    tc_fence_before();
    mbar_arrive(&P.s_free);
    const int j = u >> 1;
    mask_tail<64>(s, p.L - j * 128 - (u & 1) * 64);
    const float mx = row_max<64>(s) * sl2;
    bool need_pv = u > 0;
    if (u == 0) {
      m = mx;
    } else if (__any_sync(0xffffffffu, mx > m + kRescaleLog2)) {
      const float m_new = fmaxf(m, mx);
      const float alpha = ex2_approx(m - m_new);
      l_in *= alpha;
      l_out *= alpha;
      ok = __all_sync(0xffffffffu, sp_wait(&P.pv_done, (u - 1) & 1, ctl, p));
      if (!ok) break;
      need_pv = false;
      tc_fence_after();
      if (any_in) rescale_row<64>(tIn, alpha);
      if (any_out) rescale_row<64>(tOut, alpha);
      m = m_new;
    }
    // p = 2^(s*sl2 - m), bf16 pairs into P (after the previous PV has read it)
    uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};
    const uint64_t scale2 = f2_pack(sl2, sl2), neg_m2 = f2_pack(-m, -m);
    uint32_t pk[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const uint64_t x = ffma2(f2_pack(__uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1])), scale2, neg_m2);
      float x0, x1;
      f2_unpack(x, x0, x1);
      const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
      sum2[c & 3] = fadd2(sum2[c & 3], f2_pack(p0, p1));
      pk[c] = pack_bf16x2(p0, p1);
    }
    if (need_pv) {
      ok = __all_sync(0xffffffffu, sp_wait(&P.pv_done, (u - 1) & 1, ctl, p));
      if (!ok) break;
      tc_fence_after();
    }
    tmem_st_x32(tP, pk);
    float lo, hi;
    f2_unpack(fadd2(fadd2(sum2[0], sum2[1]), fadd2(sum2[2], sum2[3])), lo, hi);
    if (pc_kept(ctl, pipe, j)) { l_in += lo + hi; any_in = true; } else { l_out += lo + hi; any_out = true; }
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&P.p_full);
  }
  if (ok) {
    ok = __all_sync(0xffffffffu, sp_wait(&P.o_full, 0, ctl, p));
    if (ok) tc_fence_after();
  }
  // ------------------------------------------------------------- epilogue
  const int grow = qb * 128 + t;
  uint8_t* sO = base + C::OFF_Q + pipe * C::TILE;         // Q is no longer read (o_full)
  uint8_t* sRst = base + C::OFF_R + pipe * C::R_BYTES;
  if (ok) {
    const float z = l_in + l_out;
    const float inv = 1.f / z;
    const float inv_in = l_in > 0.f ? 1.f / l_in : 0.f;
    if (grow < p.L) p.rho_out[(static_cast<size_t>(b) * p.H + h) * p.L + grow] = l_in / z;
#pragma unroll
    for (int h0 = 0; h0 < 64; h0 += 32) {
      uint32_t ain[32], aout[32];
      if (any_in) tmem_ld_x32(tIn + h0, ain);
      if (any_out) tmem_ld_x32(tOut + h0, aout);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 32; c += 16) {
        float o16[16], r16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float xi = any_in ? __uint_as_float(ain[c + i]) : 0.f;
          const float xo = any_out ? __uint_as_float(aout[c + i]) : 0.f;
          o16[i] = (xi + xo) * inv;
          // masked tokens' part, or O_full - O_sparse with O_sparse = acc_in / l_in (0 with no kept key)
          r16[i] = p.r_sub ? o16[i] - xi * inv_in : xo * inv;
        }
        store_row16<64>(sO, 128, t, h0 + c, false, o16);
        store_row16<64>(sRst, 128, t, h0 + c, p.r_f32 != 0, r16);
      }
    }
  }
  fence_proxy_async_smem();
  mbar_arrive(&P.epi);
  if (t == 0) {
    if (sp_wait(&P.epi, 0, ctl, p) && !ctl.abort_flag) {
      tma_store_4d(&tm.o[0], sO, 0, qb * 128, h, b);
      if (p.r_f32) {
        tma_store_4d(&tm.r[0], sRst, 0, qb * 128, h, b);
        tma_store_4d(&tm.r[1], sRst + 128 * 128, 32, qb * 128, h, b);
      } else {
        tma_store_4d(&tm.r[0], sRst, 0, qb * 128, h, b);
      }
      tma_store_commit();
      tma_store_wait0();
    }
  }
}

template <int DPAD>
__global__ void __launch_bounds__(352, 1)
pp_calibrate_kernel(const __grid_constant__ TmaSet tm, const AttnParams p) {
  using C = PcCfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  PcCtrl& ctl = *reinterpret_cast<PcCtrl*>(base);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb0 = 2 * blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int npipes = (qb0 + 1 < p.nqb) ? 2 : 1;
  const int hm = (p.Hm == 1) ? 0 : h;

  if (threadIdx.x == 0) {
    for (int q = 0; q < 2; ++q) {
      PcPipe& P = ctl.pipe[q];
      mbar_init(&P.q_full, 1);
      mbar_init(&P.s_full, 1);
      mbar_init(&P.s_free, kSoftmaxThreads);
      mbar_init(&P.p_full, kSoftmaxThreads);
      mbar_init(&P.pv_done, 1);
      mbar_init(&P.o_full, 1);
      mbar_init(&P.epi, kSoftmaxThreads);
      mbar_init(&P.drain, 1);
    }
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(&ctl.k_full[s], 1);
      mbar_init(&ctl.v_full[s], 1);
      mbar_init(&ctl.kv_empty[s], npipes);
    }
    ctl.abort_flag = 0;
    ctl.npipes = npipes;
    fence_mbar_init();
  }
  if (warp == 8) {
    // validate both CSR rows and build their kept-block bitmaps
    for (int q = 0; q < 2; ++q) {
      for (int w = lane; w < kMaxKeyBlocks / 32; w += 32) ctl.kept_bits[q][w] = 0u;
    }
    __syncwarp();
    int bad_any = 0;
    for (int q = 0; q < npipes; ++q) {
      const int row = hm * p.nqb + qb0 + q;
      int start = 0, end = 0, bad = 0;
      if (lane == 0) {
        start = __ldg(p.row_ptr + row);
        end = __ldg(p.row_ptr + row + 1);
        if (start < 0 || end < start || static_cast<long long>(end) > p.nnz || end - start > p.nkb) bad = 1;
      }
      start = __shfl_sync(0xffffffffu, start, 0);
      end = __shfl_sync(0xffffffffu, end, 0);
      bad = __shfl_sync(0xffffffffu, bad, 0);
      if (!bad) {
        for (int i = lane; i < end - start; i += 32) {
          const int c = __ldg(p.col_idx + start + i);
          const int prev = i > 0 ? __ldg(p.col_idx + start + i - 1) : -1;
          if (c < 0 || c >= p.nkb || c <= prev) bad = 1;
          else atomicOr(&ctl.kept_bits[q][c >> 5], 1u << (c & 31));
        }
      }
      bad_any |= __any_sync(0xffffffffu, bad);
    }
    if (lane == 0) ctl.bad_index[0] = bad_any;
  }
  if (warp == 9) {
    tmem_alloc(&ctl.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;

  if (ctl.bad_index[0]) {
    if (threadIdx.x == 0) record_status(p.status, RT_ERR_BAD_INDEX);
  } else if (warp < 8) {
    const int pipe = warp >> 2;
    if (pipe < npipes) pc_softmax(tm, p, ctl, base, tmem, pipe, b, h, qb0 + pipe);
  } else if (warp == 8) {
    if (lane == 0) pc_producer(tm, p, ctl, base, b, h, qb0);
  } else if (lane == 0) {
    const int pipe = warp - 9;
    if (pipe < npipes) pc_mma(p, ctl, base, tmem, pipe);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace rtb
