// Warp-specialised sm_100a attention kernel for Re-ttention's two hot steps.
//
// CAL = true  -- calibration (full-attention) step: visits every key block,
//   keeps the kept-block and masked-block softmax sums (l_in, l_out) and
//   outputs (acc_in, acc_out) apart under one shared row max, and emits
//   O = (acc_in + acc_out) / Z, R = acc_out / Z, rho = l_in / Z with
//   Z = l_in + l_out ("Re-ttention", OpenReview replies to W1: rho = Z_sparse /
//   Z_full, the residual holds only the masked tokens' attention).
// CAL = false -- reshaped sparse step: visits only the key blocks listed in
//   the CSR block index and emits O = rho_hat * acc / l + R (O = R for an
//   empty row), rho_hat = min(1, rho * ramp_mul + ramp_add) (reply to Pwod's
//   W1: the cached rho plus a ramp-up lambda).
//
// One CTA computes one (batch, head, query block).  The query tile is always
// 128 rows (the tcgen05 M); with 64-token blocks only the first 64 rows are
// stored.  Warps 0-3 (one TMEM lane quarter each; thread t owns row t) run the
// softmax and the epilogue, warp 4 issues TMA loads, one thread of warp 5
// issues the tcgen05 MMAs.  TMEM columns: S [0,128) fp32 logits, P0/P1
// [128,256) bf16 probabilities (A operand of the PV MMA), O [256, 256+DPAD)
// (calibration: acc_in [256,384), acc_out [384,512)).
//
// Softmax: thread-per-row, so the row max and sum need no shuffles.  The
// running max is only moved (and O rescaled in TMEM) when a block's max
// exceeds it by more than 2^8; otherwise probabilities are taken against the
// stale max, which leaves O/l unchanged and keeps every p below 256.
//
// Every wait is bounded (p.wait_limit_ns).  On a timeout the CTA records
// RT_ERR_TIMEOUT, each role drains what it has in flight, TMEM is freed and the
// CTA returns.  A bad CSR row is detected before any copy or MMA is issued.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "rt.h"
#include "softmax.cuh"

namespace rtb {

constexpr int kThreads = 192;
constexpr int kSoftmaxThreads = 128;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kMaxKeyBlocks = 4096;
constexpr float kRescaleLog2 = 8.0f;
// Every p of a row block is at most the block's row sum (p >= 0, and a rounded
// sum of non-negative terms is no smaller than any of them), and x > 8 gives
// p = 2^x > 255.  A block whose row sums are all <= 255 therefore needs no
// rescale, and only then is its largest x taken (exactly) at all.
constexpr float kRescaleSum = 255.0f;
constexpr uint32_t kTmemCols = 512;

struct TmaSet {
  CUtensorMap q[2];
  CUtensorMap k[2];
  CUtensorMap v[2];
  CUtensorMap o[2];
  CUtensorMap r[4];   // bf16 residual: chunks as Q; fp32 residual: 32-column chunks
};

struct AttnParams {
  int B, H, L, d, block;
  int nqb, nkb, Hm;
  long long nnz;
  const int* row_ptr;
  const int* col_idx;
  float scale_log2;        // softmax scale * log2(e)
  const float* rho_in;     // sparse step
  const void* r_in;        // sparse step residual (read directly when fp32)
  long long stride_b, stride_h, stride_l;
  float ramp_mul, ramp_add;
  float* rho_out;          // calibration
  int r_f32;
  int use_rho, use_r;      // sparse-step epilogue: O' = (use_rho ? rho_hat : 1) * attn + (use_r ? R : 0)
  int r_sub;               // calibration: R = O_full - O_sparse (subtractive residual) instead of the masked part
  unsigned long long wait_limit_ns;
  unsigned int* status;
};

template <int DPAD, int BN>
struct Cfg {
  static_assert(DPAD == 64 || DPAD == 80 || DPAD == 96 || DPAD == 128, "padded head dim");
  static_assert(BN == 128 || (BN == 64 && DPAD == 64), "key block");
  static constexpr int C1 = DPAD - 64;            // width of the second column chunk
  static constexpr int C1B = C1 * 2;              // its row bytes (32 / 64 / 128)
  static constexpr uint32_t C1SWZ = C1 == 16 ? SWZ_32B : (C1 == 32 ? SWZ_64B : SWZ_128B);
  static constexpr int NST = DPAD <= 96 ? 3 : 2;  // K/V pipeline stages
  static constexpr int Q_BYTES = 128 * DPAD * 2;
  static constexpr int KT_BYTES = BN * DPAD * 2;
  static constexpr int STAGE_BYTES = 2 * KT_BYTES;
  static constexpr int NCH32 = (DPAD + 31) / 32;  // fp32 residual chunks of 32 columns
  static constexpr int R_MAX_BYTES = 128 * NCH32 * 128;
  static constexpr int CTRL_BYTES = 1024;
  static constexpr int OFF_Q = CTRL_BYTES;
  static constexpr int OFF_STAGE = OFF_Q + Q_BYTES;
  static constexpr int OFF_R = OFF_STAGE + NST * STAGE_BYTES;
  static constexpr int SMEM_CAL = OFF_R + 1024;               // + alignment slack
  static constexpr int SMEM_SPARSE = OFF_R + R_MAX_BYTES + 1024;
  static_assert(NST * STAGE_BYTES >= R_MAX_BYTES, "calibration residual staging fits the stages");
  static_assert(SMEM_SPARSE <= 232448, "shared memory per CTA");
  static_assert(Q_BYTES % 1024 == 0 && KT_BYTES % 1024 == 0, "1024-byte aligned regions");
  // TMEM columns
  static constexpr uint32_t T_S = 0, T_P0 = 128, T_P1 = 192, T_O = 256, T_OUT = 384;
};

struct Ctrl {
  uint64_t q_full, r_full, s_full, s_free, o_ready, o_final, drain, epi;
  uint64_t p_full[2];
  uint64_t k_full[3], v_full[3], kv_empty[3];
  uint32_t tmem_base;
  volatile int abort_flag;
  int bad_index;
  int n_blocks;
  int row_start;
  int n_kept;               // calibration: kept blocks in this row
  uint32_t kept_bits[kMaxKeyBlocks / 32];
};
static_assert(sizeof(Ctrl) <= 1024, "control block");

__device__ __forceinline__ void record_status(unsigned int* status, unsigned int code) {
  atomicCAS(status, 0u, code);
}

// Bounded mbarrier wait.  Returns false after a timeout (recorded) or when
// another role of the CTA has already aborted.
static __device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Ctrl& ctl,
                                      const AttnParams& p) {
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

// Drain wait used after an abort: ignores the abort flag and is bounded by its
// own limit (at least one second), so that copies and MMAs already in flight
// land before shared memory and TMEM are released.
constexpr uint64_t kDrainMinNs = 1000000000ull;
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (limit_ns < kDrainMinNs) limit_ns = kDrainMinNs;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) return;
  }
}

// Calibration visits every key block in ascending order; the CTAs of a head
// then stream the same K/V blocks at about the same time and share them in L2
// (a per-CTA rotated order measured slower).
__device__ __forceinline__ int cal_kb(const AttnParams&, int, int j) { return j; }

__device__ __forceinline__ bool is_kept(const Ctrl& ctl, int kb) {
  return (ctl.kept_bits[kb >> 5] >> (kb & 31)) & 1u;
}

// ------------------------------------------------------------------ descriptors
// K-major operand tile [rows][DPAD] bf16 stored as chunk 0 (64 columns, 128B
// swizzle, rows*128 bytes) followed by chunk 1 (C1 columns).  MMA k-step kk
// covers columns [16kk, 16kk+16).
template <int DPAD>
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int rows, int kk) {
  using C = Cfg<DPAD, 128>;
  if (kk < 4) return make_smem_desc(tile + kk * 32, 16, 1024, SWZ_128B);
  const uint32_t c1 = tile + rows * 128;
  return make_smem_desc(c1 + (kk - 4) * 32, 16, 8 * C::C1B, C::C1SWZ);
}

// MN-major V tile [BN keys][DPAD] (same chunked storage), k-step kk covers keys
// [16kk, 16kk+16).  chunk 0 spans 64 columns; for DPAD == 128 one descriptor
// spans both chunks through the leading byte offset (distance between chunks).
template <int DPAD, int BN>
__device__ __forceinline__ uint64_t v_desc_c0(uint32_t tile, int kk) {
  return make_smem_desc(tile + kk * 16 * 128, BN * 128, 1024, SWZ_128B);
}
template <int DPAD, int BN>
__device__ __forceinline__ uint64_t v_desc_c1(uint32_t tile, int kk) {
  using C = Cfg<DPAD, BN>;
  const uint32_t c1 = tile + BN * 128;
  return make_smem_desc(c1 + kk * 16 * C::C1B, 0, 8 * C::C1B, C::C1SWZ);
}

// ------------------------------------------------------------------ roles
template <int DPAD, int BN, bool CAL>
__device__ __forceinline__ void producer_role(const TmaSet& tm, const AttnParams& p, Ctrl& ctl,
                                              uint8_t* sQ, uint8_t* sStage, uint8_t* sR,
                                              int b, int h, int qb, int n) {
  using C = Cfg<DPAD, BN>;
  const int q_row = qb * p.block;
  int issued = 0;
  bool ok = true;
  if (!CAL && !p.use_r) {
    mbar_arrive(&ctl.r_full);               // no residual in this epilogue: nothing to load
  } else if (!CAL) {
    // residual tile for the epilogue: independent of the main loop, issue first
    const uint32_t rbytes = p.r_f32 ? p.block * C::NCH32 * 128 : p.block * DPAD * 2;
    mbar_arrive_expect_tx(&ctl.r_full, rbytes);
    if (p.r_f32) {
      for (int c = 0; c < C::NCH32; ++c)
        tma_load_4d(sR + c * p.block * 128, &tm.r[c], &ctl.r_full, c * 32, q_row, h, b);
    } else {
      tma_load_4d(sR, &tm.r[0], &ctl.r_full, 0, q_row, h, b);
      if (C::C1) tma_load_4d(sR + p.block * 128, &tm.r[1], &ctl.r_full, 64, q_row, h, b);
    }
  }
  if (n > 0) {
    mbar_arrive_expect_tx(&ctl.q_full, C::Q_BYTES);
    tma_load_4d(sQ, &tm.q[0], &ctl.q_full, 0, q_row, h, b);
    if (C::C1) tma_load_4d(sQ + 128 * 128, &tm.q[1], &ctl.q_full, 64, q_row, h, b);
  }
  for (int j = 0; j < n; ++j) {
    const int st = j % C::NST;
    const uint32_t use = j / C::NST;
    if (j >= C::NST && !wait_bar(&ctl.kv_empty[st], (use - 1) & 1, ctl, p)) { ok = false; break; }
    const int kb = CAL ? cal_kb(p, qb, j) : __ldg(p.col_idx + ctl.row_start + j);
    uint8_t* sK = sStage + st * C::STAGE_BYTES;
    uint8_t* sV = sK + C::KT_BYTES;
    mbar_arrive_expect_tx(&ctl.k_full[st], C::KT_BYTES);
    tma_load_4d(sK, &tm.k[0], &ctl.k_full[st], 0, kb * BN, h, b);
    if (C::C1) tma_load_4d(sK + BN * 128, &tm.k[1], &ctl.k_full[st], 64, kb * BN, h, b);
    mbar_arrive_expect_tx(&ctl.v_full[st], C::KT_BYTES);
    tma_load_4d(sV, &tm.v[0], &ctl.v_full[st], 0, kb * BN, h, b);
    if (C::C1) tma_load_4d(sV + BN * 128, &tm.v[1], &ctl.v_full[st], 64, kb * BN, h, b);
    issued = j + 1;
  }
  if (!ok) {
    // let every copy this thread started land before shared memory is released
    const uint64_t lim = p.wait_limit_ns;
    if (n > 0) drain_wait(&ctl.q_full, 0, lim);
    if (!CAL) drain_wait(&ctl.r_full, 0, lim);
    for (int j = (issued > C::NST ? issued - C::NST : 0); j < issued; ++j) {
      const int st = j % C::NST;
      const uint32_t par = (j / C::NST) & 1;
      drain_wait(&ctl.k_full[st], par, lim);
      drain_wait(&ctl.v_full[st], par, lim);
    }
  }
}

template <int DPAD, int BN, bool CAL>
__device__ __forceinline__ void mma_role(const AttnParams& p, Ctrl& ctl, uint8_t* sQ,
                                         uint8_t* sStage, uint32_t tmem, int n) {
  using C = Cfg<DPAD, BN>;
  constexpr uint32_t IDESC_QK = make_idesc_bf16(128, BN, 0, 0);
  constexpr uint32_t IDESC_PV_FULL = make_idesc_bf16(128, DPAD == 128 ? 128 : 64, 0, 1);
  constexpr uint32_t IDESC_PV_C1 = make_idesc_bf16(128, C::C1 > 0 ? C::C1 : 16, 0, 1);
  if (n == 0) return;
  const uint32_t q_addr = smem_u32(sQ);
  const uint32_t stage0 = smem_u32(sStage);
  bool first_in = true, first_out = true;
  bool ok = wait_bar(&ctl.q_full, 0, ctl, p);

  auto issue_pv = [&](int i) -> bool {
    const int st = i % C::NST;
    const uint32_t ph = (i / C::NST) & 1;
    if (!wait_bar(&ctl.p_full[i & 1], (i >> 1) & 1, ctl, p)) return false;
    if (!wait_bar(&ctl.v_full[st], ph, ctl, p)) return false;
    tc_fence_after();
    const uint32_t v_tile = stage0 + st * C::STAGE_BYTES + C::KT_BYTES;
    const uint32_t tp = tmem + ((i & 1) ? C::T_P1 : C::T_P0);
    uint32_t dst = tmem + C::T_O;
    bool first = (i == 0);
    if (CAL) {
      const bool kept = is_kept(ctl, cal_kb(p, blockIdx.x, i));
      dst = tmem + (kept ? C::T_O : C::T_OUT);
      first = kept ? first_in : first_out;
      if (kept) first_in = false; else first_out = false;
    }
#pragma unroll
    for (int kk = 0; kk < BN / 16; ++kk) {
      const uint32_t acc = (first && kk == 0) ? 0u : 1u;
      mma_ts(dst, tp + kk * 8, v_desc_c0<DPAD, BN>(v_tile, kk), IDESC_PV_FULL, acc);
      if (C::C1 > 0 && DPAD != 128)
        mma_ts(dst + 64, tp + kk * 8, v_desc_c1<DPAD, BN>(v_tile, kk), IDESC_PV_C1, acc);
    }
    mma_commit(&ctl.kv_empty[st]);
    mma_commit(&ctl.o_ready);
    return true;
  };

  for (int j = 0; ok && j < n; ++j) {
    const int st = j % C::NST;
    const uint32_t ph = (j / C::NST) & 1;
    if (!wait_bar(&ctl.k_full[st], ph, ctl, p)) { ok = false; break; }
    if (j > 0 && !wait_bar(&ctl.s_free, (j - 1) & 1, ctl, p)) { ok = false; break; }
    tc_fence_after();
    const uint32_t k_tile = stage0 + st * C::STAGE_BYTES;
#pragma unroll
    for (int kk = 0; kk < DPAD / 16; ++kk)
      mma_ss(tmem + C::T_S, kmajor_desc<DPAD>(q_addr, 128, kk), kmajor_desc<DPAD>(k_tile, BN, kk),
             IDESC_QK, kk > 0 ? 1u : 0u);
    mma_commit(&ctl.s_full);
    if (j > 0 && !issue_pv(j - 1)) { ok = false; break; }
  }
  if (ok) ok = issue_pv(n - 1);
  if (ok) {
    mma_commit(&ctl.o_final);
  } else {
    mma_commit(&ctl.drain);
    drain_wait(&ctl.drain, 0, p.wait_limit_ns);
  }
}

// Residual row chunk (16 columns starting at c) from a bf16 or fp32 tile in the
// chunked, swizzled shared-memory layout the TMA copies use.
template <int DPAD>
__device__ __forceinline__ void load_row16(const uint8_t* tile, int rows, int t, int c, bool f32,
                                           float (&out)[16]) {
  using C = Cfg<DPAD, 128>;
  if (f32) {
    const int ch = c >> 5, col = c & 31;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t off = swz_off(t * 128 + (col * 4 + u * 16), 128);
      const float4 v4 = *reinterpret_cast<const float4*>(tile + ch * rows * 128 + off);
      out[4 * u + 0] = v4.x; out[4 * u + 1] = v4.y; out[4 * u + 2] = v4.z; out[4 * u + 3] = v4.w;
    }
  } else {
    const bool c1 = c >= 64;
    const uint32_t rb = c1 ? C::C1B : 128;
    const uint32_t base = c1 ? rows * 128 : 0;
    const int col = c1 ? c - 64 : c;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint32_t off = swz_off(t * rb + (col * 2 + u * 16), rb);
      const uint4 v4 = *reinterpret_cast<const uint4*>(tile + base + off);
      const uint32_t w[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        out[8 * u + 2 * e] = __uint_as_float(w[e] << 16);
        out[8 * u + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
      }
    }
  }
}

template <int DPAD>
__device__ __forceinline__ void store_row16(uint8_t* tile, int rows, int t, int c, bool f32,
                                            const float (&x)[16]) {
  using C = Cfg<DPAD, 128>;
  if (f32) {
    const int ch = c >> 5, col = c & 31;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t off = swz_off(t * 128 + (col * 4 + u * 16), 128);
      *reinterpret_cast<float4*>(tile + ch * rows * 128 + off) =
          make_float4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]);
    }
  } else {
    const bool c1 = c >= 64;
    const uint32_t rb = c1 ? C::C1B : 128;
    const uint32_t base = c1 ? rows * 128 : 0;
    const int col = c1 ? c - 64 : c;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      uint4 w;
      w.x = pack_bf16x2(x[8 * u + 0], x[8 * u + 1]);
      w.y = pack_bf16x2(x[8 * u + 2], x[8 * u + 3]);
      w.z = pack_bf16x2(x[8 * u + 4], x[8 * u + 5]);
      w.w = pack_bf16x2(x[8 * u + 6], x[8 * u + 7]);
      const uint32_t off = swz_off(t * rb + (col * 2 + u * 16), rb);
      *reinterpret_cast<uint4*>(tile + base + off) = w;
    }
  }
}

template <int DPAD, int BN, bool CAL>
__device__ __forceinline__ void softmax_role(const TmaSet& tm, const AttnParams& p, Ctrl& ctl,
                                             uint8_t* sQ, uint8_t* sStage, uint8_t* sR,
                                             uint32_t tmem, int b, int h, int qb, int n) {
  using C = Cfg<DPAD, BN>;
  const int t = threadIdx.x;             // tile row
  const int warp = t >> 5;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tS = tmem + lane_base + C::T_S;
  const uint32_t tO = tmem + lane_base + C::T_O;
  const uint32_t tOut = tmem + lane_base + C::T_OUT;
  const float sl2 = p.scale_log2;
  float m = 0.f;                          // running max (log2 domain)
  float l = 0.f, l_out = 0.f;             // l (sparse) or l_in (calibration); l_out
  bool any_in = false, any_out = false;   // calibration: accumulators written so far
  bool ok = true;

  for (int j = 0; j < n; ++j) {
    ok = __all_sync(0xffffffffu, wait_bar(&ctl.s_full, j & 1, ctl, p));
    if (!ok) break;
    tc_fence_after();
    uint32_t s[BN];
    load_scores<BN>(tS, s);
    tmem_wait_ld();
    tc_fence_before();
    mbar_arrive(&ctl.s_free);

    const int kb = CAL ? cal_kb(p, qb, j) : __ldg(p.col_idx + ctl.row_start + j);
    mask_tail<BN>(s, p.L - kb * BN);                 // keys past the end of the sequence
    const float mx = row_max<BN>(s) * sl2;
    if (j == 0) {
      m = mx;
    } else if (__any_sync(0xffffffffu, mx > m + kRescaleLog2)) {
      // warp-uniform: TMEM loads/stores are .sync.aligned
      const float m_new = fmaxf(m, mx);
      const float alpha = ex2_approx(m - m_new);
      l *= alpha;
      l_out *= alpha;
      // the accumulators hold blocks 0..j-1: wait until the last of them has landed
      ok = __all_sync(0xffffffffu, wait_bar(&ctl.o_ready, (j - 1) & 1, ctl, p));
      if (!ok) break;
      tc_fence_after();
      if (!CAL || any_in) rescale_row<DPAD>(tO, alpha);
      if (CAL && any_out) rescale_row<DPAD>(tOut, alpha);
      m = m_new;
    }
    const uint32_t tP = tmem + lane_base + ((j & 1) ? C::T_P1 : C::T_P0);
    const float sum = exp_pack_store<BN>(s, sl2, m, tP);
    if (CAL) {
      if (is_kept(ctl, kb)) { l += sum; any_in = true; } else { l_out += sum; any_out = true; }
    } else {
      l += sum;
    }
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&ctl.p_full[j & 1]);
  }
  if (ok && n > 0) {
    ok = __all_sync(0xffffffffu, wait_bar(&ctl.o_final, 0, ctl, p));
    if (ok) tc_fence_after();
  }
  if (ok && !CAL) ok = __all_sync(0xffffffffu, wait_bar(&ctl.r_full, 0, ctl, p));

  // ------------------------------------------------------------- epilogue
  const int grow = qb * p.block + t;                 // sequence row of this thread
  const bool row_ok = t < p.block;                   // rows of this query block (warp-uniform)
  const size_t rho_idx = (static_cast<size_t>(b) * p.H + h) * p.L + grow;
  if (ok && row_ok) {
    float out_scale = 0.f, inv_in = 0.f;
    if (CAL) {
      out_scale = 1.f / (l + l_out);
      inv_in = l > 0.f ? 1.f / l : 0.f;
      if (grow < p.L) p.rho_out[rho_idx] = l / (l + l_out);   // correctly rounded: dense mask gives 1
    } else {
      const float rho = (p.use_rho && grow < p.L) ? __ldg(p.rho_in + rho_idx) : 0.f;
      const float rho_hat = p.use_rho ? fminf(1.f, fmaf(rho, p.ramp_mul, p.ramp_add)) : 1.f;
      out_scale = (n > 0) ? rho_hat / l : 0.f;
    }
#pragma unroll
    for (int c = 0; c < DPAD; c += 16) {
      float a[16];
      if (CAL) {
        uint32_t ain[16], aout[16];
        if (any_in) tmem_ld_x16(tO + c, ain);
        if (any_out) tmem_ld_x16(tOut + c, aout);
        tmem_wait_ld();
        float ro[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float xi = any_in ? __uint_as_float(ain[i]) : 0.f;
          const float xo = any_out ? __uint_as_float(aout[i]) : 0.f;
          a[i] = (xi + xo) * out_scale;
          // masked tokens' part, or O_full - O_sparse with O_sparse = acc_in / l_in (0 with no kept key)
          ro[i] = p.r_sub ? a[i] - xi * inv_in : xo * out_scale;
        }
        store_row16<DPAD>(sStage, p.block, t, c, p.r_f32 != 0, ro);
      } else {
        uint32_t acc[16];
        if (n > 0) { tmem_ld_x16(tO + c, acc); tmem_wait_ld(); }
        float rr[16];
        if (p.use_r) {
          load_row16<DPAD>(sR, p.block, t, c, p.r_f32 != 0, rr);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) rr[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) a[i] = (n > 0 ? __uint_as_float(acc[i]) * out_scale : 0.f) + rr[i];
      }
      store_row16<DPAD>(sQ, p.block, t, c, false, a);
    }
  }
  fence_proxy_async_smem();
  mbar_arrive(&ctl.epi);
  if (t == 0) {
    const bool all_ok = wait_bar(&ctl.epi, 0, ctl, p) && !ctl.abort_flag;
    if (all_ok) {
      const int q_row = qb * p.block;
      tma_store_4d(&tm.o[0], sQ, 0, q_row, h, b);
      if (C::C1) tma_store_4d(&tm.o[1], sQ + p.block * 128, 64, q_row, h, b);
      if (CAL) {
        if (p.r_f32) {
          for (int c = 0; c < C::NCH32; ++c)
            tma_store_4d(&tm.r[c], sStage + c * p.block * 128, c * 32, q_row, h, b);
        } else {
          tma_store_4d(&tm.r[0], sStage, 0, q_row, h, b);
          if (C::C1) tma_store_4d(&tm.r[1], sStage + p.block * 128, 64, q_row, h, b);
        }
      }
      tma_store_commit();
      tma_store_wait0();
    }
  }
}

template <int DPAD, int BN, bool CAL>
__global__ void __launch_bounds__(kThreads, 1)
attn_kernel(const __grid_constant__ TmaSet tm, const AttnParams p) {
  using C = Cfg<DPAD, BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  Ctrl& ctl = *reinterpret_cast<Ctrl*>(base);
  uint8_t* sQ = base + C::OFF_Q;
  uint8_t* sStage = base + C::OFF_STAGE;
  uint8_t* sR = base + C::OFF_R;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int hm = (p.Hm == 1) ? 0 : h;
  const int row = hm * p.nqb + qb;

  if (threadIdx.x == 0) {
    mbar_init(&ctl.q_full, 1);
    mbar_init(&ctl.r_full, 1);
    mbar_init(&ctl.s_full, 1);
    mbar_init(&ctl.s_free, kSoftmaxThreads);
    mbar_init(&ctl.o_ready, 1);
    mbar_init(&ctl.o_final, 1);
    mbar_init(&ctl.drain, 1);
    mbar_init(&ctl.epi, kSoftmaxThreads);
    mbar_init(&ctl.p_full[0], kSoftmaxThreads);
    mbar_init(&ctl.p_full[1], kSoftmaxThreads);
    for (int s = 0; s < 3; ++s) {
      mbar_init(&ctl.k_full[s], 1);
      mbar_init(&ctl.v_full[s], 1);
      mbar_init(&ctl.kv_empty[s], 1);
    }
    ctl.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp) {
    // validate this CSR row before anything is issued; build the kept bitmap
    int start = 0, end = 0, bad = 0;
    if (lane == 0) {
      start = __ldg(p.row_ptr + row);
      end = __ldg(p.row_ptr + row + 1);
      if (start < 0 || end < start || static_cast<long long>(end) > p.nnz || end - start > p.nkb) bad = 1;
    }
    start = __shfl_sync(0xffffffffu, start, 0);
    end = __shfl_sync(0xffffffffu, end, 0);
    bad = __shfl_sync(0xffffffffu, bad, 0);
    if (CAL)
      for (int w = lane; w < kMaxKeyBlocks / 32; w += 32) ctl.kept_bits[w] = 0u;
    __syncwarp();
    if (!bad) {
      for (int i = lane; i < end - start; i += 32) {
        const int c = __ldg(p.col_idx + start + i);
        const int prev = i > 0 ? __ldg(p.col_idx + start + i - 1) : -1;
        if (c < 0 || c >= p.nkb || c <= prev) bad = 1;
        else if (CAL) atomicOr(&ctl.kept_bits[c >> 5], 1u << (c & 31));
      }
    }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      ctl.bad_index = bad;
      ctl.row_start = start;
      ctl.n_blocks = CAL ? p.nkb : end - start;
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
  } else {
    const int n = ctl.n_blocks;
    if (warp == kProducerWarp) {
      if (lane == 0) producer_role<DPAD, BN, CAL>(tm, p, ctl, sQ, sStage, sR, b, h, qb, n);
    } else if (warp == kMmaWarp) {
      if (lane == 0) mma_role<DPAD, BN, CAL>(p, ctl, sQ, sStage, tmem, n);
    } else {
      softmax_role<DPAD, BN, CAL>(tm, p, ctl, sQ, sStage, sR, tmem, b, h, qb, n);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace rtb
