// Row-wise pieces of the online softmax shared by the calibration and sparse
// kernels.  Thread t owns query row t of the tile (TMEM lane t), so row
// reductions are in-thread; they are written as 8 independent chains so that
// one warp per scheduler keeps the FMNMX/FADD pipes and the MUFU busy instead
// of waiting on a serial dependency.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace rtb {

template <int BN>
__device__ __forceinline__ float row_max(const uint32_t (&s)[BN]) {
  float mx[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mx[i] = __uint_as_float(s[i]);
#pragma unroll
  for (int c = 8; c < BN; c += 2)
    mx[(c >> 1) & 7] = max3f(mx[(c >> 1) & 7], __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
  const float a = max3f(mx[0], mx[1], mx[2]);
  const float b = max3f(mx[3], mx[4], mx[5]);
  return max3f(a, b, fmaxf(mx[6], mx[7]));
}

// Set logits of key columns >= valid (keys past the end of the sequence) to -inf.
template <int BN>
__device__ __forceinline__ void mask_tail(uint32_t (&s)[BN], int valid) {
  if (valid < BN) {
#pragma unroll
    for (int c = 0; c < BN; ++c)
      if (c >= valid) s[c] = __float_as_uint(-INFINITY);
  }
}

// p_c = 2^(s_c * sl2 - m) for the whole row block; P is stored as bf16 pairs
// into TMEM columns [tP, tP + BN/2) of this thread's lane.  Returns sum_c p_c
// (of the fp32 values).  The caller waits for the stores (tmem_wait_st).
template <int BN>
__device__ __forceinline__ float exp_pack_store(const uint32_t (&s)[BN], float sl2, float m, uint32_t tP) {
  uint64_t sum[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) sum[i] = 0ull;
  const uint64_t scale2 = f2_pack(sl2, sl2);
  const uint64_t neg_m2 = f2_pack(-m, -m);
#pragma unroll
  for (int c0 = 0; c0 < BN; c0 += 64) {
    uint32_t pk[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const uint64_t x = ffma2(f2_pack(__uint_as_float(s[c0 + 2 * c]), __uint_as_float(s[c0 + 2 * c + 1])),
                               scale2, neg_m2);
      float x0, x1;
      f2_unpack(x, x0, x1);
      const float p0 = ex2_approx(x0);
      const float p1 = ex2_approx(x1);
      sum[c & 3] = fadd2(sum[c & 3], f2_pack(p0, p1));
      pk[c] = pack_bf16x2(p0, p1);
    }
    tmem_st_x32(tP + c0 / 2, pk);
  }
  const uint64_t t = fadd2(fadd2(sum[0], sum[1]), fadd2(sum[2], sum[3]));
  float lo, hi;
  f2_unpack(t, lo, hi);
  return lo + hi;
}

// Largest x = s_c * sl2 - m of the row block.  x is one rounded fma, monotone
// in s_c for sl2 > 0, so this is exactly the largest x the exponentials used.
// (Taken from the raw logits, not from the x values, so that the compiler does
// not keep the block's 128 x values live from the exponentials to this rare
// check.)
template <int BN>
__device__ __forceinline__ float xmax_of(const uint32_t (&s)[BN], float sl2, float m) {
  return fmaf(row_max<BN>(s), sl2, -m);
}

// Load BN fp32 logits of this thread's row from TMEM (caller waits with tmem_wait_ld).
template <int BN>
__device__ __forceinline__ void load_scores(uint32_t tS, uint32_t (&s)[BN]) {
  if constexpr (BN == 128) {
    tmem_ld_x128(tS, s);
  } else {
#pragma unroll
    for (int c = 0; c < BN; c += 32) tmem_ld_x32(tS + c, *reinterpret_cast<uint32_t(*)[32]>(&s[c]));
  }
}

// Rescale one TMEM accumulator row (this thread's lane) by alpha.
template <int DPAD>
__device__ __forceinline__ void rescale_row(uint32_t taddr, float alpha) {
#pragma unroll
  for (int c = 0; c < DPAD; c += 16) {
    uint32_t r[16];
    tmem_ld_x16(taddr + c, r);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
    tmem_st_x16(taddr + c, r);
  }
  tmem_wait_st();
}

}  // namespace rtb

namespace rtb {

// Two-pass form for a softmax that keeps at most 64 logits in registers: the row
// max is taken over S read from TMEM in two halves (row_max_tmem), then S is
// read again, half by half, and exponentiated (exp_pass_tmem_sep).  Keys
// c >= valid are excluded.
template <int BN>
__device__ __forceinline__ float row_max_tmem(uint32_t tS, int valid) {
  float mx[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mx[i] = -INFINITY;
#pragma unroll
  for (int h0 = 0; h0 < BN; h0 += 64) {
    uint32_t s[64];
    tmem_ld_x32(tS + h0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
    tmem_ld_x32(tS + h0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
    tmem_wait_ld();
    if (valid < h0 + 64) {
#pragma unroll
      for (int c = 0; c < 64; ++c)
        if (h0 + c >= valid) s[c] = __float_as_uint(-INFINITY);
    }
#pragma unroll
    for (int c = 0; c < 64; c += 2)
      mx[(c >> 1) & 7] = max3f(mx[(c >> 1) & 7], __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
  }
  const float a = max3f(mx[0], mx[1], mx[2]);
  const float b = max3f(mx[3], mx[4], mx[5]);
  return max3f(a, b, fmaxf(mx[6], mx[7]));
}

// p_c = 2^(s_c * sl2 - m) for a row block whose logits are read from TMEM (tS)
// in halves of 64, keys c >= valid excluded; P goes as bf16 pairs to its own
// TMEM columns tP.  on_s_read() runs once the last logits have been read (S may
// then be overwritten by the next QK^T), before_p() before the first P store
// (P's previous contents must have been consumed).  Returns sum_c p_c.
template <int BN, typename OnSRead, typename BeforeP>
__device__ __forceinline__ float exp_pass_tmem_sep(uint32_t tS, uint32_t tP, float sl2, float m, int valid,
                                                   OnSRead on_s_read, BeforeP before_p) {
  uint64_t sum[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) sum[i] = 0ull;
  const uint64_t scale2 = f2_pack(sl2, sl2);
  const uint64_t neg_m2 = f2_pack(-m, -m);
#pragma unroll
  for (int h0 = 0; h0 < BN; h0 += 64) {
    uint32_t s[64];
    tmem_ld_x32(tS + h0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
    tmem_ld_x32(tS + h0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
    tmem_wait_ld();
    if (h0 + 64 >= BN) on_s_read();
    if (valid < h0 + 64) {
#pragma unroll
      for (int c = 0; c < 64; ++c)
        if (h0 + c >= valid) s[c] = __float_as_uint(-INFINITY);
    }
    uint32_t pk[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const uint64_t x = ffma2(f2_pack(__uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1])), scale2, neg_m2);
      float x0, x1;
      f2_unpack(x, x0, x1);
      const float p0 = ex2_approx(x0);
      const float p1 = ex2_approx(x1);
      sum[c & 3] = fadd2(sum[c & 3], f2_pack(p0, p1));
      pk[c] = pack_bf16x2(p0, p1);
    }
    if (h0 == 0) before_p();
    tmem_st_x32(tP + h0 / 2, pk);
  }
  const uint64_t t = fadd2(fadd2(sum[0], sum[1]), fadd2(sum[2], sum[3]));
  float lo, hi;
  f2_unpack(t, lo, hi);
  return lo + hi;
}

}  // namespace rtb
