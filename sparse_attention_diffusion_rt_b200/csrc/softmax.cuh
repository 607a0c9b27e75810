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

// As exp_pack_store, and also returns in xmax the largest x = s_c * sl2 - m of
// the row block, so that a running max that is too small (x above the lazy
// rescale threshold) is detected without a separate max pass: the max is taken
// on the ALU pipe while the MUFU computes the exponentials.
template <int BN>
__device__ __forceinline__ float exp_pack_store_mx(const uint32_t (&s)[BN], float sl2, float m, uint32_t tP,
                                                   float& xmax) {
  uint64_t sum[4];
  float mx[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    sum[i] = 0ull;
    mx[i] = -INFINITY;
  }
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
      mx[c & 3] = max3f(mx[c & 3], x0, x1);
      const float p0 = ex2_approx(x0);
      const float p1 = ex2_approx(x1);
      sum[c & 3] = fadd2(sum[c & 3], f2_pack(p0, p1));
      pk[c] = pack_bf16x2(p0, p1);
    }
    tmem_st_x32(tP + c0 / 2, pk);
  }
  xmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
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
#pragma unroll
  for (int c = 0; c < BN; c += 32) tmem_ld_x32(tS + c, *reinterpret_cast<uint32_t(*)[32]>(&s[c]));
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

// Two-pass variants that keep at most 64 logits in registers: the row max is
// taken over S read from TMEM in two halves, then S is read again, half by half,
// exponentiated and written back as bf16 P into the first BN/2 columns of the
// same TMEM region (column 16c of P overwrites logits that were already read),
// so that P needs no TMEM of its own.  Keys c >= valid are excluded.
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

// As exp_pass_tmem but P goes to its own TMEM columns tP; on_s_read() runs once
// the last logits have been read (S may then be overwritten by the next QK^T),
// before_p() runs before the first P store (P's previous contents must have been
// consumed).
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

template <int BN>
__device__ __forceinline__ float exp_pass_tmem(uint32_t tS, float sl2, float m, int valid) {
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
    tmem_st_x32(tS + h0 / 2, pk);      // P columns [h0/2, h0/2 + 32): logits already consumed
  }
  const uint64_t t = fadd2(fadd2(sum[0], sum[1]), fadd2(sum[2], sum[3]));
  float lo, hi;
  f2_unpack(t, lo, hi);
  return lo + hi;
}

}  // namespace rtb
