/*
 * rt.h -- C ABI of the B200 (sm_100a) implementation of Re-ttention's
 * statistically reshaped static block-sparse attention.
 *
 * Source of the operations: "Re-ttention: Ultra Sparse Visual Generation via
 * Attention Statistical Reshape" -- the summary page ("Approach") and the
 * OpenReview discussion (replies to W1 of the three reviewers: the worked
 * 4-key example, rho as the ratio of sparse to full softmax denominator, the
 * residual of the masked tokens; reply to Q2: rho per head and per token;
 * reply to Q4: the residual has the attention output's shape; reply to W2:
 * static masks; reply to Pwod's W1: the ramp-up lambda).
 *
 * Notation, per batch b and head h, query row i, key j:
 *   s_ij = c <q_i, k_j>, c = softmax_scale (0 selects 1/sqrt(d), true d)
 *   M(i) = keys in the key blocks kept for i's query block; V(i) = keys j < L.
 *
 * Common conventions
 *   - Every buffer is caller-owned device memory, except where a name starts
 *     with h_ (host).  The library allocates nothing but one device status
 *     word per device (a static __device__ variable).
 *   - Q, K, V, O and R share one layout: element (b, h, l, t) is at
 *     b*stride_b + h*stride_h + l*stride_l + t (elements; t contiguous).
 *     Q, K, V and O are bf16; R is bf16 or fp32 (rt_attn_desc.r_dtype).
 *     rho is fp32 [B, H, L] contiguous.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) unless stated otherwise.  They are stateless and
 *     reentrant.  There is no CPU fallback.
 *   - Host-side validation failures return a status and launch nothing.
 *     Faults found on the device (a bad block index, a wait that ran past its
 *     limit) never trap: the kernel records the first status in the device
 *     status word, skips the affected work and returns; read it with
 *     rt_check_device_error.
 *   - Supported: 16 <= d <= 128 with d % 8 == 0 (d is padded to 64, 80, 96 or
 *     128 inside the kernels), block in {64, 128}, strides multiples of 8
 *     elements, pointers 16-byte aligned, 1 <= L and ceil(L/block) <= 4096.
 *     Other shapes return RT_ERR_UNSUPPORTED.
 *   - The strides must give every (b, h, l) row its own d elements (any
 *     permuted dense layout, e.g. [B,H,L,d] or [B,L,H,d], or a slice of one);
 *     a layout whose heads or batches alias returns RT_ERR_INVALID_ARGUMENT,
 *     and so does a call whose outputs (O; rho and R where the call writes
 *     them) overlap one of its inputs or each other.
 */
#ifndef RT_B200_H
#define RT_B200_H

#include <stdint.h>

#if defined(__GNUC__)
#define RT_API __attribute__((visibility("default")))
#else
#define RT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum rt_status {
  RT_OK = 0,
  RT_ERR_INVALID_ARGUMENT = 1, /* null/misaligned pointer, negative size, inconsistent index */
  RT_ERR_UNSUPPORTED = 2,      /* valid but outside the supported shapes above */
  RT_ERR_CAPACITY = 3,         /* output array too small (rt_build_block_index) */
  RT_ERR_CUDA = 4,             /* a CUDA runtime/driver call failed; see rt_last_cuda_error */
  RT_ERR_TIMEOUT = 5,          /* device: an mbarrier wait ran past its limit */
  RT_ERR_BAD_INDEX = 6         /* device: row_ptr/col_idx out of range or not ascending */
} rt_status;

/* Ramp-up of the cached rho with the step distance k since calibration
 * (reply to Pwod's W1: rho grows over denoising, lambda = 0.04 best).  The
 * pages give no formula; all three equal rho at lambda = 0 or k = 0 and clamp
 * at 1.  MUL_LINEAR is the default reading. */
typedef enum rt_ramp {
  RT_RAMP_MUL_LINEAR = 0, /* min(1, rho * (1 + lambda k)) */
  RT_RAMP_ADD_LINEAR = 1, /* min(1, rho + lambda k)       */
  RT_RAMP_GEOMETRIC = 2   /* min(1, rho * (1 + lambda)^k) */
} rt_ramp;

typedef enum rt_dtype { RT_BF16 = 0, RT_F32 = 1 } rt_dtype;

/* What the calibration stores as the residual R (rt_calibrate_ex).
 *   RT_RES_MASKED       Re-ttention's residual: the masked tokens' part of
 *                       the full output, R_i = sum_{V(i)\M(i)} e^{s_ij-m_i} v_j / Z_full.
 *   RT_RES_SUBTRACTIVE  DiTFastAttn's residual, the contrast the replies to W1
 *                       work through: R_i = O_i - O_sparse_i with O_sparse_i the
 *                       softmax over M(i) alone (0 when M(i) is empty). */
typedef enum rt_residual { RT_RES_MASKED = 0, RT_RES_SUBTRACTIVE = 1 } rt_residual;

/* Epilogue of the sparse step (rt_sparse_step_ex); attn_i is the softmax over
 * M(i) of the step's own inputs (0 when M(i) is empty).
 *   RT_EPI_RESHAPED  O'_i = ramp(rho_i, lambda, k) * attn_i + R_i   (Re-ttention)
 *   RT_EPI_NO_RHO    O'_i = attn_i + R_i      (ablation without the statistical
 *                    reshape; with an RT_RES_SUBTRACTIVE residual it is
 *                    DiTFastAttn's reconstruction).  rho is not read (may be NULL).
 *   RT_EPI_NO_R      O'_i = ramp(rho_i, lambda, k) * attn_i   (ablation without the
 *                    residual).  r is not read (may be NULL). */
typedef enum rt_epilogue { RT_EPI_RESHAPED = 0, RT_EPI_NO_RHO = 1, RT_EPI_NO_R = 2 } rt_epilogue;

typedef struct rt_attn_desc {
  int32_t B, H, L, d;   /* batch, heads, tokens, head dimension */
  int32_t block;        /* query and key block size: 64 or 128 */
  int64_t stride_b, stride_h, stride_l; /* element strides shared by Q, K, V, O, R */
  float softmax_scale;  /* c; 0 selects 1/sqrt(d) */
  rt_dtype r_dtype;     /* residual R element type */
} rt_attn_desc;

/* CSR block index of the static mask (device arrays).  Rows are (hm, qb)
 * flattened hm-major, hm in [0, Hm); Hm == 1 shares one mask across all
 * batches and heads, Hm == H gives each head its own.  Row r lists its kept
 * key blocks col_idx[row_ptr[r] .. row_ptr[r+1]) in strictly ascending order;
 * row_ptr[0] == 0 and row_ptr[Hm*nqb] == nnz. */
typedef struct rt_block_index {
  int32_t Hm, nqb, nkb;   /* nqb == nkb == ceil(L / block) */
  int64_t nnz;
  const int32_t* row_ptr; /* device, Hm*nqb + 1 entries */
  const int32_t* col_idx; /* device, nnz entries (may be NULL when nnz == 0) */
} rt_block_index;

/* Dense block mask -> CSR block index (the static mask is free at inference,
 * reply to W2; the index is built once per mask).
 *   d_mask      device u8 [Hm, nqb, nkb], nonzero = key block kept.
 *   d_row_ptr   device i32 [Hm*nqb + 1], written: exclusive prefix sum of row counts.
 *   d_col_idx   device i32 [col_capacity], written: kept key blocks, ascending per row.
 *   h_nnz       host, receives the total number of kept blocks.
 * Synchronises `stream` once to read nnz.  Returns RT_ERR_CAPACITY (and
 * writes only the rows that fit) when nnz > col_capacity. */
RT_API rt_status rt_build_block_index(const uint8_t* d_mask, int32_t Hm, int32_t nqb, int32_t nkb,
                               int32_t* d_row_ptr, int32_t* d_col_idx, int64_t col_capacity,
                               int64_t* h_nnz, void* stream);

/* Calibration (full-attention) step.  For every (b, h, i):
 *   O_i   = sum_{j in V(i)} e^{s_ij - m_i} v_j / Z_full          (bf16 out)
 *   rho_i = Z_sp / Z_full                                        (fp32 out)
 *   R_i   = sum_{j in V(i) \ M(i)} e^{s_ij - m_i} v_j / Z_full   (r_dtype out)
 * with Z_full = sum_{V(i)} e^{s_ij - m_i}, Z_sp = sum_{M(i)} e^{s_ij - m_i},
 * one shared row max m_i.  One tensor-core pass over all key blocks; the
 * in-mask and out-of-mask sums and outputs are kept apart. */
RT_API rt_status rt_calibrate(const rt_attn_desc* desc, const void* q, const void* k, const void* v,
                       const rt_block_index* idx, void* o, float* rho, void* r, void* stream);

/* Reshaped sparse step at step distance k >= 0 since the calibration:
 *   O'_i = ramp(rho_i, lambda, k) * sum_{j in M(i)} e^{s'_ij - m'_i} v'_j
 *                                   / sum_{j in M(i)} e^{s'_ij - m'_i}  +  R_i
 * and O'_i = R_i when M(i) is empty.  Only the kept key blocks are visited.
 * rho and r are the calibration's outputs (same layouts). */
RT_API rt_status rt_sparse_step(const rt_attn_desc* desc, const void* q, const void* k, const void* v,
                         const rt_block_index* idx, const float* rho, const void* r,
                         float lambda, int32_t step_distance, rt_ramp ramp, void* o, void* stream);

/* rt_calibrate with the residual kind chosen: rt_calibrate(...) is
 * rt_calibrate_ex(..., RT_RES_MASKED, stream).  Same arguments, layouts and
 * errors; an unknown kind returns RT_ERR_INVALID_ARGUMENT. */
RT_API rt_status rt_calibrate_ex(const rt_attn_desc* desc, const void* q, const void* k, const void* v,
                          const rt_block_index* idx, void* o, float* rho, void* r, rt_residual kind,
                          void* stream);

/* rt_sparse_step with the epilogue chosen: rt_sparse_step(...) is
 * rt_sparse_step_ex(..., RT_EPI_RESHAPED, o, stream).  rho may be NULL with
 * RT_EPI_NO_RHO and r may be NULL with RT_EPI_NO_R (they are not read);
 * otherwise as rt_sparse_step.  An unknown epilogue returns
 * RT_ERR_INVALID_ARGUMENT. */
RT_API rt_status rt_sparse_step_ex(const rt_attn_desc* desc, const void* q, const void* k, const void* v,
                            const rt_block_index* idx, const float* rho, const void* r,
                            float lambda, int32_t step_distance, rt_ramp ramp, rt_epilogue epi,
                            void* o, void* stream);

/* Denoising schedule: the pages calibrate (one full-attention step that
 * refreshes the cached rho and R) every few denoising steps and run reshaped
 * sparse steps in between, with the ramp-up growing with the distance to the
 * calibration.  Step t = 0, 1, 2, ... of a schedule is a calibration when
 * t % period == 0 and otherwise a sparse step at step distance
 * k = t % period.  epilogue / residual select the method: Re-ttention is
 * RT_EPI_RESHAPED + RT_RES_MASKED; DiTFastAttn's residual caching is
 * RT_EPI_NO_RHO + RT_RES_SUBTRACTIVE. */
typedef struct rt_schedule {
  int32_t period;         /* calibration period T >= 1 */
  float lambda;           /* ramp-up lambda of the sparse steps */
  rt_ramp ramp;
  rt_epilogue epilogue;
  rt_residual residual;
} rt_schedule;

/* Step t of the schedule on this step's q, k, v: rt_calibrate_ex into o, rho
 * and r at a calibration step, else rt_sparse_step_ex reading rho and r (the
 * caller's cache, written by the last calibration step) into o.  Errors as
 * those calls; t < 0, a NULL schedule or period < 1 return
 * RT_ERR_INVALID_ARGUMENT. */
RT_API rt_status rt_schedule_step(const rt_attn_desc* desc, const rt_schedule* sched, int32_t t,
                           const void* q, const void* k, const void* v, const rt_block_index* idx,
                           void* o, float* rho, void* r, void* stream);

/* One whole calibration cycle (steps 0 .. period-1) captured as a CUDA graph,
 * so that a cycle costs one launch.  q[t], k[t], v[t] and o[t] (arrays of
 * `period` device pointers) are step t's buffers; rho and r the cache.  The
 * graph reads and writes exactly those buffers every time it is launched.
 * `stream` must be a created stream (capture is not possible on the legacy
 * default stream: RT_ERR_INVALID_ARGUMENT).  Nothing is launched while
 * capturing.  On success *graph receives a handle that the caller owns and
 * releases with rt_cycle_graph_destroy. */
typedef struct rt_cycle_graph rt_cycle_graph;
RT_API rt_status rt_schedule_capture(const rt_attn_desc* desc, const rt_schedule* sched,
                              const void* const* q, const void* const* k, const void* const* v,
                              const rt_block_index* idx, void* const* o, float* rho, void* r,
                              void* stream, rt_cycle_graph** graph);

/* Launch a captured cycle on `stream` (asynchronous). */
RT_API rt_status rt_cycle_graph_launch(rt_cycle_graph* graph, void* stream);

/* Release a captured cycle (NULL is a no-op). */
RT_API rt_status rt_cycle_graph_destroy(rt_cycle_graph* graph);

/* Token order that makes the blocks of the static mask compact (the pages
 * lay video tokens out along a space-filling curve before blocking them).
 * Tokens in raster order are n_text text tokens, then an F x Y x X latent
 * grid with x fastest.  h_perm (host, n_text + F*Y*X entries) receives, for
 * each position i of the new order, the raster index of the token placed
 * there: the text tokens stay first, and the grid follows the Hilbert curve
 * (over the axes longer than 1) of the smallest enclosing cube of side 2^b,
 * restricted to the grid.
 * 128 consecutive tokens then fill a compact brick instead of a row strip.
 * Attention and every per-token operation commute with a fixed permutation,
 * so a model applies it once where tokens are formed (rt_permute_tokens) and
 * builds the block mask on the reordered tokens. */
RT_API rt_status rt_hilbert_token_order(int32_t n_text, int32_t F, int32_t Y, int32_t X, int32_t* h_perm);

/* Reorder the token rows of a bf16 [B, H, L, d] tensor (layout and strides of
 * `desc`; B, H, L, d and the strides are used, the rest ignored):
 *   inverse = 0: dst[b, h, i, :] = src[b, h, perm[i], :]   (raster -> new order)
 *   inverse = 1: dst[b, h, perm[i], :] = src[b, h, i, :]   (back to raster order)
 * d_perm: device i32 [L], a permutation of 0..L-1 (a bijection).  An entry
 * outside [0, L) records RT_ERR_BAD_INDEX in the device status word and its
 * row is skipped; a repeated entry is not detected (the gather copies that row
 * twice; the scatter, inverse = 1, writes one dst row twice and leaves another
 * unwritten).  src and dst must not overlap and the layout's rows must be
 * disjoint (RT_ERR_INVALID_ARGUMENT otherwise).  d % 8 == 0, 16-byte aligned
 * pointers and strides that are multiples of 8 elements.  Asynchronous on
 * `stream`. */
RT_API rt_status rt_permute_tokens(const rt_attn_desc* desc, const void* src, void* dst, const int32_t* d_perm,
                            int32_t inverse, void* stream);

/* Synchronises `stream`, returns the first device-side status recorded since
 * the last call on the current device, and clears it. */
RT_API rt_status rt_check_device_error(void* stream);

/* Static string for a status code (never NULL). */
RT_API const char* rt_status_string(rt_status s);

/* Text of the last CUDA error seen by this library on this thread ("" if none). */
RT_API const char* rt_last_cuda_error(void);

/* Upper bound, in nanoseconds, on every mbarrier wait inside the kernels
 * (default 4e9).  A wait that exceeds it records RT_ERR_TIMEOUT and the CTA
 * drains its own in-flight copies and MMAs, frees its TMEM and returns.
 * Process-wide; applies to launches made after the call.  0 restores the default. */
RT_API rt_status rt_set_wait_limit_ns(uint64_t limit_ns);

/* Test hook for the bounded-wait path: launches one CTA that waits on an
 * mbarrier no one arrives on, for at most limit_ns, then records
 * RT_ERR_TIMEOUT.  Never faults or hangs. */
RT_API rt_status rt_debug_wait_timeout(uint64_t limit_ns, void* stream);

/* Compute capability the library was built for (1000 = sm_100a). */
RT_API int32_t rt_build_arch(void);

#ifdef __cplusplus
}
#endif

#endif /* RT_B200_H */
