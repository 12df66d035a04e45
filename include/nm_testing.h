/*
 * nm_testing.h -- test and tuning hooks of libnm (sm_100a).
 *
 * Not part of the product interface in nm.h: these calls exist so that tests
 * can force a code path the library would not pick for a given shape, and
 * drive the failure path of the product kernel's bounded waits without
 * faulting the GPU.  Like every libnm call they are asynchronous on
 * `stream`, allocate nothing, and report argument errors in the returned
 * status.  (No counterpart on the pages.)
 */
#ifndef NM_TESTING_H
#define NM_TESTING_H

#include "nm.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Values of nm_spmm_test's `kernel` argument. */
enum {
    NM_SPMM_KERNEL_DEFAULT = 0,    /* the choice nm_spmm makes for the shape     */
    NM_SPMM_KERNEL_PAIR256 = 1,    /* CTA pair, 256 x 256 output tiles            */
    NM_SPMM_KERNEL_PAIR192 = 2,    /* CTA pair, 256 x 192                         */
    NM_SPMM_KERNEL_PAIR128 = 3,    /* CTA pair, 256 x 128                         */
    NM_SPMM_KERNEL_SINGLE256 = 4,  /* one CTA, 128 x 256                          */
    NM_SPMM_KERNEL_SINGLE128 = 5,  /* one CTA, 128 x 128                          */
    NM_SPMM_KERNEL_SINGLE64 = 6,   /* one CTA, 128 x 64, one CTA per SM           */
    NM_SPMM_KERNEL_SINGLE64X2 = 7, /* one CTA, 128 x 64, two CTAs per SM          */
    NM_SPMM_KERNEL_SINGLE32X2 = 8, /* one CTA, 128 x 32, two CTAs per SM          */
    NM_SPMM_KERNEL_SINGLE16X2 = 9  /* one CTA, 128 x 16, two CTAs per SM          */
};

/*
 * nm_spmm_test -- nm_spmm (same arguments, same results, same errors) with
 * four hooks:
 *   kernel         NM_SPMM_KERNEL_*; a CTA-pair kernel asked for on an odd
 *                  number of 128-row tiles falls back to the default choice;
 *                  for int8 operands the 192- and 128-column pair kernels
 *                  become the 256-column one, and for int8 and tf32 operands
 *                  the 16-column kernel the 32-column one.
 *                  Every tile configuration computes the same sums in the same
 *                  order per output, so results do not depend on it.
 *   tail_split     1: a last wave that fills at most half of the CTA pairs is
 *                  run as half-width items (nm_spmm's behaviour); 0: not.
 *   wait_limit_ns  limit of every bounded device-side wait, in nanoseconds
 *                  (0: the library's 2 s).
 *   skip_step      -1: none.  Otherwise the producer of every CTA issues no
 *                  copy and arms no barrier for its pipeline step number
 *                  skip_step (steps count 128-column K slices across the
 *                  CTA's tiles, from 0), so the consumer's wait on that stage
 *                  runs out: the kernel records NM_ERR_TIMEOUT in the device
 *                  status word (read with nm_last_device_status), stops its
 *                  other roles, lets the copies it issued land, frees its
 *                  tensor memory and returns.  Y is then undefined.  Every
 *                  later call runs normally.
 *   raster_group, raster_m_inner
 *                  0, 0: the library's tile order.  raster_group > 0: tiles
 *                  run in groups of raster_group tiles of the operand named
 *                  by raster_m_inner (1: row tiles of W, swept fastest across
 *                  every column tile of X; 0: column tiles of X, swept across
 *                  every row tile), for tuning the order against the L2.
 *                  Results do not depend on it.
 * Errors: as nm_spmm, plus NM_ERR_SHAPE for kernel outside 0..9, a negative
 * wait_limit_ns, skip_step < -1, a negative raster_group or raster_m_inner
 * outside 0..1.
 */
NM_API nm_status nm_spmm_test(const void *values, const uint8_t *meta_sm100, nm_dtype ab_dtype,
                              const void *X, int64_t ldx, void *Y, nm_dtype y_dtype, int64_t ldy,
                              int64_t R, int64_t K, int64_t T, float alpha, float beta,
                              void *workspace, size_t workspace_bytes,
                              int kernel, int tail_split, int64_t wait_limit_ns, int64_t skip_step,
                              int raster_group, int raster_m_inner, void *stream);

/*
 * nm_spmm12_test -- nm_spmm12 with a forced tile configuration (`kernel`, as
 * above) and the half-width last wave on (1) or off (0).
 */
NM_API nm_status nm_spmm12_test(const float *values, const uint8_t *meta12_sm100, const float *X, int64_t ldx,
                                void *Y, nm_dtype y_dtype, int64_t ldy, int64_t R, int64_t K, int64_t T,
                                float alpha, float beta, int kernel, int tail_split, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* NM_TESTING_H */
