/*
 * nm.h -- C ABI of libnm: N:M fine-grained structured sparsity on NVIDIA
 * B200 (sm_100a).  Mask selection, 2:4 compression / decompression, the
 * tensor-core metadata image, the 2:4-sparse x dense product, and that
 * product split by output rows over several GPUs (peer stores, completion
 * flags, IPC mappings).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Matrices are row-major.  Leading dimensions (ld*) count ELEMENTS.
 *  - W is R x C; groups are M consecutive entries of a row, i.e. along the
 *    reduction (K) dimension of the product Y = W X.  (Pages: "SR-STE sparse
 *    training", N:M concept -- N of every M consecutive parameters kept.)
 *  - Every pointer is a DEVICE pointer owned by the caller; the library
 *    allocates no device memory.  Every call is asynchronous on `stream`
 *    (a cudaStream_t passed as void*; NULL = the legacy default stream) and
 *    returns as soon as the work is enqueued.  The returned status reports
 *    argument validation and launch errors only; it never waits for the GPU.
 *  - Device pointers and leading-dimension strides (ld * element size) must
 *    be 16-byte aligned, else NM_ERR_ALIGN.  Packed arrays (values, meta)
 *    have no stride argument.  Sizes must be >= 0; R == 0 or C == 0 (or
 *    T == 0) is a no-op returning NM_OK.
 *  - Magnitude order: the IEEE bit pattern with the sign bit cleared, read as
 *    an unsigned integer (so -0 == +0, subnormals < normals < Inf < NaN).
 *    Ties: the lower in-group index wins.  Both are this library's readings;
 *    the pages leave them open.
 *
 * Canonical compressed 2:4 layout ("Accelerating Sparse Deep Neural
 * Networks" review, "Benefits of 2:4 sparsity": R*C/2 values plus a 2-bit
 * in-group index per value; groups with more zeros still store 2 values):
 *    values[r][2g+j] = W[r][4g+idx_j], idx_0 < idx_1   (R x C/2, W's dtype,
 *                      bits copied exactly, row stride C/2 elements)
 *    meta[r][k/4]    bits 2*(k%4)..+1 = idx of kept entry k = 2g+j
 *                      (R x C/8 bytes, row stride C/8)
 *
 * Tensor-core metadata image ("meta_sm100"): the layout the sm_100
 * .kind::f16 sparse MMA reads from tensor memory (PTX ISA, tcgen05 sparse
 * matrices).  Per block of 128 rows x 128 logical columns, 2048 bytes:
 * 16 bytes per tensor-memory lane L, 4 bytes per 32-column slice s; lane
 * L = r%8 + 8*((c%32)/16) + 16*((r%128)/16), bit 16*((r%16)/8) +
 * 4*((c%16)/4) of slice (c%128)/32 holds the group's idx_0 | idx_1 << 2.
 * Blocks are stored row-tile major: block (rt, kt) at byte
 * (rt*ceil(C/128) + kt) * 2048.  R and C are padded up to multiples of 128;
 * padded groups hold the pattern (0,1).  Size: nm_sizes().
 */
#ifndef NM_H
#define NM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NM_API __attribute__((visibility("default")))
#else
#define NM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NM_OK = 0,
    NM_ERR_NULL = 1,         /* a required pointer is NULL                      */
    NM_ERR_SHAPE = 2,        /* bad R / C / K / T / ld (e.g. C % M != 0)        */
    NM_ERR_ALIGN = 3,        /* pointer or row stride not 16-byte aligned       */
    NM_ERR_DTYPE = 4,        /* dtype not supported by this call                */
    NM_ERR_NM = 5,           /* N, M outside 1 <= N < M <= 8                     */
    NM_ERR_UNSUPPORTED = 6,  /* valid request the library does not implement   */
    NM_ERR_CUDA = 7,         /* a CUDA runtime / driver call failed             */
    NM_ERR_WORKSPACE = 8,    /* workspace NULL or smaller than required         */
    NM_ERR_TIMEOUT = 9       /* a bounded device-side wait gave up (see below)  */
} nm_status;

/* NM_S8: two's-complement int8 weights, magnitude |x| (so -128 ranks above 127).
 * Accepted by nm_sizes, nm_mask, nm_mask_transposable, nm_mask_compress,
 * nm_compress, nm_decompress, nm_meta_to_sm100_s8 and nm_spmm (the int8 2:4
 * product); the floating-point calls (nm_mask_scored, nm_srste_step, the 1:2
 * calls) return NM_ERR_DTYPE.
 * NM_S32: two's-complement int32, only as the output of the int8 product. */
typedef enum { NM_F32 = 0, NM_BF16 = 1, NM_F16 = 2, NM_S8 = 3, NM_S32 = 4 } nm_dtype;

/* Human-readable text for a status code (static string, never NULL). */
NM_API const char *nm_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
NM_API int nm_version(void);

/*
 * nm_sizes -- bytes of the compressed forms of an R x C matrix.
 *   values_bytes     = R * C * N / M * sizeof(dtype)
 *   meta_bytes       = R * C * N / M * 2 bits / 8  (2:4 only; 0 otherwise)
 *   meta_sm100_bytes = ceil(R/128)*128 * ceil(C/128)*128 / 8 (2:4 only)
 * Any output pointer may be NULL.  Errors: NM_ERR_NM, NM_ERR_SHAPE,
 * NM_ERR_DTYPE.  Source: "Benefits of 2:4 sparsity" (R*C/2 values and
 * R*C/2 2-bit metadata entries).
 */
NM_API nm_status nm_sizes(int64_t R, int64_t C, int N, int M, nm_dtype dtype,
                   size_t *values_bytes, size_t *meta_bytes, size_t *meta_sm100_bytes);

/*
 * nm_mask -- N:M magnitude mask.  For every group of M consecutive entries
 * of each row of W, mask = 1 at the N entries of largest |w| (ties -> lower
 * index), 0 elsewhere.  Sources: "SR-STE sparse training", SR-STE forward
 * (argsort of |w| per group, M-N smallest zeroed) and the Apex exhaustive
 * search (largest kept L1 sum), which select the same entries; review of
 * "Accelerating Sparse Deep Neural Networks", Step-2 (drop the 2 smallest of 4).
 *   W     R x C, dtype NM_F32 / NM_BF16 / NM_F16, leading dim ldw >= C
 *   mask  R x C uint8 (0 or 1), leading dim ldm >= C
 *   1 <= N < M <= 8, C % M == 0 (else NM_ERR_NM / NM_ERR_SHAPE)
 */
NM_API nm_status nm_mask(const void *W, nm_dtype dtype, int64_t R, int64_t C, int64_t ldw,
                  int N, int M, uint8_t *mask, int64_t ldm, void *stream);

/*
 * nm_mask_scored -- saliency-scored N:M mask.  Source: "sparsegpt.py"
 * (fasterprune, semi-structured branch): inside every group of M
 * consecutive columns the score of w is w^2 / d^2, with d the entry of its
 * column in the diagonal of the upper Cholesky factor of the damped inverse
 * Hessian, and the M-N smallest scores are pruned.  Here d is any
 * caller-supplied vector and the score is evaluated in binary32 as in that
 * listing, s = fl(fl(w*w) / fl(d[c]*d[c])), each operation rounded once to
 * nearest even.  mask = 1 at the N largest scores of each group, ranked by
 * the bit pattern of s with the sign cleared (0/0 gives NaN, which ranks
 * highest); equal scores keep the lower in-group index.  The weight update
 * of that listing is not part of this call.
 *   W     R x C, dtype NM_F32 / NM_BF16 / NM_F16, leading dim ldw >= C
 *   d     C floats (device), 16-byte aligned
 *   mask  R x C uint8 (0 or 1), leading dim ldm >= C
 *   1 <= N < M <= 8, C % M == 0 (else NM_ERR_NM / NM_ERR_SHAPE);
 *   NM_ERR_NULL for a null W, d or mask, NM_ERR_ALIGN as nm_mask or for d
 */
NM_API nm_status nm_mask_scored(const void *W, nm_dtype dtype, const float *d, int64_t R, int64_t C,
                         int64_t ldw, int N, int M, uint8_t *mask, int64_t ldm, void *stream);

/*
 * nm_mask_transposable -- transposable N:M mask, greedy.  Source: nubint.ai
 * review of "Accelerated Sparse Neural Training: A Provable and Efficient
 * Method to Find N:M Transposable Masks": in every M x M block keep as much
 * |w| as possible with at most N kept entries per row and per column (W and
 * W^T both N:M), found there by min-cost flow or by a fast greedy
 * 2-approximation.  This is the greedy: inside each block, entries in order
 * of decreasing magnitude (the nm_mask order; equal magnitudes by row-major
 * position within the block); an entry is kept when its row and its column
 * each hold fewer than N kept entries.  Rows or columns can end with fewer
 * than N kept entries; the kept |w| is at least half of the optimum.
 *   W     R x C, dtype NM_F32 / NM_BF16 / NM_F16, leading dim ldw >= C
 *   mask  R x C uint8 (0 or 1), leading dim ldm >= C
 *   1 <= N < M <= 8 (else NM_ERR_NM); R % M == 0 and C % M == 0 (else
 *   NM_ERR_SHAPE); alignment as nm_mask
 */
NM_API nm_status nm_mask_transposable(const void *W, nm_dtype dtype, int64_t R, int64_t C, int64_t ldw,
                               int N, int M, uint8_t *mask, int64_t ldm, void *stream);

/*
 * nm_mask_compress -- fused 2:4 mask + compression in one pass over W:
 * the 2:4 mask of nm_mask, then the kept values and their indices in the
 * canonical layout and (if meta_sm100 != NULL) in the tensor-core image.
 *   W          R x C (ldw >= C), C % 8 == 0
 *   values     R x C/2, W's dtype, packed
 *   meta       R x C/8 bytes, packed (canonical)
 *   meta_sm100 nm_sizes(...)->meta_sm100_bytes bytes, or NULL
 */
NM_API nm_status nm_mask_compress(const void *W, nm_dtype dtype, int64_t R, int64_t C, int64_t ldw,
                           void *values, uint8_t *meta, uint8_t *meta_sm100, void *stream);

/*
 * 1:2 compression (one value of every pair kept).  Source: review of
 * "Accelerating Sparse Deep Neural Networks", "Structured sparse GEMM on
 * tensor cores": sparse TF32 supports only the 1:2 pattern.  Layout (this
 * library's choice): values R x C/2 of W's dtype, values[r][p] = the kept
 * element of pair p (columns 2p, 2p+1), bits copied as stored; meta R x C/16
 * bytes, the kept index of pair p in bit p%8 of byte r*(C/16) + p/8 (LSB
 * first).  C % 16 == 0 (else NM_ERR_SHAPE); pointers and row strides of W,
 * values and mask 16-byte aligned (else NM_ERR_ALIGN).
 *
 * nm_mask_compress12 -- keep the larger magnitude of each pair (the nm_mask
 *   order with N = 1, M = 2: ties keep the first).
 * nm_compress12 -- keep what the uint8 mask (R x C, leading dim ldm) marks.
 *   A pair whose two mask bytes are not exactly one 1 and one 0 is counted
 *   into *invalid_pairs (device int32, added to atomically; NULL to skip) and
 *   stores its first element with index 0.
 * nm_decompress12 -- W_out (R x C, leading dim ldw): the kept element of each
 *   pair at its index, +0.0 at the other.
 */
NM_API nm_status nm_mask_compress12(const void *W, nm_dtype dtype, int64_t R, int64_t C, int64_t ldw,
                             void *values, uint8_t *meta, void *stream);
NM_API nm_status nm_compress12(const void *W, const uint8_t *mask, nm_dtype dtype, int64_t R, int64_t C,
                        int64_t ldw, int64_t ldm, void *values, uint8_t *meta, int32_t *invalid_pairs,
                        void *stream);
NM_API nm_status nm_decompress12(const void *values, const uint8_t *meta, nm_dtype dtype, int64_t R, int64_t C,
                          void *W_out, int64_t ldw, void *stream);

/*
 * nm_compress -- 2:4 compression under a caller-supplied mask (uint8, R x C,
 * leading dim ldm).  A valid group holds 0/1 bytes with at most two ones.
 * A group with fewer than two ("Benefits of 2:4 sparsity": a group with more
 * zeros still stores two values) is stored as its kept positions plus the
 * lowest unkept ones, in ascending order, the unkept ones with value +0.0;
 * so 1:4 masks and greedy transposable masks compress too, and decompression
 * gives W where kept and +0.0 elsewhere.  Invalid groups (more than two ones,
 * or a byte other than 0/1) are counted into *invalid_groups (a device
 * int32, added to atomically; pass NULL to skip); their output is the
 * pattern (0,1) with values W[4g], W[4g+1].  Outputs as nm_mask_compress.
 */
NM_API nm_status nm_compress(const void *W, const uint8_t *mask, nm_dtype dtype, int64_t R, int64_t C,
                      int64_t ldw, int64_t ldm, void *values, uint8_t *meta, uint8_t *meta_sm100,
                      int32_t *invalid_groups, void *stream);

/*
 * nm_compress_t -- 2:4 compression of the TRANSPOSE of W under the transpose
 * of a caller-supplied mask ("Accelerated Sparse Neural Training" review,
 * transposable N:M masks: with a mask that is 2:4 along both rows and columns
 * of W, W^T is itself 2:4-sparse along R, so the backward product
 * dX = W^T dY runs on the same sparse tensor cores as Y = W X).
 *   W, mask: R x C (leading dims ldw, ldm), R % 8 == 0, any C
 *   Output: the canonical form of Wt = W^T (C x R) with groups of four
 *   consecutive rows of a column of W:
 *     values_t  C x R/2, W's dtype, row stride R/2
 *     meta_t    C x R/8 bytes
 *     meta_t_sm100  image of the C x R matrix (nm_sizes(C, R, ...)), or NULL
 *   Groups are kept, filled and checked as by nm_compress (at most two ones
 *   among four 0/1 bytes; fewer are filled with +0.0 values at the lowest
 *   unkept positions; invalid groups are counted and stored as (0,1)).
 *   dtype: NM_F32, NM_BF16, NM_F16 or NM_S8.  One pass over W and the mask.
 *   Errors: NM_ERR_DTYPE for another dtype; NM_ERR_SHAPE if R % 8 != 0 or
 *   ldw, ldm < C; NM_ERR_NULL for a NULL W, mask, values_t or meta_t;
 *   NM_ERR_ALIGN unless W, mask, values_t, meta_t (and meta_t_sm100 when
 *   given) are 16-byte aligned, ldw * element size and ldm are multiples of
 *   16 bytes, and invalid_groups is 4-byte aligned.  R == 0 or C == 0 does
 *   nothing and returns NM_OK.
 */
NM_API nm_status nm_compress_t(const void *W, const uint8_t *mask, nm_dtype dtype, int64_t R, int64_t C,
                               int64_t ldw, int64_t ldm, void *values_t, uint8_t *meta_t,
                               uint8_t *meta_t_sm100, int32_t *invalid_groups, void *stream);

/*
 * nm_decompress -- dense R x C from the canonical 2:4 form: kept positions
 * get their values (bits copied), every other position gets +0.0.
 *   W_out R x C, leading dim ldw >= C, C % 8 == 0
 */
NM_API nm_status nm_decompress(const void *values, const uint8_t *meta, nm_dtype dtype, int64_t R,
                        int64_t C, void *W_out, int64_t ldw, void *stream);

/*
 * nm_meta_to_sm100 -- canonical metadata (R x C/8 bytes) -> tensor-core
 * metadata image (layout above).  C % 8 == 0.
 */
NM_API nm_status nm_meta_to_sm100(const uint8_t *meta, int64_t R, int64_t C, uint8_t *meta_sm100,
                           void *stream);

/*
 * nm_meta_to_sm100_s8 -- canonical 2:4 metadata of an int8 matrix (R x C/8
 * bytes) -> the tensor-core metadata image the int8 product reads
 * (.kind::i8; PTX ISA, tcgen05 sparse matrices: an int8 instruction covers 64
 * logical columns and reads their 16 group fields from two 32-bit columns of
 * the row's own lane, in the canonical order).  Layout: per block of 128 rows
 * x 128 logical columns, 2048 bytes, lane L = r%128 holding the 16 canonical
 * bytes of row r for those columns; blocks row-tile major, block (rt, kt) at
 * byte (rt*nk + kt)*2048 with nk = 2*ceil(C/256); padding rows and columns
 * hold the pattern (0,1), byte 0x44.  Size: nm_meta_s8_image_bytes(R, C)
 * = ceil(R/128)*128 * ceil(C/256)*256 / 8.  C % 8 == 0 (else NM_ERR_SHAPE);
 * meta_s8_sm100 16-byte aligned (else NM_ERR_ALIGN).
 */
NM_API size_t nm_meta_s8_image_bytes(int64_t R, int64_t C);
NM_API nm_status nm_meta_to_sm100_s8(const uint8_t *meta, int64_t R, int64_t C, uint8_t *meta_s8_sm100,
                                     void *stream);

/*
 * nm_meta12_to_sm100 -- canonical 1:2 metadata (R x C/16 bytes, from
 * nm_mask_compress12 / nm_compress12) -> the tensor-core metadata image the
 * TF32 1:2 product reads (.kind::tf32; PTX ISA, tcgen05 sparse matrices: the
 * .kind::f16 layout of the row seen as 16-bit halves, pair p being the group
 * of halves 4p..4p+3 with field 0x4 when element 0 is kept and 0xE when
 * element 1 is).  Layout: per block of 128 rows x 64 fp32 columns, 2048
 * bytes; lane L = r%8 + 8*((h%32)/16) + 16*((r%128)/16), bit
 * 16*((r%16)/8) + 4*((h%16)/4) of the 32-bit slice (h%128)/32, h = 4p; blocks
 * row-tile major, (rt, kt) at byte (rt*ceil(C/64) + kt)*2048; padding pairs
 * hold 0x4.  Size: nm_meta12_image_bytes(R, C) = ceil(R/128)*ceil(C/64)*2048.
 * C % 16 == 0 (else NM_ERR_SHAPE); meta12_sm100 16-byte aligned.
 */
NM_API size_t nm_meta12_image_bytes(int64_t R, int64_t C);
NM_API nm_status nm_meta12_to_sm100(const uint8_t *meta, int64_t R, int64_t C, uint8_t *meta12_sm100,
                                    void *stream);

/*
 * nm_srste_step -- one SR-STE training step, fused ("SR-STE sparse training",
 * SR-STE forward and backward): the N:M magnitude mask of W is recomputed
 * (same rule as nm_mask), and
 *   W_sparse = W * mask                                   (forward)
 *   grad_out = grad + decay * (1 - mask) * W              (backward)
 * evaluated as PyTorch evaluates the page's listing, whose mask is float32:
 * each product and the sum is a binary32 operation rounded on its own (no
 * fused multiply-add), and the results are returned in dtype (one more
 * rounding to nearest even for 16-bit types).  So kept entries return
 * grad + (+-0) -- grad itself, except that grad = -0 with W >= +0 gives +0 --
 * and pruned negative weights give -0 in W_sparse.  Inf and NaN inputs are
 * outside the contract.  The page's default decay is 0.0002.
 *   W, grad, W_sparse, grad_out: R x C, dtype, common leading dim ld >= C
 *   mask: R x C uint8 with row stride ld, or NULL
 *   1 <= N < M <= 8, C % M == 0
 */
NM_API nm_status nm_srste_step(const void *W, const void *grad, nm_dtype dtype, int64_t R, int64_t C,
                               int64_t ld, int N, int M, float decay, void *W_sparse, void *grad_out,
                               uint8_t *mask, void *stream);

/*
 * nm_spmm_workspace_bytes -- device scratch nm_spmm needs for this problem
 * (0 when none is needed).  NM_F32 inputs are rounded to binary16 (nearest
 * even) in the workspace before the product.
 */
NM_API size_t nm_spmm_workspace_bytes(nm_dtype ab_dtype, int64_t R, int64_t K, int64_t T);

/*
 * nm_spmm -- Y = alpha * (W (.) mask) X + beta * Y with fp32 accumulation,
 * W given in compressed 2:4 form.  Review of "Accelerating Sparse Deep
 * Neural Networks", "Structured sparse GEMM on tensor cores": sparse x dense
 * = dense; the application supplies the first operand compressed.
 *   values     R x K/2, ab_dtype (packed, row stride K/2)
 *   meta_sm100 tensor-core metadata image of W (nm_mask_compress /
 *              nm_meta_to_sm100), R and K padded to 128
 *   X          K x T, ab_dtype, leading dim ldx >= T
 *   Y          R x T, y_dtype (NM_BF16 or NM_F32), leading dim ldy >= T;
 *              read only when beta != 0.  Y needs only element alignment;
 *              16-byte aligned Y and ldy get vector stores.  Nothing outside
 *              the R x T block is written (elements between T and ldy
 *              included)
 *   X, values, meta_sm100: 16-byte aligned; ldx * element size % 16 == 0
 *   ab_dtype   NM_BF16 or NM_F16 (tensor-core path), NM_S8 (the int8 2:4
 *              tensor-core path, below), or NM_F32 (rounded to
 *              binary16 in `workspace`, then the binary16 path; binary16
 *              holds magnitudes up to 65504 and normal values down to
 *              6.1e-5, so larger fp32 inputs become +-Inf and values below
 *              about 6e-8 become zero -- scale such data first)
 *   K % 16 == 0 (the pages' rule for 16-bit sparse operands); R, T >= 1 any
 *   workspace  >= nm_spmm_workspace_bytes(...) bytes (may be NULL when 0)
 * int8 (ab_dtype NM_S8; review, "Structured sparse GEMM on tensor cores":
 * INT8 at 2:4, dimensions multiples of 32): values and X int8, meta_sm100 the
 * .kind::i8 image of nm_meta_to_sm100_s8 (NOT the nm_meta_to_sm100 image),
 * K % 32 == 0, exact s32 accumulation.  y_dtype NM_S32 stores the exact sum
 * (requires alpha == 1 and beta == 0, else NM_ERR_UNSUPPORTED; no overflow
 * while K <= 262144, since |sum| <= K/2 * 2^14); NM_F32 / NM_BF16 store
 * alpha * float(sum) + beta * Y (the conversion of sums beyond 2^24 rounds).
 * A bounded wait inside the kernel that gives up records NM_ERR_TIMEOUT in a
 * device status word, read and cleared by nm_last_device_status().
 */
NM_API nm_status nm_spmm(const void *values, const uint8_t *meta_sm100, nm_dtype ab_dtype,
                  const void *X, int64_t ldx, void *Y, nm_dtype y_dtype, int64_t ldy,
                  int64_t R, int64_t K, int64_t T, float alpha, float beta,
                  void *workspace, size_t workspace_bytes, void *stream);

/*
 * nm_spmm12 -- Y = alpha * (W (.) mask) X + beta * Y for a 1:2-sparse fp32 W
 * on the TF32 sparse tensor cores (review of "Accelerating Sparse Deep Neural
 * Networks", "Structured sparse GEMM on tensor cores": sparse TF32 only with
 * the 1:2 pattern), fp32 accumulation.
 *   values       R x K/2 fp32, the kept element of each pair (nm_mask_compress12
 *                / nm_compress12), row stride K/2
 *   meta12_sm100 the .kind::tf32 image of the 1:2 metadata (nm_meta12_to_sm100)
 *   X            K x T fp32, leading dim ldx >= T, ldx % 4 == 0
 *   Y            R x T, y_dtype NM_F32 or NM_BF16, leading dim ldy >= T
 *   K % 16 == 0; R, T any.  The tensor cores read values and X as TF32 (10
 *   fraction bits), so results carry that precision.  Errors as nm_spmm.
 */
NM_API nm_status nm_spmm12(const float *values, const uint8_t *meta12_sm100, const float *X, int64_t ldx,
                           void *Y, nm_dtype y_dtype, int64_t ldy, int64_t R, int64_t K, int64_t T,
                           float alpha, float beta, void *stream);

/*
 * nm_spmm_noalloc -- nm_spmm that allocates nothing and takes no workspace.
 * (No counterpart on the pages: this is an interface for callers.)  For
 * callers that are not allowed to allocate device memory: code running inside
 * a host framework that owns every device allocation (a serving engine or a
 * plugin host with a pre-reserved memory budget), or a latency-critical path
 * that cannot afford cudaMalloc's implicit device-wide synchronisation.
 *   Arguments as nm_spmm, without workspace / workspace_bytes.
 *   For NM_F32 inputs the binary16 staging buffers live in a fixed 16 MiB
 *   device array inside the library (held by every GPU that loads it, until
 *   exit); problems needing more (nm_spmm_workspace_bytes(...) > 16 MiB)
 *   return NM_ERR_WORKSPACE.  NM_BF16 / NM_F16 inputs need no scratch.
 *   The first NM_F32 call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.  The address is kept for the life of the
 *   process: after cudaDeviceReset on a device, do not call this entry
 *   point on that device again.
 *   Arguments are checked as nm_spmm checks them before the size limit, so a
 *   malformed call returns its own error rather than NM_ERR_WORKSPACE.
 *   All calls on a device share its one array, and it keeps the previous
 *   call's contents (every call overwrites what it reads, so nothing needs
 *   clearing).  Calls that may overlap on the same GPU -- issued to
 *   different streams, or from concurrent host threads -- race on it and
 *   must be serialised by the caller.
 */
NM_API nm_status nm_spmm_noalloc(const void *values, const uint8_t *meta_sm100, nm_dtype ab_dtype,
                                 const void *X, int64_t ldx, void *Y, nm_dtype y_dtype, int64_t ldy,
                                 int64_t R, int64_t K, int64_t T, float alpha, float beta, void *stream);

/*
 * Row-split product over several GPUs.  The pages describe the product on one
 * GPU only; these calls are this library's way of splitting it by output rows
 * (each GPU holds some rows of W and all of X) when the next step needs the
 * whole output on every GPU, as the down projection of an MLP needs all of
 * H = W_up X.  Each GPU stores its rows of the output straight into every
 * GPU's copy from the product's epilogue, then raises a flag on every GPU;
 * a GPU that needs the whole output waits for every flag.  One process per
 * GPU; the other GPUs' buffers are reached through CUDA IPC mappings.
 */
#define NM_IPC_HANDLE_BYTES 64
#define NM_MAX_PEERS 8

/*
 * nm_spmm_peers -- nm_spmm with beta = 0 and a bf16 output written into
 * rows [row0, row0 + R) of each of n_peers buffers.
 *   values, meta_sm100, X, ldx, R, K, T, alpha: as nm_spmm; ab_dtype NM_BF16
 *              or NM_F16 only (else NM_ERR_DTYPE)
 *   peer_Y     HOST array of n_peers device pointers (1 <= n_peers <= 8,
 *              else NM_ERR_SHAPE), each the start of a bf16 buffer with
 *              leading dim ldy >= T and at least row0 + R rows: this GPU's
 *              own buffer or another GPU's, mapped with nm_ipc_open; the
 *              caller owns them.  Every peer_Y[j] + row0 * ldy element must be
 *              16-byte aligned and ldy * 2 % 16 == 0 (else NM_ERR_ALIGN).
 *              Nothing outside those rows and the first T columns is written.
 *   row0 >= 0  the first output row of this GPU's slice.
 * Only the 256-column CTA-pair kernel does this: R must span an even number
 * of 128-row tiles, T > 128 and T % 8 == 0 (rows of whole 16-byte units:
 * a bulk tensor store writes the whole 16-byte unit holding a row's last
 * column), else NM_ERR_UNSUPPORTED.  Each output tile
 * leaves shared memory once per destination (bulk tensor stores, no
 * multicast).  The stores into other GPUs' buffers are complete when the
 * kernel ends; follow the call with nm_peer_signal on the same stream.
 * Errors otherwise as nm_spmm.
 */
NM_API nm_status nm_spmm_peers(const void *values, const uint8_t *meta_sm100, nm_dtype ab_dtype,
                               const void *X, int64_t ldx, void *const *peer_Y, int n_peers,
                               int64_t row0, int64_t ldy, int64_t R, int64_t K, int64_t T,
                               float alpha, void *stream);

/*
 * nm_peer_signal -- once the work issued to `stream` before it has finished,
 * stores `epoch` into slot `rank` of every GPU's flag array, with a
 * system-scope release (so a GPU that reads the flag sees every write that
 * work made to its memory).
 *   peer_flags HOST array of n_peers device pointers, 8-byte aligned, each
 *              GPU j's array of n_peers uint64 slots (own or IPC-mapped)
 *   0 <= rank < n_peers <= 8 (else NM_ERR_SHAPE)
 *   epoch      raised by the caller for every new round of stores; slots are
 *              compared with >=, so they never need resetting
 */
NM_API nm_status nm_peer_signal(uint64_t *const *peer_flags, int n_peers, int rank, uint64_t epoch,
                                void *stream);

/*
 * nm_peer_wait -- makes `stream` wait until every slot of this GPU's flag
 * array holds at least `epoch`: a one-warp kernel spins on the slots with
 * system-scope acquire loads.  The wait is bounded: after timeout_ns (> 0,
 * else NM_ERR_SHAPE) it gives up, records NM_ERR_TIMEOUT in the device status
 * word (nm_last_device_status) and lets the stream go on, so work after it
 * may then read rows that never arrived; check the status.
 *   flags      device array of n_peers uint64 slots, 8-byte aligned
 */
NM_API nm_status nm_peer_wait(const uint64_t *flags, int n_peers, uint64_t epoch, int64_t timeout_ns,
                              void *stream);

/*
 * nm_ipc_handle -- the CUDA IPC handle (NM_IPC_HANDLE_BYTES bytes written to
 * `handle`) of the device allocation holding dev_ptr, and dev_ptr's byte
 * offset in it.  nm_ipc_open(handle, offset, &p) in ANOTHER process (CUDA
 * refuses the process's own handles) maps the allocation and returns the
 * same byte in p; nm_ipc_close(p, offset) unmaps it.  The exporter keeps the
 * allocation alive while any importer has it mapped.  NM_ERR_CUDA when CUDA
 * refuses (not device memory, an allocation that cannot be exported, no
 * peer access).
 */
NM_API nm_status nm_ipc_handle(const void *dev_ptr, void *handle, int64_t *offset);
NM_API nm_status nm_ipc_open(const void *handle, int64_t offset, void **dev_ptr);
NM_API nm_status nm_ipc_close(void *dev_ptr, int64_t offset);

/*
 * nm_last_device_status -- synchronises `stream`, then returns and clears the
 * device status word written by kernels whose bounded waits gave up
 * (NM_OK if none did).  NM_ERR_CUDA if the synchronisation itself failed.
 */
NM_API nm_status nm_last_device_status(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* NM_H */
