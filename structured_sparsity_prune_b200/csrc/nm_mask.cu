// nm_mask.cu -- N:M magnitude mask (any 1 <= N < M <= 8).
//
// Pages: "SR-STE sparse training" (N of every M consecutive weights kept;
// SR-STE forward keeps the N largest |w| of each group; the Apex exhaustive
// pattern search picks the same entries) and the review of "Accelerating
// Sparse Deep Neural Networks", Network Pruning Workflow Step-2.
//
// HBM-bound streaming kernel: every weight is read once and one mask byte is
// written per weight.  The selection is integer compares on the magnitude
// bits (no floating point), M*(M-1)/2 compares per group.
//
// The saliency-scored variant ("sparsegpt.py", fasterprune, semi-structured
// branch) ranks the binary32 scores fl(fl(w*w) / fl(d*d)) instead, with d the
// caller's per-column vector; same selection, same tie rule.
#include "nm_internal.cuh"

#include <cuda_fp16.h>

namespace nm {
namespace {

// 16 consecutive elements of one row -> 16 mask bytes (one 16-byte store).
template <typename Bits> struct Chunk16;
template <> struct Chunk16<uint32_t> {
  static constexpr int kVec = 4;  // 4 x 16 B loads
};
template <> struct Chunk16<uint16_t> {
  static constexpr int kVec = 2;  // 2 x 16 B loads
};
template <> struct Chunk16<uint8_t> {
  static constexpr int kVec = 1;  // 1 x 16 B load
};

// Keep-mask bytes of one 16-byte chunk of weights, groups of M (M | 16).
template <typename Bits, int M>
__device__ __forceinline__ uint4 select_chunk(const uint4 (&v)[Chunk16<Bits>::kVec], int N) {
  const Bits* e = reinterpret_cast<const Bits*>(v);
  uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int g = 0; g < 16 / M; ++g) {
    uint32_t key[M];
#pragma unroll
    for (int i = 0; i < M; ++i) key[i] = mag_key<Bits>(e[g * M + i]);
    const uint32_t kb = keep_bits<M>(key, N);
#pragma unroll
    for (int i = 0; i < M; ++i) {
      const int pos = g * M + i;  // byte position in the 16-byte chunk
      out[pos >> 2] |= ((kb >> i) & 1u) << (8 * (pos & 3));
    }
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

// Rows r and r + the row stride of the grid per iteration, both rows' loads
// issued before selecting in either.  For 8- and 16-bit elements in groups of
// eight the selection arithmetic, not the loads, bounds the kernel, and the
// second row's registers would only cost occupancy: one row at a time there.
template <typename Bits, int M>
__global__ void __launch_bounds__(256) mask_vec16_kernel(const Bits* __restrict__ W, int64_t R,
                                                         int64_t cpr, int64_t ldw, int N,
                                                         uint8_t* __restrict__ mask, int64_t ldm) {
  static_assert(16 % M == 0, "vector path needs M | 16");
  constexpr int kVec = Chunk16<Bits>::kVec;
  constexpr int kRows = (sizeof(Bits) <= 2 && M == 8) ? 1 : 2;
  const int64_t r_step = int64_t(gridDim.y) * blockDim.y;
  const int64_t c_step = int64_t(gridDim.x) * blockDim.x;
  for (int64_t r = int64_t(blockIdx.y) * blockDim.y + threadIdx.y; r < R; r += kRows * r_step) {
    const int64_t r2 = r + r_step;
    const bool two = kRows == 2 && r2 < R;
    const uint4* wrow = reinterpret_cast<const uint4*>(W + r * ldw);
    const uint4* wrow2 = reinterpret_cast<const uint4*>(W + (two ? r2 : r) * ldw);
    for (int64_t c = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; c < cpr; c += c_step) {
      uint4 v[kVec], v2[kVec];
#pragma unroll
      for (int i = 0; i < kVec; ++i) v[i] = __ldcs(wrow + c * kVec + i);
      if (two) {
#pragma unroll
        for (int i = 0; i < kVec; ++i) v2[i] = __ldcs(wrow2 + c * kVec + i);
      }
      __stcs(reinterpret_cast<uint4*>(mask + r * ldm) + c, select_chunk<Bits, M>(v, N));
      if (two) __stcs(reinterpret_cast<uint4*>(mask + r2 * ldm) + c, select_chunk<Bits, M>(v2, N));
    }
  }
}

// M = 4 fast path: 16 elements (four groups) per thread, the branch-free
// selection of drop4 and the byte packing of keep_bytes4.  A thread takes its
// chunk of two rows (r and r + the row stride of the grid) per iteration and
// issues both rows' loads before selecting in either; five blocks share an SM
// (the grid is sized to exactly what the SMs hold).  16-bit weights under
// 2^25 entries take four rows per iteration (four blocks per SM): on a short
// launch the bytes in flight set the pace.
template <typename Bits, int N>
__device__ __forceinline__ uint4 select4_chunk(const uint4 (&v)[Chunk16<Bits>::kVec]) {
  if constexpr (sizeof(Bits) == 1) {  // one int8 group per word
    return make_uint4(keep4_s8<N>(v[0].x), keep4_s8<N>(v[0].y), keep4_s8<N>(v[0].z), keep4_s8<N>(v[0].w));
  }
  const Bits* e = reinterpret_cast<const Bits*>(v);
  uint32_t out[4];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    uint32_t x0, x1, x2, x3;
    drop4<N>(mag_key<Bits>(e[4 * g]), mag_key<Bits>(e[4 * g + 1]), mag_key<Bits>(e[4 * g + 2]),
             mag_key<Bits>(e[4 * g + 3]), x0, x1, x2, x3);
    out[g] = keep_bytes4(x0, x1, x2, x3);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

template <typename Bits, int N, int ROWS = 2>
__global__ void __launch_bounds__(256, ROWS == 2 ? 5 : 4) mask4_vec16_kernel(const Bits* __restrict__ W, int64_t R,
                                                                          int64_t cpr, int64_t ldw,
                                                                          uint8_t* __restrict__ mask, int64_t ldm) {
  constexpr int kVec = Chunk16<Bits>::kVec;
  const int64_t r_step = int64_t(gridDim.y) * blockDim.y;
  const int64_t c_step = int64_t(gridDim.x) * blockDim.x;
  if constexpr (ROWS == 2) {
    for (int64_t r = int64_t(blockIdx.y) * blockDim.y + threadIdx.y; r < R; r += 2 * r_step) {
      const int64_t r2 = r + r_step;
      const bool two = r2 < R;
      const uint4* wrow = reinterpret_cast<const uint4*>(W + r * ldw);
      const uint4* wrow2 = reinterpret_cast<const uint4*>(W + (two ? r2 : r) * ldw);
      for (int64_t c = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; c < cpr; c += c_step) {
        uint4 v[kVec], v2[kVec];
#pragma unroll
        for (int i = 0; i < kVec; ++i) v[i] = __ldcs(wrow + c * kVec + i);
        if (two) {
#pragma unroll
          for (int i = 0; i < kVec; ++i) v2[i] = __ldcs(wrow2 + c * kVec + i);
        }
        __stcs(reinterpret_cast<uint4*>(mask + r * ldm) + c, select4_chunk<Bits, N>(v));
        if (two) __stcs(reinterpret_cast<uint4*>(mask + r2 * ldm) + c, select4_chunk<Bits, N>(v2));
      }
    }
  } else {
    for (int64_t r0 = int64_t(blockIdx.y) * blockDim.y + threadIdx.y; r0 < R; r0 += ROWS * r_step) {
      for (int64_t c = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; c < cpr; c += c_step) {
        uint4 v[ROWS][kVec];
#pragma unroll
        for (int k = 0; k < ROWS; ++k) {
          const int64_t r = r0 + k * r_step;
          if (r < R) {
#pragma unroll
            for (int i = 0; i < kVec; ++i)
              v[k][i] = __ldcs(reinterpret_cast<const uint4*>(W + r * ldw) + c * kVec + i);
          }
        }
#pragma unroll
        for (int k = 0; k < ROWS; ++k) {
          const int64_t r = r0 + k * r_step;
          if (r < R) __stcs(reinterpret_cast<uint4*>(mask + r * ldm) + c, select4_chunk<Bits, N>(v[k]));
        }
      }
    }
  }
}

// Any M (2..8), any alignment: one thread per group, scalar loads/stores.
template <typename Bits, int M>
__global__ void __launch_bounds__(256) mask_scalar_kernel(const Bits* __restrict__ W, int64_t R,
                                                          int64_t gpr, int64_t ldw, int N,
                                                          uint8_t* __restrict__ mask, int64_t ldm) {
  const int64_t r_step = int64_t(gridDim.y) * blockDim.y;
  const int64_t g_step = int64_t(gridDim.x) * blockDim.x;
  for (int64_t r = int64_t(blockIdx.y) * blockDim.y + threadIdx.y; r < R; r += r_step) {
    for (int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; g < gpr; g += g_step) {
      uint32_t key[M];
#pragma unroll
      for (int i = 0; i < M; ++i) key[i] = mag_key<Bits>(W[r * ldw + g * M + i]);
      const uint32_t kb = keep_bits<M>(key, N);
#pragma unroll
      for (int i = 0; i < M; ++i) mask[r * ldm + g * M + i] = uint8_t((kb >> i) & 1u);
    }
  }
}

// ---- saliency-scored selection ---------------------------------------------
// DT: 0 binary32, 1 bfloat16, 2 binary16 -> the exact binary32 value.
template <int DT>
__device__ __forceinline__ float elem_f32(uint32_t bits) {
  if constexpr (DT == 0) return __uint_as_float(bits);
  else if constexpr (DT == 1) return __uint_as_float(bits << 16);
  else return __half2float(__ushort_as_half(static_cast<unsigned short>(bits)));
}

// Score key: the bit pattern of fl(fl(w*w) / fl(d*d)) with the sign cleared.
// Each operation is rounded to nearest even on its own (no contraction, IEEE
// quotient), so the key equals the one a plain binary32 evaluation gives.
__device__ __forceinline__ uint32_t score_key(float w, float d) {
  return __float_as_uint(__fdiv_rn(__fmul_rn(w, w), __fmul_rn(d, d))) & 0x7FFFFFFFu;
}

// 16 consecutive elements of one row (and their 16 entries of d) -> 16 mask bytes.
template <typename Bits, int DT, int M>
__global__ void __launch_bounds__(256) scored_vec16_kernel(const Bits* __restrict__ W, const float* __restrict__ d,
                                                           int64_t R, int64_t cpr, int64_t ldw, int N,
                                                           uint8_t* __restrict__ mask, int64_t ldm) {
  static_assert(16 % M == 0, "vector path needs M | 16");
  constexpr int kVec = Chunk16<Bits>::kVec;
  const int64_t r_step = int64_t(gridDim.y) * blockDim.y;
  const int64_t c_step = int64_t(gridDim.x) * blockDim.x;
  const float4* d4 = reinterpret_cast<const float4*>(d);
  for (int64_t c = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; c < cpr; c += c_step) {
    float dv[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 t = __ldg(d4 + c * 4 + i);
      dv[4 * i] = t.x; dv[4 * i + 1] = t.y; dv[4 * i + 2] = t.z; dv[4 * i + 3] = t.w;
    }
    int64_t r = int64_t(blockIdx.y) * blockDim.y + threadIdx.y;
    uint4 nxt[kVec];
    if (r < R) {
#pragma unroll
      for (int i = 0; i < kVec; ++i) nxt[i] = __ldcs(reinterpret_cast<const uint4*>(W + r * ldw) + c * kVec + i);
    }
    for (; r < R; r += r_step) {
      uint4 v[kVec];
#pragma unroll
      for (int i = 0; i < kVec; ++i) v[i] = nxt[i];
      if (r + r_step < R) {   // prefetch the next row's chunk before working on this one
#pragma unroll
        for (int i = 0; i < kVec; ++i) nxt[i] = __ldcs(reinterpret_cast<const uint4*>(W + (r + r_step) * ldw) + c * kVec + i);
      }
      const Bits* e = reinterpret_cast<const Bits*>(v);
      uint32_t out[4] = {0u, 0u, 0u, 0u};
      if constexpr (M == 4) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t k[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) k[i] = score_key(elem_f32<DT>(e[4 * g + i]), dv[4 * g + i]);
          uint32_t x0, x1, x2, x3;
          if (N == 1) drop4<1>(k[0], k[1], k[2], k[3], x0, x1, x2, x3);
          else if (N == 2) drop4<2>(k[0], k[1], k[2], k[3], x0, x1, x2, x3);
          else drop4<3>(k[0], k[1], k[2], k[3], x0, x1, x2, x3);
          out[g] = keep_bytes4(x0, x1, x2, x3);
        }
      } else {
#pragma unroll
        for (int g = 0; g < 16 / M; ++g) {
          uint32_t key[M];
#pragma unroll
          for (int i = 0; i < M; ++i) key[i] = score_key(elem_f32<DT>(e[g * M + i]), dv[g * M + i]);
          const uint32_t kb = keep_bits<M>(key, N);
#pragma unroll
          for (int i = 0; i < M; ++i) {
            const int pos = g * M + i;
            out[pos >> 2] |= ((kb >> i) & 1u) << (8 * (pos & 3));
          }
        }
      }
      __stcs(reinterpret_cast<uint4*>(mask + r * ldm) + c, make_uint4(out[0], out[1], out[2], out[3]));
    }
  }
}

// Any M, any C: one thread per group, scalar loads/stores.
template <typename Bits, int DT, int M>
__global__ void __launch_bounds__(256) scored_scalar_kernel(const Bits* __restrict__ W, const float* __restrict__ d,
                                                            int64_t R, int64_t gpr, int64_t ldw, int N,
                                                            uint8_t* __restrict__ mask, int64_t ldm) {
  const int64_t r_step = int64_t(gridDim.y) * blockDim.y;
  const int64_t g_step = int64_t(gridDim.x) * blockDim.x;
  for (int64_t r = int64_t(blockIdx.y) * blockDim.y + threadIdx.y; r < R; r += r_step) {
    for (int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; g < gpr; g += g_step) {
      uint32_t key[M];
#pragma unroll
      for (int i = 0; i < M; ++i) key[i] = score_key(elem_f32<DT>(W[r * ldw + g * M + i]), __ldg(d + g * M + i));
      const uint32_t kb = keep_bits<M>(key, N);
#pragma unroll
      for (int i = 0; i < M; ++i) mask[r * ldm + g * M + i] = uint8_t((kb >> i) & 1u);
    }
  }
}

// 2D launch shape: x over the units of a row, y over rows; about 8 blocks of
// 256 threads per SM in total.
// x over the 16-byte chunks of a row, y over rows; at most per_sm blocks per SM
// (the kernel's occupancy), so the whole grid is resident at once.
void shape2d(int64_t R, int64_t units, dim3& grid, dim3& block, int per_sm = 8) {
  const int bx = row_block_x(units);
  const int by = 256 / bx;
  const int64_t gx = (units + bx - 1) / bx;
  const int64_t want = int64_t(sm_count()) * per_sm;
  int64_t gy = (R + by - 1) / by;
  const int64_t cap_y = gx >= want ? 1 : want / gx;
  if (gy > cap_y) gy = cap_y;
  if (gy > 65535) gy = 65535;
  grid = dim3(unsigned(gx > 2147483647 ? 2147483647 : gx), unsigned(gy < 1 ? 1 : gy), 1);
  block = dim3(bx, by, 1);
}

template <typename Bits, int M>
void launch_mask(const void* W, int64_t R, int64_t C, int64_t ldw, int N, uint8_t* mask, int64_t ldm,
                 bool vec, cudaStream_t s) {
  dim3 grid, block;
  if constexpr (M == 4) {
    if (vec) {
      const Bits* w = static_cast<const Bits*>(W);
      if constexpr (sizeof(Bits) == 2) {  // fp32 and int8 spill with four rows
        if (R * C < (int64_t(1) << 25)) {  // a short launch: four rows in flight per thread
          static const int per_sm4 = blocks_per_sm(mask4_vec16_kernel<Bits, 2, 4>, 256);
          shape2d(R, C / 16, grid, block, per_sm4);
          if (N == 1) mask4_vec16_kernel<Bits, 1, 4><<<grid, block, 0, s>>>(w, R, C / 16, ldw, mask, ldm);
          else if (N == 2) mask4_vec16_kernel<Bits, 2, 4><<<grid, block, 0, s>>>(w, R, C / 16, ldw, mask, ldm);
          else mask4_vec16_kernel<Bits, 3, 4><<<grid, block, 0, s>>>(w, R, C / 16, ldw, mask, ldm);
          return;
        }
      }
      static const int per_sm = blocks_per_sm(mask4_vec16_kernel<Bits, 2>, 256);
      shape2d(R, C / 16, grid, block, per_sm);
      if (N == 1) mask4_vec16_kernel<Bits, 1><<<grid, block, 0, s>>>(w, R, C / 16, ldw, mask, ldm);
      else if (N == 2) mask4_vec16_kernel<Bits, 2><<<grid, block, 0, s>>>(w, R, C / 16, ldw, mask, ldm);
      else mask4_vec16_kernel<Bits, 3><<<grid, block, 0, s>>>(w, R, C / 16, ldw, mask, ldm);
      return;
    }
  }
  if constexpr (16 % M == 0) {
    if (vec) {
      static const int per_sm = blocks_per_sm(mask_vec16_kernel<Bits, M>, 256);
      shape2d(R, C / 16, grid, block, per_sm);
      mask_vec16_kernel<Bits, M><<<grid, block, 0, s>>>(static_cast<const Bits*>(W), R, C / 16, ldw, N,
                                                        mask, ldm);
      return;
    }
  }
  shape2d(R, C / M, grid, block);
  mask_scalar_kernel<Bits, M><<<grid, block, 0, s>>>(static_cast<const Bits*>(W), R, C / M, ldw, N, mask, ldm);
}

template <typename Bits, int DT, int M>
void launch_scored(const void* W, const float* d, int64_t R, int64_t C, int64_t ldw, int N, uint8_t* mask,
                   int64_t ldm, bool vec, cudaStream_t s) {
  dim3 grid, block;
  const Bits* w = static_cast<const Bits*>(W);
  if constexpr (16 % M == 0) {
    if (vec) {
      shape2d(R, C / 16, grid, block);
      scored_vec16_kernel<Bits, DT, M><<<grid, block, 0, s>>>(w, d, R, C / 16, ldw, N, mask, ldm);
      return;
    }
  }
  shape2d(R, C / M, grid, block);
  scored_scalar_kernel<Bits, DT, M><<<grid, block, 0, s>>>(w, d, R, C / M, ldw, N, mask, ldm);
}

template <typename Bits, int DT>
void dispatch_scored(const void* W, const float* d, int64_t R, int64_t C, int64_t ldw, int N, int M, uint8_t* mask,
                     int64_t ldm, bool vec, cudaStream_t s) {
  switch (M) {
    case 2: launch_scored<Bits, DT, 2>(W, d, R, C, ldw, N, mask, ldm, vec, s); break;
    case 3: launch_scored<Bits, DT, 3>(W, d, R, C, ldw, N, mask, ldm, vec, s); break;
    case 4: launch_scored<Bits, DT, 4>(W, d, R, C, ldw, N, mask, ldm, vec, s); break;
    case 5: launch_scored<Bits, DT, 5>(W, d, R, C, ldw, N, mask, ldm, vec, s); break;
    case 6: launch_scored<Bits, DT, 6>(W, d, R, C, ldw, N, mask, ldm, vec, s); break;
    case 7: launch_scored<Bits, DT, 7>(W, d, R, C, ldw, N, mask, ldm, vec, s); break;
    default: launch_scored<Bits, DT, 8>(W, d, R, C, ldw, N, mask, ldm, vec, s); break;
  }
}

template <typename Bits>
void dispatch_m(const void* W, int64_t R, int64_t C, int64_t ldw, int N, int M, uint8_t* mask, int64_t ldm,
                bool vec, cudaStream_t s) {
  switch (M) {
    case 2: launch_mask<Bits, 2>(W, R, C, ldw, N, mask, ldm, vec, s); break;
    case 3: launch_mask<Bits, 3>(W, R, C, ldw, N, mask, ldm, vec, s); break;
    case 4: launch_mask<Bits, 4>(W, R, C, ldw, N, mask, ldm, vec, s); break;
    case 5: launch_mask<Bits, 5>(W, R, C, ldw, N, mask, ldm, vec, s); break;
    case 6: launch_mask<Bits, 6>(W, R, C, ldw, N, mask, ldm, vec, s); break;
    case 7: launch_mask<Bits, 7>(W, R, C, ldw, N, mask, ldm, vec, s); break;
    default: launch_mask<Bits, 8>(W, R, C, ldw, N, mask, ldm, vec, s); break;
  }
}

}  // namespace
}  // namespace nm

extern "C" nm_status nm_mask(const void* W, nm_dtype dtype, int64_t R, int64_t C, int64_t ldw, int N, int M,
                             uint8_t* mask, int64_t ldm, void* stream) {
  using namespace nm;
  if (!dtype_ok_int8(dtype)) return NM_ERR_DTYPE;
  if (M < 2 || M > 8 || N < 1 || N >= M) return NM_ERR_NM;
  if (R < 0 || C < 0 || C % M != 0 || ldw < C || ldm < C) return NM_ERR_SHAPE;
  if (R == 0 || C == 0) return NM_OK;
  if (W == nullptr || mask == nullptr) return NM_ERR_NULL;
  const int es = esize_of(dtype);
  if (!aligned16(W) || !aligned16(mask) || !stride_ok(ldw, es) || !stride_ok(ldm, 1)) return NM_ERR_ALIGN;
  const bool vec = (C % 16) == 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == NM_F32)
    dispatch_m<uint32_t>(W, R, C, ldw, N, M, mask, ldm, vec, s);
  else if (dtype == NM_S8)
    dispatch_m<uint8_t>(W, R, C, ldw, N, M, mask, ldm, vec, s);
  else
    dispatch_m<uint16_t>(W, R, C, ldw, N, M, mask, ldm, vec, s);
  return launch_status();
}

extern "C" nm_status nm_mask_scored(const void* W, nm_dtype dtype, const float* d, int64_t R, int64_t C, int64_t ldw,
                                    int N, int M, uint8_t* mask, int64_t ldm, void* stream) {
  using namespace nm;
  if (!dtype_ok(dtype)) return NM_ERR_DTYPE;
  if (M < 2 || M > 8 || N < 1 || N >= M) return NM_ERR_NM;
  if (R < 0 || C < 0 || C % M != 0 || ldw < C || ldm < C) return NM_ERR_SHAPE;
  if (R == 0 || C == 0) return NM_OK;
  if (W == nullptr || mask == nullptr || d == nullptr) return NM_ERR_NULL;
  const int es = esize_of(dtype);
  if (!aligned16(W) || !aligned16(mask) || !aligned16(d) || !stride_ok(ldw, es) || !stride_ok(ldm, 1))
    return NM_ERR_ALIGN;
  const bool vec = (C % 16) == 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == NM_F32)
    dispatch_scored<uint32_t, 0>(W, d, R, C, ldw, N, M, mask, ldm, vec, s);
  else if (dtype == NM_BF16)
    dispatch_scored<uint16_t, 1>(W, d, R, C, ldw, N, M, mask, ldm, vec, s);
  else
    dispatch_scored<uint16_t, 2>(W, d, R, C, ldw, N, M, mask, ldm, vec, s);
  return launch_status();
}
