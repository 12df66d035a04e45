// nm_srste.cu -- the SR-STE training step, fused into one HBM pass.
//
// Page: "SR-STE sparse training (quantisation-friendly)", SR-STE forward and
// backward.  Every step the forward recomputes the N:M mask of |w| and
// returns the masked weight; the backward returns grad + decay * (1 - mask) * w,
// so the pruned weights receive an extra decay * w and can grow back.
//
// One kernel reads W and grad once and writes the masked weight, the new
// gradient and (optionally) the mask: 2 * s bytes in and 2 * s (+1) bytes out
// per weight.  Selection is the magnitude rule of nm_mask.  The arithmetic is
// the listing's as PyTorch evaluates it: its mask is float32 (torch.ones with
// no dtype), so the forward w * m, the decay term decay * (1 - m) * w and the
// sum with the gradient are binary32 operations, each rounded on its own
// (never contracted into a fused multiply-add), and the results go back to the
// element type, one more rounding to nearest even for 16-bit elements.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "nm_internal.cuh"

namespace nm {
namespace {

template <typename Bits> struct Elem;
template <> struct Elem<uint32_t> {  // binary32
  static __device__ __forceinline__ float to_f(uint32_t b) { return __uint_as_float(b); }
  static __device__ __forceinline__ uint32_t from_f(float x) { return __float_as_uint(x); }
};
template <> struct Elem<uint16_t> {  // bfloat16; binary16 goes through f16_to_f / f16_from_f
  static __device__ __forceinline__ float to_f(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }
  static __device__ __forceinline__ uint16_t from_f(float x) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    return *reinterpret_cast<const uint16_t*>(&h);
  }
};
__device__ __forceinline__ float f16_to_f(uint16_t b) {
  __half h = *reinterpret_cast<const __half*>(&b);
  return __half2float(h);
}
__device__ __forceinline__ uint16_t f16_from_f(float x) {
  const __half h = __float2half_rn(x);
  return *reinterpret_cast<const uint16_t*>(&h);
}

template <typename Bits, bool F16>
__device__ __forceinline__ float elem_to_f(Bits b) {
  if constexpr (F16) return f16_to_f(b);
  else return Elem<Bits>::to_f(b);
}
template <typename Bits, bool F16>
__device__ __forceinline__ Bits elem_from_f(float x) {
  if constexpr (F16) return f16_from_f(x);
  else return Elem<Bits>::from_f(x);
}

// One entry of the step, in place: w <- w * m and g <- g + decay * (1 - m) * w
// with m = 1.0 (kept) or 0.0, every product and the sum rounded to binary32 on
// its own (__fmul_rn / __fadd_rn are never contracted), then to the element type.
template <typename Bits, bool F16>
__device__ __forceinline__ void srste_entry(Bits& w, Bits& g, bool keep, float decay) {
  const float m = keep ? 1.0f : 0.0f;
  const float wf = elem_to_f<Bits, F16>(w);
  const float t = __fmul_rn(__fmul_rn(decay, __fsub_rn(1.0f, m)), wf);
  g = elem_from_f<Bits, F16>(__fadd_rn(elem_to_f<Bits, F16>(g), t));
  w = elem_from_f<Bits, F16>(__fmul_rn(wf, m));
}

// keep bits of 16 consecutive entries (groups of M, M | 16)
template <typename Bits, int M, int NT>
__device__ __forceinline__ uint32_t keep16(const Bits* e, int N) {
  uint32_t kb = 0;
#pragma unroll
  for (int g = 0; g < 16 / M; ++g) {
    if constexpr (M == 4 && NT > 0) {
      uint32_t x0, x1, x2, x3;
      drop4<NT>(mag_key<Bits>(e[4 * g]), mag_key<Bits>(e[4 * g + 1]), mag_key<Bits>(e[4 * g + 2]),
                mag_key<Bits>(e[4 * g + 3]), x0, x1, x2, x3);
      kb |= ((~x0 >> 31) | ((~x1 >> 31) << 1) | ((~x2 >> 31) << 2) | ((~x3 >> 31) << 3)) << (4 * g);
    } else {
      uint32_t key[M];
#pragma unroll
      for (int i = 0; i < M; ++i) key[i] = mag_key<Bits>(e[g * M + i]);
      kb |= keep_bits<M>(key, N) << (g * M);
    }
  }
  return kb;
}

// 16 entries per thread: 16-byte loads of W and grad, 16-byte stores.  For
// 8- and 16-bit elements a thread takes its chunk in two rows (r and r + the
// grid's row stride) and issues both rows' loads before working on either.
// NT: N as a template parameter for the M = 4 fast path (0: runtime N).
template <typename Bits, bool F16, int M, int NT>
__global__ void __launch_bounds__(256) srste_vec16_kernel(const Bits* __restrict__ W, const Bits* __restrict__ G,
                                                          int64_t R, int64_t cpr, int64_t ld, int N, float decay,
                                                          Bits* __restrict__ WS, Bits* __restrict__ GO,
                                                          uint8_t* __restrict__ mask) {
  constexpr int kVec = 16 * int(sizeof(Bits)) / 16;  // 16-byte vectors per 16 entries
  constexpr int kRows = sizeof(Bits) <= 2 ? 2 : 1;    // rows whose loads are in flight together
  const int64_t r_step = int64_t(gridDim.y) * blockDim.y;
  const int64_t c_step = int64_t(gridDim.x) * blockDim.x;
  for (int64_t r0 = int64_t(blockIdx.y) * blockDim.y + threadIdx.y; r0 < R; r0 += kRows * r_step) {
    for (int64_t c = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; c < cpr; c += c_step) {
      uint4 wv[kRows][kVec], gv[kRows][kVec];
#pragma unroll
      for (int k = 0; k < kRows; ++k) {
        const int64_t r = r0 + k * r_step;
        if (r < R) {
#pragma unroll
          for (int i = 0; i < kVec; ++i) {
            wv[k][i] = __ldcs(reinterpret_cast<const uint4*>(W + r * ld) + c * kVec + i);
            gv[k][i] = __ldcs(reinterpret_cast<const uint4*>(G + r * ld) + c * kVec + i);
          }
        }
      }
#pragma unroll
      for (int k = 0; k < kRows; ++k) {
        const int64_t r = r0 + k * r_step;
        if (r >= R) continue;
        Bits* w = reinterpret_cast<Bits*>(wv[k]);
        Bits* g = reinterpret_cast<Bits*>(gv[k]);
        const uint32_t kb = keep16<Bits, M, NT>(w, N);
#pragma unroll
        for (int i = 0; i < 16; ++i) srste_entry<Bits, F16>(w[i], g[i], (kb >> i) & 1u, decay);
#pragma unroll
        for (int i = 0; i < kVec; ++i) {
          __stcs(reinterpret_cast<uint4*>(WS + r * ld) + c * kVec + i, wv[k][i]);
          __stcs(reinterpret_cast<uint4*>(GO + r * ld) + c * kVec + i, gv[k][i]);
        }
        if (mask != nullptr) {
          uint32_t mb[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) mb[q] = (((kb >> (4 * q)) & 0xFu) * 0x00204081u) & 0x01010101u;  // nibble -> 4 bytes
          __stcs(reinterpret_cast<uint4*>(mask + r * ld) + c, make_uint4(mb[0], mb[1], mb[2], mb[3]));
        }
      }
    }
  }
}

// any M, any alignment: one thread per group
template <typename Bits, bool F16, int M>
__global__ void __launch_bounds__(256) srste_scalar_kernel(const Bits* __restrict__ W, const Bits* __restrict__ G,
                                                           int64_t R, int64_t gpr, int64_t ld, int N, float decay,
                                                           Bits* __restrict__ WS, Bits* __restrict__ GO,
                                                           uint8_t* __restrict__ mask) {
  const int64_t r_step = int64_t(gridDim.y) * blockDim.y;
  const int64_t g_step = int64_t(gridDim.x) * blockDim.x;
  for (int64_t r = int64_t(blockIdx.y) * blockDim.y + threadIdx.y; r < R; r += r_step) {
    for (int64_t gi = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; gi < gpr; gi += g_step) {
      Bits w[M], g[M];
      uint32_t key[M];
#pragma unroll
      for (int i = 0; i < M; ++i) {
        w[i] = W[r * ld + gi * M + i];
        g[i] = G[r * ld + gi * M + i];
        key[i] = mag_key<Bits>(w[i]);
      }
      const uint32_t kb = keep_bits<M>(key, N);
#pragma unroll
      for (int i = 0; i < M; ++i) {
        const bool keep = (kb >> i) & 1u;
        Bits wo = w[i], go = g[i];
        srste_entry<Bits, F16>(wo, go, keep, decay);
        WS[r * ld + gi * M + i] = wo;
        GO[r * ld + gi * M + i] = go;
        if (mask != nullptr) mask[r * ld + gi * M + i] = uint8_t(keep ? 1 : 0);
      }
    }
  }
}

// x over the units of a row, y over rows; at most per_sm blocks per SM (the
// kernel's occupancy), so the whole grid is resident at once.
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

template <typename Bits, bool F16, int M>
void launch_m(const void* W, const void* G, int64_t R, int64_t C, int64_t ld, int N, float decay, void* WS,
              void* GO, uint8_t* mask, bool vec, cudaStream_t s) {
  const Bits* w = static_cast<const Bits*>(W);
  const Bits* g = static_cast<const Bits*>(G);
  Bits* ws = static_cast<Bits*>(WS);
  Bits* go = static_cast<Bits*>(GO);
  dim3 grid, block;
  if constexpr (16 % M == 0) {
    if (vec) {
      // 16-bit elements: exactly the resident blocks.  fp32 (one row at a time)
      // measured 9 % faster with the grid oversubscribed at 8 blocks per SM.
      static const int per_sm =
          sizeof(Bits) <= 2 ? blocks_per_sm(srste_vec16_kernel<Bits, F16, M, M == 4 ? 2 : 0>, 256) : 8;
      shape2d(R, C / 16, grid, block, per_sm);
      if constexpr (M == 4) {
        if (N == 1) srste_vec16_kernel<Bits, F16, 4, 1><<<grid, block, 0, s>>>(w, g, R, C / 16, ld, N, decay, ws, go, mask);
        else if (N == 2) srste_vec16_kernel<Bits, F16, 4, 2><<<grid, block, 0, s>>>(w, g, R, C / 16, ld, N, decay, ws, go, mask);
        else srste_vec16_kernel<Bits, F16, 4, 3><<<grid, block, 0, s>>>(w, g, R, C / 16, ld, N, decay, ws, go, mask);
      } else {
        srste_vec16_kernel<Bits, F16, M, 0><<<grid, block, 0, s>>>(w, g, R, C / 16, ld, N, decay, ws, go, mask);
      }
      return;
    }
  }
  shape2d(R, C / M, grid, block);
  srste_scalar_kernel<Bits, F16, M><<<grid, block, 0, s>>>(w, g, R, C / M, ld, N, decay, ws, go, mask);
}

template <typename Bits, bool F16>
void dispatch(const void* W, const void* G, int64_t R, int64_t C, int64_t ld, int N, int M, float decay, void* WS,
              void* GO, uint8_t* mask, bool vec, cudaStream_t s) {
  switch (M) {
    case 2: launch_m<Bits, F16, 2>(W, G, R, C, ld, N, decay, WS, GO, mask, vec, s); break;
    case 3: launch_m<Bits, F16, 3>(W, G, R, C, ld, N, decay, WS, GO, mask, vec, s); break;
    case 4: launch_m<Bits, F16, 4>(W, G, R, C, ld, N, decay, WS, GO, mask, vec, s); break;
    case 5: launch_m<Bits, F16, 5>(W, G, R, C, ld, N, decay, WS, GO, mask, vec, s); break;
    case 6: launch_m<Bits, F16, 6>(W, G, R, C, ld, N, decay, WS, GO, mask, vec, s); break;
    case 7: launch_m<Bits, F16, 7>(W, G, R, C, ld, N, decay, WS, GO, mask, vec, s); break;
    default: launch_m<Bits, F16, 8>(W, G, R, C, ld, N, decay, WS, GO, mask, vec, s); break;
  }
}

}  // namespace
}  // namespace nm

extern "C" nm_status nm_srste_step(const void* W, const void* grad, nm_dtype dtype, int64_t R, int64_t C,
                                   int64_t ld, int N, int M, float decay, void* W_sparse, void* grad_out,
                                   uint8_t* mask, void* stream) {
  using namespace nm;
  if (!dtype_ok(dtype)) return NM_ERR_DTYPE;
  if (M < 2 || M > 8 || N < 1 || N >= M) return NM_ERR_NM;
  if (R < 0 || C < 0 || C % M != 0 || ld < C) return NM_ERR_SHAPE;
  if (R == 0 || C == 0) return NM_OK;
  if (W == nullptr || grad == nullptr || W_sparse == nullptr || grad_out == nullptr) return NM_ERR_NULL;
  const int es = esize_of(dtype);
  if (!aligned16(W) || !aligned16(grad) || !aligned16(W_sparse) || !aligned16(grad_out) ||
      (mask && !aligned16(mask)) || !stride_ok(ld, es))
    return NM_ERR_ALIGN;
  const bool vec = (C % 16) == 0 && (mask == nullptr || stride_ok(ld, 1));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == NM_F32) dispatch<uint32_t, false>(W, grad, R, C, ld, N, M, decay, W_sparse, grad_out, mask, vec, s);
  else if (dtype == NM_BF16) dispatch<uint16_t, false>(W, grad, R, C, ld, N, M, decay, W_sparse, grad_out, mask, vec, s);
  else dispatch<uint16_t, true>(W, grad, R, C, ld, N, M, decay, W_sparse, grad_out, mask, vec, s);
  return launch_status();
}
