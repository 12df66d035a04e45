// nm_compress12.cu -- 1:2 compression and decompression (one value of every
// pair kept), the pattern the review of "Accelerating Sparse Deep Neural
// Networks" ("Structured sparse GEMM on tensor cores") gives for sparse TF32.
//
// Layout (this library's choice): values[r][p] is the kept element of pair p
// (columns 2p, 2p+1) of row r, bits as stored; its index is bit p%8 of byte
// r*(C/16) + p/8 (LSB first).  HBM-bound streams: a thread takes units of 16
// elements (8 pairs, one metadata byte), 16-byte vector loads and stores; the
// compressors take two rows at a time with grids sized to the blocks the SMs
// hold.
#include "nm_internal.cuh"

namespace nm {
namespace {

// 16 elements of one row, as raw bits.
template <typename Bits> struct Row16 {
  static constexpr int kVec = int(sizeof(Bits));   // 16-byte vectors: 2 (16-bit) or 4 (32-bit)
  uint4 v[kVec];
  __device__ __forceinline__ void load(const Bits* p) {
#pragma unroll
    for (int i = 0; i < kVec; ++i) v[i] = __ldcs(reinterpret_cast<const uint4*>(p) + i);
  }
  __device__ __forceinline__ void store(Bits* p) const {
#pragma unroll
    for (int i = 0; i < kVec; ++i) __stcs(reinterpret_cast<uint4*>(p) + i, v[i]);
  }
  __device__ __forceinline__ Bits get(int i) const { return reinterpret_cast<const Bits*>(v)[i]; }
  __device__ __forceinline__ void set(int i, Bits b) { reinterpret_cast<Bits*>(v)[i] = b; }
};

// Eight values of one row.
template <typename Bits> struct Row8 {
  static constexpr int kVec = int(sizeof(Bits)) / 2;   // 1 (16-bit) or 2 (32-bit)
  uint4 v[kVec];
  __device__ __forceinline__ void load(const Bits* p) {
#pragma unroll
    for (int i = 0; i < kVec; ++i) v[i] = __ldcs(reinterpret_cast<const uint4*>(p) + i);
  }
  __device__ __forceinline__ void store(Bits* p) const {
#pragma unroll
    for (int i = 0; i < kVec; ++i) __stcs(reinterpret_cast<uint4*>(p) + i, v[i]);
  }
  __device__ __forceinline__ Bits get(int i) const { return reinterpret_cast<const Bits*>(v)[i]; }
  __device__ __forceinline__ void set(int i, Bits b) { reinterpret_cast<Bits*>(v)[i] = b; }
};

// MODE 0: keep the larger magnitude of each pair (ties -> the first);
// MODE 1: keep what the mask marks (exactly one 1 per pair, else the pair is
// counted as invalid and its first element kept).
template <typename Bits, int MODE>
__device__ __forceinline__ uint32_t compress12_unit(const Row16<Bits>& e, uint4 mk, Row8<Bits>& out, int& bad) {
  const uint8_t* mb = reinterpret_cast<const uint8_t*>(&mk);
  uint32_t bits = 0u;
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const Bits a = e.get(2 * p), b = e.get(2 * p + 1);
    uint32_t idx;
    if constexpr (MODE == 0) {
      idx = mag_key<Bits>(b) > mag_key<Bits>(a) ? 1u : 0u;
    } else {
      const uint32_t m0 = mb[2 * p], m1 = mb[2 * p + 1];
      const bool ok = (m0 | m1) <= 1u && m0 + m1 == 1u;
      bad += ok ? 0 : 1;
      idx = ok ? m1 : 0u;
    }
    out.set(p, idx ? b : a);
    bits |= idx << p;
  }
  return bits;
}

// A thread takes its unit in two rows (r and r + the grid's row stride) per
// iteration and issues both rows' loads before working on either.
template <typename Bits, int MODE>
__global__ void __launch_bounds__(256) compress12_kernel(const Bits* __restrict__ W, const uint8_t* __restrict__ mask,
                                                         int64_t R, int64_t upr, int64_t ldw, int64_t ldm,
                                                         Bits* __restrict__ values, uint8_t* __restrict__ meta,
                                                         int* __restrict__ invalid) {
  const int64_t r_step = int64_t(gridDim.y) * blockDim.y;
  const int64_t u_step = int64_t(gridDim.x) * blockDim.x;
  int bad = 0;
  for (int64_t r0 = int64_t(blockIdx.y) * blockDim.y + threadIdx.y; r0 < R; r0 += 2 * r_step) {
    for (int64_t u = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; u < upr; u += u_step) {
      Row16<Bits> e[2];
      uint4 mk[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int64_t r = r0 + k * r_step;
        if (r < R) {
          e[k].load(W + r * ldw + 16 * u);
          if constexpr (MODE == 1) mk[k] = __ldcs(reinterpret_cast<const uint4*>(mask + r * ldm + 16 * u));
        }
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int64_t r = r0 + k * r_step;
        if (r >= R) continue;
        Row8<Bits> out;
        const uint32_t bits = compress12_unit<Bits, MODE>(e[k], mk[k], out, bad);
        out.store(values + r * (upr * 8) + 8 * u);
        meta[r * upr + u] = uint8_t(bits);
      }
    }
  }
  if constexpr (MODE == 1) {
    if (invalid != nullptr) {
      bad = __reduce_add_sync(0xFFFFFFFFu, bad);
      if ((threadIdx.x & 31) == 0 && bad != 0) atomicAdd(invalid, bad);
    }
  }
}

// One row per iteration: the two-row form of the compressors measured 8 %
// slower here (the kernel is write-bound).
template <typename Bits>
__global__ void __launch_bounds__(256) decompress12_kernel(const Bits* __restrict__ values,
                                                           const uint8_t* __restrict__ meta, int64_t R, int64_t upr,
                                                           Bits* __restrict__ out, int64_t ldo) {
  const int64_t r_step = int64_t(gridDim.y) * blockDim.y;
  const int64_t u_step = int64_t(gridDim.x) * blockDim.x;
  for (int64_t r = int64_t(blockIdx.y) * blockDim.y + threadIdx.y; r < R; r += r_step) {
    for (int64_t u = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; u < upr; u += u_step) {
      Row8<Bits> v;
      v.load(values + r * (upr * 8) + 8 * u);
      const uint32_t bits = meta[r * upr + u];
      Row16<Bits> d;
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        const uint32_t idx = (bits >> p) & 1u;
        const Bits x = v.get(p);
        d.set(2 * p, idx ? Bits(0) : x);
        d.set(2 * p + 1, idx ? x : Bits(0));
      }
      d.store(out + r * ldo + 16 * u);
    }
  }
}

// fp32 decompression in units of 8 elements (4 pairs, half a metadata byte):
// 16 bytes of values in, 32 bytes out per thread, so a warp stores 1 KB of a
// row contiguously (the 16-element unit stores 64 bytes per thread).
__global__ void __launch_bounds__(256) decompress12_f32_kernel(const uint32_t* __restrict__ values,
                                                               const uint8_t* __restrict__ meta, int64_t R,
                                                               int64_t C, uint32_t* __restrict__ out, int64_t ldo) {
  const int64_t upr = C / 8;
  const int64_t r_step = int64_t(gridDim.y) * blockDim.y;
  const int64_t u_step = int64_t(gridDim.x) * blockDim.x;
  for (int64_t r = int64_t(blockIdx.y) * blockDim.y + threadIdx.y; r < R; r += r_step) {
    for (int64_t u = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; u < upr; u += u_step) {
      const uint4 v = __ldcs(reinterpret_cast<const uint4*>(values + r * (C / 2) + 4 * u));
      const uint32_t bits = uint32_t(meta[r * (C / 16) + u / 2]) >> (4 * (u & 1));
      const uint32_t x[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[8];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const bool second = (bits >> p) & 1u;
        o[2 * p] = second ? 0u : x[p];
        o[2 * p + 1] = second ? x[p] : 0u;
      }
      uint4* dst = reinterpret_cast<uint4*>(out + r * ldo + 8 * u);
      __stcs(dst, make_uint4(o[0], o[1], o[2], o[3]));
      __stcs(dst + 1, make_uint4(o[4], o[5], o[6], o[7]));
    }
  }
}

// x over the units of a row, y over rows; at most per_sm blocks per SM (the
// kernel's occupancy), so the whole grid is resident at once.
void shape_units(int64_t R, int64_t units, dim3& grid, dim3& block, int per_sm) {
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

nm_status check12(nm_dtype dtype, int64_t R, int64_t C) {
  if (!dtype_ok(dtype)) return NM_ERR_DTYPE;
  if (R < 0 || C < 0 || C % 16 != 0) return NM_ERR_SHAPE;
  return NM_OK;
}

template <int MODE>
nm_status run_compress12(const void* W, const uint8_t* mask, nm_dtype dtype, int64_t R, int64_t C, int64_t ldw,
                         int64_t ldm, void* values, uint8_t* meta, int32_t* invalid, void* stream) {
  nm_status st = check12(dtype, R, C);
  if (st != NM_OK) return st;
  if (ldw < C || (MODE == 1 && ldm < C)) return NM_ERR_SHAPE;
  if (R == 0 || C == 0) return NM_OK;
  if (W == nullptr || values == nullptr || meta == nullptr || (MODE == 1 && mask == nullptr)) return NM_ERR_NULL;
  const int es = esize_of(dtype);
  if (!aligned16(W) || !aligned16(values) || !stride_ok(ldw, es) ||
      (MODE == 1 && (!aligned16(mask) || !stride_ok(ldm, 1))))
    return NM_ERR_ALIGN;
  dim3 grid, block;
  static const int per_sm32 = blocks_per_sm(compress12_kernel<uint32_t, MODE>, 256);
  static const int per_sm16 = blocks_per_sm(compress12_kernel<uint16_t, MODE>, 256);
  shape_units(R, C / 16, grid, block, dtype == NM_F32 ? per_sm32 : per_sm16);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == NM_F32)
    compress12_kernel<uint32_t, MODE><<<grid, block, 0, s>>>(static_cast<const uint32_t*>(W), mask, R, C / 16, ldw,
                                                            ldm, static_cast<uint32_t*>(values), meta, invalid);
  else
    compress12_kernel<uint16_t, MODE><<<grid, block, 0, s>>>(static_cast<const uint16_t*>(W), mask, R, C / 16, ldw,
                                                            ldm, static_cast<uint16_t*>(values), meta, invalid);
  return launch_status();
}

}  // namespace
}  // namespace nm

extern "C" nm_status nm_mask_compress12(const void* W, nm_dtype dtype, int64_t R, int64_t C, int64_t ldw,
                                        void* values, uint8_t* meta, void* stream) {
  return nm::run_compress12<0>(W, nullptr, dtype, R, C, ldw, 0, values, meta, nullptr, stream);
}

extern "C" nm_status nm_compress12(const void* W, const uint8_t* mask, nm_dtype dtype, int64_t R, int64_t C,
                                   int64_t ldw, int64_t ldm, void* values, uint8_t* meta, int32_t* invalid_pairs,
                                   void* stream) {
  return nm::run_compress12<1>(W, mask, dtype, R, C, ldw, ldm, values, meta, invalid_pairs, stream);
}

extern "C" nm_status nm_decompress12(const void* values, const uint8_t* meta, nm_dtype dtype, int64_t R, int64_t C,
                                     void* W_out, int64_t ldw, void* stream) {
  using namespace nm;
  nm_status st = check12(dtype, R, C);
  if (st != NM_OK) return st;
  if (ldw < C) return NM_ERR_SHAPE;
  if (R == 0 || C == 0) return NM_OK;
  if (values == nullptr || meta == nullptr || W_out == nullptr) return NM_ERR_NULL;
  const int es = esize_of(dtype);
  if (!aligned16(values) || !aligned16(W_out) || !stride_ok(ldw, es)) return NM_ERR_ALIGN;
  dim3 grid, block;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == NM_F32) {
    shape_units(R, C / 8, grid, block, 8);
    decompress12_f32_kernel<<<grid, block, 0, s>>>(static_cast<const uint32_t*>(values), meta, R, C,
                                                   static_cast<uint32_t*>(W_out), ldw);
    return launch_status();
  }
  shape_units(R, C / 16, grid, block, 8);
  decompress12_kernel<uint16_t><<<grid, block, 0, s>>>(static_cast<const uint16_t*>(values), meta, R, C / 16,
                                                       static_cast<uint16_t*>(W_out), ldw);
  return launch_status();
}

// ---------------------------------------------------------------------------
// 1:2 metadata image for the .kind::tf32 sparse MMA (PTX ISA, tcgen05 sparse
// matrices).  A tf32 instruction reads its metadata in the .kind::f16 layout
// of the row seen as 16-bit halves: pair p (fp32 columns 2p, 2p+1) is the
// group of halves 4p..4p+3, whose 4-bit field is 0x4 when element 0 is kept
// and 0xE when element 1 is.  Per block of 128 rows x 64 fp32 columns the
// image holds the 2048 bytes one 128-lane x 128-bit copy moves into tensor
// memory: lane L, 32-bit slice s, field at bit 16*h8 + 4*q holds row
// 16*(L/16) + 8*h8 + L%8 and half-column 32*s + 16*((L/8)%2) + 4*q.  Blocks are
// row-tile major; padding rows and pairs hold 0x4.  One thread per lane row
// (16 bytes) of a block.
namespace nm {
namespace {

// A lane row holds two rows (r0 = 16*(L/16) + L%8 and r0 + 8), and for each
// row the pairs kt*32 + 8*s + 4*((L/8)%2) + q, s, q in 0..3: all inside the
// row's 32-bit metadata word kt.  So a thread reads two words and spreads
// their bits; with C % 64 == 0 (whole words per block) the words are loaded
// whole, otherwise byte by byte.
__global__ void __launch_bounds__(256) meta12_image_kernel(const uint8_t* __restrict__ meta, int64_t R, int64_t C,
                                                           int64_t kblocks, int64_t nrows16,
                                                           uint4* __restrict__ out) {
  const int64_t bpr = C / 16;  // metadata bytes per row
  const bool words = (C % 64) == 0 && (reinterpret_cast<uintptr_t>(meta) & 3u) == 0;
  for (int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; t < nrows16;
       t += int64_t(gridDim.x) * blockDim.x) {
    const int64_t blk = t >> 7;
    const int L = int(t & 127);
    const int64_t rt = blk / kblocks, kt = blk - rt * kblocks;
    uint32_t w[2];
#pragma unroll
    for (int h8 = 0; h8 < 2; ++h8) {
      const int64_t r = rt * 128 + 16 * (L >> 4) + 8 * h8 + (L & 7);
      uint32_t v = 0;                      // index bits of pairs kt*32 .. kt*32+31 (0 past the matrix: 0x4)
      if (r < R) {
        const uint8_t* src = meta + r * bpr + kt * 4;
        if (words) {
          v = __ldg(reinterpret_cast<const uint32_t*>(src));
        } else {
          for (int j = 0; j < 4 && kt * 4 + j < bpr; ++j) v |= uint32_t(src[j]) << (8 * j);
        }
      }
      w[h8] = v;
    }
    const int half = (L >> 3) & 1;
    uint32_t o[4];
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
      uint32_t word = 0;
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const int h8 = n >> 2, q = n & 3;
        const uint32_t bit = (w[h8] >> (8 * sl + 4 * half + q)) & 1u;
        word |= (bit ? 0xEu : 0x4u) << (16 * h8 + 4 * q);
      }
      o[sl] = word;
    }
    out[t] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace
}  // namespace nm

extern "C" size_t nm_meta12_image_bytes(int64_t R, int64_t C) {
  if (R <= 0 || C <= 0) return 0;
  return size_t((R + 127) / 128) * size_t((C + 63) / 64) * 2048;
}

extern "C" nm_status nm_meta12_to_sm100(const uint8_t* meta, int64_t R, int64_t C, uint8_t* meta12_sm100,
                                        void* stream) {
  using namespace nm;
  if (R < 0 || C < 0 || C % 16 != 0) return NM_ERR_SHAPE;
  if (R == 0 || C == 0) return NM_OK;
  if (meta == nullptr || meta12_sm100 == nullptr) return NM_ERR_NULL;
  if (!aligned16(meta12_sm100)) return NM_ERR_ALIGN;
  const int64_t kblocks = (C + 63) / 64;
  const int64_t rows16 = (R + 127) / 128 * kblocks * 128;
  const int64_t want = (rows16 + 255) / 256, cap = int64_t(sm_count()) * 8;
  meta12_image_kernel<<<unsigned(want < cap ? want : cap), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      meta, R, C, kblocks, rows16, reinterpret_cast<uint4*>(meta12_sm100));
  return launch_status();
}
