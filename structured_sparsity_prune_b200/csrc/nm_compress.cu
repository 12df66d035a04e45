// nm_compress.cu -- 2:4 compression, decompression and the tensor-core
// metadata image.
//
// Pages: review of "Accelerating Sparse Deep Neural Networks", "Benefits of
// 2:4 sparsity" -- the compressed matrix keeps R*C/2 values plus a 2-bit
// in-group index per value, and a group with more zeros still stores two
// values.  The hardware layout of the indices is the PTX ISA's tcgen05
// sparse-matrix metadata (the pages do not give one).
//
// All kernels here stream HBM; the int8 selections and the transposed
// compressor are bound by integer issue first.  A compressing thread takes a
// (row, 32-column) unit: it reads the unit's 32 weights with 16-byte loads,
// selects/compresses in registers, and writes its 16 values and 4 canonical
// metadata bytes with vector stores.  When C % 32 == 0 the units are streamed
// row by row (two rows per thread, whose image pieces share 4-byte words that
// the thread writes itself); otherwise a block walks 128-row x 128-column
// tiles, drops the units' 16-bit image pieces into shared memory and writes
// each finished 2048-byte image block with one coalesced 16-byte store per
// thread.  Decompression expands (row, 32- or 8-column) units; the transposed
// compressor (for the backward product) works on 32 x 32 tiles per warp in
// registers (see its comment below).
#include <cuda.h>

#include <mutex>

#include "nm_internal.cuh"

namespace nm {
namespace {

constexpr int kThreads = 256;
constexpr uint32_t kPadByte = 0x44u;  // two groups holding the pattern (0,1)

// 8 consecutive elements (one canonical metadata byte) as raw bits.
template <typename Bits> struct Oct;
template <> struct Oct<uint16_t> {
  uint4 v;
  __device__ __forceinline__ void load(const uint16_t* p) { v = __ldcs(reinterpret_cast<const uint4*>(p)); }
  __device__ __forceinline__ uint16_t operator[](int i) const {
    const uint32_t w = (&v.x)[i >> 1];
    return uint16_t((i & 1) ? (w >> 16) : (w & 0xFFFFu));
  }
};
template <> struct Oct<uint8_t> {
  uint2 v;
  __device__ __forceinline__ void load(const uint8_t* p) { v = __ldcs(reinterpret_cast<const uint2*>(p)); }
  __device__ __forceinline__ uint8_t operator[](int i) const { return uint8_t(((&v.x)[i >> 2] >> (8 * (i & 3))) & 0xFFu); }
};
template <> struct Oct<uint32_t> {
  uint4 v[2];
  __device__ __forceinline__ void load(const uint32_t* p) {
    v[0] = __ldcs(reinterpret_cast<const uint4*>(p));
    v[1] = __ldcs(reinterpret_cast<const uint4*>(p) + 1);
  }
  __device__ __forceinline__ uint32_t operator[](int i) const { return (&v[i >> 2].x)[i & 3]; }
};

// Four compressed values of one octet, stored as a unit.
template <typename Bits> struct Quad;
template <> struct Quad<uint16_t> {
  uint2 v;
  __device__ __forceinline__ void set(int i, uint16_t b) {
    uint32_t& w = (&v.x)[i >> 1];
    w = (i & 1) ? ((w & 0xFFFFu) | (uint32_t(b) << 16)) : ((w & 0xFFFF0000u) | b);
  }
  __device__ __forceinline__ void store(uint16_t* p) const { __stcs(reinterpret_cast<uint2*>(p), v); }
};
template <> struct Quad<uint8_t> {
  uint32_t v;
  __device__ __forceinline__ void set(int i, uint8_t b) { v = (v & ~(0xFFu << (8 * i))) | (uint32_t(b) << (8 * i)); }
  __device__ __forceinline__ void store(uint8_t* p) const { __stcs(reinterpret_cast<unsigned int*>(p), v); }
};
template <> struct Quad<uint32_t> {
  uint4 v;
  __device__ __forceinline__ void set(int i, uint32_t b) { (&v.x)[i] = b; }
  __device__ __forceinline__ void store(uint32_t* p) const { __stcs(reinterpret_cast<uint4*>(p), v); }
};

// ---- one group of four -> its stored pair ----------------------------------------
// The nibble idx0 | idx1 << 2 of every 4-bit keep pattern with at most two
// bits set: the kept positions, filled with the lowest unkept ones (a group
// with more zeros still stores two values).  Patterns with three or four set
// map to 0x4, the fallback (0,1) for invalid groups.
constexpr uint64_t make_pair_nib_lut() {
  uint64_t lut = 0;
  for (int k = 0; k < 16; ++k) {
    int take = k, n = ((k >> 0) & 1) + ((k >> 1) & 1) + ((k >> 2) & 1) + ((k >> 3) & 1);
    uint32_t nib = 0x4u;
    if (n <= 2) {
      for (int i = 0; i < 4 && n < 2; ++i)
        if (!((take >> i) & 1)) { take |= 1 << i; ++n; }
      int i0 = 0, i1 = 3;
      while (!((take >> i0) & 1)) ++i0;
      while (!((take >> i1) & 1)) --i1;
      nib = uint32_t(i0 | (i1 << 2));
    }
    lut |= uint64_t(nib) << (4 * k);
  }
  return lut;
}
constexpr uint64_t kPairNib = make_pair_nib_lut();

// Keep bits of four 0/1 mask bytes (bit k = bit 0 of byte k): one multiply
// gathers the four byte-aligned bits into bits 28..31 without carries.
__device__ __forceinline__ uint32_t keep_of_bytes(uint32_t w) { return ((w & 0x01010101u) * 0x10204080u) >> 28; }

struct Pick {
  uint32_t nib;   // idx0 | idx1 << 2
  bool zlo, zhi;  // the stored value is a +0.0 filler (an unkept position)
};

// Under the caller's mask (w: the group's four mask bytes).  A valid group
// holds 0/1 bytes with at most two ones; fewer are filled as above.  Anything
// else is invalid: counted, and stored as (0,1) with W's values.
__device__ __forceinline__ Pick pick_masked(uint32_t w, int& invalid) {
  const uint32_t keep = keep_of_bytes(w), n = __popc(keep);
  Pick p{0x4u, false, false};
  if ((w & 0xFEFEFEFEu) != 0 || n > 2) {
    ++invalid;
    return p;
  }
  p.nib = uint32_t(kPairNib >> (4 * keep)) & 0xFu;
  if (n < 2) {
    p.zlo = ((keep >> (p.nib & 3u)) & 1u) == 0;
    p.zhi = ((keep >> (p.nib >> 2)) & 1u) == 0;
  }
  return p;
}

// By magnitude: exactly two kept, so the first kept index is 0, 1 or 2 and
// the second 1, 2 or 3 (read off the drop signs, cheaper than the table).
template <typename Bits>
__device__ __forceinline__ Pick pick_magnitude(Bits e0, Bits e1, Bits e2, Bits e3) {
  uint32_t x0, x1, x2, x3;
  drop4<2>(mag_key<Bits>(e0), mag_key<Bits>(e1), mag_key<Bits>(e2), mag_key<Bits>(e3), x0, x1, x2, x3);
  const bool k0 = int32_t(x0) >= 0, k1 = int32_t(x1) >= 0, k2 = int32_t(x2) >= 0, k3 = int32_t(x3) >= 0;
  const uint32_t i0 = k0 ? 0u : (k1 ? 1u : 2u), i1 = k3 ? 3u : (k2 ? 2u : 1u);
  return Pick{i0 | (i1 << 2), false, false};
}

// The stored pair as packed bits.  16-bit elements: g01 holds entries 0, 1
// and g23 entries 2, 3 (entry i = bytes 2i, 2i+1 of the pair of words); one
// byte-permute picks both.  8-bit: the four entries in one word.
__device__ __forceinline__ uint32_t pair16(uint32_t g01, uint32_t g23, Pick p) {
  uint32_t v = __byte_perm(g01, g23, 34u * ((p.nib & 3u) + ((p.nib >> 2) << 8)) + 0x1010u);
  if (p.zlo) v &= 0xFFFF0000u;
  if (p.zhi) v &= 0x0000FFFFu;
  return v;
}
__device__ __forceinline__ uint32_t pair8(uint32_t g, Pick p) {
  uint32_t v = __byte_perm(g, 0u, (p.nib & 3u) | ((p.nib >> 2) << 4) | 0x4400u);
  if (p.zlo) v &= 0xFF00u;
  if (p.zhi) v &= 0x00FFu;
  return v;
}
__device__ __forceinline__ uint2 pair32(uint32_t e0, uint32_t e1, uint32_t e2, uint32_t e3, Pick p) {
  uint32_t a = sel4<uint32_t>(e0, e1, e2, e3, p.nib & 3u), b = sel4<uint32_t>(e0, e1, e2, e3, p.nib >> 2);
  if (p.zlo) a = 0u;
  if (p.zhi) b = 0u;
  return make_uint2(a, b);
}

// Compress one octet (two groups).  MODE 0 selects by magnitude; MODE 1 takes
// the caller's mask (8 bytes) and counts its invalid groups.
template <typename Bits, int MODE>
__device__ __forceinline__ uint32_t compress_octet(const Oct<Bits>& e, uint2 m, Quad<Bits>& q, int& invalid) {
  Pick p[2];
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    if constexpr (MODE == 0 && sizeof(Bits) == 1) {  // int8: the in-register rank rule
      const uint32_t keep = keep_of_bytes(keep4_s8<2>(g ? e.v.y : e.v.x));
      p[g] = Pick{uint32_t(kPairNib >> (4 * keep)) & 0xFu, false, false};
    } else if constexpr (MODE == 0) {
      p[g] = pick_magnitude<Bits>(e[4 * g], e[4 * g + 1], e[4 * g + 2], e[4 * g + 3]);
    } else {
      p[g] = pick_masked(g ? m.y : m.x, invalid);
    }
  }
  if constexpr (sizeof(Bits) == 2) {
    q.v = make_uint2(pair16(e.v.x, e.v.y, p[0]), pair16(e.v.z, e.v.w, p[1]));
  } else if constexpr (sizeof(Bits) == 1) {
    q.v = pair8(e.v.x, p[0]) | (pair8(e.v.y, p[1]) << 16);
  } else {
    const uint2 a = pair32(e.v[0].x, e.v[0].y, e.v[0].z, e.v[0].w, p[0]);
    const uint2 b = pair32(e.v[1].x, e.v[1].y, e.v[1].z, e.v[1].w, p[1]);
    q.v = make_uint4(a.x, a.y, b.x, b.y);
  }
  return p[0].nib | (p[1].nib << 4);
}

// One block walks 128x128 tiles (tile index = rt * kt_count + kt, the same
// order as the image blocks).
template <typename Bits, int MODE>
__global__ void __launch_bounds__(kThreads) compress_tiles_kernel(
    const Bits* __restrict__ W, int64_t ldw, const uint8_t* __restrict__ mask, int64_t ldm, int64_t R,
    int64_t C, Bits* __restrict__ values, uint8_t* __restrict__ meta, uint8_t* __restrict__ img,
    int32_t* __restrict__ invalid_groups) {
  __shared__ __align__(16) uint16_t s_img[1024];  // one 2048-byte image block
  const int64_t kt_count = (C + 127) / 128;
  const int64_t tiles = ((R + 127) / 128) * kt_count;
  const bool full_rows = (C % 32) == 0;  // vector stores of a whole unit are aligned
  int invalid = 0;
  for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
    const int64_t rt = tile / kt_count, kt = tile - rt * kt_count;
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
      const int u = threadIdx.x + pass * kThreads;  // 512 units: 128 rows x 4 slices
      const int64_t r = rt * 128 + (u >> 2);
      const int64_t c0 = kt * 128 + (u & 3) * 32;
      uint32_t bytes[4] = {kPadByte, kPadByte, kPadByte, kPadByte};
      if (r < R && c0 < C) {
        const Bits* wrow = W + r * ldw;
        if (full_rows) {
          // whole unit in range: 4 octets, loads first, then work
          Oct<Bits> e[4];
          uint2 m[4];
#pragma unroll
          for (int o = 0; o < 4; ++o) e[o].load(wrow + c0 + 8 * o);
          if constexpr (MODE == 1) {
            const uint4* mp = reinterpret_cast<const uint4*>(mask + r * ldm + c0);
            const uint4 a = __ldcs(mp), b = __ldcs(mp + 1);
            m[0] = make_uint2(a.x, a.y); m[1] = make_uint2(a.z, a.w);
            m[2] = make_uint2(b.x, b.y); m[3] = make_uint2(b.z, b.w);
          }
          Quad<Bits> q[4];
#pragma unroll
          for (int o = 0; o < 4; ++o) bytes[o] = compress_octet<Bits, MODE>(e[o], m[o], q[o], invalid);
          Bits* vrow = values + r * (C / 2) + c0 / 2;
#pragma unroll
          for (int o = 0; o < 4; ++o) q[o].store(vrow + 4 * o);
          const uint32_t word = bytes[0] | (bytes[1] << 8) | (bytes[2] << 16) | (bytes[3] << 24);
          __stcs(reinterpret_cast<uint32_t*>(meta + r * (C / 8) + c0 / 8), word);
        } else {
#pragma unroll
          for (int o = 0; o < 4; ++o) {
            const int64_t c = c0 + 8 * o;
            if (c < C) {
              Oct<Bits> e;
              e.load(wrow + c);
              uint2 m = make_uint2(0u, 0u);
              if constexpr (MODE == 1) m = __ldcs(reinterpret_cast<const uint2*>(mask + r * ldm + c));
              Quad<Bits> q;
              bytes[o] = compress_octet<Bits, MODE>(e, m, q, invalid);
              q.store(values + r * (C / 2) + c / 2);
              meta[r * (C / 8) + c / 8] = uint8_t(bytes[o]);
            }
          }
        }
      }
      if (img != nullptr) {
        const uint32_t rl = uint32_t(u >> 2), cl = uint32_t(u & 3) * 32u;
        s_img[sm100_piece_offset(rl, cl) >> 1] = uint16_t(bytes[0] | (bytes[1] << 8));
        s_img[sm100_piece_offset(rl, cl + 16) >> 1] = uint16_t(bytes[2] | (bytes[3] << 8));
      }
    }
    if (img != nullptr) {
      __syncthreads();
      if (threadIdx.x < 128) {
        const uint4 v = reinterpret_cast<const uint4*>(s_img)[threadIdx.x];
        __stcs(reinterpret_cast<uint4*>(img + tile * 2048) + threadIdx.x, v);
      }
      __syncthreads();
    }
  }
  if constexpr (MODE == 1) {
    if (invalid_groups != nullptr) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) invalid += __shfl_xor_sync(0xFFFFFFFFu, invalid, off);
      if ((threadIdx.x & 31) == 0 && invalid != 0) atomicAdd(invalid_groups, invalid);
    }
  }
}

// The four quads of a (row, 32-column) unit are contiguous: store them with
// as few 16-byte stores as the element size allows.
template <typename Bits>
__device__ __forceinline__ void store_unit(const Quad<Bits> (&q)[4], Bits* p) {
  uint4* d = reinterpret_cast<uint4*>(p);
  if constexpr (sizeof(Bits) == 1) {
    __stcs(d, make_uint4(q[0].v, q[1].v, q[2].v, q[3].v));
  } else if constexpr (sizeof(Bits) == 2) {
    __stcs(d, make_uint4(q[0].v.x, q[0].v.y, q[1].v.x, q[1].v.y));
    __stcs(d + 1, make_uint4(q[2].v.x, q[2].v.y, q[3].v.x, q[3].v.y));
  } else {
#pragma unroll
    for (int o = 0; o < 4; ++o) __stcs(d + o, q[o].v);
  }
}

// Row-streaming form for C % 32 == 0.  A thread takes one 32-column unit u in
// the two rows r and r + 8 with r % 16 < 8: the 16-bit image pieces of those
// two rows share each 4-byte word of the image block (low half row r, high
// half row r + 8), so the thread writes its two image words directly -- no
// shared memory, no block barrier.  Consecutive threads take consecutive units
// of the same rows, so a warp reads 32 contiguous units of each row.  The
// grid covers the image's padded extent (rows up to a multiple of 128, units
// up to a multiple of 4): threads outside the matrix write only pad pieces.
// For 8- and 16-bit elements both rows' loads are issued before either is
// used; fp32 (128 bytes per unit and row) takes the rows one after the other.
// Blocks that share an SM (MINB): two for 16- and 32-bit elements (~128
// registers a thread under a mask), more for int8, whose thread moves fewer
// bytes.  Selection by magnitude also has a three-block form (no spills) for
// weights under 2^25 entries: there a launch is short enough that the bytes
// in flight, not DRAM page traffic, set its pace (three blocks were 5 %
// slower on a 235 M-entry weight and 9 % faster on a 16.8 M one).
template <typename Bits, int MODE>
constexpr int kRowsBlocks = sizeof(Bits) == 1 ? (MODE == 0 ? 4 : 3) : 2;

template <typename Bits, int MODE, int MINB = kRowsBlocks<Bits, MODE>>
__global__ void __launch_bounds__(256, MINB) compress_rows_kernel(
    const Bits* __restrict__ W, int64_t ldw, const uint8_t* __restrict__ mask, int64_t ldm, int64_t R,
    int64_t C, Bits* __restrict__ values, uint8_t* __restrict__ meta, uint8_t* __restrict__ img,
    int32_t* __restrict__ invalid_groups) {
  constexpr int kAhead = sizeof(Bits) <= 2 ? 2 : 1;  // rows whose loads are in flight together
  const int64_t kt_count = (C + 127) / 128;
  const int64_t units = kt_count * 4;                // padded units per row
  const int64_t pairs = ((R + 127) / 128) * 64;      // padded row pairs
  const int64_t p_step = int64_t(gridDim.y) * blockDim.y;
  const int64_t u_step = int64_t(gridDim.x) * blockDim.x;
  int invalid = 0;
  for (int64_t p = int64_t(blockIdx.y) * blockDim.y + threadIdx.y; p < pairs; p += p_step) {
    const int64_t r0 = 16 * (p >> 3) + (p & 7);
    for (int64_t u = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; u < units; u += u_step) {
      const int64_t c0 = 32 * u;
      uint32_t piece[2][2];  // [row r0 / r0 + 8][columns c0 / c0 + 16]
#pragma unroll
      for (int h0 = 0; h0 < 2; h0 += kAhead) {
        Oct<Bits> e[kAhead][4];
        uint2 m[kAhead][4];
        bool in[kAhead];
#pragma unroll
        for (int k = 0; k < kAhead; ++k) {
          const int64_t r = r0 + 8 * (h0 + k);
          in[k] = r < R && c0 < C;
          if (in[k]) {
#pragma unroll
            for (int o = 0; o < 4; ++o) e[k][o].load(W + r * ldw + c0 + 8 * o);
            if constexpr (MODE == 1) {
              const uint4* mp = reinterpret_cast<const uint4*>(mask + r * ldm + c0);
              const uint4 a = __ldcs(mp), b = __ldcs(mp + 1);
              m[k][0] = make_uint2(a.x, a.y); m[k][1] = make_uint2(a.z, a.w);
              m[k][2] = make_uint2(b.x, b.y); m[k][3] = make_uint2(b.z, b.w);
            }
          }
        }
#pragma unroll
        for (int k = 0; k < kAhead; ++k) {
          const int64_t r = r0 + 8 * (h0 + k);
          uint32_t bytes[4] = {kPadByte, kPadByte, kPadByte, kPadByte};
          if (in[k]) {
            Quad<Bits> q[4];
#pragma unroll
            for (int o = 0; o < 4; ++o) bytes[o] = compress_octet<Bits, MODE>(e[k][o], m[k][o], q[o], invalid);
            store_unit<Bits>(q, values + r * (C / 2) + c0 / 2);
            __stcs(reinterpret_cast<uint32_t*>(meta + r * (C / 8) + c0 / 8),
                   bytes[0] | (bytes[1] << 8) | (bytes[2] << 16) | (bytes[3] << 24));
          }
          piece[h0 + k][0] = bytes[0] | (bytes[1] << 8);
          piece[h0 + k][1] = bytes[2] | (bytes[3] << 8);
        }
      }
      if (img != nullptr) {
        uint8_t* blk = img + ((r0 >> 7) * kt_count + (u >> 2)) * 2048;
        const uint32_t lane0 = uint32_t(r0 & 7) + 16u * uint32_t((r0 & 127) >> 4);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
          __stcs(reinterpret_cast<uint32_t*>(blk + (lane0 + 8u * hf) * 16u + (u & 3) * 4),
                 piece[0][hf] | (piece[1][hf] << 16));
      }
    }
  }
  if constexpr (MODE == 1) {
    if (invalid_groups != nullptr) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) invalid += __shfl_xor_sync(0xFFFFFFFFu, invalid, off);
      if ((threadIdx.x & 31) == 0 && invalid != 0) atomicAdd(invalid_groups, invalid);
    }
  }
}

// canonical metadata -> image, same tiling, no weights involved.  Each thread
// takes one row of the tile (16 canonical bytes, one 16-byte load when the row
// is whole) and drops its eight 16-bit pieces into the shared image block.
__global__ void __launch_bounds__(kThreads) meta_image_kernel(const uint8_t* __restrict__ meta, int64_t R,
                                                              int64_t C, uint8_t* __restrict__ img) {
  __shared__ __align__(16) uint16_t s_img[2][1024];
  const int64_t kt_count = (C + 127) / 128;
  const int64_t tiles = ((R + 127) / 128) * kt_count;
  const bool vec = (C % 128) == 0;  // whole 16-byte row pieces, 16-byte aligned
  const int half = threadIdx.x >> 7;  // two tiles per block iteration
  const int rl = threadIdx.x & 127;
  for (int64_t base = int64_t(blockIdx.x) * 2; base < tiles; base += int64_t(gridDim.x) * 2) {
    const int64_t tile = base + half;
    if (tile < tiles) {
      const int64_t rt = tile / kt_count, kt = tile - rt * kt_count;
      const int64_t r = rt * 128 + rl;
      uint32_t w[4] = {0x44444444u, 0x44444444u, 0x44444444u, 0x44444444u};
      if (r < R) {
        const uint8_t* mrow = meta + r * (C / 8) + kt * 16;
        if (vec) {
          const uint4 v = __ldcs(reinterpret_cast<const uint4*>(mrow));
          w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
        } else {
#pragma unroll
          for (int b = 0; b < 16; ++b) {
            if (kt * 128 + 8 * b < C) {
              const int wi = b >> 2, sh = 8 * (b & 3);
              w[wi] = (w[wi] & ~(0xFFu << sh)) | (uint32_t(mrow[b]) << sh);
            }
          }
        }
      }
#pragma unroll
      for (int sl = 0; sl < 4; ++sl) {
        s_img[half][sm100_piece_offset(uint32_t(rl), uint32_t(32 * sl)) >> 1] = uint16_t(w[sl] & 0xFFFFu);
        s_img[half][sm100_piece_offset(uint32_t(rl), uint32_t(32 * sl + 16)) >> 1] = uint16_t(w[sl] >> 16);
      }
    }
    __syncthreads();
    if (tile < tiles) {
      const uint4 v = reinterpret_cast<const uint4*>(s_img[half])[rl];
      __stcs(reinterpret_cast<uint4*>(img + tile * 2048) + rl, v);
    }
    __syncthreads();
  }
}

// Image from canonical metadata, row-pair form for C % 128 == 0.  A warp takes
// one 16-row group of the image and four consecutive 128-column tiles; lane
// (q, j) reads the 16 canonical bytes of rows r = 16g + q and r + 8 in tile j
// and writes the two 16-byte image chunks those rows share: chunk lanes q and
// q + 8 of the group, each word holding row r's piece in its low half and row
// r + 8's in its high half.  The eight lanes of a tile write 128 contiguous
// bytes per store; rows past R are written as pad pieces.
__global__ void __launch_bounds__(256) meta_image_rows_kernel(const uint8_t* __restrict__ meta, int64_t R,
                                                              int64_t C, uint8_t* __restrict__ img) {
  const int64_t kt_count = C / 128;
  const int64_t quads = (kt_count + 3) / 4;
  const int64_t items = ((R + 127) / 128) * 8 * quads;
  const int q = threadIdx.x & 7, j = (threadIdx.x >> 3) & 3;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  // Item it = g * quads + qd, it stepping by `warps`: (g, qd) advance by the
  // quotient and remainder of `warps`, with a carry, instead of a division per item.
  const int64_t it0 = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t groups = items / quads, d_g = warps / quads, d_qd = warps - d_g * quads;
  int64_t g = it0 / quads, qd = it0 - g * quads;
  for (; g < groups; g += d_g, qd += d_qd) {
    if (qd >= quads) {
      qd -= quads;
      ++g;
      if (g >= groups) break;
    }
    const int64_t kt = qd * 4 + j;
    if (kt >= kt_count) continue;
    const int64_t r = 16 * g + q;
    const uint4 pad = make_uint4(0x44444444u, 0x44444444u, 0x44444444u, 0x44444444u);
    uint4 a = pad, b = pad;
    if (r < R) a = __ldcs(reinterpret_cast<const uint4*>(meta + r * (C / 8) + kt * 16));
    if (r + 8 < R) b = __ldcs(reinterpret_cast<const uint4*>(meta + (r + 8) * (C / 8) + kt * 16));
    uint8_t* blk = img + ((r >> 7) * kt_count + kt) * 2048;
    const uint32_t lane0 = uint32_t(r & 7) + 16u * uint32_t((r & 127) >> 4);
    __stcs(reinterpret_cast<uint4*>(blk + lane0 * 16u),
           make_uint4(__byte_perm(a.x, b.x, 0x5410), __byte_perm(a.y, b.y, 0x5410), __byte_perm(a.z, b.z, 0x5410),
                      __byte_perm(a.w, b.w, 0x5410)));
    __stcs(reinterpret_cast<uint4*>(blk + (lane0 + 8u) * 16u),
           make_uint4(__byte_perm(a.x, b.x, 0x7632), __byte_perm(a.y, b.y, 0x7632), __byte_perm(a.z, b.z, 0x7632),
                      __byte_perm(a.w, b.w, 0x7632)));
  }
}

// Decompress: unit = one row x 8 columns (one metadata byte, four values).
template <typename Bits>
__global__ void __launch_bounds__(256) decompress_kernel(const Bits* __restrict__ values,
                                                         const uint8_t* __restrict__ meta, int64_t R,
                                                         int64_t C, Bits* __restrict__ out, int64_t ldo) {
  const int64_t opr = C / 8;
  const int64_t r_step = int64_t(gridDim.y) * blockDim.y;
  const int64_t o_step = int64_t(gridDim.x) * blockDim.x;
  for (int64_t r = int64_t(blockIdx.y) * blockDim.y + threadIdx.y; r < R; r += r_step) {
    for (int64_t o = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; o < opr; o += o_step) {
      const uint32_t mb = meta[r * (C / 8) + o];
      Bits v[4], d[8];
      if constexpr (sizeof(Bits) == 1) {
        // four int8 values in one word; each group's four outputs form one word
        const uint32_t x = __ldcs(reinterpret_cast<const unsigned int*>(values + r * (C / 2) + 4 * o));
        uint32_t gw[2];
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const uint32_t i0 = (mb >> (4 * g)) & 3u, i1 = (mb >> (4 * g + 2)) & 3u;
          gw[g] = (((x >> (16 * g)) & 0xFFu) << (8 * i0)) | (((x >> (16 * g + 8)) & 0xFFu) << (8 * i1));
        }
        __stcs(reinterpret_cast<uint2*>(out + r * ldo + 8 * o), make_uint2(gw[0], gw[1]));
        continue;
      } else if constexpr (sizeof(Bits) == 2) {
        const uint2 x = __ldcs(reinterpret_cast<const uint2*>(values + r * (C / 2) + 4 * o));
        v[0] = uint16_t(x.x & 0xFFFFu); v[1] = uint16_t(x.x >> 16);
        v[2] = uint16_t(x.y & 0xFFFFu); v[3] = uint16_t(x.y >> 16);
      } else {
        const uint4 x = __ldcs(reinterpret_cast<const uint4*>(values + r * (C / 2) + 4 * o));
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
      }
      Bits* dst = out + r * ldo + 8 * o;
      if constexpr (sizeof(Bits) == 2) {
        // each group's four outputs form one 64-bit word: the two kept values
        // shifted to 16 * idx, zeros elsewhere
        uint64_t g01[2];
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const uint32_t i0 = (mb >> (4 * g)) & 3u, i1 = (mb >> (4 * g + 2)) & 3u;
          g01[g] = (uint64_t(v[2 * g]) << (16 * i0)) | (uint64_t(v[2 * g + 1]) << (16 * i1));
        }
        uint4 y;
        y.x = uint32_t(g01[0]); y.y = uint32_t(g01[0] >> 32);
        y.z = uint32_t(g01[1]); y.w = uint32_t(g01[1] >> 32);
        __stcs(reinterpret_cast<uint4*>(dst), y);
      } else if constexpr (sizeof(Bits) == 4) {
#pragma unroll
        for (int i = 0; i < 8; ++i) d[i] = Bits(0);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t idx = (mb >> (2 * k)) & 3u;
          const int g = k >> 1;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if (idx == uint32_t(i)) d[4 * g + i] = v[k];
        }
        __stcs(reinterpret_cast<uint4*>(dst), make_uint4(d[0], d[1], d[2], d[3]));
        __stcs(reinterpret_cast<uint4*>(dst) + 1, make_uint4(d[4], d[5], d[6], d[7]));
      }
    }
  }
}

// Decompress, wide unit: one row x 32 columns (four canonical metadata bytes,
// sixteen values) per thread, 16-byte loads and stores.  Needs C % 32 == 0.
template <typename Bits>
__device__ __forceinline__ void expand32(uint32_t mw, const uint4* vv, uint4* dst) {
  const uint32_t* vw = reinterpret_cast<const uint32_t*>(vv);
  if constexpr (sizeof(Bits) == 1) {
    uint32_t o[8];  // value pair of group g: bytes 2g, 2g+1
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      const uint32_t nib = (mw >> (4 * g)) & 0xFu;
      const uint32_t w = vw[g >> 1] >> (16 * (g & 1));
      o[g] = ((w & 0xFFu) << (8 * (nib & 3u))) | (((w >> 8) & 0xFFu) << (8 * (nib >> 2)));
    }
    __stcs(dst, make_uint4(o[0], o[1], o[2], o[3]));
    __stcs(dst + 1, make_uint4(o[4], o[5], o[6], o[7]));
  } else if constexpr (sizeof(Bits) == 2) {
#pragma unroll
    for (int h = 0; h < 4; ++h) {  // two groups -> one 16-byte store; value pair of group g in word g
      uint64_t g2[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int g = 2 * h + k;
        const uint32_t nib = (mw >> (4 * g)) & 0xFu;
        const uint32_t w = vw[g];
        g2[k] = (uint64_t(w & 0xFFFFu) << (16 * (nib & 3u))) | (uint64_t(w >> 16) << (16 * (nib >> 2)));
      }
      __stcs(dst + h, make_uint4(uint32_t(g2[0]), uint32_t(g2[0] >> 32), uint32_t(g2[1]), uint32_t(g2[1] >> 32)));
    }
  } else {
#pragma unroll
    for (int g = 0; g < 8; ++g) {  // one group -> one 16-byte store
      const uint32_t nib = (mw >> (4 * g)) & 0xFu;
      const uint32_t i0 = nib & 3u, i1 = nib >> 2;
      const uint32_t v0 = vw[2 * g], v1 = vw[2 * g + 1];
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] = (uint32_t(i) == i0) ? v0 : ((uint32_t(i) == i1) ? v1 : 0u);
      __stcs(dst + g, make_uint4(o[0], o[1], o[2], o[3]));
    }
  }
}

// A thread takes its unit in two rows (r and r + the row stride of the grid)
// per iteration and issues both rows' loads before expanding either.
template <typename Bits>
__global__ void __launch_bounds__(256) decompress32_kernel(const Bits* __restrict__ values,
                                                           const uint8_t* __restrict__ meta, int64_t R,
                                                           int64_t C, Bits* __restrict__ out, int64_t ldo) {
  constexpr int kVals = 16 * int(sizeof(Bits)) / 16;  // 16-byte loads of values per unit: 1 or 2
  const int64_t upr = C / 32;
  const int64_t r_step = int64_t(gridDim.y) * blockDim.y;
  const int64_t u_step = int64_t(gridDim.x) * blockDim.x;
  for (int64_t r = int64_t(blockIdx.y) * blockDim.y + threadIdx.y; r < R; r += 2 * r_step) {
    const int64_t r2 = r + r_step;
    const bool two = r2 < R;
    for (int64_t u = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; u < upr; u += u_step) {
      uint4 vv[kVals], vv2[kVals];
      const uint32_t mw = __ldcs(reinterpret_cast<const uint32_t*>(meta + r * (C / 8) + 4 * u));
#pragma unroll
      for (int i = 0; i < kVals; ++i) vv[i] = __ldcs(reinterpret_cast<const uint4*>(values + r * (C / 2) + 16 * u) + i);
      uint32_t mw2 = 0;
      if (two) {
        mw2 = __ldcs(reinterpret_cast<const uint32_t*>(meta + r2 * (C / 8) + 4 * u));
#pragma unroll
        for (int i = 0; i < kVals; ++i)
          vv2[i] = __ldcs(reinterpret_cast<const uint4*>(values + r2 * (C / 2) + 16 * u) + i);
      }
      expand32<Bits>(mw, vv, reinterpret_cast<uint4*>(out + r * ldo + 32 * u));
      if (two) expand32<Bits>(mw2, vv2, reinterpret_cast<uint4*>(out + r2 * ldo + 32 * u));
    }
  }
}

// ---- decompression with staged reads ----------------------------------------
// The compressed inputs are packed (values R x C/2, metadata R x C/8), so the
// matrix is one stream of 8192-element units: unit u covers logical elements
// [8192u, 8192u + 8192) of the row-major R x C matrix.  One thread per CTA
// keeps kRingStages units' values and metadata in flight with bulk copies
// (cp.async.bulk, this GPU's own memory, no multicast) into a shared-memory
// ring, so the reads are never queued behind the CTA's own output stream;
// the 256 threads expand a unit from shared memory in 16-byte output chunks,
// consecutive threads on consecutive chunks, with 16-byte streaming stores.
// Needs every chunk inside one row (C % 8 == 0 for 16-bit, C % 16 for 8-bit
// elements) and R*C % 128 == 0 (whole 16-byte copies).
constexpr int kRingElems = 8192;
constexpr int kRingStages = 6;
constexpr uint64_t kRingWaitNs = 2000000000ull;  // bounded waits: 2 s

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16 bytes of decompressed output from 8 bytes of values and the groups'
// nibbles: 16-bit elements, 2 groups (4 values, nibbles in bits 0-7); 8-bit
// elements, 4 groups (8 values, nibbles in bits 0-15).  Unkept positions +0.
template <typename Bits>
__device__ __forceinline__ uint4 expand_chunk(uint2 vals, uint32_t nibs) {
  if constexpr (sizeof(Bits) == 2) {
    uint64_t g[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t nib = (nibs >> (4 * k)) & 0xFu;
      const uint32_t w = k ? vals.y : vals.x;
      g[k] = (uint64_t(w & 0xFFFFu) << (16 * (nib & 3u))) | (uint64_t(w >> 16) << (16 * (nib >> 2)));
    }
    return make_uint4(uint32_t(g[0]), uint32_t(g[0] >> 32), uint32_t(g[1]), uint32_t(g[1] >> 32));
  } else {
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t nib = (nibs >> (4 * k)) & 0xFu;
      const uint32_t w = ((k < 2 ? vals.x : vals.y) >> (16 * (k & 1))) & 0xFFFFu;
      o[k] = ((w & 0xFFu) << (8 * (nib & 3u))) | ((w >> 8) << (8 * (nib >> 2)));
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
  }
}

template <typename Bits>
__global__ void __launch_bounds__(256) decompress_ring_kernel(const Bits* __restrict__ values,
                                                              const uint8_t* __restrict__ meta, int64_t R,
                                                              int64_t C, Bits* __restrict__ out, int64_t ldo,
                                                              int* __restrict__ status) {
  constexpr int kValBytes = kRingElems / 2 * int(sizeof(Bits));
  constexpr int kMetaBytes = kRingElems / 8;
  constexpr int kStageBytes = kValBytes + kMetaBytes;
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ __align__(8) uint64_t full[kRingStages];
  const int64_t total = R * C;
  const int64_t units = (total + kRingElems - 1) / kRingElems;
  const int tid = threadIdx.x;

  auto issue = [&](int64_t u, int st) {
    const int64_t e0 = u * kRingElems;
    const int64_t n = (total - e0) < kRingElems ? (total - e0) : kRingElems;
    const uint32_t vb = uint32_t(n / 2) * uint32_t(sizeof(Bits)), mb = uint32_t(n / 8);
    const uint32_t bar = smem_addr(&full[st]);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(vb + mb) : "memory");
    uint8_t* dst = ring + st * kStageBytes;
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(dst)),
                 "l"(reinterpret_cast<const uint8_t*>(values) + (e0 / 2) * int64_t(sizeof(Bits))), "r"(vb), "r"(bar)
                 : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(dst + kValBytes)),
                 "l"(meta + e0 / 8), "r"(mb), "r"(bar)
                 : "memory");
  };

  if (tid == 0) {
    for (int st = 0; st < kRingStages; ++st)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&full[st])));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (tid == 0) {
    int st = 0;
    for (int64_t u = blockIdx.x; u < units && st < kRingStages; u += gridDim.x, ++st) issue(u, st);
  }

  int64_t it = 0;
  for (int64_t u = blockIdx.x; u < units; u += gridDim.x, ++it) {
    const int st = int(it % kRingStages);
    const uint32_t parity = uint32_t(it / kRingStages) & 1u;
    // bounded wait for this unit's copies (uniform: every thread waits on the same phase)
    bool ok = false;
    {
      const uint32_t bar = smem_addr(&full[st]);
      uint64_t t0 = 0;
      for (uint32_t spin = 0;; ++spin) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done) { ok = true; break; }
        uint64_t now;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
        if (spin == 0) t0 = now;
        else if (now - t0 > kRingWaitNs) break;
      }
    }
    if (!__syncthreads_and(ok ? 1 : 0)) {  // one decision for the whole CTA
      if (tid == 0 && status != nullptr) atomicExch(status, int(NM_ERR_TIMEOUT));
      break;
    }
    // 16 bytes of output per chunk (8 bf16 / 16 int8 columns: 2 or 4 groups),
    // chunk j of the unit handled by thread j % 256, so each warp store covers
    // 512 contiguous bytes; a chunk's 8 bytes of values and 2/es bytes of
    // metadata sit at 8j and (2/es)j in the stage
    const int64_t e0 = u * kRingElems;
    const uint8_t* src = ring + st * kStageBytes;
    constexpr int kChunks = kRingElems * int(sizeof(Bits)) / 16;
    constexpr int kCols = 16 / int(sizeof(Bits));
#pragma unroll
    for (int h = 0; h < kChunks / 256; ++h) {
      const int j = h * 256 + tid;
      const int64_t e = e0 + int64_t(j) * kCols;
      if (e < total) {
        const uint2 vals = *reinterpret_cast<const uint2*>(src + 8 * j);
        uint32_t nibs;
        if constexpr (sizeof(Bits) == 2) nibs = src[kValBytes + j];
        else nibs = *reinterpret_cast<const uint16_t*>(src + kValBytes + 2 * j);
        const int64_t r = e / C, c = e - r * C;
        __stcs(reinterpret_cast<uint4*>(out + r * ldo + c), expand_chunk<Bits>(vals, nibs));
      }
    }
    __syncthreads();  // every thread has read this stage
    if (tid == 0) {
      const int64_t un = u + int64_t(kRingStages) * gridDim.x;
      if (un < units) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic reads before the async refill
        issue(un, st);
      }
    }
  }
}

// ---- fused magnitude mask + compression with staged reads ----------------------
// nm_mask_compress on 16-bit weights with C % 256 == 0.  W comes in through a
// three-stage shared-memory ring of 64-row x 256-column tiles: four TMA boxes
// of 64 x 64 in the 128-byte swizzle per stage, issued by one thread per CTA
// (this GPU's own memory, no multicast), so the selection never waits on its
// own loads.  The threads then work as the row kernel does -- one (row pair r,
// r + 8; 32-column unit) each, the same selection, stores and image words --
// reading the unit from shared memory.  With the swizzle, the 32 threads of a
// warp (four row pairs x eight units) read eight distinct 16-byte bank groups
// per load, four deep: the minimum for 512 bytes.  Tiles cover the image's
// padded rows (a multiple of 128); rows past R arrive as zeros and only their
// image pieces (the pad pattern) are written.  Every wait is bounded and
// reports NM_ERR_TIMEOUT in the status word.
constexpr int kCRingStages = 3;
constexpr int kCRingRows = 64, kCRingCols = 256;
constexpr int kCRingBoxBytes = 64 * 128;                   // one 64 x 64 box of 16-bit weights
constexpr int kCRingStageBytes = 4 * kCRingBoxBytes;       // 32 KB
constexpr int kCRingSmem = kCRingStages * kCRingStageBytes + 1024;  // + alignment slack

__global__ void __launch_bounds__(256, 2) compress_ring_kernel(const __grid_constant__ CUtensorMap map_w,
                                                               int64_t R, int64_t C, uint16_t* __restrict__ values,
                                                               uint8_t* __restrict__ meta, uint8_t* __restrict__ img,
                                                               int* __restrict__ status) {
  extern __shared__ uint8_t cring_raw[];
  __shared__ __align__(8) uint64_t full[kCRingStages];
  // 128-byte swizzled boxes need 1024-byte aligned destinations
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(cring_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int64_t kt_count = C / 128;
  const int64_t ncb = C / kCRingCols;
  const int64_t tiles = ((R + 127) / 128) * (128 / kCRingRows) * ncb;

  auto issue = [&](int64_t t, int st) {
    const int64_t rb = t / ncb, cb = t - rb * ncb;
    const uint32_t bar = smem_addr(&full[st]);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(kCRingStageBytes)
                 : "memory");
#pragma unroll
    for (int b = 0; b < 4; ++b)
      asm volatile(
          "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
              "r"(smem_addr(ring + st * kCRingStageBytes + b * kCRingBoxBytes)),
          "l"(reinterpret_cast<uint64_t>(&map_w)), "r"(bar), "r"(int(cb * kCRingCols + 64 * b)),
          "r"(int(rb * kCRingRows))
          : "memory");
  };

  if (tid == 0) {
    for (int st = 0; st < kCRingStages; ++st)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&full[st])));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
  }
  __syncthreads();
  if (tid == 0) {
    int st = 0;
    for (int64_t t = blockIdx.x; t < tiles && st < kCRingStages; t += gridDim.x, ++st) issue(t, st);
  }

  // this thread's item inside a tile: 16-row group g, row pair p (rows 16g + p
  // and + 8), unit u (32 columns) = half h of box b
  const int g = tid >> 6, p = (tid >> 3) & 7, u = tid & 7, b = u >> 1, h = u & 1;
  const int rl = 16 * g + p;
  int64_t it = 0;
  for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
    const int st = int(it % kCRingStages);
    const uint32_t parity = uint32_t(it / kCRingStages) & 1u;
    bool ok = false;
    {
      const uint32_t bar = smem_addr(&full[st]);
      uint64_t t0 = 0;
      for (uint32_t spin = 0;; ++spin) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred q;\n\tmbarrier.try_wait.parity.shared::cta.b64 q, [%1], %2;\n\tselp.u32 %0, 1, 0, q;\n\t}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done) { ok = true; break; }
        uint64_t now;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
        if (spin == 0) t0 = now;
        else if (now - t0 > kRingWaitNs) break;
      }
    }
    if (!__syncthreads_and(ok ? 1 : 0)) {  // one decision for the whole CTA
      if (tid == 0 && status != nullptr) atomicExch(status, int(NM_ERR_TIMEOUT));
      break;
    }
    const int64_t rb = t / ncb, cb = t - rb * ncb;
    const int64_t r0 = rb * kCRingRows + rl;
    const int64_t c0 = cb * kCRingCols + 32 * u;
    const uint8_t* box = ring + st * kCRingStageBytes + b * kCRingBoxBytes;
    uint32_t piece[2][2];
    int invalid = 0;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int row = rl + 8 * k;
      const int64_t r = r0 + 8 * k;
      Oct<uint16_t> e[4];
#pragma unroll
      for (int o = 0; o < 4; ++o)  // chunk 4h + o of the row sits at (4h + o) ^ (row % 8)
        e[o].v = *reinterpret_cast<const uint4*>(box + row * 128 + (((4 * h + o) ^ (row & 7)) << 4));
      uint32_t bytes[4] = {kPadByte, kPadByte, kPadByte, kPadByte};
      if (r < R) {
        Quad<uint16_t> q[4];
#pragma unroll
        for (int o = 0; o < 4; ++o) bytes[o] = compress_octet<uint16_t, 0>(e[o], make_uint2(0u, 0u), q[o], invalid);
        store_unit<uint16_t>(q, values + r * (C / 2) + c0 / 2);
        __stcs(reinterpret_cast<uint32_t*>(meta + r * (C / 8) + c0 / 8),
               bytes[0] | (bytes[1] << 8) | (bytes[2] << 16) | (bytes[3] << 24));
      }
      piece[k][0] = bytes[0] | (bytes[1] << 8);
      piece[k][1] = bytes[2] | (bytes[3] << 8);
    }
    if (img != nullptr) {
      uint8_t* blk = img + ((r0 >> 7) * kt_count + (c0 >> 7)) * 2048;
      const uint32_t lane0 = uint32_t(r0 & 7) + 16u * uint32_t((r0 & 127) >> 4);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
        __stcs(reinterpret_cast<uint32_t*>(blk + (lane0 + 8u * hf) * 16u + ((c0 >> 5) & 3) * 4),
               piece[0][hf] | (piece[1][hf] << 16));
    }
    __syncthreads();  // every thread has read this stage
    if (tid == 0) {
      const int64_t tn = t + int64_t(kCRingStages) * gridDim.x;
      if (tn < tiles) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic reads before the async refill
        issue(tn, st);
      }
    }
  }
  // a CTA that stopped early lets its copies in flight land before leaving
  // (bounded): they complete on its barriers
  if (tid == 0) {
    const uint64_t lim = kRingWaitNs;
    uint64_t t0;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    for (int64_t k = it; k < it + kCRingStages; ++k) {
      const int64_t t = blockIdx.x + k * int64_t(gridDim.x);
      if (t >= tiles) break;
      const uint32_t bar = smem_addr(&full[int(k % kCRingStages)]);
      const uint32_t parity = uint32_t(k / kCRingStages) & 1u;
      for (;;) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred q;\n\tmbarrier.try_wait.parity.shared::cta.b64 q, [%1], %2;\n\tselp.u32 %0, 1, 0, q;\n\t}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        uint64_t now;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
        if (done || now - t0 > lim) break;
      }
    }
  }
  __syncthreads();
}

// ---- compression of the transpose ---------------------------------------------
// Wt = W^T (C x R) compressed 2:4 along R under mask^T: the operand of the
// backward product dX = W^T dY when the mask is transposable (every group of
// four consecutive rows in a column keeps at most two).  Registers only: a
// warp takes a tile of 32 rows x 32 columns of W, and lane (q, h) = (lane % 4,
// lane / 4) reads columns 8q..8q+7 of the four rows 4h..4h+3 -- one group
// down each of its eight columns -- with one 8-element load per row (a warp
// reads 64 B, 32 B or 128 B of each of 32 rows).  It compresses the eight
// groups in registers and stores each pair of values into row c of Wt (the
// eight lanes of a column chunk fill 8 consecutive groups: one 32-byte run
// of a row of Wt per store).  The lane's eight nibbles make one word, and a
// three-stage nibble transpose across the eight lanes of its column chunk
// leaves lane h holding the metadata word of row c + h of Wt (8 nibbles, 32
// columns of Wt).  Image words pair rows c and c + 8 of Wt, which are lanes q
// and q ^ 1: one more shuffle, and lane h writes the image word of row c + h.
// The warps of a block take adjacent column tiles of the same rows; the grid
// covers the image's padded extent.
template <typename Bits>
__device__ __forceinline__ Oct<Bits> make_oct(const Bits (&a)[8]) {
  Oct<Bits> e;
  if constexpr (sizeof(Bits) == 1) {
    e.v = make_uint2(uint32_t(a[0]) | (uint32_t(a[1]) << 8) | (uint32_t(a[2]) << 16) | (uint32_t(a[3]) << 24),
                     uint32_t(a[4]) | (uint32_t(a[5]) << 8) | (uint32_t(a[6]) << 16) | (uint32_t(a[7]) << 24));
  } else if constexpr (sizeof(Bits) == 2) {
    e.v = make_uint4(uint32_t(a[0]) | (uint32_t(a[1]) << 16), uint32_t(a[2]) | (uint32_t(a[3]) << 16),
                     uint32_t(a[4]) | (uint32_t(a[5]) << 16), uint32_t(a[6]) | (uint32_t(a[7]) << 16));
  } else {
    e.v[0] = make_uint4(a[0], a[1], a[2], a[3]);
    e.v[1] = make_uint4(a[4], a[5], a[6], a[7]);
  }
  return e;
}

// The lane's eight columns of one tile: pick each group down a column under
// the mask, store its pair into that column's row of Wt (vdst + j * rh), and
// return the eight nibbles as one word (nibble j = column j; pad (0,1) for
// columns past C).  kFull: all eight columns are in range, no per-column test.
template <typename Bits, bool kFull>
__device__ __forceinline__ uint32_t compress_t_columns(const Oct<Bits> (&e)[4], const uint2 (&mk)[4], int ncols,
                                                       Bits* __restrict__ vdst, int64_t rh, int& invalid) {
  uint32_t nibs = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint32_t nib = 0x4u;  // pad: pattern (0,1)
    if (kFull || j < ncols) {
      // mask byte j of rows 0..3 -> bytes 0..3 of w
      const uint32_t sel = (j & 3) | (((j & 3) + 4) << 4);  // a constant after unrolling
      const uint32_t lo = __byte_perm(j < 4 ? mk[0].x : mk[0].y, j < 4 ? mk[1].x : mk[1].y, sel);
      const uint32_t hi = __byte_perm(j < 4 ? mk[2].x : mk[2].y, j < 4 ? mk[3].x : mk[3].y, sel);
      const uint32_t w = __byte_perm(lo, hi, 0x5410);
      const Pick pk = pick_masked(w, invalid);
      nib = pk.nib;
      Bits* dst = vdst + j * rh;
      if constexpr (sizeof(Bits) == 2) {
        // entry j of rows 0..3: half j & 1 of word j / 2 of each row
        const uint32_t hsel = (j & 1) ? 0x7632u : 0x5410u;
        const uint32_t g01 = __byte_perm((&e[0].v.x)[j >> 1], (&e[1].v.x)[j >> 1], hsel);
        const uint32_t g23 = __byte_perm((&e[2].v.x)[j >> 1], (&e[3].v.x)[j >> 1], hsel);
        __stcs(reinterpret_cast<uint32_t*>(dst), pair16(g01, g23, pk));
      } else if constexpr (sizeof(Bits) == 1) {
        const uint32_t blo = __byte_perm(j < 4 ? e[0].v.x : e[0].v.y, j < 4 ? e[1].v.x : e[1].v.y, sel);
        const uint32_t bhi = __byte_perm(j < 4 ? e[2].v.x : e[2].v.y, j < 4 ? e[3].v.x : e[3].v.y, sel);
        __stcs(reinterpret_cast<unsigned short*>(dst),
               static_cast<unsigned short>(pair8(__byte_perm(blo, bhi, 0x5410), pk)));
      } else {
        __stcs(reinterpret_cast<uint2*>(dst), pair32(e[0][j], e[1][j], e[2][j], e[3][j], pk));
      }
    }
    nibs |= nib << (4 * j);
  }
  return nibs;
}

template <typename Bits>
__global__ void __launch_bounds__(256, 3) compress_t_kernel(const Bits* __restrict__ W, int64_t ldw,
                                                         const uint8_t* __restrict__ mask, int64_t ldm, int64_t R,
                                                         int64_t C, Bits* __restrict__ values,
                                                         uint8_t* __restrict__ meta, uint8_t* __restrict__ img,
                                                         int32_t* __restrict__ invalid_groups) {
  const int lane = threadIdx.x & 31, q = lane & 3, h = lane >> 2;
  const int64_t Rp = (R + 127) / 128 * 128, Cp = (C + 127) / 128 * 128;  // padded image extents
  const int64_t ct_count = Cp / 32, rt_count = Rp / 32;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const bool meta_words = R % 32 == 0;
  const int64_t rh = R / 2;
  int invalid = 0;
  // Tile t = rt * ct_count + ct, t stepping by nwarps: (rt, ct) advance by the
  // quotient and remainder of nwarps, with a carry, instead of a division per tile.
  const int64_t t0 = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  int64_t rt = t0 / ct_count, ct = t0 - rt * ct_count;
  const int64_t d_rt = nwarps / ct_count, d_ct = nwarps - d_rt * ct_count;
  for (; rt < rt_count; rt += d_rt, ct += d_ct) {
    if (ct >= ct_count) {
      ct -= ct_count;
      ++rt;
      if (rt >= rt_count) break;
    }
    const int64_t r0 = rt * 32, r = r0 + 4 * h;   // the lane's four rows: one group down each column
    const int64_t c = ct * 32 + 8 * q;
    Oct<Bits> e[4];
    uint2 mk[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) mk[k] = make_uint2(0u, 0u);
    const bool rows_in = r < R;  // R % 4 == 0: the four rows are in or out together
    const bool full = rows_in && c + 8 <= C;
    if (full) {
      const Bits* wrow = W + r * ldw + c;
      const uint8_t* mrow = mask + r * ldm + c;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        e[k].load(wrow + k * ldw);
        mk[k] = __ldcs(reinterpret_cast<const uint2*>(mrow + k * ldm));
      }
    } else if (rows_in && c < C) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        Bits a[8];
        uint8_t b[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          a[j] = c + j < C ? W[(r + k) * ldw + c + j] : Bits(0);
          b[j] = c + j < C ? mask[(r + k) * ldm + c + j] : uint8_t(0);
        }
        e[k] = make_oct<Bits>(a);
        mk[k] = make_uint2(uint32_t(b[0]) | (uint32_t(b[1]) << 8) | (uint32_t(b[2]) << 16) | (uint32_t(b[3]) << 24),
                           uint32_t(b[4]) | (uint32_t(b[5]) << 8) | (uint32_t(b[6]) << 16) | (uint32_t(b[7]) << 24));
      }
    }
    // This lane's eight nibbles (group h of columns c..c+7, nibble j = column j)
    // form one word; an 8 x 8 nibble transpose across the eight lanes of the
    // column chunk (h = lane bits 2..4) gives lane h the metadata word of row
    // c + h of Wt (nibble g = group g).  Three masked butterfly stages.
    Bits* vdst = values + c * rh + r / 2;  // dereferenced only for columns in range
    uint32_t nibs;
    if (full) {
      nibs = compress_t_columns<Bits, true>(e, mk, 8, vdst, rh, invalid);
    } else {
      const int ncols = rows_in && c < C ? int(C - c < 8 ? C - c : 8) : 0;
      nibs = compress_t_columns<Bits, false>(e, mk, ncols, vdst, rh, invalid);
    }
    {
      constexpr uint32_t kLo[3] = {0x0F0F0F0Fu, 0x00FF00FFu, 0x0000FFFFu};
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        const int d = 1 << k;
        const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, nibs, 4 * d);  // lane of group h ^ d
        nibs = (h & d) ? ((nibs & ~kLo[k]) | ((other >> (4 * d)) & kLo[k]))
                       : ((nibs & kLo[k]) | ((other << (4 * d)) & ~kLo[k]));
      }
    }
    const uint32_t mword = nibs;
    const uint32_t partner = __shfl_xor_sync(0xFFFFFFFFu, mword, 1);  // row c + h +- 8 (lane q ^ 1)
    const uint32_t iword = (q & 1) ? __byte_perm(partner, mword, 0x7632) : __byte_perm(mword, partner, 0x5410);
    const int64_t crow = c + h;  // the row of Wt this lane stores for
    if (crow < C && r0 < R) {
      uint8_t* mrow = meta + crow * (R / 8) + r0 / 8;
      if (meta_words) {
        __stcs(reinterpret_cast<uint32_t*>(mrow), mword);
      } else {
#pragma unroll
        for (int b = 0; b < 4; ++b)
          if (r0 + 8 * b < R) mrow[b] = uint8_t(mword >> (8 * b));
      }
    }
    if (img != nullptr) {
      // row pair (p, p + 8), p = crow with bit 3 cleared; even q writes the
      // half for columns r0..r0+15 of Wt, odd q the half for r0+16..r0+31
      const int64_t prow = crow & ~int64_t(8);
      const uint32_t L = uint32_t(prow & 7) + 8u * uint32_t(q & 1) + 16u * uint32_t((prow & 127) >> 4);
      uint8_t* blk = img + ((prow >> 7) * (Rp / 128) + (r0 >> 7)) * 2048;
      __stcs(reinterpret_cast<uint32_t*>(blk + L * 16u + uint32_t((r0 & 127) >> 5) * 4u), iword);
    }
  }
  if (invalid_groups != nullptr) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) invalid += __shfl_xor_sync(0xFFFFFFFFu, invalid, off);
    if (lane == 0 && invalid != 0) atomicAdd(invalid_groups, invalid);
  }
}

int tile_grid(int64_t R, int64_t C) {
  const int64_t tiles = ((R + 127) / 128) * ((C + 127) / 128);
  const int64_t want = int64_t(sm_count()) * 8;
  return int(tiles < want ? tiles : want);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda at link time)
using TensorMapEncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                       const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                       CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
TensorMapEncodeFn tensor_map_encoder() {
  static TensorMapEncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<TensorMapEncodeFn>(ptr);
  });
  return fn;
}

// The staged fused compressor (compress_ring_kernel) from this many weights
// on.  Measured on bf16 (the row kernel -> staged): 28672 x 8192, 133.1 ->
// 125.0 us; 14336 x 4096 and 4096 x 14336, 36.9 -> 38.9 us (12 tiles a CTA:
// the ring's fill and the uneven last tiles cost more than it saves); 4096^2
// no better.
constexpr int64_t kCRingMinWeights = int64_t(1) << 27;

// true when it launched the staged fused compressor (16-bit W, C % 256 == 0,
// 16-byte aligned rows); false leaves the call to the row kernel
bool launch_compress_ring(const uint16_t* w, int64_t ldw, int64_t R, int64_t C, uint16_t* v, uint8_t* meta,
                          uint8_t* img, cudaStream_t s) {
  if (C % kCRingCols != 0 || R * C < kCRingMinWeights || !aligned16(w) || !stride_ok(ldw, 2)) return false;
  TensorMapEncodeFn enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  CUtensorMap map;
  const cuuint64_t dims[2] = {cuuint64_t(C), cuuint64_t(R)};
  const cuuint64_t strides[1] = {cuuint64_t(ldw) * 2};
  const cuuint32_t box[2] = {64, cuuint32_t(kCRingRows)};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t*>(w), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(compress_ring_kernel), kCRingSmem) != NM_OK) return false;
  static const int per_sm = blocks_per_sm(compress_ring_kernel, 256, kCRingSmem);
  const int64_t tiles = ((R + 127) / 128) * (128 / kCRingRows) * (C / kCRingCols);
  const int64_t cap = int64_t(sm_count()) * (per_sm > 0 ? per_sm : 1);
  const unsigned grid = unsigned(tiles < cap ? tiles : cap);
  compress_ring_kernel<<<grid, 256, kCRingSmem, s>>>(map, R, C, v, meta, img, device_status_word());
  return true;
}

// Compressing launch: the row-streaming kernel when C % 32 == 0 (x over the
// padded units of a row, y over padded row pairs, as many blocks as the SMs
// hold at once), else the tile kernel; selection by magnitude on 16-bit
// weights with C % 256 == 0 takes the staged fused compressor instead.
template <typename Bits, int MODE>
void launch_compress(const void* W, int64_t ldw, const uint8_t* mask, int64_t ldm, int64_t R, int64_t C,
                     void* values, uint8_t* meta, uint8_t* img, int32_t* invalid_groups, cudaStream_t s) {
  const Bits* w = static_cast<const Bits*>(W);
  Bits* v = static_cast<Bits*>(values);
  if constexpr (MODE == 0 && sizeof(Bits) == 2) {
    if (launch_compress_ring(w, ldw, R, C, v, meta, img, s)) return;
  }
  if (C % 32 != 0) {
    compress_tiles_kernel<Bits, MODE><<<tile_grid(R, C), kThreads, 0, s>>>(w, ldw, mask, ldm, R, C, v, meta, img,
                                                                           invalid_groups);
    return;
  }
  constexpr bool kHasSmall = MODE == 0 && sizeof(Bits) >= 2;
  const bool small = kHasSmall && R * C < (int64_t(1) << 25);
  static const int per_sm_big = blocks_per_sm(compress_rows_kernel<Bits, MODE>, 256);
  int per_sm = per_sm_big;
  if constexpr (kHasSmall) {
    static const int per_sm_small = blocks_per_sm(compress_rows_kernel<Bits, MODE, 3>, 256);
    if (small) per_sm = per_sm_small;
  }
  const int64_t units = ((C + 127) / 128) * 4, pairs = ((R + 127) / 128) * 64;
  const int bx = row_block_x(units);
  const int by = 256 / bx;
  const int64_t gx = (units + bx - 1) / bx;
  const int64_t cap = int64_t(per_sm) * sm_count();
  int64_t gy = (pairs + by - 1) / by;
  const int64_t cap_y = gx >= cap ? 1 : cap / gx;
  if (gy > cap_y) gy = cap_y;
  if (gy > 65535) gy = 65535;
  dim3 grid(unsigned(gx > 2147483647 ? 2147483647 : gx), unsigned(gy < 1 ? 1 : gy)), block(bx, by);
  if constexpr (kHasSmall) {
    if (small) {
      compress_rows_kernel<Bits, MODE, 3><<<grid, block, 0, s>>>(w, ldw, mask, ldm, R, C, v, meta, img,
                                                                 invalid_groups);
      return;
    }
  }
  compress_rows_kernel<Bits, MODE><<<grid, block, 0, s>>>(w, ldw, mask, ldm, R, C, v, meta, img, invalid_groups);
}

nm_status check_common(const void* W, nm_dtype dtype, int64_t R, int64_t C, int64_t ldw) {
  if (!dtype_ok_int8(dtype)) return NM_ERR_DTYPE;
  if (R < 0 || C < 0 || C % 8 != 0 || ldw < C) return NM_ERR_SHAPE;
  (void)W;
  return NM_OK;
}

}  // namespace
}  // namespace nm

using namespace nm;

extern "C" nm_status nm_mask_compress(const void* W, nm_dtype dtype, int64_t R, int64_t C, int64_t ldw,
                                      void* values, uint8_t* meta, uint8_t* meta_sm100, void* stream) {
  nm_status st = check_common(W, dtype, R, C, ldw);
  if (st != NM_OK) return st;
  if (R == 0 || C == 0) return NM_OK;
  if (W == nullptr || values == nullptr || meta == nullptr) return NM_ERR_NULL;
  if (!aligned16(W) || !aligned16(values) || !aligned16(meta) || (meta_sm100 && !aligned16(meta_sm100)) ||
      !stride_ok(ldw, esize_of(dtype)))
    return NM_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == NM_F32)
    launch_compress<uint32_t, 0>(W, ldw, nullptr, 0, R, C, values, meta, meta_sm100, nullptr, s);
  else if (dtype == NM_S8)
    launch_compress<uint8_t, 0>(W, ldw, nullptr, 0, R, C, values, meta, meta_sm100, nullptr, s);
  else
    launch_compress<uint16_t, 0>(W, ldw, nullptr, 0, R, C, values, meta, meta_sm100, nullptr, s);
  return launch_status();
}

extern "C" nm_status nm_compress(const void* W, const uint8_t* mask, nm_dtype dtype, int64_t R, int64_t C,
                                 int64_t ldw, int64_t ldm, void* values, uint8_t* meta, uint8_t* meta_sm100,
                                 int32_t* invalid_groups, void* stream) {
  nm_status st = check_common(W, dtype, R, C, ldw);
  if (st != NM_OK) return st;
  if (ldm < C) return NM_ERR_SHAPE;
  if (R == 0 || C == 0) return NM_OK;
  if (W == nullptr || mask == nullptr || values == nullptr || meta == nullptr) return NM_ERR_NULL;
  if (!aligned16(W) || !aligned16(mask) || !aligned16(values) || !aligned16(meta) ||
      (meta_sm100 && !aligned16(meta_sm100)) || !stride_ok(ldw, esize_of(dtype)) || !stride_ok(ldm, 1) ||
      (invalid_groups && (reinterpret_cast<uintptr_t>(invalid_groups) & 3u)))
    return NM_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == NM_F32)
    launch_compress<uint32_t, 1>(W, ldw, mask, ldm, R, C, values, meta, meta_sm100, invalid_groups, s);
  else if (dtype == NM_S8)
    launch_compress<uint8_t, 1>(W, ldw, mask, ldm, R, C, values, meta, meta_sm100, invalid_groups, s);
  else
    launch_compress<uint16_t, 1>(W, ldw, mask, ldm, R, C, values, meta, meta_sm100, invalid_groups, s);
  return launch_status();
}

extern "C" nm_status nm_compress_t(const void* W, const uint8_t* mask, nm_dtype dtype, int64_t R, int64_t C,
                                   int64_t ldw, int64_t ldm, void* values_t, uint8_t* meta_t, uint8_t* meta_t_sm100,
                                   int32_t* invalid_groups, void* stream) {
  if (!dtype_ok_int8(dtype)) return NM_ERR_DTYPE;
  if (R < 0 || C < 0 || R % 8 != 0 || ldw < C || ldm < C) return NM_ERR_SHAPE;
  if (R == 0 || C == 0) return NM_OK;
  if (W == nullptr || mask == nullptr || values_t == nullptr || meta_t == nullptr) return NM_ERR_NULL;
  if (!aligned16(W) || !aligned16(mask) || !aligned16(values_t) || !aligned16(meta_t) ||
      (meta_t_sm100 && !aligned16(meta_t_sm100)) || !stride_ok(ldw, esize_of(dtype)) || !stride_ok(ldm, 1) ||
      (invalid_groups && (reinterpret_cast<uintptr_t>(invalid_groups) & 3u)))
    return NM_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t blocks = (((R + 127) / 128 * 4) * ((C + 127) / 128 * 4) + 7) / 8;  // eight 32x32 tiles each
  auto launch = [&](auto kernel, auto* w, auto* v) {
    const int64_t cap = int64_t(blocks_per_sm(kernel, 256)) * sm_count();
    kernel<<<unsigned(blocks < cap ? blocks : cap), 256, 0, s>>>(w, ldw, mask, ldm, R, C, v, meta_t, meta_t_sm100,
                                                                 invalid_groups);
  };
  if (dtype == NM_F32)
    launch(compress_t_kernel<uint32_t>, static_cast<const uint32_t*>(W), static_cast<uint32_t*>(values_t));
  else if (dtype == NM_S8)
    launch(compress_t_kernel<uint8_t>, static_cast<const uint8_t*>(W), static_cast<uint8_t*>(values_t));
  else
    launch(compress_t_kernel<uint16_t>, static_cast<const uint16_t*>(W), static_cast<uint16_t*>(values_t));
  return launch_status();
}

extern "C" nm_status nm_decompress(const void* values, const uint8_t* meta, nm_dtype dtype, int64_t R, int64_t C,
                                   void* W_out, int64_t ldw, void* stream) {
  nm_status st = check_common(W_out, dtype, R, C, ldw);
  if (st != NM_OK) return st;
  if (R == 0 || C == 0) return NM_OK;
  if (values == nullptr || meta == nullptr || W_out == nullptr) return NM_ERR_NULL;
  if (!aligned16(values) || !aligned16(meta) || !aligned16(W_out) || !stride_ok(ldw, esize_of(dtype)))
    return NM_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype != NM_F32 && C % (dtype == NM_S8 ? 16 : 8) == 0 && (R * C) % 128 == 0) {
    // staged reads: a bulk-copy ring per CTA, several CTAs per SM
    const int es = esize_of(dtype);
    const int smem = kRingStages * (kRingElems / 2 * es + kRingElems / 8);
    const int64_t units = (R * C + kRingElems - 1) / kRingElems;
    auto k16 = decompress_ring_kernel<uint16_t>;
    auto k8 = decompress_ring_kernel<uint8_t>;
    const void* kp = es == 2 ? reinterpret_cast<const void*>(k16) : reinterpret_cast<const void*>(k8);
    if (ensure_dynamic_smem(kp, smem) != NM_OK) return NM_ERR_CUDA;
    const int per_sm = es == 2 ? blocks_per_sm(k16, 256, smem) : blocks_per_sm(k8, 256, smem);
    const int64_t cap = int64_t(sm_count()) * per_sm;
    const unsigned grid = unsigned(units < cap ? units : cap);
    int* status = device_status_word();
    if (es == 2)
      k16<<<grid, 256, smem, s>>>(static_cast<const uint16_t*>(values), meta, R, C, static_cast<uint16_t*>(W_out),
                                  ldw, status);
    else
      k8<<<grid, 256, smem, s>>>(static_cast<const uint8_t*>(values), meta, R, C, static_cast<uint8_t*>(W_out), ldw,
                                 status);
    return launch_status();
  }
  // x over the units of a row, y over rows
  // 32-column units for 8- and 16-bit elements; fp32 takes 8-column units,
  // whose warp stores 1 KB of a row contiguously (the 32-column form's fp32
  // stores are 16-byte pieces 128 bytes apart: 2.6 against 4.3 TB/s).
  const bool wide = (C % 32) == 0 && dtype != NM_F32;
  const int64_t opr = wide ? C / 32 : C / 8;
  const int bx = row_block_x(opr);
  const int by = 256 / bx;
  const int64_t gx = (opr + bx - 1) / bx;
  static const int per_sm_wide = blocks_per_sm(decompress32_kernel<uint16_t>, 256);
  const int64_t want = int64_t(sm_count()) * (wide ? per_sm_wide : 8);
  int64_t gy = (R + by - 1) / by;
  const int64_t cap = gx >= want ? 1 : want / gx;
  if (gy > cap) gy = cap;
  if (gy > 65535) gy = 65535;
  dim3 grid(unsigned(gx), unsigned(gy < 1 ? 1 : gy)), block(bx, by);
  if (dtype == NM_S8) {
    if (wide)
      decompress32_kernel<uint8_t><<<grid, block, 0, s>>>(static_cast<const uint8_t*>(values), meta, R, C,
                                                          static_cast<uint8_t*>(W_out), ldw);
    else
      decompress_kernel<uint8_t><<<grid, block, 0, s>>>(static_cast<const uint8_t*>(values), meta, R, C,
                                                        static_cast<uint8_t*>(W_out), ldw);
  } else if (dtype == NM_F32) {
    decompress_kernel<uint32_t><<<grid, block, 0, s>>>(static_cast<const uint32_t*>(values), meta, R, C,
                                                       static_cast<uint32_t*>(W_out), ldw);
  } else {
    if (wide)
      decompress32_kernel<uint16_t><<<grid, block, 0, s>>>(static_cast<const uint16_t*>(values), meta, R, C,
                                                           static_cast<uint16_t*>(W_out), ldw);
    else
      decompress_kernel<uint16_t><<<grid, block, 0, s>>>(static_cast<const uint16_t*>(values), meta, R, C,
                                                         static_cast<uint16_t*>(W_out), ldw);
  }
  return launch_status();
}

extern "C" nm_status nm_meta_to_sm100(const uint8_t* meta, int64_t R, int64_t C, uint8_t* meta_sm100,
                                      void* stream) {
  if (R < 0 || C < 0 || C % 8 != 0) return NM_ERR_SHAPE;
  if (R == 0 || C == 0) return NM_OK;
  if (meta == nullptr || meta_sm100 == nullptr) return NM_ERR_NULL;
  if (!aligned16(meta) || !aligned16(meta_sm100)) return NM_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (C % 128 == 0) {
    static const int per_sm = blocks_per_sm(meta_image_rows_kernel, 256);
    const int64_t warps = ((R + 127) / 128) * 8 * ((C / 128 + 3) / 4);
    const int64_t blocks = (warps + 7) / 8, cap = int64_t(per_sm) * sm_count();
    meta_image_rows_kernel<<<unsigned(blocks < cap ? blocks : cap), 256, 0, s>>>(meta, R, C, meta_sm100);
  } else {
    meta_image_kernel<<<tile_grid(R, C), kThreads, 0, s>>>(meta, R, C, meta_sm100);
  }
  return launch_status();
}

// ---------------------------------------------------------------------------
// 2:4 metadata image for the int8 sparse MMA (.kind::i8; PTX ISA, tcgen05
// sparse matrices).  An i8 instruction covers 64 logical K of a row and reads
// its 16 group fields from two 32-bit tensor-memory columns of the row's own
// lane, group g at bit 4*(g%8) of column g/8: the canonical row-major order.
// The image holds, per block of 128 rows x 128 logical columns, the 2048 bytes
// one 128-lane x 128-bit copy moves: lane L gets the 16 canonical bytes of row
// 128*rt + L for those columns.  Blocks are row-tile major with
// nk = 2 * ceil(C / 256) per row tile (the product's stage is 256 columns);
// padding holds the pattern (0,1), byte 0x44.  One thread per lane row.
namespace nm {
namespace {

__global__ void __launch_bounds__(256) meta_image_s8_kernel(const uint8_t* __restrict__ meta, int64_t R, int64_t C,
                                                            int64_t nk, int64_t nrows16, uint4* __restrict__ out) {
  const int64_t bpr = C / 8;  // canonical bytes per row
  const bool rows_vec = (bpr % 16) == 0 && (reinterpret_cast<uintptr_t>(meta) & 15u) == 0;
  for (int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; t < nrows16;
       t += int64_t(gridDim.x) * blockDim.x) {
    const int64_t blk = t >> 7;
    const int64_t rt = blk / nk, kb = blk - rt * nk;
    const int64_t r = rt * 128 + (t & 127);
    const int64_t b0 = kb * 16;
    uint4 v = make_uint4(0x44444444u, 0x44444444u, 0x44444444u, 0x44444444u);
    if (r < R && b0 < bpr) {
      const uint8_t* src = meta + r * bpr + b0;
      if (rows_vec) {
        v = __ldg(reinterpret_cast<const uint4*>(src));
      } else {
        uint8_t* vb = reinterpret_cast<uint8_t*>(&v);
        for (int j = 0; j < 16 && b0 + j < bpr; ++j) vb[j] = src[j];
      }
    }
    out[t] = v;
  }
}

}  // namespace
}  // namespace nm

extern "C" size_t nm_meta_s8_image_bytes(int64_t R, int64_t C) {
  if (R <= 0 || C <= 0) return 0;
  return size_t((R + 127) / 128) * 128 * size_t((C + 255) / 256) * 256 / 8;
}

extern "C" nm_status nm_meta_to_sm100_s8(const uint8_t* meta, int64_t R, int64_t C, uint8_t* meta_s8_sm100,
                                         void* stream) {
  using namespace nm;
  if (R < 0 || C < 0 || C % 8 != 0) return NM_ERR_SHAPE;
  if (R == 0 || C == 0) return NM_OK;
  if (meta == nullptr || meta_s8_sm100 == nullptr) return NM_ERR_NULL;
  if (!aligned16(meta_s8_sm100)) return NM_ERR_ALIGN;
  const int64_t nk = (C + 255) / 256 * 2;
  const int64_t rows16 = (R + 127) / 128 * nk * 128;
  const int64_t want = (rows16 + 255) / 256, cap = int64_t(sm_count()) * 8;
  meta_image_s8_kernel<<<unsigned(want < cap ? want : cap), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      meta, R, C, nk, rows16, reinterpret_cast<uint4*>(meta_s8_sm100));
  return launch_status();
}
