// nm_internal.cuh -- helpers shared by the libnm CUDA sources (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include "../../include/nm.h"

namespace nm {

// ----------------------------------------------------------------- host side
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool stride_ok(int64_t ld_elems, int esize) { return ((ld_elems * esize) & 15) == 0; }
inline int esize_of(nm_dtype d) { return (d == NM_F32 || d == NM_S32) ? 4 : (d == NM_S8 ? 1 : 2); }
// floating-point element types
inline bool dtype_ok(int d) { return d == NM_F32 || d == NM_BF16 || d == NM_F16; }
// ... plus int8, for the calls that only select, move and pack elements
inline bool dtype_ok_int8(int d) { return dtype_ok(d) || d == NM_S8; }

// x width of a 256-thread block laid over `units` work items of a row (y
// takes the rest of the block, over rows): the widest of 32..256 that leaves
// the fewest threads of a row's last x-block idle.  A power of two at or
// above `units` when a row has fewer than 256 items; 14336 bf16 columns in
// 16-element chunks (896) take 128, not 256, which would idle 1/8 of them.
inline int row_block_x(int64_t units) {
  int best = 32;
  int64_t best_idle = -1;
  for (int bx = 32; bx <= 256; bx *= 2) {
    const int64_t idle = (units + bx - 1) / bx * bx - units;
    if (best_idle < 0 || idle <= best_idle) {
      best = bx;
      best_idle = idle;
    }
    if (bx >= units) break;
  }
  return best;
}

inline nm_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? NM_OK : NM_ERR_CUDA;
}

// SMs of the current device, cached per device ordinal.
inline int sm_count() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  const bool cached = dev >= 0 && dev < 64;
  int n = cached ? cache[dev].load(std::memory_order_relaxed) : 0;
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      (void)cudaGetLastError();
      n = 148;
    }
    if (cached) cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Device address of the status word that bounded device-side waits write
// NM_ERR_TIMEOUT into (read and cleared by nm_last_device_status), for the
// current device; nullptr if it cannot be found.  Defined in nm_spmm.cu.
int* device_status_word();

// Raises a kernel's dynamic shared-memory limit on the current device.  The
// attribute is per device, so it is set once per (kernel, device), under a
// lock shared by every host thread.
inline nm_status ensure_dynamic_smem(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::vector<std::pair<const void*, int>> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return NM_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  for (const auto& d : done)
    if (d.first == kernel && d.second == dev) return NM_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return NM_ERR_CUDA;
  done.emplace_back(kernel, dev);
  return NM_OK;
}

// Blocks of `threads` threads of kernel k that one SM holds at once (>= 1).
template <typename Kernel>
inline int blocks_per_sm(Kernel k, int threads, size_t smem = 0) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, threads, smem) != cudaSuccess || n < 1) {
    (void)cudaGetLastError();
    n = 1;
  }
  return n;
}

// ----------------------------------------------------------------- device side
// Magnitude key: IEEE bits with the sign cleared.  Elements are handled as raw
// 16- or 32-bit patterns; no floating-point arithmetic touches them.
template <typename Bits> __device__ __forceinline__ uint32_t mag_key(Bits b);
template <> __device__ __forceinline__ uint32_t mag_key<uint32_t>(uint32_t b) { return b & 0x7FFFFFFFu; }
template <> __device__ __forceinline__ uint32_t mag_key<uint16_t>(uint16_t b) { return uint32_t(b) & 0x7FFFu; }
// int8 (two's complement): |x|, 0..128
template <> __device__ __forceinline__ uint32_t mag_key<uint8_t>(uint8_t b) {
  const int v = static_cast<int8_t>(b);
  return uint32_t(v < 0 ? -v : v);
}

// Keep-bits of one group of M keys: bit i set iff fewer than N entries beat
// entry i (j beats i: key_j > key_i, or key_j == key_i and j < i).
// Each unordered pair is compared once: for i < j exactly one beats the other.
template <int M>
__device__ __forceinline__ uint32_t keep_bits(const uint32_t (&key)[M], int N) {
  int beaten[M];
#pragma unroll
  for (int i = 0; i < M; ++i) beaten[i] = 0;
#pragma unroll
  for (int i = 0; i < M; ++i) {
#pragma unroll
    for (int j = i + 1; j < M; ++j) {
      const int jw = key[j] > key[i] ? 1 : 0;  // j beats i; otherwise i beats j
      beaten[i] += jw;
      beaten[j] += 1 - jw;
    }
  }
  uint32_t bits = 0;
#pragma unroll
  for (int i = 0; i < M; ++i) bits |= (beaten[i] < N ? 1u : 0u) << i;
  return bits;
}

// Groups of four, any N (1..3), branch-free.  For i < j let d_ij = k_i - k_j
// (keys are below 2^31, so the difference is an exact int32): its sign bit is
// set iff k_j > k_i, i.e. iff j beats i; its complement says i beats j (ties go
// to the lower index).  Entry i is beaten by 0..3 others; it is dropped when
// beaten by at least N of them, which over three 0/1 terms is an OR (N = 1), a
// majority (N = 2) or an AND (N = 3) -- one 3-input logic op per entry.
// Returns x_i whose bit 31 is set iff entry i is dropped.
template <int N>
__device__ __forceinline__ void drop4(uint32_t k0, uint32_t k1, uint32_t k2, uint32_t k3, uint32_t& x0,
                                      uint32_t& x1, uint32_t& x2, uint32_t& x3) {
  const uint32_t d01 = k0 - k1, d02 = k0 - k2, d03 = k0 - k3;
  const uint32_t d12 = k1 - k2, d13 = k1 - k3, d23 = k2 - k3;
  // terms "j beats i" for each entry
  const uint32_t a0 = d01, b0 = d02, c0 = d03;     // entry 0: beaten by 1, 2, 3
  const uint32_t a1 = ~d01, b1 = d12, c1 = d13;    // entry 1: by 0, 2, 3
  const uint32_t a2 = ~d02, b2 = ~d12, c2 = d23;   // entry 2: by 0, 1, 3
  const uint32_t a3 = ~d03, b3 = ~d13, c3 = ~d23;  // entry 3: by 0, 1, 2
  if constexpr (N == 1) {
    x0 = a0 | b0 | c0; x1 = a1 | b1 | c1; x2 = a2 | b2 | c2; x3 = a3 | b3 | c3;
  } else if constexpr (N == 2) {
    x0 = (a0 & b0) | (a0 & c0) | (b0 & c0);
    x1 = (a1 & b1) | (a1 & c1) | (b1 & c1);
    x2 = (a2 & b2) | (a2 & c2) | (b2 & c2);
    x3 = (a3 & b3) | (a3 & c3) | (b3 & c3);
  } else {
    x0 = a0 & b0 & c0; x1 = a1 & b1 & c1; x2 = a2 & b2 & c2; x3 = a3 & b3 & c3;
  }
}

// Four 0/1 mask bytes (entry i in byte i) from the drop words of drop4.
__device__ __forceinline__ uint32_t keep_bytes4(uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3) {
  const uint32_t t01 = __byte_perm(x0, x1, 0x0073);  // byte0 = x0.byte3, byte1 = x1.byte3
  const uint32_t t23 = __byte_perm(x2, x3, 0x0073);
  const uint32_t t = __byte_perm(t01, t23, 0x5410);  // the four sign bytes
  return (~t >> 7) & 0x01010101u;
}

// int8 groups of four, one group per 32-bit word (entry k in byte k), the
// magnitude |x| (0..128) and the rank rule above, in-register (SWAR):
//  - per-byte |x| without carries between bytes: (x ^ m) + s with s the sign
//    bit of each byte and m = 0xFF where negative (|-128| = 0x80 fits);
//  - the six pairwise tests k_i >= k_j (i < j, "i beats j"; false = "j beats
//    i") as three 16-bit-lane subtractions (0x100 + k_i) - k_j: bit 8 of a
//    lane is set iff k_i >= k_j, and no borrow leaves the lane;
//  - each entry's three "beaten by" terms gathered into byte lanes (A, B, C,
//    polarity fixed per byte), and dropped when at least N of them hold: an
//    OR (N = 1), a majority (N = 2) or an AND (N = 3) of three 0/1 bytes.
// Returns the keep bytes (0/1 per byte) of the group.
template <int N>
__device__ __forceinline__ uint32_t keep4_s8(uint32_t w) {
  const uint32_t sgn = (w >> 7) & 0x01010101u;
  const uint32_t a = (w ^ (sgn * 0xFFu)) + sgn;                               // |x| per byte
  const uint32_t G = 0x01010101u;
  const uint32_t d1 = __byte_perm(a, G, 0x4240) - __byte_perm(a, 0u, 0x4341);  // t01 (byte 1), t23 (byte 3)
  const uint32_t x01 = __byte_perm(a, G, 0x4140);
  const uint32_t d2 = x01 - __byte_perm(a, 0u, 0x4342);                       // t02, t13
  const uint32_t d3 = x01 - __byte_perm(a, 0u, 0x4243);                       // t03, t12
  const uint32_t A = __byte_perm(__byte_perm(d1, d2, 0x0511), d3, 0x5210) ^ 0x00000001u;  // t01 t01 t02 t03
  const uint32_t B = __byte_perm(d2, d3, 0x3771) ^ 0x00000101u;                           // t02 t12 t12 t13
  const uint32_t C = __byte_perm(__byte_perm(d3, d2, 0x0071), d1, 0x7710) ^ 0x00010101u;  // t03 t13 t23 t23
  uint32_t drop;
  if constexpr (N == 1) drop = A | B | C;
  else if constexpr (N == 2) drop = (A & B) | (A & C) | (B & C);
  else drop = A & B & C;
  return drop ^ 0x01010101u;
}

// 2:4 specialisation: the two kept indices (ascending) of a group and the
// 4-bit metadata field idx0 | idx1 << 2.
struct Pick24 {
  uint32_t nib;   // idx0 | idx1 << 2
  uint32_t i0, i1;
};

__device__ __forceinline__ Pick24 pick24(uint32_t k0, uint32_t k1, uint32_t k2, uint32_t k3) {
  const uint32_t key[4] = {k0, k1, k2, k3};
  const uint32_t b = keep_bits<4>(key, 2);
  Pick24 p;
  p.i0 = __ffs(b) - 1;             // lowest set bit
  p.i1 = 31 - __clz(b);            // highest set bit
  p.nib = p.i0 | (p.i1 << 2);
  return p;
}

template <typename Bits>
__device__ __forceinline__ Bits sel4(Bits w0, Bits w1, Bits w2, Bits w3, uint32_t i) {
  Bits a = (i & 1) ? w1 : w0;
  Bits b = (i & 1) ? w3 : w2;
  return (i & 2) ? b : a;
}

// Tensor-core metadata image: byte offset of the 16-bit piece that holds the
// four group fields of row r, logical columns [c, c+16) with c % 16 == 0,
// inside its 2048-byte block (see nm.h).
__device__ __forceinline__ uint32_t sm100_piece_offset(uint32_t r, uint32_t c) {
  const uint32_t rr = r & 127u, cc = c & 127u;
  const uint32_t lane = (rr & 7u) + 8u * ((cc & 31u) >> 4) + 16u * (rr >> 4);
  const uint32_t slice = cc >> 5;
  return lane * 16u + slice * 4u + 2u * ((rr >> 3) & 1u);
}

}  // namespace nm
