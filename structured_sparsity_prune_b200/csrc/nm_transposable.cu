// nm_transposable.cu -- transposable N:M mask, greedy, one M x M block per thread.
//
// Page: nubint.ai review of "Accelerated Sparse Neural Training: A Provable
// and Efficient Method to Find N:M Transposable Masks".  In every M x M block
// the mask should keep as much |w| as possible with at most N kept entries in
// each row and in each column, so that W and its transpose are both N:M; the
// page names an exact min-cost flow and a fast greedy 2-approximation.  This
// is the greedy: entries by decreasing magnitude (ties in row-major order
// within the block), an entry kept when its row and its column each hold
// fewer than N kept entries.
//
// Each thread owns one block.  It packs every entry's magnitude key with its
// inverted in-block position into one unsigned word (larger |w| first, then
// lower position), sorts the block with Batcher's odd-even merge network
// (K. E. Batcher, "Sorting networks and their applications", AFIPS 1968;
// 543 comparators for 64 keys, each an unsigned max and min; fully unrolled,
// registers only), then walks the sorted entries once with the row and column
// counts in 4-bit fields.  The work per weight is a few dozen integer ops, so
// the kernel is bound by the integer pipe rather than by HBM.
#include "nm_internal.cuh"

#include <utility>

namespace nm {
namespace {

__host__ __device__ constexpr int pow2_at_least(int x) { return x <= 1 ? 1 : 2 * pow2_at_least((x + 1) / 2); }

__device__ __forceinline__ void cas_desc(uint32_t& x, uint32_t& y) {
  const uint32_t hi = max(x, y), lo = min(x, y);
  x = hi;
  y = lo;
}
__device__ __forceinline__ void cas_desc(unsigned long long& x, unsigned long long& y) {
  const unsigned long long hi = x > y ? x : y, lo = x > y ? y : x;
  x = hi;
  y = lo;
}

// Batcher's odd-even merge network for P keys (P a power of two, <= 64), as
// a compile-time list of comparators (lo, hi): after all of them, in order,
// have put the larger of a[lo], a[hi] into a[lo], a is in descending order.
struct SortNet {
  int n;
  unsigned char lo[544], hi[544];
};

__host__ __device__ constexpr SortNet make_sort_net(int P) {
  SortNet net{};
  net.n = 0;
  for (int p = 1; p < P; p <<= 1)
    for (int k = p; k >= 1; k >>= 1)
      for (int j = k % p; j + k < P; j += 2 * k)
        for (int i = 0; i < k && i + j + k < P; ++i)
          if ((i + j) / (2 * p) == (i + j + k) / (2 * p)) {
            net.lo[net.n] = static_cast<unsigned char>(i + j);
            net.hi[net.n] = static_cast<unsigned char>(i + j + k);
            ++net.n;
          }
  return net;
}

template <int P> struct SortNetOf {
  static constexpr SortNet net = make_sort_net(P);
};

template <typename K, int P, int... I>
__device__ __forceinline__ void apply_net(K (&a)[P], std::integer_sequence<int, I...>) {
  (cas_desc(a[SortNetOf<P>::net.lo[I]], a[SortNetOf<P>::net.hi[I]]), ...);
}

// Sort P packed keys into descending order.
template <typename K, int P>
__device__ __forceinline__ void sort_desc(K (&a)[P]) {
  apply_net<K, P>(a, std::make_integer_sequence<int, SortNetOf<P>::net.n>{});
}

// Entry key: (magnitude + 1) above 6 bits of (63 - position); position is
// 8 * row + column inside the block, which orders like row-major for M <= 8.
// Padding entries are 0 and sort after every real entry.
template <typename Bits> struct TKey;
template <> struct TKey<uint16_t> {
  using K = uint32_t;
  __device__ static K make(uint16_t bits, int pos) {
    return ((uint32_t(bits & 0x7FFFu) + 1u) << 6) | uint32_t(63 - pos);
  }
};
template <> struct TKey<uint8_t> {
  using K = uint32_t;
  __device__ static K make(uint8_t bits, int pos) { return ((mag_key<uint8_t>(bits) + 1u) << 6) | uint32_t(63 - pos); }
};
template <> struct TKey<uint32_t> {
  using K = unsigned long long;
  __device__ static K make(uint32_t bits, int pos) {
    return ((static_cast<K>(bits & 0x7FFFFFFFu) + 1ull) << 6) | static_cast<K>(63 - pos);
  }
};

// 4-bit fields: 8 - N for indexes < M, 8 (full) for the rest.
template <int M>
__device__ __forceinline__ uint32_t full_fields(int N) {
  uint32_t v = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) v |= (i < M ? uint32_t(8 - N) : 8u) << (4 * i);
  return v;
}

// Byte i of the result = bit i of x (x < 16).
__device__ __forceinline__ uint32_t spread4(uint32_t x) { return (x * 0x00204081u) & 0x01010101u; }

template <typename Bits, int M>
__global__ void __launch_bounds__(128) transposable_kernel(const Bits* __restrict__ W, int64_t RB, int64_t CB,
                                                           int64_t ldw, int N, uint8_t* __restrict__ mask,
                                                           int64_t ldm) {
  using TK = TKey<Bits>;
  using K = typename TK::K;
  constexpr int P = pow2_at_least(M * M);
  const int64_t br_step = int64_t(gridDim.y) * blockDim.y;
  const int64_t bc_step = int64_t(gridDim.x) * blockDim.x;
  for (int64_t br = int64_t(blockIdx.y) * blockDim.y + threadIdx.y; br < RB; br += br_step) {
    for (int64_t bc = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; bc < CB; bc += bc_step) {
      const Bits* w0 = W + (br * M) * ldw + bc * M;
      K a[P];
#pragma unroll
      for (int i = 0; i < M; ++i) {
        const Bits* wr = w0 + i * ldw;
        Bits e[M];
        if constexpr (M * sizeof(Bits) == 16) {
          *reinterpret_cast<uint4*>(e) = __ldcs(reinterpret_cast<const uint4*>(wr));
        } else if constexpr (M * sizeof(Bits) == 32) {
          reinterpret_cast<uint4*>(e)[0] = __ldcs(reinterpret_cast<const uint4*>(wr));
          reinterpret_cast<uint4*>(e)[1] = __ldcs(reinterpret_cast<const uint4*>(wr) + 1);
        } else if constexpr (M * sizeof(Bits) == 8) {
          *reinterpret_cast<uint2*>(e) = __ldcs(reinterpret_cast<const uint2*>(wr));
        } else {
#pragma unroll
          for (int j = 0; j < M; ++j) e[j] = wr[j];
        }
#pragma unroll
        for (int j = 0; j < M; ++j) a[i * M + j] = TK::make(e[j], 8 * i + j);
      }
#pragma unroll
      for (int t = M * M; t < P; ++t) a[t] = 0;
      sort_desc<K, P>(a);

      // Row and column counts in 4-bit fields that start at 8 - N, so a row
      // or column is full exactly when bit 3 of its field is set; fields of
      // indexes >= M start full.  keep: bit 8 * row + column (rows 0-3 in
      // keep_lo, 4-7 in keep_hi).
      const uint32_t init = full_fields<M>(N);
      uint32_t rowcnt = init, colcnt = init;
      uint32_t keep_lo = 0u, keep_hi = 0u;
      // In chunks of 8 sorted entries; once every row is full nothing more
      // can be kept and the remaining chunks are skipped.
      bool done = false;
#pragma unroll
      for (int t0 = 0; t0 < M * M; t0 += 8) {
        if (!done) {
#pragma unroll
          for (int t = t0; t < t0 + 8 && t < M * M; ++t) {
            const uint32_t npos = ~uint32_t(a[t]);                   // low 6 bits: the position
            const uint32_t rsh = (npos >> 1) & 0x1Cu;                 // 4 * row
            const uint32_t csh = (npos << 2) & 0x1Cu;                 // 4 * column
            const bool take = (((rowcnt >> rsh) | (colcnt >> csh)) & 8u) == 0u;
            const uint32_t bit = 1u << (npos & 31u);
            const bool high = (npos & 32u) != 0u;
            rowcnt += take ? (1u << rsh) : 0u;
            colcnt += take ? (1u << csh) : 0u;
            keep_lo |= (take && !high) ? bit : 0u;
            keep_hi |= (take && high) ? bit : 0u;
          }
          done = rowcnt == 0x88888888u;
        }
      }
      const unsigned long long keep = (static_cast<unsigned long long>(keep_hi) << 32) | keep_lo;

#pragma unroll
      for (int i = 0; i < M; ++i) {
        uint8_t* mr = mask + (br * M + i) * ldm + bc * M;
        const uint32_t bits = uint32_t(keep >> (8 * i)) & 0xFFu;
        if constexpr (M == 8) {
          *reinterpret_cast<uint2*>(mr) = make_uint2(spread4(bits & 15u), spread4(bits >> 4));
        } else if constexpr (M == 4) {
          *reinterpret_cast<uint32_t*>(mr) = spread4(bits);
        } else {
#pragma unroll
          for (int j = 0; j < M; ++j) mr[j] = uint8_t((bits >> j) & 1u);
        }
      }
    }
  }
}

void shape_blocks(int64_t RB, int64_t CB, dim3& grid, dim3& block) {
  int bx = 32;
  while (bx < 128 && bx < CB) bx *= 2;
  const int by = 128 / bx;
  const int64_t gx = (CB + bx - 1) / bx;
  const int64_t want = int64_t(sm_count()) * 12;
  int64_t gy = (RB + by - 1) / by;
  const int64_t cap_y = gx >= want ? 1 : want / gx;
  if (gy > cap_y) gy = cap_y;
  if (gy > 65535) gy = 65535;
  grid = dim3(unsigned(gx > 2147483647 ? 2147483647 : gx), unsigned(gy < 1 ? 1 : gy), 1);
  block = dim3(bx, by, 1);
}

template <typename Bits, int M>
void launch_transposable(const void* W, int64_t R, int64_t C, int64_t ldw, int N, uint8_t* mask, int64_t ldm,
                         cudaStream_t s) {
  dim3 grid, block;
  shape_blocks(R / M, C / M, grid, block);
  transposable_kernel<Bits, M><<<grid, block, 0, s>>>(static_cast<const Bits*>(W), R / M, C / M, ldw, N, mask, ldm);
}

template <typename Bits>
void dispatch_transposable(const void* W, int64_t R, int64_t C, int64_t ldw, int N, int M, uint8_t* mask,
                           int64_t ldm, cudaStream_t s) {
  switch (M) {
    case 2: launch_transposable<Bits, 2>(W, R, C, ldw, N, mask, ldm, s); break;
    case 3: launch_transposable<Bits, 3>(W, R, C, ldw, N, mask, ldm, s); break;
    case 4: launch_transposable<Bits, 4>(W, R, C, ldw, N, mask, ldm, s); break;
    case 5: launch_transposable<Bits, 5>(W, R, C, ldw, N, mask, ldm, s); break;
    case 6: launch_transposable<Bits, 6>(W, R, C, ldw, N, mask, ldm, s); break;
    case 7: launch_transposable<Bits, 7>(W, R, C, ldw, N, mask, ldm, s); break;
    default: launch_transposable<Bits, 8>(W, R, C, ldw, N, mask, ldm, s); break;
  }
}

}  // namespace
}  // namespace nm

extern "C" nm_status nm_mask_transposable(const void* W, nm_dtype dtype, int64_t R, int64_t C, int64_t ldw, int N,
                                          int M, uint8_t* mask, int64_t ldm, void* stream) {
  using namespace nm;
  if (!dtype_ok_int8(dtype)) return NM_ERR_DTYPE;
  if (M < 2 || M > 8 || N < 1 || N >= M) return NM_ERR_NM;
  if (R < 0 || C < 0 || R % M != 0 || C % M != 0 || ldw < C || ldm < C) return NM_ERR_SHAPE;
  if (R == 0 || C == 0) return NM_OK;
  if (W == nullptr || mask == nullptr) return NM_ERR_NULL;
  const int es = esize_of(dtype);
  if (!aligned16(W) || !aligned16(mask) || !stride_ok(ldw, es) || !stride_ok(ldm, 1)) return NM_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == NM_F32)
    dispatch_transposable<uint32_t>(W, R, C, ldw, N, M, mask, ldm, s);
  else if (dtype == NM_S8)
    dispatch_transposable<uint8_t>(W, R, C, ldw, N, M, mask, ldm, s);
  else
    dispatch_transposable<uint16_t>(W, R, C, ldw, N, M, mask, ldm, s);
  return launch_status();
}
