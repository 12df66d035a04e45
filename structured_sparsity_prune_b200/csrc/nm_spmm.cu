// nm_spmm.cu -- Y = alpha * (W (.) mask) X + beta * Y on sm_100a sparse
// tensor cores (tcgen05.mma.sp, .kind::f16, fp32 accumulation in TMEM).
//
// Pages: review of "Accelerating Sparse Deep Neural Networks", "Structured
// sparse GEMM on tensor cores" -- sparse matrix x dense matrix = dense matrix,
// only the kept values are multiplied, and the application hands the first
// operand over in compressed 2:4 form.  The Ampere design described there is
// prior art; this kernel is written for the Blackwell execution model:
//
//  * one CTA per SM (persistent), a 128-row x N_TILE-column output tile;
//  * warp 0 (one lane): TMA producer.  Per K-stage of 128 logical columns it
//    loads the compressed A tile (128 x 64 values, 128B swizzle), the X tile
//    (128 rows of K x N_TILE, 128B swizzle, N-contiguous) and the 2048-byte
//    metadata image block (one bulk copy) into a ring of STAGES slots;
//  * warp 1 (one lane): copies the stage's metadata into tensor memory
//    (tcgen05.cp 128x128b) and issues four 128 x N_TILE x 32 sparse MMAs
//    into the TMEM accumulator; tcgen05.commit frees the stage;
//  * warps 2-5: epilogue.  tcgen05.ld the accumulator (32 columns at a
//    time), apply alpha / beta in fp32, round to the output type and store.
//    With two accumulator buffers the epilogue of tile i overlaps the MMAs of
//    tile i+1.
//
// Every mbarrier wait is bounded by a wall-clock limit; on expiry the kernel
// records NM_ERR_TIMEOUT in the device status word, raises a CTA-wide abort
// flag so the other roles stop waiting, drains what it issued, frees its
// tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdlib>
#include <mutex>
#include <cstring>
#include <string>

#include "../../include/nm_testing.h"
#include "nm_internal.cuh"

namespace nm {

// Device word written by kernels whose bounded waits give up (NM_ERR_TIMEOUT).
__device__ int g_device_status = 0;

// Its device address per device, looked up once (kernels of other source
// files take it as an argument).
int* device_status_word() {
  static std::mutex mu;
  static int* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) {
      (void)cudaGetLastError();
      return nullptr;
    }
    addr[dev] = static_cast<int*>(p);
  }
  return addr[dev];
}

namespace spmm {

constexpr int kBlockM = 128;     // rows of W per tile = TMEM lanes

// Operand kinds of the sparse MMA.  Every kind moves 128 bytes of compressed
// A per row per pipeline stage and 32 bytes per instruction, so the A tile,
// its swizzle and its descriptor walk are shared; what differs is the logical
// K those bytes cover, the instruction's kind and formats, and the metadata:
//   F16 / BF16  2:4, 16-bit, 32 logical K per MMA, one 2 KB image block per
//               stage (.kind::f16, one tensor-memory column per MMA);
//   TF32        1:2, 32-bit, 16 logical K per MMA, one 2 KB block per stage
//               (.kind::tf32: the .kind::f16 layout over 16-bit halves);
//   S8          2:4, int8, 64 logical K per MMA, two 2 KB blocks per stage
//               (.kind::i8: two columns per MMA, canonical row order);
//               s32 accumulation.
enum class Kind : int { F16 = 0, BF16 = 1, TF32 = 2, S8 = 3 };

template <Kind KD>
struct KT {
  static constexpr int kEsize = KD == Kind::TF32 ? 4 : KD == Kind::S8 ? 1 : 2;
  static constexpr int kStageK = KD == Kind::TF32 ? 64 : KD == Kind::S8 ? 256 : 128;  // logical K per stage
  static constexpr int kMmaK = kStageK / 4;            // logical K per instruction (4 per stage)
  static constexpr int kStageKPhys = 128 / kEsize;     // compressed values per row per stage (128 B)
  static constexpr int kAtomCols = 128 / kEsize;       // X columns in one 128-byte swizzle row
  static constexpr int kEBytes = KD == Kind::S8 ? 4096 : 2048;  // metadata image bytes per stage
  static constexpr int kECols = kEBytes / 512;         // tensor-memory columns they fill (128 lanes x 4 B)
  static constexpr bool kAccS32 = KD == Kind::S8;
  // X (the MN-major B operand) of a tf32 instruction must sit in the 128-byte
  // swizzle with 32-byte atoms (rows of 128 bytes, 32-byte granules XORed with
  // the row index mod 4, so the pattern repeats every 4 rows): descriptor
  // layout type 1, TMA swizzle 128B_ATOM_32B.  The other kinds use the usual
  // swizzles with 16-byte granules.
  static constexpr bool kB32Atom = KD == Kind::TF32;
};
constexpr int kThreads = 192;    // 6 warps (single-CTA kernel)
constexpr int kPairThreads = 320;  // 10 warps: producer, MMA, 8 epilogue warps (CTA-pair kernel)
constexpr int kMaxPeers = 8;       // destination GPUs of the peer-store product
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far above any legitimate wait

// ----------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: true when the phase completed, false on timeout or abort.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicExch(&g_device_status, int(NM_ERR_TIMEOUT));
      return false;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Pull a tensor map (a __grid_constant__ kernel parameter) into the TMA unit's
// descriptor cache ahead of its first use.
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Shared-memory matrix descriptor (tcgen05): start, leading / stride byte
// offsets (16-byte units), version 1, layout type in bits 61..63.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  uint64_t d = 0;
  d |= uint64_t((saddr >> 4) & 0x3FFFu);
  d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(layout & 7u) << 61;
  return d;
}
constexpr uint32_t kLayoutNone = 0, kLayoutSW128_32B = 1, kLayoutSW128 = 2, kLayoutSW64 = 4, kLayoutSW32 = 6;

__device__ __forceinline__ void tmem_cp_128x128b(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

template <Kind KD>
__device__ __forceinline__ void mma_sp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t e_tmem,
                                       uint32_t idesc, uint32_t accumulate) {
  if constexpr (KD == Kind::TF32) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "tcgen05.mma.sp.cta_group::1.kind::tf32 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(e_tmem), "r"(idesc), "r"(accumulate)
        : "memory");
  } else if constexpr (KD == Kind::S8) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "tcgen05.mma.sp.cta_group::1.kind::i8 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(e_tmem), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "tcgen05.mma.sp.cta_group::1.kind::f16 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(e_tmem), "r"(idesc), "r"(accumulate)
        : "memory");
  }
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---- CTA-pair (cluster of 2) helpers for the cta_group::2 kernel
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// shared::cluster address of the same shared-memory object in CTA `rank`
__device__ __forceinline__ uint32_t mapa(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on an mbarrier of either CTA of the pair (the epilogue releasing the
// accumulator to the even CTA's MMA issuer).  What it orders is tensor memory:
// the thread's tcgen05.ld have completed (tcgen05.wait::ld) and are ordered
// before this arrive by tcgen05.fence::before_thread_sync, and the issuer
// orders its next MMAs after its wait with tcgen05.fence::after_thread_sync.
// So the arrive carries the default CTA-scope release.  With a cluster-scope
// release the MMA issuer saw the accumulator free ~1.4 us after the last
// epilogue warp reached its arrive, on every 256 x 256 tile; with this one
// the 4096-deep products run 1-4 % faster.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// TMA tile load into this CTA's shared memory whose completion is counted on
// an mbarrier of either CTA of the pair (here: the MMA-issuing CTA's).
// Output staging: a shared-memory tile written by the generic proxy and
// stored to global memory by the bulk (async) proxy.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// the bulk stores committed by this thread have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// ... and have completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int x,
                                                 int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tmem_cp_pair_128x128b(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.128x128b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

template <Kind KD>
__device__ __forceinline__ void mma_sp_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t e_tmem,
                                            uint32_t idesc, uint32_t accumulate) {
  if constexpr (KD == Kind::TF32) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "tcgen05.mma.sp.cta_group::2.kind::tf32 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(e_tmem), "r"(idesc), "r"(accumulate)
        : "memory");
  } else if constexpr (KD == Kind::S8) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "tcgen05.mma.sp.cta_group::2.kind::i8 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(e_tmem), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "tcgen05.mma.sp.cta_group::2.kind::f16 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(e_tmem), "r"(idesc), "r"(accumulate)
        : "memory");
  }
}

// completion of this thread's earlier tcgen05 ops arrives on the mbarrier at
// the same offset in both CTAs of the pair
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x32_nowait(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Instruction descriptor of a sparse MMA: bit 2 sparse; bits 4-5 the
// accumulator format (1 fp32, 2 s32); bits 7-9 and 10-12 the A and B formats
// (.kind::f16: 0 f16, 1 bf16; .kind::tf32: 2; .kind::i8: 1 signed); bit 15 A
// K-major (0); bit 16 B MN-major (1: X is K x T with T contiguous); N / 8 at
// bit 17; M / 16 at bit 24.
template <Kind KD>
__host__ __device__ constexpr uint32_t make_idesc(int n, int m = kBlockM) {
  constexpr uint32_t fmt = KD == Kind::BF16 ? 1u : KD == Kind::TF32 ? 2u : KD == Kind::S8 ? 1u : 0u;
  constexpr uint32_t acc = KD == Kind::S8 ? 2u : 1u;
  return (1u << 2) | (acc << 4) | (fmt << 7) | (fmt << 10) | (0u << 15) | (1u << 16) |
         (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}

// Metadata operand of instruction k2 (0..3) of a stage whose metadata starts
// at tensor-memory column e_tmem: the column address (even) and the selector
// that goes into the descriptor's low bits.  .kind::f16 / tf32 instructions use
// one column each (an even base plus the selector); .kind::i8 ones use two.
template <Kind KD>
__device__ __forceinline__ void meta_operand(uint32_t e_tmem, int k2, uint32_t& e_col, uint32_t& sel) {
  if constexpr (KD == Kind::S8) {
    e_col = e_tmem + uint32_t(2 * k2);
    sel = 0;
  } else {
    e_col = e_tmem + uint32_t(k2 & ~1);
    sel = uint32_t(k2 & 1);
  }
}

// Accumulator word -> fp32 for the epilogue.
template <Kind KD>
__device__ __forceinline__ float acc_to_f(uint32_t v) {
  if constexpr (KT<KD>::kAccS32) return __int2float_rn(static_cast<int>(v));
  else return __uint_as_float(v);
}

// ----------------------------------------------------------------- kernel
template <int N_TILE, int STAGES, Kind KD>
struct Cfg {
  using K_ = KT<KD>;
  static constexpr int kABytes = kBlockM * 128;                // 16 KB: 128 B of compressed A per row
  // X tile: N_TILE >= one swizzle row's worth of columns -> boxes of kAtomCols
  // columns with 128-byte rows; narrower tiles use one box whose 32- or
  // 64-byte rows carry only the columns the MMA reads, with the matching swizzle.
  static constexpr int kBoxCols = N_TILE < K_::kAtomCols ? N_TILE : K_::kAtomCols;
  static constexpr int kBRowBytes = kBoxCols * K_::kEsize;      // 32, 64 or 128
  static constexpr int kBBoxes = N_TILE < K_::kAtomCols ? 1 : N_TILE / K_::kAtomCols;
  static constexpr int kBBoxBytes = K_::kStageK * kBRowBytes;
  static constexpr int kBBytes = kBBoxes * kBBoxBytes;
  static constexpr uint32_t kBLayout = K_::kB32Atom ? kLayoutSW128_32B
                                       : kBRowBytes == 128 ? kLayoutSW128 : (kBRowBytes == 64 ? kLayoutSW64 : kLayoutSW32);
  // stride between groups of K rows that one swizzle pattern spans (8 rows;
  // 4 with 32-byte atoms)
  static constexpr uint32_t kBSbo = K_::kB32Atom ? 4 * 128 : 8 * kBRowBytes;
  static constexpr int kEBytes = K_::kEBytes;
  static constexpr int kStageBytes = kABytes + kBBytes + kEBytes;
  static constexpr int kAccCols = N_TILE;
  static constexpr int kAccBufs = (2 * N_TILE + K_::kECols * STAGES <= 512) ? 2 : 1;
  static constexpr int kECol0 = kAccBufs * N_TILE;
  static constexpr int kTmemNeed = kECol0 + K_::kECols * STAGES;
  static constexpr int kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128
                                   : kTmemNeed <= 256 ? 256 : 512;
  static constexpr int kSmemBytes = STAGES * kStageBytes + 1024 /* align */ + 256 /* barriers, flags */;
  static constexpr int kChunk = N_TILE < 32 ? N_TILE : 32;      // epilogue columns per TMEM load
  static_assert(N_TILE % K_::kAtomCols == 0 || (N_TILE < K_::kAtomCols && kBRowBytes >= 32 &&
                                                (kBRowBytes & (kBRowBytes - 1)) == 0), "N_TILE");
  static_assert(N_TILE <= 256 && N_TILE >= 16, "N_TILE");
  static_assert(!K_::kB32Atom || kBRowBytes == 128, "tf32 X rows must be whole 128-byte swizzle rows");
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
  static_assert(kECol0 + K_::kECols * STAGES <= 512, "TMEM budget");
};

struct Params {
  const uint8_t* meta_img;  // tensor-core metadata image
  void* Y;
  int64_t ldy;
  int R, T, K;
  int m_tiles, n_tiles, k_blocks;
  int m_inner;  // tile order: 1 -> m fastest inside a group of `group` m-tiles, 0 -> n fastest
  int group;    // tiles of the slow operand kept together (sized so the group stays in L2)
  int y_f32;    // 1: fp32 output, 0: bf16 output (or s32, below)
  int y_s32;    // 1: the raw s32 accumulator (int8 products; alpha == 1, beta == 0)
  int y_vec;    // 1: Y and ldy allow 16-byte vector stores
  int y_tma;    // 1: bf16 output with beta == 0 leaves through staged bulk tensor stores (pair kernel)
  // Pair kernel work list: items [0, split_from) are whole tiles; the tiles
  // from split_from on are each done as two half-width items (the last,
  // partly filled wave then takes half as long).
  int split_from, num_work;
  int n_ymaps;  // output tensor maps the staged stores go through (1, or one per destination GPU)
  float alpha, beta;
  uint64_t wait_ns;  // limit of every bounded wait (kWaitLimitNs unless a test shortens it)
  int64_t skip_it;   // test hook: the producer issues nothing for this pipeline step (-1: none)
};

// Tile order.  Tiles run in groups: with m_inner, `group` consecutive m-tiles
// (rows of W) are swept across every n-tile with m fastest, so the group's
// slices of W stay in L2 while X streams through once per group; without
// m_inner the roles of W and X swap.
__device__ __forceinline__ void grouped_tile(const Params& p, int t, int& mt, int& nt) {
  if (p.m_inner) {
    const int span = p.group * p.n_tiles;
    const int g = t / span, first = g * p.group;
    const int gm = min(p.group, p.m_tiles - first);
    const int local = t - g * span;
    mt = first + local % gm;
    nt = local / gm;
  } else {
    const int span = p.group * p.m_tiles;
    const int g = t / span, first = g * p.group;
    const int gn = min(p.group, p.n_tiles - first);
    const int local = t - g * span;
    nt = first + local % gn;
    mt = local / gn;
  }
}

// Work item w of the pair kernel: its tile (mt, nt), first output column and
// whether it is a half-width item.
struct PairWork {
  int mt, nt, col0, narrow;
};
__device__ __forceinline__ PairWork pair_work(const Params& p, int w, int n_total) {
  PairWork k;
  const bool narrow = w >= p.split_from;
  const int t = narrow ? p.split_from + ((w - p.split_from) >> 1) : w;
  grouped_tile(p, t, k.mt, k.nt);
  k.narrow = narrow ? 1 : 0;
  k.col0 = k.nt * n_total + (narrow ? ((w - p.split_from) & 1) * (n_total / 2) : 0);
  return k;
}

// Epilogue of one 32-column chunk of one output row: y = alpha * acc (+ beta * y_old),
// rounded to the output type (or the raw s32 accumulator); vector stores when Y
// allows them, scalar at the T edge.
template <int CW, Kind KD>
__device__ __forceinline__ void store_chunk_n(const Params& p, int r, int col0, const uint32_t (&v)[CW]) {
  if (r < p.R && col0 < p.T) {
    const bool full_chunk = p.y_vec && col0 + CW <= p.T;
    if (KT<KD>::kAccS32 && p.y_s32) {
      uint32_t* yrow = static_cast<uint32_t*>(p.Y) + size_t(r) * p.ldy + col0;
      if (full_chunk) {
#pragma unroll
        for (int j = 0; j < CW; j += 4) *reinterpret_cast<uint4*>(yrow + j) = make_uint4(v[j], v[j + 1], v[j + 2], v[j + 3]);
      } else {
        for (int j = 0; j < CW && col0 + j < p.T; ++j) yrow[j] = v[j];
      }
      return;
    }
    float y[CW];
#pragma unroll
    for (int j = 0; j < CW; ++j) y[j] = p.alpha * acc_to_f<KD>(v[j]);
    if (p.y_f32) {
      float* yrow = static_cast<float*>(p.Y) + size_t(r) * p.ldy + col0;
      if (full_chunk) {
        if (p.beta != 0.0f) {
#pragma unroll
          for (int j = 0; j < CW; j += 4) {
            const float4 o = *reinterpret_cast<const float4*>(yrow + j);
            y[j] += p.beta * o.x; y[j + 1] += p.beta * o.y; y[j + 2] += p.beta * o.z; y[j + 3] += p.beta * o.w;
          }
        }
#pragma unroll
        for (int j = 0; j < CW; j += 4)
          *reinterpret_cast<float4*>(yrow + j) = make_float4(y[j], y[j + 1], y[j + 2], y[j + 3]);
      } else {
        for (int j = 0; j < CW && col0 + j < p.T; ++j) {
          float o = y[j];
          if (p.beta != 0.0f) o += p.beta * yrow[j];
          yrow[j] = o;
        }
      }
    } else {
      __nv_bfloat16* yrow = static_cast<__nv_bfloat16*>(p.Y) + size_t(r) * p.ldy + col0;
      if (full_chunk) {
        if (p.beta != 0.0f) {
#pragma unroll
          for (int j = 0; j < CW; j += 8) {
            const uint4 o = *reinterpret_cast<const uint4*>(yrow + j);
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&o);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float2 f = __bfloat1622float2(h[u]);
              y[j + 2 * u] += p.beta * f.x;
              y[j + 2 * u + 1] += p.beta * f.y;
            }
          }
        }
#pragma unroll
        for (int j = 0; j < CW; j += 8) {
          uint4 o;
          __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
          for (int u = 0; u < 4; ++u) h[u] = __floats2bfloat162_rn(y[j + 2 * u], y[j + 2 * u + 1]);
          *reinterpret_cast<uint4*>(yrow + j) = o;
        }
      } else {
        for (int j = 0; j < CW && col0 + j < p.T; ++j) {
          float o = y[j];
          if (p.beta != 0.0f) o += p.beta * __bfloat162float(yrow[j]);
          yrow[j] = __float2bfloat16_rn(o);
        }
      }
    }
  }
}
template <Kind KD>
__device__ __forceinline__ void store_chunk(const Params& p, int r, int col0, const uint32_t (&v)[32]) {
  store_chunk_n<32, KD>(p, r, col0, v);
}

template <int N_TILE, int STAGES, Kind KD>
__global__ void __launch_bounds__(kThreads, Cfg<N_TILE, STAGES, KD>::kSmemBytes <= 113 * 1024 ? 2 : 1)
    spmm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b, Params p) {
  using C = Cfg<N_TILE, STAGES, KD>;
  using K_ = KT<KD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::kStageBytes);
  uint64_t* full = bars;                         // [STAGES]
  uint64_t* empty = bars + STAGES;               // [STAGES]
  uint64_t* acc_full = bars + 2 * STAGES;        // [2]
  uint64_t* acc_empty = bars + 2 * STAGES + 2;   // [2]
  uint64_t* drain = bars + 2 * STAGES + 4;       // MMA completion before TMEM release
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_tiles = p.m_tiles * p.n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&map_a);
    prefetch_tmap(&map_b);
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::kTmemCols);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  auto tile_coords = [&](int t, int& mt, int& nt) { grouped_tile(p, t, mt, nt); };

  // last round each stage's full barrier was armed in (producer lane only),
  // for the drain after an abort
  uint32_t armed_round[STAGES];
#pragma unroll
  for (int s = 0; s < STAGES; ++s) armed_round[s] = 0xFFFFFFFFu;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        int mt, nt;
        tile_coords(t, mt, nt);
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          if (int64_t(it) == p.skip_it) continue;  // test hook: this step's stage is never filled
          const int s = int(it % STAGES);
          const uint32_t round = it / STAGES;
          if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
          uint8_t* st = smem + s * C::kStageBytes;
          mbar_arrive_expect_tx(&full[s], C::kStageBytes);
          armed_round[s] = round;
          tma_load_2d(st, &map_a, &full[s], kb * K_::kStageKPhys, mt * kBlockM);
#pragma unroll
          for (int j = 0; j < C::kBBoxes; ++j)
            tma_load_2d(st + C::kABytes + j * C::kBBoxBytes, &map_b, &full[s], nt * N_TILE + K_::kAtomCols * j,
                        kb * K_::kStageK);
          const uint8_t* esrc = p.meta_img + (size_t(mt) * p.k_blocks + kb) * C::kEBytes;
          bulk_load(st + C::kABytes + C::kBBytes, esrc, C::kEBytes, &full[s]);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = make_idesc<KD>(N_TILE);
      uint32_t it = 0, local = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++local) {
        const int buf = int(local % C::kAccBufs);
        const uint32_t use = local / C::kAccBufs;
        if (!mbar_wait(&acc_empty[buf], (use & 1u) ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
        fence_after_sync();
        const uint32_t d_tmem = tmem_base + uint32_t(buf * N_TILE);
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int s = int(it % STAGES);
          const uint32_t round = it / STAGES;
          if (!mbar_wait(&full[s], round & 1u, abort_flag, p.wait_ns)) { ok = false; break; }
          fence_after_sync();
          uint8_t* st = smem + s * C::kStageBytes;
          const uint32_t a_addr = smem_u32(st);
          const uint32_t b_addr = smem_u32(st + C::kABytes);
          const uint32_t e_addr = smem_u32(st + C::kABytes + C::kBBytes);
          const uint32_t e_tmem = tmem_base + uint32_t(C::kECol0 + K_::kECols * s);
          // metadata: per 2 KB block, 128 lanes x 16 bytes, rows contiguous
          // (8-row groups 128 B apart); int8 stages carry two blocks
#pragma unroll
          for (int j = 0; j < C::kEBytes / 2048; ++j)
            tmem_cp_128x128b(e_tmem + uint32_t(4 * j), smem_desc(e_addr + uint32_t(2048 * j), 0, 128, kLayoutNone));
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2) {
            // A: K-major, 128B swizzle, rows 128 B apart, 8-row atoms 1024 B apart;
            //    32 bytes of compressed values (kMmaK logical K) further per MMA.
            const uint64_t adesc = smem_desc(a_addr + 32u * k2, 16, 1024, kLayoutSW128);
            // B: N-major, swizzled rows of kBRowBytes: atoms LBO apart, 8-row K
            //    groups SBO apart; kMmaK rows further per MMA.
            const uint64_t bdesc = smem_desc(b_addr + uint32_t(K_::kMmaK * C::kBRowBytes) * k2, C::kBBoxBytes,
                                             C::kBSbo, C::kBLayout);
            uint32_t e_col, sel;
            meta_operand<KD>(e_tmem, k2, e_col, sel);
            mma_sp<KD>(d_tmem, adesc, bdesc, e_col, idesc | sel, (kb > 0 || k2 > 0) ? 1u : 0u);
          }
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&acc_full[buf]);
      }
      // every MMA / copy this thread issued must finish before TMEM is freed
      mma_commit(drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < kWaitLimitNs) {
      }
      (void)ok;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;             // TMEM lane quarter this warp may access
    const int row_in_tile = 32 * q + lane;
    uint32_t local = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++local) {
      int mt, nt;
      tile_coords(t, mt, nt);
      const int buf = int(local % C::kAccBufs);
      const uint32_t use = local / C::kAccBufs;
      const bool ok = mbar_wait(&acc_full[buf], use & 1u, abort_flag, p.wait_ns);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;  // warp-uniform exit keeps tcgen05.ld converged
      fence_after_sync();
      const int r = mt * kBlockM + row_in_tile;
      const int c_base = nt * N_TILE;
      if constexpr (C::kChunk == 16) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem_base + (uint32_t(32 * q) << 16) + uint32_t(buf * N_TILE), v);
        store_chunk_n<16, KD>(p, r, c_base, v);
      } else {
#pragma unroll 1
        for (int c = 0; c < N_TILE; c += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tmem_base + (uint32_t(32 * q) << 16) + uint32_t(buf * N_TILE + c), v);
          store_chunk<KD>(p, r, c_base + c, v);
        }
      }
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  }

  // ---------------------------------------------------------------- teardown
  fence_before_sync();
  __syncthreads();
  // After an abort some armed stages were never consumed: their copies must
  // land before the CTA's shared memory goes away (each wait bounded).
  if (warp == 0 && lane == 0 && *abort_flag) {
    for (int s = 0; s < STAGES; ++s)
      if (armed_round[s] != 0xFFFFFFFFu) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(&full[s], armed_round[s] & 1u) && globaltimer() - t0 < 100000000ull) {
        }
      }
  }
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ----------------------------------------------------------------- CTA-pair kernel
// A cluster of two CTAs on two SMs computes a 256-row x N_TOTAL output tile with
// tcgen05.mma.sp.cta_group::2 (M = 256): each CTA stages its own 128 rows of A,
// its own metadata block and HALF of the X tile (N_TOTAL / 2 columns); the MMA
// issued by the even CTA reads both halves, so each SM's shared memory feeds
// only half of B.  Both CTAs' TMA loads complete on the even CTA's full
// barrier; the even CTA's commits arrive on both CTAs' barriers.
// Output tensor maps of the pair kernel: one over the call's Y, or, for the
// peer-store product, one per destination GPU, each over the same rows of that
// GPU's buffer. Every staged output chunk is stored through each map with the
// same coordinates, so each copy is clipped at the same R and T.
template <int NMAP>
struct YMaps {
  CUtensorMap m[NMAP];
};

template <int N_TOTAL, int STAGES, Kind KD>
struct PairCfg {
  using K_ = KT<KD>;
  static constexpr int kNHalf = N_TOTAL / 2;
  static constexpr int kABytes = kBlockM * 128;                               // 16 KB
  static constexpr int kBBoxes = (kNHalf + K_::kAtomCols - 1) / K_::kAtomCols;  // the last may be partly unused
  static constexpr int kBBoxBytes = K_::kStageK * 128;                        // 8, 16 or 32 KB
  static constexpr int kBBytes = kBBoxes * kBBoxBytes;
  static constexpr int kEBytes = K_::kEBytes;
  static constexpr int kStageBytes = kABytes + kBBytes + kEBytes;
  static constexpr int kAccBufs = (2 * N_TOTAL + K_::kECols * STAGES <= 512) ? 2 : 1;
  static constexpr int kECol0 = kAccBufs * N_TOTAL;
  static constexpr int kTmemCols = (kECol0 + K_::kECols * STAGES) <= 256 ? 256 : 512;
  // One 2 KB output slot (32 rows x 32 bf16 columns, 64-byte swizzle) per
  // epilogue warp, 1024-byte aligned after the barriers.
  static constexpr int kOutSlotBytes = 2048;
  static constexpr int kOutOff = STAGES * kStageBytes + 1024;
  static constexpr int kSmemBytes = kOutOff + 8 * kOutSlotBytes + 1024 /* base alignment */;
  // a half-width last-wave item stages one 64-column half per CTA in whole atoms
  static constexpr bool kCanSplit = N_TOTAL == 256 && K_::kAtomCols <= 64;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
  static_assert(kNHalf % 32 == 0 && N_TOTAL <= 256, "N_TOTAL");
  static_assert(kECol0 + K_::kECols * STAGES <= 512, "TMEM budget");
};

// Y4: the output is a 4-byte type (fp32 or s32); each instantiation carries
// only its own early-release epilogue, which keeps the register budget.
template <int N_TOTAL, int STAGES, Kind KD, bool Y4, int NMAP = 1>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    spmm_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                     const __grid_constant__ CUtensorMap map_e, const __grid_constant__ YMaps<NMAP> ymaps,
                     Params p) {
  const int n_ymaps = NMAP == 1 ? 1 : p.n_ymaps;
  using C = PairCfg<N_TOTAL, STAGES, KD>;
  using K_ = KT<KD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::kStageBytes);
  uint64_t* full = bars;                        // [STAGES], used in the even CTA
  uint64_t* empty = bars + STAGES;              // [STAGES], both CTAs
  uint64_t* acc_full = bars + 2 * STAGES;       // [2], both CTAs
  uint64_t* acc_empty = bars + 2 * STAGES + 2;  // [2], used in the even CTA
  uint64_t* drain = bars + 2 * STAGES + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = int(blockIdx.x >> 1), num_pairs = int(gridDim.x >> 1);
  const int num_work = p.num_work;  // m_tiles counts 256-row tiles here

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 16);  // 8 epilogue warps in each CTA
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&map_a);
    prefetch_tmap(&map_b);
    prefetch_tmap(&map_e);
    if (p.y_tma)
      for (int j = 0; j < n_ymaps; ++j) prefetch_tmap(&ymaps.m[j]);
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, C::kTmemCols);
  fence_before_sync();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive / copy
  fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  // last round each stage's full barrier was armed in (producer lane only),
  // for the drain after an abort
  uint32_t armed_round[STAGES];
#pragma unroll
  for (int s = 0; s < STAGES; ++s) armed_round[s] = 0xFFFFFFFFu;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int w = pair; w < num_work && ok; w += num_pairs) {
        const PairWork wk = pair_work(p, w, N_TOTAL);
        const int row_tile = 2 * wk.mt + int(rank);  // this CTA's 128-row tile
        // a half-width item stages 64 columns (whole atoms) per CTA
        const int b_boxes = (C::kCanSplit && wk.narrow) ? 64 / K_::kAtomCols : C::kBBoxes;
        const int b_cols = (C::kCanSplit && wk.narrow) ? 64 : C::kNHalf;
        const uint32_t tx = 2u * uint32_t(C::kABytes + b_boxes * C::kBBoxBytes + C::kEBytes);
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          if (int64_t(it) == p.skip_it) continue;  // test hook: neither CTA fills this step's stage
          const int s = int(it % STAGES);
          const uint32_t round = it / STAGES;
          if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
          uint8_t* st = smem + s * C::kStageBytes;
          if (leader) mbar_arrive_expect_tx(&full[s], tx);
          armed_round[s] = round;
          const uint32_t bar = mapa(smem_u32(&full[s]), 0);
          tma_load_2d_pair(st, &map_a, bar, kb * K_::kStageKPhys, row_tile * kBlockM);
#pragma unroll
          for (int j = 0; j < C::kBBoxes; ++j)
            if (j < b_boxes)
              tma_load_2d_pair(st + C::kABytes + j * C::kBBoxBytes, &map_b, bar,
                               wk.col0 + int(rank) * b_cols + K_::kAtomCols * j, kb * K_::kStageK);
          // the stage's image: kEBytes / 16 rows of 16 bytes
          tma_load_2d_pair(st + C::kABytes + C::kBBytes, &map_e, bar, 0,
                           (row_tile * p.k_blocks + kb) * (C::kEBytes / 16));
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && leader) {
      const uint32_t idesc_full = make_idesc<KD>(N_TOTAL, 2 * kBlockM);
      const uint32_t idesc_narrow = make_idesc<KD>(N_TOTAL / 2, 2 * kBlockM);
      uint32_t it = 0, local = 0;
      bool ok = true;
      for (int w = pair; w < num_work && ok; w += num_pairs, ++local) {
        const uint32_t idesc = w >= p.split_from ? idesc_narrow : idesc_full;
        const int buf = int(local % C::kAccBufs);
        const uint32_t use = local / C::kAccBufs;
        if (!mbar_wait(&acc_empty[buf], (use & 1u) ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
        fence_after_sync();
        const uint32_t d_tmem = tmem_base + uint32_t(buf * N_TOTAL);
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int s = int(it % STAGES);
          const uint32_t round = it / STAGES;
          if (!mbar_wait(&full[s], round & 1u, abort_flag, p.wait_ns)) { ok = false; break; }
          fence_after_sync();
          uint8_t* st = smem + s * C::kStageBytes;
          const uint32_t a_addr = smem_u32(st);
          const uint32_t b_addr = smem_u32(st + C::kABytes);
          const uint32_t e_addr = smem_u32(st + C::kABytes + C::kBBytes);
          const uint32_t e_tmem = tmem_base + uint32_t(C::kECol0 + K_::kECols * s);
#pragma unroll
          for (int j = 0; j < C::kEBytes / 2048; ++j)
            tmem_cp_pair_128x128b(e_tmem + uint32_t(4 * j),
                                  smem_desc(e_addr + uint32_t(2048 * j), 0, 128, kLayoutNone));
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2) {
            const uint64_t adesc = smem_desc(a_addr + 32u * k2, 16, 1024, kLayoutSW128);
            const uint64_t bdesc = smem_desc(b_addr + uint32_t(K_::kMmaK * 128) * k2, C::kBBoxBytes,
                                             K_::kB32Atom ? 512u : 1024u, K_::kB32Atom ? kLayoutSW128_32B : kLayoutSW128);
            uint32_t e_col, sel;
            meta_operand<KD>(e_tmem, k2, e_col, sel);
            mma_sp_pair<KD>(d_tmem, adesc, bdesc, e_col, idesc | sel, (kb > 0 || k2 > 0) ? 1u : 0u);
          }
          mma_commit_pair(&empty[s]);
        }
        if (!ok) break;
        mma_commit_pair(&acc_full[buf]);
      }
      asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                       smem_u32(drain))
                   : "memory");
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < kWaitLimitNs) {
      }
      (void)ok;
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    // Warps 2..9: warp w reads TMEM lanes 32*(w%4).. (its rows) and columns
    // [half * N/2, (half+1) * N/2) with half = (w-2)/4.  For bf16 output with
    // beta == 0 a thread converts its whole row segment into registers first
    // and releases the accumulator before storing, so the next tile's MMAs
    // overlap the global stores.
    constexpr int kCols = N_TOTAL / 2;
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row_in_tile = 32 * q + lane;
    const uint32_t acc_empty_leader[2] = {mapa(smem_u32(&acc_empty[0]), 0), mapa(smem_u32(&acc_empty[1]), 0)};
    const bool early = !Y4 && p.beta == 0.0f && p.y_vec;
    // 4-byte outputs (fp32, s32) without beta: the same early release and
    // staged bulk stores, in 32-row x 16-column chunks
    const bool early4 = Y4 && p.beta == 0.0f && p.y_vec && p.y_tma;
    const uint32_t out_slot = smem_u32(smem + C::kOutOff + (warp - 2) * C::kOutSlotBytes);
    uint32_t local = 0;
    for (int w = pair; w < num_work; w += num_pairs, ++local) {
      const PairWork wk = pair_work(p, w, N_TOTAL);
      const int mt = wk.mt;
      // columns of this warp: kc of them (kCols, or half that for a half-width
      // item); loops below run to kCols with steps past kc skipped, so the
      // register arrays keep compile-time indexes
      const int kc = wk.narrow ? kCols / 2 : kCols;
      const int buf = int(local % C::kAccBufs);
      const uint32_t use = local / C::kAccBufs;
      const bool ok = mbar_wait(&acc_full[buf], use & 1u, abort_flag, p.wait_ns);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      fence_after_sync();
      const int r = (2 * mt + int(rank)) * kBlockM + row_in_tile;
      const int c_base = wk.col0 + half * kc;
      const uint32_t taddr = tmem_base + (uint32_t(32 * q) << 16) + uint32_t(buf * N_TOTAL + half * kc);
      if (early4) {
        uint32_t v[kCols];
#pragma unroll
        for (int c = 0; c < kCols; c += 32)
          if (c < kc) tmem_ld_32x32b_x32_nowait(taddr + uint32_t(c), *reinterpret_cast<uint32_t(*)[32]>(&v[c]));
        tmem_ld_wait();
        fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(acc_empty_leader[buf]);
        if (p.y_f32) {
#pragma unroll
          for (int j = 0; j < kCols; ++j) v[j] = __float_as_uint(p.alpha * acc_to_f<KD>(v[j]));
        }
        const uint32_t slot = out_slot + uint32_t(lane) * 64u;
        const uint32_t sw = (uint32_t(lane) >> 1) & 3u;
        const int row0 = (2 * mt + int(rank)) * kBlockM + 32 * q;
#pragma unroll
        for (int c = 0; c < kCols; c += 16) {
          if (c >= kc) break;
          if (lane == 0) bulk_wait_read_all();  // the slot's previous store has read it
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 4; ++j)
            st_shared_v4(slot + 16u * (uint32_t(j) ^ sw), v[c + 4 * j], v[c + 4 * j + 1], v[c + 4 * j + 2],
                         v[c + 4 * j + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && row0 < p.R && c_base + c < p.T) {  // boxes start inside Y
            for (int j = 0; j < n_ymaps; ++j)
              tma_store_2d(&ymaps.m[j], smem + C::kOutOff + (warp - 2) * C::kOutSlotBytes, c_base + c, row0);
            bulk_commit();
          }
        }
      } else if (early) {
        uint32_t packed[kCols / 2];
        {
          // the thread's whole segment in flight at once, one wait, and the
          // accumulator released before the conversion (columns past kc of a
          // half-width item are converted but never stored)
          uint32_t v[kCols];
#pragma unroll
          for (int c = 0; c < kCols; c += 32)
            if (c < kc) tmem_ld_32x32b_x32_nowait(taddr + uint32_t(c), *reinterpret_cast<uint32_t(*)[32]>(&v[c]));
          tmem_ld_wait();
          fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(acc_empty_leader[buf]);
#pragma unroll
          for (int j = 0; j < kCols / 2; ++j)
            packed[j] = pack_bf16x2(p.alpha * acc_to_f<KD>(v[2 * j]), p.alpha * acc_to_f<KD>(v[2 * j + 1]));
        }
        if (p.y_tma) {
          // 32 x 32 chunks through this warp's slot: lane = row, four 16-byte
          // pieces per row placed with the 64-byte swizzle (piece ^ ((row >> 1) & 3)),
          // so a warp's shared stores hit all 32 banks; one bulk tensor store per
          // chunk, which the tensor map clips at R and T.
          const uint32_t slot = out_slot + uint32_t(lane) * 64u;
          const uint32_t sw = (uint32_t(lane) >> 1) & 3u;
          const int row0 = (2 * mt + int(rank)) * kBlockM + 32 * q;
#pragma unroll
          for (int c = 0; c < kCols; c += 32) {
            if (c >= kc) break;
            if (lane == 0) bulk_wait_read_all();  // the slot's previous store has read it
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 4; ++j)
              st_shared_v4(slot + 16u * (uint32_t(j) ^ sw), packed[c / 2 + 4 * j], packed[c / 2 + 4 * j + 1],
                           packed[c / 2 + 4 * j + 2], packed[c / 2 + 4 * j + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && row0 < p.R && c_base + c < p.T) {  // boxes start inside Y
              for (int j = 0; j < n_ymaps; ++j)
                tma_store_2d(&ymaps.m[j], smem + C::kOutOff + (warp - 2) * C::kOutSlotBytes, c_base + c, row0);
              bulk_commit();
            }
          }
        } else if (r < p.R) {
          __nv_bfloat16* yrow = static_cast<__nv_bfloat16*>(p.Y) + size_t(r) * p.ldy;
#pragma unroll
          for (int c = 0; c < kCols; c += 8) {
            if (c >= kc) break;
            const int col = c_base + c;
            if (col + 8 <= p.T) {
              *reinterpret_cast<uint4*>(yrow + col) =
                  make_uint4(packed[c / 2], packed[c / 2 + 1], packed[c / 2 + 2], packed[c / 2 + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                if (col + j < p.T) {
                  const uint32_t w = packed[c / 2 + j / 2];
                  const uint16_t h = uint16_t((j & 1) ? (w >> 16) : (w & 0xFFFFu));
                  reinterpret_cast<uint16_t*>(yrow)[col + j] = h;
                }
              }
            }
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < kc; c += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + uint32_t(c), v);
          store_chunk<KD>(p, r, c_base + c, v);
        }
        fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(acc_empty_leader[buf]);
      }
    }
    if (lane == 0) bulk_wait_all();  // output stores complete before the CTA leaves
  }

  // ---------------------------------------------------------------- teardown
  fence_before_sync();
  __syncthreads();
  // After an abort in either CTA, copies already issued must land before the
  // pair leaves (each wait bounded).  Both CTAs' copies complete on the even
  // CTA's full barriers, which it waits on; the odd CTA, which owns none,
  // waits 2 ms; the cluster barrier below keeps both CTAs alive until then.
  if (warp == 0) {
    if (lane == 0 && *abort_flag) {
      if (leader) {
        for (int s = 0; s < STAGES; ++s)
          if (armed_round[s] != 0xFFFFFFFFu) {
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(&full[s], armed_round[s] & 1u) && globaltimer() - t0 < 100000000ull) {
            }
          }
      } else {
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 2000000ull) {
        }
      }
    }
    __syncwarp();
  }
  cluster_sync();  // the even CTA's MMAs are done and no remote arrive is pending
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc_pair(tmem_base, C::kTmemCols);
  }
}

// f32 -> f16 (round to nearest even) staging for the NM_F32 path
__global__ void f32_to_f16_kernel(const float* __restrict__ src, int64_t rows, int64_t cols, int64_t lds,
                                  __half* __restrict__ dst, int64_t ldd) {
  const int64_t n = rows * cols;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / cols, c = i - r * cols;
    dst[r * ldd + c] = __float2half_rn(src[r * lds + c]);
  }
}

// ----------------------------------------------------------------- host side
using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn get_encode() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(ptr);
  });
  return fn;
}

// TMA element type of each operand kind.
template <Kind KD>
constexpr CUtensorMapDataType tma_type() {
  return KD == Kind::BF16   ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
         : KD == Kind::F16  ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
         : KD == Kind::TF32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                            : CU_TENSOR_MAP_DATA_TYPE_UINT8;
}

CUtensorMapSwizzle swizzle_for(int row_bytes) {
  return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
         : row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
}

// 2D tile map over a row-major [rows x cols] matrix of esize-byte elements,
// box = box_cols x box_rows.
bool make_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int esize, int64_t rows, int64_t cols,
              int64_t ld_elems, int box_cols, int box_rows, CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeFn enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(ld_elems) * cuuint64_t(esize)};
  const cuuint32_t box[2] = {cuuint32_t(box_cols), cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int N_TILE, int STAGES, Kind KD>
nm_status launch(const CUtensorMap& ma, const void* X, int64_t ldx, int64_t K, int64_t T, const Params& p,
                 cudaStream_t s) {
  using C = Cfg<N_TILE, STAGES, KD>;
  CUtensorMap mb;
  if (!make_map(&mb, X, tma_type<KD>(), KT<KD>::kEsize, K, T, ldx, C::kBoxCols, KT<KD>::kStageK,
                KT<KD>::kB32Atom ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : swizzle_for(C::kBRowBytes)))
    return NM_ERR_CUDA;
  auto kern = spmm_kernel<N_TILE, STAGES, KD>;
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(kern), C::kSmemBytes) != NM_OK) return NM_ERR_CUDA;
  const int tiles = p.m_tiles * p.n_tiles;
  const int per_sm = C::kSmemBytes <= 113 * 1024 ? 2 : 1;  // two CTAs per SM when the ring is small
  const int slots = per_sm * sm_count();
  const int grid = tiles < slots ? tiles : slots;
  kern<<<grid, kThreads, C::kSmemBytes, s>>>(ma, mb, p);
  return launch_status();
}

// 2D byte map over the metadata image seen as rows of 16 bytes (one row per
// tensor-memory lane), box = one stage's image (128 or 256 rows).
bool make_map_image(CUtensorMap* map, const uint8_t* img, int64_t rows16, int box_rows) {
  EncodeFn enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {16, cuuint64_t(rows16)};
  const cuuint64_t strides[1] = {16};
  const cuuint32_t box[2] = {16, cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(img), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int N_TOTAL, int STAGES, Kind KD, int NMAP = 1>
nm_status launch_pair(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& me, const YMaps<NMAP>& my,
                      const Params& p, bool tail_split, cudaStream_t s) {
  using C = PairCfg<N_TOTAL, STAGES, KD>;
  auto kern = (p.y_f32 || p.y_s32) ? spmm_pair_kernel<N_TOTAL, STAGES, KD, true, NMAP>
                                   : spmm_pair_kernel<N_TOTAL, STAGES, KD, false, NMAP>;
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(kern), C::kSmemBytes) != NM_OK) return NM_ERR_CUDA;
  const int tiles = p.m_tiles * p.n_tiles;
  const int max_pairs = sm_count() / 2;
  const int pairs = tiles < max_pairs ? tiles : max_pairs;
  Params q = p;
  q.split_from = tiles;
  q.num_work = tiles;
  // A last wave that fills at most half of the pairs is done in half-width
  // items (whole B atoms per CTA, so only for 256-column tiles of 16- and
  // 32-bit operands).
  const int rem = tiles % pairs;
  if (C::kCanSplit && tiles > pairs && rem > 0 && 2 * rem <= pairs && tail_split) {
    q.split_from = tiles - rem;
    q.num_work = tiles + rem;
  }
  kern<<<2 * pairs, kPairThreads, C::kSmemBytes, s>>>(ma, mb, me, my, q);
  return launch_status();
}

// Kernel choice: the CTA-pair kernel when the row tiles pair up and the
// output is wide enough to fill 128+ columns; the single-CTA kernel
// otherwise.  A test or tuning caller may force one (nm_spmm_test); a forced
// choice that does not apply (a pair kernel for an odd number of row tiles)
// falls back to the default.  int8 operands have 128-column swizzle atoms, so
// their pair kernel is the 256-column one and their narrowest tile 32 columns.
enum class Kern { Pair256, Pair192, Pair128, Single256, Single128, Single64, Single64x2, Single32x2, Single16x2 };

// Options of one call: the defaults for nm_spmm, test and tuning hooks otherwise.
struct Opts {
  int kernel = 0;          // 0: the library's choice; 1..9: Kern value + 1
  bool tail_split = true;  // half-width items for a partly filled last wave
  uint64_t wait_ns = kWaitLimitNs;
  int64_t skip_it = -1;
  int raster = 0;          // 0: the library's tile order; else 1 + 2*group + m_inner (tuning)
};

template <Kind KD>
Kern choose_kernel(int64_t R, int64_t T, int forced) {
  const bool pairable = ((R + kBlockM - 1) / kBlockM) % 2 == 0;
  const bool s8 = KD == Kind::S8;
  const bool no16 = s8 || KD == Kind::TF32;  // X rows of a 16-column tile would be narrower than the swizzle
  Kern k;
  if (pairable && T > (s8 ? 128 : 64)) k = (T > 128 || s8) ? Kern::Pair256 : Kern::Pair128;
  else if (T > 128) k = Kern::Single256;
  else if (T > 64) k = Kern::Single128;
  else if (T > 32) k = Kern::Single64x2;
  else if (T > 16 || no16) k = Kern::Single32x2;
  else k = Kern::Single16x2;
  if (forced >= 1 && forced <= 9) {
    Kern f = static_cast<Kern>(forced - 1);
    if (s8 && (f == Kern::Pair192 || f == Kern::Pair128)) f = Kern::Pair256;
    if (no16 && f == Kern::Single16x2) f = Kern::Single32x2;
    const bool is_pair = f == Kern::Pair256 || f == Kern::Pair192 || f == Kern::Pair128;
    if (!is_pair || pairable) k = f;
  }
  return k;
}

// y_kind: 0 bf16, 1 fp32, 2 s32 (int8 operands only).
// peer_y / n_peers / row0 (the peer-store product): when n_peers > 0, rows
// [row0, row0 + R) of every buffer peer_y[j] (ldy elements per row) receive
// the bf16 output and Y is ignored.  Only the 256-column CTA-pair kernel with
// bulk tensor stores does this (bf16 or fp16 operands, bf16 output, beta == 0,
// 16-byte aligned rows); any other case is NM_ERR_UNSUPPORTED.
template <Kind KD>
nm_status run(const void* values, const uint8_t* meta_img, const void* X, int64_t ldx, void* Y, int y_kind,
              int64_t ldy, int64_t R, int64_t K, int64_t T, float alpha, float beta, const Opts& o, cudaStream_t s,
              void* const* peer_y = nullptr, int n_peers = 0, int64_t row0 = 0) {
  using K_ = KT<KD>;
  if (n_peers > 0) Y = static_cast<uint8_t*>(peer_y[0]) + size_t(row0) * size_t(ldy) * 2;
  Params p;
  p.n_ymaps = 1;
  p.wait_ns = o.wait_ns;
  p.skip_it = o.skip_it;
  p.y_tma = 0;
  p.meta_img = meta_img;
  p.Y = Y;
  p.ldy = ldy;
  p.R = int(R);
  p.T = int(T);
  p.K = int(K);
  p.k_blocks = int((K + K_::kStageK - 1) / K_::kStageK);
  p.y_f32 = y_kind == 1 ? 1 : 0;
  p.y_s32 = y_kind == 2 ? 1 : 0;
  p.y_vec = (aligned16(Y) && stride_ok(ldy, y_kind == 0 ? 2 : 4)) ? 1 : 0;
  p.alpha = alpha;
  p.beta = beta;
  const Kern kern = choose_kernel<KD>(R, T, o.kernel);
  const bool pair = kern == Kern::Pair256 || kern == Kern::Pair192 || kern == Kern::Pair128;
  const int block_m = pair ? 2 * kBlockM : kBlockM;
  const int n_tile = (kern == Kern::Pair256 || kern == Kern::Single256) ? 256
                     : kern == Kern::Pair192                                 ? 192
                     : (kern == Kern::Pair128 || kern == Kern::Single128) ? 128
                     : kern == Kern::Single32x2                              ? 32
                     : kern == Kern::Single16x2                              ? 16 : 64;
  p.m_tiles = int((R + block_m - 1) / block_m);
  p.n_tiles = int((T + n_tile - 1) / n_tile);
  // Tile order.  Tiles run in groups: `group` row tiles of W swept across every
  // column tile of X (m_inner), or `group` column tiles of X swept across every
  // row tile.  A group's slice of the grouped operand is sized to about 32 MB,
  // so it stays in L2 while the other operand streams past it once per group;
  // of the two orders, the one with the smaller estimated DRAM traffic (the
  // grouped operand once, the other once per group) is taken, row groups
  // within 10 %.  On the MLP up
  // product this cut DRAM reads from 661 to 316 MB; on the TF32 8192^2 x 4096
  // product the whole-row sweep had read 1117 MB.
  {
    const double a_bytes = double(R) * (double(K) * 0.5 * K_::kEsize + double(K) / 8.0);  // values + image
    const double b_bytes = double(K) * double(T) * K_::kEsize;
    const double a_tile = a_bytes / p.m_tiles, b_tile = b_bytes / p.n_tiles;
    auto groups = [](double tile, int tiles) {
      const int g = int(32.0e6 / tile + 0.5);
      return g < 1 ? 1 : (g > tiles ? tiles : g);
    };
    const int gm = groups(a_tile, p.m_tiles), gn = groups(b_tile, p.n_tiles);
    const double est_m = a_bytes + double((p.m_tiles + gm - 1) / gm) * b_bytes;
    const double est_n = b_bytes + double((p.n_tiles + gn - 1) / gn) * a_bytes;
    p.m_inner = est_m <= 1.1 * est_n ? 1 : 0;  // near-ties: row groups (measured better on the MLP up shape)
    p.group = p.m_inner ? gm : gn;
    if (o.raster > 0) {  // a forced order: `group` tiles of the fast operand, m or n fastest
      p.m_inner = (o.raster - 1) & 1;
      const int g = (o.raster - 1) >> 1;
      const int lim = p.m_inner ? p.m_tiles : p.n_tiles;
      p.group = g < 1 ? 1 : (g > lim ? lim : g);
    }
  }

  CUtensorMap ma, mb;
  if (!make_map(&ma, values, tma_type<KD>(), K_::kEsize, R, K / 2, K / 2, K_::kStageKPhys, kBlockM))
    return NM_ERR_CUDA;
  if (!make_map(&mb, X, tma_type<KD>(), K_::kEsize, K, T, ldx, K_::kAtomCols, K_::kStageK,
                K_::kB32Atom ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B))
    return NM_ERR_CUDA;
  if (pair) {
    CUtensorMap me;
    YMaps<1> my;
    constexpr int e_rows = K_::kEBytes / 16;
    const int64_t rows16 = ((R + 127) / 128) * int64_t(p.k_blocks) * e_rows;
    if (!make_map_image(&me, meta_img, rows16, e_rows)) return NM_ERR_CUDA;
    // output without beta leaves through bulk tensor stores: 32-row boxes of
    // 64-byte rows (32 bf16 or 16 fp32 / s32 columns).  Only when a row of Y
    // is whole 16-byte units: measured on B200, a bulk tensor store clips rows
    // exactly but writes the whole 16-byte unit that holds a row's last
    // column, i.e. up to 7 bf16 (3 fp32) elements past T inside ldy.  A
    // ragged T takes the plain stores, which stop at T.
    const int y_es = y_kind == 0 ? 2 : 4;
    p.y_tma = (beta == 0.0f && p.y_vec && (int64_t(T) * y_es) % 16 == 0) ? 1 : 0;
    memset(&my, 0, sizeof(my));
    if (n_peers > 0) {
      if constexpr (KD == Kind::BF16 || KD == Kind::F16) {
        if (kern != Kern::Pair256 || y_kind != 0 || !p.y_tma || n_peers > kMaxPeers) return NM_ERR_UNSUPPORTED;
        YMaps<kMaxPeers> ym;
        memset(&ym, 0, sizeof(ym));
        for (int j = 0; j < n_peers; ++j) {
          void* dst = static_cast<uint8_t*>(peer_y[j]) + size_t(row0) * size_t(ldy) * 2;
          if (!aligned16(dst)) return NM_ERR_UNSUPPORTED;
          if (!make_map(&ym.m[j], dst, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, R, T, ldy, 32, 32,
                        CU_TENSOR_MAP_SWIZZLE_64B))
            return NM_ERR_CUDA;
        }
        p.n_ymaps = n_peers;
        return launch_pair<256, 4, KD, kMaxPeers>(ma, mb, me, ym, p, o.tail_split, s);
      } else {
        return NM_ERR_UNSUPPORTED;
      }
    }
    if (p.y_tma) {
      const bool ok = y_kind == 0 ? make_map(&my.m[0], Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, R, T, ldy, 32, 32,
                                             CU_TENSOR_MAP_SWIZZLE_64B)
                                  : make_map(&my.m[0], Y, y_kind == 1 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                                                      : CU_TENSOR_MAP_DATA_TYPE_INT32,
                                             4, R, T, ldy, 16, 32, CU_TENSOR_MAP_SWIZZLE_64B);
      if (!ok) return NM_ERR_CUDA;
    }
    if constexpr (KD == Kind::S8) {
      return launch_pair<256, 4, KD>(ma, mb, me, my, p, o.tail_split, s);
    } else {
      if (kern == Kern::Pair256) return launch_pair<256, 4, KD>(ma, mb, me, my, p, o.tail_split, s);
      if (kern == Kern::Pair192) return launch_pair<192, 4, KD>(ma, mb, me, my, p, o.tail_split, s);
      return launch_pair<128, 6, KD>(ma, mb, me, my, p, o.tail_split, s);
    }
  }
  if (n_peers > 0) return NM_ERR_UNSUPPORTED;  // the single-CTA kernels store through plain pointers
  switch (kern) {
    case Kern::Single256: return launch<256, 2, KD>(ma, X, ldx, K, T, p, s);
    case Kern::Single128: return launch<128, 4, KD>(ma, X, ldx, K, T, p, s);
    case Kern::Single64x2: return launch<64, 3, KD>(ma, X, ldx, K, T, p, s);
    case Kern::Single32x2: return launch<32, (KD == Kind::S8 ? 3 : 4), KD>(ma, X, ldx, K, T, p, s);
    case Kern::Single16x2:
      if constexpr (KD == Kind::S8 || KD == Kind::TF32) return NM_ERR_UNSUPPORTED;  // never chosen (above)
      else return launch<16, 5, KD>(ma, X, ldx, K, T, p, s);
    default: return launch<64, 6, KD>(ma, X, ldx, K, T, p, s);
  }
}

}  // namespace spmm
}  // namespace nm

using namespace nm;

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

extern "C" size_t nm_spmm_workspace_bytes(nm_dtype ab_dtype, int64_t R, int64_t K, int64_t T) {
  if (ab_dtype != NM_F32 || R <= 0 || K <= 0 || T <= 0) return 0;
  const int64_t ldx_h = (T + 7) / 8 * 8;
  return align256(size_t(R) * size_t(K / 2) * 2) + align256(size_t(K) * size_t(ldx_h) * 2);
}

namespace {

// Host checks of nm_spmm's arguments other than the workspace.  NM_OK with
// *noop set means there is nothing to compute (R == 0 or T == 0).
nm_status spmm_validate(const void* values, const uint8_t* meta_sm100, nm_dtype ab_dtype, const void* X,
                        int64_t ldx, const void* Y, nm_dtype y_dtype, int64_t ldy, int64_t R, int64_t K, int64_t T,
                        float alpha, float beta, bool* noop) {
  *noop = false;
  if (!dtype_ok_int8(ab_dtype)) return NM_ERR_DTYPE;
  if (ab_dtype == NM_S8) {
    if (y_dtype != NM_BF16 && y_dtype != NM_F32 && y_dtype != NM_S32) return NM_ERR_DTYPE;
  } else if (y_dtype != NM_BF16 && y_dtype != NM_F32) {
    return NM_ERR_DTYPE;
  }
  // int8: the compressed rows (K/2 bytes) must be whole 16-byte units, the
  // pages' "multiples of 32" for INT8 sparse operands
  const int k_mult = ab_dtype == NM_S8 ? 32 : 16;
  if (R < 0 || K < 0 || T < 0 || K % k_mult != 0 || ldx < T || ldy < T) return NM_ERR_SHAPE;
  if (R > 0x7FFFFFFF - 256 || K > 0x7FFFFFFF - 256 || T > 0x7FFFFFFF - 256) return NM_ERR_SHAPE;
  if (y_dtype == NM_S32 && (alpha != 1.0f || beta != 0.0f)) return NM_ERR_UNSUPPORTED;
  if (R == 0 || T == 0) {
    *noop = true;
    return NM_OK;
  }
  if (values == nullptr || meta_sm100 == nullptr || X == nullptr || Y == nullptr) return NM_ERR_NULL;
  const int ab_es = esize_of(ab_dtype), y_es = esize_of(y_dtype);
  if (!aligned16(values) || !aligned16(meta_sm100) || !aligned16(X) || !stride_ok(ldx, ab_es) ||
      (reinterpret_cast<uintptr_t>(Y) % uintptr_t(y_es)) != 0)
    return NM_ERR_ALIGN;
  if (K == 0) return NM_ERR_SHAPE;
  return NM_OK;
}

int y_kind_of(nm_dtype y) { return y == NM_BF16 ? 0 : y == NM_F32 ? 1 : 2; }

nm_status spmm_entry(const void* values, const uint8_t* meta_sm100, nm_dtype ab_dtype, const void* X, int64_t ldx,
                     void* Y, nm_dtype y_dtype, int64_t ldy, int64_t R, int64_t K, int64_t T, float alpha, float beta,
                     void* workspace, size_t workspace_bytes, const spmm::Opts& o, void* stream) {
  bool noop = false;
  const nm_status v =
      spmm_validate(values, meta_sm100, ab_dtype, X, ldx, Y, y_dtype, ldy, R, K, T, alpha, beta, &noop);
  if (v != NM_OK || noop) return v;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int yk = y_kind_of(y_dtype);
  using spmm::Kind;
  if (ab_dtype == NM_F32) {
    const size_t need = nm_spmm_workspace_bytes(ab_dtype, R, K, T);
    if (workspace == nullptr || workspace_bytes < need) return NM_ERR_WORKSPACE;
    if (!aligned16(workspace)) return NM_ERR_ALIGN;
    const int64_t ldx_h = (T + 7) / 8 * 8;
    __half* vh = static_cast<__half*>(workspace);
    __half* xh = reinterpret_cast<__half*>(static_cast<uint8_t*>(workspace) + align256(size_t(R) * size_t(K / 2) * 2));
    const int blocks = sm_count() * 4;
    spmm::f32_to_f16_kernel<<<blocks, 256, 0, s>>>(static_cast<const float*>(values), R, K / 2, K / 2, vh, K / 2);
    spmm::f32_to_f16_kernel<<<blocks, 256, 0, s>>>(static_cast<const float*>(X), K, T, ldx, xh, ldx_h);
    if (launch_status() != NM_OK) return NM_ERR_CUDA;
    return spmm::run<Kind::F16>(vh, meta_sm100, xh, ldx_h, Y, yk, ldy, R, K, T, alpha, beta, o, s);
  }
  if (ab_dtype == NM_S8)
    return spmm::run<Kind::S8>(values, meta_sm100, X, ldx, Y, yk, ldy, R, K, T, alpha, beta, o, s);
  if (ab_dtype == NM_BF16)
    return spmm::run<Kind::BF16>(values, meta_sm100, X, ldx, Y, yk, ldy, R, K, T, alpha, beta, o, s);
  return spmm::run<Kind::F16>(values, meta_sm100, X, ldx, Y, yk, ldy, R, K, T, alpha, beta, o, s);
}

nm_status spmm12_entry(const float* values, const uint8_t* meta12_img, const float* X, int64_t ldx, void* Y,
                       nm_dtype y_dtype, int64_t ldy, int64_t R, int64_t K, int64_t T, float alpha, float beta,
                       const spmm::Opts& o, void* stream) {
  if (y_dtype != NM_BF16 && y_dtype != NM_F32) return NM_ERR_DTYPE;
  if (R < 0 || K < 0 || T < 0 || K % 16 != 0 || ldx < T || ldy < T) return NM_ERR_SHAPE;
  if (R > 0x7FFFFFFF - 256 || K > 0x7FFFFFFF - 256 || T > 0x7FFFFFFF - 256) return NM_ERR_SHAPE;
  if (R == 0 || T == 0) return NM_OK;
  if (values == nullptr || meta12_img == nullptr || X == nullptr || Y == nullptr) return NM_ERR_NULL;
  if (!aligned16(values) || !aligned16(meta12_img) || !aligned16(X) || !stride_ok(ldx, 4) ||
      (reinterpret_cast<uintptr_t>(Y) % uintptr_t(esize_of(y_dtype))) != 0)
    return NM_ERR_ALIGN;
  if (K == 0) return NM_ERR_SHAPE;
  return spmm::run<spmm::Kind::TF32>(values, meta12_img, X, ldx, Y, y_kind_of(y_dtype), ldy, R, K, T, alpha, beta,
                                     o, static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" nm_status nm_spmm(const void* values, const uint8_t* meta_sm100, nm_dtype ab_dtype, const void* X,
                             int64_t ldx, void* Y, nm_dtype y_dtype, int64_t ldy, int64_t R, int64_t K, int64_t T,
                             float alpha, float beta, void* workspace, size_t workspace_bytes, void* stream) {
  return spmm_entry(values, meta_sm100, ab_dtype, X, ldx, Y, y_dtype, ldy, R, K, T, alpha, beta, workspace,
                    workspace_bytes, spmm::Opts(), stream);
}

extern "C" nm_status nm_spmm_peers(const void* values, const uint8_t* meta_sm100, nm_dtype ab_dtype, const void* X,
                                   int64_t ldx, void* const* peer_Y, int n_peers, int64_t row0, int64_t ldy,
                                   int64_t R, int64_t K, int64_t T, float alpha, void* stream) {
  if (ab_dtype != NM_BF16 && ab_dtype != NM_F16) return NM_ERR_DTYPE;
  if (n_peers < 1 || n_peers > spmm::kMaxPeers || row0 < 0) return NM_ERR_SHAPE;
  if (peer_Y == nullptr) return NM_ERR_NULL;
  for (int j = 0; j < n_peers; ++j)
    if (peer_Y[j] == nullptr) return NM_ERR_NULL;
  if (row0 > 0x7FFFFFFF) return NM_ERR_SHAPE;
  bool noop = false;
  void* y0 = static_cast<uint8_t*>(peer_Y[0]) + size_t(row0) * size_t(ldy < 0 ? 0 : ldy) * 2;
  const nm_status v =
      spmm_validate(values, meta_sm100, ab_dtype, X, ldx, y0, NM_BF16, ldy, R, K, T, alpha, 0.0f, &noop);
  if (v != NM_OK || noop) return v;
  if (!stride_ok(ldy, 2)) return NM_ERR_ALIGN;
  for (int j = 0; j < n_peers; ++j)
    if (!aligned16(static_cast<uint8_t*>(peer_Y[j]) + size_t(row0) * size_t(ldy) * 2)) return NM_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (ab_dtype == NM_BF16)
    return spmm::run<spmm::Kind::BF16>(values, meta_sm100, X, ldx, y0, 0, ldy, R, K, T, alpha, 0.0f, spmm::Opts(),
                                       s, peer_Y, n_peers, row0);
  return spmm::run<spmm::Kind::F16>(values, meta_sm100, X, ldx, y0, 0, ldy, R, K, T, alpha, 0.0f, spmm::Opts(), s,
                                    peer_Y, n_peers, row0);
}

extern "C" nm_status nm_spmm_test(const void* values, const uint8_t* meta_sm100, nm_dtype ab_dtype, const void* X,
                                  int64_t ldx, void* Y, nm_dtype y_dtype, int64_t ldy, int64_t R, int64_t K,
                                  int64_t T, float alpha, float beta, void* workspace, size_t workspace_bytes,
                                  int kernel, int tail_split, int64_t wait_limit_ns, int64_t skip_step,
                                  int raster_group, int raster_m_inner, void* stream) {
  if (kernel < 0 || kernel > 9 || wait_limit_ns < 0 || skip_step < -1 || raster_group < 0 ||
      raster_m_inner < 0 || raster_m_inner > 1)
    return NM_ERR_SHAPE;
  spmm::Opts o;
  o.kernel = kernel;
  o.tail_split = tail_split != 0;
  if (wait_limit_ns > 0) o.wait_ns = uint64_t(wait_limit_ns);
  o.skip_it = skip_step;
  if (raster_group > 0) o.raster = 1 + 2 * raster_group + raster_m_inner;
  return spmm_entry(values, meta_sm100, ab_dtype, X, ldx, Y, y_dtype, ldy, R, K, T, alpha, beta, workspace,
                    workspace_bytes, o, stream);
}

extern "C" nm_status nm_spmm12(const float* values, const uint8_t* meta12_sm100, const float* X, int64_t ldx,
                               void* Y, nm_dtype y_dtype, int64_t ldy, int64_t R, int64_t K, int64_t T, float alpha,
                               float beta, void* stream) {
  return spmm12_entry(values, meta12_sm100, X, ldx, Y, y_dtype, ldy, R, K, T, alpha, beta, spmm::Opts(), stream);
}

extern "C" nm_status nm_spmm12_test(const float* values, const uint8_t* meta12_sm100, const float* X, int64_t ldx,
                                    void* Y, nm_dtype y_dtype, int64_t ldy, int64_t R, int64_t K, int64_t T,
                                    float alpha, float beta, int kernel, int tail_split, void* stream) {
  if (kernel < 0 || kernel > 9) return NM_ERR_SHAPE;
  spmm::Opts o;
  o.kernel = kernel;
  o.tail_split = tail_split != 0;
  return spmm12_entry(values, meta12_sm100, X, ldx, Y, y_dtype, ldy, R, K, T, alpha, beta, o, stream);
}

extern "C" nm_status nm_last_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return NM_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, nm::g_device_status, sizeof(int)) != cudaSuccess) return NM_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(nm::g_device_status, &zero, sizeof(int)) != cudaSuccess) return NM_ERR_CUDA;
  }
  return static_cast<nm_status>(v);
}

// ---------------------------------------------------------------------------
// nm_spmm_noalloc: nm_spmm for callers that cannot allocate device memory.
// The fp32 path of nm_spmm needs scratch (inputs rounded to binary16).  This
// variant takes it from a fixed, file-scope device array instead of a
// caller-supplied workspace, so the call itself never allocates.  The array
// is part of the module: every GPU that loads the library holds it until the
// process exits.
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  Looked up once
// per device, on the first call made with that device current.  In host code
// the array's name is only a host-side stand-in, never a device address.
nm_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return NM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return NM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return NM_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return NM_OK;
}
}  // namespace

extern "C" nm_status nm_spmm_noalloc(const void* values, const uint8_t* meta_sm100, nm_dtype ab_dtype,
                                     const void* X, int64_t ldx, void* Y, nm_dtype y_dtype, int64_t ldy,
                                     int64_t R, int64_t K, int64_t T, float alpha, float beta, void* stream) {
  // the same argument checks as nm_spmm first, so a malformed call reports
  // its real fault rather than the scratch limit
  bool noop = false;
  const nm_status v =
      spmm_validate(values, meta_sm100, ab_dtype, X, ldx, Y, y_dtype, ldy, R, K, T, alpha, beta, &noop);
  if (v != NM_OK || noop) return v;
  if (ab_dtype != NM_F32)  // the 16-bit and int8 paths use no scratch at all
    return nm_spmm(values, meta_sm100, ab_dtype, X, ldx, Y, y_dtype, ldy, R, K, T, alpha, beta, nullptr, 0, stream);
  const size_t need = nm_spmm_workspace_bytes(ab_dtype, R, K, T);
  if (need > kNoAllocScratchBytes) return NM_ERR_WORKSPACE;  // problem larger than the fixed scratch
  void* scratch = nullptr;
  const nm_status st = noalloc_scratch(&scratch);
  if (st != NM_OK) return st;
  return nm_spmm(values, meta_sm100, ab_dtype, X, ldx, Y, y_dtype, ldy, R, K, T, alpha, beta, scratch,
                 kNoAllocScratchBytes, stream);
}
