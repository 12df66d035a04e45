// Cross-GPU completion flags and peer mappings for the row-split product.
//
// When the product is split by output rows over several GPUs, each GPU writes
// its rows of the output into every GPU's copy (nm_spmm_peers), then tells
// every GPU that its rows are there (nm_peer_signal), and a GPU that needs the
// whole output waits until every GPU has said so (nm_peer_wait).  The flags
// carry an epoch that the caller raises by one per step, so they never need
// to be reset.  nm_ipc_handle / nm_ipc_open map one process's device buffer
// into another process (CUDA IPC), which is how the output buffers and flag
// arrays of the other GPUs become addressable.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/nm.h"
#include "nm_internal.cuh"

namespace nm {
namespace peers {

constexpr int kMaxPeers = 8;

struct FlagPtrs {
  uint64_t* f[kMaxPeers];
};

// Thread j stores `epoch` into slot `rank` of GPU j's flag array.  The
// system-scope fence first orders every earlier write of this stream (the
// product's stores into the other GPUs' buffers, complete when its kernel
// ended) before the flag, for a reader on any GPU.
__global__ void signal_kernel(FlagPtrs fp, int n, int rank, uint64_t epoch) {
  const int j = threadIdx.x;
  if (j >= n) return;
  asm volatile("fence.sc.sys;" ::: "memory");
  asm volatile("st.release.sys.global.u64 [%0], %1;" ::"l"(fp.f[j] + rank), "l"(epoch) : "memory");
}

__device__ __forceinline__ uint64_t ld_acquire_sys(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.acquire.sys.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint64_t timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Lane j waits until slot j holds at least `epoch`, for at most limit_ns; a
// lane that gives up records NM_ERR_TIMEOUT in the device status word and
// returns.  The trailing proxy fence lets the next kernel's bulk tensor loads
// see the data the flags vouch for.
__global__ void wait_kernel(const uint64_t* flags, int n, uint64_t epoch, uint64_t limit_ns, int* status) {
  const int j = threadIdx.x;
  if (j < n) {
    const uint64_t t0 = timer_ns();
    while (ld_acquire_sys(flags + j) < epoch) {
      if (timer_ns() - t0 > limit_ns) {
        if (status != nullptr) atomicExch(status, int(NM_ERR_TIMEOUT));
        break;
      }
      __nanosleep(200);
    }
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// cuMemGetAddressRange through the runtime's driver entry point (no libcuda at link time)
using AddressRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);
AddressRangeFn address_range() {
  static AddressRangeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<AddressRangeFn>(ptr);
  });
  return fn;
}

}  // namespace peers
}  // namespace nm

using namespace nm;

extern "C" nm_status nm_peer_signal(uint64_t* const* peer_flags, int n_peers, int rank, uint64_t epoch,
                                    void* stream) {
  if (n_peers < 1 || n_peers > peers::kMaxPeers || rank < 0 || rank >= n_peers) return NM_ERR_SHAPE;
  if (peer_flags == nullptr) return NM_ERR_NULL;
  peers::FlagPtrs fp;
  memset(&fp, 0, sizeof(fp));
  for (int j = 0; j < n_peers; ++j) {
    if (peer_flags[j] == nullptr) return NM_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(peer_flags[j]) & 7u) != 0) return NM_ERR_ALIGN;
    fp.f[j] = peer_flags[j];
  }
  peers::signal_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(fp, n_peers, rank, epoch);
  return launch_status();
}

extern "C" nm_status nm_peer_wait(const uint64_t* flags, int n_peers, uint64_t epoch, int64_t timeout_ns,
                                  void* stream) {
  if (n_peers < 1 || n_peers > peers::kMaxPeers || timeout_ns <= 0) return NM_ERR_SHAPE;
  if (flags == nullptr) return NM_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(flags) & 7u) != 0) return NM_ERR_ALIGN;
  peers::wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(flags, n_peers, epoch, uint64_t(timeout_ns),
                                                                      device_status_word());
  return launch_status();
}

extern "C" nm_status nm_ipc_handle(const void* dev_ptr, void* handle, int64_t* offset) {
  if (dev_ptr == nullptr || handle == nullptr || offset == nullptr) return NM_ERR_NULL;
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, dev_ptr) != cudaSuccess || attr.type != cudaMemoryTypeDevice) {
    (void)cudaGetLastError();
    return NM_ERR_CUDA;
  }
  // The handle names the whole allocation; the offset locates dev_ptr in it.
  peers::AddressRangeFn range = peers::address_range();
  CUdeviceptr base = 0;
  size_t bytes = 0;
  if (range == nullptr || range(&base, &bytes, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
    return NM_ERR_CUDA;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) {
    (void)cudaGetLastError();
    return NM_ERR_CUDA;
  }
  static_assert(sizeof(h) == NM_IPC_HANDLE_BYTES, "CUDA IPC handle size");
  memcpy(handle, &h, sizeof(h));
  *offset = int64_t(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
  return NM_OK;
}

extern "C" nm_status nm_ipc_open(const void* handle, int64_t offset, void** dev_ptr) {
  if (handle == nullptr || dev_ptr == nullptr) return NM_ERR_NULL;
  if (offset < 0) return NM_ERR_SHAPE;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof(h));
  void* base = nullptr;
  if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
    (void)cudaGetLastError();
    return NM_ERR_CUDA;
  }
  *dev_ptr = static_cast<uint8_t*>(base) + offset;
  return NM_OK;
}

extern "C" nm_status nm_ipc_close(void* dev_ptr, int64_t offset) {
  if (dev_ptr == nullptr) return NM_ERR_NULL;
  if (offset < 0) return NM_ERR_SHAPE;
  if (cudaIpcCloseMemHandle(static_cast<uint8_t*>(dev_ptr) - offset) != cudaSuccess) {
    (void)cudaGetLastError();
    return NM_ERR_CUDA;
  }
  return NM_OK;
}
