// Host-side argument checks shared by the entry points of libshla.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/shla.h"

namespace shla {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// The kernels use tcgen05 / TMEM: compute capability 10.x only.
inline int check_device(int* sm_count = nullptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (major != 10 || minor != 0) return MLA_ERR_UNSUPPORTED;
  if (sm_count) {
    if (cudaDeviceGetAttribute(sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

inline int launch_status() {
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (kernel, device).
// Safe to call from several host threads at once: the mask is atomic, and two
// threads that both find the bit clear both set the same attribute value.
template <typename F>
inline int ensure_smem_attr(F* fn, int bytes, std::atomic<unsigned long long>* done_mask) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  const unsigned long long bit = 1ull << (dev & 63);
  if (done_mask->load(std::memory_order_acquire) & bit) return MLA_OK;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return MLA_ERR_CUDA;
  done_mask->fetch_or(bit, std::memory_order_acq_rel);
  return MLA_OK;
}

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Launch with programmatic stream serialisation: the kernel may be scheduled
// once every block of the previous kernel on the stream has executed
// griddepcontrol.launch_dependents (or exited), so its set-up overlaps that
// kernel's tail.  The kernel must execute griddepcontrol.wait before it reads
// or writes anything the previous kernel writes or reads.  Used only where
// the previous kernel is one of this library's, launched by the same call.
template <typename... KArgs, typename... Args>
inline int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

}  // namespace shla
