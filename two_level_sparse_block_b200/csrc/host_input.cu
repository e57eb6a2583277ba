// Per-step inputs straight from pinned host memory.  A decode step's query
// is tens of kilobytes; brought in by a copy-engine transfer inside a captured
// step, it lands about 2 us later than with a kernel whose loads cross PCIe
// (the copy engine's start and its hand-off to the SMs).  tls_copy_from_host
// moves such a buffer with one kernel: every thread one 16-byte load from the
// host and one store to device memory, 4 KB per CTA, all CTAs' loads in
// flight at once (one PCIe round trip for up to 2.4 MB).

#include <cuda_runtime.h>

#include <map>
#include <mutex>
#include <utility>

#include "host_common.h"

namespace tls {
namespace {

constexpr int kCopyThreads = 256;

__global__ void __launch_bounds__(kCopyThreads) copy_from_host_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                                      int64_t n16) {
  for (int64_t i = blockIdx.x * (int64_t)kCopyThreads + threadIdx.x; i < n16; i += (int64_t)gridDim.x * kCopyThreads)
    dst[i] = src[i];
}

// Device address of a pinned host range (both ends checked, as one mapped
// range), remembered per (address, size): the check runs once, outside any
// graph capture that repeats the call.
const void* mapped_source(const void* p, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<uintptr_t, size_t>, const void*> seen;
  const std::pair<uintptr_t, size_t> key((uintptr_t)p, bytes);
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = seen.find(key);
    if (it != seen.end()) return it->second;
  }
  cudaPointerAttributes a, b;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess ||
      cudaPointerGetAttributes(&b, (const uint8_t*)p + (bytes - 1)) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (a.type != cudaMemoryTypeHost || b.type != cudaMemoryTypeHost || a.devicePointer == nullptr ||
      b.devicePointer == nullptr ||
      (const uint8_t*)b.devicePointer - (const uint8_t*)a.devicePointer != (ptrdiff_t)(bytes - 1))
    return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (seen.size() >= 4096) seen.clear();  // a loop reuses a few buffers; bound the memory all the same
  seen[key] = a.devicePointer;
  return a.devicePointer;
}

}  // namespace
}  // namespace tls

using namespace tls;

extern "C" tls_status tls_copy_from_host(void* dst, const void* src, size_t bytes, void* stream) {
  NvtxRange nvtx_range("tls_copy_from_host");
  clear_error();
  if (dst == nullptr || src == nullptr) return fail(TLS_ERR_INVALID_ARG, "copy_from_host: NULL pointer");
  if (bytes == 0) return TLS_OK;
  if (bytes % 16 != 0 || !aligned16(dst) || !aligned16(src))
    return fail(TLS_ERR_INVALID_ARG, "copy_from_host: pointers and size must be multiples of 16 bytes");
  const void* dsrc = mapped_source(src, bytes);
  if (dsrc == nullptr)
    return fail(TLS_ERR_INVALID_ARG, "copy_from_host: the source is not pinned host memory the device can address");
  const int64_t n16 = (int64_t)(bytes / 16);
  const int64_t want = (n16 + kCopyThreads - 1) / kCopyThreads;
  const int grid = (int)(want < 4 * kNumSMs ? want : 4 * kNumSMs);
  copy_from_host_kernel<<<grid, kCopyThreads, 0, (cudaStream_t)stream>>>(
      reinterpret_cast<const uint4*>(dsrc), reinterpret_cast<uint4*>(dst), n16);
  return launch_check("copy_from_host: launch");
}
