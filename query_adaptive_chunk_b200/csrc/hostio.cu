// Host-side transfers of a decode step whose query and result live in pinned
// host memory.  Under unified addressing a pinned allocation is mapped into
// the device's address space, so the SMs can load from it and store to it
// across the host link directly: for the few kilobytes of one decode query
// that costs a single round trip, without the setup of a copy-engine
// transfer.  The decode kernel stores its output rows into such memory with
// its ordinary stores; the query comes in through the kernel below.
#include "internal.h"

namespace csa {
namespace {

// 16-byte words from src to dst, one word per thread.  A kernel launched
// behind it with programmatic dependent launch may start at once (it waits
// for this grid's completion before reading dst).
__global__ void copy16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int64_t n) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = src[i];
}

}  // namespace

cudaError_t launch_copy16(const Launch& l, const void* src, void* dst, size_t bytes) {
  const int64_t n = static_cast<int64_t>(bytes / 16);
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (n + threads - 1) / threads;
  copy16_kernel<<<static_cast<unsigned>(blocks), threads, 0, l.stream>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), n);
  return cudaGetLastError();
}

}  // namespace csa
