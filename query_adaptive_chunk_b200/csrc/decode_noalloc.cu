// Merged sparse decode that allocates nothing.
//
// Some callers cannot hand the library freshly allocated device memory: an
// application that owns all device memory through its own pool and forbids
// other allocations, or a latency-critical serving loop that must not call
// cudaMalloc (which can synchronise the whole device) on its hot path.  For
// them this file keeps the merged decode's scratch (split partials and
// per-unit arrival counters) in a fixed array inside the library itself.
#include <mutex>

#include "../../include/csa.h"
#include "internal.h"

namespace {

// The scratch area.  It belongs to the library's module, so every GPU that
// loads the library holds these bytes until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device.  In host code the
// array's name only stands in for the symbol, so the address is looked up
// once per device with that device current.
csa_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    csa::set_last_error(std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    return CSA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    csa::set_last_error("device ordinal out of range for the built-in scratch table");
    return CSA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      csa::set_last_error(std::string("cudaGetSymbolAddress(built-in scratch): ") +
                          cudaGetErrorString(e));
      return CSA_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return CSA_OK;
}

}  // namespace

extern "C" {

csa_status csa_sparse_decode_merged_noalloc(const void* q, const void* K, const void* V,
                                            csa_dtype dtype, const int32_t* idx,
                                            const int32_t* count, int kmax,
                                            const uint8_t* head_full, int B, int Hq, int Hkv,
                                            int D, int64_t T, int L, float scale, int num_parts,
                                            void* out, csa_dtype out_dtype, float* lse_out,
                                            csa_stream stream) {
  const int64_t need = csa_decode_workspace_bytes(B, Hq, Hkv, D, num_parts);
  if (need < 0) {
    csa::set_last_error("csa_sparse_decode_merged_noalloc: bad sizes");
    return CSA_ERR_INVALID_ARG;
  }
  if (static_cast<uint64_t>(need) > kNoAllocScratchBytes) {
    csa::set_last_error("csa_sparse_decode_merged_noalloc: this shape needs " +
                        std::to_string(need) + " bytes of scratch but the built-in area holds " +
                        std::to_string(kNoAllocScratchBytes) +
                        "; use fewer pieces (num_parts) or csa_sparse_decode_merged with a workspace");
    return CSA_ERR_UNSUPPORTED;
  }
  void* ws = nullptr;
  csa_status st = scratch_address(&ws);
  if (st != CSA_OK) return st;
  st = csa_sparse_decode_merged(q, K, V, dtype, idx, count, kmax, head_full, B, Hq, Hkv, D, T, L,
                                scale, num_parts, ws, static_cast<int64_t>(kNoAllocScratchBytes),
                                out, out_dtype, lse_out, stream);
  if (st != CSA_OK || B == 0) return st;
  // The area keeps whatever a call leaves behind.  Its arrival counters must
  // read zero when the next decode starts: the area is zero-initialised when
  // the library loads, a decode that completes leaves them zero, and every
  // call also clears them after its decode, so that a call that ended early
  // (a wait past its time limit, reported by csa_check_device_status) does
  // not leave a count behind for the next one.  The clear is one memset node
  // of B * Hkv counters on the stream (a few hundred bytes).  No test makes a
  // decode's waits run out on purpose: a limit short enough for that would
  // also cut short the wait for its own copies in flight before it retires.
  const size_t counter_bytes = (static_cast<size_t>(B) * Hkv * 4 + 255) & ~size_t(255);
  cudaError_t e = cudaMemsetAsync(ws, 0, counter_bytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    csa::set_last_error(std::string("clearing the built-in scratch counters: ") +
                        cudaGetErrorString(e));
    return CSA_ERR_CUDA;
  }
  return CSA_OK;
}

}  // extern "C"
