// C ABI of libcsa (declared in include/csa.h): argument validation, error
// reporting and the launches.  Nothing here allocates device memory.
#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstdlib>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/csa.h"
#include "internal.h"

// Device status word: [0] = first error code recorded by a kernel.
__device__ int g_csa_status[4];

// One thread waits on an mbarrier that never completes its first phase; the
// bounded wait gives up after e.wait_ns and records DEV_TIMEOUT.
__global__ void wait_timeout_selftest_kernel(csa::DevErr e) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = csa::smem_u32(&bar);
  if (threadIdx.x == 0) {
    csa::mbar_init(b, 1);
    csa::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) csa::mbar_wait(b, 0u, e);
}

namespace {

thread_local std::string t_err;

std::atomic<uint64_t>& wait_limit() {
  static std::atomic<uint64_t> v([] {
    const char* e = std::getenv("CSA_WAIT_LIMIT_NS");
    if (e && *e) {
      const unsigned long long x = std::strtoull(e, nullptr, 10);
      if (x > 0) return static_cast<uint64_t>(x);
    }
    return static_cast<uint64_t>(2000000000ull);
  }());
  return v;
}

struct DevState {
  bool ready = false;
  int* status = nullptr;
  int num_sms = 0;
};

std::mutex g_mu;
std::vector<DevState> g_dev;

csa_status fail(csa_status s, const std::string& why) {
  t_err = why;
  return s;
}

csa_status cuda_fail(cudaError_t e, const char* what) {
  t_err = std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
  return CSA_ERR_CUDA;
}

// Per-device set-up (status word address, SM count), once per device.
csa_status launch_ctx(csa_stream stream, csa::Launch* l) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lk(g_mu);
  if (static_cast<int>(g_dev.size()) <= dev) g_dev.resize(dev + 1);
  DevState& st = g_dev[dev];
  if (!st.ready) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_csa_status);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status word)");
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    st.status = static_cast<int*>(p);
    st.num_sms = sms;
    st.ready = true;
  }
  l->stream = static_cast<cudaStream_t>(stream);
  l->err.word = st.status;
  l->err.wait_ns = wait_limit().load();
  l->num_sms = st.num_sms;
  return CSA_OK;
}

// A required device pointer: not NULL, 16-byte aligned, device or managed
// memory of the current device.
csa_status check_ptr(const void* p, const char* name, bool required = true) {
  if (p == nullptr) {
    if (!required) return CSA_OK;
    return fail(CSA_ERR_INVALID_ARG, std::string(name) + " is NULL");
  }
  if (reinterpret_cast<uintptr_t>(p) % 16 != 0)
    return fail(CSA_ERR_INVALID_ARG, std::string(name) + " is not 16-byte aligned");
  cudaPointerAttributes a;
  cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(CSA_ERR_INVALID_ARG, std::string(name) + " is not a CUDA pointer");
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
    return fail(CSA_ERR_INVALID_ARG, std::string(name) + " is not device memory");
  int dev = 0;
  cudaGetDevice(&dev);
  if (a.type == cudaMemoryTypeDevice && a.device != dev)
    return fail(CSA_ERR_INVALID_ARG, std::string(name) + " lives on another device");
  return CSA_OK;
}

#define CSA_TRY(x)                     \
  do {                                 \
    csa_status _s = (x);               \
    if (_s != CSA_OK) return _s;       \
  } while (0)

#define CSA_REQUIRE(cond, msg)                                   \
  do {                                                           \
    if (!(cond)) return fail(CSA_ERR_INVALID_ARG, (msg));        \
  } while (0)

#define CSA_SUPPORT(cond, msg)                                   \
  do {                                                           \
    if (!(cond)) return fail(CSA_ERR_UNSUPPORTED, (msg));        \
  } while (0)

bool valid_dtype(csa_dtype d) { return d == CSA_F32 || d == CSA_BF16; }

csa_status finish(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return cuda_fail(e, what);
  t_err.clear();
  return CSA_OK;
}

}  // namespace

namespace csa {
void set_last_error(const std::string& why) { t_err = why; }
}  // namespace csa

extern "C" {

int csa_version(void) { return 10000; }

const char* csa_last_error_string(void) { return t_err.c_str(); }

void csa_set_wait_limit_ns(uint64_t ns) { wait_limit().store(ns > 0 ? ns : 1); }

uint64_t csa_get_wait_limit_ns(void) { return wait_limit().load(); }

csa_status csa_check_device_status(csa_stream stream) {
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  cudaError_t e = cudaStreamSynchronize(l.stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int word[4] = {0, 0, 0, 0};
  e = cudaMemcpy(word, l.err.word, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  if (word[0] != 0) {
    int zero[4] = {0, 0, 0, 0};
    e = cudaMemcpy(l.err.word, zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device status word");
  }
  switch (word[0]) {
    case 0: t_err.clear(); return CSA_OK;
    case csa::DEV_TIMEOUT: return fail(CSA_ERR_TIMEOUT, "a kernel wait exceeded its time limit");
    case csa::DEV_BAD_INDEX:
      return fail(CSA_ERR_DEVICE_INDEX, "a kernel met a chunk index or count out of range");
    default: return fail(CSA_ERR_CUDA, "unknown device status " + std::to_string(word[0]));
  }
}

csa_status csa_chunk_summaries(const void* K, csa_dtype dtype, int B, int Hkv, int64_t T, int D,
                               int L, const float* proj, int R, float* summ, csa_stream stream) {
  CSA_REQUIRE(valid_dtype(dtype), "dtype");
  CSA_REQUIRE(B >= 0 && Hkv >= 0 && T >= 0 && D > 0 && L > 0, "sizes must be non-negative, D and L positive");
  CSA_REQUIRE(T % L == 0, "T must be a multiple of L");
  CSA_SUPPORT(D == 64 || D == 128, "D must be 64 or 128");
  if (proj) CSA_SUPPORT(R == 16 || R == 32 || R == 64 || R == 128, "R must be 16, 32, 64 or 128");
  CSA_SUPPORT(T / L <= 2147483647LL, "too many chunks");
  if (static_cast<int64_t>(B) * Hkv * T == 0) return CSA_OK;
  CSA_TRY(check_ptr(K, "K"));
  CSA_TRY(check_ptr(summ, "summ"));
  CSA_TRY(check_ptr(proj, "proj", false));
  CSA_SUPPORT(static_cast<int64_t>(B) * Hkv <= 65535, "B*Hkv must be <= 65535");
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  return finish(csa::launch_chunk_summaries(l, K, dtype == CSA_BF16, B * Hkv, T, D, L, proj, R, summ),
                "chunk summaries launch");
}

csa_status csa_meta_summaries(const float* summ, int B, int Hkv, int C, int Ds, int Gm, float* meta,
                              csa_stream stream) {
  CSA_REQUIRE(B >= 0 && Hkv >= 0 && C >= 0 && Ds > 0 && Gm > 0, "bad sizes");
  CSA_REQUIRE(C % Gm == 0, "C must be a multiple of Gm");
  CSA_SUPPORT(Ds <= 1024, "Ds must be <= 1024");
  if (static_cast<int64_t>(B) * Hkv * C == 0) return CSA_OK;
  CSA_SUPPORT(static_cast<int64_t>(B) * Hkv <= 65535, "B*Hkv must be <= 65535");
  CSA_TRY(check_ptr(summ, "summ"));
  CSA_TRY(check_ptr(meta, "meta"));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  return finish(csa::launch_meta_summaries(l, summ, B * Hkv, C, Ds, Gm, meta), "meta summaries launch");
}

csa_status csa_tile_mean_q(const void* Q, csa_dtype dtype, int B, int S, int Hq, int D, int tile_m,
                           float* qbar, csa_stream stream) {
  CSA_REQUIRE(valid_dtype(dtype), "dtype");
  CSA_REQUIRE(B >= 0 && S >= 0 && Hq >= 0 && D > 0 && tile_m > 0, "bad sizes");
  CSA_REQUIRE(S % tile_m == 0, "S must be a multiple of tile_m");
  CSA_SUPPORT(D <= 1024 && Hq <= 65535 && B <= 65535, "D <= 1024, Hq and B <= 65535");
  CSA_SUPPORT((static_cast<int64_t>(Hq) * D) % (dtype == CSA_BF16 ? 8 : 4) == 0,
              "Hq * D must be a multiple of 8 (bf16) or 4 (fp32): rows are read 16 bytes at a time");
  if (static_cast<int64_t>(B) * S * Hq == 0) return CSA_OK;
  CSA_TRY(check_ptr(Q, "Q"));
  CSA_TRY(check_ptr(qbar, "qbar"));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  return finish(csa::launch_tile_mean(l, Q, dtype == CSA_BF16, B, S, Hq, D, tile_m, qbar), "tile mean launch");
}

csa_status csa_rope(const void* x, void* y, csa_dtype dtype, int64_t rows, int D, int64_t period,
                    int64_t pos0, float theta, csa_stream stream) {
  CSA_REQUIRE(valid_dtype(dtype), "dtype");
  CSA_REQUIRE(rows >= 0 && D > 0 && period > 0 && pos0 >= 0, "bad sizes");
  CSA_REQUIRE(D % 2 == 0, "D must be even");
  CSA_SUPPORT(D <= 512, "D <= 512");
  CSA_REQUIRE(std::isfinite(theta) && theta > 1.0f, "theta must be finite and > 1");
  if (rows == 0) return CSA_OK;
  CSA_TRY(check_ptr(x, "x"));
  CSA_TRY(check_ptr(y, "y"));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  return finish(csa::launch_rope(l, x, y, dtype == CSA_BF16, rows, D, period, pos0, theta),
                "rope launch");
}

csa_status csa_score_chunks(const void* q, csa_dtype q_dtype, const float* proj, int R,
                            const float* summ, int B, int Nq, int Hq, int Hkv, int D, int C,
                            const uint8_t* head_full, int causal_tile_m, int causal_L,
                            float* scores, csa_stream stream) {
  CSA_REQUIRE(valid_dtype(q_dtype), "q_dtype");
  CSA_REQUIRE(B >= 0 && Nq >= 0 && Hq > 0 && Hkv > 0 && D > 0 && C >= 0, "bad sizes");
  CSA_REQUIRE(Hq % Hkv == 0, "Hq must be a multiple of Hkv");
  CSA_REQUIRE(causal_tile_m >= 0 && (causal_tile_m == 0 || causal_L > 0), "causal_tile_m / causal_L");
  CSA_SUPPORT(D <= 1024, "D must be <= 1024");
  const int Ds = proj ? R : D;
  CSA_SUPPORT(Ds == 16 || Ds == 32 || Ds == 64 || Ds == 128, "summary width must be 16, 32, 64 or 128");
  CSA_SUPPORT(Nq <= 65535 && static_cast<int64_t>(B) * Hkv <= 65535, "Nq and B*Hkv must be <= 65535");
  if (static_cast<int64_t>(B) * Nq * C == 0) return CSA_OK;
  CSA_TRY(check_ptr(q, "q"));
  CSA_TRY(check_ptr(proj, "proj", false));
  CSA_TRY(check_ptr(summ, "summ"));
  CSA_TRY(check_ptr(head_full, "head_full", false));
  CSA_TRY(check_ptr(scores, "scores"));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  return finish(csa::launch_score(l, q, q_dtype == CSA_BF16, proj, R, summ, B, Nq, Hq, Hkv, D, C,
                                  head_full, causal_tile_m, causal_L, scores),
                "score launch");
}

csa_status csa_select_topk(const float* scores, int U, int C, const int32_t* n_valid, int k_free,
                           int n_sink, int n_local, int32_t* idx, int32_t* count, int kmax,
                           csa_stream stream) {
  CSA_REQUIRE(kmax > 0, "kmax must be positive");
  CSA_REQUIRE(U >= 0 && C >= 0 && k_free >= 0 && n_sink >= 0 && n_local >= 0, "U, C, k_free, n_sink and n_local must be non-negative");
  CSA_SUPPORT(C <= 32768, "C must be <= 32768");
  const int64_t need = std::min<int64_t>(C, static_cast<int64_t>(k_free) + n_sink + n_local);
  CSA_REQUIRE(kmax >= need, "kmax < min(C, k_free + n_sink + n_local)");
  if (U == 0) return CSA_OK;
  CSA_SUPPORT(U <= 2147483647, "U");
  CSA_TRY(check_ptr(scores, "scores", C > 0));
  CSA_TRY(check_ptr(n_valid, "n_valid", false));
  CSA_TRY(check_ptr(idx, "idx"));
  CSA_TRY(check_ptr(count, "count"));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  return finish(csa::launch_select_topk(l, scores, U, C, n_valid, k_free, n_sink, n_local, idx, count, kmax),
                "select_topk launch");
}

csa_status csa_select_topk_causal(const float* scores, int U, int C, int n_tiles, int tile_m,
                                  int L, int k_free, int n_sink, int n_local, int32_t* idx,
                                  int32_t* count, int kmax, csa_stream stream) {
  CSA_REQUIRE(kmax > 0, "kmax must be positive");
  CSA_REQUIRE(U >= 0 && C >= 0 && k_free >= 0 && n_sink >= 0 && n_local >= 0,
              "U, C, k_free, n_sink and n_local must be non-negative");
  CSA_REQUIRE(n_tiles > 0 && tile_m > 0 && L > 0, "n_tiles, tile_m and L must be positive");
  CSA_REQUIRE(U % n_tiles == 0, "U must be a multiple of n_tiles");
  CSA_SUPPORT(C <= 32768, "C must be <= 32768");
  const int64_t need = std::min<int64_t>(C, static_cast<int64_t>(k_free) + n_sink + n_local);
  CSA_REQUIRE(kmax >= need, "kmax < min(C, k_free + n_sink + n_local)");
  if (U == 0) return CSA_OK;
  CSA_TRY(check_ptr(scores, "scores", C > 0));
  CSA_TRY(check_ptr(idx, "idx"));
  CSA_TRY(check_ptr(count, "count"));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  return finish(csa::launch_select_topk(l, scores, U, C, nullptr, k_free, n_sink, n_local, idx,
                                        count, kmax, nullptr, n_tiles, tile_m, L),
                "select_topk_causal launch");
}

csa_status csa_select_topp(const float* scores, int U, int C, float logit_scale, float p, int budget,
                           int n_sink, int n_local, int32_t* idx, int32_t* count, int kmax,
                           int32_t* n_p_out, csa_stream stream) {
  CSA_REQUIRE(kmax > 0, "kmax must be positive");
  CSA_REQUIRE(U >= 0 && C > 0 && n_sink >= 0 && n_local >= 0, "U, n_sink and n_local must be non-negative and C positive");
  CSA_REQUIRE(p > 0.f && p <= 1.f, "p must be in (0, 1]");
  CSA_REQUIRE(budget >= 1, "budget must be >= 1");
  CSA_REQUIRE(logit_scale == logit_scale, "logit_scale is NaN");
  CSA_SUPPORT(budget <= 2048 && C <= 32768, "budget <= 2048 and C <= 32768");
  const int64_t need = std::min<int64_t>(C, static_cast<int64_t>(budget) + n_sink + n_local);
  CSA_REQUIRE(kmax >= need, "kmax < min(C, budget + n_sink + n_local)");
  if (U == 0) return CSA_OK;
  CSA_TRY(check_ptr(scores, "scores"));
  CSA_TRY(check_ptr(idx, "idx"));
  CSA_TRY(check_ptr(count, "count"));
  CSA_TRY(check_ptr(n_p_out, "n_p_out", false));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  return finish(csa::launch_select_topp(l, scores, U, C, logit_scale, p, budget, n_sink, n_local, idx,
                                        count, kmax, n_p_out),
                "select_topp launch");
}

}  // extern "C"

namespace {
// The selection calls with `check_only`: every argument check, then return
// before anything is enqueued (used by the one-call step to reject a bad
// selection argument before its query copy).
csa_status select_hier_impl(const void* q, csa_dtype q_dtype, const float* meta,
                            const float* summ, int B, int Hq, int Hkv, int D, int C, int Gm,
                            int top_meta, int k_free, int n_sink, int n_local, int32_t* idx,
                            int32_t* count, int kmax, csa_stream stream, bool check_only) {
  CSA_REQUIRE(valid_dtype(q_dtype), "q_dtype");
  CSA_REQUIRE(B >= 0 && Hq > 0 && Hkv > 0 && C > 0 && Gm > 0 && top_meta >= 0 && k_free >= 0 &&
                  n_sink >= 0 && n_local >= 0 && kmax > 0,
              "bad sizes");
  CSA_REQUIRE(Hq % Hkv == 0, "Hq must be a multiple of Hkv");
  CSA_REQUIRE(C % Gm == 0, "C must be a multiple of Gm");
  CSA_SUPPORT(D == 64 || D == 128, "D must be 64 or 128");
  CSA_SUPPORT(C <= 32768 && C / Gm <= 8192, "C <= 32768 and C/Gm <= 8192");
  CSA_SUPPORT(static_cast<int64_t>(std::min(top_meta, C / Gm)) * Gm <= 8192, "top_meta * Gm must be <= 8192");
  const int64_t need = std::min<int64_t>(C, static_cast<int64_t>(k_free) + n_sink + n_local);
  CSA_REQUIRE(kmax >= need, "kmax < min(C, k_free + n_sink + n_local)");
  if (B == 0) return CSA_OK;
  CSA_TRY(check_ptr(q, "q"));
  CSA_TRY(check_ptr(meta, "meta"));
  CSA_TRY(check_ptr(summ, "summ"));
  CSA_TRY(check_ptr(idx, "idx"));
  CSA_TRY(check_ptr(count, "count"));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  if (check_only) return CSA_OK;
  return finish(csa::launch_select_hier(l, q, q_dtype == CSA_BF16, meta, summ, B, Hq, Hkv, D, C, Gm,
                                        top_meta, k_free, n_sink, n_local, idx, count, kmax),
                "select_hier launch");
}
}  // namespace

extern "C" {

csa_status csa_select_hier(const void* q, csa_dtype q_dtype, const float* meta, const float* summ,
                           int B, int Hq, int Hkv, int D, int C, int Gm, int top_meta, int k_free,
                           int n_sink, int n_local, int32_t* idx, int32_t* count, int kmax,
                           csa_stream stream) {
  return select_hier_impl(q, q_dtype, meta, summ, B, Hq, Hkv, D, C, Gm, top_meta, k_free, n_sink,
                          n_local, idx, count, kmax, stream, false);
}

csa_status csa_selftest_wait_timeout(uint64_t limit_ns, csa_stream stream) {
  CSA_REQUIRE(limit_ns > 0 && limit_ns <= 10000000000ull, "limit_ns must be in (0, 1e10]");
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  csa::DevErr e = l.err;
  e.wait_ns = limit_ns;
  wait_timeout_selftest_kernel<<<1, 32, 0, l.stream>>>(e);
  return finish(cudaGetLastError(), "wait-timeout self-test launch");
}

int csa_decode_default_parts(csa_dtype dtype, int D, int L) {
  csa::Launch l;
  if (launch_ctx(nullptr, &l) != CSA_OK) return -1;
  return csa::decode_default_parts(dtype == CSA_BF16, D, L, l.num_sms);
}

}  // extern "C"

namespace {

// Shape checks shared by the two decode entry points (no CUDA call).
csa_status decode_shape_checks(csa_dtype dtype, int kmax, int B, int Hq, int Hkv, int D, int64_t T,
                               int L, float scale, int num_parts) {
  CSA_REQUIRE(valid_dtype(dtype), "dtype");
  CSA_REQUIRE(B >= 0 && Hq > 0 && Hkv > 0 && T >= 0 && L > 0 && kmax > 0 && num_parts >= 0,
              "B, T, num_parts must be non-negative; Hq, Hkv, L, kmax positive");
  CSA_REQUIRE(Hq % Hkv == 0, "Hq must be a multiple of Hkv");
  CSA_REQUIRE(T % L == 0, "T must be a multiple of L");
  CSA_SUPPORT(D == 64 || D == 128, "D must be 64 or 128");
  CSA_SUPPORT(L == 64 || L == 128, "L must be 64 or 128");
  const int G = Hq / Hkv;
  CSA_SUPPORT(G == 1 || G == 2 || G == 4 || G == 8, "Hq/Hkv must be 1, 2, 4 or 8");
  CSA_SUPPORT(static_cast<int64_t>(B) * Hkv <= 2048, "B*Hkv must be <= 2048");
  CSA_SUPPORT(static_cast<int64_t>(B) * Hkv * T < 2147483648LL, "B*Hkv*T must be < 2^31");
  CSA_SUPPORT(num_parts <= 65535, "num_parts must be <= 65535");
  CSA_REQUIRE(scale == scale, "scale is NaN");
  return CSA_OK;
}

// Pointer checks shared by the two decode entry points; returns the piece count.
csa_status decode_ptr_checks(const void* q, const void* K, const void* V, const int32_t* idx,
                             const int32_t* count, const uint8_t* head_full, bool bf16, int D,
                             int L, int num_parts, const csa::Launch& l, int* P_out) {
  CSA_TRY(check_ptr(q, "q"));
  CSA_TRY(check_ptr(K, "K"));
  CSA_TRY(check_ptr(V, "V"));
  CSA_TRY(check_ptr(head_full, "head_full", false));
  CSA_TRY(check_ptr(idx, "idx"));
  CSA_TRY(check_ptr(count, "count"));
  *P_out = num_parts > 0 ? num_parts : csa::decode_default_parts(bf16, D, L, l.num_sms);
  return CSA_OK;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

struct WorkspaceLayout {
  size_t counters, lse, o, total;
};

WorkspaceLayout workspace_layout(int B, int Hq, int Hkv, int D, int P) {
  WorkspaceLayout w;
  w.counters = 0;
  w.lse = round256(static_cast<size_t>(B) * Hkv * 4);
  w.o = w.lse + round256(static_cast<size_t>(B) * Hq * P * 4);
  w.total = w.o + static_cast<size_t>(B) * Hq * P * D * 4;
  return w;
}

}  // namespace

extern "C" {

csa_status csa_sparse_decode(const void* q, const void* K, const void* V, csa_dtype dtype,
                             const int32_t* idx, const int32_t* count, int kmax,
                             const uint8_t* head_full, int B, int Hq, int Hkv, int D, int64_t T, int L,
                             float scale, int num_parts, int max_splits, float* o_part,
                             float* lse_part, csa_stream stream) {
  CSA_REQUIRE(max_splits > 0, "max_splits must be positive");
  CSA_TRY(decode_shape_checks(dtype, kmax, B, Hq, Hkv, D, T, L, scale, num_parts));
  if (num_parts > 0) CSA_REQUIRE(max_splits >= num_parts, "max_splits must be >= num_parts");
  if (B == 0) return CSA_OK;
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  int P = 0;
  CSA_TRY(decode_ptr_checks(q, K, V, idx, count, head_full, dtype == CSA_BF16, D, L, num_parts, l, &P));
  CSA_REQUIRE(max_splits >= P, "max_splits must be >= the number of pieces (num_parts)");
  CSA_TRY(check_ptr(o_part, "o_part"));
  CSA_TRY(check_ptr(lse_part, "lse_part"));
  std::string why;
  cudaError_t e = csa::launch_decode(l, q, K, V, dtype == CSA_BF16, idx, count, kmax, head_full, B, Hq,
                                     Hkv, D, T, L, scale, P, max_splits, o_part, lse_part, nullptr, &why);
  if (e != cudaSuccess && !why.empty()) return fail(CSA_ERR_CUDA, why);
  return finish(e, "sparse decode launch");
}

int64_t csa_decode_workspace_bytes(int B, int Hq, int Hkv, int D, int num_parts) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0) return -1;
  int P = num_parts;
  if (P <= 0) {
    csa::Launch l;
    if (launch_ctx(nullptr, &l) != CSA_OK) return -1;
    P = csa::decode_default_parts(true, D, 128, l.num_sms);
  }
  return static_cast<int64_t>(workspace_layout(B, Hq, Hkv, D, P).total);
}

}  // extern "C"

namespace {
// csa_sparse_decode_merged, with the hybrid context when Kg/Vg are given.
csa_status merged_decode(const void* q, const void* K, const void* V, const void* Kg,
                         const void* Vg, int gist_scope, csa_dtype dtype, const int32_t* idx,
                         const int32_t* count, int kmax, const uint8_t* head_full, int B, int Hq,
                         int Hkv, int D, int64_t T, int L, float scale, int num_parts,
                         void* workspace, int64_t workspace_bytes, void* out,
                         csa_dtype out_dtype, float* lse_out, csa_stream stream, bool hybrid) {
  CSA_REQUIRE(valid_dtype(out_dtype), "out_dtype");
  CSA_TRY(decode_shape_checks(dtype, kmax, B, Hq, Hkv, D, T, L, scale, num_parts));
  CSA_SUPPORT(num_parts <= csa::kMergedMaxParts, "num_parts must be <= 256 for the merged decode");
  if (hybrid) {
    CSA_SUPPORT(dtype == CSA_BF16, "the hybrid context needs a bf16 cache");
    CSA_REQUIRE(gist_scope == CSA_GIST_SELECTED || gist_scope == CSA_GIST_ALL,
                "gist_scope must be CSA_GIST_SELECTED or CSA_GIST_ALL");
  }
  if (B == 0) return CSA_OK;
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  int P = 0;
  CSA_TRY(decode_ptr_checks(q, K, V, idx, count, head_full, dtype == CSA_BF16, D, L, num_parts, l, &P));
  CSA_SUPPORT(P <= csa::kMergedMaxParts, "num_parts must be <= 256 for the merged decode");
  if (hybrid) {
    CSA_TRY(check_ptr(Kg, "Kg"));
    CSA_TRY(check_ptr(Vg, "Vg"));
  }
  const WorkspaceLayout w = workspace_layout(B, Hq, Hkv, D, P);
  CSA_REQUIRE(workspace_bytes >= static_cast<int64_t>(w.total),
              "workspace smaller than csa_decode_workspace_bytes()");
  CSA_TRY(check_ptr(workspace, "workspace"));
  CSA_TRY(check_ptr(out, "out"));
  CSA_TRY(check_ptr(lse_out, "lse_out", false));
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  csa::MergeOut m{reinterpret_cast<int*>(ws + w.counters), out, out_dtype == CSA_BF16, lse_out};
  if (hybrid) {
    m.Kg = Kg;
    m.Vg = Vg;
    m.gist_selected = gist_scope == CSA_GIST_SELECTED;
  }
  m.allow_cluster = num_parts == 0;
  std::string why;
  cudaError_t e = csa::launch_decode(l, q, K, V, dtype == CSA_BF16, idx, count, kmax, head_full, B, Hq,
                                     Hkv, D, T, L, scale, P, P, reinterpret_cast<float*>(ws + w.o),
                                     reinterpret_cast<float*>(ws + w.lse), &m, &why);
  if (e != cudaSuccess && !why.empty()) return fail(CSA_ERR_CUDA, why);
  return finish(e, hybrid ? "hybrid merged decode launch" : "merged sparse decode launch");
}
}  // namespace

extern "C" {

csa_status csa_sparse_decode_merged(const void* q, const void* K, const void* V, csa_dtype dtype,
                                    const int32_t* idx, const int32_t* count, int kmax,
                                    const uint8_t* head_full, int B, int Hq, int Hkv, int D,
                                    int64_t T, int L, float scale, int num_parts, void* workspace,
                                    int64_t workspace_bytes, void* out, csa_dtype out_dtype,
                                    float* lse_out, csa_stream stream) {
  return merged_decode(q, K, V, nullptr, nullptr, 0, dtype, idx, count, kmax, head_full, B, Hq, Hkv,
                       D, T, L, scale, num_parts, workspace, workspace_bytes, out, out_dtype,
                       lse_out, stream, false);
}

csa_status csa_sparse_decode_merged_hybrid(const void* q, const void* K, const void* V,
                                           const void* Kg, const void* Vg, int gist_scope,
                                           csa_dtype dtype, const int32_t* idx,
                                           const int32_t* count, int kmax,
                                           const uint8_t* head_full, int B, int Hq, int Hkv,
                                           int D, int64_t T, int L, float scale, int num_parts,
                                           void* workspace, int64_t workspace_bytes, void* out,
                                           csa_dtype out_dtype, float* lse_out,
                                           csa_stream stream) {
  return merged_decode(q, K, V, Kg, Vg, gist_scope, dtype, idx, count, kmax, head_full, B, Hq, Hkv, D, T, L,
                       scale, num_parts, workspace, workspace_bytes, out, out_dtype, lse_out,
                       stream, true);
}

namespace {
csa_status score_select_topk_common(const void* q, csa_dtype q_dtype, const float* proj, int R,
                                    const float* summ, int B, int Hq, int Hkv, int D, int C,
                                    const uint8_t* head_full, int k_free, int n_sink, int n_local,
                                    int32_t* idx, int32_t* count, int kmax, csa_stream stream,
                                    bool per_head_union, bool check_only = false) {
  CSA_REQUIRE(valid_dtype(q_dtype), "q_dtype");
  CSA_REQUIRE(kmax > 0, "kmax must be positive");
  CSA_REQUIRE(B >= 0 && Hq > 0 && Hkv > 0 && D > 0 && C >= 0 && k_free >= 0 && n_sink >= 0 &&
                  n_local >= 0,
              "bad sizes");
  CSA_REQUIRE(Hq % Hkv == 0, "Hq must be a multiple of Hkv");
  CSA_SUPPORT(D <= 1024 && C <= 32768, "D <= 1024 and C <= 32768");
  const int Ds = proj ? R : D;
  CSA_SUPPORT(Ds == 16 || Ds == 32 || Ds == 64 || Ds == 128, "summary width must be 16, 32, 64 or 128");
  if (per_head_union) {
    const int64_t need = std::min<int64_t>(
        C, static_cast<int64_t>(Hq / Hkv) * k_free + n_sink + n_local);
    CSA_REQUIRE(kmax >= need, "kmax < min(C, (Hq/Hkv) * k_free + n_sink + n_local)");
  } else {
    const int64_t need = std::min<int64_t>(C, static_cast<int64_t>(k_free) + n_sink + n_local);
    CSA_REQUIRE(kmax >= need, "kmax < min(C, k_free + n_sink + n_local)");
  }
  if (B == 0 || C == 0) return CSA_OK;
  CSA_TRY(check_ptr(q, "q"));
  CSA_TRY(check_ptr(proj, "proj", false));
  CSA_TRY(check_ptr(summ, "summ"));
  CSA_TRY(check_ptr(head_full, "head_full", false));
  CSA_TRY(check_ptr(idx, "idx"));
  CSA_TRY(check_ptr(count, "count"));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  if (check_only) return CSA_OK;
  return finish(csa::launch_score_select_topk(l, q, q_dtype == CSA_BF16, proj, R, summ, B, Hq, Hkv, D,
                                              C, head_full, k_free, n_sink, n_local, idx, count, kmax,
                                              per_head_union),
                per_head_union ? "score_select_topk_union launch" : "score_select_topk launch");
}
}  // namespace

csa_status csa_score_select_topk(const void* q, csa_dtype q_dtype, const float* proj, int R,
                                 const float* summ, int B, int Hq, int Hkv, int D, int C,
                                 const uint8_t* head_full, int k_free, int n_sink, int n_local,
                                 int32_t* idx, int32_t* count, int kmax, csa_stream stream) {
  return score_select_topk_common(q, q_dtype, proj, R, summ, B, Hq, Hkv, D, C, head_full, k_free,
                                  n_sink, n_local, idx, count, kmax, stream, false);
}

csa_status csa_score_select_topk_union(const void* q, csa_dtype q_dtype, const float* proj, int R,
                                       const float* summ, int B, int Hq, int Hkv, int D, int C,
                                       const uint8_t* head_full, int k_free, int n_sink,
                                       int n_local, int32_t* idx, int32_t* count, int kmax,
                                       csa_stream stream) {
  return score_select_topk_common(q, q_dtype, proj, R, summ, B, Hq, Hkv, D, C, head_full, k_free,
                                  n_sink, n_local, idx, count, kmax, stream, true);
}

}  // extern "C"

namespace {
csa_status score_select_topp_impl(const void* q, csa_dtype q_dtype, const float* proj, int R,
                                  const float* summ, int B, int Hq, int Hkv, int D, int C,
                                  const uint8_t* head_full, float logit_scale, float p, int budget,
                                  int n_sink, int n_local, int32_t* idx, int32_t* count, int kmax,
                                  int32_t* n_p_out, csa_stream stream, bool check_only,
                                  bool after_query_copy = false) {
  CSA_REQUIRE(valid_dtype(q_dtype), "q_dtype");
  CSA_REQUIRE(kmax > 0, "kmax must be positive");
  CSA_REQUIRE(B >= 0 && Hq > 0 && Hkv > 0 && D > 0 && C > 0 && n_sink >= 0 && n_local >= 0,
              "bad sizes");
  CSA_REQUIRE(Hq % Hkv == 0, "Hq must be a multiple of Hkv");
  CSA_REQUIRE(p > 0.f && p <= 1.f, "p must be in (0, 1]");
  CSA_REQUIRE(budget >= 1, "budget must be >= 1");
  CSA_REQUIRE(logit_scale == logit_scale, "logit_scale is NaN");
  CSA_SUPPORT(budget <= 2048 && C <= 32768 && D <= 1024, "budget <= 2048, C <= 32768, D <= 1024");
  const int Ds = proj ? R : D;
  CSA_SUPPORT(Ds == 16 || Ds == 32 || Ds == 64 || Ds == 128, "summary width must be 16, 32, 64 or 128");
  const int64_t need = std::min<int64_t>(C, static_cast<int64_t>(budget) + n_sink + n_local);
  CSA_REQUIRE(kmax >= need, "kmax < min(C, budget + n_sink + n_local)");
  if (B == 0) return CSA_OK;
  CSA_TRY(check_ptr(q, "q"));
  CSA_TRY(check_ptr(proj, "proj", false));
  CSA_TRY(check_ptr(summ, "summ"));
  CSA_TRY(check_ptr(head_full, "head_full", false));
  CSA_TRY(check_ptr(idx, "idx"));
  CSA_TRY(check_ptr(count, "count"));
  CSA_TRY(check_ptr(n_p_out, "n_p_out", false));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  if (check_only) return CSA_OK;
  l.after_query_copy = after_query_copy;
  return finish(csa::launch_score_select_topp(l, q, q_dtype == CSA_BF16, proj, R, summ, B, Hq, Hkv, D,
                                              C, head_full, logit_scale, p, budget, n_sink, n_local,
                                              idx, count, kmax, n_p_out),
                "score_select_topp launch");
}
}  // namespace

extern "C" {

csa_status csa_score_select_topp(const void* q, csa_dtype q_dtype, const float* proj, int R,
                                 const float* summ, int B, int Hq, int Hkv, int D, int C,
                                 const uint8_t* head_full, float logit_scale, float p, int budget,
                                 int n_sink, int n_local, int32_t* idx, int32_t* count, int kmax,
                                 int32_t* n_p_out, csa_stream stream) {
  return score_select_topp_impl(q, q_dtype, proj, R, summ, B, Hq, Hkv, D, C, head_full,
                                logit_scale, p, budget, n_sink, n_local, idx, count, kmax, n_p_out,
                                stream, false);
}

}  // extern "C"

namespace {

// Pinned host memory (page-locked by cudaHostAlloc or cudaHostRegister):
// the only host memory an asynchronous copy, and a CUDA graph, can take.
csa_status check_host_ptr(const void* p, const char* name, bool required = true) {
  if (p == nullptr) {
    if (!required) return CSA_OK;
    return fail(CSA_ERR_INVALID_ARG, std::string(name) + " is NULL");
  }
  cudaPointerAttributes a;
  cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(CSA_ERR_INVALID_ARG, std::string(name) + " is not a valid pointer");
  }
  if (a.type != cudaMemoryTypeHost)
    return fail(CSA_ERR_INVALID_ARG, std::string(name) + " is not pinned host memory");
  return CSA_OK;
}

// Device address of pinned host memory (the same address under unified
// addressing), or NULL when the memory is not mapped or the address is not
// 16-byte aligned.
void* mapped_ptr(const void* h) {
  void* dp = nullptr;
  if (cudaHostGetDevicePointer(&dp, const_cast<void*>(h), 0) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return reinterpret_cast<uintptr_t>(dp) % 16 == 0 ? dp : nullptr;
}

// Host side of a step: where the query comes from and where the result goes.
struct HostIO {
  const void* q = nullptr;  // the query's source, or NULL (d->q already holds it)
  bool q_mapped = false;    // q is a device address of pinned host memory: copied by the SMs
  bool out_mapped = false;  // d->out (and d->lse_out) are device addresses of pinned host memory
};

// The decode step; with io->q the query is first copied into d->q on the
// stream, after every check of the decode's own arguments.
csa_status decode_step(const csa_decode_step_desc* d, const HostIO* io, csa_stream stream) {
  CSA_REQUIRE(d != nullptr, "descriptor is NULL");
  CSA_REQUIRE(d->mode == CSA_SELECT_TOPK || d->mode == CSA_SELECT_TOPP ||
                  d->mode == CSA_SELECT_HIER || d->mode == CSA_SELECT_TOPK_UNION,
              "mode must be CSA_SELECT_TOPK, CSA_SELECT_TOPP, CSA_SELECT_HIER or "
              "CSA_SELECT_TOPK_UNION");
  CSA_REQUIRE(valid_dtype(d->out_dtype), "out_dtype");
  CSA_TRY(decode_shape_checks(CSA_BF16, d->kmax, d->B, d->Hq, d->Hkv, d->D, d->T, d->L, d->scale,
                              d->num_parts));
  CSA_SUPPORT(d->num_parts <= csa::kMergedMaxParts, "num_parts must be <= 256");
  if (d->B == 0) return CSA_OK;
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  // decode arguments first, so that a rejected call enqueues nothing
  int P = 0;
  CSA_TRY(decode_ptr_checks(d->q, d->K, d->V, d->idx, d->count, d->head_full, true, d->D, d->L,
                            d->num_parts, l, &P));
  if (d->num_parts == 0) P = std::min(csa::kMergedMaxParts, l.num_sms);
  // The selection runs one CTA per (batch, KV head) unit; while it runs the
  // decode CTAs that find no free SM start late.  Those (the last ones of the
  // grid) take no full-head work, only the selected chunks, which cannot
  // start before the selection ends anyway.  Counted without reading
  // head_full, so the call stays free of host-device copies.
  int late = 0;
  if (d->head_full != nullptr)
    late = std::max(0, std::min(P - 1, P + d->B * d->Hkv - l.num_sms));
  const WorkspaceLayout w = workspace_layout(d->B, d->Hq, d->Hkv, d->D, P);
  CSA_REQUIRE(d->workspace_bytes >= static_cast<int64_t>(w.total),
              "workspace smaller than csa_decode_workspace_bytes()");
  CSA_TRY(check_ptr(d->workspace, "workspace"));
  if (io == nullptr || !io->out_mapped) {
    CSA_TRY(check_ptr(d->out, "out"));
    CSA_TRY(check_ptr(d->lse_out, "lse_out", false));
  }
  const bool hybrid = d->Kg != nullptr || d->Vg != nullptr;
  if (hybrid) {  // both or neither
    CSA_TRY(check_ptr(d->Kg, "Kg"));
    CSA_TRY(check_ptr(d->Vg, "Vg"));
    CSA_REQUIRE(d->gist_scope == CSA_GIST_SELECTED || d->gist_scope == CSA_GIST_ALL,
                "gist_scope must be CSA_GIST_SELECTED or CSA_GIST_ALL");
  }
  const int C = static_cast<int>(d->T / d->L);
  // the selection scores with the pre-RoPE query when one is given
  const void* qs = d->q_score != nullptr ? d->q_score : d->q;
  if (d->q_score != nullptr) CSA_TRY(check_ptr(d->q_score, "q_score"));
  // after_copy: the query copy kernel runs right before the selection (the
  // top-p selection then starts behind it with programmatic dependent launch)
  auto selection = [&](bool check_only, bool after_copy) -> csa_status {
    if (d->mode == CSA_SELECT_TOPK || d->mode == CSA_SELECT_TOPK_UNION)
      return score_select_topk_common(qs, CSA_BF16, d->proj, d->R, d->summ, d->B, d->Hq, d->Hkv,
                                      d->D, C, d->head_full, d->k_free, d->n_sink, d->n_local,
                                      d->idx, d->count, d->kmax, stream,
                                      d->mode == CSA_SELECT_TOPK_UNION, check_only);
    if (d->mode == CSA_SELECT_TOPP)
      return score_select_topp_impl(qs, CSA_BF16, d->proj, d->R, d->summ, d->B, d->Hq, d->Hkv,
                                    d->D, C, d->head_full, d->logit_scale, d->p, d->budget,
                                    d->n_sink, d->n_local, d->idx, d->count, d->kmax, d->n_p_out,
                                    stream, check_only, after_copy);
    return select_hier_impl(qs, CSA_BF16, d->meta, d->summ, d->B, d->Hq, d->Hkv, d->D, C, d->Gm,
                            d->top_meta, d->k_free, d->n_sink, d->n_local, d->idx, d->count,
                            d->kmax, stream, check_only);
  };
  // every argument of the selection too, before the query copy is enqueued
  CSA_TRY(selection(true, false));
  bool q_by_kernel = false;  // the query copied by a kernel just before the selection
  if (io != nullptr && io->q != nullptr) {
    const size_t nq = static_cast<size_t>(d->B) * d->Hq * d->D * sizeof(__nv_bfloat16);
    q_by_kernel = io->q_mapped && nq >= 16;
    if (io->q_mapped)
      CSA_TRY(finish(csa::launch_copy16(l, io->q, const_cast<void*>(d->q), nq),
                     "query copy to the device"));
    else
      CSA_TRY(finish(cudaMemcpyAsync(const_cast<void*>(d->q), io->q, nq, cudaMemcpyHostToDevice,
                                     l.stream),
                     "query copy to the device"));
  }
  const csa_status st = selection(false, q_by_kernel && d->q_score == nullptr);
  if (st != CSA_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(d->workspace);
  csa::MergeOut m{reinterpret_cast<int*>(ws + w.counters), d->out, d->out_dtype == CSA_BF16,
                  d->lse_out, true, late};
  if (hybrid) {
    m.Kg = d->Kg;
    m.Vg = d->Vg;
    m.gist_selected = d->gist_scope == CSA_GIST_SELECTED;
  }
  m.allow_cluster = d->num_parts == 0;
  std::string why;
  cudaError_t e = csa::launch_decode(l, d->q, d->K, d->V, true, d->idx, d->count, d->kmax,
                                     d->head_full, d->B, d->Hq, d->Hkv, d->D, d->T, d->L, d->scale,
                                     P, P, reinterpret_cast<float*>(ws + w.o),
                                     reinterpret_cast<float*>(ws + w.lse), &m, &why);
  if (e != cudaSuccess && !why.empty()) return fail(CSA_ERR_CUDA, why);
  return finish(e, "decode step launch");
}

}  // namespace

extern "C" {

csa_status csa_decode_step(const csa_decode_step_desc* d, csa_stream stream) {
  return decode_step(d, nullptr, stream);
}

csa_status csa_decode_step_host(const csa_decode_step_desc* d, const void* q_host, void* out_host,
                                float* lse_host, csa_stream stream) {
  CSA_REQUIRE(d != nullptr, "descriptor is NULL");
  CSA_SUPPORT(d->q_score == nullptr,
              "q_score (the RoPE-aware split) needs the query rotated on the device: use "
              "csa_rope and csa_decode_step");
  CSA_TRY(check_host_ptr(q_host, "q_host"));
  CSA_TRY(check_host_ptr(out_host, "out_host"));
  CSA_TRY(check_host_ptr(lse_host, "lse_host", false));
  CSA_REQUIRE(lse_host == nullptr || d->lse_out != nullptr, "lse_host needs lse_out");
  CSA_TRY(check_ptr(d->out, "out"));
  CSA_TRY(check_ptr(d->lse_out, "lse_out", false));
  // Mapped host memory (every pinned allocation under unified addressing):
  // the SMs read the query and the decode stores its result straight into
  // the host buffers, with no copy-engine transfer on either side.
  HostIO io;
  void* qd = mapped_ptr(q_host);
  io.q = qd != nullptr ? qd : q_host;
  io.q_mapped = qd != nullptr;
  void* od = mapped_ptr(out_host);
  void* ld = lse_host != nullptr ? mapped_ptr(lse_host) : nullptr;
  csa_decode_step_desc dd = *d;
  if (od != nullptr && (lse_host == nullptr || ld != nullptr)) {
    io.out_mapped = true;
    dd.out = od;
    dd.lse_out = lse_host != nullptr ? static_cast<float*>(ld) : d->lse_out;
  }
  CSA_TRY(decode_step(&dd, &io, stream));
  if (d->B == 0 || io.out_mapped) return CSA_OK;
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  const size_t rows = static_cast<size_t>(d->B) * d->Hq;
  const size_t no = rows * d->D * (d->out_dtype == CSA_BF16 ? 2 : 4);
  CSA_TRY(finish(cudaMemcpyAsync(out_host, d->out, no, cudaMemcpyDeviceToHost, l.stream),
                 "output copy to the host"));
  if (lse_host != nullptr)
    CSA_TRY(finish(cudaMemcpyAsync(lse_host, d->lse_out, rows * sizeof(float),
                                   cudaMemcpyDeviceToHost, l.stream),
                   "lse copy to the host"));
  return CSA_OK;
}

csa_status csa_lse_merge(const float* o_part, const float* lse_part, int rows, int max_splits, int D,
                         void* out, csa_dtype out_dtype, float* lse_out, csa_stream stream) {
  CSA_REQUIRE(valid_dtype(out_dtype), "out_dtype");
  CSA_REQUIRE(rows >= 0 && max_splits > 0 && D > 0, "bad sizes");
  CSA_SUPPORT(D % 4 == 0 && D <= 512, "D must be a multiple of 4, <= 512");
  CSA_SUPPORT(max_splits <= 16384, "max_splits must be <= 16384");
  if (rows == 0) return CSA_OK;
  CSA_TRY(check_ptr(o_part, "o_part"));
  CSA_TRY(check_ptr(lse_part, "lse_part"));
  CSA_TRY(check_ptr(out, "out"));
  CSA_TRY(check_ptr(lse_out, "lse_out", false));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  return finish(csa::launch_merge(l, o_part, lse_part, rows, max_splits, D, out, out_dtype == CSA_BF16,
                                  lse_out),
                "lse merge launch");
}

csa_status csa_block_sparse_prefill(const void* Q, const void* K, const void* V, const int32_t* idx,
                                    const int32_t* count, int kmax, int B, int S, int Hq, int Hkv,
                                    int D, int tile_m, int L, float scale, void* O,
                                    csa_stream stream) {
  CSA_REQUIRE(B >= 0 && S >= 0 && Hq > 0 && Hkv > 0 && D > 0 && tile_m > 0 && L > 0 && kmax > 0,
              "bad sizes");
  CSA_REQUIRE(Hq % Hkv == 0, "Hq must be a multiple of Hkv");
  CSA_REQUIRE(S % tile_m == 0 && S % L == 0, "S must be a multiple of tile_m and of L");
  CSA_SUPPORT(D == 128 && tile_m == 64 && L == 64 && Hq / Hkv == 4,
              "implemented for D = 128, tile_m = L = 64, Hq/Hkv = 4");
  CSA_SUPPORT(static_cast<int64_t>(B) * Hkv * S < 2147483648LL && static_cast<int64_t>(B) * S < 2147483648LL,
              "B*Hkv*S must be < 2^31");
  CSA_REQUIRE(scale == scale, "scale is NaN");
  if (static_cast<int64_t>(B) * S == 0) return CSA_OK;
  CSA_TRY(check_ptr(Q, "Q"));
  CSA_TRY(check_ptr(K, "K"));
  CSA_TRY(check_ptr(V, "V"));
  CSA_TRY(check_ptr(idx, "idx"));
  CSA_TRY(check_ptr(count, "count"));
  CSA_TRY(check_ptr(O, "O"));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  std::string why;
  cudaError_t e = csa::launch_prefill(l, Q, K, V, idx, count, kmax, B, S, Hq, Hkv, D, tile_m, L, scale, O,
                                      &why);
  if (e != cudaSuccess && !why.empty()) return fail(CSA_ERR_CUDA, why);
  return finish(e, "block-sparse prefill launch");
}


// ---------------------------------------------------------------- token-level sparsity

int64_t csa_token_importance_scratch_bytes(int B, int S, int Hq, int Hkv, int n_obs) {
  if (B < 0 || S < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || n_obs <= 0) return -1;
  return static_cast<int64_t>(csa::token_importance_scratch_bytes(B, S, Hkv, Hq / Hkv, n_obs));
}

namespace {
csa_status importance_checks(const void* Q, const void* K, int B, int S, int Hq, int Hkv, int D,
                             int n_obs, float scale) {
  CSA_REQUIRE(B >= 0 && S >= 0 && Hq > 0 && Hkv > 0 && D > 0 && n_obs > 0, "bad sizes");
  CSA_REQUIRE(Hq % Hkv == 0, "Hq must be a multiple of Hkv");
  CSA_REQUIRE(n_obs <= S || S == 0, "n_obs must be <= S");
  CSA_SUPPORT(D == 64 || D == 128, "D must be 64 or 128");
  CSA_SUPPORT(n_obs % 8 == 0 && (Hq / Hkv) * n_obs <= 512,
              "n_obs a multiple of 8 and (Hq/Hkv) * n_obs <= 512");
  CSA_REQUIRE(scale == scale && scale > 0.f, "scale must be positive");
  if (static_cast<int64_t>(B) * S == 0) return CSA_OK;
  CSA_TRY(check_ptr(Q, "Q"));
  CSA_TRY(check_ptr(K, "K"));
  return CSA_OK;
}

// Sequences longer than 32768 tokens (up to 131072): the coverage budget and
// the per-head token choice then run only on their cluster paths, which hold
// S / 8 values per CTA and need B * 8 and B * Hkv * 8 CTAs on the SMs.
constexpr int kTokenMaxS = 131072;
csa_status token_long_check(int B, int Hkv, int S, const csa::Launch& l, bool budget, bool select) {
  if (S <= 32768) return CSA_OK;
  CSA_SUPPORT(S <= kTokenMaxS, "S must be <= 131072");
  if (budget)
    CSA_SUPPORT(csa::token_budget_cluster_fits(B, l.num_sms),
                "S > 32768 needs B * 8 <= the number of SMs");
  if (select)
    CSA_SUPPORT(csa::topk_cluster_fits(B * Hkv, S, l.num_sms),
                "S > 32768 needs B * Hkv * 8 <= the number of SMs");
  return CSA_OK;
}
}  // namespace

csa_status csa_token_importance(const void* Q, const void* K, int B, int S, int Hq, int Hkv,
                                int D, int n_obs, float scale, float* imp, void* scratch,
                                int64_t scratch_bytes, csa_stream stream) {
  CSA_TRY(importance_checks(Q, K, B, S, Hq, Hkv, D, n_obs, scale));
  if (static_cast<int64_t>(B) * S == 0) return CSA_OK;
  CSA_REQUIRE(scratch_bytes >= csa_token_importance_scratch_bytes(B, S, Hq, Hkv, n_obs),
              "scratch smaller than csa_token_importance_scratch_bytes()");
  CSA_TRY(check_ptr(imp, "imp"));
  CSA_TRY(check_ptr(scratch, "scratch"));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  std::string why;
  const cudaError_t e = csa::launch_token_importance(l, Q, K, B, S, Hq, Hkv, D, n_obs, scale, imp,
                                                     static_cast<float*>(scratch), &why);
  if (e != cudaSuccess && !why.empty()) return fail(CSA_ERR_CUDA, why);
  return finish(e, "token importance launch");
}

csa_status csa_token_budget(const float* imp, int B, int S, int Hkv, float tau, int tile,
                            int32_t* k_seq, int32_t* k_unit, csa_stream stream) {
  CSA_REQUIRE(B >= 0 && S >= 0 && Hkv > 0 && tile > 0, "bad sizes");
  CSA_REQUIRE(tau == tau && tau >= 0.f && tau < 1.f, "tau must be in [0, 1)");
  CSA_SUPPORT(S <= kTokenMaxS, "S must be <= 131072");
  if (B == 0) return CSA_OK;
  CSA_TRY(check_ptr(imp, "imp"));
  CSA_TRY(check_ptr(k_seq, "k_seq"));
  CSA_TRY(check_ptr(k_unit, "k_unit"));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  CSA_TRY(token_long_check(B, Hkv, S, l, true, false));
  return finish(csa::launch_token_budget(l, imp, B, S, Hkv, tau, tile, k_seq, k_unit),
                "token budget launch");
}

namespace {
struct TsaLayout {
  size_t imp, scratch, k_unit, idx, count, qc, kc, vc, oc, inv, total;
};
TsaLayout tsa_layout(int B, int S, int Hq, int Hkv, int D, int n_obs) {
  auto r = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t U = static_cast<size_t>(B) * Hkv;
  TsaLayout w;
  size_t o = 0;
  w.imp = o; o += r(U * S * 4);
  w.scratch = o; o += r(csa::token_importance_scratch_bytes(B, S, Hkv, Hq / Hkv, n_obs));
  w.k_unit = o; o += r(U * 4);
  w.idx = o; o += r(U * S * 4);
  w.count = o; o += r(U * 4);
  w.qc = o; o += r(static_cast<size_t>(B) * S * Hq * D * 2);
  w.kc = o; o += r(U * S * D * 2);
  w.vc = o; o += r(U * S * D * 2);
  w.oc = o; o += r(static_cast<size_t>(B) * S * Hq * D * 2);
  w.inv = o; o += r(U * S * 4);
  w.total = o;
  return w;
}
}  // namespace

int64_t csa_token_sparse_workspace_bytes(int B, int S, int Hq, int Hkv, int D, int n_obs) {
  if (B < 0 || S < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || D <= 0 || n_obs <= 0 ||
      S % 64 != 0)
    return -1;
  return static_cast<int64_t>(tsa_layout(B, S, Hq, Hkv, D, n_obs).total);
}

csa_status csa_token_sparse_prefill(const void* Q, const void* K, const void* V, int B, int S,
                                    int Hq, int Hkv, int D, int n_obs, float tau, float scale,
                                    void* workspace, int64_t workspace_bytes, void* O,
                                    int32_t* budget_out, csa_stream stream) {
  CSA_TRY(importance_checks(Q, K, B, S, Hq, Hkv, D, n_obs, scale));
  CSA_REQUIRE(tau == tau && tau >= 0.f && tau < 1.f, "tau must be in [0, 1)");
  CSA_REQUIRE(S % 64 == 0, "S must be a multiple of 64");
  CSA_SUPPORT(D == 128 && Hq / Hkv == 4 && S <= kTokenMaxS,
              "implemented for D = 128, Hq/Hkv = 4 and S <= 131072");
  if (static_cast<int64_t>(B) * S == 0) return CSA_OK;
  const TsaLayout w = tsa_layout(B, S, Hq, Hkv, D, n_obs);
  CSA_REQUIRE(workspace_bytes >= static_cast<int64_t>(w.total),
              "workspace smaller than csa_token_sparse_workspace_bytes()");
  CSA_TRY(check_ptr(V, "V"));
  CSA_TRY(check_ptr(workspace, "workspace"));
  CSA_TRY(check_ptr(O, "O"));
  CSA_TRY(check_ptr(budget_out, "budget_out"));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  CSA_TRY(token_long_check(B, Hkv, S, l, true, true));
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* imp = reinterpret_cast<float*>(ws + w.imp);
  int32_t* k_unit = reinterpret_cast<int32_t*>(ws + w.k_unit);
  int32_t* idx = reinterpret_cast<int32_t*>(ws + w.idx);
  int32_t* cnt = reinterpret_cast<int32_t*>(ws + w.count);
  const int U = B * Hkv;
  std::string why;
  cudaError_t e = csa::launch_token_importance(l, Q, K, B, S, Hq, Hkv, D, n_obs, scale, imp,
                                               reinterpret_cast<float*>(ws + w.scratch), &why);
  if (e != cudaSuccess && !why.empty()) return fail(CSA_ERR_CUDA, why);
  if (e == cudaSuccess) e = csa::launch_token_budget(l, imp, B, S, Hkv, tau, 64, budget_out, k_unit);
  bool inv_ready = false;  // the selection may write the position -> slot map itself
  if (e == cudaSuccess)  // each KV head's own top tokens under the (rounded) budget
    e = csa::launch_select_topk(l, imp, U, S, nullptr, 0, 0, 0, idx, cnt, S, k_unit, 0, 0, 0,
                                reinterpret_cast<int32_t*>(ws + w.inv), &inv_ready);
  if (e != cudaSuccess) return finish(e, "token selection launch");
  // Compress, attend, decompress with no read-back of the budgets: the
  // buffers are laid out for S kept tokens, the gather writes the kept rows
  // of each unit only, and the dense causal attention takes the tiles below
  // each unit's budget (tiles past it are never visited and write nothing).
  void* Qc = ws + w.qc;
  void* Kc = ws + w.kc;
  void* Vc = ws + w.vc;
  void* Oc = ws + w.oc;
  e = csa::launch_tsa_gather(l, Q, K, V, idx, cnt, S, B, S, S, Hq, Hkv, D, Qc, Kc, Vc);
  if (e == cudaSuccess)
    e = csa::launch_prefill(l, Qc, Kc, Vc, nullptr, nullptr, 0, B, S, Hq, Hkv, D, 64, 64, scale, Oc,
                            &why, /*skip_empty=*/true, k_unit);
  if (e != cudaSuccess && !why.empty()) return fail(CSA_ERR_CUDA, why);
  if (e == cudaSuccess)
    e = csa::launch_tsa_scatter(l, Oc, idx, cnt, S, B, S, S, Hq, Hkv, D,
                                reinterpret_cast<int32_t*>(ws + w.inv), O, inv_ready);
  return finish(e, "token sparse prefill launch");
}


/* ---- the steps of csa_token_sparse_prefill as separate calls ---- */

namespace {
csa_status token_shape_checks(int B, int S, int Hq, int Hkv, int D) {
  CSA_REQUIRE(B >= 0 && S >= 0 && Hq > 0 && Hkv > 0 && D > 0, "bad sizes");
  CSA_REQUIRE(Hq % Hkv == 0, "Hq must be a multiple of Hkv");
  CSA_REQUIRE(S % 64 == 0, "S must be a multiple of 64");
  CSA_SUPPORT(D == 128 && Hq / Hkv == 4 && S <= kTokenMaxS,
              "implemented for D = 128, Hq/Hkv = 4 and S <= 131072");
  return CSA_OK;
}
}  // namespace

csa_status csa_token_select(const float* imp, int B, int S, int Hkv, const int32_t* k_unit,
                            int32_t* idx, int32_t* count, csa_stream stream) {
  CSA_REQUIRE(B >= 0 && S >= 0 && Hkv > 0, "bad sizes");
  CSA_SUPPORT(S <= kTokenMaxS, "S must be <= 131072");
  if (static_cast<int64_t>(B) * S == 0) return CSA_OK;
  CSA_TRY(check_ptr(imp, "imp"));
  CSA_TRY(check_ptr(k_unit, "k_unit"));
  CSA_TRY(check_ptr(idx, "idx"));
  CSA_TRY(check_ptr(count, "count"));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  CSA_TRY(token_long_check(B, Hkv, S, l, false, true));
  return finish(csa::launch_select_topk(l, imp, B * Hkv, S, nullptr, 0, 0, 0, idx, count, S,
                                        k_unit),
                "token select launch");
}

csa_status csa_token_compress(const void* Q, const void* K, const void* V, const int32_t* idx,
                              const int32_t* count, int B, int S, int Hq, int Hkv, int D,
                              void* Qc, void* Kc, void* Vc, csa_stream stream) {
  CSA_TRY(token_shape_checks(B, S, Hq, Hkv, D));
  if (static_cast<int64_t>(B) * S == 0) return CSA_OK;
  CSA_TRY(check_ptr(Q, "Q"));
  CSA_TRY(check_ptr(K, "K"));
  CSA_TRY(check_ptr(V, "V"));
  CSA_TRY(check_ptr(Qc, "Qc"));
  CSA_TRY(check_ptr(Kc, "Kc"));
  CSA_TRY(check_ptr(Vc, "Vc"));
  CSA_TRY(check_ptr(idx, "idx"));
  CSA_TRY(check_ptr(count, "count"));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  return finish(csa::launch_tsa_gather(l, Q, K, V, idx, count, S, B, S, S, Hq, Hkv, D, Qc, Kc, Vc),
                "token compress launch");
}

csa_status csa_token_attend(const void* Qc, const void* Kc, const void* Vc,
                            const int32_t* k_unit, int B, int S, int Hq, int Hkv, int D,
                            float scale, void* Oc, csa_stream stream) {
  CSA_TRY(token_shape_checks(B, S, Hq, Hkv, D));
  CSA_REQUIRE(scale == scale && scale > 0.f, "scale must be positive");
  if (static_cast<int64_t>(B) * S == 0) return CSA_OK;
  CSA_TRY(check_ptr(Qc, "Qc"));
  CSA_TRY(check_ptr(Kc, "Kc"));
  CSA_TRY(check_ptr(Vc, "Vc"));
  CSA_TRY(check_ptr(Oc, "Oc"));
  CSA_TRY(check_ptr(k_unit, "k_unit"));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  std::string why;
  const cudaError_t e = csa::launch_prefill(l, Qc, Kc, Vc, nullptr, nullptr, 0, B, S, Hq, Hkv, D,
                                            64, 64, scale, Oc, &why, /*skip_empty=*/true, k_unit);
  if (e != cudaSuccess && !why.empty()) return fail(CSA_ERR_CUDA, why);
  return finish(e, "token attend launch");
}

int64_t csa_token_decompress_scratch_bytes(int B, int S, int Hkv) {
  if (B < 0 || S < 0 || Hkv <= 0) return -1;
  return static_cast<int64_t>(B) * Hkv * S * 4;
}

csa_status csa_token_decompress(const void* Oc, const int32_t* idx, const int32_t* count, int B,
                                int S, int Hq, int Hkv, int D, void* scratch,
                                int64_t scratch_bytes, void* O, csa_stream stream) {
  CSA_TRY(token_shape_checks(B, S, Hq, Hkv, D));
  if (static_cast<int64_t>(B) * S == 0) return CSA_OK;
  CSA_REQUIRE(scratch_bytes >= csa_token_decompress_scratch_bytes(B, S, Hkv),
              "scratch smaller than csa_token_decompress_scratch_bytes()");
  CSA_TRY(check_ptr(Oc, "Oc"));
  CSA_TRY(check_ptr(idx, "idx"));
  CSA_TRY(check_ptr(count, "count"));
  CSA_TRY(check_ptr(scratch, "scratch"));
  CSA_TRY(check_ptr(O, "O"));
  csa::Launch l;
  CSA_TRY(launch_ctx(stream, &l));
  return finish(csa::launch_tsa_scatter(l, Oc, idx, count, S, B, S, S, Hq, Hkv, D,
                                        static_cast<int32_t*>(scratch), O),
                "token decompress launch");
}

}  // extern "C"
