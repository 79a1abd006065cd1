// Rotary position embedding of rows of a K cache or of queries.
//
// The RTPurbo review ("Full Attention Strikes Back", section 1, "Low-
// dimensional Projection") scores chunks on a projection taken before RoPE,
// because RoPE makes q.k depend on the distance between positions; the
// attention itself runs on the rotated queries and keys.  This kernel makes
// the rotated copies: row r of x (D values) sits at position
// pos0 + (r mod period) and each pair (x_i, x_{i+D/2}), i < D/2, turns by the
// angle position * theta^(-2i/D) (the rotate-half pairing).
//
// Elementwise and bound by HBM.  One thread per pair column i (a block holds
// D/2 columns x ROWS rows), so each thread computes its frequency once; the
// angle is formed and reduced modulo 2 pi in double, so that positions in
// the millions keep their accuracy, and only the reduced angle goes to the
// single-precision sine and cosine.
#include "internal.h"

namespace csa {
namespace {

constexpr int kRopeThreads = 256;

template <typename T>
__device__ __forceinline__ float load_f(const T* p);
template <>
__device__ __forceinline__ float load_f<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float load_f<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

__device__ __forceinline__ void store_f(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_f(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

template <typename T>
__global__ void __launch_bounds__(kRopeThreads) rope_kernel(const T* x, T* y, int64_t rows, int D,
                                                            int64_t period, int64_t pos0,
                                                            double log2_theta) {
  const int h = D / 2;
  const int rows_per_block = kRopeThreads / h;
  const int i = threadIdx.x % h, rr = threadIdx.x / h;
  if (rr >= rows_per_block) return;
  // theta^(-2i/D), in double
  const double freq = exp2(-2.0 * i / D * log2_theta);
  constexpr double kTwoPi = 6.283185307179586476925286766559;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * rows_per_block + rr; r < rows;
       r += static_cast<int64_t>(gridDim.x) * rows_per_block) {
    const double pos = static_cast<double>(pos0 + r % period);
    double a = pos * freq;
    a -= kTwoPi * rint(a / kTwoPi);
    float sn, cs;
    sincosf(static_cast<float>(a), &sn, &cs);
    const T* xr = x + r * D;
    const float u = load_f(xr + i), v = load_f(xr + i + h);
    T* yr = y + r * D;
    store_f(yr + i, u * cs - v * sn);
    store_f(yr + i + h, v * cs + u * sn);
  }
}

}  // namespace

cudaError_t launch_rope(const Launch& l, const void* x, void* y, bool bf16, int64_t rows, int D,
                        int64_t period, int64_t pos0, float theta) {
  if (rows == 0) return cudaSuccess;
  const int h = D / 2;
  const int rows_per_block = kRopeThreads / h;
  const int64_t need = (rows + rows_per_block - 1) / rows_per_block;
  const int grid = static_cast<int>(need < 8 * static_cast<int64_t>(l.num_sms)
                                        ? need
                                        : 8 * static_cast<int64_t>(l.num_sms));
  const double lt = log2(static_cast<double>(theta));
  if (bf16)
    rope_kernel<__nv_bfloat16><<<grid, kRopeThreads, 0, l.stream>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<__nv_bfloat16*>(y), rows, D, period, pos0,
        lt);
  else
    rope_kernel<float><<<grid, kRopeThreads, 0, l.stream>>>(
        static_cast<const float*>(x), static_cast<float*>(y), rows, D, period, pos0, lt);
  return cudaGetLastError();
}

}  // namespace csa
