// Precompute kernels: chunk summaries (chunk-mean keys, optionally projected
// to a low rank), meta-summaries (mean of Gm chunk summaries) and tile-mean
// queries.  These run once per cache / per prefill, outside the per-step path;
// each is a coalesced reduction over rows.
#include "internal.h"

namespace csa {
namespace {

template <typename T>
__device__ __forceinline__ float ld_f(const T* p);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

// One CTA per (chunk, unit); thread d sums column d over the chunk's L rows,
// in row order, in fp32.  With a projection the mean goes through shared
// memory and R threads form the [R] outputs.
template <typename T>
__global__ void chunk_summaries_kernel(const T* __restrict__ K, int64_t T_len, int D, int L,
                                       const float* __restrict__ proj, int R,
                                       float* __restrict__ summ) {
  extern __shared__ float mean_sh[];
  const int c = blockIdx.x;
  const int u = blockIdx.y;
  const int C = static_cast<int>(T_len / L);
  const T* base = K + (static_cast<int64_t>(u) * T_len + static_cast<int64_t>(c) * L) * D;
  const float invL = 1.0f / static_cast<float>(L);
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < L; ++j) acc += ld_f<T>(base + static_cast<int64_t>(j) * D + d);
    float m = acc * invL;
    if (proj == nullptr)
      summ[(static_cast<int64_t>(u) * C + c) * D + d] = m;
    else
      mean_sh[d] = m;
  }
  if (proj == nullptr) return;
  __syncthreads();
  for (int r = threadIdx.x; r < R; r += blockDim.x) {
    float acc = 0.f;
    for (int d = 0; d < D; ++d) acc += __ldg(proj + static_cast<int64_t>(d) * R + r) * mean_sh[d];
    summ[(static_cast<int64_t>(u) * C + c) * R + r] = acc;
  }
}

__global__ void meta_summaries_kernel(const float* __restrict__ summ, int C, int Ds, int Gm,
                                      float* __restrict__ meta) {
  const int m = blockIdx.x, u = blockIdx.y;
  const int M = C / Gm;
  const float inv = 1.0f / static_cast<float>(Gm);
  for (int d = threadIdx.x; d < Ds; d += blockDim.x) {
    float acc = 0.f;
    const float* p = summ + (static_cast<int64_t>(u) * C + static_cast<int64_t>(m) * Gm) * Ds + d;
    for (int j = 0; j < Gm; ++j) acc += __ldg(p + static_cast<int64_t>(j) * Ds);
    meta[(static_cast<int64_t>(u) * M + m) * Ds + d] = acc * inv;
  }
}

// Tile means: a position's Hq*D query values are one contiguous row; each
// thread owns 16 bytes of it (8 bf16 or 4 fp32 values, so a warp reads 512
// contiguous bytes per row) and sums them over the tile's rows in row order,
// eight rows in flight.  Grid: (tiles, row segments of 128 threads, batch).
constexpr int kTileMeanThreads = 128;

__device__ __forceinline__ void add16(float* acc, const uint4& v, const __nv_bfloat16*) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(h[e]);
    acc[2 * e] += f.x;
    acc[2 * e + 1] += f.y;
  }
}
__device__ __forceinline__ void add16(float* acc, const uint4& v, const float*) {
  acc[0] += __uint_as_float(v.x);
  acc[1] += __uint_as_float(v.y);
  acc[2] += __uint_as_float(v.z);
  acc[3] += __uint_as_float(v.w);
}

template <typename T>
__global__ void __launch_bounds__(kTileMeanThreads) tile_mean_kernel(
    const T* __restrict__ Q, int S, int HD, int tile_m, float* __restrict__ qbar) {
  constexpr int E = 16 / sizeof(T);  // values per thread
  const int t = blockIdx.x, b = blockIdx.z;
  const int n_tiles = S / tile_m;
  const int col = (blockIdx.y * kTileMeanThreads + threadIdx.x) * E;
  if (col >= HD) return;
  const T* p = Q + (static_cast<int64_t>(b) * S + static_cast<int64_t>(t) * tile_m) * HD + col;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  int i = 0;
  for (; i + 8 <= tile_m; i += 8) {
    uint4 v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      v[k] = __ldg(reinterpret_cast<const uint4*>(p + static_cast<int64_t>(i + k) * HD));
#pragma unroll
    for (int k = 0; k < 8; ++k) add16(acc, v[k], static_cast<const T*>(nullptr));
  }
  for (; i < tile_m; ++i)
    add16(acc, __ldg(reinterpret_cast<const uint4*>(p + static_cast<int64_t>(i) * HD)),
          static_cast<const T*>(nullptr));
  const float inv = 1.0f / static_cast<float>(tile_m);
  float4* out = reinterpret_cast<float4*>(qbar + (static_cast<int64_t>(b) * n_tiles + t) * HD + col);
#pragma unroll
  for (int e = 0; e < E; e += 4)
    out[e / 4] = make_float4(acc[e] * inv, acc[e + 1] * inv, acc[e + 2] * inv, acc[e + 3] * inv);
}

}  // namespace

cudaError_t launch_chunk_summaries(const Launch& l, const void* K, bool bf16, int U, int64_t T,
                                   int D, int L, const float* proj, int R, float* summ) {
  const int C = static_cast<int>(T / L);
  if (C == 0 || U == 0) return cudaSuccess;
  dim3 grid(C, U);
  const int threads = D >= 128 ? 128 : 64;
  const size_t sh = proj ? D * sizeof(float) : 0;
  if (bf16)
    chunk_summaries_kernel<__nv_bfloat16><<<grid, threads, sh, l.stream>>>(
        static_cast<const __nv_bfloat16*>(K), T, D, L, proj, R, summ);
  else
    chunk_summaries_kernel<float><<<grid, threads, sh, l.stream>>>(static_cast<const float*>(K), T,
                                                                   D, L, proj, R, summ);
  return cudaGetLastError();
}

cudaError_t launch_meta_summaries(const Launch& l, const float* summ, int U, int C, int Ds, int Gm,
                                  float* meta) {
  const int M = C / Gm;
  if (M == 0 || U == 0) return cudaSuccess;
  dim3 grid(M, U);
  const int threads = Ds >= 128 ? 128 : ((Ds + 31) / 32) * 32;
  meta_summaries_kernel<<<grid, threads, 0, l.stream>>>(summ, C, Ds, Gm, meta);
  return cudaGetLastError();
}

cudaError_t launch_tile_mean(const Launch& l, const void* Q, bool bf16, int B, int S, int Hq, int D,
                             int tile_m, float* qbar) {
  const int n = S / tile_m;
  if (n == 0 || B == 0 || Hq == 0) return cudaSuccess;
  const int HD = Hq * D;  // a multiple of 8 (D is 64 or 128)
  const int E = bf16 ? 8 : 4;
  dim3 grid(n, (HD / E + kTileMeanThreads - 1) / kTileMeanThreads, B);
  if (bf16)
    tile_mean_kernel<__nv_bfloat16><<<grid, kTileMeanThreads, 0, l.stream>>>(
        static_cast<const __nv_bfloat16*>(Q), S, HD, tile_m, qbar);
  else
    tile_mean_kernel<float><<<grid, kTileMeanThreads, 0, l.stream>>>(static_cast<const float*>(Q),
                                                                    S, HD, tile_m, qbar);
  return cudaGetLastError();
}

}  // namespace csa
