// Precompute kernels: chunk summaries (chunk-mean keys, optionally projected
// to a low rank), meta-summaries (mean of Gm chunk summaries) and tile-mean
// queries.  These run once per cache / per prefill, outside the per-step path;
// each is a reduction over rows with 16-byte loads, several rows in flight
// per thread.
#include "internal.h"

namespace csa {
namespace {

// Sums the E values of a 16-byte vector into acc (bf16: 8 values, fp32: 4).
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

// One CTA of kSummThreads per (chunk, unit).  A key row of D values is D / E
// 16-byte pieces (E = 8 bf16 or 4 fp32 values); thread t takes piece
// t % (D / E) of the rows rg, rg + RG, ... (rg = t / (D / E), RG row groups
// side by side), eight rows in flight, summing in fp32 in row order; the RG
// partial sums of each column then meet in shared memory and are added in
// row-group order.  With a projection R threads form the [R] outputs from
// the mean.
constexpr int kSummThreads = 128;

template <typename T, int D>
__global__ void __launch_bounds__(kSummThreads, 8) chunk_summaries_kernel(
    const T* __restrict__ K, int64_t T_len, int L, const float* __restrict__ proj, int R,
    float* __restrict__ summ) {
  constexpr int E = 16 / sizeof(T);
  constexpr int TPR = D / E;                 // threads per row
  constexpr int RG = kSummThreads / TPR;     // rows in parallel
  constexpr int UNROLL = 8;
  __shared__ float part[RG][D];
  __shared__ float mean_sh[D];
  const int c = blockIdx.x;
  const int u = blockIdx.y;
  const int C = static_cast<int>(T_len / L);
  const int piece = threadIdx.x % TPR, rg = threadIdx.x / TPR;
  const T* base =
      K + (static_cast<int64_t>(u) * T_len + static_cast<int64_t>(c) * L) * D + piece * E;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  int j = rg;
  for (; j + (UNROLL - 1) * RG < L; j += UNROLL * RG) {
    uint4 v[UNROLL];
#pragma unroll
    for (int k = 0; k < UNROLL; ++k)
      v[k] = __ldg(reinterpret_cast<const uint4*>(base + static_cast<int64_t>(j + k * RG) * D));
#pragma unroll
    for (int k = 0; k < UNROLL; ++k) add16(acc, v[k], static_cast<const T*>(nullptr));
  }
  for (; j < L; j += RG)
    add16(acc, __ldg(reinterpret_cast<const uint4*>(base + static_cast<int64_t>(j) * D)),
          static_cast<const T*>(nullptr));
#pragma unroll
  for (int e = 0; e < E; ++e) part[rg][piece * E + e] = acc[e];
  __syncthreads();
  const float invL = 1.0f / static_cast<float>(L);
  for (int d = threadIdx.x; d < D; d += kSummThreads) {
    float m = 0.f;
#pragma unroll
    for (int r = 0; r < RG; ++r) m += part[r][d];
    m *= invL;
    if (proj == nullptr)
      summ[(static_cast<int64_t>(u) * C + c) * D + d] = m;
    else
      mean_sh[d] = m;
  }
  if (proj == nullptr) return;
  __syncthreads();
  for (int r = threadIdx.x; r < R; r += kSummThreads) {
    float a = 0.f;
    for (int d = 0; d < D; ++d) a += __ldg(proj + static_cast<int64_t>(d) * R + r) * mean_sh[d];
    summ[(static_cast<int64_t>(u) * C + c) * R + r] = a;
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
  const auto* kb = static_cast<const __nv_bfloat16*>(K);
  const auto* kf = static_cast<const float*>(K);
  const int th = kSummThreads;
  if (D == 128 && bf16)
    chunk_summaries_kernel<__nv_bfloat16, 128><<<grid, th, 0, l.stream>>>(kb, T, L, proj, R, summ);
  else if (D == 128)
    chunk_summaries_kernel<float, 128><<<grid, th, 0, l.stream>>>(kf, T, L, proj, R, summ);
  else if (D == 64 && bf16)
    chunk_summaries_kernel<__nv_bfloat16, 64><<<grid, th, 0, l.stream>>>(kb, T, L, proj, R, summ);
  else if (D == 64)
    chunk_summaries_kernel<float, 64><<<grid, th, 0, l.stream>>>(kf, T, L, proj, R, summ);
  else {
    return cudaErrorInvalidValue;  // D is 64 or 128 (checked by the caller)
  }
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
