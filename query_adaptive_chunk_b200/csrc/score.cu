// Chunk scores: S[b,h,n,c] = (sum_g qt[b,n,h*G+g]) . summ[b,h,c]  (qt = q or P^T q).
//
// The group sum of the query heads is taken first (one dot product per chunk
// instead of G), then every warp streams summary rows with 128-bit loads:
// a row of Ds floats is spread over Ds/4 lanes, all eight rows of a warp are
// loaded before any arithmetic so that 8 x 512 B are in flight per warp, and
// the partial dot products are reduced with xor-shuffles inside the row's
// lanes.  One CTA covers 32 KB of summaries.
#include "internal.h"

namespace csa {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kScoreWarps = kScoreThreads / 32;
constexpr int kScoreIters = 8;  // rows per lane-group per warp

template <int DS>
__global__ void __launch_bounds__(kScoreThreads) score_kernel(
    const void* __restrict__ q, int q_bf16, const float* __restrict__ proj, int R,
    const float* __restrict__ summ, int Nq, int Hq, int Hkv, int D, int C,
    const uint8_t* __restrict__ head_full, int causal_tile_m, int causal_L,
    float* __restrict__ scores) {
  constexpr int LPR = DS / 4;          // lanes per summary row
  constexpr int RPI = 32 / LPR;        // rows per warp iteration
  constexpr int ROWS_WARP = RPI * kScoreIters;
  constexpr int ROWS_CTA = ROWS_WARP * kScoreWarps;
  __shared__ float qs[1024];
  __shared__ float qp[DS];

  const int u = blockIdx.z;  // b * Hkv + h
  const int n = blockIdx.y;
  const int h = u % Hkv, b = u / Hkv;
  if (head_full != nullptr && head_full[h]) return;
  const int G = Hq / Hkv;

  // group-summed query row (fp32)
  for (int d = threadIdx.x; d < D; d += kScoreThreads) {
    float acc = 0.f;
    for (int g = 0; g < G; ++g) {
      const int64_t off = ((static_cast<int64_t>(b) * Nq + n) * Hq + h * G + g) * D + d;
      acc += q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(q)[off])
                    : static_cast<const float*>(q)[off];
    }
    qs[d] = acc;
  }
  __syncthreads();
  const float* qv = qs;
  if (proj != nullptr) {
    // qp[r] = sum_d proj[d, r] qs[d]: thread t handles r = t / parts over the
    // d range of part t % parts (parts = 256 / R); the parts of one r sit in
    // adjacent lanes and are added by an xor-shuffle tree
    const int parts = kScoreThreads / R;
    const int r = threadIdx.x / parts, pt = threadIdx.x % parts;
    const int dchunk = (D + parts - 1) / parts;
    const int d0 = pt * dchunk, d1 = min(D, d0 + dchunk);
    float acc = 0.f;
#pragma unroll 4
    for (int d = d0; d < d1; ++d) acc += __ldg(proj + static_cast<int64_t>(d) * R + r) * qs[d];
    for (int o = parts >> 1; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (pt == 0) qp[r] = acc;
    __syncthreads();
    qv = qp;
  }

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane % LPR, rsub = lane / LPR;
  const float4 q4 = make_float4(qv[sub * 4], qv[sub * 4 + 1], qv[sub * 4 + 2], qv[sub * 4 + 3]);
  const int n_valid =
      causal_tile_m > 0 ? min(C, ((n + 1) * causal_tile_m - 1) / causal_L + 1) : C;
  const int row0 = blockIdx.x * ROWS_CTA + warp * ROWS_WARP + rsub;
  const float* sbase = summ + static_cast<int64_t>(u) * C * DS;
  float4 v[kScoreIters];
#pragma unroll
  for (int it = 0; it < kScoreIters; ++it) {
    const int c = row0 + it * RPI;
    if (c < n_valid)
      v[it] = __ldg(reinterpret_cast<const float4*>(sbase + static_cast<int64_t>(c) * DS) + sub);
    else
      v[it] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float* out = scores + (static_cast<int64_t>(u) * Nq + n) * C;
#pragma unroll
  for (int it = 0; it < kScoreIters; ++it) {
    float s = v[it].x * q4.x + v[it].y * q4.y + v[it].z * q4.z + v[it].w * q4.w;
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const int c = row0 + it * RPI;
    if (sub == 0 && c < C) out[c] = c < n_valid ? s : -INFINITY;
  }
}

// Many query rows per unit (prefill tile means): the scores of one unit are
// the product of its [Nq, DS] group-summed query rows with its [C, DS]
// summaries, so the CTA stages a 64-row block of each in shared memory
// (padded rows, no bank conflicts) and every thread accumulates a 4 x 4
// block of outputs in registers; each summary row is read once per 64 query
// rows instead of once per row.  Blocks above the causal diagonal are only
// filled with -inf.
constexpr int kTileRows = 64;
constexpr int kTileThreads = 256;

template <int DS>
__global__ void __launch_bounds__(kTileThreads) score_tiles_kernel(
    const void* __restrict__ q, int q_bf16, const float* __restrict__ summ, int Nq, int Hq,
    int Hkv, int C, const uint8_t* __restrict__ head_full, int causal_tile_m, int causal_L,
    float* __restrict__ scores) {
  constexpr int LD = DS + 1;
  extern __shared__ float sm_tile[];
  float* As = sm_tile;                   // [64][LD] query rows
  float* Bs = sm_tile + kTileRows * LD;  // [64][LD] summary rows
  const int u = blockIdx.z;
  const int h = u % Hkv, b = u / Hkv;
  if (head_full != nullptr && head_full[h]) return;
  const int G = Hq / Hkv;
  const int n0 = blockIdx.y * kTileRows, c0 = blockIdx.x * kTileRows;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;  // 16 x 16 threads, 4 x 4 outputs each
  float* out = scores + static_cast<int64_t>(u) * Nq * C;
  auto visible = [&](int n) {  // chunks [0, visible(n)) of query row n
    return causal_tile_m > 0 ? min(C, ((n + 1) * causal_tile_m - 1) / causal_L + 1) : C;
  };
  const int n_last = min(Nq, n0 + kTileRows) - 1;
  if (c0 >= visible(n_last)) {  // the whole block is masked
    for (int i = threadIdx.x; i < kTileRows * kTileRows; i += kTileThreads) {
      const int n = n0 + i / kTileRows, c = c0 + i % kTileRows;
      if (n < Nq && c < C) out[static_cast<int64_t>(n) * C + c] = -INFINITY;
    }
    return;
  }
  // stage the group-summed query rows and the summary rows, 4 floats per load
  constexpr int D4 = DS / 4;
  for (int i = threadIdx.x; i < kTileRows * D4; i += kTileThreads) {
    const int r = i / D4, d = (i % D4) * 4, n = n0 + r;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (n < Nq) {
      const int64_t row = (static_cast<int64_t>(b) * Nq + n) * Hq + h * G;
      for (int g = 0; g < G; ++g) {
        float4 x;
        if (q_bf16) {
          const __nv_bfloat162* qp = reinterpret_cast<const __nv_bfloat162*>(
              static_cast<const __nv_bfloat16*>(q) + (row + g) * DS + d);
          const float2 lo = __bfloat1622float2(qp[0]), hi = __bfloat1622float2(qp[1]);
          x = make_float4(lo.x, lo.y, hi.x, hi.y);
        } else {
          x = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(q) + (row + g) * DS + d));
        }
        acc.x += x.x;
        acc.y += x.y;
        acc.z += x.z;
        acc.w += x.w;
      }
    }
    float* ar = As + r * LD + d;
    ar[0] = acc.x;
    ar[1] = acc.y;
    ar[2] = acc.z;
    ar[3] = acc.w;
    const int c = c0 + r;
    const float4 sv = c < C ? __ldg(reinterpret_cast<const float4*>(
                                  summ + (static_cast<int64_t>(u) * C + c) * DS + d))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
    float* br = Bs + r * LD + d;
    br[0] = sv.x;
    br[1] = sv.y;
    br[2] = sv.z;
    br[3] = sv.w;
  }
  __syncthreads();
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 4
  for (int d = 0; d < DS; ++d) {
    float a[4], bb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = As[(ty * 4 + i) * LD + d];
#pragma unroll
    for (int j = 0; j < 4; ++j) bb[j] = Bs[(tx * 4 + j) * LD + d];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] += a[i] * bb[j];
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int n = n0 + ty * 4 + i;
    if (n >= Nq) continue;
    const int v = visible(n);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = c0 + tx * 4 + j;
      if (c < C) out[static_cast<int64_t>(n) * C + c] = c < v ? acc[i][j] : -INFINITY;
    }
  }
}

template <int DS>
cudaError_t launch_ds(const Launch& l, const void* q, bool bf16, const float* proj, int R,
                      const float* summ, int B, int Nq, int Hq, int Hkv, int D, int C,
                      const uint8_t* head_full, int ctm, int cL, float* scores) {
  constexpr int ROWS_CTA = (32 / (DS / 4)) * kScoreIters * kScoreWarps;
  dim3 grid((C + ROWS_CTA - 1) / ROWS_CTA, Nq, B * Hkv);
  score_kernel<DS><<<grid, kScoreThreads, 0, l.stream>>>(q, bf16 ? 1 : 0, proj, R, summ, Nq, Hq,
                                                        Hkv, D, C, head_full, ctm, cL, scores);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score(const Launch& l, const void* q, bool bf16, const float* proj, int R,
                         const float* summ, int B, int Nq, int Hq, int Hkv, int D, int C,
                         const uint8_t* head_full, int causal_tile_m, int causal_L,
                         float* scores) {
  if (B == 0 || Nq == 0 || C == 0) return cudaSuccess;
  if (proj == nullptr && Nq >= 16 && (D == 128 || D == 64)) {
    dim3 grid((C + kTileRows - 1) / kTileRows, (Nq + kTileRows - 1) / kTileRows, B * Hkv);
    const size_t sh = 2 * kTileRows * static_cast<size_t>(D + 1) * sizeof(float);
    if (D == 128) {
      cudaError_t e = cudaFuncSetAttribute(score_tiles_kernel<128>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sh);
      if (e != cudaSuccess) return e;
      score_tiles_kernel<128><<<grid, kTileThreads, sh, l.stream>>>(
          q, bf16 ? 1 : 0, summ, Nq, Hq, Hkv, C, head_full, causal_tile_m, causal_L, scores);
    } else {
      score_tiles_kernel<64><<<grid, kTileThreads, sh, l.stream>>>(
          q, bf16 ? 1 : 0, summ, Nq, Hq, Hkv, C, head_full, causal_tile_m, causal_L, scores);
    }
    return cudaGetLastError();
  }
  const int Ds = proj ? R : D;
  switch (Ds) {
    case 16: return launch_ds<16>(l, q, bf16, proj, R, summ, B, Nq, Hq, Hkv, D, C, head_full, causal_tile_m, causal_L, scores);
    case 32: return launch_ds<32>(l, q, bf16, proj, R, summ, B, Nq, Hq, Hkv, D, C, head_full, causal_tile_m, causal_L, scores);
    case 64: return launch_ds<64>(l, q, bf16, proj, R, summ, B, Nq, Hq, Hkv, D, C, head_full, causal_tile_m, causal_L, scores);
    case 128: return launch_ds<128>(l, q, bf16, proj, R, summ, B, Nq, Hq, Hkv, D, C, head_full, causal_tile_m, causal_L, scores);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace csa
