// Token Sparse Attention for prefill (gist.science/ko/paper/2602.03216,
// section 2): which tokens each KV head keeps, and the gather / scatter
// around the dense causal attention of the kept tokens.
//
//   importance   a proxy attention map of the last n_obs query rows of every
//                query head against all keys of its KV head; the importance
//                of key j is the sum over those rows of its softmax weight
//                (the rows of the GQA group's heads summed: one importance
//                per KV head).  Two passes over K on the tensor cores
//                (mma.m16n8k16): per-row max and sum over key blocks (rows
//                as M, keys as N), then, with the rows' final max and sum,
//                the weights summed per key (keys as M, rows as N).  K is
//                read twice from HBM.
//   budget       Dynamic Token Coverage: the fewest tokens whose importance
//                (summed over the KV heads, normalised) reaches 1 - tau, i.e.
//                the least important ones are dropped while their mass stays
//                within tau.  One CTA per sequence: an MSB-first radix select
//                over the masses' bits that carries each bucket's mass, so
//                the cut is found without sorting.  The budget is rounded up
//                to whole 64-row tiles for the dense attention.
//   gather       per KV head, its kept tokens' K and V rows and the group's
//                query rows, in position order, into dense compressed
//                tensors (rows past a sequence's budget are zero).
//   scatter      the compressed output back to the kept positions; every
//                other row of the output is 0 (the residual path carries the
//                skipped tokens in the model).
#include "internal.h"

namespace csa {
namespace {

constexpr int kImpThreads = 128;    // pass 2: 4 warps, 32 keys each
constexpr int kStatsThreads = 256;  // pass 1: 8 warps, 32 observed rows each per turn
constexpr int kImpKeys = 128;       // keys per CTA
constexpr float kLog2eF = 1.4426950408889634f;

// Row r of the observed block of KV head h: query head h*G + r / n_obs at
// position S - n_obs + r % n_obs.
__device__ __forceinline__ int obs_pos(int r, int n_obs, int S) { return S - n_obs + r % n_obs; }

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, bool valid) {
  // 16-byte asynchronous copy; src-size 0 fills the destination with zeros
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)),
               "l"(gsrc), "r"(valid ? 16 : 0)
               : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Asynchronous 16-byte copies of the observed query rows of (b, h) [R][D]
// into padded shared memory (row stride D + 8 bf16: conflict-free fragment
// loads); the caller commits and waits.
template <int D>
__device__ __forceinline__ void imp_load_q(const __nv_bfloat16* Q, int b, int h, int S, int Hq,
                                           int G, int n_obs, __nv_bfloat16* qs) {
  constexpr int LD = D + 8, V8 = D / 8;
  const int R = G * n_obs;
  for (int e = threadIdx.x; e < R * V8; e += blockDim.x) {
    const int r = e / V8, c = (e % V8) * 8;
    const int g = r / n_obs, pos = obs_pos(r, n_obs, S);
    cp_async16(qs + r * LD + c, Q + ((static_cast<int64_t>(b) * S + pos) * Hq + h * G + g) * D + c,
               true);
  }
}

// The same for the key block [kImpKeys][D] starting at key j0 (keys past S
// are zero-filled).
template <int D>
__device__ __forceinline__ void imp_load_k(const __nv_bfloat16* K, int b, int h, int S, int Hkv,
                                           int j0, __nv_bfloat16* ks) {
  constexpr int LD = D + 8, V8 = D / 8;
  const __nv_bfloat16* kb = K + ((static_cast<int64_t>(b) * Hkv + h) * S) * D;
  for (int e = threadIdx.x; e < kImpKeys * V8; e += blockDim.x) {
    const int r = e / V8, c = (e % V8) * 8;
    const int j = j0 + r;
    cp_async16(ks + r * LD + c, kb + static_cast<int64_t>(j < S ? j : 0) * D + c, j < S);
  }
}

// Both, all in flight at once, then waits for them (the caller's barrier
// then publishes them).
template <int D>
__device__ void imp_load(const __nv_bfloat16* Q, const __nv_bfloat16* K, int b, int h, int S,
                         int Hq, int Hkv, int G, int n_obs, int j0, __nv_bfloat16* qs,
                         __nv_bfloat16* ks) {
  imp_load_q<D>(Q, b, h, S, Hq, G, n_obs, qs);
  imp_load_k<D>(K, b, h, S, Hkv, j0, ks);
  cp_async_commit();
  cp_async_wait<0>();
}

// This warp's 32 keys (two 16-key m-tiles) as mma A fragments for every
// 16-wide slice of D, loaded once and reused for every block of query rows.
template <int D>
__device__ __forceinline__ void imp_load_a(const __nv_bfloat16* ks, int kw,
                                           uint32_t (&af)[D / 16][2][4]) {
  constexpr int LD = D + 8;
  const int lane = threadIdx.x & 31, rr = lane >> 2, cc = 2 * (lane & 3);
#pragma unroll
  for (int ks16 = 0; ks16 < D / 16; ++ks16)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      const __nv_bfloat16* kr = ks + (kw + mt * 16 + rr) * LD + ks16 * 16 + cc;
      af[ks16][mt][0] = *reinterpret_cast<const uint32_t*>(kr);
      af[ks16][mt][1] = *reinterpret_cast<const uint32_t*>(kr + 8 * LD);
      af[ks16][mt][2] = *reinterpret_cast<const uint32_t*>(kr + 8);
      af[ks16][mt][3] = *reinterpret_cast<const uint32_t*>(kr + 8 * LD + 8);
    }
}

// S^T tile of this warp's 32 keys against query rows [n0 .. n0 + 8):
// acc[mt][0..3] as the mma C layout (key = lane/4 (+8), row = n0 + 2 (lane%4)
// (+1)), unscaled.
template <int D>
__device__ __forceinline__ void imp_tile(const __nv_bfloat16* qs, const uint32_t (&af)[D / 16][2][4],
                                         int n0, float (&acc)[2][4]) {
  constexpr int LD = D + 8;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[mt][e] = 0.f;
  // B fragments of two 16-wide slices per ldmatrix: lanes 0-7 / 8-15 /
  // 16-23 / 24-31 address rows n0 .. n0 + 7 at columns +0 / +8 / +16 / +24
  const uint32_t qb_base =
      smem_u32(qs + (n0 + (lane & 7)) * LD + (lane >> 4) * 16 + ((lane >> 3) & 1) * 8);
#pragma unroll
  for (int kp = 0; kp < D / 32; ++kp) {
    uint32_t b[4];
    ldsm_x4(qb_base + kp * 32 * 2, b[0], b[1], b[2], b[3]);
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
        mma_bf16_16816(acc[mt], af[2 * kp + t][mt][0], af[2 * kp + t][mt][1],
                       af[2 * kp + t][mt][2], af[2 * kp + t][mt][3], b[2 * t], b[2 * t + 1]);
  }
}

// One warp's 32 observed rows r0 .. r0 + 31 against the key block at j0 in
// `ks`: the rows are the mma M dimension and the keys N (the layout of a
// flash-attention forward pass); the warp runs over the block's keys 64 at a
// time and every lane folds its scores into the running (max, sum) of its
// four rows over its own key columns, m/l [m-tile][row +0 / +8].  Only
// blocks that reach past the first observed position need the causal mask.
template <int D>
__device__ __forceinline__ void imp_stats_rows(const __nv_bfloat16* qs, const __nv_bfloat16* ks,
                                               int r0, int R, int S, int n_obs, int j0,
                                               bool masked, float sl2, float (&m)[2][2],
                                               float (&l)[2][2]) {
  constexpr int LD = D + 8;
  const int lane = threadIdx.x & 31, rr = lane >> 2, cc = 2 * (lane & 3);
  // A fragments by ldmatrix: lanes 0-7 / 8-15 / 16-23 / 24-31 address the
  // rows of the (rows +0, cols +0) / (+8, +0) / (+0, +8) / (+8, +8) 8x8 blocks
  uint32_t qa[D / 16][2][4];
  const uint32_t qa_base =
      smem_u32(qs + (r0 + (lane & 7) + ((lane >> 3) & 1) * 8) * LD + (lane >> 4) * 8);
#pragma unroll
  for (int k16 = 0; k16 < D / 16; ++k16)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
      ldsm_x4(qa_base + (mt * 16 * LD + k16 * 16) * 2, qa[k16][mt][0], qa[k16][mt][1],
              qa[k16][mt][2], qa[k16][mt][3]);
  // key j is visible to row r iff j <= S - n_obs + r % n_obs (which also
  // keeps j < S); rows past R (zero padding) see nothing
  int lim[2][2];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int r = r0 + mt * 16 + rr + 8 * hh;
      lim[mt][hh] = r < R ? S - n_obs + r % n_obs : -1;
    }
#pragma unroll 1
  for (int half = 0; half < kImpKeys / 64; ++half) {
    float acc[8][2][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][mt][e] = 0.f;
    // B fragments of two n-tiles per ldmatrix: lanes 0-7 / 8-15 / 16-23 /
    // 24-31 address the keys of (n-tile +0, cols +0) / (+0, +8) / (+1, +0) /
    // (+1, +8)
    const uint32_t kb_base = smem_u32(ks + (half * 64 + (lane >> 4) * 8 + (lane & 7)) * LD +
                                      ((lane >> 3) & 1) * 8);
#pragma unroll
    for (int k16 = 0; k16 < D / 16; ++k16)
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b[4];
        ldsm_x4(kb_base + (np * 16 * LD + k16 * 16) * 2, b[0], b[1], b[2], b[3]);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
            mma_bf16_16816(acc[2 * np + t][mt], qa[k16][mt][0], qa[k16][mt][1], qa[k16][mt][2],
                           qa[k16][mt][3], b[2 * t], b[2 * t + 1]);
      }
    // C layout: acc[nt][mt][e] = row r0 + mt*16 + rr + 8 (e >> 1), key
    // j0 + half*64 + nt*8 + cc + (e & 1); to the log2 domain, masked
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float v = acc[nt][mt][e] * sl2;
          if (masked && j0 + half * 64 + nt * 8 + cc + (e & 1) > lim[mt][e >> 1]) v = -INFINITY;
          acc[nt][mt][e] = v;
        }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float mx = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
          mx = fmaxf(mx, fmaxf(acc[nt][mt][2 * hh], acc[nt][mt][2 * hh + 1]));
        const float mn = fmaxf(m[mt][hh], mx);
        if (mn != -INFINITY) {
          float sum = 0.f;
#pragma unroll
          for (int nt = 0; nt < 8; ++nt)
            sum += fast_exp2(acc[nt][mt][2 * hh] - mn) + fast_exp2(acc[nt][mt][2 * hh + 1] - mn);
          l[mt][hh] = l[mt][hh] * fast_exp2(m[mt][hh] - mn) + sum;
          m[mt][hh] = mn;
        }
      }
  }
}

// Pass 1: per (b, h) and observed row, the max and the sum of 2^(s - max)
// over the visible keys of the key blocks this CTA takes -> part [b, h,
// split, R, 2].  Persistent over the key blocks: CTA (split, h, b) takes
// blocks split, split + nsplit, ...; the observed rows are loaded once and
// the key tiles double-buffered, so the next tile's copy runs under this
// tile's math.  Warp w takes the 32-row groups w, w + 8 (R <= 512) and keeps
// their per-lane running statistics across all the CTA's blocks; the four
// lanes of a row merge once at the end.
template <int D>
__global__ void __launch_bounds__(kStatsThreads) imp_stats_kernel(
    const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K, int S, int Hq,
    int Hkv, int G, int n_obs, float sl2, int nblk, float* __restrict__ part) {
  extern __shared__ __align__(16) uint8_t sm[];
  constexpr int LD = D + 8, V8 = D / 8;
  constexpr int kRowsPerTurn = (kStatsThreads / 32) * 32;
  const int R = G * n_obs, Rp = (R + 31) & ~31;
  __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(sm);  // [Rp][LD]
  __nv_bfloat16* ksb = qs + Rp * LD;                         // [2][kImpKeys][LD]
  const int nsplit = gridDim.x, split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  // rows R .. Rp - 1 of the last row group are zero (their results are dropped)
  for (int e = threadIdx.x; e < (Rp - R) * V8; e += blockDim.x)
    *reinterpret_cast<uint4*>(qs + (R + e / V8) * LD + (e % V8) * 8) = make_uint4(0u, 0u, 0u, 0u);
  imp_load_q<D>(Q, b, h, S, Hq, G, n_obs, qs);
  if (split < nblk) imp_load_k<D>(K, b, h, S, Hkv, split * kImpKeys, ksb);
  cp_async_commit();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float m[2][2][2], l[2][2][2];  // [row group of this warp][m-tile][row +0 / +8]
#pragma unroll
  for (int g2 = 0; g2 < 2; ++g2)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        m[g2][mt][hh] = -INFINITY;
        l[g2][mt][hh] = 0.f;
      }
  int it = 0;
  for (int blk = split; blk < nblk; blk += nsplit, ++it) {
    const int nxt = blk + nsplit;
    if (nxt < nblk) imp_load_k<D>(K, b, h, S, Hkv, nxt * kImpKeys, ksb + ((it + 1) & 1) * kImpKeys * LD);
    cp_async_commit();
    cp_async_wait<1>();  // all but the tile just issued
    __syncthreads();
    const __nv_bfloat16* ks = ksb + (it & 1) * kImpKeys * LD;
    const int j0 = blk * kImpKeys;
    const bool masked = j0 + kImpKeys - 1 > S - n_obs;
#pragma unroll
    for (int g2 = 0; g2 < 2; ++g2) {
      const int r0 = warp * 32 + g2 * kRowsPerTurn;
      if (r0 < R) imp_stats_rows<D>(qs, ks, r0, R, S, n_obs, j0, masked, sl2, m[g2], l[g2]);
    }
    __syncthreads();  // this buffer takes the copy issued next turn
  }
  cp_async_wait<0>();
  const int rr = lane >> 2;
  float* out = part + ((static_cast<int64_t>(b) * Hkv + h) * nsplit + split) * R * 2;
#pragma unroll
  for (int g2 = 0; g2 < 2; ++g2) {
    const int r0 = warp * 32 + g2 * kRowsPerTurn;
    if (r0 >= R) continue;  // warp-uniform
    // merge the four lanes of each row (lanes 4 rr .. 4 rr + 3)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int x = 1; x <= 2; x <<= 1) {
          const float mo = __shfl_xor_sync(0xffffffffu, m[g2][mt][hh], x);
          const float lo = __shfl_xor_sync(0xffffffffu, l[g2][mt][hh], x);
          const float mn = fmaxf(m[g2][mt][hh], mo);
          if (mn != -INFINITY) {
            l[g2][mt][hh] = l[g2][mt][hh] * fast_exp2(m[g2][mt][hh] - mn) + lo * fast_exp2(mo - mn);
            m[g2][mt][hh] = mn;
          }
        }
    if ((lane & 3) == 0) {
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int r = r0 + mt * 16 + rr + 8 * hh;
          if (r < R) {
            out[r * 2] = m[g2][mt][hh];
            out[r * 2 + 1] = l[g2][mt][hh];
          }
        }
    }
  }
}

// The rows' max and sum over all key blocks: part -> stats [b, h, R, 2].
// CTA (b*Hkv + h, y) takes rows 32 y .. 32 y + 31; its 8 warps split the key
// blocks (warp w: blocks w, w + 8, ...), lane = row, so the partials of a
// turn are one coalesced 256-byte load per warp; the warps' results merge in
// shared memory.
constexpr int kCombineWarps = 8;
__global__ void __launch_bounds__(kCombineWarps * 32) imp_combine_kernel(
    const float* __restrict__ part, int nblk, int R, float* __restrict__ stats) {
  __shared__ float2 red[kCombineWarps][32];
  const int64_t bh = blockIdx.x;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int r = blockIdx.y * 32 + lane;
  float m = -INFINITY, l = 0.f;
  if (r < R) {
    const float2* p2 = reinterpret_cast<const float2*>(part) + bh * nblk * R + r;
#pragma unroll 4
    for (int k = w; k < nblk; k += kCombineWarps) {
      const float2 v = p2[static_cast<int64_t>(k) * R];
      if (v.x == -INFINITY) continue;
      const float mn = fmaxf(m, v.x);
      l = l * exp2f(m - mn) + v.y * exp2f(v.x - mn);
      m = mn;
    }
  }
  red[w][lane] = make_float2(m, l);
  __syncthreads();
  if (w == 0 && r < R) {
    m = -INFINITY;
    l = 0.f;
    for (int x = 0; x < kCombineWarps; ++x) {
      const float2 v = red[x][lane];
      if (v.x == -INFINITY) continue;
      const float mn = fmaxf(m, v.x);
      l = l * exp2f(m - mn) + v.y * exp2f(v.x - mn);
      m = mn;
    }
    stats[(bh * R + r) * 2] = m;
    stats[(bh * R + r) * 2 + 1] = l;
  }
}

// Pass 2: importance of each key = sum over the observed rows of
// 2^(s - max_r) / sum_r -> imp [b, h, S].
template <int D>
__global__ void __launch_bounds__(kImpThreads) imp_weight_kernel(
    const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K, int S, int Hq,
    int Hkv, int G, int n_obs, float sl2, const float* __restrict__ stats, float* __restrict__ imp) {
  extern __shared__ __align__(16) uint8_t sm[];
  constexpr int LD = D + 8;
  const int R = G * n_obs;
  __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(sm);
  __nv_bfloat16* ks = qs + R * LD;
  float* st = reinterpret_cast<float*>(ks + kImpKeys * LD);  // [R][2]: max, 1/sum
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int j0 = blk * kImpKeys;
  const int64_t bh = static_cast<int64_t>(b) * Hkv + h;
  imp_load<D>(Q, K, b, h, S, Hq, Hkv, G, n_obs, j0, qs, ks);
  for (int r = threadIdx.x; r < R; r += blockDim.x) {
    st[r * 2] = stats[(bh * R + r) * 2];
    const float l = stats[(bh * R + r) * 2 + 1];
    st[r * 2 + 1] = l > 0.f ? 1.0f / l : 0.f;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kw = warp * 32, rr = lane >> 2, cc = 2 * (lane & 3);
  float wsum[4] = {0.f, 0.f, 0.f, 0.f};  // keys kw + rr + 8 t
  uint32_t af[D / 16][2][4];
  imp_load_a<D>(ks, kw, af);
  // as in pass 1: only blocks reaching past the first observed position mask
  const bool masked = j0 + kImpKeys - 1 > S - n_obs;
  const float2* st2 = reinterpret_cast<const float2*>(st);
  for (int n0 = 0; n0 < R; n0 += 8) {
    float acc[2][4];
    imp_tile<D>(qs, af, n0, acc);
    // (max, 1/sum) of this lane's two rows
    const float2 s0 = st2[n0 + cc], s1 = st2[n0 + cc + 1];
    const float nm[2] = {-s0.x, -s1.x}, il[2] = {s0.y, s1.y};
    if (!masked) {
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          wsum[mt * 2 + (e >> 1)] += fast_exp2(fmaf(acc[mt][e], sl2, nm[e & 1])) * il[e & 1];
    } else {
      const int lim[2] = {obs_pos(n0 + cc, n_obs, S), obs_pos(n0 + cc + 1, n_obs, S)};
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = mt * 2 + (e >> 1);
          if (j0 + kw + rr + t * 8 <= lim[e & 1])
            wsum[t] += fast_exp2(fmaf(acc[mt][e], sl2, nm[e & 1])) * il[e & 1];
        }
    }
  }
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    wsum[t] += __shfl_xor_sync(0xffffffffu, wsum[t], 1);
    wsum[t] += __shfl_xor_sync(0xffffffffu, wsum[t], 2);
  }
  if ((lane & 3) == 0) {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int j = j0 + kw + rr + t * 8;
      if (j < S) imp[bh * S + j] = wsum[t];
    }
  }
}

// ---------------------------------------------------------------- budget

constexpr int kBudgetThreads = 1024;

// One CTA per sequence b: the masses m_j = sum_h imp[b,h,j] (kept in shared
// memory), then the smallest k whose k largest masses reach (1 - tau) of the
// total.  Non-negative floats order like their bit patterns, so an MSB-first
// radix select over the bits, carrying each bucket's count and mass, finds
// the cut value; equal masses at the cut are taken as few as needed.
// k_seq[b] = k; k_unit[b*Hkv + h] = k rounded up to whole `tile`s (<= S).
__global__ void __launch_bounds__(kBudgetThreads) budget_kernel(const float* __restrict__ imp,
                                                                int S, int Hkv, float tau, int tile,
                                                                int32_t* __restrict__ k_seq,
                                                                int32_t* __restrict__ k_unit) {
  extern __shared__ __align__(16) uint8_t sm[];
  float* ms = reinterpret_cast<float*>(sm);  // [S]
  __shared__ unsigned int hc[256];
  __shared__ float hm[256];
  __shared__ float wsum[32];
  __shared__ unsigned int sel_sh, prefix_sh;
  __shared__ float above_m_sh;
  __shared__ unsigned int above_c_sh;
  const int b = blockIdx.x, tid = threadIdx.x;
  const float* ib = imp + static_cast<int64_t>(b) * Hkv * S;
  float part = 0.f;
  // One SM reads all B*Hkv*S importances of the sequence: keep many bytes in
  // flight per thread.  16-byte loads of four tokens, all heads at once,
  // when the rows allow it; else four tokens per thread per turn.
  const bool vec = S % 4 == 0 && (reinterpret_cast<uintptr_t>(ib) & 15u) == 0;
  for (int j4 = tid; vec && j4 < S / 4; j4 += blockDim.x) {
    float4 m4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int h = 0; h < Hkv; ++h) {
      const float4 v = reinterpret_cast<const float4*>(ib + static_cast<int64_t>(h) * S)[j4];
      m4.x += v.x;
      m4.y += v.y;
      m4.z += v.z;
      m4.w += v.w;
    }
    m4 = make_float4(fmaxf(m4.x, 0.f), fmaxf(m4.y, 0.f), fmaxf(m4.z, 0.f), fmaxf(m4.w, 0.f));
    reinterpret_cast<float4*>(ms)[j4] = m4;
    part += (m4.x + m4.y) + (m4.z + m4.w);
  }
  for (int jb = tid; !vec && jb < S; jb += 4 * blockDim.x) {
    float m[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
    for (int h = 0; h < Hkv; ++h) {
      const float* row = ib + static_cast<int64_t>(h) * S;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = jb + u * blockDim.x;
        if (j < S) m[u] += row[j];
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = jb + u * blockDim.x;
      if (j < S) {
        const float v = fmaxf(m[u], 0.f);
        ms[j] = v;
        part += v;
      }
    }
  }
#pragma unroll
  for (int x = 16; x > 0; x >>= 1) part += __shfl_xor_sync(0xffffffffu, part, x);
  if ((tid & 31) == 0) wsum[tid >> 5] = part;
  if (tid == 0) {
    prefix_sh = 0u;
    above_m_sh = 0.f;
    above_c_sh = 0u;
  }
  __syncthreads();
  float total = 0.f;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) total += wsum[w];
  const float target = (1.0f - tau) * total;
  unsigned int mask = 0u;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int d = tid; d < 256; d += blockDim.x) {
      hc[d] = 0u;
      hm[d] = 0.f;
    }
    __syncthreads();
    const unsigned int prefix = prefix_sh;
    // Most masses share a few buckets: up to three times, the lanes of a
    // warp in the bucket of its first remaining lane add their count and
    // mass by a warp reduction and one atomic each; lanes left after that
    // (buckets spread wide) add theirs one by one.
    const int lane = tid & 31;
    for (int j0 = 0; j0 < S; j0 += blockDim.x) {
      const int j = j0 + tid;
      int d = -1;
      float m = 0.f;
      if (j < S) {
        const unsigned int key = __float_as_uint(ms[j]);
        if ((key & mask) == prefix) {
          d = (key >> shift) & 255u;
          m = ms[j];
        }
      }
#pragma unroll
      for (int round = 0; round < 3; ++round) {
        const unsigned int act = __ballot_sync(0xffffffffu, d >= 0);
        if (act == 0u) break;  // warp-uniform
        const int d0 = __shfl_sync(0xffffffffu, d, __ffs(act) - 1);
        const unsigned int same = __ballot_sync(0xffffffffu, d == d0);
        float v = d == d0 ? m : 0.f;
#pragma unroll
        for (int x = 16; x > 0; x >>= 1) v += __shfl_xor_sync(0xffffffffu, v, x);
        if (lane == 0) {
          atomicAdd(&hc[d0], static_cast<unsigned int>(__popc(same)));
          atomicAdd(&hm[d0], v);
        }
        if (d == d0) d = -1;  // counted
      }
      if (d >= 0) {
        atomicAdd(&hc[d], 1u);
        atomicAdd(&hm[d], m);
      }
    }
    __syncthreads();
    // The bucket where the running mass from the top first reaches the
    // target, by warp 0: lane L holds buckets 255 - 8L .. 248 - 8L, a scan
    // over the lanes gives the mass and count above each lane's buckets.
    if (tid < 32) {
      float pm[8];
      unsigned int pc[8];
      float lm = 0.f;
      unsigned int lc = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        pm[i] = hm[255 - 8 * lane - i];
        pc[i] = hc[255 - 8 * lane - i];
        lm += pm[i];
        lc += pc[i];
      }
      float sm_ = lm;
      unsigned int sc = lc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float t = __shfl_up_sync(0xffffffffu, sm_, o);
        const unsigned int tc = __shfl_up_sync(0xffffffffu, sc, o);
        if (lane >= o) {
          sm_ += t;
          sc += tc;
        }
      }
      float em = __shfl_up_sync(0xffffffffu, sm_, 1);
      unsigned int ec = __shfl_up_sync(0xffffffffu, sc, 1);
      if (lane == 0) {
        em = 0.f;
        ec = 0u;
      }
      float am = above_m_sh + em;
      unsigned int ac = above_c_sh + ec;
      int sel = -1, low = -1;
      float am_sel = 0.f, am_low = 0.f;
      unsigned int ac_sel = 0u, ac_low = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (sel < 0 && pc[i] != 0u) {
          if (am + pm[i] >= target) {
            sel = 255 - 8 * lane - i;
            am_sel = am;
            ac_sel = ac;
          } else {
            am_low = am;  // the mass above this bucket, were it the cut
            ac_low = ac;
            am += pm[i];
            ac += pc[i];
            low = 255 - 8 * lane - i;
          }
        }
      }
      const unsigned int hit = __ballot_sync(0xffffffffu, sel >= 0);
      int src;
      if (hit != 0u) {
        src = __ffs(hit) - 1;  // the first crossing from the top
      } else {  // the sums fell short of the target by rounding: cut in the lowest bucket
        const unsigned int nz = __ballot_sync(0xffffffffu, low >= 0);
        src = nz != 0u ? 31 - __clz(nz) : 0;
        sel = low < 0 ? 0 : low;
        am_sel = low < 0 ? am : am_low;
        ac_sel = low < 0 ? ac : ac_low;
      }
      sel = __shfl_sync(0xffffffffu, sel, src);
      am_sel = __shfl_sync(0xffffffffu, am_sel, src);
      ac_sel = __shfl_sync(0xffffffffu, ac_sel, src);
      if (lane == 0) {
        above_m_sh = am_sel;
        above_c_sh = ac_sel;
        sel_sh = static_cast<unsigned int>(sel);
        prefix_sh = prefix | (static_cast<unsigned int>(sel) << shift);
      }
    }
    __syncthreads();
    mask |= 255u << shift;
    if (shift == 0) break;
  }
  if (tid == 0) {
    int k;
    if (!(target > 0.f)) {
      k = 0;
    } else {
      const float v = __uint_as_float(prefix_sh);
      const unsigned int n_eq = hc[sel_sh];
      const float need = target - above_m_sh;
      unsigned int take = n_eq;
      if (v > 0.f && need > 0.f) {
        const float t = ceilf(need / v);
        take = t < static_cast<float>(n_eq) ? static_cast<unsigned int>(fmaxf(t, 1.f)) : n_eq;
      } else if (!(need > 0.f)) {
        take = 0u;
      }
      k = static_cast<int>(above_c_sh + take);
    }
    k = min(k, S);
    k_seq[b] = k;
    const int kt = min(S, (k + tile - 1) / tile * tile);
    for (int h = 0; h < Hkv; ++h) k_unit[static_cast<int64_t>(b) * Hkv + h] = kt;
  }
}

// ---------------------------------------------------------------- budget, one cluster per sequence
//
// The same cut as budget_kernel, over a cluster of kBudgetCS CTAs: CTA r
// holds the masses of tokens [r S / CS, (r + 1) S / CS) in shared memory and
// builds its own 256-bucket histogram (count and mass) per radix pass; the
// CTAs then read every CTA's histogram through distributed shared memory and
// add them in rank order, so each finds the same cut bucket, and the next
// pass narrows the prefix.  The first CTA writes the budgets.

constexpr int kBudgetCS = 8;
constexpr int kBudgetCThreads = 512;

__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

__global__ void __launch_bounds__(kBudgetCThreads) budget_cluster_kernel(
    const float* __restrict__ imp, int S, int Hkv, float tau, int tile, int32_t* __restrict__ k_seq,
    int32_t* __restrict__ k_unit) {
  cluster_arrive_relaxed();
  extern __shared__ __align__(16) uint8_t sm[];
  float* ms = reinterpret_cast<float*>(sm);  // [S / CS] this CTA's masses
  __shared__ unsigned int hc[256];           // this CTA's histogram of the pass
  __shared__ float hm[256];
  __shared__ unsigned int gc[256];           // the cluster's
  __shared__ float gm[256];
  __shared__ float wsum[32], tot_parts[kBudgetCS];
  __shared__ unsigned int prefix_sh, sel_sh;
  __shared__ float above_m_sh;
  __shared__ unsigned int above_c_sh;
  const int CS = static_cast<int>(cluster_size());
  const int rank = static_cast<int>(cluster_rank());
  const int b = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
  const int lo = static_cast<int>(static_cast<int64_t>(S) * rank / CS);
  const int n = static_cast<int>(static_cast<int64_t>(S) * (rank + 1) / CS) - lo;
  const float* ib = imp + static_cast<int64_t>(b) * Hkv * S + lo;
  float part = 0.f;
  for (int j = tid; j < n; j += blockDim.x) {
    float m = 0.f;
#pragma unroll 8
    for (int h = 0; h < Hkv; ++h) m += ib[static_cast<int64_t>(h) * S + j];
    m = fmaxf(m, 0.f);
    ms[j] = m;
    part += m;
  }
#pragma unroll
  for (int x = 16; x > 0; x >>= 1) part += __shfl_xor_sync(0xffffffffu, part, x);
  if (lane == 0) wsum[tid >> 5] = part;
  if (tid == 0) {
    prefix_sh = 0u;
    above_m_sh = 0.f;
    above_c_sh = 0u;
  }
  __syncthreads();
  cluster_wait();  // (phase 1) every CTA is running: its part of the total to all
  if (tid == 0) {
    float t = 0.f;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += wsum[w];
    for (int r = 0; r < CS; ++r) st_cluster_f32(cluster_map(smem_u32(tot_parts + rank), r), t);
  }
  cluster_arrive();
  cluster_wait();
  float total = 0.f;
  for (int r = 0; r < CS; ++r) total += tot_parts[r];  // rank order: the same sum in every CTA
  const float target = (1.0f - tau) * total;
  unsigned int mask = 0u;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int d = tid; d < 256; d += blockDim.x) {
      hc[d] = 0u;
      hm[d] = 0.f;
    }
    __syncthreads();
    const unsigned int prefix = prefix_sh;
    for (int j0 = 0; j0 < n; j0 += blockDim.x) {
      const int j = j0 + tid;
      int d = -1;
      float m = 0.f;
      if (j < n) {
        const unsigned int key = __float_as_uint(ms[j]);
        if ((key & mask) == prefix) {
          d = (key >> shift) & 255u;
          m = ms[j];
        }
      }
#pragma unroll
      for (int round = 0; round < 3; ++round) {
        const unsigned int act = __ballot_sync(0xffffffffu, d >= 0);
        if (act == 0u) break;  // warp-uniform
        const int d0 = __shfl_sync(0xffffffffu, d, __ffs(act) - 1);
        const unsigned int same = __ballot_sync(0xffffffffu, d == d0);
        float v = d == d0 ? m : 0.f;
#pragma unroll
        for (int x = 16; x > 0; x >>= 1) v += __shfl_xor_sync(0xffffffffu, v, x);
        if (lane == 0) {
          atomicAdd(&hc[d0], static_cast<unsigned int>(__popc(same)));
          atomicAdd(&hm[d0], v);
        }
        if (d == d0) d = -1;  // counted
      }
      if (d >= 0) {
        atomicAdd(&hc[d], 1u);
        atomicAdd(&hm[d], m);
      }
    }
    cluster_arrive();  // every CTA's histogram of this pass is complete
    cluster_wait();
    for (int d = tid; d < 256; d += blockDim.x) {  // the cluster's, added in rank order
      unsigned int c = 0u;
      float mm = 0.f;
      for (int r = 0; r < CS; ++r) {
        c += ld_cluster_u32(cluster_map(smem_u32(hc + d), r));
        mm += ld_cluster_f32(cluster_map(smem_u32(hm + d), r));
      }
      gc[d] = c;
      gm[d] = mm;
    }
    cluster_arrive();  // every CTA has read the others' histograms (they may be cleared)
    cluster_wait();
    // the bucket where the running mass from the top first reaches the
    // target, by warp 0 (as budget_kernel), on the cluster's histogram
    if (tid < 32) {
      float pm[8];
      unsigned int pc[8];
      float lm = 0.f;
      unsigned int lc = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        pm[i] = gm[255 - 8 * lane - i];
        pc[i] = gc[255 - 8 * lane - i];
        lm += pm[i];
        lc += pc[i];
      }
      float sm_ = lm;
      unsigned int sc = lc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float t = __shfl_up_sync(0xffffffffu, sm_, o);
        const unsigned int tc = __shfl_up_sync(0xffffffffu, sc, o);
        if (lane >= o) {
          sm_ += t;
          sc += tc;
        }
      }
      float em = __shfl_up_sync(0xffffffffu, sm_, 1);
      unsigned int ec = __shfl_up_sync(0xffffffffu, sc, 1);
      if (lane == 0) {
        em = 0.f;
        ec = 0u;
      }
      float am = above_m_sh + em;
      unsigned int ac = above_c_sh + ec;
      int sel = -1, low = -1;
      float am_sel = 0.f, am_low = 0.f;
      unsigned int ac_sel = 0u, ac_low = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (sel < 0 && pc[i] != 0u) {
          if (am + pm[i] >= target) {
            sel = 255 - 8 * lane - i;
            am_sel = am;
            ac_sel = ac;
          } else {
            am_low = am;
            ac_low = ac;
            am += pm[i];
            ac += pc[i];
            low = 255 - 8 * lane - i;
          }
        }
      }
      const unsigned int hit = __ballot_sync(0xffffffffu, sel >= 0);
      int src;
      if (hit != 0u) {
        src = __ffs(hit) - 1;
      } else {
        const unsigned int nz = __ballot_sync(0xffffffffu, low >= 0);
        src = nz != 0u ? 31 - __clz(nz) : 0;
        sel = low < 0 ? 0 : low;
        am_sel = low < 0 ? am : am_low;
        ac_sel = low < 0 ? ac : ac_low;
      }
      sel = __shfl_sync(0xffffffffu, sel, src);
      am_sel = __shfl_sync(0xffffffffu, am_sel, src);
      ac_sel = __shfl_sync(0xffffffffu, ac_sel, src);
      if (lane == 0) {
        above_m_sh = am_sel;
        above_c_sh = ac_sel;
        sel_sh = static_cast<unsigned int>(sel);
        prefix_sh = prefix | (static_cast<unsigned int>(sel) << shift);
      }
    }
    __syncthreads();
    mask |= 255u << shift;
  }
  if (rank == 0 && tid == 0) {
    int k;
    if (!(target > 0.f)) {
      k = 0;
    } else {
      const float v = __uint_as_float(prefix_sh);
      const unsigned int n_eq = gc[sel_sh];
      const float need = target - above_m_sh;
      unsigned int take = n_eq;
      if (v > 0.f && need > 0.f) {
        const float t = ceilf(need / v);
        take = t < static_cast<float>(n_eq) ? static_cast<unsigned int>(fmaxf(t, 1.f)) : n_eq;
      } else if (!(need > 0.f)) {
        take = 0u;
      }
      k = static_cast<int>(above_c_sh + take);
    }
    k = min(k, S);
    k_seq[b] = k;
    const int kt = min(S, (k + tile - 1) / tile * tile);
    for (int h = 0; h < Hkv; ++h) k_unit[static_cast<int64_t>(b) * Hkv + h] = kt;
  }
}

// ---------------------------------------------------------------- gather / scatter

// Compressed row t < count[u] of (b, h): the kept token idx[u, t]; rows
// past the unit's count are not written (no causal list reaches them).
// Q^ [B, Sc, Hq, D] takes the G query heads of the group; K^, V^
// [B, Hkv, Sc, D].  16 bytes per thread.
__global__ void tsa_gather_kernel(const __nv_bfloat16* __restrict__ Q,
                                  const __nv_bfloat16* __restrict__ K,
                                  const __nv_bfloat16* __restrict__ V,
                                  const int32_t* __restrict__ idx, const int32_t* __restrict__ count,
                                  int kmax, int S, int Sc, int Hq, int Hkv, int D,
                                  __nv_bfloat16* __restrict__ Qc, __nv_bfloat16* __restrict__ Kc,
                                  __nv_bfloat16* __restrict__ Vc) {
  // one warp per compressed row t of unit u = b * Hkv + h: its (G + 2) * D / 8
  // pieces (G query rows, then K, then V) spread over the lanes
  const int G = Hq / Hkv, V8 = D / 8;
  const int per_row = (G + 2) * V8;
  const int64_t u = blockIdx.y;
  const int b = static_cast<int>(u / Hkv), h = static_cast<int>(u % Hkv);
  const int n = min(count[u], Sc);
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < n; t += gridDim.x * wpb) {
    const int p = idx[u * kmax + t];
#pragma unroll 3
    for (int w = lane; w < per_row; w += 32) {
      const int part = w / V8, c = (w % V8) * 8;
      int4 v = make_int4(0, 0, 0, 0);
      if (part < G) {  // query head h*G + part
        if (p >= 0 && p < S)
          v = *reinterpret_cast<const int4*>(
              Q + ((static_cast<int64_t>(b) * S + p) * Hq + h * G + part) * D + c);
        *reinterpret_cast<int4*>(Qc + ((static_cast<int64_t>(b) * Sc + t) * Hq + h * G + part) * D +
                                 c) = v;
      } else {
        const __nv_bfloat16* src = part == G ? K : V;
        __nv_bfloat16* dst = part == G ? Kc : Vc;
        if (p >= 0 && p < S) v = *reinterpret_cast<const int4*>(src + (u * S + p) * D + c);
        *reinterpret_cast<int4*>(dst + (u * Sc + t) * D + c) = v;
      }
    }
  }
}

// Dense causal chunk lists of the compressed sequences: tile t of (b, h)
// sees chunks 0..t (chunk = tile = 64 rows); tiles past the unit's budget
// k_unit (a multiple of the tile) see none and are skipped by the dense
// attention.
__global__ void tsa_lists_kernel(const int32_t* __restrict__ k_unit, int n_tiles, int tile,
                                 int32_t* __restrict__ lists, int32_t* __restrict__ counts) {
  const int64_t ut = blockIdx.x;  // (b * Hkv + h) * n_tiles + t
  const int t = static_cast<int>(ut % n_tiles);
  const int64_t u = ut / n_tiles;
  const bool live = t * tile < k_unit[u];
  for (int c = threadIdx.x; c < n_tiles; c += blockDim.x)
    lists[ut * n_tiles + c] = (live && c <= t) ? c : -1;
  if (threadIdx.x == 0) counts[ut] = live ? t + 1 : 0;
}

__global__ void tsa_inverse_kernel(const int32_t* __restrict__ idx,
                                   const int32_t* __restrict__ count, int kmax, int S,
                                   int32_t* __restrict__ inv) {
  const int64_t u = blockIdx.x;
  for (int s = threadIdx.x; s < S; s += blockDim.x) inv[u * S + s] = -1;
  __syncthreads();
  const int n = count[u];
  for (int t = threadIdx.x; t < n; t += blockDim.x) {
    const int p = idx[u * kmax + t];
    if (p >= 0 && p < S) inv[u * S + p] = t;
  }
}

// O[b, s, h*G + g] = O^[b, inv, h*G + g] for kept positions, else 0.
__global__ void tsa_scatter_kernel(const __nv_bfloat16* __restrict__ Oc,
                                   const int32_t* __restrict__ inv, int S, int Sc, int Hq, int Hkv,
                                   int D, int B, __nv_bfloat16* __restrict__ O) {
  // one warp per output position (b, s): its Hq * D / 8 pieces over the lanes
  const int G = Hq / Hkv, V8 = D / 8, per_row = Hq * V8;
  const int lane = threadIdx.x & 31;
  const int64_t wpb = blockDim.x >> 5;
  for (int64_t bs = blockIdx.x * wpb + (threadIdx.x >> 5); bs < static_cast<int64_t>(B) * S;
       bs += gridDim.x * wpb) {
    const int b = static_cast<int>(bs / S), s = static_cast<int>(bs % S);
    const int32_t* invb = inv + static_cast<int64_t>(b) * Hkv * S + s;
#pragma unroll 4
    for (int q = lane; q < per_row; q += 32) {
      const int hq = q / V8, c = (q % V8) * 8;
      const int t = invb[static_cast<int64_t>(hq / G) * S];
      int4 v = make_int4(0, 0, 0, 0);
      if (t >= 0)
        v = *reinterpret_cast<const int4*>(Oc + ((static_cast<int64_t>(b) * Sc + t) * Hq + hq) * D + c);
      *reinterpret_cast<int4*>(O + (bs * Hq + hq) * D + c) = v;
    }
  }
}

cudaError_t set_smem_ts(const void* fn, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bytes));
}

}  // namespace

cudaError_t launch_token_budget(const Launch& l, const float* imp, int B, int S, int Hkv,
                                float tau, int tile, int32_t* k_seq, int32_t* k_unit) {
  if (B == 0) return cudaSuccess;
  if (B <= 65535 && static_cast<int64_t>(B) * kBudgetCS <= l.num_sms) {  // one cluster per sequence
    const size_t shc = static_cast<size_t>((S + kBudgetCS - 1) / kBudgetCS) * 4;
    cudaError_t e = set_smem_ts(reinterpret_cast<const void*>(budget_cluster_kernel), shc);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kBudgetCS, B);
    cfg.blockDim = dim3(kBudgetCThreads);
    cfg.dynamicSmemBytes = shc;
    cfg.stream = l.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kBudgetCS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, budget_cluster_kernel, imp, S, Hkv, tau, tile, k_seq, k_unit);
  }
  const size_t sh = static_cast<size_t>(S) * 4;
  cudaError_t e = set_smem_ts(reinterpret_cast<const void*>(budget_kernel), sh);
  if (e != cudaSuccess) return e;
  budget_kernel<<<B, kBudgetThreads, sh, l.stream>>>(imp, S, Hkv, tau, tile, k_seq, k_unit);
  return cudaGetLastError();
}

cudaError_t launch_tsa_gather(const Launch& l, const void* Q, const void* K, const void* V,
                              const int32_t* idx, const int32_t* count, int kmax, int B, int S,
                              int Sc, int Hq, int Hkv, int D, void* Qc, void* Kc, void* Vc) {
  if (B == 0 || Sc == 0) return cudaSuccess;
  const dim3 grid(8 * l.num_sms / (B * Hkv) + 1, B * Hkv);
  tsa_gather_kernel<<<grid, 256, 0, l.stream>>>(
      static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K),
      static_cast<const __nv_bfloat16*>(V), idx, count, kmax, S, Sc, Hq, Hkv, D,
      static_cast<__nv_bfloat16*>(Qc), static_cast<__nv_bfloat16*>(Kc),
      static_cast<__nv_bfloat16*>(Vc));
  return cudaGetLastError();
}

cudaError_t launch_tsa_lists(const Launch& l, const int32_t* k_unit, int U, int n_tiles, int tile,
                             int32_t* lists, int32_t* counts) {
  if (U == 0 || n_tiles == 0) return cudaSuccess;
  tsa_lists_kernel<<<U * n_tiles, 128, 0, l.stream>>>(k_unit, n_tiles, tile, lists, counts);
  return cudaGetLastError();
}

cudaError_t launch_tsa_scatter(const Launch& l, const void* Oc, const int32_t* idx,
                               const int32_t* count, int kmax, int B, int S, int Sc, int Hq,
                               int Hkv, int D, int32_t* inv, void* O) {
  if (B == 0 || S == 0) return cudaSuccess;
  tsa_inverse_kernel<<<B * Hkv, 512, 0, l.stream>>>(idx, count, kmax, S, inv);
  tsa_scatter_kernel<<<8 * l.num_sms, 256, 0, l.stream>>>(
      static_cast<const __nv_bfloat16*>(Oc), inv, S, Sc, Hq, Hkv, D, B,
      static_cast<__nv_bfloat16*>(O));
  return cudaGetLastError();
}

size_t token_importance_scratch_bytes(int B, int S, int Hkv, int G, int n_obs) {
  const int64_t nblk = (S + kImpKeys - 1) / kImpKeys;
  const int64_t R = static_cast<int64_t>(G) * n_obs;
  return static_cast<size_t>(B) * Hkv * R * 2 * 4 * (nblk + 1);
}

cudaError_t launch_token_importance(const Launch& l, const void* Q, const void* K, int B, int S,
                                    int Hq, int Hkv, int D, int n_obs, float scale, float* imp,
                                    float* scratch) {
  if (B == 0 || S == 0) return cudaSuccess;
  const int G = Hq / Hkv, R = G * n_obs;
  const int nblk = (S + kImpKeys - 1) / kImpKeys;
  float* part = scratch;
  float* stats = scratch + static_cast<size_t>(B) * Hkv * nblk * R * 2;
  const size_t lds = static_cast<size_t>(D + 8) * 2;
  const size_t sh1 = ((R + 31) / 32 * 32 + 2 * kImpKeys) * lds;
  // pass 1 is persistent: about one CTA per SM over the (b, h) pairs
  const int nsplit = std::max(1, std::min(nblk, l.num_sms / std::max(1, B * Hkv)));
  const size_t sh2 = (R + kImpKeys) * lds + static_cast<size_t>(R) * 2 * 4;
  const dim3 grid(nblk, Hkv, B);
  const float sl2 = scale * kLog2eF;
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(Q);
  const __nv_bfloat16* k = static_cast<const __nv_bfloat16*>(K);
  cudaError_t e;
  if (D == 128) {
    e = set_smem_ts(reinterpret_cast<const void*>(imp_stats_kernel<128>), sh1);
    if (e == cudaSuccess) e = set_smem_ts(reinterpret_cast<const void*>(imp_weight_kernel<128>), sh2);
    if (e != cudaSuccess) return e;
    imp_stats_kernel<128><<<dim3(nsplit, Hkv, B), kStatsThreads, sh1, l.stream>>>(
        q, k, S, Hq, Hkv, G, n_obs, sl2, nblk, part);
    imp_combine_kernel<<<dim3(B * Hkv, (R + 31) / 32), kCombineWarps * 32, 0, l.stream>>>(
        part, nsplit, R, stats);
    imp_weight_kernel<128><<<grid, kImpThreads, sh2, l.stream>>>(q, k, S, Hq, Hkv, G, n_obs, sl2,
                                                                 stats, imp);
  } else {
    e = set_smem_ts(reinterpret_cast<const void*>(imp_stats_kernel<64>), sh1);
    if (e == cudaSuccess) e = set_smem_ts(reinterpret_cast<const void*>(imp_weight_kernel<64>), sh2);
    if (e != cudaSuccess) return e;
    imp_stats_kernel<64><<<dim3(nsplit, Hkv, B), kStatsThreads, sh1, l.stream>>>(
        q, k, S, Hq, Hkv, G, n_obs, sl2, nblk, part);
    imp_combine_kernel<<<dim3(B * Hkv, (R + 31) / 32), kCombineWarps * 32, 0, l.stream>>>(
        part, nsplit, R, stats);
    imp_weight_kernel<64><<<grid, kImpThreads, sh2, l.stream>>>(q, k, S, Hq, Hkv, G, n_obs, sl2,
                                                                stats, imp);
  }
  return cudaGetLastError();
}

}  // namespace csa
