// Token Sparse Attention for prefill (gist.science/ko/paper/2602.03216,
// section 2): which tokens each KV head keeps, and the gather / scatter
// around the dense causal attention of the kept tokens.
//
//   importance   a proxy attention map of the last n_obs query rows of every
//                query head against all keys of its KV head; the importance
//                of key j is the sum over those rows of its softmax weight
//                (the rows of the GQA group's heads summed: one importance
//                per KV head).  Two passes over K on the tensor cores
//                (tcgen05, accumulators in tensor memory): per-row max and
//                sum over key blocks (rows as M, keys as N), then, with the
//                rows' final max and sum, the weights summed per key (keys
//                as M, rows as N).  K is read twice.
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
#include <algorithm>

#include "internal.h"
#include "tcgen05.cuh"

namespace csa {
namespace {

// ---------------------------------------------------------------- importance
//
// Both passes are persistent over blocks of kTcKeys keys: CTA (split, h, b)
// takes blocks split, split + nsplit, ... of KV head h of sequence b.  The
// head's observed query rows (R = G * n_obs of them, padded with zero rows
// to Rp, a multiple of 128) are copied once into shared memory by TMA as
// 64-column slabs with the 128-byte swizzle; the key blocks stream through a
// ring of TMA stages; one thread issues the MMAs into a double-buffered
// accumulator in tensor memory:
//   pass 1   S = Q_obs K_blk^T, M = 128 observed rows per MMA (Rp / 128 of
//            them), N = 128 keys.  TMEM lane = row: each epilogue thread
//            keeps its row's running max and sum of 2^(s - max).
//   pass 2   S^T = K_blk Q_obs^T, M = 128 keys, N = the observed rows (up to
//            256 per MMA).  TMEM lane = key: each thread sums its key's
//            weights 2^(s - max_r - log2 sum_r) along its own TMEM lane.
// Warp 0 issues the TMA copies, warp 1 owns the tensor memory and one of its
// threads issues the MMAs, warps 2-17 are four warpgroups that read the
// accumulators (warp w reaches TMEM lanes 32 (w % 4) .. + 31): in pass 1
// warpgroup g takes the 128-row tiles g % 2 and g % 2 + 2, keys of half g / 2
// of each block (the halves keep separate row statistics, written as two
// splits); in pass 2 it takes a quarter of the observed rows, and the
// quarters' sums meet in shared memory.  A third of the exponentials run on
// the FMA pipe.  Pass 2 is launched behind pass 1
// with programmatic dependent launch: its copies and MMAs start while pass 1
// drains, and its epilogue waits (griddepcontrol.wait) for pass 1's per-split
// row statistics, which it combines itself.  Pass 1 reads K with the default
// L2 policy so that pass 2, which reads it last, finds much of it in L2.

constexpr int kTcKeys = 128;
constexpr int kTcEpiWarps = 16;
constexpr int kTcThreads = (2 + kTcEpiWarps) * 32;
constexpr int kTcMaxNS = 4;
constexpr size_t kTcMinSmem = 120 * 1024;  // one CTA per SM: it allocates all 512 TMEM columns
constexpr size_t kTcMaxSmem = 232448;      // 227 KB per block
constexpr int kTcEmuPeriod = 3;            // one pair of exponentials in 3 on the FMA pipe
constexpr float kLog2eF = 1.4426950408889634f;

struct ImpParams {
  int S, Hkv, G, n_obs, R, Rp, D, nblk, nsplit, NS, qbox;
  float sl2;    // scale * log2(e)
  float2* part;  // [B, Hkv, 2 nsplit, R]: (max, sum of 2^(s - max)) per split and key half, log2 units
  float* imp;    // [B, Hkv, S]
  DevErr err;
};

// Shared-memory layout, offsets from the 1024-aligned base: Q slabs | K
// stages | mbarriers + TMEM slot | pass 2: bias[Rp], lim[Rp], red[2][3][128].
struct ImpLayout {
  int kv_off, stage_bytes, bar_off, bias_off, lim_off, red_off;
  size_t total;
};

__host__ __device__ inline ImpLayout imp_layout(int Rp, int D, int NS) {
  ImpLayout y;
  y.kv_off = Rp * D * 2;
  y.stage_bytes = kTcKeys * D * 2;
  y.bar_off = y.kv_off + NS * y.stage_bytes;
  y.bias_off = y.bar_off + 256;
  y.lim_off = y.bias_off + Rp * 4;
  y.red_off = y.lim_off + Rp * 4;
  y.total = 1024 + static_cast<size_t>(y.red_off) + 2 * 3 * kTcKeys * 4;
  return y;
}

__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Named barrier over the eight epilogue warps.
__device__ __forceinline__ void epi_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kTcEpiWarps * 32) : "memory");
}

__device__ __forceinline__ int imp_blocks(const ImpParams& p, int split) {
  return split < p.nblk ? (p.nblk - split + p.nsplit - 1) / p.nsplit : 0;
}

// Warp 0, lane 0: the observed rows once, then this CTA's key blocks into
// the ring.  Returns the number of key blocks issued.
__device__ uint32_t imp_produce(const ImpParams& p, const CUtensorMap* tmQ, const CUtensorMap* tmK,
                                uint32_t sQ, uint32_t sKV, uint32_t stage_bytes, uint32_t q_full,
                                uint32_t kv_full, uint32_t kv_empty, int b, int h, int split,
                                bool evict_first) {
  const int nslab = p.D / 64;
  mbar_arrive_expect_tx(q_full, static_cast<uint32_t>(p.R) * p.D * 2);
  for (int g = 0; g < p.G; ++g)
    for (int i = 0; i < p.n_obs; i += p.qbox)
      for (int sl = 0; sl < nslab; ++sl)
        tma_load_2d(sQ + sl * p.Rp * 128 + (g * p.n_obs + i) * 128, tmQ,
                    (h * p.G + g) * p.D + sl * 64, b * p.S + p.S - p.n_obs + i, q_full);
  const uint64_t pol = evict_first ? l2_policy_evict_first() : 0;
  const int krow0 = (b * p.Hkv + h) * p.S;
  uint32_t it = 0;
  for (int blk = split; blk < p.nblk; blk += p.nsplit, ++it) {
    const uint32_t s = it % p.NS;
    if (!mbar_wait(kv_empty + 8 * s, ((it / p.NS) & 1u) ^ 1u, p.err)) break;
    const uint32_t fb = kv_full + 8 * s;
    mbar_arrive_expect_tx(fb, stage_bytes);
    for (int sl = 0; sl < nslab; ++sl) {
      const uint32_t dst = sKV + s * stage_bytes + sl * (kTcKeys * 128);
      if (evict_first)
        tma_load_2d_hint(dst, tmK, sl * 64, krow0 + blk * kTcKeys, fb, pol);
      else
        tma_load_2d(dst, tmK, sl * 64, krow0 + blk * kTcKeys, fb);
    }
  }
  // no copy may still be landing when the CTA retires
  const uint32_t first = it > static_cast<uint32_t>(p.NS) ? it - p.NS : 0u;
  for (uint32_t i = first; i < it; ++i)
    mbar_wait(kv_full + 8 * (i % p.NS), (i / p.NS) & 1u, p.err);
  mbar_wait(q_full, 0u, p.err);
  return it;
}

// Warp 1, lane 0: the MMAs of every key block this CTA takes.  Pass 1:
// D[buf][128 mt .. + 128) = Q rows of tile mt x K_blk^T for each 128-row
// tile; pass 2: D[buf][n0 .. + N) = K_blk x Q rows n0 .. n0 + N - 1.  Each
// block's stage is released and its accumulator published by commits.
template <bool kPass2>
__device__ void imp_mma(const ImpParams& p, uint32_t tmem, uint32_t sQ, uint32_t sKV,
                        uint32_t stage_bytes, uint32_t q_full, uint32_t kv_full,
                        uint32_t kv_empty, uint32_t tm_full, uint32_t tm_free, uint32_t drain,
                        int nb) {
  const int nbuf = 2 * p.Rp <= 512 ? 2 : 1;
  const int ksteps = p.D / 16;
  bool ok = mbar_wait(q_full, 0u, p.err);
  for (int i = 0; i < nb && ok; ++i) {
    const uint32_t s = i % p.NS;
    const int buf = i % nbuf, use = i / nbuf;
    if (!mbar_wait(kv_full + 8 * s, (i / p.NS) & 1u, p.err)) break;
    if (use > 0 && !mbar_wait(tm_free + 8 * buf, (use - 1) & 1u, p.err)) break;
    tc_fence_after();
    const uint32_t kb = sKV + s * stage_bytes;
    const uint32_t d0 = tmem + buf * p.Rp;
    if (!kPass2) {
      const uint32_t idesc = idesc_bf16(128, kTcKeys, 0);
      for (int mt = 0; mt < p.Rp / 128; ++mt)
        for (int kk = 0; kk < ksteps; ++kk) {
          const uint32_t qa = sQ + (kk >> 2) * (p.Rp * 128) + mt * 16384 + (kk & 3) * 32;
          const uint32_t ka = kb + (kk >> 2) * (kTcKeys * 128) + (kk & 3) * 32;
          umma_ss(d0 + mt * 128, smem_desc(qa, 16, 1024), smem_desc(ka, 16, 1024), idesc,
                  kk > 0 ? 1u : 0u);
        }
    } else {
      for (int n0 = 0; n0 < p.Rp; n0 += 256) {
        const int n = min(256, p.Rp - n0);
        const uint32_t idesc = idesc_bf16(128, n, 0);
        for (int kk = 0; kk < ksteps; ++kk) {
          const uint32_t ka = kb + (kk >> 2) * (kTcKeys * 128) + (kk & 3) * 32;
          const uint32_t qa = sQ + (kk >> 2) * (p.Rp * 128) + n0 * 128 + (kk & 3) * 32;
          umma_ss(d0 + n0, smem_desc(ka, 16, 1024), smem_desc(qa, 16, 1024), idesc,
                  kk > 0 ? 1u : 0u);
        }
      }
    }
    umma_commit(kv_empty + 8 * s);
    umma_commit(tm_full + 8 * buf);
  }
  // every MMA issued here has finished before the tensor memory is freed
  umma_commit(drain);
  mbar_wait(drain, 0u, p.err);
}

// 2^x of a pair, every kTcEmuPeriod-th pair on the FMA pipe.
__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ int2 lds_s2(uint32_t addr) {
  int2 v;
  asm volatile("ld.shared.v2.s32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// Pass 1 epilogue, one row against 64 keys of a block: x = the raw scores,
// keys i <= lim visible (lim >= 63: all); folds them into the running (m:
// max of s * sl2, l: sum of 2^(s sl2 - m)).
__device__ __forceinline__ void stats_fold(const uint32_t (&r)[2][32], int lim, float sl2,
                                           float& m, float& l) {
  float x[64];
#pragma unroll
  for (int i = 0; i < 64; ++i) x[i] = __uint_as_float(r[i >> 5][i & 31]);
  if (lim < 63) {
#pragma unroll
    for (int i = 0; i < 64; ++i) x[i] = i <= lim ? x[i] : -INFINITY;
  }
  float mq[2];
#pragma unroll
  for (int a = 0; a < 2; ++a) {
    float v = fmax3(x[32 * a], x[32 * a + 1], x[32 * a + 2]);
#pragma unroll
    for (int k = 3; k < 31; k += 2) v = fmax3(v, x[32 * a + k], x[32 * a + k + 1]);
    mq[a] = fmaxf(v, x[32 * a + 31]);
  }
  const float mn = fmaxf(mq[0], mq[1]) * sl2;
  const float mnew = fmaxf(m, mn);
  if (mnew == -INFINITY) return;  // no visible key yet
  const float2 sc = make_float2(sl2, sl2), nb = make_float2(-mnew, -mnew);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                   make_float2(0.f, 0.f)};
#pragma unroll
  for (int q = 0; q < 32; q += kTcEmuPeriod * 2) {
#pragma unroll
    for (int t = 0; t < kTcEmuPeriod * 2; ++t) {
      if (q + t < 32) {
        const float2 a = __ffma2_rn(make_float2(x[2 * (q + t)], x[2 * (q + t) + 1]), sc, nb);
        float2 e;
        if (t % kTcEmuPeriod == kTcEmuPeriod - 1) e = exp2_fma2(a);
        else e = make_float2(fast_exp2(a.x), fast_exp2(a.y));
        acc[(q + t) & 3] = __fadd2_rn(acc[(q + t) & 3], e);
      }
    }
  }
  const float2 s01 = __fadd2_rn(acc[0], acc[1]), s23 = __fadd2_rn(acc[2], acc[3]);
  l = l * fast_exp2(m - mnew) + ((s01.x + s01.y) + (s23.x + s23.y));
  m = mnew;
}

// Pass 2 epilogue, one key against 32 observed rows c0 .. c0 + 31: adds
// 2^(s sl2 + bias_c) over the rows it may see (all unless `masked`: then
// only rows whose position lim_c >= j).
__device__ __forceinline__ void weight_fold(const uint32_t (&r)[32], uint32_t bias_a,
                                            uint32_t lim_a, int c0, bool masked, int j, float sl2,
                                            float2 (&acc)[4]) {
  const float2 sc = make_float2(sl2, sl2);
#pragma unroll
  for (int q = 0; q < 16; q += kTcEmuPeriod * 2) {
#pragma unroll
    for (int t = 0; t < kTcEmuPeriod * 2; ++t) {
      if (q + t < 16) {
        const int pr = q + t, c = c0 + 2 * pr;
        const float2 bb = lds_f2(bias_a + c * 4);
        const float2 a =
            __ffma2_rn(make_float2(__uint_as_float(r[2 * pr]), __uint_as_float(r[2 * pr + 1])), sc, bb);
        float2 ev;
        if (t % kTcEmuPeriod == kTcEmuPeriod - 1) ev = exp2_fma2(a);
        else ev = make_float2(fast_exp2(a.x), fast_exp2(a.y));
        if (masked) {
          const int2 lm = lds_s2(lim_a + c * 4);
          ev.x = j <= lm.x ? ev.x : 0.f;
          ev.y = j <= lm.y ? ev.y : 0.f;
        }
        acc[pr & 3] = __fadd2_rn(acc[pr & 3], ev);
      }
    }
  }
}

template <bool kPass2>
__global__ void __launch_bounds__(kTcThreads, 1)
    imp_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ ImpParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const ImpLayout Y = imp_layout(p.Rp, p.D, p.NS);
  const uint32_t sb = smem_u32(smem);
  const uint32_t sQ = sb, sKV = sb + Y.kv_off;
  const uint32_t kv_full = sb + Y.bar_off, kv_empty = kv_full + 8 * kTcMaxNS;
  const uint32_t tm_full = kv_empty + 8 * kTcMaxNS, tm_free = tm_full + 16;  // [2] each
  const uint32_t q_full = tm_free + 16, drain = q_full + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Y.bar_off + 8 * (2 * kTcMaxNS + 6));
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = imp_blocks(p, split);
  const int nbuf = 2 * p.Rp <= 512 ? 2 : 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.NS; ++s) {
      mbar_init(kv_full + 8 * s, 1);
      mbar_init(kv_empty + 8 * s, 1);
    }
    // pass 1: the warps of the warpgroups that have a 128-row tile read the
    // accumulator (two per tile parity); pass 2: all of them
    const int readers = kPass2 ? kTcEpiWarps : 8 * min(2, p.Rp / 128);
    for (int k = 0; k < 2; ++k) {
      mbar_init(tm_full + 8 * k, 1);
      mbar_init(tm_free + 8 * k, readers);
    }
    mbar_init(q_full, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
  }
  if (warp == 1) tmem_alloc<512>(tmem_slot);
  if (warp >= 2 && p.Rp > p.R) {  // zero the padding rows of every slab (MMA operands)
    const int pad16 = (p.Rp - p.R) * 8;  // 16-byte pieces per slab
    for (int e = threadIdx.x - 64; e < pad16 * (p.D / 64); e += kTcEpiWarps * 32) {
      const int sl = e / pad16, o = e % pad16;
      *reinterpret_cast<uint4*>(smem + sl * p.Rp * 128 + p.R * 128 + o * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (!kPass2) grid_dependents_launch();  // pass 2 may start its copies as SMs free up

  if (warp == 0) {
    if (lane == 0)
      imp_produce(p, &tmQ, &tmK, sQ, sKV, Y.stage_bytes, q_full, kv_full, kv_empty, b, h, split,
                  kPass2);
  } else if (warp == 1) {
    if (lane == 0)
      imp_mma<kPass2>(p, tmem, sQ, sKV, Y.stage_bytes, q_full, kv_full, kv_empty, tm_full, tm_free,
                      drain, nb);
    __syncwarp();
  } else {
    const int e = warp - 2, grp = e >> 2, quarter = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int64_t bh = static_cast<int64_t>(b) * p.Hkv + h;
    if (!kPass2) {
      // ------------------------------------------------ pass 1: row statistics
      const int tp = grp & 1, kh = grp >> 1;  // tile parity, key half
      float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
      const int nmt = p.Rp / 128;
      for (int i = 0; i < nb && tp < nmt; ++i) {
        const int buf = i % nbuf, use = i / nbuf;
        const int j0 = (split + i * p.nsplit) * kTcKeys + kh * 64;
        if (!warp_wait(tm_full + 8 * buf, use & 1u, p.err)) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int mt = tp + 2 * k;
          if (mt >= nmt) break;
          uint32_t r[2][32];
          const uint32_t ta = tmem + lane_base + buf * p.Rp + mt * 128 + kh * 64;
          tmem_ld32(ta, r[0]);
          tmem_ld32(ta + 32, r[1]);
          tmem_wait_ld();
          if (mt + 2 >= nmt) {  // this warp's last read of the buffer
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tm_free + 8 * buf);
          }
          const int row = mt * 128 + quarter * 32 + lane;
          // keys past the first observed position are masked per row
          const int lim = (j0 + 63 > p.S - p.n_obs) ? p.S - p.n_obs + (row % p.n_obs) - j0 : 63;
          stats_fold(r, lim, p.sl2, m[k], l[k]);
        }
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int row = (tp + 2 * k) * 128 + quarter * 32 + lane;
        if (tp + 2 * k < nmt && row < p.R)
          p.part[(bh * 2 * p.nsplit + 2 * split + kh) * p.R + row] = make_float2(m[k], l[k]);
      }
    } else {
      // ------------------------------------------------ pass 2: weights per key
      float* bias = reinterpret_cast<float*>(smem + Y.bias_off);
      int* lim = reinterpret_cast<int*>(smem + Y.lim_off);
      float* red = reinterpret_cast<float*>(smem + Y.red_off);  // [2][3][128]
      grid_dependency_wait();  // pass 1's statistics are complete and visible
      const int nparts = 2 * p.nsplit;
      for (int r = threadIdx.x - 64; r < p.Rp; r += kTcEpiWarps * 32) {
        float bv = -INFINITY;
        int lv = -1;
        if (r < p.R) {
          // the row's (max, sum) over the splits, kStatBatch splits' loads in
          // flight at a time and folded online (each batch rescales the sum)
          constexpr int kStatBatch = 16;
          const float2* pr = p.part + bh * nparts * p.R + r;
          float M = -INFINITY, Ls = 0.f;
          for (int s0 = 0; s0 < nparts; s0 += kStatBatch) {
            float2 v[kStatBatch];
#pragma unroll
            for (int k = 0; k < kStatBatch; ++k)
              v[k] = s0 + k < nparts ? pr[static_cast<int64_t>(s0 + k) * p.R]
                                     : make_float2(-INFINITY, 0.f);
            float bm = M;
#pragma unroll
            for (int k = 0; k < kStatBatch; ++k) bm = fmaxf(bm, v[k].x);
            if (bm == -INFINITY) continue;
            Ls = M == -INFINITY ? 0.f : Ls * exp2f(M - bm);
#pragma unroll
            for (int k = 0; k < kStatBatch; ++k)
              if (v[k].x != -INFINITY) Ls += v[k].y * exp2f(v[k].x - bm);
            M = bm;
          }
          // weight of score s: 2^(s sl2 - M) / Ls = 2^(s sl2 + bias)
          bv = Ls > 0.f ? -(M + log2f(Ls)) : -INFINITY;
          lv = p.S - p.n_obs + r % p.n_obs;
        }
        bias[r] = bv;
        lim[r] = lv;
      }
      epi_sync();
      const uint32_t bias_a = smem_u32(bias), lim_a = smem_u32(lim);
      const int quarter_cols = p.Rp / 4, c_begin = grp * quarter_cols;
      const int key = quarter * 32 + lane;
      // every epilogue warp meets the others once per block, also after a
      // timed-out wait (it then reads nothing more), so the named barrier
      // never waits for a warp that left
      bool ok = true;
      for (int i = 0; i < nb; ++i) {
        const int buf = i % nbuf, use = i / nbuf;
        const int j0 = (split + i * p.nsplit) * kTcKeys, j = j0 + key;
        const bool masked = j0 + kTcKeys - 1 > p.S - p.n_obs;
        if (ok) ok = warp_wait(tm_full + 8 * buf, use & 1u, p.err);
        tc_fence_after();
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
        // this warpgroup's columns, two 32-column loads in flight when there are two
        for (int c0 = c_begin; ok && c0 < c_begin + quarter_cols; c0 += 64) {
          const bool two = c0 + 32 < c_begin + quarter_cols;
          uint32_t r0[32], r1[32];
          const uint32_t ta = tmem + lane_base + buf * p.Rp + c0;
          tmem_ld32(ta, r0);
          if (two) tmem_ld32(ta + 32, r1);
          tmem_wait_ld();
          if (c0 + 64 >= c_begin + quarter_cols) {  // this warp's last read of the buffer
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tm_free + 8 * buf);
          }
          weight_fold(r0, bias_a, lim_a, c0, masked, j, p.sl2, acc);
          if (two) weight_fold(r1, bias_a, lim_a, c0 + 32, masked, j, p.sl2, acc);
        }
        const float2 s01 = __fadd2_rn(acc[0], acc[1]), s23 = __fadd2_rn(acc[2], acc[3]);
        const float w = (s01.x + s01.y) + (s23.x + s23.y);
        float* rb = red + (i & 1) * 3 * kTcKeys;
        if (grp > 0) rb[(grp - 1) * kTcKeys + key] = w;
        epi_sync();
        if (ok && grp == 0 && j < p.S)
          p.imp[bh * p.S + j] = ((w + rb[key]) + rb[kTcKeys + key]) + rb[2 * kTcKeys + key];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<512>(tmem);
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

__global__ void __launch_bounds__(kBudgetCThreads) budget_cluster_kernel(
    const float* __restrict__ imp, int S, int Hkv, float tau, int tile, int32_t* __restrict__ k_seq,
    int32_t* __restrict__ k_unit) {
  cluster_arrive_relaxed();
  extern __shared__ __align__(16) uint8_t sm[];
  constexpr int kWarps = kBudgetCThreads / 32;
  unsigned int* whc = reinterpret_cast<unsigned int*>(sm);  // [kWarps][256] per-warp counts
  float* whm = reinterpret_cast<float*>(whc + kWarps * 256);  // [kWarps][256] per-warp masses
  float* ms = whm + kWarps * 256;            // [S / CS] this CTA's masses
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
  // rounds of kBudgetJ * blockDim.x tokens (one round up to S = 32768 over
  // kBudgetCS CTAs), each unrolled so that every load of the thread in the
  // round is in flight together
  constexpr int kBudgetJ = 8;
  for (int j0 = 0; j0 < n; j0 += kBudgetJ * kBudgetCThreads) {
#pragma unroll
    for (int k = 0; k < kBudgetJ; ++k) {
      const int j = j0 + tid + k * kBudgetCThreads;
      if (j < n) {
        float m = 0.f;
#pragma unroll 8
        for (int h = 0; h < Hkv; ++h) m += ib[static_cast<int64_t>(h) * S + j];
        m = fmaxf(m, 0.f);
        ms[j] = m;
        part += m;
      }
    }
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
    // each warp's own histogram (shared-memory atomics contend only within
    // the warp: the masses' high bytes take few values), then the CTA's as
    // their sum in warp order
    unsigned int* wc = whc + (tid >> 5) * 256;
    float* wm = whm + (tid >> 5) * 256;
    for (int d = lane; d < 256; d += 32) {
      wc[d] = 0u;
      wm[d] = 0.f;
    }
    __syncwarp();
    const unsigned int prefix = prefix_sh;
    for (int j = tid; j < n; j += blockDim.x) {
      const unsigned int key = __float_as_uint(ms[j]);
      if ((key & mask) == prefix) {
        const int d = static_cast<int>((key >> shift) & 255u);
        atomicAdd(&wc[d], 1u);
        atomicAdd(&wm[d], ms[j]);
      }
    }
    __syncthreads();
    for (int d = tid; d < 256; d += blockDim.x) {
      unsigned int c = 0u;
      float mm = 0.f;
#pragma unroll 4
      for (int w = 0; w < kWarps; ++w) {
        c += whc[w * 256 + d];
        mm += whm[w * 256 + d];
      }
      hc[d] = c;
      hm[d] = mm;
    }
    cluster_arrive();  // every CTA's histogram of this pass is complete
    cluster_wait();
    for (int d = tid; d < 256; d += blockDim.x) {  // the cluster's, added in rank order
      unsigned int c = 0u;
      float mm = 0.f;
      // all the cluster's loads in flight at once (the launch's cluster has
      // kBudgetCS CTAs), then added in rank order
      unsigned int cr[kBudgetCS];
      float mr[kBudgetCS];
#pragma unroll
      for (int r = 0; r < kBudgetCS; ++r) {
        cr[r] = ld_cluster_u32(cluster_map(smem_u32(hc + d), r));
        mr[r] = ld_cluster_f32(cluster_map(smem_u32(hm + d), r));
      }
#pragma unroll
      for (int r = 0; r < kBudgetCS; ++r) {
        c += cr[r];
        mm += mr[r];
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
  const int stride = gridDim.x * wpb;
  int t = blockIdx.x * wpb + (threadIdx.x >> 5);
  int p_next = t < n ? idx[u * kmax + t] : 0;
  for (; t < n; t += stride) {
    const int p = p_next;
    // the next row's position is loaded while this row's pieces move
    if (t + stride < n) p_next = idx[u * kmax + t + stride];
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

// O[b, s, h*G + g] = O^[b, inv, h*G + g] for kept positions, else 0.  CTA
// (chunk, b) takes kScatterRows positions: the inverse entries of every KV
// head for them into shared memory (one coalesced row per head), then the
// threads move independent 16-byte pieces, consecutive threads consecutive
// pieces of an output row (coalesced stores; a kept row reads each head's
// D contiguous elements of O^), eight rows in flight per thread.
constexpr int kScatterRows = 32;
constexpr int kScatterThreads = 256;
template <int D>
__global__ void __launch_bounds__(kScatterThreads) tsa_scatter_kernel(
    const __nv_bfloat16* __restrict__ Oc, const int32_t* __restrict__ inv, int S, int Sc, int Hq,
    int Hkv, __nv_bfloat16* __restrict__ O) {
  extern __shared__ int inv_s[];  // [Hkv][kScatterRows]
  constexpr int V8 = D / 8;
  const int b = blockIdx.y, s0 = blockIdx.x * kScatterRows;
  const int nrow = min(kScatterRows, S - s0);
  for (int e = threadIdx.x; e < Hkv * kScatterRows; e += blockDim.x) {
    const int h = e / kScatterRows, r = e % kScatterRows;
    int t = r < nrow ? inv[(static_cast<int64_t>(b) * Hkv + h) * S + s0 + r] : -1;
    inv_s[e] = t < Sc ? t : -1;
  }
  __syncthreads();
  const int G = Hq / Hkv, per_row = Hq * V8;
  const __nv_bfloat16* ob = Oc + static_cast<int64_t>(b) * Sc * Hq * D;
  __nv_bfloat16* dst = O + (static_cast<int64_t>(b) * S + s0) * Hq * D;
  for (int q = threadIdx.x; q < per_row; q += blockDim.x) {
    const int hq = q / V8, c = (q % V8) * 8;
    const int* it = inv_s + (hq / G) * kScatterRows;
#pragma unroll 8
    for (int r = 0; r < nrow; ++r) {
      const int t = it[r];
      int4 v = make_int4(0, 0, 0, 0);
      if (t >= 0)
        v = __ldcs(reinterpret_cast<const int4*>(ob + (static_cast<int64_t>(t) * Hq + hq) * D + c));
      // O is written once and not read again here: streaming (evict-first) stores
      __stcs(reinterpret_cast<int4*>(dst + (static_cast<int64_t>(r) * Hq + hq) * D + c), v);
    }
  }
}

cudaError_t set_smem_ts(const void* fn, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bytes));
}

}  // namespace

bool token_budget_cluster_fits(int B, int num_sms) {
  return B <= 65535 && static_cast<int64_t>(B) * kBudgetCS <= num_sms;
}

cudaError_t launch_token_budget(const Launch& l, const float* imp, int B, int S, int Hkv,
                                float tau, int tile, int32_t* k_seq, int32_t* k_unit) {
  if (B == 0) return cudaSuccess;
  if (token_budget_cluster_fits(B, l.num_sms)) {  // one cluster per sequence
    const size_t shc = static_cast<size_t>((S + kBudgetCS - 1) / kBudgetCS) * 4 +
                       static_cast<size_t>(kBudgetCThreads / 32) * 256 * 8;
    // always set: with its static histograms the kernel may pass 48 KB in all
    cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(budget_cluster_kernel),
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(shc));
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

cudaError_t launch_tsa_scatter(const Launch& l, const void* Oc, const int32_t* idx,
                               const int32_t* count, int kmax, int B, int S, int Sc, int Hq,
                               int Hkv, int D, int32_t* inv, void* O, bool inv_ready) {
  if (B == 0 || S == 0) return cudaSuccess;
  if (!inv_ready) tsa_inverse_kernel<<<B * Hkv, 512, 0, l.stream>>>(idx, count, kmax, S, inv);
  const dim3 grid((S + kScatterRows - 1) / kScatterRows, B);
  const size_t sh = static_cast<size_t>(Hkv) * kScatterRows * 4;
  const auto* oc = static_cast<const __nv_bfloat16*>(Oc);
  auto* o = static_cast<__nv_bfloat16*>(O);
  if (D == 128) {
    cudaError_t e = set_smem_ts(reinterpret_cast<const void*>(tsa_scatter_kernel<128>), sh);
    if (e != cudaSuccess) return e;
    tsa_scatter_kernel<128><<<grid, kScatterThreads, sh, l.stream>>>(oc, inv, S, Sc, Hq, Hkv, o);
  } else {
    cudaError_t e = set_smem_ts(reinterpret_cast<const void*>(tsa_scatter_kernel<64>), sh);
    if (e != cudaSuccess) return e;
    tsa_scatter_kernel<64><<<grid, kScatterThreads, sh, l.stream>>>(oc, inv, S, Sc, Hq, Hkv, o);
  }
  return cudaGetLastError();
}

size_t token_importance_scratch_bytes(int B, int S, int Hkv, int G, int n_obs) {
  // row statistics of pass 1 per split and key half: at most one split per
  // key block
  const int64_t nblk = (S + kTcKeys - 1) / kTcKeys;
  const int64_t R = static_cast<int64_t>(G) * n_obs;
  return static_cast<size_t>(B) * Hkv * R * 2 * 4 * 2 * nblk;
}

cudaError_t launch_token_importance(const Launch& l, const void* Q, const void* K, int B, int S,
                                    int Hq, int Hkv, int D, int n_obs, float scale, float* imp,
                                    float* scratch, std::string* why) {
  if (B == 0 || S == 0) return cudaSuccess;
  ImpParams p{};
  p.S = S;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.n_obs = n_obs;
  p.R = p.G * n_obs;
  p.Rp = (p.R + 127) & ~127;
  p.D = D;
  p.nblk = (S + kTcKeys - 1) / kTcKeys;
  // about one CTA per SM over the (b, h) pairs
  p.nsplit = std::max(1, std::min(p.nblk, l.num_sms / std::max(1, B * Hkv)));
  p.qbox = std::min(256, n_obs & -n_obs);  // n_obs is a multiple of 8
  p.sl2 = scale * kLog2eF;
  p.part = reinterpret_cast<float2*>(scratch);
  p.imp = imp;
  p.err = l.err;
  const int stage = kTcKeys * D * 2;
  const size_t fixed = imp_layout(p.Rp, D, 0).total;
  p.NS = static_cast<int>(std::min<size_t>(kTcMaxNS, (kTcMaxSmem - fixed) / stage));
  if (p.NS < 2) {
    if (why) *why = "token importance: observed rows do not fit in shared memory";
    return cudaErrorInvalidValue;
  }
  const size_t smem = std::max(kTcMinSmem, imp_layout(p.Rp, D, p.NS).total);
  CUtensorMap tmQ, tmK;
  if (!make_tmap_bf16_2d(&tmQ, Q, static_cast<uint64_t>(B) * S, static_cast<uint64_t>(Hq) * D,
                         static_cast<uint64_t>(Hq) * D, p.qbox, 64, why))
    return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tmK, K, static_cast<uint64_t>(B) * Hkv * S, D, D, kTcKeys, 64, why))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(imp_tc_kernel<false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(imp_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(p.nsplit, Hkv, B);
  imp_tc_kernel<false><<<grid, kTcThreads, smem, l.stream>>>(tmQ, tmK, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // pass 2 behind pass 1 (programmatic dependent launch)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = l.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, imp_tc_kernel<true>, tmQ, tmK, p);
}

}  // namespace csa
