// Block-sparse causal prefill on the 5th-generation tensor cores (tcgen05,
// accumulators in tensor memory).
//
// Work unit = (sequence b, KV head h, query tile t): the 64 query rows of
// the tile for each of the G = 4 query heads of the group, stacked into 256
// rows (head-major) that share the tile's chunk list.  The 256 rows are two
// 128-row halves, each an M = 128 MMA operand.  Per selected chunk (64 keys):
//   S_half = Q_half K^T      tcgen05.mma M=128 N=64 K=128, A/B from shared memory
//   P_half = softmax rows    one warpgroup per half reads S with tcgen05.ld,
//                            keeps the running max/sum per row and writes P
//                            back to tensor memory as bf16 pairs (tcgen05.st)
//   O_half += P_half V       tcgen05.mma M=128 N=128 K=64, A = P from tensor
//                            memory, B = V from shared memory (MN-major)
// The softmax releases S as soon as it holds it in registers, so QK^T of
// chunk j+1 runs while it computes the exponentials of chunk j; the running
// max is lazily updated (O is rescaled in TMEM only when a row max grows by
// more than 2^8).  Half of the exponentials are
// computed on the FMA pipe (2^x = 2^rint(x) * cubic(x - rint(x))) so that the
// special-function unit, which otherwise needs as many cycles per chunk as
// the tensor core, stops being the bound.
// P is double-buffered in tensor memory: the softmax of chunk j + 1 writes
// its P while the PV of chunk j still reads the other buffer, so it waits
// only for the PV two chunks back (and for the previous one when O has to be
// rescaled).
// Warp roles: warp 0 issues TMA (each half of the Q tile once per unit, K/V
// per chunk into a 3-stage ring), warp 1 allocates TMEM, one thread of warp
// 1 issues the MMAs of half 0 and one thread of warp 2 those of half 1 (in
// the order QK(j+1) PV(j) per chunk j, so that neither half's chain waits
// on the other's softmax), warps 4-7 and 8-11 are the softmax/epilogue
// warpgroups of half 0 and half 1 (a warpgroup's warp w may touch TMEM
// lanes 32*(w%4)..+31, so the four warps cover the 128 rows).
// Every wait is a bounded mbarrier wait; the grid is persistent (one CTA per
// SM, the whole 512-column TMEM), heaviest tiles first.
#include <algorithm>

#include "internal.h"
#include "tcgen05.cuh"

namespace csa {
namespace {

constexpr int kPfThreads = 384;
constexpr int kNS = 3;                         // K/V stages
constexpr int kQHalfBytes = 128 * 128 * 2;     // 32 KB: one 128-row half of the Q tile
constexpr int kKVBytes = 64 * 128 * 2;         // 16 KB per K (or V) chunk
constexpr int kStageBytes = 2 * kKVBytes;
constexpr int kQOff = 0;
constexpr int kKVOff = 2 * kQHalfBytes;
constexpr int kOStageBytes = 32768;            // per half: all 128 output columns of its 128 rows
constexpr int kOOff = kKVOff + kNS * kStageBytes;
constexpr int kBarOff = kOOff + 2 * kOStageBytes;
constexpr int kSmemBytes = 1024 + kBarOff + 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kEmuPeriod = 2;  // one pair of exponentials in kEmuPeriod on the FMA pipe

// TMEM columns: S of half h at 64 h, P buffer u (bf16 pairs) of half h at
// 128 + 64 u + 32 h, O of half h at 256 + 128 h
constexpr uint32_t kColP = 128, kColO = 256;

// instruction descriptors: QK^T M = 128, N = 64 (both K-major); PV M = 128,
// N = 128 (V MN-major)
constexpr uint32_t kIdescQK = idesc_bf16(128, 64, 0);
constexpr uint32_t kIdescPV = idesc_bf16(128, 128, 1);

// Bulk tensor store of a [64 x 64] bf16 box from shared memory (128-byte
// swizzle) at (col, row) of the output map; completion tracked per thread
// by bulk groups.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// The shared-memory sources of this thread's stores have been read.
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// This thread's stores are complete.
__device__ __forceinline__ void bulk_wait0() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

struct PrefillParams {
  const int32_t* idx;
  const int32_t* count;
  int kmax;
  int B, S, Hq, Hkv, n_tiles, C;
  float scale_log2;
  __nv_bfloat16* O;
  DevErr err;
  int skip_empty;  // units with no chunk write nothing (else their rows get 0)
  // dense causal mode (no index lists): unit (b, h, t) holds chunks 0 .. t
  // when t * 64 < dense_k[b * Hkv + h], else none
  const int32_t* dense_k;
};

// Tiles that can hold work: all of them, or in dense causal mode those below
// the largest dense_k (the launch's units beyond it are never visited).
__device__ __forceinline__ int active_tiles(const PrefillParams& p) {
  if (p.dense_k == nullptr) return p.n_tiles;
  int mx = 0;
  for (int bh = 0; bh < p.B * p.Hkv; ++bh) mx = max(mx, __ldg(p.dense_k + bh));
  return min(p.n_tiles, (mx + 63) / 64);
}

// Unit w of T active tiles: heaviest (latest) tiles first.
__device__ __forceinline__ void unit_coords(const PrefillParams& p, int T, int w, int& b, int& h,
                                            int& t) {
  const int bh = p.B * p.Hkv;
  t = T - 1 - w / bh;
  const int r = w % bh;
  b = r / p.Hkv;
  h = r % p.Hkv;
}

__device__ __forceinline__ int unit_n(const PrefillParams& p, int sel_row) {
  if (p.dense_k != nullptr) {
    const int t = sel_row % p.n_tiles;
    return t * 64 < __ldg(p.dense_k + sel_row / p.n_tiles) ? t + 1 : 0;
  }
  int n = p.count[sel_row];
  if (n < 0 || n > p.kmax) {
    dev_flag(p.err, DEV_BAD_INDEX);
    n = max(0, min(n, p.kmax));
  }
  return n;
}

__device__ __forceinline__ int unit_chunk(const PrefillParams& p, int sel_row, int j) {
  if (p.dense_k != nullptr) return j;
  int c = p.idx[static_cast<int64_t>(sel_row) * p.kmax + j];
  if (c < 0 || c >= p.C) {
    dev_flag(p.err, DEV_BAD_INDEX);
    c = 0;
  }
  return c;
}

__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t sQ = sb + kQOff;
  const uint32_t sKV = sb + kKVOff;
  const uint32_t bar = sb + kBarOff;
  const uint32_t q_full = bar, q_empty = bar + 16;          // [2] each
  const uint32_t kv_full = bar + 32, kv_empty = kv_full + 8 * kNS;
  const uint32_t s_full = kv_empty + 8 * kNS;               // [2]
  const uint32_t s_free = s_full + 16;                      // [2]
  const uint32_t p_full = s_free + 16;                      // [2 halves][2 P buffers]
  const uint32_t pv_done = p_full + 32;                     // [2][2]
  const uint32_t drain = pv_done + 32;                      // [2]
  const uint32_t o_full = drain + 16;                       // [2] a half's staged O columns
  const uint32_t o_free = o_full + 16;                      // [2] ... have been read by the store
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + (o_free + 16 - bar));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int h = 0; h < 2; ++h) {
      mbar_init(q_full + 8 * h, 1);
      mbar_init(q_empty + 8 * h, 1);
      mbar_init(s_full + 8 * h, 1);
      mbar_init(s_free + 8 * h, 128);
      for (int u = 0; u < 2; ++u) {
        mbar_init(p_full + 8 * (2 * h + u), 128);
        mbar_init(pv_done + 8 * (2 * h + u), 1);
      }
    }
    for (int s = 0; s < kNS; ++s) {
      mbar_init(kv_full + 8 * s, 1);
      mbar_init(kv_empty + 8 * s, 2);  // released by both halves' MMA issuers
    }
    mbar_init(drain, 1);
    mbar_init(drain + 8, 1);
    for (int h = 0; h < 2; ++h) {
      mbar_init(o_full + 8 * h, 128);
      mbar_init(o_free + 8 * h, 1);
    }
    fence_barrier_init();
  }
  __shared__ int tiles_sh;
  if (warp == 1) {
    tmem_alloc<512>(tmem_slot);
  }
  if (threadIdx.x == 64) tiles_sh = active_tiles(p);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int T = tiles_sh;
  const int n_units = p.B * p.Hkv * T;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    uint32_t q_phase[2] = {0, 0}, kv_it = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < n_units && ok; w += gridDim.x) {
      int b, h, t;
      unit_coords(p, T, w, b, h, t);
      const int sel = (b * p.Hkv + h) * p.n_tiles + t;
      const int n = unit_n(p, sel);
      if (n == 0) continue;
      if (lane == 0) {
        const int qrow = b * p.S + t * 64;
        for (int hf = 0; hf < 2 && ok; ++hf) {
          // a half is free once the last QK^T of the previous unit that reads it is done
          if (!mbar_wait(q_empty + 8 * hf, q_phase[hf] ^ 1u, p.err)) ok = false;
          q_phase[hf] ^= 1u;
          if (!ok) break;
          const uint32_t fb = q_full + 8 * hf;
          mbar_arrive_expect_tx(fb, kQHalfBytes);
          for (int gg = 0; gg < 2; ++gg)
            for (int dbx = 0; dbx < 2; ++dbx)
              tma_load_2d(sQ + hf * kQHalfBytes + dbx * 16384 + gg * 8192, &tmQ,
                          (h * 4 + 2 * hf + gg) * 128 + dbx * 64, qrow, fb);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      for (int j0 = 0; j0 < n && ok; j0 += 32) {
        const int myc = j0 + lane < n ? unit_chunk(p, sel, j0 + lane) : 0;
        const int nb = min(32, n - j0);
        for (int j = 0; j < nb; ++j) {
          const int c = __shfl_sync(0xffffffffu, myc, j);
          int good = 1;
          if (lane == 0) {
            const int s = kv_it % kNS;
            if (!mbar_wait(kv_empty + 8 * s, ((kv_it / kNS) & 1u) ^ 1u, p.err)) {
              good = 0;
            } else {
              const uint32_t fb = kv_full + 8 * s;
              mbar_arrive_expect_tx(fb, kStageBytes);
              const int krow = (b * p.Hkv + h) * p.S + c * 64;
              const uint32_t dst = sKV + s * kStageBytes;
              tma_load_2d(dst, &tmK, 0, krow, fb);
              tma_load_2d(dst + 8192, &tmK, 64, krow, fb);
              tma_load_2d(dst + kKVBytes, &tmV, 0, krow, fb);
              tma_load_2d(dst + kKVBytes + 8192, &tmV, 64, krow, fb);
            }
          }
          ++kv_it;
          good = __shfl_sync(0xffffffffu, good, 0);
          if (!good) {
            ok = false;
            break;
          }
        }
      }
    }
    // let every copy in flight land before the CTA retires
    if (lane == 0) {
      const uint32_t first = kv_it > kNS ? kv_it - kNS : 0u;
      for (uint32_t i = first; i < kv_it; ++i)
        mbar_wait(kv_full + 8 * (i % kNS), (i / kNS) & 1u, p.err);
    }
  } else if (warp == 1 || warp == 2) {
    // ---------------------------------------------------------------- MMA issuers
    // One thread per 128-row half (warp 1: half 0, warp 2: half 1), so each
    // half's QK^T -> softmax -> PV chain runs at its own pace.
    const int hf = warp - 1;
    if (lane == 0) {
      uint32_t q_phase = 0, s_cnt = 0, kv_it = 0;
      bool ok = true;
      const uint32_t qa = sQ + hf * kQHalfBytes;
      // S of this half is overwritten only after the softmax has loaded the
      // previous S (s_free), so QK^T of chunk j+1 runs during its exponentials
      auto qk = [&](uint32_t stage) -> bool {
        if (s_cnt > 0 && !mbar_wait(s_free + 8 * hf, (s_cnt - 1) & 1u, p.err)) return false;
        tc_fence_after();
        const uint32_t d = tmem + hf * 64;
        const uint32_t kb = sKV + stage * kStageBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off_q = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t off_k = (kk >> 2) * 8192 + (kk & 3) * 32;
          umma_ss(d, smem_desc(qa + off_q, 16, 1024), smem_desc(kb + off_k, 16, 1024), kIdescQK,
                  kk > 0 ? 1u : 0u);
        }
        umma_commit(s_full + 8 * hf);
        ++s_cnt;
        return true;
      };
      // PV of this half's chunk k (kv_it) reads P buffer k & 1 and signals
      // pv_done[hf][k & 1]
      auto pv = [&](uint32_t stage, bool acc, uint32_t k) {
        const uint32_t d = tmem + kColO + hf * 128;
        const uint32_t pa = tmem + kColP + (k & 1u) * 64 + hf * 32;
        const uint32_t vb = sKV + stage * kStageBytes + kKVBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ts(d, pa + kk * 8, smem_desc(vb + kk * 2048, 8192, 1024), kIdescPV,
                  (acc || kk > 0) ? 1u : 0u);
        umma_commit(pv_done + 8 * (2 * hf + (k & 1u)));
      };
      for (int w = blockIdx.x; w < n_units && ok; w += gridDim.x) {
        int b, h, t;
        unit_coords(p, T, w, b, h, t);
        const int n = unit_n(p, (b * p.Hkv + h) * p.n_tiles + t);
        if (n == 0) continue;
        const uint32_t st0 = kv_it % kNS;
        if (!mbar_wait(kv_full + 8 * st0, (kv_it / kNS) & 1u, p.err)) break;
        if (!mbar_wait(q_full + 8 * hf, q_phase, p.err)) break;
        q_phase ^= 1u;
        if (!qk(st0)) break;
        if (n == 1) umma_commit(q_empty + 8 * hf);
        for (int j = 0; j < n; ++j) {
          const uint32_t cur = kv_it % kNS, nxt = (kv_it + 1) % kNS;
          if (j + 1 < n) {
            if (!mbar_wait(kv_full + 8 * nxt, ((kv_it + 1) / kNS) & 1u, p.err)) { ok = false; break; }
            if (!qk(nxt)) { ok = false; break; }
            if (j + 2 == n) umma_commit(q_empty + 8 * hf);
          }
          // P of chunk j written (its buffer's (kv_it / 2)-th fill)
          if (!mbar_wait(p_full + 8 * (2 * hf + (kv_it & 1u)), (kv_it >> 1) & 1u, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          pv(cur, j > 0, kv_it);
          umma_commit(kv_empty + 8 * cur);  // the stage is free once both halves' reads are done
          ++kv_it;
        }
      }
      // every MMA this thread issued has finished before TMEM is released
      umma_commit(drain + 8 * hf);
      mbar_wait(drain + 8 * hf, 0u, p.err);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- softmax + epilogue
    const int half = (warp - 4) >> 2;
    const int r = ((warp & 3) << 5) + lane;  // row within the half == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + half * 64;
    const uint32_t tP = tmem + lane_base + kColP + half * 32;  // + 64 per buffer
    const uint32_t tO = tmem + lane_base + kColO + half * 128;
    const int g = half * 2 + (r >> 6);  // query head within the group
    const int i = r & 63;               // row within the tile
    const float sl = p.scale_log2;
    uint32_t s_cnt = 0, o_cnt = 0;  // s_cnt: this half's chunks so far (chunk k has PV k)
    int64_t pv_seen = -1;            // the latest PV known complete (all earlier ones too)
    bool ok = true;
    // Wait until PV k is complete: the (k / 2)-th completion of pv_done[half][k & 1];
    // waits come in increasing k, and PV k + 2 needs a P written after this wait
    auto wait_pv = [&](int64_t k) -> bool {
      if (k <= pv_seen) return true;
      if (!warp_wait(pv_done + 8 * (2 * half + static_cast<int>(k & 1)),
                     static_cast<uint32_t>(k >> 1) & 1u, p.err))
        return false;
      pv_seen = k;
      tc_fence_after();
      return true;
    };
    for (int w = blockIdx.x; w < n_units && ok; w += gridDim.x) {
      int b, h, t;
      unit_coords(p, T, w, b, h, t);
      const int sel = (b * p.Hkv + h) * p.n_tiles + t;
      const int n = unit_n(p, sel);
      const int qpos = t * 64 + i;
      __nv_bfloat16* orow = p.O + ((static_cast<int64_t>(b) * p.S + qpos) * p.Hq + h * 4 + g) * 128;
      if (n == 0) {
        if (!p.skip_empty)
          for (int c = 0; c < 128; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
        continue;
      }
      float m = -INFINITY, l = 0.f;  // running max of the raw scores, sum of 2^((s - m) sl)
      int c_next = unit_chunk(p, sel, 0);
      for (int j = 0; j < n; ++j) {
        const int c = c_next;
        if (j + 1 < n) c_next = unit_chunk(p, sel, j + 1);
        const uint32_t sph = s_cnt & 1u;
        const int64_t kc = s_cnt;  // this chunk's index: P buffer kc & 1, PV kc
        ++s_cnt;
        // wait results are made warp-uniform: the TMEM accesses below are
        // warp-collective
        if (!warp_wait(s_full + 8 * half, sph, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[2][32];
        tmem_ld32(tS, sr[0]);
        tmem_ld32(tS + 32, sr[1]);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(s_free + 8 * half);  // S is in registers: QK^T of the next chunk may overwrite it
        float x[64];
#pragma unroll
        for (int jj = 0; jj < 64; ++jj) x[jj] = __uint_as_float(sr[jj >> 5][jj & 31]);
        // only a chunk reaching past the tile's first row needs the causal mask
        const bool masked = c * 64 + 63 > t * 64;
        if (masked) {
          const int lim = qpos - c * 64;  // keys jj <= lim are visible
#pragma unroll
          for (int jj = 0; jj < 64; ++jj) x[jj] = jj <= lim ? x[jj] : -INFINITY;
        }
        float mq[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          float v = fmax3(x[16 * a], x[16 * a + 1], x[16 * a + 2]);
#pragma unroll
          for (int k = 3; k < 15; k += 2) v = fmax3(v, x[16 * a + k], x[16 * a + k + 1]);
          mq[a] = fmaxf(v, x[16 * a + 15]);
        }
        const float mnew = fmaxf(fmax3(mq[0], mq[1], mq[2]), fmaxf(mq[3], m));
        // this chunk's P buffer is free once the PV two chunks back is done
        if (!wait_pv(kc - 2)) {
          ok = false;
          break;
        }
        // Lazy rescale: a row moves its max only when it grew by more than
        // 2^8.  tcgen05.ld/st are warp-collective, so the warp rescales
        // together when any of its rows needs it (the others by 1).
        const bool grow = m != -INFINITY && (mnew - m) * sl > kRescaleLog2;
        float alpha = 1.f;
        if (grow) {
          alpha = fast_exp2((m - mnew) * sl);
          l *= alpha;
          m = mnew;
        }
        if (m == -INFINITY) m = mnew;  // first visible keys: nothing accumulated in O yet
        if (__any_sync(0xffffffffu, grow)) {
          // O is rescaled in place: every PV issued so far has to be done
          if (!wait_pv(kc - 1)) {
            ok = false;
            break;
          }
#pragma unroll 1
          for (int cc = 0; cc < 128; cc += 32) {
            uint32_t ov[32];
            tmem_ld32(tO + cc, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st32(tO + cc, ov);
          }
          tmem_wait_st();
        }
        const float nm = m == -INFINITY ? 0.f : -m * sl;
        const float2 sl2 = make_float2(sl, sl), nm2 = make_float2(nm, nm);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
        uint32_t pk[32];
        if (!masked) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float2 xe = __ffma2_rn(make_float2(x[2 * e], x[2 * e + 1]), sl2, nm2);
            float2 pe;
            if (e % kEmuPeriod == kEmuPeriod - 1) {
              pe = exp2_fma2(xe);
            } else {
              pe.x = fast_exp2(xe.x);
              pe.y = fast_exp2(xe.y);
            }
            acc[e & 3] = __fadd2_rn(acc[e & 3], pe);
            pk[e] = pack_bf16x2(pe.x, pe.y);
          }
        } else {  // masked keys must give exactly 0: special-function unit only
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float2 xe = __ffma2_rn(make_float2(x[2 * e], x[2 * e + 1]), sl2, nm2);
            const float2 pe = make_float2(fast_exp2(xe.x), fast_exp2(xe.y));
            acc[e & 3] = __fadd2_rn(acc[e & 3], pe);
            pk[e] = pack_bf16x2(pe.x, pe.y);
          }
        }
        l += (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y) + (acc[2].x + acc[2].y) +
             (acc[3].x + acc[3].y);
        // P row r (bf16 pairs), the A operand of this half's PV
        tmem_st32(tP + static_cast<uint32_t>(kc & 1) * 64, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full + 8 * (2 * half + static_cast<int>(kc & 1)));
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 rows, once the unit's last PV is done
      if (!wait_pv(static_cast<int64_t>(s_cnt) - 1)) {
        ok = false;
        break;
      }
      const float inv = l > 0.f ? 1.0f / l : 0.f;
      // O / l as bf16 into this half's staging area, laid out as the output
      // map's [64 x 64] boxes (128-byte swizzle), kOStageBytes / 256 columns
      // per round; one thread then writes the boxes with bulk tensor stores.
      constexpr int CW = kOStageBytes / 256, NBX = CW / 64;
      const uint32_t so = sb + kOOff + half * kOStageBytes;
      const uint32_t srow = so + (r >> 6) * NBX * 8192 + i * 128;
#pragma unroll 1
      for (int cc = 0; cc < 128; cc += CW) {
        uint32_t pk[CW / 2];
#pragma unroll
        for (int c0 = 0; c0 < CW; c0 += 64) {
          uint32_t ov[2][32];
          tmem_ld32(tO + cc + c0, ov[0]);
          tmem_ld32(tO + cc + c0 + 32, ov[1]);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e)
            pk[c0 / 2 + e] = pack_bf16x2(__uint_as_float(ov[e >> 4][2 * (e & 15)]) * inv,
                                         __uint_as_float(ov[e >> 4][2 * (e & 15) + 1]) * inv);
        }
        // the area is free once the bulk store of the previous round has read it
        if (o_cnt > 0) {
          if (r == 0) {
            bulk_wait_read0();
            mbar_arrive(o_free + 8 * half);
          }
          __syncwarp();
          if (!warp_wait(o_free + 8 * half, (o_cnt - 1) & 1u, p.err)) {
            ok = false;
            break;
          }
        }
#pragma unroll
        for (int j = 0; j < CW / 8; ++j) {
          const uint32_t dst = srow + (j >> 3) * 8192 + (((j & 7) ^ (i & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(pk[4 * j]),
                       "r"(pk[4 * j + 1]), "r"(pk[4 * j + 2]), "r"(pk[4 * j + 3])
                       : "memory");
        }
        fence_proxy_async_smem();  // the writes, for the bulk store
        mbar_arrive(o_full + 8 * half);
        if (r == 0) {
          if (mbar_wait(o_full + 8 * half, o_cnt & 1u, p.err)) {
            const int orow0 = b * p.S + t * 64;
#pragma unroll
            for (int gq = 0; gq < 2; ++gq)
#pragma unroll
              for (int bx = 0; bx < NBX; ++bx)
                tma_store_2d(&tmO, so + (gq * NBX + bx) * 8192,
                             (h * 4 + half * 2 + gq) * 128 + cc + bx * 64, orow0);
            bulk_commit();
          } else {
            ok = false;
          }
        }
        __syncwarp();
        ++o_cnt;
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
      }
      if (!ok) break;
      // the next unit's first PV overwrites O: it is issued after this
      // warpgroup's next p_full arrival, which follows these loads
      tc_fence_before();
    }
    if (r == 0) bulk_wait0();  // the last bulk stores are complete before the CTA retires
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1)
    tmem_dealloc<512>(tmem);
}

}  // namespace

cudaError_t launch_prefill(const Launch& l, const void* Q, const void* K, const void* V,
                           const int32_t* idx, const int32_t* count, int kmax, int B, int S,
                           int Hq, int Hkv, int D, int tile_m, int L, float scale, void* O,
                           std::string* why, bool skip_empty, const int32_t* dense_k) {
  (void)D;
  (void)tile_m;
  (void)L;
  CUtensorMap tmQ, tmK, tmV, tmO;
  if (!make_tmap_bf16_2d(&tmO, O, static_cast<uint64_t>(B) * S, static_cast<uint64_t>(Hq) * 128,
                         static_cast<uint64_t>(Hq) * 128, 64, 64, why))
    return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tmQ, Q, static_cast<uint64_t>(B) * S, static_cast<uint64_t>(Hq) * 128,
                         static_cast<uint64_t>(Hq) * 128, 64, 64, why))
    return cudaErrorInvalidValue;
  const uint64_t kv_rows = static_cast<uint64_t>(B) * Hkv * S;
  if (!make_tmap_bf16_2d(&tmK, K, kv_rows, 128, 128, 64, 64, why)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tmV, V, kv_rows, 128, 128, 64, 64, why)) return cudaErrorInvalidValue;
  PrefillParams p{};
  p.idx = idx;
  p.count = count;
  p.kmax = kmax;
  p.B = B;
  p.S = S;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.n_tiles = S / 64;
  p.C = S / 64;
  p.scale_log2 = scale * kLog2e;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.err = l.err;
  p.skip_empty = skip_empty ? 1 : 0;
  p.dense_k = dense_k;
  const int n_units = B * Hkv * p.n_tiles;
  if (n_units == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
  if (e != cudaSuccess) return e;
  const int grid = std::min(n_units, l.num_sms);
  prefill_kernel<<<grid, kPfThreads, kSmemBytes, l.stream>>>(tmQ, tmK, tmV, tmO, p);
  return cudaGetLastError();
}

}  // namespace csa
