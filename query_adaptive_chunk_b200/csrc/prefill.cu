// Block-sparse causal prefill on the 5th-generation tensor cores (tcgen05,
// accumulators in tensor memory).
//
// Work unit = (sequence b, KV head h, query tile t): the 64 query rows of
// the tile for each of the G = 4 query heads of the group, stacked into 256
// rows (head-major) that share the tile's chunk list.  The 256 rows are two
// 128-row halves, each an M = 128 MMA operand.  Per selected chunk (64 keys):
//   S_half = Q_half K^T      tcgen05.mma M=128 N=64 K=128, A/B from shared memory
//   P_half = softmax rows    two warpgroups (one per half) read S from TMEM with
//                            tcgen05.ld, keep the running max/sum per row, write
//                            P back to TMEM as packed bf16
//   O_half += P_half V       tcgen05.mma M=128 N=128 K=64, A = P from TMEM,
//                            B = V from shared memory (MN-major)
// The running max is lazily updated: O is rescaled (tcgen05.ld/st by the
// owning softmax thread) only when a row max grows by more than 2^8.
// Warp roles: warp 0 issues TMA (Q tile once per unit, K/V per chunk into a
// 4-stage ring), warp 1 allocates TMEM and one of its threads issues every MMA
// and tcgen05.commit, warps 4-7 and 8-11 are the softmax/epilogue warpgroups
// of half 0 and half 1 (a warpgroup's warp w may touch TMEM lanes
// 32*(w%4)..+31, so the four warps cover the 128 rows).  MMA order
//   QK0(0) QK1(0) | PV0(j) QK0(j+1) PV1(j) QK1(j+1) | ...
// lets one half's softmax run while the tensor core works on the other half.
// A commit tracks every earlier MMA of the issuing thread, so "S_h(j+1) is
// ready" also means "PV_h(j) has finished": the softmax may then overwrite P_h
// and rescale O_h without a separate wait.
// Every wait is a bounded mbarrier wait; the grid is persistent (one CTA per
// SM, the whole 512-column TMEM), heaviest tiles first.
#include <algorithm>

#include "internal.h"

namespace csa {
namespace {

constexpr int kPfThreads = 384;
constexpr int kNS = 4;                         // K/V stages
constexpr int kQBytes = 256 * 128 * 2;         // 64 KB Q tile
constexpr int kKVBytes = 64 * 128 * 2;         // 16 KB per K (or V) chunk
constexpr int kStageBytes = 2 * kKVBytes;
constexpr int kQOff = 0;
constexpr int kKVOff = kQBytes;
constexpr int kBarOff = kKVOff + kNS * kStageBytes;
constexpr int kSmemBytes = 1024 + kBarOff + 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;

// TMEM columns
constexpr uint32_t kColS0 = 0, kColS1 = 64, kColP0 = 128, kColP1 = 160, kColO0 = 256,
                   kColO1 = 384;

// instruction descriptors (kind::f16): D fp32, A/B bf16, M = 128
constexpr uint32_t kIdescQK = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (0u << 16) |
                              ((64u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) |
                              ((128u >> 3) << 17) | ((128u >> 4) << 24);

// shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((addr & 0x3ffffu) >> 4) |
         (static_cast<uint64_t>(lbo >> 4) << 16) | (static_cast<uint64_t>(sbo >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void umma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void umma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                        uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

#define CSA_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), \
                  "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define CSA_W8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), "r"(r[i + 4]), \
                  "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])

// 32 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : CSA_R8(0), CSA_R8(8), CSA_R8(16), CSA_R8(24)
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      CSA_W8(0), CSA_W8(8), CSA_W8(16), CSA_W8(24)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

struct PrefillParams {
  const int32_t* idx;
  const int32_t* count;
  int kmax;
  int B, S, Hq, Hkv, n_tiles, C;
  float scale_log2;
  __nv_bfloat16* O;
  DevErr err;
};

__device__ __forceinline__ void unit_coords(const PrefillParams& p, int w, int& b, int& h, int& t) {
  const int bh = p.B * p.Hkv;
  t = p.n_tiles - 1 - w / bh;  // heaviest (latest) tiles first
  const int r = w % bh;
  b = r / p.Hkv;
  h = r % p.Hkv;
}

__device__ __forceinline__ int unit_n(const PrefillParams& p, int sel_row) {
  int n = p.count[sel_row];
  if (n < 0 || n > p.kmax) {
    dev_flag(p.err, DEV_BAD_INDEX);
    n = max(0, min(n, p.kmax));
  }
  return n;
}

__device__ __forceinline__ int unit_chunk(const PrefillParams& p, int sel_row, int j) {
  int c = p.idx[static_cast<int64_t>(sel_row) * p.kmax + j];
  if (c < 0 || c >= p.C) {
    dev_flag(p.err, DEV_BAD_INDEX);
    c = 0;
  }
  return c;
}

__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t sQ = sb + kQOff;
  const uint32_t sKV = sb + kKVOff;
  const uint32_t bar = sb + kBarOff;
  const uint32_t q_full = bar, q_empty = bar + 8;
  const uint32_t kv_full = bar + 16, kv_empty = kv_full + 8 * kNS;
  const uint32_t s_full = kv_empty + 8 * kNS;  // [2]
  const uint32_t p_full = s_full + 16;         // [2]
  const uint32_t o_full = p_full + 16;         // [2]
  const uint32_t o_empty = o_full + 16;        // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + 8 * (2 + 2 * kNS + 8));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kNS; ++s) {
      mbar_init(kv_full + 8 * s, 1);
      mbar_init(kv_empty + 8 * s, 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(s_full + 8 * h, 1);
      mbar_init(p_full + 8 * h, 128);
      mbar_init(o_full + 8 * h, 1);
      mbar_init(o_empty + 8 * h, 128);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_units = p.B * p.Hkv * p.n_tiles;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    uint32_t q_phase = 0, kv_it = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < n_units && ok; w += gridDim.x) {
      int b, h, t;
      unit_coords(p, w, b, h, t);
      const int sel = (b * p.Hkv + h) * p.n_tiles + t;
      const int n = unit_n(p, sel);
      if (n == 0) continue;
      if (lane == 0) {
        if (!mbar_wait(q_empty, q_phase ^ 1u, p.err)) ok = false;
        q_phase ^= 1u;
        if (ok) {
          mbar_arrive_expect_tx(q_full, kQBytes);
          const int qrow = b * p.S + t * 64;
          for (int g = 0; g < 4; ++g)
            for (int dbx = 0; dbx < 2; ++dbx)
              tma_load_2d(sQ + (g >> 1) * 32768 + dbx * 16384 + (g & 1) * 8192, &tmQ,
                          (h * 4 + g) * 128 + dbx * 64, qrow, q_full);
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
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t q_phase = 0, kv_it = 0;
      uint32_t p_phase[2] = {0, 0}, oe_phase[2] = {0, 0};
      bool ok = true;
      auto qk = [&](int half, uint32_t stage) {
        const uint32_t d = tmem + (half ? kColS1 : kColS0);
        const uint32_t qa = sQ + half * 32768;
        const uint32_t kb = sKV + stage * kStageBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off_q = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t off_k = (kk >> 2) * 8192 + (kk & 3) * 32;
          umma_ss(d, smem_desc(qa + off_q, 16, 1024), smem_desc(kb + off_k, 16, 1024), kIdescQK,
                  kk > 0 ? 1u : 0u);
        }
      };
      auto pv = [&](int half, uint32_t stage, bool acc) {
        const uint32_t d = tmem + (half ? kColO1 : kColO0);
        const uint32_t a = tmem + (half ? kColP1 : kColP0);
        const uint32_t vb = sKV + stage * kStageBytes + kKVBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ts(d, a + kk * 8, smem_desc(vb + kk * 2048, 8192, 1024), kIdescPV,
                  (acc || kk > 0) ? 1u : 0u);
      };
      for (int w = blockIdx.x; w < n_units && ok; w += gridDim.x) {
        int b, h, t;
        unit_coords(p, w, b, h, t);
        const int n = unit_n(p, (b * p.Hkv + h) * p.n_tiles + t);
        if (n == 0) continue;
        if (!mbar_wait(q_full, q_phase, p.err)) break;
        q_phase ^= 1u;
        uint32_t st = kv_it % kNS;
        if (!mbar_wait(kv_full + 8 * st, (kv_it / kNS) & 1u, p.err)) break;
        tc_fence_after();
        qk(0, st);
        umma_commit(s_full);
        qk(1, st);
        umma_commit(s_full + 8);
        for (int j = 0; j < n; ++j) {
          const uint32_t cur = kv_it % kNS;
          const bool last = j + 1 == n;
          // half 0
          if (!mbar_wait(p_full, p_phase[0], p.err)) { ok = false; break; }
          p_phase[0] ^= 1u;
          if (j == 0) {
            if (!mbar_wait(o_empty, oe_phase[0] ^ 1u, p.err)) { ok = false; break; }
            oe_phase[0] ^= 1u;
          }
          tc_fence_after();
          pv(0, cur, j > 0);
          if (last) umma_commit(o_full);
          uint32_t nxt = (kv_it + 1) % kNS;
          if (!last) {
            if (!mbar_wait(kv_full + 8 * nxt, ((kv_it + 1) / kNS) & 1u, p.err)) { ok = false; break; }
            tc_fence_after();
            qk(0, nxt);
            umma_commit(s_full);
          }
          // half 1
          if (!mbar_wait(p_full + 8, p_phase[1], p.err)) { ok = false; break; }
          p_phase[1] ^= 1u;
          if (j == 0) {
            if (!mbar_wait(o_empty + 8, oe_phase[1] ^ 1u, p.err)) { ok = false; break; }
            oe_phase[1] ^= 1u;
          }
          tc_fence_after();
          pv(1, cur, j > 0);
          umma_commit(kv_empty + 8 * cur);
          if (last) {
            umma_commit(o_full + 8);
            umma_commit(q_empty);
          } else {
            qk(1, nxt);
            umma_commit(s_full + 8);
          }
          ++kv_it;
        }
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- softmax + epilogue
    const int half = (warp - 4) >> 2;
    const int r = ((warp & 3) << 5) + lane;  // row within the half == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + (half ? kColS1 : kColS0);
    const uint32_t tP = tmem + lane_base + (half ? kColP1 : kColP0);
    const uint32_t tO = tmem + lane_base + (half ? kColO1 : kColO0);
    const uint32_t my_s_full = s_full + 8 * half, my_p_full = p_full + 8 * half;
    const uint32_t my_o_full = o_full + 8 * half, my_o_empty = o_empty + 8 * half;
    const int g = half * 2 + (r >> 6);  // query head within the group
    const int i = r & 63;               // row within the tile
    uint32_t s_phase = 0, of_phase = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < n_units && ok; w += gridDim.x) {
      int b, h, t;
      unit_coords(p, w, b, h, t);
      const int sel = (b * p.Hkv + h) * p.n_tiles + t;
      const int n = unit_n(p, sel);
      const int qpos = t * 64 + i;
      __nv_bfloat16* orow = p.O + ((static_cast<int64_t>(b) * p.S + qpos) * p.Hq + h * 4 + g) * 128;
      if (n == 0) {
        for (int c = 0; c < 128; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
        continue;
      }
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < n; ++j) {
        const int c = unit_chunk(p, sel, j);
        if (!mbar_wait(my_s_full, s_phase, p.err)) { ok = false; break; }
        s_phase ^= 1u;
        tc_fence_after();
        uint32_t sr[2][32];
        tmem_ld32(tS, sr[0]);
        tmem_ld32(tS + 32, sr[1]);
        tmem_wait_ld();
        const int lim = qpos - c * 64;  // keys jj <= lim are visible
        float x[64];
        float rmax = -INFINITY;
#pragma unroll
        for (int jj = 0; jj < 64; ++jj) {
          const float v = __uint_as_float(sr[jj >> 5][jj & 31]) * p.scale_log2;
          x[jj] = jj <= lim ? v : -INFINITY;
          rmax = fmaxf(rmax, x[jj]);
        }
        float mnew = fmaxf(m, rmax);
        if (m == -INFINITY) {
          m = mnew;  // first visible keys: nothing accumulated in O yet
        } else if (mnew > m + kRescaleLog2) {
          const float alpha = fast_exp2(m - mnew);
          l *= alpha;
          m = mnew;
#pragma unroll 1
          for (int cc = 0; cc < 128; cc += 32) {
            uint32_t ov[32];
            tmem_ld32(tO + cc, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st32(tO + cc, ov);
          }
        }
        const float mu = m == -INFINITY ? 0.f : m;
        uint32_t pk[32];
        float ls = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float p0 = fast_exp2(x[2 * e] - mu), p1 = fast_exp2(x[2 * e + 1] - mu);
          ls += p0 + p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        l += ls;
        tmem_st32(tP, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(my_p_full);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 rows
      if (!mbar_wait(my_o_full, of_phase, p.err)) { ok = false; break; }
      of_phase ^= 1u;
      tc_fence_after();
      const float inv = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll 1
      for (int cc = 0; cc < 128; cc += 32) {
        uint32_t ov[32];
        tmem_ld32(tO + cc, ov);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * inv, __uint_as_float(ov[2 * e + 1]) * inv);
        uint4* dst = reinterpret_cast<uint4*>(orow + cc);
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
      }
      tc_fence_before();
      mbar_arrive(my_o_empty);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
}

}  // namespace

cudaError_t launch_prefill(const Launch& l, const void* Q, const void* K, const void* V,
                           const int32_t* idx, const int32_t* count, int kmax, int B, int S,
                           int Hq, int Hkv, int D, int tile_m, int L, float scale, void* O,
                           std::string* why) {
  (void)D;
  (void)tile_m;
  (void)L;
  CUtensorMap tmQ, tmK, tmV;
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
  const int n_units = B * Hkv * p.n_tiles;
  if (n_units == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
  if (e != cudaSuccess) return e;
  const int grid = std::min(n_units, l.num_sms);
  prefill_kernel<<<grid, kPfThreads, kSmemBytes, l.stream>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace csa
