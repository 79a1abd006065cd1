// Sparse split-K decode over the gathered raw KV of the selected chunks, and
// the log-sum-exp merge of its partials.
//
// bf16 path (the hot one).  A persistent grid of P CTAs, one per SM.  The
// units' chunk lists are laid end to end and cut into P equal pieces, so
// every CTA streams the same number of chunks whatever mix of full-attention
// heads (all chunks) and sparse heads (a few hundred) the step holds.
//   * warp 4 (producer): resolves chunk ids 32 at a time (one lane each) and
//     issues, per chunk, 2-D TMA loads of the chunk's K and V rows
//     ([L x 64] boxes, 128-byte swizzle) into a ring of stages that fills
//     ~192 KB of shared memory (3 stages of 64 KB at L = 128, D = 128), i.e.
//     enough bytes in flight per SM to cover HBM latency.  With the first
//     chunk of each unit it also copies the unit's query rows into the
//     stage's q slot, on the same barrier.
//   * warps 0-3 (consumers): each takes L/4 tokens of every chunk.  S^T =
//     K q^T runs on the tensor cores as mma.m16n8k16 with the tokens as M and
//     the query heads of the GQA group as N (up to 8); the online softmax
//     stays in registers (per-head running max/sum); P is moved into the B
//     layout with movmatrix and O^T += V^T P^T runs as a second mma.  The
//     math per 64 KB chunk is a few hundred warp instructions, so the SM
//     stays bound by the copy engine, not by issue.  At a unit boundary each
//     warp drops its (m, l, O) into a flush buffer (two, double-buffered)
//     and streams on.
//   * warp 5 (epilogue): combines the four warps' partials of each unit into
//     one split partial (o normalised, lse), or the output when the unit has
//     a single split, and in merged mode counts the split in; the CTA that
//     brings a unit's last split merges it after its main loop, with the
//     partials staged through shared memory.
// Every wait is an mbarrier wait with a time limit; there is no named
// barrier, so a timeout anywhere makes the kernel wind down, never hang.
//
// fp32 path: a plain CUDA-core kernel with the same partition, used for fp32
// caches (parity workloads); it does the dot products in fp32.
#include <algorithm>

#include "internal.h"

namespace csa {
namespace {

constexpr int kConsumerWarps = 4;                    // warps 0-3
constexpr int kProducerWarp = kConsumerWarps;        // warp 4
constexpr int kEpilogueWarp = kConsumerWarps + 1;    // warp 5
constexpr int kDecodeThreads = (kConsumerWarps + 2) * 32;
constexpr int kStageBudget = 192 * 1024;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kDeferMax = 32;  // merges a CTA can postpone to the end of its work

// e^x and ln x on the special-function unit (ex2.approx / lg2.approx): the
// weights and lse of a merge need no more, and the short instruction
// sequences keep the end-of-launch merge code small.
__device__ __forceinline__ float sfu_exp(float x) { return fast_exp2(x * kLog2e); }
__device__ __forceinline__ float sfu_log(float x) { return __log2f(x) * kLn2; }

struct DecodeParams {
  const void* q;  // [B, Hq, D]
  const float* Kf;  // fp32 path only
  const float* Vf;
  const int32_t* idx;
  const int32_t* count;
  int kmax;
  const uint8_t* head_full;
  int U, Hkv, G, Hq, C, L, D;
  int64_t T;
  float scale_log2;
  int max_splits;
  float* o_part;
  float* lse_part;
  DevErr err;
  // merged variant: the last CTA of a unit combines its splits into out/lse_out
  int merged;
  int* counters;   // [U] arrivals, zero between calls
  void* out;       // [B, Hq, D] fp32 or bf16
  int out_bf16;
  float* lse_out;  // [B, Hq] or null
  // phased: full-head units first (no dependency on the selection), then,
  // after griddepcontrol.wait, the sparse units (launched with programmatic
  // dependent launch behind the selection kernel); pdl: that launch (the
  // cluster kernel has no phases but waits the same way)
  int phased;
  int pdl;
  // phased: the last `late` CTAs of the grid take no phase-1 work (they can
  // only start once the selection's CTAs have left their SMs)
  int late;
  // hybrid context (bf16 merged), over every chunk's gist row: every sparse
  // unit also attends over its gist rows, gist_rows (= C) per unit in
  // [B*Hkv*gist_rows, D] bf16 tensors, streamed as n_gist = ceil(gist_rows /
  // L) extra chunks after its selected ones (the last one ragged, its rows
  // past gist_rows masked); 0 = off
  int n_gist;
  int gist_rows;
  // hybrid context over the selected chunks' own gist rows: each sparse unit
  // with n selected chunks attends over their n gist rows (rows u*C + c of
  // Kg/Vg), gathered by the producer warp with 16-byte cp.async copies into
  // ceil(n / L) extra chunks after the selected ones; 0 = off
  int gist_sel;
  const __nv_bfloat16* Kg;
  const __nv_bfloat16* Vg;
};

// Unit sets of a phase: 0 = every unit, 1 = full-head units, 2 = sparse units.
__device__ __forceinline__ bool unit_in(const DecodeParams& p, int u, int mode) {
  if (mode == 0) return true;
  const bool full = p.head_full != nullptr && p.head_full[u % p.Hkv];
  return mode == 1 ? full : !full;
}

// Selected chunks of sparse unit u (its count, clamped to [0, kmax]).
__device__ __forceinline__ int sel_count(const DecodeParams& p, int u) {
  int n = p.count[u];
  if (n < 0 || n > p.kmax) {
    dev_flag(p.err, DEV_BAD_INDEX);
    n = max(0, min(n, p.kmax));
  }
  return n;
}

// Gist chunks and gist rows of a hybrid sparse unit with n selected chunks
// (both 0 without the hybrid context).
__device__ __forceinline__ int gist_chunks(const DecodeParams& p, int n) {
  return p.gist_sel ? (n + p.L - 1) / p.L : p.n_gist;
}
__device__ __forceinline__ int gist_rows_of(const DecodeParams& p, int n) {
  return p.gist_sel ? n : p.gist_rows;
}

__device__ __forceinline__ int unit_count(const DecodeParams& p, int u, int mode = 0) {
  const bool full = p.head_full != nullptr && p.head_full[u % p.Hkv];
  if (mode == 1) return full ? p.C : 0;
  if (full) return mode == 2 ? 0 : p.C;
  const int n = sel_count(p, u);
  return n + gist_chunks(p, n);  // a sparse unit's gist chunks come after its selected ones
}

__device__ __forceinline__ int unit_chunk(const DecodeParams& p, int u, int pos) {
  if (p.head_full != nullptr && p.head_full[u % p.Hkv]) return pos;
  int c = p.idx[static_cast<int64_t>(u) * p.kmax + pos];
  if (c < 0 || c >= p.C) {
    dev_flag(p.err, DEV_BAD_INDEX);
    c = 0;
  }
  return c;
}

// Row of the chunk at position pos of unit u: the raw K/V row of a selected
// (or, for a full unit, every) chunk, or for a hybrid unit's gist chunk j
// the first gist row, encoded as -(row + 1).  In the selected-gist scope a
// gist chunk has no contiguous rows: *gsel then gets the offset u*kmax + j*L
// of its first chunk id in idx (else -1).
__device__ __forceinline__ int unit_row(const DecodeParams& p, int u, int pos, int L, int* gsel) {
  *gsel = -1;
  if ((p.n_gist > 0 || p.gist_sel) && !(p.head_full != nullptr && p.head_full[u % p.Hkv])) {
    const int j = pos - sel_count(p, u);
    if (j >= 0) {
      if (p.gist_sel) {
        *gsel = u * p.kmax + j * L;
        return 0;
      }
      return -(u * p.gist_rows + j * L) - 1;
    }
  }
  const int c = unit_chunk(p, u, pos);
  return static_cast<int>(u * p.T + static_cast<int64_t>(c) * L);
}

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}

// The arrive-on of `bar` waits for this thread's earlier cp.async copies (the
// pending count goes up by one now and down by one when they land).
__device__ __forceinline__ void cp_async_mbar_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Selected-gist scope: the gist K and V rows of the chunk ids idx[off ..
// off + L) of unit u = off / kmax (those below the unit's count; the rest of
// the stage is zero-filled) into stage `dst`, laid out as the TMA boxes
// ([L x 64] per 64 columns, 128-byte swizzle).  All 32 lanes of the calling
// warp copy (lane r takes rows r, r + 32, ...) and arrive on `bar` through
// cp.async.mbarrier.arrive; the caller then makes the barrier's own arrival.
template <int D, int L>
__device__ __forceinline__ void gather_gist_rows(const DecodeParams& p, int off, uint32_t dst,
                                                 uint32_t bar) {
  constexpr int KV_BYTES = L * D * 2, BOX_BYTES = L * 128, PIECES = D / 8;
  const int lane = threadIdx.x & 31;
  const int u = off / p.kmax, r0 = off - u * p.kmax;
  const int n = sel_count(p, u);
#pragma unroll 1
  for (int r = lane; r < L; r += 32) {
    const bool valid = r0 + r < n;
    int c = valid ? p.idx[off + r] : 0;
    if (c < 0 || c >= p.C) {
      dev_flag(p.err, DEV_BAD_INDEX);
      c = 0;
    }
    const int64_t row = static_cast<int64_t>(u) * p.C + c;
    const __nv_bfloat16* ks = p.Kg + row * D;
    const __nv_bfloat16* vs = p.Vg + row * D;
    const uint32_t bytes = valid ? 16u : 0u;
#pragma unroll
    for (int pc = 0; pc < PIECES; ++pc) {
      const uint32_t o = (pc >> 3) * BOX_BYTES + r * 128 + (((pc & 7) ^ (r & 7)) << 4);
      cp_async_16(dst + o, ks + pc * 8, bytes);
      cp_async_16(dst + KV_BYTES + o, vs + pc * 8, bytes);
    }
  }
  cp_async_mbar_arrive(bar);
}

// prefix[0..U] of the effective chunk counts of a phase (all threads of the block).
__device__ void build_prefix(const DecodeParams& p, int* prefix, int* scan_sh, int mode = 0) {
  const int seg = (p.U + blockDim.x - 1) / blockDim.x;
  const int lo = min(p.U, static_cast<int>(threadIdx.x) * seg), hi = min(p.U, lo + seg);
  int loc = 0;
  for (int u = lo; u < hi; ++u) loc += unit_count(p, u, mode);
  int total = 0;
  int run = block_exclusive_scan(loc, scan_sh, &total);
  for (int u = lo; u < hi; ++u) {
    prefix[u] = run;
    run += unit_count(p, u, mode);
  }
  if (threadIdx.x == 0) prefix[p.U] = total;
  __syncthreads();
}

// The same by one warp (the producer), without a block barrier.
__device__ void warp_build_prefix(const DecodeParams& p, int* prefix, int mode) {
  const int lane = threadIdx.x & 31;
  const int seg = (p.U + 31) / 32;
  const int lo = min(p.U, lane * seg), hi = min(p.U, lo + seg);
  int loc = 0;
  for (int u = lo; u < hi; ++u) loc += unit_count(p, u, mode);
  int inc = loc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  int run = inc - loc;
  for (int u = lo; u < hi; ++u) {
    prefix[u] = run;
    run += unit_count(p, u, mode);
  }
  if (lane == 31) prefix[p.U] = inc;
  __syncwarp();
}

__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Unit owning global chunk g (prefix[u] <= g < prefix[u+1]); empty units skipped.
__device__ __forceinline__ int unit_of(const int* prefix, int U, int64_t g) {
  int lo = 0, hi = U - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= g) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Piece c of P over N chunks: [N c / P, N (c + 1) / P); CTAs c >= P (the
// late ones of phase 1) get an empty piece at N.
__device__ __forceinline__ void piece_range(int64_t N, int64_t P, int64_t c, int64_t& a,
                                            int64_t& bnd) {
  a = c < P ? N * c / P : N;
  bnd = c < P ? N * (c + 1) / P : N;
}

__device__ __forceinline__ int64_t piece_of(int64_t g, int64_t N, int64_t P) {
  return ((g + 1) * P - 1) / N;
}

// Splits of a unit = the non-empty pieces meeting its range [lo, hi).  With
// N >= P every piece holds >= 1 chunk; with N < P a non-empty piece holds
// exactly one chunk, so splits are counted in chunks.
__device__ __forceinline__ int split_count(int64_t lo, int64_t hi, int64_t N, int64_t P) {
  if (hi <= lo) return 0;
  return N >= P ? static_cast<int>(piece_of(hi - 1, N, P) - piece_of(lo, N, P) + 1)
                : static_cast<int>(hi - lo);
}

// Split index, within unit [lo, ...), of the piece `c` that starts at chunk a.
__device__ __forceinline__ int split_slot(int64_t lo, int64_t a, int64_t c, int64_t N, int64_t P) {
  return N >= P ? static_cast<int>(c - piece_of(lo, N, P)) : static_cast<int>(a - lo);
}

__device__ __forceinline__ void store_out(const DecodeParams& p, int64_t idx, float v) {
  if (p.out_bf16)
    static_cast<__nv_bfloat16*>(p.out)[idx] = __float2bfloat16_rn(v);
  else
    static_cast<float*>(p.out)[idx] = v;
}

// Merged mode: units of the phase with no chunk get out = 0, lse = -inf
// (no split exists to merge them); CTA c covers units c, c + P, ...
__device__ void zero_empty_units(const DecodeParams& p, const int* prefix, int mode, int nthreads) {
  for (int u = blockIdx.x; u < p.U; u += gridDim.x) {
    if (!unit_in(p, u, mode) || prefix[u + 1] > prefix[u]) continue;
    const int b = u / p.Hkv, h = u % p.Hkv;
    const int64_t row0 = static_cast<int64_t>(b) * p.Hq + h * p.G;
    for (int e = threadIdx.x; e < p.G * p.D; e += nthreads) store_out(p, row0 * p.D + e, 0.f);
    if (p.lse_out)
      for (int g = threadIdx.x; g < p.G; g += nthreads) p.lse_out[row0 + g] = -INFINITY;
  }
}

// Slots of unit u beyond its split count get lse = -inf (CTA c covers units
// u = c, c + P, ...).  Threads [0, nthreads) of the block take part.
__device__ void fill_empty_slots(const DecodeParams& p, const int* prefix, int nthreads) {
  const int64_t N = prefix[p.U], P = gridDim.x;
  for (int u = blockIdx.x; u < p.U; u += gridDim.x) {
    const int64_t lo = prefix[u], hi = prefix[u + 1];
    const int nsplit = split_count(lo, hi, N, P);
    const int b = u / p.Hkv, h = u % p.Hkv;
    if (p.merged && nsplit == 0) {  // no split will merge this unit: write its rows here
      const int64_t row0 = static_cast<int64_t>(b) * p.Hq + h * p.G;
      const int D = p.D;
      for (int e = threadIdx.x; e < p.G * D; e += nthreads) store_out(p, row0 * D + e, 0.f);
      if (p.lse_out)
        for (int g = threadIdx.x; g < p.G; g += nthreads) p.lse_out[row0 + g] = -INFINITY;
    }
    const int nfill = p.max_splits - nsplit;
    for (int e = threadIdx.x; e < p.G * nfill; e += nthreads) {
      const int g = e / nfill, s = nsplit + e % nfill;
      p.lse_part[(static_cast<int64_t>(b) * p.Hq + h * p.G + g) * p.max_splits + s] = -INFINITY;
    }
  }
}

// Combine the ns split partials of unit u (already in L2, read with ld.cg)
// into the unit's G output rows.  `wts` holds >= G * ns floats of shared
// memory; `nthr` threads take part, `tid` in [0, nthr) numbering them by
// whole warps; `sync` is a barrier over them that returns false on a timeout.
template <int D, int BATCH, typename Sync>
__device__ bool merge_unit(const DecodeParams& p, int u, int ns, float* wts, int tid, int nthr,
                           Sync sync) {
  constexpr int D4 = D / 4;
  const int b = u / p.Hkv, h = u % p.Hkv, G = p.G;
  const int64_t row0 = static_cast<int64_t>(b) * p.Hq + h * G;
  const int lane = tid & 31, warp = tid >> 5, nw = nthr >> 5;
  // Output items e = (head g, float4 column c4).  The partial loads of this
  // thread's first item do not depend on the weights: issue them first so
  // they are in flight during the lse phase.
  const int n_items = G * D4;
  float4 pre[BATCH];
  const int e0 = tid;
  if (e0 < n_items) {
    const float4* src = reinterpret_cast<const float4*>(
                            p.o_part + (row0 + e0 / D4) * p.max_splits * D) + (e0 % D4);
#pragma unroll
    for (int k = 0; k < BATCH; ++k)
      pre[k] = k < ns ? __ldcg(src + static_cast<int64_t>(k) * D4) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int e = tid; e < G * ns; e += nthr) {
    const int g = e / ns, sl = e % ns;
    wts[e] = __ldcg(p.lse_part + (row0 + g) * p.max_splits + sl);
  }
  if (!sync()) return false;
  for (int g = warp; g < G; g += nw) {
    float mx = -INFINITY;
    for (int sl = lane; sl < ns; sl += 32) mx = fmaxf(mx, wts[g * ns + sl]);
#pragma unroll
    for (int x = 16; x > 0; x >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, x));
    float sum = 0.f;
    for (int sl = lane; sl < ns; sl += 32) sum += sfu_exp(wts[g * ns + sl] - mx);
#pragma unroll
    for (int x = 16; x > 0; x >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, x);
    const float lse = mx + sfu_log(sum);
    __syncwarp();
    for (int sl = lane; sl < ns; sl += 32) wts[g * ns + sl] = sfu_exp(wts[g * ns + sl] - lse);
    if (lane == 0 && p.lse_out) p.lse_out[row0 + g] = lse;
  }
  if (!sync()) return false;
  for (int e = tid; e < n_items; e += nthr) {
    const int g = e / D4, c4 = e % D4;
    const float4* src = reinterpret_cast<const float4*>(p.o_part + (row0 + g) * p.max_splits * D) + c4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int s0 = 0;
    if (e == e0) {
#pragma unroll
      for (int k = 0; k < BATCH; ++k) {
        const float wk = k < ns ? wts[g * ns + k] : 0.f;
        acc.x += wk * pre[k].x;
        acc.y += wk * pre[k].y;
        acc.z += wk * pre[k].z;
        acc.w += wk * pre[k].w;
      }
      s0 = BATCH;
    }
    for (; s0 < ns; s0 += BATCH) {
      float4 x[BATCH];
#pragma unroll
      for (int k = 0; k < BATCH; ++k)
        x[k] = s0 + k < ns ? __ldcg(src + static_cast<int64_t>(s0 + k) * D4) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < BATCH; ++k) {
        const float wk = s0 + k < ns ? wts[g * ns + s0 + k] : 0.f;
        acc.x += wk * x[k].x;
        acc.y += wk * x[k].y;
        acc.z += wk * x[k].z;
        acc.w += wk * x[k].w;
      }
    }
    const int64_t o = (row0 + g) * D + c4 * 4;
    store_out(p, o, acc.x);
    store_out(p, o + 1, acc.y);
    store_out(p, o + 2, acc.z);
    store_out(p, o + 3, acc.w);
  }
  return sync();
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Shared-memory layout of the bf16 kernel, offsets from the 1024-aligned base:
// K/V stages | q slots (one per stage) | flush buffers | mbarriers | prefix[2][U+1].
struct DecLayout {
  int nf;        // flush buffers: 2, or 1 when two do not fit
  int fb_bytes;  // one flush buffer: per consumer warp O [G][D], m [8], l [8]
  int q_off, fb_off, bar_off, prefix_off;
  size_t total;  // dynamic shared memory to request (with the alignment slack)
};

constexpr int kQSlotHeads = 8;          // a q slot holds up to 8 query heads
constexpr size_t kMaxDynSmem = 232448;  // 227 KB per block

template <int D, int L>
struct DecodeShape {
  static constexpr int KV_BYTES = L * D * 2;
  static constexpr int STAGE_BYTES = 2 * KV_BYTES;
  static constexpr int NS = kStageBudget / STAGE_BYTES;
  static constexpr int QSLOT_BYTES = kQSlotHeads * D * 2;
};

__host__ __device__ inline DecLayout dec_layout(int D, int L, int G, int U, int nf) {
  const int stage_bytes = 2 * L * D * 2;
  const int ns = kStageBudget / stage_bytes;
  DecLayout y;
  y.nf = nf;
  y.fb_bytes = (kConsumerWarps * G * D * 4 + 2 * kConsumerWarps * 8 * 4 + 127) & ~127;
  y.q_off = ns * stage_bytes;
  y.fb_off = y.q_off + ns * kQSlotHeads * D * 2;
  y.bar_off = y.fb_off + nf * y.fb_bytes;
  y.prefix_off = y.bar_off + (2 * ns + 8) * 8;  // full[ns], empty[ns], fb_full[2], fb_empty[2], phase, end, merge, spare
  y.total = 1024 + static_cast<size_t>(y.prefix_off) + 2 * static_cast<size_t>(U + 1) * 4;
  return y;
}

__host__ __device__ inline DecLayout dec_layout(int D, int L, int G, int U) {
  DecLayout y = dec_layout(D, L, G, U, 2);
  if (y.total > kMaxDynSmem) y = dec_layout(D, L, G, U, 1);
  return y;
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Release/acquire fence at GPU scope: orders this thread's partial writes
// before its arrival count (release), and the count before the reads of a
// merge (acquire).  Lighter than the sequentially consistent __threadfence.
__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

__device__ __forceinline__ int atom_add_acq_rel_gpu(int* ptr, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(ptr), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* ptr) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// An opaque copy of v: the compiler cannot tell which loop pass a flag made
// from it is set on, so it keeps one copy of the loop body for all passes
// (a dry first pass then runs the same instructions as the real ones).
__device__ __forceinline__ int opaque(int v) {
  asm volatile("" : "+r"(v));
  return v;
}

// Merge of unit u by one warp, straight from global memory (rarely used:
// more merges fell to one CTA than its deferred list holds).
template <int D>
__device__ void merge_unit_warp(const DecodeParams& p, int u, int ns) {
  constexpr int D4 = D / 4;
  const int lane = threadIdx.x & 31;
  const int b = u / p.Hkv, h = u % p.Hkv;
  for (int g = 0; g < p.G; ++g) {
    const int64_t row = static_cast<int64_t>(b) * p.Hq + h * p.G + g;
    const float* ls = p.lse_part + row * p.max_splits;
    float mx = -INFINITY;
    for (int s = lane; s < ns; s += 32) mx = fmaxf(mx, __ldcg(ls + s));
#pragma unroll
    for (int x = 16; x > 0; x >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, x));
    float sum = 0.f;
    for (int s = lane; s < ns; s += 32) sum += sfu_exp(__ldcg(ls + s) - mx);
#pragma unroll
    for (int x = 16; x > 0; x >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, x);
    const float lse = mx + sfu_log(sum);
    if (lane < D4) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      const float4* src = reinterpret_cast<const float4*>(p.o_part + row * p.max_splits * D) + lane;
      for (int s = 0; s < ns; ++s) {
        const float wgt = sfu_exp(__ldcg(ls + s) - lse);
        const float4 x = __ldcg(src + static_cast<int64_t>(s) * D4);
        acc.x += wgt * x.x;
        acc.y += wgt * x.y;
        acc.z += wgt * x.z;
        acc.w += wgt * x.w;
      }
      const int64_t o = row * D + lane * 4;
      store_out(p, o, acc.x);
      store_out(p, o + 1, acc.y);
      store_out(p, o + 2, acc.z);
      store_out(p, o + 3, acc.w);
    }
    if (lane == 0 && p.lse_out) p.lse_out[row] = lse;
  }
}

// Shared-memory staging of a unit's merge: the ns partial rows of each head
// ([G][ns][D]) and, when rows start on 16-byte boundaries, its lse rows
// ([G][ns4], each copied rounded up to 4 floats: the workspace holds more
// after the last row), in the idle K/V stage ring; its last 8 KB hold the
// split weights.
struct MergeGeom {
  uint32_t head_bytes, lse_bytes;
  int ns4;
  bool fits;
};

template <int D>
__device__ __forceinline__ MergeGeom merge_geom(const DecodeParams& p, int ns, int area_bytes) {
  MergeGeom m;
  m.head_bytes = static_cast<uint32_t>(ns) * D * 4;
  m.ns4 = (ns + 3) & ~3;
  m.lse_bytes = (p.max_splits & 3) == 0 ? static_cast<uint32_t>(m.ns4) * 4 : 0u;
  m.fits = ns <= 256 && static_cast<size_t>(p.G) * (m.head_bytes + m.lse_bytes) <=
                            static_cast<size_t>(area_bytes) - 8192;
  return m;
}

// Issues the bulk copies of unit u's partials (and lse rows) into `area`,
// completing mbarrier `bar`.  The calling thread must have acquired the
// unit's final arrival count (the partials are other CTAs' writes).
template <int D>
__device__ void merge_bulk_issue(const DecodeParams& p, int u, int ns, const MergeGeom& m,
                                 uint8_t* area, uint32_t bar) {
  const int G = p.G;
  const int64_t row0 = static_cast<int64_t>(u / p.Hkv) * p.Hq + (u % p.Hkv) * G;
  float* st = reinterpret_cast<float*>(area);
  float* sl_rows = st + static_cast<size_t>(G) * ns * D;
  fence_proxy_async_global();  // read through the async proxy
  fence_proxy_async_shared();  // the area may last have been written by cp.async
  mbar_arrive_expect_tx(bar, static_cast<uint32_t>(G) * (m.head_bytes + m.lse_bytes));
  for (int g = 0; g < G; ++g) {
    bulk_load(smem_u32(st + static_cast<size_t>(g) * ns * D),
              p.o_part + (row0 + g) * p.max_splits * D, m.head_bytes, bar);
    if (m.lse_bytes)
      bulk_load(smem_u32(sl_rows + g * m.ns4), p.lse_part + (row0 + g) * p.max_splits,
                m.lse_bytes, bar);
  }
}

// Merge of unit u from its staged partials (merge_geom): one bulk copy per
// head row set, so the partials cross from L2 in a single round trip (issued
// here by tid 0, or earlier when `issued`); `bar` is an mbarrier of this CTA
// (count 1) and `n_bulk` counts the copies that completed it so far.  Then
// each warp takes whole heads: the head's lse and split weights stay in the
// warp (shuffles and a per-warp slice of the weights), and the lanes
// accumulate float4 columns, with no block barrier in between.  `nthr`
// (<= 256) threads numbered `tid` by whole warps take part; `sync` is a
// barrier over them (bounded).  Falls back to merge_unit when the partials
// do not fit.
template <int D, typename Sync>
__device__ bool merge_staged(const DecodeParams& p, int u, int ns, uint8_t* area, int area_bytes,
                             uint32_t bar, uint32_t& n_bulk, bool issued, int tid, int nthr,
                             Sync sync) {
  constexpr int D4 = D / 4;
  const int G = p.G;
  const int64_t row0 = static_cast<int64_t>(u / p.Hkv) * p.Hq + (u % p.Hkv) * G;
  const MergeGeom m = merge_geom<D>(p, ns, area_bytes);
  float* wts = reinterpret_cast<float*>(area + area_bytes - 8192);
  if (!m.fits) return merge_unit<D, 8>(p, u, ns, wts, tid, nthr, sync);
  const uint32_t phase = n_bulk & 1u;
  ++n_bulk;
  float* st = reinterpret_cast<float*>(area);                    // [G][ns][D]
  float* sl_rows = st + static_cast<size_t>(G) * ns * D;         // [G][ns4]
  const bool lse_bulk = m.lse_bytes != 0;
  const int ns4 = m.ns4;
  if (!issued && tid == 0) merge_bulk_issue<D>(p, u, ns, m, area, bar);
  const int lane = tid & 31, warp = tid >> 5, nw = nthr >> 5;
  float* ww = wts + warp * 256;  // this warp's split weights
  bool ok = warp_wait(bar, phase, p.err);
  for (int g = warp; g < G && ok; g += nw) {
    const float* lsp = p.lse_part + (row0 + g) * p.max_splits;
    float mx = -INFINITY;
    for (int sl = lane; sl < ns; sl += 32) {
      const float v = lse_bulk ? sl_rows[g * ns4 + sl] : __ldcg(lsp + sl);
      ww[sl] = v;
      mx = fmaxf(mx, v);
    }
#pragma unroll
    for (int x = 16; x > 0; x >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, x));
    float sum = 0.f;
    for (int sl = lane; sl < ns; sl += 32) sum += sfu_exp(ww[sl] - mx);
#pragma unroll
    for (int x = 16; x > 0; x >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, x);
    const float lse = mx + sfu_log(sum);
    for (int sl = lane; sl < ns; sl += 32) ww[sl] = sfu_exp(ww[sl] - lse);
    __syncwarp();
    if (lane == 0 && p.lse_out) p.lse_out[row0 + g] = lse;
    for (int c4 = lane; c4 < D4; c4 += 32) {
      const float* src = st + static_cast<size_t>(g) * ns * D + c4 * 4;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int sl = 0; sl < ns; ++sl) {
        const float wk = ww[sl];
        const float4 x = *reinterpret_cast<const float4*>(src + static_cast<size_t>(sl) * D);
        acc.x += wk * x.x;
        acc.y += wk * x.y;
        acc.z += wk * x.z;
        acc.w += wk * x.w;
      }
      const int64_t o = (row0 + g) * D + c4 * 4;
      store_out(p, o, acc.x);
      store_out(p, o + 1, acc.y);
      store_out(p, o + 2, acc.z);
      store_out(p, o + 3, acc.w);
    }
    __syncwarp();
  }
  return sync() && ok;  // the area is free again
}

// The epilogue warp's work for one flushed unit: combine the four consumer
// warps' (m, l, O) from flush buffer `fo` into the unit's split partial (or
// its output when ns == 1), release the buffer, and count the split in.
// Returns 1 when this CTA brought the unit's last split (its merge is
// deferred), 2 when it also started the merge's copy already (the CTA's last
// flush), else 0.  `dry`: the same instructions with every write, release
// and count left out (a first pass that only fetches the code).
template <int D>
__device__ __forceinline__ int epilogue_unit(const DecodeParams& p, const float* fo, int u,
                                             int slot, int ns, bool final_flush, uint8_t* area,
                                             int area_bytes, uint32_t merge_bar,
                                             uint32_t fb_empty, int* pre_u, int* pre_ns,
                                             bool dry) {
  static_assert(kConsumerWarps == 4, "four partials per head");
  const int lane = threadIdx.x & 31, G = p.G;
  const float* fm = fo + kConsumerWarps * G * D;
  const float* fl = fm + kConsumerWarps * 8;
  const int64_t row0 = static_cast<int64_t>(u / p.Hkv) * p.Hq + (u % p.Hkv) * G;
  const bool direct = p.merged && ns == 1;  // the only split: it is the output
  // Lane g < G: head g's max over the warps, and the weights of the warps'
  // partials normalised by the total sum; it also writes the head's lse.
  float wn[kConsumerWarps] = {0.f, 0.f, 0.f, 0.f};
  if (lane < G) {
    float M = -INFINITY, Ls = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, fm[w * 8 + lane]);
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      wn[w] = fast_exp2(fm[w * 8 + lane] - M);
      Ls += fl[w * 8 + lane] * wn[w];
    }
    const float inv = 1.0f / Ls;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) wn[w] *= inv;
    const float lse = (M + __log2f(Ls)) * kLn2;
    if (dry) {
    } else if (!direct) {
      p.lse_part[(row0 + lane) * p.max_splits + slot] = lse;
    } else if (p.lse_out) {
      p.lse_out[row0 + lane] = lse;
    }
  }
  // Every lane: columns lane + 32 j of every head, all independent (the
  // weights of all heads first, then the loads and stores).
  float wg[8][kConsumerWarps];
#pragma unroll
  for (int g = 0; g < 8; ++g)
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) wg[g][w] = __shfl_sync(0xffffffffu, wn[w], g);
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    if (g < G) {
      const int64_t row = row0 + g;
#pragma unroll
      for (int d = lane; d < D; d += 32) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) acc += fo[(w * G + g) * D + d] * wg[g][w];
        if (dry) continue;
        if (direct) store_out(p, row * D + d, acc);
        else p.o_part[(row * p.max_splits + slot) * D + d] = acc;
      }
    }
  }
  __syncwarp();
  if (dry) return 0;
  if (lane == 0) mbar_arrive(fb_empty);  // the consumers may refill it
  if (!p.merged || direct) return 0;
  fence_acq_rel_gpu();  // this lane's partial writes before the arrival count
  __syncwarp();
  int last = 0;
  if (lane == 0) {
    last = atom_add_acq_rel_gpu(p.counters + u, 1) == ns - 1;
    const MergeGeom mg = merge_geom<D>(p, ns, area_bytes);
    if (last && final_flush && mg.fits) {  // start the merge's copy now, before the CTA barrier
      merge_bulk_issue<D>(p, u, ns, mg, area, merge_bar);
      *pre_u = u;
      *pre_ns = ns;
      last = 2;
    }
  }
  return __shfl_sync(0xffffffffu, last, 0);
}

// ---------------------------------------------------------------- producer

// The K/V tensor maps of a launch: raw rows [B*Hkv*T, D] and gist rows.
struct KVMaps {
  const CUtensorMap* K;
  const CUtensorMap* V;
  const CUtensorMap* Kg;
  const CUtensorMap* Vg;
};

// Fill ring slot i % ns (stage at `dst`, barriers full/empty) with one chunk:
// row >= 0 a raw K/V row block and row < 0 the gist rows -(row + 1).. (both
// by TMA, issued by lane 0), or gsel >= 0 a gathered gist chunk (all 32
// lanes).  qu >= 0: unit qu's query rows ride along into q slot `qdst`.
// Called by the whole producer warp with warp-uniform arguments; false when
// the wait for the slot ran out of time.
template <int D, int L>
__device__ __forceinline__ bool issue_stage(const DecodeParams& p, const KVMaps& m, int64_t i,
                                            int ns, uint32_t dst, uint32_t full_bar,
                                            uint32_t empty_bar, int row, int gsel, int qu,
                                            uint32_t qdst, uint64_t kv_policy,
                                            uint32_t& cp_stages) {
  constexpr int KV_BYTES = L * D * 2, STAGE_BYTES = 2 * KV_BYTES, BOX_BYTES = L * 128;
  const int lane = threadIdx.x & 31;
  const int s = static_cast<int>(i % ns);
  const uint32_t fb = full_bar + 8 * s;
  const uint32_t q_bytes = static_cast<uint32_t>(p.G) * D * 2;
  const __nv_bfloat16* qsrc = nullptr;
  if (qu >= 0)
    qsrc = static_cast<const __nv_bfloat16*>(p.q) +
           (static_cast<int64_t>(qu / p.Hkv) * p.Hq + (qu % p.Hkv) * p.G) * D;
  int good = 1;
  if (lane == 0) {
    const uint32_t it = static_cast<uint32_t>(i / ns);
    if (!mbar_wait(empty_bar + 8 * s, (it & 1u) ^ 1u, p.err)) {
      good = 0;
    } else if (gsel < 0) {
      if (cp_stages & (1u << s)) {  // the copies that filled it last were cp.async
        fence_proxy_async_shared();
        cp_stages &= ~(1u << s);
      }
      mbar_arrive_expect_tx(fb, STAGE_BYTES + (qu >= 0 ? q_bytes : 0u));
      if (qu >= 0) bulk_load(qdst, qsrc, q_bytes, fb);
      const bool gist = row < 0;  // rows of a ragged last gist chunk past
      const int r = gist ? -row - 1 : row;  // the tensor read as zeros
      const CUtensorMap* mk = gist ? m.Kg : m.K;
      const CUtensorMap* mv = gist ? m.Vg : m.V;
#pragma unroll
      for (int bx = 0; bx < D / 64; ++bx) {
        tma_load_2d_hint(dst + bx * BOX_BYTES, mk, bx * 64, r, fb, kv_policy);
        tma_load_2d_hint(dst + KV_BYTES + bx * BOX_BYTES, mv, bx * 64, r, fb, kv_policy);
      }
    }
  }
  good = __shfl_sync(0xffffffffu, good, 0);
  if (good && gsel >= 0) {  // warp-uniform: a gathered gist chunk
    gather_gist_rows<D, L>(p, gsel, dst, fb);
    __syncwarp();  // every lane's pending arrival before the barrier's own
    if (lane == 0) {
      cp_stages |= 1u << s;
      if (qu >= 0) {
        mbar_arrive_expect_tx(fb, q_bytes);
        bulk_load(qdst, qsrc, q_bytes, fb);
      } else {
        mbar_arrive(fb);
      }
    }
  }
  return good != 0;
}

// ---------------------------------------------------------------- per-warp attention
//
// A consumer warp takes L/4 tokens of every chunk.  S^T = K q^T runs as
// mma.m16n8k16 with the tokens as M and the query heads of the GQA group as
// N (lane l holds heads hA = 2 (l % 4) and hB = hA + 1); the online softmax
// (log2 domain) stays in registers; P goes into the B layout with movmatrix
// and O^T += V^T P^T runs as a second mma.

template <int D>
struct WarpAcc {
  uint32_t qf[D / 16][2];  // the unit's query heads as B fragments
  float o[D / 16][4];      // O^T tiles: d = 16 dt + lane/4 (+8), heads hA / hB
  float m0, m1, l0, l1;    // running max (log2 domain) and sum of heads hA / hB
};

// Start a unit: its G query rows from a q slot ([8][D] bf16), accumulators zeroed.
template <int D>
__device__ __forceinline__ void acc_begin(WarpAcc<D>& w, const __nv_bfloat16* qs, int G,
                                          int lane) {
  const int n = lane >> 2;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const int d0 = ks * 16 + 2 * (lane & 3);
    if (n < G) {
      w.qf[ks][0] = *reinterpret_cast<const uint32_t*>(qs + n * D + d0);
      w.qf[ks][1] = *reinterpret_cast<const uint32_t*>(qs + n * D + d0 + 8);
    } else {
      w.qf[ks][0] = 0u;
      w.qf[ks][1] = 0u;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) w.o[ks][e] = 0.f;
  }
  w.m0 = w.m1 = -INFINITY;
  w.l0 = w.l1 = 0.f;
}

// One stage (K at sK, V at sK + L*D*2, each as [L x 64] boxes with the
// 128-byte swizzle) into the warp's accumulators; rows >= valid take no part.
template <int D, int L>
__device__ __forceinline__ void acc_stage(WarpAcc<D>& w, uint32_t sK, int warp, int lane,
                                          float scale_log2, int valid) {
  constexpr int TOK_W = L / kConsumerWarps;  // tokens per consumer warp
  constexpr int MT = TOK_W / 16;             // 16-token m-tiles per warp
  constexpr int KS = D / 16;                 // k-steps (QK) / d-tiles (PV)
  constexpr int KV_BYTES = L * D * 2, BOX_BYTES = L * 128;
  const uint32_t sV = sK + KV_BYTES;
  const int tok0 = warp * TOK_W;
  // S^T = K q^T over this warp's tokens
  float sc[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) sc[mt][e] = 0.f;
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int bx = ks >> 2, colb = (ks & 3) * 16;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int row = tok0 + mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int col = colb + (lane >> 4) * 8;
      uint32_t a0, a1, a2, a3;
      ldsm_x4(sK + bx * BOX_BYTES + sw128_offset(row, col), a0, a1, a2, a3);
      mma_bf16_16816(sc[mt], a0, a1, a2, a3, w.qf[ks][0], w.qf[ks][1]);
    }
  }
  if (valid < L) {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (tok0 + mt * 16 + (lane >> 2) + (e >> 1) * 8 >= valid) sc[mt][e] = -INFINITY;
  }
  // online softmax (log2 domain), per head hA / hB of this lane
  float cm0 = -INFINITY, cm1 = -INFINITY;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) sc[mt][e] *= scale_log2;
    cm0 = fmaxf(cm0, fmaxf(sc[mt][0], sc[mt][2]));
    cm1 = fmaxf(cm1, fmaxf(sc[mt][1], sc[mt][3]));
  }
#pragma unroll
  for (int x = 4; x < 32; x <<= 1) {
    cm0 = fmaxf(cm0, __shfl_xor_sync(0xffffffffu, cm0, x));
    cm1 = fmaxf(cm1, __shfl_xor_sync(0xffffffffu, cm1, x));
  }
  const float mn0 = fmaxf(w.m0, cm0), mn1 = fmaxf(w.m1, cm1);
  // exponent reference: 0 while every row this warp has seen was masked
  // (max -inf), so that no -inf - -inf arises
  const float rf0 = mn0 == -INFINITY ? 0.f : mn0, rf1 = mn1 == -INFINITY ? 0.f : mn1;
  const float al0 = fast_exp2(w.m0 - rf0), al1 = fast_exp2(w.m1 - rf1);
  w.m0 = mn0;
  w.m1 = mn1;
  uint32_t pb[MT][2];
  float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const float p0 = fast_exp2(sc[mt][0] - rf0), p1 = fast_exp2(sc[mt][1] - rf1);
    const float p2 = fast_exp2(sc[mt][2] - rf0), p3 = fast_exp2(sc[mt][3] - rf1);
    ps0 += p0 + p2;
    ps1 += p1 + p3;
    pb[mt][0] = movmatrix_trans(pack_bf16x2(p0, p1));
    pb[mt][1] = movmatrix_trans(pack_bf16x2(p2, p3));
  }
  w.l0 = w.l0 * al0 + ps0;
  w.l1 = w.l1 * al1 + ps1;
#pragma unroll
  for (int dt = 0; dt < KS; ++dt) {
    w.o[dt][0] *= al0;
    w.o[dt][1] *= al1;
    w.o[dt][2] *= al0;
    w.o[dt][3] *= al1;
  }
  // O^T += V^T P^T
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int dt = 0; dt < KS; ++dt) {
      const int bx = dt >> 2, colb = (dt & 3) * 16;
      const int mi = lane >> 3;
      const int tok = tok0 + mt * 16 + (lane & 7) + (mi >> 1) * 8;
      const int col = colb + (mi & 1) * 8;
      uint32_t a0, a1, a2, a3;
      ldsm_x4_trans(sV + bx * BOX_BYTES + sw128_offset(tok, col), a0, a1, a2, a3);
      mma_bf16_16816(w.o[dt], a0, a1, a2, a3, pb[mt][0], pb[mt][1]);
    }
  }
}

// The warp's (m, l, O) into a flush buffer: O [kConsumerWarps][G][D], then
// m [kConsumerWarps][8], l [kConsumerWarps][8] (fp32); the sums are reduced
// over the lanes of a head first.
template <int D>
__device__ __forceinline__ void acc_write(WarpAcc<D>& w, float* fo, int G, int warp, int lane) {
#pragma unroll
  for (int x = 4; x < 32; x <<= 1) {
    w.l0 += __shfl_xor_sync(0xffffffffu, w.l0, x);
    w.l1 += __shfl_xor_sync(0xffffffffu, w.l1, x);
  }
  const int hA = 2 * (lane & 3), hB = hA + 1;
  float* fm = fo + kConsumerWarps * G * D;
  float* fl = fm + kConsumerWarps * 8;
  if (lane < 4) {
    fm[warp * 8 + hA] = w.m0;
    fm[warp * 8 + hB] = w.m1;
    fl[warp * 8 + hA] = w.l0;
    fl[warp * 8 + hB] = w.l1;
  }
#pragma unroll
  for (int dt = 0; dt < D / 16; ++dt) {
    const int d = dt * 16 + (lane >> 2);
    if (hA < G) {
      fo[(warp * G + hA) * D + d] = w.o[dt][0];
      fo[(warp * G + hA) * D + d + 8] = w.o[dt][2];
    }
    if (hB < G) {
      fo[(warp * G + hB) * D + d] = w.o[dt][1];
      fo[(warp * G + hB) * D + d + 8] = w.o[dt][3];
    }
  }
}

template <int D, int L>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    decode_bf16_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmKg,
                       const __grid_constant__ CUtensorMap tmVg,
                       const __grid_constant__ DecodeParams p) {
  using Sh = DecodeShape<D, L>;
  constexpr int NS = Sh::NS;
  const DecLayout Y = dec_layout(D, L, p.G, p.U);
  const int G = p.G;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t full_bar = sbase + Y.bar_off;
  const uint32_t empty_bar = full_bar + NS * 8;
  const uint32_t fb_full = empty_bar + NS * 8;  // [2]
  const uint32_t fb_empty = fb_full + 16;       // [2]
  const uint32_t phase_bar = fb_empty + 16;
  const uint32_t end_bar = phase_bar + 8;
  const uint32_t merge_bar = end_bar + 8;  // completed by the final merges' bulk copies
  int* prefix = reinterpret_cast<int*>(smem + Y.prefix_off);  // [U+1]
  int* prefix2 = prefix + (p.U + 1);  // phase 2 (sparse units), built by the producer
  __shared__ int scan_sh[33];
  __shared__ int defer_u[kDeferMax], defer_ns[kDeferMax];
  __shared__ int n_defer_sh, pre_u_sh, pre_ns_sh, own_ok_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // split partials out (no merge here): the merge kernel launched behind this
  // one may become resident now; it waits for this grid before reading them
  if (!p.merged) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full_bar + 8 * s, 1);
      mbar_init(empty_bar + 8 * s, kConsumerWarps);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(fb_full + 8 * k, kConsumerWarps * 32);
      mbar_init(fb_empty + 8 * k, 1);
    }
    mbar_init(phase_bar, 1);
    mbar_init(end_bar, (kConsumerWarps + 1) * 32);
    mbar_init(merge_bar, 1);
    n_defer_sh = 0;
    pre_u_sh = -1;
    fence_barrier_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    if (p.n_gist > 0) {
      prefetch_tensormap(&tmKg);
      prefetch_tensormap(&tmVg);
    }
  }
  build_prefix(p, prefix, scan_sh, p.phased ? 1 : 0);  // ends with __syncthreads (also publishes the barriers)
  const int n_phase = p.phased ? 2 : 1;
  // pieces per phase: phase 1 of a phased launch leaves out the late CTAs
  const int64_t P_all = gridDim.x;
  auto phase_parts = [&](int ph) -> int64_t {
    return (p.phased && ph == 0) ? P_all - p.late : P_all;
  };
  // merged phased launches: the late CTAs merge the full-head units
  const bool own_full = p.merged && p.phased && p.late > 0;

  if (warp == kProducerWarp) {
    // ---------------------------------------------------------------- producer
    const KVMaps maps{&tmK, &tmV, &tmKg, &tmVg};
    // K/V is read once: first out of L2, so that what the kernel reads again
    // (its instructions, parameters, the partials and counters) stays there
    const uint64_t kv_policy = l2_policy_evict_first();
    uint32_t cp_stages = 0;  // lane 0: stages last filled by cp.async (selected-gist chunks)
    int64_t issued = 0;
    bool ok = true;
    for (int ph = 0; ph < n_phase && ok; ++ph) {
      const int* pre = prefix;
      if (ph == 1) {  // the selection has to be complete from here on
        grid_dependency_wait();
        warp_build_prefix(p, prefix2, 2);
        if (lane == 0) mbar_arrive(phase_bar);
        pre = prefix2;
      }
      const int64_t N = pre[p.U];
      int64_t a, bnd;
      piece_range(N, phase_parts(ph), blockIdx.x, a, bnd);
      for (int64_t g0 = a; g0 < bnd && ok; g0 += 32) {
        const int64_t g = g0 + lane;
        int row = 0, qu = -1, gsel = -1;
        if (g < bnd) {
          const int u = unit_of(pre, p.U, g);
          row = unit_row(p, u, static_cast<int>(g - pre[u]), L, &gsel);
          if (g == a || g == pre[u]) qu = u;  // first chunk of a unit here: its q rides along
        }
        const int nb = static_cast<int>(bnd - g0 < 32 ? bnd - g0 : 32);
        for (int j = 0; j < nb; ++j) {
          const int row_j = __shfl_sync(0xffffffffu, row, j);
          const int qu_j = __shfl_sync(0xffffffffu, qu, j);
          const int gs_j = __shfl_sync(0xffffffffu, gsel, j);
          const int s = static_cast<int>(issued % NS);
          const bool good = issue_stage<D, L>(p, maps, issued, NS, sbase + s * Sh::STAGE_BYTES,
                                              full_bar, empty_bar, row_j, gs_j, qu_j,
                                              sbase + Y.q_off + s * Sh::QSLOT_BYTES, kv_policy,
                                              cp_stages);
          if (!good) {
            ok = false;
            break;
          }
          ++issued;
        }
      }
    }
    if (!ok && p.phased) {  // never leave the other warps waiting: hand them an empty phase
      for (int u = lane; u <= p.U; u += 32) prefix2[u] = 0;
      __syncwarp();
      if (lane == 0) mbar_arrive(phase_bar);
    }
    // no copy may still be landing when the CTA retires
    if (lane == 0) {
      const int64_t first = issued > NS ? issued - NS : 0;
      for (int64_t i = first; i < issued; ++i)
        mbar_wait(full_bar + 8 * static_cast<int>(i % NS), static_cast<uint32_t>(i / NS) & 1u, p.err);
    }
    return;
  }

  // consumers and the epilogue warp meet at the end (merged mode) to run
  // the merges that fell to this CTA
  uint32_t end_phase = 0;
  auto end_sync = [&]() -> bool {
    mbar_arrive(end_bar);
    const bool r = warp_wait(end_bar, end_phase, p.err);
    end_phase ^= 1u;
    return r;
  };
  auto final_merges = [&](int tid) {
    if (!end_sync()) return;
    const int nd = n_defer_sh, pu = pre_u_sh;
    uint32_t n_bulk = 0;
    if (nd > 0 || pu >= 0) {
      // the arrival counts seen (by the epilogue's atomics) before partials are
      // read by these threads; not needed when the only merge's partials and
      // lse rows come by the bulk copy its own issuer ordered
      if (nd > 0 || (p.max_splits & 3) != 0) fence_acq_rel_gpu();
      if (pu >= 0) {  // the last unit of the CTA: its copy is already in flight
        if (!merge_staged<D>(p, pu, pre_ns_sh, smem, NS * Sh::STAGE_BYTES, merge_bar, n_bulk,
                             true, tid, (kConsumerWarps + 1) * 32, end_sync))
          return;
        if (tid == 0) p.counters[pu] = 0;  // ready for the next call
      }
      for (int k = 0; k < nd; ++k) {
        const int u = defer_u[k];
        if (!merge_staged<D>(p, u, defer_ns[k], smem, NS * Sh::STAGE_BYTES, merge_bar, n_bulk,
                             false, tid, (kConsumerWarps + 1) * 32, end_sync))
          return;
        if (tid == 0) p.counters[u] = 0;  // ready for the next call
      }
    }
    // A late CTA of a merged phased launch merges the full-head units assigned
    // to it (the k-th such unit to late CTA k mod late): their splits all come
    // in phase 1, while the late CTAs' own work is phase 2 only, so these
    // merges run beside the other CTAs' streaming instead of at the end.
    if (own_full && static_cast<int64_t>(blockIdx.x) >= P_all - p.late) {
      const int64_t N1 = prefix[p.U], P1 = P_all - p.late;
      const int li = static_cast<int>(blockIdx.x - P1);
      int kf = 0;
      for (int u = 0; u < p.U; ++u) {
        if (prefix[u + 1] <= prefix[u]) continue;  // not a phase-1 unit
        if (kf++ % p.late != li) continue;
        const int ns = split_count(prefix[u], prefix[u + 1], N1, P1);
        if (ns <= 1) continue;  // one split writes the unit's rows itself
        if (tid == 0) {  // every split counted in (bounded)
          int ok = 1;
          const uint64_t t0 = globaltimer_ns();
          while (ld_acquire_gpu(p.counters + u) < ns) {
            if (globaltimer_ns() - t0 > p.err.wait_ns) {
              dev_flag(p.err, DEV_TIMEOUT);
              ok = 0;
              break;
            }
            __nanosleep(64);
          }
          own_ok_sh = ok;
        }
        if (!end_sync() || !own_ok_sh) return;
        if (!merge_staged<D>(p, u, ns, smem, NS * Sh::STAGE_BYTES, merge_bar, n_bulk, false, tid,
                             (kConsumerWarps + 1) * 32, end_sync))
          return;
        if (tid == 0) p.counters[u] = 0;  // ready for the next call
      }
    }
  };

  if (warp == kEpilogueWarp) {
    // ---------------------------------------------------------------- epilogue
    // Takes each unit's four per-warp partials from a flush buffer, combines
    // them into the unit's split partial (or its output when it has one
    // split), and counts the split in (merged mode) while the consumers
    // stream on.
    bool ok = true;
    int nseen = 0, n_defer = 0;
    for (int ph = 0; ph < n_phase && ok; ++ph) {
      const int* pre = prefix;
      if (ph == 1) {
        if (!warp_wait(phase_bar, 0u, p.err)) {
          ok = false;
          break;
        }
        pre = prefix2;
      }
      const int64_t N = pre[p.U], P = phase_parts(ph);
      int64_t a, bnd;
      piece_range(N, P, blockIdx.x, a, bnd);
      if (a >= bnd) continue;
      const int u0 = unit_of(pre, p.U, a), u1 = unit_of(pre, p.U, bnd - 1);
      // phase 0 starts with a dry pass of the loop body (no wait, nothing
      // written) while the first stages are in flight: its code is then in
      // the instruction caches for the real flushes
      for (int u = u0 - (ph == 0 ? 1 : 0); u <= u1 && ok; ++u) {
        const bool dry = opaque(u < u0 ? 1 : 0) != 0;
        if (!dry && pre[u + 1] <= pre[u]) continue;  // no chunk: never flushed
        // the split's slot and count before the wait (64-bit divisions)
        const int slot = dry ? 0 : split_slot(pre[u], a, blockIdx.x, N, P);
        const int ns = dry ? 2 : split_count(pre[u], pre[u + 1], N, P);
        const int k = dry ? 0 : (Y.nf == 2 ? (nseen & 1) : 0);
        const int use = Y.nf == 2 ? (nseen >> 1) : nseen;
        if (!dry && !warp_wait(fb_full + 8 * k, static_cast<uint32_t>(use) & 1u, p.err)) {
          ok = false;
          break;
        }
        if (!dry) ++nseen;
        const float* fo = reinterpret_cast<const float*>(smem + Y.fb_off + k * Y.fb_bytes);
        // the CTA's last flush: the consumers are done with the stage ring
        const bool final_flush = !dry && ph == n_phase - 1 && u == u1;
        int last = epilogue_unit<D>(p, fo, dry ? u0 : u, slot, ns, final_flush, smem,
                                    NS * Sh::STAGE_BYTES, merge_bar, fb_empty + 8 * k, &pre_u_sh,
                                    &pre_ns_sh, dry);
        if (dry || last != 1) continue;
        if (ph == 0 && own_full) continue;  // a late CTA merges it
        if (n_defer < kDeferMax) {  // merged after the main loop, off the hot path
          if (lane == 0) {
            defer_u[n_defer] = u;
            defer_ns[n_defer] = ns;
          }
          ++n_defer;
        } else {
          fence_acq_rel_gpu();
          merge_unit_warp<D>(p, u, ns);
          __syncwarp();
          if (lane == 0) p.counters[u] = 0;
        }
      }
    }
    if (!p.merged) return;
    if (lane == 0) n_defer_sh = n_defer;
    __syncwarp();
    final_merges(kConsumerWarps * 32 + lane);
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int* pre = prefix;
  int64_t N = pre[p.U];
  int64_t a, bnd;
  piece_range(N, phase_parts(0), blockIdx.x, a, bnd);
  if (p.merged) zero_empty_units(p, pre, p.phased ? 1 : 0, kConsumerWarps * 32);
  else fill_empty_slots(p, pre, kConsumerWarps * 32);
  const float scale_log2 = p.scale_log2;
  WarpAcc<D> acc;
  int cur_u = -1, nflush = 0;
  bool cur_full = false;  // hybrid launches: the current unit is a full-attention one
  int cur_ns = 0;         // hybrid launches: the current unit's selected chunks
  const bool hybrid = p.n_gist > 0 || p.gist_sel;
  bool ok = true;

  // Hand this warp's (m, l, O) of unit u to the epilogue warp and go on.
  auto flush_async = [&](int u) -> bool {
    (void)u;
    const int k = Y.nf == 2 ? (nflush & 1) : 0;
    const int use = Y.nf == 2 ? (nflush >> 1) : nflush;
    if (use > 0 && !warp_wait(fb_empty + 8 * k, static_cast<uint32_t>(use - 1) & 1u, p.err))
      return false;
    acc_write<D>(acc, reinterpret_cast<float*>(smem + Y.fb_off + k * Y.fb_bytes), G, warp, lane);
    mbar_arrive(fb_full + 8 * k);
    ++nflush;
    return true;
  };

  int64_t i = 0;
  for (int ph = 0; ph < n_phase && ok; ++ph) {
    if (ph == 1) {
      if (cur_u >= 0) {  // phases hold different units
        if (!flush_async(cur_u)) {
          ok = false;
          break;
        }
        cur_u = -1;
      }
      if (!warp_wait(phase_bar, 0u, p.err)) {
        ok = false;
        break;
      }
      grid_dependency_wait();
      pre = prefix2;
      N = pre[p.U];
      piece_range(N, phase_parts(1), blockIdx.x, a, bnd);
      zero_empty_units(p, pre, 2, kConsumerWarps * 32);
    }
    // phase 0 starts with a dry pass of the loop body over stage 0 (no
    // wait, nothing released or kept; the accumulator is set up again by the
    // first real chunk) while the first stages are in flight: its code is
    // then in the instruction caches when the data arrives
    for (int64_t g = (ph == 0 && a < bnd) ? a - 1 : a; g < bnd; ++g) {
      const bool dry = opaque(g < a ? 1 : 0) != 0;
      const int s = dry ? 0 : static_cast<int>(i % NS);
      const uint32_t it = static_cast<uint32_t>(i / NS);
      if (!dry && !warp_wait(full_bar + 8 * s, it & 1u, p.err)) {
        ok = false;
        break;
      }
      if (!dry && (cur_u < 0 || g >= pre[cur_u + 1])) {
        if (cur_u >= 0 && !flush_async(cur_u)) {
          ok = false;
          break;
        }
        cur_u = unit_of(pre, p.U, g);
        cur_full = hybrid && p.head_full != nullptr && p.head_full[cur_u % p.Hkv];
        if (hybrid && !cur_full) cur_ns = sel_count(p, cur_u);
        // the unit's q arrived with this stage
        acc_begin<D>(acc,
                     reinterpret_cast<const __nv_bfloat16*>(smem + Y.q_off + s * Sh::QSLOT_BYTES),
                     G, lane);
      }
      int valid = L;
      if (!dry && hybrid && !cur_full) {
        // a hybrid unit's last gist chunk is ragged: rows past its gist rows
        // (the next unit's, zeros past the tensor, or the zero-filled rows of
        // a gathered chunk) take no part
        const int j = static_cast<int>(g - pre[cur_u]) - cur_ns;
        if (j >= 0) valid = min(L, gist_rows_of(p, cur_ns) - j * L);
      }
      acc_stage<D, L>(acc, sbase + s * Sh::STAGE_BYTES, warp, lane, scale_log2, valid);
      __syncwarp();
      if (dry) continue;
      if (lane == 0) mbar_arrive(empty_bar + 8 * s);
      ++i;
    }
  }
  if (ok && cur_u >= 0) ok = flush_async(cur_u);
  if (!p.merged) return;
  final_merges(threadIdx.x);
}

// ------------------------------------------------------------------ cluster path
//
// Steps with few chunks per unit: one thread-block cluster of CS CTAs per
// unit, CTA r of the cluster streaming the r-th of CS equal parts of the
// unit's list (its chunks, then its gist chunks).  The parts are combined
// through distributed shared memory: each CTA folds its four consumer
// warps' (m, l, O) into one partial and writes it into a slot of the
// cluster's first CTA, which writes the unit's output rows and lse after a
// cluster barrier.  No partial leaves the cluster, so there is no global
// workspace traffic, arrival counter or separate merge.  Warps 0-3 consume,
// warp 4 produces (as in the persistent kernel).  Both cluster barriers are
// reached by every thread on every path (a timed-out wait only skips work),
// so a wait that ran out of time cannot leave the cluster waiting.

constexpr int kClusterThreads = (kConsumerWarps + 1) * 32;
constexpr int kClusterMax = 8;  // portable cluster size

// Shared memory of the cluster kernel, offsets from the 1024-aligned base:
// K/V stages | q slot | flush buffer | CS partial slots | mbarriers.
struct ClLayout {
  int ns;                                   // ring stages
  int q_off, fo_off, part_off, part_stride, bar_off;
  size_t total;
};

__host__ __device__ inline ClLayout cl_layout(int D, int L, int G, int CS) {
  const int stage_bytes = 2 * L * D * 2;
  ClLayout y;
  const int fo_bytes = (kConsumerWarps * G * D + 2 * kConsumerWarps * 8) * 4;
  y.part_stride = (G * D + 16) * 4;  // per slot: M [8], Lsum [8], O [G][D] (fp32)
  const int fixed = kQSlotHeads * D * 2 + ((fo_bytes + 127) & ~127) +
                    ((CS * y.part_stride + 127) & ~127) + 64 * 8;
  int ns = kStageBudget / stage_bytes;
  const int room = static_cast<int>(kMaxDynSmem) - 1024 - fixed;
  if (ns * stage_bytes > room) ns = room / stage_bytes;
  y.ns = ns;
  y.q_off = ns * stage_bytes;
  y.fo_off = y.q_off + kQSlotHeads * D * 2;
  y.part_off = y.fo_off + ((fo_bytes + 127) & ~127);
  y.bar_off = y.part_off + ((CS * y.part_stride + 127) & ~127);
  y.total = 1024 + static_cast<size_t>(y.bar_off) + (2 * ns + 2) * 8;
  return y;
}

template <int D, int L>
__global__ void __launch_bounds__(kClusterThreads, 1)
    decode_cluster_kernel(const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV,
                          const __grid_constant__ CUtensorMap tmKg,
                          const __grid_constant__ CUtensorMap tmVg,
                          const __grid_constant__ DecodeParams p) {
  cluster_arrive_relaxed();  // every CTA of the cluster has started by the matching wait
  const int G = p.G;
  const int CS = static_cast<int>(cluster_size());
  const int rank = static_cast<int>(cluster_rank());
  const int u = blockIdx.y;
  const ClLayout Y = cl_layout(D, L, G, CS);
  const int NS = Y.ns;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t full_bar = sbase + Y.bar_off;
  const uint32_t empty_bar = full_bar + NS * 8;
  const uint32_t fo_bar = empty_bar + NS * 8;
  float* fo = reinterpret_cast<float*>(smem + Y.fo_off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int k = 0; k < NS; ++k) {
      mbar_init(full_bar + 8 * k, 1);
      mbar_init(empty_bar + 8 * k, kConsumerWarps);
    }
    mbar_init(fo_bar, kConsumerWarps * 32);
    fence_barrier_init();
  }
  if (warp == kConsumerWarps && lane == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    if (p.n_gist > 0) {
      prefetch_tensormap(&tmKg);
      prefetch_tensormap(&tmVg);
    }
  }
  __syncthreads();
  const bool full = p.head_full != nullptr && p.head_full[u % p.Hkv];
  if (!full && p.pdl) grid_dependency_wait();  // the selection's lists are complete
  const int n_all = unit_count(p, u);
  const int lo = static_cast<int>(static_cast<int64_t>(n_all) * rank / CS);
  const int hi = static_cast<int>(static_cast<int64_t>(n_all) * (rank + 1) / CS);
  const int STAGE_BYTES = 2 * L * D * 2;
  bool ok = true;

  if (warp == kConsumerWarps) {
    // ---------------------------------------------------------------- producer
    const KVMaps maps{&tmK, &tmV, &tmKg, &tmVg};
    const uint64_t kv_policy = l2_policy_evict_first();
    uint32_t cp_stages = 0;
    int64_t issued = 0;
    for (int g0 = lo; g0 < hi && ok; g0 += 32) {
      int row = 0, gsel = -1;
      if (g0 + lane < hi) row = unit_row(p, u, g0 + lane, L, &gsel);
      const int nb = min(32, hi - g0);
      for (int j = 0; j < nb; ++j) {
        const int row_j = __shfl_sync(0xffffffffu, row, j);
        const int gs_j = __shfl_sync(0xffffffffu, gsel, j);
        const int s = static_cast<int>(issued % NS);
        if (!issue_stage<D, L>(p, maps, issued, NS, sbase + s * STAGE_BYTES, full_bar,
                               empty_bar, row_j, gs_j, g0 + j == lo ? u : -1,
                               sbase + Y.q_off, kv_policy, cp_stages)) {
          ok = false;
          break;
        }
        ++issued;
      }
    }
    // no copy may still be landing when the CTA retires
    if (lane == 0) {
      const int64_t first = issued > NS ? issued - NS : 0;
      for (int64_t i = first; i < issued; ++i)
        mbar_wait(full_bar + 8 * static_cast<int>(i % NS), static_cast<uint32_t>(i / NS) & 1u,
                  p.err);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- consumers
    WarpAcc<D> acc;
    acc.m0 = acc.m1 = -INFINITY;
    acc.l0 = acc.l1 = 0.f;
    for (int ks = 0; ks < D / 16; ++ks)
      for (int e = 0; e < 4; ++e) acc.o[ks][e] = 0.f;
    const bool hybrid = (p.n_gist > 0 || p.gist_sel) && !full;
    const int ns_sel = hybrid ? sel_count(p, u) : 0;
    for (int g = lo; g < hi; ++g) {
      const int64_t i = g - lo;
      const int s = static_cast<int>(i % NS);
      if (!warp_wait(full_bar + 8 * s, static_cast<uint32_t>(i / NS) & 1u, p.err)) {
        ok = false;
        break;
      }
      if (g == lo)  // the unit's q arrived with the first stage
        acc_begin<D>(acc, reinterpret_cast<const __nv_bfloat16*>(smem + Y.q_off), G, lane);
      int valid = L;
      if (hybrid) {
        const int j = g - ns_sel;
        if (j >= 0) valid = min(L, gist_rows_of(p, ns_sel) - j * L);
      }
      acc_stage<D, L>(acc, sbase + s * STAGE_BYTES, warp, lane, p.scale_log2, valid);
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar + 8 * s);
    }
    acc_write<D>(acc, fo, G, warp, lane);
    mbar_arrive(fo_bar);
    const bool have = warp_wait(fo_bar, 0u, p.err);
    // this CTA's part: the four warps folded into one (M, Lsum, O) per head
    const float* fm = fo + kConsumerWarps * G * D;
    const float* fl = fm + kConsumerWarps * 8;
    cluster_wait();  // (phase 1) every CTA of the cluster is running
    const uint32_t slot = cluster_map(smem_u32(smem + Y.part_off + rank * Y.part_stride), 0);
    const int tid = threadIdx.x;  // 0 .. 127
    for (int e = tid; e < G * D && have; e += kConsumerWarps * 32) {
      const int g = e / D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, fm[w * 8 + g]);
      float O = 0.f, Ls = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float wt = fast_exp2(fm[w * 8 + g] - M);
          O += fo[(w * G + g) * D + (e % D)] * wt;
          Ls += fl[w * 8 + g] * wt;
        }
      }
      st_cluster_f32(slot + (16 + e) * 4, O);
      if (e % D == 0) {
        st_cluster_f32(slot + g * 4, M);
        st_cluster_f32(slot + (8 + g) * 4, Ls);
      }
    }
  }
  if (warp == kConsumerWarps) cluster_wait();  // (phase 1) for the producer warp
  cluster_arrive();  // (phase 2) the parts are in the first CTA's slots
  cluster_wait();
  if (rank != 0) return;
  // ---------------------------------------------------------------- the unit's rows
  const float* part = reinterpret_cast<const float*>(smem + Y.part_off);
  const int pst = Y.part_stride / 4;
  const int64_t row0 = static_cast<int64_t>(u / p.Hkv) * p.Hq + (u % p.Hkv) * G;
  for (int e = threadIdx.x; e < G * D; e += kClusterThreads) {
    const int g = e / D;
    float M = -INFINITY;
    for (int r = 0; r < CS; ++r) M = fmaxf(M, part[r * pst + g]);
    float O = 0.f, Ls = 0.f;
    if (M != -INFINITY) {
      for (int r = 0; r < CS; ++r) {
        const float wt = fast_exp2(part[r * pst + g] - M);
        O += part[r * pst + 16 + e] * wt;
        Ls += part[r * pst + 8 + g] * wt;
      }
    }
    store_out(p, row0 * D + e, Ls > 0.f ? O / Ls : 0.f);
    if (e % D == 0 && p.lse_out)
      p.lse_out[row0 + g] = Ls > 0.f ? (M + __log2f(Ls)) * kLn2 : -INFINITY;
  }
}

// ------------------------------------------------------------------ fp32 path

constexpr int kF32Threads = 128;
constexpr int kMergeWts = 2048;  // G * splits per unit in merged mode (8 * 256)

template <int D>
__global__ void __launch_bounds__(kF32Threads) decode_f32_kernel(const DecodeParams p) {
  extern __shared__ __align__(16) uint8_t smem_f[];
  float* qs = reinterpret_cast<float*>(smem_f);   // [8][D]
  float* sc = qs + 8 * D;                          // [8][128]
  float* mh = sc + 8 * 128;                        // [8]
  float* lh = mh + 8;                              // [8]
  float* ah = lh + 8;                              // [8]
  float* wts = ah + 8;                             // [kMergeWts] merge weights
  float* ks = wts + kMergeWts;                     // [L][D + 1] the chunk's keys (padded rows)
  float* vs = ks + 128 * (D + 1);                  // [L][D] its values (16-byte aligned)
  int* prefix = reinterpret_cast<int*>(vs + 128 * D);  // [U+1]
  __shared__ int scan_sh[33];
  __shared__ int last_sh;
  // split partials out: the merge kernel behind this one may become resident
  if (!p.merged) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  build_prefix(p, prefix, scan_sh);
  fill_empty_slots(p, prefix, kF32Threads);
  const int64_t N = prefix[p.U], P = gridDim.x;
  const int64_t a = N * blockIdx.x / P, bnd = N * (blockIdx.x + 1) / P;
  const int L = p.L, G = p.G;
  const int tid = threadIdx.x;
  float o[8];
  int cur_u = -1;

  auto flush = [&](int u) {
    const int b = u / p.Hkv, h = u % p.Hkv;
    const int slot = split_slot(prefix[u], a, blockIdx.x, N, P);
    const int ns = split_count(prefix[u], prefix[u + 1], N, P);
    const bool direct = p.merged && ns == 1;
    for (int g = 0; g < G; ++g) {
      const int64_t row = static_cast<int64_t>(b) * p.Hq + h * G + g;
      const float lse = (mh[g] + log2f(lh[g])) * kLn2;
      if (direct) {
        if (tid < D) store_out(p, row * D + tid, o[g] / lh[g]);
        if (tid == 0 && p.lse_out) p.lse_out[row] = lse;
      } else {
        if (tid < D) p.o_part[(row * p.max_splits + slot) * D + tid] = o[g] / lh[g];
        if (tid == 0) p.lse_part[row * p.max_splits + slot] = lse;
      }
    }
    __syncthreads();
    if (p.merged && !direct) {
      if (tid == 0) {
        __threadfence();
        last_sh = atomicAdd(p.counters + u, 1) == ns - 1;
      }
      __syncthreads();
      if (last_sh) {
        __threadfence();
        merge_unit<D, 8>(p, u, ns, wts, tid, kF32Threads, [] { __syncthreads(); return true; });
        if (tid == 0) p.counters[u] = 0;
      }
    }
    __syncthreads();
  };

  for (int64_t g = a; g < bnd; ++g) {
    if (cur_u < 0 || g >= prefix[cur_u + 1]) {
      if (cur_u >= 0) flush(cur_u);
      cur_u = unit_of(prefix, p.U, g);
      const int b = cur_u / p.Hkv, h = cur_u % p.Hkv;
      const float* qf = static_cast<const float*>(p.q);
      for (int e = tid; e < G * D; e += kF32Threads)
        qs[e] = qf[(static_cast<int64_t>(b) * p.Hq + h * G) * D + e];
      if (tid < 8) {
        mh[tid] = -INFINITY;
        lh[tid] = 0.f;
      }
#pragma unroll
      for (int x = 0; x < 8; ++x) o[x] = 0.f;
      __syncthreads();
    }
    const int u = cur_u;
    const int c = unit_chunk(p, u, static_cast<int>(g - prefix[u]));
    const int64_t row0 = u * p.T + static_cast<int64_t>(c) * L;
    {
      // the chunk's K and V rows into shared memory: 16-byte loads, up to
      // eight of each in flight per thread (one round for L = D = 64)
      constexpr int D4 = D / 4;
      const float4* kg = reinterpret_cast<const float4*>(p.Kf + row0 * D);
      const float4* vg = reinterpret_cast<const float4*>(p.Vf + row0 * D);
      const int n4 = L * D4;
      for (int e0 = 0; e0 < n4; e0 += 8 * kF32Threads) {
        float4 kv[8], vv[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int e = e0 + k * kF32Threads + tid;
          if (e < n4) {
            kv[k] = __ldg(kg + e);
            vv[k] = __ldg(vg + e);
          }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int e = e0 + k * kF32Threads + tid;
          if (e < n4) {
            float* kd = ks + (e / D4) * (D + 1) + (e % D4) * 4;
            kd[0] = kv[k].x;
            kd[1] = kv[k].y;
            kd[2] = kv[k].z;
            kd[3] = kv[k].w;
            reinterpret_cast<float4*>(vs)[e] = vv[k];
          }
        }
      }
    }
    __syncthreads();
    if (tid < L) {
      const float* kr = ks + tid * (D + 1);
      for (int x = 0; x < G; ++x) {
        float acc = 0.f;
        for (int d = 0; d < D; ++d) acc += qs[x * D + d] * kr[d];
        sc[x * 128 + tid] = acc * p.scale_log2;
      }
    }
    __syncthreads();
    if (tid < G) {
      float cm = -INFINITY;
      for (int j = 0; j < L; ++j) cm = fmaxf(cm, sc[tid * 128 + j]);
      const float mn = fmaxf(mh[tid], cm);
      ah[tid] = exp2f(mh[tid] - mn);
      mh[tid] = mn;
    }
    __syncthreads();
    if (tid < L)
      for (int x = 0; x < G; ++x) sc[x * 128 + tid] = exp2f(sc[x * 128 + tid] - mh[x]);
    __syncthreads();
    if (tid < G) {
      float s = 0.f;
      for (int j = 0; j < L; ++j) s += sc[tid * 128 + j];
      lh[tid] = lh[tid] * ah[tid] + s;
    }
    if (tid < D) {
      for (int x = 0; x < G; ++x) {
        float acc = 0.f;
        for (int j = 0; j < L; ++j) acc += sc[x * 128 + j] * vs[j * D + tid];
        o[x] = o[x] * ah[x] + acc;
      }
    }
    __syncthreads();
  }
  if (cur_u >= 0) flush(cur_u);
}

// ------------------------------------------------------------------ merge

constexpr int kMergeThreads = 128;
constexpr int kMergeWarps = kMergeThreads / 32;

// One CTA per row.  The valid slots (lse > -inf) are compacted in slot order
// with their weights exp(lse_s - lse); warp w then accumulates slots w, w+4,
// ... over its lanes' float4 columns and the four partial sums are added in
// a fixed order, so the result does not depend on timing.
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(
    const float* __restrict__ o_part, const float* __restrict__ lse_part, int rows, int S, int D,
    void* __restrict__ out, int out_bf16, float* __restrict__ lse_out) {
  extern __shared__ __align__(16) float msm[];
  float* acc_sh = msm;                                        // [kMergeWarps][D] (float4 stores)
  float* wts = msm + kMergeWarps * D;                         // [S]
  int* slots = reinterpret_cast<int*>(wts + S);               // [S]
  __shared__ int scan_sh[33];
  __shared__ float red[kMergeWarps];
  __shared__ float lse_sh;
  const int r = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* lrow = lse_part + static_cast<int64_t>(r) * S;
  // launched behind the split decode (programmatic dependent launch): the
  // CTAs wait here, resident, until its partials are complete and visible
  grid_dependency_wait();
  // row max
  float mx = -INFINITY;
  for (int s = threadIdx.x; s < S; s += kMergeThreads) mx = fmaxf(mx, lrow[s]);
#pragma unroll
  for (int x = 16; x > 0; x >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, x));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  mx = red[0];
#pragma unroll
  for (int w = 1; w < kMergeWarps; ++w) mx = fmaxf(mx, red[w]);
  __syncthreads();
  // ordered compaction of the valid slots (contiguous segments per thread)
  const int seg = (S + kMergeThreads - 1) / kMergeThreads;
  const int lo = min(S, static_cast<int>(threadIdx.x) * seg), hi = min(S, lo + seg);
  int nv = 0;
  for (int s = lo; s < hi; ++s) nv += (mx != -INFINITY && lrow[s] != -INFINITY);
  int total = 0;
  int pos = block_exclusive_scan(nv, scan_sh, &total);
  for (int s = lo; s < hi; ++s)
    if (mx != -INFINITY && lrow[s] != -INFINITY) {
      slots[pos] = s;
      wts[pos] = expf(lrow[s] - mx);
      ++pos;
    }
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
    for (int i = 0; i < total; ++i) tot += wts[i];
    lse_sh = total > 0 ? mx + logf(tot) : -INFINITY;
    if (lse_out) lse_out[r] = lse_sh;
    const float inv = total > 0 ? 1.0f / tot : 0.f;
    for (int i = 0; i < total; ++i) wts[i] *= inv;
  }
  __syncthreads();
  const int nv4 = D / 4;
  for (int v4 = lane; v4 < nv4; v4 += 32) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int i = warp;
    for (; i + 3 * kMergeWarps < total; i += 4 * kMergeWarps) {
      float4 x[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        x[k] = __ldg(reinterpret_cast<const float4*>(
                         o_part + (static_cast<int64_t>(r) * S + slots[i + k * kMergeWarps]) * D) + v4);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float wgt = wts[i + k * kMergeWarps];
        acc.x += wgt * x[k].x;
        acc.y += wgt * x[k].y;
        acc.z += wgt * x[k].z;
        acc.w += wgt * x[k].w;
      }
    }
    for (; i < total; i += kMergeWarps) {
      const float4 x = __ldg(reinterpret_cast<const float4*>(
                                 o_part + (static_cast<int64_t>(r) * S + slots[i]) * D) + v4);
      const float wgt = wts[i];
      acc.x += wgt * x.x;
      acc.y += wgt * x.y;
      acc.z += wgt * x.z;
      acc.w += wgt * x.w;
    }
    reinterpret_cast<float4*>(acc_sh + warp * D)[v4] = acc;
  }
  __syncthreads();
  for (int d = threadIdx.x; d < D; d += kMergeThreads) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) v += acc_sh[w * D + d];
    if (out_bf16)
      static_cast<__nv_bfloat16*>(out)[static_cast<int64_t>(r) * D + d] = __float2bfloat16_rn(v);
    else
      static_cast<float*>(out)[static_cast<int64_t>(r) * D + d] = v;
  }
}

template <int D, int L>
cudaError_t launch_bf16(const Launch& l, const DecodeParams& p, const void* K, const void* V,
                        const void* Kg, const void* Vg, int B, int Hkv, int P, std::string* why) {
  CUtensorMap tmK, tmV, tmKg, tmVg;
  const uint64_t rows = static_cast<uint64_t>(B) * Hkv * p.T;
  if (!make_tmap_bf16_2d(&tmK, K, rows, D, D, L, 64, why)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tmV, V, rows, D, D, L, 64, why)) return cudaErrorInvalidValue;
  if (p.n_gist > 0) {  // the gist rows: [B*Hkv*gist_rows, D], the same boxes
    const uint64_t grows = static_cast<uint64_t>(B) * Hkv * p.gist_rows;
    if (!make_tmap_bf16_2d(&tmKg, Kg, grows, D, D, L, 64, why)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16_2d(&tmVg, Vg, grows, D, D, L, 64, why)) return cudaErrorInvalidValue;
  } else {
    tmKg = tmK;
    tmVg = tmV;
  }
  const size_t sh = dec_layout(D, L, p.G, p.U).total;
  if (sh > kMaxDynSmem) {
    *why = "too many (batch, KV head) units for one decode launch: " + std::to_string(p.U);
    return cudaErrorInvalidValue;
  }
  auto fn = decode_bf16_kernel<D, L>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(sh));
  if (e != cudaSuccess) return e;
  if (!p.pdl) {
    fn<<<P, kDecodeThreads, sh, l.stream>>>(tmK, tmV, tmKg, tmVg, p);
    return cudaGetLastError();
  }
  // programmatic dependent launch: the grid may start while the selection
  // kernel before it still runs; the kernel waits (griddepcontrol.wait)
  // before it reads anything the selection writes
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P);
  cfg.blockDim = dim3(kDecodeThreads);
  cfg.dynamicSmemBytes = sh;
  cfg.stream = l.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, tmK, tmV, tmKg, tmVg, p);
}

template <int D, int L>
cudaError_t launch_cluster(const Launch& l, const DecodeParams& p, const void* K, const void* V,
                           const void* Kg, const void* Vg, int B, int Hkv, int CS,
                           std::string* why) {
  CUtensorMap tmK, tmV, tmKg, tmVg;
  const uint64_t rows = static_cast<uint64_t>(B) * Hkv * p.T;
  if (!make_tmap_bf16_2d(&tmK, K, rows, D, D, L, 64, why)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tmV, V, rows, D, D, L, 64, why)) return cudaErrorInvalidValue;
  if (p.n_gist > 0) {
    const uint64_t grows = static_cast<uint64_t>(B) * Hkv * p.gist_rows;
    if (!make_tmap_bf16_2d(&tmKg, Kg, grows, D, D, L, 64, why)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16_2d(&tmVg, Vg, grows, D, D, L, 64, why)) return cudaErrorInvalidValue;
  } else {
    tmKg = tmK;
    tmVg = tmV;
  }
  const size_t sh = cl_layout(D, L, p.G, CS).total;
  auto fn = decode_cluster_kernel<D, L>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(sh));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CS, p.U);
  cfg.blockDim = dim3(kClusterThreads);
  cfg.dynamicSmemBytes = sh;
  cfg.stream = l.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  int na = 1;
  if (p.pdl) {  // behind the selection: wait for it on the device (griddepcontrol.wait)
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    na = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, fn, tmK, tmV, tmKg, tmVg, p);
}

// Cluster size for the cluster path, or 0 for the persistent one.  Without
// full-attention heads (which the host cannot see without reading device
// memory) and with at most ~512 KB of K/V per CTA at the largest possible
// list (kmax chunks plus the gist chunks), CS is the largest power of two
// <= 8 with B*Hkv*CS CTAs on the SMs.
int cluster_size_for(const DecodeParams& p, bool head_full, int num_sms) {
  if (head_full || p.U <= 0 || p.U > 65535) return 0;
  int CS = kClusterMax;
  while (CS > 1 && static_cast<int64_t>(p.U) * CS > num_sms) CS >>= 1;
  if (static_cast<int64_t>(p.U) * CS > num_sms) return 0;
  int n_max = std::min(p.C, p.kmax);
  n_max += p.gist_sel ? (std::min(p.C, p.kmax) + p.L - 1) / p.L : p.n_gist;
  const int64_t per_cta = static_cast<int64_t>((n_max + CS - 1) / CS) * 2 * p.L * p.D * 2;
  if (per_cta > 512 * 1024) return 0;
  if (cl_layout(p.D, p.L, p.G, CS).ns < 2) return 0;
  return CS;
}

}  // namespace

int decode_default_parts(bool bf16, int D, int L, int num_sms) {
  (void)bf16;
  (void)D;
  (void)L;
  return num_sms;  // one persistent CTA per SM
}

size_t decode_f32_smem_bytes(int D, int U) {
  return static_cast<size_t>(8 * D + 8 * 128 + 24 + kMergeWts + 128 * (D + 1) + 128 * D + U + 1) *
         4;
}

cudaError_t launch_decode(const Launch& l, const void* q, const void* K, const void* V, bool bf16,
                          const int32_t* idx, const int32_t* count, int kmax,
                          const uint8_t* head_full, int B, int Hq, int Hkv, int D, int64_t T,
                          int L, float scale, int num_parts, int max_splits, float* o_part,
                          float* lse_part, const MergeOut* merge, std::string* why) {
  DecodeParams p{};
  if (merge != nullptr) {
    p.merged = 1;
    p.counters = merge->counters;
    p.out = merge->out;
    p.out_bf16 = merge->out_bf16 ? 1 : 0;
    p.lse_out = merge->lse_out;
    p.pdl = (merge->phased && bf16) ? 1 : 0;
    p.phased = p.pdl;
    p.late = p.phased ? merge->late : 0;
    if (merge->Kg != nullptr && bf16) {
      if (merge->gist_selected) {
        p.gist_sel = 1;
        p.Kg = static_cast<const __nv_bfloat16*>(merge->Kg);
        p.Vg = static_cast<const __nv_bfloat16*>(merge->Vg);
      } else {
        p.gist_rows = static_cast<int>(T / L);
        p.n_gist = (p.gist_rows + L - 1) / L;
      }
    }
  }
  p.D = D;
  p.q = q;
  p.Kf = static_cast<const float*>(K);
  p.Vf = static_cast<const float*>(V);
  p.idx = idx;
  p.count = count;
  p.kmax = kmax;
  p.head_full = head_full;
  p.U = B * Hkv;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.Hq = Hq;
  p.C = static_cast<int>(T / L);
  p.L = L;
  p.T = T;
  p.scale_log2 = scale * kLog2e;
  p.max_splits = max_splits;
  p.o_part = o_part;
  p.lse_part = lse_part;
  p.err = l.err;
  const int P = num_parts > 0 ? num_parts : decode_default_parts(bf16, D, L, l.num_sms);
  if (p.U == 0) return cudaSuccess;
  if (!bf16) {
    const size_t sh = decode_f32_smem_bytes(D, p.U);
    cudaError_t e;
    if (D == 128) {
      e = cudaFuncSetAttribute(decode_f32_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sh));
      if (e != cudaSuccess) return e;
      decode_f32_kernel<128><<<P, kF32Threads, sh, l.stream>>>(p);
    } else {
      e = cudaFuncSetAttribute(decode_f32_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sh));
      if (e != cudaSuccess) return e;
      decode_f32_kernel<64><<<P, kF32Threads, sh, l.stream>>>(p);
    }
    return cudaGetLastError();
  }
  const void* Kg = merge != nullptr ? merge->Kg : nullptr;
  const void* Vg = merge != nullptr ? merge->Vg : nullptr;
  const int CS = (merge != nullptr && merge->allow_cluster)
                     ? cluster_size_for(p, head_full != nullptr, l.num_sms)
                     : 0;
  if (CS > 0) {
    if (D == 128 && L == 128) return launch_cluster<128, 128>(l, p, K, V, Kg, Vg, B, Hkv, CS, why);
    if (D == 128 && L == 64) return launch_cluster<128, 64>(l, p, K, V, Kg, Vg, B, Hkv, CS, why);
    if (D == 64 && L == 128) return launch_cluster<64, 128>(l, p, K, V, Kg, Vg, B, Hkv, CS, why);
    return launch_cluster<64, 64>(l, p, K, V, Kg, Vg, B, Hkv, CS, why);
  }
  if (D == 128 && L == 128) return launch_bf16<128, 128>(l, p, K, V, Kg, Vg, B, Hkv, P, why);
  if (D == 128 && L == 64) return launch_bf16<128, 64>(l, p, K, V, Kg, Vg, B, Hkv, P, why);
  if (D == 64 && L == 128) return launch_bf16<64, 128>(l, p, K, V, Kg, Vg, B, Hkv, P, why);
  return launch_bf16<64, 64>(l, p, K, V, Kg, Vg, B, Hkv, P, why);
}

cudaError_t launch_merge(const Launch& l, const float* o_part, const float* lse_part, int rows,
                         int max_splits, int D, void* out, bool out_bf16, float* lse_out) {
  if (rows == 0) return cudaSuccess;
  const size_t sh = (2 * static_cast<size_t>(max_splits) + kMergeWarps * D) * 4;
  if (sh > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sh));
    if (e != cudaSuccess) return e;
  }
  // behind the kernel that writes the partials: may start early (it waits
  // on the device for that kernel to complete)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows);
  cfg.blockDim = dim3(kMergeThreads);
  cfg.dynamicSmemBytes = sh;
  cfg.stream = l.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, merge_kernel, o_part, lse_part, rows, max_splits, D, out,
                            out_bf16 ? 1 : 0, lse_out);
}

}  // namespace csa
