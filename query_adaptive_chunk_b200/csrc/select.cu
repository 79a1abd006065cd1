// Chunk selection, one CTA per unit, entirely in shared memory.
//
// Scores become order-preserving uint32 keys (0 = not a candidate).  The
// k-th largest key tau is found by an MSB-first radix select (4 passes of
// 8 bits, warp-aggregated shared-memory histograms).  The chosen set is every
// candidate with key > tau plus the first (k - #greater) candidates with key
// == tau in index order, which realises the (score desc, index asc) order
// exactly.  Results are written ascending through a block-wide scan.
//
// top-k: radix select over the non-forced chunks.
// top-p: radix select of the `budget` best chunks, a bitonic sort of just
//        those, an ordered prefix scan of their softmax mass, and a cut at the
//        first prefix reaching p (or at the budget).
// hier:  meta scores -> radix select of top_meta metas -> child scores ->
//        radix select of k_free children.
#include "internal.h"

namespace csa {
namespace {

constexpr int kSelThreads = 512;

__device__ __forceinline__ float key_to_float(uint32_t k) {
  uint32_t b = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(b);
}

struct SelScratch {
  int hist[256];
  int bcast[2];
  int scan[33];
  float fscan[33];
  int misc[4];
};

// k-th largest candidate key among keys[0, n) (0 = not a candidate);
// 1 <= k <= number of candidates.  *n_gt = candidates strictly above it.
__device__ uint32_t radix_select(const uint32_t* keys, int n, int k, SelScratch& s, int* n_gt) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0, mask = 0;
  int krem = k;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) s.hist[i] = 0;
    __syncthreads();
    for (int base = 0; base < n; base += blockDim.x) {
      const int c = base + threadIdx.x;
      const uint32_t key = c < n ? keys[c] : 0u;
      const bool valid = key != 0u && (key & mask) == prefix;
      const uint32_t bucket = (key >> shift) & 255u;
      const unsigned peers = __match_any_sync(0xffffffffu, valid ? bucket : 256u + lane);
      if (valid && lane == __ffs(peers) - 1) atomicAdd(&s.hist[bucket], __popc(peers));
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      int cnt[8], tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        cnt[i] = s.hist[255 - 8 * lane - i];
        tot += cnt[i];
      }
      int inc = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const int exc = inc - tot;
      if (exc < krem && krem <= inc) {
        int run = exc;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (run + cnt[i] >= krem) {
            s.bcast[0] = 255 - 8 * lane - i;
            s.bcast[1] = run;
            break;
          }
          run += cnt[i];
        }
      }
    }
    __syncthreads();
    krem -= s.bcast[1];
    prefix |= static_cast<uint32_t>(s.bcast[0]) << shift;
    mask |= 0xffu << shift;
    __syncthreads();
  }
  *n_gt = k - krem;
  return prefix;
}

// Mark in flags[] the candidates with key > tau and the first take_eq with
// key == tau (index order).  Threads own contiguous segments so that the
// block scan follows index order.
__device__ void mark_top(const uint32_t* keys, int n, uint32_t tau, int take_eq, uint8_t* flags,
                         SelScratch& s) {
  const int seg = (n + blockDim.x - 1) / blockDim.x;
  const int lo = min(n, static_cast<int>(threadIdx.x) * seg), hi = min(n, lo + seg);
  int eq = 0;
  for (int c = lo; c < hi; ++c) eq += keys[c] == tau;
  int rank = block_exclusive_scan(eq, s.scan, nullptr);
  for (int c = lo; c < hi; ++c) {
    const uint32_t k = keys[c];
    if (k == 0u) continue;
    if (k > tau) flags[c] = 1;
    else if (k == tau) {
      if (rank < take_eq) flags[c] = 1;
      ++rank;
    }
  }
  __syncthreads();
}

// Choose the k best candidates of keys[0, n) into flags (k clamped to the
// number of candidates n_cand).
__device__ void choose_best(const uint32_t* keys, int n, int n_cand, int k, uint8_t* flags,
                            SelScratch& s) {
  k = min(k, n_cand);
  if (k <= 0) return;
  if (k == n_cand) {
    for (int c = threadIdx.x; c < n; c += blockDim.x)
      if (keys[c] != 0u) flags[c] = 1;
    __syncthreads();
    return;
  }
  int n_gt = 0;
  const uint32_t tau = radix_select(keys, n, k, s, &n_gt);
  mark_top(keys, n, tau, k - n_gt, flags, s);
}

// Write the positions of set flags in [0, n) ascending into row[0:total],
// fill row[total:kmax] with -1 and store total.
__device__ void emit_ascending(const uint8_t* flags, int n, int32_t* row, int32_t* count,
                               int kmax, SelScratch& s) {
  const int seg = (n + blockDim.x - 1) / blockDim.x;
  const int lo = min(n, static_cast<int>(threadIdx.x) * seg), hi = min(n, lo + seg);
  int cnt = 0;
  for (int c = lo; c < hi; ++c) cnt += flags[c];
  int total = 0;
  int pos = block_exclusive_scan(cnt, s.scan, &total);
  for (int c = lo; c < hi; ++c)
    if (flags[c]) {
      if (pos < kmax) row[pos] = c;
      ++pos;
    }
  for (int i = total + threadIdx.x; i < kmax; i += blockDim.x) row[i] = -1;
  if (threadIdx.x == 0) *count = min(total, kmax);
}

__device__ __forceinline__ bool is_forced(int c, int v, int n_sink, int n_local) {
  return c < n_sink || c >= v - n_local;
}

__device__ __forceinline__ int forced_count(int v, int n_sink, int n_local) {
  const int a = min(n_sink, v);
  const int b0 = max(v - n_local, 0);
  return a + (v - b0) - max(0, a - b0);  // |[0,a) U [b0,v)|
}

__global__ void __launch_bounds__(kSelThreads) select_topk_kernel(
    const float* __restrict__ scores, int C, const int32_t* __restrict__ n_valid, int k_free,
    int n_sink, int n_local, int32_t* __restrict__ idx, int32_t* __restrict__ count, int kmax) {
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ SelScratch s;
  uint32_t* keys = reinterpret_cast<uint32_t*>(sm);
  uint8_t* flags = sm + static_cast<size_t>(C) * 4;
  const int u = blockIdx.x;
  const int v = n_valid ? max(0, min(C, n_valid[u])) : C;
  const float* row = scores + static_cast<int64_t>(u) * C;
  for (int c = threadIdx.x; c < v; c += blockDim.x) {
    const bool f = is_forced(c, v, n_sink, n_local);
    keys[c] = f ? 0u : float_key(row[c]);
    flags[c] = f ? 1 : 0;
  }
  __syncthreads();
  const int n_cand = v - forced_count(v, n_sink, n_local);
  choose_best(keys, v, n_cand, k_free, flags, s);
  emit_ascending(flags, v, idx + static_cast<int64_t>(u) * kmax, count + u, kmax, s);
}

// Block sum of one float per thread in a fixed order (deterministic).
__device__ float block_sum(float v, SelScratch& s) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) s.fscan[warp] = v;
  __syncthreads();
  float t = 0.f;
  for (int w = 0; w < nw; ++w) t += s.fscan[w];
  __syncthreads();
  return t;
}

__device__ float block_max(float v, SelScratch& s) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) s.fscan[warp] = v;
  __syncthreads();
  float t = -INFINITY;
  for (int w = 0; w < nw; ++w) t = fmaxf(t, s.fscan[w]);
  __syncthreads();
  return t;
}

// Exclusive block scan of floats, fixed order.
__device__ float block_exclusive_scan_f(float v, SelScratch& s) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  float x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s.fscan[warp] = x;
  __syncthreads();
  float base = 0.f;
  for (int w = 0; w < warp; ++w) base += s.fscan[w];
  (void)nw;
  __syncthreads();
  return base + x - v;
}

__global__ void __launch_bounds__(kSelThreads) select_topp_kernel(
    const float* __restrict__ scores, int C, float logit_scale, float p, int budget, int n_sink,
    int n_local, int32_t* __restrict__ idx, int32_t* __restrict__ count, int kmax,
    int32_t* __restrict__ n_p_out, int SN) {
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ SelScratch s;
  uint64_t* sortbuf = reinterpret_cast<uint64_t*>(sm);            // [SN]
  float* cum = reinterpret_cast<float*>(sm + static_cast<size_t>(SN) * 8);  // [SN]
  uint32_t* keys = reinterpret_cast<uint32_t*>(sm + static_cast<size_t>(SN) * 12);  // [C]
  uint8_t* flags = sm + static_cast<size_t>(SN) * 12 + static_cast<size_t>(C) * 4;  // [C]
  const int u = blockIdx.x;
  const float* row = scores + static_cast<int64_t>(u) * C;

  float mx = -INFINITY;
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    const float x = row[c];
    keys[c] = float_key(x);
    flags[c] = 0;
    mx = fmaxf(mx, x);
  }
  mx = block_max(mx, s);  // includes the __syncthreads that publishes keys
  float part = 0.f;
  for (int c = threadIdx.x; c < C; c += blockDim.x)
    part += expf((key_to_float(keys[c]) - mx) * logit_scale);
  const float Z = block_sum(part, s);

  // the nb best chunks (by score, lower index first) into flags as a pool
  const int nb = min(budget, C);
  choose_best(keys, C, C, nb, flags, s);
  // if even those nb chunks hold less than p of the mass, n_p > budget and the
  // cap decides: the pool is the answer, no ordering of it is needed
  {
    float mpart = 0.f;
    for (int c = threadIdx.x; c < C; c += blockDim.x)
      if (flags[c]) mpart += expf((key_to_float(keys[c]) - mx) * logit_scale);
    const float mass_nb = block_sum(mpart, s);
    if (nb < C && mass_nb < p * Z) {
      for (int c = threadIdx.x; c < C; c += blockDim.x)
        if (is_forced(c, C, n_sink, n_local)) flags[c] = 1;
      __syncthreads();
      if (n_p_out && threadIdx.x == 0) n_p_out[u] = nb + 1;
      emit_ascending(flags, C, idx + static_cast<int64_t>(u) * kmax, count + u, kmax, s);
      return;
    }
  }
  // compact them, in index order, into the sort buffer as 64-bit keys
  {
    const int seg = (C + blockDim.x - 1) / blockDim.x;
    const int lo = min(C, static_cast<int>(threadIdx.x) * seg), hi = min(C, lo + seg);
    int cnt = 0;
    for (int c = lo; c < hi; ++c) cnt += flags[c];
    int pos = block_exclusive_scan(cnt, s.scan, nullptr);
    for (int c = lo; c < hi; ++c)
      if (flags[c]) {
        sortbuf[pos++] = (static_cast<uint64_t>(keys[c]) << 32) | (0xffffffffu - static_cast<uint32_t>(c));
        flags[c] = 0;
      }
    for (int i = nb + threadIdx.x; i < SN; i += blockDim.x) sortbuf[i] = 0ull;
    __syncthreads();
  }
  // bitonic sort, descending: (key desc, index asc)
  for (int k = 2; k <= SN; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < SN; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint64_t a = sortbuf[i], b = sortbuf[ixj];
          const bool desc = (i & k) == 0;
          if (desc ? (a < b) : (a > b)) {
            sortbuf[i] = b;
            sortbuf[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  // ordered inclusive prefix of the softmax mass (unnormalised), first n with cum >= p*Z
  {
    const int seg = (nb + blockDim.x - 1) / blockDim.x;
    const int lo = min(nb, static_cast<int>(threadIdx.x) * seg), hi = min(nb, lo + seg);
    float loc = 0.f;
    for (int i = lo; i < hi; ++i) {
      const float x = key_to_float(static_cast<uint32_t>(sortbuf[i] >> 32));
      loc += expf((x - mx) * logit_scale);
      cum[i] = loc;
    }
    const float base = block_exclusive_scan_f(loc, s);
    if (threadIdx.x == 0) s.misc[0] = 0x7fffffff;
    __syncthreads();
    const float target = p * Z;
    for (int i = lo; i < hi; ++i) {
      cum[i] += base;
      if (cum[i] >= target) {
        atomicMin(&s.misc[0], i);
        break;
      }
    }
    __syncthreads();
  }
  const int first = s.misc[0];
  const bool found = first != 0x7fffffff;
  const int n_take = found ? first + 1 : nb;
  for (int i = threadIdx.x; i < n_take; i += blockDim.x)
    flags[0xffffffffu - static_cast<uint32_t>(sortbuf[i] & 0xffffffffull)] = 1;
  for (int c = threadIdx.x; c < C; c += blockDim.x)
    if (is_forced(c, C, n_sink, n_local)) flags[c] = 1;
  __syncthreads();
  if (n_p_out && threadIdx.x == 0) n_p_out[u] = found ? first + 1 : (nb < C ? nb + 1 : C);
  emit_ascending(flags, C, idx + static_cast<int64_t>(u) * kmax, count + u, kmax, s);
}

// Group-summed dot products of `nrows` rows (row ids rows[i], or i when rows
// is null) of a [*, D] fp32 matrix with qs, into keys (0 where skip(c)).
template <bool kSkipForced>
__device__ void score_rows(const float* __restrict__ mat, int D, const float* qs, const int* rows,
                           int nrows, uint32_t* keys, int C, int n_sink, int n_local) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  constexpr int BATCH = 8;
  for (int i0 = warp * BATCH; i0 < nrows; i0 += nw * BATCH) {
    float4 v[BATCH];
#pragma unroll
    for (int b = 0; b < BATCH; ++b) {
      const int i = i0 + b;
      v[b] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < nrows && lane * 4 < D) {
        const int r = rows ? rows[i] : i;
        v[b] = __ldg(reinterpret_cast<const float4*>(mat + static_cast<int64_t>(r) * D) + lane);
      }
    }
    // D == 128: one float4 per lane; D == 64: lanes 0..15
    const float4 q4 = lane * 4 < D ? make_float4(qs[lane * 4], qs[lane * 4 + 1], qs[lane * 4 + 2],
                                                 qs[lane * 4 + 3])
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int b = 0; b < BATCH; ++b) {
      float x = v[b].x * q4.x + v[b].y * q4.y + v[b].z * q4.z + v[b].w * q4.w;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      const int i = i0 + b;
      if (lane == 0 && i < nrows) {
        const int r = rows ? rows[i] : i;
        keys[i] = (kSkipForced && is_forced(r, C, n_sink, n_local)) ? 0u : float_key(x);
      }
    }
  }
}

__global__ void __launch_bounds__(kSelThreads) select_hier_kernel(
    const void* __restrict__ q, int q_bf16, const float* __restrict__ meta,
    const float* __restrict__ summ, int Hq, int Hkv, int D, int C, int Gm, int top_meta,
    int k_free, int n_sink, int n_local, int32_t* __restrict__ idx, int32_t* __restrict__ count,
    int kmax) {
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ SelScratch s;
  __shared__ float qs[128];
  const int M = C / Gm;
  const int k1 = min(top_meta, M);
  const int NCH = k1 * Gm;
  uint32_t* mkeys = reinterpret_cast<uint32_t*>(sm);                        // [M]
  int* clist = reinterpret_cast<int*>(sm + static_cast<size_t>(M) * 4);     // [NCH]
  uint32_t* ckeys = reinterpret_cast<uint32_t*>(clist + NCH);              // [NCH]
  int* mlist = reinterpret_cast<int*>(ckeys + NCH);                         // [k1]
  uint8_t* mflags = reinterpret_cast<uint8_t*>(mlist + k1);                 // [M]
  uint8_t* cflags = mflags + M;                                             // [NCH]
  uint8_t* flags = cflags + NCH;                                            // [C]

  const int u = blockIdx.x;
  const int h = u % Hkv, b = u / Hkv;
  const int G = Hq / Hkv;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    for (int g = 0; g < G; ++g) {
      const int64_t off = (static_cast<int64_t>(b) * Hq + h * G + g) * D + d;
      acc += q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(q)[off])
                    : static_cast<const float*>(q)[off];
    }
    qs[d] = acc;
  }
  for (int i = threadIdx.x; i < M; i += blockDim.x) mflags[i] = 0;
  for (int i = threadIdx.x; i < NCH; i += blockDim.x) cflags[i] = 0;
  for (int c = threadIdx.x; c < C; c += blockDim.x) flags[c] = is_forced(c, C, n_sink, n_local);
  __syncthreads();

  // level 1: meta-chunks
  score_rows<false>(meta + static_cast<int64_t>(u) * M * D, D, qs, nullptr, M, mkeys, C, 0, 0);
  __syncthreads();
  choose_best(mkeys, M, M, k1, mflags, s);
  {  // ascending list of kept metas -> ascending list of their children
    const int seg = (M + blockDim.x - 1) / blockDim.x;
    const int lo = min(M, static_cast<int>(threadIdx.x) * seg), hi = min(M, lo + seg);
    int cnt = 0;
    for (int m = lo; m < hi; ++m) cnt += mflags[m];
    int pos = block_exclusive_scan(cnt, s.scan, nullptr);
    for (int m = lo; m < hi; ++m)
      if (mflags[m]) mlist[pos++] = m;
    __syncthreads();
    for (int i = threadIdx.x; i < NCH; i += blockDim.x) clist[i] = mlist[i / Gm] * Gm + (i % Gm);
    __syncthreads();
  }
  // level 2: children of the kept metas, forced chunks excluded from the pool
  score_rows<true>(summ + static_cast<int64_t>(u) * C * D, D, qs, clist, NCH, ckeys, C, n_sink,
                   n_local);
  __syncthreads();
  int n_cand = 0;
  {
    int loc = 0;
    for (int i = threadIdx.x; i < NCH; i += blockDim.x) loc += ckeys[i] != 0u;
    int tot = 0;
    block_exclusive_scan(loc, s.scan, &tot);
    n_cand = tot;
  }
  choose_best(ckeys, NCH, n_cand, k_free, cflags, s);
  for (int i = threadIdx.x; i < NCH; i += blockDim.x)
    if (cflags[i]) flags[clist[i]] = 1;
  __syncthreads();
  emit_ascending(flags, C, idx + static_cast<int64_t>(u) * kmax, count + u, kmax, s);
}

int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

cudaError_t set_smem(const void* fn, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bytes));
}

}  // namespace

cudaError_t launch_select_topk(const Launch& l, const float* scores, int U, int C,
                               const int32_t* n_valid, int k_free, int n_sink, int n_local,
                               int32_t* idx, int32_t* count, int kmax) {
  if (U == 0) return cudaSuccess;
  const size_t sh = static_cast<size_t>(C) * 5 + 16;
  cudaError_t e = set_smem(reinterpret_cast<const void*>(select_topk_kernel), sh);
  if (e != cudaSuccess) return e;
  select_topk_kernel<<<U, kSelThreads, sh, l.stream>>>(scores, C, n_valid, k_free, n_sink, n_local,
                                                       idx, count, kmax);
  return cudaGetLastError();
}

cudaError_t launch_select_topp(const Launch& l, const float* scores, int U, int C,
                               float logit_scale, float p, int budget, int n_sink, int n_local,
                               int32_t* idx, int32_t* count, int kmax, int32_t* n_p_out) {
  if (U == 0) return cudaSuccess;
  const int SN = next_pow2(std::min(budget, C));
  const size_t sh = static_cast<size_t>(SN) * 12 + static_cast<size_t>(C) * 5 + 16;
  cudaError_t e = set_smem(reinterpret_cast<const void*>(select_topp_kernel), sh);
  if (e != cudaSuccess) return e;
  select_topp_kernel<<<U, kSelThreads, sh, l.stream>>>(scores, C, logit_scale, p, budget, n_sink,
                                                       n_local, idx, count, kmax, n_p_out, SN);
  return cudaGetLastError();
}

cudaError_t launch_select_hier(const Launch& l, const void* q, bool bf16, const float* meta,
                               const float* summ, int B, int Hq, int Hkv, int D, int C, int Gm,
                               int top_meta, int k_free, int n_sink, int n_local, int32_t* idx,
                               int32_t* count, int kmax) {
  const int U = B * Hkv;
  if (U == 0) return cudaSuccess;
  const int M = C / Gm;
  const int k1 = std::min(top_meta, M);
  const int NCH = k1 * Gm;
  const size_t sh = static_cast<size_t>(M) * 5 + static_cast<size_t>(NCH) * 9 +
                    static_cast<size_t>(k1) * 4 + static_cast<size_t>(C) + 16;
  cudaError_t e = set_smem(reinterpret_cast<const void*>(select_hier_kernel), sh);
  if (e != cudaSuccess) return e;
  select_hier_kernel<<<U, kSelThreads, sh, l.stream>>>(q, bf16 ? 1 : 0, meta, summ, Hq, Hkv, D, C,
                                                       Gm, top_meta, k_free, n_sink, n_local, idx,
                                                       count, kmax);
  return cudaGetLastError();
}

}  // namespace csa
