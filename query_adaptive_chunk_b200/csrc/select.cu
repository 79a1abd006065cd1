// Chunk selection, one CTA per unit, entirely on chip.
//
// Scores become order-preserving uint32 keys (0 = not a candidate) and
// 64-bit composites (key << 32 | ~index), whose descending order is exactly
// (score desc, index asc).
//
// Up to 2048 candidates (every workload here): a register-resident bitonic
// sort of the composites (shuffles inside a warp, shared memory only for the
// cross-warp stages) gives the order directly.
//   top-k: the first k_free sort positions of the non-forced chunks;
//   top-p: an ordered block scan of exp((s - max) * scale) over the first
//          `budget` positions; the cut is the first position whose prefix
//          reaches p * Z (Z from a fixed-order (max, sum-exp) reduction), or
//          the budget when none does;
//   hier:  the same sort-and-mark for the metas, then for their children.
// Larger C falls back to an MSB-first radix select (4 passes of 8 bits over
// shared-memory histograms) that finds the k-th key, keeps the keys above it
// and the first of the equal keys in index order.
// Results are written ascending through a block-wide scan of per-chunk flags.
#include "internal.h"

namespace csa {
namespace {

constexpr int kSelThreads = 512;

// Shared-memory exchange buffer of the register sort (0 when C is too large
// for it): one 64-bit slot per sort position, at least one per thread.
__host__ __device__ __forceinline__ int sort_exch_bytes(int C) {
  int p = 1;
  while (p < C) p <<= 1;
  if (p > 2048) return 0;
  return 8 * (p < kSelThreads ? kSelThreads : p);
}

// Lets a grid launched behind this one with programmatic dependent launch
// start now; that grid still waits for this one's completion before it reads
// what this one writes.
__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Waits until the grid this one was launched behind (programmatic dependent
// launch) has completed and its writes are visible; returns at once otherwise.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ float key_to_float(uint32_t k) {
  uint32_t b = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(b);
}

struct __align__(16) SelScratch {
  int hist[256];
  int bcast[2];
  int scan[33];
  float fscan[33];
  int misc[4];
};

// Bucket-select scratch (see bucket_mark).
constexpr int kBuckets = 1024;
constexpr int kBoundaryMax = 256;

struct BucketScratch {
  int hist[kBuckets];
  uint64_t bnd[kBoundaryMax];
  int n_bnd, above, bstar;
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
      // lane j owns buckets 255-8j down to 248-8j (two 16-byte reads)
      const int4 hi = reinterpret_cast<const int4*>(s.hist)[(252 - 8 * lane) >> 2];
      const int4 lo = reinterpret_cast<const int4*>(s.hist)[(248 - 8 * lane) >> 2];
      const int cnt[8] = {hi.w, hi.z, hi.y, hi.x, lo.w, lo.z, lo.y, lo.x};
      int tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) tot += cnt[i];
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

__device__ __forceinline__ float key_to_float(uint32_t k);
__device__ float block_sum(float v, SelScratch& s);

// Mark in flags[] the candidates with key > tau and the first take_eq with
// key == tau (index order).  Threads own contiguous segments so that the
// block scan follows index order.  With mass != null, also returns the sum
// of exp((score - mx) * scale) over the marked candidates.
__device__ void mark_top(const uint32_t* keys, int n, uint32_t tau, int take_eq, uint8_t* flags,
                         SelScratch& s, float* mass = nullptr, float mx = 0.f, float scale = 0.f) {
  const int seg = (n + blockDim.x - 1) / blockDim.x;
  const int lo = min(n, static_cast<int>(threadIdx.x) * seg), hi = min(n, lo + seg);
  int eq = 0;
  for (int c = lo; c < hi; ++c) eq += keys[c] == tau;
  int rank = block_exclusive_scan(eq, s.scan, nullptr);
  float m = 0.f;
  for (int c = lo; c < hi; ++c) {
    const uint32_t k = keys[c];
    if (k == 0u) continue;
    bool take = false;
    if (k > tau) take = true;
    else if (k == tau) {
      take = rank < take_eq;
      ++rank;
    }
    if (take) {
      flags[c] = 1;
      if (mass) m += expf((key_to_float(k) - mx) * scale);
    }
  }
  if (mass) *mass = block_sum(m, s);  // ends with a barrier
  else __syncthreads();
}

// Choose the k best candidates of keys[0, n) into flags (k clamped to the
// number of candidates n_cand); optionally the softmax mass of the chosen.
__device__ void choose_best(const uint32_t* keys, int n, int n_cand, int k, uint8_t* flags,
                            SelScratch& s, float* mass = nullptr, float mx = 0.f,
                            float scale = 0.f) {
  k = min(k, n_cand);
  if (k <= 0) {
    if (mass) *mass = 0.f;
    return;
  }
  if (k == n_cand) {
    mark_top(keys, n, 0u, 0, flags, s, mass, mx, scale);  // every non-zero key is > 0
    return;
  }
  int n_gt = 0;
  const uint32_t tau = radix_select(keys, n, k, s, &n_gt);
  mark_top(keys, n, tau, k - n_gt, flags, s, mass, mx, scale);
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

// Top-k over keys[0, v) already loaded (forced chunks: key 0, flag 1).
__device__ bool try_sorted_mark(const uint32_t* keys, uint8_t* flags, int v, int k_take,
                                uint64_t* exch);

__device__ void mark_best(const uint32_t* keys, uint8_t* flags, int n, int n_cand, int k,
                          uint64_t* exch, BucketScratch& bs, SelScratch& s);

__device__ void topk_from_keys(const uint32_t* keys, uint8_t* flags, int v, int n_sink,
                               int n_local, int k_free, int32_t* row, int32_t* cnt, int kmax,
                               SelScratch& s, uint64_t* exch, BucketScratch& bs) {
  const int n_cand = v - forced_count(v, n_sink, n_local);
  mark_best(keys, flags, v, n_cand, k_free, exch, bs, s);
  emit_ascending(flags, v, row, cnt, kmax, s);
}

// Causal prefill units (causal_tiles > 0): unit u is query tile t = u mod
// causal_tiles, which sees the chunks c < ((t + 1) * tile_m - 1) / L + 1.
struct CausalRows {
  int tiles, tile_m, L;
};

__global__ void __launch_bounds__(kSelThreads) select_topk_kernel(
    const float* __restrict__ scores, int C, const int32_t* __restrict__ n_valid, int k_free,
    int n_sink, int n_local, int32_t* __restrict__ idx, int32_t* __restrict__ count, int kmax,
    const int32_t* __restrict__ k_dev, CausalRows causal) {
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ SelScratch s;
  __shared__ BucketScratch bs;
  const int exch_bytes = sort_exch_bytes(C);
  uint64_t* exch = exch_bytes ? reinterpret_cast<uint64_t*>(sm) : nullptr;
  uint32_t* keys = reinterpret_cast<uint32_t*>(sm + exch_bytes);
  uint8_t* flags = sm + exch_bytes + static_cast<size_t>(C) * 4;
  const int u = blockIdx.x;
  int v = n_valid ? max(0, min(C, n_valid[u])) : C;
  if (causal.tiles > 0) {
    const int64_t t = u % causal.tiles;
    const int64_t vis = ((t + 1) * causal.tile_m - 1) / causal.L + 1;
    v = static_cast<int>(vis < C ? vis : C);
  }
  const float* row = scores + static_cast<int64_t>(u) * C;
  for (int c = threadIdx.x; c < v; c += blockDim.x) {
    const bool f = is_forced(c, v, n_sink, n_local);
    keys[c] = f ? 0u : float_key(row[c]);
    flags[c] = f ? 1 : 0;
  }
  __syncthreads();
  // k_dev: a per-unit k computed on the device (token budgets), else k_free
  const int k = k_dev ? max(0, min(k_dev[u], kmax)) : k_free;
  topk_from_keys(keys, flags, v, n_sink, n_local, k, idx + static_cast<int64_t>(u) * kmax,
                 count + u, kmax, s, exch, bs);
}

// Block sum of one float per thread in a fixed order (deterministic): a
// warp xor-tree, then every warp reduces the per-warp totals the same way.
__device__ float block_sum(float v, SelScratch& s) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) s.fscan[warp] = v;
  __syncthreads();
  float t = lane < nw ? s.fscan[lane] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  __syncthreads();
  return t;
}


// Running (max m, sum s of exp((x - m) * scale)) of a stream of scores.
__device__ __forceinline__ void ms_add(float& m, float& sum, float x, float scale) {
  if (x > m) {
    sum = sum * expf((m - x) * scale) + 1.f;
    m = x;
  } else {
    sum += expf((x - m) * scale);
  }
}

__device__ __forceinline__ void ms_merge(float& m, float& sum, float m2, float s2, float scale) {
  if (m2 == -INFINITY) return;
  if (m == -INFINITY) {
    m = m2;
    sum = s2;
    return;
  }
  const float M = fmaxf(m, m2);
  sum = sum * expf((m - M) * scale) + s2 * expf((m2 - M) * scale);
  m = M;
}

// Block-wide (max, sum-exp) in a fixed tree order; every thread gets the result.
__device__ void block_max_sumexp(float& m, float& sum, float scale, SelScratch& s) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, sum, o);
    ms_merge(m, sum, m2, s2, scale);
  }
  if (lane == 0) {
    s.fscan[warp] = m;
    s.fscan[16 + warp] = sum;
  }
  __syncthreads();
  m = lane < nw ? s.fscan[lane] : -INFINITY;
  sum = lane < nw ? s.fscan[16 + lane] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, sum, o);
    ms_merge(m, sum, m2, s2, scale);
  }
  __syncthreads();
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

// Top-p over keys[0, C) already loaded (every chunk a candidate, flags 0)
// with mx = the largest score.
// ---------------------------------------------------------------- register bitonic sort
//
// For up to 2048 candidates the whole selection is a sort: thread t holds
// the E = SN/256 consecutive sort positions t*E .. t*E+E-1 in registers as
// 64-bit composites (score key << 32 | ~index), so descending order is
// (score desc, index asc) and 0 marks padding or an excluded chunk.  Stages
// whose partner is in the same thread need nothing, partners in another
// lane of the warp come by shuffle, and only partners in another warp go
// through shared memory with a barrier (6 of the 55 stages at SN = 1024).

constexpr int kSortedMax = 2048;

__device__ __forceinline__ uint64_t composite(uint32_t key, int c) {
  return key ? ((static_cast<uint64_t>(key) << 32) | (0xffffffffu - static_cast<uint32_t>(c))) : 0ull;
}
__device__ __forceinline__ int comp_index(uint64_t v) {
  return static_cast<int>(0xffffffffu - static_cast<uint32_t>(v & 0xffffffffull));
}
__device__ __forceinline__ uint32_t comp_key(uint64_t v) { return static_cast<uint32_t>(v >> 32); }

__device__ __forceinline__ int pow2_at_least(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

template <int E>
__device__ void bitonic_desc(uint64_t (&v)[E], uint64_t* exch, int SN) {
  const int tid = threadIdx.x, lane = tid & 31;
  for (int k = 2; k <= SN; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j < E) {
        // partner in this thread: unrolled per stride so indices are constants
#pragma unroll
        for (int jj = 1; jj < E; jj <<= 1) {
          if (jj != j) continue;
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const int pe = e ^ jj;
            if (pe > e) {
              const bool desc = ((tid * E + e) & k) == 0;
              const uint64_t a = v[e], b = v[pe];
              if (desc ? (a < b) : (a > b)) {
                v[e] = b;
                v[pe] = a;
              }
            }
          }
        }
      } else if (j < 32 * E) {
        const int lm = j / E;
        const bool lower = (lane & lm) == 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const uint64_t o = __shfl_xor_sync(0xffffffffu, v[e], lm);
          const bool keep_max = (((tid * E + e) & k) == 0) == lower;
          v[e] = keep_max ? (v[e] > o ? v[e] : o) : (v[e] < o ? v[e] : o);
        }
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) exch[tid * E + e] = v[e];
        __syncthreads();
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = tid * E + e;
          const uint64_t o = exch[i ^ j];
          const bool keep_max = ((i & k) == 0) == ((i & j) == 0);
          v[e] = keep_max ? (v[e] > o ? v[e] : o) : (v[e] < o ? v[e] : o);
        }
        __syncthreads();
      }
    }
  }
}

// Mark in flags the k_take best of keys[0, v) (0 = excluded) by sorting.
template <int E>
__device__ void sorted_mark(const uint32_t* keys, uint8_t* flags, int v, int k_take,
                            uint64_t* exch) {
  const int SN = pow2_at_least(max(v, 1));
  uint64_t x[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int c = threadIdx.x * E + e;
    x[e] = c < v ? composite(keys[c], c) : 0ull;
  }
  bitonic_desc<E>(x, exch, SN);
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (static_cast<int>(threadIdx.x) * E + e < k_take && x[e] != 0ull) flags[comp_index(x[e])] = 1;
  __syncthreads();
}

// Dispatch on the sort width; false (nothing done) when v is too large.
__device__ bool try_sorted_mark(const uint32_t* keys, uint8_t* flags, int v, int k_take,
                                uint64_t* exch) {
  const int SN = pow2_at_least(max(v, 1));
  if (exch == nullptr || SN > kSortedMax) return false;
  // E sort positions per thread: E * blockDim.x >= SN, and the exchange
  // buffer holds E * blockDim.x = max(SN, blockDim.x) entries
  const int E = SN <= static_cast<int>(blockDim.x) ? 1 : SN / static_cast<int>(blockDim.x);
  if (E == 1) sorted_mark<1>(keys, flags, v, k_take, exch);
  else if (E == 2) sorted_mark<2>(keys, flags, v, k_take, exch);
  else if (E == 4) sorted_mark<4>(keys, flags, v, k_take, exch);
  else sorted_mark<8>(keys, flags, v, k_take, exch);
  return true;
}

// ---------------------------------------------------------------- bucket select
//
// Top-k without ordering the whole set: scores are binned linearly between
// their min and max (the map x -> floor((x - lo) * NB / (hi - lo)) is
// monotone, and equal scores share a bin), one shared-memory histogram and
// one descending scan find the bin b* holding the k-th best; every chunk in
// a higher bin is chosen, and only the few chunks of bin b* are ranked
// exactly by (key desc, index asc).  Degenerate inputs (all candidates
// equal, or too many in one bin) report false and the caller sorts.


__device__ void block_minmax(float& lo, float& hi, SelScratch& s) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    s.fscan[warp] = lo;
    s.fscan[16 + warp] = hi;
  }
  __syncthreads();
  lo = lane < nw ? s.fscan[lane] : INFINITY;
  hi = lane < nw ? s.fscan[16 + lane] : -INFINITY;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  __syncthreads();
}

__device__ __forceinline__ int bucket_of(float x, float lo, float scale) {
  return min(kBuckets - 1, static_cast<int>((x - lo) * scale));
}

// Marks in flags the k_take best of keys[0, v) (0 = excluded); returns
// false when the input is degenerate for binning (flags then hold a subset
// of the answer, which a sort on top completes).
__device__ bool bucket_mark(const uint32_t* keys, uint8_t* flags, int v, int k_take,
                            BucketScratch& bs, SelScratch& s) {
  if (k_take <= 0) return true;
  float lo = INFINITY, hi = -INFINITY;
  for (int c = threadIdx.x; c < v; c += blockDim.x)
    if (keys[c]) {
      const float x = key_to_float(keys[c]);
      lo = fminf(lo, x);
      hi = fmaxf(hi, x);
    }
  for (int b = threadIdx.x; b < kBuckets; b += blockDim.x) bs.hist[b] = 0;
  if (threadIdx.x == 0) {
    bs.n_bnd = 0;
    bs.bstar = -1;
  }
  block_minmax(lo, hi, s);  // barriers also publish the cleared histogram
  if (!(hi > lo)) return false;
  const float scale = static_cast<float>(kBuckets) / (hi - lo);
  if (!(scale < INFINITY)) return false;
  for (int c = threadIdx.x; c < v; c += blockDim.x)
    if (keys[c]) atomicAdd(&bs.hist[bucket_of(key_to_float(keys[c]), lo, scale)], 1);
  __syncthreads();
  // descending scan over the bins: thread t owns bins NB-1-t*seg down to NB-(t+1)*seg
  const int seg = kBuckets / blockDim.x;
  const int top = kBuckets - 1 - static_cast<int>(threadIdx.x) * seg;
  int loc = 0;
  for (int i = 0; i < seg; ++i) loc += bs.hist[top - i];
  const int exc = block_exclusive_scan(loc, s.scan, nullptr);
  if (exc < k_take && k_take <= exc + loc) {
    int run = exc;
    for (int i = 0; i < seg; ++i) {
      const int h = bs.hist[top - i];
      if (run + h >= k_take) {
        bs.bstar = top - i;
        bs.above = run;
        break;
      }
      run += h;
    }
  }
  __syncthreads();
  const int bstar = bs.bstar;
  if (bstar < 0) return false;
  for (int c = threadIdx.x; c < v; c += blockDim.x) {
    const uint32_t k = keys[c];
    if (!k) continue;
    const int b = bucket_of(key_to_float(k), lo, scale);
    if (b > bstar) {
      flags[c] = 1;
    } else if (b == bstar) {
      const int pos = atomicAdd(&bs.n_bnd, 1);
      if (pos < kBoundaryMax) bs.bnd[pos] = composite(k, c);
    }
  }
  __syncthreads();
  const int m = bs.n_bnd, need = k_take - bs.above;
  if (m > kBoundaryMax) return false;
  for (int j = threadIdx.x; j < m; j += blockDim.x) {
    const uint64_t mine = bs.bnd[j];
    int rank = 0;
    for (int i = 0; i < m; ++i) rank += bs.bnd[i] > mine;
    if (rank < need) flags[comp_index(mine)] = 1;
  }
  __syncthreads();
  return true;
}

// Top-p by sorting all C chunks: the ordered prefix mass over the first
// nb = min(budget, C) sort positions is a block scan; the cut is the first
// position where it reaches p * Z, or nb when it never does.
template <int E>
__device__ void sorted_topp(const uint32_t* keys, uint8_t* flags, int C, float mx, float Z,
                            float logit_scale, float p, int budget, int n_sink, int n_local,
                            uint64_t* exch, int32_t* row, int32_t* cnt, int kmax,
                            int32_t* n_p_slot, SelScratch& s) {
  const int SN = pow2_at_least(C);
  uint64_t x[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int c = threadIdx.x * E + e;
    x[e] = c < C ? composite(keys[c], c) : 0ull;
  }
  bitonic_desc<E>(x, exch, SN);
  const int nb = min(budget, C);
  float ev[E];
  float loc = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int r = threadIdx.x * E + e;
    ev[e] = (r < nb && x[e] != 0ull) ? expf((key_to_float(comp_key(x[e])) - mx) * logit_scale) : 0.f;
    loc += ev[e];
  }
  if (threadIdx.x == 0) s.misc[0] = 0x7fffffff;
  float run = block_exclusive_scan_f(loc, s);  // its barriers also publish misc[0]
  const float target = p * Z;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    run += ev[e];
    const int r = threadIdx.x * E + e;
    if (r < nb && run >= target) {
      atomicMin(&s.misc[0], r);
      break;
    }
  }
  __syncthreads();
  const int first = s.misc[0];
  const bool found = first != 0x7fffffff;
  const int n_take = found ? first + 1 : nb;
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (static_cast<int>(threadIdx.x) * E + e < n_take && x[e] != 0ull) flags[comp_index(x[e])] = 1;
  for (int c = threadIdx.x; c < C; c += blockDim.x)
    if (is_forced(c, C, n_sink, n_local)) flags[c] = 1;
  __syncthreads();
  if (n_p_slot && threadIdx.x == 0) *n_p_slot = found ? first + 1 : (nb < C ? nb + 1 : C);
  emit_ascending(flags, C, row, cnt, kmax, s);
}

__device__ bool try_sorted_topp(const uint32_t* keys, uint8_t* flags, int C, float mx, float Z,
                                float logit_scale, float p, int budget, int n_sink, int n_local,
                                uint64_t* exch, int32_t* row, int32_t* cnt, int kmax,
                                int32_t* n_p_slot, SelScratch& s) {
  const int SN = pow2_at_least(C);
  if (SN > kSortedMax) return false;
  const int E = SN <= static_cast<int>(blockDim.x) ? 1 : SN / static_cast<int>(blockDim.x);
  if (E == 1)
    sorted_topp<1>(keys, flags, C, mx, Z, logit_scale, p, budget, n_sink, n_local, exch, row, cnt, kmax, n_p_slot, s);
  else if (E == 2)
    sorted_topp<2>(keys, flags, C, mx, Z, logit_scale, p, budget, n_sink, n_local, exch, row, cnt, kmax, n_p_slot, s);
  else if (E == 4)
    sorted_topp<4>(keys, flags, C, mx, Z, logit_scale, p, budget, n_sink, n_local, exch, row, cnt, kmax, n_p_slot, s);
  else
    sorted_topp<8>(keys, flags, C, mx, Z, logit_scale, p, budget, n_sink, n_local, exch, row, cnt, kmax, n_p_slot, s);
  return true;
}

// Mark the k best of keys[0, n) (n_cand candidates, 0 = excluded): bucket
// select, else a register sort (n <= 2048), else radix select.
__device__ void mark_best(const uint32_t* keys, uint8_t* flags, int n, int n_cand, int k,
                          uint64_t* exch, BucketScratch& bs, SelScratch& s) {
  const int k_take = min(k, n_cand);
  if (k_take <= 0) return;
  if (k_take >= n_cand) {
    for (int c = threadIdx.x; c < n; c += blockDim.x)
      if (keys[c]) flags[c] = 1;
    __syncthreads();
    return;
  }
  if (bucket_mark(keys, flags, n, k_take, bs, s)) return;
  if (try_sorted_mark(keys, flags, n, k_take, exch)) return;
  choose_best(keys, n, n_cand, k_take, flags, s);
}

// Bytes before the keys in the top-p kernels' shared memory: the register
// sort's exchange buffer when C is small enough, else the radix path's
// sort buffer and prefix array for the budget's SN entries.
__host__ __device__ __forceinline__ size_t topp_head_bytes(int C, int SN) {
  const int ex = sort_exch_bytes(C);
  const size_t radix = static_cast<size_t>(SN) * 12;
  return ex ? (static_cast<size_t>(ex) > radix ? static_cast<size_t>(ex) : radix) : radix;
}

// Top-p over keys[0, C) already loaded (every chunk a candidate, flags 0),
// mx = the largest score, Z = sum_c exp((score_c - mx) * logit_scale).
__device__ void topp_from_keys(const uint32_t* keys, uint8_t* flags, uint64_t* sortbuf,
                               float* cum, int C, float mx, float Z, float logit_scale, float p,
                               int budget, int n_sink, int n_local, int32_t* idx, int32_t* count,
                               int kmax, int32_t* n_p_out, int SN, int u, SelScratch& s) {
  // the nb best chunks (by score, lower index first) into flags as a pool,
  // with their softmax mass
  const int nb = min(budget, C);
  float mass_nb = 0.f;
  choose_best(keys, C, C, nb, flags, s, &mass_nb, mx, logit_scale);
  // if even those nb chunks hold less than p of the mass, n_p > budget and the
  // cap decides: the pool is the answer, no ordering of it is needed
  if (nb < C && mass_nb < p * Z) {
    for (int c = threadIdx.x; c < C; c += blockDim.x)
      if (is_forced(c, C, n_sink, n_local)) flags[c] = 1;
    __syncthreads();
    if (n_p_out && threadIdx.x == 0) n_p_out[u] = nb + 1;
    emit_ascending(flags, C, idx + static_cast<int64_t>(u) * kmax, count + u, kmax, s);
    return;
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


// Top-p driver: when the budget caps the prefix (the usual case on long
// contexts) the answer is the budget's best set, found by bucket select,
// whose mass is checked against p; only when that set reaches p is the exact
// ordered prefix needed, from a sort (or the radix path beyond 2048 chunks).
__device__ void topp_select(const uint32_t* keys, uint8_t* flags, uint64_t* sortbuf, float* cum,
                            int C, float mx, float Z, float logit_scale, float p, int budget,
                            int n_sink, int n_local, int32_t* idx, int32_t* count, int kmax,
                            int32_t* n_p_out, int SN, int u, SelScratch& s, BucketScratch& bs) {
  const int nb = min(budget, C);
  int32_t* row = idx + static_cast<int64_t>(u) * kmax;
  if (nb < C && bucket_mark(keys, flags, C, nb, bs, s)) {
    float m = 0.f;
    for (int c = threadIdx.x; c < C; c += blockDim.x)
      if (flags[c]) m += expf((key_to_float(keys[c]) - mx) * logit_scale);
    const float mass_nb = block_sum(m, s);
    if (mass_nb < p * Z) {
      for (int c = threadIdx.x; c < C; c += blockDim.x)
        if (is_forced(c, C, n_sink, n_local)) flags[c] = 1;
      __syncthreads();
      if (n_p_out && threadIdx.x == 0) n_p_out[u] = nb + 1;
      emit_ascending(flags, C, row, count + u, kmax, s);
      return;
    }
  }
  for (int c = threadIdx.x; c < C; c += blockDim.x) flags[c] = 0;
  __syncthreads();
  if (try_sorted_topp(keys, flags, C, mx, Z, logit_scale, p, budget, n_sink, n_local, sortbuf, row,
                      count + u, kmax, n_p_out ? n_p_out + u : nullptr, s))
    return;
  topp_from_keys(keys, flags, sortbuf, cum, C, mx, Z, logit_scale, p, budget, n_sink, n_local, idx,
                 count, kmax, n_p_out, SN, u, s);
}

__global__ void __launch_bounds__(kSelThreads) select_topp_kernel(
    const float* __restrict__ scores, int C, float logit_scale, float p, int budget, int n_sink,
    int n_local, int32_t* __restrict__ idx, int32_t* __restrict__ count, int kmax,
    int32_t* __restrict__ n_p_out, int SN) {
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ SelScratch s;
  __shared__ BucketScratch bs;
  const size_t head = topp_head_bytes(C, SN);
  uint64_t* sortbuf = reinterpret_cast<uint64_t*>(sm);            // [SN] or the sort exchange
  float* cum = reinterpret_cast<float*>(sm + static_cast<size_t>(SN) * 8);  // [SN]
  uint32_t* keys = reinterpret_cast<uint32_t*>(sm + head);  // [C]
  uint8_t* flags = sm + head + static_cast<size_t>(C) * 4;  // [C]
  const int u = blockIdx.x;
  const float* row = scores + static_cast<int64_t>(u) * C;
  float mx = -INFINITY, Z = 0.f;
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    const float x = row[c];
    keys[c] = float_key(x);
    flags[c] = 0;
    ms_add(mx, Z, x, logit_scale);
  }
  block_max_sumexp(mx, Z, logit_scale, s);  // its barriers also publish keys
  topp_select(keys, flags, sortbuf, cum, C, mx, Z, logit_scale, p, budget, n_sink, n_local, idx,
              count, kmax, n_p_out, SN, u, s, bs);
}

// Group-summed dot products of `nrows` rows (row ids rows[i], or i when rows
// is null) of a [*, D] fp32 matrix with qs, into keys (0 where skip(c)).
template <bool kSkipForced>
__device__ void score_rows(const float* __restrict__ mat, int D, const float* qs, const int* rows,
                           int nrows, uint32_t* keys, int C, int n_sink, int n_local) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  constexpr int BATCH = 16;
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
  allow_dependent_launch();
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ SelScratch s;
  __shared__ BucketScratch bs;
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
  const int exch_bytes = sort_exch_bytes(max(M, NCH));
  uint64_t* exch = exch_bytes ? reinterpret_cast<uint64_t*>(
                                    sm + ((static_cast<size_t>(5) * M + 9 * NCH + 4 * k1 + C + 15) & ~size_t(15)))
                              : nullptr;

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
  mark_best(mkeys, mflags, M, M, k1, exch, bs, s);
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
  mark_best(ckeys, cflags, NCH, n_cand, k_free, exch, bs, s);
  for (int i = threadIdx.x; i < NCH; i += blockDim.x)
    if (cflags[i]) flags[clist[i]] = 1;
  __syncthreads();
  emit_ascending(flags, C, idx + static_cast<int64_t>(u) * kmax, count + u, kmax, s);
}

// Selection by rank for small candidate sets (n <= kRankMax): thread i counts
// the composite keys above its own (composites are unique: ties go to the
// lower chunk index), and keeps i when fewer than k are above it.  Key 0 is
// "not a candidate".  n^2 / blockDim comparisons, all shared-memory
// broadcasts, and a single barrier.
constexpr int kRankMax = 512;

__device__ void rank_select(const uint64_t* comp, int n, int k, uint8_t* sel) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const uint64_t me = comp[i];
    int above = 0;
    if (me != 0ull)
      for (int j = 0; j < n; ++j) above += comp[j] > me;
    sel[i] = (me != 0ull && above < k) ? 1 : 0;
  }
  __syncthreads();
}

// Hierarchical selection when both levels have at most kRankMax candidates:
// rank selection at each level, and the list written directly as sink
// chunks, the chosen children (ascending already: the kept metas are
// ascending and so are their children) and the local chunks.
__global__ void __launch_bounds__(kSelThreads) select_hier_rank_kernel(
    const void* __restrict__ q, int q_bf16, const float* __restrict__ meta,
    const float* __restrict__ summ, int Hq, int Hkv, int D, int C, int Gm, int top_meta,
    int k_free, int n_sink, int n_local, int32_t* __restrict__ idx, int32_t* __restrict__ count,
    int kmax) {
  allow_dependent_launch();
  __shared__ SelScratch s;
  __shared__ float qs[128];
  __shared__ uint32_t keys[kRankMax];
  __shared__ uint64_t comp[kRankMax];
  __shared__ int clist[kRankMax];
  __shared__ uint8_t sel[kRankMax];
  __shared__ int mlist[kRankMax];
  const int M = C / Gm;
  const int k1 = min(top_meta, M);
  const int NCH = k1 * Gm;
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
  __syncthreads();
  // level 1: meta-chunks (every meta is a candidate)
  score_rows<false>(meta + static_cast<int64_t>(u) * M * D, D, qs, nullptr, M, keys, C, 0, 0);
  __syncthreads();
  for (int i = threadIdx.x; i < M; i += blockDim.x) comp[i] = composite(keys[i], i);
  __syncthreads();
  rank_select(comp, M, k1, sel);
  {  // ascending list of the kept metas, then their children
    int pos = block_exclusive_scan(threadIdx.x < M ? sel[threadIdx.x] : 0, s.scan, nullptr);
    if (threadIdx.x < M && sel[threadIdx.x]) mlist[pos] = threadIdx.x;
    __syncthreads();
    for (int i = threadIdx.x; i < NCH; i += blockDim.x) clist[i] = mlist[i / Gm] * Gm + (i % Gm);
    __syncthreads();
  }
  // level 2: the children, forced chunks excluded from the pool (key 0)
  score_rows<true>(summ + static_cast<int64_t>(u) * C * D, D, qs, clist, NCH, keys, C, n_sink,
                   n_local);
  __syncthreads();
  for (int i = threadIdx.x; i < NCH; i += blockDim.x) comp[i] = composite(keys[i], clist[i]);
  __syncthreads();
  rank_select(comp, NCH, k_free, sel);
  // list = sink chunks, chosen children (ascending), local chunks
  int nsel = 0;
  const int pos = block_exclusive_scan(threadIdx.x < NCH ? sel[threadIdx.x] : 0, s.scan, &nsel);
  const int n_s = min(n_sink, C);
  const int loc0 = max(C - n_local, n_s);
  const int n_l = C - loc0;
  const int total = n_s + nsel + n_l;
  int32_t* row = idx + static_cast<int64_t>(u) * kmax;
  if (threadIdx.x < NCH && sel[threadIdx.x] && n_s + pos < kmax) row[n_s + pos] = clist[threadIdx.x];
  for (int j = threadIdx.x; j < n_s && j < kmax; j += blockDim.x) row[j] = j;
  for (int j = threadIdx.x; j < n_l; j += blockDim.x)
    if (n_s + nsel + j < kmax) row[n_s + nsel + j] = loc0 + j;
  for (int j = total + threadIdx.x; j < kmax; j += blockDim.x) row[j] = -1;
  if (threadIdx.x == 0) count[u] = min(total, kmax);
}

// ---------------------------------------------------------------- fused score + select

// Group-summed query of unit (b, h) into qs[0, D) and, with a projection,
// proj^T qs into qv[0, R).  Same partition and order as the score kernel
// (256 threads split the d range), so the scores match it bit for bit.
__device__ void unit_query(const void* __restrict__ q, int q_bf16, int64_t head0, int G, int D,
                           const float* __restrict__ proj, int R, float* qs, float* qv,
                           float* part) {
  // this thread's projection entries are loaded together with the query
  // (they do not depend on it), so the two global round trips overlap
  constexpr int kPre = 8;
  float pw[kPre];
  const int parts = proj != nullptr ? 256 / R : 1;
  const int pr = threadIdx.x / parts, ppt = threadIdx.x % parts;
  const int dchunk = (D + parts - 1) / parts;
  const int pd0 = ppt * dchunk, pd1 = min(D, pd0 + dchunk);
  const bool pre_ok = proj != nullptr && threadIdx.x < 256 && dchunk <= kPre;
#pragma unroll
  for (int k = 0; k < kPre; ++k)
    pw[k] = pre_ok && pd0 + k < pd1 ? __ldg(proj + static_cast<int64_t>(pd0 + k) * R + pr) : 0.f;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    for (int g = 0; g < G; ++g) {
      const int64_t off = (head0 + g) * D + d;
      acc += q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(q)[off])
                    : static_cast<const float*>(q)[off];
    }
    qs[d] = acc;
  }
  __syncthreads();
  if (proj == nullptr) return;
  // 256 threads: thread t handles r = t / parts over the d range of part
  // t % parts; the parts of one r sit in adjacent lanes and are added by an
  // xor-shuffle tree (same order as the score kernel)
  if (threadIdx.x < 256) {
    float acc = 0.f;
    if (pre_ok) {
#pragma unroll
      for (int k = 0; k < kPre; ++k)
        if (pd0 + k < pd1) acc += pw[k] * qs[pd0 + k];
    } else {
#pragma unroll 4
      for (int d = pd0; d < pd1; ++d) acc += __ldg(proj + static_cast<int64_t>(d) * R + pr) * qs[d];
    }
    for (int o = parts >> 1; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (ppt == 0) qv[pr] = acc;
  }
  (void)part;
  __syncthreads();
}

constexpr int kRowBatch = 8;  // summary rows per lane group in flight

// First round of summary rows of a unit (issued before the query is ready).
template <int DS>
__device__ __forceinline__ void rows_load(const float* __restrict__ summ_u, int C, int base,
                                          float4 (&v)[kRowBatch]) {
  constexpr int LPR = DS / 4, RPI = 32 / LPR;
  const int lane = threadIdx.x & 31;
  const int sub = lane % LPR, rsub = lane / LPR;
#pragma unroll
  for (int b = 0; b < kRowBatch; ++b) {
    const int c = base + b * RPI + rsub;
    v[b] = c < C ? __ldg(reinterpret_cast<const float4*>(summ_u + static_cast<int64_t>(c) * DS) + sub)
                 : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

template <int DS>
__device__ __forceinline__ int rows_first_base() {
  constexpr int RPI = 32 / (DS / 4);
  return (threadIdx.x >> 5) * RPI * kRowBatch;
}

// keys[c] = key of (qv . summ_u[c]) for c < C (0 for forced chunks when
// skip_forced), with the running (max, sum-exp) of the scores when scale != 0.
// Rows of DS floats over DS/4 lanes, kRowBatch rows per lane group in flight;
// `pre` holds the first round, loaded by rows_load.
template <int DS>
__device__ void summaries_to_keys(const float* __restrict__ summ_u, int C, const float* qv,
                                  uint32_t* keys, int n_sink, int n_local, bool skip_forced,
                                  float& mx, float& sum, float scale,
                                  const float4 (&pre)[kRowBatch]) {
  constexpr int LPR = DS / 4, RPI = 32 / LPR;
  const int lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int sub = lane % LPR, rsub = lane / LPR;
  const float4 q4 = make_float4(qv[sub * 4], qv[sub * 4 + 1], qv[sub * 4 + 2], qv[sub * 4 + 3]);
  mx = -INFINITY;
  sum = 0.f;
  const int first = rows_first_base<DS>();
  for (int base = first; base < C; base += nw * RPI * kRowBatch) {
    float4 v[kRowBatch];
    if (base == first) {
#pragma unroll
      for (int b = 0; b < kRowBatch; ++b) v[b] = pre[b];
    } else {
      rows_load<DS>(summ_u, C, base, v);
    }
#pragma unroll
    for (int b = 0; b < kRowBatch; ++b) {
      float x = v[b].x * q4.x + v[b].y * q4.y + v[b].z * q4.z + v[b].w * q4.w;
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      const int c = base + b * RPI + rsub;
      if (sub == 0 && c < C) {
        keys[c] = (skip_forced && is_forced(c, C, n_sink, n_local)) ? 0u : float_key(x);
        if (scale != 0.f) ms_add(mx, sum, x, scale);
      }
    }
  }
}

struct FusedSmem {
  float qs[1024];
  float qv[128];
  float part[256];
};

// Fused score + top-k, one CTA per unit.  kUnion: per-head top-k with the
// GQA union (each query head of the group scores the chunks with its own
// query and marks its k_free best; the unit keeps the union, loaded once by
// the decode); otherwise one top-k over the group-summed score.
template <int DS, bool kUnion>
__global__ void __launch_bounds__(kSelThreads) score_select_topk_kernel(
    const void* __restrict__ q, int q_bf16, const float* __restrict__ proj, int R,
    const float* __restrict__ summ, int Hq, int Hkv, int D, int C,
    const uint8_t* __restrict__ head_full, int k_free, int n_sink, int n_local,
    int32_t* __restrict__ idx, int32_t* __restrict__ count, int kmax) {
  allow_dependent_launch();
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ SelScratch s;
  __shared__ BucketScratch bs;
  __shared__ FusedSmem f;
  const int exch_bytes = sort_exch_bytes(C);
  uint64_t* exch = exch_bytes ? reinterpret_cast<uint64_t*>(sm) : nullptr;
  uint32_t* keys = reinterpret_cast<uint32_t*>(sm + exch_bytes);
  uint8_t* flags = sm + exch_bytes + static_cast<size_t>(C) * 4;
  const int u = blockIdx.x, h = u % Hkv, b = u / Hkv, G = Hq / Hkv;
  int32_t* row = idx + static_cast<int64_t>(u) * kmax;
  if (head_full != nullptr && head_full[h]) {  // full heads read every chunk: no list
    for (int i = threadIdx.x; i < kmax; i += blockDim.x) row[i] = -1;
    if (threadIdx.x == 0) count[u] = 0;
    return;
  }
  const float* summ_u = summ + static_cast<int64_t>(u) * C * DS;
  const int64_t head0 = static_cast<int64_t>(b) * Hq + h * G;
  float4 pre[kRowBatch];
  rows_load<DS>(summ_u, C, rows_first_base<DS>(), pre);  // in flight during the query phase
  unit_query(q, q_bf16, head0, kUnion ? 1 : G, D, proj, R, f.qs, f.qv, f.part);
  for (int c = threadIdx.x; c < C; c += blockDim.x) flags[c] = is_forced(c, C, n_sink, n_local);
  float mx_unused = 0.f, sum_unused = 0.f;
  summaries_to_keys<DS>(summ_u, C, proj ? f.qv : f.qs, keys, n_sink, n_local, true, mx_unused,
                        sum_unused, 0.f, pre);
  __syncthreads();
  if (!kUnion) {
    topk_from_keys(keys, flags, C, n_sink, n_local, k_free, row, count + u, kmax, s, exch, bs);
    return;
  }
  const int n_cand = C - forced_count(C, n_sink, n_local);
  for (int g = 0;;) {
    mark_best(keys, flags, C, n_cand, k_free, exch, bs, s);  // sets flags; never clears them
    __syncthreads();
    if (++g == G) break;
    rows_load<DS>(summ_u, C, rows_first_base<DS>(), pre);
    unit_query(q, q_bf16, head0 + g, 1, D, proj, R, f.qs, f.qv, f.part);
    summaries_to_keys<DS>(summ_u, C, proj ? f.qv : f.qs, keys, n_sink, n_local, true, mx_unused,
                          sum_unused, 0.f, pre);
    __syncthreads();
  }
  emit_ascending(flags, C, row, count + u, kmax, s);
}

template <int DS>
__global__ void __launch_bounds__(kSelThreads) score_select_topp_kernel(
    const void* __restrict__ q, int q_bf16, const float* __restrict__ proj, int R,
    const float* __restrict__ summ, int Hq, int Hkv, int D, int C,
    const uint8_t* __restrict__ head_full, float logit_scale, float p, int budget, int n_sink,
    int n_local, int32_t* __restrict__ idx, int32_t* __restrict__ count, int kmax,
    int32_t* __restrict__ n_p_out, int SN, int q_after_copy) {
  // q_after_copy: launched behind the kernel that writes q (programmatic
  // dependent launch); the grid behind this one may start only once q is
  // complete, since it reads q without waiting for this grid
  if (!q_after_copy) allow_dependent_launch();
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ SelScratch s;
  __shared__ BucketScratch bs;
  __shared__ FusedSmem f;
  const size_t head = topp_head_bytes(C, SN);
  uint64_t* sortbuf = reinterpret_cast<uint64_t*>(sm);
  float* cum = reinterpret_cast<float*>(sm + static_cast<size_t>(SN) * 8);
  uint32_t* keys = reinterpret_cast<uint32_t*>(sm + head);
  uint8_t* flags = sm + head + static_cast<size_t>(C) * 4;
  const int u = blockIdx.x, h = u % Hkv, b = u / Hkv, G = Hq / Hkv;
  if (head_full != nullptr && head_full[h]) {
    int32_t* row = idx + static_cast<int64_t>(u) * kmax;
    for (int i = threadIdx.x; i < kmax; i += blockDim.x) row[i] = -1;
    if (threadIdx.x == 0) {
      count[u] = 0;
      if (n_p_out) n_p_out[u] = 0;
    }
    return;
  }
  const float* summ_u = summ + static_cast<int64_t>(u) * C * DS;
  float4 pre[kRowBatch];
  rows_load<DS>(summ_u, C, rows_first_base<DS>(), pre);  // in flight during the query phase
  if (q_after_copy) {
    grid_dependency_wait();  // the query copy is complete and visible
    allow_dependent_launch();
  }
  unit_query(q, q_bf16, static_cast<int64_t>(b) * Hq + h * G, G, D, proj, R, f.qs, f.qv, f.part);
  for (int c = threadIdx.x; c < C; c += blockDim.x) flags[c] = 0;
  float mx = -INFINITY, Z = 0.f;
  summaries_to_keys<DS>(summ_u, C, proj ? f.qv : f.qs, keys, 0, 0, false, mx, Z, logit_scale, pre);
  block_max_sumexp(mx, Z, logit_scale, s);  // its barriers also publish keys
  topp_select(keys, flags, sortbuf, cum, C, mx, Z, logit_scale, p, budget, n_sink, n_local, idx,
              count, kmax, n_p_out, SN, u, s, bs);
}

// ---------------------------------------------------------------- cluster score + top-k
//
// Short selections: one cluster of CS CTAs per unit.  CTA r scores the r-th
// of CS equal ranges of the unit's chunks (one round of summary loads) and
// keeps its best min(k_free, candidates) by rank: the 64-bit composites
// (score key << 32 | ~index) are unique, so a chunk is kept when fewer than
// k_free composites of the range exceed its own.  The kept candidates meet
// in the first CTA's shared memory, which ranks them again the same way,
// adds the forced chunks and writes the ascending list.  The result is the
// unit's top-k: a chunk among the best k_free overall is among the best
// k_free of its own range.

constexpr int kClSelThreads = 256;
constexpr int kClRangeMax = 512;  // chunks scored by one CTA
constexpr int kClCandMax = 512;   // candidates meeting in the first CTA
constexpr int kClRowBatch = 16;   // summary rows per warp in flight

// One warp's round of summary rows: local rows base + b * RPI + (lane /
// (DS/4)), b < kClRowBatch, each lane holding one float4 of its row.
template <int DS>
__device__ __forceinline__ void rows_issue(const float* __restrict__ summ_u, int lo, int n,
                                           const int* rows, int base, float4 (&v)[kClRowBatch]) {
  constexpr int LPR = DS / 4, RPI = 32 / LPR;
  const int lane = threadIdx.x & 31;
  const int sub = lane % LPR, rsub = lane / LPR;
#pragma unroll
  for (int b = 0; b < kClRowBatch; ++b) {
    const int i = base + b * RPI + rsub;
    const int r = i < n ? (rows ? rows[lo + i] : lo + i) : 0;
    v[b] = i < n ? __ldg(reinterpret_cast<const float4*>(summ_u + static_cast<int64_t>(r) * DS) + sub)
                 : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

template <int DS>
__device__ __forceinline__ int rows_first(int n) {
  constexpr int RPI = 32 / (DS / 4);
  return (threadIdx.x >> 5) * RPI * kClRowBatch;
}

// Composite keys of n summary rows of a unit (row of local index i: lo + i,
// or rows[lo + i] when a row list is given) against the (projected,
// group-summed) query qv; forced chunks (skip_forced) get 0.  `pre` holds
// this warp's first round when `prefetched` (rows_issue before the query
// was ready).
template <int DS>
__device__ __forceinline__ void cluster_scores(const float* __restrict__ summ_u, int lo, int n,
                                               int C, const float* qv, int n_sink, int n_local,
                                               uint64_t* comp, const int* rows, bool skip_forced,
                                               const float4 (&pre)[kClRowBatch], bool prefetched) {
  constexpr int LPR = DS / 4, RPI = 32 / LPR;  // lanes per row, rows per warp step
  const int lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int sub = lane % LPR, rsub = lane / LPR;
  const float4 q4 = make_float4(qv[sub * 4], qv[sub * 4 + 1], qv[sub * 4 + 2], qv[sub * 4 + 3]);
  const int first = rows_first<DS>(n);
  for (int base = first; base < n; base += nw * RPI * kClRowBatch) {
    float4 v[kClRowBatch];
    if (prefetched && base == first) {
#pragma unroll
      for (int b = 0; b < kClRowBatch; ++b) v[b] = pre[b];
    } else {
      rows_issue<DS>(summ_u, lo, n, rows, base, v);
    }
#pragma unroll
    for (int b = 0; b < kClRowBatch; ++b) {
      float x = v[b].x * q4.x + v[b].y * q4.y + v[b].z * q4.z + v[b].w * q4.w;
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      const int i = base + b * RPI + rsub;
      if (sub == 0 && i < n) {
        const int c = rows ? rows[lo + i] : lo + i;
        comp[i] = (skip_forced && is_forced(c, C, n_sink, n_local)) ? 0ull
                                                                     : composite(float_key(x), c);
      }
    }
  }
}

// comp[0, n) -> kept[0, *n_kept): the composites with fewer than k of the
// others above them (all composites distinct, 0 = none).  Ends with a barrier.
__device__ __forceinline__ void rank_keep(const uint64_t* comp, int n, int k, uint64_t* kept,
                                          int* n_kept) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const uint64_t me = comp[i];
    if (me == 0ull) continue;
    int above = 0;
    for (int j = 0; j < n; ++j) above += comp[j] > me;
    if (above < k) kept[atomicAdd(n_kept, 1)] = me;
  }
  __syncthreads();
}

// The first CTA's ascending list of the chosen chunks sel[0, n_sel) and the
// forced ones (the first n_sink and last n_local of C), written to the
// unit's index row.  The chunks are distinct; `buf` has room for all.
__device__ void emit_with_forced(int32_t* buf, int n_sel, int C, int n_sink, int n_local,
                                 int32_t* row, int32_t* cnt, int kmax) {
  const int ns_ = min(n_sink, C), loc0 = max(C - n_local, ns_);
  for (int j = threadIdx.x; j < ns_; j += blockDim.x) buf[n_sel + j] = j;
  for (int j = threadIdx.x; j < C - loc0; j += blockDim.x) buf[n_sel + ns_ + j] = loc0 + j;
  const int total = n_sel + ns_ + (C - loc0);
  __syncthreads();
  // each chunk's place is the number of smaller ones
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    const int me = buf[i];
    int pos = 0;
    for (int j = 0; j < total; ++j) pos += buf[j] < me;
    if (pos < kmax) row[pos] = me;
  }
  for (int i = total + threadIdx.x; i < kmax; i += blockDim.x) row[i] = -1;
  if (threadIdx.x == 0) *cnt = min(total, kmax);
}

template <int DS>
__global__ void __launch_bounds__(kClSelThreads) score_select_topk_cluster_kernel(
    const void* __restrict__ q, int q_bf16, const float* __restrict__ proj, int R,
    const float* __restrict__ summ, int Hq, int Hkv, int D, int C,
    const uint8_t* __restrict__ head_full, int k_free, int n_sink, int n_local,
    int32_t* __restrict__ idx, int32_t* __restrict__ count, int kmax) {
  allow_dependent_launch();
  cluster_arrive_relaxed();  // every CTA of the cluster runs by the matching wait
  __shared__ FusedSmem f;
  __shared__ uint64_t comp[kClRangeMax];
  __shared__ uint64_t kept[kClRangeMax];
  __shared__ uint64_t cand[kClCandMax];
  __shared__ int32_t out_l[kClCandMax + 64];
  __shared__ int n_kept, n_out;
  const int CS = static_cast<int>(cluster_size());
  const int rank = static_cast<int>(cluster_rank());
  const int u = blockIdx.y, h = u % Hkv, b = u / Hkv, G = Hq / Hkv;
  const int lo = static_cast<int>(static_cast<int64_t>(C) * rank / CS);
  const int n = static_cast<int>(static_cast<int64_t>(C) * (rank + 1) / CS) - lo;
  const int KL = (k_free < (C + CS - 1) / CS) ? k_free : (C + CS - 1) / CS;  // slots per CTA
  const bool full = head_full != nullptr && head_full[h];
  if (threadIdx.x == 0) n_kept = 0;
  if (!full) {
    const float* summ_u = summ + static_cast<int64_t>(u) * C * DS;
    float4 pre[kClRowBatch];
    rows_issue<DS>(summ_u, lo, n, nullptr, rows_first<DS>(n), pre);  // in flight with the query
    unit_query(q, q_bf16, static_cast<int64_t>(b) * Hq + h * G, G, D, proj, R, f.qs, f.qv,
               f.part);  // ends with a barrier
    cluster_scores<DS>(summ_u, lo, n, C, proj ? f.qv : f.qs, n_sink, n_local, comp, nullptr, true,
                       pre, true);
    __syncthreads();
    rank_keep(comp, n, k_free, kept, &n_kept);
  }
  __syncthreads();
  cluster_wait();  // (phase 1)
  if (!full) {  // this CTA's kept candidates into its slots of the first CTA (zeros pad)
    const uint32_t dst = cluster_map(smem_u32(cand + rank * KL), 0);
    const int nk = n_kept;
    for (int i = threadIdx.x; i < KL; i += blockDim.x)
      st_cluster_u64(dst + i * 8, i < nk ? kept[i] : 0ull);
  }
  cluster_arrive();  // (phase 2)
  cluster_wait();
  if (rank != 0) return;
  int32_t* row = idx + static_cast<int64_t>(u) * kmax;
  if (full) {  // full heads read every chunk: no list
    for (int i = threadIdx.x; i < kmax; i += blockDim.x) row[i] = -1;
    if (threadIdx.x == 0) count[u] = 0;
    return;
  }
  // the unit's best k_free among the candidates, then the forced chunks
  const int nc = CS * KL;
  if (threadIdx.x == 0) n_out = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < nc; i += blockDim.x) {
    const uint64_t me = cand[i];
    if (me == 0ull) continue;
    int above = 0;
    for (int j = 0; j < nc; ++j) above += cand[j] > me;
    if (above < k_free) out_l[atomicAdd(&n_out, 1)] = comp_index(me);
  }
  __syncthreads();
  emit_with_forced(out_l, n_out, C, n_sink, n_local, row, count + u, kmax);
}

// Per-head top-k with the GQA union by a cluster of CS CTAs per unit: CTA r
// loads the summary rows of the r-th range of the unit's chunks once and
// scores them against each of the G query heads' own (projected) queries;
// per head it keeps its best min(k_free, candidates) by rank.  The first
// CTA gathers every head's candidates, takes each head's k_free best (the
// same argument as for one head: a chunk among a head's best k_free overall
// is among that head's best of its own range), marks their union, adds the
// forced chunks and writes the ascending list.
template <int DS>
__device__ __forceinline__ void cluster_scores_heads(const float* __restrict__ summ_u, int lo,
                                                     int n, int C, const float* qall, int G,
                                                     int n_sink, int n_local, uint64_t* comp,
                                                     int stride,
                                                     const float4 (&pre)[kClRowBatch]) {
  constexpr int LPR = DS / 4, RPI = 32 / LPR;
  const int lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int sub = lane % LPR, rsub = lane / LPR;
  const int first = rows_first<DS>(n);
  for (int base = first; base < n; base += nw * RPI * kClRowBatch) {
    float4 v[kClRowBatch];
    if (base == first) {
#pragma unroll
      for (int b = 0; b < kClRowBatch; ++b) v[b] = pre[b];
    } else {
      rows_issue<DS>(summ_u, lo, n, nullptr, base, v);
    }
    for (int g = 0; g < G; ++g) {
      const float* qv = qall + g * DS;
      const float4 q4 = make_float4(qv[sub * 4], qv[sub * 4 + 1], qv[sub * 4 + 2], qv[sub * 4 + 3]);
#pragma unroll
      for (int b = 0; b < kClRowBatch; ++b) {
        float x = v[b].x * q4.x + v[b].y * q4.y + v[b].z * q4.z + v[b].w * q4.w;
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        const int i = base + b * RPI + rsub;
        if (sub == 0 && i < n) {
          const int c = lo + i;
          comp[g * stride + i] = is_forced(c, C, n_sink, n_local) ? 0ull : composite(float_key(x), c);
        }
      }
    }
  }
}

// Dynamic shared memory of the union kernel: qall [G][DS] f32 | comp
// [G][per] | kept [G][KL] | cand [G][CS][KL] (u64) | out_l [C + 64] i32 |
// flags [C] u8.
__host__ __device__ inline size_t union_cl_bytes(int G, int DS, int per, int KL, int CS, int C) {
  return static_cast<size_t>(G) * DS * 4 + static_cast<size_t>(G) * (per + KL + CS * KL) * 8 +
         static_cast<size_t>(C + 64) * 4 + static_cast<size_t>(C + 15) / 16 * 16;
}

template <int DS>
__global__ void __launch_bounds__(kClSelThreads) score_select_union_cluster_kernel(
    const void* __restrict__ q, int q_bf16, const float* __restrict__ proj, int R,
    const float* __restrict__ summ, int Hq, int Hkv, int D, int C,
    const uint8_t* __restrict__ head_full, int k_free, int n_sink, int n_local,
    int32_t* __restrict__ idx, int32_t* __restrict__ count, int kmax) {
  allow_dependent_launch();
  cluster_arrive_relaxed();  // every CTA of the cluster runs by the matching wait
  __shared__ FusedSmem f;
  __shared__ int n_kept[8];
  __shared__ int n_out;
  extern __shared__ __align__(16) uint8_t dsm[];
  const int CS = static_cast<int>(cluster_size());
  const int rank = static_cast<int>(cluster_rank());
  const int u = blockIdx.y, h = u % Hkv, b = u / Hkv, G = Hq / Hkv;
  const int per = (C + CS - 1) / CS;
  const int lo = static_cast<int>(static_cast<int64_t>(C) * rank / CS);
  const int n = static_cast<int>(static_cast<int64_t>(C) * (rank + 1) / CS) - lo;
  const int KL = k_free < per ? k_free : per;  // slots per CTA and head
  float* qall = reinterpret_cast<float*>(dsm);
  uint64_t* comp = reinterpret_cast<uint64_t*>(dsm + static_cast<size_t>(G) * DS * 4);
  uint64_t* kept = comp + static_cast<size_t>(G) * per;
  uint64_t* cand = kept + static_cast<size_t>(G) * KL;
  int32_t* out_l = reinterpret_cast<int32_t*>(cand + static_cast<size_t>(G) * CS * KL);
  uint8_t* flags = reinterpret_cast<uint8_t*>(out_l + C + 64);
  const bool full = head_full != nullptr && head_full[h];
  if (threadIdx.x < 8) n_kept[threadIdx.x] = 0;
  if (!full) {
    const float* summ_u = summ + static_cast<int64_t>(u) * C * DS;
    float4 pre[kClRowBatch];
    rows_issue<DS>(summ_u, lo, n, nullptr, rows_first<DS>(n), pre);  // in flight with the queries
    // the G heads' queries in one round of loads, then each projected (the
    // same partition and order as unit_query)
    const int64_t head0 = static_cast<int64_t>(b) * Hq + h * G;
    float* qs_all = proj ? f.qs : qall;  // [G][D]
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
      const int64_t off = head0 * D + e;
      qs_all[e] = q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(q)[off])
                         : static_cast<const float*>(q)[off];
    }
    __syncthreads();
    if (proj) {
      const int parts = 256 / R;
      for (int g = 0; g < G; ++g) {
        if (threadIdx.x < 256) {
          const int r = threadIdx.x / parts, pt = threadIdx.x % parts;
          const int dchunk = (D + parts - 1) / parts;
          const int d0 = pt * dchunk, d1 = min(D, d0 + dchunk);
          float acc = 0.f;
#pragma unroll 4
          for (int d = d0; d < d1; ++d)
            acc += __ldg(proj + static_cast<int64_t>(d) * R + r) * qs_all[g * D + d];
          for (int o = parts >> 1; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
          if (pt == 0) qall[g * DS + r] = acc;
        }
      }
      __syncthreads();
    }
    cluster_scores_heads<DS>(summ_u, lo, n, C, qall, G, n_sink, n_local, comp, per, pre);
    __syncthreads();
    for (int g = 0; g < G; ++g) rank_keep(comp + g * per, n, k_free, kept + g * KL, &n_kept[g]);
  }
  __syncthreads();
  cluster_wait();  // (phase 1)
  if (!full) {  // each head's kept candidates into this CTA's slots of the first CTA
    for (int g = 0; g < G; ++g) {
      const uint32_t dst = cluster_map(smem_u32(cand + (static_cast<size_t>(g) * CS + rank) * KL), 0);
      const int nk = n_kept[g];
      for (int i = threadIdx.x; i < KL; i += blockDim.x)
        st_cluster_u64(dst + i * 8, i < nk ? kept[g * KL + i] : 0ull);
    }
  }
  cluster_arrive();  // (phase 2)
  cluster_wait();
  if (rank != 0) return;
  int32_t* row = idx + static_cast<int64_t>(u) * kmax;
  if (full) {  // full heads read every chunk: no list
    for (int i = threadIdx.x; i < kmax; i += blockDim.x) row[i] = -1;
    if (threadIdx.x == 0) count[u] = 0;
    return;
  }
  for (int c = threadIdx.x; c < C; c += blockDim.x) flags[c] = 0;
  if (threadIdx.x == 0) n_out = 0;
  __syncthreads();
  const int nc = CS * KL;
  for (int e = threadIdx.x; e < G * nc; e += blockDim.x) {  // each head's k_free best
    const uint64_t* hc = cand + static_cast<size_t>(e / nc) * nc;
    const uint64_t me = hc[e % nc];
    if (me == 0ull) continue;
    int above = 0;
    for (int j = 0; j < nc; ++j) above += hc[j] > me;
    if (above < k_free) flags[comp_index(me)] = 1;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += blockDim.x)
    if (flags[c]) out_l[atomicAdd(&n_out, 1)] = c;
  __syncthreads();
  emit_with_forced(out_l, n_out, C, n_sink, n_local, row, count + u, kmax);
}

// Two-level selection by a cluster of CS CTAs per unit: the meta-chunks'
// scores split over the CTAs, each keeping its best by rank; the first CTA
// ranks the kept metas and hands the ascending list of the top_meta best to
// every CTA of the cluster; the children of those metas split over the CTAs
// the same way (forced chunks out of the pool); the first CTA ranks the kept
// children and writes them with the forced chunks, ascending.
__global__ void __launch_bounds__(kClSelThreads) select_hier_cluster_kernel(
    const void* __restrict__ q, int q_bf16, const float* __restrict__ meta,
    const float* __restrict__ summ, int Hq, int Hkv, int D, int C, int Gm, int top_meta,
    int k_free, int n_sink, int n_local, int32_t* __restrict__ idx, int32_t* __restrict__ count,
    int kmax) {
  allow_dependent_launch();
  cluster_arrive_relaxed();
  __shared__ float qs[128];
  __shared__ uint64_t comp[kClRangeMax];
  __shared__ uint64_t kept[kClRangeMax];
  __shared__ uint64_t cand[kClCandMax];
  __shared__ uint8_t chosen[kClCandMax];
  __shared__ int32_t mlist[kClRangeMax];
  __shared__ int32_t out_l[kClCandMax + 64];
  __shared__ int n_kept, n_out;
  const int CS = static_cast<int>(cluster_size());
  const int rank = static_cast<int>(cluster_rank());
  const int u = blockIdx.y, h = u % Hkv, b = u / Hkv, G = Hq / Hkv;
  const int M = C / Gm, k1 = min(top_meta, M), NCH = k1 * Gm;
  // level 1: this CTA's share of the metas (every meta is a candidate); its
  // rows are in flight while the query is summed
  const int lo1 = static_cast<int>(static_cast<int64_t>(M) * rank / CS);
  const int n1 = static_cast<int>(static_cast<int64_t>(M) * (rank + 1) / CS) - lo1;
  const int KL1 = min(k1, (M + CS - 1) / CS);
  const float* meta_u = meta + static_cast<int64_t>(u) * M * D;
  float4 pre[kClRowBatch];
  rows_issue<128>(meta_u, lo1, n1, nullptr, rows_first<128>(n1), pre);
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    for (int g = 0; g < G; ++g) {
      const int64_t off = (static_cast<int64_t>(b) * Hq + h * G + g) * D + d;
      acc += q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(q)[off])
                    : static_cast<const float*>(q)[off];
    }
    qs[d] = acc;
  }
  if (threadIdx.x == 0) n_kept = 0;
  __syncthreads();
  cluster_scores<128>(meta_u, lo1, n1, C, qs, 0, 0, comp, nullptr, false, pre, true);
  __syncthreads();
  rank_keep(comp, n1, k1, kept, &n_kept);
  cluster_wait();  // (phase 1)
  {
    const uint32_t dst = cluster_map(smem_u32(cand + rank * KL1), 0);
    for (int i = threadIdx.x; i < KL1; i += blockDim.x)
      st_cluster_u64(dst + i * 8, i < n_kept ? kept[i] : 0ull);
  }
  cluster_arrive();  // (phase 2) the meta candidates are in the first CTA
  cluster_wait();
  if (rank == 0) {  // the top_meta best metas, ascending, into every CTA's mlist
    const int nc = CS * KL1;
    for (int i = threadIdx.x; i < nc; i += blockDim.x) {
      const uint64_t me = cand[i];
      int above = 0;
      if (me != 0ull)
        for (int j = 0; j < nc; ++j) above += cand[j] > me;
      chosen[i] = me != 0ull && above < k1;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nc; i += blockDim.x) {
      if (!chosen[i]) continue;
      const int m = comp_index(cand[i]);
      int pos = 0;
      for (int j = 0; j < nc; ++j) pos += chosen[j] && comp_index(cand[j]) < m;
      for (int r = 0; r < CS; ++r) st_cluster_u32(cluster_map(smem_u32(mlist + pos), r), m);
    }
  }
  cluster_arrive();  // (phase 3) every CTA holds the kept metas
  cluster_wait();
  // level 2: this CTA's share of the kept metas' children
  if (threadIdx.x == 0) n_kept = 0;
  const int lo2 = static_cast<int>(static_cast<int64_t>(NCH) * rank / CS);
  const int n2 = static_cast<int>(static_cast<int64_t>(NCH) * (rank + 1) / CS) - lo2;
  const int KL2 = min(k_free, (NCH + CS - 1) / CS);
  int32_t* clist = out_l;  // chunk of child i: meta mlist[i / Gm], child i % Gm
  for (int i = threadIdx.x; i < n2; i += blockDim.x)
    clist[lo2 + i - lo2] = mlist[(lo2 + i) / Gm] * Gm + (lo2 + i) % Gm;
  __syncthreads();
  cluster_scores<128>(summ + static_cast<int64_t>(u) * C * D, 0, n2, C, qs, n_sink, n_local,
                      comp, clist, true, pre, false);
  __syncthreads();
  rank_keep(comp, n2, k_free, kept, &n_kept);
  {
    const uint32_t dst = cluster_map(smem_u32(cand + rank * KL2), 0);
    for (int i = threadIdx.x; i < KL2; i += blockDim.x)
      st_cluster_u64(dst + i * 8, i < n_kept ? kept[i] : 0ull);
  }
  cluster_arrive();  // (phase 4) the child candidates are in the first CTA
  cluster_wait();
  if (rank != 0) return;
  if (threadIdx.x == 0) n_out = 0;
  __syncthreads();
  const int nc2 = CS * KL2;
  for (int i = threadIdx.x; i < nc2; i += blockDim.x) {
    const uint64_t me = cand[i];
    if (me == 0ull) continue;
    int above = 0;
    for (int j = 0; j < nc2; ++j) above += cand[j] > me;
    if (above < k_free) out_l[atomicAdd(&n_out, 1)] = comp_index(me);
  }
  __syncthreads();
  emit_with_forced(out_l, n_out, C, n_sink, n_local, idx + static_cast<int64_t>(u) * kmax,
                   count + u, kmax);
}

int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

// ------------------------------------------------------------------ long rows (cluster)
//
// Top-k over long score rows with no forced entries (the Token Sparse
// tokens, C >= kClTopkMinC): one cluster of kClTopkCS CTAs per unit, CTA r
// holding the keys of positions [C r / CS, C (r + 1) / CS) in shared memory.
// An MSB-first radix select over the keys' four bytes finds the k-th largest
// key tau, the CTAs' 256-bucket histograms of each pass added through
// distributed shared memory in rank order (integer counts: every CTA takes
// the same bucket); the keys equal to tau are taken lowest position first
// (the CTAs' counts of them meet the same way), and each CTA writes its kept
// positions, ascending, after those of the CTAs before it.  `inv` (optional,
// [U, C]): for every position its slot in the unit's list, or -1.
constexpr int kClTopkCS = 8;
constexpr int kClTopkThreads = 512;
constexpr int kClTopkMinC = 8192;

__global__ void __launch_bounds__(kClTopkThreads) topk_cluster_kernel(
    const float* __restrict__ scores, int C, int k_free, const int32_t* __restrict__ k_dev,
    int32_t* __restrict__ idx, int32_t* __restrict__ count, int kmax, int32_t* __restrict__ inv) {
  cluster_arrive_relaxed();
  extern __shared__ __align__(16) uint8_t sm[];
  uint32_t* keys = reinterpret_cast<uint32_t*>(sm);  // this CTA's positions
  __shared__ unsigned int hc[256];                   // this CTA's histogram of the pass
  __shared__ unsigned int gc[256];                   // the cluster's
  __shared__ unsigned int part_eq[kClTopkCS], part_sel[kClTopkCS];
  __shared__ int scan_sh[33];
  __shared__ unsigned int pick_sh[2];  // the pass's bucket and the count above it
  const int CS = static_cast<int>(cluster_size());
  const int rank = static_cast<int>(cluster_rank());
  const int u = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
  const int lo = static_cast<int>(static_cast<int64_t>(C) * rank / CS);
  const int n = static_cast<int>(static_cast<int64_t>(C) * (rank + 1) / CS) - lo;
  const float* row = scores + static_cast<int64_t>(u) * C + lo;
  for (int j = tid; j < n; j += blockDim.x) keys[j] = float_key(row[j]);
  const int k = min(k_dev ? max(0, min(k_dev[u], kmax)) : max(0, min(k_free, kmax)), C);
  __syncthreads();
  cluster_wait();  // (phase 1) every CTA of the cluster is running
  // keys > tau are taken, and the first `need` keys equal to tau
  uint32_t tau = 0u;
  unsigned int need = 0u;
  if (k == 0) {
    tau = 0xffffffffu;
  } else if (k < C) {
    uint32_t prefix = 0u, mask = 0u;
    need = static_cast<unsigned int>(k);
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int d = tid; d < 256; d += blockDim.x) hc[d] = 0u;
      __syncthreads();
      for (int j0 = 0; j0 < n; j0 += blockDim.x) {
        const int j = j0 + tid;
        int d = -1;
        if (j < n) {
          const uint32_t key = keys[j];
          if ((key & mask) == prefix) d = static_cast<int>((key >> shift) & 255u);
        }
        const unsigned int act = __ballot_sync(0xffffffffu, d >= 0);
        if (d >= 0) {  // one shared atomic per distinct bucket of the warp
          const unsigned int peers = __match_any_sync(act, d);
          if (lane == __ffs(peers) - 1) atomicAdd(&hc[d], static_cast<unsigned int>(__popc(peers)));
        }
      }
      cluster_arrive();  // every CTA's histogram of this pass is complete
      cluster_wait();
      for (int d = tid; d < 256; d += blockDim.x) {
        unsigned int c = 0u;
        unsigned int cr[kClTopkCS];  // the launch's cluster has kClTopkCS CTAs: all loads in flight
#pragma unroll
        for (int r = 0; r < kClTopkCS; ++r) cr[r] = ld_cluster_u32(cluster_map(smem_u32(hc + d), r));
#pragma unroll
        for (int r = 0; r < kClTopkCS; ++r) c += cr[r];
        gc[d] = c;
      }
      cluster_arrive();  // every CTA has read the others' histograms (they may be cleared)
      cluster_wait();
      if (tid < 32) {  // the bucket where the count from the top reaches `need`
        unsigned int pc[8], lc = 0u;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          pc[i] = gc[255 - 8 * lane - i];
          lc += pc[i];
        }
        unsigned int sc = lc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned int t = __shfl_up_sync(0xffffffffu, sc, o);
          if (lane >= o) sc += t;
        }
        unsigned int above = sc - lc;  // count in the buckets above this lane's eight
        int sel = -1;
        unsigned int above_sel = 0u;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (sel < 0) {
            if (above + pc[i] >= need) {
              sel = 255 - 8 * lane - i;
              above_sel = above;
            } else {
              above += pc[i];
            }
          }
        }
        // `need` never exceeds the count of keys under the prefix: a bucket is hit
        const unsigned int hit = __ballot_sync(0xffffffffu, sel >= 0);
        if (lane == (hit ? __ffs(hit) - 1 : 0)) {
          pick_sh[0] = sel < 0 ? 0u : static_cast<unsigned int>(sel);
          pick_sh[1] = above_sel;
        }
      }
      __syncthreads();
      prefix |= pick_sh[0] << shift;
      mask |= 255u << shift;
      need -= pick_sh[1];
      __syncthreads();  // pick_sh read before the next pass writes it
    }
    tau = prefix;
  }
  // this thread's segment of the CTA's positions: keys above tau, keys at tau
  const int seg = (n + blockDim.x - 1) / blockDim.x;
  const int s0 = min(n, tid * seg), s1 = min(n, s0 + seg);
  int c_gt = 0, c_eq = 0;
  for (int j = s0; j < s1; ++j) {
    const uint32_t key = keys[j];
    c_gt += key > tau;
    c_eq += key == tau;
  }
  int eq_tot = 0;
  const int eq_base = block_exclusive_scan(c_eq, scan_sh, &eq_tot);
  if (tid < CS) st_cluster_u32(cluster_map(smem_u32(part_eq + rank), tid), static_cast<unsigned int>(eq_tot));
  cluster_arrive();
  cluster_wait();
  int eq_before = 0;
  for (int r = 0; r < rank; ++r) eq_before += static_cast<int>(part_eq[r]);
  const int take = max(0, min(static_cast<int>(need) - eq_before, eq_tot));  // ties kept here
  const int c_sel = c_gt + max(0, min(take - eq_base, c_eq));
  int sel_tot = 0;
  const int sel_base = block_exclusive_scan(c_sel, scan_sh, &sel_tot);
  if (tid < CS) st_cluster_u32(cluster_map(smem_u32(part_sel + rank), tid), static_cast<unsigned int>(sel_tot));
  cluster_arrive();
  cluster_wait();  // the last access to another CTA's shared memory is before this barrier
  int sel_before = 0, total = 0;
  for (int r = 0; r < CS; ++r) {
    const int v = static_cast<int>(part_sel[r]);
    if (r < rank) sel_before += v;
    total += v;
  }
  int32_t* out = idx + static_cast<int64_t>(u) * kmax;
  int32_t* inv_row = inv ? inv + static_cast<int64_t>(u) * C + lo : nullptr;
  int pos = sel_before + sel_base, eq_seen = eq_base;
  for (int j = s0; j < s1; ++j) {
    const uint32_t key = keys[j];
    bool t = key > tau;
    if (key == tau) {
      t = eq_seen < take;
      ++eq_seen;
    }
    if (inv_row) inv_row[j] = t && pos < kmax ? pos : -1;
    if (t) {
      if (pos < kmax) out[pos] = lo + j;
      ++pos;
    }
  }
  const int tot = min(total, kmax);
  const int f0 = tot + static_cast<int>(static_cast<int64_t>(kmax - tot) * rank / CS);
  const int f1 = tot + static_cast<int>(static_cast<int64_t>(kmax - tot) * (rank + 1) / CS);
  for (int i = f0 + tid; i < f1; i += blockDim.x) out[i] = -1;
  if (rank == 0 && tid == 0) count[u] = tot;
}

cudaError_t set_smem(const void* fn, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bytes));
}

}  // namespace

bool topk_cluster_fits(int U, int C, int num_sms) {
  return C >= kClTopkMinC && U <= 65535 && static_cast<int64_t>(U) * kClTopkCS <= num_sms;
}

cudaError_t launch_select_topk(const Launch& l, const float* scores, int U, int C,
                               const int32_t* n_valid, int k_free, int n_sink, int n_local,
                               int32_t* idx, int32_t* count, int kmax, const int32_t* k_dev,
                               int causal_tiles, int causal_tile_m, int causal_L, int32_t* inv,
                               bool* inv_done) {
  if (inv_done) *inv_done = false;
  if (U == 0) return cudaSuccess;
  if (n_valid == nullptr && causal_tiles == 0 && n_sink == 0 && n_local == 0 &&
      topk_cluster_fits(U, C, l.num_sms)) {
    // long rows, nothing forced: one cluster per unit
    const size_t shc = static_cast<size_t>((C + kClTopkCS - 1) / kClTopkCS) * 4;
    cudaError_t e = set_smem(reinterpret_cast<const void*>(topk_cluster_kernel), shc);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kClTopkCS, U);
    cfg.blockDim = dim3(kClTopkThreads);
    cfg.dynamicSmemBytes = shc;
    cfg.stream = l.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kClTopkCS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel, scores, C, k_free, k_dev, idx, count, kmax,
                           inv);
    if (e == cudaSuccess && inv_done) *inv_done = inv != nullptr;
    return e;
  }
  const size_t sh = sort_exch_bytes(C) + static_cast<size_t>(C) * 5 + 16;
  cudaError_t e = set_smem(reinterpret_cast<const void*>(select_topk_kernel), sh);
  if (e != cudaSuccess) return e;
  const CausalRows causal{causal_tiles, causal_tile_m, causal_L};
  // short rows (C <= 1024: at most 8 sort positions per thread) take 128
  // threads, so four times as many units are in flight per SM (64 threads
  // for C <= 512 measured the same)
  const int threads = C <= 1024 ? 128 : kSelThreads;
  select_topk_kernel<<<U, threads, sh, l.stream>>>(scores, C, n_valid, k_free, n_sink, n_local,
                                                   idx, count, kmax, k_dev, causal);
  return cudaGetLastError();
}

cudaError_t launch_select_topp(const Launch& l, const float* scores, int U, int C,
                               float logit_scale, float p, int budget, int n_sink, int n_local,
                               int32_t* idx, int32_t* count, int kmax, int32_t* n_p_out) {
  if (U == 0) return cudaSuccess;
  const int SN = next_pow2(std::min(budget, C));
  const size_t sh = topp_head_bytes(C, SN) + static_cast<size_t>(C) * 5 + 16;
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
  if (D == 128 && n_sink + n_local <= 64 && U <= 65535) {  // one cluster per unit
    for (int CS = 8; CS >= 2; CS >>= 1) {
      if (static_cast<int64_t>(U) * CS > l.num_sms) continue;
      const int per1 = (M + CS - 1) / CS, per2 = (NCH + CS - 1) / CS;
      if (per1 > kClRangeMax || per2 > kClRangeMax || CS * std::min(k1, per1) > kClCandMax ||
          CS * std::min(k_free, per2) > kClCandMax || k1 > kClRangeMax)
        continue;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(CS, U);
      cfg.blockDim = dim3(kClSelThreads);
      cfg.stream = l.stream;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = CS;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      return cudaLaunchKernelEx(&cfg, select_hier_cluster_kernel, q, bf16 ? 1 : 0, meta, summ, Hq,
                                Hkv, D, C, Gm, top_meta, k_free, n_sink, n_local, idx, count,
                                kmax);
    }
  }
  if (M <= kRankMax && NCH <= kRankMax && D <= 128) {
    select_hier_rank_kernel<<<U, kSelThreads, 0, l.stream>>>(q, bf16 ? 1 : 0, meta, summ, Hq, Hkv,
                                                             D, C, Gm, top_meta, k_free, n_sink,
                                                             n_local, idx, count, kmax);
    return cudaGetLastError();
  }
  const size_t base = (static_cast<size_t>(M) * 5 + static_cast<size_t>(NCH) * 9 +
                       static_cast<size_t>(k1) * 4 + static_cast<size_t>(C) + 15) & ~size_t(15);
  const size_t sh = base + sort_exch_bytes(std::max(M, NCH)) + 16;
  cudaError_t e = set_smem(reinterpret_cast<const void*>(select_hier_kernel), sh);
  if (e != cudaSuccess) return e;
  select_hier_kernel<<<U, kSelThreads, sh, l.stream>>>(q, bf16 ? 1 : 0, meta, summ, Hq, Hkv, D, C,
                                                       Gm, top_meta, k_free, n_sink, n_local, idx,
                                                       count, kmax);
  return cudaGetLastError();
}


namespace {
template <int DS, bool kUnion>
cudaError_t fused_topk_kernel(const Launch& l, const void* q, bool bf16, const float* proj, int R,
                              const float* summ, int U, int Hq, int Hkv, int D, int C,
                              const uint8_t* head_full, int k_free, int n_sink, int n_local,
                              int32_t* idx, int32_t* count, int kmax) {
  const size_t sh = sort_exch_bytes(C) + static_cast<size_t>(C) * 5 + 16;
  cudaError_t e = set_smem(reinterpret_cast<const void*>(score_select_topk_kernel<DS, kUnion>), sh);
  if (e != cudaSuccess) return e;
  score_select_topk_kernel<DS, kUnion><<<U, kSelThreads, sh, l.stream>>>(
      q, bf16 ? 1 : 0, proj, R, summ, Hq, Hkv, D, C, head_full, k_free, n_sink, n_local, idx,
      count, kmax);
  return cudaGetLastError();
}

template <int DS>
cudaError_t fused_topk_ds(const Launch& l, const void* q, bool bf16, const float* proj, int R,
                          const float* summ, int U, int Hq, int Hkv, int D, int C,
                          const uint8_t* head_full, int k_free, int n_sink, int n_local,
                          int32_t* idx, int32_t* count, int kmax, bool per_head_union) {
  if (per_head_union)
    return fused_topk_kernel<DS, true>(l, q, bf16, proj, R, summ, U, Hq, Hkv, D, C, head_full,
                                       k_free, n_sink, n_local, idx, count, kmax);
  return fused_topk_kernel<DS, false>(l, q, bf16, proj, R, summ, U, Hq, Hkv, D, C, head_full,
                                      k_free, n_sink, n_local, idx, count, kmax);
}

template <int DS>
cudaError_t fused_topp_ds(const Launch& l, const void* q, bool bf16, const float* proj, int R,
                          const float* summ, int U, int Hq, int Hkv, int D, int C,
                          const uint8_t* head_full, float logit_scale, float p, int budget,
                          int n_sink, int n_local, int32_t* idx, int32_t* count, int kmax,
                          int32_t* n_p_out) {
  const int SN = next_pow2(std::min(budget, C));
  const size_t sh = topp_head_bytes(C, SN) + static_cast<size_t>(C) * 5 + 16;
  cudaError_t e = set_smem(reinterpret_cast<const void*>(score_select_topp_kernel<DS>), sh);
  if (e != cudaSuccess) return e;
  if (!l.after_query_copy) {
    score_select_topp_kernel<DS><<<U, kSelThreads, sh, l.stream>>>(
        q, bf16 ? 1 : 0, proj, R, summ, Hq, Hkv, D, C, head_full, logit_scale, p, budget, n_sink,
        n_local, idx, count, kmax, n_p_out, SN, 0);
    return cudaGetLastError();
  }
  // behind the query copy: start now, wait for it before reading q
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(U);
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = sh;
  cfg.stream = l.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, score_select_topp_kernel<DS>, q, bf16 ? 1 : 0, proj, R, summ,
                            Hq, Hkv, D, C, head_full, logit_scale, p, budget, n_sink, n_local, idx,
                            count, kmax, n_p_out, SN, 1);
}
}  // namespace

namespace {
// Cluster size for the cluster top-k, or 0: the largest power of two <= 8
// with B*Hkv*CS CTAs on the SMs, each CTA scoring at most kClRangeMax chunks
// and the kept candidates fitting the first CTA's kClCandMax slots.
int select_cluster_size(int U, int C, int k_free, int n_sink, int n_local, int num_sms) {
  if (U <= 0 || U > 65535 || C <= 0 || n_sink + n_local > 64) return 0;
  for (int CS = 8; CS >= 2; CS >>= 1) {
    if (static_cast<int64_t>(U) * CS > num_sms) continue;
    const int per = (C + CS - 1) / CS;
    const int KL = std::min(k_free, per);
    if (per <= kClRangeMax && CS * KL <= kClCandMax) return CS;
  }
  return 0;
}

// Cluster size for the per-head union (G query heads per unit), or 0.
int union_cluster_size(int U, int G, int C, int k_free, int n_sink, int n_local, int DS,
                       bool projected, int D, int num_sms) {
  if (U <= 0 || U > 65535 || C <= 0 || G > 8 || n_sink + n_local > 64) return 0;
  if (projected && G * D > 1024) return 0;  // the heads' raw queries share one 1024-float buffer
  for (int CS = 8; CS >= 2; CS >>= 1) {
    if (static_cast<int64_t>(U) * CS > num_sms) continue;
    const int per = (C + CS - 1) / CS;
    const int KL = std::min(k_free, per);
    if (per <= kClRangeMax && CS * KL <= kClCandMax &&
        union_cl_bytes(G, DS, per, KL, CS, C) <= 160 * 1024)
      return CS;
  }
  return 0;
}

template <int DS>
cudaError_t cluster_union_kernel(const Launch& l, const void* q, bool bf16, const float* proj,
                                 int R, const float* summ, int U, int Hq, int Hkv, int D, int C,
                                 const uint8_t* head_full, int k_free, int n_sink, int n_local,
                                 int32_t* idx, int32_t* count, int kmax, int CS) {
  const int G = Hq / Hkv, per = (C + CS - 1) / CS;
  const size_t sh = union_cl_bytes(G, DS, per, std::min(k_free, per), CS, C);
  cudaError_t e = set_smem(reinterpret_cast<const void*>(score_select_union_cluster_kernel<DS>), sh);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CS, U);
  cfg.blockDim = dim3(kClSelThreads);
  cfg.dynamicSmemBytes = sh;
  cfg.stream = l.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, score_select_union_cluster_kernel<DS>, q, bf16 ? 1 : 0, proj, R,
                            summ, Hq, Hkv, D, C, head_full, k_free, n_sink, n_local, idx, count,
                            kmax);
}

template <int DS>
cudaError_t cluster_topk_kernel(const Launch& l, const void* q, bool bf16, const float* proj,
                                int R, const float* summ, int U, int Hq, int Hkv, int D, int C,
                                const uint8_t* head_full, int k_free, int n_sink, int n_local,
                                int32_t* idx, int32_t* count, int kmax, int CS) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CS, U);
  cfg.blockDim = dim3(kClSelThreads);
  cfg.stream = l.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, score_select_topk_cluster_kernel<DS>, q, bf16 ? 1 : 0, proj, R,
                            summ, Hq, Hkv, D, C, head_full, k_free, n_sink, n_local, idx, count,
                            kmax);
}
}  // namespace

cudaError_t launch_score_select_topk(const Launch& l, const void* q, bool bf16, const float* proj,
                                     int R, const float* summ, int B, int Hq, int Hkv, int D, int C,
                                     const uint8_t* head_full, int k_free, int n_sink, int n_local,
                                     int32_t* idx, int32_t* count, int kmax, bool per_head_union) {
  const int U = B * Hkv;
  if (U == 0) return cudaSuccess;
  const int DSel = proj ? R : D;
  const int CSu = per_head_union ? union_cluster_size(U, Hq / Hkv, C, k_free, n_sink, n_local,
                                                      DSel, proj != nullptr, D, l.num_sms)
                                 : 0;
  if (CSu > 0) {
    switch (DSel) {
      case 16: return cluster_union_kernel<16>(l, q, bf16, proj, R, summ, U, Hq, Hkv, D, C, head_full, k_free, n_sink, n_local, idx, count, kmax, CSu);
      case 32: return cluster_union_kernel<32>(l, q, bf16, proj, R, summ, U, Hq, Hkv, D, C, head_full, k_free, n_sink, n_local, idx, count, kmax, CSu);
      case 64: return cluster_union_kernel<64>(l, q, bf16, proj, R, summ, U, Hq, Hkv, D, C, head_full, k_free, n_sink, n_local, idx, count, kmax, CSu);
      case 128: return cluster_union_kernel<128>(l, q, bf16, proj, R, summ, U, Hq, Hkv, D, C, head_full, k_free, n_sink, n_local, idx, count, kmax, CSu);
      default: return cudaErrorInvalidValue;
    }
  }
  const int CS = per_head_union ? 0 : select_cluster_size(U, C, k_free, n_sink, n_local, l.num_sms);
  if (CS > 0) {
    switch (proj ? R : D) {
      case 16: return cluster_topk_kernel<16>(l, q, bf16, proj, R, summ, U, Hq, Hkv, D, C, head_full, k_free, n_sink, n_local, idx, count, kmax, CS);
      case 32: return cluster_topk_kernel<32>(l, q, bf16, proj, R, summ, U, Hq, Hkv, D, C, head_full, k_free, n_sink, n_local, idx, count, kmax, CS);
      case 64: return cluster_topk_kernel<64>(l, q, bf16, proj, R, summ, U, Hq, Hkv, D, C, head_full, k_free, n_sink, n_local, idx, count, kmax, CS);
      case 128: return cluster_topk_kernel<128>(l, q, bf16, proj, R, summ, U, Hq, Hkv, D, C, head_full, k_free, n_sink, n_local, idx, count, kmax, CS);
      default: return cudaErrorInvalidValue;
    }
  }
  const bool pu = per_head_union;
  switch (proj ? R : D) {
    case 16: return fused_topk_ds<16>(l, q, bf16, proj, R, summ, U, Hq, Hkv, D, C, head_full, k_free, n_sink, n_local, idx, count, kmax, pu);
    case 32: return fused_topk_ds<32>(l, q, bf16, proj, R, summ, U, Hq, Hkv, D, C, head_full, k_free, n_sink, n_local, idx, count, kmax, pu);
    case 64: return fused_topk_ds<64>(l, q, bf16, proj, R, summ, U, Hq, Hkv, D, C, head_full, k_free, n_sink, n_local, idx, count, kmax, pu);
    case 128: return fused_topk_ds<128>(l, q, bf16, proj, R, summ, U, Hq, Hkv, D, C, head_full, k_free, n_sink, n_local, idx, count, kmax, pu);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_score_select_topp(const Launch& l, const void* q, bool bf16, const float* proj,
                                     int R, const float* summ, int B, int Hq, int Hkv, int D, int C,
                                     const uint8_t* head_full, float logit_scale, float p,
                                     int budget, int n_sink, int n_local, int32_t* idx,
                                     int32_t* count, int kmax, int32_t* n_p_out) {
  const int U = B * Hkv;
  if (U == 0) return cudaSuccess;
  switch (proj ? R : D) {
    case 16: return fused_topp_ds<16>(l, q, bf16, proj, R, summ, U, Hq, Hkv, D, C, head_full, logit_scale, p, budget, n_sink, n_local, idx, count, kmax, n_p_out);
    case 32: return fused_topp_ds<32>(l, q, bf16, proj, R, summ, U, Hq, Hkv, D, C, head_full, logit_scale, p, budget, n_sink, n_local, idx, count, kmax, n_p_out);
    case 64: return fused_topp_ds<64>(l, q, bf16, proj, R, summ, U, Hq, Hkv, D, C, head_full, logit_scale, p, budget, n_sink, n_local, idx, count, kmax, n_p_out);
    case 128: return fused_topp_ds<128>(l, q, bf16, proj, R, summ, U, Hq, Hkv, D, C, head_full, logit_scale, p, budget, n_sink, n_local, idx, count, kmax, n_p_out);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace csa
