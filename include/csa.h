/*
 * csa.h — C ABI of libcsa.so: query-adaptive chunk-sparse attention on NVIDIA
 * B200 (sm_100a).
 *
 * The method (pages of the surveyed subject):
 *   - the KV sequence is cut into chunks of L tokens, each summarised by one
 *     key (SSA summary, aitrends.kr/articles/69798, section "기술 상세";
 *     HiLS review "Hierarchical Sparse Attention Done Right", section 1,
 *     "Landmark Token"); this library summarises a chunk by the mean of its
 *     keys, optionally projected to a low rank (RTPurbo review "Full Attention
 *     Strikes Back", section 1, "Low-dimensional Projection");
 *   - each chunk is scored by the inner product of the query with its
 *     summary, s = q^T k_summary (SSA summary, section "방법론"), summed over
 *     the query heads of a GQA group (HiLS review, section 1, "GQA");
 *   - a chunk set is picked per (sequence, KV head) by top-k (SSA summary,
 *     "방법론"), dynamic top-p (RTPurbo review, section 1, "Dynamic Top-p
 *     Selection") or two-level meta-chunk -> chunk selection (SSA summary,
 *     "핵심 기여", H-SSA), always keeping sink and local chunks;
 *   - exact softmax attention runs over the raw KV of the chosen chunks as
 *     split-K partials from a compact index list, combined afterwards (SSA
 *     summary, "핵심 기여", decode kernel); full-attention and sparse heads run
 *     in one launch (Elastic Attention summary, section 2.3, fused kernel);
 *   - prefill runs block-sparse causal attention over a chunk set per query
 *     tile (SSA summary, "핵심 기여", block-skip prefill; HiLS review, section 3,
 *     union chunks of adjacent queries).
 *
 * Conventions for every call:
 *   - Every data pointer is a DEVICE pointer (cudaMalloc'd, or managed)
 *     owned by the caller, except the pinned host buffers of
 *     csa_decode_step_host.  The library allocates nothing, frees nothing and
 *     never blocks the host; each call enqueues kernels on `stream` (a
 *     cudaStream_t; NULL = legacy default stream) and returns.
 *   - Tensors are dense, row-major (last index fastest), in the layouts given
 *     per call.  K/V caches are [B, Hkv, T, D]: chunk c of head (b, h) is the
 *     contiguous block of rows [c*L, (c+1)*L).
 *   - Pointers must be 16-byte aligned.  A host pointer, a NULL required
 *     pointer, a non-positive size, or an inconsistent shape is rejected with
 *     CSA_ERR_INVALID_ARG before anything is launched; shapes outside what the
 *     kernels implement are rejected with CSA_ERR_UNSUPPORTED.  On any error
 *     nothing is enqueued, and csa_last_error_string() (thread-local) says why.
 *   - Faults the kernels detect on the device (an index out of range, a wait
 *     that exceeded its time limit) do not trap: the kernel records a code in
 *     a device-side status word and carries on or returns.
 *     csa_check_device_status() reads and clears it.
 *   - Calls on one stream are ordered; the library keeps no state between
 *     calls other than the device status word and process-wide settings
 *     (wait limit).
 */
#ifndef CSA_H_
#define CSA_H_

#include <stdint.h>

#if defined(__GNUC__)
#define CSA_API __attribute__((visibility("default")))
#else
#define CSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum csa_status {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = 1,  /* NULL / host pointer, bad size, misalignment, kmax too small */
  CSA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. D not in {64,128}) */
  CSA_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  CSA_ERR_TIMEOUT = 4,      /* a device-side bounded wait expired (read back later) */
  CSA_ERR_DEVICE_INDEX = 5  /* a kernel met a chunk index or count out of range */
} csa_status;

typedef enum csa_dtype { CSA_F32 = 0, CSA_BF16 = 1 } csa_dtype;

typedef void* csa_stream; /* a cudaStream_t */

/* Version of this ABI (major * 10000 + minor * 100 + patch). */
CSA_API int csa_version(void);

/* Why the last call on this thread failed ("" after success). */
CSA_API const char* csa_last_error_string(void);

/* Waits for `stream` to finish, then reads and clears the device status
 * word of the current device: CSA_OK, CSA_ERR_TIMEOUT or CSA_ERR_DEVICE_INDEX
 * (or CSA_ERR_CUDA if the synchronisation itself failed).  This is the one
 * call that blocks the host. */
CSA_API csa_status csa_check_device_status(csa_stream stream);

/* Time limit of every spin-wait inside the kernels, in nanoseconds (process
 * wide; default 2e9, or the CSA_WAIT_LIMIT_NS environment variable).  A wait
 * that exceeds it records CSA_ERR_TIMEOUT and the kernel returns. */
CSA_API void csa_set_wait_limit_ns(uint64_t ns);
CSA_API uint64_t csa_get_wait_limit_ns(void);

/* Diagnostic (no counterpart in the pages): launches one CTA that waits on
 * an mbarrier nothing ever arrives on, with a limit of `limit_ns`.  The wait
 * runs out, the kernel records CSA_ERR_TIMEOUT and returns, and the next
 * csa_check_device_status() reports it.  Shows that a stuck wait ends as a
 * status code, not a hang or a trap, and that the context stays usable. */
CSA_API csa_status csa_selftest_wait_timeout(uint64_t limit_ns, csa_stream stream);

/* ---------------------------------------------------------------- a0
 * Chunk summaries (precompute, once per cache).
 * summ[b,h,c,:] = (1/L) * sum_{j<L} K[b,h,c*L+j,:]            (proj == NULL, Ds = D)
 * summ[b,h,c,r] = sum_d proj[d,r] * (1/L) sum_j K[b,h,c*L+j,d]  (proj [D,R] fp32, Ds = R)
 * Basis: chunk summary keys (SSA summary "기술 상세"; HiLS review section 1)
 * with the chunk mean standing in for a learned gist/landmark key; low-rank
 * projection (RTPurbo review section 1).
 *   K     [B, Hkv, T, D] of `dtype`;  summ [B, Hkv, T/L, Ds] fp32 (output)
 *   D in {64, 128}, L >= 1, T % L == 0, R in {16, 32, 64, 128} when proj != NULL.
 * fp32 accumulation in row order. */
CSA_API csa_status csa_chunk_summaries(const void* K, csa_dtype dtype, int B, int Hkv, int64_t T,
                               int D, int L, const float* proj, int R, float* summ,
                               csa_stream stream);

/* Meta-summaries for two-level selection (H-SSA meta-gist stand-in, SSA
 * summary "핵심 기여" and glossary "Hierarchical Gist-of-Gist"):
 * meta[b,h,m,:] = (1/Gm) * sum_{j<Gm} summ[b,h,m*Gm+j,:].
 *   summ [B, Hkv, C, Ds] fp32 -> meta [B, Hkv, C/Gm, Ds] fp32;  C % Gm == 0, Ds <= 1024. */
CSA_API csa_status csa_meta_summaries(const float* summ, int B, int Hkv, int C, int Ds, int Gm,
                              float* meta, csa_stream stream);

/* ---------------------------------------------------------------- RoPE
 * Rotary position embedding, for the RoPE-aware split of the RTPurbo review
 * (section 1, "Low-dimensional Projection": the scoring projection is taken
 * before RoPE, which makes scores depend on distance): chunks are scored on
 * the pre-RoPE keys and query (summaries of the pre-RoPE cache,
 * csa_decode_step_desc.q_score), and attention runs on the rotated ones made
 * here.  The pages do not write RoPE out; this is the rotate-half form:
 * row r of x sits at position p = pos0 + (r mod period), and for i < D/2
 *   y[r,i]     = x[r,i] cos(p w_i) - x[r,i+D/2] sin(p w_i)
 *   y[r,i+D/2] = x[r,i+D/2] cos(p w_i) + x[r,i] sin(p w_i),  w_i = theta^(-2i/D).
 * The angle is reduced modulo 2 pi in double precision.
 *   x, y [rows, D] of `dtype` (y == x allowed); a K cache [B, H, T, D] is
 *   rows = B*H*T with period T, pos0 0; a decode query [B, Hq, D] at position
 *   t is rows = B*Hq with period 1, pos0 t.  D even, D <= 512, theta > 1. */
CSA_API csa_status csa_rope(const void* x, void* y, csa_dtype dtype, int64_t rows, int D,
                            int64_t period, int64_t pos0, float theta, csa_stream stream);

/* ---------------------------------------------------------------- token-level sparsity
 * Token Sparse Attention for prefill (Token Sparse Attention summary,
 * gist.science/ko/paper/2602.03216, section 2).  bf16 Q [B, S, Hq, D] and
 * K, V [B, Hkv, S, D]; the GQA group of KV head h is query heads h*G..h*G+G-1.
 *
 * csa_token_importance: importance of every key from a proxy attention map
 * of the recent queries ("동적 토큰 커버리지"): the last n_obs query rows of
 * every query head of the group attend causally (key j <= the row's
 * position) with softmax(scale * q.k); imp[b, h, j] = the sum over those
 * G*n_obs rows of key j's weight.  Two passes over K on the tensor cores.
 * imp [B, Hkv, S] fp32 (output); scratch >= csa_token_importance_scratch_bytes.
 * D 64 or 128; n_obs a multiple of 8 with (Hq/Hkv) * n_obs <= 512. */
CSA_API int64_t csa_token_importance_scratch_bytes(int B, int S, int Hq, int Hkv, int n_obs);
CSA_API csa_status csa_token_importance(const void* Q, const void* K, int B, int S, int Hq,
                                        int Hkv, int D, int n_obs, float scale, float* imp,
                                        void* scratch, int64_t scratch_bytes,
                                        csa_stream stream);

/* csa_token_budget: Dynamic Token Coverage.  The masses m_j = sum_h
 * imp[b, h, j] are normalised; the least important tokens are dropped while
 * their mass stays <= tau, i.e. k_seq[b] = the fewest tokens whose mass
 * reaches 1 - tau.  k_unit[b*Hkv + h] = k_seq[b] rounded up to a multiple of
 * `tile` (at most S): the token count every KV head of sequence b keeps.
 * Float sums: a cut within rounding of a tie may land one token apart from
 * exact arithmetic.  tau in [0, 1); S <= 32768, or up to 131072 when B * 8
 * <= the number of SMs (one cluster of 8 CTAs per sequence); other sizes
 * return CSA_ERR_UNSUPPORTED. */
CSA_API csa_status csa_token_budget(const float* imp, int B, int S, int Hkv, float tau, int tile,
                                    int32_t* k_seq, int32_t* k_unit, csa_stream stream);

/* csa_token_sparse_prefill: the whole prefill ("핵심 아키텍처", "헤드별 선택"):
 * importance and budget as above (tile 64), each KV head's own k_unit most
 * important tokens (score desc, lower index on ties; csa_select_topk's
 * order), then compress: the kept tokens' K and V rows and the group's query
 * rows, in position order, into dense tensors; dense causal attention of the
 * compressed sequences on the tensor cores (the block-sparse prefill kernel
 * with every earlier tile visible); decompress: each output row back to its
 * position, every other row of O set to 0.
 *   O [B, S, Hq, D] bf16 (output); budget_out [B] int32 device (output, the
 *   unrounded k_seq).  D = 128, Hq/Hkv = 4, S % 64 == 0, S <= 32768, or up
 *   to 131072 when B * Hkv * 8 <= the number of SMs (the budget and the
 *   token choice then run on their cluster paths); else CSA_ERR_UNSUPPORTED.
 *   workspace >= csa_token_sparse_workspace_bytes(B, S, Hq, Hkv, D, n_obs).
 * Every step runs on the device from the budgets the device computed: the
 * compressed buffers are laid out for S kept tokens, and the dense attention
 * runs over the tiles within each KV head's budget, skipping the rest.  The
 * call never blocks the host; it enqueues only kernel launches on `stream`. */
CSA_API int64_t csa_token_sparse_workspace_bytes(int B, int S, int Hq, int Hkv, int D, int n_obs);
CSA_API csa_status csa_token_sparse_prefill(const void* Q, const void* K, const void* V, int B,
                                            int S, int Hq, int Hkv, int D, int n_obs, float tau,
                                            float scale, void* workspace,
                                            int64_t workspace_bytes, void* O,
                                            int32_t* budget_out, csa_stream stream);

/* The steps of csa_token_sparse_prefill after the budget, as separate calls
 * (the same kernels, in the same order): compress ("핵심 아키텍처": gather
 * the kept tokens), attend (dense causal attention of the compressed
 * sequences) and decompress (scatter back).  Same shapes and limits as the
 * whole call (D = 128, Hq/Hkv = 4, S % 64 == 0, S <= 131072; csa_token_select
 * above 32768 only when B * Hkv * 8 <= the number of SMs); compressed
 * buffers Qc [B, S, Hq, D], Kc/Vc [B, Hkv, S, D], Oc [B, S, Hq, D] bf16,
 * laid out for S kept tokens.
 *
 * csa_token_select: each KV head's own k_unit[b*Hkv + h] most important
 *   tokens (importance desc, lower position on ties), ascending, into
 *   idx [B*Hkv, S] int32 (unused slots -1) and count [B*Hkv] int32 ("헤드별
 *   선택"); imp and k_unit as csa_token_importance / csa_token_budget give
 *   them.
 * csa_token_compress: compressed row t < count[u] of unit u = b*Hkv + h gets
 *   token idx[u, t]: its K and V rows into Kc/Vc[b, h, t], the query rows of
 *   the group's heads into Qc[b, t, h*G .. h*G+G-1].  Rows past a unit's
 *   count are not written.
 * csa_token_attend: dense causal attention of each unit's first k_unit[u]
 *   compressed rows (k_unit a multiple of 64, as csa_token_budget gives it),
 *   64-row tile t attending to tiles 0 .. t; the rows of Oc past a unit's
 *   k_unit are not written.  No scratch: the tiles are read from k_unit on
 *   the device.
 * csa_token_decompress: O[b, s, h*G+g] = Oc[b, t, h*G+g] where idx[u, t] = s,
 *   0 for the positions a head did not keep; every row of O is written.
 *   scratch >= csa_token_decompress_scratch_bytes(B, S, Hkv) (the inverse
 *   map). */
CSA_API csa_status csa_token_select(const float* imp, int B, int S, int Hkv,
                                    const int32_t* k_unit, int32_t* idx, int32_t* count,
                                    csa_stream stream);
CSA_API csa_status csa_token_compress(const void* Q, const void* K, const void* V,
                                      const int32_t* idx, const int32_t* count, int B, int S,
                                      int Hq, int Hkv, int D, void* Qc, void* Kc, void* Vc,
                                      csa_stream stream);
CSA_API csa_status csa_token_attend(const void* Qc, const void* Kc, const void* Vc,
                                    const int32_t* k_unit, int B, int S, int Hq, int Hkv, int D,
                                    float scale, void* Oc, csa_stream stream);
CSA_API int64_t csa_token_decompress_scratch_bytes(int B, int S, int Hkv);
CSA_API csa_status csa_token_decompress(const void* Oc, const int32_t* idx, const int32_t* count,
                                        int B, int S, int Hq, int Hkv, int D, void* scratch,
                                        int64_t scratch_bytes, void* O, csa_stream stream);

/* ---------------------------------------------------------------- a7
 * Tile-mean queries for prefill (HiLS review section 3: adjacent queries
 * share one chunk union):  qbar[b,t,h,:] = (1/tile_m) sum_{i<tile_m} Q[b,t*tile_m+i,h,:].
 *   Q [B, S, Hq, D] of `dtype` -> qbar [B, S/tile_m, Hq, D] fp32;  S % tile_m == 0, D <= 1024,
 *   Hq*D a multiple of 8 (bf16) or 4 (fp32), else CSA_ERR_UNSUPPORTED. */
CSA_API csa_status csa_tile_mean_q(const void* Q, csa_dtype dtype, int B, int S, int Hq, int D,
                           int tile_m, float* qbar, csa_stream stream);

/* ---------------------------------------------------------------- a1
 * Chunk scores (SSA summary "방법론": s_{t,m} = q_t^T k_{g_m}; group-level
 * selection for GQA, HiLS review section 1):
 *   scores[b,h,n,c] = sum_{g<G} qt[b,n,h*G+g,:] . summ[b,h,c,:],   G = Hq/Hkv,
 *   qt = q (proj == NULL, Ds = D) or qt = proj^T q (proj [D,R] fp32, Ds = R).
 *   q      [B, Nq, Hq, D] of `q_dtype` (decode: Nq = 1; prefill: the tile means, Nq = tiles)
 *   summ   [B, Hkv, C, Ds] fp32;  scores [B, Hkv, Nq, C] fp32 (output)
 *   head_full  NULL or [Hkv] bytes: rows of heads with head_full[h] != 0 are not
 *              written (those heads attend to every chunk).
 *   causal_tile_m, causal_L: 0, 0 for no mask; otherwise row n sees the chunks
 *              c < ((n+1)*causal_tile_m - 1)/causal_L + 1 and the others get -inf.
 *   Ds in {16, 32, 64, 128}; D <= 1024; Hq % Hkv == 0. */
CSA_API csa_status csa_score_chunks(const void* q, csa_dtype q_dtype, const float* proj, int R,
                            const float* summ, int B, int Nq, int Hq, int Hkv, int D, int C,
                            const uint8_t* head_full, int causal_tile_m, int causal_L,
                            float* scores, csa_stream stream);

/* ---------------------------------------------------------------- a2
 * Top-k chunk selection per unit (SSA summary "방법론"; the compact list of
 * the decode kernel, "핵심 기여").  Unit u sees chunks [0, v) with
 * v = n_valid ? n_valid[u] : C.  Forced set F = the first n_sink and the last
 * n_local of [0, v).  The other chunks are ranked by (score desc, index asc;
 * -0 == +0) and the first k_free are kept.  Result F U top, ascending.
 *   scores [U, C] fp32 (finite);  n_valid NULL or [U] int32 in [0, C]
 *   idx [U, kmax] int32 (output, ascending, unused slots = -1);  count [U] int32 (output)
 *   kmax >= min(C, k_free + n_sink + n_local);  C <= 32768. */
CSA_API csa_status csa_select_topk(const float* scores, int U, int C, const int32_t* n_valid,
                           int k_free, int n_sink, int n_local, int32_t* idx, int32_t* count,
                           int kmax, csa_stream stream);

/* csa_select_topk for the query tiles of a causal prefill (SSA summary
 * "핵심 기여": block-skip prefill; HiLS review section 3: one chunk union per
 * group of adjacent queries): unit u is tile t = u mod n_tiles of its
 * (sequence, KV head), and sees the chunks [0, v) with
 *   v = min(C, ((t + 1) * tile_m - 1) / L + 1)
 * (every chunk holding a key at or before the tile's last row), so that the
 * forced local chunk (n_local = 1) is the diagonal one.  Arguments and
 * results otherwise as csa_select_topk; U % n_tiles == 0. */
CSA_API csa_status csa_select_topk_causal(const float* scores, int U, int C, int n_tiles,
                                          int tile_m, int L, int k_free, int n_sink, int n_local,
                                          int32_t* idx, int32_t* count, int kmax,
                                          csa_stream stream);

/* ---------------------------------------------------------------- a3
 * Dynamic top-p selection per unit (RTPurbo review section 1, "Dynamic Top-p
 * Selection"; chunk mass from the HiLS review's chunk-mass surrogate):
 * pi_c = softmax_c(scores[u,c] * logit_scale) over all C chunks; chunks
 * ordered by (pi desc, index asc); n_p = smallest n with sum of the first n
 * pi >= p; the first min(n_p, budget) are kept, then F (first n_sink, last
 * n_local) is added.  Result ascending.
 *   scores [U, C] fp32;  idx [U, kmax] int32, count [U] int32 (outputs)
 *   n_p_out NULL or [U] int32: n_p when n_p <= budget, else budget + 1
 *   0 < p <= 1;  1 <= budget <= 2048;  kmax >= min(C, budget + n_sink + n_local);  C <= 32768. */
CSA_API csa_status csa_select_topp(const float* scores, int U, int C, float logit_scale, float p,
                           int budget, int n_sink, int n_local, int32_t* idx, int32_t* count,
                           int kmax, int32_t* n_p_out, csa_stream stream);

/* ---------------------------------------------------------------- a4
 * Two-level selection per unit (b, h) (SSA summary "핵심 기여", H-SSA:
 * coarse selection on meta-gists, then re-scoring inside the kept segments):
 * meta score = sum_g q[b,h*G+g,:] . meta[b,h,m,:]; keep the top_meta metas by
 * (score desc, index asc); score their children the same way; among children
 * not in F keep the k_free best; add F (first n_sink, last n_local of [0, C)).
 *   q [B, Hq, D] of `q_dtype`;  meta [B, Hkv, C/Gm, D] fp32;  summ [B, Hkv, C, D] fp32
 *   idx [B*Hkv, kmax] int32, count [B*Hkv] int32 (outputs, ascending)
 *   D in {64, 128};  top_meta * Gm <= 8192;  C / Gm <= 8192;  C <= 32768;
 *   kmax >= min(C, k_free + n_sink + n_local). */
CSA_API csa_status csa_select_hier(const void* q, csa_dtype q_dtype, const float* meta,
                           const float* summ, int B, int Hq, int Hkv, int D, int C, int Gm,
                           int top_meta, int k_free, int n_sink, int n_local, int32_t* idx,
                           int32_t* count, int kmax, csa_stream stream);

/* ---------------------------------------------------------------- a5
 * Sparse split-K decode (SSA summary "핵심 기여": compact index list + split-K
 * partial attention; Elastic Attention summary section 2.3: full and sparse
 * heads in one launch).
 * Unit u = b*Hkv + h owns the chunk list idx[u, 0:count[u]] (or, if
 * head_full[h] != 0, every chunk 0..T/L-1; idx/count of that unit are not
 * read).  All units' lists are laid end to end (unit-major), N chunks in all,
 * and cut into num_parts pieces [floor(c*N/P), floor((c+1)*N/P)); the s-th
 * non-empty intersection of unit u with a piece is split s of that unit.  For
 * every query head g of the unit and every split s:
 *   o_part[b, h*G+g, s, :] = sum_j softmax(scale * q.k_j) v_j over the split's tokens,
 *   lse_part[b, h*G+g, s]  = log sum_j exp(scale * q.k_j)          (natural log)
 * and slots s >= the unit's split count get lse = -inf (their o is not written).
 *   q [B, Hq, D], K/V [B, Hkv, T, D] of `dtype` (CSA_BF16: bf16 tensor-core
 *   dot products with fp32 accumulation; CSA_F32: fp32 throughout)
 *   idx [B*Hkv, kmax] int32 in [0, T/L);  count [B*Hkv] int32 in [0, kmax]
 *   num_parts: 0 = csa_decode_default_parts(); max_splits >= the effective num_parts
 *   o_part [B, Hq, max_splits, D] fp32;  lse_part [B, Hq, max_splits] fp32 (outputs)
 *   D in {64, 128};  L in {64, 128};  T % L == 0;  Hq/Hkv in {1, 2, 4, 8};
 *   B*Hkv <= 4096;  B*Hkv*T < 2^31.
 * An idx entry out of range or count > kmax records CSA_ERR_DEVICE_INDEX
 * (the chunk is replaced by chunk 0 / the count clamped) instead of faulting. */
CSA_API csa_status csa_sparse_decode(const void* q, const void* K, const void* V, csa_dtype dtype,
                             const int32_t* idx, const int32_t* count, int kmax,
                             const uint8_t* head_full, int B, int Hq, int Hkv, int D, int64_t T,
                             int L, float scale, int num_parts, int max_splits, float* o_part,
                             float* lse_part, csa_stream stream);

/* Number of pieces csa_sparse_decode uses when num_parts == 0, on the
 * current device (a multiple of the SM count); < 0 on error. */
CSA_API int csa_decode_default_parts(csa_dtype dtype, int D, int L);

/* Fused a1 + a2 (decode, Nq = 1): the scores of csa_score_chunks computed
 * straight into shared memory (one CTA per unit, or one thread-block cluster
 * per unit when the lists are short), then the top-k of csa_select_topk;
 * same arithmetic, so the index lists equal the two-call path's bit for bit.  Units of heads with head_full[h] != 0 get count 0 and
 * an all -1 row (csa_sparse_decode reads every chunk for them).
 *   q [B, Hq, D];  proj NULL or [D, R];  summ [B, Hkv, C, Ds] fp32
 *   idx [B*Hkv, kmax], count [B*Hkv] (outputs);  same limits as the two calls. */
CSA_API csa_status csa_score_select_topk(const void* q, csa_dtype q_dtype, const float* proj, int R,
                                         const float* summ, int B, int Hq, int Hkv, int D, int C,
                                         const uint8_t* head_full, int k_free, int n_sink,
                                         int n_local, int32_t* idx, int32_t* count, int kmax,
                                         csa_stream stream);

/* Per-head top-k with the GQA union (SSA summary, glossary entry
 * "Grouped-Query Attention": each query head selects its own top-k chunks and
 * the group loads the union of the selected chunks once, so the decode reads
 * each KV chunk once per group).  Per unit (b, h): for each query head g of
 * the group, S_g[c] = q~_g . summ[b, h, c] (q~ = P^T q_g with a projection);
 * head g keeps its k_free best non-forced chunks by (score desc, index asc);
 * the list is the ascending union over the heads plus the forced set (first
 * n_sink and last n_local chunks).  Arguments, layouts, full-head handling
 * and errors as csa_score_select_topk, except that kmax must be
 * >= min(C, (Hq/Hkv) * k_free + n_sink + n_local). */
CSA_API csa_status csa_score_select_topk_union(const void* q, csa_dtype q_dtype, const float* proj,
                                               int R, const float* summ, int B, int Hq, int Hkv,
                                               int D, int C, const uint8_t* head_full, int k_free,
                                               int n_sink, int n_local, int32_t* idx,
                                               int32_t* count, int kmax, csa_stream stream);

/* Fused a1 + a3 (decode): csa_score_chunks then csa_select_topp in one CTA
 * per unit (bit-identical to the two calls); full heads as above (n_p_out 0). */
CSA_API csa_status csa_score_select_topp(const void* q, csa_dtype q_dtype, const float* proj, int R,
                                         const float* summ, int B, int Hq, int Hkv, int D, int C,
                                         const uint8_t* head_full, float logit_scale, float p,
                                         int budget, int n_sink, int n_local, int32_t* idx,
                                         int32_t* count, int kmax, int32_t* n_p_out,
                                         csa_stream stream);

/* Bytes of device workspace csa_sparse_decode_merged needs (num_parts 0 =
 * the default piece count of the current device); < 0 on bad sizes. */
CSA_API int64_t csa_decode_workspace_bytes(int B, int Hq, int Hkv, int D, int num_parts);

/* a5 + a6 in one launch (SSA summary "핵심 기여": split-K partials combined):
 * the decode of csa_sparse_decode, after which the last CTA to finish a unit
 * merges that unit's splits (the log-sum-exp merge of csa_lse_merge) into
 *   out[b, h*G+g, :] (out_dtype) and lse_out[b, h*G+g] (natural log; NULL ok).
 * A unit with a single split writes its output directly; a unit with no
 * chunks gets out = 0, lse = -inf.
 * `workspace` (caller-owned device memory, >= csa_decode_workspace_bytes())
 * holds the split partials and one arrival counter per unit.  The counters
 * must be zero before the first call (zero the workspace once); every call
 * that completes leaves them zero again.  After a call that reported
 * CSA_ERR_TIMEOUT, zero the workspace before reusing it.  Calls that share a
 * workspace must not overlap on the GPU.
 *   num_parts <= 256 (0 = default); other arguments as csa_sparse_decode. */
CSA_API csa_status csa_sparse_decode_merged(const void* q, const void* K, const void* V,
                                            csa_dtype dtype, const int32_t* idx,
                                            const int32_t* count, int kmax,
                                            const uint8_t* head_full, int B, int Hq, int Hkv,
                                            int D, int64_t T, int L, float scale, int num_parts,
                                            void* workspace, int64_t workspace_bytes, void* out,
                                            csa_dtype out_dtype, float* lse_out,
                                            csa_stream stream);

/* The merged decode above for callers that cannot allocate device memory
 * (the pages have no counterpart: this is a deployment convenience).  An
 * application that manages all device memory through its own pool and
 * forbids other allocations, or a serving loop that must not call cudaMalloc
 * (which can synchronise the device) on its hot path, can call this instead
 * of csa_sparse_decode_merged: it takes the same arguments minus the
 * workspace and allocates nothing.  Its scratch (split partials and per-unit
 * counters) is a fixed 16 MiB area inside the library, held by every GPU
 * that loads the library until the process exits.
 *   - Shapes whose scratch (csa_decode_workspace_bytes()) exceeds 16 MiB are
 *     rejected with CSA_ERR_UNSUPPORTED (use fewer pieces, or the
 *     workspace variant).
 *   - The first call on a device looks up the area's device address; make
 *     that first call before any stream capture on that device.
 *   - The area starts zeroed when the library loads and keeps what each
 *     call leaves; every call clears its counters on `stream` after its
 *     decode, so the next call starts clean.  All calls share the one area:
 *     calls that overlap on the GPU (other streams, other host threads)
 *     race and must be serialised by the caller.  A call rejected on its
 *     arguments enqueues nothing. */
CSA_API csa_status csa_sparse_decode_merged_noalloc(const void* q, const void* K, const void* V,
                                                    csa_dtype dtype, const int32_t* idx,
                                                    const int32_t* count, int kmax,
                                                    const uint8_t* head_full, int B, int Hq,
                                                    int Hkv, int D, int64_t T, int L, float scale,
                                                    int num_parts, void* out, csa_dtype out_dtype,
                                                    float* lse_out, csa_stream stream);

/* ---------------------------------------------------------------- hybrid context
 * The merged decode over the hybrid context of the SSA summary: each sparse
 * unit's query heads attend, in one softmax and with the same scale for gist
 * and raw logits, over the raw tokens of its selected chunks and over gist
 * rows, as `gist_scope` says:
 *   CSA_GIST_SELECTED: the gist rows of the selected chunks only (SSA
 *     summary, sections "방법론" and "기술 상세": only the top-k chunks are
 *     brought back, each with its gist KV and its raw KV; K_hybrid / V_hybrid
 *     are the union of the gist and raw KV of I_t).
 *   CSA_GIST_ALL: the gist row of every chunk of the unit (the glossary entry
 *     "Selective Unfolding" read as the context: the query meets every
 *     chunk's gist token and the raw tokens of the top-k chunks are added).
 * Full-attention KV heads (head_full) attend over their raw tokens only.  A
 * sparse unit with no selected chunk gets out = 0, lse = -inf in the
 * selected scope (an empty context), and its gist rows alone in the other.
 *   Kg, Vg [B, Hkv, C, D] bf16, C = T / L, 16-byte aligned: gist key / value
 *   of chunk c of unit (b, h) at row c (the model's gist KV; a synthetic
 *   workload draws them or uses the chunk means as a stand-in).
 *   Other arguments, outputs, workspace and errors as
 *   csa_sparse_decode_merged; bf16 caches only (CSA_ERR_UNSUPPORTED for
 *   fp32); CSA_ERR_INVALID_ARG for a gist_scope outside the enum.  The gist
 *   rows are read as extra chunks of each sparse unit: ceil(C/L) chunks of
 *   contiguous rows (scope ALL, by TMA), or ceil(n/L) chunks of the n
 *   selected chunks' rows gathered with 16-byte copies (scope SELECTED); K
 *   and V: 2*D*2 bytes per gist row. */
typedef enum csa_gist_scope {
  CSA_GIST_SELECTED = 0,
  CSA_GIST_ALL = 1
} csa_gist_scope;

CSA_API csa_status csa_sparse_decode_merged_hybrid(const void* q, const void* K, const void* V,
                                                   const void* Kg, const void* Vg,
                                                   int gist_scope, csa_dtype dtype,
                                                   const int32_t* idx, const int32_t* count,
                                                   int kmax, const uint8_t* head_full, int B,
                                                   int Hq, int Hkv, int D, int64_t T, int L,
                                                   float scale, int num_parts, void* workspace,
                                                   int64_t workspace_bytes, void* out,
                                                   csa_dtype out_dtype, float* lse_out,
                                                   csa_stream stream);

/* ---------------------------------------------------------------- a1-a6 in one call
 * A whole decode step: the selection (csa_score_select_topk,
 * csa_score_select_topk_union, csa_score_select_topp or csa_select_hier,
 * by `mode`) followed by the merged split-K
 * decode (csa_sparse_decode_merged), with the same results.  The decode is
 * launched with programmatic dependent launch and works in two phases: the
 * chunks of full-attention heads first, which do not depend on the
 * selection and so stream while it runs, then the selected chunks of the
 * sparse heads once the selection has completed (SSA summary "핵심 기여";
 * Elastic Attention summary section 2.3: full and sparse heads in one pass).
 * bf16 caches only.  Fields of the descriptor are the arguments of those
 * calls.  num_parts 0 = the number of SMs (at most 256).  When head_full is
 * given, the last min(B*Hkv + P - #SMs, P - 1) CTAs (those that find the
 * selection's CTAs on their SMs and start late) take only selected chunks.
 * The workspace must be sized for the P the
 * call uses (csa_decode_workspace_bytes(B, Hq, Hkv, D, num_parts) with the
 * same num_parts, 0 included, is always enough) and start zeroed once; each
 * call leaves it zeroed again.  Errors: as the underlying calls; nothing is
 * enqueued when an argument is rejected, and CSA_ERR_UNSUPPORTED for a
 * fp32 cache (use the separate calls).  The step is two kernel launches on
 * one stream and is safe to capture in a CUDA graph. */
typedef enum csa_select_mode {
  CSA_SELECT_TOPK = 0,
  CSA_SELECT_TOPP = 1,
  CSA_SELECT_HIER = 2,
  CSA_SELECT_TOPK_UNION = 3 /* csa_score_select_topk_union */
} csa_select_mode;

typedef struct csa_decode_step_desc {
  /* query and KV cache */
  const void* q;       /* [B, Hq, D] bf16 */
  const void* K;       /* [B, Hkv, T, D] bf16 */
  const void* V;       /* [B, Hkv, T, D] bf16 */
  int B, Hq, Hkv, D;
  int64_t T;
  int L;
  float scale;
  const uint8_t* head_full; /* NULL or [Hkv] */
  /* selection */
  int mode;            /* csa_select_mode */
  const float* summ;   /* [B, Hkv, C, Ds] fp32 */
  const float* proj;   /* top-k / top-p: NULL or [D, R] fp32 */
  int R;
  const float* meta;   /* hierarchical: [B, Hkv, C/Gm, D] fp32 */
  int Gm, top_meta;
  int k_free, n_sink, n_local;
  float logit_scale, p;  /* top-p */
  int budget;            /* top-p */
  int32_t* idx;          /* [B*Hkv, kmax] (output) */
  int32_t* count;        /* [B*Hkv] (output) */
  int kmax;
  int32_t* n_p_out;      /* top-p: NULL or [B*Hkv] (output) */
  /* decode and merge */
  int num_parts;
  void* workspace;       /* >= csa_decode_workspace_bytes(B, Hq, Hkv, D, num_parts) */
  int64_t workspace_bytes;
  void* out;             /* [B, Hq, D] of out_dtype (output) */
  csa_dtype out_dtype;
  float* lse_out;        /* NULL or [B, Hq] (output) */
  /* hybrid context (as csa_sparse_decode_merged_hybrid): NULL, NULL = off,
   * else both [B, Hkv, T/L, D] bf16 gist keys and values, over the gist rows
   * of gist_scope (csa_gist_scope; 0 = CSA_GIST_SELECTED) */
  const void* Kg;
  const void* Vg;
  int gist_scope;
  /* RoPE-aware split (see csa_rope): NULL = score with q; else the pre-RoPE
   * query [B, Hq, D] bf16 the selection scores with (against summaries of
   * the pre-RoPE keys), while the decode attends with q (rotated) over the
   * rotated cache K */
  const void* q_score;
} csa_decode_step_desc;

CSA_API csa_status csa_decode_step(const csa_decode_step_desc* d, csa_stream stream);

/* The same step with the query and the result in host memory, for a caller
 * whose query arrives on the host: q_host ([B, Hq, D] bf16) is brought into
 * the device buffer d->q, the step of csa_decode_step runs, and its output
 * ([B, Hq, D] of out_dtype) lands in out_host and, when lse_host is given,
 * its lse ([B, Hq] fp32; d->lse_out then required) in lse_host.  All on
 * `stream`, asynchronous: the host reads out_host after synchronising it.
 * q_host, out_host and lse_host must be pinned host memory (cudaHostAlloc
 * or cudaHostRegister), else CSA_ERR_INVALID_ARG.  When that memory is
 * mapped into the device's address space (every pinned allocation under
 * unified addressing) and 16-byte aligned, the SMs read the query from it
 * (one small copy kernel) and the decode stores the result straight into
 * it; d->out and d->lse_out are then left as they were.  Otherwise the
 * copies are cudaMemcpyAsync transfers and d->out / d->lse_out hold the
 * result too.  Either way the transfers happen when the stream reaches
 * them: q_host must keep the query, and out_host / lse_host must not be
 * read, until the stream has passed the call.  The call captures into a CUDA graph, whose replays read and
 * write the same host buffers.  CSA_ERR_UNSUPPORTED with q_score set (the
 * RoPE-aware split rotates the query on the device: csa_rope, then
 * csa_decode_step).  Every argument, the selection's included, is checked
 * before the query copy: a rejected call enqueues nothing. */
CSA_API csa_status csa_decode_step_host(const csa_decode_step_desc* d, const void* q_host,
                                        void* out_host, float* lse_host, csa_stream stream);

/* ---------------------------------------------------------------- a6
 * Log-sum-exp merge of split-K partials (SSA summary "핵심 기여": split-K
 * partials combined):
 *   lse[r] = log sum_s exp(lse_part[r,s]);  out[r,:] = sum_s exp(lse_part[r,s] - lse[r]) o_part[r,s,:]
 * over the slots with lse_part > -inf (others are not read; a row with none
 * gives out = 0, lse = -inf).
 *   o_part [rows, max_splits, D] fp32;  lse_part [rows, max_splits] fp32
 *   out [rows, D] of out_dtype (output);  lse_out NULL or [rows] fp32 (output)
 *   D % 4 == 0, D <= 512, max_splits <= 16384. */
CSA_API csa_status csa_lse_merge(const float* o_part, const float* lse_part, int rows, int max_splits,
                         int D, void* out, csa_dtype out_dtype, float* lse_out,
                         csa_stream stream);

/* ---------------------------------------------------------------- a8
 * Block-sparse causal prefill (SSA summary "핵심 기여": block-skip prefill;
 * HiLS review section 3: one chunk union per group of adjacent queries).
 * For query tile t (rows t*tile_m .. +tile_m) and KV head h, the tile's chunk
 * list is idx[u, 0:count[u]], u = (b*Hkv + h)*(S/tile_m) + t.  Query row i of
 * head g in the group attends causally to the tokens j of those chunks with
 * j <= t*tile_m + i:
 *   O[b, t*tile_m+i, h*G+g, :] = sum_j softmax(scale * q.k_j) v_j   (bf16 out)
 * Rows with no visible token get 0.  Tensor-core (tcgen05) bf16 products,
 * fp32 accumulation and softmax.
 *   Q [B, S, Hq, D] bf16;  K/V [B, Hkv, S, D] bf16;  O [B, S, Hq, D] bf16 (output)
 *   idx [B*Hkv*(S/tile_m), kmax] int32 ascending in [0, S/L);  count [same] int32
 *   implemented: D = 128, tile_m = L = 64, Hq/Hkv = 4;  B*Hkv*S < 2^31. */
CSA_API csa_status csa_block_sparse_prefill(const void* Q, const void* K, const void* V,
                                    const int32_t* idx, const int32_t* count, int kmax, int B,
                                    int S, int Hq, int Hkv, int D, int tile_m, int L,
                                    float scale, void* O, csa_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H_ */
