// Internal launcher interface between the C ABI (api.cu) and the kernel files.
// Launchers assume validated arguments and return the launch's cudaError_t.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "common.cuh"

namespace csa {

// Sets the thread-local message returned by csa_last_error_string().
void set_last_error(const std::string& why);

struct Launch {
  cudaStream_t stream;
  DevErr err;
  int num_sms;
  // the launch follows a kernel that writes the query it reads (a host-query
  // copy): a launcher that supports it starts behind that kernel with
  // programmatic dependent launch and waits for it before reading the query
  bool after_query_copy = false;
};

// summaries.cu
cudaError_t launch_chunk_summaries(const Launch& l, const void* K, bool bf16, int U, int64_t T,
                                   int D, int L, const float* proj, int R, float* summ);
cudaError_t launch_meta_summaries(const Launch& l, const float* summ, int U, int C, int Ds, int Gm,
                                  float* meta);
cudaError_t launch_tile_mean(const Launch& l, const void* Q, bool bf16, int B, int S, int Hq, int D,
                             int tile_m, float* qbar);

// score.cu
cudaError_t launch_score(const Launch& l, const void* q, bool bf16, const float* proj, int R,
                         const float* summ, int B, int Nq, int Hq, int Hkv, int D, int C,
                         const uint8_t* head_full, int causal_tile_m, int causal_L,
                         float* scores);

// select.cu
// causal_tiles > 0: unit u is query tile u % causal_tiles of a causal
// prefill and sees the chunks c < ((t + 1) * causal_tile_m - 1) / causal_L + 1
// (n_valid is then ignored).  inv (optional, [U, C]): when the long-row
// cluster kernel runs, it also writes every position's slot in its unit's
// list (or -1) and sets *inv_done; otherwise *inv_done is false.
// The long-row top-k (one cluster of 8 CTAs per unit) runs for these sizes
// (rows of C >= 8192 keys, nothing forced).
bool topk_cluster_fits(int U, int C, int num_sms);
cudaError_t launch_select_topk(const Launch& l, const float* scores, int U, int C,
                               const int32_t* n_valid, int k_free, int n_sink, int n_local,
                               int32_t* idx, int32_t* count, int kmax,
                               const int32_t* k_dev = nullptr, int causal_tiles = 0,
                               int causal_tile_m = 0, int causal_L = 0, int32_t* inv = nullptr,
                               bool* inv_done = nullptr);
cudaError_t launch_select_topp(const Launch& l, const float* scores, int U, int C,
                               float logit_scale, float p, int budget, int n_sink, int n_local,
                               int32_t* idx, int32_t* count, int kmax, int32_t* n_p_out);
cudaError_t launch_select_hier(const Launch& l, const void* q, bool bf16, const float* meta,
                               const float* summ, int B, int Hq, int Hkv, int D, int C, int Gm,
                               int top_meta, int k_free, int n_sink, int n_local, int32_t* idx,
                               int32_t* count, int kmax);

cudaError_t launch_score_select_topk(const Launch& l, const void* q, bool bf16, const float* proj,
                                     int R, const float* summ, int B, int Hq, int Hkv, int D, int C,
                                     const uint8_t* head_full, int k_free, int n_sink, int n_local,
                                     int32_t* idx, int32_t* count, int kmax,
                                     bool per_head_union = false);
cudaError_t launch_score_select_topp(const Launch& l, const void* q, bool bf16, const float* proj,
                                     int R, const float* summ, int B, int Hq, int Hkv, int D, int C,
                                     const uint8_t* head_full, float logit_scale, float p,
                                     int budget, int n_sink, int n_local, int32_t* idx,
                                     int32_t* count, int kmax, int32_t* n_p_out);

// token_sparse.cu
size_t token_importance_scratch_bytes(int B, int S, int Hkv, int G, int n_obs);
cudaError_t launch_token_importance(const Launch& l, const void* Q, const void* K, int B, int S,
                                    int Hq, int Hkv, int D, int n_obs, float scale, float* imp,
                                    float* scratch, std::string* why);
// The coverage budget runs one cluster of 8 CTAs per sequence for these
// sizes (else one CTA per sequence, S <= 32768).
bool token_budget_cluster_fits(int B, int num_sms);
cudaError_t launch_token_budget(const Launch& l, const float* imp, int B, int S, int Hkv,
                                float tau, int tile, int32_t* k_seq, int32_t* k_unit);
cudaError_t launch_tsa_gather(const Launch& l, const void* Q, const void* K, const void* V,
                              const int32_t* idx, const int32_t* count, int kmax, int B, int S,
                              int Sc, int Hq, int Hkv, int D, void* Qc, void* Kc, void* Vc);
// inv [B*Hkv, S] (scratch): built here from idx/count unless inv_ready (the
// selection wrote it)
cudaError_t launch_tsa_scatter(const Launch& l, const void* Oc, const int32_t* idx,
                               const int32_t* count, int kmax, int B, int S, int Sc, int Hq,
                               int Hkv, int D, int32_t* inv, void* O, bool inv_ready = false);

// rope.cu
cudaError_t launch_rope(const Launch& l, const void* x, void* y, bool bf16, int64_t rows, int D,
                        int64_t period, int64_t pos0, float theta);

// decode.cu
int decode_default_parts(bool bf16, int D, int L, int num_sms);
// Merged mode: the last CTA of each unit combines the unit's splits.
struct MergeOut {
  int* counters;   // [B*Hkv], zero on entry, left zero on a normal exit
  void* out;       // [B, Hq, D]
  bool out_bf16;
  float* lse_out;  // [B, Hq] or null
  // bf16 only: full-head units first, then (after the selection kernel that
  // precedes it on the stream completes) the sparse units; the decode is
  // launched with programmatic dependent launch
  bool phased = false;
  // phased: CTAs at the end of the grid that take no full-head work (they
  // start only after the selection's CTAs leave their SMs)
  int late = 0;
  // bf16 hybrid context: gist K/V rows [B, Hkv, C, D] (C = T / L) that every
  // sparse unit attends over next to its selected chunks; null = off.
  // gist_selected: only the gist rows of the unit's selected chunks, else
  // every chunk's gist row
  const void* Kg = nullptr;
  const void* Vg = nullptr;
  bool gist_selected = false;
  // the caller left the number of pieces to the library: steps with few
  // chunks per unit and no full-attention heads may run as one cluster of
  // CTAs per unit (its parts combined in distributed shared memory)
  bool allow_cluster = false;
};
constexpr int kMergedMaxParts = 256;
cudaError_t launch_decode(const Launch& l, const void* q, const void* K, const void* V, bool bf16,
                          const int32_t* idx, const int32_t* count, int kmax,
                          const uint8_t* head_full, int B, int Hq, int Hkv, int D, int64_t T,
                          int L, float scale, int num_parts, int max_splits, float* o_part,
                          float* lse_part, const MergeOut* merge, std::string* why);
cudaError_t launch_merge(const Launch& l, const float* o_part, const float* lse_part, int rows,
                         int max_splits, int D, void* out, bool out_bf16, float* lse_out);

// hostio.cu: bytes / 16 words from src to dst (both 16-byte aligned; src may
// be mapped pinned host memory)
cudaError_t launch_copy16(const Launch& l, const void* src, void* dst, size_t bytes);

// prefill.cu
// skip_empty: units with no chunk write nothing (else their rows get 0).
// dense_k (dense causal mode; idx/count unused): tile t of (b, h) attends
// to chunks 0 .. t when t * 64 < dense_k[b * Hkv + h], else it is empty.
cudaError_t launch_prefill(const Launch& l, const void* Q, const void* K, const void* V,
                           const int32_t* idx, const int32_t* count, int kmax, int B, int S,
                           int Hq, int Hkv, int D, int tile_m, int L, float scale, void* O,
                           std::string* why, bool skip_empty = false,
                           const int32_t* dense_k = nullptr);

// tma_host.cu: 2-D bf16 tensor map over a row-major [rows, cols] matrix with
// `row_stride` elements between rows, box [box_rows, box_cols], 128-byte swizzle.
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                       uint64_t row_stride, uint32_t box_rows, uint32_t box_cols,
                       std::string* why);

}  // namespace csa
