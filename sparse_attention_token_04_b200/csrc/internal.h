// Internal launch interface between the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/dsa_indexer.h"

namespace dsa {

struct PrefillLaunch {
  const uint8_t* q;
  const float* q_scale;
  const float* w;
  const uint8_t* k;
  const float* k_scale;
  int32_t Lk, q_pos0, Lq, H, d, topk;
  int32_t* out_idx;
  float* out_score;
  void* ws;
  size_t ws_bytes;
  cudaStream_t stream;
  uint64_t budget_ns;
  int num_sms;
};

struct DecodeLaunch {
  const uint8_t* q;
  const float* q_scale;
  const float* w;
  const uint8_t* k_cache;
  const float* k_scale_cache;
  int32_t n_blocks, block_size;
  const int32_t* block_table;
  int32_t max_blocks;
  const int32_t* seq_lens;
  int32_t B, H, d, topk;
  int32_t* out_idx;
  float* out_score;
  void* ws;
  size_t ws_bytes;
  cudaStream_t stream;
  uint64_t budget_ns;
  int num_sms;
};

struct AttentionLaunch {
  const uint16_t* q;
  const uint16_t* latent;
  int32_t n_blocks, block_size;
  const int32_t* block_table;
  int32_t max_blocks;
  const int32_t* seq_lens;
  const int32_t* idx;
  int32_t B, topk;
  float scale;
  float* out;
  void* ws;
  cudaStream_t stream;
  uint64_t budget_ns;
};

// Prefill workspace layout. Every query row owns 4 * seg_stride candidate entries: four warp
// segments, seg_stride entries apart. The lean pass may fill a segment up to lean_segcap
// (about 3k/4 + 128: it expects k + 6.5 sqrt(k S) keys per row), the exact pass up to
// exact_segcap (k/2 + 128: its cut-backs leave at most (k + 131) / 4 per segment), and the
// sample pass up to seg_stride.
struct PrefillLayout {
  uint32_t seg_stride, lean_segcap, exact_segcap;
  size_t cand_off, thr_off, counts_off, flags_off, list_off, count_off, total;
};
__host__ __device__ constexpr uint32_t prefill_exact_cap(int topk) {
  return (2u * static_cast<uint32_t>(topk) + 512u + 127u) & ~127u;
}
constexpr uint32_t kPrefillExactCapMax = prefill_exact_cap(DSA_MAX_TOPK);
inline PrefillLayout prefill_layout(int Lq, int topk) {
  PrefillLayout L{};
  const uint32_t lean_cap = (3u * static_cast<uint32_t>(topk) + 512u + 127u) & ~127u;
  const uint32_t pitch = lean_cap > prefill_exact_cap(topk) ? lean_cap : prefill_exact_cap(topk);
  L.seg_stride = pitch / 4u;
  L.lean_segcap = lean_cap / 4u;
  L.exact_segcap = prefill_exact_cap(topk) / 4u;
  const size_t rows = static_cast<size_t>(Lq);
  const size_t nqb = rows;  // at least one flag / list slot per row covers every block size
  size_t off = DSA_WS_HEADER_BYTES;
  L.cand_off = off;
  off += rows * pitch * sizeof(uint64_t);
  L.thr_off = off;
  off += rows * sizeof(uint64_t);
  L.counts_off = off;
  off += rows * 4 * sizeof(uint32_t);
  L.flags_off = off;
  off += nqb * sizeof(uint32_t);
  L.list_off = off;
  off += nqb * sizeof(int32_t);
  L.count_off = off;
  off += 16;
  L.total = off;
  return L;
}
inline int prefill_queries_per_block(int H) { return 2 * (256 / H); }

size_t prefill_workspace_bytes(int Lq, int H, int d, int topk, int num_sms);
size_t decode_workspace_bytes(int B, int max_len, int H, int d, int topk);

// Decode workspace after the header: the scores [B][max_len] fp32 the scoring kernel writes,
// the per-request score histograms [B][kDecodeScoreBins] u32, the per-request collection state
// [B][4] u32 (candidate count, largest ordered score, complement of the smallest, candidate
// count the histogram predicts) and the per-request candidate keys [B][kDecodeCandCap] u64.
// Histograms and state are adjacent so that one small kernel (decode_clear_kernel) clears both.
constexpr int kDecodeScoreBins = 2048;
constexpr uint32_t kDecodeCandCap = 8192;
struct DecodeLayout {
  size_t scores, bins, state, cand, total;
};
constexpr size_t align_256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
// n_scores = B * max_len.
constexpr DecodeLayout decode_layout(size_t B, size_t n_scores) {
  DecodeLayout L{};
  L.scores = DSA_WS_HEADER_BYTES;
  L.bins = align_256(L.scores + n_scores * sizeof(float));
  L.state = L.bins + B * kDecodeScoreBins * sizeof(uint32_t);
  L.cand = align_256(L.state + B * 4 * sizeof(uint32_t));
  L.total = L.cand + B * kDecodeCandCap * sizeof(uint64_t);
  return L;
}

dsa_status launch_prefill(const PrefillLaunch& a);
// Exact top-k of every row's candidate buffer, ordered and written to out_idx / out_score.
dsa_status launch_prefill_finish(const uint64_t* cand, const uint32_t* counts,
                                 const uint64_t* thr, uint32_t pitch, int rows, int topk,
                                 int32_t* out_idx, float* out_score, int num_sms,
                                 cudaStream_t stream);
// Per prefill row, the threshold of the lean pass from the row's sampled keys.
dsa_status launch_prefill_sample_threshold(const uint64_t* cand, const uint32_t* counts,
                                           uint64_t* thr, uint32_t seg_stride, int rows,
                                           int q_pos0, int Lk, int topk, uint32_t max_samples,
                                           cudaStream_t stream);
dsa_status launch_decode(const DecodeLaunch& a);
// Exact top-k of every decode request's stored scores: a collection pass (several CTAs per
// request) gathers the keys at or above the request's boundary histogram bin into its
// candidate list, a rank pass (one CTA per request) orders them and writes the outputs.
dsa_status launch_decode_topk(void* ws, const DecodeLayout& lay, int max_len,
                              const int32_t* seq_lens, int B, int topk, int32_t* out_idx,
                              float* out_score, uint64_t budget_ns, cudaStream_t stream);
// Sparse attention of decode queries over their selected latents (attention.cu).
size_t attention_workspace_bytes(int B, int topk);
dsa_status launch_attention(const AttentionLaunch& a);
dsa_status launch_overlap(const int32_t* const* layer_idx, int32_t n_layers, int32_t rows,
                          int32_t topk, int32_t n_keys, uint64_t* out_counts, uint64_t* out_valid,
                          double* out_overlap, void* ws, cudaStream_t stream, int num_sms);
dsa_status launch_selftest_wait(void* ws, uint64_t budget_ns, cudaStream_t stream);
// Top-k of the union of n_lists sorted top-k lists per row (dsa_topk_merge).
dsa_status launch_topk_merge(const float* scores, const int32_t* idx, const int32_t* offsets,
                             int n_lists, int rows, int topk, int32_t* out_idx, float* out_score,
                             cudaStream_t stream);

// Tensor-map encoding through the driver entry point (no link-time libcuda dependency).
// Rows of row_bytes bytes, row_stride bytes apart (0: packed), boxes of box_rows rows.
bool encode_tmap_2d_u8(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows,
                       uint32_t box_rows, uint64_t row_stride = 0);

inline dsa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

}  // namespace dsa
