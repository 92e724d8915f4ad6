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

// Candidate-buffer capacity (entries) per query of the streaming prefill top-k: four warp
// segments of cap/4 entries. A segment is cut back as soon as it holds more than cap/4 - 32
// keys (a tile adds at most 32), and a cut-back leaves at most (k + 131) / 4 keys in it.
__host__ __device__ constexpr uint32_t prefill_cand_cap(int topk) {
  return (2u * static_cast<uint32_t>(topk) + 512u + 127u) & ~127u;
}
constexpr uint32_t kPrefillCapMax = prefill_cand_cap(DSA_MAX_TOPK);
inline int prefill_queries_per_block(int H) { return 2 * (256 / H); }

size_t prefill_workspace_bytes(int Lq, int H, int d, int topk, int num_sms);
size_t decode_workspace_bytes(int B, int max_len, int H, int d, int topk);

dsa_status launch_prefill(const PrefillLaunch& a);
// Exact top-k of every row's candidate buffer, ordered and written to out_idx / out_score.
dsa_status launch_prefill_finish(const uint64_t* cand, const uint32_t* counts, uint32_t cap,
                                 int rows, int topk, int32_t* out_idx, float* out_score,
                                 cudaStream_t stream);
dsa_status launch_decode(const DecodeLaunch& a);
dsa_status launch_decode_topk(const float* scores, int max_len, const int32_t* seq_lens,
                              const uint32_t* bins, int B, int topk, int32_t* out_idx,
                              float* out_score, void* ws, cudaStream_t stream);
dsa_status launch_overlap(const int32_t* const* layer_idx, int32_t n_layers, int32_t rows,
                          int32_t topk, int32_t n_keys, uint64_t* out_counts, uint64_t* out_valid,
                          double* out_overlap, void* ws, cudaStream_t stream, int num_sms);
dsa_status launch_selftest_wait(void* ws, uint64_t budget_ns, cudaStream_t stream);

// Tensor-map encoding through the driver entry point (no link-time libcuda dependency).
bool encode_tmap_2d_u8(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows,
                       uint32_t box_rows);

inline dsa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

}  // namespace dsa
