// C-ABI entry points: host-side validation, workspace sizing, tensor-map encoding, the
// IndexCache layer driver and device-status reporting. No device memory is allocated here.
#include <cstdlib>
#include <cstring>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {

namespace {

uint64_t wait_budget_ns() {
  const char* env = std::getenv("DSA_WAIT_BUDGET_NS");
  if (env && *env) {
    char* end = nullptr;
    unsigned long long v = std::strtoull(env, &end, 10);
    if (end && *end == '\0' && v > 0) return static_cast<uint64_t>(v);
  }
  return 2000000000ull;
}

int current_num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return n;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool prefill_shape_supported(int H, int d) { return (H == 64 && d == 128) || (H == 8 && d == 64); }

dsa_status check_prefill(const uint8_t* q, const float* q_scale, const float* w, const uint8_t* k,
                         const float* k_scale, int32_t Lk, int32_t q_pos0, int32_t Lq, int32_t H,
                         int32_t d, int32_t topk, const int32_t* out_idx) {
  if (!q || !q_scale || !w || !k || !k_scale || !out_idx) return DSA_ERR_INVALID;
  if (Lq < 1 || Lk < 1 || q_pos0 < 0 || static_cast<int64_t>(q_pos0) + Lq > Lk) return DSA_ERR_INVALID;
  if (topk < 1 || H < 1 || d < 1) return DSA_ERR_INVALID;
  if (!aligned(q, 16) || !aligned(k, 16)) return DSA_ERR_INVALID;
  if (!prefill_shape_supported(H, d) || topk > DSA_MAX_TOPK) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

dsa_status check_decode(const uint8_t* q, const float* q_scale, const float* w,
                        const uint8_t* k_cache, const float* k_scale_cache, int32_t n_blocks,
                        int32_t block_size, const int32_t* block_table, int32_t max_blocks,
                        const int32_t* seq_lens, int32_t B, int32_t H, int32_t d, int32_t topk,
                        const int32_t* out_idx) {
  if (!q || !q_scale || !w || !k_cache || !k_scale_cache || !block_table || !seq_lens || !out_idx)
    return DSA_ERR_INVALID;
  if (B < 1 || n_blocks < 1 || max_blocks < 1 || block_size < 1 || topk < 1 || H < 1 || d < 1)
    return DSA_ERR_INVALID;
  if (static_cast<int64_t>(max_blocks) * block_size > INT32_MAX) return DSA_ERR_INVALID;
  if (!aligned(q, 16) || !aligned(k_cache, 16)) return DSA_ERR_INVALID;
  if (!(H == 64 && d == 128) || block_size != 64 || topk > DSA_MAX_TOPK) return DSA_ERR_UNSUPPORTED;
  if (B > DSA_DECODE_MAX_REQUESTS) return DSA_ERR_UNSUPPORTED;  // one grid row per request
  return DSA_OK;
}

}  // namespace

bool encode_tmap_2d_u8(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows,
                       uint32_t box_rows, uint64_t row_stride) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qres) != cudaSuccess ||
        qres != cudaDriverEntryPointSuccess || !fn)
      return false;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_stride ? row_stride : row_bytes};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(row_bytes), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle swz =
      row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace dsa

using namespace dsa;

extern "C" {

DSA_API int32_t dsa_abi_version(void) { return DSA_ABI_VERSION; }

DSA_API const char* dsa_status_string(int32_t status) {
  switch (status) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_TIMEOUT: return "device wait timed out";
    case DSA_ERR_DEVICE: return "device-side input check failed";
    default: return "unknown status";
  }
}

DSA_API dsa_status dsa_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace || workspace_bytes < DSA_WS_HEADER_BYTES) return DSA_ERR_INVALID;
  return cuda_status(
      cudaMemsetAsync(workspace, 0, DSA_WS_HEADER_BYTES, static_cast<cudaStream_t>(stream)));
}

DSA_API dsa_status dsa_read_device_status(void* workspace, void* stream, int32_t* status_out,
                                          int32_t* detail_out) {
  if (!workspace) return DSA_ERR_INVALID;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t h[2] = {0, 0};
  if (cudaStreamSynchronize(s) != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaMemcpyAsync(h, workspace, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, sizeof(h), s) != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DSA_ERR_CUDA;
  if (status_out) *status_out = static_cast<int32_t>(h[0]);
  if (detail_out) *detail_out = static_cast<int32_t>(h[1]);
  return DSA_OK;
}

DSA_API size_t dsa_prefill_workspace_bytes(int32_t Lq, int32_t H, int32_t d, int32_t topk) {
  if (Lq < 1 || topk < 1 || topk > DSA_MAX_TOPK || !prefill_shape_supported(H, d)) return 0;
  const int sms = current_num_sms();
  if (sms < 1) return 0;
  return prefill_workspace_bytes(Lq, H, d, topk, sms);
}

DSA_API dsa_status dsa_indexer_prefill(const uint8_t* q, const float* q_scale, const float* w,
                                       const uint8_t* k, const float* k_scale, int32_t Lk,
                                       int32_t q_pos0, int32_t Lq, int32_t H, int32_t d,
                                       int32_t topk, int32_t* out_idx, float* out_score,
                                       void* workspace, size_t workspace_bytes, void* stream) {
  dsa_status st = check_prefill(q, q_scale, w, k, k_scale, Lk, q_pos0, Lq, H, d, topk, out_idx);
  if (st != DSA_OK) return st;
  if (!workspace || !aligned(workspace, 256)) return DSA_ERR_INVALID;
  const int sms = current_num_sms();
  if (sms < 1) return DSA_ERR_CUDA;
  if (workspace_bytes < prefill_workspace_bytes(Lq, H, d, topk, sms)) return DSA_ERR_INVALID;
  PrefillLaunch a{q, q_scale, w, k, k_scale, Lk, q_pos0, Lq, H, d, topk, out_idx, out_score,
                  workspace, workspace_bytes, static_cast<cudaStream_t>(stream), wait_budget_ns(), sms};
  return launch_prefill(a);
}

DSA_API size_t dsa_decode_workspace_bytes(int32_t B, int32_t max_len, int32_t H, int32_t d,
                                          int32_t topk) {
  if (B < 1 || max_len < 1 || topk < 1) return 0;
  return decode_workspace_bytes(B, max_len, H, d, topk);
}

DSA_API dsa_status dsa_indexer_decode(const uint8_t* q, const float* q_scale, const float* w,
                                      const uint8_t* k_cache, const float* k_scale_cache,
                                      int32_t n_blocks, int32_t block_size,
                                      const int32_t* block_table, int32_t max_blocks,
                                      const int32_t* seq_lens, int32_t B, int32_t H, int32_t d,
                                      int32_t topk, int32_t* out_idx, float* out_score,
                                      void* workspace, size_t workspace_bytes, void* stream) {
  dsa_status st = check_decode(q, q_scale, w, k_cache, k_scale_cache, n_blocks, block_size,
                               block_table, max_blocks, seq_lens, B, H, d, topk, out_idx);
  if (st != DSA_OK) return st;
  if (!workspace || !aligned(workspace, 256)) return DSA_ERR_INVALID;
  if (workspace_bytes < decode_workspace_bytes(B, max_blocks * block_size, H, d, topk)) return DSA_ERR_INVALID;
  const int sms = current_num_sms();
  if (sms < 1) return DSA_ERR_CUDA;
  DecodeLaunch a{q, q_scale, w, k_cache, k_scale_cache, n_blocks, block_size, block_table,
                 max_blocks, seq_lens, B, H, d, topk, out_idx, out_score, workspace,
                 workspace_bytes, static_cast<cudaStream_t>(stream), wait_budget_ns(), sms};
  return launch_decode(a);
}

DSA_API size_t dsa_sparse_attention_workspace_bytes(int32_t B, int32_t topk) {
  if (B < 1 || topk < 256 || topk > DSA_MAX_TOPK || topk % 256 != 0) return 0;
  return attention_workspace_bytes(B, topk);
}

DSA_API dsa_status dsa_sparse_attention_decode(const uint16_t* q, const uint16_t* latent,
                                               int32_t n_blocks, int32_t block_size,
                                               const int32_t* block_table, int32_t max_blocks,
                                               const int32_t* seq_lens, const int32_t* idx,
                                               int32_t B, int32_t Hq, int32_t dqk, int32_t dv,
                                               int32_t topk, float scale, float* out,
                                               void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !latent || !block_table || !seq_lens || !idx || !out) return DSA_ERR_INVALID;
  if (B < 1 || n_blocks < 1 || block_size < 1 || max_blocks < 1 || topk < 1) return DSA_ERR_INVALID;
  if (static_cast<int64_t>(max_blocks) * block_size > INT32_MAX ||
      static_cast<int64_t>(n_blocks) * block_size > INT32_MAX)
    return DSA_ERR_INVALID;
  if (!(scale > 0.0f) || !(scale < 1e30f)) return DSA_ERR_INVALID;
  if (!aligned(q, 16) || !aligned(latent, 16) || !aligned(out, 16)) return DSA_ERR_INVALID;
  if (Hq != 128 || dqk != 576 || dv != 512 || topk % 256 != 0 || topk > DSA_MAX_TOPK ||
      B > DSA_DECODE_MAX_REQUESTS)
    return DSA_ERR_UNSUPPORTED;
  if (!workspace || !aligned(workspace, 256)) return DSA_ERR_INVALID;
  if (workspace_bytes < attention_workspace_bytes(B, topk)) return DSA_ERR_INVALID;
  AttentionLaunch a{q, latent, n_blocks, block_size, block_table, max_blocks, seq_lens, idx, B, topk,
                    scale, out, workspace, static_cast<cudaStream_t>(stream), wait_budget_ns()};
  return launch_attention(a);
}

DSA_API size_t dsa_indexcache_workspace_bytes(const dsa_indexer_shape* shape) {
  if (!shape) return 0;
  if (shape->mode == DSA_MODE_PREFILL)
    return dsa_prefill_workspace_bytes(shape->Lq, shape->H, shape->d, shape->topk);
  if (shape->mode == DSA_MODE_DECODE) {
    if (static_cast<int64_t>(shape->max_blocks) * shape->block_size > INT32_MAX) return 0;
    return dsa_decode_workspace_bytes(shape->B, shape->max_blocks * shape->block_size, shape->H,
                                      shape->d, shape->topk);
  }
  return 0;
}

// Validates an IndexCache call (pattern, buffers, every Full layer's inputs, workspace) before
// anything is enqueued; returns the number of Full layers in *n_full.
static dsa_status check_indexcache(const char* pattern, int32_t n_layers,
                                   const dsa_indexer_shape* shape, const dsa_layer_inputs* layers,
                                   int32_t* const* f_bufs, const int32_t** out_layer_idx,
                                   void* workspace, size_t workspace_bytes, int* n_full) {
  if (!pattern || !shape || !layers || !f_bufs || !out_layer_idx || n_layers < 1) return DSA_ERR_INVALID;
  if (static_cast<int64_t>(std::strlen(pattern)) != n_layers) return DSA_ERR_INVALID;
  *n_full = 0;
  for (int l = 0; l < n_layers; ++l) {
    if (pattern[l] == 'F') ++*n_full;
    else if (pattern[l] != 'S') return DSA_ERR_INVALID;
  }
  if (pattern[0] != 'F') return DSA_ERR_INVALID;  // the first layer is always Full
  if (shape->mode != DSA_MODE_PREFILL && shape->mode != DSA_MODE_DECODE) return DSA_ERR_INVALID;
  for (int l = 0; l < n_layers; ++l) {
    if (pattern[l] != 'F') continue;
    const dsa_layer_inputs& in = layers[l];
    dsa_status st;
    if (shape->mode == DSA_MODE_PREFILL)
      st = check_prefill(in.q, in.q_scale, in.w, in.k, in.k_scale, shape->Lk, shape->q_pos0,
                         shape->Lq, shape->H, shape->d, shape->topk, f_bufs[0]);
    else
      st = check_decode(in.q, in.q_scale, in.w, in.k, in.k_scale, shape->n_blocks,
                        shape->block_size, shape->block_table, shape->max_blocks, shape->seq_lens,
                        shape->B, shape->H, shape->d, shape->topk, f_bufs[0]);
    if (st != DSA_OK) return st;
  }
  const size_t need = dsa_indexcache_workspace_bytes(shape);
  if (!workspace || need == 0 || workspace_bytes < need || !aligned(workspace, 256)) return DSA_ERR_INVALID;
  return DSA_OK;
}

// One Full layer's indexer into buf on stream.
static dsa_status run_full_layer(const dsa_indexer_shape* shape, const dsa_layer_inputs& in,
                                 int32_t* buf, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  if (shape->mode == DSA_MODE_PREFILL)
    return dsa_indexer_prefill(in.q, in.q_scale, in.w, in.k, in.k_scale, shape->Lk, shape->q_pos0,
                               shape->Lq, shape->H, shape->d, shape->topk, buf, in.out_score,
                               workspace, workspace_bytes, stream);
  return dsa_indexer_decode(in.q, in.q_scale, in.w, in.k, in.k_scale, shape->n_blocks,
                            shape->block_size, shape->block_table, shape->max_blocks,
                            shape->seq_lens, shape->B, shape->H, shape->d, shape->topk, buf,
                            in.out_score, workspace, workspace_bytes, stream);
}

DSA_API dsa_status indexcache_run(const char* pattern, int32_t n_layers,
                                  const dsa_indexer_shape* shape, const dsa_layer_inputs* layers,
                                  int32_t* const* f_bufs, int32_t n_fbufs,
                                  const int32_t** out_layer_idx, dsa_after_layer_fn after_layer,
                                  void* user, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  int n_full = 0;
  dsa_status st = check_indexcache(pattern, n_layers, shape, layers, f_bufs, out_layer_idx,
                                   workspace, workspace_bytes, &n_full);
  if (st != DSA_OK) return st;
  if (n_fbufs != 1 && n_fbufs != n_full) return DSA_ERR_INVALID;
  for (int m = 0; m < n_fbufs; ++m)
    if (!f_bufs[m]) return DSA_ERR_INVALID;

  int m = 0;
  const int32_t* cached = nullptr;
  for (int l = 0; l < n_layers; ++l) {
    if (pattern[l] == 'F') {
      int32_t* buf = f_bufs[n_fbufs == 1 ? 0 : m];
      ++m;
      if ((st = run_full_layer(shape, layers[l], buf, workspace, workspace_bytes, stream)) != DSA_OK)
        return st;
      cached = buf;
    }
    out_layer_idx[l] = cached;  // an S layer reads T_f(l): the buffer of the last F layer
    if (after_layer) after_layer(l, cached, user);
  }
  return DSA_OK;
}

DSA_API dsa_status indexcache_run_lagged(const char* pattern, int32_t n_layers,
                                         const dsa_indexer_shape* shape,
                                         const dsa_layer_inputs* layers, int32_t* const* f_bufs,
                                         int32_t n_fbufs, const int32_t** out_layer_idx,
                                         dsa_after_layer_fn consume, void* user, void* workspace,
                                         size_t workspace_bytes, void* stream,
                                         void* indexer_stream) {
  int n_full = 0;
  dsa_status st = check_indexcache(pattern, n_layers, shape, layers, f_bufs, out_layer_idx,
                                   workspace, workspace_bytes, &n_full);
  if (st != DSA_OK) return st;
  // A Full layer's consumer reads the previous Full layer's buffer while the layer's own
  // indexer writes: two buffers at least (one suffices for a single Full layer).
  const int min_bufs = n_full >= 2 ? 2 : 1;
  if (n_fbufs < min_bufs || n_fbufs > (n_full > 2 ? n_full : 2)) return DSA_ERR_INVALID;
  for (int m = 0; m < n_fbufs; ++m)
    if (!f_bufs[m]) return DSA_ERR_INVALID;
  if (stream == indexer_stream) return DSA_ERR_INVALID;  // the point is two streams
  cudaStream_t main_s = static_cast<cudaStream_t>(stream);
  cudaStream_t idx_s = static_cast<cudaStream_t>(indexer_stream);

  // One completion event per Full layer (the indexer's work on indexer_stream) and one event
  // marking where each Full layer's inputs are ready on the consumer stream.
  const int n_events = n_full + 1;
  cudaEvent_t* ev = new cudaEvent_t[n_events];
  int made = 0;
  for (; made < n_events; ++made)
    if (cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming) != cudaSuccess) break;
  auto cleanup = [&](dsa_status s) {
    for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]);  // released once they complete
    delete[] ev;
    return s;
  };
  if (made < n_events) return cleanup(DSA_ERR_CUDA);
  cudaEvent_t ready = ev[n_full];

  int m = -1;  // index of the last Full layer so far
  for (int l = 0; l < n_layers; ++l) {
    int src;
    if (pattern[l] == 'F') {
      ++m;
      // Everything enqueued on the consumer stream so far (the layer's inputs; every consumer
      // that may still read the buffer about to be rewritten) precedes this indexer.
      if (cudaEventRecord(ready, main_s) != cudaSuccess || cudaStreamWaitEvent(idx_s, ready, 0) != cudaSuccess)
        return cleanup(DSA_ERR_CUDA);
      if ((st = run_full_layer(shape, layers[l], f_bufs[m % n_fbufs], workspace, workspace_bytes,
                               idx_s)) != DSA_OK)
        return cleanup(st);
      if (cudaEventRecord(ev[m], idx_s) != cudaSuccess) return cleanup(DSA_ERR_CUDA);
      src = (m == 0) ? 0 : m - 1;  // the previous indexer layer; layer 0 has only its own
    } else {
      src = m;  // the source Full layer, whose indexer ran during that layer's consumer
    }
    if (cudaStreamWaitEvent(main_s, ev[src], 0) != cudaSuccess) return cleanup(DSA_ERR_CUDA);
    out_layer_idx[l] = f_bufs[src % n_fbufs];
    if (consume) consume(l, out_layer_idx[l], user);
  }
  if (cudaStreamWaitEvent(main_s, ev[m], 0) != cudaSuccess) return cleanup(DSA_ERR_CUDA);
  return cleanup(DSA_OK);
}

DSA_API dsa_status topk_overlap(const int32_t* const* layer_idx, int32_t n_layers, int32_t rows,
                                int32_t topk, int32_t n_keys, uint64_t* out_counts,
                                uint64_t* out_valid, double* out_overlap, void* workspace,
                                size_t workspace_bytes, void* stream) {
  if (!layer_idx || !out_counts || !out_valid || !workspace) return DSA_ERR_INVALID;
  if (n_layers < 1 || n_layers > DSA_MAX_LAYERS || rows < 0 || topk < 1 || n_keys < 1)
    return DSA_ERR_INVALID;
  if (n_keys > 1500000) return DSA_ERR_UNSUPPORTED;
  if (workspace_bytes < DSA_WS_HEADER_BYTES || !aligned(workspace, 256)) return DSA_ERR_INVALID;
  for (int i = 0; i < n_layers; ++i)
    if (!layer_idx[i] && rows > 0) return DSA_ERR_INVALID;  // zero rows read no layer
  const int sms = current_num_sms();
  if (sms < 1) return DSA_ERR_CUDA;
  return launch_overlap(layer_idx, n_layers, rows, topk, n_keys, out_counts, out_valid, out_overlap,
                        workspace, static_cast<cudaStream_t>(stream), sms);
}

DSA_API dsa_status dsa_topk_merge(const float* scores, const int32_t* idx, const int32_t* idx_offset,
                                  int32_t n_lists, int32_t rows, int32_t topk, int32_t* out_idx,
                                  float* out_score, void* stream) {
  if (!scores || !idx || !out_idx) return DSA_ERR_INVALID;
  if (n_lists < 1 || n_lists > DSA_MAX_LAYERS || rows < 1 || topk < 1) return DSA_ERR_INVALID;
  if (topk > DSA_MAX_TOPK) return DSA_ERR_UNSUPPORTED;
  return launch_topk_merge(scores, idx, idx_offset, n_lists, rows, topk, out_idx, out_score,
                           static_cast<cudaStream_t>(stream));
}

DSA_API dsa_status dsa_selftest_wait_timeout(void* workspace, size_t workspace_bytes,
                                             uint64_t budget_ns, void* stream) {
  if (!workspace || workspace_bytes < DSA_WS_HEADER_BYTES || !aligned(workspace, 256) ||
      budget_ns == 0 || budget_ns > 10000000000ull)
    return DSA_ERR_INVALID;
  return launch_selftest_wait(workspace, budget_ns, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
