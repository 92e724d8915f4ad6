// Decode indexer entry point that allocates nothing.
//
// Some callers cannot hand the library a workspace: for example a plugin running inside a host
// application whose allocator owns all of the device memory, or a latency-critical decode loop
// that must not call cudaMalloc / cudaFree at step time (cudaFree synchronises the whole
// device). For them, dsa_indexer_decode_noalloc runs the same decode kernels with their scratch
// (the status header, one fp32 score per cached key and per-request selection state) placed
// in a fixed array that lives in this file, instead of in a caller-provided workspace.
//
// The array is a file-scope __device__ variable, so every GPU that loads this library holds it
// until the process exits. Its name is only a host-side stand-in for the device variable: host
// code must never pass it to a kernel. Instead, the first call on each device (with that device
// current) asks the runtime for the variable's device address with cudaGetSymbolAddress and
// caches it; every later call on that device reuses the cached address.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

// The decode workspace of the largest call it takes: status header, one fp32 score slot per
// cached key, and per request a 2048-bin score histogram, 16 bytes of collection state and
// 8192 candidate keys.
constexpr size_t kScratchBytes =
    decode_layout(DSA_NOALLOC_MAX_REQUESTS, static_cast<size_t>(DSA_NOALLOC_MAX_SCORES)).total;

// Zero at load time. Every call clears the status header on its stream before its kernels, so a
// call reports only its own device-side errors, even after an earlier call that failed part-way
// (the decode launch itself clears the histograms it uses).
static __device__ __align__(256) uint8_t g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (set up once per device).
dsa_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
      return DSA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return DSA_OK;
}

}  // namespace
}  // namespace dsa

extern "C" DSA_API dsa_status dsa_indexer_decode_noalloc(
    const uint8_t* q, const float* q_scale, const float* w, const uint8_t* k_cache,
    const float* k_scale_cache, int32_t n_blocks, int32_t block_size, const int32_t* block_table,
    int32_t max_blocks, const int32_t* seq_lens, int32_t B, int32_t H, int32_t d, int32_t topk,
    int32_t* out_idx, float* out_score, int32_t* device_status_out, void* stream) {
  using namespace dsa;
  if (B >= 1 && max_blocks >= 1 && block_size >= 1 &&
      (B > DSA_NOALLOC_MAX_REQUESTS ||
       static_cast<int64_t>(B) * max_blocks * block_size > static_cast<int64_t>(DSA_NOALLOC_MAX_SCORES) ||
       dsa_decode_workspace_bytes(B, max_blocks * block_size, H, d, topk) > kScratchBytes))
    return DSA_ERR_UNSUPPORTED;  // more requests or cached-key slots than the fixed scratch holds
  void* scratch = nullptr;
  dsa_status st = scratch_address(&scratch);
  if (st != DSA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, DSA_WS_HEADER_BYTES, s) != cudaSuccess) return DSA_ERR_CUDA;
  st = dsa_indexer_decode(q, q_scale, w, k_cache, k_scale_cache, n_blocks, block_size, block_table,
                          max_blocks, seq_lens, B, H, d, topk, out_idx, out_score, scratch,
                          kScratchBytes, stream);
  if (st != DSA_OK) return st;
  if (device_status_out)
    return cuda_status(cudaMemcpyAsync(device_status_out, scratch, 2 * sizeof(int32_t),
                                       cudaMemcpyDeviceToDevice, s));
  return DSA_OK;
}
