// Cross-layer top-k overlap: C[i][j] = sum over rows of |T_i(row) ∩ T_j(row)|.
//
// Integer work bound by reading the N index tensors (N * rows * topk * 4 bytes). Each CTA
// walks rows; for a row and each layer i it marks T_i(row) in a shared-memory bitmap over
// [0, n_keys), probes the entries of T_j(row), j >= i, against it, and clears the marked
// words again. Counts accumulate in shared 64-bit counters per CTA and are added to the
// output once per CTA. A finishing kernel mirrors the upper triangle and forms C / V.
#include "common.cuh"
#include "internal.h"

namespace dsa {

struct OverlapParams {
  const int32_t* layers[DSA_MAX_LAYERS];
  int32_t N, rows, topk, n_keys;
  unsigned long long* counts;
  unsigned long long* valid;
  WsHeader* hdr;
};

constexpr int kOverlapThreads = 256;

__global__ void __launch_bounds__(kOverlapThreads)
    overlap_kernel(const __grid_constant__ OverlapParams p) {
  extern __shared__ uint8_t smem_raw[];
  const int N = p.N;
  unsigned long long* acc = reinterpret_cast<unsigned long long*>(smem_raw);     // [N*N + 1]
  uint32_t* bits = reinterpret_cast<uint32_t*>(acc + (N * N + 1));               // [W]
  const int W = (p.n_keys + 31) / 32;
  for (int e = threadIdx.x; e < N * N + 1; e += kOverlapThreads) acc[e] = 0ull;
  for (int e = threadIdx.x; e < W; e += kOverlapThreads) bits[e] = 0u;
  __syncthreads();
  const uint32_t lane = threadIdx.x & 31u;
  for (int row = blockIdx.x; row < p.rows; row += gridDim.x) {
    const size_t off = static_cast<size_t>(row) * p.topk;
    for (int i = 0; i < N; ++i) {
      const int32_t* Ti = p.layers[i] + off;
      for (int e = threadIdx.x; e < p.topk; e += kOverlapThreads) {
        const int32_t v = __ldg(&Ti[e]);
        if (v >= 0 && v < p.n_keys) {
          atomicOr(&bits[v >> 5], 1u << (v & 31));
        } else if (v != -1) {
          record_error(p.hdr, DSA_ERR_DEVICE, DETAIL_BAD_INDEX);
        }
      }
      __syncthreads();
      for (int j = i; j < N; ++j) {
        const int32_t* Tj = p.layers[j] + off;
        uint32_t c = 0;
        for (int e = threadIdx.x; e < p.topk; e += kOverlapThreads) {
          const int32_t v = __ldg(&Tj[e]);
          if (v >= 0 && v < p.n_keys) c += (bits[v >> 5] >> (v & 31)) & 1u;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
        if (lane == 0 && c) atomicAdd(&acc[i * N + j], static_cast<unsigned long long>(c));
      }
      __syncthreads();
      for (int e = threadIdx.x; e < p.topk; e += kOverlapThreads) {
        const int32_t v = __ldg(&Ti[e]);
        if (v >= 0 && v < p.n_keys) bits[v >> 5] = 0u;
      }
      __syncthreads();
    }
    uint32_t c = 0;
    for (int e = threadIdx.x; e < p.topk; e += kOverlapThreads) c += (__ldg(&p.layers[0][off + e]) >= 0) ? 1u : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
    if (lane == 0 && c) atomicAdd(&acc[N * N], static_cast<unsigned long long>(c));
  }
  __syncthreads();
  for (int e = threadIdx.x; e < N * N; e += kOverlapThreads)
    if (acc[e]) atomicAdd(&p.counts[e], acc[e]);
  if (threadIdx.x == 0 && acc[N * N]) atomicAdd(p.valid, acc[N * N]);
}

__global__ void overlap_finish_kernel(unsigned long long* counts, const unsigned long long* valid,
                                      double* overlap, int N) {
  for (int e = threadIdx.x; e < N * N; e += blockDim.x) {
    const int i = e / N, j = e % N;
    if (j < i) counts[e] = counts[j * N + i];
  }
  __syncthreads();
  if (overlap) {
    const unsigned long long v = *valid;
    for (int e = threadIdx.x; e < N * N; e += blockDim.x)
      overlap[e] = v ? static_cast<double>(counts[e]) / static_cast<double>(v) : 0.0;
  }
}

dsa_status launch_overlap(const int32_t* const* layer_idx, int32_t n_layers, int32_t rows,
                          int32_t topk, int32_t n_keys, uint64_t* out_counts, uint64_t* out_valid,
                          double* out_overlap, void* ws, cudaStream_t stream, int num_sms) {
  OverlapParams p;
  for (int i = 0; i < DSA_MAX_LAYERS; ++i) p.layers[i] = i < n_layers ? layer_idx[i] : nullptr;
  p.N = n_layers;
  p.rows = rows;
  p.topk = topk;
  p.n_keys = n_keys;
  p.counts = reinterpret_cast<unsigned long long*>(out_counts);
  p.valid = reinterpret_cast<unsigned long long*>(out_valid);
  p.hdr = static_cast<WsHeader*>(ws);
  const size_t nn = static_cast<size_t>(n_layers) * n_layers;
  if (cudaMemsetAsync(out_counts, 0, nn * sizeof(uint64_t), stream) != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaMemsetAsync(out_valid, 0, sizeof(uint64_t), stream) != cudaSuccess) return DSA_ERR_CUDA;
  if (rows > 0) {
    const size_t smem = (nn + 1) * sizeof(unsigned long long) + static_cast<size_t>((n_keys + 31) / 32) * 4;
    if (cudaFuncSetAttribute(overlap_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return DSA_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, overlap_kernel, kOverlapThreads, smem) !=
        cudaSuccess)
      return DSA_ERR_CUDA;
    if (per_sm < 1) return DSA_ERR_UNSUPPORTED;
    const int grid = rows < per_sm * num_sms ? rows : per_sm * num_sms;
    overlap_kernel<<<grid, kOverlapThreads, smem, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  }
  overlap_finish_kernel<<<1, 256, 0, stream>>>(p.counts, p.valid, out_overlap, n_layers);
  return cuda_status(cudaGetLastError());
}

}  // namespace dsa
