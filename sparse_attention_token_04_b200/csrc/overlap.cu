// Cross-layer top-k overlap: C[i][j] = sum over rows of |T_i(row) ∩ T_j(row)|.
//
// Integer work bound by reading the N index tensors (N * rows * topk * 4 bytes, each byte once)
// and by the shared-memory marks: every listed index sets one bit with a shared atomic, about
// 3.5 bank wavefronts per warp instruction for random indices. Small CTAs (four warps, up to
// eight per SM) walk rows independently, so while some mark, others load or count. For a row a
// CTA marks every layer's indices in per-layer shared-memory bitmaps over the row's index range,
// one layer's loads in flight at a time, counts each pair (i <= j) as the popcount of the AND of
// the two bitmaps and clears the bitmaps. When the N bitmaps over [0, n_keys) do not fit in
// shared memory, one bitmap at a time is built and the other layers' entries are probed against
// it. Counts accumulate in shared 64-bit counters per CTA and are added to the output once per
// CTA; a finishing kernel mirrors the upper triangle and forms C / V.
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

constexpr int kOverlapThreads = 128;
constexpr int kOverlapMinBlocks = 8;  // CTAs per SM the register budget is sized for
constexpr size_t kOverlapSmemBudget = 200 * 1024;

__device__ __forceinline__ unsigned long long* overlap_acc(uint8_t* smem) {
  return reinterpret_cast<unsigned long long*>(smem);
}

// All N bitmaps resident: bits[i][w], W words per layer. With N <= kOvGroup (SMALL) each
// thread keeps its pair counts in registers across rows, two 16-bit counts per register, and
// reduces them into the shared counters before a count can wrap (a row adds at most 32 per
// word a thread counts) and at the end; otherwise each row's pair counts are reduced per warp
// into the shared counters. VEC: rows start 16-byte aligned, indices are loaded as int4.
constexpr int kOvGroup = 8;
constexpr int kOvPerThread = DSA_MAX_TOPK / kOverlapThreads;  // indices per thread per layer
constexpr int kOvPairs = kOvGroup * (kOvGroup + 1) / 2;
static_assert(DSA_MAX_TOPK % (4 * kOverlapThreads) == 0, "indices per thread");

template <bool SMALL, bool VEC>
__global__ void __launch_bounds__(kOverlapThreads, kOverlapMinBlocks)
    overlap_bitmaps_kernel(const __grid_constant__ OverlapParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int N = p.N;
  // Pair counters (SMALL: the kOvGroup x kOvGroup triangle, whatever N), then one spare word.
  const int npairs = SMALL ? kOvPairs : N * (N + 1) / 2;
  unsigned long long* acc = overlap_acc(smem_raw);                        // [npairs + 1]
  int* row_max = reinterpret_cast<int*>(acc + npairs + 1);                 // [1] (+pad)
  uint32_t* bits = reinterpret_cast<uint32_t*>(row_max + 4);               // [N][W]
  const int W = (p.n_keys + 31) / 32;
  for (int e = threadIdx.x; e < npairs + 1; e += kOverlapThreads) acc[e] = 0ull;
  for (int e = threadIdx.x; e < N * W; e += kOverlapThreads) bits[e] = 0u;
  if (threadIdx.x == 0) *row_max = -1;
  __syncthreads();
  const uint32_t lane = threadIdx.x & 31u;
  // Pair q's count in half q & 1 of creg[q / 2].
  uint32_t creg[(kOvPairs + 1) / 2];
#pragma unroll
  for (int q = 0; q < (kOvPairs + 1) / 2; ++q) creg[q] = 0u;
  const int words_pt = (W + kOverlapThreads - 1) / kOverlapThreads;
  const int flush_rows = 65535 / (32 * words_pt);  // >= 1: W <= 51200 words in the budget
  // Adds the register pair counts into the shared counters (all threads of the CTA).
  auto flush_creg = [&]() {
#pragma unroll
    for (int q = 0; q < kOvPairs; ++q) {
      const uint32_t c = __reduce_add_sync(0xFFFFFFFFu, (creg[q >> 1] >> (16 * (q & 1))) & 0xFFFFu);
      if (lane == 0 && c) atomicAdd(&acc[q], static_cast<unsigned long long>(c));
    }
#pragma unroll
    for (int q = 0; q < (kOvPairs + 1) / 2; ++q) creg[q] = 0u;
  };
  int it = 0;
  for (int row = blockIdx.x; row < p.rows; row += gridDim.x) {
    const size_t off = static_cast<size_t>(row) * p.topk;
    int local_max = -1;
    for (int i = 0; i < N; ++i) {
      int32_t v[kOvPerThread];
      if constexpr (VEC) {
        const int4* src = reinterpret_cast<const int4*>(p.layers[i] + off);
#pragma unroll
        for (int q4 = 0; q4 < kOvPerThread / 4; ++q4) {
          const int e4 = static_cast<int>(threadIdx.x) + q4 * kOverlapThreads;
          const int4 t = 4 * e4 < p.topk ? __ldcs(src + e4) : make_int4(-1, -1, -1, -1);
          v[4 * q4 + 0] = t.x;
          v[4 * q4 + 1] = t.y;
          v[4 * q4 + 2] = t.z;
          v[4 * q4 + 3] = t.w;
        }
      } else {
#pragma unroll
        for (int q = 0; q < kOvPerThread; ++q) {
          const int e = static_cast<int>(threadIdx.x) + q * kOverlapThreads;
          v[q] = e < p.topk ? __ldcs(p.layers[i] + off + e) : -1;
        }
      }
      uint32_t* bi = bits + i * W;
#pragma unroll
      for (int q = 0; q < kOvPerThread; ++q) {
        const int32_t x = v[q];
        if (x >= 0 && x < p.n_keys) {
          atomicOr(&bi[x >> 5], __funnelshift_l(0u, 1u, static_cast<uint32_t>(x)));  // 1 << (x mod 32)
          local_max = x > local_max ? x : local_max;
        } else if (x != -1) {
          record_error(p.hdr, DSA_ERR_DEVICE, DETAIL_BAD_INDEX);
        }
      }
    }
    local_max = __reduce_max_sync(0xFFFFFFFFu, local_max);  // one shared atomic per warp
    if (lane == 0 && local_max >= 0) atomicMax(row_max, local_max);
    __syncthreads();
    const int wr = (*row_max >> 5) + 1;  // words that can hold a mark in this row
    if constexpr (SMALL) {
      for (int w = threadIdx.x; w < wr; w += kOverlapThreads) {
        uint32_t m[kOvGroup];
#pragma unroll
        for (int i = 0; i < kOvGroup; ++i) m[i] = i < N ? bits[i * W + w] : 0u;
        int q = 0;
#pragma unroll
        for (int i = 0; i < kOvGroup; ++i)
#pragma unroll
          for (int j = i; j < kOvGroup; ++j, ++q)
            creg[q >> 1] += static_cast<uint32_t>(__popc(m[i] & m[j])) << (16 * (q & 1));
      }
    } else {
      int pair = 0;
      for (int i = 0; i < N; ++i) {
        const uint32_t* bi = bits + i * W;
        for (int j = i; j < N; ++j, ++pair) {
          const uint32_t* bj = bits + j * W;
          uint32_t c = 0;
          for (int w = threadIdx.x; w < wr; w += kOverlapThreads) c += __popc(bi[w] & bj[w]);
          c = __reduce_add_sync(0xFFFFFFFFu, c);
          if (lane == 0 && c) atomicAdd(&acc[pair], static_cast<unsigned long long>(c));
        }
      }
    }
    __syncthreads();
    for (int i = 0; i < N; ++i)
      for (int w = threadIdx.x; w < wr; w += kOverlapThreads) bits[i * W + w] = 0u;
    if (threadIdx.x == 0) *row_max = -1;
    if constexpr (SMALL) {
      if (++it == flush_rows) {
        flush_creg();
        it = 0;
      }
    }
    __syncthreads();
  }
  if constexpr (SMALL) {
    // Register pair q (i <= j over kOvGroup layers) is shared pair (i, j) over N layers.
    flush_creg();
    __syncthreads();
    if (threadIdx.x == 0) {
      int q = 0;
      for (int i = 0; i < kOvGroup; ++i)
        for (int j = i; j < kOvGroup; ++j, ++q)
          if (j < N && acc[q]) atomicAdd(&p.counts[i * N + j], acc[q]);
      // V: a row lists a key once, so layer 0's in-range entries are its pair count C[0][0].
      if (acc[0]) atomicAdd(p.valid, acc[0]);
    }
  } else {
    __syncthreads();
    int pair = 0;
    for (int i = 0; i < N; ++i)
      for (int j = i; j < N; ++j, ++pair)
        if (threadIdx.x == 0 && acc[pair]) atomicAdd(&p.counts[i * N + j], acc[pair]);
    if (threadIdx.x == 0 && acc[0]) atomicAdd(p.valid, acc[0]);  // V = C[0][0]
  }
}

// One bitmap at a time (wide index ranges or many layers).
__global__ void __launch_bounds__(kOverlapThreads)
    overlap_probe_kernel(const __grid_constant__ OverlapParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int N = p.N;
  unsigned long long* acc = overlap_acc(smem_raw);                        // [N*N + 1]
  uint32_t* bits = reinterpret_cast<uint32_t*>(acc + (N * N + 1));        // [W]
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
        if (v >= 0 && v < p.n_keys) atomicOr(&bits[v >> 5], 1u << (v & 31));
        else if (v != -1) record_error(p.hdr, DSA_ERR_DEVICE, DETAIL_BAD_INDEX);
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

template <class Kern>
static dsa_status launch_overlap_kernel(Kern kern, const OverlapParams& p, size_t smem, int rows,
                                        cudaStream_t stream, int num_sms) {
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return DSA_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kOverlapThreads, smem) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (per_sm < 1) return DSA_ERR_UNSUPPORTED;
  const int grid = rows < per_sm * num_sms ? rows : per_sm * num_sms;
  kern<<<grid, kOverlapThreads, smem, stream>>>(p);
  return cuda_status(cudaGetLastError());
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
    const size_t words = static_cast<size_t>((n_keys + 31) / 32);
    const size_t npairs = n_layers <= kOvGroup ? static_cast<size_t>(kOvPairs)
                                               : static_cast<size_t>(n_layers) * (n_layers + 1) / 2;
    const size_t smem_all = (npairs + 1) * 8 + 16 + static_cast<size_t>(n_layers) * words * 4;
    dsa_status st;
    bool vec = topk % 4 == 0;
    for (int i = 0; i < n_layers; ++i) vec = vec && (reinterpret_cast<uintptr_t>(layer_idx[i]) & 15u) == 0;
    const bool small = n_layers <= kOvGroup;
    if (smem_all <= kOverlapSmemBudget)
      st = small ? (vec ? launch_overlap_kernel(overlap_bitmaps_kernel<true, true>, p, smem_all, rows, stream, num_sms)
                        : launch_overlap_kernel(overlap_bitmaps_kernel<true, false>, p, smem_all, rows, stream, num_sms))
                 : (vec ? launch_overlap_kernel(overlap_bitmaps_kernel<false, true>, p, smem_all, rows, stream, num_sms)
                        : launch_overlap_kernel(overlap_bitmaps_kernel<false, false>, p, smem_all, rows, stream, num_sms));
    else
      st = launch_overlap_kernel(overlap_probe_kernel, p, (nn + 1) * 8 + words * 4, rows, stream,
                                 num_sms);
    if (st != DSA_OK) return st;
  }
  overlap_finish_kernel<<<1, 256, 0, stream>>>(p.counts, p.valid, out_overlap, n_layers);
  return cuda_status(cudaGetLastError());
}

}  // namespace dsa
