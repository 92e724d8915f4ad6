// Exact merge of top-k lists computed over disjoint key ranges of the same rows.
//
// When one long decode request's keys are split across GPUs, each GPU selects the top-k of its
// own range; the global top-k is contained in the union of those lists, so the top-k of the
// union is the exact result. dsa_topk_merge takes that union per row.
//
// One CTA per row. Every entry becomes the 64-bit selection key (order-preserving score bits,
// complement of the index): larger key = higher score, then lower index, and an empty slot is
// key 0. The lists are merged one after another into a running top-k in shared memory. One
// merge step places every element by its rank: an element of the running list A at position i
// lands at i + |{b in B : b > a}|, an element of the incoming list B at position j at
// j + |{a in A : a >= b}|, each count found by a binary search over the other sorted list;
// positions below k are kept. Positions are distinct, so the step needs no atomics.
#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int kMergeThreads = 512;

// Number of elements of the descending list v[0..n) that are > x (strict) or >= x.
template <bool STRICT>
__device__ __forceinline__ uint32_t count_above(const uint64_t* v, uint32_t n, uint64_t x) {
  uint32_t lo = 0, hi = n;  // v[0..lo) qualify, v[hi..n) do not
  while (lo < hi) {
    const uint32_t mid = (lo + hi) >> 1;
    const bool above = STRICT ? (v[mid] > x) : (v[mid] >= x);
    if (above) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

__global__ void __launch_bounds__(kMergeThreads)
    topk_merge_kernel(const float* __restrict__ scores, const int32_t* __restrict__ idx,
                      const int32_t* __restrict__ offsets, int n_lists, int rows, int topk,
                      int32_t* __restrict__ out_idx, float* __restrict__ out_score) {
  extern __shared__ uint64_t smem[];
  uint64_t* a = smem;             // running top-k
  uint64_t* b = smem + topk;      // incoming list
  uint64_t* c = smem + 2 * topk;  // merge output
  const int row = blockIdx.x;
  const uint32_t k = static_cast<uint32_t>(topk);
  auto load = [&](int l, uint64_t* dst) {
    const size_t base = (static_cast<size_t>(l) * rows + row) * k;
    const int32_t off = offsets ? offsets[static_cast<size_t>(l) * rows + row] : 0;
    for (uint32_t e = threadIdx.x; e < k; e += blockDim.x) {
      const int32_t i = idx[base + e];
      dst[e] = i >= 0 ? make_key(scores[base + e], static_cast<uint32_t>(i + off)) : 0ull;
    }
  };
  load(0, a);
  for (int l = 1; l < n_lists; ++l) {
    load(l, b);
    __syncthreads();
    for (uint32_t e = threadIdx.x; e < k; e += blockDim.x) {
      const uint32_t pa = e + count_above<true>(b, k, a[e]);
      if (pa < k) c[pa] = a[e];
      const uint32_t pb = e + count_above<false>(a, k, b[e]);
      if (pb < k) c[pb] = b[e];
    }
    __syncthreads();
    uint64_t* t = a;
    a = c;
    c = t;
  }
  __syncthreads();
  const size_t o = static_cast<size_t>(row) * k;
  for (uint32_t e = threadIdx.x; e < k; e += blockDim.x) {
    out_idx[o + e] = key_index(a[e]);
    if (out_score) out_score[o + e] = key_score(a[e]);
  }
}

}  // namespace

dsa_status launch_topk_merge(const float* scores, const int32_t* idx, const int32_t* offsets,
                             int n_lists, int rows, int topk, int32_t* out_idx, float* out_score,
                             cudaStream_t stream) {
  const size_t smem = 3u * static_cast<size_t>(topk) * sizeof(uint64_t);
  if (cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return DSA_ERR_CUDA;
  topk_merge_kernel<<<rows, kMergeThreads, smem, stream>>>(scores, idx, offsets, n_lists, rows, topk,
                                                           out_idx, out_score);
  return cuda_status(cudaGetLastError());
}

}  // namespace dsa
