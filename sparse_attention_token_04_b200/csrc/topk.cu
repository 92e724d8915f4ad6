// Top-k finishing kernels.
//   sort_rows_kernel   : orders each row's exact top-k keys (prefill winners) by key
//                        descending = (score descending, index ascending) and writes
//                        out_idx / out_score with -1 / -inf padding.
//   decode_topk_kernel : per request, exact top-k of its n_b stored scores (radix select on
//                        the 64-bit (score, position) key), then the same ordering.
#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace dsa {

__device__ __forceinline__ uint32_t next_pow2(uint32_t x) {
  uint32_t p = 1;
  while (p < x) p <<= 1;
  return p;
}

constexpr int kSortThreads = 256;

__global__ void __launch_bounds__(kSortThreads)
    sort_rows_kernel(const uint64_t* __restrict__ win, int topk, int32_t* __restrict__ out_idx,
                     float* __restrict__ out_score) {
  __shared__ uint64_t s[DSA_MAX_TOPK];
  const GroupSync<kSortThreads> gs{0};
  const uint32_t rank = threadIdx.x;
  const size_t row = blockIdx.x;
  const uint32_t P = next_pow2(static_cast<uint32_t>(topk));
  const uint64_t* src = win + row * topk;
  for (uint32_t e = rank; e < P; e += kSortThreads) s[e] = (e < static_cast<uint32_t>(topk)) ? src[e] : 0ull;
  gs.sync();
  group_bitonic_sort_desc<kSortThreads>(s, P, rank, gs);
  for (uint32_t e = rank; e < static_cast<uint32_t>(topk); e += kSortThreads) {
    const uint64_t key = s[e];
    out_idx[row * topk + e] = key_index(key);
    if (out_score) out_score[row * topk + e] = key_score(key);
  }
}

dsa_status launch_sort_rows(const uint64_t* win, int rows, int topk, int32_t* out_idx,
                            float* out_score, cudaStream_t stream) {
  sort_rows_kernel<<<rows, kSortThreads, 0, stream>>>(win, topk, out_idx, out_score);
  return cuda_status(cudaGetLastError());
}

constexpr int kDecodeTopkThreads = 1024;

__global__ void __launch_bounds__(kDecodeTopkThreads)
    decode_topk_kernel(const float* __restrict__ scores, int max_len,
                       const int32_t* __restrict__ seq_lens, int topk,
                       int32_t* __restrict__ out_idx, float* __restrict__ out_score,
                       WsHeader* hdr) {
  __shared__ uint64_t s[DSA_MAX_TOPK];
  __shared__ uint32_t hist[kHistBins];
  __shared__ uint32_t scr[kDecodeTopkThreads / 32 + 2];
  const GroupSync<kDecodeTopkThreads> gs{0};
  const uint32_t rank = threadIdx.x;
  const int b = blockIdx.x;
  int n = seq_lens[b];
  if (n < 1 || n > max_len) {
    if (rank == 0) record_error(hdr, DSA_ERR_DEVICE, DETAIL_BAD_SEQ_LEN);
    n = n < 1 ? 1 : max_len;
  }
  const float* row = scores + static_cast<size_t>(b) * max_len;
  auto key_at = [&](uint32_t e) { return make_key(row[e], e); };
  const uint32_t P = next_pow2(static_cast<uint32_t>(topk));
  const uint32_t un = static_cast<uint32_t>(n), uk = static_cast<uint32_t>(topk);
  if (un <= uk) {
    for (uint32_t e = rank; e < P; e += kDecodeTopkThreads) s[e] = (e < un) ? key_at(e) : 0ull;
  } else {
    for (uint32_t e = uk + rank; e < P; e += kDecodeTopkThreads) s[e] = 0ull;
    const uint64_t T = group_kth_threshold<kDecodeTopkThreads>(key_at, un, uk, rank, hist, scr, gs);
    group_compact_ge<kDecodeTopkThreads>(key_at, un, T, [&](uint32_t pos, uint64_t key) { if (pos < uk) s[pos] = key; },
                                         rank, scr, gs);
  }
  gs.sync();
  group_bitonic_sort_desc<kDecodeTopkThreads>(s, P, rank, gs);
  for (uint32_t e = rank; e < uk; e += kDecodeTopkThreads) {
    const uint64_t key = s[e];
    out_idx[static_cast<size_t>(b) * topk + e] = key_index(key);
    if (out_score) out_score[static_cast<size_t>(b) * topk + e] = key_score(key);
  }
}

dsa_status launch_decode_topk(const float* scores, int max_len, const int32_t* seq_lens, int B,
                              int topk, int32_t* out_idx, float* out_score, void* ws,
                              cudaStream_t stream) {
  decode_topk_kernel<<<B, kDecodeTopkThreads, 0, stream>>>(
      scores, max_len, seq_lens, topk, out_idx, out_score, static_cast<WsHeader*>(ws));
  return cuda_status(cudaGetLastError());
}

}  // namespace dsa
