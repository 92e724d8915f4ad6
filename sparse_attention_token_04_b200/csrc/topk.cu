// Top-k finishing kernels.
//   prefill_finish_kernel : per prefill query, the exact top-k of the candidate buffer the
//                           fused scoring kernel left (four warp segments), ordered by
//                           (score descending, index ascending) and padded with -1 / -inf.
//   decode_topk_kernel    : per request, exact top-k of its n_b stored scores. The scoring
//                           kernel has already counted the request's scores in 2048 bins of
//                           their order-preserving top 11 bits; the bin holding the k-th score
//                           bounds the candidates, which one pass over the scores collects into
//                           shared memory. An exact radix select there and a merge sort finish
//                           the row, in the same order and padding.
#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace dsa {

constexpr int kSortBuf = sort_buffer_len(DSA_MAX_TOPK);

constexpr int kFinishThreads = 256;

struct FinishSmem {
  uint64_t stage[kPrefillCapMax];   // the row's candidates; later the two sort buffers
  uint64_t win[DSA_MAX_TOPK];       // the k winners, contiguous
  uint32_t hist[kHistBins];
  GroupScratch<kFinishThreads> sc;
};
static_assert(kPrefillCapMax >= 2u * static_cast<uint32_t>(kSortBuf), "sort buffers in the stage");

__global__ void __launch_bounds__(kFinishThreads)
    prefill_finish_kernel(const uint64_t* __restrict__ cand, const uint32_t* __restrict__ counts,
                          uint32_t cap, int topk, int32_t* __restrict__ out_idx,
                          float* __restrict__ out_score) {
  extern __shared__ uint8_t smem_raw[];
  FinishSmem& sm = *reinterpret_cast<FinishSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~static_cast<uintptr_t>(15));
  const GroupSync<kFinishThreads> gs{0};
  const uint32_t rank = threadIdx.x;
  const size_t row = blockIdx.x;
  const uint32_t k = static_cast<uint32_t>(topk);
  const uint32_t segcap = cap / 4u;
  const uint64_t* buf = cand + row * cap;
  uint32_t c[4], n = 0;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const uint32_t v = __ldcg(counts + row * 4 + w);
    c[w] = v < segcap ? v : segcap;
    n += c[w];
  }
  // Stage the four segments contiguously, four independent loads in flight per thread.
  const uint32_t o1 = c[0], o2 = o1 + c[1], o3 = o2 + c[2];
  auto src_of = [&](uint32_t e) -> const uint64_t* {
    const uint32_t w = (e >= o1 ? 1u : 0u) + (e >= o2 ? 1u : 0u) + (e >= o3 ? 1u : 0u);
    const uint32_t start = e >= o3 ? o3 : (e >= o2 ? o2 : (e >= o1 ? o1 : 0u));
    return buf + w * segcap + (e - start);
  };
  uint32_t e = rank;
  for (; e + 3 * kFinishThreads < n; e += 4 * kFinishThreads) {
    const uint64_t a0 = __ldcg(src_of(e)), a1 = __ldcg(src_of(e + kFinishThreads)),
                   a2 = __ldcg(src_of(e + 2 * kFinishThreads)), a3 = __ldcg(src_of(e + 3 * kFinishThreads));
    sm.stage[e] = a0;
    sm.stage[e + kFinishThreads] = a1;
    sm.stage[e + 2 * kFinishThreads] = a2;
    sm.stage[e + 3 * kFinishThreads] = a3;
  }
  for (; e < n; e += kFinishThreads) sm.stage[e] = __ldcg(src_of(e));
  for (uint32_t b = rank; b < kHistBins; b += kFinishThreads) sm.hist[b] = 0u;
  gs.sync();
  auto key_at = [&](uint32_t i) { return sm.stage[i]; };
  const uint64_t T = n > k ? group_kth_threshold<kFinishThreads>(key_at, n, k, rank, sm.hist, sm.sc, gs)
                           : 0ull;
  uint32_t n_win = group_compact_ge<kFinishThreads>(
      key_at, n, T, [&](uint32_t pos, uint64_t key) { if (pos < k) sm.win[pos] = key; }, rank, sm.sc, gs);
  n_win = n_win < k ? n_win : k;
  const uint64_t* s = group_merge_sort_desc<kFinishThreads>(
      [&](uint32_t i) { return i < n_win ? sm.win[i] : 0ull; }, sm.stage, sm.stage + kSortBuf,
      sort_size(k), rank, gs);
  int32_t* oi = out_idx + row * k;
  float* os = out_score ? out_score + row * k : nullptr;
  for (uint32_t i = rank; i < k; i += kFinishThreads) {
    const uint64_t key = s[spad(i)];
    oi[i] = key_index(key);
    if (os) os[i] = key_score(key);
  }
}

dsa_status launch_prefill_finish(const uint64_t* cand, const uint32_t* counts, uint32_t cap,
                                 int rows, int topk, int32_t* out_idx, float* out_score,
                                 cudaStream_t stream) {
  const size_t smem = sizeof(FinishSmem) + 16;
  if (cudaFuncSetAttribute(prefill_finish_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return DSA_ERR_CUDA;
  prefill_finish_kernel<<<rows, kFinishThreads, smem, stream>>>(cand, counts, cap, topk, out_idx,
                                                                out_score);
  return cuda_status(cudaGetLastError());
}

constexpr int kDecodeTopkThreads = 1024;
constexpr uint32_t kDecodeCandCap = 8192;

struct DecodeTopkSmem {
  uint64_t a[kSortBuf];             // sort buffer
  uint64_t win[DSA_MAX_TOPK];       // the k winners, contiguous
  uint64_t cand[kDecodeCandCap];    // candidates; later the second sort buffer
  uint32_t hist[kHistBins];
  GroupScratch<kDecodeTopkThreads> sc;
  uint32_t n_cand;
};
static_assert(kDecodeCandCap >= static_cast<uint32_t>(kSortBuf), "second sort buffer");

__global__ void __launch_bounds__(kDecodeTopkThreads)
    decode_topk_kernel(const float* __restrict__ scores, int max_len,
                       const int32_t* __restrict__ seq_lens, const uint32_t* __restrict__ bins,
                       int topk, int32_t* __restrict__ out_idx, float* __restrict__ out_score,
                       WsHeader* hdr) {
  extern __shared__ uint8_t smem_raw[];
  DecodeTopkSmem& sm = *reinterpret_cast<DecodeTopkSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~static_cast<uintptr_t>(15));
  const GroupSync<kDecodeTopkThreads> gs{0};
  const uint32_t rank = threadIdx.x, lane = rank & 31u;
  const int req = blockIdx.x;
  int n = seq_lens[req];
  if (n < 1 || n > max_len) {
    if (rank == 0) record_error(hdr, DSA_ERR_DEVICE, DETAIL_BAD_SEQ_LEN);
    n = n < 1 ? 1 : max_len;
  }
  const float* row = scores + static_cast<size_t>(req) * max_len;
  auto key_at = [&](uint32_t e) { return make_key(__ldcg(row + e), e); };
  const uint32_t un = static_cast<uint32_t>(n), k = static_cast<uint32_t>(topk);
  const uint32_t P = sort_size(k);
  uint32_t n_win = un < k ? un : k;

  if (un > k) {
    // Boundary bin: the highest bin where the count of scores at or above it reaches k.
    for (uint32_t b = rank; b < kHistBins; b += kDecodeTopkThreads)
      sm.hist[b] = bins[static_cast<size_t>(req) * kHistBins + b];
    if (rank == 0) sm.n_cand = 0;
    gs.sync();
    constexpr int BPT = kHistBins / kDecodeTopkThreads;
    uint32_t local = 0;
#pragma unroll
    for (int i = 0; i < BPT; ++i) local += sm.hist[rank * BPT + i];
    uint32_t acc = group_suffix_exclusive<kDecodeTopkThreads>(local, rank, sm.sc.w, gs, nullptr);
#pragma unroll
    for (int i = BPT - 1; i >= 0; --i) {
      const uint32_t c = sm.hist[rank * BPT + i];
      if (acc < k && acc + c >= k) {
        sm.sc.w[kDecodeTopkThreads / 32] = rank * BPT + i;
        sm.sc.w[kDecodeTopkThreads / 32 + 1] = acc + c;
      }
      acc += c;
    }
    gs.sync();
    const uint32_t bstar = sm.sc.w[kDecodeTopkThreads / 32];
    const uint32_t n_cand = sm.sc.w[kDecodeTopkThreads / 32 + 1];
    gs.sync();
    for (uint32_t b = rank; b < kHistBins; b += kDecodeTopkThreads) sm.hist[b] = 0u;  // selects below need it zero
    gs.sync();
    uint64_t T;
    if (n_cand <= kDecodeCandCap) {
      // One pass: keys whose bin is at or above the boundary bin, eight loads in flight.
      for (uint32_t e0 = 0; e0 < un; e0 += 8 * kDecodeTopkThreads) {
        uint64_t v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t e = e0 + i * kDecodeTopkThreads + rank;
          v[i] = e < un ? key_at(e) : 0ull;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const bool take = v[i] != 0ull && static_cast<uint32_t>(v[i] >> 53) >= bstar;
          const uint32_t m = __ballot_sync(0xFFFFFFFFu, take);
          if (m) {
            uint32_t base = 0;
            if (lane == 0) base = atomicAdd(&sm.n_cand, static_cast<uint32_t>(__popc(m)));
            base = __shfl_sync(0xFFFFFFFFu, base, 0);
            const uint32_t pos = base + __popc(m & ((1u << lane) - 1u));
            if (take && pos < kDecodeCandCap) sm.cand[pos] = v[i];
          }
        }
      }
      gs.sync();
      const uint32_t got = sm.n_cand < kDecodeCandCap ? sm.n_cand : kDecodeCandCap;
      if (got != n_cand && rank == 0) record_error(hdr, DSA_ERR_DEVICE, DETAIL_HIST_MISMATCH);
      auto cand_at = [&](uint32_t e) { return sm.cand[e]; };
      T = got > k ? group_kth_threshold<kDecodeTopkThreads>(cand_at, got, k, rank, sm.hist, sm.sc, gs)
                  : 0ull;
      n_win = group_compact_ge<kDecodeTopkThreads>(
          cand_at, got, T, [&](uint32_t pos, uint64_t key) { if (pos < k) sm.win[pos] = key; }, rank,
          sm.sc, gs);
    } else {
      // Too many keys share the boundary bin (heavy ties): radix select over global memory.
      T = group_kth_threshold<kDecodeTopkThreads>(key_at, un, k, rank, sm.hist, sm.sc, gs);
      n_win = group_compact_ge<kDecodeTopkThreads>(
          key_at, un, T, [&](uint32_t pos, uint64_t key) { if (pos < k) sm.win[pos] = key; }, rank,
          sm.sc, gs);
    }
    n_win = n_win < k ? n_win : k;
  } else {
    for (uint32_t e = rank; e < un; e += kDecodeTopkThreads) sm.win[e] = key_at(e);
  }
  gs.sync();
  const uint64_t* s = group_merge_sort_desc<kDecodeTopkThreads>(
      [&](uint32_t e) { return e < n_win ? sm.win[e] : 0ull; }, sm.a, sm.cand, P, rank, gs);
  for (uint32_t e = rank; e < k; e += kDecodeTopkThreads) {
    const uint64_t key = s[spad(e)];
    out_idx[static_cast<size_t>(req) * topk + e] = key_index(key);
    if (out_score) out_score[static_cast<size_t>(req) * topk + e] = key_score(key);
  }
}

dsa_status launch_decode_topk(const float* scores, int max_len, const int32_t* seq_lens,
                              const uint32_t* bins, int B, int topk, int32_t* out_idx,
                              float* out_score, void* ws, cudaStream_t stream) {
  const size_t smem = sizeof(DecodeTopkSmem) + 16;
  if (cudaFuncSetAttribute(decode_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return DSA_ERR_CUDA;
  decode_topk_kernel<<<B, kDecodeTopkThreads, smem, stream>>>(
      scores, max_len, seq_lens, bins, topk, out_idx, out_score, static_cast<WsHeader*>(ws));
  return cuda_status(cudaGetLastError());
}

}  // namespace dsa
