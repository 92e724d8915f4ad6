// Top-k kernels.
//   prefill_sample_threshold_kernel : per prefill query, the lean pass's threshold from the
//                           query's sampled keys.
//   prefill_finish_kernel : per prefill query, the exact top-k of the candidate buffer the
//                           fused scoring kernel left (four warp segments and a threshold),
//                           ordered by (score descending, index ascending) and padded with
//                           -1 / -inf.
//   decode_collect_kernel : per decode request, the candidates of its exact top-k. The scoring
//                           kernel has already counted the request's scores in 2048 bins of
//                           their order-preserving top 11 bits; the bin holding the k-th score
//                           bounds the candidates, which several CTAs per request gather from
//                           the stored scores into the request's candidate list.
//   decode_rank_kernel    : per decode request, the candidates ordered by the bucket ranking of
//                           the finish kernel (radix select + merge sort with heavy ties), same
//                           order and padding.
#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace dsa {

constexpr int kSortBuf = sort_buffer_len(DSA_MAX_TOPK);

// Prefill finish. Every key a row's candidate buffer holds is at or above the row's threshold
// (the lean pass appends only such keys, the exact pass compacts to them), so the buffer is the
// candidate set itself. Persistent CTAs walk rows r, r + G, ...; while one row is ranked, the
// next row's buffer is copied into the other half of shared memory with cp.async. The ranking
// is group_bucket_rank (4096 value-linear buckets); a row with heavy ties (a bucket over
// kBucketMax keys) or more keys than a staging buffer holds falls back to an exact radix select
// and a merge sort. The k largest keys are written in order, padded with -1 / -inf.
constexpr int kFinishThreads = 512;
constexpr uint32_t kFinishTmp = 4608;
constexpr int kFinishKPT = kFinishTmp / kFinishThreads;  // keys ranked per thread
constexpr int kFinishBuckets = 4096;
constexpr uint32_t kBucketMax = 256;

struct FinishSmem {
  uint64_t buf[2][kFinishTmp];   // staged candidates of the current and the next row
  uint32_t bk[kFinishBuckets];   // bucket counts / radix histogram, then (select path) winners
  GroupScratch<kFinishThreads> sc;
  uint32_t n[2];                 // candidates of the row staged in each buffer
  uint32_t big;
  uint32_t omin, omax;           // order-preserving score bits of the smallest / largest key
};
static_assert(kFinishTmp % kFinishThreads == 0, "keys per thread");
static_assert(kFinishTmp >= 2u * static_cast<uint32_t>(kSortBuf), "merge-sort buffers in a staging buffer");
static_assert(kFinishBuckets * sizeof(uint32_t) >= DSA_MAX_TOPK * sizeof(uint64_t), "winners in bk");
static_assert(kFinishBuckets >= kHistBins, "radix histogram in bk");

struct RowSegments {
  const uint64_t* buf;
  uint32_t o1, o2, o3, n, segcap;
  __device__ __forceinline__ const uint64_t* at(uint32_t e) const {
    const uint32_t w = (e >= o1 ? 1u : 0u) + (e >= o2 ? 1u : 0u) + (e >= o3 ? 1u : 0u);
    const uint32_t start = e >= o3 ? o3 : (e >= o2 ? o2 : (e >= o1 ? o1 : 0u));
    return buf + w * segcap + (e - start);
  }
};

__device__ __forceinline__ RowSegments row_segments(const uint64_t* cand, const uint32_t* counts,
                                                    uint32_t pitch, size_t row) {
  RowSegments r;
  r.segcap = pitch / 4u;
  r.buf = cand + row * pitch;
  uint32_t c[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const uint32_t v = __ldcg(counts + row * 4 + w);
    c[w] = v < r.segcap ? v : r.segcap;
  }
  r.o1 = c[0];
  r.o2 = r.o1 + c[1];
  r.o3 = r.o2 + c[2];
  r.n = r.o3 + c[3];
  return r;
}

__global__ void __launch_bounds__(kFinishThreads, 2)
    prefill_finish_kernel(const uint64_t* __restrict__ cand, const uint32_t* __restrict__ counts,
                          uint32_t pitch, int rows, int topk, int32_t* __restrict__ out_idx,
                          float* __restrict__ out_score) {
  extern __shared__ uint8_t smem_raw[];
  FinishSmem& sm = *reinterpret_cast<FinishSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~static_cast<uintptr_t>(15));
  const GroupSync<kFinishThreads> gs{0};
  const uint32_t rank = threadIdx.x, lane = rank & 31u;
  const uint32_t k = static_cast<uint32_t>(topk);
  const int G = gridDim.x;

  // Copies a row's candidates into buf[b] (one cp.async group per thread, possibly empty).
  auto stage = [&](int row, int b) {
    const RowSegments seg = row_segments(cand, counts, pitch, static_cast<size_t>(row));
    if (seg.n <= kFinishTmp)
      for (uint32_t e = rank; e < seg.n; e += kFinishThreads) cp_async_8(&sm.buf[b][e], seg.at(e));
    cp_async_commit();
    if (rank == 0) sm.n[b] = seg.n;
  };

  for (uint32_t b = rank; b < kFinishBuckets; b += kFinishThreads) sm.bk[b] = 0u;
  if (static_cast<int>(blockIdx.x) < rows) stage(blockIdx.x, 0);
  int i = 0;
  for (int row = blockIdx.x; row < rows; row += G, ++i) {
    const int b = i & 1;
    // Prefetch the next row into the other buffer (free since the previous row's last barrier).
    if (row + G < rows) stage(row + G, b ^ 1);
    else cp_async_commit();
    if (rank == 0) {
      sm.omin = 0xFFFFFFFFu;
      sm.omax = 0u;
    }
    cp_async_wait<1>();  // this thread's copies of the current row have landed
    gs.sync();
    const uint32_t n = sm.n[b];
    uint64_t* keys = sm.buf[b];
    const uint64_t* res = keys;
    bool padded = false;
    uint32_t n_res = 0;
    bool need_select = n > kFinishTmp;
    if (!need_select && n > 0) {
      uint32_t lmin = 0xFFFFFFFFu, lmax = 0u;
      for (uint32_t e = rank; e < n; e += kFinishThreads) {
        const uint32_t o = static_cast<uint32_t>(keys[e] >> 32);
        lmin = o < lmin ? o : lmin;
        lmax = o > lmax ? o : lmax;
      }
      lmin = __reduce_min_sync(0xFFFFFFFFu, lmin);
      lmax = __reduce_max_sync(0xFFFFFFFFu, lmax);
      if (lane == 0) {
        atomicMin(&sm.omin, lmin);
        atomicMax(&sm.omax, lmax);
      }
      gs.sync();
      if (group_bucket_rank<kFinishThreads, kFinishKPT, kFinishBuckets>(
              keys, n, k, sm.omin, sm.omax, kBucketMax, sm.bk, &sm.big, sm.sc, gs, rank))
        n_res = n < k ? n : k;
      else
        need_select = true;  // bk is zero again
    }
    if (need_select) {
      // Exact radix select of the k-th key and a merge sort of the winners (bk is zero here).
      uint64_t* win = reinterpret_cast<uint64_t*>(sm.bk);
      uint32_t nw;
      if (n <= kFinishTmp) {
        auto key_at = [keys](uint32_t e) { return keys[e]; };
        const uint64_t T = n > k ? group_kth_threshold<kFinishThreads>(key_at, n, k, rank, sm.bk, sm.sc, gs) : 0ull;
        nw = group_compact_ge<kFinishThreads>(
            key_at, n, T, [&](uint32_t pos, uint64_t key) { if (pos < k) win[pos] = key; }, rank, sm.sc, gs);
      } else {
        const RowSegments seg = row_segments(cand, counts, pitch, static_cast<size_t>(row));
        auto key_at = [&](uint32_t e) { return __ldcg(seg.at(e)); };
        const uint64_t T = group_kth_threshold<kFinishThreads>(key_at, n, k, rank, sm.bk, sm.sc, gs);
        nw = group_compact_ge<kFinishThreads>(
            key_at, n, T, [&](uint32_t pos, uint64_t key) { if (pos < k) win[pos] = key; }, rank, sm.sc, gs);
      }
      nw = nw < k ? nw : k;
      res = group_merge_sort_desc<kFinishThreads>(
          [&](uint32_t e) { return e < nw ? win[e] : 0ull; }, keys, keys + kSortBuf, sort_size(k), rank, gs);
      padded = true;
      n_res = nw;
    }
    int32_t* oi = out_idx + static_cast<size_t>(row) * k;
    float* os = out_score ? out_score + static_cast<size_t>(row) * k : nullptr;
    for (uint32_t e = rank; e < k; e += kFinishThreads) {
      const uint64_t key = e < n_res ? res[padded ? spad(e) : e] : 0ull;
      oi[e] = key_index(key);
      if (os) os[e] = key_score(key);
    }
    gs.sync();  // the row's buffers are free
    for (uint32_t bb = rank; bb < kFinishBuckets; bb += kFinishThreads) sm.bk[bb] = 0u;
  }
  cp_async_wait<0>();
}

dsa_status launch_prefill_finish(const uint64_t* cand, const uint32_t* counts,
                                 const uint64_t* thr, uint32_t pitch, int rows, int topk,
                                 int32_t* out_idx, float* out_score, int num_sms, cudaStream_t stream) {
  (void)thr;  // every buffered key is at or above the row's threshold already
  const size_t smem = sizeof(FinishSmem) + 16;
  if (cudaFuncSetAttribute(prefill_finish_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return DSA_ERR_CUDA;
  const int grid = rows < 2 * num_sms ? rows : 2 * num_sms;
  prefill_finish_kernel<<<grid, kFinishThreads, smem, stream>>>(cand, counts, pitch, rows, topk,
                                                                out_idx, out_score);
  return cuda_status(cudaGetLastError());
}

// Lean-pass threshold of one prefill query from a uniform sample of its keys. The query's row
// holds n keys, n_s of them sampled (four segments, seg_stride apart); about rho = k n_s / n
// sampled keys lie above the row's k-th largest key, with a binomial spread of sqrt(rho). T is
// the r-th largest sampled key for r = rho + 6.5 sqrt(rho) + 1: more than r sampled keys above
// the k-th largest key is a 6.5-sigma event, and otherwise at least k keys of the row are >= T.
// A row with r >= n_s (short rows, n <= k) gets T = 0: every key is kept. (The lean pass checks
// the count it actually appended and hands the rare failure to the exact pass.)
// Per prefill row (one warp), the lean pass's threshold: the sampled key of rank r (largest
// first), by radix passes with 8-bit digits below the bits every sample shares. STAGED: the
// row's samples are read from global memory once into the warp's shared-memory stage and the
// passes read the stage (rows of up to kThrStageMax samples, eight warps per block); otherwise
// every pass reads global memory with eight loads in flight per lane, which keeps many more
// rows in flight than a stage of a long row's samples would allow.
constexpr int kThrWarps = 8;
constexpr uint32_t kThrStageMax = 1024;

template <bool STAGED>
__global__ void __launch_bounds__(32 * kThrWarps)
    prefill_sample_threshold_kernel(const uint64_t* __restrict__ cand, const uint32_t* __restrict__ counts,
                                    uint64_t* __restrict__ thr, uint32_t seg_stride, int rows, int q_pos0,
                                    int Lk, int topk) {
  __shared__ uint32_t hist_all[kThrWarps][256];
  extern __shared__ uint64_t stage_all[];  // STAGED: kThrWarps x kThrStageMax keys
  const uint32_t lane = threadIdx.x & 31u, wi = threadIdx.x >> 5;
  const int row = blockIdx.x * kThrWarps + static_cast<int>(wi);
  if (row >= rows) return;  // warp-uniform; the block has no barrier
  uint32_t* hist = hist_all[wi];
  uint64_t* stage = stage_all + (STAGED ? wi * kThrStageMax : 0u);
  const uint64_t* buf = cand + static_cast<size_t>(row) * 4u * seg_stride;
  uint32_t c[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const uint32_t v = __ldcg(counts + static_cast<size_t>(row) * 4 + w);
    c[w] = v < seg_stride ? v : seg_stride;
  }
  const uint32_t o1 = c[0], o2 = o1 + c[1], o3 = o2 + c[2];
  const uint32_t ns = STAGED ? min(o3 + c[3], kThrStageMax) : o3 + c[3];
  const int keys = min(q_pos0 + row + 1, Lk);
  const double rho = static_cast<double>(topk) * ns / keys;
  const double rr = rho + 6.5 * sqrt(rho) + 1.0;
  if (rr >= static_cast<double>(ns)) {
    if (lane == 0) thr[row] = 0ull;
    return;
  }
  const uint32_t r = static_cast<uint32_t>(ceil(rr));
  auto global_at = [&](uint32_t e) {
    const uint32_t w = (e >= o1 ? 1u : 0u) + (e >= o2 ? 1u : 0u) + (e >= o3 ? 1u : 0u);
    const uint32_t start = e >= o3 ? o3 : (e >= o2 ? o2 : (e >= o1 ? o1 : 0u));
    return __ldcg(buf + w * seg_stride + (e - start));
  };
  // First pass: the samples' range (and, STAGED, the stage).
  constexpr int kBatch = 8;
  uint64_t mn = ~0ull, mx = 0ull;
  for (uint32_t e0 = 0; e0 < ns; e0 += 32 * kBatch) {
    uint64_t v[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const uint32_t e = e0 + i * 32 + lane;
      v[i] = e < ns ? global_at(e) : 0ull;
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const uint32_t e = e0 + i * 32 + lane;
      if (e < ns) {
        if (STAGED) stage[e] = v[i];
        mn = v[i] < mn ? v[i] : mn;
        mx = v[i] > mx ? v[i] : mx;
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const uint64_t a = __shfl_xor_sync(0xFFFFFFFFu, mn, off), b = __shfl_xor_sync(0xFFFFFFFFu, mx, off);
    mn = a < mn ? a : mn;
    mx = b > mx ? b : mx;
  }
  __syncwarp();
  // Bits common to every sampled key are fixed from the start.
  int hb = 63 - __clzll(static_cast<long long>(mn ^ mx));
  uint64_t mask = (hb >= 63) ? 0ull : ~((2ull << hb) - 1ull);
  uint64_t prefix = mx & mask;
  uint32_t need = r, taken = 0;
  while (true) {
    const int shift = hb >= 7 ? hb - 7 : 0;
    const uint32_t dmask = (2u << (hb - shift)) - 1u;
#pragma unroll
    for (int i = 0; i < 8; ++i) hist[lane * 8 + i] = 0u;
    __syncwarp();
    if constexpr (STAGED) {
      for (uint32_t e = lane; e < ns; e += 32) {
        const uint64_t v = stage[e];
        if ((v & mask) == prefix) atomicAdd(&hist[static_cast<uint32_t>(v >> shift) & dmask], 1u);
      }
    } else {
      for (uint32_t e0 = 0; e0 < ns; e0 += 32 * kBatch) {
        uint64_t v[kBatch];
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
          const uint32_t e = e0 + i * 32 + lane;
          v[i] = e < ns ? global_at(e) : 0ull;
        }
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
          const uint32_t e = e0 + i * 32 + lane;
          if (e < ns && (v[i] & mask) == prefix)
            atomicAdd(&hist[static_cast<uint32_t>(v[i] >> shift) & dmask], 1u);
        }
      }
    }
    __syncwarp();
    // Bins 8*lane .. 8*lane+7; keys in higher bins come first.
    uint32_t cb[8], local = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      cb[i] = hist[lane * 8 + i];
      local += cb[i];
    }
    uint32_t suf = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t o = __shfl_down_sync(0xFFFFFFFFu, suf, off);
      if (lane + off < 32) suf += o;
    }
    uint32_t acc = suf - local;
    uint32_t hit = 0xFFFFFFFFu, hit_above = 0, hit_in = 0;
#pragma unroll
    for (int i = 7; i >= 0; --i) {
      if (acc < need && acc + cb[i] >= need) {
        hit = lane * 8 + i;
        hit_above = acc;
        hit_in = cb[i];
      }
      acc += cb[i];
    }
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, hit != 0xFFFFFFFFu);
    const int src = __ffs(bal) - 1;  // exactly one lane holds the bin of the need-th key
    const uint32_t bin = __shfl_sync(0xFFFFFFFFu, hit, src);
    const uint32_t above = __shfl_sync(0xFFFFFFFFu, hit_above, src);
    const uint32_t in_bin = __shfl_sync(0xFFFFFFFFu, hit_in, src);
    need -= above;
    taken += above;
    prefix |= static_cast<uint64_t>(bin) << shift;
    mask |= static_cast<uint64_t>(dmask) << shift;
    __syncwarp();
    if (taken + in_bin <= r || shift == 0) break;
    hb = shift - 1;
  }
  if (lane == 0) thr[row] = prefix;
}

dsa_status launch_prefill_sample_threshold(const uint64_t* cand, const uint32_t* counts,
                                           uint64_t* thr, uint32_t seg_stride, int rows,
                                           int q_pos0, int Lk, int topk, uint32_t max_samples,
                                           cudaStream_t stream) {
  // A row holds at most max_samples sampled keys (and at most its four segments).
  const uint32_t most = max_samples < 4u * seg_stride ? max_samples : 4u * seg_stride;
  const int grid = (rows + kThrWarps - 1) / kThrWarps;
  if (most <= kThrStageMax) {
    constexpr size_t smem = static_cast<size_t>(kThrWarps) * kThrStageMax * sizeof(uint64_t);
    if (cudaFuncSetAttribute(prefill_sample_threshold_kernel<true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
      return DSA_ERR_CUDA;
    prefill_sample_threshold_kernel<true><<<grid, 32 * kThrWarps, smem, stream>>>(cand, counts, thr, seg_stride,
                                                                                rows, q_pos0, Lk, topk);
  } else
    prefill_sample_threshold_kernel<false><<<grid, 32 * kThrWarps, 0, stream>>>(cand, counts, thr, seg_stride,
                                                                              rows, q_pos0, Lk, topk);
  return cuda_status(cudaGetLastError());
}

// Decode collection: CTA (c, b) takes scores [c * kCollectChunk, (c + 1) * kCollectChunk) of
// request b. Two bulk copies bring its scores into shared memory while the CTA finds the
// request's boundary bin from the histogram: the highest bin at or above which at least k
// scores lie (bin 0 when the request has at most k keys: every key is a winner). The keys at or
// above that bin are appended to the request's candidate list, with one atomic reservation per
// CTA, and the CTA's ordered score range is merged into the request's state (two more atomics).
constexpr int kCollectThreads = 512;
constexpr int kCollectParts = 2;
constexpr int kCollectPart = 4096;  // scores per bulk copy
constexpr int kCollectChunk = kCollectParts * kCollectPart;
static_assert(kDecodeScoreBins == 4 * kCollectThreads, "four histogram bins per thread");
static_assert(kCollectPart == 8 * kCollectThreads, "two float4 per thread per part");

struct CollectSmem {
  float4 v[kCollectChunk / 4];
  uint64_t bar[kCollectParts];
  GroupScratch<kCollectThreads> sc;
  uint32_t bstar, n_cand, base, omin, omax;
  int abort;
};

__global__ void __launch_bounds__(kCollectThreads)
    decode_collect_kernel(const float* __restrict__ scores, int max_len,
                          const int32_t* __restrict__ seq_lens, const uint32_t* __restrict__ bins,
                          uint32_t* __restrict__ state, uint64_t* __restrict__ cand, int topk,
                          WsHeader* hdr, uint64_t budget_ns) {
  extern __shared__ uint8_t smem_raw[];
  CollectSmem& sm = *reinterpret_cast<CollectSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~static_cast<uintptr_t>(15));
  const GroupSync<kCollectThreads> gs{0};
  const uint32_t rank = threadIdx.x, lane = rank & 31u;
  const int req = blockIdx.y;
  int n = seq_lens[req];  // a bad length is recorded by the rank pass
  n = n < 1 ? 1 : (n > max_len ? max_len : n);
  const uint32_t un = static_cast<uint32_t>(n), k = static_cast<uint32_t>(topk);
  const uint32_t c0 = blockIdx.x * static_cast<uint32_t>(kCollectChunk);
  if (c0 >= un) return;
  const uint32_t len = min(un - c0, static_cast<uint32_t>(kCollectChunk));
  const uint32_t parts = (len + kCollectPart - 1) / kCollectPart;
  const float* src = scores + static_cast<size_t>(req) * max_len + c0;
  // Everything above reads only what was complete before the scoring kernel started; the
  // scores and the histogram below are that kernel's output.
  grid_dependency_wait();
  if (rank == 0) {
    for (uint32_t q = 0; q < parts; ++q) mbar_init(&sm.bar[q], 1);
    fence_mbar_init();
    // Every copy starts 16-byte aligned (rows of a multiple of 64 scores); the last one is
    // rounded up to whole float4, which stays inside the row.
    for (uint32_t q = 0; q < parts; ++q) {
      const uint32_t cnt = min(len - q * kCollectPart, static_cast<uint32_t>(kCollectPart));
      const uint32_t bytes = ((cnt + 3u) & ~3u) * static_cast<uint32_t>(sizeof(float));
      mbar_arrive_expect_tx(&sm.bar[q], bytes);
      bulk_load_1d(&sm.v[q * (kCollectPart / 4)], src + q * kCollectPart, bytes, &sm.bar[q]);
    }
    sm.abort = 0;
    sm.omin = 0xFFFFFFFFu;
    sm.omax = 0u;
    sm.bstar = 0u;
    sm.n_cand = un;
  }
  // Boundary bin from the request's histogram (complete: the scoring kernel has finished).
  if (un > k) {
    const uint4 h = __ldcg(reinterpret_cast<const uint4*>(bins + static_cast<size_t>(req) * kDecodeScoreBins) + rank);
    const uint32_t c[4] = {h.x, h.y, h.z, h.w};
    uint32_t acc = group_suffix_exclusive<kCollectThreads>(c[0] + c[1] + c[2] + c[3], rank, sm.sc.w, gs, nullptr);
#pragma unroll
    for (int i = 3; i >= 0; --i) {
      if (acc < k && acc + c[i] >= k) {
        sm.bstar = rank * 4u + static_cast<uint32_t>(i);
        sm.n_cand = acc + c[i];
      }
      acc += c[i];
    }
  }
  gs.sync();
  const uint32_t bstar = sm.bstar, n_cand = sm.n_cand;
  if (blockIdx.x == 0 && rank == 0) state[req * 4 + 3] = n_cand;
  const bool collect = n_cand <= kDecodeCandCap;  // else the rank pass selects from the scores
  const WaitCtl ctl{hdr, &sm.abort, budget_ns};

  // Pass 1: mark this thread's candidates (bit 8q + 4i + j: part q, float4 i, lane j).
  uint32_t mask = 0u, lmin = 0xFFFFFFFFu, lmax = 0u;
  bool ok = true;
  for (uint32_t q = 0; q < parts && collect; ++q) {
    ok = mbar_wait(&sm.bar[q], 0, ctl, DETAIL_WAIT_SCORES);
    if (!ok) break;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint32_t f4 = q * (kCollectPart / 4) + static_cast<uint32_t>(i) * kCollectThreads + rank;
      const float4 v = sm.v[f4];
      const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t o = float_to_ordered(vv[j] + 0.0f);
        if (4u * f4 + j < len && (o >> 21) >= bstar) {
          mask |= 1u << (8u * q + 4u * i + j);
          lmin = min(lmin, o);
          lmax = max(lmax, o);
        }
      }
    }
  }
  ok = named_bar_and(0, kCollectThreads, ok);
  if (collect && ok) {
    // Pass 2: reserve this CTA's slice of the candidate list, then write the keys.
    uint32_t total = 0;
    const uint32_t off = group_prefix_exclusive<kCollectThreads>(__popc(mask), rank, sm.sc.w, gs, &total);
    lmin = __reduce_min_sync(0xFFFFFFFFu, lmin);
    lmax = __reduce_max_sync(0xFFFFFFFFu, lmax);
    if (lane == 0 && lmax != 0u) {
      atomicMin(&sm.omin, lmin);
      atomicMax(&sm.omax, lmax);
    }
    gs.sync();
    if (rank == 0 && total > 0) {
      sm.base = atomicAdd(&state[req * 4 + 0], total);
      atomicMax(&state[req * 4 + 1], sm.omax);
      atomicMax(&state[req * 4 + 2], ~sm.omin);
    }
    gs.sync();
    uint64_t* dst = cand + static_cast<size_t>(req) * kDecodeCandCap;
    uint32_t pos = sm.base + off;
    while (mask) {
      const uint32_t bit = __ffs(mask) - 1u;
      mask &= mask - 1u;
      const uint32_t f4 = (bit >> 3) * (kCollectPart / 4) + ((bit >> 2) & 1u) * kCollectThreads + rank;
      const float v = reinterpret_cast<const float*>(sm.v)[4u * f4 + (bit & 3u)];
      if (pos < kDecodeCandCap) dst[pos] = make_key(v, c0 + 4u * f4 + (bit & 3u));
      ++pos;
    }
  } else if (rank == 0) {
    // Let every copy this CTA issued land before it exits (bounded).
    for (uint32_t q = 0; q < parts; ++q) mbar_wait_drain(&sm.bar[q], 0, budget_ns);
  }
  grid_launch_dependents();
}

// Decode rank: one CTA per request orders the request's candidates (group_bucket_rank; heavy
// ties fall back to a radix select and a merge sort) and writes the k best, padded with -1 / -inf.
// A request whose boundary bin holds too many keys for the candidate list is selected from its
// stored scores directly.
constexpr int kDecodeTopkThreads = 1024;
constexpr int kDecodeBuckets = 4096;

struct DecodeTopkSmem {
  uint64_t a[kSortBuf];             // sort buffer; before that the bucket counts of the ranking
  uint64_t win[DSA_MAX_TOPK];       // the k winners, contiguous (select path)
  uint64_t cand[kDecodeCandCap];    // candidates, ranked in place; or the second sort buffer
  uint32_t hist[kHistBins];
  GroupScratch<kDecodeTopkThreads> sc;
  uint32_t big;
};
static_assert(kDecodeCandCap >= static_cast<uint32_t>(kSortBuf), "second sort buffer");
static_assert(sizeof(uint64_t) * kSortBuf >= sizeof(uint32_t) * kDecodeBuckets, "bucket counts in a");

__global__ void __launch_bounds__(kDecodeTopkThreads)
    decode_rank_kernel(const float* __restrict__ scores, int max_len,
                       const int32_t* __restrict__ seq_lens, const uint32_t* __restrict__ state,
                       const uint64_t* __restrict__ cand_all, int topk,
                       int32_t* __restrict__ out_idx, float* __restrict__ out_score, WsHeader* hdr) {
  extern __shared__ uint8_t smem_raw[];
  DecodeTopkSmem& sm = *reinterpret_cast<DecodeTopkSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~static_cast<uintptr_t>(15));
  const GroupSync<kDecodeTopkThreads> gs{0};
  const uint32_t rank = threadIdx.x;
  const int req = blockIdx.x;
  int n = seq_lens[req];
  if (n < 1 || n > max_len) {
    if (rank == 0) record_error(hdr, DSA_ERR_DEVICE, DETAIL_BAD_SEQ_LEN);
    n = n < 1 ? 1 : max_len;
  }
  const float* row = scores + static_cast<size_t>(req) * max_len;
  auto key_at = [&](uint32_t e) { return make_key(__ldcg(row + e), e); };
  const uint32_t un = static_cast<uint32_t>(n), k = static_cast<uint32_t>(topk);
  uint32_t* bk = reinterpret_cast<uint32_t*>(sm.a);
  for (uint32_t b = rank; b < static_cast<uint32_t>(kDecodeBuckets); b += kDecodeTopkThreads) bk[b] = 0u;
  for (uint32_t b = rank; b < kHistBins; b += kDecodeTopkThreads) sm.hist[b] = 0u;  // selects need it zero
  // The collection pass (and, before it, the scoring kernel) has completed past this point.
  grid_dependency_wait();
  const uint4 st = __ldcg(reinterpret_cast<const uint4*>(state) + req);
  const uint32_t n_cand = st.w;

  const uint64_t* res = sm.cand;
  bool padded = false;
  uint32_t n_res = 0;
  if (n_cand <= kDecodeCandCap) {
    const uint32_t got = st.x < kDecodeCandCap ? st.x : kDecodeCandCap;
    const uint64_t* src = cand_all + static_cast<size_t>(req) * kDecodeCandCap;
    for (uint32_t e = rank; e < got; e += kDecodeTopkThreads) sm.cand[e] = __ldcg(src + e);
    gs.sync();
    if (got != n_cand && rank == 0) record_error(hdr, DSA_ERR_DEVICE, DETAIL_HIST_MISMATCH);
    if (got > 0 &&
        group_bucket_rank<kDecodeTopkThreads, kDecodeCandCap / kDecodeTopkThreads, kDecodeBuckets>(
            sm.cand, got, k, ~st.z, st.y, 256u, bk, &sm.big, sm.sc, gs, rank)) {
      n_res = got < k ? got : k;
    } else {
      // Heavy ties: exact radix select over the candidates, then a merge sort.
      auto cand_at = [&](uint32_t e) { return sm.cand[e]; };
      const uint64_t T = got > k ? group_kth_threshold<kDecodeTopkThreads>(cand_at, got, k, rank, sm.hist, sm.sc, gs)
                                 : 0ull;
      uint32_t nw = group_compact_ge<kDecodeTopkThreads>(
          cand_at, got, T, [&](uint32_t pos, uint64_t key) { if (pos < k) sm.win[pos] = key; }, rank,
          sm.sc, gs);
      nw = nw < k ? nw : k;
      res = group_merge_sort_desc<kDecodeTopkThreads>(
          [&](uint32_t e) { return e < nw ? sm.win[e] : 0ull; }, sm.a, sm.cand, sort_size(k), rank, gs);
      padded = true;
      n_res = nw;
    }
  } else {
    // Too many keys share the boundary bin (heavy ties): radix select over global memory.
    gs.sync();
    const uint64_t T = group_kth_threshold<kDecodeTopkThreads>(key_at, un, k, rank, sm.hist, sm.sc, gs);
    uint32_t nw = group_compact_ge<kDecodeTopkThreads>(
        key_at, un, T, [&](uint32_t pos, uint64_t key) { if (pos < k) sm.win[pos] = key; }, rank,
        sm.sc, gs);
    nw = nw < k ? nw : k;
    res = group_merge_sort_desc<kDecodeTopkThreads>(
        [&](uint32_t e) { return e < nw ? sm.win[e] : 0ull; }, sm.a, sm.cand, sort_size(k), rank, gs);
    padded = true;
    n_res = nw;
  }
  for (uint32_t e = rank; e < k; e += kDecodeTopkThreads) {
    const uint64_t key = e < n_res ? res[padded ? spad(e) : e] : 0ull;
    out_idx[static_cast<size_t>(req) * topk + e] = key_index(key);
    if (out_score) out_score[static_cast<size_t>(req) * topk + e] = key_score(key);
  }
}

dsa_status launch_decode_topk(void* ws, const DecodeLayout& lay, int max_len,
                              const int32_t* seq_lens, int B, int topk, int32_t* out_idx,
                              float* out_score, uint64_t budget_ns, cudaStream_t stream) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  const float* scores = reinterpret_cast<const float*>(base + lay.scores);
  const uint32_t* bins = reinterpret_cast<const uint32_t*>(base + lay.bins);
  uint32_t* state = reinterpret_cast<uint32_t*>(base + lay.state);
  uint64_t* cand = reinterpret_cast<uint64_t*>(base + lay.cand);
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  const size_t csmem = sizeof(CollectSmem) + 16;
  if (cudaFuncSetAttribute(decode_collect_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(csmem)) != cudaSuccess)
    return DSA_ERR_CUDA;
  // Both passes are launched as programmatic dependents of the kernel before them, so their
  // launch and prologue overlap its last CTAs; each waits for it before reading its output.
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((max_len + kCollectChunk - 1) / kCollectChunk, B);
  cfg.blockDim = dim3(kCollectThreads);
  cfg.dynamicSmemBytes = csmem;
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, decode_collect_kernel, scores, max_len, seq_lens, bins, state, cand, topk,
                         hdr, budget_ns) != cudaSuccess)
    return DSA_ERR_CUDA;
  const size_t smem = sizeof(DecodeTopkSmem) + 16;
  if (cudaFuncSetAttribute(decode_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return DSA_ERR_CUDA;
  cfg.gridDim = dim3(B);
  cfg.blockDim = dim3(kDecodeTopkThreads);
  cfg.dynamicSmemBytes = smem;
  if (cudaLaunchKernelEx(&cfg, decode_rank_kernel, scores, max_len, seq_lens,
                         static_cast<const uint32_t*>(state), static_cast<const uint64_t*>(cand), topk,
                         out_idx, out_score, hdr) != cudaSuccess)
    return DSA_ERR_CUDA;
  return cuda_status(cudaGetLastError());
}

}  // namespace dsa
