// Top-k kernels.
//   prefill_sample_threshold_kernel : per prefill query, the lean pass's threshold from the
//                           query's sampled keys.
//   prefill_finish_kernel : per prefill query, the exact top-k of the candidate buffer the
//                           fused scoring kernel left (four warp segments and a threshold),
//                           ordered by (score descending, index ascending) and padded with
//                           -1 / -inf.
//   decode_topk_kernel    : per request, exact top-k of its n_b stored scores. The scoring
//                           kernel has already counted the request's scores in 2048 bins of
//                           their order-preserving top 11 bits; the bin holding the k-th score
//                           bounds the candidates, which one pass over the scores collects into
//                           shared memory. The bucket ranking of the finish kernel orders them
//                           (radix select + merge sort with heavy ties), same order and padding.
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
// One warp per row: a radix select on the 64-bit keys with digits of up to 8 bits, starting at
// the highest bit where the row's smallest and largest sampled key differ, with a warp-private
// 256-bin histogram; no block-wide barrier.
constexpr int kThrWarps = 8;

__global__ void __launch_bounds__(32 * kThrWarps)
    prefill_sample_threshold_kernel(const uint64_t* __restrict__ cand, const uint32_t* __restrict__ counts,
                                    uint64_t* __restrict__ thr, uint32_t seg_stride, int rows, int q_pos0,
                                    int Lk, int topk) {
  __shared__ uint32_t hist_all[kThrWarps][256];
  const uint32_t lane = threadIdx.x & 31u, wi = threadIdx.x >> 5;
  const int row = blockIdx.x * kThrWarps + static_cast<int>(wi);
  if (row >= rows) return;  // warp-uniform; the block has no barrier
  uint32_t* hist = hist_all[wi];
  const uint64_t* buf = cand + static_cast<size_t>(row) * 4u * seg_stride;
  uint32_t c[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const uint32_t v = __ldcg(counts + static_cast<size_t>(row) * 4 + w);
    c[w] = v < seg_stride ? v : seg_stride;
  }
  const uint32_t o1 = c[0], o2 = o1 + c[1], o3 = o2 + c[2], ns = o3 + c[3];
  const int keys = min(q_pos0 + row + 1, Lk);
  const double rho = static_cast<double>(topk) * ns / keys;
  const double rr = rho + 6.5 * sqrt(rho) + 1.0;
  if (rr >= static_cast<double>(ns)) {
    if (lane == 0) thr[row] = 0ull;
    return;
  }
  const uint32_t r = static_cast<uint32_t>(ceil(rr));
  auto key_at = [&](uint32_t e) {
    const uint32_t w = (e >= o1 ? 1u : 0u) + (e >= o2 ? 1u : 0u) + (e >= o3 ? 1u : 0u);
    const uint32_t start = e >= o3 ? o3 : (e >= o2 ? o2 : (e >= o1 ? o1 : 0u));
    return __ldcg(buf + w * seg_stride + (e - start));
  };
  // Bits common to every sampled key are fixed from the start.
  // Eight independent loads in flight per lane in every pass over the samples.
  constexpr int kBatch = 8;
  uint64_t mn = ~0ull, mx = 0ull;
  for (uint32_t e0 = 0; e0 < ns; e0 += 32 * kBatch) {
    uint64_t v[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const uint32_t e = e0 + i * 32 + lane;
      v[i] = e < ns ? key_at(e) : 0ull;
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const uint32_t e = e0 + i * 32 + lane;
      if (e < ns) {
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
    for (uint32_t e0 = 0; e0 < ns; e0 += 32 * kBatch) {
      uint64_t v[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const uint32_t e = e0 + i * 32 + lane;
        v[i] = e < ns ? key_at(e) : 0ull;
      }
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const uint32_t e = e0 + i * 32 + lane;
        if (e < ns && (v[i] & mask) == prefix)
          atomicAdd(&hist[static_cast<uint32_t>(v[i] >> shift) & dmask], 1u);
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
  (void)max_samples;
  const int grid = (rows + kThrWarps - 1) / kThrWarps;
  prefill_sample_threshold_kernel<<<grid, 32 * kThrWarps, 0, stream>>>(cand, counts, thr, seg_stride, rows,
                                                                      q_pos0, Lk, topk);
  return cuda_status(cudaGetLastError());
}

constexpr int kDecodeTopkThreads = 1024;
constexpr uint32_t kDecodeCandCap = 8192;
constexpr int kDecodeBuckets = 4096;

struct DecodeTopkSmem {
  uint64_t a[kSortBuf];             // sort buffer; before that the bucket counts of the ranking
  uint64_t win[DSA_MAX_TOPK];       // the k winners, contiguous (select path)
  uint64_t cand[kDecodeCandCap];    // candidates, ranked in place; or the second sort buffer
  uint32_t hist[kHistBins];
  GroupScratch<kDecodeTopkThreads> sc;
  uint32_t n_cand, big, omin, omax;
};
static_assert(kDecodeCandCap >= static_cast<uint32_t>(kSortBuf), "second sort buffer");
static_assert(sizeof(uint64_t) * kSortBuf >= sizeof(uint32_t) * kDecodeBuckets, "bucket counts in a");

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
  uint32_t* bk = reinterpret_cast<uint32_t*>(sm.a);
  for (uint32_t b = rank; b < static_cast<uint32_t>(kDecodeBuckets); b += kDecodeTopkThreads) bk[b] = 0u;
  if (rank == 0) {
    sm.n_cand = 0u;
    sm.omin = 0xFFFFFFFFu;
    sm.omax = 0u;
  }

  // Boundary bin: the highest bin where the count of scores at or above it reaches k (bin 0
  // when the request has at most k keys: every key is a winner).
  uint32_t bstar = 0, n_cand = un;
  if (un > k) {
    for (uint32_t b = rank; b < kHistBins; b += kDecodeTopkThreads)
      sm.hist[b] = bins[static_cast<size_t>(req) * kHistBins + b];
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
    bstar = sm.sc.w[kDecodeTopkThreads / 32];
    n_cand = sm.sc.w[kDecodeTopkThreads / 32 + 1];
    gs.sync();
  }
  for (uint32_t b = rank; b < kHistBins; b += kDecodeTopkThreads) sm.hist[b] = 0u;  // selects below need it zero
  gs.sync();

  const uint64_t* res = sm.cand;
  bool padded = false;
  uint32_t n_res = 0;
  if (n_cand <= kDecodeCandCap) {
    // One pass: keys whose bin is at or above the boundary bin, 32 score loads in flight per
    // thread (a 200000-key request in seven rounds), with their score range.
    constexpr int kInFlight = 32;
    uint32_t lmin = 0xFFFFFFFFu, lmax = 0u;
    for (uint32_t e0 = 0; e0 < un; e0 += kInFlight * kDecodeTopkThreads) {
      float v[kInFlight];
#pragma unroll
      for (int i = 0; i < kInFlight; ++i) {
        const uint32_t e = e0 + i * kDecodeTopkThreads + rank;
        v[i] = e < un ? __ldcg(row + e) : 0.0f;
      }
#pragma unroll
      for (int i = 0; i < kInFlight; ++i) {
        const uint32_t e = e0 + i * kDecodeTopkThreads + rank;
        const uint64_t key = make_key(v[i], e);
        const bool take = e < un && static_cast<uint32_t>(key >> 53) >= bstar;
        const uint32_t m = __ballot_sync(0xFFFFFFFFu, take);
        if (m) {
          uint32_t base = 0;
          if (lane == 0) base = atomicAdd(&sm.n_cand, static_cast<uint32_t>(__popc(m)));
          base = __shfl_sync(0xFFFFFFFFu, base, 0);
          const uint32_t pos = base + __popc(m & ((1u << lane) - 1u));
          if (take && pos < kDecodeCandCap) sm.cand[pos] = key;
          if (take) {
            const uint32_t o = static_cast<uint32_t>(key >> 32);
            lmin = o < lmin ? o : lmin;
            lmax = o > lmax ? o : lmax;
          }
        }
      }
    }
    lmin = __reduce_min_sync(0xFFFFFFFFu, lmin);
    lmax = __reduce_max_sync(0xFFFFFFFFu, lmax);
    if (lane == 0 && lmax != 0u) {
      atomicMin(&sm.omin, lmin);
      atomicMax(&sm.omax, lmax);
    }
    gs.sync();
    const uint32_t got = sm.n_cand < kDecodeCandCap ? sm.n_cand : kDecodeCandCap;
    if (got != n_cand && rank == 0) record_error(hdr, DSA_ERR_DEVICE, DETAIL_HIST_MISMATCH);
    if (got > 0 &&
        group_bucket_rank<kDecodeTopkThreads, kDecodeCandCap / kDecodeTopkThreads, kDecodeBuckets>(
            sm.cand, got, k, sm.omin, sm.omax, 256u, bk, &sm.big, sm.sc, gs, rank)) {
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
