// Exact top-k selection primitives on 64-bit (score, index) keys for a group of NT threads
// that synchronise on one named barrier. Keys are distinct (the low word encodes the index),
// so "the k largest keys" is one well-defined set: the k best scores with ties going to the
// lower index.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kHistBins = 2048;  // radix digits of up to 11 bits

template <int NT>
struct GroupSync {
  uint32_t bar_id;
  __device__ __forceinline__ void sync() const { named_bar(bar_id, NT); }
};

// Scratch words a group needs: NT/32 + 4 (u32) and 2 * NT/32 (u64).
template <int NT>
struct GroupScratch {
  uint32_t w[NT / 32 + 4];
  uint64_t w64[2 * (NT / 32)];
};

// Sum of `v` over the threads of the group whose rank is HIGHER than this thread's
// (exclusive suffix sum), and the group total.
template <int NT>
__device__ __forceinline__ uint32_t group_suffix_exclusive(uint32_t v, uint32_t rank,
                                                           uint32_t* scratch,
                                                           const GroupSync<NT>& gs,
                                                           uint32_t* total) {
  constexpr int NW = NT / 32;
  const uint32_t lane = rank & 31u, warp = rank >> 5;
  uint32_t s = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    uint32_t o = __shfl_down_sync(0xFFFFFFFFu, s, off);
    if (lane + off < 32) s += o;
  }
  if (lane == 0) scratch[warp] = s;
  gs.sync();
  uint32_t above = 0, all = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    uint32_t x = scratch[w];
    all += x;
    if (w > static_cast<int>(warp)) above += x;
  }
  gs.sync();
  if (total) *total = all;
  return above + (s - v);
}

// Exclusive prefix sum over ranks (lower ranks first), and the group total.
template <int NT>
__device__ __forceinline__ uint32_t group_prefix_exclusive(uint32_t v, uint32_t rank,
                                                           uint32_t* scratch,
                                                           const GroupSync<NT>& gs,
                                                           uint32_t* total) {
  constexpr int NW = NT / 32;
  const uint32_t lane = rank & 31u, warp = rank >> 5;
  uint32_t s = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    uint32_t o = __shfl_up_sync(0xFFFFFFFFu, s, off);
    if (lane >= static_cast<uint32_t>(off)) s += o;
  }
  if (lane == 31) scratch[warp] = s;
  gs.sync();
  uint32_t below = 0, all = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    uint32_t x = scratch[w];
    all += x;
    if (w < static_cast<int>(warp)) below += x;
  }
  gs.sync();
  if (total) *total = all;
  return below + (s - v);
}

// Smallest and largest of the n keys key_at(e), over the group.
template <int NT, class KeyAt>
__device__ void group_minmax(KeyAt key_at, uint32_t n, uint32_t rank, GroupScratch<NT>& sc,
                             const GroupSync<NT>& gs, uint64_t* mn, uint64_t* mx) {
  constexpr int NW = NT / 32;
  uint64_t lo = ~0ull, hi = 0ull;
  for (uint32_t e = rank; e < n; e += NT) {
    const uint64_t v = key_at(e);
    lo = v < lo ? v : lo;
    hi = v > hi ? v : hi;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const uint64_t a = __shfl_xor_sync(0xFFFFFFFFu, lo, off);
    const uint64_t b = __shfl_xor_sync(0xFFFFFFFFu, hi, off);
    lo = a < lo ? a : lo;
    hi = b > hi ? b : hi;
  }
  if ((rank & 31u) == 0) {
    sc.w64[2 * (rank >> 5)] = lo;
    sc.w64[2 * (rank >> 5) + 1] = hi;
  }
  gs.sync();
  lo = ~0ull;
  hi = 0ull;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const uint64_t a = sc.w64[2 * w], b = sc.w64[2 * w + 1];
    lo = a < lo ? a : lo;
    hi = b > hi ? b : hi;
  }
  gs.sync();
  *mn = lo;
  *mx = hi;
}

// Radix selection on the n distinct keys key_at(e), e in [0, n), with 0 < k < n.
// Digits of up to 11 bits start at the highest bit where the smallest and largest key differ
// (the bits above it are common to every key), so the first histogram spreads over all bins
// instead of the few bins that keys of similar magnitude share. After each pass the highest bin
// holding the k-th key is known; with `taken` keys in higher bins and `in_bin` keys in it,
// every key >= the bin's lower edge E is among the taken + in_bin largest. The select stops as
// soon as taken + in_bin <= relax_limit and returns E: relax_limit = k gives the exact k-th
// threshold (exactly k keys >= E); a larger limit returns after fewer passes with
// k <= count(keys >= E) <= relax_limit. *count receives count(keys >= E).
// `hist` (kHistBins words) must be zero on entry and is zero again on return.
template <int NT, class KeyAt>
__device__ uint64_t group_select_threshold(KeyAt key_at, uint32_t n, uint32_t k, uint32_t relax_limit,
                                           uint32_t rank, uint32_t* hist, GroupScratch<NT>& sc,
                                           const GroupSync<NT>& gs, uint32_t* count) {
  constexpr int BPT = kHistBins / NT;  // bins owned per thread
  uint64_t mn, mx;
  group_minmax<NT>(key_at, n, rank, sc, gs, &mn, &mx);
  int hb = 63 - __clzll(static_cast<long long>(mn ^ mx));
  uint64_t mask = (hb >= 63) ? 0ull : ~((2ull << hb) - 1ull);
  uint64_t prefix = mx & mask;
  uint32_t need = k, taken = 0;
#pragma unroll 1
  while (true) {
    const int shift = hb >= 10 ? hb - 10 : 0;
    const uint32_t digit_mask = (2u << (hb - shift)) - 1u;
    for (uint32_t e = rank; e < n; e += NT) {
      const uint64_t key = key_at(e);
      if ((key & mask) == prefix)
        atomicAdd(&hist[static_cast<uint32_t>(key >> shift) & digit_mask], 1u);
    }
    gs.sync();
    uint32_t local = 0;
#pragma unroll
    for (int i = 0; i < BPT; ++i) local += hist[rank * BPT + i];
    uint32_t acc = group_suffix_exclusive<NT>(local, rank, sc.w, gs, nullptr);
#pragma unroll
    for (int i = BPT - 1; i >= 0; --i) {
      const uint32_t c = hist[rank * BPT + i];
      if (acc < need && acc + c >= need) {
        sc.w[NT / 32] = rank * BPT + i;
        sc.w[NT / 32 + 1] = acc;
        sc.w[NT / 32 + 2] = c;
      }
      acc += c;
    }
    gs.sync();
    const uint32_t bin = sc.w[NT / 32];
    const uint32_t above = sc.w[NT / 32 + 1];
    const uint32_t in_bin = sc.w[NT / 32 + 2];
#pragma unroll
    for (int i = 0; i < BPT; ++i) hist[rank * BPT + i] = 0u;  // ready for the next pass / call
    gs.sync();
    need -= above;
    taken += above;
    prefix |= static_cast<uint64_t>(bin) << shift;
    mask |= static_cast<uint64_t>(digit_mask) << shift;
    if (taken + in_bin <= relax_limit || shift == 0) {
      *count = taken + in_bin;
      return prefix;
    }
    hb = shift - 1;
  }
}

// Exact k-th threshold: exactly k keys are >= the returned value.
template <int NT, class KeyAt>
__device__ uint64_t group_kth_threshold(KeyAt key_at, uint32_t n, uint32_t k, uint32_t rank,
                                        uint32_t* hist, GroupScratch<NT>& sc,
                                        const GroupSync<NT>& gs) {
  uint32_t cnt;
  return group_select_threshold<NT>(key_at, n, k, k, rank, hist, sc, gs, &cnt);
}

// Stable compaction: writes the keys key_at(e) >= T, e in [0, n), in element order to
// out(pos, key) and returns their number. Warp w owns the elements
// [w * per, (w + 1) * per); a ballot pass counts its keeps, one barrier exchanges the warps'
// totals, and a ballot pass writes. No atomics; loads within a pass are independent.
template <int NT, class KeyAt, class Out>
__device__ uint32_t group_compact_ge(KeyAt key_at, uint32_t n, uint64_t T, Out out, uint32_t rank,
                                     GroupScratch<NT>& sc, const GroupSync<NT>& gs) {
  constexpr int NW = NT / 32;
  const uint32_t lane = rank & 31u, warp = rank >> 5;
  const uint32_t per = (((n + NW - 1) / NW) + 31u) & ~31u;
  const uint32_t beg = min(n, warp * per), end = min(n, beg + per);
  uint32_t mine = 0;
  for (uint32_t e0 = beg; e0 < end; e0 += 128) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t e = e0 + i * 32 + lane;
      mine += __popc(__ballot_sync(0xFFFFFFFFu, e < end && key_at(e) >= T));
    }
  }
  if (lane == 0) sc.w[warp] = mine;
  gs.sync();
  uint32_t base = 0, total = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const uint32_t t = sc.w[w];
    base += (w < static_cast<int>(warp)) ? t : 0u;
    total += t;
  }
  const uint32_t lt = (1u << lane) - 1u;
  for (uint32_t e0 = beg; e0 < end; e0 += 32) {
    const uint32_t e = e0 + lane;
    const uint64_t key = e < end ? key_at(e) : 0ull;
    const bool keep = e < end && key >= T;
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, keep);
    if (keep) out(base + __popc(m & lt), key);
    base += __popc(m);
  }
  gs.sync();
  return total;
}

// Same contract; kept under this name for the selection code that does not need the order.
template <int NT, class KeyAt, class Out>
__device__ __forceinline__ uint32_t group_compact_ge_unordered(KeyAt key_at, uint32_t n, uint64_t T,
                                                               Out out, uint32_t rank,
                                                               GroupScratch<NT>& sc,
                                                               const GroupSync<NT>& gs) {
  return group_compact_ge<NT>(key_at, n, T, out, rank, sc, gs);
}

// Descending compare-exchange of a 64-bit pair held by one thread.
__device__ __forceinline__ void cx_desc(uint64_t& a, uint64_t& b, bool desc) {
  const uint64_t hi = a > b ? a : b, lo = a > b ? b : a;
  a = desc ? hi : lo;
  b = desc ? lo : hi;
}

// One bitonic stage (size, stride known at compile time) over 16 * NT keys held 16 per thread:
// element i = rank * 16 + r lives in v[r]. Strides below 16 stay in registers, strides up to
// 256 exchange with warp shuffles, larger strides through xbuf (16 * NT keys).
template <int NT, int SIZE, int STRIDE>
__device__ __forceinline__ void bitonic_stage(uint64_t (&v)[16], uint32_t rank, uint64_t* xbuf,
                                              const GroupSync<NT>& gs) {
  if constexpr (STRIDE < 16) {
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      if ((r & STRIDE) == 0) {
        const bool desc = (SIZE < 16) ? ((r & SIZE) == 0) : ((rank & (SIZE >> 4)) == 0);
        cx_desc(v[r], v[r | STRIDE], desc);
      }
    }
  } else {
    const bool desc = ((rank & (SIZE >> 4)) == 0);
    const bool lower = ((rank & (STRIDE >> 4)) == 0);
    const bool keep_max = (lower == desc);
    if constexpr (STRIDE <= 256) {
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const uint64_t o = __shfl_xor_sync(0xFFFFFFFFu, v[r], STRIDE >> 4);
        v[r] = keep_max ? (v[r] > o ? v[r] : o) : (v[r] > o ? o : v[r]);
      }
    } else {
#pragma unroll
      for (int r = 0; r < 16; ++r) xbuf[r * NT + rank] = v[r];
      gs.sync();
      const uint32_t partner = rank ^ (STRIDE >> 4);
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const uint64_t o = xbuf[r * NT + partner];
        v[r] = keep_max ? (v[r] > o ? v[r] : o) : (v[r] > o ? o : v[r]);
      }
      gs.sync();
    }
  }
}

template <int NT, int SIZE, int STRIDE>
__device__ __forceinline__ void bitonic_merge_stages(uint64_t (&v)[16], uint32_t rank, uint64_t* xbuf,
                                                     const GroupSync<NT>& gs) {
  bitonic_stage<NT, SIZE, STRIDE>(v, rank, xbuf, gs);
  if constexpr (STRIDE > 1) bitonic_merge_stages<NT, SIZE, STRIDE / 2>(v, rank, xbuf, gs);
}

template <int NT, int SIZE>
__device__ __forceinline__ void bitonic_sizes(uint64_t (&v)[16], uint32_t rank, uint64_t* xbuf,
                                              const GroupSync<NT>& gs) {
  bitonic_merge_stages<NT, SIZE, SIZE / 2>(v, rank, xbuf, gs);
  if constexpr (SIZE < 16 * NT) bitonic_sizes<NT, SIZE * 2>(v, rank, xbuf, gs);
}

// Sorts the 16 * NT keys held 16 per thread into descending order: afterwards thread `rank`
// holds elements rank * 16 .. rank * 16 + 15 of the sorted sequence in v[0..15].
template <int NT>
__device__ void group_bitonic_sort_regs(uint64_t (&v)[16], uint32_t rank, uint64_t* xbuf,
                                        const GroupSync<NT>& gs) {
  static_assert(NT <= 512, "exchange strides");
  bitonic_sizes<NT, 2>(v, rank, xbuf, gs);
}

// Sorts the 16 keys of one thread in descending order (bitonic network, fully unrolled).
__device__ __forceinline__ void sort16_desc(uint64_t (&v)[16]) {
#pragma unroll
  for (int size = 2; size <= 16; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;
          const uint64_t a = v[i], b = v[j];
          const bool swap = desc ? (a < b) : (a > b);
          v[i] = swap ? b : a;
          v[j] = swap ? a : b;
        }
      }
    }
  }
}

// Smallest power of two >= max(k, 16): the size the merge sort works on.
__device__ __forceinline__ uint32_t sort_size(uint32_t k) {
  uint32_t p = 16;
  while (p < k) p <<= 1;
  return p;
}

// Shared-memory index of element x of a sort buffer: one padding slot after every 16 keys,
// so that the 16-key runs of consecutive threads fall into different banks.
__device__ __forceinline__ uint32_t spad(uint32_t x) { return x + (x >> 4); }
__host__ __device__ constexpr int sort_buffer_len(int P) { return P + P / 16; }

// Sorts P keys (P a power of two, 16 <= P <= 16 * NT) in descending order. load(e) supplies
// key e (e < P). Each of the first P/16 threads loads 16 keys with a coalesced stride, sorts
// them in registers and writes them as one run; runs are then merged pairwise, every thread
// emitting 16 consecutive outputs found by a merge-path search. a and b hold
// sort_buffer_len(P) keys each (padded layout, see spad). Returns the buffer holding the result.
template <int NT, class Load>
__device__ uint64_t* group_merge_sort_desc(Load load, uint64_t* a, uint64_t* b, uint32_t P,
                                           uint32_t rank, const GroupSync<NT>& gs) {
  const uint32_t active = P / 16;
  if (rank < active) {
    uint64_t v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = load(i * active + rank);
    sort16_desc(v);
#pragma unroll
    for (int i = 0; i < 16; ++i) a[spad(rank * 16 + i)] = v[i];
  }
  gs.sync();
  uint64_t* src = a;
  uint64_t* dst = b;
  for (uint32_t r = 16; r < P; r <<= 1) {
    if (rank < active) {
      const uint32_t out0 = rank * 16;
      const uint32_t base = out0 & ~(2 * r - 1);  // start of this pair of runs
      const uint32_t o = out0 - base;             // output offset within the pair
      uint32_t lo = o > r ? o - r : 0, hi = o < r ? o : r;
      while (lo < hi) {  // number of run-A keys among the first o outputs
        const uint32_t mid = (lo + hi) >> 1;
        if (src[spad(base + mid)] > src[spad(base + r + o - mid - 1)]) lo = mid + 1;
        else hi = mid;
      }
      uint32_t ia = lo, ib = o - lo;
      uint64_t va = src[spad(base + (ia < r ? ia : r - 1))];
      uint64_t vb = src[spad(base + r + (ib < r ? ib : r - 1))];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const bool take_a = ib >= r || (ia < r && va > vb);
        dst[spad(out0 + i)] = take_a ? va : vb;
        if (take_a) {
          ++ia;
          va = src[spad(base + (ia < r ? ia : r - 1))];
        } else {
          ++ib;
          vb = src[spad(base + r + (ib < r ? ib : r - 1))];
        }
      }
    }
    gs.sync();
    uint64_t* t = src;
    src = dst;
    dst = t;
  }
  return src;
}

}  // namespace dsa

namespace dsa {

// Ranks the m distinct keys tmp[0..m) (m <= KPT * NT) by a bucket sort and leaves the
// min(m, k) largest in tmp[0..min(m, k)) in descending order. NBK buckets of equal width in
// score value span [score(omin), score(omax)] (omin / omax: order-preserving score bits of the
// smallest and largest key); the fp32 map from score to bucket is monotone, so a larger key
// never lands in a lower bucket. A suffix scan gives each bucket's first rank, the buckets'
// keys are placed side by side, and a key's rank is its bucket's first rank plus the number
// of larger keys in its bucket. bk (NBK words) must be zero on entry. Returns false, with bk
// zero again and tmp unchanged, when some bucket holds more than max_bucket keys (heavy ties,
// scores bunched in a sliver of the span): the caller then sorts another way.
template <int NT, int KPT, int NBK>
__device__ bool group_bucket_rank(uint64_t* tmp, uint32_t m, uint32_t k, uint32_t omin, uint32_t omax,
                                  uint32_t max_bucket, uint32_t* bk, uint32_t* flag,
                                  GroupScratch<NT>& sc, const GroupSync<NT>& gs, uint32_t rank) {
  static_assert(NBK % NT == 0, "buckets per thread");
  const float smin = ordered_to_float(omin), smax = ordered_to_float(omax);
  const float span = smax - smin;
  // A zero (or overflowing) span puts every key in bucket 0.
  const float scale = (span > 0.0f && span < 3.0e38f) ? (NBK - 0.5f) / span : 0.0f;
  if (rank == 0) *flag = 0u;
  gs.sync();
  uint64_t v[KPT];
  uint32_t bs[KPT];  // bucket << 16 | slot in the bucket; later the key's rank (~0: no winner)
  uint32_t bs_bucket[KPT];
#pragma unroll
  for (int i = 0; i < KPT; ++i) {
    const uint32_t e = rank + i * NT;
    v[i] = 0ull;
    bs[i] = 0u;
    if (e < m) {
      v[i] = tmp[e];
      const float f = (key_score(v[i]) - smin) * scale;
      const uint32_t b = min(static_cast<uint32_t>(f > 0.0f ? f : 0.0f), static_cast<uint32_t>(NBK - 1));
      const uint32_t slot = atomicAdd(&bk[b], 1u);
      bs[i] = (b << 16) | slot;
      if (slot >= max_bucket) *flag = 1u;
    }
    bs_bucket[i] = bs[i] >> 16;
  }
  gs.sync();
  if (*flag) {
    for (uint32_t b = rank; b < static_cast<uint32_t>(NBK); b += NT) bk[b] = 0u;
    gs.sync();
    return false;
  }
  // First rank of each bucket: keys in higher buckets (exclusive suffix sum), in place.
  constexpr int BPT = NBK / NT;
  uint32_t cnt[BPT];
  uint32_t local = 0;
#pragma unroll
  for (int i = 0; i < BPT; ++i) {
    cnt[i] = bk[rank * BPT + i];
    local += cnt[i];
  }
  uint32_t acc = group_suffix_exclusive<NT>(local, rank, sc.w, gs, nullptr);
#pragma unroll
  for (int i = BPT - 1; i >= 0; --i) {
    bk[rank * BPT + i] = acc;
    acc += cnt[i];
  }
  gs.sync();
  // Bucket members side by side (every key is in registers by now); buckets that start at
  // rank k or later hold no winner and are left out.
#pragma unroll
  for (int i = 0; i < KPT; ++i) {
    const uint32_t e = rank + i * NT;
    if (e < m) {
      const uint32_t s0 = bk[bs[i] >> 16];
      if (s0 < k) tmp[s0 + (bs[i] & 0xFFFFu)] = v[i];
    }
  }
  gs.sync();
#pragma unroll
  for (int i = 0; i < KPT; ++i) {
    const uint32_t e = rank + i * NT;
    bs[i] = 0xFFFFFFFFu;
    if (e < m) {
      const uint32_t b = bs_bucket[i];
      const uint32_t s0 = bk[b];
      if (s0 < k) {
        const uint32_t nb = (b == 0 ? m : bk[b - 1]) - s0;
        uint32_t r = s0;
        for (uint32_t j = 0; j < nb; ++j) r += tmp[s0 + j] > v[i] ? 1u : 0u;
        bs[i] = r;
      }
    }
  }
  gs.sync();
#pragma unroll
  for (int i = 0; i < KPT; ++i) {
    const uint32_t e = rank + i * NT;
    if (e < m && bs[i] < k) tmp[bs[i]] = v[i];
  }
  gs.sync();
  return true;
}

}  // namespace dsa
