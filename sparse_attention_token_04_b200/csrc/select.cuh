// Exact top-k selection primitives on 64-bit (score, index) keys for a group of NT threads
// that synchronise on one named barrier. Keys are distinct (the low word encodes the index),
// so "the k largest keys" is one well-defined set: the k best scores with ties going to the
// lower index.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kHistBins = 2048;  // 11-bit radix digits

// Digits of the 64-bit key, most significant first: the score word in 11/11/10 bits, then
// the index word in 11/11/10 bits.
__device__ __forceinline__ int radix_shift(int pass) {
  constexpr int s[6] = {53, 42, 32, 21, 10, 0};
  return s[pass];
}
__device__ __forceinline__ int radix_bits(int pass) {
  constexpr int b[6] = {11, 11, 10, 11, 11, 10};
  return b[pass];
}

template <int NT>
struct GroupSync {
  uint32_t bar_id;
  __device__ __forceinline__ void sync() const { named_bar(bar_id, NT); }
};

// Sum of `v` over the threads of the group whose rank is HIGHER than this thread's
// (exclusive suffix sum), and the group total. `scratch` holds NT/32 words.
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

// Returns T such that exactly k of the n keys produced by key_at(e), e in [0, n), satisfy
// key >= T. Requires 0 < k < n and distinct keys. `hist` holds kHistBins words and
// `scratch` at least NT/32 + 2 words, both private to the group.
template <int NT, class KeyAt>
__device__ uint64_t group_kth_threshold(KeyAt key_at, uint32_t n, uint32_t k, uint32_t rank,
                                        uint32_t* hist, uint32_t* scratch,
                                        const GroupSync<NT>& gs) {
  constexpr int BPT = kHistBins / NT;  // bins owned per thread
  uint64_t prefix = 0, mask = 0;
  uint32_t need = k;
#pragma unroll 1
  for (int pass = 0; pass < 6; ++pass) {
    const int shift = radix_shift(pass);
    const uint32_t digit_mask = (1u << radix_bits(pass)) - 1u;
    for (uint32_t b = rank; b < kHistBins; b += NT) hist[b] = 0;
    gs.sync();
    for (uint32_t e = rank; e < n; e += NT) {
      const uint64_t key = key_at(e);
      if ((key & mask) == prefix)
        atomicAdd(&hist[static_cast<uint32_t>(key >> shift) & digit_mask], 1u);
    }
    gs.sync();
    uint32_t local = 0;
#pragma unroll
    for (int i = 0; i < BPT; ++i) local += hist[rank * BPT + i];
    uint32_t acc = group_suffix_exclusive<NT>(local, rank, scratch, gs, nullptr);
#pragma unroll
    for (int i = BPT - 1; i >= 0; --i) {
      const uint32_t c = hist[rank * BPT + i];
      if (acc < need && acc + c >= need) {
        scratch[NT / 32] = rank * BPT + i;
        scratch[NT / 32 + 1] = acc;
      }
      acc += c;
    }
    gs.sync();
    const uint32_t bin = scratch[NT / 32];
    const uint32_t above = scratch[NT / 32 + 1];
    const uint32_t in_bin = hist[bin];
    gs.sync();
    need -= above;
    prefix |= static_cast<uint64_t>(bin) << shift;
    mask |= static_cast<uint64_t>(digit_mask) << shift;
    if (in_bin == need) break;  // every key of this bin is selected
  }
  return prefix;
}

// Stable compaction: writes, in order, the keys key_at(e) >= T to out(pos, key) and returns
// their number. Each thread walks one contiguous segment.
template <int NT, class KeyAt, class Out>
__device__ uint32_t group_compact_ge(KeyAt key_at, uint32_t n, uint64_t T, Out out, uint32_t rank,
                                     uint32_t* scratch, const GroupSync<NT>& gs) {
  const uint32_t seg = (n + NT - 1) / NT;
  const uint32_t beg = min(n, rank * seg), end = min(n, beg + seg);
  uint32_t c = 0;
  for (uint32_t e = beg; e < end; ++e) c += (key_at(e) >= T) ? 1u : 0u;
  uint32_t total;
  uint32_t pos = group_prefix_exclusive<NT>(c, rank, scratch, gs, &total);
  for (uint32_t e = beg; e < end; ++e) {
    const uint64_t key = key_at(e);
    if (key >= T) out(pos++, key);
  }
  return total;
}

// Sorts s[0..P) (P a power of two) in descending key order.
template <int NT>
__device__ void group_bitonic_sort_desc(uint64_t* s, uint32_t P, uint32_t rank,
                                        const GroupSync<NT>& gs) {
  for (uint32_t size = 2; size <= P; size <<= 1) {
    for (uint32_t stride = size >> 1; stride > 0; stride >>= 1) {
      for (uint32_t e = rank; e < (P >> 1); e += NT) {
        const uint32_t i = 2 * e - (e & (stride - 1));
        const uint32_t j = i + stride;
        const bool desc = (i & size) == 0;
        const uint64_t a = s[i], b = s[j];
        if ((a < b) == desc) {
          s[i] = b;
          s[j] = a;
        }
      }
      gs.sync();
    }
  }
}

}  // namespace dsa
