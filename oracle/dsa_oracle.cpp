// Oracle for the DSA lightning indexer, its top-k selection, IndexCache layer reuse and the
// cross-layer top-k overlap, in plain single-threaded C++ with fp64 arithmetic.
//
// TEST INFRASTRUCTURE ONLY. Nothing on the product path (the CUDA library and its Python
// binding) includes, links or calls this file; only the tests, the smoke check and the
// benchmark's CPU-baseline leg do. It shares no code, table or helper with the CUDA path, and
// none with the numpy oracle next to it either: the two are written independently so that each
// checks the other.
//
// Pages followed (by title and section):
//   * "IndexShare deep-dive report" (深度解读报告), §1.1: the lightning indexer is a multi-head,
//     ReLU-gated dot product over FP8 inputs that scores the whole prefix and keeps the top-k
//     keys (k = 2048 in the abstract).
//   * same report, §2.1: Full layers run the indexer and overwrite the cached indices; a Shared
//     layer reads T_f(l) with f(l) = max{j < l : c_j = F}; the first layer is always F.
//   * same report, §1.2: the overlap of layers i and j is |T(i) ∩ T(j)| / k.
//   * "ADIndex以分组蒸馏重构长上下文稀疏注意力索引", section 索引器为何成为长上下文瓶颈: every
//     query scans its whole causal prefix (keys s <= t).
// The indexer formula, which the pages describe only in words, is read as
//     I[t,s] = sum_j w[t,j] * max(0, q_scale[t] * k_scale[s] * D_j),
//     D_j = sum_c e4m3(q8[t][j][c]) * e4m3(k8[s][c]),
// heads summed in ascending j, ties in the top-k going to the lower key index, rows written by
// (score descending, index ascending) and padded with index -1 / score -inf.
//
// Every step is a plain loop. D_j is exact in fp64: E4M3 values are multiples of 2^-9 below
// 2^9, so each product is a multiple of 2^-18 below 2^18 and a sum of at most d = 128 of them
// stays below 2^25 -- 43 significant bits, within the 53 of a double. Build with
// -ffp-contract=off so that no multiply-add is fused.
//
// n_threads > 1 runs the same per-row function on that many std::threads over rows (row r on
// thread r % n_threads): the all-cores CPU baseline. n_threads = 1 is the plain single-threaded
// oracle.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <limits>
#include <thread>
#include <vector>

namespace {

// OCP 8-bit floating point, E4M3 variant: sign, 4 exponent bits (bias 7), 3 mantissa bits;
// exponent field 0 encodes subnormals m/8 * 2^-6; S.1111.111 is NaN; no infinities.
double e4m3_value(unsigned code) {
  const double sign = (code & 0x80u) ? -1.0 : 1.0;
  const unsigned e = (code >> 3) & 0xFu;
  const unsigned m = code & 0x7u;
  if (e == 0xFu && m == 0x7u) return std::numeric_limits<double>::quiet_NaN();
  if (e == 0u) return sign * (static_cast<double>(m) / 8.0) * std::ldexp(1.0, -6);
  return sign * (1.0 + static_cast<double>(m) / 8.0) * std::ldexp(1.0, static_cast<int>(e) - 7);
}

struct E4M3 {
  double v[256];
  E4M3() {
    for (unsigned c = 0; c < 256; ++c) v[c] = e4m3_value(c);
  }
};
const E4M3& table() {
  static const E4M3 t;
  return t;
}

bool is_nan_code(uint8_t c) { return (c & 0x7Fu) == 0x7Fu; }

// Scores of one query against n keys given by a key accessor. q8: [H][d] codes of the query.
// key(s) returns the pointer to key s's d codes, kscale(s) its scale.
template <class KeyAt, class ScaleAt>
bool score_row(const uint8_t* q8, double q_scale, const float* w, int H, int d, int n, KeyAt key,
               ScaleAt kscale, std::vector<double>& scores) {
  const E4M3& T = table();
  std::vector<double> qv(static_cast<size_t>(H) * d);
  for (int i = 0; i < H * d; ++i) {
    if (is_nan_code(q8[i])) return false;
    qv[i] = T.v[q8[i]];
  }
  std::vector<double> kv(d);
  scores.assign(n, 0.0);
  for (int s = 0; s < n; ++s) {
    const uint8_t* k8 = key(s);
    for (int c = 0; c < d; ++c) {
      if (is_nan_code(k8[c])) return false;
      kv[c] = T.v[k8[c]];
    }
    const double qk = q_scale * static_cast<double>(kscale(s));
    double total = 0.0;
    for (int j = 0; j < H; ++j) {
      double dot = 0.0;
      for (int c = 0; c < d; ++c) dot += qv[static_cast<size_t>(j) * d + c] * kv[c];
      const double x = qk * dot;
      const double relu = x > 0.0 ? x : 0.0;
      total = total + static_cast<double>(w[j]) * relu;
    }
    scores[s] = total;
  }
  return true;
}

// The k largest scores, ties to the lower index, listed by (score desc, index asc); padding
// with -1 / -inf when fewer than k keys exist. A full sort, as plain as it gets.
void select_topk(const std::vector<double>& scores, int topk, int64_t* idx, double* val) {
  const int n = static_cast<int>(scores.size());
  std::vector<int> order(n);
  for (int s = 0; s < n; ++s) order[s] = s;
  std::sort(order.begin(), order.end(), [&](int a, int b) {
    if (scores[a] != scores[b]) return scores[a] > scores[b];
    return a < b;
  });
  const int take = std::min(topk, n);
  for (int i = 0; i < topk; ++i) {
    if (i < take) {
      idx[i] = order[i];
      val[i] = scores[order[i]];
    } else {
      idx[i] = -1;
      val[i] = -std::numeric_limits<double>::infinity();
    }
  }
}

template <class Fn>
bool for_rows(int n_rows, int n_threads, Fn fn) {
  if (n_threads <= 1 || n_rows <= 1) {
    bool ok = true;
    for (int r = 0; r < n_rows; ++r) ok = fn(r) && ok;
    return ok;
  }
  const int nt = std::min(n_threads, n_rows);
  std::vector<char> ok(nt, 1);
  std::vector<std::thread> pool;
  for (int p = 0; p < nt; ++p)
    pool.emplace_back([&, p] {
      for (int r = p; r < n_rows; r += nt) ok[p] = fn(r) && ok[p];
    });
  for (auto& th : pool) th.join();
  return std::all_of(ok.begin(), ok.end(), [](char c) { return c != 0; });
}

}  // namespace

extern "C" {

// The decoded value of every E4M3 code (NaN for 0x7F / 0xFF).
void oracle_e4m3_table(double* out) {
  for (int c = 0; c < 256; ++c) out[c] = table().v[c];
}

// Prefill rows. q [*][H][d] holds the chunk's queries; row r of the request is local query
// rows[r], at position t = q_pos0 + rows[r], scoring keys 0..t of k [Lk][d].
// out_idx / out_val [n_rows][topk]; out_scores [n_rows][scores_stride] (nullable) receives the
// scores of keys 0..t. Returns 0, or -1 on a NaN code or a row beyond the keys.
int oracle_prefill_rows(const uint8_t* q, const float* q_scale, const float* w, const uint8_t* k,
                        const float* k_scale, int Lk, int H, int d, int q_pos0, const int32_t* rows,
                        int n_rows, int topk, int64_t* out_idx, double* out_val, double* out_scores,
                        int64_t scores_stride, int n_threads) {
  const bool ok = for_rows(n_rows, n_threads, [&](int r) {
    const int i = rows[r];
    const int t = q_pos0 + i;
    if (i < 0 || t < 0 || t >= Lk) return false;
    std::vector<double> scores;
    const bool good = score_row(
        q + static_cast<size_t>(i) * H * d, static_cast<double>(q_scale[i]),
        w + static_cast<size_t>(i) * H, H, d, t + 1,
        [&](int s) { return k + static_cast<size_t>(s) * d; }, [&](int s) { return k_scale[s]; },
        scores);
    if (!good) return false;
    select_topk(scores, topk, out_idx + static_cast<size_t>(r) * topk,
                out_val + static_cast<size_t>(r) * topk);
    if (out_scores)
      std::copy(scores.begin(), scores.end(), out_scores + static_cast<size_t>(r) * scores_stride);
    return true;
  });
  return ok ? 0 : -1;
}

// Prefill rows given as separate queries: row r is the query q_rows[r] ([H][d] codes, scale
// q_scale[r], weights w[r]) at position positions[r], scoring keys 0..positions[r] of k.
// Outputs as oracle_prefill_rows.
int oracle_prefill_positions(const uint8_t* q_rows, const float* q_scale, const float* w,
                             const uint8_t* k, const float* k_scale, int Lk, int H, int d,
                             const int32_t* positions, int n_rows, int topk, int64_t* out_idx,
                             double* out_val, double* out_scores, int64_t scores_stride,
                             int n_threads) {
  const bool ok = for_rows(n_rows, n_threads, [&](int r) {
    const int t = positions[r];
    if (t < 0 || t >= Lk) return false;
    std::vector<double> scores;
    const bool good = score_row(
        q_rows + static_cast<size_t>(r) * H * d, static_cast<double>(q_scale[r]),
        w + static_cast<size_t>(r) * H, H, d, t + 1,
        [&](int s) { return k + static_cast<size_t>(s) * d; }, [&](int s) { return k_scale[s]; },
        scores);
    if (!good) return false;
    select_topk(scores, topk, out_idx + static_cast<size_t>(r) * topk,
                out_val + static_cast<size_t>(r) * topk);
    if (out_scores)
      std::copy(scores.begin(), scores.end(), out_scores + static_cast<size_t>(r) * scores_stride);
    return true;
  });
  return ok ? 0 : -1;
}

// Decode rows: request b has one query at position seq_lens[b] - 1 and scores its
// seq_lens[b] cached keys; logical key s lives in block block_table[b][s / block_size], slot
// s % block_size. Output indices are logical positions. Returns -1 on a NaN code or a block
// table entry outside [0, n_blocks).
int oracle_decode_rows(const uint8_t* q, const float* q_scale, const float* w,
                       const uint8_t* k_cache, const float* k_scale_cache, int n_blocks,
                       int block_size, const int32_t* block_table, int max_blocks,
                       const int32_t* seq_lens, int H, int d, const int32_t* reqs, int n_reqs,
                       int topk, int64_t* out_idx, double* out_val, double* out_scores,
                       int64_t scores_stride, int n_threads) {
  const bool ok = for_rows(n_reqs, n_threads, [&](int r) {
    const int b = reqs[r];
    const int n = seq_lens[b];
    const int32_t* row = block_table + static_cast<size_t>(b) * max_blocks;
    if (n < 1 || n > max_blocks * block_size) return false;
    for (int i = 0; i < (n + block_size - 1) / block_size; ++i)
      if (row[i] < 0 || row[i] >= n_blocks) return false;
    auto slot = [&](int s) {
      return static_cast<size_t>(row[s / block_size]) * block_size + static_cast<size_t>(s % block_size);
    };
    std::vector<double> scores;
    const bool good = score_row(
        q + static_cast<size_t>(b) * H * d, static_cast<double>(q_scale[b]),
        w + static_cast<size_t>(b) * H, H, d, n,
        [&](int s) { return k_cache + slot(s) * d; }, [&](int s) { return k_scale_cache[slot(s)]; },
        scores);
    if (!good) return false;
    select_topk(scores, topk, out_idx + static_cast<size_t>(r) * topk,
                out_val + static_cast<size_t>(r) * topk);
    if (out_scores)
      std::copy(scores.begin(), scores.end(), out_scores + static_cast<size_t>(r) * scores_stride);
    return true;
  });
  return ok ? 0 : -1;
}

// IndexCache sources: src[l] = l for a Full layer, the most recent Full layer before l for a
// Shared one. Returns -1 for a character other than F / S or a leading S.
int oracle_indexcache_sources(const char* pattern, int n_layers, int32_t* src) {
  int last_full = -1;
  for (int l = 0; l < n_layers; ++l) {
    if (pattern[l] == 'F') {
      last_full = l;
    } else if (pattern[l] != 'S' || last_full < 0) {
      return -1;
    }
    src[l] = last_full;
  }
  return n_layers > 0 ? 0 : -1;
}

// Overlap counts: C[i][j] = sum over rows of |T_i(row) ∩ T_j(row)| with -1 entries excluded,
// each row's two index sets sorted and merged; V = the valid (non-negative) entries of layer 0.
int oracle_topk_overlap(const int32_t* const* layers, int n_layers, int rows, int topk,
                        uint64_t* counts, uint64_t* valid) {
  for (int i = 0; i < n_layers * n_layers; ++i) counts[i] = 0;
  *valid = 0;
  std::vector<std::vector<int32_t>> sets(n_layers);
  for (int t = 0; t < rows; ++t) {
    for (int i = 0; i < n_layers; ++i) {
      sets[i].clear();
      const int32_t* r = layers[i] + static_cast<size_t>(t) * topk;
      uint64_t n_valid = 0;
      for (int e = 0; e < topk; ++e)
        if (r[e] >= 0) {
          sets[i].push_back(r[e]);
          ++n_valid;
        }
      std::sort(sets[i].begin(), sets[i].end());
      sets[i].erase(std::unique(sets[i].begin(), sets[i].end()), sets[i].end());
      if (i == 0) *valid += n_valid;
    }
    for (int i = 0; i < n_layers; ++i) {
      for (int j = i; j < n_layers; ++j) {
        uint64_t c = 0;
        size_t a = 0, b = 0;
        while (a < sets[i].size() && b < sets[j].size()) {
          if (sets[i][a] < sets[j][b]) {
            ++a;
          } else if (sets[j][b] < sets[i][a]) {
            ++b;
          } else {
            ++c;
            ++a;
            ++b;
          }
        }
        counts[static_cast<size_t>(i) * n_layers + j] += c;
        if (j != i) counts[static_cast<size_t>(j) * n_layers + i] += c;
      }
    }
  }
  return 0;
}

}  // extern "C"
