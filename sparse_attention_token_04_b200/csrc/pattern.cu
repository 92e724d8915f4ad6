// Layer-pattern diagnostics from the cross-layer top-k overlap matrix (host code).
//
// "IndexShare deep-dive report" §1.2 and §3.1: the overlap heat map of a DSA model is organised
// in blocks of layers whose selections agree closely, with sharp drops at a few transition
// layers; uniform F/S interleaving ignores that structure. §5.2 of the same report warns that a
// similarity proxy does not predict model quality, so nothing here chooses a pattern for
// serving: these functions describe an overlap matrix.
//
//   dsa_overlap_blocks       splits the layers into maximal runs whose adjacent-layer overlap
//                            stays at or above a threshold (a new block starts at a layer whose
//                            overlap with the layer before it drops below the threshold).
//   dsa_pattern_from_overlap the F/S pattern with a given number of Full layers (layer 0 always
//                            Full) that keeps the most overlap: every layer l is served by the
//                            last Full layer at or before it, f(l), and the pattern maximises
//                            sum_l O[l][f(l)] (O[l][l] = 1 for a Full layer). Exact, by dynamic
//                            programming over the position of each Full layer.
#include <cstring>
#include <vector>

#include "internal.h"

extern "C" {

DSA_API int32_t dsa_overlap_blocks(const double* overlap, int32_t n_layers, double threshold,
                                   int32_t* block_of_layer) {
  if (!overlap || !block_of_layer || n_layers < 1 || n_layers > DSA_MAX_LAYERS) return -1;
  int32_t block = 0;
  block_of_layer[0] = 0;
  for (int l = 1; l < n_layers; ++l) {
    const double adj = overlap[static_cast<size_t>(l) * n_layers + (l - 1)];
    if (!(adj >= threshold)) ++block;
    block_of_layer[l] = block;
  }
  return block + 1;
}

DSA_API dsa_status dsa_pattern_from_overlap(const double* overlap, int32_t n_layers, int32_t n_full,
                                            char* pattern_out, double* retained_out) {
  if (!overlap || !pattern_out || n_layers < 1 || n_layers > DSA_MAX_LAYERS || n_full < 1 ||
      n_full > n_layers)
    return DSA_ERR_INVALID;
  const int N = n_layers;
  auto O = [&](int i, int j) { return overlap[static_cast<size_t>(i) * N + j]; };
  // seg[p][e]: overlap kept by layers p..e-1 when all are served by a Full layer at p.
  std::vector<double> seg(static_cast<size_t>(N + 1) * (N + 1), 0.0);
  for (int p = 0; p < N; ++p) {
    double s = 0.0;
    for (int e = p + 1; e <= N; ++e) {
      s += (e - 1 == p) ? 1.0 : O(e - 1, p);
      seg[static_cast<size_t>(p) * (N + 1) + e] = s;
    }
  }
  const double NEG = -1e300;
  // best[c][e]: most overlap kept by layers 0..e-1 with c Full layers, the next Full layer (or
  // the end) at e; from[c][e]: the position of the c-th Full layer in that optimum.
  std::vector<double> best(static_cast<size_t>(n_full + 1) * (N + 1), NEG);
  std::vector<int> from(static_cast<size_t>(n_full + 1) * (N + 1), -1);
  auto B = [&](int c, int e) -> double& { return best[static_cast<size_t>(c) * (N + 1) + e]; };
  auto F = [&](int c, int e) -> int& { return from[static_cast<size_t>(c) * (N + 1) + e]; };
  for (int e = 1; e <= N; ++e) {
    B(1, e) = seg[e];  // the first Full layer is layer 0
    F(1, e) = 0;
  }
  for (int c = 2; c <= n_full; ++c) {
    for (int e = c; e <= N; ++e) {
      for (int p = c - 1; p < e; ++p) {  // the c-th Full layer at p, the (c-1)-th segment ends at p
        const double prev = B(c - 1, p);
        if (prev == NEG) continue;
        const double v = prev + seg[static_cast<size_t>(p) * (N + 1) + e];
        if (v > B(c, e)) {
          B(c, e) = v;
          F(c, e) = p;
        }
      }
    }
  }
  if (B(n_full, N) == NEG) return DSA_ERR_INVALID;
  std::memset(pattern_out, 'S', static_cast<size_t>(N));
  pattern_out[N] = '\0';
  int e = N;
  for (int c = n_full; c >= 1; --c) {
    const int p = F(c, e);
    pattern_out[p] = 'F';
    e = p;
  }
  if (retained_out) *retained_out = B(n_full, N) / N;
  return DSA_OK;
}

}  // extern "C"
