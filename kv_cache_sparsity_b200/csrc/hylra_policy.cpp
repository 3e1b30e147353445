// hylra_policy.cpp - offline policy of HyLRA on the host (see include/hylra.h).
//
// "HyLRA: Hybrid Layer Reuse Attention for Efficient Long-Context Inference"
// (gist.science technical summary of arXiv 2602.00777), §2.2 "Offline Policy
// Optimization via Dynamic Programming":
//   * the overlap matrix M of top-k indices between a source and a target
//     layer (lower-triangular), from a profiling run with every layer full;
//   * the policy: a path over states (i, j) - layer j reuses the indices of
//     reset layer i - with reset jumps (j, j) and vertical moves (i, j) ->
//     (i, j+1) allowed while the similarity exceeds theta; fewest full
//     attention layers first, then the largest cumulative similarity.
#include <algorithm>
#include <cmath>
#include <vector>

#include "hylra.h"

namespace {

// Sorted distinct valid (>= 0) entries of one k-long index list.
std::vector<int32_t> index_set(const int32_t* list, int k) {
  std::vector<int32_t> v;
  v.reserve(k);
  for (int i = 0; i < k; ++i)
    if (list[i] >= 0) v.push_back(list[i]);
  std::sort(v.begin(), v.end());
  v.erase(std::unique(v.begin(), v.end()), v.end());
  return v;
}

long long intersection_size(const std::vector<int32_t>& a, const std::vector<int32_t>& b) {
  long long n = 0;
  size_t i = 0, j = 0;
  while (i < a.size() && j < b.size()) {
    if (a[i] < b[j]) {
      ++i;
    } else if (b[j] < a[i]) {
      ++j;
    } else {
      ++n;
      ++i;
      ++j;
    }
  }
  return n;
}

// Best way found so far to reach "layer i is a reset": resets, cumulative
// similarity and the policy of layers 0..i.
struct Path {
  bool valid = false;
  int resets = 0;
  double sim = 0.0;
  std::vector<uint8_t> policy;
};

// Preference between two complete-or-equal-length paths: fewer resets, then
// more similarity, then the lexicographically smaller policy (reuse < reset).
bool preferred(int r1, double s1, const std::vector<uint8_t>& p1, const Path& b) {
  if (!b.valid) return true;
  if (r1 != b.resets) return r1 < b.resets;
  if (s1 != b.sim) return s1 > b.sim;
  return p1 < b.policy;
}

}  // namespace

extern "C" {

int hylra_overlap_counts(int32_t num_layers, int32_t num_sets, int32_t k, const int32_t* topk,
                         int64_t* inter, int64_t* total) {
  if (num_layers < 1 || num_sets < 0 || k < 1 || !inter || !total || (num_sets > 0 && !topk))
    return HYLRA_ERR_INVALID;
  const int L = num_layers, S = num_sets;
  std::vector<std::vector<int32_t>> sets((size_t)L * S);
  for (int l = 0; l < L; ++l)
    for (int u = 0; u < S; ++u)
      sets[(size_t)l * S + u] = index_set(topk + ((size_t)l * S + u) * k, k);
  for (int t = 0; t < L; ++t) {
    long long tot = 0;
    for (int u = 0; u < S; ++u) tot += (long long)sets[(size_t)t * S + u].size();
    total[t] = tot;
    for (int s = 0; s < L; ++s) {
      long long n = 0;
      if (s <= t)
        for (int u = 0; u < S; ++u)
          n += intersection_size(sets[(size_t)s * S + u], sets[(size_t)t * S + u]);
      inter[(size_t)t * L + s] = n;
    }
  }
  return HYLRA_OK;
}

int hylra_similarity_from_counts(int32_t num_layers, const int64_t* inter, const int64_t* total,
                                 double* M) {
  if (num_layers < 1 || !inter || !total || !M) return HYLRA_ERR_INVALID;
  const int L = num_layers;
  for (int t = 0; t < L; ++t) {
    if (total[t] < 0) return HYLRA_ERR_INVALID;
    for (int s = 0; s < L; ++s) {
      const int64_t n = inter[(size_t)t * L + s];
      if (n < 0 || n > total[t] || (s > t && n != 0)) return HYLRA_ERR_INVALID;
    }
  }
  for (int t = 0; t < L; ++t)
    for (int s = 0; s < L; ++s)
      M[(size_t)t * L + s] = (s <= t && total[t] > 0)
                                 ? (double)inter[(size_t)t * L + s] / (double)total[t]
                                 : 0.0;
  return HYLRA_OK;
}

int hylra_similarity(int32_t num_layers, int32_t num_sets, int32_t k, const int32_t* topk,
                     double* M) {
  if (num_layers < 1 || num_sets < 0 || k < 1 || !M || (num_sets > 0 && !topk))
    return HYLRA_ERR_INVALID;
  std::vector<int64_t> inter((size_t)num_layers * num_layers), total(num_layers);
  int rc = hylra_overlap_counts(num_layers, num_sets, k, topk, inter.data(), total.data());
  if (rc) return rc;
  return hylra_similarity_from_counts(num_layers, inter.data(), total.data(), M);
}

int hylra_token_topk(int32_t num_lists, int32_t n, const float* scores, const int32_t* lengths,
                     int32_t k, int32_t* topk) {
  if (num_lists < 0 || n < 0 || k < 1 || !topk || (num_lists > 0 && n > 0 && !scores))
    return HYLRA_ERR_INVALID;
  for (int u = 0; u < num_lists; ++u) {
    const int len = lengths ? lengths[u] : n;
    if (len < 0 || len > n) return HYLRA_ERR_INVALID;
    for (int t = 0; t < len; ++t) {
      const float v = scores[(size_t)u * n + t];
      if (!std::isfinite(v) || v < 0.f) return HYLRA_ERR_INVALID;
    }
  }
  std::vector<int32_t> order;
  for (int u = 0; u < num_lists; ++u) {
    const int len = lengths ? lengths[u] : n;
    const float* sc = scores + (size_t)u * n;
    const int kp = std::min(k, len);
    order.resize(len);
    for (int t = 0; t < len; ++t) order[t] = t;
    // score descending, lower index first among equal scores
    std::partial_sort(order.begin(), order.begin() + kp, order.end(), [sc](int32_t a, int32_t b) {
      return sc[a] != sc[b] ? sc[a] > sc[b] : a < b;
    });
    int32_t* dst = topk + (size_t)u * k;
    for (int e = 0; e < k; ++e) dst[e] = e < kp ? order[e] : -1;
  }
  return HYLRA_OK;
}

int hylra_dp_policy(int32_t num_layers, const double* M, double theta, uint8_t* policy,
                    int32_t* num_resets, double* cum_similarity) {
  if (num_layers < 1 || !M || !policy || std::isnan(theta)) return HYLRA_ERR_INVALID;
  const int L = num_layers;
  // reset[i]: best path whose layer i is a reset.  Every candidate for
  // reset[j+1] comes from a state (i, j) with i <= j, so visiting i in
  // increasing order settles reset[i] before it is extended.
  std::vector<Path> reset(L);
  reset[0].valid = true;
  reset[0].resets = 1;
  reset[0].sim = 0.0;
  reset[0].policy.assign(1, 1);
  Path best;
  for (int i = 0; i < L; ++i) {
    const Path& from = reset[i];
    if (!from.valid) continue;
    std::vector<uint8_t> pol = from.policy;  // policy of layers 0..j
    double sim = from.sim;
    for (int j = i;; ++j) {
      // at state (i, j)
      if (j == L - 1) {
        if (preferred(from.resets, sim, pol, best)) {
          best.valid = true;
          best.resets = from.resets;
          best.sim = sim;
          best.policy = pol;
        }
        break;
      }
      // reset jump to (j+1, j+1)
      pol.push_back(1);
      if (preferred(from.resets + 1, sim, pol, reset[j + 1])) {
        Path& to = reset[j + 1];
        to.valid = true;
        to.resets = from.resets + 1;
        to.sim = sim;
        to.policy = pol;
      }
      pol.pop_back();
      // vertical move to (i, j+1), only while the similarity exceeds theta
      const double mv = M[(size_t)(j + 1) * L + i];
      if (!(mv > theta)) break;
      sim += mv;
      pol.push_back(0);
    }
  }
  for (int l = 0; l < L; ++l) policy[l] = best.policy[l];
  if (num_resets) *num_resets = best.resets;
  if (cum_similarity) *cum_similarity = best.sim;
  return HYLRA_OK;
}

int hylra_static_policy(int32_t num_layers, int32_t period, uint8_t* policy,
                        int32_t* num_resets) {
  if (num_layers < 1 || period < 1 || !policy) return HYLRA_ERR_INVALID;
  int32_t resets = 0;
  for (int32_t l = 0; l < num_layers; ++l) {
    policy[l] = (l % period == 0) ? 1 : 0;
    resets += policy[l];
  }
  if (num_resets) *num_resets = resets;
  return HYLRA_OK;
}

}  // extern "C"
