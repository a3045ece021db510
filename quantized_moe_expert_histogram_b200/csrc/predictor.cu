// Next-layer expert predictor for the offload mode (EdgeMoE, expert
// preloading: a statistical profile keyed by the experts activated at the
// two preceding MoE layers gives the probability of each expert at the next
// layer, and the experts are preloaded in order of that probability;
// ExactMoE/D2MoE: load the next experts while computing the current ones).
//
// Learned online from the routed ids of earlier steps, per choice position
// j of a token (the path a token's j-th assignment takes through the
// layers):
//   counts1[l][a][b]     assignments at expert a at layer l-1 that went to
//                        expert b at layer l
//   counts2[l][c][a][b]  the same, keyed by the pair (expert c at layer l-2,
//                        expert a at layer l-1)   (kept for E <= 64)
// A prediction for layer l scores each expert b by the sum over the
// assignments of P(b | key), using the pair key when that pair has been seen
// at least kPairSupport times and the one-layer key otherwise (the expected
// number of assignments routed to b), and returns the best-scoring experts
// whose score reaches min_score (ties to the lower id).  Host-only
// bookkeeping: the caller passes host arrays (the routed ids it already
// copied for moe_slot_stage).
#include <algorithm>
#include <new>
#include <vector>

#include "common.cuh"

using namespace moeq;

namespace {
constexpr int kPairMaxE = 64;    // pair tables: layers * E^3 counters
constexpr uint64_t kPairSupport = 2;
}  // namespace

struct moe_route_predictor {
  int layers = 0, E = 0;
  std::vector<uint32_t> counts1;   // [layers][E][E]
  std::vector<uint64_t> sum1;      // [layers][E]
  std::vector<uint32_t> counts2;   // [layers][E][E][E] (E <= kPairMaxE), else empty
  std::vector<uint64_t> sum2;      // [layers][E][E]
};

extern "C" {

moe_status_t moe_predictor_create(int layers, int E, moe_route_predictor** out) {
  if (!out || layers <= 0 || E <= 0 || E > 256) {
    set_error("moe_predictor_create: bad arguments");
    return MOE_ERR_INVALID_ARG;
  }
  *out = nullptr;
  moe_route_predictor* p = new (std::nothrow) moe_route_predictor();
  if (!p) {
    set_error("moe_predictor_create: out of host memory");
    return MOE_ERR_OOM;
  }
  p->layers = layers;
  p->E = E;
  try {
    const size_t L = layers, e = E;
    p->counts1.assign(L * e * e, 0u);
    p->sum1.assign(L * e, 0u);
    if (E <= kPairMaxE) {
      p->counts2.assign(L * e * e * e, 0u);
      p->sum2.assign(L * e * e, 0u);
    }
  } catch (...) {
    delete p;
    set_error("moe_predictor_create: out of host memory");
    return MOE_ERR_OOM;
  }
  *out = p;
  return MOE_OK;
}

void moe_predictor_destroy(moe_route_predictor* p) { delete p; }

moe_status_t moe_predictor_observe(moe_route_predictor* p, int layer, const int32_t* prev2_ids,
                                   const int32_t* prev_ids, const int32_t* cur_ids, int T, int k) {
  if (!p || layer <= 0 || layer >= p->layers || T < 0 || k <= 0 || (T > 0 && (!prev_ids || !cur_ids)) ||
      (prev2_ids && layer < 2)) {
    set_error("moe_predictor_observe: bad arguments");
    return MOE_ERR_INVALID_ARG;
  }
  const size_t E = p->E;
  for (int i = 0; i < T * k; ++i) {
    const int c = prev2_ids ? prev2_ids[i] : 0, a = prev_ids[i], b = cur_ids[i];
    if (a < 0 || a >= p->E || b < 0 || b >= p->E || c < 0 || c >= p->E) {
      set_error("moe_predictor_observe: expert id out of range");
      return MOE_ERR_INVALID_ARG;
    }
  }
  for (int i = 0; i < T * k; ++i) {
    const size_t a = prev_ids[i], b = cur_ids[i];
    ++p->counts1[(layer * E + a) * E + b];
    ++p->sum1[layer * E + a];
    if (prev2_ids && !p->counts2.empty()) {
      const size_t c = prev2_ids[i];
      ++p->counts2[((layer * E + c) * E + a) * E + b];
      ++p->sum2[(layer * E + c) * E + a];
    }
  }
  return MOE_OK;
}

moe_status_t moe_predictor_predict(const moe_route_predictor* p, int layer, const int32_t* prev2_ids,
                                   const int32_t* prev_ids, int T, int k, int max_out, double min_score,
                                   int32_t* out_ids, int32_t* n_out) {
  if (!p || layer <= 0 || layer >= p->layers || T < 0 || k <= 0 || max_out < 0 || !n_out ||
      (T > 0 && !prev_ids) || (max_out > 0 && !out_ids) || (prev2_ids && layer < 2)) {
    set_error("moe_predictor_predict: bad arguments");
    return MOE_ERR_INVALID_ARG;
  }
  const size_t E = p->E;
  std::vector<double> score(E, 0.0);
  for (int i = 0; i < T * k; ++i) {
    const int a = prev_ids[i], c = prev2_ids ? prev2_ids[i] : 0;
    if (a < 0 || a >= p->E || c < 0 || c >= p->E) {
      set_error("moe_predictor_predict: expert id out of range");
      return MOE_ERR_INVALID_ARG;
    }
    const uint32_t* row = nullptr;
    uint64_t rs = 0;
    if (prev2_ids && !p->counts2.empty()) {
      const size_t key = (layer * E + c) * E + a;
      if (p->sum2[key] >= kPairSupport) {
        row = &p->counts2[key * E];
        rs = p->sum2[key];
      }
    }
    if (!row) {
      row = &p->counts1[(layer * E + a) * E];
      rs = p->sum1[layer * E + a];
    }
    if (!rs) continue;
    for (size_t b = 0; b < E; ++b)
      if (row[b]) score[b] += static_cast<double>(row[b]) / static_cast<double>(rs);
  }
  std::vector<int> order;
  for (size_t b = 0; b < E; ++b)
    if (score[b] > 0.0 && score[b] >= min_score) order.push_back(static_cast<int>(b));
  std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return score[x] > score[y]; });
  const int n = std::min<int>(max_out, static_cast<int>(order.size()));
  for (int i = 0; i < n; ++i) out_ids[i] = order[i];
  *n_out = n;
  return MOE_OK;
}

}  // extern "C"
