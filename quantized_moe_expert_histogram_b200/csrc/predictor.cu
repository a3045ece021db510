// Next-layer expert predictor for the offload mode (EdgeMoE's statistical
// profile of expert activations, keyed here by the previous layer's experts;
// ExactMoE/D2MoE: load the next experts while computing the current ones).
//
// counts[layer][a][b] = how often an assignment routed to expert a at layer
// layer-1 was routed, at the same choice position j of the same token, to
// expert b at layer `layer`.  A prediction for layer l from the routed ids
// of layer l-1 scores each expert b by sum over the assignments of
// counts[l][a][b] / sum_b' counts[l][a][b'] (the expected number of
// assignments routed to b) and returns the best-scoring experts whose score
// reaches min_score (ties to the lower id).  Host-only bookkeeping: the caller passes
// host arrays (the routed ids it already copied for moe_slot_stage).
#include <algorithm>
#include <new>
#include <vector>

#include "common.cuh"

using namespace moeq;

struct moe_route_predictor {
  int layers = 0, E = 0;
  std::vector<uint32_t> counts;  // [layers][E][E]
  std::vector<uint64_t> row_sum;  // [layers][E]
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
    p->counts.assign(static_cast<size_t>(layers) * E * E, 0u);
    p->row_sum.assign(static_cast<size_t>(layers) * E, 0u);
  } catch (...) {
    delete p;
    set_error("moe_predictor_create: out of host memory");
    return MOE_ERR_OOM;
  }
  *out = p;
  return MOE_OK;
}

void moe_predictor_destroy(moe_route_predictor* p) { delete p; }

moe_status_t moe_predictor_observe(moe_route_predictor* p, int layer, const int32_t* prev_ids,
                                   const int32_t* cur_ids, int T, int k) {
  if (!p || layer <= 0 || layer >= p->layers || T < 0 || k <= 0 || (T > 0 && (!prev_ids || !cur_ids))) {
    set_error("moe_predictor_observe: bad arguments");
    return MOE_ERR_INVALID_ARG;
  }
  const int E = p->E;
  for (int i = 0; i < T * k; ++i) {
    const int a = prev_ids[i], b = cur_ids[i];
    if (a < 0 || a >= E || b < 0 || b >= E) {
      set_error("moe_predictor_observe: expert id out of range");
      return MOE_ERR_INVALID_ARG;
    }
    ++p->counts[(static_cast<size_t>(layer) * E + a) * E + b];
    ++p->row_sum[static_cast<size_t>(layer) * E + a];
  }
  return MOE_OK;
}

moe_status_t moe_predictor_predict(const moe_route_predictor* p, int layer, const int32_t* prev_ids, int T,
                                   int k, int max_out, double min_score, int32_t* out_ids, int32_t* n_out) {
  if (!p || layer <= 0 || layer >= p->layers || T < 0 || k <= 0 || max_out < 0 || !n_out ||
      (T > 0 && !prev_ids) || (max_out > 0 && !out_ids)) {
    set_error("moe_predictor_predict: bad arguments");
    return MOE_ERR_INVALID_ARG;
  }
  const int E = p->E;
  std::vector<double> score(E, 0.0);
  for (int i = 0; i < T * k; ++i) {
    const int a = prev_ids[i];
    if (a < 0 || a >= E) {
      set_error("moe_predictor_predict: expert id out of range");
      return MOE_ERR_INVALID_ARG;
    }
    const uint64_t rs = p->row_sum[static_cast<size_t>(layer) * E + a];
    if (!rs) continue;
    const uint32_t* row = &p->counts[(static_cast<size_t>(layer) * E + a) * E];
    for (int b = 0; b < E; ++b)
      if (row[b]) score[b] += static_cast<double>(row[b]) / static_cast<double>(rs);
  }
  std::vector<int> order;
  for (int b = 0; b < E; ++b)
    if (score[b] > 0.0 && score[b] >= min_score) order.push_back(b);
  std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return score[x] > score[y]; });
  const int n = std::min<int>(max_out, static_cast<int>(order.size()));
  for (int i = 0; i < n; ++i) out_ids[i] = order[i];
  *n_out = n;
  return MOE_OK;
}

}  // extern "C"
