// Offload mode: a per-layer GPU slot cache of expert blobs fed from pinned
// host memory with cudaMemcpyAsync on a copy stream, overlapped with the
// grouped FFN on the compute stream.
//
// A layer-step's distinct experts are ordered hits first, then the experts
// that need copies by descending row count (the hottest expert is loaded
// first; in plane mode resident experts that need more planes before the
// ones that are not resident), and cut into waves of at most slots/2
// experts.  Waves alternate
// between slot sets in LRU order and never into a slot of the previous wave,
// so the copies of wave w+1 overlap the compute of wave w (load E2 while
// computing E1).  A slot is overwritten only after the compute that last
// read it has finished (per-slot event), and a wave computes only after its
// copies have landed (per-wave event).  The FFN of a wave sees a device
// table slot_of[E] listing just that wave's experts.
//
// Plane mode (nested-width blobs): a slot records the widest width whose bit
// planes it holds.  An expert is copied only up to the widest width its
// assignments of the step use -- the Q2 planes and the scales for width 2,
// plus D3 for 3, plus D4 for 4 -- and a resident expert needed wider later
// receives only the missing planes.  The blob is laid out width by width
// (Q2 of the three matrices and the scales, then D3, then D4), so either is
// one contiguous copy -- the range between the ends of two widths -- with
// an expert's base planes first (the bit order of D2MoE's
// Hottest-Expert-Bit-First schedule, whose expert order is the wave order).
#include <algorithm>
#include <atomic>
#include <new>
#include <vector>

#include "common.cuh"

using namespace moeq;

namespace {
std::atomic<int> g_fault_what{0};
std::atomic<int> g_fault_count{0};

bool take_fault(int what) {
  if (g_fault_what.load() != what) return false;
  int c = g_fault_count.load();
  while (c > 0) {
    if (g_fault_count.compare_exchange_weak(c, c - 1)) return true;
  }
  return false;
}

inline cudaStream_t S(moe_stream_t s) { return static_cast<cudaStream_t>(s); }

// One planned copy: expert e into slot s, planes of widths (from, to]
// (from = 0: a fresh load, including the scales).
struct SlotCopy {
  int e, s, from, to;
};
}  // namespace

struct moe_slot_cache {
  int E = 0, S = 0, max_waves = 0;
  size_t blob_bytes = 0;
  const uint8_t* host = nullptr;
  uint8_t* pool = nullptr;
  // plane mode: byte ranges of the blob format (gate, up, down)
  bool planes = false;
  size_t width_end[5] = {};  // plane mode: blob bytes holding the planes up to width b (b = 2, 3, 4)
  std::vector<int> slot_of;        // expert -> slot, -1 when not resident
  std::vector<int> expert_in;      // slot -> expert, -1 when empty
  std::vector<int> width_in;       // slot -> widest width whose planes it holds (4 in blob mode)
  std::vector<uint64_t> last_use;  // slot -> logical time of last use
  uint64_t clock = 1;
  std::vector<cudaEvent_t> slot_free;  // recorded after the last compute reading the slot
  std::vector<char> slot_free_valid;
  std::vector<cudaEvent_t> copy_done;  // per wave
  std::vector<char> copy_pending;      // per wave: wave has copies to wait for
  cudaEvent_t prefetch_done = nullptr;  // after the last moe_slot_prefetch copies
  bool prefetch_pending = false;        // the next moe_slot_ffn waits for them
  cudaEvent_t tables_done = nullptr;
  bool tables_done_valid = false;
  int32_t* d_tables = nullptr;  // device [max_waves][E]
  int32_t* h_tables = nullptr;  // pinned host [max_waves][E]
  // plan of the current step
  std::vector<std::vector<int>> waves;             // experts per wave
  std::vector<std::vector<SlotCopy>> wave_copies;  // copies per wave
  std::vector<std::vector<int>> wave_slots;        // slot of each expert of the wave
  int copies_issued = 0;                           // waves whose copies were issued
  bool staged = false;  // a plan is staged and its moe_slot_ffn has not run yet
  // busy-time measurement (moe_slot_timing): event pairs around each wave's
  // copies and each wave's FFN, recorded after the waits on the other stream
  bool timing = false;
  std::vector<cudaEvent_t> tev[2];  // [0] copies, [1] FFN: start, end, start, end, ...
  size_t tev_used[2] = {0, 0};
  int64_t stats[3] = {0, 0, 0};
};

namespace {

// Bytes a copy of widths (from, to] moves.
size_t copy_bytes(const moe_slot_cache* c, const SlotCopy& k) {
  if (!c->planes) return c->blob_bytes;
  return c->width_end[k.to] - c->width_end[k.from];
}

// After a failed copy: the slots of waves >= w that were to receive copies
// hold stale bytes, so their experts are dropped, and the plan is dropped.
void invalidate_from(moe_slot_cache* c, int w) {
  for (size_t v = static_cast<size_t>(w); v < c->waves.size(); ++v)
    for (const SlotCopy& k : c->wave_copies[v]) {
      if (c->expert_in[k.s] == k.e) c->expert_in[k.s] = -1;
      c->width_in[k.s] = 0;
      c->slot_of[k.e] = -1;
    }
  c->waves.clear();
  c->wave_copies.clear();
  c->wave_slots.clear();
  c->staged = false;
}

// Record the next timing event of kind k (0 copies, 1 FFN) on stream s.
moe_status_t timing_mark(moe_slot_cache* c, int k, cudaStream_t s) {
  if (!c->timing) return MOE_OK;
  auto& v = c->tev[k];
  if (c->tev_used[k] == v.size()) {
    cudaEvent_t e = nullptr;
    moe_status_t st = cuda_check(cudaEventCreate(&e), "timing event");
    if (st != MOE_OK) return st;
    v.push_back(e);
  }
  return cuda_check(cudaEventRecord(v[c->tev_used[k]++], s), "timing event record");
}

moe_status_t h2d(moe_slot_cache* c, int s, int e, size_t off, size_t len, cudaStream_t copy) {
  return cuda_check(cudaMemcpyAsync(c->pool + static_cast<size_t>(s) * c->blob_bytes + off,
                                    c->host + static_cast<size_t>(e) * c->blob_bytes + off, len,
                                    cudaMemcpyHostToDevice, copy),
                    "slot H2D copy");
}

// Issue the copies `todo` on `copy` after their slots are free: one copy
// per expert (plane mode: the blob range between the ends of widths from
// and to).
moe_status_t issue(moe_slot_cache* c, const std::vector<SlotCopy>& todo, cudaStream_t copy) {
  for (const SlotCopy& k : todo) {
    if (c->slot_free_valid[k.s]) {
      moe_status_t st = cuda_check(cudaStreamWaitEvent(copy, c->slot_free[k.s], 0), "slot wait free");
      if (st != MOE_OK) return st;
    }
  }
  moe_status_t st = timing_mark(c, 0, copy);
  if (st != MOE_OK) return st;
  for (const SlotCopy& k : todo) {
    const size_t off = c->planes ? c->width_end[k.from] : 0;
    if ((st = h2d(c, k.s, k.e, off, copy_bytes(c, k), copy)) != MOE_OK) return st;
  }
  return timing_mark(c, 0, copy);
}

moe_status_t issue_copies(moe_slot_cache* c, int w, cudaStream_t copy) {
  const auto& todo = c->wave_copies[w];
  for (size_t i = 0; i < todo.size(); ++i)
    if (take_fault(2)) {
      set_error("moe_slot_stage: injected copy failure (expert %d)", todo[i].e);
      return MOE_ERR_FAULT_INJECTED;
    }
  c->copy_pending[w] = !todo.empty();
  if (todo.empty()) return MOE_OK;
  moe_status_t st = issue(c, todo, copy);
  if (st != MOE_OK) return st;
  return cuda_check(cudaEventRecord(c->copy_done[w], copy), "slot copy event");
}

moe_status_t create(int E, int slots, size_t blob_bytes, const void* host_blobs, void* device_pool,
                    const BlobLayout* planes, moe_slot_cache** out) {
  if (!out || !host_blobs || !device_pool || E <= 0 || E > 256 || slots < 2 || blob_bytes == 0) {
    set_error("moe_slot_cache_create: bad arguments");
    return MOE_ERR_INVALID_ARG;
  }
  if (blob_bytes % 16) {
    set_error("moe_slot_cache_create: blob_bytes must be a multiple of 16");
    return MOE_ERR_INVALID_ARG;
  }
  *out = nullptr;
  moe_slot_cache* c = new (std::nothrow) moe_slot_cache();
  if (!c) {
    set_error("moe_slot_cache_create: out of host memory");
    return MOE_ERR_OOM;
  }
  c->E = E;
  c->S = slots;
  c->blob_bytes = blob_bytes;
  c->host = static_cast<const uint8_t*>(host_blobs);
  c->pool = static_cast<uint8_t*>(device_pool);
  if (planes) {  // width by width: [Q2 x3 | scales x3 | D3 x3 | D4 x3]
    c->planes = true;
    c->width_end[2] = planes->d3[0];
    c->width_end[3] = planes->d4[0];
    c->width_end[4] = planes->bytes;
  }
  c->slot_of.assign(E, -1);
  c->expert_in.assign(slots, -1);
  c->width_in.assign(slots, 0);
  c->last_use.assign(slots, 0);
  c->slot_free.assign(slots, nullptr);
  c->slot_free_valid.assign(slots, 0);
  // at most E distinct experts, at least 1 per wave
  c->max_waves = E;
  c->copy_done.assign(c->max_waves, nullptr);
  c->copy_pending.assign(c->max_waves, 0);
  moe_status_t st = MOE_OK;
  for (int s = 0; s < slots && st == MOE_OK; ++s)
    st = cuda_check(cudaEventCreateWithFlags(&c->slot_free[s], cudaEventDisableTiming), "event");
  for (int w = 0; w < c->max_waves && st == MOE_OK; ++w)
    st = cuda_check(cudaEventCreateWithFlags(&c->copy_done[w], cudaEventDisableTiming), "event");
  if (st == MOE_OK)
    st = cuda_check(cudaEventCreateWithFlags(&c->tables_done, cudaEventDisableTiming), "event");
  if (st == MOE_OK)
    st = cuda_check(cudaEventCreateWithFlags(&c->prefetch_done, cudaEventDisableTiming), "event");
  if (st == MOE_OK)
    st = cuda_check(cudaMalloc(&c->d_tables, sizeof(int32_t) * c->max_waves * E), "table alloc");
  if (st == MOE_OK)
    st = cuda_check(cudaHostAlloc(&c->h_tables, sizeof(int32_t) * c->max_waves * E,
                                  cudaHostAllocDefault),
                    "table host alloc");
  if (st != MOE_OK) {
    moe_slot_cache_destroy(c);
    return st;
  }
  *out = c;
  return MOE_OK;
}

}  // namespace

extern "C" {

void moe_debug_inject_fault(int what, int count) {
  g_fault_what.store(what);
  g_fault_count.store(what ? count : 0);
}

moe_status_t moe_slot_cache_create(int E, int slots, size_t blob_bytes, const void* host_blobs,
                                   void* device_pool, moe_slot_cache** out) {
  return create(E, slots, blob_bytes, host_blobs, device_pool, nullptr, out);
}

moe_status_t moe_slot_cache_create_planes(int E, int slots, int d, int F, int group, const void* host_blobs,
                                          void* device_pool, moe_slot_cache** out) {
  const BlobLayout L = blob_layout(d, F, group, MOE_LAYOUT_PLANES);
  if (!L.valid) {
    set_error("moe_slot_cache_create_planes: unsupported shape d=%d F=%d group=%d", d, F, group);
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  return create(E, slots, L.bytes, host_blobs, device_pool, &L, out);
}

void moe_slot_cache_destroy(moe_slot_cache* c) {
  if (!c) return;
  for (auto e : c->slot_free)
    if (e) {
      cudaEventSynchronize(e);
      cudaEventDestroy(e);
    }
  for (auto e : c->copy_done)
    if (e) {
      cudaEventSynchronize(e);
      cudaEventDestroy(e);
    }
  if (c->tables_done) {
    cudaEventSynchronize(c->tables_done);
    cudaEventDestroy(c->tables_done);
  }
  if (c->prefetch_done) {
    cudaEventSynchronize(c->prefetch_done);
    cudaEventDestroy(c->prefetch_done);
  }
  for (int k = 0; k < 2; ++k)
    for (auto e : c->tev[k]) {
      cudaEventSynchronize(e);
      cudaEventDestroy(e);
    }
  if (c->d_tables) cudaFree(c->d_tables);
  if (c->h_tables) cudaFreeHost(c->h_tables);
  delete c;
}

moe_status_t moe_slot_timing(moe_slot_cache* c, int enable) {
  if (!c) {
    set_error("moe_slot_timing: null cache");
    return MOE_ERR_INVALID_ARG;
  }
  c->timing = enable != 0;
  c->tev_used[0] = c->tev_used[1] = 0;
  return MOE_OK;
}

moe_status_t moe_slot_timing_read(moe_slot_cache* c, double* copy_ms, double* ffn_ms) {
  if (!c || !copy_ms || !ffn_ms) {
    set_error("moe_slot_timing_read: bad arguments");
    return MOE_ERR_INVALID_ARG;
  }
  double sum[2] = {0.0, 0.0};
  for (int k = 0; k < 2; ++k) {
    for (size_t i = 0; i + 1 < c->tev_used[k]; i += 2) {
      moe_status_t st = cuda_check(cudaEventSynchronize(c->tev[k][i + 1]), "timing event wait");
      if (st != MOE_OK) return st;
      float ms = 0.f;
      st = cuda_check(cudaEventElapsedTime(&ms, c->tev[k][i], c->tev[k][i + 1]), "timing elapsed");
      if (st != MOE_OK) return st;
      sum[k] += ms;
    }
    c->tev_used[k] = 0;
  }
  *copy_ms = sum[0];
  *ffn_ms = sum[1];
  return MOE_OK;
}

moe_status_t moe_slot_stage(moe_slot_cache* c, const int32_t* ids_host, const uint8_t* bits_host, int n_ids,
                            moe_stream_t copy_stream, moe_stream_t compute_stream,
                            int32_t* n_waves, int64_t* stats_host) {
  (void)compute_stream;
  if (!c || !n_waves || n_ids < 0 || (n_ids > 0 && !ids_host)) {
    set_error("moe_slot_stage: bad arguments");
    return MOE_ERR_INVALID_ARG;
  }
  if (take_fault(1)) {
    set_error("moe_slot_stage: injected fault before any work");
    return MOE_ERR_FAULT_INJECTED;
  }
  std::vector<int> cnt(c->E, 0), need(c->E, 0);
  for (int i = 0; i < n_ids; ++i) {
    const int e = ids_host[i];
    if (e < 0 || e >= c->E) {
      set_error("moe_slot_stage: expert id %d out of range [0,%d)", e, c->E);
      return MOE_ERR_INVALID_ARG;
    }
    int b = 4;
    if (c->planes && bits_host) {
      b = bits_host[i];
      if (b < 2 || b > 4) {
        set_error("moe_slot_stage: bit width %d not in {2, 3, 4}", b);
        return MOE_ERR_INVALID_ARG;
      }
    }
    ++cnt[e];
    need[e] = std::max(need[e], b);
  }
  // hits: resident with every plane the step needs; upgrades (plane mode):
  // resident but missing planes; misses: not resident.  Resident experts
  // come first (hits, then upgrades hottest first), then misses hottest
  // first, so that every wave after them holds only experts that are not
  // resident yet -- the slots a later wave pins are then only those of the
  // wave before it.
  std::vector<int> hits, upgrades, misses;
  for (int e = 0; e < c->E; ++e) {
    if (!cnt[e]) continue;
    const int s = c->slot_of[e];
    if (s < 0) misses.push_back(e);
    else (c->width_in[s] >= need[e] ? hits : upgrades).push_back(e);
  }
  auto hotter = [&](int a, int b) { return cnt[a] > cnt[b]; };
  std::stable_sort(upgrades.begin(), upgrades.end(), hotter);
  std::stable_sort(misses.begin(), misses.end(), hotter);
  std::vector<int> order(hits);
  order.insert(order.end(), upgrades.begin(), upgrades.end());
  order.insert(order.end(), misses.begin(), misses.end());
  const int W = std::max(1, c->S / 2);
  const int nw = static_cast<int>((order.size() + W - 1) / W);
  c->waves.assign(nw, {});
  c->wave_copies.assign(nw, {});
  c->wave_slots.assign(nw, {});
  for (size_t i = 0; i < order.size(); ++i) c->waves[i / W].push_back(order[i]);

  // Assign slots wave by wave.  Resident experts keep their slot; a fresh
  // load takes the least recently used slot that holds nothing needed by
  // this wave or later ones.
  std::vector<int> slot_of = c->slot_of, expert_in = c->expert_in, width_in = c->width_in;
  std::vector<uint64_t> last_use = c->last_use;
  uint64_t clock = c->clock;
  std::vector<char> needed_later(c->E, 0);
  for (int e : order) needed_later[e] = 1;
  int64_t n_hits = 0, n_copy = 0, bytes = 0;
  std::vector<int> prev_slots;  // slots of wave w-1: its compute may still be unqueued
  for (int w = 0; w < nw; ++w) {
    const uint64_t t = ++clock;
    std::vector<char> pinned(c->S, 0);
    for (int s : prev_slots) pinned[s] = 1;
    for (int e : c->waves[w])
      if (slot_of[e] >= 0) pinned[slot_of[e]] = 1;
    for (int s = 0; s < c->S; ++s)
      if (expert_in[s] >= 0 && needed_later[expert_in[s]]) pinned[s] = 1;
    for (int e : c->waves[w]) {
      int s = slot_of[e];
      if (s >= 0 && width_in[s] >= need[e]) {
        ++n_hits;
      } else {
        SlotCopy k{e, s, 0, need[e]};
        if (s >= 0) {
          k.from = width_in[s];  // plane mode: only the missing planes
        } else {
          int best = -1;
          for (int cand = 0; cand < c->S; ++cand) {
            if (pinned[cand]) continue;
            if (best < 0 || last_use[cand] < last_use[best]) best = cand;
          }
          if (best < 0) {
            set_error("moe_slot_stage: no free slot (slots=%d)", c->S);
            return MOE_ERR_INVALID_ARG;
          }
          s = best;
          if (expert_in[s] >= 0) slot_of[expert_in[s]] = -1;
          expert_in[s] = e;
          slot_of[e] = s;
          pinned[s] = 1;
          k.s = s;
        }
        width_in[s] = c->planes ? need[e] : 4;
        if (!c->planes) k.to = 4;
        c->wave_copies[w].push_back(k);
        bytes += static_cast<int64_t>(copy_bytes(c, k));
        ++n_copy;
      }
      last_use[s] = t;
      c->wave_slots[w].push_back(s);
    }
    for (int e : c->waves[w]) needed_later[e] = 0;
    prev_slots = c->wave_slots[w];
  }
  c->slot_of.swap(slot_of);
  c->expert_in.swap(expert_in);
  c->width_in.swap(width_in);
  c->last_use.swap(last_use);
  c->clock = clock;
  // Device tables of this step: the previous step's uploads must have run
  // before the pinned staging rows are rewritten.
  if (c->tables_done_valid) {
    moe_status_t st = cuda_check(cudaEventSynchronize(c->tables_done), "slot table reuse");
    if (st != MOE_OK) return st;
  }
  for (int w = 0; w < nw; ++w) {
    int32_t* row = c->h_tables + static_cast<size_t>(w) * c->E;
    for (int e = 0; e < c->E; ++e) row[e] = -1;
    for (size_t i = 0; i < c->waves[w].size(); ++i) row[c->waves[w][i]] = c->wave_slots[w][i];
  }
  c->copies_issued = 0;
  for (int w = 0; w < std::min(nw, 2); ++w) {
    moe_status_t st = issue_copies(c, w, S(copy_stream));
    if (st != MOE_OK) {
      invalidate_from(c, w);
      return st;
    }
    c->copies_issued = w + 1;
  }
  *n_waves = nw;
  c->staged = true;
  c->stats[0] = n_hits;
  c->stats[1] = n_copy;
  c->stats[2] = bytes;
  if (stats_host) {
    stats_host[0] = c->stats[0];
    stats_host[1] = c->stats[1];
    stats_host[2] = c->stats[2];
  }
  return MOE_OK;
}

moe_status_t moe_slot_prefetch(moe_slot_cache* c, const int32_t* ids_host, int n_ids, int max_copies,
                               moe_stream_t copy_stream, int32_t* n_copied) {
  if (!c || n_ids < 0 || max_copies < 0 || (n_ids > 0 && !ids_host)) {
    set_error("moe_slot_prefetch: bad arguments");
    return MOE_ERR_INVALID_ARG;
  }
  if (n_copied) *n_copied = 0;
  if (c->staged) {
    // the staged plan's slots (hits, and copies of waves issued later) must
    // keep their experts until its moe_slot_ffn has run
    set_error("moe_slot_prefetch: called between moe_slot_stage and moe_slot_ffn of the same cache");
    return MOE_ERR_INVALID_ARG;
  }
  // Victims: least recently used slots, never one filled by this call; each
  // copy (every plane) waits for the compute that last read its slot (a step
  // of this layer whose FFN may still run).
  std::vector<char> pinned(c->S, 0);
  std::vector<SlotCopy> todo;
  for (int i = 0; i < n_ids && static_cast<int>(todo.size()) < max_copies; ++i) {
    const int e = ids_host[i];
    if (e < 0 || e >= c->E) {
      set_error("moe_slot_prefetch: expert id %d out of range [0,%d)", e, c->E);
      return MOE_ERR_INVALID_ARG;
    }
    if (c->slot_of[e] >= 0) continue;
    int best = -1;
    for (int cand = 0; cand < c->S; ++cand) {
      if (pinned[cand]) continue;
      if (best < 0 || c->last_use[cand] < c->last_use[best]) best = cand;
    }
    if (best < 0) break;
    if (take_fault(2)) {
      set_error("moe_slot_prefetch: injected copy failure (expert %d)", e);
      return MOE_ERR_FAULT_INJECTED;
    }
    if (c->expert_in[best] >= 0) c->slot_of[c->expert_in[best]] = -1;
    c->expert_in[best] = e;
    c->slot_of[e] = best;
    c->width_in[best] = 4;
    c->last_use[best] = ++c->clock;
    pinned[best] = 1;
    todo.push_back(SlotCopy{e, best, 0, 4});
  }
  if (!todo.empty()) {
    moe_status_t st = issue(c, todo, S(copy_stream));
    if (st != MOE_OK) return st;
    st = cuda_check(cudaEventRecord(c->prefetch_done, S(copy_stream)), "slot prefetch event");
    if (st != MOE_OK) return st;
    c->prefetch_pending = true;
  }
  if (n_copied) *n_copied = static_cast<int32_t>(todo.size());
  return MOE_OK;
}

moe_status_t moe_slot_ffn(moe_slot_cache* c, const void* x_perm, const int32_t* offsets,
                          int total_rows, int T, int d, int F, int group, int layout,
                          void* workspace, size_t workspace_bytes, void* y_perm,
                          int32_t* status, moe_stream_t copy_stream,
                          moe_stream_t compute_stream) {
  if (!c) {
    set_error("moe_slot_ffn: null cache");
    return MOE_ERR_INVALID_ARG;
  }
  if (c->planes && layout != MOE_LAYOUT_PLANES) {
    set_error("moe_slot_ffn: a plane-mode cache holds nested-plane blobs (layout %d given)", layout);
    return MOE_ERR_INVALID_ARG;
  }
  const int nw = static_cast<int>(c->waves.size());
  const size_t table_bytes = sizeof(int32_t) * c->E;
  if (c->prefetch_pending) {  // experts staged ahead by moe_slot_prefetch count as hits
    moe_status_t st = cuda_check(cudaStreamWaitEvent(S(compute_stream), c->prefetch_done, 0),
                                 "slot wait prefetch");
    if (st != MOE_OK) return st;
    c->prefetch_pending = false;
  }
  for (int w = 0; w < nw; ++w) {
    if (c->copy_pending[w]) {
      moe_status_t st = cuda_check(cudaStreamWaitEvent(S(compute_stream), c->copy_done[w], 0),
                                   "slot wait copies");
      if (st != MOE_OK) return st;
    }
    int32_t* dt = c->d_tables + static_cast<size_t>(w) * c->E;
    moe_status_t st = cuda_check(cudaMemcpyAsync(dt, c->h_tables + static_cast<size_t>(w) * c->E,
                                                 table_bytes, cudaMemcpyHostToDevice,
                                                 S(compute_stream)),
                                 "slot table upload");
    if (st != MOE_OK) return st;
    if (w == nw - 1) {
      st = cuda_check(cudaEventRecord(c->tables_done, S(compute_stream)), "table event");
      if (st != MOE_OK) return st;
      c->tables_done_valid = true;
    }
    st = timing_mark(c, 1, S(compute_stream));
    if (st != MOE_OK) return st;
    st = moe_grouped_ffn_wq(x_perm, offsets, c->pool, dt, total_rows, T, c->E, d, F, group, layout,
                            workspace, workspace_bytes, y_perm, status, compute_stream);
    if (st != MOE_OK) return st;
    st = timing_mark(c, 1, S(compute_stream));
    if (st != MOE_OK) return st;
    for (int s : c->wave_slots[w]) {
      st = cuda_check(cudaEventRecord(c->slot_free[s], S(compute_stream)), "slot free event");
      if (st != MOE_OK) return st;
      c->slot_free_valid[s] = 1;
    }
    const int nxt = w + 2;
    if (nxt < nw && nxt >= c->copies_issued) {
      st = issue_copies(c, nxt, S(copy_stream));
      if (st != MOE_OK) {
        invalidate_from(c, nxt);
        return st;
      }
      c->copies_issued = nxt + 1;
    }
  }
  c->staged = false;
  return MOE_OK;
}

}  // extern "C"
