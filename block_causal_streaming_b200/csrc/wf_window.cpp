// wf_window.cpp -- host-side planner of a rolling context window (include/wf.h, wf_window_*).
//
// Each round of a streaming wavefront advances the diagonal of active cells by one chunk; a
// finished chunk gets a store pass whose K/V become history (KipQuest summary of arXiv
// 2611.00859, "The deep dive").  This file maps a round number to the chunks of that round and to
// the fixed chunk slots they occupy, with the anchor pinned in slot 0 and the history kept as a
// ring, so nothing that persists is ever moved (the project page's fixed attention slots, "03
// End-to-end KV transport", item 03 "Layout").  Pure host code: no CUDA call.
#include <cstdint>

#include "../../include/wf.h"

namespace {

int check_window(const wf_window_t* w, int32_t* slots, int64_t* tokens) {
  if (w == nullptr || w->stages == nullptr) return WF_ERR_INVALID_ARG;
  if (w->chunk_len < 1 || w->num_stages < 1 || w->history < 0) return WF_ERR_SHAPE;
  for (int i = 0; i < w->num_stages; ++i) {
    if (w->stages[i] <= 0) return WF_ERR_SHAPE;
    if (i > 0 && w->stages[i] >= w->stages[i - 1]) return WF_ERR_SHAPE;   // noisiest first
  }
  const int64_t n = 2 + static_cast<int64_t>(w->history) + w->num_stages;
  if (n > WF_MAX_CHUNKS) return WF_ERR_SHAPE;
  const int64_t t = n * w->chunk_len;
  if (t > INT32_MAX) return WF_ERR_SHAPE;
  if (slots != nullptr) *slots = static_cast<int32_t>(n);
  if (tokens != nullptr) *tokens = t;
  return WF_OK;
}

// Slot kept by stored chunk c: the anchor (c = 0) in slot 0, the others in the history ring.
int ring_slot(const wf_window_t* w, int64_t c) {
  return c == 0 ? 0 : 1 + static_cast<int>((c - 1) % w->history);
}

}  // namespace

int wf_window_slots(const wf_window_t* window, int32_t* slots, int64_t* tokens) {
  if (slots == nullptr || tokens == nullptr) return WF_ERR_INVALID_ARG;
  return check_window(window, slots, tokens);
}

int wf_window_round(const wf_window_t* w, int64_t round, wf_round_t* out) {
  if (out == nullptr) return WF_ERR_INVALID_ARG;
  const int rc = check_window(w, nullptr, nullptr);
  if (rc) return rc;
  if (round < 0) return WF_ERR_INVALID_ARG;
  const int64_t S = w->num_stages, H = w->history;
  int n = 0;
  auto put = [&](int64_t id, int role, int32_t stage) {
    out->chunk_id[n] = id;
    out->role[n] = role;
    out->chunk_stage[n] = stage;
    ++n;
  };
  const int64_t last_stored = round - S - 1;     // chunks <= this have finished their store pass
  if (last_stored >= 0) {
    put(0, WF_ROLE_ANCHOR, 0);
    if (H > 0) {
      // the kept history chunks, placed in ring-slot order: slot 1 + (c - 1) mod H
      const int64_t first = last_stored - H + 1 > 1 ? last_stored - H + 1 : 1;
      const int64_t count = last_stored - first + 1;
      for (int64_t s = 1; s <= H && count > 0; ++s) {
        // the kept chunk whose ring slot is s, if any: c = first + ((s - 1 - (first - 1)) mod H)
        const int64_t off = ((s - 1) - (first - 1) % H + H) % H;
        const int64_t c = first + off;
        if (off < count) put(c, WF_ROLE_HISTORY, 0);
      }
    }
  }
  out->num_ctx_chunks = n;
  const int64_t store = round - S;
  out->store_to = -1;
  out->evicted = -1;
  if (store >= 0) {
    put(store, WF_ROLE_STORE, 0);
    if (store >= 1 && H > 0 && store - H >= 1) {   // the ring is full: hand over after attention
      out->evicted = store - H;
      out->store_to = ring_slot(w, store);
    }
  }
  for (int64_t c = (round - S + 1 > 0 ? round - S + 1 : 0); c <= round; ++c)
    put(c, WF_ROLE_ACTIVE, w->stages[round - c]);     // in flight, oldest (cleanest) first
  out->round = round;
  out->num_chunks = n;
  for (int i = 0; i <= n; ++i) out->chunk_offsets[i] = i * w->chunk_len;
  // the store pass is the first query chunk: its rows see the slots up to its own
  out->store_kv_end = -1;
  for (int i = 0; i < n; ++i)
    if (out->role[i] == WF_ROLE_STORE) out->store_kv_end = out->chunk_offsets[i + 1];
  return WF_OK;
}

int wf_window_round_ring(const wf_window_t* w, int64_t round, wf_round_t* out) {
  if (out == nullptr) return WF_ERR_INVALID_ARG;
  const int rc = check_window(w, nullptr, nullptr);
  if (rc) return rc;
  if (round < 0) return WF_ERR_INVALID_ARG;
  const int64_t S = w->num_stages, H = w->history, R = H + 1;   // ring slots
  const int64_t store = round - S;                 // the chunk in its store pass, if >= 0
  int n = 0;
  auto put = [&](int64_t id, int role, int32_t stage) {
    out->chunk_id[n] = id;
    out->role[n] = role;
    out->chunk_stage[n] = stage;
    ++n;
  };
  out->store_to = -1;
  out->evicted = -1;
  out->store_kv_end = -1;
  int ctx = 0;
  if (store >= 0) {
    // slot 0: the anchor (chunk 0), in its store pass at round S
    put(0, store == 0 ? WF_ROLE_STORE : WF_ROLE_ANCHOR, 0);
    if (store >= 1) {
      // ring slots 1 .. min(store, R): stored chunks max(1, store - H) .. store, each in slot
      // 1 + (c - 1) mod R; the slots fill in order, so the occupied ones are contiguous
      const int64_t occupied = store < R ? store : R;
      const int64_t first = store - H > 1 ? store - H : 1;
      for (int64_t slot = 1; slot <= occupied; ++slot) {
        // the chunk in `slot`: the one in [first, store] congruent to slot - 1 modulo R
        const int64_t c = first + (((slot - 1) - (first - 1)) % R + R) % R;
        put(c, c == store ? WF_ROLE_STORE : WF_ROLE_HISTORY, 0);
      }
      if (store - R >= 1) out->evicted = store - R;   // its slot now holds the store pass
    }
    for (int i = 0; i < n; ++i) ctx += out->role[i] != WF_ROLE_STORE ? 1 : 0;
  }
  const int ring_end = n;                           // slots of anchor + occupied ring
  for (int64_t c = (round - S + 1 > 0 ? round - S + 1 : 0); c <= round; ++c)
    put(c, WF_ROLE_ACTIVE, w->stages[round - c]);     // in flight, oldest (cleanest) first
  out->round = round;
  out->num_chunks = n;
  out->num_ctx_chunks = ctx;
  for (int i = 0; i <= n; ++i) out->chunk_offsets[i] = i * w->chunk_len;
  if (store >= 0) out->store_kv_end = out->chunk_offsets[ring_end];
  return WF_OK;
}
