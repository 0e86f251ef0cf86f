// Per-layer LFU expert-slot cache: host planner and staging engine.
//
// Source: "TurboFieldfare: Gemma 4 26B on an 8 GB MacBook, in ~2 GB of RAM"
// (blog-mushroom.pages.dev), section "Why 26B Fits in 2 GB": per token the
// host checks the 8 selected experts against a 16-slot LFU cache of that
// layer; hits reuse the resident copy, misses fetch the expert blob, and the
// shared-expert branch runs while the fetches complete.  Here the blobs live
// in pinned host memory and a miss is one cudaMemcpyAsync into a device slot
// on a side stream.
//
// Policy (the pages say only "16-slot LFU"): counts live while an expert is
// resident (insert 1, hit +1); within a step hits are taken first, then
// misses, each in the step's order; a global tick advances per access; a miss
// fills the lowest empty slot, else evicts, among slots not used by the
// current step, the smallest (count, last tick, slot index).
//
// Optional lookahead prefetch (off unless set): after a streamed layer call,
// up to P experts of that layer are staged ahead of their next use -- the
// non-resident ones accessed most often so far in the run (ties to the lower
// id), each into the slot a miss would take, and only while that slot is
// empty or its resident's count is below the candidate's access total.  A
// prefetched expert enters with count 0; it is one more step of the layer
// and is logged with hit = 2.
#include <chrono>
#include <cstdint>
#include <cstdio>
#include <algorithm>
#include <cstring>
#include <mutex>
#include <thread>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/moe.h"

namespace moe {
int fail(int code, const char* fmt, ...);
int cuda_check(cudaError_t e, const char* what);
}  // namespace moe

struct moe_lfu {
  int L = 0, E = 0, S = 0;
  size_t blob_bytes = 0, slot_stride = 0;
  const void* const* host_blobs = nullptr;    // [L*E] pinned host pointers (null: plan only)
  unsigned char* pool = nullptr;              // device, L*S*slot_stride
  std::vector<int32_t> expert, count, steps;  // [L*S], [L*S], [L]
  std::vector<int32_t> freq;                  // [L*E] accesses per expert over the run (prefetch ranking)
  int prefetch_n = 0;                         // experts prefetched per streamed layer call (0: off)
  std::vector<int64_t> last;                  // [L*S]
  int64_t tick = 0;
  std::vector<int32_t> log;                   // records of 5
  // device pointer tables: host mirror (pinned) per layer
  std::vector<void**> mirror;                 // [L] pinned arrays of E pointers
  std::vector<cudaEvent_t> mirror_ev;         // [L] table copy done
  int fault_kind = 0, fault_after = -1;
  long copies = 0;
  int64_t bytes_copied = 0;
  // A slot whose bytes do not hold the expert that expert[] names: a call that
  // failed after issuing copies was rolled back (its plan undone) while the
  // copies it had issued still overwrite their slots.  The next hit on such a
  // slot copies the blob again.
  std::vector<char> dirty;                    // [L*S]
  // Transaction of one call (moe_lfu_step, or a whole streamed layer call that
  // makes several steps): the layer's state as it was before the call, and
  // the slots that copies issued during the call write.  A failure restores
  // the state, so that repeating the call plans exactly as the first attempt.
  int txn_depth = 0, txn_layer = -1;
  std::vector<int32_t> snap_expert, snap_count, snap_freq;
  std::vector<int64_t> snap_last;
  int64_t snap_tick = 0;
  int32_t snap_steps = 0;
  size_t snap_log = 0;
  std::vector<int32_t> txn_written;
  // streamed layer forward: per-layer "slots read" events, pinned staging
  std::vector<cudaEvent_t> consumed;          // [L] recorded after the expert kernels of a layer
  cudaEvent_t done = nullptr, idx_ready = nullptr, stage_free = nullptr;
  // The kernels that last read each slot (streamed layer forward): read_ev is
  // a ring of events recorded on the main stream after a step's expert
  // kernels, read_seq counts the steps recorded, slot_read[l*S+s] is the
  // read_seq of the last step that read slot s (-1: not known, wait for all
  // of the layer's kernels).  A copy into a slot waits only for that event;
  // an event re-recorded by a later step only makes the wait longer.
  static constexpr int READ_RING = 64;
  std::vector<cudaEvent_t> read_ev;           // [READ_RING]
  int64_t read_seq = 0;
  int64_t read_done = 0;                      // every step below this one is known complete
  cudaStream_t read_stream = nullptr;         // the stream the read events were recorded on
  std::vector<int64_t> slot_read;             // [L*S]
  int32_t* pin_idx = nullptr;                 // pinned [cap_rows * 8]
  int32_t* pin_act = nullptr;                 // pinned [groups * (E + 1)]
  int cap_rows = 0;
};

namespace {

int victim(moe_lfu* h, int layer, const std::vector<char>& used) {
  int32_t* ex = &h->expert[static_cast<size_t>(layer) * h->S];
  for (int s = 0; s < h->S; ++s)
    if (ex[s] < 0) return s;
  int best = -1;
  for (int s = 0; s < h->S; ++s) {
    if (used[s]) continue;
    if (best < 0) { best = s; continue; }
    const size_t a = static_cast<size_t>(layer) * h->S + s, b = static_cast<size_t>(layer) * h->S + best;
    if (h->count[a] < h->count[b] || (h->count[a] == h->count[b] && h->last[a] < h->last[b])) best = s;
  }
  return best;
}

void txn_begin(moe_lfu* h, int layer) {
  if (h->txn_depth++ > 0) return;
  const size_t b = static_cast<size_t>(layer) * h->S;
  h->txn_layer = layer;
  h->snap_expert.assign(h->expert.begin() + b, h->expert.begin() + b + h->S);
  h->snap_count.assign(h->count.begin() + b, h->count.begin() + b + h->S);
  h->snap_last.assign(h->last.begin() + b, h->last.begin() + b + h->S);
  const size_t fb = static_cast<size_t>(layer) * h->E;
  h->snap_freq.assign(h->freq.begin() + fb, h->freq.begin() + fb + h->E);
  h->snap_tick = h->tick;
  h->snap_steps = h->steps[layer];
  h->snap_log = h->log.size();
  h->txn_written.clear();
}

void txn_commit(moe_lfu* h) {
  if (h->txn_depth > 0) --h->txn_depth;
}

// Undo the plan of the current transaction (every step of it) and mark the
// slots its issued copies overwrite.  Returns `status` for the caller to pass on.
int txn_rollback(moe_lfu* h, int status) {
  if (h->txn_depth == 0) return status;
  const int layer = h->txn_layer;
  const size_t b = static_cast<size_t>(layer) * h->S;
  std::copy(h->snap_expert.begin(), h->snap_expert.end(), h->expert.begin() + b);
  std::copy(h->snap_count.begin(), h->snap_count.end(), h->count.begin() + b);
  std::copy(h->snap_last.begin(), h->snap_last.end(), h->last.begin() + b);
  std::copy(h->snap_freq.begin(), h->snap_freq.end(), h->freq.begin() + static_cast<size_t>(layer) * h->E);
  h->tick = h->snap_tick;
  h->steps[layer] = h->snap_steps;
  h->log.resize(h->snap_log);
  if (!h->dirty.empty())
    for (int32_t s : h->txn_written) h->dirty[b + s] = 1;
  if (!h->slot_read.empty())
    for (int s = 0; s < h->S; ++s) h->slot_read[b + s] = -1;
  h->txn_written.clear();
  h->txn_depth = 0;
  return status;
}

// Plan one step: slots_out[i] / hit_out[i] for ids[i].  Updates the state and the log.
int plan(moe_lfu* h, int layer, const int32_t* ids, int n, int32_t* slots_out, int32_t* hit_out) {
  if (layer < 0 || layer >= h->L) return moe::fail(MOE_ERR_INVALID_ARG, "lfu: layer %d out of range", layer);
  if (n < 0 || n > h->S) return moe::fail(MOE_ERR_INVALID_ARG, "lfu: %d ids in a step (slots %d)", n, h->S);
  for (int i = 0; i < n; ++i) {
    if (ids[i] < 0 || ids[i] >= h->E) return moe::fail(MOE_ERR_INVALID_ARG, "lfu: expert id %d out of range", ids[i]);
    for (int j = 0; j < i; ++j)
      if (ids[j] == ids[i]) return moe::fail(MOE_ERR_INVALID_ARG, "lfu: expert %d twice in one step", ids[i]);
  }
  const size_t base = static_cast<size_t>(layer) * h->S;
  const int st = h->steps[layer]++;
  std::vector<char> used(h->S, 0);
  auto find = [&](int e) {
    for (int s = 0; s < h->S; ++s)
      if (h->expert[base + s] == e) return s;
    return -1;
  };
  for (int pass = 0; pass < 2; ++pass) {          // hits, then misses
    for (int i = 0; i < n; ++i) {
      const int e = ids[i];
      const int s0 = find(e);
      if (pass == 0 && s0 < 0) continue;
      if (pass == 1 && s0 >= 0 && hit_out[i] == 1) continue;
      int s;
      int hit;
      if (pass == 0) {
        s = s0;
        hit = 1;
        h->count[base + s] += 1;
      } else {
        s = victim(h, layer, used);
        hit = 0;
        h->expert[base + s] = e;
        h->count[base + s] = 1;
      }
      h->tick += 1;
      h->last[base + s] = h->tick;
      h->freq[static_cast<size_t>(layer) * h->E + e] += 1;
      used[s] = 1;
      slots_out[i] = s;
      hit_out[i] = hit;
      const int32_t rec[5] = {layer, st, e, hit, s};
      h->log.insert(h->log.end(), rec, rec + 5);
    }
  }
  return MOE_OK;
}

// Plan a lookahead prefetch of up to P experts of `layer` (the policy in the
// file header): ids_out / slots_out get the chosen experts and their slots.
int plan_prefetch(moe_lfu* h, int layer, int P, std::vector<int32_t>& ids_out, std::vector<int32_t>& slots_out) {
  ids_out.clear();
  slots_out.clear();
  if (P <= 0) return MOE_OK;
  const size_t base = static_cast<size_t>(layer) * h->S, fb = static_cast<size_t>(layer) * h->E;
  std::vector<char> res(h->E, 0);
  for (int s = 0; s < h->S; ++s)
    if (h->expert[base + s] >= 0) res[h->expert[base + s]] = 1;
  std::vector<int32_t> cand;
  for (int e = 0; e < h->E; ++e)
    if (!res[e] && h->freq[fb + e] > 0) cand.push_back(e);
  std::stable_sort(cand.begin(), cand.end(), [&](int32_t a, int32_t b) { return h->freq[fb + a] > h->freq[fb + b]; });
  const int st = h->steps[layer]++;
  std::vector<char> used(h->S, 0);
  for (size_t i = 0; i < cand.size() && static_cast<int>(ids_out.size()) < P; ++i) {
    const int e = cand[i];
    const int s = victim(h, layer, used);
    if (s < 0) break;
    if (h->expert[base + s] >= 0 && h->count[base + s] >= h->freq[fb + e]) break;   // no colder resident
    h->expert[base + s] = e;
    h->count[base + s] = 0;
    h->tick += 1;
    h->last[base + s] = h->tick;
    used[s] = 1;
    ids_out.push_back(e);
    slots_out.push_back(s);
    const int32_t rec[5] = {layer, st, e, 2, s};
    h->log.insert(h->log.end(), rec, rec + 5);
  }
  return MOE_OK;
}

// Bounded host wait for an event: polled without sleeping for the first
// millisecond (the waits on the layer path -- routing, table copies -- end
// within tens of microseconds, and a sleep of the thread overshoots by the
// scheduler's timer slack), then with 20 us sleeps until timeout_ms.
int wait_event(cudaEvent_t ev, int timeout_ms) {
  const auto t0 = std::chrono::steady_clock::now();
  while (true) {
    const cudaError_t e = cudaEventQuery(ev);
    if (e == cudaSuccess) return MOE_OK;
    if (e != cudaErrorNotReady) return moe::cuda_check(e, "lfu: event query");
    const auto waited = std::chrono::steady_clock::now() - t0;
    if (waited > std::chrono::milliseconds(timeout_ms))
      return moe::fail(MOE_ERR_TIMEOUT, "lfu: wait ran out after %d ms", timeout_ms);
    if (waited > std::chrono::milliseconds(1)) std::this_thread::sleep_for(std::chrono::microseconds(20));
  }
}

}  // namespace

extern "C" {

MOE_API int moe_lfu_create(int n_layers, int n_experts, int n_slots, size_t blob_bytes,
                           const void* const* host_blobs, void* slot_pool, size_t slot_stride, moe_lfu** out) {
  if (!out) return moe::fail(MOE_ERR_INVALID_ARG, "lfu_create: out is NULL");
  *out = nullptr;
  if (n_layers <= 0 || n_experts <= 0 || n_slots <= 0 || n_slots > 1024)
    return moe::fail(MOE_ERR_INVALID_ARG, "lfu_create: bad sizes");
  if ((host_blobs == nullptr) != (slot_pool == nullptr))
    return moe::fail(MOE_ERR_INVALID_ARG, "lfu_create: give both host blobs and a slot pool, or neither");
  if (slot_pool && (slot_stride < blob_bytes || slot_stride % 16 || blob_bytes == 0))
    return moe::fail(MOE_ERR_INVALID_ARG, "lfu_create: slot stride must be >= blob bytes and a multiple of 16");
  moe_lfu* h = new moe_lfu();
  h->L = n_layers; h->E = n_experts; h->S = n_slots;
  h->blob_bytes = blob_bytes; h->slot_stride = slot_stride;
  h->host_blobs = host_blobs;
  h->pool = static_cast<unsigned char*>(slot_pool);
  h->expert.assign(static_cast<size_t>(n_layers) * n_slots, -1);
  h->count.assign(static_cast<size_t>(n_layers) * n_slots, 0);
  h->last.assign(static_cast<size_t>(n_layers) * n_slots, 0);
  h->steps.assign(n_layers, 0);
  h->freq.assign(static_cast<size_t>(n_layers) * n_experts, 0);
  if (slot_pool) h->dirty.assign(static_cast<size_t>(n_layers) * n_slots, 0);
  if (slot_pool) {
    h->mirror.assign(n_layers, nullptr);
    h->mirror_ev.assign(n_layers, nullptr);
    for (int l = 0; l < n_layers; ++l) {
      void* p = nullptr;
      if (cudaHostAlloc(&p, sizeof(void*) * n_experts, cudaHostAllocDefault) != cudaSuccess ||
          cudaEventCreateWithFlags(&h->mirror_ev[l], cudaEventDisableTiming) != cudaSuccess) {
        const int st = moe::cuda_check(cudaGetLastError(), "lfu_create: pinned table");
        moe_lfu_destroy(h);
        return st ? st : MOE_ERR_CUDA;
      }
      h->mirror[l] = static_cast<void**>(p);
      for (int e = 0; e < n_experts; ++e) h->mirror[l][e] = nullptr;
    }
  }
  if (slot_pool) {
    h->consumed.assign(n_layers, nullptr);
    bool ok = true;
    for (int l = 0; l < n_layers && ok; ++l) ok = cudaEventCreateWithFlags(&h->consumed[l], cudaEventDisableTiming) == cudaSuccess;
    ok = ok && cudaEventCreateWithFlags(&h->done, cudaEventDisableTiming) == cudaSuccess;
    ok = ok && cudaEventCreateWithFlags(&h->idx_ready, cudaEventDisableTiming) == cudaSuccess;
    ok = ok && cudaEventCreateWithFlags(&h->stage_free, cudaEventDisableTiming) == cudaSuccess;
    h->read_ev.assign(moe_lfu::READ_RING, nullptr);
    for (int i = 0; i < moe_lfu::READ_RING && ok; ++i)
      ok = cudaEventCreateWithFlags(&h->read_ev[i], cudaEventDisableTiming) == cudaSuccess;
    h->slot_read.assign(static_cast<size_t>(n_layers) * n_slots, -1);
    void* p = nullptr;
    ok = ok && cudaHostAlloc(&p, sizeof(int32_t) * (n_experts + 1) * (n_experts + 1), 0) == cudaSuccess;
    h->pin_act = static_cast<int32_t*>(p);
    if (!ok) {
      const int st = moe::cuda_check(cudaGetLastError(), "lfu_create: events/pinned staging");
      moe_lfu_destroy(h);
      return st ? st : MOE_ERR_CUDA;
    }
  }
  *out = h;
  return MOE_OK;
}

MOE_API int moe_lfu_plan(moe_lfu* h, int layer, const int32_t* ids, int n, int32_t* slots_out, int32_t* hit_out) {
  if (!h || (n > 0 && (!ids || !slots_out || !hit_out))) return moe::fail(MOE_ERR_INVALID_ARG, "lfu_plan: NULL");
  std::vector<int32_t> hit(n, 0);
  const int st = plan(h, layer, ids, n, slots_out, hit.data());
  if (st == MOE_OK)
    for (int i = 0; i < n; ++i) hit_out[i] = hit[i];
  return st;
}

namespace {

// One step.  per_slot = false: every copy waits for wait_event (the public
// call).  per_slot = true (the streamed layer forward): a copy waits only for
// the kernels that last read its slot, and the device table copy (read by the
// previous step's kernels) waits for wait_event.  slots_out: the step's slots.
int lfu_step_impl(moe_lfu* h, int layer, const int32_t* ids, int n, void* side_stream, void* wait_event_,
                  bool per_slot, void* done_event, void** dev_table, int timeout_ms, int32_t* slots_out) {
  if (!h || !h->pool) return moe::fail(MOE_ERR_INVALID_ARG, "lfu_step: handle has no slot pool");
  if (n > 0 && !ids) return moe::fail(MOE_ERR_INVALID_ARG, "lfu_step: NULL ids");
  if (!dev_table || !done_event) return moe::fail(MOE_ERR_INVALID_ARG, "lfu_step: NULL table or event");
  if (layer < 0 || layer >= h->L) return moe::fail(MOE_ERR_INVALID_ARG, "lfu_step: layer %d out of range", layer);
  if (h->txn_depth > 0 && h->txn_layer != layer)
    return moe::fail(MOE_ERR_INVALID_ARG, "lfu_step: layer %d inside a call on layer %d", layer, h->txn_layer);
  cudaStream_t s = static_cast<cudaStream_t>(side_stream);
  cudaEvent_t wait_all = static_cast<cudaEvent_t>(wait_event_);
  std::vector<int32_t> slots(n), hit(n, 0);
  txn_begin(h, layer);
  int st = plan(h, layer, ids, n, slots.data(), hit.data());
  if (st) return txn_rollback(h, st);
  const size_t base = static_cast<size_t>(layer) * h->S;
  auto needs_copy = [&](int i) { return !hit[i] || h->dirty[base + slots[i]]; };
  // slots are overwritten only after the kernels that read them are done
  if (!per_slot || h->slot_read.empty()) {
    if (wait_all && (st = moe::cuda_check(cudaStreamWaitEvent(s, wait_all, 0), "lfu_step: wait")))
      return txn_rollback(h, st);
  } else {
    std::vector<char> waited(moe_lfu::READ_RING, 0);
    bool all = false;
    for (int i = 0; i < n && !all; ++i) {
      if (!needs_copy(i)) continue;
      const int64_t q = h->slot_read[base + slots[i]];
      if (q < 0) { all = true; break; }
      if (q < h->read_done) continue;         // its kernels have finished
      const int r = static_cast<int>(q % moe_lfu::READ_RING);
      if (waited[r]) continue;
      waited[r] = 1;
      if ((st = moe::cuda_check(cudaStreamWaitEvent(s, h->read_ev[r], 0), "lfu_step: wait slot reader")))
        return txn_rollback(h, st);
    }
    if (all && wait_all && (st = moe::cuda_check(cudaStreamWaitEvent(s, wait_all, 0), "lfu_step: wait")))
      return txn_rollback(h, st);
  }
  for (int i = 0; i < n; ++i) {
    unsigned char* slot = h->pool + (base + slots[i]) * h->slot_stride;
    // a miss, or a hit on a slot that a rolled-back call overwrote
    if (needs_copy(i)) {
      ++h->copies;
      if (h->fault_kind == MOE_LFU_FAULT_COPY_FAILS && h->fault_after >= 0 && h->copies > h->fault_after)
        return txn_rollback(h, moe::fail(MOE_ERR_CUDA, "lfu_step: injected copy failure (copy %ld)", h->copies));
      if (h->fault_kind == MOE_LFU_FAULT_SLOW_COPY && h->fault_after >= 0 && h->copies > h->fault_after)
        std::this_thread::sleep_for(std::chrono::milliseconds(50));
      const void* src = h->host_blobs[static_cast<size_t>(layer) * h->E + ids[i]];
      if ((st = moe::cuda_check(cudaMemcpyAsync(slot, src, h->blob_bytes, cudaMemcpyHostToDevice, s),
                                "lfu_step: copy")))
        return txn_rollback(h, st);
      h->txn_written.push_back(slots[i]);
      h->dirty[base + slots[i]] = 0;
      h->bytes_copied += static_cast<int64_t>(h->blob_bytes);
    }
  }
  // the device table is read by the previous step's kernels
  if (per_slot && wait_all && (st = moe::cuda_check(cudaStreamWaitEvent(s, wait_all, 0), "lfu_step: wait table")))
    return txn_rollback(h, st);
  // the pinned table mirror may still feed the previous copy of this layer's table
  if ((st = wait_event(h->mirror_ev[layer], timeout_ms))) return txn_rollback(h, st);
  for (int i = 0; i < n; ++i)
    h->mirror[layer][ids[i]] = h->pool + (base + slots[i]) * h->slot_stride;
  if ((st = moe::cuda_check(cudaMemcpyAsync(dev_table, h->mirror[layer], sizeof(void*) * h->E,
                                            cudaMemcpyHostToDevice, s), "lfu_step: table")))
    return txn_rollback(h, st);
  if ((st = moe::cuda_check(cudaEventRecord(h->mirror_ev[layer], s), "lfu_step: record")))
    return txn_rollback(h, st);
  if ((st = moe::cuda_check(cudaEventRecord(static_cast<cudaEvent_t>(done_event), s), "lfu_step: done event")))
    return txn_rollback(h, st);
  if (slots_out)
    for (int i = 0; i < n; ++i) slots_out[i] = slots[i];
  txn_commit(h);
  return MOE_OK;
}

}  // namespace

MOE_API int moe_lfu_step(moe_lfu* h, int layer, const int32_t* ids, int n, void* side_stream, void* wait_event_,
                         void* done_event, void** dev_table, int timeout_ms) {
  std::vector<int32_t> sl(n > 0 ? n : 0);
  const int st = lfu_step_impl(h, layer, ids, n, side_stream, wait_event_, false, done_event, dev_table, timeout_ms,
                               sl.data());
  // the caller's kernels read these slots, ordered by the caller's own events
  if (st == MOE_OK && !h->slot_read.empty())
    for (int i = 0; i < n; ++i) h->slot_read[static_cast<size_t>(layer) * h->S + sl[i]] = -1;
  return st;
}

MOE_API int moe_lfu_wait(void* event, int timeout_ms) {
  if (!event) return moe::fail(MOE_ERR_INVALID_ARG, "lfu_wait: NULL event");
  return wait_event(static_cast<cudaEvent_t>(event), timeout_ms);
}

MOE_API int moe_lfu_get_log(moe_lfu* h, int32_t* buf, size_t cap_records, size_t* n_records) {
  if (!h || !n_records) return moe::fail(MOE_ERR_INVALID_ARG, "lfu_get_log: NULL");
  const size_t n = h->log.size() / 5;
  *n_records = n;
  if (buf) std::memcpy(buf, h->log.data(), sizeof(int32_t) * 5 * (n < cap_records ? n : cap_records));
  return MOE_OK;
}

MOE_API int moe_lfu_stats(moe_lfu* h, int64_t* hits, int64_t* misses, int64_t* bytes_copied) {
  if (!h) return moe::fail(MOE_ERR_INVALID_ARG, "lfu_stats: NULL");
  int64_t nh = 0, nm = 0;
  for (size_t i = 0; i + 4 < h->log.size(); i += 5) {      // prefetch records (hit = 2) are neither
    if (h->log[i + 3] == 1) ++nh;
    else if (h->log[i + 3] == 0) ++nm;
  }
  if (hits) *hits = nh;
  if (misses) *misses = nm;
  if (bytes_copied) *bytes_copied = h->bytes_copied;
  return MOE_OK;
}

MOE_API int moe_lfu_set_fault(moe_lfu* h, int kind, int after_n) {
  if (!h || kind < 0 || kind > 2) return moe::fail(MOE_ERR_INVALID_ARG, "lfu_set_fault: bad arguments");
  h->fault_kind = kind;
  h->fault_after = after_n;
  return MOE_OK;
}

MOE_API int moe_lfu_set_prefetch(moe_lfu* h, int per_call) {
  if (!h || per_call < 0 || per_call > h->S) return moe::fail(MOE_ERR_INVALID_ARG, "lfu_set_prefetch: bad arguments");
  h->prefetch_n = per_call;
  return MOE_OK;
}

MOE_API int moe_lfu_plan_prefetch(moe_lfu* h, int layer, int per_call, int32_t* ids_out, int32_t* slots_out,
                                  int* n_out) {
  if (!h || !n_out || (per_call > 0 && (!ids_out || !slots_out)))
    return moe::fail(MOE_ERR_INVALID_ARG, "lfu_plan_prefetch: NULL");
  if (layer < 0 || layer >= h->L || per_call < 0 || per_call > h->S)
    return moe::fail(MOE_ERR_INVALID_ARG, "lfu_plan_prefetch: bad arguments");
  std::vector<int32_t> ids, slots;
  plan_prefetch(h, layer, per_call, ids, slots);
  for (size_t i = 0; i < ids.size(); ++i) { ids_out[i] = ids[i]; slots_out[i] = slots[i]; }
  *n_out = static_cast<int>(ids.size());
  return MOE_OK;
}

MOE_API int moe_lfu_destroy(moe_lfu* h) {
  if (!h) return MOE_OK;
  for (cudaEvent_t e : h->consumed) if (e) { cudaEventSynchronize(e); cudaEventDestroy(e); }
  for (cudaEvent_t e : {h->done, h->idx_ready, h->stage_free}) if (e) { cudaEventSynchronize(e); cudaEventDestroy(e); }
  for (cudaEvent_t e : h->read_ev) if (e) { cudaEventSynchronize(e); cudaEventDestroy(e); }
  if (h->pin_idx) cudaFreeHost(h->pin_idx);
  if (h->pin_act) cudaFreeHost(h->pin_act);
  for (size_t l = 0; l < h->mirror.size(); ++l) {
    if (h->mirror_ev[l]) {
      cudaEventSynchronize(h->mirror_ev[l]);
      cudaEventDestroy(h->mirror_ev[l]);
    }
    if (h->mirror[l]) cudaFreeHost(h->mirror[l]);
  }
  delete h;
  return MOE_OK;
}

}  // extern "C"

// ------------------------------------------------------------ streamed layer
extern "C" {

MOE_API size_t moe_streamed_workspace_size(int T, int H, int I, int Is, int E, int k) {
  return moe_layer_workspace_size(T, H, I, Is, E, k) + 256 + sizeof(int32_t) * (E + 1) * (E + 1);
}

MOE_API int moe_streamed_layer_forward(moe_lfu* h, int layer, float* hres, int T, int H, int I, int Is, int E, int k,
                                       const moe_qmat* router, const float* bias, int bias_per_row,
                                       const moe_qmat* shared, void** dev_table, uint16_t* x_out, uint16_t* y_out,
                                       int32_t* idx_out, void* ws, size_t ws_bytes, int flags, void* main_stream,
                                       void* side_stream, int timeout_ms) {
  if (!h || !h->pool) return moe::fail(MOE_ERR_INVALID_ARG, "streamed: handle has no slot pool");
  if (!hres || !dev_table || !ws || T < 0 || k < 1 || k > 8 || E != h->E || layer < 0 || layer >= h->L)
    return moe::fail(MOE_ERR_INVALID_ARG, "streamed: bad arguments");
  if (T == 0) return MOE_OK;
  if (ws_bytes < moe_streamed_workspace_size(T, H, I, Is, E, k))
    return moe::fail(MOE_ERR_INVALID_ARG, "streamed: workspace too small");
  cudaStream_t ms = static_cast<cudaStream_t>(main_stream);
  // workspace: the per-layer buffers (same carving as moe_layer_forward), then device active lists
  auto al = [](size_t n) { return (n + 255) / 256 * 256; };
  char* p = static_cast<char*>(ws);
  auto take = [&](size_t n) { char* q = p; p += al(n); return q; };
  uint16_t* x = reinterpret_cast<uint16_t*>(take(static_cast<size_t>(T) * H * 2));
  int32_t* idx = reinterpret_cast<int32_t*>(take(static_cast<size_t>(T) * k * 4));
  float* gates = reinterpret_cast<float*>(take(static_cast<size_t>(T) * k * 4));
  int32_t* offsets = reinterpret_cast<int32_t*>(take(static_cast<size_t>(E + 1) * 4));
  int32_t* pairs = reinterpret_cast<int32_t*>(take(static_cast<size_t>(T) * k * 4));
  int32_t* active = reinterpret_cast<int32_t*>(take(static_cast<size_t>(E) * 4));
  int32_t* n_active = reinterpret_cast<int32_t*>(take(4));
  float* y_pairs = reinterpret_cast<float*>(take(static_cast<size_t>(T) * k * H * 4));
  float* ysh = reinterpret_cast<float*>(take(static_cast<size_t>(T) * H * 4));
  const size_t ews = moe_expert_workspace_size(T, H, I, k);
  void* ew = take(ews);
  const size_t sws = moe_shared_workspace_size(T, H, Is);
  void* sw = take(sws);
  int32_t* dev_act = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (E + 1) * (E + 1)));
  (void)active; (void)n_active;
  int st;
  if ((st = moe_rmsnorm(hres, T, H, 1e-6f, x, ms))) return st;
  if ((st = moe_router_topk(x, T, H, router, bias, bias_per_row, E, k, idx, gates, nullptr, ms))) return st;
  if ((st = moe_bucket(idx, T, k, E, offsets, pairs, active, n_active, ms))) return st;
  // the routing to the host (pinned), then the shared expert, which overlaps the copies
  if (h->cap_rows < T) {
    if (h->pin_idx) { cudaStreamSynchronize(ms); cudaFreeHost(h->pin_idx); h->pin_idx = nullptr; }
    void* q = nullptr;
    if ((st = moe::cuda_check(cudaHostAlloc(&q, sizeof(int32_t) * T * 8, 0), "streamed: pinned idx"))) return st;
    h->pin_idx = static_cast<int32_t*>(q);
    h->cap_rows = T;
  }
  if ((st = moe::cuda_check(cudaMemcpyAsync(h->pin_idx, idx, sizeof(int32_t) * T * k, cudaMemcpyDeviceToHost, ms),
                            "streamed: idx to host")))
    return st;
  if ((st = moe::cuda_check(cudaEventRecord(h->idx_ready, ms), "streamed: record"))) return st;
  if ((st = moe_shared_forward(x, T, H, Is, shared, ysh, sw, sws, flags, ms))) return st;
  if ((st = wait_event(h->idx_ready, timeout_ms))) return st;
  // the routing follows every earlier step's kernels on the main stream, when
  // they were issued on this same stream; readers recorded on another stream
  // are forgotten (their slots then wait for the layer's last kernels)
  if (ms == h->read_stream) {
    h->read_done = h->read_seq;
  } else {
    h->read_stream = ms;
    std::fill(h->slot_read.begin(), h->slot_read.end(), -1);
  }
  // steps: one token's ids in selection order, or the chunk's distinct experts,
  // resident ones first (ascending), then the rest (ascending), k at a time
  std::vector<std::vector<int32_t>> steps;
  if (T == 1) {
    steps.emplace_back(h->pin_idx, h->pin_idx + k);
  } else {
    std::vector<char> seen(E, 0);
    for (int i = 0; i < T * k; ++i) seen[h->pin_idx[i]] = 1;
    std::vector<char> res(E, 0);
    for (int s2 = 0; s2 < h->S; ++s2) {
      const int e = h->expert[static_cast<size_t>(layer) * h->S + s2];
      if (e >= 0) res[e] = 1;
    }
    std::vector<int32_t> order;
    for (int e = 0; e < E; ++e) if (seen[e] && res[e]) order.push_back(e);
    for (int e = 0; e < E; ++e) if (seen[e] && !res[e]) order.push_back(e);
    for (size_t i = 0; i < order.size(); i += k)
      steps.emplace_back(order.begin() + i, order.begin() + std::min(order.size(), i + static_cast<size_t>(k)));
  }
  // the pinned active-list staging of the previous call must have been consumed
  if ((st = wait_event(h->stage_free, timeout_ms))) return st;
  // every step of this call is one transaction: a failure in any of them
  // undoes the plan of all of them (a repeated call then plans the same way)
  txn_begin(h, layer);
  // a failed call still marks its pinned staging (the active lists already
  // queued for copying) so that the next call waits before reusing it
  auto abort_call = [&](int status) {
    cudaEventRecord(h->stage_free, ms);
    return txn_rollback(h, status);
  };
  for (size_t g = 0; g < steps.size(); ++g) {
    const auto& ids = steps[g];
    const int n = static_cast<int>(ids.size());
    std::vector<int32_t> sl(n);
    if ((st = lfu_step_impl(h, layer, ids.data(), n, side_stream, h->consumed[layer], true, h->done, dev_table,
                            timeout_ms, sl.data())))
      return abort_call(st);
    if ((st = moe::cuda_check(cudaStreamWaitEvent(ms, h->done, 0), "streamed: wait copies"))) return abort_call(st);
    int32_t* pa = h->pin_act + g * (E + 1);
    pa[0] = n;
    for (int i = 0; i < n; ++i) pa[1 + i] = ids[i];
    int32_t* da = dev_act + g * (E + 1);
    if ((st = moe::cuda_check(cudaMemcpyAsync(da, pa, sizeof(int32_t) * (n + 1), cudaMemcpyHostToDevice, ms),
                              "streamed: active list")))
      return abort_call(st);
    if ((st = moe_expert_forward(x, T, H, I, E, k, const_cast<const void* const*>(dev_table), offsets, pairs, da + 1,
                                 da, y_pairs, ew, ews, flags, ms)))
      return abort_call(st);
    if ((st = moe::cuda_check(cudaEventRecord(h->consumed[layer], ms), "streamed: record consumed")))
      return abort_call(st);
    // this step's kernels read its slots; the last step's event is never
    // waited for (the next call's routing wait covers it), so it is not
    // recorded
    const int r = static_cast<int>(h->read_seq % moe_lfu::READ_RING);
    if (g + 1 < steps.size() &&
        (st = moe::cuda_check(cudaEventRecord(h->read_ev[r], ms), "streamed: record slot readers")))
      return abort_call(st);
    for (int i = 0; i < n; ++i) h->slot_read[static_cast<size_t>(layer) * h->S + sl[i]] = h->read_seq;
    ++h->read_seq;
  }
  // lookahead prefetch (part of the call's transaction): the copies follow
  // the call's expert kernels on the side stream, since a victim slot may be
  // one they read
  if (h->prefetch_n > 0) {
    std::vector<int32_t> pids, pslots;
    plan_prefetch(h, layer, h->prefetch_n, pids, pslots);
    if (!pids.empty() &&
        (st = moe::cuda_check(cudaStreamWaitEvent(static_cast<cudaStream_t>(side_stream), h->consumed[layer], 0),
                              "streamed: prefetch wait")))
      return abort_call(st);
    const size_t base = static_cast<size_t>(layer) * h->S;
    for (size_t i = 0; i < pids.size(); ++i) {
      ++h->copies;
      if (h->fault_kind == MOE_LFU_FAULT_COPY_FAILS && h->fault_after >= 0 && h->copies > h->fault_after)
        return abort_call(moe::fail(MOE_ERR_CUDA, "streamed: injected copy failure (copy %ld)", h->copies));
      unsigned char* slot = h->pool + (base + pslots[i]) * h->slot_stride;
      const void* src = h->host_blobs[static_cast<size_t>(layer) * h->E + pids[i]];
      if ((st = moe::cuda_check(cudaMemcpyAsync(slot, src, h->blob_bytes, cudaMemcpyHostToDevice,
                                                static_cast<cudaStream_t>(side_stream)), "streamed: prefetch copy")))
        return abort_call(st);
      h->txn_written.push_back(pslots[i]);
      h->dirty[base + pslots[i]] = 0;
      h->bytes_copied += static_cast<int64_t>(h->blob_bytes);
    }
  }
  txn_commit(h);
  if ((st = moe::cuda_check(cudaEventRecord(h->stage_free, ms), "streamed: record staging"))) return st;
  if ((st = moe_combine(y_pairs, gates, ysh, T, H, k, y_out, hres, ms))) return st;
  if (x_out && (st = moe::cuda_check(cudaMemcpyAsync(x_out, x, static_cast<size_t>(T) * H * 2,
                                                     cudaMemcpyDeviceToDevice, ms), "streamed: x_out")))
    return st;
  if (idx_out && (st = moe::cuda_check(cudaMemcpyAsync(idx_out, idx, static_cast<size_t>(T) * k * 4,
                                                       cudaMemcpyDeviceToDevice, ms), "streamed: idx_out")))
    return st;
  return MOE_OK;
}

}  // extern "C"
