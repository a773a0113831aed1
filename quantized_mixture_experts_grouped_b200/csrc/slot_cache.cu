// GPU-resident expert slot cache refilled from pinned host memory ("Every Expert Counts:
// ExactMoE for Memory-Efficient W4A16 Inference", Abstract: experts stored in pinned host
// memory and executed through a configurable GPU-resident slot cache).
//
// Host-side LRU bookkeeping; refills are cudaMemcpyAsync copies on a caller-given copy stream,
// ordered after the last kernel that read the pool through an event. A routed set larger than
// the pool runs in waves; the FFN of each wave sees only that wave's experts (others -1) and
// accumulates into the workspace's fp32 accumulator, the last wave writing the bf16 output.
#include <algorithm>
#include <cstring>
#include <vector>

#include "common.cuh"

struct moe_slot_cache {
  int E, S, H, I;
  const uint8_t* bank_w13; const uint16_t* bank_s13;
  const uint8_t* bank_w2; const uint16_t* bank_s2;
  uint8_t* pool_w13; uint16_t* pool_s13;
  uint8_t* pool_w2; uint16_t* pool_s2;
  size_t w13_bytes, s13_bytes, w2_bytes, s2_bytes;   // per expert
  std::vector<int32_t> slot_expert;                  // [S], -1 free
  std::vector<int64_t> last_used;                    // [S]
  int64_t clock = 0;
  cudaEvent_t wave_done[2] = {nullptr, nullptr};    // FFN of the last even / odd wave done
  cudaEvent_t loaded = nullptr;
  cudaStream_t copy2 = nullptr;                      // second refill stream (two copies in flight
  cudaEvent_t fork = nullptr, join = nullptr;        // on the link), forked from and joined to the
                                                     // caller's copy stream per wave
  int32_t* wave_tables = nullptr;                    // host copies of every wave's table, pinned
                                                     // ([E + 1][E]: the uploads stay asynchronous)
  std::vector<int32_t> idx_host;
  int fail_copies_after = -1;                        // test hook: fail the n-th next copy
  bool dry_run = false;                              // test hook: plan and commit, copy nothing
};

namespace moe {

// Test hook: makes the n-th next refill copy (0 = the next one) of this cache report failure
// as if cudaMemcpyAsync had returned an error; -1 disables.
MOE_API void moe_slot_cache_fail_copy_after(moe_slot_cache* c, int n) {
  if (c) c->fail_copies_after = n;
}

// Test hook: with dry != 0 refills are planned and committed exactly as usual but no copy is
// issued, so the replacement policy runs on a machine without a GPU; 0 restores the copies.
MOE_API void moe_slot_cache_dry_run(moe_slot_cache* c, int dry) {
  if (c) c->dry_run = dry != 0;
}

namespace {

cudaError_t refill_copy(moe_slot_cache* c, void* dst, const void* src, size_t bytes, cudaStream_t s) {
  if (c->fail_copies_after == 0) {
    c->fail_copies_after = -1;
    return cudaErrorInvalidValue;
  }
  if (c->fail_copies_after > 0) c->fail_copies_after--;
  if (c->dry_run) return cudaSuccess;
  return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, s);
}

// The events that order refills against the FFN launches of moe_slot_cache_layer, created on
// its first call (creating the cache itself makes no CUDA call).
int ensure_events(moe_slot_cache* c) {
  for (cudaEvent_t& e : c->wave_done)
    if (!e)
      if (int rc = check_cuda(cudaEventCreateWithFlags(&e, cudaEventDisableTiming), "event create")) return rc;
  if (!c->loaded)
    if (int rc = check_cuda(cudaEventCreateWithFlags(&c->loaded, cudaEventDisableTiming), "event create"))
      return rc;
  if (!c->wave_tables)
    if (int rc = check_cuda(cudaHostAlloc(reinterpret_cast<void**>(&c->wave_tables),
                                          sizeof(int32_t) * (size_t)c->E * (c->E + 1), cudaHostAllocDefault),
                            "pinned wave tables"))
      return rc;
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

MOE_API int moe_slot_cache_create(int E, int S, int H, int I, const uint8_t* bank_w13, const uint16_t* bank_s13,
                                  const uint8_t* bank_w2, const uint16_t* bank_s2, uint8_t* pool_w13,
                                  uint16_t* pool_s13, uint8_t* pool_w2, uint16_t* pool_s2, moe_slot_cache** out) {
  if (!out) return fail(MOE_ERR_ARG, "moe_slot_cache_create: null out");
  *out = nullptr;
  if (E < 1 || S < 1 || E > kMaxExperts) return fail(MOE_ERR_ARG, "moe_slot_cache_create: E=%d S=%d", E, S);
  if (H <= 0 || I <= 0 || H % kRowBlock || I % kRowBlock)
    return fail(MOE_ERR_SHAPE, "moe_slot_cache_create: H=%d I=%d must be multiples of 128", H, I);
  if (!bank_w13 || !bank_s13 || !bank_w2 || !bank_s2 || !pool_w13 || !pool_s13 || !pool_w2 || !pool_s2)
    return fail(MOE_ERR_ARG, "moe_slot_cache_create: null bank or pool pointer");
  moe_slot_cache* c = new moe_slot_cache();
  c->E = E; c->S = S; c->H = H; c->I = I;
  c->bank_w13 = bank_w13; c->bank_s13 = bank_s13; c->bank_w2 = bank_w2; c->bank_s2 = bank_s2;
  c->pool_w13 = pool_w13; c->pool_s13 = pool_s13; c->pool_w2 = pool_w2; c->pool_s2 = pool_s2;
  c->w13_bytes = (size_t)2 * I * H / 2;
  c->s13_bytes = sizeof(uint16_t) * (size_t)2 * I * (H / kGroup);
  c->w2_bytes = (size_t)H * I / 2;
  c->s2_bytes = sizeof(uint16_t) * (size_t)H * (I / kGroup);
  c->slot_expert.assign(S, -1);
  c->last_used.assign(S, 0);
  *out = c;
  return MOE_OK;
}

MOE_API void moe_slot_cache_destroy(moe_slot_cache* c) {
  if (!c) return;
  for (cudaEvent_t e : c->wave_done)
    if (e) cudaEventDestroy(e);
  if (c->wave_tables) cudaFreeHost(c->wave_tables);
  if (c->fork) cudaEventDestroy(c->fork);
  if (c->join) cudaEventDestroy(c->join);
  if (c->copy2) cudaStreamDestroy(c->copy2);
  if (c->loaded) cudaEventDestroy(c->loaded);
  delete c;
}

MOE_API int64_t moe_slot_cache_state(const moe_slot_cache* c, int32_t* slot_expert, int64_t* last_used) {
  if (!c) return -1;
  if (slot_expert) std::copy(c->slot_expert.begin(), c->slot_expert.end(), slot_expert);
  if (last_used) std::copy(c->last_used.begin(), c->last_used.end(), last_used);
  return c->clock;
}

MOE_API int slot_table_update(moe_slot_cache* c, uint64_t* needed_mask, int32_t* wave_table, int32_t* misses,
                              int* n_misses, moe_stream_t copy_stream, moe_event_t reuse_ok, moe_event_t loaded) {
  return slot_table_update_ex(c, needed_mask, wave_table, misses, n_misses, copy_stream, reuse_ok, loaded, 0,
                              nullptr);
}

MOE_API int slot_table_update_ex(moe_slot_cache* c, uint64_t* needed_mask, int32_t* wave_table, int32_t* misses,
                                 int* n_misses, moe_stream_t copy_stream, moe_event_t reuse_ok, moe_event_t loaded,
                                 int max_wave, const uint8_t* protect) {
  if (!c || !needed_mask || !wave_table || !misses || !n_misses)
    return fail(MOE_ERR_ARG, "slot_table_update: null pointer");
  const int E = c->E, S = c->S;
  const int cap = max_wave <= 0 ? S : max_wave;
  if (cap > S) return fail(MOE_ERR_ARG, "slot_table_update: max_wave %d exceeds the %d slots", max_wave, S);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(copy_stream);
  auto needed = [&](int e) { return (needed_mask[e >> 6] >> (e & 63)) & 1ull; };
  std::vector<int> slot_of(E, -1);
  for (int s = 0; s < S; ++s)
    if (c->slot_expert[s] >= 0) slot_of[c->slot_expert[s]] = s;
  std::vector<int> hits, miss;
  for (int e = 0; e < E; ++e)
    if (needed(e)) (slot_of[e] >= 0 ? hits : miss).push_back(e);
  // the wave: the first min(cap, hits) hits, then misses up to cap, both in ascending id
  std::vector<char> in_wave(E, 0);
  const int n_hit = std::min(cap, (int)hits.size());
  for (int i = 0; i < n_hit; ++i) in_wave[hits[i]] = 1;
  const int n_new = std::min(cap - n_hit, (int)miss.size());
  for (int i = 0; i < n_new; ++i) in_wave[miss[i]] = 1;

  // plan on a copy of the state so that a failed copy can leave the committed state alone
  std::vector<int32_t> se = c->slot_expert;
  std::vector<int> loads_e, loads_s;
  for (int i = 0; i < n_new; ++i) {
    const int e = miss[i];
    int pick = -1;
    for (int s = 0; s < S && pick < 0; ++s)
      if (se[s] < 0) pick = s;
    if (pick < 0)   // least recently used, neither protected nor holding an expert still needed
      for (int s = 0; s < S; ++s) {
        if (se[s] >= 0 && (in_wave[se[s]] || needed(se[s]))) continue;
        if (protect && protect[s]) continue;
        if (pick < 0 || c->last_used[s] < c->last_used[pick]) pick = s;
      }
    if (pick < 0)
      return fail(MOE_ERR_ARG, "slot_table_update: no evictable slot (protected slots and needed experts hold all)");
    if (se[pick] >= 0) slot_of[se[pick]] = -1;
    se[pick] = e;
    slot_of[e] = pick;
    loads_e.push_back(e);
    loads_s.push_back(pick);
  }

  if (!loads_e.empty() && reuse_ok)
    if (int rc = check_cuda(cudaStreamWaitEvent(cs, reinterpret_cast<cudaEvent_t>(reuse_ok), 0),
                            "slot_table_update: wait for pool reuse"))
      return rc;
  // Two refill streams keep two copies on the link at once. For this copy pattern one stream
  // measured 39.0 GB/s and two 43.6 GB/s on one B200 machine (four no more than two); where one
  // stream already reaches ~44 GB/s the second changes nothing. The second stream is forked
  // from the copy stream (so it waits for everything the copy stream waits for) and joined back
  // before `loaded`. Experts alternate between the two; the issue order of the copies is
  // unchanged.
  cudaStream_t cs2 = cs;
  if (loads_e.size() >= 2 && !c->dry_run) {
    if (!c->copy2) {
      if (int rc = check_cuda(cudaStreamCreateWithFlags(&c->copy2, cudaStreamNonBlocking), "second refill stream"))
        return rc;
      if (int rc = check_cuda(cudaEventCreateWithFlags(&c->fork, cudaEventDisableTiming), "event create")) return rc;
      if (int rc = check_cuda(cudaEventCreateWithFlags(&c->join, cudaEventDisableTiming), "event create")) return rc;
    }
    if (int rc = check_cuda(cudaEventRecord(c->fork, cs), "slot_table_update: fork")) return rc;
    if (int rc = check_cuda(cudaStreamWaitEvent(c->copy2, c->fork, 0), "slot_table_update: fork")) return rc;
    cs2 = c->copy2;
  }
  for (size_t i = 0; i < loads_e.size(); ++i) {
    const size_t e = loads_e[i], s = loads_s[i];
    cudaStream_t st = (i & 1) ? cs2 : cs;
    cudaError_t err = refill_copy(c, c->pool_w13 + s * c->w13_bytes, c->bank_w13 + e * c->w13_bytes, c->w13_bytes, st);
    if (err == cudaSuccess)
      err = refill_copy(c, reinterpret_cast<char*>(c->pool_s13) + s * c->s13_bytes,
                        reinterpret_cast<const char*>(c->bank_s13) + e * c->s13_bytes, c->s13_bytes, st);
    if (err == cudaSuccess)
      err = refill_copy(c, c->pool_w2 + s * c->w2_bytes, c->bank_w2 + e * c->w2_bytes, c->w2_bytes, st);
    if (err == cudaSuccess)
      err = refill_copy(c, reinterpret_cast<char*>(c->pool_s2) + s * c->s2_bytes,
                        reinterpret_cast<const char*>(c->bank_s2) + e * c->s2_bytes, c->s2_bytes, st);
    if (err != cudaSuccess) {
      // slots written so far no longer hold what the committed state says: mark them free
      for (size_t j = 0; j <= i; ++j) c->slot_expert[loads_s[j]] = -1;
      *n_misses = 0;
      if (cs2 != cs && cudaEventRecord(c->join, cs2) == cudaSuccess)   // keep the copy stream after both
        cudaStreamWaitEvent(cs, c->join, 0);
      return fail(MOE_ERR_CUDA, "slot_table_update: refill of expert %zu into slot %zu failed: %s", e, s,
                  cudaGetErrorString(err));
    }
  }
  if (cs2 != cs) {
    if (int rc = check_cuda(cudaEventRecord(c->join, cs2), "slot_table_update: join")) return rc;
    if (int rc = check_cuda(cudaStreamWaitEvent(cs, c->join, 0), "slot_table_update: join")) return rc;
  }
  if (loaded)
    if (int rc = check_cuda(cudaEventRecord(reinterpret_cast<cudaEvent_t>(loaded), cs), "slot_table_update: record"))
      return rc;

  c->slot_expert = se;
  for (int e = 0; e < E; ++e) {
    wave_table[e] = in_wave[e] ? slot_of[e] : -1;
    if (in_wave[e]) {
      c->last_used[slot_of[e]] = c->clock;
      needed_mask[e >> 6] &= ~(1ull << (e & 63));
    }
  }
  c->clock += 1;
  for (size_t i = 0; i < loads_e.size(); ++i) misses[i] = loads_e[i];
  *n_misses = (int)loads_e.size();
  return MOE_OK;
}

MOE_API int moe_slot_cache_layer(moe_slot_cache* c, const uint16_t* x, const uint16_t* logits, int T, int k,
                                 int32_t* idx, float* wts, int32_t* wave_tables, void* workspace,
                                 size_t workspace_bytes, uint16_t* out, int path, moe_stream_t stream,
                                 moe_stream_t copy_stream, int* n_waves, int* n_loads) {
  if (!c || !wave_tables || !n_waves || !n_loads) return fail(MOE_ERR_ARG, "moe_slot_cache_layer: null pointer");
  if (T < 0 || k < 1 || k > c->E) return fail(MOE_ERR_ARG, "moe_slot_cache_layer: bad sizes");
  *n_waves = 0;
  *n_loads = 0;
  if (T == 0) return MOE_OK;
  if (int rc = ensure_events(c)) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int E = c->E;
  if (int rc = moe_route_topk(logits, T, E, k, idx, wts, stream)) return rc;
  c->idx_host.resize((size_t)T * k);
  if (int rc = check_cuda(cudaMemcpyAsync(c->idx_host.data(), idx, sizeof(int32_t) * T * k, cudaMemcpyDeviceToHost, s),
                          "moe_slot_cache_layer: read routed experts"))
    return rc;
  if (int rc = check_cuda(cudaStreamSynchronize(s), "moe_slot_cache_layer: sync")) return rc;
  uint64_t mask[kMaxExperts / 64] = {0, 0, 0, 0};
  for (int32_t e : c->idx_host) {
    if (e < 0 || e >= E) return fail(MOE_ERR_ARG, "moe_slot_cache_layer: routed expert %d out of range", e);
    mask[e >> 6] |= 1ull << (e & 63);
  }
  // Waves overlap their refills with the FFN of the wave before: with two or more slots a wave
  // holds at most S/2 experts and may not overwrite the slots of the wave before it (still
  // running), so its copies only wait for the wave two back. With one slot every refill waits
  // for the wave before. The first wave waits for nothing: the host synchronised above, after
  // every earlier kernel of this stream. The device tables are reused in turn: their uploads
  // run on the compute stream, after the FFN that read the previous contents.
  const int S = c->S;
  const bool overlap = S >= 2;
  const int cap = overlap ? S / 2 : S, n_dev_tables = (E + S - 1) / S + 1;
  std::vector<int32_t> miss(S);
  std::vector<uint8_t> prot(S, 0);
  int wave = 0;
  auto any = [&]() { return (mask[0] | mask[1] | mask[2] | mask[3]) != 0; };
  while (any()) {
    if (wave >= E) return fail(MOE_ERR_ARG, "moe_slot_cache_layer: too many waves (internal)");
    int32_t* table_h = c->wave_tables + (size_t)wave * E;
    int nm = 0;
    cudaEvent_t reuse = nullptr;
    if (overlap && wave >= 2) reuse = c->wave_done[wave & 1];
    if (!overlap && wave >= 1) reuse = c->wave_done[(wave - 1) & 1];
    if (int rc = slot_table_update_ex(c, mask, table_h, miss.data(), &nm, copy_stream,
                                      reinterpret_cast<moe_event_t>(reuse), reinterpret_cast<moe_event_t>(c->loaded),
                                      cap, overlap ? prot.data() : nullptr))
      return rc;
    *n_loads += nm;
    int32_t* table_d = wave_tables + (size_t)(wave % n_dev_tables) * E;
    if (int rc = check_cuda(cudaMemcpyAsync(table_d, table_h, sizeof(int32_t) * E, cudaMemcpyHostToDevice, s),
                            "moe_slot_cache_layer: upload wave table"))
      return rc;
    if (int rc = check_cuda(cudaStreamWaitEvent(s, c->loaded, 0), "moe_slot_cache_layer: wait refill")) return rc;
    const bool last = !any();
    // wave 0 stores its sum into the fp32 accumulator without reading it (no zero precondition
    // on the accumulator, even after an earlier call ended early); later waves add to it; the
    // last wave writes out
    const int flags = (path & MOE_PATH_MASK) | (wave > 0 ? MOE_FLAG_ACCUMULATE : 0);
    if (int rc = moe_w4a16_ffn(x, T, c->H, c->I, E, k, idx, wts, c->pool_w13, c->pool_s13, c->pool_w2, c->pool_s2,
                               table_d, workspace, workspace_bytes, last ? out : nullptr, flags, stream))
      return rc;
    if (int rc = check_cuda(cudaEventRecord(c->wave_done[wave & 1], s), "moe_slot_cache_layer: record")) return rc;
    std::fill(prot.begin(), prot.end(), 0);
    for (int e = 0; e < E; ++e)
      if (table_h[e] >= 0) prot[table_h[e]] = 1;
    ++wave;
  }
  *n_waves = wave;
  return MOE_OK;
}
