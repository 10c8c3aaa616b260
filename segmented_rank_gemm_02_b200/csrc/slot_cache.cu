// slot_cache.cu -- mlora_slot_cache: host-side adapter cache over the slots of a pool.
//
// Which adapter (a caller-chosen 64-bit id) each slot holds, how many in-flight
// batches pin it, and least-recently-used order among the unpinned slots.  A miss
// takes a never-used slot first, then the least recently released unpinned one; a
// pinned slot is never evicted (page "Multi-LoRA Serving: adapter batching", section
// "Eviction cannot look only at LRU").  Host code only: no device memory, no CUDA
// calls.  Every entry point takes the cache's mutex.
#include <cstdint>
#include <list>
#include <mutex>
#include <new>
#include <unordered_map>
#include <vector>

#include "mlora.h"

namespace {
constexpr uint64_t kNone = UINT64_MAX;
}

struct mlora_slot_cache {
    mutable std::mutex mu;
    int32_t n = 0;
    std::vector<uint64_t> id;                       // adapter held by each slot, kNone if empty
    std::vector<int32_t> pins;                      // pins per slot
    std::vector<std::list<int32_t>::iterator> pos;  // position in `lru` (unpinned, used slots)
    std::vector<bool> in_lru;
    std::list<int32_t> lru;                         // front = least recently released
    std::vector<int32_t> fresh;                     // never-used slots (taken from the back)
    std::unordered_map<uint64_t, int32_t> where;    // adapter -> slot
    int64_t hits = 0, misses = 0, evictions = 0;
};

extern "C" {

mlora_status mlora_slot_cache_create(int32_t n_slots, mlora_slot_cache **out)
{
    if (out == nullptr) return MLORA_ERR_INVALID_ARG;
    *out = nullptr;
    if (n_slots <= 0) return MLORA_ERR_INVALID_ARG;
    mlora_slot_cache *c = new (std::nothrow) mlora_slot_cache();
    if (c == nullptr) return MLORA_ERR_OUT_OF_MEMORY;
    try {
        c->n = n_slots;
        c->id.assign(n_slots, kNone);
        c->pins.assign(n_slots, 0);
        c->pos.resize(n_slots);
        c->in_lru.assign(n_slots, false);
        c->fresh.reserve(n_slots);
        for (int32_t s = n_slots - 1; s >= 0; --s) c->fresh.push_back(s);   // slot 0 first
        c->where.reserve((size_t)n_slots * 2);
    } catch (...) {
        delete c;
        return MLORA_ERR_OUT_OF_MEMORY;
    }
    *out = c;
    return MLORA_OK;
}

mlora_status mlora_slot_cache_destroy(mlora_slot_cache *cache)
{
    delete cache;
    return MLORA_OK;
}

mlora_status mlora_slot_cache_acquire(mlora_slot_cache *c, uint64_t adapter_id, int32_t *slot,
                                      int32_t *needs_load, uint64_t *evicted_id)
{
    if (c == nullptr || slot == nullptr || needs_load == nullptr || adapter_id == kNone)
        return MLORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(c->mu);
    auto it = c->where.find(adapter_id);
    if (it != c->where.end()) {
        const int32_t s = it->second;
        if (c->in_lru[s]) {
            c->lru.erase(c->pos[s]);
            c->in_lru[s] = false;
        }
        ++c->pins[s];
        ++c->hits;
        *slot = s;
        *needs_load = 0;
        if (evicted_id) *evicted_id = kNone;
        return MLORA_OK;
    }
    int32_t s;
    if (!c->fresh.empty()) {
        s = c->fresh.back();
        c->fresh.pop_back();
    } else if (!c->lru.empty()) {
        s = c->lru.front();
        c->lru.pop_front();
        c->in_lru[s] = false;
    } else {
        return MLORA_ERR_NO_SLOT;
    }
    const uint64_t old = c->id[s];
    if (old != kNone) {
        c->where.erase(old);
        ++c->evictions;
    }
    try {
        c->where[adapter_id] = s;
    } catch (...) {
        c->id[s] = kNone;   // keep the slot usable for a later miss
        c->pos[s] = c->lru.insert(c->lru.begin(), s);
        c->in_lru[s] = true;
        return MLORA_ERR_OUT_OF_MEMORY;
    }
    c->id[s] = adapter_id;
    c->pins[s] = 1;
    ++c->misses;
    *slot = s;
    *needs_load = 1;
    if (evicted_id) *evicted_id = old;
    return MLORA_OK;
}

mlora_status mlora_slot_cache_release(mlora_slot_cache *c, int32_t slot)
{
    if (c == nullptr || slot < 0 || slot >= c->n) return MLORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(c->mu);
    if (c->pins[slot] <= 0) return MLORA_ERR_INVALID_ARG;
    if (--c->pins[slot] == 0) {
        if (c->id[slot] == kNone) {
            c->pos[slot] = c->lru.insert(c->lru.begin(), slot);   // empty: reuse it first
        } else {
            c->pos[slot] = c->lru.insert(c->lru.end(), slot);
        }
        c->in_lru[slot] = true;
    }
    return MLORA_OK;
}

mlora_status mlora_slot_cache_invalidate(mlora_slot_cache *c, int32_t slot)
{
    if (c == nullptr || slot < 0 || slot >= c->n) return MLORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(c->mu);
    if (c->id[slot] != kNone) {
        c->where.erase(c->id[slot]);
        c->id[slot] = kNone;
    }
    if (c->in_lru[slot]) {   // an empty unpinned slot is the next to be reused
        c->lru.erase(c->pos[slot]);
        c->pos[slot] = c->lru.insert(c->lru.begin(), slot);
    }
    return MLORA_OK;
}

mlora_status mlora_slot_cache_lookup(const mlora_slot_cache *c, uint64_t adapter_id, int32_t *slot)
{
    if (c == nullptr || slot == nullptr) return MLORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(c->mu);
    auto it = c->where.find(adapter_id);
    *slot = it == c->where.end() ? -1 : it->second;
    return MLORA_OK;
}

mlora_status mlora_slot_cache_stats(const mlora_slot_cache *c, int64_t *hits, int64_t *misses,
                                    int64_t *evictions)
{
    if (c == nullptr) return MLORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(c->mu);
    if (hits) *hits = c->hits;
    if (misses) *misses = c->misses;
    if (evictions) *evictions = c->evictions;
    return MLORA_OK;
}

}  // extern "C"
