// Slot manager of the adapter pool: which adapter lives in which slot, and
// which slot to reuse when a new adapter must be brought in.
//
// Page "LoRA Adapters at Serve Time with vLLM Multi-LoRA", section "The
// Inference Mechanism: A Worked Scenario", step "Eviction": when every slot
// is taken, the least recently used adapter is swapped out to make room.
// Page "Multi-LoRA Serving Architecture ... (2026)", section "An
// adapter-cache LRU simulator": an LRU over a fixed slot count, measured by its
// hit rate; the same page notes that the slots of a batching engine hold the
// adapters of the running batch, which this manager models with pin counts:
// a pinned slot is never chosen for eviction.
//
// Host bookkeeping only: the manager never touches device memory.  The caller
// moves the weights (lora_pool_evict / lora_pool_load on its own stream), so
// a load for the next batch can run on a second stream while the current
// batch computes.
#include <cstdint>
#include <mutex>
#include <new>
#include <unordered_map>
#include <vector>

#include "lora.h"

namespace {

struct SlotEntry {
    int64_t key = -1;   // adapter held, -1 = empty
    int pins = 0;
    int prev = -1;      // recency list: toward the least recently used end
    int next = -1;      // toward the most recently used end
};

}  // namespace

struct lora_slot_cache_s {
    std::mutex mu;
    std::vector<SlotEntry> slot;
    std::unordered_map<int64_t, int> where;   // key -> slot
    std::vector<int> empty;                    // empty slots, lowest id last
    int lru = -1;                              // least recently used resident slot
    int mru = -1;                              // most recently used resident slot
    int64_t hits = 0, misses = 0, evictions = 0;

    void unlink(int s) {
        SlotEntry &e = slot[s];
        if (e.prev >= 0) slot[e.prev].next = e.next; else lru = e.next;
        if (e.next >= 0) slot[e.next].prev = e.prev; else mru = e.prev;
        e.prev = e.next = -1;
    }
    void push_mru(int s) {
        SlotEntry &e = slot[s];
        e.prev = mru;
        e.next = -1;
        if (mru >= 0) slot[mru].next = s; else lru = s;
        mru = s;
    }
};

extern "C" int lora_slot_cache_create(int num_slots, lora_slot_cache_t *out) {
    if (!out || num_slots < 1 || num_slots > LORA_MAX_SLOTS) return LORA_ERR_INVALID_ARG;
    lora_slot_cache_s *c = new (std::nothrow) lora_slot_cache_s();
    if (!c) return LORA_ERR_INVALID_ARG;
    c->slot.resize((size_t)num_slots);
    c->empty.reserve((size_t)num_slots);
    for (int s = num_slots - 1; s >= 0; --s) c->empty.push_back(s);
    *out = c;
    return LORA_OK;
}

extern "C" int lora_slot_cache_destroy(lora_slot_cache_t c) {
    if (!c) return LORA_ERR_INVALID_ARG;
    delete c;
    return LORA_OK;
}

extern "C" int lora_slot_cache_acquire(lora_slot_cache_t c, int64_t key, int pin, int *slot_out, int *hit_out,
                                       int64_t *evicted_key_out) {
    if (!c || key < 0 || !slot_out || !hit_out || !evicted_key_out) return LORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(c->mu);
    *evicted_key_out = -1;
    auto it = c->where.find(key);
    int s;
    if (it != c->where.end()) {
        s = it->second;
        c->unlink(s);
        *hit_out = 1;
        ++c->hits;
    } else {
        if (!c->empty.empty()) {
            s = c->empty.back();
            c->empty.pop_back();
        } else {
            s = c->lru;   // the least recently used slot that no batch holds
            while (s >= 0 && c->slot[s].pins > 0) s = c->slot[s].next;
            if (s < 0) return LORA_ERR_ALL_PINNED;
            c->unlink(s);
            *evicted_key_out = c->slot[s].key;
            c->where.erase(c->slot[s].key);
            ++c->evictions;
        }
        c->slot[s].key = key;
        c->where[key] = s;
        *hit_out = 0;
        ++c->misses;
    }
    c->push_mru(s);
    if (pin) ++c->slot[s].pins;
    *slot_out = s;
    return LORA_OK;
}

extern "C" int lora_slot_cache_unpin(lora_slot_cache_t c, int slot) {
    if (!c) return LORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(c->mu);
    if (slot < 0 || slot >= (int)c->slot.size()) return LORA_ERR_BAD_SLOT;
    if (c->slot[slot].pins <= 0) return LORA_ERR_INVALID_ARG;
    --c->slot[slot].pins;
    return LORA_OK;
}

extern "C" int lora_slot_cache_invalidate(lora_slot_cache_t c, int slot) {
    if (!c) return LORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(c->mu);
    if (slot < 0 || slot >= (int)c->slot.size()) return LORA_ERR_BAD_SLOT;
    SlotEntry &e = c->slot[slot];
    if (e.key < 0) return LORA_OK;
    if (e.pins > 0) return LORA_ERR_ALL_PINNED;
    c->unlink(slot);
    c->where.erase(e.key);
    e.key = -1;
    c->empty.push_back(slot);
    return LORA_OK;
}

extern "C" int lora_slot_cache_lookup(lora_slot_cache_t c, int64_t key, int *slot_out) {
    if (!c || !slot_out) return LORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(c->mu);
    auto it = c->where.find(key);
    *slot_out = it == c->where.end() ? -1 : it->second;
    return LORA_OK;
}

extern "C" int lora_slot_cache_stats(lora_slot_cache_t c, int64_t *hits, int64_t *misses, int64_t *evictions) {
    if (!c || !hits || !misses || !evictions) return LORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(c->mu);
    *hits = c->hits;
    *misses = c->misses;
    *evictions = c->evictions;
    return LORA_OK;
}
