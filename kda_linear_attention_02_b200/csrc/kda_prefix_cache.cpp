// kda_prefix_cache.cpp -- host-side prefix-reuse directory for the recurrent state.
//
// orkas.ai "Kimi K3 architecture" post, section "비용은 서빙 스택에서 돌아옵니다", prefix-reuse item:
// per-token pages and the per-request fixed state must be restorable at the same boundary, so the
// granularities are decoupled -- a hash every 512 tokens, allocation in 1024-6144-token units, and
// state checkpoints kept sparsely at some hash ends.  This file keeps the hash -> checkpoint directory;
// the states live in a caller-owned device pool filled from kda_chunk_fwd's checkpoints.
//
// Block hashes are chained 64-bit FNV-1a (Fowler-Noll-Vo, variant 1a: for each byte, xor then multiply
// by the 64-bit FNV prime, starting from the 64-bit offset basis).  Eviction is least-recently-used.
#include <cstdint>
#include <cstring>
#include <mutex>
#include <set>
#include <unordered_map>
#include <utility>
#include <vector>

#include "kda.h"

namespace {

constexpr uint64_t kFnvOffset = 14695981039346656037ull;
constexpr uint64_t kFnvPrime = 1099511628211ull;

inline uint64_t fnv1a_bytes(uint64_t h, const unsigned char* p, size_t n) {
    for (size_t i = 0; i < n; ++i) {
        h ^= p[i];
        h *= kFnvPrime;
    }
    return h;
}

inline void le64(uint64_t x, unsigned char* out) {
    for (int i = 0; i < 8; ++i) out[i] = static_cast<unsigned char>(x >> (8 * i));
}

struct Entry {
    uint64_t last_use = 0;
    int32_t slot = -1;
};

}  // namespace

struct kda_prefix_cache {
    int64_t max_blocks;
    int n_slots;
    int unit_blocks;
    uint64_t clock = 0;
    std::unordered_map<uint64_t, Entry> blocks;
    std::set<std::pair<uint64_t, uint64_t>> lru;         // (last_use, hash) of every entry
    std::set<std::pair<uint64_t, uint64_t>> lru_slots;   // (last_use, hash) of entries holding a slot
    std::vector<int32_t> free_slots;
    // Per slot: handed out by an insert whose state copy has not been committed yet, and the number
    // of lookups that named it as a resume point and have not released it.  A slot in either state is
    // never returned by a lookup (pending) nor handed to another entry (pending or pinned).
    std::vector<uint8_t> pending;
    std::vector<int32_t> pins;
    std::vector<uint64_t> owner;   // hash of the entry holding each slot (meaningful while it is held)
    mutable std::mutex mu;

    bool slot_busy(int32_t s) const { return s >= 0 && (pending[s] || pins[s] > 0); }
    void touch(uint64_t h, Entry& e) {
        lru.erase({e.last_use, h});
        if (e.slot >= 0) lru_slots.erase({e.last_use, h});
        e.last_use = ++clock;
        lru.insert({e.last_use, h});
        if (e.slot >= 0) lru_slots.insert({e.last_use, h});
    }
    void drop_slot(uint64_t h, Entry& e) {
        if (e.slot < 0) return;
        lru_slots.erase({e.last_use, h});
        free_slots.push_back(e.slot);
        pending[e.slot] = 0;
        e.slot = -1;
    }
    // Evicts the least recently used entry that was last used before `start` and whose slot (if any)
    // is neither pending nor pinned, together with its slot.  False if there is none.
    bool evict_block(uint64_t start) {
        for (auto it = lru.begin(); it != lru.end() && it->first <= start; ++it) {
            const uint64_t h = it->second;
            Entry& e = blocks[h];
            if (slot_busy(e.slot)) continue;
            drop_slot(h, e);
            lru.erase(it);
            blocks.erase(h);
            return true;
        }
        return false;
    }
    // Frees the slot of the least recently used slot-holding entry last used before `start` whose slot
    // is committed and unpinned (the entry keeps its hash).  False if there is none.
    bool free_lru_slot(uint64_t start) {
        for (auto it = lru_slots.begin(); it != lru_slots.end() && it->first <= start; ++it) {
            const uint64_t h = it->second;
            Entry& e = blocks[h];
            if (slot_busy(e.slot)) continue;
            drop_slot(h, e);
            return true;
        }
        return false;
    }
};

extern "C" {

int64_t kda_prefix_block_hashes(const int32_t* tokens, int64_t n_tokens, uint64_t seed, uint64_t* hashes) {
    if (n_tokens < 0 || (n_tokens > 0 && !tokens)) return -1;
    const int64_t nb = n_tokens / KDA_PREFIX_BLOCK;
    if (nb > 0 && !hashes) return -1;
    uint64_t prev = seed;
    unsigned char buf[8 + 4 * KDA_PREFIX_BLOCK];
    for (int64_t b = 0; b < nb; ++b) {
        le64(prev, buf);
        for (int i = 0; i < KDA_PREFIX_BLOCK; ++i) {
            const uint32_t t = static_cast<uint32_t>(tokens[b * KDA_PREFIX_BLOCK + i]);
            for (int k = 0; k < 4; ++k) buf[8 + 4 * i + k] = static_cast<unsigned char>(t >> (8 * k));
        }
        prev = fnv1a_bytes(kFnvOffset, buf, sizeof(buf));
        hashes[b] = prev;
    }
    return nb;
}

kda_status_t kda_prefix_cache_create(int64_t max_blocks, int n_slots, int unit_blocks, kda_prefix_cache** out) {
    if (!out || max_blocks <= 0 || n_slots < 0 || unit_blocks < 2 || unit_blocks > 12) return KDA_ERR_ARG;
    kda_prefix_cache* c = new (std::nothrow) kda_prefix_cache();
    if (!c) return KDA_ERR_ARG;
    c->max_blocks = max_blocks;
    c->n_slots = n_slots;
    c->unit_blocks = unit_blocks;
    c->free_slots.reserve(n_slots);
    c->pending.assign(static_cast<size_t>(n_slots), 0);
    c->pins.assign(static_cast<size_t>(n_slots), 0);
    c->owner.assign(static_cast<size_t>(n_slots), 0);
    for (int s = n_slots - 1; s >= 0; --s) c->free_slots.push_back(s);   // slot 0 handed out first
    *out = c;
    return KDA_OK;
}

void kda_prefix_cache_destroy(kda_prefix_cache* cache) { delete cache; }

kda_status_t kda_prefix_cache_lookup(kda_prefix_cache* c, const uint64_t* hashes, int64_t n_blocks,
                                     int64_t* matched_blocks, int64_t* resume_blocks, int32_t* resume_slot) {
    if (!c || n_blocks < 0 || (n_blocks > 0 && !hashes) || !matched_blocks || !resume_blocks || !resume_slot)
        return KDA_ERR_ARG;
    std::lock_guard<std::mutex> lock(c->mu);
    int64_t m = 0, r = 0;
    int32_t slot = -1;
    for (; m < n_blocks; ++m) {
        auto it = c->blocks.find(hashes[m]);
        if (it == c->blocks.end()) break;
        c->touch(it->first, it->second);
        const int32_t sl = it->second.slot;
        if (sl >= 0 && !c->pending[sl]) {   // only a checkpoint whose state has been committed
            r = m + 1;
            slot = sl;
        }
    }
    if (slot >= 0) ++c->pins[slot];          // held until kda_prefix_cache_release
    *matched_blocks = m;
    *resume_blocks = r;
    *resume_slot = slot;
    return KDA_OK;
}

int64_t kda_prefix_cache_plan(const kda_prefix_cache* c, int64_t n_blocks, int64_t resume_blocks, int64_t* out_ends,
                              int64_t max_out) {
    if (!c || n_blocks < 0 || resume_blocks < 0 || resume_blocks > n_blocks || max_out < 0 ||
        (max_out > 0 && !out_ends))
        return -1;
    int64_t k = 0;
    auto emit = [&](int64_t e) {
        if (k < max_out) out_ends[k] = e;
        ++k;
    };
    const int64_t u = c->unit_blocks;
    for (int64_t e = (resume_blocks / u + 1) * u; e < n_blocks; e += u) emit(e);
    if (n_blocks > resume_blocks) emit(n_blocks);
    return k;
}

kda_status_t kda_prefix_cache_insert(kda_prefix_cache* c, const uint64_t* hashes, int64_t n_blocks,
                                     const int64_t* ends, int64_t n_ends, int32_t* out_slots) {
    if (!c || n_blocks < 0 || n_ends < 0 || (n_blocks > 0 && !hashes) || (n_ends > 0 && (!ends || !out_slots)))
        return KDA_ERR_ARG;
    for (int64_t i = 0; i < n_ends; ++i)
        if (ends[i] < 1 || ends[i] > n_blocks) return KDA_ERR_ARG;
    std::lock_guard<std::mutex> lock(c->mu);
    const uint64_t start = c->clock;   // entries touched by this request have last_use > start
    for (int64_t b = 0; b < n_blocks; ++b) {
        auto it = c->blocks.find(hashes[b]);
        if (it == c->blocks.end()) {
            while (static_cast<int64_t>(c->blocks.size()) >= c->max_blocks && c->evict_block(start)) {
            }
            if (static_cast<int64_t>(c->blocks.size()) >= c->max_blocks) break;   // this request fills the cache
            it = c->blocks.emplace(hashes[b], Entry{}).first;
        }
        c->touch(it->first, it->second);
    }
    for (int64_t i = 0; i < n_ends; ++i) {
        out_slots[i] = KDA_PREFIX_NO_SLOT;
        auto it = c->blocks.find(hashes[ends[i] - 1]);
        if (it == c->blocks.end()) continue;
        Entry& e = it->second;
        if (e.slot >= 0) {                     // stored already (or being stored): nothing to copy
            out_slots[i] = KDA_PREFIX_STORED;
            continue;
        }
        if (c->free_slots.empty()) c->free_lru_slot(start);
        if (c->free_slots.empty()) continue;
        e.slot = c->free_slots.back();
        c->free_slots.pop_back();
        c->pending[e.slot] = 1;                // until the caller commits the copied state
        c->owner[e.slot] = it->first;
        c->lru_slots.insert({e.last_use, it->first});
        out_slots[i] = e.slot;
    }
    return KDA_OK;
}

kda_status_t kda_prefix_cache_commit(kda_prefix_cache* c, const int32_t* slots, int64_t n) {
    if (!c || n < 0 || (n > 0 && !slots)) return KDA_ERR_ARG;
    std::lock_guard<std::mutex> lock(c->mu);
    for (int64_t i = 0; i < n; ++i)
        if (slots[i] >= c->n_slots) return KDA_ERR_ARG;
    for (int64_t i = 0; i < n; ++i)
        if (slots[i] >= 0) c->pending[slots[i]] = 0;   // negative entries (no slot, stored) are skipped
    return KDA_OK;
}

kda_status_t kda_prefix_cache_abort(kda_prefix_cache* c, const int32_t* slots, int64_t n) {
    if (!c || n < 0 || (n > 0 && !slots)) return KDA_ERR_ARG;
    std::lock_guard<std::mutex> lock(c->mu);
    for (int64_t i = 0; i < n; ++i)
        if (slots[i] >= c->n_slots) return KDA_ERR_ARG;
    for (int64_t i = 0; i < n; ++i) {
        const int32_t s = slots[i];
        if (s < 0 || !c->pending[s]) continue;   // only slots still waiting for their state
        auto it = c->blocks.find(c->owner[s]);
        if (it != c->blocks.end() && it->second.slot == s) c->drop_slot(it->first, it->second);
    }
    return KDA_OK;
}

kda_status_t kda_prefix_cache_release(kda_prefix_cache* c, int32_t slot) {
    if (!c) return KDA_ERR_ARG;
    if (slot < 0) return KDA_OK;               // a lookup that named no slot holds nothing
    std::lock_guard<std::mutex> lock(c->mu);
    if (slot >= c->n_slots || c->pins[slot] <= 0) return KDA_ERR_ARG;
    --c->pins[slot];
    return KDA_OK;
}

kda_status_t kda_prefix_cache_stats(const kda_prefix_cache* c, int64_t* n_blocks_cached, int32_t* n_slots_used) {
    if (!c || !n_blocks_cached || !n_slots_used) return KDA_ERR_ARG;
    std::lock_guard<std::mutex> lock(c->mu);
    *n_blocks_cached = static_cast<int64_t>(c->blocks.size());
    *n_slots_used = c->n_slots - static_cast<int32_t>(c->free_slots.size());
    return KDA_OK;
}

}  // extern "C"
