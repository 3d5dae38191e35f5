// Host-side block allocator and block tables (see include/pa_block_manager.h for
// the contract and the page passages it follows).
//
// Data structures: a LIFO free stack of block ids, a reference count per block,
// and a hash map from sequence id to (token count, block table).  Every mutating
// call first works out how many fresh blocks it needs and fails with PA_ERR_OOM
// before touching anything if too few can be had, so a failed call leaves the
// manager exactly as it was.
//
// Automatic prefix caching (sequences created from prompt tokens): a full prompt
// block is indexed by (parent block, parent's generation, its 16 token ids); a
// block's generation counts how often it was handed out, so a key never matches
// a block that has since been reused.  Cached blocks whose count drops to zero
// stay indexed on an evictable list (least recently freed first, and a freed
// sequence's blocks tail first) and are reclaimed only when the free stack is
// empty.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <list>
#include <memory>
#include <new>
#include <unordered_map>
#include <vector>

#include "pa_block_manager.h"

namespace {

struct Sequence {
    int64_t tokens = 0;
    std::vector<int32_t> blocks;  // logical block j -> physical block blocks[j]
};

struct CacheKey {
    int32_t parent = -1;     // physical block before this one in the prompt (-1: first)
    uint32_t parent_gen = 0;
    std::vector<int32_t> tokens;
};

// FNV-1a taken over 32-bit words (one xor and one multiply per word) with a final
// xor-shift, over (parent, parent generation, token ids).  Collisions are harmless:
// every hit is verified against the stored key.
uint64_t key_hash(int32_t parent, uint32_t parent_gen, const int32_t *tokens, size_t n) {
    uint64_t h = 1469598103934665603ull;
    auto mix = [&](uint32_t w) {
        h ^= w;
        h *= 1099511628211ull;
    };
    mix((uint32_t)parent);
    mix(parent_gen);
    for (size_t i = 0; i < n; ++i) mix((uint32_t)tokens[i]);
    return h ^ (h >> 29);
}
uint64_t key_hash(const CacheKey &k) { return key_hash(k.parent, k.parent_gen, k.tokens.data(), k.tokens.size()); }

}  // namespace

struct pa_block_manager {
    int32_t num_blocks = 0;
    int32_t block_size = 0;
    std::vector<int32_t> free_stack;  // back() is the next block handed out
    std::vector<int32_t> refs;
    std::vector<uint32_t> gen;        // times each block was handed out
    std::unordered_map<int64_t, Sequence> seqs;
    // prefix cache
    std::vector<char> cached;                      // block is in the index
    std::vector<CacheKey> keys;                    // its key while cached
    std::unordered_multimap<uint64_t, int32_t> index;
    std::list<int32_t> evictable;                  // cached, count 0; front = next reclaimed
    std::vector<std::list<int32_t>::iterator> evict_pos;
    std::vector<char> on_evictable;

    int32_t available() const { return (int32_t)(free_stack.size() + evictable.size()); }

    void uncache(int32_t b) {
        auto range = index.equal_range(key_hash(keys[b]));
        for (auto it = range.first; it != range.second; ++it)
            if (it->second == b) {
                index.erase(it);
                break;
            }
        cached[b] = 0;
        keys[b] = CacheKey{};
    }
    int32_t take() {
        int32_t b;
        if (!free_stack.empty()) {
            b = free_stack.back();
            free_stack.pop_back();
        } else {  // reclaim the least recently freed cached block
            b = evictable.front();
            evictable.pop_front();
            on_evictable[b] = 0;
            uncache(b);
        }
        refs[b] = 1;
        ++gen[b];
        return b;
    }
    // drop a reference; a block reaching zero goes to the free stack, or (cached)
    // is returned for the caller to put on the evictable list
    bool release(int32_t b) {
        if (--refs[b] != 0) return false;
        if (cached[b]) return true;
        free_stack.push_back(b);
        return false;
    }
    void make_evictable(int32_t b) {
        evict_pos[b] = evictable.insert(evictable.end(), b);
        on_evictable[b] = 1;
    }
    void revive(int32_t b) {  // a hit on a cached block
        if (on_evictable[b]) {
            evictable.erase(evict_pos[b]);
            on_evictable[b] = 0;
        }
        ++refs[b];
    }
    // cached block whose key is (parent, parent_gen, tokens[0..block_size)), or -1
    int32_t lookup(int32_t parent, uint32_t parent_gen, const int32_t *tokens) const {
        auto range = index.equal_range(key_hash(parent, parent_gen, tokens, (size_t)block_size));
        for (auto it = range.first; it != range.second; ++it) {
            const CacheKey &k = keys[it->second];
            if (k.parent == parent && k.parent_gen == parent_gen && k.tokens.size() == (size_t)block_size &&
                std::memcmp(k.tokens.data(), tokens, sizeof(int32_t) * (size_t)block_size) == 0)
                return it->second;
        }
        return -1;
    }
    void insert(int32_t b, CacheKey k) {
        index.emplace(key_hash(k), b);
        keys[b] = std::move(k);
        cached[b] = 1;
    }
    static int64_t blocks_for(int64_t tokens, int32_t bs) { return (tokens + bs - 1) / bs; }
};

// Host allocation failures (std::bad_alloc from the containers) must not cross the
// C boundary: they become PA_ERR_OOM, and the manager's state is then unspecified.
template <typename F>
pa_status guarded(F &&f) {
    try {
        return f();
    } catch (const std::bad_alloc &) {
        return PA_ERR_OOM;
    } catch (...) {
        return PA_ERR_INVALID_ARG;
    }
}

extern "C" {

pa_status pa_bm_create(int32_t num_blocks, int32_t block_size, const int32_t *free_order,
                       pa_block_manager **out) {
    if (!out || num_blocks < 0 || block_size <= 0) return PA_ERR_INVALID_ARG;
    *out = nullptr;
    return guarded([&]() -> pa_status {
        std::unique_ptr<pa_block_manager> owner(new pa_block_manager);
        pa_block_manager *bm = owner.get();
        bm->num_blocks = num_blocks;
        bm->block_size = block_size;
        bm->refs.assign(num_blocks, 0);
        bm->gen.assign(num_blocks, 0);
        bm->cached.assign(num_blocks, 0);
        bm->keys.resize(num_blocks);
        bm->evict_pos.resize(num_blocks);
        bm->on_evictable.assign(num_blocks, 0);
        bm->free_stack.resize(num_blocks);
        if (free_order) {
            std::vector<char> seen(num_blocks, 0);
            for (int32_t i = 0; i < num_blocks; ++i) {
                int32_t b = free_order[i];
                if (b < 0 || b >= num_blocks || seen[b]) return PA_ERR_INVALID_ARG;
                seen[b] = 1;
                bm->free_stack[i] = b;
            }
        } else {
            for (int32_t i = 0; i < num_blocks; ++i) bm->free_stack[i] = i;
        }
        *out = owner.release();
        return PA_OK;
    });
}

void pa_bm_destroy(pa_block_manager *bm) { delete bm; }

pa_status pa_bm_add_seq(pa_block_manager *bm, int64_t seq_id) {
    return guarded([&]() -> pa_status {
        if (!bm) return PA_ERR_INVALID_ARG;
        if (bm->seqs.count(seq_id)) return PA_ERR_INVALID_ARG;
        bm->seqs.emplace(seq_id, Sequence{});
        return PA_OK;
    });
}

pa_status pa_bm_add_seq_tokens(pa_block_manager *bm, int64_t seq_id, const int32_t *tokens, int32_t n,
                               int64_t *slots_out, int32_t *num_cached_out) {
    return guarded([&]() -> pa_status {
        if (!bm || n < 0 || (n > 0 && !tokens)) return PA_ERR_INVALID_ARG;
        if (bm->seqs.count(seq_id)) return PA_ERR_INVALID_ARG;
        const int32_t bs = bm->block_size;
        // Plan: the longest run of leading full blocks already cached.
        std::vector<int32_t> hits;
        int32_t parent = -1;
        uint32_t pgen = 0;
        int32_t hits_evictable = 0;
        for (int64_t j = 0; j < n / bs; ++j) {
            const int32_t b = bm->lookup(parent, pgen, tokens + j * bs);
            if (b < 0) break;
            hits.push_back(b);
            hits_evictable += bm->on_evictable[b] ? 1 : 0;
            parent = b;
            pgen = bm->gen[b];
        }
        const int64_t need = pa_block_manager::blocks_for(n, bs) - (int64_t)hits.size();
        if (need > (int64_t)bm->available() - hits_evictable) return PA_ERR_OOM;
        // Commit: reuse the hits, allocate the rest, index each new full block.
        for (int32_t b : hits) bm->revive(b);
        Sequence sq;
        sq.blocks = hits;
        int64_t k_out = 0;
        for (int64_t i = (int64_t)hits.size() * bs; i < n; ++i) {
            const int64_t offset = i % bs;
            if (offset == 0) sq.blocks.push_back(bm->take());
            if (slots_out) slots_out[k_out++] = (int64_t)sq.blocks.back() * bs + offset;
            if (offset == bs - 1) {
                const int64_t j = i / bs;
                const int32_t par = j > 0 ? sq.blocks[j - 1] : -1;
                bm->insert(sq.blocks[j], CacheKey{par, par >= 0 ? bm->gen[par] : 0u,
                                                  std::vector<int32_t>(tokens + j * bs, tokens + (j + 1) * bs)});
            }
        }
        sq.tokens = n;
        bm->seqs.emplace(seq_id, std::move(sq));
        if (num_cached_out) *num_cached_out = (int32_t)hits.size() * bs;
        return PA_OK;
    });
}

pa_status pa_bm_append_slots(pa_block_manager *bm, int64_t seq_id, int32_t n, int64_t *slots_out,
                             int32_t *cow_pairs_out, int32_t cow_capacity, int32_t *num_cow_out) {
    return guarded([&]() -> pa_status {
        if (!bm || n < 0) return PA_ERR_INVALID_ARG;
        auto it = bm->seqs.find(seq_id);
        if (it == bm->seqs.end()) return PA_ERR_NOT_FOUND;
        Sequence &sq = it->second;
        const int32_t bs = bm->block_size;
        // Plan first: fresh blocks for new block boundaries, plus one copy if the
        // first token lands in a shared, partly filled last block.
        const bool cow = n > 0 && (sq.tokens % bs) != 0 && bm->refs[sq.blocks.back()] > 1;
        const int64_t fresh =
            pa_block_manager::blocks_for(sq.tokens + n, bs) - pa_block_manager::blocks_for(sq.tokens, bs);
        if (fresh + (cow ? 1 : 0) > (int64_t)bm->available()) return PA_ERR_OOM;
        if (cow && cow_pairs_out && cow_capacity < 1) return PA_ERR_INVALID_ARG;
        int32_t ncow = 0;
        for (int32_t i = 0; i < n; ++i) {
            const int64_t offset = sq.tokens % bs;
            if (offset == 0) {
                sq.blocks.push_back(bm->take());
            } else if (bm->refs[sq.blocks.back()] > 1) {
                const int32_t old_block = sq.blocks.back();
                const int32_t new_block = bm->take();
                if (cow_pairs_out) {
                    cow_pairs_out[2 * ncow] = old_block;
                    cow_pairs_out[2 * ncow + 1] = new_block;
                }
                ++ncow;
                if (bm->release(old_block)) bm->make_evictable(old_block);
                sq.blocks.back() = new_block;
            }
            if (slots_out) slots_out[i] = (int64_t)sq.blocks.back() * bs + offset;
            ++sq.tokens;
        }
        if (num_cow_out) *num_cow_out = ncow;
        return PA_OK;
    });
}

pa_status pa_bm_append_step(pa_block_manager *bm, const int64_t *seq_ids, const int32_t *counts, int32_t n,
                            int64_t *slots_out, int32_t *cow_pairs_out, int32_t cow_capacity,
                            int32_t *num_cow_out) {
    return guarded([&]() -> pa_status {
        if (!bm || n < 0 || (n > 0 && !seq_ids) || cow_capacity < 0) return PA_ERR_INVALID_ARG;
        const int32_t bs = bm->block_size;
        // Plan the whole step in order: fresh blocks at block boundaries, and a copy
        // when a token goes into a partly filled last block still shared at that
        // moment (an earlier sibling's copy in this step drops the count by one).
        std::unordered_map<int64_t, char> seen;
        std::unordered_map<int32_t, int32_t> dropped;  // references given up by copies so far
        seen.reserve((size_t)n * 2);
        int64_t need = 0, cows = 0;
        std::vector<Sequence *> seq(n);
        for (int32_t i = 0; i < n; ++i) {
            const int32_t c = counts ? counts[i] : 1;
            if (c < 0) return PA_ERR_INVALID_ARG;
            if (!seen.emplace(seq_ids[i], 1).second) return PA_ERR_INVALID_ARG;  // one entry per sequence
            auto it = bm->seqs.find(seq_ids[i]);
            if (it == bm->seqs.end()) return PA_ERR_NOT_FOUND;
            seq[i] = &it->second;
            const Sequence &sq = it->second;
            if (c > 0 && sq.tokens % bs != 0) {
                const int32_t last = sq.blocks.back();
                auto d = dropped.find(last);
                const int32_t refs_now = bm->refs[last] - (d == dropped.end() ? 0 : d->second);
                if (refs_now > 1) {
                    ++need;
                    ++cows;
                    ++dropped[last];
                }
            }
            need += pa_block_manager::blocks_for(sq.tokens + c, bs) - pa_block_manager::blocks_for(sq.tokens, bs);
        }
        if (cow_pairs_out && cows > cow_capacity) return PA_ERR_INVALID_ARG;
        if (need > (int64_t)bm->available()) return PA_ERR_OOM;
        // Commit: the same steps as pa_bm_append_slots, sequence by sequence.
        int64_t k = 0;
        int32_t ncow = 0;
        for (int32_t i = 0; i < n; ++i) {
            Sequence &sq = *seq[i];
            const int32_t c = counts ? counts[i] : 1;
            for (int32_t t = 0; t < c; ++t) {
                const int64_t offset = sq.tokens % bs;
                if (offset == 0) {
                    sq.blocks.push_back(bm->take());
                } else if (bm->refs[sq.blocks.back()] > 1) {
                    const int32_t old_block = sq.blocks.back();
                    const int32_t new_block = bm->take();
                    if (cow_pairs_out) {
                        cow_pairs_out[2 * ncow] = old_block;
                        cow_pairs_out[2 * ncow + 1] = new_block;
                    }
                    ++ncow;
                    if (bm->release(old_block)) bm->make_evictable(old_block);
                    sq.blocks.back() = new_block;
                }
                if (slots_out) slots_out[k] = (int64_t)sq.blocks.back() * bs + offset;
                ++k;
                ++sq.tokens;
            }
        }
        if (num_cow_out) *num_cow_out = ncow;
        return PA_OK;
    });
}

pa_status pa_bm_fork(pa_block_manager *bm, int64_t parent_id, int64_t child_id) {
    return guarded([&]() -> pa_status {
        if (!bm) return PA_ERR_INVALID_ARG;
        auto p = bm->seqs.find(parent_id);
        if (p == bm->seqs.end()) return PA_ERR_NOT_FOUND;
        if (bm->seqs.count(child_id)) return PA_ERR_INVALID_ARG;
        Sequence child = p->second;  // copies token count and table
        for (int32_t b : child.blocks) ++bm->refs[b];
        bm->seqs.emplace(child_id, std::move(child));
        return PA_OK;
    });
}

pa_status pa_bm_free_seq(pa_block_manager *bm, int64_t seq_id) {
    return guarded([&]() -> pa_status {
        if (!bm) return PA_ERR_INVALID_ARG;
        auto it = bm->seqs.find(seq_id);
        if (it == bm->seqs.end()) return PA_ERR_NOT_FOUND;
        // references drop in logical order; cached blocks reaching zero become
        // evictable from the last to the first, so a prefix's tail goes before its head
        std::vector<int32_t> to_evictable;
        for (int32_t b : it->second.blocks)
            if (bm->release(b)) to_evictable.push_back(b);
        for (auto r = to_evictable.rbegin(); r != to_evictable.rend(); ++r) bm->make_evictable(*r);
        bm->seqs.erase(it);
        return PA_OK;
    });
}

int64_t pa_bm_num_tokens(const pa_block_manager *bm, int64_t seq_id) {
    if (!bm) return -1;
    auto it = bm->seqs.find(seq_id);
    return it == bm->seqs.end() ? -1 : it->second.tokens;
}

int32_t pa_bm_num_seq_blocks(const pa_block_manager *bm, int64_t seq_id) {
    if (!bm) return -1;
    auto it = bm->seqs.find(seq_id);
    return it == bm->seqs.end() ? -1 : (int32_t)it->second.blocks.size();
}

int32_t pa_bm_max_seq_blocks(const pa_block_manager *bm, const int64_t *seq_ids, int32_t n) {
    if (!bm || n < 0 || (n > 0 && !seq_ids)) return -1;
    int32_t mx = 0;
    for (int32_t i = 0; i < n; ++i) {
        auto it = bm->seqs.find(seq_ids[i]);
        if (it == bm->seqs.end()) return -1;
        mx = std::max(mx, (int32_t)it->second.blocks.size());
    }
    return mx;
}

pa_status pa_bm_block_table(const pa_block_manager *bm, int64_t seq_id, int32_t *out,
                            int32_t capacity, int32_t *len_out) {
    if (!bm || capacity < 0 || (capacity > 0 && !out)) return PA_ERR_INVALID_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return PA_ERR_NOT_FOUND;
    const auto &b = it->second.blocks;
    const int32_t k = (int32_t)b.size() < capacity ? (int32_t)b.size() : capacity;
    if (k > 0) std::memcpy(out, b.data(), sizeof(int32_t) * k);
    if (len_out) *len_out = (int32_t)b.size();
    return PA_OK;
}

pa_status pa_bm_build_tables(const pa_block_manager *bm, const int64_t *seq_ids, int32_t n,
                             int32_t max_blocks, int32_t *tables_out, int32_t *lens_out) {
    if (!bm || n < 0 || max_blocks < 0 || (n > 0 && (!seq_ids || !tables_out)))
        return PA_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n; ++i) {
        auto it = bm->seqs.find(seq_ids[i]);
        if (it == bm->seqs.end()) return PA_ERR_NOT_FOUND;
        if ((int64_t)it->second.blocks.size() > max_blocks) return PA_ERR_INVALID_ARG;
    }
    for (int32_t i = 0; i < n; ++i) {
        const Sequence &sq = bm->seqs.find(seq_ids[i])->second;
        int32_t *row = tables_out + (int64_t)i * max_blocks;
        const int32_t k = (int32_t)sq.blocks.size();
        if (k > 0) std::memcpy(row, sq.blocks.data(), sizeof(int32_t) * k);
        for (int32_t j = k; j < max_blocks; ++j) row[j] = -1;
        if (lens_out) lens_out[i] = (int32_t)sq.tokens;
    }
    return PA_OK;
}

int32_t pa_bm_refcount(const pa_block_manager *bm, int32_t block) {
    if (!bm || block < 0 || block >= bm->num_blocks) return -1;
    return bm->refs[block];
}

int32_t pa_bm_num_free(const pa_block_manager *bm) {
    return bm ? (int32_t)bm->free_stack.size() : -1;
}

int32_t pa_bm_num_blocks(const pa_block_manager *bm) { return bm ? bm->num_blocks : -1; }
int32_t pa_bm_block_size(const pa_block_manager *bm) { return bm ? bm->block_size : -1; }

int32_t pa_bm_num_evictable(const pa_block_manager *bm) {
    return bm ? (int32_t)bm->evictable.size() : -1;
}

int32_t pa_bm_num_cached(const pa_block_manager *bm) { return bm ? (int32_t)bm->index.size() : -1; }

int32_t pa_bm_evictable(const pa_block_manager *bm, int32_t *out, int32_t capacity) {
    if (!bm) return -1;
    int32_t k = 0;
    for (int32_t b : bm->evictable) {
        if (out && k < capacity) out[k] = b;
        ++k;
    }
    return k;
}

int32_t pa_bm_free_stack(const pa_block_manager *bm, int32_t *out, int32_t capacity) {
    if (!bm) return -1;
    const int32_t k = (int32_t)bm->free_stack.size();
    if (out) {
        const int32_t m = k < capacity ? k : capacity;
        if (m > 0) std::memcpy(out, bm->free_stack.data(), sizeof(int32_t) * m);
    }
    return k;
}

int64_t pa_bm_tokens_stored(const pa_block_manager *bm) {
    if (!bm) return -1;
    int64_t total = 0;
    for (const auto &kv : bm->seqs) total += kv.second.tokens;
    return total;
}

}  // extern "C"

// ---- snapshot / restore ---------------------------------------------------------
// Byte format (host byte order): "PABM", u32 version 1, i32 num_blocks, i32 block_size,
// u32 n + i32[n] free stack (bottom first), i32[num_blocks] counts, u32[num_blocks]
// generations, u32 n + per sequence in ascending id (i64 id, i64 tokens, u32 k, i32[k]
// blocks), u32 n + per cached block in ascending id (i32 block, i32 parent, u32 parent
// generation, u32 k, i32[k] tokens), u32 n + i32[n] evictable list (next reclaimed first).

namespace {

struct Writer {
    unsigned char *p;
    size_t cap, len = 0;
    template <typename T>
    void put(const T &v) {
        if (p && len + sizeof(T) <= cap) std::memcpy(p + len, &v, sizeof(T));
        len += sizeof(T);
    }
    void put_ids(const int32_t *v, size_t n) {
        if (p && len + 4 * n <= cap && n) std::memcpy(p + len, v, 4 * n);
        len += 4 * n;
    }
};

struct Reader {
    const unsigned char *p;
    size_t len, at = 0;
    bool ok = true;
    template <typename T>
    T get() {
        T v{};
        if (at + sizeof(T) > len) {
            ok = false;
            return v;
        }
        std::memcpy(&v, p + at, sizeof(T));
        at += sizeof(T);
        return v;
    }
    bool get_ids(std::vector<int32_t> &v, size_t n) {
        if (n > (len - at) / 4) return ok = false;
        v.resize(n);
        if (n) std::memcpy(v.data(), p + at, 4 * n);
        at += 4 * n;
        return true;
    }
};

constexpr uint32_t kSnapshotVersion = 1;

size_t write_snapshot(const pa_block_manager &bm, unsigned char *buf, size_t cap) {
    Writer w{buf, cap};
    uint32_t magic;
    std::memcpy(&magic, "PABM", 4);
    w.put(magic);
    w.put(kSnapshotVersion);
    w.put(bm.num_blocks);
    w.put(bm.block_size);
    w.put((uint32_t)bm.free_stack.size());
    w.put_ids(bm.free_stack.data(), bm.free_stack.size());
    w.put_ids(bm.refs.data(), bm.refs.size());
    w.put_ids(reinterpret_cast<const int32_t *>(bm.gen.data()), bm.gen.size());
    std::vector<int64_t> ids;
    ids.reserve(bm.seqs.size());
    for (const auto &kv : bm.seqs) ids.push_back(kv.first);
    std::sort(ids.begin(), ids.end());
    w.put((uint32_t)ids.size());
    for (int64_t id : ids) {
        const Sequence &sq = bm.seqs.at(id);
        w.put(id);
        w.put(sq.tokens);
        w.put((uint32_t)sq.blocks.size());
        w.put_ids(sq.blocks.data(), sq.blocks.size());
    }
    uint32_t ncached = 0;
    for (int32_t b = 0; b < bm.num_blocks; ++b) ncached += bm.cached[b] ? 1u : 0u;
    w.put(ncached);
    for (int32_t b = 0; b < bm.num_blocks; ++b) {
        if (!bm.cached[b]) continue;
        const CacheKey &k = bm.keys[b];
        w.put(b);
        w.put(k.parent);
        w.put(k.parent_gen);
        w.put((uint32_t)k.tokens.size());
        w.put_ids(k.tokens.data(), k.tokens.size());
    }
    w.put((uint32_t)bm.evictable.size());
    for (int32_t b : bm.evictable) w.put(b);
    return w.len;
}

// Cross-checks of a parsed snapshot, so that a restored manager can never hand a
// block that a sequence still holds to another one:
//  * each block's count equals the number of table entries naming it;
//  * every block is in exactly one state: free (on the free stack once, count 0,
//    not in the prefix index), evictable (indexed, count 0, on the evictable
//    list), or held (count > 0).
bool consistent(const pa_block_manager &bm) {
    const size_t nb = (size_t)bm.num_blocks;
    std::vector<int64_t> held(nb, 0);
    for (const auto &kv : bm.seqs)
        for (int32_t b : kv.second.blocks) ++held[(size_t)b];
    std::vector<char> on_free(nb, 0);
    for (int32_t b : bm.free_stack) {
        if (on_free[(size_t)b]) return false;  // listed twice
        on_free[(size_t)b] = 1;
    }
    for (size_t b = 0; b < nb; ++b) {
        if (held[b] != bm.refs[b]) return false;
        const bool is_free = on_free[b] != 0, is_evictable = bm.on_evictable[b] != 0;
        if (bm.refs[b] > 0) {
            if (is_free || is_evictable) return false;
        } else if (is_free == is_evictable) {
            return false;  // a count-0 block must be free or evictable, not both or neither
        } else if (is_free && bm.cached[b]) {
            return false;  // a free block is not in the prefix index
        }
    }
    return true;
}

}  // namespace

extern "C" {

size_t pa_bm_snapshot_size(const pa_block_manager *bm) {
    if (!bm) return 0;
    try {
        return write_snapshot(*bm, nullptr, 0);
    } catch (...) {
        return 0;
    }
}

pa_status pa_bm_snapshot(const pa_block_manager *bm, void *buf, size_t capacity, size_t *len_out) {
    return guarded([&]() -> pa_status {
        if (!bm || (capacity > 0 && !buf)) return PA_ERR_INVALID_ARG;
        const size_t need = write_snapshot(*bm, nullptr, 0);
        if (len_out) *len_out = need;
        if (capacity < need) return PA_ERR_INVALID_ARG;
        write_snapshot(*bm, static_cast<unsigned char *>(buf), capacity);
        return PA_OK;
    });
}

pa_status pa_bm_restore(const void *buf, size_t len, pa_block_manager **out) {
    if (!out || (len > 0 && !buf)) return PA_ERR_INVALID_ARG;
    *out = nullptr;
    return guarded([&]() -> pa_status {
        Reader r{static_cast<const unsigned char *>(buf), len};
        const uint32_t magic = r.get<uint32_t>();
        uint32_t want_magic;
        std::memcpy(&want_magic, "PABM", 4);
        if (!r.ok || magic != want_magic || r.get<uint32_t>() != kSnapshotVersion) return PA_ERR_INVALID_ARG;
        const int32_t nb = r.get<int32_t>(), bs = r.get<int32_t>();
        if (!r.ok || nb < 0 || bs <= 0) return PA_ERR_INVALID_ARG;
        std::unique_ptr<pa_block_manager> owner(new pa_block_manager);
        pa_block_manager &bm = *owner;
        bm.num_blocks = nb;
        bm.block_size = bs;
        auto in_pool = [&](int32_t b) { return b >= 0 && b < nb; };
        std::vector<int32_t> tmp;
        if (!r.get_ids(bm.free_stack, r.get<uint32_t>()) || bm.free_stack.size() > (size_t)nb) return PA_ERR_INVALID_ARG;
        for (int32_t b : bm.free_stack)
            if (!in_pool(b)) return PA_ERR_INVALID_ARG;
        if (!r.get_ids(bm.refs, (size_t)nb) || !r.get_ids(tmp, (size_t)nb)) return PA_ERR_INVALID_ARG;
        bm.gen.assign(tmp.begin(), tmp.end());
        for (int32_t c : bm.refs)
            if (c < 0) return PA_ERR_INVALID_ARG;
        const uint32_t nseq = r.get<uint32_t>();
        for (uint32_t i = 0; r.ok && i < nseq; ++i) {
            const int64_t id = r.get<int64_t>();
            Sequence sq;
            sq.tokens = r.get<int64_t>();
            if (!r.ok || !r.get_ids(sq.blocks, r.get<uint32_t>())) return PA_ERR_INVALID_ARG;
            for (int32_t b : sq.blocks)
                if (!in_pool(b)) return PA_ERR_INVALID_ARG;
            if (sq.tokens < 0 || pa_block_manager::blocks_for(sq.tokens, bs) != (int64_t)sq.blocks.size())
                return PA_ERR_INVALID_ARG;
            if (!bm.seqs.emplace(id, std::move(sq)).second) return PA_ERR_INVALID_ARG;
        }
        bm.cached.assign(nb, 0);
        bm.keys.resize(nb);
        bm.evict_pos.resize(nb);
        bm.on_evictable.assign(nb, 0);
        const uint32_t ncached = r.get<uint32_t>();
        for (uint32_t i = 0; r.ok && i < ncached; ++i) {
            const int32_t b = r.get<int32_t>();
            CacheKey k;
            k.parent = r.get<int32_t>();
            k.parent_gen = r.get<uint32_t>();
            if (!r.ok || !r.get_ids(k.tokens, r.get<uint32_t>())) return PA_ERR_INVALID_ARG;
            if (!in_pool(b) || bm.cached[b] || (k.parent != -1 && !in_pool(k.parent)) ||
                k.tokens.size() != (size_t)bs)
                return PA_ERR_INVALID_ARG;
            bm.insert(b, std::move(k));
        }
        const uint32_t nev = r.get<uint32_t>();
        for (uint32_t i = 0; r.ok && i < nev; ++i) {
            const int32_t b = r.get<int32_t>();
            if (!r.ok || !in_pool(b) || !bm.cached[b] || bm.on_evictable[b] || bm.refs[b] != 0)
                return PA_ERR_INVALID_ARG;
            bm.make_evictable(b);
        }
        if (!r.ok || r.at != len) return PA_ERR_INVALID_ARG;
        if (!consistent(bm)) return PA_ERR_INVALID_ARG;
        *out = owner.release();
        return PA_OK;
    });
}

}  // extern "C"
