// Host block manager: free stack, refcounts, per-sequence block tables,
// slot reservation with copy-on-write.
//
// Follows "What problem does PagedAttention solve, and what is continuous
// batching?", section "How PagedAttention works" (fixed-size blocks, a block
// table per request, any free block will do, shared blocks and copy-on-write)
// and section "A concrete memory example" (a finished request's blocks return
// to the pool at once), and "Continuous Batching & Paged Attention", section
// "Paged attention borrows a trick from operating systems" (a growing request
// gets another block).  The policy choices the pages leave open -- LIFO reuse
// over a caller-given order, logical-order reference drops, whole-call
// rollback -- are documented in include/pa.h.
#include <algorithm>
#include <cstring>
#include <new>

#include "pool.hpp"

namespace pa_internal {
static thread_local std::string g_last_error;
std::atomic<uint64_t> launch_count{0};

pa_status fail(pa_status st, const std::string &msg) {
    g_last_error = msg;
    return st;
}
pa_status ok() { return PA_OK; }
}  // namespace pa_internal

using pa_internal::fail;

namespace {

bool valid_block(const pa_pool *p, int32_t b) { return b >= 0 && b < p->cfg.num_blocks; }

void add_ref(pa_pool *p, int32_t b) {
    if (++p->refcount[b] == 2) ++p->num_shared;
}

// Drop a reference that is known to be > 0; returns true when it reached zero.
bool drop_ref(pa_pool *p, int32_t b) {
    int32_t r = --p->refcount[b];
    if (r == 1) --p->num_shared;
    return r == 0;
}

void note_usage(pa_pool *p) {
    int32_t used = p->cfg.num_blocks - (int32_t)p->free_stack.size() - p->ev_count;
    p->peak_used = std::max(p->peak_used, used);
}

// ---- evictable queue (registered blocks with refcount 0), oldest at the head
void ev_push_back(pa_pool *p, int32_t b) {
    p->ev_prev[b] = p->ev_tail;
    p->ev_next[b] = -1;
    if (p->ev_tail >= 0) p->ev_next[p->ev_tail] = b; else p->ev_head = b;
    p->ev_tail = b;
    p->in_ev[b] = 1;
    ++p->ev_count;
}

void ev_push_front(pa_pool *p, int32_t b) {
    p->ev_prev[b] = -1;
    p->ev_next[b] = p->ev_head;
    if (p->ev_head >= 0) p->ev_prev[p->ev_head] = b; else p->ev_tail = b;
    p->ev_head = b;
    p->in_ev[b] = 1;
    ++p->ev_count;
}

void ev_unlink(pa_pool *p, int32_t b) {
    const int32_t pr = p->ev_prev[b], nx = p->ev_next[b];
    if (pr >= 0) p->ev_next[pr] = nx; else p->ev_head = nx;
    if (nx >= 0) p->ev_prev[nx] = pr; else p->ev_tail = pr;
    p->in_ev[b] = 0;
    --p->ev_count;
}

void unregister(pa_pool *p, int32_t b) {
    p->block_of.erase(p->key_of[b]);
    p->has_key[b] = 0;
}

void register_key(pa_pool *p, int32_t b, uint64_t key) {
    p->block_of.emplace(key, b);
    p->key_of[b] = key;
    p->has_key[b] = 1;
}

// A block whose last reference went away: cached blocks stay findable in the queue.
void release(pa_pool *p, int32_t b) {
    if (p->has_key[b]) ev_push_back(p, b); else p->free_stack.push_back(b);
}

// Take a block: the free stack first, else evict the least recently released cached
// block.  *evicted_key is set (and *was_evicted true) when a cached block was reclaimed.
pa_status pop_block(pa_pool *p, int32_t *b, bool *was_evicted, uint64_t *evicted_key) {
    *was_evicted = false;
    if (p->fail_alloc_after == 0) {
        p->fail_alloc_after = -1;
        return fail(PA_ERR_OUT_OF_BLOCKS, "block allocation failed (injected)");
    }
    if (p->free_stack.empty() && p->ev_head < 0)
        return fail(PA_ERR_OUT_OF_BLOCKS, "no free KV blocks left in the pool");
    if (p->fail_alloc_after > 0) --p->fail_alloc_after;
    if (!p->free_stack.empty()) {
        *b = p->free_stack.back();
        p->free_stack.pop_back();
    } else {
        *b = p->ev_head;
        ev_unlink(p, *b);
        *was_evicted = true;
        *evicted_key = p->key_of[*b];
        unregister(p, *b);
        ++p->cache_evictions;
    }
    p->refcount[*b] = 1;
    return PA_OK;
}

// Undo journal for pa_reserve_slots: every mutation is recorded and replayed
// backwards if the call runs out of blocks part way.
struct Undo {
    enum Kind { kAlloc, kEvict, kDrop, kPush, kSet, kLen, kCow } kind;
    int32_t seq;
    int32_t a;
    int32_t b;
    uint64_t key;
};

}  // namespace

extern "C" {

const char *pa_last_error(void) { return pa_internal::g_last_error.c_str(); }

const char *pa_status_string(pa_status s) {
    switch (s) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
    case PA_ERR_OUT_OF_BLOCKS: return "PA_ERR_OUT_OF_BLOCKS";
    case PA_ERR_DOUBLE_FREE: return "PA_ERR_DOUBLE_FREE";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
    }
    return "PA_ERR_UNKNOWN";
}

pa_status pa_pool_create(const pa_pool_config *cfg, void *k_pool, void *v_pool,
                         const int32_t *free_order, pa_pool **out) {
    if (!cfg || !out) return fail(PA_ERR_INVALID_ARG, "pa_pool_create: null config or out");
    *out = nullptr;
    if (cfg->num_layers < 1 || cfg->num_blocks < 1 || cfg->num_kv_heads < 1 ||
        cfg->block_size < 1 || cfg->head_dim < 1)
        return fail(PA_ERR_INVALID_ARG, "pa_pool_create: sizes must be positive");
    if (cfg->dtype != PA_F32 && cfg->dtype != PA_F16 && cfg->dtype != PA_BF16 && cfg->dtype != PA_FP8_E4M3)
        return fail(PA_ERR_INVALID_ARG, "pa_pool_create: unknown dtype");
    if (cfg->dtype == PA_FP8_E4M3 && cfg->act_dtype != PA_F16 && cfg->act_dtype != PA_BF16)
        return fail(PA_ERR_INVALID_ARG, "pa_pool_create: an FP8 pool needs act_dtype PA_F16 or PA_BF16");
    if (cfg->dtype == PA_FP8_E4M3 && cfg->block_size % 16 != 0)
        return fail(PA_ERR_UNSUPPORTED, "pa_pool_create: FP8 pools need a block_size that is a multiple of 16");
    if ((k_pool == nullptr) != (v_pool == nullptr))
        return fail(PA_ERR_INVALID_ARG, "pa_pool_create: give both pools or neither");
    if (((uintptr_t)k_pool | (uintptr_t)v_pool) & 15)
        return fail(PA_ERR_INVALID_ARG, "pa_pool_create: pools must be 16-byte aligned");
    pa_pool *p = new (std::nothrow) pa_pool();
    if (!p) return fail(PA_ERR_INVALID_ARG, "pa_pool_create: out of host memory");
    p->cfg = *cfg;
    p->k_pool = k_pool;
    p->v_pool = v_pool;
    const int32_t nb = cfg->num_blocks;
    p->refcount.assign(nb, 0);
    p->key_of.assign(nb, 0);
    p->has_key.assign(nb, 0);
    p->ev_prev.assign(nb, -1);
    p->ev_next.assign(nb, -1);
    p->in_ev.assign(nb, 0);
    p->free_stack.resize(nb);
    if (free_order) {
        std::vector<char> seen(nb, 0);
        for (int32_t i = 0; i < nb; ++i) {
            int32_t b = free_order[i];
            if (b < 0 || b >= nb || seen[b]) {
                delete p;
                return fail(PA_ERR_INVALID_ARG, "pa_pool_create: free_order is not a permutation");
            }
            seen[b] = 1;
            p->free_stack[nb - 1 - i] = b;   // free_order[0] ends on top
        }
    } else {
        for (int32_t i = 0; i < nb; ++i) p->free_stack[nb - 1 - i] = i;
    }
    *out = p;
    return PA_OK;
}

pa_status pa_pool_set_scales(pa_pool *pool, void *scales) {
    if (!pool || !scales) return fail(PA_ERR_INVALID_ARG, "pa_pool_set_scales: null argument");
    if (!pool->fp8()) return fail(PA_ERR_INVALID_ARG, "pa_pool_set_scales: only FP8 pools carry scales");
    if ((uintptr_t)scales & 15) return fail(PA_ERR_INVALID_ARG, "pa_pool_set_scales: scales must be 16-byte aligned");
    pool->scales = scales;
    return PA_OK;
}

pa_status pa_pool_destroy(pa_pool *pool) {
    if (!pool) return fail(PA_ERR_INVALID_ARG, "pa_pool_destroy: null pool");
    delete pool;
    return PA_OK;
}

pa_status pa_pool_stats(const pa_pool *p, pa_pool_stats_t *o) {
    if (!p || !o) return fail(PA_ERR_INVALID_ARG, "pa_pool_stats: null argument");
    o->num_blocks = p->cfg.num_blocks;
    o->num_free = (int32_t)p->free_stack.size() + p->ev_count;
    o->num_shared = p->num_shared;
    o->num_seqs = (int32_t)p->seqs.size();
    o->num_tokens = p->num_tokens;
    o->cow_copies = p->cow_copies;
    o->peak_used = p->peak_used;
    o->num_cached = (int32_t)p->block_of.size();
    o->num_evictable = p->ev_count;
    o->cache_hits = p->cache_hits;
    o->cache_evictions = p->cache_evictions;
    return PA_OK;
}

pa_status pa_alloc_block(pa_pool *p, int32_t *block) {
    if (!p || !block) return fail(PA_ERR_INVALID_ARG, "pa_alloc_block: null argument");
    bool ev;
    uint64_t key;
    pa_status st = pop_block(p, block, &ev, &key);
    if (st == PA_OK) note_usage(p);
    return st;
}

pa_status pa_free_block(pa_pool *p, int32_t block) {
    if (!p || !valid_block(p, block)) return fail(PA_ERR_INVALID_ARG, "pa_free_block: bad block id");
    if (p->refcount[block] == 0)
        return fail(PA_ERR_DOUBLE_FREE, "pa_free_block: block " + std::to_string(block) + " is already free");
    if (drop_ref(p, block)) release(p, block);
    return PA_OK;
}

pa_status pa_incref_block(pa_pool *p, int32_t block) {
    if (!p || !valid_block(p, block)) return fail(PA_ERR_INVALID_ARG, "pa_incref_block: bad block id");
    if (p->refcount[block] == 0) return fail(PA_ERR_INVALID_ARG, "pa_incref_block: block is free");
    add_ref(p, block);
    return PA_OK;
}

pa_status pa_block_refcount(const pa_pool *p, int32_t block, int32_t *rc) {
    if (!p || !rc || !valid_block(p, block)) return fail(PA_ERR_INVALID_ARG, "pa_block_refcount: bad argument");
    *rc = p->refcount[block];
    return PA_OK;
}

pa_status pa_num_free_blocks(const pa_pool *p, int32_t *n) {
    if (!p || !n) return fail(PA_ERR_INVALID_ARG, "pa_num_free_blocks: null argument");
    *n = (int32_t)p->free_stack.size() + p->ev_count;
    return PA_OK;
}

pa_status pa_free_list(const pa_pool *p, int32_t *out, int32_t cap, int32_t *n) {
    if (!p || !n || (cap > 0 && !out)) return fail(PA_ERR_INVALID_ARG, "pa_free_list: bad argument");
    *n = (int32_t)p->free_stack.size();
    int32_t m = std::min<int32_t>(cap, *n);
    if (m > 0) std::memcpy(out, p->free_stack.data(), sizeof(int32_t) * (size_t)m);
    return PA_OK;
}

pa_status pa_debug_fail_alloc_after(pa_pool *p, int64_t n) {
    if (!p) return fail(PA_ERR_INVALID_ARG, "pa_debug_fail_alloc_after: null pool");
    p->fail_alloc_after = n < 0 ? -1 : n;
    return PA_OK;
}

pa_status pa_seq_add(pa_pool *p, int32_t *seq_id) {
    if (!p || !seq_id) return fail(PA_ERR_INVALID_ARG, "pa_seq_add: null argument");
    if (p->next_seq == INT32_MAX) return fail(PA_ERR_INVALID_ARG, "pa_seq_add: sequence ids exhausted");
    *seq_id = p->next_seq++;
    p->seqs.emplace(*seq_id, pa_pool::Seq());
    return PA_OK;
}

pa_status pa_seq_fork(pa_pool *p, int32_t parent, int32_t *child) {
    if (!p || !child) return fail(PA_ERR_INVALID_ARG, "pa_seq_fork: null argument");
    auto it = p->seqs.find(parent);
    if (it == p->seqs.end()) return fail(PA_ERR_INVALID_ARG, "pa_seq_fork: unknown parent");
    if (it->second.swapped) return fail(PA_ERR_INVALID_ARG, "pa_seq_fork: parent is swapped out");
    if (p->next_seq == INT32_MAX) return fail(PA_ERR_INVALID_ARG, "pa_seq_fork: sequence ids exhausted");
    pa_pool::Seq s = it->second;          // copy of table and length
    for (int32_t b : s.table) add_ref(p, b);
    *child = p->next_seq++;
    p->num_tokens += s.len;
    p->seqs.emplace(*child, std::move(s));
    return PA_OK;
}

pa_status pa_seq_free(pa_pool *p, int32_t seq_id) {
    pa_internal::TraceRange trace_("pa_seq_free");
    if (!p) return fail(PA_ERR_INVALID_ARG, "pa_seq_free: null pool");
    auto it = p->seqs.find(seq_id);
    if (it == p->seqs.end()) return fail(PA_ERR_INVALID_ARG, "pa_seq_free: unknown sequence");
    for (int32_t b : it->second.table)
        if (drop_ref(p, b)) release(p, b);
    p->num_tokens -= it->second.len;
    p->seqs.erase(it);
    return PA_OK;
}

pa_status pa_seq_info(const pa_pool *p, int32_t seq_id, int32_t *len, int32_t *table, int32_t cap,
                      int32_t *nblk) {
    if (!p) return fail(PA_ERR_INVALID_ARG, "pa_seq_info: null pool");
    auto it = p->seqs.find(seq_id);
    if (it == p->seqs.end()) return fail(PA_ERR_INVALID_ARG, "pa_seq_info: unknown sequence");
    const pa_pool::Seq &s = it->second;
    if (len) *len = s.len;
    if (nblk) *nblk = (int32_t)s.table.size();
    if (table && cap > 0) {
        int32_t m = std::min<int32_t>(cap, (int32_t)s.table.size());
        std::memcpy(table, s.table.data(), sizeof(int32_t) * (size_t)m);
    }
    return PA_OK;
}

pa_status pa_reserve_slots(pa_pool *p, const int32_t *seq_ids, const int32_t *ntok, int32_t n,
                           int64_t *slot_mapping_out, int32_t *cow_pairs_out, int32_t *n_cow) {
    pa_internal::TraceRange trace_("pa_reserve_slots");
    if (!p || n < 0 || (n > 0 && (!seq_ids || !ntok)))
        return fail(PA_ERR_INVALID_ARG, "pa_reserve_slots: bad argument");
    int64_t total = 0;
    std::vector<pa_pool::Seq *> seqs((size_t)n);
    const uint64_t call = ++p->batch_calls;   // a sequence listed twice in this call is seen twice
    for (int32_t i = 0; i < n; ++i) {
        auto it = p->seqs.find(seq_ids[i]);
        if (it == p->seqs.end() || ntok[i] < 0)
            return fail(PA_ERR_INVALID_ARG, "pa_reserve_slots: unknown sequence or negative count");
        if (it->second.swapped) return fail(PA_ERR_INVALID_ARG, "pa_reserve_slots: sequence is swapped out");
        if ((int64_t)it->second.len + ntok[i] > INT32_MAX)
            return fail(PA_ERR_INVALID_ARG, "pa_reserve_slots: sequence too long");
        if (it->second.seen == call) return fail(PA_ERR_INVALID_ARG, "pa_reserve_slots: duplicate sequence id");
        it->second.seen = call;
        seqs[i] = &it->second;
        total += ntok[i];
    }
    if (total > 0 && !slot_mapping_out) return fail(PA_ERR_INVALID_ARG, "pa_reserve_slots: null slot_mapping_out");

    const int32_t B = p->cfg.block_size;
    // Blocks the call must open at block boundaries (copies on write need more): a
    // request that cannot fit fails here, before anything is allocated, so a huge
    // count costs nothing and the journal below is sized by what can really happen.
    int64_t opened = 0;
    for (int32_t i = 0; i < n; ++i)
        opened += ((int64_t)seqs[i]->len + ntok[i] + B - 1) / B - (int64_t)seqs[i]->table.size();
    if (opened > (int64_t)p->free_stack.size() + p->ev_count)
        return fail(PA_ERR_OUT_OF_BLOCKS, "pa_reserve_slots: no free KV blocks left in the pool (needs " +
                                              std::to_string(opened) + " new blocks; no change made)");
    std::vector<Undo> journal;
    int32_t cows = 0;
    int64_t k = 0;
    pa_status st = PA_OK;
    try {
    // one length record per token and two per opened block; a copy on write adds four
    journal.reserve((size_t)(total + 2 * opened + 16));
    for (int32_t i = 0; i < n && st == PA_OK; ++i) {
        pa_pool::Seq &s = *seqs[i];
        for (int32_t t = 0; t < ntok[i]; ++t) {
            const int32_t L = s.len;
            bool ev;
            uint64_t key;
            if (L % B == 0) {
                int32_t b;
                st = pop_block(p, &b, &ev, &key);
                if (st != PA_OK) break;
                journal.push_back({ev ? Undo::kEvict : Undo::kAlloc, seq_ids[i], b, 0, key});
                s.table.push_back(b);
                journal.push_back({Undo::kPush, seq_ids[i], 0, 0, 0});
            } else {
                const int32_t tail = s.table.back();
                if (p->refcount[tail] > 1) {
                    int32_t nb;
                    st = pop_block(p, &nb, &ev, &key);
                    if (st != PA_OK) break;
                    journal.push_back({ev ? Undo::kEvict : Undo::kAlloc, seq_ids[i], nb, 0, key});
                    drop_ref(p, tail);
                    journal.push_back({Undo::kDrop, seq_ids[i], tail, 0, 0});
                    const int32_t idx = (int32_t)s.table.size() - 1;
                    s.table[idx] = nb;
                    journal.push_back({Undo::kSet, seq_ids[i], idx, tail, 0});
                    if (cow_pairs_out) {
                        cow_pairs_out[2 * cows] = tail;
                        cow_pairs_out[2 * cows + 1] = nb;
                    }
                    ++cows;
                    journal.push_back({Undo::kCow, seq_ids[i], 0, 0, 0});
                }
            }
            slot_mapping_out[k++] = (int64_t)s.table[L / B] * B + L % B;
            s.len = L + 1;
            journal.push_back({Undo::kLen, seq_ids[i], L, 0, 0});
        }
    }
    } catch (const std::bad_alloc &) {   // host memory for the journal or a table: undo, report
        st = fail(PA_ERR_HOST_MEMORY, "host memory allocation failed");
    }
    if (st != PA_OK) {
        std::string msg = pa_last_error();
        for (auto it = journal.rbegin(); it != journal.rend(); ++it) {
            pa_pool::Seq &s = p->seqs[it->seq];
            switch (it->kind) {
            case Undo::kAlloc:
                p->refcount[it->a] = 0;
                p->free_stack.push_back(it->a);
                break;
            case Undo::kEvict:   // it was the head of the queue when it was taken
                p->refcount[it->a] = 0;
                register_key(p, it->a, it->key);
                ev_push_front(p, it->a);
                --p->cache_evictions;
                break;
            case Undo::kDrop: add_ref(p, it->a); break;
            case Undo::kPush: s.table.pop_back(); break;
            case Undo::kSet: s.table[it->a] = it->b; break;
            case Undo::kLen: s.len = it->a; break;
            case Undo::kCow: break;
            }
        }
        return fail(st, "pa_reserve_slots: " + msg + " (no change made)");
    }
    p->num_tokens += total;
    p->cow_copies += cows;
    if (n_cow) *n_cow = cows;
    note_usage(p);
    return PA_OK;
}

pa_status pa_build_block_tables(const pa_pool *p, const int32_t *seq_ids, int32_t n, int32_t max_blocks,
                                int32_t *tables_out, int32_t *lens_out) {
    pa_internal::TraceRange trace_("pa_build_block_tables");
    if (!p || n < 0 || max_blocks < 1 || (n > 0 && (!seq_ids || !tables_out || !lens_out)))
        return fail(PA_ERR_INVALID_ARG, "pa_build_block_tables: bad argument");
    for (int32_t i = 0; i < n; ++i) {
        auto it = p->seqs.find(seq_ids[i]);
        if (it == p->seqs.end()) return fail(PA_ERR_INVALID_ARG, "pa_build_block_tables: unknown sequence");
        if (it->second.swapped) return fail(PA_ERR_INVALID_ARG, "pa_build_block_tables: sequence is swapped out");
        if ((int32_t)it->second.table.size() > max_blocks)
            return fail(PA_ERR_INVALID_ARG, "pa_build_block_tables: sequence has more than max_blocks blocks");
    }
    for (int32_t i = 0; i < n; ++i) {
        const pa_pool::Seq &s = p->seqs.find(seq_ids[i])->second;
        int32_t *row = tables_out + (size_t)i * max_blocks;
        const size_t nb = s.table.size();
        if (nb) std::memcpy(row, s.table.data(), sizeof(int32_t) * nb);
        std::fill(row + nb, row + max_blocks, -1);
        lens_out[i] = s.len;
    }
    return PA_OK;
}

pa_status pa_prefix_register(pa_pool *p, int32_t seq_id, const uint64_t *keys, int32_t n_blocks,
                             int32_t *n_new) {
    if (!p || n_blocks < 0 || (n_blocks > 0 && !keys)) return fail(PA_ERR_INVALID_ARG, "pa_prefix_register: bad argument");
    auto it = p->seqs.find(seq_id);
    if (it == p->seqs.end()) return fail(PA_ERR_INVALID_ARG, "pa_prefix_register: unknown sequence");
    if (it->second.swapped) return fail(PA_ERR_INVALID_ARG, "pa_prefix_register: sequence is swapped out");
    const pa_pool::Seq &s = it->second;
    if ((int64_t)n_blocks * p->cfg.block_size > s.len)
        return fail(PA_ERR_INVALID_ARG, "pa_prefix_register: only full blocks can be registered");
    int32_t added = 0;
    for (int32_t i = 0; i < n_blocks; ++i) {
        const int32_t b = s.table[i];
        if (p->has_key[b] || p->block_of.count(keys[i])) continue;
        register_key(p, b, keys[i]);
        ++added;
    }
    if (n_new) *n_new = added;
    return PA_OK;
}

pa_status pa_seq_add_cached(pa_pool *p, const uint64_t *keys, int32_t n_keys, int32_t *seq_id, int32_t *n_hit) {
    if (!p || !seq_id || !n_hit || n_keys < 0 || (n_keys > 0 && !keys))
        return fail(PA_ERR_INVALID_ARG, "pa_seq_add_cached: bad argument");
    if (p->next_seq == INT32_MAX) return fail(PA_ERR_INVALID_ARG, "pa_seq_add_cached: sequence ids exhausted");
    pa_pool::Seq s;
    for (int32_t i = 0; i < n_keys; ++i) {
        auto f = p->block_of.find(keys[i]);
        if (f == p->block_of.end()) break;
        const int32_t b = f->second;
        if (p->refcount[b] == 0) ev_unlink(p, b);
        add_ref(p, b);
        s.table.push_back(b);
    }
    s.len = (int32_t)s.table.size() * p->cfg.block_size;
    *n_hit = (int32_t)s.table.size();
    *seq_id = p->next_seq++;
    p->num_tokens += s.len;
    p->cache_hits += *n_hit;
    p->seqs.emplace(*seq_id, std::move(s));
    note_usage(p);
    return PA_OK;
}

pa_status pa_prefix_evictable(const pa_pool *p, int32_t *out, int32_t cap, int32_t *n) {
    if (!p || !n || (cap > 0 && !out)) return fail(PA_ERR_INVALID_ARG, "pa_prefix_evictable: bad argument");
    *n = p->ev_count;
    int32_t k = 0;
    for (int32_t b = p->ev_head; b >= 0 && k < cap; b = p->ev_next[b]) out[k++] = b;
    return PA_OK;
}

static size_t swap_bytes_of(const pa_pool *p, int32_t len) {
    const size_t nblk = (size_t)((len + p->cfg.block_size - 1) / p->cfg.block_size);
    return nblk * (size_t)p->cfg.num_layers * p->swap_record_bytes();
}

pa_status pa_swap_bytes(const pa_pool *p, int32_t seq_id, size_t *bytes) {
    if (!p || !bytes) return fail(PA_ERR_INVALID_ARG, "pa_swap_bytes: null argument");
    auto it = p->seqs.find(seq_id);
    if (it == p->seqs.end()) return fail(PA_ERR_INVALID_ARG, "pa_swap_bytes: unknown sequence");
    *bytes = swap_bytes_of(p, it->second.len);
    return PA_OK;
}

pa_status pa_swap_out(pa_pool *p, int32_t seq_id, void *host_buf, size_t buf_bytes, pa_stream stream) {
    pa_internal::TraceRange trace_("pa_swap_out");
    if (!p) return fail(PA_ERR_INVALID_ARG, "pa_swap_out: null pool");
    auto it = p->seqs.find(seq_id);
    if (it == p->seqs.end()) return fail(PA_ERR_INVALID_ARG, "pa_swap_out: unknown sequence");
    pa_pool::Seq &s = it->second;
    if (s.swapped) return fail(PA_ERR_INVALID_ARG, "pa_swap_out: sequence is already swapped out");
    if (p->k_pool) {
        if (!host_buf || buf_bytes < swap_bytes_of(p, s.len))
            return fail(PA_ERR_INVALID_ARG, "pa_swap_out: host buffer missing or smaller than pa_swap_bytes");
        pa_status st = pa_internal::swap_copy(p, s.table.data(), (int32_t)s.table.size(), host_buf, true, stream);
        if (st != PA_OK) return st;
    }
    for (int32_t b : s.table)
        if (drop_ref(p, b)) release(p, b);
    s.table.clear();
    s.swapped = true;
    return PA_OK;
}

pa_status pa_swap_in(pa_pool *p, int32_t seq_id, const void *host_buf, size_t buf_bytes, pa_stream stream) {
    pa_internal::TraceRange trace_("pa_swap_in");
    if (!p) return fail(PA_ERR_INVALID_ARG, "pa_swap_in: null pool");
    auto it = p->seqs.find(seq_id);
    if (it == p->seqs.end()) return fail(PA_ERR_INVALID_ARG, "pa_swap_in: unknown sequence");
    pa_pool::Seq &s = it->second;
    if (!s.swapped) return fail(PA_ERR_INVALID_ARG, "pa_swap_in: sequence is not swapped out");
    if (p->k_pool && (!host_buf || buf_bytes < swap_bytes_of(p, s.len)))
        return fail(PA_ERR_INVALID_ARG, "pa_swap_in: host buffer missing or smaller than pa_swap_bytes");
    const int32_t n = (s.len + p->cfg.block_size - 1) / p->cfg.block_size;
    std::vector<int32_t> blocks;
    std::vector<std::pair<int32_t, uint64_t>> evicted;   // for rollback
    for (int32_t i = 0; i < n; ++i) {
        int32_t b;
        bool ev;
        uint64_t key;
        pa_status st = pop_block(p, &b, &ev, &key);
        if (st != PA_OK) {
            std::string msg = pa_last_error();
            for (int32_t j = (int32_t)blocks.size() - 1; j >= 0; --j) {   // undo in reverse
                const int32_t x = blocks[j];
                p->refcount[x] = 0;
                if (evicted[j].first) {
                    register_key(p, x, evicted[j].second);
                    ev_push_front(p, x);
                    --p->cache_evictions;
                } else {
                    p->free_stack.push_back(x);
                }
            }
            return fail(st, "pa_swap_in: " + msg + " (no change made)");
        }
        blocks.push_back(b);
        evicted.push_back({ev ? 1 : 0, key});
    }
    if (p->k_pool) {
        pa_status st = pa_internal::swap_copy(p, blocks.data(), n, const_cast<void *>(host_buf), false, stream);
        if (st != PA_OK) {   // launch failed: give the blocks back
            for (int32_t j = n - 1; j >= 0; --j) {
                p->refcount[blocks[j]] = 0;
                p->free_stack.push_back(blocks[j]);
            }
            return st;
        }
    }
    s.table = std::move(blocks);
    s.swapped = false;
    note_usage(p);
    return PA_OK;
}

uint64_t pa_launch_count(void) { return pa_internal::launch_count.load(); }

}  // extern "C"
