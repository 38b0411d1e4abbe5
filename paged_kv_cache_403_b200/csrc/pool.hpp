// Internal definition of the opaque pa_pool and shared host helpers.
#pragma once

#include <cuda.h>

#include <atomic>
#include <cstdint>
#include <string>
#include <unordered_map>
#include <vector>

#include "pa.h"

struct pa_pool {
    pa_pool_config cfg;
    void *k_pool = nullptr;   // device, [L][NB][Hkv][B][D]
    void *v_pool = nullptr;

    // Free list: a LIFO stack; back() is handed out next.
    std::vector<int32_t> free_stack;
    std::vector<int32_t> refcount;

    struct Seq {
        std::vector<int32_t> table;   // logical block -> physical block
        int32_t len = 0;              // tokens
        bool swapped = false;         // blocks live in host memory (pa_swap_out)
    };
    std::unordered_map<int32_t, Seq> seqs;
    int32_t next_seq = 0;

    int64_t num_tokens = 0;
    int64_t cow_copies = 0;
    int32_t num_shared = 0;           // blocks with refcount > 1
    int32_t peak_used = 0;
    int64_t fail_alloc_after = -1;    // host fault injection (< 0: off)

    // Prefix caching: registered full blocks (key <-> block) and the queue of
    // registered blocks whose refcount fell to zero, least recently released first
    // (an intrusive doubly linked list over block ids).
    std::unordered_map<uint64_t, int32_t> block_of;
    std::vector<uint64_t> key_of;
    std::vector<char> has_key;
    std::vector<int32_t> ev_prev, ev_next;
    std::vector<char> in_ev;
    int32_t ev_head = -1, ev_tail = -1, ev_count = 0;
    int64_t cache_hits = 0, cache_evictions = 0;

    // TMA descriptors over the whole key / value pools, viewed as 2-D tensors of
    // [num_layers * num_blocks * num_kv_heads * block_size rows][head_dim]; built on
    // the first decode call (16-bit caches only).
    bool tmaps_ready = false;
    CUtensorMap tmap_k;
    CUtensorMap tmap_v;

    size_t elem_bytes() const { return cfg.dtype == PA_F32 ? 4 : 2; }
    // bytes of one (block, kv-head) tile and of one block across heads
    size_t tile_bytes() const { return (size_t)cfg.block_size * cfg.head_dim * elem_bytes(); }
    size_t block_bytes() const { return tile_bytes() * cfg.num_kv_heads; }
    size_t layer_bytes() const { return block_bytes() * (size_t)cfg.num_blocks; }
};

namespace pa_internal {
// Records `msg` as this thread's last error and returns `st`.
pa_status fail(pa_status st, const std::string &msg);
pa_status ok();
extern std::atomic<uint64_t> launch_count;
// Device side of swapping (kernels.cu): copy `blocks` between the pools and a host
// buffer laid out [block][layer][K, V][Hkv][B][D]; to_host selects the direction.
pa_status swap_copy(const pa_pool *pool, const int32_t *blocks, int32_t n, void *host_buf, bool to_host,
                    void *stream);
}  // namespace pa_internal
