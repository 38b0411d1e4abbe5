// Internal definition of the opaque pa_pool and shared host helpers.
#pragma once

#include <cuda.h>
#include <nvtx3/nvToolsExt.h>

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
    void *scales = nullptr;   // FP8 pools: device scale bytes [L][NB][Hkv][K, V][B]

    // Free list: a LIFO stack; back() is handed out next.
    std::vector<int32_t> free_stack;
    std::vector<int32_t> refcount;

    struct Seq {
        std::vector<int32_t> table;   // logical block -> physical block
        int32_t len = 0;              // tokens
        bool swapped = false;         // blocks live in host memory (pa_swap_out)
        uint64_t seen = 0;            // last batch call that listed this sequence
    };
    std::unordered_map<int32_t, Seq> seqs;
    int32_t next_seq = 0;
    uint64_t batch_calls = 0;         // numbers batch calls, for the duplicate-id check

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
    int tmap_rows = 0;                // box height of the cached descriptors
    CUtensorMap tmap_k;
    CUtensorMap tmap_v;

    bool fp8() const { return cfg.dtype == PA_FP8_E4M3; }
    // type of queries, appended rows and 16-bit outputs
    pa_dtype act_dtype() const { return fp8() ? cfg.act_dtype : cfg.dtype; }
    size_t elem_bytes() const { return cfg.dtype == PA_F32 ? 4 : fp8() ? 1 : 2; }
    size_t act_bytes() const { return act_dtype() == PA_F32 ? 4 : 2; }
    // FP8 pools: scale bytes of one block (all heads, K and V) in one layer, and of a layer
    size_t scale_block_bytes() const { return fp8() ? (size_t)2 * cfg.num_kv_heads * cfg.block_size : 0; }
    size_t scale_layer_bytes() const { return scale_block_bytes() * (size_t)cfg.num_blocks; }
    // one [block][layer] record of a swap buffer: K codes, V codes, then the scales
    size_t swap_record_bytes() const { return 2 * block_bytes() + scale_block_bytes(); }
    bool device_ready() const { return k_pool && (!fp8() || scales); }
    // bytes of one (block, kv-head) tile and of one block across heads
    size_t tile_bytes() const { return (size_t)cfg.block_size * cfg.head_dim * elem_bytes(); }
    size_t block_bytes() const { return tile_bytes() * cfg.num_kv_heads; }
    size_t layer_bytes() const { return block_bytes() * (size_t)cfg.num_blocks; }
};

namespace pa_internal {
// NVTX range named after a library call, so profiler timelines (Nsight Systems, the
// NVTX filters of Nsight Compute) show where each call's host work and launches sit.
// Without a tool attached a push or pop is a check of one function pointer.
struct TraceRange {
    explicit TraceRange(const char *name) { nvtxRangePushA(name); }
    ~TraceRange() { nvtxRangePop(); }
    TraceRange(const TraceRange &) = delete;
    TraceRange &operator=(const TraceRange &) = delete;
};

// Records `msg` as this thread's last error and returns `st`.
pa_status fail(pa_status st, const std::string &msg);
pa_status ok();
extern std::atomic<uint64_t> launch_count;
// Device side of swapping (kernels.cu): copy `blocks` between the pools and a host
// buffer of [block][layer] records (K codes, V codes, then for FP8 pools the block's
// scale bytes); to_host selects the direction.
pa_status swap_copy(const pa_pool *pool, const int32_t *blocks, int32_t n, void *host_buf, bool to_host,
                    void *stream);
}  // namespace pa_internal
