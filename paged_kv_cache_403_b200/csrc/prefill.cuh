// Paged chunked-prefill attention on the 5th-generation tensor cores (tcgen05, TMEM).
// Included by kernels.cu (shares its device error word, mbarrier and TMA helpers).
//
// "What problem does PagedAttention solve, and what is continuous batching?": prefill
// is the compute-heavy pass over the prompt ("Why the KV cache becomes the problem")
// and long prompts are broken into chunks ("The prefill and decode phases need careful
// scheduling").  A chunk is the last C tokens of a sequence whose keys and values are
// already in the paged cache; query i of the chunk (absolute position L - C + i)
// attends to keys 0 .. L - C + i, read through the block table.
//
// One CTA per (256 query rows, KV head, sequence): two 128-row tiles A and B whose rows
// are (token, query head of the GQA group) pairs, row = token * G + head, so every
// query head of the group shares each key/value tile.  Warp roles:
//   warps 0-7        softmax, one thread per row: warp w serves tile w / 4 and rows
//                    32 (w % 4) .. +31 (its TMEM lane quarter), so each SM sub-partition
//                    holds one softmax warp of each tile.  Per row and key tile: the
//                    128 scores come out of TMEM in four loads with one wait, the row
//                    maximum needs no other thread, a causal / length mask by select on
//                    the last tiles only, base-2 online softmax with a lazily moved
//                    maximum (the O row is rescaled in TMEM only when a score passes the
//                    running maximum by 2^8), and P written back to TMEM (tcgen05.st) as
//                    the A operand of P V: for bf16 a truncated high part plus the
//                    truncated remainder, for fp16 once;
//   warp 8           tensor-core issue, one thread: S_t = Q_t K^T (M=128, N=128 keys,
//                    both operands in shared memory) and O_t += P_t V (M=128,
//                    N=head_dim, per part of P; A = P from TMEM, B = V from shared
//                    memory).  The tensor core keeps almost no queue of its own, so this
//                    thread does nothing but wait and issue: a cycle it spends elsewhere
//                    is a cycle the tensor core idles;
//   warp 9           TMA producer: 128-key tiles of K and V (2-D tensor loads, 128-byte
//                    swizzle) into a 2-stage ring, walking the block table; it also zeroes
//                    the last value tile's rows past the sequence end.
// Tiles of 128 keys make S = Q K^T an M=128, N=128 product (64 cycles at the dense
// rate; an N=64 product takes 48, two thirds of that rate).  TMEM then holds O and S of both query tiles (512
// columns), so P is written over S in place: the 16 columns of each 16-key group of S
// take that group's P (8 columns of high parts, 8 of low parts), and the next S of the
// tile is issued after the P V that reads them (one thread's tcgen05.mma run in order).
// The two tiles ping-pong: while one tile's softmax computes exponentials the tensor
// core works on the other tile.  Every hand-off is an mbarrier; every wait is bounded and
// sets a shared abort flag that all roles check; TMEM is always freed.  Value rows past
// the sequence end are zeroed in shared memory before P V (weight 0, but 0 * NaN would
// not be 0).
namespace prefill {

constexpr int kRows = 128;           // MMA M: rows of one query tile
constexpr int kTiles = 2;            // query tiles per CTA (ping-pong)
constexpr int kKeys = 128;           // keys per K/V tile
constexpr int kSoftmaxWarps = kTiles * kRows / 32;   // one thread per query row
constexpr int kThreads = kSoftmaxWarps * 32 + 64;   // + tensor-core issue warp + TMA warp
constexpr int kMmaWarp = kSoftmaxWarps, kTmaWarp = kMmaWarp + 1;
constexpr int kD = 128;              // head_dim
// TMEM columns: O_A [0,128) O_B [128,256) S_A [256,384) S_B [384,512); after the
// softmax, columns [16g, 16g+8) of S_t hold the high parts of keys 16g..16g+15 of P_t
// (two 16-bit values per column) and [16g+8, 16g+16) the low parts.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 0, kSCol = 256;
constexpr int kQBytes = kRows * kD * 2;         // 32 KB per tile: [2 halves][128 rows][128 B]
constexpr int kKVBytes = kKeys * kD * 2;        // 32 KB: [2 halves][128 rows][128 B]
constexpr int kStages = 2;
// s_full, p_full, o_done per tile; k/v full, empty per stage; v_fixed (the last value
// tile after its rows past the sequence end were zeroed)
constexpr int kNumBars = 3 * kTiles + 4 * kStages + 1;
constexpr int kSmemBytes = 1024 + kTiles * kQBytes + kStages * 2 * kKVBytes + kNumBars * 8 + 16;

// --- tcgen05 wrappers --------------------------------------------------------------
// Shared-memory matrix descriptor, 128-byte swizzle: start address, leading and stride
// byte offsets in 16-byte units, descriptor version 1, layout code 2 (SWIZZLE_128B).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor of kind::f16: fp32 accumulator, A/B format (0 = f16, 1 = bf16),
// A/B major-ness (0 = K-major, 1 = MN-major), N / 8 and M / 16.
__host__ __device__ constexpr uint32_t instr_desc(uint32_t fmt, uint32_t m, uint32_t n, uint32_t a_mn,
                                                  uint32_t b_mn) {
    return (1u << 4) | (fmt << 7) | (fmt << 10) | (a_mn << 15) | (b_mn << 16) | ((n >> 3) << 17) |
           ((m >> 4) << 24);
}

__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

// the same with A read from tensor memory (a_tmem: lane = row, two 16-bit K elements
// per 32-bit column, 8 columns per K = 16 step)
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// generic-proxy shared-memory writes become visible to the tensor core (async proxy)
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Bounded wait for a whole warp (lanes leave together); gives up when another role has
// set the abort flag or after the wait bound (wait_limit_ns()), setting the flag itself then.
__device__ __forceinline__ bool wait_warp(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    uint64_t t0 = 0, limit = kWaitLimitNs;
    for (uint32_t it = 0;; ++it) {
        const bool done = mbar_try_wait(bar, parity);
        if (__all_sync(0xffffffffu, done)) return true;
        if (it == 0) {
            t0 = global_timer_ns();
            limit = wait_limit_ns();
        }
        const bool give_up = *abort_flag || global_timer_ns() - t0 > limit;
        if (__any_sync(0xffffffffu, give_up)) {
            if ((threadIdx.x & 31) == 0 && !*abort_flag) {
                raise_error(kErrTimeout);
                *abort_flag = 1;
            }
            return false;
        }
    }
}

// The same for one thread (the tensor-core issuer): the tensor core's queue is short, so
// every cycle this thread spends outside tcgen05.mma is a cycle the tensor core may idle.
__device__ __forceinline__ bool wait_one(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns(), limit = wait_limit_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag || global_timer_ns() - t0 > limit) {
            if (!*abort_flag) {
                raise_error(kErrTimeout);
                *abort_flag = 1;
            }
            return false;
        }
    }
    return true;
}

// Operand format code of the instruction descriptor, and how P enters P V: bf16 P
// keeps 8 significant bits, too few for the 2e-3 bound on peaky rows, so a bf16 P is a
// high part (the truncation of p to bf16) plus the truncation of the exact remainder
// p - high (>= 14 bits together, two products), both taken with byte permutes so the
// conversion unit only computes exponentials; an fp16 P keeps 11 bits and enters once.
template <typename T>
struct Fmt;
template <>
struct Fmt<__half> {
    static constexpr uint32_t code = 0;
    static constexpr bool two_parts = false;
};
template <>
struct Fmt<__nv_bfloat16> {
    static constexpr uint32_t code = 1;
    static constexpr bool two_parts = true;
};

// Pairs of fp32 values in one 64-bit register (element 0 in the low half) and the packed
// fp32x2 arithmetic of sm_100, which does two fp32 operations per instruction.
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void unpack_f32x2(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ uint32_t byte_perm(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}


struct Params {
    CUtensorMap tmap_k;
    CUtensorMap tmap_v;
    const void *q;              // [total_q][Hq][D]
    void *out;                  // [total_q][Hq][D]
    const int32_t *tables;      // [n][max_blocks]
    const int32_t *lens;        // [n] total tokens (context + chunk)
    const int32_t *q_start;     // [n + 1]
    int32_t max_blocks, num_blocks, num_kv_heads, num_q_heads, layer, block_size, out_f32;
    int32_t debug_withhold;     // see copies_withheld(); -1 outside wait-expiry tests
    float scale_log2;
};

template <typename T, int B>
__global__ void __launch_bounds__(kThreads, 1) paged_prefill_kernel(const __grid_constant__ Params p) {
    constexpr int BLOCKS_PER_TILE = kKeys / B;
    constexpr uint32_t IDESC_S = instr_desc(Fmt<T>::code, kRows, kKeys, 0, 0);
    constexpr uint32_t IDESC_O = instr_desc(Fmt<T>::code, kRows, kD, 0, 1);
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    unsigned char *sQ = smem;                                       // tile t at t * kQBytes
    unsigned char *sKV = sQ + kTiles * kQBytes;                     // stage st: K then V
    uint64_t *bars = reinterpret_cast<uint64_t *>(sKV + kStages * 2 * kKVBytes);
    // K and V slots are released separately: a K tile is free once both query tiles'
    // S used it, long before P V is done with the V tile beside it
    uint64_t *k_full = bars, *k_empty = bars + kStages, *v_full = bars + 2 * kStages, *v_empty = bars + 3 * kStages;
    uint64_t *s_full = bars + 4 * kStages, *p_full = s_full + kTiles, *o_done = p_full + kTiles;
    uint64_t *v_fixed = o_done + kTiles;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kNumBars);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int s = blockIdx.z;
    const int g = blockIdx.y;
    const int group = p.num_q_heads / p.num_kv_heads;
    const int tokens_per_cta = kTiles * kRows / group;
    const int q0 = p.q_start[s];
    const int C = p.q_start[s + 1] - q0;
    const int t0 = blockIdx.x * tokens_per_cta;
    if (t0 >= C) return;
    const int L = p.lens[s];
    const int nblk = (L + B - 1) / B;
    if (L < 1 || C > L || nblk > p.max_blocks) {
        if (threadIdx.x == 0) raise_error(kErrBadLen);
        return;
    }
    const int P0 = L - C;                                    // position of the chunk's first token
    const int t_last = min(C, t0 + tokens_per_cta) - 1;
    const int n_tiles = (P0 + t_last) / kKeys + 1;           // keys 0 .. P0 + t_last
    const bool has_b = t0 + kRows / group < C;               // tile B holds at least one token
    const int n_qt = has_b ? 2 : 1;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
        }
        for (int t = 0; t < kTiles; ++t) {
            mbar_init(&s_full[t], 1);
            mbar_init(&p_full[t], 4);   // the four softmax warps of the tile
            mbar_init(&o_done[t], 1);
        }
        mbar_init(v_fixed, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == kMmaWarp) {   // TMEM: the issuing warp allocates and frees
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // softmax warp w: tile w / 4, lane quarter w % 4; each loads its query row (rows past
    // the chunk are zero)
    const int quarter = warp & 3;
    const int qtile = (warp >> 2) & 1;
    const int row = quarter * 32 + lane;
    const int my_t = t0 + (qtile * kRows + row) / group;
    const int my_h = g * group + row % group;
    const bool row_valid = warp < kSoftmaxWarps && my_t < C;
    if (warp < kSoftmaxWarps) {
        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const T *>(p.q) +
                                                            ((size_t)(q0 + (row_valid ? my_t : 0)) * p.num_q_heads + my_h) * kD);
        unsigned char *dst = sQ + qtile * kQBytes;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const uint4 v = row_valid ? src[c] : make_uint4(0, 0, 0, 0);
            const int half = c >> 3, cc = c & 7;
            *reinterpret_cast<uint4 *>(dst + half * (kQBytes / 2) + row * 128 + ((cc ^ (row & 7)) << 4)) = v;
        }
        fence_proxy_async();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == kTmaWarp) {
        // ---------------- producer: walk the table, keep the ring full
        const int32_t *trow = p.tables + (size_t)s * p.max_blocks;
        int issued_k = 0, issued_v = 0;   // tiles whose K / V copies were issued
        // a wait-expiry test withholds every copy of one CTA: its other roles' waits run out
        const int to_issue = copies_withheld(p.debug_withhold) ? 0 : n_tiles;
        for (int j = 0; j < to_issue; ++j) {
            const int st = j % kStages;
            int blk = 0;
            if (lane < BLOCKS_PER_TILE) {
                const int lb = j * BLOCKS_PER_TILE + lane;
                blk = trow[lb < nblk ? lb : 0];      // past the end: finite data, masked and zeroed
                if ((unsigned)blk >= (unsigned)p.num_blocks) {
                    raise_error(kErrBadBlock);
                    blk = 0;
                }
            }
            unsigned char *k_dst = sKV + st * 2 * kKVBytes;
            for (int kv = 0; kv < 2; ++kv) {
                uint64_t *full = kv == 0 ? &k_full[st] : &v_full[st];
                uint64_t *empty = kv == 0 ? &k_empty[st] : &v_empty[st];
                if (j >= kStages && !wait_warp(empty, ((j / kStages) - 1) & 1, abort_flag)) break;
                if (lane == 0) mbar_arrive_expect_tx(full, kKVBytes);
#pragma unroll
                for (int b = 0; b < BLOCKS_PER_TILE; ++b) {
                    const int bb = __shfl_sync(0xffffffffu, blk, b);
                    if (lane == 0) {
                        const int r0 = ((p.layer * p.num_blocks + bb) * p.num_kv_heads + g) * B;
                        for (int h = 0; h < 2; ++h)
                            tma_load_2d(k_dst + kv * kKVBytes + h * (kKVBytes / 2) + b * B * 128,
                                        kv == 0 ? &p.tmap_k : &p.tmap_v, h * 64, r0, full);
                    }
                }
                if (kv == 0)
                    issued_k = j + 1;
                else
                    issued_v = j + 1;
            }
            if (*abort_flag) break;
            __syncwarp();
        }
        // Value rows past the sequence end (only the last tile has any) are zeroed here, once
        // that tile's copy has landed, and handed to the tensor-core thread through v_fixed:
        // their weights are 0, but 0 * NaN would not be 0.
        const int last = n_tiles - 1;
        const int first_bad = L - last * kKeys;
        if (issued_v == n_tiles && first_bad < kKeys &&
            wait_warp(&v_full[last % kStages], (last / kStages) & 1, abort_flag)) {
            unsigned char *v_st = sKV + (last % kStages) * 2 * kKVBytes + kKVBytes;
            for (int rr = lane; rr < 2 * kKeys; rr += 32) {
                const int r = rr >> 1, half = rr & 1;
                if (r >= first_bad) {
                    uint4 *dst = reinterpret_cast<uint4 *>(v_st + half * (kKVBytes / 2) + r * 128);
#pragma unroll
                    for (int c = 0; c < 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
                }
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(v_fixed);
        }
        // every issued copy lands before the CTA frees its shared memory, also after an abort
        if (lane == 0) {
            drain_copies(k_full, issued_k, kStages);
            drain_copies(v_full, issued_v, kStages);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ---------------- tensor-core issue, one thread (the others wait at the end)
        if (lane == 0) {
            const int last = n_tiles - 1;
            const bool fixed_last = L - last * kKeys < kKeys;   // the producer zeroes its tail rows
            auto ready_k = [&](int j) -> bool {
                if (!wait_one(&k_full[j % kStages], (j / kStages) & 1, abort_flag)) return false;
                fence_after_sync();
                return true;
            };
            auto ready_v = [&](int j) -> bool {
                if (!wait_one(&v_full[j % kStages], (j / kStages) & 1, abort_flag)) return false;
                if (j == last && fixed_last && !wait_one(v_fixed, 0, abort_flag)) return false;
                fence_after_sync();
                return true;
            };
            // Descriptors are built once: the start address sits in the low 14 bits as
            // addr >> 4 (shared memory < 256 KB), so moving to another tile, stage or K step
            // is one add of offset >> 4.
            const uint64_t q_desc = smem_desc(smem_addr(sQ), 16, 1024);
            const uint64_t k_desc = smem_desc(smem_addr(sKV), 16, 1024);
            const uint64_t v_desc = smem_desc(smem_addr(sKV + kKVBytes), kKVBytes / 2, 1024);
            auto issue_s = [&](int t, int j) {
                const uint64_t qa = q_desc + (uint64_t)((t * kQBytes) >> 4);
                const uint64_t kb = k_desc + (uint64_t)(((j % kStages) * 2 * kKVBytes) >> 4);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t qo = ((kk >> 2) * (kQBytes / 2) + (kk & 3) * 32) >> 4;
                    const uint32_t ko = ((kk >> 2) * (kKVBytes / 2) + (kk & 3) * 32) >> 4;
                    umma(tmem + kSCol + t * kKeys, qa + qo, kb + ko, IDESC_S, kk > 0);
                }
                umma_commit(&s_full[t]);
            };
            auto issue_pv = [&](int t, int j) {
                const uint32_t pcol = tmem + kSCol + t * kKeys;
                const uint64_t vb = v_desc + (uint64_t)(((j % kStages) * 2 * kKVBytes) >> 4);
#pragma unroll
                for (int kk = 0; kk < kKeys / 16; ++kk) {
                    const uint64_t b = vb + (uint64_t)((kk * 16 * 128) >> 4);
                    umma_ts(tmem + kOCol + t * kD, pcol + kk * 16, b, IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
                    if (Fmt<T>::two_parts) umma_ts(tmem + kOCol + t * kD, pcol + kk * 16 + 8, b, IDESC_O, 1u);
                }
                umma_commit(&o_done[t]);
            };
            bool ok = ready_k(0);
            if (ok) {
                for (int t = 0; t < n_qt; ++t) issue_s(t, 0);
                umma_commit(&k_empty[0]);   // K(0) free once both S(0) are done
            }
            for (int j = 0; j < n_tiles && ok; ++j) {
                for (int t = 0; t < n_qt; ++t) {
                    // softmax t read S_t(j) and wrote P_t(j)
                    if (!(ok = wait_one(&p_full[t], j & 1, abort_flag))) break;
                    fence_after_sync();
                    if (t == 0 && !(ok = ready_v(j))) break;
                    // P_t(j) V(j) first: S_t(j+1) overwrites the columns P_t(j) is read from
                    issue_pv(t, j);
                    if (t == n_qt - 1) umma_commit(&v_empty[j % kStages]);   // V(j) read for the last time
                    if (j + 1 < n_tiles) {
                        if (t == 0 && !(ok = ready_k(j + 1))) break;
                        issue_s(t, j + 1);
                    }
                }
                if (ok && j + 1 < n_tiles) umma_commit(&k_empty[(j + 1) % kStages]);
            }
        }
        __syncwarp();
    } else {
        // ---------------- softmax of tile qtile, one thread per row = TMEM lane
        const bool tile_used = qtile < n_qt;
        const int kmax = row_valid ? P0 + my_t : -1;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t s_col = kSCol + qtile * kKeys;
        const uint32_t o_col = kOCol + qtile * kD;
        const float sl = p.scale_log2;
        float m = -INFINITY, l = 0.f;
        bool ok = tile_used;
        for (int j = 0; j < n_tiles && ok; ++j) {
            ok = wait_warp(&s_full[qtile], j & 1, abort_flag);
            if (!ok) break;
            fence_after_sync();
            const int key0 = j * kKeys;
            // the row's 128 scores: four loads in flight, one wait
            uint32_t v[kKeys / 32][32];
#pragma unroll
            for (int c = 0; c < kKeys / 32; ++c) tmem_ld32(tmem + lane_base + s_col + 32 * c, v[c]);
            tmem_wait_ld();
            // interior tiles need no mask; the last ones mask by select (keys past this
            // row's position or past the sequence end get weight 0)
            if (!(key0 + kKeys - 1 <= kmax && key0 + kKeys <= L)) {
#pragma unroll
                for (int e = 0; e < kKeys; ++e) {
                    const int key = key0 + e;
                    if (!(key <= kmax && key < L)) v[e >> 5][e & 31] = __float_as_uint(-INFINITY);
                }
            }
            // maximum on raw scores (scale > 0 keeps the order), 8 chains
            float mx8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) mx8[e] = -INFINITY;
#pragma unroll
            for (int e = 0; e < kKeys; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], __uint_as_float(v[e >> 5][e & 31]));
            const float tmax = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                     fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * sl;
            // The running maximum moves only when a score passes it by 2^8; the O row is
            // then rescaled by f below, after P is written (the scores are dead by then).
            const bool need = tmax > m + kRescaleThreshold;
            const float f = need ? ex2(m - tmax) : 1.f;
            if (need) {
                l *= f;
                m = tmax;
            }
            // p = 2^(s * scale_log2 - m), one FMA and one ex2 per score (-inf -> 0), written
            // over the row's own S columns: per 16 keys, 8 columns of high parts then 8 of
            // low parts
            const float neg_m = m == -INFINITY ? 0.f : -m;
            const uint64_t sl2 = f32x2(sl, sl), nm2 = f32x2(neg_m, neg_m);
            uint64_t lp2[2] = {0ull, 0ull};                   // two pairs of running sums
#pragma unroll
            for (int c = 0; c < kKeys / 32; ++c) {
                uint32_t pw[32];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float x0, x1;
                    unpack_f32x2(fma_f32x2(f32x2(__uint_as_float(v[c][2 * e]), __uint_as_float(v[c][2 * e + 1])), sl2,
                                           nm2),
                                 x0, x1);
                    const float p0 = ex2(x0), p1 = ex2(x1);
                    const uint64_t p2 = f32x2(p0, p1);
                    const int slot = (e >> 3) * 16 + (e & 7);     // key group e/8, pair e%8
                    if (Fmt<T>::two_parts) {
                        // high halves of the two fp32 words = their bf16 truncations; the
                        // remainders (exact in fp32, >= 0) truncated the same way
                        const uint32_t b0 = __float_as_uint(p0), b1 = __float_as_uint(p1);
                        pw[slot] = byte_perm(b0, b1, 0x7632u);
                        float r0, r1;
                        unpack_f32x2(add_f32x2(p2, f32x2(__uint_as_float((b0 & 0xffff0000u) ^ 0x80000000u),
                                                         __uint_as_float((b1 & 0xffff0000u) ^ 0x80000000u))),
                                     r0, r1);
                        pw[slot + 8] = byte_perm(__float_as_uint(r0), __float_as_uint(r1), 0x7632u);
                    } else {
                        pw[slot] = Mma<T>::pack(p0, p1);
                        pw[slot + 8] = 0u;
                    }
                    lp2[e & 1] = add_f32x2(lp2[e & 1], p2);
                }
                tmem_st32(tmem + lane_base + s_col + 32 * c, pw);
            }
            {
                float a0, a1, b0, b1;
                unpack_f32x2(lp2[0], a0, a1);
                unpack_f32x2(lp2[1], b0, b1);
                l += (a0 + a1) + (b0 + b1);
            }
            // The rescale is warp-wide (tcgen05.ld / st are); rows that do not need it scale
            // by 1.  P_t(j-1) V(j-1) completed before S_t(j) (issued after it on the same
            // thread), so O_t is settled, and P_t(j) V(j) waits for this tile's arrival.
            if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
                for (int c0 = 0; c0 < kD; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_base + o_col + c0, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
                    tmem_st32(tmem + lane_base + o_col + c0, o);
                }
            }
            tmem_wait_st();
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[qtile]);
        }
        if (ok) ok = wait_warp(&o_done[qtile], (n_tiles - 1) & 1, abort_flag);
        if (ok) {
            fence_after_sync();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const size_t orow = ((size_t)(q0 + my_t) * p.num_q_heads + my_h) * kD;
#pragma unroll
            for (int c0 = 0; c0 < kD; c0 += 32) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_base + o_col + c0, o);
                tmem_wait_ld();
                if (row_valid) {
                    if (p.out_f32) {
                        float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.out) + orow + c0);
#pragma unroll
                        for (int c = 0; c < 32; c += 4)
                            dst[c / 4] = make_float4(__uint_as_float(o[c]) * inv, __uint_as_float(o[c + 1]) * inv,
                                                     __uint_as_float(o[c + 2]) * inv, __uint_as_float(o[c + 3]) * inv);
                    } else {
                        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<T *>(p.out) + orow + c0);
#pragma unroll
                        for (int c = 0; c < 32; c += 8) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                w[e] = Mma<T>::pack(__uint_as_float(o[c + 2 * e]) * inv,
                                                    __uint_as_float(o[c + 2 * e + 1]) * inv);
                            dst[c / 8] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        fence_after_sync();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace prefill
