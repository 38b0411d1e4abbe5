// FP8 (E4M3) KV cache: quantising append and tensor-core decode attention.
// Included by kernels.cu after the 16-bit decode kernel, whose PTX wrappers
// (mbarriers, TMA, ldmatrix, movmatrix, mma) it reuses.
//
// Why: "What problem does PagedAttention solve, and what is continuous batching?",
// section "Common misconception" -- paging leaves the bytes per cached token as they
// are; KV-cache quantisation reduces them.  Decode attention reads every cached byte
// once, so at the same HBM roofline half the bytes is twice the tokens per second.
//
// Format (stated in pa.h): E4M3 codes, plus one power-of-two scale per (token, KV
// head) row stored as a byte e (factor 2^(e - 127)) in separate scale arrays
// [layer][block][kv head][block_size].  The value of element i of a row is
// E4M3(code_i) * 2^(e - 127).
//
// Decode design (head_dim 128).  Same skeleton as the 16-bit tensor-core kernel: a
// producer warp fills a ring of shared-memory stages by TMA (one 2-D box of rows x
// 128 code bytes for K and one for V, 128-byte swizzle, plus one 1-D bulk copy of the
// tile's scale bytes), and four consumer warps each take whole tiles.  A tile holds
// one block of HEADS neighbouring KV heads: at 1 byte per element a single head's
// block is only block_size x 128 bytes, and copies that small left the copy engine,
// not HBM, as the limit.  E4M3 values are
// exact in fp16 (times 2^-8, folded into the scale factors), so the consumers widen
// codes with a byte permute, a shift and a mask and run the same m16n8k16 fp16
// products:
//   S^T[16 tok][8 heads] = K[16][128] . Q^T   ldmatrix reads 4 code bytes of a row per
//                                             lane; the query fragments use the same
//                                             order of the head dimension, so the
//                                             products pair the right elements.
//   O^T[128][8]         += V^T . P^T          ldmatrix.trans + two byte permutes give a
//                                             lane the codes of tokens 2t, 2t+1, 2t+8,
//                                             2t+9 for two neighbouring dims 2g, 2g+1;
//                                             the output rows are relabelled to match.
// Scales: a key row's 2^X multiplies that token's scores (folded into the score
// factor with scale * log2(e) and the query's own power-of-two prescale).  A value
// row's 2^X multiplies that token's softmax weight, and a large value exponent can
// outweigh a small weight, so the output keeps its own running reference: weights for
// P.V are 2^(s + X_v - m_o), with m_o a lazily raised maximum of s + X_v, while the
// denominator sums 2^(s - m) against the usual running maximum m of the scores.  Both
// stay <= 2^8, in fp16 range, and the end multiplies the output by 2^(m_o - m).  The
// query is multiplied by a power of two that puts its largest element in [2^14, 2^15)
// before it is rounded to fp16, so bf16 queries keep their bits.
namespace fp8 {

constexpr int kD = 128;

// round two fp32 values to E4M3 (nearest, ties to even, saturating); `lo` -> byte 0
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// Two E4M3 codes -> an f16x2 word holding value * 2^-8 each, exactly (normal and
// subnormal codes alike: the code's 4 exponent and 3 mantissa bits become f16
// exponent bits 13..10 and mantissa bits 9..7, and the two biases differ by 8).
// `sel` is a byte-permute selector over the eight bytes of (a, b) that puts code A in
// byte 0, A's sign replicated in byte 1, code B in byte 2 and B's sign in byte 3.
// The shift by 7 moves each code's low seven bits into place and a sign byte's lowest
// bit onto bit 15 of its half; the mask drops the code's own sign (now bit 14) and
// what the low sign byte spilled into the high half.  Integer pipes only, where the
// hardware conversion (cvt.f16x2.e4m3x2) would queue on the conversion unit.
__device__ __forceinline__ uint32_t codes_to_f16x2(uint32_t a, uint32_t b, uint32_t sel) {
    return (prmt(a, b, sel) << 7) & 0xBF80BF80u;
}

// 2^k for an exponent field k (1..254 -> normal powers of two; <= 0 -> 0)
__device__ __forceinline__ float pow2_field(int k) { return k > 0 ? __uint_as_float((uint32_t)min(k, 254) << 23) : 0.f; }

// ------------------------------------------------------------------ append
struct AppendParams {
    unsigned char *k_layer;         // codes of this layer [NB][Hkv][B][D]
    unsigned char *v_layer;
    unsigned char *s_layer;         // scale bytes of this layer [NB][Hkv][K, V][B]
    const unsigned char *k_new;     // [n][Hkv][D] of the activation type
    const unsigned char *v_new;
    const int64_t *slots;
    int32_t n_tokens, block_size, num_kv_heads;
    int64_t num_blocks;
    Div32 by_heads, by_block;       // num_kv_heads, block_size (32-bit index form)
};

// kAppendLanes lanes per (token, head) row of K or V, so a warp quantises 32 / kAppendLanes
// rows at once and the per-row work (index arithmetic, slot check, the exponent) is shared
// by lanes of D / kAppendLanes elements each -- with a warp per row the kernel was bound by
// instruction issue, not memory.  amax by a max over the row's lanes of the fp32 bit
// patterns (non-negative floats order like their bits), the row exponent from the bits of
// amax, one fp32 multiply by 2^-X per element, then E4M3 rounding.  The rows of a warp may
// take different paths (a padding slot, a bad slot), so every shuffle is executed by the
// whole warp and only the stores are guarded.
constexpr int kAppendLanes = 4;
template <typename T, int D, bool NARROW>
__global__ void __launch_bounds__(256) append_kernel(const AppendParams p) {
    constexpr int LPR = kAppendLanes, RPW = 32 / LPR;   // lanes per row, rows per warp
    constexpr int EPL = D / LPR;                         // elements per lane: 8, 16 or 32
    static_assert(EPL == 8 || EPL == 16 || EPL == 32, "head_dim 64 or 128");
    constexpr int NQ = EPL / 8;                          // 16-byte loads per lane
    const int lane = threadIdx.x & 31;
    const int rl = lane % LPR;                           // lane within the row
    const int64_t rows = (int64_t)p.n_tokens * p.num_kv_heads;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); RPW * w < 2 * rows; w += warps) {
        const int64_t r = RPW * w + lane / LPR;           // this row: K rows, then V rows
        bool valid = r < 2 * rows;
        const bool is_v = r >= rows;
        const int64_t rr = is_v ? r - rows : r;
        int64_t i = 0;
        int h = 0;
        if (valid) {
            if constexpr (NARROW) {   // 32-bit index arithmetic (see Div32)
                i = div32((uint32_t)rr, p.by_heads);
                h = (int)((uint32_t)rr - (uint32_t)i * (uint32_t)p.num_kv_heads);
            } else {
                i = rr / p.num_kv_heads;
                h = (int)(rr % p.num_kv_heads);
            }
        }
        // the row is read before the slot is looked at, so the loads overlap
        uint4 u[NQ] = {};
        int64_t slot = -1;
        if (valid) {
            const uint4 *src = reinterpret_cast<const uint4 *>((is_v ? p.v_new : p.k_new) +
                                                               (size_t)(rr * D + rl * EPL) * sizeof(T));
#pragma unroll
            for (int k = 0; k < NQ; ++k) u[k] = src[k];
            slot = p.slots[i];
        }
        if (valid && slot >= p.num_blocks * p.block_size) {
            if (rl == 0 && !is_v) raise_error(kErrBadSlot);
            valid = false;
        }
        if (slot < 0) valid = false;             // padding row
        float x[EPL];
#pragma unroll
        for (int k = 0; k < NQ; ++k) {
            Elem<T>::widen2(u[k].x, x + 8 * k);
            Elem<T>::widen2(u[k].y, x + 8 * k + 2);
            Elem<T>::widen2(u[k].z, x + 8 * k + 4);
            Elem<T>::widen2(u[k].w, x + 8 * k + 6);
        }
        uint32_t a = 0;
#pragma unroll
        for (int e = 0; e < EPL; ++e) a = max(a, __float_as_uint(x[e]) & 0x7fffffffu);
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) a = max(a, __shfl_xor_sync(0xffffffffu, a, o));   // within the row
        if (!valid) continue;
        int64_t blk;
        int off;
        if constexpr (NARROW) {
            blk = div32((uint32_t)slot, p.by_block);
            off = (int)((uint32_t)slot - (uint32_t)blk * (uint32_t)p.block_size);
        } else {
            blk = slot / p.block_size;
            off = (int)(slot % p.block_size);
        }
        // smallest X with amax <= 448 * 2^X: amax = 1.M * 2^(E-127) <= 1.75 * 2^(8+X)
        const int E = (int)(a >> 23);
        int X = E == 0 ? -127 : ((a & 0x7fffffu) <= 0x600000u ? E - 135 : E - 134);
        X = max(-127, min(127, X));
        const float f = __uint_as_float((uint32_t)(127 - X) << 23);   // 2^-X (127 - X >= 6)
        uint32_t codes[EPL / 4];
#pragma unroll
        for (int k = 0; k < EPL / 4; ++k)
            codes[k] = f32x2_to_e4m3x2(x[4 * k] * f, x[4 * k + 1] * f) |
                       (f32x2_to_e4m3x2(x[4 * k + 2] * f, x[4 * k + 3] * f) << 16);
        const size_t row = ((size_t)blk * p.num_kv_heads + h) * p.block_size + off;
        unsigned char *dst = (is_v ? p.v_layer : p.k_layer) + row * D + rl * EPL;
        if constexpr (EPL >= 16) {
#pragma unroll
            for (int k = 0; k < EPL / 16; ++k)
                reinterpret_cast<uint4 *>(dst)[k] =
                    make_uint4(codes[4 * k], codes[4 * k + 1], codes[4 * k + 2], codes[4 * k + 3]);
        } else {
            *reinterpret_cast<uint2 *>(dst) = make_uint2(codes[0], codes[1]);
        }
        if (rl == 0)
            p.s_layer[(((size_t)blk * p.num_kv_heads + h) * 2 + (is_v ? 1 : 0)) * p.block_size + off] =
                (unsigned char)(X + 127);
    }
}

// ------------------------------------------------------------------ decode attention
struct Params {
    CUtensorMap tmap_k;             // codes as [L*NB*Hkv*B rows][128] bytes, boxes of HEADS*B rows
    CUtensorMap tmap_v;
    const unsigned char *s_layer;   // this layer's scale bytes [NB][Hkv][K, V][B]
    const void *q;                  // [n][Hq][128] activation type
    void *out;
    const int32_t *tables;
    const int32_t *lens;
    float *ws_acc;
    float *ws_ml;
    const int32_t *order;           // longest-first range order, or null (launch order)
    int32_t *counters;              // [n_seqs][head_groups] split-merge counters
    int32_t max_blocks, num_blocks, num_kv_heads, num_q_heads, layer;
    int32_t split_blocks, max_splits, out_f32, group, head_groups;
    int32_t debug_withhold;         // see copies_withheld(); -1 outside wait-expiry tests
    float scale_log2;
};

// A CTA serves HEADS neighbouring KV heads (their rows of a block are contiguous, so
// one TMA box fetches all of them) and their HEADS * group <= 8 query heads, which
// fill the 8 columns of the m16n8 products.
template <int B, int HEADS>
struct Shape {
    static constexpr int kRows = HEADS * B;                          // rows of a K (or V) tile
    static constexpr int kTileBytes = kRows * kD;
    static constexpr int kStages = 32768 / kTileBytes;               // 64 KB of codes in flight
    static constexpr int kScaleBytes = 2 * kRows;                    // [heads][K, V][B] of a tile
    static constexpr int kRingBytes = kStages * 2 * kTileBytes;
    static constexpr int kScaleRing = kStages * kScaleBytes;
    static constexpr int kRedBytes = kConsumerWarps * 8 * (2 + kD) * 4;
    static_assert(kRedBytes <= kRingBytes, "reduction area reuses the ring");
    static_assert(kStages % kConsumerWarps == 0, "each stage must belong to one consumer warp");
    static_assert(kScaleBytes % 16 == 0, "bulk copies move multiples of 16 bytes");
    static constexpr size_t kSmemBytes = 1024 + kRingBytes + kScaleRing + 2 * kStages * sizeof(uint64_t);
};

template <typename T, int B, int HEADS>
__global__ void __launch_bounds__(kDecodeThreads, 3) decode_kernel(const __grid_constant__ Params p) {
    using SH = Shape<B, HEADS>;
    using M = Mma<__half>;
    constexpr int STAGES = SH::kStages, TILE = SH::kTileBytes, SCB = SH::kScaleBytes;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);

    // one CTA per (range, head group); ranges longest first when an order is given
    const int hg = (int)(blockIdx.x % (unsigned)p.head_groups);
    const int rank = (int)(blockIdx.x / (unsigned)p.head_groups);
    const int item = p.order ? p.order[rank] : rank;
    const int s = item / p.max_splits;
    const int split = item % p.max_splits;
    const int g0 = hg * HEADS;              // first KV head of this CTA
    const int group = p.group;
    const int hpc = HEADS * group;          // query heads of this CTA (<= 8)
    const int h0 = g0 * group;

    int L = p.lens[s];
    if (L < 1 || (L + B - 1) / B > p.max_blocks) {
        if (threadIdx.x == 0 && hg == 0 && split == 0) raise_error(kErrBadLen);
        if (L < 1) {
            if (split == 0)
                for (int t = threadIdx.x; t < hpc * kD; t += blockDim.x) {
                    const size_t idx = ((size_t)s * p.num_q_heads + h0 + t / kD) * kD + t % kD;
                    if (p.out_f32)
                        static_cast<float *>(p.out)[idx] = 0.f;
                    else
                        static_cast<T *>(p.out)[idx] = Elem<T>::narrow(0.f);
                }
            return;
        }
        L = p.max_blocks * B;
    }
    const int nblk = (L + B - 1) / B;
    const SplitRange rg = split_range(nblk, p.split_blocks, split);
    if (split >= rg.n) return;
    const int b0 = rg.b0;
    const int ntiles = rg.b1 - rg.b0;
    const int nsplit = rg.n;

    unsigned char *scl = smem + SH::kRingBytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(scl + SH::kScaleRing);
    uint64_t *empty = full + STAGES;
    float *red_m = reinterpret_cast<float *>(smem);   // [warps][8], after the loop
    float *red_l = red_m + kConsumerWarps * 8;
    float *red_o = red_l + kConsumerWarps * 8;        // [warps][8][128]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_fence_init();
    }
    __syncthreads();

    const int gq = lane >> 2;
    const int tq = lane & 3;
    // KV head (within the CTA) of this lane's accumulator columns 2tq, 2tq+1 (one head:
    // a CTA serves several heads only for groups of 2 or 4) and of its P^T column gq
    // (columns past the CTA's query heads are zero queries; clamp their head index)
    const int hd = HEADS == 1 ? 0 : min(HEADS - 1, (2 * tq) / group);
    const int hb = HEADS == 1 ? 0 : gq / group;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // scores of columns 2tq, 2tq+1
    float mo0 = -INFINITY, mo1 = -INFINITY;                    // scores + value exponents
    float o[8][4];

    if (warp == kConsumerWarps) {
        // ---------------- producer
        const int32_t *trow = p.tables + (size_t)s * p.max_blocks + b0;
        bool ok = true;
        int issued = 0;
        const int to_issue = copies_withheld(p.debug_withhold) ? 0 : ntiles;
        for (int base = 0; base < to_issue && ok; base += 32) {
            int blk = 0;
            if (base + lane < ntiles) {
                blk = trow[base + lane];
                if ((unsigned)blk >= (unsigned)p.num_blocks) {
                    raise_error(kErrBadBlock);
                    blk = 0;
                }
            }
            const int cnt = min(32, ntiles - base);
            for (int j = 0; j < cnt; ++j) {
                const int b = __shfl_sync(0xffffffffu, blk, j);
                const int i = base + j;
                const int st = i % STAGES;
                if (lane == 0) {
                    if (i >= STAGES) ok = mbar_wait_thread(&empty[st], ((i / STAGES) - 1) & 1);
                    if (ok) {
                        const size_t hb0 = (size_t)b * p.num_kv_heads + g0;   // (block, first head) in the layer
                        const int row = (int)(((size_t)p.layer * p.num_blocks * p.num_kv_heads + hb0) * B);
                        unsigned char *dst = smem + st * 2 * TILE;
                        mbar_arrive_expect_tx(&full[st], 2 * TILE + SCB);
                        tma_load_2d(dst, &p.tmap_k, 0, row, &full[st]);
                        tma_load_2d(dst + TILE, &p.tmap_v, 0, row, &full[st]);
                        bulk_g2s(scl + st * SCB, p.s_layer + hb0 * 2 * B, SCB, &full[st]);
                        issued = i + 1;
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
        }
        if (lane == 0) drain_copies(full, issued, STAGES);
        __syncwarp();
    } else {
        // ---------------- consumers
        // Q^T fragments: column gq is query head h0 + gq; lane (gq, tq) holds dims
        // 16c + 4tq .. 16c + 4tq + 3 of k-step c (the order the K codes arrive in).
        uint32_t qb[8][2];
        int qexp;
        {
            const bool qv = gq < hpc;
            const unsigned char *qrow = static_cast<const unsigned char *>(p.q) +
                                        ((size_t)s * p.num_q_heads + h0 + (qv ? gq : 0)) * kD * sizeof(T);
            float x[8][4];
            uint32_t amax = 0;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint2 u = *reinterpret_cast<const uint2 *>(qrow + (16 * c + 4 * tq) * sizeof(T));
                Elem<T>::widen2(u.x, x[c]);
                Elem<T>::widen2(u.y, x[c] + 2);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (!qv) x[c][e] = 0.f;
                    amax = max(amax, __float_as_uint(x[c][e]) & 0x7fffffffu);
                }
            }
            amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            // prescale 2^P with the largest |q| in [2^14, 2^15): P = 141 - E (biased E)
            const int E = (int)(amax >> 23);
            qexp = E == 0 ? 127 : max(-126, min(127, 141 - E));
            const float f = __uint_as_float((uint32_t)(qexp + 127) << 23);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                qb[c][0] = M::pack(x[c][0] * f, x[c][1] * f);
                qb[c][1] = M::pack(x[c][2] * f, x[c][3] * f);
            }
        }
        // score exponent offsets of this lane's two columns: 8 - P (the 2^-8 of the
        // widened codes and the query prescale)
        const int pq0 = 8 - __shfl_sync(0xffffffffu, qexp, 8 * tq);
        const int pq1 = 8 - __shfl_sync(0xffffffffu, qexp, 8 * tq + 4);
#pragma unroll
        for (int dm = 0; dm < 8; ++dm) o[dm][0] = o[dm][1] = o[dm][2] = o[dm][3] = 0.f;
        const float sl = p.scale_log2;

        for (int i = warp; i < ntiles; i += kConsumerWarps) {
            const int st = i % STAGES;
            if (!mbar_wait_warp(&full[st], (i / STAGES) & 1)) break;
            const uint32_t kbase = smem_addr(smem + st * 2 * TILE);
            const uint32_t vbase = kbase + TILE;
            const unsigned char *ksc = scl + st * SCB + hd * 2 * B;   // this lane's head: K bytes
            const unsigned char *vsc = ksc + B;                        // V bytes
            const int tok0 = (b0 + i) * B;
            const int valid = min(B, L - tok0);
#pragma unroll
            for (int j = 0; j < B / 16; ++j) {
                if (j * 16 >= valid) break;
                const int ra = j * 16 + gq, rb = ra + 8;          // this lane's two token rows
                const int eka = ksc[ra], ekb = ksc[rb], eva = vsc[ra], evb = vsc[rb];
                float c[4];
#pragma unroll
                for (int hh = 0; hh < HEADS; ++hh) {
                    float t[4] = {0.f, 0.f, 0.f, 0.f};
                    const int r = hh * B + j * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
                    for (int cc = 0; cc < 8; cc += 2) {
                        const int chunk = cc + (lane >> 4);
                        uint32_t k4[4], a[4];
                        ldsm_x4(k4, kbase + r * 128 + ((chunk ^ (r & 7)) << 4));
                        // k4[x] holds dims 4tq..4tq+3 of a 16-dim chunk: codes 0,1 -> a0/a1,
                        // codes 2,3 -> a2/a3 (the query fragments use the same order)
                        a[0] = codes_to_f16x2(k4[0], k4[0], 0x9180u);
                        a[2] = codes_to_f16x2(k4[0], k4[0], 0xB3A2u);
                        a[1] = codes_to_f16x2(k4[1], k4[1], 0x9180u);
                        a[3] = codes_to_f16x2(k4[1], k4[1], 0xB3A2u);
                        M::mma(t, a, qb[cc][0], qb[cc][1]);
                        a[0] = codes_to_f16x2(k4[2], k4[2], 0x9180u);
                        a[2] = codes_to_f16x2(k4[2], k4[2], 0xB3A2u);
                        a[1] = codes_to_f16x2(k4[3], k4[3], 0x9180u);
                        a[3] = codes_to_f16x2(k4[3], k4[3], 0xB3A2u);
                        M::mma(t, a, qb[cc + 1][0], qb[cc + 1][1]);
                    }
                    // keep the product with this lane's own KV head
#pragma unroll
                    for (int e = 0; e < 4; ++e) c[e] = (hh == 0 || hd == hh) ? t[e] : c[e];
                }
                const bool v0 = ra < valid, v1 = rb < valid;
                // 2^(X_k + 8 - P): key scale, the codes' 2^-8 and the query prescale
                const float s0 = v0 ? c[0] * (sl * pow2_field(eka + pq0)) : -INFINITY;
                const float s1 = v0 ? c[1] * (sl * pow2_field(eka + pq1)) : -INFINITY;
                const float s2 = v1 ? c[2] * (sl * pow2_field(ekb + pq0)) : -INFINITY;
                const float s3 = v1 ? c[3] * (sl * pow2_field(ekb + pq1)) : -INFINITY;
                const bool need = fmaxf(s0, s2) > m0 + kRescaleThreshold || fmaxf(s1, s3) > m1 + kRescaleThreshold;
                if (__any_sync(0xffffffffu, need)) {
                    float t0 = fmaxf(s0, s2), t1 = fmaxf(s1, s3);
#pragma unroll
                    for (int off = 4; off < 32; off <<= 1) {
                        t0 = fmaxf(t0, __shfl_xor_sync(0xffffffffu, t0, off));
                        t1 = fmaxf(t1, __shfl_xor_sync(0xffffffffu, t1, off));
                    }
                    const float n0 = fmaxf(m0, t0), n1 = fmaxf(m1, t1);
                    l0 *= ex2(m0 - n0);
                    l1 *= ex2(m1 - n1);
                    m0 = n0;
                    m1 = n1;
                }
                // the same for the output's reference over s + X_v; byte - 127 as a float
                // without a conversion instruction: (2^23 + byte) - (2^23 + 127)
                const float xa = __uint_as_float(0x4B000000u | (uint32_t)eva) - 8388735.0f;
                const float xb = __uint_as_float(0x4B000000u | (uint32_t)evb) - 8388735.0f;
                const float u0 = s0 + xa, u1 = s1 + xa, u2 = s2 + xb, u3 = s3 + xb;
                const bool need_o =
                    fmaxf(u0, u2) > mo0 + kRescaleThreshold || fmaxf(u1, u3) > mo1 + kRescaleThreshold;
                if (__any_sync(0xffffffffu, need_o)) {
                    float t0 = fmaxf(u0, u2), t1 = fmaxf(u1, u3);
#pragma unroll
                    for (int off = 4; off < 32; off <<= 1) {
                        t0 = fmaxf(t0, __shfl_xor_sync(0xffffffffu, t0, off));
                        t1 = fmaxf(t1, __shfl_xor_sync(0xffffffffu, t1, off));
                    }
                    const float n0 = fmaxf(mo0, t0), n1 = fmaxf(mo1, t1);
                    const float f0 = ex2(mo0 - n0), f1 = ex2(mo1 - n1);
#pragma unroll
                    for (int dm = 0; dm < 8; ++dm) {
                        o[dm][0] *= f0;
                        o[dm][2] *= f0;
                        o[dm][1] *= f1;
                        o[dm][3] *= f1;
                    }
                    mo0 = n0;
                    mo1 = n1;
                }
                l0 += ex2(s0 - m0) + ex2(s2 - m0);
                l1 += ex2(s1 - m1) + ex2(s3 - m1);
                // weights for P.V, <= 2^8; past-the-end rows have u = -inf and weight 0
                const float w0 = ex2(u0 - mo0), w1 = ex2(u1 - mo1), w2 = ex2(u2 - mo0), w3 = ex2(u3 - mo1);
                const uint32_t h01 = M::pack(w0, w1), h23 = M::pack(w2, w3);
                const uint32_t r01 = M::pack(w0 - M::low(h01), w1 - M::high(h01));
                const uint32_t r23 = M::pack(w2 - M::low(h23), w3 - M::high(h23));
                const uint32_t bh0 = transpose8x8(h01), bh1 = transpose8x8(h23);
                const uint32_t bl0 = transpose8x8(r01), bl1 = transpose8x8(r23);
                // Past-the-end slots carry weight 0 but arbitrary codes (0x7F is NaN, and
                // 0 * NaN is NaN): zero them.  a0/a1 hold tokens 2tq, 2tq+1 and a2/a3
                // tokens 2tq+8, 2tq+9 of the group.
                const int left = valid - j * 16;
                uint32_t keep01 = 0xffffffffu, keep89 = 0xffffffffu;
                if (left < 16) {
                    const int t0 = 2 * tq;
                    keep01 = (t0 < left ? 0x0000ffffu : 0u) | (t0 + 1 < left ? 0xffff0000u : 0u);
                    keep89 = (t0 + 8 < left ? 0x0000ffffu : 0u) | (t0 + 9 < left ? 0xffff0000u : 0u);
                }
                const int mi = lane >> 3;
#pragma unroll
                for (int hh = 0; hh < HEADS; ++hh) {
                    // P^T columns of the other heads' queries are zero for this head's values
                    const bool mine = HEADS == 1 || hb == hh;
                    const uint32_t ph0 = mine ? bh0 : 0u, ph1 = mine ? bh1 : 0u;
                    const uint32_t pl0 = mine ? bl0 : 0u, pl1 = mine ? bl1 : 0u;
                    const int r = hh * B + j * 16 + (lane & 7) + (mi & 1) * 8;
#pragma unroll
                    for (int cc = 0; cc < 8; cc += 2) {
                        const int chunk = cc + (mi >> 1);
                        uint32_t v4[4];
                        ldsm_x4_trans(v4, vbase + r * 128 + ((chunk ^ (r & 7)) << 4));
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) {
                            // v4[2h2] holds tokens 2tq, 2tq+1 and v4[2h2+1] tokens 2tq+8, 2tq+9,
                            // each as codes (dim 2gq, dim 2gq+1): byte k = token k/2, dim k%2.
                            // Rows gq / gq+8 of the A fragment are dims 16(cc+h2) + 2gq / + 1.
                            const uint32_t x = v4[2 * h2], y = v4[2 * h2 + 1];
                            uint32_t a[4];
                            a[0] = codes_to_f16x2(x, y, 0xA280u) & keep01;   // even dim, tokens 2tq, 2tq+1
                            a[2] = codes_to_f16x2(x, y, 0xE6C4u) & keep89;   // even dim, tokens 2tq+8, 2tq+9
                            a[1] = codes_to_f16x2(x, y, 0xB391u) & keep01;   // odd dim
                            a[3] = codes_to_f16x2(x, y, 0xF7D5u) & keep89;
                            M::mma(o[cc + h2], a, ph0, ph1);
                            M::mma(o[cc + h2], a, pl0, pl1);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, off);
            l1 += __shfl_xor_sync(0xffffffffu, l1, off);
        }
    }
    __syncthreads();   // every stage consumed and every copy landed: the ring is free
    if (warp < kConsumerWarps) {
        if (gq == 0) {
            red_m[warp * 8 + 2 * tq] = m0;
            red_m[warp * 8 + 2 * tq + 1] = m1;
            red_l[warp * 8 + 2 * tq] = l0;
            red_l[warp * 8 + 2 * tq + 1] = l1;
        }
        // bring the output to the denominator's reference, x 2^(m_o - m), and undo the
        // 2^-8 of the widened value codes
        const float f0 = m0 == -INFINITY ? 0.f : ex2(mo0 - m0) * 256.f;
        const float f1 = m1 == -INFINITY ? 0.f : ex2(mo1 - m1) * 256.f;
#pragma unroll
        for (int dm = 0; dm < 8; ++dm) {
            // accumulator rows gq / gq + 8 are dims 16dm + 2gq / 16dm + 2gq + 1
            float *c0 = red_o + (warp * 8 + 2 * tq) * kD + dm * 16 + 2 * gq;
            float *c1 = c0 + kD;
            c0[0] = o[dm][0] * f0;
            c1[0] = o[dm][1] * f1;
            c0[1] = o[dm][2] * f0;
            c1[1] = o[dm][3] * f1;
        }
    }
    __syncthreads();

    for (int t = threadIdx.x; t < hpc * kD; t += blockDim.x) {
        const int h = t / kD;
        const int d = t % kD;
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) mx = fmaxf(mx, red_m[w * 8 + h]);
        float lsum = 0.f, osum = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const float mw = red_m[w * 8 + h];
            const float f = (mw == -INFINITY) ? 0.f : ex2(mw - mx);
            lsum += red_l[w * 8 + h] * f;
            osum += red_o[(w * 8 + h) * kD + d] * f;
        }
        const int hq = h0 + h;
        if (nsplit == 1) {
            const size_t idx = ((size_t)s * p.num_q_heads + hq) * kD + d;
            if (p.out_f32)
                static_cast<float *>(p.out)[idx] = osum / lsum;
            else
                static_cast<T *>(p.out)[idx] = Elem<T>::narrow(osum / lsum);
        } else {
            const size_t part = ((size_t)s * p.max_splits + split) * p.num_q_heads + hq;
            p.ws_acc[part * kD + d] = osum;
            if (d == 0) {
                p.ws_ml[part * 2] = mx;
                p.ws_ml[part * 2 + 1] = lsum;
            }
        }
    }
    if (nsplit > 1) {
        // (the range is looked up again rather than kept in registers across the loop)
        const int hg2 = (int)(blockIdx.x % (unsigned)p.head_groups);
        const int rank2 = (int)(blockIdx.x / (unsigned)p.head_groups);
        const int s2 = (p.order ? p.order[rank2] : rank2) / p.max_splits;
        merge_splits_if_last<T>(p.ws_acc, p.ws_ml, p.counters + (size_t)s2 * p.head_groups + hg2, p.out, p.out_f32,
                                s2, p.num_q_heads, p.max_splits, nsplit, hg2 * HEADS * p.group, HEADS * p.group, kD,
                                reinterpret_cast<float *>(smem), SH::kRingBytes / 4);
    }
}

// KV heads per CTA for a GQA group: 8 / group for groups of 2 and 4 (so the query
// heads fill the 8 product columns and each lane's two columns stay in one head),
// at most 64 rows per tile, and dividing the KV heads; else 1.
inline int heads_per_cta(int group, int num_kv_heads, int block_size) {
    if (group != 2 && group != 4) return 1;
    int h = 8 / group;
    while (h > 1 && (h * block_size > 64 || num_kv_heads % h != 0)) h /= 2;
    return h;
}

}  // namespace fp8
