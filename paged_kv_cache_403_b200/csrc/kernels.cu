// sm_100a kernels of the paged decode path and their C ABI entry points.
//
//  paged_decode_simt_kernel  -- single-query decode attention through the block
//                          table ("What problem does PagedAttention solve, and
//                          what is continuous batching?", "How PagedAttention
//                          works": the kernel follows the table when it reads
//                          keys and values).  One CTA per (sequence, group of up
//                          to 4 query heads sharing one KV head, split).
//  split_reduce_kernel  -- log-sum-exp merge of the splits of long sequences.
//  append_kv_kernel     -- reshape-and-cache: new K/V rows into their slots
//                          (same page, "Why the KV cache becomes the problem":
//                          decode appends a small amount of new data).
//  copy_blocks_kernel   -- copy-on-write block copies (same page, "How
//                          PagedAttention works").
//  paged_decode_mma_kernel (below), prefill.cuh and fp8.cuh hold the tensor-core
//  decode, the tcgen05 chunked prefill and the FP8-cache append and decode.
//
// Design (B200): each (block, KV head) tile of keys or values is one contiguous
// block_size x head_dim run in HBM, fetched whole by a 1-D TMA bulk copy
// (cp.async.bulk, no tensor map, no multicast) into a ring of shared-memory
// stages guarded by mbarriers.  A producer warp walks the block table and keeps
// the ring full; four consumer warps each own whole tiles.  Inside a warp eight
// lanes share one token (16-byte vector reads of the row), so a pass covers four
// tokens; dot products reduce over the eight lanes with xor shuffles.  Every
// query head of the GQA group reuses the same key/value registers, so K and V
// are read from HBM once per KV head.  The softmax is online in base 2 (q is
// pre-scaled by scale*log2(e)); the running maximum is only moved when a score
// exceeds it by more than 2^8, which keeps rescaling off the common path and is
// exact because the final division uses the same reference maximum.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <string>
#include <type_traits>

#include "pool.hpp"

using pa_internal::fail;

namespace {

// ------------------------------------------------------------------ device error word
constexpr unsigned kErrBadBlock = 1u, kErrBadLen = 2u, kErrTimeout = 4u, kErrBadSlot = 8u;
__device__ unsigned int g_device_error = 0;

__device__ __forceinline__ void raise_error(unsigned e) { atomicOr(&g_device_error, e); }

// Division of 32-bit indices by a divisor fixed for the launch: a shift when it is a power
// of two, else the hardware's 32-bit division.  The append kernels' index arithmetic in 64
// bits (emulated division) cost more than their memory traffic; the host launches the
// 32-bit form only when every index of the launch fits.
struct Div32 {
    uint32_t d;
    int32_t shift;   // >= 0: d == 1 << shift
};
inline Div32 make_div32(uint32_t d) {
    return {d, (d && !(d & (d - 1))) ? __builtin_ctz(d) : -1};
}
__device__ __forceinline__ uint32_t div32(uint32_t n, Div32 d) { return d.shift >= 0 ? n >> d.shift : n / d.d; }

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Waits are bounded: after g_wait_limit_ns (kWaitLimitNs unless a test lowers it
// through pa_debug_wait_test) the waiter records kErrTimeout and gives up.  The bound
// is read only once a wait has to spin, so the common path never loads it.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
__device__ uint64_t g_wait_limit_ns = kWaitLimitNs;

__device__ __forceinline__ uint64_t wait_limit_ns() { return *static_cast<volatile uint64_t *>(&g_wait_limit_ns); }

// A wait-expiry test (pa_debug_wait_test) names one decode or prefill CTA, by its
// linear block index, whose producer issues no copies, so that the waits of its other
// warps run out.
__device__ __forceinline__ bool copies_withheld(int32_t withhold) {
    return withhold >= 0 &&
           (int64_t)blockIdx.x + (int64_t)gridDim.x * (blockIdx.y + (int64_t)gridDim.y * blockIdx.z) == withhold;
}

// One thread waits (the producer lane).
__device__ __forceinline__ bool mbar_wait_thread(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns(), limit = wait_limit_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit) {
            raise_error(kErrTimeout);
            return false;
        }
    }
    return true;
}

// Before its ring is reused or the CTA exits, the issuing lane waits (bounded) until
// the last copy it put into each stage has landed: fill i went to stage i % stages as
// that stage's phase i / stages, and only the last `stages` fills can still be in
// flight.  In a normal run they landed long before; after a consumer gave up on a
// wait this keeps a late copy from writing into shared memory that is reused.
__device__ __forceinline__ void drain_copies(uint64_t *full, int issued, int stages) {
    for (int i = issued > stages ? issued - stages : 0; i < issued; ++i)
        if (!mbar_wait_thread(&full[i % stages], (uint32_t)(i / stages) & 1u)) return;
}

// A whole warp waits and leaves together, so later full-warp shuffles stay converged.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t *bar, uint32_t parity) {
    uint64_t t0 = 0, limit = kWaitLimitNs;
    for (uint32_t it = 0;; ++it) {
        const bool done = mbar_try_wait(bar, parity);
        if (__all_sync(0xffffffffu, done)) return true;
        if (it == 0) {
            t0 = global_timer_ns();
            limit = wait_limit_ns();
        }
        const bool late = global_timer_ns() - t0 > limit;
        if (__any_sync(0xffffffffu, late)) {
            if ((threadIdx.x & 31) == 0) raise_error(kErrTimeout);
            return false;
        }
    }
}

// 1-D TMA bulk copy global -> shared, completing `bytes` transactions on `bar`.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ------------------------------------------------------------------ element types
template <typename T>
struct Elem;

template <>
struct Elem<float> {
    static constexpr int kVec = 4;   // elements per 16 bytes
    __device__ __forceinline__ static void widen(const uint4 &u, float *f) {
        f[0] = __uint_as_float(u.x);
        f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z);
        f[3] = __uint_as_float(u.w);
    }
    __device__ __forceinline__ static float narrow(float x) { return x; }
};

template <>
struct Elem<__half> {
    static constexpr int kVec = 8;
    __device__ __forceinline__ static void widen2(uint32_t w, float *f) {
        __half2 h;
        memcpy(&h, &w, 4);
        const float2 x = __half22float2(h);
        f[0] = x.x;
        f[1] = x.y;
    }
    __device__ __forceinline__ static void widen(const uint4 &u, float *f) {
        widen2(u.x, f);
        widen2(u.y, f + 2);
        widen2(u.z, f + 4);
        widen2(u.w, f + 6);
    }
    __device__ __forceinline__ static __half narrow(float x) { return __float2half_rn(x); }
};

template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kVec = 8;
    // bf16 is the top half of an fp32: the low element of a word is (w << 16),
    // the high one (w & 0xffff0000).
    __device__ __forceinline__ static void widen2(uint32_t w, float *f) {
        f[0] = __uint_as_float(w << 16);
        f[1] = __uint_as_float(w & 0xffff0000u);
    }
    __device__ __forceinline__ static void widen(const uint4 &u, float *f) {
        widen2(u.x, f);
        widen2(u.y, f + 2);
        widen2(u.z, f + 4);
        widen2(u.w, f + 6);
    }
    __device__ __forceinline__ static __nv_bfloat16 narrow(float x) { return __float2bfloat16_rn(x); }
};

// ------------------------------------------------------------------ decode attention
constexpr int kLanesPerToken = 8;                        // lanes sharing one token row
constexpr int kTokensPerPass = 32 / kLanesPerToken;      // tokens a warp covers per pass
constexpr int kConsumerWarps = 4;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;  // + one producer warp
constexpr float kRescaleThreshold = 8.0f;                // log2 units: 2^8 headroom

// Split ranges.  A sequence of nblk blocks, more than split_blocks of them, is cut
// into n = ceil(nblk / split_blocks) ranges of nearly equal length: with
// nblk = q * n + r, the first r ranges hold q + 1 blocks and the others q, so a range
// holds at most split_blocks blocks and, when there are several, at least
// split_blocks / 2 (rounded down).
// Range lengths then spread with the sequence lengths instead of piling up at
// split_blocks, where CTAs of equal length would end (and their successors ramp up)
// at the same moment all over the GPU.
struct SplitRange {
    int b0, b1, n;   // blocks [b0, b1) of range z; n ranges; b0 >= nblk when z >= n
};

__device__ __forceinline__ SplitRange split_range(int nblk, int split_blocks, int z) {
    SplitRange r;
    r.n = nblk > 0 ? (nblk + split_blocks - 1) / split_blocks : 0;
    if (z >= r.n) {
        r.b0 = r.b1 = nblk;
        return r;
    }
    const int q = nblk / r.n, rem = nblk % r.n;
    r.b0 = z * q + min(z, rem);
    r.b1 = r.b0 + q + (z < rem ? 1 : 0);
    return r;
}

struct DecodeParams {
    const unsigned char *k_layer;   // this layer's key pool [NB][Hkv][B][D]
    const unsigned char *v_layer;
    const void *q;                  // [n][Hq][D]
    void *out;                      // [n][Hq][D]
    const int32_t *tables;          // [n][max_blocks]
    const int32_t *lens;            // [n]
    float *ws_acc;                  // [n][max_splits][Hq][D]
    float *ws_ml;                   // [n][max_splits][Hq][2]
    int32_t n_seqs, max_blocks, num_blocks, num_kv_heads, num_q_heads;
    int32_t split_blocks, max_splits, out_f32;
    int32_t debug_withhold;         // see copies_withheld(); -1 outside wait-expiry tests
    float scale_log2;
};

template <typename T, int B, int D>
struct DecodeShape {
    static constexpr int kVec = Elem<T>::kVec;
    static constexpr int kElems = D / kLanesPerToken;      // elements of a row per lane
    static constexpr int kChunks = kElems / kVec;          // 16-byte chunks per lane
    static constexpr int kRowBytes = D * (int)sizeof(T);
    static constexpr int kTileBytes = B * kRowBytes;
    static constexpr int kStages = (2 * kTileBytes <= 8192) ? 8 : 4;
    static_assert(kChunks >= 1 && kElems % kVec == 0, "row must split into 16-byte chunks");
    static_assert(kStages % kConsumerWarps == 0, "each stage must belong to one consumer warp");
    static constexpr int kRingBytes = kStages * 2 * kTileBytes;
};

template <int HPC, int D>
constexpr int reduce_bytes() {
    return kConsumerWarps * HPC * (2 + D) * 4;
}

template <typename T, int B, int D, int HPC>
constexpr size_t decode_smem_bytes() {
    using S = DecodeShape<T, B, D>;
    return (size_t)S::kRingBytes + 2 * S::kStages * sizeof(uint64_t) + reduce_bytes<HPC, D>();
}

template <typename T>
__device__ __forceinline__ void store_out(const DecodeParams &p, size_t idx, float v) {
    if (p.out_f32)
        static_cast<float *>(p.out)[idx] = v;
    else
        static_cast<T *>(p.out)[idx] = Elem<T>::narrow(v);
}

template <typename T, int B, int D, int HPC>
__global__ void __launch_bounds__(kDecodeThreads) paged_decode_simt_kernel(const DecodeParams p) {
    using EL = Elem<T>;
    using SH = DecodeShape<T, B, D>;
    constexpr int VEC = SH::kVec, E = SH::kElems, NCH = SH::kChunks, ROW = SH::kRowBytes;
    constexpr int TILE = SH::kTileBytes, STAGES = SH::kStages;
    extern __shared__ __align__(128) unsigned char smem[];

    const int s = blockIdx.x;
    const int hg = blockIdx.y;
    const int split = blockIdx.z;

    int L = p.lens[s];
    if (L < 1 || (L + B - 1) / B > p.max_blocks) {
        if (threadIdx.x == 0 && hg == 0 && split == 0) raise_error(kErrBadLen);
        if (L < 1) {   // nothing to attend to: defined output 0
            if (split == 0)
                for (int t = threadIdx.x; t < HPC * D; t += blockDim.x)
                    store_out<T>(p, ((size_t)s * p.num_q_heads + hg * HPC + t / D) * D + t % D, 0.f);
            return;
        }
        L = p.max_blocks * B;
    }
    const int nblk = (L + B - 1) / B;
    const SplitRange rg = split_range(nblk, p.split_blocks, split);
    if (split >= rg.n) return;
    const int b0 = rg.b0;
    const int b1 = rg.b1;
    const int ntiles = b1 - b0;
    const int nsplit = rg.n;
    const int group = p.num_q_heads / p.num_kv_heads;
    const int h0 = hg * HPC;
    const int g = h0 / group;

    uint64_t *full = reinterpret_cast<uint64_t *>(smem + SH::kRingBytes);
    uint64_t *empty = full + STAGES;
    float *red_m = reinterpret_cast<float *>(empty + STAGES);   // [warps][HPC]
    float *red_l = red_m + kConsumerWarps * HPC;                 // [warps][HPC]
    float *red_o = red_l + kConsumerWarps * HPC;                 // [warps][HPC][D]

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

    if (warp == kConsumerWarps) {
        // ---------------- producer: walk the table, keep the ring full
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
                    blk = 0;   // stay in bounds; the error word reports the bad table
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
                        const size_t off = ((size_t)b * p.num_kv_heads + g) * TILE;
                        unsigned char *dst = smem + st * 2 * TILE;
                        mbar_arrive_expect_tx(&full[st], 2 * TILE);
                        bulk_g2s(dst, p.k_layer + off, TILE, &full[st]);
                        bulk_g2s(dst + TILE, p.v_layer + off, TILE, &full[st]);
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
        const int c = lane % kLanesPerToken;       // which 16-byte chunks of the row
        const int slot = lane / kLanesPerToken;    // which token of the pass
        float q[HPC][E];
#pragma unroll
        for (int h = 0; h < HPC; ++h) {
            const T *qrow = static_cast<const T *>(p.q) + ((size_t)s * p.num_q_heads + h0 + h) * D;
#pragma unroll
            for (int k = 0; k < NCH; ++k) {
                const uint4 u = *reinterpret_cast<const uint4 *>(qrow + (k * kLanesPerToken + c) * VEC);
                float f[VEC];
                EL::widen(u, f);
#pragma unroll
                for (int v = 0; v < VEC; ++v) q[h][k * VEC + v] = f[v] * p.scale_log2;
            }
        }
        float m[HPC], l[HPC], o[HPC][E];
#pragma unroll
        for (int h = 0; h < HPC; ++h) {
            m[h] = -INFINITY;
            l[h] = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) o[h][e] = 0.f;
        }

        for (int i = warp; i < ntiles; i += kConsumerWarps) {
            const int st = i % STAGES;
            if (!mbar_wait_warp(&full[st], (i / STAGES) & 1)) break;
            const unsigned char *kt = smem + st * 2 * TILE;
            const unsigned char *vt = kt + TILE;
            const int tok0 = (b0 + i) * B;
#pragma unroll 2
            for (int ps = 0; ps < B / kTokensPerPass; ++ps) {
                const int r = ps * kTokensPerPass + slot;
                const bool valid = tok0 + r < L;
                float kf[E];
#pragma unroll
                for (int k = 0; k < NCH; ++k) {
                    const uint4 u = *reinterpret_cast<const uint4 *>(kt + r * ROW + (k * kLanesPerToken + c) * 16);
                    EL::widen(u, &kf[k * VEC]);
                }
                float sc[HPC];
#pragma unroll
                for (int h = 0; h < HPC; ++h) {
                    float a0 = 0.f, a1 = 0.f;
#pragma unroll
                    for (int e = 0; e < E; e += 2) {
                        a0 = fmaf(q[h][e], kf[e], a0);
                        a1 = fmaf(q[h][e + 1], kf[e + 1], a1);
                    }
                    sc[h] = a0 + a1;
                }
#pragma unroll
                for (int off = 1; off < kLanesPerToken; off <<= 1)
#pragma unroll
                    for (int h = 0; h < HPC; ++h) sc[h] += __shfl_xor_sync(0xffffffffu, sc[h], off);
                float pr[HPC];
#pragma unroll
                for (int h = 0; h < HPC; ++h) {
                    const float sv = valid ? sc[h] : -INFINITY;
                    if (sv > m[h] + kRescaleThreshold) {
                        const float f = ex2(m[h] - sv);
                        l[h] *= f;
#pragma unroll
                        for (int e = 0; e < E; ++e) o[h][e] *= f;
                        m[h] = sv;
                    }
                    pr[h] = valid ? ex2(sv - m[h]) : 0.f;
                    l[h] += pr[h];
                }
                if (valid) {
                    float vf[E];
#pragma unroll
                    for (int k = 0; k < NCH; ++k) {
                        const uint4 u =
                            *reinterpret_cast<const uint4 *>(vt + r * ROW + (k * kLanesPerToken + c) * 16);
                        EL::widen(u, &vf[k * VEC]);
                    }
#pragma unroll
                    for (int h = 0; h < HPC; ++h)
#pragma unroll
                        for (int e = 0; e < E; ++e) o[h][e] = fmaf(pr[h], vf[e], o[h][e]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }

        // merge the four token slots of the warp (lanes differing in bits 3 and 4)
#pragma unroll
        for (int off = kLanesPerToken; off < 32; off <<= 1) {
#pragma unroll
            for (int h = 0; h < HPC; ++h) {
                const float mo = __shfl_xor_sync(0xffffffffu, m[h], off);
                const float lo = __shfl_xor_sync(0xffffffffu, l[h], off);
                const float mn = fmaxf(m[h], mo);
                const float fa = (m[h] == -INFINITY) ? 0.f : ex2(m[h] - mn);
                const float fb = (mo == -INFINITY) ? 0.f : ex2(mo - mn);
                l[h] = l[h] * fa + lo * fb;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float oo = __shfl_xor_sync(0xffffffffu, o[h][e], off);
                    o[h][e] = o[h][e] * fa + oo * fb;
                }
                m[h] = mn;
            }
        }
        if (lane < kLanesPerToken) {
#pragma unroll
            for (int h = 0; h < HPC; ++h) {
                if (lane == 0) {
                    red_m[warp * HPC + h] = m[h];
                    red_l[warp * HPC + h] = l[h];
                }
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int d = ((e / VEC) * kLanesPerToken + c) * VEC + e % VEC;
                    red_o[(warp * HPC + h) * D + d] = o[h][e];
                }
            }
        }
    }
    __syncthreads();

    // merge the consumer warps and write the result or this split's partial
    for (int t = threadIdx.x; t < HPC * D; t += blockDim.x) {
        const int h = t / D;
        const int d = t % D;
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) mx = fmaxf(mx, red_m[w * HPC + h]);
        float lsum = 0.f, osum = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const float mw = red_m[w * HPC + h];
            const float f = (mw == -INFINITY) ? 0.f : ex2(mw - mx);
            lsum += red_l[w * HPC + h] * f;
            osum += red_o[(w * HPC + h) * D + d] * f;
        }
        const int hq = h0 + h;
        if (nsplit == 1) {
            store_out<T>(p, ((size_t)s * p.num_q_heads + hq) * D + d, osum / lsum);
        } else {
            const size_t part = ((size_t)s * p.max_splits + split) * p.num_q_heads + hq;
            p.ws_acc[part * D + d] = osum;
            if (d == 0) {
                p.ws_ml[part * 2] = mx;
                p.ws_ml[part * 2 + 1] = lsum;
            }
        }
    }
}

// ------------------------------------------------------------------ split reduce
struct ReduceParams {
    const int32_t *lens;
    void *out;
    const float *ws_acc;
    const float *ws_ml;
    int32_t max_blocks, num_q_heads, split_blocks, max_splits, out_f32;
};

template <typename T, int B, int D>
__global__ void __launch_bounds__(D) split_reduce_kernel(const ReduceParams p) {
    const int s = blockIdx.x;
    const int hq = blockIdx.y;
    const int d = threadIdx.x;
    int L = p.lens[s];
    if (L < 1) return;
    if ((L + B - 1) / B > p.max_blocks) L = p.max_blocks * B;
    const int nblk = (L + B - 1) / B;
    const int nsplit = (nblk + p.split_blocks - 1) / p.split_blocks;
    if (nsplit <= 1) return;
    const size_t base = (size_t)s * p.max_splits * p.num_q_heads + hq;
    float mx = -INFINITY;
    for (int x = 0; x < nsplit; ++x) mx = fmaxf(mx, p.ws_ml[(base + (size_t)x * p.num_q_heads) * 2]);
    float lsum = 0.f, osum = 0.f;
    for (int x = 0; x < nsplit; ++x) {
        const size_t part = base + (size_t)x * p.num_q_heads;
        const float f = ex2(p.ws_ml[part * 2] - mx);
        lsum += p.ws_ml[part * 2 + 1] * f;
        osum += p.ws_acc[part * D + d] * f;
    }
    const float v = osum / lsum;
    const size_t idx = ((size_t)s * p.num_q_heads + hq) * D + d;
    if (p.out_f32)
        static_cast<float *>(p.out)[idx] = v;
    else
        static_cast<T *>(p.out)[idx] = Elem<T>::narrow(v);
}

// ------------------------------------------------------------------ longest ranges first
// The decode grid has one CTA per (sequence, split range, head group), and ranges range
// from a few tokens to a whole split.  The block scheduler starts CTAs in index order,
// so a long range that starts late keeps a few SMs busy after the rest are idle.  One
// CTA of this kernel sorts the (sequence, split) ranges by tile count, longest first
// (a counting sort over the counts), and the decode kernels take their range from
// that order: the greedy longest-first schedule.  Ranges of equal length may come in
// any order; each range's result is the same wherever it runs.
constexpr int kPlanThreads = 1024;
constexpr int kPlanBuckets = 4096;   // counts >= 4095 tiles share the first bucket

struct PlanParams {
    const int32_t *lens;
    int32_t *order;                  // [n_seqs * max_splits] range ids s * max_splits + z
    int32_t *counters;               // [n_counters] split-merge counters to zero
    int32_t n_seqs, max_blocks, block_size, split_blocks, max_splits, n_counters;
};

__device__ __forceinline__ int plan_bucket(const PlanParams &p, int item) {
    const int s = item / p.max_splits, z = item % p.max_splits;
    const int L = p.lens[s];
    const int nblk = L < 1 ? 0 : min((L + p.block_size - 1) / p.block_size, p.max_blocks);
    const SplitRange r = split_range(nblk, p.split_blocks, z);
    const int t = r.b1 - r.b0;
    return kPlanBuckets - 1 - min(t, kPlanBuckets - 1);   // longest ranges in the lowest bucket
}

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const PlanParams p) {
    __shared__ int start[kPlanBuckets];
    __shared__ int warp_sum[kPlanThreads / 32];
    constexpr int PER = kPlanBuckets / kPlanThreads;
    const int n_items = p.n_seqs * p.max_splits;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < p.n_counters; i += kPlanThreads) p.counters[i] = 0;
    for (int b = threadIdx.x; b < kPlanBuckets; b += kPlanThreads) start[b] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n_items; i += kPlanThreads) atomicAdd(&start[plan_bucket(p, i)], 1);
    __syncthreads();
    // exclusive prefix sum of the bucket counts: PER buckets per thread, then warps
    int cnt[PER], sum = 0;
#pragma unroll
    for (int k = 0; k < PER; ++k) {
        cnt[k] = start[threadIdx.x * PER + k];
        sum += cnt[k];
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = warp_sum[lane];
        int wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += v;
        }
        warp_sum[lane] = wi - w;
    }
    __syncthreads();
    int run = warp_sum[warp] + incl - sum;
#pragma unroll
    for (int k = 0; k < PER; ++k) {
        start[threadIdx.x * PER + k] = run;
        run += cnt[k];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n_items; i += kPlanThreads) p.order[atomicAdd(&start[plan_bucket(p, i)], 1)] = i;
}

// ------------------------------------------------------------------ in-kernel split merge
// The tensor-core decode kernels merge split partials themselves: every split CTA of a
// (sequence, head group) writes its partial, fences, and bumps that range's counter;
// the CTA that brings the counter to the number of splits merges all partials of its
// query heads (the same log-sum-exp merge as split_reduce_kernel) and writes the
// output, then resets the counter.  The counters are zeroed by plan_kernel, which
// runs before every split launch.  This saves the reduce launch and its re-read of
// cold partials (the last CTA finds most of them in L2).
template <typename T>
__device__ __forceinline__ void merge_splits_if_last(const float *ws_acc, const float *ws_ml, int32_t *counter,
                                                     void *out, int out_f32, int s, int num_q_heads,
                                                     int max_splits, int nsplit, int h0, int hpc, int D,
                                                     float *scratch, int scratch_floats) {
    __shared__ int is_last;
    __threadfence();          // this CTA's partial is visible before the count moves
    __syncthreads();
    if (threadIdx.x == 0) {
        const int prev = atomicAdd(counter, 1);
        is_last = prev == nsplit - 1;
        if (is_last) *counter = 0;
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    const size_t base = (size_t)s * max_splits * num_q_heads + h0;   // partial (s, split 0, head h0)
    const int nml = nsplit * hpc;
    if (nml * 3 + 16 <= scratch_floats && D % 4 == 0) {
        // The partials sit in L2; every load of a phase is independent of the others,
        // so each phase costs about one L2 round trip.  Phase 1: every (m, l) pair.
        float *sm = scratch;              // [nsplit][hpc] running maxima
        float *sl = sm + nml;             // [nsplit][hpc] sums
        float *sw = sl + nml;             // [nsplit][hpc] weights 2^(m - M) / l_total
        float *smax = sw + nml;           // [hpc] M
        float *sinv = smax + 8;           // [hpc] 1 / l_total
        for (int i = threadIdx.x; i < nml; i += blockDim.x) {
            const int x = i / hpc, h = i % hpc;
            const float2 ml = __ldcg(reinterpret_cast<const float2 *>(ws_ml) + base + (size_t)x * num_q_heads + h);
            sm[i] = ml.x;
            sl[i] = ml.y;
        }
        __syncthreads();
        if (threadIdx.x < hpc) {
            const int h = threadIdx.x;
            float mx = -INFINITY;
            for (int x = 0; x < nsplit; ++x) mx = fmaxf(mx, sm[x * hpc + h]);
            float lsum = 0.f;
            for (int x = 0; x < nsplit; ++x) lsum += sl[x * hpc + h] * ex2(sm[x * hpc + h] - mx);
            smax[h] = mx;
            sinv[h] = 1.f / lsum;
        }
        __syncthreads();
        for (int i = threadIdx.x; i < nml; i += blockDim.x) {
            const int h = i % hpc;
            sw[i] = ex2(sm[i] - smax[h]) * sinv[h];
        }
        __syncthreads();
        // Phase 2: four output columns per thread, all splits' partials loaded together.
        const int q4 = D / 4;
        for (int it = threadIdx.x; it < hpc * q4; it += blockDim.x) {
            const int h = it / q4, d4 = it % q4;
            const float4 *src = reinterpret_cast<const float4 *>(ws_acc + (base + h) * D) + d4;
            const size_t stride = (size_t)num_q_heads * D / 4;   // float4s from one split to the next
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
            for (int x = 0; x < nsplit; ++x) {
                const float4 a = __ldcg(src + (size_t)x * stride);
                const float w = sw[x * hpc + h];
                acc.x += w * a.x;
                acc.y += w * a.y;
                acc.z += w * a.z;
                acc.w += w * a.w;
            }
            const size_t idx = ((size_t)s * num_q_heads + h0 + h) * D + 4 * d4;
            if (out_f32) {
                float *o = static_cast<float *>(out) + idx;
                o[0] = acc.x;
                o[1] = acc.y;
                o[2] = acc.z;
                o[3] = acc.w;
            } else {
                T *o = static_cast<T *>(out) + idx;
                o[0] = Elem<T>::narrow(acc.x);
                o[1] = Elem<T>::narrow(acc.y);
                o[2] = Elem<T>::narrow(acc.z);
                o[3] = Elem<T>::narrow(acc.w);
            }
        }
        return;
    }
    // very many splits: one output element per thread, partials read split by split
    for (int t = threadIdx.x; t < hpc * D; t += blockDim.x) {
        const int h = t / D;
        const int d = t % D;
        const size_t hb = base + h;
        float mx = -INFINITY;
        for (int x = 0; x < nsplit; ++x) mx = fmaxf(mx, __ldcg(ws_ml + (hb + (size_t)x * num_q_heads) * 2));
        float lsum = 0.f, osum = 0.f;
        for (int x = 0; x < nsplit; ++x) {
            const size_t part = hb + (size_t)x * num_q_heads;
            const float f = ex2(__ldcg(ws_ml + part * 2) - mx);
            lsum += __ldcg(ws_ml + part * 2 + 1) * f;
            osum += __ldcg(ws_acc + part * D + d) * f;
        }
        const size_t idx = ((size_t)s * num_q_heads + h0 + h) * D + d;
        if (out_f32)
            static_cast<float *>(out)[idx] = osum / lsum;
        else
            static_cast<T *>(out)[idx] = Elem<T>::narrow(osum / lsum);
    }
}

// ------------------------------------------------------------------ tensor-core decode (fp16 / bf16)
// Per consumer warp and per 16-token group of a tile:
//   S^T[16 tok][8 heads]  = K[16][D] . Q^T[D][8]       mma.m16n8k16, K rows via ldmatrix
//   online softmax down the columns of S^T (one column per query head)
//   O^T[D][8 heads]      += V^T[D][16] . P^T[16][8]     mma.m16n8k16, V via ldmatrix.trans,
//                                                       P^T from S^T's layout by movmatrix.trans
// Query heads beyond the GQA group are zero columns.  P enters the second product as
// a hi + lo pair of 16-bit halves, so the weights keep about 16 bits.  K and V tiles
// arrive by 2-D TMA tensor loads with 128-byte swizzle (16-byte chunk c of row r sits
// at chunk c ^ (r % 8) of a 128-byte row), which makes the ldmatrix reads free of
// bank conflicts.
template <typename T>
struct Mma;

template <>
struct Mma<__nv_bfloat16> {
    __device__ __forceinline__ static void mma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
        asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
    // two floats -> one register, `lo` in the low half
    __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
        uint32_t r;
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
        return r;
    }
    __device__ __forceinline__ static float low(uint32_t r) { return __uint_as_float(r << 16); }
    __device__ __forceinline__ static float high(uint32_t r) { return __uint_as_float(r & 0xffff0000u); }
};

template <>
struct Mma<__half> {
    __device__ __forceinline__ static void mma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
        asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
    __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
        uint32_t r;
        asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
        return r;
    }
    __device__ __forceinline__ static float low(uint32_t r) {
        return __half2float(__ushort_as_half((unsigned short)(r & 0xffffu)));
    }
    __device__ __forceinline__ static float high(uint32_t r) {
        return __half2float(__ushort_as_half((unsigned short)(r >> 16)));
    }
};

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ uint32_t transpose8x8(uint32_t x) {
    uint32_t r;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
    return r;
}

// 2-D TMA tensor load (no multicast) completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

struct MmaParams {
    CUtensorMap tmap_k;             // [L*NB*Hkv*B rows][D] key pool
    CUtensorMap tmap_v;
    const void *q;
    void *out;
    const int32_t *tables;
    const int32_t *lens;
    float *ws_acc;
    float *ws_ml;
    const int32_t *order;           // longest-first range order, or null (launch order)
    int32_t *counters;              // [n_seqs][head_groups] split-merge counters
    int32_t max_blocks, num_blocks, num_kv_heads, num_q_heads, layer;
    int32_t split_blocks, max_splits, out_f32, heads_per_cta, head_groups;
    int32_t debug_withhold;         // see copies_withheld(); -1 outside wait-expiry tests
    float scale_log2;
};

template <int B, int D>
struct MmaShape {
    static constexpr int kBoxes = D / 64;                 // 128-byte column boxes per row
    static constexpr int kBoxBytes = B * 128;             // one box: B rows x 128 bytes
    static constexpr int kTileBytes = kBoxes * kBoxBytes;  // B x D x 2 bytes
    static constexpr int kStages = (2 * kTileBytes <= 8192) ? 8 : 4;
    static constexpr int kRingBytes = kStages * 2 * kTileBytes;
    static constexpr int kRedBytes = kConsumerWarps * 8 * (2 + D) * 4;
    static_assert(kRedBytes <= kRingBytes, "reduction area reuses the ring");
    static_assert(kStages % kConsumerWarps == 0, "each stage must belong to one consumer warp");
    static constexpr size_t kSmemBytes = 1024 + kRingBytes + 2 * kStages * sizeof(uint64_t);
};

template <typename T, int B, int D>
__global__ void __launch_bounds__(kDecodeThreads, 3) paged_decode_mma_kernel(const __grid_constant__ MmaParams p) {
    using SH = MmaShape<B, D>;
    using M = Mma<T>;
    constexpr int STAGES = SH::kStages, TILE = SH::kTileBytes, BOX = SH::kBoxBytes, KD = D / 16;
    extern __shared__ unsigned char smem_raw[];
    // 128-byte swizzled TMA destinations want 1024-byte alignment
    unsigned char *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);

    // one CTA per (range, head group); ranges longest first when an order is given
    const int hg = (int)(blockIdx.x % (unsigned)p.head_groups);
    const int rank = (int)(blockIdx.x / (unsigned)p.head_groups);
    const int item = p.order ? p.order[rank] : rank;
    const int s = item / p.max_splits;
    const int split = item % p.max_splits;
    const int hpc = p.heads_per_cta;

    int L = p.lens[s];
    if (L < 1 || (L + B - 1) / B > p.max_blocks) {
        if (threadIdx.x == 0 && hg == 0 && split == 0) raise_error(kErrBadLen);
        if (L < 1) {
            if (split == 0)
                for (int t = threadIdx.x; t < hpc * D; t += blockDim.x) {
                    const size_t idx = ((size_t)s * p.num_q_heads + hg * hpc + t / D) * D + t % D;
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
    const int group = p.num_q_heads / p.num_kv_heads;
    const int h0 = hg * hpc;
    const int g = h0 / group;

    uint64_t *full = reinterpret_cast<uint64_t *>(smem + SH::kRingBytes);
    uint64_t *empty = full + STAGES;
    float *red_m = reinterpret_cast<float *>(smem);               // [warps][8], after the loop
    float *red_l = red_m + kConsumerWarps * 8;                     // [warps][8]
    float *red_o = red_l + kConsumerWarps * 8;                     // [warps][8][D]

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

    const int gq = lane >> 2;   // accumulator row group
    const int tq = lane & 3;    // accumulator column pair
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // heads 2tq, 2tq+1
    float o[KD][4];

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
                        const int row = ((p.layer * p.num_blocks + b) * p.num_kv_heads + g) * B;
                        unsigned char *dst = smem + st * 2 * TILE;
                        mbar_arrive_expect_tx(&full[st], 2 * TILE);
#pragma unroll
                        for (int bx = 0; bx < SH::kBoxes; ++bx) {
                            tma_load_2d(dst + bx * BOX, &p.tmap_k, bx * 64, row, &full[st]);
                            tma_load_2d(dst + TILE + bx * BOX, &p.tmap_v, bx * 64, row, &full[st]);
                        }
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
        uint32_t qb[KD][2];   // Q^T fragments: column gq is query head h0 + gq
        {
            const bool qv = gq < hpc;
            const uint32_t *qrow = reinterpret_cast<const uint32_t *>(
                static_cast<const T *>(p.q) + ((size_t)s * p.num_q_heads + h0 + (qv ? gq : 0)) * D);
#pragma unroll
            for (int kk = 0; kk < KD; ++kk) {
                qb[kk][0] = qv ? qrow[(kk * 16 + 2 * tq) / 2] : 0u;
                qb[kk][1] = qv ? qrow[(kk * 16 + 8 + 2 * tq) / 2] : 0u;
            }
        }
#pragma unroll
        for (int dm = 0; dm < KD; ++dm) o[dm][0] = o[dm][1] = o[dm][2] = o[dm][3] = 0.f;
        const float sl = p.scale_log2;

        for (int i = warp; i < ntiles; i += kConsumerWarps) {
            const int st = i % STAGES;
            if (!mbar_wait_warp(&full[st], (i / STAGES) & 1)) break;
            const uint32_t kbase = smem_addr(smem + st * 2 * TILE);
            const uint32_t vbase = kbase + TILE;
            const int tok0 = (b0 + i) * B;
#pragma unroll
            for (int j = 0; j < B / 16; ++j) {
                if (tok0 + j * 16 >= L) break;          // nothing valid in this group
                float c[4] = {0.f, 0.f, 0.f, 0.f};
                {
                    const int r = j * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
                    for (int kk = 0; kk < KD; ++kk) {
                        const int chunk = (kk & 3) * 2 + (lane >> 4);
                        uint32_t a[4];
                        ldsm_x4(a, kbase + (kk >> 2) * BOX + r * 128 + ((chunk ^ (r & 7)) << 4));
                        M::mma(c, a, qb[kk][0], qb[kk][1]);
                    }
                }
                const bool v0 = tok0 + j * 16 + gq < L;
                const bool v1 = tok0 + j * 16 + gq + 8 < L;
                const float s0 = v0 ? c[0] * sl : -INFINITY, s1 = v0 ? c[1] * sl : -INFINITY;
                const float s2 = v1 ? c[2] * sl : -INFINITY, s3 = v1 ? c[3] * sl : -INFINITY;
                const bool need = fmaxf(s0, s2) > m0 + kRescaleThreshold || fmaxf(s1, s3) > m1 + kRescaleThreshold;
                if (__any_sync(0xffffffffu, need)) {
                    float t0 = fmaxf(s0, s2), t1 = fmaxf(s1, s3);
#pragma unroll
                    for (int off = 4; off < 32; off <<= 1) {
                        t0 = fmaxf(t0, __shfl_xor_sync(0xffffffffu, t0, off));
                        t1 = fmaxf(t1, __shfl_xor_sync(0xffffffffu, t1, off));
                    }
                    const float n0 = fmaxf(m0, t0), n1 = fmaxf(m1, t1);
                    const float f0 = ex2(m0 - n0), f1 = ex2(m1 - n1);
                    l0 *= f0;
                    l1 *= f1;
#pragma unroll
                    for (int dm = 0; dm < KD; ++dm) {
                        o[dm][0] *= f0;
                        o[dm][2] *= f0;
                        o[dm][1] *= f1;
                        o[dm][3] *= f1;
                    }
                    m0 = n0;
                    m1 = n1;
                }
                const float p0 = ex2(s0 - m0), p1 = ex2(s1 - m1), p2 = ex2(s2 - m0), p3 = ex2(s3 - m1);
                l0 += p0 + p2;
                l1 += p1 + p3;
                const uint32_t h01 = M::pack(p0, p1), h23 = M::pack(p2, p3);
                const uint32_t r01 = M::pack(p0 - M::low(h01), p1 - M::high(h01));
                const uint32_t r23 = M::pack(p2 - M::low(h23), p3 - M::high(h23));
                const uint32_t bh0 = transpose8x8(h01), bh1 = transpose8x8(h23);
                const uint32_t bl0 = transpose8x8(r01), bl1 = transpose8x8(r23);
                {
                    const int mi = lane >> 3;
                    const int r = j * 16 + (lane & 7) + (mi >> 1) * 8;
                    // Slots past the sequence end carry weight 0, but their values are
                    // whatever the pool holds (possibly NaN bit patterns) and 0 * NaN is
                    // NaN: zero those tokens in the V^T fragments.  Lane (gq, tq) holds
                    // tokens 2tq, 2tq+1 in a0/a1 and 2tq+8, 2tq+9 in a2/a3.
                    const int left = L - (tok0 + j * 16);           // valid tokens in this group
                    uint32_t keep01 = 0xffffffffu, keep89 = 0xffffffffu;
                    if (left < 16) {
                        const int t0 = 2 * tq;
                        keep01 = (t0 < left ? 0x0000ffffu : 0u) | (t0 + 1 < left ? 0xffff0000u : 0u);
                        keep89 = (t0 + 8 < left ? 0x0000ffffu : 0u) | (t0 + 9 < left ? 0xffff0000u : 0u);
                    }
#pragma unroll
                    for (int dm = 0; dm < KD; ++dm) {
                        const int chunk = (dm & 3) * 2 + (mi & 1);
                        uint32_t a[4];
                        ldsm_x4_trans(a, vbase + (dm >> 2) * BOX + r * 128 + ((chunk ^ (r & 7)) << 4));
                        a[0] &= keep01;
                        a[1] &= keep01;
                        a[2] &= keep89;
                        a[3] &= keep89;
                        M::mma(o[dm], a, bh0, bh1);
                        M::mma(o[dm], a, bl0, bl1);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        // l: sum over the eight token rows held by lanes differing in bits 2..4
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
#pragma unroll
        for (int dm = 0; dm < KD; ++dm) {
            float *c0 = red_o + (warp * 8 + 2 * tq) * D + dm * 16 + gq;
            float *c1 = c0 + D;
            c0[0] = o[dm][0];
            c1[0] = o[dm][1];
            c0[8] = o[dm][2];
            c1[8] = o[dm][3];
        }
    }
    __syncthreads();

    for (int t = threadIdx.x; t < hpc * D; t += blockDim.x) {
        const int h = t / D;
        const int d = t % D;
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) mx = fmaxf(mx, red_m[w * 8 + h]);
        float lsum = 0.f, osum = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const float mw = red_m[w * 8 + h];
            const float f = (mw == -INFINITY) ? 0.f : ex2(mw - mx);
            lsum += red_l[w * 8 + h] * f;
            osum += red_o[(w * 8 + h) * D + d] * f;
        }
        const int hq = h0 + h;
        if (nsplit == 1) {
            const size_t idx = ((size_t)s * p.num_q_heads + hq) * D + d;
            if (p.out_f32)
                static_cast<float *>(p.out)[idx] = osum / lsum;
            else
                static_cast<T *>(p.out)[idx] = Elem<T>::narrow(osum / lsum);
        } else {
            const size_t part = ((size_t)s * p.max_splits + split) * p.num_q_heads + hq;
            p.ws_acc[part * D + d] = osum;
            if (d == 0) {
                p.ws_ml[part * 2] = mx;
                p.ws_ml[part * 2 + 1] = lsum;
            }
        }
    }
    if (nsplit > 1)
        merge_splits_if_last<T>(p.ws_acc, p.ws_ml, p.counters + (size_t)s * p.head_groups + hg, p.out, p.out_f32, s,
                                p.num_q_heads, p.max_splits, nsplit, h0, hpc, D, reinterpret_cast<float *>(smem),
                                SH::kRingBytes / 4);
}

#include "prefill.cuh"
#include "fp8.cuh"

// ------------------------------------------------------------------ append / copy
struct AppendParams {
    unsigned char *k_layer;
    unsigned char *v_layer;
    const unsigned char *k_new;     // [n][Hkv][D]
    const unsigned char *v_new;
    const int64_t *slots;
    int32_t n_tokens, block_size, num_kv_heads, row_chunks;   // row_chunks = D*e/16
    int64_t num_blocks;
    Div32 by_chunks, by_block, by_row_chunks;                 // Hkv*row_chunks, block_size, row_chunks
};

// One thread per 16-byte chunk of a new row (all tokens, heads and chunks flattened,
// grid-stride); the source read is issued before the slot lookup, so a thread's loads
// are in flight together.
template <bool NARROW>
__global__ void __launch_bounds__(256) append_kv_kernel(const AppendParams p) {
    const int64_t chunks = (int64_t)p.num_kv_heads * p.row_chunks;   // 16-byte chunks per token
    const int64_t total = (int64_t)p.n_tokens * chunks;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < total; g += stride) {
        int64_t i;
        int t;
        if constexpr (NARROW) {
            i = div32((uint32_t)g, p.by_chunks);
            t = (int)((uint32_t)g - (uint32_t)i * (uint32_t)chunks);
        } else {
            i = g / chunks;
            t = (int)(g - i * chunks);
        }
        const uint4 kx = reinterpret_cast<const uint4 *>(p.k_new)[g];   // [n][Hkv][row_chunks]
        const uint4 vx = reinterpret_cast<const uint4 *>(p.v_new)[g];
        const int64_t slot = p.slots[i];
        if (slot < 0) continue;                                            // padding row
        int64_t blk;
        int off, h;
        if constexpr (NARROW) {
            if (slot >= p.num_blocks * p.block_size) {
                if (t == 0) raise_error(kErrBadSlot);
                continue;
            }
            blk = div32((uint32_t)slot, p.by_block);
            off = (int)((uint32_t)slot - (uint32_t)blk * (uint32_t)p.block_size);
            h = (int)div32((uint32_t)t, p.by_row_chunks);
        } else {
            blk = slot / p.block_size;
            off = (int)(slot % p.block_size);
            if (blk >= p.num_blocks) {
                if (t == 0) raise_error(kErrBadSlot);
                continue;
            }
            h = t / p.row_chunks;
        }
        const int c = t - h * p.row_chunks;
        const size_t dst = (((size_t)blk * p.num_kv_heads + h) * p.block_size + off) * p.row_chunks + c;
        reinterpret_cast<uint4 *>(p.k_layer)[dst] = kx;
        reinterpret_cast<uint4 *>(p.v_layer)[dst] = vx;
    }
}

struct CopyParams {
    unsigned char *k_pool;
    unsigned char *v_pool;
    unsigned char *scales;    // FP8 pools: scale bytes (null otherwise)
    const int32_t *pairs;     // [n][2] (src, dst)
    int64_t block_chunks;     // 16-byte chunks per block (all heads)
    int64_t layer_chunks;     // 16-byte chunks per layer
    int64_t scale_block_chunks, scale_layer_chunks;
    int32_t num_blocks;
};

__global__ void __launch_bounds__(256) copy_blocks_kernel(const CopyParams p) {
    const int pair = blockIdx.x;
    const int layer = blockIdx.y;
    const int src = p.pairs[2 * pair];
    const int dst = p.pairs[2 * pair + 1];
    if ((unsigned)src >= (unsigned)p.num_blocks || (unsigned)dst >= (unsigned)p.num_blocks) {
        if (threadIdx.x == 0) raise_error(kErrBadBlock);
        return;
    }
    uint4 *pool = reinterpret_cast<uint4 *>(blockIdx.z == 0 ? p.k_pool : p.v_pool);
    uint4 *from = pool + layer * p.layer_chunks + (int64_t)src * p.block_chunks;
    uint4 *to = pool + layer * p.layer_chunks + (int64_t)dst * p.block_chunks;
    for (int64_t t = threadIdx.x; t < p.block_chunks; t += blockDim.x) to[t] = from[t];
    if (p.scales && blockIdx.z == 0) {
        uint4 *sc = reinterpret_cast<uint4 *>(p.scales) + layer * p.scale_layer_chunks;
        for (int64_t t = threadIdx.x; t < p.scale_block_chunks; t += blockDim.x)
            sc[(int64_t)dst * p.scale_block_chunks + t] = sc[(int64_t)src * p.scale_block_chunks + t];
    }
}

// ------------------------------------------------------------------ swap copies
constexpr int kSwapChunk = 256;   // block ids passed by value per launch

struct SwapParams {
    unsigned char *k_pool;
    unsigned char *v_pool;
    unsigned char *scales;        // FP8 pools: scale bytes (null otherwise)
    unsigned char *host;          // device-visible address of the page-locked host buffer
    int64_t block_chunks;         // 16-byte chunks of one block (all heads) in one layer
    int64_t layer_chunks;         // 16-byte chunks of one layer of the pool
    int64_t scale_block_chunks, scale_layer_chunks;
    int64_t record_chunks;        // one [block][layer] record of the host buffer
    int32_t num_blocks, first, count, to_host;
    int32_t blocks[kSwapChunk];
};

// grid (block in chunk, layer, K|V): one CTA moves one block of one layer of K or V.
__global__ void __launch_bounds__(256) swap_copy_kernel(const __grid_constant__ SwapParams p) {
    const int i = blockIdx.x;
    const int layer = blockIdx.y;
    const int kv = blockIdx.z;
    const int blk = p.blocks[i];
    if ((unsigned)blk >= (unsigned)p.num_blocks) {
        if (threadIdx.x == 0) raise_error(kErrBadBlock);
        return;
    }
    uint4 *pool = reinterpret_cast<uint4 *>(kv == 0 ? p.k_pool : p.v_pool) + layer * p.layer_chunks +
                  (int64_t)blk * p.block_chunks;
    const int64_t layers = gridDim.y;
    uint4 *rec = reinterpret_cast<uint4 *>(p.host) + ((int64_t)(p.first + i) * layers + layer) * p.record_chunks;
    uint4 *host = rec + kv * p.block_chunks;
    if (p.to_host)
        for (int64_t t = threadIdx.x; t < p.block_chunks; t += blockDim.x) host[t] = pool[t];
    else
        for (int64_t t = threadIdx.x; t < p.block_chunks; t += blockDim.x) pool[t] = host[t];
    if (p.scales && kv == 0) {
        uint4 *sc = reinterpret_cast<uint4 *>(p.scales) + layer * p.scale_layer_chunks + (int64_t)blk * p.scale_block_chunks;
        uint4 *hs = rec + 2 * p.block_chunks;
        if (p.to_host)
            for (int64_t t = threadIdx.x; t < p.scale_block_chunks; t += blockDim.x) hs[t] = sc[t];
        else
            for (int64_t t = threadIdx.x; t < p.scale_block_chunks; t += blockDim.x) sc[t] = hs[t];
    }
}

// ------------------------------------------------------------------ host dispatch
pa_status check_launch(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
    return PA_OK;
}

// Raise the dynamic shared-memory limit of one kernel once per device; `done` is
// the caller's per-kernel flag array (one per template instantiation).
template <typename K>
pa_status ensure_smem(K kernel, size_t bytes, bool (&done)[64]) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return fail(PA_ERR_CUDA, "cudaGetDevice failed");
    if (dev < 64 && done[dev]) return PA_OK;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
    if (dev < 64) done[dev] = true;
    return PA_OK;
}

template <typename T, int B, int D>
pa_status launch_reduce(const ReduceParams &r, int n_seqs, cudaStream_t stream) {
    if (r.max_splits <= 1) return PA_OK;
    split_reduce_kernel<T, B, D><<<dim3(n_seqs, r.num_q_heads), D, 0, stream>>>(r);
    pa_internal::launch_count.fetch_add(1);
    return check_launch("split_reduce_kernel");
}

template <typename T, int B, int D, int HPC>
pa_status launch_simt(const DecodeParams &p, const ReduceParams &r, cudaStream_t stream) {
    constexpr size_t smem = decode_smem_bytes<T, B, D, HPC>();
    auto kernel = paged_decode_simt_kernel<T, B, D, HPC>;
    static bool smem_set[64] = {};
    pa_status st = ensure_smem(kernel, smem, smem_set);
    if (st != PA_OK) return st;
    dim3 grid(p.n_seqs, p.num_q_heads / HPC, p.max_splits);
    kernel<<<grid, kDecodeThreads, smem, stream>>>(p);
    pa_internal::launch_count.fetch_add(1);
    st = check_launch("paged_decode_simt_kernel");
    if (st != PA_OK) return st;
    return launch_reduce<T, B, D>(r, p.n_seqs, stream);
}

template <typename T, int B, int D>
pa_status dispatch_hpc(const DecodeParams &p, const ReduceParams &r, int hpc, cudaStream_t stream) {
    switch (hpc) {
    case 1: return launch_simt<T, B, D, 1>(p, r, stream);
    case 2: return launch_simt<T, B, D, 2>(p, r, stream);
    case 4: return launch_simt<T, B, D, 4>(p, r, stream);
    }
    return fail(PA_ERR_UNSUPPORTED, "unsupported query heads per KV head");
}

template <typename T>
pa_status dispatch_simt(const DecodeParams &p, const ReduceParams &r, int B, int D, int hpc, cudaStream_t stream) {
    if (B == 16 && D == 128) return dispatch_hpc<T, 16, 128>(p, r, hpc, stream);
    if (B == 32 && D == 128) return dispatch_hpc<T, 32, 128>(p, r, hpc, stream);
    if (B == 16 && D == 64) return dispatch_hpc<T, 16, 64>(p, r, hpc, stream);
    if (B == 32 && D == 64) return dispatch_hpc<T, 32, 64>(p, r, hpc, stream);
    return fail(PA_ERR_UNSUPPORTED, "block_size must be 16 or 32 and head_dim 64 or 128");
}

template <typename T, int B, int D>
pa_status launch_mma(const MmaParams &p, const ReduceParams &r, int n_seqs, cudaStream_t stream) {
    constexpr size_t smem = MmaShape<B, D>::kSmemBytes;
    auto kernel = paged_decode_mma_kernel<T, B, D>;
    static bool smem_set[64] = {};
    pa_status st = ensure_smem(kernel, smem, smem_set);
    if (st != PA_OK) return st;
    const dim3 grid((unsigned)((int64_t)n_seqs * p.max_splits * p.head_groups));
    kernel<<<grid, kDecodeThreads, smem, stream>>>(p);
    pa_internal::launch_count.fetch_add(1);
    return check_launch("paged_decode_mma_kernel");   // splits are merged in the kernel
}

template <typename T>
pa_status dispatch_mma(const MmaParams &p, const ReduceParams &r, int n_seqs, int B, int D, cudaStream_t stream) {
    if (B == 16 && D == 128) return launch_mma<T, 16, 128>(p, r, n_seqs, stream);
    if (B == 32 && D == 128) return launch_mma<T, 32, 128>(p, r, n_seqs, stream);
    if (B == 16 && D == 64) return launch_mma<T, 16, 64>(p, r, n_seqs, stream);
    if (B == 32 && D == 64) return launch_mma<T, 32, 64>(p, r, n_seqs, stream);
    return fail(PA_ERR_UNSUPPORTED, "block_size must be 16 or 32 and head_dim 64 or 128");
}

template <typename T, int B, int HEADS>
pa_status launch_fp8(const fp8::Params &p, const ReduceParams &r, int n_seqs, cudaStream_t stream) {
    constexpr size_t smem = fp8::Shape<B, HEADS>::kSmemBytes;
    auto kernel = fp8::decode_kernel<T, B, HEADS>;
    static bool smem_set[64] = {};
    pa_status st = ensure_smem(kernel, smem, smem_set);
    if (st != PA_OK) return st;
    const dim3 grid((unsigned)((int64_t)n_seqs * p.max_splits * p.head_groups));
    kernel<<<grid, kDecodeThreads, smem, stream>>>(p);
    pa_internal::launch_count.fetch_add(1);
    return check_launch("fp8::decode_kernel");   // splits are merged in the kernel
}

// TMA descriptors over a 16-bit or FP8 pool: 2-D [rows][head_dim], boxes of 128
// bytes (the 128-byte swizzle span: 64 16-bit elements or 128 codes) by block_size rows.
pa_status ensure_tensor_maps(pa_pool *pool, int box_rows) {
    if (pool->tmaps_ready && pool->tmap_rows == box_rows) return PA_OK;
    using Encode = PFN_cuTensorMapEncodeTiled_v12000;
    static Encode encode = nullptr;
    if (!encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
        encode = reinterpret_cast<Encode>(fn);
    }
    const pa_pool_config &c = pool->cfg;
    const uint64_t rows = (uint64_t)c.num_layers * c.num_blocks * c.num_kv_heads * c.block_size;
    if (rows >= (1ull << 31))
        return fail(PA_ERR_UNSUPPORTED, "pool too large for 32-bit TMA row coordinates");
    const CUtensorMapDataType dt = c.dtype == PA_BF16       ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                   : c.dtype == PA_FP8_E4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                                            : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const size_t eb = pool->elem_bytes();
    cuuint64_t dims[2] = {(cuuint64_t)c.head_dim, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(c.head_dim * eb)};
    cuuint32_t box[2] = {(cuuint32_t)(128 / eb), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    void *bases[2] = {pool->k_pool, pool->v_pool};
    CUtensorMap *maps[2] = {&pool->tmap_k, &pool->tmap_v};
    for (int i = 0; i < 2; ++i) {
        CUresult r = encode(maps[i], dt, 2, bases[i], dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (" + std::to_string((int)r) + ")");
    }
    pool->tmaps_ready = true;
    pool->tmap_rows = box_rows;
    return PA_OK;
}

// One shared-memory flag per kernel instantiation (the flag must not be shared between
// kernels of the same pointer type).
template <typename T, int B>
pa_status launch_prefill(const prefill::Params &p, dim3 grid, cudaStream_t stream) {
    auto kernel = prefill::paged_prefill_kernel<T, B>;
    static bool smem_set[64] = {};
    pa_status st = ensure_smem(kernel, prefill::kSmemBytes, smem_set);
    if (st != PA_OK) return st;
    kernel<<<grid, prefill::kThreads, prefill::kSmemBytes, stream>>>(p);
    pa_internal::launch_count.fetch_add(1);
    return check_launch("paged_prefill_kernel");
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Decode or prefill CTA whose copies a wait-expiry test withholds (pa_debug_wait_test),
// else -1.
std::atomic<int32_t> g_debug_withhold{-1};

// Decode workspace: split partials (acc [parts][D] then (m, l) [parts][2], fp32) when a
// sequence can have more than one split, then the longest-first range order
// (int32 [n_seqs * max_splits]), each part rounded up to 16 bytes.
size_t partial_bytes(int32_t n_seqs, int32_t num_q_heads, int32_t head_dim, int32_t max_splits) {
    if (max_splits <= 1) return 0;
    const size_t parts = (size_t)n_seqs * max_splits * num_q_heads;
    return (parts * head_dim * sizeof(float) + parts * 2 * sizeof(float) + 15) & ~(size_t)15;
}

size_t order_bytes(int32_t n_seqs, int32_t max_splits) {
    return ((size_t)n_seqs * max_splits * sizeof(int32_t) + 15) & ~(size_t)15;
}

// split-merge counters, one per (sequence, head group) -- at most num_q_heads groups
size_t counter_bytes(int32_t n_seqs, int32_t num_q_heads, int32_t max_splits) {
    if (max_splits <= 1) return 0;
    return ((size_t)n_seqs * num_q_heads * sizeof(int32_t) + 15) & ~(size_t)15;
}

}  // namespace

// ------------------------------------------------------------------ allocation-free decode
// Split-K scratch for pa_decode_attention_static: a fixed array in this library's
// device memory.  Every GPU that loads the library holds these bytes until the
// process exits; every call of pa_decode_attention_static on a device shares them.
static __device__ __align__(256) unsigned char pa_static_split_scratch[PA_STATIC_WORKSPACE_BYTES];

namespace {

// Device address of the scratch array on the current device.  Host code cannot pass
// the array's name to a kernel (on the host it is only a stand-in symbol), so the
// first call on each device looks the address up with that device current and
// keeps it.  Host threads may make their first calls at the same time: each looks
// the address up (the same value) and publishes it atomically.  The kept address
// belongs to the device's current context; after cudaDeviceReset it is stale.
pa_status static_scratch_address(void **out) {
    static std::atomic<void *> addr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    if (dev < 0 || dev >= 64) return fail(PA_ERR_UNSUPPORTED, "pa_decode_attention_static: device ordinal >= 64");
    void *p = addr[dev].load(std::memory_order_acquire);
    if (!p) {
        e = cudaGetSymbolAddress(&p, pa_static_split_scratch);
        if (e != cudaSuccess || !p)
            return fail(PA_ERR_CUDA, std::string("cudaGetSymbolAddress(split scratch): ") + cudaGetErrorString(e));
        addr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return PA_OK;
}

}  // namespace

extern "C" {

int32_t pa_decode_max_splits(int32_t block_size, int32_t max_blocks, int32_t split_tokens) {
    if (block_size < 1 || max_blocks < 1 || split_tokens < 0) return 0;
    if (split_tokens == 0) return 1;
    const int32_t split_blocks = split_tokens / block_size;
    if (split_blocks < 1) return 0;
    return (max_blocks + split_blocks - 1) / split_blocks;
}

size_t pa_decode_workspace_bytes(int32_t n_seqs, int32_t num_q_heads, int32_t head_dim, int32_t max_splits) {
    if (n_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_splits < 1) return 0;
    return partial_bytes(n_seqs, num_q_heads, head_dim, max_splits) + order_bytes(n_seqs, max_splits) +
           counter_bytes(n_seqs, num_q_heads, max_splits);
}

pa_status pa_decode_attention(pa_pool *pool, int32_t layer, const void *q, void *out, pa_dtype out_dtype,
                              const int32_t *block_tables_dev, int32_t max_blocks, const int32_t *seq_lens_dev,
                              int32_t n_seqs, int32_t num_q_heads, float scale, int32_t split_tokens,
                              void *workspace, size_t ws_bytes, pa_stream stream) {
    pa_internal::TraceRange trace_("pa_decode_attention");
    if (!pool || !pool->device_ready())
        return fail(PA_ERR_INVALID_ARG, "pa_decode_attention: pool has no device memory (or no FP8 scales)");
    const pa_pool_config &c = pool->cfg;
    if (layer < 0 || layer >= c.num_layers) return fail(PA_ERR_INVALID_ARG, "pa_decode_attention: layer out of range");
    if (n_seqs < 0 || max_blocks < 1) return fail(PA_ERR_INVALID_ARG, "pa_decode_attention: bad n_seqs/max_blocks");
    if (n_seqs == 0) return PA_OK;
    if (!q || !out || !block_tables_dev || !seq_lens_dev)
        return fail(PA_ERR_INVALID_ARG, "pa_decode_attention: null device pointer");
    if (!aligned16(q) || !aligned16(out) || ((uintptr_t)block_tables_dev & 3) || ((uintptr_t)seq_lens_dev & 3))
        return fail(PA_ERR_INVALID_ARG, "pa_decode_attention: misaligned pointer");
    if (out_dtype != PA_F32 && out_dtype != pool->act_dtype())
        return fail(PA_ERR_INVALID_ARG, "pa_decode_attention: out_dtype must be PA_F32 or the pool's query type");
    if (pool->fp8() && c.head_dim != fp8::kD)
        return fail(PA_ERR_UNSUPPORTED, "pa_decode_attention: FP8 pools need head_dim 128");
    if (num_q_heads < 1 || num_q_heads % c.num_kv_heads != 0)
        return fail(PA_ERR_INVALID_ARG, "pa_decode_attention: num_q_heads must be a multiple of num_kv_heads");
    const int group = num_q_heads / c.num_kv_heads;
    if (group != 1 && group != 2 && group != 4 && group != 8)
        return fail(PA_ERR_UNSUPPORTED, "pa_decode_attention: query heads per KV head must be 1, 2, 4 or 8");
    if (!std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "pa_decode_attention: scale must be finite");
    if (split_tokens < 0 || (split_tokens > 0 && split_tokens % c.block_size != 0))
        return fail(PA_ERR_INVALID_ARG, "pa_decode_attention: split_tokens must be 0 or a multiple of block_size");
    const int32_t max_splits = pa_decode_max_splits(c.block_size, max_blocks, split_tokens);
    if (max_splits > 65535 || num_q_heads > 65535)
        return fail(PA_ERR_UNSUPPORTED, "pa_decode_attention: grid too large");
    const size_t need_partials = partial_bytes(n_seqs, num_q_heads, c.head_dim, max_splits);
    const size_t need = pa_decode_workspace_bytes(n_seqs, num_q_heads, c.head_dim, max_splits);
    if (workspace && !aligned16(workspace))
        return fail(PA_ERR_INVALID_ARG, "pa_decode_attention: workspace must be 16-byte aligned");
    if (need_partials > 0 && (!workspace || ws_bytes < need_partials))
        return fail(PA_ERR_INVALID_ARG, "pa_decode_attention: workspace missing or smaller than " +
                                            std::to_string(need) + " bytes");

    const size_t parts = (size_t)n_seqs * max_splits * num_q_heads;
    float *ws_acc = static_cast<float *>(workspace);
    float *ws_ml = need_partials > 0 ? static_cast<float *>(workspace) + parts * c.head_dim : nullptr;
    const int32_t split_blocks = split_tokens > 0 ? split_tokens / c.block_size : max_blocks;
    const float scale_log2 = (float)((double)scale * 1.4426950408889634);   // scale * log2(e)
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // Longest ranges first, when the workspace has room for the order and the grid is
    // more than about two CTAs per SM (below that there is no tail to shape).
    const int head_groups = c.dtype == PA_F32 ? 0
                            : pool->fp8() ? c.num_kv_heads / fp8::heads_per_cta(group, c.num_kv_heads, c.block_size)
                                          : c.num_kv_heads;
    if ((int64_t)n_seqs * max_splits * (head_groups > 0 ? head_groups : 1) >= (1ll << 31))
        return fail(PA_ERR_UNSUPPORTED, "pa_decode_attention: grid too large");
    // Tensor-core paths: with splits the full workspace is needed (partials, order,
    // merge counters) and the plan kernel runs first (it zeroes the counters); without
    // splits the order is used when there is room for it and the grid is more than
    // about two CTAs per SM (below that there is no tail to shape).
    if (head_groups > 0 && max_splits > 1 && ws_bytes < need)
        return fail(PA_ERR_INVALID_ARG, "pa_decode_attention: workspace smaller than " + std::to_string(need) +
                                            " bytes");
    int32_t *order = nullptr, *counters = nullptr;
    if (head_groups > 0 && workspace && ws_bytes >= need &&
        (max_splits > 1 || (int64_t)n_seqs * max_splits * head_groups > 2 * 148)) {
        unsigned char *w = static_cast<unsigned char *>(workspace);
        order = reinterpret_cast<int32_t *>(w + need_partials);
        counters = max_splits > 1 ? reinterpret_cast<int32_t *>(w + need_partials + order_bytes(n_seqs, max_splits))
                                  : nullptr;
        PlanParams pp;
        pp.lens = seq_lens_dev;
        pp.order = order;
        pp.counters = counters;
        pp.n_seqs = n_seqs;
        pp.max_blocks = max_blocks;
        pp.block_size = c.block_size;
        pp.split_blocks = split_blocks;
        pp.max_splits = max_splits;
        pp.n_counters = counters ? n_seqs * head_groups : 0;
        plan_kernel<<<1, kPlanThreads, 0, st>>>(pp);
        pa_internal::launch_count.fetch_add(1);
        pa_status ps = check_launch("plan_kernel");
        if (ps != PA_OK) return ps;
    }

    ReduceParams r;
    r.lens = seq_lens_dev;
    r.out = out;
    r.ws_acc = ws_acc;
    r.ws_ml = ws_ml;
    r.max_blocks = max_blocks;
    r.num_q_heads = num_q_heads;
    r.split_blocks = split_blocks;
    r.max_splits = max_splits;
    r.out_f32 = out_dtype == PA_F32;

    if (c.dtype == PA_F32) {
        // fp32 caches: CUDA-core kernel (the tensor-core path takes 16-bit operands only)
        DecodeParams p;
        p.k_layer = static_cast<const unsigned char *>(pool->k_pool) + (size_t)layer * pool->layer_bytes();
        p.v_layer = static_cast<const unsigned char *>(pool->v_pool) + (size_t)layer * pool->layer_bytes();
        p.q = q;
        p.out = out;
        p.tables = block_tables_dev;
        p.lens = seq_lens_dev;
        p.ws_acc = ws_acc;
        p.ws_ml = ws_ml;
        p.n_seqs = n_seqs;
        p.max_blocks = max_blocks;
        p.num_blocks = c.num_blocks;
        p.num_kv_heads = c.num_kv_heads;
        p.num_q_heads = num_q_heads;
        p.split_blocks = split_blocks;
        p.max_splits = max_splits;
        p.out_f32 = r.out_f32;
        p.scale_log2 = scale_log2;
        p.debug_withhold = g_debug_withhold.load(std::memory_order_relaxed);
        const int hpc = group < 4 ? group : 4;
        return dispatch_simt<float>(p, r, c.block_size, c.head_dim, hpc, st);
    }
    if (pool->fp8()) {
        const int heads = fp8::heads_per_cta(group, c.num_kv_heads, c.block_size);
        pa_status s2 = ensure_tensor_maps(pool, heads * c.block_size);
        if (s2 != PA_OK) return s2;
        fp8::Params p;
        p.tmap_k = pool->tmap_k;
        p.tmap_v = pool->tmap_v;
        p.s_layer = static_cast<const unsigned char *>(pool->scales) + (size_t)layer * pool->scale_layer_bytes();
        p.q = q;
        p.out = out;
        p.tables = block_tables_dev;
        p.lens = seq_lens_dev;
        p.ws_acc = ws_acc;
        p.ws_ml = ws_ml;
        p.max_blocks = max_blocks;
        p.num_blocks = c.num_blocks;
        p.num_kv_heads = c.num_kv_heads;
        p.num_q_heads = num_q_heads;
        p.layer = layer;
        p.split_blocks = split_blocks;
        p.max_splits = max_splits;
        p.out_f32 = r.out_f32;
        p.group = group;
        p.head_groups = head_groups;
        p.order = order;
        p.counters = counters;
        p.scale_log2 = scale_log2;
        p.debug_withhold = g_debug_withhold.load(std::memory_order_relaxed);
        const bool bf = c.act_dtype == PA_BF16;
#define PA_FP8_LAUNCH(B, H) \
    (bf ? launch_fp8<__nv_bfloat16, B, H>(p, r, n_seqs, st) : launch_fp8<__half, B, H>(p, r, n_seqs, st))
        if (c.block_size == 16) {
            if (heads == 4) return PA_FP8_LAUNCH(16, 4);
            if (heads == 2) return PA_FP8_LAUNCH(16, 2);
            return PA_FP8_LAUNCH(16, 1);
        }
        if (c.block_size == 32) {
            if (heads == 2) return PA_FP8_LAUNCH(32, 2);
            return PA_FP8_LAUNCH(32, 1);
        }
#undef PA_FP8_LAUNCH
        return fail(PA_ERR_UNSUPPORTED, "pa_decode_attention: block_size must be 16 or 32");
    }
    pa_status s2 = ensure_tensor_maps(pool, c.block_size);
    if (s2 != PA_OK) return s2;
    MmaParams p;
    p.tmap_k = pool->tmap_k;
    p.tmap_v = pool->tmap_v;
    p.q = q;
    p.out = out;
    p.tables = block_tables_dev;
    p.lens = seq_lens_dev;
    p.ws_acc = ws_acc;
    p.ws_ml = ws_ml;
    p.max_blocks = max_blocks;
    p.num_blocks = c.num_blocks;
    p.num_kv_heads = c.num_kv_heads;
    p.num_q_heads = num_q_heads;
    p.layer = layer;
    p.split_blocks = split_blocks;
    p.max_splits = max_splits;
    p.out_f32 = r.out_f32;
    p.heads_per_cta = group;   // the whole GQA group (<= 8) shares one CTA
    p.head_groups = head_groups;
    p.order = order;
    p.counters = counters;
    p.scale_log2 = scale_log2;
    p.debug_withhold = g_debug_withhold.load(std::memory_order_relaxed);
    if (c.dtype == PA_BF16) return dispatch_mma<__nv_bfloat16>(p, r, n_seqs, c.block_size, c.head_dim, st);
    return dispatch_mma<__half>(p, r, n_seqs, c.block_size, c.head_dim, st);
}

pa_status pa_prefill_attention(pa_pool *pool, int32_t layer, const void *q, void *out, pa_dtype out_dtype,
                               const int32_t *block_tables_dev, int32_t max_blocks, const int32_t *seq_lens_dev,
                               const int32_t *q_start_dev, int32_t n_seqs, int32_t max_q_len, int32_t num_q_heads,
                               float scale, pa_stream stream) {
    pa_internal::TraceRange trace_("pa_prefill_attention");
    if (!pool || !pool->k_pool) return fail(PA_ERR_INVALID_ARG, "pa_prefill_attention: pool has no device memory");
    const pa_pool_config &c = pool->cfg;
    if (layer < 0 || layer >= c.num_layers) return fail(PA_ERR_INVALID_ARG, "pa_prefill_attention: layer out of range");
    if (n_seqs < 0 || max_blocks < 1 || max_q_len < 0)
        return fail(PA_ERR_INVALID_ARG, "pa_prefill_attention: bad n_seqs / max_blocks / max_q_len");
    if (n_seqs == 0 || max_q_len == 0) return PA_OK;
    if (!q || !out || !block_tables_dev || !seq_lens_dev || !q_start_dev)
        return fail(PA_ERR_INVALID_ARG, "pa_prefill_attention: null device pointer");
    if (!aligned16(q) || !aligned16(out) || ((uintptr_t)block_tables_dev & 3) || ((uintptr_t)seq_lens_dev & 3) ||
        ((uintptr_t)q_start_dev & 3))
        return fail(PA_ERR_INVALID_ARG, "pa_prefill_attention: misaligned pointer");
    if (c.dtype == PA_F32 || c.dtype == PA_FP8_E4M3)
        return fail(PA_ERR_UNSUPPORTED, "pa_prefill_attention: the tensor-core path takes fp16 / bf16 caches");
    if (c.head_dim != 128 || (c.block_size != 16 && c.block_size != 32))
        return fail(PA_ERR_UNSUPPORTED, "pa_prefill_attention: head_dim 128 and block_size 16 or 32 only");
    if (out_dtype != PA_F32 && out_dtype != c.dtype)
        return fail(PA_ERR_INVALID_ARG, "pa_prefill_attention: out_dtype must be PA_F32 or the pool dtype");
    if (num_q_heads < 1 || num_q_heads % c.num_kv_heads != 0)
        return fail(PA_ERR_INVALID_ARG, "pa_prefill_attention: num_q_heads must be a multiple of num_kv_heads");
    const int group = num_q_heads / c.num_kv_heads;
    if (group != 1 && group != 2 && group != 4 && group != 8)
        return fail(PA_ERR_UNSUPPORTED, "pa_prefill_attention: query heads per KV head must be 1, 2, 4 or 8");
    if (!std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "pa_prefill_attention: scale must be finite");
    const int64_t tiles = ((int64_t)max_q_len * group + prefill::kTiles * prefill::kRows - 1) /
                          (prefill::kTiles * prefill::kRows);
    if (tiles > INT32_MAX || c.num_kv_heads > 65535 || n_seqs > 65535)
        return fail(PA_ERR_UNSUPPORTED, "pa_prefill_attention: grid too large");
    pa_status st = ensure_tensor_maps(pool, c.block_size);
    if (st != PA_OK) return st;
    prefill::Params p;
    p.tmap_k = pool->tmap_k;
    p.tmap_v = pool->tmap_v;
    p.q = q;
    p.out = out;
    p.tables = block_tables_dev;
    p.lens = seq_lens_dev;
    p.q_start = q_start_dev;
    p.max_blocks = max_blocks;
    p.num_blocks = c.num_blocks;
    p.num_kv_heads = c.num_kv_heads;
    p.num_q_heads = num_q_heads;
    p.layer = layer;
    p.block_size = c.block_size;
    p.out_f32 = out_dtype == PA_F32;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634);
    p.debug_withhold = g_debug_withhold.load(std::memory_order_relaxed);
    const dim3 grid((unsigned)tiles, c.num_kv_heads, n_seqs);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (c.dtype == PA_BF16)
        return c.block_size == 16 ? launch_prefill<__nv_bfloat16, 16>(p, grid, cs)
                                  : launch_prefill<__nv_bfloat16, 32>(p, grid, cs);
    return c.block_size == 16 ? launch_prefill<__half, 16>(p, grid, cs) : launch_prefill<__half, 32>(p, grid, cs);
}

pa_status pa_append_kv(pa_pool *pool, int32_t layer, const void *k_new, const void *v_new,
                       const int64_t *slot_mapping_dev, int32_t n_tokens, pa_stream stream) {
    pa_internal::TraceRange trace_("pa_append_kv");
    if (!pool || !pool->device_ready())
        return fail(PA_ERR_INVALID_ARG, "pa_append_kv: pool has no device memory (or no FP8 scales)");
    if (layer < 0 || layer >= pool->cfg.num_layers) return fail(PA_ERR_INVALID_ARG, "pa_append_kv: layer out of range");
    if (n_tokens < 0) return fail(PA_ERR_INVALID_ARG, "pa_append_kv: negative n_tokens");
    if (n_tokens == 0) return PA_OK;
    if (!k_new || !v_new || !slot_mapping_dev || !aligned16(k_new) || !aligned16(v_new) ||
        ((uintptr_t)slot_mapping_dev & 7))
        return fail(PA_ERR_INVALID_ARG, "pa_append_kv: null or misaligned device pointer");
    if (pool->fp8()) {
        const pa_pool_config &c = pool->cfg;
        if (c.head_dim != 64 && c.head_dim != 128)
            return fail(PA_ERR_UNSUPPORTED, "pa_append_kv: FP8 pools need head_dim 64 or 128");
        fp8::AppendParams p;
        p.k_layer = static_cast<unsigned char *>(pool->k_pool) + (size_t)layer * pool->layer_bytes();
        p.v_layer = static_cast<unsigned char *>(pool->v_pool) + (size_t)layer * pool->layer_bytes();
        p.s_layer = static_cast<unsigned char *>(pool->scales) + (size_t)layer * pool->scale_layer_bytes();
        p.k_new = static_cast<const unsigned char *>(k_new);
        p.v_new = static_cast<const unsigned char *>(v_new);
        p.slots = slot_mapping_dev;
        p.n_tokens = n_tokens;
        p.block_size = c.block_size;
        p.num_kv_heads = c.num_kv_heads;
        p.num_blocks = c.num_blocks;
        const int64_t rows2 = 2 * (int64_t)n_tokens * c.num_kv_heads;   // K rows, then V rows
        const int64_t warps = (rows2 + 32 / fp8::kAppendLanes - 1) / (32 / fp8::kAppendLanes);
        const int grid = (int)std::min<int64_t>((warps + 7) / 8, 148 * 16);
        p.by_heads = make_div32((uint32_t)c.num_kv_heads);
        p.by_block = make_div32((uint32_t)c.block_size);
        const bool narrow = rows2 < INT32_MAX && (int64_t)c.num_blocks * c.block_size < INT32_MAX;
        cudaStream_t cs = static_cast<cudaStream_t>(stream);
        const bool bf = c.act_dtype == PA_BF16;
#define PA_FP8_APPEND(TT, DD)                                                          \
    (narrow ? fp8::append_kernel<TT, DD, true><<<grid, 256, 0, cs>>>(p)              \
            : fp8::append_kernel<TT, DD, false><<<grid, 256, 0, cs>>>(p))
        if (c.head_dim == 128) {
            if (bf)
                PA_FP8_APPEND(__nv_bfloat16, 128);
            else
                PA_FP8_APPEND(__half, 128);
        } else {
            if (bf)
                PA_FP8_APPEND(__nv_bfloat16, 64);
            else
                PA_FP8_APPEND(__half, 64);
        }
#undef PA_FP8_APPEND
        pa_internal::launch_count.fetch_add(1);
        return check_launch("fp8::append_kernel");
    }
    const size_t row_bytes = (size_t)pool->cfg.head_dim * pool->elem_bytes();
    if (row_bytes % 16) return fail(PA_ERR_UNSUPPORTED, "pa_append_kv: head_dim * element size must be a multiple of 16");
    AppendParams p;
    p.k_layer = static_cast<unsigned char *>(pool->k_pool) + (size_t)layer * pool->layer_bytes();
    p.v_layer = static_cast<unsigned char *>(pool->v_pool) + (size_t)layer * pool->layer_bytes();
    p.k_new = static_cast<const unsigned char *>(k_new);
    p.v_new = static_cast<const unsigned char *>(v_new);
    p.slots = slot_mapping_dev;
    p.n_tokens = n_tokens;
    p.block_size = pool->cfg.block_size;
    p.num_kv_heads = pool->cfg.num_kv_heads;
    p.row_chunks = (int32_t)(row_bytes / 16);
    p.num_blocks = pool->cfg.num_blocks;
    const int64_t threads = (int64_t)n_tokens * p.num_kv_heads * p.row_chunks;
    const int grid = (int)std::min<int64_t>((threads + 255) / 256, 148 * 16);
    p.by_chunks = make_div32((uint32_t)(p.num_kv_heads * p.row_chunks));
    p.by_block = make_div32((uint32_t)p.block_size);
    p.by_row_chunks = make_div32((uint32_t)p.row_chunks);
    const bool narrow = threads < INT32_MAX && p.num_blocks * p.block_size < INT32_MAX;
    if (narrow)
        append_kv_kernel<true><<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    else
        append_kv_kernel<false><<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    pa_internal::launch_count.fetch_add(1);
    return check_launch("append_kv_kernel");
}

pa_status pa_copy_blocks(pa_pool *pool, const int32_t *pairs_dev, int32_t n_pairs, pa_stream stream) {
    pa_internal::TraceRange trace_("pa_copy_blocks");
    if (!pool || !pool->device_ready())
        return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks: pool has no device memory (or no FP8 scales)");
    if (n_pairs < 0) return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks: negative n_pairs");
    if (n_pairs == 0) return PA_OK;
    if (!pairs_dev || ((uintptr_t)pairs_dev & 3)) return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks: bad pairs pointer");
    if (pool->block_bytes() % 16) return fail(PA_ERR_UNSUPPORTED, "pa_copy_blocks: block bytes not a multiple of 16");
    if (pool->cfg.num_layers > 65535) return fail(PA_ERR_UNSUPPORTED, "pa_copy_blocks: too many layers");
    CopyParams p;
    p.k_pool = static_cast<unsigned char *>(pool->k_pool);
    p.v_pool = static_cast<unsigned char *>(pool->v_pool);
    p.scales = static_cast<unsigned char *>(pool->scales);
    p.pairs = pairs_dev;
    p.block_chunks = (int64_t)(pool->block_bytes() / 16);
    p.layer_chunks = (int64_t)(pool->layer_bytes() / 16);
    p.scale_block_chunks = (int64_t)(pool->scale_block_bytes() / 16);
    p.scale_layer_chunks = (int64_t)(pool->scale_layer_bytes() / 16);
    p.num_blocks = pool->cfg.num_blocks;
    copy_blocks_kernel<<<dim3(n_pairs, pool->cfg.num_layers, 2), 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    pa_internal::launch_count.fetch_add(1);
    return check_launch("copy_blocks_kernel");
}

pa_status pa_decode_attention_static(pa_pool *pool, int32_t layer, const void *q, void *out, pa_dtype out_dtype,
                                     const int32_t *block_tables_dev, int32_t max_blocks, const int32_t *seq_lens_dev,
                                     int32_t n_seqs, int32_t num_q_heads, float scale, int32_t split_tokens,
                                     pa_stream stream) {
    pa_internal::TraceRange trace_("pa_decode_attention_static");
    if (!pool) return fail(PA_ERR_INVALID_ARG, "pa_decode_attention_static: null pool");
    if (n_seqs < 0 || max_blocks < 1 || split_tokens < 0)
        return fail(PA_ERR_INVALID_ARG, "pa_decode_attention_static: bad n_seqs, max_blocks or split_tokens");
    const int32_t max_splits = pa_decode_max_splits(pool->cfg.block_size, max_blocks, split_tokens);
    if (max_splits < 1)
        return fail(PA_ERR_INVALID_ARG, "pa_decode_attention_static: split_tokens must be 0 or a multiple of block_size");
    const size_t need = pa_decode_workspace_bytes(n_seqs, num_q_heads, pool->cfg.head_dim, max_splits);
    if (need > (size_t)PA_STATIC_WORKSPACE_BYTES)
        return fail(PA_ERR_INVALID_ARG,
                    "pa_decode_attention_static: this batch needs " + std::to_string(need) +
                        " bytes of split scratch but the built-in array holds " +
                        std::to_string((size_t)PA_STATIC_WORKSPACE_BYTES) +
                        "; use a larger split_tokens (or 0), a smaller batch, or pa_decode_attention with a "
                        "caller-owned workspace");
    void *ws = nullptr;
    if (need > 0) {
        pa_status st = static_scratch_address(&ws);
        if (st != PA_OK) return st;
    }
    return pa_decode_attention(pool, layer, q, out, out_dtype, block_tables_dev, max_blocks, seq_lens_dev, n_seqs,
                               num_q_heads, scale, split_tokens, ws, need > 0 ? (size_t)PA_STATIC_WORKSPACE_BYTES : 0,
                               stream);
}

pa_status pa_debug_wait_test(int64_t wait_limit_ns, int32_t withhold_cta) {
    if (withhold_cta < -1) return fail(PA_ERR_INVALID_ARG, "pa_debug_wait_test: withhold_cta must be >= -1");
    const uint64_t limit = wait_limit_ns > 0 ? (uint64_t)wait_limit_ns : kWaitLimitNs;
    cudaError_t e = cudaDeviceSynchronize();   // no launch in flight sees a half-changed setting
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_wait_limit_ns, &limit, sizeof limit);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, std::string("pa_debug_wait_test: ") + cudaGetErrorString(e));
    g_debug_withhold.store(withhold_cta, std::memory_order_relaxed);
    return PA_OK;
}

pa_status pa_device_error(int32_t *code, int32_t clear) {
    if (!code) return fail(PA_ERR_INVALID_ARG, "pa_device_error: null code");
    unsigned v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof v);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, std::string("pa_device_error: ") + cudaGetErrorString(e));
    *code = (int32_t)v;
    if (clear) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero);
        if (e != cudaSuccess) return fail(PA_ERR_CUDA, std::string("pa_device_error: ") + cudaGetErrorString(e));
    }
    return PA_OK;
}

}  // extern "C"

namespace pa_internal {

pa_status swap_copy(const pa_pool *pool, const int32_t *blocks, int32_t n, void *host_buf, bool to_host,
                    void *stream) {
    if (n == 0) return PA_OK;
    cudaPointerAttributes attr;
    cudaError_t e = cudaPointerGetAttributes(&attr, host_buf);
    if (e != cudaSuccess || attr.type != cudaMemoryTypeHost || !attr.devicePointer) {
        cudaGetLastError();
        return fail(PA_ERR_INVALID_ARG, "swap: the host buffer must be page-locked host memory the GPU can reach");
    }
    if (((uintptr_t)attr.devicePointer & 15) || pool->block_bytes() % 16)
        return fail(PA_ERR_INVALID_ARG, "swap: host buffer must be 16-byte aligned");
    if (!pool->device_ready()) return fail(PA_ERR_INVALID_ARG, "swap: the FP8 pool has no scale arrays");
    if (pool->cfg.num_layers > 65535) return fail(PA_ERR_UNSUPPORTED, "swap: too many layers");
    SwapParams p;
    p.k_pool = static_cast<unsigned char *>(pool->k_pool);
    p.v_pool = static_cast<unsigned char *>(pool->v_pool);
    p.scales = static_cast<unsigned char *>(pool->scales);
    p.host = static_cast<unsigned char *>(attr.devicePointer);
    p.block_chunks = (int64_t)(pool->block_bytes() / 16);
    p.layer_chunks = (int64_t)(pool->layer_bytes() / 16);
    p.scale_block_chunks = (int64_t)(pool->scale_block_bytes() / 16);
    p.scale_layer_chunks = (int64_t)(pool->scale_layer_bytes() / 16);
    p.record_chunks = (int64_t)(pool->swap_record_bytes() / 16);
    p.num_blocks = pool->cfg.num_blocks;
    p.to_host = to_host ? 1 : 0;
    for (int32_t first = 0; first < n; first += kSwapChunk) {
        p.first = first;
        p.count = n - first < kSwapChunk ? n - first : kSwapChunk;
        for (int32_t j = 0; j < p.count; ++j) p.blocks[j] = blocks[first + j];
        swap_copy_kernel<<<dim3(p.count, pool->cfg.num_layers, 2), 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
        launch_count.fetch_add(1);
        pa_status st = check_launch("swap_copy_kernel");
        if (st != PA_OK) return st;
    }
    return PA_OK;
}

}  // namespace pa_internal
