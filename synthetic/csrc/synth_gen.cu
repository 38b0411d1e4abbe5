// Device-side counter-based synthetic values (input generation, not part of the
// paged decode path).  Second implementation, written separately, of the
// generator described in synthetic/values.py: element value =
// narrow(fp32(centred sum of the four 16-bit fields of SplitMix64 output
// number c of the stream seeded `seed`) * unit), with counter
// c = kind<<62 | uid<<40 | layer<<34 | token<<14 | head<<8 | dim.
// SplitMix64: Steele, Lea & Flood, "Fast splittable pseudorandom number
// generators" (OOPSLA 2014).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint64_t splitmix_output(uint64_t seed, uint64_t index) {
    uint64_t z = seed + (index + 1ull) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__device__ __forceinline__ float value_f32(uint64_t seed, uint64_t ctr, float unit) {
    const uint64_t z = splitmix_output(seed, ctr);
    const int32_t s = (int32_t)(z & 0xFFFF) + (int32_t)((z >> 16) & 0xFFFF) + (int32_t)((z >> 32) & 0xFFFF) +
                      (int32_t)((z >> 48) & 0xFFFF) - 131070;
    return __fmul_rn((float)s, unit);
}

// out[i][h][d] for rows (uids[i], tokens[i]); dtype 0 = fp32, 1 = fp16, 2 = bf16.
__global__ void fill_rows_kernel(void *out, int dtype, int kind, uint64_t seed, int layer, const int32_t *uids,
                                 const int32_t *tokens, int64_t n_rows, int heads, int dim, float unit) {
    const int64_t per_row = (int64_t)heads * dim;
    const int64_t total = n_rows * per_row;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = idx / per_row;
        const int h = (int)((idx % per_row) / dim);
        const int d = (int)(idx % dim);
        const uint64_t ctr = ((uint64_t)kind << 62) | ((uint64_t)uids[i] << 40) | ((uint64_t)layer << 34) |
                             ((uint64_t)tokens[i] << 14) | ((uint64_t)h << 8) | (uint64_t)d;
        const float v = value_f32(seed, ctr, unit);
        if (dtype == 0)
            static_cast<float *>(out)[idx] = v;
        else if (dtype == 1)
            static_cast<__half *>(out)[idx] = __float2half_rn(v);
        else
            static_cast<__nv_bfloat16 *>(out)[idx] = __float2bfloat16_rn(v);
    }
}

}  // namespace

extern "C" int synth_fill_rows(void *out, int dtype, int kind, uint64_t seed, int layer, const int32_t *uids,
                               const int32_t *tokens, int64_t n_rows, int heads, int dim, float unit,
                               void *stream) {
    if (n_rows <= 0) return 0;
    const int64_t total = n_rows * heads * dim;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 148 * 64) blocks = 148 * 64;
    fill_rows_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        out, dtype, kind, seed, layer, uids, tokens, n_rows, heads, dim, unit);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}
