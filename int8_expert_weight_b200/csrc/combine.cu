// Weighted combine of a token's two expert outputs: y_t = bf16(out[t][0] + out[t][1]).
// The routing weights were already applied by the down-projection epilogue; the two fp32
// slots are added in a fixed order (slot 0 then slot 1) and rounded once, so y is deterministic.
// HBM-bound: 8 bytes read and 2 bytes written per output.
#include "common.cuh"

namespace jmoe {

__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ slots, int64_t T, int64_t d,
                                                      uint16_t* __restrict__ y) {
    pdl_wait();
    pdl_trigger();
    const int64_t quads = T * d / 4;  // d % 4 == 0
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < quads; q += stride) {
        const int64_t t = (q * 4) / d, i = (q * 4) % d;
        const float4 a = __ldcs(reinterpret_cast<const float4*>(slots + (t * kTopK + 0) * d + i));
        const float4 b = __ldcs(reinterpret_cast<const float4*>(slots + (t * kTopK + 1) * d + i));
        const uint32_t lo = (uint32_t)f32_to_bf16_bits(a.x + b.x) | ((uint32_t)f32_to_bf16_bits(a.y + b.y) << 16);
        const uint32_t hi = (uint32_t)f32_to_bf16_bits(a.z + b.z) | ((uint32_t)f32_to_bf16_bits(a.w + b.w) << 16);
        *reinterpret_cast<uint2*>(y + t * d + i) = make_uint2(lo, hi);
    }
}

cudaError_t launch_combine(const float* slots, int64_t T, int64_t d, uint16_t* y, cudaStream_t st, int num_sms) {
    int64_t blocks = (T * d / 4 + 255) / 256;
    if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
    if (blocks < 1) blocks = 1;
    return launch_pdl(combine_kernel, dim3((unsigned)blocks), dim3(256), 0, st, slots, T, d, y);
}

}  // namespace jmoe
