// ExpertsInt8 weight quantization (Jamba-1.5 paper, §3.1 "ExpertsInt8": MoE weights are quantized
// to INT8 at model loading, in seconds, without calibration).
//
// One warp per output row: pass 1 finds amax with 16-byte loads, the scale is amax / 127 in IEEE
// fp32 (a row of zeros gets scale 1), pass 2 re-reads the row (now in L2) and writes 16 int8
// codes per lane per step.  HBM-bound: 2 bytes read + 1 byte written per weight (+ the second
// read, served by L2).
//
// Rounding without a division per element: n0 = rint(w * (1/s)) is within one of the nearest
// integer to the exact quotient w / s (the product is off by at most ~3e-5 for |w/s| <= 127.5).
// The residual d = w - n0 * s comes from one fp32 fma.  Whenever |w| >= s/2, w is a multiple of
// ulp(s) (a bf16 has 8 significant bits, s has 24), so d is a multiple of ulp(s) with |d| < s
// and the fma is exact; when |w| < s/2, n0 is 0 (d = w, exact) unless w sits within rounding
// distance of s/2, which again needs |w| >= s/2 - tiny and hence the exact case.  Comparing
// 2|d| with s therefore decides exactly whether to step to n0 +- 1, and exact ties go to the
// even integer.  Scales below 1e-30 (1/s would overflow) take an fp64 division instead.
#include "common.cuh"

namespace jmoe {

__device__ __forceinline__ int quantize_one(float w, float s, float inv_s, bool tiny) {
    if (tiny) {
        // scale so small that 1/s overflows fp32: take the quotient in fp64 (exact tie decisions too)
        double r = rint(__ddiv_rn((double)w, (double)s));
        return (int)fmin(fmax(r, -127.0), 127.0);
    }
    float n0 = rintf(w * inv_s);
    const float d = fmaf(-n0, s, w);
    const float twice = 2.0f * fabsf(d);
    if (twice > s) {
        n0 += (d > 0.0f) ? 1.0f : -1.0f;
    } else if (twice == s) {
        // exact tie between n0 and n0 + sign(d): take the even one
        const float other = n0 + ((d > 0.0f) ? 1.0f : -1.0f);
        if (fmodf(n0, 2.0f) != 0.0f) n0 = other;
    }
    n0 = fminf(fmaxf(n0, -127.0f), 127.0f);
    return (int)n0;
}

__global__ void __launch_bounds__(256) quantize_rows_kernel(const uint16_t* __restrict__ W, int64_t rows,
                                                            int64_t cols, int8_t* __restrict__ Q,
                                                            float* __restrict__ S) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t chunks = cols / 16;  // 16 weights = 32 bytes in, 16 bytes out
    for (int64_t r = warp; r < rows; r += nwarps) {
        const uint16_t* wr = W + r * cols;
        uint32_t amax_bits = 0;  // max of |w| as an IEEE bit pattern (monotone for non-negative floats)
#pragma unroll 4
        for (int64_t c = lane; c < chunks; c += 32) {
            const uint4 a = ld_nc_v4(wr + c * 16);
            const uint4 b = ld_nc_v4(wr + c * 16 + 8);
            const uint32_t v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                amax_bits = max(amax_bits, (v[i] & 0x7FFFu) << 16);
                amax_bits = max(amax_bits, v[i] & 0x7FFF0000u);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax_bits = max(amax_bits, __shfl_xor_sync(0xffffffffu, amax_bits, o));
        const float amax = __uint_as_float(amax_bits);
        const float s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 127.0f);
        const float inv_s = __frcp_rn(s);
        const bool tiny = s < 1.0e-30f;
        if (lane == 0) S[r] = s;
        int8_t* qr = Q + r * cols;
        for (int64_t c = lane; c < chunks; c += 32) {
            const uint4 a = ld_nc_v4(wr + c * 16);
            const uint4 b = ld_nc_v4(wr + c * 16 + 8);
            const uint32_t v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            uint32_t out[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int q0 = quantize_one(bf16_bits_to_f32(v[2 * i] & 0xFFFFu), s, inv_s, tiny);
                const int q1 = quantize_one(bf16_bits_to_f32(v[2 * i] >> 16), s, inv_s, tiny);
                const int q2 = quantize_one(bf16_bits_to_f32(v[2 * i + 1] & 0xFFFFu), s, inv_s, tiny);
                const int q3 = quantize_one(bf16_bits_to_f32(v[2 * i + 1] >> 16), s, inv_s, tiny);
                out[i] = (uint32_t)(q0 & 0xFF) | ((uint32_t)(q1 & 0xFF) << 8) | ((uint32_t)(q2 & 0xFF) << 16) |
                         ((uint32_t)(q3 & 0xFF) << 24);
            }
            *reinterpret_cast<uint4*>(qr + c * 16) = make_uint4(out[0], out[1], out[2], out[3]);
        }
    }
}

cudaError_t launch_quantize(const uint16_t* W, int64_t rows, int64_t cols, int8_t* Q, float* S, cudaStream_t st,
                            int num_sms) {
    const int threads = 256;
    int64_t blocks = (rows + 7) / 8;
    const int64_t cap = (int64_t)num_sms * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    quantize_rows_kernel<<<(unsigned)blocks, threads, 0, st>>>(W, rows, cols, Q, S);
    return cudaGetLastError();
}

}  // namespace jmoe
