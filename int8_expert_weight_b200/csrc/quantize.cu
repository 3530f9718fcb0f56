// ExpertsInt8 weight quantization (Jamba-1.5 paper, §3.1 "ExpertsInt8": MoE weights are quantized
// to INT8 at model loading, in seconds, without calibration).
//
// HBM-bound: 2 bytes read + 1 byte written per weight.  A row of up to 32768 weights takes 32, 64,
// 128 or 256 threads (the fewest that hold it in 16 chunks of 8 weights each): the row is read once
// with 16-byte loads into registers, amax is reduced across the row, the scale is amax / 127 in IEEE
// fp32 (a row of zeros gets scale 1), and the codes are computed from the registers and written 8
// per store.  Longer rows take one warp per row and two passes (the second read is served by L2).
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

// Codes of 8 weights (one 16-byte chunk) as two words, byte i = code of weight i, by the exact
// rule of quantize_one; out of line, for the rare chunks the fast rounding cannot decide.
__device__ __noinline__ uint2 quantize_chunk_exact(const uint4 v, float s, float inv_s, bool tiny) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t q0 = (uint32_t)quantize_one(__uint_as_float(w[i] << 16), s, inv_s, tiny) & 0xFFu;
        const uint32_t q1 = (uint32_t)quantize_one(__uint_as_float(w[i] & 0xFFFF0000u), s, inv_s, tiny) & 0xFFu;
        out[i >> 1] |= (q0 | (q1 << 8)) << (16 * (i & 1));
    }
    return make_uint2(out[0], out[1]);
}

// The same codes on the fast path.  m = fma(w, 1/s, 1.5 * 2^23) rounds w/s (to within the error
// of 1/s) to an integer n held in the low mantissa bits of m, two's complement, so the code is
// byte 0 of m.  n is the nearest integer to w/s whenever the exact residual |w - n*s| (one fma, exact
// where it matters, see above) is below s/2; a chunk with any other weight takes the exact rule.
__device__ __forceinline__ uint2 quantize_chunk(const uint4 v, float s, float inv_s, float half_s, bool tiny) {
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t m[8];
    bool ok = !tiny;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float a0 = __uint_as_float(w[i] << 16), a1 = __uint_as_float(w[i] & 0xFFFF0000u);
        const float m0 = fmaf(a0, inv_s, kMagic), m1 = fmaf(a1, inv_s, kMagic);
        ok &= fabsf(fmaf(-(m0 - kMagic), s, a0)) < half_s;
        ok &= fabsf(fmaf(-(m1 - kMagic), s, a1)) < half_s;
        m[2 * i] = __float_as_uint(m0);
        m[2 * i + 1] = __float_as_uint(m1);
    }
    if (!ok) return quantize_chunk_exact(v, s, inv_s, tiny);
    const uint32_t lo = __byte_perm(__byte_perm(m[0], m[1], 0x0040), __byte_perm(m[2], m[3], 0x0040), 0x5410);
    const uint32_t hi = __byte_perm(__byte_perm(m[4], m[5], 0x0040), __byte_perm(m[6], m[7], 0x0040), 0x5410);
    return make_uint2(lo, hi);
}

constexpr int kQChunks = 16;  // 8-weight chunks a thread holds in registers

// kRowThreads threads per row (a multiple of 32 up to 256); 256 / kRowThreads rows per CTA step.
template <int kRowThreads>
__global__ void __launch_bounds__(256, 2) quantize_rows_reg_kernel(const uint16_t* __restrict__ W, int64_t rows,
                                                                   int64_t cols, int8_t* __restrict__ Q,
                                                                   float* __restrict__ S) {
    constexpr int kRowsPerCta = 256 / kRowThreads;
    constexpr int kWarpsPerRow = kRowThreads / 32;
    __shared__ uint32_t part[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t = tid % kRowThreads;
    const int64_t chunks = cols / 8;
    for (int64_t r0 = (int64_t)blockIdx.x * kRowsPerCta; r0 < rows; r0 += (int64_t)gridDim.x * kRowsPerCta) {
        const int64_t r = r0 + tid / kRowThreads;
        const bool live = r < rows;
        const uint16_t* wr = W + (live ? r : 0) * cols;
        uint4 v[kQChunks];
#pragma unroll
        for (int i = 0; i < kQChunks; ++i) {
            const int64_t c = t + (int64_t)i * kRowThreads;
            v[i] = (live && c < chunks) ? ld_stream_v4(wr + c * 8) : make_uint4(0, 0, 0, 0);
        }
        uint32_t m2 = 0;  // two 16-bit maxima of |w| bit patterns (monotone for non-negative values)
#pragma unroll
        for (int i = 0; i < kQChunks; ++i) {
            m2 = __vmaxu2(m2, v[i].x & 0x7FFF7FFFu);
            m2 = __vmaxu2(m2, v[i].y & 0x7FFF7FFFu);
            m2 = __vmaxu2(m2, v[i].z & 0x7FFF7FFFu);
            m2 = __vmaxu2(m2, v[i].w & 0x7FFF7FFFu);
        }
        uint32_t amax_bits = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax_bits = max(amax_bits, __shfl_xor_sync(0xffffffffu, amax_bits, o));
        if (kWarpsPerRow > 1) {  // across the warps of the row (every thread takes part: no early exit above)
            if (lane == 0) part[warp] = amax_bits;
            __syncthreads();
            const int w0 = (warp / kWarpsPerRow) * kWarpsPerRow;
#pragma unroll
            for (int w = 0; w < kWarpsPerRow; ++w) amax_bits = max(amax_bits, part[w0 + w]);
            __syncthreads();  // part is rewritten by the next row
        }
        const float amax = __uint_as_float(amax_bits << 16);
        const float s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 127.0f);
        const float inv_s = __frcp_rn(s);
        const bool tiny = s < 1.0e-30f;
        if (!live) continue;
        if (t == 0) S[r] = s;
        int8_t* qr = Q + r * cols;
#pragma unroll
        for (int i = 0; i < kQChunks; ++i) {
            const int64_t c = t + (int64_t)i * kRowThreads;
            if (c < chunks) *reinterpret_cast<uint2*>(qr + c * 8) = quantize_chunk(v[i], s, inv_s, 0.5f * s, tiny);
        }
    }
}

template <int kRowThreads>
static void launch_reg(const uint16_t* W, int64_t rows, int64_t cols, int8_t* Q, float* S, cudaStream_t st,
                       int64_t cap) {
    constexpr int kRowsPerCta = 256 / kRowThreads;
    int64_t blocks = (rows + kRowsPerCta - 1) / kRowsPerCta;
    blocks = blocks > cap ? cap : (blocks < 1 ? 1 : blocks);
    quantize_rows_reg_kernel<kRowThreads><<<(unsigned)blocks, 256, 0, st>>>(W, rows, cols, Q, S);
}

cudaError_t launch_quantize(const uint16_t* W, int64_t rows, int64_t cols, int8_t* Q, float* S, cudaStream_t st,
                            int num_sms) {
    const int64_t cap = (int64_t)num_sms * 8;
    const int64_t per_thread = kQChunks * 8;  // weights a thread holds
    if (cols <= 32 * per_thread) {
        launch_reg<32>(W, rows, cols, Q, S, st, cap);
    } else if (cols <= 64 * per_thread) {
        launch_reg<64>(W, rows, cols, Q, S, st, cap);
    } else if (cols <= 128 * per_thread) {
        launch_reg<128>(W, rows, cols, Q, S, st, cap);
    } else if (cols <= 256 * per_thread) {
        launch_reg<256>(W, rows, cols, Q, S, st, cap);
    } else {
        int64_t blocks = (rows + 7) / 8;
        blocks = blocks > cap ? cap : (blocks < 1 ? 1 : blocks);
        quantize_rows_kernel<<<(unsigned)blocks, 256, 0, st>>>(W, rows, cols, Q, S);
    }
    return cudaGetLastError();
}

}  // namespace jmoe
