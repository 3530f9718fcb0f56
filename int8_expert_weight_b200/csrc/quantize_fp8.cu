// FP8 (E4M3) quantization for the FP8 comparator layer (Jamba-1.5 paper, §3.1 compares ExpertsInt8
// with FP8 serving).  Per row: amax, scale = amax / 448 in IEEE fp32 (a row of zeros gets scale 1
// and code 0), code = the E4M3 number nearest to the exact quotient v / scale, ties to the even
// code, saturating at +-448 (E4M3: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no
// infinities, subnormals m * 2^-9).  Used for the weights (per output channel, load time), for the
// activations x (per token) and for the SwiGLU intermediate h (per permuted row); all bf16 rows.
//
// Fast path: the hardware conversion of the fp32 product v * (1/scale), whenever that product is
// provably on the same side of every E4M3 rounding boundary as the exact quotient (see e4m3_safe).
// Near a boundary (a tie, a near tie, the E4M3 subnormal range) that code is at most one step off
// and an exact fp32 residual settles it (e4m3_fix); scales below 2^-100 take the fp64 quotient,
// rounded to the E4M3 grid by power-of-two scaling and rint.
#include "common.cuh"

namespace jmoe {

// Value of an E4M3 code (not the NaN codes): its exponent and mantissa bits placed in an fp32 at
// bits 20..26 denote 2^(e-127) (1 + m/8) (or m 2^-129 for e = 0); times 2^120 that is the E4M3
// value, exactly.
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
    const float mag = __uint_as_float((code & 0x7Fu) << 20) * 0x1p120f;
    return (code & 0x80u) ? -mag : mag;
}

// Two codes from two floats by the hardware conversion (nearest even, saturating): a -> byte 0.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float a, float b) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
    return r;
}

// Exact E4M3 rounding of v / s (s > 0, finite): the fp64 quotient, its binade, and rint.
__device__ __noinline__ uint32_t e4m3_exact(float v, float s) {
    const double q = __ddiv_rn((double)v, (double)s);
    const uint32_t sign = signbit(q) ? 0x80u : 0u;
    const double a = fabs(q);
    if (a >= 448.0) return sign | 0x7Eu;
    if (a == 0.0) return sign;
    int eb = ilogb(a);
    if (eb < -6) eb = -6;
    double n = rint(scalbn(a, 3 - eb));
    if (n >= 16.0) {
        eb += 1;
        n = 8.0;
    }
    if (eb == -6 && n < 8.0) return sign | (uint32_t)n;
    return sign | (uint32_t)(((eb + 7) << 3) | ((int)n - 8));
}

// t = v * (1/s) in fp32 is within 2 ulps of the exact quotient q = v / s (two roundings of 2^-24
// relative each).  E4M3 keeps 3 fraction bits, so in the normal E4M3 range [2^-6, 448) the rounding
// boundaries of a binade are where the 20 fraction bits below those 3 read 0x80000; if t's bits are
// more than 3 ulps away from that pattern, no boundary lies between t and q and the hardware rounding
// of t is the rounding of q.  |t| >= 448 saturates either way; zero is exact; the E4M3 subnormal
// range and everything else near a boundary go to the exact path.
__device__ __forceinline__ bool e4m3_safe(float t) {
    const uint32_t a = __float_as_uint(t) & 0x7FFFFFFFu;
    if (a >= 0x43E00000u) return true;   // |t| >= 448
    if (a < 0x3C800000u) return a == 0;  // |t| < 2^-6
    const int32_t dist = (int32_t)(a & 0xFFFFFu) - 0x80000;
    return dist > 3 || dist < -3;
}

// The correctly rounded code of v / s, given a code c at most one step away from it (v a bf16
// value, s >= 2^-100).  The residual d = |v| - |c| s is exact as one fp32 fma: |c| has 4
// significant bits and s 24, so |c| s and |v| (8 bits) are multiples of a common quantum q, and
// |d| < (grid step) * s gives |d| / q < 2^24; half a grid step times s is exact too.  d against
// half the step on its side decides between c and that neighbour; equality is a tie, to the even
// code.
__device__ __noinline__ uint32_t e4m3_fix(float v, float s, uint32_t c) {
    const uint32_t sign = c & 0x80u, mc = c & 0x7Fu;
    const float d = fmaf(-e4m3_to_f32(mc), s, fabsf(v));
    const uint32_t E = mc >> 3;
    const float half_above = __uint_as_float((127u + (E > 0 ? E : 1u) - 11u) << 23);  // 2^(max(E,1) - 11)
    const float half_below = ((mc & 7u) == 0 && E >= 2) ? 0.5f * half_above : half_above;
    uint32_t r = mc;
    if (d > 0.0f && mc != 0x7Eu) {  // above c (at 448: saturated)
        const float thr = half_above * s;
        if (d > thr || (d == thr && (mc & 1u))) r = mc + 1;
    } else if (d < 0.0f) {
        const float thr = half_below * s;
        if (-d > thr || (-d == thr && (mc & 1u))) r = mc - 1;
    }
    return sign | r;
}

// Codes of 8 values (one chunk) as two words, byte i = code of value i.
__device__ __forceinline__ uint2 fp8_chunk(const float (&v)[8], float s, float inv_s) {
    uint32_t w[4];
    if (s < 0x1p-100f) {  // scales this small: the exact quotient for every value
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] = e4m3_exact(v[2 * i], s) | (e4m3_exact(v[2 * i + 1], s) << 8);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float t0 = v[2 * i] * inv_s, t1 = v[2 * i + 1] * inv_s;
            w[i] = cvt_e4m3x2(t0, t1);
            const bool ok0 = e4m3_safe(t0), ok1 = e4m3_safe(t1);
            if (!(ok0 && ok1)) {  // near a rounding boundary: settle it with the exact residual
                const uint32_t c0 = ok0 ? (w[i] & 0xFFu) : e4m3_fix(v[2 * i], s, w[i] & 0xFFu);
                const uint32_t c1 = ok1 ? (w[i] >> 8) : e4m3_fix(v[2 * i + 1], s, w[i] >> 8);
                w[i] = c0 | (c1 << 8);
            }
        }
    }
    return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

// bf16 rows; one row per kRowThreads threads, up to kChunks chunks of 8 values per thread held in
// registers (as loaded) between the amax reduction and the conversion.  With a permutation, rows
// whose entry is -1 (padding) are skipped and only rows below *n_live are taken.
template <int kRowThreads, int kChunks>
__global__ void __launch_bounds__(256) quantize_fp8_rows_kernel(const uint16_t* __restrict__ W, int64_t rows,
                                                                int64_t cols, uint8_t* __restrict__ Q,
                                                                float* __restrict__ S,
                                                                const int32_t* __restrict__ live_rows,
                                                                const int32_t* __restrict__ n_live) {
    constexpr int kRowsPerCta = 256 / kRowThreads;
    constexpr int kWarpsPerRow = kRowThreads / 32;
    __shared__ float part[8];
    pdl_wait();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t = tid % kRowThreads;
    const int64_t chunks = cols / 8;
    if (n_live) rows = min(rows, (int64_t)*n_live);  // rows past the last expert segment hold nothing
    for (int64_t r0 = (int64_t)blockIdx.x * kRowsPerCta; r0 < rows; r0 += (int64_t)gridDim.x * kRowsPerCta) {
        const int64_t r = r0 + tid / kRowThreads;
        const bool live = r < rows && (!live_rows || live_rows[r] >= 0);
        uint4 raw[kChunks];
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < kChunks; ++i) {
            const int64_t c = t + (int64_t)i * kRowThreads;
            raw[i] = (live && c < chunks) ? ld_stream_v4(W + r * cols + c * 8) : make_uint4(0, 0, 0, 0);
            const uint32_t m2 = __vmaxu2(__vmaxu2(raw[i].x & 0x7FFF7FFFu, raw[i].y & 0x7FFF7FFFu),
                                         __vmaxu2(raw[i].z & 0x7FFF7FFFu, raw[i].w & 0x7FFF7FFFu));
            amax = fmaxf(amax, __uint_as_float(max(m2 & 0xFFFFu, m2 >> 16) << 16));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (kWarpsPerRow > 1) {
            if (lane == 0) part[warp] = amax;
            __syncthreads();
            const int w0 = (warp / kWarpsPerRow) * kWarpsPerRow;
#pragma unroll
            for (int w = 0; w < kWarpsPerRow; ++w) amax = fmaxf(amax, part[w0 + w]);
            __syncthreads();
        }
        const float s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
        const float inv_s = __frcp_rn(s);
        if (!live) continue;
        if (t == 0) S[r] = s;
        uint8_t* qr = Q + r * cols;
#pragma unroll
        for (int i = 0; i < kChunks; ++i) {
            const int64_t c = t + (int64_t)i * kRowThreads;
            if (c < chunks) {
                const uint32_t u[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
                float v[8];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    v[2 * k] = __uint_as_float(u[k] << 16);
                    v[2 * k + 1] = __uint_as_float(u[k] & 0xFFFF0000u);
                }
                *reinterpret_cast<uint2*>(qr + c * 8) = (amax == 0.0f) ? make_uint2(0u, 0u) : fp8_chunk(v, s, inv_s);
            }
        }
    }
    pdl_trigger();
}

// Rows longer than the register-resident kernels hold: one warp per row, amax pass + code pass.
__global__ void __launch_bounds__(256) quantize_fp8_long_kernel(const uint16_t* __restrict__ W, int64_t rows,
                                                                int64_t cols, uint8_t* __restrict__ Q,
                                                                float* __restrict__ S,
                                                                const int32_t* __restrict__ live_rows,
                                                                const int32_t* __restrict__ n_live) {
    pdl_wait();
    if (n_live) rows = min(rows, (int64_t)*n_live);
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5), nwarps = (int64_t)gridDim.x * 8;
    for (int64_t r = warp; r < rows; r += nwarps) {
        if (live_rows && live_rows[r] < 0) continue;
        const uint16_t* wr = W + r * cols;
        float amax = 0.0f;
        for (int64_t i = lane; i < cols; i += 32) amax = fmaxf(amax, fabsf(__uint_as_float((uint32_t)wr[i] << 16)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
        const float inv_s = __frcp_rn(s);
        if (lane == 0) S[r] = s;
        for (int64_t c = lane; c < cols / 8; c += 32) {
            float v[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = __uint_as_float((uint32_t)wr[c * 8 + k] << 16);
            *reinterpret_cast<uint2*>(Q + r * cols + c * 8) =
                (amax == 0.0f) ? make_uint2(0u, 0u) : fp8_chunk(v, s, inv_s);
        }
    }
    pdl_trigger();
}

template <int kRowThreads, int kChunks>
static cudaError_t launch_fp8_reg(const uint16_t* W, int64_t rows, int64_t cols, uint8_t* Q, float* S,
                                  const int32_t* live, const int32_t* n_live, cudaStream_t st, int64_t cap) {
    constexpr int kRowsPerCta = 256 / kRowThreads;
    int64_t blocks = (rows + kRowsPerCta - 1) / kRowsPerCta;
    blocks = blocks > cap ? cap : (blocks < 1 ? 1 : blocks);
    return launch_pdl(quantize_fp8_rows_kernel<kRowThreads, kChunks>, dim3((unsigned)blocks), dim3(256), 0, st, W,
                      rows, cols, Q, S, live, n_live);
}

// bf16 rows [rows][cols] (cols % 8 == 0) -> E4M3 codes and per-row scales.  perm / n_live (both may
// be null): skip rows whose permutation entry is -1 and rows from *n_live on.  Few rows (activations
// of a decode step) take a whole CTA each; many rows the fewest threads that hold a row.
cudaError_t launch_quantize_fp8(const uint16_t* W, int64_t rows, int64_t cols, uint8_t* Q, float* S,
                                const int32_t* perm, const int32_t* n_live, cudaStream_t st, int num_sms) {
    const int64_t cap = (int64_t)num_sms * 8;
    constexpr int kC = 16;
    const bool few = rows <= (int64_t)num_sms * 16;
    if (cols <= 32 * kC * 8 && !few) return launch_fp8_reg<32, kC>(W, rows, cols, Q, S, perm, n_live, st, cap);
    if (cols <= 64 * kC * 8 && !few) return launch_fp8_reg<64, kC>(W, rows, cols, Q, S, perm, n_live, st, cap);
    if (cols <= 128 * kC * 8 && !few) return launch_fp8_reg<128, kC>(W, rows, cols, Q, S, perm, n_live, st, cap);
    if (cols <= 256 * 4 * 8) return launch_fp8_reg<256, 4>(W, rows, cols, Q, S, perm, n_live, st, cap);
    if (cols <= 256 * kC * 8) return launch_fp8_reg<256, kC>(W, rows, cols, Q, S, perm, n_live, st, cap);
    int64_t blocks = (rows + 7) / 8;
    blocks = blocks > cap ? cap : (blocks < 1 ? 1 : blocks);
    return launch_pdl(quantize_fp8_long_kernel, dim3((unsigned)blocks), dim3(256), 0, st, W, rows, cols, Q, S, perm,
                      n_live);
}

}  // namespace jmoe
