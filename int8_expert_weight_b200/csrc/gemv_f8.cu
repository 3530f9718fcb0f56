// Decode path of the FP8 (E4M3) comparator layer: weights and activations are both E4M3 codes, so
// the tensor cores take them as they are loaded (mma.sync m16n8k32 with e4m3 operands, fp32
// accumulation) and no conversion is needed; the row scales of the weights and the per-row scales
// of the activations are applied to the fp32 totals.
//
//   gemv13: h[r][j] = bf16( SiLU(S1[j] sx_t (x8_t . Q1[j])) * (S3[j] sx_t (x8_t . Q3[j])) )   (t = token of r)
//   gemv2:  out[a][i] = p_a * S2[i] * sh_r * (h8_r . Q2[i])                          (a = assignment of r)
//
// CTA = (one touched expert, 16 weight rows), 8 warps splitting K into interleaved 64-wide steps.
// Per step a lane loads 16 consecutive codes of weight rows g and g+8 and of each token's row
// (16-byte loads) and feeds two m16n8k32 MMAs: a k-permutation applied to both operands leaves the
// dot product unchanged, so the lane's 16 consecutive k fill exactly the fragment slots it owns
// (bytes 0-3 / 4-7 of the first MMA's A and B registers, bytes 8-15 of the second's).  Partial sums
// of the 8 warps are added in a fixed order in shared memory.
#include "common.cuh"

namespace jmoe {

constexpr int kF8Warps = 8;
constexpr int kF8Rows = 16;

struct GemvF8Args {
    const WsHeader* hdr;
    const int32_t* perm;     // [rows] assignment (t*K + k) of each permuted row, -1 = padding
    const uint8_t* act;      // gemv13: x8 [T][d] (row = token); gemv2: h8 [rows][F] (row = permuted row)
    const float* act_scale;  // gemv13: sx [T]; gemv2: sh [rows]
    const uint8_t* qa;       // gemv13: Q1 [E][F][d]; gemv2: Q2 [E][d][F]  (E4M3 codes)
    const uint8_t* qb;       // gemv13: Q3 [E][F][d]
    const float* sa;         // S1 [E][F] / S2 [E][d]
    const float* sb;         // S3 [E][F]
    const float* wts;        // gemv2: routing weight of each assignment
    uint16_t* h_out;         // gemv13: h [rows][F] in bf16
    float* slot_out;         // gemv2: out_slot [T*K][d]
    int64_t K, N;
};

__device__ __forceinline__ void mma_e4m3_16832(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The two MMAs of one 64-wide step: w0, w1 = 16 codes of rows g and g+8, x = 16 codes of a token.
__device__ __forceinline__ void mma_step_f8(float (&acc)[4], const uint4& w0, const uint4& w1, const uint4& x) {
    mma_e4m3_16832(acc, w0.x, w1.x, w0.y, w1.y, x.x, x.y);
    mma_e4m3_16832(acc, w0.z, w1.z, w0.w, w1.w, x.z, x.w);
}

template <int NT, bool kDual>
__global__ void __launch_bounds__(kF8Warps * 32, (NT == 1) ? ((kDual) ? 3 : 4) : (NT <= 2 ? 2 : 1))
    gemv_f8_kernel(GemvF8Args p) {
    constexpr int kU = 2;  // k-steps a warp loads before consuming them
    __shared__ __align__(16) float red[kF8Warps * 2 * NT * 128];
    pdl_wait();
    const WsHeader* hdr = p.hdr;
    if ((int)blockIdx.y >= hdr->n_touched) return;
    const int e = hdr->touched[blockIdx.y];
    const int m = hdr->counts[e];
    const int64_t row0 = hdr->seg_start[e];
    const int64_t j0 = (int64_t)blockIdx.x * kF8Rows;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int64_t K = p.K;
    const int steps = (int)(K / 64);
    constexpr int kStride = kF8Warps * 64;
    for (int n0 = 0; n0 < m; n0 += 8 * NT) {
        const uint8_t* px[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int n = n0 + nt * 8 + g;
            const int nn = n < m ? n : 0;  // past the count: any valid row, its column is ignored
            const int64_t arow = kDual ? (int64_t)(p.perm[row0 + nn] / kTopK) : row0 + nn;
            px[nt] = p.act + arow * K + 16 * c + warp * 64;
        }
        const uint8_t* pa0 = p.qa + ((int64_t)e * p.N + j0 + g) * K + 16 * c + warp * 64;
        const uint8_t* pa1 = pa0 + 8 * K;
        const uint8_t* pb0 = kDual ? p.qb + ((int64_t)e * p.N + j0 + g) * K + 16 * c + warp * 64 : nullptr;
        const uint8_t* pb1 = kDual ? pb0 + 8 * K : nullptr;
        float acc_a[NT][4], acc_b[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc_a[nt][i] = acc_b[nt][i] = 0.0f;
        for (int s0 = warp; s0 < steps; s0 += kF8Warps * kU) {
            uint4 wa0[kU], wa1[kU], wb0[kU], wb1[kU], xa[kU][NT];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                if (s0 + u * kF8Warps < steps) {
                    wa0[u] = ld_stream_v4(pa0 + u * kStride);
                    wa1[u] = ld_stream_v4(pa1 + u * kStride);
                    if (kDual) {
                        wb0[u] = ld_stream_v4(pb0 + u * kStride);
                        wb1[u] = ld_stream_v4(pb1 + u * kStride);
                    }
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) xa[u][nt] = ld_nc_v4(px[nt] + u * kStride);
                }
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                if (s0 + u * kF8Warps < steps) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        mma_step_f8(acc_a[nt], wa0[u], wa1[u], xa[u][nt]);
                        if (kDual) mma_step_f8(acc_b[nt], wb0[u], wb1[u], xa[u][nt]);
                    }
                }
            }
            pa0 += kU * kStride;
            pa1 += kU * kStride;
            if (kDual) {
                pb0 += kU * kStride;
                pb1 += kU * kStride;
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) px[nt] += kU * kStride;
        }
        // fixed-order cross-warp reduction
        float* mine = red + (size_t)warp * 2 * NT * 128;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            *reinterpret_cast<float4*>(mine + nt * 128 + lane * 4) =
                make_float4(acc_a[nt][0], acc_a[nt][1], acc_a[nt][2], acc_a[nt][3]);
            if (kDual)
                *reinterpret_cast<float4*>(mine + (NT + nt) * 128 + lane * 4) =
                    make_float4(acc_b[nt][0], acc_b[nt][1], acc_b[nt][2], acc_b[nt][3]);
        }
        __syncthreads();
        for (int o = threadIdx.x; o < (kDual ? 2 : 1) * NT * 128; o += blockDim.x) {
            float sum = 0.0f;
#pragma unroll
            for (int w = 0; w < kF8Warps; ++w) sum += red[(size_t)w * 2 * NT * 128 + o];
            red[o] = sum;
        }
        __syncthreads();
        pdl_trigger();
        // epilogue: o = (nt, lane', i) of the C fragment (lane' = 4g' + c'): i = 0,1 -> row g',
        // tokens 2c', 2c'+1; i = 2,3 -> row g'+8, same tokens
        for (int o = threadIdx.x; o < NT * 128; o += blockDim.x) {
            const int nt = o >> 7, l2 = (o >> 2) & 31, i = o & 3;
            const int row = (l2 >> 2) + ((i & 2) ? 8 : 0);
            const int n = n0 + nt * 8 + 2 * (l2 & 3) + (i & 1);
            if (n >= m) continue;
            const int64_t jr = j0 + row;
            const int32_t a = p.perm[row0 + n];
            if (kDual) {
                const float xs = p.act_scale[a / kTopK];
                const float a1 = red[o] * xs * p.sa[(int64_t)e * p.N + jr];
                const float a3 = red[NT * 128 + o] * xs * p.sb[(int64_t)e * p.N + jr];
                p.h_out[(row0 + n) * p.N + jr] = f32_to_bf16_bits(silu(a1) * a3);
            } else {
                const float v = red[o] * p.act_scale[row0 + n] * p.sa[(int64_t)e * p.N + jr];
                p.slot_out[(int64_t)a * p.N + jr] = p.wts[a] * v;
            }
        }
        __syncthreads();  // red is reused by the next pass
    }
}

static int gemv_f8_nt(int64_t T) {
    const int64_t avg = (T * kTopK + kExperts - 1) / kExperts;
    return avg <= 6 ? 1 : (avg <= 12 ? 2 : 4);
}

template <bool kDual>
static cudaError_t launch_gemv_f8_t(const GemvF8Args& p, int64_t T, cudaStream_t st) {
    dim3 grid((unsigned)(p.N / kF8Rows), kExperts);
    const int nt = gemv_f8_nt(T);
    if (nt == 1) return launch_pdl(gemv_f8_kernel<1, kDual>, grid, dim3(kF8Warps * 32), 0, st, p);
    if (nt == 2) return launch_pdl(gemv_f8_kernel<2, kDual>, grid, dim3(kF8Warps * 32), 0, st, p);
    return launch_pdl(gemv_f8_kernel<4, kDual>, grid, dim3(kF8Warps * 32), 0, st, p);
}

cudaError_t launch_gemv13_f8(const WsHeader* hdr, const int32_t* perm, const uint8_t* x8, const float* sx,
                             const uint8_t* Q1, const float* S1, const uint8_t* Q3, const float* S3, uint16_t* h,
                             int64_t T, int64_t d, int64_t F, cudaStream_t st) {
    GemvF8Args p{hdr, perm, x8, sx, Q1, Q3, S1, S3, nullptr, h, nullptr, d, F};
    return launch_gemv_f8_t<true>(p, T, st);
}

cudaError_t launch_gemv2_f8(const WsHeader* hdr, const int32_t* perm, const uint8_t* h8, const float* sh,
                            const uint8_t* Q2, const float* S2, const float* wts, float* out_slot, int64_t T,
                            int64_t d, int64_t F, cudaStream_t st) {
    GemvF8Args p{hdr, perm, h8, sh, Q2, nullptr, S2, nullptr, wts, nullptr, out_slot, F, d};
    return launch_gemv_f8_t<false>(p, T, st);
}

}  // namespace jmoe
