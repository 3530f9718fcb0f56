// Decode path of the expert FFN: few tokens per expert, so the work is bound by streaming the
// int8 weights from HBM (Jamba rebuttal page, reply on MoE and Mamba layer interaction: these
// layers are limited by memory traffic, not arithmetic; Jamba-1.5 paper, §3.1: the weights cross
// HBM -> SRAM as int8, half the bytes of BF16, and are turned into BF16 right before the math).
//
//   gemv13: h[r][j]      = bf16( SiLU(S1[j] * (x_r . Q1[j])) * (S3[j] * (x_r . Q3[j])) )
//   gemv2:  out[a][i]    = p_a * S2[i] * (h_r . Q2[i])        (a = the assignment of permuted row r)
//
// CTA = (one touched expert, 16 weight rows), 8 warps splitting K into interleaved 64-wide
// steps.  Each lane streams 16 contiguous int8 weights of rows g and g+8 (g = lane / 4) per step
// with 128-bit no-L1 loads, converts them exactly to bf16 in registers (bit trick, no conversion
// unit) and feeds mma.sync m16n8k16 with the weights as A (16 rows) and up to 8*NT tokens as B.
// Because a k-permutation applied to both operands leaves a dot product unchanged, each lane's
// 16 consecutive k are mapped onto the fragment positions it owns, so activations are also read
// with plain 16-byte loads (from L1/L2: they are tiny and shared by all CTAs of an expert).
// Partial sums of the 8 warps are added in a fixed order in shared memory (deterministic), then
// scales, SiLU * up and the routing weight are applied in fp32.
#include "common.cuh"

namespace jmoe {

constexpr int kGemvWarps = 8;
constexpr int kGemvRows = 16;

struct GemvArgs {
    const WsHeader* hdr;
    const int32_t* perm;   // [rows] assignment index (t*K + k) of each permuted row, -1 = padding
    const uint16_t* act;   // gemv13: x [T][d]; gemv2: h [rows][F]
    const void* qa;        // gemv13: W1 [E][F][d]; gemv2: W2 [E][d][F] (int8 codes, or bf16 weights)
    const void* qb;        // gemv13: W3 [E][F][d]; gemv2: unused
    const float* sa;       // S1 [E][F] / S2 [E][d] (int8 codes only)
    const float* sb;       // S3 [E][F]
    const float* wts;      // gemv2: routing weight of each assignment [T*K]
    uint16_t* h_out;       // gemv13: h [rows][F]
    float* slot_out;       // gemv2: out_slot [T*K][d]
    int64_t K;             // reduction length: d (gemv13) or F (gemv2)
    int64_t N;             // weight rows per expert: F (gemv13) or d (gemv2)
    uint16_t* y_out;       // gemv2 of the dense MLP: y [T][d] in bf16, written instead of out_slot
    int list;              // experts this launch serves: kAllTouched, kFewOnly or kManyOnly
    int k_div;             // assignments per activation row of gemv13 (x row = assignment / k_div; 0: K)
};
enum { kAllTouched = 0, kFewOnly = 1, kManyOnly = 2 };

// One k-step (16 consecutive k per lane) of weights for rows g and g+8: int8 codes fill one
// 16-byte vector per row, bf16 weights two.
template <bool kDual, bool kW8>
struct WeightRegs {
    static constexpr int kV = kW8 ? 1 : 2;
    uint4 a0[kV], a1[kV], b0[kV], b1[kV];  // rows g and g+8 of matrix a (and b)
};

__device__ __forceinline__ uint32_t word(const uint4& v, int j) {
    return j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w));
}
// Word m (0..7) of 16 consecutive bf16 values held in two vectors.
__device__ __forceinline__ uint32_t word8(const uint4 (&v)[2], int m) { return word(v[m >> 2], m & 3); }
__device__ __forceinline__ uint32_t word8(const uint4 (&v)[1], int m) { return word(v[0], m & 3); }

template <int NT, bool kDual, bool kW8>
__device__ __forceinline__ void mma_step(float (&acc_a)[NT][4], float (&acc_b)[NT][4],
                                         const WeightRegs<kDual, kW8>& w, const uint4 (&xa)[NT][2],
                                         const S8Consts& k) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t a0, a1, a2, a3, c0 = 0, c1 = 0, c2 = 0, c3 = 0;
        uint32_t b0[NT], b1[NT];
        if (kW8) {
            // A fragment: k positions (2c, 2c+1) <- bytes 4j, 4j+2; (2c+8, 2c+9) <- bytes 4j+1, 4j+3.
            const uint32_t wa0 = word(w.a0[0], j), wa1 = word(w.a1[0], j);
            a0 = s8x2_even_to_bf16x2(wa0, k);
            a1 = s8x2_even_to_bf16x2(wa1, k);
            a2 = s8x2_odd_to_bf16x2(wa0, k);
            a3 = s8x2_odd_to_bf16x2(wa1, k);
            if (kDual) {
                const uint32_t wb0 = word(w.b0[0], j), wb1 = word(w.b1[0], j);
                c0 = s8x2_even_to_bf16x2(wb0, k);
                c1 = s8x2_even_to_bf16x2(wb1, k);
                c2 = s8x2_odd_to_bf16x2(wb0, k);
                c3 = s8x2_odd_to_bf16x2(wb1, k);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                // activations 4j..4j+3 of this lane's 16: words 2j = (4j, 4j+1), 2j+1 = (4j+2, 4j+3)
                const uint32_t lo = word8(xa[nt], 2 * j), hi = word8(xa[nt], 2 * j + 1);
                b0[nt] = pair_lo(lo, hi);
                b1[nt] = pair_hi(lo, hi);
            }
        } else {
            // bf16 weights: k positions (2c, 2c+1) <- elements 4j, 4j+1; (2c+8, 2c+9) <- 4j+2, 4j+3
            a0 = word8(w.a0, 2 * j);
            a2 = word8(w.a0, 2 * j + 1);
            a1 = word8(w.a1, 2 * j);
            a3 = word8(w.a1, 2 * j + 1);
            if (kDual) {
                c0 = word8(w.b0, 2 * j);
                c2 = word8(w.b0, 2 * j + 1);
                c1 = word8(w.b1, 2 * j);
                c3 = word8(w.b1, 2 * j + 1);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                b0[nt] = word8(xa[nt], 2 * j);
                b1[nt] = word8(xa[nt], 2 * j + 1);
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            mma_bf16_16816(acc_a[nt], a0, a1, a2, a3, b0[nt], b1[nt]);
            if (kDual) mma_bf16_16816(acc_b[nt], c0, c1, c2, c3, b0[nt], b1[nt]);
        }
    }
}

// One pass over K for up to 8*NT tokens of expert e, rows [j0, j0+16).  Warp w takes the k-steps
// w, w+8, w+16, ...; U consecutive steps of a warp are loaded into separate registers before any is
// consumed, so each lane keeps U*(2 or 4)*16 bytes of weights in flight.  Addresses advance by one
// pointer increment per batch; the U steps are immediate offsets from it.  Rows of tokens past the
// expert's count point at a valid row: their MMA columns are computed and then ignored.
// Returns the CTA-reduced accumulators in shared memory red[mat][nt][lane*4 + i].
template <int NT, bool kDual, bool kW8, int U>
__device__ __forceinline__ void gemv_pass(const GemvArgs& p, int e, int64_t j0, const uint16_t* const (&rows)[NT],
                                          float* red /* [kGemvWarps][2][NT][128] */) {
    using W = WeightRegs<kDual, kW8>;
    constexpr int kEl = kW8 ? 1 : 2;  // bytes per weight
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int64_t K = p.K;
    constexpr int kStride = kGemvWarps * 64;  // elements between a warp's steps
    const uint8_t* pa0 =
        static_cast<const uint8_t*>(p.qa) + (((int64_t)e * p.N + j0 + g) * K + 16 * c + warp * 64) * kEl;
    const uint8_t* pa1 = pa0 + 8 * K * kEl;
    const uint8_t* pb0 =
        kDual ? static_cast<const uint8_t*>(p.qb) + (((int64_t)e * p.N + j0 + g) * K + 16 * c + warp * 64) * kEl
              : nullptr;
    const uint8_t* pb1 = kDual ? pb0 + 8 * K * kEl : nullptr;
    const uint16_t* px[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) px[nt] = rows[nt] + 16 * c + warp * 64;

    float acc_a[NT][4], acc_b[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc_a[nt][i] = acc_b[nt][i] = 0.0f;

    const int steps = (int)(K / 64);
    const S8Consts k = s8_consts();
    for (int s0 = warp; s0 < steps; s0 += kGemvWarps * U) {
        W w[U];
        uint4 xa[U][NT][2];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (s0 + u * kGemvWarps < steps) {
#pragma unroll
                for (int v = 0; v < W::kV; ++v) {
                    w[u].a0[v] = ld_stream_v4(pa0 + u * kStride * kEl + 16 * v);
                    w[u].a1[v] = ld_stream_v4(pa1 + u * kStride * kEl + 16 * v);
                    if (kDual) {
                        w[u].b0[v] = ld_stream_v4(pb0 + u * kStride * kEl + 16 * v);
                        w[u].b1[v] = ld_stream_v4(pb1 + u * kStride * kEl + 16 * v);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    xa[u][nt][0] = ld_nc_v4(px[nt] + u * kStride);
                    xa[u][nt][1] = ld_nc_v4(px[nt] + u * kStride + 8);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (s0 + u * kGemvWarps < steps) mma_step<NT, kDual, kW8>(acc_a, acc_b, w[u], xa[u], k);
        pa0 += U * kStride * kEl;
        pa1 += U * kStride * kEl;
        if (kDual) {
            pb0 += U * kStride * kEl;
            pb1 += U * kStride * kEl;
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) px[nt] += U * kStride;
    }
    // fixed-order cross-warp reduction
    float* mine = red + (size_t)warp * 2 * NT * 128;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        *reinterpret_cast<float4*>(mine + (0 * NT + nt) * 128 + lane * 4) =
            make_float4(acc_a[nt][0], acc_a[nt][1], acc_a[nt][2], acc_a[nt][3]);
        if (kDual)
            *reinterpret_cast<float4*>(mine + (1 * NT + nt) * 128 + lane * 4) =
                make_float4(acc_b[nt][0], acc_b[nt][1], acc_b[nt][2], acc_b[nt][3]);
    }
    __syncthreads();
    for (int o = threadIdx.x; o < (kDual ? 2 : 1) * NT * 128; o += blockDim.x) {
        float sum = 0.0f;
#pragma unroll
        for (int w = 0; w < kGemvWarps; ++w) sum += red[(size_t)w * 2 * NT * 128 + o];
        red[o] = sum;  // warp 0's slice now holds the totals
    }
    __syncthreads();
}

template <int NT, bool kDual, bool kW8>
__global__ void __launch_bounds__(kGemvWarps * 32,
                                  kW8 ? ((NT == 1) ? ((kDual) ? 3 : 4) : (NT <= 2 ? ((kDual) ? 2 : 4) : 2))
                                      : ((NT == 1) ? 2 : 1))
    gemv_kernel(GemvArgs p) {
    __shared__ __align__(16) float red[kGemvWarps * 2 * NT * 128];
    pdl_wait();
    const WsHeader* hdr = p.hdr;
    const int n_list = p.list == kFewOnly ? hdr->n_few : (p.list == kManyOnly ? hdr->n_many : hdr->n_touched);
    if ((int)blockIdx.y >= n_list) return;
    const int e = (p.list == kFewOnly ? hdr->few : (p.list == kManyOnly ? hdr->many : hdr->touched))[blockIdx.y];
    const int m = hdr->counts[e];
    const int64_t row0 = hdr->seg_start[e];
    const int64_t j0 = (int64_t)blockIdx.x * kGemvRows;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2;
    for (int n0 = 0; n0 < m; n0 += 8 * NT) {
        const uint16_t* rows[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int n = n0 + nt * 8 + g;
            const int nn = n < m ? n : 0;  // past the count: any valid row, its column is ignored
            if (kDual) {
                const int32_t a = p.perm[row0 + nn];
                rows[nt] = p.act + (int64_t)(a / p.k_div) * p.K;
            } else {
                rows[nt] = p.act + (row0 + nn) * p.K;
            }
        }
        // W2 with 16 tokens per pass: one k-step in flight per warp and 4 CTAs per SM stream faster
        // than two steps at 2 CTAs per SM; W1/W3 with 32 tokens per pass: one k-step (registers)
        gemv_pass<NT, kDual, kW8, (kW8 && ((!kDual && NT == 2) || (kDual && NT == 4))) ? 1 : 2>(p, e, j0, rows, red);
        pdl_trigger();  // main loop done: the next kernel may start launching
        // epilogue over the totals: o = (mat, nt, lane', i); C fragment (lane' = 4g' + c'):
        // i = 0,1 -> row g', tokens 2c', 2c'+1; i = 2,3 -> row g'+8, same tokens.
        for (int o = threadIdx.x; o < NT * 128; o += blockDim.x) {
            const int nt = o >> 7, l2 = (o >> 2) & 31, i = o & 3;
            const int row = (l2 >> 2) + ((i & 2) ? 8 : 0);
            const int n = n0 + nt * 8 + 2 * (l2 & 3) + (i & 1);
            if (n >= m) continue;
            const int64_t jr = j0 + row;
            if (kDual) {
                const float a1 = kW8 ? red[o] * p.sa[(int64_t)e * p.N + jr] : red[o];
                const float a3 = kW8 ? red[NT * 128 + o] * p.sb[(int64_t)e * p.N + jr] : red[NT * 128 + o];
                p.h_out[(row0 + n) * p.N + jr] = f32_to_bf16_bits(silu(a1) * a3);
            } else {
                const int32_t a = p.perm[row0 + n];
                const float v = kW8 ? p.sa[(int64_t)e * p.N + jr] * red[o] : red[o];
                if (p.y_out)  // one assignment per token: round its output to bf16 here
                    p.y_out[(int64_t)(a / kTopK) * p.N + jr] = f32_to_bf16_bits(p.wts[a] * v);
                else
                    p.slot_out[(int64_t)a * p.N + jr] = p.wts[a] * v;
            }
        }
        __syncthreads();  // red is reused by the next pass
    }
}

static int gemv_nt(int64_t T) {
    const int64_t avg = (T * kTopK + kExperts - 1) / kExperts;
    return avg <= 6 ? 1 : (avg <= 12 ? 2 : 4);
}

// Tokens per pass of the dense MLP, where all T tokens take the one weight matrix.
static int gemv_nt_dense(int64_t T) { return T <= 8 ? 1 : (T <= 16 ? 2 : 4); }

template <bool kDual, bool kW8>
static cudaError_t launch_gemv_nt(const GemvArgs& p, int nt, cudaStream_t st, int experts) {
    dim3 grid((unsigned)(p.N / kGemvRows), (unsigned)experts);
    if (nt == 1) return launch_pdl(gemv_kernel<1, kDual, kW8>, grid, dim3(kGemvWarps * 32), 0, st, p);
    if (nt == 2) return launch_pdl(gemv_kernel<2, kDual, kW8>, grid, dim3(kGemvWarps * 32), 0, st, p);
    return launch_pdl(gemv_kernel<4, kDual, kW8>, grid, dim3(kGemvWarps * 32), 0, st, p);
}

// Passes of 16 tokens (nt = 2) stream the weights slower than passes of 8 (nt = 1: more CTAs per
// SM).  When the batch calls for 16-token passes, experts with at most 8 tokens take one launch of
// the 8-token kernel and the others one launch of the 16-token kernel, so each expert's weights
// are still streamed once.
template <bool kDual, bool kW8>
static cudaError_t launch_gemv_t(GemvArgs p, int nt, cudaStream_t st, int experts = kExperts) {
    if (p.k_div <= 0) p.k_div = kTopK;
    if (nt != 2 || experts != kExperts) {
        p.list = kAllTouched;
        return launch_gemv_nt<kDual, kW8>(p, nt, st, experts);
    }
    p.list = kFewOnly;
    cudaError_t e = launch_gemv_nt<kDual, kW8>(p, 1, st, experts);
    if (e != cudaSuccess) return e;
    p.list = kManyOnly;
    return launch_gemv_nt<kDual, kW8>(p, 2, st, experts);
}

cudaError_t launch_gemv13(const WsHeader* hdr, const int32_t* perm, const uint16_t* x, const int8_t* Q1,
                          const float* S1, const int8_t* Q3, const float* S3, uint16_t* h, int64_t T, int64_t d,
                          int64_t F, cudaStream_t st, int k_div) {
    GemvArgs p{hdr, perm, x, Q1, Q3, S1, S3, nullptr, h, nullptr, d, F};
    p.k_div = k_div;
    return launch_gemv_t<true, true>(p, gemv_nt(T), st);
}

cudaError_t launch_gemv2(const WsHeader* hdr, const int32_t* perm, const uint16_t* h, const int8_t* Q2,
                         const float* S2, const float* wts, float* out_slot, int64_t T, int64_t d, int64_t F,
                         cudaStream_t st) {
    GemvArgs p{hdr, perm, h, Q2, nullptr, S2, nullptr, wts, nullptr, out_slot, F, d};
    return launch_gemv_t<false, true>(p, gemv_nt(T), st);
}

// The same two kernels with unquantized bf16 weights (no dequantization, no scales).
cudaError_t launch_gemv13_bf16w(const WsHeader* hdr, const int32_t* perm, const uint16_t* x, const uint16_t* W1,
                                const uint16_t* W3, uint16_t* h, int64_t T, int64_t d, int64_t F, cudaStream_t st) {
    GemvArgs p{hdr, perm, x, W1, W3, nullptr, nullptr, nullptr, h, nullptr, d, F};
    return launch_gemv_t<true, false>(p, gemv_nt(T), st);
}

cudaError_t launch_gemv2_bf16w(const WsHeader* hdr, const int32_t* perm, const uint16_t* h, const uint16_t* W2,
                               const float* wts, float* out_slot, int64_t T, int64_t d, int64_t F, cudaStream_t st) {
    GemvArgs p{hdr, perm, h, W2, nullptr, nullptr, nullptr, wts, nullptr, out_slot, F, d};
    return launch_gemv_t<false, false>(p, gemv_nt(T), st);
}

// The dense MLP (one weight matrix, every token with weight 1): one expert's rows of CTAs, and
// gemv2 writes y in bf16 directly.
cudaError_t launch_gemv13_dense(const WsHeader* hdr, const int32_t* perm, const uint16_t* x, const int8_t* Q1,
                                const float* S1, const int8_t* Q3, const float* S3, uint16_t* h, int64_t T,
                                int64_t d, int64_t F, cudaStream_t st) {
    GemvArgs p{hdr, perm, x, Q1, Q3, S1, S3, nullptr, h, nullptr, d, F, nullptr};
    return launch_gemv_t<true, true>(p, gemv_nt_dense(T), st, 1);
}

cudaError_t launch_gemv2_dense(const WsHeader* hdr, const int32_t* perm, const uint16_t* h, const int8_t* Q2,
                               const float* S2, const float* wts, uint16_t* y, int64_t T, int64_t d, int64_t F,
                               cudaStream_t st) {
    GemvArgs p{hdr, perm, h, Q2, nullptr, S2, nullptr, wts, nullptr, nullptr, F, d, y};
    return launch_gemv_t<false, true>(p, gemv_nt_dense(T), st, 1);
}

}  // namespace jmoe
