// MoE router (Jamba-1.5 paper, "Model Architecture": n = 16 experts, top K = 2 per token).
//
// logits z_e = sum_i x_i Wr[e][i] (+ b_e) on CUDA cores in fp32 (the top-2 decision needs fp32,
// not TF32), softmax over the 16 logits, the two largest logits in descending order (equal
// logits: lower expert index first), weights = their softmax probabilities, not renormalised.
//
// Large batches: a CTA of 128 threads takes 4 tokens; thread t owns the 8-wide column chunks t,
// t+128, ... of d, keeps 4 x 16 partial sums in registers (x read once from HBM, Wr re-read from L2
// once per 4 tokens), and the 128 partials of each (token, expert) are added in a fixed order
// through shared memory.  Small batches (T <= 512): one CTA per token (see router_token_kernel).
// Either way the result is deterministic.
#include "common.cuh"

namespace jmoe {

// Softmax over the 16 logits of one token, top-2 by logit (equal logits: lower index first),
// weights = probabilities of the chosen two, written to the workspace and (if given) the caller.
__device__ __forceinline__ void finish_token(const float* z, int64_t t, int32_t* ids_ws, float* w_ws,
                                             int32_t* ids_user, float* w_user) {
    float zmax = z[0];
#pragma unroll
    for (int e = 1; e < kExperts; ++e) zmax = fmaxf(zmax, z[e]);
    float denom = 0.0f;
#pragma unroll
    for (int e = 0; e < kExperts; ++e) denom += expf(z[e] - zmax);
    int first = 0;
#pragma unroll
    for (int e = 1; e < kExperts; ++e)
        if (z[e] > z[first]) first = e;
    int second = (first == 0) ? 1 : 0;
#pragma unroll
    for (int e = 0; e < kExperts; ++e)
        if (e != first && z[e] > z[second]) second = e;
    const float p1 = expf(z[first] - zmax) / denom, p2 = expf(z[second] - zmax) / denom;
    ids_ws[t * 2] = first;
    ids_ws[t * 2 + 1] = second;
    w_ws[t * 2] = p1;
    w_ws[t * 2 + 1] = p2;
    if (ids_user) {
        ids_user[t * 2] = first;
        ids_user[t * 2 + 1] = second;
    }
    if (w_user) {
        w_user[t * 2] = p1;
        w_user[t * 2 + 1] = p2;
    }
}

constexpr int kRouterThreads = 128;
constexpr int kRouterTokens = 4;

__global__ void __launch_bounds__(kRouterThreads) router_kernel(const uint16_t* __restrict__ x,
                                                                const float* __restrict__ Wr,
                                                                const float* __restrict__ bias, int64_t T,
                                                                int64_t d, int32_t* __restrict__ ids_ws,
                                                                float* __restrict__ w_ws,
                                                                int32_t* __restrict__ ids_user,
                                                                float* __restrict__ w_user) {
    __shared__ float red[kRouterThreads][kRouterTokens * kExperts + 1];
    __shared__ float logits[kRouterTokens][kExperts];
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x;
    const int64_t t0 = (int64_t)blockIdx.x * kRouterTokens;

    float acc[kRouterTokens][kExperts];
#pragma unroll
    for (int a = 0; a < kRouterTokens; ++a)
#pragma unroll
        for (int e = 0; e < kExperts; ++e) acc[a][e] = 0.0f;

    const int64_t chunks = d / 8;
    for (int64_t c = tid; c < chunks; c += kRouterThreads) {
        float xv[kRouterTokens][8];
#pragma unroll
        for (int a = 0; a < kRouterTokens; ++a) {
            uint4 raw = make_uint4(0, 0, 0, 0);
            if (t0 + a < T) raw = ld_nc_v4(x + (t0 + a) * d + c * 8);
            const uint32_t v[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                xv[a][2 * i] = bf16_bits_to_f32(v[i] & 0xFFFFu);
                xv[a][2 * i + 1] = bf16_bits_to_f32(v[i] >> 16);
            }
        }
#pragma unroll
        for (int e = 0; e < kExperts; ++e) {
            const float4 w0 = __ldg(reinterpret_cast<const float4*>(Wr + e * d + c * 8));
            const float4 w1 = __ldg(reinterpret_cast<const float4*>(Wr + e * d + c * 8 + 4));
            const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
            for (int a = 0; a < kRouterTokens; ++a)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[a][e] = fmaf(xv[a][i], wv[i], acc[a][e]);
        }
    }
#pragma unroll
    for (int a = 0; a < kRouterTokens; ++a)
#pragma unroll
        for (int e = 0; e < kExperts; ++e) red[tid][a * kExperts + e] = acc[a][e];
    __syncthreads();
    if (tid < kRouterTokens * kExperts) {
        float s = 0.0f;
        for (int r = 0; r < kRouterThreads; ++r) s += red[r][tid];
        const int e = tid % kExperts;
        if (bias) s += bias[e];
        logits[tid / kExperts][e] = s;
    }
    __syncthreads();
    if (tid < kRouterTokens && t0 + tid < T) finish_token(logits[tid], t0 + tid, ids_ws, w_ws, ids_user, w_user);
}

// Small batches: one CTA of 256 threads per token, so that a decode step spreads the router over
// T SMs.  Thread t owns the 8-wide chunks t, t+256, ...; the 16 partial sums are reduced with warp
// shuffles and then across the 8 warps in shared memory, in a fixed order.
constexpr int kRouterSmallThreads = 256;
__global__ void __launch_bounds__(kRouterSmallThreads) router_token_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ Wr, const float* __restrict__ bias, int64_t d,
    int32_t* __restrict__ ids_ws, float* __restrict__ w_ws, int32_t* __restrict__ ids_user,
    float* __restrict__ w_user) {
    __shared__ float part[kRouterSmallThreads / 32][kExperts];
    __shared__ float logits[kExperts];
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t t = blockIdx.x;
    float acc[kExperts];
#pragma unroll
    for (int e = 0; e < kExperts; ++e) acc[e] = 0.0f;
    for (int64_t c = tid; c < d / 8; c += kRouterSmallThreads) {
        const uint4 raw = ld_nc_v4(x + t * d + c * 8);
        const uint32_t v[4] = {raw.x, raw.y, raw.z, raw.w};
        float xv[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            xv[2 * i] = bf16_bits_to_f32(v[i] & 0xFFFFu);
            xv[2 * i + 1] = bf16_bits_to_f32(v[i] >> 16);
        }
#pragma unroll
        for (int e = 0; e < kExperts; ++e) {
            const float4 w0 = __ldg(reinterpret_cast<const float4*>(Wr + e * d + c * 8));
            const float4 w1 = __ldg(reinterpret_cast<const float4*>(Wr + e * d + c * 8 + 4));
            const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[e] = fmaf(xv[i], wv[i], acc[e]);
        }
    }
#pragma unroll
    for (int e = 0; e < kExperts; ++e) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    }
    if (lane == 0) {
#pragma unroll
        for (int e = 0; e < kExperts; ++e) part[warp][e] = acc[e];
    }
    __syncthreads();
    if (tid < kExperts) {
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < kRouterSmallThreads / 32; ++w) s += part[w][tid];
        if (bias) s += bias[tid];
        logits[tid] = s;
    }
    __syncthreads();
    if (tid == 0) finish_token(logits, t, ids_ws, w_ws, ids_user, w_user);
}

cudaError_t launch_router(const uint16_t* x, const float* Wr, const float* bias, int64_t T, int64_t d,
                          int32_t* ids_ws, float* w_ws, int32_t* ids_user, float* w_user, cudaStream_t st) {
    if (T <= 512) {
        return launch_pdl(router_token_kernel, dim3((unsigned)T), dim3(kRouterSmallThreads), 0, st, x, Wr, bias, d,
                          ids_ws, w_ws, ids_user, w_user);
    } else {
        const int64_t blocks = (T + kRouterTokens - 1) / kRouterTokens;
        return launch_pdl(router_kernel, dim3((unsigned)blocks), dim3(kRouterThreads), 0, st, x, Wr, bias, T, d,
                          ids_ws, w_ws, ids_user, w_user);
    }
    return cudaGetLastError();
}

}  // namespace jmoe
