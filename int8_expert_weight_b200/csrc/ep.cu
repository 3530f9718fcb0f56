// Expert parallelism across GPUs (Jamba-1.5 paper, "Model Architecture": ExpertsInt8 lets
// Jamba-1.5-Large be served on one machine of eight 80 GB GPUs; "Training Infrastructure": expert
// parallelism).  With G ranks, rank g owns experts [g*16/G, (g+1)*16/G).  One layer call is
//
//   dispatch (this file)   router + permutation of the rank's own T tokens, then the rows of x
//                          packed by destination rank: assignment a = t*K + k of expert e goes to
//                          position pos[a] = (assignments of experts < e) + (its rank in e)
//   exchange (NCCL)        all-to-all of the per-rank row counts, then of the packed rows, their
//                          local expert index and routing weight (the caller's collective)
//   experts (this file)    the local experts on the N received rows, one assignment per row:
//                          permutation by local expert, then the ExpertsInt8 expert kernels of the
//                          single-GPU layer; out[n] = w_n * E(x_n) in fp32
//   exchange back (NCCL)   all-to-all of the outputs in reverse, into the send order
//   combine (this file)    y[t] = bf16(ret[pos[t*K]] + ret[pos[t*K+1]]), slot 0 then slot 1
//
// Every rank's y equals the single-GPU layer's: each output row depends only on its own token
// and on its expert's weights, and the two slots are added in the same fixed order.
#include "common.cuh"

namespace jmoe {

// Rows of x in send order, their local expert index and weight, and pos[a] for every assignment.
// One warp per permuted row; 16-byte copies.
__global__ void __launch_bounds__(256) ep_pack_kernel(const uint16_t* __restrict__ x, const WsHeader* __restrict__ hdr,
                                                      const int32_t* __restrict__ perm,
                                                      const float* __restrict__ wts, int64_t d, int experts_per_rank,
                                                      uint16_t* __restrict__ send_x, int32_t* __restrict__ send_e,
                                                      float* __restrict__ send_w, int32_t* __restrict__ pos) {
    __shared__ int seg[kExperts + 1], cum[kExperts + 1], cnt[kExperts];
    pdl_wait();
    pdl_trigger();
    if (threadIdx.x == 0) {
        int c = 0;
        for (int e = 0; e < kExperts; ++e) {
            seg[e] = hdr->seg_start[e];
            cnt[e] = hdr->counts[e];
            cum[e] = c;
            c += cnt[e];
        }
        seg[kExperts] = hdr->seg_start[kExperts];
        cum[kExperts] = c;
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t nrows = seg[kExperts];
    for (int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); r < nrows; r += (int64_t)gridDim.x * 8) {
        int e = 0;
        while (e + 1 < kExperts && r >= seg[e + 1]) ++e;
        const int64_t local = r - seg[e];
        if (local >= cnt[e]) continue;  // padding row
        const int32_t a = perm[r];
        const int64_t p = cum[e] + local;
        if (lane == 0) {
            send_e[p] = e % experts_per_rank;
            send_w[p] = wts[a];
            pos[a] = (int32_t)p;
        }
        const uint4* src = reinterpret_cast<const uint4*>(x + (int64_t)(a / kTopK) * d);
        uint4* dst = reinterpret_cast<uint4*>(send_x + p * d);
        for (int64_t c = lane; c < d / 8; c += 32) dst[c] = ld_nc_v4(src + c);
    }
}

// send_counts[g] = rows for rank g.
__global__ void ep_counts_kernel(const WsHeader* __restrict__ hdr, int experts_per_rank, int n_ranks,
                                 int32_t* __restrict__ send_counts) {
    pdl_wait();
    pdl_trigger();
    const int g = threadIdx.x;
    if (g < n_ranks) {
        int c = 0;
        for (int e = g * experts_per_rank; e < (g + 1) * experts_per_rank; ++e) c += hdr->counts[e];
        send_counts[g] = c;
    }
}

// y[t] = bf16(ret[pos[t*K]] + ret[pos[t*K+1]]): the fixed slot order of the single-GPU combine.
__global__ void __launch_bounds__(256) ep_combine_kernel(const float* __restrict__ ret, const int32_t* __restrict__ pos,
                                                         int64_t T, int64_t d, uint16_t* __restrict__ y) {
    pdl_wait();
    pdl_trigger();
    const int64_t quads = T * d / 4;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < quads; q += stride) {
        const int64_t t = (q * 4) / d, i = (q * 4) % d;
        // a position outside the send buffer (an assignment the dispatch skipped as out of range)
        // contributes nothing
        const int64_t p0 = pos[t * kTopK + 0], p1 = pos[t * kTopK + 1];
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 a = (p0 >= 0 && p0 < T * kTopK) ? *reinterpret_cast<const float4*>(ret + p0 * d + i) : z;
        const float4 b = (p1 >= 0 && p1 < T * kTopK) ? *reinterpret_cast<const float4*>(ret + p1 * d + i) : z;
        const uint32_t lo = (uint32_t)f32_to_bf16_bits(a.x + b.x) | ((uint32_t)f32_to_bf16_bits(a.y + b.y) << 16);
        const uint32_t hi = (uint32_t)f32_to_bf16_bits(a.z + b.z) | ((uint32_t)f32_to_bf16_bits(a.w + b.w) << 16);
        *reinterpret_cast<uint2*>(y + t * d + i) = make_uint2(lo, hi);
    }
}

cudaError_t launch_ep_pack(const uint16_t* x, const WsHeader* hdr, const int32_t* perm, const float* wts, int64_t d,
                           int64_t rows_cap, int experts_per_rank, int n_ranks, uint16_t* send_x, int32_t* send_e,
                           float* send_w, int32_t* pos, int32_t* send_counts, cudaStream_t st, int num_sms) {
    int64_t blocks = (rows_cap + 7) / 8;
    if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
    if (blocks < 1) blocks = 1;
    cudaError_t e = launch_pdl(ep_pack_kernel, dim3((unsigned)blocks), dim3(256), 0, st, x, hdr, perm, wts, d,
                               experts_per_rank, send_x, send_e, send_w, pos);
    if (e != cudaSuccess) return e;
    return launch_pdl(ep_counts_kernel, dim3(1), dim3(32), 0, st, hdr, experts_per_rank, n_ranks, send_counts);
}

cudaError_t launch_ep_combine(const float* ret, const int32_t* pos, int64_t T, int64_t d, uint16_t* y, cudaStream_t st,
                              int num_sms) {
    int64_t blocks = (T * d / 4 + 255) / 256;
    if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
    if (blocks < 1) blocks = 1;
    return launch_pdl(ep_combine_kernel, dim3((unsigned)blocks), dim3(256), 0, st, ret, pos, T, d, y);
}

}  // namespace jmoe
