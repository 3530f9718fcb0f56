// Expert histogram, padded prefix sum and stable token permutation (the batching of tokens per
// expert that lets each expert run as one GEMM; Jamba rebuttal page, reply on MoE and Mamba layer
// interaction: a token's two experts are independent pieces of work, which is what lets them be
// grouped by expert).
//
// One CTA of 1024 threads:
//   1. histogram of the T*K routing assignments (shared-memory integer atomics: exact),
//   2. exclusive scan with each expert's segment padded to a multiple of 128 rows (one GEMM
//      M tile), the list of experts that got tokens, and the per-expert M-tile offsets,
//   3. placement in rounds of 1024 assignments: within a warp, lanes with the same expert are
//      ranked with __match_any_sync, warps are ranked by a fixed-order scan, so an expert's rows
//      keep token order (stable) and the permutation is deterministic,
//   4. padding rows get assignment -1.
// The gather kernel copies x rows into the permuted, padded order for the GEMM path.
#include "common.cuh"

namespace jmoe {

constexpr int kPermThreads = 1024;

__global__ void __launch_bounds__(kPermThreads) permute_kernel(const int32_t* __restrict__ ids, int64_t TK,
                                                               WsHeader* __restrict__ hdr,
                                                               int32_t* __restrict__ perm,
                                                               int32_t* __restrict__ inv, int n_valid) {
    __shared__ int hist[kExperts];
    __shared__ int seg[kExperts + 1];
    __shared__ int base[kExperts];
    __shared__ int wcount[kPermThreads / 32][kExperts];
    __shared__ int wpre[kPermThreads / 32][kExperts];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();
    pdl_trigger();
    if (tid < kExperts) hist[tid] = 0;
    if (tid == 0) {  // first kernel of a forward call to touch the header
        hdr->status = 0;
        hdr->sched[0] = 0;
        hdr->sched[1] = 0;
    }
    __syncthreads();
    bool bad = false;
    for (int64_t a = tid; a < TK; a += kPermThreads) {
        const int e = ids[a];
        if (e < 0 || e >= n_valid) {
            bad = true;
            continue;
        }
        atomicAdd(&hist[e], 1);
    }
    if (bad) set_status(hdr, JMOE_DEV_BAD_INDEX);
    __syncthreads();
    if (tid == 0) {
        int s = 0, nt = 0;
        for (int e = 0; e < kExperts; ++e) {
            seg[e] = s;
            hdr->counts[e] = hist[e];
            hdr->seg_start[e] = s;
            hdr->tile_start[e] = s / kRowPad;
            if (hist[e] > 0) hdr->touched[nt++] = e;
            s += (hist[e] + kRowPad - 1) / kRowPad * kRowPad;
            base[e] = 0;
        }
        seg[kExperts] = s;
        hdr->seg_start[kExperts] = s;
        hdr->tile_start[kExperts] = s / kRowPad;
        for (int e = nt; e < kExperts; ++e) hdr->touched[e] = -1;
        hdr->n_touched = nt;
        int nf = 0, nm = 0;
        for (int e = 0; e < kExperts; ++e) {
            if (hist[e] > kFewTokens) hdr->many[nm++] = e;
            else if (hist[e] > 0) hdr->few[nf++] = e;
        }
        for (int e = nf; e < kExperts; ++e) hdr->few[e] = -1;
        for (int e = nm; e < kExperts; ++e) hdr->many[e] = -1;
        hdr->n_few = nf;
        hdr->n_many = nm;
    }
    __syncthreads();
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int64_t r0 = 0; r0 < TK; r0 += kPermThreads) {
        const int64_t a = r0 + tid;
        int e = -1;
        if (a < TK) {
            e = ids[a];
            if (e < 0 || e >= n_valid) e = -1;
        }
        if (tid < kPermThreads / 32 * kExperts) wcount[tid / kExperts][tid % kExperts] = 0;
        __syncthreads();
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(same & lt_mask);
        if (e >= 0 && rank == 0) wcount[warp][e] = __popc(same);
        __syncthreads();
        if (tid < kExperts) {
            int run = 0;
            for (int w = 0; w < kPermThreads / 32; ++w) {
                wpre[w][tid] = run;
                run += wcount[w][tid];
            }
        }
        __syncthreads();
        if (e >= 0) {
            const int pos = seg[e] + base[e] + wpre[warp][e] + rank;
            perm[pos] = (int32_t)a;
            inv[a] = pos;
        }
        __syncthreads();
        if (tid < kExperts) base[tid] += wpre[kPermThreads / 32 - 1][tid] + wcount[kPermThreads / 32 - 1][tid];
        __syncthreads();
    }
    for (int e = 0; e < kExperts; ++e)
        for (int r = seg[e] + hist[e] + tid; r < seg[e + 1]; r += kPermThreads) perm[r] = -1;
}

// x_perm[r] = x[perm[r] / k_div] for real rows (k_div = K: assignment a belongs to token a / K) (with `swap`, elements 1 and 2 of every group of 4
// swapped: the k order of the int8 tensor-core path), zeros for padding rows; rows past the last
// segment are left alone.  16-byte vector copies, one warp per row.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ x,
                                                          const int32_t* __restrict__ perm,
                                                          const WsHeader* __restrict__ hdr, int64_t d,
                                                          int64_t cap_rows, uint16_t* __restrict__ x_perm,
                                                          int swap, int k_div) {
    const int lane = threadIdx.x & 31;
    pdl_wait();
    pdl_trigger();
    const int64_t nrows = min((int64_t)hdr->seg_start[kExperts], cap_rows);
    const int64_t chunks = d / 8;
    for (int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); r < nrows; r += (int64_t)gridDim.x * 8) {
        const int32_t a = perm[r];
        uint4* dst = reinterpret_cast<uint4*>(x_perm + r * d);
        if (a < 0) {
            for (int64_t c = lane; c < chunks; c += 32) dst[c] = make_uint4(0, 0, 0, 0);
        } else {
            // with int8 weights, elements 1 and 2 of every group of 4 swapped: the k order of the
            // converted weight tiles
            const uint4* src = reinterpret_cast<const uint4*>(x + (int64_t)(a / k_div) * d);
            for (int64_t c = lane; c < chunks; c += 32) {
                const uint4 v = ld_nc_v4(src + c);
                dst[c] = swap ? make_uint4(__byte_perm(v.x, v.y, 0x5410), __byte_perm(v.x, v.y, 0x7632),
                                           __byte_perm(v.z, v.w, 0x5410), __byte_perm(v.z, v.w, 0x7632))
                              : v;
            }
        }
    }
}

// The routing table of the dense MLP, which every token takes with weight 1: the MLP is run as a
// one-expert layer whose expert 0 holds all T tokens in token order.  Token t is assignment t*K
// (the other K-1 assignment slots of a token stay unused), with weight 1; rows T.. of the segment,
// up to the next multiple of kRowPad, are padding (-1).
__global__ void __launch_bounds__(256) dense_setup_kernel(int64_t T, WsHeader* __restrict__ hdr,
                                                          int32_t* __restrict__ perm, float* __restrict__ wts) {
    pdl_wait();
    pdl_trigger();
    const int64_t R = (T + kRowPad - 1) / kRowPad * kRowPad;
    if (blockIdx.x == 0 && threadIdx.x < kExperts) {
        const int e = threadIdx.x;
        if (e == 0) {  // first kernel of a forward call to touch the header
            hdr->status = 0;
            hdr->sched[0] = 0;
            hdr->sched[1] = 0;
        }
        hdr->counts[e] = (e == 0) ? (int32_t)T : 0;
        hdr->seg_start[e] = (e == 0) ? 0 : (int32_t)R;
        hdr->tile_start[e] = (e == 0) ? 0 : (int32_t)(R / kRowPad);
        hdr->touched[e] = (e == 0) ? 0 : -1;
        hdr->few[e] = (e == 0 && T <= kFewTokens) ? 0 : -1;
        hdr->many[e] = (e == 0 && T > kFewTokens) ? 0 : -1;
        if (e == 0) {
            hdr->seg_start[kExperts] = (int32_t)R;
            hdr->tile_start[kExperts] = (int32_t)(R / kRowPad);
            hdr->n_touched = 1;
            hdr->n_few = (T <= kFewTokens) ? 1 : 0;
            hdr->n_many = (T > kFewTokens) ? 1 : 0;
        }
    }
    for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < R; r += (int64_t)gridDim.x * blockDim.x) {
        perm[r] = (r < T) ? (int32_t)(r * kTopK) : -1;
        if (r < T) wts[r * kTopK] = 1.0f;
    }
}

cudaError_t launch_dense_setup(int64_t T, WsHeader* hdr, int32_t* perm, float* wts, cudaStream_t st, int num_sms) {
    const int64_t R = (T + kRowPad - 1) / kRowPad * kRowPad;
    int64_t blocks = (R + 255) / 256;
    if (blocks > num_sms) blocks = num_sms;
    return launch_pdl(dense_setup_kernel, dim3((unsigned)blocks), dim3(256), 0, st, T, hdr, perm, wts);
}

cudaError_t launch_permute(const int32_t* ids, int64_t T, WsHeader* hdr, int32_t* perm, int32_t* inv,
                           cudaStream_t st) {
    return launch_pdl(permute_kernel, dim3(1), dim3(kPermThreads), 0, st, ids, T * kTopK, hdr, perm, inv, kExperts);
}

// The same over TK routing ids of any layout (one id per row: the rows an expert-parallel rank
// received) naming experts 0 .. n_valid-1; other ids are skipped and reported (JMOE_DEV_BAD_INDEX).
cudaError_t launch_permute_tk(const int32_t* ids, int64_t TK, int n_valid, WsHeader* hdr, int32_t* perm, int32_t* inv,
                              cudaStream_t st) {
    return launch_pdl(permute_kernel, dim3(1), dim3(kPermThreads), 0, st, ids, TK, hdr, perm, inv, n_valid);
}

cudaError_t launch_gather(const uint16_t* x, const int32_t* perm, const WsHeader* hdr, int64_t d, int64_t cap_rows,
                          uint16_t* x_perm, cudaStream_t st, int num_sms, bool swap_mid, int k_div) {
    int64_t blocks = (cap_rows + 7) / 8;
    if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
    if (blocks < 1) blocks = 1;
    return launch_pdl(gather_rows_kernel, dim3((unsigned)blocks), dim3(256), 0, st, x, perm, hdr, d, cap_rows,
                      x_perm, swap_mid ? 1 : 0, k_div);
}

}  // namespace jmoe
