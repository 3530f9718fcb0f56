// Debug checks of a forward call, off by default (jamba_moe_debug_checks): they replace the memory
// checkers that cannot run here with checks the kernels make themselves, and report through the
// workspace status word without trapping.
//
//   tables_check_kernel  after the permutation: the routing tables must describe a valid
//                        permutation of the T*K assignments (JMOE_DEV_BAD_TABLE otherwise)
//   canary_fill_kernel   at the start of the call: a fixed pattern into the guard gaps the
//                        workspace layout leaves after each of its regions
//   canary_check_kernel  after the last kernel: the pattern must be intact (JMOE_DEV_CANARY),
//                        so a kernel that wrote past the end of its region is caught
#include "common.cuh"

namespace jmoe {

constexpr uint32_t kCanary = 0xC0DEC0DEu;
constexpr int kCheckThreads = 1024;

// Every invariant the expert kernels rely on:
//   counts sum to TK; seg_start[0] = 0 and each segment is its count rounded up to 128 rows;
//   tile_start = seg_start / 128; touched lists the experts with tokens, ascending;
//   row r of expert e's segment holds, for r - seg_start[e] < counts[e], an assignment a with
//   ids[a] = e and inv[a] = r (so no assignment appears twice), and -1 past the count.
__global__ void __launch_bounds__(kCheckThreads) tables_check_kernel(WsHeader* __restrict__ hdr,
                                                                     const int32_t* __restrict__ ids,
                                                                     const int32_t* __restrict__ perm,
                                                                     const int32_t* __restrict__ inv, int64_t TK,
                                                                     int64_t rows_cap) {
    __shared__ int bad;
    __shared__ int seg[kExperts + 1], cnt[kExperts];
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x;
    if (tid == 0) {
        bad = 0;
        int64_t total = 0;
        int s = 0, nt = 0;
        if (hdr->seg_start[0] != 0) bad = 1;
        for (int e = 0; e < kExperts; ++e) {
            const int c = hdr->counts[e];
            cnt[e] = c;
            seg[e] = hdr->seg_start[e];
            if (c < 0 || seg[e] != s || hdr->tile_start[e] != s / kRowPad) bad = 1;
            if (c > 0) {
                if (nt >= kExperts || hdr->touched[nt] != e) bad = 1;
                ++nt;
            }
            total += c;
            s += (c + kRowPad - 1) / kRowPad * kRowPad;
        }
        seg[kExperts] = hdr->seg_start[kExperts];
        if (seg[kExperts] != s || hdr->tile_start[kExperts] != s / kRowPad || hdr->n_touched != nt) bad = 1;
        if (total != TK || s > rows_cap) bad = 1;
    }
    __syncthreads();
    if (!bad) {
        bool my_bad = false;
        for (int e = 0; e < kExperts; ++e) {
            for (int64_t r = seg[e] + tid; r < seg[e + 1]; r += kCheckThreads) {
                const int32_t a = perm[r];
                if (r - seg[e] < cnt[e]) {
                    if (a < 0 || a >= TK || ids[a] != e || inv[a] != r) my_bad = true;
                } else if (a != -1) {
                    my_bad = true;
                }
            }
        }
        if (my_bad) bad = 1;
    }
    __syncthreads();
    if (tid == 0 && bad) set_status(hdr, JMOE_DEV_BAD_TABLE);
}

// One CTA per guard gap.
__global__ void canary_fill_kernel(uint8_t* __restrict__ ws, const GuardGaps g) {
    pdl_wait();
    pdl_trigger();
    uint32_t* w = reinterpret_cast<uint32_t*>(ws + g.off[blockIdx.x]);
    for (uint32_t i = threadIdx.x; i < kGuardBytes / 4; i += blockDim.x) w[i] = kCanary;
}

__global__ void canary_check_kernel(const uint8_t* __restrict__ ws, const GuardGaps g, WsHeader* __restrict__ hdr) {
    pdl_wait();
    pdl_trigger();
    const uint32_t* w = reinterpret_cast<const uint32_t*>(ws + g.off[blockIdx.x]);
    bool bad = false;
    for (uint32_t i = threadIdx.x; i < kGuardBytes / 4; i += blockDim.x) bad |= (w[i] != kCanary);
    if (__syncthreads_or(bad) && threadIdx.x == 0) set_status(hdr, JMOE_DEV_CANARY);
}

cudaError_t launch_tables_check(WsHeader* hdr, const int32_t* ids, const int32_t* perm, const int32_t* inv, int64_t TK,
                                int64_t rows_cap, cudaStream_t st) {
    return launch_pdl(tables_check_kernel, dim3(1), dim3(kCheckThreads), 0, st, hdr, ids, perm, inv, TK, rows_cap);
}

cudaError_t launch_canary_fill(uint8_t* ws, const GuardGaps& g, cudaStream_t st) {
    if (g.n <= 0) return cudaSuccess;
    return launch_pdl(canary_fill_kernel, dim3((unsigned)g.n), dim3(64), 0, st, ws, g);
}

cudaError_t launch_canary_check(const uint8_t* ws, const GuardGaps& g, WsHeader* hdr, cudaStream_t st) {
    if (g.n <= 0) return cudaSuccess;
    return launch_pdl(canary_check_kernel, dim3((unsigned)g.n), dim3(64), 0, st, ws, g, hdr);
}

}  // namespace jmoe
