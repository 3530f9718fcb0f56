// Prefill path of the expert FFN with ExpertsInt8 weights: grouped GEMMs on the 5th-generation
// tensor cores, with each int8 weight tile turned into BF16 inside the kernel right before the
// matrix math (Jamba-1.5 paper, §3.1 ExpertsInt8: int8 weights cross HBM -> SRAM at half the
// bytes and are dequantized to BF16 there; BF16 activations).
//
// The weights are the MMA's A operand and live in tensor memory (TMEM); the tokens are B, in
// shared memory.  One tile = 128 weight rows (M) x up to 256 tokens (N) of one expert:
//
//   gemm13: rows 32q .. 32q+15 of the tile are W1 rows j0+16q .. j0+16q+15 and rows 32q+16 ..
//           32q+31 the W3 rows with the same j (q = 0..3), so gate and up of one j sit in lanes l
//           and l+16 of the same warp and meet with one shuffle:
//           h[t][j] = bf16( SiLU(S1[j] * (x_t . Q1[j])) * (S3[j] * (x_t . Q3[j])) ), 64 j per tile
//   gemm2:  out[a][i] = p_a * S2[i] * (h_t . Q2[i]), 128 i per tile (fp32 slot of assignment a), or
//           y[a / K][i] in bf16 for the dense MLP (one assignment per token)
//
// Each converted weight element is used by up to 256 tokens (the 128-token tiles of an M = 128,
// N = 256 layout use it 128 times), and the BF16 weights never go back through shared memory:
// the converters read the int8 tile from shared memory and write BF16 pairs straight into TMEM
// with tcgen05.st, from where the MMA reads them.
//
// Persistent, one CTA per SM, 864 threads in roles.  A pipeline stage covers 128 of K as two
// 64-wide sub-steps: every hand-off between the roles (copy landed, weights converted, MMAs done)
// is one mbarrier round trip per 128 K, whose fixed latency would otherwise set the pace.
//   warp 0       tile scheduler (first tile = CTA index, then an atomic counter in the workspace
//                header, claimed one tile ahead) and token copies: per stage two TMA boxes of the
//                bf16 token tile [256][64] SWIZZLE_128B (a partial tile: only its 32-row boxes)
//   warp 26      int8 weight copies: per stage two TMA boxes of the tile [128][64] SWIZZLE_64B
//   warp 1       TMEM allocator and MMA issuer: tcgen05.mma kind::f16, A from TMEM, B from smem,
//                M = 128, N = tokens of the tile rounded up to 16, K = 16 (8 per stage)
//   warps 2-9    converters: int8 -> bf16 (exact), two warps per TMEM lane quarter taking turns
//                by stage; each converts the 128 K of its 32 rows and stores them with tcgen05.st
//                into a 4-stage TMEM ring
//   warps 10-25  epilogue: tcgen05.ld of the accumulator, four warps per lane quarter (64 tokens
//                each), scales, SiLU * up or routing weight, global stores.  The MMA of the next
//                tile waits until the accumulator is read out, so the epilogue is split over
//                as many warps as the register budget allows
// TMEM: 256 accumulator columns (fp32 [128][256]) + 256 columns of converted weights (4 stages of
// 64 columns = 128 bf16 per lane).  Rings: 3 token stages (64 KB each), 2 int8 stages (16 KB),
// 4 TMEM stages, 4 tile slots.  Every mbarrier wait is bounded: on timeout the kernel records
// JMOE_DEV_TIMEOUT in the workspace status word, the other roles stop at their next wait,
// in-flight copies and MMAs are waited for (bounded), TMEM is released and the CTA returns.
//
// Tile order: expert by expert; inside an expert, bands of token tiles whose activations stay in
// L2 while every weight tile streams past once per band; token tiles fastest inside a band, so the
// CTAs working at the same time share each weight tile.
//
// k order: the converters turn bytes (b0, b1, b2, b3) of a 4-byte word into the bf16 pairs
// (b0, b2) and (b1, b3), so TMEM holds every group of 4 K elements in the order 0, 2, 1, 3; the
// token operands of this path (x_perm from the gather kernel, h from the gemm13 epilogue) are stored
// with elements 1 and 2 of every group of 4 swapped to match.  A k-permutation applied to both
// operands leaves every dot product unchanged.
#include <cuda.h>

#include <atomic>

#include "common.cuh"
#include "tc.cuh"

namespace jmoe {
namespace ts {

constexpr int kWRows = 128;   // weight rows per tile (MMA M, TMEM lanes)
constexpr int kTokMax = 256;  // tokens per tile at most (MMA N)
constexpr int kAccBufs = 1;   // TMEM accumulators (one of 256 columns leaves 256 for the weight ring)
constexpr int kBK = 64;       // K elements per copy box and converted sub-step
constexpr int kSub = 2;       // sub-steps per pipeline stage (one barrier hand-off per 128 K)
constexpr int kXStages = 3;
constexpr int kQStages = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kACol0 = kAccBufs * kTokMax;  // first TMEM column of the converted-weight ring
constexpr int kAStages = (int)(kTmemCols - kACol0) / (32 * kSub);  // 32 columns = 64 bf16 per lane per sub-step
constexpr int kTileSlots = 4;
constexpr int kConvWarps = 8;                // two per TMEM lane quarter
constexpr int kConvGroups = kConvWarps / 4;  // warps of a quarter take turns: stage g goes to group g % 2
constexpr int kEpiWarps = 16;                // four per TMEM lane quarter
constexpr int kEpiParts = kEpiWarps / 4;     // column ranges of the accumulator, one per warp of a quarter
constexpr int kEpiCols = kTokMax / kEpiParts;
constexpr int kQWarp = 2 + kConvWarps + kEpiWarps;  // the weight-copy warp, after the epilogue warps
constexpr int kThreads = (kQWarp + 1) * 32;
constexpr int kXSub = kTokMax * kBK * 2;  // bf16 tokens of one sub-step, 128-byte rows
constexpr int kXBytes = kSub * kXSub;
constexpr int kXBoxRows = 32;                // rows of the copies that fill a partial token tile
constexpr int kQSub = kWRows * kBK;       // 8 KB: int8 weights of one sub-step, 64-byte rows
constexpr int kQBytes = kSub * kQSub;
constexpr int kBarBytes = 512;
constexpr int kSmem = kXStages * kXBytes + kQStages * kQBytes + kBarBytes + 1024;
constexpr uint32_t kMaxPolls = 1u << 22;      // ~0.3 s of polling: far above any healthy wait
constexpr uint32_t kTestMaxPolls = 1u << 14;  // short bound used together with the test hook
static_assert(kSmem <= 227 * 1024, "shared memory");
static_assert(kAStages >= 4 && kTokMax % 32 == 0 && kTokMax <= 256, "TMEM ring, tile width");

struct Args {
    WsHeader* hdr;
    const int32_t* perm;  // assignment index of each permuted row, -1 = padding
    const float* sa;      // gemm13: S1 [E][N]; gemm2: S2 [E][N]
    const float* sb;      // gemm13: S3 [E][N]
    const float* wts;     // gemm2: routing weight per assignment
    uint16_t* h_out;      // gemm13: h [rows][N]
    float* slot_out;      // gemm2 (MoE): out_slot [T*K][N]
    uint16_t* y_out;      // gemm2 (dense MLP): y [T][N] in bf16
    int K;                // d (gemm13) or ffn (gemm2)
    int N;                // weight rows per expert and matrix: ffn (gemm13) or d (gemm2)
    int n_wt;             // weight tiles per expert: N / 64 (gemm13) or N / 128 (gemm2)
    int band_max;         // token tiles per L2 band, at most
    int sched;            // which tile counter of the header this GEMM uses
    uint32_t max_polls;   // bound of every mbarrier wait
    int skip_copy;        // test hook: CTA 0 skips the copies of the second stage of its first tile
};

struct Tile {
    int e, m, n;  // expert, token tile, weight tile
    int row0;     // first permuted row of the token tile
    int ntok;     // rows of the token tile holding tokens (1 .. 256)
};

__device__ __forceinline__ int tok_tiles(int count) { return (count + kTokMax - 1) / kTokMax; }

__device__ __forceinline__ int count_tiles(const WsHeader* hdr, int n_wt) {
    int total = 0;
#pragma unroll 1
    for (int e = 0; e < kExperts; ++e) total += tok_tiles(hdr->counts[e]) * n_wt;
    return total;
}

// Tile L of the list (see the order above).  Inside an expert with nt token tiles, the bands are
// as even as possible with at most band_max tiles each.
__device__ __forceinline__ bool tile_at(const WsHeader* hdr, const Args& p, int L, Tile& t) {
    int base = 0;
#pragma unroll 1
    for (int e = 0; e < kExperts; ++e) {
        const int count = hdr->counts[e];
        const int nt = tok_tiles(count);
        const int tiles = nt * p.n_wt;
        if (L < base + tiles) {
            const int local = L - base;
            const int nb = (nt + p.band_max - 1) / p.band_max;
            const int bfull = (nt + nb - 1) / nb;
            const int band = local / (bfull * p.n_wt);
            const int m_first = band * bfull;
            const int bsz = min(bfull, nt - m_first);
            const int within = local - band * bfull * p.n_wt;
            t.e = e;
            t.n = within / bsz;
            t.m = m_first + within % bsz;
            t.row0 = hdr->seg_start[e] + t.m * kTokMax;
            t.ntok = min(kTokMax, count - t.m * kTokMax);
            return true;
        }
        base += tiles;
    }
    return false;
}

// tcgen05.st of a converter's bf16 pairs: 8 or 16 columns.
__device__ __forceinline__ void tmem_st_n(uint32_t taddr, const uint32_t (&r)[8]) { tc::tmem_st8(taddr, r); }
__device__ __forceinline__ void tmem_st_n(uint32_t taddr, const uint32_t (&r)[16]) { tc::tmem_st16(taddr, r); }

// SiLU with the fast exponential and division intrinsics: a few fp32 ulps from the exact value,
// far below the bf16 rounding of h that follows.
__device__ __forceinline__ float silu_fast(float a) { return __fdividef(a, 1.0f + __expf(-a)); }

__device__ __forceinline__ void fail(WsHeader* hdr, volatile int* abort) {
    *abort = 1;
    set_status(hdr, JMOE_DEV_TIMEOUT);
}

// Position of k inside its group of 4 in the token operands: elements 1 and 2 swapped.
__device__ __forceinline__ int kpos(int k) { return (k & ~3) | ((k & 1) << 1) | ((k >> 1) & 1); }

template <bool kDual>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_ts_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmXs,
                   const __grid_constant__ CUtensorMap tmQ0, const __grid_constant__ CUtensorMap tmQ1, Args p) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t tmem_holder;
    __shared__ volatile int abort_flag;
    __shared__ volatile int tile_slot[kTileSlots];

    pdl_wait();
    const WsHeader* hdr = p.hdr;
    const int total = count_tiles(hdr, p.n_wt);
    if ((int)blockIdx.x >= total) return;  // no tile for this CTA: nothing was taken yet

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sX = smem;                                // [kXStages][kSub][256 rows][128 B]
    uint8_t* sQ = smem + kXStages * kXBytes;           // [kQStages][kSub][128 rows][64 B]
    uint64_t* bars = reinterpret_cast<uint64_t*>(sQ + kQStages * kQBytes);
    uint64_t* x_full = bars;                           // [kXStages] token tile landed (TMA bytes)
    uint64_t* x_empty = x_full + kXStages;             // [kXStages] MMAs reading it are done
    uint64_t* q_full = x_empty + kXStages;             // [kQStages] int8 tile landed
    uint64_t* q_empty = q_full + kQStages;             // [kQStages] read by every converter warp
    uint64_t* a_full = q_empty + kQStages;             // [kAStages] bf16 weights stored in TMEM
    uint64_t* a_empty = a_full + kAStages;             // [kAStages] MMAs reading them are done
    uint64_t* t_full = a_empty + kAStages;             // [kTileSlots] tile index published
    uint64_t* t_empty = t_full + kTileSlots;           // [kTileSlots] read by every consumer
    uint64_t* acc_full = t_empty + kTileSlots;         // [kAccBufs] accumulator complete
    uint64_t* acc_empty = acc_full + kAccBufs;         // [kAccBufs] accumulator read out by the epilogue
    uint64_t* mma_done = acc_empty + kAccBufs;         // every issued MMA complete (teardown)
    static_assert((2 * kXStages + 2 * kQStages + 2 * kAStages + 2 * kTileSlots + 2 * kAccBufs + 1) * 8 <= kBarBytes,
                  "barriers");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kXStages; ++s) {
            tc::mbar_init(&x_full[s], 1);
            tc::mbar_init(&x_empty[s], 1);
        }
        for (int s = 0; s < kQStages; ++s) {
            tc::mbar_init(&q_full[s], 1);
            tc::mbar_init(&q_empty[s], 4);
        }
        for (int s = 0; s < kAStages; ++s) {
            tc::mbar_init(&a_full[s], 4);
            tc::mbar_init(&a_empty[s], 1);
        }
        for (int s = 0; s < kTileSlots; ++s) {
            tc::mbar_init(&t_full[s], 1);
            tc::mbar_init(&t_empty[s], 2 + kConvWarps + kEpiWarps);  // MMA, converters, epilogue, weight copies
        }
        for (int b = 0; b < kAccBufs; ++b) {
            tc::mbar_init(&acc_full[b], 1);
            tc::mbar_init(&acc_empty[b], kEpiWarps);
        }
        tc::mbar_init(mma_done, 1);
        abort_flag = 0;
        tc::mbar_fence_init();
    }
    if (warp == 0 && lane == 0) {
        tc::prefetch_tmap(&tmX);
        tc::prefetch_tmap(&tmXs);
        tc::prefetch_tmap(&tmQ0);
        if (kDual) tc::prefetch_tmap(&tmQ1);
    }
    if (warp == 1) tc::tmem_alloc(&tmem_holder, kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = tmem_holder;
    const int KB = p.K / (kBK * kSub);
    int issued_x[kXStages], issued_q[kQStages];  // producer: last round issued on each stage (-1: none)
#pragma unroll
    for (int s = 0; s < kXStages; ++s) issued_x[s] = -1;
#pragma unroll
    for (int s = 0; s < kQStages; ++s) issued_q[s] = -1;
    int mma_issued = 0;

    // Consumers: the index of tile `it` (-1 past the last), or -2 after an abort.
    auto next_tile = [&](int it) -> int {
        const int slot = it % kTileSlots, u = it / kTileSlots;
        const bool ok = tc::mbar_wait_bounded(&t_full[slot], u & 1, &abort_flag, p.max_polls);
        if (!ok) {
            if (!abort_flag) fail(p.hdr, &abort_flag);
            return -2;
        }
        return tile_slot[slot];
    };

    if (warp == 0) {
        // ---------------- scheduler + token-tile copies
        if (lane == 0) {
            int g = 0;
            Tile t;
            // the next tile's index is claimed one tile ahead, so the atomic's latency hides
            // behind the current tile's copies
            int L_next = (int)blockIdx.x;
            for (int it = 0;; ++it) {
                int L = L_next;
                if (L >= total || abort_flag) L = -1;
                const int slot = it % kTileSlots, u = it / kTileSlots;
                if (u > 0 && !tc::mbar_wait_bounded(&t_empty[slot], (u - 1) & 1, &abort_flag, p.max_polls)) {
                    if (!abort_flag) fail(p.hdr, &abort_flag);
                    break;
                }
                tile_slot[slot] = L;
                tc::mbar_arrive(&t_full[slot]);  // release: the slot write is visible to the waiters
                if (L < 0) break;
                L_next = (int)gridDim.x + atomicAdd(&p.hdr->sched[p.sched], 1);
                tile_at(hdr, p, L, t);
                // a full tile takes one 256-row copy; a partial one only the 32-row boxes it uses
                const int n_box = (t.ntok == kTokMax) ? 0 : (((t.ntok + 15) & ~15) + kXBoxRows - 1) / kXBoxRows;
                const uint32_t x_bytes = n_box == 0 ? (uint32_t)kXBytes : (uint32_t)(kSub * n_box * kXBoxRows * 128);
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    const int sx = g % kXStages, rx = g / kXStages;
                    if (rx > 0 && !tc::mbar_wait_bounded(&x_empty[sx], (rx - 1) & 1, &abort_flag, p.max_polls)) {
                        ok = false;
                        break;
                    }
                    if (p.skip_copy && blockIdx.x == 0 && it == 0 && kb == 1) continue;
                    tc::mbar_arrive_expect_tx(&x_full[sx], x_bytes);
                    for (int sub = 0; sub < kSub; ++sub) {
                        uint8_t* dx = sX + sx * kXBytes + sub * kXSub;
                        const int kx = (kb * kSub + sub) * kBK;
                        if (n_box == 0) {
                            tc::tma_load_2d(dx, &tmX, &x_full[sx], kx, t.row0);
                        } else {
                            for (int i = 0; i < n_box; ++i)
                                tc::tma_load_2d(dx + i * kXBoxRows * 128, &tmXs, &x_full[sx], kx, t.row0 + i * kXBoxRows);
                        }
                    }
                    issued_x[sx] = rx;
                }
                if (!ok) {
                    if (!abort_flag) fail(p.hdr, &abort_flag);
                    break;
                }
            }
        }
    } else if (warp == kQWarp) {
        // ---------------- int8 weight-tile copies, running ahead of the token copies as far as
        // the (deeper) weight ring allows
        if (lane == 0) {
            int g = 0;
            Tile t;
            for (int it = 0;; ++it) {
                const int L = next_tile(it);
                if (L < 0) break;
                tc::mbar_arrive(&t_empty[it % kTileSlots]);
                tile_at(hdr, p, L, t);
                const int w_row0 = t.e * p.N + t.n * (kDual ? kWRows / 2 : kWRows);
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    const int sq = g % kQStages, rq = g / kQStages;
                    if (rq > 0 && !tc::mbar_wait_bounded(&q_empty[sq], (rq - 1) & 1, &abort_flag, p.max_polls)) {
                        ok = false;
                        break;
                    }
                    tc::mbar_arrive_expect_tx(&q_full[sq], kQBytes);
                    for (int sub = 0; sub < kSub; ++sub) {
                        uint8_t* dq = sQ + sq * kQBytes + sub * kQSub;
                        const int kx = (kb * kSub + sub) * kBK;
                        tc::tma_load_2d(dq, &tmQ0, &q_full[sq], kx, w_row0);
                        if (kDual) tc::tma_load_2d(dq + kQSub / 2, &tmQ1, &q_full[sq], kx, w_row0);
                    }
                    issued_q[sq] = rq;
                }
                if (!ok) {
                    if (!abort_flag) fail(p.hdr, &abort_flag);
                    break;
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            int g = 0;
            Tile t;
            for (int it = 0;; ++it) {
                const int L = next_tile(it);
                if (L < 0) break;
                tc::mbar_arrive(&t_empty[it % kTileSlots]);
                tile_at(hdr, p, L, t);
                const int n_mma = (t.ntok + 15) & ~15;
                const uint32_t idesc = tc::idesc_bf16_f32(kWRows, n_mma);
                const int b = it % kAccBufs, u = it / kAccBufs;
                if (u > 0 && !tc::mbar_wait_bounded(&acc_empty[b], (u - 1) & 1, &abort_flag, p.max_polls)) {
                    if (!abort_flag) fail(p.hdr, &abort_flag);
                    break;
                }
                const uint32_t d_tmem = tmem + (uint32_t)(b * kTokMax);
                tc::tc_fence_after();
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    const int sx = g % kXStages, rx = g / kXStages;
                    const int sa = g % kAStages, ra = g / kAStages;
                    if (!tc::mbar_wait_bounded(&x_full[sx], rx & 1, &abort_flag, p.max_polls) ||
                        !tc::mbar_wait_bounded(&a_full[sa], ra & 1, &abort_flag, p.max_polls)) {
                        if (!abort_flag) fail(p.hdr, &abort_flag);
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
#pragma unroll
                    for (int sub = 0; sub < kSub; ++sub) {
                        const uint64_t bdesc = tc::sw128_kmajor_desc(tc::smem_u32(sX + sx * kXBytes + sub * kXSub));
                        const uint32_t a_col = tmem + kACol0 + (uint32_t)(sa * 32 * kSub + sub * 32);
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk)  // 16 bf16 = 8 TMEM columns of A, 32 bytes of B
                            tc::mma_bf16_ts(d_tmem, a_col + 8 * kk, bdesc + 2 * kk, idesc, (kb | sub | kk) != 0);
                    }
                    tc::mma_commit(&x_empty[sx]);
                    tc::mma_commit(&a_empty[sa]);
                    ++mma_issued;
                }
                if (!ok) break;
                tc::mma_commit(&acc_full[b]);
            }
            tc::mma_commit(mma_done);  // arrives once every MMA issued above has completed
        }
        __syncwarp();
    } else if (warp < 2 + kConvWarps) {
        // ---------------- converters: int8 [128][64] (SWIZZLE_64B: 16-byte chunk c of row r at
        // chunk c ^ ((r >> 1) & 3)) -> bf16 pairs in TMEM lane = tile row
        const int cw = warp - 2, qd = warp & 3, grp = cw >> 2;
        const int trow = 32 * qd + lane;  // TMEM lane = tile row this thread converts
        const int srow = kDual ? ((lane < 16) ? 16 * qd + lane : kWRows / 2 + 16 * qd + lane - 16) : trow;
        const int sw = (srow >> 1) & 3;
        uint32_t coff[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) coff[i] = (uint32_t)(srow * 64 + ((i ^ sw) << 4));
        const uint32_t t_lane = tmem + ((uint32_t)(32 * qd) << 16) + kACol0;
        const S8Consts k8 = s8_consts();
        int g = 0;
        for (int it = 0;; ++it) {
            const int L = next_tile(it);
            __syncwarp();
            if (lane == 0 && L >= 0) tc::mbar_arrive(&t_empty[it % kTileSlots]);
            if (!__all_sync(0xffffffffu, L >= 0)) break;  // warp-uniform
            bool ok = true;
            for (int kb = 0; kb < KB; ++kb, ++g) {
                if (g % kConvGroups != grp) continue;  // another warp of this quarter takes this step
                const int sq = g % kQStages, rq = g / kQStages;
                const int sa = g % kAStages, ra = g / kAStages;
                bool landed = tc::mbar_wait_bounded(&q_full[sq], rq & 1, &abort_flag, p.max_polls);
                if (!__all_sync(0xffffffffu, landed)) {  // warp-uniform: the collectives below need all lanes
                    if (!abort_flag) fail(p.hdr, &abort_flag);
                    ok = false;
                    break;
                }
                const uint8_t* q8 = sQ + sq * kQBytes;
                bool free_ = true;
#pragma unroll
                for (int sub = 0; sub < kSub; ++sub) {
                    uint4 v[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) v[i] = *reinterpret_cast<const uint4*>(q8 + sub * kQSub + coff[i]);
                    if (sub == kSub - 1) {
                        __syncwarp();
                        if (lane == 0) tc::mbar_arrive(&q_empty[sq]);
                    }
                    uint32_t o0[16], o1[16];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            uint32_t* o = (i < 2) ? o0 : o1;
                            o[8 * (i & 1) + 2 * j] = s8x2_even_to_bf16x2(w[j], k8);
                            o[8 * (i & 1) + 2 * j + 1] = s8x2_odd_to_bf16x2(w[j], k8);
                        }
                    }
                    if (sub == 0) {
                        free_ = ra == 0 || tc::mbar_wait_bounded(&a_empty[sa], (ra - 1) & 1, &abort_flag, p.max_polls);
                        if (!__all_sync(0xffffffffu, free_)) break;
                        tc::tc_fence_after();
                    }
                    tc::tmem_st16(t_lane + (uint32_t)(sa * 32 * kSub + sub * 32), o0);
                    tc::tmem_st16(t_lane + (uint32_t)(sa * 32 * kSub + sub * 32 + 16), o1);
                }
                if (!__all_sync(0xffffffffu, free_)) {
                    if (!abort_flag) fail(p.hdr, &abort_flag);
                    ok = false;
                    break;
                }
                tc::tmem_wait_st();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&a_full[sa]);
            }
            if (!ok) break;
        }
    } else {
        // ---------------- epilogue
        const int ew = warp - 2 - kConvWarps, qd = warp & 3, cpart = ew >> 2;
        const uint32_t t_quarter = tmem + ((uint32_t)(32 * qd) << 16);
        Tile t;
        for (int it = 0;; ++it) {
            const int L = next_tile(it);
            __syncwarp();
            if (lane == 0 && L >= 0) tc::mbar_arrive(&t_empty[it % kTileSlots]);
            if (!__all_sync(0xffffffffu, L >= 0)) break;  // warp-uniform
            tile_at(hdr, p, L, t);
            const int b = it % kAccBufs, u = it / kAccBufs;
            const int n_mma = (t.ntok + 15) & ~15;
            constexpr int kChunks = kEpiCols / 32;  // 32-token chunks of this warp's part of the tile
            const int c0 = cpart * kEpiCols;
            // everything the epilogue needs besides the accumulator is loaded before waiting for it:
            // the row scale and (W2) each chunk's assignment and routing weight for this lane's token
            const int jl = 16 * qd + (lane & 15);  // W1/W3: lanes l and l + 16 hold gate and up of j0 + jl
            const int il = 32 * qd + lane;         // W2: the output channel of this lane
            const float sc = kDual ? __ldg((lane < 16 ? p.sa : p.sb) + (int64_t)t.e * p.N + t.n * (kWRows / 2) + jl)
                                   : __ldg(p.sa + (int64_t)t.e * p.N + t.n * kWRows + il);
            int32_t a_l[kChunks];
            float w_l[kChunks];
            if constexpr (!kDual) {
#pragma unroll
                for (int ci = 0; ci < kChunks; ++ci) {
                    const int tok = c0 + 32 * ci + lane;
                    a_l[ci] = (tok < t.ntok) ? p.perm[t.row0 + tok] : -1;
                    w_l[ci] = a_l[ci] >= 0 ? p.wts[a_l[ci]] : 0.0f;
                }
            }
            bool ok = tc::mbar_wait_bounded(&acc_full[b], u & 1, &abort_flag, p.max_polls);
            if (!ok && !abort_flag) fail(p.hdr, &abort_flag);
            if (!__all_sync(0xffffffffu, ok)) break;  // tcgen05.ld below is warp-collective
            tc::tc_fence_after();
            const uint32_t t_lane = t_quarter + (uint32_t)(b * kTokMax);
            // the accumulator is released as soon as this warp's last chunk is in registers, so the
            // next tile's MMAs overlap the math and stores of that chunk
            const int c_end = min(c0 + kEpiCols, n_mma);
            bool released = false;
            auto release = [&]() {
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&acc_empty[b]);
                released = true;
            };
            if constexpr (kDual) {
                uint16_t* hcol = p.h_out + (int64_t)t.n * (kWRows / 2) + kpos(jl);
#pragma unroll 1
                for (int c = c0; c < c_end; c += 32) {
                    uint32_t v[32];
                    tc::tmem_ld32(t_lane + (uint32_t)c, v);
                    tc::tmem_wait_ld();
                    if (c + 32 >= c_end) release();
                    // lanes < 16 keep the gate of tokens c .. c+15 and take the up values from lane + 16;
                    // lanes >= 16 keep the up of tokens c+16 .. c+31 and take the gate values from lane - 16
                    const int tok0 = c + ((lane < 16) ? 0 : 16);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float own_keep = __uint_as_float(v[(lane < 16) ? i : 16 + i]) * sc;
                        const float own_send = __uint_as_float(v[(lane < 16) ? 16 + i : i]) * sc;
                        const float other = __shfl_xor_sync(0xffffffffu, own_send, 16);
                        const float gt = (lane < 16) ? own_keep : other;
                        const float up = (lane < 16) ? other : own_keep;
                        const int tok = tok0 + i;
                        if (tok < n_mma)
                            hcol[(int64_t)(t.row0 + tok) * p.N] = f32_to_bf16_bits(silu_fast(gt) * up);
                    }
                }
            } else {
                const int ig = t.n * kWRows + il;
#pragma unroll
                for (int ci = 0; ci < kChunks; ++ci) {
                    const int c = c0 + 32 * ci;
                    if (c >= n_mma) break;
                    uint32_t v[32];
                    tc::tmem_ld32(t_lane + (uint32_t)c, v);
                    tc::tmem_wait_ld();
                    if (c + 32 >= c_end) release();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int32_t a = __shfl_sync(0xffffffffu, a_l[ci], i);
                        const float wt = __shfl_sync(0xffffffffu, w_l[ci], i);
                        if (a >= 0) {
                            const float o = wt * (sc * __uint_as_float(v[i]));
                            if (p.y_out)
                                p.y_out[(int64_t)(a / kTopK) * p.N + ig] = f32_to_bf16_bits(o);
                            else
                                p.slot_out[(int64_t)a * p.N + ig] = o;
                        }
                    }
                }
            }
            if (!released) release();  // a warp whose columns hold no tokens of this tile
        }
    }

    // ---- teardown: after an abort, let in-flight copies and MMAs finish (bounded) before TMEM goes
    pdl_trigger();
    tc::tc_fence_before();
    __syncthreads();
    if (abort_flag) {
        // a copy of round r completes phase r of its full barrier; these waits ignore the abort flag
        if (warp == 0 && lane == 0) {
            for (int s = 0; s < kXStages; ++s)
                for (uint32_t i = 0; issued_x[s] >= 0 && i < p.max_polls &&
                                     !tc::mbar_try_wait(&x_full[s], issued_x[s] & 1);
                     ++i)
                    __nanosleep(64);
        }
        if (warp == kQWarp && lane == 0) {
            for (int s = 0; s < kQStages; ++s)
                for (uint32_t i = 0; issued_q[s] >= 0 && i < p.max_polls &&
                                     !tc::mbar_try_wait(&q_full[s], issued_q[s] & 1);
                     ++i)
                    __nanosleep(64);
        }
        if (warp == 1 && lane == 0 && mma_issued > 0) {
            for (uint32_t i = 0; i < p.max_polls && !tc::mbar_try_wait(mma_done, 0); ++i) __nanosleep(64);
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Looked up once; the initialisation of a function-local static is thread-safe.
EncodeTiledFn encode_fn() {
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(f);
        return nullptr;
    }();
    return fn;
}

// 2D row-major [rows][cols] tensor, box [box_rows][box_cols].
bool make_map(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, int elem_bytes, uint64_t rows, uint64_t cols,
              uint32_t box_rows, uint32_t box_cols, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * elem_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Token tiles per band: the band's activations (band * 256 rows * K bf16) near 48 MB of L2.
int band_for(int64_t K) {
    const int64_t per_tile = (int64_t)kTokMax * K * 2;
    int64_t b = (48ll << 20) / per_tile;
    return (int)(b < 1 ? 1 : (b > 64 ? 64 : b));
}

int sm_count() {
    static std::atomic<int> cache[64];  // per device; zero-initialised (static storage)
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) {
        int n = cache[dev].load(std::memory_order_relaxed);
        if (n <= 0 && cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
            cache[dev].store(n, std::memory_order_relaxed);
        if (n > 0) sms = n;
    }
    return sms;
}

template <bool kDual>
cudaError_t launch(const CUtensorMap& tx, const CUtensorMap& txs, const CUtensorMap& tq0, const CUtensorMap& tq1,
                   const Args& p, int64_t rows_cap, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(gemm_ts_kernel<kDual>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    // persistent: one CTA per SM (fewer when the row capacity allows fewer tiles)
    int64_t grid = (rows_cap / 128) * p.n_wt;  // an upper bound of the tile count
    const int sms = sm_count();
    if (grid > sms) grid = sms;
    if (grid < 1) grid = 1;
    return launch_pdl(gemm_ts_kernel<kDual>, dim3((unsigned)grid), dim3(kThreads), kSmem, st, tx, txs, tq0, tq1, p);
}

int g_skip_copy = 0;  // set by jamba_moe_debug_skip_copy (tests only)

}  // namespace ts

// h = SwiGLU(x_perm . Q1^T, x_perm . Q3^T) per expert segment; rows_cap = permuted-row capacity;
// n_exp = experts held by Q1/Q3 (16, or 1 for the dense MLP).
cudaError_t launch_gemm13(WsHeader* hdr, const int32_t* perm, const uint16_t* x_perm, const int8_t* Q1,
                          const float* S1, const int8_t* Q3, const float* S3, uint16_t* h, int64_t rows_cap,
                          int64_t d, int64_t F, cudaStream_t st, int n_exp) {
    using namespace ts;
    CUtensorMap tx, txs, tq0, tq1;
    if (!make_map(&tx, x_perm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows_cap, d, kTokMax, kBK,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&txs, x_perm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows_cap, d, kXBoxRows, kBK,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tq0, Q1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)n_exp * F, d, kWRows / 2, kBK,
                  CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map(&tq1, Q3, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)n_exp * F, d, kWRows / 2, kBK,
                  CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    Args p{};
    p.hdr = hdr;
    p.perm = perm;
    p.sa = S1;
    p.sb = S3;
    p.h_out = h;
    p.K = (int)d;
    p.N = (int)F;
    p.n_wt = (int)(F / (kWRows / 2));
    p.band_max = band_for(d);
    p.sched = 0;
    p.max_polls = g_skip_copy ? kTestMaxPolls : kMaxPolls;
    p.skip_copy = g_skip_copy;
    return launch<true>(tx, txs, tq0, tq1, p, rows_cap, st);
}

// out_slot[a] = p_a * S2 . (h_perm . Q2^T) per expert segment, or, given y (the dense MLP, one
// assignment per token), y[a / K] = bf16(p_a * S2 . (h_perm . Q2^T)).
cudaError_t launch_gemm2(WsHeader* hdr, const int32_t* perm, const uint16_t* h, const int8_t* Q2, const float* S2,
                         const float* wts, float* out_slot, int64_t rows_cap, int64_t d, int64_t F, cudaStream_t st,
                         int n_exp, uint16_t* y) {
    using namespace ts;
    CUtensorMap tx, txs, tq0;
    if (!make_map(&tx, h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows_cap, F, kTokMax, kBK,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&txs, h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows_cap, F, kXBoxRows, kBK,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tq0, Q2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)n_exp * d, F, kWRows, kBK,
                  CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    Args p{};
    p.hdr = hdr;
    p.perm = perm;
    p.sa = S2;
    p.wts = wts;
    p.slot_out = out_slot;
    p.y_out = y;
    p.K = (int)F;
    p.N = (int)d;
    p.n_wt = (int)(d / kWRows);
    p.band_max = band_for(F);
    p.sched = 1;
    p.max_polls = g_skip_copy ? kTestMaxPolls : kMaxPolls;
    p.skip_copy = 0;
    return launch<false>(tx, txs, tq0, tq0, p, rows_cap, st);
}

}  // namespace jmoe

// Test hook: while `on` is non-zero, the W1/W3 tensor-core GEMM's CTA 0 skips the copies of the
// second pipeline stage of its first tile, so the wait for them runs out (after a short bound)
// and the kernel must report JMOE_DEV_TIMEOUT, release its resources and return.  Nothing faults
// or hangs.
extern "C" int jamba_moe_debug_skip_copy(int on) {
    jmoe::ts::g_skip_copy = on ? 1 : 0;
    return JMOE_OK;
}
