// Prefill path of the two comparator layers: grouped GEMMs on the 5th-generation tensor cores
// (tcgen05) for unquantized bf16 weights and for FP8 (E4M3) weights and activations, the layers
// the Jamba-1.5 paper measures ExpertsInt8 against (§3.1).  The ExpertsInt8 GEMMs themselves are
// in gemm_ts.cu.
//
//   gemm13: h[r][j] = bf16( SiLU(g_r . W1[j]) * (u_r . W3[j]) )     tile: 128 rows x (128 j of W1 |
//           the same 128 j of W3), so both halves of SwiGLU meet in one accumulator
//   gemm2:  out[a][i] = p_a * (h_r . W2[i])                         tile: 128 rows x BN i
//
// Persistent: one CTA per SM; 192 threads in roles:
//   warp 0       tile scheduler (first tile = CTA index, then an atomic counter in the workspace
//                header, claimed one tile ahead and published through a 4-slot ring) and TMA
//                producer: activation tile + weight tile per K step, both straight into the
//                MMA's SWIZZLE_128B K-major layout (128 bytes of K per row)
//   warp 1       TMEM allocator and MMA issuer: tcgen05.mma kind::f16 (bf16) or kind::f8f6f4 (E4M3),
//                M=128, N=BN, fp32 accumulators in TMEM
//   warps 2-5    epilogue: tcgen05.ld, scales, SiLU * up or routing weight, global stores
// A 4-stage ring of (activation, weight) buffers with full / empty mbarriers, and two TMEM
// accumulators (full / empty mbarriers) so that a tile's epilogue overlaps the next tile's main
// loop.  Every wait is bounded: on timeout the kernel records JMOE_DEV_TIMEOUT in the workspace
// status word, the other roles stop at their next wait, outstanding copies and MMAs are waited
// for (bounded), TMEM is released and the CTA returns.
//
// Tiles are ordered expert by expert; inside an expert, bands of M tiles keep their activations
// resident in L2 while every N tile of the weights streams past once per band.  Tiles are handed
// out in list order as CTAs become free (not by a fixed stride), so the CTAs that share a weight
// tile start it together and read it while it is still in L2.
//
// FP8 (kF8): E4M3 activations and weights, 128 K elements per stage, kind::f8f6f4 MMAs, per-row
// activation scales and per-channel weight scales in the epilogue, bf16 h.
#include <cuda.h>

#include <atomic>

#include "common.cuh"
#include "tc.cuh"

namespace jmoe {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kEpiWarps = 4;
constexpr int kGemmThreads = (2 + kEpiWarps) * 32;
constexpr uint32_t kMaxPolls = 1u << 22;       // ~0.3 s of polling: far above any healthy wait

struct GemmArgs {
    WsHeader* hdr;
    const int32_t* perm;  // assignment index of each permuted row, -1 = padding
    const float* sa;      // FP8 gemm13: S1 [E][N]; FP8 gemm2: S2 [E][N]
    const float* sb;      // FP8 gemm13: S3 [E][N]
    const float* wts;     // gemm2: routing weight per assignment
    uint16_t* h_out;      // gemm13: h [rows][N]
    float* slot_out;      // gemm2: out_slot [T*K][N]
    int K;                // d (gemm13) or ffn (gemm2)
    int N;                // weight rows per expert and matrix: ffn (gemm13) or d (gemm2)
    int n_tiles;          // N tiles per M tile
    int band;             // M tiles per raster band
    uint32_t max_polls;   // bound of every mbarrier wait
    // FP8 layer only: per-row activation scale (gemm13: per token, indexed by assignment / K;
    // gemm2: per permuted row)
    const float* a_scale;
    int sched;  // which tile counter of the header this GEMM uses (zeroed by the permutation)
};
constexpr int kTileSlots = 4;

// Shared-memory ring: per stage the activation tile and the weight tile, both as the MMA reads
// them (128 bytes of K per row: 64 bf16 or 128 E4M3).
template <int BN>
struct StageLayout {
    static constexpr int kStages = 4;
    static constexpr int kA = kBM * 128;              // activations
    static constexpr int kB = BN * 128;               // weights
    static constexpr int kStage = kA + kB;
    static constexpr int kSmem = kStages * kStage + 1024 + 256;
};

__device__ __forceinline__ void fail(WsHeader* hdr, volatile int* abort) {
    *abort = 1;
    set_status(hdr, JMOE_DEV_TIMEOUT);
}

struct TileCoord {
    int e, m_tile, n_tile;
};

// Tile L of the list: expert by expert; inside an expert, bands of `band` M tiles, N tiles of a
// band in order, M tiles of the band fastest.  Returns false past the last tile.
__device__ __forceinline__ bool tile_coord(const WsHeader* hdr, const GemmArgs& p, int L, TileCoord& t) {
    int base = 0;
    for (int i = 0; i < kExperts; ++i) {
        const int mt = hdr->tile_start[i + 1] - hdr->tile_start[i];
        if (L < base + mt * p.n_tiles) {
            const int local = L - base;
            const int band = local / (p.band * p.n_tiles);
            const int m_first = band * p.band;
            const int bsz = min(p.band, mt - m_first);
            const int within = local - band * p.band * p.n_tiles;
            t.e = i;
            t.n_tile = within / bsz;
            t.m_tile = m_first + within % bsz;
            return true;
        }
        base += mt * p.n_tiles;
    }
    return false;
}

// kF8: both operands E4M3 codes copied by TMA into the MMA's layout (no conversion), 128 K
// elements (128 bytes) per stage, kind::f8f6f4 MMAs, activation and weight scales in the epilogue.
template <bool kDual, int BN, bool kF8>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmB1, GemmArgs p) {
    using SL = StageLayout<BN>;
    constexpr int kStages = SL::kStages;
    static_assert(!kDual || BN == 256, "the SwiGLU tile pairs 128 gate rows with 128 up rows");
    constexpr uint32_t kTmemCols = 2 * BN;  // two accumulators
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t tmem_holder;
    __shared__ volatile int abort_flag;
    __shared__ volatile int tile_slot[kTileSlots];

    pdl_wait();
    const WsHeader* hdr = p.hdr;
    const int total = hdr->tile_start[kExperts] * p.n_tiles;
    if ((int)blockIdx.x >= total) return;  // no tile for this CTA: nothing was taken yet

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * SL::kStage);
    uint64_t* full_tma = bars;                  // [kStages] TMA bytes landed
    uint64_t* empty = bars + kStages;           // [kStages] MMAs reading the stage are done
    uint64_t* acc_full = bars + 2 * kStages;    // [2] accumulator complete
    uint64_t* acc_empty = acc_full + 2;         // [2] accumulator read out by the epilogue
    uint64_t* mma_done = acc_empty + 2;         // every issued MMA complete (teardown)
    uint64_t* t_full = mma_done + 1;            // [kTileSlots] tile index published
    uint64_t* t_empty = t_full + kTileSlots;    // [kTileSlots] read by the MMA and epilogue warps
    static_assert((2 * kStages + 5 + 2 * kTileSlots) * 8 <= 256, "barriers");
    auto sA = [&](int s) { return smem + s * SL::kStage; };
    auto sB = [&](int s) { return smem + s * SL::kStage + SL::kA; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(&full_tma[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(&acc_full[b], 1);
            tc::mbar_init(&acc_empty[b], kEpiWarps);
        }
        tc::mbar_init(mma_done, 1);
        for (int s = 0; s < kTileSlots; ++s) {
            tc::mbar_init(&t_full[s], 1);
            tc::mbar_init(&t_empty[s], 1 + kEpiWarps);
        }
        abort_flag = 0;
        tc::mbar_fence_init();
    }
    if (warp == 0 && lane == 0) {
        tc::prefetch_tmap(&tmA);
        tc::prefetch_tmap(&tmB0);
        if (kDual) tc::prefetch_tmap(&tmB1);
    }
    if (warp == 1) tc::tmem_alloc(&tmem_holder, kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = tmem_holder;
    constexpr int kKStage = kF8 ? 128 : kBK;  // K elements per stage (128 bytes per row either way)
    const int KB = p.K / kKStage;
    constexpr uint32_t kTxBytes = SL::kA + SL::kB;
    constexpr uint32_t kIdesc = tc::idesc_bf16_f32(kBM, BN);
    constexpr uint32_t kIdescF8 = tc::idesc_e4m3_f32(kBM, BN);
    int issued_round[kStages];  // producer: last round issued on each stage (-1: none)
#pragma unroll
    for (int s = 0; s < kStages; ++s) issued_round[s] = -1;
    int mma_issued = 0;

    // MMA and epilogue warps: the index of tile `it` (-1 past the last), or -2 after an abort.
    auto next_tile = [&](int it) -> int {
        const int slot = it % kTileSlots, u = it / kTileSlots;
        if (!tc::mbar_wait_bounded(&t_full[slot], u & 1, &abort_flag, p.max_polls)) {
            if (!abort_flag) fail(p.hdr, &abort_flag);
            return -2;
        }
        return tile_slot[slot];
    };

    if (warp == 0) {
        // ---------------- tile scheduler + TMA producer
        if (lane == 0) {
            int g = 0;
            TileCoord t;
            // the next tile's index is claimed one tile ahead, so the atomic's latency hides behind
            // the current tile's copies
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
                tile_coord(hdr, p, L, t);
                const int a_row0 = hdr->seg_start[t.e] + t.m_tile * kBM;
                const int w_row0 = t.e * p.N + t.n_tile * (kDual ? BN / 2 : BN);
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    const int s = g % kStages, r = g / kStages;
                    if (r > 0 && !tc::mbar_wait_bounded(&empty[s], (r - 1) & 1, &abort_flag, p.max_polls)) {
                        if (!abort_flag) fail(p.hdr, &abort_flag);
                        ok = false;
                        break;
                    }
                    tc::mbar_arrive_expect_tx(&full_tma[s], kTxBytes);
                    tc::tma_load_2d(sA(s), &tmA, &full_tma[s], kb * kKStage, a_row0);
                    tc::tma_load_2d(sB(s), &tmB0, &full_tma[s], kb * kKStage, w_row0);
                    if (kDual) tc::tma_load_2d(sB(s) + (BN / 2) * 128, &tmB1, &full_tma[s], kb * kKStage, w_row0);
                    issued_round[s] = r;
                }
                if (!ok) break;
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            int g = 0;
            for (int it = 0;; ++it) {
                const int L = next_tile(it);
                if (L < 0) break;
                tc::mbar_arrive(&t_empty[it % kTileSlots]);
                const int b = it & 1, u = it >> 1;
                if (u > 0 && !tc::mbar_wait_bounded(&acc_empty[b], (u - 1) & 1, &abort_flag, p.max_polls)) {
                    if (!abort_flag) fail(p.hdr, &abort_flag);
                    break;
                }
                tc::tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(b * BN);
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    const int s = g % kStages, r = g / kStages;
                    if (!tc::mbar_wait_bounded(&full_tma[s], r & 1, &abort_flag, p.max_polls)) {
                        if (!abort_flag) fail(p.hdr, &abort_flag);
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint64_t adesc = tc::sw128_kmajor_desc(tc::smem_u32(sA(s)));
                    const uint64_t bdesc = tc::sw128_kmajor_desc(tc::smem_u32(sB(s)));
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {  // +32 bytes per K step (16 bf16 or 32 fp8) = +2 in the address field
                        if (kF8)
                            tc::mma_f8_ss(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, kIdescF8, (kb | kk) != 0);
                        else
                            tc::mma_bf16_ss(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, kIdesc, (kb | kk) != 0);
                    }
                    tc::mma_commit(&empty[s]);
                    ++mma_issued;
                }
                if (!ok) break;
                tc::mma_commit(&acc_full[b]);
            }
            tc::mma_commit(mma_done);  // arrives once every MMA issued above has completed
        }
        __syncwarp();
    } else {
        // ---------------- epilogue
        const int q = warp & 3;  // TMEM lanes 32q .. 32q+31 belong to this warp
        const int row = q * 32 + lane;
        TileCoord t;
        for (int it = 0;; ++it) {
            const int L = next_tile(it);
            __syncwarp();
            if (lane == 0 && L >= 0) tc::mbar_arrive(&t_empty[it % kTileSlots]);
            if (!__all_sync(0xffffffffu, L >= 0)) break;  // warp-uniform
            const int b = it & 1, u = it >> 1;
            bool ok = tc::mbar_wait_bounded(&acc_full[b], u & 1, &abort_flag, p.max_polls);
            if (!ok && !abort_flag) fail(p.hdr, &abort_flag);
            ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
            if (!ok) break;
            tc::tc_fence_after();
            tile_coord(hdr, p, L, t);
            const int64_t gr = (int64_t)hdr->seg_start[t.e] + t.m_tile * kBM + row;
            const uint32_t tbase = tmem + (uint32_t)(b * BN) + ((uint32_t)(q * 32) << 16);
            if constexpr (kDual && kF8) {
                // FP8: scales of the weight rows and of the token's activations; bf16 h in natural k
                // order (quantized per row by the next kernel)
                const int j0 = t.n_tile * (BN / 2);
                const float* s1 = p.sa + (int64_t)t.e * p.N + j0;
                const float* s3 = p.sb + (int64_t)t.e * p.N + j0;
                const int32_t a = p.perm[gr];
                const float as = a >= 0 ? p.a_scale[a / kTopK] : 0.0f;
                uint4* hrow = reinterpret_cast<uint4*>(p.h_out + gr * p.N + j0);
#pragma unroll 1
                for (int c = 0; c < BN / 2; c += 32) {
                    uint32_t a1[32], a3[32];
                    tc::tmem_ld32(tbase + c, a1);
                    tc::tmem_ld32(tbase + BN / 2 + c, a3);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint32_t pk[4];
#pragma unroll
                        for (int k = 0; k < 8; k += 2) {
                            const float g0 = __uint_as_float(a1[i + k]) * as * __ldg(s1 + c + i + k);
                            const float u0 = __uint_as_float(a3[i + k]) * as * __ldg(s3 + c + i + k);
                            const float g1 = __uint_as_float(a1[i + k + 1]) * as * __ldg(s1 + c + i + k + 1);
                            const float u1 = __uint_as_float(a3[i + k + 1]) * as * __ldg(s3 + c + i + k + 1);
                            pk[k / 2] = (uint32_t)f32_to_bf16_bits(silu(g0) * u0) |
                                        ((uint32_t)f32_to_bf16_bits(silu(g1) * u1) << 16);
                        }
                        hrow[(c + i) / 8] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    }
                }
            } else if (kDual) {
                const int j0 = t.n_tile * (BN / 2);
                uint16_t* hrow = p.h_out + gr * p.N + j0;
#pragma unroll 1
                for (int c = 0; c < BN / 2; c += 32) {
                    uint32_t a1[32], a3[32];
                    tc::tmem_ld32(tbase + c, a1);
                    tc::tmem_ld32(tbase + BN / 2 + c, a3);
                    tc::tmem_wait_ld();
                    uint32_t packed[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {  // bf16 weights: no scales
                        const float g0 = __uint_as_float(a1[i]), g1 = __uint_as_float(a1[i + 1]);
                        const float u0 = __uint_as_float(a3[i]), u1 = __uint_as_float(a3[i + 1]);
                        packed[i / 2] = (uint32_t)f32_to_bf16_bits(silu(g0) * u0) |
                                        ((uint32_t)f32_to_bf16_bits(silu(g1) * u1) << 16);
                    }
                    uint4* dst = reinterpret_cast<uint4*>(hrow + c);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
                }
            } else {
                const int i0 = t.n_tile * BN;
                const int32_t a = p.perm[gr];
                // FP8: the routing weight times the row's activation (h) scale
                const float wt = a >= 0 ? p.wts[a] * (kF8 ? p.a_scale[gr] : 1.0f) : 0.0f;
                const float* s2 = kF8 ? p.sa + (int64_t)t.e * p.N + i0 : nullptr;
                {
                    float* orow = p.slot_out + (int64_t)(a >= 0 ? a : 0) * p.N + i0;
#pragma unroll 1
                    for (int c = 0; c < BN; c += 32) {
                        uint32_t v[32];
                        tc::tmem_ld32(tbase + c, v);
                        tc::tmem_wait_ld();
                        if (a >= 0) {
                            float4* dst = reinterpret_cast<float4*>(orow + c);
#pragma unroll
                            for (int k = 0; k < 8; ++k) {
                                float4 o;
                                o.x = wt * ((kF8 ? __ldg(s2 + c + 4 * k + 0) : 1.0f) * __uint_as_float(v[4 * k + 0]));
                                o.y = wt * ((kF8 ? __ldg(s2 + c + 4 * k + 1) : 1.0f) * __uint_as_float(v[4 * k + 1]));
                                o.z = wt * ((kF8 ? __ldg(s2 + c + 4 * k + 2) : 1.0f) * __uint_as_float(v[4 * k + 2]));
                                o.w = wt * ((kF8 ? __ldg(s2 + c + 4 * k + 3) : 1.0f) * __uint_as_float(v[4 * k + 3]));
                                dst[k] = o;
                            }
                        }
                    }
                }
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&acc_empty[b]);
        }
    }

    // ---- teardown: after an abort, let in-flight copies and MMAs finish (bounded) before TMEM goes
    pdl_trigger();
    tc::tc_fence_before();
    __syncthreads();
    if (abort_flag) {
        if (warp == 0 && lane == 0) {
            for (int s = 0; s < kStages; ++s) {
                if (issued_round[s] < 0) continue;
                // a copy of round r completes phase r of full_tma[s]; this wait ignores the abort flag
                for (uint32_t i = 0; i < p.max_polls && !tc::mbar_try_wait(&full_tma[s], issued_round[s] & 1); ++i)
                    __nanosleep(64);
            }
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
namespace {

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

int band_for(int K, int act_bytes) {
    // keep a band's activation tiles (band * 128 rows * K elements) near 24 MB of L2
    const int64_t per_tile = (int64_t)kBM * K * act_bytes;
    int b = (int)((24ll << 20) / per_tile);
    return b < 1 ? 1 : (b > 16 ? 16 : b);
}

template <bool kDual, int BN, bool kF8>
cudaError_t launch_gemm_t(const CUtensorMap& ta, const CUtensorMap& tb0, const CUtensorMap& tb1, const GemmArgs& p,
                          int64_t m_tiles_cap, cudaStream_t st) {
    using SL = StageLayout<BN>;
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<kDual, BN, kF8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SL::kSmem);
    if (e != cudaSuccess) return e;
    // persistent: one CTA per SM (fewer when there are fewer tile slots)
    static std::atomic<int> sms_cache[64];  // per device; zero-initialised (static storage)
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) {
        int n = sms_cache[dev].load(std::memory_order_relaxed);
        if (n <= 0 && cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
            sms_cache[dev].store(n, std::memory_order_relaxed);
        if (n > 0) sms = n;
    }
    int64_t grid = m_tiles_cap * p.n_tiles;
    if (grid > sms) grid = sms;
    return launch_pdl(gemm_tc_kernel<kDual, BN, kF8>, dim3((unsigned)grid), dim3(kGemmThreads), SL::kSmem, st, ta,
                      tb0, tb1, p);
}

}  // namespace

// The same two GEMMs with unquantized bf16 weights: the weight tiles are TMA-loaded in the
// MMA's layout, nothing is converted, no scales are applied, and activations keep their k order.
cudaError_t launch_gemm13_bf16w(WsHeader* hdr, const int32_t* perm, const uint16_t* x_perm, const uint16_t* W1,
                                const uint16_t* W3, uint16_t* h, int64_t rows_cap, int64_t d, int64_t F,
                                cudaStream_t st) {
    CUtensorMap ta, tb0, tb1;
    if (!make_map(&ta, x_perm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows_cap, d, kBM, kBK,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tb0, W1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)kExperts * F, d, 128, kBK,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tb1, W3, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)kExperts * F, d, 128, kBK,
                  CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    GemmArgs p{hdr,          perm,          nullptr,     nullptr,
               nullptr,      h,             nullptr,     (int)d,
               (int)F,       (int)(F / 128), band_for((int)d, 2), kMaxPolls,
               nullptr,      0};
    return launch_gemm_t<true, 256, false>(ta, tb0, tb1, p, rows_cap / kBM, st);
}

cudaError_t launch_gemm2_bf16w(WsHeader* hdr, const int32_t* perm, const uint16_t* h, const uint16_t* W2,
                               const float* wts, float* out_slot, int64_t rows_cap, int64_t d, int64_t F,
                               cudaStream_t st) {
    const int BN = (d % 256 == 0) ? 256 : 128;
    CUtensorMap ta, tb0;
    if (!make_map(&ta, h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows_cap, F, kBM, kBK, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tb0, W2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)kExperts * d, F, BN, kBK,
                  CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    GemmArgs p{hdr,         perm,         nullptr,     nullptr,
               wts,         nullptr,      out_slot,    (int)F,
               (int)d,      (int)(d / BN), band_for((int)F, 2), kMaxPolls,
               nullptr,     1};
    if (BN == 256) return launch_gemm_t<false, 256, false>(ta, tb0, tb0, p, rows_cap / kBM, st);
    return launch_gemm_t<false, 128, false>(ta, tb0, tb0, p, rows_cap / kBM, st);
}

// The FP8 layer's GEMMs: E4M3 activations x8_perm [rows_cap][d] (per-token scales sx, indexed by
// assignment / K) and weights Q1, Q3 [E][F][d] (scales S1, S3); h = SwiGLU in bf16.
cudaError_t launch_gemm13_f8(WsHeader* hdr, const int32_t* perm, const uint8_t* x8_perm, const float* sx,
                             const uint8_t* Q1, const float* S1, const uint8_t* Q3, const float* S3, uint16_t* h,
                             int64_t rows_cap, int64_t d, int64_t F, cudaStream_t st) {
    CUtensorMap ta, tb0, tb1;
    if (!make_map(&ta, x8_perm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows_cap, d, kBM, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tb0, Q1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)kExperts * F, d, 128, 128,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tb1, Q3, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)kExperts * F, d, 128, 128,
                  CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    GemmArgs p{hdr,          perm,          S1,          S3,
               nullptr,      h,             nullptr,     (int)d,
               (int)F,       (int)(F / 128), band_for((int)d, 1), kMaxPolls,
               sx,           0};
    return launch_gemm_t<true, 256, true>(ta, tb0, tb1, p, rows_cap / kBM, st);
}

// out_slot[a] = p_a * sh_r * S2 . (h8_r . Q2^T): E4M3 h8 [rows_cap][F] with per-row scales sh.
cudaError_t launch_gemm2_f8(WsHeader* hdr, const int32_t* perm, const uint8_t* h8, const float* sh, const uint8_t* Q2,
                            const float* S2, const float* wts, float* out_slot, int64_t rows_cap, int64_t d, int64_t F,
                            cudaStream_t st) {
    const int BN = (d % 256 == 0) ? 256 : 128;
    CUtensorMap ta, tb0;
    if (!make_map(&ta, h8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows_cap, F, kBM, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tb0, Q2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)kExperts * d, F, BN, 128,
                  CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    GemmArgs p{hdr,         perm,         S2,          nullptr,
               wts,         nullptr,      out_slot,    (int)F,
               (int)d,      (int)(d / BN), band_for((int)F, 1), kMaxPolls,
               sh,          1};
    if (BN == 256) return launch_gemm_t<false, 256, true>(ta, tb0, tb0, p, rows_cap / kBM, st);
    return launch_gemm_t<false, 128, true>(ta, tb0, tb0, p, rows_cap / kBM, st);
}

}  // namespace jmoe
