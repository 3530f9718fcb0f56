// Device helpers shared by the kernels of the ExpertsInt8 MoE layer (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/jmoe.h"

namespace jmoe {

constexpr int kExperts = 16;
constexpr int kTopK = 2;
constexpr int kRowPad = 128;  // each expert's segment of permuted rows starts on a multiple of this

// ------------------------------------------------------------------ workspace header
// The first kHeaderBytes of the workspace hold the routing tables the kernels exchange.
struct WsHeader {
    uint32_t status;              // JMOE_OK or a JMOE_DEV_* code (first error wins)
    int32_t sched[2];             // tile counters of the two tensor-core GEMMs (dynamic scheduling)
    uint32_t pad0[13];
    int32_t counts[kExperts];     // tokens routed to each expert
    int32_t seg_start[kExperts + 1];  // first permuted row of each expert (multiple of kRowPad)
    int32_t pad1[15];
    int32_t tile_start[kExperts + 1];  // cumulative count of 128-row M tiles (GEMM path)
    int32_t pad2[15];
    int32_t touched[kExperts];    // experts with at least one token, ascending
    int32_t n_touched;
    int32_t pad3[15];
    // the touched experts split by count (decode path: one pass of 8 tokens, or passes of 16)
    int32_t few[kExperts];        // 1 .. kFewTokens tokens, ascending
    int32_t n_few;
    int32_t pad4[15];
    int32_t many[kExperts];       // more than kFewTokens tokens, ascending
    int32_t n_many;
    int32_t pad5[15];
};
constexpr int kFewTokens = 8;
constexpr size_t kHeaderBytes = 4096;
static_assert(sizeof(WsHeader) <= kHeaderBytes, "header too large");

__device__ __forceinline__ void set_status(WsHeader* h, uint32_t code) { atomicCAS(&h->status, 0u, code); }

// Guard gaps of a workspace layout: kGuardBytes after each region, filled with a canary pattern
// and checked when the debug checks are on (byte offsets from the workspace start).
constexpr uint32_t kGuardBytes = 256;
constexpr int kMaxGuards = 16;
struct GuardGaps {
    uint64_t off[kMaxGuards];
    int n;
};

// ------------------------------------------------------------------ loads
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    // Weights are read exactly once per launch: keep them out of L1.
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

// ------------------------------------------------------------------ int8 -> bf16, exact
// For a byte b (two's complement q), the bf16 with exponent 0x86 and mantissa b & 0x7F is
// 128 + (b & 0x7F); subtracting 128 (b >= 0) or 256 (b < 0) leaves exactly q.  Both bf16
// operands and the integer result (|q| <= 128) are exact, so the subtraction is exact.  It is
// done as one bf16x2 fma, c * (-1) + v.
__device__ __forceinline__ uint32_t bf16x2_v_minus_c(uint32_t v, uint32_t c) {
    uint32_t r;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(c), "r"(0xBF80BF80u), "r"(v));
    return r;
}
// The three bit masks of the conversion, held in registers: as immediates the compiler splits each
// (w & mask) | exponent into two logic instructions; with all operands in registers it is one lop3.
struct S8Consts {
    uint32_t low7, sign, expo;
};
__device__ __forceinline__ S8Consts s8_consts() {
    S8Consts k;
    asm volatile("mov.b32 %0, 0x007F007F;" : "=r"(k.low7));
    asm volatile("mov.b32 %0, 0x00800080;" : "=r"(k.sign));
    asm volatile("mov.b32 %0, 0x43004300;" : "=r"(k.expo));
    return k;
}
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {  // (a & b) | c
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
// Bytes 0 and 2 of a 32-bit word as a bf16x2 (byte 0 in the low half).
__device__ __forceinline__ uint32_t s8x2_even_to_bf16x2(uint32_t w, const S8Consts& k) {
    return bf16x2_v_minus_c(and_or(w, k.low7, k.expo), and_or(w, k.sign, k.expo));
}
// Bytes 1 and 3 of the word.
__device__ __forceinline__ uint32_t s8x2_odd_to_bf16x2(uint32_t w, const S8Consts& k) {
    return s8x2_even_to_bf16x2(w >> 8, k);
}

// bf16 pairs (e0, e2) and (e1, e3) from two bf16x2 words holding (e0, e1) and (e2, e3).
__device__ __forceinline__ uint32_t pair_lo(uint32_t a, uint32_t b) { return __byte_perm(a, b, 0x5410); }
__device__ __forceinline__ uint32_t pair_hi(uint32_t a, uint32_t b) { return __byte_perm(a, b, 0x7632); }

// ------------------------------------------------------------------ warp MMA
// D = A * B + D, A 16x16 bf16 (row), B 16x8 bf16 (col), D 16x8 fp32.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float silu(float a) { return a / (1.0f + expf(-a)); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
    __nv_bfloat16 b = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&b);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// ------------------------------------------------------------------ programmatic dependent launch
// Forward-pass kernels are launched with programmatic stream serialization: a kernel may be
// scheduled while its predecessor in the stream is still finishing, and waits in pdl_wait() until
// the predecessor has completed and its writes are visible.  pdl_wait() is called before any read
// of a predecessor's output and before any write a predecessor might still read.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Lets the next kernel in the stream be scheduled once every CTA of this one has called it (or
// exited); correctness never depends on where it is called.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace jmoe
