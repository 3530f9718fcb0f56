// C ABI of the ExpertsInt8 MoE layer: argument checks, workspace layout, kernel sequencing and
// the optional per-launch event timing.  Declared in include/jmoe.h.
#include <atomic>
#include <vector>

#include "common.cuh"

namespace jmoe {

cudaError_t launch_quantize(const uint16_t* W, int64_t rows, int64_t cols, int8_t* Q, float* S, cudaStream_t st,
                            int num_sms);
cudaError_t launch_router(const uint16_t* x, const float* Wr, const float* bias, int64_t T, int64_t d,
                          int32_t* ids_ws, float* w_ws, int32_t* ids_user, float* w_user, cudaStream_t st);
cudaError_t launch_permute(const int32_t* ids, int64_t T, WsHeader* hdr, int32_t* perm, int32_t* inv,
                           cudaStream_t st);
cudaError_t launch_gather(const uint16_t* x, const int32_t* perm, const WsHeader* hdr, int64_t d, int64_t cap_rows,
                          uint16_t* x_perm, cudaStream_t st, int num_sms, bool swap_mid, int k_div = kTopK);
cudaError_t launch_gemv13_bf16w(const WsHeader* hdr, const int32_t* perm, const uint16_t* x, const uint16_t* W1,
                                const uint16_t* W3, uint16_t* h, int64_t T, int64_t d, int64_t F, cudaStream_t st);
cudaError_t launch_gemv2_bf16w(const WsHeader* hdr, const int32_t* perm, const uint16_t* h, const uint16_t* W2,
                               const float* wts, float* out_slot, int64_t T, int64_t d, int64_t F, cudaStream_t st);
cudaError_t launch_gemm13_bf16w(WsHeader* hdr, const int32_t* perm, const uint16_t* x_perm, const uint16_t* W1,
                                const uint16_t* W3, uint16_t* h, int64_t rows_cap, int64_t d, int64_t F,
                                cudaStream_t st);
cudaError_t launch_gemm2_bf16w(WsHeader* hdr, const int32_t* perm, const uint16_t* h, const uint16_t* W2,
                               const float* wts, float* out_slot, int64_t rows_cap, int64_t d, int64_t F,
                               cudaStream_t st);
cudaError_t launch_gemv13(const WsHeader* hdr, const int32_t* perm, const uint16_t* x, const int8_t* Q1,
                          const float* S1, const int8_t* Q3, const float* S3, uint16_t* h, int64_t T, int64_t d,
                          int64_t F, cudaStream_t st, int k_div = kTopK);
cudaError_t launch_gemv2(const WsHeader* hdr, const int32_t* perm, const uint16_t* h, const int8_t* Q2,
                         const float* S2, const float* wts, float* out_slot, int64_t T, int64_t d, int64_t F,
                         cudaStream_t st);
cudaError_t launch_combine(const float* slots, int64_t T, int64_t d, uint16_t* y, cudaStream_t st, int num_sms);
cudaError_t launch_gemm13(WsHeader* hdr, const int32_t* perm, const uint16_t* x_perm, const int8_t* Q1,
                          const float* S1, const int8_t* Q3, const float* S3, uint16_t* h, int64_t rows_cap,
                          int64_t d, int64_t F, cudaStream_t st, int n_exp);
cudaError_t launch_gemm2(WsHeader* hdr, const int32_t* perm, const uint16_t* h, const int8_t* Q2, const float* S2,
                         const float* wts, float* out_slot, int64_t rows_cap, int64_t d, int64_t F, cudaStream_t st,
                         int n_exp, uint16_t* y);
cudaError_t launch_dense_setup(int64_t T, WsHeader* hdr, int32_t* perm, float* wts, cudaStream_t st, int num_sms);
cudaError_t launch_gemv13_dense(const WsHeader* hdr, const int32_t* perm, const uint16_t* x, const int8_t* Q1,
                                const float* S1, const int8_t* Q3, const float* S3, uint16_t* h, int64_t T,
                                int64_t d, int64_t F, cudaStream_t st);
cudaError_t launch_gemv2_dense(const WsHeader* hdr, const int32_t* perm, const uint16_t* h, const int8_t* Q2,
                               const float* S2, const float* wts, uint16_t* y, int64_t T, int64_t d, int64_t F,
                               cudaStream_t st);

cudaError_t launch_quantize_fp8(const uint16_t* W, int64_t rows, int64_t cols, uint8_t* Q, float* S,
                                const int32_t* perm, const int32_t* n_live, cudaStream_t st, int num_sms);
cudaError_t launch_gemv13_f8(const WsHeader* hdr, const int32_t* perm, const uint8_t* x8, const float* sx,
                             const uint8_t* Q1, const float* S1, const uint8_t* Q3, const float* S3, uint16_t* h,
                             int64_t T, int64_t d, int64_t F, cudaStream_t st);
cudaError_t launch_gemv2_f8(const WsHeader* hdr, const int32_t* perm, const uint8_t* h8, const float* sh,
                            const uint8_t* Q2, const float* S2, const float* wts, float* out_slot, int64_t T,
                            int64_t d, int64_t F, cudaStream_t st);
cudaError_t launch_gemm13_f8(WsHeader* hdr, const int32_t* perm, const uint8_t* x8_perm, const float* sx,
                             const uint8_t* Q1, const float* S1, const uint8_t* Q3, const float* S3, uint16_t* h,
                             int64_t rows_cap, int64_t d, int64_t F, cudaStream_t st);
cudaError_t launch_gemm2_f8(WsHeader* hdr, const int32_t* perm, const uint8_t* h8, const float* sh, const uint8_t* Q2,
                            const float* S2, const float* wts, float* out_slot, int64_t rows_cap, int64_t d, int64_t F,
                            cudaStream_t st);

cudaError_t launch_tables_check(WsHeader* hdr, const int32_t* ids, const int32_t* perm, const int32_t* inv, int64_t TK,
                                int64_t rows_cap, cudaStream_t st);
cudaError_t launch_canary_fill(uint8_t* ws, const GuardGaps& g, cudaStream_t st);
cudaError_t launch_canary_check(const uint8_t* ws, const GuardGaps& g, WsHeader* hdr, cudaStream_t st);

namespace {

constexpr int64_t kMaxT = int64_t(1) << 20;
constexpr int64_t kMaxDim = 32768;
constexpr int64_t kGemvMaxTokens = 128;  // auto path: GEMV up to 2*128/16 = 16 rows per expert on average

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

struct Layout {
    int64_t rows_cap;  // permuted rows incl. per-expert padding
    size_t hdr, ids, wts, inv, perm, x_perm, h, slots, total;
    GuardGaps guards;  // a canary gap after every region
};

// Region allocator of the workspace layouts: 256-byte aligned regions, each followed by a guard
// gap of kGuardBytes (checked for overwrites when the debug checks are on).
struct Regions {
    size_t off = 0;
    GuardGaps g{};
    size_t take(size_t bytes) {
        const size_t at = off;
        off = (off + bytes + 255) & ~size_t(255);
        if (g.n < kMaxGuards) g.off[g.n++] = off;
        off += kGuardBytes;
        return at;
    }
};

// Test hooks (host-side state, not thread-safe): debug checks on every forward call, and a one-shot
// corruption of the next call's routing state, made from the host with in-bounds copies.
int g_debug_checks = 0;
int g_corrupt = 0;  // JMOE_CORRUPT_*

bool shape_ok(int64_t T, int64_t d, int64_t F, int E, int K) {
    if (E != kExperts || K != kTopK) return false;
    if (T < 0 || T > kMaxT) return false;
    if (d < 128 || d > kMaxDim || d % 128 != 0) return false;
    if (F < 128 || F > kMaxDim || F % 128 != 0) return false;
    return true;
}

Layout make_layout(int64_t T, int64_t d, int64_t F) {
    Layout L{};
    const int64_t TK = T * kTopK;
    L.rows_cap = (TK + int64_t(kExperts) * (kRowPad - 1) + kRowPad - 1) / kRowPad * kRowPad;
    Regions R;
    L.hdr = R.take(kHeaderBytes);
    L.ids = R.take(sizeof(int32_t) * TK);
    L.wts = R.take(sizeof(float) * TK);
    L.inv = R.take(sizeof(int32_t) * TK);
    L.perm = R.take(sizeof(int32_t) * L.rows_cap);
    L.x_perm = R.take(sizeof(uint16_t) * L.rows_cap * d);
    L.h = R.take(sizeof(uint16_t) * L.rows_cap * F);
    L.slots = R.take(sizeof(float) * TK * d);
    L.total = R.off;
    L.guards = R.g;
    return L;
}

// The debug-check and corruption steps of a MoE forward call, at the points the call reaches.
enum Step { kAtStart, kAfterRouter, kAfterPermute, kAtEnd };
cudaError_t debug_step(Step at, char* ws, const GuardGaps& guards, WsHeader* hdr, int32_t* ids, const int32_t* perm,
                       const int32_t* inv, int64_t TK, int64_t rows_cap, cudaStream_t st) {
    cudaError_t e = cudaSuccess;
    uint8_t* w8 = reinterpret_cast<uint8_t*>(ws);
    switch (at) {
        case kAtStart:
            if (g_debug_checks) e = launch_canary_fill(w8, guards, st);
            break;
        case kAfterRouter:
            if (g_corrupt == JMOE_CORRUPT_ROUTE_ID) {  // routing id of assignment 0 := 0x7F7F7F7F
                g_corrupt = 0;
                e = cudaMemsetAsync(ids, 0x7F, sizeof(int32_t), st);
            }
            break;
        case kAfterPermute:
            if (g_corrupt == JMOE_CORRUPT_PERM_ROW) {  // permuted row 1 := permuted row 0
                g_corrupt = 0;
                e = cudaMemcpyAsync(const_cast<int32_t*>(perm) + 1, perm, sizeof(int32_t), cudaMemcpyDeviceToDevice,
                                    st);
            }
            if (e == cudaSuccess && g_debug_checks) e = launch_tables_check(hdr, ids, perm, inv, TK, rows_cap, st);
            break;
        case kAtEnd:
            if (g_corrupt == JMOE_CORRUPT_CANARY && guards.n > 1) {  // one byte of the second guard gap
                g_corrupt = 0;
                e = cudaMemsetAsync(w8 + guards.off[1] + 17, 0x5A, 1, st);
            }
            if (e == cudaSuccess && g_debug_checks) e = launch_canary_check(w8, guards, hdr, st);
            break;
    }
    return e;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// SM count of the current device, looked up once per device (relaxed atomics: several host
// threads may race to fill an entry, all with the same value).
int num_sms_current() {
    static std::atomic<int> cache[64];  // zero-initialised (static storage)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// ---------------------------------------------------------------- launch timing
struct Timing {
    std::vector<cudaEvent_t> start, stop;
    std::vector<int> kind;
    int used = 0;
    bool on = false;
} g_timing;

struct TimedLaunch {
    cudaStream_t st;
    int slot = -1;
    TimedLaunch(int kind, cudaStream_t s) : st(s) {
        if (g_timing.on && g_timing.used < (int)g_timing.start.size()) {
            slot = g_timing.used++;
            g_timing.kind[slot] = kind;
            cudaEventRecord(g_timing.start[slot], st);
        }
    }
    ~TimedLaunch() {
        if (slot >= 0) cudaEventRecord(g_timing.stop[slot], st);
    }
};

int to_status(cudaError_t e) { return e == cudaSuccess ? JMOE_OK : JMOE_ERR_CUDA; }

}  // namespace
}  // namespace jmoe

using namespace jmoe;

extern "C" {

int jamba_moe_quantize(const uint16_t* W, int64_t n_mats, int64_t rows, int64_t cols, int8_t* Q, float* S,
                       void* stream) {
    if (!W || !Q || !S) return JMOE_ERR_NULL;
    if (n_mats < 1 || rows < 1 || cols < 16 || cols > (int64_t(1) << 20) || cols % 16 != 0) return JMOE_ERR_SHAPE;
    if (n_mats > (int64_t(1) << 40) / rows) return JMOE_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(Q) || (reinterpret_cast<uintptr_t>(S) & 3)) return JMOE_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    TimedLaunch t(JMOE_KERNEL_QUANTIZE, st);
    return to_status(launch_quantize(W, n_mats * rows, cols, Q, S, st, num_sms_current()));
}

size_t jamba_moe_workspace_size(int64_t T, int64_t d, int64_t ffn, int n_experts, int top_k) {
    if (!shape_ok(T, d, ffn, n_experts, top_k)) return 0;
    return make_layout(T, d, ffn).total;
}

}  // extern "C"

namespace {

// The layer with either int8 weights (codes + per-row scales, w8) or unquantized bf16 weights.
int forward_impl(const uint16_t* x, const float* router_W, const float* router_bias, const void* W1,
                 const float* S1, const void* W3, const float* S3, const void* W2, const float* S2, bool w8,
                 int64_t T, int64_t d, int64_t ffn, int n_experts, int top_k, uint16_t* y, int32_t* topk_ids,
                 float* topk_w, void* workspace, size_t workspace_bytes, void* stream, int path) {
    if (!shape_ok(T, d, ffn, n_experts, top_k)) return JMOE_ERR_SHAPE;
    if (path != JMOE_PATH_AUTO && path != JMOE_PATH_GEMV && path != JMOE_PATH_GEMM) return JMOE_ERR_SHAPE;
    if (T == 0) return JMOE_OK;  // no token: nothing to read or write
    if (!x || !router_W || !W1 || !W3 || !W2 || !y || !workspace) return JMOE_ERR_NULL;
    if (w8 && (!S1 || !S3 || !S2)) return JMOE_ERR_NULL;
    const void* ptrs16[] = {x, W1, W3, W2, y, router_W};
    for (const void* p : ptrs16)
        if (!aligned16(p)) return JMOE_ERR_ALIGN;
    const void* ptrs4[] = {router_bias, S1, S3, S2, topk_ids, topk_w};
    for (const void* p : ptrs4)
        if (reinterpret_cast<uintptr_t>(p) & 3) return JMOE_ERR_ALIGN;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return JMOE_ERR_WORKSPACE;
    const Layout L = make_layout(T, d, ffn);
    if (workspace_bytes < L.total) return JMOE_ERR_WORKSPACE;

    char* ws = static_cast<char*>(workspace);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + L.hdr);
    int32_t* ids = reinterpret_cast<int32_t*>(ws + L.ids);
    float* wts = reinterpret_cast<float*>(ws + L.wts);
    int32_t* inv = reinterpret_cast<int32_t*>(ws + L.inv);
    int32_t* perm = reinterpret_cast<int32_t*>(ws + L.perm);
    uint16_t* x_perm = reinterpret_cast<uint16_t*>(ws + L.x_perm);
    uint16_t* h = reinterpret_cast<uint16_t*>(ws + L.h);
    float* slots = reinterpret_cast<float*>(ws + L.slots);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int sms = num_sms_current();
    // Few tokens per expert: stream the weights (GEMV); otherwise grouped tensor-core GEMMs.
    if (path == JMOE_PATH_AUTO) path = (T <= kGemvMaxTokens) ? JMOE_PATH_GEMV : JMOE_PATH_GEMM;
    const int8_t* Q1 = static_cast<const int8_t*>(W1);
    const int8_t* Q3 = static_cast<const int8_t*>(W3);
    const int8_t* Q2 = static_cast<const int8_t*>(W2);
    const uint16_t* B1 = static_cast<const uint16_t*>(W1);
    const uint16_t* B3 = static_cast<const uint16_t*>(W3);
    const uint16_t* B2 = static_cast<const uint16_t*>(W2);

    const int64_t TK = T * kTopK;
    cudaError_t e = debug_step(kAtStart, ws, L.guards, hdr, ids, perm, inv, TK, L.rows_cap, st);
    if (e != cudaSuccess) return JMOE_ERR_CUDA;
    {
        TimedLaunch t(JMOE_KERNEL_ROUTER, st);
        e = launch_router(x, router_W, router_bias, T, d, ids, wts, topk_ids, topk_w, st);
    }
    if (e != cudaSuccess) return JMOE_ERR_CUDA;
    if (debug_step(kAfterRouter, ws, L.guards, hdr, ids, perm, inv, TK, L.rows_cap, st) != cudaSuccess)
        return JMOE_ERR_CUDA;
    {
        TimedLaunch t(JMOE_KERNEL_PERMUTE, st);
        e = launch_permute(ids, T, hdr, perm, inv, st);
    }
    if (e != cudaSuccess) return JMOE_ERR_CUDA;
    if (debug_step(kAfterPermute, ws, L.guards, hdr, ids, perm, inv, TK, L.rows_cap, st) != cudaSuccess)
        return JMOE_ERR_CUDA;
    if (path == JMOE_PATH_GEMV) {
        {
            TimedLaunch t(JMOE_KERNEL_GEMV13, st);
            e = w8 ? launch_gemv13(hdr, perm, x, Q1, S1, Q3, S3, h, T, d, ffn, st)
                   : launch_gemv13_bf16w(hdr, perm, x, B1, B3, h, T, d, ffn, st);
        }
        if (e != cudaSuccess) return JMOE_ERR_CUDA;
        {
            TimedLaunch t(JMOE_KERNEL_GEMV2, st);
            e = w8 ? launch_gemv2(hdr, perm, h, Q2, S2, wts, slots, T, d, ffn, st)
                   : launch_gemv2_bf16w(hdr, perm, h, B2, wts, slots, T, d, ffn, st);
        }
        if (e != cudaSuccess) return JMOE_ERR_CUDA;
    } else {
        {
            TimedLaunch t(JMOE_KERNEL_GATHER, st);
            e = launch_gather(x, perm, hdr, d, L.rows_cap, x_perm, st, sms, w8);
        }
        if (e != cudaSuccess) return JMOE_ERR_CUDA;
        {
            TimedLaunch t(JMOE_KERNEL_GEMM13, st);
            e = w8 ? launch_gemm13(hdr, perm, x_perm, Q1, S1, Q3, S3, h, L.rows_cap, d, ffn, st, kExperts)
                   : launch_gemm13_bf16w(hdr, perm, x_perm, B1, B3, h, L.rows_cap, d, ffn, st);
        }
        if (e != cudaSuccess) return JMOE_ERR_CUDA;
        {
            TimedLaunch t(JMOE_KERNEL_GEMM2, st);
            e = w8 ? launch_gemm2(hdr, perm, h, Q2, S2, wts, slots, L.rows_cap, d, ffn, st, kExperts, nullptr)
                   : launch_gemm2_bf16w(hdr, perm, h, B2, wts, slots, L.rows_cap, d, ffn, st);
        }
        if (e != cudaSuccess) return JMOE_ERR_CUDA;
    }
    {
        TimedLaunch t(JMOE_KERNEL_COMBINE, st);
        e = launch_combine(slots, T, d, y, st, sms);
    }
    if (e != cudaSuccess) return JMOE_ERR_CUDA;
    return to_status(debug_step(kAtEnd, ws, L.guards, hdr, ids, perm, inv, TK, L.rows_cap, st));
}

}  // namespace

namespace {

// ---------------------------------------------------------------- dense MLP
// The MLP runs as a one-expert layer: a table kernel in place of router + permute, the same
// expert kernels, and a down-projection that writes y in bf16 (no slots, no combine).
constexpr int64_t kMlpGemvMaxTokens = 64;

Layout make_layout_mlp(int64_t T, int64_t d, int64_t F) {
    Layout L{};
    L.rows_cap = (T + kRowPad - 1) / kRowPad * kRowPad;
    size_t off = 0;
    L.hdr = off;
    off = align256(off + kHeaderBytes);
    L.wts = off;
    off = align256(off + sizeof(float) * T * kTopK);
    L.perm = off;
    off = align256(off + sizeof(int32_t) * L.rows_cap);
    L.x_perm = off;
    off = align256(off + sizeof(uint16_t) * L.rows_cap * d);
    L.h = off;
    off = align256(off + sizeof(uint16_t) * L.rows_cap * F);
    L.ids = L.inv = L.slots = off;  // unused
    L.total = off;
    return L;
}

int mlp_impl(const uint16_t* x, const int8_t* Q1, const float* S1, const int8_t* Q3, const float* S3,
             const int8_t* Q2, const float* S2, int64_t T, int64_t d, int64_t ffn, uint16_t* y, void* workspace,
             size_t workspace_bytes, void* stream, int path) {
    if (!shape_ok(T, d, ffn, kExperts, kTopK)) return JMOE_ERR_SHAPE;
    if (path != JMOE_PATH_AUTO && path != JMOE_PATH_GEMV && path != JMOE_PATH_GEMM) return JMOE_ERR_SHAPE;
    if (T == 0) return JMOE_OK;
    if (!x || !Q1 || !S1 || !Q3 || !S3 || !Q2 || !S2 || !y || !workspace) return JMOE_ERR_NULL;
    const void* ptrs16[] = {x, Q1, Q3, Q2, y};
    for (const void* p : ptrs16)
        if (!aligned16(p)) return JMOE_ERR_ALIGN;
    const void* ptrs4[] = {S1, S3, S2};
    for (const void* p : ptrs4)
        if (reinterpret_cast<uintptr_t>(p) & 3) return JMOE_ERR_ALIGN;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return JMOE_ERR_WORKSPACE;
    const Layout L = make_layout_mlp(T, d, ffn);
    if (workspace_bytes < L.total) return JMOE_ERR_WORKSPACE;

    char* ws = static_cast<char*>(workspace);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + L.hdr);
    float* wts = reinterpret_cast<float*>(ws + L.wts);
    int32_t* perm = reinterpret_cast<int32_t*>(ws + L.perm);
    uint16_t* x_perm = reinterpret_cast<uint16_t*>(ws + L.x_perm);
    uint16_t* h = reinterpret_cast<uint16_t*>(ws + L.h);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int sms = num_sms_current();
    if (path == JMOE_PATH_AUTO) path = (T <= kMlpGemvMaxTokens) ? JMOE_PATH_GEMV : JMOE_PATH_GEMM;

    cudaError_t e;
    {
        TimedLaunch t(JMOE_KERNEL_PERMUTE, st);
        e = launch_dense_setup(T, hdr, perm, wts, st, sms);
    }
    if (e != cudaSuccess) return JMOE_ERR_CUDA;
    if (path == JMOE_PATH_GEMV) {
        {
            TimedLaunch t(JMOE_KERNEL_GEMV13, st);
            e = launch_gemv13_dense(hdr, perm, x, Q1, S1, Q3, S3, h, T, d, ffn, st);
        }
        if (e != cudaSuccess) return JMOE_ERR_CUDA;
        TimedLaunch t(JMOE_KERNEL_GEMV2, st);
        return to_status(launch_gemv2_dense(hdr, perm, h, Q2, S2, wts, y, T, d, ffn, st));
    }
    {
        TimedLaunch t(JMOE_KERNEL_GATHER, st);
        e = launch_gather(x, perm, hdr, d, L.rows_cap, x_perm, st, sms, true);
    }
    if (e != cudaSuccess) return JMOE_ERR_CUDA;
    {
        TimedLaunch t(JMOE_KERNEL_GEMM13, st);
        e = launch_gemm13(hdr, perm, x_perm, Q1, S1, Q3, S3, h, L.rows_cap, d, ffn, st, 1);
    }
    if (e != cudaSuccess) return JMOE_ERR_CUDA;
    TimedLaunch t(JMOE_KERNEL_GEMM2, st);
    return to_status(launch_gemm2(hdr, perm, h, Q2, S2, wts, nullptr, L.rows_cap, d, ffn, st, 1, y));
}

}  // namespace

namespace {

// ---------------------------------------------------------------- FP8 (E4M3) comparator layer
struct LayoutF8 {
    int64_t rows_cap;
    size_t hdr, ids, wts, inv, perm, x8, sx, x8_perm, h, h8, sh, slots, total;
    GuardGaps guards;
};

LayoutF8 make_layout_f8(int64_t T, int64_t d, int64_t F) {
    LayoutF8 L{};
    const int64_t TK = T * kTopK;
    L.rows_cap = (TK + int64_t(kExperts) * (kRowPad - 1) + kRowPad - 1) / kRowPad * kRowPad;
    Regions R;
    auto take = [&](size_t bytes) { return R.take(bytes); };
    L.hdr = take(kHeaderBytes);
    L.ids = take(sizeof(int32_t) * TK);
    L.wts = take(sizeof(float) * TK);
    L.inv = take(sizeof(int32_t) * TK);
    L.perm = take(sizeof(int32_t) * L.rows_cap);
    L.x8 = take((size_t)T * d);
    L.sx = take(sizeof(float) * T);
    L.x8_perm = take((size_t)L.rows_cap * d);
    L.h = take(sizeof(uint16_t) * L.rows_cap * F);
    L.h8 = take((size_t)L.rows_cap * F);
    L.sh = take(sizeof(float) * L.rows_cap);
    L.slots = take(sizeof(float) * TK * d);
    L.total = R.off;
    L.guards = R.g;
    return L;
}

int forward_f8(const uint16_t* x, const float* router_W, const float* router_bias, const uint8_t* Q1, const float* S1,
               const uint8_t* Q3, const float* S3, const uint8_t* Q2, const float* S2, int64_t T, int64_t d,
               int64_t ffn, int n_experts, int top_k, uint16_t* y, int32_t* topk_ids, float* topk_w, void* workspace,
               size_t workspace_bytes, void* stream, int path) {
    if (!shape_ok(T, d, ffn, n_experts, top_k)) return JMOE_ERR_SHAPE;
    if (path != JMOE_PATH_AUTO && path != JMOE_PATH_GEMV && path != JMOE_PATH_GEMM) return JMOE_ERR_SHAPE;
    if (T == 0) return JMOE_OK;
    if (!x || !router_W || !Q1 || !S1 || !Q3 || !S3 || !Q2 || !S2 || !y || !workspace) return JMOE_ERR_NULL;
    const void* ptrs16[] = {x, Q1, Q3, Q2, y, router_W};
    for (const void* p : ptrs16)
        if (!aligned16(p)) return JMOE_ERR_ALIGN;
    const void* ptrs4[] = {router_bias, S1, S3, S2, topk_ids, topk_w};
    for (const void* p : ptrs4)
        if (reinterpret_cast<uintptr_t>(p) & 3) return JMOE_ERR_ALIGN;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return JMOE_ERR_WORKSPACE;
    const LayoutF8 L = make_layout_f8(T, d, ffn);
    if (workspace_bytes < L.total) return JMOE_ERR_WORKSPACE;

    char* ws = static_cast<char*>(workspace);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + L.hdr);
    int32_t* ids = reinterpret_cast<int32_t*>(ws + L.ids);
    float* wts = reinterpret_cast<float*>(ws + L.wts);
    int32_t* inv = reinterpret_cast<int32_t*>(ws + L.inv);
    int32_t* perm = reinterpret_cast<int32_t*>(ws + L.perm);
    uint8_t* x8 = reinterpret_cast<uint8_t*>(ws + L.x8);
    float* sx = reinterpret_cast<float*>(ws + L.sx);
    uint8_t* x8_perm = reinterpret_cast<uint8_t*>(ws + L.x8_perm);
    uint16_t* h = reinterpret_cast<uint16_t*>(ws + L.h);
    uint8_t* h8 = reinterpret_cast<uint8_t*>(ws + L.h8);
    float* sh = reinterpret_cast<float*>(ws + L.sh);
    float* slots = reinterpret_cast<float*>(ws + L.slots);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int sms = num_sms_current();
    if (path == JMOE_PATH_AUTO) path = (T <= kGemvMaxTokens) ? JMOE_PATH_GEMV : JMOE_PATH_GEMM;

    const int64_t TK = T * kTopK;
    cudaError_t e = debug_step(kAtStart, ws, L.guards, hdr, ids, perm, inv, TK, L.rows_cap, st);
    if (e != cudaSuccess) return JMOE_ERR_CUDA;
    {
        TimedLaunch t(JMOE_KERNEL_ROUTER, st);
        e = launch_router(x, router_W, router_bias, T, d, ids, wts, topk_ids, topk_w, st);
    }
    if (e != cudaSuccess) return JMOE_ERR_CUDA;
    if (debug_step(kAfterRouter, ws, L.guards, hdr, ids, perm, inv, TK, L.rows_cap, st) != cudaSuccess)
        return JMOE_ERR_CUDA;
    {
        TimedLaunch t(JMOE_KERNEL_PERMUTE, st);
        e = launch_permute(ids, T, hdr, perm, inv, st);
    }
    if (e != cudaSuccess) return JMOE_ERR_CUDA;
    if (debug_step(kAfterPermute, ws, L.guards, hdr, ids, perm, inv, TK, L.rows_cap, st) != cudaSuccess)
        return JMOE_ERR_CUDA;
    {
        TimedLaunch t(JMOE_KERNEL_ACT_QUANT, st);  // per-token E4M3 activations
        e = launch_quantize_fp8(x, T, d, x8, sx, nullptr, nullptr, st, sms);
    }
    if (e != cudaSuccess) return JMOE_ERR_CUDA;
    const int32_t* n_rows = &hdr->seg_start[kExperts];
    if (path == JMOE_PATH_GEMV) {
        {
            TimedLaunch t(JMOE_KERNEL_GEMV13, st);
            e = launch_gemv13_f8(hdr, perm, x8, sx, Q1, S1, Q3, S3, h, T, d, ffn, st);
        }
        if (e != cudaSuccess) return JMOE_ERR_CUDA;
        {
            TimedLaunch t(JMOE_KERNEL_ACT_QUANT, st);  // per-row E4M3 intermediate
            e = launch_quantize_fp8(h, L.rows_cap, ffn, h8, sh, perm, n_rows, st, sms);
        }
        if (e != cudaSuccess) return JMOE_ERR_CUDA;
        {
            TimedLaunch t(JMOE_KERNEL_GEMV2, st);
            e = launch_gemv2_f8(hdr, perm, h8, sh, Q2, S2, wts, slots, T, d, ffn, st);
        }
        if (e != cudaSuccess) return JMOE_ERR_CUDA;
    } else {
        {
            TimedLaunch t(JMOE_KERNEL_GATHER, st);  // E4M3 rows, moved as pairs of bytes
            e = launch_gather(reinterpret_cast<const uint16_t*>(x8), perm, hdr, d / 2, L.rows_cap,
                              reinterpret_cast<uint16_t*>(x8_perm), st, sms, false);
        }
        if (e != cudaSuccess) return JMOE_ERR_CUDA;
        {
            TimedLaunch t(JMOE_KERNEL_GEMM13, st);
            e = launch_gemm13_f8(hdr, perm, x8_perm, sx, Q1, S1, Q3, S3, h, L.rows_cap, d, ffn, st);
        }
        if (e != cudaSuccess) return JMOE_ERR_CUDA;
        {
            TimedLaunch t(JMOE_KERNEL_ACT_QUANT, st);
            e = launch_quantize_fp8(h, L.rows_cap, ffn, h8, sh, perm, n_rows, st, sms);
        }
        if (e != cudaSuccess) return JMOE_ERR_CUDA;
        {
            TimedLaunch t(JMOE_KERNEL_GEMM2, st);
            e = launch_gemm2_f8(hdr, perm, h8, sh, Q2, S2, wts, slots, L.rows_cap, d, ffn, st);
        }
        if (e != cudaSuccess) return JMOE_ERR_CUDA;
    }
    {
        TimedLaunch t(JMOE_KERNEL_COMBINE, st);
        e = launch_combine(slots, T, d, y, st, sms);
    }
    if (e != cudaSuccess) return JMOE_ERR_CUDA;
    return to_status(debug_step(kAtEnd, ws, L.guards, hdr, ids, perm, inv, TK, L.rows_cap, st));
}

}  // namespace

extern "C" {

int jamba_moe_quantize_fp8(const uint16_t* W, int64_t n_mats, int64_t rows, int64_t cols, uint8_t* Q, float* S,
                           void* stream) {
    if (!W || !Q || !S) return JMOE_ERR_NULL;
    if (n_mats < 1 || rows < 1 || cols < 16 || cols > (int64_t(1) << 20) || cols % 16 != 0) return JMOE_ERR_SHAPE;
    if (n_mats > (int64_t(1) << 40) / rows) return JMOE_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(Q) || (reinterpret_cast<uintptr_t>(S) & 3)) return JMOE_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    TimedLaunch t(JMOE_KERNEL_QUANTIZE, st);
    return to_status(launch_quantize_fp8(W, n_mats * rows, cols, Q, S, nullptr, nullptr, st, num_sms_current()));
}

size_t jamba_moe_workspace_size_fp8(int64_t T, int64_t d, int64_t ffn, int n_experts, int top_k) {
    if (!shape_ok(T, d, ffn, n_experts, top_k)) return 0;
    return make_layout_f8(T, d, ffn).total;
}

int jamba_moe_forward_fp8(const uint16_t* x, const float* router_W, const float* router_bias, const uint8_t* Q1,
                          const float* S1, const uint8_t* Q3, const float* S3, const uint8_t* Q2, const float* S2,
                          int64_t T, int64_t d, int64_t ffn, int n_experts, int top_k, uint16_t* y, int32_t* topk_ids,
                          float* topk_w, void* workspace, size_t workspace_bytes, void* stream, int path) {
    return forward_f8(x, router_W, router_bias, Q1, S1, Q3, S3, Q2, S2, T, d, ffn, n_experts, top_k, y, topk_ids,
                      topk_w, workspace, workspace_bytes, stream, path);
}

}  // extern "C"

extern "C" {

size_t jamba_mlp_workspace_size(int64_t T, int64_t d, int64_t ffn) {
    if (!shape_ok(T, d, ffn, kExperts, kTopK)) return 0;
    return make_layout_mlp(T, d, ffn).total;
}

int jamba_mlp_forward_path(const uint16_t* x, const int8_t* Q1, const float* S1, const int8_t* Q3, const float* S3,
                           const int8_t* Q2, const float* S2, int64_t T, int64_t d, int64_t ffn, uint16_t* y,
                           void* workspace, size_t workspace_bytes, void* stream, int path) {
    return mlp_impl(x, Q1, S1, Q3, S3, Q2, S2, T, d, ffn, y, workspace, workspace_bytes, stream, path);
}

int jamba_mlp_forward(const uint16_t* x, const int8_t* Q1, const float* S1, const int8_t* Q3, const float* S3,
                      const int8_t* Q2, const float* S2, int64_t T, int64_t d, int64_t ffn, uint16_t* y,
                      void* workspace, size_t workspace_bytes, void* stream) {
    return mlp_impl(x, Q1, S1, Q3, S3, Q2, S2, T, d, ffn, y, workspace, workspace_bytes, stream, JMOE_PATH_AUTO);
}

int jamba_moe_forward_path(const uint16_t* x, const float* router_W, const float* router_bias, const int8_t* Q1,
                           const float* S1, const int8_t* Q3, const float* S3, const int8_t* Q2, const float* S2,
                           int64_t T, int64_t d, int64_t ffn, int n_experts, int top_k, uint16_t* y,
                           int32_t* topk_ids, float* topk_w, void* workspace, size_t workspace_bytes, void* stream,
                           int path) {
    return forward_impl(x, router_W, router_bias, Q1, S1, Q3, S3, Q2, S2, true, T, d, ffn, n_experts, top_k, y,
                        topk_ids, topk_w, workspace, workspace_bytes, stream, path);
}

int jamba_moe_forward_bf16w(const uint16_t* x, const float* router_W, const float* router_bias, const uint16_t* W1,
                            const uint16_t* W3, const uint16_t* W2, int64_t T, int64_t d, int64_t ffn, int n_experts,
                            int top_k, uint16_t* y, int32_t* topk_ids, float* topk_w, void* workspace,
                            size_t workspace_bytes, void* stream, int path) {
    return forward_impl(x, router_W, router_bias, W1, nullptr, W3, nullptr, W2, nullptr, false, T, d, ffn, n_experts,
                        top_k, y, topk_ids, topk_w, workspace, workspace_bytes, stream, path);
}

int jamba_moe_forward(const uint16_t* x, const float* router_W, const float* router_bias, const int8_t* Q1,
                      const float* S1, const int8_t* Q3, const float* S3, const int8_t* Q2, const float* S2,
                      int64_t T, int64_t d, int64_t ffn, int n_experts, int top_k, uint16_t* y, int32_t* topk_ids,
                      float* topk_w, void* workspace, size_t workspace_bytes, void* stream) {
    return jamba_moe_forward_path(x, router_W, router_bias, Q1, S1, Q3, S3, Q2, S2, T, d, ffn, n_experts, top_k, y,
                                  topk_ids, topk_w, workspace, workspace_bytes, stream, JMOE_PATH_AUTO);
}

int jamba_moe_read_device_status(const void* workspace, void* stream) {
    if (!workspace) return JMOE_ERR_NULL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t status = 0;
    if (cudaMemcpyAsync(&status, workspace, sizeof(status), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return JMOE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return JMOE_ERR_CUDA;
    return (int)status;
}

const char* jamba_moe_status_string(int status) {
    switch (status) {
        case JMOE_OK: return "ok";
        case JMOE_ERR_NULL: return "a required pointer is NULL";
        case JMOE_ERR_SHAPE: return "unsupported or inconsistent sizes";
        case JMOE_ERR_WORKSPACE: return "workspace too small or not 256-byte aligned";
        case JMOE_ERR_CUDA: return "CUDA runtime call or kernel launch failed";
        case JMOE_DEV_TIMEOUT: return "a kernel gave up waiting on a pipeline barrier";
        case JMOE_DEV_BAD_INDEX: return "a kernel saw an out-of-range routing index";
        case JMOE_ERR_ALIGN: return "a pointer is not 16-byte aligned";
        case JMOE_DEV_BAD_TABLE: return "a debug check found inconsistent routing tables";
        case JMOE_DEV_CANARY: return "a debug check found a workspace guard gap overwritten";
        default: return "unknown status";
    }
}

int jamba_moe_debug_checks(int on) {
    g_debug_checks = on ? 1 : 0;
    return JMOE_OK;
}

int jamba_moe_debug_corrupt(int what) {
    if (what < 0 || what > JMOE_CORRUPT_CANARY) return JMOE_ERR_SHAPE;
    g_corrupt = what;
    return JMOE_OK;
}

int jamba_moe_timing_start(int max_launches) {
    for (cudaEvent_t ev : g_timing.start) cudaEventDestroy(ev);
    for (cudaEvent_t ev : g_timing.stop) cudaEventDestroy(ev);
    g_timing.start.clear();
    g_timing.stop.clear();
    g_timing.kind.clear();
    g_timing.used = 0;
    g_timing.on = false;
    if (max_launches <= 0) return JMOE_OK;
    g_timing.start.resize(max_launches);
    g_timing.stop.resize(max_launches);
    g_timing.kind.assign(max_launches, -1);
    for (int i = 0; i < max_launches; ++i) {
        if (cudaEventCreate(&g_timing.start[i]) != cudaSuccess || cudaEventCreate(&g_timing.stop[i]) != cudaSuccess) {
            g_timing.start.resize(i);
            g_timing.stop.resize(i);
            return JMOE_ERR_CUDA;
        }
    }
    g_timing.on = true;
    return JMOE_OK;
}

int jamba_moe_timing_collect(double* total_ms, int64_t* launches, int n_kinds) {
    if (!total_ms || !launches || n_kinds < 0) return -JMOE_ERR_NULL;
    const int n = n_kinds < JMOE_KERNEL_KINDS ? n_kinds : JMOE_KERNEL_KINDS;
    for (int k = 0; k < n; ++k) {
        total_ms[k] = 0.0;
        launches[k] = 0;
    }
    for (int i = 0; i < g_timing.used; ++i) {
        if (cudaEventSynchronize(g_timing.stop[i]) != cudaSuccess) return -JMOE_ERR_CUDA;
        float ms = 0.0f;
        if (cudaEventElapsedTime(&ms, g_timing.start[i], g_timing.stop[i]) != cudaSuccess) return -JMOE_ERR_CUDA;
        const int k = g_timing.kind[i];
        if (k >= 0 && k < n) {
            total_ms[k] += ms;
            launches[k] += 1;
        }
    }
    return n;
}

const char* jamba_moe_kernel_name(int kind) {
    static const char* names[JMOE_KERNEL_KINDS] = {"quantize", "router", "permute", "gather", "gemv13",
                                                   "gemv2", "gemm13", "gemm2", "combine", "act_quant"};
    return (kind >= 0 && kind < JMOE_KERNEL_KINDS) ? names[kind] : "unknown";
}

}  // extern "C"

// ---------------------------------------------------------------- expert parallelism (ep.cu)
namespace jmoe {
cudaError_t launch_permute_tk(const int32_t* ids, int64_t TK, int n_valid, WsHeader* hdr, int32_t* perm, int32_t* inv,
                              cudaStream_t st);
cudaError_t launch_ep_pack(const uint16_t* x, const WsHeader* hdr, const int32_t* perm, const float* wts, int64_t d,
                           int64_t rows_cap, int experts_per_rank, int n_ranks, uint16_t* send_x, int32_t* send_e,
                           float* send_w, int32_t* pos, int32_t* send_counts, cudaStream_t st, int num_sms);
cudaError_t launch_ep_combine(const float* ret, const int32_t* pos, int64_t T, int64_t d, uint16_t* y, cudaStream_t st,
                              int num_sms);
}  // namespace jmoe

namespace {

bool ranks_ok(int n_ranks) { return n_ranks >= 1 && n_ranks <= kExperts && kExperts % n_ranks == 0; }

// Dispatch workspace: routing tables of the rank's own tokens.
Layout make_layout_ep_dispatch(int64_t T) {
    Layout L{};
    const int64_t TK = T * kTopK;
    L.rows_cap = (TK + int64_t(kExperts) * (kRowPad - 1) + kRowPad - 1) / kRowPad * kRowPad;
    Regions R;
    L.hdr = R.take(kHeaderBytes);
    L.ids = R.take(sizeof(int32_t) * TK);
    L.wts = R.take(sizeof(float) * TK);
    L.inv = R.take(sizeof(int32_t) * TK);
    L.perm = R.take(sizeof(int32_t) * L.rows_cap);
    L.total = R.off;
    L.guards = R.g;
    return L;
}

// Expert workspace: the received rows' routing tables, permuted rows and SwiGLU intermediate.
Layout make_layout_ep_experts(int64_t N, int64_t d, int64_t F) {
    Layout L{};
    L.rows_cap = (N + int64_t(kExperts) * (kRowPad - 1) + kRowPad - 1) / kRowPad * kRowPad;
    Regions R;
    L.hdr = R.take(kHeaderBytes);
    L.inv = R.take(sizeof(int32_t) * (N > 0 ? N : 1));
    L.perm = R.take(sizeof(int32_t) * L.rows_cap);
    L.x_perm = R.take(sizeof(uint16_t) * L.rows_cap * d);
    L.h = R.take(sizeof(uint16_t) * L.rows_cap * F);
    L.total = R.off;
    L.guards = R.g;
    return L;
}

}  // namespace

extern "C" {

size_t jamba_moe_ep_dispatch_workspace_size(int64_t T, int64_t d, int n_experts, int top_k) {
    if (!shape_ok(T, d, 128, n_experts, top_k)) return 0;
    return make_layout_ep_dispatch(T).total;
}

int jamba_moe_ep_dispatch(const uint16_t* x, const float* router_W, const float* router_bias, int64_t T, int64_t d,
                          int n_experts, int top_k, int n_ranks, uint16_t* send_x, int32_t* send_expert,
                          float* send_w, int32_t* send_counts, int32_t* pos, int32_t* topk_ids, float* topk_w,
                          void* workspace, size_t workspace_bytes, void* stream) {
    if (!shape_ok(T, d, 128, n_experts, top_k) || !ranks_ok(n_ranks)) return JMOE_ERR_SHAPE;
    if (!send_counts) return JMOE_ERR_NULL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) return to_status(cudaMemsetAsync(send_counts, 0, sizeof(int32_t) * n_ranks, st));
    if (!x || !router_W || !send_x || !send_expert || !send_w || !pos || !workspace) return JMOE_ERR_NULL;
    if (!aligned16(x) || !aligned16(router_W) || !aligned16(send_x)) return JMOE_ERR_ALIGN;
    const void* ptrs4[] = {router_bias, send_expert, send_w, send_counts, pos, topk_ids, topk_w};
    for (const void* p : ptrs4)
        if (reinterpret_cast<uintptr_t>(p) & 3) return JMOE_ERR_ALIGN;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return JMOE_ERR_WORKSPACE;
    const Layout L = make_layout_ep_dispatch(T);
    if (workspace_bytes < L.total) return JMOE_ERR_WORKSPACE;
    char* ws = static_cast<char*>(workspace);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + L.hdr);
    int32_t* ids = reinterpret_cast<int32_t*>(ws + L.ids);
    float* wts = reinterpret_cast<float*>(ws + L.wts);
    int32_t* inv = reinterpret_cast<int32_t*>(ws + L.inv);
    int32_t* perm = reinterpret_cast<int32_t*>(ws + L.perm);
    cudaError_t e;
    {
        TimedLaunch t(JMOE_KERNEL_ROUTER, st);
        e = launch_router(x, router_W, router_bias, T, d, ids, wts, topk_ids, topk_w, st);
    }
    if (e != cudaSuccess) return JMOE_ERR_CUDA;
    {
        TimedLaunch t(JMOE_KERNEL_PERMUTE, st);
        e = launch_permute(ids, T, hdr, perm, inv, st);
    }
    if (e != cudaSuccess) return JMOE_ERR_CUDA;
    TimedLaunch t(JMOE_KERNEL_GATHER, st);
    return to_status(launch_ep_pack(x, hdr, perm, wts, d, L.rows_cap, kExperts / n_ranks, n_ranks, send_x, send_expert,
                                    send_w, pos, send_counts, st, num_sms_current()));
}

size_t jamba_moe_ep_experts_workspace_size(int64_t N, int64_t d, int64_t ffn) {
    if (!shape_ok(N, d, ffn, kExperts, kTopK)) return 0;
    return make_layout_ep_experts(N, d, ffn).total;
}

int jamba_moe_ep_experts(const uint16_t* xr, const int32_t* expert, const float* w, int64_t N, int64_t d, int64_t ffn,
                         int n_local, const int8_t* Q1, const float* S1, const int8_t* Q3, const float* S3,
                         const int8_t* Q2, const float* S2, float* out, void* workspace, size_t workspace_bytes,
                         void* stream, int path) {
    if (!shape_ok(N, d, ffn, kExperts, kTopK) || n_local < 1 || n_local > kExperts) return JMOE_ERR_SHAPE;
    if (path != JMOE_PATH_AUTO && path != JMOE_PATH_GEMV && path != JMOE_PATH_GEMM) return JMOE_ERR_SHAPE;
    if (N == 0) return JMOE_OK;
    if (!xr || !expert || !w || !Q1 || !S1 || !Q3 || !S3 || !Q2 || !S2 || !out || !workspace) return JMOE_ERR_NULL;
    const void* ptrs16[] = {xr, Q1, Q3, Q2, out};
    for (const void* p : ptrs16)
        if (!aligned16(p)) return JMOE_ERR_ALIGN;
    const void* ptrs4[] = {expert, w, S1, S3, S2};
    for (const void* p : ptrs4)
        if (reinterpret_cast<uintptr_t>(p) & 3) return JMOE_ERR_ALIGN;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return JMOE_ERR_WORKSPACE;
    const Layout L = make_layout_ep_experts(N, d, ffn);
    if (workspace_bytes < L.total) return JMOE_ERR_WORKSPACE;
    char* ws = static_cast<char*>(workspace);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + L.hdr);
    int32_t* inv = reinterpret_cast<int32_t*>(ws + L.inv);
    int32_t* perm = reinterpret_cast<int32_t*>(ws + L.perm);
    uint16_t* x_perm = reinterpret_cast<uint16_t*>(ws + L.x_perm);
    uint16_t* h = reinterpret_cast<uint16_t*>(ws + L.h);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // one assignment per received row (k_div = 1); the GEMV pass width follows the rows per local
    // expert, given to the launcher as the token count whose K assignments spread over 16 experts
    const int64_t rows_per_expert = (N + n_local - 1) / n_local;
    const int64_t T_equiv = (rows_per_expert * kExperts + kTopK - 1) / kTopK;
    if (path == JMOE_PATH_AUTO) path = (T_equiv <= kGemvMaxTokens) ? JMOE_PATH_GEMV : JMOE_PATH_GEMM;
    cudaError_t e;
    {
        TimedLaunch t(JMOE_KERNEL_PERMUTE, st);
        e = launch_permute_tk(expert, N, n_local, hdr, perm, inv, st);
    }
    if (e != cudaSuccess) return JMOE_ERR_CUDA;
    if (path == JMOE_PATH_GEMV) {
        {
            TimedLaunch t(JMOE_KERNEL_GEMV13, st);
            e = launch_gemv13(hdr, perm, xr, Q1, S1, Q3, S3, h, T_equiv, d, ffn, st, 1);
        }
        if (e != cudaSuccess) return JMOE_ERR_CUDA;
        TimedLaunch t(JMOE_KERNEL_GEMV2, st);
        return to_status(launch_gemv2(hdr, perm, h, Q2, S2, w, out, T_equiv, d, ffn, st));
    }
    {
        TimedLaunch t(JMOE_KERNEL_GATHER, st);
        e = launch_gather(xr, perm, hdr, d, L.rows_cap, x_perm, st, num_sms_current(), true, 1);
    }
    if (e != cudaSuccess) return JMOE_ERR_CUDA;
    {
        TimedLaunch t(JMOE_KERNEL_GEMM13, st);
        e = launch_gemm13(hdr, perm, x_perm, Q1, S1, Q3, S3, h, L.rows_cap, d, ffn, st, n_local);
    }
    if (e != cudaSuccess) return JMOE_ERR_CUDA;
    TimedLaunch t(JMOE_KERNEL_GEMM2, st);
    return to_status(launch_gemm2(hdr, perm, h, Q2, S2, w, out, L.rows_cap, d, ffn, st, n_local, nullptr));
}

int jamba_moe_ep_combine(const float* ret, const int32_t* pos, int64_t T, int64_t d, uint16_t* y, void* stream) {
    if (!shape_ok(T, d, 128, kExperts, kTopK)) return JMOE_ERR_SHAPE;
    if (T == 0) return JMOE_OK;
    if (!ret || !pos || !y) return JMOE_ERR_NULL;
    if (!aligned16(ret) || !aligned16(y) || (reinterpret_cast<uintptr_t>(pos) & 3)) return JMOE_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    TimedLaunch t(JMOE_KERNEL_COMBINE, st);
    return to_status(launch_ep_combine(ret, pos, T, d, y, st, num_sms_current()));
}

}  // extern "C"
