// jamba_moe_forward_noalloc: the MoE layer on the decode (weight-streaming) path for callers that
// cannot allocate device memory themselves — code that runs inside a memory pool it does not own,
// a host process that must not call cudaMalloc once serving has started (cudaMalloc synchronises
// the device and can fail under fragmentation), or a plugin boundary that only passes tensors in
// and out.  Its scratch lives in one file-scope __device__ array instead of a caller workspace.
//
// Facts a caller must know (also stated in include/jmoe.h):
//   - The array is kNoAllocScratchBytes (64 MiB) per GPU and exists on every GPU that loads this
//     library, from load until process exit.
//   - The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
//     that device current; make that first call before any stream capture.
//   - All calls share the array and it keeps the last call's contents.  Every byte a call reads
//     is written earlier in the same call (the permutation kernel rewrites the routing header,
//     status word included); the header is also cleared at the start of each call, as a defence.
//   - jamba_moe_noalloc_read_device_status reads the array's status word (the device-side error
//     report of the last call on the current device).
//   - Two calls that may overlap on the GPU (other streams, other host threads) race on the array.
//   - Sizes whose scratch does not fit return JMOE_ERR_WORKSPACE.
//   - No cudaMalloc, cudaFree or allocating library routine is called.
#include <mutex>

#include "common.cuh"

namespace jmoe {

cudaError_t launch_router(const uint16_t* x, const float* Wr, const float* bias, int64_t T, int64_t d,
                          int32_t* ids_ws, float* w_ws, int32_t* ids_user, float* w_user, cudaStream_t st);
cudaError_t launch_permute(const int32_t* ids, int64_t T, WsHeader* hdr, int32_t* perm, int32_t* inv,
                           cudaStream_t st);
cudaError_t launch_gemv13(const WsHeader* hdr, const int32_t* perm, const uint16_t* x, const int8_t* Q1,
                          const float* S1, const int8_t* Q3, const float* S3, uint16_t* h, int64_t T, int64_t d,
                          int64_t F, cudaStream_t st, int k_div = kTopK);
cudaError_t launch_gemv2(const WsHeader* hdr, const int32_t* perm, const uint16_t* h, const int8_t* Q2,
                         const float* S2, const float* wts, float* out_slot, int64_t T, int64_t d, int64_t F,
                         cudaStream_t st);
cudaError_t launch_combine(const float* slots, int64_t T, int64_t d, uint16_t* y, cudaStream_t st, int num_sms);

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {nullptr};
int g_sms[kMaxDevices] = {0};

inline size_t up256(size_t v) { return (v + 255) & ~size_t(255); }
inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
inline bool al4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3) == 0; }

// Device address of the static scratch on the current device, looked up once per device.
int scratch_for_current_device(void** addr, int* sms) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return JMOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return JMOE_ERR_CUDA;
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        g_scratch_addr[dev] = p;
        g_sms[dev] = n;
    }
    *addr = g_scratch_addr[dev];
    *sms = g_sms[dev];
    return JMOE_OK;
}

}  // namespace
}  // namespace jmoe

using namespace jmoe;

extern "C" size_t jamba_moe_noalloc_scratch_capacity(void) { return kNoAllocScratchBytes; }

extern "C" size_t jamba_moe_noalloc_scratch_needed(int64_t T, int64_t d, int64_t ffn) {
    if (T < 1 || T > (int64_t(1) << 20) || d < 128 || d > 32768 || d % 128 || ffn < 128 || ffn > 32768 || ffn % 128)
        return 0;
    const int64_t TK = T * kTopK;
    const int64_t rows = (TK + int64_t(kExperts) * (kRowPad - 1) + kRowPad - 1) / kRowPad * kRowPad;
    size_t n = up256(kHeaderBytes);
    n += 3 * up256(sizeof(int32_t) * TK);            // ids, weights, inverse permutation
    n += up256(sizeof(int32_t) * rows);              // permutation
    n += up256(sizeof(uint16_t) * rows * ffn);       // SwiGLU intermediate
    n += up256(sizeof(float) * TK * d);              // weighted per-slot outputs
    return n;
}

extern "C" int jamba_moe_forward_noalloc(const uint16_t* x, const float* router_W, const float* router_bias,
                                         const int8_t* Q1, const float* S1, const int8_t* Q3, const float* S3,
                                         const int8_t* Q2, const float* S2, int64_t T, int64_t d, int64_t ffn,
                                         int n_experts, int top_k, uint16_t* y, int32_t* topk_ids, float* topk_w,
                                         void* stream) {
    if (!x || !router_W || !Q1 || !S1 || !Q3 || !S3 || !Q2 || !S2 || !y) return JMOE_ERR_NULL;
    if (n_experts != kExperts || top_k != kTopK) return JMOE_ERR_SHAPE;
    const size_t need = jamba_moe_noalloc_scratch_needed(T, d, ffn);
    if (need == 0) return JMOE_ERR_SHAPE;
    if (need > kNoAllocScratchBytes) return JMOE_ERR_WORKSPACE;
    if (!al16(x) || !al16(Q1) || !al16(Q3) || !al16(Q2) || !al16(y) || !al16(router_W)) return JMOE_ERR_ALIGN;
    if (!al4(router_bias) || !al4(S1) || !al4(S3) || !al4(S2) || !al4(topk_ids) || !al4(topk_w)) return JMOE_ERR_ALIGN;

    void* base = nullptr;
    int sms = 148;
    const int rc = scratch_for_current_device(&base, &sms);
    if (rc != JMOE_OK) return rc;
    const int64_t TK = T * kTopK;
    const int64_t rows = (TK + int64_t(kExperts) * (kRowPad - 1) + kRowPad - 1) / kRowPad * kRowPad;
    char* p = static_cast<char*>(base);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(p);
    p += up256(kHeaderBytes);
    int32_t* ids = reinterpret_cast<int32_t*>(p);
    p += up256(sizeof(int32_t) * TK);
    float* wts = reinterpret_cast<float*>(p);
    p += up256(sizeof(float) * TK);
    int32_t* inv = reinterpret_cast<int32_t*>(p);
    p += up256(sizeof(int32_t) * TK);
    int32_t* perm = reinterpret_cast<int32_t*>(p);
    p += up256(sizeof(int32_t) * rows);
    uint16_t* h = reinterpret_cast<uint16_t*>(p);
    p += up256(sizeof(uint16_t) * rows * ffn);
    float* slots = reinterpret_cast<float*>(p);

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // defensive: the permutation kernel rewrites every header field the later kernels read, the
    // status word included, but a header left over from an earlier call is cleared all the same
    if (cudaMemsetAsync(hdr, 0, kHeaderBytes, st) != cudaSuccess) return JMOE_ERR_CUDA;
    if (launch_router(x, router_W, router_bias, T, d, ids, wts, topk_ids, topk_w, st) != cudaSuccess)
        return JMOE_ERR_CUDA;
    if (launch_permute(ids, T, hdr, perm, inv, st) != cudaSuccess) return JMOE_ERR_CUDA;
    if (launch_gemv13(hdr, perm, x, Q1, S1, Q3, S3, h, T, d, ffn, st) != cudaSuccess) return JMOE_ERR_CUDA;
    if (launch_gemv2(hdr, perm, h, Q2, S2, wts, slots, T, d, ffn, st) != cudaSuccess) return JMOE_ERR_CUDA;
    if (launch_combine(slots, T, d, y, st, sms) != cudaSuccess) return JMOE_ERR_CUDA;
    return JMOE_OK;
}

// The status word of the static scratch on the current device: what the kernels of the last
// jamba_moe_forward_noalloc call there reported (JMOE_OK, JMOE_DEV_TIMEOUT or JMOE_DEV_BAD_INDEX).
// Synchronises `stream` first; reads 4 bytes into a host variable, allocates nothing.
extern "C" int jamba_moe_noalloc_read_device_status(void* stream) {
    void* base = nullptr;
    int sms = 0;
    const int rc = scratch_for_current_device(&base, &sms);
    if (rc != JMOE_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t status = 0;
    if (cudaMemcpyAsync(&status, base, sizeof(status), cudaMemcpyDeviceToHost, st) != cudaSuccess) return JMOE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return JMOE_ERR_CUDA;
    return (int)status;
}
