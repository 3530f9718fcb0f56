/*
 * jmoe.h — C ABI of the ExpertsInt8 mixture-of-experts layer for NVIDIA B200 (sm_100a).
 *
 * The layer (Jamba-1.5: Hybrid Transformer-Mamba Models at Scale, "Model Architecture":
 * n = 16 experts, two of them serving every token; §3.1 "ExpertsInt8": expert weights are kept
 * as 8-bit integer codes and converted into BF16 inside the expert GEMM kernel just before the
 * matrix math) computes, for every token x_t (a row of d bf16 values):
 *
 *     z_e   = sum_i x_ti * Wr[e][i] (+ b_e)                  router logits, fp32
 *     p     = softmax(z)                                      over all 16 experts
 *     e_t1, e_t2 = the two largest logits, in descending order
 *     y_t   = p_{e_t1} * E_{e_t1}(x_t) + p_{e_t2} * E_{e_t2}(x_t)   (weights not renormalised)
 *     E_e(x) = W2_e ( SiLU(W1_e x) * (W3_e x) )               SwiGLU expert
 *
 * with W1_e, W3_e: [ffn][d] and W2_e: [d][ffn] held as int8 codes Q plus one fp32 scale S per
 * output row (W[r][c] ~= Q[r][c] * S[r]).
 *
 * Conventions for every call below
 *   - "bf16" buffers are arrays of uint16_t holding bfloat16 bit patterns.
 *   - Every pointer is a DEVICE pointer owned by the caller, unless a comment says otherwise.
 *     The library allocates no device memory, never synchronises the stream (except where
 *     stated) and launches its kernels only on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream).
 *   - Tensors are dense, row-major, with the last dimension contiguous.  Activation, weight and
 *     output pointers must be 16-byte aligned; scale, bias and routing-output pointers 4-byte
 *     aligned; workspaces 256-byte aligned (JMOE_ERR_ALIGN / JMOE_ERR_WORKSPACE otherwise).
 *   - Calls return a jmoe_status.  Argument errors are detected on the host before anything is
 *     launched and leave all buffers untouched.  Launch failures return JMOE_ERR_CUDA.  No call
 *     aborts, throws or prints.
 *   - Calls are asynchronous: results are ready when `stream` reaches the point of the call.
 *   - Host threads: the quantize, workspace-size and forward calls may be made from several
 *     threads at once (each with its own workspace and outputs); the timing calls, the test hooks
 *     and jamba_moe_forward_noalloc (one shared scratch array) may not.
 *   - Supported shapes: n_experts == 16, top_k == 2, d and ffn multiples of 128 with
 *     128 <= d, ffn <= 32768, 0 <= T <= 1048576.  Anything else returns JMOE_ERR_SHAPE.
 *   - T = 0 (no token) is valid for every forward call but jamba_moe_forward_noalloc: it returns
 *     JMOE_OK at once, after the size checks, without touching any pointer (they may be NULL) and
 *     without launching anything.
 */
#ifndef JMOE_H
#define JMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    JMOE_OK = 0,
    JMOE_ERR_NULL = 1,       /* a required pointer is NULL */
    JMOE_ERR_SHAPE = 2,      /* unsupported or inconsistent sizes */
    JMOE_ERR_WORKSPACE = 3,  /* workspace too small or misaligned */
    JMOE_ERR_CUDA = 4,       /* a CUDA runtime call or kernel launch failed */
    JMOE_DEV_TIMEOUT = 5,    /* a kernel gave up waiting on a pipeline barrier (device status) */
    JMOE_DEV_BAD_INDEX = 6,  /* a kernel saw an out-of-range routing index (device status) */
    JMOE_ERR_ALIGN = 7,      /* a pointer is not 16-byte aligned */
    JMOE_DEV_BAD_TABLE = 8,  /* debug checks: the routing tables are not a valid permutation (device status) */
    JMOE_DEV_CANARY = 9      /* debug checks: a workspace guard gap was overwritten (device status) */
} jmoe_status;

/* Forward-path selection for jamba_moe_forward_path. */
enum {
    JMOE_PATH_AUTO = 0,  /* decode GEMV path when T <= 128, grouped tensor-core GEMM otherwise */
    JMOE_PATH_GEMV = 1,  /* weight-streaming path for few tokens per expert */
    JMOE_PATH_GEMM = 2   /* tcgen05 grouped GEMM path (prefill) */
};

/*
 * jamba_moe_quantize — ExpertsInt8 weight quantization (Jamba-1.5 paper, §3.1: weights are
 * quantized to INT8 at model loading, without calibration).
 *
 *   W: bf16 [n_mats][rows][cols]   input weights, out x in (one row per output channel)
 *   Q: int8 [n_mats][rows][cols]   output codes
 *   S: fp32 [n_mats][rows]         output scales, one per row
 *
 * For each row r: amax = max_c |W[r][c]|; S[r] = amax / 127 (fp32, round to nearest even);
 * Q[r][c] = the integer nearest to W[r][c] / S[r] (exact quotient; halfway cases to even),
 * within [-127, 127].  A row of zeros gets S = 1 and Q = 0.  The scale granularity (per output
 * channel), the symmetric range and the rounding rule are this library's reading of what the
 * page leaves open.  Results are bit-exact and deterministic.
 * Sizes: n_mats >= 1, 1 <= rows, 16 <= cols <= 1<<20 with cols % 16 == 0; W, Q 16-byte aligned.
 */
int jamba_moe_quantize(const uint16_t* W, int64_t n_mats, int64_t rows, int64_t cols, int8_t* Q, float* S,
                       void* stream);

/*
 * jamba_moe_workspace_size — bytes of device scratch jamba_moe_forward needs for these sizes
 * (routing tables, the permuted activations, the SwiGLU intermediate and the per-slot
 * outputs).  Returns 0 for unsupported sizes.  Host only; touches no device.
 */
size_t jamba_moe_workspace_size(int64_t T, int64_t d, int64_t ffn, int n_experts, int top_k);

/*
 * jamba_moe_forward — the MoE layer on T tokens (formula at the top of this file).
 *
 *   x:           bf16 [T][d]                 activations
 *   router_W:    fp32 [n_experts][d]         router weight
 *   router_bias: fp32 [n_experts] or NULL    added to the logits (NULL = no bias)
 *   Q1, Q3:      int8 [n_experts][ffn][d]    with S1, S3 fp32 [n_experts][ffn]  (gate, up)
 *   Q2:          int8 [n_experts][d][ffn]    with S2 fp32 [n_experts][d]        (down)
 *   y:           bf16 [T][d]                 output (written)
 *   topk_ids:    int32 [T][top_k] or NULL    chosen experts, descending logit (written if given)
 *   topk_w:      fp32 [T][top_k] or NULL     their softmax probabilities (written if given)
 *   workspace:   device scratch of at least jamba_moe_workspace_size(...) bytes, 256-byte
 *                aligned, owned by the caller; its contents on entry do not matter.  One
 *                workspace must not be used by two calls that may overlap on the GPU.
 *
 * Numerics: router in fp32; int8 codes converted exactly to bf16 inside the GEMM kernels,
 * bf16 x bf16 products accumulated in fp32, per-row scales applied to the fp32 accumulators;
 * the SwiGLU intermediate is rounded to bf16; the two weighted expert outputs of a token are
 * added in fp32 in a fixed order (slot 0 then slot 1) and rounded once to bf16.  The result
 * is deterministic (no floating-point atomics).  Experts that receive no token are skipped and
 * their weights are not read.
 */
int jamba_moe_forward(const uint16_t* x, const float* router_W, const float* router_bias, const int8_t* Q1,
                      const float* S1, const int8_t* Q3, const float* S3, const int8_t* Q2, const float* S2,
                      int64_t T, int64_t d, int64_t ffn, int n_experts, int top_k, uint16_t* y,
                      int32_t* topk_ids, float* topk_w, void* workspace, size_t workspace_bytes, void* stream);

/*
 * jamba_moe_forward_path — jamba_moe_forward with the expert-GEMM path chosen explicitly
 * (JMOE_PATH_*).  Both paths compute the same function; tests use this to run each path on
 * every shape.  An unknown path value returns JMOE_ERR_SHAPE.
 */
int jamba_moe_forward_path(const uint16_t* x, const float* router_W, const float* router_bias,
                           const int8_t* Q1, const float* S1, const int8_t* Q3, const float* S3,
                           const int8_t* Q2, const float* S2, int64_t T, int64_t d, int64_t ffn, int n_experts,
                           int top_k, uint16_t* y, int32_t* topk_ids, float* topk_w, void* workspace,
                           size_t workspace_bytes, void* stream, int path);

/*
 * jamba_moe_forward_bf16w — the same layer with unquantized bf16 expert weights (no ExpertsInt8):
 * W1, W3 bf16 [n_experts][ffn][d], W2 bf16 [n_experts][d][ffn]; everything else as in
 * jamba_moe_forward_path (same workspace size, same paths, same numerics minus the scales).  It
 * is the comparator the Jamba-1.5 paper measures ExpertsInt8 against (§3.1 reports ExpertsInt8 at
 * no extra latency, even slightly faster, than BF16 weights): here the decode path streams twice
 * the weight bytes, and the prefill path loads the weight tiles straight into the MMA's layout
 * without conversion.
 */
int jamba_moe_forward_bf16w(const uint16_t* x, const float* router_W, const float* router_bias,
                            const uint16_t* W1, const uint16_t* W3, const uint16_t* W2, int64_t T, int64_t d,
                            int64_t ffn, int n_experts, int top_k, uint16_t* y, int32_t* topk_ids, float* topk_w,
                            void* workspace, size_t workspace_bytes, void* stream, int path);

/*
 * FP8 comparator layer.  The Jamba-1.5 paper (§3.1) compares ExpertsInt8 with FP8 serving (on H100,
 * the two run with equal latency; FP8 needs FP8 hardware and, unlike ExpertsInt8, does not keep
 * BF16 activations) without defining the FP8 scheme.  This library's reading: both GEMM operands
 * are OCP FP8 E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no infinities, largest
 * finite 448, subnormals m * 2^-9); weights carry one fp32 scale per output channel, the
 * activations x one dynamic fp32 scale per token and the SwiGLU intermediate one per expert row
 * (scale = amax / 448 in fp32, code = the E4M3 value nearest to the exact quotient, ties to the
 * even code, saturating at +-448; a row of zeros gets scale 1).  Router and combine as in
 * jamba_moe_forward.
 *
 * jamba_moe_quantize_fp8 — as jamba_moe_quantize with E4M3 codes: Q uint8 [n_mats][rows][cols].
 * Bit-exact and deterministic.
 */
int jamba_moe_quantize_fp8(const uint16_t* W, int64_t n_mats, int64_t rows, int64_t cols, uint8_t* Q, float* S,
                           void* stream);

/* jamba_moe_workspace_size_fp8 — device scratch bytes of jamba_moe_forward_fp8 (0: unsupported sizes). */
size_t jamba_moe_workspace_size_fp8(int64_t T, int64_t d, int64_t ffn, int n_experts, int top_k);

/*
 * jamba_moe_forward_fp8 — the FP8 layer: arguments as jamba_moe_forward_path, with Q1, Q3
 * uint8 [n_experts][ffn][d] and Q2 uint8 [n_experts][d][ffn] E4M3 codes from
 * jamba_moe_quantize_fp8 and their scales.  x is quantized per token, the fp32 SwiGLU output of
 * the first GEMM per expert row; the GEMMs multiply E4M3 by E4M3 with fp32 accumulation (tcgen05
 * kind::f8f6f4 on the tensor-core path, mma.sync e4m3 on the decode path) and apply the weight and
 * activation scales to the fp32 totals.  Deterministic; errors as jamba_moe_forward.
 */
int jamba_moe_forward_fp8(const uint16_t* x, const float* router_W, const float* router_bias, const uint8_t* Q1,
                          const float* S1, const uint8_t* Q3, const float* S3, const uint8_t* Q2, const float* S2,
                          int64_t T, int64_t d, int64_t ffn, int n_experts, int top_k, uint16_t* y,
                          int32_t* topk_ids, float* topk_w, void* workspace, size_t workspace_bytes, void* stream,
                          int path);

/*
 * jamba_mlp_workspace_size — bytes of device scratch jamba_mlp_forward needs for these sizes.
 * Returns 0 for unsupported sizes.  Host only; touches no device.
 */
size_t jamba_mlp_workspace_size(int64_t T, int64_t d, int64_t ffn);

/*
 * jamba_mlp_forward — the dense MLP of the layers without MoE, on ExpertsInt8 weights (Jamba-1.5
 * paper, §3.1: the MLP weights are quantized and dequantized like the experts'; "Model
 * Architecture": one layer in e = 2 has an MoE block, the other an MLP):
 *
 *     y_t = bf16( S2 * (Q2 . h_t) ),  h_t = bf16( SiLU(S1 * (Q1 . x_t)) * (S3 * (Q3 . x_t)) )
 *
 *   x:       bf16 [T][d]                        activations
 *   Q1, Q3:  int8 [ffn][d] with S1, S3 fp32 [ffn]  (gate, up; from jamba_moe_quantize)
 *   Q2:      int8 [d][ffn] with S2 fp32 [d]        (down)
 *   y:       bf16 [T][d]                        output (written)
 *   workspace: device scratch of at least jamba_mlp_workspace_size(...) bytes, 256-byte aligned,
 *            owned by the caller, contents on entry irrelevant; not shared by overlapping calls.
 *
 * It runs the kernels of jamba_moe_forward as a layer of one expert that every token takes with
 * weight 1 (no router, no combine: the down-projection writes y in bf16 directly).  Numerics as
 * in jamba_moe_forward: exact int8 -> bf16, fp32 accumulation, scales on the accumulators, h in
 * bf16; deterministic.  Sizes: 0 <= T <= 1<<20, d and ffn multiples of 128 in [128, 32768];
 * x, y, Q1, Q3, Q2 16-byte aligned, scales 4-byte aligned.  Errors as in jamba_moe_forward.
 */
int jamba_mlp_forward(const uint16_t* x, const int8_t* Q1, const float* S1, const int8_t* Q3, const float* S3,
                      const int8_t* Q2, const float* S2, int64_t T, int64_t d, int64_t ffn, uint16_t* y,
                      void* workspace, size_t workspace_bytes, void* stream);

/* jamba_mlp_forward_path — jamba_mlp_forward with the path chosen explicitly (JMOE_PATH_*; AUTO
 * takes the weight-streaming path for T <= 64 tokens, the tensor-core GEMMs above). */
int jamba_mlp_forward_path(const uint16_t* x, const int8_t* Q1, const float* S1, const int8_t* Q3, const float* S3,
                           const int8_t* Q2, const float* S2, int64_t T, int64_t d, int64_t ffn, uint16_t* y,
                           void* workspace, size_t workspace_bytes, void* stream, int path);

/*
 * jamba_moe_read_device_status — synchronises `stream`, then returns the status word the
 * kernels of the last forward call on `workspace` left there: JMOE_OK, JMOE_DEV_TIMEOUT (a
 * pipeline wait ran out of its bounded number of polls; the kernel released its resources and
 * returned early, so y is not valid) or JMOE_DEV_BAD_INDEX.  JMOE_ERR_CUDA if the copy fails.
 */
int jamba_moe_read_device_status(const void* workspace, void* stream);

/* jamba_moe_status_string — static, human-readable text for a jmoe_status value (host only). */
const char* jamba_moe_status_string(int status);

/*
 * jamba_moe_debug_skip_copy — test hook for failure detection, off by default.  While `on` is
 * non-zero, the next forward calls on the tensor-core (prefill) path make CTA 0 of the W1/W3 GEMM
 * skip the copies of its second pipeline stage, with every wait bounded by a short poll limit:
 * the wait for those copies runs out, the kernel records JMOE_DEV_TIMEOUT in the workspace status
 * word, waits (bounded) for its other in-flight copies and MMAs, releases its tensor memory and
 * returns; the output of that call is not valid.  Nothing faults, traps or hangs, and the CUDA
 * context stays usable.  Host only; not thread-safe.
 */
int jamba_moe_debug_skip_copy(int on);

/*
 * jamba_moe_debug_checks — debug checks, off by default.  While `on` is non-zero, every MoE
 * forward call (jamba_moe_forward, _path, _bf16w, _fp8) also launches: at its start, a kernel that
 * fills the guard gaps the workspace layout leaves after each of its regions with a canary pattern;
 * after the permutation, a kernel that checks the routing tables (counts sum to T*K, every
 * expert's segment is its count rounded up to 128 rows, each permuted row holds -1 or an
 * assignment routed to that expert whose inverse entry points back at the row, so no assignment
 * is held twice); at its end, a kernel that checks the canaries.  A failed check sets
 * JMOE_DEV_BAD_TABLE or JMOE_DEV_CANARY in the status word (first error wins) and traps nothing.
 * Host only; not thread-safe.
 *
 * jamba_moe_debug_corrupt — test hook for those checks: the next MoE forward call (one shot)
 * corrupts its own state from the host, with in-bounds copies that no kernel can turn into a
 * memory fault:
 *   JMOE_CORRUPT_ROUTE_ID  after the router, routing id 0 := 0x7F7F7F7F (out of range: the
 *                          permutation kernel skips it and reports JMOE_DEV_BAD_INDEX);
 *   JMOE_CORRUPT_PERM_ROW  after the permutation, permuted row 1 := permuted row 0 (an assignment
 *                          held twice: the table check reports JMOE_DEV_BAD_TABLE);
 *   JMOE_CORRUPT_CANARY    before the final check, one byte of a guard gap (JMOE_DEV_CANARY).
 * The output of that call is not valid.  0 cancels a pending corruption.  Host only.
 */
enum { JMOE_CORRUPT_NONE = 0, JMOE_CORRUPT_ROUTE_ID = 1, JMOE_CORRUPT_PERM_ROW = 2, JMOE_CORRUPT_CANARY = 3 };
int jamba_moe_debug_checks(int on);
int jamba_moe_debug_corrupt(int what);

/*
 * jamba_moe_forward_noalloc — jamba_moe_forward on the decode (weight-streaming) path for callers
 * that cannot allocate device memory: code running inside a memory pool it does not own, a
 * serving process that must not call cudaMalloc after start-up (it synchronises the device and
 * can fail under fragmentation), or a plugin interface that only hands over inputs and outputs.
 * The pages describe no such entry point; it has no counterpart there.
 *
 * Arguments are those of jamba_moe_forward without the workspace.  The scratch is one static
 * device array of jamba_moe_noalloc_scratch_capacity() bytes (64 MiB), present on every GPU that
 * loads this library until the process exits.  Sizes needing more
 * (jamba_moe_noalloc_scratch_needed) return JMOE_ERR_WORKSPACE; other checks as in
 * jamba_moe_forward.  The first call on a device looks the array's address up with that device
 * current: make it before any stream capture.  Every call shares the array, which keeps the last
 * call's contents (each call clears what it needs cleared); calls that may overlap on the GPU
 * race on it.  Calls no cudaMalloc, cudaFree or allocating library routine.
 */
int jamba_moe_forward_noalloc(const uint16_t* x, const float* router_W, const float* router_bias,
                              const int8_t* Q1, const float* S1, const int8_t* Q3, const float* S3,
                              const int8_t* Q2, const float* S2, int64_t T, int64_t d, int64_t ffn, int n_experts,
                              int top_k, uint16_t* y, int32_t* topk_ids, float* topk_w, void* stream);
size_t jamba_moe_noalloc_scratch_capacity(void);
/* Scratch bytes jamba_moe_forward_noalloc needs for these sizes (0 = unsupported sizes). */
size_t jamba_moe_noalloc_scratch_needed(int64_t T, int64_t d, int64_t ffn);
/*
 * jamba_moe_noalloc_read_device_status — jamba_moe_read_device_status for the static scratch of
 * jamba_moe_forward_noalloc on the current device: synchronises `stream`, then returns the status
 * word its last call left there (JMOE_OK, JMOE_DEV_TIMEOUT or JMOE_DEV_BAD_INDEX); JMOE_ERR_CUDA
 * if the lookup or the 4-byte copy fails.  Allocates nothing.
 */
int jamba_moe_noalloc_read_device_status(void* stream);

/*
 * Expert parallelism over G ranks (one GPU each; Jamba-1.5 paper, "Model Architecture": with
 * ExpertsInt8, Jamba-1.5-Large is served on one machine of eight 80 GB GPUs; "Training
 * Infrastructure": expert parallelism).  Rank g (0 <= g < G, G divides 16) holds the int8
 * weights of experts [g*16/G, (g+1)*16/G) only, and its own batch of T tokens.  One layer call:
 *
 *   1. jamba_moe_ep_dispatch     router + permutation of the rank's tokens; rows of x packed in
 *                                send order (grouped by destination rank, then expert, then token)
 *   2. the caller's all-to-all   of send_counts, then of send_x / send_expert / send_w with those
 *                                counts (e.g. torch.distributed.all_to_all_single over NCCL)
 *   3. jamba_moe_ep_experts      the rank's experts on the N rows it received
 *   4. the caller's all-to-all   of `out` back, in reverse, into a buffer `ret` in send order
 *   5. jamba_moe_ep_combine      y[t] = bf16(ret[pos[t][0]] + ret[pos[t][1]])
 *
 * The rows cross the interconnect once each way; y equals jamba_moe_forward's up to the choice of
 * expert path (both are within the same tolerance of the exact layer), the two slots being added
 * in the same fixed order.
 *
 * jamba_moe_ep_dispatch — x bf16 [T][d], router as in jamba_moe_forward; n_ranks = G.  Writes
 * send_x bf16 [T*2][d], send_expert int32 [T*2] (expert index local to the destination rank),
 * send_w fp32 [T*2] (routing weight), send_counts int32 [G] (rows for each rank, in rank order:
 * the first send_counts[0] rows go to rank 0, ...), pos int32 [T][2] (the send row of each
 * assignment) and, if given, topk_ids / topk_w.  Only the first sum(send_counts) = 2T rows are
 * written.  T = 0 writes zero counts.  workspace: jamba_moe_ep_dispatch_workspace_size bytes.
 */
size_t jamba_moe_ep_dispatch_workspace_size(int64_t T, int64_t d, int n_experts, int top_k);
int jamba_moe_ep_dispatch(const uint16_t* x, const float* router_W, const float* router_bias, int64_t T, int64_t d,
                          int n_experts, int top_k, int n_ranks, uint16_t* send_x, int32_t* send_expert,
                          float* send_w, int32_t* send_counts, int32_t* pos, int32_t* topk_ids, float* topk_w,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * jamba_moe_ep_experts — the rank's n_local experts on N received rows: xr bf16 [N][d],
 * expert int32 [N] in [0, n_local) (other values are skipped and reported as JMOE_DEV_BAD_INDEX in
 * the workspace status word), w fp32 [N]; Q1, Q3 int8 [n_local][ffn][d], Q2 int8 [n_local][d][ffn]
 * with their scales.  out fp32 [N][d]: out[n] = w[n] * E_expert[n](xr[n]) with the numerics of
 * jamba_moe_forward (exact int8 -> bf16, fp32 accumulation, bf16 SwiGLU intermediate).  path as in
 * jamba_moe_forward_path (AUTO: weight streaming when the rows per local expert are few).
 * workspace: jamba_moe_ep_experts_workspace_size(N, d, ffn) bytes; N = 0 is a no-op.
 */
size_t jamba_moe_ep_experts_workspace_size(int64_t N, int64_t d, int64_t ffn);
int jamba_moe_ep_experts(const uint16_t* xr, const int32_t* expert, const float* w, int64_t N, int64_t d, int64_t ffn,
                         int n_local, const int8_t* Q1, const float* S1, const int8_t* Q3, const float* S3,
                         const int8_t* Q2, const float* S2, float* out, void* workspace, size_t workspace_bytes,
                         void* stream, int path);

/* jamba_moe_ep_combine — ret fp32 [T*2][d] (the outputs back in send order), pos from the
 * dispatch: y bf16 [T][d] = bf16(ret[pos[t][0]] + ret[pos[t][1]]), slot 0 then slot 1. */
int jamba_moe_ep_combine(const float* ret, const int32_t* pos, int64_t T, int64_t d, uint16_t* y, void* stream);

/*
 * Kernel timing (for the benchmark's roofline figures).
 * jamba_moe_timing_start(max_launches) makes every following launch of this library record a
 * pair of CUDA events on its stream, until max_launches pairs are recorded, and forgets any
 * earlier records; max_launches <= 0 switches recording off.  jamba_moe_timing_collect
 * synchronises those events and writes, for each kernel kind k < n_kinds (JMOE_KERNEL_*),
 * total_ms[k] (sum of event-measured durations) and launches[k]; it returns the number of
 * kinds written.  Host pointers.  Not thread-safe: one timing session per process.
 */
enum {
    JMOE_KERNEL_QUANTIZE = 0,
    JMOE_KERNEL_ROUTER = 1,
    JMOE_KERNEL_PERMUTE = 2,
    JMOE_KERNEL_GATHER = 3,
    JMOE_KERNEL_GEMV13 = 4,
    JMOE_KERNEL_GEMV2 = 5,
    JMOE_KERNEL_GEMM13 = 6,
    JMOE_KERNEL_GEMM2 = 7,
    JMOE_KERNEL_COMBINE = 8,
    JMOE_KERNEL_ACT_QUANT = 9, /* FP8 layer: per-row E4M3 quantization of x and of the intermediate h */
    JMOE_KERNEL_KINDS = 10
};
int jamba_moe_timing_start(int max_launches);
int jamba_moe_timing_collect(double* total_ms, int64_t* launches, int n_kinds);
const char* jamba_moe_kernel_name(int kind);

#ifdef __cplusplus
}
#endif

#endif /* JMOE_H */
