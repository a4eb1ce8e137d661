/*
 * moe_q4.h -- C ABI of the B200 (sm_100a) 4-bit Mixture-of-Experts expert FFN.
 *
 * The layer computed here is the MoE part of the model in "A 35B
 * Hybrid-Attention Mixture-of-Experts Model on a 6GB 2011 GPU: Hand-Written
 * 4-bit CUDA Inference for Fermi" (Dutch technical summary,
 * gist.science/nl/paper/2606.24031):
 *   - Methodologie 1: the prefill runs a grouped 4-bit GEMM over the routed
 *     experts; the decode runs a W4A8 integer kernel (4-bit weights, 8-bit
 *     activations, integer multiply-adds).
 *   - Methodologie 2: weights are group-wise symmetric 4-bit (Q4_0 family),
 *     activations 8-bit, 128 experts per layer after pruning.
 *   - Methodologie 4: the whole prompt in one pass, so each expert's GEMM
 *     sees all of its tokens at once.
 *
 * Formats (the readings of the "Q4_0 family" and "8-bit activations"):
 *   Q4_0 block = 18 bytes: binary16 scale d (little endian), then qs[16];
 *     weight i<16 = low nibble of qs[i], weight i+16 = high nibble;
 *     value = (nibble - 8) * d.
 *   Q8_0 block = 32 int8 q plus a binary16 scale: d = amax/127 (binary32
 *     division), q = round-half-away-from-zero(x/d) (binary32 division),
 *     stored scale = binary16(d), nearest-even; all-zero block -> d = 0, q = 0.
 *
 * Layer: y[t] = sum_j w[t,j] * FFN_{idx[t,j]}(x[t]) + FFN_shared(x[t]), where
 *   logits = x.Wr^T (+ bias), idx = top-k (descending, ties to the lower
 *   expert index), w = softmax over the k chosen logits, and
 *   FFN_e(x) = Wd_e . Q8_0( silu(Wg_e . Q8_0(x)) * (Wu_e . Q8_0(x)) ).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers (except the *_host entry),
 *     row-major, owned by the caller.  The library never allocates, frees or
 *     synchronises; all work is enqueued on `stream` (NULL = legacy default
 *     stream) and faults surface at the caller's next synchronisation.
 *   - Pointers must be 16-byte aligned, workspaces 256-byte aligned.
 *   - hidden and ffn must be positive multiples of 256; 1 <= top_k <=
 *     min(n_experts, 16); 1 <= n_experts <= 256; 0 <= T <= 2^24.  T == 0 is
 *     a no-op that returns MOE_Q4_OK.
 *   - Inputs must be finite.  A binary16 scale that overflows (block amax >
 *     65504*127) is reported in the device status word, never by a trap.
 *   - The device must be compute capability 10.0 (B200, sm_100a).
 *   - Return value: MOE_Q4_OK (0) or a negative MOE_Q4_ERR_* code; nothing is
 *     enqueued when an argument check fails.
 */
#ifndef MOE_Q4_H
#define MOE_Q4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_q4_stream_t; /* a cudaStream_t */

enum {
    MOE_Q4_OK = 0,
    MOE_Q4_ERR_INVALID_ARG = -1, /* null pointer, T < 0 or too large, bad k/E */
    MOE_Q4_ERR_SHAPE = -2,       /* hidden or ffn not a positive multiple of 256 */
    MOE_Q4_ERR_ALIGN = -3,       /* pointer not 16-byte (workspace: 256-byte) aligned */
    MOE_Q4_ERR_WORKSPACE = -4,   /* workspace smaller than moe_q4_ffn_workspace_bytes() */
    MOE_Q4_ERR_ARCH = -5,        /* current device is not compute capability 10.0 */
    MOE_Q4_ERR_CUDA = -6,        /* a CUDA runtime call or kernel launch failed */
    MOE_Q4_ERR_OVERLAP = -7      /* output buffer overlaps an input */
};

/* Bits of the device status word (first uint32 of a workspace, or the
 * optional `status` argument): set with atomicOr, never cleared by the
 * library except at the start of a forward call (moe_q4_ffn_forward and its
 * variants clear it per call; moe_q4_stack_forward once per call, so it
 * accumulates over the layers). */
#define MOE_Q4_STATUS_SCALE_OVERFLOW 0x1u /* a binary16 Q8_0 scale overflowed */
#define MOE_Q4_STATUS_SPIN_TIMEOUT 0x2u   /* a bounded device-side wait gave up */
#define MOE_Q4_STATUS_NONFINITE_LOGIT 0x4u /* a router logit was NaN or infinite: NaN ranks below
                                              every number, so the token still gets k distinct
                                              experts in [0, E), but its weights are undefined */
#define MOE_Q4_STATUS_BAD_EXPERT_INDEX 0x8u /* the permutation met an expert index outside [0, E)
                                               (counted as expert 0; the top-k never produces one) */

/* One MoE layer.  Expert e's matrices are consecutive Q4_0 blocks:
 *   w_gate, w_up : [n_experts][ffn][hidden/32] blocks (18 B each)
 *   w_down       : [n_experts][hidden][ffn/32] blocks
 *   sh_*         : the always-on shared expert, same layout with one expert;
 *                  all three NULL iff has_shared == 0.
 *   w_router     : [n_experts][hidden] fp32;  router_bias: [n_experts] or NULL. */
typedef struct {
    int32_t hidden, ffn, n_experts, top_k, has_shared;
    const float* w_router;
    const float* router_bias;
    const uint8_t* w_gate;
    const uint8_t* w_up;
    const uint8_t* w_down;
    const uint8_t* sh_gate;
    const uint8_t* sh_up;
    const uint8_t* sh_down;
} moe_q4_layer;

/* Q8_0 activation quantisation (Methodologie 1 and 2: the 8-bit activations
 * of the W4A8 kernel).  x [T][H] fp32 -> q [T][H] int8 and d [T][H/32]
 * binary16 bits.  `status` (device uint32, may be NULL) receives
 * MOE_Q4_STATUS_SCALE_OVERFLOW.  H must be a positive multiple of 32. */
int moe_q4_quantize_act(const float* x, int64_t T, int32_t H, int8_t* q, uint16_t* d,
                        uint32_t* status, moe_q4_stream_t stream);

/* Router (Methodologie 1: "MoE-routing" of the grouped GEMM): logits [T][E]
 * fp32 = x.Wr^T (+ bias), then per token the top-k experts (descending logit,
 * ties to the lower index) into topk_idx [T][k] int32 and their softmax
 * weights into topk_w [T][k] fp32.  `logits` is a caller buffer that
 * receives the logits (required). */
int moe_q4_route(const moe_q4_layer* L, const float* x, int64_t T, int32_t* topk_idx,
                 float* topk_w, float* logits, moe_q4_stream_t stream);

/* Bytes of device workspace moe_q4_ffn_forward needs for up to T_max tokens
 * (0 on invalid arguments). */
size_t moe_q4_ffn_workspace_bytes(const moe_q4_layer* L, int64_t T_max);

/* The whole MoE expert FFN layer (Methodologie 1: grouped 4-bit GEMM for
 * prefill, W4A8 kernel for decode; Methodologie 4: all T tokens in one pass).
 * x [T][H] fp32 in, y [T][H] fp32 out (overwritten; must not overlap x or the
 * workspace).  The workspace must hold moe_q4_ffn_workspace_bytes(L, T) bytes;
 * its first uint32 is the device status word (cleared by this call).
 * Kernel choice by T is internal; results do not depend on it beyond fp32
 * summation order. */
int moe_q4_ffn_forward(const moe_q4_layer* L, const float* x, int64_t T, float* y,
                       void* workspace, size_t ws_bytes, moe_q4_stream_t stream);

/* Bytes of device workspace moe_q4_ffn_forward_host needs: the forward's
 * workspace plus device staging for x and y. */
size_t moe_q4_ffn_host_workspace_bytes(const moe_q4_layer* L, int64_t T_max);

/* moe_q4_ffn_forward with x and y in HOST memory (pinned for asynchronous
 * copies): enqueues the host-to-device copy of x, the forward, and the
 * device-to-host copy of y on `stream`.  y is valid after the caller
 * synchronises the stream.  For one token with both x and y page-locked (and
 * 16-byte aligned) the copies are made by kernels of the decode chain (a
 * first one reads x, a last one writes y over the bus), with no copy node
 * between the kernels.  That first kernel is a programmatic dependent launch
 * and reads x before its dependency wait: x may be read as soon as the kernel
 * enqueued just before the call lets its dependents launch.  A kernel of the
 * caller's that writes x must therefore not release its dependents early
 * (the default).  The previous one-token host call's y on the same stream is
 * tracked by the library: when x overlaps it, x is read after the wait. */
int moe_q4_ffn_forward_host(const moe_q4_layer* L, const float* x_host, int64_t T, float* y_host,
                            void* workspace, size_t ws_bytes, moe_q4_stream_t stream);

/* The paper has no counterpart of this entry point; it exists for callers
 * that cannot allocate device memory.  Examples: a host runtime or plugin
 * whose device memory is reserved up front by someone else, a latency-critical
 * decode loop that cannot pay for cudaMalloc's implicit device
 * synchronisation, and code that may not allocate while it records a CUDA
 * graph.
 * moe_q4_ffn_forward with the workspace replaced by a static device array of
 * MOE_Q4_NOALLOC_SCRATCH_BYTES owned by the library.  Nothing is allocated
 * or freed by the call.  The array occupies device memory on each GPU where
 * this entry is used, from its first call there (CUDA's default lazy module
 * loading places it then; with lazy loading off, when the library's module is
 * loaded into the device's context) until the process exits.
 *   - x, y: as for moe_q4_ffn_forward (caller-owned device buffers).
 *   - The device is checked (MOE_Q4_ERR_ARCH) before the scratch is touched.
 *   - A problem whose workspace (moe_q4_ffn_workspace_bytes(L, T)) exceeds
 *     the scratch returns MOE_Q4_ERR_WORKSPACE and enqueues nothing; for a
 *     layer with hidden 2048, ffn 512, 128 experts, top-8 and a shared expert
 *     that allows T up to 542 tokens.
 *   - The first call on a device looks up the scratch's device address (once
 *     per device, with that device current); make that first call before any
 *     stream capture.
 *   - All calls share the one array, which keeps the last call's contents.
 *     Each call writes every scratch value it later reads (the status word,
 *     the first uint32 of the scratch, is cleared at the start), so nothing
 *     needs clearing between calls.  Calls that overlap on the GPU (other
 *     streams, other host threads) race on the scratch: serialise them. */
#define MOE_Q4_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
int moe_q4_ffn_forward_noalloc(const moe_q4_layer* L, const float* x, int64_t T, float* y,
                               moe_q4_stream_t stream);

/* ---------------------------------------------------------------------
 * Stacks of layers.
 *
 * The page runs the MoE layers one after another (Methodologie 1: expert
 * weights are streamed layer by layer) but fixes no step between them.  The
 * multi-layer workload joins them by a residual add; without a normalisation
 * the activations grow by about 25x per layer and the binary16 Q8_0 scales
 * overflow within a few layers.  The step taken between layers is
 *     x_{l+1} = x_l + MoE_l(RMSNorm(x_l)),
 * RMSNorm with unit gain over H: rms = sqrt(mean_h x^2 + eps) with the mean
 * of squares accumulated in binary64, xn = binary32(x / rms) (binary64
 * division, one rounding).
 * --------------------------------------------------------------------- */

/* x [T][H] fp32 (in place), y [T][H] fp32 or NULL, xn [T][H] fp32 or NULL:
 *   if y: x <- binary32(x + y);  then if xn: xn = RMSNorm(x).
 * H a positive multiple of 256, eps finite and >= 0, 0 <= T <= 2^24;
 * 16-byte aligned pointers; xn must not overlap x or y (x and y must not
 * overlap either).  Returns MOE_Q4_OK or an error code; T == 0 is a no-op. */
int moe_q4_residual_rmsnorm(float* x, const float* y, int64_t T, int32_t H, float eps, float* xn,
                            moe_q4_stream_t stream);

/* Workspace of moe_q4_stack_forward for layers shaped like *L and up to T_max
 * tokens: RMSNorm output and layer output [T_max][H] fp32 each, then one layer
 * workspace.  0 for an invalid layer or T_max. */
size_t moe_q4_stack_workspace_bytes(const moe_q4_layer* L, int64_t T_max);

/* n_layers >= 1 layers (an array of descriptors, all with the same hidden,
 * ffn, n_experts, top_k and has_shared) applied in order to x [T][H] fp32 in
 * place: for each layer, x <- x + MoE_l(RMSNorm(x)).  Same conventions and
 * errors as moe_q4_ffn_forward; MOE_Q4_ERR_SHAPE if the layers differ in
 * shape.  The device status word (the first uint32 of the layer workspace,
 * which starts after the two [T_max][H] fp32 buffers, each rounded up to 256
 * bytes) is cleared once at the start of the call and accumulates the
 * conditions of every layer. */
int moe_q4_stack_forward(const moe_q4_layer* layers, int32_t n_layers, float* x, int64_t T, float eps,
                         void* workspace, size_t ws_bytes, moe_q4_stream_t stream);

/* ---------------------------------------------------------------------
 * Host-streamed experts.
 *
 * The page keeps its expert weights in page-locked host memory and streams
 * them to a small GPU layer by layer (Methodologie 1 and 2).  Here the
 * expert matrices of L (w_gate, w_up, w_down and the shared ones) are
 * PAGE-LOCKED HOST pointers (cudaHostAlloc / cudaHostRegister; pageable
 * memory is rejected with MOE_Q4_ERR_INVALID_ARG), while w_router,
 * router_bias, x, y, the workspace and `staging` are device memory.  Each
 * call routes the tokens on the device, copies exactly the experts that the
 * routing selects (and the shared expert) into `staging` (at least
 * moe_q4_staging_bytes(L) bytes, 256-byte aligned: a device copy laid out
 * like the layer), with the GPU reading the host pages directly, and then
 * runs moe_q4_ffn_forward on the staged copy.  No host synchronisation:
 * the call is stream-ordered and graph-capturable.  Same results as
 * moe_q4_ffn_forward on a resident copy of the layer.
 * --------------------------------------------------------------------- */
size_t moe_q4_staging_bytes(const moe_q4_layer* L);
int moe_q4_ffn_forward_streamed(const moe_q4_layer* L, const float* x, int64_t T, float* y, void* workspace,
                                size_t ws_bytes, void* staging, size_t staging_bytes, moe_q4_stream_t stream);

/* ---------------------------------------------------------------------
 * W4A8 GEMV of one large Q4_0 matrix (the LM head).
 *
 * The page reports the LM head run on the GPU against the CPU (Resultaten,
 * 116 -> 139 ms/token on Fermi).  Here it is the decode path's W4A8 GEMV
 * applied to one vocabulary-sized matrix: x [T][H] fp32 (1 <= T <= 8) is
 * quantised to Q8_0 exactly as moe_q4_quantize_act does, and
 *     y[t][n] = sum_b dW[n,b] * dA[t,b] * I_{n,b,t}   (binary32)
 * with I the exact per-block integer dot product, for the N rows of
 * W [N][H/32] Q4_0 blocks (18 B each).  y is [T][N] fp32, overwritten.
 * H a positive multiple of 256 up to 16384, 1 <= N <= 2^30; pointers 16-byte
 * aligned, the workspace 256-byte aligned and at least
 * moe_q4_gemv_workspace_bytes(T, H) bytes (status word, Q8_0 of x); y must
 * not overlap x or the workspace.  The status word (first uint32 of the
 * workspace) reports a binary16 scale overflow.
 * --------------------------------------------------------------------- */
size_t moe_q4_gemv_workspace_bytes(int64_t T, int32_t H);
int moe_q4_gemv(const uint8_t* W, int64_t N, int32_t H, const float* x, int64_t T, float* y, void* workspace,
                size_t ws_bytes, moe_q4_stream_t stream);

/* Static description of an error code. */
const char* moe_q4_status_string(int status);

/* Description of the CUDA runtime error behind the last MOE_Q4_ERR_CUDA that
 * an entry point returned on the calling thread ("no CUDA error" if none). */
const char* moe_q4_last_cuda_error(void);

/* ---------------------------------------------------------------------
 * Inspection entry points used by the parity tests.
 * --------------------------------------------------------------------- */

/* Byte offsets, inside a forward workspace sized for T tokens, of the
 * intermediate arrays, in this order (MOE_Q4_WS_* indices):
 *   status u32[4] | logits f32[T][E] | topk_idx i32[T][k] | topk_w f32[T][k]
 *   | qa i8[T][H] | da u16[T][H/32] | cnt i32[E+1] | off i32[E+2]
 *   | tile_off i32[E+2] | chunk_cnt i32[C][E] | chunk_base i32[C][E]
 *   | sorted i32[P] | pos i32[P] | hq i8[P+S*T][F] | dh u16[P+S*T][F/32]
 *   | total
 * with P = T*k routed pairs and S = has_shared.  Slots (rows of hq/dh) are
 * grouped by expert: routed expert e owns slots off[e]..off[e+1]-1 holding
 * pairs sorted[...] = t*k+j in increasing (t, j) order; the shared expert
 * owns slots P..P+T-1 (slot P+t = token t).  pos is the inverse of sorted.
 * Fills n <= MOE_Q4_WS_COUNT entries of `offsets`; returns MOE_Q4_OK or an
 * error code. */
enum {
    MOE_Q4_WS_STATUS = 0, MOE_Q4_WS_LOGITS, MOE_Q4_WS_TOPK_IDX, MOE_Q4_WS_TOPK_W, MOE_Q4_WS_QA,
    MOE_Q4_WS_DA, MOE_Q4_WS_CNT, MOE_Q4_WS_OFF, MOE_Q4_WS_TILE_OFF, MOE_Q4_WS_CHUNK_CNT,
    MOE_Q4_WS_CHUNK_BASE, MOE_Q4_WS_SORTED, MOE_Q4_WS_POS, MOE_Q4_WS_HQ, MOE_Q4_WS_DH,
    MOE_Q4_WS_TOTAL, MOE_Q4_WS_COUNT
};
int moe_q4_workspace_layout(const moe_q4_layer* L, int64_t T, size_t* offsets, int n);

/* Kernel family selectors for moe_q4_ffn_forward_debug. */
enum {
    MOE_Q4_PATH_AUTO = 0,     /* what moe_q4_ffn_forward does */
    MOE_Q4_PATH_GROUPED_DP4A = 1,
    MOE_Q4_PATH_DECODE = 2,
    MOE_Q4_PATH_TENSOR_CORE = 3,     /* tensor cores, tile width chosen by T */
    MOE_Q4_PATH_TENSOR_CORE_N32 = 4, /* tensor cores, tiles of 32 slots */
    MOE_Q4_PATH_TENSOR_CORE_N128 = 5, /* tensor cores, tiles of 128 slots */
    MOE_Q4_PATH_TENSOR_CORE_N64 = 6   /* tensor cores, tiles of 64 slots */
};

typedef struct {
    float* h_out;     /* [P+S*T][F] fp32 SwiGLU output before requantisation, slot order; or NULL */
    int32_t path;     /* MOE_Q4_PATH_* */
    void* ev_start;   /* cudaEvent_t recorded just before the dominant (gate/up) kernel, or NULL */
    void* ev_stop;    /* cudaEvent_t recorded just after it, or NULL */
    int32_t force_spin_timeout;  /* nonzero: one CTA of the fused T = 1 FFN kernel waits for 16 bytes
                                    more than its weight copies deliver, so its bounded wait runs out;
                                    the call completes with correct results and
                                    MOE_Q4_STATUS_SPIN_TIMEOUT in the status word (tests of the timeout
                                    report; about half a second per call) */
    /* Per-block integer dot products I_b = sum_{i<32} (nibble_i - 8) * q_i of
     * the grouped paths (tensor-core and streaming), exactly as the projection
     * kernel computed them (the tensor-core path: the MMA's accumulator before
     * the rescale), for one row block of one expert group:
     *   block_dots_out[s][r][b], s = slot - off[g] over the group's slots in
     *   slot order, r < R rows of the row block, b < K/32 blocks along K.
     * Tensor-core paths: R = 128; gate/up rows r < 64 are gate rows 64 rb + r,
     * r >= 64 the up rows 64 rb + r - 64; down rows are 128 rb + r.
     * Streaming path: R = 64; gate/up rows r < 32 are gate rows 32 rb + r,
     * r >= 32 the up rows 32 rb + r - 32; down rows are 64 rb + r.
     * The buffer must hold count(g) * R * K/32 int32 (K = hidden for gate/up,
     * ffn for down); ignored by the T = 1 fused path.  NULL: no capture. */
    int32_t* block_dots_out;
    int32_t block_dots_down;   /* 0: the gate/up projection, 1: the down projection */
    int32_t block_dots_group;  /* expert group g (n_experts: the shared expert) */
    int32_t block_dots_rb;     /* row block */
    /* Fused T = 1 path only: device uint64[3], 8-byte aligned; per call, in
     * the FFN kernel's first CTA (%globaltimer ns, inside the programmatic-
     * launch chain, with no event between the kernels): [0] += the span from
     * its wait on the router kernel returning to its end, [1] += 1, [2] +=
     * the span from its start (the launch overlaps the router kernel, so
     * this includes the wait) to its end.  NULL: not timed. */
    unsigned long long* decode_kernel_ns;
} moe_q4_debug;

/* moe_q4_ffn_forward with inspection options (see moe_q4_debug). */
int moe_q4_ffn_forward_debug(const moe_q4_layer* L, const float* x, int64_t T, float* y,
                             void* workspace, size_t ws_bytes, const moe_q4_debug* dbg,
                             moe_q4_stream_t stream);

/* Test hook: with enable != 0 every entry point sees the current device as
 * compute capability major.minor instead of asking the driver, so the
 * MOE_Q4_ERR_ARCH rejection (anything but 10.0, checked before any CUDA call
 * and before anything is enqueued) can be exercised on any host; enable == 0
 * restores the real query.  Not thread-safe: for tests only.  Returns
 * MOE_Q4_OK. */
int moe_q4_test_override_device(int32_t enable, int32_t major, int32_t minor);

/* Per-block W4A8 integer dot products through the device routine every
 * projection kernel uses: out[i] = sum_{j<32} (nibble_j(w[i]) - 8) * qa[32*i+j]
 * for n Q4_0 blocks w (18 B each, consecutive; n a multiple of 8) and n*32 int8
 * activations. */
int moe_q4_block_dots(const uint8_t* w_blocks, const int8_t* qa, int64_t n, int32_t* out,
                      moe_q4_stream_t stream);

/* Measurement aid: the tensor-core projections' epilogue rescale on its own
 * (the per-block step acc += I_b * dW * dA that follows every 32-wide block's
 * MMA; "Methodologie 1" of the Dutch technical summary page, the W4A8 block
 * arithmetic).  One CTA per SM runs `iters` (1 .. 2^20) operand stages of the
 * epilogue's inner loop -- TMEM loads, block scales from shared memory, the
 * packed fp32 rescale, and with int8_operands != 0 the int8 path's bias
 * removal and TMEM reset -- over its whole TMEM, with no other role, so its
 * rate is the ceiling the rescale puts on the projection kernels.  Writes one
 * float (a checksum that keeps the work live) to sink (device, 4-byte
 * aligned) and the number of accumulator elements rescaled to *elements
 * (host); each element stands for 32 int8 multiply-adds.  Asynchronous on
 * `stream`; time it with events around the call. */
int moe_q4_rescale_ceiling(int32_t int8_operands, int32_t iters, float* sink, int64_t* elements,
                           moe_q4_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_Q4_H */
