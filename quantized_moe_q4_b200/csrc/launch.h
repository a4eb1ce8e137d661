// launch.h -- host-side launchers of the kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moeq4 {

// Shapes and device pointers of one layer as the kernels see them.
struct LayerView {
    int H, F, E, k, S;
    const float* w_router;
    const float* router_bias;
    const uint8_t* w_gate;
    const uint8_t* w_up;
    const uint8_t* w_down;
    const uint8_t* sh_gate;
    const uint8_t* sh_up;
    const uint8_t* sh_down;
};

// Pointers into a forward workspace.
struct Workspace {
    uint32_t* status;
    float* logits;
    int32_t* topk_idx;
    float* topk_w;
    int8_t* qa;
    uint16_t* da;
    int32_t* cnt;
    int32_t* off;
    int32_t* tile_off;
    int32_t* chunk_cnt;
    int32_t* chunk_base;
    int32_t* sorted;
    int32_t* pos;
    int8_t* hq;
    uint16_t* dh;
};

// Test capture of the per-block integer dot products I_b of one row block of
// one expert group (moe_q4_debug.block_dots_*): out[slot - off[g]][row][block].
struct BlockDotCapture {
    int32_t* out;
    int down;   // 0: gate/up projection, 1: down projection
    int group;  // expert group (E: the shared expert)
    int rb;     // row block of the kernel family
};

struct DeviceInfo {
    int sm_count;
    int max_smem_optin;
};

// k_route.cu
// status_clear (may be NULL): a status word the first thread zeroes.
cudaError_t launch_router_logits(const LayerView& L, const float* x, int64_t T, float* logits,
                                 uint32_t* status_clear, cudaStream_t s);
// status (may be NULL) receives STATUS_NONFINITE_LOGIT.
cudaError_t launch_topk(const float* logits, int64_t T, int E, int k, int32_t* idx, float* w,
                        uint32_t* status, cudaStream_t s);

// k_quant_perm.cu
cudaError_t launch_quantize(const float* x, int64_t T, int H, int8_t* q, uint16_t* d,
                            uint32_t* status, float* y_zero, cudaStream_t s);
cudaError_t launch_permute(const int32_t* idx, int64_t T, int k, int E, int S, int tile_tokens,
                           const Workspace& ws, cudaStream_t s);

// k_grouped_dp4a.cu
// cap (may be NULL): capture the block dot products of one row block.
cudaError_t launch_gateup_dp4a(const LayerView& L, int64_t T, const Workspace& ws, float* h_dbg,
                               const DeviceInfo& dev, const BlockDotCapture* cap, cudaStream_t s);
cudaError_t launch_down_dp4a(const LayerView& L, int64_t T, const Workspace& ws, float* y,
                             const DeviceInfo& dev, const BlockDotCapture* cap, cudaStream_t s);
// y[t][n] (t < T <= 8, n < N) = W4A8 product of Q4_0 rows W [N][H/32] with the
// Q8_0 activations qa/da of T tokens (the streaming kernel's GEMV mode).
cudaError_t launch_gemv_dp4a(const uint8_t* W, int64_t N, int H, const int8_t* qa, const uint16_t* da, int T,
                             float* y, uint32_t* status, const DeviceInfo& dev, cudaStream_t s);
// k_tc_grouped.cu: grouped projections on tcgen05 (kind::f16, TMEM) with
// tiles of `tile` slots (32 or 128); the permutation must have been built with
// the same tile width.  tc_tile_tokens: the width for T tokens (force = 32 or
// 128 picks one, else automatic).
int tc_tile_tokens(const LayerView& L, int64_t T, int force);
cudaError_t launch_gateup_tc(const LayerView& L, int64_t T, const Workspace& ws, float* h_dbg, const DeviceInfo& dev,
                             int tile, const BlockDotCapture* cap, cudaStream_t s);
cudaError_t launch_down_tc(const LayerView& L, int64_t T, const Workspace& ws, float* y, const DeviceInfo& dev,
                           int tile, const BlockDotCapture* cap, cudaStream_t s);

// k_decode.cu: the fused T=1 path (router kernel + FFN kernel,
// chained with programmatic dependent launch).  Events, if given, bracket the
// FFN kernel.
bool decode_eligible(const LayerView& L, int64_t T, const DeviceInfo& dev);
// force_timeout: one gate/up copy barrier of CTA 0 expects 16 bytes that
// never arrive (the bounded wait runs out; used only to test the timeout report).
// clear_status: zero the status word (else the kernels only OR into it).
// kernel_ns (may be NULL): [0] += the FFN kernel's span in CTA 0 (globaltimer
// ns, entry to exit), [1] += 1, per launch.  x_host / y_host (may be NULL):
// page-locked host memory that a first kernel of the chain copies into x (a
// device buffer then) / a last kernel copies y into.
cudaError_t launch_decode(const LayerView& L, const float* x, float* y, const Workspace& ws, float* h_dbg,
                          const DeviceInfo& dev, cudaEvent_t ev_start, cudaEvent_t ev_stop, bool force_timeout,
                          bool clear_status, unsigned long long* kernel_ns, const float* x_host, float* y_host,
                          bool x_host_early, cudaStream_t s);

cudaError_t launch_block_dots(const uint8_t* w, const int8_t* qa, int64_t n, int32_t* out,
                              cudaStream_t s);

// k_tc_grouped.cu: the tensor-core epilogue's per-block rescale on its own
// (one CTA per SM, iters operand stages); *elements = accumulator elements
// rescaled (each one 32 int8 multiply-adds of the projection).
cudaError_t launch_rescale_ceiling(bool int8_operands, int iters, float* sink, const DeviceInfo& dev,
                                   int64_t* elements, cudaStream_t s);

// k_stage.cu: copy the experts with cnt[g] > 0 (and the shared expert) from
// pinned host memory (h_*) into the device staging copy (d_*).
struct StageParams {
    int E, S;
    size_t gu_bytes, dn_bytes;  // one expert's gate (or up) matrix, one down matrix
    const int32_t* cnt;
    const uint8_t* h_gate;
    const uint8_t* h_up;
    const uint8_t* h_down;
    const uint8_t* h_sh_gate;
    const uint8_t* h_sh_up;
    const uint8_t* h_sh_down;
    uint8_t* d_gate;
    uint8_t* d_up;
    uint8_t* d_down;
    uint8_t* d_sh_gate;
    uint8_t* d_sh_up;
    uint8_t* d_sh_down;
};
cudaError_t launch_stage_experts(const StageParams& p, const DeviceInfo& dev, cudaStream_t s);

// k_stack.cu: x += y (if y), then xn = RMSNorm(x) (if xn); H a multiple of 128.
cudaError_t launch_residual_rmsnorm(float* x, const float* y, int64_t T, int H, float eps, float* xn,
                                    cudaStream_t s);

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// MOE_Q4_OK if the current device is compute capability 10.0, else
// MOE_Q4_ERR_ARCH (or MOE_Q4_ERR_CUDA if it cannot be queried); abi.cu.
int check_device();

// Resident CTAs per SM of `kernel` at `threads` and `smem` dynamic bytes, with
// the dynamic shared-memory limit raised to `smem` first.  Cached per device,
// kernel and size, so the CUDA attribute calls happen on the first (eager)
// launch only, never while a stream is being captured.  At least 1.
cudaError_t kernel_occupancy(const void* kernel, int threads, size_t smem, int* per_sm);

// cudaEventRecord that also works inside stream capture (as an external event
// record node whose timestamp can be read after each graph launch).
cudaError_t record_event(cudaEvent_t ev, cudaStream_t s);

}  // namespace moeq4
