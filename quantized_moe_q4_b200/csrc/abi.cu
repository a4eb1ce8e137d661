// abi.cu -- the extern "C" entry points of include/moe_q4.h: argument checks,
// workspace layout, kernel-family dispatch.  No allocation, no host sync.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <utility>

#include "moe_q4.h"
#include "common.cuh"
#include "launch.h"

namespace moeq4 {

static constexpr int64_t T_LIMIT = int64_t(1) << 24;
// Token count from which the automatic choice uses the tensor-core kernels.
static constexpr int64_t TC_MIN_TOKENS = 48;   // measured crossover of the dp4a and tensor-core paths
static constexpr int MAX_DEVICES = 64;

struct DeviceState {
    int checked;  // 0 unknown, 1 ok, -1 wrong arch
    DeviceInfo info;
};
static DeviceState g_dev[MAX_DEVICES];

// Test override of the device's compute capability (moe_q4_test_override_device).
static int g_cc_override[3] = {0, 0, 0};  // enabled, major, minor

static int current_device(DeviceInfo* out) {
    if (g_cc_override[0] && !(g_cc_override[1] == 10 && g_cc_override[2] == 0)) return MOE_Q4_ERR_ARCH;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return MOE_Q4_ERR_CUDA;
    DeviceState& st = g_dev[dev];
    if (st.checked == 0) {
        int major = 0, minor = 0, sms = 0, smem = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return MOE_Q4_ERR_CUDA;
        st.info.sm_count = sms;
        st.info.max_smem_optin = smem;
        st.checked = (major == 10 && minor == 0) ? 1 : -1;
    }
    if (st.checked < 0) return MOE_Q4_ERR_ARCH;
    *out = st.info;
    return MOE_Q4_OK;
}

struct OccEntry {
    int dev;
    const void* kernel;
    int threads;
    size_t smem;
    int per_sm;
};
static OccEntry g_occ[256];
static int g_occ_n = 0;
static std::mutex g_occ_mu;

static size_t kernel_static_smem(const void* kernel) {
    cudaFuncAttributes a;
    if (cudaFuncGetAttributes(&a, kernel) != cudaSuccess) return 0;
    return a.sharedSizeBytes;
}

// Last CUDA error seen by an entry point of this thread (for error messages).
static thread_local cudaError_t g_last_cuda_error = cudaSuccess;

cudaError_t kernel_occupancy(const void* kernel, int threads, size_t smem, int* per_sm) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_occ_mu);
    bool kernel_seen = false;
    for (int i = 0; i < g_occ_n; ++i) {
        const OccEntry& o = g_occ[i];
        if (o.dev != dev || o.kernel != kernel) continue;
        kernel_seen = true;
        if (o.threads == threads && o.smem == smem) {
            *per_sm = o.per_sm;
            return cudaSuccess;
        }
    }
    // The dynamic shared-memory limit is one attribute per function: raise it
    // once to the device's opt-in maximum, so launches of every size (cached
    // or not) stay within it.
    if (!kernel_seen) {
        int max_optin = 0;
        e = cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return e;
        const int dyn_max = max_optin - (int)kernel_static_smem(kernel);
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_max);
        if (e != cudaSuccess) return e;
    }
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem);
    if (e != cudaSuccess) return e;
    if (n < 1) n = 1;
    if (g_occ_n < 256) g_occ[g_occ_n++] = OccEntry{dev, kernel, threads, smem, n};
    *per_sm = n;
    return cudaSuccess;
}

cudaError_t record_event(cudaEvent_t ev, cudaStream_t s) {
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(s, &st);
    if (e != cudaSuccess) return e;
    if (st == cudaStreamCaptureStatusActive) return cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
    return cudaEventRecord(ev, s);
}

static bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

static bool overlap(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return na && nb && x < y + nb && y < x + na;
}

static int check_layer(const moe_q4_layer* L) {
    if (!L) return MOE_Q4_ERR_INVALID_ARG;
    if (L->n_experts < 1 || L->n_experts > 256 || L->top_k < 1 || L->top_k > 16 || L->top_k > L->n_experts)
        return MOE_Q4_ERR_INVALID_ARG;
    if (L->has_shared != 0 && L->has_shared != 1) return MOE_Q4_ERR_INVALID_ARG;
    if (!L->w_router || !L->w_gate || !L->w_up || !L->w_down) return MOE_Q4_ERR_INVALID_ARG;
    const bool sh = L->sh_gate || L->sh_up || L->sh_down;
    if (L->has_shared && !(L->sh_gate && L->sh_up && L->sh_down)) return MOE_Q4_ERR_INVALID_ARG;
    if (!L->has_shared && sh) return MOE_Q4_ERR_INVALID_ARG;
    if (L->hidden <= 0 || L->ffn <= 0 || L->hidden % 256 || L->ffn % 256 || L->hidden > 16384 || L->ffn > 16384)
        return MOE_Q4_ERR_SHAPE;
    const void* ptrs[] = {L->w_router, L->w_gate, L->w_up, L->w_down, L->sh_gate, L->sh_up, L->sh_down};
    for (const void* q : ptrs)
        if (q && !aligned(q, 16)) return MOE_Q4_ERR_ALIGN;
    if (L->router_bias && !aligned(L->router_bias, 4)) return MOE_Q4_ERR_ALIGN;
    return MOE_Q4_OK;
}

static LayerView view(const moe_q4_layer* L) {
    LayerView v;
    v.H = L->hidden; v.F = L->ffn; v.E = L->n_experts; v.k = L->top_k; v.S = L->has_shared;
    v.w_router = L->w_router; v.router_bias = L->router_bias;
    v.w_gate = L->w_gate; v.w_up = L->w_up; v.w_down = L->w_down;
    v.sh_gate = L->sh_gate; v.sh_up = L->sh_up; v.sh_down = L->sh_down;
    return v;
}

static size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

static void layout(const LayerView& L, int64_t T, size_t off[WS_COUNT]) {
    const int64_t P = T * L.k;
    const int64_t slots = P + (L.S ? T : 0);
    const int64_t C = ceil_div(P, PERM_CHUNK);
    const size_t sz[WS_COUNT - 1] = {
        16,                                            // status
        sizeof(float) * (size_t)(T * L.E),             // logits
        sizeof(int32_t) * (size_t)P,                   // topk_idx
        sizeof(float) * (size_t)P,                     // topk_w
        (size_t)(T * L.H),                             // qa
        sizeof(uint16_t) * (size_t)(T * (L.H / QK)),   // da
        sizeof(int32_t) * (size_t)(L.E + 1),           // cnt
        sizeof(int32_t) * (size_t)(L.E + 2),           // off
        sizeof(int32_t) * (size_t)(L.E + 2),           // tile_off
        sizeof(int32_t) * (size_t)(C * L.E),           // chunk_cnt
        sizeof(int32_t) * (size_t)(C * L.E),           // chunk_base
        sizeof(int32_t) * (size_t)P,                   // sorted
        sizeof(int32_t) * (size_t)P,                   // pos
        (size_t)(slots * L.F),                         // hq
        sizeof(uint16_t) * (size_t)(slots * (L.F / QK)),  // dh
    };
    size_t o = 0;
    for (int i = 0; i < WS_COUNT - 1; ++i) {
        off[i] = o;
        o += align256(sz[i]);
    }
    off[WS_TOTAL] = o;
}

static Workspace carve(void* base, const size_t off[WS_COUNT]) {
    char* b = static_cast<char*>(base);
    Workspace w;
    w.status = reinterpret_cast<uint32_t*>(b + off[WS_STATUS]);
    w.logits = reinterpret_cast<float*>(b + off[WS_LOGITS]);
    w.topk_idx = reinterpret_cast<int32_t*>(b + off[WS_TOPK_IDX]);
    w.topk_w = reinterpret_cast<float*>(b + off[WS_TOPK_W]);
    w.qa = reinterpret_cast<int8_t*>(b + off[WS_QA]);
    w.da = reinterpret_cast<uint16_t*>(b + off[WS_DA]);
    w.cnt = reinterpret_cast<int32_t*>(b + off[WS_CNT]);
    w.off = reinterpret_cast<int32_t*>(b + off[WS_OFF]);
    w.tile_off = reinterpret_cast<int32_t*>(b + off[WS_TILE_OFF]);
    w.chunk_cnt = reinterpret_cast<int32_t*>(b + off[WS_CHUNK_CNT]);
    w.chunk_base = reinterpret_cast<int32_t*>(b + off[WS_CHUNK_BASE]);
    w.sorted = reinterpret_cast<int32_t*>(b + off[WS_SORTED]);
    w.pos = reinterpret_cast<int32_t*>(b + off[WS_POS]);
    w.hq = reinterpret_cast<int8_t*>(b + off[WS_HQ]);
    w.dh = reinterpret_cast<uint16_t*>(b + off[WS_DH]);
    return w;
}

// Page-locked host memory the GPU can address (unified addressing), or device
// memory, by the runtime's pointer attributes.
static bool pinned_host(const void* p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeHost;
}

static bool on_device(const void* p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

static int cuda_rc(cudaError_t e) {
    if (e == cudaSuccess) return MOE_Q4_OK;
    g_last_cuda_error = e;
    return MOE_Q4_ERR_CUDA;
}

#define MOE_TRY(expr)                          \
    do {                                       \
        cudaError_t e_ = (expr);               \
        if (e_ != cudaSuccess) return cuda_rc(e_); \
    } while (0)

// clear_status: zero the workspace's status word first (every public forward
// does; the stack entry clears it once and lets it accumulate over layers).
static int forward_impl(const moe_q4_layer* Lp, const float* x, int64_t T, float* y, void* ws, size_t ws_bytes,
                        const moe_q4_debug* dbg, cudaStream_t s, bool clear_status = true) {
    int rc = check_layer(Lp);
    if (rc) return rc;
    if (T < 0 || T > T_LIMIT) return MOE_Q4_ERR_INVALID_ARG;
    if (T == 0) return MOE_Q4_OK;
    if (!x || !y || !ws) return MOE_Q4_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(ws, 256)) return MOE_Q4_ERR_ALIGN;
    const LayerView L = view(Lp);
    size_t off[WS_COUNT];
    layout(L, T, off);
    if (ws_bytes < off[WS_TOTAL]) return MOE_Q4_ERR_WORKSPACE;
    const size_t xy_bytes = sizeof(float) * (size_t)(T * L.H);
    if (overlap(x, xy_bytes, y, xy_bytes) || overlap(y, xy_bytes, ws, off[WS_TOTAL])) return MOE_Q4_ERR_OVERLAP;
    if (dbg && dbg->h_out && !aligned(dbg->h_out, 4)) return MOE_Q4_ERR_ALIGN;
    if (dbg && dbg->decode_kernel_ns && !aligned(dbg->decode_kernel_ns, 8)) return MOE_Q4_ERR_ALIGN;
    if (dbg && dbg->block_dots_out &&
        (!aligned(dbg->block_dots_out, 4) || dbg->block_dots_group < 0 ||
         dbg->block_dots_group > Lp->n_experts - (Lp->has_shared ? 0 : 1) || dbg->block_dots_rb < 0))
        return MOE_Q4_ERR_INVALID_ARG;
    DeviceInfo dev;
    rc = current_device(&dev);
    if (rc) return rc;

    const Workspace w = carve(ws, off);
    cudaEvent_t ev0 = dbg ? static_cast<cudaEvent_t>(dbg->ev_start) : nullptr;
    cudaEvent_t ev1 = dbg ? static_cast<cudaEvent_t>(dbg->ev_stop) : nullptr;
    const int path = dbg ? dbg->path : MOE_Q4_PATH_AUTO;
    if ((path == MOE_Q4_PATH_AUTO || path == MOE_Q4_PATH_DECODE) && decode_eligible(L, T, dev))
        return cuda_rc(launch_decode(L, x, y, w, dbg ? dbg->h_out : nullptr, dev, ev0, ev1,
                                     dbg && dbg->force_spin_timeout, clear_status,
                                     dbg ? dbg->decode_kernel_ns : nullptr, nullptr, nullptr, false, s));

    // grouped paths: tensor cores once experts see tens of tokens, else dp4a
    const bool tc = (path == MOE_Q4_PATH_TENSOR_CORE) || (path == MOE_Q4_PATH_TENSOR_CORE_N32) ||
                    (path == MOE_Q4_PATH_TENSOR_CORE_N64) || (path == MOE_Q4_PATH_TENSOR_CORE_N128) ||
                    (path == MOE_Q4_PATH_AUTO && T >= TC_MIN_TOKENS);
    const int tile = tc ? tc_tile_tokens(L, T, path == MOE_Q4_PATH_TENSOR_CORE_N32    ? 32
                                               : path == MOE_Q4_PATH_TENSOR_CORE_N64  ? 64
                                               : path == MOE_Q4_PATH_TENSOR_CORE_N128 ? 128
                                                                                      : 0)
                        : DP4A_TT;
    MOE_TRY(launch_router_logits(L, x, T, w.logits, clear_status ? w.status : nullptr, s));
    MOE_TRY(launch_topk(w.logits, T, L.E, L.k, w.topk_idx, w.topk_w, w.status, s));
    MOE_TRY(launch_quantize(x, T, L.H, w.qa, w.da, w.status, y, s));
    MOE_TRY(launch_permute(w.topk_idx, T, L.k, L.E, L.S, tile, w, s));
    BlockDotCapture cap_store;
    const BlockDotCapture* cap = nullptr;
    if (dbg && dbg->block_dots_out) {
        cap_store = BlockDotCapture{dbg->block_dots_out, dbg->block_dots_down ? 1 : 0, dbg->block_dots_group,
                                    dbg->block_dots_rb};
        cap = &cap_store;
    }
    if (ev0) MOE_TRY(record_event(ev0, s));
    if (tc)
        MOE_TRY(launch_gateup_tc(L, T, w, dbg ? dbg->h_out : nullptr, dev, tile, cap, s));
    else
        MOE_TRY(launch_gateup_dp4a(L, T, w, dbg ? dbg->h_out : nullptr, dev, cap, s));
    if (ev1) MOE_TRY(record_event(ev1, s));
    if (tc)
        MOE_TRY(launch_down_tc(L, T, w, y, dev, tile, cap, s));
    else
        MOE_TRY(launch_down_dp4a(L, T, w, y, dev, cap, s));
    return MOE_Q4_OK;
}

int check_device() {
    DeviceInfo dev;
    return current_device(&dev);
}

}  // namespace moeq4

using namespace moeq4;

extern "C" {

const char* moe_q4_last_cuda_error(void) {
    return g_last_cuda_error == cudaSuccess ? "no CUDA error" : cudaGetErrorString(g_last_cuda_error);
}

const char* moe_q4_status_string(int status) {
    switch (status) {
        case MOE_Q4_OK: return "ok";
        case MOE_Q4_ERR_INVALID_ARG: return "invalid argument";
        case MOE_Q4_ERR_SHAPE: return "hidden and ffn must be positive multiples of 256 (at most 16384)";
        case MOE_Q4_ERR_ALIGN: return "pointer not 16-byte aligned (workspace: 256-byte)";
        case MOE_Q4_ERR_WORKSPACE: return "workspace too small";
        case MOE_Q4_ERR_ARCH: return "device is not compute capability 10.0 (sm_100a)";
        case MOE_Q4_ERR_CUDA: return "CUDA runtime error";
        case MOE_Q4_ERR_OVERLAP: return "output overlaps an input or the workspace";
        default: return "unknown status";
    }
}

int moe_q4_quantize_act(const float* x, int64_t T, int32_t H, int8_t* q, uint16_t* d, uint32_t* status,
                        moe_q4_stream_t stream) {
    if (T < 0 || T > T_LIMIT || H <= 0 || H % QK) return MOE_Q4_ERR_INVALID_ARG;
    if (T == 0) return MOE_Q4_OK;
    if (!x || !q || !d) return MOE_Q4_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(d, 2) || (status && !aligned(status, 4)))
        return MOE_Q4_ERR_ALIGN;
    DeviceInfo dev;
    int rc = current_device(&dev);
    if (rc) return rc;
    return cuda_rc(launch_quantize(x, T, H, q, d, status, nullptr, reinterpret_cast<cudaStream_t>(stream)));
}

int moe_q4_route(const moe_q4_layer* L, const float* x, int64_t T, int32_t* topk_idx, float* topk_w, float* logits,
                 moe_q4_stream_t stream) {
    int rc = check_layer(L);
    if (rc) return rc;
    if (T < 0 || T > T_LIMIT) return MOE_Q4_ERR_INVALID_ARG;
    if (T == 0) return MOE_Q4_OK;
    if (!x || !topk_idx || !topk_w || !logits) return MOE_Q4_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(topk_idx, 4) || !aligned(topk_w, 4) || !aligned(logits, 4))
        return MOE_Q4_ERR_ALIGN;
    DeviceInfo dev;
    rc = current_device(&dev);
    if (rc) return rc;
    const LayerView v = view(L);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    MOE_TRY(launch_router_logits(v, x, T, logits, nullptr, s));
    MOE_TRY(launch_topk(logits, T, v.E, v.k, topk_idx, topk_w, nullptr, s));
    return MOE_Q4_OK;
}

size_t moe_q4_ffn_workspace_bytes(const moe_q4_layer* L, int64_t T_max) {
    if (check_layer(L) || T_max < 0 || T_max > T_LIMIT) return 0;
    size_t off[WS_COUNT];
    layout(view(L), std::max<int64_t>(T_max, 1), off);
    return off[WS_TOTAL];
}

int moe_q4_workspace_layout(const moe_q4_layer* L, int64_t T, size_t* offsets, int n) {
    int rc = check_layer(L);
    if (rc) return rc;
    if (T < 0 || T > T_LIMIT || !offsets || n < 0) return MOE_Q4_ERR_INVALID_ARG;
    size_t off[WS_COUNT];
    layout(view(L), std::max<int64_t>(T, 1), off);
    for (int i = 0; i < n && i < WS_COUNT; ++i) offsets[i] = off[i];
    return MOE_Q4_OK;
}

int moe_q4_ffn_forward(const moe_q4_layer* L, const float* x, int64_t T, float* y, void* workspace,
                       size_t ws_bytes, moe_q4_stream_t stream) {
    return forward_impl(L, x, T, y, workspace, ws_bytes, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

int moe_q4_ffn_forward_debug(const moe_q4_layer* L, const float* x, int64_t T, float* y, void* workspace,
                             size_t ws_bytes, const moe_q4_debug* dbg, moe_q4_stream_t stream) {
    if (dbg && (dbg->path < MOE_Q4_PATH_AUTO || dbg->path > MOE_Q4_PATH_TENSOR_CORE_N64)) return MOE_Q4_ERR_INVALID_ARG;
    return forward_impl(L, x, T, y, workspace, ws_bytes, dbg, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

// The one-token host path's copy-in kernel may read x_host before the kernel
// ahead of it on the stream has finished (see decode_copy_in_kernel), if that
// kernel lets its dependents launch early.  Of this library's kernels, the
// one that can then still be writing host memory is the previous call's
// copy-out kernel on the same stream; a caller's kernel that writes x_host
// must not release its dependents early (include/moe_q4.h).  So x_host is
// read early unless it overlaps the previous host call's y_host, tracked per
// stream here.
namespace {
std::mutex g_host_y_mu;
std::unordered_map<cudaStream_t, std::pair<uintptr_t, uintptr_t>> g_host_y;   // [begin, end)
}  // namespace

static bool x_host_read_early(cudaStream_t s, const float* x_host, const float* y_host, size_t bytes) {
    const uintptr_t xb = reinterpret_cast<uintptr_t>(x_host), yb = reinterpret_cast<uintptr_t>(y_host);
    std::lock_guard<std::mutex> lk(g_host_y_mu);
    auto it = g_host_y.find(s);
    const bool early = it == g_host_y.end() || xb + bytes <= it->second.first || it->second.second <= xb;
    g_host_y[s] = {yb, yb + bytes};
    return early;
}

// Any other kind of call on the stream ends with a copy or kernel that does
// not release the next launch early.
static void forget_host_y(cudaStream_t s) {
    std::lock_guard<std::mutex> lk(g_host_y_mu);
    g_host_y.erase(s);
}

extern "C" {

size_t moe_q4_ffn_host_workspace_bytes(const moe_q4_layer* L, int64_t T_max) {
    const size_t base = moe_q4_ffn_workspace_bytes(L, T_max);
    if (!base) return 0;
    const size_t xy = align256(sizeof(float) * (size_t)(std::max<int64_t>(T_max, 1) * L->hidden));
    return base + 2 * xy;
}

int moe_q4_ffn_forward_host(const moe_q4_layer* L, const float* x_host, int64_t T, float* y_host, void* workspace,
                            size_t ws_bytes, moe_q4_stream_t stream) {
    int rc = check_layer(L);
    if (rc) return rc;
    if (T < 0 || T > T_LIMIT) return MOE_Q4_ERR_INVALID_ARG;
    if (T == 0) return MOE_Q4_OK;
    if (!x_host || !y_host || !workspace) return MOE_Q4_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return MOE_Q4_ERR_ALIGN;
    size_t off[WS_COUNT];
    layout(view(L), T, off);
    const size_t xy = align256(sizeof(float) * (size_t)(T * L->hidden));
    if (ws_bytes < off[WS_TOTAL] + 2 * xy) return MOE_Q4_ERR_WORKSPACE;
    char* base = static_cast<char*>(workspace);
    float* x_dev = reinterpret_cast<float*>(base + off[WS_TOTAL]);
    float* y_dev = reinterpret_cast<float*>(base + off[WS_TOTAL] + xy);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t bytes = sizeof(float) * (size_t)(T * L->hidden);
    DeviceInfo dev;
    rc = current_device(&dev);
    if (rc) return rc;
    // one token with page-locked x and y: kernels of the decode chain copy x
    // in and y out over the bus, so the call stays one programmatic-launch
    // chain (a copy node would end it)
    const LayerView Lv = view(L);
    if (T == 1 && decode_eligible(Lv, T, dev) && aligned(x_host, 16) && aligned(y_host, 16) && pinned_host(x_host) &&
        pinned_host(y_host)) {
        const Workspace w = carve(workspace, off);
        const bool early = x_host_read_early(s, x_host, y_host, bytes);
        return cuda_rc(launch_decode(Lv, x_dev, y_dev, w, nullptr, dev, nullptr, nullptr, false, true, nullptr,
                                     x_host, y_host, early, s));
    }
    forget_host_y(s);
    MOE_TRY(cudaMemcpyAsync(x_dev, x_host, bytes, cudaMemcpyHostToDevice, s));
    rc = forward_impl(L, x_dev, T, y_dev, workspace, off[WS_TOTAL], nullptr, s);
    if (rc) return rc;
    MOE_TRY(cudaMemcpyAsync(y_host, y_dev, bytes, cudaMemcpyDeviceToHost, s));
    return MOE_Q4_OK;
}

int moe_q4_residual_rmsnorm(float* x, const float* y, int64_t T, int32_t H, float eps, float* xn,
                            moe_q4_stream_t stream) {
    if (T < 0 || T > T_LIMIT || H <= 0 || H % 256 || !(eps >= 0.0f) || !(eps < INFINITY))
        return MOE_Q4_ERR_INVALID_ARG;
    if (T == 0) return MOE_Q4_OK;
    if (!x) return MOE_Q4_ERR_INVALID_ARG;
    if (!aligned(x, 16) || (y && !aligned(y, 16)) || (xn && !aligned(xn, 16))) return MOE_Q4_ERR_ALIGN;
    const size_t bytes = sizeof(float) * (size_t)T * (size_t)H;
    if ((y && overlap(x, bytes, y, bytes)) || (xn && overlap(x, bytes, xn, bytes)) ||
        (xn && y && overlap(y, bytes, xn, bytes)))
        return MOE_Q4_ERR_OVERLAP;
    DeviceInfo dev;
    int rc = current_device(&dev);
    if (rc) return rc;
    return cuda_rc(launch_residual_rmsnorm(x, y, T, H, eps, xn, reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_q4_stack_workspace_bytes(const moe_q4_layer* L, int64_t T_max) {
    const size_t base = moe_q4_ffn_workspace_bytes(L, T_max);
    if (!base) return 0;
    const size_t xy = align256(sizeof(float) * (size_t)(std::max<int64_t>(T_max, 1) * L->hidden));
    return 2 * xy + base;
}

int moe_q4_stack_forward(const moe_q4_layer* layers, int32_t n_layers, float* x, int64_t T, float eps,
                         void* workspace, size_t ws_bytes, moe_q4_stream_t stream) {
    if (!layers || n_layers < 1 || !(eps >= 0.0f) || !(eps < INFINITY)) return MOE_Q4_ERR_INVALID_ARG;
    for (int32_t l = 0; l < n_layers; ++l) {
        const int rc = check_layer(&layers[l]);
        if (rc) return rc;
        const moe_q4_layer& a = layers[0];
        const moe_q4_layer& b = layers[l];
        if (a.hidden != b.hidden || a.ffn != b.ffn || a.n_experts != b.n_experts || a.top_k != b.top_k ||
            (a.has_shared != 0) != (b.has_shared != 0))
            return MOE_Q4_ERR_SHAPE;
    }
    if (T < 0 || T > T_LIMIT) return MOE_Q4_ERR_INVALID_ARG;
    if (T == 0) return MOE_Q4_OK;
    if (!x || !workspace) return MOE_Q4_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(workspace, 256)) return MOE_Q4_ERR_ALIGN;
    const int32_t H = layers[0].hidden;
    const size_t xy = align256(sizeof(float) * (size_t)(T * H));
    size_t off[WS_COUNT];
    layout(view(&layers[0]), T, off);
    if (ws_bytes < 2 * xy + off[WS_TOTAL]) return MOE_Q4_ERR_WORKSPACE;
    if (overlap(x, sizeof(float) * (size_t)(T * H), workspace, 2 * xy + off[WS_TOTAL])) return MOE_Q4_ERR_OVERLAP;
    char* base = static_cast<char*>(workspace);
    float* xn = reinterpret_cast<float*>(base);
    float* y = reinterpret_cast<float*>(base + xy);
    void* lws = base + 2 * xy;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    DeviceInfo dev;
    int rc0 = current_device(&dev);
    if (rc0) return rc0;
    // one status word for the whole call: cleared here, then every layer's
    // kernels OR their conditions into it
    MOE_TRY(cudaMemsetAsync(static_cast<char*>(lws) + off[WS_STATUS], 0, 16, s));
    for (int32_t l = 0; l < n_layers; ++l) {
        int rc = moe_q4_residual_rmsnorm(x, l ? y : nullptr, T, H, eps, xn, stream);
        if (rc) return rc;
        rc = forward_impl(&layers[l], xn, T, y, lws, off[WS_TOTAL], nullptr, s, /*clear_status=*/false);
        if (rc) return rc;
    }
    return moe_q4_residual_rmsnorm(x, y, T, H, eps, nullptr, stream);
}

size_t moe_q4_gemv_workspace_bytes(int64_t T, int32_t H) {
    if (T < 1 || T > 8 || H <= 0 || H % 256 || H > 16384) return 0;
    return 256 + align256((size_t)T * H) + align256((size_t)T * (H / QK) * 2);
}

int moe_q4_gemv(const uint8_t* W, int64_t N, int32_t H, const float* x, int64_t T, float* y, void* workspace,
                size_t ws_bytes, moe_q4_stream_t stream) {
    if (T < 0 || T > 8 || N < 1 || N > (int64_t(1) << 30)) return MOE_Q4_ERR_INVALID_ARG;
    if (H <= 0 || H % 256 || H > 16384) return MOE_Q4_ERR_SHAPE;
    if (T == 0) return MOE_Q4_OK;
    if (!W || !x || !y || !workspace) return MOE_Q4_ERR_INVALID_ARG;
    if (!aligned(W, 16) || !aligned(x, 16) || !aligned(y, 16) || !aligned(workspace, 256)) return MOE_Q4_ERR_ALIGN;
    const size_t need = moe_q4_gemv_workspace_bytes(T, H);
    if (ws_bytes < need) return MOE_Q4_ERR_WORKSPACE;
    const size_t ybytes = sizeof(float) * (size_t)T * (size_t)N, xbytes = sizeof(float) * (size_t)T * H;
    if (overlap(y, ybytes, x, xbytes) || overlap(y, ybytes, workspace, need)) return MOE_Q4_ERR_OVERLAP;
    DeviceInfo dev;
    int rc = current_device(&dev);
    if (rc) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char* base = static_cast<char*>(workspace);
    uint32_t* status = reinterpret_cast<uint32_t*>(base);
    int8_t* qa = reinterpret_cast<int8_t*>(base + 256);
    uint16_t* da = reinterpret_cast<uint16_t*>(base + 256 + align256((size_t)T * H));
    MOE_TRY(cudaMemsetAsync(status, 0, sizeof(uint32_t), s));
    MOE_TRY(launch_quantize(x, T, H, qa, da, status, nullptr, s));
    return cuda_rc(launch_gemv_dp4a(W, N, H, qa, da, (int)T, y, status, dev, s));
}

// Staging copy of a layer's experts on the device: gate [E] | up [E] | down [E]
// | shared gate | shared up | shared down, each region 256-byte aligned.
static void staging_layout(const moe_q4_layer* L, size_t off[7]) {
    const size_t gu = (size_t)L->ffn * (L->hidden / QK) * Q4_BYTES;
    const size_t dn = (size_t)L->hidden * (L->ffn / QK) * Q4_BYTES;
    const size_t E = (size_t)L->n_experts, S = L->has_shared ? 1 : 0;
    const size_t sz[6] = {E * gu, E * gu, E * dn, S * gu, S * gu, S * dn};
    off[0] = 0;
    for (int i = 0; i < 6; ++i) off[i + 1] = off[i] + align256(sz[i]);
}

size_t moe_q4_staging_bytes(const moe_q4_layer* L) {
    if (check_layer(L)) return 0;
    size_t off[7];
    staging_layout(L, off);
    return off[6];
}

int moe_q4_ffn_forward_streamed(const moe_q4_layer* L, const float* x, int64_t T, float* y, void* workspace,
                                size_t ws_bytes, void* staging, size_t staging_bytes, moe_q4_stream_t stream) {
    int rc = check_layer(L);
    if (rc) return rc;
    if (T < 0 || T > T_LIMIT) return MOE_Q4_ERR_INVALID_ARG;
    if (T == 0) return MOE_Q4_OK;
    if (!x || !y || !workspace || !staging) return MOE_Q4_ERR_INVALID_ARG;
    if (!aligned(staging, 256) || !aligned(workspace, 256)) return MOE_Q4_ERR_ALIGN;
    size_t soff[7];
    staging_layout(L, soff);
    if (staging_bytes < soff[6]) return MOE_Q4_ERR_WORKSPACE;
    DeviceInfo dev;
    rc = current_device(&dev);
    if (rc) return rc;
    // the experts must be page-locked host memory (read by the GPU through
    // unified addressing); the router weights and x, y device memory
    const void* host_mats[6] = {L->w_gate, L->w_up, L->w_down, L->sh_gate, L->sh_up, L->sh_down};
    for (int i = 0; i < (L->has_shared ? 6 : 3); ++i)
        if (!pinned_host(host_mats[i])) return MOE_Q4_ERR_INVALID_ARG;
    if (!on_device(L->w_router) || (L->router_bias && !on_device(L->router_bias)) || !on_device(x) ||
        !on_device(y) || !on_device(staging) || !on_device(workspace))
        return MOE_Q4_ERR_INVALID_ARG;
    const LayerView Lv = view(L);
    size_t off[WS_COUNT];
    layout(Lv, T, off);
    if (ws_bytes < off[WS_TOTAL]) return MOE_Q4_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const Workspace w = carve(workspace, off);
    // routing and its per-expert counts, on the device
    MOE_TRY(launch_router_logits(Lv, x, T, w.logits, w.status, s));
    MOE_TRY(launch_topk(w.logits, T, Lv.E, Lv.k, w.topk_idx, w.topk_w, w.status, s));
    MOE_TRY(launch_permute(w.topk_idx, T, Lv.k, Lv.E, Lv.S, DP4A_TT, w, s));
    uint8_t* st = static_cast<uint8_t*>(staging);
    StageParams sp;
    sp.E = Lv.E; sp.S = Lv.S;
    sp.gu_bytes = (size_t)Lv.F * (Lv.H / QK) * Q4_BYTES;
    sp.dn_bytes = (size_t)Lv.H * (Lv.F / QK) * Q4_BYTES;
    sp.cnt = w.cnt;
    sp.h_gate = L->w_gate; sp.h_up = L->w_up; sp.h_down = L->w_down;
    sp.h_sh_gate = L->sh_gate; sp.h_sh_up = L->sh_up; sp.h_sh_down = L->sh_down;
    sp.d_gate = st + soff[0]; sp.d_up = st + soff[1]; sp.d_down = st + soff[2];
    sp.d_sh_gate = st + soff[3]; sp.d_sh_up = st + soff[4]; sp.d_sh_down = st + soff[5];
    MOE_TRY(launch_stage_experts(sp, dev, s));
    moe_q4_layer Ls = *L;
    Ls.w_gate = sp.d_gate; Ls.w_up = sp.d_up; Ls.w_down = sp.d_down;
    if (L->has_shared) {
        Ls.sh_gate = sp.d_sh_gate; Ls.sh_up = sp.d_sh_up; Ls.sh_down = sp.d_sh_down;
    }
    return forward_impl(&Ls, x, T, y, workspace, ws_bytes, nullptr, s);
}

int moe_q4_test_override_device(int32_t enable, int32_t major, int32_t minor) {
    g_cc_override[1] = major;
    g_cc_override[2] = minor;
    g_cc_override[0] = enable ? 1 : 0;
    return MOE_Q4_OK;
}

int moe_q4_block_dots(const uint8_t* w_blocks, const int8_t* qa, int64_t n, int32_t* out, moe_q4_stream_t stream) {
    if (n < 0 || n > (int64_t(1) << 31) || (n % 8)) return MOE_Q4_ERR_INVALID_ARG;
    if (n == 0) return MOE_Q4_OK;
    if (!w_blocks || !qa || !out) return MOE_Q4_ERR_INVALID_ARG;
    if (!aligned(w_blocks, 16) || !aligned(qa, 16) || !aligned(out, 4)) return MOE_Q4_ERR_ALIGN;
    DeviceInfo dev;
    int rc = current_device(&dev);
    if (rc) return rc;
    return cuda_rc(launch_block_dots(w_blocks, qa, n, out, reinterpret_cast<cudaStream_t>(stream)));
}

int moe_q4_rescale_ceiling(int32_t int8_operands, int32_t iters, float* sink, int64_t* elements,
                           moe_q4_stream_t stream) {
    if (iters < 1 || iters > (1 << 20) || !sink || !elements) return MOE_Q4_ERR_INVALID_ARG;
    if (!aligned(sink, 4)) return MOE_Q4_ERR_ALIGN;
    DeviceInfo dev;
    int rc = current_device(&dev);
    if (rc) return rc;
    return cuda_rc(launch_rescale_ceiling(int8_operands != 0, iters, sink, dev, elements,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
