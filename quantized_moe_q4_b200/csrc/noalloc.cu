// noalloc.cu -- moe_q4_ffn_forward_noalloc: the whole layer with its scratch in
// a fixed device array owned by the library, for callers that cannot allocate.
//
// Who needs it: code that must not call cudaMalloc or an allocator in the
// middle of a step -- a host runtime or plugin whose device memory is
// reserved up front by someone else, a latency-critical decode loop that
// cannot afford cudaMalloc's implicit device synchronisation, or code that
// builds CUDA graphs and may not allocate while doing so.  Such a caller still
// owns x and y; only the scratch moves into the library.
//
// Cost: MOE_Q4_NOALLOC_SCRATCH_BYTES of device memory on each GPU where the
// entry is used, until the process exits.  With CUDA's default lazy module
// loading the array is placed on a device by the first call there (its
// address lookup loads the module); with lazy loading off, when the
// library's module is loaded into that device's context.
#include <mutex>

#include "moe_q4.h"
#include "launch.h"

namespace {

constexpr size_t kScratchBytes = MOE_Q4_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// The scratch.  In host code this name is only a stand-in for the device
// array (using it as a pointer would read host memory or fault); the device
// address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

void* g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch on the current device, looked up once per
// device with that device current.  Returns MOE_Q4_OK or MOE_Q4_ERR_CUDA.
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_Q4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MOE_Q4_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return MOE_Q4_OK;
}

}  // namespace

extern "C" int moe_q4_ffn_forward_noalloc(const moe_q4_layer* L, const float* x, int64_t T, float* y,
                                          moe_q4_stream_t stream) {
    const size_t need = moe_q4_ffn_workspace_bytes(L, T);
    // An invalid layer or T: the forward's own checks name the error and
    // return before touching the (absent) workspace.
    if (need == 0) return moe_q4_ffn_forward(L, x, T, y, nullptr, 0, stream);
    if (need > kScratchBytes) return MOE_Q4_ERR_WORKSPACE;
    if (T == 0) return MOE_Q4_OK;
    // the architecture first: on another device the lookup itself would fail
    int rc = moeq4::check_device();
    if (rc != MOE_Q4_OK) return rc;
    void* scratch = nullptr;
    rc = scratch_address(&scratch);
    if (rc != MOE_Q4_OK) return rc;
    return moe_q4_ffn_forward(L, x, T, y, scratch, kScratchBytes, stream);
}
