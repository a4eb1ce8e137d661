// k_stage.cu -- host-streamed experts: copy the experts a call activates from
// pinned host memory into a device staging copy of the layer.
//
// The page keeps the 10.5 GB of expert weights in page-locked host memory and
// streams them to the 6 GB GPU layer by layer ("A 35B Hybrid-Attention
// Mixture-of-Experts Model on a 6GB 2011 GPU", Dutch technical summary,
// Methodologie 1 and 2).  Here only the experts that the call's routing
// selects (plus the shared expert) cross the link: the copy kernel reads the
// per-expert pair counts of the permutation on the device, so no host round
// trip sits between routing and the copies, and the whole call stays
// capturable in a CUDA graph.  The GPU reads the pinned host pages directly
// (unified addressing) with 16-byte loads from many CTAs at once.
#include "common.cuh"
#include "launch.h"

namespace moeq4 {

namespace {
constexpr size_t CHUNK = 64 * 1024;  // bytes a CTA copies per work item
}

__global__ void __launch_bounds__(256) stage_experts_kernel(StageParams p) {
    const int ngroups = p.E + p.S;
    const int64_t per_gu = (int64_t)((p.gu_bytes + CHUNK - 1) / CHUNK);
    const int64_t per_dn = (int64_t)((p.dn_bytes + CHUNK - 1) / CHUNK);
    const int64_t per_group = 2 * per_gu + per_dn;
    const int64_t n_items = (int64_t)ngroups * per_group;
    for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int g = (int)(item / per_group);
        if (g < p.E && p.cnt[g] == 0) continue;   // expert not selected by any token
        int64_t r = item - (int64_t)g * per_group;
        const uint8_t* src;
        uint8_t* dst;
        size_t bytes;
        const bool sh = g >= p.E;
        if (r < 2 * per_gu) {
            const int mat = (int)(r / per_gu);
            r -= (int64_t)mat * per_gu;
            const uint8_t* base = sh ? (mat ? p.h_sh_up : p.h_sh_gate) : (mat ? p.h_up : p.h_gate) + (size_t)g * p.gu_bytes;
            uint8_t* dbase = sh ? (mat ? p.d_sh_up : p.d_sh_gate) : (mat ? p.d_up : p.d_gate) + (size_t)g * p.gu_bytes;
            src = base + r * CHUNK;
            dst = dbase + r * CHUNK;
            bytes = min(CHUNK, p.gu_bytes - (size_t)r * CHUNK);
        } else {
            r -= 2 * per_gu;
            const uint8_t* base = sh ? p.h_sh_down : p.h_down + (size_t)g * p.dn_bytes;
            uint8_t* dbase = sh ? p.d_sh_down : p.d_down + (size_t)g * p.dn_bytes;
            src = base + r * CHUNK;
            dst = dbase + r * CHUNK;
            bytes = min(CHUNK, p.dn_bytes - (size_t)r * CHUNK);
        }
        // matrix sizes are multiples of 16 bytes (rows of 144-byte multiples)
        const int4* s4 = reinterpret_cast<const int4*>(src);
        int4* d4 = reinterpret_cast<int4*>(dst);
        const int n4 = (int)(bytes / 16);
        for (int i = threadIdx.x; i < n4; i += blockDim.x) d4[i] = s4[i];
    }
}

cudaError_t launch_stage_experts(const StageParams& p, const DeviceInfo& dev, cudaStream_t s) {
    stage_experts_kernel<<<(unsigned)(dev.sm_count * 4), 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace moeq4
