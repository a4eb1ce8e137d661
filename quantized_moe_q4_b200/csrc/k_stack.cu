// k_stack.cu -- the glue between the layers of a stack of MoE layers.
//
// The page runs its MoE layers one after another ("A 35B Hybrid-Attention
// Mixture-of-Experts Model on a 6GB 2011 GPU", Dutch technical summary,
// Methodologie 1: expert weights are streamed layer by layer) and fixes no
// step between them.  The multi-layer workload joins them by a residual add;
// without a normalisation the activations grow by about 25x per layer and the
// binary16 Q8_0 scales overflow within a few layers, so the step taken is
//   x <- x + y_prev (binary32, one rounding),  xn = x / sqrt(mean_h x^2 + eps)
// with a unit-gain RMSNorm whose mean of squares is accumulated in binary64
// (every square of a binary32 value is exact there) and whose division is the
// IEEE binary64 one, rounded once to binary32.
#include "common.cuh"
#include "launch.h"

namespace moeq4 {

namespace {
constexpr int ROWS_PER_CTA = 4;  // one warp per row
}

__global__ void __launch_bounds__(32 * ROWS_PER_CTA)
    residual_rmsnorm_kernel(float* __restrict__ x, const float* __restrict__ y, int64_t T, int H, float eps,
                            float* __restrict__ xn) {
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * ROWS_PER_CTA + (threadIdx.x >> 5);
    if (t >= T) return;
    float* xr = x + t * H;
    const float* yr = y ? y + t * H : nullptr;
    double ss = 0.0;
    for (int h = 4 * lane; h < H; h += 128) {
        float4 v = *reinterpret_cast<const float4*>(xr + h);
        if (yr) {
            const float4 u = *reinterpret_cast<const float4*>(yr + h);
            v.x = __fadd_rn(v.x, u.x);
            v.y = __fadd_rn(v.y, u.y);
            v.z = __fadd_rn(v.z, u.z);
            v.w = __fadd_rn(v.w, u.w);
            *reinterpret_cast<float4*>(xr + h) = v;
        }
        ss = __fma_rn((double)v.x, (double)v.x, ss);
        ss = __fma_rn((double)v.y, (double)v.y, ss);
        ss = __fma_rn((double)v.z, (double)v.z, ss);
        ss = __fma_rn((double)v.w, (double)v.w, ss);
    }
    if (!xn) return;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const double rms = __dsqrt_rn(__dadd_rn(__ddiv_rn(ss, (double)H), (double)eps));
    float* nr = xn + t * H;
    for (int h = 4 * lane; h < H; h += 128) {
        const float4 v = *reinterpret_cast<const float4*>(xr + h);
        float4 o;
        o.x = __double2float_rn(__ddiv_rn((double)v.x, rms));
        o.y = __double2float_rn(__ddiv_rn((double)v.y, rms));
        o.z = __double2float_rn(__ddiv_rn((double)v.z, rms));
        o.w = __double2float_rn(__ddiv_rn((double)v.w, rms));
        *reinterpret_cast<float4*>(nr + h) = o;
    }
}

cudaError_t launch_residual_rmsnorm(float* x, const float* y, int64_t T, int H, float eps, float* xn,
                                    cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const int64_t grid = (T + ROWS_PER_CTA - 1) / ROWS_PER_CTA;
    residual_rmsnorm_kernel<<<(unsigned)grid, 32 * ROWS_PER_CTA, 0, s>>>(x, y, T, H, eps, xn);
    return cudaGetLastError();
}

}  // namespace moeq4
