// k_route.cu -- router logits and top-k softmax.
//
// The pages ("A 35B Hybrid-Attention Mixture-of-Experts Model on a 6GB 2011
// GPU", Dutch technical summary, Methodologie 1) name the MoE routing that
// feeds the grouped 4-bit GEMM; the rule implemented is: logits = x.Wr^T
// (+ bias) in binary32, the k largest logits per token in descending order
// (equal logits: lower expert index first), weights = softmax over those k.
#include <float.h>

#include "common.cuh"
#include "launch.h"

namespace moeq4 {

// ---------------------------------------------------------------------------
// Logits, up to a few hundred tokens: one CTA per (expert, tile of RT tokens);
// its 8 warps split H into 8 slices, and the slices' sums are added in a fixed
// order (deterministic), so even a handful of tokens spreads over E CTAs.
// ---------------------------------------------------------------------------
constexpr int RT = 8;

__global__ void __launch_bounds__(256) router_logits_split(const float* __restrict__ x, int T, int H,
                                                            const float* __restrict__ Wr,
                                                            const float* __restrict__ bias, int E,
                                                            float* __restrict__ logits,
                                                            uint32_t* __restrict__ status_clear) {
    if (status_clear && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *status_clear = 0u;
    __shared__ float part[8][RT];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x;
    const int t0 = blockIdx.y * RT;
    const int slice = H / 8;                      // a multiple of 32 floats
    const int h4_0 = warp * (slice >> 2), h4_1 = h4_0 + (slice >> 2);
    const float4* wr = reinterpret_cast<const float4*>(Wr + (size_t)e * H);
    float acc[RT];
#pragma unroll
    for (int t = 0; t < RT; ++t) acc[t] = 0.0f;
    for (int h4 = h4_0 + lane; h4 < h4_1; h4 += 32) {
        const float4 w = __ldg(wr + h4);
#pragma unroll
        for (int t = 0; t < RT; ++t) {
            if (t0 + t < T) {
                const float4 v = __ldg(reinterpret_cast<const float4*>(x + (size_t)(t0 + t) * H) + h4);
                acc[t] = fmaf(w.x, v.x, acc[t]);
                acc[t] = fmaf(w.y, v.y, acc[t]);
                acc[t] = fmaf(w.z, v.z, acc[t]);
                acc[t] = fmaf(w.w, v.w, acc[t]);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < RT; ++t) {
        float a = acc[t];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (lane == 0) part[warp][t] = a;
    }
    __syncthreads();
    if (threadIdx.x < RT && t0 + (int)threadIdx.x < T) {
        float a = part[0][threadIdx.x];
#pragma unroll
        for (int w = 1; w < 8; ++w) a += part[w][threadIdx.x];
        logits[(size_t)(t0 + threadIdx.x) * E + e] = a + (bias ? __ldg(bias + e) : 0.0f);
    }
}

// ---------------------------------------------------------------------------
// Logits, many tokens: 64x64 output tile per CTA, K step 16, 4x4 per thread.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) router_logits_tiled(const float* __restrict__ x, int T, int H,
                                                            const float* __restrict__ Wr,
                                                            const float* __restrict__ bias, int E,
                                                            float* __restrict__ logits,
                                                            uint32_t* __restrict__ status_clear) {
    if (status_clear && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *status_clear = 0u;
    __shared__ __align__(16) float As[16][68];
    __shared__ __align__(16) float Bs[16][68];
    const int tid = threadIdx.x;
    const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
    const int tm = tid >> 4, tn = tid & 15;
    const int lr = tid >> 2, lc = (tid & 3) * 4;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
    const bool arow = (m0 + lr) < T, brow = (n0 + lr) < E;
    const float* xa = x + (size_t)(arow ? m0 + lr : 0) * H + lc;
    const float* wb = Wr + (size_t)(brow ? n0 + lr : 0) * H + lc;
    for (int k0 = 0; k0 < H; k0 += 16) {
        const float4 a = arow ? __ldg(reinterpret_cast<const float4*>(xa + k0)) : make_float4(0, 0, 0, 0);
        const float4 b = brow ? __ldg(reinterpret_cast<const float4*>(wb + k0)) : make_float4(0, 0, 0, 0);
        As[lc + 0][lr] = a.x; As[lc + 1][lr] = a.y; As[lc + 2][lr] = a.z; As[lc + 3][lr] = a.w;
        Bs[lc + 0][lr] = b.x; Bs[lc + 1][lr] = b.y; Bs[lc + 2][lr] = b.z; Bs[lc + 3][lr] = b.w;
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            const float4 av = *reinterpret_cast<const float4*>(&As[kk][tm * 4]);
            const float4 bv = *reinterpret_cast<const float4*>(&Bs[kk][tn * 4]);
            const float ar[4] = {av.x, av.y, av.z, av.w};
            const float br[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(ar[i], br[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = m0 + tm * 4 + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = n0 + tn * 4 + j;
            if (e < E) logits[(size_t)t * E + e] = acc[i][j] + (bias ? __ldg(bias + e) : 0.0f);
        }
    }
}

// ---------------------------------------------------------------------------
// Top-k + softmax over the chosen logits: one warp per token, E <= 256.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) topk_softmax_kernel(const float* __restrict__ logits, int T, int E,
                                                            int k, int32_t* __restrict__ idx,
                                                            float* __restrict__ w) {
    const int lane = threadIdx.x & 31;
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = i * 32 + lane;
        v[i] = (e < E) ? logits[(size_t)t * E + e] : -FLT_MAX;
    }
    uint32_t taken = 0;
    for (int i = 0; i < 8; ++i)
        if (i * 32 + lane >= E) taken |= 1u << i;
    float my_l = 0.0f;
    int my_e = 0;
    for (int j = 0; j < k; ++j) {
        float bv = -FLT_MAX;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = i * 32 + lane;
            if (!((taken >> i) & 1u) && (v[i] > bv || (v[i] == bv && e < be))) {
                bv = v[i];
                be = e;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (ov > bv || (ov == bv && oe < be)) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == j) {
            my_l = bv;
            my_e = be;
        }
    }
    const float lmax = __shfl_sync(0xffffffffu, my_l, 0);
    const float ex = (lane < k) ? expf(my_l - lmax) : 0.0f;
    float z = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (lane < k) {
        idx[(size_t)t * k + lane] = my_e;
        w[(size_t)t * k + lane] = __fdiv_rn(ex, z);
    }
}

cudaError_t launch_router_logits(const LayerView& L, const float* x, int64_t T, float* logits,
                                 uint32_t* status_clear, cudaStream_t s) {
    if (T <= 512) {
        // x rows are re-read once per expert from L2 (at most 512 x H x 4 x E bytes)
        dim3 grid((unsigned)L.E, (unsigned)ceil_div(T, RT));
        router_logits_split<<<grid, 256, 0, s>>>(x, (int)T, L.H, L.w_router, L.router_bias, L.E, logits,
                                                 status_clear);
    } else {
        dim3 grid((unsigned)ceil_div(L.E, 64), (unsigned)ceil_div(T, 64));
        router_logits_tiled<<<grid, 256, 0, s>>>(x, (int)T, L.H, L.w_router, L.router_bias, L.E, logits,
                                                 status_clear);
    }
    return cudaGetLastError();
}

cudaError_t launch_topk(const float* logits, int64_t T, int E, int k, int32_t* idx, float* w,
                        cudaStream_t s) {
    const unsigned blocks = (unsigned)ceil_div(T, 8);
    topk_softmax_kernel<<<blocks, 256, 0, s>>>(logits, (int)T, E, k, idx, w);
    return cudaGetLastError();
}

}  // namespace moeq4
