// k_route.cu -- router logits and top-k softmax.
//
// The pages ("A 35B Hybrid-Attention Mixture-of-Experts Model on a 6GB 2011
// GPU", Dutch technical summary, Methodologie 1) name the MoE routing that
// feeds the grouped 4-bit GEMM; the rule implemented is: logits = x.Wr^T
// (+ bias) in binary32, the k largest logits per token in descending order
// (equal logits: lower expert index first), weights = softmax over those k.
#include <float.h>

#include <cooperative_groups.h>

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
// Logits, many tokens: a 64-token x 64-expert output tile per cluster of RKS
// CTAs.  CTA z of the cluster covers one contiguous slice of H (whole 32-wide
// chunks), with the next chunk's loads in flight while the current one is
// multiplied (4x4 outputs a thread); the RKS partial tiles are then added
// through distributed shared memory in rank order, each CTA finishing a
// quarter of the tile, so the sum order is fixed (deterministic).  Splitting
// H spreads a 947-token batch over 120 SMs instead of 30, and the prefetch
// hides the L2 latency that a load-then-sync loop pays once per chunk.
// ---------------------------------------------------------------------------
constexpr int RKS = 4;     // CTAs per cluster (slices of H)
constexpr int RBK = 32;    // K chunk
constexpr int RLD = 68;    // padded row length of the staged tiles

__global__ void __cluster_dims__(1, 1, RKS) __launch_bounds__(256)
    router_logits_tiled(const float* __restrict__ x, int T, int H, const float* __restrict__ Wr,
                        const float* __restrict__ bias, int E, float* __restrict__ logits,
                        uint32_t* __restrict__ status_clear) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    if (status_clear && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) *status_clear = 0u;
    __shared__ __align__(16) float As[2][RBK][RLD];   // [buffer][k][token]
    __shared__ __align__(16) float Bs[2][RBK][RLD];   // [buffer][k][expert]
    const int tid = threadIdx.x;
    const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
    const int rank = (int)cluster.block_rank();
    const int tm = tid >> 4, tn = tid & 15;
    // loader: row lr of the tile, k offsets lc and lc + 16 of the chunk
    const int lr = tid >> 2, lc = (tid & 3) * 4;
    const bool arow = (m0 + lr) < T, brow = (n0 + lr) < E;
    const float* xa = x + (size_t)(arow ? m0 + lr : 0) * H + lc;
    const float* wb = Wr + (size_t)(brow ? n0 + lr : 0) * H + lc;
    const int nch = H / RBK;
    const int c0 = rank * nch / RKS, c1 = (rank + 1) * nch / RKS;

    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;

    float4 a0 = make_float4(0, 0, 0, 0), a1 = a0, b0 = a0, b1 = a0;
    auto load = [&](int c) {
        const int k0 = c * RBK;
        a0 = arow ? __ldg(reinterpret_cast<const float4*>(xa + k0)) : make_float4(0, 0, 0, 0);
        a1 = arow ? __ldg(reinterpret_cast<const float4*>(xa + k0 + 16)) : make_float4(0, 0, 0, 0);
        b0 = brow ? __ldg(reinterpret_cast<const float4*>(wb + k0)) : make_float4(0, 0, 0, 0);
        b1 = brow ? __ldg(reinterpret_cast<const float4*>(wb + k0 + 16)) : make_float4(0, 0, 0, 0);
    };
    auto stage = [&](int buf) {
        As[buf][lc + 0][lr] = a0.x; As[buf][lc + 1][lr] = a0.y; As[buf][lc + 2][lr] = a0.z; As[buf][lc + 3][lr] = a0.w;
        As[buf][lc + 16][lr] = a1.x; As[buf][lc + 17][lr] = a1.y; As[buf][lc + 18][lr] = a1.z; As[buf][lc + 19][lr] = a1.w;
        Bs[buf][lc + 0][lr] = b0.x; Bs[buf][lc + 1][lr] = b0.y; Bs[buf][lc + 2][lr] = b0.z; Bs[buf][lc + 3][lr] = b0.w;
        Bs[buf][lc + 16][lr] = b1.x; Bs[buf][lc + 17][lr] = b1.y; Bs[buf][lc + 18][lr] = b1.z; Bs[buf][lc + 19][lr] = b1.w;
    };
    if (c0 < c1) {
        load(c0);
        stage(0);
    }
    __syncthreads();
    for (int c = c0; c < c1; ++c) {
        const int buf = (c - c0) & 1;
        if (c + 1 < c1) load(c + 1);   // in flight while this chunk is multiplied
#pragma unroll
        for (int kk = 0; kk < RBK; ++kk) {
            const float4 av = *reinterpret_cast<const float4*>(&As[buf][kk][tm * 4]);
            const float4 bv = *reinterpret_cast<const float4*>(&Bs[buf][kk][tn * 4]);
            const float ar[4] = {av.x, av.y, av.z, av.w};
            const float br[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(ar[i], br[j], acc[i][j]);
        }
        // the other buffer was last read in the previous chunk, before the
        // barrier that ended it
        if (c + 1 < c1) stage(buf ^ 1);
        __syncthreads();
    }

    // this CTA's partial tile [token][expert] (stride 65) in the A staging area
    float* part = &As[0][0][0];
    static_assert(sizeof(As) >= 64 * 65 * sizeof(float), "partial tile fits the A staging area");
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) part[(tm * 4 + i) * 65 + tn * 4 + j] = acc[i][j];
    cluster.sync();
    // CTA `rank` adds rows 16 rank .. 16 rank + 15 of the RKS partials in rank order
    float* parts[RKS];
#pragma unroll
    for (int q = 0; q < RKS; ++q) parts[q] = cluster.map_shared_rank(part, q);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int idx = u * 256 + tid;            // 0 .. 1023 over 16 rows x 64 columns
        const int r = rank * 16 + (idx >> 6), col = idx & 63;
        float v = parts[0][r * 65 + col];
#pragma unroll
        for (int q = 1; q < RKS; ++q) v += parts[q][r * 65 + col];
        const int t = m0 + r, e = n0 + col;
        if (t < T && e < E) logits[(size_t)t * E + e] = v + (bias ? __ldg(bias + e) : 0.0f);
    }
    cluster.sync();   // the partials stay alive until every CTA of the cluster has read them
}

// ---------------------------------------------------------------------------
// Top-k + softmax over the chosen logits: one warp per token, E <= 256.
// A NaN logit ranks as -infinity (below every number; equal keys go to the
// lower expert index), so every pick is an expert in [0, E) whatever the
// logits hold; a NaN or infinite logit sets STATUS_NONFINITE_LOGIT in
// *status (if given), and the weights of such a token are then undefined.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) topk_softmax_kernel(const float* __restrict__ logits, int T, int E,
                                                            int k, int32_t* __restrict__ idx,
                                                            float* __restrict__ w, uint32_t* __restrict__ status) {
    const int lane = threadIdx.x & 31;
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    float v[8];
    bool nonfinite = false;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = i * 32 + lane;
        float l = (e < E) ? logits[(size_t)t * E + e] : -INFINITY;
        if (e < E && !isfinite(l)) nonfinite = true;
        v[i] = (l != l) ? -INFINITY : l;
    }
    if (status && __any_sync(0xffffffffu, nonfinite) && lane == 0) atomicOr(status, STATUS_NONFINITE_LOGIT);
    uint32_t taken = 0;
    for (int i = 0; i < 8; ++i)
        if (i * 32 + lane >= E) taken |= 1u << i;
    float my_l = 0.0f;
    int my_e = 0;
    for (int j = 0; j < k; ++j) {
        // every untaken expert beats the start value (-inf with an index
        // above any expert's), and k <= E leaves at least one untaken
        float bv = -INFINITY;
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
    if (T <= 128) {
        // x rows are re-read once per expert from L2 (at most 128 x H x 4 x E bytes)
        dim3 grid((unsigned)L.E, (unsigned)ceil_div(T, RT));
        router_logits_split<<<grid, 256, 0, s>>>(x, (int)T, L.H, L.w_router, L.router_bias, L.E, logits,
                                                 status_clear);
    } else {
        // grid.y holds the 64-token tiles, at most 65535 a launch: larger
        // batches take several launches over consecutive token ranges
        const int64_t max_tokens = (int64_t)65535 * 64;
        for (int64_t t0 = 0; t0 < T; t0 += max_tokens) {
            const int64_t Tc = (T - t0 < max_tokens) ? T - t0 : max_tokens;
            dim3 grid((unsigned)ceil_div(L.E, 64), (unsigned)ceil_div(Tc, 64), RKS);
            router_logits_tiled<<<grid, 256, 0, s>>>(x + t0 * L.H, (int)Tc, L.H, L.w_router, L.router_bias, L.E,
                                                     logits + t0 * L.E, t0 == 0 ? status_clear : nullptr);
        }
    }
    return cudaGetLastError();
}

cudaError_t launch_topk(const float* logits, int64_t T, int E, int k, int32_t* idx, float* w,
                        uint32_t* status, cudaStream_t s) {
    const unsigned blocks = (unsigned)ceil_div(T, 8);
    topk_softmax_kernel<<<blocks, 256, 0, s>>>(logits, (int)T, E, k, idx, w, status);
    return cudaGetLastError();
}

}  // namespace moeq4
