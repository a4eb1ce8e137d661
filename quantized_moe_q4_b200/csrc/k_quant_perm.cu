// k_quant_perm.cu -- Q8_0 activation quantisation and the token-to-expert
// permutation (histogram -> scan -> stable scatter).
//
// Q8_0 is the 8-bit activation format of the W4A8 kernel ("A 35B
// Hybrid-Attention Mixture-of-Experts Model on a 6GB 2011 GPU", Dutch technical
// summary, Methodologie 1 and 2).  The permutation groups the (token, slot)
// pairs by expert so the grouped 4-bit GEMM of Methodologie 1 sees each
// expert's tokens as one contiguous batch.
#include "common.cuh"
#include "launch.h"

namespace moeq4 {

// One warp per 32-value block, lane = element.  Optionally zeroes y (same
// [T][H] shape as x) so the down projection can accumulate into it.
__global__ void __launch_bounds__(256) quantize_q8_0_kernel(const float* __restrict__ x, int64_t nblocks,
                                                             int8_t* __restrict__ q,
                                                             uint16_t* __restrict__ d,
                                                             uint32_t* __restrict__ status,
                                                             float* __restrict__ y_zero) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t b = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); b < nblocks; b += nwarps) {
        const float v = __ldg(x + b * QK + lane);
        uint16_t db;
        bool ov;
        const int qi = q8_0_lane(v, db, ov);
        q[b * QK + lane] = (int8_t)qi;
        if (lane == 0) {
            d[b] = db;
            if (ov && status) atomicOr(status, STATUS_SCALE_OVERFLOW);
        }
        if (y_zero) y_zero[b * QK + lane] = 0.0f;
    }
}

cudaError_t launch_quantize(const float* x, int64_t T, int H, int8_t* q, uint16_t* d, uint32_t* status,
                            float* y_zero, cudaStream_t s) {
    const int64_t nblocks = T * (H / QK);
    int64_t ctas = ceil_div(nblocks, 8);
    if (ctas > 148 * 16) ctas = 148 * 16;
    quantize_q8_0_kernel<<<(unsigned)ctas, 256, 0, s>>>(x, nblocks, q, d, status, y_zero);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Permutation.  Pairs p = t*k + j.  Groups g = 0..E-1 are the routed experts,
// group E the shared expert (count S*T, slots P..P+S*T-1).
// ---------------------------------------------------------------------------

// Expert of pair p.  The top-k kernels only produce experts in [0, E); an
// index outside it (which would address the counters out of bounds) is
// counted as expert 0 by both the histogram and the scatter, so the
// permutation stays a bijection, and reported as STATUS_BAD_EXPERT_INDEX.
__device__ __forceinline__ int pair_expert(const int32_t* idx, int64_t p, int E, uint32_t* status) {
    const int e = __ldg(idx + p);
    if ((unsigned)e < (unsigned)E) return e;
    if (status) atomicOr(status, STATUS_BAD_EXPERT_INDEX);
    return 0;
}

// Per-chunk expert histogram.
__global__ void __launch_bounds__(PERM_CHUNK) perm_hist_kernel(const int32_t* __restrict__ idx, int64_t P,
                                                                int E, int32_t* __restrict__ chunk_cnt,
                                                                uint32_t* __restrict__ status) {
    __shared__ int cnt[256];
    for (int i = threadIdx.x; i < E; i += blockDim.x) cnt[i] = 0;
    __syncthreads();
    const int64_t p = (int64_t)blockIdx.x * PERM_CHUNK + threadIdx.x;
    if (p < P) atomicAdd(&cnt[pair_expert(idx, p, E, status)], 1);
    __syncthreads();
    for (int i = threadIdx.x; i < E; i += blockDim.x) chunk_cnt[(size_t)blockIdx.x * E + i] = cnt[i];
}

// Block-wide exclusive scan of one int per thread (blockDim.x == 512).
__device__ int block_exclusive_scan_512(int v, int* total) {
    __shared__ int warp_sums[16];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int ws = (lane < 16) ? warp_sums[lane] : 0;
        int wi = ws;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        if (lane < 16) warp_sums[lane] = wi - ws;  // exclusive warp prefix
        if (lane == 15) warp_sums[0] = warp_sums[0];
        if (lane == 15) *total = wi;
    }
    __syncthreads();
    const int r = warp_sums[warp] + incl - v;
    __syncthreads();
    return r;
}

// Totals, group offsets, work-tile offsets and per-chunk bases (one CTA).
__global__ void __launch_bounds__(512) perm_scan_kernel(const int32_t* __restrict__ chunk_cnt, int nchunks, int E,
                                                         int S, int64_t T, int k, int tile_tokens,
                                                         int32_t* __restrict__ cnt, int32_t* __restrict__ off,
                                                         int32_t* __restrict__ tile_off,
                                                         int32_t* __restrict__ chunk_base) {
    __shared__ int s_total[2];
    const int g = threadIdx.x;
    int c_g = 0;
    if (g < E) {
        for (int c = 0; c < nchunks; ++c) c_g += __ldg(chunk_cnt + (size_t)c * E + g);
    } else if (g == E) {
        c_g = S ? (int)T : 0;
    }
    const int o_g = block_exclusive_scan_512(c_g, &s_total[0]);
    const int tiles = (c_g + tile_tokens - 1) / tile_tokens;
    const int to_g = block_exclusive_scan_512(tiles, &s_total[1]);
    if (g <= E) {
        cnt[g] = c_g;
        off[g] = o_g;
        tile_off[g] = to_g;
    }
    if (g == E) {
        off[E + 1] = o_g + c_g;
        tile_off[E + 1] = to_g + tiles;
    }
    if (g < E) {
        int run = o_g;
        for (int c = 0; c < nchunks; ++c) {
            chunk_base[(size_t)c * E + g] = run;
            run += __ldg(chunk_cnt + (size_t)c * E + g);
        }
    }
}

// Stable scatter: the r-th pair of expert e (in increasing p) goes to slot
// off[e] + r.  Within a chunk, rank = pairs of e in earlier warps + earlier
// lanes of this warp.
__global__ void __launch_bounds__(PERM_CHUNK) perm_scatter_kernel(const int32_t* __restrict__ idx, int64_t P,
                                                                   int E, const int32_t* __restrict__ chunk_base,
                                                                   int32_t* __restrict__ sorted,
                                                                   int32_t* __restrict__ pos) {
    // (a bad index was reported by the histogram; the same mapping here)
    __shared__ int wcnt[PERM_CHUNK / 32][256];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < (PERM_CHUNK / 32) * 256; i += blockDim.x) (&wcnt[0][0])[i] = 0;
    __syncthreads();
    const int64_t p = (int64_t)blockIdx.x * PERM_CHUNK + threadIdx.x;
    const bool valid = p < P;
    const int e = valid ? pair_expert(idx, p, E, nullptr) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (valid && rank == 0) wcnt[warp][e] = __popc(peers);
    __syncthreads();
    if (valid) {
        int pre = 0;
        for (int w = 0; w < warp; ++w) pre += wcnt[w][e];
        const int slot = __ldg(chunk_base + (size_t)blockIdx.x * E + e) + pre + rank;
        sorted[slot] = (int32_t)p;
        pos[p] = slot;
    }
}

cudaError_t launch_permute(const int32_t* idx, int64_t T, int k, int E, int S, int tile_tokens,
                           const Workspace& ws, cudaStream_t s) {
    const int64_t P = T * k;
    const int nchunks = (int)ceil_div(P, PERM_CHUNK);
    perm_hist_kernel<<<nchunks, PERM_CHUNK, 0, s>>>(idx, P, E, ws.chunk_cnt, ws.status);
    perm_scan_kernel<<<1, 512, 0, s>>>(ws.chunk_cnt, nchunks, E, S, T, k, tile_tokens, ws.cnt, ws.off,
                                       ws.tile_off, ws.chunk_base);
    perm_scatter_kernel<<<nchunks, PERM_CHUNK, 0, s>>>(idx, P, E, ws.chunk_base, ws.sorted, ws.pos);
    return cudaGetLastError();
}

}  // namespace moeq4
