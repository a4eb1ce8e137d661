// k_grouped_dp4a.cu -- grouped W4A8 projections on the integer dp4a pipe.
//
// The grouped 4-bit GEMM of "A 35B Hybrid-Attention Mixture-of-Experts Model
// on a 6GB 2011 GPU" (Dutch technical summary, Methodologie 1), computed as
// per-block exact integer dot products (the W4A8 integer multiply-adds of the
// same section) scaled by the two binary16 block scales and summed in binary32:
//   g[s,n] = sum_b dWg[e,n,b] * dA[t,b] * I_b,   I_b = sum_i (nib_i - 8) q_i.
// Work items are (expert group, tile of up to DP4A_TT of its slots, block of
// rows), consumed by a persistent grid; the item list is built on the device
// by the permutation, so the host never learns the per-expert counts.
//
//   gate/up item: 32 rows of F of both Wg and Wu, then SwiGLU and the Q8_0
//                 requantisation of those 32 values per slot (one block).
//   down item:    64 rows of H of Wd; each slot's result, times its routing
//                 weight (1 for the shared expert), is added into y[t].
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace moeq4 {

struct ItemRange {
    int g;       // group: routed expert 0..E-1, or E = shared expert
    int slot0;   // first slot of the tile
    int nslots;  // slots in the tile (1..DP4A_TT)
    int rb;      // row block
};

// Largest g in [0, ngroups) with tile_off[g] <= tile (tile_off ascending).
__device__ __forceinline__ int find_group(const int* tile_off, int ngroups, int tile) {
    int lo = 0, hi = ngroups;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tile_off[mid] <= tile) lo = mid; else hi = mid;
    }
    return lo;
}

__device__ __forceinline__ ItemRange decode_item(int item, int n_rb, const int* tile_off_s, const int* off_s,
                                                 int ngroups) {
    ItemRange r;
    const int tile = item / n_rb;
    r.rb = item - tile * n_rb;
    r.g = find_group(tile_off_s, ngroups, tile);
    r.slot0 = off_s[r.g] + (tile - tile_off_s[r.g]) * DP4A_TT;
    r.nslots = min(DP4A_TT, off_s[r.g + 1] - r.slot0);
    return r;
}

// Token of a slot and its routing weight.
__device__ __forceinline__ void slot_token(int s, int g, int E, int k, int P, const int32_t* sorted,
                                           const float* topk_w, int& t, float& w) {
    if (g < E) {
        const int pair = __ldg(sorted + s);
        t = pair / k;
        w = __ldg(topk_w + pair);
    } else {
        t = s - P;
        w = 1.0f;
    }
}

struct GroupedParams {
    int H, F, E, k, P;
    const uint8_t* w_gate;
    const uint8_t* w_up;
    const uint8_t* w_down;
    const uint8_t* sh_gate;
    const uint8_t* sh_up;
    const uint8_t* sh_down;
    const int8_t* qa;
    const uint16_t* da;
    const int32_t* off;
    const int32_t* tile_off;
    const int32_t* sorted;
    const float* topk_w;
    int8_t* hq;
    uint16_t* dh;
    float* h_dbg;
    float* y;
    uint32_t* status;
};

// Stage the int8 rows of the tile's slots, their block scales and block sums.
// src row of slot i is row `rows[i]` of q [*, K] / d [*, K/32].
__device__ __forceinline__ void stage_q8_rows(const int8_t* __restrict__ q, const uint16_t* __restrict__ d, int K,
                                              const int* rows, int nslots, int8_t* q_s, float* d_s, int* sum_s) {
    const int nb = K / QK;
    const int chunks = K / 16;  // int4 chunks per row
    for (int i = threadIdx.x; i < nslots * chunks; i += blockDim.x) {
        const int r = i / chunks, c = i - r * chunks;
        reinterpret_cast<int4*>(q_s + (size_t)r * K)[c] =
            __ldg(reinterpret_cast<const int4*>(q + (size_t)rows[r] * K) + c);
    }
    for (int i = threadIdx.x; i < nslots * nb; i += blockDim.x) {
        const int r = i / nb, b = i - r * nb;
        d_s[i] = half_bits_to_float(__ldg(d + (size_t)rows[r] * nb + b));
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nslots * nb; i += blockDim.x) {
        const int r = i / nb, b = i - r * nb;
        const int* qw = reinterpret_cast<const int*>(q_s + (size_t)r * K + b * QK);
        int s = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) s = __dp4a(qw[j], 0x01010101, s);
        sum_s[i] = s;
    }
    __syncthreads();
}

// Dot products of one Q4_0 row (nb blocks) with the staged slots; the LPR
// lanes of a lane group split the blocks and reduce at the end.
template <int LPR>
__device__ __forceinline__ void row_dots(const uint8_t* __restrict__ wrow, int nb, int K, int sub, int nslots,
                                         const int8_t* q_s, const float* d_s, const int* sum_s,
                                         float acc[DP4A_TT]) {
#pragma unroll
    for (int t = 0; t < DP4A_TT; ++t) acc[t] = 0.0f;
    for (int b = sub; b < nb; b += LPR) {
        uint32_t qs[4], dbits;
        load_q4_block(wrow + (size_t)b * Q4_BYTES, qs, dbits);
        const float dw = half_bits_to_float(dbits);
#pragma unroll
        for (int t = 0; t < DP4A_TT; ++t) {
            if (t < nslots) {
                const int4* qv = reinterpret_cast<const int4*>(q_s + (size_t)t * K + b * QK);
                const int4 a0 = qv[0], a1 = qv[1];
                const int qa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                const int I = q4_q8_dot(qs, qa, sum_s[t * nb + b]);
                acc[t] = fmaf((float)I, dw * d_s[t * nb + b], acc[t]);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < DP4A_TT; ++t) {
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
    }
}

template <int LPR>
__global__ void __launch_bounds__(256) gateup_dp4a_kernel(GroupedParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int tile_off_s[258];
    __shared__ int off_s[258];
    __shared__ int rows_s[DP4A_TT];
    __shared__ float gs[GU_ROWS][DP4A_TT];
    __shared__ float us[GU_ROWS][DP4A_TT];
    const int H = p.H, F = p.F, nb = H / QK;
    int8_t* q_s = reinterpret_cast<int8_t*>(smem);
    float* d_s = reinterpret_cast<float*>(smem + (size_t)DP4A_TT * H);
    int* sum_s = reinterpret_cast<int*>(d_s + DP4A_TT * nb);
    const int ngroups = p.E + 1;
    for (int i = threadIdx.x; i <= ngroups; i += blockDim.x) {
        tile_off_s[i] = p.tile_off[i];
        off_s[i] = p.off[i];
    }
    __syncthreads();
    const int n_rb = F / GU_ROWS;
    const int n_items = tile_off_s[ngroups] * n_rb;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane % LPR, lgrp = lane / LPR;
    constexpr int ROWS_PER_PASS = 32 / LPR;
    const size_t gu_stride = (size_t)F * nb * Q4_BYTES;

    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const ItemRange it = decode_item(item, n_rb, tile_off_s, off_s, ngroups);
        if (threadIdx.x < it.nslots) {
            int t;
            float w;
            slot_token(it.slot0 + threadIdx.x, it.g, p.E, p.k, p.P, p.sorted, p.topk_w, t, w);
            rows_s[threadIdx.x] = t;
        }
        __syncthreads();
        stage_q8_rows(p.qa, p.da, H, rows_s, it.nslots, q_s, d_s, sum_s);

        const uint8_t* Wg = (it.g < p.E) ? p.w_gate + it.g * gu_stride : p.sh_gate;
        const uint8_t* Wu = (it.g < p.E) ? p.w_up + it.g * gu_stride : p.sh_up;
        const int n0 = it.rb * GU_ROWS;
        // 64 row jobs (32 gate + 32 up), 8 per warp
        for (int j0 = warp * 8; j0 < warp * 8 + 8; j0 += ROWS_PER_PASS) {
            const int job = j0 + lgrp;
            const int mat = job >> 5, rloc = job & 31;
            const uint8_t* wrow = (mat ? Wu : Wg) + (size_t)(n0 + rloc) * nb * Q4_BYTES;
            float acc[DP4A_TT];
            row_dots<LPR>(wrow, nb, H, sub, it.nslots, q_s, d_s, sum_s, acc);
            if (sub == 0) {
#pragma unroll
                for (int t = 0; t < DP4A_TT; ++t) (mat ? us : gs)[rloc][t] = acc[t];
            }
        }
        __syncthreads();
        // epilogue: one warp per slot, lane = row of the 32-row block
        for (int t = warp; t < it.nslots; t += 8) {
            const int slot = it.slot0 + t;
            const float h = swiglu(gs[lane][t], us[lane][t]);
            if (p.h_dbg) p.h_dbg[(size_t)slot * F + n0 + lane] = h;
            uint16_t db;
            bool ov;
            const int q = q8_0_lane(h, db, ov);
            p.hq[(size_t)slot * F + n0 + lane] = (int8_t)q;
            if (lane == 0) {
                p.dh[(size_t)slot * (F / QK) + it.rb] = db;
                if (ov) atomicOr(p.status, STATUS_SCALE_OVERFLOW);
            }
        }
        __syncthreads();
    }
}

template <int LPR>
__global__ void __launch_bounds__(256) down_dp4a_kernel(GroupedParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int tile_off_s[258];
    __shared__ int off_s[258];
    __shared__ int slots_s[DP4A_TT];
    __shared__ int tok_s[DP4A_TT];
    __shared__ float wgt_s[DP4A_TT];
    const int H = p.H, F = p.F, nbF = F / QK;
    int8_t* q_s = reinterpret_cast<int8_t*>(smem);
    float* d_s = reinterpret_cast<float*>(smem + (size_t)DP4A_TT * F);
    int* sum_s = reinterpret_cast<int*>(d_s + DP4A_TT * nbF);
    const int ngroups = p.E + 1;
    for (int i = threadIdx.x; i <= ngroups; i += blockDim.x) {
        tile_off_s[i] = p.tile_off[i];
        off_s[i] = p.off[i];
    }
    __syncthreads();
    const int n_rb = H / DN_ROWS;
    const int n_items = tile_off_s[ngroups] * n_rb;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane % LPR, lgrp = lane / LPR;
    constexpr int ROWS_PER_PASS = 32 / LPR;
    const size_t dn_stride = (size_t)H * nbF * Q4_BYTES;

    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const ItemRange it = decode_item(item, n_rb, tile_off_s, off_s, ngroups);
        if (threadIdx.x < it.nslots) {
            int t;
            float w;
            slot_token(it.slot0 + threadIdx.x, it.g, p.E, p.k, p.P, p.sorted, p.topk_w, t, w);
            slots_s[threadIdx.x] = it.slot0 + threadIdx.x;
            tok_s[threadIdx.x] = t;
            wgt_s[threadIdx.x] = w;
        }
        __syncthreads();
        stage_q8_rows(p.hq, p.dh, F, slots_s, it.nslots, q_s, d_s, sum_s);

        const uint8_t* Wd = (it.g < p.E) ? p.w_down + it.g * dn_stride : p.sh_down;
        const int n0 = it.rb * DN_ROWS;
        for (int r0 = warp * 8; r0 < warp * 8 + 8; r0 += ROWS_PER_PASS) {
            const int n = n0 + r0 + lgrp;
            const uint8_t* wrow = Wd + (size_t)n * nbF * Q4_BYTES;
            float acc[DP4A_TT];
            row_dots<LPR>(wrow, nbF, F, sub, it.nslots, q_s, d_s, sum_s, acc);
            if (sub == 0) {
#pragma unroll
                for (int t = 0; t < DP4A_TT; ++t)
                    if (t < it.nslots) atomicAdd(p.y + (size_t)tok_s[t] * H + n, wgt_s[t] * acc[t]);
            }
        }
        __syncthreads();
    }
}

static int lanes_per_row(int nblocks) { return nblocks >= 32 ? 32 : (nblocks >= 16 ? 16 : 8); }

static GroupedParams make_params(const LayerView& L, int64_t T, const Workspace& ws, float* h_dbg, float* y) {
    GroupedParams p;
    p.H = L.H; p.F = L.F; p.E = L.E; p.k = L.k; p.P = (int)(T * L.k);
    p.w_gate = L.w_gate; p.w_up = L.w_up; p.w_down = L.w_down;
    p.sh_gate = L.sh_gate; p.sh_up = L.sh_up; p.sh_down = L.sh_down;
    p.qa = ws.qa; p.da = ws.da; p.off = ws.off; p.tile_off = ws.tile_off; p.sorted = ws.sorted;
    p.topk_w = ws.topk_w; p.hq = ws.hq; p.dh = ws.dh; p.h_dbg = h_dbg; p.y = y; p.status = ws.status;
    return p;
}

// Upper bound of the work tiles over all groups: sum_g ceil(c_g / TT).
static int64_t max_tiles(const LayerView& L, int64_t T) {
    const int64_t P = T * L.k;
    return ceil_div(P, DP4A_TT) + std::min<int64_t>(L.E, P) + (L.S ? ceil_div(T, DP4A_TT) : 0);
}

template <typename K>
static cudaError_t launch_persistent(K kernel, int64_t items, size_t smem, const DeviceInfo& dev,
                                     const GroupedParams& p, cudaStream_t s) {
    int per_sm = 0;
    cudaError_t err = kernel_occupancy(reinterpret_cast<const void*>(kernel), 256, smem, &per_sm);
    if (err != cudaSuccess) return err;
    int64_t grid = std::min<int64_t>(items, (int64_t)dev.sm_count * per_sm);
    if (grid < 1) grid = 1;
    kernel<<<(unsigned)grid, 256, smem, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_gateup_dp4a(const LayerView& L, int64_t T, const Workspace& ws, float* h_dbg,
                               const DeviceInfo& dev, cudaStream_t s) {
    const GroupedParams p = make_params(L, T, ws, h_dbg, nullptr);
    const int nb = L.H / QK;
    const size_t smem = (size_t)DP4A_TT * L.H + (size_t)DP4A_TT * nb * 8;
    const int64_t items = max_tiles(L, T) * (L.F / GU_ROWS);
    switch (lanes_per_row(nb)) {
        case 32: return launch_persistent(gateup_dp4a_kernel<32>, items, smem, dev, p, s);
        case 16: return launch_persistent(gateup_dp4a_kernel<16>, items, smem, dev, p, s);
        default: return launch_persistent(gateup_dp4a_kernel<8>, items, smem, dev, p, s);
    }
}

cudaError_t launch_down_dp4a(const LayerView& L, int64_t T, const Workspace& ws, float* y,
                             const DeviceInfo& dev, cudaStream_t s) {
    const GroupedParams p = make_params(L, T, ws, nullptr, y);
    const int nbF = L.F / QK;
    const size_t smem = (size_t)DP4A_TT * L.F + (size_t)DP4A_TT * nbF * 8;
    const int64_t items = max_tiles(L, T) * (L.H / DN_ROWS);
    switch (lanes_per_row(nbF)) {
        case 32: return launch_persistent(down_dp4a_kernel<32>, items, smem, dev, p, s);
        case 16: return launch_persistent(down_dp4a_kernel<16>, items, smem, dev, p, s);
        default: return launch_persistent(down_dp4a_kernel<8>, items, smem, dev, p, s);
    }
}

// ---------------------------------------------------------------------------
// Test export: per-block integer dot products through the same routines.
// ---------------------------------------------------------------------------
__global__ void block_dots_kernel(const uint8_t* __restrict__ w, const int8_t* __restrict__ qa, int64_t n,
                                  int32_t* __restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    uint32_t qs[4], dbits;
    load_q4_block(w + i * Q4_BYTES, qs, dbits);
    const int4* qv = reinterpret_cast<const int4*>(qa + i * QK);
    const int4 a0 = __ldg(qv), a1 = __ldg(qv + 1);
    const int q[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    out[i] = q4_q8_dot(qs, q, q8_block_sum(q));
}

cudaError_t launch_block_dots(const uint8_t* w, const int8_t* qa, int64_t n, int32_t* out, cudaStream_t s) {
    block_dots_kernel<<<(unsigned)ceil_div(n, 256), 256, 0, s>>>(w, qa, n, out);
    return cudaGetLastError();
}

}  // namespace moeq4
