// k_tc_grouped.cu -- grouped W4A8 projections on the 5th-generation tensor
// cores (tcgen05.mma kind::i8, accumulators in TMEM).
//
// The grouped 4-bit GEMM of the prefill ("A 35B Hybrid-Attention
// Mixture-of-Experts Model on a 6GB 2011 GPU", Dutch technical summary,
// Methodologie 1), with the page's single-pass prefill (Methodologie 4): every
// expert sees all of its tokens at once, so its weights are read once per
// token tile.
//
// Orientation: the MMA's M dimension is 128 weight rows (gate/up: 64 gate rows
// + the same 64 up rows; down: 128 rows of H), N is a tile of 64 slots of one
// expert, K runs over Q4_0 blocks.  Each 32-wide block is one MMA (K = 32)
// into its own TMEM buffer, because every block has its own pair of binary16
// scales: the epilogue reads the exact int32 block sums and accumulates
// dW[row,b] * dA[slot,b] * I_b in fp32 registers (lane = row).
//
// Per K chunk of 8 blocks:
//   1. bulk copies of the 128 packed weight rows (144 B each) into staging;
//      16-byte cp.async gathers of the 64 slots' int8 activations straight
//      into the K-major operand layout (8-row x 16-byte core matrices);
//   2. each thread unpacks one weight row: nibbles -> signed int8 (nib - 8)
//      into the same operand layout, scales -> shared memory;
//   3. one thread issues the 8 MMAs and commits them to an mbarrier;
//   4. the four warps read their 32 TMEM lanes and rescale.
// After the last chunk: gate/up -> SwiGLU and Q8_0 requantisation of h
// (a warp's 32 lanes are the 32 rows of one Q8_0 block); down -> y[t] +=
// w_slot * o (fp32 atomics).
#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"
#include "tc.cuh"

namespace moeq4 {

constexpr int TC_M = 128;
constexpr int TC_N = 64;
constexpr int TC_KB = 8;                     // Q4_0 blocks per K chunk
constexpr int TC_THREADS = 128;              // one thread per TMEM lane
constexpr uint32_t TC_TMEM_COLS = TC_KB * TC_N;  // one 64-column buffer per block
constexpr int TC_STAGE_ROW = TC_KB * Q4_BYTES;   // 144 packed bytes per row per chunk

constexpr size_t TC_SMEM_A = (size_t)TC_KB * TC_M * QK;     // 32 KB
constexpr size_t TC_SMEM_B = (size_t)TC_KB * TC_N * QK;     // 16 KB
constexpr size_t TC_SMEM_STAGE = (size_t)TC_M * TC_STAGE_ROW;  // 18 KB
// more than half of an SM's shared memory: one CTA per SM, so the 512 TMEM
// columns one CTA allocates are always free
constexpr size_t TC_SMEM_TOTAL = 120 * 1024;

enum { TC_GATEUP = 0, TC_DOWN = 1 };

struct TcParams {
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

// nibble bytes (0..15) -> signed int8 bytes (nib - 8): for nib >= 8 the value
// is nib ^ 8; for nib < 8 it is 0xF8 | nib, i.e. nib ^ 8 with the top four bits
// set, and (~nib & 8) * 0x1E supplies exactly those bits without carries.
__device__ __forceinline__ uint32_t nib_to_s8(uint32_t n) {
    return (n ^ 0x08080808u) | ((~n & 0x08080808u) * 0x1Eu);
}

// Offset of the 16-byte piece kc (0: K bytes 0..15, 1: 16..31) of row r of
// block kb in a K-major operand tile of `rows` rows (8-row x 16-byte core
// matrices; K core matrices 128 B apart, 8-row groups 256 B apart).
__device__ __forceinline__ uint32_t op_offset(int kb, int rows, int r, int kc) {
    return (uint32_t)(kb * rows * QK + (r >> 3) * 256 + kc * 128 + (r & 7) * 16);
}

__device__ __forceinline__ int find_group_tc(const int* tile_off, int ngroups, int tile) {
    int lo = 0, hi = ngroups;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tile_off[mid] <= tile) lo = mid; else hi = mid;
    }
    return lo;
}

template <int MODE>
__global__ void __launch_bounds__(TC_THREADS, 1) tc_grouped_kernel(TcParams p) {
    extern __shared__ __align__(1024) unsigned char smem[];
    __shared__ __align__(8) uint64_t bar_w, bar_mma;
    __shared__ uint32_t tmem_base_s;
    __shared__ int tile_off_s[258];
    __shared__ int off_s[258];
    __shared__ int tok_s[TC_N];
    __shared__ float wgt_s[TC_N];
    __shared__ const int8_t* act_row_s[TC_N];
    __shared__ const uint16_t* act_scale_s[TC_N];

    uint8_t* A = smem;
    uint8_t* B = A + TC_SMEM_A;
    uint8_t* stage = B + TC_SMEM_B;
    float* dw_s = reinterpret_cast<float*>(stage + TC_SMEM_STAGE);
    float* da_s = dw_s + TC_M * TC_KB;
    float* xch = reinterpret_cast<float*>(A);  // 128 x 65 floats, reuses A and B after the K loop

    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int H = p.H, F = p.F, E = p.E;
    const int K = (MODE == TC_GATEUP) ? H : F;
    const int nbK = K / QK, nchunks = nbK / TC_KB;
    const int nbF = F / QK;
    const size_t wrow = (size_t)nbK * Q4_BYTES;  // bytes per weight row
    const size_t mat_stride = (MODE == TC_GATEUP) ? (size_t)F * wrow : (size_t)H * wrow;
    const int n_rb = (MODE == TC_GATEUP) ? F / 64 : H / TC_M;
    const int ngroups = E + 1;

    if (warp == 0) {
        tmem_alloc(&tmem_base_s, TC_TMEM_COLS);
        tmem_relinquish();
    }
    if (t == 0) {
        mbar_init(&bar_w, TC_THREADS);
        mbar_init(&bar_mma, 1);
        mbar_fence_init();
    }
    for (int i = t; i <= ngroups; i += TC_THREADS) {
        tile_off_s[i] = p.tile_off[i];
        off_s[i] = p.off[i];
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = tmem_base_s;
    const uint32_t idesc = idesc_i8(TC_M, TC_N);
    const int n_items = tile_off_s[ngroups] * n_rb;
    uint32_t phase = 0;
    bool timed_out = false;

    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int tile = item / n_rb, rb = item - tile * n_rb;
        const int g = find_group_tc(tile_off_s, ngroups, tile);
        const int slot0 = off_s[g] + (tile - tile_off_s[g]) * TC_N;
        const int nslots = min(TC_N, off_s[g + 1] - slot0);
        if (t < TC_N) {
            int tok = 0;
            float w = 0.0f;
            if (t < nslots) {
                const int s = slot0 + t;
                if (g < E) {
                    const int pair = __ldg(p.sorted + s);
                    tok = pair / p.k;
                    w = __ldg(p.topk_w + pair);
                } else {
                    tok = s - p.P;
                    w = 1.0f;
                }
                if (MODE == TC_GATEUP) {
                    act_row_s[t] = p.qa + (size_t)tok * H;
                    act_scale_s[t] = p.da + (size_t)tok * (H / QK);
                } else {
                    act_row_s[t] = p.hq + (size_t)s * F;
                    act_scale_s[t] = p.dh + (size_t)s * nbF;
                }
            }
            tok_s[t] = tok;
            wgt_s[t] = w;
        }
        // this thread's weight row
        const uint8_t* wsrc;
        if (MODE == TC_GATEUP) {
            const int f = rb * 64 + (t & 63);
            const uint8_t* base = (t < 64) ? ((g < E) ? p.w_gate + g * mat_stride : p.sh_gate)
                                           : ((g < E) ? p.w_up + g * mat_stride : p.sh_up);
            wsrc = base + (size_t)f * wrow;
        } else {
            wsrc = ((g < E) ? p.w_down + g * mat_stride : p.sh_down) + (size_t)(rb * TC_M + t) * wrow;
        }
        __syncthreads();

        float acc[TC_N];
#pragma unroll
        for (int n = 0; n < TC_N; ++n) acc[n] = 0.0f;

        for (int c = 0; c < nchunks; ++c) {
            // 1. packed weight rows -> staging; activations -> operand B
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&bar_w, (uint32_t)TC_STAGE_ROW);
            bulk_g2s(stage + t * TC_STAGE_ROW, wsrc + (size_t)c * TC_STAGE_ROW, (uint32_t)TC_STAGE_ROW, &bar_w);
            for (int i = t; i < TC_N * TC_KB * 2; i += TC_THREADS) {
                const int n = i / (TC_KB * 2), kb = (i >> 1) % TC_KB, kc = i & 1;
                uint8_t* dst = B + op_offset(kb, TC_N, n, kc);
                if (n < nslots)
                    cp_async16(dst, act_row_s[n] + (size_t)(c * TC_KB + kb) * QK + kc * 16);
                else
                    *reinterpret_cast<int4*>(dst) = make_int4(0, 0, 0, 0);
            }
            for (int i = t; i < TC_N * TC_KB; i += TC_THREADS) {
                const int n = i / TC_KB, kb = i % TC_KB;
                da_s[i] = (n < nslots) ? half_bits_to_float(__ldg(act_scale_s[n] + c * TC_KB + kb)) : 0.0f;
            }
            cp_async_wait_all();
            if (!mbar_wait_bounded(&bar_w, phase & 1, 1u << 20)) timed_out = true;

            // 2. unpack this thread's row: nibbles -> signed int8 operand A
            const uint8_t* srow = stage + t * TC_STAGE_ROW;
#pragma unroll
            for (int kb = 0; kb < TC_KB; ++kb) {
                uint32_t qs[4], dbits;
                load_q4_block_smem(srow + kb * Q4_BYTES, qs, dbits);
                dw_s[t * TC_KB + kb] = half_bits_to_float(dbits);
                int4 lo, hi;
                lo.x = (int)nib_to_s8(qs[0] & 0x0f0f0f0fu);
                lo.y = (int)nib_to_s8(qs[1] & 0x0f0f0f0fu);
                lo.z = (int)nib_to_s8(qs[2] & 0x0f0f0f0fu);
                lo.w = (int)nib_to_s8(qs[3] & 0x0f0f0f0fu);
                hi.x = (int)nib_to_s8((qs[0] >> 4) & 0x0f0f0f0fu);
                hi.y = (int)nib_to_s8((qs[1] >> 4) & 0x0f0f0f0fu);
                hi.z = (int)nib_to_s8((qs[2] >> 4) & 0x0f0f0f0fu);
                hi.w = (int)nib_to_s8((qs[3] >> 4) & 0x0f0f0f0fu);
                *reinterpret_cast<int4*>(A + op_offset(kb, TC_M, t, 0)) = lo;
                *reinterpret_cast<int4*>(A + op_offset(kb, TC_M, t, 1)) = hi;
            }
            fence_proxy_async_smem();  // operand writes -> visible to the tensor core
            tc_fence_before_sync();
            __syncthreads();
            tc_fence_after_sync();

            // 3. one MMA per block into its own TMEM buffer
            if (t == 0) {
#pragma unroll
                for (int kb = 0; kb < TC_KB; ++kb) {
                    const uint64_t da = smem_desc_kmajor(A + (size_t)kb * TC_M * QK, 128, 256);
                    const uint64_t db = smem_desc_kmajor(B + (size_t)kb * TC_N * QK, 128, 256);
                    mma_i8(tmem + kb * TC_N, da, db, idesc, false);
                }
                mma_commit(&bar_mma);
            }
            if (!mbar_wait_bounded(&bar_mma, phase & 1, 1u << 20)) timed_out = true;
            tc_fence_after_sync();

            // 4. rescale: lane = row t, 64 slot columns per block
            const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
            for (int kb = 0; kb < TC_KB; ++kb) {
                const float dw = dw_s[t * TC_KB + kb];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r[32];
                    tmem_ld32(lane_addr + kb * TC_N + half * 32, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int n = half * 32 + j;
                        acc[n] = fmaf((float)(int)r[j], dw * da_s[n * TC_KB + kb], acc[n]);
                    }
                }
            }
            tc_fence_before_sync();
            __syncthreads();  // staging, operands and TMEM buffers are free again
            phase ^= 1u;
        }

        if (MODE == TC_GATEUP) {
            // rows t < 64: gate row f0 + t; rows 64 + t: up row f0 + t
            const int f0 = rb * 64;
#pragma unroll
            for (int n = 0; n < TC_N; ++n) xch[t * 65 + n] = acc[n];
            __syncthreads();
            if (t < 64) {
#pragma unroll 1
                for (int n = 0; n < TC_N; ++n) {
                    // all 32 lanes of the warp take every column: the Q8_0
                    // block of h is the warp's 32 rows
                    const float h = swiglu(xch[t * 65 + n], xch[(t + 64) * 65 + n]);
                    uint16_t db;
                    bool ov;
                    const int q = q8_0_lane(h, db, ov);
                    if (n < nslots) {
                        const int s = slot0 + n;
                        if (p.h_dbg) p.h_dbg[(size_t)s * F + f0 + t] = h;
                        p.hq[(size_t)s * F + f0 + t] = (int8_t)q;
                        if (lane == 0) {
                            p.dh[(size_t)s * nbF + (f0 >> 5) + warp] = db;
                            if (ov) atomicOr(p.status, STATUS_SCALE_OVERFLOW);
                        }
                    }
                }
            }
        } else {
            const int h0 = rb * TC_M;
#pragma unroll
            for (int n = 0; n < TC_N; ++n)
                if (n < nslots) atomicAdd(p.y + (size_t)tok_s[n] * H + h0 + t, wgt_s[n] * acc[n]);
        }
        __syncthreads();
    }

    if (timed_out) atomicOr(p.status, STATUS_SPIN_TIMEOUT);
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, TC_TMEM_COLS);
}

static TcParams make_tc_params(const LayerView& L, int64_t T, const Workspace& ws, float* h_dbg, float* y) {
    TcParams p;
    p.H = L.H; p.F = L.F; p.E = L.E; p.k = L.k; p.P = (int)(T * L.k);
    p.w_gate = L.w_gate; p.w_up = L.w_up; p.w_down = L.w_down;
    p.sh_gate = L.sh_gate; p.sh_up = L.sh_up; p.sh_down = L.sh_down;
    p.qa = ws.qa; p.da = ws.da; p.off = ws.off; p.tile_off = ws.tile_off; p.sorted = ws.sorted;
    p.topk_w = ws.topk_w; p.hq = ws.hq; p.dh = ws.dh; p.h_dbg = h_dbg; p.y = y; p.status = ws.status;
    return p;
}

static int64_t tc_max_tiles(const LayerView& L, int64_t T) {
    const int64_t P = T * L.k;
    return ceil_div(P, TC_N) + std::min<int64_t>(L.E, P) + (L.S ? ceil_div(T, TC_N) : 0);
}

template <int MODE>
static cudaError_t launch_tc(const LayerView& L, int64_t T, const Workspace& ws, float* h_dbg, float* y,
                             const DeviceInfo& dev, cudaStream_t s) {
    int per_sm = 0;
    cudaError_t e = kernel_occupancy(reinterpret_cast<const void*>(tc_grouped_kernel<MODE>), TC_THREADS,
                                     TC_SMEM_TOTAL, &per_sm);
    if (e != cudaSuccess) return e;
    const int n_rb = (MODE == TC_GATEUP) ? L.F / 64 : L.H / TC_M;
    const int64_t items = tc_max_tiles(L, T) * n_rb;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(items, dev.sm_count));
    tc_grouped_kernel<MODE><<<(unsigned)grid, TC_THREADS, TC_SMEM_TOTAL, s>>>(make_tc_params(L, T, ws, h_dbg, y));
    return cudaGetLastError();
}

cudaError_t launch_gateup_tc(const LayerView& L, int64_t T, const Workspace& ws, float* h_dbg, const DeviceInfo& dev,
                             cudaStream_t s) {
    return launch_tc<TC_GATEUP>(L, T, ws, h_dbg, nullptr, dev, s);
}

cudaError_t launch_down_tc(const LayerView& L, int64_t T, const Workspace& ws, float* y, const DeviceInfo& dev,
                           cudaStream_t s) {
    return launch_tc<TC_DOWN>(L, T, ws, nullptr, y, dev, s);
}

}  // namespace moeq4
