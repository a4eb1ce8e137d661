// k_grouped_dp4a.cu -- grouped W4A8 projections for few tokens per expert, on
// the integer dp4a pipe, streaming the weights.
//
// The grouped 4-bit GEMM of "A 35B Hybrid-Attention Mixture-of-Experts Model
// on a 6GB 2011 GPU" (Dutch technical summary, Methodologie 1), computed with
// the W4A8 integer multiply-adds of the same section: per-block exact integer
// dot products scaled by the two binary16 block scales and summed in binary32,
//   g[s,n] = sum_b dWg[e,n,b] * dA[t,b] * I_b,   I_b = sum_i (nib_i - 8) q_i.
// When every expert sees only a few tokens (small batches, decode of several
// sequences) the layer is bound by streaming the active experts' weights, so
// this kernel is built around that stream:
//   - a work item is (expert group, tile of up to 8 of its slots, 64 weight
//     rows: 32 rows of Wg + the same 32 of Wu, or 64 rows of Wd); items come
//     from the device-built tile list and are consumed by one persistent CTA
//     per SM;
//   - a producer warp moves each item's weights in chunks of 64 rows x 32
//     blocks with one or two 2D tensor copies (TMA; 8-byte elements, so a
//     box row is a whole 576-byte chunk row), and the tile's int8
//     activations and scales with 16-byte cp.async, three chunks in flight;
//   - sixteen compute warps: a lane owns 2 weight rows and every 16th block of
//     the chunk, keeps its slots' activation blocks in registers and its
//     2 x 8 (row, slot) sums in registers across the item's chunks; the 16
//     lanes of a row group add their sums with shuffles once per item;
//   - epilogue: gate/up -> SwiGLU + Q8_0 requantisation of each slot's 32-row
//     block of h; down -> y[t] += w * o (fp32 atomics; weight 1 for the
//     shared expert).
// Every wait is bounded; a wait that runs out releases every role and records
// STATUS_SPIN_TIMEOUT.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace moeq4 {

namespace {

constexpr int SR = 64;                 // weight rows per item
constexpr int ST = DP4A_TT;            // slots per tile (8)
constexpr int KCMAX = 32;              // blocks per chunk, at most
// Blocks per chunk for rows of nb blocks (nb a multiple of 8): the largest of
// 32, 24, 16, 8 that divides nb, so the chunks tile the row exactly.
__host__ __device__ constexpr int chunk_blocks(int nb) {
    return nb % 32 == 0 ? 32 : nb % 24 == 0 ? 24 : nb % 16 == 0 ? 16 : 8;
}
constexpr int NST = 3;                 // chunks in flight
constexpr int NCW = 16;                // compute warps
constexpr int RPL = 2;                 // weight rows per lane
constexpr int THREADS = (NCW + 1) * 32;
constexpr uint32_t LIMIT = 1u << 22;
constexpr size_t SZ_W = (size_t)SR * KCMAX * Q4_BYTES;    // 36,864
constexpr size_t SZ_A = (size_t)ST * KCMAX * QK;          // 8,192
constexpr size_t SZ_D = (size_t)ST * KCMAX * 2;           // 512
constexpr size_t SZ_STAGE = SZ_W + SZ_A + SZ_D;           // 45,568 = 356 x 128
constexpr size_t OFF_RES = NST * SZ_STAGE;
constexpr size_t SMEM_BYTES = OFF_RES + (size_t)SR * ST * 4;
constexpr size_t SMEM_ALLOC = SMEM_BYTES + 128;           // slack to align the stages to 128 B
static_assert(SZ_STAGE % 128 == 0, "TMA destinations need 128-byte alignment");
static_assert(SMEM_ALLOC <= 200 * 1024, "shared memory map too large");

enum { GATEUP = 0, DOWN = 1, GEMV = 2 };

// 2D views of the weight matrices for TMA, in 8-byte elements so that one
// row segment of a box is a whole chunk row (KC blocks x 18 B, up to 576 B)
// rather than many short ones.  gate/up: [0] gate, [1] up, [2] shared gate,
// [3] shared up; down: [0] down, [2] shared down.
struct StreamMaps {
    CUtensorMap m[4];
};

struct StreamParams {
    int H, F, E, k, P;
    int N, T;  // GEMV: rows of the matrix, tokens (the slots of the one tile)
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
    int32_t* cap_out;  // block-dot capture (the CAP instantiation only)
    int cap_group, cap_rb;
};

// Where a capturing item writes its block dot products: cap + ((slot_rel + j)
// * SR + row) * nb + block, for the lane's rows and blocks.
struct CapPtr {
    int32_t* out;  // NULL when this item is not captured
    int slot_rel;  // first slot of the tile minus the group's first slot
    int row0;      // this lane's first row within the item
    int nb;        // blocks along K
    int blk;       // block index along K of the current block
};

__device__ __forceinline__ void mbar_arrive1(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void cp_async16_(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all_() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void cp_async_arrive_noinc_(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tma_load_2d_(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Bounded wait; once any wait of the CTA has run out, every later one
// returns false soon after.
__device__ __forceinline__ bool wait_phase_s(uint64_t* bar, uint32_t parity, volatile int* abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 100000u)) return true;   // sleeps instead of spinning
        if (*abort) return false;
        if (global_ns() - t0 > 2000000000ull) break;                  // 2 s bound
    }
    *abort = 1;
    return false;
}

// Barrier of the compute warps (one arrival per warp), bounded.
__device__ __forceinline__ bool compute_sync(uint64_t* bar, uint32_t use, volatile int* abort) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive1(bar);
    return wait_phase_s(bar, use & 1, abort);
}

__device__ __forceinline__ int find_group_s(const int* tile_off, int ngroups, int tile) {
    int lo = 0, hi = ngroups;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tile_off[mid] <= tile) lo = mid; else hi = mid;
    }
    return lo;
}

struct SItem {
    int g, slot0, nslots, rb;
};

__device__ __forceinline__ SItem item_of(int item, int n_rb, const int* tile_off_s, const int* off_s, int ngroups) {
    SItem t;
    const int tile = item / n_rb;
    t.rb = item - tile * n_rb;
    t.g = find_group_s(tile_off_s, ngroups, tile);
    t.slot0 = off_s[t.g] + (tile - tile_off_s[t.g]) * ST;
    t.nslots = min(ST, off_s[t.g + 1] - t.slot0);
    return t;
}

// Token and routing weight of slot s of group g (group E: the shared expert,
// slot P + t is token t, weight 1).
__device__ __forceinline__ void slot_tok(const StreamParams& p, int g, int s, int& tok, float& w) {
    if (g < p.E) {
        const int pair = __ldg(p.sorted + s);
        tok = pair / p.k;
        w = __ldg(p.topk_w + pair);
    } else {
        tok = s - p.P;
        w = 1.0f;
    }
}

// binary32 value of an integer |I| < 2^22, exactly, without the slow int->float
// conversion: the integer is placed in the mantissa of 1.5 * 2^23.
__device__ __forceinline__ float int_to_float_exact(int I) {
    return __fsub_rn(__int_as_float(I + 0x4B400000), 12582912.0f);
}

// acc[r][s0 + j] += the W4A8 block term of block b for slots s0 .. s0 + SPW - 1
// (activations of a slot: [half][block][16 B] at sa + slot * KC * 32).
template <int SPW, int RPL_, int ST_, bool CAP>
__device__ __forceinline__ void block_slots(float (&acc)[RPL_][ST_], int s0, const uint32_t (&qs)[RPL_][4],
                                            const float (&dW)[RPL_], const int8_t* sa, const uint16_t* sd, int KC,
                                            int b, const CapPtr& cap) {
    int qa[SPW][8];
    int base[SPW];
    float dA[SPW];
#pragma unroll
    for (int j = 0; j < SPW; ++j) {
        const int8_t* a = sa + (size_t)(s0 + j) * KC * QK;
        const int4 a0 = *reinterpret_cast<const int4*>(a + b * 16);
        const int4 a1 = *reinterpret_cast<const int4*>(a + (size_t)KC * 16 + b * 16);
        qa[j][0] = a0.x; qa[j][1] = a0.y; qa[j][2] = a0.z; qa[j][3] = a0.w;
        qa[j][4] = a1.x; qa[j][5] = a1.y; qa[j][6] = a1.z; qa[j][7] = a1.w;
        int sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) sum = __dp4a(qa[j][i], 0x01010101, sum);
        base[j] = -8 * sum;
        dA[j] = half_bits_to_float(sd[(s0 + j) * KC + b]);
    }
#pragma unroll
    for (int r = 0; r < RPL_; ++r) {
#pragma unroll
        for (int j = 0; j < SPW; ++j) {
            // low nibbles as they are; high nibbles masked in place (16 x the
            // nibble), their chain divided by 16 once (exact)
            int lo = base[j], hi = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                lo = dp4a_u8s8(qs[r][i] & 0x0f0f0f0fu, qa[j][i], lo);
                hi = dp4a_u8s8(qs[r][i] & 0xf0f0f0f0u, qa[j][4 + i], hi);
            }
            const int I = lo + (hi >> 4);
            if (CAP && cap.out) cap.out[((size_t)(cap.slot_rel + s0 + j) * SR + cap.row0 + r) * cap.nb + cap.blk] = I;
            acc[r][s0 + j] = fmaf(int_to_float_exact(I), dW[r] * dA[j], acc[r][s0 + j]);
        }
    }
}

}  // namespace

// CAP: also write the per-block integer dot products of one row block of one
// group to p.cap_out (test instantiation).
template <int MODE, bool CAP>
__global__ void __maxnreg__(96) stream_dp4a_kernel(StreamParams p, const __grid_constant__ StreamMaps maps) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
    __shared__ __align__(8) uint64_t full[NST], empty[NST], cbar;
    __shared__ int abort_s;
    __shared__ int tile_off_s[258], off_s[258];
    __shared__ const int8_t* arow_s[ST];
    __shared__ const uint16_t* ascale_s[ST];
    float* res = reinterpret_cast<float*>(smem + OFF_RES);
    volatile int* abort = &abort_s;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = p.H, F = p.F, E = p.E;
    const int K = (MODE == DOWN) ? F : H;
    const int nb = K / QK;
    const int KC = chunk_blocks(nb);
    const int nchunk = nb / KC;
    const int n_rb = (MODE == GATEUP) ? F / 32 : ((MODE == DOWN) ? H / SR : (p.N + SR - 1) / SR);
    const int ngroups = E + 1;
    const uint32_t chunk_bytes = (uint32_t)(SR * KC * Q4_BYTES);

    if (tid == 0) {
        abort_s = 0;
        for (int i = 0; i < NST; ++i) {
            mbar_init(&full[i], 64);   // 32 producer arrivals + 32 cp.async arrivals
            mbar_init(&empty[i], NCW);
        }
        mbar_init(&cbar, NCW);
        mbar_fence_init();
    }
    if (MODE != GEMV) {
        for (int i = tid; i <= ngroups; i += THREADS) {
            tile_off_s[i] = p.tile_off[i];
            off_s[i] = p.off[i];
        }
    }
    __syncthreads();
    const int n_items = (MODE == GEMV) ? n_rb : tile_off_s[ngroups] * n_rb;

    if (warp == NCW) {
        // ------------------------------------------------------------ producer
        uint32_t ic = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            const SItem it = (MODE == GEMV) ? SItem{0, 0, p.T, item} : item_of(item, n_rb, tile_off_s, off_s, ngroups);
            const bool sh = (MODE != GEMV) && it.g >= E;
            if (MODE == GEMV && lane < it.nslots) {
                arow_s[lane] = p.qa + (size_t)lane * H;
                ascale_s[lane] = p.da + (size_t)lane * (H / QK);
            } else if (MODE != GEMV && lane < it.nslots) {
                int tok;
                float w;
                const int s = it.slot0 + lane;
                slot_tok(p, it.g, s, tok, w);
                if (MODE == GATEUP) {
                    arow_s[lane] = p.qa + (size_t)tok * H;
                    ascale_s[lane] = p.da + (size_t)tok * (H / QK);
                } else {
                    arow_s[lane] = p.hq + (size_t)s * F;
                    ascale_s[lane] = p.dh + (size_t)s * (F / QK);
                }
            }
            __syncwarp();
            const CUtensorMap* m0 = &maps.m[sh ? 2 : 0];
            const CUtensorMap* m1 = &maps.m[sh ? 3 : 1];
            const int z = (MODE == GEMV) ? it.rb * SR
                                         : (sh ? 0 : it.g * ((MODE == GATEUP) ? F : H)) + it.rb * ((MODE == GATEUP) ? 32 : SR);
            for (int c = 0; c < nchunk; ++c, ++ic) {
                const int st = ic % NST;
                if (!wait_phase_s(&empty[st], ((ic / NST) & 1) ^ 1, abort)) { ok = false; break; }
                unsigned char* sw = smem + st * SZ_STAGE;
                int8_t* sa = reinterpret_cast<int8_t*>(sw + SZ_W);
                unsigned char* sd = sw + SZ_W + SZ_A;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[st], chunk_bytes);
                    const int x8 = c * KC * Q4_BYTES / 8;   // chunk start in 8-byte elements (16-B multiple)
                    if (MODE == GATEUP) {
                        tma_load_2d_(sw, m0, x8, z, &full[st]);
                        tma_load_2d_(sw + (size_t)32 * KC * Q4_BYTES, m1, x8, z, &full[st]);
                    } else {
                        tma_load_2d_(sw, m0, x8, z, &full[st]);
                    }
                } else {
                    mbar_arrive1(&full[st]);
                }
                for (int n = 0; n < it.nslots; ++n) {
                    const int8_t* src = arow_s[n] + (size_t)c * KC * QK;
                    int8_t* dst = sa + (size_t)n * KC * QK;
                    // activations as [half][block][16 B]: the 16 lanes that own
                    // consecutive blocks read 256 contiguous bytes
                    for (int j = lane; j < 2 * KC; j += 32)
                        cp_async16_(dst + (size_t)(j & 1) * KC * 16 + (j >> 1) * 16, src + j * 16);
                    if (lane < KC / 8)                                                               // binary16 scales
                        cp_async16_(sd + (size_t)n * KC * 2 + lane * 16, ascale_s[n] + (size_t)c * KC + lane * 8);
                }
                cp_async_arrive_noinc_(&full[st]);
            }
            __syncwarp();
        }
        cp_async_wait_all_();
        if (ic > 0) mbar_wait_bounded(&full[(ic - 1) % NST], ((ic - 1) / NST) & 1, LIMIT);
    } else {
        // ------------------------------------------------------------ compute
        const int rg = 2 * warp + (lane >> 4);   // row group: rows RPL rg .. RPL rg + RPL - 1
        const int ks = lane & 15;                // this lane's blocks: ks, ks + 16, ...
        uint32_t ic = 0, cuse = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            const SItem it = (MODE == GEMV) ? SItem{0, 0, p.T, item} : item_of(item, n_rb, tile_off_s, off_s, ngroups);
            float acc[RPL][ST];
#pragma unroll
            for (int r = 0; r < RPL; ++r)
#pragma unroll
                for (int s = 0; s < ST; ++s) acc[r][s] = 0.0f;
            for (int c = 0; c < nchunk; ++c, ++ic) {
                const int st = ic % NST;
                if (!wait_phase_s(&full[st], (ic / NST) & 1, abort)) { ok = false; break; }
                const unsigned char* sw = smem + st * SZ_STAGE;
                const int8_t* sa = reinterpret_cast<const int8_t*>(sw + SZ_W);
                const uint16_t* sd = reinterpret_cast<const uint16_t*>(sw + SZ_W + SZ_A);
                CapPtr cap{nullptr, 0, RPL * rg, nb, 0};
                if (CAP && MODE != GEMV && it.g == p.cap_group && it.rb == p.cap_rb) {
                    cap.out = p.cap_out;
                    cap.slot_rel = it.slot0 - off_s[it.g];
                }
                for (int b = ks; b < KC; b += 16) {
                    cap.blk = c * KC + b;
                    // this lane's weight blocks (its RPL rows, block b), loaded once
                    uint32_t qs[RPL][4];
                    float dW[RPL];
#pragma unroll
                    for (int r = 0; r < RPL; ++r) {
                        uint32_t dbits;
                        load_q4_block_smem(sw + (size_t)(RPL * rg + r) * KC * Q4_BYTES + b * Q4_BYTES, qs[r], dbits);
                        dW[r] = half_bits_to_float(dbits);
                    }
                    // slot passes of 4, 2 or 1 as many slots as the tile holds
#pragma unroll
                    for (int sp = 0; sp < ST; sp += 4) {
                        const int rem = it.nslots - sp;
                        if (rem >= 4) {
                            block_slots<4, RPL, ST, CAP>(acc, sp, qs, dW, sa, sd, KC, b, cap);
                        } else if (rem >= 2) {
                            block_slots<2, RPL, ST, CAP>(acc, sp, qs, dW, sa, sd, KC, b, cap);
                            if (rem == 3) block_slots<1, RPL, ST, CAP>(acc, sp + 2, qs, dW, sa, sd, KC, b, cap);
                        } else if (rem == 1) {
                            block_slots<1, RPL, ST, CAP>(acc, sp, qs, dW, sa, sd, KC, b, cap);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive1(&empty[st]);
            }
            if (!ok) break;
            // the 16 lanes of a row group hold partial sums over their blocks
#pragma unroll
            for (int r = 0; r < RPL; ++r)
#pragma unroll
                for (int s = 0; s < ST; ++s) {
                    if (s < it.nslots) {
                        float v = acc[r][s];
                        v += __shfl_xor_sync(0xffffffffu, v, 8);
                        v += __shfl_xor_sync(0xffffffffu, v, 4);
                        v += __shfl_xor_sync(0xffffffffu, v, 2);
                        v += __shfl_xor_sync(0xffffffffu, v, 1);
                        if (ks == 0) res[(RPL * rg + r) * ST + s] = v;
                    }
                }
            if (!compute_sync(&cbar, cuse++, abort)) break;
            if (MODE == GATEUP) {
                // warp w < 8: slot w; lane = row f0 + lane of the 32-row block of h
                const int s = warp;
                if (s < it.nslots && s < ST) {
                    const int slot = it.slot0 + s;
                    const int f0 = it.rb * 32;
                    const float h = swiglu(res[lane * ST + s], res[(32 + lane) * ST + s]);
                    if (p.h_dbg) p.h_dbg[(size_t)slot * F + f0 + lane] = h;
                    uint16_t db;
                    bool ov;
                    const int q = q8_0_lane(h, db, ov);
                    p.hq[(size_t)slot * F + f0 + lane] = (int8_t)q;
                    if (lane == 0) {
                        p.dh[(size_t)slot * (F / QK) + it.rb] = db;
                        if (ov) atomicOr(p.status, STATUS_SCALE_OVERFLOW);
                    }
                }
            } else if (MODE == GEMV) {
                // warp w: token w & 7, rows 32 (w >> 3) .. + 31 of the item's 64 rows
                const int s = warp & (ST - 1), r = 32 * (warp / ST) + lane;
                const int n = it.rb * SR + r;
                if (s < it.nslots && n < p.N) p.y[(size_t)s * p.N + n] = res[r * ST + s];
            } else {
                // warp w: slot w & 7, rows 32 (w >> 3) .. + 31 of the 64 rows of H
                const int s = warp & (ST - 1), r = 32 * (warp / ST) + lane;
                if (s < it.nslots) {
                    int tok;
                    float w;
                    slot_tok(p, it.g, it.slot0 + s, tok, w);
                    atomicAdd(p.y + (size_t)tok * H + it.rb * SR + r, w * res[r * ST + s]);
                }
            }
            if (!compute_sync(&cbar, cuse++, abort)) break;  // res is free for the next item
        }
    }
    __syncthreads();
    if (tid == 0 && abort_s) atomicOr(p.status, STATUS_SPIN_TIMEOUT);
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 stream_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// `rows` rows of nb 18-byte blocks at `base` (row bytes a multiple of 144),
// viewed as [rows][nb * 18 / 8] 8-byte elements, copied as boxes of box_rows
// rows x KC blocks.
cudaError_t encode_rows_2d(CUtensorMap* map, const uint8_t* base, uint64_t rows, int nb, int KC, uint32_t box_rows) {
    const PFN_cuTensorMapEncodeTiled_v12000 enc = stream_encoder();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {(cuuint64_t)nb * Q4_BYTES / 8, rows};
    const cuuint64_t strides[1] = {(cuuint64_t)nb * Q4_BYTES};
    const cuuint32_t box[2] = {(cuuint32_t)(KC * Q4_BYTES / 8), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

StreamParams make_stream_params(const LayerView& L, int64_t T, const Workspace& ws, float* h_dbg, float* y) {
    StreamParams p;
    p.H = L.H; p.F = L.F; p.E = L.E; p.k = L.k; p.P = (int)(T * L.k);
    p.N = 0; p.T = 0;
    p.qa = ws.qa; p.da = ws.da; p.off = ws.off; p.tile_off = ws.tile_off; p.sorted = ws.sorted;
    p.topk_w = ws.topk_w; p.hq = ws.hq; p.dh = ws.dh; p.h_dbg = h_dbg; p.y = y; p.status = ws.status;
    p.cap_out = nullptr; p.cap_group = -1; p.cap_rb = -1;
    return p;
}

// Upper bound of the work tiles over all groups: sum_g ceil(c_g / ST).
int64_t stream_max_tiles(const LayerView& L, int64_t T) {
    const int64_t P = T * L.k;
    return ceil_div(P, ST) + std::min<int64_t>(L.E, P) + (L.S ? ceil_div(T, ST) : 0);
}

template <int MODE>
cudaError_t launch_stream(const LayerView& L, int64_t T, const Workspace& ws, float* h_dbg, float* y,
                          const DeviceInfo& dev, const BlockDotCapture* cap, cudaStream_t s) {
    const bool capture = cap && cap->down == (MODE == DOWN ? 1 : 0);
    const void* kfn = capture ? reinterpret_cast<const void*>(stream_dp4a_kernel<MODE, true>)
                              : reinterpret_cast<const void*>(stream_dp4a_kernel<MODE, false>);
    int per_sm = 0;
    cudaError_t e = kernel_occupancy(kfn, THREADS, SMEM_ALLOC, &per_sm);
    if (e != cudaSuccess) return e;
    StreamMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    const uint64_t E = (uint64_t)L.E, F = (uint64_t)L.F, H = (uint64_t)L.H;
    if (MODE == GATEUP) {
        const int nb = L.H / QK, KC = chunk_blocks(nb);
        e = encode_rows_2d(&maps.m[0], L.w_gate, E * F, nb, KC, 32);
        if (e == cudaSuccess) e = encode_rows_2d(&maps.m[1], L.w_up, E * F, nb, KC, 32);
        if (e == cudaSuccess && L.S) e = encode_rows_2d(&maps.m[2], L.sh_gate, F, nb, KC, 32);
        if (e == cudaSuccess && L.S) e = encode_rows_2d(&maps.m[3], L.sh_up, F, nb, KC, 32);
    } else {
        const int nb = L.F / QK, KC = chunk_blocks(nb);
        e = encode_rows_2d(&maps.m[0], L.w_down, E * H, nb, KC, SR);
        if (e == cudaSuccess && L.S) e = encode_rows_2d(&maps.m[2], L.sh_down, H, nb, KC, SR);
    }
    if (e != cudaSuccess) return e;
    const int n_rb = (MODE == GATEUP) ? L.F / 32 : L.H / SR;
    const int64_t items = stream_max_tiles(L, T) * n_rb;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(items, dev.sm_count));
    StreamParams p = make_stream_params(L, T, ws, h_dbg, y);
    if (capture) {
        p.cap_out = cap->out;
        p.cap_group = cap->group;
        p.cap_rb = cap->rb;
        stream_dp4a_kernel<MODE, true><<<(unsigned)grid, THREADS, SMEM_ALLOC, s>>>(p, maps);
    } else {
        stream_dp4a_kernel<MODE, false><<<(unsigned)grid, THREADS, SMEM_ALLOC, s>>>(p, maps);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemv_dp4a(const uint8_t* W, int64_t N, int H, const int8_t* qa, const uint16_t* da, int T,
                             float* y, uint32_t* status, const DeviceInfo& dev, cudaStream_t s) {
    int per_sm = 0;
    cudaError_t e =
        kernel_occupancy(reinterpret_cast<const void*>(stream_dp4a_kernel<GEMV, false>), THREADS, SMEM_ALLOC, &per_sm);
    if (e != cudaSuccess) return e;
    StreamMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    const int nb = H / QK, KC = chunk_blocks(nb);
    e = encode_rows_2d(&maps.m[0], W, (uint64_t)N, nb, KC, SR);
    if (e != cudaSuccess) return e;
    StreamParams p;
    std::memset(&p, 0, sizeof(p));
    p.H = H; p.N = (int)N; p.T = T; p.qa = qa; p.da = da; p.y = y; p.status = status;
    const int64_t items = ceil_div(N, SR);
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(items, dev.sm_count));
    p.cap_out = nullptr; p.cap_group = -1; p.cap_rb = -1;
    stream_dp4a_kernel<GEMV, false><<<(unsigned)grid, THREADS, SMEM_ALLOC, s>>>(p, maps);
    return cudaGetLastError();
}

cudaError_t launch_gateup_dp4a(const LayerView& L, int64_t T, const Workspace& ws, float* h_dbg,
                               const DeviceInfo& dev, const BlockDotCapture* cap, cudaStream_t s) {
    return launch_stream<GATEUP>(L, T, ws, h_dbg, nullptr, dev, cap, s);
}

cudaError_t launch_down_dp4a(const LayerView& L, int64_t T, const Workspace& ws, float* y,
                             const DeviceInfo& dev, const BlockDotCapture* cap, cudaStream_t s) {
    return launch_stream<DOWN>(L, T, ws, nullptr, y, dev, cap, s);
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
