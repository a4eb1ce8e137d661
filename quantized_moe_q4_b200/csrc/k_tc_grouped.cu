// k_tc_grouped.cu -- grouped W4A8 projections on the 5th-generation tensor
// cores (tcgen05.mma, accumulators in TMEM), warp-specialised and pipelined.
//
// The grouped 4-bit GEMM of the prefill ("A 35B Hybrid-Attention
// Mixture-of-Experts Model on a 6GB 2011 GPU", Dutch technical summary,
// Methodologie 1), with the page's single-pass prefill (Methodologie 4): every
// expert sees all of its tokens at once.
//
// Arithmetic.  Every Q4_0 block (32 weights along K) carries its own binary16
// scale, and so does every Q8_0 block of the activations, so the sum over K is
// sum_b dW[row,b] * dA[slot,b] * I_b with I_b the exact integer block dot
// product.  The tensor core computes I_b: operands hold the exact small
// integers (nibble - 8 in [-8, 7], q in [-127, 127]) as binary16, products and
// 32-term sums are exact in the fp32 accumulator, so each 32-wide block is two
// K=16 MMAs into its own TMEM buffer.  The epilogue then accumulates
// acc += I_b * (dW * dA) in fp32 registers (packed f32x2 FMUL + FFMA; the
// product of two binary16 scales is exact in binary32).  Binary16 rather than
// int8 operands spare an int32 -> fp32 conversion per accumulator element per
// block, which on B200 issues at about a quarter of the FMA rate and would
// bound the kernel.
//
// Tile: 128 weight rows (gate/up: 64 gate rows + the same 64 up rows; down:
// 128 rows of H) x 64 slots of one expert (MMA M = 128, N = 64).
//
// Warp roles (14 warps):
//   0      producer: 2D tensor copies (TMA) of the packed weight rows (a box
//          of 64 or 128 rows x 144 B = 8 blocks) and 16-byte cp.async gathers
//          of the slots' int8 activations and their scales, two input stages
//          of 8 blocks in flight;
//   1..4   converters: nibbles -> binary16 (nib - 8) for the A operand and
//          int8 -> binary16 activations for the B operand, both written into
//          the K-major shared-memory layout (8-row x 16-byte core matrices);
//          two operand stages of 4 blocks; block scales into a ring shared
//          with the epilogue;
//   5      MMA issuer (one thread): two MMAs per block (A and B from shared
//          memory), descriptors precomputed; one wait and one commit per
//          operand stage for its quad of accumulators;
//   6..13  epilogue: 4 TMEM lane quarters x 2 column halves; per quad of
//          blocks one wait, then two passes of two TMEM loads of 32 columns
//          and the rescale-accumulate; after the last block of a tile gate/up
//          -> SwiGLU + Q8_0 requantisation, down -> y += w_slot * o (fp32
//          atomics).
// TMEM: eight accumulators of 64 columns (all 512 columns), handed between the
// MMA issuer and the epilogue a quad (one operand stage) at a time; a 16-entry
// scale ring (so the converters run up to four operand stages ahead of the
// epilogue); full/empty mbarriers between every pair of roles; every wait
// bounded, and one that runs out makes every role leave its loop and records
// STATUS_SPIN_TIMEOUT.
// Why quads: the kernel is bound by its hand-off skeleton rather than by any
// role's arithmetic (measured on B200: with every role's work removed half of
// the time remains).  One mbarrier phase per block in each direction became
// one per pair (-10 to -12%) and then one per quad (-4 to -5% more, which
// needs all of TMEM for the accumulators and so the A operand in shared
// memory); deeper rings or more input stages changed nothing.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"
#include "tc.cuh"

namespace moeq4 {

namespace {

constexpr int TM = 128;            // MMA M: weight rows per tile
constexpr int TN = TC_TILE_TOKENS; // MMA N: slots per tile
constexpr int IN_KB = 8;           // Q4_0 blocks per input stage (144-byte rows: a 16-byte multiple)
constexpr int OP_KB = 4;           // blocks per operand stage
constexpr int NIN = 2, NOP = 2, NTM = 8, NSC = 16;  // input, operand, accumulator and scale ring depths
constexpr int IN_ROW = IN_KB * Q4_BYTES;          // 144
constexpr int THREADS = 14 * 32;  // 4 warps on some SM sub-partitions: at most 128 registers a thread
constexpr int W_PROD = 0, W_CONV0 = 1, W_MMA = 5, W_EPI0 = 6;
constexpr int N_CONV = 128, N_EPI = 256;
constexpr uint32_t TMEM_COLS = 512;
static_assert(NTM * TN <= TMEM_COLS, "TMEM budget");
static_assert(NTM == 2 * OP_KB, "two quads of accumulators, one per operand stage");
constexpr uint32_t LIMIT = 1u << 22;
static_assert(TN == 64, "the epilogue maps two warps of 32 columns onto a tile");

// dynamic shared memory map (bytes)
constexpr size_t SZ_IN_W = (size_t)TM * IN_ROW;           // one input stage of packed weight rows
constexpr size_t SZ_IN_B = (size_t)TN * IN_KB * QK;       // int8 activations, [16-byte chunk][slot]
constexpr size_t SZ_IN_DA = (size_t)TN * IN_KB * 2;       // activation scale bits, [slot][block]
constexpr size_t SZ_KSTEP_B = (size_t)TN * 32;
constexpr size_t SZ_OP_B = (size_t)OP_KB * 2 * SZ_KSTEP_B;
constexpr int XCH_LD = TN + 1;
constexpr size_t OFF_IN_W = 0;
constexpr size_t OFF_IN_B = OFF_IN_W + NIN * SZ_IN_W;
constexpr size_t OFF_IN_DA = OFF_IN_B + NIN * SZ_IN_B;
constexpr size_t OFF_OP_B = (OFF_IN_DA + NIN * SZ_IN_DA + 1023) & ~size_t(1023);
constexpr size_t SZ_KSTEP_A = (size_t)TM * 32;
constexpr size_t SZ_OP_A = (size_t)OP_KB * 2 * SZ_KSTEP_A;
constexpr size_t OFF_OP_A = OFF_OP_B + NOP * SZ_OP_B;
constexpr size_t OFF_DW = OFF_OP_A + NOP * SZ_OP_A;
constexpr size_t OFF_DA = OFF_DW + (size_t)NSC * TM * 4;
constexpr size_t OFF_XCH = OFF_DA + (size_t)NSC * TN * 4;
constexpr size_t SMEM_BYTES = OFF_XCH + (size_t)TM * XCH_LD * 4;
constexpr size_t SMEM_ALLOC = SMEM_BYTES + 1024;          // slack to align the map to 1024 B
static_assert(SMEM_ALLOC <= 220 * 1024, "shared memory map too large");

enum { GATEUP = 0, DOWN = 1 };

// Tensor maps of the weight matrices, rows of 18-byte blocks viewed as bytes:
// gate/up: [0] all experts' gate rows, [1] up rows, [2] shared gate, [3]
// shared up; down: [0] all experts' down rows, [2] shared down.
struct TcMaps {
    CUtensorMap m[4];
};

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
    int32_t* cap_out;  // block-dot capture (the CAP instantiation only)
    int cap_group, cap_rb;
};

// ---------------------------------------------------------------- helpers

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Arrive on `bar` once this thread's earlier cp.async copies complete; the
// arrival counts towards the barrier's expected count.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}


// Bounded wait shared by all roles: once any wait of the CTA has run out,
// `abort` is set and every later wait returns false soon after.
// The waiting thread sleeps in try_wait (suspend hint) rather than spinning;
// the bound is 2 s of wall time (globaltimer).
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, volatile int* abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 100000u)) return true;
        if (*abort) return false;
        if (global_ns() - t0 > 2000000000ull) break;
    }
    *abort = 1;
    return false;
}

// Barrier of the epilogue warps (one arrival per warp), bounded like every
// other wait so that a role that gave up cannot strand the others.
__device__ __forceinline__ bool epi_sync(uint64_t* bar, uint32_t use, volatile int* abort) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
    return wait_phase(bar, use & 1, abort);
}

// 2D tiled tensor copy global -> shared (no multicast), completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// acc[slot pair j] += I (32 columns of one block) * dW * dA[slot].
__device__ __forceinline__ void rescale_acc(float2 (&acc)[16], const uint32_t (&r)[32], float dwv, const float* da) {
    const float4* da4 = reinterpret_cast<const float4*>(da);
    const float2 dw2 = make_float2(dwv, dwv);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float4 d = da4[j];
        const float2 s0 = __fmul2_rn(dw2, make_float2(d.x, d.y));
        const float2 s1 = __fmul2_rn(dw2, make_float2(d.z, d.w));
        acc[2 * j] = __ffma2_rn(make_float2(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1])), s0, acc[2 * j]);
        acc[2 * j + 1] =
            __ffma2_rn(make_float2(__uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])), s1, acc[2 * j + 1]);
    }
}

// D[tmem] (=|+=) A[smem] x B[smem]^T, binary16 operands, fp32 accumulator;
// both operands K-major in 8-row x 16-byte core matrices.
__device__ __forceinline__ void mma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
        : "memory");
}

// kind::f16 instruction descriptor: binary16 A and B, fp32 accumulator, both
// operands K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
    return (1u << 4)                        // accumulator format: F32
           | ((uint32_t)(N >> 3) << 17)     // N / 8
           | ((uint32_t)(M >> 4) << 24);    // M / 16
}

// Four unsigned bytes u_i of w -> binary16 (1024 + u_i) - bias, two per word:
// 1024 + u has the bit pattern 0x6400 | u for u < 256, and the subtraction of
// two exact small integers is exact.
__device__ __forceinline__ uint2 bytes_to_f16(uint32_t w, uint32_t bias2) {
    const uint32_t lo = __byte_perm(w, 0x64646464u, 0x4140);
    const uint32_t hi = __byte_perm(w, 0x64646464u, 0x4342);
    const __half2 b = *reinterpret_cast<const __half2*>(&bias2);
    const __half2 a0 = __hsub2(*reinterpret_cast<const __half2*>(&lo), b);
    const __half2 a1 = __hsub2(*reinterpret_cast<const __half2*>(&hi), b);
    return make_uint2(*reinterpret_cast<const uint32_t*>(&a0), *reinterpret_cast<const uint32_t*>(&a1));
}

constexpr uint32_t BIAS_NIB = 0x64086408u;   // binary16 1032, twice: 1024 + n - 1032 = n - 8
constexpr uint32_t BIAS_ACT = 0x64806480u;   // binary16 1152, twice: 1024 + (q ^ 0x80) - 1152 = q

// Byte offset of the 16-byte core-matrix piece `core` (0/1) of row r in K-step
// `ks` of block `kb` of an operand stage with `rows` rows: K-steps are 32-byte
// (16 x binary16) slabs; inside one, 8-row groups are 256 B apart and the two
// pieces of a row 128 B apart (the descriptor's SBO and LBO).
__device__ __forceinline__ uint32_t op_off(int kb, int ks, int rows, int r, int core) {
    return (uint32_t)((kb * 2 + ks) * rows * 32 + (r >> 3) * 256 + core * 128 + (r & 7) * 16);
}

__device__ __forceinline__ int find_group(const int* tile_off, int ngroups, int tile) {
    int lo = 0, hi = ngroups;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tile_off[mid] <= tile) lo = mid; else hi = mid;
    }
    return lo;
}

struct Tile {
    int g, slot0, nslots, rb;
};

// Work item -> (group, first slot, slots in the tile, row block).
__device__ __forceinline__ Tile tile_of(int item, int n_rb, const int* tile_off_s, const int* off_s, int ngroups) {
    Tile t;
    const int tile = item / n_rb;
    t.rb = item - tile * n_rb;
    t.g = find_group(tile_off_s, ngroups, tile);
    t.slot0 = off_s[t.g] + (tile - tile_off_s[t.g]) * TN;
    t.nslots = min(TN, off_s[t.g + 1] - t.slot0);
    return t;
}

// Token and routing weight of slot s of group g (group E: the shared expert,
// slot P + t is token t with weight 1).
__device__ __forceinline__ void slot_info(const TcParams& p, int g, int s, int& tok, float& w) {
    if (g < p.E) {
        const int pair = __ldg(p.sorted + s);
        tok = pair / p.k;
        w = __ldg(p.topk_w + pair);
    } else {
        tok = s - p.P;
        w = 1.0f;
    }
}

}  // namespace

// CAP: also write the per-block integer sums (the MMA accumulators before the
// rescale) of one row block of one group to p.cap_out (test instantiation).
template <int MODE, bool CAP>
__global__ void __launch_bounds__(THREADS, 1) tc_grouped_kernel(TcParams p, const __grid_constant__ TcMaps maps) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t in_full[NIN], in_empty[NIN], op_full[NOP], op_empty[NOP], tm_full[2],
        tm_empty[2], sc_full[NSC], sc_empty[NSC], epi_bar;
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    __shared__ int tile_off_s[258], off_s[258];

    uint8_t* in_w = smem + OFF_IN_W;
    int8_t* in_b = reinterpret_cast<int8_t*>(smem + OFF_IN_B);
    uint16_t* in_da = reinterpret_cast<uint16_t*>(smem + OFF_IN_DA);
    uint8_t* op_b = smem + OFF_OP_B;
    uint8_t* op_a = smem + OFF_OP_A;
    float* dw_ring = reinterpret_cast<float*>(smem + OFF_DW);
    float* da_ring = reinterpret_cast<float*>(smem + OFF_DA);
    float* xch = reinterpret_cast<float*>(smem + OFF_XCH);
    volatile int* abort = &abort_s;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = p.H, F = p.F, E = p.E;
    const int K = (MODE == GATEUP) ? H : F;
    const int nbK = K / QK;
    const int nbF = F / QK;
    const int n_rb = (MODE == GATEUP) ? F / 64 : H / TM;
    const int ngroups = E + 1;

    if (warp == W_PROD) {
        tmem_alloc(&tmem_base_s, TMEM_COLS);
        tmem_relinquish();
    }
    if (tid == 32) {
        abort_s = 0;
        for (int i = 0; i < NIN; ++i) {
            mbar_init(&in_full[i], 64);   // 32 producer-lane arrivals + 32 cp.async arrivals
            mbar_init(&in_empty[i], N_CONV);
        }
        for (int i = 0; i < NOP; ++i) {
            mbar_init(&op_full[i], N_CONV);
            mbar_init(&op_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {  // one quad of accumulators each
            mbar_init(&tm_full[i], 1);
            mbar_init(&tm_empty[i], N_EPI / 32);
        }
        for (int i = 0; i < NSC; ++i) {
            mbar_init(&sc_full[i], N_CONV / 32);
            mbar_init(&sc_empty[i], N_EPI / 32);
        }
        mbar_init(&epi_bar, N_EPI / 32);
        mbar_fence_init();
    }
    for (int i = tid; i <= ngroups; i += THREADS) {
        tile_off_s[i] = p.tile_off[i];
        off_s[i] = p.off[i];
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = tmem_base_s;
    const int n_items = tile_off_s[ngroups] * n_rb;

    if (warp == W_PROD) {
        // ------------------------------------------------------------ producer
        uint32_t i_in = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            const Tile T = tile_of(item, n_rb, tile_off_s, off_s, ngroups);
            // weight rows of this item: one box of 64 gate + one of 64 up rows, or 128 down rows
            const bool shared_g = T.g >= E;
            const CUtensorMap* map0 = &maps.m[shared_g ? 2 : 0];
            const CUtensorMap* map1 = &maps.m[shared_g ? 3 : 1];
            const int wy = (shared_g ? 0 : T.g * ((MODE == GATEUP) ? F : H)) + T.rb * ((MODE == GATEUP) ? 64 : TM);
            const int8_t* arow[2];
            const uint16_t* ascale[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int n = lane + 32 * j;
                arow[j] = nullptr;
                ascale[j] = nullptr;
                if (n < T.nslots) {
                    const int s = T.slot0 + n;
                    int tok;
                    float w;
                    slot_info(p, T.g, s, tok, w);
                    if (MODE == GATEUP) {
                        arow[j] = p.qa + (size_t)tok * H;
                        ascale[j] = p.da + (size_t)tok * (H / QK);
                    } else {
                        arow[j] = p.hq + (size_t)s * F;
                        ascale[j] = p.dh + (size_t)s * nbF;
                    }
                }
            }
            for (int c = 0; c < nbK / IN_KB; ++c, ++i_in) {
                const int s = i_in % NIN;
                if (!wait_phase(&in_empty[s], ((i_in / NIN) & 1) ^ 1, abort)) { ok = false; break; }
                uint8_t* dw = in_w + (size_t)s * SZ_IN_W;
                int8_t* db = in_b + (size_t)s * SZ_IN_B;
                uint16_t* dda = in_da + (size_t)s * TN * IN_KB;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&in_full[s], (uint32_t)(TM * IN_ROW));
                    tma_load_2d(dw, map0, c * IN_ROW, wy, &in_full[s]);
                    if (MODE == GATEUP) tma_load_2d(dw + 64 * IN_ROW, map1, c * IN_ROW, wy, &in_full[s]);
                } else {
                    mbar_arrive(&in_full[s]);
                }
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    if (arow[j]) {
                        const int n = lane + 32 * j;
                        const int8_t* src = arow[j] + (size_t)c * IN_KB * QK;
#pragma unroll
                        for (int q = 0; q < IN_KB * 2; ++q) cp_async16(db + ((size_t)q * TN + n) * 16, src + q * 16);
                        cp_async16(dda + n * IN_KB, ascale[j] + c * IN_KB);   // 8 binary16 scales
                    }
                }
                cp_async_arrive_noinc(&in_full[s]);
            }
        }
        // let the copies in flight land before the CTA can exit
        cp_async_wait_all();
        if (i_in > 0) mbar_wait_bounded(&in_full[(i_in - 1) % NIN], ((i_in - 1) / NIN) & 1, LIMIT);
    } else if (warp >= W_CONV0 && warp < W_CONV0 + 4) {
        // ------------------------------------------------------------ converters
        const int ct = tid - W_CONV0 * 32;        // slot column ct & 63 of the activation work
        const int crow = 32 * (warp & 3) + lane;  // weight row this thread converts
        uint32_t i_op = 0, gb = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            const Tile T = tile_of(item, n_rb, tile_off_s, off_s, ngroups);
            for (int c = 0; c < nbK / OP_KB && ok; ++c, ++i_op, gb += OP_KB) {
                const uint32_t i_in = i_op >> 1;
                const int s = i_in % NIN, sub = i_op & 1;
                if (sub == 0 && !wait_phase(&in_full[s], (i_in / NIN) & 1, abort)) { ok = false; break; }
                const int o = i_op % NOP;
                if (!wait_phase(&op_empty[o], ((i_op / NOP) & 1) ^ 1, abort)) { ok = false; break; }
                tc_fence_after_sync();
                uint8_t* ob = op_b + (size_t)o * SZ_OP_B;

                // weights: this row's 4 blocks, 72 bytes at an 8-byte boundary
                uint32_t w[18];
                const uint2* wsrc = reinterpret_cast<const uint2*>(in_w + (size_t)s * SZ_IN_W + (size_t)crow * IN_ROW +
                                                                   sub * OP_KB * Q4_BYTES);
#pragma unroll
                for (int i = 0; i < 9; ++i) {
                    const uint2 v = wsrc[i];
                    w[2 * i] = v.x;
                    w[2 * i + 1] = v.y;
                }
                float dws[OP_KB];
                uint32_t v[OP_KB * 16];  // the 4 blocks' binary16 pairs of this row, in K order
#pragma unroll
                for (int kb = 0; kb < OP_KB; ++kb) {
                    // block kb starts at byte 18 kb: scale, then 16 nibble bytes
                    const int bw = (18 * kb) / 4;
                    uint32_t qs[4], dbits;
                    if ((kb & 1) == 0) {
                        dbits = w[bw] & 0xffffu;
#pragma unroll
                        for (int i = 0; i < 4; ++i) qs[i] = __funnelshift_r(w[bw + i], w[bw + i + 1], 16);
                    } else {
                        dbits = w[bw] >> 16;
#pragma unroll
                        for (int i = 0; i < 4; ++i) qs[i] = w[bw + 1 + i];
                    }
                    dws[kb] = half_bits_to_float(dbits);
                    // columns 0..7 of a block: low nibbles (weights 0..15), 8..15: high nibbles (16..31)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint2 lo = bytes_to_f16(qs[i] & 0x0f0f0f0fu, BIAS_NIB);
                        const uint2 hi = bytes_to_f16((qs[i] >> 4) & 0x0f0f0f0fu, BIAS_NIB);
                        v[16 * kb + 2 * i] = lo.x;
                        v[16 * kb + 2 * i + 1] = lo.y;
                        v[16 * kb + 8 + 2 * i] = hi.x;
                        v[16 * kb + 8 + 2 * i + 1] = hi.y;
                    }
                }
                // this row of the A operand: block kb, K-step ks, core matrix
                // `core` holds binary16 pairs 16 kb + 8 ks + 4 core .. + 3
                uint8_t* oa = op_a + (size_t)o * SZ_OP_A;
#pragma unroll
                for (int kb = 0; kb < OP_KB; ++kb)
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                        for (int core = 0; core < 2; ++core) {
                            const int c0 = 16 * kb + 8 * ks + 4 * core;
                            *reinterpret_cast<uint4*>(oa + op_off(kb, ks, TM, crow, core)) =
                                make_uint4(v[c0], v[c0 + 1], v[c0 + 2], v[c0 + 3]);
                        }
                // activations: slot n = ct & 63, blocks (ct >> 6) and (ct >> 6) + 2
                const int n = ct & 63;
                const bool valid = n < T.nslots;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int kb = (ct >> 6) + 2 * j;
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        uint4 v = make_uint4(0, 0, 0, 0), u = make_uint4(0, 0, 0, 0);
                        if (valid) {
                            const int q = (sub * OP_KB + kb) * 2 + ks;
                            const uint4 a = *reinterpret_cast<const uint4*>(in_b + (size_t)s * SZ_IN_B +
                                                                            ((size_t)q * TN + n) * 16);
                            const uint2 a0 = bytes_to_f16(a.x ^ 0x80808080u, BIAS_ACT);
                            const uint2 a1 = bytes_to_f16(a.y ^ 0x80808080u, BIAS_ACT);
                            const uint2 a2 = bytes_to_f16(a.z ^ 0x80808080u, BIAS_ACT);
                            const uint2 a3 = bytes_to_f16(a.w ^ 0x80808080u, BIAS_ACT);
                            v = make_uint4(a0.x, a0.y, a1.x, a1.y);
                            u = make_uint4(a2.x, a2.y, a3.x, a3.y);
                        }
                        *reinterpret_cast<uint4*>(ob + op_off(kb, ks, TN, n, 0)) = v;
                        *reinterpret_cast<uint4*>(ob + op_off(kb, ks, TN, n, 1)) = u;
                    }
                }
                // this slot's activation scales, read before the input stage is released
                float das[OP_KB];
#pragma unroll
                for (int kb = 0; kb < OP_KB; ++kb)
                    das[kb] = valid ? half_bits_to_float(in_da[(size_t)s * TN * IN_KB + n * IN_KB + sub * OP_KB + kb])
                                    : 0.0f;
                fence_proxy_async_smem();
                tc_fence_before_sync();
                mbar_arrive(&op_full[o]);
                if (sub == 1) mbar_arrive(&in_empty[s]);
                // scales of these 4 blocks into the ring read by the epilogue; the
                // epilogue frees the last entry of each group of four, in order
                const uint32_t glast = gb + OP_KB - 1, buf0 = gb % NSC;
                if (!wait_phase(&sc_empty[glast % NSC], ((glast / NSC) & 1) ^ 1, abort)) { ok = false; break; }
#pragma unroll
                for (int kb = 0; kb < OP_KB; ++kb) {
                    dw_ring[(buf0 + kb) * TM + crow] = dws[kb];
                    if (ct < TN) da_ring[(buf0 + kb) * TN + ct] = das[kb];
                }
                __syncwarp();
                if (lane == 0) {
#pragma unroll
                    for (int kb = 0; kb < OP_KB; ++kb) mbar_arrive(&sc_full[buf0 + kb]);
                }
            }
        }
    } else if (warp == W_MMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16(TM, TN);
            // descriptors of the first K-step of each operand stage; a later
            // K-step adds its byte offset / 16 to the start-address field
            const uint64_t b0 = smem_desc_kmajor(op_b, 128, 256), b1 = smem_desc_kmajor(op_b + SZ_OP_B, 128, 256);
            const uint64_t a0 = smem_desc_kmajor(op_a, 128, 256), a1 = smem_desc_kmajor(op_a + SZ_OP_A, 128, 256);
            static_assert(NOP == 2, "two operand stages");
            uint32_t i_op = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
                for (int c = 0; c < nbK / OP_KB; ++c, ++i_op) {
                    const int o = i_op & 1;
                    if (!wait_phase(&op_full[o], (i_op / NOP) & 1, abort)) {
                        ok = false;
                        break;
                    }
                    // the quad of accumulators of this operand stage: buffers 4o .. 4o + 3,
                    // freed by the epilogue two stages ago
                    if (!wait_phase(&tm_empty[o], ((i_op / 2) & 1) ^ 1, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint64_t bd = o ? b1 : b0, ad = o ? a1 : a0;
#pragma unroll
                    for (int kb = 0; kb < OP_KB; ++kb) {
                        const uint32_t d = tmem + (uint32_t)(OP_KB * o + kb) * TN;
                        mma_f16_ss(d, ad + (uint64_t)((kb * 2) * (SZ_KSTEP_A >> 4)),
                                   bd + (uint64_t)((kb * 2) * (SZ_KSTEP_B >> 4)), idesc, false);
                        mma_f16_ss(d, ad + (uint64_t)((kb * 2 + 1) * (SZ_KSTEP_A >> 4)),
                                   bd + (uint64_t)((kb * 2 + 1) * (SZ_KSTEP_B >> 4)), idesc, true);
                    }
                    mma_commit(&tm_full[o]);  // covers the quad's eight MMAs
                    mma_commit(&op_empty[o]);
                    if (!ok) break;
                }
            }
            // the last commit's arrival must land before the CTA can exit
            if (i_op > 0) mbar_wait_bounded(&op_empty[(i_op - 1) % NOP], ((i_op - 1) / NOP) & 1, LIMIT);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                   // TMEM lane quarter this warp may access
        const int hcol = (warp - W_EPI0) >> 2;    // column half: slots 32 hcol .. 32 hcol + 31
        const int row = 32 * q + lane;            // weight row (TMEM lane) of this thread
        const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + 32 * hcol;
        uint32_t gb = 0, epi_phase = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            const Tile T = tile_of(item, n_rb, tile_off_s, off_s, ngroups);
            float2 acc[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = make_float2(0.0f, 0.0f);
            // one wait per quad of blocks (one operand stage); two blocks per pass,
            // both TMEM loads in flight before either is used
            for (int b = 0; b < nbK; b += OP_KB, gb += OP_KB) {
                const uint32_t qd = (gb / OP_KB) & 1, qpar = (gb / (2 * OP_KB)) & 1;
                const uint32_t s0 = gb % NSC, spar = (gb / NSC) & 1;
                // the converters arrive on the four scale entries in order, so the
                // last one complete means all four are
                if (!wait_phase(&tm_full[qd], qpar, abort) || !wait_phase(&sc_full[s0 + 3], spar, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const uint32_t bb = OP_KB * qd + 2 * h2, sa = s0 + 2 * h2;
                    uint32_t r0[32], r1[32];
                    tmem_ld32(taddr + bb * TN, r0);
                    tmem_ld32(taddr + (bb + 1) * TN, r1);
                    tmem_wait_ld();
                    if (CAP && T.g == p.cap_group && T.rb == p.cap_rb) {
                        // exact integers held in binary32: convert back without rounding
                        const size_t s0 = (size_t)(T.slot0 - off_s[T.g]);
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int n = 32 * hcol + j;
                            if (n < T.nslots) {
                                int32_t* o = p.cap_out + ((s0 + n) * TM + row) * nbK + b + 2 * h2;
                                o[0] = __float2int_rn(__uint_as_float(r0[j]));
                                o[1] = __float2int_rn(__uint_as_float(r1[j]));
                            }
                        }
                    }
                    rescale_acc(acc, r0, dw_ring[sa * TM + row], da_ring + sa * TN + 32 * hcol);
                    rescale_acc(acc, r1, dw_ring[(sa + 1) * TM + row], da_ring + (sa + 1) * TN + 32 * hcol);
                }
                tc_fence_before_sync();
                __syncwarp();
                // the converters wait only on the last entry of each group of four
                if (lane == 0) {
                    mbar_arrive(&tm_empty[qd]);
                    mbar_arrive(&sc_empty[s0 + 3]);
                }
            }
            if (!ok) break;
            if (MODE == GATEUP) {
                float* xr = xch + (size_t)row * XCH_LD + 32 * hcol;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    xr[2 * j] = acc[j].x;
                    xr[2 * j + 1] = acc[j].y;
                }
                if (!epi_sync(&epi_bar, epi_phase++, abort)) break;
                // SwiGLU + Q8_0 of h.  A unit is one 32-row block of h (gate rows
                // 32 fb .. 32 fb + 31) of one slot n; two lanes share a unit, 16
                // rows each, so every value is independent of the others and a
                // single shuffle gives the block's absolute maximum.  Both
                // divisions of the Q8_0 rule stay IEEE (div.rn).
                const int u = ((warp - W_EPI0) * 32 + lane) >> 1;   // 0..127
                const int n = u & 63, fb = u >> 6, half = lane & 1;
                const int r0 = 32 * fb + 16 * half;
                const int f0 = T.rb * 64;
                float h[16];
                float amax = 0.0f;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    h[j] = swiglu(xch[(size_t)(r0 + j) * XCH_LD + n], xch[(size_t)(64 + r0 + j) * XCH_LD + n]);
                    amax = fmaxf(amax, fabsf(h[j]));
                }
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
                const float d = __fdiv_rn(amax, 127.0f);
                const uint16_t dbits = __half_as_ushort(__float2half_rn(d));
                uint32_t packed[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    int qv = 0;
                    if (d != 0.0f) qv = max(-127, min(127, round_half_away(__fdiv_rn(h[j], d))));
                    packed[j >> 2] |= (uint32_t)(qv & 0xff) << (8 * (j & 3));
                }
                if (n < T.nslots) {
                    const int sl = T.slot0 + n;
                    *reinterpret_cast<uint4*>(p.hq + (size_t)sl * F + f0 + r0) =
                        make_uint4(packed[0], packed[1], packed[2], packed[3]);
                    if (p.h_dbg) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) p.h_dbg[(size_t)sl * F + f0 + r0 + j] = h[j];
                    }
                    if (half == 0) {
                        p.dh[(size_t)sl * nbF + (f0 >> 5) + fb] = dbits;
                        if ((dbits & 0x7fffu) == 0x7c00u) atomicOr(p.status, STATUS_SCALE_OVERFLOW);
                    }
                }
                if (!epi_sync(&epi_bar, epi_phase++, abort)) break;  // xch is free for the next tile
            } else {
                int tok = 0;
                float w = 0.0f;
                const int n_me = 32 * hcol + lane;
                if (n_me < T.nslots) slot_info(p, T.g, T.slot0 + n_me, tok, w);
                const int h0 = T.rb * TM;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int tj = __shfl_sync(0xffffffffu, tok, j);
                    const float wj = __shfl_sync(0xffffffffu, w, j);
                    const float v = (j & 1) ? acc[j >> 1].y : acc[j >> 1].x;
                    if (32 * hcol + j < T.nslots) atomicAdd(p.y + (size_t)tj * H + h0 + row, wj * v);
                }
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (tid == 0 && abort_s) atomicOr(p.status, STATUS_SPIN_TIMEOUT);
    if (warp == W_PROD) tmem_dealloc(tmem, TMEM_COLS);
}

static TcParams make_tc_params(const LayerView& L, int64_t T, const Workspace& ws, float* h_dbg, float* y) {
    TcParams p;
    p.H = L.H; p.F = L.F; p.E = L.E; p.k = L.k; p.P = (int)(T * L.k);
    p.w_gate = L.w_gate; p.w_up = L.w_up; p.w_down = L.w_down;
    p.sh_gate = L.sh_gate; p.sh_up = L.sh_up; p.sh_down = L.sh_down;
    p.qa = ws.qa; p.da = ws.da; p.off = ws.off; p.tile_off = ws.tile_off; p.sorted = ws.sorted;
    p.topk_w = ws.topk_w; p.hq = ws.hq; p.dh = ws.dh; p.h_dbg = h_dbg; p.y = y; p.status = ws.status;
    p.cap_out = nullptr; p.cap_group = -1; p.cap_rb = -1;
    return p;
}

static int64_t tc_max_tiles(const LayerView& L, int64_t T) {
    const int64_t P = T * L.k;
    return ceil_div(P, TN) + std::min<int64_t>(L.E, P) + (L.S ? ceil_div(T, TN) : 0);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// dependency on the driver library).
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// `rows` rows of `row_bytes` bytes at `base` (16-byte aligned, row_bytes a
// multiple of 16), copied as boxes of `box_rows` rows x 144 bytes.
static cudaError_t encode_rows(CUtensorMap* map, const uint8_t* base, uint64_t rows, uint64_t row_bytes,
                               uint32_t box_rows) {
    const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {row_bytes, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)IN_ROW, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int MODE>
static cudaError_t make_maps(const LayerView& L, TcMaps* maps) {
    std::memset(maps, 0, sizeof(TcMaps));
    const uint64_t E = (uint64_t)L.E, F = (uint64_t)L.F, H = (uint64_t)L.H;
    cudaError_t e = cudaSuccess;
    if (MODE == GATEUP) {
        const uint64_t rb = H / QK * Q4_BYTES;
        if (e == cudaSuccess) e = encode_rows(&maps->m[0], L.w_gate, E * F, rb, 64);
        if (e == cudaSuccess) e = encode_rows(&maps->m[1], L.w_up, E * F, rb, 64);
        if (L.S && e == cudaSuccess) e = encode_rows(&maps->m[2], L.sh_gate, F, rb, 64);
        if (L.S && e == cudaSuccess) e = encode_rows(&maps->m[3], L.sh_up, F, rb, 64);
    } else {
        const uint64_t rb = F / QK * Q4_BYTES;
        if (e == cudaSuccess) e = encode_rows(&maps->m[0], L.w_down, E * H, rb, TM);
        if (L.S && e == cudaSuccess) e = encode_rows(&maps->m[2], L.sh_down, H, rb, TM);
    }
    return e;
}

template <int MODE>
static cudaError_t launch_tc(const LayerView& L, int64_t T, const Workspace& ws, float* h_dbg, float* y,
                             const DeviceInfo& dev, const BlockDotCapture* cap, cudaStream_t s) {
    const bool capture = cap && cap->down == (MODE == DOWN ? 1 : 0);
    const void* kfn = capture ? reinterpret_cast<const void*>(tc_grouped_kernel<MODE, true>)
                              : reinterpret_cast<const void*>(tc_grouped_kernel<MODE, false>);
    int per_sm = 0;
    cudaError_t e = kernel_occupancy(kfn, THREADS, SMEM_ALLOC, &per_sm);
    if (e != cudaSuccess) return e;
    TcMaps maps;
    e = make_maps<MODE>(L, &maps);
    if (e != cudaSuccess) return e;
    const int n_rb = (MODE == GATEUP) ? L.F / 64 : L.H / TM;
    const int64_t items = tc_max_tiles(L, T) * n_rb;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(items, dev.sm_count));
    TcParams p = make_tc_params(L, T, ws, h_dbg, y);
    if (capture) {
        p.cap_out = cap->out;
        p.cap_group = cap->group;
        p.cap_rb = cap->rb;
        tc_grouped_kernel<MODE, true><<<(unsigned)grid, THREADS, SMEM_ALLOC, s>>>(p, maps);
    } else {
        tc_grouped_kernel<MODE, false><<<(unsigned)grid, THREADS, SMEM_ALLOC, s>>>(p, maps);
    }
    return cudaGetLastError();
}

cudaError_t launch_gateup_tc(const LayerView& L, int64_t T, const Workspace& ws, float* h_dbg, const DeviceInfo& dev,
                             const BlockDotCapture* cap, cudaStream_t s) {
    return launch_tc<GATEUP>(L, T, ws, h_dbg, nullptr, dev, cap, s);
}

cudaError_t launch_down_tc(const LayerView& L, int64_t T, const Workspace& ws, float* y, const DeviceInfo& dev,
                           const BlockDotCapture* cap, cudaStream_t s) {
    return launch_tc<DOWN>(L, T, ws, nullptr, y, dev, cap, s);
}

}  // namespace moeq4
