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
// product.  The tensor core computes I_b into its own TMEM buffer, from the
// exact small integers (nibble - 8 in [-8, 7], q in [-127, 127]) held either
// as int8 (kind::i8, one K = 32 MMA a block, int32 accumulator started at a
// bias that makes its bits an fp32 1.5 * 2^23 + I_b) or as binary16
// (kind::f16, two K = 16 MMAs a block; products and 32-term sums are exact in
// the fp32 accumulator).  The epilogue then accumulates acc += I_b * (dW * dA)
// in fp32 registers (packed f32x2 FMUL + FFMA, plus one packed FADD taking
// the bias off for int8; the product of two binary16 scales is exact in
// binary32).  int8 operands spare the converters the activations altogether
// (the MMA reads the codes where the producer copied them) and halve the
// weight bytes, but cost the epilogue the FADD and the TMEM reset: they win
// on 32-slot tiles, which also take 8 blocks per operand stage, and lose on
// 64- and 128-slot tiles, whose epilogues have more columns per block.
//
// Tile: 128 weight rows (gate/up: 64 gate rows + the same 64 up rows; down:
// 128 rows of H) x TN slots of one expert (MMA M = 128, N = TN), TN = 32, 64
// or 128, chosen per call from the routed slots per expert (tc_tile_tokens):
// a weight block converted once serves TN slots.
//
// Warp roles (18 warps for TN = 32 and 64, 14 for 128); the pipeline depths
// and stage sizes per width are in TcCfg:
//   0      producer: 2D tensor copies (TMA) of the packed weight rows (a box
//          of 64 or 128 rows x 144 B = 8 blocks), and the activation ring's
//          cp.async copies (a slot's codes and scales per operand stage),
//          issued as far ahead as the ring allows;
//   1..    converters (8 warps, 4 for TN = 128): a pair of blocks of a weight
//          row per thread (two pairs on 32-slot tiles): nibbles -> nib - 8
//          (int8 or binary16) for the A operand, read as 16-byte loads of the
//          window around the pair.  binary16 tiles: the threads also turn
//          slots' codes from the ring into binary16 for the B operand (128
//          slots: the pair of slot `row`; 64 slots: one block each, so every
//          thread has the same share).  int8 tiles: the MMA reads B in the
//          ring, and the first TN / 32 warps take the slots' scales.  Operands
//          are K-major (8-row x 16-byte core matrices); block scales go into a
//          ring read by the epilogue;
//   then   the MMA issuer (one thread): one (int8) or two (binary16) MMAs per
//          block, A and B from shared memory; one wait and one commit per
//          operand stage, for its set of accumulators;
//   last   epilogue (8 warps): 4 TMEM lane quarters x TN / CW column groups
//          (CW = 16, 32 or 64 for TN = 32, 64, 128); per operand stage one
//          wait, TMEM loads of 16 columns software-pipelined against the
//          rescale-accumulate, the accumulator set released as soon as its
//          last chunk is in registers; after the last block of a tile
//          gate/up -> SwiGLU + Q8_0 requantisation, down -> y += w_slot * o
//          with vector reductions (red.v4.f32) of 4 consecutive rows of H of
//          one token.
// TMEM: two sets of OP_KB accumulators of TN columns (all 512 columns),
// handed between the MMA issuer and the epilogue a set (one operand stage) at
// a time; full/empty mbarriers between every pair of roles; every wait
// bounded, and one that runs out makes every role leave its loop and records
// STATUS_SPIN_TIMEOUT.
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
constexpr int IN_KB = 8;           // Q4_0 blocks per input stage (144-byte rows: a 16-byte multiple)
constexpr int IN_ROW = IN_KB * Q4_BYTES;          // 144
constexpr int W_PROD = 0, W_CONV0 = 1;
constexpr uint32_t LIMIT = 1u << 22;
constexpr size_t SZ_IN_W = (size_t)TM * IN_ROW;           // one input stage of packed weight rows

// Per tile width TN (slots, the MMA N): the blocks per operand stage, the
// epilogue's column groups of 4 warps (one per TMEM lane quarter), and the
// shared-memory map.
template <int TN>
struct TcCfg {
    static_assert(TN == 32 || TN == 64 || TN == 128, "tile widths");
    // blocks per operand stage: each stage is one hand-off between the roles,
    // so narrower tiles (less epilogue work a block) take more blocks a stage:
    // eight for 32 slots, four for 64, two for 128 (TMEM holds 512 columns)
    static constexpr int OP_KB = (TN == 128) ? 2 : (TN == 64) ? 4 : 8;
    // pipeline depths: input stages of weight rows (NIN), operand stages
    // (NOP), accumulator sets in TMEM (NTS), the scale ring (NSC) and the
    // activation ring (NPF: operand stages of a slot's OP_KB blocks of int8
    // codes and their binary16 scales, copied by the producer warp); the
    // narrow tiles have the shared memory to run deeper
    static constexpr int NIN = (TN == 32) ? 3 : 2;
    static constexpr int NOP = 2;
    static constexpr int NTS = 2;
    static constexpr int NSC = 4;
    static constexpr int NPF = (TN == 32) ? 6 : 4;
    static constexpr int NACC = NTS * OP_KB;              // accumulators: NTS sets of OP_KB
    // operand type: int8 (kind::i8, one K = 32 MMA a block) for 32-slot tiles,
    // binary16 (kind::f16, two K = 16 MMAs a block) for wider ones
    static constexpr bool I8 = (TN == 32);
    static constexpr int OPB = I8 ? 1 : 2;                // bytes per operand element
    static constexpr size_t SZ_OP_A = (size_t)OP_KB * OPB * TM * 32;   // one operand stage of A
    // a ring entry: OP_KB x 32 codes, OP_KB binary16 scales, padded to 16 bytes
    static constexpr size_t BPF_SLOT = ((size_t)OP_KB * (QK + 2) + 15) & ~size_t(15);
    // epilogue: a thread owns one accumulator row x CW columns; 4 warps (the
    // TMEM lane quarters) per CW-wide column group: 8 warps at every width
    // (16 on 64-slot tiles or on 128-slot ones measured slower)
    static constexpr int CW = (TN == 128) ? 64 : (TN == 64) ? 32 : 16;
    static constexpr int N_EPI = 4 * (TN / CW) * 32;
    // converters: PPT pairs of blocks of a weight row (and on binary16 tiles
    // of a slot) per thread, OP_KB / 2 / PPT threads a row: 8 warps for 8- and
    // 4-block stages, 4 for 2
    static constexpr int PPT = (OP_KB == 8) ? 2 : 1;
    static constexpr int N_CONV = TM * OP_KB / 2 / PPT;
    static constexpr int W_MMA = W_CONV0 + N_CONV / 32, W_EPI0 = W_MMA + 1;
    static constexpr int THREADS = (W_EPI0 * 32) + N_EPI;  // 18, 18 or 14 warps
    static constexpr uint32_t TMEM_COLS = (NACC * TN <= 256) ? 256 : 512;   // a power of two
    // binary16 tiles convert the activations into B operand stages; int8
    // tiles read B straight from the activation ring, whose entries then hold
    // the codes in the MMA's core-matrix layout followed by the scales
    static constexpr size_t SZ_OP_B = I8 ? 0 : (size_t)OP_KB * OPB * TN * 32;
    static constexpr size_t BPF_CODES = (size_t)OP_KB * TN * 32;
    static constexpr size_t BPF_ENTRY = I8 ? ((BPF_CODES + (size_t)TN * OP_KB * 2 + 15) & ~size_t(15))
                                           : (size_t)TN * BPF_SLOT;
    static constexpr int XCH_LD = TN + 1;
    static constexpr size_t OFF_IN_W = 0;
    static constexpr size_t OFF_OP_A = (OFF_IN_W + NIN * SZ_IN_W + 1023) & ~size_t(1023);
    static constexpr size_t OFF_OP_B = OFF_OP_A + NOP * SZ_OP_A;
    static constexpr size_t OFF_DW = OFF_OP_B + NOP * SZ_OP_B;
    static constexpr size_t OFF_DA = OFF_DW + (size_t)NSC * OP_KB * TM * 4;
    static constexpr size_t OFF_XCH = OFF_DA + (size_t)NSC * OP_KB * TN * 4;
    static constexpr size_t OFF_BPF = OFF_XCH + (size_t)TM * XCH_LD * 4;
    static constexpr size_t SMEM_BYTES = OFF_BPF + (size_t)NPF * BPF_ENTRY;
    static constexpr size_t SMEM_ALLOC = SMEM_BYTES + 1024;   // slack to align the map to 1024 B
    static_assert(SMEM_ALLOC <= 226 * 1024, "shared memory map too large");
    static_assert(TMEM_COLS <= 512, "TMEM budget");
};

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

__device__ __forceinline__ void cp_async4(void* dst_smem, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst_smem)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(void* dst_smem, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst_smem)), "l"(src) : "memory");
}
// arrive on bar once this thread's earlier cp.async copies have landed (the
// barrier's count includes the arrival)
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// y[0..3] += v (one vector reduction at L2; y 16-byte aligned)
__device__ __forceinline__ void red_add_v4(float* y, float4 v) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(y), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

// 16 consecutive 32-bit columns of this warp's 32 TMEM lanes (lane = row).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

// 16 consecutive 32-bit columns of this warp's 32 TMEM lanes, all set to v.
__device__ __forceinline__ void tmem_st16_fill(uint32_t taddr, uint32_t v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr),
        "r"(v)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// int8 operands: every accumulator starts at ACC_BIAS and the MMAs add the
// int32 block dot I (|I| <= 8 * 127 * 32 < 2^22) to it.  The int32
// ACC_BIAS + I read as binary32 is exactly 1.5 * 2^23 + I (the significand
// field of ACC_BIAS is 2^22, so adding I never carries into the exponent),
// and one packed subtraction of 1.5 * 2^23 gives I exactly, with no
// int32 -> fp32 conversion.
constexpr uint32_t ACC_BIAS = 0x4B400000u;
constexpr float ACC_BIAS_F = 12582912.0f;   // 1.5 * 2^23

// The 16 block dots of one chunk as fp32 pairs: binary16 operands leave
// exact fp32 integers; int8 operands leave them offset by ACC_BIAS.
template <bool I8>
__device__ __forceinline__ float2 block_dots2(uint32_t a, uint32_t b) {
    const float2 v = make_float2(__uint_as_float(a), __uint_as_float(b));
    if constexpr (I8) return __fadd2_rn(v, make_float2(-ACC_BIAS_F, -ACC_BIAS_F));
    return v;
}

// acc[slot pair h8 + j] += I (16 columns of one block) * dW * dA[slot].
template <bool I8, int NA>
__device__ __forceinline__ void rescale_acc16(float2 (&acc)[NA], int h8, const uint32_t (&r)[16], float dwv,
                                              const float* da) {
    const float4* da4 = reinterpret_cast<const float4*>(da);
    const float2 dw2 = make_float2(dwv, dwv);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float4 d = da4[j];
        const float2 s0 = __fmul2_rn(dw2, make_float2(d.x, d.y));
        const float2 s1 = __fmul2_rn(dw2, make_float2(d.z, d.w));
        acc[h8 + 2 * j] = __ffma2_rn(block_dots2<I8>(r[4 * j], r[4 * j + 1]), s0, acc[h8 + 2 * j]);
        acc[h8 + 2 * j + 1] = __ffma2_rn(block_dots2<I8>(r[4 * j + 2], r[4 * j + 3]), s1, acc[h8 + 2 * j + 1]);
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

// Byte offset of the 16-byte core-matrix piece `core` (0/1) of row r in K-step
// `ks` of block `kb` of an operand stage of `rows` rows.  A K-step is one
// 32-byte slab per row (int8: the whole block, K = 32; binary16: half of it,
// K = 16, so OPB = 2 K-steps a block); inside it, 8-row groups are 256 B
// apart and the two pieces of a row 128 B apart (the descriptor's SBO and LBO).
template <int OPB>
__device__ __forceinline__ uint32_t op_off(int rows, int kb, int ks, int r, int core) {
    return (uint32_t)((kb * OPB + ks) * rows * 32 + (r >> 3) * 256 + core * 128 + (r & 7) * 16);
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

// Four nibbles n (one per byte, high bits clear) -> the bytes n - 8 as int8:
// n + 0x78 stays below 0x88 (no carry between bytes) and flipping its top bit
// subtracts 0x80.
__device__ __forceinline__ uint32_t nib_to_s8(uint32_t w) { return (w + 0x78787878u) ^ 0x80808080u; }

// One Q4_0 block (qs as four words) -> weight row r of block kb in the A
// operand: the low nibbles are weights 0..15 of the block, the high nibbles
// 16..31, each minus 8.
template <bool I8>
__device__ __forceinline__ void store_weights(uint8_t* oa, int kb, int r, const uint32_t (&qs)[4]) {
    if constexpr (I8) {
        *reinterpret_cast<uint4*>(oa + op_off<1>(TM, kb, 0, r, 0)) =
            make_uint4(nib_to_s8(qs[0] & 0x0f0f0f0fu), nib_to_s8(qs[1] & 0x0f0f0f0fu),
                       nib_to_s8(qs[2] & 0x0f0f0f0fu), nib_to_s8(qs[3] & 0x0f0f0f0fu));
        *reinterpret_cast<uint4*>(oa + op_off<1>(TM, kb, 0, r, 1)) =
            make_uint4(nib_to_s8((qs[0] >> 4) & 0x0f0f0f0fu), nib_to_s8((qs[1] >> 4) & 0x0f0f0f0fu),
                       nib_to_s8((qs[2] >> 4) & 0x0f0f0f0fu), nib_to_s8((qs[3] >> 4) & 0x0f0f0f0fu));
    } else {
        uint32_t v[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint2 lo = bytes_to_f16(qs[i] & 0x0f0f0f0fu, BIAS_NIB);
            const uint2 hi = bytes_to_f16((qs[i] >> 4) & 0x0f0f0f0fu, BIAS_NIB);
            v[2 * i] = lo.x;
            v[2 * i + 1] = lo.y;
            v[8 + 2 * i] = hi.x;
            v[8 + 2 * i + 1] = hi.y;
        }
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
#pragma unroll
            for (int core = 0; core < 2; ++core) {
                const int c0 = 8 * ks + 4 * core;
                *reinterpret_cast<uint4*>(oa + op_off<2>(TM, kb, ks, r, core)) =
                    make_uint4(v[c0], v[c0 + 1], v[c0 + 2], v[c0 + 3]);
            }
    }
}

// 16 activation codes (one 16-byte load: half `h` of block kb) -> slot n of
// the B operand: as they are (int8), or as binary16 (one K-step).
template <bool I8>
__device__ __forceinline__ void store_act16(uint8_t* ob, int rows, int kb, int h, int n, uint4 a) {
    if constexpr (I8) {
        *reinterpret_cast<uint4*>(ob + op_off<1>(rows, kb, 0, n, h)) = a;
    } else {
        const uint2 a0 = bytes_to_f16(a.x ^ 0x80808080u, BIAS_ACT);
        const uint2 a1 = bytes_to_f16(a.y ^ 0x80808080u, BIAS_ACT);
        const uint2 a2 = bytes_to_f16(a.z ^ 0x80808080u, BIAS_ACT);
        const uint2 a3 = bytes_to_f16(a.w ^ 0x80808080u, BIAS_ACT);
        *reinterpret_cast<uint4*>(ob + op_off<2>(rows, kb, h, n, 0)) = make_uint4(a0.x, a0.y, a1.x, a1.y);
        *reinterpret_cast<uint4*>(ob + op_off<2>(rows, kb, h, n, 1)) = make_uint4(a2.x, a2.y, a3.x, a3.y);
    }
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
template <int TN>
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

// w[i] = win[i + OFS] (zero past the window)
template <int OFS, int N, int M>
__device__ __forceinline__ void take_words(uint32_t (&w)[N], const uint32_t (&win)[M]) {
#pragma unroll
    for (int i = 0; i < N; ++i) w[i] = (i + OFS < M) ? win[i + OFS] : 0u;
}

// ---------------------------------------------------------------------------
// The epilogue's per-block rescale on its own (a measurement aid): one CTA per
// SM of RC_WARPS warps, each owning TMEM lane quarter warp % 4 and 128 of the
// 512 columns, runs `iters` operand stages of the epilogue's inner loop over
// them -- 16-column TMEM loads software-pipelined against rescale_acc16, the
// block scales read from shared memory, and for int8 operands the reset of
// every chunk to ACC_BIAS and the wait for it -- with nothing handed between
// roles, so its rate bounds the rescale of the projection kernels.  A stage
// is 4 blocks x 32 columns per thread, as in the 32- and 64-slot tiles.
constexpr int RC_WARPS = 16;

template <bool I8>
__global__ void __launch_bounds__(RC_WARPS * 32, 1) rescale_ceiling_kernel(int iters, float* sink) {
    __shared__ uint32_t tmem_base_s;
    __shared__ __align__(16) float da_s[4 * 4 * 32];     // 4 scale-ring entries x 4 blocks x 32 slots
    __shared__ float dw_s[4 * 4 * 128];                  // 4 entries x 4 blocks x 128 rows
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < 4 * 4 * 32; i += RC_WARPS * 32) da_s[i] = 1.0f + (float)(i & 63) * (1.0f / 1024.0f);
    for (int i = tid; i < 4 * 4 * 128; i += RC_WARPS * 32) dw_s[i] = 1.0f / 4096.0f + (float)(i & 31) * 1e-6f;
    if (warp == 0) {
        tmem_alloc(&tmem_base_s, 512);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const int q = warp & 3, cg = warp >> 2;            // lane quarter, group of 128 columns
    const int row = 32 * q + lane;
    const uint32_t taddr = tmem_base_s + ((uint32_t)(32 * q) << 16) + 128u * cg;
    // small exact integers (1 + the column) as the accumulators' contents
#pragma unroll
    for (int c = 0; c < 8; ++c) tmem_st16_fill(taddr + 16 * c, I8 ? ACC_BIAS + 1u + c : __float_as_uint(1.0f + c));
    tmem_wait_st();
    tc_fence_before_sync();
    __syncwarp();
    tc_fence_after_sync();
    float2 acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = make_float2(0.0f, 0.0f);
    for (int it = 0; it < iters; ++it) {
        const int sc = it & 3;
        uint32_t rA[16], rB[16];
        tmem_ld16(taddr, rA);
        tmem_wait_ld();
        if constexpr (I8) tmem_st16_fill(taddr, ACC_BIAS + 1u);
#pragma unroll
        for (int qc = 0; qc < 8; ++qc) {           // 4 blocks x 2 chunks of 16 columns
            const int kb = qc >> 1, hf = qc & 1;
            if (qc + 1 < 8) tmem_ld16(taddr + 16 * (qc + 1), (qc & 1) ? rA : rB);
            const uint32_t(&r)[16] = (qc & 1) ? rB : rA;
            rescale_acc16<I8>(acc, 8 * hf, r, dw_s[(sc * 4 + kb) * 128 + row], da_s + (sc * 4 + kb) * 32 + 16 * hf);
            if (qc + 1 < 8) {
                tmem_wait_ld();
                if constexpr (I8) tmem_st16_fill(taddr + 16 * (qc + 1), ACC_BIAS + 1u + (qc + 1));
            }
            if (qc + 2 == 8) {
                if constexpr (I8) tmem_wait_st();
                tc_fence_before_sync();
                __syncwarp();
                tc_fence_after_sync();
            }
        }
    }
    float t = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) t += acc[j].x + acc[j].y;
    if (blockIdx.x == 0 && tid == 0) *sink = t;
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem_base_s, 512);
}

}  // namespace

// CAP: also write the per-block integer sums (the MMA accumulators before the
// rescale) of one row block of one group to p.cap_out (test instantiation).
template <int MODE, int TN, bool CAP>
__global__ void __launch_bounds__(TcCfg<TN>::THREADS, 1)
    tc_grouped_kernel(TcParams p, const __grid_constant__ TcMaps maps) {
    using C = TcCfg<TN>;
    constexpr int N_EPI = C::N_EPI, THREADS = C::THREADS, XCH_LD = C::XCH_LD, CW = C::CW, NCH = CW / 16;
    constexpr int N_CONV = C::N_CONV, W_MMA = C::W_MMA, W_EPI0 = C::W_EPI0;
    constexpr int OP_KB = C::OP_KB;
    constexpr size_t SZ_OP_A = C::SZ_OP_A, BPF_SLOT = C::BPF_SLOT;
    constexpr bool I8 = C::I8;
    constexpr uint32_t TMEM_COLS = C::TMEM_COLS;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    constexpr int NIN = C::NIN, NOP = C::NOP, NTS = C::NTS, NSC = C::NSC, NPF = C::NPF;
    __shared__ __align__(8) uint64_t in_full[NIN], in_empty[NIN], op_full[NOP], op_empty[NOP], tm_full[NTS],
        tm_empty[NTS], sc_full[NSC], sc_empty[NSC], epi_bar, b_full[NPF], b_empty[NPF];
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    __shared__ int tile_off_s[258], off_s[258];
    __shared__ int tok_s[TN];
    __shared__ float wt_s[TN];

    uint8_t* in_w = smem + C::OFF_IN_W;
    uint8_t* op_a = smem + C::OFF_OP_A;
    uint8_t* op_b = smem + C::OFF_OP_B;
    float* dw_ring = reinterpret_cast<float*>(smem + C::OFF_DW);
    float* da_ring = reinterpret_cast<float*>(smem + C::OFF_DA);
    float* xch = reinterpret_cast<float*>(smem + C::OFF_XCH);
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
            mbar_init(&in_full[i], 1);
            mbar_init(&in_empty[i], N_CONV);
        }
        for (int i = 0; i < NOP; ++i) {
            mbar_init(&op_full[i], N_CONV);
            mbar_init(&op_empty[i], 1);
        }
        for (int i = 0; i < NTS; ++i) {  // one set of accumulators each
            mbar_init(&tm_full[i], 1);
            mbar_init(&tm_empty[i], N_EPI / 32);
        }
        for (int i = 0; i < NSC; ++i) {
            mbar_init(&sc_full[i], N_CONV / 32);
            mbar_init(&sc_empty[i], N_EPI / 32);
        }
        for (int i = 0; i < NPF; ++i) {
            mbar_init(&b_full[i], 32);              // the producer's 32 lanes, after their copies land
            // binary16: the converter warps, after reading the entry; int8:
            // the MMAs' commit and the converter warp that takes the scales
            mbar_init(&b_empty[i], I8 ? 1 + TN / 32 : N_CONV / 32);
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
        // weights: TMA copies of each input stage; activations: for each of
        // its operand stages, the codes and scales of every slot of the tile
        // (lane l: slots l, l + 32, ..) into a ring entry by cp.async, whose
        // landing the lane reports on the entry's barrier
        uint8_t* bpf = smem + C::OFF_BPF;
        constexpr int SPL = (TN + 31) / 32;          // slots per lane
        uint32_t i_in = 0, i_b = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            const Tile T = tile_of<TN>(item, n_rb, tile_off_s, off_s, ngroups);
            const int8_t* arow[SPL];
            const uint16_t* ascale[SPL];
#pragma unroll
            for (int q = 0; q < SPL; ++q) {
                arow[q] = nullptr;
                ascale[q] = nullptr;
                const int n = lane + 32 * q;
                if (n < TN && n < T.nslots) {
                    const int sl = T.slot0 + n;
                    int tok;
                    float w;
                    slot_info(p, T.g, sl, tok, w);
                    if (MODE == GATEUP) {
                        arow[q] = p.qa + (size_t)tok * H;
                        ascale[q] = p.da + (size_t)tok * (H / QK);
                    } else {
                        arow[q] = p.hq + (size_t)sl * F;
                        ascale[q] = p.dh + (size_t)sl * nbF;
                    }
                }
            }
            // weight rows of this item: one box of 64 gate + one of 64 up rows, or 128 down rows
            const bool shared_g = T.g >= E;
            const CUtensorMap* map0 = &maps.m[shared_g ? 2 : 0];
            const CUtensorMap* map1 = &maps.m[shared_g ? 3 : 1];
            const int wy = (shared_g ? 0 : T.g * ((MODE == GATEUP) ? F : H)) + T.rb * ((MODE == GATEUP) ? 64 : TM);
            for (int c = 0; c < nbK / IN_KB; ++c, ++i_in) {
                const int s = i_in % NIN;
                if (!wait_phase(&in_empty[s], ((i_in / NIN) & 1) ^ 1, abort)) { ok = false; break; }
                uint8_t* dw = in_w + (size_t)s * SZ_IN_W;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&in_full[s], (uint32_t)(TM * IN_ROW));
                    tma_load_2d(dw, map0, c * IN_ROW, wy, &in_full[s]);
                    if (MODE == GATEUP) tma_load_2d(dw + 64 * IN_ROW, map1, c * IN_ROW, wy, &in_full[s]);
                }
                __syncwarp();
                for (int sb = 0; sb < IN_KB / OP_KB; ++sb, ++i_b) {
                    const int r = i_b % NPF;
                    if (!wait_phase(&b_empty[r], ((i_b / NPF) & 1) ^ 1, abort)) { ok = false; break; }
                    const int cb = c * (IN_KB / OP_KB) + sb;   // operand stage within the item
#pragma unroll
                    for (int q = 0; q < SPL; ++q) {
                        if (!arow[q]) continue;
                        const int n = lane + 32 * q;
                        const int8_t* src = arow[q] + (size_t)cb * OP_KB * QK;
                        if constexpr (I8) {
                            // codes into the B operand layout (block kb: a K = 32
                            // slab of TN rows), scales after them
                            uint8_t* ent = bpf + (size_t)r * C::BPF_ENTRY;
#pragma unroll
                            for (int kb = 0; kb < OP_KB; ++kb)
#pragma unroll
                                for (int h = 0; h < 2; ++h)
                                    cp_async16(ent + op_off<1>(TN, kb, 0, n, h), src + 32 * kb + 16 * h);
                            if constexpr (OP_KB == 8)
                                cp_async16(ent + C::BPF_CODES + 16 * n, ascale[q] + cb * OP_KB);
                            else
                                cp_async8(ent + C::BPF_CODES + 8 * n, ascale[q] + cb * OP_KB);
                        } else {
                            uint8_t* dst = bpf + (size_t)r * C::BPF_ENTRY + (size_t)n * BPF_SLOT;
#pragma unroll
                            for (int i = 0; i < 2 * OP_KB; ++i) cp_async16(dst + 16 * i, src + 16 * i);
                            if (OP_KB == 4) cp_async8(dst + OP_KB * QK, ascale[q] + cb * OP_KB);
                            else cp_async4(dst + OP_KB * QK, ascale[q] + cb * OP_KB);
                        }
                    }
                    cp_async_arrive_noinc(&b_full[r]);
                }
                if (!ok) break;
            }
        }
        // let the copies in flight land before the CTA can exit
        cp_async_wait_all();
        if (i_in > 0) mbar_wait_bounded(&in_full[(i_in - 1) % NIN], ((i_in - 1) / NIN) & 1, LIMIT);
    } else if (warp >= W_CONV0 && warp < W_MMA) {
        // ------------------------------------------------------------ converters
        // thread ct converts PPT pairs of blocks (kb0 + 2 G j, kb0 + 2 G j + 1;
        // G = N_CONV / 128 threads a row) of weight row ct mod 128 and, on
        // binary16 tiles, (row < TN) of the activations of that slot, which
        // the producer has copied into the ring
        constexpr int PPT = C::PPT, G = N_CONV / TM;
        const int ct = tid - W_CONV0 * 32;
        const int row = ct % TM, kb0 = 2 * (ct / TM);
        const uint8_t* bpf = smem + C::OFF_BPF;
        const int nst = nbK / OP_KB;                      // operand stages per item
        uint32_t i_op = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            const Tile T = tile_of<TN>(item, n_rb, tile_off_s, off_s, ngroups);
            const bool valid = row < T.nslots;
            for (int c = 0; c < nst && ok; ++c, ++i_op) {
                const uint32_t i_in = i_op / (IN_KB / OP_KB);
                const int s = i_in % NIN, sub = i_op % (IN_KB / OP_KB);
                if (sub == 0 && !wait_phase(&in_full[s], (i_in / NIN) & 1, abort)) { ok = false; break; }
                const int o = i_op % NOP;
                if (!wait_phase(&op_empty[o], ((i_op / NOP) & 1) ^ 1, abort)) { ok = false; break; }
                tc_fence_after_sync();

                // weights: each of this thread's pairs of blocks (36 bytes at a
                // 4-byte boundary), read as 16-byte loads of the window from the
                // 16-byte boundary at or below it: rows are 144 bytes apart, so
                // a quarter-warp's loads fall in distinct banks
                uint8_t* oa = op_a + (size_t)o * SZ_OP_A;
                float dws[2 * PPT];
#pragma unroll
                for (int j = 0; j < PPT; ++j) {
                    const int kp = kb0 + 2 * G * j;               // first block of the pair
                    uint32_t w[9];
                    {
                        constexpr int NW = (4 * 3 + 2 * Q4_BYTES + 15) / 16;   // 3 loads, inside the row
                        const int gb = (sub * OP_KB + kp) * Q4_BYTES;
                        const uint4* wsrc = reinterpret_cast<const uint4*>(in_w + (size_t)s * SZ_IN_W +
                                                                           (size_t)row * IN_ROW + (gb & ~15));
                        uint32_t win[4 * NW];
#pragma unroll
                        for (int i = 0; i < NW; ++i) {
                            const uint4 v = wsrc[i];
                            win[4 * i] = v.x; win[4 * i + 1] = v.y; win[4 * i + 2] = v.z; win[4 * i + 3] = v.w;
                        }
                        switch ((gb & 15) >> 2) {   // the same in every lane of the warp
                            case 0: take_words<0>(w, win); break;
                            case 1: take_words<1>(w, win); break;
                            case 2: take_words<2>(w, win); break;
                            default: take_words<3>(w, win); break;
                        }
                    }
                    // the pair's first block starts at its byte 0 (scale, then
                    // 16 nibble bytes), the second at byte 18
                    uint32_t qs[4];
                    dws[2 * j] = half_bits_to_float(w[0] & 0xffffu);
#pragma unroll
                    for (int i = 0; i < 4; ++i) qs[i] = __funnelshift_r(w[i], w[i + 1], 16);
                    store_weights<I8>(oa, kp, row, qs);
                    dws[2 * j + 1] = half_bits_to_float(w[4] >> 16);
#pragma unroll
                    for (int i = 0; i < 4; ++i) qs[i] = w[5 + i];
                    store_weights<I8>(oa, kp + 1, row, qs);
                }
                // activations.  binary16 tiles: slot `row`'s codes from the ring
                // into the B operand (zeros past the tile's slots).  int8 tiles:
                // the MMA reads the codes in the ring; the first TN / 32
                // converter warps take the scales of slot ct (all OP_KB blocks)
                uint32_t dab = 0;
                uint32_t dsl[OP_KB / 2];                          // int8: the slot's OP_KB scales
#pragma unroll
                for (int i = 0; i < OP_KB / 2; ++i) dsl[i] = 0;
                if constexpr (I8) {
                    if (ct < TN) {   // slot ct: warp-uniform
                        if (!wait_phase(&b_full[i_op % NPF], (i_op / NPF) & 1, abort)) { ok = false; break; }
                        if (valid) {
                            const uint8_t* sp = bpf + (size_t)(i_op % NPF) * C::BPF_ENTRY + C::BPF_CODES + 2 * OP_KB * ct;
                            if constexpr (OP_KB == 8) {
                                const uint4 v = *reinterpret_cast<const uint4*>(sp);
                                dsl[0] = v.x; dsl[1] = v.y; dsl[2] = v.z; dsl[3] = v.w;
                            } else {
                                const uint2 v = *reinterpret_cast<const uint2*>(sp);
                                dsl[0] = v.x; dsl[1] = v.y;
                            }
                        }
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&b_empty[i_op % NPF]);   // with the MMAs' commit: entry free
                    }
                } else {
                    uint8_t* ob = op_b + (size_t)o * C::SZ_OP_B;
                    if (!wait_phase(&b_full[i_op % NPF], (i_op / NPF) & 1, abort)) { ok = false; break; }
                    if constexpr (TN * 2 == TM) {
                        // 64-slot tiles: one block of one slot per thread (slot
                        // row mod 64, block kb0 + row / 64), so every converter
                        // thread carries the same share of the activations
                        const int sl = row % TN, kb = kb0 + row / TN;
                        const uint8_t* src = bpf + (size_t)(i_op % NPF) * C::BPF_ENTRY + (size_t)sl * BPF_SLOT;
                        const bool v = sl < T.nslots;
#pragma unroll
                        for (int h = 0; h < 2; ++h)
                            store_act16<I8>(ob, TN, kb, h, sl,
                                            v ? *reinterpret_cast<const uint4*>(src + 16 * (2 * kb + h))
                                              : make_uint4(0, 0, 0, 0));
                        if (v) dab = *reinterpret_cast<const uint16_t*>(src + OP_KB * QK + 2 * kb);
                    } else if (row < TN) {
                        const uint8_t* src = bpf + (size_t)(i_op % NPF) * C::BPF_ENTRY + (size_t)row * BPF_SLOT;
#pragma unroll
                        for (int kb = kb0; kb < kb0 + 2; ++kb)
#pragma unroll
                            for (int h = 0; h < 2; ++h)
                                store_act16<I8>(ob, TN, kb, h, row,
                                                valid ? *reinterpret_cast<const uint4*>(src + 16 * (2 * kb + h))
                                                      : make_uint4(0, 0, 0, 0));
                        if (valid) dab = *reinterpret_cast<const uint32_t*>(src + OP_KB * QK + 2 * kb0);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&b_empty[i_op % NPF]);   // the ring entry is free again
                }
                fence_proxy_async_smem();
                tc_fence_before_sync();
                mbar_arrive(&op_full[o]);
                if (sub == IN_KB / OP_KB - 1) mbar_arrive(&in_empty[s]);
                // block scales into the ring read by the epilogue
                const int sc = i_op % NSC;
                if (!wait_phase(&sc_empty[sc], ((i_op / NSC) & 1) ^ 1, abort)) { ok = false; break; }
#pragma unroll
                for (int j = 0; j < PPT; ++j)
#pragma unroll
                    for (int i = 0; i < 2; ++i) dw_ring[(sc * OP_KB + kb0 + 2 * G * j + i) * TM + row] = dws[2 * j + i];
                if constexpr (I8) {
                    static_assert(!I8 || OP_KB == 4 || OP_KB == 8, "int8 tiles: 4- or 8-block stages");
                    if (ct < TN) {
#pragma unroll
                        for (int kb = 0; kb < OP_KB; ++kb)
                            da_ring[(sc * OP_KB + kb) * TN + ct] =
                                valid ? half_bits_to_float((kb & 1) ? (dsl[kb >> 1] >> 16) : (dsl[kb >> 1] & 0xffffu))
                                      : 0.0f;
                    }
                } else {
                    static_assert(I8 || PPT == 1, "binary16 tiles: a pair a thread");
                    if constexpr (TN * 2 == TM) {
                        const int sl = row % TN, kb = kb0 + row / TN;
                        da_ring[(sc * OP_KB + kb) * TN + sl] = sl < T.nslots ? half_bits_to_float(dab) : 0.0f;
                    } else {
#pragma unroll
                        for (int i = 0; i < 2; ++i)
                            if (row < TN)
                                da_ring[(sc * OP_KB + kb0 + i) * TN + row] =
                                    valid ? half_bits_to_float(i ? (dab >> 16) : dab) : 0.0f;
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sc_full[sc]);
            }
        }
    } else if (warp == W_MMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = I8 ? idesc_i8(TM, TN) : idesc_f16(TM, TN);
            // descriptors of the first K-step of operand stage 0; a later
            // stage or K-step adds its byte offset / 16 to the start-address
            // field (shared-memory offsets stay below 2^18: no carry out)
            const uint64_t b00 = smem_desc_kmajor(I8 ? smem + C::OFF_BPF : op_b, 128, 256);
            const uint64_t a00 = smem_desc_kmajor(op_a, 128, 256);
            uint32_t i_op = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
                for (int c = 0; c < nbK / OP_KB; ++c, ++i_op) {
                    const int o = i_op % NOP, ts = i_op % NTS;
                    if (!wait_phase(&op_full[o], (i_op / NOP) & 1, abort)) {
                        ok = false;
                        break;
                    }
                    // the set of accumulators of this operand stage, released by
                    // the epilogue (int8 operands: reset to ACC_BIAS); its first
                    // phase is the epilogue's start-up arrival
                    if (!wait_phase(&tm_empty[ts], (i_op / NTS) & 1, abort)) {
                        ok = false;
                        break;
                    }
                    if constexpr (I8) {
                        // the B operand is the ring entry the producer's
                        // cp.async copies filled (generic proxy): order them
                        // before the MMA's reads (async proxy)
                        if (!wait_phase(&b_full[i_op % NPF], (i_op / NPF) & 1, abort)) {
                            ok = false;
                            break;
                        }
                        fence_proxy_async_smem();
                    }
                    tc_fence_after_sync();
                    const uint64_t bd = I8 ? b00 + (uint64_t)(((i_op % NPF) * C::BPF_ENTRY) >> 4)
                                           : b00 + (uint64_t)((o * C::SZ_OP_B) >> 4);
                    const uint64_t ad = a00 + (uint64_t)((o * SZ_OP_A) >> 4);
#pragma unroll
                    for (int kb = 0; kb < OP_KB; ++kb) {
                        const uint32_t d = tmem + (uint32_t)(OP_KB * ts + kb) * TN;
                        constexpr uint64_t KA = (uint64_t)TM * 32 >> 4, KB = (uint64_t)TN * 32 >> 4;  // K-step / 16
                        if constexpr (I8) {
                            mma_i8(d, ad + (uint64_t)kb * KA, bd + (uint64_t)kb * KB, idesc, true);  // onto ACC_BIAS
                        } else {
                            mma_f16_ss(d, ad + (uint64_t)(kb * 2) * KA, bd + (uint64_t)(kb * 2) * KB, idesc, false);
                            mma_f16_ss(d, ad + (uint64_t)(kb * 2 + 1) * KA, bd + (uint64_t)(kb * 2 + 1) * KB, idesc,
                                       true);
                        }
                    }
                    mma_commit(&tm_full[ts]);  // covers the set's MMAs
                    mma_commit(&op_empty[o]);
                    if constexpr (I8) mma_commit(&b_empty[i_op % NPF]);
                }
            }
            // the last commit's arrival must land before the CTA can exit
            if (i_op > 0) mbar_wait_bounded(&op_empty[(i_op - 1) % NOP], ((i_op - 1) / NOP) & 1, LIMIT);
            if (I8 && i_op > 0) mbar_wait_bounded(&b_empty[(i_op - 1) % NPF], ((i_op - 1) / NPF) & 1, LIMIT);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = tid - W_EPI0 * 32;         // 0 .. N_EPI - 1
        const int q = warp & 3;                   // TMEM lane quarter this warp may access
        const int cq = (warp - W_EPI0) >> 2;      // column group: slots CW cq .. CW cq + CW - 1
        const int row = 32 * q + lane;            // weight row (TMEM lane) of this thread
        const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + CW * cq;
        uint32_t i_op = 0, epi_phase = 0;
        bool ok = true;
        // both sets of accumulators start at ACC_BIAS (int8 operands)
        if constexpr (I8) {
#pragma unroll
            for (int a = 0; a < C::NACC; ++a)
#pragma unroll
                for (int hf = 0; hf < NCH; ++hf) tmem_st16_fill(taddr + a * TN + 16 * hf, ACC_BIAS);
            tmem_wait_st();
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) {
            for (int i = 0; i < NTS; ++i) mbar_arrive(&tm_empty[i]);
        }
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            const Tile T = tile_of<TN>(item, n_rb, tile_off_s, off_s, ngroups);
            if (MODE == DOWN && et < TN) {
                // token and weight of each slot, for the combine at the tile's end
                // (the previous tile's readers passed the barrier that ended it)
                int tok = 0;
                float w = 0.0f;
                if (et < T.nslots) slot_info(p, T.g, T.slot0 + et, tok, w);
                tok_s[et] = tok;
                wt_s[et] = w;
            }
            float2 acc[CW / 2];
#pragma unroll
            for (int j = 0; j < CW / 2; ++j) acc[j] = make_float2(0.0f, 0.0f);
            for (int b = 0; b < nbK; b += OP_KB, ++i_op) {
                const uint32_t pr = i_op % NTS, ppar = (i_op / NTS) & 1;
                const uint32_t sc = i_op % NSC, spar = (i_op / NSC) & 1;
                if (!wait_phase(&tm_full[pr], ppar, abort) || !wait_phase(&sc_full[sc], spar, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                // chunks of 16 columns (OP_KB blocks x CW / 16), software pipelined:
                // the TMEM load of chunk qc + 1 is in flight while chunk qc is
                // rescaled; int8 operands: each chunk is reset to ACC_BIAS
                // once it is in registers, and the set is released once every
                // reset landed
                uint32_t rA[16], rB[16];
                tmem_ld16(taddr + (OP_KB * pr) * TN, rA);
                tmem_wait_ld();
                if constexpr (I8) tmem_st16_fill(taddr + (OP_KB * pr) * TN, ACC_BIAS);
#pragma unroll
                for (int qc = 0; qc < NCH * OP_KB; ++qc) {
                    const int kb = qc / NCH, hf = qc % NCH;
                    if (qc + 1 < NCH * OP_KB) {
                        const int kb1 = (qc + 1) / NCH, hf1 = (qc + 1) % NCH;
                        tmem_ld16(taddr + (OP_KB * pr + kb1) * TN + 16 * hf1, (qc & 1) ? rA : rB);
                    }
                    const uint32_t(&r)[16] = (qc & 1) ? rB : rA;
                    if (CAP && T.g == p.cap_group && T.rb == p.cap_rb) {
                        // the int32 block dots as the tensor cores left them
                        const size_t s0 = (size_t)(T.slot0 - off_s[T.g]);
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int n = CW * cq + 16 * hf + j;
                            if (n < T.nslots)
                                p.cap_out[((s0 + n) * TM + row) * nbK + b + kb] =
                                    I8 ? (int)(r[j] - ACC_BIAS) : __float2int_rn(__uint_as_float(r[j]));
                        }
                    }
                    rescale_acc16<I8>(acc, 8 * hf, r, dw_ring[(sc * OP_KB + kb) * TM + row],
                                  da_ring + (sc * OP_KB + kb) * TN + CW * cq + 16 * hf);
                    if (qc + 1 < NCH * OP_KB) {
                        tmem_wait_ld();
                        const int kb1 = (qc + 1) / NCH, hf1 = (qc + 1) % NCH;
                        if constexpr (I8) tmem_st16_fill(taddr + (OP_KB * pr + kb1) * TN + 16 * hf1, ACC_BIAS);
                    }
                    if (qc + 2 == NCH * OP_KB) {
                        // every chunk of the set is loaded and reset: the accumulators are free
                        if constexpr (I8) tmem_wait_st();
                        tc_fence_before_sync();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&tm_empty[pr]);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sc_empty[sc]);
            }
            if (!ok) break;
            // this thread's row x CW slots into the exchange tile
            float* xr = xch + (size_t)row * XCH_LD + CW * cq;
#pragma unroll
            for (int j = 0; j < CW / 2; ++j) {
                xr[2 * j] = acc[j].x;
                xr[2 * j + 1] = acc[j].y;
            }
            if (!epi_sync(&epi_bar, epi_phase++, abort)) break;
            if (MODE == GATEUP) {
                // SwiGLU + Q8_0 of h.  A unit is one 32-row block of h (gate rows
                // 32 fb .. 32 fb + 31) of one slot n; two lanes share a unit, 16
                // rows each, so every value is independent of the others and a
                // single shuffle gives the block's absolute maximum.  Both
                // divisions of the Q8_0 rule stay IEEE (div.rn).
#pragma unroll 1
                for (int u = et >> 1; u < 2 * TN; u += N_EPI / 2) {   // 2 TN units
                const int n = u % TN, fb = u / TN, half = lane & 1;
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
                }
            } else {
                // y[token][h0 + 4 i .. + 3] += w * o: one vector reduction per
                // (slot, 4 consecutive rows of H)
                const int h0 = T.rb * TM;
#pragma unroll
                for (int i = 0; i < TM * TN / 4 / N_EPI; ++i) {
                    const int u = et + N_EPI * i;
                    const int n = u % TN, rq = u / TN;
                    if (n < T.nslots) {
                        const float w = wt_s[n];
                        const float* xc = xch + (size_t)(4 * rq) * XCH_LD + n;
                        red_add_v4(p.y + (size_t)tok_s[n] * H + h0 + 4 * rq,
                                   make_float4(w * xc[0], w * xc[XCH_LD], w * xc[2 * XCH_LD], w * xc[3 * XCH_LD]));
                    }
                }
            }
            if (!epi_sync(&epi_bar, epi_phase++, abort)) break;  // xch is free for the next tile
        }
        if constexpr (I8) tmem_wait_st();   // no reset may still be in flight when TMEM is freed
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

static int64_t tc_max_tiles(const LayerView& L, int64_t T, int TN) {
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

template <int MODE, int TN, bool CAP>
static cudaError_t launch_tc_inst(const LayerView& L, int64_t T, const TcParams& p, const TcMaps& maps,
                                  const DeviceInfo& dev, cudaStream_t s) {
    using C = TcCfg<TN>;
    int per_sm = 0;
    cudaError_t e = kernel_occupancy(reinterpret_cast<const void*>(tc_grouped_kernel<MODE, TN, CAP>), C::THREADS,
                                     C::SMEM_ALLOC, &per_sm);
    if (e != cudaSuccess) return e;
    const int n_rb = (MODE == GATEUP) ? L.F / 64 : L.H / TM;
    const int64_t items = tc_max_tiles(L, T, TN) * n_rb;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(items, dev.sm_count));
    tc_grouped_kernel<MODE, TN, CAP><<<(unsigned)grid, C::THREADS, C::SMEM_ALLOC, s>>>(p, maps);
    return cudaGetLastError();
}

template <int MODE>
static cudaError_t launch_tc(const LayerView& L, int64_t T, const Workspace& ws, float* h_dbg, float* y,
                             const DeviceInfo& dev, int tile, const BlockDotCapture* cap, cudaStream_t s) {
    if (tile != 32 && tile != 64 && tile != 128) return cudaErrorInvalidValue;
    const bool capture = cap && cap->down == (MODE == DOWN ? 1 : 0);
    TcMaps maps;
    cudaError_t e = make_maps<MODE>(L, &maps);
    if (e != cudaSuccess) return e;
    TcParams p = make_tc_params(L, T, ws, h_dbg, y);
    if (capture) {
        p.cap_out = cap->out;
        p.cap_group = cap->group;
        p.cap_rb = cap->rb;
        return tile == 128 ? launch_tc_inst<MODE, 128, true>(L, T, p, maps, dev, s)
               : tile == 64 ? launch_tc_inst<MODE, 64, true>(L, T, p, maps, dev, s)
                            : launch_tc_inst<MODE, 32, true>(L, T, p, maps, dev, s);
    }
    return tile == 128 ? launch_tc_inst<MODE, 128, false>(L, T, p, maps, dev, s)
           : tile == 64 ? launch_tc_inst<MODE, 64, false>(L, T, p, maps, dev, s)
                        : launch_tc_inst<MODE, 32, false>(L, T, p, maps, dev, s);
}

int tc_tile_tokens(const LayerView& L, int64_t T, int force) {
    if (force == 32 || force == 64 || force == 128) return force;
    // routed slots per expert on average, against the measured crossovers of
    // the three widths (one 2048/512 layer, 128 experts top-8): 32 slots still
    // lead at 32 per expert (T = 512: 351 against 372 us) and 64 at 59 (a
    // 947-token prompt: 0.475 against 0.521 ms), so 64 from 44, between them;
    // 128 from 96 (a 16384-token batch's 1024)
    const int64_t per_expert = T * L.k / L.E;
    return per_expert >= 96 ? 128 : per_expert >= 44 ? 64 : 32;
}

cudaError_t launch_gateup_tc(const LayerView& L, int64_t T, const Workspace& ws, float* h_dbg, const DeviceInfo& dev,
                             int tile, const BlockDotCapture* cap, cudaStream_t s) {
    return launch_tc<GATEUP>(L, T, ws, h_dbg, nullptr, dev, tile, cap, s);
}

cudaError_t launch_down_tc(const LayerView& L, int64_t T, const Workspace& ws, float* y, const DeviceInfo& dev,
                           int tile, const BlockDotCapture* cap, cudaStream_t s) {
    return launch_tc<DOWN>(L, T, ws, nullptr, y, dev, tile, cap, s);
}

cudaError_t launch_rescale_ceiling(bool int8_operands, int iters, float* sink, const DeviceInfo& dev,
                                   int64_t* elements, cudaStream_t s) {
    const dim3 grid((unsigned)dev.sm_count), block(RC_WARPS * 32);
    if (int8_operands)
        rescale_ceiling_kernel<true><<<grid, block, 0, s>>>(iters, sink);
    else
        rescale_ceiling_kernel<false><<<grid, block, 0, s>>>(iters, sink);
    *elements = (int64_t)dev.sm_count * RC_WARPS * 32 * 128 * (int64_t)iters;
    return cudaGetLastError();
}

}  // namespace moeq4
