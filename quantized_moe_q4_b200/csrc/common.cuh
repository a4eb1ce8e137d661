// common.cuh -- device building blocks shared by the kernels of the 4-bit MoE
// expert FFN (W4A8: Q4_0 weights, Q8_0 activations).
//
// Method: "A 35B Hybrid-Attention Mixture-of-Experts Model on a 6GB 2011 GPU:
// Hand-Written 4-bit CUDA Inference for Fermi", Dutch technical summary,
// Methodologie 1 (W4A8 integer multiply-adds; grouped 4-bit GEMM) and
// Methodologie 2 (group-wise symmetric Q4_0-family weights, 8-bit activations).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moeq4 {

constexpr int QK = 32;          // values per Q4_0 / Q8_0 block
constexpr int Q4_BYTES = 18;    // binary16 scale + 16 nibble bytes

// Workspace layout (indices match MOE_Q4_WS_* of the public header).
enum WsIndex {
    WS_STATUS = 0, WS_LOGITS, WS_TOPK_IDX, WS_TOPK_W, WS_QA, WS_DA, WS_CNT, WS_OFF, WS_TILE_OFF,
    WS_CHUNK_CNT, WS_CHUNK_BASE, WS_SORTED, WS_POS, WS_HQ, WS_DH, WS_TOTAL, WS_COUNT
};

// Token-to-expert permutation chunk: pairs handled by one CTA of the
// histogram and scatter kernels.
constexpr int PERM_CHUNK = 1024;

// Tokens per work tile of the grouped dp4a kernels.
constexpr int DP4A_TT = 8;
// Rows per work item: gate/up items cover one Q8_0 block of the SwiGLU
// output (32 rows of F); down items cover 64 rows of H.
constexpr int GU_ROWS = 32;
constexpr int DN_ROWS = 64;

// Status word bits (the public header's MOE_Q4_STATUS_*).
constexpr uint32_t STATUS_SCALE_OVERFLOW = 0x1u;
constexpr uint32_t STATUS_SPIN_TIMEOUT = 0x2u;
constexpr uint32_t STATUS_NONFINITE_LOGIT = 0x4u;
constexpr uint32_t STATUS_BAD_EXPERT_INDEX = 0x8u;

// ---------------------------------------------------------------------------
// Scalar rules
// ---------------------------------------------------------------------------

// Round half away from zero of a binary32 value.  v - trunc(v) is exact in
// binary32, so the comparison with 0.5 decides ties correctly (adding 0.5 and
// flooring would not: 0.49999997 + 0.5 rounds up to 1 in binary32).
__device__ __forceinline__ int round_half_away(float v) {
    float t = truncf(v);
    int q = (int)t;
    if (fabsf(v - t) >= 0.5f) q += (v < 0.0f) ? -1 : 1;
    return q;
}

// Q8_0 of one 32-value block held one value per lane of a full warp.
// Returns this lane's code; `dbits` receives the binary16 scale bits and
// `overflow` whether that scale overflowed to infinity.  Both divisions are
// IEEE binary32 (div.rn), never a reciprocal multiply.
__device__ __forceinline__ int q8_0_lane(float x, uint16_t& dbits, bool& overflow) {
    float a = fabsf(x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    const float d = __fdiv_rn(a, 127.0f);
    int q = 0;
    if (d != 0.0f) {
        q = round_half_away(__fdiv_rn(x, d));
        q = max(-127, min(127, q));
    }
    dbits = __half_as_ushort(__float2half_rn(d));
    overflow = (dbits & 0x7fffu) == 0x7c00u;
    return q;
}

__device__ __forceinline__ float half_bits_to_float(uint32_t bits) {
    return __half2float(__ushort_as_half((unsigned short)(bits & 0xffffu)));
}

// ---------------------------------------------------------------------------
// W4A8 block dot product
// ---------------------------------------------------------------------------

// d = c + sum_i a.u8[i] * b.s8[i]
__device__ __forceinline__ int dp4a_u8s8(uint32_t a, int b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Exact sum_i (nibble_i - 8) * q_i of one Q4_0 block (nibble bytes qs as four
// little-endian words) against 32 int8 activations (eight words).  The low
// nibbles (weights 0..15) go through dp4a as they are; the high nibbles
// (weights 16..31) are masked in place, so each byte holds 16 x the nibble,
// and their chain is divided by 16 once at the end (exact: every term is a
// multiple of 16, and the sum stays below 2^20).  The -8 offset is applied
// once through the activations' block sum qsum.
__device__ __forceinline__ int q4_q8_dot(const uint32_t qs[4], const int qa[8], int qsum) {
    int lo = 0, hi = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        lo = dp4a_u8s8(qs[j] & 0x0f0f0f0fu, qa[j], lo);       // weights 4j..4j+3
        hi = dp4a_u8s8(qs[j] & 0xf0f0f0f0u, qa[4 + j], hi);   // 16 x weights 16+4j..
    }
    return lo + (hi >> 4) - 8 * qsum;
}

// Sum of the 32 int8 values held as eight words.
__device__ __forceinline__ int q8_block_sum(const int qa[8]) {
    int s = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) s = __dp4a(qa[j], 0x01010101, s);
    return s;
}

// Load one 18-byte Q4_0 block whose first byte is at `p` (2-byte aligned) as
// five aligned 32-bit words, then realign: scale bits and qs[16].
__device__ __forceinline__ void load_q4_block(const uint8_t* p, uint32_t qs[4], uint32_t& dbits) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    const uint32_t* w = reinterpret_cast<const uint32_t*>(a & ~uintptr_t(3));
    const uint32_t sh = (uint32_t)(a & 2u) * 8u;  // 0 or 16
    uint32_t w0 = __ldg(w + 0), w1 = __ldg(w + 1), w2 = __ldg(w + 2), w3 = __ldg(w + 3), w4 = __ldg(w + 4);
    dbits = __funnelshift_r(w0, w1, sh) & 0xffffu;
    qs[0] = __funnelshift_rc(w0, w1, 16u + sh);
    qs[1] = __funnelshift_rc(w1, w2, 16u + sh);
    qs[2] = __funnelshift_rc(w2, w3, 16u + sh);
    qs[3] = __funnelshift_rc(w3, w4, 16u + sh);
}

// Same from shared memory (no read-only cache path).
__device__ __forceinline__ void load_q4_block_smem(const uint8_t* p, uint32_t qs[4], uint32_t& dbits) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    const uint32_t* w = reinterpret_cast<const uint32_t*>(a & ~uintptr_t(3));
    const uint32_t sh = (uint32_t)(a & 2u) * 8u;
    uint32_t w0 = w[0], w1 = w[1], w2 = w[2], w3 = w[3], w4 = w[4];
    dbits = __funnelshift_r(w0, w1, sh) & 0xffffu;
    qs[0] = __funnelshift_rc(w0, w1, 16u + sh);
    qs[1] = __funnelshift_rc(w1, w2, 16u + sh);
    qs[2] = __funnelshift_rc(w2, w3, 16u + sh);
    qs[3] = __funnelshift_rc(w3, w4, 16u + sh);
}

// silu(g) * u in binary32 (expf, IEEE division).
__device__ __forceinline__ float swiglu(float g, float u) {
    return __fdiv_rn(g, 1.0f + expf(-g)) * u;
}

}  // namespace moeq4
