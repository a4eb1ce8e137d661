// k_decode.cu -- fused single-token (T=1) decode path of the MoE expert FFN.
//
// The decode step of "A 35B Hybrid-Attention Mixture-of-Experts Model on a
// 6GB 2011 GPU" (Dutch technical summary, Methodologie 1: a W4A8 integer
// kernel that reads the 4-bit weights of the active experts directly; the
// pages ran it on CPU SIMD because the Fermi card lacked fast integer dot
// products).  On B200 the step is bound by HBM bandwidth over the active
// experts' bytes plus the latency of the routing dependency.  Two kernels,
// chained with programmatic dependent launch (PDL):
//
//   decode_router_kernel: one CTA per expert.  Before waiting on the previous
//     kernel it loads its router row into registers and prefetches x into
//     L2; then the logit (four independent FMA chains); y is zeroed (the FFN
//     kernel accumulates into it).
//   decode_ffn_kernel: a grid of (k+S) x F/32 CTAs (one wave), one per (expert
//     of the token, 32-row block of h).  The shared expert's weights are
//     copied before the wait on the router (they do not depend on the
//     routing).  Warp 0 selects the top-k straight from the logits (one warp
//     max and one warp min per round); the CTA of rank j issues its copies as
//     soon as round j names its expert: the block's 32 gate rows and 32 up
//     rows (bulk copies) and its column of the down matrix (block hb of all H
//     rows, 2D tensor copies of 32 bytes x 256 rows) at once, while the
//     other warps quantise x (Q8_0) themselves.  Gate/up dot products,
//     SwiGLU and the Q8_0 requantisation give the CTA's h block; the down
//     column against that block gives its share of every output row, added
//     into y with vector reductions (red.v4.f32).
//
// No CTA waits for another: a CTA's h block is all its down column needs, so
// nothing is exchanged between CTAs and y collects (k+S) x F/32 partial sums
// per element.  (An earlier design split the down rows over groups of 8 CTAs,
// which exchanged their h blocks through L2 behind a release/acquire counter:
// about 2 us more per token.)  The order of the partial sums added into an
// element of y is not fixed: results agree across runs to binary32 rounding,
// not bit for bit.
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

constexpr uint32_t MBAR_LIMIT = 1u << 20;   // bounded waits: about 0.5 s
constexpr int FFN_THREADS = 512;            // 16 warps
constexpr int FFN_WARPS = FFN_THREADS / 32;
constexpr int DN_BOX_BYTES = 32;            // bytes of each down row per tensor copy (holds the 18-byte block)
constexpr int DN_BOX_ROWS = 256;            // rows per 2D tensor copy of the down column
constexpr int ROUTER_STEPS = 5;             // float4 steps of 128 in a router row: H <= 2560

struct DecodeParams {
    int H, F, E, k, S;
    int nbF;             // h blocks per expert (F / 32) = CTAs per expert
    int clear_status;    // the router kernel zeroes the status word (else it accumulates)
    int force_timeout;   // CTA 0's first gate/up barrier expects 16 bytes that never come
    const float* x;
    const float* w_router;
    const float* bias;
    const uint8_t* w_gate;
    const uint8_t* w_up;
    const uint8_t* sh_gate;
    const uint8_t* sh_up;
    float* logits;
    int32_t* topk_idx;
    float* topk_w;
    int8_t* qa;
    uint16_t* da;
    int32_t* cnt;
    int32_t* off;
    int32_t* sorted;
    int32_t* pos;
    int8_t* hq;
    uint16_t* dh;
    float* h_dbg;
    float* y;
    uint32_t* status;
    unsigned long long* kernel_ns;  // optional: CTA 0's spans, [0] from the wait, [2] from the start; [1] += 1
};

// 2D views of the down matrices for the tensor copies: rows of F/32 blocks of
// 18 bytes; a box is 32 bytes (from a 16-byte boundary, so it holds one whole
// block) x 256 rows, written to shared memory with the 32-byte swizzle.
struct DecodeMaps {
    CUtensorMap down, sh_down;
};

// ---------------------------------------------------------------------------
// Butterfly reductions: V per-lane values summed over groups of W lanes.  At
// each of the first log2(V) steps a lane keeps half of its values and trades
// the other half, so V sums cost (V - 1) + log2(W / V) shuffles instead of
// V * log2(W).  Afterwards lane l of a group holds the total of value
// bf_index<V, W>(l); lanes with bf_owner<V, W>(l) hold distinct totals.
// ---------------------------------------------------------------------------
template <int V, int W>
__device__ __forceinline__ float butterfly(float (&v)[V]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int half = V / 2, o = W / 2; half >= 1; half >>= 1, o >>= 1) {
        const bool hi = lane & o;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = hi ? v[i] : v[i + half];
            const float keep = hi ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    float s = v[0];
#pragma unroll
    for (int o = W / (2 * V); o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}

template <int V, int W>
__device__ __forceinline__ int bf_index(int lane) {
    int idx = 0;
#pragma unroll
    for (int half = V / 2, o = W / 2; half >= 1; half >>= 1, o >>= 1)
        if (lane & o) idx += half;
    return idx;
}

template <int V, int W>
__device__ __forceinline__ bool bf_owner(int lane) {
    return (lane & (W / V - 1)) == 0;
}

// acc[r] += W4A8 terms of a pair of blocks (36 bytes from a 4-byte boundary:
// the pair's first byte is at 36 p) in NR rows (stride row_bytes), against
// the pair's two Q8_0 blocks in registers.  Nine 32-bit loads a row; lanes
// taking consecutive pairs hit banks 9 l + i, all distinct.
template <int NR>
__device__ __forceinline__ void pair_rows(const uint8_t* rows, size_t row_bytes, const int (&qa0)[8],
                                          const int (&qa1)[8], int qs0, int qs1, float da0, float da1,
                                          float (&acc)[NR]) {
#pragma unroll
    for (int r = 0; r < NR; ++r) {
        const uint32_t* w = reinterpret_cast<const uint32_t*>(rows + (size_t)r * row_bytes);
        uint32_t v[9];
#pragma unroll
        for (int i = 0; i < 9; ++i) v[i] = w[i];
        // block 0: scale in bytes 0-1, nibbles in 2-17; block 1: scale in 18-19, nibbles in 20-35
        uint32_t q0[4], q1[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            q0[i] = __funnelshift_r(v[i], v[i + 1], 16);
            q1[i] = v[5 + i];
        }
        acc[r] = fmaf((float)q4_q8_dot(q0, qa0, qs0), half_bits_to_float(v[0] & 0xffffu) * da0, acc[r]);
        acc[r] = fmaf((float)q4_q8_dot(q1, qa1, qs1), half_bits_to_float(v[4] >> 16) * da1, acc[r]);
    }
}

// Q8_0 codes of x in shared memory: the codes of block pair p (64 bytes) at
// byte 80 p, so that 16-byte loads by lanes taking consecutive pairs fall in
// distinct banks.
__host__ __device__ constexpr int qa_pair_off(int p) { return 80 * p; }

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// y[0..3] += v (one vector reduction at L2; y 16-byte aligned)
__device__ __forceinline__ void red_add_v4(float* y, float4 v) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(y), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

}  // namespace

// ---------------------------------------------------------------------------
// K1: router logits (one CTA per expert), y zeroed.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) decode_router_kernel(DecodeParams p) {
    __shared__ float red[4];
    const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = p.H;
    // the router row (a weight: read before the wait) into registers, float4
    // steps tid, tid + 128, .. (at most ROUTER_STEPS of them)
    const float4* w4 = reinterpret_cast<const float4*>(p.w_router + (size_t)e * H);
    float4 w[ROUTER_STEPS];
#pragma unroll
    for (int i = 0; i < ROUTER_STEPS; ++i)
        w[i] = (tid + 128 * i < H / 4) ? __ldg(w4 + tid + 128 * i) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    // x into L2 ahead of the wait: a prefetch returns no data, and L2 is where
    // the previous kernel's stores land, so the loads after the wait still see
    // them (each CTA fetches its share of the 128-byte lines)
    for (int i = e * 128 + tid; i < H / 32; i += (int)gridDim.x * 128)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(p.x + 32 * i));
    const float bias = p.bias ? __ldg(p.bias + e) : 0.0f;
    pdl_launch_dependents();
    pdl_wait();  // x and the workspace are now the previous kernels' results
    if (e == 0 && tid == 0 && p.clear_status) p.status[0] = 0u;
    for (int i = e * 128 + tid; i < H; i += (int)gridDim.x * 128) p.y[i] = 0.0f;
    const float4* x4 = reinterpret_cast<const float4*>(p.x);
    float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;  // four independent chains
#pragma unroll
    for (int i = 0; i < ROUTER_STEPS; ++i) {
        if (tid + 128 * i < H / 4) {
            const float4 a = __ldcg(x4 + tid + 128 * i), b = w[i];
            a0 = fmaf(a.x, b.x, a0);
            a1 = fmaf(a.y, b.y, a1);
            a2 = fmaf(a.z, b.z, a2);
            a3 = fmaf(a.w, b.w, a3);
        }
    }
    float acc = (a0 + a1) + (a2 + a3);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) red[warp] = acc;
    __syncthreads();
    if (tid == 0) {
        p.logits[e] = (red[0] + red[1]) + (red[2] + red[3]) + bias;
    }
}

// ---------------------------------------------------------------------------
// K2: top-k, Q8_0 of x, gate/up + SwiGLU + requant, down column + combine.
// ---------------------------------------------------------------------------
struct DecodeSmem {
    size_t gu, dn, qa, da, qsum, o, total;  // byte offsets
};

__host__ __device__ inline size_t al128(size_t v) { return (v + 127) & ~size_t(127); }

__host__ __device__ inline DecodeSmem decode_smem_layout(int H) {
    const int nbH = H / QK;
    DecodeSmem L;
    size_t o = 0;
    L.gu = o;   o += al128((size_t)64 * nbH * Q4_BYTES);       // 32 gate + 32 up rows
    o = (o + 1023) & ~size_t(1023);                               // swizzle pattern boundary
    L.dn = o;   o += al128((size_t)H * DN_BOX_BYTES);              // H rows x 32 bytes
    L.qa = o;   o += al128((size_t)qa_pair_off(H / 64));
    L.da = o;   o += al128((size_t)nbH * 4);
    L.qsum = o; o += al128((size_t)nbH * 4);
    L.o = o;    o += al128((size_t)H * 4);
    L.total = o + 1024;  // slack to align the map to 1024 bytes
    return L;
}

// Order key of a logit: unsigned integers in the order of the values, with
// -0 folded into +0 (equal logits compare equal).  Key 0 lies below every
// logit's key (-infinity's is 0x007fffff) and marks an expert that is out of
// range or already chosen.
__device__ __forceinline__ uint32_t logit_key(float l) {
    const uint32_t u = __float_as_uint(l == 0.0f ? 0.0f : l);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_logit(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Top-k of E <= 32 NK logits by one warp (a NaN ranks as -infinity): lane l
// holds the keys of experts l, l + 32, ...; each of the k rounds takes the
// largest key (warp max), the lowest expert index among equal keys (warp
// min) and retires it, so round r names the expert of rank r (descending
// logits, equal logits by the lower index).  on_round(r, e, logit) runs in
// every lane after round r.  Returns the status bits of non-finite logits.
template <int NK, class OnRound>
__device__ __forceinline__ int topk_rounds(const float* __restrict__ logits, int E, int k, int lane,
                                           OnRound&& on_round) {
    uint32_t key[NK];
    unsigned fl = 0;
#pragma unroll
    for (int i = 0; i < NK; ++i) {
        const int e = lane + 32 * i;
        key[i] = 0u;
        if (e < E) {
            const float l = __ldcg(logits + e);
            if (!isfinite(l)) fl |= STATUS_NONFINITE_LOGIT;
            key[i] = logit_key(l != l ? -INFINITY : l);
        }
    }
    for (int r = 0; r < k; ++r) {
        uint32_t lm = key[0];
#pragma unroll
        for (int i = 1; i < NK; ++i) lm = max(lm, key[i]);
        const uint32_t m = __reduce_max_sync(0xffffffffu, lm);
        uint32_t cand = 0xffffffffu;
#pragma unroll
        for (int i = NK - 1; i >= 0; --i)
            if (key[i] == m) cand = (uint32_t)(lane + 32 * i);
        const uint32_t win = __reduce_min_sync(0xffffffffu, cand);
#pragma unroll
        for (int i = 0; i < NK; ++i)
            if ((uint32_t)(lane + 32 * i) == win) key[i] = 0u;
        on_round(r, (int)win, key_logit(m));
    }
    return (int)__reduce_or_sync(0xffffffffu, fl);
}

// The down column of one h block: o[n] = wj * (I_n * (dW_n * dh)) for every
// row n < H, I_n the integer dot of row n's block (at byte 4A + sh/8 of the
// row's 32 copied bytes) with the h codes hv (sum hsum).
template <int A>
__device__ __forceinline__ void down_column(const uint8_t* dn_s, int H, uint32_t sh, const int (&hv)[8], int hsum,
                                            float dh, float wj, float* o_s) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll 4
    for (int n = warp * 32 + lane; n < H; n += FFN_THREADS) {
        const int sw = (n >> 2) & 1;
        const uint4 c0 = *reinterpret_cast<const uint4*>(dn_s + (size_t)n * DN_BOX_BYTES + 16 * sw);
        const uint4 c1 = *reinterpret_cast<const uint4*>(dn_s + (size_t)n * DN_BOX_BYTES + 16 * (sw ^ 1));
        const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        const uint32_t dbits = __funnelshift_r(w[A], w[A + 1], sh) & 0xffffu;
        uint32_t qs[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) qs[i] = __funnelshift_rc(w[A + i], w[A + i + 1], 16u + sh);
        o_s[n] = wj * ((float)q4_q8_dot(qs, hv, hsum) * (half_bits_to_float(dbits) * dh));
    }
}

__global__ void __launch_bounds__(FFN_THREADS, 1) decode_ffn_kernel(DecodeParams p,
                                                                    const __grid_constant__ DecodeMaps maps) {
    extern __shared__ __align__(16) unsigned char dsm_raw[];
    // tensor-copy destinations 1024-byte aligned (the allocation has 1024 bytes of slack)
    unsigned char* dsm = dsm_raw + ((1024u - (smem_u32(dsm_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t bar_gu[4];
    __shared__ __align__(8) uint64_t bar_dn;
    __shared__ int idx_s[16];
    __shared__ float ex_s[16];
    __shared__ float w_s[16];
    __shared__ int slot_s[17];
    __shared__ float gs[32], us[32];
    __shared__ __align__(16) int8_t hq_w[FFN_WARPS * 32];
    __shared__ int flags_s;

    unsigned long long t_entry = 0;
    if (p.kernel_ns && blockIdx.x == 0 && threadIdx.x == 0) t_entry = global_ns();

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = p.H, F = p.F, E = p.E, k = p.k;
    const int nbH = H / QK, nbF = F / QK;
    const int j = blockIdx.x / p.nbF;               // expert of the token: rank j < k, or k = shared
    const int hb = blockIdx.x % p.nbF;              // this CTA's h block
    const bool is_shared = (j == k);
    // this CTA's column of the down matrix: block hb of every row, inside a
    // 32-byte box from the 16-byte boundary at or below it
    const int dn_x0 = (hb * Q4_BYTES) & ~15;
    const int dn_off = hb * Q4_BYTES - dn_x0;       // 0, 2, .., 14
    const size_t row_gu = (size_t)nbH * Q4_BYTES;
    const size_t gu_stride = (size_t)F * row_gu;    // bytes of one expert's gate (or up) matrix
    const DecodeSmem SL = decode_smem_layout(H);
    uint8_t* gu_s = dsm + SL.gu;
    uint8_t* dn_s = dsm + SL.dn;
    int8_t* qa_s = reinterpret_cast<int8_t*>(dsm + SL.qa);
    float* da_s = reinterpret_cast<float*>(dsm + SL.da);
    int* qsum_s = reinterpret_cast<int*>(dsm + SL.qsum);
    float* o_s = reinterpret_cast<float*>(dsm + SL.o);
    bool timed_out = false;

    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bar_gu[i], 1);
        mbar_init(&bar_dn, 1);
        mbar_fence_init();
        flags_s = 0;
    }
    __syncthreads();

    // copies of this CTA's weights, issued by warp 0's lanes at once: lane
    // i < 4 gate/up chunk i = 8 gate rows + the same 8 up rows on bar_gu[i];
    // lanes 4, 5, .. one 256-row box each of the down column on bar_dn
    const uint32_t chunk_bytes = (uint32_t)(8 * row_gu);
    const int n_dn_box = H / DN_BOX_ROWS;
    auto issue_copies = [&](const uint8_t* Wg, const uint8_t* Wu, const CUtensorMap* dmap, int drow0) {
        if (lane < 4) {
            const int ch = lane;
            const uint32_t extra = (p.force_timeout && blockIdx.x == 0 && ch == 0) ? 16u : 0u;
            mbar_arrive_expect_tx(&bar_gu[ch], 2u * chunk_bytes + extra);
            const size_t src = (size_t)(hb * 32 + 8 * ch) * row_gu;
            bulk_g2s(gu_s + (size_t)(8 * ch) * row_gu, Wg + src, chunk_bytes, &bar_gu[ch]);
            bulk_g2s(gu_s + (size_t)(32 + 8 * ch) * row_gu, Wu + src, chunk_bytes, &bar_gu[ch]);
        }
        if (lane == 4) mbar_arrive_expect_tx(&bar_dn, (uint32_t)(H * DN_BOX_BYTES));
        __syncwarp();
        const int bx = lane - 4;
        if (bx >= 0 && bx < n_dn_box)
            tma_load_2d(dn_s + (size_t)bx * DN_BOX_ROWS * DN_BOX_BYTES, dmap, dn_x0, drow0 + bx * DN_BOX_ROWS,
                        &bar_dn);
    };

    // ---- prologue: the shared expert's copies do not depend on the routing;
    // the down matrices' tensor-map descriptors are fetched ahead of their use
    if (tid == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.down)) : "memory");
        if (p.S) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.sh_down)) : "memory");
    }
    if (is_shared && warp == 0) issue_copies(p.sh_gate, p.sh_up, &maps.sh_down, 0);

    pdl_wait();  // logits, Q8_0 of x and the zeroed y are visible
    pdl_launch_dependents();
    unsigned long long t_ready = 0;
    if (p.kernel_ns && blockIdx.x == 0 && threadIdx.x == 0) t_ready = global_ns();

    if (warp == 0) {
        // ---- top-k by warp 0, straight from the logits in L2 (a NaN ranks as
        // -infinity).  The CTA of routed rank j issues its copies as soon as
        // round j has named its expert; lane r < k keeps round r's expert.
        int e_r = 0;
        float l_r = 0.0f, l_0 = 0.0f;
        auto on_round = [&](int rr, int e, float l) {
            if (rr == 0) l_0 = l;
            if (lane == rr) {
                e_r = e;
                l_r = l;
            }
            if (!is_shared && rr == j) {
                const size_t eo = (size_t)e * gu_stride;
                issue_copies(p.w_gate + eo, p.w_up + eo, &maps.down, e * H);
            }
        };
        const int fl = (E <= 128) ? topk_rounds<4>(p.logits, E, k, lane, on_round)
                                  : topk_rounds<8>(p.logits, E, k, lane, on_round);
        if (fl && lane == 0) atomicOr(&flags_s, fl);
        // softmax over the k chosen logits (terms relative to the largest,
        // summed in rank order) and the slots: slot of a chosen expert = the
        // number of chosen experts with a lower index (slots are grouped by
        // ascending expert, as in the grouped path)
        if (lane < k) {
            idx_s[lane] = e_r;
            ex_s[lane] = expf(l_r - l_0);
        }
        __syncwarp();
        if (lane < k) {
            float z = 0.0f;
            int before = 0;
            for (int i = 0; i < k; ++i) {
                z += ex_s[i];
                before += (idx_s[i] < e_r) ? 1 : 0;
            }
            w_s[lane] = __fdiv_rn(ex_s[lane], z);
            slot_s[lane] = before;
        }
        if (lane == 0) slot_s[k] = k;  // the shared expert's slot: P + t
    } else {
        // ---- warps 1..: the Q8_0 of x, all blocks in one pass: thread t
        // quantises values 4t .. 4t + 3 (8 threads a block: the block's
        // absolute maximum over 8 lanes, then per value the arithmetic of
        // every Q8_0 step: d = amax / 127, q = round half away from zero of
        // x / d, clamped to +-127); codes into shared memory (pair layout),
        // scales and code sums beside them; CTA 0 also writes them to the
        // workspace.  A binary16 scale overflow is reported.
        for (int t4 = tid - 32; t4 < H / 4; t4 += FFN_THREADS - 32) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(p.x) + t4);
            float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
            for (int o = 4; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
            const float d = __fdiv_rn(a, 127.0f);
            int q0 = 0, q1 = 0, q2 = 0, q3 = 0;
            if (d != 0.0f) {
                q0 = max(-127, min(127, round_half_away(__fdiv_rn(v.x, d))));
                q1 = max(-127, min(127, round_half_away(__fdiv_rn(v.y, d))));
                q2 = max(-127, min(127, round_half_away(__fdiv_rn(v.z, d))));
                q3 = max(-127, min(127, round_half_away(__fdiv_rn(v.w, d))));
            }
            const uint32_t word = (uint32_t)(q0 & 0xff) | ((uint32_t)(q1 & 0xff) << 8) |
                                  ((uint32_t)(q2 & 0xff) << 16) | ((uint32_t)(q3 & 0xff) << 24);
            const int b = t4 >> 3, part = t4 & 7;   // block, word within it
            *reinterpret_cast<uint32_t*>(qa_s + qa_pair_off(b >> 1) + QK * (b & 1) + 4 * part) = word;
            int qs = (q0 + q1) + (q2 + q3);
#pragma unroll
            for (int o = 4; o > 0; o >>= 1) qs += __shfl_xor_sync(0xffffffffu, qs, o);
            const uint16_t db = __half_as_ushort(__float2half_rn(d));
            if (part == 0) {
                da_s[b] = half_bits_to_float(db);
                qsum_s[b] = qs;
                if ((db & 0x7fffu) == 0x7c00u) atomicOr(&flags_s, (int)STATUS_SCALE_OVERFLOW);
            }
            if (blockIdx.x == 0) {
                reinterpret_cast<uint32_t*>(p.qa)[t4] = word;
                if (part == 0) p.da[b] = db;
            }
        }
    }
    __syncthreads();

    // ---- gate/up: warp w computes rows 4w .. 4w + 3 of the 64 (0..31 gate,
    // 32..63 up), from chunk (w mod 8) / 2; lanes split the blocks along H
    {
        if (!mbar_wait_bounded(&bar_gu[(warp & 7) >> 1], 0, MBAR_LIMIT)) timed_out = true;
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        const uint8_t* rows4 = gu_s + (size_t)(warp * 4) * row_gu;
        // lane l takes block pairs l, l + 32, ..
#pragma unroll 1
        for (int pr = lane; pr < nbH / 2; pr += 32) {
            const int4* a = reinterpret_cast<const int4*>(qa_s + qa_pair_off(pr));
            const int4 a0 = a[0], a1 = a[1], a2 = a[2], a3 = a[3];
            const int qa0[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const int qa1[8] = {a2.x, a2.y, a2.z, a2.w, a3.x, a3.y, a3.z, a3.w};
            pair_rows<4>(rows4 + (size_t)pr * 2 * Q4_BYTES, row_gu, qa0, qa1, qsum_s[2 * pr], qsum_s[2 * pr + 1],
                         da_s[2 * pr], da_s[2 * pr + 1], acc);
        }
        const float s = butterfly<4, 32>(acc);
        if (bf_owner<4, 32>(lane)) {
            const int row64 = warp * 4 + bf_index<4, 32>(lane);
            (row64 < 32 ? gs : us)[row64 & 31] = s;
        }
    }
    __syncthreads();

    // ---- SwiGLU + Q8_0 of this CTA's h block, by every warp (each needs all
    // 32 codes for the down column; the arithmetic is the same in every warp):
    // lane l's code into the warp's own 32 bytes of shared memory, read back as
    // eight words.  Warp 0 writes h, the codes and the scale to the workspace.
    const int slot = slot_s[j];
    int hv[8], hsum;
    float dh;
    float h_mine = 0.0f;      // warp 0: lane's h value, code and the scale, written out at the end
    int q_mine = 0;
    uint16_t db_mine = 0;
    {
        const float h = swiglu(gs[lane], us[lane]);
        uint16_t db;
        bool ov;
        const int q = q8_0_lane(h, db, ov);
        int8_t* hw = hq_w + 32 * warp;
        hw[lane] = (int8_t)q;
        __syncwarp();
        const int4 h0 = reinterpret_cast<const int4*>(hw)[0], h1 = reinterpret_cast<const int4*>(hw)[1];
        hv[0] = h0.x; hv[1] = h0.y; hv[2] = h0.z; hv[3] = h0.w;
        hv[4] = h1.x; hv[5] = h1.y; hv[6] = h1.z; hv[7] = h1.w;
        hsum = q8_block_sum(hv);
        dh = half_bits_to_float(db);
        if (warp == 0) {
            h_mine = h;
            q_mine = q;
            db_mine = db;
            if (ov && lane == 0) atomicOr(&flags_s, (int)STATUS_SCALE_OVERFLOW);
        }
    }

    // ---- down: o[n] = w_j * (block hb of row n against the h block), every
    // row n < H; thread rows n = 32 w + lane + 512 i.  Row n's 32 bytes hold
    // 16-byte chunk c at 32 n + 16 (c ^ bit 2 of n) (the copy's swizzle), so
    // a warp's 16-byte loads of 32 consecutive rows hit distinct banks.
    {
        const float wj = is_shared ? 1.0f : w_s[j];
        if (!mbar_wait_bounded(&bar_dn, 0, MBAR_LIMIT)) timed_out = true;
        const uint32_t sh = (uint32_t)(dn_off & 2) * 8u;
        switch (dn_off >> 2) {
            case 0: down_column<0>(dn_s, H, sh, hv, hsum, dh, wj, o_s); break;
            case 1: down_column<1>(dn_s, H, sh, hv, hsum, dh, wj, o_s); break;
            case 2: down_column<2>(dn_s, H, sh, hv, hsum, dh, wj, o_s); break;
            default: down_column<3>(dn_s, H, sh, hv, hsum, dh, wj, o_s); break;
        }
    }
    if (timed_out) atomicOr(&flags_s, (int)STATUS_SPIN_TIMEOUT);
    __syncthreads();
    // ---- combine: y[n] += o[n], vector reductions at L2
    for (int t = tid; t < H / 4; t += FFN_THREADS)
        red_add_v4(p.y + 4 * t, reinterpret_cast<const float4*>(o_s)[t]);
    if (tid == 0 && flags_s) atomicOr(p.status, (uint32_t)flags_s);
    // the h block, its codes and scale, and the inspection arrays of the
    // workspace (the same as the grouped path's), written last: nothing in
    // the call reads them
    if (warp == 0) {
        if (p.h_dbg) p.h_dbg[(size_t)slot * F + hb * QK + lane] = h_mine;
        p.hq[(size_t)slot * F + hb * QK + lane] = (int8_t)q_mine;
        if (lane == 0) p.dh[(size_t)slot * nbF + hb] = db_mine;
    }
    if (blockIdx.x == 0) {
        for (int e = tid; e <= E + 1; e += FFN_THREADS) {
            int o = 0, chosen = 0;
            for (int i = 0; i < k; ++i) {
                o += (idx_s[i] < e) ? 1 : 0;
                chosen |= (idx_s[i] == e) ? 1 : 0;
            }
            if (e < E) p.cnt[e] = chosen;
            if (e == E) p.cnt[E] = p.S;
            p.off[e] = (e <= E) ? o : k + p.S;
        }
        if (tid < k) {
            p.topk_idx[tid] = idx_s[tid];
            p.topk_w[tid] = w_s[tid];
            p.pos[tid] = slot_s[tid];
            p.sorted[slot_s[tid]] = tid;
        }
    }

    if (p.kernel_ns && blockIdx.x == 0 && tid == 0) {
        const unsigned long long t_end = global_ns();
        atomicAdd(p.kernel_ns, t_end - t_ready);
        atomicAdd(p.kernel_ns + 1, 1ull);
        atomicAdd(p.kernel_ns + 2, t_end - t_entry);
    }
}

// ---------------------------------------------------------------------------
// K0 / K3 (host entry only): x copied from and y copied to page-locked host
// memory by the GPU, so the call stays one programmatic-launch chain with no
// copy node in it (one CTA reads x over the bus once; the router's CTAs then
// read the device copy).
// ---------------------------------------------------------------------------
constexpr int COPY_IN_VEC = 4;   // float4 loads a thread: H <= 4 * 4 * 256

// EARLY: x_host is read into registers before the dependency wait, so the
// bus round trip overlaps the previous call's tail; only the store into the
// device copy (which the previous call's kernels may still read) waits.  The
// host side uses it unless x_host overlaps the previous call's y_host on the
// same stream (whose copy-out may still be writing it).
template <bool EARLY>
__global__ void __launch_bounds__(256) decode_copy_in_kernel(const float* __restrict__ x_host, float* __restrict__ x,
                                                             int H) {
    pdl_launch_dependents();
    const float4* src = reinterpret_cast<const float4*>(x_host);
    float4 v[COPY_IN_VEC];
    if (!EARLY) pdl_wait();  // the previous call's kernels no longer read x, nor write x_host
#pragma unroll
    for (int j = 0; j < COPY_IN_VEC; ++j) {
        const int i = threadIdx.x + 256 * j;
        if (i < H / 4) v[j] = src[i];
    }
    if (EARLY) pdl_wait();  // the previous call's kernels no longer read x
#pragma unroll
    for (int j = 0; j < COPY_IN_VEC; ++j) {
        const int i = threadIdx.x + 256 * j;
        if (i < H / 4) reinterpret_cast<float4*>(x)[i] = v[j];
    }
}

__global__ void __launch_bounds__(256) decode_copy_out_kernel(const float* __restrict__ y, float* __restrict__ y_host,
                                                              int H) {
    pdl_launch_dependents();
    pdl_wait();  // the FFN kernel's partial sums are all in y
    for (int i = threadIdx.x; i < H / 4; i += blockDim.x)
        reinterpret_cast<float4*>(y_host)[i] = __ldcg(reinterpret_cast<const float4*>(y) + i);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 decode_encoder() {
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

// Tensor map of a down matrix ([rows][F/32 blocks of 18 bytes], a row a
// multiple of 16 bytes): boxes of 32 bytes x 256 rows, 32-byte swizzle.
cudaError_t encode_down(CUtensorMap* map, const uint8_t* base, uint64_t rows, int F) {
    const PFN_cuTensorMapEncodeTiled_v12000 enc = decode_encoder();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t row_bytes = (cuuint64_t)(F / QK) * Q4_BYTES;
    const cuuint64_t dims[2] = {row_bytes, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)DN_BOX_BYTES, (cuuint32_t)DN_BOX_ROWS};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}



}  // namespace

bool decode_eligible(const LayerView& L, int64_t T, const DeviceInfo& dev) {
    if (T != 1 || L.E > 256 || L.k > 16) return false;
    // one CTA per SM in a single wave
    if ((int64_t)(L.k + L.S) * (L.F / QK) > dev.sm_count) return false;
    // one lane of warp 0 per 256-row box of the down column (lanes 4..31)
    if (L.H / DN_BOX_ROWS > 28) return false;
    const DecodeSmem SL = decode_smem_layout(L.H);
    // the FFN kernel must fit with room for the router kernel's CTA beside it
    return L.H / 4 <= 128 * ROUTER_STEPS && SL.total <= (size_t)std::min(dev.max_smem_optin - 4096, 200 * 1024);
}

cudaError_t launch_decode(const LayerView& L, const float* x, float* y, const Workspace& ws, float* h_dbg,
                          const DeviceInfo& dev, cudaEvent_t ev_start, cudaEvent_t ev_stop, bool force_timeout,
                          bool clear_status, unsigned long long* kernel_ns, const float* x_host, float* y_host,
                          bool x_host_early, cudaStream_t s) {
    DecodeParams p;
    p.H = L.H; p.F = L.F; p.E = L.E; p.k = L.k; p.S = L.S;
    p.nbF = L.F / QK;
    p.clear_status = clear_status ? 1 : 0;
    p.force_timeout = force_timeout ? 1 : 0;
    p.x = x; p.w_router = L.w_router; p.bias = L.router_bias;
    p.w_gate = L.w_gate; p.w_up = L.w_up; p.sh_gate = L.sh_gate; p.sh_up = L.sh_up;
    p.logits = ws.logits; p.topk_idx = ws.topk_idx; p.topk_w = ws.topk_w; p.qa = ws.qa; p.da = ws.da;
    p.cnt = ws.cnt; p.off = ws.off; p.sorted = ws.sorted; p.pos = ws.pos; p.hq = ws.hq; p.dh = ws.dh;
    p.h_dbg = h_dbg; p.y = y; p.status = ws.status; p.kernel_ns = kernel_ns;

    DecodeMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    cudaError_t e = encode_down(&maps.down, L.w_down, (uint64_t)L.E * L.H, L.F);
    if (e == cudaSuccess && L.S) e = encode_down(&maps.sh_down, L.sh_down, (uint64_t)L.H, L.F);
    if (e != cudaSuccess) return e;

    int per_sm = 0;
    e = kernel_occupancy(reinterpret_cast<const void*>(decode_router_kernel), 128, 0, &per_sm);
    if (e != cudaSuccess) return e;
    const DecodeSmem SL = decode_smem_layout(L.H);
    e = kernel_occupancy(reinterpret_cast<const void*>(decode_ffn_kernel), FFN_THREADS, SL.total, &per_sm);
    if (e != cudaSuccess) return e;

    cudaLaunchAttribute attrs[1];
    attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = s;
    cfg.attrs = attrs;
    if (x_host) {
        if (L.H / 4 > 256 * COPY_IN_VEC) return cudaErrorInvalidValue;
        cfg.gridDim = dim3(1);
        cfg.blockDim = dim3(256);
        cfg.dynamicSmemBytes = 0;
        cfg.numAttrs = 1;
        e = x_host_early ? cudaLaunchKernelEx(&cfg, decode_copy_in_kernel<true>, x_host, const_cast<float*>(x), L.H)
                         : cudaLaunchKernelEx(&cfg, decode_copy_in_kernel<false>, x_host, const_cast<float*>(x), L.H);
        if (e != cudaSuccess) return e;
    }
    cfg.gridDim = dim3((unsigned)L.E);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, decode_router_kernel, p);
    if (e != cudaSuccess) return e;

    if (ev_start && (e = record_event(ev_start, s)) != cudaSuccess) return e;
    cfg.gridDim = dim3((unsigned)((L.k + L.S) * p.nbF));
    cfg.blockDim = dim3(FFN_THREADS);
    cfg.dynamicSmemBytes = SL.total;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, decode_ffn_kernel, p, maps);
    if (e != cudaSuccess) return e;
    if (ev_stop && (e = record_event(ev_stop, s)) != cudaSuccess) return e;
    if (y_host) {
        cfg.gridDim = dim3(1);
        cfg.blockDim = dim3(256);
        cfg.dynamicSmemBytes = 0;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, decode_copy_out_kernel, (const float*)y, y_host, L.H);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace moeq4
