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
//     kernel it bulk-copies its router row into shared memory; then the logit
//     (four independent FMA chains), and the first H/32 CTAs quantise one
//     Q8_0 block of x each.  CTA 0 zeroes the status word and the grid-barrier
//     counter of the next kernel.
//   decode_ffn_kernel: cooperative, one CTA of 16 warps per SM.  Before
//     waiting on the router, bulk-copies the shared expert's weights
//     (routing-independent); then the top-k (every thread ranks one logit),
//     bulk copies of its gate/up row block (32 rows of F = one Q8_0 block of
//     h) and of its slice of down rows for all k+1 experts; gate/up dot
//     products (the activation block loaded once for four rows, four
//     independent chains per lane), SwiGLU, requantisation; one bounded grid
//     barrier; down dot products (eight rows per lane group) and the
//     router-weighted combine into y in a fixed order (no atomics).
//
// Every phase runs once per launch on every SM, so each is written as short,
// independent dependency chains: measured on B200, the same arithmetic with
// one row at a time and a reduction per row took 3.7x longer.
#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace moeq4 {

constexpr uint32_t MBAR_LIMIT = 1u << 20;

struct DecodeParams {
    int H, F, E, k, S;
    int rows_per_cta;  // down rows of H per FFN CTA
    int nctas;         // grid of decode_ffn_kernel
    int barrier_target;  // arrivals the grid barrier waits for (nctas; nctas + 1 only in the timeout test)
    int clear_status;    // the router kernel zeroes the status word (else it accumulates)
    const float* x;
    const float* w_router;
    const float* bias;
    const uint8_t* w_gate;
    const uint8_t* w_up;
    const uint8_t* w_down;
    const uint8_t* sh_gate;
    const uint8_t* sh_up;
    const uint8_t* sh_down;
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
    uint32_t* status;  // status[0] = status word, status[1] = grid-barrier counter
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

// ---------------------------------------------------------------------------
// K1: router logits (one CTA per expert) + Q8_0 of x.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) decode_router_kernel(DecodeParams p) {
    extern __shared__ __align__(16) unsigned char dsm[];
    float* wr_s = reinterpret_cast<float*>(dsm);
    __shared__ __align__(8) uint64_t bar;
    __shared__ float red[4];
    const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = p.H;
    if (tid == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    if (tid == 0) {
        mbar_arrive_expect_tx(&bar, (uint32_t)H * 4u);
        bulk_g2s(wr_s, p.w_router + (size_t)e * H, (uint32_t)H * 4u, &bar);
    }
    pdl_launch_dependents();
    pdl_wait();  // x and the workspace are now the previous kernels' results
    if (e == 0 && tid == 0) {
        if (p.clear_status) p.status[0] = 0u;  // status word
        p.status[1] = 0u;  // grid-barrier counter of decode_ffn_kernel
    }
    const bool ok = mbar_wait_bounded(&bar, 0, MBAR_LIMIT);
    const float4* x4 = reinterpret_cast<const float4*>(p.x);
    const float4* w4 = reinterpret_cast<const float4*>(wr_s);
    float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;  // four independent chains
    for (int h4 = tid; h4 < H / 4; h4 += 128) {
        const float4 a = __ldcg(x4 + h4), b = w4[h4];
        a0 = fmaf(a.x, b.x, a0);
        a1 = fmaf(a.y, b.y, a1);
        a2 = fmaf(a.z, b.z, a2);
        a3 = fmaf(a.w, b.w, a3);
    }
    float acc = (a0 + a1) + (a2 + a3);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) red[warp] = acc;
    __syncthreads();
    if (tid == 0) {
        const float l = (red[0] + red[1]) + (red[2] + red[3]) + (p.bias ? __ldg(p.bias + e) : 0.0f);
        p.logits[e] = ok ? l : __int_as_float(0x7fc00000);  // a NaN logit reports the timeout
    }
    // Q8_0 of x: block b by warp 0 of CTA b (and CTA b + E, ... when H/32 > E).
    // A binary16 scale overflow is visible to the next kernel as an infinite scale.
    if (warp == 0) {
        for (int b = e; b < H / QK; b += gridDim.x) {
            uint16_t db;
            bool ov;
            const int q = q8_0_lane(__ldcg(p.x + b * QK + lane), db, ov);
            p.qa[b * QK + lane] = (int8_t)q;
            if (lane == 0) p.da[b] = db;
        }
    }
}

// ---------------------------------------------------------------------------
// K2: top-k, gate/up + SwiGLU + requant, grid barrier, down + combine.
// ---------------------------------------------------------------------------
struct DecodeSmem {
    size_t gu, dn, qa, da, qsum, hq, dhs, hsum, o, total;  // byte offsets
};

__host__ __device__ inline size_t al16(size_t v) { return (v + 15) & ~size_t(15); }

__host__ __device__ inline DecodeSmem decode_smem_layout(int H, int F, int J, int R) {
    const int nbH = H / QK, nbF = F / QK;
    DecodeSmem L;
    size_t o = 0;
    L.gu = o;   o += al16((size_t)64 * nbH * Q4_BYTES);
    L.dn = o;   o += al16((size_t)J * R * nbF * Q4_BYTES);
    L.qa = o;   o += al16((size_t)H);
    L.da = o;   o += al16((size_t)nbH * 4);
    L.qsum = o; o += al16((size_t)nbH * 4);
    L.hq = o;   o += al16((size_t)J * F);
    L.dhs = o;  o += al16((size_t)J * nbF * 4);
    L.hsum = o; o += al16((size_t)J * nbF * 4);
    L.o = o;    o += al16((size_t)J * R * 4);
    L.total = o;
    return L;
}

// acc[r] += W4A8 term of block b of NR rows (stride row_bytes) against one
// staged Q8_0 block, the activation loaded once for all rows: NR independent
// dependency chains per lane.
template <int NR>
__device__ __forceinline__ void block_rows(const uint8_t* rows, size_t row_bytes, int nrows, int b, const int8_t* q_s,
                                           int qsum, float da, float (&acc)[NR]) {
    const int4* qv = reinterpret_cast<const int4*>(q_s + b * QK);
    const int4 a0 = qv[0], a1 = qv[1];
    const int qa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
    for (int r = 0; r < NR; ++r) {
        if (r < nrows) {
            uint32_t qs[4], dbits;
            load_q4_block_smem(rows + (size_t)r * row_bytes + (size_t)b * Q4_BYTES, qs, dbits);
            acc[r] = fmaf((float)q4_q8_dot(qs, qa, qsum), half_bits_to_float(dbits) * da, acc[r]);
        }
    }
}

// Down projection for the CTA's rows: tasks (pair jj, chunk of 8 rows), one per
// lane group of W lanes; lanes split the F/32 blocks.
template <int W>
__device__ __forceinline__ void down_tasks(const uint8_t* dn_s, size_t row_dn, int R, int rows, int J, int nbF, int F,
                                           const int8_t* hq_s, const float* dh_s, const int* hsum_s, const int* slot_s,
                                           float* o_s, int warp, int n_warps) {
    constexpr int G = 32 / W;  // lane groups per warp
    const int lane = threadIdx.x & 31, grp = lane / W, sub = lane % W;
    const int chunks = (rows + 7) / 8;
    const int n_tasks = J * chunks;
#pragma unroll 1
    for (int t0 = warp * G; t0 < n_tasks; t0 += n_warps * G) {  // warp-uniform trip count
        const int task = min(t0 + grp, n_tasks - 1);
        const int jj = task / chunks, r0 = (task % chunks) * 8;
        const int nr = min(8, rows - r0);
        const int slot = slot_s[jj];
        const int8_t* q = hq_s + (size_t)slot * F;
        const uint8_t* base = dn_s + ((size_t)jj * R + r0) * row_dn;
        float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll 1
        for (int b = sub; b < nbF; b += W)
            block_rows<8>(base, row_dn, nr, b, q, hsum_s[slot * nbF + b], dh_s[slot * nbF + b], acc);
        const float s = butterfly<8, W>(acc);
        const int r = bf_index<8, W>(sub);
        if (bf_owner<8, W>(sub) && t0 + grp < n_tasks && r < nr) o_s[jj * R + r0 + r] = s;
    }
}

constexpr int FFN_THREADS = 512;  // 16 warps
constexpr int FFN_WARPS = FFN_THREADS / 32;

// At most 96 registers per thread: 512 x 96 plus the router kernel's CTAs fit
// one SM's register file, so the next router kernel can become resident
// beside this one under programmatic dependent launch.
__global__ void __maxnreg__(96) decode_ffn_kernel(DecodeParams p) {
    extern __shared__ __align__(16) unsigned char dsm[];
    __shared__ __align__(8) uint64_t bar_gu[4];
    __shared__ __align__(8) uint64_t bar_dn;
    __shared__ __align__(16) float logit_s[256];  // E rounded up to 16
    __shared__ int idx_s[16];
    __shared__ float w_s[16];
    __shared__ float ex_s[16];
    __shared__ int slot_s[17];
    __shared__ int warp_chosen[FFN_WARPS];
    __shared__ float gs[32], us[32];
    __shared__ int flags_s;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = p.H, F = p.F, E = p.E, k = p.k, S = p.S;
    const int J = k + S, nbH = H / QK, nbF = F / QK, nrb = F / GU_ROWS;
    const int R = p.rows_per_cta;
    const size_t row_gu = (size_t)nbH * Q4_BYTES, row_dn = (size_t)nbF * Q4_BYTES;
    const size_t gu_stride = (size_t)F * row_gu, dn_stride = (size_t)H * row_dn;
    const DecodeSmem SL = decode_smem_layout(H, F, J, R);
    uint8_t* gu_s = dsm + SL.gu;
    uint8_t* dn_s = dsm + SL.dn;
    int8_t* qa_s = reinterpret_cast<int8_t*>(dsm + SL.qa);
    float* da_s = reinterpret_cast<float*>(dsm + SL.da);
    int* qsum_s = reinterpret_cast<int*>(dsm + SL.qsum);
    int8_t* hq_s = reinterpret_cast<int8_t*>(dsm + SL.hq);
    float* dh_s = reinterpret_cast<float*>(dsm + SL.dhs);
    int* hsum_s = reinterpret_cast<int*>(dsm + SL.hsum);
    float* o_s = reinterpret_cast<float*>(dsm + SL.o);

    const int n_items = J * nrb;
    const int n0 = blockIdx.x * R;
    const int rows = max(0, min(R, H - n0));
    bool timed_out = false;

    if (tid == 0) {
        for (int c = 0; c < 4; ++c) mbar_init(&bar_gu[c], 1);
        mbar_init(&bar_dn, 1);
        mbar_fence_init();
        flags_s = 0;
    }
    __syncthreads();

    // gate/up copies of one item, issued by warp 0: chunk c = 8 gate rows + 8
    // up rows on bar_gu[c]; lane 2c + mat issues one copy
    const uint32_t chunk_bytes = (uint32_t)(8 * row_gu);
    auto issue_gateup = [&](const uint8_t* Wg, const uint8_t* Wu, int rb) {
        if (lane < 4) mbar_arrive_expect_tx(&bar_gu[lane], 2u * chunk_bytes);
        __syncwarp();
        if (lane < 8) {
            const int c = lane >> 1, mat = lane & 1;
            bulk_g2s(gu_s + (size_t)(mat * 32 + 8 * c) * row_gu, (mat ? Wu : Wg) + (size_t)(rb * GU_ROWS + 8 * c) * row_gu,
                     chunk_bytes, &bar_gu[c]);
        }
    };

    // ---- prologue: routing-independent copies (the shared expert), before the wait
    const int item0 = blockIdx.x;
    const bool item0_shared = S && item0 < n_items && (item0 / nrb) == k;
    if (warp == 0) {
        if (rows > 0 && lane == 0) {
            mbar_arrive_expect_tx(&bar_dn, (uint32_t)(J * rows * row_dn));
            if (S)
                bulk_g2s(dn_s + (size_t)k * R * row_dn, p.sh_down + (size_t)n0 * row_dn, (uint32_t)(rows * row_dn),
                         &bar_dn);
        }
        if (item0_shared) issue_gateup(p.sh_gate, p.sh_up, item0 % nrb);
    }

    pdl_wait();  // logits, Q8_0 of x and the zeroed status words are visible
    pdl_launch_dependents();

    // ---- top-k: expert e is ranked by P consecutive threads (P = 4 for
    // E <= 128, else 2), each comparing logit e with a 1/P share of the logits
    // (descending, equal logits by expert index); the P partial ranks are
    // summed with shuffles.  Ranks below k are the chosen experts, in order.
    const int E16 = (E + 15) & ~15;
    const int P = (E16 <= FFN_THREADS / 4) ? 4 : 2;
    // a NaN logit (non-finite data, or the router kernel's timeout report)
    // ranks as -infinity, so the ranks below stay a permutation of [0, E)
    for (int e = tid; e < E16; e += blockDim.x) {
        float l = (e < E) ? __ldcg(p.logits + e) : -INFINITY;
        if (e < E && !isfinite(l)) atomicOr(&flags_s, (int)STATUS_NONFINITE_LOGIT);
        logit_s[e] = (l != l) ? -INFINITY : l;
    }
    for (int i = tid; i < H / 16; i += blockDim.x)
        reinterpret_cast<int4*>(qa_s)[i] = __ldcg(reinterpret_cast<const int4*>(p.qa) + i);
    for (int b = tid; b < nbH; b += blockDim.x) {
        const uint32_t bits = __ldcg(p.da + b);
        if ((bits & 0x7fffu) == 0x7c00u) atomicOr(&flags_s, (int)STATUS_SCALE_OVERFLOW);
        da_s[b] = half_bits_to_float(bits);
    }
    __syncthreads();
    const int e_me = tid / P, part = tid % P;
    float my_l = 0.0f;
    int rank = 0;
    if (e_me < E) {
        my_l = logit_s[e_me];
        const float4* l4 = reinterpret_cast<const float4*>(logit_s);
        const int per4 = E16 / (4 * P);
#pragma unroll 4
        for (int e4 = part * per4; e4 < (part + 1) * per4; ++e4) {
            const float4 v = l4[e4];
            const int e = 4 * e4;
            rank += (v.x > my_l || (v.x == my_l && e < e_me)) ? 1 : 0;
            rank += (v.y > my_l || (v.y == my_l && e + 1 < e_me)) ? 1 : 0;
            rank += (v.z > my_l || (v.z == my_l && e + 2 < e_me)) ? 1 : 0;
            rank += (v.w > my_l || (v.w == my_l && e + 3 < e_me)) ? 1 : 0;
        }
    }
    rank += __shfl_xor_sync(0xffffffffu, rank, 1);
    if (P == 4) rank += __shfl_xor_sync(0xffffffffu, rank, 2);
    const int my_rank = (e_me < E) ? rank : k;
    if (part == 0 && my_rank < k) idx_s[my_rank] = e_me;
    // slot of a chosen expert = number of chosen experts with a lower index
    // (slots are grouped by ascending expert, as in the grouped path)
    const bool chosen = part == 0 && my_rank < k;
    const unsigned chosen_mask = __ballot_sync(0xffffffffu, chosen);
    if (lane == 0) warp_chosen[warp] = __popc(chosen_mask);
    for (int b = tid; b < nbH; b += blockDim.x) {
        const int* qw = reinterpret_cast<const int*>(qa_s + b * QK);
        int s = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) s = __dp4a(qw[j], 0x01010101, s);
        qsum_s[b] = s;
    }
    __syncthreads();
    if (chosen) {
        int before = __popc(chosen_mask & ((1u << lane) - 1u));
        for (int w2 = 0; w2 < warp; ++w2) before += warp_chosen[w2];
        slot_s[my_rank] = before;
        ex_s[my_rank] = expf(my_l - logit_s[idx_s[0]]);
    }
    if (tid == 0) slot_s[k] = k;  // the shared expert's slot: P + t
    __syncthreads();

    // ---- routed copies (warp 0), softmax weights (warp 1), inspection arrays (CTA 0)
    if (warp == 0) {
        // gate/up first: the grid barrier waits for the last CTA's gate/up
        // data, while the down rows are needed only after it
        if (item0 < n_items && !item0_shared) {
            const size_t eo = (size_t)idx_s[item0 / nrb] * gu_stride;
            issue_gateup(p.w_gate + eo, p.w_up + eo, item0 % nrb);
        }
        __syncwarp();
        if (rows > 0 && lane < k)
            bulk_g2s(dn_s + (size_t)lane * R * row_dn, p.w_down + (size_t)idx_s[lane] * dn_stride + (size_t)n0 * row_dn,
                     (uint32_t)(rows * row_dn), &bar_dn);
    } else if (warp == 1 && lane < k) {
        float z = 0.0f;
        for (int j = 0; j < k; ++j) z += ex_s[j];
        w_s[lane] = __fdiv_rn(ex_s[lane], z);
    }
    if (blockIdx.x == 0) {
        if (part == 0 && e_me < E) p.cnt[e_me] = chosen ? 1 : 0;
        if (tid == 0) p.cnt[E] = S;
        for (int e = tid; e <= E + 1; e += blockDim.x) {
            int o = 0;
            if (e <= E)
                for (int j = 0; j < k; ++j) o += (idx_s[j] < e) ? 1 : 0;
            p.off[e] = (e <= E) ? o : k + S;
        }
    }
    __syncthreads();
    if (blockIdx.x == 0 && tid < k) {
        p.topk_idx[tid] = idx_s[tid];
        p.topk_w[tid] = w_s[tid];
        p.pos[tid] = slot_s[tid];
        p.sorted[slot_s[tid]] = tid;
    }

    // ---- gate/up + SwiGLU + requant, one item per pass.  Warp w computes the
    // rows 4w..4w+3 of the 64 (0..31 gate, 32..63 up): chunk (w mod 8) / 2.
    uint32_t gu_phase = 0;
    for (int item = item0; item < n_items; item += gridDim.x) {
        const int j = item / nrb, rb = item % nrb;
        if (item != item0 && warp == 0) {
            if (lane == 0) fence_proxy_async_smem();
            __syncwarp();
            const size_t eo = (j < k) ? (size_t)idx_s[j] * gu_stride : 0;
            issue_gateup((j < k) ? p.w_gate + eo : p.sh_gate, (j < k) ? p.w_up + eo : p.sh_up, rb);
        }
        if (!mbar_wait_bounded(&bar_gu[(warp & 7) >> 1], gu_phase, MBAR_LIMIT)) timed_out = true;
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        const uint8_t* rows4 = gu_s + (size_t)(warp * 4) * row_gu;
#pragma unroll 1
        for (int b = lane; b < nbH; b += 32) block_rows<4>(rows4, row_gu, 4, b, qa_s, qsum_s[b], da_s[b], acc);
        const float s = butterfly<4, 32>(acc);
        if (bf_owner<4, 32>(lane)) {
            const int row64 = warp * 4 + bf_index<4, 32>(lane);
            (row64 < 32 ? gs : us)[row64 & 31] = s;
        }
        __syncthreads();
        if (warp == 0) {
            const int slot = slot_s[j];
            const float h = swiglu(gs[lane], us[lane]);
            if (p.h_dbg) p.h_dbg[(size_t)slot * F + rb * GU_ROWS + lane] = h;
            uint16_t db;
            bool ov;
            const int q = q8_0_lane(h, db, ov);
            p.hq[(size_t)slot * F + rb * GU_ROWS + lane] = (int8_t)q;
            if (lane == 0) {
                p.dh[(size_t)slot * nbF + rb] = db;
                if (ov) atomicOr(&flags_s, (int)STATUS_SCALE_OVERFLOW);
            }
        }
        gu_phase ^= 1u;
        __syncthreads();
    }

    // ---- every CTA's requantised rows are written: grid barrier
    __threadfence();
    grid_barrier_bounded(p.status + 1, (uint32_t)p.barrier_target, p.status, STATUS_SPIN_TIMEOUT);

    if (rows > 0) {
        // requantised SwiGLU rows of all k+1 slots (L2: written by other SMs)
        for (int i = tid; i < J * F / 16; i += blockDim.x)
            reinterpret_cast<int4*>(hq_s)[i] = __ldcg(reinterpret_cast<const int4*>(p.hq) + i);
        for (int i = tid; i < J * nbF; i += blockDim.x) dh_s[i] = half_bits_to_float(__ldcg(p.dh + i));
        __syncthreads();
        for (int i = tid; i < J * nbF; i += blockDim.x) {
            const int* qw = reinterpret_cast<const int*>(hq_s + i * QK);
            int s = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) s = __dp4a(qw[q], 0x01010101, s);
            hsum_s[i] = s;
        }
        __syncthreads();
        if (!mbar_wait_bounded(&bar_dn, 0, MBAR_LIMIT)) timed_out = true;
        if (nbF >= 32)
            down_tasks<32>(dn_s, row_dn, R, rows, J, nbF, F, hq_s, dh_s, hsum_s, slot_s, o_s, warp, FFN_WARPS);
        else if (nbF >= 16)
            down_tasks<16>(dn_s, row_dn, R, rows, J, nbF, F, hq_s, dh_s, hsum_s, slot_s, o_s, warp, FFN_WARPS);
        else
            down_tasks<8>(dn_s, row_dn, R, rows, J, nbF, F, hq_s, dh_s, hsum_s, slot_s, o_s, warp, FFN_WARPS);
        __syncthreads();
        for (int r = tid; r < rows; r += blockDim.x) {
            float acc = 0.0f;
            for (int j = 0; j < k; ++j) acc = fmaf(w_s[j], o_s[j * R + r], acc);
            if (S) acc += o_s[k * R + r];
            p.y[n0 + r] = acc;
        }
    }
    if (timed_out) atomicOr(&flags_s, (int)STATUS_SPIN_TIMEOUT);
    __syncthreads();
    if (tid == 0 && flags_s) atomicOr(p.status, (uint32_t)flags_s);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static int decode_rows_per_cta(int H, int G) { return (int)ceil_div(H, G); }

static size_t router_smem(const LayerView& L) { return (size_t)L.H * 4; }

bool decode_eligible(const LayerView& L, int64_t T, const DeviceInfo& dev) {
    if (T != 1 || L.E > 256 || L.k > 16) return false;
    const int G = dev.sm_count;
    const int R = decode_rows_per_cta(L.H, G);
    const DecodeSmem SL = decode_smem_layout(L.H, L.F, L.k + L.S, R);
    // the FFN kernel must fit with room for the router kernel's CTA beside it
    return SL.total <= (size_t)std::min(dev.max_smem_optin - 4096, 200 * 1024) && router_smem(L) <= 96 * 1024;
}

cudaError_t launch_decode(const LayerView& L, const float* x, float* y, const Workspace& ws, float* h_dbg,
                          const DeviceInfo& dev, cudaEvent_t ev_start, cudaEvent_t ev_stop, bool force_timeout,
                          bool clear_status, cudaStream_t s) {
    DecodeParams p;
    p.clear_status = clear_status ? 1 : 0;
    p.H = L.H; p.F = L.F; p.E = L.E; p.k = L.k; p.S = L.S;
    p.nctas = dev.sm_count;
    p.barrier_target = p.nctas + (force_timeout ? 1 : 0);
    p.rows_per_cta = decode_rows_per_cta(L.H, p.nctas);
    p.x = x; p.w_router = L.w_router; p.bias = L.router_bias;
    p.w_gate = L.w_gate; p.w_up = L.w_up; p.w_down = L.w_down;
    p.sh_gate = L.sh_gate; p.sh_up = L.sh_up; p.sh_down = L.sh_down;
    p.logits = ws.logits; p.topk_idx = ws.topk_idx; p.topk_w = ws.topk_w; p.qa = ws.qa; p.da = ws.da;
    p.cnt = ws.cnt; p.off = ws.off; p.sorted = ws.sorted; p.pos = ws.pos; p.hq = ws.hq; p.dh = ws.dh;
    p.h_dbg = h_dbg; p.y = y; p.status = ws.status;

    int per_sm = 0;
    const size_t smem1 = router_smem(L);
    cudaError_t e = kernel_occupancy(reinterpret_cast<const void*>(decode_router_kernel), 128, smem1, &per_sm);
    if (e != cudaSuccess) return e;
    const DecodeSmem SL = decode_smem_layout(L.H, L.F, L.k + L.S, p.rows_per_cta);
    e = kernel_occupancy(reinterpret_cast<const void*>(decode_ffn_kernel), FFN_THREADS, SL.total, &per_sm);
    if (e != cudaSuccess) return e;

    cudaLaunchAttribute attrs[2];
    attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)L.E);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = smem1;
    cfg.stream = s;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, decode_router_kernel, p);
    if (e != cudaSuccess) return e;

    if (ev_start && (e = record_event(ev_start, s)) != cudaSuccess) return e;
    attrs[1].id = cudaLaunchAttributeCooperative;
    attrs[1].val.cooperative = 1;
    cfg.gridDim = dim3((unsigned)p.nctas);
    cfg.blockDim = dim3(FFN_THREADS);
    cfg.dynamicSmemBytes = SL.total;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, decode_ffn_kernel, p);
    if (e != cudaSuccess) return e;
    if (ev_stop && (e = record_event(ev_stop, s)) != cudaSuccess) return e;
    return cudaSuccess;
}

}  // namespace moeq4
