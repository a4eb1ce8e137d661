/*
 * moe_q4_oracle.c -- plain, slow CPU oracle of the 4-bit MoE expert FFN.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file.  Its users are the tests, the smoke check of the package
 * entry module and the CPU-baseline leg of the benchmark script.  It shares
 * no code, header, table or constant with the CUDA library.
 *
 * Source of the method: the Dutch technical summary of "A 35B Hybrid-Attention
 * Mixture-of-Experts Model on a 6GB 2011 GPU: Hand-Written 4-bit CUDA
 * Inference for Fermi" (gist.science/nl/paper/2606.24031):
 *   - Methodologie 1 "Hybride GPU-Prefill / CPU-Decode": prefill runs a
 *     grouped 4-bit GEMM for the MoE layers; decode runs a W4A8 integer kernel
 *     (4-bit weights, 8-bit activations, integer multiply-adds).
 *   - Methodologie 2 "Geheugen en Kwantisatie": group-wise symmetric 4-bit
 *     weights of the Q4_0 family, 8-bit activations on the decode path,
 *     128 experts per layer after pruning.
 * The page fixes no bit layout.  The readings taken here (all of them listed
 * in the design notes) are:
 *   Q4_0 block: 32 weights, 18 bytes: bytes 0-1 the scale d as IEEE binary16,
 *     little endian; bytes 2..17 qs[16]; weight i (i<16) is the low nibble of
 *     qs[i], weight i+16 its high nibble; value = (nibble - 8) * d.
 *   Q8_0 block: 32 activations, amax = max |x_i|, d = amax/127 as one IEEE
 *     binary32 division, q_i = round-half-away-from-zero(x_i / d) as one
 *     binary32 division, clamped to [-127, 127]; the stored scale is d rounded
 *     to binary16 (nearest, ties to even); value = q * fp16(d).
 *   Router: fp32 logits x.Wr (+ bias), top-k largest (ties to the lower expert
 *     index), softmax over the k chosen logits.
 *   Expert FFN: h = silu(x.Wg) * (x.Wu), h requantised to Q8_0 along F, then
 *     o = h.Wd; y = sum_j w_j o_j + o_shared (shared expert weight 1).
 *
 * Arithmetic: every block dot product is an exact integer sum; every sum of
 * scaled block terms is taken in binary64 and rounded to binary32 exactly where
 * a GPU kernel would store binary32 (logits, weights, g, u, h, o, y).
 * Loops follow the definitions; the only parallelism is an OpenMP loop over
 * independent tokens, used for timing.  Build with -ffp-contract=off.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define QK 32             /* values per Q4_0 / Q8_0 block */
#define Q4_BYTES 18       /* bytes per Q4_0 block */

/* ------------------------------------------------------------------ */
/* IEEE 754 binary16 <-> binary64 / binary32, from the format definition */
/* ------------------------------------------------------------------ */

/* Value of a binary16 bit pattern: sign, 5-bit exponent (bias 15), 10-bit
 * fraction; exponent 0 = subnormal (fraction * 2^-24), 31 = inf/nan. */
double orc_half_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int ex = (h >> 10) & 0x1f;
    int fr = h & 0x3ff;
    double v;
    if (ex == 0)
        v = ldexp((double)fr, -24);
    else if (ex == 31)
        v = fr ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + fr), ex - 25);
    return sign ? -v : v;
}

/* Nearest binary16 to a binary32 value, ties to even; |f| beyond the largest
 * finite half (65504) rounds to infinity from the halfway point 65520 up. */
uint16_t orc_float_to_half_rne(float f) {
    uint16_t sign = signbit(f) ? 0x8000 : 0;
    double a = fabs((double)f);
    if (isnan(f)) return (uint16_t)(sign | 0x7e00);
    if (a >= 65520.0) return (uint16_t)(sign | 0x7c00);
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: quantum 2^-24; rint() rounds half to even */
        double m = rint(a * ldexp(1.0, 24));
        /* m == 1024 lands exactly on the smallest normal, whose bit pattern
         * is 0x0400 = 1024: the same formula covers it. */
        return (uint16_t)(sign | (uint16_t)m);
    }
    int e2;
    frexp(a, &e2);                   /* a = f * 2^e2, f in [0.5, 1) */
    int e = e2 - 1;                  /* a in [2^e, 2^(e+1)) */
    double m = rint(a * ldexp(1.0, 10 - e));   /* 1024 <= m <= 2048 */
    if (m == 2048.0) { m = 1024.0; e += 1; }
    if (e > 15) return (uint16_t)(sign | 0x7c00);
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)(m - 1024.0));
}

/* Round half away from zero of a binary32 value (the addition is exact in
 * binary64 because v has 24 significant bits). */
int orc_round_half_away(float v) {
    double r = floor(fabs((double)v) + 0.5);
    return (int)(v < 0 ? -r : r);
}

/* ------------------------------------------------------------------ */
/* Q8_0 activation quantisation                                        */
/* ------------------------------------------------------------------ */

/* Quantise n values (n a multiple of 32) block by block.
 * q[i] int8, d[i/32] binary16 bits.  Returns 1 if some binary16 scale
 * overflowed to infinity, else 0. */
int orc_quantize_q8_0(const float* x, int64_t n, int8_t* q, uint16_t* d) {
    int overflow = 0;
    for (int64_t b = 0; b < n / QK; ++b) {
        const float* xb = x + b * QK;
        float amax = 0.0f;
        for (int i = 0; i < QK; ++i) {
            float a = fabsf(xb[i]);
            if (a > amax) amax = a;
        }
        float d32 = amax / 127.0f;            /* one binary32 division */
        for (int i = 0; i < QK; ++i) {
            int qi = 0;
            if (d32 != 0.0f) {
                float v = xb[i] / d32;        /* one binary32 division */
                qi = orc_round_half_away(v);
                if (qi > 127) qi = 127;
                if (qi < -127) qi = -127;
            }
            q[b * QK + i] = (int8_t)qi;
        }
        d[b] = orc_float_to_half_rne(d32);
        if ((d[b] & 0x7fff) == 0x7c00) overflow = 1;
    }
    return overflow;
}

/* ------------------------------------------------------------------ */
/* Q4_0 weights                                                        */
/* ------------------------------------------------------------------ */

/* Signed 4-bit value (nibble - 8) of weight i in one 18-byte block. */
static int q4_weight(const uint8_t* blk, int i) {
    const uint8_t* qs = blk + 2;
    int nib = (i < 16) ? (qs[i] & 0x0f) : (qs[i - 16] >> 4);
    return nib - 8;
}

static uint16_t q4_scale_bits(const uint8_t* blk) {
    return (uint16_t)(blk[0] | (blk[1] << 8));
}

/* Dequantise nblocks consecutive Q4_0 blocks into binary64 values. */
void orc_q4_0_dequant(const uint8_t* blocks, int64_t nblocks, double* out) {
    for (int64_t b = 0; b < nblocks; ++b) {
        const uint8_t* blk = blocks + b * Q4_BYTES;
        double d = orc_half_to_double(q4_scale_bits(blk));
        for (int i = 0; i < QK; ++i) out[b * QK + i] = (double)q4_weight(blk, i) * d;
    }
}

/* Exact integer dot product of one Q4_0 block with 32 Q8_0 values:
 * sum_i (nibble_i - 8) * q_i.  |result| <= 32*8*127 = 32512. */
int32_t orc_block_dot(const uint8_t* blk, const int8_t* qa) {
    int32_t s = 0;
    for (int i = 0; i < QK; ++i) s += q4_weight(blk, i) * (int32_t)qa[i];
    return s;
}

/* out[i] = orc_block_dot(blocks[i], qa[32 i .. 32 i + 31]) for n blocks (18
 * bytes each, consecutive) against n * 32 int8 activations. */
void orc_block_dots(const uint8_t* blocks, int64_t n, const int8_t* qa, int32_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_block_dot(blocks + i * Q4_BYTES, qa + i * QK);
}

/* out[n] = fp32( sum_b d_w[n,b] * d_a[b] * I[n,b] ) for a Q4_0 matrix of N
 * rows and K inputs (row n = K/32 consecutive blocks) against one Q8_0 row.
 * Each term is exact in binary64 (11+11+15 significant bits). */
void orc_q4_matvec(const uint8_t* W, int N, int K, const int8_t* qa,
                   const uint16_t* da, float* out) {
    int nb = K / QK;
    for (int n = 0; n < N; ++n) {
        const uint8_t* row = W + (int64_t)n * nb * Q4_BYTES;
        double acc = 0.0;
        for (int b = 0; b < nb; ++b) {
            const uint8_t* blk = row + (int64_t)b * Q4_BYTES;
            int32_t I = orc_block_dot(blk, qa + b * QK);
            acc += orc_half_to_double(q4_scale_bits(blk)) * orc_half_to_double(da[b]) * (double)I;
        }
        out[n] = (float)acc;
    }
}

/* ------------------------------------------------------------------ */
/* Router                                                              */
/* ------------------------------------------------------------------ */

/* logits[t,e] = fp32( sum_h x[t,h] Wr[e,h] + b[e] ), binary64 sum. */
void orc_router_logits(const float* x, int64_t T, int H, const float* Wr,
                       const float* bias, int E, float* logits) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int h = 0; h < H; ++h)
                acc += (double)x[t * H + h] * (double)Wr[(int64_t)e * H + h];
            if (bias) acc += (double)bias[e];
            logits[t * E + e] = (float)acc;
        }
    }
}

/* Per token: the k largest logits in descending order (equal logits: lower
 * expert index first) and the softmax over those k logits. */
void orc_topk_softmax(const float* logits, int64_t T, int E, int k,
                      int32_t* idx, float* w) {
    for (int64_t t = 0; t < T; ++t) {
        const float* l = logits + t * E;
        int32_t* it = idx + t * k;
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                int taken = 0;
                for (int i = 0; i < j; ++i) taken |= (it[i] == e);
                if (taken) continue;
                if (best < 0 || l[e] > l[best]) best = e;   /* strict: ties keep the lower e */
            }
            it[j] = best;
        }
        double lmax = l[it[0]];
        double z = 0.0;
        for (int j = 0; j < k; ++j) z += exp((double)l[it[j]] - lmax);
        for (int j = 0; j < k; ++j) w[t * k + j] = (float)(exp((double)l[it[j]] - lmax) / z);
    }
}

/* ------------------------------------------------------------------ */
/* Token -> expert permutation (counting sort, stable in (t, j) order)  */
/* ------------------------------------------------------------------ */

/* cnt[e] = number of pairs routed to e; off = exclusive prefix sum of cnt
 * (off[E] = T*k); sorted[off[e] + r] = t*k + j for the r-th pair of expert e
 * in increasing (t, j) order; pos is the inverse of sorted. */
void orc_permute(const int32_t* idx, int64_t T, int k, int E, int32_t* cnt,
                 int32_t* off, int32_t* sorted, int32_t* pos) {
    int64_t P = T * k;
    for (int e = 0; e < E; ++e) cnt[e] = 0;
    for (int64_t p = 0; p < P; ++p) cnt[idx[p]] += 1;
    off[0] = 0;
    for (int e = 0; e < E; ++e) off[e + 1] = off[e] + cnt[e];
    int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    for (int64_t p = 0; p < P; ++p) {
        int e = idx[p];
        int32_t s = off[e] + fill[e]++;
        sorted[s] = (int32_t)p;
        pos[p] = s;
    }
    free(fill);
}

/* ------------------------------------------------------------------ */
/* The MoE expert FFN layer                                            */
/* ------------------------------------------------------------------ */

typedef struct {
    int32_t hidden, ffn, n_experts, top_k, has_shared;
    const float* w_router;      /* [E][H] */
    const float* router_bias;   /* [E] or NULL */
    const uint8_t* w_gate;      /* [E][F][H/32] blocks */
    const uint8_t* w_up;        /* [E][F][H/32] blocks */
    const uint8_t* w_down;      /* [E][H][F/32] blocks */
    const uint8_t* sh_gate;     /* [F][H/32] or NULL */
    const uint8_t* sh_up;
    const uint8_t* sh_down;     /* [H][F/32] */
} orc_layer;

/* Optional outputs (any pointer may be NULL).  Pair index pj = t*(k+S) + j;
 * j = k is the shared expert. */
typedef struct {
    float* logits;      /* [T][E] */
    int32_t* idx;       /* [T][k] */
    float* w;           /* [T][k] */
    int8_t* qa;         /* [T][H] */
    uint16_t* da;       /* [T][H/32] */
    float* g;           /* [T][k+S][F] */
    float* u;           /* [T][k+S][F] */
    float* h;           /* [T][k+S][F] */
    int8_t* hq;         /* [T][k+S][F] */
    uint16_t* dh;       /* [T][k+S][F/32] */
    float* o;           /* [T][k+S][H] */
    int32_t* overflow;  /* [1] set to 1 if a binary16 scale overflowed */
} orc_debug;

static double silu(double g) { return g / (1.0 + exp(-g)); }

/* y[t] for T tokens.  forced_idx/forced_w replace the router (teacher
 * forcing); forced_hq/forced_dh ([T][k+S][F], [T][k+S][F/32]) replace the
 * requantised SwiGLU output.  Returns 0, or -1 on bad arguments. */
int orc_moe_forward(const orc_layer* L, const float* x, int64_t T, float* y,
                    const int32_t* forced_idx, const float* forced_w,
                    const int8_t* forced_hq, const uint16_t* forced_dh,
                    orc_debug* dbg) {
    const int H = L->hidden, F = L->ffn, E = L->n_experts, k = L->top_k;
    const int S = L->has_shared ? 1 : 0;
    const int J = k + S;
    if (H % QK || F % QK || k < 1 || k > E || T < 0) return -1;
    if (T == 0) return 0;

    float* logits = (float*)malloc(sizeof(float) * (size_t)T * E);
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)T * k);
    float* w = (float*)malloc(sizeof(float) * (size_t)T * k);
    int8_t* qa = (int8_t*)malloc((size_t)T * H);
    uint16_t* da = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)T * (H / QK));
    int overflow = 0;

    if (forced_idx) {
        memcpy(idx, forced_idx, sizeof(int32_t) * (size_t)T * k);
        memcpy(w, forced_w, sizeof(float) * (size_t)T * k);
    } else {
        orc_router_logits(x, T, H, L->w_router, L->router_bias, E, logits);
        orc_topk_softmax(logits, T, E, k, idx, w);
        if (dbg && dbg->logits) memcpy(dbg->logits, logits, sizeof(float) * (size_t)T * E);
    }
    for (int64_t t = 0; t < T; ++t)
        overflow |= orc_quantize_q8_0(x + t * H, H, qa + t * H, da + t * (H / QK));

    const int64_t gu_stride = (int64_t)F * (H / QK) * Q4_BYTES;   /* bytes per expert */
    const int64_t dn_stride = (int64_t)H * (F / QK) * Q4_BYTES;

#pragma omp parallel for schedule(dynamic, 1) reduction(| : overflow)
    for (int64_t t = 0; t < T; ++t) {
        float* g = (float*)malloc(sizeof(float) * F);
        float* u = (float*)malloc(sizeof(float) * F);
        float* h = (float*)malloc(sizeof(float) * F);
        int8_t* hq = (int8_t*)malloc((size_t)F);
        uint16_t* dh = (uint16_t*)malloc(sizeof(uint16_t) * (F / QK));
        float* o = (float*)malloc(sizeof(float) * H);
        double* acc = (double*)calloc((size_t)H, sizeof(double));
        for (int j = 0; j < J; ++j) {
            const uint8_t *Wg, *Wu, *Wd;
            double wj;
            if (j < k) {
                int e = idx[t * k + j];
                Wg = L->w_gate + e * gu_stride;
                Wu = L->w_up + e * gu_stride;
                Wd = L->w_down + e * dn_stride;
                wj = (double)w[t * k + j];
            } else {
                Wg = L->sh_gate; Wu = L->sh_up; Wd = L->sh_down;
                wj = 1.0;
            }
            const int8_t* qt = qa + t * H;
            const uint16_t* dt = da + t * (H / QK);
            orc_q4_matvec(Wg, F, H, qt, dt, g);
            orc_q4_matvec(Wu, F, H, qt, dt, u);
            for (int n = 0; n < F; ++n) h[n] = (float)(silu((double)g[n]) * (double)u[n]);
            int64_t pj = t * J + j;
            if (forced_hq) {
                memcpy(hq, forced_hq + pj * F, (size_t)F);
                memcpy(dh, forced_dh + pj * (F / QK), sizeof(uint16_t) * (F / QK));
            } else {
                overflow |= orc_quantize_q8_0(h, F, hq, dh);
            }
            orc_q4_matvec(Wd, H, F, hq, dh, o);
            for (int n = 0; n < H; ++n) acc[n] += wj * (double)o[n];
            if (dbg) {
                if (dbg->g) memcpy(dbg->g + pj * F, g, sizeof(float) * F);
                if (dbg->u) memcpy(dbg->u + pj * F, u, sizeof(float) * F);
                if (dbg->h) memcpy(dbg->h + pj * F, h, sizeof(float) * F);
                if (dbg->hq) memcpy(dbg->hq + pj * F, hq, (size_t)F);
                if (dbg->dh) memcpy(dbg->dh + pj * (F / QK), dh, sizeof(uint16_t) * (F / QK));
                if (dbg->o) memcpy(dbg->o + pj * H, o, sizeof(float) * H);
            }
        }
        for (int n = 0; n < H; ++n) y[t * H + n] = (float)acc[n];
        free(g); free(u); free(h); free(hq); free(dh); free(o); free(acc);
    }

    if (dbg) {
        if (dbg->idx) memcpy(dbg->idx, idx, sizeof(int32_t) * (size_t)T * k);
        if (dbg->w) memcpy(dbg->w, w, sizeof(float) * (size_t)T * k);
        if (dbg->qa) memcpy(dbg->qa, qa, (size_t)T * H);
        if (dbg->da) memcpy(dbg->da, da, sizeof(uint16_t) * (size_t)T * (H / QK));
        if (dbg->overflow) dbg->overflow[0] = overflow;
    }
    free(logits); free(idx); free(w); free(qa); free(da);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Glue between the layers of a stack                                  */
/* ------------------------------------------------------------------ */

/* The page runs the MoE layers one after another (Methodologie 1: expert
 * weights are streamed layer by layer) but fixes no step between them; the
 * multi-layer workload joins them by a residual add.  Without a normalisation
 * the activations grow by about 25x per layer and the binary16 Q8_0 scales
 * overflow within a few layers, so the reading taken is
 * x_{l+1} = x_l + MoE_l(RMSNorm(x_l)) with a unit-gain RMSNorm over H:
 * rms = sqrt(mean_h x^2 + eps), the mean taken in binary64;
 * xn = binary32(x / rms). */
void orc_rmsnorm(const float* x, int64_t T, int H, float eps, float* xn) {
    for (int64_t t = 0; t < T; ++t) {
        const float* r = x + t * H;
        double ss = 0.0;
        for (int h = 0; h < H; ++h) ss += (double)r[h] * (double)r[h];
        const double rms = sqrt(ss / (double)H + (double)eps);
        for (int h = 0; h < H; ++h) xn[t * H + h] = (float)((double)r[h] / rms);
    }
}

/* x <- binary32(x + y): the exact sum rounded once. */
void orc_residual_add(float* x, const float* y, int64_t n) {
    for (int64_t i = 0; i < n; ++i) x[i] = (float)((double)x[i] + (double)y[i]);
}

/* Thread count used by the OpenMP loops (timing only); returns the count. */
int orc_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}
