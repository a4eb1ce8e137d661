/*
 * w4a8_simd.c -- the decode side of the page's method on the host CPU, with
 * SIMD integer multiply-adds: a timed CPU baseline for the GPU library.
 *
 * "A 35B Hybrid-Attention Mixture-of-Experts Model on a 6GB 2011 GPU" (Dutch
 * technical summary, Methodologie 1 and Resultaten): decode runs a W4A8
 * kernel on the CPU, unpacking 4-bit weights and multiplying them with 8-bit
 * activations on the SIMD integer units (SSSE3 pmaddubsw on the authors'
 * Xeon).  Here the same idea on x86-64 AVX2 (vpmaddubsw + vpmaddwd), or the
 * fused u8 x s8 dot-product instruction (vpdpbusd) where the build machine
 * has AVX-VNNI.  Independent of the CUDA library and of the oracle; tested
 * against the oracle (per-block integer sums bit for bit, the layer within
 * tolerance).
 *
 * Per token: fp32 router logits, top-k (ties to the lower expert index) and
 * softmax over the k chosen logits, Q8_0 of x (IEEE binary32 divisions,
 * round half away from zero, binary16 scale), then for the k routed experts
 * and the shared expert: gate/up rows (Q4_0 x Q8_0 block dot products in
 * integers, scaled and summed in binary32), SwiGLU, Q8_0 of h, down rows,
 * and y = sum_j w_j o_j + o_shared.  Tokens are independent: OpenMP over
 * tokens.
 */
#include <immintrin.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define QK 32
#define Q4B 18

typedef struct {
    int H, F, E, k, S;
    const float* w_router;  /* [E][H] */
    const float* bias;      /* [E] or NULL */
    const uint8_t* w_gate;  /* [E][F][H/32][18] */
    const uint8_t* w_up;
    const uint8_t* w_down;  /* [E][H][F/32][18] */
    const uint8_t* sh_gate;
    const uint8_t* sh_up;
    const uint8_t* sh_down;
} simd_layer;

static float half_to_float(uint16_t h) { return _cvtsh_ss(h); }
static uint16_t float_to_half(float f) { return _cvtss_sh(f, _MM_FROUND_TO_NEAREST_INT | _MM_FROUND_NO_EXC); }

/* Q8_0 of n values (n a multiple of 32): codes q, binary16 scale bits d. */
static void quantize_q8_0(const float* x, int n, int8_t* q, uint16_t* d) {
    for (int b = 0; b < n / QK; ++b) {
        const float* v = x + b * QK;
        float amax = 0.0f;
        for (int i = 0; i < QK; ++i) amax = fmaxf(amax, fabsf(v[i]));
        const float s = amax / 127.0f;
        d[b] = float_to_half(s);
        for (int i = 0; i < QK; ++i) {
            int r = 0;
            if (s != 0.0f) {
                const float t = v[i] / s;
                const float tr = truncf(t);
                r = (int)tr;
                if (fabsf(t - tr) >= 0.5f) r += (t < 0.0f) ? -1 : 1;
                r = r < -127 ? -127 : (r > 127 ? 127 : r);
            }
            q[b * QK + i] = (int8_t)r;
        }
    }
}

/* sum_i nib_i * q_i over one block (nibbles unsigned 0..15) and sum_i q_i. */
static inline int block_dot_u(const uint8_t* blk, const int8_t* q, int qsum) {
    const __m128i qs = _mm_loadu_si128((const __m128i*)(blk + 2));
    const __m128i lo = _mm_and_si128(qs, _mm_set1_epi8(0x0f));
    const __m128i hi = _mm_and_si128(_mm_srli_epi16(qs, 4), _mm_set1_epi8(0x0f));
    const __m256i w = _mm256_set_m128i(hi, lo);  /* weights 0..15 then 16..31 */
    const __m256i a = _mm256_loadu_si256((const __m256i*)q);
#if defined(__AVXVNNI__)
    __m256i acc = _mm256_dpbusd_avx_epi32(_mm256_setzero_si256(), w, a);
#elif defined(__AVX512VNNI__) && defined(__AVX512VL__)
    __m256i acc = _mm256_dpbusd_epi32(_mm256_setzero_si256(), w, a);
#else
    const __m256i p16 = _mm256_maddubs_epi16(w, a);  /* |pair| <= 2*15*127: no saturation */
    __m256i acc = _mm256_madd_epi16(p16, _mm256_set1_epi16(1));
#endif
    __m128i s = _mm_add_epi32(_mm256_castsi256_si128(acc), _mm256_extracti128_si256(acc, 1));
    s = _mm_add_epi32(s, _mm_shuffle_epi32(s, 0x4e));
    s = _mm_add_epi32(s, _mm_shuffle_epi32(s, 0xb1));
    return _mm_cvtsi128_si32(s) - 8 * qsum;
}

/* Exact per-block integer dot products of n blocks (test export). */
void simd_block_dots(const uint8_t* w, const int8_t* qa, int64_t n, int32_t* out) {
    for (int64_t i = 0; i < n; ++i) {
        int qsum = 0;
        for (int j = 0; j < QK; ++j) qsum += qa[i * QK + j];
        out[i] = block_dot_u(w + i * Q4B, qa + i * QK, qsum);
    }
}

/* out[r] = sum_b dW[r,b] * dA[b] * I_{r,b} for R rows of nb blocks. */
static void q4_rows(const uint8_t* W, int R, int nb, const int8_t* qa, const float* dA, const int* qsum, float* out) {
    for (int r = 0; r < R; ++r) {
        const uint8_t* row = W + (size_t)r * nb * Q4B;
        float acc = 0.0f;
        for (int b = 0; b < nb; ++b) {
            const uint8_t* blk = row + b * Q4B;
            uint16_t db;
            memcpy(&db, blk, 2);
            acc += (float)block_dot_u(blk, qa + b * QK, qsum[b]) * (half_to_float(db) * dA[b]);
        }
        out[r] = acc;
    }
}

static void block_sums(const int8_t* q, int nb, int* s) {
    for (int b = 0; b < nb; ++b) {
        int t = 0;
        for (int i = 0; i < QK; ++i) t += q[b * QK + i];
        s[b] = t;
    }
}

int simd_moe_forward(const simd_layer* L, const float* x, int64_t T, float* y) {
    const int H = L->H, F = L->F, E = L->E, k = L->k, S = L->S;
    const int nbH = H / QK, nbF = F / QK;
    if (k < 1 || k > E || k > 16 || H % 256 || F % 256) return -1;
#pragma omp parallel
    {
        float* logits = malloc(sizeof(float) * E);
        int8_t* qa = malloc(H);
        uint16_t* da16 = malloc(2 * nbH);
        float* dA = malloc(sizeof(float) * nbH);
        int* qs = malloc(sizeof(int) * nbH);
        float* g = malloc(sizeof(float) * F);
        float* u = malloc(sizeof(float) * F);
        float* h = malloc(sizeof(float) * F);
        int8_t* hq = malloc(F);
        uint16_t* dh16 = malloc(2 * nbF);
        float* dH = malloc(sizeof(float) * nbF);
        int* hs = malloc(sizeof(int) * nbF);
        float* o = malloc(sizeof(float) * H);
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < T; ++t) {
            const float* xt = x + t * H;
            float* yt = y + t * H;
            /* router */
            for (int e = 0; e < E; ++e) {
                const float* wr = L->w_router + (size_t)e * H;
                __m256 a8 = _mm256_setzero_ps();
                for (int i = 0; i < H; i += 8) a8 = _mm256_fmadd_ps(_mm256_loadu_ps(wr + i), _mm256_loadu_ps(xt + i), a8);
                __m128 s4 = _mm_add_ps(_mm256_castps256_ps128(a8), _mm256_extractf128_ps(a8, 1));
                s4 = _mm_add_ps(s4, _mm_movehl_ps(s4, s4));
                s4 = _mm_add_ss(s4, _mm_movehdup_ps(s4));
                logits[e] = _mm_cvtss_f32(s4) + (L->bias ? L->bias[e] : 0.0f);
            }
            int idx[16];
            float wsel[16];
            unsigned char taken[256] = {0};
            for (int j = 0; j < k; ++j) {
                int be = -1;
                for (int e = 0; e < E; ++e)
                    if (!taken[e] && (be < 0 || logits[e] > logits[be])) be = e;
                taken[be] = 1;
                idx[j] = be;
            }
            float z = 0.0f;
            for (int j = 0; j < k; ++j) {
                wsel[j] = expf(logits[idx[j]] - logits[idx[0]]);
                z += wsel[j];
            }
            for (int j = 0; j < k; ++j) wsel[j] /= z;
            /* Q8_0 of x */
            quantize_q8_0(xt, H, qa, da16);
            for (int b = 0; b < nbH; ++b) dA[b] = half_to_float(da16[b]);
            block_sums(qa, nbH, qs);
            for (int i = 0; i < H; ++i) yt[i] = 0.0f;
            for (int j = 0; j < k + S; ++j) {
                const int sh = j == k;
                const size_t gs = (size_t)F * nbH * Q4B, ds = (size_t)H * nbF * Q4B;
                const uint8_t* Wg = sh ? L->sh_gate : L->w_gate + idx[j] * gs;
                const uint8_t* Wu = sh ? L->sh_up : L->w_up + idx[j] * gs;
                const uint8_t* Wd = sh ? L->sh_down : L->w_down + idx[j] * ds;
                q4_rows(Wg, F, nbH, qa, dA, qs, g);
                q4_rows(Wu, F, nbH, qa, dA, qs, u);
                for (int i = 0; i < F; ++i) h[i] = g[i] / (1.0f + expf(-g[i])) * u[i];
                quantize_q8_0(h, F, hq, dh16);
                for (int b = 0; b < nbF; ++b) dH[b] = half_to_float(dh16[b]);
                block_sums(hq, nbF, hs);
                q4_rows(Wd, H, nbF, hq, dH, hs, o);
                const float wj = sh ? 1.0f : wsel[j];
                for (int i = 0; i < H; ++i) yt[i] += wj * o[i];
            }
        }
        free(logits); free(qa); free(da16); free(dA); free(qs); free(g); free(u); free(h);
        free(hq); free(dh16); free(dH); free(hs); free(o);
    }
    return 0;
}

int simd_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}
