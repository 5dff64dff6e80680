/*
 * oracle.c -- plain, slow, single-threaded CPU restatement of the BitLinear
 * forward pass (BitNet b1.58 / Sparse-BitNet).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file.  Only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or constant
 * generator with the CUDA library; the packed layouts below are re-derived
 * here from their written definition.
 *
 * Sources (web pages, cited by title and section):
 *  [b158]  "BitNet 1-Bit LLM" blog (youngju.dev), section "BitNet b1.58:
 *          Absmean quantization function" -- weight_quant_ternary,
 *          activation_quant, BitLinear_b158.forward.
 *  [2B4T]  "BitNet b1.58 2B4T Technical Report" summary (greeksharifa),
 *          section 2 Architecture (absmean ternary weights, per-token absmax
 *          8-bit activations) and section 5.1 GPU Inference (four ternary
 *          values packed per byte).
 *  [I2S]   "BitNet 1-Bit LLM" blog, section "bitnet.cpp inference framework /
 *          Architecture overview": I2_S code map -1 -> 00, 0 -> 01, +1 -> 10,
 *          sixteen weights per 32-bit word.
 *  [SBN]   "Sparse-BitNet" review (manon006.tistory.com), section 3.2 (mask
 *          from master-weight magnitude, top-N per block of M, quant then
 *          mask) and section 4 (6:8 main pattern, 2:4 and N:8 sweep).
 *
 * Readings taken where the pages are silent or inconsistent (each is also
 * listed in the design notes):
 *  - Q_b is a parameter.  The product uses 127 for both quantisation and
 *    dequantisation; [b158] prints 2**(bits-1) = 128.
 *  - eps = 1e-5 is added to the scale only in the divisor ([b158]).
 *  - Rounding is round-half-to-even (torch.round), evaluated in fp32 for the
 *    code decisions: r = RN(v * Qb) / RN(scale + eps).
 *  - alpha = mean |W| over the whole matrix, summed in fp64 in row-major
 *    order, divided in fp64, then rounded once to fp32.
 *  - y = acc * alpha * gamma / Qb evaluated in fp64, rounded once to bf16
 *    (round-half-to-even).
 *  - N:M blocks are M consecutive positions along K inside one output row;
 *    ties in |W| go to the lower position; the mask is applied after
 *    ternarisation; alpha comes from the dense latent matrix.
 *  - RMSNorm before the activation quantisation ([b158] BitLinear_b158.forward
 *    normalises x first; nn.RMSNorm with a per-feature weight g): the mean of
 *    x^2 is summed in fp64 and rounded once to fp32 (ms); the reciprocal root
 *    r = 1 / sqrt(ms + eps) is evaluated in fp64 and rounded once to fp32;
 *    xn = RN(RN(x * r) * g) in fp32 and is not rounded to bf16 before the
 *    quantisation.  eps is a parameter (the page's nn.RMSNorm leaves it to
 *    the dtype's default).
 *
 *  - H-BitLinear ("BitNet v2" page of brain.hanbit.co.kr, the paragraphs on
 *    the H-BitLinear module and on native 4-bit activations: an online
 *    Hadamard transform of the activations, then 4-bit activation
 *    quantisation, then the ternary linear map).  The pages give neither the
 *    transform's size, normalisation or evaluation order nor the 4-bit
 *    quantiser, so: the Sylvester-order Walsh-Hadamard matrix of size B = the
 *    largest power of two dividing K, applied to each of the K / B blocks of
 *    a row; evaluated in fp32 by the in-place fast transform (stages
 *    h = 1, 2, 4, ..., B/2, each pair (j, j + h) with bit h of j clear becomes
 *    (a + b, a - b), one fp32 rounding per sum), then scaled by one fp32
 *    multiply with RN32(1 / sqrt(B)) so the transform is orthonormal; 4-bit
 *    codes by the absmax formula with Q_b = 7 clamped to [-8, 7]; the weights
 *    are the ternary matrix of the rotated-basis latent weights (the
 *    transform is not applied to them at run time).
 *
 * Build: gcc -O2 -std=gnu11 -fPIC -shared -pthread -ffp-contract=off -fno-fast-math
 */
#include <fenv.h>
#include <math.h>
#include <pthread.h>
#include <unistd.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_EPS 1e-5f

/* ------------------------------------------------------------------------ */
/* bf16 helpers (bit patterns held in uint16_t)                              */
/* ------------------------------------------------------------------------ */

/* bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits. */
static float orc_bf16_to_f32(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a double once to the nearest bf16 (ties to even).  bf16 keeps 8
 * significant bits; below 2^-126 the spacing is fixed at 2^-133. */
uint16_t orc_bf16_from_f64(double d) {
    if (d == 0.0) return signbit(d) ? 0x8000u : 0x0000u;
    if (isnan(d)) return 0x7FC0u;
    int sign = d < 0.0;
    double a = fabs(d);
    int e;
    (void)frexp(a, &e);           /* a = m * 2^e, m in [0.5, 1) */
    int qexp = e - 8;             /* spacing of 8-bit significands in [2^(e-1), 2^e) */
    if (qexp < -133) qexp = -133; /* subnormal bf16 spacing */
    double r = nearbyint(ldexp(a, -qexp)); /* exact scaling, then RNE */
    double v = ldexp(r, qexp);
    float f = (float)v;           /* exact: v has <= 8 significant bits */
    if (isinf(f) || v > 3.3895313892515355e38) f = INFINITY;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint16_t out = (uint16_t)(u >> 16);
    if (sign) out |= 0x8000u;
    return out;
}

/* ------------------------------------------------------------------------ */
/* Weight quantisation ([b158] weight_quant_ternary, [2B4T] sec. 2)          */
/* ------------------------------------------------------------------------ */

/* alpha = mean |W| over all count entries: fp64 sum in storage order. */
float orc_absmean(const float* W, int64_t count) {
    double s = 0.0;
    for (int64_t i = 0; i < count; ++i) s += fabs((double)W[i]);
    return (float)(s / (double)count);
}

/* W_t = clamp(round(W / (alpha + eps)), -1, 1), fp32 division, RNE. */
void orc_ternarize(const float* W, int64_t count, float alpha, int8_t* Wt) {
    fesetround(FE_TONEAREST);
    volatile float d = alpha + ORC_EPS;
    for (int64_t i = 0; i < count; ++i) {
        volatile float r = W[i] / d;
        float q = nearbyintf(r);
        if (q > 1.0f) q = 1.0f;
        if (q < -1.0f) q = -1.0f;
        Wt[i] = (int8_t)q;
    }
}

/* ------------------------------------------------------------------------ */
/* N:M magnitude mask ([SBN] sec. 3.2)                                       */
/* ------------------------------------------------------------------------ */

/* For every block of m consecutive k inside a row, keep the n entries with
 * the largest |W|; ties go to the lower k.  K must be a multiple of m.
 * mask[i] = 1 if kept.  The ranking is a stable insertion sort of the block
 * by decreasing |W|. */
void orc_nm_mask(const float* W, int N, int K, int n, int m, uint8_t* mask) {
    int idx[64];
    for (int r = 0; r < N; ++r) {
        for (int b = 0; b < K / m; ++b) {
            const float* w = W + (int64_t)r * K + (int64_t)b * m;
            for (int j = 0; j < m; ++j) idx[j] = j;
            for (int j = 1; j < m; ++j) { /* stable: only strictly larger moves up */
                int cur = idx[j];
                int t = j - 1;
                while (t >= 0 && fabsf(w[idx[t]]) < fabsf(w[cur])) {
                    idx[t + 1] = idx[t];
                    --t;
                }
                idx[t + 1] = cur;
            }
            uint8_t* mk = mask + (int64_t)r * K + (int64_t)b * m;
            for (int j = 0; j < m; ++j) mk[j] = 0;
            for (int j = 0; j < n; ++j) mk[idx[j]] = 1;
        }
    }
}

/* Quant-then-mask: W_eff = W_t * mask. */
void orc_apply_mask(int8_t* Wt, const uint8_t* mask, int64_t count) {
    for (int64_t i = 0; i < count; ++i)
        if (!mask[i]) Wt[i] = 0;
}

/* ------------------------------------------------------------------------ */
/* Packed layouts ([2B4T] sec. 5.1, [I2S])                                   */
/*                                                                          */
/* Dense: code = W_t + 1 (00 = -1, 01 = 0, 10 = +1; 11 unused).  Row r takes */
/* ld = 16 * ceil(K / 64) bytes; weight k sits in byte k / 4 at bits          */
/* 2*(k % 4) .. 2*(k % 4) + 1 (first weight in the least significant bits),  */
/* so one 32-bit little-endian word carries sixteen consecutive weights.     */
/* Unused tail positions of a row hold code 01.                              */
/*                                                                          */
/* N:M (2:4, or n:8 with 1 <= n <= 7; K a multiple of m):                    */
/*  values: the n kept codes of every block, in increasing k, blocks in      */
/*          order, 2 bits each as above; row stride 16*ceil(K*n/m / 64)      */
/*          bytes, unused tail codes 01.                                     */
/*  meta 2:4: per block a nibble i0 | i1 << 2 (kept positions, i0 < i1);     */
/*          block b in byte b / 2, low nibble first.                         */
/*  meta n:8: per block one byte, bit j set when position j is kept.         */
/*  meta row stride 16 * ceil(K / 128) bytes, unused bytes 0.                */
/* ------------------------------------------------------------------------ */

int64_t orc_dense_ld(int K) { return 16 * (int64_t)((K + 63) / 64); }

int64_t orc_nm_values_ld(int K, int n, int m) {
    int64_t kept = (int64_t)K / m * n;
    return 16 * ((kept + 63) / 64);
}

int64_t orc_nm_meta_ld(int K) { return 16 * (int64_t)((K + 127) / 128); }

static void orc_put_code(uint8_t* row, int64_t pos, int code) {
    row[pos / 4] = (uint8_t)((row[pos / 4] & ~(3u << (2 * (pos % 4)))) | ((unsigned)code << (2 * (pos % 4))));
}

static int orc_get_code(const uint8_t* row, int64_t pos) {
    return (row[pos / 4] >> (2 * (pos % 4))) & 3;
}

void orc_pack_dense(const int8_t* Wt, int N, int K, uint8_t* codes) {
    int64_t ld = orc_dense_ld(K);
    for (int r = 0; r < N; ++r) {
        uint8_t* row = codes + (int64_t)r * ld;
        memset(row, 0x55, (size_t)ld); /* every position starts as code 01 */
        for (int k = 0; k < K; ++k) orc_put_code(row, k, Wt[(int64_t)r * K + k] + 1);
    }
}

void orc_unpack_dense(const uint8_t* codes, int N, int K, int8_t* Wt) {
    int64_t ld = orc_dense_ld(K);
    for (int r = 0; r < N; ++r)
        for (int k = 0; k < K; ++k)
            Wt[(int64_t)r * K + k] = (int8_t)(orc_get_code(codes + (int64_t)r * ld, k) - 1);
}

/* Returns 0 on success, -1 for an unsupported pattern or K. */
int orc_pack_nm(const int8_t* Wt, const uint8_t* mask, int N, int K, int n, int m,
                uint8_t* values, uint8_t* meta) {
    if (!((n == 2 && m == 4) || (m == 8 && n >= 1 && n <= 7)) || K % m != 0) return -1;
    int64_t ldv = orc_nm_values_ld(K, n, m), ldm = orc_nm_meta_ld(K);
    for (int r = 0; r < N; ++r) {
        uint8_t* vrow = values + (int64_t)r * ldv;
        uint8_t* mrow = meta + (int64_t)r * ldm;
        memset(vrow, 0x55, (size_t)ldv);
        memset(mrow, 0x00, (size_t)ldm);
        int64_t out = 0;
        for (int b = 0; b < K / m; ++b) {
            int kept_pos[8], nk = 0;
            for (int j = 0; j < m; ++j) {
                int64_t i = (int64_t)r * K + (int64_t)b * m + j;
                if (mask[i]) {
                    kept_pos[nk++] = j;
                    orc_put_code(vrow, out++, Wt[i] + 1);
                }
            }
            if (nk != n) return -1;
            if (m == 4) {
                unsigned nib = (unsigned)kept_pos[0] | ((unsigned)kept_pos[1] << 2);
                mrow[b / 2] |= (uint8_t)(nib << (4 * (b % 2)));
            } else {
                unsigned bits = 0;
                for (int j = 0; j < nk; ++j) bits |= 1u << kept_pos[j];
                mrow[b] = (uint8_t)bits;
            }
        }
    }
    return 0;
}

/* Expands the compressed form back to a dense ternary matrix (pruned = 0). */
int orc_unpack_nm(const uint8_t* values, const uint8_t* meta, int N, int K, int n, int m, int8_t* Wt) {
    if (!((n == 2 && m == 4) || (m == 8 && n >= 1 && n <= 7)) || K % m != 0) return -1;
    int64_t ldv = orc_nm_values_ld(K, n, m), ldm = orc_nm_meta_ld(K);
    for (int r = 0; r < N; ++r) {
        const uint8_t* vrow = values + (int64_t)r * ldv;
        const uint8_t* mrow = meta + (int64_t)r * ldm;
        int64_t in = 0;
        for (int b = 0; b < K / m; ++b) {
            int8_t* w = Wt + (int64_t)r * K + (int64_t)b * m;
            for (int j = 0; j < m; ++j) w[j] = 0;
            if (m == 4) {
                unsigned nib = (mrow[b / 2] >> (4 * (b % 2))) & 0xF;
                int i0 = nib & 3, i1 = (nib >> 2) & 3;
                w[i0] = (int8_t)(orc_get_code(vrow, in++) - 1);
                w[i1] = (int8_t)(orc_get_code(vrow, in++) - 1);
            } else {
                for (int j = 0; j < 8; ++j)
                    if ((mrow[b] >> j) & 1) w[j] = (int8_t)(orc_get_code(vrow, in++) - 1);
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Activation quantisation ([b158] activation_quant, per token)              */
/* ------------------------------------------------------------------------ */

/* gamma_m = max_k |x_mk|; q = clamp(round(RN(x * Qb) / RN(gamma + eps)),
 * -128, 127) (the int8 range; with Qb = 127 the codes stay in [-127, 127]);
 * rowsum_m = sum_k q (may be NULL). */
void orc_quant_act(const uint16_t* x, int M, int K, int Qb, int8_t* q, float* gamma, int32_t* rowsum) {
    fesetround(FE_TONEAREST);
    for (int r = 0; r < M; ++r) {
        const uint16_t* xr = x + (int64_t)r * K;
        float g = 0.0f;
        for (int k = 0; k < K; ++k) {
            float a = fabsf(orc_bf16_to_f32(xr[k]));
            if (a > g) g = a;
        }
        gamma[r] = g;
        volatile float d = g + ORC_EPS;
        int64_t s = 0;
        for (int k = 0; k < K; ++k) {
            volatile float t = orc_bf16_to_f32(xr[k]) * (float)Qb;
            volatile float v = t / d;
            float c = nearbyintf(v);
            if (c > 127.0f) c = 127.0f;
            if (c < -128.0f) c = -128.0f;
            q[(int64_t)r * K + k] = (int8_t)c;
            s += (int64_t)c;
        }
        if (rowsum) rowsum[r] = (int32_t)s;
    }
}

/* ------------------------------------------------------------------------ */
/* RMSNorm, then activation quantisation ([b158] BitLinear_b158.forward:      */
/* x = self.norm(x) before activation_quant)                                  */
/* ------------------------------------------------------------------------ */

/* xn[m][k] = RN(RN(x[m][k] * r_m) * g[k]) with r_m = RN32(1 / sqrt(ms_m + eps))
 * (fp64), ms_m = RN32(sum_k x[m][k]^2 / K) (fp64 sum in index order). */
void orc_rmsnorm(const uint16_t* x, const float* g, int M, int K, float eps, float* xn) {
    fesetround(FE_TONEAREST);
    for (int r = 0; r < M; ++r) {
        const uint16_t* xr = x + (int64_t)r * K;
        double ss = 0.0;
        for (int k = 0; k < K; ++k) {
            const double v = (double)orc_bf16_to_f32(xr[k]);
            ss += v * v;
        }
        const float ms = (float)(ss / (double)K);
        const float rr = (float)(1.0 / sqrt((double)ms + (double)eps));
        for (int k = 0; k < K; ++k) {
            volatile float a = orc_bf16_to_f32(xr[k]) * rr;
            volatile float b = a * g[k];
            xn[(int64_t)r * K + k] = b;
        }
    }
}

/* Activation quantisation of fp32 rows: gamma = max |xn|,
 * q = clamp(rne(RN(xn * Qb) / RN(gamma + eps)), -128, 127). */
void orc_quant_act_f32(const float* xn, int M, int K, int Qb, int8_t* q, float* gamma, int32_t* rowsum) {
    fesetround(FE_TONEAREST);
    for (int r = 0; r < M; ++r) {
        const float* xr = xn + (int64_t)r * K;
        float g = 0.0f;
        for (int k = 0; k < K; ++k) {
            float a = fabsf(xr[k]);
            if (a > g) g = a;
        }
        gamma[r] = g;
        volatile float d = g + ORC_EPS;
        int64_t s = 0;
        for (int k = 0; k < K; ++k) {
            volatile float t = xr[k] * (float)Qb;
            volatile float v = t / d;
            float c = nearbyintf(v);
            if (c > 127.0f) c = 127.0f;
            if (c < -128.0f) c = -128.0f;
            q[(int64_t)r * K + k] = (int8_t)c;
            s += (int64_t)c;
        }
        if (rowsum) rowsum[r] = (int32_t)s;
    }
}

/* ------------------------------------------------------------------------ */
/* Integer contraction and dequantisation ([b158] BitLinear_b158.forward)    */
/* ------------------------------------------------------------------------ */

/* acc[m][n] = sum_k q[m][k] * Wt[n][k].  Returns -1 if a sum leaves int32. */
int orc_matmul_i32(const int8_t* q, const int8_t* Wt, int M, int N, int K, int32_t* acc) {
    int bad = 0;
    for (int i = 0; i < M; ++i)
        for (int j = 0; j < N; ++j) {
            int64_t s = 0;
            const int8_t* a = q + (int64_t)i * K;
            const int8_t* w = Wt + (int64_t)j * K;
            for (int k = 0; k < K; ++k) s += (int64_t)a[k] * (int64_t)w[k];
            if (s > INT32_MAX || s < INT32_MIN) bad = 1;
            acc[(int64_t)i * N + j] = (int32_t)s;
        }
    return bad ? -1 : 0;
}

/* The same contraction spread over nthreads POSIX threads, each running the
 * loop above on its own band of output columns j (no other change: the
 * timed all-cores baseline of the benchmark, not a second definition).
 * Returns -1 if a sum leaves int32 or a thread cannot be started. */
typedef struct {
    const int8_t* q;
    const int8_t* Wt;
    int M, N, K, j0, j1, bad;
    int32_t* acc;
} orc_band;

static void* orc_band_run(void* arg) {
    orc_band* b = (orc_band*)arg;
    for (int i = 0; i < b->M; ++i)
        for (int j = b->j0; j < b->j1; ++j) {
            int64_t s = 0;
            const int8_t* a = b->q + (int64_t)i * b->K;
            const int8_t* w = b->Wt + (int64_t)j * b->K;
            for (int k = 0; k < b->K; ++k) s += (int64_t)a[k] * (int64_t)w[k];
            if (s > INT32_MAX || s < INT32_MIN) b->bad = 1;
            b->acc[(int64_t)i * b->N + j] = (int32_t)s;
        }
    return NULL;
}

int orc_matmul_i32_threads(const int8_t* q, const int8_t* Wt, int M, int N, int K, int32_t* acc, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > N) nthreads = N;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    orc_band* bands = (orc_band*)malloc(sizeof(orc_band) * (size_t)nthreads);
    if (!th || !bands) {
        free(th);
        free(bands);
        return -1;
    }
    int started = 0, bad = 0;
    for (int t = 0; t < nthreads; ++t) {
        orc_band* b = &bands[t];
        b->q = q; b->Wt = Wt; b->M = M; b->N = N; b->K = K; b->acc = acc; b->bad = 0;
        b->j0 = (int)((int64_t)N * t / nthreads);
        b->j1 = (int)((int64_t)N * (t + 1) / nthreads);
        if (pthread_create(&th[t], NULL, orc_band_run, b) != 0) {
            bad = 1;
            break;
        }
        ++started;
    }
    for (int t = 0; t < started; ++t) {
        pthread_join(th[t], NULL);
        bad |= bands[t].bad;
    }
    free(th);
    free(bands);
    return bad ? -1 : 0;
}

/* Number of host threads the system reports online. */
int orc_online_cpus(void) { return (int)sysconf(_SC_NPROCESSORS_ONLN); }

/* y = acc * alpha * gamma_m / Qb in fp64, rounded once to bf16. */
void orc_dequant(const int32_t* acc, const float* gamma, float alpha, int M, int N, int Qb, uint16_t* y) {
    for (int i = 0; i < M; ++i)
        for (int j = 0; j < N; ++j) {
            double v = (double)acc[(int64_t)i * N + j] * (double)alpha * (double)gamma[i] / (double)Qb;
            y[(int64_t)i * N + j] = orc_bf16_from_f64(v);
        }
}

/* Squared-ReLU gate of the FFN pair.  BitNet b1.58 2B4T technical report
 * summary (greeksharifa.github.io page), section 2 "Architecture": the FFN
 * sublayer uses squared ReLU, the rectified activation squared.  With the
 * block's gate and up projections (both BitLinears of the same x, outputs g
 * and u in bf16), the reading taken here is h = ReLU(g)^2 * u elementwise,
 * every bf16 operation rounded once: sq = RN_bf16(max(g, 0)^2), then
 * h = RN_bf16(sq * u).  Both products are exact in double (8-bit significands),
 * so each line rounds exactly once. */
void orc_relu2_glu(const uint16_t* g, const uint16_t* u, int64_t count, uint16_t* h) {
    for (int64_t i = 0; i < count; ++i) {
        double gv = (double)orc_bf16_to_f32(g[i]);
        double r = gv > 0.0 ? gv : 0.0;
        uint16_t sq = orc_bf16_from_f64(r * r);
        h[i] = orc_bf16_from_f64((double)orc_bf16_to_f32(sq) * (double)orc_bf16_to_f32(u[i]));
    }
}

/* Whole forward for a dense ternary matrix: quantise activations, contract,
 * dequantise.  q_out/acc_out/gamma_out may be NULL.  Returns 0 or -1. */
int orc_forward(const uint16_t* x, int M, int K, const int8_t* Wt, int N, float alpha, int Qb,
                uint16_t* y, int8_t* q_out, int32_t* acc_out, float* gamma_out) {
    int8_t* q = q_out ? q_out : (int8_t*)malloc((size_t)M * (size_t)K);
    int32_t* acc = acc_out ? acc_out : (int32_t*)malloc((size_t)M * (size_t)N * sizeof(int32_t));
    float* g = gamma_out ? gamma_out : (float*)malloc((size_t)M * sizeof(float));
    int rc = -1;
    if (q && acc && g) {
        orc_quant_act(x, M, K, Qb, q, g, NULL);
        rc = orc_matmul_i32(q, Wt, M, N, K, acc);
        orc_dequant(acc, g, alpha, M, N, Qb, y);
    }
    if (!q_out) free(q);
    if (!acc_out) free(acc);
    if (!gamma_out) free(g);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* H-BitLinear: online Hadamard transform, 4-bit activations ("BitNet v2"   */
/* page, brain.hanbit.co.kr: the H-BitLinear and native 4-bit paragraphs)   */
/* ------------------------------------------------------------------------ */

/* Largest power of two that divides K (1 for odd K). */
int orc_hadamard_block(int K) {
    int b = 1;
    while (K % (2 * b) == 0) b *= 2;
    return b;
}

/* xh = RN32(1 / sqrt(B)) * H_B x on every B-block of every bf16 row, with the
 * unnormalised transform formed by the in-place fast Walsh-Hadamard butterflies
 * in fp32 (stage h = 1, 2, ..., B/2: (a, b) -> (a + b, a - b) for j with
 * bit h clear and its partner j + h). */
void orc_hadamard_rows(const uint16_t* x, int M, int K, int B, float* xh) {
    fesetround(FE_TONEAREST);
    const float scale = (float)(1.0 / sqrt((double)B));
    for (int r = 0; r < M; ++r) {
        float* row = xh + (int64_t)r * K;
        for (int k = 0; k < K; ++k) row[k] = orc_bf16_to_f32(x[(int64_t)r * K + k]);
        for (int b0 = 0; b0 < K; b0 += B) {
            float* v = row + b0;
            for (int h = 1; h < B; h *= 2)
                for (int j = 0; j < B; ++j)
                    if ((j & h) == 0) {
                        volatile float a = v[j], b = v[j + h];
                        volatile float s = a + b, d = a - b;
                        v[j] = s;
                        v[j + h] = d;
                    }
            for (int j = 0; j < B; ++j) {
                volatile float t = v[j] * scale;
                v[j] = t;
            }
        }
    }
}

/* 4-bit activation codes of fp32 rows: gamma = max |xh|,
 * q = clamp(rne(RN(xh * 7) / RN(gamma + eps)), -8, 7). */
void orc_quant_act4(const float* xh, int M, int K, int8_t* q, float* gamma, int32_t* rowsum) {
    fesetround(FE_TONEAREST);
    for (int r = 0; r < M; ++r) {
        const float* xr = xh + (int64_t)r * K;
        float g = 0.0f;
        for (int k = 0; k < K; ++k) {
            float a = fabsf(xr[k]);
            if (a > g) g = a;
        }
        gamma[r] = g;
        volatile float d = g + ORC_EPS;
        int64_t s = 0;
        for (int k = 0; k < K; ++k) {
            volatile float t = xr[k] * 7.0f;
            volatile float v = t / d;
            float c = nearbyintf(v);
            if (c > 7.0f) c = 7.0f;
            if (c < -8.0f) c = -8.0f;
            q[(int64_t)r * K + k] = (int8_t)c;
            s += (int64_t)c;
        }
        if (rowsum) rowsum[r] = (int32_t)s;
    }
}

/* H-BitLinear forward: transform, 4-bit codes, contraction with the ternary
 * matrix, y = acc * alpha * gamma / 7 in fp64 rounded once to bf16. */
int orc_forward_hbit(const uint16_t* x, int M, int K, const int8_t* Wt, int N, float alpha, uint16_t* y,
                     int8_t* q_out, int32_t* acc_out, float* gamma_out) {
    float* xh = (float*)malloc((size_t)M * (size_t)K * sizeof(float));
    int8_t* q = q_out ? q_out : (int8_t*)malloc((size_t)M * (size_t)K);
    int32_t* acc = acc_out ? acc_out : (int32_t*)malloc((size_t)M * (size_t)N * sizeof(int32_t));
    float* g = gamma_out ? gamma_out : (float*)malloc((size_t)M * sizeof(float));
    int rc = -1;
    if (xh && q && acc && g) {
        orc_hadamard_rows(x, M, K, orc_hadamard_block(K), xh);
        orc_quant_act4(xh, M, K, q, g, NULL);
        rc = orc_matmul_i32(q, Wt, M, N, K, acc);
        orc_dequant(acc, g, alpha, M, N, 7, y);
    }
    free(xh);
    if (!q_out) free(q);
    if (!acc_out) free(acc);
    if (!gamma_out) free(g);
    return rc;
}
