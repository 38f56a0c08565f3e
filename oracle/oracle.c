/*
 * CPU oracle for quantized video-DiT self-attention.  TEST INFRASTRUCTURE
 * ONLY: the tests, the smoke check and the benchmark's CPU-baseline leg call
 * it; the product library never does.  It shares no code with the CUDA path.
 *
 * Source: page 1 of the TMAP / Taobao Faxiang image-to-video write-up
 * (ai.aiking123.com/155823.html), section "Attention performance
 * optimisation": the op replaced is aten.scaled_dot_product_flash_attention
 * (73.76% of DiT FLOPs, "Background"); it is swapped for the SageAttention
 * operator ("attention quantization"); an all-zero channel made the
 * per-channel quantization coefficient divide by zero and produced NaN, which
 * was fixed ("operator details"); some layers stay at original precision
 * ("keeping video quality").  The step-by-step scheme the pages leave open is
 * taken in its plainest reading:
 *
 *   O1  exact attention  O = softmax(Q K^T / sqrt(d)) V, in fp64.
 *   O2  scalar emulation of the quantized scheme:
 *       a1 K channel mean over real tokens (fp64 sums per 128-token tile in
 *          ascending token order, tile partials in ascending order, / N in
 *          fp64, rounded to fp32);
 *       a2 Ks = fp32(K) - mean (fp32); per 128-token block amax = max|Ks|,
 *          k_scale = amax / 127, code = clamp(rne(Ks * (127 / amax)), +-127),
 *          amax == 0 -> scale 0 and codes 0 (the zero-scale guard);
 *       a3 the same for Q without smoothing;
 *       a4 per channel amax over tokens of V, v_scale = amax / 448,
 *          code = e4m3_rne_satfinite(V * (448 / amax)), same guard;
 *       a5 S = Q_i8 . K_i8 in exact integers;
 *       a6 s = S * (q_scale * k_scale * (log2(e) / sqrt(d))), keys >= N
 *          masked, online softmax over 128-key tiles in ascending order with
 *          running max m, p = 2^(s - m), row sum l of fp32 p;
 *       a7 P8 = e4m3_rne_satfinite(p * 448);
 *       a8 acc = acc * 2^(m_old - m_new) + sum_j P8_j V8_j   (fp32);
 *       a9 O = acc * v_scale / (448 * l), rounded to bf16.
 *
 * FP8 e4m3 follows the OCP 8-bit floating point specification (v1.0): sign,
 * 4 exponent bits with bias 7, 3 mantissa bits, no infinities, S.1111.111 is
 * NaN, largest finite 448, smallest normal 2^-6, subnormals m * 2^-9.
 *
 * Every floating-point step is written with explicit float / double types and
 * compiled with -ffp-contract=off so no multiply-add is fused.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_TILE 128

static inline float bf16f(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static inline uint16_t f32_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* Round to nearest integer, ties to even, of a finite double. */
static inline double rne(double x) {
    double f = floor(x);
    double r = x - f;
    if (r > 0.5) return f + 1.0;
    if (r < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* ---------------- FP8 e4m3 (OCP) ---------------- */

double orc_e4m3_decode(uint8_t x) {
    int s = x >> 7, e = (x >> 3) & 0xF, m = x & 7;
    if (e == 0xF && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round to nearest (ties to even), saturating to +-448; NaN -> 0x7F. */
uint8_t orc_e4m3_encode(float xf) {
    if (isnan(xf)) return 0x7F;
    uint8_t sign = signbit(xf) ? 0x80 : 0x00;
    double a = fabs((double)xf);
    if (a >= 448.0) return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {             /* subnormal grid: multiples of 2^-9 */
        double q = rne(a * 512.0);        /* 0..8; 8 is the smallest normal */
        return sign | (uint8_t)q;
    }
    int e2;
    frexp(a, &e2);                        /* a = f * 2^e2, f in [0.5, 1) */
    int e = e2 - 1;                       /* a in [2^e, 2^(e+1)) */
    double q = rne(ldexp(a, 3 - e));      /* in [8, 16] */
    if (q == 16.0) { q = 8.0; e += 1; }
    if (e + 7 > 15 || (e + 7 == 15 && q - 8.0 > 6.0)) return sign | 0x7E;
    return sign | (uint8_t)(((e + 7) << 3) | (int)(q - 8.0));
}

/* ---------------- a1: K channel mean ---------------- */

/* k: bf16 [B,H,N,d] -> mean fp32 [B,H,d] */
void orc_k_mean(const uint16_t* k, int B, int H, int N, int d, float* mean) {
    long BH = (long)B * H;
#pragma omp parallel for schedule(static)
    for (long bh = 0; bh < BH; ++bh) {
        const uint16_t* kh = k + bh * (long)N * d;
        for (int c = 0; c < d; ++c) {
            double total = 0.0;
            for (int t0 = 0; t0 < N; t0 += ORC_TILE) {
                double part = 0.0;
                int t1 = t0 + ORC_TILE < N ? t0 + ORC_TILE : N;
                for (int n = t0; n < t1; ++n) part += (double)bf16f(kh[(long)n * d + c]);
                total += part;
            }
            mean[bh * d + c] = (float)(total / (double)N);
        }
    }
}

/* ---------------- a2/a3: per-block INT8 ---------------- */

/*
 * Quantizes one tensor x (bf16 [B,H,N,d]) per 128-token block, optionally
 * subtracting a per-(b,h,c) fp32 mean first (mean == NULL: no smoothing).
 * codes: int8 [B,H,N,d] (natural layout); scale: fp32 [B,H,ceil(N/128)].
 */
void orc_quant_int8_blocks(const uint16_t* x, const float* mean, int B, int H, int N, int d,
                           int8_t* codes, float* scale) {
    long BH = (long)B * H;
    int nb = (N + ORC_TILE - 1) / ORC_TILE;
#pragma omp parallel for schedule(static)
    for (long blk = 0; blk < BH * nb; ++blk) {
        long bh = blk / nb;
        int b0 = (int)(blk % nb) * ORC_TILE;
        int b1 = b0 + ORC_TILE < N ? b0 + ORC_TILE : N;
        const uint16_t* xh = x + bh * (long)N * d;
        const float* mh = mean ? mean + bh * d : NULL;
        float amax = 0.0f;
        for (int n = b0; n < b1; ++n)
            for (int c = 0; c < d; ++c) {
                float v = bf16f(xh[(long)n * d + c]);
                if (mh) v = v - mh[c];
                float a = fabsf(v);
                if (a > amax) amax = a;
            }
        int8_t* ch = codes + bh * (long)N * d;
        if (amax == 0.0f) {                 /* zero-scale guard */
            scale[blk] = 0.0f;
            for (int n = b0; n < b1; ++n) memset(ch + (long)n * d, 0, (size_t)d);
            continue;
        }
        float sc = amax / 127.0f;
        float inv = 127.0f / amax;
        scale[blk] = sc;
        for (int n = b0; n < b1; ++n)
            for (int c = 0; c < d; ++c) {
                float v = bf16f(xh[(long)n * d + c]);
                if (mh) v = v - mh[c];
                float t = v * inv;
                double r = rne((double)t);
                if (r > 127.0) r = 127.0;
                if (r < -127.0) r = -127.0;
                ch[(long)n * d + c] = (int8_t)r;
            }
    }
}

/*
 * The same quantization with a block of `rows` consecutive tokens (rows = 1:
 * one scale per token, the finer Q granularity).  codes: int8 [B,H,N,d];
 * scale: fp32 [B,H,ceil(N/rows)].  Same formula and zero guard as above.
 */
void orc_quant_int8_rows(const uint16_t* x, const float* mean, int B, int H, int N, int d, int rows,
                         int8_t* codes, float* scale) {
    long BH = (long)B * H;
    int nb = (N + rows - 1) / rows;
#pragma omp parallel for schedule(static)
    for (long blk = 0; blk < BH * nb; ++blk) {
        long bh = blk / nb;
        int b0 = (int)(blk % nb) * rows;
        int b1 = b0 + rows < N ? b0 + rows : N;
        const uint16_t* xh = x + bh * (long)N * d;
        const float* mh = mean ? mean + bh * d : NULL;
        float amax = 0.0f;
        for (int n = b0; n < b1; ++n)
            for (int c = 0; c < d; ++c) {
                float v = bf16f(xh[(long)n * d + c]);
                if (mh) v = v - mh[c];
                float a = fabsf(v);
                if (a > amax) amax = a;
            }
        int8_t* ch = codes + bh * (long)N * d;
        if (amax == 0.0f) {
            scale[blk] = 0.0f;
            for (int n = b0; n < b1; ++n) memset(ch + (long)n * d, 0, (size_t)d);
            continue;
        }
        float inv = 127.0f / amax;
        scale[blk] = amax / 127.0f;
        for (int n = b0; n < b1; ++n)
            for (int c = 0; c < d; ++c) {
                float v = bf16f(xh[(long)n * d + c]);
                if (mh) v = v - mh[c];
                double r = rne((double)(v * inv));
                if (r > 127.0) r = 127.0;
                if (r < -127.0) r = -127.0;
                ch[(long)n * d + c] = (int8_t)r;
            }
    }
}

/* ---------------- a4: per-channel FP8 V ---------------- */

/* v: bf16 [B,H,N,d] -> codes e4m3 [B,H,N,d] (natural layout), scale fp32 [B,H,d] */
void orc_quant_v_fp8(const uint16_t* v, int B, int H, int N, int d, uint8_t* codes, float* scale) {
    long BH = (long)B * H;
#pragma omp parallel for schedule(static)
    for (long bh = 0; bh < BH; ++bh) {
        const uint16_t* vh = v + bh * (long)N * d;
        uint8_t* ch = codes + bh * (long)N * d;
        for (int c = 0; c < d; ++c) {
            float amax = 0.0f;
            for (int n = 0; n < N; ++n) {
                float a = fabsf(bf16f(vh[(long)n * d + c]));
                if (a > amax) amax = a;
            }
            if (amax == 0.0f) {             /* zero-scale guard */
                scale[bh * d + c] = 0.0f;
                for (int n = 0; n < N; ++n) ch[(long)n * d + c] = 0;
                continue;
            }
            scale[bh * d + c] = amax / 448.0f;
            float inv = 448.0f / amax;
            for (int n = 0; n < N; ++n) {
                float t = bf16f(vh[(long)n * d + c]) * inv;
                ch[(long)n * d + c] = orc_e4m3_encode(t);
            }
        }
    }
}

/* ---------------- a5: integer QK^T tile ---------------- */

/*
 * S[i, j] = sum_c q[qb*128+i, c] * k[kb*128+j, c] for one (bh, qb, kb) tile,
 * with rows/keys beyond N treated as zero (the padding the path uses).
 * q, k: int8 [B*H, N, d]; out: int32 [128, 128].
 */
void orc_qk_tile(const int8_t* q, const int8_t* k, int N, int d, long bh, int qb, int kb, int32_t* out) {
    const int8_t* qh = q + bh * (long)N * d;
    const int8_t* kh = k + bh * (long)N * d;
    for (int i = 0; i < ORC_TILE; ++i)
        for (int j = 0; j < ORC_TILE; ++j) {
            int qi = qb * ORC_TILE + i, kj = kb * ORC_TILE + j;
            int64_t acc = 0;
            if (qi < N && kj < N)
                for (int c = 0; c < d; ++c) acc += (int64_t)qh[(long)qi * d + c] * (int64_t)kh[(long)kj * d + c];
            out[i * ORC_TILE + j] = (int32_t)acc;
        }
}

/* ---------------- O1: exact attention (fp64) ---------------- */

/*
 * For each (bh, row) in rows[0..n_rows) over every bh: out[bh][r][c] in fp64,
 * O = softmax(q k^T / sqrt(d)) v computed with a max-shifted two-pass softmax.
 * q, k, v: bf16 [B,H,N,d]; rows: query indices; out: double [B*H, n_rows, d].
 */
void orc_attn_exact(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int H, int N, int d,
                    const int* rows, int n_rows, double* out) {
    long BH = (long)B * H;
    double inv_sqrt_d = 1.0 / sqrt((double)d);
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)N);
        double* qv = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
        for (long w = 0; w < BH * n_rows; ++w) {
            long bh = w / n_rows;
            int i = rows[w % n_rows];
            const uint16_t* qh = q + bh * (long)N * d;
            const uint16_t* kh = k + bh * (long)N * d;
            const uint16_t* vh = v + bh * (long)N * d;
            for (int c = 0; c < d; ++c) qv[c] = (double)bf16f(qh[(long)i * d + c]);
            double m = -INFINITY;
            for (int j = 0; j < N; ++j) {
                double acc = 0.0;
                for (int c = 0; c < d; ++c) acc += qv[c] * (double)bf16f(kh[(long)j * d + c]);
                s[j] = acc * inv_sqrt_d;
                if (s[j] > m) m = s[j];
            }
            double l = 0.0;
            for (int j = 0; j < N; ++j) { s[j] = exp(s[j] - m); l += s[j]; }
            double* o = out + w * d;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            for (int j = 0; j < N; ++j) {
                double p = s[j] / l;
                for (int c = 0; c < d; ++c) o[c] += p * (double)bf16f(vh[(long)j * d + c]);
            }
        }
        free(s);
        free(qv);
    }
}

/* ---------------- O2: scalar emulation of a5..a9 ---------------- */

/*
 * flags: bit 0 keep P in fp32 (skip a7's e4m3 rounding, scale stays 448),
 *        bit 1 use dequantized-exact V (v8 * v_scale replaced by bf16 V; needs v_bf16),
 *        bit 2 use the bf16 Q/K instead of the INT8 codes (needs q_bf16/k_bf16),
 *        bit 3 one key tile spanning all N (no tiling of the online softmax),
 *        bit 4 q_scale holds one scale per query token ([B*H, N]) instead of
 *              one per 128-token block (the finer Q granularity).
 * The bits exist only to pin the emulation against O1 as quantization is
 * switched off step by step.
 *
 * q8: int8 [B*H, N, d]; q_scale [B*H, nQ]; k8 int8 [B*H, N, d]; k_scale [B*H, nK];
 * v8: e4m3 [B*H, N, d]; v_scale [B*H, d]; rows as in orc_attn_exact;
 * out: fp32 [B*H, n_rows, d] (before bf16 rounding) and, if out_bf16 != NULL,
 * the bf16 bits of the same values.
 */
void orc_attn_emul(const int8_t* q8, const float* q_scale, const int8_t* k8, const float* k_scale,
                   const uint8_t* v8, const float* v_scale, int B, int H, int N, int d,
                   const int* rows, int n_rows, int flags,
                   const uint16_t* q_bf16, const uint16_t* k_bf16, const uint16_t* v_bf16,
                   float* out, uint16_t* out_bf16) {
    long BH = (long)B * H;
    int nT = (N + ORC_TILE - 1) / ORC_TILE;
    int tile = (flags & 8) ? N : ORC_TILE;
    int n_kt = (N + tile - 1) / tile;
    /* log2(e) / sqrt(d), formed in fp64 and rounded once to fp32 */
    float c_scale = (float)(1.4426950408889634073599246810019 / sqrt((double)d));
    double v_lut[256];
    for (int i = 0; i < 256; ++i) v_lut[i] = orc_e4m3_decode((uint8_t)i);
#pragma omp parallel
    {
        float* s = (float*)malloc(sizeof(float) * (size_t)tile);
        float* acc = (float*)malloc(sizeof(float) * (size_t)d);
        float* vrow = (float*)malloc(sizeof(float) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
        for (long w = 0; w < BH * n_rows; ++w) {
            long bh = w / n_rows;
            int i = rows[w % n_rows];
            int qb = i / ORC_TILE;
            const int8_t* qh = q8 + bh * (long)N * d;
            const int8_t* kh = k8 + bh * (long)N * d;
            const uint8_t* vh = v8 + bh * (long)N * d;
            float m = -INFINITY, l = 0.0f;
            for (int c = 0; c < d; ++c) acc[c] = 0.0f;
            for (int kt = 0; kt < n_kt; ++kt) {
                int j0 = kt * tile;
                int j1 = j0 + tile < N ? j0 + tile : N;
                float tmax = -INFINITY;
                for (int j = j0; j < j1; ++j) {
                    float sj;
                    if (flags & 4) {
                        double a = 0.0;
                        for (int c = 0; c < d; ++c)
                            a += (double)bf16f(q_bf16[(bh * (long)N + i) * d + c]) *
                                 (double)bf16f(k_bf16[(bh * (long)N + j) * d + c]);
                        sj = (float)a * c_scale;
                    } else {
                        int32_t S = 0;
                        for (int c = 0; c < d; ++c) S += (int32_t)qh[(long)i * d + c] * (int32_t)kh[(long)j * d + c];
                        float qsc = (flags & 16) ? q_scale[bh * (long)N + i] : q_scale[bh * nT + qb];
                        float sc = qsc * k_scale[bh * nT + j / ORC_TILE];
                        sc = sc * c_scale;
                        sj = (float)S * sc;
                    }
                    s[j - j0] = sj;
                    if (sj > tmax) tmax = sj;
                }
                float m_new = tmax > m ? tmax : m;
                float alpha = (m == -INFINITY) ? 0.0f : (float)exp2((double)(m - m_new));
                float psum = 0.0f;
                for (int c = 0; c < d; ++c) vrow[c] = 0.0f;
                for (int j = j0; j < j1; ++j) {
                    float p = (float)exp2((double)(s[j - j0] - m_new));
                    psum = psum + p;
                    float pq = p * 448.0f;
                    if (!(flags & 1)) pq = (float)v_lut[orc_e4m3_encode(pq)];
                    for (int c = 0; c < d; ++c) {
                        float vv;
                        if (flags & 2) vv = bf16f(v_bf16[(bh * (long)N + j) * d + c]) * 448.0f;
                        else vv = (float)v_lut[vh[(long)j * d + c]];
                        vrow[c] = vrow[c] + pq * vv;
                    }
                }
                l = l * alpha + psum;
                for (int c = 0; c < d; ++c) acc[c] = acc[c] * alpha + vrow[c];
                m = m_new;
            }
            float* o = out + w * d;
            for (int c = 0; c < d; ++c) {
                float vs = (flags & 2) ? (1.0f / 448.0f) : v_scale[bh * d + c];
                o[c] = (acc[c] * vs) / (448.0f * l);
                if (out_bf16) out_bf16[w * d + c] = f32_bf16_rne(o[c]);
            }
        }
        free(s);
        free(acc);
        free(vrow);
    }
}

/* ---------------- W8A8 linear with 128x128 block scales ---------------- */

/*
 * Page 1 of the TMAP write-up, "FFN performance optimisation / linear layer
 * quantization": linear-layer weights and activations in 8 bits with a
 * 128 x 128 per-block quantization operator.  Reading: a bf16 matrix
 * X [R, K] (K a multiple of 128) is cut into 128 x 128 blocks; per block
 * scale = fl(amax / 127), code = clamp(rne(x * fl(127 / amax)), +-127), the
 * zero guard of the attention prepass.  codes int8 [R, K]; scales fp32
 * [ceil(R/128), K/128].
 */
void orc_quant_blocks_2d(const uint16_t* x, int R, int K, int8_t* codes, float* scales) {
    int nr = (R + 127) / 128, nk = K / 128;
#pragma omp parallel for schedule(static)
    for (long blk = 0; blk < (long)nr * nk; ++blk) {
        int rb = (int)(blk / nk), kb = (int)(blk % nk);
        int r0 = rb * 128, r1 = r0 + 128 < R ? r0 + 128 : R;
        float amax = 0.0f;
        for (int r = r0; r < r1; ++r)
            for (int c = kb * 128; c < kb * 128 + 128; ++c) {
                float a = fabsf(bf16f(x[(long)r * K + c]));
                if (a > amax) amax = a;
            }
        if (amax == 0.0f) {
            scales[blk] = 0.0f;
            for (int r = r0; r < r1; ++r) memset(codes + (long)r * K + kb * 128, 0, 128);
            continue;
        }
        float inv = 127.0f / amax;
        scales[blk] = amax / 127.0f;
        for (int r = r0; r < r1; ++r)
            for (int c = kb * 128; c < kb * 128 + 128; ++c) {
                double q = rne((double)(bf16f(x[(long)r * K + c]) * inv));
                if (q > 127.0) q = 127.0;
                if (q < -127.0) q = -127.0;
                codes[(long)r * K + c] = (int8_t)q;
            }
    }
}

/*
 * Y[m, n] = sum over K blocks kb (ascending) of
 *           fl(sx[m/128, kb] * sw[n/128, kb]) * S_kb[m, n],
 * S_kb[m, n] = sum_{k in kb} xq[m, k] * wq[n, k] in exact integers (|S| <
 * 2^21, so exact in fp32 too); the sum over kb in fp32, each block's term
 * added with one fused multiply-add (one rounding: the page fixes no
 * rounding, a fused multiply-add is the plain fp32 "acc += scale * S");
 * then + bias[n] (bf16, may be NULL) in fp32, rounded to bf16.
 * xq [M, K], wq [N, K] int8; sx [ceil(M/128), K/128]; sw [ceil(N/128), K/128];
 * only the rows in `rows` (n_rows entries) are computed: y fp32 [n_rows, N]
 * and, if y_bf16, the bf16 bits.
 */
void orc_linear_w8a8(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, const uint16_t* bias,
                     int M, int N, int K, const int* rows, int n_rows, float* y, uint16_t* y_bf16) {
    int nk = K / 128;
#pragma omp parallel for schedule(dynamic, 4)
    for (long w = 0; w < (long)n_rows * N; ++w) {
        int m = rows[w / N], n = (int)(w % N);
        float acc = 0.0f;
        for (int kb = 0; kb < nk; ++kb) {
            int64_t s = 0;
            for (int k = kb * 128; k < kb * 128 + 128; ++k) s += (int64_t)xq[(long)m * K + k] * wq[(long)n * K + k];
            float sc = sx[(long)(m / 128) * nk + kb] * sw[(long)(n / 128) * nk + kb];
            acc = fmaf(sc, (float)s, acc);          /* one rounding per block */
        }
        if (bias) acc = acc + bf16f(bias[n]);
        y[w] = acc;
        if (y_bf16) y_bf16[w] = f32_bf16_rne(acc);
    }
}

/*
 * W8A16 weights (TMAP write-up, FFN section: weights kept in 8 bits while
 * some layers compute with 16-bit activations): the bf16 weight a 16-bit
 * GEMM consumes is the block-scaled code rounded to bf16,
 * w[r, k] = bf16_rne(fl(scales[r/128, k/128] * codes[r, k])).
 */
void orc_dequant_blocks_2d(const int8_t* codes, const float* scales, int R, int K, uint16_t* out) {
    int nk = K / 128;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < (long)R; ++r)
        for (int k = 0; k < K; ++k) {
            float v = scales[(r / 128) * nk + k / 128] * (float)codes[r * K + k];
            out[r * K + k] = f32_bf16_rne(v);
        }
}

/* ---------------- a11: layer schedule ---------------- */

/*
 * modes[l] = 0 (BF16) for layers in the full-precision set, 1 (INT8/FP8)
 * otherwise; the same table serves every denoising step.  Returns -1 on an
 * out-of-range layer index or bad size.
 */
int orc_layer_schedule(int num_layers, const int* fp_layers, int n_fp, int8_t* modes) {
    if (num_layers < 0 || n_fp < 0 || (n_fp > 0 && !fp_layers)) return -1;
    for (int i = 0; i < n_fp; ++i)
        if (fp_layers[i] < 0 || fp_layers[i] >= num_layers) return -1;
    for (int l = 0; l < num_layers; ++l) modes[l] = 1;
    for (int i = 0; i < n_fp; ++i) modes[fp_layers[i]] = 0;
    return 0;
}

/* ---------------- f2: per-layer error and the full-precision layer set ---------------- */

/*
 * Page 1, "Attention performance optimisation / Keeping video quality": the
 * attention error of every layer was measured at every denoising iteration,
 * and the layers whose error stayed large keep the original precision.
 *
 * The error of one layer at one iteration: the relative L2 distance of the
 * quantized output a from the full-precision output b over every element of
 * the layer's output (all heads), sqrt(sum (a - b)^2 / sum b^2), with both
 * sums in fp64 in ascending element order.  b == 0 everywhere gives 0 when a
 * is also 0 and +inf otherwise.
 */
double orc_rel_l2(const uint16_t* a, const uint16_t* b, long n) {
    double num = 0.0, den = 0.0;
    for (long i = 0; i < n; ++i) {
        const double x = (double)bf16f(a[i]), y = (double)bf16f(b[i]);
        const double diff = x - y;
        num += diff * diff;
        den += y * y;
    }
    if (den == 0.0) return num == 0.0 ? 0.0 : INFINITY;
    return sqrt(num / den);
}

/*
 * The full-precision set from the error table err[layer][iteration]:
 *   rule 0: a layer whose error exceeds the threshold at EVERY iteration (the
 *           page's "large at every iteration");
 *   rule 1: a layer whose mean error over the iterations exceeds it.
 * Writes the chosen layers in ascending order; returns how many, or -1 on a
 * bad size, an unknown rule or a non-finite error.
 */
int orc_select_layers(const double* err, int num_layers, int num_iters, double threshold, int rule, int* out) {
    if (num_layers < 0 || num_iters < 1 || (rule != 0 && rule != 1)) return -1;
    int n = 0;
    for (int l = 0; l < num_layers; ++l) {
        int every = 1;
        double sum = 0.0;
        for (int i = 0; i < num_iters; ++i) {
            const double e = err[(long)l * num_iters + i];
            if (!isfinite(e)) return -1;
            if (!(e > threshold)) every = 0;
            sum += e;
        }
        const int pick = rule == 0 ? every : (sum / (double)num_iters > threshold);
        if (pick) out[n++] = l;
    }
    return n;
}
