/*
 * Seeded synthetic Q/K/V generator for the video-DiT self-attention workloads.
 *
 * This module holds no attention or quantization arithmetic: it only draws
 * numbers.  Both the CUDA path (through the tests and the benchmark) and the
 * CPU oracle consume the bytes it writes, so the two sides see identical
 * inputs.
 *
 * Generator (counter based, so any element can be drawn independently):
 *   splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
 *   generators", OOPSLA 2014) as the mixing function;
 *   uniform u = (splitmix64(ctr) >> 11) * 2^-53 in [0, 1);
 *   Box-Muller (1958): z = sqrt(-2 ln(1 - u1)) * cos(2 pi u2), in fp64.
 * Element e of stream (seed, tensor) draws its two uniforms at counters
 * key + 2e and key + 2e + 1, key = splitmix64(splitmix64(seed) ^ tensor * C).
 *
 * Workload recipe (video DiT self-attention, page 1 "Attention performance
 * optimisation" of the TMAP write-up profiles this op on CogVideoX / Wan):
 *   Q, V ~ N(0,1); K ~ N(0,1) + off[b,h,c] with off ~ N(0, k_off_std^2)
 *   broadcast over tokens; optional outlier channels: a seeded set of
 *   round(frac*H*d) distinct (h,c) pairs whose Q and K values are multiplied by
 *   outlier_scale before the K offset is added; optional all-zero K channel.
 *   Values are formed in fp64, rounded to fp32 (RNE) and then to bf16 (RNE).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SYN_Q 1u
#define SYN_K 2u
#define SYN_V 3u
#define SYN_KOFF 4u
#define SYN_OUTLIER 5u
#define SYN_ROWS 6u
#define SYN_LX 7u
#define SYN_LW 8u
#define SYN_LB 9u
#define SYN_LOUT 10u

static inline uint64_t splitmix64(uint64_t x) {
    x += 0x9E3779B97F4A7C15ull;
    x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
    x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
    return x ^ (x >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t tensor) {
    return splitmix64(splitmix64(seed) ^ (tensor * 0xD1B54A32D192ED03ull));
}

static inline double uniform01(uint64_t ctr) {
    return (double)(splitmix64(ctr) >> 11) * (1.0 / 9007199254740992.0);
}

static inline double normal_at(uint64_t key, uint64_t e) {
    double u1 = uniform01(key + 2 * e);
    double u2 = uniform01(key + 2 * e + 1);
    double r = sqrt(-2.0 * log(1.0 - u1));
    return r * cos(6.283185307179586476925286766559 * u2);
}

/* fp32 -> bf16 bits, round to nearest even (inputs here are finite). */
static inline uint16_t f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

double synth_normal(uint64_t seed, uint32_t tensor, uint64_t e) {
    return normal_at(stream_key(seed, tensor), e);
}

/* Marks the outlier (h, c) pairs: the n_out pairs with the smallest hash. */
static void outlier_mask_t(uint64_t seed, uint32_t tensor, int H, int d, int n_out, uint8_t* mask) {
    int total = H * d;
    memset(mask, 0, (size_t)total);
    if (n_out <= 0) return;
    uint64_t key = stream_key(seed, tensor);
    uint64_t* h = (uint64_t*)malloc(sizeof(uint64_t) * (size_t)total);
    for (int i = 0; i < total; ++i) h[i] = splitmix64(key + (uint64_t)i);
    for (int k = 0; k < n_out && k < total; ++k) {
        int best = -1;
        for (int i = 0; i < total; ++i)
            if (!mask[i] && (best < 0 || h[i] < h[best])) best = i;
        mask[best] = 1;
    }
    free(h);
}

static void outlier_mask(uint64_t seed, int H, int d, int n_out, uint8_t* mask) {
    outlier_mask_t(seed, SYN_OUTLIER, H, d, n_out, mask);
}

int synth_outlier_pairs(uint64_t seed, int H, int d, int n_out, uint8_t* mask_out) {
    if (H <= 0 || d <= 0 || n_out < 0 || n_out > H * d) return -1;
    outlier_mask(seed, H, d, n_out, mask_out);
    return 0;
}

/*
 * Writes bf16 bit patterns of Q, K, V, each [B, H, N, d] row-major (any of the
 * three pointers may be NULL to skip that tensor).
 *   k_off_std      standard deviation of the per-(b,h,c) K offset (0: none)
 *   n_outlier      number of (h, c) outlier pairs (0: none)
 *   outlier_scale  factor applied to Q and K on outlier pairs
 *   zero_k_channel channel c whose K values are all zero (-1: none)
 */
int synth_qkv(uint64_t seed, int B, int H, int N, int d, double k_off_std,
              int n_outlier, double outlier_scale, int zero_k_channel,
              uint16_t* q, uint16_t* k, uint16_t* v) {
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return -1;
    if (n_outlier < 0 || n_outlier > H * d) return -1;
    uint8_t* mask = (uint8_t*)malloc((size_t)H * d);
    outlier_mask(seed, H, d, n_outlier, mask);
    double* off = (double*)malloc(sizeof(double) * (size_t)B * H * d);
    uint64_t koff = stream_key(seed, SYN_KOFF);
    for (long i = 0; i < (long)B * H * d; ++i) off[i] = k_off_std * normal_at(koff, (uint64_t)i);
    const uint64_t kq = stream_key(seed, SYN_Q), kk = stream_key(seed, SYN_K), kv = stream_key(seed, SYN_V);
    const long rows = (long)B * H * N;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        long bh = r / N;
        int h = (int)(bh % H);
        for (int c = 0; c < d; ++c) {
            uint64_t e = (uint64_t)r * (uint64_t)d + (uint64_t)c;
            double scale = mask[h * d + c] ? outlier_scale : 1.0;
            if (q) q[e] = f32_to_bf16((float)(normal_at(kq, e) * scale));
            if (k) {
                double x = normal_at(kk, e) * scale + off[bh * d + c];
                if (c == zero_k_channel) x = 0.0;
                k[e] = f32_to_bf16((float)x);
            }
            if (v) v[e] = f32_to_bf16((float)normal_at(kv, e));
        }
    }
    free(off);
    free(mask);
    return 0;
}

/*
 * Seeded sample of n distinct query rows of [0, N): always row 0, row N-1 and
 * the first row of the last 128-row tile, the rest drawn uniformly.  Rows are
 * returned sorted.  Returns the number written (min(n, N)).
 */
static int cmp_int(const void* a, const void* b) {
    int x = *(const int*)a, y = *(const int*)b;
    return (x > y) - (x < y);
}

int synth_sample_rows(uint64_t seed, int N, int n, int* rows) {
    if (N <= 0 || n <= 0) return 0;
    if (n >= N) {
        for (int i = 0; i < N; ++i) rows[i] = i;
        return N;
    }
    uint8_t* taken = (uint8_t*)calloc((size_t)N, 1);
    int cnt = 0;
    int fixed[3] = {0, N - 1, ((N - 1) / 128) * 128};
    for (int i = 0; i < 3 && cnt < n; ++i)
        if (!taken[fixed[i]]) { taken[fixed[i]] = 1; rows[cnt++] = fixed[i]; }
    uint64_t key = stream_key(seed, SYN_ROWS);
    uint64_t ctr = 0;
    while (cnt < n) {
        int r = (int)(splitmix64(key + ctr++) % (uint64_t)N);
        if (!taken[r]) { taken[r] = 1; rows[cnt++] = r; }
    }
    free(taken);
    qsort(rows, (size_t)cnt, sizeof(int), cmp_int);
    return cnt;
}

/*
 * Linear-layer operands, bf16 bit patterns, row-major:
 *   x [M, K]  N(0,1), the n_outlier channels k with the smallest hash scaled
 *             by outlier_scale (activation outlier channels)
 *   w [N, K]  N(0,1) / sqrt(K)
 *   bias [N]  0.02 * N(0,1)
 * Any pointer may be NULL to skip that tensor.
 */
int synth_linear(uint64_t seed, int M, int N, int K, int n_outlier, double outlier_scale,
                 uint16_t* x, uint16_t* w, uint16_t* bias) {
    if (M <= 0 || N <= 0 || K <= 0 || n_outlier < 0 || n_outlier > K) return -1;
    uint8_t* mask = (uint8_t*)malloc((size_t)K);
    outlier_mask_t(seed, SYN_LOUT, 1, K, n_outlier, mask);
    const uint64_t kx = stream_key(seed, SYN_LX), kw = stream_key(seed, SYN_LW), kb = stream_key(seed, SYN_LB);
    const double wstd = 1.0 / sqrt((double)K);
    if (x) {
#pragma omp parallel for schedule(static)
        for (long r = 0; r < (long)M; ++r)
            for (int c = 0; c < K; ++c) {
                uint64_t e = (uint64_t)r * (uint64_t)K + (uint64_t)c;
                x[e] = f32_to_bf16((float)(normal_at(kx, e) * (mask[c] ? outlier_scale : 1.0)));
            }
    }
    if (w) {
#pragma omp parallel for schedule(static)
        for (long r = 0; r < (long)N; ++r)
            for (int c = 0; c < K; ++c) {
                uint64_t e = (uint64_t)r * (uint64_t)K + (uint64_t)c;
                w[e] = f32_to_bf16((float)(normal_at(kw, e) * wstd));
            }
    }
    if (bias)
        for (int n = 0; n < N; ++n) bias[n] = f32_to_bf16((float)(0.02 * normal_at(kb, (uint64_t)n)));
    free(mask);
    return 0;
}
