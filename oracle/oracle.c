/*
 * oracle.c -- plain CPU reference for the NVFP4 attention hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; it is used by the test-suite, by the smoke check and by the
 * CPU-baseline leg of the benchmark.  It shares no code, header, table or
 * constant generator with the CUDA path.
 *
 * Every function restates one step of the method as the web pages describe it,
 * in the pages' order, with no blocking, fusion or reordering beyond what the
 * definition fixes.  Floating point that decides an integer (a code, a scale,
 * a ScaleSearch choice, a selector mask) is done in FP32 exactly as defined
 * below; everything else (scores, softmax, outputs) is FP64.
 *
 * Sources (page title -- section):
 *  [SS]  "Search Your Block Floating Point Scales!" (gist.science summary):
 *        "특수 하드웨어: NVFP4", "문제 제기", "방법론 / ScaleSearch"
 *        ("메커니즘", "검색 전략", "근거"), "ScaleSearchAttention"
 *        ("네이티브 NVFP4 실행", "어텐션 싱크 인식 혼합 정밀도 캐싱").
 *  [SA]  "SageAttention: Accurate 8-Bit Attention for Plug-and-play Inference
 *        Acceleration" (hotpaper.ai): "핵심 기여도", "기술적 접근법"
 *        (per-channel smoothing of K).
 *  [SA3] SageAttention3 article (dasgeld.co): FP4 tensor-core attention.
 *  [TA]  "ThriftAttention: 5%의 연산량으로 90%의 품질 유지" (molayo1419.me):
 *        first and third paragraphs (about 5 % of query-key blocks in high
 *        precision, one joint softmax).
 *
 * Where the pages are silent the readings used here are:
 *  - block = 16 elements; Q/K blocks run along head_dim, V blocks along
 *    tokens, P blocks along keys (a block-scaled MMA can only scale along its
 *    reduction dimension, which for P.V is the key axis);
 *  - two-level scaling: FP32 per-tensor g = amax/2688 (2688 = 6 * 448 maps the
 *    tensor amax onto the largest E2M1 value times the largest E4M3 value),
 *    E4M3 block scale, E2M1 codes;
 *  - "round" is round-to-nearest, ties to the even code, saturating;
 *  - ScaleSearch offsets f run over the half-open range [f_lo, f_hi), default
 *    [-2, 6) = 8 candidates; f = 0 is the starting best and wins ties, then
 *    the lowest f; the error is the FP32 sum of squares in the g-normalised
 *    domain with two interleaved fmaf accumulators;
 *  - K smoothing subtracts the per-(batch, head, channel) mean over tokens,
 *    summed in FP64 in a fixed order (tokens ascending inside 128-token tiles,
 *    then tile partials ascending);
 *  - P is requantised per 16 keys with a fixed second-level scale 1/2688 and
 *    max-scaling; the denominator l sums the dequantised P;
 *  - the selector mean-pools 128-row tiles of raw Q and K into bf16, scores
 *    with an FP32 fmaf chain, and keeps the top ceil(frac * valid) blocks per
 *    head, ties broken by the lower block index;
 *  - incoherence processing rotates Q and K by a signed Hadamard matrix and
 *    balances each channel with a diagonal R (the minimiser of the summed
 *    squared magnitudes), per (batch, head);
 *  - the attention-sink-aware decode cache keeps whole 128-key tiles at full
 *    precision: a count of tiles at the start and at the end of the cache,
 *    with the raw bf16 operands, bf16-rounded P and the smoothed keys' mean
 *    offset, as the mixed blocks of the prefill schedule do.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define TILE 128
#define BLK 16
#define AMAX_NORM 2688.0f /* 6 (largest E2M1) * 448 (largest E4M3) */

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

/* E2M1 (NVFP4 element): sign, 2 exponent bits with bias 1, 1 mantissa bit,
 * no infinities or NaN.  Exponent field 0 is subnormal (0 or 0.5). */
double orc_e2m1_value(int code)
{
    int sign = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return sign ? -mag : mag;
}

/* E4M3 (NVFP4 block scale, "UE4M3" as used here: sign bit always 0):
 * 4 exponent bits with bias 7, 3 mantissa bits, code 0x7F is NaN. */
double orc_e4m3_value(int code)
{
    int e = (code >> 3) & 15;
    int m = code & 7;
    if ((code & 0x7F) == 0x7F) return NAN;
    double mag = (e == 0) ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
    return (code & 0x80) ? -mag : mag;
}

static double E2M1_MAG[8];
static double E4M3_MAG[127];
static int formats_ready = 0;

static void init_formats(void)
{
    if (formats_ready) return;
    for (int c = 0; c < 8; c++) E2M1_MAG[c] = orc_e2m1_value(c);
    for (int c = 0; c < 127; c++) E4M3_MAG[c] = orc_e4m3_value(c);
    formats_ready = 1;
}

/* Nearest representable magnitude among codes 0..ncodes-1 (ascending values),
 * ties to the even code.  Anything above the largest value maps to it, which
 * is the saturating behaviour. */
static int nearest_code(double a, const double* mags, int ncodes)
{
    /* saturating: at or above the largest value (this also keeps huge inputs,
     * whose distances to the top two values round to the same double, on the
     * largest code) */
    if (a >= mags[ncodes - 1]) return ncodes - 1;
    int best = 0;
    double bd = fabs(a - mags[0]);
    for (int c = 1; c < ncodes; c++) {
        double d = fabs(a - mags[c]);
        if (d < bd || (d == bd && (c & 1) == 0)) {
            best = c;
            bd = d;
        }
    }
    return best;
}

/* E2M1 code of a float: the sign is kept (a negative value that rounds to
 * magnitude 0 gives code 0x8), magnitude by nearest_code. */
int orc_e2m1_code(float x)
{
    init_formats();
    int mag = nearest_code(fabs((double)x), E2M1_MAG, 8);
    return (signbit(x) ? 8 : 0) | mag;
}

/* Non-negative E4M3 scale code of a float, round to nearest even, saturating
 * to 448 (code 0x7E). */
int orc_e4m3_code(float x)
{
    init_formats();
    return nearest_code(fabs((double)x), E4M3_MAG, 127);
}

/* bf16 is the upper half of an IEEE float. */
static float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round a float to bf16, nearest with ties to even (finite inputs). */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)(u >> 16); /* inf/nan */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------ */
/* Quantisation of one tensor (Q, K or V)                                    */
/* ------------------------------------------------------------------------ */

/* Per-tensor scale pair: g = A/2688, 1/g = 2688/A, both rounded to FP32;
 * an all-zero tensor uses g = 1. */
void orc_tensor_scale(float amax, float* g, float* inv_g)
{
    if (amax == 0.0f) {
        *g = 1.0f;
        *inv_g = 1.0f;
        return;
    }
    *g = amax / AMAX_NORM;
    *inv_g = AMAX_NORM / amax;
}

/* Codes of one 16-element block of g-normalised values for scale code c:
 * r = 1/s in FP32, y = x~ * r in FP32, code = E2M1(y).  Scale code 0 gives
 * all-zero codes. */
static void encode_block(const float* xt, int c, uint8_t* code16)
{
    if (c == 0) {
        for (int i = 0; i < BLK; i++) code16[i] = 0;
        return;
    }
    float s = (float)E4M3_MAG[c];
    float r = 1.0f / s;
    for (int i = 0; i < BLK; i++) {
        float y = xt[i] * r;
        code16[i] = (uint8_t)orc_e2m1_code(y);
    }
}

/* ScaleSearch error of a block: e_i = x~_i - v_i*s (v_i*s is exact in FP32),
 * two accumulators a_(i mod 2) = fmaf(e_i, e_i, a_(i mod 2)), err = a0 + a1. */
static float block_err(const float* xt, const uint8_t* code16, int c)
{
    float s = (float)E4M3_MAG[c];
    float a0 = 0.0f, a1 = 0.0f;
    for (int i = 0; i < BLK; i++) {
        float vs = (float)(orc_e2m1_value(code16[i]) * (double)s);
        float e = xt[i] - vs;
        if ((i & 1) == 0)
            a0 = fmaf(e, e, a0);
        else
            a1 = fmaf(e, e, a1);
    }
    return a0 + a1;
}

/* Quantise one block of 16 g-normalised values.
 * Max-scaling [SS "메커니즘"]: s0 = E4M3(max|x~| / 6).
 * ScaleSearch [SS "메커니즘", "검색 전략"]: candidates are the scale codes
 * c0 + f (the int8 reinterpretation of the E4M3 byte plus an integer offset);
 * keep the candidate with the lowest block squared error. */
static void quant_block(const float* xt, int search, int f_lo, int f_hi, uint8_t* code16,
                        uint8_t* scale_out, int8_t* off_out)
{
    float amax = 0.0f;
    for (int i = 0; i < BLK; i++) {
        float a = fabsf(xt[i]);
        if (a > amax) amax = a;
    }
    int c0 = orc_e4m3_code(amax / 6.0f);
    int best = c0, bestf = 0;
    encode_block(xt, c0, code16);
    if (search && c0 != 0) {
        float best_err = block_err(xt, code16, c0);
        uint8_t tmp[BLK];
        for (int f = f_lo; f < f_hi; f++) {
            if (f == 0) continue;
            int c = c0 + f;
            if (c < 0 || c > 0x7E) continue;
            encode_block(xt, c, tmp);
            float e = block_err(xt, tmp, c);
            if (e < best_err) {
                best_err = e;
                best = c;
                bestf = f;
            }
        }
        encode_block(xt, best, code16);
    }
    *scale_out = (uint8_t)best;
    if (off_out) *off_out = (int8_t)bestf;
}

/* K smoothing mean [SA "기술적 접근법"]: mean over tokens of each
 * (batch, head, channel), FP64, tokens ascending inside 128-token tiles and the
 * tile partials ascending, then rounded to FP32. */
static void k_channel_mean(const uint16_t* x, int N, int D, float* mu)
{
    for (int c = 0; c < D; c++) {
        double total = 0.0;
        for (int t0 = 0; t0 < N; t0 += TILE) {
            double part = 0.0;
            int t1 = t0 + TILE < N ? t0 + TILE : N;
            for (int t = t0; t < t1; t++) part += (double)bf16_to_f32(x[(size_t)t * D + c]);
            total += part;
        }
        mu[c] = (float)(total / (double)N);
    }
}

/*
 * Quantise a bf16 tensor x[B,H,N,D] to NVFP4.
 *  role 0 = Q, 1 = K, 2 = V.  Q and K blocks: 16 consecutive channels of one
 *  token; codes [B,H,N,D/2], scales [B,H,N,D/16].  V blocks: 16 consecutive
 *  tokens of one channel; codes [B,H,D,N/2], scales [B,H,D,N/16].
 *  Two codes per byte, the even element in the low nibble.
 *  smooth (K only): subtract the channel mean first; k_mean receives it.
 *  g2 receives {g, 1/g}.  ss_off (optional) receives the chosen offset f per
 *  block, in the scales' layout.
 * Returns 0, or -1 for bad arguments, -2 for non-finite input.
 */
int orc_quant_nvfp4(const uint16_t* x, int B, int H, int N, int D, int role, int smooth, int search,
                    int f_lo, int f_hi, uint8_t* codes, uint8_t* scales, float* g2, float* k_mean,
                    int8_t* ss_off)
{
    init_formats();
    if (B < 0 || H < 0 || N < 0 || D <= 0 || D % BLK) return -1;
    if (role == 2 && N % BLK) return -1;
    if (role != 1) smooth = 0;
    size_t BH = (size_t)B * H, per = (size_t)N * D, total = BH * per;

    /* non-finite check */
    for (size_t i = 0; i < total; i++) {
        float f = bf16_to_f32(x[i]);
        if (!isfinite(f)) return -2;
    }

    float* mu = NULL;
    if (smooth) {
        mu = (float*)malloc(sizeof(float) * (BH * D > 0 ? BH * D : 1));
#pragma omp parallel for schedule(static)
        for (long bh = 0; bh < (long)BH; bh++) k_channel_mean(x + bh * per, N, D, mu + bh * D);
        if (k_mean) memcpy(k_mean, mu, sizeof(float) * BH * D);
    }

    /* per-tensor amax of the (smoothed) values: max |fl(x - mu)| */
    float amax = 0.0f;
#pragma omp parallel for reduction(max : amax) schedule(static)
    for (long bh = 0; bh < (long)BH; bh++) {
        for (size_t i = 0; i < per; i++) {
            float v = bf16_to_f32(x[bh * per + i]);
            if (smooth) v = v - mu[bh * D + i % D];
            float a = fabsf(v);
            if (a > amax) amax = a;
        }
    }
    float g, inv_g;
    orc_tensor_scale(amax, &g, &inv_g);
    g2[0] = g;
    g2[1] = inv_g;

    if (role != 2) {
        size_t rows = BH * N;
        int nb = D / BLK;
#pragma omp parallel for schedule(static)
        for (long r = 0; r < (long)rows; r++) {
            size_t bh = (size_t)r / N;
            const uint16_t* xr = x + (size_t)r * D;
            for (int b = 0; b < nb; b++) {
                float xt[BLK];
                uint8_t c16[BLK];
                for (int i = 0; i < BLK; i++) {
                    int c = b * BLK + i;
                    float v = bf16_to_f32(xr[c]);
                    if (smooth) v = v - mu[bh * D + c];
                    xt[i] = v * inv_g;
                }
                uint8_t sc;
                int8_t off;
                quant_block(xt, search, f_lo, f_hi, c16, &sc, &off);
                for (int i = 0; i < BLK / 2; i++)
                    codes[(size_t)r * (D / 2) + b * (BLK / 2) + i] =
                        (uint8_t)((c16[2 * i] & 15) | ((c16[2 * i + 1] & 15) << 4));
                scales[(size_t)r * nb + b] = sc;
                if (ss_off) ss_off[(size_t)r * nb + b] = off;
            }
        }
    } else {
        int nb = N / BLK;
#pragma omp parallel for schedule(static)
        for (long rc = 0; rc < (long)(BH * D); rc++) {
            size_t bh = (size_t)rc / D;
            int c = (int)((size_t)rc % D);
            const uint16_t* xb = x + bh * per;
            for (int b = 0; b < nb; b++) {
                float xt[BLK];
                uint8_t c16[BLK];
                for (int i = 0; i < BLK; i++) xt[i] = bf16_to_f32(xb[(size_t)(b * BLK + i) * D + c]) * inv_g;
                uint8_t sc;
                int8_t off;
                quant_block(xt, search, f_lo, f_hi, c16, &sc, &off);
                for (int i = 0; i < BLK / 2; i++)
                    codes[(size_t)rc * (N / 2) + b * (BLK / 2) + i] =
                        (uint8_t)((c16[2 * i] & 15) | ((c16[2 * i + 1] & 15) << 4));
                scales[(size_t)rc * nb + b] = sc;
                if (ss_off) ss_off[(size_t)rc * nb + b] = off;
            }
        }
    }
    free(mu);
    return 0;
}

/*
 * Quantise FP32 rows x[rows, D] (Q/K layout: blocks of 16 consecutive
 * channels of a row) to NVFP4 with the same per-tensor scale and block rule
 * as orc_quant_nvfp4 (no smoothing: the caller has applied any transform).
 * Returns 0, -1 for bad arguments, -2 for non-finite input.
 */
int orc_quant_rows_f32(const float* x, long rows, int D, int search, int f_lo, int f_hi, uint8_t* codes,
                       uint8_t* scales, float* g2, int8_t* ss_off)
{
    init_formats();
    if (rows < 0 || D <= 0 || D % BLK) return -1;
    size_t total = (size_t)rows * D;
    float amax = 0.0f;
    for (size_t i = 0; i < total; i++) {
        if (!isfinite(x[i])) return -2;
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    float g, inv_g;
    orc_tensor_scale(amax, &g, &inv_g);
    g2[0] = g;
    g2[1] = inv_g;
    int nb = D / BLK;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; r++) {
        for (int b = 0; b < nb; b++) {
            float xt[BLK];
            uint8_t c16[BLK];
            for (int i = 0; i < BLK; i++) xt[i] = x[(size_t)r * D + b * BLK + i] * inv_g;
            uint8_t sc;
            int8_t off;
            quant_block(xt, search, f_lo, f_hi, c16, &sc, &off);
            for (int i = 0; i < BLK / 2; i++)
                codes[(size_t)r * (D / 2) + b * (BLK / 2) + i] =
                    (uint8_t)((c16[2 * i] & 15) | ((c16[2 * i + 1] & 15) << 4));
            scales[(size_t)r * nb + b] = sc;
            if (ss_off) ss_off[(size_t)r * nb + b] = off;
        }
    }
    return 0;
}

/*
 * Incoherence processing [SS "ScaleSearchAttention", "비일관성 처리 (IP) 및
 * 크기 감소"]: a Hadamard transform of Q and K (following QuIP#: the
 * orthonormal Sylvester matrix H_D, entries (-1)^popcount(i & j) / sqrt(D),
 * followed by a diagonal of random signs S, given as input), then a linear
 * pair Q' = Q~ R^-T, K' = K~ R that keeps every score Q' K'^T = Q~ K~^T and
 * lowers the mean squared magnitude.  Reading: R is diagonal per (b, h,
 * channel), the minimiser of |Q~ R^-1|^2 + |K~ R|^2 over diagonal R:
 * r_c = (sum_t q~_tc^2 / sum_t k~_tc^2)^(1/4) (r_c = 1 when either sum is 0).
 * Here Q~ = Q H S and K~ = (K - mu) H S, with mu the K channel mean (k_mean,
 * nullable: no smoothing).
 * Arithmetic (the pages fix none; the codes of Q' and K' are integers decided
 * from these values, so this is the precision both sides use): the rotation
 * in FP32 as the fast Walsh-Hadamard butterfly (stages of span 1, 2, ...,
 * D/2, each pair (a, b) -> (a + b, a - b)), then y_j = fl(t_j * hn) * s_j with
 * hn = fl32(1/sqrt(D)); K's input x_i = fl32(k_i - mu_i).  The sums of
 * squares in FP64: rows ascending inside 128-row tiles, then the tile
 * partials ascending.  r in FP64; R^-1 as the diagonal of FP64 reciprocals
 * 1/r (the pair is Q~ R^-1, K~ R); Q' = fl32(y * (1/r)), K' = fl32(y * r).
 *  q, k: bf16 [B, H, N, D], D a power of two; signs: D entries of +-1.
 *  q_out, k_out: FP32 [B, H, N, D]; r_out: FP32 [B, H, D].
 */
static void fwht_f32(float* y, int D)
{
    for (int h = 1; h < D; h <<= 1)
        for (int i = 0; i < D; i += 2 * h)
            for (int j = i; j < i + h; j++) {
                float a = y[j], b = y[j + h];
                y[j] = a + b;
                y[j + h] = a - b;
            }
}

int orc_incoherence(const uint16_t* q, const uint16_t* k, const float* k_mean, int B, int H, int N, int D,
                    const int8_t* signs, float* q_out, float* k_out, float* r_out)
{
    if (B < 0 || H < 0 || N <= 0 || D <= 0 || (D & (D - 1))) return -1;
    for (int j = 0; j < D; j++)
        if (signs[j] != 1 && signs[j] != -1) return -1;
    const float hn = (float)(1.0 / sqrt((double)D));
    const long BH = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; bh++) {
        float* yq = (float*)malloc(sizeof(float) * (size_t)N * D);
        float* yk = (float*)malloc(sizeof(float) * (size_t)N * D);
        for (int t = 0; t < N; t++) {
            for (int pass = 0; pass < 2; pass++) {
                const uint16_t* src = (pass ? k : q) + ((size_t)bh * N + t) * D;
                float* y = (pass ? yk : yq) + (size_t)t * D;
                for (int i = 0; i < D; i++) {
                    float v = bf16_to_f32(src[i]);
                    if (pass && k_mean) v = v - k_mean[(size_t)bh * D + i];
                    y[i] = v;
                }
                fwht_f32(y, D);
                for (int j = 0; j < D; j++) y[j] = (y[j] * hn) * (float)signs[j];
            }
        }
        for (int j = 0; j < D; j++) {
            double a = 0.0, b = 0.0;
            for (int t0 = 0; t0 < N; t0 += TILE) {
                double pa = 0.0, pb = 0.0;
                for (int t = t0; t < N && t < t0 + TILE; t++) {
                    double vq = yq[(size_t)t * D + j], vk = yk[(size_t)t * D + j];
                    pa += vq * vq;
                    pb += vk * vk;
                }
                a += pa;
                b += pb;
            }
            double r = (a > 0.0 && b > 0.0) ? sqrt(sqrt(a / b)) : 1.0;
            double rinv = 1.0 / r;
            r_out[(size_t)bh * D + j] = (float)r;
            for (int t = 0; t < N; t++) {
                q_out[((size_t)bh * N + t) * D + j] = (float)((double)yq[(size_t)t * D + j] * rinv);
                k_out[((size_t)bh * N + t) * D + j] = (float)((double)yk[(size_t)t * D + j] * r);
            }
        }
        free(yq);
        free(yk);
    }
    return 0;
}

/* Dequantise codes/scales (the layout orc_quant_nvfp4 writes) to FP64:
 * value = E2M1(code) * E4M3(scale) * g.  rows x cols logical matrix with
 * blocks of 16 along cols. */
void orc_dequant(const uint8_t* codes, const uint8_t* scales, float g, size_t rows, int cols, double* out)
{
    init_formats();
#pragma omp parallel for schedule(static)
    for (long r = 0; r < (long)rows; r++) {
        for (int c = 0; c < cols; c++) {
            uint8_t byte = codes[(size_t)r * (cols / 2) + c / 2];
            int code = (c & 1) ? (byte >> 4) : (byte & 15);
            double s = orc_e4m3_value(scales[(size_t)r * (cols / BLK) + c / BLK]);
            out[(size_t)r * cols + c] = orc_e2m1_value(code) * s * (double)g;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* P requantisation inside attention                                         */
/* ------------------------------------------------------------------------ */

/* One 16-key block of probabilities P~ (FP64, in [0,1]) to NVFP4 with the
 * fixed second-level scale 1/2688, i.e. the block of g-normalised values
 * p~ = fl32(P~ * 2688) (a ragged tail is padded with zeros, which change
 * neither the block max nor the error).  Max-scaling (search = 0) or
 * ScaleSearch over the scale codes c0 + f, f in [-2, 6) (search = 1), as for
 * Q, K and V [SS "메커니즘", "검색 전략"].  Returns the dequantised values
 * P^ = E2M1 * E4M3 / 2688 and the chosen scale code. */
static int requant_p_block(const double* pt, int n, double* ph, int search)
{
    float pn[BLK];
    for (int i = 0; i < BLK; i++) pn[i] = i < n ? (float)(pt[i] * 2688.0) : 0.0f;
    uint8_t code16[BLK], c;
    int8_t off;
    quant_block(pn, search, -2, 6, code16, &c, &off);
    const double s = E4M3_MAG[c];
    for (int i = 0; i < n; i++) ph[i] = c ? orc_e2m1_value(code16[i]) * s / 2688.0 : 0.0;
    return c;
}

/* ------------------------------------------------------------------------ */
/* Attention schedule                                                        */
/* ------------------------------------------------------------------------ */

/* One query row over keys [0, nkeys) of one (batch, head), key tiles of 128 in
 * ascending order, online softmax [SS "네이티브 NVFP4 실행"], P requantised
 * per 16 keys, l summing the dequantised P.  Keys j > causal_limit are
 * masked (causal_limit < 0: none).  Mixed blocks [TA] use raw bf16 q and k
 * (k minus its channel mean, so FP4 and bf16 blocks share one score offset),
 * bf16-rounded P and raw V, inside the same running max / sum / output.
 * quant_p: 0 keeps P~ unquantised, 1 requantises it with max-scaling, 2 with
 * ScaleSearch.  Returns m and l through the pointers; o receives the
 * unnormalised sum. */
static void attn_row(const double* q, const double* kh, const double* vh, int nkeys, int D, long causal_limit,
                     double sm_scale, int quant_p, const uint8_t* mixed_tiles, const double* q_raw,
                     const double* k_raw_smoothed, const double* v_raw, double* m_out, double* l_out, double* o)
{
    double m = -INFINITY, l = 0.0;
    double S[TILE], Pt[TILE], Ph[TILE];
    int valid[TILE];
    for (int d = 0; d < D; d++) o[d] = 0.0;
    int ntiles = (nkeys + TILE - 1) / TILE;
    for (int u = 0; u < ntiles; u++) {
        int j0 = u * TILE;
        if (causal_limit >= 0 && j0 > causal_limit) break;
        int n = nkeys - j0 < TILE ? nkeys - j0 : TILE;
        int mixed = mixed_tiles && mixed_tiles[u];
        const double* qq = mixed ? q_raw : q;
        const double* kk = mixed ? k_raw_smoothed : kh;
        const double* vv = mixed ? v_raw : vh;
        double mt = -INFINITY;
        for (int jj = 0; jj < n; jj++) {
            long j = j0 + jj;
            valid[jj] = !(causal_limit >= 0 && j > causal_limit);
            double acc = 0.0;
            for (int d = 0; d < D; d++) acc += qq[d] * kk[(size_t)j * D + d];
            S[jj] = sm_scale * acc;
            if (valid[jj] && S[jj] > mt) mt = S[jj];
        }
        double m_new = m > mt ? m : mt;
        double alpha = exp(m - m_new);
        for (int jj = 0; jj < n; jj++) Pt[jj] = valid[jj] ? exp(S[jj] - m_new) : 0.0;
        if (mixed) {
            for (int jj = 0; jj < n; jj++) Ph[jj] = (double)bf16_to_f32(orc_f32_to_bf16((float)Pt[jj]));
        } else if (quant_p) {
            for (int b0 = 0; b0 < n; b0 += BLK) {
                int nb = n - b0 < BLK ? n - b0 : BLK;
                requant_p_block(Pt + b0, nb, Ph + b0, quant_p == 2);
            }
        } else {
            for (int jj = 0; jj < n; jj++) Ph[jj] = Pt[jj];
        }
        l *= alpha;
        for (int d = 0; d < D; d++) o[d] *= alpha;
        for (int jj = 0; jj < n; jj++) {
            l += Ph[jj];
            const double* vr = vv + (size_t)(j0 + jj) * D;
            for (int d = 0; d < D; d++) o[d] += Ph[jj] * vr[d];
        }
        m = m_new;
    }
    *m_out = m;
    *l_out = l;
}

/*
 * Attention over FP64 operands (already dequantised, or raw for the
 * unquantised path).  q, k, v: [BH, N, D] row-major (V token-major here).
 * rows/nrows: query rows to compute per (batch, head) (NULL = all N rows);
 * out: [BH, nrows, D], lse (nullable): [BH, nrows] natural-log units.
 * mask (nullable): [BH, T, T] mixed-precision block flags; q_raw,
 * k_raw_smoothed, v_raw then hold the raw operands for those blocks.
 */
int orc_attn_f64(const double* q, const double* k, const double* v, long BH, int N, int D, int causal,
                 double sm_scale, int quant_p, const uint8_t* mask, const double* q_raw,
                 const double* k_raw_smoothed, const double* v_raw, const int32_t* rows, int nrows,
                 double* out, double* lse)
{
    init_formats();
    if (N <= 0 || D <= 0) return -1;
    int T = (N + TILE - 1) / TILE;
    int nr = rows ? nrows : N;
#pragma omp parallel for collapse(2) schedule(dynamic, 4)
    for (long bh = 0; bh < BH; bh++) {
        for (int ri = 0; ri < nr; ri++) {
            int i = rows ? rows[ri] : ri;
            size_t base = (size_t)bh * N * D;
            const uint8_t* mt = mask ? mask + ((size_t)bh * T + i / TILE) * T : NULL;
            double m, l;
            double* o = out + ((size_t)bh * nr + ri) * D;
            attn_row(q + base + (size_t)i * D, k + base, v + base, N, D, causal ? i : -1, sm_scale, quant_p, mt,
                     mask ? q_raw + base + (size_t)i * D : NULL, mask ? k_raw_smoothed + base : NULL,
                     mask ? v_raw + base : NULL, &m, &l, o);
            for (int d = 0; d < D; d++) o[d] /= l;
            if (lse) lse[(size_t)bh * nr + ri] = m + log(l);
        }
    }
    return 0;
}

/*
 * Decode over an NVFP4 KV cache (one query token per sequence), grouped-query
 * heads: query head h reads kv head h / (Hq/Hkv).  The keys are processed in
 * splits of `split` keys, each split with its own online softmax from
 * m = -inf; the splits are then merged exactly:
 *   O = sum_s e^(m_s - M) O_s / sum_s e^(m_s - M) l_s,  M = max_s m_s.
 * q: [B, Hq, D] FP64 (already quantised/dequantised), k, v: [B, Hkv, L, D].
 * pairs/npairs: (b, hq) flat indices to compute (NULL = all); out [npairs, D].
 *
 * Attention-sink-aware mixed-precision cache [SS "ScaleSearchAttention",
 * attention-sink-aware mixed-precision caching]: the first sink_first and the
 * last sink_last 128-key tiles of the cache are kept at full precision and the
 * rest in NVFP4.  Those tiles take the mixed-block arithmetic of attn_row:
 * raw bf16 q (q_raw [B, Hq, D]), raw bf16 k minus its channel mean
 * (k_raw_smoothed [B, Hkv, L, D]), bf16-rounded P and raw bf16 v (v_raw), in
 * the same split-wise online softmax.  sink_first = sink_last = 0 is the plain
 * NVFP4 decode and needs no raw operands.
 */
int orc_decode_sink_f64(const double* q, const double* k, const double* v, int B, int Hq, int Hkv, int L, int D,
                        double sm_scale, int quant_p, int split, int sink_first, int sink_last, const double* q_raw,
                        const double* k_raw_smoothed, const double* v_raw, const int32_t* pairs, int npairs,
                        double* out)
{
    init_formats();
    if (Hkv <= 0 || Hq % Hkv || L <= 0 || split <= 0 || split % TILE) return -1;
    if (sink_first < 0 || sink_last < 0) return -1;
    const int mixed = sink_first > 0 || sink_last > 0;
    if (mixed && (!q_raw || !k_raw_smoothed || !v_raw)) return -1;
    int grp = Hq / Hkv;
    int np = pairs ? npairs : B * Hq;
    int nsplit = (L + split - 1) / split;
    int T = (L + TILE - 1) / TILE;  /* key tiles of the whole cache */
#pragma omp parallel for schedule(dynamic, 1)
    for (int pi = 0; pi < np; pi++) {
        int flat = pairs ? pairs[pi] : pi;
        int b = flat / Hq, hq = flat % Hq, hk = hq / grp;
        size_t kvo = ((size_t)b * Hkv + hk) * L * D;
        const double* qr = q + (size_t)flat * D;
        const double* kb = k + kvo;
        const double* vb = v + kvo;
        double* ms = (double*)malloc(sizeof(double) * nsplit);
        double* ls = (double*)malloc(sizeof(double) * nsplit);
        double* os = (double*)malloc(sizeof(double) * nsplit * D);
        uint8_t* flags = (uint8_t*)malloc((size_t)split / TILE);
        double M = -INFINITY;
        for (int s = 0; s < nsplit; s++) {
            int k0 = s * split;
            int n = L - k0 < split ? L - k0 : split;
            int nt = (n + TILE - 1) / TILE;
            for (int u = 0; u < nt; u++) {
                int g = k0 / TILE + u; /* tile index in the cache */
                flags[u] = (uint8_t)(g < sink_first || g >= T - sink_last);
            }
            attn_row(qr, kb + (size_t)k0 * D, vb + (size_t)k0 * D, n, D, -1, sm_scale, quant_p,
                     mixed ? flags : NULL, mixed ? q_raw + (size_t)flat * D : NULL,
                     mixed ? k_raw_smoothed + kvo + (size_t)k0 * D : NULL, mixed ? v_raw + kvo + (size_t)k0 * D : NULL,
                     &ms[s], &ls[s], os + (size_t)s * D);
            if (ms[s] > M) M = ms[s];
        }
        double den = 0.0;
        double* o = out + (size_t)pi * D;
        for (int d = 0; d < D; d++) o[d] = 0.0;
        for (int s = 0; s < nsplit; s++) {
            double w = exp(ms[s] - M);
            den += w * ls[s];
            for (int d = 0; d < D; d++) o[d] += w * os[(size_t)s * D + d];
        }
        for (int d = 0; d < D; d++) o[d] /= den;
        free(ms);
        free(ls);
        free(os);
        free(flags);
    }
    return 0;
}

/* The plain NVFP4-KV decode: no full-precision tiles. */
int orc_decode_f64(const double* q, const double* k, const double* v, int B, int Hq, int Hkv, int L, int D,
                   double sm_scale, int quant_p, int split, const int32_t* pairs, int npairs, double* out)
{
    return orc_decode_sink_f64(q, k, v, B, Hq, Hkv, L, D, sm_scale, quant_p, split, 0, 0, NULL, NULL, NULL, pairs,
                               npairs, out);
}

/* ------------------------------------------------------------------------ */
/* ThriftAttention-style block selector [TA]                                 */
/* ------------------------------------------------------------------------ */

typedef struct {
    float score;
    int32_t idx;
} scored_t;

static int cmp_scored(const void* a, const void* b)
{
    const scored_t* x = (const scored_t*)a;
    const scored_t* y = (const scored_t*)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

/* Mean of one 128-row tile of bf16 rows, per channel: FP32 sum over the
 * rows in ascending order (of fl(x - mu_c) when mu is given, else of x),
 * divided by the row count, rounded to bf16. */
static void pool_tile(const uint16_t* x, const float* mu, int r0, int r1, int D, float* out)
{
    for (int c = 0; c < D; c++) {
        float acc = 0.0f;
        for (int r = r0; r < r1; r++) {
            float v = bf16_to_f32(x[(size_t)r * D + c]);
            if (mu) v = v - mu[c];
            acc = acc + v;
        }
        out[c] = bf16_to_f32(orc_f32_to_bf16(acc / (float)(r1 - r0)));
    }
}

/*
 * Select the top frac_bp/10000 of valid (query tile, key tile) blocks by the
 * score qbar_t . kbar_u (FP32 fmaf chain over channels ascending).  Valid
 * blocks: all, or u <= t when causal.  Ranking: score descending, then the
 * lower block index.
 *  per_row = 0: one budget per (batch, head), ceil(n_valid * frac_bp / 10000);
 *  per_row = 1: one budget per query tile t, ceil(n_valid_t * frac_bp / 10000)
 *               over that row's valid key tiles.
 *  k_mean (nullable, [B,H,D]): pool the smoothed keys fl(k - mu) instead of
 *               the raw ones.  The per-row ranking is unchanged by any channel
 *               offset up to the bf16 rounding of the means, since the offset
 *               shifts every score of a row by the same q_t . mu.
 * mask: [B,H,T,T] (1 = high precision); nsel (nullable): [B,H] blocks
 * selected; scores (nullable): [B,H,T,T].
 */
int orc_thrift_select_ex(const uint16_t* q, const uint16_t* k, const float* k_mean, int B, int H, int N, int D,
                         int causal, int frac_bp, int per_row, uint8_t* mask, int32_t* nsel, float* scores)
{
    if (N <= 0 || D <= 0 || frac_bp < 0 || frac_bp > 10000) return -1;
    int T = (N + TILE - 1) / TILE;
    long BH = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; bh++) {
        const uint16_t* qb = q + (size_t)bh * N * D;
        const uint16_t* kb = k + (size_t)bh * N * D;
        const float* mu = k_mean ? k_mean + (size_t)bh * D : NULL;
        float* qbar = (float*)malloc(sizeof(float) * T * D);
        float* kbar = (float*)malloc(sizeof(float) * T * D);
        scored_t* list = (scored_t*)malloc(sizeof(scored_t) * (size_t)T * T);
        for (int t = 0; t < T; t++) {
            int r1 = (t + 1) * TILE < N ? (t + 1) * TILE : N;
            pool_tile(qb, NULL, t * TILE, r1, D, qbar + (size_t)t * D);
            pool_tile(kb, mu, t * TILE, r1, D, kbar + (size_t)t * D);
        }
        uint8_t* mb = mask + (size_t)bh * T * T;
        long total = 0, nvalid = 0;
        for (int t = 0; t < T; t++) {
            long row0 = nvalid;
            for (int u = 0; u < T; u++) {
                float acc = 0.0f;
                for (int c = 0; c < D; c++) acc = fmaf(qbar[(size_t)t * D + c], kbar[(size_t)u * D + c], acc);
                if (scores) scores[((size_t)bh * T + t) * T + u] = acc;
                mb[(size_t)t * T + u] = 0;
                if (causal && u > t) continue;
                list[nvalid].score = acc;
                list[nvalid].idx = t * T + u;
                nvalid++;
            }
            if (per_row) {
                long n = nvalid - row0, ksel = (n * (long)frac_bp + 9999) / 10000;
                qsort(list + row0, (size_t)n, sizeof(scored_t), cmp_scored);
                for (long i = 0; i < ksel; i++) mb[list[row0 + i].idx] = 1;
                total += ksel;
            }
        }
        if (!per_row) {
            long ksel = (nvalid * (long)frac_bp + 9999) / 10000;
            qsort(list, (size_t)nvalid, sizeof(scored_t), cmp_scored);
            for (long i = 0; i < ksel; i++) mb[list[i].idx] = 1;
            total = ksel;
        }
        if (nsel) nsel[bh] = (int32_t)total;
        free(qbar);
        free(kbar);
        free(list);
    }
    return 0;
}

/* The selector of the benchmark configuration: raw keys, one budget per head. */
int orc_thrift_select(const uint16_t* q, const uint16_t* k, int B, int H, int N, int D, int causal, int frac_bp,
                      uint8_t* mask, int32_t* nsel, float* scores)
{
    return orc_thrift_select_ex(q, k, NULL, B, H, N, D, causal, frac_bp, 0, mask, nsel, scores);
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Block-level entry points used by the worked-example tests                 */
/* ------------------------------------------------------------------------ */

/* Quantise one block of 16 g-normalised values; err_out (nullable) receives
 * the ScaleSearch error of the chosen scale. */
void orc_quant_block(const float* xt, int search, int f_lo, int f_hi, uint8_t* code16, uint8_t* scale_out,
                     int8_t* off_out, float* err_out)
{
    init_formats();
    quant_block(xt, search, f_lo, f_hi, code16, scale_out, off_out);
    if (err_out) *err_out = block_err(xt, code16, *scale_out);
}

/* ScaleSearch error of a block for a given scale code (codes recomputed). */
float orc_block_err(const float* xt, int c)
{
    init_formats();
    uint8_t c16[BLK];
    encode_block(xt, c, c16);
    return block_err(xt, c16, c);
}

/* P requantisation of n <= 16 probabilities. */
void orc_requant_p(const double* pt, int n, double* ph)
{
    init_formats();
    requant_p_block(pt, n, ph, 0);
}

/* P requantisation of one block with max-scaling (search 0) or ScaleSearch
 * (search 1); returns the chosen E4M3 scale code. */
int orc_requant_p_mode(const double* pt, int n, double* ph, int search)
{
    init_formats();
    return requant_p_block(pt, n, ph, search);
}
