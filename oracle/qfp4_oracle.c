/*
 * qfp4_oracle.c - plain, slow CPU oracle of the FP4 quantized-linear path.
 *
 * TEST INFRASTRUCTURE. Only the test-suite, the package's smoke check and the
 * benchmark's CPU-baseline leg load this library. The CUDA path never does, and
 * the two share no code, header, table or constant.
 *
 * Every decision that produces an integer (an E2M1 code, an E4M3/E8M0 scale
 * code) is taken on fp32 values computed in the same fp32 operation order the
 * method is stated in, so that its result is exactly defined. Distances to grid
 * points are compared in fp64, where they are exact. Build with
 * -ffp-contract=off (no fused multiply-add but the one written out, fmaf in
 * dot_tree) and without fast-math.
 *
 * Sources (web pages on FP4 training; no code is printed on any of them):
 *  [Quartet II]  "Quartet II - obuchenie v NVFP4 s tochnymi nesmeshchyonnymi
 *                gradientami" (stuffynlp post 238): random rotations, FP8 scales,
 *                stochastic rounding of the renormalisation into the FP8 scale.
 *  [AMD MXFP4]   "New AMD paper overturns conventional wisdom: FP4 training..."
 *                sections "Chto takoe MXFP4" (micro-scaling, 32-element blocks,
 *                E8M0 shared exponent, round-to-nearest FP4 elements) and
 *                "Poiskovaya eksperimental'naya rabota" (Fprop/Dgrad/Wgrad,
 *                stochastic rounding, random vs deterministic Hadamard).
 *  [NVIDIA NVFP4] "NVIDIA sozdala metod obucheniya neyrosetey v 4-bit tochnosti",
 *                section "Kak eto rabotaet" (16x16 random Hadamard, stochastic
 *                rounding).
 * Where the pages leave a step open, the reading taken is stated at the step.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { FMT_NVFP4 = 0, FMT_MXFP4 = 1, FMT_MXFP4_RU = 2 };
enum { RND_RTN = 0, RND_SR = 1, RND_QUARTET2 = 2 };
enum { HAD_NONE = 0, HAD_DET16 = 1, HAD_DET32 = 2, HAD_RAND16 = 3, HAD_RAND32 = 4 };
enum { AXIS_ROW = 0, AXIS_COL = 1 };
/* Philox counter word 2 holds a tag: what the random word is for. */
enum { TAG_ELEMENT = 0, TAG_SCALE = 1, TAG_SIGN = 2 };

/* ------------------------------------------------------------------------ */
/* bf16 input: widening to fp32 is exact (bf16 is the top half of binary32).  */
static float bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------------------------ */
/* Philox4x32-10, the counter-based generator of Salmon, Moraes, Dror and
 * Shaw, "Parallel random numbers: as easy as 1, 2, 3" (SC'11): ten rounds of
 * two 32x32->64 multiplications by fixed constants, with the key bumped by the
 * two Weyl constants between rounds. */
void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
    uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u; /* golden ratio */
            k1 += 0xBB67AE85u; /* sqrt(3) - 1  */
        }
        uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)x0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)x2;
        uint32_t y0 = (uint32_t)(p1 >> 32) ^ x1 ^ k0;
        uint32_t y1 = (uint32_t)p1;
        uint32_t y2 = (uint32_t)(p0 >> 32) ^ x3 ^ k1;
        uint32_t y3 = (uint32_t)p0;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* The random word for item i of a stream: key = the 64-bit seed, counter =
 * (i/4 as 64 bits, tag | stream << 4, 0); the word used is i mod 4. */
static uint32_t random_word(uint64_t seed, uint32_t tag, uint32_t stream, uint64_t i) {
    uint32_t ctr[4] = {(uint32_t)(i >> 2), (uint32_t)(i >> 34), tag | (stream << 4), 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    oracle_philox4x32_10(ctr, key, out);
    return out[i & 3u];
}

/* A uniform in [0, 1) on a 2^-24 grid from the top 24 bits of a word. */
static float uniform24(uint32_t w) { return (float)(w >> 8) * 0x1p-24f; }

uint32_t oracle_random_word(uint64_t seed, uint32_t tag, uint32_t stream, uint64_t i) {
    return random_word(seed, tag, stream, i);
}

/* The uniform of element i's stochastic rounding. The pages ([AMD MXFP4]
 * glossary: rounding whose error has zero expectation; [NVIDIA NVFP4] "Kak
 * eto rabotaet"; [Quartet II]) fix no width for the random draw. Reading: 16
 * bits per element, half (i mod 2) of word floor(i/2) of the element stream
 * (the low half for even i), rho = half * 2^-16, so one Philox call serves
 * eight elements. Rounding up iff rho < p (p the exact fraction) then has
 * probability ceil(p 2^16) / 2^16: a bias below 2^-16 of the grid gap. */
static float element_uniform(uint64_t seed, uint32_t stream, uint64_t i) {
    const uint32_t w = random_word(seed, TAG_ELEMENT, stream, i >> 1);
    return (float)((w >> (16u * (uint32_t)(i & 1u))) & 0xFFFFu) * 0x1p-16f;
}

float oracle_element_uniform(uint64_t seed, uint32_t stream, uint64_t i) {
    return element_uniform(seed, stream, i);
}

/* ------------------------------------------------------------------------ */
/* E2M1: the 4-bit float element of both formats ([AMD MXFP4] "Chto takoe
 * MXFP4": each element is a 4-bit floating-point number). Code = sign << 3 |
 * index into the magnitude set {0, 0.5, 1, 1.5, 2, 3, 4, 6}. */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double oracle_e2m1_value(uint8_t code) {
    double m = E2M1_MAG[code & 7u];
    return (code & 8u) ? -m : m;
}

/* Round to the nearest representable E2M1 value ([AMD MXFP4] "Chto takoe
 * MXFP4": Q_FP4 is the value rounded to the nearest representable 4-bit
 * float). Reading: a tie goes to the even code index (IEEE
 * round-half-to-even), magnitudes above 6 saturate to 6, and a result of
 * magnitude 0 is code 0 whatever the sign. */
uint8_t oracle_e2m1_rtn(float u) {
    double a = fabs((double)u);
    int idx = 7;
    if (a <= 6.0) {
        double best = a;
        idx = 0;
        for (int j = 1; j < 8; ++j) {
            double d = fabs(a - E2M1_MAG[j]);
            if (d < best || (d == best && (j % 2) == 0)) {
                best = d;
                idx = j;
            }
        }
    }
    if (idx == 0) return 0;
    return (uint8_t)(idx | (u < 0.0f ? 8 : 0));
}

/* Stochastic rounding onto E2M1 ([Quartet II] on NVIDIA's recipe;
 * [AMD MXFP4] "Poiskovaya..."; [NVIDIA NVFP4] "Kak eto rabotaet"): round up
 * to the next grid magnitude with probability equal to the distance from the
 * lower one divided by the gap, so the expected result is the input. rho is
 * the uniform in [0, 1). Magnitudes at or above 6 give 6. */
uint8_t oracle_e2m1_sr(float u, float rho) {
    float a = fabsf(u);
    int idx;
    if (a >= 6.0f) {
        idx = 7;
    } else {
        int lo = 0;
        while (lo < 7 && E2M1_MAG[lo + 1] <= (double)a) ++lo;
        float lo_v = (float)E2M1_MAG[lo];
        float gap = (float)(E2M1_MAG[lo + 1] - E2M1_MAG[lo]);
        float p = (a - lo_v) / gap; /* both steps exact: Sterbenz, power-of-two gap */
        idx = (rho < p) ? lo + 1 : lo;
    }
    if (idx == 0) return 0;
    return (uint8_t)(idx | (u < 0.0f ? 8 : 0));
}

/* ------------------------------------------------------------------------ */
/* E4M3 (FP8, OCP "FN" variant): bias 7, no infinities, 0x7F / 0xFF are NaN,
 * largest finite 448. The NVFP4 block scale ([Quartet II]: NVFP4 uses more
 * precise FP8 scales). */
double oracle_e4m3_value(uint8_t code) {
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round a non-negative fp32 to the nearest E4M3 value, ties to the even code,
 * saturating at 448 (the largest finite value). Brute force over the codes. */
uint8_t oracle_e4m3_rne_sat(float t) {
    double a = (double)t;
    if (!(a < 448.0)) return 0x7E;
    uint8_t best_c = 0;
    double best = a;
    for (int c = 1; c <= 0x7E; ++c) {
        double d = fabs(a - oracle_e4m3_value((uint8_t)c));
        if (d < best || (d == best && (c % 2) == 0)) {
            best = d;
            best_c = (uint8_t)c;
        }
    }
    return best_c;
}

/* Stochastic rounding of a non-negative fp32 onto the E4M3 grid: the Quartet
 * II step that writes the renormalised scale into FP8 ([Quartet II]: the
 * renormalisation is "sewn into" the FP8 scales with SR). Values at or above
 * 448 give 448. */
uint8_t oracle_e4m3_sr(float t, float rho) {
    if (!(t < 448.0f)) return 0x7E;
    int lo = 0;
    while (lo < 0x7E && oracle_e4m3_value((uint8_t)(lo + 1)) <= (double)t) ++lo;
    float lo_v = (float)oracle_e4m3_value((uint8_t)lo);
    float gap = (float)(oracle_e4m3_value((uint8_t)(lo + 1)) - oracle_e4m3_value((uint8_t)lo));
    float p = (t - lo_v) / gap; /* exact: Sterbenz, power-of-two gap */
    return (uint8_t)((rho < p) ? lo + 1 : lo);
}

/* ------------------------------------------------------------------------ */
/* E8M0: the MXFP4 shared exponent ([AMD MXFP4] "Chto takoe MXFP4": one common
 * exponent per block, format E8M0). Value 2^(code-127); code 255 is NaN. */
double oracle_e8m0_value(uint8_t code) {
    if (code == 255) return NAN;
    return ldexp(1.0, (int)code - 127);
}

/* floor(log2(a)) of a positive finite fp32, exactly (frexp is exact). */
static int floor_log2f(float a) {
    int e;
    (void)frexpf(a, &e); /* a = f * 2^e with f in [0.5, 1) */
    return e - 1;
}

/* Stochastic rounding of a positive fp32 onto powers of two (E8M0 grid). The
 * Quartet II step applied to an E8M0 scale (an extension: the pages define it
 * for FP8 scales only). Returns the E8M0 code, clamped to [0, 254]. */
uint8_t oracle_e8m0_sr(float t, float rho) {
    int e = floor_log2f(t);
    float lo = ldexpf(1.0f, e);
    float p = (t - lo) / lo; /* exact: t in [lo, 2 lo) */
    if (rho < p) e += 1;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return (uint8_t)(e + 127);
}

/* ------------------------------------------------------------------------ */
/* Hadamard transform ([NVIDIA NVFP4] "Kak eto rabotaet": 16x16 random
 * Hadamard transforms; [AMD MXFP4] "Poiskovaya...": randomized Hadamard with
 * random sign flips vs the deterministic Hadamard; [Quartet II]: random
 * rotations). Sylvester matrix H[i][j] = (-1)^popcount(i & j). */
void oracle_hadamard_matrix(int n, int8_t* H) {
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j) H[i * n + j] = (__builtin_popcount((unsigned)(i & j)) & 1) ? -1 : 1;
}

/* In-place unnormalised fast Walsh-Hadamard transform, w -> H w, in fp32.
 * Reading: stages in ascending half-width h = 1, 2, 4, ...; in each pair
 * (j, j + h) of a 2h-block, (a, b) -> (a + b, a - b). */
void oracle_fwht(float* w, int n) {
    for (int h = 1; h < n; h <<= 1)
        for (int j0 = 0; j0 < n; j0 += 2 * h)
            for (int j = j0; j < j0 + h; ++j) {
                float a = w[j], b = w[j + h];
                w[j] = a + b;
                w[j + h] = a - b;
            }
}

/* The random sign vector D of a random Hadamard: bit b of word 0 of
 * Philox(key = rot seed, counter = (0, 0, TAG_SIGN | stream << 4, 0)); a set
 * bit flips the sign of position b. Reading: one vector of length n_h per
 * call, shared by every block and by both operands of a GEMM, so the rotation
 * cancels in the product. A deterministic Hadamard has D = I. */
uint32_t oracle_sign_bits(uint64_t rot_seed, uint32_t rot_stream) {
    return random_word(rot_seed, TAG_SIGN, rot_stream, 0);
}

static int had_size(int had) {
    return (had == HAD_DET16 || had == HAD_RAND16) ? 16 : (had == HAD_DET32 || had == HAD_RAND32) ? 32 : 0;
}

/* Rotate one quantized-axis segment of length k in place: per n_h chunk,
 * v = c * H * (D x), c = fp32(1/sqrt(n_h)) applied as one fp32 multiply after
 * the butterflies (reading: orthonormal transform; values stay fp32). */
static void rotate_segment(float* seg, int64_t k, int nh, uint32_t sign_bits) {
    if (nh == 0) return;
    const float c = (float)(1.0 / sqrt((double)nh));
    for (int64_t j0 = 0; j0 < k; j0 += nh) {
        float* w = seg + j0;
        for (int j = 0; j < nh; ++j)
            if ((sign_bits >> j) & 1u) w[j] = -w[j];
        oracle_fwht(w, nh);
        for (int j = 0; j < nh; ++j) w[j] = w[j] * c;
    }
}

/* Sum of n fp32 terms by the halving-stride tree: for stride n/2, ..., 1,
 * s[j] += s[j + stride] for j < stride. Reading: a fixed order, so the
 * Quartet II renormalisation is exactly defined. */
static float tree_sum(float* s, int n) {
    for (int stride = n / 2; stride >= 1; stride /= 2)
        for (int j = 0; j < stride; ++j) s[j] = s[j] + s[j + stride];
    return s[0];
}

/* <a, b> of n <= 32 fp32 terms in the same halving-stride order, the first
 * stride taking the products: s[j] = a[j] b[j] + a[j + n/2] b[j + n/2] as one
 * fused multiply-add of a[j] b[j] onto the rounded product a[j + n/2] b[j +
 * n/2] (fmaf: exact product and sum, one rounding), then tree_sum of the n/2
 * partial sums. Reading: the pages fix neither the precision nor the order of
 * the Quartet II sums; this one is exactly defined, and the multiply-add
 * leaves one rounding fewer per pair than a product followed by a sum. */
static float dot_tree(const float* a, const float* b, int n) {
    float s[16];
    const int h = n / 2;
    for (int j = 0; j < h; ++j) s[j] = fmaf(a[j], b[j], a[j + h] * b[j + h]);
    return tree_sum(s, h);
}

/* Load quantized-axis segment `row` (length k) of x into seg as fp32. */
static void load_segment(const uint16_t* x, int64_t ld, int axis, int64_t row, int64_t k, float* seg) {
    if (axis == AXIS_ROW)
        for (int64_t j = 0; j < k; ++j) seg[j] = bf16_to_f32(x[row * ld + j]);
    else
        for (int64_t j = 0; j < k; ++j) seg[j] = bf16_to_f32(x[j * ld + row]);
}

/*
 * Quantize x (bf16, R x C, row stride ld) to FP4.
 *   axis ROW: quantize along C; the result is rows = R, k = C.
 *   axis COL: quantize along R; the result is the quantized transpose,
 *             rows = C, k = R (element (c, r) is x[r][c]).
 * Outputs: codes [rows][k/2] (element j in the low nibble of byte j/2 when j is
 * even, high nibble when odd), scales [rows][k/nb] canonical row-major codes
 * (E4M3 for NVFP4, E8M0 for MXFP4), *g_out the NVFP4 per-tensor scale (1 for
 * MXFP4), alpha_out (optional) [rows][k/nb] the Quartet II renormalisation.
 * amax_in (optional) replaces the tensor amax of step 2.
 * sel (optional, nsel entries): quantize only these rows of the quantized
 * orientation; row sel[i] goes to output row i. Everything else is as for the
 * whole tensor: the tensor amax is over all rows, and the random words are
 * those of the row's own index.
 * Returns 0, or -1 on an invalid argument.
 */
int oracle_quantize_rows(const uint16_t* x, int64_t R, int64_t C, int64_t ld, int fmt, int rnd, int had,
                         int axis, uint64_t rot_seed, uint32_t rot_stream, uint64_t sr_seed, uint32_t sr_stream,
                         const float* amax_in, const int64_t* sel, int64_t nsel, uint8_t* codes, uint8_t* scales,
                         float* g_out, float* alpha_out) {
    if (fmt != FMT_NVFP4 && fmt != FMT_MXFP4 && fmt != FMT_MXFP4_RU) return -1;
    if (rnd < RND_RTN || rnd > RND_QUARTET2) return -1;
    if (had < HAD_NONE || had > HAD_RAND32) return -1;
    if (axis != AXIS_ROW && axis != AXIS_COL) return -1;
    if (R < 0 || C < 0 || ld < C) return -1;
    const int64_t rows = (axis == AXIS_ROW) ? R : C;
    const int64_t k = (axis == AXIS_ROW) ? C : R;
    const int nb = (fmt == FMT_NVFP4) ? 16 : 32;
    const int nh = had_size(had);
    if (k % nb != 0 || (nh && k % nh != 0)) return -1;
    const uint32_t signs = (had == HAD_RAND16 || had == HAD_RAND32) ? oracle_sign_bits(rot_seed, rot_stream) : 0u;
    const int64_t nblk = k / nb;
    if (sel) {
        if (nsel < 0) return -1;
        for (int64_t i = 0; i < nsel; ++i)
            if (sel[i] < 0 || sel[i] >= rows) return -1;
    }
    const int64_t n_out = sel ? nsel : rows;

    /* Step 1-2: the NVFP4 per-tensor scale from the amax of the rotated tensor.
     * Reading (NVFP4 two-level scaling, FP32 tensor scale): amax maps to 6 * 448,
     * the top of E2M1 times the top of E4M3; s_enc = 2688 / amax and
     * g = amax / 2688 (fp32 divisions); an all-zero tensor gives s_enc = g = 1. */
    float amax = 0.0f;
    if (fmt == FMT_NVFP4) {
        if (amax_in) {
            amax = *amax_in;
        } else {
#pragma omp parallel
            {
                float* seg = (float*)malloc(sizeof(float) * (size_t)(k > 0 ? k : 1));
                float local = 0.0f;
#pragma omp for schedule(static)
                for (int64_t r = 0; r < rows; ++r) {
                    load_segment(x, ld, axis, r, k, seg);
                    rotate_segment(seg, k, nh, signs);
                    for (int64_t j = 0; j < k; ++j) local = fmaxf(local, fabsf(seg[j]));
                }
#pragma omp critical
                amax = fmaxf(amax, local);
                free(seg);
            }
        }
    }
    float s_enc = 1.0f, g = 1.0f;
    if (fmt == FMT_NVFP4 && amax > 0.0f) {
        s_enc = 2688.0f / amax;
        if (s_enc > FLT_MAX) s_enc = FLT_MAX;
        g = amax / 2688.0f;
    }
    if (g_out) *g_out = g;

#pragma omp parallel
    {
        float* seg = (float*)malloc(sizeof(float) * (size_t)(k > 0 ? k : 1));
        float u[32], qval[32];
        uint8_t q[32];
#pragma omp for schedule(static)
        for (int64_t ro = 0; ro < n_out; ++ro) {
            const int64_t r = sel ? sel[ro] : ro; /* row of the quantized orientation */
            load_segment(x, ld, axis, r, k, seg);
            rotate_segment(seg, k, nh, signs);
            for (int64_t b = 0; b < nblk; ++b) {
                const float* v = seg + b * nb;
                const int64_t blk_index = r * nblk + b; /* block index in the quantized orientation */
                const int64_t blk_out = ro * nblk + b;  /* where it is stored */
                /* Step 3: block scale from the block amax. */
                float amax_b = 0.0f;
                for (int j = 0; j < nb; ++j) amax_b = fmaxf(amax_b, fabsf(v[j]));
                uint8_t s_code;
                float s_val, rmul;
                if (fmt == FMT_NVFP4) {
                    /* S = E4M3_RN_sat(fp32(amax_b / 6) * s_enc); r = s_enc / S. */
                    float d = amax_b / 6.0f;
                    float t = d * s_enc;
                    s_code = oracle_e4m3_rne_sat(t);
                    s_val = (float)oracle_e4m3_value(s_code);
                    rmul = (s_val == 0.0f) ? 0.0f : s_enc / s_val;
                } else {
                    /* [AMD MXFP4] "Chto takoe MXFP4": the shared exponent is the largest
                     * exponent in the block. Reading (OCP MX): E = floor(log2 amax_b) - 2,
                     * 2 being the largest E2M1 exponent, clamped to [-127, 127]; larger
                     * elements saturate to 6. An all-zero block has code 0 and r = 0. */
                    if (amax_b == 0.0f) {
                        s_code = 0;
                        s_val = (float)oracle_e8m0_value(0);
                        rmul = 0.0f;
                    } else {
                        int E = floor_log2f(amax_b) - 2;
                        if (fmt == FMT_MXFP4_RU) {
                            /* Round-up variant, not on the pages (they give the
                             * shared exponent only as the block's largest one):
                             * the smallest E with amax_b <= 6 * 2^E, so that no
                             * element of the block clips; searched upward from one
                             * below the floor rule's E, 6 * 2^E exact in double. */
                            E -= 1;
                            while ((double)amax_b > 6.0 * ldexp(1.0, E)) E += 1;
                        }
                        if (E < -127) E = -127;
                        if (E > 127) E = 127;
                        s_code = (uint8_t)(E + 127);
                        s_val = ldexpf(1.0f, E);
                        rmul = ldexpf(1.0f, -E);
                    }
                }
                /* Step 4-5: scaled values and element rounding. */
                for (int j = 0; j < nb; ++j) u[j] = v[j] * rmul;
                if (rnd == RND_SR) {
                    for (int j = 0; j < nb; ++j) {
                        const uint64_t i = (uint64_t)(r * k + b * nb + j);
                        q[j] = oracle_e2m1_sr(u[j], element_uniform(sr_seed, sr_stream, i));
                    }
                } else {
                    for (int j = 0; j < nb; ++j) q[j] = oracle_e2m1_rtn(u[j]);
                }
                float alpha = 1.0f;
                if (rnd == RND_QUARTET2) {
                    /* [Quartet II]: the quantized rotated block is collinear with the
                     * original in expectation; renormalising by alpha = <u,u>/<u,q> (the
                     * projection of u on q) makes it unbiased; alpha (about 0.94-1.06) is
                     * too fine for an FP8 scale, so S * alpha is stochastically rounded
                     * into the scale. The element codes stay round-to-nearest. */
                    for (int j = 0; j < nb; ++j) qval[j] = (float)oracle_e2m1_value(q[j]);
                    float num = dot_tree(u, u, nb);
                    float den = dot_tree(u, qval, nb);
                    alpha = (den == 0.0f) ? 1.0f : num / den;
                    float t = s_val * alpha;
                    float rho = uniform24(random_word(sr_seed, TAG_SCALE, sr_stream, (uint64_t)blk_index));
                    s_code = (fmt == FMT_NVFP4) ? oracle_e4m3_sr(t, rho) : oracle_e8m0_sr(t, rho);
                }
                if (alpha_out) alpha_out[blk_out] = alpha;
                scales[blk_out] = s_code;
                /* Step 6: pack two codes per byte, the lower index in the low nibble. */
                uint8_t* out = codes + ro * (k / 2) + b * (nb / 2);
                for (int j = 0; j < nb; j += 2) out[j / 2] = (uint8_t)(q[j] | (q[j + 1] << 4));
            }
        }
        free(seg);
    }
    return 0;
}

int oracle_quantize(const uint16_t* x, int64_t R, int64_t C, int64_t ld, int fmt, int rnd, int had,
                    int axis, uint64_t rot_seed, uint32_t rot_stream, uint64_t sr_seed, uint32_t sr_stream,
                    const float* amax_in, uint8_t* codes, uint8_t* scales, float* g_out, float* alpha_out) {
    return oracle_quantize_rows(x, R, C, ld, fmt, rnd, had, axis, rot_seed, rot_stream, sr_seed, sr_stream, amax_in,
                                NULL, 0, codes, scales, g_out, alpha_out);
}

/* The rotated, unquantized values v of the quantized orientation, [rows][k]
 * fp32 (used by statistical tests to compare the estimate with its target). */
int oracle_rotate(const uint16_t* x, int64_t R, int64_t C, int64_t ld, int had, int axis, uint64_t rot_seed,
                  uint32_t rot_stream, float* v) {
    const int64_t rows = (axis == AXIS_ROW) ? R : C;
    const int64_t k = (axis == AXIS_ROW) ? C : R;
    const int nh = had_size(had);
    if (nh && k % nh != 0) return -1;
    const uint32_t signs = (had == HAD_RAND16 || had == HAD_RAND32) ? oracle_sign_bits(rot_seed, rot_stream) : 0u;
    for (int64_t r = 0; r < rows; ++r) {
        load_segment(x, ld, axis, r, k, v + r * k);
        rotate_segment(v + r * k, k, nh, signs);
    }
    return 0;
}
