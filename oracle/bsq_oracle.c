/*
 * bsq_oracle.c -- the plain, slow, scalar CPU oracle for block-scaled
 * quantization (NVFP4, MXFP8, MXFP4), the 16-point random Hadamard transform and the
 * block-scaled GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  The tests, the package's smoke check and the
 * bench's CPU-baseline leg call it; the library under fp8_math_b200/ never
 * links, imports or calls it, and it shares no code, header, table or constant
 * with that library.
 *
 * Build (see oracle.py): gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math
 * -fPIC -shared.  On x86-64 every float operation below is one IEEE-754
 * binary32 operation rounded to nearest-even, executed in the order written
 * (no contraction into FMA, no excess precision).  Reductions that produce
 * a GEMM value use binary64.
 *
 * Sources (web pages, cited by title and section):
 *   [MX]   "Microscaling (MX) and block-scaled 4-bit formats" -- sections
 *          "The problem", "Microscaling", "NVFP4", "Hardware and kernels",
 *          "Open points", "Words on this page" (stochastic rounding).
 *   [FP4]  "08 -- FP4, MXFP4, NVFP4: The Blackwell Frontier" -- sections
 *          "Bit layout of FP4 E2M1", "The two Blackwell formats: MXFP4 vs
 *          NVFP4", "The OCP Microscaling (MX) spec".
 *   [RL]   "LMSYS and humans& ... Blackwell-native low-precision recipes" --
 *          section "Recipe 1: End-to-end MXFP8".
 *   [TML]  "Thinking Machines ... Inkling 2 Small end-to-end 4-bit training"
 *          -- sections "A precision choice for each stage", "Why
 *          communication became the next bottleneck".
 * Readings where the pages are silent are named R<n> in comments; the same
 * numbering is used in the design notes.
 *
 * Parity unpinned (no value on the pages or in mathematics fixes them beyond
 * CPU/GPU agreement): the Philox bit stream is pinned only against an
 * independent library implementation in the tests; the Four-Over-Six error
 * summation order (R9) and the operation order of the NVFP4 block scale (R3)
 * are readings, pinned by invariants only.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

/* ------------------------------------------------------------------------ */
/* bf16 <-> fp32                                                              */
/* ------------------------------------------------------------------------ */

/* bf16 is the top 16 bits of a binary32. */
float ora_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round a finite binary32 to bf16, nearest, ties to even. */
uint16_t ora_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t keep = u >> 16;
    uint32_t rest = u & 0xFFFFu;
    if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u)))
        keep += 1u;
    return (uint16_t)keep;
}

/* ------------------------------------------------------------------------ */
/* E2M1 (FP4) -- [FP4] "Bit layout of FP4 E2M1": bits S E E M, exponent     */
/* bias 1, E=0 is subnormal with value M * 0.5; [MX] "The problem" lists the  */
/* non-negative values 0, 0.5, 1, 1.5, 2, 3, 4, 6.                            */
/* ------------------------------------------------------------------------ */

float ora_e2m1_value(uint8_t code)
{
    int s = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    float mag = (e == 0) ? 0.5f * (float)m : ldexpf(1.0f + 0.5f * (float)m, e - 1);
    return s ? -mag : mag;
}

/* Nearest E2M1 value, ties to the code with mantissa bit 0, saturating at
 * +-6 (round-to-nearest as [MX] "Open points" names it; saturation per the
 * configuration's "E2M1 by RNE with saturation at +-6").  The sign bit is the
 * sign of v, so a negative input that rounds to zero gives code 0x8 (R5). */
uint8_t ora_e2m1_rne_sat(float v)
{
    float a = fabsf(v);
    uint8_t mag = 7;
    for (uint8_t c = 0; c < 7; c++) {
        float lo = ora_e2m1_value(c), hi = ora_e2m1_value((uint8_t)(c + 1));
        if (a < hi) {
            float mid = 0.5f * (lo + hi); /* exact: at most 3 significant bits */
            if (a < mid)
                mag = c;
            else if (a > mid)
                mag = (uint8_t)(c + 1);
            else
                mag = (c & 1) ? (uint8_t)(c + 1) : c;
            break;
        }
    }
    return (uint8_t)((signbit(v) ? 8 : 0) | mag);
}

/* ------------------------------------------------------------------------ */
/* E4M3 (the "FN" variant: no infinities, S.1111.111 is NaN, max 448)        */
/* [RL] "Recipe 1": MXFP8 elements are E4M3; [MX] "NVFP4": the NVFP4 block   */
/* scale is E4M3.  Bias 7; E=0 is subnormal with value M * 2^-9.             */
/* ------------------------------------------------------------------------ */

float ora_e4m3_value(uint8_t code)
{
    int s = code >> 7;
    int e = (code >> 3) & 15;
    int m = code & 7;
    if (e == 15 && m == 7)
        return NAN;
    float mag = (e == 0) ? ldexpf((float)m, -9) : ldexpf(1.0f + (float)m / 8.0f, e - 7);
    return s ? -mag : mag;
}

/* Nearest E4M3 value, ties to even mantissa, saturating at +-448 (R11).
 * Codes 0x00..0x7E are the non-negative finite values in increasing order. */
uint8_t ora_e4m3_rne_sat(float v)
{
    float a = fabsf(v);
    uint8_t mag;
    if (a >= 448.0f) {
        mag = 0x7E;
    } else {
        int lo = 0, hi = 0x7E; /* invariant: value(lo) <= a < value(hi) */
        while (hi - lo > 1) {
            int mid = (lo + hi) / 2;
            if (ora_e4m3_value((uint8_t)mid) <= a)
                lo = mid;
            else
                hi = mid;
        }
        float vlo = ora_e4m3_value((uint8_t)lo), vhi = ora_e4m3_value((uint8_t)hi);
        float midv = 0.5f * (vlo + vhi); /* exact: 5 significant bits */
        if (a < midv)
            mag = (uint8_t)lo;
        else if (a > midv)
            mag = (uint8_t)hi;
        else
            mag = (lo & 1) ? (uint8_t)hi : (uint8_t)lo;
    }
    return (uint8_t)((signbit(v) ? 0x80 : 0) | mag);
}

/* ------------------------------------------------------------------------ */
/* E8M0 -- [FP4] "The OCP Microscaling (MX) spec": exponent only, no sign,   */
/* range 2^-127 .. 2^127, one code for NaN.                                   */
/* ------------------------------------------------------------------------ */

float ora_e8m0_value(uint8_t code)
{
    if (code == 255)
        return NAN;
    return ldexpf(1.0f, (int)code - 127);
}

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as   */
/* easy as 1, 2, 3", SC'11): ten rounds of two 32x32->64 multiplies; the key */
/* is bumped by the Weyl constants between rounds.                            */
/* ------------------------------------------------------------------------ */

void ora_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; round++) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)c0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)c2;
        uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
        uint32_t n1 = (uint32_t)p1;
        uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
        uint32_t n3 = (uint32_t)p0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* R12: the 16-bit draw for output element idx of one stochastic-rounding
 * pass.  One Philox call covers 8 consecutive elements: counter =
 * (lo32(idx>>3), hi32(idx>>3), stream_id, 0), key = (lo32(seed), hi32(seed));
 * the element takes the low (idx even) or high (idx odd) half of word
 * (idx>>1)&3. */
uint16_t ora_sr_draw(uint64_t seed, uint32_t stream_id, uint64_t idx)
{
    uint64_t g = idx >> 3;
    uint32_t ctr[4] = {(uint32_t)g, (uint32_t)(g >> 32), stream_id, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t w[4];
    ora_philox4x32_10(ctr, key, w);
    uint32_t word = w[(idx >> 1) & 3];
    return (idx & 1) ? (uint16_t)(word >> 16) : (uint16_t)(word & 0xFFFFu);
}

/* R14: the RHT sign vector of a seed is bits 0..15 of word 0 of
 * Philox4x32-10(counter 0, key seed); bit i set means s_i = -1. */
uint16_t ora_rht_sign_mask(uint64_t seed)
{
    uint32_t ctr[4] = {0u, 0u, 0u, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t w[4];
    ora_philox4x32_10(ctr, key, w);
    return (uint16_t)(w[0] & 0xFFFFu);
}

/* ------------------------------------------------------------------------ */
/* Stochastic rounding to E4M3 -- [MX] "Words on this page": round up or     */
/* down at random in proportion to closeness; [TML] "A precision choice for  */
/* each stage": the expected value is preserved.                             */
/* v must already be clamped to [-448, 448].                                 */
/* ------------------------------------------------------------------------ */

uint8_t ora_e4m3_sr(float v, uint16_t r16)
{
    uint8_t s = signbit(v) ? 0x80 : 0;
    float a = fabsf(v);
    if (a == 0.0f)
        return s;
    int e2;
    frexpf(a, &e2);           /* a = f * 2^e2, f in [0.5, 1) */
    int fl = e2 - 1;          /* floor(log2 a) */
    int ue = (fl > -6 ? fl : -6) - 3;
    float ulp = ldexpf(1.0f, ue);            /* spacing of E4M3 around a */
    float lo = floorf(a / ulp) * ulp;        /* representable neighbour below */
    float frac = (a - lo) / ulp;             /* in [0, 1), exact */
    float u = (float)r16 * (1.0f / 65536.0f);
    float mag = (u < frac) ? lo + ulp : lo;
    return (uint8_t)(s | ora_e4m3_rne_sat(mag)); /* mag is representable */
}

/* ------------------------------------------------------------------------ */
/* Stochastic rounding to E2M1 -- [MX] "NVFP4": the NVFP4 pretraining recipe */
/* rounds gradients stochastically; [MX] "Words on this page": round up or   */
/* down at random in proportion to closeness.  Same rule and draws as the    */
/* E4M3 form (R12): with lo <= |v| < hi the neighbouring E2M1 values, round   */
/* up iff r16 * 2^-16 < (|v| - lo) / (hi - lo).  v must already be clamped to */
/* [-6, 6]; the sign bit is the sign of v (R5).                              */
/* ------------------------------------------------------------------------ */

uint8_t ora_e2m1_sr(float v, uint16_t r16)
{
    uint8_t s = signbit(v) ? 8 : 0;
    float a = fabsf(v);
    uint8_t c = 0;
    while (c < 7 && ora_e2m1_value((uint8_t)(c + 1)) <= a)
        c++;                                   /* E2M1(c) <= a < E2M1(c + 1) */
    if (c == 7)
        return (uint8_t)(s | 7);
    float lo = ora_e2m1_value(c), hi = ora_e2m1_value((uint8_t)(c + 1));
    float frac = (a - lo) / (hi - lo);         /* exact: the gap is 0.5, 1 or 2 */
    float u = (float)r16 * (1.0f / 65536.0f);
    return (uint8_t)(s | ((u < frac) ? c + 1 : c));
}

/* ------------------------------------------------------------------------ */
/* 16-point random Hadamard transform -- [MX] "NVFP4": random Hadamard       */
/* transforms bound block outliers; [TML] "Why communication became the next */
/* bottleneck": a random Hadamard rotation that the receiver reverses.       */
/* R14: y = 1/4 * H16 * diag(s) * x with H16 the Sylvester matrix,          */
/* H[i][j] = (-1)^popcount(i & j), evaluated by butterflies of stride 1, 2,   */
/* 4, 8 in that order, every add and subtract one binary32 operation.         */
/* ------------------------------------------------------------------------ */

void ora_rht16(const float x[16], uint16_t sign_mask, float y[16])
{
    float u[16];
    for (int i = 0; i < 16; i++)
        u[i] = ((sign_mask >> i) & 1) ? -x[i] : x[i];
    for (int h = 1; h < 16; h <<= 1) {
        for (int base = 0; base < 16; base += 2 * h) {
            for (int i = base; i < base + h; i++) {
                float a = u[i], b = u[i + h];
                u[i] = a + b;
                u[i + h] = a - b;
            }
        }
    }
    for (int i = 0; i < 16; i++)
        y[i] = 0.25f * u[i];
}

/* Load row `src` of a bf16 matrix into fp32, applying the RHT to each group of
 * 16 along K when enabled. */
static void load_row(const uint16_t *x, int64_t ldx, int64_t src, int64_t K,
                     int rht, uint16_t mask, float *out)
{
    const uint16_t *p = x + src * ldx;
    for (int64_t k = 0; k < K; k++)
        out[k] = ora_bf16_to_f32(p[k]);
    if (rht) {
        for (int64_t g = 0; g < K; g += 16) {
            float y[16];
            ora_rht16(out + g, mask, y);
            memcpy(out + g, y, sizeof y);
        }
    }
}

/* The fused path's RHT output, binary32, for every group of 16 along K of a
 * row-major M x K bf16 matrix (what the amax and NVFP4 passes consume). */
int ora_rht_f32(const uint16_t *x, float *y, int64_t M, int64_t K, uint16_t mask)
{
    if (K % 16)
        return 1;
    for (int64_t m = 0; m < M; m++)
        load_row(x, K, m, K, 1, mask, y + m * K);
    return 0;
}

/* Standalone RHT: bf16 in, bf16 (nearest-even) out, along K in groups of 16. */
int ora_rht_bf16(const uint16_t *x, uint16_t *y, int64_t M, int64_t K, int64_t ld, uint16_t mask)
{
    if (K % 16)
        return 1;
    float *row = (float *)malloc(sizeof(float) * (size_t)K);
    for (int64_t m = 0; m < M; m++) {
        load_row(x, ld, m, K, 1, mask, row);
        for (int64_t k = 0; k < K; k++)
            y[m * ld + k] = ora_f32_to_bf16(row[k]);
    }
    free(row);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Tensor amax -- the first level of NVFP4's two-level scale ([MX] "NVFP4":  */
/* a second-level per-tensor FP32 scale).  Exact max of |x| over fp32(bf16)  */
/* (after the RHT when enabled); row_index, when given, selects the rows.    */
/* ------------------------------------------------------------------------ */

float ora_amax(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
               int rht, uint16_t mask, const int32_t *row_index)
{
    float *row = (float *)malloc(sizeof(float) * (size_t)(K > 0 ? K : 1));
    float amax = 0.0f;
    for (int64_t m = 0; m < M; m++) {
        load_row(x, ldx, row_index ? row_index[m] : m, K, rht, mask, row);
        for (int64_t k = 0; k < K; k++) {
            float a = fabsf(row[k]);
            if (a > amax)
                amax = a;
        }
    }
    free(row);
    return amax;
}

/* ------------------------------------------------------------------------ */
/* NVFP4 quantize -- [MX] "NVFP4": E2M1 elements in blocks of 16, one E4M3   */
/* scale per block, one FP32 per-tensor scale; two-dimensional (16x16)       */
/* weight blocks.  [FP4] "The two Blackwell formats": group 16, E4M3 block   */
/* scale, FP32 per-tensor scale.  The configuration fixes                     */
/*   s_g = amax / (6 * 448),  s_b = E4M3_RNE(block_amax / 6 / s_g),           */
/* and the elements as E2M1 by nearest-even with saturation at +-6.         */
/* R2: amax == 0 gives s_g = 1.  R3: two binary32 divisions, left to right.  */
/* R4: each element is x * r with r = 1 / (fp32(s_b) * s_g), one reciprocal */
/* per block.  A block with s_b == 0 stores all codes +0.                     */
/* [TML] "A precision choice for each stage": Four Over Six picks between   */
/* two block scales to lower the quantization error.  R9: candidates         */
/* block_amax/6 and block_amax/4 (same s_g); error = sum of squared          */
/* (x - E2M1(code) * den) over a fixed pairwise tree; the /4 candidate wins   */
/* only if its error is strictly smaller.                                     */
/* Outputs: codes [M][K/2], element 2j in the low nibble of byte j (R24);    */
/* sf [M][K/16] canonical row-major E4M3 codes (a 16x16 tile's scale is      */
/* written for each of its 16 rows, R8).                                       */
/* ------------------------------------------------------------------------ */

typedef struct {
    float den;      /* fp32(s_b) * s_g */
    uint8_t sb;     /* E4M3 code */
    uint8_t code[16];
} nv_cand;

static void nv_candidate(const float *x, int n, float bamax, float divisor, float s_g, nv_cand *c)
{
    float t = (bamax / divisor) / s_g;
    c->sb = ora_e4m3_rne_sat(t);
    float sbv = ora_e4m3_value(c->sb);
    if (sbv == 0.0f) {
        c->den = 0.0f;
        for (int i = 0; i < n; i++)
            c->code[i] = 0;
        return;
    }
    c->den = sbv * s_g;
    float r = 1.0f / c->den;
    for (int i = 0; i < n; i++)
        c->code[i] = ora_e2m1_rne_sat(x[i] * r);
}

/* R9: squared error of a 1x16 candidate, summed pairwise: (0+1),(2+3),... then
 * pairs of those, four levels in all. */
static float nv_block_err(const float *x, const nv_cand *c)
{
    float e[16];
    for (int i = 0; i < 16; i++) {
        float deq = ora_e2m1_value(c->code[i]) * c->den;
        float d = x[i] - deq;
        e[i] = d * d;
    }
    for (int w = 16; w > 1; w >>= 1)
        for (int i = 0; i < w / 2; i++)
            e[i] = e[2 * i] + e[2 * i + 1];
    return e[0];
}

float ora_nvfp4_global_scale(float amax)
{
    return (amax == 0.0f) ? 1.0f : amax / 2688.0f;
}

/* R29 -- sr != 0: the elements are rounded stochastically instead (ora_e2m1_sr of
 * x * r clamped to +-6, the draw of output element m * K + k with the given
 * seed and stream id); block scales and s_g are unchanged.  Not combined with
 * Four Over Six.  row0 is the index, in the whole output tensor, of the first
 * output row computed here (0 for a whole tensor): it only offsets the draw
 * index, so a band of rows can be computed on its own. */
static int quant_nvfp4_impl(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                            int block_2d, int four_over_six, int rht, uint16_t mask,
                            const int32_t *row_index, const float *amax_in,
                            int sr, uint64_t seed, uint32_t stream_id, int64_t row0,
                            float *s_g_out, uint8_t *codes, uint8_t *sf)
{
    if (K % 16 || (block_2d && M % 16) || (block_2d && four_over_six) || (sr && four_over_six))
        return 1;
    float amax = amax_in ? *amax_in : ora_amax(x, M, K, ldx, rht, mask, row_index);
    float s_g = ora_nvfp4_global_scale(amax);
    *s_g_out = s_g;
    int64_t KB = K / 16;
    int64_t stripe = block_2d ? 16 : 1;
    float *buf = (float *)malloc(sizeof(float) * (size_t)(stripe * (K > 0 ? K : 1)));
    for (int64_t m0 = 0; m0 < M; m0 += stripe) {
        for (int64_t r = 0; r < stripe; r++) {
            int64_t m = m0 + r;
            load_row(x, ldx, row_index ? row_index[m] : m, K, rht, mask, buf + r * K);
        }
        for (int64_t kb = 0; kb < KB; kb++) {
            float bamax = 0.0f;
            for (int64_t r = 0; r < stripe; r++)
                for (int i = 0; i < 16; i++) {
                    float a = fabsf(buf[r * K + kb * 16 + i]);
                    if (a > bamax)
                        bamax = a;
                }
            for (int64_t r = 0; r < stripe; r++) {
                const float *xb = buf + r * K + kb * 16;
                nv_cand c6, c4;
                nv_candidate(xb, 16, bamax, 6.0f, s_g, &c6);
                const nv_cand *pick = &c6;
                if (four_over_six) {
                    nv_candidate(xb, 16, bamax, 4.0f, s_g, &c4);
                    if (nv_block_err(xb, &c4) < nv_block_err(xb, &c6))
                        pick = &c4;
                }
                int64_t m = m0 + r;
                if (sr && c6.den != 0.0f) {
                    float rc = 1.0f / c6.den;
                    for (int i = 0; i < 16; i++) {
                        float q = xb[i] * rc;
                        if (q > 6.0f)
                            q = 6.0f;
                        if (q < -6.0f)
                            q = -6.0f;
                        c6.code[i] = ora_e2m1_sr(q, ora_sr_draw(seed, stream_id,
                                                                (uint64_t)((row0 + m) * K + kb * 16 + i)));
                    }
                }
                sf[m * KB + kb] = pick->sb;
                for (int i = 0; i < 16; i += 2)
                    codes[m * (K / 2) + kb * 8 + i / 2] =
                        (uint8_t)(pick->code[i] | (pick->code[i + 1] << 4));
            }
        }
    }
    free(buf);
    return 0;
}

int ora_quant_nvfp4(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                    int block_2d, int four_over_six, int rht, uint16_t mask,
                    const int32_t *row_index, const float *amax_in,
                    float *s_g_out, uint8_t *codes, uint8_t *sf)
{
    return quant_nvfp4_impl(x, M, K, ldx, block_2d, four_over_six, rht, mask, row_index, amax_in,
                            0, 0, 0, 0, s_g_out, codes, sf);
}

int ora_quant_nvfp4_sr_rows(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                            int block_2d, int rht, uint16_t mask,
                            const int32_t *row_index, const float *amax_in,
                            uint64_t seed, uint32_t stream_id, int64_t row0,
                            float *s_g_out, uint8_t *codes, uint8_t *sf)
{
    return quant_nvfp4_impl(x, M, K, ldx, block_2d, 0, rht, mask, row_index, amax_in,
                            1, seed, stream_id, row0, s_g_out, codes, sf);
}

int ora_quant_nvfp4_sr(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                       int block_2d, int rht, uint16_t mask,
                       const int32_t *row_index, const float *amax_in,
                       uint64_t seed, uint32_t stream_id,
                       float *s_g_out, uint8_t *codes, uint8_t *sf)
{
    return ora_quant_nvfp4_sr_rows(x, M, K, ldx, block_2d, rht, mask, row_index, amax_in,
                                   seed, stream_id, 0, s_g_out, codes, sf);
}

/* ------------------------------------------------------------------------ */
/* MXFP4 quantize -- [FP4] "The two Blackwell formats": E2M1 elements in     */
/* groups of 32 with one E8M0 (power-of-two) scale, 4 + 8/32 = 4.25 bits;    */
/* [MX] "Microscaling": the block shares one exponent.  R28 (the pages give  */
/* no scale rule): as MXFP8's 2^(floor(log2 amax) - 8), with E2M1's largest  */
/* exponent in place of E4M3's -- 6 = 1.5 * 2^2 -- so E = floor(log2 amax)   */
/* - 2, clamped to [-127, 127]; elements x * 2^-E clamped to +-6 (values in  */
/* (6, 8) * 2^E saturate), then nearest-even or stochastic rounding (draw of */
/* output element r * K + k).  An all-zero block has scale code 0 and codes  */
/* +0.  Outputs: codes [M][K/2] (element 2j in the low nibble of byte j),    */
/* sf [M][K/32] canonical E8M0 codes.                                         */
/* ------------------------------------------------------------------------ */

int ora_quant_mxfp4_rows(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, int sr,
                         uint64_t seed, uint32_t stream_id, int64_t row0, uint8_t *codes, uint8_t *sf)
{
    if (K % 32)
        return 1;
    for (int64_t r = 0; r < M; r++) {
        for (int64_t kb = 0; kb < K / 32; kb++) {
            float v[32], bamax = 0.0f;
            for (int i = 0; i < 32; i++) {
                v[i] = ora_bf16_to_f32(x[r * ldx + kb * 32 + i]);
                if (fabsf(v[i]) > bamax)
                    bamax = fabsf(v[i]);
            }
            uint8_t c[32];
            if (bamax == 0.0f) {
                sf[r * (K / 32) + kb] = 0;
                memset(c, 0, sizeof c);
            } else {
                int e2;
                frexpf(bamax, &e2);
                int E = (e2 - 1) - 2;
                if (E < -127)
                    E = -127;
                if (E > 127)
                    E = 127;
                sf[r * (K / 32) + kb] = (uint8_t)(E + 127);
                for (int i = 0; i < 32; i++) {
                    float q = ldexpf(v[i], -E);
                    if (q > 6.0f)
                        q = 6.0f;
                    if (q < -6.0f)
                        q = -6.0f;
                    c[i] = sr ? ora_e2m1_sr(q, ora_sr_draw(seed, stream_id, (uint64_t)((row0 + r) * K + kb * 32 + i)))
                              : ora_e2m1_rne_sat(q);
                }
            }
            for (int i = 0; i < 32; i += 2)
                codes[r * (K / 2) + kb * 16 + i / 2] = (uint8_t)(c[i] | (c[i + 1] << 4));
        }
    }
    return 0;
}

/* The whole tensor (row0 = 0); ora_quant_mxfp4_rows computes a band of rows
 * whose first row is row row0 of the whole output (the SR draw index). */
int ora_quant_mxfp4(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, int sr,
                    uint64_t seed, uint32_t stream_id, uint8_t *codes, uint8_t *sf)
{
    return ora_quant_mxfp4_rows(x, M, K, ldx, sr, seed, stream_id, 0, codes, sf);
}

/* ------------------------------------------------------------------------ */
/* MXFP8 quantize -- [RL] "Recipe 1": 32 consecutive E4M3 share one E8M0     */
/* scale, one-dimensional blocks; [MX] "Microscaling": the shared scale is a  */
/* pure power of two.  The configuration fixes scale = 2^(floor(log2 amax)-8). */
/* R10: floor(log2) from the binary32 exponent (frexp), clamped to           */
/* [-127, 127]; elements x * 2^-E, clamped to +-448, then nearest-even or    */
/* stochastic rounding.  An all-zero block has scale code 0 and codes +0.    */
/* A block is 32 consecutive elements of an output row; idx0 is the output   */
/* row-major linear index of its first element (used for the SR draw).       */
/* ------------------------------------------------------------------------ */

static uint8_t mx_block(const float v[32], int sr, uint64_t seed, uint32_t sid,
                        uint64_t idx0, uint8_t out[32])
{
    float bamax = 0.0f;
    for (int i = 0; i < 32; i++) {
        float a = fabsf(v[i]);
        if (a > bamax)
            bamax = a;
    }
    if (bamax == 0.0f) {
        for (int i = 0; i < 32; i++)
            out[i] = 0;
        return 0;
    }
    int e2;
    frexpf(bamax, &e2);
    int E = (e2 - 1) - 8;
    if (E < -127)
        E = -127;
    if (E > 127)
        E = 127;
    for (int i = 0; i < 32; i++) {
        float s = ldexpf(v[i], -E);
        if (s > 448.0f)
            s = 448.0f;
        if (s < -448.0f)
            s = -448.0f;
        out[i] = sr ? ora_e4m3_sr(s, ora_sr_draw(seed, sid, idx0 + (uint64_t)i))
                    : ora_e4m3_rne_sat(s);
    }
    return (uint8_t)(E + 127);
}

/* Quantize x [M][K] (bf16) to MXFP8.  colwise == 0: output codes [M][K], sf
 * [M][K/32]; colwise == 1: output is the quantization of x^T, codes [K][M],
 * sf [K][M/32] (blocks of 32 along the original M).  out_row0 is the index,
 * in the full output tensor, of the first output row computed here (0 for a
 * whole tensor): it only offsets the element indices of the SR draws, so a
 * band of output rows can be computed on its own. */
int ora_quant_mxfp8_rows(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, int colwise,
                         int sr, uint64_t seed, uint32_t stream_id, int64_t out_row0,
                         uint8_t *codes, uint8_t *sf)
{
    int64_t R = colwise ? K : M, C = colwise ? M : K;
    if (C % 32)
        return 1;
    float v[32];
    for (int64_t r = 0; r < R; r++) {
        for (int64_t cb = 0; cb < C / 32; cb++) {
            for (int i = 0; i < 32; i++) {
                int64_t c = cb * 32 + i;
                v[i] = colwise ? ora_bf16_to_f32(x[c * ldx + r]) : ora_bf16_to_f32(x[r * ldx + c]);
            }
            sf[r * (C / 32) + cb] = mx_block(v, sr, seed, stream_id,
                                             (uint64_t)((out_row0 + r) * C + cb * 32), codes + r * C + cb * 32);
        }
    }
    return 0;
}

int ora_quant_mxfp8(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, int colwise,
                    int sr, uint64_t seed, uint32_t stream_id, uint8_t *codes, uint8_t *sf)
{
    return ora_quant_mxfp8_rows(x, M, K, ldx, colwise, sr, seed, stream_id, 0, codes, sf);
}

/* ------------------------------------------------------------------------ */
/* Dequantize -> transpose -> requantize -- [TML] "A precision choice for    */
/* each stage": saved values are dequantized, transposed at higher precision  */
/* and stochastically re-quantized to MXFP8.  R15: the new blocks are 32     */
/* consecutive old-M indices.  The dequantized value E4M3(code) * 2^E is     */
/* exact in binary32 (inputs must keep it finite).                            */
/* ------------------------------------------------------------------------ */

int ora_requant_transpose_rows(const uint8_t *codes_row, const uint8_t *sf_row, int64_t M, int64_t K,
                               int sr, uint64_t seed, uint32_t stream_id, int64_t k0, int64_t k1,
                               uint8_t *codes_col, uint8_t *sf_col)
{
    if (K % 32 || M % 32 || k0 < 0 || k1 > K || k0 > k1)
        return 1;
    float v[32];
    for (int64_t k = k0; k < k1; k++) {
        for (int64_t mb = 0; mb < M / 32; mb++) {
            for (int i = 0; i < 32; i++) {
                int64_t m = mb * 32 + i;
                v[i] = ora_e4m3_value(codes_row[m * K + k]) * ora_e8m0_value(sf_row[m * (K / 32) + k / 32]);
            }
            sf_col[k * (M / 32) + mb] =
                mx_block(v, sr, seed, stream_id, (uint64_t)(k * M + mb * 32), codes_col + k * M + mb * 32);
        }
    }
    return 0;
}

/* The whole output (rows 0 .. K-1); ora_requant_transpose_rows computes output
 * rows k0 .. k1-1 only, into the same full-size output arrays. */
int ora_requant_transpose(const uint8_t *codes_row, const uint8_t *sf_row, int64_t M, int64_t K,
                          int sr, uint64_t seed, uint32_t stream_id,
                          uint8_t *codes_col, uint8_t *sf_col)
{
    return ora_requant_transpose_rows(codes_row, sf_row, M, K, sr, seed, stream_id, 0, K, codes_col, sf_col);
}

/* ------------------------------------------------------------------------ */
/* NVFP4 -> MXFP8 column-wise requantize -- [TML] "A precision choice for   */
/* each stage": tensors saved in the forward pass (NVFP4, the weights in     */
/* 16x16 blocks) are dequantized, transposed at higher precision and         */
/* requantized to MXFP8 for the backward pass.  R30: the dequantized value   */
/* is binary32 RN((E2M1(code) * E4M3(s_b)) * s_g) -- the first product is    */
/* exact (at most six significant bits), the multiply by the FP32 tensor    */
/* scale rounds once; the transpose's rows are then quantized to MXFP8 as   */
/* in ora_quant_mxfp8 (blocks of 32 along the old rows, RNE or SR with the  */
/* draw of output element c * R + r).  Input: codes [R][C/2], canonical sf  */
/* [R][C/16], s_g; output rows c0 .. c1-1 of codes_out [C][R] and sf_out    */
/* [C][R/32].                                                                 */
/* ------------------------------------------------------------------------ */

int ora_requant_nvfp4_mxfp8_rows(const uint8_t *codes, const uint8_t *sf, float s_g, int64_t R, int64_t C,
                                 int sr, uint64_t seed, uint32_t stream_id, int64_t c0, int64_t c1,
                                 uint8_t *codes_out, uint8_t *sf_out)
{
    if (R % 32 || C % 16 || c0 < 0 || c1 > C || c0 > c1)
        return 1;
    float v[32];
    for (int64_t c = c0; c < c1; c++) {
        for (int64_t rb = 0; rb < R / 32; rb++) {
            for (int i = 0; i < 32; i++) {
                int64_t r = rb * 32 + i;
                uint8_t byte = codes[r * (C / 2) + c / 2];
                uint8_t e2 = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
                float elem_scale = ora_e2m1_value(e2) * ora_e4m3_value(sf[r * (C / 16) + c / 16]);
                v[i] = elem_scale * s_g;
            }
            sf_out[c * (R / 32) + rb] = mx_block(v, sr, seed, stream_id, (uint64_t)(c * R + rb * 32),
                                                 codes_out + c * R + rb * 32);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* S2F6 combine compression -- [TML] "Why communication became the next     */
/* bottleneck": the combined MoE outputs are rotated by a random Hadamard   */
/* transform, sent in block-scaled S2F6 ("an 8-bit fixed-point format") at  */
/* 8.25 bits per value, and the receiver reconstructs and combines them,     */
/* then reverses the transform.                                               */
/* R34: S2F6 is two's-complement fixed point with two integer bits (the     */
/* sign among them) and six fraction bits: code q in [-128, 127], value     */
/* q / 64.  R35: 32 consecutive values share one E8M0 scale (8 + 8/32 =     */
/* 8.25 bits): E = floor(log2 block_amax) clamped to [-127, 127], so that   */
/* block_amax / 2^E lies in [1, 2); q = nearest-even integer of            */
/* x * 2^(6 - E) (exact scaling), clamped to [-128, 127]; an all-zero block  */
/* has scale code 0 and zero codes.  The transform is the 16-point RHT of    */
/* R14 applied first (binary32).                                             */
/* ------------------------------------------------------------------------ */

static int8_t s2f6_round(float s)
{
    float r = rintf(s); /* the default rounding mode: nearest, ties to even */
    if (r > 127.0f)
        r = 127.0f;
    if (r < -128.0f)
        r = -128.0f;
    return (int8_t)r;
}

int ora_quant_s2f6(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, int rht, uint16_t mask,
                   int8_t *codes, uint8_t *sf)
{
    if (K % 32)
        return 1;
    float *row = (float *)malloc(sizeof(float) * (size_t)K);
    for (int64_t m = 0; m < M; m++) {
        load_row(x, ldx, m, K, rht, mask, row);
        for (int64_t b = 0; b < K / 32; b++) {
            float bamax = 0.0f;
            for (int i = 0; i < 32; i++)
                if (fabsf(row[b * 32 + i]) > bamax)
                    bamax = fabsf(row[b * 32 + i]);
            if (bamax == 0.0f) {
                sf[m * (K / 32) + b] = 0;
                for (int i = 0; i < 32; i++)
                    codes[m * K + b * 32 + i] = 0;
                continue;
            }
            int e2;
            frexpf(bamax, &e2);
            int E = e2 - 1;
            if (E < -127)
                E = -127;
            if (E > 127)
                E = 127;
            sf[m * (K / 32) + b] = (uint8_t)(E + 127);
            for (int i = 0; i < 32; i++)
                codes[m * K + b * 32 + i] = s2f6_round(ldexpf(row[b * 32 + i], 6 - E));
        }
    }
    free(row);
    return 0;
}

/* R36, the receiver: token t's output is the sum, over the rows listed for
 * it (rows[off[t]] .. rows[off[t+1]-1], in that order), of weight * value
 * (binary32: each value q / 64 * 2^E is exact, each product and each
 * addition one RN operation), then the inverse transform of each group of
 * 16: x = 1/4 * D * H16 * acc (butterflies of stride 1, 2, 4, 8, RN; the
 * quarter and the signs exact), rounded once to bf16 (nearest-even). */
int ora_combine_s2f6(const int8_t *codes, const uint8_t *sf, int64_t K, const int32_t *off,
                     const int32_t *rows, const float *weights, int64_t T, uint16_t mask, uint16_t *out)
{
    if (K % 32)
        return 1;
    float *acc = (float *)malloc(sizeof(float) * (size_t)K);
    for (int64_t t = 0; t < T; t++) {
        for (int64_t k = 0; k < K; k++)
            acc[k] = 0.0f;
        for (int32_t j = off[t]; j < off[t + 1]; j++) {
            const int64_t r = rows[j];
            for (int64_t k = 0; k < K; k++) {
                float v = ldexpf((float)codes[r * K + k], (int)sf[r * (K / 32) + k / 32] - 127 - 6);
                acc[k] = acc[k] + weights[j] * v;
            }
        }
        for (int64_t g = 0; g < K; g += 16) {
            float u[16];
            for (int i = 0; i < 16; i++)
                u[i] = acc[g + i];
            for (int h = 1; h < 16; h <<= 1)
                for (int base = 0; base < 16; base += 2 * h)
                    for (int i = base; i < base + h; i++) {
                        float a = u[i], b = u[i + h];
                        u[i] = a + b;
                        u[i + h] = a - b;
                    }
            for (int i = 0; i < 16; i++) {
                float y = 0.25f * u[i];
                out[t * K + g + i] = ora_f32_to_bf16(((mask >> i) & 1) ? -y : y);
            }
        }
    }
    free(acc);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Scale-factor layout for the tensor-core MMA -- [MX] "Hardware and         */
/* kernels": a block-scaled GEMM needs a particular scale-factor memory      */
/* layout; the pages do not give it.  R23 (Blackwell block-scaled MMA        */
/* layout): 128-row x 4-block atoms of 512 bytes; inside an atom, row r and  */
/* block b sit at (r % 32) * 16 + (r / 32) * 4 + b; atoms are ordered row-   */
/* tile major, then block tile.  Rows pad to 128 and blocks to 4, with zero. */
/* ------------------------------------------------------------------------ */

int64_t ora_sf_swizzled_bytes(int64_t rows, int64_t nblk)
{
    int64_t rp = (rows + 127) / 128 * 128, bp = (nblk + 3) / 4 * 4;
    return rp * bp;
}

int64_t ora_sf_offset(int64_t r, int64_t b, int64_t nblk)
{
    int64_t bt = (nblk + 3) / 4;
    int64_t atom = (r / 128) * bt + b / 4;
    return atom * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + (b % 4);
}

void ora_sf_swizzle(const uint8_t *sf, int64_t rows, int64_t nblk, uint8_t *out)
{
    memset(out, 0, (size_t)ora_sf_swizzled_bytes(rows, nblk));
    for (int64_t r = 0; r < rows; r++)
        for (int64_t b = 0; b < nblk; b++)
            out[ora_sf_offset(r, b, nblk)] = sf[r * nblk + b];
}

void ora_sf_unswizzle(const uint8_t *in, int64_t rows, int64_t nblk, uint8_t *sf)
{
    for (int64_t r = 0; r < rows; r++)
        for (int64_t b = 0; b < nblk; b++)
            sf[r * nblk + b] = in[ora_sf_offset(r, b, nblk)];
}

/* ------------------------------------------------------------------------ */
/* Decode and GEMM -- [MX] "Microscaling": a block decodes as scale x        */
/* element; NVFP4 multiplies the per-tensor scale too ([MX] "NVFP4").         */
/* [MX] "Hardware and kernels": the tensor core applies the scales inside    */
/* the matrix instruction; the oracle instead decodes to binary64 (exact)    */
/* and sums in binary64, k ascending.                                          */
/* fmt 0 = NVFP4 (codes [R][K/2], sf [R][K/16] canonical, s_g),              */
/* fmt 1 = MXFP8 (codes [R][K], sf [R][K/32] canonical).                      */
/* ------------------------------------------------------------------------ */

static double decode_one(int fmt, const uint8_t *codes, const uint8_t *sf, float s_g,
                         int64_t K, int64_t r, int64_t k)
{
    if (fmt == 0) {
        uint8_t byte = codes[r * (K / 2) + k / 2];
        uint8_t c = (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
        return (double)ora_e2m1_value(c) * (double)ora_e4m3_value(sf[r * (K / 16) + k / 16]) * (double)s_g;
    }
    if (fmt == 2) { /* MXFP4 */
        uint8_t byte = codes[r * (K / 2) + k / 2];
        uint8_t c = (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
        return (double)ora_e2m1_value(c) * (double)ora_e8m0_value(sf[r * (K / 32) + k / 32]);
    }
    return (double)ora_e4m3_value(codes[r * K + k]) * (double)ora_e8m0_value(sf[r * (K / 32) + k / 32]);
}

void ora_dequant(int fmt, const uint8_t *codes, const uint8_t *sf, float s_g,
                 int64_t R, int64_t K, double *out)
{
    for (int64_t r = 0; r < R; r++)
        for (int64_t k = 0; k < K; k++)
            out[r * K + k] = decode_one(fmt, codes, sf, s_g, K, r, k);
}

/* C[m][n] = sum_k A[m][k] * B[n][k] and ref_abs = sum_k |A[m][k] B[n][k]|. */
void ora_gemm_f64(const double *A, const double *B, int64_t M, int64_t N, int64_t K,
                  double *C, double *ref_abs)
{
    for (int64_t m = 0; m < M; m++)
        for (int64_t n = 0; n < N; n++) {
            double s = 0.0, sa = 0.0;
            for (int64_t k = 0; k < K; k++) {
                double p = A[m * K + k] * B[n * K + k];
                s += p;
                sa += fabs(p);
            }
            C[m * N + n] = s;
            ref_abs[m * N + n] = sa;
        }
}

/* The same sum for a list of (m, n) points, decoding quantized operands on
 * the fly (no dequantized copy of a large operand is made). */
void ora_gemm_points(int fmt, const uint8_t *codesA, const uint8_t *sfA, float sgA,
                     const uint8_t *codesB, const uint8_t *sfB, float sgB, int64_t K,
                     int64_t npts, const int64_t *pm, const int64_t *pn,
                     double *C, double *ref_abs)
{
    for (int64_t p = 0; p < npts; p++) {
        double s = 0.0, sa = 0.0;
        for (int64_t k = 0; k < K; k++) {
            double prod = decode_one(fmt, codesA, sfA, sgA, K, pm[p], k) *
                          decode_one(fmt, codesB, sfB, sgB, K, pn[p], k);
            s += prod;
            sa += fabs(prod);
        }
        C[p] = s;
        ref_abs[p] = sa;
    }
}
