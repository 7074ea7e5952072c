/*
 * wq_oracle.c -- TEST INFRASTRUCTURE, not part of the library.
 *
 * A plain, slow, single-threaded CPU restatement of per-group round-to-nearest
 * (RTN) weight quantization and of the W4A16 decode linear that consumes it.
 * Only the tests, the smoke check and the CPU-baseline leg of the benchmark
 * load this file; the CUDA library never includes, links or calls it, and it
 * shares no code, header or table with the CUDA library.
 *
 * Sources (page title, then section / equation):
 *   [PTQ]   "后训练量化（PTQ, Post-Training Quantization）", section 基础量化公式
 *           (q = round(x/s)+z, x_hat = s(q-z), s = (max-min)/(2^b-1),
 *           z = round(-min/s); symmetric z = 0, s = max|x|/(2^(b-1)-1)),
 *           section 量化粒度 (per-group, group_size = 128), section AWQ
 *           (W' = W diag(s), Y = X diag(s)^-1 quant(W')).
 *   [3.6]   "3.6 量化(Quantization)", section 对称与非对称量化 (both
 *           closed forms, clamp to [-qmax, qmax] / [0, 2^b-1], error <= s/2),
 *           section 粒度 (G = 128 along the input dimension), section 代码
 *           (division by s, round half to even, range floor 1e-8, fp32),
 *           section 实例演算 (worked 8-value example).
 *   [Comp]  "量化" (AI 推理 compendium, ch. 17.01), section 量化方程
 *           (x_q = clamp(round(x/scale)+zero_point, q_min, q_max)).
 *   [Pano]  "大模型量化全景解析", section 粒度和矩阵维度的关系
 *           (Y = X W^T, W: [out_features, in_features], groups along
 *           in_features), section dtype、storage dtype、compute dtype.
 *
 * Readings taken where the pages are silent:
 *   - the integer codes are computed with the fp16-rounded scale s16 (the
 *     stored one) and, for the asymmetric form, with the fp16-stored zero z16,
 *     so the stored metadata reproduce x_hat exactly;
 *   - a zero point of 0 is stored as +0;
 *   - an fp16 scale that underflows to 0 is replaced by the smallest fp16
 *     subnormal 2^-24;
 *   - a group holding a non-finite value, or whose fp16 scale or zero
 *     overflows, is "non-finite": it is counted, its stored nibbles are 0 and
 *     its scale (and zero) are the fp16 quiet NaN 0x7E00.
 *
 * Floating point: quantization runs in fp32 (the pages' code works on fp32
 * tensors); the linear is accumulated in fp64.  Build with
 * -ffp-contract=off so no multiply-add is fused behind our back.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

/* ------------------------------------------------------------------ */
/* Number formats                                                       */
/* ------------------------------------------------------------------ */

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
float or_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* IEEE 754 binary16 -> double, exact, written from the format definition:
 * 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double or_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int ex = (h >> 10) & 0x1F;
    int fr = h & 0x3FF;
    double v;
    if (ex == 0x1F)
        v = fr ? NAN : INFINITY;
    else if (ex == 0)
        v = ldexp((double)fr, -24);                 /* subnormal: fr * 2^-24 */
    else
        v = ldexp((double)(fr | 0x400), ex - 25);   /* (1024+fr) * 2^(ex-25) */
    return sign ? -v : v;
}

float or_f16_to_f32(uint16_t h) { return (float)or_f16_to_f64(h); }

void or_f16_to_f64_array(const uint16_t* h, double* out, int64_t n)
{
    for (int64_t i = 0; i < n; i++) out[i] = or_f16_to_f64(h[i]);
}

/* binary32 -> binary16, round to nearest, ties to even, written from the
 * format definition.  |f| is first written exactly as m * 2^e (m an
 * integer); the binary16 quantum at that magnitude is 2^(floor(log2|f|)-10)
 * in the normal range and 2^-24 below it; |f| / quantum is rounded to an
 * integer n with ties to even, and n is encoded (n = 2048 carries into the
 * next binade, a biased exponent of 31 or more is infinity). */
uint16_t or_f32_to_f16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t ex = (u >> 23) & 0xFFu, fr = u & 0x7FFFFFu;
    if (ex == 0xFF)
        return (uint16_t)(sign | (fr ? 0x7E00u : 0x7C00u));
    if (ex == 0 && fr == 0)
        return sign;

    uint64_t m;
    int e;
    if (ex == 0) { m = fr; e = -149; }
    else         { m = fr | 0x800000u; e = (int)ex - 150; }

    int lg = e;                         /* floor(log2 |f|) */
    for (uint64_t t = m; t > 1; t >>= 1) lg++;
    int qe = (lg >= -14) ? lg - 10 : -24;

    uint64_t n;
    if (e >= qe) {
        n = m << (e - qe);
    } else {
        int sh = qe - e;
        if (sh > 40) {
            n = 0;                      /* far below half a quantum */
        } else {
            uint64_t q = m >> sh;
            uint64_t rem = m & ((1ull << sh) - 1);
            uint64_t half = 1ull << (sh - 1);
            n = q + ((rem > half || (rem == half && (q & 1))) ? 1 : 0);
        }
    }
    if (n == 0)
        return sign;
    if (n < 1024)                       /* only reachable with qe == -24 */
        return (uint16_t)(sign | n);
    if (n == 2048) { n = 1024; qe += 1; }
    int be = qe + 25;                   /* value = n * 2^qe, n in [1024,2047] */
    if (be >= 31)
        return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | ((uint32_t)be << 10) | (uint32_t)(n - 1024));
}

void or_f32_to_f16_array(const float* x, uint16_t* h, int64_t n)
{
    for (int64_t i = 0; i < n; i++) h[i] = or_f32_to_f16(x[i]);
}

/* Round to the nearest integer, ties to even (the rounding of the pages'
 * torch.round / jnp.round).  Values of magnitude >= 2^23 are integers. */
float or_round_half_even(float v)
{
    if (!(fabsf(v) < 8388608.0f))
        return v;
    float fl = floorf(v);
    float d = v - fl;                   /* exact: 0 <= d < 1 */
    if (d > 0.5f) return fl + 1.0f;
    if (d < 0.5f) return fl;
    return (fmodf(fl, 2.0f) == 0.0f) ? fl : fl + 1.0f;
}

static int is_f16_inf_or_nan(uint16_t h) { return (h & 0x7C00u) == 0x7C00u; }

/* ------------------------------------------------------------------ */
/* Per-group RTN quantization ([PTQ] 基础量化公式, [3.6] 对称与非对称量化,  */
/* [Comp] 量化方程), generic bit width b and group size G.               */
/* ------------------------------------------------------------------ */

/* w: fp32 [rows][cols], groups of G consecutive columns (G divides cols).
 * Outputs per element the signed integer code q (symmetric: [-qmax, qmax],
 * qmax = 2^(b-1)-1; asymmetric: [0, 2^b-1]); per group the fp16 scale s16
 * and, asymmetric only, the fp16 zero z16 (z16 may be NULL when sym).
 * Returns the number of non-finite groups. */
int64_t or_quantize_f32(const float* w, int64_t rows, int64_t cols, int64_t G,
                        int bits, int sym, int32_t* q, uint16_t* s16, uint16_t* z16)
{
    const int qmax_sym = (1 << (bits - 1)) - 1;
    const int qlo = sym ? -qmax_sym : 0;
    const int qhi = sym ? qmax_sym : (1 << bits) - 1;
    const float qden = sym ? (float)qmax_sym : (float)((1 << bits) - 1);
    const int64_t NG = cols / G;
    int64_t bad_groups = 0;

    for (int64_t r = 0; r < rows; r++) {
        for (int64_t g = 0; g < NG; g++) {
            const float* v = w + r * cols + g * G;
            int32_t* qo = q + r * cols + g * G;
            int bad = 0;

            /* group range: max|w| (sym) or min, max (asym), exact in fp32 */
            float amax = 0.0f, mn = v[0], mx = v[0];
            for (int64_t i = 0; i < G; i++) {
                if (!isfinite(v[i])) bad = 1;
                float a = fabsf(v[i]);
                if (a > amax) amax = a;
                if (v[i] < mn) mn = v[i];
                if (v[i] > mx) mx = v[i];
            }

            uint16_t hs = 0, hz = 0;
            float sf = 0.0f, zf = 0.0f;
            if (!bad) {
                float range = sym ? amax : (mx - mn);
                if (range < 1e-8f) range = 1e-8f;          /* clamp(min=1e-8) */
                float s32 = range / qden;                   /* IEEE fp32 division */
                hs = or_f32_to_f16(s32);
                if (hs == 0) hs = 0x0001;                   /* underflow -> 2^-24 */
                if (is_f16_inf_or_nan(hs)) bad = 1;
                sf = or_f16_to_f32(hs);
            }
            if (!bad && !sym) {
                zf = or_round_half_even(-mn / sf) + 0.0f;   /* +0.0 turns -0 into +0 */
                hz = or_f32_to_f16(zf);
                if (is_f16_inf_or_nan(hz)) bad = 1;
                zf = or_f16_to_f32(hz);
            }

            if (bad) {
                bad_groups++;
                for (int64_t i = 0; i < G; i++) qo[i] = sym ? -(1 << (bits - 1)) : 0;
                s16[r * NG + g] = 0x7E00;
                if (!sym) z16[r * NG + g] = 0x7E00;
                continue;
            }
            for (int64_t i = 0; i < G; i++) {
                float t = or_round_half_even(v[i] / sf) + zf;
                if (t < (float)qlo) t = (float)qlo;
                if (t > (float)qhi) t = (float)qhi;
                qo[i] = (int32_t)t;
            }
            s16[r * NG + g] = hs;
            if (!sym) z16[r * NG + g] = hz;
        }
    }
    return bad_groups;
}

/* The weight-side AWQ fold ([PTQ] AWQ step 3, [3.6] AWQ): w'[n][k] = w[n][k] *
 * s[k], one fp32 product rounded to nearest. */
void or_awq_fold_weight(const float* w, const float* s, int64_t rows, int64_t cols, float* out)
{
    for (int64_t r = 0; r < rows; r++)
        for (int64_t k = 0; k < cols; k++)
            out[r * cols + k] = w[r * cols + k] * s[k];
}

/* 4-bit RTN of a bf16 weight matrix W [N][K] (row n = output channel,
 * groups along the input dimension K, [Pano] 粒度和矩阵维度的关系), with
 * the optional AWQ per-input-channel scale folded in first. */
int64_t or_quantize_bf16(const uint16_t* W, const float* awq_s, int64_t N, int64_t K,
                         int64_t G, int sym, int32_t* q, uint16_t* s16, uint16_t* z16)
{
    int64_t bad = 0;
    float* row = (float*)malloc((size_t)K * sizeof(float));   /* one row at a time */
    if (!row) return -1;
    for (int64_t n = 0; n < N; n++) {
        for (int64_t k = 0; k < K; k++) row[k] = or_bf16_to_f32(W[n * K + k]);
        if (awq_s) or_awq_fold_weight(row, awq_s, 1, K, row);
        bad += or_quantize_f32(row, 1, K, G, 4, sym, q + n * K, s16 + n * (K / G),
                               sym ? NULL : z16 + n * (K / G));
    }
    free(row);
    return bad;
}

/* ------------------------------------------------------------------ */
/* uint4 packing: element k = 8j + i of a row lives in bits [4i, 4i+4) of  */
/* word j of that row; symmetric codes are stored as q + 8.              */
/* ------------------------------------------------------------------ */

void or_pack_u4(const int32_t* q, int64_t N, int64_t K, int sym, uint32_t* P)
{
    for (int64_t n = 0; n < N; n++)
        for (int64_t j = 0; j < K / 8; j++) {
            uint32_t word = 0;
            for (int i = 0; i < 8; i++) {
                int32_t c = q[n * K + 8 * j + i] + (sym ? 8 : 0);
                word |= ((uint32_t)c & 0xFu) << (4 * i);
            }
            P[n * (K / 8) + j] = word;
        }
}

void or_unpack_u4(const uint32_t* P, int64_t N, int64_t K, int sym, int32_t* q)
{
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) {
            uint32_t word = P[n * (K / 8) + k / 8];
            int32_t c = (int32_t)((word >> (4 * (k % 8))) & 0xFu);
            q[n * K + k] = c - (sym ? 8 : 0);
        }
}

/* ------------------------------------------------------------------ */
/* Dequantization and the W4A16 linear                                  */
/* ------------------------------------------------------------------ */

/* x_hat = s16 * (q - z16) for one row, in fp64 (exact: an 11-bit fp16
 * significand times an integer of at most a few bits). */
static void dequant_row(const uint32_t* Prow, const uint16_t* srow, const uint16_t* zrow,
                        int64_t K, int64_t G, int sym, double* out)
{
    for (int64_t k = 0; k < K; k++) {
        uint32_t word = Prow[k / 8];
        int32_t c = (int32_t)((word >> (4 * (k % 8))) & 0xFu);
        double s = or_f16_to_f64(srow[k / G]);
        double z = sym ? 8.0 : or_f16_to_f64(zrow[k / G]);
        out[k] = s * ((double)c - z);
    }
}

void or_dequant(const uint32_t* P, const uint16_t* s16, const uint16_t* z16,
                int64_t N, int64_t K, int64_t G, int sym, double* out)
{
    for (int64_t n = 0; n < N; n++)
        dequant_row(P + n * (K / 8), s16 + n * (K / G), sym ? NULL : z16 + n * (K / G),
                    K, G, sym, out + n * K);
}

/* y[m][i] = sum_k x'[m][k] * x_hat[rows[i]][k], accumulated in fp64, with
 * x' = x (bf16, exact) or, with the AWQ fold, x' = x / s[k] ([PTQ] AWQ step 5:
 * Y = X diag(s)^-1 quant(W')).  rows == NULL selects every row (nrows = N).
 * Y = X W_hat^T follows [Pano] 公式补课 (Y_hat = X W_hat^T). */
void or_linear(const uint16_t* x, const float* awq_s, int64_t M,
               const uint32_t* P, const uint16_t* s16, const uint16_t* z16,
               int64_t N, int64_t K, int64_t G, int sym,
               const int64_t* rows, int64_t nrows, double* y, double* scratch /* [K] */)
{
    if (!rows) nrows = N;
    for (int64_t i = 0; i < nrows; i++) {
        int64_t n = rows ? rows[i] : i;
        dequant_row(P + n * (K / 8), s16 + n * (K / G), sym ? NULL : z16 + n * (K / G),
                    K, G, sym, scratch);
        for (int64_t m = 0; m < M; m++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++) {
                double xv = (double)or_bf16_to_f32(x[m * K + k]);
                if (awq_s) xv = xv / (double)awq_s[k];
                acc += xv * scratch[k];
            }
            y[m * nrows + i] = acc;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Kernel layout 1 ("tiled"): the byte permutation wq_pack_layout must     */
/* produce.  A tile holds 128 rows x one K-slab of 4 groups (512 inputs;   */
/* the last slab may hold fewer groups).  Tiles are stored slab by slab,   */
/* row-tile by row-tile.  Inside a tile: first the codes, row r taking     */
/* gs*64 bytes (the row's words for the slab's groups, in order), then the */
/* metadata, entry (r, g) at (r*gs + g) * meta bytes: symmetric: the fp16  */
/* scale (2 bytes); asymmetric: the fp16 scale in the low half and the     */
/* fp16 zero in the high half of a little-endian uint32.  Each code word   */
/* is the canonical word with its nibbles interleaved: nibble slot t       */
/* (bits [4t, 4t+4)) holds canonical nibble 2t for t < 4 and 2(t-4)+1 for  */
/* t >= 4, so slots t and t+4 hold the adjacent inputs 2t and 2t+1.        */
/* Rows N..ceil(N/128)*128-1 are padding and hold zero bytes.              */
/* ------------------------------------------------------------------ */

uint32_t or_interleave_word(uint32_t w)
{
    uint32_t out = 0;
    for (int t = 0; t < 8; t++) {
        int src = (t < 4) ? 2 * t : 2 * (t - 4) + 1;
        out |= ((w >> (4 * src)) & 0xFu) << (4 * t);
    }
    return out;
}

#define OR_TILE_ROWS 128
#define OR_SLAB_GROUPS 4

int64_t or_layout_bytes(int64_t N, int64_t K, int sym)
{
    int64_t NG = K / 128, NS = (NG + OR_SLAB_GROUPS - 1) / OR_SLAB_GROUPS;
    int64_t NB = (N + OR_TILE_ROWS - 1) / OR_TILE_ROWS;
    int64_t per_group = 64 + (sym ? 2 : 4);
    int64_t last = NG - OR_SLAB_GROUPS * (NS - 1);
    return (NS - 1) * NB * OR_TILE_ROWS * OR_SLAB_GROUPS * per_group
         + NB * OR_TILE_ROWS * last * per_group;
}

static void put_u16(uint8_t* p, uint16_t v) { p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); }
static void put_u32(uint8_t* p, uint32_t v)
{
    for (int b = 0; b < 4; b++) p[b] = (uint8_t)(v >> (8 * b));
}

void or_relayout(const uint32_t* P, const uint16_t* s16, const uint16_t* z16,
                 int64_t N, int64_t K, int sym, uint8_t* out)
{
    int64_t NG = K / 128, NS = (NG + OR_SLAB_GROUPS - 1) / OR_SLAB_GROUPS;
    int64_t NB = (N + OR_TILE_ROWS - 1) / OR_TILE_ROWS;
    int64_t meta = sym ? 2 : 4, per_group = 64 + meta;
    int64_t full_tile = OR_TILE_ROWS * OR_SLAB_GROUPS * per_group;
    memset(out, 0, (size_t)or_layout_bytes(N, K, sym));
    for (int64_t s = 0; s < NS; s++) {
        int64_t gs = NG - OR_SLAB_GROUPS * s;
        if (gs > OR_SLAB_GROUPS) gs = OR_SLAB_GROUPS;
        int64_t tile = OR_TILE_ROWS * gs * per_group;
        for (int64_t b = 0; b < NB; b++) {
            uint8_t* base = out + s * NB * full_tile + b * tile;
            uint8_t* mbase = base + OR_TILE_ROWS * gs * 64;
            for (int64_t r = 0; r < OR_TILE_ROWS; r++) {
                int64_t n = b * OR_TILE_ROWS + r;
                if (n >= N) continue;
                for (int64_t g = 0; g < gs; g++) {
                    int64_t gg = OR_SLAB_GROUPS * s + g;
                    for (int64_t w = 0; w < 16; w++)
                        put_u32(base + r * gs * 64 + g * 64 + w * 4,
                                or_interleave_word(P[n * (K / 8) + gg * 16 + w]));
                    uint8_t* mp = mbase + (r * gs + g) * meta;
                    if (sym) put_u16(mp, s16[n * NG + gg]);
                    else put_u32(mp, (uint32_t)s16[n * NG + gg] | ((uint32_t)z16[n * NG + gg] << 16));
                }
            }
        }
    }
}
