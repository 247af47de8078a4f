/*
 * synth.c -- seeded, counter-based synthetic inputs for the block-quantised
 * MoE FFN (codes, block scales, activations, router logits).
 *
 * This module is the ONLY code shared by the fp64 oracle side and the CUDA
 * side: it draws raw inputs and holds none of the method's arithmetic (no
 * dequantisation, no packing, no GEMV, no routing).  Both sides consume the
 * same arrays it writes.
 *
 * Generator: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014).  The n-th output of a
 * SplitMix64 stream started at state s is mix64(s + (n+1)*GAMMA), so every
 * draw is addressable by (stream key, counter) and any block of any expert can
 * be regenerated without storing the layer.
 *
 * Distributions (the synthetic workload recipe):
 *   codes   uniform over the 2^b levels of the format (b = 2, 3, 4)
 *   scales  0.02 * 2^u, u ~ U(-1, 1) on a 65536-point midpoint grid,
 *           rounded to IEEE binary16 (nearest-even) for the 2/3-bit formats,
 *           or to the nearest power of two (E8M0 byte, bias 127) for 4-bit
 *   x       N(0,1) by Box-Muller in fp64, rounded to fp32 then to bf16 (RNE)
 *   logits  fp32(N(0,1) + b_e); b_e = ln p_{pi(e)} with Zipf(s) popularity
 *           p_r = r^-s / sum_r' r'^-s over a seeded permutation pi of experts,
 *           or b_e = 0 for uniform routing
 */
#include <stdint.h>
#include <stddef.h>
#include <math.h>
#include <string.h>
#include <stdlib.h>

#define SYNTH_GAMMA 0x9e3779b97f4a7c15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
    return z ^ (z >> 31);
}

/* n-th (0-based) output of the SplitMix64 stream whose state starts at key. */
uint64_t synth_draw(uint64_t key, uint64_t n) { return mix64(key + (n + 1) * SYNTH_GAMMA); }

/* Stream key for (seed, a, b, c): three chained SplitMix64 hashes. */
uint64_t synth_key(uint64_t seed, uint64_t a, uint64_t b, uint64_t c) {
    uint64_t k = mix64(seed + SYNTH_GAMMA);
    k = mix64(k ^ mix64(a + 1 * SYNTH_GAMMA));
    k = mix64(k ^ mix64(b + 2 * SYNTH_GAMMA));
    k = mix64(k ^ mix64(c + 3 * SYNTH_GAMMA));
    return k;
}

/* ---- binary16 / bfloat16 encoders (input rounding only) ---- */

static uint16_t f64_to_f16_rne(double v) {
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    if (a == 0.0) return sign;
    if (a >= 65520.0) return (uint16_t)(sign | 0x7c00u);
    int e;
    (void)frexp(a, &e);             /* a = m * 2^e, m in [0.5, 1) */
    int E = e - 1;                  /* a = 1.f * 2^E */
    if (E < -14) {                  /* subnormal: integer multiples of 2^-24 */
        double r = nearbyint(a * 16777216.0);
        return (uint16_t)(sign | (uint16_t)r);
    }
    double r = nearbyint(ldexp(a, 10 - E));   /* in [1024, 2048] */
    if (r == 2048.0) { r = 1024.0; E += 1; }
    if (E > 15) return (uint16_t)(sign | 0x7c00u);
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)((int)r - 1024));
}

static uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u); /* NaN */
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* ---- block-scale table: 65536 midpoints of U(-1,1) ---- */

static uint16_t g_scale_f16[65536];
static uint8_t  g_scale_e8m0[65536];
static int      g_table_ready = 0;

static void build_tables(void) {
    if (g_table_ready) return;
    const double l2base = log2(0.02);
    for (int i = 0; i < 65536; ++i) {
        double u = -1.0 + (2.0 * i + 1.0) / 65536.0;
        g_scale_f16[i] = f64_to_f16_rne(0.02 * exp2(u));
        int e = (int)floor(l2base + u + 0.5);      /* nearest power of two */
        g_scale_e8m0[i] = (uint8_t)(127 + e);
    }
    g_table_ready = 1;
}

void synth_init(void) { build_tables(); }

/* Copy of the 65536-entry scale tables (for the device twin of this module). */
void synth_scale_tables(uint16_t* f16, uint8_t* e8m0) {
    build_tables();
    memcpy(f16, g_scale_f16, sizeof(g_scale_f16));
    memcpy(e8m0, g_scale_e8m0, sizeof(g_scale_e8m0));
}

/*
 * Codes of rows [row0, row0+nrows) of a [rows][cols] matrix (cols % 32 == 0),
 * one code per byte, row-major: out[(r - row0) * cols + k].
 * Block beta = r * (cols/32) + k/32.  2-bit: one draw per block, code j in
 * bits [2j, 2j+2).  3-bit: draws 2beta, 2beta+1, codes 0..15 in bits [3j, 3j+3)
 * of the first, 16..31 of the second.  4-bit: draws 2beta, 2beta+1, 16 codes
 * of 4 bits each.
 */
int synth_codes(uint64_t key, int bits, int64_t row0, int64_t nrows, int64_t cols, uint8_t* out) {
    if (cols % 32 != 0 || (bits != 2 && bits != 3 && bits != 4) || nrows < 0) return -1;
    const int64_t nb = cols / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nrows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            uint64_t beta = (uint64_t)((row0 + r) * nb + b);
            uint8_t* o = out + r * cols + b * 32;
            if (bits == 2) {
                uint64_t d = synth_draw(key, beta);
                for (int j = 0; j < 32; ++j) o[j] = (uint8_t)((d >> (2 * j)) & 3u);
            } else if (bits == 3) {
                uint64_t d0 = synth_draw(key, 2 * beta), d1 = synth_draw(key, 2 * beta + 1);
                for (int j = 0; j < 16; ++j) o[j] = (uint8_t)((d0 >> (3 * j)) & 7u);
                for (int j = 0; j < 16; ++j) o[16 + j] = (uint8_t)((d1 >> (3 * j)) & 7u);
            } else {
                uint64_t d0 = synth_draw(key, 2 * beta), d1 = synth_draw(key, 2 * beta + 1);
                for (int j = 0; j < 16; ++j) o[j] = (uint8_t)((d0 >> (4 * j)) & 15u);
                for (int j = 0; j < 16; ++j) o[16 + j] = (uint8_t)((d1 >> (4 * j)) & 15u);
            }
        }
    }
    return 0;
}

/*
 * Block scales of rows [row0, row0+nrows): out is uint16 (binary16 bits) for
 * bits 2/3 and uint8 (E8M0) for bits 4, layout [nrows][cols/32].
 */
int synth_scales(uint64_t key, int bits, int64_t row0, int64_t nrows, int64_t cols, void* out) {
    if (cols % 32 != 0 || (bits != 2 && bits != 3 && bits != 4) || nrows < 0) return -1;
    build_tables();
    const int64_t nb = cols / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nrows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            uint64_t beta = (uint64_t)((row0 + r) * nb + b);
            unsigned i = (unsigned)(synth_draw(key, beta) >> 48);
            if (bits == 4) ((uint8_t*)out)[r * nb + b] = g_scale_e8m0[i];
            else ((uint16_t*)out)[r * nb + b] = g_scale_f16[i];
        }
    }
    return 0;
}

static double normal_pair(uint64_t key, uint64_t pair, int which) {
    uint64_t r1 = synth_draw(key, 2 * pair), r2 = synth_draw(key, 2 * pair + 1);
    double u1 = ((double)((r1 >> 11) + 1)) * 0x1.0p-53;   /* (0, 1] */
    double u2 = ((double)(r2 >> 11)) * 0x1.0p-53;         /* [0, 1) */
    double rad = sqrt(-2.0 * log(u1));
    double ang = 6.283185307179586476925286766559 * u2;
    return which ? rad * sin(ang) : rad * cos(ang);
}

/* out[i] = N(0,1) draw i + n0 of stream key, as fp64. */
void synth_normal_f64(uint64_t key, int64_t n0, int64_t n, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint64_t idx = (uint64_t)(n0 + i);
        out[i] = normal_pair(key, idx >> 1, (int)(idx & 1));
    }
}

/* out[i] = bf16 bits of fp32(N(0,1) draw i + n0). */
void synth_normal_bf16(uint64_t key, int64_t n0, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint64_t idx = (uint64_t)(n0 + i);
        out[i] = f32_to_bf16_rne((float)normal_pair(key, idx >> 1, (int)(idx & 1)));
    }
}

/*
 * Per-expert log-popularity bias b_e = ln p_{pi(e)}, p_r = r^-s / sum r'^-s,
 * pi a Fisher-Yates permutation drawn from key.  s <= 0 gives b_e = 0.
 */
void synth_zipf_bias(uint64_t key, int E, double s, double* bias) {
    if (s <= 0.0) { for (int e = 0; e < E; ++e) bias[e] = 0.0; return; }
    int* perm = (int*)malloc(sizeof(int) * (size_t)E);
    for (int e = 0; e < E; ++e) perm[e] = e;
    for (int i = E - 1; i > 0; --i) {
        int j = (int)(synth_draw(key, (uint64_t)i) % (uint64_t)(i + 1));
        int t = perm[i]; perm[i] = perm[j]; perm[j] = t;
    }
    double z = 0.0;
    for (int r = 1; r <= E; ++r) z += pow((double)r, -s);
    for (int e = 0; e < E; ++e) bias[e] = log(pow((double)(perm[e] + 1), -s) / z);
    free(perm);
}

/*
 * logits[t][e] = fp32(N(0,1) + bias[e]) for tokens [tok0, tok0+T) of stream
 * key; token t uses normal draws t*E .. t*E+E-1.
 */
void synth_logits(uint64_t key, const double* bias, int64_t tok0, int64_t T, int E, float* out) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            uint64_t idx = (uint64_t)((tok0 + t) * E + e);
            double z = normal_pair(key, idx >> 1, (int)(idx & 1));
            out[t * E + e] = (float)(z + (bias ? bias[e] : 0.0));
        }
    }
}
