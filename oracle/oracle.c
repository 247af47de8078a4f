/*
 * oracle.c -- plain fp64 CPU reference of the block-quantised MoE FFN step.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load or call this library.  It shares no code with
 * the CUDA library: it reads the raw codes and scales written by the input
 * generator (never the packed bytes) and computes every step from its
 * definition in double precision, with no blocking, fusion or reordering.
 *
 * Sources (web pages, cited by title and section):
 *  [TZ]  taozi.news, "DeepSeek V4 Flash 在 128GB 锐龙 AI MAX+ 上跑到 32 tok/s",
 *        section "ROCmFPX：把 284B 权重压进 128 GB": a block stores the low-bit
 *        codes of 32 weights plus its scale; ROCmFP2 = 10 bytes per block
 *        (~2.50 bit/weight), ROCmFP3 ~3.50 bit, ROCmFP4 ~4.25 bit; routed
 *        gate/up in FP2, routed down in FP3, sensitive projections in FP4.
 *  [AI]  ainomam.com, "APU 实现 token 自由：AMD Ryzen AI MAX+ 395 跑 DeepSeek V4
 *        Flash，284B 模型跑出 32 tok/s", section "Lucebox 的优化三板斧": 256
 *        routed experts plus 1 shared, 6 active per layer; each packed weight
 *        is decoded once and applied to all 4 verify columns; TOP-K/ARGSORT
 *        routing kernels.
 *  [MZ]  m.mzlw.cn, "Lucebox专攻DeepSeek V4：DSpark草稿模型、MoE专家并行与
 *        ROCmFPX量化达成42 tok/s", section "MoE 专家并行": 43 MoE layers, each
 *        with 256 routed experts, top-6, plus 1 shared expert.
 *
 * The pages give only the block size and the bytes per block.  The format this
 * library fixes (its readings, not the pages'):
 *   FP2: 8 B of 2-bit codes + binary16 scale     levels c - 1.5  (-1.5..1.5)
 *   FP3: 12 B of 3-bit codes + binary16 scale    levels c - 3.5  (-3.5..3.5)
 *   FP4: 16 B of 4-bit codes + E8M0 scale byte   levels c - 7.5  (-7.5..7.5)
 *   W[n][k] = scale[n][k/32] * level(code[n][k]); blocks run along k (the
 *   reduction dimension) of one output row.
 * Expert FFN: h = silu(Wg x) * (Wu x), silu(z) = z / (1 + e^-z); d = Wd h.
 * Routing: the k largest logits (ties to the lower expert index), weights =
 * softmax over the k selected logits; shared expert weight 1.
 */
#include <stdint.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

typedef struct {
    int bits;                /* 2, 3 or 4 */
    const uint8_t* codes;    /* [rows][cols], one code per byte */
    const void* scales;      /* [rows][cols/32]: uint16 binary16 (2/3) or uint8 E8M0 (4) */
} oracle_mat;

/* ---- format definition ---- */

/* Bytes of one 32-weight block: 32*b bits of codes + the scale (2 B binary16,
 * or 1 B power-of-two for FP4). */
int oracle_block_bytes(int bits) {
    if (bits == 2) return 32 * 2 / 8 + 2;
    if (bits == 3) return 32 * 3 / 8 + 2;
    if (bits == 4) return 32 * 4 / 8 + 1;
    return -1;
}

double oracle_bits_per_weight(int bits) {
    int b = oracle_block_bytes(bits);
    return b < 0 ? -1.0 : (double)b * 8.0 / 32.0;
}

/* Level of code c in a b-bit format: evenly spaced, unit step, symmetric. */
double oracle_level(int bits, int c) { return (double)c - ((double)((1 << bits) - 1)) / 2.0; }

/* IEEE binary16 bits -> value (finite only; returns NAN otherwise). */
static double f16_value(uint16_t h) {
    int s = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 31) return NAN;
    if (e == 0) v = ldexp((double)m, -24);
    else v = ldexp((double)(1024 + m), e - 25);
    return s ? -v : v;
}

/* Scale of block i of a matrix. */
static double scale_value(int bits, const void* scales, int64_t i) {
    if (bits == 4) {
        uint8_t e = ((const uint8_t*)scales)[i];
        if (e == 0xFF) return NAN;
        return ldexp(1.0, (int)e - 127);
    }
    return f16_value(((const uint16_t*)scales)[i]);
}

/* Round a double to the nearest bfloat16 value (ties to even), result as double. */
double oracle_bf16_round(double v) {
    if (v == 0.0 || !isfinite(v)) return v;
    double a = fabs(v);
    double r;
    if (a < 0x1.0p-126) {
        r = ldexp(nearbyint(ldexp(a, 133)), -133);      /* subnormal spacing 2^-133 */
    } else {
        int e;
        double m = frexp(a, &e);                        /* a = m 2^e, m in [0.5,1) */
        r = ldexp(nearbyint(ldexp(m, 8)), e - 8);       /* 8 significant bits */
    }
    return v < 0 ? -r : r;
}

/* W[rows][cols] = scale * level, element by element. */
int oracle_dequant(int bits, const uint8_t* codes, const void* scales, int64_t rows, int64_t cols, double* W) {
    if (oracle_block_bytes(bits) < 0 || cols % 32 != 0) return -1;
    const int64_t nb = cols / 32;
    for (int64_t n = 0; n < rows; ++n)
        for (int64_t k = 0; k < cols; ++k) {
            double s = scale_value(bits, scales, n * nb + k / 32);
            if (isnan(s)) return -2;
            W[n * cols + k] = s * oracle_level(bits, codes[n * cols + k]);
        }
    return 0;
}

/* Element W[n][k] of a matrix, optionally rounded to bf16 (prefill operands). */
static inline double w_elem(const oracle_mat* M, int64_t cols, int64_t n, int64_t k, int bf16_ops) {
    double w = scale_value(M->bits, M->scales, n * (cols / 32) + k / 32) * oracle_level(M->bits, M->codes[n * cols + k]);
    return bf16_ops ? oracle_bf16_round(w) : w;
}

/*
 * y[c][n] = sum_k W[n][k] x[c][k] for c < q, and, if mag != NULL,
 * mag[c][n] = sum_k |W[n][k]| |x[c][k]|.
 */
static int gemv_mat(const oracle_mat* M, int64_t N, int64_t K, const double* x, int q, double* y, double* mag, int bf16_ops) {
    if (oracle_block_bytes(M->bits) < 0 || K % 32 != 0) return -1;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(|:bad)
    for (int64_t n = 0; n < N; ++n) {
        for (int c = 0; c < q; ++c) {
            double acc = 0.0, am = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double w = w_elem(M, K, n, k, bf16_ops);
                if (isnan(w)) bad = 1;
                acc += w * x[(int64_t)c * K + k];
                am += fabs(w) * fabs(x[(int64_t)c * K + k]);
            }
            y[(int64_t)c * N + n] = acc;
            if (mag) mag[(int64_t)c * N + n] = am;
        }
    }
    return bad ? -2 : 0;
}

int oracle_gemv(int bits, const uint8_t* codes, const void* scales, int64_t N, int64_t K,
                const double* x, int q, double* y, double* mag) {
    oracle_mat M = {bits, codes, scales};
    return gemv_mat(&M, N, K, x, q, y, mag, 0);
}

/*
 * The same with every weight rounded to bf16 (nearest even) from its exact
 * value: the prefill operand precision (the prefill of the pages' model runs
 * the experts as dense contractions on bf16 tensor-core operands, here
 * dequantised once per weight and rounded once).
 */
int oracle_gemv_bf16w(int bits, const uint8_t* codes, const void* scales, int64_t N, int64_t K,
                      const double* x, int q, double* y, double* mag) {
    oracle_mat M = {bits, codes, scales};
    return gemv_mat(&M, N, K, x, q, y, mag, 1);
}

/*
 * Router: for each token the k largest logits, ordered by descending value,
 * equal values by ascending expert index; w = softmax over the k selected.
 */
int oracle_router_topk(const float* logits, int64_t T, int E, int k, int32_t* idx, double* w) {
    if (k < 1 || k > E) return -1;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(|:bad)
    for (int64_t t = 0; t < T; ++t) {
        const float* l = logits + t * E;
        unsigned char* taken = (unsigned char*)calloc((size_t)E, 1);
        if (!taken) { bad = 1; continue; }
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e;   /* strict: lower index wins ties */
            }
            taken[best] = 1;
            idx[t * k + j] = best;
        }
        double vmax = (double)l[idx[t * k]];
        double z = 0.0;
        for (int j = 0; j < k; ++j) z += exp((double)l[idx[t * k + j]] - vmax);
        for (int j = 0; j < k; ++j) w[t * k + j] = exp((double)l[idx[t * k + j]] - vmax) / z;
        free(taken);
    }
    return bad ? -2 : 0;
}

double oracle_silu(double z) { return z / (1.0 + exp(-z)); }

/*
 * One expert applied to one token column x[H]:
 *   g = Wg x, u = Wu x (Wg, Wu: [I][H]); h = silu(g) * u; d = Wd h (Wd: [H][I]).
 * mag[H] = sum_i |Wd| |h| (the per-element scale of the accumulation error).
 * bf16_ops: round every weight and h to bfloat16 before use (prefill operand
 * precision); x is bf16 already.
 */
int oracle_expert_ffn(int H, int I, const oracle_mat* gate, const oracle_mat* up, const oracle_mat* down,
                      const double* x, int bf16_ops, double* d, double* mag, double* h_out) {
    double* g = (double*)malloc(sizeof(double) * (size_t)I);
    double* u = (double*)malloc(sizeof(double) * (size_t)I);
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
    int rc = (g && u && h) ? 0 : -3;
    if (!rc) rc = gemv_mat(gate, I, H, x, 1, g, NULL, bf16_ops);
    if (!rc) rc = gemv_mat(up, I, H, x, 1, u, NULL, bf16_ops);
    if (!rc) {
        for (int i = 0; i < I; ++i) {
            h[i] = oracle_silu(g[i]) * u[i];
            if (bf16_ops) h[i] = oracle_bf16_round(h[i]);
            if (h_out) h_out[i] = h[i];
        }
        rc = gemv_mat(down, H, I, h, 1, d, mag, bf16_ops);
    }
    free(g); free(u); free(h);
    return rc;
}

/*
 * MoE FFN for one token: y = sum_j w[j] * FFN_{e_j}(x) + FFN_shared(x).
 * gate/up/down hold the k selected experts' matrices in routing order;
 * shared (3 matrices) may be NULL.  mag[H] = sum_j |w_j| mag_j + mag_shared.
 */
int oracle_moe_token(int H, int I, int k, const oracle_mat* gate, const oracle_mat* up, const oracle_mat* down,
                     const double* w, const oracle_mat* shared, const double* x, int bf16_ops,
                     double* y, double* mag) {
    double* d = (double*)malloc(sizeof(double) * (size_t)H);
    double* m = (double*)malloc(sizeof(double) * (size_t)H);
    if (!d || !m) { free(d); free(m); return -3; }
    for (int i = 0; i < H; ++i) { y[i] = 0.0; mag[i] = 0.0; }
    int rc = 0;
    for (int j = 0; j < k && !rc; ++j) {
        rc = oracle_expert_ffn(H, I, &gate[j], &up[j], &down[j], x, bf16_ops, d, m, NULL);
        for (int i = 0; i < H && !rc; ++i) { y[i] += w[j] * d[i]; mag[i] += fabs(w[j]) * m[i]; }
    }
    if (!rc && shared) {
        rc = oracle_expert_ffn(H, I, &shared[0], &shared[1], &shared[2], x, bf16_ops, d, m, NULL);
        for (int i = 0; i < H && !rc; ++i) { y[i] += d[i]; mag[i] += m[i]; }
    }
    free(d); free(m);
    return rc;
}

/* Layer chaining: x_next = bf16(y / sqrt(mean(y^2))). */
void oracle_rms_bf16(const double* y, int64_t H, double* xnext) {
    double ss = 0.0;
    for (int64_t i = 0; i < H; ++i) ss += y[i] * y[i];
    double r = sqrt(ss / (double)H);
    for (int64_t i = 0; i < H; ++i) xnext[i] = oracle_bf16_round(y[i] / r);
}
