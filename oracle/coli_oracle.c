/*
 * coli_oracle.c -- the ORACLE for one GLM-5.2-shaped MoE layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, the package smoke check and the
 * CPU-baseline leg of bench.py may load or call this library.  The CUDA
 * library never links it, includes it or calls it, and this file shares no
 * code, header, table or constant generator with the CUDA sources: the two
 * implement the same written definition independently.
 *
 * What it computes (one MoE layer, every token independent):
 *   x (F32) --Q8_0--> xq, xd                       activation quantiser
 *   x (F32) --router GEMV, sigmoid--> s            router (kept in F32)
 *   s + bias --top-k--> idx, w                     selection and weights
 *   (idx) --bucket--> counts, offsets, perm        "batched MoE" grouping
 *   xq --gate/up int4 dots, SwiGLU, Q8_0--> hq     routed + shared experts
 *   hq --down int4 dots--> y
 *   out = sum_k w_k y_k + y_shared                 weighted combine
 *
 * Sources (page title, then section):
 *  [W] "GLM-5.2-colibri-int4架构解析MoE专家混合与INT4量化原理" (wmrh.cn):
 *      "GLM-5.2的MoE实现" (256 routed experts, 1 shared, 8 per token,
 *      hidden 6144, expert inter 2048); "MoE的工作原理" (router scores, pick
 *      the 8 best, weighted sum of the 8 outputs); "GLM-5.2-colibri-int4的
 *      量化流程" (int4 by np.rint == lrintf, one F32 scale per weight row,
 *      packed into U8); "高级配置选项 / 路由策略定制" (topk_method,
 *      routed_scaling_factor, norm_topk_prob); "量化保留模块"
 *      (modules_to_not_convert stay F32: the router).
 *  [C] "Colibri：在笔记本上跑744B参数的AI模型", "关键特性": DeepSeek-V3 style
 *      sigmoid router plus shared expert; integer dot-product kernels with
 *      Q8_0-style int8 activations (AVX2 maddubs); int8 / packed int4 kernels.
 *  [D] "如何在普通电脑上运行 7440 亿参数神经网络" (devtrends.cc), "引擎是如何
 *      工作的": requests for the same expert are merged into one batch.
 *  [H] HN summary (hn.213312.xyz, article 48842459), "已实现的功能":
 *      batched MoE (an expert shared by several positions is read once);
 *      efficient integer kernels.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - nibble format: two's complement, element 2j in the low nibble of byte j;
 *    int4 scale = absmax/7, q clamped to [-8,7]; Q8 scale = absmax/127, F32,
 *    q clamped to [-127,127]; both round half to even (rintf).
 *  - router: DeepSeek-V3 "noaux_tc" reading: the correction bias changes the
 *    selection only, weights come from the unbiased sigmoid scores, ties go
 *    to the lower expert index, optional renormalisation, then
 *    routed_scaling_factor; no expert groups.
 *  - the down projection's input is re-quantised to Q8_0 along the
 *    intermediate dimension; the shared expert is int4 like the routed ones
 *    and enters the combine with weight 1.
 *  - float evaluation order is fixed by three contracts so that a second
 *    implementation can match bit for bit:
 *      R (router logit): element h feeds accumulator l = (h/4) mod 32; each
 *        accumulator starts at +0 and takes its elements in ascending h with
 *        fmaf; the logit is acc_0 + acc_1 + ... + acc_31 added left to right.
 *      F (row fold): acc = 0; for each 32-block b ascending:
 *        acc = fmaf(d_x[b], (float)isum[b], acc); y = s_w * acc.
 *      C (combine): acc = 0; for k in rank order acc = fmaf(w_k, y_k, acc);
 *        then out = acc + y_shared_0 (+ y_shared_1 ...).
 *  - exp: our own, Cody & Waite argument reduction (W. J. Cody, W. Waite,
 *    "Software Manual for the Elementary Functions", 1980) with a degree-7
 *    Taylor polynomial, so that no libm exp enters a result (see ora_exp).
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math -fPIC -shared.
 * With those flags every float expression is one binary32 operation,
 * round-to-nearest-even, in the order written.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORA_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* exp, sigmoid, SiLU                                                        */
/* ------------------------------------------------------------------------ */

/* Constants of the exp definition.  LOG2E is log2(e) rounded to binary32.
 * LN2_HI is ln 2 with the mantissa cut to 15 significant bits, so k*LN2_HI is
 * exact for |k| <= 255 (Cody-Waite); LN2_LO = ln 2 - LN2_HI rounded to
 * binary32.  C2..C7 are 1/n! rounded to binary32 (Taylor series of e^r). */
static const float ORA_LOG2E = 0x1.715476p+0f;
static const float ORA_LN2_HI = 0x1.62e4p-1f;
static const float ORA_LN2_LO = 0x1.7f7d1cp-20f;
static const float ORA_C2 = 0x1.0p-1f;
static const float ORA_C3 = 0x1.555556p-3f;
static const float ORA_C4 = 0x1.555556p-5f;
static const float ORA_C5 = 0x1.111112p-7f;
static const float ORA_C6 = 0x1.6c16c2p-10f;
static const float ORA_C7 = 0x1.a01a02p-13f;
/* Above EXP_HI the result overflows binary32; below EXP_LO it is below half
 * the smallest subnormal. */
static const float ORA_EXP_HI = 0x1.62e43p+6f;   /*  88.7228394 */
static const float ORA_EXP_LO = -0x1.9fe36ap+6f; /* -103.972084 */

/* 2^k as a binary32 built from its exponent field, -126 <= k <= 127. */
static float ora_pow2i(int k) {
    uint32_t bits = (uint32_t)(k + 127) << 23;
    float f;
    memcpy(&f, &bits, sizeof f);
    return f;
}

/* e^x.  Steps: k = rint(x*log2 e); r = x - k*ln2 in two fmaf steps
 * (Cody-Waite); p = sum_{n=0..7} r^n/n! by Horner with fmaf; result
 * p * 2^k applied as two exact-range factors 2^(k/2) and 2^(k - k/2), so the
 * only rounding of the scaling is the last multiply. */
ORA_API float ora_exp(float x) {
    if (x != x) return x;
    if (x > ORA_EXP_HI) return INFINITY;
    if (x < ORA_EXP_LO) return 0.0f;
    float k = rintf(x * ORA_LOG2E);
    float r = fmaf(-k, ORA_LN2_HI, x);
    r = fmaf(-k, ORA_LN2_LO, r);
    float p = ORA_C7;
    p = fmaf(p, r, ORA_C6);
    p = fmaf(p, r, ORA_C5);
    p = fmaf(p, r, ORA_C4);
    p = fmaf(p, r, ORA_C3);
    p = fmaf(p, r, ORA_C2);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    int ki = (int)k;
    int k1 = ki / 2; /* C division truncates toward zero */
    int k2 = ki - k1;
    return (p * ora_pow2i(k1)) * ora_pow2i(k2);
}

/* Logistic sigmoid of the router ([C] "DeepSeek-V3 风格的 sigmoid 路由器"). */
ORA_API float ora_sigmoid(float x) { return 1.0f / (1.0f + ora_exp(-x)); }

/* SiLU(g) = g * sigmoid(g), the gate activation of a SwiGLU expert. */
ORA_API float ora_silu(float g) { return g * ora_sigmoid(g); }

/* Element-wise forms of the three functions above (for sweeps). */
ORA_API void ora_exp_n(const float* x, int64_t n, float* y) {
    for (int64_t i = 0; i < n; ++i) y[i] = ora_exp(x[i]);
}
ORA_API void ora_sigmoid_n(const float* x, int64_t n, float* y) {
    for (int64_t i = 0; i < n; ++i) y[i] = ora_sigmoid(x[i]);
}
ORA_API void ora_silu_n(const float* x, int64_t n, float* y) {
    for (int64_t i = 0; i < n; ++i) y[i] = ora_silu(x[i]);
}

/* ------------------------------------------------------------------------ */
/* int4 packing and the per-row int4 weight quantiser ([W] 量化流程)         */
/* ------------------------------------------------------------------------ */

/* Pack n int4 values (each in [-8,7]) two per byte: element 2j goes to the
 * low nibble of byte j, element 2j+1 to the high nibble, two's complement.
 * n must be even. */
ORA_API void ora_pack_int4(const int8_t* q, int64_t n, uint8_t* out) {
    for (int64_t j = 0; j < n / 2; ++j) {
        unsigned lo = (unsigned)q[2 * j] & 0xFu;
        unsigned hi = (unsigned)q[2 * j + 1] & 0xFu;
        out[j] = (uint8_t)(lo | (hi << 4));
    }
}

/* Sign-extend one nibble: 0..7 -> 0..7, 8..15 -> -8..-1. */
static int ora_nibble_value(unsigned nib) { return nib >= 8u ? (int)nib - 16 : (int)nib; }

/* Element i of a packed int4 row. */
static int ora_int4_at(const uint8_t* packed, int64_t i) {
    unsigned byte = packed[i / 2];
    unsigned nib = (i % 2 == 0) ? (byte & 0xFu) : (byte >> 4);
    return ora_nibble_value(nib);
}

/* Unpack n int4 values (inverse of ora_pack_int4). */
ORA_API void ora_unpack_int4(const uint8_t* packed, int64_t n, int8_t* q) {
    for (int64_t i = 0; i < n; ++i) q[i] = (int8_t)ora_int4_at(packed, i);
}

static int ora_clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* Per-row int4 quantiser: scale = absmax/7 (F32 division); q = rint(w/scale)
 * clamped to [-8,7]; an all-zero row gets scale 0 and q = 0.  Output rows
 * are cols/2 bytes; cols must be even. */
ORA_API void ora_quantize_rows_int4(const float* w, int64_t rows, int64_t cols, uint8_t* q_out,
                                    float* scale_out) {
    int8_t* q = (int8_t*)malloc((size_t)cols);
    for (int64_t r = 0; r < rows; ++r) {
        const float* row = w + r * cols;
        float amax = 0.0f;
        for (int64_t c = 0; c < cols; ++c) {
            float a = fabsf(row[c]);
            if (a > amax) amax = a;
        }
        float scale = amax / 7.0f;
        for (int64_t c = 0; c < cols; ++c) {
            if (amax == 0.0f) {
                q[c] = 0;
            } else {
                q[c] = (int8_t)ora_clampi((int)rintf(row[c] / scale), -8, 7);
            }
        }
        scale_out[r] = scale;
        ora_pack_int4(q, cols, q_out + r * (cols / 2));
    }
    free(q);
}

/* Per-row int8 weight quantiser, the int8 variant of the expert weights
 * ([C] "关键特性": quantisation kernels int8 / packed int4 / packed int2).
 * Reading: the int4 recipe with the int8 range -- scale = absmax/127 (F32
 * division), q = rint(w/scale) clamped to [-127,127] (round half to even),
 * one byte per element; an all-zero row gets scale 0 and q = 0. */
ORA_API void ora_quantize_rows_int8(const float* w, int64_t rows, int64_t cols, int8_t* q_out,
                                    float* scale_out) {
    for (int64_t r = 0; r < rows; ++r) {
        const float* row = w + r * cols;
        float amax = 0.0f;
        for (int64_t c = 0; c < cols; ++c) {
            float a = fabsf(row[c]);
            if (a > amax) amax = a;
        }
        float scale = amax / 127.0f;
        for (int64_t c = 0; c < cols; ++c)
            q_out[r * cols + c] = (amax == 0.0f) ? 0 : (int8_t)ora_clampi((int)rintf(row[c] / scale), -127, 127);
        scale_out[r] = scale;
    }
}

/* ------------------------------------------------------------------------ */
/* FP8 -> int4 requantiser ([W] "GLM-5.2-colibri-int4的量化流程": the source */
/* is the FP8 (e4m3) model, dequantised to F32 and then quantised per row as */
/* above; its config: fmt e4m3, weight_block_size [128, 128])                */
/* ------------------------------------------------------------------------ */

/* e4m3 ("fn" variant: no infinities): bit 7 sign, bits 6..3 exponent with
 * bias 7, bits 2..0 mantissa.  Exponent 0: subnormal, (m/8) * 2^-6.
 * Exponent 15 with mantissa 7: NaN.  Otherwise (1 + m/8) * 2^(e-7).
 * Every code is exact in F32. */
ORA_API float ora_e4m3_to_f32(uint8_t b) {
    const int sign = (b >> 7) & 1, e = (b >> 3) & 15, m = b & 7;
    float v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexpf((float)m / 8.0f, -6);
    else
        v = ldexpf(1.0f + (float)m / 8.0f, e - 7);
    return sign ? -v : v;
}

/* Reading (the pages give the flow, not the arithmetic): element (r, c) of
 * the F32 matrix is e4m3(w8[r, c]) * block_scale[r / block, c / block], one
 * F32 multiply (DeepSeek-V3's weight_scale_inv convention: the stored factor
 * multiplies the FP8 value); an element whose product is not finite (a NaN
 * code, or an overflow) counts as 0; then each row is quantised to int4
 * exactly as ora_quantize_rows_int4.  block_scale is
 * [ceil(rows/block) x ceil(cols/block)], row-major. */
ORA_API void ora_requantize_fp8_int4(const uint8_t* w8, const float* block_scale, int64_t rows, int64_t cols,
                                     int64_t block, uint8_t* q_out, float* scale_out) {
    const int64_t bcols = (cols + block - 1) / block;
    float* row = (float*)malloc((size_t)cols * sizeof(float));
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < cols; ++c) {
            float v = ora_e4m3_to_f32(w8[r * cols + c]) * block_scale[(r / block) * bcols + c / block];
            if (!(fabsf(v) <= FLT_MAX)) v = 0.0f;
            row[c] = v;
        }
        ora_quantize_rows_int4(row, 1, cols, q_out + r * (cols / 2), scale_out + r);
    }
    free(row);
}

/* ------------------------------------------------------------------------ */
/* Q8_0-style activation quantiser ([C] "Q8_0 风格的 int8 激活")             */
/* ------------------------------------------------------------------------ */

/* Each token's vector is cut into 32-element blocks; per block d = absmax/127
 * (F32), q = rint(x/d) clamped to [-127,127]; an all-zero block has d = 0 and
 * q = 0.  dim must be a multiple of 32; d has n_tok * dim/32 entries. */
ORA_API void ora_quantize_act_q8(const float* x, int64_t n_tok, int64_t dim, int8_t* q_out,
                                 float* d_out) {
    int64_t nb = dim / 32;
    for (int64_t t = 0; t < n_tok; ++t) {
        for (int64_t b = 0; b < nb; ++b) {
            const float* blk = x + t * dim + b * 32;
            int8_t* qb = q_out + t * dim + b * 32;
            float amax = 0.0f;
            for (int j = 0; j < 32; ++j) {
                float a = fabsf(blk[j]);
                if (a > amax) amax = a;
            }
            float d = amax / 127.0f;
            for (int j = 0; j < 32; ++j) {
                qb[j] = (amax == 0.0f) ? 0 : (int8_t)ora_clampi((int)rintf(blk[j] / d), -127, 127);
            }
            d_out[t * nb + b] = d;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Router ([W] MoE的工作原理, 路由策略定制, 量化保留模块; [C] 关键特性)       */
/* ------------------------------------------------------------------------ */

/* Router logit of one token against one router row, contract R. */
ORA_API float ora_router_logit(const float* x, const float* w, int64_t H) {
    float acc[32];
    for (int l = 0; l < 32; ++l) acc[l] = 0.0f;
    for (int64_t h = 0; h < H; ++h) {
        int l = (int)((h / 4) % 32);
        acc[l] = fmaf(x[h], w[h], acc[l]);
    }
    float logit = acc[0];
    for (int l = 1; l < 32; ++l) logit = logit + acc[l];
    return logit;
}

/* Full router for n_tok tokens.
 *   scores[t,e] = sigmoid(logit(x_t, W_r[e]))                     (F32)
 *   select K experts by descending scores[t,e] + bias[e], ties to the lower
 *   e; idx[t, 0..K) is that list in rank order.
 *   denom = s_r0 + s_r1 + ... (left to right, rank order);
 *   w_k = (s_rk / denom) * rsf if norm_topk_prob, else s_rk * rsf.
 * Any of scores_out / idx_out / w_out may be NULL. */
ORA_API void ora_route(const float* x, const float* w_router, const float* bias, int64_t n_tok,
                       int64_t E, int64_t H, int32_t K, int32_t norm_topk_prob, float rsf,
                       float* scores_out, int32_t* idx_out, float* w_out) {
    float* s = (float*)malloc((size_t)E * sizeof(float));
    float* b = (float*)malloc((size_t)E * sizeof(float));
    unsigned char* taken = (unsigned char*)malloc((size_t)E);
    int32_t* idx = (int32_t*)malloc((size_t)K * sizeof(int32_t));
    for (int64_t t = 0; t < n_tok; ++t) {
        for (int64_t e = 0; e < E; ++e) {
            s[e] = ora_sigmoid(ora_router_logit(x + t * H, w_router + e * H, H));
            b[e] = s[e] + bias[e];
            taken[e] = 0;
            if (scores_out) scores_out[t * E + e] = s[e];
        }
        for (int32_t k = 0; k < K; ++k) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; ++e) {
                if (taken[e]) continue;
                /* strict '>' keeps the lower index when two values tie */
                if (best < 0 || b[e] > b[best]) best = e;
            }
            taken[best] = 1;
            idx[k] = (int32_t)best;
        }
        float denom = s[idx[0]];
        for (int32_t k = 1; k < K; ++k) denom = denom + s[idx[k]];
        for (int32_t k = 0; k < K; ++k) {
            float wk = norm_topk_prob ? (s[idx[k]] / denom) * rsf : s[idx[k]] * rsf;
            if (idx_out) idx_out[t * K + k] = idx[k];
            if (w_out) w_out[t * K + k] = wk;
        }
    }
    free(s);
    free(b);
    free(taken);
    free(idx);
}

/* ------------------------------------------------------------------------ */
/* Bucketing ("batched MoE", [D] 引擎是如何工作的, [H] 已实现的功能)          */
/* ------------------------------------------------------------------------ */

/* Group the n_tok*K (token, slot) pairs by expert: counts[e] pairs per
 * expert, offsets = exclusive prefix sum (offsets[E] = n_tok*K), and perm
 * lists the flat pair ids t*K + k sorted by (expert, token).  Each expert's
 * tokens then form one contiguous group, so its weights are read once. */
ORA_API void ora_bucket(const int32_t* idx, int64_t n_tok, int32_t K, int32_t E, int32_t* counts,
                        int32_t* offsets, int32_t* perm) {
    for (int32_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t i = 0; i < n_tok * K; ++i) counts[idx[i]] += 1;
    offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int64_t pos = 0;
    for (int32_t e = 0; e < E; ++e)
        for (int64_t t = 0; t < n_tok; ++t)
            for (int32_t k = 0; k < K; ++k)
                if (idx[t * K + k] == e) perm[pos++] = (int32_t)(t * K + k);
}

/* ------------------------------------------------------------------------ */
/* Integer row dots and the expert FFN ([C] 整数点积内核; [H] 高效整数内核)   */
/* ------------------------------------------------------------------------ */

/* Per-32-block integer partial sums of one packed int4 row against one
 * Q8 activation vector: isum[b] = sum_{j<32} q_w[32b+j] * q_x[32b+j]. */
ORA_API void ora_block_isums(const uint8_t* qrow, const int8_t* xq, int64_t dim_in, int32_t* isum) {
    for (int64_t b = 0; b < dim_in / 32; ++b) {
        int32_t acc = 0;
        for (int j = 0; j < 32; ++j) {
            int64_t i = b * 32 + j;
            acc += (int32_t)ora_int4_at(qrow, i) * (int32_t)xq[i];
        }
        isum[b] = acc;
    }
}

/* The same for an int8 weight row (one signed byte per element). */
ORA_API void ora_block_isums_int8(const int8_t* qrow, const int8_t* xq, int64_t dim_in, int32_t* isum) {
    for (int64_t b = 0; b < dim_in / 32; ++b) {
        int32_t acc = 0;
        for (int j = 0; j < 32; ++j) acc += (int32_t)qrow[b * 32 + j] * (int32_t)xq[b * 32 + j];
        isum[b] = acc;
    }
}

/* One output of a weight x Q8 matrix-vector product, contract F: the weight
 * row is packed int4 (bits 4) or int8 (bits 8). */
static float ora_row_dot_bits(const uint8_t* qrow, int bits, float s_w, const int8_t* xq, const float* xd,
                              int64_t dim_in) {
    int64_t nb = dim_in / 32;
    int32_t* isum = (int32_t*)malloc((size_t)nb * sizeof(int32_t));
    if (bits == 8)
        ora_block_isums_int8((const int8_t*)qrow, xq, dim_in, isum);
    else
        ora_block_isums(qrow, xq, dim_in, isum);
    float acc = 0.0f;
    for (int64_t b = 0; b < nb; ++b) acc = fmaf(xd[b], (float)isum[b], acc);
    free(isum);
    return s_w * acc;
}

/* One output of an int4 x Q8 matrix-vector product, contract F. */
ORA_API float ora_row_dot(const uint8_t* qrow, float s_w, const int8_t* xq, const float* xd,
                          int64_t dim_in) {
    int64_t nb = dim_in / 32;
    int32_t* isum = (int32_t*)malloc((size_t)nb * sizeof(int32_t));
    ora_block_isums(qrow, xq, dim_in, isum);
    float acc = 0.0f;
    for (int64_t b = 0; b < nb; ++b) acc = fmaf(xd[b], (float)isum[b], acc);
    free(isum);
    return s_w * acc;
}

/* One expert's weights, row-major [out x in] matrices: packed int4 (in/2
 * bytes per row) when bits is 4 (or 0), int8 (in bytes per row) when 8. */
typedef struct {
    const uint8_t* gate_q; /* [inter x hidden*bits/8] */
    const float* gate_s;   /* [inter] */
    const uint8_t* up_q;   /* [inter x hidden*bits/8] */
    const float* up_s;     /* [inter] */
    const uint8_t* down_q; /* [hidden x inter*bits/8] */
    const float* down_s;   /* [hidden] */
    int32_t bits;
} ora_expert;

/* SwiGLU expert on one Q8 token:
 *   g[o] = row_dot(gate o), u[o] = row_dot(up o)          o < inter
 *   h[o] = (g * sigmoid(g)) * u
 *   h -> Q8_0 (32-blocks along inter)
 *   y[o'] = row_dot(down o', hq, hd)                      o' < hidden
 * hq_out / hd_out (may be NULL) receive the re-quantised intermediate. */
ORA_API void ora_expert_ffn_token(const ora_expert* ex, int64_t hidden, int64_t inter,
                                  const int8_t* xq, const float* xd, float* y, int8_t* hq_out,
                                  float* hd_out) {
    float* h = (float*)malloc((size_t)inter * sizeof(float));
    int8_t* hq = (int8_t*)malloc((size_t)inter);
    float* hd = (float*)malloc((size_t)(inter / 32) * sizeof(float));
    const int bits = ex->bits == 8 ? 8 : 4;
    const int64_t rb_in = hidden * bits / 8, rb_h = inter * bits / 8; /* bytes per weight row */
    for (int64_t o = 0; o < inter; ++o) {
        float g = ora_row_dot_bits(ex->gate_q + o * rb_in, bits, ex->gate_s[o], xq, xd, hidden);
        float u = ora_row_dot_bits(ex->up_q + o * rb_in, bits, ex->up_s[o], xq, xd, hidden);
        float sg = ora_sigmoid(g);
        h[o] = (g * sg) * u;
    }
    ora_quantize_act_q8(h, 1, inter, hq, hd);
    for (int64_t o = 0; o < hidden; ++o)
        y[o] = ora_row_dot_bits(ex->down_q + o * rb_h, bits, ex->down_s[o], hq, hd, inter);
    if (hq_out) memcpy(hq_out, hq, (size_t)inter);
    if (hd_out) memcpy(hd_out, hd, (size_t)(inter / 32) * sizeof(float));
    free(h);
    free(hq);
    free(hd);
}

/* The same expert on n_tok Q8 tokens: y is [n_tok x hidden]. */
ORA_API void ora_expert_ffn(const ora_expert* ex, int64_t hidden, int64_t inter, const int8_t* xq,
                            const float* xd, int64_t n_tok, float* y) {
    for (int64_t t = 0; t < n_tok; ++t)
        ora_expert_ffn_token(ex, hidden, inter, xq + t * hidden, xd + t * (hidden / 32),
                             y + t * hidden, NULL, NULL);
}

/* ------------------------------------------------------------------------ */
/* The layer                                                                 */
/* ------------------------------------------------------------------------ */

typedef struct {
    int32_t hidden, inter, n_experts, top_k, n_shared, shared_inter, norm_topk_prob;
    float routed_scaling_factor;
    const float* w_router;     /* [E x hidden] F32 */
    const float* bias;         /* [E] F32 correction bias */
    const ora_expert* experts; /* [E]; an entry with gate_q == NULL is "not supplied" */
    const ora_expert* shared;  /* [n_shared] */
} ora_layer;

/* out[t] = sum_k w[t,k] * E_{idx[t,k]}(x_t) + sum_s S_s(x_t), contracts R,F,C.
 * idx_out / w_out (may be NULL) receive the routing.  Returns 0, or -1 when
 * a selected expert was not supplied (the caller supplies only the experts
 * the routing needs, which it can learn from ora_route first). */
ORA_API int ora_moe_layer(const ora_layer* L, const float* x, int64_t n_tok, float* out,
                          int32_t* idx_out, float* w_out) {
    const int64_t H = L->hidden, K = L->top_k;
    int rc = 0;
    int8_t* xq = (int8_t*)malloc((size_t)(n_tok * H));
    float* xd = (float*)malloc((size_t)(n_tok * (H / 32)) * sizeof(float));
    int32_t* idx = (int32_t*)malloc((size_t)(n_tok * K) * sizeof(int32_t));
    float* w = (float*)malloc((size_t)(n_tok * K) * sizeof(float));
    float* yk = (float*)malloc((size_t)(K > 0 ? K : 1) * (size_t)H * sizeof(float));
    float* ys = (float*)malloc((size_t)(L->n_shared > 0 ? L->n_shared : 1) * (size_t)H * sizeof(float));

    ora_quantize_act_q8(x, n_tok, H, xq, xd);
    ora_route(x, L->w_router, L->bias, n_tok, L->n_experts, H, (int32_t)K, L->norm_topk_prob,
              L->routed_scaling_factor, NULL, idx, w);
    for (int64_t t = 0; t < n_tok && rc == 0; ++t) {
        const int8_t* xqt = xq + t * H;
        const float* xdt = xd + t * (H / 32);
        for (int64_t k = 0; k < K; ++k) {
            const ora_expert* ex = &L->experts[idx[t * K + k]];
            if (ex->gate_q == NULL) { rc = -1; break; }
            ora_expert_ffn_token(ex, H, L->inter, xqt, xdt, yk + k * H, NULL, NULL);
        }
        if (rc != 0) break;
        for (int32_t s = 0; s < L->n_shared; ++s)
            ora_expert_ffn_token(&L->shared[s], H, L->shared_inter, xqt, xdt, ys + (int64_t)s * H,
                                 NULL, NULL);
        for (int64_t o = 0; o < H; ++o) {
            float acc = 0.0f;
            for (int64_t k = 0; k < K; ++k) acc = fmaf(w[t * K + k], yk[k * H + o], acc);
            for (int32_t s = 0; s < L->n_shared; ++s) acc = acc + ys[(int64_t)s * H + o];
            out[t * H + o] = acc;
        }
    }
    if (idx_out) memcpy(idx_out, idx, (size_t)(n_tok * K) * sizeof(int32_t));
    if (w_out) memcpy(w_out, w, (size_t)(n_tok * K) * sizeof(float));
    free(xq);
    free(xd);
    free(idx);
    free(w);
    free(yk);
    free(ys);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Between layers of a stack: RMSNorm and the residual                       */
/* ------------------------------------------------------------------------ */

/* RMSNorm with weight 1: ss = sum of x[h]^2 under contract R (the same
 * 32-accumulator order as the router logit, so a parallel implementation can
 * reproduce it); mean = ss / H; r = 1 / sqrtf(mean + eps); y = x * r.
 * (A pre-norm reading of "RMSNorm and a residual between layers"; the pages
 * do not describe the norm.)  H must be a multiple of 128. */
ORA_API void ora_rmsnorm(const float* x, int64_t n_tok, int64_t H, float eps, float* y) {
    for (int64_t t = 0; t < n_tok; ++t) {
        const float* xt = x + t * H;
        float ss = ora_router_logit(xt, xt, H);
        float mean = ss / (float)H;
        float r = 1.0f / sqrtf(mean + eps);
        for (int64_t h = 0; h < H; ++h) y[t * H + h] = xt[h] * r;
    }
}

/* x_next = x + m, element by element (the residual of a pre-norm stack). */
ORA_API void ora_residual_add(const float* x, const float* m, int64_t n, float* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = x[i] + m[i];
}
