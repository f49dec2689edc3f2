/*
 * CPU oracle for MoE token dispatch / combine.  TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, obviously correct C (C11, fp64 arithmetic, no vector tricks).
 * Only the tests, the smoke check and the bench's CPU-baseline leg may load
 * this library.  It shares no code, header, table or helper with the CUDA
 * path under combine_moe_route_11_b200/, and the CUDA path never calls it.
 *
 * What it computes, step by step, and the passage each step follows:
 *
 *   router    logits = x W_r^T per token (bf16 rows and router weights,
 *             summed in double, rounded to fp32): the gate ahead of top-k.
 *   route     top-k experts per token, ties to the lower expert id, and the
 *             gate weights as a softmax over the k selected logits.  The pages
 *             only fix the shape of the selection ([N, top_k] expert indices,
 *             "backends/mlx: runtime MoE expert-sort for decode", author update
 *             on the sorted path); the softmax-over-the-selected-k gating and
 *             the lower-id tie-break are the readings taken here.
 *   counts    number of (token, choice) pairs per expert.
 *   offsets   first slot of every expert inside a rank-major receive buffer:
 *             virtual rank r owns experts [r*E/R, (r+1)*E/R) and a region of
 *             C_r = N*min(k, E/R) rows at the fixed base r*C_r, so no rank
 *             needs another rank's counts before writing ("One-Sided
 *             Expert-Parallel All-to-All for Mixture-of-Experts Inference over
 *             NVLink", abstract: push without a metadata exchange into
 *             rank-major buffers that the grouped GEMM reads in place).
 *   slots     inside a region experts ascend by id and inside an expert rows
 *             ascend by source token: slot(t,j) = off[e] + #{t' < t picking e}.
 *             With one rank this is the stable sort of the flattened [N*k]
 *             expert indices ("backends/mlx: runtime MoE expert-sort for
 *             decode", the sorted gather that flattens before the argsort).
 *   dispatch  recv[slot(t,j)] = x[t] byte for byte, scales alongside
 *             ("MLX expert parallelism all_to_all PR 3158", Facts: the
 *             dispatch_local / dispatch_scatter_remote data-movement kernels).
 *   expert    identity (FP8 rows dequantised to bf16: code * block scale) or
 *             SwiGLU: H = bf16(silu(x Wg^T) * (x Wu^T)), Y = bf16(H Wd^T).
 *             With FP8 rows the SwiGLU experts are FP8 too, reading the
 *             dispatched codes and scales in place (the interface is agnostic
 *             to the activation quantisation format, arXiv 2611.13188
 *             abstract; the pages fix no FP8 GEMM format, so the readings
 *             are: weights in e4m3 with one fp32 scale per 128x128 block, the
 *             same 128-column granularity as the rows, and H quantised to
 *             e4m3 per row and 128 columns by the rows' own amax / 448 rule).
 *   combine   out[t] = sum_j w[t,j] * Y[slot(t,j)] (Facts of PR 3158:
 *             combine_gather_remote and combine_weighted_sum).
 *
 * Floating point is accumulated in double and rounded once to the output
 * type (fp32: C's round-to-nearest-even conversion; bf16: the rounding
 * written out in bf16_from_double below).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG -1
#define ORACLE_NONFINITE -2
#define ORACLE_BAD_INDEX -3

/* dtype codes shared with the Python wrapper of this file only */
#define DT_F32 0
#define DT_BF16 1
#define DT_FP8_E4M3 2

/* ---------------------------------------------------------------- numbers */

/* bf16 is the upper half of an IEEE binary32: widen by appending 16 zero bits. */
static double bf16_to_double(uint16_t b) {
    uint32_t bits = (uint32_t)b << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16, ties to even, straight from the format:
 * 8 significant bits, binary32's exponent range (normal min 2^-126, subnormal
 * quantum 2^-133, largest finite (2 - 2^-7) * 2^127). */
static uint16_t bf16_from_double(double v) {
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7F80;
    int e;
    frexp(a, &e);                  /* a in [2^(e-1), 2^e) */
    int q_exp = e - 8;             /* weight of the last of 8 significant bits */
    if (q_exp < -133) q_exp = -133;
    double q = nearbyint(ldexp(a, -q_exp)); /* default mode: nearest, ties even */
    double r = ldexp(q, q_exp);
    const double bf16_max = ldexp(255.0, 120);  /* 0x7F7F = 1.9921875 * 2^127 */
    if (r > bf16_max) return sign | 0x7F80;
    float f = (float)r;            /* exact: r has at most 8 significant bits */
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    return sign | (uint16_t)(bits >> 16);
}

/* OCP FP8 E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; exponent 0 is
 * subnormal (m/8 * 2^-6); S.1111.111 is NaN; there is no infinity. */
static double e4m3_to_double(uint8_t b) {
    int s = b >> 7, ex = (b >> 3) & 0xF, m = b & 7;
    if (ex == 0xF && m == 7) return NAN;
    double v = (ex == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, ex - 7);
    return s ? -v : v;
}

static double load_elem(const void* base, int dtype, int64_t i) {
    switch (dtype) {
    case DT_F32: return (double)((const float*)base)[i];
    case DT_BF16: return bf16_to_double(((const uint16_t*)base)[i]);
    default: return e4m3_to_double(((const uint8_t*)base)[i]);
    }
}

static void store_elem(void* base, int dtype, int64_t i, double v) {
    if (dtype == DT_F32) ((float*)base)[i] = (float)v;
    else ((uint16_t*)base)[i] = bf16_from_double(v);
}

/* Exported for the pins: the number formats by themselves. */
double oracle_bf16_to_double(uint16_t b) { return bf16_to_double(b); }
uint16_t oracle_bf16_from_double(double v) { return bf16_from_double(v); }
double oracle_e4m3_to_double(uint8_t b) { return e4m3_to_double(b); }

/* ---------------------------------------------------------------- routing */

/* Top-k selection by k passes of "largest remaining logit, lowest id on a tie",
 * then softmax over the selected logits:
 *   w_j = exp(L_j - L_0) / sum_i exp(L_i - L_0)    (L_0 is the largest). */
int oracle_route(int64_t n, int32_t n_experts, int32_t top_k, const float* logits,
                 int32_t* topk_idx, float* topk_w) {
    if (n < 0 || n_experts <= 0 || top_k <= 0 || top_k > n_experts) return ORACLE_BAD_ARG;
    unsigned char picked[4096];
    if (n_experts > 4096) return ORACLE_BAD_ARG;
    for (int64_t t = 0; t < n; ++t) {
        const float* row = logits + t * n_experts;
        for (int32_t e = 0; e < n_experts; ++e) {
            if (!isfinite(row[e])) return ORACLE_NONFINITE;
            picked[e] = 0;
        }
        double sel[64];
        if (top_k > 64) return ORACLE_BAD_ARG;
        for (int32_t j = 0; j < top_k; ++j) {
            int32_t best = -1;
            for (int32_t e = 0; e < n_experts; ++e) {
                if (picked[e]) continue;
                if (best < 0 || (double)row[e] > (double)row[best]) best = e;
            }
            picked[best] = 1;
            topk_idx[t * top_k + j] = best;
            sel[j] = (double)row[best];
        }
        double denom = 0.0;
        for (int32_t j = 0; j < top_k; ++j) denom += exp(sel[j] - sel[0]);
        for (int32_t j = 0; j < top_k; ++j)
            topk_w[t * top_k + j] = (float)(exp(sel[j] - sel[0]) / denom);
    }
    return ORACLE_OK;
}

/* Router logits: logits[t, e] = sum_d x[t, d] * w_router[e, d] -- the gate
 * that produces the [N, top_k] expert indices of "backends/mlx: runtime MoE
 * expert-sort for decode" (author updates on the sorted path) is a linear
 * map of the token's hidden row; the pages do not spell it out, so the
 * reading is the plain dot product of the bf16 row with each expert's bf16
 * router row, summed in double in increasing d and rounded once to fp32.
 * oracle_route then selects the top k of these logits. */
int oracle_router_logits(int64_t n, int32_t hidden, int32_t n_experts, const uint16_t* x,
                         const uint16_t* w_router, float* logits) {
    if (n < 0 || hidden <= 0 || n_experts <= 0) return ORACLE_BAD_ARG;
    for (int64_t t = 0; t < n; ++t) {
        const uint16_t* xr = x + t * hidden;
        for (int32_t e = 0; e < n_experts; ++e) {
            const uint16_t* wr = w_router + (int64_t)e * hidden;
            double acc = 0.0;
            for (int32_t d = 0; d < hidden; ++d) acc += bf16_to_double(xr[d]) * bf16_to_double(wr[d]);
            logits[t * n_experts + e] = (float)acc;
        }
    }
    return ORACLE_OK;
}

/* counts[e] = #{(t, j) : topk_idx[t, j] == e} */
int oracle_counts(int64_t n, int32_t n_experts, int32_t top_k, const int32_t* topk_idx,
                  int32_t* counts) {
    for (int32_t e = 0; e < n_experts; ++e) counts[e] = 0;
    for (int64_t i = 0; i < n * top_k; ++i) {
        int32_t e = topk_idx[i];
        if (e < 0 || e >= n_experts) return ORACLE_BAD_INDEX;
        counts[e] += 1;
    }
    return ORACLE_OK;
}

/* Rows of one virtual-rank region: a token picks k distinct experts, so it can
 * send at most min(k, E/R) rows to one rank. */
int64_t oracle_region_rows(int64_t n, int32_t n_experts, int32_t top_k, int32_t n_ranks) {
    int32_t per_rank = n_experts / n_ranks;
    return n * (int64_t)(top_k < per_rank ? top_k : per_rank);
}

/* expert_off[e] = (e / (E/R)) * C_r + sum of counts of the lower experts of the
 * same rank; expert_off[E] = R * C_r (the whole buffer). */
int oracle_offsets(int64_t n, int32_t n_experts, int32_t top_k, int32_t n_ranks,
                   const int32_t* counts, int64_t* expert_off) {
    if (n_ranks <= 0 || n_experts % n_ranks) return ORACLE_BAD_ARG;
    int32_t per_rank = n_experts / n_ranks;
    int64_t c_r = oracle_region_rows(n, n_experts, top_k, n_ranks);
    for (int32_t e = 0; e < n_experts; ++e) {
        int32_t r = e / per_rank;
        int64_t off = r * c_r;
        for (int32_t e2 = r * per_rank; e2 < e; ++e2) off += counts[e2];
        expert_off[e] = off;
    }
    expert_off[n_experts] = (int64_t)n_ranks * c_r;
    return ORACLE_OK;
}

/* slot(t, j) = expert_off[e] + #{t' < t : e among the picks of t'}, e = idx[t, j].
 * Walking tokens in order and keeping one fill counter per expert counts
 * exactly those earlier tokens, since a token picks an expert at most once.
 * src_of[slot] = t*k + j on filled slots, -1 elsewhere. */
int oracle_slots(int64_t n, int32_t n_experts, int32_t top_k, const int32_t* topk_idx,
                 const int64_t* expert_off, int64_t total_slots, int32_t* slot_of,
                 int32_t* src_of) {
    int64_t fill[4096];
    if (n_experts > 4096) return ORACLE_BAD_ARG;
    for (int32_t e = 0; e < n_experts; ++e) fill[e] = 0;
    for (int64_t s = 0; s < total_slots; ++s) src_of[s] = -1;
    for (int64_t t = 0; t < n; ++t) {
        for (int32_t j = 0; j < top_k; ++j) {
            int32_t e = topk_idx[t * top_k + j];
            if (e < 0 || e >= n_experts) return ORACLE_BAD_INDEX;
            int64_t s = expert_off[e] + fill[e];
            if (s < 0 || s >= total_slots) return ORACLE_BAD_INDEX;
            fill[e] += 1;
            slot_of[t * top_k + j] = (int32_t)s;
            src_of[s] = (int32_t)(t * top_k + j);
        }
    }
    return ORACLE_OK;
}

/* recv[slot_of[t, j]] = src[t], rows of row_bytes opaque bytes. */
int oracle_scatter_rows(int64_t n, int32_t top_k, int64_t row_bytes, const uint8_t* src,
                        const int32_t* slot_of, int64_t total_slots, uint8_t* recv) {
    for (int64_t t = 0; t < n; ++t)
        for (int32_t j = 0; j < top_k; ++j) {
            int64_t s = slot_of[t * top_k + j];
            if (s < 0 || s >= total_slots) return ORACLE_BAD_INDEX;
            memcpy(recv + s * row_bytes, src + t * row_bytes, (size_t)row_bytes);
        }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------- experts */

/* Identity expert on an FP8 row: Y[c] = bf16(code[c] * scale[c / block]). */
int oracle_dequant_rows(int64_t n_rows, const int32_t* rows, int32_t hidden, int32_t block,
                        const uint8_t* q, const float* scale, uint16_t* y) {
    int32_t n_blocks = hidden / block;
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t s = rows[i];
        for (int32_t c = 0; c < hidden; ++c) {
            double v = e4m3_to_double(q[s * hidden + c]) * (double)scale[s * n_blocks + c / block];
            y[s * hidden + c] = bf16_from_double(v);
        }
    }
    return ORACLE_OK;
}

/* SwiGLU expert on the listed rows of a bf16 buffer X, row s using expert
 * row_expert[i]:  g = x Wg[e]^T, u = x Wu[e]^T (Wg = rows [0, I) of
 * w_gate_up[e], Wu = rows [I, 2I)), h = bf16(silu(g) * u) with
 * silu(z) = z / (1 + exp(-z)), y = bf16(h Wd[e]^T).  h_out may be NULL. */
int oracle_swiglu_rows(int64_t n_rows, const int32_t* rows, const int32_t* row_expert,
                       int32_t hidden, int32_t inter, const uint16_t* x,
                       const uint16_t* w_gate_up, const uint16_t* w_down, uint16_t* h_out,
                       uint16_t* y) {
    static double hbuf[65536];
    if (inter > 65536) return ORACLE_BAD_ARG;
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t s = rows[i];
        int64_t e = row_expert[i];
        const uint16_t* xr = x + s * hidden;
        const uint16_t* wg = w_gate_up + e * 2 * (int64_t)inter * hidden;
        const uint16_t* wu = wg + (int64_t)inter * hidden;
        for (int32_t c = 0; c < inter; ++c) {
            double g = 0.0, u = 0.0;
            for (int32_t d = 0; d < hidden; ++d) {
                double xv = bf16_to_double(xr[d]);
                g += xv * bf16_to_double(wg[(int64_t)c * hidden + d]);
                u += xv * bf16_to_double(wu[(int64_t)c * hidden + d]);
            }
            double silu = g / (1.0 + exp(-g));
            uint16_t hb = bf16_from_double(silu * u);
            if (h_out) h_out[s * inter + c] = hb;
            hbuf[c] = bf16_to_double(hb);
        }
        const uint16_t* wd = w_down + e * (int64_t)hidden * inter;
        for (int32_t c = 0; c < hidden; ++c) {
            double acc = 0.0;
            for (int32_t d = 0; d < inter; ++d) acc += hbuf[d] * bf16_to_double(wd[(int64_t)c * inter + d]);
            y[s * hidden + c] = bf16_from_double(acc);
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------- FP8 experts */

/* e4m3_to_double of every code, filled on first use (the GEMM loops below
 * decode billions of codes at full layer sizes). */
static const double* e4m3_values(void) {
    static double tab[256];
    static int ready = 0;
    if (!ready) {
        for (int c = 0; c < 256; ++c) tab[c] = e4m3_to_double((uint8_t)c);
        ready = 1;
    }
    return tab;
}

/* Nearest finite e4m3 value to v, ties to the code whose last mantissa bit is
 * 0, magnitudes of 448 and above giving +-448 (saturation instead of NaN;
 * stated as a rule because distances to huge values round to ties).  Below
 * 448, found by scanning the 127 non-negative finite codes in increasing
 * order, where neighbouring codes are neighbouring values.  NaN inputs are
 * outside the contract. */
static uint8_t e4m3_from_float_satfinite(float v) {
    double a = fabs((double)v);
    uint8_t sign = signbit(v) ? 0x80 : 0;
    if (a >= 448.0) return sign | 0x7E;
    int best = 0;
    double best_d = a;
    for (int c = 1; c <= 0x7E; ++c) {
        double d = fabs(e4m3_to_double((uint8_t)c) - a);
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return sign | (uint8_t)best;
}

uint8_t oracle_e4m3_from_float(float v) { return e4m3_from_float_satfinite(v); }

/* FP8 quantisation of the listed bf16 rows, one fp32 scale per `block`
 * columns: s = amax / 448 (1 for an all-zero block), code = e4m3(h / s).
 * Both quotients are fp32 values: each is computed in double and rounded once
 * to float, which is the correctly rounded fp32 quotient because double
 * carries more than twice float's precision plus two bits (Figueroa, "When is
 * double rounding innocuous?", 1995). */
int oracle_quant_rows(int64_t n_rows, const int32_t* rows, int32_t width, int32_t block,
                      const uint16_t* h, uint8_t* q, float* scale) {
    if (block <= 0 || width % block) return ORACLE_BAD_ARG;
    int32_t n_blocks = width / block;
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t s = rows[i];
        for (int32_t b = 0; b < n_blocks; ++b) {
            const uint16_t* hb = h + s * width + (int64_t)b * block;
            double amax = 0.0;
            for (int32_t c = 0; c < block; ++c) {
                double a = fabs(bf16_to_double(hb[c]));
                if (a > amax) amax = a;
            }
            float sc = amax > 0.0 ? (float)(amax / 448.0) : 1.0f;
            scale[s * n_blocks + b] = sc;
            for (int32_t c = 0; c < block; ++c) {
                float v = (float)(bf16_to_double(hb[c]) / (double)sc);
                q[s * width + (int64_t)b * block + c] = e4m3_from_float_satfinite(v);
            }
        }
    }
    return ORACLE_OK;
}

/* FP8 SwiGLU gate/up step on the listed rows of the e4m3 buffer X (scales xs,
 * one per row and `block` columns), row s using expert row_expert[i], whose
 * e4m3 weights w_gate_up[e] (rows [0, I) gate, [I, 2I) up) carry one scale
 * per block x block tile, ws[e][row / block][col / block]:
 *   g[c] = sum_d (X[s,d] xs[s,d/block]) (Wg[c,d] ws[e][c/block][d/block])
 *   u[c] = the same with row I + c,       h[c] = bf16(silu(g[c]) u[c])
 * summed in double.  g_out, u_out (double [T, I]) may be NULL. */
int oracle_fp8_gate_up_rows(int64_t n_rows, const int32_t* rows, const int32_t* row_expert,
                            int32_t hidden, int32_t inter, int32_t block, const uint8_t* xq,
                            const float* xs, const uint8_t* w_gate_up, const float* w_gate_up_s,
                            uint16_t* h_out, double* g_out, double* u_out) {
    if (block <= 0 || hidden % block || inter % block) return ORACLE_BAD_ARG;
    int32_t kb = hidden / block;               /* scale blocks along the reduction */
    int32_t rb = 2 * inter / block;            /* scale blocks along an expert's rows */
    const double* dec = e4m3_values();
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t s = rows[i];
        int64_t e = row_expert[i];
        const uint8_t* xr = xq + s * hidden;
        const float* xsr = xs + s * kb;
        const uint8_t* w = w_gate_up + e * 2 * (int64_t)inter * hidden;
        const float* wsc = w_gate_up_s + e * (int64_t)rb * kb;
        for (int32_t c = 0; c < inter; ++c) {
            int64_t cu = (int64_t)inter + c;
            double g = 0.0, u = 0.0;
            for (int32_t d = 0; d < hidden; ++d) {
                double xv = dec[xr[d]] * (double)xsr[d / block];
                g += xv * (dec[w[(int64_t)c * hidden + d]] *
                           (double)wsc[(int64_t)(c / block) * kb + d / block]);
                u += xv * (dec[w[cu * hidden + d]] *
                           (double)wsc[(cu / block) * kb + d / block]);
            }
            if (g_out) g_out[s * inter + c] = g;
            if (u_out) u_out[s * inter + c] = u;
            h_out[s * inter + c] = bf16_from_double(g / (1.0 + exp(-g)) * u);
        }
    }
    return ORACLE_OK;
}

/* FP8 down projection on the listed rows of the e4m3 buffer H (scales hs, one
 * per row and `block` columns), with expert e's e4m3 w_down[e] [D, I] and its
 * per-tile scales wds[e][row / block][col / block]:
 *   y[c] = bf16( sum_d (H[s,d] hs[s,d/block]) (Wd[c,d] wds[e][c/block][d/block]) ). */
int oracle_fp8_down_rows(int64_t n_rows, const int32_t* rows, const int32_t* row_expert,
                         int32_t hidden, int32_t inter, int32_t block, const uint8_t* hq,
                         const float* hs, const uint8_t* w_down, const float* w_down_s,
                         uint16_t* y) {
    if (block <= 0 || hidden % block || inter % block) return ORACLE_BAD_ARG;
    int32_t kb = inter / block;
    int32_t rb = hidden / block;
    const double* dec = e4m3_values();
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t s = rows[i];
        int64_t e = row_expert[i];
        const uint8_t* hr = hq + s * inter;
        const float* hsr = hs + s * kb;
        const uint8_t* w = w_down + e * (int64_t)hidden * inter;
        const float* wsc = w_down_s + e * (int64_t)rb * kb;
        for (int32_t c = 0; c < hidden; ++c) {
            double acc = 0.0;
            for (int32_t d = 0; d < inter; ++d)
                acc += (dec[hr[d]] * (double)hsr[d / block]) *
                       (dec[w[(int64_t)c * inter + d]] *
                        (double)wsc[(int64_t)(c / block) * kb + d / block]);
            y[s * hidden + c] = bf16_from_double(acc);
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------- combine */

/* out[t, c] = sum_j w[t, j] * Y[slot_of[t, j], c], summed in double. */
int oracle_combine(int64_t n, int32_t top_k, int32_t hidden, int y_dtype, const void* y,
                   const float* topk_w, const int32_t* slot_of, int64_t total_slots,
                   int out_dtype, void* out) {
    if (out_dtype == DT_FP8_E4M3) return ORACLE_BAD_ARG;
    for (int64_t t = 0; t < n; ++t) {
        for (int32_t c = 0; c < hidden; ++c) {
            double acc = 0.0;
            for (int32_t j = 0; j < top_k; ++j) {
                int64_t s = slot_of[t * top_k + j];
                if (s < 0 || s >= total_slots) return ORACLE_BAD_INDEX;
                acc += (double)topk_w[t * top_k + j] * load_elem(y, y_dtype, s * hidden + c);
            }
            store_elem(out, out_dtype, t * hidden + c, acc);
        }
    }
    return ORACLE_OK;
}

/* Per-element bound used by the tolerance check: sum_j |w[t,j] * Y[slot,c]|. */
int oracle_combine_abs(int64_t n, int32_t top_k, int32_t hidden, int y_dtype, const void* y,
                       const float* topk_w, const int32_t* slot_of, int64_t total_slots,
                       double* out) {
    for (int64_t t = 0; t < n; ++t)
        for (int32_t c = 0; c < hidden; ++c) {
            double acc = 0.0;
            for (int32_t j = 0; j < top_k; ++j) {
                int64_t s = slot_of[t * top_k + j];
                if (s < 0 || s >= total_slots) return ORACLE_BAD_INDEX;
                acc += fabs((double)topk_w[t * top_k + j] * load_elem(y, y_dtype, s * hidden + c));
            }
            out[t * hidden + c] = acc;
        }
    return ORACLE_OK;
}
