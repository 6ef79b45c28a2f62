/*
 * Plain CPU oracle of the forward pass of the biased-sigmoid-routed MoE FFN layer
 * (Step-3.5-Flash / Step-5-Preview), written from the method's description.
 *
 * TEST INFRASTRUCTURE ONLY. Tests, the package's smoke check and the benchmark's
 * CPU-baseline leg may load this library; the product path never does. It shares
 * no code, header or constant with the CUDA library.
 *
 * Sources (page titles and sections):
 *  [MAX-MoE]    "MAX 中 Step-3.5-Flash 架构解析", section "MoE共享专家、sigmoid 路由与激活裁剪":
 *               scores = sigmoid(gate(x)) with the gate matmul forced to FP32; the fp32
 *               per-expert router_bias is added for top-k selection only; the weights
 *               come from the uncorrected scores, are optionally normalised to sum 1
 *               and then multiplied by the routing scale; indices are clamped to
 *               [0, E-1]; output = routed_moe(x) + shared_expert(x); routed and shared
 *               experts take their own SwiGLU clip limit.
 *  [MAX-Config] same page, section "Step3p5Config配置项全解": moe_top_k,
 *               moe_router_scaling_factor = 3.0, norm_expert_weight, swiglu_limits /
 *               swiglu_limits_shared with 0.0 meaning no clip.
 *  [MAX-Weights] same page, section "权重适配从 HF checkpoint 到 MAX 布局": experts
 *               stacked [num_experts, ...], router_bias kept in float32.
 *  [miles-5.3]  miles Step-5-Preview recipe page, section 5.3: 24 MiB and 12 MiB BF16
 *               expert tensors, i.e. a fused [2I, H] gate_up and a [H, I] down matrix.
 *  [miles-5.1]  same page, section 1: the checkpoint's routed experts are FP8 E4M3 with
 *               128x128 block scales, dequantized on load (the FP8 functions at the end).
 *
 * Readings where the pages leave a step open (all restated in the design notes):
 *  - clip form: a = min(silu(g), L), u = clamp(u, -L, L), h = a*u; L = 0 means no clip;
 *  - gate_up rows: gate rows first, then up rows;
 *  - selection order: biased score descending, ties to the lower expert index, a NaN
 *    biased score below every number (ties among NaNs by index), -0.0 equal to +0.0;
 *  - normalisation has no epsilon; if the selected scores sum to 0 every selected
 *    weight is scale/k; without normalisation the weight is scale*s;
 *  - margin = (k-th biased score) - ((k+1)-th biased score) in fp32, +inf when k = E;
 *  - backward (oracle_backward): no gradient through the top-k selection (the bias gets
 *    none), clips pass the gradient at their boundary.
 *
 * Precision: inputs are bf16 bit patterns (decoded exactly). The router logit is the
 * dot product accumulated in double and rounded once to fp32 (the FP32 gate); the
 * score is sigmoid evaluated in double from that fp32 logit and rounded to fp32; the
 * biased score is an fp32 addition. Everything after selection (weights, expert
 * MLPs, combine) is evaluated in double; nothing is rounded to bf16.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* [MAX-MoE] gate(x) in FP32: logits[t,e] = fp32( sum_h x[t,h] * Wr[e,h] ), summed in
 * ascending h in double. */
void oracle_router_logits(int64_t T, int H, int E, const uint16_t *x, const uint16_t *Wr,
                          float *logits)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const uint16_t *xr = x + t * (int64_t)H;
        for (int e = 0; e < E; ++e) {
            const uint16_t *wr = Wr + (int64_t)e * H;
            double acc = 0.0;
            for (int h = 0; h < H; ++h)
                acc += bf(xr[h]) * bf(wr[h]);
            logits[t * (int64_t)E + e] = (float)acc;
        }
    }
}

/* Selection order (reading stated above): is expert a ranked before expert b? */
static int ranks_before(float ba, int ea, float bb, int eb)
{
    int na = isnan(ba), nb = isnan(bb);
    if (na != nb)
        return nb; /* the number ranks before the NaN */
    if (!na && ba != bb)
        return ba > bb;
    return ea < eb;
}

/* [MAX-MoE], [MAX-Config]: for each token, s = sigmoid(logit) in fp32,
 * corrected = s + router_bias (fp32), top-k on corrected, weights from s,
 * normalised to sum 1 when norm != 0, times scale. Ids are reported in rank order.
 * w64 (double) and w32 (fp32 rounding of w64) may each be NULL, as may margin and
 * scores. */
void oracle_router_select(int64_t T, int E, int k, const float *logits, const float *bias,
                          float scale, int norm, int32_t *idx, float *w32, double *w64,
                          float *margin, float *scores)
{
#pragma omp parallel
    {
        float *s = (float *)malloc(sizeof(float) * (size_t)E);
        float *b = (float *)malloc(sizeof(float) * (size_t)E);
        char *taken = (char *)malloc((size_t)E);
        int *order = (int *)malloc(sizeof(int) * (size_t)(k + 1));
#pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            const float *l = logits + t * (int64_t)E;
            for (int e = 0; e < E; ++e) {
                s[e] = (float)(1.0 / (1.0 + exp(-(double)l[e])));
                b[e] = s[e] + bias[e];
                taken[e] = 0;
                if (scores)
                    scores[t * (int64_t)E + e] = s[e];
            }
            int nrank = k < E ? k + 1 : E;
            /* selection by repeated scan: rank r takes the best expert not yet taken */
            for (int r = 0; r < nrank; ++r) {
                int best = -1;
                for (int e = 0; e < E; ++e) {
                    if (taken[e])
                        continue;
                    if (best < 0 || ranks_before(b[e], e, b[best], best))
                        best = e;
                }
                taken[best] = 1;
                order[r] = best;
            }
            double sum = 0.0;
            for (int j = 0; j < k; ++j)
                sum += (double)s[order[j]];
            for (int j = 0; j < k; ++j) {
                int e = order[j];
                /* [MAX-MoE] clamp to [0, E-1] as a guard (always in range here) */
                if (e < 0)
                    e = 0;
                if (e > E - 1)
                    e = E - 1;
                double w;
                if (norm)
                    w = sum > 0.0 ? (double)scale * (double)s[e] / sum : (double)scale / k;
                else
                    w = (double)scale * (double)s[e];
                idx[t * k + j] = e;
                if (w64)
                    w64[t * k + j] = w;
                if (w32)
                    w32[t * k + j] = (float)w;
            }
            if (margin)
                margin[t] = k < E ? b[order[k - 1]] - b[order[k]] : INFINITY;
        }
        free(s);
        free(b);
        free(taken);
        free(order);
    }
}

/* Token -> slot permutation (histogram, exclusive scan, stable scatter) as a plain
 * counting sort by expert, stable in token order. Group E is the shared expert: it
 * holds every token in order. counts[E+1], offsets[E+2], perm_token[T*k+T],
 * slot_of[T*k]. Returns -1 (and writes nothing further) on an id outside [0, E-1]. */
int oracle_permute(int64_t T, int k, int E, const int32_t *idx, int32_t *counts,
                   int32_t *offsets, int32_t *perm_token, int32_t *slot_of)
{
    for (int e = 0; e <= E; ++e)
        counts[e] = 0;
    for (int64_t n = 0; n < T * k; ++n) {
        if (idx[n] < 0 || idx[n] >= E)
            return -1;
        counts[idx[n]] += 1;
    }
    counts[E] = (int32_t)T;
    offsets[0] = 0;
    for (int e = 0; e <= E; ++e)
        offsets[e + 1] = offsets[e] + counts[e];
    int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));
    for (int e = 0; e <= E; ++e)
        cursor[e] = offsets[e];
    for (int64_t t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int e = idx[t * k + j];
            int32_t slot = cursor[e]++;
            perm_token[slot] = (int32_t)t;
            slot_of[t * k + j] = slot;
        }
        perm_token[cursor[E]++] = (int32_t)t;
    }
    free(cursor);
    return 0;
}

/* SwiGLU hidden activation of one token through one expert ([MAX-MoE] clipped
 * activation; [miles-5.3] fused [2I, H] gate_up, gate rows first):
 *   g_i = sum_h Wgu[i,h] x_h, u_i = sum_h Wgu[I+i,h] x_h,
 *   a_i = silu(g_i), clipped a_i = min(a_i, L), u_i = clamp(u_i, -L, L) when L > 0,
 *   hid_i = a_i * u_i. */
void oracle_swiglu_hidden(int H, int Iw, const uint16_t *x_row, const uint16_t *Wgu,
                          double limit, double *hid)
{
    for (int i = 0; i < Iw; ++i) {
        const uint16_t *wg = Wgu + (int64_t)i * H;
        const uint16_t *wu = Wgu + (int64_t)(Iw + i) * H;
        double g = 0.0, u = 0.0;
        for (int h = 0; h < H; ++h) {
            double xv = bf(x_row[h]);
            g += bf(wg[h]) * xv;
            u += bf(wu[h]) * xv;
        }
        double a = g / (1.0 + exp(-g));
        if (limit > 0.0) {
            if (a > limit)
                a = limit;
            if (u > limit)
                u = limit;
            if (u < -limit)
                u = -limit;
        }
        hid[i] = a * u;
    }
}

/* One expert MLP on one token: out_f = sum_i Wd[f,i] * hid_i, Wd [H, Iw]. */
void oracle_swiglu_mlp(int H, int Iw, const uint16_t *x_row, const uint16_t *Wgu,
                       const uint16_t *Wd, double limit, double *out, double *hid)
{
    oracle_swiglu_hidden(H, Iw, x_row, Wgu, limit, hid);
    for (int f = 0; f < H; ++f) {
        const uint16_t *wd = Wd + (int64_t)f * Iw;
        double acc = 0.0;
        for (int i = 0; i < Iw; ++i)
            acc += bf(wd[i]) * hid[i];
        out[f] = acc;
    }
}

/* [MAX-MoE] layer output for a list of tokens:
 *   y = sum_j w_j * MLP_{e_j}(x; L_routed) + MLP_shared(x; L_shared),
 * routed terms summed in rank order, then the shared expert, in double.
 * Routed weights are given per expert id (Wgu_by_e[e] -> [2I, H], Wd_by_e[e] ->
 * [H, I]); an entry may be NULL when no listed token selects that expert.
 * Returns -1 if a selected expert's pointer is NULL, else 0. idx, w and margin
 * (each optional) receive the routing of every listed token. */
int oracle_forward_tokens(int64_t ntok, int H, int E, int k, int I, int Is, float scale,
                          int norm, float limit_routed, float limit_shared,
                          const uint16_t *x_rows, const uint16_t *Wr, const float *bias,
                          const uint16_t *const *Wgu_by_e, const uint16_t *const *Wd_by_e,
                          const uint16_t *Wsh_gu, const uint16_t *Wsh_d, double *y,
                          int32_t *idx_out, double *w_out, float *margin_out)
{
    float *logits = (float *)malloc(sizeof(float) * (size_t)(ntok * E));
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)(ntok * k));
    double *w = (double *)malloc(sizeof(double) * (size_t)(ntok * k));
    float *margin = (float *)malloc(sizeof(float) * (size_t)ntok);
    oracle_router_logits(ntok, H, E, x_rows, Wr, logits);
    oracle_router_select(ntok, E, k, logits, bias, scale, norm, idx, NULL, w, margin, NULL);
    int missing = 0;
    for (int64_t n = 0; n < ntok * k; ++n)
        if (!Wgu_by_e[idx[n]] || !Wd_by_e[idx[n]])
            missing = 1;
    if (!missing) {
#pragma omp parallel
        {
            int Imax = I > Is ? I : Is;
            double *hid = (double *)malloc(sizeof(double) * (size_t)Imax);
            double *o = (double *)malloc(sizeof(double) * (size_t)H);
#pragma omp for schedule(dynamic, 1)
            for (int64_t t = 0; t < ntok; ++t) {
                const uint16_t *xr = x_rows + t * (int64_t)H;
                double *yr = y + t * (int64_t)H;
                for (int f = 0; f < H; ++f)
                    yr[f] = 0.0;
                for (int j = 0; j < k; ++j) {
                    int e = idx[t * k + j];
                    oracle_swiglu_mlp(H, I, xr, Wgu_by_e[e], Wd_by_e[e], limit_routed, o, hid);
                    for (int f = 0; f < H; ++f)
                        yr[f] += w[t * k + j] * o[f];
                }
                oracle_swiglu_mlp(H, Is, xr, Wsh_gu, Wsh_d, limit_shared, o, hid);
                for (int f = 0; f < H; ++f)
                    yr[f] += o[f];
            }
            free(hid);
            free(o);
        }
    }
    if (idx_out)
        memcpy(idx_out, idx, sizeof(int32_t) * (size_t)(ntok * k));
    if (w_out)
        memcpy(w_out, w, sizeof(double) * (size_t)(ntok * k));
    if (margin_out)
        memcpy(margin_out, margin, sizeof(float) * (size_t)ntok);
    free(logits);
    free(idx);
    free(w);
    free(margin);
    return missing ? -1 : 0;
}

/* Layer output with the routing supplied by the caller (routing replay; the pages' fake
 * balanced static expert routing): y = sum_j w[t,j] * MLP_{idx[t,j]}(x; L_routed) +
 * MLP_shared(x; L_shared), routed terms summed in the given order, in double. Ids are
 * clamped to [0, E-1] like the router's. Returns -1 if a used expert's pointer is NULL. */
int oracle_forward_given_routing(int64_t ntok, int H, int E, int k, int I, int Is, float limit_routed,
                                 float limit_shared, const uint16_t *x_rows, const int32_t *idx,
                                 const float *w, const uint16_t *const *Wgu_by_e,
                                 const uint16_t *const *Wd_by_e, const uint16_t *Wsh_gu,
                                 const uint16_t *Wsh_d, double *y)
{
    for (int64_t n = 0; n < ntok * k; ++n) {
        int e = idx[n] < 0 ? 0 : (idx[n] > E - 1 ? E - 1 : idx[n]);
        if (!Wgu_by_e[e] || !Wd_by_e[e])
            return -1;
    }
#pragma omp parallel
    {
        int Imax = I > Is ? I : Is;
        double *hid = (double *)malloc(sizeof(double) * (size_t)Imax);
        double *o = (double *)malloc(sizeof(double) * (size_t)H);
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < ntok; ++t) {
            const uint16_t *xr = x_rows + t * (int64_t)H;
            double *yr = y + t * (int64_t)H;
            for (int f = 0; f < H; ++f)
                yr[f] = 0.0;
            for (int j = 0; j < k; ++j) {
                int e = idx[t * k + j];
                e = e < 0 ? 0 : (e > E - 1 ? E - 1 : e);
                oracle_swiglu_mlp(H, I, xr, Wgu_by_e[e], Wd_by_e[e], limit_routed, o, hid);
                for (int f = 0; f < H; ++f)
                    yr[f] += (double)w[t * k + j] * o[f];
            }
            oracle_swiglu_mlp(H, Is, xr, Wsh_gu, Wsh_d, limit_shared, o, hid);
            for (int f = 0; f < H; ++f)
                yr[f] += o[f];
        }
        free(hid);
        free(o);
    }
    return 0;
}

/* Dense brute force of the same layer: every expert runs on every token and a
 * [T, E] mask-weight matrix (the selection weight, 0 for unselected experts) mixes
 * them, experts summed in ascending index order, plus the shared expert. Stacked
 * weights: W_gate_up [E, 2I, H], W_down [E, H, I]. */
void oracle_forward_dense(int64_t T, int H, int E, int k, int I, int Is, float scale,
                          int norm, float limit_routed, float limit_shared,
                          const uint16_t *x, const uint16_t *Wr, const float *bias,
                          const uint16_t *W_gate_up, const uint16_t *W_down,
                          const uint16_t *Wsh_gu, const uint16_t *Wsh_d, double *y)
{
    float *logits = (float *)malloc(sizeof(float) * (size_t)(T * E));
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T * k));
    double *w = (double *)malloc(sizeof(double) * (size_t)(T * k));
    double *mask = (double *)calloc((size_t)(T * E), sizeof(double));
    oracle_router_logits(T, H, E, x, Wr, logits);
    oracle_router_select(T, E, k, logits, bias, scale, norm, idx, NULL, w, NULL, NULL);
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j)
            mask[t * E + idx[t * k + j]] = w[t * k + j];
#pragma omp parallel
    {
        int Imax = I > Is ? I : Is;
        double *hid = (double *)malloc(sizeof(double) * (size_t)Imax);
        double *o = (double *)malloc(sizeof(double) * (size_t)H);
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < T; ++t) {
            const uint16_t *xr = x + t * (int64_t)H;
            double *yr = y + t * (int64_t)H;
            for (int f = 0; f < H; ++f)
                yr[f] = 0.0;
            for (int e = 0; e < E; ++e) {
                oracle_swiglu_mlp(H, I, xr, W_gate_up + (int64_t)e * 2 * I * H,
                                  W_down + (int64_t)e * H * I, limit_routed, o, hid);
                for (int f = 0; f < H; ++f)
                    yr[f] += mask[t * E + e] * o[f];
            }
            oracle_swiglu_mlp(H, Is, xr, Wsh_gu, Wsh_d, limit_shared, o, hid);
            for (int f = 0; f < H; ++f)
                yr[f] += o[f];
        }
        free(hid);
        free(o);
    }
    free(logits);
    free(idx);
    free(w);
    free(mask);
}

/* ------------------------------------------------------------------------------------
 * FP8 routed experts. [miles-5.1] miles Step-5-Preview recipe page, section 1 ("FP8
 * checkpoint"): the routed experts are stored in FP8 E4M3 with one scale per 128x128
 * block and are dequantized on load; the shared expert is not among them and stays BF16.
 * Reading taken: the dequantized weight is w[r][c] = e4m3(q[r][c]) * scale[r/128][c/128],
 * the product rounded once to fp32, the scale an fp32 value.
 */

/* Value of one E4M3 code (OCP 8-bit floating point, E4M3 variant): sign bit, 4 exponent
 * bits with bias 7, 3 mantissa bits; exponent field 0 encodes subnormals m/8 * 2^-6;
 * exponent field 15 with mantissa 7 is NaN (the variant has no infinities), so the
 * largest finite magnitude is 1.75 * 2^8 = 448. */
double oracle_e4m3_value(uint8_t q)
{
    const int sign = q >> 7, ex = (q >> 3) & 15, man = q & 7;
    double v;
    if (ex == 15 && man == 7)
        return NAN;
    if (ex == 0)
        v = ldexp((double)man / 8.0, -6);
    else
        v = ldexp(1.0 + (double)man / 8.0, ex - 7);
    return sign ? -v : v;
}

/* Dequantize a [rows, cols] E4M3 matrix with 128x128 block scales
 * (scale [ceil(rows/128), ceil(cols/128)], row-major) to fp32. */
void oracle_dequant_block128(int64_t rows, int64_t cols, const uint8_t *q, const float *scale, float *out)
{
    const int64_t bc = (cols + 127) / 128;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            out[r * cols + c] = (float)(oracle_e4m3_value(q[r * cols + c]) * (double)scale[(r / 128) * bc + c / 128]);
}

/* The SwiGLU hidden activation and expert MLP of oracle_swiglu_hidden / oracle_swiglu_mlp
 * for fp32 weights (dequantized FP8 experts): the same sums, clip and product. */
static void swiglu_mlp_f32w(int H, int Iw, const uint16_t *x_row, const float *Wgu, const float *Wd,
                            double limit, double *out, double *hid)
{
    for (int i = 0; i < Iw; ++i) {
        const float *wg = Wgu + (int64_t)i * H;
        const float *wu = Wgu + (int64_t)(Iw + i) * H;
        double g = 0.0, u = 0.0;
        for (int h = 0; h < H; ++h) {
            double xv = bf(x_row[h]);
            g += (double)wg[h] * xv;
            u += (double)wu[h] * xv;
        }
        double a = g / (1.0 + exp(-g));
        if (limit > 0.0) {
            if (a > limit)
                a = limit;
            if (u > limit)
                u = limit;
            if (u < -limit)
                u = -limit;
        }
        hid[i] = a * u;
    }
    for (int f = 0; f < H; ++f) {
        const float *wd = Wd + (int64_t)f * Iw;
        double acc = 0.0;
        for (int i = 0; i < Iw; ++i)
            acc += (double)wd[i] * hid[i];
        out[f] = acc;
    }
}

/* Expert part of the layer for a given routing with fp32 routed-expert weights (the
 * dequantized FP8 experts, Wgu_by_e[e] -> [2I, H], Wd_by_e[e] -> [H, I]) and the BF16
 * shared expert: y = sum_j w[t,j] * MLP_{idx[t,j]}(x; L_routed) + MLP_shared(x; L_shared),
 * routed terms in the given order, in double. Returns -1 if a used expert's pointer is
 * NULL or an id is out of range. */
int oracle_experts_f32w(int64_t ntok, int H, int E, int k, int I, int Is, float limit_routed,
                        float limit_shared, const uint16_t *x_rows, const int32_t *idx, const double *w,
                        const float *const *Wgu_by_e, const float *const *Wd_by_e, const uint16_t *Wsh_gu,
                        const uint16_t *Wsh_d, double *y)
{
    for (int64_t n = 0; n < ntok * k; ++n)
        if (idx[n] < 0 || idx[n] >= E || !Wgu_by_e[idx[n]] || !Wd_by_e[idx[n]])
            return -1;
#pragma omp parallel
    {
        int Imax = I > Is ? I : Is;
        double *hid = (double *)malloc(sizeof(double) * (size_t)Imax);
        double *o = (double *)malloc(sizeof(double) * (size_t)H);
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < ntok; ++t) {
            const uint16_t *xr = x_rows + t * (int64_t)H;
            double *yr = y + t * (int64_t)H;
            for (int f = 0; f < H; ++f)
                yr[f] = 0.0;
            for (int j = 0; j < k; ++j) {
                int e = idx[t * k + j];
                swiglu_mlp_f32w(H, I, xr, Wgu_by_e[e], Wd_by_e[e], limit_routed, o, hid);
                for (int f = 0; f < H; ++f)
                    yr[f] += w[t * k + j] * o[f];
            }
            oracle_swiglu_mlp(H, Is, xr, Wsh_gu, Wsh_d, limit_shared, o, hid);
            for (int f = 0; f < H; ++f)
                yr[f] += o[f];
        }
        free(hid);
        free(o);
    }
    return 0;
}

/* ------------------------------------------------------------------------------------
 * Backward pass of the layer (the layer is trained: NeMo AutoModel Step-5-Preview page,
 * benchmark recipe runs forward, backward and optimizer steps; miles page: BF16 training).
 * The pages give no formulas; this is the chain rule on the forward above, with two
 * readings: no gradient flows through the top-k selection (the selected set is a step
 * function of the biased scores, so the router bias receives none and the logits only
 * through the selected experts' weights), and a clip passes the gradient at its boundary
 * (a == L, |u| == L), as an inclusive clamp does.
 *
 * Given dy = dLoss/dy [ntok, H] (fp32), with the forward's selection (ids e_j, scores s):
 *   per selected (t, j), expert e = e_j, weight w_j:
 *     g = Wg_e x, u = Wu_e x, a = silu(g), clipped a_c, u_c, h = a_c u_c, o = Wd_e h
 *     dW_down_e += (w_j dy) h^T;  dh = w_j Wd_e^T dy;  dw_j = dy . o
 *     da = dh u_c [a <= L],  du = dh a_c [-L <= u <= L]   (masks only when L > 0)
 *     dg = da silu'(g),  silu'(g) = sig(g) (1 + g (1 - sig(g)))
 *     dWg_e += dg x^T, dWu_e += du x^T,  dx += Wg_e^T dg + Wu_e^T du
 *   the shared expert the same with weight 1 and no dw;
 *   router, normalised (Z = sum of the k selected scores, c = scale): w_j = c s_j / Z,
 *     ds_i = (c / Z) dw_i - (c / Z^2) sum_j dw_j s_j;  otherwise w_j = c s_j, ds_i = c dw_i;
 *     dlogit_i = ds_i s_i (1 - s_i) for the selected experts, 0 for the others;
 *     dWr[e] += dlogit_e x,  dx += sum_e dlogit_e Wr[e].
 * Everything in double; weights stacked: W_gate_up [E, 2I, H] (gate rows first),
 * W_down [E, H, I]. Outputs are overwritten. Returns 0.
 */
static void mlp_backward(int H, int Iw, const uint16_t *x_row, const uint16_t *Wgu, const uint16_t *Wd,
                         double limit, double wgt, const float *dy_row, double *dWgu, double *dWd, double *dx_row,
                         double *dw_out, double *hid, double *gpre, double *upre, double *dh)
{
    for (int i = 0; i < Iw; ++i) {
        const uint16_t *wg = Wgu + (int64_t)i * H;
        const uint16_t *wu = Wgu + (int64_t)(Iw + i) * H;
        double g = 0.0, u = 0.0;
        for (int h = 0; h < H; ++h) {
            double xv = bf(x_row[h]);
            g += bf(wg[h]) * xv;
            u += bf(wu[h]) * xv;
        }
        gpre[i] = g;
        upre[i] = u;
        double a = g / (1.0 + exp(-g)), uc = u;
        if (limit > 0.0) {
            if (a > limit)
                a = limit;
            if (uc > limit)
                uc = limit;
            if (uc < -limit)
                uc = -limit;
        }
        hid[i] = a * uc;
    }
    /* dw = dy . (Wd h); dh = w Wd^T dy; dWd += (w dy) h^T */
    double dw = 0.0;
    for (int i = 0; i < Iw; ++i)
        dh[i] = 0.0;
    for (int f = 0; f < H; ++f) {
        const uint16_t *wd = Wd + (int64_t)f * Iw;
        const double d = (double)dy_row[f];
        double o = 0.0;
        for (int i = 0; i < Iw; ++i) {
            o += bf(wd[i]) * hid[i];
            dh[i] += bf(wd[i]) * d;
        }
        dw += d * o;
        double *dwd = dWd + (int64_t)f * Iw;
        for (int i = 0; i < Iw; ++i)
            dwd[i] += wgt * d * hid[i];
    }
    if (dw_out)
        *dw_out = dw;
    for (int i = 0; i < Iw; ++i) {
        const double g = gpre[i], u = upre[i];
        const double sg = 1.0 / (1.0 + exp(-g));
        const double a = g * sg;
        double ac = a, uc = u, ma = 1.0, mu = 1.0;
        if (limit > 0.0) {
            if (a > limit) {
                ac = limit;
                ma = 0.0;
            }
            if (u > limit) {
                uc = limit;
                mu = 0.0;
            } else if (u < -limit) {
                uc = -limit;
                mu = 0.0;
            }
        }
        const double dhi = wgt * dh[i];
        const double dg = dhi * uc * ma * sg * (1.0 + g * (1.0 - sg));
        const double du = dhi * ac * mu;
        const uint16_t *wg = Wgu + (int64_t)i * H;
        const uint16_t *wu = Wgu + (int64_t)(Iw + i) * H;
        double *dwg = dWgu + (int64_t)i * H;
        double *dwu = dWgu + (int64_t)(Iw + i) * H;
        for (int h = 0; h < H; ++h) {
            const double xv = bf(x_row[h]);
            dwg[h] += dg * xv;
            dwu[h] += du * xv;
            dx_row[h] += bf(wg[h]) * dg + bf(wu[h]) * du;
        }
    }
}

int oracle_backward(int64_t T, int H, int E, int k, int I, int Is, float scale, int norm, float limit_routed,
                    float limit_shared, const uint16_t *x, const uint16_t *Wr, const float *bias,
                    const uint16_t *W_gate_up, const uint16_t *W_down, const uint16_t *Wsh_gu,
                    const uint16_t *Wsh_d, const float *dy, double *dx, double *dWr, double *dWgu, double *dWd,
                    double *dWsh_gu, double *dWsh_d, int32_t *idx_out, double *w_out, double *dw_out)
{
    float *logits = (float *)malloc(sizeof(float) * (size_t)(T * E));
    float *scores = (float *)malloc(sizeof(float) * (size_t)(T * E));
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T * k));
    double *w = (double *)malloc(sizeof(double) * (size_t)(T * k));
    double *dw = (double *)malloc(sizeof(double) * (size_t)(T * k));
    oracle_router_logits(T, H, E, x, Wr, logits);
    oracle_router_select(T, E, k, logits, bias, scale, norm, idx, NULL, w, NULL, scores);
    memset(dx, 0, sizeof(double) * (size_t)(T * H));
    memset(dWr, 0, sizeof(double) * (size_t)E * H);
    memset(dWgu, 0, sizeof(double) * (size_t)E * 2 * I * H);
    memset(dWd, 0, sizeof(double) * (size_t)E * H * I);
    memset(dWsh_gu, 0, sizeof(double) * (size_t)2 * Is * H);
    memset(dWsh_d, 0, sizeof(double) * (size_t)H * Is);
    int Imax = I > Is ? I : Is;
    double *buf = (double *)malloc(sizeof(double) * (size_t)4 * Imax);
    /* experts, token by token in order (weight gradients accumulate in token order) */
    for (int64_t t = 0; t < T; ++t) {
        const uint16_t *xr = x + t * (int64_t)H;
        const float *dyr = dy + t * (int64_t)H;
        double *dxr = dx + t * (int64_t)H;
        for (int j = 0; j < k; ++j) {
            const int e = idx[t * k + j];
            mlp_backward(H, I, xr, W_gate_up + (int64_t)e * 2 * I * H, W_down + (int64_t)e * H * I, limit_routed,
                         w[t * k + j], dyr, dWgu + (int64_t)e * 2 * I * H, dWd + (int64_t)e * H * I, dxr,
                         &dw[t * k + j], buf, buf + Imax, buf + 2 * Imax, buf + 3 * Imax);
        }
        mlp_backward(H, Is, xr, Wsh_gu, Wsh_d, limit_shared, 1.0, dyr, dWsh_gu, dWsh_d, dxr, NULL, buf,
                     buf + Imax, buf + 2 * Imax, buf + 3 * Imax);
        /* router: selected experts only */
        double Z = 0.0, sdw = 0.0;
        for (int j = 0; j < k; ++j) {
            const double s = scores[t * E + idx[t * k + j]];
            Z += s;
            sdw += dw[t * k + j] * s;
        }
        for (int j = 0; j < k; ++j) {
            const int e = idx[t * k + j];
            const double s = scores[t * E + e];
            double ds;
            if (norm && Z > 0.0)
                ds = (double)scale / Z * dw[t * k + j] - (double)scale / (Z * Z) * sdw;
            else if (norm)
                ds = 0.0; /* all selected scores underflowed: the weights are constant scale/k */
            else
                ds = (double)scale * dw[t * k + j];
            const double dl = ds * s * (1.0 - s);
            const uint16_t *wr = Wr + (int64_t)e * H;
            double *dwr = dWr + (int64_t)e * H;
            for (int h = 0; h < H; ++h) {
                dwr[h] += dl * bf(xr[h]);
                dxr[h] += dl * bf(wr[h]);
            }
        }
    }
    if (idx_out)
        memcpy(idx_out, idx, sizeof(int32_t) * (size_t)(T * k));
    if (w_out)
        memcpy(w_out, w, sizeof(double) * (size_t)(T * k));
    if (dw_out)
        memcpy(dw_out, dw, sizeof(double) * (size_t)(T * k));
    free(buf);
    free(logits);
    free(scores);
    free(idx);
    free(w);
    free(dw);
    return 0;
}
