/*
 * gdn_oracle.c -- fp64 CPU oracle for the Gated DeltaNet recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
 * its Python binding) may include, link, load or call this file.  Only the
 * tests, the package smoke check and the benchmark's CPU-baseline leg use it.
 * It shares no code, header, table or helper with the CUDA path.
 *
 * What it computes, and where the pages say so:
 *
 *  - The delta rule.  The Qwen3.8-27B architecture page (2kiu.com, "From
 *    parameter race to efficiency revolution: dissecting Qwen3.8-27B's dense
 *    architecture and long-context hybrid attention"), section 2.2, states the
 *    update S_t = S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T: the value
 *    stored under key k_t is erased, then v_t is written, with beta_t as the
 *    write strength.  Section 2.2 also keeps this state in float32
 *    (mamba_ssm_dtype).
 *  - The gate.  The same page names A_log, dt_bias, in_proj_a and in_proj_b
 *    per linear-attention layer (section 2.1) and calls the layer "Gated"
 *    (section 2.2) but prints no gate formula.  The reading used here: a decay
 *    alpha_t = exp(-exp(A_log) * softplus(a_t + dt_bias)) scales the whole
 *    erased state, S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T)
 *    + beta_t v_t k_t^T, with beta_t = sigmoid(b_t).  With alpha = 1 this is
 *    exactly the page's rule.
 *  - Output o_t = scale * S_t q_t from the state after the update, scale =
 *    1/sqrt(d_k).
 *  - Heads.  Section 2.1 gives 16 key heads and 48 value heads of width 128
 *    (linear_num_key_heads / linear_num_value_heads).  Value head h reads key
 *    head h / (Hv/Hqk) (contiguous groups of three).
 *  - Front end.  Section 2.1 gives linear_conv_kernel_dim = 4 and a
 *    conv1d.weight per layer: a causal depthwise 4-tap convolution over time,
 *    then SiLU on every channel, then q and k are divided by their L2 norm
 *    per head: y / sqrt(sum y^2 + 1e-6).
 *
 * Every function is a plain loop in the order the method states it; nothing is
 * blocked, fused or reordered.  The only exception is gdn_oracle_prefill_chunked,
 * which exists to check the chunked (WY / UT) algebra against the plain
 * recurrence, and is written out step by step from that algebra:
 *   A_ij = beta_i e^{G_i-G_j} k_i.k_j (j<i),  T = (I+A)^{-1} by forward
 *   substitution,  W = T diag(beta e^G) K,  U' = T diag(beta) V,
 *   U = U' - W S0^T,  o = scale (diag(e^G) Q S0^T + (M o QK^T) U),
 *   S = e^{G_C} S0 + U^T diag(e^{G_C-G}) K,  with G the running sum of
 *   log(alpha) inside the chunk.
 *
 * Inputs q, k, v may be given either as bf16 bit patterns (uint16) or as
 * float64; bf16 is widened exactly.  All arithmetic is in double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- element fetch: exact widening of bf16 bits or plain f64 ---------------- */

static double bf16_bits_to_f64(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* copies n contiguous elements starting at element offset off */
static void fetch(const void* base, int is_f64, int64_t off, int n, double* dst) {
    if (is_f64) {
        const double* p = (const double*)base + off;
        for (int i = 0; i < n; ++i) dst[i] = p[i];
    } else {
        const uint16_t* p = (const uint16_t*)base + off;
        for (int i = 0; i < n; ++i) dst[i] = bf16_bits_to_f64(p[i]);
    }
}

/* ---- gates ------------------------------------------------------------------ */

/* softplus(x) = log(1 + e^x), evaluated without overflow */
static double softplus(double x) {
    if (x > 0.0) return x + log1p(exp(-x));
    return log1p(exp(x));
}

/* log(alpha) = -exp(A_log) * softplus(a + dt_bias) */
double gdn_oracle_log_alpha(double a, double A_log, double dt_bias) {
    return -exp(A_log) * softplus(a + dt_bias);
}

double gdn_oracle_beta(double b) { return 1.0 / (1.0 + exp(-b)); }

/* ---- one recurrence step on one head --------------------------------------- */

/* S (dv x dk, row-major) <- alpha S (I - beta k k^T) + beta v k^T,
 * then o = scale * S q.  Written as x = S k, S = alpha S + beta (v - alpha x) k^T,
 * which is the same product expanded. */
static void delta_step(double* S, int dv, int dk, const double* q, const double* k,
                       const double* v, double alpha, double beta, double scale,
                       double* o /* may be NULL */, double* x /* scratch dv */) {
    for (int i = 0; i < dv; ++i) {
        double acc = 0.0;
        for (int j = 0; j < dk; ++j) acc += S[(int64_t)i * dk + j] * k[j];
        x[i] = acc;
    }
    for (int i = 0; i < dv; ++i) {
        double u = beta * (v[i] - alpha * x[i]);
        for (int j = 0; j < dk; ++j)
            S[(int64_t)i * dk + j] = alpha * S[(int64_t)i * dk + j] + u * k[j];
    }
    if (o) {
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[(int64_t)i * dk + j] * q[j];
            o[i] = scale * acc;
        }
    }
}

static int set_threads(int threads) {
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
    return omp_get_max_threads();
#else
    (void)threads;
    return 1;
#endif
}

int gdn_oracle_max_threads(int threads) { return set_threads(threads); }

/* ---- prefill: the plain sequential recurrence ------------------------------ */

/*
 * q [T, Hqk, dk], k [T, Hqk, dk], v [T, Hv, dv]   (bf16 bits or f64, see is_f64)
 * a, b [T, Hv] float;  A_log, dt_bias [Hv] float
 * cu_seqlens [n_seq + 1] int32 (NULL: one sequence of length T)
 * initial_state [n_seq, Hv, dv, dk] float (NULL: zeros)
 * Only value heads h_begin <= h < h_end are computed; nh = h_end - h_begin.
 * o [T, nh, dv] double (NULL: not written)
 * final_state [n_seq, nh, dv, dk] double (NULL: not written)
 * seq_mask [n_seq] (NULL: all sequences) -- sequences with mask 0 are skipped.
 * Returns 0, or -1 on bad arguments.
 */
int gdn_oracle_prefill(const void* q, const void* k, const void* v, int is_f64,
                       const float* a, const float* b, const float* A_log, const float* dt_bias,
                       const int32_t* cu_seqlens, int32_t n_seq, int64_t T,
                       int32_t Hqk, int32_t Hv, int32_t dk, int32_t dv, double scale,
                       const float* initial_state, int32_t h_begin, int32_t h_end,
                       const uint8_t* seq_mask, double* o, double* final_state, int threads) {
    if (Hqk <= 0 || Hv <= 0 || Hv % Hqk || h_begin < 0 || h_end > Hv || h_begin >= h_end)
        return -1;
    if (n_seq <= 0 || T < 0) return -1;
    if (!cu_seqlens && n_seq != 1) return -1;
    set_threads(threads);
    const int nh = h_end - h_begin;
    const int grp = Hv / Hqk;
    const int64_t units = (int64_t)n_seq * nh;
    int bad = 0;

#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t u = 0; u < units; ++u) {
        const int n = (int)(u / nh);
        const int hl = (int)(u % nh);
        const int h = h_begin + hl;
        const int g = h / grp;
        if (seq_mask && !seq_mask[n]) continue;
        const int64_t bos = cu_seqlens ? cu_seqlens[n] : 0;
        const int64_t eos = cu_seqlens ? cu_seqlens[n + 1] : T;
        if (bos < 0 || eos < bos || eos > T) { bad = 1; continue; }

        double* S = (double*)calloc((size_t)dv * dk, sizeof(double));
        double* qt = (double*)malloc(sizeof(double) * dk);
        double* kt = (double*)malloc(sizeof(double) * dk);
        double* vt = (double*)malloc(sizeof(double) * dv);
        double* x = (double*)malloc(sizeof(double) * dv);
        double* ot = (double*)malloc(sizeof(double) * dv);
        if (initial_state) {
            const float* s0 = initial_state + ((int64_t)n * Hv + h) * dv * dk;
            for (int64_t i = 0; i < (int64_t)dv * dk; ++i) S[i] = s0[i];
        }
        for (int64_t t = bos; t < eos; ++t) {
            fetch(q, is_f64, (t * Hqk + g) * dk, dk, qt);
            fetch(k, is_f64, (t * Hqk + g) * dk, dk, kt);
            fetch(v, is_f64, (t * Hv + h) * dv, dv, vt);
            const double la = gdn_oracle_log_alpha(a[t * Hv + h], A_log[h], dt_bias[h]);
            const double alpha = exp(la);
            const double beta = gdn_oracle_beta(b[t * Hv + h]);
            delta_step(S, dv, dk, qt, kt, vt, alpha, beta, scale, o ? ot : NULL, x);
            if (o) {
                double* dst = o + (t * nh + hl) * dv;
                for (int i = 0; i < dv; ++i) dst[i] = ot[i];
            }
        }
        if (final_state) {
            double* dst = final_state + ((int64_t)n * nh + hl) * dv * dk;
            memcpy(dst, S, sizeof(double) * dv * dk);
        }
        free(S); free(qt); free(kt); free(vt); free(x); free(ot);
    }
    return bad ? -1 : 0;
}

/* ---- prefill: chunked WY / UT form (checks the chunk algebra only) --------- */

/*
 * Same arguments as gdn_oracle_prefill plus the chunk length C >= 1.  Chunks
 * restart at every sequence start; the last chunk of a sequence may be short.
 */
int gdn_oracle_prefill_chunked(const void* q, const void* k, const void* v, int is_f64,
                               const float* a, const float* b, const float* A_log,
                               const float* dt_bias, const int32_t* cu_seqlens, int32_t n_seq,
                               int64_t T, int32_t Hqk, int32_t Hv, int32_t dk, int32_t dv,
                               double scale, const float* initial_state, int32_t h_begin,
                               int32_t h_end, int32_t C, double* o, double* final_state,
                               int threads) {
    if (Hqk <= 0 || Hv <= 0 || Hv % Hqk || h_begin < 0 || h_end > Hv || h_begin >= h_end)
        return -1;
    if (n_seq <= 0 || T < 0 || C < 1) return -1;
    if (!cu_seqlens && n_seq != 1) return -1;
    set_threads(threads);
    const int nh = h_end - h_begin;
    const int grp = Hv / Hqk;
    const int64_t units = (int64_t)n_seq * nh;
    int bad = 0;

#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t u = 0; u < units; ++u) {
        const int n = (int)(u / nh);
        const int hl = (int)(u % nh);
        const int h = h_begin + hl;
        const int g = h / grp;
        const int64_t bos = cu_seqlens ? cu_seqlens[n] : 0;
        const int64_t eos = cu_seqlens ? cu_seqlens[n + 1] : T;
        if (bos < 0 || eos < bos || eos > T) { bad = 1; continue; }

        double* S = (double*)calloc((size_t)dv * dk, sizeof(double));   /* dv x dk */
        double* Q = (double*)malloc(sizeof(double) * C * dk);
        double* K = (double*)malloc(sizeof(double) * C * dk);
        double* V = (double*)malloc(sizeof(double) * C * dv);
        double* G = (double*)malloc(sizeof(double) * C);
        double* be = (double*)malloc(sizeof(double) * C);
        double* A = (double*)malloc(sizeof(double) * C * C);
        double* Tm = (double*)malloc(sizeof(double) * C * C);
        double* W = (double*)malloc(sizeof(double) * C * dk);
        double* Up = (double*)malloc(sizeof(double) * C * dv);
        double* U = (double*)malloc(sizeof(double) * C * dv);
        double* Sn = (double*)malloc(sizeof(double) * dv * dk);
        if (initial_state) {
            const float* s0 = initial_state + ((int64_t)n * Hv + h) * dv * dk;
            for (int64_t i = 0; i < (int64_t)dv * dk; ++i) S[i] = s0[i];
        }
        for (int64_t c0 = bos; c0 < eos; c0 += C) {
            const int L = (int)((eos - c0) < C ? (eos - c0) : C);
            /* load the chunk and its gates; G = running sum of log(alpha) */
            double run = 0.0;
            for (int t = 0; t < L; ++t) {
                const int64_t tt = c0 + t;
                fetch(q, is_f64, (tt * Hqk + g) * dk, dk, Q + (int64_t)t * dk);
                fetch(k, is_f64, (tt * Hqk + g) * dk, dk, K + (int64_t)t * dk);
                fetch(v, is_f64, (tt * Hv + h) * dv, dv, V + (int64_t)t * dv);
                run += gdn_oracle_log_alpha(a[tt * Hv + h], A_log[h], dt_bias[h]);
                G[t] = run;
                be[t] = gdn_oracle_beta(b[tt * Hv + h]);
            }
            /* A_ij = beta_i e^{G_i - G_j} (k_i . k_j) for j < i, else 0 */
            for (int i = 0; i < L; ++i)
                for (int j = 0; j < L; ++j) {
                    double val = 0.0;
                    if (j < i) {
                        double kk = 0.0;
                        for (int e = 0; e < dk; ++e) kk += K[(int64_t)i * dk + e] * K[(int64_t)j * dk + e];
                        val = be[i] * exp(G[i] - G[j]) * kk;
                    }
                    A[i * C + j] = val;
                }
            /* T = (I + A)^{-1}, lower unit triangular, by forward substitution:
             * row i of T is e_i - sum_{m<i} A_im T_m */
            for (int i = 0; i < L; ++i)
                for (int j = 0; j < L; ++j) {
                    double val = (i == j) ? 1.0 : 0.0;
                    for (int m = j; m < i; ++m) val -= A[i * C + m] * Tm[m * C + j];
                    Tm[i * C + j] = (j <= i) ? val : 0.0;
                }
            /* W = T diag(beta e^G) K ;  U' = T diag(beta) V */
            for (int i = 0; i < L; ++i) {
                for (int e = 0; e < dk; ++e) {
                    double acc = 0.0;
                    for (int j = 0; j <= i; ++j)
                        acc += Tm[i * C + j] * be[j] * exp(G[j]) * K[(int64_t)j * dk + e];
                    W[(int64_t)i * dk + e] = acc;
                }
                for (int e = 0; e < dv; ++e) {
                    double acc = 0.0;
                    for (int j = 0; j <= i; ++j) acc += Tm[i * C + j] * be[j] * V[(int64_t)j * dv + e];
                    Up[(int64_t)i * dv + e] = acc;
                }
            }
            /* U = U' - W S0^T   (S0 is dv x dk, so (W S0^T)_{i,e} = sum_f W_if S0_ef) */
            for (int i = 0; i < L; ++i)
                for (int e = 0; e < dv; ++e) {
                    double acc = 0.0;
                    for (int f = 0; f < dk; ++f) acc += W[(int64_t)i * dk + f] * S[(int64_t)e * dk + f];
                    U[(int64_t)i * dv + e] = Up[(int64_t)i * dv + e] - acc;
                }
            /* o_i = scale (e^{G_i} S0 q_i + sum_{j<=i} e^{G_i-G_j} (q_i . k_j) u_j) */
            if (o) {
                for (int i = 0; i < L; ++i) {
                    double* dst = o + ((c0 + i) * nh + hl) * dv;
                    for (int e = 0; e < dv; ++e) {
                        double inter = 0.0;
                        for (int f = 0; f < dk; ++f) inter += S[(int64_t)e * dk + f] * Q[(int64_t)i * dk + f];
                        double intra = 0.0;
                        for (int j = 0; j <= i; ++j) {
                            double qk = 0.0;
                            for (int f = 0; f < dk; ++f) qk += Q[(int64_t)i * dk + f] * K[(int64_t)j * dk + f];
                            intra += exp(G[i] - G[j]) * qk * U[(int64_t)j * dv + e];
                        }
                        dst[e] = scale * (exp(G[i]) * inter + intra);
                    }
                }
            }
            /* S = e^{G_L} S0 + sum_j e^{G_L - G_j} u_j k_j^T */
            const double GL = G[L - 1];
            for (int e = 0; e < dv; ++e)
                for (int f = 0; f < dk; ++f) {
                    double acc = exp(GL) * S[(int64_t)e * dk + f];
                    for (int j = 0; j < L; ++j)
                        acc += exp(GL - G[j]) * U[(int64_t)j * dv + e] * K[(int64_t)j * dk + f];
                    Sn[(int64_t)e * dk + f] = acc;
                }
            memcpy(S, Sn, sizeof(double) * dv * dk);
        }
        if (final_state) {
            double* dst = final_state + ((int64_t)n * nh + hl) * dv * dk;
            memcpy(dst, S, sizeof(double) * dv * dk);
        }
        free(S); free(Q); free(K); free(V); free(G); free(be); free(A); free(Tm);
        free(W); free(Up); free(U); free(Sn);
    }
    return bad ? -1 : 0;
}

/* ---- decode: one recurrence step per (sequence, layer) unit ---------------- */

/*
 * Units u = s * L + l for sequence s < n_seq and layer l < L.
 * q, k [U, Hqk, dk]; v [U, Hv, dv] (bf16 bits or f64); a, b [U, Hv] float;
 * A_log, dt_bias [L, Hv] float; state [U, Hv, dv, dk] float (read only here).
 * units_sel [n_sel] lists the units to compute (NULL: all units, n_sel = U).
 * o [n_sel, Hv, dv] double; state_out [n_sel, Hv, dv, dk] double (either may be NULL).
 */
int gdn_oracle_decode(const void* q, const void* k, const void* v, int is_f64, const float* a,
                      const float* b, const float* A_log, const float* dt_bias, int32_t n_seq,
                      int32_t L, int32_t Hqk, int32_t Hv, int32_t dk, int32_t dv, double scale,
                      const float* state, const int64_t* units_sel, int64_t n_sel, double* o,
                      double* state_out, int threads) {
    if (Hqk <= 0 || Hv <= 0 || Hv % Hqk || n_seq <= 0 || L <= 0) return -1;
    const int64_t U = (int64_t)n_seq * L;
    if (!units_sel) n_sel = U;
    set_threads(threads);
    const int grp = Hv / Hqk;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t w = 0; w < n_sel * Hv; ++w) {
        const int64_t si = w / Hv;
        const int h = (int)(w % Hv);
        const int64_t u = units_sel ? units_sel[si] : si;
        if (u < 0 || u >= U) { bad = 1; continue; }
        const int l = (int)(u % L);
        const int g = h / grp;
        double* S = (double*)malloc(sizeof(double) * dv * dk);
        double* qt = (double*)malloc(sizeof(double) * dk);
        double* kt = (double*)malloc(sizeof(double) * dk);
        double* vt = (double*)malloc(sizeof(double) * dv);
        double* x = (double*)malloc(sizeof(double) * dv);
        double* ot = (double*)malloc(sizeof(double) * dv);
        const float* s0 = state + (u * Hv + h) * (int64_t)dv * dk;
        for (int64_t i = 0; i < (int64_t)dv * dk; ++i) S[i] = s0[i];
        fetch(q, is_f64, (u * Hqk + g) * dk, dk, qt);
        fetch(k, is_f64, (u * Hqk + g) * dk, dk, kt);
        fetch(v, is_f64, (u * Hv + h) * dv, dv, vt);
        const double alpha = exp(gdn_oracle_log_alpha(a[u * Hv + h], A_log[l * Hv + h], dt_bias[l * Hv + h]));
        const double beta = gdn_oracle_beta(b[u * Hv + h]);
        delta_step(S, dv, dk, qt, kt, vt, alpha, beta, scale, ot, x);
        if (o) memcpy(o + (si * Hv + h) * dv, ot, sizeof(double) * dv);
        if (state_out) memcpy(state_out + (si * Hv + h) * (int64_t)dv * dk, S, sizeof(double) * dv * dk);
        free(S); free(qt); free(kt); free(vt); free(x); free(ot);
    }
    return bad ? -1 : 0;
}

/* ---- front end: causal depthwise 4-tap conv, SiLU, per-head L2 norm -------- */

/*
 * x [T, Ctot] bf16 bits, channels ordered [q heads | k heads | v heads], each
 * head d channels wide, Ctot = (2 Hqk + Hv) d.  w [Ctot, 4] float; tap j
 * multiplies x[t - 3 + j] (tap 3 is the current token).  History before a
 * sequence start is conv_state_in[n, c, 0..2] = x[bos-3 .. bos-1] (NULL: zeros);
 * no history crosses a cu_seqlens boundary.
 * Outputs (double): q [T, Hqk, d], k [T, Hqk, d], v [T, Hv, d] (any may be NULL),
 * conv_state_out [n_seq, Ctot, 3] = the last three inputs of each sequence,
 * oldest first (NULL: not written).
 */
int gdn_oracle_conv1d_silu(const uint16_t* x, const float* w, const int32_t* cu_seqlens,
                           int32_t n_seq, int64_t T, int32_t Hqk, int32_t Hv, int32_t d,
                           const float* conv_state_in, double* q, double* k, double* v,
                           double* conv_state_out, int threads) {
    if (Hqk <= 0 || Hv <= 0 || d <= 0 || n_seq <= 0 || T < 0) return -1;
    if (!cu_seqlens && n_seq != 1) return -1;
    set_threads(threads);
    const int64_t Ctot = (int64_t)(2 * Hqk + Hv) * d;
    const int64_t n_heads = 2 * Hqk + Hv;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t u = 0; u < (int64_t)n_seq * n_heads; ++u) {
        const int n = (int)(u / n_heads);
        const int hh = (int)(u % n_heads);          /* head index in the packed order */
        const int64_t bos = cu_seqlens ? cu_seqlens[n] : 0;
        const int64_t eos = cu_seqlens ? cu_seqlens[n + 1] : T;
        if (bos < 0 || eos < bos || eos > T) { bad = 1; continue; }
        double* y = (double*)malloc(sizeof(double) * d);
        for (int64_t t = bos; t < eos; ++t) {
            double ss = 0.0;
            for (int e = 0; e < d; ++e) {
                const int64_t c = (int64_t)hh * d + e;
                double acc = 0.0;
                for (int j = 0; j < 4; ++j) {
                    const int64_t tau = t - 3 + j;
                    double xv;
                    if (tau >= bos) xv = bf16_bits_to_f64(x[tau * Ctot + c]);
                    else {
                        /* position bos - m (m = 1..3) is history slot 3 - m */
                        const int64_t m = bos - tau;
                        xv = conv_state_in ? conv_state_in[((int64_t)n * Ctot + c) * 3 + (3 - m)] : 0.0;
                    }
                    acc += (double)w[c * 4 + j] * xv;
                }
                const double s = acc / (1.0 + exp(-acc));   /* SiLU */
                y[e] = s;
                ss += s * s;
            }
            if (hh < 2 * Hqk) {
                const double inv = 1.0 / sqrt(ss + 1e-6);
                for (int e = 0; e < d; ++e) y[e] *= inv;
            }
            double* dst;
            if (hh < Hqk) dst = q ? q + (t * Hqk + hh) * d : NULL;
            else if (hh < 2 * Hqk) dst = k ? k + (t * Hqk + (hh - Hqk)) * d : NULL;
            else dst = v ? v + (t * Hv + (hh - 2 * Hqk)) * d : NULL;
            if (dst) memcpy(dst, y, sizeof(double) * d);
        }
        if (conv_state_out) {
            for (int e = 0; e < d; ++e) {
                const int64_t c = (int64_t)hh * d + e;
                for (int s = 0; s < 3; ++s) {
                    const int64_t tau = eos - 3 + s;
                    double xv;
                    if (tau >= bos) xv = bf16_bits_to_f64(x[tau * Ctot + c]);
                    else {
                        const int64_t m = bos - tau;
                        xv = conv_state_in ? conv_state_in[((int64_t)n * Ctot + c) * 3 + (3 - m)] : 0.0;
                    }
                    conv_state_out[((int64_t)n * Ctot + c) * 3 + s] = xv;
                }
            }
        }
        free(y);
    }
    return bad ? -1 : 0;
}

/*
 * Gated output norm of the linear-attention layer.  The architecture page
 * (section 2.1) lists the weights `norm` and `in_proj_z` of every
 * linear-attention layer and prints no formula.  Reading used: per (token t,
 * value head h) an RMS norm over the d_v channels, one weight vector per layer
 * shared by the heads (row t uses layer t % layers), eps as given (the layer's
 * other norms use 1e-6), gated by SiLU of z:
 *     y[t,h,e] = w[l][e] * o[t,h,e] / sqrt(mean_e' o[t,h,e']^2 + eps)
 *                * z[t,h,e] / (1 + exp(-z[t,h,e])).
 * o, z, w, y in double; z may carry bf16 values widened exactly by the caller.
 */
int gdn_oracle_gated_norm(const double* o, const double* z, const double* w, int64_t T, int Hv, int d,
                          int layers, double eps, double* y) {
    if (T < 0 || Hv <= 0 || d <= 0 || layers <= 0 || !(eps >= 0.0)) return -1;
    for (int64_t t = 0; t < T; ++t) {
        const double* wl = w + (int64_t)(t % layers) * d;
        for (int h = 0; h < Hv; ++h) {
            const int64_t row = (t * Hv + h) * (int64_t)d;
            double ss = 0.0;
            for (int e = 0; e < d; ++e) ss += o[row + e] * o[row + e];
            const double inv = 1.0 / sqrt(ss / d + eps);
            for (int e = 0; e < d; ++e) {
                const double g = z[row + e] / (1.0 + exp(-z[row + e]));
                y[row + e] = wl[e] * (o[row + e] * inv) * g;
            }
        }
    }
    return 0;
}

/* ---- everything in double: forward and its gradient ------------------------ */

/*
 * gdn_oracle_prefill_f64 -- the same sequential recurrence as
 * gdn_oracle_prefill with every input in double (q, k, v, gates, initial
 * state), for the finite-difference checks of the gradient below.  One call
 * covers all value heads; o [T, Hv, dv] and final_state [n_seq, Hv, dv, dk]
 * may be NULL.
 */
int gdn_oracle_prefill_f64(const double* q, const double* k, const double* v, const double* a,
                           const double* b, const double* A_log, const double* dt_bias,
                           const int32_t* cu_seqlens, int32_t n_seq, int64_t T, int32_t Hqk,
                           int32_t Hv, int32_t dk, int32_t dv, double scale,
                           const double* initial_state, double* o, double* final_state) {
    if (Hqk <= 0 || Hv <= 0 || Hv % Hqk || n_seq <= 0 || T < 0) return -1;
    if (!cu_seqlens && n_seq != 1) return -1;
    const int grp = Hv / Hqk;
    double* S = (double*)malloc(sizeof(double) * dv * dk);
    double* x = (double*)malloc(sizeof(double) * dv);
    double* ot = (double*)malloc(sizeof(double) * dv);
    for (int n = 0; n < n_seq; ++n) {
        const int64_t bos = cu_seqlens ? cu_seqlens[n] : 0;
        const int64_t eos = cu_seqlens ? cu_seqlens[n + 1] : T;
        for (int h = 0; h < Hv; ++h) {
            const int g = h / grp;
            for (int64_t i = 0; i < (int64_t)dv * dk; ++i)
                S[i] = initial_state ? initial_state[((int64_t)n * Hv + h) * dv * dk + i] : 0.0;
            for (int64_t t = bos; t < eos; ++t) {
                const double alpha = exp(gdn_oracle_log_alpha(a[t * Hv + h], A_log[h], dt_bias[h]));
                const double beta = gdn_oracle_beta(b[t * Hv + h]);
                delta_step(S, dv, dk, q + (t * Hqk + g) * dk, k + (t * Hqk + g) * dk, v + (t * Hv + h) * dv,
                           alpha, beta, scale, o ? ot : NULL, x);
                if (o)
                    for (int i = 0; i < dv; ++i) o[(t * Hv + h) * dv + i] = ot[i];
            }
            if (final_state) memcpy(final_state + ((int64_t)n * Hv + h) * dv * dk, S, sizeof(double) * dv * dk);
        }
    }
    free(S); free(x); free(ot);
    return 0;
}

/*
 * gdn_oracle_prefill_backward -- the gradient of a scalar loss through the
 * recurrence, by reverse-mode differentiation of each step in turn (the step
 * of the architecture page, section 2.2, with the gate reading of
 * gdn_oracle_log_alpha):
 *     S_t = alpha_t S (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   S = S_{t-1},
 *     o_t = scale S_t q_t.
 * Given d_o = dL/do [T, Hv, dv] and d_final = dL/dS_T [n_seq, Hv, dv, dk]
 * (NULL: 0), with G = dL/dS_t collected from the later steps plus the
 * output's scale d_o_t q_t^T, one step back gives
 *     dq_t += scale S_t^T d_o_t
 *     dv_t  = beta G k                       (G k written g)
 *     dk_t += -alpha beta (S^T g + G^T S k) + beta G^T v
 *     dalpha = <G, S> - beta (S k).g          dbeta = -alpha (S k).g + v.g
 *     dL/dS_{t-1} = alpha (G - beta g k^T)
 * and through the gates (log alpha = -exp(A_log) softplus(a + dt_bias),
 * beta = sigmoid(b)):
 *     da_t = dalpha alpha (-exp(A_log) sigmoid(a_t + dt_bias)),
 *     ddt_bias += da_t,  dA_log += dalpha alpha log(alpha_t),
 *     db_t = dbeta beta (1 - beta).
 * dq and dk sum over the value heads that share a key head.  The states S_t
 * are kept for the whole sequence (small inputs only).  All inputs double;
 * outputs dq, dk [T, Hqk, dk], dv [T, Hv, dv], da, db [T, Hv], dA_log,
 * ddt_bias [Hv], d_initial [n_seq, Hv, dv, dk] (NULL: not written).
 */
int gdn_oracle_prefill_backward(const double* q, const double* k, const double* v, const double* a,
                                const double* b, const double* A_log, const double* dt_bias,
                                const int32_t* cu_seqlens, int32_t n_seq, int64_t T, int32_t Hqk,
                                int32_t Hv, int32_t dk, int32_t dv, double scale,
                                const double* initial_state, const double* d_o, const double* d_final,
                                double* dq, double* dkk, double* dvv, double* da, double* db,
                                double* dA_log, double* ddt_bias, double* d_initial) {
    if (Hqk <= 0 || Hv <= 0 || Hv % Hqk || n_seq <= 0 || T < 0) return -1;
    if (!cu_seqlens && n_seq != 1) return -1;
    const int grp = Hv / Hqk;
    const int64_t sz = (int64_t)dv * dk;
    memset(dq, 0, sizeof(double) * T * Hqk * dk);
    memset(dkk, 0, sizeof(double) * T * Hqk * dk);
    memset(dA_log, 0, sizeof(double) * Hv);
    memset(ddt_bias, 0, sizeof(double) * Hv);
    double* G = (double*)malloc(sizeof(double) * sz);
    double* Sk = (double*)malloc(sizeof(double) * dv);
    double* g = (double*)malloc(sizeof(double) * dv);
    double* x = (double*)malloc(sizeof(double) * dv);
    for (int n = 0; n < n_seq; ++n) {
        const int64_t bos = cu_seqlens ? cu_seqlens[n] : 0;
        const int64_t eos = cu_seqlens ? cu_seqlens[n + 1] : T;
        const int64_t len = eos - bos;
        for (int h = 0; h < Hv; ++h) {
            const int gk = h / grp;
            /* states S_{bos-1} .. S_{eos-1}: hist[j] is the state before token bos + j */
            double* hist = (double*)malloc(sizeof(double) * sz * (len + 1));
            for (int64_t i = 0; i < sz; ++i)
                hist[i] = initial_state ? initial_state[((int64_t)n * Hv + h) * sz + i] : 0.0;
            for (int64_t j = 0; j < len; ++j) {
                const int64_t t = bos + j;
                memcpy(hist + (j + 1) * sz, hist + j * sz, sizeof(double) * sz);
                const double alpha = exp(gdn_oracle_log_alpha(a[t * Hv + h], A_log[h], dt_bias[h]));
                const double beta = gdn_oracle_beta(b[t * Hv + h]);
                delta_step(hist + (j + 1) * sz, dv, dk, q + (t * Hqk + gk) * dk, k + (t * Hqk + gk) * dk,
                           v + (t * Hv + h) * dv, alpha, beta, scale, NULL, x);
            }
            for (int64_t i = 0; i < sz; ++i) G[i] = d_final ? d_final[((int64_t)n * Hv + h) * sz + i] : 0.0;
            for (int64_t j = len - 1; j >= 0; --j) {
                const int64_t t = bos + j;
                const double* S = hist + j * sz;          /* S_{t-1} */
                const double* St = hist + (j + 1) * sz;   /* S_t */
                const double* qt = q + (t * Hqk + gk) * dk;
                const double* kt = k + (t * Hqk + gk) * dk;
                const double* vt = v + (t * Hv + h) * dv;
                const double* dot = d_o + (t * Hv + h) * dv;
                const double la = gdn_oracle_log_alpha(a[t * Hv + h], A_log[h], dt_bias[h]);
                const double alpha = exp(la);
                const double beta = gdn_oracle_beta(b[t * Hv + h]);
                /* the output of step t: o_t = scale S_t q_t */
                for (int e = 0; e < dk; ++e) {
                    double acc = 0.0;
                    for (int i = 0; i < dv; ++i) acc += St[(int64_t)i * dk + e] * dot[i];
                    dq[(t * Hqk + gk) * dk + e] += scale * acc;
                }
                for (int i = 0; i < dv; ++i)
                    for (int e = 0; e < dk; ++e) G[(int64_t)i * dk + e] += scale * dot[i] * qt[e];
                /* back through the update */
                double GS = 0.0;
                for (int64_t i = 0; i < sz; ++i) GS += G[i] * S[i];
                for (int i = 0; i < dv; ++i) {
                    double s1 = 0.0, s2 = 0.0;
                    for (int e = 0; e < dk; ++e) {
                        s1 += S[(int64_t)i * dk + e] * kt[e];
                        s2 += G[(int64_t)i * dk + e] * kt[e];
                    }
                    Sk[i] = s1;
                    g[i] = s2;
                }
                double Skg = 0.0, vg = 0.0;
                for (int i = 0; i < dv; ++i) { Skg += Sk[i] * g[i]; vg += vt[i] * g[i]; }
                const double dalpha = GS - beta * Skg;
                const double dbeta = -alpha * Skg + vg;
                for (int i = 0; i < dv; ++i) dvv[(t * Hv + h) * dv + i] = beta * g[i];
                for (int e = 0; e < dk; ++e) {
                    double sg = 0.0, gs = 0.0, gv = 0.0;
                    for (int i = 0; i < dv; ++i) {
                        sg += S[(int64_t)i * dk + e] * g[i];
                        gs += G[(int64_t)i * dk + e] * Sk[i];
                        gv += G[(int64_t)i * dk + e] * vt[i];
                    }
                    dkk[(t * Hqk + gk) * dk + e] += -alpha * beta * (sg + gs) + beta * gv;
                }
                const double xg = a[t * Hv + h] + dt_bias[h];
                const double sig = 1.0 / (1.0 + exp(-xg));
                const double dla = dalpha * alpha;
                const double dat = dla * (-exp(A_log[h]) * sig);
                da[t * Hv + h] = dat;
                ddt_bias[h] += dat;
                dA_log[h] += dla * la;
                db[t * Hv + h] = dbeta * beta * (1.0 - beta);
                /* dL/dS_{t-1} = alpha (G - beta g k^T) */
                for (int i = 0; i < dv; ++i)
                    for (int e = 0; e < dk; ++e)
                        G[(int64_t)i * dk + e] = alpha * (G[(int64_t)i * dk + e] - beta * g[i] * kt[e]);
            }
            if (d_initial) memcpy(d_initial + ((int64_t)n * Hv + h) * sz, G, sizeof(double) * sz);
            free(hist);
        }
    }
    free(G); free(Sk); free(g); free(x);
    return 0;
}

/*
 * gdn_oracle_prefill_backward_chunked -- the same gradient as
 * gdn_oracle_prefill_backward, taken through the chunked (WY / UT) form of
 * gdn_oracle_prefill_chunked, chunk by chunk from the last: the algebra a
 * tensor-core backward follows.  Within a chunk of L tokens with start state S
 * (G the running sum of log alpha, gam_i = e^{G_i}, Gam_ij = e^{G_i - G_j},
 * kap_j = e^{G_{L-1} - G_j}):
 *     A = strict_lower(diag(beta) Gam o K K^T),  T = (I + A)^{-1},
 *     W = T diag(beta gam) K,  U' = T diag(beta) V,  U = U' - W S^T,
 *     P = lower(Gam o Q K^T),  O = scale (diag(gam) Q S^T + P U),
 *     S_end = gam_{L-1} S + U^T diag(kap) K.
 * Each of these is differentiated in reverse order: S_end, O, P, U, U', W, then
 * T (dA = -T^T dT T^T on the strictly lower part), A, and the decays through
 * G (dG_i collects gam, Gam and kap terms; d log alpha_m = sum_{i >= m} dG_i).
 * The gradient at the chunk start becomes dL/dS_end of the chunk before.
 * Arguments and outputs as for gdn_oracle_prefill_backward, plus the chunk
 * length C >= 1.
 */
int gdn_oracle_prefill_backward_chunked(const double* q, const double* k, const double* v, const double* a,
                                        const double* b, const double* A_log, const double* dt_bias,
                                        const int32_t* cu_seqlens, int32_t n_seq, int64_t T, int32_t Hqk,
                                        int32_t Hv, int32_t dk, int32_t dv, double scale,
                                        const double* initial_state, const double* d_o, const double* d_final,
                                        int32_t C, double* dq, double* dkk, double* dvv, double* da, double* db,
                                        double* dA_log, double* ddt_bias, double* d_initial) {
    if (Hqk <= 0 || Hv <= 0 || Hv % Hqk || n_seq <= 0 || T < 0 || C < 1) return -1;
    if (!cu_seqlens && n_seq != 1) return -1;
    const int grp = Hv / Hqk;
    const int64_t sz = (int64_t)dv * dk;
    memset(dq, 0, sizeof(double) * T * Hqk * dk);
    memset(dkk, 0, sizeof(double) * T * Hqk * dk);
    memset(dA_log, 0, sizeof(double) * Hv);
    memset(ddt_bias, 0, sizeof(double) * Hv);
    /* chunk scratch */
    double *Q = malloc(sizeof(double) * C * dk), *K = malloc(sizeof(double) * C * dk), *V = malloc(sizeof(double) * C * dv);
    double *G = malloc(sizeof(double) * C), *lg = malloc(sizeof(double) * C), *be = malloc(sizeof(double) * C);
    double *gam = malloc(sizeof(double) * C), *kap = malloc(sizeof(double) * C);
    double *KK = malloc(sizeof(double) * C * C), *QK = malloc(sizeof(double) * C * C), *Gm = malloc(sizeof(double) * C * C);
    double *A = malloc(sizeof(double) * C * C), *Tm = malloc(sizeof(double) * C * C), *P = malloc(sizeof(double) * C * C);
    double *W = malloc(sizeof(double) * C * dk), *Up = malloc(sizeof(double) * C * dv), *U = malloc(sizeof(double) * C * dv);
    double *dU = malloc(sizeof(double) * C * dv), *dK = malloc(sizeof(double) * C * dk), *dQ = malloc(sizeof(double) * C * dk);
    double *dV = malloc(sizeof(double) * C * dv), *dW = malloc(sizeof(double) * C * dk);
    double *dbe = malloc(sizeof(double) * C), *dgam = malloc(sizeof(double) * C), *dkap = malloc(sizeof(double) * C);
    double *dGm = malloc(sizeof(double) * C * C), *dT = malloc(sizeof(double) * C * C), *dA = malloc(sizeof(double) * C * C);
    double *tmp = malloc(sizeof(double) * C * C), *dG = malloc(sizeof(double) * C);
    double *TtdUp = malloc(sizeof(double) * C * dv), *TtdW = malloc(sizeof(double) * C * dk);
    double *dS = malloc(sizeof(double) * sz), *dSn = malloc(sizeof(double) * sz);
    for (int n = 0; n < n_seq; ++n) {
        const int64_t bos = cu_seqlens ? cu_seqlens[n] : 0;
        const int64_t eos = cu_seqlens ? cu_seqlens[n + 1] : T;
        const int64_t nch = (eos - bos + C - 1) / C;
        for (int h = 0; h < Hv; ++h) {
            const int gk = h / grp;
            /* chunk-start states by the chunked forward: starts[c] */
            double* starts = malloc(sizeof(double) * sz * (nch + 1));
            for (int64_t i = 0; i < sz; ++i)
                starts[i] = initial_state ? initial_state[((int64_t)n * Hv + h) * sz + i] : 0.0;
            /* one chunk's forward quantities (shared by the forward sweep and the backward one) */
#define GDN_CHUNK_FORWARD(c0, L, S)                                                                          \
    do {                                                                                                     \
        double run_ = 0.0;                                                                                   \
        for (int t_ = 0; t_ < (L); ++t_) {                                                                   \
            const int64_t tt_ = (c0) + t_;                                                                   \
            memcpy(Q + (int64_t)t_ * dk, q + (tt_ * Hqk + gk) * dk, sizeof(double) * dk);                    \
            memcpy(K + (int64_t)t_ * dk, k + (tt_ * Hqk + gk) * dk, sizeof(double) * dk);                    \
            memcpy(V + (int64_t)t_ * dv, v + (tt_ * Hv + h) * dv, sizeof(double) * dv);                      \
            lg[t_] = gdn_oracle_log_alpha(a[tt_ * Hv + h], A_log[h], dt_bias[h]);                            \
            run_ += lg[t_];                                                                                  \
            G[t_] = run_;                                                                                    \
            be[t_] = gdn_oracle_beta(b[tt_ * Hv + h]);                                                       \
        }                                                                                                    \
        for (int i_ = 0; i_ < (L); ++i_) {                                                                   \
            gam[i_] = exp(G[i_]);                                                                            \
            kap[i_] = exp(G[(L) - 1] - G[i_]);                                                               \
            for (int j_ = 0; j_ < (L); ++j_) {                                                               \
                double kk_ = 0.0, qk_ = 0.0;                                                                 \
                for (int e_ = 0; e_ < dk; ++e_) {                                                            \
                    kk_ += K[(int64_t)i_ * dk + e_] * K[(int64_t)j_ * dk + e_];                              \
                    qk_ += Q[(int64_t)i_ * dk + e_] * K[(int64_t)j_ * dk + e_];                              \
                }                                                                                            \
                KK[i_ * C + j_] = kk_;                                                                       \
                QK[i_ * C + j_] = qk_;                                                                       \
                Gm[i_ * C + j_] = j_ <= i_ ? exp(G[i_] - G[j_]) : 0.0;                                       \
                A[i_ * C + j_] = j_ < i_ ? be[i_] * Gm[i_ * C + j_] * kk_ : 0.0;                             \
                P[i_ * C + j_] = j_ <= i_ ? Gm[i_ * C + j_] * qk_ : 0.0;                                     \
            }                                                                                                \
        }                                                                                                    \
        for (int i_ = 0; i_ < (L); ++i_)                                                                     \
            for (int j_ = 0; j_ < (L); ++j_) {                                                               \
                double val_ = (i_ == j_) ? 1.0 : 0.0;                                                        \
                for (int m_ = j_; m_ < i_; ++m_) val_ -= A[i_ * C + m_] * Tm[m_ * C + j_];                   \
                Tm[i_ * C + j_] = (j_ <= i_) ? val_ : 0.0;                                                   \
            }                                                                                                \
        for (int i_ = 0; i_ < (L); ++i_) {                                                                   \
            for (int e_ = 0; e_ < dk; ++e_) {                                                                \
                double acc_ = 0.0;                                                                           \
                for (int j_ = 0; j_ <= i_; ++j_) acc_ += Tm[i_ * C + j_] * be[j_] * gam[j_] * K[(int64_t)j_ * dk + e_]; \
                W[(int64_t)i_ * dk + e_] = acc_;                                                             \
            }                                                                                                \
            for (int e_ = 0; e_ < dv; ++e_) {                                                                \
                double acc_ = 0.0;                                                                           \
                for (int j_ = 0; j_ <= i_; ++j_) acc_ += Tm[i_ * C + j_] * be[j_] * V[(int64_t)j_ * dv + e_]; \
                Up[(int64_t)i_ * dv + e_] = acc_;                                                            \
            }                                                                                                \
            for (int e_ = 0; e_ < dv; ++e_) {                                                                \
                double acc_ = 0.0;                                                                           \
                for (int f_ = 0; f_ < dk; ++f_) acc_ += W[(int64_t)i_ * dk + f_] * (S)[(int64_t)e_ * dk + f_]; \
                U[(int64_t)i_ * dv + e_] = Up[(int64_t)i_ * dv + e_] - acc_;                                 \
            }                                                                                                \
        }                                                                                                    \
    } while (0)
            for (int64_t c = 0; c < nch; ++c) {
                const int64_t c0 = bos + c * C;
                const int L = (int)((eos - c0) < C ? (eos - c0) : C);
                const double* S = starts + c * sz;
                double* Sn = starts + (c + 1) * sz;
                GDN_CHUNK_FORWARD(c0, L, S);
                for (int e = 0; e < dv; ++e)
                    for (int f = 0; f < dk; ++f) {
                        double acc = gam[L - 1] * S[(int64_t)e * dk + f];
                        for (int j = 0; j < L; ++j) acc += kap[j] * U[(int64_t)j * dv + e] * K[(int64_t)j * dk + f];
                        Sn[(int64_t)e * dk + f] = acc;
                    }
            }
            for (int64_t i = 0; i < sz; ++i) dSn[i] = d_final ? d_final[((int64_t)n * Hv + h) * sz + i] : 0.0;
            for (int64_t c = nch - 1; c >= 0; --c) {
                const int64_t c0 = bos + c * C;
                const int L = (int)((eos - c0) < C ? (eos - c0) : C);
                const double* S = starts + c * sz;
                GDN_CHUNK_FORWARD(c0, L, S);
                memset(dU, 0, sizeof(double) * C * dv);
                memset(dK, 0, sizeof(double) * C * dk);
                memset(dQ, 0, sizeof(double) * C * dk);
                memset(dV, 0, sizeof(double) * C * dv);
                memset(dbe, 0, sizeof(double) * C);
                memset(dgam, 0, sizeof(double) * C);
                memset(dkap, 0, sizeof(double) * C);
                memset(dGm, 0, sizeof(double) * C * C);
                memset(dT, 0, sizeof(double) * C * C);
                memset(dS, 0, sizeof(double) * sz);
                /* 1. S_end = gam_{L-1} S + U^T diag(kap) K */
                double dSS = 0.0;
                for (int64_t i = 0; i < sz; ++i) { dS[i] += gam[L - 1] * dSn[i]; dSS += dSn[i] * S[i]; }
                dgam[L - 1] += dSS;
                for (int j = 0; j < L; ++j) {
                    double s_ = 0.0;
                    for (int e = 0; e < dv; ++e) {
                        double dk_ = 0.0;
                        for (int f = 0; f < dk; ++f) dk_ += dSn[(int64_t)e * dk + f] * K[(int64_t)j * dk + f];
                        dU[(int64_t)j * dv + e] += kap[j] * dk_;
                        s_ += U[(int64_t)j * dv + e] * dk_;
                    }
                    dkap[j] = s_;
                    for (int f = 0; f < dk; ++f) {
                        double acc = 0.0;
                        for (int e = 0; e < dv; ++e) acc += U[(int64_t)j * dv + e] * dSn[(int64_t)e * dk + f];
                        dK[(int64_t)j * dk + f] += kap[j] * acc;
                    }
                }
                /* 2. O = scale (diag(gam) Q S^T + P U);  3. P = lower(Gam o Q K^T) */
                for (int i = 0; i < L; ++i) {
                    const double* doi = d_o + ((c0 + i) * Hv + h) * dv;
                    double sqd = 0.0;
                    for (int e = 0; e < dv; ++e) {
                        double sq = 0.0;
                        for (int f = 0; f < dk; ++f) sq += S[(int64_t)e * dk + f] * Q[(int64_t)i * dk + f];
                        sqd += doi[e] * sq;
                    }
                    dgam[i] += scale * sqd;
                    for (int f = 0; f < dk; ++f) {
                        double acc = 0.0;
                        for (int e = 0; e < dv; ++e) acc += doi[e] * S[(int64_t)e * dk + f];
                        dQ[(int64_t)i * dk + f] += scale * gam[i] * acc;
                    }
                    for (int e = 0; e < dv; ++e)
                        for (int f = 0; f < dk; ++f) dS[(int64_t)e * dk + f] += scale * gam[i] * doi[e] * Q[(int64_t)i * dk + f];
                    for (int j = 0; j <= i; ++j) {
                        double dP = 0.0;
                        for (int e = 0; e < dv; ++e) {
                            dP += doi[e] * U[(int64_t)j * dv + e];
                            dU[(int64_t)j * dv + e] += scale * P[i * C + j] * doi[e];
                        }
                        dP *= scale;
                        for (int f = 0; f < dk; ++f) {
                            dQ[(int64_t)i * dk + f] += dP * Gm[i * C + j] * K[(int64_t)j * dk + f];
                            dK[(int64_t)j * dk + f] += dP * Gm[i * C + j] * Q[(int64_t)i * dk + f];
                        }
                        dGm[i * C + j] += dP * QK[i * C + j];
                    }
                }
                /* 4. U = U' - W S^T */
                for (int i = 0; i < L; ++i)
                    for (int f = 0; f < dk; ++f) {
                        double acc = 0.0;
                        for (int e = 0; e < dv; ++e) acc += dU[(int64_t)i * dv + e] * S[(int64_t)e * dk + f];
                        dW[(int64_t)i * dk + f] = -acc;
                    }
                for (int e = 0; e < dv; ++e)
                    for (int f = 0; f < dk; ++f) {
                        double acc = 0.0;
                        for (int i = 0; i < L; ++i) acc += dU[(int64_t)i * dv + e] * W[(int64_t)i * dk + f];
                        dS[(int64_t)e * dk + f] -= acc;
                    }
                /* 5. U' = T diag(beta) V  (dU' = dU);  6. W = T diag(beta gam) K */
                for (int i = 0; i < L; ++i)
                    for (int j = 0; j <= i; ++j) {
                        double a1 = 0.0, a2 = 0.0;
                        for (int e = 0; e < dv; ++e) a1 += dU[(int64_t)i * dv + e] * V[(int64_t)j * dv + e];
                        for (int f = 0; f < dk; ++f) a2 += dW[(int64_t)i * dk + f] * K[(int64_t)j * dk + f];
                        dT[i * C + j] += be[j] * a1 + be[j] * gam[j] * a2;
                    }
                for (int j = 0; j < L; ++j) {
                    for (int e = 0; e < dv; ++e) {
                        double acc = 0.0;
                        for (int i = j; i < L; ++i) acc += Tm[i * C + j] * dU[(int64_t)i * dv + e];
                        TtdUp[(int64_t)j * dv + e] = acc;
                    }
                    for (int f = 0; f < dk; ++f) {
                        double acc = 0.0;
                        for (int i = j; i < L; ++i) acc += Tm[i * C + j] * dW[(int64_t)i * dk + f];
                        TtdW[(int64_t)j * dk + f] = acc;
                    }
                    double sv = 0.0, sk = 0.0;
                    for (int e = 0; e < dv; ++e) {
                        dV[(int64_t)j * dv + e] += be[j] * TtdUp[(int64_t)j * dv + e];
                        sv += TtdUp[(int64_t)j * dv + e] * V[(int64_t)j * dv + e];
                    }
                    for (int f = 0; f < dk; ++f) {
                        dK[(int64_t)j * dk + f] += be[j] * gam[j] * TtdW[(int64_t)j * dk + f];
                        sk += TtdW[(int64_t)j * dk + f] * K[(int64_t)j * dk + f];
                    }
                    dbe[j] += sv + gam[j] * sk;
                    dgam[j] += be[j] * sk;
                }
                /* 7. T = (I + A)^{-1}: dA = -T^T dT T^T on the strictly lower part */
                for (int i = 0; i < L; ++i)
                    for (int j = 0; j < L; ++j) {
                        double acc = 0.0;
                        for (int m = 0; m < L; ++m) acc += Tm[m * C + i] * dT[m * C + j];   /* (T^T dT)_ij */
                        tmp[i * C + j] = acc;
                    }
                for (int i = 0; i < L; ++i)
                    for (int j = 0; j < L; ++j) {
                        double acc = 0.0;
                        for (int m = 0; m < L; ++m) acc += tmp[i * C + m] * Tm[j * C + m];   /* (. T^T)_ij */
                        dA[i * C + j] = j < i ? -acc : 0.0;
                    }
                /* 8. A_ij = beta_i Gam_ij (k_i . k_j), j < i */
                for (int i = 0; i < L; ++i)
                    for (int j = 0; j < i; ++j) {
                        const double dAij = dA[i * C + j];
                        dbe[i] += dAij * Gm[i * C + j] * KK[i * C + j];
                        dGm[i * C + j] += dAij * be[i] * KK[i * C + j];
                        const double E = dAij * be[i] * Gm[i * C + j];
                        for (int f = 0; f < dk; ++f) {
                            dK[(int64_t)i * dk + f] += E * K[(int64_t)j * dk + f];
                            dK[(int64_t)j * dk + f] += E * K[(int64_t)i * dk + f];
                        }
                    }
                /* 9. decays: G_i = sum_{m <= i} log alpha_m */
                double kk_sum = 0.0;
                for (int i = 0; i < L; ++i) kk_sum += kap[i] * dkap[i];
                for (int i = 0; i < L; ++i) {
                    double acc = gam[i] * dgam[i] - kap[i] * dkap[i];
                    for (int j = 0; j <= i; ++j) acc += Gm[i * C + j] * dGm[i * C + j];
                    for (int i2 = i; i2 < L; ++i2) acc -= Gm[i2 * C + i] * dGm[i2 * C + i];
                    dG[i] = acc;
                }
                dG[L - 1] += kk_sum;
                double suffix = 0.0;
                for (int m = L - 1; m >= 0; --m) {
                    suffix += dG[m];
                    const int64_t tt = c0 + m;
                    const double la = lg[m];
                    const double xg = a[tt * Hv + h] + dt_bias[h];
                    const double sig = 1.0 / (1.0 + exp(-xg));
                    const double dat = suffix * (-exp(A_log[h]) * sig);
                    da[tt * Hv + h] = dat;
                    ddt_bias[h] += dat;
                    dA_log[h] += suffix * la;
                    db[tt * Hv + h] = dbe[m] * be[m] * (1.0 - be[m]);
                    for (int e = 0; e < dv; ++e) dvv[(tt * Hv + h) * dv + e] = dV[(int64_t)m * dv + e];
                    for (int f = 0; f < dk; ++f) {
                        dq[(tt * Hqk + gk) * dk + f] += dQ[(int64_t)m * dk + f];
                        dkk[(tt * Hqk + gk) * dk + f] += dK[(int64_t)m * dk + f];
                    }
                }
                memcpy(dSn, dS, sizeof(double) * sz);
            }
#undef GDN_CHUNK_FORWARD
            if (d_initial) memcpy(d_initial + ((int64_t)n * Hv + h) * sz, dSn, sizeof(double) * sz);
            free(starts);
        }
    }
    free(Q); free(K); free(V); free(G); free(lg); free(be); free(gam); free(kap); free(KK); free(QK); free(Gm);
    free(A); free(Tm); free(P); free(W); free(Up); free(U); free(dU); free(dK); free(dQ); free(dV); free(dW);
    free(dbe); free(dgam); free(dkap); free(dGm); free(dT); free(dA); free(tmp); free(dG); free(TtdUp);
    free(TtdW); free(dS); free(dSn);
    return 0;
}

/*
 * Front end with every input in double (x [T, Ctot], w [Ctot, 4], conv_state
 * [n_seq, Ctot, 3] or NULL): the same arithmetic as gdn_oracle_conv1d_silu,
 * for finite differences of the front end's gradient.  Outputs as there
 * (q, k, v; no conv_state_out).
 */
static double gdn_oracle_front_x(const double* x, const double* cs, int64_t Ctot, int n, int64_t bos,
                                 int64_t tau, int64_t c) {
    if (tau >= bos) return x[tau * Ctot + c];
    const int64_t m = bos - tau;                       /* position bos - m is history slot 3 - m */
    return cs ? cs[((int64_t)n * Ctot + c) * 3 + (3 - m)] : 0.0;
}

int gdn_oracle_conv1d_silu_f64(const double* x, const double* w, const int32_t* cu_seqlens, int32_t n_seq,
                               int64_t T, int32_t Hqk, int32_t Hv, int32_t d, const double* conv_state_in,
                               double* q, double* k, double* v) {
    if (Hqk <= 0 || Hv <= 0 || d <= 0 || n_seq <= 0 || T < 0) return -1;
    if (!cu_seqlens && n_seq != 1) return -1;
    const int64_t n_heads = 2 * Hqk + Hv, Ctot = n_heads * d;
    double* y = malloc(sizeof(double) * d);
    for (int n = 0; n < n_seq; ++n) {
        const int64_t bos = cu_seqlens ? cu_seqlens[n] : 0, eos = cu_seqlens ? cu_seqlens[n + 1] : T;
        for (int64_t hh = 0; hh < n_heads; ++hh)
            for (int64_t t = bos; t < eos; ++t) {
                double ss = 0.0;
                for (int e = 0; e < d; ++e) {
                    const int64_t c = hh * d + e;
                    double acc = 0.0;
                    for (int j = 0; j < 4; ++j)
                        acc += w[c * 4 + j] * gdn_oracle_front_x(x, conv_state_in, Ctot, n, bos, t - 3 + j, c);
                    y[e] = acc / (1.0 + exp(-acc));
                    ss += y[e] * y[e];
                }
                const double inv = hh < 2 * Hqk ? 1.0 / sqrt(ss + 1e-6) : 1.0;
                double* dst = hh < Hqk ? q + (t * Hqk + hh) * d
                            : hh < 2 * Hqk ? k + (t * Hqk + (hh - Hqk)) * d : v + (t * Hv + (hh - 2 * Hqk)) * d;
                for (int e = 0; e < d; ++e) dst[e] = y[e] * inv;
            }
    }
    free(y);
    return 0;
}

/*
 * gdn_oracle_conv1d_silu_backward -- the gradient of the front end (conv1d,
 * SiLU, per-head L2 norm of q and k) given dL/dq, dL/dk [T, Hqk, d] and dL/dv
 * [T, Hv, d].  Reverse mode through each step of the forward:
 *   out = a / n with n = sqrt(sum a^2 + 1e-6) (q, k heads; out = a for v):
 *       da = (dout - out <dout, out>) / n;
 *   a = silu(y) = y sigma(y):  dy = da sigma(y) (1 + y (1 - sigma(y)));
 *   y[t, c] = sum_j w[c, j] x~[t - 3 + j, c]:  dx~ += w dy, dw += dy x~,
 * where x~ before a sequence's first token is its conv_state history (or
 * zero).  Outputs (all overwritten): dx [T, Ctot], dw [Ctot, 4] (summed over
 * every token of every sequence), dconv_state [n_seq, Ctot, 3] or NULL.
 * Parallel over heads only, so each sum has a fixed order.
 */
int gdn_oracle_conv1d_silu_backward(const double* x, const double* w, const int32_t* cu_seqlens, int32_t n_seq,
                                    int64_t T, int32_t Hqk, int32_t Hv, int32_t d, const double* conv_state_in,
                                    const double* dq, const double* dk, const double* dv, double* dx, double* dw,
                                    double* dconv_state, int threads) {
    if (Hqk <= 0 || Hv <= 0 || d <= 0 || n_seq <= 0 || T < 0) return -1;
    if (!cu_seqlens && n_seq != 1) return -1;
    set_threads(threads);
    const int64_t n_heads = 2 * Hqk + Hv, Ctot = n_heads * d;
    memset(dx, 0, sizeof(double) * T * Ctot);
    memset(dw, 0, sizeof(double) * Ctot * 4);
    if (dconv_state) memset(dconv_state, 0, sizeof(double) * n_seq * Ctot * 3);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t hh = 0; hh < n_heads; ++hh) {
        double* yv = malloc(sizeof(double) * d);
        double* av = malloc(sizeof(double) * d);
        for (int n = 0; n < n_seq; ++n) {
            const int64_t bos = cu_seqlens ? cu_seqlens[n] : 0, eos = cu_seqlens ? cu_seqlens[n + 1] : T;
            for (int64_t t = bos; t < eos; ++t) {
                double ss = 0.0;
                for (int e = 0; e < d; ++e) {
                    const int64_t c = hh * d + e;
                    double acc = 0.0;
                    for (int j = 0; j < 4; ++j)
                        acc += w[c * 4 + j] * gdn_oracle_front_x(x, conv_state_in, Ctot, n, bos, t - 3 + j, c);
                    yv[e] = acc;
                    av[e] = acc / (1.0 + exp(-acc));
                    ss += av[e] * av[e];
                }
                const double* dout = hh < Hqk ? dq + (t * Hqk + hh) * d
                                   : hh < 2 * Hqk ? dk + (t * Hqk + (hh - Hqk)) * d
                                                  : dv + (t * Hv + (hh - 2 * Hqk)) * d;
                const int normed = hh < 2 * Hqk;
                const double nrm = normed ? sqrt(ss + 1e-6) : 1.0;
                double dot = 0.0;
                if (normed)
                    for (int e = 0; e < d; ++e) dot += dout[e] * av[e] / nrm;
                for (int e = 0; e < d; ++e) {
                    const int64_t c = hh * d + e;
                    const double da = normed ? (dout[e] - av[e] / nrm * dot) / nrm : dout[e];
                    const double sg = 1.0 / (1.0 + exp(-yv[e]));
                    const double dy = da * sg * (1.0 + yv[e] * (1.0 - sg));
                    for (int j = 0; j < 4; ++j) {
                        const int64_t tau = t - 3 + j;
                        dw[c * 4 + j] += dy * gdn_oracle_front_x(x, conv_state_in, Ctot, n, bos, tau, c);
                        if (tau >= bos) dx[tau * Ctot + c] += w[c * 4 + j] * dy;
                        else if (dconv_state) dconv_state[((int64_t)n * Ctot + c) * 3 + (3 - (bos - tau))] += w[c * 4 + j] * dy;
                    }
                }
            }
        }
        free(yv);
        free(av);
    }
    return 0;
}

/*
 * gdn_oracle_gated_norm_backward -- the gradient of gdn_oracle_gated_norm
 * (y = w[l] * o * r * silu(z), r = 1 / sqrt(mean(o^2) + eps), l = t % layers)
 * given dL/dy.  With u = w g dy (g = silu(z)):
 *     do = r u - (r^3 / d) o <o, u>,
 *     dz = dy w r o silu'(z),  silu'(z) = sigma(z) (1 + z (1 - sigma(z))),
 *     dw[l] = sum over the rows of layer l of dy r o g.
 * Rows are summed in order (t, then h).  Outputs overwritten.
 */
int gdn_oracle_gated_norm_backward(const double* o, const double* z, const double* w, int64_t T, int Hv, int d,
                                   int layers, double eps, const double* dy, double* d_o, double* dz, double* dw) {
    if (T < 0 || Hv <= 0 || d <= 0 || layers <= 0 || !(eps >= 0.0)) return -1;
    memset(dw, 0, sizeof(double) * (size_t)layers * d);
    for (int64_t t = 0; t < T; ++t) {
        const int l = (int)(t % layers);
        const double* wl = w + (int64_t)l * d;
        for (int h = 0; h < Hv; ++h) {
            const int64_t row = (t * Hv + h) * (int64_t)d;
            double ss = 0.0, ou = 0.0;
            for (int e = 0; e < d; ++e) ss += o[row + e] * o[row + e];
            const double r = 1.0 / sqrt(ss / d + eps);
            for (int e = 0; e < d; ++e) {
                const double sg = 1.0 / (1.0 + exp(-z[row + e]));
                ou += o[row + e] * wl[e] * z[row + e] * sg * dy[row + e];
            }
            for (int e = 0; e < d; ++e) {
                const double sg = 1.0 / (1.0 + exp(-z[row + e]));
                const double g = z[row + e] * sg;
                const double u = wl[e] * g * dy[row + e];
                d_o[row + e] = r * u - r * r * r / d * o[row + e] * ou;
                dz[row + e] = dy[row + e] * wl[e] * r * o[row + e] * sg * (1.0 + z[row + e] * (1.0 - sg));
                dw[(int64_t)l * d + e] += dy[row + e] * r * o[row + e] * g;
            }
        }
    }
    return 0;
}
