/*
 * CPU oracle for the AdaFuse fused gated multi-LoRA path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code, header, table or helper with the CUDA library.
 *
 * Method: "AdaFuse: Accelerating Dynamic Adapter Inference via Token-Level
 * Pre-Gating and Fused Kernel Optimization" (gist.science summaries, pt and ja).
 *   - section 2.A / 2.1 (token-level pre-gating): one top-2 router at the first
 *     adapted layer decides, once per token, which LoRA experts are active for
 *     every layer that follows;
 *   - section 2.B / 2.2 (SGMM): the activated adapters' down (A) and up (B)
 *     projections are concatenated and fused into the backbone weights,
 *     W' = W + sum_s g_s B_s A_s, for every targeted linear;
 *   - section 2.B (switching): the previous token's fusion is undone and the
 *     current one applied;
 *   - the segmented-gather form for mixed batches,
 *     y = x W^T + sum_s g_s (x A_s^T) B_s^T.
 * The pages give no formulas, scaling, gate normalisation or precision; the
 * readings taken here are: LoRA scale 1 (any alpha/r is folded into B), gates
 * are the full softmax probabilities of the selected experts (optional
 * renormalisation), selection on the logits with ties to the lower index,
 * W stored [d_out, d_in] row-major, A_e [r, d_in], B_e [d_out, r].
 *
 * Precision.  Merge, apply and gates are computed in fp64 from the exact bf16
 * (or fp32) inputs and rounded once, to bf16 with round-to-nearest-even.  The
 * router logits decide an integer (the top-k), so they are computed in fp32 in
 * the plainest order: the products x_j * w_j, each rounded to fp32, added in
 * ascending j (no fused multiply-add; build with -ffp-contract=off).
 *
 * Every function here is pinned by a test against something other than itself
 * (closed forms, brute force, library routines); see tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <fenv.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ bf16 */

/* bf16 bit pattern -> its exact value. */
double orc_bf16_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a double to the nearest bf16, ties to even, in one step (no detour
 * through fp32, which could round twice).  bf16 has an 8-bit significand and
 * fp32's exponent range: quantum 2^(e-7) for |v| in [2^e, 2^(e+1)), e >= -126,
 * and 2^-133 below 2^-126 (subnormals). */
uint16_t orc_bf16_from_double(double v)
{
    if (isnan(v)) return 0x7FC0;
    double a = fabs(v);
    double q;
    if (a < ldexp(1.0, -126)) {
        q = ldexp(1.0, -133);
    } else {
        int e;
        frexp(a, &e);          /* a = m * 2^e, m in [0.5, 1) -> a in [2^(e-1), 2^e) */
        q = ldexp(1.0, (e - 1) - 7);
    }
    double n = nearbyint(a / q);           /* exact scaling; ties to even */
    double rv = n * q;
    float f;
    if (rv >= ldexp(1.0, 128)) {
        f = INFINITY;
    } else {
        f = (float)rv;                     /* exact: rv has <= 8 significant bits */
    }
    if (signbit(v)) f = -f;              /* the sign of a zero result is the operand's */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

void orc_bf16_from_double_array(const double* v, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_from_double(v[i]);
}

/* ---------------------------------------------------------------- router */

/* Router logits z[t,e] = sum_j x[t,j] * W_r[e,j] (+ b_r[e]), fp32, products
 * rounded to fp32 and summed in ascending j; the bias, when given, is added
 * after the sum.  (Token-level pre-gating: section 2.A / 2.1.) */
void orc_router_logits(const uint16_t* x, int64_t T, int32_t H, int64_t ldx,
                       const float* Wr, const float* br, int32_t E, float* z)
{
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t e = 0; e < E; ++e) {
            float acc = 0.0f;
            for (int32_t j = 0; j < H; ++j) {
                float xj = (float)orc_bf16_to_double(x[t * ldx + j]);
                float p = xj * Wr[(int64_t)e * H + j];
                acc = acc + p;
            }
            if (br) acc = acc + br[e];
            z[t * E + e] = acc;
        }
    }
}

/* Sequence-level routing input: the mean of the T rows, fp32, summed in
 * ascending t and divided by T ("the whole sentence or its first token",
 * section "O essencial" / 1: Guardião na Entrada). */
void orc_pool_mean(const uint16_t* x, int64_t T, int32_t H, int64_t ldx, float* xbar)
{
    for (int32_t j = 0; j < H; ++j) {
        float acc = 0.0f;
        for (int64_t t = 0; t < T; ++t) acc = acc + (float)orc_bf16_to_double(x[t * ldx + j]);
        xbar[j] = acc / (float)T;
    }
}

/* Logits of one fp32 input row (used with the pooled row). */
void orc_router_logits_f32(const float* xrow, int32_t H, const float* Wr, const float* br,
                           int32_t E, float* z)
{
    for (int32_t e = 0; e < E; ++e) {
        float acc = 0.0f;
        for (int32_t j = 0; j < H; ++j) {
            float p = xrow[j] * Wr[(int64_t)e * H + j];
            acc = acc + p;
        }
        if (br) acc = acc + br[e];
        z[e] = acc;
    }
}

/* Is expert a ranked before expert b?  Larger logit first; equal logits go to
 * the lower index; a NaN logit ranks as -infinity. */
static int ranks_before(const float* z, int a, int b)
{
    float za = z[a], zb = z[b];
    int na = isnan(za), nb = isnan(zb);
    if (na && nb) return a < b;
    if (na) return 0;
    if (nb) return 1;
    if (za > zb) return 1;
    if (za < zb) return 0;
    return a < b;
}

/* Top-k selection and gates for each token: idx = the k best experts in rank
 * order; gate = their softmax probabilities over all E experts, computed in
 * fp64 from the fp32 logits with the maximum subtracted; with renorm != 0 the
 * k gates are divided by their sum.  NaN logits take no probability mass. */
void orc_topk_softmax(const float* z, int64_t T, int32_t E, int32_t k, int32_t renorm,
                      int32_t* idx, double* gate)
{
    for (int64_t t = 0; t < T; ++t) {
        const float* zt = z + t * E;
        /* selection: repeatedly take the best not yet taken */
        int taken[64] = {0};
        for (int32_t s = 0; s < k; ++s) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || ranks_before(zt, e, best)) best = e;
            }
            taken[best] = 1;
            idx[t * k + s] = best;
        }
        /* softmax over all experts */
        double m = -INFINITY;
        for (int e = 0; e < E; ++e) if (!isnan(zt[e]) && (double)zt[e] > m) m = (double)zt[e];
        double sum = 0.0;
        for (int e = 0; e < E; ++e) if (!isnan(zt[e])) sum += exp((double)zt[e] - m);
        double gs = 0.0;
        for (int32_t s = 0; s < k; ++s) {
            float zi = zt[idx[t * k + s]];
            double p = isnan(zi) ? 0.0 : exp((double)zi - m) / sum;
            gate[t * k + s] = p;
            gs += p;
        }
        if (renorm) for (int32_t s = 0; s < k; ++s) gate[t * k + s] /= gs;
    }
}

/* ----------------------------------------------------------------- merge */

/* All-layer fused merge, one linear (section 2.B / 2.2, SGMM):
 *   W'[o,i] = bf16( W[o,i] + sum_{s<ns} g_s * sum_{j<r} B_{e_s}[o,j] * A_{e_s}[j,i] )
 * for rows o in [row0, row1).  A slot whose expert index lies outside [0, E)
 * is skipped.  Switching (undo the previous selection, apply the current one)
 * is this same function over the concatenated slot list with the previous
 * gates negated.  W and W_out are [d_out, d_in] row-major; A is
 * A[e*a_es + j*d_in + i], B is B[e*b_es + o*r + j]. */
void orc_merge_linear(const uint16_t* W, uint16_t* Wout,
                      const uint16_t* A, const uint16_t* B,
                      int32_t d_out, int32_t d_in, int32_t E, int32_t r,
                      int64_t a_es, int64_t b_es,
                      const int32_t* eidx, const double* g, int32_t ns,
                      int64_t row0, int64_t row1, int32_t nthreads)
{
    (void)d_out;
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(static) num_threads(nthreads)
#endif
    for (int64_t o = row0; o < row1; ++o) {
        for (int64_t i = 0; i < d_in; ++i) {
            double acc = orc_bf16_to_double(W[o * d_in + i]);
            for (int32_t s = 0; s < ns; ++s) {
                int32_t e = eidx[s];
                if (e < 0 || e >= E) continue;
                double d = 0.0;
                for (int32_t j = 0; j < r; ++j)
                    d += orc_bf16_to_double(B[e * b_es + o * r + j]) *
                         orc_bf16_to_double(A[e * a_es + (int64_t)j * d_in + i]);
                acc += g[s] * d;
            }
            Wout[(o - row0) * d_in + i] = orc_bf16_from_double(acc);
        }
    }
}

/* ----------------------------------------------------------------- apply */

/* Unmerged mixed-batch apply for one linear (segmented-gather form):
 *   u[t,s,j] = sum_i A_{e_ts}[j,i] * x[t,i]
 *   y[t,o]   = sum_i x[t,i] W[o,i] + sum_s g[t,s] sum_j B_{e_ts}[o,j] u[t,s,j]
 * for tokens t in [t0, t1).  Slots with an index outside [0, E) are skipped.
 * x is [T, d_in] row-major; the result rows [t1-t0, d_out] go to y16 rounded
 * once to bf16 (orc_apply_linear), or to y64 unrounded (orc_apply_linear_f64:
 * the partial output of a row-parallel shard, whose sum over the shards is
 * rounded once after the all-reduce). */
static void apply_rows(const uint16_t* x, const uint16_t* W,
                       const uint16_t* A, const uint16_t* B,
                       int32_t d_out, int32_t d_in, int32_t E, int32_t r,
                       int64_t a_es, int64_t b_es,
                       const int32_t* idx, const double* gate, int32_t k,
                       int64_t t0, int64_t t1, uint16_t* y16, double* y64, int32_t nthreads)
{
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(static) num_threads(nthreads)
#endif
    for (int64_t t = t0; t < t1; ++t) {
        double* u = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1) * (size_t)(r > 0 ? r : 1));
        for (int32_t s = 0; s < k; ++s) {
            int32_t e = idx[t * k + s];
            for (int32_t j = 0; j < r; ++j) {
                double acc = 0.0;
                if (e >= 0 && e < E)
                    for (int64_t i = 0; i < d_in; ++i)
                        acc += orc_bf16_to_double(A[e * a_es + (int64_t)j * d_in + i]) *
                               orc_bf16_to_double(x[t * d_in + i]);
                u[s * r + j] = acc;
            }
        }
        for (int64_t o = 0; o < d_out; ++o) {
            double acc = 0.0;
            for (int64_t i = 0; i < d_in; ++i)
                acc += orc_bf16_to_double(x[t * d_in + i]) * orc_bf16_to_double(W[o * d_in + i]);
            for (int32_t s = 0; s < k; ++s) {
                int32_t e = idx[t * k + s];
                if (e < 0 || e >= E) continue;
                double d = 0.0;
                for (int32_t j = 0; j < r; ++j)
                    d += orc_bf16_to_double(B[e * b_es + o * r + j]) * u[s * r + j];
                acc += gate[t * k + s] * d;
            }
            if (y16) y16[(t - t0) * d_out + o] = orc_bf16_from_double(acc);
            if (y64) y64[(t - t0) * d_out + o] = acc;
        }
        free(u);
    }
}

void orc_apply_linear(const uint16_t* x, const uint16_t* W,
                      const uint16_t* A, const uint16_t* B,
                      int32_t d_out, int32_t d_in, int32_t E, int32_t r,
                      int64_t a_es, int64_t b_es,
                      const int32_t* idx, const double* gate, int32_t k,
                      int64_t t0, int64_t t1, uint16_t* y, int32_t nthreads)
{
    apply_rows(x, W, A, B, d_out, d_in, E, r, a_es, b_es, idx, gate, k, t0, t1, y, NULL, nthreads);
}

void orc_apply_linear_f64(const uint16_t* x, const uint16_t* W,
                          const uint16_t* A, const uint16_t* B,
                          int32_t d_out, int32_t d_in, int32_t E, int32_t r,
                          int64_t a_es, int64_t b_es,
                          const int32_t* idx, const double* gate, int32_t k,
                          int64_t t0, int64_t t1, double* y, int32_t nthreads)
{
    apply_rows(x, W, A, B, d_out, d_in, E, r, a_es, b_es, idx, gate, k, t0, t1, NULL, y, nthreads);
}

/* -------------------------------------------------------------- segments */

/* Segments of a mixed batch ("Segmented Gather"): the T*k (token, slot) pairs,
 * numbered p = t*k + s, stably sorted by their expert index.  offsets[e] ..
 * offsets[e+1] is expert e's segment of perm; pairs with an index outside
 * [0, E) are left out, and their count is returned. */
int32_t orc_segments(const int32_t* idx, int64_t T, int32_t k, int32_t E,
                     int32_t* offsets, int32_t* perm)
{
    int64_t P = T * k;
    int32_t bad = 0;
    for (int32_t e = 0; e <= E; ++e) offsets[e] = 0;
    for (int64_t p = 0; p < P; ++p) {
        int32_t e = idx[p];
        if (e < 0 || e >= E) { ++bad; continue; }
        offsets[e + 1] += 1;
    }
    for (int32_t e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
    int32_t* fill = (int32_t*)calloc((size_t)E + 1, sizeof(int32_t));
    for (int64_t p = 0; p < P; ++p) {
        int32_t e = idx[p];
        if (e < 0 || e >= E) continue;
        perm[offsets[e] + fill[e]] = (int32_t)p;
        fill[e] += 1;
    }
    free(fill);
    return bad;
}

int32_t orc_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
