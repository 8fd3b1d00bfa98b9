/*
 * moe_oracle.c -- plain, slow, fp64 CPU oracle of the Grok-1 mixture-of-experts
 * feed-forward layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
 * benchmark's CPU-baseline / reference leg may load or call this library.  The
 * product path (the CUDA library and its binding) never does, and the two share
 * no code, header, table or helper.
 *
 * What it computes, and the passage each step follows:
 *
 *   routing   "Grok-1 Admin & Architecture Guide", section 3 "The Model",
 *             "Mixture of Experts (MoELayer + Router)", steps 1-2: routing
 *             logits in fp32, softmax to per-token expert probabilities, top-2
 *             experts per token ("num_selected_experts" = 2 in "Configuration
 *             objects").
 *   experts   same section, step 3: each expert is a gated-GELU MLP,
 *             linear_1( gelu(linear(x)) * linear_v(x) ).
 *   weights   same guide, section 3 "Quantized weights": 8-bit values times
 *             scales, w.weight * w.scales, dequantised on the fly.
 *   combine   same section, step 4: expert outputs combined, each scaled by
 *             its routing gate.
 *   width     "llm-architectures-explained: Grok-1", table "Every architecture
 *             field", row ffns.moe.d_expert: ffn = int(8 * 6144) * 2 // 3
 *             rounded up to a multiple of 8 = 32768.
 *   blocks    "Grok-1 Admin & Architecture Guide", section 3 "Transformer stack
 *             and language model head" (pre/post RMSNorm around the MoE block,
 *             residual h += h_dense) and the grok-field-guide source-code map,
 *             fourth stop (moe(rms_norm(h)) added to h).
 *
 * Readings taken where the pages are silent:
 *   - the gate is the full 8-way softmax probability of the chosen expert; the
 *     two gates are not renormalised (the pages name no such step);
 *   - slot 0 holds the larger probability; equal logits go to the lower index;
 *   - "gelu" is the tanh approximation (the default of the JAX gelu the pages'
 *     framework uses); the erf form is available as gelu_kind = 1;
 *   - one scale per output channel, broadcast over the input dimension;
 *   - weights are stored [E, in, out] row-major (x @ W orientation);
 *   - no biases in the expert linears or the router;
 *   - the routing logits are the exact dot product rounded once to fp32 (the
 *     precision the pages fix for routing); the selection is taken on those
 *     fp32 logits; softmax and everything after it is evaluated in fp64.
 *
 * Everything else is IEEE fp64 in the plain summation order of the definition.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_API __attribute__((visibility("default")))

enum { OR_OK = 0, OR_EINVAL = -1, OR_ENOMEM = -2 };

/* ---- number formats ------------------------------------------------------ */

/* bf16 -> fp64: the 16 stored bits are the top half of an fp32. Exact. */
static double bf16_to_f64(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* fp64 -> nearest bf16 value (round half to even, 8 significant bits), kept
 * as an fp64.  Used where the method stores a tensor in bf16 (the stacked
 * workload's residual stream and MoE input). */
ORACLE_API double moe_oracle_round_bf16(double x)
{
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    frexp(x, &e);                         /* x = m * 2^e with 0.5 <= |m| < 1 */
    double scale = ldexp(1.0, 8 - e);     /* |x| * scale in [128, 256)         */
    return nearbyint(x * scale) / scale;  /* default rounding mode: to even    */
}

ORACLE_API void moe_oracle_round_bf16_array(long n, const double *in, double *out)
{
    for (long i = 0; i < n; ++i) out[i] = moe_oracle_round_bf16(in[i]);
}

/* ---- GELU ---------------------------------------------------------------- */

/* tanh approximation: 0.5 a (1 + tanh( sqrt(2/pi) (a + 0.044715 a^3) )) */
static double gelu_tanh(double a)
{
    const double c = sqrt(2.0 / acos(-1.0));   /* sqrt(2/pi) */
    return 0.5 * a * (1.0 + tanh(c * (a + 0.044715 * a * a * a)));
}

/* exact form: a * Phi(a) = 0.5 a (1 + erf(a / sqrt 2)) */
static double gelu_erf(double a) { return 0.5 * a * (1.0 + erf(a / sqrt(2.0))); }

ORACLE_API double moe_oracle_gelu(double a, int gelu_kind)
{
    return gelu_kind == 1 ? gelu_erf(a) : gelu_tanh(a);
}

/* ---- shape rule ---------------------------------------------------------- */

/* ffn_size(emb, widening) = int(widening * emb) * 2 // 3, rounded up to a
 * multiple of 8 ("llm-architectures-explained: Grok-1", ffns.moe.d_expert; the
 * admin guide's note under "Mixture of Experts"). */
ORACLE_API long moe_oracle_ffn_size(long emb, double widening)
{
    long f = ((long)(widening * (double)emb)) * 2 / 3;
    return ((f + 7) / 8) * 8;
}

/* ---- router: logits, softmax, top-2 ------------------------------------- */

/*
 * For each token t:
 *   L[e]  = fp32( sum_i x[t,i] * router_w[i,e] ) + bias[e]   (exact sum, one rounding)
 *   p     = softmax(L) in fp64
 *   e0    = argmax_e L[e], e1 = argmax_{e != e0} L[e], equal logits -> lower e
 *   gate  = p[e0], p[e1]
 * x is bf16 [T,d]; router_w fp32 [d,E] row-major; bias fp32 [E] or NULL.
 * Outputs (any may be NULL): logits fp32 [T,E], probs fp64 [T,E],
 * idx int32 [T,2], gate fp64 [T,2].
 */
ORACLE_API int moe_oracle_route(int T, int d, int E, const uint16_t *x, const float *router_w,
                                const float *bias, float *logits, double *probs, int32_t *idx,
                                double *gate)
{
    if (T < 0 || d <= 0 || E < 2 || E > 64 || !x || !router_w) return OR_EINVAL;
    double acc[64];
    float L[64];
    double p[64];
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) acc[e] = 0.0;
        for (int i = 0; i < d; ++i) {
            double xi = bf16_to_f64(x[(size_t)t * d + i]);
            for (int e = 0; e < E; ++e) acc[e] += xi * (double)router_w[(size_t)i * E + e];
        }
        for (int e = 0; e < E; ++e) {
            float l = (float)acc[e];                 /* routing logits in fp32 */
            if (bias) l = l + bias[e];               /* fp32 add of the test bias */
            L[e] = l;
        }
        double m = L[0];
        for (int e = 1; e < E; ++e)
            if (L[e] > m) m = L[e];
        double s = 0.0;
        for (int e = 0; e < E; ++e) {
            p[e] = exp((double)L[e] - m);
            s += p[e];
        }
        for (int e = 0; e < E; ++e) p[e] /= s;
        int e0 = 0;
        for (int e = 1; e < E; ++e)
            if (L[e] > L[e0]) e0 = e;
        int e1 = (e0 == 0) ? 1 : 0;
        for (int e = 0; e < E; ++e)
            if (e != e0 && L[e] > L[e1]) e1 = e;
        if (logits)
            for (int e = 0; e < E; ++e) logits[(size_t)t * E + e] = L[e];
        if (probs)
            for (int e = 0; e < E; ++e) probs[(size_t)t * E + e] = p[e];
        if (idx) {
            idx[2 * t] = e0;
            idx[2 * t + 1] = e1;
        }
        if (gate) {
            gate[2 * t] = p[e0];
            gate[2 * t + 1] = p[e1];
        }
    }
    return OR_OK;
}

/* ---- dispatch: group routes by expert ----------------------------------- */

/*
 * Route (t, j) is token t's j-th pick, id r = 2t + j.  counts[e] = number of
 * routes to e; offsets = exclusive prefix sum (E+1 entries); within expert e the
 * routes are ordered by ascending token index (a token reaches an expert at most
 * once): perm[offsets[e] + rank] = r.
 */
ORACLE_API int moe_oracle_dispatch(int T, int E, const int32_t *idx, int32_t *counts,
                                   int32_t *offsets, int32_t *perm)
{
    if (T < 0 || E < 1 || (T > 0 && !idx) || !offsets) return OR_EINVAL;
    int32_t *cnt = calloc((size_t)E, sizeof *cnt);
    if (!cnt) return OR_ENOMEM;
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < 2; ++j) {
            int e = idx[2 * t + j];
            if (e == -1) continue;   /* a padding token's route: not dispatched */
            if (e < 0 || e >= E) { free(cnt); return OR_EINVAL; }
            cnt[e]++;
        }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + cnt[e];
    if (counts) memcpy(counts, cnt, (size_t)E * sizeof *cnt);
    if (perm) {
        memset(cnt, 0, (size_t)E * sizeof *cnt);
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < 2; ++j) {
                int e = idx[2 * t + j];
                if (e >= 0) perm[offsets[e] + cnt[e]++] = 2 * t + j;
            }
    }
    free(cnt);
    return OR_OK;
}

/* ---- one expert's gated-GELU FFN ---------------------------------------- */

typedef struct {
    int d, F, gelu_kind;
    const double *xt;                 /* [d] token, fp64                      */
    const int8_t *wl, *wv, *w1;       /* [d,F], [d,F], [F,d] int8 of expert e */
    const uint16_t *sl, *sv, *s1;     /* bf16 scales: [F], [F], [d] per output channel, or
                                         [d/kb,F], [d/kb,F], [F/kb,d] per block of kb inputs */
    int kb;                           /* scale block along the input dimension; 0: none */
    double *h;                        /* [F] gelu(linear) * linear_v           */
    double *y;                        /* [d] linear_1(h)                      */
    int lo, hi;                       /* this worker's output column range     */
} ffn_job;

/* linear and linear_v over output columns f in [lo, hi):
 *   a[f] = sum_i x[i] * (Wl[i,f] * sl[f]),  v[f] = sum_i x[i] * (Wv[i,f] * sv[f])
 *   h[f] = gelu(a[f]) * v[f]
 * (with block scales, sl[i / kb, f] and sv[i / kb, f]: "Grok-1 Admin & Architecture
 * Guide", section 3 "Quantized weights", per-block dequant scales).
 * The dequantised weight Wl[i,f]*sl[f] is formed first (exact in fp64: an
 * 8-bit integer times an 8-bit-significand scale), then the dot product. */
static void *ffn_up_worker(void *arg)
{
    ffn_job *j = arg;
    int n = j->hi - j->lo;
    if (n <= 0) return NULL;
    double *restrict a = calloc((size_t)n, sizeof(double));
    double *restrict v = calloc((size_t)n, sizeof(double));
    double *restrict s_l = malloc((size_t)n * sizeof(double));
    double *restrict s_v = malloc((size_t)n * sizeof(double));
    if (!a || !v || !s_l || !s_v) { free(a); free(v); free(s_l); free(s_v); return (void *)1; }
    for (int i = 0; i < j->d; ++i) {
        if (i == 0 || (j->kb && i % j->kb == 0)) {   /* the scale row of this input */
            const size_t row = j->kb ? (size_t)(i / j->kb) * j->F : 0;
            for (int f = 0; f < n; ++f) {
                s_l[f] = bf16_to_f64(j->sl[row + j->lo + f]);
                s_v[f] = bf16_to_f64(j->sv[row + j->lo + f]);
            }
        }
        const double xi = j->xt[i];
        const int8_t *restrict rl = j->wl + (size_t)i * j->F + j->lo;
        const int8_t *restrict rv = j->wv + (size_t)i * j->F + j->lo;
        for (int f = 0; f < n; ++f) {
            a[f] += xi * ((double)rl[f] * s_l[f]);
            v[f] += xi * ((double)rv[f] * s_v[f]);
        }
    }
    for (int f = 0; f < n; ++f) {
        double g = j->gelu_kind == 1 ? gelu_erf(a[f]) : gelu_tanh(a[f]);
        j->h[j->lo + f] = g * v[f];
    }
    free(a); free(v); free(s_l); free(s_v);
    return NULL;
}

/* linear_1 over output columns c in [lo, hi):  y[c] = sum_f h[f] * (W1[f,c] * s1[c])
 * (with block scales, s1[f / kb, c]) */
static void *ffn_down_worker(void *arg)
{
    ffn_job *j = arg;
    int n = j->hi - j->lo;
    if (n <= 0) return NULL;
    double *restrict acc = calloc((size_t)n, sizeof(double));
    double *restrict s = malloc((size_t)n * sizeof(double));
    if (!acc || !s) { free(acc); free(s); return (void *)1; }
    for (int f = 0; f < j->F; ++f) {
        if (f == 0 || (j->kb && f % j->kb == 0)) {
            const size_t row = j->kb ? (size_t)(f / j->kb) * j->d : 0;
            for (int c = 0; c < n; ++c) s[c] = bf16_to_f64(j->s1[row + j->lo + c]);
        }
        const double hf = j->h[f];
        const int8_t *restrict r = j->w1 + (size_t)f * j->d + j->lo;
        for (int c = 0; c < n; ++c) acc[c] += hf * ((double)r[c] * s[c]);
    }
    for (int c = 0; c < n; ++c) j->y[j->lo + c] = acc[c];
    free(acc); free(s);
    return NULL;
}

static int default_threads(int n)
{
    if (n > 0) return n;
    long c = sysconf(_SC_NPROCESSORS_ONLN);
    return c > 0 ? (int)c : 1;
}

static int run_split(void *(*fn)(void *), ffn_job *base, int ncols, int nthreads)
{
    if (nthreads > ncols / 16) nthreads = ncols / 16 > 0 ? ncols / 16 : 1;
    pthread_t *th = malloc((size_t)nthreads * sizeof *th);
    ffn_job *jobs = malloc((size_t)nthreads * sizeof *jobs);
    if (!th || !jobs) { free(th); free(jobs); return OR_ENOMEM; }
    int rc = OR_OK;
    for (int w = 0; w < nthreads; ++w) {
        jobs[w] = *base;
        jobs[w].lo = (int)((long)ncols * w / nthreads);
        jobs[w].hi = (int)((long)ncols * (w + 1) / nthreads);
        if (pthread_create(&th[w], NULL, fn, &jobs[w]) != 0) {
            fn(&jobs[w]);   /* run inline if no thread could be started */
            th[w] = 0;
        }
    }
    for (int w = 0; w < nthreads; ++w) {
        void *ret = NULL;
        if (th[w]) pthread_join(th[w], &ret);
        if (ret) rc = OR_ENOMEM;
    }
    free(th); free(jobs);
    return rc;
}

/*
 * One expert e on one token: y = linear_1( gelu(linear(x)) * linear_v(x) ).
 * xt fp64 [d]; wl, wv int8 [d,F]; w1 int8 [F,d]; scales bf16, per output channel
 * (kb = 0: sl, sv [F], s1 [d]) or per block of kb inputs (sl, sv [d/kb,F], s1 [F/kb,d]),
 * all already offset to expert e; y fp64 [d].  h (fp64 [F]) may be NULL.
 */
ORACLE_API int moe_oracle_expert_ffn(int d, int F, const double *xt, const int8_t *wl,
                                     const uint16_t *sl, const int8_t *wv, const uint16_t *sv,
                                     const int8_t *w1, const uint16_t *s1, double *h_out,
                                     double *y, int nthreads, int gelu_kind, int kb)
{
    if (d <= 0 || F <= 0 || !xt || !wl || !sl || !wv || !sv || !w1 || !s1 || !y) return OR_EINVAL;
    if (kb < 0 || (kb && (d % kb || F % kb))) return OR_EINVAL;
    double *h = h_out ? h_out : malloc((size_t)F * sizeof(double));
    if (!h) return OR_ENOMEM;
    ffn_job base = {d, F, gelu_kind, xt, wl, wv, w1, sl, sv, s1, kb, h, y, 0, 0};
    nthreads = default_threads(nthreads);
    int rc = run_split(ffn_up_worker, &base, F, nthreads);
    if (rc == OR_OK) rc = run_split(ffn_down_worker, &base, d, nthreads);
    if (!h_out) free(h);
    return rc;
}

/* ---- the layer ----------------------------------------------------------- */

/*
 * out[s,:] = gate0 * FFN_{e0}(x[t]) + gate1 * FFN_{e1}(x[t]) for each selected
 * token t = tokens[s] (s = 0..n_sel-1; tokens == NULL means every token).
 * The experts and gates come from moe_oracle_route on that token, unless
 * forced_idx (int32 [n_sel,2], may be NULL) names the two experts to use; the
 * gates are then those experts' softmax probabilities.
 * Weights: wl, wv int8 [E,d,F], w1 int8 [E,F,d]; sl, sv bf16 [E,F]; s1 bf16 [E,d].
 * kb: scale block along the input dimension (0: one scale per output channel), as
 * in moe_oracle_expert_ffn.
 * mask (uint8 [T], may be NULL = every token real): a token t with mask[t] == 0 is
 * padding, the padding_mask of the MoE call in the grok-field-guide source-code map,
 * fourth stop (moe(rms_norm(h), padding_mask)); it is routed nowhere: out row 0,
 * experts -1 and gates 0.
 * Outputs: out fp64 [n_sel,d]; idx int32 [n_sel,2] and gate fp64 [n_sel,2] (may be NULL).
 */
ORACLE_API int moe_oracle_forward(int T, int d, int F, int E, const uint16_t *x,
                                  const float *router_w, const float *bias, const int8_t *wl,
                                  const uint16_t *sl, const int8_t *wv, const uint16_t *sv,
                                  const int8_t *w1, const uint16_t *s1, const int32_t *tokens,
                                  int n_sel, const int32_t *forced_idx, const uint8_t *mask, double *out,
                                  int32_t *idx, double *gate, int nthreads, int gelu_kind, int kb)
{
    if (T < 0 || d <= 0 || F <= 0 || E < 2 || E > 64 || !x || !router_w || !wl || !sl || !wv ||
        !sv || !w1 || !s1 || !out)
        return OR_EINVAL;
    if (!tokens) n_sel = T;
    double *xt = malloc((size_t)d * sizeof(double));
    double *y = malloc((size_t)d * sizeof(double));
    double probs[64];
    if (!xt || !y) { free(xt); free(y); return OR_ENOMEM; }
    int rc = OR_OK;
    for (int s = 0; s < n_sel && rc == OR_OK; ++s) {
        int t = tokens ? tokens[s] : s;
        if (t < 0 || t >= T) { rc = OR_EINVAL; break; }
        const uint16_t *xrow = x + (size_t)t * d;
        if (mask && !mask[t]) {
            for (int i = 0; i < d; ++i) out[(size_t)s * d + i] = 0.0;
            if (idx) { idx[2 * s] = -1; idx[2 * s + 1] = -1; }
            if (gate) { gate[2 * s] = 0.0; gate[2 * s + 1] = 0.0; }
            continue;
        }
        int32_t sel[2];
        rc = moe_oracle_route(1, d, E, xrow, router_w, bias, NULL, probs, sel, NULL);
        if (rc != OR_OK) break;
        if (forced_idx) {
            sel[0] = forced_idx[2 * s];
            sel[1] = forced_idx[2 * s + 1];
            if (sel[0] < 0 || sel[0] >= E || sel[1] < 0 || sel[1] >= E) { rc = OR_EINVAL; break; }
        }
        for (int i = 0; i < d; ++i) xt[i] = bf16_to_f64(xrow[i]);
        double *o = out + (size_t)s * d;
        for (int i = 0; i < d; ++i) o[i] = 0.0;
        for (int j = 0; j < 2 && rc == OR_OK; ++j) {
            int e = sel[j];
            /* per expert: F (or d/kb * F) scales of linear / linear_v, d (or F/kb * d) of linear_1 */
            const size_t up_s = kb ? (size_t)(d / kb) * F : (size_t)F;
            const size_t dn_s = kb ? (size_t)(F / kb) * d : (size_t)d;
            rc = moe_oracle_expert_ffn(d, F, xt, wl + (size_t)e * d * F, sl + (size_t)e * up_s,
                                       wv + (size_t)e * d * F, sv + (size_t)e * up_s,
                                       w1 + (size_t)e * F * d, s1 + (size_t)e * dn_s, NULL, y,
                                       nthreads, gelu_kind, kb);
            /* combine in route order: slot 0 first, then slot 1 */
            for (int i = 0; i < d; ++i) o[i] += probs[e] * y[i];
        }
        if (idx) { idx[2 * s] = sel[0]; idx[2 * s + 1] = sel[1]; }
        if (gate) { gate[2 * s] = probs[sel[0]]; gate[2 * s + 1] = probs[sel[1]]; }
    }
    free(xt); free(y);
    return rc;
}

/* ---- RMSNorm (stacked workload) ----------------------------------------- */

/* out[t,i] = z[t,i] / sqrt( mean_i z[t,i]^2 + eps ) * gamma[i], all fp64.
 * gamma is bf16 [d] (NULL = all ones). */
ORACLE_API int moe_oracle_rmsnorm(int T, int d, const double *z, const uint16_t *gamma, double eps,
                                  double *out)
{
    if (T < 0 || d <= 0 || !z || !out) return OR_EINVAL;
    for (int t = 0; t < T; ++t) {
        const double *zr = z + (size_t)t * d;
        double ss = 0.0;
        for (int i = 0; i < d; ++i) ss += zr[i] * zr[i];
        double r = 1.0 / sqrt(ss / d + eps);
        for (int i = 0; i < d; ++i)
            out[(size_t)t * d + i] = zr[i] * r * (gamma ? bf16_to_f64(gamma[i]) : 1.0);
    }
    return OR_OK;
}
