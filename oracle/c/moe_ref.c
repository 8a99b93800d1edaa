/* Plain C oracle of the routed-expert MoE step (Route -> Union -> int4 SwiGLU -> combine).
 *
 * TEST INFRASTRUCTURE.  Only tests/ load this library (through oracle/cref.py);
 * the product path never calls it and shares no code with it.
 *
 * A second, independent statement of the layer that oracle/moe.py (numpy,
 * float64) states: same readings of the pages, different means.  Where the
 * numpy oracle leans on library steps (frexp/rint rounding, lexsort, argsort,
 * BLAS dot products) this file works from the definitions: number formats
 * decoded from their bit fields, bf16 rounding done on the bit pattern, top-k
 * as k selection passes, the union as a counting sort, every dot product a
 * sequential loop in double.  Compiled with -ffp-contract=off.
 *
 * The passages it follows (the pages give no formula; the numerics are the
 * layer statement this library implements):
 *   - per token and per layer, Route then Union then the expert matmuls
 *     (Colibri README, "Come funziona", "Il percorso di ogni token";
 *     getting-started guide, "トークンごとの処理経路", steps 1 and 2);
 *   - a batch reads each selected expert once (README, "Mai aspettare il disco
 *     due volte": batch-union);
 *   - routed experts in an int4 container (README, "L'idea"); the MTP head in
 *     int8 (README, "Decodifica speculativa, onestamente", "2. Scarica il
 *     modello"); the gs64 container (README, "2. Scarica il modello").
 *
 * Every exported function returns 0, or a negative value for arguments it
 * cannot take (COLI_REF_EARG) or a failed allocation (COLI_REF_ENOMEM).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define COLI_REF_EARG (-1)
#define COLI_REF_ENOMEM (-2)
#define ST_NONFINITE 1

/* ------------------------------------------------------------------------
 * number formats
 * ------------------------------------------------------------------------ */

/* IEEE binary16: sign, 5-bit exponent (bias 15), 10-bit fraction. */
static double fp16_value(uint16_t b)
{
    int neg = b >> 15, ex = (b >> 10) & 0x1f, fr = b & 0x3ff;
    double v;
    if (ex == 0)
        v = ldexp((double)fr, -24);                 /* fr/2^10 * 2^-14 */
    else if (ex == 31)
        v = fr ? NAN : INFINITY;
    else
        v = ldexp((double)(0x400 | fr), ex - 25);   /* (1 + fr/2^10) * 2^(ex-15) */
    return neg ? -v : v;
}

/* bfloat16: sign, 8-bit exponent (bias 127), 7-bit fraction. */
static double bf16_value(uint16_t b)
{
    int neg = b >> 15, ex = (b >> 7) & 0xff, fr = b & 0x7f;
    double v;
    if (ex == 0)
        v = ldexp((double)fr, -133);                /* fr/2^7 * 2^-126 */
    else if (ex == 255)
        v = fr ? NAN : INFINITY;
    else
        v = ldexp((double)(0x80 | fr), ex - 134);   /* (1 + fr/2^7) * 2^(ex-127) */
    return neg ? -v : v;
}

/* Nearest bfloat16 value of v (ties to even), straight from the double.
 * Normal range (|v| >= 2^-126): a bfloat16 keeps the top 7 of the double's 52
 * fraction bits; the 45 dropped bits decide the rounding, and a carry out of
 * the kept bits steps the exponent.  Below 2^-126 bfloat16 values are the
 * integer multiples of 2^-133; |v| * 2^133 < 128 is exact in double and is
 * rounded to an integer.  Results above the largest finite bfloat16
 * ((2 - 2^-7) * 2^127) become infinities. */
static double round_bf16(double v)
{
    if (isnan(v) || isinf(v) || v == 0.0)
        return v;
    uint64_t u;
    memcpy(&u, &v, 8);
    uint64_t sign = u & 0x8000000000000000ull, mag = u & 0x7fffffffffffffffull;
    int e = (int)(mag >> 52) - 1023;
    double r;
    if (e >= -126) {
        const uint64_t half = 1ull << 44, low = mag & ((1ull << 45) - 1);
        uint64_t keep = mag >> 45;
        if (low > half || (low == half && (keep & 1)))
            keep += 1;
        uint64_t m2 = keep << 45;
        memcpy(&r, &m2, 8);
        if (r > ldexp(255.0, 120))                  /* (2^8 - 1) * 2^120 */
            r = INFINITY;
    } else {
        double n = ldexp(fabs(v), 133);
        double fl = floor(n), fr = n - fl;
        if (fr > 0.5 || (fr == 0.5 && fmod(fl, 2.0) != 0.0))
            fl += 1.0;
        r = ldexp(fl, -133);
    }
    return sign ? -r : r;
}

/* Bit pattern of a double that holds a bfloat16 value (or an infinity/NaN):
 * the top half of its binary32 form, which is exact. */
static uint16_t bf16_bits_of(double v)
{
    float f = (float)v;
    uint32_t b;
    memcpy(&b, &f, 4);
    if (isnan(v))
        b = 0x7fc00000u | (b & 0x80000000u);
    return (uint16_t)(b >> 16);
}

/* ------------------------------------------------------------------------
 * the int4 / int8 group-quantised container
 * ------------------------------------------------------------------------ */

/* READING (the pages say only "int4 container"): row-major, K contiguous;
 * int4 element c of a row in byte c/2, low nibble when c is even, nibble n
 * read as n - 16 when n >= 8; int8 element c in byte c, two's complement;
 * one fp16 scale per `group` consecutive elements of a row. */
static int code_at(const uint8_t *row, int c, int bits)
{
    if (bits == 8)
        return (int)(int8_t)row[c];
    int byte = row[c >> 1];
    int nib = (c & 1) ? (byte >> 4) : (byte & 0xf);
    return nib >= 8 ? nib - 16 : nib;
}

static double weight_at(const uint8_t *q, const uint16_t *s, int K, int group, int bits, int r, int c)
{
    const uint8_t *row = q + (size_t)r * (size_t)(K * bits / 8);
    return (double)code_at(row, c, bits) * fp16_value(s[(size_t)r * (K / group) + c / group]);
}

static int container_ok(int K, int group, int bits)
{
    return (bits == 4 || bits == 8) && group > 0 && K > 0 && K % group == 0 && (bits == 8 || K % 2 == 0);
}

int coli_ref_dequant(int rows, int K, int group, int bits, const uint8_t *q, const uint16_t *s, double *out)
{
    if (rows < 0 || !container_ok(K, group, bits))
        return COLI_REF_EARG;
    for (int r = 0; r < rows; ++r)
        for (int c = 0; c < K; ++c)
            out[(size_t)r * K + c] = weight_at(q, s, K, group, bits, r, c);
    return 0;
}

int coli_ref_round_bf16(long n, const double *in, double *out, uint16_t *bits)
{
    for (long i = 0; i < n; ++i) {
        double r = round_bf16(in[i]);
        if (out)
            out[i] = r;
        if (bits)
            bits[i] = bf16_bits_of(r);
    }
    return 0;
}

int coli_ref_decode(long n, const uint16_t *in, int is_bf16, double *out)
{
    for (long i = 0; i < n; ++i)
        out[i] = is_bf16 ? bf16_value(in[i]) : fp16_value(in[i]);
    return 0;
}

/* ------------------------------------------------------------------------
 * router logits, bias, Route
 * ------------------------------------------------------------------------ */

/* l[t][e] = sum_h x[t][h] * W_r[e][h], summed in double in h order; l32 is
 * that sum rounded once to binary32.  x is bf16 [T][H], W_r fp32 [E][H]. */
int coli_ref_router_logits(int T, int E, int H, const uint16_t *x, const float *wr, double *l64, float *l32)
{
    if (T < 0 || E <= 0 || H <= 0)
        return COLI_REF_EARG;
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int h = 0; h < H; ++h)
                acc += bf16_value(x[(size_t)t * H + h]) * (double)wr[(size_t)e * H + h];
            if (l64)
                l64[(size_t)t * E + e] = acc;
            l32[(size_t)t * E + e] = (float)acc;
        }
    return 0;
}

/* Top-k per token under the order (logit descending, expert index
 * ascending); a NaN logit ranks as -inf and -0.0 ties +0.0.  Slot j holds the
 * j-th pick.  Weights w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0) over the k
 * picks (the softmax over all E restricted to the picks and renormalised).
 * flags[t] gets ST_NONFINITE when a logit is NaN or +inf or a pick is -inf.
 * READING: the per-expert bias, when given, is added to the logit in binary32
 * before both the selection and the weights. */
int coli_ref_route(int T, int E, int k, const float *l32, const float *bias, int32_t *ids, double *w,
                   int32_t *flags)
{
    if (T < 0 || E <= 0 || k <= 0 || k > E)
        return COLI_REF_EARG;
    double *key = malloc(sizeof(double) * (size_t)E);
    char *taken = malloc((size_t)E);
    if (!key || !taken) {
        free(key);
        free(taken);
        return COLI_REF_ENOMEM;
    }
    for (int t = 0; t < T; ++t) {
        int flag = 0;
        for (int e = 0; e < E; ++e) {
            float l = l32[(size_t)t * E + e];
            if (bias)
                l = l + bias[e];                    /* one binary32 addition */
            if (isnan(l) || (isinf(l) && l > 0))
                flag = ST_NONFINITE;
            key[e] = isnan(l) ? -INFINITY : (double)l;
            taken[e] = 0;
        }
        double sel[k > 0 ? k : 1];
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || key[e] > key[best]))
                    best = e;
            taken[best] = 1;
            ids[(size_t)t * k + j] = best;
            sel[j] = key[best];
            if (isinf(key[best]) && key[best] < 0)
                flag = ST_NONFINITE;
        }
        double sum = 0.0;
        for (int j = 0; j < k; ++j)
            sum += exp(sel[j] - sel[0]);
        for (int j = 0; j < k; ++j)
            w[(size_t)t * k + j] = exp(sel[j] - sel[0]) / sum;
        flags[t] = flag;
    }
    free(key);
    free(taken);
    return 0;
}

/* ------------------------------------------------------------------------
 * Union: the batch's selected experts, once each
 * ------------------------------------------------------------------------ */

/* Pairs p = t*k + j of the flattened ids [P].  A counting sort by expert:
 * unique[] = experts with at least one pair, ascending (*n_unique of them);
 * seg_off[u]..seg_off[u+1] = the positions in perm[] of unique[u]'s pairs,
 * in pair order; pair_pos[] = the inverse of perm[]. */
int coli_ref_union(int P, int E, const int32_t *flat, int32_t *unique, int32_t *n_unique, int32_t *seg_off,
                   int32_t *perm, int32_t *pair_pos)
{
    if (P < 0 || E <= 0)
        return COLI_REF_EARG;
    for (int p = 0; p < P; ++p)
        if (flat[p] < 0 || flat[p] >= E)
            return COLI_REF_EARG;
    int32_t *count = calloc((size_t)E, sizeof(int32_t)), *start = calloc((size_t)E, sizeof(int32_t));
    if (!count || !start) {
        free(count);
        free(start);
        return COLI_REF_ENOMEM;
    }
    for (int p = 0; p < P; ++p)
        count[flat[p]] += 1;
    int U = 0, pos = 0;
    seg_off[0] = 0;
    for (int e = 0; e < E; ++e) {
        start[e] = pos;
        if (count[e]) {
            unique[U] = e;
            pos += count[e];
            seg_off[++U] = pos;
        }
    }
    for (int p = 0; p < P; ++p) {
        int at = start[flat[p]]++;
        perm[at] = p;
        pair_pos[p] = at;
    }
    *n_unique = U;
    free(count);
    free(start);
    return 0;
}

/* ------------------------------------------------------------------------
 * expert SwiGLU FFN, combine, the layer
 * ------------------------------------------------------------------------ */

/* One pointer per expert and matrix: codes [I][H*bits/8] (gate, up) and
 * [H][I*bits/8] (down), scales [I][H/group] and [H][I/group]. */
typedef struct {
    int H, I, group, bits;
    const uint8_t *const *gate_q, *const *up_q, *const *down_q;
    const uint16_t *const *gate_s, *const *up_s, *const *down_s;
} Experts;

static int expert_present(const Experts *X, int e)
{
    return X->gate_q[e] && X->up_q[e] && X->down_q[e] && X->gate_s[e] && X->up_s[e] && X->down_s[e];
}

static double silu(double g) { return g / (1.0 + exp(-g)); }

/* y = W_down[e] . h, h_i = bf16( silu(W_gate[e]_i . x) * (W_up[e]_i . x) ).
 * READING: h is rounded to bf16 (the layer's tensor-core forms take a bf16
 * operand); every sum is double.  hbuf holds I doubles. */
static void expert_ffn(const Experts *X, int e, const double *x, double *hbuf, double *y)
{
    const int H = X->H, I = X->I, G = X->group, B = X->bits;
    const uint8_t *gq = X->gate_q[e], *uq = X->up_q[e], *dq = X->down_q[e];
    const uint16_t *gs = X->gate_s[e], *us = X->up_s[e], *ds = X->down_s[e];
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int c = 0; c < H; ++c) {
            g += weight_at(gq, gs, H, G, B, i, c) * x[c];
            u += weight_at(uq, us, H, G, B, i, c) * x[c];
        }
        hbuf[i] = round_bf16(silu(g) * u);
    }
    for (int r = 0; r < H; ++r) {
        double acc = 0.0;
        for (int i = 0; i < I; ++i)
            acc += weight_at(dq, ds, I, G, B, r, i) * hbuf[i];
        y[r] = acc;
    }
}

/* One layer: logits (or the given fp32 logits) -> Route -> Union -> FFN of
 * every unique expert over its tokens -> combine.
 *   out[t] = bf16( sum_j w[t][j] y_{ids[t][j]}(x_t) + sum_s y_{E+s}(x_t) + residual[t] )
 * with the sum in double (routed experts in ascending expert order, then the
 * shared experts, then the residual) and one rounding.  READING: S shared
 * experts (ids E..E+S-1) run on every token with weight 1, outside the
 * renormalisation.  Inputs: x bf16 [T][H]; router_w fp32 [E][H] or NULL when
 * logits_in fp32 [T][E] is given; bias fp32 [E] or NULL; residual bf16 [T][H]
 * or NULL.  Outputs (caller-owned): l64 [T][E] (NULL allowed), l32 [T][E],
 * ids [T][k], w [T][k], flags [T], acc [T][H] (NULL allowed), out bf16 bits
 * [T][H]. */
static int moe_layer(int T, int E, int k, int S, const Experts *X, const uint16_t *x, const float *router_w,
                     const float *logits_in, const float *bias, const uint16_t *residual, double *l64, float *l32,
                     int32_t *ids, double *w, int32_t *flags, double *acc_out, uint16_t *out)
{
    const int H = X->H, I = X->I;
    if (T < 0 || H <= 0 || I <= 0 || E <= 0 || k <= 0 || k > E || S < 0 || !container_ok(H, X->group, X->bits) ||
        !container_ok(I, X->group, X->bits) || (!router_w && !logits_in))
        return COLI_REF_EARG;
    int rc;
    if (logits_in) {
        for (long i = 0; i < (long)T * E; ++i) {
            l32[i] = logits_in[i];
            if (l64)
                l64[i] = (double)logits_in[i];
        }
    } else if ((rc = coli_ref_router_logits(T, E, H, x, router_w, l64, l32)) != 0) {
        return rc;
    }
    if ((rc = coli_ref_route(T, E, k, l32, bias, ids, w, flags)) != 0)
        return rc;

    const int P = T * k;
    int32_t *unique = malloc(sizeof(int32_t) * (size_t)(E + 1)), *seg = malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t *perm = malloc(sizeof(int32_t) * (size_t)(P + 1)), *pos = malloc(sizeof(int32_t) * (size_t)(P + 1));
    double *acc = calloc((size_t)T * H + 1, sizeof(double)), *xt = malloc(sizeof(double) * (size_t)H);
    double *hb = malloc(sizeof(double) * (size_t)I), *y = malloc(sizeof(double) * (size_t)H);
    rc = COLI_REF_ENOMEM;
    if (!unique || !seg || !perm || !pos || !acc || !xt || !hb || !y)
        goto done;
    int32_t U = 0;
    if ((rc = coli_ref_union(P, E, ids, unique, &U, seg, perm, pos)) != 0)
        goto done;
    rc = COLI_REF_EARG;                         /* an expert the layer reads was not given */
    for (int u = 0; u < U; ++u)
        if (!expert_present(X, unique[u]))
            goto done;
    for (int s = 0; s < S && T > 0; ++s)
        if (!expert_present(X, E + s))
            goto done;

    for (int u = 0; u < U; ++u)
        for (int at = seg[u]; at < seg[u + 1]; ++at) {
            int t = perm[at] / k, j = perm[at] % k;
            for (int c = 0; c < H; ++c)
                xt[c] = bf16_value(x[(size_t)t * H + c]);
            expert_ffn(X, unique[u], xt, hb, y);
            for (int c = 0; c < H; ++c)
                acc[(size_t)t * H + c] += w[(size_t)t * k + j] * y[c];
        }
    for (int t = 0; t < T; ++t) {
        for (int c = 0; c < H; ++c)
            xt[c] = bf16_value(x[(size_t)t * H + c]);
        for (int s = 0; s < S; ++s) {
            expert_ffn(X, E + s, xt, hb, y);
            for (int c = 0; c < H; ++c)
                acc[(size_t)t * H + c] += y[c];
        }
        if (residual)
            for (int c = 0; c < H; ++c)
                acc[(size_t)t * H + c] += bf16_value(residual[(size_t)t * H + c]);
        for (int c = 0; c < H; ++c) {
            double a = acc[(size_t)t * H + c];
            if (acc_out)
                acc_out[(size_t)t * H + c] = a;
            out[(size_t)t * H + c] = bf16_bits_of(round_bf16(a));
        }
    }
    rc = 0;
done:
    free(unique);
    free(seg);
    free(perm);
    free(pos);
    free(acc);
    free(xt);
    free(hb);
    free(y);
    return rc;
}

/* The layer with every expert's matrices in contiguous arrays with a leading
 * axis of E+S: gate_q/up_q [E+S][I][H*bits/8], down_q [E+S][H][I*bits/8],
 * gate_s/up_s [E+S][I][H/group], down_s [E+S][H][I/group]. */
int coli_ref_moe_layer(int T, int H, int I, int E, int k, int S, int group, int bits,
                       const uint8_t *gate_q, const uint16_t *gate_s, const uint8_t *up_q, const uint16_t *up_s,
                       const uint8_t *down_q, const uint16_t *down_s, const uint16_t *x, const float *router_w,
                       const float *logits_in, const float *bias, const uint16_t *residual, double *l64,
                       float *l32, int32_t *ids, double *w, int32_t *flags, double *acc_out, uint16_t *out)
{
    if (E <= 0 || S < 0 || !container_ok(H, group, bits) || !container_ok(I, group, bits))
        return COLI_REF_EARG;
    const int n = E + S;
    const size_t gu_codes = (size_t)I * H * bits / 8, gu_scales = (size_t)I * (H / group);
    const size_t dn_codes = (size_t)H * I * bits / 8, dn_scales = (size_t)H * (I / group);
    const uint8_t **q = malloc(sizeof(*q) * 3 * (size_t)n);
    const uint16_t **sc = malloc(sizeof(*sc) * 3 * (size_t)n);
    if (!q || !sc) {
        free(q);
        free(sc);
        return COLI_REF_ENOMEM;
    }
    for (int e = 0; e < n; ++e) {
        q[e] = gate_q + e * gu_codes;
        q[n + e] = up_q + e * gu_codes;
        q[2 * n + e] = down_q + e * dn_codes;
        sc[e] = gate_s + e * gu_scales;
        sc[n + e] = up_s + e * gu_scales;
        sc[2 * n + e] = down_s + e * dn_scales;
    }
    const Experts X = {H, I, group, bits, q, q + n, q + 2 * n, sc, sc + n, sc + 2 * n};
    int rc = moe_layer(T, E, k, S, &X, x, router_w, logits_in, bias, residual, l64, l32, ids, w, flags, acc_out, out);
    free(q);
    free(sc);
    return rc;
}

/* The layer with one pointer per expert and matrix (arrays of E+S pointers);
 * an expert the batch does not select may be NULL.  A NULL expert that the
 * layer would read gives COLI_REF_EARG. */
int coli_ref_moe_layer_experts(int T, int H, int I, int E, int k, int S, int group, int bits,
                               const uint8_t *const *gate_q, const uint16_t *const *gate_s,
                               const uint8_t *const *up_q, const uint16_t *const *up_s,
                               const uint8_t *const *down_q, const uint16_t *const *down_s, const uint16_t *x,
                               const float *router_w, const float *logits_in, const float *bias,
                               const uint16_t *residual, double *l64, float *l32, int32_t *ids, double *w,
                               int32_t *flags, double *acc_out, uint16_t *out)
{
    const Experts X = {H, I, group, bits, gate_q, up_q, down_q, gate_s, up_s, down_s};
    return moe_layer(T, E, k, S, &X, x, router_w, logits_in, bias, residual, l64, l32, ids, w, flags, acc_out, out);
}

/* n = bf16( h / sqrt(mean(h^2) + 1e-6) ) per token, double inside.
 * READING: the weightless pre-norm of the 16-layer stack (the pages name no
 * normalisation; the literal stack h + MoE(h) overflows bf16 in a few layers). */
int coli_ref_rms_norm(int T, int H, const uint16_t *h, uint16_t *out)
{
    if (T < 0 || H <= 0)
        return COLI_REF_EARG;
    for (int t = 0; t < T; ++t) {
        double ss = 0.0;
        for (int c = 0; c < H; ++c) {
            double v = bf16_value(h[(size_t)t * H + c]);
            ss += v * v;
        }
        double r = 1.0 / sqrt(ss / H + 1e-6);
        for (int c = 0; c < H; ++c)
            out[(size_t)t * H + c] = bf16_bits_of(round_bf16(bf16_value(h[(size_t)t * H + c]) * r));
    }
    return 0;
}
