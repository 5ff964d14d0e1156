/*
 * spkv_oracle.c -- plain, slow, fp64 CPU oracle for Spherical KV angle-domain
 * attention (ADA) decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or load
 * this file: only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline /
 * reference arm use it.  It shares no code, header, table or constant generator
 * with the CUDA library, and it imports nothing from it.
 *
 * Source of every definition below ("the pages"): the summary pages of
 *   "SPHERICAL KV: Angle-Domain Attention and Rate-Distortion Retention for
 *    Efficient Long-Context Inference" (gist.science/{es,fr,de}/paper/2605.18856),
 * technical summary section 2.1 "Angle-Domain Attention (ADA)":
 *   - spherical parametrisation  r = ||k||,  phi = Phi(k/||k||);
 *   - compressed-domain logit    l(q,k) ~= ||q|| * r~ * f_b(c_q, c_k);
 *   - f_b is the cosine similarity evaluated from the angle codes;
 *   - the no-reconstruction invariant (a property of the GPU kernel, not of
 *     the arithmetic, so the oracle is free to rebuild unit vectors).
 * The pages leave the coordinate convention, the quantisers, the radius code
 * and the softmax open.  The readings taken here (numbered R1..R8, the same
 * numbers the design notes use) are:
 *   R1  Phi is the textbook n-sphere chart: S_i = sum_{j>=i} x_j^2,
 *       phi_i = atan2(sqrt(S_{i+1}), x_i) in [0, pi] for i < d-2 (0-based),
 *       phi_{d-2} = atan2(x_{d-1}, x_{d-2}) taken in [0, 2 pi).
 *       atan2(0, 0) = 0, so an all-zero tail gives zero angles.
 *       Angles are quantised by a uniform mid-rise quantiser with b bits:
 *       c = floor(phi * 2^b / pi) (polar) or floor(phi * 2^b / (2 pi))
 *       (azimuth), clamped to 2^b - 1; reconstruction at the cell midpoint.
 *   R2  f_b is the exact cosine of the two decoded unit vectors; the prefix
 *       (sum of products) form and the nested form are the same number.
 *   R3  the query is coded too, at the bit width of the key's page.
 *   R4  radius code: c_r = clamp(floor((log2 r - L)/Delta + 1/2), 0, 255),
 *       r~ = 2^(L + c_r Delta); L, Delta per kv head; r = 0 gives c_r = 0.
 *   R6  logits are divided by sqrt(d) (standard attention scale).
 *   R7  softmax over retained slots only; an empty set gives a zero output.
 *   R13 exact-query variant (section 2.1 leaves f_b open; the coded query of
 *       R3 is the literal reading): f = <q/||q||, u~(c_k)>, the unquantised
 *       unit query against the decoded key; a zero query gives f = 0.
 * Arithmetic is IEEE fp64 throughout; bf16 inputs are widened exactly and
 * -0 is normalised to +0.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SPKV_ORACLE_PI 3.14159265358979323846

/* ---------------------------------------------------------------- helpers */

/* Exact bf16 -> fp64 widening (bf16 is the top half of an IEEE fp32). */
double spkv_oracle_bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    double x = (double)f;
    if (x == 0.0) x = 0.0; /* -0 -> +0 */
    return x;
}

/* fp64 -> bf16, rounding the fp64 value directly to 8 significant bits with
 * round-half-even.  Magnitudes below the fp32 normal range flush to +0.
 * NaN and overflow are not produced by the oracle's inputs. */
uint16_t spkv_oracle_f64_to_bf16(double x)
{
    if (x == 0.0 || fabs(x) < 0x1p-126) return 0; /* below the fp32 normal range */
    int e;
    double m = frexp(fabs(x), &e);       /* |x| = m 2^e, m in [0.5, 1) */
    /* keep 8 significant bits: scale m to [128, 256) and round half even */
    double s = ldexp(m, 8);
    double r = nearbyint(s);            /* default rounding mode: half even */
    double y = ldexp(r, e - 8);
    if (x < 0) y = -y;
    float f = (float)y;                 /* exact: y has 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* --------------------------------------------------- R1: angles and codes */

/* Hyperspherical angles of x (length d >= 2) into phi[0..d-2]. */
void spkv_oracle_angles(int d, const double *x, double *phi)
{
    double *S = (double *)malloc(sizeof(double) * (size_t)(d + 1));
    S[d] = 0.0;
    for (int i = d - 1; i >= 0; --i) S[i] = x[i] * x[i] + S[i + 1];
    for (int i = 0; i < d - 2; ++i) phi[i] = atan2(sqrt(S[i + 1]), x[i]);
    double a = atan2(x[d - 1], x[d - 2]);
    if (a < 0.0) a += 2.0 * SPKV_ORACLE_PI;
    phi[d - 2] = a;
    free(S);
}

/* Scaled position of an angle on the b-bit grid: phi * 2^b / pi for polar
 * angles, phi * 2^b / (2 pi) for the azimuth.  Its floor is the code. */
double spkv_oracle_angle_pos(double phi, int b, int is_azimuth)
{
    double range = is_azimuth ? 2.0 * SPKV_ORACLE_PI : SPKV_ORACLE_PI;
    return phi * ldexp(1.0, b) / range;
}

int32_t spkv_oracle_angle_code(double phi, int b, int is_azimuth)
{
    double t = floor(spkv_oracle_angle_pos(phi, b, is_azimuth));
    double top = ldexp(1.0, b) - 1.0;
    if (t > top) t = top; /* phi == pi (polar) or a rounded 2 pi (azimuth) */
    if (t < 0.0) t = 0.0;
    return (int32_t)t;
}

/* Cell midpoint of a code. */
double spkv_oracle_angle_mid(int32_t c, int b, int is_azimuth)
{
    double range = is_azimuth ? 2.0 * SPKV_ORACLE_PI : SPKV_ORACLE_PI;
    return ((double)c + 0.5) * range / ldexp(1.0, b);
}

void spkv_oracle_angle_codes(int d, const double *phi, int b, int32_t *codes)
{
    for (int i = 0; i < d - 1; ++i) codes[i] = spkv_oracle_angle_code(phi[i], b, i == d - 2);
}

/* Inverse chart: unit vector from (any) angles.
 * u_0 = cos phi_0, u_j = prod_{i<j} sin phi_i * cos phi_j (j <= d-2),
 * u_{d-1} = prod_{i<d-1} sin phi_i. */
void spkv_oracle_unit_from_angles(int d, const double *phi, double *u)
{
    double P = 1.0;
    for (int j = 0; j < d - 1; ++j) {
        u[j] = P * cos(phi[j]);
        P *= sin(phi[j]);
    }
    u[d - 1] = P;
}

/* R1/R2: decoded unit vector u~(c) from b-bit codes (midpoint angles). */
void spkv_oracle_unit_from_codes(int d, const int32_t *codes, int b, double *u)
{
    double *phi = (double *)malloc(sizeof(double) * (size_t)(d - 1));
    for (int i = 0; i < d - 1; ++i) phi[i] = spkv_oracle_angle_mid(codes[i], b, i == d - 2);
    spkv_oracle_unit_from_angles(d, phi, u);
    free(phi);
}

/* R2, prefix form: f_b = <u~(c_q), u~(c_k)>. */
double spkv_oracle_fb(int d, const int32_t *cq, const int32_t *ck, int b)
{
    double *uq = (double *)malloc(sizeof(double) * (size_t)d);
    double *uk = (double *)malloc(sizeof(double) * (size_t)d);
    spkv_oracle_unit_from_codes(d, cq, b, uq);
    spkv_oracle_unit_from_codes(d, ck, b, uk);
    double s = 0.0;
    for (int j = 0; j < d; ++j) s += uq[j] * uk[j];
    free(uq);
    free(uk);
    return s;
}

/* R2, nested form: s = cos(a_q - a_k) for the azimuth, then
 * s <- cos a_q cos a_k + sin a_q sin a_k s for the polar angles, last to first. */
double spkv_oracle_fb_nested(int d, const int32_t *cq, const int32_t *ck, int b)
{
    double aq = spkv_oracle_angle_mid(cq[d - 2], b, 1);
    double ak = spkv_oracle_angle_mid(ck[d - 2], b, 1);
    double s = cos(aq - ak);
    for (int i = d - 3; i >= 0; --i) {
        aq = spkv_oracle_angle_mid(cq[i], b, 0);
        ak = spkv_oracle_angle_mid(ck[i], b, 0);
        s = cos(aq) * cos(ak) + sin(aq) * sin(ak) * s;
    }
    return s;
}

/* ---------------------------------------------------------- R4: radius */

/* Scaled radius position (log2 r - L)/Delta + 1/2; its floor is the code
 * before clamping.  r = 0 gives -inf. */
double spkv_oracle_radius_pos(double r, double L, double Delta)
{
    if (r <= 0.0) return -INFINITY;
    return (log2(r) - L) / Delta + 0.5;
}

int32_t spkv_oracle_radius_code(double r, double L, double Delta)
{
    double t = spkv_oracle_radius_pos(r, L, Delta);
    if (!(t > 0.0)) return 0; /* also r = 0 (-inf) */
    t = floor(t);
    if (t > 255.0) t = 255.0;
    return (int32_t)t;
}

double spkv_oracle_radius_value(int32_t c, double L, double Delta)
{
    return exp2(L + (double)c * Delta);
}

/* --------------------------------------------------------------- encode */

/* Encode n keys (bf16 bits, [n, d]) at per-key bit widths bits[n].
 * codes: [n, d-1] angle codes; rcode: [n] radius codes.
 * Optional outputs (NULL to skip): apos [n, d-1] scaled angle positions,
 * rpos [n] scaled radius positions, used to find codes that sit on a
 * quantisation boundary. */
void spkv_oracle_encode(int d, int n, const uint16_t *keys, const int32_t *bits, double L,
                        double Delta, int32_t *codes, uint8_t *rcode, double *apos, double *rpos)
{
    double *x = (double *)malloc(sizeof(double) * (size_t)d);
    double *phi = (double *)malloc(sizeof(double) * (size_t)(d - 1));
    for (int t = 0; t < n; ++t) {
        const uint16_t *kt = keys + (size_t)t * d;
        double S = 0.0;
        for (int j = d - 1; j >= 0; --j) {
            x[j] = spkv_oracle_bf16_to_f64(kt[j]);
            S += x[j] * x[j];
        }
        double r = sqrt(S);
        spkv_oracle_angles(d, x, phi);
        int b = bits[t];
        for (int i = 0; i < d - 1; ++i) {
            int az = (i == d - 2);
            codes[(size_t)t * (d - 1) + i] = spkv_oracle_angle_code(phi[i], b, az);
            if (apos) apos[(size_t)t * (d - 1) + i] = spkv_oracle_angle_pos(phi[i], b, az);
        }
        rcode[t] = (uint8_t)spkv_oracle_radius_code(r, L, Delta);
        if (rpos) rpos[t] = spkv_oracle_radius_pos(r, L, Delta);
    }
    free(x);
    free(phi);
}

/* Dense key reconstruction k~ = r~ u~(c), rounded to bf16 (the strawman
 * "decompress, then dot" path of the pages' problem statement). */
void spkv_oracle_decompress(int d, int n, const int32_t *codes, const int32_t *bits,
                            const uint8_t *rcode, double L, double Delta, uint16_t *kout)
{
    double *u = (double *)malloc(sizeof(double) * (size_t)d);
    for (int t = 0; t < n; ++t) {
        spkv_oracle_unit_from_codes(d, codes + (size_t)t * (d - 1), bits[t], u);
        double r = spkv_oracle_radius_value(rcode[t], L, Delta);
        for (int j = 0; j < d; ++j) kout[(size_t)t * d + j] = spkv_oracle_f64_to_bf16(r * u[j]);
    }
    free(u);
}

/* ------------------------------------------------------------ attention */

/* Softmax over the retained logits, then the weighted sum of values.
 * logit[t] is ignored where keep[t] == 0.  Empty set -> zero output. */
static void softmax_pv(int d, int T, const double *logit, const uint8_t *keep, const uint16_t *v,
                       double *out)
{
    double m = -INFINITY;
    for (int t = 0; t < T; ++t)
        if (keep[t] && logit[t] > m) m = logit[t];
    for (int j = 0; j < d; ++j) out[j] = 0.0;
    if (m == -INFINITY) return;
    double den = 0.0;
    for (int t = 0; t < T; ++t) {
        if (!keep[t]) continue;
        double p = exp(logit[t] - m);
        den += p;
        for (int j = 0; j < d; ++j) out[j] += p * spkv_oracle_bf16_to_f64(v[(size_t)t * d + j]);
    }
    for (int j = 0; j < d; ++j) out[j] /= den;
}

/* ADA attention for the G query heads that share one kv head.
 *   q       [G, d]      bf16 bits
 *   kcodes  [T, d-1]    angle codes of the keys
 *   kbits   [T]         bit width of each key (the tier of its page)
 *   rcode   [T]         radius codes, or NULL when r_exact is given
 *   r_exact [T]         exact radii (test mode), or NULL
 *   keep    [T]         1 = retained, 0 = evicted; NULL = all retained
 *   v       [T, d]      bf16 bits
 *   out     [G, d]      fp64 attention output
 *   logits  [G, T]      fp64 logits (natural-log units), -inf where evicted;
 *                       NULL to skip
 * logit(q_g, k_t) = ||q_g|| r~_t f_b(c_q(b_t), c_k(t)) / sqrt(d). */
static void ada_group_impl(int d, int G, int T, const uint16_t *q, const int32_t *kcodes,
                           const int32_t *kbits, const uint8_t *rcode, const double *r_exact,
                           double L, double Delta, const uint8_t *keep, const uint16_t *v,
                           double *out, double *logits, int exact_q)
{
    double *x = (double *)malloc(sizeof(double) * (size_t)d);
    double *phi = (double *)malloc(sizeof(double) * (size_t)(d - 1));
    int32_t *cq = (int32_t *)malloc(sizeof(int32_t) * (size_t)(d - 1));
    double *uq = (double *)malloc(sizeof(double) * (size_t)d);
    double *uk = (double *)malloc(sizeof(double) * (size_t)d);
    double *lg = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    uint8_t *kp = (uint8_t *)malloc((size_t)(T > 0 ? T : 1));
    for (int t = 0; t < T; ++t) kp[t] = keep ? (keep[t] != 0) : 1;

    for (int g = 0; g < G; ++g) {
        double qn2 = 0.0;
        for (int j = d - 1; j >= 0; --j) {
            x[j] = spkv_oracle_bf16_to_f64(q[(size_t)g * d + j]);
            qn2 += x[j] * x[j];
        }
        double qn = sqrt(qn2);
        spkv_oracle_angles(d, x, phi);
        if (exact_q) /* R13: the unquantised unit query */
            for (int j = 0; j < d; ++j) uq[j] = qn > 0.0 ? x[j] / qn : 0.0;
        int qb = -1;
        for (int t = 0; t < T; ++t) {
            int b = kbits[t];
            if (!exact_q && b != qb) { /* R3: the query is coded at the key's bit width */
                spkv_oracle_angle_codes(d, phi, b, cq);
                spkv_oracle_unit_from_codes(d, cq, b, uq);
                qb = b;
            }
            spkv_oracle_unit_from_codes(d, kcodes + (size_t)t * (d - 1), b, uk);
            double f = 0.0;
            for (int j = 0; j < d; ++j) f += uq[j] * uk[j];
            double r = r_exact ? r_exact[t] : spkv_oracle_radius_value(rcode[t], L, Delta);
            lg[t] = qn * r * f / sqrt((double)d);
        }
        softmax_pv(d, T, lg, kp, v, out + (size_t)g * d);
        if (logits)
            for (int t = 0; t < T; ++t) logits[(size_t)g * T + t] = kp[t] ? lg[t] : -INFINITY;
    }
    free(x); free(phi); free(cq); free(uq); free(uk); free(lg); free(kp);
}

void spkv_oracle_ada_group(int d, int G, int T, const uint16_t *q, const int32_t *kcodes,
                           const int32_t *kbits, const uint8_t *rcode, const double *r_exact,
                           double L, double Delta, const uint8_t *keep, const uint16_t *v,
                           double *out, double *logits)
{
    ada_group_impl(d, G, T, q, kcodes, kbits, rcode, r_exact, L, Delta, keep, v, out, logits, 0);
}

/* The exact-query variant (R13): as spkv_oracle_ada_group, with
 * f = <q/||q||, u~(c_k)> in place of the coded query. */
void spkv_oracle_ada_group_exact_q(int d, int G, int T, const uint16_t *q, const int32_t *kcodes,
                                   const int32_t *kbits, const uint8_t *rcode, const double *r_exact,
                                   double L, double Delta, const uint8_t *keep, const uint16_t *v,
                                   double *out, double *logits)
{
    ada_group_impl(d, G, T, q, kcodes, kbits, rcode, r_exact, L, Delta, keep, v, out, logits, 1);
}

/* Dense attention for G query heads over bf16 keys:
 * logit = q . k / sqrt(d), softmax over retained slots, times V. */
void spkv_oracle_dense_group(int d, int G, int T, const uint16_t *q, const uint16_t *k,
                             const uint8_t *keep, const uint16_t *v, double *out, double *logits)
{
    double *lg = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    uint8_t *kp = (uint8_t *)malloc((size_t)(T > 0 ? T : 1));
    for (int t = 0; t < T; ++t) kp[t] = keep ? (keep[t] != 0) : 1;
    for (int g = 0; g < G; ++g) {
        for (int t = 0; t < T; ++t) {
            double s = 0.0;
            for (int j = 0; j < d; ++j)
                s += spkv_oracle_bf16_to_f64(q[(size_t)g * d + j]) *
                     spkv_oracle_bf16_to_f64(k[(size_t)t * d + j]);
            lg[t] = s / sqrt((double)d);
        }
        softmax_pv(d, T, lg, kp, v, out + (size_t)g * d);
        if (logits)
            for (int t = 0; t < T; ++t) logits[(size_t)g * T + t] = kp[t] ? lg[t] : -INFINITY;
    }
    free(lg); free(kp);
}

/* ------------------------------------------------------------ RDR controller
 * Rate-distortion retention (technical summary section 2.2): for every
 * state, a residency decision and a precision tier under a hard memory
 * budget, from a distortion surrogate built on the angular error of the
 * codes scaled by the query and key magnitudes, with protected states kept
 * at the top tier.  The section leaves the formulas open; the readings are:
 *   R14 the decision unit is a token: its kv heads share a page, so they
 *       share its tier b (b = 0: evicted);
 *   R15 distortion D_t(b) = w_t eps_b with w_t = sum_h qn_h ||k_{t,h}|| and
 *       eps_b = pi / (2^b sqrt 12), the RMS error of one uniformly coded
 *       angle; an evicted token costs eps = 1 (its whole logit is lost);
 *   R16 rate R(b) = H_kv (16 b + 1 + 256) bytes for a resident token (codes,
 *       radius byte, bf16 value row), 0 when evicted;
 *   R17 protected tokens take b_max (the largest tier allowed) and count
 *       against the budget.
 * Solver (the Lagrangian relaxation): every token minimises
 * D_t(b) + lambda R(b) on its own (equal costs: the larger b); lambda is the
 * smallest value, found by doubling then 100 bisection steps, whose total
 * rate fits the budget.  Returns 0, or 1 when the protected tokens alone
 * exceed the budget (then all others are evicted and lambda = +inf).  keys [T, H_kv, d] bf16;
 * qn [H_kv]; protect [T] or NULL; tier_mask bit t: b = {3,4,6,8}[t]. */
static const int kRdrBits[4] = {3, 4, 6, 8};

static double rdr_eps(int b) { return b == 0 ? 1.0 : SPKV_ORACLE_PI / (ldexp(1.0, b) * sqrt(12.0)); }

static double rdr_rate(int b, int Hkv) { return b == 0 ? 0.0 : (double)Hkv * (16.0 * b + 1.0 + 256.0); }

static double rdr_assign(int T, int Hkv, const double *w, const uint8_t *protect, uint32_t tier_mask, int bmax,
                         double lambda, int32_t *tier)
{
    double rate = 0.0;
    for (int t = 0; t < T; ++t) {
        int best = 0;
        if (protect && protect[t]) {
            best = bmax;
        } else {
            double bc = w[t] * rdr_eps(0) + lambda * rdr_rate(0, Hkv);
            for (int i = 0; i < 4; ++i) {
                if (!((tier_mask >> i) & 1u)) continue;
                const int b = kRdrBits[i];
                const double c = w[t] * rdr_eps(b) + lambda * rdr_rate(b, Hkv);
                if (c <= bc) { bc = c; best = b; }
            }
        }
        tier[t] = best;
        rate += rdr_rate(best, Hkv);
    }
    return rate;
}

int spkv_oracle_rdr_plan(int d, int T, int Hkv, const uint16_t *keys, const double *qn, const uint8_t *protect,
                         double budget, uint32_t tier_mask, int32_t *tier, double *lambda_out, double *rate_out,
                         double *dist_out)
{
    int bmax = 0, status = 0;
    for (int i = 0; i < 4; ++i)
        if ((tier_mask >> i) & 1u) bmax = kRdrBits[i];
    double *w = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    for (int t = 0; t < T; ++t) {
        double wt = 0.0;
        for (int h = 0; h < Hkv; ++h) {
            double n2 = 0.0;
            for (int j = 0; j < d; ++j) {
                const double x = spkv_oracle_bf16_to_f64(keys[((size_t)t * Hkv + h) * d + j]);
                n2 += x * x;
            }
            wt += qn[h] * sqrt(n2);
        }
        w[t] = wt;
    }
    double lambda = 0.0;
    double rate = rdr_assign(T, Hkv, w, protect, tier_mask, bmax, 0.0, tier);
    if (rate > budget) {
        double prot_rate = 0.0;
        for (int t = 0; t < T; ++t)
            if (protect && protect[t]) prot_rate += rdr_rate(bmax, Hkv);
        if (prot_rate > budget) {
            /* the protected tokens alone exceed the budget: no multiplier
             * fits; they stay at b_max and every other token is evicted */
            status = 1;
            lambda = INFINITY;
            for (int t = 0; t < T; ++t) tier[t] = (protect && protect[t]) ? bmax : 0;
            rate = prot_rate;
        } else {
            /* a multiplier large enough that the rate fits (at worst every
             * unprotected token evicted), then bisection on [0, hi] */
            double hi = 1.0;
            int n = 0;
            while (rdr_assign(T, Hkv, w, protect, tier_mask, bmax, hi, tier) > budget && n < 2000) {
                hi *= 2.0;
                ++n;
            }
            double lo = 0.0;
            for (int it = 0; it < 100; ++it) {
                const double mid = 0.5 * (lo + hi);
                if (rdr_assign(T, Hkv, w, protect, tier_mask, bmax, mid, tier) > budget) lo = mid;
                else hi = mid;
            }
            lambda = hi;
            rate = rdr_assign(T, Hkv, w, protect, tier_mask, bmax, lambda, tier);
        }
    }
    double dist = 0.0;
    for (int t = 0; t < T; ++t) dist += w[t] * rdr_eps(tier[t]);
    if (lambda_out) *lambda_out = lambda;
    if (rate_out) *rate_out = rate;
    if (dist_out) *dist_out = dist;
    free(w);
    return status;
}

/* The assignment at one multiplier (the step the bisection repeats): tiers of
 * every token at lambda and their total rate, with the weights w_t as in
 * spkv_oracle_rdr_plan.  Exposed for the pins of the solver. */
double spkv_oracle_rdr_assign(int d, int T, int Hkv, const uint16_t *keys, const double *qn, const uint8_t *protect,
                              uint32_t tier_mask, double lambda, int32_t *tier)
{
    int bmax = 0;
    for (int i = 0; i < 4; ++i)
        if ((tier_mask >> i) & 1u) bmax = kRdrBits[i];
    double *w = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    for (int t = 0; t < T; ++t) {
        double wt = 0.0;
        for (int h = 0; h < Hkv; ++h) {
            double n2 = 0.0;
            for (int j = 0; j < d; ++j) {
                const double x = spkv_oracle_bf16_to_f64(keys[((size_t)t * Hkv + h) * d + j]);
                n2 += x * x;
            }
            wt += qn[h] * sqrt(n2);
        }
        w[t] = wt;
    }
    const double rate = rdr_assign(T, Hkv, w, protect, tier_mask, bmax, lambda, tier);
    free(w);
    return rate;
}
