/*
 * e8_oracle.c -- plain, slow, fp64 CPU reference for the E8 quantize path.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load this file's library.  It shares no code,
 * header, table or constant generator with the CUDA library; nothing here
 * is fast on purpose.
 *
 * Sources (titles of the pages this follows):
 *   [E8QAT-abs]  "E8-QAT: Efficient 2-Bit Quantization-Aware Training with
 *                Implicit Lattice Codebooks", abstract: the E8 lattice is an
 *                implicit 8-D codebook; weight groups are projected onto it
 *                by arithmetic; a 2-bit core encoding plus sparse extension
 *                keeps the selected lattice point exactly.
 *   [E8QAT-F2]   same paper, Figure 2 caption: fixed E8 core; arithmetic
 *                lattice projection with identity STE; core indices plus
 *                sparse escape records; Hadamard transforms and
 *                reconstruction scales applied around the projection.
 *   [E8QAT-T3]   same paper, appendix Table 3: all 65,536 core codewords
 *                decode identically; every escaped group's residual is one
 *                element of the root set R.
 *   [E8QAT-T10]  same paper, appendix Table 10: payload b = 2 + 20*rho bits
 *                per weight with 20-byte coordinate records.
 *
 * Conventions where the pages are silent (each is listed with its reason in
 * the design notes): doubled coordinates P = 2p; the core is the 65,536 E8
 * points that come first in (|p|^2, lexicographic P) order and a core index
 * is the rank in that order; the 240 roots are numbered in lexicographic
 * order; Conway-Sloane D8 rounding with round-half-even and lowest-index
 * tie break for the parity fix; coset tie goes to D8; the escape root is
 * the one giving the smallest core index; the RHT is the Sylvester Hadamard
 * in natural order, orthonormal (1/sqrt(B)), sign flip before it.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define EO_CORE 65536
#define EO_NROOTS 240
#define EO_MAXN2 48 /* |P|^2 bound of the enumeration: |p|^2 <= 12 */

typedef struct {
    int32_t n2;
    int8_t c[8];
} eo_pt;

static eo_pt* g_pts = 0;      /* every E8 point with |P|^2 <= 48, sorted */
static int64_t g_npts = 0;
static int8_t g_roots[EO_NROOTS][8];
static int g_ready = 0;

/* (|P|^2, then P lexicographically, most negative first) */
static int eo_cmp(const void* a, const void* b)
{
    const eo_pt* p = (const eo_pt*)a;
    const eo_pt* q = (const eo_pt*)b;
    if (p->n2 != q->n2) return p->n2 < q->n2 ? -1 : 1;
    for (int i = 0; i < 8; i++)
        if (p->c[i] != q->c[i]) return p->c[i] < q->c[i] ? -1 : 1;
    return 0;
}

/* E8 = D8 u (D8 + 1/2): in doubled coordinates, all entries even or all
 * odd, and sum(P) divisible by 4 (sum(p) even). */
static int eo_is_e8(const int32_t* P)
{
    int par = P[0] & 1;
    int32_t s = 0;
    for (int i = 0; i < 8; i++) {
        if ((P[i] & 1) != par) return 0;
        s += P[i];
    }
    return (s % 4) == 0;
}

/* Enumerate every E8 point of |p|^2 <= 12, sort it, pick out the roots. */
int eo_init(void)
{
    if (g_ready) return 0;
    /* upper bound: 7^8 even-type + 6^8 odd-type candidates */
    int64_t cap = 200000;
    g_pts = (eo_pt*)malloc(sizeof(eo_pt) * cap);
    if (!g_pts) return -1;
    g_npts = 0;
    for (int type = 0; type < 2; type++) {
        int nv = type ? 6 : 7;
        int vals[7];
        for (int k = 0; k < nv; k++) vals[k] = type ? (2 * k - 5) : (2 * k - 6);
        int d[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (;;) {
            int32_t P[8];
            int32_t n2 = 0;
            for (int i = 0; i < 8; i++) {
                P[i] = vals[d[i]];
                n2 += P[i] * P[i];
            }
            if (n2 <= EO_MAXN2 && eo_is_e8(P)) {
                if (g_npts >= cap) return -2;
                g_pts[g_npts].n2 = n2;
                for (int i = 0; i < 8; i++) g_pts[g_npts].c[i] = (int8_t)P[i];
                g_npts++;
            }
            int i = 7;
            while (i >= 0 && ++d[i] == nv) d[i--] = 0;
            if (i < 0) break;
        }
    }
    qsort(g_pts, (size_t)g_npts, sizeof(eo_pt), eo_cmp);
    int nr = 0;
    for (int64_t k = 0; k < g_npts; k++) {
        if (g_pts[k].n2 == 8) {
            if (nr >= EO_NROOTS) return -3;
            memcpy(g_roots[nr], g_pts[k].c, 8);
            nr++;
        }
    }
    if (nr != EO_NROOTS || g_npts < EO_CORE) return -4;
    g_ready = 1;
    return 0;
}

int64_t eo_num_points(void) { return g_npts; }

/* Export the sorted list: coords [n][8] and |P|^2 [n]. */
void eo_points(int8_t* coords, int32_t* n2)
{
    for (int64_t k = 0; k < g_npts; k++) {
        memcpy(coords + 8 * k, g_pts[k].c, 8);
        n2[k] = g_pts[k].n2;
    }
}

void eo_roots(int8_t* out) { memcpy(out, g_roots, sizeof(g_roots)); }

/* Rank of P in the sorted enumeration, or -1 when P is not an E8 point of
 * |p|^2 <= 12.  A rank below 65,536 means P is in the core and the rank is
 * its core index [E8QAT-F2, E8QAT-T3]. */
int64_t eo_rank(const int32_t* P)
{
    if (!eo_is_e8(P)) return -1;
    eo_pt key;
    key.n2 = 0;
    for (int i = 0; i < 8; i++) {
        if (P[i] < -6 || P[i] > 6) return -1;
        key.c[i] = (int8_t)P[i];
        key.n2 += P[i] * P[i];
    }
    if (key.n2 > EO_MAXN2) return -1;
    const eo_pt* hit = (const eo_pt*)bsearch(&key, g_pts, (size_t)g_npts, sizeof(eo_pt), eo_cmp);
    return hit ? (int64_t)(hit - g_pts) : -1;
}

/* ---------------------------------------------------------------------
 * Nearest-point projection [E8QAT-abs, E8QAT-F2 (b)]: Conway & Sloane's
 * decoder for E8 = D8 u (D8 + 1/2).  D8 rounding: round every coordinate
 * to the nearest integer; if the sum is odd, move the coordinate that was
 * rounded furthest one step the other way.  Do it for x and for x - 1/2
 * (then add 1/2 back) and keep whichever result is closer to x.
 * ------------------------------------------------------------------- */
static void eo_d8_round(const double* y, double* f)
{
    double s = 0.0;
    for (int i = 0; i < 8; i++) {
        f[i] = nearbyint(y[i]); /* default rounding mode: half to even */
        s += f[i];
    }
    if (fmod(s, 2.0) != 0.0) {
        int k = 0;
        double worst = -1.0;
        for (int i = 0; i < 8; i++) {
            double e = fabs(y[i] - f[i]);
            if (e > worst) { /* strict: the lowest index wins a tie */
                worst = e;
                k = i;
            }
        }
        f[k] += (y[k] >= f[k]) ? 1.0 : -1.0;
    }
}

void eo_nearest(const double* x, int32_t* P)
{
    double a[8], b[8], xm[8];
    eo_d8_round(x, a);
    for (int i = 0; i < 8; i++) xm[i] = x[i] - 0.5;
    eo_d8_round(xm, b);
    for (int i = 0; i < 8; i++) b[i] += 0.5;
    double da = 0.0, db = 0.0;
    for (int i = 0; i < 8; i++) {
        da += (x[i] - a[i]) * (x[i] - a[i]);
        db += (x[i] - b[i]) * (x[i] - b[i]);
    }
    const double* c = (db < da) ? b : a; /* a tie keeps the D8 point */
    for (int i = 0; i < 8; i++) P[i] = (int32_t)llround(2.0 * c[i]);
}

/* How far x is from a second nearest lattice point: min over roots r of
 * |x - p - r|^2 - |x - p|^2.  The roots are the Voronoi-relevant vectors of
 * E8, so this is the nearest-vs-second-nearest gap. */
double eo_margin(const double* x, const int32_t* P)
{
    double best = INFINITY;
    for (int k = 0; k < EO_NROOTS; k++) {
        double dot = 0.0;
        for (int i = 0; i < 8; i++) dot += (x[i] - 0.5 * P[i]) * (0.5 * g_roots[k][i]);
        double m = 2.0 - 2.0 * dot; /* |r|^2 = 2 */
        if (m < best) best = m;
    }
    return best;
}

/* ---------------------------------------------------------------------
 * Encoding [E8QAT-abs, E8QAT-F2 (c), E8QAT-T3]: a point in the core is its
 * core index.  Otherwise look for a root r with P - 2r in the core and keep
 * the one whose core index is smallest (escape record: core index + root);
 * if there is none, the point needs a full coordinate record (overflow).
 * Returns 0 core, 1 escape, 2 overflow.
 * ------------------------------------------------------------------- */
int eo_encode_point(const int32_t* P, int32_t* idx, int32_t* root)
{
    int64_t r = eo_rank(P);
    *root = -1;
    if (r >= 0 && r < EO_CORE) {
        *idx = (int32_t)r;
        return 0;
    }
    int64_t best = -1;
    int bestk = -1;
    for (int k = 0; k < EO_NROOTS; k++) {
        int32_t Q[8];
        for (int i = 0; i < 8; i++) Q[i] = P[i] - g_roots[k][i];
        int64_t rq = eo_rank(Q);
        if (rq >= 0 && rq < EO_CORE && (best < 0 || rq < best)) {
            best = rq;
            bestk = k;
        }
    }
    if (best >= 0) {
        *idx = (int32_t)best;
        *root = bestk;
        return 1;
    }
    *idx = 0;
    return 2;
}

/* Core codeword (doubled coordinates) of a core index. */
int eo_core_point(int32_t idx, int32_t* P)
{
    if (idx < 0 || idx >= EO_CORE) return -1;
    for (int i = 0; i < 8; i++) P[i] = g_pts[idx].c[i];
    return 0;
}

/* ---------------------------------------------------------------------
 * Hadamard transform [E8QAT-F2: "Hadamard transforms"].  H_B is the
 * Sylvester matrix, H[i][j] = (-1)^popcount(i & j).  Two forms: the
 * definition (dense sum) and the fast butterfly, unnormalised.
 * ------------------------------------------------------------------- */
void eo_hadamard_dense(const double* u, int64_t n, double* v)
{
    for (int64_t i = 0; i < n; i++) {
        double acc = 0.0;
        for (int64_t j = 0; j < n; j++) acc += (__builtin_popcountll((unsigned long long)(i & j)) & 1) ? -u[j] : u[j];
        v[i] = acc;
    }
}

void eo_fwht(double* v, int64_t n)
{
    for (int64_t h = 1; h < n; h *= 2)
        for (int64_t i = 0; i < n; i += 2 * h)
            for (int64_t j = i; j < i + h; j++) {
                double a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
}

/* ---------------------------------------------------------------------
 * bf16 with one round-half-even step from an exact double.
 * ------------------------------------------------------------------- */
uint16_t eo_bf16_bits(double v)
{
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7F80;
    int e;
    frexp(a, &e);          /* a = m * 2^e, 0.5 <= m < 1 */
    int q = e - 8;         /* bf16 keeps 8 significant bits */
    if (q < -133) q = -133; /* spacing of the subnormal range */
    double k = nearbyint(ldexp(a, -q));
    double r = ldexp(k, q);
    float f = (float)r; /* exact: r has at most 8 significant bits (inf past the top) */
    uint32_t bits;
    memcpy(&bits, &f, 4);
    return (uint16_t)(sign | (bits >> 16));
}

/* ---------------------------------------------------------------------
 * Row pipeline [E8QAT-F2]: u = d * w; v = blockwise H_B u / sqrt(B);
 * s = sqrt(mean v^2) / kappa (the reconstruction scale, one per row);
 * x = v / s; every 8-group of x is projected and encoded.  Non-finite
 * inputs are read as 0 and counted.  B = 1 means no transform.
 *
 * w      [R][C] (values of the stored input, exact in double)
 * d      [C] of +-1
 * outputs: scale[R], x[R][C] (nullable), P[G][8], margin[G] (nullable),
 *          idx[G], kind[G], root[G]; returns the count of non-finite inputs.
 * ------------------------------------------------------------------- */
int64_t eo_project_encode_rows(const double* w, int64_t R, int64_t C, const int8_t* d, int64_t B, double kappa,
                               double* scale, double* xout, int32_t* P, double* margin, int32_t* idx, int32_t* kind,
                               int32_t* root)
{
    int64_t nonfinite = 0;
    double* v = (double*)malloc(sizeof(double) * (size_t)(C > 0 ? C : 1));
    int64_t gpr = C / 8;
    for (int64_t r = 0; r < R; r++) {
        for (int64_t c = 0; c < C; c++) {
            double t = w[r * C + c];
            if (!isfinite(t)) {
                t = 0.0;
                nonfinite++;
            }
            v[c] = (double)d[c] * t;
        }
        if (B > 1) {
            double inv = 1.0 / sqrt((double)B);
            for (int64_t b0 = 0; b0 < C; b0 += B) {
                eo_fwht(v + b0, B);
                for (int64_t j = 0; j < B; j++) v[b0 + j] *= inv;
            }
        }
        double ss = 0.0;
        for (int64_t c = 0; c < C; c++) ss += v[c] * v[c];
        double s = (C > 0) ? sqrt(ss / (double)C) / kappa : 0.0;
        scale[r] = s;
        for (int64_t c = 0; c < C; c++) v[c] = (s > 0.0) ? v[c] / s : 0.0;
        if (xout) memcpy(xout + r * C, v, sizeof(double) * (size_t)C);
        for (int64_t g = 0; g < gpr; g++) {
            int64_t G = r * gpr + g;
            eo_nearest(v + 8 * g, P + 8 * G);
            if (margin) margin[G] = eo_margin(v + 8 * g, P + 8 * G);
            kind[G] = eo_encode_point(P + 8 * G, idx + G, root + G);
        }
    }
    free(v);
    return nonfinite;
}

/* ---------------------------------------------------------------------
 * Core-clipped projection [E8QAT-F2 (a): post-training quantisation starts
 * the latent weights from a fixed E8 core; (b) contrasts it with the
 * unclipped projection used during QAT]: the core point nearest to x,
 * found by searching all 65,536 core codewords in fp64.  Equal distances
 * go to the smaller core index.  margin = second-smallest minus smallest
 * squared distance (x units) over the core.
 * ------------------------------------------------------------------- */
int32_t eo_nearest_core(const double* x, double* margin)
{
    if (eo_init() != 0) return -1;
    double best = INFINITY, second = INFINITY;
    int32_t bi = 0;
    for (int32_t k = 0; k < EO_CORE; k++) {
        const int8_t* P = g_pts[k].c;
        double dd = 0.0;
        for (int i = 0; i < 8; i++) {
            double t = x[i] - 0.5 * (double)P[i];
            dd += t * t;
        }
        if (dd < best) {
            second = best;
            best = dd;
            bi = k;
        } else if (dd < second) {
            second = dd;
        }
    }
    if (margin) *margin = second - best;
    return bi;
}

/* Row pipeline with the core-clipped projection: the transform and scale of
 * eo_project_encode_rows, then the nearest core point of every group
 * (idx[G]; P[G][8] its doubled coordinates; margin[G] nullable). */
int64_t eo_project_core_rows(const double* w, int64_t R, int64_t C, const int8_t* d, int64_t B, double kappa,
                             double* scale, int32_t* P, double* margin, int32_t* idx)
{
    int64_t nonfinite = 0;
    double* v = (double*)malloc(sizeof(double) * (size_t)(C > 0 ? C : 1));
    int64_t gpr = C / 8;
    for (int64_t r = 0; r < R; r++) {
        for (int64_t c = 0; c < C; c++) {
            double t = w[r * C + c];
            if (!isfinite(t)) {
                t = 0.0;
                nonfinite++;
            }
            v[c] = (double)d[c] * t;
        }
        if (B > 1) {
            double inv = 1.0 / sqrt((double)B);
            for (int64_t b0 = 0; b0 < C; b0 += B) {
                eo_fwht(v + b0, B);
                for (int64_t j = 0; j < B; j++) v[b0 + j] *= inv;
            }
        }
        double ss = 0.0;
        for (int64_t c = 0; c < C; c++) ss += v[c] * v[c];
        double s = (C > 0) ? sqrt(ss / (double)C) / kappa : 0.0;
        scale[r] = s;
        for (int64_t c = 0; c < C; c++) v[c] = (s > 0.0) ? v[c] / s : 0.0;
        for (int64_t g = 0; g < gpr; g++) {
            int64_t G = r * gpr + g;
            idx[G] = eo_nearest_core(v + 8 * g, margin ? margin + G : NULL);
            for (int i = 0; i < 8; i++) P[8 * G + i] = g_pts[idx[G]].c[i];
        }
    }
    free(v);
    return nonfinite;
}

/* Project and encode free 8-vectors (no transform, no scale). */
void eo_project_encode_vectors(const double* x, int64_t n, int32_t* P, double* margin, int32_t* idx, int32_t* kind,
                               int32_t* root)
{
    for (int64_t k = 0; k < n; k++) {
        eo_nearest(x + 8 * k, P + 8 * k);
        if (margin) margin[k] = eo_margin(x + 8 * k, P + 8 * k);
        kind[k] = eo_encode_point(P + 8 * k, idx + k, root + k);
    }
}

/* ---------------------------------------------------------------------
 * Decode [E8QAT-abs: "preserve the selected lattice points exactly"]:
 * p = core[idx] (+ root when escaped), or the overflow coordinates.
 * Dequantised weight, rotated basis: bf16(s * p), one rounding of the exact
 * product.  Original basis: d * H_B (s * p) / sqrt(B), in double, then one
 * rounding to bf16 (this is the identity-STE forward weight).
 *
 * P  [R*C/8][8]  lattice points already assembled by the caller
 * s  [R]         the stored fp32 scales, as doubles
 * basis 0 rotated, 1 original; out_bits [R][C]; out_f64 (nullable) gets the
 * unrounded original-basis weights (basis 1 only).
 * ------------------------------------------------------------------- */
void eo_dequant_rows(const int32_t* P, const double* s, int64_t R, int64_t C, const int8_t* d, int64_t B, int basis,
                     uint16_t* out_bits, double* out_f64)
{
    double* v = (double*)malloc(sizeof(double) * (size_t)(C > 0 ? C : 1));
    for (int64_t r = 0; r < R; r++) {
        for (int64_t c = 0; c < C; c++) v[c] = s[r] * (0.5 * (double)P[r * C + c]);
        if (basis == 1) {
            if (B > 1) {
                double inv = 1.0 / sqrt((double)B);
                for (int64_t b0 = 0; b0 < C; b0 += B) {
                    eo_fwht(v + b0, B);
                    for (int64_t j = 0; j < B; j++) v[b0 + j] *= inv;
                }
            }
            for (int64_t c = 0; c < C; c++) v[c] *= (double)d[c];
            if (out_f64) memcpy(out_f64 + r * C, v, sizeof(double) * (size_t)C);
        }
        for (int64_t c = 0; c < C; c++) out_bits[r * C + c] = eo_bf16_bits(v[c]);
    }
    free(v);
}

/* Blockwise RHT of activation rows: x_rot = H_B (d * x) / sqrt(B). */
void eo_rht_vectors(const double* x, int64_t nb, int64_t C, const int8_t* d, int64_t B, double* out)
{
    double inv = (B > 1) ? 1.0 / sqrt((double)B) : 1.0;
    for (int64_t b = 0; b < nb; b++) {
        double* v = out + b * C;
        for (int64_t c = 0; c < C; c++) v[c] = (double)d[c] * x[b * C + c];
        if (B > 1)
            for (int64_t b0 = 0; b0 < C; b0 += B) {
                eo_fwht(v + b0, B);
                for (int64_t j = 0; j < B; j++) v[b0 + j] *= inv;
            }
    }
}
