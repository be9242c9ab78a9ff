/*
 * nm_oracle.c -- plain, slow, fp64 CPU oracle for the N:M-pruned linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark load this library.  It shares no code, header
 * or table with the CUDA library and must never be used by the product path.
 *
 * Every function is the plain definition written out as loops, in the order
 * the definition states.  Passages followed (page title, section):
 *   - SparseForge (arXiv 2605.06402), "Estimativa de Importância Consciente do
 *     Hessiano": importance score s = (H + eps) * W^2; "Mistura Progressiva":
 *     the hard target keeps the top-N entries of each group by that score.
 *   - Sparsity Induction (arXiv 2602.21652), section 2C "Snelle Hessian Update":
 *     the diagonal Gauss-Newton proxy of the input activations, read here as
 *     H_j = mean_t x_{t,j}^2.
 *   - Sparse-BitNet (arXiv 2603.05168), section 1/2: N:M keeps at most N of
 *     every M consecutive weights; the mask is taken from latent magnitudes;
 *     quantise first, then mask; ternary values gamma*{-1,0,+1}.
 *   - SlideSparse (arXiv 2603.05232), section 2A "Decomposição por Janela
 *     Deslizante": a (2N-2):2N group is covered by N-1 width-4 windows at
 *     stride 2, each 2:4; section 2B "Elevação de Ativação": activation columns
 *     are duplicated so the lifted product equals the original one.
 *
 * Readings of points the pages leave open (each also listed in the design
 * notes): mean (1/T) with no factor 2 for H; a mean is the exact sum of its
 * terms (every term here is a dyadic rational) rounded once to fp64, to
 * nearest with ties to even, then one IEEE division by the count -- so no
 * summation order enters the definition; S rounded once from fp64 to fp32;
 * groups run along the input (K) dimension; ties go to the lower index; a
 * ragged tail group is zero-padded (score 0, value 0); survivor k of a group
 * goes to window k/2.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fPIC -shared (no fast-math, no
 * FMA contraction), so every fp64 operation rounds exactly once as written.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 bit pattern -> fp64 (exact: bf16 is the top half of an fp32). */
static double bf16_to_f64(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static float bf16_to_f32(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* fp64 -> bf16, round to nearest even, straight from the fp64 value (no fp32
 * step).  Written from the IEEE-754 rounding definition for normal numbers; a
 * value outside the normal bf16 range returns 0xFFFF (signalled to caller). */
static uint16_t f64_to_bf16_rne(double v) {
    uint64_t u;
    memcpy(&u, &v, sizeof u);
    uint16_t sign = (uint16_t)((u >> 63) << 15);
    int e = (int)((u >> 52) & 0x7FF);
    if (e == 0 && (u & 0xFFFFFFFFFFFFFull) == 0) return sign; /* +-0 */
    int exp_unbiased = e - 1023;
    if (exp_unbiased < -126 || exp_unbiased > 127) return 0xFFFF;
    uint64_t mant = (u & 0xFFFFFFFFFFFFFull) | (1ull << 52); /* 53-bit significand */
    /* keep 8 significant bits (1 implicit + 7): drop 45 bits, ties to even */
    uint64_t keep = mant >> 45;
    uint64_t rem = mant & ((1ull << 45) - 1);
    uint64_t half = 1ull << 44;
    if (rem > half || (rem == half && (keep & 1))) keep += 1;
    if (keep == (1ull << 8)) { keep >>= 1; exp_unbiased += 1; }
    if (exp_unbiased > 127) return 0xFFFF;
    return (uint16_t)(sign | ((uint16_t)(exp_unbiased + 127) << 7) | (uint16_t)(keep & 0x7F));
}

static int64_t groups_of(int64_t K, int m) { return (K + m - 1) / m; }

/* ------------------------------------------------------------------------ */
/* Exact sums of bf16-derived terms.  A finite bf16 value with exponent field
 * e and fraction f has the significand m = 128 + f (e >= 1) or m = f (e = 0)
 * and the value m * 2^(max(e,1) - 134).  So |x| is an integer multiple of
 * 2^-134 and x^2 an integer multiple of 2^-268: both sums below are sums of
 * integers, formed exactly with integer arithmetic and rounded once.        */

#define ORACLE_DIGITS 24   /* 768-bit unsigned integer, 32-bit digits */

/* n += v << shift (v < 2^64) */
static void big_add_shifted(uint32_t *n, uint64_t v, int shift) {
    int d = shift / 32, b = shift % 32;
    /* v << b spans at most three digits */
    uint64_t lo = (v << b) & 0xFFFFFFFFull;
    uint64_t mid = b ? ((v >> (32 - b)) & 0xFFFFFFFFull) : ((v >> 32) & 0xFFFFFFFFull);
    uint64_t hi = b ? (v >> (64 - b)) : 0;
    uint64_t carry = 0;
    uint64_t part[3] = {lo, mid, hi};
    for (int i = d; i < ORACLE_DIGITS; ++i) {
        uint64_t add = (i - d < 3) ? part[i - d] : 0;
        uint64_t s = (uint64_t)n[i] + add + carry;
        n[i] = (uint32_t)s;
        carry = s >> 32;
        if (i - d >= 2 && carry == 0) break;
    }
}

/* the integer n times 2^-scale, rounded to the nearest fp64 (ties to even).
 * n < 2^767 and scale <= 268 keep the result a normal, finite double. */
static double big_round_to_double(const uint32_t *n, int scale) {
    int top = -1;
    for (int i = ORACLE_DIGITS - 1; i >= 0 && top < 0; --i)
        if (n[i])
            for (int b = 31; b >= 0; --b)
                if ((n[i] >> b) & 1u) { top = 32 * i + b; break; }
    if (top < 0) return 0.0;
    /* bit p of n */
    #define BIT(p) (((p) >= 0) ? ((n[(p) / 32] >> ((p) % 32)) & 1u) : 0u)
    uint64_t sig = 0;                        /* the 53 bits from `top` down */
    for (int p = top; p > top - 53; --p) sig = (sig << 1) | BIT(p);
    int low = top - 53;                      /* the first bit below the kept ones */
    int round_bit = (int)BIT(low);
    int sticky = 0;
    for (int p = low - 1; p >= 0 && !sticky; --p) sticky = (int)BIT(p);
    #undef BIT
    if (round_bit && (sticky || (sig & 1u))) sig += 1;   /* 2^53 stays exact */
    return ldexp((double)sig, low + 1 - scale);
}

/* ------------------------------------------------------------------------ */
/* O1: diagonal Gauss-Newton proxy H_j = (1/T) sum_t x_{t,j}^2:
 *   the exact sum of the squares rounded once to fp64, then divided by T.
 * Any NaN in a column makes its H NaN; otherwise any infinity makes it +inf. */
void oracle_hessian_diag(const uint16_t *X, int64_t T, int64_t K, int64_t ldx, double *H) {
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < K; ++j) {
        uint64_t count[256];   /* sum of m^2 over the values with exponent field e */
        memset(count, 0, sizeof count);
        int nan = 0, inf = 0;
        for (int64_t t = 0; t < T; ++t) {
            uint16_t b = X[t * ldx + j];
            int e = (b >> 7) & 0xFF, f = b & 0x7F;
            if (e == 0xFF) {
                if (f) nan = 1; else inf = 1;
                continue;
            }
            uint64_t m = e ? (uint64_t)(128 + f) : (uint64_t)f;
            count[e] += m * m;
        }
        if (nan) { H[j] = NAN; continue; }
        if (inf) { H[j] = INFINITY; continue; }
        uint32_t n[ORACLE_DIGITS];
        memset(n, 0, sizeof n);
        for (int e = 0; e < 255; ++e)
            if (count[e]) big_add_shifted(n, count[e], 2 * (e ? e : 1));  /* units of 2^-268 */
        double sum = big_round_to_double(n, 268);
        H[j] = sum / (double)T;
    }
}

/* O(d_in) refresh of H under per-channel equivalent scaling (Sparsity
 * Induction, sec. 2C "Snelle Hessian Update"): with W' = W diag(s) and
 * X' = X diag(1/s) the product is unchanged and the proxy of X' is
 *   H'_j = H_j / (s_j * s_j)     (fp64: one multiply, one division),
 * so the scores of W' are refreshed without re-reading X.                  */
void oracle_hessian_rescale(const double *H, const double *s, int64_t K, double *out) {
    for (int64_t j = 0; j < K; ++j) out[j] = H[j] / (s[j] * s[j]);
}

/* Hutchinson's stochastic estimate of diag(A), A = X^T X / T (the Gram
 * matrix whose diagonal is H), the Rademacher-vector estimator of SparseForge
 * (arXiv 2605.06402), "Estimativa de Importancia Consciente do Hessiano":
 *   D_k = (1/S) sum_s z_s[k] (A z_s)[k],   z_s in {-1, +1}^K
 * with A z = X^T (X z) / T.  Sign s of column k: bit k % 32 of word k / 32
 * of row s of zbits set = -1.  Plain fp64 loops.                           */
void oracle_hutchinson_diag(const uint16_t *X, int64_t T, int64_t K, int64_t ldx, const uint32_t *zbits,
                            int64_t S, double *D) {
    const int64_t words = (K + 31) / 32;
    double *u = (double *)malloc((size_t)T * sizeof(double));
    for (int64_t k = 0; k < K; ++k) D[k] = 0.0;
    for (int64_t s = 0; s < S; ++s) {
        const uint32_t *zs = zbits + s * words;
        #pragma omp parallel for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            double acc = 0.0;
            for (int64_t j = 0; j < K; ++j) {
                const double x = bf16_to_f64(X[t * ldx + j]);
                acc = acc + (((zs[j >> 5] >> (j & 31)) & 1u) ? -x : x);
            }
            u[t] = acc;
        }
        #pragma omp parallel for schedule(static)
        for (int64_t k = 0; k < K; ++k) {
            double v = 0.0;
            for (int64_t t = 0; t < T; ++t) v = v + bf16_to_f64(X[t * ldx + k]) * u[t];
            const double z = ((zs[k >> 5] >> (k & 31)) & 1u) ? -1.0 : 1.0;
            D[k] = D[k] + z * (v / (double)T);
        }
    }
    for (int64_t k = 0; k < K; ++k) D[k] = D[k] / (double)S;
    free(u);
}

/* Same quantity, one sequential fp64 sum over all tokens in ascending t
 * (diagnostic only: rounds at every addition, so it depends on the order). */
void oracle_hessian_diag_naive(const uint16_t *X, int64_t T, int64_t K, int64_t ldx, double *H) {
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < K; ++j) {
        double total = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            double x = bf16_to_f64(X[t * ldx + j]);
            total = total + x * x;
        }
        H[j] = total / (double)T;
    }
}

/* ------------------------------------------------------------------------ */
/* O2: importance score S_ij = fp32( (H_j + eps) * W_ij^2 ), one rounding.   */
void oracle_score_hessian(const double *H, double eps, const uint16_t *W, int64_t R, int64_t K,
                          int64_t ldw, float *S) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < R; ++i) {
        for (int64_t j = 0; j < K; ++j) {
            double w = bf16_to_f64(W[i * ldw + j]);
            double h = H[j] + eps;
            double w2 = w * w;
            double s = h * w2;
            S[i * K + j] = (float)s;
        }
    }
}

/* Latent-magnitude score S_ij = |W_ij| (exact in fp32). */
void oracle_score_magnitude(const uint16_t *W, int64_t R, int64_t K, int64_t ldw, float *S) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < R; ++i)
        for (int64_t j = 0; j < K; ++j)
            S[i * K + j] = fabsf(bf16_to_f32(W[i * ldw + j]));
}

/* ------------------------------------------------------------------------ */
/* O3/O4: per-group top-n selection (ties -> lower index), compression of the
 * kept values in ascending column order, 2:4 metadata when m == 4.
 *   mask   : [R x ceil(G*m/32)] u32, bit (c % 32) of word c/32 = position c kept
 *   vals   : [R x G*n] bf16 bits
 *   meta24 : [R x ceil(G/2)] bytes, only for 2:4 (n == 2, m == 4): nibble
 *            idx0 | idx1<<2, even group in the low nibble
 * Returns 0, or -1 on an unsupported n:m or a non-finite / negative score.   */
int oracle_prune(const float *S, int64_t lds, const uint16_t *V, int64_t ldv, int64_t R, int64_t K,
                 int n, int m, uint32_t *mask, uint16_t *vals, uint8_t *meta24) {
    if (m < 2 || m > 16 || n < 1 || n >= m) return -1;
    const int64_t G = groups_of(K, m);
    const int64_t mwords = (G * m + 31) / 32;
    const int64_t mbytes = (G + 1) / 2;
    int bad = 0;
    #pragma omp parallel for schedule(static) reduction(|:bad)
    for (int64_t i = 0; i < R; ++i) {
        uint32_t *mrow = mask + i * mwords;
        memset(mrow, 0, (size_t)mwords * sizeof(uint32_t));
        if (m == 4 && n == 2 && meta24) memset(meta24 + i * mbytes, 0, (size_t)mbytes);
        for (int64_t g = 0; g < G; ++g) {
            float s[16];
            uint16_t v[16];
            for (int q = 0; q < m; ++q) {
                int64_t c = g * m + q;
                if (c < K) {
                    s[q] = S[i * lds + c];
                    v[q] = V[i * ldv + c];
                    if (!(s[q] >= 0.0f) || isinf(s[q])) bad = 1;
                } else {
                    s[q] = 0.0f; /* zero-padded tail */
                    v[q] = 0;
                }
            }
            int kept = 0;
            int idx[16];
            for (int q = 0; q < m; ++q) {
                int rank = 0;
                for (int p = 0; p < m; ++p)
                    if (s[p] > s[q] || (s[p] == s[q] && p < q)) ++rank;
                if (rank < n) idx[kept++] = q; /* ascending q */
            }
            for (int k = 0; k < kept; ++k) {
                int64_t c = g * m + idx[k];
                mrow[c / 32] |= 1u << (c % 32);
                vals[i * (G * n) + g * n + k] = v[idx[k]];
            }
            if (kept != n) bad = 1;
            if (m == 4 && n == 2 && meta24) {
                uint8_t nib = (uint8_t)(idx[0] | (idx[1] << 2));
                meta24[i * mbytes + g / 2] |= (uint8_t)(nib << (4 * (g % 2)));
            }
        }
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------ */
/* O5: sliding-window decomposition of a (2Ns-2):2Ns mask into Ns-1 windows
 * (width 4, stride 2).  Survivor k of a group (0-based, ascending position q_k)
 * goes to window k/2 with in-window index q_k - 2*(k/2).
 *   wmeta : [R x ceil(G*(Ns-1)/2)] bytes, one nibble idx0 | idx1<<2 per window,
 *           windows in (group, window) order, even window in the low nibble.
 * Returns 0, or -1 if a group does not hold exactly m-2 survivors or an index
 * falls outside its window.                                                  */
int oracle_slide_pack(const uint32_t *mask, int64_t R, int64_t K, int m, uint8_t *wmeta) {
    if (m < 4 || m % 2) return -1;
    const int Ns = m / 2;
    const int64_t G = groups_of(K, m);
    const int64_t mwords = (G * m + 31) / 32;
    const int64_t nw = G * (Ns - 1);
    const int64_t wbytes = (nw + 1) / 2;
    int bad = 0;
    #pragma omp parallel for schedule(static) reduction(|:bad)
    for (int64_t i = 0; i < R; ++i) {
        const uint32_t *mrow = mask + i * mwords;
        uint8_t *wrow = wmeta + i * wbytes;
        memset(wrow, 0, (size_t)wbytes);
        for (int64_t g = 0; g < G; ++g) {
            int q[16], cnt = 0;
            for (int p = 0; p < m; ++p) {
                int64_t c = g * m + p;
                if ((mrow[c / 32] >> (c % 32)) & 1u) q[cnt++] = p;
            }
            if (cnt != m - 2) { bad = 1; continue; }
            for (int w = 0; w < Ns - 1; ++w) {
                int a = q[2 * w] - 2 * w, b = q[2 * w + 1] - 2 * w;
                if (a < 0 || a > 3 || b < 0 || b > 3 || a >= b) bad = 1;
                int64_t wi = g * (Ns - 1) + w;
                wrow[wi / 2] |= (uint8_t)(((a & 3) | ((b & 3) << 2)) << (4 * (wi % 2)));
            }
        }
    }
    return bad ? -1 : 0;
}

/* Inverse of the pack: rebuild the dense masked matrix (mask (.) V) [R x K]
 * from the window values and window metadata. Returns -1 on a bad nibble.    */
int oracle_slide_unpack(const uint16_t *vals, const uint8_t *wmeta, int64_t R, int64_t K, int m,
                        uint16_t *Wd) {
    if (m < 4 || m % 2) return -1;
    const int Ns = m / 2, n = m - 2;
    const int64_t G = groups_of(K, m);
    const int64_t nw = G * (Ns - 1);
    const int64_t wbytes = (nw + 1) / 2;
    int bad = 0;
    #pragma omp parallel for schedule(static) reduction(|:bad)
    for (int64_t i = 0; i < R; ++i) {
        memset(Wd + i * K, 0, (size_t)K * sizeof(uint16_t));
        for (int64_t g = 0; g < G; ++g)
            for (int w = 0; w < Ns - 1; ++w) {
                int64_t wi = g * (Ns - 1) + w;
                int nib = (wmeta[i * wbytes + wi / 2] >> (4 * (wi % 2))) & 0xF;
                int a = nib & 3, b = nib >> 2;
                if (a >= b) bad = 1;
                int64_t ca = g * m + 2 * w + a, cb = g * m + 2 * w + b;
                uint16_t va = vals[i * (G * n) + g * n + 2 * w];
                uint16_t vb = vals[i * (G * n) + g * n + 2 * w + 1];
                if (ca < K) Wd[i * K + ca] = va; else if (va & 0x7FFF) bad = 1;
                if (cb < K) Wd[i * K + cb] = vb; else if (vb & 0x7FFF) bad = 1;
            }
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------ */
/* O6: activation lifting X'[t, g*4(Ns-1) + 4w + i] = X[t, g*m + 2w + i],
 * zero where the source column is past K.  XL is [T x G*(Ns-1)*4].          */
int oracle_lift(const uint16_t *X, int64_t T, int64_t K, int64_t ldx, int m, uint16_t *XL) {
    if (m < 4 || m % 2) return -1;
    const int Ns = m / 2;
    const int64_t G = groups_of(K, m);
    const int64_t KL = G * (Ns - 1) * 4;
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t g = 0; g < G; ++g)
            for (int w = 0; w < Ns - 1; ++w)
                for (int c = 0; c < 4; ++c) {
                    int64_t src = g * m + 2 * w + c;
                    XL[t * KL + g * (Ns - 1) * 4 + 4 * w + c] = src < K ? X[t * ldx + src] : 0;
                }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* O7: Y64[t, r] = sum over kept k (ascending) of X[t,k] * V[r,k], in fp64.
 * rows (may be NULL = all tokens) selects which token rows to compute;
 * Y is [nrows x R] in the order of rows.                                     */
void oracle_gemm_masked(const uint16_t *X, int64_t T, int64_t K, int64_t ldx,
                        const uint32_t *mask, int m, const uint16_t *V, int64_t ldv, int64_t R,
                        const int64_t *rows, int64_t nrows, double *Y) {
    const int64_t G = groups_of(K, m);
    const int64_t mwords = (G * m + 31) / 32;
    if (!rows) nrows = T;
    #pragma omp parallel for schedule(dynamic, 1) collapse(2)
    for (int64_t a = 0; a < nrows; ++a) {
        for (int64_t r = 0; r < R; ++r) {
            int64_t t = rows ? rows[a] : a;
            const uint32_t *mrow = mask + r * mwords;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                if (!((mrow[k / 32] >> (k % 32)) & 1u)) continue;
                double p = bf16_to_f64(X[t * ldx + k]) * bf16_to_f64(V[r * ldv + k]);
                acc = acc + p;
            }
            Y[a * R + r] = acc;
        }
    }
}

/* Dense fp64 product Y64 = X * Wd^T, sequential ascending k, zero products
 * skipped (so it equals oracle_gemm_masked when Wd = mask (.) V).            */
void oracle_gemm_dense(const uint16_t *X, int64_t T, int64_t K, int64_t ldx,
                       const uint16_t *Wd, int64_t ldw, int64_t R,
                       const int64_t *rows, int64_t nrows, double *Y) {
    if (!rows) nrows = T;
    #pragma omp parallel for schedule(dynamic, 1) collapse(2)
    for (int64_t a = 0; a < nrows; ++a) {
        for (int64_t r = 0; r < R; ++r) {
            int64_t t = rows ? rows[a] : a;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double w = bf16_to_f64(Wd[r * ldw + k]);
                if (w == 0.0) continue;
                acc = acc + bf16_to_f64(X[t * ldx + k]) * w;
            }
            Y[a * R + r] = acc;
        }
    }
}

/* Lifted product: Y64[t, r] = sum over windows (ascending K' order) of the two
 * selected products XL[t, window col] * window value, in fp64.              */
void oracle_gemm_lifted(const uint16_t *XL, int64_t T, int64_t KL, const uint16_t *vals,
                        const uint8_t *wmeta, int64_t R, int64_t K, int m,
                        const int64_t *rows, int64_t nrows, double *Y) {
    const int Ns = m / 2, n = m - 2;
    const int64_t G = groups_of(K, m);
    const int64_t nw = G * (Ns - 1);
    const int64_t wbytes = (nw + 1) / 2;
    if (!rows) nrows = T;
    #pragma omp parallel for schedule(dynamic, 1) collapse(2)
    for (int64_t a = 0; a < nrows; ++a) {
        for (int64_t r = 0; r < R; ++r) {
            int64_t t = rows ? rows[a] : a;
            double acc = 0.0;
            for (int64_t wi = 0; wi < nw; ++wi) {
                int nib = (wmeta[r * wbytes + wi / 2] >> (4 * (wi % 2))) & 0xF;
                int64_t g = wi / (Ns - 1);
                int w = (int)(wi % (Ns - 1));
                int sel[2] = {nib & 3, nib >> 2};
                for (int s = 0; s < 2; ++s) {
                    double x = bf16_to_f64(XL[t * KL + 4 * wi + sel[s]]);
                    double v = bf16_to_f64(vals[r * (G * n) + g * n + 2 * w + s]);
                    acc = acc + x * v;
                }
            }
            Y[a * R + r] = acc;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Ternary absmean quantisation (Sparse-BitNet, "O Problema" item 1):
 *   gamma = mean |W| over the tensor: the exact sum of the |w| rounded once to
 *           fp64, then divided by R*K;
 *   q     = clip(rint(W / gamma), -1, 1), ties to even;
 *   W_q   = q * bf16(gamma), bf16(gamma) rounded to nearest even from fp64.
 * Returns gamma (fp64), or -1.0 if bf16(gamma) is out of the normal range or
 * W holds a NaN or an infinity.                                              */
double oracle_ternary(const uint16_t *W, int64_t R, int64_t K, int64_t ldw, uint16_t *Wq) {
    uint64_t count[256];   /* sum of m over the values with exponent field e */
    memset(count, 0, sizeof count);
    int bad = 0;
    /* integer counts: each thread counts its rows, the counts are added after */
    #pragma omp parallel reduction(|:bad)
    {
        uint64_t mine[256];
        memset(mine, 0, sizeof mine);
        #pragma omp for schedule(static)
        for (int64_t i = 0; i < R; ++i)
            for (int64_t j = 0; j < K; ++j) {
                uint16_t b = W[i * ldw + j];
                int e = (b >> 7) & 0xFF, f = b & 0x7F;
                if (e == 0xFF) { bad = 1; continue; }
                mine[e] += e ? (uint64_t)(128 + f) : (uint64_t)f;
            }
        #pragma omp critical
        for (int e = 0; e < 256; ++e) count[e] += mine[e];
    }
    if (bad) return -1.0;
    uint32_t n[ORACLE_DIGITS];
    memset(n, 0, sizeof n);
    for (int e = 0; e < 255; ++e)
        if (count[e]) big_add_shifted(n, count[e], e ? e : 1);   /* units of 2^-134 */
    double total = big_round_to_double(n, 134);
    double gamma = total / ((double)R * (double)K);
    uint16_t gb = f64_to_bf16_rne(gamma);
    if (gb == 0xFFFF || gamma == 0.0) return -1.0;
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < R; ++i)
        for (int64_t j = 0; j < K; ++j) {
            double q = rint(bf16_to_f64(W[i * ldw + j]) / gamma);
            if (q > 1.0) q = 1.0;
            if (q < -1.0) q = -1.0;
            Wq[i * K + j] = q == 0.0 ? 0 : (q > 0 ? gb : (uint16_t)(gb | 0x8000));
        }
    return gamma;
}

/* Exposed for tests of the rounding helper. */
/* ------------------------------------------------------------------------ */
/* FP8 path (SlideSparse sec. 2B: the lift is fused into the per-token
 * INT8/FP8/FP4 quantisation of the activations; sec. 2C: online, one fused
 * quantise-and-lift kernel, then the sparse GEMM).  Format: E4M3 -- sign,
 * 4 exponent bits (bias 7), 3 mantissa bits; code e > 0 has the value
 * 2^(e-7) (1 + m/8), code e = 0 the value m 2^-9; e = 15, m = 7 is NaN, so
 * the largest finite value is 448 (code 0x7E).  Rounding: to the nearest
 * finite value, ties to the even code, magnitudes beyond 448 clamp to 448.
 * Scales (a reading: the pages fix no scale rule): per token (activations)
 * and per weight row, scale = amax / 448 in fp32 (1 when amax = 0); a value
 * x becomes the code of fp32(x * inv), inv = fp32(1 / scale) (multiplying by
 * the reciprocal, as per-token FP8 quantisers commonly do).                 */
double oracle_e4m3_value(uint8_t c) {
    const int e = (c >> 3) & 15, mant = c & 7;
    const double v = e == 0 ? ldexp((double)mant, -9) : ldexp(1.0 + mant / 8.0, e - 7);
    return (c & 0x80) ? -v : v;
}

/* nearest finite E4M3 code by search over all 127 non-negative codes; codes
 * are monotone in value and the last code bit is the last mantissa bit, so
 * "even" is "code bit 0 clear" */
uint8_t oracle_e4m3_encode(float x) {
    const double a = fabs((double)x);
    uint8_t best = 0;
    double bd = a;
    for (int c = 1; c <= 0x7E; ++c) {
        const double d = fabs(oracle_e4m3_value((uint8_t)c) - a);
        if (d < bd || (d == bd && (c & 1) == 0)) { bd = d; best = (uint8_t)c; }
    }
    return signbit(x) ? (uint8_t)(best | 0x80) : best;
}

static float f8_scale(float amax) { return amax > 0.0f ? amax / 448.0f : 1.0f; }

/* lifted activations (natural window order, as oracle_lift) quantised per
 * token: Q [T x ldq] codes, columns past the lifted width zero; scale [T] */
int oracle_quant_lift_f8(const uint16_t *X, int64_t T, int64_t K, int64_t ldx, int m, int64_t ldq, uint8_t *Q,
                         float *scale) {
    if (m < 4 || m % 2) return -1;
    const int Ns = m / 2;
    const int64_t G = groups_of(K, m);
    const int64_t KL = G * (Ns - 1) * 4;
    if (ldq < KL) return -1;
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            const float v = fabsf(bf16_to_f32(X[t * ldx + k]));
            if (v > amax) amax = v;
        }
        const float s = f8_scale(amax), inv = 1.0f / s;
        scale[t] = s;
        for (int64_t c = 0; c < ldq; ++c) Q[t * ldq + c] = 0;
        for (int64_t g = 0; g < G; ++g)
            for (int w = 0; w < Ns - 1; ++w)
                for (int c = 0; c < 4; ++c) {
                    const int64_t src = g * m + 2 * w + c;
                    const float v = src < K ? bf16_to_f32(X[t * ldx + src]) : 0.0f;
                    Q[t * ldq + g * (Ns - 1) * 4 + 4 * w + c] = oracle_e4m3_encode(v * inv);
                }
    }
    return 0;
}

/* kept weight values [R x L] (bf16) quantised per row: Q [R x L], scale [R] */
void oracle_quant_rows_f8(const uint16_t *V, int64_t R, int64_t L, uint8_t *Q, float *scale) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        float amax = 0.0f;
        for (int64_t j = 0; j < L; ++j) {
            const float v = fabsf(bf16_to_f32(V[r * L + j]));
            if (v > amax) amax = v;
        }
        const float s = f8_scale(amax), inv = 1.0f / s;
        scale[r] = s;
        for (int64_t j = 0; j < L; ++j) Q[r * L + j] = oracle_e4m3_encode(bf16_to_f32(V[r * L + j]) * inv);
    }
}

uint16_t oracle_f64_to_bf16(double v) { return f64_to_bf16_rne(v); }
