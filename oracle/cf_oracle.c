/*
 * cf_oracle.c -- plain CPU oracle of the residual-compression activation codec.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously correct
 * statement of what the codec computes.  Only the tests, the smoke check and
 * the CPU-baseline leg of the benchmark load it; the product path never does.
 * It shares no code, header, table or constant generator with the CUDA path.
 *
 * Sources (page title, then section):
 *  - "Accelerating Parallel Diffusion Model Serving with Residual Compression"
 *    (arXiv 2507.17511), abstract: only the compressed difference between an
 *    activation and its value at the previous denoising step is sent, and a
 *    cheap error-feedback term keeps compression error from building up.
 *  - Same paper, reproducibility table, "Dataset Splits" row (Appendix D,
 *    Figure 8): a 1-step uncompressed warmup initialises the base tensor used
 *    for later residuals.
 *  - Same paper, reproducibility table, "Pseudocode" row, Algorithm 3
 *    (Subspace Iteration, rank r): random start Q, orthonormalise; T times
 *    Z = A^T A Q then orthonormalise; U = A Q, orthonormalise U; V = Q.
 *  - xDiT issue 573 ("Proposal: Integrating a compression-based acceleration
 *    method into xDiT"): compressed residuals plus error feedback cut
 *    communication 8-16x.
 *
 * The pages give no quantiser formula.  The readings taken here (symmetric
 * per-group absmax with L = 2^(k-1)-1 levels each side, scaled sign with the
 * mean |A| scale for k = 1, LSB-first bit packing, fp32 group scales, RNE,
 * no FMA) are the plainest ones the pages support; every floating-point
 * operation of the quantised path is a single IEEE-754 binary32 operation,
 * so the CUDA path must reproduce codes, scales, E, base and C bit for bit.
 * Build flags: -O2 -ffp-contract=off -fno-fast-math (no contraction, no
 * reassociation).
 *
 * Parity pins: every function here is checked in tests/ against closed forms,
 * invariants, hand-worked groups and library routines (numpy SVD); none is
 * "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define CFO_OK 0
#define CFO_E_ARG 1
#define CFO_E_NOMEM 5
#define CFO_FLAG_NONFINITE 0x1u

/* A group whose scale is below 2^-120 is an all-zero group: this keeps
 * L / s finite for every k (L <= 7). */
static const float CFO_SCALE_MIN = 7.52316384526264e-37f; /* 2^-120 */

/* ---------------------------------------------------------------- bf16 -- */

static float bf16_to_float(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a float to bf16 with round-to-nearest-even on the 16 dropped bits
 * (a NaN stays a quiet NaN). */
static uint16_t float_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
    const uint32_t lsb = (u >> 16) & 1u;
    return (uint16_t)((u + 0x7fffu + lsb) >> 16);
}

/* bf16 copy of the receiver's reconstruction, for a consumer that reads K or
 * V in bf16: out[i] = float_to_bf16(in[i]). */
int cfo_to_bf16(int64_t n, const float *in, uint16_t *out)
{
    if (n < 0 || (n > 0 && (!in || !out))) return CFO_E_ARG;
    for (int64_t i = 0; i < n; ++i) out[i] = float_to_bf16(in[i]);
    return CFO_OK;
}

/* ------------------------------------------------------- bit stream ----- */

/* The payload is one bit stream per slot, bytes in increasing address order,
 * least significant bit first: the code of element i occupies bits
 * [i*k, i*k + k).  Group g therefore starts at byte g*G*k/8. */
static void put_code(uint8_t *stream, int64_t i, int k, unsigned code)
{
    for (int b = 0; b < k; ++b) {
        int64_t bit = i * k + b;
        if ((code >> b) & 1u)
            stream[bit >> 3] |= (uint8_t)(1u << (bit & 7));
        else
            stream[bit >> 3] &= (uint8_t)~(1u << (bit & 7));
    }
}

static unsigned get_code(const uint8_t *stream, int64_t i, int k)
{
    unsigned code = 0;
    for (int b = 0; b < k; ++b) {
        int64_t bit = i * k + b;
        code |= ((unsigned)(stream[bit >> 3] >> (bit & 7)) & 1u) << b;
    }
    return code;
}

int cfo_put_code(uint8_t *stream, int64_t i, int k, unsigned code)
{
    if (k != 1 && k != 2 && k != 4) return CFO_E_ARG;
    put_code(stream, i, k, code);
    return CFO_OK;
}

int cfo_get_code(const uint8_t *stream, int64_t i, int k, unsigned *code)
{
    if (k != 1 && k != 2 && k != 4) return CFO_E_ARG;
    *code = get_code(stream, i, k);
    return CFO_OK;
}

/* ----------------------------------------------------------- levels ----- */

static int half_levels(int k) { return k >= 2 ? (1 << (k - 1)) - 1 : 1; }

/* Dequantised level of code c: t_c = (c - L) / L, one correctly rounded
 * division. */
static float level(unsigned c, int L) { return (float)((int)c - L) / (float)L; }

/* Perfect binary-tree sum: sum(v, n) = sum(left half) + sum(right half). */
static float tree_sum(const float *v, int n)
{
    if (n == 1) return v[0];
    float left = tree_sum(v, n / 2);
    float right = tree_sum(v + n / 2, n / 2);
    return left + right;
}

static int valid_quant(int64_t n, int k, int G)
{
    if (n < 0) return 0;
    if (k != 1 && k != 2 && k != 4) return 0;
    if (G < 8 || G > 256 || (G & (G - 1)) != 0) return 0;
    if (n % G != 0) return 0;
    return 1;
}

/* ------------------------------------------------------ warmup (t=0) ---- */

/* Sender side of the 1-step warmup: the uncompressed X_0 becomes the base
 * tensor and the error-feedback buffer starts at zero. */
int cfo_warmup_sender(int64_t n, const uint16_t *x, uint16_t *base, float *err)
{
    if (n < 0) return CFO_E_ARG;
    for (int64_t i = 0; i < n; ++i) {
        base[i] = x[i];
        err[i] = 0.0f;
    }
    return CFO_OK;
}

/* Receiver side of the warmup: the raw X_0 seeds the reconstruction cache. */
int cfo_warmup_receiver(int64_t n, const uint16_t *x, float *cache)
{
    if (n < 0) return CFO_E_ARG;
    for (int64_t i = 0; i < n; ++i) cache[i] = bf16_to_float(x[i]);
    return CFO_OK;
}

/* ------------------------------------------------------ residual + EF --- */

/* A = (X_t - X_{t-1}) + E_{t-1}: the step-wise difference against the base
 * tensor plus the carried error; the base then advances to X_t. */
int cfo_residual(int64_t n, const uint16_t *x, uint16_t *base, const float *err, float *a_out)
{
    if (n < 0) return CFO_E_ARG;
    for (int64_t i = 0; i < n; ++i) {
        float diff = bf16_to_float(x[i]) - bf16_to_float(base[i]);
        a_out[i] = diff + err[i];
        base[i] = x[i];
    }
    return CFO_OK;
}

/* ------------------------------------------------- quantised compress --- */

/* Quantise one group of G residual values a[0..G).  Writes codes into the
 * slot's bit stream at element offset i0, returns the scale, and leaves the
 * local dequantised values in d[0..G).  *flags gets CFO_FLAG_NONFINITE for a
 * group whose scale is not finite (then the group is sent as all-zero). */
static float quantise_group(const float *a, int G, int k, int sign_scale,
                            uint8_t *codes, int64_t i0, float *d, uint32_t *flags)
{
    const int L = half_levels(k);
    float s;
    if (k == 1 && sign_scale == 0) {
        float absval[256];
        for (int j = 0; j < G; ++j) absval[j] = fabsf(a[j]);
        s = tree_sum(absval, G) / (float)G;
    } else {
        s = 0.0f;
        for (int j = 0; j < G; ++j) {
            float m = fabsf(a[j]);
            /* NaN compares false, so test it explicitly: the scale must
             * report a non-finite input. */
            if (m != m || m > s) s = m;
            if (s != s) break;
        }
    }

    int zero_group = 0;
    if (!isfinite(s)) {
        *flags |= CFO_FLAG_NONFINITE;
        zero_group = 1;
    } else if (s < CFO_SCALE_MIN) {
        zero_group = 1;
    }
    if (zero_group) {
        const unsigned zc = (k == 1) ? 1u : (unsigned)L;
        for (int j = 0; j < G; ++j) {
            put_code(codes, i0 + j, k, zc);
            d[j] = 0.0f;
        }
        return 0.0f;
    }

    if (k == 1) {
        for (int j = 0; j < G; ++j) {
            unsigned c = (a[j] >= 0.0f) ? 1u : 0u;
            put_code(codes, i0 + j, k, c);
            d[j] = c ? s : -s;
        }
    } else {
        const float inv = (float)L / s;
        for (int j = 0; j < G; ++j) {
            float y = a[j] * inv;
            float r = rintf(y); /* round half to even (default mode) */
            int q = (int)r;
            if (q > L) q = L;
            if (q < -L) q = -L;
            unsigned c = (unsigned)(q + L);
            put_code(codes, i0 + j, k, c);
            d[j] = level(c, L) * s;
        }
    }
    return s;
}

/* Sender, step t >= 1: residual + EF, per-group quantise, pack, local
 * dequantise, new error E = A - d, base <- X_t.  Returns flags. */
int cfo_compress(int64_t n, int k, int G, int sign_scale, const uint16_t *x, uint16_t *base,
                 float *err, uint8_t *codes, float *scales, uint32_t *flags_out)
{
    if (!valid_quant(n, k, G) || (sign_scale != 0 && sign_scale != 1)) return CFO_E_ARG;
    uint32_t flags = 0;
    float a[256], d[256];
    for (int64_t g = 0; g < n / G; ++g) {
        const int64_t i0 = g * G;
        for (int j = 0; j < G; ++j) {
            float diff = bf16_to_float(x[i0 + j]) - bf16_to_float(base[i0 + j]);
            a[j] = diff + err[i0 + j];
            base[i0 + j] = x[i0 + j];
        }
        scales[g] = quantise_group(a, G, k, sign_scale, codes, i0, d, &flags);
        for (int j = 0; j < G; ++j) err[i0 + j] = a[j] - d[j];
    }
    if (flags_out) *flags_out = flags;
    return CFO_OK;
}

/* Receiver, step t >= 1: unpack, dequantise, accumulate into the cache. */
int cfo_decompress(int64_t n, int k, int G, const uint8_t *codes, const float *scales, float *cache)
{
    if (!valid_quant(n, k, G)) return CFO_E_ARG;
    const int L = half_levels(k);
    for (int64_t g = 0; g < n / G; ++g) {
        const float s = scales[g];
        for (int j = 0; j < G; ++j) {
            const int64_t i = g * G + j;
            const unsigned c = get_code(codes, i, k);
            float dv;
            if (k == 1)
                dv = c ? s : -s;
            else
                dv = level(c, L) * s;
            cache[i] = cache[i] + dv;
        }
    }
    return CFO_OK;
}

/* Bytes of one quantised payload: codes plus fp32 group scales. */
int64_t cfo_payload_bytes(int64_t n, int k, int G)
{
    if (!valid_quant(n, k, G)) return -1;
    return n * k / 8 + 4 * (n / G);
}

/* ============================================ low-rank (fp64 answer) ==== */

/* CholeskyQR of a tall block Z (rows x r, row-major, fp64):
 *   G = Z^T Z, R = chol(G) upper with G = R^T R, Q = Z R^{-1}.
 * Q may alias Z.  Returns CFO_E_ARG if G is not positive definite. */
int cfo_cholqr(int64_t rows, int r, const double *Z, double *Q, double *R)
{
    if (rows < r || r < 1 || r > 64) return CFO_E_ARG;
    double *Gm = (double *)calloc((size_t)r * r, sizeof(double));
    if (!Gm) return CFO_E_NOMEM;
    for (int64_t i = 0; i < rows; ++i)
        for (int p = 0; p < r; ++p)
            for (int q = 0; q < r; ++q) Gm[p * r + q] += Z[i * r + p] * Z[i * r + q];

    /* Upper Cholesky: R[p][p] = sqrt(G[p][p] - sum_k R[k][p]^2),
     * R[p][q] = (G[p][q] - sum_k R[k][p] R[k][q]) / R[p][p]. */
    memset(R, 0, sizeof(double) * (size_t)r * r);
    for (int p = 0; p < r; ++p) {
        double diag = Gm[p * r + p];
        for (int k = 0; k < p; ++k) diag -= R[k * r + p] * R[k * r + p];
        if (!(diag > 0.0)) {
            free(Gm);
            return CFO_E_ARG;
        }
        R[p * r + p] = sqrt(diag);
        for (int q = p + 1; q < r; ++q) {
            double v = Gm[p * r + q];
            for (int k = 0; k < p; ++k) v -= R[k * r + p] * R[k * r + q];
            R[p * r + q] = v / R[p * r + p];
        }
    }
    free(Gm);

    /* Q = Z R^{-1}: each row q solves q R = z by forward substitution. */
    for (int64_t i = 0; i < rows; ++i) {
        double row[64];
        for (int c = 0; c < r; ++c) {
            double v = Z[i * r + c];
            for (int k = 0; k < c; ++k) v -= row[k] * R[k * r + c];
            row[c] = v / R[c * r + c];
        }
        for (int c = 0; c < r; ++c) Q[i * r + c] = row[c];
    }
    return CFO_OK;
}

/* P = A Q  (A: m x n fp32 row-major, Q: n x r fp64, P: m x r fp64). */
static void mat_AQ(int64_t m, int64_t n, int r, const float *A, const double *Q, double *P)
{
    for (int64_t i = 0; i < m; ++i) {
        double acc[64];
        for (int c = 0; c < r; ++c) acc[c] = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            const double aij = (double)A[i * n + j];
            for (int c = 0; c < r; ++c) acc[c] += aij * Q[j * r + c];
        }
        for (int c = 0; c < r; ++c) P[i * r + c] = acc[c];
    }
}

/* Z = A^T P  (Z: n x r fp64). */
static void mat_AtP(int64_t m, int64_t n, int r, const float *A, const double *P, double *Z)
{
    memset(Z, 0, sizeof(double) * (size_t)n * r);
    for (int64_t i = 0; i < m; ++i)
        for (int64_t j = 0; j < n; ++j) {
            const double aij = (double)A[i * n + j];
            for (int c = 0; c < r; ++c) Z[j * r + c] += aij * P[i * r + c];
        }
}

/* Algorithm 3 (subspace iteration, rank r, T iterations), orthogonalisation
 * by CholeskyQR:
 *   Q = orth(Q0);  repeat T: Z = A^T (A Q), Q = orth(Z);
 *   P = A Q;  (U, R) = CholeskyQR(P);  V = Q.
 * The reconstruction is D = U R V^T (= A Q Q^T).  Outputs are fp64. */
int cfo_subspace_iteration(int64_t m, int64_t n, int r, int T, const float *A, const float *Q0,
                           double *U, double *R, double *V)
{
    if (r < 1 || r > 64 || m < r || n < r || T < 0) return CFO_E_ARG;
    double *Q = (double *)malloc(sizeof(double) * (size_t)n * r);
    double *P = (double *)malloc(sizeof(double) * (size_t)m * r);
    double *Rs = (double *)malloc(sizeof(double) * (size_t)r * r);
    if (!Q || !P || !Rs) {
        free(Q); free(P); free(Rs);
        return CFO_E_NOMEM;
    }
    int rc = CFO_OK;
    for (int64_t i = 0; i < n * r; ++i) Q[i] = (double)Q0[i];
    rc = cfo_cholqr(n, r, Q, Q, Rs);
    for (int t = 0; t < T && rc == CFO_OK; ++t) {
        mat_AQ(m, n, r, A, Q, P);
        mat_AtP(m, n, r, A, P, Q);
        rc = cfo_cholqr(n, r, Q, Q, Rs);
    }
    if (rc == CFO_OK) {
        mat_AQ(m, n, r, A, Q, P);
        rc = cfo_cholqr(m, r, P, U, R);
        memcpy(V, Q, sizeof(double) * (size_t)n * r);
    }
    free(Q); free(P); free(Rs);
    return rc;
}

/* Low-rank apply: D = U (R V^T); E = A - D (if E); C_out = C_in + D (if C).
 * All outputs fp64 [m, n]; C_in is fp32. */
int cfo_lowrank_apply(int64_t m, int64_t n, int r, const float *A, const double *U, const double *R,
                      const double *V, double *D, double *E, const float *C_in, double *C_out)
{
    if (r < 1 || r > 64) return CFO_E_ARG;
    double *W = (double *)malloc(sizeof(double) * (size_t)r * n); /* W = R V^T, r x n */
    if (!W) return CFO_E_NOMEM;
    for (int p = 0; p < r; ++p)
        for (int64_t j = 0; j < n; ++j) {
            double v = 0.0;
            for (int q = 0; q < r; ++q) v += R[p * r + q] * V[j * r + q];
            W[p * n + j] = v;
        }
    for (int64_t i = 0; i < m; ++i)
        for (int64_t j = 0; j < n; ++j) {
            double dv = 0.0;
            for (int p = 0; p < r; ++p) dv += U[i * r + p] * W[p * n + j];
            if (D) D[i * n + j] = dv;
            if (E) E[i * n + j] = (double)A[i * n + j] - dv;
            if (C_out) C_out[i * n + j] = (double)C_in[i * n + j] + dv;
        }
    free(W);
    return CFO_OK;
}

/* ======================================== lean state (bf16 E and C) ==== */
/* The same codec with the error-feedback buffer E and the receiver cache C
 * kept in bf16: every arithmetic step stays one binary32 operation, and the
 * new E and C are rounded to bf16 (RNE) when they are stored.  The payload
 * (codes, scales) is the same as in the fp32-state codec for the same A. */

int cfo_warmup_sender_lean(int64_t n, const uint16_t *x, uint16_t *base, uint16_t *err)
{
    if (n < 0) return CFO_E_ARG;
    for (int64_t i = 0; i < n; ++i) {
        base[i] = x[i];
        err[i] = 0;
    }
    return CFO_OK;
}

int cfo_warmup_receiver_lean(int64_t n, const uint16_t *x, uint16_t *cache)
{
    if (n < 0) return CFO_E_ARG;
    for (int64_t i = 0; i < n; ++i) cache[i] = x[i];
    return CFO_OK;
}

int cfo_compress_lean(int64_t n, int k, int G, int sign_scale, const uint16_t *x, uint16_t *base, uint16_t *err,
                      uint8_t *codes, float *scales, uint32_t *flags_out)
{
    if (!valid_quant(n, k, G) || (sign_scale != 0 && sign_scale != 1)) return CFO_E_ARG;
    uint32_t flags = 0;
    float a[256], d[256];
    for (int64_t g = 0; g < n / G; ++g) {
        const int64_t i0 = g * G;
        for (int j = 0; j < G; ++j) {
            float diff = bf16_to_float(x[i0 + j]) - bf16_to_float(base[i0 + j]);
            a[j] = diff + bf16_to_float(err[i0 + j]);
            base[i0 + j] = x[i0 + j];
        }
        scales[g] = quantise_group(a, G, k, sign_scale, codes, i0, d, &flags);
        for (int j = 0; j < G; ++j) err[i0 + j] = float_to_bf16(a[j] - d[j]);
    }
    if (flags_out) *flags_out = flags;
    return CFO_OK;
}

int cfo_decompress_lean(int64_t n, int k, int G, const uint8_t *codes, const float *scales, uint16_t *cache)
{
    if (!valid_quant(n, k, G)) return CFO_E_ARG;
    const int L = half_levels(k);
    for (int64_t g = 0; g < n / G; ++g) {
        const float s = scales[g];
        for (int j = 0; j < G; ++j) {
            const int64_t i = g * G + j;
            const unsigned c = get_code(codes, i, k);
            const float dv = (k == 1) ? (c ? s : -s) : level(c, L) * s;
            cache[i] = float_to_bf16(bf16_to_float(cache[i]) + dv);
        }
    }
    return CFO_OK;
}

/* ------------------------------------------------------------ attention -- */

/* "Accelerating Parallel Diffusion Model Serving with Residual Compression",
 * reproducibility table, "Pseudocode" row, Algorithms 1 and 2: each device
 * attends with its queries over the key/value blocks it receives.  Standard
 * scaled dot-product attention per head of 64 channels (channels
 * [64 h, 64 h + 64) of the token-major layout), in fp64:
 *   score(i, j) = (q_i . k_j) / 8          (8 = sqrt(64))
 *   w(i, j)     = exp(score(i, j) - max_j score(i, j)) / sum_j (same)
 *   out(i, c)   = sum_j w(i, j) v(j, c)
 *   lse(i)      = log sum_j exp(score(i, j))   (if lse is not NULL)
 * The log-sum-exp of a row is what merges partial results over several K/V
 * blocks (ring attention, Algorithm 2): the softmax over their union weighs
 * each block's output by exp(lse_block - lse_union).
 * q, k, v are bf16 bit patterns; out is fp64 [lq x cols], lse fp64
 * [lq x cols / 64] (query-major). */
int cfo_attention(int64_t lq, int64_t lk, int64_t cols, const uint16_t *q, const uint16_t *k, const uint16_t *v,
                  double *out, double *lse)
{
    if (lq < 0 || lk < 1 || cols < 64 || cols % 64 != 0) return CFO_E_ARG;
    double *w = (double *)malloc((size_t)lk * sizeof(double));
    if (!w) return CFO_E_NOMEM;
    for (int64_t h = 0; h < cols / 64; ++h) {
        const int64_t c0 = h * 64;
        for (int64_t i = 0; i < lq; ++i) {
            double mx = -INFINITY;
            for (int64_t j = 0; j < lk; ++j) {
                double s = 0.0;
                for (int c = 0; c < 64; ++c)
                    s += (double)bf16_to_float(q[i * cols + c0 + c]) * (double)bf16_to_float(k[j * cols + c0 + c]);
                w[j] = s / 8.0;
                if (w[j] > mx) mx = w[j];
            }
            double z = 0.0;
            for (int64_t j = 0; j < lk; ++j) {
                w[j] = exp(w[j] - mx);
                z += w[j];
            }
            for (int c = 0; c < 64; ++c) {
                double o = 0.0;
                for (int64_t j = 0; j < lk; ++j) o += w[j] * (double)bf16_to_float(v[j * cols + c0 + c]);
                out[i * cols + c0 + c] = o / z;
            }
            if (lse) lse[i * (cols / 64) + h] = mx + log(z);
        }
    }
    free(w);
    return CFO_OK;
}
