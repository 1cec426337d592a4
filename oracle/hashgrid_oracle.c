/*
 * hashgrid_oracle.c -- plain, slow, CPU-only oracle for the multiresolution hash-grid
 * encoding (Instant-NGP style), forward and backward.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check of the package entry file and
 * the CPU-baseline leg of the benchmark may load or call this code. The CUDA library shares
 * no code, header, table or constant with it, and neither side includes the other.
 *
 * Sources, cited by page and section (the pages are web articles; they print no worked
 * numbers, so every check of this file is self-made, see the test suite):
 *   [NeRFace-HG]  "NeRFace + Instant-NGP hash encoding" article (ipipp.com, 0929/63223),
 *                 section 2 (二, multiresolution feature grids): per-level table of T
 *                 F-wide learnable features, resolution growing geometrically from N_min to
 *                 N_max, voxel of x with its 8 corners, corner hash, trilinear interpolation,
 *                 concatenation of the L levels into an L*F vector; the backward pass only
 *                 updates the sampled features (end of section 2 and section 3, 三).
 *   [Repro-HG]    "Reproduce Instant-NGP's hash-encoding layer in PyTorch" (jsqmd.com,
 *                 news/998204): section 2.1 (level table: coarsest 16^3, finest 512^3,
 *                 T = 2^19, F = 2), section 2.2 (hash = XOR over axes of coordinate times a
 *                 per-axis prime, modulo T), section 3 (the layer), section 5 (half-precision
 *                 tables to save memory).
 *   [Overview-HG] Instant-NGP overview (ijyty.com, news/1538821), section 2.2: the hash
 *                 h(x) = (XOR_i x_i * pi_i) mod T.
 *
 * Readings taken where the pages are silent or disagree (each one is listed in the design
 * notes of the repository):
 *   - resolution: N_l is the exact-math value of N_min * b^l, floored (R1 below);
 *   - the point is scaled by N_l, not N_l - 1 (the NeRFace article's reading);
 *   - the hash is evaluated in unsigned 32-bit wraparound arithmetic; for a power-of-two T
 *     the "mod T" of the pages' 64-bit products keeps the same low bits;
 *   - every level is hashed, including coarse levels whose vertices would fit in T;
 *   - the offset along axis i is weighted by frac_i (true trilinear interpolation); the
 *     pages' own snippets pair the x fraction with the z offset, which is not trilinear;
 *   - the point is scaled in fp32 (the pages scale an fp32 coordinate tensor), so the voxel
 *     decision x*N_l -> floor is taken in fp32 on both sides; everything after that here
 *     is fp64.
 *
 * Corner numbering (shared convention of the C ABI, not arithmetic): corner c in 0..7 has
 * offsets d0 = c & 1 (x), d1 = (c >> 1) & 1 (y), d2 = (c >> 2) & 1 (z).
 *
 * Table layout: table[l][i][f] at element (l*T + i)*F + f.  Output layout: out[p][l*F + f].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_PRIME_X 1u
#define ORACLE_PRIME_Y 2654435761u
#define ORACLE_PRIME_Z 805459861u

/* ------------------------------------------------------------------------------------ */
/* Resolution schedule.                                                                   */
/* [NeRFace-HG] section 2: b = exp((ln N_max - ln N_min)/(L - 1)), N_l = floor(N_min b^l). */
/* [Repro-HG] section 2.1 prints 16^3 for the coarsest and 512^3 for the finest level.     */
/* R1: computed literally in double, N_min*b^l can land a few ulp below an integer that    */
/* it equals in exact arithmetic (16*b^15 = 4095.99999... for N_max = 4096), and the floor */
/* then loses one. The reading taken: when v is within 1e-9*v of an integer, that integer  */
/* is the exact value and is used; otherwise floor(v). With L = 1 the formula divides by   */
/* zero; the reading taken is b = 1, allowed only when N_min == N_max.                     */
/* Returns 0 on success, -1 on invalid arguments.                                          */
/* ------------------------------------------------------------------------------------ */
int oracle_resolutions(int L, int N_min, int N_max, int *res)
{
    if (L < 1 || N_min < 1 || N_max < N_min || res == NULL)
        return -1;
    if (L == 1) {
        if (N_min != N_max)
            return -1;
        res[0] = N_min;
        return 0;
    }
    double b = exp((log((double)N_max) - log((double)N_min)) / (double)(L - 1));
    for (int l = 0; l < L; ++l) {
        double v = (double)N_min * pow(b, (double)l);
        double r = nearbyint(v);
        if (fabs(v - r) <= 1e-9 * v)
            res[l] = (int)r;
        else
            res[l] = (int)floor(v);
    }
    return 0;
}

/* ------------------------------------------------------------------------------------ */
/* Spatial hash of one integer vertex.                                                    */
/* [NeRFace-HG] section 2 and [Repro-HG] section 2.2: each coordinate is multiplied by its */
/* axis prime (1, 2654435761, 805459861) and the products are XORed. [Overview-HG] §2.2    */
/* writes the same formula. Coordinates are taken modulo 2^32 (two's complement for        */
/* negative vertices) and the products wrap at 2^32.                                      */
/* ------------------------------------------------------------------------------------ */
uint32_t oracle_hash3(int64_t c0, int64_t c1, int64_t c2)
{
    uint32_t u0 = (uint32_t)c0, u1 = (uint32_t)c1, u2 = (uint32_t)c2;
    return (u0 * ORACLE_PRIME_X) ^ (u1 * ORACLE_PRIME_Y) ^ (u2 * ORACLE_PRIME_Z);
}

/* ------------------------------------------------------------------------------------ */
/* IEEE 754 binary16 -> double, from the format's definition (1 sign bit, 5 exponent bits */
/* with bias 15, 10 fraction bits; exponent 0 = subnormal m * 2^-24; exponent 31 = inf or */
/* NaN). [Repro-HG] section 5 suggests half-precision tables; their values are decoded     */
/* exactly here (every binary16 value is exact in double).                                 */
/* ------------------------------------------------------------------------------------ */
double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = (m == 0) ? INFINITY : NAN;
    else
        v = ldexp((double)(1024 + m), e - 25);
    return sign ? -v : v;
}

/* Table element as double. dtype 0 = fp32, 1 = fp16 bits. */
static double table_value(const void *table, int dtype, size_t elem)
{
    if (dtype == 0)
        return (double)((const float *)table)[elem];
    return oracle_half_to_double(((const uint16_t *)table)[elem]);
}

/* ------------------------------------------------------------------------------------ */
/* Voxel and fraction of one point at one level.                                         */
/* [NeRFace-HG] section 2: the point is scaled by the level's resolution, floored to the  */
/* voxel's lower vertex, and the remainder is the position inside the voxel. The scaling  */
/* is one fp32 multiply (the pages scale an fp32 tensor); the remainder xs - floor(xs) is */
/* exact in fp32.                                                                         */
/* ------------------------------------------------------------------------------------ */
static void locate(const float *xp, int res_l, int64_t v[3], double frac[3])
{
    for (int i = 0; i < 3; ++i) {
        float xs = xp[i] * (float)res_l;
        float fl = floorf(xs);
        v[i] = (int64_t)fl;
        frac[i] = (double)(xs - fl);
    }
}

/* Corner c of the voxel: its vertex and its trilinear weight (product over axes of       */
/* frac_i for offset 1 and 1 - frac_i for offset 0), [NeRFace-HG] section 2.              */
static double corner(const int64_t v[3], const double frac[3], int c, int64_t vc[3])
{
    double w = 1.0;
    for (int i = 0; i < 3; ++i) {
        int d = (c >> i) & 1;
        vc[i] = v[i] + d;
        w *= d ? frac[i] : 1.0 - frac[i];
    }
    return w;
}

/* ------------------------------------------------------------------------------------ */
/* Hash indices of every corner: idx[p][l][c] = hash(corner) mod T, T = 2^log2T.          */
/* Levels l0 <= l < l1 are written; idx has room for all L levels per point.             */
/* ------------------------------------------------------------------------------------ */
void oracle_indices(int L, int log2T, const int *res, const float *x, int64_t N,
                    int l0, int l1, uint32_t *idx)
{
    uint32_t mask = (uint32_t)((1ull << log2T) - 1ull);
    for (int64_t p = 0; p < N; ++p) {
        for (int l = l0; l < l1; ++l) {
            int64_t v[3], vc[3];
            double frac[3];
            locate(x + 3 * p, res[l], v, frac);
            for (int c = 0; c < 8; ++c) {
                (void)corner(v, frac, c, vc);
                idx[((size_t)p * L + l) * 8 + c] = oracle_hash3(vc[0], vc[1], vc[2]) & mask;
            }
        }
    }
}

/* ------------------------------------------------------------------------------------ */
/* Forward pass. [NeRFace-HG] section 2 and [Repro-HG] section 3:                         */
/*   out[p][l*F + f] = sum_c w_c * table[l][hash(corner_c) mod T][f]                      */
/* with the sum and weights in fp64. Levels l0 <= l < l1 are written (the rest of out is */
/* untouched). Parallel over points when nthreads > 1: every point is independent, so    */
/* the result does not depend on the thread count.                                        */
/* ------------------------------------------------------------------------------------ */
void oracle_forward(int L, int F, int log2T, const int *res, int dtype, const void *table,
                    const float *x, int64_t N, int l0, int l1, double *out, int nthreads)
{
    size_t T = (size_t)1 << log2T;
    uint32_t mask = (uint32_t)(T - 1);
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel for schedule(static) num_threads(nthreads)
    for (int64_t p = 0; p < N; ++p) {
        for (int l = l0; l < l1; ++l) {
            int64_t v[3], vc[3];
            double frac[3];
            double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            locate(x + 3 * p, res[l], v, frac);
            for (int c = 0; c < 8; ++c) {
                double w = corner(v, frac, c, vc);
                uint32_t h = oracle_hash3(vc[0], vc[1], vc[2]) & mask;
                for (int f = 0; f < F; ++f)
                    acc[f] += w * table_value(table, dtype, ((size_t)l * T + h) * F + f);
            }
            for (int f = 0; f < F; ++f)
                out[(size_t)p * L * F + (size_t)l * F + f] = acc[f];
        }
    }
}

/* ------------------------------------------------------------------------------------ */
/* Backward pass with respect to the tables. The forward pass is linear in the table, so */
/* each corner passes its weight times the upstream gradient to the entry it read; only  */
/* the sampled entries receive gradient ([NeRFace-HG] end of section 2 and section 3).   */
/*   dtable[l][hash(corner_c) mod T][f] += w_c * g[p][l*F + f]                            */
/* Accumulates into dtable (fp64, caller zeroes it). Within one level the order is p, c. */
/* Levels are disjoint slices, so running levels on separate threads gives the same bits */
/* as a serial run.                                                                      */
/* ------------------------------------------------------------------------------------ */
void oracle_backward(int L, int F, int log2T, const int *res, const float *x, const float *g,
                     int64_t N, int l0, int l1, double *dtable, int nthreads)
{
    size_t T = (size_t)1 << log2T;
    uint32_t mask = (uint32_t)(T - 1);
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int l = l0; l < l1; ++l) {
        for (int64_t p = 0; p < N; ++p) {
            int64_t v[3], vc[3];
            double frac[3];
            locate(x + 3 * p, res[l], v, frac);
            for (int c = 0; c < 8; ++c) {
                double w = corner(v, frac, c, vc);
                uint32_t h = oracle_hash3(vc[0], vc[1], vc[2]) & mask;
                for (int f = 0; f < F; ++f)
                    dtable[((size_t)l * T + h) * F + f] +=
                        w * (double)g[(size_t)p * L * F + (size_t)l * F + f];
            }
        }
    }
}

/* ------------------------------------------------------------------------------------ */
/* Backward pass with respect to the input coordinates. [NeRFace-HG] section 3 applies    */
/* the encoder to coordinates produced by a learned transform, which needs dL/dx. Inside */
/* the voxel that floor() selects, frac_i = x_i * N_l - v_i, so d frac_i / d x_i = N_l,  */
/* and the weight of corner c changes along axis i by                                    */
/*   d w_c / d x_i = N_l * (d_i ? +1 : -1) * prod_{j != i} (d_j ? frac_j : 1 - frac_j).  */
/* (On a voxel face the encoding is continuous but has a kink; this is the derivative    */
/* from the voxel that contains x, i.e. the one-sided derivative towards +x.)             */
/*   dL_dx[p][i] = sum_l sum_c sum_f dL_dout[p][l*F + f] * table[l][idx_c][f] * dw_c/dx_i */
/* Overwrites dx [N][3] (fp64). Levels l0 <= l < l1 are summed.                           */
/* ------------------------------------------------------------------------------------ */
void oracle_backward_x(int L, int F, int log2T, const int *res, int dtype, const void *table,
                       const float *x, const float *g, int64_t N, int l0, int l1, double *dx,
                       int nthreads)
{
    size_t T = (size_t)1 << log2T;
    uint32_t mask = (uint32_t)(T - 1);
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel for schedule(static) num_threads(nthreads)
    for (int64_t p = 0; p < N; ++p) {
        double acc[3] = {0.0, 0.0, 0.0};
        for (int l = l0; l < l1; ++l) {
            int64_t v[3], vc[3];
            double frac[3];
            locate(x + 3 * p, res[l], v, frac);
            for (int c = 0; c < 8; ++c) {
                (void)corner(v, frac, c, vc);
                uint32_t h = oracle_hash3(vc[0], vc[1], vc[2]) & mask;
                double ge = 0.0;  /* sum_f g * e_c[f] */
                for (int f = 0; f < F; ++f)
                    ge += (double)g[(size_t)p * L * F + (size_t)l * F + f] *
                          table_value(table, dtype, ((size_t)l * T + h) * F + f);
                for (int i = 0; i < 3; ++i) {
                    double dw = (double)res[l] * (((c >> i) & 1) ? 1.0 : -1.0);
                    for (int j = 0; j < 3; ++j) {
                        if (j == i)
                            continue;
                        dw *= ((c >> j) & 1) ? frac[j] : 1.0 - frac[j];
                    }
                    acc[i] += ge * dw;
                }
            }
        }
        for (int i = 0; i < 3; ++i)
            dx[3 * p + i] = acc[i];
    }
}

/* ------------------------------------------------------------------------------------ */
/* Sparse Adam step on the tables. [NeRFace-HG] sections 3 and 4: the tables are trained  */
/* with Adam, without weight decay, at a learning rate several times the MLP's; only the  */
/* sampled entries receive gradient in a step. [Overview-HG] sections 4-5: Adam, learning */
/* rate 1e-2 to 1e-3. Adam (Kingma and Ba), for step t >= 1:                               */
/*   m = b1 m + (1 - b1) g;  v = b2 v + (1 - b2) g^2;                                     */
/*   theta -= lr * (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps).                        */
/* Reading taken for "sparse": an element whose gradient is exactly zero was not sampled */
/* in this step and is left entirely unchanged (theta, m and v). All fp64.               */
/* param/m/v are updated in place (fp64 arrays of n elements).                           */
/* ------------------------------------------------------------------------------------ */
void oracle_adam_step(int64_t n, double *param, double *m, double *v, const float *grad,
                      int64_t step, double lr, double beta1, double beta2, double eps)
{
    double c1 = 1.0 - pow(beta1, (double)step);
    double c2 = 1.0 - pow(beta2, (double)step);
    for (int64_t i = 0; i < n; ++i) {
        double g = (double)grad[i];
        if (g == 0.0)
            continue;
        m[i] = beta1 * m[i] + (1.0 - beta1) * g;
        v[i] = beta2 * v[i] + (1.0 - beta2) * g * g;
        double mhat = m[i] / c1;
        double vhat = v[i] / c2;
        param[i] -= lr * mhat / (sqrt(vhat) + eps);
    }
}

/* ------------------------------------------------------------------------------------ */
/* bfloat16 -> double: the bf16 format is the upper 16 bits of an IEEE binary32 value.  */
/* ------------------------------------------------------------------------------------ */
double oracle_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------------------ */
/* Encoding followed by the small MLP that consumes it. [NeRFace-HG] section 3: a three- */
/* layer network of 64 units with ReLU after the hash features; [Repro-HG] section 4:     */
/* Linear(in, 64), ReLU, Linear(64, 64), ReLU, Linear(64, 4). Here in = L*F (the encoding */
/* alone; the pages' extra inputs -- expression code, raw x -- are the caller's):         */
/*   a1 = relu(W1 e + b1), a2 = relu(W2 a1 + b2), y = W3 a2 + b3                         */
/* Weights are bf16 bit patterns, row-major [out][in] (W1 [64][in], W2 [64][64],         */
/* W3 [4][64]), biases fp32; everything is evaluated in fp64 on the fp64 encoding.       */
/* y: [N][4] fp64.                                                                       */
/* ------------------------------------------------------------------------------------ */
void oracle_mlp_forward(int L, int F, int log2T, const int *res, int dtype, const void *table,
                        const float *x, int64_t N, const uint16_t *w1, const float *b1,
                        const uint16_t *w2, const float *b2, const uint16_t *w3, const float *b3,
                        double *y, int nthreads)
{
    const int in = L * F, hid = 64, nout = 4;
    double *e = (double *)malloc(sizeof(double) * (size_t)N * in);
    if (e == NULL)
        return;
    oracle_forward(L, F, log2T, res, dtype, table, x, N, 0, L, e, nthreads);
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel for schedule(static) num_threads(nthreads)
    for (int64_t p = 0; p < N; ++p) {
        double a1[64], a2[64];
        const double *ep = e + (size_t)p * in;
        for (int o = 0; o < hid; ++o) {
            double s = (double)b1[o];
            for (int k = 0; k < in; ++k)
                s += oracle_bf16_to_double(w1[o * in + k]) * ep[k];
            a1[o] = s > 0.0 ? s : 0.0;
        }
        for (int o = 0; o < hid; ++o) {
            double s = (double)b2[o];
            for (int k = 0; k < hid; ++k)
                s += oracle_bf16_to_double(w2[o * hid + k]) * a1[k];
            a2[o] = s > 0.0 ? s : 0.0;
        }
        for (int o = 0; o < nout; ++o) {
            double s = (double)b3[o];
            for (int k = 0; k < hid; ++k)
                s += oracle_bf16_to_double(w3[o * hid + k]) * a2[k];
            y[(size_t)p * nout + o] = s;
        }
    }
    free(e);
}

/* ------------------------------------------------------------------------------------ */
/* D-dimensional inputs. [Repro-HG] section 2.2 writes the hash for coordinates of any   */
/* dimension d as the XOR over axes of coordinate_i * pi_i, and section 3 lists the       */
/* primes (1, 2654435761, 805459861, 3674653429, 2097192037, 1434869437, 2165219737);    */
/* the encoding of a D-dimensional point interpolates the 2^D corners of its cell with   */
/* multilinear weights prod_i (d_i ? frac_i : 1 - frac_i). Corner c has offset bit i =   */
/* (c >> i) & 1. x is [N][D]. D = 3 reproduces the functions above.                       */
/* ------------------------------------------------------------------------------------ */
static const uint32_t ORACLE_PRIMES7[7] = {1u, 2654435761u, 805459861u, 3674653429u,
                                           2097192037u, 1434869437u, 2165219737u};

uint32_t oracle_hash_nd(int D, const int64_t *c)
{
    uint32_t h = 0;
    for (int i = 0; i < D; ++i)
        h ^= (uint32_t)c[i] * ORACLE_PRIMES7[i];
    return h;
}

static void locate_nd(int D, const float *xp, int res_l, int64_t *v, double *frac)
{
    for (int i = 0; i < D; ++i) {
        float xs = xp[i] * (float)res_l;
        float fl = floorf(xs);
        v[i] = (int64_t)fl;
        frac[i] = (double)(xs - fl);
    }
}

static double corner_nd(int D, const int64_t *v, const double *frac, int c, int64_t *vc)
{
    double w = 1.0;
    for (int i = 0; i < D; ++i) {
        int d = (c >> i) & 1;
        vc[i] = v[i] + d;
        w *= d ? frac[i] : 1.0 - frac[i];
    }
    return w;
}

void oracle_indices_nd(int D, int L, int log2T, const int *res, const float *x, int64_t N, uint32_t *idx)
{
    uint32_t mask = (uint32_t)((1ull << log2T) - 1ull);
    int nc = 1 << D;
    for (int64_t p = 0; p < N; ++p)
        for (int l = 0; l < L; ++l) {
            int64_t v[7], vc[7];
            double frac[7];
            locate_nd(D, x + (size_t)D * p, res[l], v, frac);
            for (int c = 0; c < nc; ++c) {
                (void)corner_nd(D, v, frac, c, vc);
                idx[((size_t)p * L + l) * nc + c] = oracle_hash_nd(D, vc) & mask;
            }
        }
}

void oracle_forward_nd(int D, int L, int F, int log2T, const int *res, int dtype, const void *table,
                       const float *x, int64_t N, double *out, int nthreads)
{
    size_t T = (size_t)1 << log2T;
    uint32_t mask = (uint32_t)(T - 1);
    int nc = 1 << D;
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel for schedule(static) num_threads(nthreads)
    for (int64_t p = 0; p < N; ++p)
        for (int l = 0; l < L; ++l) {
            int64_t v[7], vc[7];
            double frac[7], acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            locate_nd(D, x + (size_t)D * p, res[l], v, frac);
            for (int c = 0; c < nc; ++c) {
                double w = corner_nd(D, v, frac, c, vc);
                uint32_t h = oracle_hash_nd(D, vc) & mask;
                for (int f = 0; f < F; ++f)
                    acc[f] += w * table_value(table, dtype, ((size_t)l * T + h) * F + f);
            }
            for (int f = 0; f < F; ++f)
                out[(size_t)p * L * F + (size_t)l * F + f] = acc[f];
        }
}

void oracle_backward_nd(int D, int L, int F, int log2T, const int *res, const float *x, const float *g,
                        int64_t N, double *dtable, int nthreads)
{
    size_t T = (size_t)1 << log2T;
    uint32_t mask = (uint32_t)(T - 1);
    int nc = 1 << D;
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int l = 0; l < L; ++l)
        for (int64_t p = 0; p < N; ++p) {
            int64_t v[7], vc[7];
            double frac[7];
            locate_nd(D, x + (size_t)D * p, res[l], v, frac);
            for (int c = 0; c < nc; ++c) {
                double w = corner_nd(D, v, frac, c, vc);
                uint32_t h = oracle_hash_nd(D, vc) & mask;
                for (int f = 0; f < F; ++f)
                    dtable[((size_t)l * T + h) * F + f] += w * (double)g[(size_t)p * L * F + (size_t)l * F + f];
            }
        }
}

/* dL/dx_i = sum_l N_l sum_c (sum_f g e_c[f]) (d_i ? +1 : -1) prod_{j != i} (d_j ? frac_j : 1 - frac_j) */
void oracle_backward_x_nd(int D, int L, int F, int log2T, const int *res, int dtype, const void *table,
                          const float *x, const float *g, int64_t N, double *dx, int nthreads)
{
    size_t T = (size_t)1 << log2T;
    uint32_t mask = (uint32_t)(T - 1);
    int nc = 1 << D;
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel for schedule(static) num_threads(nthreads)
    for (int64_t p = 0; p < N; ++p) {
        double acc[7] = {0, 0, 0, 0, 0, 0, 0};
        for (int l = 0; l < L; ++l) {
            int64_t v[7], vc[7];
            double frac[7];
            locate_nd(D, x + (size_t)D * p, res[l], v, frac);
            for (int c = 0; c < nc; ++c) {
                (void)corner_nd(D, v, frac, c, vc);
                uint32_t h = oracle_hash_nd(D, vc) & mask;
                double ge = 0.0;
                for (int f = 0; f < F; ++f)
                    ge += (double)g[(size_t)p * L * F + (size_t)l * F + f] *
                          table_value(table, dtype, ((size_t)l * T + h) * F + f);
                for (int i = 0; i < D; ++i) {
                    double dw = (double)res[l] * (((c >> i) & 1) ? 1.0 : -1.0);
                    for (int j = 0; j < D; ++j)
                        if (j != i)
                            dw *= ((c >> j) & 1) ? frac[j] : 1.0 - frac[j];
                    acc[i] += ge * dw;
                }
            }
        }
        for (int i = 0; i < D; ++i)
            dx[(size_t)D * p + i] = acc[i];
    }
}
