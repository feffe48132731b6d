/*
 * grinqh_oracle.c -- TEST INFRASTRUCTURE, not part of the product.
 *
 * A plain, slow, obviously correct CPU restatement (fp64) of the GRINQH
 * batch-1 decode path: precision assignment, per-plane row lists, bit-plane
 * packing/unpacking, weight reconstruction with the midpoint truncation-bias
 * correction, and the GEMV y = W_hat^T x.  Only tests/, the smoke check of
 * __graft_entry__ and the cpu_baseline / reference legs of bench.py may load
 * this library.  It shares no code, header or table with the CUDA library.
 *
 * Sources (the pages' own words are not quoted; each step is restated):
 *   [KD1] "GRINQH: Graded Input-Based Quantization Hierarchy for Efficient LLM
 *         Generation" (papernotes summary), section "Key design 1: dynamic
 *         activation-graded precision mapping", the b_i equation.
 *   [KD2] same page, "Key design 2: hierarchical bit-plane interleaved storage
 *         and sparse memory access".
 *   [KD3] same page, "Key design 3: midpoint truncation-bias correction", the
 *         w_hat equation and the definition of phi.
 *   [FW]  same page, "Method / overall framework" (assignment -> plane load ->
 *         on-chip reconstruction -> GEMV).
 *
 * Readings where the pages are silent or garbled (each one is listed in the
 * design notes of the repository):
 *   R1  Theta has P = b_max/2 increasing entries theta_1..theta_P; level k
 *       (bit width 2k) covers |x| in [theta_k, theta_{k+1}) with theta_0 = 0,
 *       theta_{P+1} = +inf.  Equivalently b = 2 * #{k : theta_k <= |x|}.
 *   R2  Intervals are closed on the left: |x| == theta_k takes the higher level.
 *   R3  -0 -> |x| = 0; +-Inf -> b_max; NaN -> b = 0 (every comparison false).
 *   R4  phi_b = 2^(b_max-b-1) for b < b_max and phi_{b_max} = 0 (nothing is
 *       truncated at full width, so no midpoint shift is applied).
 *   R5  s and z are fp16 per (128-row group, output channel); z is an additive
 *       float offset: w_hat = s * (Q + phi) + z.
 *   R6  Field t (0..15) of word j of a (row, plane) region holds output 16j+t
 *       in bits [2t+1 : 2t]; plane 0 is the most significant 2-bit slice; the
 *       region of (row i, plane p) starts at word (i*P + p) * d_out/16.
 *   R7  List p holds, in ascending order, every row i with b_i > 2p.
 *   R8  Rows with b_i = 0 contribute nothing to y (not even z).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_GROUP 128

/* fp16 bit pattern -> double, written from the IEEE-754 binary16 definition:
 * 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_f16_to_f64(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24); /* subnormal: f * 2^-14 * 2^-10 */
    } else if (e == 31) {
        v = (f == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(1024 + f), e - 25); /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* [KD3] with reading R4: phi for level k (bit width b = 2k), k = 0..P.
 * phi[0] is never used (a b = 0 row is skipped) and is set to 0. */
void oracle_phi_default(int b_max, double *phi) {
    int P = b_max / 2;
    phi[0] = 0.0;
    for (int k = 1; k <= P; k++) {
        int b = 2 * k;
        phi[k] = (b < b_max) ? ldexp(1.0, b_max - b - 1) : 0.0;
    }
}

/* [KD1] with readings R1-R3: b_i = 2 * #{k in 1..P : theta_k <= |x_i|}.
 * The comparison is made in double on exactly converted fp16/fp32 values,
 * which is the same decision as an fp32 comparison. */
void oracle_assign(const uint16_t *x, const float *theta, int d_in, int b_max,
                   uint8_t *b) {
    int P = b_max / 2;
    for (int i = 0; i < d_in; i++) {
        double a = fabs(oracle_f16_to_f64(x[i]));
        int count = 0;
        for (int k = 0; k < P; k++) {
            if ((double)theta[k] <= a) count++;
        }
        b[i] = (uint8_t)(2 * count);
    }
}

/* Reading R7: list p = ascending rows with b_i > 2p; counts[p] = its length.
 * lists is [P][d_in]; entries past counts[p] are left untouched. */
void oracle_lists(const uint8_t *b, int d_in, int b_max, int32_t *lists,
                  int32_t *counts) {
    int P = b_max / 2;
    for (int p = 0; p < P; p++) {
        int n = 0;
        for (int i = 0; i < d_in; i++) {
            if (b[i] > 2 * p) {
                lists[(size_t)p * d_in + n] = i;
                n++;
            }
        }
        counts[p] = n;
    }
}

/* [KD2] with reading R6, one bit at a time: plane p of a code q is the 2-bit
 * slice (q >> 2(P-1-p)) & 3; field t of word j of region (i, p) is that
 * slice of output 16j+t. */
void oracle_pack(const uint8_t *q, int d_in, int d_out, int b_max,
                 uint32_t *planes) {
    int P = b_max / 2;
    int W = d_out / 16;
    for (int i = 0; i < d_in; i++) {
        for (int p = 0; p < P; p++) {
            for (int j = 0; j < W; j++) {
                uint32_t word = 0;
                for (int t = 0; t < 16; t++) {
                    int code = q[(size_t)i * d_out + 16 * j + t];
                    for (int bit = 0; bit < 2; bit++) {
                        int src = 2 * (P - 1 - p) + bit; /* bit of the code */
                        int dst = 2 * t + bit;           /* bit of the word */
                        if ((code >> src) & 1) word |= (uint32_t)1 << dst;
                    }
                }
                planes[((size_t)i * P + p) * W + j] = word;
            }
        }
    }
}

/* Inverse of oracle_pack, one bit at a time. */
void oracle_unpack(const uint32_t *planes, int d_in, int d_out, int b_max,
                   uint8_t *q) {
    int P = b_max / 2;
    int W = d_out / 16;
    for (int i = 0; i < d_in; i++) {
        for (int o = 0; o < d_out; o++) {
            int code = 0;
            for (int p = 0; p < P; p++) {
                uint32_t word = planes[((size_t)i * P + p) * W + o / 16];
                for (int bit = 0; bit < 2; bit++) {
                    int src = 2 * (o % 16) + bit;
                    int dst = 2 * (P - 1 - p) + bit;
                    if ((word >> src) & 1) code |= 1 << dst;
                }
            }
            q[(size_t)i * d_out + o] = (uint8_t)code;
        }
    }
}

/* [KD2]: the truncated code q_b of row i, output o, read from the packed
 * planes: only the first b/2 planes are read (the rest are never touched), and
 * each 2-bit slice is put back at its significance 4^(P-1-p).  The result is
 * the integer q_b * 2^(b_max-b) of [KD3]. */
static double truncated_code(const uint32_t *planes, int i, int o, int b,
                             int P, int W) {
    double Q = 0.0;
    for (int p = 0; p < b / 2; p++) {
        uint32_t word = planes[((size_t)i * P + p) * W + o / 16];
        int slice = (int)((word >> (2 * (o % 16))) & 3u);
        Q += (double)slice * ldexp(1.0, 2 * (P - 1 - p));
    }
    return Q;
}

/* [KD3] with R4/R5: w_hat = s * (Q + phi_b) + z, in fp64. */
static double reconstruct(const uint32_t *planes, const uint16_t *s,
                          const uint16_t *z, const double *phi, int i, int o,
                          int b, int P, int W, int d_out) {
    int g = i / ORACLE_GROUP;
    double sv = oracle_f16_to_f64(s[(size_t)g * d_out + o]);
    double zv = oracle_f16_to_f64(z[(size_t)g * d_out + o]);
    double Q = truncated_code(planes, i, o, b, P, W);
    return sv * (Q + phi[b / 2]) + zv;
}

/* Exposed for tests: one reconstructed weight. */
double oracle_reconstruct(const uint32_t *planes, const uint16_t *s,
                          const uint16_t *z, const double *phi, int d_out,
                          int b_max, int i, int o, int b) {
    int P = b_max / 2;
    return reconstruct(planes, s, z, phi, i, o, b, P, d_out / 16, d_out);
}

/* Exposed for tests: the truncated code of one weight (integer valued). */
double oracle_truncated_code(const uint32_t *planes, int d_out, int b_max,
                             int i, int o, int b) {
    return truncated_code(planes, i, o, b, b_max / 2, d_out / 16);
}

/* [FW] + [KD1]/[KD3] with R8: for each output o (in outs[], or every output
 * when outs is NULL), y_o = sum over rows i with b_i > 0, in ascending i, of
 * x_i * w_hat(i, o); bound_o = sum of |w_hat(i, o)| * |x_i| over the same
 * rows.  Results go to y[n] / bound[n] for the n-th requested output.
 * Outputs are split over n_threads OpenMP threads; each output's sum is
 * still taken serially in row order, so the result does not depend on it. */
void oracle_gemv(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                 const uint16_t *x, const uint8_t *b, const double *phi,
                 int d_in, int d_out, int b_max, const int32_t *outs,
                 int n_outs, double *y, double *bound, int n_threads) {
    int P = b_max / 2;
    int W = d_out / 16;
    int n = outs ? n_outs : d_out;
#ifdef _OPENMP
    if (n_threads < 1) n_threads = 1;
#pragma omp parallel for schedule(dynamic, 64) num_threads(n_threads)
#endif
    for (int k = 0; k < n; k++) {
        int o = outs ? outs[k] : k;
        double acc = 0.0, acc_abs = 0.0;
        for (int i = 0; i < d_in; i++) {
            if (b[i] == 0) continue; /* R8: skipped row, no load */
            double xv = oracle_f16_to_f64(x[i]);
            double w = reconstruct(planes, s, z, phi, i, o, b[i], P, W, d_out);
            acc += xv * w;
            acc_abs += fabs(w) * fabs(xv);
        }
        y[k] = acc;
        bound[k] = acc_abs;
    }
}

/* ---- Dense 4-bit comparator (not a GRINQH step; the same-shape fixed-width
 * baseline the throughput table compares against, "4-bit MARLIN").
 * Layout: word j of row i holds outputs 8j..8j+7, output 8j+t in bits
 * [4t+3 : 4t]; w_hat = s * q4 + z with the same fp16 s/z grouping. ---- */
void oracle_pack_dense4(const uint8_t *q4, int d_in, int d_out, uint32_t *w4) {
    int W = d_out / 8;
    for (int i = 0; i < d_in; i++) {
        for (int j = 0; j < W; j++) {
            uint32_t word = 0;
            for (int t = 0; t < 8; t++) {
                int code = q4[(size_t)i * d_out + 8 * j + t];
                for (int bit = 0; bit < 4; bit++) {
                    if ((code >> bit) & 1) word |= (uint32_t)1 << (4 * t + bit);
                }
            }
            w4[(size_t)i * W + j] = word;
        }
    }
}

void oracle_unpack_dense4(const uint32_t *w4, int d_in, int d_out, uint8_t *q4) {
    int W = d_out / 8;
    for (int i = 0; i < d_in; i++) {
        for (int o = 0; o < d_out; o++) {
            uint32_t word = w4[(size_t)i * W + o / 8];
            int code = 0;
            for (int bit = 0; bit < 4; bit++) {
                if ((word >> (4 * (o % 8) + bit)) & 1) code |= 1 << bit;
            }
            q4[(size_t)i * d_out + o] = (uint8_t)code;
        }
    }
}

void oracle_gemv_dense4(const uint32_t *w4, const uint16_t *s,
                        const uint16_t *z, const uint16_t *x, int d_in,
                        int d_out, const int32_t *outs, int n_outs, double *y,
                        double *bound, int n_threads) {
    int W = d_out / 8;
    int n = outs ? n_outs : d_out;
#ifdef _OPENMP
    if (n_threads < 1) n_threads = 1;
#pragma omp parallel for schedule(dynamic, 64) num_threads(n_threads)
#endif
    for (int k = 0; k < n; k++) {
        int o = outs ? outs[k] : k;
        double acc = 0.0, acc_abs = 0.0;
        for (int i = 0; i < d_in; i++) {
            int g = i / ORACLE_GROUP;
            uint32_t word = w4[(size_t)i * W + o / 8];
            double code = (double)((word >> (4 * (o % 8))) & 0xfu);
            double sv = oracle_f16_to_f64(s[(size_t)g * d_out + o]);
            double zv = oracle_f16_to_f64(z[(size_t)g * d_out + o]);
            double w = sv * code + zv;
            double xv = oracle_f16_to_f64(x[i]);
            acc += xv * w;
            acc_abs += fabs(w) * fabs(xv);
        }
        y[k] = acc;
        bound[k] = acc_abs;
    }
}

/* Number of OpenMP threads the library would use by default. */
int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
