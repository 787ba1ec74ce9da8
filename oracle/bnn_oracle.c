/*
 * CPU oracle for the binary (+1/-1) matrix product.  TEST INFRASTRUCTURE ONLY:
 * only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * load this library.  It shares no code with the CUDA path.
 *
 * Every routine here is the plain definition, written out with +1/-1 values
 * materialised as int8 and integer multiply-accumulate.  No bit tricks, no
 * blocking, no reordering beyond an OpenMP split over independent outputs
 * (each output is still one thread's plain loop over k, so the split does not
 * change any result).
 *
 * Sources (page title, section / equation):
 *  - "Extreme Quantization: Binary, Ternary & 1-bit LLMs", Notation:
 *    sign(x) = +1 for x >= 0 and -1 for x < 0; XNOR-Net section, eq. (4):
 *    both weights and activations pass through sign().
 *  - same page, Binary Neural Networks section, eq. (1): y = alpha * (w_b^T x),
 *    alpha = (1/n) sum_i |w_i|.
 *  - "First Principles: Why Binary Ops Can Be Exponentially Faster",
 *    section "1. Arithmetic: MAC -> XNOR + popcount": bit 0 encodes +1 and bit 1
 *    encodes -1; bits are packed into machine words; pad bits encode +1.
 *
 * Readings where the pages are silent:
 *  - NaN: sign(NaN) = +1 (NaN is not < 0).  -0.0 is not < 0, so it maps to +1.
 *  - bit j of word w holds element 32*w + j (least significant bit first);
 *    rows are padded to a multiple of 4 words, pad bits and pad words are 0.
 *  - convolution padding pads the real input with zeros, so a padded tap is
 *    sign(0) = +1.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Number of 32-bit words in one packed row of K elements: ceil(K/32) rounded
 * up to a multiple of 4 (so that every row starts on a 16-byte boundary). */
int64_t oracle_ld_words(int64_t K) {
    int64_t words = (K + 31) / 32;
    return (words + 3) / 4 * 4;
}

/* sign() of the Notation section: -1 exactly when x < 0, else +1. */
void oracle_sign_f32(const float* x, int64_t n, int8_t* out) {
    for (int64_t i = 0; i < n; ++i) {
        double v = (double)x[i];
        out[i] = (v < 0.0) ? (int8_t)-1 : (int8_t)1;
    }
}

/* Pack +1/-1 values into words: bit 1 for -1, bit 0 for +1.  Element k of a
 * row goes to bit (k % 32) of word (k / 32).  Words past the last element,
 * up to ld_words, are zero (pad encodes +1). */
void oracle_pack_pm1(const int8_t* b, int64_t rows, int64_t K,
                     uint32_t* out, int64_t ld_words) {
    for (int64_t r = 0; r < rows; ++r) {
        uint32_t* orow = out + r * ld_words;
        for (int64_t w = 0; w < ld_words; ++w) orow[w] = 0u;
        for (int64_t k = 0; k < K; ++k) {
            int8_t v = b[r * K + k];
            if (v == -1) orow[k / 32] |= (uint32_t)1u << (uint32_t)(k % 32);
        }
    }
}

/* alpha_r = (1/K) * sum_k |w_rk|, accumulated in double over the true K
 * (eq. (1) of the Binary Neural Networks section). */
void oracle_alpha_f32(const float* w, int64_t rows, int64_t K, double* alpha) {
    for (int64_t r = 0; r < rows; ++r) {
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) acc += fabs((double)w[r * K + k]);
        alpha[r] = acc / (double)K;
    }
}

/* s[m, n] = sum_k a[m, k] * w[n, k] with a, w in {-1, +1}: the plain
 * definition of w_b^T x_b (left-hand side of eq. (6)). */
void oracle_matmul_pm1(const int8_t* a, const int8_t* w, int64_t M, int64_t N,
                       int64_t K, int32_t* s) {
    int64_t job;
    /* One job per output (m, n), so that a single row (a GEMV) also spreads
     * over the threads. */
#pragma omp parallel for schedule(static)
    for (job = 0; job < M * N; ++job) {
        const int64_t m = job / N, n = job % N;
        const int8_t* arow = a + m * K;
        const int8_t* wrow = w + n * K;
        int32_t acc = 0;
        for (int64_t k = 0; k < K; ++k) acc += (int32_t)arow[k] * (int32_t)wrow[k];
        s[m * N + n] = acc;
    }
}

/* 2-D convolution of +1/-1 input with +1/-1 filters, NCHW input and output,
 * OIHW filters, square kernel kk x kk.  Taps outside the image read +1
 * (zero-padded real input, then sign). */
void oracle_conv2d_pm1(const int8_t* x, int64_t n, int64_t c, int64_t h, int64_t wd,
                       const int8_t* f, int64_t cout, int64_t kk,
                       int64_t stride, int64_t pad, int32_t* out) {
    int64_t oh = (h + 2 * pad - kk) / stride + 1;
    int64_t ow = (wd + 2 * pad - kk) / stride + 1;
    int64_t job;
#pragma omp parallel for schedule(static)
    for (job = 0; job < n * cout; ++job) {
        int64_t b = job / cout, co = job % cout;
        for (int64_t y = 0; y < oh; ++y) {
            for (int64_t xo = 0; xo < ow; ++xo) {
                int32_t acc = 0;
                for (int64_t ci = 0; ci < c; ++ci) {
                    for (int64_t ky = 0; ky < kk; ++ky) {
                        for (int64_t kx = 0; kx < kk; ++kx) {
                            int64_t iy = y * stride - pad + ky;
                            int64_t ix = xo * stride - pad + kx;
                            int32_t v = 1;
                            if (iy >= 0 && iy < h && ix >= 0 && ix < wd)
                                v = x[((b * c + ci) * h + iy) * wd + ix];
                            int32_t fw = f[((co * c + ci) * kk + ky) * kk + kx];
                            acc += v * fw;
                        }
                    }
                }
                out[((b * cout + co) * oh + y) * ow + xo] = acc;
            }
        }
    }
}

/* Thread count for the OpenMP loops above (timing of the oracle on one core
 * and on all cores); it changes no result. */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
