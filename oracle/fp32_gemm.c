/*
 * Oracle for the fp32 prompt-phase projection K = X·W_K with a fixed
 * accumulation order. TEST INFRASTRUCTURE ONLY: used by tests/ and nothing
 * on the product path.
 *
 * Source: Slim Attention article, section "K-Cache is All You Need": in the
 * prompt phase K is formed for all prompt tokens and cached (row vectors,
 * K = X·W_K).
 *
 * Definition written out: Y[i][j] = fmaf(X[i][d-1], W[d-1][j], ... fmaf(X[i][0],
 * W[0][j], 0.0f)), i.e. one fp32 accumulator per output, k ascending, each step
 * a single correctly rounded fused multiply-add. fmaf is correctly rounded by
 * the C standard, so this order fixes every bit of the result.
 */
#include <math.h>
#include <stdint.h>

void oracle_gemm_f32_fmaf(const float *X, const float *W, float *Y,
                          int64_t n, int64_t d_in, int64_t d_out) {
  for (int64_t i = 0; i < n; ++i) {
    for (int64_t j = 0; j < d_out; ++j) {
      float acc = 0.0f;
      for (int64_t k = 0; k < d_in; ++k) {
        acc = fmaf(X[i * d_in + k], W[k * d_out + j], acc);
      }
      Y[i * d_out + j] = acc;
    }
  }
}
