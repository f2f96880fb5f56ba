/*
 * gear_oracle.c -- plain, slow CPU oracle of the GEAR KV-cache codec.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or
 * execute this file; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark use it. It shares no code, header, table or constant
 * generator with the CUDA library: it is written from the method's
 * description, step by step, in the order the pages give it.
 *
 * Pages (cited by title and section):
 *   [summary] GEAR: Efficient KV Cache Compression for LLM Inference,
 *             question Q3 (how the method works);
 *   [cites]   GEAR: An Efficient KV Cache Compression Recipe for
 *             Near-Lossless Generative Inference of LLM, the Cites list (the
 *             paper's own sentences, filed under the work each one cites).
 *
 * Precision: the quantization decisions (outlier choice, min/max, scale,
 * codes, dequantized value, residual) are taken in IEEE binary32 with
 * round-to-nearest-even, exactly as the codec defines them; the power
 * iteration, the reconstruction and attention run in binary64.
 * Build with -O2 -ffp-contract=off and without -ffast-math so that every
 * float operation is a single correctly rounded IEEE operation.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Step 1: outlier extraction.                                               */
/* [cites] SqueezeLLM entry: the entries of largest magnitude stay exact, held */
/* as a sparse matrix S = Filter_s(X); [cites] ZeroQuant entry: the sparsity   */
/* ratio s is fixed at 2 %. Reading: Filter_s acts per token and keeps         */
/* k = ceil(s*d) entries (at least a fraction s is kept).                     */
/* ------------------------------------------------------------------------ */
int32_t oracle_num_outliers(float s, int32_t d) {
  double v = (double)s * (double)d - 1e-9;
  if (v <= 0.0) return 0;
  int32_t k = (int32_t)ceil(v);
  return k > d ? d : k;
}

/* The k channels of one token with the largest |x|. Ties in |x| go to the
 * lower channel; +0 and -0 are equal. Returned in ascending channel order. */
void oracle_select_outliers(const float* x, int32_t d, int32_t k, int32_t* idx_out) {
  char* taken = (char*)calloc((size_t)d, 1);
  for (int32_t i = 0; i < k; ++i) {
    int32_t best = -1;
    float best_abs = 0.0f;
    for (int32_t c = 0; c < d; ++c) {
      if (taken[c]) continue;
      float a = fabsf(x[c]);
      if (best < 0 || a > best_abs) { best = c; best_abs = a; }
    }
    taken[best] = 1;
  }
  int32_t m = 0;
  for (int32_t c = 0; c < d; ++c)
    if (taken[c]) idx_out[m++] = c;
  free(taken);
}

/* ------------------------------------------------------------------------ */
/* Step 2: uniform group-wise quantization of the extracted matrix.          */
/* [summary] Q3: the bulk of the entries, which have similar magnitudes, are  */
/* quantized to very few bits (4, for instance); [cites] SqueezeLLM entry:    */
/* the quantizer runs on the matrix left once the outliers are taken out;     */
/* [cites] FlexGen entry: the quantizer groups channels finely within each    */
/* token. Reading: asymmetric                                                 */
/* min-max quantization (zero point = group minimum) over the non-outlier     */
/* entries of each group of g channels of a token:                            */
/*   scale = (mx - mn) / (2^b - 1)                                            */
/*   code  = clamp(round_half_even((x - mn) / scale), 0, 2^b - 1), 0 if scale */
/*           is 0 and at outlier slots                                        */
/*   dhat  = fma(code, scale, mn)                                             */
/* Step 3: residual r = x - dhat at non-outlier slots, 0 at outlier slots.    */
/* ------------------------------------------------------------------------ */
void oracle_quantize_token(const float* x, int32_t d, int32_t bits, int32_t g,
                           const int32_t* oidx, int32_t k, int32_t meta_f16,
                           uint32_t* codes, float* scale_out, float* zero_out,
                           float* dhat_out, float* resid_out) {
  const int32_t levels = (1 << bits) - 1;
  const int32_t words = d * bits / 32;
  char* is_out = (char*)calloc((size_t)d, 1);
  for (int32_t i = 0; i < k; ++i) is_out[oidx[i]] = 1;
  for (int32_t w = 0; w < words; ++w) codes[w] = 0u;

  for (int32_t grp = 0; grp < d / g; ++grp) {
    int32_t c0 = grp * g;
    int have = 0;
    float mn = 0.0f, mx = 0.0f;
    for (int32_t c = c0; c < c0 + g; ++c) {
      if (is_out[c]) continue;
      if (!have) { mn = x[c]; mx = x[c]; have = 1; }
      if (x[c] < mn) mn = x[c];
      if (x[c] > mx) mx = x[c];
    }
    /* Reading: the zero point and the maximum are stored with -0 replaced by
       +0 (v + 0.0f under round-to-nearest), so they do not depend on the order
       in which +0 and -0 occur in the group. */
    mn = mn + 0.0f;
    mx = mx + 0.0f;
    float scale = (mx - mn) / (float)levels;
    if (meta_f16) {
      /* Reading (byte-lean metadata): scale and zero point are stored as
         binary16, rounded to nearest even from the binary32 values, and the
         codes below are decided against the stored values. */
      scale = (float)(_Float16)scale;
      mn = (float)(_Float16)mn + 0.0f;
    }
    scale_out[grp] = scale;
    zero_out[grp] = mn;
    for (int32_t c = c0; c < c0 + g; ++c) {
      uint32_t code = 0u;
      if (!is_out[c] && scale != 0.0f) {
        float q = (x[c] - mn) / scale;
        float qr = nearbyintf(q); /* default rounding mode: ties to even */
        if (qr < 0.0f) qr = 0.0f;
        if (qr > (float)levels) qr = (float)levels;
        code = (uint32_t)qr;
      }
      int32_t bit = c * bits;
      codes[bit / 32] |= code << (bit % 32);
      float dh = fmaf((float)code, scale, mn);
      dhat_out[c] = dh;
      resid_out[c] = is_out[c] ? 0.0f : x[c] - dh;
    }
  }
  free(is_out);
}

/* ------------------------------------------------------------------------ */
/* Step 2, KIVI-combined variant (keys): per-channel groups across tokens.   */
/* [cites] KIVI entries: combining GEAR with KIVI requires a buffer at least */
/* as large as the group size; the same page's list of works citing GEAR,    */
/* TailorKV entry: KIVI quantizes keys per channel and values per token.     */
/* Reading: the                                                              */
/* tokens of a block form groups of g consecutive tokens (the last group may */
/* be shorter); within each group every channel gets its own min-max         */
/* quantizer over the group's non-outlier entries, with the same formulas as */
/* oracle_quantize_token (zero point = minimum, -0 stored as +0, codes       */
/* rounded half to even, code 0 at outlier slots and where scale is 0).      */
/* X is n x d; is_out marks outlier entries (n x d); codes are packed per    */
/* token as in the per-token quantizer; scale and zero are [ngroups][d].     */
/* ------------------------------------------------------------------------ */
void oracle_quantize_channels(const float* X, int32_t n, int32_t d, int32_t bits, int32_t g,
                              const char* is_out, uint32_t* codes, float* scale_out, float* zero_out,
                              float* resid_out) {
  const int32_t levels = (1 << bits) - 1;
  const int32_t words = d * bits / 32;
  for (size_t w = 0; w < (size_t)n * words; ++w) codes[w] = 0u;
  const int32_t ngroups = (n + g - 1) / g;
  for (int32_t j = 0; j < ngroups; ++j) {
    const int32_t t0 = j * g, t1 = (t0 + g < n) ? t0 + g : n;
    for (int32_t c = 0; c < d; ++c) {
      int have = 0;
      float mn = 0.0f, mx = 0.0f;
      for (int32_t t = t0; t < t1; ++t) {
        if (is_out[(size_t)t * d + c]) continue;
        float x = X[(size_t)t * d + c];
        if (!have) { mn = x; mx = x; have = 1; }
        if (x < mn) mn = x;
        if (x > mx) mx = x;
      }
      mn = mn + 0.0f;
      mx = mx + 0.0f;
      float scale = (mx - mn) / (float)levels;
      scale_out[(size_t)j * d + c] = scale;
      zero_out[(size_t)j * d + c] = mn;
      for (int32_t t = t0; t < t1; ++t) {
        uint32_t code = 0u;
        const int out = is_out[(size_t)t * d + c];
        if (!out && scale != 0.0f) {
          float q = (X[(size_t)t * d + c] - mn) / scale;
          float qr = nearbyintf(q);
          if (qr < 0.0f) qr = 0.0f;
          if (qr > (float)levels) qr = (float)levels;
          code = (uint32_t)qr;
        }
        int32_t bit = c * bits;
        codes[(size_t)t * words + bit / 32] |= code << (bit % 32);
        float dh = fmaf((float)code, scale, mn);
        resid_out[(size_t)t * d + c] = out ? 0.0f : X[(size_t)t * d + c] - dh;
      }
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Step 4: seeded start matrix of the power iteration. splitmix64 as         */
/* published by Steele, Lea & Flood (OOPSLA 2014, "Fast splittable          */
/* pseudorandom number generators"): the state advances by the golden-ratio */
/* increment and each output is the state passed through the mix function.  */
/* Q0[i][j] = top 24 bits of output number i*r+j, mapped to u*2^-23 - 1.    */
/* ------------------------------------------------------------------------ */
uint64_t oracle_splitmix64_next(uint64_t* state) {
  *state += 0x9E3779B97F4A7C15ull;
  uint64_t z = *state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

void oracle_start_matrix(uint64_t seed, int32_t d, int32_t r, double* q0) {
  uint64_t state = seed;
  for (int32_t i = 0; i < d; ++i)
    for (int32_t j = 0; j < r; ++j) {
      uint64_t z = oracle_splitmix64_next(&state);
      uint32_t u = (uint32_t)(z >> 40);
      q0[(size_t)i * r + j] = (double)u * ldexp(1.0, -23) - 1.0;
    }
}

/* ------------------------------------------------------------------------ */
/* Step 5: low-rank approximation of the residual by power iteration.       */
/* [summary] Q3: a low-rank matrix, found by singular value decomposition,   */
/* models the error that quantization leaves; [cites] PowerSGD entry: the   */
/* method cites the power-iteration compressor, used here for the SVD.      */
/* For t = 1..T:  P = orthonormalize(R Q),  Q = R^T P;  L = P_T, Rf = Q_T.   */
/* Orthonormalization: modified Gram-Schmidt in binary64; a column whose     */
/* norm after removing the earlier columns is at most 1e-10 of its norm      */
/* before (or zero) is set to the zero column.                               */
/* R is n x d (row-major float), Q0 is d x r, L is n x r, Rf is d x r.       */
/* ------------------------------------------------------------------------ */
void oracle_power_iteration(const float* R, int32_t n, int32_t d, int32_t r, int32_t T,
                            const double* q0, double* L, double* Rf) {
  double* Q = (double*)malloc(sizeof(double) * (size_t)d * (size_t)(r > 0 ? r : 1));
  double* P = (double*)malloc(sizeof(double) * (size_t)n * (size_t)(r > 0 ? r : 1));
  memcpy(Q, q0, sizeof(double) * (size_t)d * (size_t)r);
  for (int32_t t = 0; t < T; ++t) {
    /* P = R Q */
    for (int32_t i = 0; i < n; ++i)
      for (int32_t j = 0; j < r; ++j) {
        double acc = 0.0;
        for (int32_t c = 0; c < d; ++c) acc += (double)R[(size_t)i * d + c] * Q[(size_t)c * r + j];
        P[(size_t)i * r + j] = acc;
      }
    /* modified Gram-Schmidt on the columns of P */
    for (int32_t j = 0; j < r; ++j) {
      double before = 0.0;
      for (int32_t i = 0; i < n; ++i) before += P[(size_t)i * r + j] * P[(size_t)i * r + j];
      before = sqrt(before);
      for (int32_t m = 0; m < j; ++m) {
        double dot = 0.0;
        for (int32_t i = 0; i < n; ++i) dot += P[(size_t)i * r + m] * P[(size_t)i * r + j];
        for (int32_t i = 0; i < n; ++i) P[(size_t)i * r + j] -= dot * P[(size_t)i * r + m];
      }
      double after = 0.0;
      for (int32_t i = 0; i < n; ++i) after += P[(size_t)i * r + j] * P[(size_t)i * r + j];
      after = sqrt(after);
      if (before == 0.0 || after <= 1e-10 * before) {
        for (int32_t i = 0; i < n; ++i) P[(size_t)i * r + j] = 0.0;
      } else {
        for (int32_t i = 0; i < n; ++i) P[(size_t)i * r + j] /= after;
      }
    }
    /* Q = R^T P */
    for (int32_t c = 0; c < d; ++c)
      for (int32_t j = 0; j < r; ++j) {
        double acc = 0.0;
        for (int32_t i = 0; i < n; ++i) acc += (double)R[(size_t)i * d + c] * P[(size_t)i * r + j];
        Q[(size_t)c * r + j] = acc;
      }
  }
  memcpy(L, P, sizeof(double) * (size_t)n * (size_t)r);
  memcpy(Rf, Q, sizeof(double) * (size_t)d * (size_t)r);
  free(P);
  free(Q);
}

/* ------------------------------------------------------------------------ */
/* One unit (n tokens x d channels) through steps 1-5.                        */
/* Inputs are the exact binary32 values of the KV entries. Outputs:          */
/*   codes [n][d*b/32], scale [n][d/g], zero [n][d/g], oidx [n][k],          */
/*   oval [n][k], resid [n][d], L [n][r], Rf [d][r].                          */
/* ------------------------------------------------------------------------ */
void oracle_encode_unit(const float* X, int32_t n, int32_t d, int32_t bits, int32_t g,
                        int32_t k, int32_t meta_f16, int32_t r, int32_t T, uint64_t seed,
                        uint32_t* codes, float* scale, float* zero, int32_t* oidx,
                        float* oval, float* resid, double* L, double* Rf) {
  const int32_t words = d * bits / 32;
  const int32_t G = d / g;
  float* dhat = (float*)malloc(sizeof(float) * (size_t)d);
  for (int32_t t = 0; t < n; ++t) {
    const float* x = X + (size_t)t * d;
    oracle_select_outliers(x, d, k, oidx + (size_t)t * k);
    for (int32_t i = 0; i < k; ++i) oval[(size_t)t * k + i] = x[oidx[(size_t)t * k + i]];
    oracle_quantize_token(x, d, bits, g, oidx + (size_t)t * k, k, meta_f16, codes + (size_t)t * words,
                          scale + (size_t)t * G, zero + (size_t)t * G, dhat,
                          resid + (size_t)t * d);
  }
  free(dhat);
  if (r > 0) {
    double* q0 = (double*)malloc(sizeof(double) * (size_t)d * (size_t)r);
    oracle_start_matrix(seed, d, r, q0);
    oracle_power_iteration(resid, n, d, r, T, q0, L, Rf);
    free(q0);
  }
}

/* The KIVI-combined key encoding of one unit: steps 1 (per token), 2 with  */
/* per-channel token groups of g (oracle_quantize_channels), 3-5 as above.  */
/* scale and zero are [ceil(n/g)][d].                                        */
void oracle_encode_unit_channels(const float* X, int32_t n, int32_t d, int32_t bits, int32_t g,
                                 int32_t k, int32_t r, int32_t T, uint64_t seed, uint32_t* codes,
                                 float* scale, float* zero, int32_t* oidx, float* oval, float* resid,
                                 double* L, double* Rf) {
  char* is_out = (char*)calloc((size_t)n * d, 1);
  for (int32_t t = 0; t < n; ++t) {
    const float* x = X + (size_t)t * d;
    oracle_select_outliers(x, d, k, oidx + (size_t)t * k);
    for (int32_t i = 0; i < k; ++i) {
      oval[(size_t)t * k + i] = x[oidx[(size_t)t * k + i]];
      is_out[(size_t)t * d + oidx[(size_t)t * k + i]] = 1;
    }
  }
  oracle_quantize_channels(X, n, d, bits, g, is_out, codes, scale, zero, resid);
  free(is_out);
  if (r > 0) {
    double* q0 = (double*)malloc(sizeof(double) * (size_t)d * (size_t)r);
    oracle_start_matrix(seed, d, r, q0);
    oracle_power_iteration(resid, n, d, r, T, q0, L, Rf);
    free(q0);
  }
}

/* ------------------------------------------------------------------------ */
/* Step 6: reconstruction, X ~ D + L Rf^T with the outlier slots holding    */
/* their exact values ([cites] LoftQ and Zafrir et al. entries: the low-rank */
/* part carries the error shared across entries, the sparse part fixes the  */
/* individual outliers).                                                     */
/* ------------------------------------------------------------------------ */
void oracle_reconstruct_unit(int32_t n, int32_t d, int32_t bits, int32_t g, int32_t k,
                             int32_t r, const uint32_t* codes, const float* scale,
                             const float* zero, const int32_t* oidx, const float* oval,
                             const double* L, const double* Rf, double* Xhat) {
  const int32_t words = d * bits / 32;
  const int32_t G = d / g;
  const uint32_t mask = (bits == 32) ? 0xFFFFFFFFu : ((1u << bits) - 1u);
  for (int32_t t = 0; t < n; ++t) {
    for (int32_t c = 0; c < d; ++c) {
      int32_t bit = c * bits;
      uint32_t code = (codes[(size_t)t * words + bit / 32] >> (bit % 32)) & mask;
      int32_t grp = c / g;
      double v = (double)fmaf((float)code, scale[(size_t)t * G + grp], zero[(size_t)t * G + grp]);
      for (int32_t j = 0; j < r; ++j) v += L[(size_t)t * r + j] * Rf[(size_t)c * r + j];
      Xhat[(size_t)t * d + c] = v;
    }
    for (int32_t i = 0; i < k; ++i)
      Xhat[(size_t)t * d + oidx[(size_t)t * k + i]] = (double)oval[(size_t)t * k + i];
  }
}

/* Step 6 for a KIVI-combined key unit: the group of token t is t / g.      */
void oracle_reconstruct_unit_channels(int32_t n, int32_t d, int32_t bits, int32_t g, int32_t k,
                                      int32_t r, const uint32_t* codes, const float* scale,
                                      const float* zero, const int32_t* oidx, const float* oval,
                                      const double* L, const double* Rf, double* Xhat) {
  const int32_t words = d * bits / 32;
  const uint32_t mask = (1u << bits) - 1u;
  for (int32_t t = 0; t < n; ++t) {
    const int32_t j = t / g;
    for (int32_t c = 0; c < d; ++c) {
      int32_t bit = c * bits;
      uint32_t code = (codes[(size_t)t * words + bit / 32] >> (bit % 32)) & mask;
      double v = (double)fmaf((float)code, scale[(size_t)j * d + c], zero[(size_t)j * d + c]);
      for (int32_t q = 0; q < r; ++q) v += L[(size_t)t * r + q] * Rf[(size_t)c * r + q];
      Xhat[(size_t)t * d + c] = v;
    }
    for (int32_t i = 0; i < k; ++i)
      Xhat[(size_t)t * d + oidx[(size_t)t * k + i]] = (double)oval[(size_t)t * k + i];
  }
}

/* ------------------------------------------------------------------------ */
/* Step 7: the decode-step attention that consumes the cache: one query     */
/* vector against n reconstructed keys and values, in binary64:              */
/*   o = sum_t softmax_t(scale * q . K_t) V_t.                                */
/* ------------------------------------------------------------------------ */
void oracle_attention(const double* q, const double* K, const double* V, int32_t n,
                      int32_t d, double scale, double* out) {
  double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  double mx = -INFINITY;
  for (int32_t t = 0; t < n; ++t) {
    double acc = 0.0;
    for (int32_t c = 0; c < d; ++c) acc += q[c] * K[(size_t)t * d + c];
    s[t] = scale * acc;
    if (s[t] > mx) mx = s[t];
  }
  double den = 0.0;
  for (int32_t t = 0; t < n; ++t) { s[t] = exp(s[t] - mx); den += s[t]; }
  for (int32_t c = 0; c < d; ++c) out[c] = 0.0;
  for (int32_t t = 0; t < n; ++t)
    for (int32_t c = 0; c < d; ++c) out[c] += (s[t] / den) * V[(size_t)t * d + c];
  free(s);
}
