/*
 * tq_oracle.c -- the oracle: a plain, slow, fp64 CPU restatement of what the
 * trellis-decode matmul path computes.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark load this file.  It shares no code, header,
 * table or constant with the CUDA library (decode_matmul_b200/csrc); the two
 * sides meet only through the seeded inputs that tqsynth produces.
 *
 * Sources (cited by page title and section):
 *  - "Pingala-8" landing page, section "How it works" (仕組み): weights are
 *    coded in groups of four by an 8-state trellis code; a small state carried
 *    from one group to the next decides which values the next group may use;
 *    a random Hadamard rotation is applied before encoding.
 *  - "Bonsai 2 27B" article, section on the change of basis: the rotation is
 *    folded into the stored weights and the matching transform is applied to
 *    the activations at run time.
 *  - "8 open models ... what 2-bit quantization costs", section "Size": the
 *    per-block scales cost bits on top of the 2-bit codes.
 * The pages fix no bit layout; the layout restated here is the one this
 * project adopts (one byte per group of four, state = low 3 bits of the
 * previous code, reset every 256 weights, one fp16 scale per 256 weights,
 * 8 codebooks of 256 fp16 4-vectors, RHT = Sylvester Hadamard of order 512
 * after a seeded +-1 diagonal).
 *
 * Every function here follows the plain definition, step by step, with no
 * blocking, fusion or reordering.  Rounding to fp16/bf16 is written out from
 * the IEEE-754 round-to-nearest-even definition.
 *
 * Parity pins (what each function is checked against, in tests/):
 *   orc_mix64 / orc_draw      published SplitMix64 output for state 0
 *   orc_f16_from_f64          numpy float16 (library) over every scale x
 *                             codebook product the format can produce
 *   orc_bf16_from_f64         brute force nearest-neighbour search
 *   orc_decode                hand-worked examples with exact codebooks
 *   orc_rht                   H*H^T = I, norm preservation, closed forms,
 *                             scipy.linalg.hadamard (library)
 *   orc_matmul                numpy matmul (library), linearity
 *   orc_viterbi               brute force over all code sequences (tiny rows)
 *   orc_viterbi32             brute force in binary64 (its path is optimal to
 *                             within binary32 rounding), the binary64 Viterbi
 *   orc_refit32               exact least-squares cases (w = 2^e * path)
 *   orc_encode32              closed-form scales, zero-error round trips,
 *                             monotone refits, Gaussian MSE between the
 *                             rate-distortion bound and the best 2-bit
 *                             scalar quantizer
 *   orc_ldlq32                U = 0 reduces to orc_encode32; the proxy-loss
 *                             identity tr(E H E^T) = sum of block errors for
 *                             H = (I+U)(I+U)^T (binary64 check); lower proxy
 *                             loss than plain encoding
 * Compile: gcc -O2 -ffp-contract=off -fPIC -shared (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Counter-based generator: SplitMix64 (Steele, Lea & Flood, OOPSLA 2014;    */
/* Vigna's public reference splitmix64.c).  The i-th output (i = 0, 1, ...)  */
/* of a generator whose state starts at `key` is mix64(key + (i+1)*gamma).   */
/* The RHT signs are drawn from it; the oracle implements it on its own.     */
/* ------------------------------------------------------------------------ */
static const uint64_t ORC_GAMMA = 0x9E3779B97F4A7C15ULL;

uint64_t orc_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

uint64_t orc_draw(uint64_t key, uint64_t i) { return orc_mix64(key + (i + 1) * ORC_GAMMA); }

/* Sign of the RHT diagonal at input feature k: -1 when the top bit of the
 * k-th draw is set, else +1. */
int orc_rht_sign(uint64_t seed, int64_t k) { return (orc_draw(seed, (uint64_t)k) >> 63) ? -1 : 1; }

/* Seed of the RHT used by phase p (0..3) of layer l of a layer stack. */
uint64_t orc_stack_phase_seed(uint64_t seed, int32_t layer, int32_t phase) {
  uint64_t tag = 0x516E0000ULL | ((uint64_t)layer << 2) | (uint64_t)phase;
  return orc_mix64(seed ^ orc_mix64(tag));
}

/* ------------------------------------------------------------------------ */
/* IEEE-754 binary16 / bfloat16 <-> binary64                                 */
/* ------------------------------------------------------------------------ */
double orc_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1, e = (h >> 10) & 0x1F, m = h & 0x3FF;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24); /* subnormal: m * 2^-24 */
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
  return sign ? -v : v;
}

double orc_bf16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1, e = (h >> 7) & 0xFF, m = h & 0x7F;
  double v;
  if (e == 0)
    v = ldexp((double)m, -133); /* subnormal: m * 2^-133 */
  else if (e == 255)
    v = m ? NAN : INFINITY;
  else
    v = ldexp((double)(128 + m), e - 134); /* (1 + m/128) * 2^(e-127) */
  return sign ? -v : v;
}

/* Round x to the nearest value of a binary format with `mbits` stored
 * mantissa bits, minimum normal exponent `emin` and maximum exponent `emax`,
 * ties to even, keeping subnormals; returns the encoded bits (sign included).
 * Steps: quantum q = 2^(max(e, emin) - mbits) for |x| in [2^e, 2^(e+1));
 * r = nearest integer to |x|/q (ties to even; |x|/q is exact in binary64);
 * value = r*q, re-encoded. */
static uint16_t round_to_format(double x, int mbits, int emin, int emax, int ebias) {
  uint16_t sign = signbit(x) ? 0x8000 : 0; /* both formats are 16 bits wide */
  int expbits = 15 - mbits;
  uint16_t inf = (uint16_t)(((1u << expbits) - 1) << mbits);
  double ax = fabs(x);
  if (isnan(x)) return (uint16_t)(sign | inf | (1u << (mbits - 1)));
  if (isinf(x)) return (uint16_t)(sign | inf);
  if (ax == 0.0) return sign;
  int E;
  (void)frexp(ax, &E); /* ax = f * 2^E, f in [0.5, 1) */
  int e = E - 1;        /* ax in [2^e, 2^(e+1)) */
  int qe = (e < emin ? emin : e) - mbits;
  double n = ldexp(ax, -qe);
  double r = nearbyint(n); /* default rounding mode: to nearest, ties to even */
  uint32_t ri = (uint32_t)r;
  if (e < emin) {
    /* subnormal range: bits are r itself (r == 2^mbits is the smallest normal) */
    return (uint16_t)(sign | ri);
  }
  if (ri == (1u << (mbits + 1))) { /* rounded up into the next binade */
    ri = 1u << mbits;
    e += 1;
  }
  if (e > emax) return (uint16_t)(sign | inf);
  return (uint16_t)(sign | ((uint32_t)(e + ebias) << mbits) | (ri - (1u << mbits)));
}

uint16_t orc_f16_from_f64(double x) { return round_to_format(x, 10, -14, 15, 15); }
uint16_t orc_bf16_from_f64(double x) { return round_to_format(x, 7, -126, 127, 127); }

void orc_f16_from_f64_array(const double* x, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_f16_from_f64(x[i]);
}

void orc_bf16_from_f64_array(const double* x, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_from_f64(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Decode ("How it works": groups of 4 coded in order; the state carried     */
/* from the previous group selects the codebook of the next group).          */
/*   s_g = 0                      if g mod 64 == 0 (start of a 256-block)    */
/*       = codes[n][g-1] & 7      otherwise                                  */
/*   W[n][4g+j] = fp16_RNE( scale[n][g/64] * cb[s_g][codes[n][g]][j] )       */
/* codes: uint8 [n][k/4]; scales: fp16 [n][k/256]; cb: fp16 [8][256][4].     */
/* ------------------------------------------------------------------------ */
void orc_decode_rows(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb, int64_t k,
                     int64_t row_begin, int64_t row_end, uint16_t* w) {
  int64_t groups = k / 4, blocks = (k + 255) / 256; /* rows shorter than 256 (tiny tests) use one block */
  for (int64_t n = row_begin; n < row_end; ++n) {
    for (int64_t g = 0; g < groups; ++g) {
      int s = (g % 64 == 0) ? 0 : (codes[n * groups + g - 1] & 7);
      int c = codes[n * groups + g];
      double sc = orc_f16_to_f64(scales[n * blocks + g / 64]);
      for (int j = 0; j < 4; ++j) {
        double e = orc_f16_to_f64(cb[((int64_t)s * 256 + c) * 4 + j]);
        w[(n - row_begin) * k + 4 * g + j] = orc_f16_from_f64(sc * e);
      }
    }
  }
}

void orc_decode(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb, int64_t n, int64_t k,
                uint16_t* w) {
  orc_decode_rows(codes, scales, cb, k, 0, n, w);
}

/* ------------------------------------------------------------------------ */
/* Randomized Hadamard transform on activations (landing page "How it        */
/* works"; "Bonsai 2" article, change of basis): first the +-1 diagonal D,   */
/* then the orthonormal Hadamard matrix of order 512 in natural (Sylvester)  */
/* order, H[i][j] = (-1)^popcount(i & j) / sqrt(512), on each contiguous     */
/* block of 512 features of each row.  Written as the plain O(512^2) sum.    */
/* x: bf16 [m][k]; out: fp64 [m][k].                                         */
/* ------------------------------------------------------------------------ */
void orc_rht(const uint16_t* x, int64_t m, int64_t k, uint64_t seed, double* out) {
  const double inv = 1.0 / sqrt(512.0);
  double* dx = (double*)malloc(sizeof(double) * 512);
  for (int64_t r = 0; r < m; ++r) {
    for (int64_t b = 0; b < k / 512; ++b) {
      for (int j = 0; j < 512; ++j) {
        int64_t kk = b * 512 + j;
        dx[j] = orc_rht_sign(seed, kk) * orc_bf16_to_f64(x[r * k + kk]);
      }
      for (int i = 0; i < 512; ++i) {
        double acc = 0.0;
        for (int j = 0; j < 512; ++j) acc += (__builtin_popcount((unsigned)(i & j)) & 1) ? -dx[j] : dx[j];
        out[r * k + b * 512 + i] = acc * inv;
      }
    }
  }
  free(dx);
}

/* Same transform on fp64 input (used to pin H and D on exact vectors). */
void orc_rht_f64(const double* x, int64_t m, int64_t k, uint64_t seed, double* out) {
  const double inv = 1.0 / sqrt(512.0);
  double* dx = (double*)malloc(sizeof(double) * 512);
  for (int64_t r = 0; r < m; ++r) {
    for (int64_t b = 0; b < k / 512; ++b) {
      for (int j = 0; j < 512; ++j) dx[j] = orc_rht_sign(seed, b * 512 + j) * x[r * k + b * 512 + j];
      for (int i = 0; i < 512; ++i) {
        double acc = 0.0;
        for (int j = 0; j < 512; ++j) acc += (__builtin_popcount((unsigned)(i & j)) & 1) ? -dx[j] : dx[j];
        out[r * k + b * 512 + i] = acc * inv;
      }
    }
  }
  free(dx);
}

/* ------------------------------------------------------------------------ */
/* Matmul: y[t][n] = sum_k W[n][k] * x'[t][k], fp64, k ascending.            */
/* w: fp16 [rows][k]; xr: fp64 [m][k]; y: fp64 [m][rows].                    */
/* ------------------------------------------------------------------------ */
void orc_matmul(const uint16_t* w, const double* xr, int64_t m, int64_t rows, int64_t k, double* y) {
  for (int64_t t = 0; t < m; ++t)
    for (int64_t n = 0; n < rows; ++n) {
      double acc = 0.0;
      for (int64_t kk = 0; kk < k; ++kk) acc += orc_f16_to_f64(w[n * k + kk]) * xr[t * k + kk];
      y[t * rows + n] = acc;
    }
}

/* Decode + matmul for the rows [row_begin, row_end) of one trellis-coded
 * weight: y[t][n - row_begin] for every token t.  Used for sampled checks on
 * large matrices and for the CPU baseline; it calls the two functions above
 * row by row and adds no step of its own. */
void orc_linear_rows(const uint8_t* codes, const uint16_t* scales, const uint16_t* cb, int64_t k,
                     const double* xr, int64_t m, int64_t row_begin, int64_t row_end, double* y) {
  uint16_t* w = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)k);
  double* yrow = (double*)malloc(sizeof(double) * (size_t)m);
  int64_t rows = row_end - row_begin;
  for (int64_t n = row_begin; n < row_end; ++n) {
    orc_decode_rows(codes, scales, cb, k, n, n + 1, w);
    orc_matmul(w, xr, m, 1, k, yrow);
    for (int64_t t = 0; t < m; ++t) y[t * rows + (n - row_begin)] = yrow[t];
  }
  free(yrow);
  free(w);
}

/* ------------------------------------------------------------------------ */
/* Viterbi encoder (tiny rows; test tool).  Chooses codes c_0..c_{G-1} that  */
/* minimise sum_g ||w_g - dec(s_g, c_g)||^2 where dec(s, c)[j] =             */
/* fp16_RNE(scale_b * cb[s][c][j]), s_0 = 0 at each 256-block start and      */
/* s_{g+1} = c_g & 7 inside a block.  End state free.  Ties: the first       */
/* candidate in (code, predecessor state) ascending order is kept.           */
/* w: fp64 [k]; scales: fp16 [k/256] (k < 256 uses scales[0]);              */
/* codes out: uint8 [k/4].  Returns the minimum cost.                        */
/* ------------------------------------------------------------------------ */
double orc_viterbi(const double* w, int64_t k, const uint16_t* cb, const uint16_t* scales, uint8_t* codes) {
  int64_t groups = k / 4;
  double total = 0.0;
  /* per block DP; back-pointers: best (prev state, code) for each (g, state) */
  int* bp_state = (int*)malloc(sizeof(int) * 64 * 8);
  int* bp_code = (int*)malloc(sizeof(int) * 64 * 8);
  for (int64_t g0 = 0; g0 < groups; g0 += 64) {
    int64_t gn = (groups - g0 < 64) ? groups - g0 : 64;
    double sc = orc_f16_to_f64(scales[g0 / 64]);
    double J[8], Jn[8];
    for (int s = 0; s < 8; ++s) J[s] = (s == 0) ? 0.0 : INFINITY;
    for (int64_t g = 0; g < gn; ++g) {
      for (int s = 0; s < 8; ++s) Jn[s] = INFINITY;
      for (int c = 0; c < 256; ++c) {
        for (int s = 0; s < 8; ++s) {
          if (isinf(J[s])) continue;
          double err = 0.0;
          for (int j = 0; j < 4; ++j) {
            double d = orc_f16_to_f64(orc_f16_from_f64(sc * orc_f16_to_f64(cb[((int64_t)s * 256 + c) * 4 + j])));
            double diff = w[4 * (g0 + g) + j] - d;
            err += diff * diff;
          }
          double cost = J[s] + err;
          int ns = c & 7;
          if (cost < Jn[ns]) {
            Jn[ns] = cost;
            bp_state[g * 8 + ns] = s;
            bp_code[g * 8 + ns] = c;
          }
        }
      }
      memcpy(J, Jn, sizeof J);
    }
    int best = 0;
    for (int s = 1; s < 8; ++s)
      if (J[s] < J[best]) best = s;
    total += J[best];
    int s = best;
    for (int64_t g = gn - 1; g >= 0; --g) {
      codes[g0 + g] = (uint8_t)bp_code[g * 8 + s];
      s = bp_state[g * 8 + s];
    }
  }
  free(bp_state);
  free(bp_code);
  return total;
}

/* Squared error of a given code sequence (same cost as orc_viterbi). */
double orc_code_cost(const double* w, int64_t k, const uint16_t* cb, const uint16_t* scales, const uint8_t* codes) {
  int64_t groups = k / 4;
  double total = 0.0;
  for (int64_t g = 0; g < groups; ++g) {
    int s = (g % 64 == 0) ? 0 : (codes[g - 1] & 7);
    double sc = orc_f16_to_f64(scales[g / 64]);
    for (int j = 0; j < 4; ++j) {
      double d = orc_f16_to_f64(orc_f16_from_f64(sc * orc_f16_to_f64(cb[((int64_t)s * 256 + codes[g]) * 4 + j])));
      double diff = w[4 * g + j] - d;
      total += diff * diff;
    }
  }
  return total;
}

/* ======================================================================== */
/* Trellis encoder with binary32 decisions.                                  */
/*                                                                           */
/* "Pingala-8" landing page, "How it works": the groups of four weights are  */
/* coded in order, the state carried from one group selects the values the   */
/* next group may use, and the result lands closer to the weights at the     */
/* same bits; a random Hadamard rotation is applied to the weights first.    */
/* The pages give no encoding procedure.  Readings adopted here:             */
/*  - per 256-weight block the code path of least squared error is found by  */
/*    dynamic programming over the 8 states (Viterbi), start state 0, end    */
/*    state free;                                                            */
/*  - the block's fp16 scale starts at RMS(block) * gain and is refitted by  */
/*    least squares on the chosen path (sum w*e / sum e*e, e the unscaled    */
/*    codebook values) up to `refits` times, a refit kept only when its      */
/*    path costs less;                                                       */
/*  - every decision (scale roundings, path choices) is taken in binary32 in */
/*    the order written below, so that any implementation with this order    */
/*    chooses identical codes.  orc_viterbi above is the binary64 reference. */
/*                                                                           */
/* Candidate cost of code c from state s for group weights w (u = -2 w):     */
/*   t = J[s] + N[s][c];  t = fma(u3, D3, t); ... t = fma(u0, D0, t)          */
/* with D = fp16_RNE(scale * cb[s][c]) and N = ((D0*D0 + D1*D1) + D2*D2) +   */
/* D3*D3 (each "a*a + r" one fma).  t equals the squared error minus |w|^2,  */
/* a constant of the group.  The new state c & 7 keeps the least t; ties go  */
/* to the smaller code, then the smaller predecessor state.  Sums over a     */
/* block use the fold order: v[i] += v[i + h] for h = 128, 64, ..., 1.       */
/* ======================================================================== */

static float f32_of_f16(uint16_t h) { return (float)orc_f16_to_f64(h); }
static uint16_t f16_of_f32(float x) { return orc_f16_from_f64((double)x); }

/* Fold-order sum of n (a power of two) values; v is overwritten. */
static float fold_sum(float* v, int n) {
  for (int h = n / 2; h >= 1; h /= 2)
    for (int i = 0; i < h; ++i) v[i] = v[i] + v[i + h];
  return v[0];
}

/* Viterbi over `groups` groups (1..64) of w at fp16 scale bits `scale`.
 * codes out: uint8 [groups].  Returns the least final path cost t (squared
 * error minus the sum of |w_g|^2). */
float orc_viterbi32(const float* w, int groups, const uint16_t* cb, uint16_t scale, uint8_t* codes) {
  float D[8][256][4], N[8][256];
  uint8_t bp[64][8];
  float sigma = f32_of_f16(scale);
  for (int s = 0; s < 8; ++s)
    for (int c = 0; c < 256; ++c) {
      for (int j = 0; j < 4; ++j) D[s][c][j] = f32_of_f16(f16_of_f32(sigma * f32_of_f16(cb[(s * 256 + c) * 4 + j])));
      float nn = D[s][c][0] * D[s][c][0];
      nn = fmaf(D[s][c][1], D[s][c][1], nn);
      nn = fmaf(D[s][c][2], D[s][c][2], nn);
      N[s][c] = fmaf(D[s][c][3], D[s][c][3], nn);
    }
  float J[8];
  for (int s = 0; s < 8; ++s) J[s] = (s == 0) ? 0.0f : INFINITY;
  for (int g = 0; g < groups; ++g) {
    float u[4];
    for (int j = 0; j < 4; ++j) u[j] = -2.0f * w[4 * g + j];
    float Jn[8];
    for (int ns = 0; ns < 8; ++ns) {
      float best = 0.0f;
      int bc = -1, bs = -1;
      for (int c = ns; c < 256; c += 8)
        for (int s = 0; s < 8; ++s) {
          float t = J[s] + N[s][c];
          t = fmaf(u[3], D[s][c][3], t);
          t = fmaf(u[2], D[s][c][2], t);
          t = fmaf(u[1], D[s][c][1], t);
          t = fmaf(u[0], D[s][c][0], t);
          if (bc < 0 || t < best) {
            best = t;
            bc = c;
            bs = s;
          }
        }
      Jn[ns] = best;
      bp[g][ns] = (uint8_t)((bc & 0xF8) | bs);
    }
    memcpy(J, Jn, sizeof J);
  }
  int st = 0;
  for (int s = 1; s < 8; ++s)
    if (J[s] < J[st]) st = s;
  float jmin = J[st];
  for (int g = groups - 1; g >= 0; --g) {
    codes[g] = (uint8_t)((bp[g][st] & 0xF8) | st);
    st = bp[g][st] & 7;
  }
  return jmin;
}

/* Least-squares scale of one 256-weight block for fixed codes:
 * fp16_RNE(sum w*e / sum e*e), clamped to +-65504.  Returns 0 (no refit)
 * when sum e*e is not positive or the ratio is not a number. */
int orc_refit32(const float* w, const uint8_t* codes, const uint16_t* cb, uint16_t* scale) {
  float p[256], q[256];
  for (int i = 0; i < 256; ++i) {
    int g = i / 4, j = i % 4;
    int s = (g == 0) ? 0 : (codes[g - 1] & 7);
    float e = f32_of_f16(cb[(s * 256 + codes[g]) * 4 + j]);
    p[i] = w[i] * e;
    q[i] = e * e;
  }
  float num = fold_sum(p, 256), den = fold_sum(q, 256);
  if (!(den > 0.0f)) return 0;
  float r = num / den;
  if (isnan(r)) return 0;
  if (r > 65504.0f) r = 65504.0f;
  if (r < -65504.0f) r = -65504.0f;
  *scale = f16_of_f32(r);
  return 1;
}

/* Encode one 256-weight block wb: codes64 out, *scale out, *err out (fold-
 * order sum of (w - w_hat)^2 of the chosen encoding); wh out (may be NULL):
 * the decoded block as binary32. */
static void encode_block32(const float* wb, const uint16_t* cb, float gain, int refits, uint8_t* codes64,
                           uint16_t* scale, float* err, float* wh) {
  float v[256];
  for (int i = 0; i < 256; ++i) v[i] = wb[i] * wb[i];
  float ss = fold_sum(v, 256);
  float rs = sqrtf(ss * 0.00390625f) * gain;
  if (!(rs <= 65504.0f)) rs = 65504.0f;
  uint16_t best_scale = f16_of_f32(rs);
  uint8_t best[64], cand[64];
  float best_j = orc_viterbi32(wb, 64, cb, best_scale, best);
  for (int it = 0; it < refits; ++it) {
    uint16_t s1;
    if (!orc_refit32(wb, best, cb, &s1) || s1 == best_scale) break;
    float j1 = orc_viterbi32(wb, 64, cb, s1, cand);
    if (!(j1 < best_j)) break;
    best_j = j1;
    best_scale = s1;
    memcpy(best, cand, 64);
  }
  memcpy(codes64, best, 64);
  *scale = best_scale;
  float sigma = f32_of_f16(best_scale);
  for (int i = 0; i < 256; ++i) {
    int g = i / 4, j = i % 4;
    int s = (g == 0) ? 0 : (best[g - 1] & 7);
    float d = f32_of_f16(f16_of_f32(sigma * f32_of_f16(cb[(s * 256 + best[g]) * 4 + j])));
    if (wh) wh[i] = d;
    float e = wb[i] - d;
    v[i] = e * e;
  }
  *err = fold_sum(v, 256);
}

/* Encode n rows of k rotated weights (k a multiple of 256).
 * w: fp32 [n][k]; cb: fp16 [8][256][4]; codes out uint8 [n][k/4]; scales out
 * fp16 [n][k/256]; err out fp32 [n][k/256] = fold-order sum of (w - w_hat)^2
 * of the chosen encoding (may be NULL). */
void orc_encode32(const float* w, int64_t n, int64_t k, const uint16_t* cb, float gain, int refits, uint8_t* codes,
                  uint16_t* scales, float* err) {
  int64_t nb = k / 256;
  for (int64_t r = 0; r < n; ++r)
    for (int64_t b = 0; b < nb; ++b) {
      float e;
      encode_block32(w + r * k + b * 256, cb, gain, refits, codes + r * (k / 4) + b * 64, &scales[r * nb + b], &e,
                     NULL);
      if (err) err[r * nb + b] = e;
    }
}

/* ======================================================================== */
/* Block LDLQ with the trellis encoder.                                      */
/*                                                                           */
/* LDLQ, named on the "Pingala-8" landing page ("How it works"): the coding */
/* error of the columns already coded is fed forward.  Reading adopted: with */
/* the proxy Hessian factored as H = (I + U) D (I + U)^T, U strictly upper   */
/* triangular by 256-column blocks, block b of each row is encoded from       */
/*   w~_b = w_b + (w - w_hat)_{<b} U_{<b,b}                                  */
/* (the errors of all earlier blocks, fed forward through U), and the error  */
/* w - w_hat of block b is kept for the blocks after it.  Then               */
/* (w - w_hat)(I + U) = (w~ - w_hat) blockwise, so the proxy loss            */
/* tr((w - w_hat) H (w - w_hat)^T) equals the D-weighted quantization error   */
/* of the adjusted blocks.  binary32, fixed order: each w~ element starts at */
/* w and adds the products delta_i * U[i][j] by fma in ascending i.          */
/* w: fp32 [n][k]; u: fp32 [k][k] row-major (only the block strictly upper   */
/* part is read); outputs as orc_encode32, err = per block sum of            */
/* (w~ - w_hat)^2 in fold order.                                             */
/* ======================================================================== */
void orc_ldlq32(const float* w, int64_t n, int64_t k, const float* u, const uint16_t* cb, float gain, int refits,
                uint8_t* codes, uint16_t* scales, float* err) {
  int64_t nb = k / 256;
  float* delta = (float*)malloc(sizeof(float) * (size_t)k);
  float wt[256], wh[256];
  for (int64_t r = 0; r < n; ++r) {
    const float* wr = w + r * k;
    for (int64_t b = 0; b < nb; ++b) {
      for (int j = 0; j < 256; ++j) {
        int64_t col = b * 256 + j;
        float acc = wr[col];
        for (int64_t i = 0; i < b * 256; ++i) acc = fmaf(delta[i], u[i * k + col], acc);
        wt[j] = acc;
      }
      float e;
      encode_block32(wt, cb, gain, refits, codes + r * (k / 4) + b * 64, &scales[r * nb + b], &e, wh);
      if (err) err[r * nb + b] = e;
      for (int j = 0; j < 256; ++j) delta[b * 256 + j] = wr[b * 256 + j] - wh[j];
    }
  }
  free(delta);
}
