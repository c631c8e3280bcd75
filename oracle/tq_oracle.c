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
