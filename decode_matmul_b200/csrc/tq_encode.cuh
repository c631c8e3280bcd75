// tq_encode.cuh -- trellis encoder: least-squared-error code path per
// 256-weight block by dynamic programming over the 8 states (Viterbi).
//
// "Pingala-8" landing page, "How it works": the groups of four weights are
// coded in order; the state carried from one group selects the values the
// next group may use, so the code lands closer to the weights at the same
// bits; a random Hadamard rotation is applied to the weights first (tq_rht
// on the weight rows gives exactly the rotation the matmul applies to the
// activations).  The pages give no encoding procedure.  This kernel:
//   - fits the block's fp16 scale as fp16_RNE(RMS(block) * gain) (clamped to
//     65504), finds the least-cost path from state 0 (end state free), then
//     refits the scale by least squares on that path (sum w*e / sum e*e, e the
//     unscaled codebook values) up to `refits` times, keeping a refit only
//     when its path costs less;
//   - takes every decision in binary32 in one fixed order, so the result is
//     reproducible bit for bit:
//       D[s][c] = fp16_RNE(scale * cb[s][c]),
//       N[s][c] = fma(D3,D3, fma(D2,D2, fma(D1,D1, D0*D0))),
//       candidate (s, c) of a group w, u = -2w:
//         t = fma(u0,D0, fma(u1,D1, fma(u2,D2, fma(u3,D3, J[s] + N[s][c])))),
//       (t is the squared error minus |w|^2, a constant of the group);
//       J'[c & 7] = the least t, ties to the smaller code, then the smaller
//       predecessor state; block sums in fold order v[i] += v[i+h],
//       h = 128, 64, ..., 1.
//
// Work split.  One CTA of 256 threads encodes one block at a time (grid-stride
// over the n * k/256 blocks).  Warp w evaluates predecessor state s = w; lane
// l serves new state ns = l & 7 and the eight codes c = 8*(8*(l>>3) + i) + ns,
// i = 0..7, whose scaled entries and norms it keeps in registers for the whole
// pass.  Per group: eight candidates per lane, a minimum over the four lanes
// that share ns (two shuffles), one shared-memory exchange between the eight
// warps with one barrier, after which warp s reduces the eight predecessors of
// new state s and lane 0 records the back-pointer (code high bits | state).
// The bound is the FP32 pipe: 5 FP32 operations per candidate, 2048
// candidates per group.
#pragma once

#include <stddef.h>

#include "tq_common.cuh"

namespace tq {

constexpr int kEncThreads = 256;

struct EncShared {
  float w[256];          // the block's rotated weights
  uint8_t cur[64];       // codes of the last pass (16-byte aligned: offset 1024)
  uint8_t best[64];      // codes of the best pass so far (offset 1088)
  float red[2][256];     // fold-sum scratch
  float kt[2][8][8];     // per group: [buffer][predecessor s][new state] least cost
  uint32_t kc[2][8][8];  //   and its code
  uint8_t bp[64][8];     // back-pointers: (code & 0xF8) | predecessor state
  float jf[8];           // final path cost per end state
  float bc[2];           // broadcast slots
};
static_assert(offsetof(EncShared, best) % 16 == 0, "codes are stored with 16-byte writes");

__device__ __forceinline__ float enc_rnd16(float x) { return __half2float(__float2half_rn(x)); }

__device__ __forceinline__ uint16_t enc_f16_bits(float x) { return __half_as_ushort(__float2half_rn(x)); }

// Fold-order sums of two values held one per thread (v[i] += v[i + h] for
// h = 128 ... 1), returned to every thread.
__device__ __forceinline__ float2 enc_fold2(EncShared& S, float a, float b) {
  const int tid = threadIdx.x;
  S.red[0][tid] = a;
  S.red[1][tid] = b;
  __syncthreads();
  if (tid < 128) {
    S.red[0][tid] = __fadd_rn(S.red[0][tid], S.red[0][tid + 128]);
    S.red[1][tid] = __fadd_rn(S.red[1][tid], S.red[1][tid + 128]);
  }
  __syncthreads();
  if (tid < 64) {
    S.red[0][tid] = __fadd_rn(S.red[0][tid], S.red[0][tid + 64]);
    S.red[1][tid] = __fadd_rn(S.red[1][tid], S.red[1][tid + 64]);
  }
  __syncthreads();
  if (tid < 32) {
    float x = __fadd_rn(S.red[0][tid], S.red[0][tid + 32]);
    float y = __fadd_rn(S.red[1][tid], S.red[1][tid + 32]);
#pragma unroll
    for (int h = 16; h >= 1; h >>= 1) {
      x = __fadd_rn(x, __shfl_down_sync(0xffffffffu, x, h));
      y = __fadd_rn(y, __shfl_down_sync(0xffffffffu, y, h));
    }
    if (tid == 0) {
      S.bc[0] = x;
      S.bc[1] = y;
    }
  }
  __syncthreads();
  return make_float2(S.bc[0], S.bc[1]);
}

// Unscaled codebook value of weight i of the block under the codes `cd`.
__device__ __forceinline__ float enc_path_value(const uint16_t* __restrict__ cb, const uint8_t* cd, int i) {
  const int g = i >> 2;
  const uint32_t st = g ? (cd[g - 1] & 7u) : 0u;
  return __half2float(__ushort_as_half(__ldg(cb + (((st << 8) | cd[g]) << 2) + (i & 3))));
}

// (t, key) pairs ordered by t, then key; keys are distinct.
__device__ __forceinline__ bool enc_before(float t_o, uint32_t k_o, float t, uint32_t k) {
  return t_o < t || (t_o == t && k_o < k);
}

// One Viterbi pass over the block in S.w at fp16 scale `scale_bits`; the codes
// go to `out` (shared memory) and the least final cost is returned to every
// thread.
__device__ float enc_viterbi(EncShared& S, const uint16_t* __restrict__ cb, uint16_t scale_bits, uint8_t* out) {
  const int tid = threadIdx.x, s = tid >> 5, lane = tid & 31, ns = lane & 7, hq = lane >> 3;
  const float sigma = __half2float(__ushort_as_half(scale_bits));
  float D[8][4], N[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t c = ((uint32_t)(hq * 8 + i) << 3) | (uint32_t)ns;
    const uint2 e = __ldg(reinterpret_cast<const uint2*>(cb + ((((uint32_t)s << 8) | c) << 2)));
    const float2 e01 = h2_to_f2(e.x), e23 = h2_to_f2(e.y);
    D[i][0] = enc_rnd16(__fmul_rn(sigma, e01.x));
    D[i][1] = enc_rnd16(__fmul_rn(sigma, e01.y));
    D[i][2] = enc_rnd16(__fmul_rn(sigma, e23.x));
    D[i][3] = enc_rnd16(__fmul_rn(sigma, e23.y));
    N[i] = fmaf(D[i][3], D[i][3], fmaf(D[i][2], D[i][2], fmaf(D[i][1], D[i][1], __fmul_rn(D[i][0], D[i][0]))));
  }
  float J = (s == 0) ? 0.0f : __int_as_float(0x7f800000);
  for (int g = 0; g < 64; ++g) {
    const float4 wg = *reinterpret_cast<const float4*>(S.w + 4 * g);
    const float u0 = -2.0f * wg.x, u1 = -2.0f * wg.y, u2 = -2.0f * wg.z, u3 = -2.0f * wg.w;
    float bt = 0.0f;
    int bi = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float t = __fadd_rn(J, N[i]);
      t = fmaf(u3, D[i][3], t);
      t = fmaf(u2, D[i][2], t);
      t = fmaf(u1, D[i][1], t);
      t = fmaf(u0, D[i][0], t);
      if (i == 0 || t < bt) {
        bt = t;
        bi = i;
      }
    }
    uint32_t bc = ((uint32_t)(hq * 8 + bi) << 3) | (uint32_t)ns;
#pragma unroll
    for (int o = 8; o <= 16; o <<= 1) {
      const float to = __shfl_xor_sync(0xffffffffu, bt, o);
      const uint32_t co = __shfl_xor_sync(0xffffffffu, bc, o);
      if (enc_before(to, co, bt, bc)) {
        bt = to;
        bc = co;
      }
    }
    const int buf = g & 1;
    if (hq == 0) {
      S.kt[buf][s][ns] = bt;
      S.kc[buf][s][ns] = bc;
    }
    __syncthreads();
    // warp s now owns new state s; lane & 7 is the predecessor state
    const int sp = lane & 7;
    float t2 = S.kt[buf][sp][s];
    uint32_t k2 = (S.kc[buf][sp][s] << 3) | (uint32_t)sp;
#pragma unroll
    for (int o = 1; o <= 4; o <<= 1) {
      const float to = __shfl_xor_sync(0xffffffffu, t2, o);
      const uint32_t ko = __shfl_xor_sync(0xffffffffu, k2, o);
      if (enc_before(to, ko, t2, k2)) {
        t2 = to;
        k2 = ko;
      }
    }
    J = t2;
    if (lane == 0) S.bp[g][s] = (uint8_t)(((k2 >> 3) & 0xF8u) | (k2 & 7u));
  }
  if (lane == 0) S.jf[s] = J;
  __syncthreads();
  if (tid == 0) {
    int st = 0;
    for (int q = 1; q < 8; ++q)
      if (S.jf[q] < S.jf[st]) st = q;
    S.bc[0] = S.jf[st];
    for (int g = 63; g >= 0; --g) {
      const uint32_t b = S.bp[g][st];
      out[g] = (uint8_t)((b & 0xF8u) | (uint32_t)st);
      st = (int)(b & 7u);
    }
  }
  __syncthreads();
  return S.bc[0];
}

// Encode n rows x k rotated weights (see the file comment).  blocks = n * k/256.
__global__ void __launch_bounds__(kEncThreads, 3)
    encode_kernel(const float* __restrict__ w, long long blocks, const uint16_t* __restrict__ cb, float gain,
                  int refits, uint8_t* __restrict__ codes, uint16_t* __restrict__ scales, float* __restrict__ err) {
  __shared__ __align__(16) EncShared S;
  const int tid = threadIdx.x;
  for (long long blk = blockIdx.x; blk < blocks; blk += gridDim.x) {
    const float wv = __ldg(w + blk * 256 + tid);
    S.w[tid] = wv;
    const float ss = enc_fold2(S, __fmul_rn(wv, wv), 0.0f).x;
    float rs = __fmul_rn(__fsqrt_rn(__fmul_rn(ss, 0.00390625f)), gain);
    if (!(rs <= 65504.0f)) rs = 65504.0f;
    uint16_t best_scale = enc_f16_bits(rs);
    float best_j = enc_viterbi(S, cb, best_scale, S.best);
    for (int it = 0; it < refits; ++it) {
      const float e = enc_path_value(cb, S.best, tid);
      const float2 nd = enc_fold2(S, __fmul_rn(wv, e), __fmul_rn(e, e));
      if (!(nd.y > 0.0f)) break;
      float r = __fdiv_rn(nd.x, nd.y);
      if (isnan(r)) break;
      r = fminf(fmaxf(r, -65504.0f), 65504.0f);
      const uint16_t s1 = enc_f16_bits(r);
      if (s1 == best_scale) break;
      const float j1 = enc_viterbi(S, cb, s1, S.cur);
      if (!(j1 < best_j)) break;
      best_j = j1;
      best_scale = s1;
      if (tid < 16) reinterpret_cast<uint32_t*>(S.best)[tid] = reinterpret_cast<const uint32_t*>(S.cur)[tid];
      __syncthreads();
    }
    if (tid < 4) reinterpret_cast<uint4*>(codes + blk * 64)[tid] = reinterpret_cast<const uint4*>(S.best)[tid];
    if (tid == 0) scales[blk] = best_scale;
    if (err != nullptr) {
      const float sigma = __half2float(__ushort_as_half(best_scale));
      const float wh = enc_rnd16(__fmul_rn(sigma, enc_path_value(cb, S.best, tid)));
      const float d = __fsub_rn(wv, wh);
      const float e2 = enc_fold2(S, __fmul_rn(d, d), 0.0f).x;
      if (tid == 0) err[blk] = e2;
    }
    __syncthreads();
  }
}

}  // namespace tq
