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
// Work split.  One CTA of 128 threads encodes one block at a time (grid-stride
// over the n * k/256 blocks).  Warp w evaluates the predecessor states
// s = 2w and 2w+1; lane l serves new state ns = l & 7 and the eight codes
// c = 8*(8*(l>>3) + i) + ns, i = 0..7, whose scaled entries and norms (for both
// of its states) it keeps in registers for the whole pass.  Per group: sixteen
// candidates per lane, a minimum over the four lanes that share ns (two
// shuffles), one shared-memory exchange between the four warps with one
// barrier, after which warp w reduces the four partial minima of new states 2w
// (lanes 0-15) and 2w+1 (lanes 16-31) and records their back-pointers (code
// high bits | predecessor state).  The bound is the FP32 pipe: 5 FP32
// operations per candidate, 2048 candidates per group.
#pragma once

#include <stddef.h>

#include "tq_common.cuh"

namespace tq {

constexpr int kEncWarps = 4;                 // each warp: two predecessor states
constexpr int kEncThreads = 32 * kEncWarps;  // two weights of the block per thread

struct EncShared {
  float w[256];          // the block's rotated weights
  uint8_t cur[64];       // codes of the last pass (16-byte aligned: offset 1024)
  uint8_t best[64];      // codes of the best pass so far (offset 1088)
  float red[2][128];     // fold-sum scratch
  float kt[2][8][4];     // per group: [buffer][new state][warp] least cost
  uint32_t kc[2][8][4];  //   and its key (code << 3 | predecessor state)
  uint8_t bp[64][8];     // back-pointers: (code & 0xF8) | predecessor state
  float jf[8];           // final path cost per end state
  float bc[2];           // broadcast slots
};
static_assert(offsetof(EncShared, best) % 16 == 0, "codes are stored with 16-byte writes");

__device__ __forceinline__ float enc_rnd16(float x) { return __half2float(__float2half_rn(x)); }

__device__ __forceinline__ uint16_t enc_f16_bits(float x) { return __half_as_ushort(__float2half_rn(x)); }

// Fold-order sums (v[i] += v[i + h] for h = 128 ... 1) of two 256-element
// vectors a and b, thread t holding elements t and t + 128 of each; returned
// to every thread.
__device__ __forceinline__ float2 enc_fold2(EncShared& S, float a0, float a1, float b0, float b1) {
  const int tid = threadIdx.x;
  S.red[0][tid] = __fadd_rn(a0, a1);
  S.red[1][tid] = __fadd_rn(b0, b1);
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
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, ns = lane & 7, hq = lane >> 3;
  const float sigma = __half2float(__ushort_as_half(scale_bits));
  float D[2][8][4], N[2][8];
#pragma unroll
  for (int sl = 0; sl < 2; ++sl)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t s = 2 * warp + sl, c = ((uint32_t)(hq * 8 + i) << 3) | (uint32_t)ns;
      const uint2 e = __ldg(reinterpret_cast<const uint2*>(cb + (((s << 8) | c) << 2)));
      const float2 e01 = h2_to_f2(e.x), e23 = h2_to_f2(e.y);
      D[sl][i][0] = enc_rnd16(__fmul_rn(sigma, e01.x));
      D[sl][i][1] = enc_rnd16(__fmul_rn(sigma, e01.y));
      D[sl][i][2] = enc_rnd16(__fmul_rn(sigma, e23.x));
      D[sl][i][3] = enc_rnd16(__fmul_rn(sigma, e23.y));
      N[sl][i] = fmaf(D[sl][i][3], D[sl][i][3],
                      fmaf(D[sl][i][2], D[sl][i][2], fmaf(D[sl][i][1], D[sl][i][1], __fmul_rn(D[sl][i][0], D[sl][i][0]))));
    }
  const float inf = __int_as_float(0x7f800000);
  float J0 = (warp == 0) ? 0.0f : inf, J1 = inf;  // path costs of states 2w and 2w+1
  for (int g = 0; g < 64; ++g) {
    const float4 wg = *reinterpret_cast<const float4*>(S.w + 4 * g);
    const float u0 = -2.0f * wg.x, u1 = -2.0f * wg.y, u2 = -2.0f * wg.z, u3 = -2.0f * wg.w;
    // candidate index x = 2i + sl orders the lane's candidates by (code, state)
    float tv[16];
    int ti[16];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int sl = 0; sl < 2; ++sl) {
        float t = __fadd_rn(sl ? J1 : J0, N[sl][i]);
        t = fmaf(u3, D[sl][i][3], t);
        t = fmaf(u2, D[sl][i][2], t);
        t = fmaf(u1, D[sl][i][1], t);
        tv[2 * i + sl] = fmaf(u0, D[sl][i][0], t);
        ti[2 * i + sl] = 2 * i + sl;
      }
    // least (t, x) by a tree; the right operand holds the larger x, so it wins
    // only when strictly smaller
#pragma unroll
    for (int h = 1; h < 16; h <<= 1)
#pragma unroll
      for (int x = 0; x < 16; x += 2 * h)
        if (tv[x + h] < tv[x]) {
          tv[x] = tv[x + h];
          ti[x] = ti[x + h];
        }
    float bt = tv[0];
    uint32_t bk = ((((uint32_t)(hq * 8 + (ti[0] >> 1)) << 3) | (uint32_t)ns) << 3) | (uint32_t)(2 * warp + (ti[0] & 1));
#pragma unroll
    for (int o = 8; o <= 16; o <<= 1) {
      const float to = __shfl_xor_sync(0xffffffffu, bt, o);
      const uint32_t ko = __shfl_xor_sync(0xffffffffu, bk, o);
      if (enc_before(to, ko, bt, bk)) {
        bt = to;
        bk = ko;
      }
    }
    const int buf = g & 1;
    if (hq == 0) {
      S.kt[buf][ns][warp] = bt;
      S.kc[buf][ns][warp] = bk;
    }
    __syncthreads();
    // warp w now owns new states 2w (lanes 0-15) and 2w+1 (lanes 16-31);
    // lane & 3 picks the partial minimum of one warp
    const int nn = 2 * warp + (lane >> 4);
    float t2 = S.kt[buf][nn][lane & 3];
    uint32_t k2 = S.kc[buf][nn][lane & 3];
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      const float to = __shfl_xor_sync(0xffffffffu, t2, o);
      const uint32_t ko = __shfl_xor_sync(0xffffffffu, k2, o);
      if (enc_before(to, ko, t2, k2)) {
        t2 = to;
        k2 = ko;
      }
    }
    J0 = __shfl_sync(0xffffffffu, t2, 0);
    J1 = __shfl_sync(0xffffffffu, t2, 16);
    if ((lane & 15) == 0) S.bp[g][nn] = (uint8_t)(((k2 >> 3) & 0xF8u) | (k2 & 7u));
  }
  if (lane == 0) {
    S.jf[2 * warp] = J0;
    S.jf[2 * warp + 1] = J1;
  }
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
__global__ void __launch_bounds__(kEncThreads, 4)
    encode_kernel(const float* __restrict__ w, long long blocks, const uint16_t* __restrict__ cb, float gain,
                  int refits, uint8_t* __restrict__ codes, uint16_t* __restrict__ scales, float* __restrict__ err) {
  __shared__ __align__(16) EncShared S;
  const int tid = threadIdx.x;
  for (long long blk = blockIdx.x; blk < blocks; blk += gridDim.x) {
    const float w0 = __ldg(w + blk * 256 + tid), w1 = __ldg(w + blk * 256 + tid + 128);
    S.w[tid] = w0;
    S.w[tid + 128] = w1;
    const float ss = enc_fold2(S, __fmul_rn(w0, w0), __fmul_rn(w1, w1), 0.0f, 0.0f).x;
    float rs = __fmul_rn(__fsqrt_rn(__fmul_rn(ss, 0.00390625f)), gain);
    if (!(rs <= 65504.0f)) rs = 65504.0f;
    uint16_t best_scale = enc_f16_bits(rs);
    float best_j = enc_viterbi(S, cb, best_scale, S.best);
    for (int it = 0; it < refits; ++it) {
      const float e0 = enc_path_value(cb, S.best, tid), e1 = enc_path_value(cb, S.best, tid + 128);
      const float2 nd = enc_fold2(S, __fmul_rn(w0, e0), __fmul_rn(w1, e1), __fmul_rn(e0, e0), __fmul_rn(e1, e1));
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
      const float d0 = __fsub_rn(w0, enc_rnd16(__fmul_rn(sigma, enc_path_value(cb, S.best, tid))));
      const float d1 = __fsub_rn(w1, enc_rnd16(__fmul_rn(sigma, enc_path_value(cb, S.best, tid + 128))));
      const float e2 = enc_fold2(S, __fmul_rn(d0, d0), __fmul_rn(d1, d1), 0.0f, 0.0f).x;
      if (tid == 0) err[blk] = e2;
    }
    __syncthreads();
  }
}

}  // namespace tq
