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

// One encoder launch: blocks (r, j), r < n, j < nbl, read at w + r*ldw + 256j
// and written to output block column b0 + j of rows with kb blocks.  With
// `delta`, the launch also stores delta = w_ref - w_hat for those columns
// (the error the block LDLQ feeds forward).
struct EncArgs {
  const float* w;
  long long ldw;
  long long blocks;  // n * nbl
  int nbl, b0, kb;
  const uint16_t* cb;
  float gain;
  int refits;
  uint8_t* codes;     // [n][kb * 64]
  uint16_t* scales;   // [n][kb]
  float* err;         // [n][kb] or null
  const float* w_ref; // [n][ldr], with delta
  long long ldr;
  float* delta;       // [n][ldr] or null
};

__global__ void __launch_bounds__(kEncThreads, 4) encode_kernel(EncArgs a) {
  __shared__ __align__(16) EncShared S;
  const int tid = threadIdx.x;
  const uint16_t* __restrict__ cb = a.cb;
  for (long long blk = blockIdx.x; blk < a.blocks; blk += gridDim.x) {
    const long long r = blk / a.nbl;
    const int j = (int)(blk - r * a.nbl);
    const float* wb = a.w + r * a.ldw + 256LL * j;
    const long long ob = r * a.kb + a.b0 + j;
    const float w0 = __ldg(wb + tid), w1 = __ldg(wb + tid + 128);
    S.w[tid] = w0;
    S.w[tid + 128] = w1;
    const float ss = enc_fold2(S, __fmul_rn(w0, w0), __fmul_rn(w1, w1), 0.0f, 0.0f).x;
    float rs = __fmul_rn(__fsqrt_rn(__fmul_rn(ss, 0.00390625f)), a.gain);
    if (!(rs <= 65504.0f)) rs = 65504.0f;
    uint16_t best_scale = enc_f16_bits(rs);
    float best_j = enc_viterbi(S, cb, best_scale, S.best);
    for (int it = 0; it < a.refits; ++it) {
      const float e0 = enc_path_value(cb, S.best, tid), e1 = enc_path_value(cb, S.best, tid + 128);
      const float2 nd = enc_fold2(S, __fmul_rn(w0, e0), __fmul_rn(w1, e1), __fmul_rn(e0, e0), __fmul_rn(e1, e1));
      if (!(nd.y > 0.0f)) break;
      float q = __fdiv_rn(nd.x, nd.y);
      if (isnan(q)) break;
      q = fminf(fmaxf(q, -65504.0f), 65504.0f);
      const uint16_t s1 = enc_f16_bits(q);
      if (s1 == best_scale) break;
      const float j1 = enc_viterbi(S, cb, s1, S.cur);
      if (!(j1 < best_j)) break;
      best_j = j1;
      best_scale = s1;
      if (tid < 16) reinterpret_cast<uint32_t*>(S.best)[tid] = reinterpret_cast<const uint32_t*>(S.cur)[tid];
      __syncthreads();
    }
    if (tid < 4) reinterpret_cast<uint4*>(a.codes + ob * 64)[tid] = reinterpret_cast<const uint4*>(S.best)[tid];
    if (tid == 0) a.scales[ob] = best_scale;
    if (a.err != nullptr || a.delta != nullptr) {
      const float sigma = __half2float(__ushort_as_half(best_scale));
      const float h0 = enc_rnd16(__fmul_rn(sigma, enc_path_value(cb, S.best, tid)));
      const float h1 = enc_rnd16(__fmul_rn(sigma, enc_path_value(cb, S.best, tid + 128)));
      if (a.delta != nullptr) {
        const long long o = r * a.ldr + 256LL * (a.b0 + j);
        a.delta[o + tid] = __fsub_rn(__ldg(a.w_ref + o + tid), h0);
        a.delta[o + tid + 128] = __fsub_rn(__ldg(a.w_ref + o + tid + 128), h1);
      }
      if (a.err != nullptr) {
        const float d0 = __fsub_rn(w0, h0), d1 = __fsub_rn(w1, h1);
        const float e2 = enc_fold2(S, __fmul_rn(d0, d0), __fmul_rn(d1, d1), 0.0f, 0.0f).x;
        if (tid == 0) a.err[ob] = e2;
      }
    }
    __syncthreads();
  }
}

// ---- block LDLQ feedback --------------------------------------------------------
// LDLQ, named on the "Pingala-8" landing page ("How it works"): the coding
// error of the columns already coded is fed forward.  With the proxy Hessian factored as
// H = (I + U) D (I + U)^T (U strictly upper by 256-column blocks), block b of
// each row is encoded from
//   wt[r][j] = w[r][256b + j] + sum_{i < 256b} delta[r][i] * U[i][256b + j],
// each element summed by fma in ascending i (binary32), delta = w - w_hat of the
// blocks already coded.  A plain tiled SIMT GEMM: 16 TM x 64 outputs per CTA
// (TM = 4, or 2 when there are too few rows to fill the GPU with 64-row
// tiles), a TM x 4 register tile per thread, 32-deep k tiles in shared
// memory; every output keeps its own accumulator, so the order per output is
// ascending i.
constexpr int kFbCols = 64, kFbDepth = 32;

template <int TM>
__global__ void __launch_bounds__(256) ldlq_feedback_kernel(const float* __restrict__ w, const float* __restrict__ delta,
                                                            const float* __restrict__ u, int n, int k, int b,
                                                            float* __restrict__ wt) {
  constexpr int ROWS = 16 * TM;                              // rows of the CTA tile
  constexpr int PER = ROWS * kFbDepth / 256;                 // delta values each thread stages (8 or 4)
  __shared__ __align__(16) float As[kFbDepth][ROWS + 4];     // delta tile, [i][row]
  __shared__ __align__(16) float Bs[kFbDepth][kFbCols];      // U tile, [i][col]
  const int tid = threadIdx.x, tr = tid >> 4, tc = tid & 15;
  const int row0 = blockIdx.x * ROWS, col0 = blockIdx.y * kFbCols;
  const long long cw = 256LL * b + col0 + tc * 4;  // this thread's first column in w / U
  float acc[TM][4];
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int r = row0 + tr * TM + i;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < n) v = __ldg(reinterpret_cast<const float4*>(w + (long long)r * k + cw));
    acc[i][0] = v.x;
    acc[i][1] = v.y;
    acc[i][2] = v.z;
    acc[i][3] = v.w;
  }
  const int lr = tid / (kFbDepth / PER), lk = (tid % (kFbDepth / PER)) * PER;  // delta loads: row lr, PER values
  const int ui = tid >> 3, uc = (tid & 7) * 8;                                 // U tile loads: row ui, 8 values
  const int kend = 256 * b;
  for (int k0 = 0; k0 < kend; k0 += kFbDepth) {
    float dv[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) dv[e] = 0.f;
    if (row0 + lr < n) {
      const float* dp = delta + (long long)(row0 + lr) * k + k0 + lk;
#pragma unroll
      for (int e = 0; e < PER; e += 4) {
        const float4 d4 = __ldg(reinterpret_cast<const float4*>(dp + e));
        dv[e] = d4.x;
        dv[e + 1] = d4.y;
        dv[e + 2] = d4.z;
        dv[e + 3] = d4.w;
      }
    }
    const float* up = u + (long long)(k0 + ui) * k + 256LL * b + col0 + uc;
    const float4 u0 = __ldg(reinterpret_cast<const float4*>(up)), u1 = __ldg(reinterpret_cast<const float4*>(up + 4));
#pragma unroll
    for (int e = 0; e < PER; ++e) As[lk + e][lr] = dv[e];
    *reinterpret_cast<float4*>(&Bs[ui][uc]) = u0;
    *reinterpret_cast<float4*>(&Bs[ui][uc + 4]) = u1;
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kFbDepth; ++kk) {
      float a4[TM];
      if (TM == 4) {
        const float4 av = *reinterpret_cast<const float4*>(&As[kk][tr * 4]);
        a4[0] = av.x;
        a4[1] = av.y;
        a4[2 % TM] = av.z;
        a4[3 % TM] = av.w;
      } else {
        const float2 av = *reinterpret_cast<const float2*>(&As[kk][tr * 2]);
        a4[0] = av.x;
        a4[1] = av.y;
      }
      const float4 bv = *reinterpret_cast<const float4*>(&Bs[kk][tc * 4]);
      const float b4[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a4[i], b4[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int r = row0 + tr * TM + i;
    if (r < n)
      *reinterpret_cast<float4*>(wt + (long long)r * 256 + col0 + tc * 4) =
          make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
  }
}

}  // namespace tq
