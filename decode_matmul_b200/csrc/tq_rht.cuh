// tq_rht.cuh -- randomized Walsh-Hadamard transform of activations.
//
// "Pingala-8" landing page, "How it works": a random Hadamard rotation is
// applied before the weights are encoded; "Bonsai 2 27B" article, change of
// basis: the rotation lives in the stored weights and the matching transform
// runs on the activations at run time.  Here: x' = H_512 D x per 512-block,
// H in natural (Sylvester) order, orthonormal (1/sqrt(512)), D = diag(+-1)
// drawn from SplitMix64.
//
// One warp owns one 512-block of one row.  Lane l holds elements 16l..16l+15
// in registers: index bits 0-3 are register bits, bits 4-8 are lane bits.
// The 9 butterfly stages are 4 in-register stages and 5 shfl.xor stages.
#pragma once

#include "tq_common.cuh"

namespace tq {

// In-place unnormalised Sylvester transform of the 512 values held by a warp.
__device__ __forceinline__ void wht512_warp(float v[16]) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      if (!(r & h)) {
        float a = v[r], b = v[r | h];
        v[r] = a + b;
        v[r | h] = a - b;
      }
    }
  }
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    // upper lane: o - v, lower lane: v + o -- one exact fma with a +-1 factor
    const float sg = (lane & m) ? -1.f : 1.f;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      const float o = __shfl_xor_sync(0xffffffffu, v[r], m);
      v[r] = fmaf(sg, v[r], o);
    }
  }
}

// Load this lane's 16 bf16 inputs of block `blk` of row `x_row`, apply D,
// transform, scale by 1/sqrt(512).  Returns values for elements 16*lane + r.
__device__ __forceinline__ void rht512_warp(const uint16_t* __restrict__ x_row, int blk, uint64_t seed,
                                            float v[16]) {
  const int lane = threadIdx.x & 31;
  const int base = blk * 512 + lane * 16;
  const uint4* src = reinterpret_cast<const uint4*>(x_row + base);
  uint4 p0 = src[0], p1 = src[1];
  uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t lo = w[i] & 0xFFFFu, hi = w[i] >> 16;
    uint32_t k0 = (uint32_t)(base + 2 * i), k1 = k0 + 1;
    // D: flip the sign bit of the bf16 value where d[k] = -1 (exact)
    if (rht_sign_negative(seed, k0)) lo ^= 0x8000u;
    if (rht_sign_negative(seed, k1)) hi ^= 0x8000u;
    v[2 * i] = bf16_bits_to_f(lo);
    v[2 * i + 1] = bf16_bits_to_f(hi);
  }
  wht512_warp(v);
  const float inv = 0.044194173824159216f;  // 1/sqrt(512)
#pragma unroll
  for (int r = 0; r < 16; ++r) v[r] *= inv;
}

// Offset of element kk of token t in "fragment order", the small-batch
// kernel's x' layout.  Tokens go in groups of 8 (group t / 8 takes 8 k
// elements per feature); inside a group's 256-weight block b, the 64 groups
// of 4 weights (group 16q + j is read by lanes with q = lane % 4 at MMA step
// j) of token g = t % 8 are stored as [j / 2][g][q][j % 2]: a lane's quads of
// steps j and j + 1 are one 16-byte load, and the 32 lanes (g, q) of a step
// pair read 512 contiguous bytes (four shared-memory-sized wavefronts; with
// one row per token they touched eight lines).  Buffers hold whole groups of
// 8 tokens; the rows past m are never written and feed only MMA columns whose
// outputs are discarded.
__host__ __device__ __forceinline__ size_t xt_pos(int t, int kk, int k) {
  const int b = kk >> 8, G = (kk & 255) >> 2, e = kk & 3;
  const int j = G & 15, q = G >> 4;
  return (size_t)(t >> 3) * 8 * k + (size_t)((b << 3) + (j >> 1)) * 256 + ((t & 7) << 5) + (q << 3) + ((j & 1) << 2) + e;
}

// Standalone RHT.  CTA (blk, y) transforms 512-block `blk` of rows 8y + warp
// (grid-stride in y): the 512 diagonal signs of the block are hashed once per
// CTA (two per thread, packed by ballot into shared memory, before the wait for
// the preceding kernel) and shared by its eight rows.  MODE 0: fp32 row-major;
// 1: fp16 row-major; 2: fp16 in fragment order (xt_pos).
template <int MODE>
__global__ void __launch_bounds__(256) rht_kernel(const uint16_t* __restrict__ x, int m, int k, uint64_t seed,
                                                  void* __restrict__ out) {
  __shared__ uint32_t smask[16];  // bit e % 32 of word e / 32: d[512 blk + e] = -1
  const int blk = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t e0 = (uint32_t)blk * 512u + (uint32_t)tid;
  const uint32_t b0 = __ballot_sync(0xffffffffu, rht_sign_negative(seed, e0));
  const uint32_t b1 = __ballot_sync(0xffffffffu, rht_sign_negative(seed, e0 + 256u));
  if (lane == 0) {
    smask[warp] = b0;
    smask[8 + warp] = b1;
  }
  __syncthreads();
  const uint32_t mask16 = (smask[lane >> 1] >> ((lane & 1) * 16)) & 0xFFFFu;  // elements 16 lane .. +15
  pdl_wait();
  pdl_launch_dependents();
  for (int rg = blockIdx.y; rg * 8 < m; rg += gridDim.y) {
    const int row = rg * 8 + warp;
    if (row >= m) break;
    const int base = blk * 512 + lane * 16;
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)row * k + base);
    const uint4 p0 = src[0], p1 = src[1];
    const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    float v[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      // D: flip the sign bit of the bf16 value where d = -1 (exact)
      const uint32_t f = ((mask16 >> (2 * i)) & 1u) << 15 | ((mask16 >> (2 * i + 1)) & 1u) << 31;
      const uint32_t ww = w[i] ^ f;
      v[2 * i] = bf16_bits_to_f(ww & 0xFFFFu);
      v[2 * i + 1] = bf16_bits_to_f(ww >> 16);
    }
    wht512_warp(v);
    const float inv = 0.044194173824159216f;  // 1/sqrt(512)
#pragma unroll
    for (int r = 0; r < 16; ++r) v[r] *= inv;
    const size_t o = (size_t)row * k + (size_t)blk * 512 + lane * 16;
    if (MODE == 1) {
      uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(out) + o);
      dst[0] = make_uint4(f2_to_h2(v[0], v[1]), f2_to_h2(v[2], v[3]), f2_to_h2(v[4], v[5]), f2_to_h2(v[6], v[7]));
      dst[1] = make_uint4(f2_to_h2(v[8], v[9]), f2_to_h2(v[10], v[11]), f2_to_h2(v[12], v[13]),
                          f2_to_h2(v[14], v[15]));
    } else if (MODE == 2) {
#pragma unroll
      for (int r4 = 0; r4 < 4; ++r4) {
        const int kk = blk * 512 + lane * 16 + 4 * r4;
        *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(out) + xt_pos(row, kk, k)) =
            make_uint2(f2_to_h2(v[4 * r4], v[4 * r4 + 1]), f2_to_h2(v[4 * r4 + 2], v[4 * r4 + 3]));
      }
    } else {
      float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + o);
#pragma unroll
      for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
  }
}

// Grid of rht_kernel for m rows of k features.
inline dim3 rht_grid(int m, int k) {
  const int groups = (m + 7) / 8;
  return dim3((unsigned)(k / 512), (unsigned)(groups < 65535 ? groups : 65535));
}

// fp16 [m][k] row-major -> fragment order (one thread per group of 4).
__global__ void __launch_bounds__(256) frag_permute_kernel(const uint16_t* __restrict__ x, int m, int k,
                                                           uint16_t* __restrict__ out) {
  const long long groups = (long long)m * (k / 4);
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < groups;
       i += (long long)gridDim.x * blockDim.x) {
    const long long row = i / (k / 4);
    const int kk = (int)(i - row * (k / 4)) * 4;
    *reinterpret_cast<uint2*>(out + xt_pos((int)row, kk, k)) = *reinterpret_cast<const uint2*>(x + row * k + kk);
  }
}

}  // namespace tq
