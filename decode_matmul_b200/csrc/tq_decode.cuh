// tq_decode.cuh -- materialise the decoded fp16 weight (inspection/test export).
//
// "Pingala-8" landing page, "How it works": groups of 4 weights are coded in
// order and the state carried from the previous group selects the codebook
// of the next one.  Layout used here: state = previous code & 7, reset to 0
// at every 256-weight block; W = fp16_RNE(scale * codebook[state][code]).
#pragma once

#include "tq_common.cuh"

namespace tq {

// One thread per group of 4 weights.  The product of two fp16 values is exact
// in fp32, so __hmul2 (one IEEE round-to-nearest-even) gives the single
// rounding the format defines.
__global__ void __launch_bounds__(256) decode_kernel(const uint8_t* __restrict__ codes,
                                                     const uint16_t* __restrict__ scales,
                                                     const uint16_t* __restrict__ codebook, int n, int k,
                                                     uint16_t* __restrict__ w) {
  const long long groups = (long long)n * (k / 4);
  const int gpr = k / 4;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < groups;
       i += (long long)gridDim.x * blockDim.x) {
    const int row = (int)(i / gpr), g = (int)(i % gpr);
    const uint32_t c = codes[i];
    const uint32_t s = (g % 64 == 0) ? 0u : (codes[i - 1] & 7u);
    const uint32_t sc = scales[(size_t)row * (k / 256) + g / 64];
    const uint32_t sc2 = sc | (sc << 16);
    const uint2 e = *reinterpret_cast<const uint2*>(codebook + ((s << 8) | c) * 4);
    uint2 out;
    out.x = hmul2_u32(e.x, sc2);
    out.y = hmul2_u32(e.y, sc2);
    *reinterpret_cast<uint2*>(w + (size_t)row * k + 4 * (size_t)g) = out;
  }
}

}  // namespace tq
