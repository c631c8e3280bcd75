// tq_stackn.cuh -- the layer stack for small batches (2-16 tokens) in one
// persistent kernel.
//
// The batch-1 design (tq_stack1.cuh) with three changes for m tokens:
//   * the transform of each phase's input is split over the whole grid: one
//     warp per (token, 512-block) task writes x' (fp16, fragment order) to a
//     global buffer, and a second grid barrier per phase orders those writes
//     before the unit loops read them (through L2);
//   * unit loops run the m16n8k16 register-decode with NT 8-token column
//     tiles ("8 open models" article, "Speed": one read of the weights is
//     shared by all tokens of the batch);
//   * warp and CTA partial sums hold 16 rows x 8 NT tokens; a CTA partial of a
//     tile that straddles CTAs is stored token-major, so the task that needs
//     one token's 16 rows reads them contiguously.
// The unit split and the order of every sum are those of the single-phase
// kernel, so both give identical bits.
#pragma once

#include "tq_stack1.cuh"

namespace tq {

// The CTA's shared tiles after its unit loops (and a __syncthreads): tiles
// inside the CTA are summed in warp order and written (y, handoff); a tile
// that straddles CTAs leaves the CTA's sum, token-major, in gp[cta][s][MC][16]
// (s = 0 for the CTA's first tile, 1 for its last).  One warp per tile.
template <int NT>
__device__ __forceinline__ void stackn_cta_reduce(const DmmaParams& p, const int32_t* wbeg, const int32_t* wfirst,
                                                  const float* wslots, float* gp, int warp, int lane) {
  constexpr int MC = NT * 8, SLOT = 16 * MC;
  const int32_t b0 = wbeg[0], b1 = wbeg[DMMA_WARPS];
  if (b0 >= b1) return;
  const int32_t B = p.blocks;
  const int T0 = wfirst[0], T1 = (b1 - 1) / B;
  const int lw = lane & (DMMA_WARPS - 1);
  const int32_t lb = wbeg[lw], le = wbeg[lw + 1], lf = wfirst[lw];
  for (int t = T0 + warp; t <= T1; t += DMMA_WARPS) {
    const int32_t t0 = t * B, t1 = t0 + B;
    const uint32_t meet = __ballot_sync(0xffffffffu, lane < DMMA_WARPS && lb < le && lb < t1 && le > t0);
    const int wa = __ffs(meet) - 1, wz = 31 - __clz(meet);
    const bool one = wa == wz && __shfl_sync(0xffffffffu, lb, wa) <= t0 && __shfl_sync(0xffffffffu, le, wa) >= t1;
    if (one) continue;  // finished by that warp
    const int ls = (lf == t) ? 0 : 1;  // lane w: warp w's slot of tile t
    int sw[DMMA_WARPS];
#pragma unroll
    for (int w = 0; w < DMMA_WARPS; ++w) sw[w] = __shfl_sync(0xffffffffu, ls, w);
    const bool inside = t0 >= b0 && t1 <= b1;
    for (int e = lane; e < SLOT; e += 32) {
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < DMMA_WARPS; ++w)
        if (w >= wa && w <= wz) v += wslots[(w * 2 + sw[w]) * SLOT + e];
      const int row = e / MC, tok = e - row * MC;
      if (inside) {
        const int R = t * 16 + row;
        const float fin = 0.f + v;  // the single-phase kernel's association: 0 + group sum
        if (tok < p.m && R < p.n_total) {
          if (p.y) p.y[(size_t)tok * p.n_total + R] = fin;
          if (R < p.handoff_rows) p.handoff[(size_t)tok * p.handoff_rows + R] = f_to_bf16_bits(p.alpha * fin);
        }
      } else {
        __stcg(gp + (((size_t)blockIdx.x * 2 + (t == T0 ? 0 : 1)) * MC + tok) * 16 + row, v);
      }
    }
  }
}

// Four rows (i0 .. i0+3) of token tok of a straddling tile of phase q: the
// sum of its CTA partials (token-major, gq) in CTA order.
template <int NT>
__device__ __forceinline__ float4 skn_sum4(const float* gq, int ca, int cz, int s0, int tok, int i0) {
  constexpr int MC = NT * 8;
  float4 a[2];
#pragma unroll
  for (int i = 0; i < 2; ++i)
    a[i] = (ca + i <= cz)
               ? __ldcg(reinterpret_cast<const float4*>(gq + (((size_t)(ca + i) * 2 + (i ? 0 : s0)) * MC + tok) * 16 + i0))
               : make_float4(0.f, 0.f, 0.f, 0.f);
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 2; ++i)
    if (ca + i <= cz) {
      v.x += a[i].x;
      v.y += a[i].y;
      v.z += a[i].z;
      v.w += a[i].w;
    }
  for (int cc = ca + 2; cc <= cz; ++cc) {  // a tile over more than two CTAs
    const float4 w = __ldcg(reinterpret_cast<const float4*>(gq + (((size_t)cc * 2) * MC + tok) * 16 + i0));
    v.x += w.x;
    v.y += w.y;
    v.z += w.z;
    v.w += w.w;
  }
  return v;
}

// The phase's x' = RHT(x) for all m tokens, split over the grid: warp gw
// takes the (token, 512-block) tasks gw, gw + nw, ...  A lane whose 16 inputs
// (tile 32 B + lane of phase q) straddle CTAs sums them from the CTA partials
// gq and rounds them as the handoff is.  x' goes to xq in fragment order.
template <int NT>
__device__ __forceinline__ void stackn_rht(const DmmaParams& p, const DmmaParams* q, const float* gq,
                                           const uint32_t* signs, uint16_t* xq, int64_t gw, int64_t nw, int lane) {
  const int nb = p.k / 512;
  const int64_t ntask = (int64_t)p.m * nb;
  for (int64_t task = gw; task < ntask; task += nw) {
    const int t = (int)(task / nb), blk = (int)(task - (int64_t)t * nb);
    RhtIn r = rht_table_load(p.x_bf16 + (size_t)t * p.k, blk, signs);
    int ca, cz, s0;
    if (q && sk_straddle(*q, blk * 32 + lane, ca, cz, s0)) {
      uint32_t w[8];
#pragma unroll
      for (int i4 = 0; i4 < 4; ++i4) {
        const float4 v = skn_sum4<NT>(gq, ca, cz, s0, t, 4 * i4);
        w[2 * i4] = f_to_bf16_bits(q->alpha * v.x) | (f_to_bf16_bits(q->alpha * v.y) << 16);
        w[2 * i4 + 1] = f_to_bf16_bits(q->alpha * v.z) | (f_to_bf16_bits(q->alpha * v.w) << 16);
      }
      r.p0 = make_uint4(w[0], w[1], w[2], w[3]);
      r.p1 = make_uint4(w[4], w[5], w[6], w[7]);
    }
    const uint32_t w[8] = {r.p0.x, r.p0.y, r.p0.z, r.p0.w, r.p1.x, r.p1.y, r.p1.z, r.p1.w};
    float v[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = bf16_bits_to_f((w[i] & 0xFFFFu) ^ (((r.bits >> (2 * i)) & 1u) << 15));
      v[2 * i + 1] = bf16_bits_to_f((w[i] >> 16) ^ (((r.bits >> (2 * i + 1)) & 1u) << 15));
    }
    wht512_warp(v);
    const float inv = 0.044194173824159216f;  // 1/sqrt(512)
#pragma unroll
    for (int r4 = 0; r4 < 4; ++r4) {
      const int kk = blk * 512 + lane * 16 + 4 * r4;
      *reinterpret_cast<uint2*>(xq + xt_pos(t, kk, p.k)) =
          make_uint2(f2_to_h2(v[4 * r4] * inv, v[4 * r4 + 1] * inv), f2_to_h2(v[4 * r4 + 2] * inv, v[4 * r4 + 3] * inv));
    }
  }
}

// The outputs (y, handoff; every token) of the straddling tile of phase q that
// starts in this CTA's range, if any; one warp, lane = (token, 4-row group).
template <int NT>
__device__ __forceinline__ void stackn_own_straddle(const DmmaParams& q, const float* gq, int lane) {
  const int64_t B = q.blocks;
  const int64_t b0 = sk_cta_begin(q, blockIdx.x), b1 = sk_cta_begin(q, blockIdx.x + 1);
  if (b0 >= b1) return;
  const int T = (int)((b1 - 1) / B);
  const int64_t t0 = (int64_t)T * B, t1 = t0 + B;
  if (t0 < b0 || t1 <= b1) return;  // starts in an earlier CTA, or ends inside this one
  const int cz = sk_cta_of(q, t1 - 1);
  const int s0 = (b0 / B == T) ? 0 : 1;
  for (int idx = lane; idx < q.m * 4; idx += 32) {
    const int tok = idx >> 2, i0 = (idx & 3) * 4;
    const float4 v = skn_sum4<NT>(gq, blockIdx.x, cz, s0, tok, i0);
    const float vv[4] = {v.x, v.y, v.z, v.w};
    for (int e = 0; e < 4; ++e) {
      const int R = T * 16 + i0 + e;
      if (R < q.n_total) {
        if (q.y) q.y[(size_t)tok * q.n_total + R] = vv[e];
        if (R < q.handoff_rows) q.handoff[(size_t)tok * q.handoff_rows + R] = f_to_bf16_bits(q.alpha * vv[e]);
      }
    }
  }
}

template <int LV, int NT>
__global__ void __launch_bounds__(DMMA_THREADS, 1) stackn_kernel(const __grid_constant__ StackParams sp) {
  constexpr int MC = NT * 8, SLOT = 16 * MC;
  extern __shared__ __align__(128) uint8_t smem[];
  float* wslots = reinterpret_cast<float*>(smem + (16384 << LV));           // [warp][2][16 * MC]
  uint4* slots = reinterpret_cast<uint4*>(wslots + DMMA_WARPS * 2 * SLOT);  // 4 parameter slots
  int32_t* wbegt = reinterpret_cast<int32_t*>(slots + 4 * PARAM_QUADS);     // [2][DMMA_WARPS + 1]
  int32_t* wfirstt = wbegt + 2 * (DMMA_WARPS + 1);                          // [2][DMMA_WARPS + 1]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(wfirstt + 2 * (DMMA_WARPS + 1));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grid_warps = gridDim.x * DMMA_WARPS;
  const int64_t W = (int64_t)blockIdx.x * DMMA_WARPS + warp;
  const int nphases = 4 * sp.n_layers;
  const size_t gstride = (size_t)gridDim.x * 2 * SLOT;  // floats of one phase's CTA partials
  auto slot = [&](int f) -> DmmaParams& { return *reinterpret_cast<DmmaParams*>(slots + (f & 3) * PARAM_QUADS); };
  auto wbeg = [&](int f) { return wbegt + (f & 1) * (DMMA_WARPS + 1); };
  auto wfirst = [&](int f) { return wfirstt + (f & 1) * (DMMA_WARPS + 1); };
  auto parts = [&](int f) { return sp.partials + (size_t)(f % 3) * gstride; };

  if (tid == 0) {
    *abort_flag = 0;
    stack_phase_params(sp, 0, slot(0), grid_warps);
  }
  if (tid == 32 && nphases > 1) stack_phase_params(sp, 1, slot(1), grid_warps);
  // every phase's parameters, one thread each, into the table read later
  for (int f = blockIdx.x * DMMA_THREADS + tid; f < nphases; f += gridDim.x * DMMA_THREADS) {
    DmmaParams pf;
    stack_phase_params(sp, f, pf, grid_warps);
    const uint4* src = reinterpret_cast<const uint4*>(&pf);
    for (int i = 0; i < (int)(sizeof(DmmaParams) / 16); ++i) sp.phase_table[(size_t)f * PARAM_QUADS + i] = src[i];
    if (sizeof(DmmaParams) % 16) {
      uint4 tail = make_uint4(0u, 0u, 0u, 0u);
      memcpy(&tail, reinterpret_cast<const uint8_t*>(&pf) + (sizeof(DmmaParams) / 16) * 16, sizeof(DmmaParams) % 16);
      sp.phase_table[(size_t)f * PARAM_QUADS + sizeof(DmmaParams) / 16] = tail;
    }
  }
  build_views<LV>(smem, sp.codebook, tid, DMMA_THREADS);

  // RHT sign table: word j holds d[32j .. 32j+31] of the phase it belongs to.
  for (uint32_t j = blockIdx.x * DMMA_THREADS + tid; j < sp.sign_words; j += gridDim.x * DMMA_THREADS) {
    int l = 0;
    while (l + 1 < sp.n_layers && sp.layers[l + 1].sign_off[0] <= j) ++l;
    int ph = 0;
    while (ph < 3 && sp.layers[l].sign_off[ph + 1] <= j) ++ph;
    const uint64_t tag = 0x516E0000ULL | ((uint64_t)l << 2) | (uint64_t)ph;
    const uint64_t seed_lp = mix64(sp.seed ^ mix64(tag));
    const uint32_t k0 = (j - sp.layers[l].sign_off[ph]) * 32;
    uint32_t bits = 0;
    for (int i = 0; i < 32; ++i) bits |= (rht_sign_negative(seed_lp, k0 + i) ? 1u : 0u) << i;
    sp.signs[j] = bits;
  }
  grid_arrive(sp, (int)blockIdx.x != sp.skip_arrive_cta);  // its __syncthreads publishes slots 0 and 1
  uint32_t epoch = 1;
  stack_warp_tables(slot(0), wbeg(0), wfirst(0), tid);
  if (!grid_wait(sp, epoch * gridDim.x, abort_flag)) return;

  DmmaCursor c;
  for (int f = 0; f < nphases; ++f) {
    const int l = f >> 2, ph = f & 3;
    const DmmaParams& p = slot(f);
    // parameters of phase f+2 come from the table while the transform runs
    uint4 nq = make_uint4(0u, 0u, 0u, 0u);
    const bool fetch = tid < PARAM_QUADS && f + 2 < nphases;
    if (fetch) nq = __ldcg(sp.phase_table + (size_t)(f + 2) * PARAM_QUADS + tid);
    // x' of this phase, split over the grid
    stackn_rht<NT>(p, f > 0 ? &slot(f - 1) : nullptr, parts(f + 2), sp.signs + sp.layers[l].sign_off[ph], sp.xq, W,
                   grid_warps, lane);
    // the outputs of the previous phase's straddling tile that starts in this
    // CTA (its partials stay until phase f+2 overwrites them)
    if (f > 0 && warp == DMMA_WARPS - 1) stackn_own_straddle<NT>(slot(f - 1), parts(f - 1), lane);
    if (fetch) slots[((f + 2) & 3) * PARAM_QUADS + tid] = nq;  // slot of phase f-2: no reader left
    if (f + 1 < nphases) stack_warp_tables(slot(f + 1), wbeg(f + 1), wfirst(f + 1), tid);  // read after a barrier
    stack_begin(p, wbeg(f), wfirst(f), warp, lane, c);  // first code chunk before the wait
    grid_arrive(sp);  // x' of every token is in
    ++epoch;
    if (!grid_wait(sp, epoch * gridDim.x, abort_flag)) return;
    dmma_units<LV, NT, false, true, true>(p, smem, nullptr, W, c, lane, wslots + warp * 2 * SLOT);
    __syncthreads();
    stackn_cta_reduce<NT>(p, wbeg(f), wfirst(f), wslots, parts(f), warp, lane);
    grid_arrive(sp);  // its __syncthreads ends every use of the warp tables, slots and slots' partials
    ++epoch;
    if (!grid_wait(sp, epoch * gridDim.x, abort_flag)) return;
  }
  // the last phase's straddling tiles (every CTA partial is in)
  if (warp == 0) stackn_own_straddle<NT>(slot(nphases - 1), parts(nphases - 1), lane);
}

}  // namespace tq
