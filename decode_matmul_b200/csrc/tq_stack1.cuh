// tq_stack1.cuh -- the whole batch-1 layer stack in one persistent kernel.
//
// At batch 1 each phase of a layer (RHT -> decode-GEMV -> handoff) reads a
// few MB of codes, a few microseconds of work, so separate launches would
// spend as long in launch, codebook set-up and tail as in the work itself
// ("8 open models" article, "Speed": batch-1 generation is one read of the
// weights per token).  Here one cooperative launch (one CTA per SM) runs
// every phase of every layer:
//   * the codebook views are built once; the RHT sign bits of every phase
//     are drawn once into a table;
//   * between phases a grid barrier (atomic arrive + bounded acquire poll)
//     orders the handoff of phase f before the RHT of phase f+1; each warp
//     loads the first code chunk of phase f+1 before waiting at the barrier;
//   * each phase is the same warp-level unit split and deterministic
//     last-arriver reduction as the single-phase kernel.
// Every wait is bounded: on timeout the kernel records TQ_ERR_TIMEOUT in the
// status word and all CTAs leave.
#pragma once

#include "tq_dmma.cuh"

namespace tq {

constexpr int STACK_MAX_LAYERS = 128;
constexpr int STACK_TIMEOUT_STATUS = 7;  // TQ_ERR_TIMEOUT

struct StackLayerDev {
  const uint8_t* codes[7];  // q k v o gate up down
  const uint16_t* scales[7];
  int32_t n[7];
  int32_t k[4];           // input width of each phase
  uint32_t sign_off[4];   // first word of each phase's RHT sign bits
  float alpha[4];         // handoff gain of each phase
};

struct StackParams {
  StackLayerDev layers[STACK_MAX_LAYERS];
  int32_t n_layers;
  int32_t lv;
  const uint16_t* codebook;
  const uint16_t* h_in;
  uint16_t* h_out;
  uint16_t* buf[4];       // phase handoffs: q, o, gate, layer output
  float* y;               // every phase's outputs (k, v and up land here)
  uint32_t* signs;        // sign bits, bit set = the diagonal entry is -1
  uint32_t sign_words;
  uint64_t seed;
  float* partials;
  int32_t* counters;
  uint32_t* sync;         // barrier counter, zero at launch
  int32_t* status;
  uint32_t spin_limit;
};

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// RHT of one 512-block with the diagonal taken from the sign table.  The
// input and the table were written by other CTAs of this launch, so they are
// read through L2 (ld.global.cg), never from a possibly stale L1 line.
__device__ __forceinline__ void rht512_warp_table(const uint16_t* x, int blk, const uint32_t* signs, float v[16]) {
  const int lane = threadIdx.x & 31;
  const int base = blk * 512 + lane * 16;
  const uint4* src = reinterpret_cast<const uint4*>(x + base);
  const uint4 p0 = __ldcg(src), p1 = __ldcg(src + 1);
  const uint32_t bits = __ldcg(signs + (base >> 5)) >> (base & 16);
  const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t lo = (w[i] & 0xFFFFu) ^ (((bits >> (2 * i)) & 1u) << 15);
    const uint32_t hi = (w[i] >> 16) ^ (((bits >> (2 * i + 1)) & 1u) << 15);
    v[2 * i] = bf16_bits_to_f(lo);
    v[2 * i + 1] = bf16_bits_to_f(hi);
  }
  wht512_warp(v);
  const float inv = 0.044194173824159216f;  // 1/sqrt(512)
#pragma unroll
  for (int r = 0; r < 16; ++r) v[r] *= inv;
}

// Phase f = 4l + p as single-phase parameters.
__device__ __forceinline__ void stack_phase_params(const StackParams& sp, int f, DmmaParams& p, int grid_warps) {
  const int l = f >> 2, ph = f & 3;
  const StackLayerDev& L = sp.layers[l];
  const int first = ph == 0 ? 0 : (ph == 1 ? 3 : (ph == 2 ? 4 : 6));
  const int nops = ph == 0 ? 3 : (ph == 2 ? 2 : 1);
  int32_t row0 = 0;
  for (int i = 0; i < 3; ++i) {
    const int op = first + (i < nops ? i : 0);
    p.seg[i].codes = L.codes[op];
    p.seg[i].scales = L.scales[op];
    p.seg[i].rows = i < nops ? L.n[op] : 0;
    p.seg[i].row0 = row0;
    if (i < nops) row0 += L.n[op];
  }
  p.nseg = nops;
  p.codebook = sp.codebook;
  p.n_total = row0;
  p.k = L.k[ph];
  p.m = 1;
  p.x_f32 = nullptr;
  p.x_f16 = nullptr;
  p.x_bf16 = ph == 0 ? (l == 0 ? sp.h_in : sp.buf[3]) : sp.buf[ph - 1];
  p.rht_seed = 0;
  p.y = sp.y;
  p.handoff = (ph == 3 && l == sp.n_layers - 1) ? sp.h_out : sp.buf[ph];
  p.handoff_rows = L.n[first];
  p.alpha = L.alpha[ph];
  p.partials = sp.partials;
  p.counters = sp.counters;
  p.tiles = (p.n_total + 15) / 16;
  p.blocks = p.k / 256;
  p.units = (int64_t)p.tiles * p.blocks;
  p.active_warps = (int32_t)(p.units < grid_warps ? p.units : grid_warps);
}

// Arrive at the grid barrier (after the whole CTA finished its writes).
__device__ __forceinline__ void grid_arrive(const StackParams& sp) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(sp.sync, 1u);
  }
}

// Wait until `target` arrivals; false (and the status word set) on timeout.
__device__ __forceinline__ bool grid_wait(const StackParams& sp, uint32_t target, volatile int* abort_flag) {
  if (threadIdx.x == 0) {
    uint32_t spins = 0;
    while (ld_acquire_gpu(sp.sync) < target) {
      if (++spins > sp.spin_limit) {
        *abort_flag = 1;
        atomicExch(sp.status, STACK_TIMEOUT_STATUS);
        break;
      }
      __nanosleep(64);
    }
  }
  __syncthreads();
  return *abort_flag == 0;
}

template <int LV>
__global__ void __launch_bounds__(DMMA_THREADS, 1) stack1_kernel(const __grid_constant__ StackParams sp) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* xs = smem + (16384 << LV);
  int kmax = 0;
  for (int l = 0; l < sp.n_layers; ++l)
    for (int ph = 0; ph < 4; ++ph) kmax = max(kmax, sp.layers[l].k[ph]);
  DmmaParams* pp = reinterpret_cast<DmmaParams*>(xs + (size_t)kmax * 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(pp + 1);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grid_warps = gridDim.x * DMMA_WARPS;
  const int64_t W = (int64_t)blockIdx.x * DMMA_WARPS + warp;
  const int nphases = 4 * sp.n_layers;

  if (tid == 0) *abort_flag = 0;
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
  grid_arrive(sp);
  uint32_t epoch = 1;

  // first phase's parameters and code chunk, then the barrier
  if (tid == 0) stack_phase_params(sp, 0, *pp, grid_warps);
  __syncthreads();
  DmmaCursor c;
  dmma_begin(*pp, W, lane >> 2, lane & 3, c);
  if (!grid_wait(sp, epoch * gridDim.x, abort_flag)) return;

  for (int f = 0; f < nphases; ++f) {
    const int l = f >> 2, ph = f & 3;
    // batch-1 activations of this phase: RHT with the table, hi/lo split
    const uint32_t* sg = sp.signs + sp.layers[l].sign_off[ph];
    for (int blk = warp; blk < pp->k / 512; blk += DMMA_WARPS) {
      float v[16];
      rht512_warp_table(pp->x_bf16, blk, sg, v);
#pragma unroll
      for (int r4 = 0; r4 < 4; ++r4)
        store_hilo(xs, blk * 128 + lane * 4 + r4, v[4 * r4], v[4 * r4 + 1], v[4 * r4 + 2], v[4 * r4 + 3]);
    }
    __syncthreads();
    dmma_units<LV, 1, true>(*pp, smem, xs, W, c, lane);
    grid_arrive(sp);
    ++epoch;
    if (f + 1 == nphases) break;
    // next phase: parameters and first code chunk before the barrier wait
    if (tid == 0) stack_phase_params(sp, f + 1, *pp, grid_warps);
    __syncthreads();
    dmma_begin(*pp, W, lane >> 2, lane & 3, c);
    if (!grid_wait(sp, epoch * gridDim.x, abort_flag)) return;
  }
}

}  // namespace tq
