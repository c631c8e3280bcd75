// tq_stack1.cuh -- the whole batch-1 layer stack in one persistent kernel.
//
// At batch 1 each phase of a layer (RHT -> decode-GEMV -> handoff) reads a
// few MB of codes, a few microseconds of work, so separate launches would
// spend as long in launch, codebook set-up and tail as in the work itself
// ("8 open models" article, "Speed": batch-1 generation is one read of the
// weights per token).  Here one cooperative launch (one CTA per SM) runs
// every phase of every layer:
//   * the codebook views are built once; the RHT sign bits and the unit
//     split of every phase are computed once into tables;
//   * between phases a grid barrier (atomic arrive + bounded acquire poll)
//     orders the outputs of phase f before the RHT of phase f+1; each warp
//     loads the first code chunk of phase f+1 before waiting at the barrier;
//   * units are split over warps exactly as in the single-phase kernel, but
//     the reduction has two levels and no global round trip inside a phase:
//     warps that share a tile leave their partial sums in shared memory and
//     the CTA sums them; a tile that straddles CTAs leaves one partial per
//     CTA in global memory, and the next phase sums those (in CTA order)
//     while it loads its input, after the barrier.  Grouping the sums by CTA
//     gives the same bits as the single-phase kernel's last-arriver sum.
// Every wait is bounded: on timeout the kernel records TQ_ERR_TIMEOUT in the
// status word and all CTAs leave.
#pragma once

#include "tq_dmma.cuh"

namespace tq {

constexpr int STACK_MAX_LAYERS = 128;
constexpr int STACK_TIMEOUT_STATUS = 7;  // TQ_ERR_TIMEOUT

// Copies of each CTA partial of a straddling tile: every CTA reads all of
// them after a barrier, and spreading the readers over copies keeps them off
// the same L2 lines.
constexpr int STACK_PART_COPIES = 8;

constexpr int PARAM_QUADS = (int)((sizeof(DmmaParams) + 15) / 16);  // 16-byte words of one DmmaParams

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
  float* y[4];            // outputs of each phase type (k, v and up land here too)
  uint32_t* signs;        // sign bits, bit set = the diagonal entry is -1
  uint32_t sign_words;
  uint64_t seed;
  float* partials;        // per-CTA partials of straddling tiles: [3][STACK_PART_COPIES][grid][2][16]
  int32_t* counters;
  int32_t m;              // tokens (1 for stack1_kernel)
  uint16_t* xq;           // small batch: x' fp16 [m][k] in fragment order, written each phase
  uint32_t* sync;         // barrier counter, zero at launch
  uint4* phase_table;     // [4 * n_layers][PARAM_QUADS]: every phase's parameters
  int32_t* status;
  uint32_t spin_limit;
  int32_t skip_arrive_cta;  // test hook: this CTA does not arrive at the launch's first barrier (-1: none)
};

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
  return v;
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
  p.m = sp.m;
  p.x_f32 = nullptr;
  p.x_f16 = sp.xq;
  p.x_bf16 = ph == 0 ? (l == 0 ? sp.h_in : sp.buf[3]) : sp.buf[ph - 1];
  p.rht_seed = 0;
  p.y = sp.y[ph];
  p.handoff = (ph == 3 && l == sp.n_layers - 1) ? sp.h_out : sp.buf[ph];
  p.handoff_rows = L.n[first];
  p.alpha = L.alpha[ph];
  p.partials = sp.partials;
  p.counters = sp.counters;
  p.tiles = (p.n_total + 15) / 16;
  p.blocks = p.k / 256;
  p.units = (int64_t)p.tiles * p.blocks;
  p.active_warps = (int32_t)(p.units < grid_warps ? p.units : grid_warps);
  p.rcp_active = ~0ULL / (uint64_t)p.active_warps;
  p.rcp_units = ~0ULL / (uint64_t)p.units;
}

// Arrive at the grid barrier (after the whole CTA finished its writes).
// With arrive = false the CTA only synchronises itself (the test hook that
// makes every bounded wait of the barrier run out).
__device__ __forceinline__ void grid_arrive(const StackParams& sp, bool arrive = true) {
  __syncthreads();
  if (threadIdx.x == 0 && arrive) {
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

// floor(n / d) for n < 2^53 and 0 < d < 2^32, given r = floor((2^64 - 1) / d):
// the multiply-high is floor(n / d) or one less (the error of r is below
// n / 2^64 < 1), and one step corrects it.
__device__ __forceinline__ uint64_t div_rcp(uint64_t n, uint64_t d, uint64_t r) {
  uint64_t q = __umul64hi(n, r);
  if ((q + 1) * d <= n) ++q;
  return q;
}

// The unit split of dmma_warp_begin / dmma_warp_of, per warp and per CTA
// (CTA c holds warps DMMA_WARPS*c .. DMMA_WARPS*c + DMMA_WARPS-1).
__device__ __forceinline__ int64_t sk_warp_begin(const DmmaParams& p, int64_t w) {
  return (int64_t)div_rcp((uint64_t)w * (uint64_t)p.units, (uint64_t)p.active_warps, p.rcp_active);
}
__device__ __forceinline__ int64_t sk_cta_begin(const DmmaParams& p, int c) {
  return sk_warp_begin(p, min((int64_t)c * DMMA_WARPS, (int64_t)p.active_warps));
}
__device__ __forceinline__ int sk_cta_of(const DmmaParams& p, int64_t u) {
  const uint64_t w = div_rcp((uint64_t)(u + 1) * (uint64_t)p.active_warps + (uint64_t)p.units - 1,
                             (uint64_t)p.units, p.rcp_units) - 1;
  return (int)(w / DMMA_WARPS);
}

// y and handoff of one output row.
__device__ __forceinline__ void stack_store_row(const DmmaParams& p, int R, float v) {
  if (R < p.n_total) {
    if (p.y) p.y[R] = v;
    if (R < p.handoff_rows) p.handoff[R] = f_to_bf16_bits(p.alpha * v);
  }
}

// After the unit loop and a __syncthreads: the tiles this CTA touched that no
// single warp finished.  Warp w's partial of tile t sits in its slot 0 when t
// is the first tile of its range, else in slot 1.  A tile inside the CTA is
// summed here in warp order and written; a tile that straddles CTAs leaves
// the CTA's sum in gp[copy][cta][s] (s = 0 for the CTA's first tile, 1 for
// its last; every copy) for the next phase.  `wbeg` = first unit of each warp of the CTA
// (17 entries), `wfirst` = first tile of each warp.
__device__ __forceinline__ void stack_cta_reduce(const DmmaParams& p, const int32_t* wbeg, const int32_t* wfirst,
                                                 const float* wslots, float* gp, int warp, int lane) {
  const int32_t b0 = wbeg[0], b1 = wbeg[DMMA_WARPS];
  if (b0 >= b1) return;
  const int32_t B = p.blocks;
  const int T0 = wfirst[0], T1 = (b1 - 1) / B;
  const int lw = lane & (DMMA_WARPS - 1);
  const int32_t lb = wbeg[lw], le = wbeg[lw + 1], lf = wfirst[lw];
  for (int t = T0 + warp; t <= T1; t += DMMA_WARPS) {
    const int32_t t0 = t * B, t1 = t0 + B;
    // warps of this CTA whose (non-empty) ranges meet the tile
    const uint32_t meet = __ballot_sync(0xffffffffu, lane < DMMA_WARPS && lb < le && lb < t1 && le > t0);
    const int wa = __ffs(meet) - 1, wz = 31 - __clz(meet);
    const bool one = wa == wz && __shfl_sync(0xffffffffu, lb, wa) <= t0 && __shfl_sync(0xffffffffu, le, wa) >= t1;
    if (one) continue;  // finished by that warp
    // this lane's contributor slot: every contributor's value is loaded, then summed in warp order
    const int ls = (lf == t) ? 0 : 1;
    float v = 0.f;
    if (lane < 16) {
      float part[DMMA_WARPS];
#pragma unroll
      for (int w = 0; w < DMMA_WARPS; ++w) {
        const int sw = __shfl_sync(0x0000ffffu, ls, w);
        part[w] = (w >= wa && w <= wz) ? wslots[(w * 2 + sw) * 16 + lane] : 0.f;
      }
#pragma unroll
      for (int w = 0; w < DMMA_WARPS; ++w)
        if (w >= wa && w <= wz) v += part[w];
      if (t0 >= b0 && t1 <= b1) {
        // the association of the single-phase kernel: (0 + group sum) + 0
        stack_store_row(p, t * 16 + lane, (0.f + v) + 0.f);
      } else {
        const size_t o = ((size_t)blockIdx.x * 2 + (t == T0 ? 0 : 1)) * 16 + lane;
#pragma unroll
        for (int r = 0; r < STACK_PART_COPIES; ++r) __stcg(gp + (size_t)r * gridDim.x * 32 + o, v);
      }
    }
  }
}

// Tile T of phase q (units T*B .. T*B+B-1) straddles CTAs when its first and
// last units belong to different CTAs ca < cz; s0 is the slot of ca's partial
// (0 when T is the first tile of ca's range).
__device__ __forceinline__ bool sk_straddle(const DmmaParams& q, int T, int& ca, int& cz, int& s0) {
  const int64_t t0 = (int64_t)T * q.blocks, t1 = t0 + q.blocks;
  ca = sk_cta_of(q, t0);
  cz = sk_cta_of(q, t1 - 1);
  if (ca == cz) return false;
  s0 = sk_cta_begin(q, ca) >= t0 ? 0 : 1;
  return true;
}

// Rows i0 .. i0+n-1 (n = 16 or 8) of a straddling tile: the sum of its CTA
// partials (gq = this CTA's copy) in CTA order, with the association of the
// single-phase kernel's last-arriver sum ((0 + group sums) + 0).  Two
// contributors' loads are in flight together.
template <int N>
__device__ __forceinline__ void sk_sum_rows(const float* gq, int ca, int cz, int s0, int i0, float (&v)[N]) {
  static_assert(N % 4 == 0, "rows in float4s");
  float4 a[2][N / 4];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float4* src = reinterpret_cast<const float4*>(gq + ((size_t)(ca + i) * 2 + (i ? 0 : s0)) * 16 + i0);
#pragma unroll
    for (int u = 0; u < N / 4; ++u) a[i][u] = (ca + i <= cz) ? __ldcg(src + u) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int e = 0; e < N; ++e) v[e] = 0.f;
#pragma unroll
  for (int i = 0; i < 2; ++i)
    if (ca + i <= cz) {
      const float* aa = reinterpret_cast<const float*>(&a[i][0]);
#pragma unroll
      for (int e = 0; e < N; ++e) v[e] += aa[e];
    }
  for (int cc = ca + 2; cc <= cz; ++cc) {  // a tile over more than two CTAs
    const float4* src = reinterpret_cast<const float4*>(gq + (size_t)cc * 2 * 16 + i0);
#pragma unroll
    for (int u = 0; u < N / 4; ++u) {
      const float4 w = __ldcg(src + u);
      v[4 * u] += w.x;
      v[4 * u + 1] += w.y;
      v[4 * u + 2] += w.z;
      v[4 * u + 3] += w.w;
    }
  }
#pragma unroll
  for (int e = 0; e < N; ++e) v[e] = v[e] + 0.f;
}

// The outputs (y, handoff) of the straddling tile of phase q that starts in
// this CTA's range, if any; lanes 0-3, four rows each.  Every such tile
// starts in exactly one CTA, so each is written once.
__device__ __forceinline__ void stack_own_straddle(const DmmaParams& q, const float* gq, int tid) {
  if (tid >= 4) return;
  const int64_t B = q.blocks;
  const int64_t b0 = sk_cta_begin(q, blockIdx.x), b1 = sk_cta_begin(q, blockIdx.x + 1);
  if (b0 >= b1) return;
  const int T = (int)((b1 - 1) / B);
  const int64_t t0 = (int64_t)T * B, t1 = t0 + B;
  if (t0 < b0 || t1 <= b1) return;  // starts in an earlier CTA, or ends inside this one
  const int cz = sk_cta_of(q, t1 - 1);
  float v[4];
  sk_sum_rows<4>(gq, blockIdx.x, cz, (b0 / B == T) ? 0 : 1, tid * 4, v);
  for (int e = 0; e < 4; ++e) stack_store_row(q, T * 16 + tid * 4 + e, v[e]);
}

// RHT of one 512-block with the diagonal taken from the sign table, in two
// steps so that a warp issues the loads of all its blocks before the first
// transform.  The input and the table were written by other CTAs of this
// launch, so they are read through L2 (ld.global.cg), never from a possibly
// stale L1 line.
struct RhtIn {
  uint4 p0, p1;
  uint32_t bits;
};

__device__ __forceinline__ RhtIn rht_table_load(const uint16_t* x, int blk, const uint32_t* signs) {
  const int lane = threadIdx.x & 31;
  const int base = blk * 512 + lane * 16;
  const uint4* src = reinterpret_cast<const uint4*>(x + base);
  RhtIn r;
  r.p0 = __ldcg(src);
  r.p1 = __ldcg(src + 1);
  r.bits = __ldcg(signs + (base >> 5)) >> (base & 16);
  return r;
}

// Transform block blk and store it as hi/lo quads, then mark the block ready
// for this CTA's unit loops (xflag[blk] = tag).  With q, a lane whose 16
// inputs (tile 32 blk + lane of phase q) straddle CTAs sums them from the CTA
// partials gq and rounds them as the handoff is, instead of the handoff value
// in global memory (written by its own CTA only after this phase's barrier).
__device__ __forceinline__ void rht_block(RhtIn r, int blk, const DmmaParams* q, const float* gq, uint8_t* xs,
                                          volatile int* xflag, int tag) {
  const int lane = threadIdx.x & 31;
  int ca, cz, s0;
  if (q && sk_straddle(*q, blk * 32 + lane, ca, cz, s0)) {
    float v[16];
    sk_sum_rows<16>(gq, ca, cz, s0, 0, v);
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      w[i] = f_to_bf16_bits(q->alpha * v[2 * i]) | (f_to_bf16_bits(q->alpha * v[2 * i + 1]) << 16);
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
  for (int i = 0; i < 16; ++i) v[i] *= inv;
#pragma unroll
  for (int r4 = 0; r4 < 4; ++r4)
    store_hilo(xs, blk * 128 + lane * 4 + r4, v[4 * r4], v[4 * r4 + 1], v[4 * r4 + 2], v[4 * r4 + 3]);
  __syncwarp();
  __threadfence_block();
  if (lane == 0) xflag[blk] = tag;
}

// This warp's share of the phase's activations x' = RHT(x): blocks warp,
// warp + 16, ... one after the other (holding several blocks' loads at once
// costs register spills in the unit loops).  No CTA-wide synchronisation:
// each block is flagged when it is stored.
__device__ __forceinline__ void stack_rht(const DmmaParams& p, const DmmaParams* q, const float* gq,
                                          const uint32_t* signs, uint8_t* xs, volatile int* xflag, int tag,
                                          int warp) {
  const int nb = p.k / 512;
  for (int blk = warp; blk < nb; blk += DMMA_WARPS)
    rht_block(rht_table_load(p.x_bf16, blk, signs), blk, q, gq, xs, xflag, tag);
}

// First unit and first tile of each warp of this CTA in phase p.
__device__ __forceinline__ void stack_warp_tables(const DmmaParams& p, int32_t* wbeg, int32_t* wfirst, int tid) {
  if (tid <= DMMA_WARPS) {
    const int64_t w = min((int64_t)blockIdx.x * DMMA_WARPS + tid, (int64_t)p.active_warps);
    const int32_t b = (int32_t)sk_warp_begin(p, w);
    wbeg[tid] = b;
    wfirst[tid] = b / p.blocks;
  }
}

// dmma_begin with the unit range of this warp taken from the tables.
__device__ __forceinline__ void stack_begin(const DmmaParams& p, const int32_t* wbeg, const int32_t* wfirst, int warp,
                                            int lane, DmmaCursor& c) {
  c.wb = wbeg[warp];
  c.we = wbeg[warp + 1];
  c.t = c.b = 0;
  if (c.wb < c.we) {
    c.t = wfirst[warp];
    c.b = (int)(c.wb - (int64_t)c.t * p.blocks);
    c.rows = dmma_rows(p, c.t, lane >> 2, lane & 3);
    c.cur = dmma_fetch(c.rows, c.b, c.spa, c.spb, true);
  }
}

template <int LV>
__global__ void __launch_bounds__(DMMA_THREADS, 1) stack1_kernel(const __grid_constant__ StackParams sp) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* xs = smem + (16384 << LV);
  int kmax = 0;
  for (int l = 0; l < sp.n_layers; ++l)
    for (int ph = 0; ph < 4; ++ph) kmax = max(kmax, sp.layers[l].k[ph]);
  // four parameter slots: previous, running, next and next-but-one phase
  uint4* slots = reinterpret_cast<uint4*>(xs + (size_t)kmax * 4);
  float* wslots = reinterpret_cast<float*>(slots + 4 * PARAM_QUADS);       // [warp][2][16]
  int32_t* wbegt = reinterpret_cast<int32_t*>(wslots + DMMA_WARPS * 32);    // [2][DMMA_WARPS + 1]
  int32_t* wfirstt = wbegt + 2 * (DMMA_WARPS + 1);                          // [2][DMMA_WARPS + 1]
  volatile int* xflag = reinterpret_cast<volatile int*>(wfirstt + 2 * (DMMA_WARPS + 1));  // [kmax / 512]
  volatile int* abort_flag = xflag + kmax / 512;
  int* duty = const_cast<int*>(abort_flag + 1);  // last phase whose straddle duty was taken
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grid_warps = gridDim.x * DMMA_WARPS;
  const int64_t W = (int64_t)blockIdx.x * DMMA_WARPS + warp;
  const int nphases = 4 * sp.n_layers;
  const size_t gstride = (size_t)STACK_PART_COPIES * gridDim.x * 32;  // floats of one phase's CTA partials
  const size_t gcopy = (size_t)(blockIdx.x % STACK_PART_COPIES) * gridDim.x * 32;  // this CTA's copy
  auto slot = [&](int f) -> DmmaParams& { return *reinterpret_cast<DmmaParams*>(slots + (f & 3) * PARAM_QUADS); };
  auto wbeg = [&](int f) { return wbegt + (f & 1) * (DMMA_WARPS + 1); };
  auto wfirst = [&](int f) { return wfirstt + (f & 1) * (DMMA_WARPS + 1); };
  auto parts = [&](int f) { return sp.partials + (size_t)(f % 3) * gstride; };

  if (tid == 0) {
    *abort_flag = 0;
    *duty = 0;
    stack_phase_params(sp, 0, slot(0), grid_warps);
  }
  if (tid == 32 && nphases > 1) stack_phase_params(sp, 1, slot(1), grid_warps);
  for (int i = tid; i < kmax / 512; i += DMMA_THREADS) xflag[i] = -1;
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

  // first phase's tables and code chunk, then the barrier
  stack_warp_tables(slot(0), wbeg(0), wfirst(0), tid);
  __syncthreads();
  DmmaCursor c;
  stack_begin(slot(0), wbeg(0), wfirst(0), warp, lane, c);
  if (!grid_wait(sp, epoch * gridDim.x, abort_flag)) return;

  for (int f = 0; f < nphases; ++f) {
    const int l = f >> 2, ph = f & 3;
    const DmmaParams& p = slot(f);
    // parameters of phase f+2 come from the table while the RHT runs
    uint4 nq = make_uint4(0u, 0u, 0u, 0u);
    const bool fetch = tid < PARAM_QUADS && f + 2 < nphases;
    if (fetch) nq = __ldcg(sp.phase_table + (size_t)(f + 2) * PARAM_QUADS + tid);
    // this warp's blocks of x' (each flagged when stored), then its units,
    // which wait only for the blocks they read
    stack_rht(p, f > 0 ? &slot(f - 1) : nullptr, parts(f + 2) + gcopy, sp.signs + sp.layers[l].sign_off[ph], xs,
              xflag, f, warp);
    if (fetch) slots[((f + 2) & 3) * PARAM_QUADS + tid] = nq;  // slot of phase f-2: no reader left
    if (f + 1 < nphases) stack_warp_tables(slot(f + 1), wbeg(f + 1), wfirst(f + 1), tid);  // read after the barrier
    dmma_units<LV, 1, true, false, true>(p, smem, xs, W, c, lane, wslots + warp * 32, xflag, f, sp.status,
                                           sp.spin_limit);
    // the first warp done writes the outputs of the previous phase's
    // straddling tile that starts in this CTA (its partials stay until phase
    // f+2 overwrites them), off the critical path of the slowest warp
    if (f > 0) {
      int won = 0;
      if (lane == 0) won = atomicCAS(duty, f - 1, f) == f - 1;
      if (__shfl_sync(0xffffffffu, won, 0)) stack_own_straddle(slot(f - 1), parts(f - 1) + gcopy, lane);
    }
    __syncthreads();
    stack_cta_reduce(p, wbeg(f), wfirst(f), wslots, parts(f), warp, lane);
    grid_arrive(sp);  // its __syncthreads ends every use of the warp tables, slots and x'
    ++epoch;
    if (f + 1 == nphases) break;
    // next phase: first code chunk before the barrier wait
    stack_begin(slot(f + 1), wbeg(f + 1), wfirst(f + 1), warp, lane, c);
    if (!grid_wait(sp, epoch * gridDim.x, abort_flag)) return;
  }
  // the last phase's straddling tiles: summed once every CTA partial is in
  if (!grid_wait(sp, epoch * gridDim.x, abort_flag)) return;
  stack_own_straddle(slot(nphases - 1), parts(nphases - 1) + gcopy, tid);
}

}  // namespace tq
