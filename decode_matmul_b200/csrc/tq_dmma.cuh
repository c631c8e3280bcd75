// tq_dmma.cuh -- decode-in-registers matmul for batch 1 and small batches.
//
// Computes y[t][n] = sum_k W[n][k] x'[t][k] where W is decoded on the fly
// from the trellis codes ("Pingala-8" landing page, "How it works"; "8 open
// models" article, "Speed": at batch 1 the work is one read of the packed
// weights per token).
//
// Design (B200, sm_100a):
//  * Work unit = 16 weight rows x one 256-weight block (64 code bytes per
//    row).  Units are ordered tile-major and split evenly over all active
//    warps of the grid (contiguous ranges), so every SM gets the same number
//    of code bytes whatever n and k are.  A tile whose units span several
//    warps is summed by the last warp to arrive, in warp order (deterministic),
//    through a small workspace of partial sums and per-tile counters.
//  * Lane (g = lane/4, q = lane%4) streams 16 code bytes of row g and 16 of
//    row g+8 (one 128-bit load each; 4 lanes cover a row's 64 codes), i.e. the
//    m16n8k16 A-fragment owner of those rows.  The K order inside the MMA is
//    permuted so that a lane's four A slots {2q,2q+1,2q+8,2q+9} hold the four
//    weights of ONE code; B (the activations) uses the same permutation.
//  * The state of code j is the low 3 bits of code j-1: the same 32-bit word
//    or the previous word for 15 of 16 codes, the previous lane's last byte
//    (one shuffle) for the first; lanes with q == 0 start a 256-block (state 0).
//  * The codebook (16 KB) is replicated V times in shared memory as "views":
//    entry e of view v lives at byte (e * 8V + 8v), so lanes with different
//    v % V land in different bank pairs.  The gather is the in-core limit.
//  * Decode is exact: W = fp16_RNE(scale * cb) by __hmul2, then mma.sync
//    (fp16 x fp16 -> fp32).  Batch 1 takes fp32 x' and splits it into
//    hi + lo fp16 columns of the MMA (x' = hi + lo to ~22 bits), so the fp32
//    activation is not rounded to fp16.
#pragma once

#include "tq_common.cuh"
#include "tq_rht.cuh"

namespace tq {

constexpr int DMMA_WARPS = 16;
constexpr int DMMA_THREADS = DMMA_WARPS * 32;
constexpr int DMMA_MAX_WARPS = 8192;  // bound on active warps (workspace sizing)

struct DmmaSeg {
  const uint8_t* codes;
  const uint16_t* scales;
  int32_t rows;
  int32_t row0;  // first row of this segment in the concatenated output
};

struct DmmaParams {
  DmmaSeg seg[3];
  int32_t nseg;
  const uint16_t* codebook;
  int32_t n_total;
  int32_t k;
  int32_t m;
  const float* x_f32;      // batch 1: x' fp32 [k]
  const uint16_t* x_bf16;  // batch 1, fused RHT: x bf16 [k]
  uint64_t rht_seed;
  const uint16_t* x_f16;   // small batch: x' fp16 in fragment order (xt_pos), whole groups of 8 tokens
  float* y;                // [m][n_total] or null
  uint16_t* handoff;       // [m][handoff_rows] bf16 or null
  int32_t handoff_rows;
  float alpha;
  float* partials;         // [active_warps][2][16 * MC]
  int32_t* counters;       // [tiles]
  int32_t tiles;
  int32_t blocks;          // k / 256
  int64_t units;           // tiles * blocks
  int32_t active_warps;
  uint64_t rcp_active;     // floor((2^64 - 1) / active_warps), floor((2^64 - 1) / units):
  uint64_t rcp_units;      // exact divisions by multiply-high (persistent stack kernel)
};

__host__ __device__ __forceinline__ int64_t dmma_warp_begin(int64_t w, int64_t units, int64_t active) {
  return (w * units) / active;
}
// The warp whose range contains unit u.
__host__ __device__ __forceinline__ int64_t dmma_warp_of(int64_t u, int64_t units, int64_t active) {
  return ((u + 1) * active + units - 1) / units - 1;
}

// Shared-memory offset of the hi (n=0) or lo (n=1) fp16 quad of group G
// (group 16q + j of a 256-block is read by lanes with q = lane % 4 at MMA step
// j), stored as [block][j / 2][q][n][j % 2]: a lane's quads of steps j and
// j + 1 are one 16-byte load, and the 8 lanes that read a step pair hit 128
// contiguous bytes.
__device__ __forceinline__ uint32_t xs_offset(int G, int n) {
  const int b = G >> 6, j = G & 15, q = (G >> 4) & 3;
  return (uint32_t)((((((b << 3) + (j >> 1)) << 2) + q) * 2 + n) * 2 + (j & 1)) * 8;
}

__device__ __forceinline__ void store_hilo(uint8_t* xs, int G, float a, float b, float c, float d) {
  uint32_t h0 = f2_to_h2(a, b), h1 = f2_to_h2(c, d);
  float2 f0 = h2_to_f2(h0), f1 = h2_to_f2(h1);
  uint32_t l0 = f2_to_h2(a - f0.x, b - f0.y), l1 = f2_to_h2(c - f1.x, d - f1.y);
  *reinterpret_cast<uint2*>(xs + xs_offset(G, 0)) = make_uint2(h0, h1);
  *reinterpret_cast<uint2*>(xs + xs_offset(G, 1)) = make_uint2(l0, l1);
}

struct DmmaChunk {
  uint4 ca, cb;    // 16 code bytes of rows g and g+8
  uint32_t sa, sb; // fp16 scales of rows g and g+8 (block b)
};

__device__ __forceinline__ void seg_lookup(const DmmaParams& p, int row, const uint8_t*& codes,
                                           const uint16_t*& scales, int& local) {
  int s = 0;
  if (p.nseg > 1 && row >= p.seg[1].row0) s = 1;
  if (p.nseg > 2 && row >= p.seg[2].row0) s = 2;
  codes = s == 0 ? p.seg[0].codes : (s == 1 ? p.seg[1].codes : p.seg[2].codes);
  scales = s == 0 ? p.seg[0].scales : (s == 1 ? p.seg[1].scales : p.seg[2].scales);
  local = row - (s == 0 ? p.seg[0].row0 : (s == 1 ? p.seg[1].row0 : p.seg[2].row0));
}

// Pointers of this lane's two rows (g, g+8) of tile t at block 0: code bytes
// of chunk q and the row's scales.  Rows past the end are clamped (their
// results are never stored).
struct DmmaRows {
  const uint8_t* ca;
  const uint8_t* cb;
  const uint16_t* sa;
  const uint16_t* sb;
};

__device__ __forceinline__ DmmaRows dmma_rows(const DmmaParams& p, int t, int g, int q) {
  const int r0 = min(t * 16 + g, p.n_total - 1), r1 = min(t * 16 + g + 8, p.n_total - 1);
  const uint8_t *c0, *c1;
  const uint16_t *s0, *s1;
  int l0, l1;
  seg_lookup(p, r0, c0, s0, l0);
  seg_lookup(p, r1, c1, s1, l1);
  const int gpr = p.k >> 2;
  DmmaRows r;
  r.ca = c0 + (size_t)l0 * gpr + q * 16;
  r.cb = c1 + (size_t)l1 * gpr + q * 16;
  r.sa = s0 + (size_t)l0 * p.blocks;
  r.sb = s1 + (size_t)l1 * p.blocks;
  return r;
}

// Codes of block b, and its scales from the scale-pair words (spa, spb) of
// blocks (b & ~1, b | 1): loaded here when b is even or `fresh` (the first
// block of a range), else left from the fetch of block b - 1.  Rows hold an
// even number of blocks (k is a multiple of 512), so the words are aligned.
__device__ __forceinline__ DmmaChunk dmma_fetch(const DmmaRows& r, int b, uint32_t& spa, uint32_t& spb,
                                               bool fresh) {
  DmmaChunk ch;
  ch.ca = ldg_stream_u4(r.ca + b * 64);
  ch.cb = ldg_stream_u4(r.cb + b * 64);
  if (fresh || (b & 1) == 0) {
    spa = __ldg(reinterpret_cast<const uint32_t*>(r.sa + (b & ~1)));
    spb = __ldg(reinterpret_cast<const uint32_t*>(r.sb + (b & ~1)));
  }
  ch.sa = (b & 1) ? (spa >> 16) : (spa & 0xFFFFu);
  ch.sb = (b & 1) ? (spb >> 16) : (spb & 0xFFFFu);
  return ch;
}

// Offsets (bytes, relative to the views base) of the 4 codebook entries of
// one 32-bit code word.  `r` is the byte-reversed word, `prev_hi` holds the
// previous code in bits 0-7.  Entry e = (prev & 7) << 8 | code sits at
// e << SH (+ view offset); the shifts put code at bit SH and prev at SH + 8.
template <int SH>
__device__ __forceinline__ void word_offsets(uint32_t r, uint32_t prev_hi, uint32_t vofs, uint32_t off[4]) {
  constexpr uint32_t MASK = 0x7FFu << SH;
  off[0] = (__funnelshift_r(r, prev_hi, 24 - SH) & MASK) | vofs;
  off[1] = ((r >> (16 - SH)) & MASK) | vofs;
  off[2] = ((r >> (8 - SH)) & MASK) | vofs;
  off[3] = ((r << SH) & MASK) | vofs;
}

template <int NT, bool HILO>
__device__ __forceinline__ void dmma_epilogue(const DmmaParams& p, int t, int g, int q, const float (&v)[NT][4]) {
  const int R0 = t * 16 + g, R1 = R0 + 8;
  if (HILO) {
    if (q != 0) return;
    const float y0 = v[0][0] + v[0][1], y1 = v[0][2] + v[0][3];
    if (R0 < p.n_total) {
      if (p.y) p.y[R0] = y0;
      if (R0 < p.handoff_rows) p.handoff[R0] = f_to_bf16_bits(p.alpha * y0);
    }
    if (R1 < p.n_total) {
      if (p.y) p.y[R1] = y1;
      if (R1 < p.handoff_rows) p.handoff[R1] = f_to_bf16_bits(p.alpha * y1);
    }
  } else {
#pragma unroll
    for (int jt = 0; jt < NT; ++jt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int tok = jt * 8 + 2 * q + e;
        if (tok >= p.m) continue;
        if (R0 < p.n_total) {
          const float y = v[jt][e];
          if (p.y) p.y[(size_t)tok * p.n_total + R0] = y;
          if (R0 < p.handoff_rows) p.handoff[(size_t)tok * p.handoff_rows + R0] = f_to_bf16_bits(p.alpha * y);
        }
        if (R1 < p.n_total) {
          const float y = v[jt][2 + e];
          if (p.y) p.y[(size_t)tok * p.n_total + R1] = y;
          if (R1 < p.handoff_rows) p.handoff[(size_t)tok * p.handoff_rows + R1] = f_to_bf16_bits(p.alpha * y);
        }
      }
    }
  }
}

// Element index (within a tile's 16 x MC partial) of accumulator value (jt, i).
template <int NT, bool HILO>
__device__ __forceinline__ int partial_index(int g, int q, int jt, int i) {
  constexpr int MC = HILO ? 1 : NT * 8;
  if (HILO) return (i < 2) ? g : g + 8;
  const int row = (i < 2) ? g : g + 8;
  return row * MC + jt * 8 + 2 * q + (i & 1);
}

// A tile whose units span several warps: each contributor writes its partial
// sum (slot 0 = the contributor's first tile, slot 1 = a later one), bumps the
// tile's counter, and the last to arrive sums all of them in warp order.
template <int NT, bool HILO>
__device__ __forceinline__ void dmma_write_partial(const DmmaParams& p, int64_t W, int slot, int g, int q,
                                                   const float (&acc)[NT][4]) {
  constexpr int MC = HILO ? 1 : NT * 8;
  float* part = p.partials + ((size_t)W * 2 + slot) * (16 * MC);
  if (HILO) {
    if (q == 0) {
      part[g] = acc[0][0] + acc[0][1];
      part[g + 8] = acc[0][2] + acc[0][3];
    }
  } else {
#pragma unroll
    for (int jt = 0; jt < NT; ++jt)
#pragma unroll
      for (int i = 0; i < 4; ++i) part[partial_index<NT, HILO>(g, q, jt, i)] = acc[jt][i];
  }
}

// Called by the tile's last contributor (after its counter increment saw
// every other one): sum the partials in warp order (grouped by CTA), write
// y / handoff, and leave the counter at zero for the next call.
template <int NT, bool HILO>
__device__ __forceinline__ void dmma_reduce_tile(const DmmaParams& p, int t, int g, int q) {
  constexpr int MC = HILO ? 1 : NT * 8;
  const int lane = threadIdx.x & 31;
  const int64_t B = p.blocks;
  const int64_t t0 = (int64_t)t * B, t1 = t0 + B;
  const int64_t wa = dmma_warp_of(t0, p.units, p.active_warps);
  const int64_t wz = dmma_warp_of(t1 - 1, p.units, p.active_warps);
  __threadfence();
  // Only the first contributor can have started before the tile (then the
  // tile is its slot 1); every later one starts inside it (slot 0).  Loads
  // are issued CB contributors at a time.
  constexpr int CB = NT >= 8 ? 1 : 8 / NT;
  // Partials are summed per group of DMMA_WARPS consecutive warps (one CTA)
  // first, then the group sums in order: the same association as a two-level
  // (CTA, then grid) reduction, so both give identical bits.
  float sum[NT][4], gsum[NT][4];
#pragma unroll
  for (int jt = 0; jt < NT; ++jt)
#pragma unroll
    for (int i = 0; i < 4; ++i) sum[jt][i] = gsum[jt][i] = 0.f;
  const int first_slot = (dmma_warp_begin(wa, p.units, p.active_warps) >= t0) ? 0 : 1;
  const int ncontrib = (int)(wz - wa) + 1;
  for (int c0 = 0; c0 < ncontrib; c0 += CB) {
    float v[CB][NT][4];
#pragma unroll
    for (int c = 0; c < CB; ++c) {
      const int cc = min(c0 + c, ncontrib - 1);
      const int64_t w = wa + cc;
      const int s = (cc == 0) ? first_slot : 0;
      const float* src = p.partials + ((size_t)w * 2 + s) * (16 * MC);
#pragma unroll
      for (int jt = 0; jt < NT; ++jt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (HILO) {
            v[c][jt][i] = (jt == 0 && (i == 0 || i == 2)) ? __ldcg(src + (i == 0 ? g : g + 8)) : 0.f;
          } else {
            v[c][jt][i] = __ldcg(src + partial_index<NT, HILO>(g, q, jt, i));
          }
        }
    }
#pragma unroll
    for (int c = 0; c < CB; ++c)
      if (c0 + c < ncontrib) {
        if (c0 + c > 0 && ((wa + c0 + c) % DMMA_WARPS) == 0) {  // next CTA-sized group
#pragma unroll
          for (int jt = 0; jt < NT; ++jt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              sum[jt][i] += gsum[jt][i];
              gsum[jt][i] = 0.f;
            }
        }
#pragma unroll
        for (int jt = 0; jt < NT; ++jt)
#pragma unroll
          for (int i = 0; i < 4; ++i) gsum[jt][i] += v[c][jt][i];
      }
  }
#pragma unroll
  for (int jt = 0; jt < NT; ++jt)
#pragma unroll
    for (int i = 0; i < 4; ++i) sum[jt][i] += gsum[jt][i];
  dmma_epilogue<NT, HILO>(p, t, g, q, sum);
  if (lane == 0) p.counters[t] = 0;  // leave the counter ready for the next call
}

// Number of warps whose unit ranges meet tile t.
__device__ __forceinline__ int dmma_contributors(const DmmaParams& p, int t) {
  const int64_t t0 = (int64_t)t * p.blocks, t1 = t0 + p.blocks;
  return (int)(dmma_warp_of(t1 - 1, p.units, p.active_warps) - dmma_warp_of(t0, p.units, p.active_warps)) + 1;
}

// End of a warp's unit range: publish the (at most two) tiles it shares with
// other warps -- the first tile of the range (its sums kept in registers
// since that tile ended) and the last -- with ONE fence, then finish the ones
// this warp was last to reach.  Deferring the first tile keeps the fence and
// the counter round trip out of the code stream.
template <int NT, bool HILO>
__device__ __forceinline__ void dmma_publish(const DmmaParams& p, int64_t W, int g, int q, bool has_head, int head_t,
                                             const float (&hacc)[NT][4], bool has_tail, int tail_t, int tail_slot,
                                             const float (&tacc)[NT][4]) {
  const int lane = threadIdx.x & 31;
  if (has_head) dmma_write_partial<NT, HILO>(p, W, 0, g, q, hacc);
  if (has_tail) dmma_write_partial<NT, HILO>(p, W, tail_slot, g, q, tacc);
  __threadfence();
  __syncwarp();
  int oh = 0, ot = 0;
  if (lane == 0) {
    if (has_head) oh = atomicAdd(p.counters + head_t, 1);
    if (has_tail) ot = atomicAdd(p.counters + tail_t, 1);
  }
  oh = __shfl_sync(0xffffffffu, oh, 0);
  ot = __shfl_sync(0xffffffffu, ot, 0);
  if (has_head && oh == dmma_contributors(p, head_t) - 1) dmma_reduce_tile<NT, HILO>(p, head_t, g, q);
  if (has_tail && ot == dmma_contributors(p, tail_t) - 1) dmma_reduce_tile<NT, HILO>(p, tail_t, g, q);
}

// Replicate the codebook into V = 2^LV shared-memory views (entry e of view
// v at byte e*8V + 8v).
template <int LV>
__device__ __forceinline__ void build_views(uint8_t* smem, const uint16_t* __restrict__ codebook, int tid,
                                            int nthreads) {
  constexpr int V = 1 << LV;
  constexpr int SH = 3 + LV;
  for (int e = tid; e < 2048; e += nthreads) {
    const uint2 ent = reinterpret_cast<const uint2*>(codebook)[e];
    uint8_t* dst = smem + (e << SH);
    if (V == 1) {
      *reinterpret_cast<uint2*>(dst) = ent;
    } else {
#pragma unroll
      for (int v = 0; v < V; v += 2)
        *reinterpret_cast<uint4*>(dst + 8 * v) = make_uint4(ent.x, ent.y, ent.x, ent.y);
    }
  }
}

// Units [wb, we) of global warp W, the tile/block it starts at and its first
// chunk of code bytes (loaded ahead: the weights never depend on activations).
struct DmmaCursor {
  int64_t wb, we;
  int t, b;
  DmmaRows rows;
  DmmaChunk cur;
  uint32_t spa, spb;  // scale-pair words of block b's pair (see dmma_fetch)
};

__device__ __forceinline__ void dmma_begin(const DmmaParams& p, int64_t W, int g, int q, DmmaCursor& c) {
  const bool active = W < p.active_warps;
  c.wb = active ? dmma_warp_begin(W, p.units, p.active_warps) : 0;
  c.we = active ? dmma_warp_begin(W + 1, p.units, p.active_warps) : 0;
  c.t = c.b = 0;
  if (c.wb < c.we) {
    c.t = (int)(c.wb / p.blocks);
    c.b = (int)(c.wb - (int64_t)c.t * p.blocks);
    c.rows = dmma_rows(p, c.t, g, q);
    c.cur = dmma_fetch(c.rows, c.b, c.spa, c.spb, true);
  }
}

// Batch-1 activation quads of two MMA steps for lanes 0-7 (lanes g = 0 / 1
// hold the hi / lo column); the other lanes own MMA columns that are never
// read and skip the load (predicated, no branch).
__device__ __forceinline__ uint4 lds_b_hilo(const uint8_t* addr, int lane) {
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  asm volatile(
      "{\n .reg .pred p;\n setp.lt.u32 p, %4, 8;\n @p ld.shared.v4.u32 {%0,%1,%2,%3}, [%5];\n}\n"
      : "+r"(v.x), "+r"(v.y), "+r"(v.z), "+r"(v.w)
      : "r"(lane), "r"(smem_u32(addr)));
  return v;
}

// The unit loop of one warp: decode its units, run the MMAs, flush tiles.
// `smem` holds the codebook views, `xs` the batch-1 activations (hi/lo).
// With `wslots` (batch 1 only) the tiles this warp shares with other warps
// are not published through global memory: their partial sums go to this
// warp's two shared-memory slots ([2][16] floats, slot 0 = the range's first
// tile), for a reduction by the whole CTA.
// With `xflag` (batch 1, persistent stack) the activations are produced
// block by block while the units run: before reading the x' of a 512-block
// for the first time, the warp waits (bounded; on timeout the status word
// gets TQ_ERR_TIMEOUT) until xflag[block] == xtag.
__device__ __forceinline__ void wait_xflag(const volatile int* xflag, int blk, int xtag, int32_t* status,
                                           uint32_t spin_limit) {
  const int lane = threadIdx.x & 31;
  if (lane == 0) {
    uint32_t spins = 0;
    while (xflag[blk] != xtag) {
      if (++spins > spin_limit) {
        if (status) atomicExch(status, 7);  // TQ_ERR_TIMEOUT
        break;
      }
      __nanosleep(20);
    }
  }
  __syncwarp();
  __threadfence_block();
}

// XCG: the small-batch activations were written earlier in the same launch
// (persistent stack), so they are read with coherent loads (ld.global.ca)
// instead of the read-only path: the writes are released before the grid
// barrier and acquired by the barrier's waiting thread, whose CTA barrier
// then orders every thread's later loads after that acquire, so L1 holds no
// stale line of them; a CTA's units reuse each block of x' across tiles.
// A warp's partial of one tile into its shared-memory slot (16 rows x MC
// tokens, the layout of the global partials).
template <int NT, bool HILO>
__device__ __forceinline__ void dmma_slot_store(float* wslots, int slot, int g, int q, const float (&acc)[NT][4]) {
  constexpr int MC = HILO ? 1 : NT * 8;
  float* s = wslots + slot * 16 * MC;
  if (HILO) {
    if (q == 0) {
      s[g] = acc[0][0] + acc[0][1];
      s[g + 8] = acc[0][2] + acc[0][3];
    }
  } else {
#pragma unroll
    for (int jt = 0; jt < NT; ++jt)
#pragma unroll
      for (int i = 0; i < 4; ++i) s[partial_index<NT, HILO>(g, q, jt, i)] = acc[jt][i];
  }
}

// SLOTS: tiles shared with other warps go to the warp's shared-memory slots
// (wslots, persistent stack kernels) as soon as they end, holding no register
// copy of the first tile until the end of the range.
template <int LV, int NT, bool HILO, bool XCG = false, bool SLOTS = false>
__device__ __forceinline__ void dmma_units(const DmmaParams& p, const uint8_t* smem, const uint8_t* xs, int64_t W,
                                           DmmaCursor& c, int lane, float* wslots = nullptr,
                                           const volatile int* xflag = nullptr, int xtag = 0,
                                           int32_t* status = nullptr, uint32_t spin_limit = 0) {
  constexpr int V = 1 << LV;
  constexpr int SH = 3 + LV;
  const int g = lane >> 2, q = lane & 3;
  if (c.wb >= c.we) return;
  int t = c.t, b = c.b;
  DmmaRows rows = c.rows;
  DmmaChunk cur = c.cur;
  uint32_t spa = c.spa, spb = c.spb;
  const uint32_t vofs = (uint32_t)((lane & (V - 1)) << 3);
  // two accumulator sets (even / odd code steps) halve the MMA dependency chain
  float acc[NT][4], acc2[NT][4];
#pragma unroll
  for (int jt = 0; jt < NT; ++jt)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[jt][i] = acc2[jt][i] = 0.f;

  const int nunits = (int)(c.we - c.wb);
  int ready_rb = -1;  // x' block known to be stored (xflag mode)
  bool has_head = false, has_tail = false;
  int head_t = 0, tail_t = 0;
  float hacc[NT][4];
#pragma unroll
  for (int jt = 0; jt < NT; ++jt)
#pragma unroll
    for (int i = 0; i < 4; ++i) hacc[jt][i] = 0.f;
  for (int iu = 0; iu < nunits; ++iu) {
    int tn = t, bn = b + 1;
    if (bn == p.blocks) {
      bn = 0;
      ++tn;
    }
    DmmaRows nrows = rows;
    DmmaChunk nxt;
    if (iu + 1 < nunits) {
      if (bn == 0) nrows = dmma_rows(p, tn, g, q);
      nxt = dmma_fetch(nrows, bn, spa, spb, false);
    }

    if (HILO && xflag && (b >> 1) != ready_rb) {
      ready_rb = b >> 1;
      wait_xflag(xflag, ready_rb, xtag, status, spin_limit);
    }
    const uint8_t* xs_lane = xs + ((((b << 3) << 2) + q) * 2 + (g & 1)) * 16;  // step pair 0
    uint4 bw2 = make_uint4(0u, 0u, 0u, 0u);
    const uint16_t* xg_lane[NT];
    uint4 bpair[NT];
#pragma unroll
    for (int jt = 0; jt < NT; ++jt)  // step pair 0 of block b, tokens 8 jt .. 8 jt + 7 (xt_pos); column
      // tiles past the last group of 8 tokens re-read it (their outputs are discarded)
      xg_lane[jt] = p.x_f16 + (size_t)min(jt, (p.m - 1) >> 3) * 8 * p.k + (size_t)b * 2048 + lane * 8;
    // previous code byte of each row chunk (state of code 0); 0 at a block start
    uint32_t pa = __shfl_up_sync(0xffffffffu, cur.ca.w, 1) >> 24;
    uint32_t pb = __shfl_up_sync(0xffffffffu, cur.cb.w, 1) >> 24;
    if (q == 0) pa = pb = 0;
    const uint32_t wa[4] = {cur.ca.x, cur.ca.y, cur.ca.z, cur.ca.w};
    const uint32_t wbw[4] = {cur.cb.x, cur.cb.y, cur.cb.z, cur.cb.w};
    const uint32_t sa2 = cur.sa | (cur.sa << 16), sb2 = cur.sb | (cur.sb << 16);

#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t ra = __byte_perm(wa[i], 0, 0x0123), rb = __byte_perm(wbw[i], 0, 0x0123);
      const uint32_t ha = (i == 0) ? pa : __byte_perm(wa[i - 1], 0, 0x0123);
      const uint32_t hb = (i == 0) ? pb : __byte_perm(wbw[i - 1], 0, 0x0123);
      uint32_t oa[4], ob[4];
      word_offsets<SH>(ra, ha, vofs, oa);
      word_offsets<SH>(rb, hb, vofs, ob);
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int j = i * 4 + jj;
        const uint2 ea = *reinterpret_cast<const uint2*>(smem + oa[jj]);
        const uint2 eb = *reinterpret_cast<const uint2*>(smem + ob[jj]);
        uint32_t a[4];
        a[0] = hmul2_u32(ea.x, sa2);
        a[2] = hmul2_u32(ea.y, sa2);
        a[1] = hmul2_u32(eb.x, sb2);
        a[3] = hmul2_u32(eb.y, sb2);
        // B columns other than the live ones (hi/lo at batch 1, tokens < m
        // otherwise) only feed C columns that are never read.
        if (HILO) {
          if ((j & 1) == 0) bw2 = lds_b_hilo(xs_lane + (j >> 1) * 128, lane);  // steps j, j + 1
          mma_16816((j & 1) ? acc2[0] : acc[0], a, (j & 1) ? bw2.z : bw2.x, (j & 1) ? bw2.w : bw2.y);
        } else {
          // one 16-byte load holds this lane's quads of steps j and j + 1
          if ((j & 1) == 0) {
#pragma unroll
            for (int jt = 0; jt < NT; ++jt)
              bpair[jt] = XCG ? __ldca(reinterpret_cast<const uint4*>(xg_lane[jt] + 128 * j))
                              : __ldg(reinterpret_cast<const uint4*>(xg_lane[jt] + 128 * j));
          }
#pragma unroll
          for (int jt = 0; jt < NT; ++jt) {
            const uint32_t b0 = (j & 1) ? bpair[jt].z : bpair[jt].x, b1 = (j & 1) ? bpair[jt].w : bpair[jt].y;
            mma_16816((j & 1) ? acc2[jt] : acc[jt], a, b0, b1);
          }
        }
      }
    }

    if (iu + 1 == nunits || bn == 0) {  // tile t ends here (for this warp)
#pragma unroll
      for (int jt = 0; jt < NT; ++jt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[jt][i] += acc2[jt][i];
      const int64_t t0 = (int64_t)t * p.blocks;
      if (t0 >= c.wb && t0 + p.blocks <= c.we) {
        dmma_epilogue<NT, HILO>(p, t, g, q, acc);  // the whole tile ran in this warp
      } else if (iu + 1 < nunits) {
        // the range's first tile, shared with earlier warps: publish it at the
        // end (8 column tiles keep no second register copy: publish now)
        if (SLOTS) {
          dmma_slot_store<NT, HILO>(wslots, 0, g, q, acc);
        } else if (NT <= 4) {
          has_head = true;
          head_t = t;
#pragma unroll
          for (int jt = 0; jt < NT; ++jt)
#pragma unroll
            for (int i = 0; i < 4; ++i) hacc[jt][i] = acc[jt][i];
        } else {
          dmma_publish<NT, HILO>(p, W, g, q, true, t, acc, false, 0, 0, acc);
        }
      } else {
        has_tail = true;
        tail_t = t;
      }
      if (iu + 1 < nunits || !has_tail) {
#pragma unroll
        for (int jt = 0; jt < NT; ++jt)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[jt][i] = acc2[jt][i] = 0.f;
      }
    }
    t = tn;
    b = bn;
    rows = nrows;
    cur = nxt;
  }
  if (has_head || has_tail) {
    // slot 0 holds the range's first tile, slot 1 a later one
    const int tail_slot = (tail_t == (int)(c.wb / p.blocks)) ? 0 : 1;
    if (SLOTS) {
      if (has_tail) dmma_slot_store<NT, HILO>(wslots, tail_slot, g, q, acc);  // the head is already in slot 0
    } else {
      dmma_publish<NT, HILO>(p, W, g, q, has_head, head_t, hacc, has_tail, tail_t, tail_slot, acc);
    }
  }
}

// Batch-1 activations of the block: x' = RHT(x_bf16) computed here, or x' fp32
// given, split into hi/lo fp16 quads in shared memory.
__device__ __forceinline__ void dmma_prologue_hilo(const DmmaParams& p, uint8_t* xs, int tid, int nthreads) {
  const int lane = tid & 31, warp = tid >> 5, nwarps = nthreads >> 5;
  if (p.x_bf16) {
    for (int blk = warp; blk < p.k / 512; blk += nwarps) {
      float v[16];
      rht512_warp(p.x_bf16, blk, p.rht_seed, v);
#pragma unroll
      for (int r4 = 0; r4 < 4; ++r4)
        store_hilo(xs, blk * 128 + lane * 4 + r4, v[4 * r4], v[4 * r4 + 1], v[4 * r4 + 2], v[4 * r4 + 3]);
    }
  } else {
    for (int G = tid; G < (p.k >> 2); G += nthreads) {
      const float4 x = reinterpret_cast<const float4*>(p.x_f32)[G];
      store_hilo(xs, G, x.x, x.y, x.z, x.w);
    }
  }
}

// LV = log2(number of codebook views); NT = number of 8-token MMA column
// tiles (small batch); HILO = batch-1 mode with fp32 x' split in hi/lo.
template <int LV, int NT, bool HILO>
__global__ void __launch_bounds__(DMMA_THREADS, 1) dmma_kernel(const __grid_constant__ DmmaParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* xs = smem + (16384 << LV);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  pdl_launch_dependents();
  build_views<LV>(smem, p.codebook, tid, DMMA_THREADS);  // no kernel of the stream writes the codebook
  const int64_t W = (int64_t)blockIdx.x * DMMA_WARPS + warp;
  DmmaCursor c;
  dmma_begin(p, W, lane >> 2, lane & 3, c);  // weights: prefetched before waiting on the previous kernel
  pdl_wait();
  if (HILO) dmma_prologue_hilo(p, xs, tid, DMMA_THREADS);
  __syncthreads();
  dmma_units<LV, NT, HILO>(p, smem, xs, W, c, lane);
}

// ---- two row tiles per warp (17-32 tokens) ------------------------------------
//
// At 17-32 tokens (four 8-token column tiles) the unit loop above spends as
// many L1 wavefronts on x' as on the codebook gathers: every 16-row unit loads
// its 16 KB of x' again.  Here a warp's unit is 32 rows x one 256-weight block:
// lane (g, q) decodes rows g, g+8, g+16 and g+24, and both 16-row MMA tiles
// use the same x' registers, so x' costs half as many wavefronts per weight.
// The extra registers (codes, scales and accumulators of two more rows) do not
// fit 16 warps at 128 registers each, so this kernel runs 8 warps per SM with
// up to 255 registers.  Tiles are 32 rows; a tile split across warps is summed
// by the last warp to arrive, in warp order.  Batch 1 and the persistent stack
// kernels keep the 16-row loop above.
constexpr int DMMA2_WARPS = 8;
constexpr int DMMA2_THREADS = DMMA2_WARPS * 32;

struct DmmaRows2 {
  const uint8_t* c[4];  // code bytes of rows g + 8 i, chunk q, block 0
  const uint16_t* s[4]; // their scales
};

struct DmmaChunk2 {
  uint4 c[4];
  uint32_t s[4];
};

__device__ __forceinline__ DmmaRows2 dmma2_rows(const DmmaParams& p, int t, int g, int q) {
  DmmaRows2 r;
  const int gpr = p.k >> 2;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = min(t * 32 + g + 8 * i, p.n_total - 1);  // rows past the end are clamped, never stored
    const uint8_t* c;
    const uint16_t* sc;
    int l;
    seg_lookup(p, row, c, sc, l);
    r.c[i] = c + (size_t)l * gpr + q * 16;
    r.s[i] = sc + (size_t)l * p.blocks;
  }
  return r;
}

// Codes of block b, scales from the scale-pair words (see dmma_fetch).
__device__ __forceinline__ DmmaChunk2 dmma2_fetch(const DmmaRows2& r, int b, uint32_t (&sp)[4], bool fresh) {
  DmmaChunk2 ch;
#pragma unroll
  for (int i = 0; i < 4; ++i) ch.c[i] = ldg_stream_u4(r.c[i] + b * 64);
  if (fresh || (b & 1) == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) sp[i] = __ldg(reinterpret_cast<const uint32_t*>(r.s[i] + (b & ~1)));
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) ch.s[i] = (b & 1) ? (sp[i] >> 16) : (sp[i] & 0xFFFFu);
  return ch;
}

// Element of a 32-row x MC partial for accumulator value (h, jt, i) of lane (g, q).
template <int NT>
__device__ __forceinline__ int dmma2_pidx(int g, int q, int h, int jt, int i) {
  constexpr int MC = NT * 8;
  return (16 * h + g + ((i < 2) ? 0 : 8)) * MC + jt * 8 + 2 * q + (i & 1);
}

template <int NT>
__device__ __forceinline__ void dmma2_epilogue(const DmmaParams& p, int t, int g, int q, const float (&v)[2][NT][4]) {
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int jt = 0; jt < NT; ++jt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int tok = jt * 8 + 2 * q + (i & 1);
        const int row = t * 32 + 16 * h + g + ((i < 2) ? 0 : 8);
        if (tok < p.m && row < p.n_total) {
          const float y = v[h][jt][i];
          if (p.y) p.y[(size_t)tok * p.n_total + row] = y;
          if (row < p.handoff_rows) p.handoff[(size_t)tok * p.handoff_rows + row] = f_to_bf16_bits(p.alpha * y);
        }
      }
}

template <int NT>
__device__ __forceinline__ void dmma2_write_partial(const DmmaParams& p, int64_t W, int slot, int g, int q,
                                                    const float (&acc)[2][NT][4]) {
  constexpr int MC = NT * 8;
  float* part = p.partials + ((size_t)W * 2 + slot) * (32 * MC);
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int jt = 0; jt < NT; ++jt)
#pragma unroll
      for (int i = 0; i < 4; ++i) part[dmma2_pidx<NT>(g, q, h, jt, i)] = acc[h][jt][i];
}

// The last contributor of tile t sums every contributor's partial in warp order.
template <int NT>
__device__ __forceinline__ void dmma2_reduce_tile(const DmmaParams& p, int t, int g, int q) {
  constexpr int MC = NT * 8;
  const int lane = threadIdx.x & 31;
  const int64_t t0 = (int64_t)t * p.blocks, t1 = t0 + p.blocks;
  const int64_t wa = dmma_warp_of(t0, p.units, p.active_warps);
  const int64_t wz = dmma_warp_of(t1 - 1, p.units, p.active_warps);
  __threadfence();
  const int first_slot = (dmma_warp_begin(wa, p.units, p.active_warps) >= t0) ? 0 : 1;
  float sum[2][NT][4];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int jt = 0; jt < NT; ++jt)
#pragma unroll
      for (int i = 0; i < 4; ++i) sum[h][jt][i] = 0.f;
  for (int64_t w = wa; w <= wz; ++w) {
    const int s = (w == wa) ? first_slot : 0;
    const float* src = p.partials + ((size_t)w * 2 + s) * (32 * MC);
    float v[2][NT][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int jt = 0; jt < NT; ++jt)
#pragma unroll
        for (int i = 0; i < 4; ++i) v[h][jt][i] = __ldcg(src + dmma2_pidx<NT>(g, q, h, jt, i));
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int jt = 0; jt < NT; ++jt)
#pragma unroll
        for (int i = 0; i < 4; ++i) sum[h][jt][i] += v[h][jt][i];
  }
  dmma2_epilogue<NT>(p, t, g, q, sum);
  if (lane == 0) p.counters[t] = 0;  // leave the counter ready for the next call
}

template <int NT>
__device__ __forceinline__ void dmma2_publish(const DmmaParams& p, int64_t W, int g, int q, bool has_head, int head_t,
                                              const float (&hacc)[2][NT][4], bool has_tail, int tail_t, int tail_slot,
                                              const float (&tacc)[2][NT][4]) {
  const int lane = threadIdx.x & 31;
  if (has_head) dmma2_write_partial<NT>(p, W, 0, g, q, hacc);
  if (has_tail) dmma2_write_partial<NT>(p, W, tail_slot, g, q, tacc);
  __threadfence();
  __syncwarp();
  int oh = 0, ot = 0;
  if (lane == 0) {
    if (has_head) oh = atomicAdd(p.counters + head_t, 1);
    if (has_tail) ot = atomicAdd(p.counters + tail_t, 1);
  }
  oh = __shfl_sync(0xffffffffu, oh, 0);
  ot = __shfl_sync(0xffffffffu, ot, 0);
  if (has_head && oh == dmma_contributors(p, head_t) - 1) dmma2_reduce_tile<NT>(p, head_t, g, q);
  if (has_tail && ot == dmma_contributors(p, tail_t) - 1) dmma2_reduce_tile<NT>(p, tail_t, g, q);
}

// Units [wb, we) of warp W and its first chunk of codes (loaded ahead: the
// weights never depend on activations).
struct DmmaCursor2 {
  int64_t wb, we;
  int t, b;
  DmmaRows2 rows;
  DmmaChunk2 cur;
  uint32_t sp[4];
};

__device__ __forceinline__ void dmma2_begin(const DmmaParams& p, int64_t W, int g, int q, DmmaCursor2& c) {
  const bool active = W < p.active_warps;
  c.wb = active ? dmma_warp_begin(W, p.units, p.active_warps) : 0;
  c.we = active ? dmma_warp_begin(W + 1, p.units, p.active_warps) : 0;
  c.t = c.b = 0;
  if (c.wb < c.we) {
    c.t = (int)(c.wb / p.blocks);
    c.b = (int)(c.wb - (int64_t)c.t * p.blocks);
    c.rows = dmma2_rows(p, c.t, g, q);
    c.cur = dmma2_fetch(c.rows, c.b, c.sp, true);
  }
}

template <int LV, int NT>
__device__ __forceinline__ void dmma2_units(const DmmaParams& p, const uint8_t* smem, int64_t W, int lane,
                                            DmmaCursor2& c) {
  constexpr int V = 1 << LV;
  constexpr int SH = 3 + LV;
  const int g = lane >> 2, q = lane & 3;
  const int64_t wb = c.wb, we = c.we;
  if (wb >= we) return;
  int t = c.t, b = c.b;
  DmmaRows2 rows = c.rows;
  uint32_t sp[4] = {c.sp[0], c.sp[1], c.sp[2], c.sp[3]};
  DmmaChunk2 cur = c.cur;
  const uint32_t vofs = (uint32_t)((lane & (V - 1)) << 3);
  const int jt_last = (p.m - 1) >> 3;  // column tiles past it re-read it (their outputs are discarded)
  float acc[2][NT][4], hacc[2][NT][4];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int jt = 0; jt < NT; ++jt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[h][jt][i] = hacc[h][jt][i] = 0.f;
  bool has_head = false, has_tail = false;
  int head_t = 0, tail_t = 0;
  const int nunits = (int)(we - wb);
  for (int iu = 0; iu < nunits; ++iu) {
    int tn = t, bn = b + 1;
    if (bn == p.blocks) {
      bn = 0;
      ++tn;
    }
    DmmaRows2 nrows = rows;
    DmmaChunk2 nxt;
    if (iu + 1 < nunits) {
      if (bn == 0) nrows = dmma2_rows(p, tn, g, q);
      nxt = dmma2_fetch(nrows, bn, sp, false);
    }
    const uint16_t* xg_lane[NT];
#pragma unroll
    for (int jt = 0; jt < NT; ++jt)  // step pair 0 of block b, tokens of column tile jt (xt_pos)
      xg_lane[jt] = p.x_f16 + (size_t)min(jt, jt_last) * 8 * p.k + (size_t)b * 2048 + lane * 8;
    // previous code byte of each row chunk (state of code 0); 0 at a block start
    uint32_t pv[4], s2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      pv[i] = __shfl_up_sync(0xffffffffu, cur.c[i].w, 1) >> 24;
      if (q == 0) pv[i] = 0;
      s2[i] = cur.s[i] | (cur.s[i] << 16);
    }
    uint4 bpair[NT];
#pragma unroll
    for (int i4 = 0; i4 < 4; ++i4) {
      uint32_t off[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t w4[4] = {cur.c[i].x, cur.c[i].y, cur.c[i].z, cur.c[i].w};
        const uint32_t r = __byte_perm(w4[i4], 0, 0x0123);
        const uint32_t hp = (i4 == 0) ? pv[i] : __byte_perm(w4[i4 > 0 ? i4 - 1 : 0], 0, 0x0123);
        word_offsets<SH>(r, hp, vofs, off[i]);
      }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int j = i4 * 4 + jj;
        uint32_t a[2][4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint2 ea = *reinterpret_cast<const uint2*>(smem + off[2 * h][jj]);
          const uint2 eb = *reinterpret_cast<const uint2*>(smem + off[2 * h + 1][jj]);
          a[h][0] = hmul2_u32(ea.x, s2[2 * h]);
          a[h][2] = hmul2_u32(ea.y, s2[2 * h]);
          a[h][1] = hmul2_u32(eb.x, s2[2 * h + 1]);
          a[h][3] = hmul2_u32(eb.y, s2[2 * h + 1]);
        }
        // one 16-byte load holds this lane's quads of steps j and j + 1
        if ((j & 1) == 0) {
#pragma unroll
          for (int jt = 0; jt < NT; ++jt) bpair[jt] = __ldg(reinterpret_cast<const uint4*>(xg_lane[jt] + 128 * j));
        }
#pragma unroll
        for (int jt = 0; jt < NT; ++jt) {
          const uint32_t b0 = (j & 1) ? bpair[jt].z : bpair[jt].x, b1 = (j & 1) ? bpair[jt].w : bpair[jt].y;
#pragma unroll
          for (int h = 0; h < 2; ++h) mma_16816(acc[h][jt], a[h], b0, b1);
        }
      }
    }
    if (iu + 1 == nunits || bn == 0) {  // tile t ends here (for this warp)
      const int64_t t0 = (int64_t)t * p.blocks;
      if (t0 >= wb && t0 + p.blocks <= we) {
        dmma2_epilogue<NT>(p, t, g, q, acc);  // the whole tile ran in this warp
      } else if (iu + 1 < nunits) {
        has_head = true;  // the range's first tile, shared with earlier warps: published at the end
        head_t = t;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int jt = 0; jt < NT; ++jt)
#pragma unroll
            for (int i = 0; i < 4; ++i) hacc[h][jt][i] = acc[h][jt][i];
      } else {
        has_tail = true;
        tail_t = t;
      }
      if (iu + 1 < nunits) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int jt = 0; jt < NT; ++jt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[h][jt][i] = 0.f;
      }
    }
    t = tn;
    b = bn;
    rows = nrows;
    cur = nxt;
  }
  if (has_head || has_tail) {
    const int tail_slot = (tail_t == (int)(wb / p.blocks)) ? 0 : 1;  // slot 0 holds the range's first tile
    dmma2_publish<NT>(p, W, g, q, has_head, head_t, hacc, has_tail, tail_t, tail_slot, acc);
  }
}

template <int LV, int NT>
__global__ void __launch_bounds__(DMMA2_THREADS, 1) dmma_kernel_r2(const __grid_constant__ DmmaParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_launch_dependents();
  build_views<LV>(smem, p.codebook, tid, DMMA2_THREADS);  // no kernel of the stream writes the codebook
  const int64_t W = (int64_t)blockIdx.x * DMMA2_WARPS + warp;
  DmmaCursor2 c;
  dmma2_begin(p, W, lane >> 2, lane & 3, c);  // weights: requested before waiting on the previous kernel
  pdl_wait();
  __syncthreads();
  dmma2_units<LV, NT>(p, smem, W, lane, c);
}

}  // namespace tq
