// tq_umma.cuh -- decode-to-shared-memory tcgen05 GEMM for larger batches.
//
// y[t][n] = sum_k W[n][k] x'[t][k] with W decoded from the trellis codes
// ("Pingala-8" landing page, "How it works") straight into the shared-memory
// operand of the 5th-generation tensor cores; at a few dozen tokens and more
// the decoded contraction is a dense fp16 GEMM (the prompt-processing case of
// the landing page's "Limitations" list).
//
// One CTA computes a 128-row (weights) x BN-column (tokens) tile of y, over
// a contiguous range of 256-weight blocks of k (split-k when the tile count
// alone cannot fill the GPU):
//   warp 0      TMA producer: x' tile [BN x 64] (128B swizzle) and the code
//               tile [128 rows x 16 bytes] of each 64-wide k step
//   warp 1      TMEM allocation; one thread issues tcgen05.mma (M=128,
//               N=BN, K=16, fp16 x fp16 -> fp32) and tcgen05.commit
//   warps 4-11  decoders: two threads per row, 8 codes each (codebook in
//               shared memory, exact fp16 scale * entry), into the MMA's A
//               operand; then the epilogue (tcgen05.ld), warps 4-7 and 8-11
//               taking one half of the columns each
// Where A lives depends on the tile width:
//   * at 64 and 256 tokens, in tensor memory (tcgen05.st by the decoders; row
//     r of the tile in TMEM lane r, the fp16 pair (2c, 2c+1) of the k step in
//     column c of the stage).  At 256 tokens the loop is bound by shared
//     memory, where a decoded tile costs a 16 KB write and a 16 KB MMA read
//     per k step (without them: 16% faster on the Qwen3-4B gate|up shape at
//     512 tokens).  At 64 tokens the loop is bound by the latency of the
//     stage round trip (TMA in, decode, MMA, release); A out of shared memory
//     leaves room for 12 stages of 10 KB (6 stages of 26 KB with A in shared
//     memory were 15% faster than 4 on the 27B-class gate|up shape at 32
//     tokens, 12 in TMEM another 4-5% at 64 tokens);
//   * at 128 tokens, in shared memory (the K-major 128B-swizzled tile),
//     except in the two-CTA form (PAIR, below), which keeps it in TMEM.
// Stages are handed over with mbarriers; every wait is bounded and, when it
// runs out, the kernel records TQ_ERR_TIMEOUT in the status word and drains.
#pragma once

#include <cuda.h>

#include "tq_common.cuh"

namespace tq {

constexpr int UM_BM = 128;
constexpr int UM_BK = 64;
constexpr int UM_DEC_THREADS = 256;             // 8 decoder warps: 2 threads per row
constexpr int UM_THREADS = 128 + UM_DEC_THREADS;
constexpr int UM_TIMEOUT_STATUS = 7;  // TQ_ERR_TIMEOUT
constexpr int UM_SPLIT_BATCH = 4;     // split partials loaded together in the split-k sum

struct UmmaParams {
  CUtensorMap tmap_x;         // x' fp16 [m][k]: box {64, BN}, 128B swizzle
  CUtensorMap tmap_codes[3];  // codes uint8 [rows][k/4]: box {16, 128}
  const uint16_t* scales[3];
  int32_t seg_row0[3];        // first output row of each segment (multiple of 128)
  int32_t seg_rows[3];
  int32_t nseg;
  const uint16_t* codebook;
  int32_t n_total, k, m;
  float* y;            // [m][n_total] or null
  uint16_t* handoff;   // [m][handoff_rows] or null
  int32_t handoff_rows;
  float alpha;
  float* partials;     // [tiles][splits][BN][128]
  int32_t* counters;   // [tiles]
  int32_t* status;     // error word or null
  int32_t row_tiles, tok_tiles, splits;
  uint32_t spin_limit;  // bounded waits
  int32_t skip_arrive_cta;  // timeout test hook: this CTA's decoded-stage barriers expect one arrival
                            // too many, so its MMA wait runs out (-1 = off)
};

// ---- PTX wrappers -------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: false when the limit ran out.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t limit) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];\n" ::"r"(
          dst),
      "l"(map), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ uint64_t umma_smem_desc(uint32_t addr) {
  // K-major, 128-byte swizzle: 8-row core groups 1024 B apart (SBO), LBO
  // unused (16 B), descriptor version 1, layout type 2 (128B swizzle).
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// kind::f16 instruction descriptor: D f32, A/B f16, both K-major, M = 128, N = bn.
__host__ __device__ constexpr uint32_t umma_idesc(int bn) {
  return (1u << 4) | ((uint32_t)(bn >> 3) << 17) | ((uint32_t)(UM_BM >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// The same MMA with A read from tensor memory (tmem_a: lane = row, 32-bit
// column = two consecutive k).
__device__ __forceinline__ void umma_f16_tmem_a(uint32_t tmem_d, uint32_t tmem_a, uint64_t b, uint32_t idesc,
                                                uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(
          tmem_d),
      "r"(tmem_a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// 16 consecutive 32-bit TMEM columns of this thread's lane (warp-collective:
// lanes 32 (warp % 4) .. + 31).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

// 32 lanes x 32 consecutive 32-bit columns of TMEM into 32 registers.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// ---- shared-memory layout ---------------------------------------------------------

// PAIR: two CTAs per SM: A in tensor memory, 4 stages, 4 codebook views at 64
// tokens (2 at 128) and 256 TMEM columns each, so that two fit one SM; the
// tiles run in fewer waves and each SM has two independent stage pipelines
// for the latency-bound loop (27B-class gate|up shape, 272 tiles: 75.9 ->
// 52.7 us at 64 tokens, 87.0 -> 62.3 us at 128; at 64 tokens 4 stages with 4
// views measured 6% faster than 6 stages with 2).  The host takes it for 64-
// and 128-token tiles when there are at least as many tiles as SMs, and at 64
// tokens also for split-k shapes whose splits (sized for two CTAs per SM)
// keep at least 5 blocks each (27B-class down projection 46.8 -> 38.2 us);
// shorter splits are faster in the single-CTA form.  At 256-token tiles two
// CTAs do not fit (their accumulators alone take all of TMEM).
template <int BN, bool PAIR = false>
struct UmmaSmem {
  static_assert(!PAIR || BN <= 128, "two CTAs per SM at 64- and 128-token tiles only");
  // A in tensor memory at 64 and 256 tokens and in PAIR (see the file header)
  static constexpr bool TMEM_A = PAIR || BN != 128;
  // stages: 12 at 64 tokens, 4 above and in PAIR; the codebook as 4 views
  // (64 KB), 2 in PAIR at 128 tokens (4 stages of 18 KB leave no room for more)
  static constexpr int STAGES = PAIR ? 4 : (BN == 64 ? 12 : 4);
  static constexpr int LV = (PAIR && BN == 128) ? 1 : 2;
  // TMEM columns: the fp32 accumulator [0, BN), then (TMEM_A) 32 per stage
  static constexpr uint32_t A_COL0 = BN;
  static constexpr uint32_t TMEM_COLS = PAIR ? 256 : (TMEM_A ? 512 : BN);
  static constexpr uint32_t A_BYTES = TMEM_A ? 0 : UM_BM * 128;  // 16 KB per stage in shared memory
  static constexpr uint32_t B_BYTES = BN * 128;        // BN rows of 64 fp16
  static constexpr uint32_t C_BYTES = UM_BM * 16;      // 16 code bytes per row
  static constexpr uint32_t A_OFF = 0;
  static constexpr uint32_t B_OFF = A_OFF + STAGES * A_BYTES;
  static constexpr uint32_t C_OFF = B_OFF + STAGES * B_BYTES;
  static constexpr uint32_t CB_OFF = C_OFF + STAGES * C_BYTES;
  static constexpr uint32_t BAR_OFF = CB_OFF + (16384u << LV);  // full[S], decoded[S], empty[S], accum
  static constexpr uint32_t MISC_OFF = BAR_OFF + (3 * STAGES + 1) * 8;
  static constexpr uint32_t BYTES = MISC_OFF + 64;
  static constexpr uint32_t ALLOC = BYTES + 1024;  // slack to align the base to 1024
  static_assert(ALLOC <= (PAIR ? 113 : 227) * 1024, "shared memory per block");
  static_assert(!TMEM_A || A_COL0 + 32 * STAGES <= TMEM_COLS, "tensor memory columns");
};

template <int BN, bool PAIR = false>
__global__ void __launch_bounds__(UM_THREADS, PAIR ? 2 : 1) umma_kernel(const __grid_constant__ UmmaParams p) {
  using L = UmmaSmem<BN, PAIR>;
  const int splits = p.splits;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sm = smem_raw + (base - raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // tile coordinates
  const int tile = blockIdx.x / splits, split = blockIdx.x - tile * splits;
  const int rt = tile / p.tok_tiles, tt = tile - rt * p.tok_tiles;
  const int row0 = rt * UM_BM, tok0 = tt * BN;
  int seg = 0;
  if (p.nseg > 1 && row0 >= p.seg_row0[1]) seg = 1;
  if (p.nseg > 2 && row0 >= p.seg_row0[2]) seg = 2;
  const int seg_row = row0 - p.seg_row0[seg];
  const int blocks = p.k / 256;
  const int b_lo = (int)((int64_t)split * blocks / splits);
  const int b_hi = (int)((int64_t)(split + 1) * blocks / splits);
  const int it0 = b_lo * 4, it1 = b_hi * 4;  // 64-wide k steps of this split
  const int niters = it1 - it0;

  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::MISC_OFF + 8);
  int* bcast = reinterpret_cast<int*>(sm + L::MISC_OFF + 16);
  constexpr int ST = L::STAGES;
  const uint32_t bar_full = base + L::BAR_OFF, bar_dec = bar_full + 8 * ST, bar_empty = bar_dec + 8 * ST,
                 bar_acc = bar_empty + 8 * ST;

  pdl_launch_dependents();
  if (tid == 0) {
    *abort_flag = 0;
    for (int s = 0; s < ST; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_dec + 8 * s, UM_DEC_THREADS + ((int)blockIdx.x == p.skip_arrive_cta ? 1 : 0));
      mbar_init(bar_empty + 8 * s, 1);
    }
    mbar_init(bar_acc, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  // codebook into shared memory as 2^LV interleaved views (entry e of view v
  // at byte 8(e 2^LV + v)): decoder lane l reads view l % 2^LV, so with 4
  // views the four lanes of a half-warp that share a view spread over four
  // bank pairs (with one copy, 32 random 8-byte gathers cost ~7.7
  // shared-memory wavefronts)
  for (int e = tid; e < 2048; e += UM_THREADS) {
    const uint2 ent = reinterpret_cast<const uint2*>(p.codebook)[e];
    uint8_t* dst = sm + L::CB_OFF + (e << (3 + L::LV));
    if (L::LV == 0) {
      *reinterpret_cast<uint2*>(dst) = ent;
    } else {
#pragma unroll
      for (int v = 0; v < (1 << L::LV); v += 2)
        *reinterpret_cast<uint4*>(dst + 8 * v) = make_uint4(ent.x, ent.y, ent.x, ent.y);
    }
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_slot)),
                 "r"(L::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  pdl_wait();  // x' is written by the preceding kernel

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const uint32_t tx = L::B_BYTES + L::C_BYTES;
      int issued = 0;
      for (int i = 0; i < niters; ++i) {
        const int s = i % ST, r = i / ST;
        if (r > 0 && !mbar_wait(bar_empty + 8 * s, (r - 1) & 1, p.spin_limit)) {
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        mbar_expect_tx(bar_full + 8 * s, tx);
        const int kk = it0 + i;
        tma_load_2d(base + L::B_OFF + s * L::B_BYTES, &p.tmap_x, bar_full + 8 * s, kk * UM_BK, tok0);
        tma_load_2d(base + L::C_OFF + s * L::C_BYTES, &p.tmap_codes[seg], bar_full + 8 * s, kk * 16, seg_row);
        issued = i + 1;
      }
      if (*abort_flag) {
        // the copies still in flight belong to the last (up to) ST issued
        // stages: let them land before the CTA leaves
        for (int i = issued - ST < 0 ? 0 : issued - ST; i < issued; ++i)
          (void)mbar_wait(bar_full + 8 * (i % ST), (i / ST) & 1, p.spin_limit);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = umma_idesc(BN);
      for (int i = 0; i < niters; ++i) {
        const int s = i % ST, r = i / ST;
        if (*abort_flag || !mbar_wait(bar_dec + 8 * s, r & 1, p.spin_limit)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t b0 = base + L::B_OFF + s * L::B_BYTES;
        if (L::TMEM_A) {
          const uint32_t a0 = tmem + L::A_COL0 + s * 32;
#pragma unroll
          for (int k16 = 0; k16 < UM_BK / 16; ++k16)
            umma_f16_tmem_a(tmem, a0 + k16 * 8, umma_smem_desc(b0 + k16 * 32), idesc, (i > 0 || k16 > 0) ? 1u : 0u);
        } else {
          const uint32_t a0 = base + L::A_OFF + s * L::A_BYTES;
#pragma unroll
          for (int k16 = 0; k16 < UM_BK / 16; ++k16)
            umma_f16(tmem, umma_smem_desc(a0 + k16 * 32), umma_smem_desc(b0 + k16 * 32), idesc,
                     (i > 0 || k16 > 0) ? 1u : 0u);
        }
        umma_commit(bar_empty + 8 * s);
      }
      umma_commit(bar_acc);  // arrives once every MMA issued above has completed
    }
  } else if (warp >= 4) {
    // ---------------- decoders ----------------
    const int dt = tid - 128;
    const int r = dt & (UM_BM - 1);  // row of the tile
    const int h = dt >> 7;           // codes 8h .. 8h+7 of each 16-code chunk
    // (TMEM_A) this thread's TMEM lane (row r: warps 4-7 and 8-11 hold rows
    // 32 (warp % 4) ..) and its 16 columns (codes 8h .. 8h+7) of a stage
    const uint32_t a_thr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + L::A_COL0 + 16 * h;
    const int grow = min(row0 + r, p.n_total - 1);
    const uint16_t* srow = p.scales[seg] + (size_t)(grow - p.seg_row0[seg]) * blocks;
    const uint8_t* cbs = sm + L::CB_OFF + ((lane & ((1 << L::LV) - 1)) << 3);
    uint32_t carry = 0;  // last code of this row in the previous k step
    uint32_t sc_next = __ldg(srow + b_lo);
    uint32_t sc2 = 0;
    for (int i = 0; i < niters; ++i) {
      const int s = i % ST, rr = i / ST;
      if ((i & 3) == 0) {  // block start: state resets, scale of this block
        carry = 0;
        sc2 = sc_next | (sc_next << 16);
        const int bn = b_lo + (i >> 2) + 1;
        if (bn < b_hi) sc_next = __ldg(srow + bn);
      }
      // the stop decision is warp-uniform: the warp-collective ops below need every lane
      if (!__all_sync(0xffffffffu, !*abort_flag && mbar_wait(bar_full + 8 * s, rr & 1, p.spin_limit))) {
        *abort_flag = 1;
        break;
      }
      const uint4 cw = *reinterpret_cast<const uint4*>(sm + L::C_OFF + s * L::C_BYTES + r * 16);
      const uint32_t w0 = h ? cw.z : cw.x, w1 = h ? cw.w : cw.y;
      uint32_t prev = h ? (cw.y >> 24) : carry;
      carry = cw.w >> 24;
      uint32_t out[16];  // 4-byte words 2j, 2j + 1: weights (0, 1), (2, 3) of code 8h + j
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t code = ((j < 4 ? w0 : w1) >> (8 * (j & 3))) & 0xFFu;
        const uint32_t e = ((prev & 7u) << 8) | code;
        const uint2 ent = *reinterpret_cast<const uint2*>(cbs + (e << (3 + L::LV)));
        out[2 * j] = hmul2_u32(ent.x, sc2);
        out[2 * j + 1] = hmul2_u32(ent.y, sc2);
        prev = code;
      }
      if (L::TMEM_A) {
        tc_fence_after();  // the stage's previous MMAs (released through bar_full's producer wait) are done
        tmem_st16(a_thr + s * 32, out);
        tmem_wait_st();
        tc_fence_before();
      } else {
        uint8_t* arow = sm + L::A_OFF + s * L::A_BYTES + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c)  // 16-byte chunk 4h + c = codes 8h+2c, 8h+2c+1
          *reinterpret_cast<uint4*>(arow + (((4 * h + c) ^ (r & 7)) << 4)) =
              make_uint4(out[4 * c], out[4 * c + 1], out[4 * c + 2], out[4 * c + 3]);
        fence_async_smem();
      }
      mbar_arrive(bar_dec + 8 * s);
    }
  }

  // ---------------- epilogue (warps 4-11; TMEM lanes 32*(warp%4) ..) ----------------
  if (warp >= 4) {
    const int wq = warp & 3;
    const int half = (warp - 4) >> 2;  // column half
    // always wait for the MMAs issued so far (TMEM is freed below), read only
    // when nothing timed out
    const bool done = mbar_wait(bar_acc, 0, p.spin_limit);
    const bool ok = __all_sync(0xffffffffu, done && !*abort_flag);  // tcgen05.ld is warp-collective
    if (!ok) *abort_flag = 1;
    tc_fence_after();
    const int n = row0 + wq * 32 + lane;
    float* part = p.partials + ((size_t)tile * splits + split) * (size_t)(BN * UM_BM);
    for (int c0 = half * (BN / 2); c0 < (half + 1) * (BN / 2); c0 += 32) {
      float v[32];
      if (ok) {
        tmem_ld32(tmem + ((uint32_t)(wq * 32) << 16) + c0, v);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0.f;
      }
      if (splits == 1) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int tok = tok0 + c0 + j;
          if (tok < p.m && n < p.n_total) {
            if (p.y) p.y[(size_t)tok * p.n_total + n] = v[j];
            if (n < p.handoff_rows) p.handoff[(size_t)tok * p.handoff_rows + n] = f_to_bf16_bits(p.alpha * v[j]);
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) part[(size_t)(c0 + j) * UM_BM + wq * 32 + lane] = v[j];
      }
    }
    if (splits > 1) {
      // the last split of this tile to finish sums all of them in split order,
      // 4 rows per float4, every epilogue thread in parallel
      __threadfence();
      asm volatile("bar.sync 1, 256;\n" ::: "memory");
      if (tid == 128) bcast[0] = atomicAdd(p.counters + tile, 1);
      asm volatile("bar.sync 1, 256;\n" ::: "memory");
      if (bcast[0] == splits - 1) {
        __threadfence();
        const float4* tp = reinterpret_cast<const float4*>(p.partials + (size_t)tile * splits * (size_t)(BN * UM_BM));
        constexpr int Q = BN * UM_BM / 4;  // float4s per split tile
        const int et = tid - 128;
        for (int i0 = et; i0 < Q; i0 += 4 * UM_DEC_THREADS) {
          float4 acc[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          // the loads of up to UM_SPLIT_BATCH splits are all in flight before
          // the first add (the sum is latency-bound otherwise)
          constexpr int SB = PAIR ? 2 : UM_SPLIT_BATCH;  // fewer in flight in PAIR (register budget)
          for (int sp0 = 0; sp0 < splits; sp0 += SB) {
            float4 v4[SB][4];
#pragma unroll
            for (int b = 0; b < SB; ++b)
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * UM_DEC_THREADS;
                v4[b][u] = (i < Q && sp0 + b < splits) ? __ldcg(tp + (size_t)(sp0 + b) * Q + i)
                                                         : make_float4(0.f, 0.f, 0.f, 0.f);
              }
#pragma unroll
            for (int b = 0; b < SB; ++b)
              if (sp0 + b < splits)
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  acc[u].x += v4[b][u].x;
                  acc[u].y += v4[b][u].y;
                  acc[u].z += v4[b][u].z;
                  acc[u].w += v4[b][u].w;
                }
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * UM_DEC_THREADS;
            if (i >= Q) continue;
            const int tok = tok0 + i / (UM_BM / 4);
            const int nb = row0 + (i % (UM_BM / 4)) * 4;
            const float vv[4] = {acc[u].x, acc[u].y, acc[u].z, acc[u].w};
            if (tok < p.m) {
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int nn = nb + e;
                if (nn < p.n_total) {
                  if (p.y) p.y[(size_t)tok * p.n_total + nn] = vv[e];
                  if (nn < p.handoff_rows)
                    p.handoff[(size_t)tok * p.handoff_rows + nn] = f_to_bf16_bits(p.alpha * vv[e]);
                }
              }
            }
          }
        }
        if (tid == 128) p.counters[tile] = 0;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  // after the barrier: every role has set the flag by now if its wait ran out
  // (a producer with no more k steps than stages never waits, and would
  // otherwise read the flag before the MMA thread sets it)
  if (*abort_flag && tid == 0 && p.status) atomicExch(p.status, UM_TIMEOUT_STATUS);
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(L::TMEM_COLS));
  }
}

}  // namespace tq
