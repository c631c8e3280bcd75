// tq_api.cu -- the C ABI of libtq (see include/tq.h): argument checks, kernel
// selection and launches.  No allocation, no synchronisation.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "../../include/tq.h"
#include "tq_common.cuh"
#include "tq_decode.cuh"
#include "tq_dmma.cuh"
#include "tq_encode.cuh"
#include "tq_rht.cuh"
#include "tq_stack1.cuh"
#include "tq_stackn.cuh"
#include "tq_umma.cuh"

#include <cudaTypedefs.h>

namespace {

thread_local int g_last_cuda_error = 0;

int cuda_fail(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return TQ_ERR_CUDA;
}

#define TQ_CUDA(call)                           \
  do {                                          \
    cudaError_t e_ = (call);                    \
    if (e_ != cudaSuccess) return cuda_fail(e_); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kMaxDevices = 64;
int g_arch_ok[kMaxDevices];  // 0 unknown, 1 ok, 2 bad
int g_num_sms[kMaxDevices];

// Current device must be compute capability 10.0 (B200, sm_100a).
int check_arch(int* num_sms) {
  int dev = 0;
  TQ_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return TQ_ERR_ARCH;
  if (g_arch_ok[dev] == 0) {
    int major = 0, minor = 0, sms = 0;
    TQ_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    TQ_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
    TQ_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    g_num_sms[dev] = sms;
    g_arch_ok[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  if (g_arch_ok[dev] != 1) return TQ_ERR_ARCH;
  if (num_sms) *num_sms = g_num_sms[dev];
  return TQ_OK;
}

bool k_ok(int32_t k) { return k > 0 && k % 512 == 0; }

int check_weight(const tq_weight_t* w) {
  if (!w) return TQ_ERR_NULL;
  if (w->n < 1 || !k_ok(w->k)) return TQ_ERR_SHAPE;
  if (!w->codes_d || !w->scales_d || !w->codebook_d) return TQ_ERR_NULL;
  if (!aligned16(w->codes_d) || !aligned16(w->codebook_d)) return TQ_ERR_ALIGN;
  if (reinterpret_cast<uintptr_t>(w->scales_d) & 3) return TQ_ERR_ALIGN;  // read two blocks' scales at a time
  return TQ_OK;
}

// Launch with the programmatic-stream-serialization attribute so that a
// kernel may start its weight prefetch while the previous one finishes.
template <typename... KArgs, typename... Args>
int launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
#ifdef TQ_NO_PDL
  cfg.numAttrs = 0;  // build option: plain stream ordering
#else
  cfg.numAttrs = 1;
#endif
  TQ_CUDA(cudaLaunchKernelEx(&cfg, kernel, args...));
  return TQ_OK;
}

// ---- decode-MMA configuration ------------------------------------------------

using tq::DmmaParams;

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Columns of one partial-sum tile: 1 at batch 1 (hi+lo summed), else 8 * NT.
int dmma_nt_for(int32_t m) {
  if (m <= 8) return 1;
  if (m <= 16) return 2;
  return 4;
}
constexpr int kDmmaMaxM = 32;  // one dmma launch covers up to 32 tokens (4 column tiles)

struct DmmaWs {
  size_t counters_off, partials_off, bytes;
};

// Every workspace starts with a fixed region of per-tile arrival counters
// (kCounterBytes, so every call, whatever its shape, finds its counters in
// the same zeroed bytes; each call leaves them zero).  Everything after it
// (partial sums, activation scratch) is written before it is read.
constexpr size_t kCounterBytes = 64 * 1024;
constexpr int64_t kMaxTiles = kCounterBytes / 4 - 1;  // the last slot holds the status word

DmmaWs dmma_ws_layout(int64_t n_total, int32_t k, int mc) {
  const int64_t tiles = (n_total + 15) / 16;
  const int64_t units = tiles * (k / 256);
  const int64_t warps = units < tq::DMMA_MAX_WARPS ? units : tq::DMMA_MAX_WARPS;
  DmmaWs w;
  w.counters_off = 0;
  w.partials_off = kCounterBytes;
  w.bytes = w.partials_off + (size_t)warps * 2 * 16 * mc * sizeof(float);
  return w;
}

// views: pick the largest replication that fits next to the activations.
int dmma_lv_for(bool hilo, int32_t k) {
  const size_t xs = hilo ? (size_t)k * 4 : 0;
  const size_t limit = 227 * 1024;
  for (int lv = 3; lv > 0; --lv)
    if ((16384u << lv) + xs <= limit) return lv;
  return 0;
}

// Largest k of the batch-1 kernel: its 4 bytes of hi/lo activations per
// feature sit in shared memory beside one 16 KB codebook copy (227 KB per
// block), rounded down to a multiple of 512.
constexpr int32_t kGemvMaxK = (int32_t)(((227 * 1024 - 16384) / 4) / 512 * 512);

template <int LV, int NT, bool HILO>
int dmma_launch_t(DmmaParams& p, int num_sms, cudaStream_t stream, bool dry_run) {
  auto kern = tq::dmma_kernel<LV, NT, HILO>;
  const size_t smem = (16384u << LV) + (HILO ? (size_t)p.k * 4 : 0);
  if (smem > 227 * 1024) return TQ_ERR_SHAPE;
  // per instantiation and device: opt in to large shared memory once and
  // remember the occupancy for each shared-memory size (in KB) seen
  static int occ_cache[kMaxDevices][228];
  int dev = 0;
  TQ_CUDA(cudaGetDevice(&dev));
  const int cls = (int)((smem + 1023) >> 10);
  int occ = occ_cache[dev][cls];
  if (occ == 0) {
    TQ_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024));
    TQ_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, tq::DMMA_THREADS, cls << 10));
    if (occ < 1) return TQ_ERR_SHAPE;
    occ_cache[dev][cls] = occ;
  }
  if (dry_run) return TQ_OK;
  int64_t grid = (int64_t)num_sms * occ;
  const int64_t need = (p.units + tq::DMMA_WARPS - 1) / tq::DMMA_WARPS;
  if (grid > need) grid = need;
  if (grid * tq::DMMA_WARPS > tq::DMMA_MAX_WARPS) grid = tq::DMMA_MAX_WARPS / tq::DMMA_WARPS;
  int64_t aw = grid * tq::DMMA_WARPS;
  if (aw > p.units) aw = p.units;
  p.active_warps = (int32_t)aw;
  return launch(kern, dim3((unsigned)grid), dim3(tq::DMMA_THREADS), smem, stream, p);
}

// Units per warp from which the two-row-tile kernel is used (measured at 32
// tokens: 5.1 and more faster, e.g. 34816 x 5120 58 vs 68 us; 4.3 even;
// 2.6 and fewer slower, e.g. 4096 x 4096 25 vs 21 us).
constexpr int kDmma2MinUnits = 5;

// The two-row-tile kernel (17-32 tokens): 32-row tiles, 8 warps per CTA.
// Its partial sums take 32 x MC floats per warp and slot; the active warps
// are capped at half the 16-row unit count so they fit the workspace that
// dmma_ws_layout sizes for the 16-row kernel.
template <int LV, int NT>
int dmma2_launch_t(DmmaParams& p, int num_sms, cudaStream_t stream, bool dry_run) {
  auto kern = tq::dmma_kernel_r2<LV, NT>;
  const size_t smem = 16384u << LV;
  static int occ_cache[kMaxDevices];
  int dev = 0;
  TQ_CUDA(cudaGetDevice(&dev));
  int occ = occ_cache[dev];
  if (occ == 0) {
    TQ_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    TQ_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, tq::DMMA2_THREADS, smem));
    if (occ < 1) return TQ_ERR_SHAPE;
    occ_cache[dev] = occ;
  }
  if (dry_run) return TQ_OK;
  const int64_t units16 = p.units;  // 16-row units (the workspace layout's count)
  p.tiles = (p.n_total + 31) / 32;
  p.units = (int64_t)p.tiles * p.blocks;
  int64_t aw = (int64_t)num_sms * occ * tq::DMMA2_WARPS;
  if (aw > p.units) aw = p.units;
  if (aw > units16 / 2) aw = units16 / 2 > 0 ? units16 / 2 : 1;
  p.active_warps = (int32_t)aw;
  const int64_t grid = (aw + tq::DMMA2_WARPS - 1) / tq::DMMA2_WARPS;
  return launch(kern, dim3((unsigned)grid), dim3(tq::DMMA2_THREADS), smem, stream, p);
}

template <int NT, bool HILO>
int dmma_launch_lv(DmmaParams& p, int lv, int num_sms, cudaStream_t stream, bool dry_run) {
  switch (lv) {
    case 3: return dmma_launch_t<3, NT, HILO>(p, num_sms, stream, dry_run);
    case 2: return dmma_launch_t<2, NT, HILO>(p, num_sms, stream, dry_run);
    case 1: return dmma_launch_t<1, NT, HILO>(p, num_sms, stream, dry_run);
    default: return dmma_launch_t<0, NT, HILO>(p, num_sms, stream, dry_run);
  }
}

// Fill the shape / workspace fields of p and launch.  p.m <= 32.  With
// dry_run every check (shape, workspace, shared-memory fit, occupancy) runs
// and nothing is launched.
int dmma_run(DmmaParams& p, bool hilo, void* ws, size_t ws_bytes, int num_sms, cudaStream_t stream,
             bool dry_run = false) {
  const int nt = hilo ? 1 : dmma_nt_for(p.m);
  const int mc = hilo ? 1 : nt * 8;
  if (hilo && p.k > kGemvMaxK) return TQ_ERR_SHAPE;
  const DmmaWs L = dmma_ws_layout(p.n_total, p.k, mc);
  if (!ws) return TQ_ERR_WORKSPACE;
  if (ws_bytes < L.bytes) return TQ_ERR_WORKSPACE;
  if (!aligned16(ws)) return TQ_ERR_ALIGN;
  p.tiles = (p.n_total + 15) / 16;
  if (p.tiles > kMaxTiles) return TQ_ERR_SHAPE;
  p.blocks = p.k / 256;
  p.units = (int64_t)p.tiles * p.blocks;
  p.counters = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + L.counters_off);
  p.partials = reinterpret_cast<float*>(static_cast<char*>(ws) + L.partials_off);
  const int lv = dmma_lv_for(hilo, p.k);
  if (hilo) return dmma_launch_lv<1, true>(p, lv, num_sms, stream, dry_run);
  switch (nt) {
    case 1: return dmma_launch_lv<1, false>(p, lv, num_sms, stream, dry_run);
    case 2: return dmma_launch_lv<2, false>(p, lv, num_sms, stream, dry_run);
    default:
      // 17-32 tokens: two 16-row tiles per warp (x' loaded once for both)
      // where that gives each of its warps at least kDmma2MinUnits 32-row
      // units; on smaller shapes (few units per warp, most tiles split across
      // warps) 16 warps of one row tile measured faster
      if ((int64_t)((p.n_total + 31) / 32) * p.blocks < (int64_t)kDmma2MinUnits * num_sms * tq::DMMA2_WARPS)
        return dmma_launch_lv<4, false>(p, lv, num_sms, stream, dry_run);
      switch (lv) {
        case 3: return dmma2_launch_t<3, 4>(p, num_sms, stream, dry_run);
        case 2: return dmma2_launch_t<2, 4>(p, num_sms, stream, dry_run);
        case 1: return dmma2_launch_t<1, 4>(p, num_sms, stream, dry_run);
        default: return dmma2_launch_t<0, 4>(p, num_sms, stream, dry_run);
      }
  }
}

void dmma_single(DmmaParams& p, const tq_weight_t* w) {
  memset(&p, 0, sizeof(p));
  p.seg[0].codes = w->codes_d;
  p.seg[0].scales = w->scales_d;
  p.seg[0].rows = w->n;
  p.seg[0].row0 = 0;
  p.nseg = 1;
  p.codebook = w->codebook_d;
  p.n_total = w->n;
  p.k = w->k;
}

// ---- tcgen05 GEMM configuration -------------------------------------------------

constexpr int kUmmaMinM = 33;  // from this many tokens on the decoded GEMM uses tcgen05 (measured crossover)
constexpr int kSplitTarget = 148;    // split k until about one CTA per SM (B200 SM count; two in PAIR)
constexpr int kStatusOff = (int)kCounterBytes - 4;  // error word: last 4 bytes of the counter region
static_assert(kStatusOff == TQ_STATUS_OFFSET, "the status word offset is part of the interface");

PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;

int get_encode_tiled() {
  if (g_encode_tiled) return TQ_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  TQ_CUDA(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
  if (q != cudaDriverEntryPointSuccess || !fn) return cuda_fail(cudaErrorNotSupported);
  g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return TQ_OK;
}

int umma_bn_for(int32_t m) { return m <= 64 ? 64 : (m <= 128 ? 128 : 256); }

// Least 256-weight blocks per split for the two-CTA form of a split 64-token
// tile (measured: 9.7 and 5 blocks faster, e.g. 5120 x 17408 46.8 -> 38.2 us;
// 3.4 and 2.7 slower).
constexpr int kPairMinBlocks = 5;

struct UmmaShape {
  int bn, row_tiles, tok_tiles, splits;
  bool pair;  // two CTAs per SM (tq::UmmaSmem)
  size_t partial_bytes;
};

UmmaShape umma_shape(int64_t n_total, int32_t k, int32_t m) {
  UmmaShape u;
  u.bn = umma_bn_for(m);
  u.row_tiles = (int)((n_total + tq::UM_BM - 1) / tq::UM_BM);
  u.tok_tiles = (m + u.bn - 1) / u.bn;
  const int tiles = u.row_tiles * u.tok_tiles;
  const int blocks = k / 256;
  int sp = kSplitTarget / tiles;
  if (sp < 1) sp = 1;
  if (sp > blocks) sp = blocks;
  u.pair = u.bn <= 128 && tiles >= kSplitTarget;  // sp == 1 there
  if (u.bn == 64 && tiles < kSplitTarget) {
    // two CTAs per SM with splits sized for both, where each keeps at least
    // kPairMinBlocks blocks (shorter splits measured faster one per SM)
    int sp2 = 2 * kSplitTarget / tiles;
    if (sp2 > blocks) sp2 = blocks;
    if (blocks >= kPairMinBlocks * sp2) {
      u.pair = true;
      sp = sp2;
    }
  }
  u.splits = sp;
  u.partial_bytes = sp > 1 ? (size_t)tiles * sp * u.bn * tq::UM_BM * sizeof(float) : 0;
  return u;
}

size_t umma_ws_bytes(int64_t n_total, int32_t k, int32_t m) {
  return kCounterBytes + umma_shape(n_total, k, m).partial_bytes;
}

// Segments must start on 128-row boundaries for the tile -> segment lookup.
bool umma_ok(int32_t m, const int32_t* rows, int nseg) {
  if (m < kUmmaMinM) return false;
  for (int i = 0; i + 1 < nseg; ++i)
    if (rows[i] % tq::UM_BM != 0) return false;
  return true;
}

int encode_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* ptr, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_in, uint32_t box_out, CUtensorMapSwizzle sw) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_in, box_out};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode_tiled(map, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return TQ_OK;
}

template <int BN, bool PAIR = false>
int umma_launch_t(tq::UmmaParams& p, int grid, cudaStream_t stream) {
  auto kern = tq::umma_kernel<BN, PAIR>;
  const size_t smem = tq::UmmaSmem<BN, PAIR>::ALLOC;
  static int configured[kMaxDevices];
  int dev = 0;
  TQ_CUDA(cudaGetDevice(&dev));
  if (!configured[dev]) {
    TQ_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    configured[dev] = 1;
  }
  return launch(kern, dim3((unsigned)grid), dim3(tq::UM_THREADS), smem, stream, p);
}

// y (and handoff) for m tokens of a weight made of `nseg` row segments sharing
// k and the codebook.  x_f16: device fp16 [m][k].
int umma_run(const uint8_t* const* codes, const uint16_t* const* scales, const int32_t* rows, int nseg,
             const uint16_t* codebook, int32_t k, int32_t m, const uint16_t* x_f16, float* y, uint16_t* handoff,
             float alpha, void* ws, size_t ws_bytes, cudaStream_t stream, const tq_stack_options_t* opt = nullptr) {
  if (opt && opt->test_skip_arrive < -1) return TQ_ERR_VALUE;
  int st = get_encode_tiled();
  if (st != TQ_OK) return st;
  int64_t n_total = 0;
  for (int i = 0; i < nseg; ++i) n_total += rows[i];
  const UmmaShape u = umma_shape(n_total, k, m);
  if ((int64_t)u.row_tiles * u.tok_tiles > kMaxTiles - 1) return TQ_ERR_SHAPE;
  if (ws_bytes < kCounterBytes + u.partial_bytes) return TQ_ERR_WORKSPACE;
  tq::UmmaParams p;
  memset(&p, 0, sizeof(p));
  st = encode_2d(&p.tmap_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x_f16, (uint64_t)k, (uint64_t)m, (uint64_t)k * 2,
                 tq::UM_BK, (uint32_t)u.bn, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != TQ_OK) return st;
  int32_t row0 = 0;
  for (int i = 0; i < nseg; ++i) {
    st = encode_2d(&p.tmap_codes[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, codes[i], (uint64_t)k / 4, (uint64_t)rows[i],
                   (uint64_t)k / 4, 16, tq::UM_BM, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != TQ_OK) return st;
    p.scales[i] = scales[i];
    p.seg_row0[i] = row0;
    p.seg_rows[i] = rows[i];
    row0 += rows[i];
  }
  p.nseg = nseg;
  p.codebook = codebook;
  p.n_total = (int32_t)n_total;
  p.k = k;
  p.m = m;
  p.y = y;
  p.handoff = handoff;
  p.handoff_rows = handoff ? rows[0] : 0;
  p.alpha = alpha;
  p.counters = static_cast<int32_t*>(ws);
  p.status = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + kStatusOff);
  p.partials = reinterpret_cast<float*>(static_cast<char*>(ws) + kCounterBytes);
  p.row_tiles = u.row_tiles;
  p.tok_tiles = u.tok_tiles;
  p.splits = u.splits;
  p.spin_limit = (opt && opt->spin_limit) ? opt->spin_limit : 1u << 21;  // try_wait polls; far above any healthy wait
  p.skip_arrive_cta = opt ? opt->test_skip_arrive : -1;
  const int grid = u.row_tiles * u.tok_tiles * u.splits;
  switch (u.bn) {
    case 64: return u.pair ? umma_launch_t<64, true>(p, grid, stream) : umma_launch_t<64>(p, grid, stream);
    case 128: return u.pair ? umma_launch_t<128, true>(p, grid, stream) : umma_launch_t<128>(p, grid, stream);
    default: return umma_launch_t<256>(p, grid, stream);
  }
}

// ---- layer stack helpers -------------------------------------------------------

const double kScaleLo = 0.005, kScaleHi = 0.03;

float stack_alpha(int32_t k) {
  const double es2 = (kScaleHi * kScaleHi * kScaleHi - kScaleLo * kScaleLo * kScaleLo) / (3.0 * (kScaleHi - kScaleLo));
  return (float)(1.0 / sqrt((double)k * es2));
}

// ops of phase p (first one is handed on)
int phase_ops(const tq_layer_t* L, int phase, const tq_weight_t* ops[3]) {
  switch (phase) {
    case 0: ops[0] = &L->q; ops[1] = &L->k; ops[2] = &L->v; return 3;
    case 1: ops[0] = &L->o; return 1;
    case 2: ops[0] = &L->gate; ops[1] = &L->up; return 2;
    case 3: ops[0] = &L->down; return 1;
    default: return 0;
  }
}

int phase_check(const tq_layer_t* L, int phase, int* nops, const tq_weight_t* ops[3], int64_t* n_total) {
  if (!L) return TQ_ERR_NULL;
  *nops = phase_ops(L, phase, ops);
  if (*nops == 0) return TQ_ERR_SHAPE;
  int64_t n = 0;
  for (int i = 0; i < *nops; ++i) {
    int st = check_weight(ops[i]);
    if (st != TQ_OK) return st;
    if (ops[i]->k != ops[0]->k || ops[i]->codebook_d != ops[0]->codebook_d) return TQ_ERR_SHAPE;
    n += ops[i]->n;
  }
  if (n > 0x7fffffff) return TQ_ERR_SHAPE;
  *n_total = n;
  return TQ_OK;
}

// Workspace of one phase call at m tokens:
//  [counters | partial sums (largest kernel choice)][x' fp16 [m][k] when m > 1]
size_t matmul_ws_bytes(int64_t n_total, int32_t k, int32_t m) {
  const int mc = (m <= 1) ? 1 : dmma_nt_for(m < kDmmaMaxM ? m : kDmmaMaxM) * 8;
  size_t b = dmma_ws_layout(n_total, k, mc).bytes;
  if (m >= kUmmaMinM) {
    const size_t u = umma_ws_bytes(n_total, k, m);
    if (u > b) b = u;
  }
  return round_up(b, 256);
}

// Bytes of x' for m tokens of k features: fp16, whole groups of 8 tokens
// (the small-batch kernel's fragment order, tq::xt_pos).
size_t xt_bytes(int64_t m, int64_t k) { return round_up((size_t)((m + 7) / 8 * 8) * k * 2, 256); }

size_t phase_ws_bytes(int64_t n_total, int32_t k, int32_t m) {
  size_t b = matmul_ws_bytes(n_total, k, m);
  if (m > 1) b += xt_bytes(m, k);
  return b;
}

int run_phase(const tq_layer_t* L, int phase, const uint16_t* x, int32_t m, uint64_t seed, float* y,
              uint16_t* handoff, void* ws, size_t ws_bytes, int num_sms, cudaStream_t stream) {
  int nops = 0;
  const tq_weight_t* ops[3];
  int64_t n_total = 0;
  int st = phase_check(L, phase, &nops, ops, &n_total);
  if (st != TQ_OK) return st;
  const int32_t k = ops[0]->k;
  if (ws_bytes < phase_ws_bytes(n_total, k, m)) return TQ_ERR_WORKSPACE;
  DmmaParams p;
  memset(&p, 0, sizeof(p));
  int32_t row0 = 0;
  for (int i = 0; i < nops; ++i) {
    p.seg[i].codes = ops[i]->codes_d;
    p.seg[i].scales = ops[i]->scales_d;
    p.seg[i].rows = ops[i]->n;
    p.seg[i].row0 = row0;
    row0 += ops[i]->n;
  }
  p.nseg = nops;
  p.codebook = ops[0]->codebook_d;
  p.n_total = (int32_t)n_total;
  p.k = k;
  p.y = y;
  p.handoff = handoff;
  p.handoff_rows = ops[0]->n;
  p.alpha = stack_alpha(k);
  if (m == 1) {
    p.m = 1;
    p.x_bf16 = x;
    p.rht_seed = seed;
    return dmma_run(p, true, ws, ws_bytes, num_sms, stream);
  }
  // m > 1: RHT to fp16 in the workspace tail, then the tcgen05 GEMM (m >= 33)
  // or the small-batch kernel in chunks of up to 32 tokens.
  const size_t dm_bytes = matmul_ws_bytes(n_total, k, m);
  uint16_t* xr = reinterpret_cast<uint16_t*>(static_cast<char*>(ws) + dm_bytes);
  int32_t rows[3];
  const uint8_t* cptr[3];
  const uint16_t* sptr[3];
  for (int i = 0; i < nops; ++i) {
    rows[i] = ops[i]->n;
    cptr[i] = ops[i]->codes_d;
    sptr[i] = ops[i]->scales_d;
  }
  const bool use_umma = umma_ok(m, rows, nops);
  {
    // x' fp16: row-major for the TMA of the tcgen05 GEMM, fragment order for
    // the small-batch kernel
    st = launch(use_umma ? tq::rht_kernel<1> : tq::rht_kernel<2>, tq::rht_grid(m, k), dim3(256), 0, stream, x,
                (int)m, (int)k, seed, (void*)xr);
    if (st != TQ_OK) return st;
  }
  if (use_umma)
    return umma_run(cptr, sptr, rows, nops, ops[0]->codebook_d, k, m, xr, y, handoff, p.alpha, ws, dm_bytes, stream);
  for (int32_t t0 = 0; t0 < m; t0 += kDmmaMaxM) {
    DmmaParams pc = p;
    pc.m = (m - t0) < kDmmaMaxM ? (m - t0) : kDmmaMaxM;
    pc.x_f16 = xr + (size_t)t0 * k;
    pc.y = y ? y + (size_t)t0 * n_total : nullptr;
    pc.handoff = handoff ? handoff + (size_t)t0 * ops[0]->n : nullptr;
    st = dmma_run(pc, false, ws, dm_bytes, num_sms, stream);
    if (st != TQ_OK) return st;
  }
  return TQ_OK;
}

}  // namespace

extern "C" {

int tq_pack_info(int32_t n, int32_t k, tq_pack_info_t* out) {
  if (!out) return TQ_ERR_NULL;
  if (n < 1 || !k_ok(k)) return TQ_ERR_SHAPE;
  out->n = n;
  out->k = k;
  out->group = 4;
  out->block = 256;
  out->rht_block = 512;
  out->n_states = 8;
  out->code_bytes = (int64_t)n * (k / 4);
  out->scale_bytes = (int64_t)n * (k / 256) * 2;
  out->codebook_bytes = 8 * 256 * 4 * 2;
  out->packed_bytes = out->code_bytes + out->scale_bytes;
  out->bits_per_weight = 8.0 * (double)out->packed_bytes / ((double)n * (double)k);
  return TQ_OK;
}

int tq_decode(const tq_weight_t* w, uint16_t* w_f16_d, void* stream) {
  int st = check_weight(w);
  if (st != TQ_OK) return st;
  if (!w_f16_d) return TQ_ERR_NULL;
  if (!aligned16(w_f16_d)) return TQ_ERR_ALIGN;
  int sms = 0;
  st = check_arch(&sms);
  if (st != TQ_OK) return st;
  const int64_t groups = (int64_t)w->n * (w->k / 4);
  int64_t blocks = (groups + 255) / 256;
  if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
  return launch(tq::decode_kernel, dim3((unsigned)blocks), dim3(256), 0, (cudaStream_t)stream, w->codes_d, w->scales_d,
                w->codebook_d, (int)w->n, (int)w->k, w_f16_d);
}

int tq_rht(const uint16_t* x_bf16_d, int32_t m, int32_t k, uint64_t seed, void* x_rot_d, int32_t out_dtype,
           void* stream) {
  if (m < 0 || !k_ok(k)) return TQ_ERR_SHAPE;
  if (out_dtype != TQ_F32 && out_dtype != TQ_F16) return TQ_ERR_SHAPE;
  if (m == 0) return TQ_OK;
  if (!x_bf16_d || !x_rot_d) return TQ_ERR_NULL;
  if (!aligned16(x_bf16_d) || !aligned16(x_rot_d)) return TQ_ERR_ALIGN;
  int sms = 0;
  int st = check_arch(&sms);
  if (st != TQ_OK) return st;
  if (out_dtype == TQ_F16)
    return launch(tq::rht_kernel<1>, tq::rht_grid(m, k), dim3(256), 0, (cudaStream_t)stream, x_bf16_d, (int)m,
                  (int)k, seed, x_rot_d);
  return launch(tq::rht_kernel<0>, tq::rht_grid(m, k), dim3(256), 0, (cudaStream_t)stream, x_bf16_d, (int)m,
                (int)k, seed, x_rot_d);
}

int tq_gemv_workspace(int32_t n, int32_t k, size_t* bytes) {
  if (!bytes) return TQ_ERR_NULL;
  if (n < 1 || !k_ok(k)) return TQ_ERR_SHAPE;
  *bytes = dmma_ws_layout(n, k, 1).bytes;
  return TQ_OK;
}

int tq_gemv(const tq_weight_t* w, const float* x_rot_d, float* y_d, void* workspace_d, size_t ws_bytes,
            void* stream) {
  int st = check_weight(w);
  if (st != TQ_OK) return st;
  if (w->k > kGemvMaxK) return TQ_ERR_SHAPE;
  if (!x_rot_d || !y_d) return TQ_ERR_NULL;
  if (!aligned16(x_rot_d) || !aligned16(y_d)) return TQ_ERR_ALIGN;
  int sms = 0;
  st = check_arch(&sms);
  if (st != TQ_OK) return st;
  DmmaParams p;
  dmma_single(p, w);
  p.m = 1;
  p.x_f32 = x_rot_d;
  p.y = y_d;
  return dmma_run(p, true, workspace_d, ws_bytes, sms, (cudaStream_t)stream);
}

int tq_gemm_workspace(int32_t n, int32_t k, int32_t m, size_t* bytes) {
  if (!bytes) return TQ_ERR_NULL;
  if (n < 1 || !k_ok(k) || m < 0 || m > 4096) return TQ_ERR_SHAPE;
  *bytes = matmul_ws_bytes(n, k, m < 1 ? 1 : m);
  if (m > 1 && m < kUmmaMinM) *bytes += xt_bytes(m, k);  // x' in fragment order
  return TQ_OK;
}

int tq_gemm(const tq_weight_t* w, const uint16_t* x_rot_f16_d, int32_t m, float* y_d, void* workspace_d,
            size_t ws_bytes, void* stream) {
  return tq_gemm_ex(w, x_rot_f16_d, m, y_d, workspace_d, ws_bytes, nullptr, stream);
}

int tq_gemm_ex(const tq_weight_t* w, const uint16_t* x_rot_f16_d, int32_t m, float* y_d, void* workspace_d,
               size_t ws_bytes, const tq_stack_options_t* options, void* stream) {
  if (options && options->test_skip_arrive < -1) return TQ_ERR_VALUE;
  int st = check_weight(w);
  if (st != TQ_OK) return st;
  if (m < 0 || m > 4096) return TQ_ERR_SHAPE;
  if (m == 0) return TQ_OK;
  if (!x_rot_f16_d || !y_d) return TQ_ERR_NULL;
  if (!aligned16(x_rot_f16_d) || !aligned16(y_d)) return TQ_ERR_ALIGN;
  int sms = 0;
  st = check_arch(&sms);
  if (st != TQ_OK) return st;
  if (m >= kUmmaMinM) {
    const uint8_t* c = w->codes_d;
    const uint16_t* sc = w->scales_d;
    const int32_t rows = w->n;
    return umma_run(&c, &sc, &rows, 1, w->codebook_d, w->k, m, x_rot_f16_d, y_d, nullptr, 0.f, workspace_d, ws_bytes,
                    (cudaStream_t)stream, options);
  }
  // the small-batch kernel reads x' in fragment order: permute it into the
  // workspace after the matmul scratch
  const size_t mm_bytes = matmul_ws_bytes(w->n, w->k, m);
  if (ws_bytes < mm_bytes + xt_bytes(m, w->k)) return TQ_ERR_WORKSPACE;
  uint16_t* xp = reinterpret_cast<uint16_t*>(static_cast<char*>(workspace_d) + mm_bytes);
  {
    const int64_t groups = (int64_t)m * (w->k / 4);
    int64_t blocks = (groups + 255) / 256;
    if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
    st = launch(tq::frag_permute_kernel, dim3((unsigned)blocks), dim3(256), 0, (cudaStream_t)stream, x_rot_f16_d,
                (int)m, (int)w->k, xp);
    if (st != TQ_OK) return st;
  }
  for (int32_t t0 = 0; t0 < m; t0 += kDmmaMaxM) {
    DmmaParams p;
    dmma_single(p, w);
    p.m = (m - t0) < kDmmaMaxM ? (m - t0) : kDmmaMaxM;
    p.x_f16 = xp + (size_t)t0 * w->k;
    p.y = y_d + (size_t)t0 * w->n;
    st = dmma_run(p, false, workspace_d, ws_bytes, sms, (cudaStream_t)stream);
    if (st != TQ_OK) return st;
  }
  return TQ_OK;
}

int tq_workspace_status(const void* workspace_d, int32_t* status, void* stream) {
  if (!workspace_d || !status) return TQ_ERR_NULL;
  int32_t v = 0;
  cudaStream_t s = (cudaStream_t)stream;
  TQ_CUDA(cudaMemcpyAsync(&v, static_cast<const char*>(workspace_d) + TQ_STATUS_OFFSET, sizeof(v),
                          cudaMemcpyDeviceToHost, s));
  TQ_CUDA(cudaStreamSynchronize(s));
  *status = v;
  return TQ_OK;
}

int tq_workspace_init(void* workspace_d, size_t bytes, void* stream) {
  if (bytes == 0) return TQ_OK;
  if (!workspace_d) return TQ_ERR_NULL;
  TQ_CUDA(cudaMemsetAsync(workspace_d, 0, bytes, (cudaStream_t)stream));
  return TQ_OK;
}

uint64_t tq_stack_phase_seed(uint64_t seed, int32_t layer, int32_t phase) {
  const uint64_t tag = 0x516E0000ULL | ((uint64_t)(uint32_t)layer << 2) | (uint64_t)(uint32_t)phase;
  return tq::mix64(seed ^ tq::mix64(tag));
}

int tq_layer_phase_workspace(const tq_layer_t* layer, int32_t phase, int32_t m, size_t* bytes) {
  if (!bytes) return TQ_ERR_NULL;
  if (m < 0 || m > 4096) return TQ_ERR_SHAPE;
  int nops = 0;
  const tq_weight_t* ops[3];
  int64_t n_total = 0;
  int st = phase_check(layer, phase, &nops, ops, &n_total);
  if (st != TQ_OK) return st;
  *bytes = phase_ws_bytes(n_total, ops[0]->k, m < 1 ? 1 : m);
  return TQ_OK;
}

int tq_layer_phase(const tq_layer_t* layer, int32_t phase, const uint16_t* x_bf16_d, int32_t m, uint64_t phase_seed,
                   float* y_d, uint16_t* handoff_bf16_d, void* workspace_d, size_t ws_bytes, void* stream) {
  if (m < 0 || m > 4096) return TQ_ERR_SHAPE;
  int nops = 0;
  const tq_weight_t* ops[3];
  int64_t n_total = 0;
  int st = phase_check(layer, phase, &nops, ops, &n_total);
  if (st != TQ_OK) return st;
  if (m == 0) return TQ_OK;
  if (!x_bf16_d || !handoff_bf16_d || !workspace_d) return TQ_ERR_NULL;
  if (!aligned16(x_bf16_d) || (y_d && !aligned16(y_d)) || !aligned16(workspace_d)) return TQ_ERR_ALIGN;
  int sms = 0;
  st = check_arch(&sms);
  if (st != TQ_OK) return st;
  return run_phase(layer, phase, x_bf16_d, m, phase_seed, y_d, handoff_bf16_d, workspace_d, ws_bytes, sms,
                   (cudaStream_t)stream);
}

// Stack workspace: [phase workspace][y fp32 [m][max n]][a bf16 [m][q]]
// [b bf16 [m][hidden]][c bf16 [m][inter]][h bf16 [m][hidden]][RHT sign bits]
// [per-phase parameter table (batch-1 persistent kernel)][barrier word]
constexpr int kStackMaxCtas = 256;  // bound on the persistent stack kernel's grid

constexpr int kStackMaxM = 16;  // the persistent stack kernels run batches of 1 .. 16 tokens

struct StackWs {
  size_t phase, y, a, b, c, h, signs, params, xq, sync, total;
  uint32_t sign_words;
};

static int stack_layout(const tq_layer_t* layers, int32_t n_layers, int32_t m, StackWs* L) {
  if (!layers) return TQ_ERR_NULL;
  if (n_layers < 1 || m < 1 || m > 4096) return TQ_ERR_SHAPE;
  size_t phase = 0;
  int64_t ymax = 0, amax = 0, bmax = 0, cmax = 0, hmax = 0;
  for (int l = 0; l < n_layers; ++l) {
    for (int p = 0; p < 4; ++p) {
      int nops = 0;
      const tq_weight_t* ops[3];
      int64_t n_total = 0;
      int st = phase_check(&layers[l], p, &nops, ops, &n_total);
      if (st != TQ_OK) return st;
      size_t b = phase_ws_bytes(n_total, ops[0]->k, m);
      if (b > phase) phase = b;
      if (n_total > ymax) ymax = n_total;
    }
    const tq_layer_t& L0 = layers[l];
    // the chain of shapes: h -> q|k|v (k = hidden) -> o (k = q.n) -> gate|up (k = o.n) -> down (k = gate.n)
    if (L0.o.k != L0.q.n || L0.gate.k != L0.o.n || L0.down.k != L0.gate.n || L0.down.n != L0.q.k)
      return TQ_ERR_SHAPE;
    if (l > 0 && L0.q.k != layers[l - 1].down.n) return TQ_ERR_SHAPE;
    if (L0.q.n > amax) amax = L0.q.n;
    if (L0.o.n > bmax) bmax = L0.o.n;
    if (L0.gate.n > cmax) cmax = L0.gate.n;
    if (L0.down.n > hmax) hmax = L0.down.n;
  }
  // at batch 1 the persistent stack kernel keeps two partial-sum slots for
  // every warp it may run (at most DMMA_MAX_WARPS)
  if (m == 1) {
    const size_t pk = kCounterBytes + (size_t)tq::DMMA_MAX_WARPS * 2 * 16 * sizeof(float);
    if (phase < pk) phase = pk;
  } else if (m <= kStackMaxM) {
    // the small-batch persistent kernel: three phases of CTA partials (two
    // tiles of 16 rows x 16 tokens per CTA)
    const size_t pk = kCounterBytes + (size_t)3 * kStackMaxCtas * 2 * 16 * 16 * sizeof(float);
    if (phase < pk) phase = pk;
  }
  int64_t kmax = 0;
  for (int l = 0; l < n_layers; ++l) {
    const int64_t ks[4] = {layers[l].q.k, layers[l].o.k, layers[l].gate.k, layers[l].down.k};
    for (int p = 0; p < 4; ++p) kmax = ks[p] > kmax ? ks[p] : kmax;
  }
  uint64_t words = 0;
  for (int l = 0; l < n_layers; ++l)
    words += ((uint64_t)layers[l].q.k + layers[l].o.k + layers[l].gate.k + layers[l].down.k) / 32;
  L->phase = 0;
  L->y = round_up(phase, 256);
  // persistent kernels (m <= 16): one output region per phase type, the
  // down phase's first so that L->y always holds the last phase's outputs
  const size_t yb = round_up((size_t)m * ymax * 4, 256);
  L->a = L->y + (m <= kStackMaxM ? 4 : 1) * yb;
  L->b = L->a + round_up((size_t)m * amax * 2, 256);
  L->c = L->b + round_up((size_t)m * bmax * 2, 256);
  L->h = L->c + round_up((size_t)m * cmax * 2, 256);
  L->signs = L->h + round_up((size_t)m * hmax * 2, 256);
  L->sign_words = (uint32_t)words;
  L->params = L->signs + round_up((size_t)words * 4, 256);
  L->xq = L->params + round_up((size_t)n_layers * 4 * tq::PARAM_QUADS * 16, 256);
  L->sync = L->xq + (m > 1 && m <= kStackMaxM ? xt_bytes(m, kmax) : 0);
  L->total = L->sync + 256;
  return TQ_OK;
}

// Output regions of the four phase types: at m <= 16 one each, down first (at
// L.y), then q|k|v, o, gate|up; beyond, one shared region.
static size_t stack_y_offset(const StackWs& L, int32_t m, int phase) {
  if (m > kStackMaxM) return L.y;
  const size_t yb = (L.a - L.y) / 4;
  const int order[4] = {1, 2, 3, 0};
  return L.y + order[phase] * yb;
}

// The whole stack as one cooperative persistent kernel: stack1_kernel at
// batch 1, stackn_kernel for 2-16 tokens.  Returns TQ_ERR_SHAPE (and launches
// nothing) when the stack does not qualify: more than STACK_MAX_LAYERS layers,
// phases with different codebooks, or a phase too wide for shared memory.
static int stack_run(const tq_layer_t* layers, int32_t n_layers, const uint16_t* h_in, int32_t m, uint64_t seed,
                     uint16_t* h_out, char* ws, const StackWs& L, int sms, const tq_stack_options_t* opt,
                     cudaStream_t s) {
  if (n_layers > tq::STACK_MAX_LAYERS || sms > kStackMaxCtas) return TQ_ERR_SHAPE;
  static thread_local tq::StackParams sp;  // large (~25 KB): per-thread storage, copied into the launch
  memset(&sp, 0, sizeof(sp));
  const uint16_t* cb = layers[0].q.codebook_d;
  int32_t kmax = 0;
  uint32_t off = 0;
  for (int l = 0; l < n_layers; ++l) {
    const tq_layer_t& ly = layers[l];
    const tq_weight_t* ops[7] = {&ly.q, &ly.k, &ly.v, &ly.o, &ly.gate, &ly.up, &ly.down};
    tq::StackLayerDev& d = sp.layers[l];
    for (int i = 0; i < 7; ++i) {
      if (ops[i]->codebook_d != cb) return TQ_ERR_SHAPE;
      d.codes[i] = ops[i]->codes_d;
      d.scales[i] = ops[i]->scales_d;
      d.n[i] = ops[i]->n;
    }
    const int32_t ks[4] = {ly.q.k, ly.o.k, ly.gate.k, ly.down.k};
    const int32_t nt[4] = {ly.q.n + ly.k.n + ly.v.n, ly.o.n, ly.gate.n + ly.up.n, ly.down.n};
    for (int ph = 0; ph < 4; ++ph) {
      d.k[ph] = ks[ph];
      d.sign_off[ph] = off;
      off += (uint32_t)ks[ph] / 32;
      d.alpha[ph] = stack_alpha(ks[ph]);
      if (ks[ph] > kmax) kmax = ks[ph];
      if ((nt[ph] + 15) / 16 > kMaxTiles) return TQ_ERR_SHAPE;
    }
  }
  const int nt = m <= 8 ? 1 : 2;  // 8-token column tiles of the small-batch kernel
  const int lv = m == 1 ? dmma_lv_for(true, kmax) : 3;
  const size_t smem = m == 1 ? (16384u << lv) + (size_t)kmax * 4 + 4 * tq::PARAM_QUADS * 16 +
                                   tq::DMMA_WARPS * 32 * sizeof(float) + 4 * (tq::DMMA_WARPS + 1) * sizeof(int32_t) +
                                   (size_t)kmax / 512 * sizeof(int32_t) + 32
                             : (16384u << lv) + (size_t)tq::DMMA_WARPS * 2 * 16 * nt * 8 * sizeof(float) +
                                   4 * tq::PARAM_QUADS * 16 + 4 * (tq::DMMA_WARPS + 1) * sizeof(int32_t) + 32;
  if (smem > 227 * 1024) return TQ_ERR_SHAPE;
  sp.m = m;
  sp.xq = m > 1 ? reinterpret_cast<uint16_t*>(ws + L.xq) : nullptr;
  sp.n_layers = n_layers;
  sp.lv = lv;
  sp.codebook = cb;
  sp.h_in = h_in;
  sp.h_out = h_out;
  sp.buf[0] = reinterpret_cast<uint16_t*>(ws + L.a);
  sp.buf[1] = reinterpret_cast<uint16_t*>(ws + L.b);
  sp.buf[2] = reinterpret_cast<uint16_t*>(ws + L.c);
  sp.buf[3] = reinterpret_cast<uint16_t*>(ws + L.h);
  for (int ph = 0; ph < 4; ++ph) sp.y[ph] = reinterpret_cast<float*>(ws + stack_y_offset(L, m, ph));
  sp.signs = reinterpret_cast<uint32_t*>(ws + L.signs);
  sp.sign_words = L.sign_words;
  sp.seed = seed;
  sp.counters = reinterpret_cast<int32_t*>(ws);
  sp.status = reinterpret_cast<int32_t*>(ws + kStatusOff);
  sp.partials = reinterpret_cast<float*>(ws + kCounterBytes);
  sp.sync = reinterpret_cast<uint32_t*>(ws + L.sync);
  sp.phase_table = reinterpret_cast<uint4*>(ws + L.params);
  sp.spin_limit = (opt && opt->spin_limit) ? opt->spin_limit : (1u << 24);  // x 64 ns sleeps: ~1 s by default
  sp.skip_arrive_cta = opt ? opt->test_skip_arrive : -1;
  void (*kern)(tq::StackParams);
  if (m > 1) {
    kern = nt == 1 ? tq::stackn_kernel<3, 1> : tq::stackn_kernel<3, 2>;
  } else {
    switch (lv) {
      case 3: kern = tq::stack1_kernel<3>; break;
      case 2: kern = tq::stack1_kernel<2>; break;
      case 1: kern = tq::stack1_kernel<1>; break;
      default: kern = tq::stack1_kernel<0>; break;
    }
  }
  TQ_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024));
  int occ = 0;
  TQ_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, tq::DMMA_THREADS, smem));
  if (occ < 1) return TQ_ERR_SHAPE;
  // partial sums of straddling tiles: three phases x copies x every CTA x two tiles
  const size_t part_bytes = m == 1 ? (size_t)3 * tq::STACK_PART_COPIES * sms * 2 * 16 * sizeof(float)
                                   : (size_t)3 * sms * 2 * 16 * nt * 8 * sizeof(float);
  if (part_bytes > L.y - kCounterBytes) return TQ_ERR_SHAPE;
  TQ_CUDA(cudaMemsetAsync(ws + L.sync, 0, 256, s));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)sms);
  cfg.blockDim = dim3(tq::DMMA_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  TQ_CUDA(cudaLaunchKernelEx(&cfg, kern, sp));
  return TQ_OK;
}

int tq_layer_stack_buffers(const tq_layer_t* layers, int32_t n_layers, int32_t m, size_t offsets[5]) {
  if (!offsets) return TQ_ERR_NULL;
  StackWs L;
  int st = stack_layout(layers, n_layers, m, &L);
  if (st != TQ_OK) return st;
  offsets[0] = L.a;
  offsets[1] = L.b;
  offsets[2] = L.c;
  offsets[3] = L.h;
  offsets[4] = L.y;
  return TQ_OK;
}

int tq_layer_stack_outputs(const tq_layer_t* layers, int32_t n_layers, int32_t m, size_t offsets[4]) {
  if (!offsets) return TQ_ERR_NULL;
  StackWs L;
  int st = stack_layout(layers, n_layers, m, &L);
  if (st != TQ_OK) return st;
  for (int p = 0; p < 4; ++p) offsets[p] = stack_y_offset(L, m, p);
  return TQ_OK;
}

int tq_layer_stack_workspace(const tq_layer_t* layers, int32_t n_layers, int32_t m, size_t* bytes) {
  if (!bytes) return TQ_ERR_NULL;
  StackWs L;
  int st = stack_layout(layers, n_layers, m, &L);
  if (st != TQ_OK) return st;
  *bytes = L.total;
  return TQ_OK;
}

int tq_layer_stack(const tq_layer_t* layers, int32_t n_layers, const uint16_t* h_in_bf16_d, int32_t m, uint64_t seed,
                   uint16_t* h_out_bf16_d, void* workspace_d, size_t ws_bytes, void* stream) {
  return tq_layer_stack_ex(layers, n_layers, h_in_bf16_d, m, seed, h_out_bf16_d, workspace_d, ws_bytes, nullptr,
                           stream);
}

int tq_layer_stack_ex(const tq_layer_t* layers, int32_t n_layers, const uint16_t* h_in_bf16_d, int32_t m,
                      uint64_t seed, uint16_t* h_out_bf16_d, void* workspace_d, size_t ws_bytes,
                      const tq_stack_options_t* options, void* stream) {
  if (options && options->test_skip_arrive < -1) return TQ_ERR_VALUE;
  if (m == 0) return TQ_OK;
  StackWs L;
  int st = stack_layout(layers, n_layers, m, &L);
  if (st != TQ_OK) return st;
  if (!h_in_bf16_d || !h_out_bf16_d || !workspace_d) return TQ_ERR_NULL;
  if (!aligned16(h_in_bf16_d) || !aligned16(h_out_bf16_d) || !aligned16(workspace_d)) return TQ_ERR_ALIGN;
  if (ws_bytes < L.total) return TQ_ERR_WORKSPACE;
  int sms = 0;
  st = check_arch(&sms);
  if (st != TQ_OK) return st;
  char* ws = static_cast<char*>(workspace_d);
  uint16_t* a = reinterpret_cast<uint16_t*>(ws + L.a);
  uint16_t* b = reinterpret_cast<uint16_t*>(ws + L.b);
  uint16_t* c = reinterpret_cast<uint16_t*>(ws + L.c);
  uint16_t* h = reinterpret_cast<uint16_t*>(ws + L.h);
  const size_t phase_bytes = L.y;
  cudaStream_t s = (cudaStream_t)stream;
  if (m <= kStackMaxM) {
    st = stack_run(layers, n_layers, h_in_bf16_d, m, seed, h_out_bf16_d, ws, L, sms, options, s);
    if (st != TQ_ERR_SHAPE) return st;  // TQ_ERR_SHAPE: not eligible, run phase by phase
  }
  for (int l = 0; l < n_layers; ++l) {
    const uint16_t* in0 = (l == 0) ? h_in_bf16_d : h;
    uint16_t* out3 = (l == n_layers - 1) ? h_out_bf16_d : h;
    const uint16_t* ins[4] = {in0, a, b, c};
    uint16_t* outs[4] = {a, b, c, out3};
    for (int p = 0; p < 4; ++p) {
      float* yp = reinterpret_cast<float*>(ws + stack_y_offset(L, m, p));
      st = run_phase(&layers[l], p, ins[p], m, tq_stack_phase_seed(seed, l, p), yp, outs[p], ws, phase_bytes, sms, s);
      if (st != TQ_OK) return st;
    }
  }
  return TQ_OK;
}

// ---- batch-1 GEMV with built-in scratch ---------------------------------------
// For callers that cannot hand the library device memory.  The scratch lives
// in a file-scope device array; host code only ever passes its device address,
// which cudaGetSymbolAddress returns for the current device.

static __device__ __align__(256) unsigned char g_gemv_scratch[TQ_GEMV_NOALLOC_SCRATCH_BYTES];
static void* g_gemv_scratch_addr[kMaxDevices];  // device address of g_gemv_scratch, per device

static_assert(TQ_GEMV_NOALLOC_SCRATCH_BYTES >= kCounterBytes + (size_t)tq::DMMA_MAX_WARPS * 2 * 16 * sizeof(float),
              "built-in scratch must hold the counters and the batch-1 partial sums");

int tq_gemv_noalloc(const tq_weight_t* w, const float* x_rot_d, float* y_d, void* stream) {
  int st = check_weight(w);
  if (st != TQ_OK) return st;
  if (w->k > kGemvMaxK) return TQ_ERR_SHAPE;
  if (!x_rot_d || !y_d) return TQ_ERR_NULL;
  if (!aligned16(x_rot_d) || !aligned16(y_d)) return TQ_ERR_ALIGN;
  if ((int64_t)(w->n + 15) / 16 > kMaxTiles || dmma_ws_layout(w->n, w->k, 1).bytes > TQ_GEMV_NOALLOC_SCRATCH_BYTES)
    return TQ_ERR_SCRATCH;
  int sms = 0;
  st = check_arch(&sms);
  if (st != TQ_OK) return st;
  int dev = 0;
  TQ_CUDA(cudaGetDevice(&dev));
  if (!g_gemv_scratch_addr[dev]) {  // first call on this device: look up the array's device address
    void* addr = nullptr;
    TQ_CUDA(cudaGetSymbolAddress(&addr, g_gemv_scratch));
    g_gemv_scratch_addr[dev] = addr;
  }
  void* ws = g_gemv_scratch_addr[dev];
  cudaStream_t s = (cudaStream_t)stream;
  DmmaParams p;
  dmma_single(p, w);
  p.m = 1;
  p.x_f32 = x_rot_d;
  p.y = y_d;
  // every check first (nothing is enqueued on an error) ...
  st = dmma_run(p, true, ws, TQ_GEMV_NOALLOC_SCRATCH_BYTES, sms, s, /*dry_run=*/true);
  if (st != TQ_OK) return st;
  // ... then the arrival counters, which must start at zero whatever an
  // earlier call left, and the launch
  TQ_CUDA(cudaMemsetAsync(ws, 0, kCounterBytes, s));
  return dmma_run(p, true, ws, TQ_GEMV_NOALLOC_SCRATCH_BYTES, sms, s);
}

namespace {

int enc_grid(long long blocks, int sms, int* grid) {
  static int per_sm = 0;
  if (per_sm == 0) {
    int b = 0;
    TQ_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, tq::encode_kernel, tq::kEncThreads, 0));
    per_sm = b > 0 ? b : 1;
  }
  long long g = (long long)sms * per_sm;
  *grid = (int)(g < blocks ? g : blocks);
  return TQ_OK;
}

int enc_check(const float* w_d, int32_t n, int32_t k, const uint16_t* codebook_d, float gain, int32_t refits,
              const uint8_t* codes_d, const uint16_t* scales_d, const float* err_d) {
  if (n < 1 || !k_ok(k)) return TQ_ERR_SHAPE;
  if (!(gain > 0.0f) || !(gain <= 3.0e38f) || refits < 0 || refits > TQ_ENCODE_MAX_REFITS) return TQ_ERR_VALUE;
  if (!w_d || !codebook_d || !codes_d || !scales_d) return TQ_ERR_NULL;
  if (!aligned16(w_d) || !aligned16(codebook_d) || !aligned16(codes_d)) return TQ_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(scales_d) & 3) || (reinterpret_cast<uintptr_t>(err_d) & 3)) return TQ_ERR_ALIGN;
  return TQ_OK;
}

}  // namespace

int tq_encode(const float* w_rot_d, int32_t n, int32_t k, const uint16_t* codebook_d, float gain, int32_t refits,
              uint8_t* codes_d, uint16_t* scales_d, float* err_d, void* stream) {
  int st = enc_check(w_rot_d, n, k, codebook_d, gain, refits, codes_d, scales_d, err_d);
  if (st != TQ_OK) return st;
  int sms = 0;
  st = check_arch(&sms);
  if (st != TQ_OK) return st;
  tq::EncArgs a = {};
  a.w = w_rot_d;
  a.ldw = k;
  a.nbl = k / 256;
  a.blocks = (long long)n * a.nbl;
  a.b0 = 0;
  a.kb = k / 256;
  a.cb = codebook_d;
  a.gain = gain;
  a.refits = refits;
  a.codes = codes_d;
  a.scales = scales_d;
  a.err = err_d;
  int grid = 0;
  st = enc_grid(a.blocks, sms, &grid);
  if (st != TQ_OK) return st;
  return launch(tq::encode_kernel, dim3((unsigned)grid), dim3(tq::kEncThreads), 0, (cudaStream_t)stream, a);
}

int tq_ldlq_workspace(int32_t n, int32_t k, size_t* bytes) {
  if (!bytes) return TQ_ERR_NULL;
  if (n < 1 || !k_ok(k)) return TQ_ERR_SHAPE;
  *bytes = (size_t)n * (size_t)(k + 256) * sizeof(float);
  return TQ_OK;
}

int tq_ldlq_encode(const float* w_rot_d, int32_t n, int32_t k, const float* u_d, const uint16_t* codebook_d, float gain,
                   int32_t refits, uint8_t* codes_d, uint16_t* scales_d, float* err_d, void* workspace_d,
                   size_t ws_bytes, void* stream) {
  int st = enc_check(w_rot_d, n, k, codebook_d, gain, refits, codes_d, scales_d, err_d);
  if (st != TQ_OK) return st;
  if (!u_d) return TQ_ERR_NULL;
  if (!aligned16(u_d)) return TQ_ERR_ALIGN;
  size_t need = 0;
  tq_ldlq_workspace(n, k, &need);
  if (!workspace_d || ws_bytes < need) return TQ_ERR_WORKSPACE;
  if (!aligned16(workspace_d)) return TQ_ERR_ALIGN;
  int sms = 0;
  st = check_arch(&sms);
  if (st != TQ_OK) return st;
  float* delta = static_cast<float*>(workspace_d);    // [n][k]
  float* wt = delta + (size_t)n * (size_t)k;          // [n][256]
  const int kb = k / 256;
  int grid = 0;
  st = enc_grid(n, sms, &grid);
  if (st != TQ_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  for (int b = 0; b < kb; ++b) {
    if (b > 0) {
      // 64-row tiles when they give at least one per SM, else 32-row tiles
      const bool wide = (int64_t)((n + 63) / 64) * (256 / tq::kFbCols) >= sms;
      if (wide)
        st = launch(tq::ldlq_feedback_kernel<4>, dim3((unsigned)((n + 63) / 64), 256 / tq::kFbCols), dim3(256), 0, s,
                    w_rot_d, (const float*)delta, u_d, (int)n, (int)k, b, wt);
      else
        st = launch(tq::ldlq_feedback_kernel<2>, dim3((unsigned)((n + 31) / 32), 256 / tq::kFbCols), dim3(256), 0, s,
                    w_rot_d, (const float*)delta, u_d, (int)n, (int)k, b, wt);
      if (st != TQ_OK) return st;
    }
    tq::EncArgs a = {};
    a.w = b > 0 ? wt : w_rot_d;
    a.ldw = b > 0 ? 256 : k;
    a.nbl = 1;
    a.blocks = n;
    a.b0 = b;
    a.kb = kb;
    a.cb = codebook_d;
    a.gain = gain;
    a.refits = refits;
    a.codes = codes_d;
    a.scales = scales_d;
    a.err = err_d;
    a.w_ref = w_rot_d;
    a.ldr = k;
    a.delta = (b + 1 < kb) ? delta : nullptr;
    st = launch(tq::encode_kernel, dim3((unsigned)grid), dim3(tq::kEncThreads), 0, s, a);
    if (st != TQ_OK) return st;
  }
  return TQ_OK;
}

const char* tq_status_string(int status) {
  switch (status) {
    case TQ_OK: return "ok";
    case TQ_ERR_SHAPE: return "bad shape (k must be a positive multiple of 512, n >= 1, 0 <= m <= 4096)";
    case TQ_ERR_ALIGN: return "pointer not 16-byte aligned";
    case TQ_ERR_NULL: return "required pointer is NULL";
    case TQ_ERR_ARCH: return "device is not compute capability 10.0 (sm_100a)";
    case TQ_ERR_WORKSPACE: return "workspace missing or too small";
    case TQ_ERR_CUDA: return "CUDA runtime error (see tq_last_cuda_error)";
    case TQ_ERR_TIMEOUT: return "bounded device wait expired";
    case TQ_ERR_SCRATCH: return "problem larger than the built-in scratch of tq_gemv_noalloc (n > 262128)";
    case TQ_ERR_VALUE: return "a scalar argument is out of range";
    default: return "unknown status";
  }
}

int tq_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"
