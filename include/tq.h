/*
 * tq.h -- C ABI of libtq, the B200 (sm_100a) trellis-decode matmul library.
 *
 * The method (pages cited by title and section):
 *   "Pingala-8" landing page, "How it works": linear-layer weights are stored
 *   as an 8-state trellis code over groups of 4 weights, coded in order; a
 *   small state carried from one group to the next selects the set of values
 *   the next group may use.  A random Hadamard rotation is applied to the
 *   weights before encoding.
 *   "Bonsai 2 27B" article, change-of-basis paragraph: the rotation is folded
 *   into the stored weights; the matching transform runs on the activations
 *   at inference time.
 *   "8 open models ... what 2-bit quantization costs", "Size": per-block
 *   scales add bits on top of the 2-bit codes; "Speed": batch-1 decoding is
 *   a matter of reading the weights from memory once per token.
 *
 * Format (the pages fix no bit layout; this is the layout the library uses):
 *   codes     uint8  [n][k/4]   one code c per group of 4 weights, row-major
 *   scales    fp16   [n][k/256] one scale per row and 256-weight block
 *   codebook  fp16   [8][256][4] entry (s, c) is a 4-vector
 *   state     s_g = 0 when g % 64 == 0, else codes[n][g-1] & 7
 *   weight    W[n][4g+j] = fp16_RNE(scale[n][g/64] * codebook[s_g][c_g][j])
 *   size      n*k/4 + 2*n*k/256 bytes = 2.0625 bits per weight
 *   RHT       x'[m][512b+i] = (1/sqrt(512)) sum_j H[i][j] d[512b+j] x[m][512b+j],
 *             H[i][j] = (-1)^popcount(i&j) (natural / Sylvester order),
 *             d[k] = -1 if bit 63 of splitmix64_k(seed) is set, else +1,
 *             where splitmix64_k(seed) is the k-th (0-based) output of a
 *             SplitMix64 generator whose state starts at `seed`.
 *   linear    y[m][n] = sum_k W[n][k] x'[m][k]   (fp32 output)
 *
 * Conventions for every call:
 *   - Pointers named *_d are DEVICE pointers and are caller-owned; the library
 *     never allocates device memory and never frees what it is given.
 *     Host pointers (structs, `out` arguments) are read or written before the
 *     call returns.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     are asynchronous on it; none synchronises, except tq_workspace_status,
 *     which reads a word of device memory back to the host.
 *   - Return value: TQ_OK or one TQ_ERR_* code.  On an error nothing is
 *     launched.  No C++ exception crosses this interface.
 *   - k must be a positive multiple of 512.  n >= 1.  m >= 0 (m == 0 and
 *     n == 0 are accepted as empty work and return TQ_OK without a launch
 *     where stated).
 *   - codes_d, x and y pointers must be 16-byte aligned (TQ_ERR_ALIGN).
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TQ_API __attribute__((visibility("default")))
#else
#define TQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
#define TQ_OK 0
#define TQ_ERR_SHAPE 1     /* a size is out of range (k % 512, n < 1, m < 0, m too large) */
#define TQ_ERR_ALIGN 2     /* a pointer is not 16-byte aligned */
#define TQ_ERR_NULL 3      /* a required pointer is NULL */
#define TQ_ERR_ARCH 4      /* the current device is not compute capability 10.0 */
#define TQ_ERR_WORKSPACE 5 /* workspace missing or smaller than the *_workspace query */
#define TQ_ERR_CUDA 6      /* a CUDA runtime call failed; tq_last_cuda_error() has its code */
#define TQ_ERR_TIMEOUT 7   /* a bounded device-side wait expired (reported by the status word) */
#define TQ_ERR_SCRATCH 8   /* the problem does not fit the built-in scratch of tq_gemv_noalloc */
#define TQ_ERR_VALUE 9     /* a scalar argument (not a size) is out of range */

/* output element types */
#define TQ_F32 0
#define TQ_F16 1

/* One trellis-coded weight.  All pointers are device pointers (caller-owned).
 * codes_d: uint8 [n][k/4], 16-byte aligned.  scales_d: fp16 bits [n][k/256],
 * 4-byte aligned (the kernels read the scales of two blocks at a time).
 * codebook_d: fp16 bits [8][256][4] (16384 bytes), 16-byte aligned. */
typedef struct tq_weight {
  const uint8_t* codes_d;
  const uint16_t* scales_d;
  const uint16_t* codebook_d;
  int32_t n;
  int32_t k;
} tq_weight_t;

/* Sizes of one packed n x k weight ("Size" section: codes plus per-block
 * scales).  packed_bytes = code_bytes + scale_bytes = n*k*33/128. */
typedef struct tq_pack_info {
  int32_t n, k;
  int32_t group;     /* 4 weights per code */
  int32_t block;     /* 256 weights per scale and per state reset */
  int32_t rht_block; /* 512 */
  int32_t n_states;  /* 8 */
  int64_t code_bytes;
  int64_t scale_bytes;
  int64_t codebook_bytes; /* 16384, shared by all rows */
  int64_t packed_bytes;
  double bits_per_weight; /* 2.0625 */
} tq_pack_info_t;

/* Host-only.  Fills *out for an n x k weight.  TQ_ERR_SHAPE unless n >= 1 and
 * k is a positive multiple of 512; TQ_ERR_NULL if out is NULL. */
TQ_API int tq_pack_info(int32_t n, int32_t k, tq_pack_info_t* out);

/* Decode the whole weight to fp16 (test and inspection export; the matmul
 * calls never materialise W).  Definition: the "weight" line of the format
 * above ("How it works": the previous group's state selects the codebook).
 * w_f16_d: device, fp16 bits [n][k], caller-owned, 16-byte aligned. */
TQ_API int tq_decode(const tq_weight_t* w, uint16_t* w_f16_d, void* stream);

/* Randomized Hadamard transform of the activations ("How it works" and the
 * "Bonsai 2" change-of-basis paragraph): x' = H_512 . D . x on each block of
 * 512 features of each of the m rows.
 * x_bf16_d: device bf16 bits [m][k], 16-byte aligned.
 * x_rot_d:  device [m][k], fp32 (out_dtype TQ_F32) or fp16 (TQ_F16, rounded
 *           to nearest even), 16-byte aligned.
 * m == 0 returns TQ_OK without a launch. */
TQ_API int tq_rht(const uint16_t* x_bf16_d, int32_t m, int32_t k, uint64_t seed, void* x_rot_d, int32_t out_dtype,
           void* stream);

/* Bytes of device workspace tq_gemv needs for an n x k weight (split-row
 * partial sums and per-tile arrival counters). */
TQ_API int tq_gemv_workspace(int32_t n, int32_t k, size_t* bytes);

/* Batch-1 decode-GEMV: y[n] = sum_k W[n][k] x_rot[k] with W decoded on the
 * fly from the codes ("Speed": one read of the packed weight per token).
 * x_rot_d: device fp32 [k] (already rotated, e.g. by tq_rht), 16-byte aligned.
 * y_d: device fp32 [n], 16-byte aligned.
 * workspace_d: device, >= tq_gemv_workspace bytes, 16-byte aligned.  Every
 * workspace begins with a 64 KB region of per-tile counters that must be zero
 * before the first call (tq_workspace_init); every call of this library leaves
 * it zero again, so one workspace may serve calls of any shape in turn.  The
 * rest is scratch.  Calls that share a workspace must not overlap on the GPU.
 * n is limited to 262128 rows per call and k to TQ_GEMV_MAX_K (the kernel
 * keeps 4 bytes of activations per feature in shared memory beside a 16 KB
 * codebook copy); beyond either, TQ_ERR_SHAPE before anything is launched. */
#define TQ_GEMV_MAX_K 53760
TQ_API int tq_gemv(const tq_weight_t* w, const float* x_rot_d, float* y_d, void* workspace_d, size_t ws_bytes,
            void* stream);

/* Batch-1 decode-GEMV that allocates nothing and takes no workspace.
 * No counterpart on the pages: this is an interface for callers that cannot
 * give the library device memory -- for example a runtime that owns every
 * device allocation and has no workspace hook for a custom op, or a latency
 * path that must not call cudaMalloc (which can synchronise the device).
 * Same arguments and result as tq_gemv, without the workspace.
 * Scratch: a file-scope device array of TQ_GEMV_NOALLOC_SCRATCH_BYTES
 * (1 MiB + 64 KiB), which every GPU that loads the library holds until the
 * process exits.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress) for that device; make that first call before
 * any stream capture.  Each call clears the array's counter region on
 * `stream` before the kernel, and calls no cudaMalloc, cudaFree or other
 * allocating routine.  Every call on a device shares that device's copy of
 * the array, which keeps the last call's contents: calls that overlap on the
 * GPU (for example on two streams) race and give wrong results, so run them
 * one after another.
 * Limits: n <= 262128 rows (TQ_ERR_SCRATCH beyond it); k a positive
 * multiple of 512 up to TQ_GEMV_MAX_K (TQ_ERR_SHAPE beyond it).  Every check
 * runs before the counter clear is enqueued: on an error nothing is
 * enqueued. */
#define TQ_GEMV_NOALLOC_SCRATCH_BYTES ((size_t)(1u << 20) + (size_t)(64u << 10))
TQ_API int tq_gemv_noalloc(const tq_weight_t* w, const float* x_rot_d, float* y_d, void* stream);

/* Bytes of device workspace tq_gemm needs for an n x k weight and m tokens. */
TQ_API int tq_gemm_workspace(int32_t n, int32_t k, int32_t m, size_t* bytes);

/* Small-batch / prompt matmul: y[t][n] = sum_k W[n][k] x_rot[t][k] for m
 * tokens.  x_rot_f16_d: device fp16 [m][k] (tq_rht with TQ_F16), 16-byte
 * aligned.  y_d: device fp32 [m][n], 16-byte aligned.  The kernel is chosen by
 * m: register-decode warp MMAs up to 32 tokens, tcgen05 MMAs with TMEM
 * accumulators from 33 (the decoded weights staged in tensor memory for
 * 64- and 256-token tiles, in shared memory for 128-token tiles).  Same
 * workspace rules as tq_gemv.
 * m == 0 returns TQ_OK without a launch; m > 4096 is TQ_ERR_SHAPE. */
TQ_API int tq_gemm(const tq_weight_t* w, const uint16_t* x_rot_f16_d, int32_t m, float* y_d, void* workspace_d,
            size_t ws_bytes, void* stream);

/* tq_gemm with options (tq_stack_options_t, declared with tq_layer_stack_ex;
 * NULL = the defaults, which is tq_gemm).  They act on the tcgen05 kernel
 * (m >= 33) only: spin_limit = try-wait polls of each of its bounded mbarrier
 * waits (0 = the default, 2^21); test_skip_arrive = c >= 0 makes thread block
 * c's decoded-stage barriers expect one arrival more than its decoders make,
 * so that block's MMA wait runs out: the launch ends with TQ_ERR_TIMEOUT in
 * the workspace's status word and undefined outputs (a test hook of the
 * timeout path; -1 = off, below -1 = TQ_ERR_VALUE).  The register-decode
 * kernel (m <= 32) has no wait on other thread blocks and ignores them. */
typedef struct tq_stack_options tq_stack_options_t;
TQ_API int tq_gemm_ex(const tq_weight_t* w, const uint16_t* x_rot_f16_d, int32_t m, float* y_d, void* workspace_d,
                      size_t ws_bytes, const tq_stack_options_t* options, void* stream);

/* Zero a workspace (cudaMemsetAsync on `stream`). */
TQ_API int tq_workspace_init(void* workspace_d, size_t bytes, void* stream);

/* ---- device-side status ------------------------------------------------------
 * Kernels that wait on other thread blocks (the tcgen05 GEMM's pipeline
 * barriers, the persistent stack kernels' grid barriers and block flags) bound
 * every wait.  When a wait runs out, the kernel writes TQ_ERR_TIMEOUT into the
 * 32-bit status word at byte TQ_STATUS_OFFSET of the workspace it was given
 * (the last word of the 64 KB counter region), stops and returns; its outputs
 * are then undefined.  The host calls return before the kernels run, so they
 * cannot report it: read the word after the stream has reached the call.
 * No call of this library clears it except tq_workspace_init, and after a
 * timeout the counter region may hold non-zero counts, so re-initialise the
 * workspace (tq_workspace_init) before using it again.
 * The batch-1 GEMV (tq_gemv, tq_gemv_noalloc) has no device-side wait (its
 * split tiles are summed by the last block to arrive), so it never sets it. */
#define TQ_STATUS_OFFSET 65532

/* Copy the status word of `workspace_d` to *status (TQ_OK or TQ_ERR_TIMEOUT)
 * after everything enqueued on `stream` before it.  The one call of this
 * library that synchronises: it waits for `stream`.  Does not clear the word. */
TQ_API int tq_workspace_status(const void* workspace_d, int32_t* status, void* stream);

/* ---- layer stack ----------------------------------------------------------
 * One layer = q, k, v, o, gate, up, down.  Per layer, four phases run in
 * order; each starts with the RHT of its input and ends with the handoff
 * h' = bf16_RNE(alpha(k_op) * y_op) of one op's output, where
 * alpha(k) = 1/sqrt(k * E[s^2]) and E[s^2] = (0.03^3 - 0.005^3)/(3*0.025)
 * (the second moment of a U[0.005, 0.03] scale), so that every handoff has
 * about unit variance:
 *   phase 0: x' = RHT(h)        -> q, k, v       handoff alpha(k_q) * q
 *   phase 1: x' = RHT(phase 0)  -> o             handoff alpha(k_o) * o
 *   phase 2: x' = RHT(phase 1)  -> gate, up      handoff alpha(k_gate) * gate
 *   phase 3: x' = RHT(phase 2)  -> down          handoff alpha(k_down) * down = next h
 * The k, v and up outputs are computed (and written to y) but not consumed:
 * they stand in for attention and the gated product, which are not part of
 * the trellis-decode path.  The RHT of phase p of layer l uses the seed
 * tq_stack_phase_seed(seed, l, p).  All ops of one phase must share k and the
 * codebook pointer (TQ_ERR_SHAPE otherwise). */
typedef struct tq_layer {
  tq_weight_t q, k, v, o, gate, up, down;
} tq_layer_t;

/* mix64(seed ^ mix64(0x516E0000 | layer << 2 | phase)), mix64 = the
 * SplitMix64 output function. */
TQ_API uint64_t tq_stack_phase_seed(uint64_t seed, int32_t layer, int32_t phase);

/* Workspace bytes for one phase / for a whole stack at m tokens. */
TQ_API int tq_layer_phase_workspace(const tq_layer_t* layer, int32_t phase, int32_t m, size_t* bytes);
TQ_API int tq_layer_stack_workspace(const tq_layer_t* layers, int32_t n_layers, int32_t m, size_t* bytes);

/* One phase of one layer.
 * x_bf16_d: device bf16 [m][k_phase] input.
 * y_d: device fp32 [m][n_phase] (the phase's ops concatenated in the order
 *      listed above), or NULL to skip writing it.
 * handoff_bf16_d: device bf16 [m][n_handoff] (n of q / o / gate / down).
 * phase_seed: the RHT seed of this phase. */
TQ_API int tq_layer_phase(const tq_layer_t* layer, int32_t phase, const uint16_t* x_bf16_d, int32_t m, uint64_t phase_seed,
                   float* y_d, uint16_t* handoff_bf16_d, void* workspace_d, size_t ws_bytes, void* stream);

/* The whole stack: h_out = layers[n-1] o ... o layers[0] (h_in).
 * layers: HOST array of n_layers tq_layer_t (device pointers inside).
 * h_in_bf16_d / h_out_bf16_d: device bf16 [m][hidden]; they may alias.
 * For 1 <= m <= 16 every phase of every layer runs in ONE cooperative
 * persistent launch: one thread block per SM, all of them resident at once,
 * with bounded grid-wide waits between phases (the launch fails with
 * TQ_ERR_CUDA when the blocks cannot all be resident, e.g. when other work
 * holds SMs; a wait that runs out leaves TQ_ERR_TIMEOUT in the status word).
 * A stack that does not fit that kernel (more than 128 layers, phases with
 * different codebooks, a phase too wide for shared memory) and m > 16 run as
 * 4 launch groups per layer (RHT + matmul), PDL-chained on `stream`.  Either
 * way the work is enqueued on `stream` and can be captured in a CUDA graph. */
TQ_API int tq_layer_stack(const tq_layer_t* layers, int32_t n_layers, const uint16_t* h_in_bf16_d, int32_t m, uint64_t seed,
                   uint16_t* h_out_bf16_d, void* workspace_d, size_t ws_bytes, void* stream);

/* Options of tq_layer_stack_ex.
 * spin_limit: polls each bounded wait of the persistent kernels makes before
 *   it gives up (each poll is one L2 round trip plus a 64 ns sleep); 0 = the
 *   default, about a second, far above any healthy wait.
 * test_skip_arrive: a fault-injection hook for tests of the timeout path.
 *   -1 = off.  c >= 0: thread block c of the persistent kernel does not
 *   arrive at the launch's first grid barrier, so every block's bounded wait
 *   there runs out; the launch ends early with TQ_ERR_TIMEOUT in the status
 *   word and undefined outputs.  Values below -1 are TQ_ERR_VALUE; a block
 *   index past the grid makes nothing happen.  Ignored by the per-phase path
 *   (m > 16). */
struct tq_stack_options {
  uint32_t spin_limit;
  int32_t test_skip_arrive;
};

/* tq_layer_stack with options (NULL = the defaults, which is tq_layer_stack). */
TQ_API int tq_layer_stack_ex(const tq_layer_t* layers, int32_t n_layers, const uint16_t* h_in_bf16_d, int32_t m,
                             uint64_t seed, uint16_t* h_out_bf16_d, void* workspace_d, size_t ws_bytes,
                             const tq_stack_options_t* options, void* stream);

/* Byte offsets, inside a tq_layer_stack workspace for these layers and m,
 * of the bf16 buffers that hold the last layer's phase handoffs when
 * tq_layer_stack has returned: offsets[0] = q handoff [m][q.n], offsets[1] =
 * o handoff [m][o.n], offsets[2] = gate handoff [m][gate.n], offsets[3] = the
 * last layer's input h [m][hidden] (for n_layers >= 2; with one layer the
 * input is h_in); offsets[4] = fp32 y of the last phase (down) [m][down.n].
 * The last phase's handoff is h_out itself.  For inspection and tests; the
 * buffers are scratch for the next call. */
TQ_API int tq_layer_stack_buffers(const tq_layer_t* layers, int32_t n_layers, int32_t m, size_t offsets[5]);

/* Byte offsets, inside a tq_layer_stack workspace for these layers and m, of
 * the fp32 outputs y [m][n_phase] of the last layer's four phases (q|k|v,
 * o, gate|up, down: every op of the phase, concatenated by rows) when
 * tq_layer_stack has returned.  At m <= 16 each phase has its own buffer;
 * beyond, the phases share one buffer (all four offsets are equal) and only
 * the last phase's outputs are left in it.  offsets[3] equals
 * tq_layer_stack_buffers' offsets[4].  For inspection and tests; the
 * pages define no such query.  TQ_ERR_NULL / TQ_ERR_SHAPE as
 * tq_layer_stack_workspace. */
TQ_API int tq_layer_stack_outputs(const tq_layer_t* layers, int32_t n_layers, int32_t m, size_t offsets[4]);

/* ---- encoder ----------------------------------------------------------------
 * Trellis encoder ("Pingala-8" landing page, "How it works": groups of four
 * weights are coded in order, the state carried from one group selects the
 * values the next may use, and a random Hadamard rotation is applied to the
 * weights before encoding).  The pages give no encoding procedure; this is
 * the one the library implements, per row and 256-weight block b:
 *   1. scale = fp16_RNE(min(sqrt(sum_i w_i^2 / 256) * gain, 65504));
 *   2. the code path of least squared error sum_i (w_i - W_i)^2, W the
 *      decoded block (the "weight" line of the format above), from state 0
 *      with a free end state, by dynamic programming over the 8 states;
 *   3. up to `refits` times: scale' = fp16_RNE(sum w_i e_i / sum e_i^2), e the
 *      unscaled codebook values on the path (clamped to +-65504); a new path
 *      at scale'; kept only when it costs less, otherwise stop (also when
 *      scale' equals the scale or sum e_i^2 is not positive).
 * Decisions are taken in binary32 in one fixed order (see tq_encode.cuh), so
 * results are reproducible bit for bit.
 * w_rot_d:   device fp32 [n][k], the rotated weights (tq_rht of the bf16
 *            weight rows with TQ_F32 and the seed the activations will use),
 *            16-byte aligned, finite; |w| should stay well inside the fp16
 *            range (a scaled codebook entry that overflows fp16 makes that
 *            block's result unspecified).
 * codebook_d: fp16 bits [8][256][4], 16-byte aligned.
 * gain:      > 0 and finite; 1 / RMS(codebook entries) matches the block RMS
 *            to the codebook's (TQ_ERR_VALUE otherwise).
 * refits:    0 .. TQ_ENCODE_MAX_REFITS (TQ_ERR_VALUE otherwise).
 * codes_d:   device uint8 [n][k/4] out, 16-byte aligned.
 * scales_d:  device fp16 bits [n][k/256] out, 4-byte aligned.
 * err_d:     device fp32 [n][k/256] out, or NULL: per block, the squared
 *            error of the chosen encoding summed in fold order
 *            (v[i] += v[i + h], h = 128 ... 1), 4-byte aligned.
 * k must be a positive multiple of 512 and n >= 1 (TQ_ERR_SHAPE). */
#define TQ_ENCODE_MAX_REFITS 16
TQ_API int tq_encode(const float* w_rot_d, int32_t n, int32_t k, const uint16_t* codebook_d, float gain, int32_t refits,
                     uint8_t* codes_d, uint16_t* scales_d, float* err_d, void* stream);

/* Block LDLQ with the trellis encoder (the LDLQ step named on the
 * "Pingala-8" landing page, section "How it works"; the feedback it applies
 * is the equation below).  The proxy Hessian of the layer's inputs is given by its factor:
 * H = (I + U) D (I + U)^T with U strictly upper triangular by 256-column
 * blocks (U[i][j] = 0 unless i/256 < j/256; D, block diagonal, is not needed).
 * For each 256-column block b in order, every row is encoded (as tq_encode)
 * from
 *   w~[r][256b + j] = w[r][256b + j] + sum_{i < 256b} E[r][i] U[i][256b + j],
 * E = w - w_hat over the blocks already coded, each element summed by fma in
 * ascending i in binary32.  Then E (I + U) = w~ - w_hat blockwise: the proxy
 * loss tr(E H E^T) is the D-weighted error of the adjusted blocks.
 * w_rot_d, codebook_d, gain, refits, codes_d, scales_d: as tq_encode.
 * u_d:      device fp32 [k][k] row-major, 16-byte aligned (only the block
 *           strictly upper part is read).
 * err_d:    device fp32 [n][k/256] or NULL: per block, the fold-order sum of
 *           (w~ - w_hat)^2.
 * workspace_d: device, >= tq_ldlq_workspace bytes = 4 n (k + 256), 16-byte
 *           aligned (E and the adjusted block; no initial contents needed).
 * Errors: those of tq_encode; TQ_ERR_NULL for a NULL u_d; TQ_ERR_ALIGN for
 * u_d or workspace_d; TQ_ERR_WORKSPACE for a missing or short workspace.
 * Enqueues 2*(k/256) - 1 launches on `stream`. */
TQ_API int tq_ldlq_workspace(int32_t n, int32_t k, size_t* bytes);
TQ_API int tq_ldlq_encode(const float* w_rot_d, int32_t n, int32_t k, const float* u_d, const uint16_t* codebook_d,
                          float gain, int32_t refits, uint8_t* codes_d, uint16_t* scales_d, float* err_d,
                          void* workspace_d, size_t ws_bytes, void* stream);

/* Human-readable text of a status code (static storage). */
TQ_API const char* tq_status_string(int status);

/* The cudaError_t value behind the last TQ_ERR_CUDA returned on this thread. */
TQ_API int tq_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
