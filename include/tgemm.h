/*
 * tgemm.h -- C ABI of the B200 (sm_100a) ternary / 4-bit dequant-fused matmul library
 * (libtgemm.so).
 *
 * What is computed (page title, section):
 *   Q2_0 ternary weights -- "We're Teaching Your Browser to Paint: A 4B Image Model on
 *     WebGPU", section "The lucky break that wasn't luck": blocks of 128 weights along
 *     the input axis with one f16 scale d; 2-bit codes q in {0,1,2}, four per byte,
 *     least-significant bits first; w = (q - 1) * d.  The converter's only rounding is
 *     the scale's f32 -> f16 conversion, and it must round-trip exactly.
 *   4-bit group weights -- "You Can Now Just Ask for an Image -- and Your Browser Draws
 *     It", section "The bug that hid in one flipped bit": two codes per byte, code t of
 *     a row is (byte[t/2] >> ((t & 1) * 4)) & 0xF (even index in the low nibble);
 *     "We're Teaching...", section "What's left": w = (q - z) * s.
 *   Low-rank side branch -- "mindview-t2i-turbo", section "One step": y = W x + B (A x).
 *   Row slicing -- "We're Teaching...", section "The GPU driver, and the bug that looked
 *     like broken math": quantized rows are independent byte runs, so rows [n0, n1) of a
 *     packed matrix are the pointers wq + n0*K/4, d + n0*K/128 (Q2) or wq + n0*K/2,
 *     sz + n0*(K/64)*2 (4-bit), with N = n1 - n0.
 *
 * Layouts (all row-major, the input axis K innermost):
 *   x      bf16 bit patterns [M][K]                 activations
 *   Q2:    wq  uint8 [N][K/4]     d  f16 [N][K/128]   (K a multiple of 128)
 *   4-bit: wq  uint8 [N][K/2]     sz f16 [N][K/64][2], (s, z) per group of 64 (K % 64 == 0)
 *   a      bf16 [r][K], b bf16 [N][r]                side-branch factors, 1 <= r <= 256
 *   y      [M][N], f32 (TGEMM_OUT_F32) or bf16 (TGEMM_OUT_BF16, round to nearest even)
 *   y[m][n] = sum_k w[n][k] * x[m][k]  (+ sum_i b[n][i] * sum_k a[i][k] * x[m][k])
 *
 * Ownership and memory: every pointer argument is a DEVICE pointer owned by the caller;
 * the library keeps no reference after a call returns and allocates no device memory.
 * Scratch space the matmuls need (an f16 copy of x for the tensor-core path, the side
 * branch's A x) lives in a caller-provided workspace whose size tgemm_workspace_size()
 * returns.
 *
 * Execution and errors: every call is asynchronous on `stream` (a cudaStream_t, or NULL
 * for the legacy default stream).  The return value reports only what can be known on
 * the host: argument checks and launch failures.  Results, pack status words and the
 * device error word are valid once the stream has been synchronized.  No kernel traps:
 * pack problems are reported through a status word, and a device-side wait that runs
 * out of time sets a bit in the device error word (tgemm_device_error) and returns.
 *
 * Accuracy: the matmuls accumulate in f32.  The tensor-core path multiplies f16
 * operands: x is converted bf16 -> f16 (exact for |x| in f16's normal range; x must be
 * finite with |x| < 65504), Q2 weights (q-1)*d are exact in f16, 4-bit weights are the
 * f16 rounding of (q - z) * s.
 */
#ifndef TGEMM_H
#define TGEMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes (return values) ------------------------------------------------ */
#define TGEMM_OK          0
#define TGEMM_EINVAL     -1 /* null pointer, non-positive size, K not a multiple of the
                               block, r outside [1,256], unknown out_dtype/op/path */
#define TGEMM_EALIGN     -2 /* a pointer is not aligned as documented for its argument */
#define TGEMM_ECUDA      -3 /* a CUDA runtime call or kernel launch failed */
#define TGEMM_EARCH      -4 /* the current device is not compute capability 10.0 */
#define TGEMM_EWORKSPACE -5 /* workspace missing or smaller than tgemm_workspace_size_min() */
#define TGEMM_ETOOLARGE  -6 /* tgemm_q2_noalloc: the problem needs more scratch than its
                               built-in buffer (TGEMM_NOALLOC_SCRATCH_BYTES) holds;
                               q2_from_gemlite: more than 2^31 - 1 transpose tiles */

/* ---- output element types ---------------------------------------------------------- */
#define TGEMM_OUT_F32  0
#define TGEMM_OUT_BF16 1

/* ---- pack status bits (OR-ed into the caller's device status word) ----------------- */
#define TGEMM_PACK_BAD_CODE  1u /* a Q2 code > 2 or a 4-bit code > 15 (stored masked) */
#define TGEMM_PACK_INEXACT   2u /* a scale/zero is not exactly representable in f16 */
#define TGEMM_PACK_NONFINITE 4u /* a scale/zero is inf or NaN */
#define TGEMM_PACK_ZERO_MISMATCH  8u  /* q2_from_gemlite: some zero != -scale */
#define TGEMM_PACK_GROUP_MISMATCH 16u /* q2_from_gemlite: groups of one 128-block differ */

/* ---- device error word bits (tgemm_device_error) ----------------------------------- */
#define TGEMM_DEVERR_TIMEOUT 1u /* a pipeline wait in a matmul kernel ran out of time */

/* ---- operations, for tgemm_workspace_size ----------------------------------------- */
#define TGEMM_OP_Q2      0
#define TGEMM_OP_Q2_LORA 1
#define TGEMM_OP_Q4      2

/* ---- kernel path selection (tgemm_set_path) --------------------------------------- */
#define TGEMM_PATH_AUTO    0 /* M <= 16: small-M path; otherwise the tensor-core kernel */
#define TGEMM_PATH_SMALL_M 1 /* always the small-M (mma.sync) path, its form chosen per shape */
#define TGEMM_PATH_TENSOR  2 /* always the tcgen05 tensor-core kernel */
#define TGEMM_PATH_SMALL_M_PASS 3   /* small-M path, per-pass form only (for comparisons) */
#define TGEMM_PATH_SMALL_M_STREAM 4 /* small-M path, streaming form wherever its layout fits
                                       (M <= 16, one input, no branch; for tests) */

/*
 * q2_pack -- Q2_0 packing ("We're Teaching...", "The lucky break that wasn't luck").
 *   codes  uint8 [N][K], each in {0,1,2}             (16-byte aligned)
 *   scale  f32   [N][K/128], the block scales         (4-byte aligned)
 *   wq     uint8 [N][K/4]  out: code k of a row goes to bits 2*(k%4) of byte k/4 (16-byte aligned)
 *   d      f16   [N][K/128] out: scale rounded to f16 (nearest even)  (2-byte aligned)
 *   status uint32 device word (4-byte aligned), zeroed by the caller; receives
 *          TGEMM_PACK_* bits.  A code above 2 is stored as (code & 3) and sets BAD_CODE;
 *          a scale whose f16 value differs from it sets INEXACT (NONFINITE for inf/NaN).
 *          A caller following the pages aborts on any nonzero status.
 *   Requires N >= 1, K >= 128, K % 128 == 0.
 */
int q2_pack(const uint8_t* codes, const float* scale, uint8_t* wq, uint16_t* d, int N, int K,
            uint32_t* status, void* stream);

/*
 * q2_from_gemlite -- import a gemlite-int2 matrix as Q2_0, on the device ("We're Teaching
 * Your Browser to Paint...", "The lucky break that wasn't luck": gemlite's codes are
 * {0,1,2}, LSB-first, four per byte along the input axis, dequantized as
 * (q - zero) * scale with zeros == -scales, so the conversion is a transpose and regroup
 * with no numeric change; the scale's f32 -> f16 rounding must be exact).
 *   wq_g   uint8 [K/4][N]: byte (i, n) holds the codes of k = 4i..4i+3 of output row n
 *          (the input axis is the outer one; this layout is a reading, the pages do not
 *          print it)                                   (any alignment)
 *   scale, zero  f32 [N][K/g]: group j of a row covers k in [j g, (j + 1) g)  (4-byte aligned)
 *   wq, d  Q2_0 out, as from q2_pack: byte (i, n) of wq_g becomes wq[n][i] unchanged, and
 *          block b of row n gets the f16 of the scale of the groups covering
 *          [128 b, 128 b + 128)                       (16- and 2-byte aligned)
 *   status as for q2_pack, plus ZERO_MISMATCH (a zero that is not -scale) and
 *          GROUP_MISMATCH (g < 128 and the groups of one block have different scales).
 *   Requires N >= 1, K % 128 == 0, and g a multiple of 4 dividing 128 or a multiple of
 *   128 dividing K.  Load-time work.
 */
int q2_from_gemlite(const uint8_t* wq_g, const float* scale, const float* zero, int N, int K,
                    int g, uint8_t* wq, uint16_t* d, uint32_t* status, void* stream);

/*
 * q4_pack -- 4-bit packing ("You Can Now Just Ask...", "The bug that hid in one flipped bit").
 *   codes  uint8 [N][K], each in 0..15               (16-byte aligned)
 *   s, z   f32   [N][K/64], per-group scale and zero (4-byte aligned)
 *   wq     uint8 [N][K/2] out: code t in the low nibble of byte t/2 when t is even, the
 *          high nibble when t is odd                  (16-byte aligned)
 *   sz     f16   [N][K/64][2] out: (s, z) rounded to f16 (4-byte aligned)
 *   status as for q2_pack (BAD_CODE for codes > 15, stored as code & 15).
 *   Requires N >= 1, K >= 64, K % 64 == 0.
 */
int q4_pack(const uint8_t* codes, const float* s, const float* z, uint8_t* wq, uint16_t* sz,
            int N, int K, uint32_t* status, void* stream);

/*
 * q2_dequant / q4_dequant -- the weights a packed matrix stands for, in f32 [N][K]
 * (16-byte aligned): (q - 1) * d, or (q - z) * s computed as two rounded f32 operations.
 * wq 4-byte aligned; d 2-byte, sz 4-byte aligned.  Requires N >= 1 and K a multiple of
 * 128 (Q2) or 64 (4-bit).  Test hooks: they unpack the codes as the matmul kernels do.
 */
int q2_dequant(const uint8_t* wq, const uint16_t* d, float* w, int N, int K, void* stream);
int q4_dequant(const uint8_t* wq, const uint16_t* sz, float* w, int N, int K, void* stream);

/*
 * tgemm_selftest_wait_timeout -- test hook for failure detection.  Launches one CTA
 * whose wait (the same bounded mbarrier wait every pipeline of the library uses) can
 * never be satisfied: after the wait limit (1 s) it gives up, sets TGEMM_DEVERR_TIMEOUT
 * in the device error word and returns.  Nothing faults, traps or hangs, and the
 * context stays usable; read and clear the bit with tgemm_device_error.  The pages have
 * no counterpart: it checks this library's own error reporting.
 */
int tgemm_selftest_wait_timeout(void* stream);

/*
 * tgemm_selftest_bad_launch -- test hook for launch-error reporting.  Asks the CUDA
 * runtime for a launch it refuses on the host (2048 threads in one block) and returns
 * TGEMM_ECUDA; nothing reaches the GPU.  The refused launch's error is left in the
 * runtime's last-error slot, as an unrelated caller's failed launch would leave it: the
 * next matmul call must still return TGEMM_OK, since every call of this library reports
 * only its own launches' results.  The pages have no counterpart.
 */
int tgemm_selftest_bad_launch(void* stream);

/*
 * tgemm_mma_rate -- measurement hook behind two design choices (the small-M tile width
 * and the 8-bit-activation variant); the pages have no counterpart.  One CTA per SM
 * issues `iters` back-to-back operations of one kind and writes the cycles they took to
 * out[cta] (device, 8-byte aligned, nout >= the SM count); read after synchronizing.
 *   mode 0: tcgen05.mma kind::f16 (f16 x f16 -> f32), M = 128, N = n, K = 16, A and B in
 *           shared memory;  1: the same with A in tensor memory;
 *   mode 2: tcgen05.mma kind::i8 (s8 x s8 -> s32), M = 128, N = n, K = 32, both in shared
 *           memory;
 *   mode 3: tcgen05.ld of 32 lanes x 16 columns per warp (4 warps), each waited for;
 *   mode 4: warp mma.sync m16n8k16 bf16 -> f32, 5: mma.sync m16n8k32 s8 -> s32, each of
 *           4 warps running 8 independent accumulator chains (`iters` per warp);
 *   modes 6-8: `iters` 128-k blocks of an 8-bit-activation pipeline: four kind::i8 MMAs
 *           (M = 128, N = 256) per block into one of two int32 accumulators, each block
 *           drained by 16 warps (64 columns each) into f32 running sums in registers
 *           (sum += d * float(int)); 6: MMAs and drains overlapped, int -> float by cvt;
 *           7: drains alone; 8: as 6 with the exponent-trick conversion; 9: as 8 and
 *           10: as 6, with packed f32x2 subtract and multiply-add.  n is ignored.
 * n: 16..256, a multiple of 16 (modes 0-2).  Operands are zeros (or TMEM contents); the
 * results are not read.
 */
int tgemm_mma_rate(int mode, int n, int iters, unsigned long long* out, int nout, void* stream);

/*
 * tgemm_gemv_plan -- introspection of the small-M streaming kernel's launch plan for a
 * matmul of format `fmt` (0 Q2_0, 1 4-bit) with M <= 16 tokens on a GPU of `sms` SMs:
 * plan[0..16] = token tiles of 8 (T), weights per pass over K, passes, grid (one CTA per
 * SM), ring slots, units of 128 along K, most 32-row tiles of a CTA, shared-memory bytes,
 * weight boxes (32 rows x 128 bytes) per ring slot, activation row stride, then the
 * offsets of the activations, correction sums, warp partial sums (two buffers), pass
 * partial sums, staged scales, ring and barriers in shared memory.  TGEMM_ETOOLARGE when no layout fits (the per-pass
 * kernel then serves the call).
 */
int tgemm_gemv_plan(int fmt, int M, int N, int K, int sms, int* plan);

/*
 * tgemm_workspace_size -- bytes of workspace the matmul `op` (TGEMM_OP_*) needs for
 * these sizes under the current path setting to run its fastest schedule (0 when it
 * needs none).  On the tensor-core path that schedule may split tiles between CTAs
 * when the tiles fill the SMs unevenly, and then the size includes f32 partial sums
 * (2 x 128 KB per CTA) and arrival counters; it depends on the current device's SM
 * count (148 is assumed when no device is visible).  r is ignored unless op is
 * TGEMM_OP_Q2_LORA.  Returns 0 for invalid arguments as well; the matmul call then
 * reports the argument error.
 */
size_t tgemm_workspace_size(int op, int M, int N, int K, int r);

/*
 * tgemm_workspace_size_min -- the smallest workspace the matmul accepts (0 when it
 * needs none).  With less than tgemm_workspace_size() bytes the call keeps whole tiles
 * per CTA; the results agree to f32 rounding of the partial sums.  Same arguments and
 * error behaviour as tgemm_workspace_size.
 */
size_t tgemm_workspace_size_min(int op, int M, int N, int K, int r);

/*
 * tgemm_tc_plan -- the schedule the tensor-core kernel uses for matmul `op` with these
 * sizes on a device of `sms` SMs, when the workspace has tgemm_workspace_size() bytes
 * (with only the minimum it keeps whole tiles: plan[3] = 0, plan[5] = 0, plan[7] = 0).
 * Host computation only; no device is touched.  K2 > 0 adds a second input of width K2
 * (op must be TGEMM_OP_Q2, as for tgemm_q2_dual); r as for tgemm_workspace_size.
 * A tile is 128 weight rows x 256 tokens; a unit is one of its 128-k stages (the
 * low-rank branch adds its own stages).  Tiles and units are numbered tile-major; tile t
 * covers tokens 256 (t % tiles_m) and rows 128 (t / tiles_m).  CTA c runs the split-region
 * units sk_t0 * ksteps + [c * upc, (c + 1) * upc) first, then the whole-tile units
 * [c * dpc, (c + 1) * dpc), both clipped to their region; a tile whose units are spread
 * over several CTAs is summed from their f32 partial sums in k order.
 *   plan[8] receives: tiles_m, num_tiles, ksteps, sk_t0, upc, dpc, grid (CTAs launched),
 *   split (1 when some tile is shared between CTAs).
 * Returns TGEMM_OK, or TGEMM_EINVAL for a NULL plan, sizes < 1, sms < 1 or an invalid op.
 */
int tgemm_tc_plan(int op, int M, int N, int K, int r, int K2, int sms, int* plan);

/*
 * tgemm_q2 -- y = x . W^T for Q2_0 weights, W = (q - 1) * d ("We're Teaching...", "The
 * lucky break that wasn't luck"; the ternary linears of "A Browser Tab Just Rendered
 * This Fox...", "The claim").  M <= 16 runs the small-M kernel, larger M the tensor-core
 * kernel (tgemm_set_path overrides this for tests).
 *   x [M][K] bf16 (16-byte aligned), wq [N][K/4] (16-byte aligned), d [N][K/128] f16
 *   (2-byte aligned), y [M][N] (16-byte aligned), out_dtype TGEMM_OUT_*.
 *   workspace: device memory of tgemm_workspace_size(TGEMM_OP_Q2, M, N, K, 0) bytes, or
 *   at least tgemm_workspace_size_min() (256-byte aligned; may be NULL when that is 0).
 *   The call overwrites it; calls sharing a workspace must not overlap on the GPU.
 *   Requires M, N >= 1, K % 128 == 0.
 *   Packed weights are read early: every matmul kernel starts loading wq and its scales
 *   (and the tensor-core kernel starts dequantizing them) before it waits for the kernels
 *   ahead of it on the stream (programmatic dependent launch), so that the fetch overlaps
 *   the end of those kernels.  wq and the
 *   scales must therefore not be written by a matmul call of this library that is still
 *   ahead on the stream.  Weights written by q2_pack, q4_pack or q2_from_gemlite (which
 *   let no later kernel start before they finish), by host copies or by other libraries'
 *   kernels are safe.  x is read only after that wait.
 */
int tgemm_q2(const uint16_t* x, const uint8_t* wq, const uint16_t* d, void* y, int M, int N,
             int K, int out_dtype, void* workspace, size_t ws_bytes, void* stream);

/*
 * tgemm_q2_lora -- y = x . W^T + (x . A^T) . B^T ("mindview-t2i-turbo", "One step").
 *   As tgemm_q2, plus a [r][K] bf16 (4-byte aligned) and b [N][r] bf16 (2-byte aligned),
 *   1 <= r <= 256, and workspace of tgemm_workspace_size(TGEMM_OP_Q2_LORA, M, N, K, r).
 *   The branch has no extra scale factor.  u = x . A^T is accumulated in f32; both
 *   paths feed it to the MMA as a bf16 pair (hi + lo) so that its rounding error stays
 *   near 2^-16 relative.  a and b are weights and are read early like wq (see tgemm_q2):
 *   neither may be written by a matmul call of this library still ahead on the stream.
 */
int tgemm_q2_lora(const uint16_t* x, const uint8_t* wq, const uint16_t* d, const uint16_t* a,
                  const uint16_t* b, int r, void* y, int M, int N, int K, int out_dtype,
                  void* workspace, size_t ws_bytes, void* stream);

/*
 * tgemm_q2_lora_bt -- tgemm_q2_lora with B given transposed: bt [r][N] bf16 (2-byte
 * aligned), element (i, n) = B[n][i].  The branches in the model file are stored as
 * <branch>.<matrix>.a and <branch>.<matrix>.bt ("mindview-t2i-turbo", "Running it"),
 * so they load without a transpose.  The same workspace as tgemm_q2_lora; the
 * result is bit-identical to tgemm_q2_lora on the transposed copy.
 */
int tgemm_q2_lora_bt(const uint16_t* x, const uint8_t* wq, const uint16_t* d, const uint16_t* a,
                     const uint16_t* bt, int r, void* y, int M, int N, int K, int out_dtype,
                     void* workspace, size_t ws_bytes, void* stream);

/*
 * tgemm_q2_noalloc -- tgemm_q2 for callers that cannot allocate device memory.
 *   The pages have no counterpart to this call; it exists for code that may not call
 *   cudaMalloc or any allocator: plugins inside hosts that own all device memory, code
 *   paths that run while a stream is being captured, real-time loops that must not
 *   allocate.  It computes exactly what tgemm_q2 computes (same kernels), but instead of
 *   a caller workspace it uses one scratch buffer compiled into the library: a
 *   file-scope device array of TGEMM_NOALLOC_SCRATCH_BYTES (40 MiB), which every GPU
 *   that loads the library holds until the process exits.
 *   Limit: the tensor-core path needs M*K*2 bytes of scratch (an f16 copy of x), so
 *   M*K may be at most 20 Mi elements (e.g. 1536 x 12288); larger problems return
 *   TGEMM_ETOOLARGE before launching anything.  The small-M path (M <= 16) needs none.
 *   The first call on a device looks up that device's address of the buffer
 *   (cudaGetSymbolAddress, with that device current); make that first call before any
 *   stream capture.  The address is kept per device and context: after a device reset
 *   (a new primary context, with a new context id) the next call looks it up again, so
 *   make that call before any capture too.  All calls share the one buffer and it keeps the last call's
 *   contents (nothing in it has to start at zero: every call rewrites what it reads).
 *   Calls that overlap on the GPU -- on different streams, or from different threads --
 *   race on the buffer: serialize them.  Arguments, layouts and errors as tgemm_q2.
 */
#define TGEMM_NOALLOC_SCRATCH_BYTES (40u * 1024u * 1024u)
int tgemm_q2_noalloc(const uint16_t* x, const uint8_t* wq, const uint16_t* d, void* y, int M,
                     int N, int K, int out_dtype, void* stream);

/*
 * tgemm_q2_dual -- y = x1 . W1^T + x2 . W2^T for Q2_0 weights: a projection whose input
 *   is two activations concatenated per token, split along its input axis into two
 *   matmuls that are summed ("We're Teaching Your Browser to Paint", section "The GPU
 *   driver, and the bug that looked like broken math", "Slice weights, not
 *   activations").  Both products accumulate into one f32 accumulator in one kernel (no
 *   intermediate y).
 *   x1 [M][K1] and x2 [M][K2] bf16 (16-byte aligned); wq1 [N][K1/4], d1 [N][K1/128] and
 *   wq2 [N][K2/4], d2 [N][K2/128] as for tgemm_q2; y [M][N] (16-byte aligned).
 *   Requires M, N >= 1, K1 and K2 multiples of 128.  Workspace of
 *   tgemm_q2_dual_workspace_size(M, N, K1, K2) bytes, or at least
 *   tgemm_q2_dual_workspace_size_min() (whole tiles per CTA); 256-byte aligned.
 */
int tgemm_q2_dual(const uint16_t* x1, const uint8_t* wq1, const uint16_t* d1, int K1,
                  const uint16_t* x2, const uint8_t* wq2, const uint16_t* d2, int K2, void* y,
                  int M, int N, int out_dtype, void* workspace, size_t ws_bytes, void* stream);
size_t tgemm_q2_dual_workspace_size(int M, int N, int K1, int K2);
size_t tgemm_q2_dual_workspace_size_min(int M, int N, int K1, int K2);

/*
 * tgemm_q4 -- y = x . W^T for 4-bit group weights, W = (q - z) * s with the codes unpacked
 * as in q4_pack ("You Can Now Just Ask...", "The bug that hid in one flipped bit";
 * "We're Teaching...", "What's left").  Dispatch as for tgemm_q2.
 *   x [M][K] bf16 (16-byte aligned), wq [N][K/2] (16-byte aligned), sz [N][K/64][2] f16
 *   (4-byte aligned), y [M][N] (16-byte aligned), workspace as for tgemm_q2 with
 *   TGEMM_OP_Q4.  Requires M, N >= 1, K % 64 == 0.  wq and sz are read before the wait for
 *   the kernels ahead on the stream, under the same rule as tgemm_q2.
 */
int tgemm_q4(const uint16_t* x, const uint8_t* wq, const uint16_t* sz, void* y, int M, int N,
             int K, int out_dtype, void* workspace, size_t ws_bytes, void* stream);

/* tgemm_strerror -- a static string describing a TGEMM_* status code. */
const char* tgemm_strerror(int status);

/*
 * tgemm_set_path -- choose which matmul kernel runs (TGEMM_PATH_*); returns the previous
 * setting, or TGEMM_EINVAL.  Process-wide; meant for tests and benchmarks.
 */
int tgemm_set_path(int path);

/*
 * tgemm_device_error -- synchronize the current device, copy its device error word
 * (TGEMM_DEVERR_* bits, accumulated since load or the last clear) to *bits, and clear
 * it if `clear` is nonzero.
 */
int tgemm_device_error(uint32_t* bits, int clear);

/* tgemm_version -- library version, major * 10000 + minor * 100 + patch. */
int tgemm_version(void);

/* ---- measurement hooks ------------------------------------------------------------ */
/* Kernel kinds for tgemm_profile_read. */
#define TGEMM_KIND_TC_Q2       0 /* tensor-core Q2_0 matmul kernel */
#define TGEMM_KIND_TC_Q2_LORA  1 /* tensor-core Q2_0 matmul + low-rank branch kernel */
#define TGEMM_KIND_TC_Q4       2 /* tensor-core 4-bit matmul kernel */
#define TGEMM_KIND_GEMV_Q2     3 /* small-M Q2_0 kernel (with or without the branch) */
#define TGEMM_KIND_GEMV_Q4     4 /* small-M 4-bit kernel */
#define TGEMM_KIND_PREP        5 /* activation conversion and u = x A^T kernels */
#define TGEMM_NUM_KINDS        6

/*
 * tgemm_profile_enable -- `kinds` is a bit mask of (1 << TGEMM_KIND_*): every subsequent
 * launch of a kernel kind whose bit is set records a pair of CUDA events around itself
 * on the call's stream (host cost: two event records per such launch; do not enable
 * while capturing a CUDA graph).  TGEMM_PROFILE_ALL enables every kind, 0 disables.
 * Returns the previous mask.
 */
#define TGEMM_PROFILE_ALL ((1 << TGEMM_NUM_KINDS) - 1)
int tgemm_profile_enable(int kinds);

/*
 * tgemm_profile_read -- wait for the recorded events of `kind` (TGEMM_KIND_*), store the
 * summed device time in *total_ms and the number of launches in *launches; forget them
 * if `reset` is nonzero.
 */
int tgemm_profile_read(int kind, double* total_ms, int64_t* launches, int reset);

/* tgemm_launch_count -- kernels launched by this library since it was loaded. */
int64_t tgemm_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* TGEMM_H */
