// tgemm.cu -- the C ABI of libtgemm.so: argument checks, workspace layout, dispatch.
//
// One translation unit (kernels are in the included .cuh files) so that every kernel
// sees the same device error word.  Built for sm_100a only.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>
#include <cstdio>
#include <mutex>
#include <type_traits>
#include <vector>

#include "../../include/tgemm.h"
#include "common.cuh"
#include "gemm_tc.cuh"
#include "prep.cuh"
#include "gemv.cuh"
#include "gemv_stream.cuh"
#include "mma_rate.cuh"
#include "pack.cuh"

namespace tgemm {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kSmallM = 16;

std::atomic<int> g_path{TGEMM_PATH_AUTO};

struct DeviceInfo {
  int checked = 0;  // 0 unknown, 1 ok, -1 wrong architecture
  int sms = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

int current_device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TGEMM_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return TGEMM_ECUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& di = g_dev[dev];
  if (di.checked == 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return TGEMM_ECUDA;
    di.checked = (major == 10 && minor == 0) ? 1 : -1;
    di.sms = sms;
  }
  if (di.checked < 0) return TGEMM_EARCH;
  *out = di;
  return TGEMM_OK;
}

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// ---- launch accounting and optional per-launch event timing ---------------------------

std::atomic<int64_t> g_launches{0};
std::atomic<int> g_profile{0};
struct ProfRecord {
  int kind;
  cudaEvent_t begin, end;
};
std::vector<ProfRecord> g_records;
std::vector<cudaEvent_t> g_event_pool;
std::mutex g_prof_mu;

cudaEvent_t take_event() {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Launch `kernel` on `st` with programmatic stream serialization: it may be scheduled
// while the previous kernel on the stream is finishing (every kernel of the library
// waits for its predecessors with griddepcontrol.wait before touching global memory).
template <typename... KArgs, typename... Args>
cudaError_t pdl_launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Run `launch_fn` (one kernel launch on `st`, returning its cudaError_t), count it, and
// time it when profiling.
template <typename Fn>
int launch(int kind, cudaStream_t st, Fn&& launch_fn) {
  cudaEvent_t b = nullptr, e = nullptr;
  if (g_profile.load(std::memory_order_relaxed) & (1 << kind)) {
    b = take_event();
    e = take_event();
    if (b && e) cudaEventRecord(b, st);
  }
  // The launch's own return value is its status.  The runtime's last-error slot is left
  // alone: reading it (cudaGetLastError) would clear, and blame this call for, an error
  // that an earlier, unrelated launch left there.
  const cudaError_t le = launch_fn();
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (b && e) {
    cudaEventRecord(e, st);
    std::lock_guard<std::mutex> lock(g_prof_mu);
    g_records.push_back({kind, b, e});
  }
  return le == cudaSuccess ? TGEMM_OK : TGEMM_ECUDA;
}

int grid_for(int64_t work_items, int per_block, int sms) {
  int64_t g = (work_items + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

// ---- TMA descriptors -------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

int encoder(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  std::call_once(g_encode_once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  if (!g_encode) return TGEMM_ECUDA;
  *fn = g_encode;
  return TGEMM_OK;
}

// 2-D row-major tensor [rows][cols] of `esize`-byte elements, box [box_rows][box_cols].
int make_map_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int esize,
                uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows,
                CUtensorMapSwizzle swizzle) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  if (int st = encoder(&enc)) return st;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * static_cast<uint64_t>(esize)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? TGEMM_OK : TGEMM_ECUDA;
}

// ---- kernel attribute setup (once per instantiation) ------------------------------------

template <int FMT, bool LORA, bool DUAL, bool HYB>
int tc_prepare() {
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    err = cudaFuncSetAttribute(tc_gemm_kernel<FMT, LORA, DUAL, HYB>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               TcFmt<FMT>::kSmemBytes);
  });
  return err == cudaSuccess ? TGEMM_OK : TGEMM_ECUDA;
}

// ---- workspace layout -----------------------------------------------------------------

int choose_path(int M) {
  const int p = g_path.load();
  if (p == TGEMM_PATH_SMALL_M || p == TGEMM_PATH_SMALL_M_PASS || p == TGEMM_PATH_SMALL_M_STREAM)
    return TGEMM_PATH_SMALL_M;
  if (p == TGEMM_PATH_TENSOR) return TGEMM_PATH_TENSOR;
  return M <= kSmallM ? TGEMM_PATH_SMALL_M : TGEMM_PATH_TENSOR;
}

struct LoraDims {
  int R;       // round_up(r, 16)
  int wcat;    // width of [u_hi | u_lo | 0], a multiple of the tensor-core stage (128)
  int L;       // pipeline stages for the branch
  int rpad;    // round_up(r, 64): columns of the partial sums
  int slices;  // K slices of the partial sums
};

LoraDims lora_dims(int r, int K) {
  LoraDims d;
  d.R = (r + 15) / 16 * 16;
  d.wcat = (2 * d.R + kTcBK - 1) / kTcBK * kTcBK;
  d.L = d.wcat / kTcBK;
  d.rpad = (r + 63) / 64 * 64;
  d.slices = (K + kLoraKc - 1) / kLoraKc;
  return d;
}

// Tensor-core schedule (see gemm_tc.cuh): units (tile, 128-k stage), tile-major, in a
// whole-tile region of floor(tiles / SMs) tiles per CTA and a split region where the
// remaining tiles' units are cut into equal contiguous ranges, one per CTA.  It is the
// split form only when it saves more than the split tiles' charge over whole tiles alone
// (a larger charge when the CTAs also run whole tiles).
constexpr int kDefaultSms = 148;    // sizes workspaces when no device is visible (B200)
// Units a pure-split schedule is charged for its partial sums and fix-ups, which come at
// the end of every CTA's work: measured against whole tiles, 1536 tokens x 3072 x
// (3072 + 12288) ran 120 us split against 105 us whole (117 + 2 units against 120), and
// 256 x 9216 x 3072 32 us against 30 us (12 against 24 units), while the 4-bit encoder
// shapes stayed faster split (40 against 46 us at 21 against 40 units).
constexpr int kSplitPenalty = 13;
// Next to whole tiles a CTA's split share costs more: writing its partial sums and fixing
// up shared tiles keeps the epilogue warps from draining the following whole tile, which
// stalls the MMAs (measured: 4096 tokens x 9216 x 3072 ran 6 % slower split than whole at
// a 2-unit charge, 1280 tokens with the r = 64 branch ran 5 % faster split).
constexpr int kHybridPenalty = 8;
constexpr int kMaxShare = 4;        // CTAs that may share a split tile next to whole tiles

struct TcSchedule {
  int ksteps = 0, tiles_m = 0, num_tiles = 0, units = 0, grid = 0;
  int sk_t0 = 0;  // first tile of the split region
  int upc = 0;    // split-region units per CTA
  int dpc = 0;    // whole-tile units per CTA before the split region (0: none)
  bool split = false;
};

// Whole tiles only: ceil(tiles / CTAs) per CTA, expressed as a split region of whole tiles.
void tc_schedule_whole(TcSchedule& s, int sms) {
  s.split = false;
  s.sk_t0 = 0;
  s.dpc = 0;
  s.upc = (s.num_tiles + sms - 1) / sms * s.ksteps;
  s.grid = (s.units + s.upc - 1) / s.upc;
}

TcSchedule tc_schedule(int M, int N, int K, int kt_lora, int sms) {
  TcSchedule s;
  s.ksteps = (K + kTcBK - 1) / kTcBK + kt_lora;
  s.tiles_m = (M + kTcTok - 1) / kTcTok;
  s.num_tiles = s.tiles_m * ((N + kTcRows - 1) / kTcRows);
  s.units = s.num_tiles * s.ksteps;
  tc_schedule_whole(s, sms);
  const int whole = s.upc;                       // the longest CTA's units, whole tiles
  int wf = s.num_tiles / sms;                    // whole tiles every CTA gets
  if (wf * sms == s.num_tiles) return s;         // the tiles fill the SMs evenly
  // A few remainder tiles cut over all CTAs would each be summed from many partial sums
  // by one CTA; give the split region one more wave of tiles instead.
  if (wf > 0 && (s.num_tiles - wf * sms) * kMaxShare < sms) --wf;
  const int sk_t0 = wf * sms;
  const int upc = ((s.num_tiles - sk_t0) * s.ksteps + sms - 1) / sms;
  if (wf * s.ksteps + upc + (wf > 0 ? kHybridPenalty : kSplitPenalty) >= whole) return s;
  s.split = true;
  s.sk_t0 = sk_t0;
  s.upc = upc;
  s.dpc = wf * s.ksteps;
  s.grid = wf > 0 ? sms : ((s.units + upc - 1) / upc);
  return s;
}

int sms_for_sizing() {
  DeviceInfo di;
  if (current_device_info(&di) == TGEMM_OK && di.sms > 0) return di.sms;
  return kDefaultSms;
}

struct Workspace {
  size_t x16 = 0, x16_bytes = 0;    // f16 activations (tensor-core path)
  size_t ucat = 0, ucat_bytes = 0;  // [u_hi | u_lo] (tensor-core path)
  size_t u32 = 0, u32_bytes = 0;    // f32 u (small-M path)
  size_t part = 0, part_bytes = 0;  // f32 partial sums of u
  size_t slots = 0, slots_bytes = 0;  // split tiles: f32 partial sums, 2 per CTA
  size_t cnt = 0, cnt_bytes = 0;      // split tiles: arrival counters
  size_t total = 0;
  size_t total_whole = 0;           // the same without the split-tile part
};

// K2 > 0: a second input of width K2 (a projection split along its input axis).
Workspace workspace_layout(int op, int M, int N, int K, int r, int path, int sms, int K2 = 0) {
  Workspace w;
  size_t off = 0;
  const bool lora = op == TGEMM_OP_Q2_LORA;
  if (path == TGEMM_PATH_TENSOR) {
    w.x16 = off;
    w.x16_bytes = static_cast<size_t>(M) * (K + K2) * 2;
    off = round_up(off + w.x16_bytes, 256);
    if (lora) {
      w.ucat = off;
      w.ucat_bytes = static_cast<size_t>(M) * lora_dims(r, K).wcat * 2;
      off = round_up(off + w.ucat_bytes, 256);
    }
  } else if (lora) {
    w.u32 = off;
    w.u32_bytes = static_cast<size_t>(M) * r * 4;
    off = round_up(off + w.u32_bytes, 256);
  }
  if (lora && path == TGEMM_PATH_TENSOR) {
    const LoraDims ld = lora_dims(r, K);
    w.part = off;
    w.part_bytes = static_cast<size_t>(ld.slices) * M * ld.rpad * 4;
    off = round_up(off + w.part_bytes, 256);
  }
  w.total_whole = off;
  if (path == TGEMM_PATH_TENSOR) {
    const TcSchedule sc = tc_schedule(M, N, K + K2, lora ? lora_dims(r, K).L : 0, sms);
    if (sc.split) {
      w.slots = off;
      w.slots_bytes = static_cast<size_t>(2) * sc.grid * kTcSlotFloats * 4;
      off = round_up(off + w.slots_bytes, 256);
      w.cnt = off;
      w.cnt_bytes = static_cast<size_t>(sc.num_tiles - sc.sk_t0) * kTcEpiWarps * 4;
      off = round_up(off + w.cnt_bytes, 256);
    }
  }
  w.total = off;
  return w;
}

// Small-M path: u = x A^T into u32 (f32 [M][r]), one launch.
int launch_lora_down_small(const uint16_t* x, const uint16_t* la, int M, int K, int r, float* u32,
                           cudaStream_t st) {
  const dim3 grid((r + 7) / 8, (M + 15) / 16);
  return launch(TGEMM_KIND_PREP, st, [&] {
    if (aligned(la, 8))
      return pdl_launch(lora_down_small_kernel<true>, grid, kLdWarps * 32, 0, st, x, la, M, K, r, u32);
    return pdl_launch(lora_down_small_kernel<false>, grid, kLdWarps * 32, 0, st, x, la, M, K, r, u32);
  });
}

int prep_lora_prepare() {
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    err = cudaFuncSetAttribute(prep_lora_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kPlSmemBytes);
  });
  return err == cudaSuccess ? TGEMM_OK : TGEMM_ECUDA;
}

template <int FMT, int T, bool LORA, bool DUAL = false>
int gemv_prepare() {
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    err = cudaFuncSetAttribute(gemv_kernel<FMT, T, LORA, DUAL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kGvXBudget);
  });
  return err == cudaSuccess ? TGEMM_OK : TGEMM_ECUDA;
}

// ---- small-M streaming kernel: plan and launch ------------------------------------------

constexpr int kGsSmemMax = 232448;  // dynamic shared memory a CTA may use on sm_100
constexpr int kGsSmemHalf = 115712; // the most each of two CTAs on one SM may use

struct GsPlan {
  GsParams p;
  int smem = 0;
  bool ok = false;
};

// Shared-memory layout of the streaming kernel for `passes` passes over K and `S` ring
// slots; fills p and returns the bytes.
size_t gs_layout(GsParams& p, int fmt, int T, int passes, int S) {
  const int upass = (p.U + passes - 1) / passes;
  const int n8 = (p.N + 7) / 8;
  p.kp = upass * kGsUnit;
  p.passes = (p.U + upass - 1) / upass;
  p.j_max = (8 * ((n8 + p.grid - 1) / p.grid) + kGsRows - 1) / kGsRows;
  p.S = S;
  p.nbox = (p.kp / (fmt == 0 ? 4 : 2) + 127) / 128;
  p.xs_stride = p.kp * 2 + 16;  // 16 modulo 128: ldmatrix rows hit distinct banks
  size_t off = 0;
  p.off_x = 0;
  off += static_cast<size_t>(p.M) * p.xs_stride;  // the M real token rows
  off = round_up(off, 16);
  p.off_corr = static_cast<int>(off);
  off += static_cast<size_t>(upass) * (fmt == 0 ? 1 : 2) * 16 * 4;
  off = round_up(off, 16);
  p.off_red = static_cast<int>(off);
  off += static_cast<size_t>(2) * kGsWarps * 32 * 8 * T * 4;  // two buffers
  off = round_up(off, 16);
  p.off_acc = static_cast<int>(off);
  if (p.passes > 1) off += static_cast<size_t>(p.j_max) * kGsRows * 8 * T * 4;
  off = round_up(off, 16);
  p.off_sc = static_cast<int>(off);  // every scale of the CTA's rows: Q2 d, 4-bit (s, z)
  off += static_cast<size_t>(p.j_max) * kGsRows * p.U * (fmt == 0 ? 2 : 8);
  off = round_up(off, 1024);
  p.off_ring = static_cast<int>(off);
  off += static_cast<size_t>(S) * p.nbox * kGsBoxBytes;
  off = round_up(off, 8);
  p.off_bar = static_cast<int>(off);
  off += static_cast<size_t>(2 * S) * 8 + 8;
  off += 1024;  // slack: the kernel aligns its shared memory to 1024 bytes
  return off;
}

// Whether two CTAs of the one-token-tile streaming kernel fit on an SM with `smem` bytes
// each (true without a device: the layout already fits half the shared memory).
bool gs_two_fit(int fmt, int smem) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return true;
  int n = 0;
  const cudaError_t e = fmt == 0
      ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gemv_stream_kernel<0, 1>, kGsThreads, smem)
      : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gemv_stream_kernel<1, 1>, kGsThreads, smem);
  if (e != cudaSuccess) {
    cudaGetLastError();  // the query's own error, not a pending one of another call
    return false;
  }
  return n >= 2;
}

// One CTA per SM; the fewest passes over K (each at most 4096 weights, the activations of
// a pass staged whole) whose layout fits with at least 2 ring slots, and up to 4 slots.
GsPlan gs_plan(int fmt, const uint16_t* x, const uint8_t* wq, const uint16_t* scales, void* y,
               int M, int N, int K, int out_f32, int sms) {
  GsPlan best;
  if (M < 1 || M > 16) return best;
  const int T = M <= 8 ? 1 : 2;
  GsParams p = {};
  p.x = x;
  p.wq = wq;
  p.scales = scales;
  p.y = y;
  p.M = M;
  p.N = N;
  p.K = K;
  p.out_f32 = out_f32;
  p.U = (K + kGsUnit - 1) / kGsUnit;
  const int min_passes = (p.U + kGsMaxUW * kGsWarps - 1) / (kGsMaxUW * kGsWarps);
  // up to 8 tokens, two CTAs per SM when a one-pass layout fits in half the shared memory
  // (and, with a device current, the occupancy calculator confirms two fit)
  for (int per_sm = T == 1 ? 2 : 1; per_sm >= 1; --per_sm) {
    const int limit = per_sm == 2 ? kGsSmemHalf : kGsSmemMax;
    p.grid = per_sm * sms;
    for (int passes = min_passes; passes <= (per_sm == 2 ? min_passes : p.U); ++passes) {
      for (int S = 4; S >= 2; --S) {
        GsParams q = p;
        const size_t bytes = gs_layout(q, fmt, T, passes, S);
        if (bytes > static_cast<size_t>(limit)) continue;
        if (per_sm == 2 && !gs_two_fit(fmt, static_cast<int>(bytes))) continue;
        best.p = q;
        best.smem = static_cast<int>(bytes);
        best.ok = true;
        return best;
      }
    }
  }
  return best;
}

template <int FMT, int T>
int launch_gemv_stream(const GsPlan& pl, cudaStream_t st) {
  // packed weights as a [N][row bytes] u8 tensor, boxes of 32 rows x 128 bytes, 128-byte swizzle
  CUtensorMap tm_w;
  const uint64_t row_bytes = FMT == 0 ? static_cast<uint64_t>(pl.p.K) / 4 : static_cast<uint64_t>(pl.p.K) / 2;
  if (int e = make_map_2d(&tm_w, pl.p.wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, row_bytes, pl.p.N, 128,
                          kGsRows, CU_TENSOR_MAP_SWIZZLE_128B))
    return e;
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    err = cudaFuncSetAttribute(gemv_stream_kernel<FMT, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kGsSmemMax);
  });
  if (err != cudaSuccess) return TGEMM_ECUDA;
  return launch(FMT == 0 ? TGEMM_KIND_GEMV_Q2 : TGEMM_KIND_GEMV_Q4, st, [&] {
    return pdl_launch(gemv_stream_kernel<FMT, T>, dim3(static_cast<unsigned>(pl.p.grid)), kGsThreads,
                      static_cast<size_t>(pl.smem), st, tm_w, pl.p);
  });
}

// The streaming kernel when it applies (M <= 16, one input, no branch, a layout that fits)
// and is the faster form; returns 1 when it does not apply.  Measured (chained calls over
// weights larger than L2): it beats the per-pass kernel for up to 8 tokens with all of K
// in one pass on the large linears (M = 1: 12288 x 3072 8.5 against 10.1 us, 21504 x 3072
// 11.7 against 16.8 us, 4-bit 9728 x 2560 9.3 against 10.4 us), and loses on 3072 x 3072
// (5.6 against 3.1 us) and with several passes; at 9..16 tokens the two are close.
int try_gemv_stream(int fmt, const uint16_t* x, const uint8_t* wq, const uint16_t* scales, void* y,
                    int M, int N, int K, int out_f32, int sms, cudaStream_t st) {
  const int path = g_path.load();
  if (path == TGEMM_PATH_SMALL_M_PASS || M > 16) return 1;
  const GsPlan pl = gs_plan(fmt, x, wq, scales, y, M, N, K, out_f32, sms);
  if (!pl.ok) return 1;
  if (path != TGEMM_PATH_SMALL_M_STREAM && (M > 8 || pl.p.passes > 1 || N < 6144)) return 1;
  const bool t1 = M <= 8;
  if (fmt == 0) return t1 ? launch_gemv_stream<0, 1>(pl, st) : launch_gemv_stream<0, 2>(pl, st);
  return t1 ? launch_gemv_stream<1, 1>(pl, st) : launch_gemv_stream<1, 2>(pl, st);
}

// One small-M launch: T token tiles of 8 per pass over the weights.
template <int FMT, int T, bool LORA, bool DUAL>
int launch_gemv(int grid, size_t smem, cudaStream_t st, const uint16_t* x, const uint8_t* wq,
                const uint16_t* scales, void* y, int M, int N, int K, int out_f32, const float* u32,
                const uint16_t* lb, int r, int lb_sn, int lb_si, int kp, const uint16_t* x2,
                const uint8_t* wq2, const uint16_t* d2, int K2) {
  if (int e = gemv_prepare<FMT, T, LORA, DUAL>()) return e;
  return launch(FMT == 0 ? TGEMM_KIND_GEMV_Q2 : TGEMM_KIND_GEMV_Q4, st, [&] {
    return pdl_launch(gemv_kernel<FMT, T, LORA, DUAL>, grid, 256, smem, st, x, wq, scales, y, M, N, K,
                      out_f32, u32, lb, r, lb_sn, lb_si, kp, x2, wq2, d2, K2);
  });
}

// ---- the matmul driver ---------------------------------------------------------------

// The optional second input of a projection split along its input axis (Q2 only).
struct SecondInput {
  const uint16_t* x = nullptr;
  const uint8_t* wq = nullptr;
  const uint16_t* d = nullptr;
  int K = 0;
};

// lb_t: the branch's B is given transposed, [r][N] instead of [N][r].
int run_gemm(int fmt, const uint16_t* x, const uint8_t* wq, const uint16_t* scales,
             const uint16_t* la, const uint16_t* lb, int r, void* y, int M, int N, int K,
             int out_dtype, void* workspace, size_t ws_bytes, void* stream,
             const SecondInput& in2 = SecondInput(), bool lb_t = false) {
  const bool lora = la != nullptr;
  const bool dual = in2.K > 0;
  const int K2 = in2.K;
  const int op = fmt == 1 ? TGEMM_OP_Q4 : (lora ? TGEMM_OP_Q2_LORA : TGEMM_OP_Q2);
  const int kblock = fmt == 0 ? 128 : 64;
  if (!x || !wq || !scales || !y) return TGEMM_EINVAL;
  if (M < 1 || N < 1 || K < kblock || K % kblock) return TGEMM_EINVAL;
  if (out_dtype != TGEMM_OUT_F32 && out_dtype != TGEMM_OUT_BF16) return TGEMM_EINVAL;
  if (lora && (!lb || r < 1 || r > 256)) return TGEMM_EINVAL;
  if (!aligned(x, 16) || !aligned(wq, 16) || !aligned(y, 16)) return TGEMM_EALIGN;
  if (!aligned(scales, fmt == 0 ? 2 : 4)) return TGEMM_EALIGN;
  if (lora && (!aligned(la, 4) || !aligned(lb, 2))) return TGEMM_EALIGN;
  if (dual) {
    if (fmt != 0 || lora || !in2.x || !in2.wq || !in2.d || K2 < 128 || K2 % 128) return TGEMM_EINVAL;
    if (!aligned(in2.x, 16) || !aligned(in2.wq, 16) || !aligned(in2.d, 2)) return TGEMM_EALIGN;
  }
  const int lb_sn = lb_t ? 1 : r, lb_si = lb_t ? N : 1;  // B's element strides
  const int path = choose_path(M);
  // the required size does not depend on the device (only the optional split-tile part does)
  const size_t required = workspace_layout(op, M, N, K, r, path, kDefaultSms, K2).total_whole;
  if (required > 0) {
    if (!workspace || ws_bytes < required) return TGEMM_EWORKSPACE;
    if (!aligned(workspace, 256)) return TGEMM_EALIGN;
  }
  DeviceInfo di;
  if (int st = current_device_info(&di)) return st;
  const Workspace wl = workspace_layout(op, M, N, K, r, path, di.sms, K2);
  // split tiles only when the workspace has room for their partial sums
  const bool split_ok = wl.slots_bytes > 0 && ws_bytes >= wl.total;
  const cudaStream_t st = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int out_f32 = out_dtype == TGEMM_OUT_F32 ? 1 : 0;
  const LoraDims ld = lora ? lora_dims(r, K) : LoraDims{0, 0, 0, 0, 0};
  float* part = lora ? reinterpret_cast<float*>(ws + wl.part) : nullptr;

  if (path == TGEMM_PATH_SMALL_M) {
    float* u32 = nullptr;
    if (lora) {
      u32 = reinterpret_cast<float*>(ws + wl.u32);
      if (int e = launch_lora_down_small(x, la, M, K, r, u32, st)) return e;
    }
    if (!lora && !dual) {
      const int e = try_gemv_stream(fmt, x, wq, scales, y, M, N, K, out_f32, di.sms, st);
      if (e <= 0) return e;  // launched (TGEMM_OK) or failed
    }
    const int grid = (N + kGvRows - 1) / kGvRows;
    const int mrows = M < 16 ? M : 16;
    const bool t1 = M <= 8;  // one token tile of 8, else two
    const int T = t1 ? 1 : 2, rl = lora ? r : 0;
    const int kp = gemv_pass_k(fmt, mrows, K > K2 ? K : K2, T, gemv_lora_bytes(T, rl));
    const size_t smem = gemv_smem_bytes(mrows, kp, T, rl);
    const uint16_t* x2 = in2.x;
    const uint8_t* wq2 = in2.wq;
    const uint16_t* d2 = in2.d;
    if (fmt == 0 && lora)
      return t1 ? launch_gemv<0, 1, true, false>(grid, smem, st, x, wq, scales, y, M, N, K, out_f32, u32, lb, r, lb_sn, lb_si, kp, nullptr, nullptr, nullptr, 0)
                : launch_gemv<0, 2, true, false>(grid, smem, st, x, wq, scales, y, M, N, K, out_f32, u32, lb, r, lb_sn, lb_si, kp, nullptr, nullptr, nullptr, 0);
    if (fmt == 0 && dual)
      return t1 ? launch_gemv<0, 1, false, true>(grid, smem, st, x, wq, scales, y, M, N, K, out_f32, nullptr, nullptr, 0, 0, 0, kp, x2, wq2, d2, K2)
                : launch_gemv<0, 2, false, true>(grid, smem, st, x, wq, scales, y, M, N, K, out_f32, nullptr, nullptr, 0, 0, 0, kp, x2, wq2, d2, K2);
    if (fmt == 0)
      return t1 ? launch_gemv<0, 1, false, false>(grid, smem, st, x, wq, scales, y, M, N, K, out_f32, nullptr, nullptr, 0, 0, 0, kp, nullptr, nullptr, nullptr, 0)
                : launch_gemv<0, 2, false, false>(grid, smem, st, x, wq, scales, y, M, N, K, out_f32, nullptr, nullptr, 0, 0, 0, kp, nullptr, nullptr, nullptr, 0);
    return t1 ? launch_gemv<1, 1, false, false>(grid, smem, st, x, wq, scales, y, M, N, K, out_f32, nullptr, nullptr, 0, 0, 0, kp, nullptr, nullptr, nullptr, 0)
              : launch_gemv<1, 2, false, false>(grid, smem, st, x, wq, scales, y, M, N, K, out_f32, nullptr, nullptr, 0, 0, 0, kp, nullptr, nullptr, nullptr, 0);
  }

  // ---- tensor-core path
  TcSchedule sc = tc_schedule(M, N, K + K2, lora ? ld.L : 0, di.sms);
  if (sc.split && !split_ok) {
    // whole tiles per CTA (the workspace holds no partial-sum slots)
    tc_schedule_whole(sc, di.sms);
  }
  int* cnt = sc.split ? reinterpret_cast<int*>(ws + wl.cnt) : nullptr;
  const int ncnt = sc.split ? (sc.num_tiles - sc.sk_t0) * kTcEpiWarps : 0;
  uint16_t* x16 = reinterpret_cast<uint16_t*>(ws + wl.x16);
  uint16_t* ucat = nullptr;
  if (lora) {
    // one pass over x: the f16 copy and the slices of u = x A^T; then u -> [u_hi | u_lo]
    ucat = reinterpret_cast<uint16_t*>(ws + wl.ucat);
    if (int e = prep_lora_prepare()) return e;
    const dim3 grid((M + kPlTok - 1) / kPlTok, ld.slices);
    const int a_vec = aligned(la, 16) ? 1 : 0;
    if (int e = launch(TGEMM_KIND_PREP, st, [&] {
          return pdl_launch(prep_lora_kernel<0>, grid, 256, kPlSmemBytes, st, x, x16, la, M, K, r, ld.rpad, part,
                                                               cnt, ncnt, a_vec);
        }))
      return e;
    const int fgrid = grid_for(static_cast<int64_t>(M) * ld.wcat, 256, di.sms);
    if (int e = launch(TGEMM_KIND_PREP, st, [&] {
          return pdl_launch(lora_finalize_kernel, fgrid, 256, 0, st, part, ld.slices, M, r, ld.rpad, ld.R,
                            ld.wcat, ucat);
        }))
      return e;
  } else {
    const int64_t ngroups = static_cast<int64_t>(M) * K / 16;
    const int pgrid = grid_for(ngroups, 256, di.sms);
    if (int e = launch(TGEMM_KIND_PREP, st, [&] {
          if (fmt == 0)
            return pdl_launch(prep_x16_kernel<0>, pgrid, 256, 0, st, x, x16, ngroups, cnt, ncnt);
          else
            return pdl_launch(prep_x16_kernel<1>, pgrid, 256, 0, st, x, x16, ngroups, cnt, ncnt);
        }))
      return e;
  }
  // the second input's f16 copy follows the first's in the workspace
  uint16_t* x16b = x16 + static_cast<int64_t>(M) * K;
  if (dual) {
    const int64_t ngroups2 = static_cast<int64_t>(M) * K2 / 16;
    const int pgrid2 = grid_for(ngroups2, 256, di.sms);
    if (int e = launch(TGEMM_KIND_PREP, st, [&] {
          return pdl_launch(prep_x16_kernel<0>, pgrid2, 256, 0, st, in2.x, x16b, ngroups2,
                            static_cast<int*>(nullptr), 0);
        }))
      return e;
  }
  CUtensorMap tm_x, tm_u;
  if (int e = make_map_2d(&tm_x, x16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, K, M, kTcBox, kTcTok,
                          CU_TENSOR_MAP_SWIZZLE_128B))
    return e;
  if (lora) {
    if (int e = make_map_2d(&tm_u, ucat, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ld.wcat, M, kTcBox,
                            kTcTok, CU_TENSOR_MAP_SWIZZLE_128B))
      return e;
  } else {
    tm_u = tm_x;  // unused
  }
  // packed weights as a [N][row bytes] u8 tensor, boxes of one stage x 128 rows
  CUtensorMap tm_w;
  const uint64_t wq_row_bytes = fmt == 0 ? static_cast<uint64_t>(K) / 4 : static_cast<uint64_t>(K) / 2;
  if (int e = make_map_2d(&tm_w, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, wq_row_bytes, N,
                          fmt == 0 ? TcFmt<0>::kWqRowBytes : TcFmt<1>::kWqRowBytes, kTcRows,
                          CU_TENSOR_MAP_SWIZZLE_NONE))
    return e;
  CUtensorMap tm_x2 = tm_x, tm_w2 = tm_w;  // unused with one input
  if (dual) {
    if (int e = make_map_2d(&tm_x2, x16b, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, K2, M, kTcBox, kTcTok,
                            CU_TENSOR_MAP_SWIZZLE_128B))
      return e;
    if (int e = make_map_2d(&tm_w2, in2.wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1,
                            static_cast<uint64_t>(K2) / 4, N, TcFmt<0>::kWqRowBytes, kTcRows,
                            CU_TENSOR_MAP_SWIZZLE_NONE))
      return e;
  }
  TcParams p;
  // bf16 Q2 output of whole tiles goes through the output boxes when 4 rows are 8 bytes
  p.y_box = fmt == 0 && !out_f32 && N % 4 == 0 ? 1 : 0;
  p.M = M;
  p.N = N;
  p.K = K;
  p.K2 = K2;
  p.scales2 = in2.d;
  p.tiles_m = sc.tiles_m;
  p.num_tiles = sc.num_tiles;
  p.kt1 = (K + kTcBK - 1) / kTcBK;
  p.kt_main = p.kt1 + (K2 + kTcBK - 1) / kTcBK;
  p.kt_lora = lora ? ld.L : 0;
  p.ksteps = sc.ksteps;
  p.sk_t0 = sc.sk_t0;
  p.upc = sc.upc;
  p.dpc = sc.dpc;
  p.units = sc.units;
  p.lora_mmas = lora ? 2 * ld.R / 16 : 0;
  p.R = ld.R;
  p.r = r;
  p.out_f32 = out_f32;
  p.wq = wq;
  p.scales = scales;
  p.lb = lb;
  p.lb_sn = lb_sn;
  p.lb_si = lb_si;
  p.y = y;
  p.part = sc.split ? reinterpret_cast<float*>(ws + wl.slots) : nullptr;
  p.cnt = cnt;
  const int grid = sc.grid;
  // one instantiation per (format, branch, second input, whole-tile region)
  auto run_tc = [&](auto fmt_c, auto lora_c, auto dual_c, auto hyb_c, int kind) -> int {
    constexpr int kF = decltype(fmt_c)::value;
    constexpr bool kL = decltype(lora_c)::value, kD = decltype(dual_c)::value;
    constexpr bool kH = decltype(hyb_c)::value;
    if (int e = tc_prepare<kF, kL, kD, kH>()) return e;
    return launch(kind, st, [&] {
      return pdl_launch(tc_gemm_kernel<kF, kL, kD, kH>, grid, kTcThreads, TcFmt<kF>::kSmemBytes, st,
                        tm_x, tm_u, tm_w, tm_x2, tm_w2, p);
    });
  };
  using F0 = std::integral_constant<int, 0>;
  using F1 = std::integral_constant<int, 1>;
  using On = std::true_type;
  using Off = std::false_type;
  const bool hyb = sc.dpc > 0;
  if (dual)
    return hyb ? run_tc(F0{}, Off{}, On{}, On{}, TGEMM_KIND_TC_Q2) : run_tc(F0{}, Off{}, On{}, Off{}, TGEMM_KIND_TC_Q2);
  if (fmt == 0 && !lora)
    return hyb ? run_tc(F0{}, Off{}, Off{}, On{}, TGEMM_KIND_TC_Q2) : run_tc(F0{}, Off{}, Off{}, Off{}, TGEMM_KIND_TC_Q2);
  if (fmt == 0)
    return hyb ? run_tc(F0{}, On{}, Off{}, On{}, TGEMM_KIND_TC_Q2_LORA)
               : run_tc(F0{}, On{}, Off{}, Off{}, TGEMM_KIND_TC_Q2_LORA);
  return hyb ? run_tc(F1{}, Off{}, Off{}, On{}, TGEMM_KIND_TC_Q4) : run_tc(F1{}, Off{}, Off{}, Off{}, TGEMM_KIND_TC_Q4);
}

// Failure-detection self test: one CTA waits on an mbarrier phase that nothing ever
// completes.  The library's bounded wait gives up after kWaitLimitNs, records
// TGEMM_DEVERR_TIMEOUT in the device error word and returns; the context stays usable.
__global__ void __launch_bounds__(32) selftest_wait_kernel() {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_word;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_word = 0u;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_trigger_and_wait();
  mbar_wait(smem_u32(&bar), 0u, &abort_word);  // no thread arrives on `bar`
}

__global__ void selftest_noop_kernel() {}

}  // namespace
}  // namespace tgemm

// ---- scratch for tgemm_q2_noalloc ------------------------------------------------------
// Compiled into the library so that tgemm_q2_noalloc never allocates.  In host code the
// name is only a stand-in for the symbol; the device address comes from
// cudaGetSymbolAddress, once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[TGEMM_NOALLOC_SCRATCH_BYTES];

namespace tgemm {
namespace {
// The buffer's device address, looked up once per device and context.  The address
// belongs to the context the module was loaded in: after a device reset the primary
// context (and the module) is created anew, with a new context id, and the address is
// looked up again.
struct NoallocScratch {
  unsigned long long ctx_id = 0;
  void* ptr = nullptr;
};
NoallocScratch g_noalloc[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// The current context's unique id (never reused within a process).
int current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(f);
  });
  if (!get_current || !get_id) return TGEMM_ECUDA;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return TGEMM_ECUDA;
  if (get_id(ctx, id) != CUDA_SUCCESS) return TGEMM_ECUDA;
  return TGEMM_OK;
}

int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TGEMM_ECUDA;
  // No context may be current yet (the runtime creates the primary context lazily);
  // then the lookup below creates it, and its id is read afterwards.
  unsigned long long id = 0;
  const bool have_id = current_context_id(&id) == TGEMM_OK;
  std::lock_guard<std::mutex> lock(g_mu);
  NoallocScratch& s = g_noalloc[dev];
  if (!have_id || s.ptr == nullptr || s.ctx_id != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return TGEMM_ECUDA;
    if (!have_id && current_context_id(&id) != TGEMM_OK) return TGEMM_ECUDA;
    s.ptr = p;
    s.ctx_id = id;
  }
  *out = s.ptr;
  return TGEMM_OK;
}
}  // namespace
}  // namespace tgemm

using namespace tgemm;

extern "C" {

int q2_pack(const uint8_t* codes, const float* scale, uint8_t* wq, uint16_t* d, int N, int K,
            uint32_t* status, void* stream) {
  if (!codes || !scale || !wq || !d || !status) return TGEMM_EINVAL;
  if (N < 1 || K < 128 || K % 128) return TGEMM_EINVAL;
  if (!aligned(codes, 16) || !aligned(wq, 16) || !aligned(scale, 4) || !aligned(d, 2) ||
      !aligned(status, 4))
    return TGEMM_EALIGN;
  DeviceInfo di;
  if (int st = current_device_info(&di)) return st;
  const int64_t units = static_cast<int64_t>(N) * K / 64;
  const int64_t scales = static_cast<int64_t>(N) * K / 128;
  const cudaStream_t st = as_stream(stream);
  return launch(TGEMM_KIND_PREP, st, [&] {
    return pdl_launch(q2_pack_kernel, grid_for(units, 256, di.sms), 256, 0, st, codes, scale, wq, d, units, scales, status);
  });
}

int q2_from_gemlite(const uint8_t* wq_g, const float* scale, const float* zero, int N, int K,
                    int g, uint8_t* wq, uint16_t* d, uint32_t* status, void* stream) {
  if (!wq_g || !scale || !zero || !wq || !d || !status) return TGEMM_EINVAL;
  if (N < 1 || K < 128 || K % 128 || g < 4) return TGEMM_EINVAL;
  const bool small_groups = 128 % g == 0 && g % 4 == 0;
  const bool large_groups = g % 128 == 0 && K % g == 0;
  if (!small_groups && !large_groups) return TGEMM_EINVAL;
  if (!aligned(wq, 16) || !aligned(scale, 4) || !aligned(zero, 4) || !aligned(d, 2) ||
      !aligned(status, 4))
    return TGEMM_EALIGN;
  DeviceInfo di;
  if (int st = current_device_info(&di)) return st;
  const int tiles_n = (N + kGlTileN - 1) / kGlTileN;
  const int64_t tiles = static_cast<int64_t>(K / 4 / kGlTileI) * tiles_n;
  if (tiles > 0x7FFFFFFF) return TGEMM_ETOOLARGE;
  const cudaStream_t st = as_stream(stream);
  return launch(TGEMM_KIND_PREP, st, [&] {
    return pdl_launch(q2_from_gemlite_kernel, static_cast<int>(tiles), 256, 0, st, wq_g, scale, zero,
                      wq, d, N, K, g, tiles_n, status);
  });
}

int q4_pack(const uint8_t* codes, const float* s, const float* z, uint8_t* wq, uint16_t* sz,
            int N, int K, uint32_t* status, void* stream) {
  if (!codes || !s || !z || !wq || !sz || !status) return TGEMM_EINVAL;
  if (N < 1 || K < 64 || K % 64) return TGEMM_EINVAL;
  if (!aligned(codes, 16) || !aligned(wq, 16) || !aligned(s, 4) || !aligned(z, 4) ||
      !aligned(sz, 4) || !aligned(status, 4))
    return TGEMM_EALIGN;
  DeviceInfo di;
  if (int st = current_device_info(&di)) return st;
  const int64_t units = static_cast<int64_t>(N) * K / 32;
  const int64_t groups = static_cast<int64_t>(N) * K / 64;
  const cudaStream_t st = as_stream(stream);
  return launch(TGEMM_KIND_PREP, st, [&] {
    return pdl_launch(q4_pack_kernel, grid_for(units, 256, di.sms), 256, 0, st, codes, s, z, wq, sz, units, groups, status);
  });
}

int q2_dequant(const uint8_t* wq, const uint16_t* d, float* w, int N, int K, void* stream) {
  if (!wq || !d || !w) return TGEMM_EINVAL;
  if (N < 1 || K < 128 || K % 128) return TGEMM_EINVAL;
  if (!aligned(wq, 4) || !aligned(d, 2) || !aligned(w, 16)) return TGEMM_EALIGN;
  DeviceInfo di;
  if (int st = current_device_info(&di)) return st;
  const int64_t words = static_cast<int64_t>(N) * K / 16;
  const cudaStream_t st = as_stream(stream);
  return launch(TGEMM_KIND_PREP, st, [&] {
    return pdl_launch(q2_dequant_kernel, grid_for(words, 256, di.sms), 256, 0, st, wq, d, w, words, K);
  });
}

int q4_dequant(const uint8_t* wq, const uint16_t* sz, float* w, int N, int K, void* stream) {
  if (!wq || !sz || !w) return TGEMM_EINVAL;
  if (N < 1 || K < 64 || K % 64) return TGEMM_EINVAL;
  if (!aligned(wq, 4) || !aligned(sz, 4) || !aligned(w, 16)) return TGEMM_EALIGN;
  DeviceInfo di;
  if (int st = current_device_info(&di)) return st;
  const int64_t words = static_cast<int64_t>(N) * K / 8;
  const cudaStream_t st = as_stream(stream);
  return launch(TGEMM_KIND_PREP, st, [&] {
    return pdl_launch(q4_dequant_kernel, grid_for(words, 256, di.sms), 256, 0, st, wq, sz, w, words, K);
  });
}

int tgemm_selftest_wait_timeout(void* stream) {
  DeviceInfo di;
  if (int st = current_device_info(&di)) return st;
  const cudaStream_t st = as_stream(stream);
  return launch(TGEMM_KIND_PREP, st, [&] { return pdl_launch(selftest_wait_kernel, 1, 32, 0, st); });
}

int tgemm_mma_rate(int mode, int n, int iters, unsigned long long* out, int nout, void* stream) {
  if (!out || mode < 0 || mode > 10 || iters < 1 || iters > (1 << 20)) return TGEMM_EINVAL;
  if (mode <= 2 && (n < 16 || n > 256 || n % 16)) return TGEMM_EINVAL;
  if (!aligned(out, 8)) return TGEMM_EALIGN;
  DeviceInfo di;
  if (int st = current_device_info(&di)) return st;
  if (nout < di.sms) return TGEMM_EINVAL;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(mma_rate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRateSmem);
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(drain_rate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRateSmem);
  });
  if (attr_err != cudaSuccess) return TGEMM_ECUDA;
  const cudaStream_t st = as_stream(stream);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(di.sms));
  cfg.blockDim = dim3(mode >= 6 ? kDrainThreads : 128);
  cfg.dynamicSmemBytes = kRateSmem;
  cfg.stream = st;
  const cudaError_t le = mode >= 6 ? cudaLaunchKernelEx(&cfg, drain_rate_kernel, mode, iters, out)
                                   : cudaLaunchKernelEx(&cfg, mma_rate_kernel, mode, n, iters, out);
  return le == cudaSuccess ? TGEMM_OK : TGEMM_ECUDA;
}

int tgemm_selftest_bad_launch(void* stream) {
  DeviceInfo di;
  if (int st = current_device_info(&di)) return st;
  const cudaStream_t st = as_stream(stream);
  // 2048 threads per block is over the 1024 limit: the runtime refuses the launch on the
  // host, returns the error and leaves it in its last-error slot; nothing reaches the GPU.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(2048);
  cfg.stream = st;
  const cudaError_t le = cudaLaunchKernelEx(&cfg, selftest_noop_kernel);
  return le == cudaSuccess ? TGEMM_OK : TGEMM_ECUDA;
}

size_t tgemm_workspace_size(int op, int M, int N, int K, int r) {
  if (M < 1 || N < 1 || K < 1) return 0;
  if (op != TGEMM_OP_Q2 && op != TGEMM_OP_Q2_LORA && op != TGEMM_OP_Q4) return 0;
  if (op == TGEMM_OP_Q2_LORA && (r < 1 || r > 256)) return 0;
  return workspace_layout(op, M, N, K, r, choose_path(M), sms_for_sizing()).total;
}

size_t tgemm_workspace_size_min(int op, int M, int N, int K, int r) {
  if (M < 1 || N < 1 || K < 1) return 0;
  if (op != TGEMM_OP_Q2 && op != TGEMM_OP_Q2_LORA && op != TGEMM_OP_Q4) return 0;
  if (op == TGEMM_OP_Q2_LORA && (r < 1 || r > 256)) return 0;
  return workspace_layout(op, M, N, K, r, choose_path(M), kDefaultSms).total_whole;
}

int tgemm_tc_plan(int op, int M, int N, int K, int r, int K2, int sms, int* plan) {
  if (!plan || M < 1 || N < 1 || K < 1 || K2 < 0 || sms < 1) return TGEMM_EINVAL;
  if (op != TGEMM_OP_Q2 && op != TGEMM_OP_Q2_LORA && op != TGEMM_OP_Q4) return TGEMM_EINVAL;
  if (op == TGEMM_OP_Q2_LORA && (r < 1 || r > 256)) return TGEMM_EINVAL;
  if (K2 > 0 && op != TGEMM_OP_Q2) return TGEMM_EINVAL;
  const int kt_lora = op == TGEMM_OP_Q2_LORA ? lora_dims(r, K).L : 0;
  const TcSchedule sc = tc_schedule(M, N, K + K2, kt_lora, sms);
  plan[0] = sc.tiles_m;
  plan[1] = sc.num_tiles;
  plan[2] = sc.ksteps;
  plan[3] = sc.sk_t0;
  plan[4] = sc.upc;
  plan[5] = sc.dpc;
  plan[6] = sc.grid;
  plan[7] = sc.split ? 1 : 0;
  return TGEMM_OK;
}

int tgemm_gemv_plan(int fmt, int M, int N, int K, int sms, int* plan) {
  if (!plan || M < 1 || M > 16 || N < 1 || K < 1 || sms < 1) return TGEMM_EINVAL;
  if ((fmt != 0 && fmt != 1) || K % (fmt == 0 ? 128 : 64)) return TGEMM_EINVAL;
  const GsPlan pl = gs_plan(fmt, nullptr, nullptr, nullptr, nullptr, M, N, K, 0, sms);
  if (!pl.ok) return TGEMM_ETOOLARGE;
  const GsParams& q = pl.p;
  const int vals[17] = {M <= 8 ? 1 : 2, q.kp, q.passes, q.grid, q.S, q.U, q.j_max, pl.smem,
                        q.nbox, q.xs_stride, q.off_x, q.off_corr, q.off_red, q.off_acc,
                        q.off_sc, q.off_ring, q.off_bar};
  for (int i = 0; i < 17; ++i) plan[i] = vals[i];
  return TGEMM_OK;
}

int tgemm_q2(const uint16_t* x, const uint8_t* wq, const uint16_t* d, void* y, int M, int N,
             int K, int out_dtype, void* workspace, size_t ws_bytes, void* stream) {
  return run_gemm(0, x, wq, d, nullptr, nullptr, 0, y, M, N, K, out_dtype, workspace, ws_bytes,
                  stream);
}

int tgemm_q2_lora(const uint16_t* x, const uint8_t* wq, const uint16_t* d, const uint16_t* a,
                  const uint16_t* b, int r, void* y, int M, int N, int K, int out_dtype,
                  void* workspace, size_t ws_bytes, void* stream) {
  if (!a) return TGEMM_EINVAL;
  return run_gemm(0, x, wq, d, a, b, r, y, M, N, K, out_dtype, workspace, ws_bytes, stream);
}

int tgemm_q2_lora_bt(const uint16_t* x, const uint8_t* wq, const uint16_t* d, const uint16_t* a,
                     const uint16_t* bt, int r, void* y, int M, int N, int K, int out_dtype,
                     void* workspace, size_t ws_bytes, void* stream) {
  if (!a) return TGEMM_EINVAL;
  return run_gemm(0, x, wq, d, a, bt, r, y, M, N, K, out_dtype, workspace, ws_bytes, stream,
                  SecondInput(), true);
}

int tgemm_q2_noalloc(const uint16_t* x, const uint8_t* wq, const uint16_t* d, void* y, int M,
                     int N, int K, int out_dtype, void* stream) {
  if (!x || !wq || !d || !y) return TGEMM_EINVAL;
  if (M < 1 || N < 1 || K < 128 || K % 128) return TGEMM_EINVAL;
  const size_t need =
      workspace_layout(TGEMM_OP_Q2, M, N, K, 0, choose_path(M), sms_for_sizing()).total_whole;
  if (need > TGEMM_NOALLOC_SCRATCH_BYTES) return TGEMM_ETOOLARGE;
  void* scratch = nullptr;
  if (need > 0) {
    if (int e = noalloc_scratch(&scratch)) return e;
  }
  return run_gemm(0, x, wq, d, nullptr, nullptr, 0, y, M, N, K, out_dtype, scratch,
                  need > 0 ? static_cast<size_t>(TGEMM_NOALLOC_SCRATCH_BYTES) : 0, stream);
}

size_t tgemm_q2_dual_workspace_size(int M, int N, int K1, int K2) {
  if (M < 1 || N < 1 || K1 < 1 || K2 < 1) return 0;
  return workspace_layout(TGEMM_OP_Q2, M, N, K1, 0, choose_path(M), sms_for_sizing(), K2).total;
}

size_t tgemm_q2_dual_workspace_size_min(int M, int N, int K1, int K2) {
  if (M < 1 || N < 1 || K1 < 1 || K2 < 1) return 0;
  return workspace_layout(TGEMM_OP_Q2, M, N, K1, 0, choose_path(M), kDefaultSms, K2).total_whole;
}

int tgemm_q2_dual(const uint16_t* x1, const uint8_t* wq1, const uint16_t* d1, int K1,
                  const uint16_t* x2, const uint8_t* wq2, const uint16_t* d2, int K2, void* y,
                  int M, int N, int out_dtype, void* workspace, size_t ws_bytes, void* stream) {
  if (K2 < 1) return TGEMM_EINVAL;
  SecondInput in2;
  in2.x = x2;
  in2.wq = wq2;
  in2.d = d2;
  in2.K = K2;
  return run_gemm(0, x1, wq1, d1, nullptr, nullptr, 0, y, M, N, K1, out_dtype, workspace,
                  ws_bytes, stream, in2);
}

int tgemm_q4(const uint16_t* x, const uint8_t* wq, const uint16_t* sz, void* y, int M, int N,
             int K, int out_dtype, void* workspace, size_t ws_bytes, void* stream) {
  return run_gemm(1, x, wq, sz, nullptr, nullptr, 0, y, M, N, K, out_dtype, workspace, ws_bytes,
                  stream);
}

const char* tgemm_strerror(int status) {
  switch (status) {
    case TGEMM_OK: return "success";
    case TGEMM_EINVAL: return "invalid argument";
    case TGEMM_EALIGN: return "misaligned pointer";
    case TGEMM_ECUDA: return "CUDA runtime or launch failure";
    case TGEMM_EARCH: return "device is not compute capability 10.0 (sm_100)";
    case TGEMM_EWORKSPACE: return "workspace missing or too small";
    case TGEMM_ETOOLARGE: return "problem too large for this call (built-in scratch or tile count)";
    default: return "unknown status";
  }
}

int tgemm_set_path(int path) {
  if (path != TGEMM_PATH_AUTO && path != TGEMM_PATH_SMALL_M && path != TGEMM_PATH_TENSOR &&
      path != TGEMM_PATH_SMALL_M_PASS && path != TGEMM_PATH_SMALL_M_STREAM)
    return TGEMM_EINVAL;
  return g_path.exchange(path);
}

int tgemm_device_error(uint32_t* bits, int clear) {
  if (!bits) return TGEMM_EINVAL;
  if (cudaDeviceSynchronize() != cudaSuccess) return TGEMM_ECUDA;
  if (cudaMemcpyFromSymbol(bits, g_device_error, sizeof(uint32_t)) != cudaSuccess)
    return TGEMM_ECUDA;
  if (clear) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(uint32_t)) != cudaSuccess)
      return TGEMM_ECUDA;
  }
  return TGEMM_OK;
}

int tgemm_version(void) { return 100; }

int tgemm_profile_enable(int kinds) { return g_profile.exchange(kinds & TGEMM_PROFILE_ALL); }

int tgemm_profile_read(int kind, double* total_ms, int64_t* launches, int reset) {
  if (kind < 0 || kind >= TGEMM_NUM_KINDS || !total_ms || !launches) return TGEMM_EINVAL;
  std::lock_guard<std::mutex> lock(g_prof_mu);
  double sum = 0.0;
  int64_t n = 0;
  int status = TGEMM_OK;
  std::vector<ProfRecord> keep;
  for (const ProfRecord& rec : g_records) {
    if (rec.kind != kind) {
      keep.push_back(rec);
      continue;
    }
    float ms = 0.f;
    if (cudaEventSynchronize(rec.end) != cudaSuccess ||
        cudaEventElapsedTime(&ms, rec.begin, rec.end) != cudaSuccess)
      status = TGEMM_ECUDA;
    sum += ms;
    ++n;
    if (reset) {
      g_event_pool.push_back(rec.begin);
      g_event_pool.push_back(rec.end);
    } else {
      keep.push_back(rec);
    }
  }
  g_records.swap(keep);
  *total_ms = sum;
  *launches = n;
  return status;
}

int64_t tgemm_launch_count(void) { return g_launches.load(); }

}  // extern "C"
