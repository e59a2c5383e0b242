// tgemm.cu -- the C ABI of libtgemm.so: argument checks, workspace layout, dispatch.
//
// One translation unit (kernels are in the included .cuh files) so that every kernel
// sees the same device error word.  Built for sm_100a only.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/tgemm.h"
#include "common.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"
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

inline int launch_status() {
  return cudaGetLastError() == cudaSuccess ? TGEMM_OK : TGEMM_ECUDA;
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

template <int FMT, bool LORA>
int tc_prepare() {
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    err = cudaFuncSetAttribute(tc_gemm_kernel<FMT, LORA>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               TcFmt<FMT>::kSmemBytes);
  });
  return err == cudaSuccess ? TGEMM_OK : TGEMM_ECUDA;
}

// ---- workspace layout -----------------------------------------------------------------

int choose_path(int M) {
  const int p = g_path.load();
  if (p == TGEMM_PATH_SMALL_M) return TGEMM_PATH_SMALL_M;
  if (p == TGEMM_PATH_TENSOR) return TGEMM_PATH_TENSOR;
  return M <= kSmallM ? TGEMM_PATH_SMALL_M : TGEMM_PATH_TENSOR;
}

struct LoraDims {
  int R;     // round_up(r, 16)
  int wcat;  // width of [u_hi | u_lo | 0], a multiple of 64
  int L;     // pipeline stages for the branch
};

LoraDims lora_dims(int r) {
  LoraDims d;
  d.R = (r + 15) / 16 * 16;
  d.wcat = (2 * d.R + 63) / 64 * 64;
  d.L = d.wcat / 64;
  return d;
}

struct Workspace {
  size_t x16 = 0, x16_bytes = 0;  // f16 activations (tensor-core path)
  size_t ucat = 0, ucat_bytes = 0;
  size_t u32 = 0, u32_bytes = 0;  // f32 u (small-M path)
  size_t total = 0;
};

Workspace workspace_layout(int op, int M, int K, int r, int path) {
  Workspace w;
  size_t off = 0;
  if (path == TGEMM_PATH_TENSOR) {
    w.x16 = off;
    w.x16_bytes = static_cast<size_t>(M) * K * 2;
    off = round_up(off + w.x16_bytes, 256);
    if (op == TGEMM_OP_Q2_LORA) {
      w.ucat = off;
      w.ucat_bytes = static_cast<size_t>(M) * lora_dims(r).wcat * 2;
      off = round_up(off + w.ucat_bytes, 256);
    }
  } else if (op == TGEMM_OP_Q2_LORA) {
    w.u32 = off;
    w.u32_bytes = static_cast<size_t>(M) * r * 4;
    off = round_up(off + w.u32_bytes, 256);
  }
  w.total = off;
  return w;
}

// ---- the matmul driver ---------------------------------------------------------------

int run_gemm(int fmt, const uint16_t* x, const uint8_t* wq, const uint16_t* scales,
             const uint16_t* la, const uint16_t* lb, int r, void* y, int M, int N, int K,
             int out_dtype, void* workspace, size_t ws_bytes, void* stream) {
  const bool lora = la != nullptr;
  const int op = fmt == 1 ? TGEMM_OP_Q4 : (lora ? TGEMM_OP_Q2_LORA : TGEMM_OP_Q2);
  const int kblock = fmt == 0 ? 128 : 64;
  if (!x || !wq || !scales || !y) return TGEMM_EINVAL;
  if (M < 1 || N < 1 || K < kblock || K % kblock) return TGEMM_EINVAL;
  if (out_dtype != TGEMM_OUT_F32 && out_dtype != TGEMM_OUT_BF16) return TGEMM_EINVAL;
  if (lora && (!lb || r < 1 || r > 256)) return TGEMM_EINVAL;
  if (!aligned(x, 16) || !aligned(wq, 16) || !aligned(y, 16)) return TGEMM_EALIGN;
  if (!aligned(scales, fmt == 0 ? 2 : 4)) return TGEMM_EALIGN;
  if (lora && (!aligned(la, 4) || !aligned(lb, 2))) return TGEMM_EALIGN;
  const int path = choose_path(M);
  const Workspace wl = workspace_layout(op, M, K, r, path);
  if (wl.total > 0) {
    if (!workspace || ws_bytes < wl.total) return TGEMM_EWORKSPACE;
    if (!aligned(workspace, 256)) return TGEMM_EALIGN;
  }
  DeviceInfo di;
  if (int st = current_device_info(&di)) return st;
  const cudaStream_t st = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int out_f32 = out_dtype == TGEMM_OUT_F32 ? 1 : 0;
  const LoraDims ld = lora ? lora_dims(r) : LoraDims{0, 0, 0};

  if (path == TGEMM_PATH_SMALL_M) {
    float* u32 = nullptr;
    if (lora) {
      u32 = reinterpret_cast<float*>(ws + wl.u32);
      const dim3 grid((M + 15) / 16, (r + 63) / 64);
      lora_down_kernel<<<grid, 256, 0, st>>>(x, la, M, K, r, ld.R, ld.wcat, u32, nullptr);
    }
    const int grid = (N + kGvRows - 1) / kGvRows;
    if (fmt == 0) {
      if (lora)
        gemv_kernel<0, true><<<grid, 256, 0, st>>>(x, wq, scales, y, M, N, K, out_f32, u32, lb, r);
      else
        gemv_kernel<0, false><<<grid, 256, 0, st>>>(x, wq, scales, y, M, N, K, out_f32, nullptr, nullptr, 0);
    } else {
      gemv_kernel<1, false><<<grid, 256, 0, st>>>(x, wq, scales, y, M, N, K, out_f32, nullptr, nullptr, 0);
    }
    return launch_status();
  }

  // ---- tensor-core path
  uint16_t* x16 = reinterpret_cast<uint16_t*>(ws + wl.x16);
  const int64_t ngroups = static_cast<int64_t>(M) * K / 16;
  if (fmt == 0)
    prep_x16_kernel<0><<<grid_for(ngroups, 256, di.sms), 256, 0, st>>>(x, x16, ngroups);
  else
    prep_x16_kernel<1><<<grid_for(ngroups, 256, di.sms), 256, 0, st>>>(x, x16, ngroups);
  uint16_t* ucat = nullptr;
  if (lora) {
    ucat = reinterpret_cast<uint16_t*>(ws + wl.ucat);
    const dim3 grid((M + 15) / 16, (ld.R + 63) / 64);
    lora_down_kernel<<<grid, 256, 0, st>>>(x, la, M, K, r, ld.R, ld.wcat, nullptr, ucat);
  }
  CUtensorMap tm_x, tm_w, tm_u;
  if (int e = make_map_2d(&tm_x, x16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, K, M, kTcBK, kTcBM,
                          CU_TENSOR_MAP_SWIZZLE_128B))
    return e;
  const int wq_row_bytes = fmt == 0 ? 16 : 32;
  const uint64_t wq_cols = fmt == 0 ? K / 4 : K / 2;
  if (int e = make_map_2d(&tm_w, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, wq_cols, N, wq_row_bytes,
                          kTcBN, CU_TENSOR_MAP_SWIZZLE_NONE))
    return e;
  if (lora) {
    if (int e = make_map_2d(&tm_u, ucat, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ld.wcat, M, kTcBK,
                            kTcBM, CU_TENSOR_MAP_SWIZZLE_128B))
      return e;
  } else {
    tm_u = tm_x;  // unused
  }
  TcParams p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.tiles_m = (M + kTcBM - 1) / kTcBM;
  const int tiles_n = (N + kTcBN - 1) / kTcBN;
  p.num_tiles = p.tiles_m * tiles_n;
  p.kt_main = K / kTcBK;
  p.kt_lora = lora ? ld.L : 0;
  p.lora_mmas = lora ? 2 * ld.R / 16 : 0;
  p.R = ld.R;
  p.r = r;
  p.out_f32 = out_f32;
  const int esize = out_f32 ? 4 : 2;
  p.vec_store = (static_cast<int64_t>(N) * esize) % 16 == 0 ? 1 : 0;
  p.scales = scales;
  p.lb = lb;
  p.y = y;
  const int grid = p.num_tiles < di.sms ? p.num_tiles : di.sms;
  if (fmt == 0 && !lora) {
    if (int e = tc_prepare<0, false>()) return e;
    tc_gemm_kernel<0, false><<<grid, kTcThreads, TcFmt<0>::kSmemBytes, st>>>(tm_x, tm_w, tm_u, p);
  } else if (fmt == 0) {
    if (int e = tc_prepare<0, true>()) return e;
    tc_gemm_kernel<0, true><<<grid, kTcThreads, TcFmt<0>::kSmemBytes, st>>>(tm_x, tm_w, tm_u, p);
  } else {
    if (int e = tc_prepare<1, false>()) return e;
    tc_gemm_kernel<1, false><<<grid, kTcThreads, TcFmt<1>::kSmemBytes, st>>>(tm_x, tm_w, tm_u, p);
  }
  return launch_status();
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
  q2_pack_kernel<<<grid_for(units, 256, di.sms), 256, 0, as_stream(stream)>>>(codes, scale, wq, d, units, scales, status);
  return launch_status();
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
  q4_pack_kernel<<<grid_for(units, 256, di.sms), 256, 0, as_stream(stream)>>>(codes, s, z, wq, sz, units, groups, status);
  return launch_status();
}

int q2_dequant(const uint8_t* wq, const uint16_t* d, float* w, int N, int K, void* stream) {
  if (!wq || !d || !w) return TGEMM_EINVAL;
  if (N < 1 || K < 128 || K % 128) return TGEMM_EINVAL;
  if (!aligned(wq, 4) || !aligned(d, 2) || !aligned(w, 16)) return TGEMM_EALIGN;
  DeviceInfo di;
  if (int st = current_device_info(&di)) return st;
  const int64_t words = static_cast<int64_t>(N) * K / 16;
  q2_dequant_kernel<<<grid_for(words, 256, di.sms), 256, 0, as_stream(stream)>>>(wq, d, w, words, K);
  return launch_status();
}

int q4_dequant(const uint8_t* wq, const uint16_t* sz, float* w, int N, int K, void* stream) {
  if (!wq || !sz || !w) return TGEMM_EINVAL;
  if (N < 1 || K < 64 || K % 64) return TGEMM_EINVAL;
  if (!aligned(wq, 4) || !aligned(sz, 4) || !aligned(w, 16)) return TGEMM_EALIGN;
  DeviceInfo di;
  if (int st = current_device_info(&di)) return st;
  const int64_t words = static_cast<int64_t>(N) * K / 8;
  q4_dequant_kernel<<<grid_for(words, 256, di.sms), 256, 0, as_stream(stream)>>>(wq, sz, w, words, K);
  return launch_status();
}

size_t tgemm_workspace_size(int op, int M, int N, int K, int r) {
  (void)N;
  if (M < 1 || K < 1) return 0;
  if (op != TGEMM_OP_Q2 && op != TGEMM_OP_Q2_LORA && op != TGEMM_OP_Q4) return 0;
  if (op == TGEMM_OP_Q2_LORA && (r < 1 || r > 256)) return 0;
  return workspace_layout(op, M, K, r, choose_path(M)).total;
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
    default: return "unknown status";
  }
}

int tgemm_set_path(int path) {
  if (path != TGEMM_PATH_AUTO && path != TGEMM_PATH_SMALL_M && path != TGEMM_PATH_TENSOR)
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

}  // extern "C"
