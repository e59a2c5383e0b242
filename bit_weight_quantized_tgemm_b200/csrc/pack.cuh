// pack.cuh -- load-time packing of Q2_0 and 4-bit weights, and the dequant test hooks.
//
// Q2_0 ("We're Teaching Your Browser to Paint...", section "The lucky break that wasn't
// luck"): code k of a row lands in bits 2*(k%4) of byte k/4; the f32 block scale becomes
// an f16 that must round-trip exactly.  4-bit ("You Can Now Just Ask for an Image...",
// section "The bug that hid in one flipped bit"): code t lands in the low nibble of byte
// t/2 when t is even, the high nibble when odd.  Problems are reported through the
// caller's status word; nothing traps.
#pragma once

#include "common.cuh"

namespace tgemm {

constexpr uint32_t kPackBadCode = 1u;
constexpr uint32_t kPackInexact = 2u;
constexpr uint32_t kPackNonFinite = 4u;
constexpr uint32_t kPackZeroMismatch = 8u;
constexpr uint32_t kPackGroupMismatch = 16u;

// OR `bits` into *status once per warp (only lanes with something to report take part).
__device__ __forceinline__ void report_status(uint32_t* status, uint32_t bits) {
  const uint32_t all = __reduce_or_sync(0xFFFFFFFFu, bits);
  if (all && (threadIdx.x & 31u) == 0u) atomicOr(status, all);
}

// f32 -> f16 (nearest even) plus the round-trip classification.
__device__ __forceinline__ uint16_t scale_to_f16(float v, uint32_t& flags) {
  const __half h = __float2half_rn(v);
  if (!isfinite(v)) {
    flags |= kPackNonFinite;
  } else if (__half2float(h) != v) {
    flags |= kPackInexact;
  }
  return __half_as_ushort(h);
}

// One thread packs 64 codes (64 bytes in) into 16 bytes out.
__global__ void __launch_bounds__(256) q2_pack_kernel(const uint8_t* __restrict__ codes,
                                                      const float* __restrict__ scale,
                                                      uint8_t* __restrict__ wq,
                                                      uint16_t* __restrict__ d, int64_t n_units,
                                                      int64_t n_scales, uint32_t* status) {
  // no early trigger: kernels after this one on the stream start only once it has
  // finished, so they may read the packed weights before their own dependency wait
  pdl_wait();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t iters = (n_units > n_scales ? n_units : n_scales);
  for (int64_t base = 0; base < iters; base += stride) {
    const int64_t u = base + tid;
    uint32_t flags = 0;
    if (u < n_units) {
      const uint4* src = reinterpret_cast<const uint4*>(codes + u * 64);
      uint32_t out[4];
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 c = __ldg(src + v);
        const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          // cw[b] holds codes 4b..4b+3 of this 16-code group, one per byte.
          const uint32_t q0 = cw[b] & 0xFFu, q1 = (cw[b] >> 8) & 0xFFu;
          const uint32_t q2 = (cw[b] >> 16) & 0xFFu, q3 = cw[b] >> 24;
          if ((q0 > 2u) | (q1 > 2u) | (q2 > 2u) | (q3 > 2u)) flags |= kPackBadCode;
          const uint32_t byte = (q0 & 3u) | ((q1 & 3u) << 2) | ((q2 & 3u) << 4) | ((q3 & 3u) << 6);
          word |= byte << (8 * b);
        }
        out[v] = word;
      }
      reinterpret_cast<uint4*>(wq)[u] = make_uint4(out[0], out[1], out[2], out[3]);
    }
    if (u < n_scales) d[u] = scale_to_f16(scale[u], flags);
    report_status(status, flags);
  }
}

// gemlite-int2 -> Q2_0 ("We're Teaching Your Browser to Paint...", section "The lucky
// break that wasn't luck": same codes, same bit order, dequant (q - zero) * scale with
// zeros == -scales, so the conversion is a transpose and regroup).  The gemlite bytes are
// [K/4][N] (byte (i, n): codes of k = 4i..4i+3 of row n), so byte (i, n) moves unchanged
// to wq[n][i].  Each CTA transposes one tile of 32 byte-rows x 128 rows n through shared
// memory; then all threads regroup the f32 scales [N][K/g] into f16 block scales, checking
// zero == -scale for every group and that the groups of one 128-block agree.
constexpr int kGlTileI = 32;   // gemlite byte-rows (4 k each) per tile
constexpr int kGlTileN = 128;  // output rows per tile

__global__ void __launch_bounds__(256) q2_from_gemlite_kernel(
    const uint8_t* __restrict__ wq_g, const float* __restrict__ scale,
    const float* __restrict__ zero, uint8_t* __restrict__ wq, uint16_t* __restrict__ d, int N,
    int K, int g, int tiles_n, uint32_t* status) {
  __shared__ uint8_t tile[kGlTileI][kGlTileN + 4];
  // no early trigger: kernels after this one on the stream start only once it has
  // finished, so they may read the packed weights before their own dependency wait
  pdl_wait();
  const int kq = K / 4;
  const int i0 = (static_cast<int>(blockIdx.x) / tiles_n) * kGlTileI;
  const int n0 = (static_cast<int>(blockIdx.x) % tiles_n) * kGlTileN;
  uint32_t flags = 0;
  // load: 32 byte-rows x 128 bytes along n (lanes read consecutive n)
#pragma unroll
  for (int r = 0; r < kGlTileI * kGlTileN / 256; ++r) {
    const int idx = r * 256 + static_cast<int>(threadIdx.x);
    const int ii = idx / kGlTileN, nn = idx % kGlTileN;
    uint32_t byte = 0x55u;  // rows past N: four codes 1, never stored
    if (n0 + nn < N) {
      byte = __ldg(wq_g + static_cast<int64_t>(i0 + ii) * N + n0 + nn);
      if (byte & (byte >> 1) & 0x55u) flags |= kPackBadCode;  // a 2-bit field equal to 3
    }
    tile[ii][nn] = static_cast<uint8_t>(byte);
  }
  __syncthreads();
  // store: row n0 + nn gets bytes [i0, i0 + 32) as eight 4-byte words
#pragma unroll
  for (int r = 0; r < kGlTileI * kGlTileN / 4 / 256; ++r) {
    const int w = r * 256 + static_cast<int>(threadIdx.x);
    const int nn = w / (kGlTileI / 4), wi = w % (kGlTileI / 4);
    if (n0 + nn < N) {
      const uint32_t word = static_cast<uint32_t>(tile[4 * wi][nn]) |
                            (static_cast<uint32_t>(tile[4 * wi + 1][nn]) << 8) |
                            (static_cast<uint32_t>(tile[4 * wi + 2][nn]) << 16) |
                            (static_cast<uint32_t>(tile[4 * wi + 3][nn]) << 24);
      *reinterpret_cast<uint32_t*>(wq + static_cast<int64_t>(n0 + nn) * kq + i0 + 4 * wi) = word;
    }
  }
  report_status(status, flags);
  // regroup the scales: block b of row n takes the scale of the groups covering it
  const int nb = K / 128, ng = K / g;
  const int64_t n_blocks = static_cast<int64_t>(N) * nb;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (int64_t base = 0; base < n_blocks; base += stride) {
    const int64_t u = base + tid;
    uint32_t f = 0;
    if (u < n_blocks) {
      const int64_t n = u / nb;
      const int b = static_cast<int>(u - n * nb);
      const float* srow = scale + n * ng;
      const float* zrow = zero + n * ng;
      const int j0 = 128 * b / g;
      const float sv = __ldg(srow + j0);
      for (int j = j0; j * g < 128 * b + 128; ++j) {
        const float sj = __ldg(srow + j);
        if (!(sj == sv)) f |= kPackGroupMismatch;
        if (!(__ldg(zrow + j) == -sj)) f |= kPackZeroMismatch;
      }
      d[u] = scale_to_f16(sv, f);
    }
    report_status(status, f);
  }
}

// One thread packs 32 codes (32 bytes in) into 16 bytes out.
__global__ void __launch_bounds__(256) q4_pack_kernel(const uint8_t* __restrict__ codes,
                                                      const float* __restrict__ s,
                                                      const float* __restrict__ z,
                                                      uint8_t* __restrict__ wq,
                                                      uint16_t* __restrict__ sz, int64_t n_units,
                                                      int64_t n_groups, uint32_t* status) {
  // no early trigger: kernels after this one on the stream start only once it has
  // finished, so they may read the packed weights before their own dependency wait
  pdl_wait();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t iters = (n_units > n_groups ? n_units : n_groups);
  for (int64_t base = 0; base < iters; base += stride) {
    const int64_t u = base + tid;
    uint32_t flags = 0;
    if (u < n_units) {
      const uint4* src = reinterpret_cast<const uint4*>(codes + u * 32);
      uint32_t out[4];
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        const uint4 c = __ldg(src + v);
        const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t word = 0;
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            const uint32_t w4 = cw[2 * h + b];  // codes 4j..4j+3 of the group, one per byte
            const uint32_t q0 = w4 & 0xFFu, q1 = (w4 >> 8) & 0xFFu;
            const uint32_t q2 = (w4 >> 16) & 0xFFu, q3 = w4 >> 24;
            if ((q0 > 15u) | (q1 > 15u) | (q2 > 15u) | (q3 > 15u)) flags |= kPackBadCode;
            // even index -> low nibble, odd index -> high nibble
            const uint32_t b0 = (q0 & 15u) | ((q1 & 15u) << 4);
            const uint32_t b1 = (q2 & 15u) | ((q3 & 15u) << 4);
            word |= (b0 | (b1 << 8)) << (16 * b);
          }
          out[2 * v + h] = word;
        }
      }
      reinterpret_cast<uint4*>(wq)[u] = make_uint4(out[0], out[1], out[2], out[3]);
    }
    if (u < n_groups) {
      const uint16_t hs = scale_to_f16(s[u], flags);
      const uint16_t hz = scale_to_f16(z[u], flags);
      reinterpret_cast<uint32_t*>(sz)[u] = static_cast<uint32_t>(hs) | (static_cast<uint32_t>(hz) << 16);
    }
    report_status(status, flags);
  }
}

// (q - 1) * d for every weight, f32 out; one thread per 16 weights (one 32-bit word).
__global__ void __launch_bounds__(256) q2_dequant_kernel(const uint8_t* __restrict__ wq,
                                                         const uint16_t* __restrict__ d,
                                                         float* __restrict__ w, int64_t n_words,
                                                         int K) {
  pdl_trigger_and_wait();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t words_per_row = K / 16;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_words;
       i += stride) {
    const int64_t row = i / words_per_row;
    const int64_t kw = (i % words_per_row) * 16;  // first k of this word
    const uint32_t word = reinterpret_cast<const uint32_t*>(wq)[i];
    const float dd = __half2float(__ushort_as_half(d[row * (K / 128) + kw / 128]));
    float out[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int q = static_cast<int>((word >> (2 * j)) & 3u);
      out[j] = static_cast<float>(q - 1) * dd;
    }
    float4* dst = reinterpret_cast<float4*>(w + row * K + kw);
#pragma unroll
    for (int j = 0; j < 4; ++j) dst[j] = make_float4(out[4 * j], out[4 * j + 1], out[4 * j + 2], out[4 * j + 3]);
  }
}

// (q - z) * s for every weight, two rounded f32 operations; one thread per 8 weights.
__global__ void __launch_bounds__(256) q4_dequant_kernel(const uint8_t* __restrict__ wq,
                                                         const uint16_t* __restrict__ sz,
                                                         float* __restrict__ w, int64_t n_words,
                                                         int K) {
  pdl_trigger_and_wait();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t words_per_row = K / 8;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_words;
       i += stride) {
    const int64_t row = i / words_per_row;
    const int64_t t0 = (i % words_per_row) * 8;
    const uint32_t word = reinterpret_cast<const uint32_t*>(wq)[i];
    const uint32_t szw = reinterpret_cast<const uint32_t*>(sz)[row * (K / 64) + t0 / 64];
    const float sc = __half2float(__ushort_as_half(static_cast<uint16_t>(szw & 0xFFFFu)));
    const float ze = __half2float(__ushort_as_half(static_cast<uint16_t>(szw >> 16)));
    float out[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float q = static_cast<float>((word >> (4 * j)) & 15u);
      out[j] = __fmul_rn(__fsub_rn(q, ze), sc);
    }
    float4* dst = reinterpret_cast<float4*>(w + row * K + t0);
    dst[0] = make_float4(out[0], out[1], out[2], out[3]);
    dst[1] = make_float4(out[4], out[5], out[6], out[7]);
  }
}

}  // namespace tgemm
