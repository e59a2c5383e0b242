// gemv.cuh -- small-M path (up to 16 tokens per pass over the weights): HBM-bound on the
// packed weights, and at these sizes bound by the latency of one trip to memory, so the
// kernel is laid out to need exactly one such trip after its dependency wait.
//
// Each CTA owns 16 weight rows (the M side of mma.sync m16n8k16); its 8 warps split K in
// units of 128 weights; the tokens are the mma's N side (8 per tile, one or two tiles).
// Per pass over up to kp weights along K:
//   * lanes of warp 0 start one bulk copy (cp.async.bulk) per token row of the pass's
//     activations into shared memory, in their natural order, completing on an mbarrier;
//   * meanwhile every lane loads, straight into registers, all the packed codes it needs
//     for the pass (lane (g, c): rows g and g+8, bytes [8c, 8c+8) of each of its 32-byte
//     Q2 row-units, or bytes [8c, 8c+8) and [32+8c, 32+8c+8) of its 64-byte 4-bit
//     row-units: each 32-byte sector is requested once), and the CTA loads the pass's
//     scales of its 16 rows with consecutive threads on consecutive scales;
//   * the codes of one byte (Q2) or byte pair (4-bit) become an A fragment pair with a
//     byte permute, a mask-and-or that sets a bf16 exponent (the code then reads as an
//     exact integer plus a known offset), and one subtraction;
//   * the B fragments (activations) are one 8-byte shared-memory load per k16 step.
// Block scales are applied to the f32 partial sums after each block:
//   Q2_0:  A = base + q (base 128 or 32 by k slot), C = sum of (base + 1) x (an mma against
//          constants), then y += d * (sum - C)                    (128-weight block)
//   4-bit: A = 128 + q, S = sum of x over the group (an mma against ones),
//          then y += s * (sum - (128 + z) * S)                      (64-weight group)
// which equals sum_k (q - 1) d x  and  sum_k (q - z) s x  up to f32 rounding (all products
// of the bf16 operands are exact in the f32 accumulators).
// The warps' partial sums are reduced through shared memory; the optional low-rank
// branch adds sum_i B[n][i] u[m][i] (u = A x in f32, from the lora kernels).
//
// k order inside an mma.  Lane (g, c) supplies the k slots {2c, 2c+1, 2c+8, 2c+9} of A
// (weight rows g, g+8) and of B (token g).  In k16 step s of a 128-k unit those slots hold
// four consecutive codes -- one Q2 byte, or two 4-bit bytes -- in the slot order
//   Q2:    codes 32c + 4s + (0, 1 | 2, 3)
//   4-bit: codes 16c + 4s + (0, 2 | 1, 3)  (steps 0-3, the first 64-weight group), and
//          64 + 16c + 4(s-4) + (0, 2 | 1, 3)  (steps 4-7, the second group)
// so that all codes of a 4-bit step share one group.  Any assignment of codes to slots
// gives the same contraction as long as A and B agree, and every lane's codes for all eight
// steps are the 8 (Q2) or 16 (4-bit) bytes it loaded.
#pragma once

#include "common.cuh"

namespace tgemm {

constexpr int kGvRows = 16;   // weight rows per CTA
constexpr int kGvWarps = 8;   // warps per CTA, splitting K
constexpr int kGvUnit = 128;  // K per unit (one Q2 block, two 4-bit groups)
// units per warp per pass: the codes of a pass are held in registers
template <int FMT>
struct GvFmt {
  static constexpr int kMaxU = FMT == 0 ? 6 : 4;
  static constexpr int kKPMax = kMaxU * kGvWarps * kGvUnit;  // 6144 (Q2), 4096 (4-bit)
  static constexpr int kUnitBytes = FMT == 0 ? 32 : 64;      // packed bytes of a row-unit
  static constexpr int kWords = FMT == 0 ? 2 : 4;             // 32-bit code words per lane
};
// Dynamic shared memory per CTA: the staged activations (whose space the warps' partial
// sums reuse once the last pass is done) and, with the low-rank branch, u and B.  Two CTAs
// fit on one SM at this size: 2 x (111360 + at most 4224 static + 1024 reserved) is within
// the SM's 233472 bytes.  16 tokens x 3072 (and, with the branch, up to r = 112) take one pass.
constexpr int kGvXBudget = 111360;

__host__ __device__ constexpr int gemv_row_stride_bytes(int kp) { return 2 * kp + 16; }
__host__ __device__ constexpr int gemv_round16(int b) { return (b + 15) / 16 * 16; }
// the warps' partial sums: f32 [warp][row][token], kTok + 1 tokens per row
__host__ __device__ constexpr int gemv_red_bytes(int T) { return kGvWarps * kGvRows * (8 * T + 1) * 4; }
// the activation rows of a pass, or the partial sums, whichever is larger
__host__ __device__ constexpr int gemv_xreg_bytes(int mrows, int kp, int T) {
  return gemv_round16(mrows * gemv_row_stride_bytes(kp) > gemv_red_bytes(T)
                          ? mrows * gemv_row_stride_bytes(kp) : gemv_red_bytes(T));
}
// Branch operands in shared memory, bf16, the rank padded with zeros to a multiple of 16 and
// rows gemv_lb_pitch(r) elements apart (= 8 mod 16, so a fragment's 32 words hit 32 banks):
// the CTA's 16 rows of B, then u of the pass's 8 T tokens as u_hi = bf16(u) and
// u_lo = bf16(u - u_hi).
__host__ __device__ constexpr int gemv_lb_pitch(int r) { return (r + 15) / 16 * 16 + 8; }
__host__ __device__ constexpr int gemv_lora_bytes(int T, int r) {
  return r > 0 ? gemv_round16((kGvRows + 16 * T) * gemv_lb_pitch(r) * 2) : 0;
}
// K per pass: the largest multiple of 128 (at most the format's kKPMax) whose staged
// activation rows (`mrows` tokens, token tiles of 8 T) fit kGvXBudget next to `extra`
// bytes; never more than K needs.
__host__ __device__ inline int gemv_pass_k(int fmt, int mrows, int K, int T = 2, int extra = 0) {
  const int kmax = fmt == 0 ? GvFmt<0>::kKPMax : GvFmt<1>::kKPMax;
  int kp = (K + kGvUnit - 1) / kGvUnit * kGvUnit;
  if (kp > kmax) kp = kmax;
  while (kp > kGvUnit && gemv_xreg_bytes(mrows, kp, T) + extra > kGvXBudget) kp -= kGvUnit;
  return kp;
}
__host__ __device__ constexpr int gemv_smem_bytes(int mrows, int kp, int T = 2, int r = 0) {
  return gemv_xreg_bytes(mrows, kp, T) + gemv_lora_bytes(T, r);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// Q2: byte `b` of w (codes q0..q3 at bits 0-1, 2-3, 4-5, 6-7) -> two bf16x2 pairs
// (128 + q0, 32 + q1) and (128 + q2, 32 + q3).  The byte is copied into both halves; the
// low half keeps bits 0-1 under the exponent of 128 (ulp 1), the high half bits 2-3 (its
// bits 18-19) under the exponent of 32 (ulp 1/4, so bit 2 is worth 1).  The offsets are
// removed after the mma: sum_k (q - 1) x = sum_k (base_k + q) x - sum_k (base_k + 1) x,
// the last term being one more mma of x against the constant pairs (129, 33).
constexpr uint32_t kQ2Offset1 = 0x42044301u;  // bf16x2 (129, 33)
__device__ __forceinline__ void q2_byte_pairs(uint32_t w, int b, uint32_t& lo, uint32_t& hi) {
  const uint32_t p = prmt(w, 0u, static_cast<uint32_t>(b) | 0x4040u | (static_cast<uint32_t>(b) << 8));
  lo = lop3_and_or(p, 0x000C0003u, 0x42004300u);
  hi = lop3_and_or(p >> 4, 0x000C0003u, 0x42004300u);
}

// 4-bit: bytes 2h and 2h+1 of w (codes q0, q1 | q2, q3, low nibble first) -> bf16x2 pairs
// (128 + q0, 128 + q2) and (128 + q1, 128 + q3), each nibble under the exponent of 128;
// the offset joins the zero point: (q - z) = (128 + q) - (128 + z).
__device__ __forceinline__ void q4_bytes_pairs(uint32_t w, int h, uint32_t& lo, uint32_t& hi) {
  const uint32_t sel = static_cast<uint32_t>(2 * h) | 0x40u | (static_cast<uint32_t>(2 * h + 1) << 8) | 0x4000u;
  const uint32_t p = prmt(w, 0u, sel);
  lo = lop3_and_or(p, 0x000F000Fu, 0x43004300u);
  hi = lop3_and_or(p >> 4, 0x000F000Fu, 0x43004300u);
}

// DUAL: a second input (x2, wq2, scales2, K2) whose product adds into the same sums.
// T: token tiles of 8 per pass (1 for up to 8 tokens, 2 for up to 16).
template <int FMT, int T, bool LORA, bool DUAL>
__global__ void __launch_bounds__(256, 2) gemv_kernel(
    const uint16_t* __restrict__ x, const uint8_t* __restrict__ wq,
    const uint16_t* __restrict__ scales, void* __restrict__ y, int M, int N, int K, int out_f32,
    const float* __restrict__ u, const uint16_t* __restrict__ lb, int r, int lb_sn, int lb_si,
    int kp,
    const uint16_t* __restrict__ x2, const uint8_t* __restrict__ wq2,
    const uint16_t* __restrict__ scales2, int K2) {
  using F = GvFmt<FMT>;
  constexpr int kTok = 8 * T;  // tokens per pass over the weights
  extern __shared__ __align__(128) uint8_t gv_smem[];
  __shared__ __align__(8) uint64_t xbar;              // the activation copies of a pass
  __shared__ uint32_t abort_word;
  // the pass's scales of the CTA's rows: Q2 d per unit, 4-bit (s, z) per group
  constexpr int kScl = FMT == 0 ? F::kMaxU * kGvWarps : 2 * F::kMaxU * kGvWarps;
  constexpr int kSclPerThread = kGvRows * kScl / 256;
  static_assert(kSclPerThread * 256 == kGvRows * kScl,
                "the 256 threads must stage every scale of a pass, none twice");
  __shared__ uint32_t scl[kGvRows][kScl];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int n0 = blockIdx.x * kGvRows;
  const uint32_t xs = smem_u32(gv_smem);
  const uint32_t bar = smem_u32(&xbar);
  const int rs = gemv_row_stride_bytes(kp);
  // the warps' partial sums [warp][row][token] reuse the activations' space after the last pass
  float* red = reinterpret_cast<float*>(gv_smem);
  // branch operands: the CTA's rows of B [row][lbp], u_hi and u_lo [token][lbp]
  const int lbp = gemv_lb_pitch(r), r16 = lbp - 8;
  uint16_t* bs = reinterpret_cast<uint16_t*>(gv_smem + gemv_xreg_bytes(min(M, kTok), kp, T));
  uint16_t* uhs = bs + kGvRows * lbp;
  uint16_t* uls = uhs + kTok * lbp;
  volatile uint32_t* abort_flag = &abort_word;
  if (tid == 0) {
    mbar_init(bar, 1);
    abort_word = 0u;
    fence_mbar_init();
  }
  pdl_trigger();
  // Every packed-code load of a pass goes straight into registers: lane (g, c) takes rows g
  // and g + 8, bytes [8c, 8c + 8) of each of its 32-byte Q2 row-units (or [8c, 8c + 8) and
  // [32 + 8c, 32 + 8c + 8) of its 64-byte 4-bit row-units).
  uint32_t wreg[F::kMaxU][2][F::kWords];
  auto load_codes = [&](const uint8_t* wqq, int64_t row_bytes, int Kq, int u_base, int u_end) {
#pragma unroll
    for (int i = 0; i < F::kMaxU; ++i) {
      const int unit = u_base + warp + kGvWarps * i;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int row = n0 + 8 * j + g;
        const bool ok = unit < u_end && row < N;
        const uint8_t* base = wqq + static_cast<int64_t>(row) * row_bytes +
                              static_cast<int64_t>(unit) * F::kUnitBytes;
        if (FMT == 0) {
          // codes 32c..32c+31 of the unit (code 1 = weight 0 where there is no row)
          uint2 a = make_uint2(0x55555555u, 0x55555555u);
          if (ok) a = __ldg(reinterpret_cast<const uint2*>(base + 8 * c));
          wreg[i][j][0] = a.x;
          wreg[i][j][1] = a.y;
        } else {
          // codes 16c..16c+15 and 64+16c..64+16c+15; the unit's second 64 codes exist
          // only where K reaches them
          const bool ok2 = ok && static_cast<int64_t>(unit) * kGvUnit + 64 < Kq;
          uint2 a = make_uint2(0u, 0u), b = make_uint2(0u, 0u);
          if (ok) a = __ldg(reinterpret_cast<const uint2*>(base + 8 * c));
          if (ok2) b = __ldg(reinterpret_cast<const uint2*>(base + 32 + 8 * c));
          wreg[i][j][0] = a.x;
          wreg[i][j][1] = a.y;
          wreg[i][j][2] = b.x;
          wreg[i][j][3] = b.y;
        }
      }
    }
  };
  // The pass's scales of the CTA's rows (consecutive threads, consecutive scales) -> shared.
  auto stage_scales = [&](const uint16_t* sq, int nscale, int u_base, int u_end) {
    const int s_base = FMT == 0 ? u_base : 2 * u_base;
    const int s_cnt = FMT == 0 ? u_end - u_base : min(nscale - s_base, 2 * (u_end - u_base));
    uint32_t sv[kSclPerThread];
#pragma unroll
    for (int e = 0; e < kSclPerThread; ++e) {
      const int it = tid + 256 * e;
      const int rl = it / s_cnt, si = it - rl * s_cnt;
      const int n = n0 + rl;
      sv[e] = 0u;
      if (rl < kGvRows && n < N) {
        const int64_t idx = static_cast<int64_t>(n) * nscale + s_base + si;
        sv[e] = FMT == 0 ? static_cast<uint32_t>(__ldg(sq + idx))
                         : __ldg(reinterpret_cast<const uint32_t*>(sq) + idx);
      }
    }
#pragma unroll
    for (int e = 0; e < kSclPerThread; ++e) {
      const int it = tid + 256 * e;
      const int rl = it / s_cnt, si = it - rl * s_cnt;
      if (rl < kGvRows) scl[rl][si] = sv[e];
    }
  };
  // The first pass's codes and scales load before the dependency wait: the packed weights
  // are not an output of the kernels ahead on the stream, so their trip to memory overlaps
  // the end of those kernels; only the activations are fetched after the wait.
  {
    const int u_end0 = (min(kp, K) + kGvUnit - 1) / kGvUnit;
    load_codes(wq, FMT == 0 ? K / 4 : K / 2, K, 0, u_end0);
    stage_scales(scales, FMT == 0 ? K / 128 : K / 64, 0, u_end0);
  }
  if (LORA) {
    // The CTA's rows of B (a weight, like the codes) -> shared memory, zero past r and N,
    // in the order that keeps consecutive threads on consecutive addresses of its layout.
    const bool by_row = lb_si == 1;
    for (int i0 = tid; i0 < kGvRows * r16; i0 += 4 * 256) {
      uint16_t v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = i0 + e * 256;
        const int nn = by_row ? i / r16 : i % kGvRows, k = by_row ? i % r16 : i / kGvRows;
        v[e] = 0;
        if (i < kGvRows * r16 && k < r && n0 + nn < N)
          v[e] = __ldg(lb + static_cast<int64_t>(n0 + nn) * lb_sn + static_cast<int64_t>(k) * lb_si);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = i0 + e * 256;
        const int nn = by_row ? i / r16 : i % kGvRows, k = by_row ? i % r16 : i / kGvRows;
        if (i < kGvRows * r16) bs[nn * lbp + k] = v[e];
      }
    }
  }
  __syncthreads();  // the barrier's initialisation and the first scales are visible
  pdl_wait();

  uint32_t phase = 0;  // completed activation copies (the mbarrier's phase parity)
  bool first = true;   // the first (token pass, input, k pass) has its weights loaded
  for (int m0 = 0; m0 < M; m0 += kTok) {
    const int mt = min(kTok, M - m0);  // tokens in this pass over the weights
    float acc[T][4];
#pragma unroll
    for (int t = 0; t < T; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[t][e] = 0.f;
    if (LORA && warp > 0) {
      // Warps 1-7 copy u of this pass's tokens to shared memory as (u_hi, u_lo), zero past
      // r and the pass's tokens, while warp 0 starts the activation copies; they are read
      // after the last pass.
      const int nt = blockDim.x - 32;
      for (int i0 = tid - 32; i0 < kTok * r16; i0 += 8 * nt) {
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int i = i0 + e * nt, mm = i / r16, k = i % r16;
          v[e] = i < kTok * r16 && mm < mt && k < r ? __ldg(u + static_cast<int64_t>(m0 + mm) * r + k) : 0.f;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int i = i0 + e * nt, mm = i / r16, k = i % r16;
          if (i < kTok * r16) {
            const __nv_bfloat16 h = __float2bfloat16_rn(v[e]);
            uhs[mm * lbp + k] = __bfloat16_as_ushort(h);
            uls[mm * lbp + k] = __bfloat16_as_ushort(__float2bfloat16_rn(v[e] - __bfloat162float(h)));
          }
        }
      }
    }

    // one input, or two (a projection split along its input axis: their products add
    // into the same partial sums)
    for (int part = 0; part < (DUAL ? 2 : 1); ++part) {
      const uint16_t* xq = part ? x2 : x;
      const uint8_t* wqq = part ? wq2 : wq;
      const uint16_t* sq = part ? scales2 : scales;
      const int Kq = part ? K2 : K;
      const int64_t row_bytes = FMT == 0 ? Kq / 4 : Kq / 2;
      const int nscale = FMT == 0 ? Kq / 128 : Kq / 64;
      for (int k0 = 0; k0 < Kq; k0 += kp) {
        const int kpass = min(kp, Kq - k0);
        const int u_base = k0 / kGvUnit;
        const int u_end = (k0 + kpass + kGvUnit - 1) / kGvUnit;
        // ---- the pass's activation rows -> shared memory (async)
        if (warp == 0) {
          if (lane == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(mt * kpass * 2));
          __syncwarp();
          if (lane < mt)
            bulk_copy_g2s(xs + lane * rs, xq + static_cast<int64_t>(m0 + lane) * Kq + k0,
                          static_cast<uint32_t>(kpass * 2), bar);
        }
        // the next pass's rows -> L2
        if (k0 + kp < Kq) {
          const int nb = FMT == 0 ? min(kp, Kq - k0 - kp) / 4 : min(kp, Kq - k0 - kp) / 2;
          const int lines = (nb + 127) / 128;
          for (int i = tid; i < kGvRows * lines; i += blockDim.x) {
            const int row = n0 + i / lines;
            if (row < N)
              prefetch_l2(wqq + static_cast<int64_t>(row) * row_bytes +
                          (FMT == 0 ? (k0 + kp) / 4 : (k0 + kp) / 2) + (i % lines) * 128);
          }
        }
        // ---- this pass's codes and scales (the very first pass's are already loaded)
        if (!first) {
          load_codes(wqq, row_bytes, Kq, u_base, u_end);
          stage_scales(sq, nscale, u_base, u_end);
        }
        first = false;
        // ---- wait for the activations (bounded); every thread must agree before going on
        const bool got = mbar_wait(bar, phase, abort_flag);
        phase ^= 1u;
        if (!__syncthreads_and(got)) {
          // give the copies in flight a bounded time to land before the CTA leaves
          if (tid == 0) mbar_wait_drain(bar, phase ^ 1u);
          return;
        }
        // ---- the warp's units
#pragma unroll
        for (int i = 0; i < F::kMaxU; ++i) {
          const int unit = u_base + warp + kGvWarps * i;
          if (unit >= u_end) break;
          const int ui = unit - u_base;  // the unit within the pass
          if (FMT == 0) {
            float pacc[T][4], corr[T][4];
#pragma unroll
            for (int t = 0; t < T; ++t)
#pragma unroll
              for (int e = 0; e < 4; ++e) pacc[t][e] = corr[t][e] = 0.f;
            const uint32_t off[4] = {kQ2Offset1, kQ2Offset1, kQ2Offset1, kQ2Offset1};
#pragma unroll
            for (int s = 0; s < 8; ++s) {
              uint32_t af[4];
              q2_byte_pairs(wreg[i][0][s >> 2], s & 3, af[0], af[2]);
              q2_byte_pairs(wreg[i][1][s >> 2], s & 3, af[1], af[3]);
              // activations 32c + 4s .. +3 of the unit, token g (+8t)
              const uint32_t xo = xs + 2 * (ui * kGvUnit + 32 * c + 4 * s);
#pragma unroll
              for (int t = 0; t < T; ++t) {
                uint2 bv = make_uint2(0u, 0u);
                if (g + 8 * t < mt) bv = ld_shared_v2(xo + (g + 8 * t) * rs);
                mma_bf16_16816(pacc[t], af, bv.x, bv.y);
                mma_bf16_16816(corr[t], off, bv.x, bv.y);
              }
            }
            // pacc[t][e]: weight row g (+8 for e >= 2), token 2c + (e & 1) + 8t; corr[t][e]
            // is the same for every row
            const float d0 = __half2float(__ushort_as_half(static_cast<uint16_t>(scl[g][ui])));
            const float d1 = __half2float(__ushort_as_half(static_cast<uint16_t>(scl[g + 8][ui])));
#pragma unroll
            for (int t = 0; t < T; ++t) {
              acc[t][0] = fmaf(d0, pacc[t][0] - corr[t][0], acc[t][0]);
              acc[t][1] = fmaf(d0, pacc[t][1] - corr[t][1], acc[t][1]);
              acc[t][2] = fmaf(d1, pacc[t][2] - corr[t][0], acc[t][2]);
              acc[t][3] = fmaf(d1, pacc[t][3] - corr[t][1], acc[t][3]);
            }
          } else {
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {  // the unit's two 64-weight groups
              if (h2 == 1 && static_cast<int64_t>(unit) * kGvUnit + 64 >= Kq) break;
              float pacc[T][4], ssum[T][4];
#pragma unroll
              for (int t = 0; t < T; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) pacc[t][e] = ssum[t][e] = 0.f;
#pragma unroll
              for (int sq4 = 0; sq4 < 4; ++sq4) {
                const int s = 4 * h2 + sq4;
                uint32_t af[4];
                q4_bytes_pairs(wreg[i][0][s >> 1], s & 1, af[0], af[2]);
                q4_bytes_pairs(wreg[i][1][s >> 1], s & 1, af[1], af[3]);
                // activations 64 h2 + 16c + 4 sq4 .. +3 of the unit, token g (+8t)
                const uint32_t xo = xs + 2 * (ui * kGvUnit + 64 * h2 + 16 * c + 4 * sq4);
                const uint32_t ones[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};
#pragma unroll
                for (int t = 0; t < T; ++t) {
                  uint2 bv = make_uint2(0u, 0u);
                  if (g + 8 * t < mt) bv = ld_shared_v2(xo + (g + 8 * t) * rs);
                  const uint32_t b0 = prmt(bv.x, bv.y, 0x5410u);  // (x0, x2)
                  const uint32_t b1 = prmt(bv.x, bv.y, 0x7632u);  // (x1, x3)
                  mma_bf16_16816(pacc[t], af, b0, b1);
                  mma_bf16_16816(ssum[t], ones, b0, b1);  // S: sum of x per token
                }
              }
              // ssum[t][0] = S of token 2c + 8t, ssum[t][1] = S of token 2c + 1 + 8t
              const uint32_t v0 = scl[g][2 * ui + h2], v1 = scl[g + 8][2 * ui + h2];
              // codes arrive as 128 + q: the zero point becomes 128 + z (exact in f32)
              const float s0 = __half2float(__ushort_as_half(static_cast<uint16_t>(v0 & 0xFFFFu)));
              const float z0 = 128.f + __half2float(__ushort_as_half(static_cast<uint16_t>(v0 >> 16)));
              const float s1 = __half2float(__ushort_as_half(static_cast<uint16_t>(v1 & 0xFFFFu)));
              const float z1 = 128.f + __half2float(__ushort_as_half(static_cast<uint16_t>(v1 >> 16)));
#pragma unroll
              for (int t = 0; t < T; ++t) {
                acc[t][0] = fmaf(s0, fmaf(-z0, ssum[t][0], pacc[t][0]), acc[t][0]);
                acc[t][1] = fmaf(s0, fmaf(-z0, ssum[t][1], pacc[t][1]), acc[t][1]);
                acc[t][2] = fmaf(s1, fmaf(-z1, ssum[t][0], pacc[t][2]), acc[t][2]);
                acc[t][3] = fmaf(s1, fmaf(-z1, ssum[t][1], pacc[t][3]), acc[t][3]);
              }
            }
          }
        }
        // the next pass's bulk copies (the async proxy) overwrite these activations: order
        // this thread's generic-proxy reads of them before those writes
        fence_proxy_async_smem();
        __syncthreads();  // everyone is done with this pass's activations
      }
    }

    // ---- the branch: acc += B (u_hi + u_lo)^T, its rank's 16-wide steps spread over the
    // warps (bf16 products are exact in the f32 accumulators)
    if (LORA) {
      for (int s = warp; s < r16 / 16; s += kGvWarps) {
        // rank slots 2c, 2c+1 (word 0) and 2c+8, 2c+9 (word 4) of step s
        const uint32_t* b0 = reinterpret_cast<const uint32_t*>(bs + g * lbp + 16 * s + 2 * c);
        const uint32_t* b1 = reinterpret_cast<const uint32_t*>(bs + (g + 8) * lbp + 16 * s + 2 * c);
        const uint32_t af[4] = {b0[0], b1[0], b0[4], b1[4]};
#pragma unroll
        for (int t = 0; t < T; ++t) {
          const uint32_t* uh = reinterpret_cast<const uint32_t*>(uhs + (g + 8 * t) * lbp + 16 * s + 2 * c);
          const uint32_t* ul = reinterpret_cast<const uint32_t*>(uls + (g + 8 * t) * lbp + 16 * s + 2 * c);
          mma_bf16_16816(acc[t], af, uh[0], uh[4]);
          mma_bf16_16816(acc[t], af, ul[0], ul[4]);
        }
      }
    }

    // ---- reduce the warps' partial sums and write y ---------------------------------
    // (the last pass ended with a barrier: nobody reads the activations any more)
    auto red_at = [&](int w, int nn, int mm) -> float& {
      return red[(w * kGvRows + nn) * (kTok + 1) + mm];
    };
#pragma unroll
    for (int t = 0; t < T; ++t) {
      red_at(warp, g, 2 * c + 8 * t) = acc[t][0];
      red_at(warp, g, 2 * c + 1 + 8 * t) = acc[t][1];
      red_at(warp, g + 8, 2 * c + 8 * t) = acc[t][2];
      red_at(warp, g + 8, 2 * c + 1 + 8 * t) = acc[t][3];
    }
    __syncthreads();
    for (int o = tid; o < kTok * kGvRows; o += blockDim.x) {
      const int mm = o / kGvRows, nn = o % kGvRows;
      const int m = m0 + mm, n = n0 + nn;
      if (mm >= mt || n >= N) continue;
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kGvWarps; ++w) v += red_at(w, nn, mm);
      if (out_f32)
        reinterpret_cast<float*>(y)[static_cast<int64_t>(m) * N + n] = v;
      else
        reinterpret_cast<__nv_bfloat16*>(y)[static_cast<int64_t>(m) * N + n] = __float2bfloat16_rn(v);
    }
    // the next token pass's bulk copies (the async proxy) overwrite the partial sums
    fence_proxy_async_smem();
    __syncthreads();
  }
}

// u = x A^T for the low-rank branch on the small-M path, in one launch.  CTA (16 tokens, 8
// columns of u = 8 rows of A) runs over the whole of K: its 16 warps take interleaved k16
// steps on mma.sync (A operand: the token rows of x; B operand: the rows of A; bf16 in, f32
// accumulate), and the warps' sums are added in warp order through shared memory -- a fixed
// order, no atomics and no second kernel.  The CTA's rows of A (a weight) are prefetched
// into L2 before the dependency wait.  Lane (g, c) feeds the k slots {2c, 2c+1, 2c+8, 2c+9}
// of a step with its elements 4c..4c+3 (one 8-byte load per row); both operands use that
// map, so the contraction is unchanged.  A8: A is 8-byte aligned (else two 4-byte loads).
constexpr int kLdWarps = 16;
constexpr int kLdBatch = 12;  // k16 steps a warp loads before their mma (one trip when K <= 3072)
template <bool A8>
__global__ void __launch_bounds__(kLdWarps * 32) lora_down_small_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ a, int M, int K, int r,
    float* __restrict__ u) {
  __shared__ float red[kLdWarps][16][8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int j0 = blockIdx.x * 8, m0 = blockIdx.y * 16;
  const int64_t row_bytes = static_cast<int64_t>(K) * 2;
  pdl_trigger();
  {
    const int lines = static_cast<int>((row_bytes + 127) / 128);
    for (int i = threadIdx.x; i < 8 * lines; i += blockDim.x) {
      const int j = j0 + i / lines;
      if (j < r) prefetch_l2(reinterpret_cast<const uint8_t*>(a) + j * row_bytes + (i % lines) * 128);
    }
  }
  pdl_wait();
  const bool ok0 = m0 + g < M, ok1 = m0 + g + 8 < M, okb = j0 + g < r;
  // rows clamped into range (a row that does not exist contributes zeros); element 4c
  const uint2* x0 = reinterpret_cast<const uint2*>(x + static_cast<int64_t>(min(m0 + g, M - 1)) * K) + c;
  const uint2* x1 = reinterpret_cast<const uint2*>(x + static_cast<int64_t>(min(m0 + g + 8, M - 1)) * K) + c;
  const uint16_t* arow = a + static_cast<int64_t>(min(j0 + g, r - 1)) * K + 4 * c;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  const int steps = K / 16;
  for (int kb0 = warp; kb0 < steps; kb0 += kLdWarps * kLdBatch) {
    uint2 f0[kLdBatch], f1[kLdBatch], fb[kLdBatch];
#pragma unroll
    for (int i = 0; i < kLdBatch; ++i) {
      const int kb = kb0 + i * kLdWarps;
      const bool in = kb < steps;
      const uint2 z = make_uint2(0u, 0u);
      f0[i] = in && ok0 ? __ldg(x0 + 4 * kb) : z;
      f1[i] = in && ok1 ? __ldg(x1 + 4 * kb) : z;
      if (A8) {
        fb[i] = in && okb ? __ldg(reinterpret_cast<const uint2*>(arow + 16 * kb)) : z;
      } else {
        const uint32_t* p = reinterpret_cast<const uint32_t*>(arow + 16 * kb);
        fb[i] = in && okb ? make_uint2(__ldg(p), __ldg(p + 1)) : z;
      }
    }
#pragma unroll
    for (int i = 0; i < kLdBatch; ++i) {
      const uint32_t af[4] = {f0[i].x, f1[i].x, f0[i].y, f1[i].y};
      mma_bf16_16816(acc, af, fb[i].x, fb[i].y);
    }
  }
  // acc: u[m0 + g (+8)][j0 + 2c (+1)]
  red[warp][g][2 * c] = acc[0];
  red[warp][g][2 * c + 1] = acc[1];
  red[warp][g + 8][2 * c] = acc[2];
  red[warp][g + 8][2 * c + 1] = acc[3];
  __syncthreads();
  if (threadIdx.x < 128) {
    const int mm = threadIdx.x >> 3, jj = threadIdx.x & 7;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kLdWarps; ++w) v += red[w][mm][jj];
    if (m0 + mm < M && j0 + jj < r) u[static_cast<int64_t>(m0 + mm) * r + j0 + jj] = v;
  }
}

}  // namespace tgemm
