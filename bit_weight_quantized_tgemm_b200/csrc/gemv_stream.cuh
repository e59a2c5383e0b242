// gemv_stream.cuh -- small-M path (1..16 tokens), streaming form: a persistent grid of
// thread-block clusters that streams the packed weights from HBM through a ring of
// shared-memory slots and splits K across the CTAs of a cluster.
//
// Work split.  The rows of W are cut into `nclus` contiguous ranges (multiples of 8 rows),
// one per cluster; the K axis is cut into units of 128 weights and the units into C
// contiguous slices, one per CTA of the cluster.  A CTA works through its cluster's rows
// in tiles of 16 (the M side of mma.sync m16n8k16); compute warp w takes tiles w, w+8, ...
// and runs every unit of the CTA's K slice for them, so no warp shares a tile with another
// warp of its CTA.  With C > 1 the C partial sums of a tile meet in one CTA of the cluster
// (distributed shared memory) and are added in a fixed order: the result does not depend
// on timing.
//
// Data movement.
//   * Weights: one producer warp copies, per tile, each row's packed codes of the CTA's K
//     slice (cp.async.bulk, one copy per row) into a ring of slots, completing on the
//     slot's mbarrier.  The first slots are issued before the kernel waits for the kernels
//     ahead of it on the stream (griddepcontrol.wait): the packed weights are not an output
//     of those kernels, so their fetch overlaps the end of the previous kernel.
//   * Scales of every tile of the CTA are staged in shared memory, also before the wait.
//   * Activations (the kernels ahead may have written them): after the wait, the compute
//     warps copy the CTA's K slice of x into shared memory with its k order permuted
//     (below), and meanwhile form the per-(unit, token) correction sums.
//
// The unpack.  Inside a 32-bit word of packed codes, a bf16 whose exponent makes a field's
// lowest bit worth 1 reads as base + q, so one lop3 (mask the field, or in the exponent)
// turns a pair of codes 16 bits apart into an exact bf16 pair (base + q_lo, base + q_hi):
//   Q2_0 word (16 codes, code i at bits 2i): pairs (i, i+8), i < 8.  Fields at bits 0, 2,
//        4 use the exponents of 128, 32, 8; the word shifted by 6 and by 12 gives the rest:
//        bases 128, 32, 8, 128, 32, 8, 128, 32 for i = 0..7.
//   4-bit word (8 codes, code i at bits 4i): pairs (i, i+4), i < 4, from the word shifted
//        by 4i, base 128.
// The offsets are removed after the products, per unit (Q2) or group (4-bit):
//   Q2:    y += d * (sum_k (base_k + q_k) x_k - sum_k (base_k + 1) x_k)
//   4-bit: y += s * (sum_k (128 + q_k) x_k - (128 + z) sum_k x_k)
// which is sum_k (q - 1) d x and sum_k (q - z) s x up to f32 rounding (the products of the
// bf16 operands are exact in the f32 accumulators).
//
// k order.  In k16 step s of a unit, lane (g, c) of the MMA supplies the A slots
// {2c, 2c+1 | 2c+8, 2c+9} of weight rows g and g+8; they are two code pairs of one word of
// that lane: Q2 word c + 4 (s / 4), pairs 2 (s % 4) and 2 (s % 4) + 1; 4-bit word
// c + 4 (s / 2), pairs 2 (s % 2) and 2 (s % 2) + 1.  The staged activations put the matching
// x values at those slots, so the B fragments come from ldmatrix (8 consecutive staged
// values per token row).  The mapping is the same for A and B, so the contraction is
// unchanged; gs_stage_k() states it.
#pragma once

#include "common.cuh"

namespace tgemm {

constexpr int kGsWarps = 8;                      // compute warps
constexpr int kGsThreads = (kGsWarps + 1) * 32;  // + the weight producer warp
constexpr int kGsTile = 16;                      // weight rows per tile (mma M)
constexpr int kGsUnit = 128;                     // k per unit
constexpr int kGsMaxCluster = 8;                 // CTAs per cluster (portable limit)
constexpr int kGsRedSlots = 2;                   // partial-sum slots per reduced warp

template <int FMT>
struct GsFmt {
  static constexpr int kUnitBytes = FMT == 0 ? 32 : 64;  // packed bytes of one row-unit
  static constexpr int kWordsPerUnit = kUnitBytes / 4;
  static constexpr int kScl = FMT == 0 ? 1 : 2;          // scale entries per row-unit
  static constexpr int kSclBytes = FMT == 0 ? 2 : 4;     // bytes of one entry
  static constexpr int kCorr = FMT == 0 ? 1 : 2;         // correction sums per (unit, token)
};

// Staged position 16 s + j of a unit (s = k16 step, j = slot) holds the activation of
// unit-relative k = gs_stage_k(s, j).  Slots 2c + e (e = 0, 1) and 8 + 2c + e of lane
// column c hold the low/high halves of the lane's two code pairs for the step.
template <int FMT>
__host__ __device__ constexpr int gs_stage_k(int s, int j) {
  const int c = (j & 7) >> 1, e = j & 1, hi = j >> 3;
  if (FMT == 0) {
    const int w = c + 4 * (s >> 2), sp = s & 3;  // word of the lane, pair 2 sp + hi
    return 16 * w + 2 * sp + hi + 8 * e;          // pair i = (code i, code i + 8)
  } else {
    const int w = c + 4 * (s >> 1), h = s & 1;   // word of the lane, pair 2 h + hi
    return 8 * w + 2 * h + hi + 4 * e;            // pair i = (code i, code i + 4)
  }
}

// Q2 base of code i of a word (its pair i % 8): 128, 32, 8, 128, 32, 8, 128, 32.
__host__ __device__ constexpr int gs_q2_base(int i) {
  return (i & 7) % 3 == 0 ? 128 : ((i & 7) % 3 == 1 ? 32 : 8);
}

struct GsParams {
  const uint16_t* x;
  const uint8_t* wq;
  const uint16_t* scales;  // Q2: d [N][K/128]; 4-bit: sz [N][K/64][2]
  void* y;
  int M, N, K, out_f32;
  int U;          // units along K: ceil(K / 128)
  int C;          // CTAs per cluster (slices of K)
  int nclus;      // clusters (row ranges)
  int uq_max;     // most units of any CTA's slice
  int j_max;      // most tiles of any cluster's row range
  int S;          // ring slots
  int row_stride;  // bytes per row in a ring slot (uq_max * unit bytes + 16)
  int xs_stride;   // bytes per token row of the staged activations (uq_max * 256 + 16)
  int off_x, off_corr, off_sc, off_ring, off_red, off_bar;  // shared-memory layout
};

// ---- cluster helpers (distributed shared memory) -----------------------------------

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}

// This CTA's shared address `a` as the same variable in cluster CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void st_cluster_v4(uint32_t a, float v0, float v1, float v2, float v3) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(v0), "f"(v1),
               "f"(v2), "f"(v3)
               : "memory");
}

// Arrive on an mbarrier of a cluster CTA (address from mapa), releasing this thread's
// earlier writes at cluster scope.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t a) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(a) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait (acquire at cluster scope) for a phase completed by arrivals from other
// CTAs of the cluster; warp-uniform answer.
__device__ __forceinline__ bool mbar_wait_cluster_warp(uint32_t bar, uint32_t parity,
                                                       volatile uint32_t* abort_flag) {
  bool ok = mbar_try_wait_cluster(bar, parity);
  if (!__all_sync(0xFFFFFFFFu, ok)) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
      ok = mbar_try_wait_cluster(bar, parity);
      if (__all_sync(0xFFFFFFFFu, ok)) break;
      if ((i & 63u) == 0u) {
        int give_up = 0;
        if ((threadIdx.x & 31) == 0) {
          if (*abort_flag) {
            give_up = 1;
          } else if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort_flag = 1u;
            atomicOr(&g_device_error, kDevErrTimeout);
            give_up = 1;
          }
        }
        if (__shfl_sync(0xFFFFFFFFu, give_up, 0)) return false;
      }
    }
  }
  return true;
}

__device__ __forceinline__ void ldmatrix_x2(uint32_t saddr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(saddr));
}

__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t saddr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(saddr) : "memory");
  return v;
}

// Q2: the 8 code pairs (i, i+8) of a word as bf16 pairs (base_i + q_i, base_i + q_{i+8}).
__device__ __forceinline__ void gs_q2_pairs(uint32_t w, uint32_t (&p)[8]) {
  const uint32_t w6 = w >> 6, w12 = w >> 12;
  p[0] = lop3_and_or(w, 0x00030003u, 0x43004300u);    // 128
  p[1] = lop3_and_or(w, 0x000C000Cu, 0x42004200u);    // 32
  p[2] = lop3_and_or(w, 0x00300030u, 0x41004100u);    // 8
  p[3] = lop3_and_or(w6, 0x00030003u, 0x43004300u);   // 128
  p[4] = lop3_and_or(w6, 0x000C000Cu, 0x42004200u);   // 32
  p[5] = lop3_and_or(w6, 0x00300030u, 0x41004100u);   // 8
  p[6] = lop3_and_or(w12, 0x00030003u, 0x43004300u);  // 128
  p[7] = lop3_and_or(w12, 0x000C000Cu, 0x42004200u);  // 32
}

// 4-bit: the 4 code pairs (i, i+4) of a word as bf16 pairs (128 + q_i, 128 + q_{i+4}).
__device__ __forceinline__ void gs_q4_pairs(uint32_t w, uint32_t (&p)[4]) {
  p[0] = lop3_and_or(w, 0x000F000Fu, 0x43004300u);
  p[1] = lop3_and_or(w >> 4, 0x000F000Fu, 0x43004300u);
  p[2] = lop3_and_or(w >> 8, 0x000F000Fu, 0x43004300u);
  p[3] = lop3_and_or(w >> 12, 0x000F000Fu, 0x43004300u);
}

// T: token tiles of 8 (1 for up to 8 tokens, 2 for up to 16).
template <int FMT, int T>
__global__ void __launch_bounds__(kGsThreads, 1) gemv_stream_kernel(const GsParams p) {
  using F = GsFmt<FMT>;
  constexpr int kTok = 8 * T;
  extern __shared__ __align__(128) uint8_t gs_smem[];
  const uint32_t sb = smem_u32(gs_smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;

  const int C = p.C;
  const int q = C > 1 ? static_cast<int>(cluster_ctarank()) : 0;  // this CTA's K slice
  const int gcl = C > 1 ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  const int ua = q * p.U / C, ub = (q + 1) * p.U / C;  // units [ua, ub)
  const int uq = ub - ua;
  const int n8 = (p.N + 7) / 8;
  const int r0 = 8 * static_cast<int>(static_cast<int64_t>(gcl) * n8 / p.nclus);
  const int r1 = min(p.N, 8 * static_cast<int>(static_cast<int64_t>(gcl + 1) * n8 / p.nclus));
  const int J = r1 > r0 ? (r1 - r0 + kGsTile - 1) / kGsTile : 0;  // tiles of this cluster
  const int64_t row_bytes = FMT == 0 ? p.K / 4 : p.K / 2;
  const int kend = min(p.K, ub * kGsUnit);               // last k of the slice (exclusive)
  const int copy_bytes = FMT == 0 ? (kend - ua * kGsUnit) / 4 : (kend - ua * kGsUnit) / 2;

  // barriers: full[S], empty[S], rfull[8][R], rfree[8][R], then the abort word
  const uint32_t bar0 = sb + p.off_bar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (p.S + s); };
  auto rfull_bar = [&](int i, int s) { return bar0 + 8u * (2 * p.S + i * kGsRedSlots + s); };
  auto rfree_bar = [&](int w, int s) {
    return bar0 + 8u * (2 * p.S + kGsWarps * kGsRedSlots + w * kGsRedSlots + s);
  };
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(
      gs_smem + p.off_bar + 8 * (2 * p.S + 2 * kGsWarps * kGsRedSlots));

  if (tid == 0) {
    for (int s = 0; s < p.S; ++s) {
      mbar_init(full_bar(s), 1);   // the producer's expect_tx
      mbar_init(empty_bar(s), 1);  // the consuming warp
    }
    for (int i = 0; i < kGsWarps; ++i)
      for (int s = 0; s < kGsRedSlots; ++s) {
        mbar_init(rfull_bar(i, s), 32 * C);  // every lane of the warp in each CTA
        mbar_init(rfree_bar(i, s), 32);      // every lane of the reducing warp
      }
    *abort_flag = 0u;
    fence_mbar_init();
  }
  pdl_trigger();
  __syncwarp();
  if (C > 1) {
    cluster_sync_all();  // every CTA's barriers exist before any remote arrive
  } else {
    __syncthreads();
  }

  if (warp == kGsWarps) {
    // ---------------------------------------------------------- weight producer
    // Packed weights are not written by the kernels ahead on the stream, so the copies
    // start before the dependency wait.
    const uint32_t ring = sb + p.off_ring;
    const uint32_t slot_bytes = static_cast<uint32_t>(kGsTile * p.row_stride);
    int j = 0;
    bool ok = true;
    for (; ok && j < J; ++j) {
      const int s = j % p.S;
      const uint32_t ph = static_cast<uint32_t>(j / p.S) & 1u;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(empty_bar(s), ph ^ 1u, abort_flag))) {
        ok = false;
        break;
      }
      const int row0 = r0 + j * kGsTile;
      const int rows = min(kGsTile, r1 - row0);
      if (lane == 0) mbar_arrive_expect_tx(full_bar(s), static_cast<uint32_t>(rows * copy_bytes));
      __syncwarp();
      if (lane < rows)
        bulk_copy_g2s(ring + s * slot_bytes + lane * p.row_stride,
                      p.wq + static_cast<int64_t>(row0 + lane) * row_bytes +
                          static_cast<int64_t>(ua) * F::kUnitBytes,
                      static_cast<uint32_t>(copy_bytes), full_bar(s));
    }
    // every copy issued must land before the CTA may exit
    if (lane == 0)
      for (int jj = max(0, j - p.S); jj < j; ++jj)
        mbar_wait_drain(full_bar(jj % p.S), static_cast<uint32_t>(jj / p.S) & 1u);
    __syncwarp();
  } else {
    // ---------------------------------------------------------- compute warps
    const int nsc = FMT == 0 ? p.K / 128 : p.K / 64;  // scale entries per row
    // scales of every tile of the CTA -> shared memory (zero for rows past the range)
    {
      const int per_row = uq * F::kScl;
      const int total = J * kGsTile * per_row;
      for (int e = tid; e < total; e += kGsWarps * 32) {
        const int rt = e / per_row, si = e - rt * per_row;
        const int n = r0 + rt;
        const int sidx = ua * F::kScl + si;  // entry within the row
        uint32_t v = 0u;
        if (n < r1 && sidx < nsc) {
          const int64_t idx = static_cast<int64_t>(n) * nsc + sidx;
          v = FMT == 0 ? static_cast<uint32_t>(__ldcg(p.scales + idx))
                       : __ldcg(reinterpret_cast<const uint32_t*>(p.scales) + idx);
        }
        if (FMT == 0)
          reinterpret_cast<uint16_t*>(gs_smem + p.off_sc)[e] = static_cast<uint16_t>(v);
        else
          reinterpret_cast<uint32_t*>(gs_smem + p.off_sc)[e] = v;
      }
    }
    pdl_wait();  // the activations may come from the kernels ahead
    // activations -> shared memory in the staged order, and the correction sums
    {
      const int items = p.M * uq;
      for (int it = tid; it < items; it += kGsWarps * 32) {
        const int m = it / uq, u = it - m * uq;
        const int k0 = (ua + u) * kGsUnit;
        const int kv = min(kGsUnit, p.K - k0);  // 128, or 64 for a 4-bit half unit
        const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(m) * p.K + k0);
        uint32_t v[64];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          uint4 t = make_uint4(0u, 0u, 0u, 0u);
          if (8 * i < kv) t = __ldg(src + i);
          v[4 * i] = t.x;
          v[4 * i + 1] = t.y;
          v[4 * i + 2] = t.z;
          v[4 * i + 3] = t.w;
        }
        auto xk = [&](int k) -> uint32_t { return (v[k >> 1] >> (16 * (k & 1))) & 0xFFFFu; };
        const uint32_t dst = sb + p.off_x + m * p.xs_stride + u * (2 * kGsUnit);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          uint32_t o[8];
#pragma unroll
          for (int h = 0; h < 8; ++h)
            o[h] = xk(gs_stage_k<FMT>(s, 2 * h)) | (xk(gs_stage_k<FMT>(s, 2 * h + 1)) << 16);
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst + 32 * s), "r"(o[0]),
                       "r"(o[1]), "r"(o[2]), "r"(o[3])
                       : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst + 32 * s + 16), "r"(o[4]),
                       "r"(o[5]), "r"(o[6]), "r"(o[7])
                       : "memory");
        }
        float* corr = reinterpret_cast<float*>(gs_smem + p.off_corr);
        if (FMT == 0) {
          float sum = 0.f;  // sum_k (base_k + 1) x_k, k ascending
#pragma unroll
          for (int k = 0; k < kGsUnit; ++k)
            sum = fmaf(static_cast<float>(gs_q2_base(k) + 1), bf16_bits_to_f32(xk(k)), sum);
          corr[u * 16 + m] = sum;
        } else {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float sum = 0.f;  // sum_k x_k over the group, k ascending
#pragma unroll
            for (int k = 0; k < 64; ++k) sum += bf16_bits_to_f32(xk(64 * h + k));
            corr[(2 * u + h) * 16 + m] = sum;
          }
        }
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kGsWarps * 32) : "memory");  // compute warps only

    const uint32_t xs = sb + p.off_x;
    const float* corr = reinterpret_cast<const float*>(gs_smem + p.off_corr);
    // ldmatrix row addresses: lane l -> matrix l / 8 (token block l / 16, slot half (l / 8) % 2)
    const uint32_t lm_addr = xs + ((lane >> 4) * 8 + (lane & 7)) * p.xs_stride + ((lane >> 3) & 1) * 16;
    const uint32_t ring = sb + p.off_ring;
    const uint32_t slot_bytes = static_cast<uint32_t>(kGsTile * p.row_stride);
    bool ok = true;
    for (int kt = 0; ok; ++kt) {
      const int j = warp + kGsWarps * kt;  // this warp's k-th tile
      if (j >= J) break;
      const int s = j % p.S;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(full_bar(s), static_cast<uint32_t>(j / p.S) & 1u, abort_flag))) {
        ok = false;
        break;
      }
      float acc[T][4];
#pragma unroll
      for (int t = 0; t < T; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[t][e] = 0.f;
      const uint32_t rg = ring + s * slot_bytes + g * p.row_stride;  // row g of the slot
      const uint32_t rg8 = rg + 8 * p.row_stride;                      // row g + 8
      const int sc_row = j * kGsTile + g;                                // staged scale rows
      for (int u = 0; u < uq; ++u) {
        const uint32_t ub_off = u * F::kUnitBytes;
        if (FMT == 0) {
          const float d0 = __half2float(__ushort_as_half(
              reinterpret_cast<const uint16_t*>(gs_smem + p.off_sc)[sc_row * uq + u]));
          const float d1 = __half2float(__ushort_as_half(
              reinterpret_cast<const uint16_t*>(gs_smem + p.off_sc)[(sc_row + 8) * uq + u]));
          float pacc[T][4];
#pragma unroll
          for (int t = 0; t < T; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) pacc[t][e] = 0.f;
#pragma unroll
          for (int hw = 0; hw < 2; ++hw) {  // the lane's words c and c + 4
            uint32_t pa[8], pb[8];
            gs_q2_pairs(ld_shared_u32(rg + ub_off + 4 * (c + 4 * hw)), pa);
            gs_q2_pairs(ld_shared_u32(rg8 + ub_off + 4 * (c + 4 * hw)), pb);
#pragma unroll
            for (int sp = 0; sp < 4; ++sp) {
              const int st = 4 * hw + sp;  // k16 step of the unit
              const uint32_t a[4] = {pa[2 * sp], pb[2 * sp], pa[2 * sp + 1], pb[2 * sp + 1]};
              const uint32_t baddr = lm_addr + (u * kGsUnit + 16 * st) * 2;
              if (T == 1) {
                uint32_t b0, b1;
                ldmatrix_x2(baddr, b0, b1);
                mma_bf16_16816(pacc[0], a, b0, b1);
              } else {
                uint32_t b[4];
                ldmatrix_x4(baddr, b);
                mma_bf16_16816(pacc[0], a, b[0], b[1]);
                mma_bf16_16816(pacc[T - 1], a, b[2], b[3]);
              }
            }
          }
#pragma unroll
          for (int t = 0; t < T; ++t) {
            const float c0 = corr[u * 16 + 2 * c + 8 * t], c1 = corr[u * 16 + 2 * c + 1 + 8 * t];
            acc[t][0] = fmaf(d0, pacc[t][0] - c0, acc[t][0]);
            acc[t][1] = fmaf(d0, pacc[t][1] - c1, acc[t][1]);
            acc[t][2] = fmaf(d1, pacc[t][2] - c0, acc[t][2]);
            acc[t][3] = fmaf(d1, pacc[t][3] - c1, acc[t][3]);
          }
        } else {
          const int ng = (ua + u) * kGsUnit + 64 < p.K ? 2 : 1;  // groups in this unit
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            if (h2 >= ng) break;
            float pacc[T][4];
#pragma unroll
            for (int t = 0; t < T; ++t)
#pragma unroll
              for (int e = 0; e < 4; ++e) pacc[t][e] = 0.f;
#pragma unroll
            for (int hw = 0; hw < 2; ++hw) {  // words c + 4 (2 h2 + hw): steps 4 h2 + 2 hw + {0, 1}
              const int word = c + 4 * (2 * h2 + hw);
              uint32_t pa[4], pb[4];
              gs_q4_pairs(ld_shared_u32(rg + ub_off + 4 * word), pa);
              gs_q4_pairs(ld_shared_u32(rg8 + ub_off + 4 * word), pb);
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                const int st = 4 * h2 + 2 * hw + hh;
                const uint32_t a[4] = {pa[2 * hh], pb[2 * hh], pa[2 * hh + 1], pb[2 * hh + 1]};
                const uint32_t baddr = lm_addr + (u * kGsUnit + 16 * st) * 2;
                if (T == 1) {
                  uint32_t b0, b1;
                  ldmatrix_x2(baddr, b0, b1);
                  mma_bf16_16816(pacc[0], a, b0, b1);
                } else {
                  uint32_t b[4];
                  ldmatrix_x4(baddr, b);
                  mma_bf16_16816(pacc[0], a, b[0], b[1]);
                  mma_bf16_16816(pacc[T - 1], a, b[2], b[3]);
                }
              }
            }
            const uint32_t* scs = reinterpret_cast<const uint32_t*>(gs_smem + p.off_sc);
            const uint32_t v0 = scs[sc_row * (2 * uq) + 2 * u + h2];
            const uint32_t v1 = scs[(sc_row + 8) * (2 * uq) + 2 * u + h2];
            const float s0 = __half2float(__ushort_as_half(static_cast<uint16_t>(v0 & 0xFFFFu)));
            const float z0 = 128.f + __half2float(__ushort_as_half(static_cast<uint16_t>(v0 >> 16)));
            const float s1 = __half2float(__ushort_as_half(static_cast<uint16_t>(v1 & 0xFFFFu)));
            const float z1 = 128.f + __half2float(__ushort_as_half(static_cast<uint16_t>(v1 >> 16)));
#pragma unroll
            for (int t = 0; t < T; ++t) {
              const float S0 = corr[(2 * u + h2) * 16 + 2 * c + 8 * t];
              const float S1 = corr[(2 * u + h2) * 16 + 2 * c + 1 + 8 * t];
              acc[t][0] = fmaf(s0, fmaf(-z0, S0, pacc[t][0]), acc[t][0]);
              acc[t][1] = fmaf(s0, fmaf(-z0, S1, pacc[t][1]), acc[t][1]);
              acc[t][2] = fmaf(s1, fmaf(-z1, S0, pacc[t][2]), acc[t][2]);
              acc[t][3] = fmaf(s1, fmaf(-z1, S1, pacc[t][3]), acc[t][3]);
            }
          }
        }
      }
      // the slot's codes are read: order those generic-proxy reads before the producer's
      // next bulk copy into the slot, then release it
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(s));

      // ---- the tile's result: this CTA's K slice alone, or the cluster's sum
      const int row0 = r0 + j * kGsTile;
      if (C > 1) {
        const int rq = warp % C, ri = warp / C;  // reducing CTA and its slot set
        const int rs = kt % kGsRedSlots;
        const uint32_t rph = static_cast<uint32_t>(kt / kGsRedSlots) & 1u;
        // the reducing CTA has read this slot's previous use
        if (kt >= kGsRedSlots && !mbar_wait_cluster_warp(rfree_bar(warp, rs), rph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t red_local = sb + p.off_red +
                                   static_cast<uint32_t>((((ri * kGsRedSlots + rs) * C + q) * 32 + lane) * 16 * T);
        const uint32_t red = mapa_shared(red_local, static_cast<uint32_t>(rq));
#pragma unroll
        for (int t = 0; t < T; ++t) st_cluster_v4(red + 16 * t, acc[t][0], acc[t][1], acc[t][2], acc[t][3]);
        mbar_arrive_remote(mapa_shared(rfull_bar(ri, rs), static_cast<uint32_t>(rq)));
        if (q != rq) continue;
        // this CTA adds the C partial sums of the tile, in slice order, and stores y
        if (!mbar_wait_cluster_warp(rfull_bar(ri, rs), rph, abort_flag)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int t = 0; t < T; ++t)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[t][e] = 0.f;
        for (int qq = 0; qq < C; ++qq) {
          const float* src = reinterpret_cast<const float*>(
              gs_smem + p.off_red + (((ri * kGsRedSlots + rs) * C + qq) * 32 + lane) * 16 * T);
#pragma unroll
          for (int t = 0; t < T; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[t][e] += src[4 * t + e];
        }
        // the slot may be reused: tell every CTA's writer warp
        for (int qq = 0; qq < C; ++qq) mbar_arrive_remote(mapa_shared(rfree_bar(warp, rs), static_cast<uint32_t>(qq)));
      }
      // y[m][n]: rows g, g + 8 of the tile; tokens 2c, 2c + 1 (+ 8t)
#pragma unroll
      for (int t = 0; t < T; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int n = row0 + g + 8 * (e >> 1);
          const int m = 2 * c + (e & 1) + 8 * t;
          if (n >= r1 || m >= p.M) continue;
          if (p.out_f32)
            reinterpret_cast<float*>(p.y)[static_cast<int64_t>(m) * p.N + n] = acc[t][e];
          else
            reinterpret_cast<__nv_bfloat16*>(p.y)[static_cast<int64_t>(m) * p.N + n] =
                __float2bfloat16_rn(acc[t][e]);
        }
    }
    (void)kTok;
  }

  // ---------------------------------------------------------- teardown
  // No CTA leaves while another CTA of its cluster may still write into its shared memory
  // or arrive on its barriers (every wait above is bounded, so all CTAs get here).
  __syncwarp();
  if (C > 1) cluster_sync_all();
}

}  // namespace tgemm
