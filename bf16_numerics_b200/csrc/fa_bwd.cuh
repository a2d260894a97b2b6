// Backward kernels: delta preprocess, the dQ/dK/dV main kernel, dQ convert.
//
// Gradient of O = softmax(S) V with S = Q K^T * scale (the standard
// attention backward; the pages name its delta step -- 91haoming.cn page,
// section 3: an elementwise product of two matrices followed by a row sum --
// and the dP term -- itsolotime.com/archives/23922, "core finding"):
//   delta = rowsum(dO o O)
//   P     = softmax(S), recomputed from the saved statistics
//   dV = P^T dO,  dP = dO V^T,  dS = P o (dP - delta),
//   dQ = dS K * scale,  dK = dS^T Q * scale.
// The recompute follows the softmax mode:
//   standard   : P = exp(S - lse)
//   stabilised : P_bar = exp(S - m), P = P_bar * (1/l), l = exp(lse - m),
//                with m the row shift the forward selected.
//
// Main kernel: one CTA per (batch, head, 128-key block), looping over the
// 128-query blocks that see those keys.  It works in the transposed
// orientation so that P^T and dS^T (lane = key) feed the dV and dK products
// straight from TMEM:
//   warps 0-3  softmax/dS: thread t owns key t of the block;
//   warps 4-7  dQ drain: thread t owns query t of the current block and adds
//              its row of the dQ partial into an fp32 accumulator with
//              vector reductions;
//   warp  8    TMA producer (K, V once; Q_i, dO_i through a ring);
//   warp  9    MMA issuer and TMEM owner.
// Products per query block (M = N = 128 unless noted, K-dim 16 per MMA):
//   S^T  = K  Q_i^T   (A: K  smem K-major, B: Q_i  smem K-major)
//   dP^T = V  dO_i^T  (A: V  smem K-major, B: dO_i smem K-major)
//   dV  += P^T  dO_i  (A: P^T  TMEM,     B: dO_i smem MN-major, N = d)
//   dK  += dS^T Q_i   (A: dS^T TMEM,     B: Q_i  smem MN-major, N = d)
//   dQ_i = dS   K     (A: dS smem MN-major (written from dS^T), B: K MN-major)
#pragma once

#include "fa_fwd.cuh"

namespace fa {

// ------------------------------------------------------------------ delta
// delta[r] = sum_c dO[r,c] * O[r,c] in fp32; also clears the dQ accumulator
// row.  O is the bf16 output of the forward, or (OT = float) its fp32 value
// before rounding (the high-precision O_hp of the pages).
// Memory bound: each row of O and dO is read once with 16-byte loads, LPR
// lanes per row (8 elements of dO per lane); every warp takes U row groups at
// a time and issues all of their loads before using any, so enough bytes are
// in flight to cover the DRAM latency.
// 8 consecutive elements of O as they sit in memory (16 bytes of bf16 or
// 32 bytes of fp32), and their dot product with 8 bf16 elements of dO
template <typename OT>
struct ORaw;
template <>
struct ORaw<__nv_bfloat16> {
  uint4 v;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { v = __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ __forceinline__ void zero() { v = make_uint4(0u, 0u, 0u, 0u); }
  __device__ __forceinline__ float dot(const uint4& d, float acc) const {
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&v);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&d);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 a = __bfloat1622float2(pa[i]), b = __bfloat1622float2(pb[i]);
      acc = fmaf(a.x, b.x, acc);
      acc = fmaf(a.y, b.y, acc);
    }
    return acc;
  }
};
template <>
struct ORaw<float> {
  float4 lo, hi;
  __device__ __forceinline__ void load(const float* p) {
    lo = __ldg(reinterpret_cast<const float4*>(p));
    hi = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ void zero() { lo = hi = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ float dot(const uint4& d, float acc) const {
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&d);
    float2 b = __bfloat1622float2(pb[0]);
    acc = fmaf(lo.x, b.x, acc);
    acc = fmaf(lo.y, b.y, acc);
    b = __bfloat1622float2(pb[1]);
    acc = fmaf(lo.z, b.x, acc);
    acc = fmaf(lo.w, b.y, acc);
    b = __bfloat1622float2(pb[2]);
    acc = fmaf(hi.x, b.x, acc);
    acc = fmaf(hi.y, b.y, acc);
    b = __bfloat1622float2(pb[3]);
    acc = fmaf(hi.z, b.x, acc);
    acc = fmaf(hi.w, b.y, acc);
    return acc;
  }
};

template <int D, typename OT>
__global__ void __launch_bounds__(256)
fa_bwd_delta_kernel(const OT* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
                    float* __restrict__ delta, float* __restrict__ dq_acc, long long rows) {
  constexpr int LPR = D / 8;               // lanes per row (8 elements per lane)
  constexpr int RPW = 32 / LPR;            // rows per warp per group
  constexpr int U = 4;                     // row groups per warp per pass
  const int lane = threadIdx.x & 31;
  const long long warp_global = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const int sub = lane / LPR, li = lane % LPR;
  grid_launch_dependents();
  grid_dependency_wait();  // O comes from the forward grid
  for (long long r0 = warp_global * (RPW * U); r0 < rows; r0 += n_warps * (RPW * U)) {
    ORaw<OT> a[U];
    uint4 b[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long r = r0 + u * RPW + sub;
      if (r < rows) {
        a[u].load(o + r * D + 8 * li);
        b[u] = __ldg(reinterpret_cast<const uint4*>(dO + r * D) + li);
      } else {
        a[u].zero();
        b[u] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long r = r0 + u * RPW + sub;
      if (r < rows) {
        float4* z = reinterpret_cast<float4*>(dq_acc + r * D) + 2 * li;
        z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float acc = a[u].dot(b[u], 0.f);
#pragma unroll
      for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      const long long r = r0 + u * RPW + sub;
      if (r < rows && li == 0) delta[r] = acc;
    }
  }
}

// --------------------------------------------------------------- dQ convert
// dq = bf16(dq_acc), 8 values per thread and chunk, U chunks per thread per
// pass with all loads issued first; the accumulator is dead afterwards, so
// it is read with the streaming (evict-first) hint.
__global__ void __launch_bounds__(256)
fa_bwd_dq_convert_kernel(const float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dq, long long n8) {
  constexpr int U = 4;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  grid_launch_dependents();
  grid_dependency_wait();  // the accumulator is complete once the main grid is
  for (long long i0 = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i0 < n8; i0 += stride * U) {
    float4 a[U], b[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long i = i0 + u * stride;
      if (i < n8) {
        a[u] = __ldcs(reinterpret_cast<const float4*>(dq_acc) + 2 * i);
        b[u] = __ldcs(reinterpret_cast<const float4*>(dq_acc) + 2 * i + 1);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long i = i0 + u * stride;
      if (i < n8) {
        uint4 w;
        w.x = pack_bf16x2(a[u].x, a[u].y);
        w.y = pack_bf16x2(a[u].z, a[u].w);
        w.z = pack_bf16x2(b[u].x, b[u].y);
        w.w = pack_bf16x2(b[u].z, b[u].w);
        reinterpret_cast<uint4*>(dq)[i] = w;
      }
    }
  }
}

// --------------------------------------------------------------- main kernel
struct BwdParams {
  const float* lse;    // [BH, N]
  const float* row_m;  // [BH, N], stabilised mode only
  const float* delta;  // [BH, N]
  float* dq_acc;       // [BH, N, D] fp32, zeroed by the delta kernel
  __nv_bfloat16* dk;   // [BH, N, D]
  __nv_bfloat16* dv;   // [BH, N, D]
  int BH, N, n_blk;
  int causal, mode;
  float scale;
};

template <int D>
struct BwdLayout {
  static constexpr int B = 128;                // keys per CTA, queries per step
  static constexpr int TILE = B * D * 2;
  static constexpr int HALF = 128 * 128;
  static constexpr int ST = (D == 64) ? 2 : 1; // Q/dO ring depth
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + TILE;
  static constexpr int Q_OFF = V_OFF + TILE;            // ST tiles
  static constexpr int DO_OFF = Q_OFF + ST * TILE;      // ST tiles
  static constexpr int DS_OFF = DO_OFF + ST * TILE;     // dS^T, [keys][queries], two 64-query halves
  static constexpr int VEC_OFF = DS_OFF + 2 * HALF;     // per query: a, b, delta (fp32 x 128 each)
  static constexpr int BAR_OFF = VEC_OFF + 3 * 128 * 4;
  enum { KV_FULL = 0, Q_FULL = 1, Q_EMPTY = 1 + ST, S_FULL = 1 + 2 * ST, DP_FULL, PDS_FULL, DQ_FULL, DQ_FREE,
         ACC_DONE, TEARDOWN, NBAR };
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int USED = MISC_OFF + 16;
  static constexpr int SMEM_BYTES = (USED + 1024 > 120 * 1024 ? USED + 1024 : 120 * 1024);
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t ST_COL = 0, DPT_COL = 128, DV_COL = 256, DK_COL = 256 + D;
  static constexpr uint32_t DQ_COL = (D == 64) ? 384 : 0;  // d = 128: dQ reuses the S^T columns
};

template <int D>
__global__ void __launch_bounds__(320, 1)
fa_bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                   const BwdParams p) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);
  auto bar = [&](int i) { return base + L::BAR_OFF + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  float* vec_a = reinterpret_cast<float*>(smem + L::VEC_OFF);  // mode 0: lse*log2e; mode 1: m
  float* vec_b = vec_a + 128;                                  // mode 1: 1/l
  float* vec_d = vec_b + 128;                                  // delta
  const BoundedWait wait{abort_flag, 2u};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = p.BH;
  const int kblk = blockIdx.x / BH;  // low key blocks (most query blocks when causal) first
  const int bh = blockIdx.x - kblk * BH;
  const int i0 = p.causal ? kblk : 0;
  const int n_it = p.n_blk - i0;

  if (threadIdx.x == 0) {
    mbar_init(bar(L::KV_FULL), 1);
    for (int s = 0; s < L::ST; ++s) {
      mbar_init(bar(L::Q_FULL + s), 1);
      mbar_init(bar(L::Q_EMPTY + s), 1);
    }
    mbar_init(bar(L::S_FULL), 1);
    mbar_init(bar(L::DP_FULL), 1);
    mbar_init(bar(L::PDS_FULL), 128);
    mbar_init(bar(L::DQ_FULL), 1);
    mbar_init(bar(L::DQ_FREE), 128);
    mbar_init(bar(L::ACC_DONE), 1);
    mbar_init(bar(L::TEARDOWN), 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
    tmem_relinquish();
  }
  grid_launch_dependents();
  grid_dependency_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_expect_tx(bar(L::KV_FULL), 2 * L::TILE);
      for (int h = 0; h < D / 64; ++h) {
        tma_load_3d(base + L::K_OFF + h * L::HALF, &tm_k, bar(L::KV_FULL), 64 * h, kblk * L::B, bh);
        tma_load_3d(base + L::V_OFF + h * L::HALF, &tm_v, bar(L::KV_FULL), 64 * h, kblk * L::B, bh);
      }
      int issued[L::ST];
      for (int s = 0; s < L::ST; ++s) issued[s] = -1;
      for (int it = 0; it < n_it; ++it) {
        const int s = it % L::ST, use = it / L::ST;
        if (use > 0 && !wait(bar(L::Q_EMPTY + s), (use - 1) & 1, 1)) break;
        const int row0 = (i0 + it) * L::B;
        mbar_expect_tx(bar(L::Q_FULL + s), 2 * L::TILE);
        for (int h = 0; h < D / 64; ++h) {
          tma_load_3d(base + L::Q_OFF + s * L::TILE + h * L::HALF, &tm_q, bar(L::Q_FULL + s), 64 * h, row0, bh);
          tma_load_3d(base + L::DO_OFF + s * L::TILE + h * L::HALF, &tm_do, bar(L::Q_FULL + s), 64 * h, row0, bh);
        }
        issued[s] = it;
      }
      volatile int never = 0;
      const BoundedWait drain{&never, 2u};
      drain(bar(L::KV_FULL), 0, 20);
      for (int s = 0; s < L::ST; ++s)
        if (issued[s] >= 0) drain(bar(L::Q_FULL + s), (issued[s] / L::ST) & 1, 21);
    }
    __syncwarp();
  } else if (warp == 9) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_SQ = idesc_bf16_f32(128, 128, false, false);  // S^T, dP^T
      constexpr uint32_t IDESC_KV = idesc_bf16_f32(128, D, false, true);     // dV, dK
      constexpr uint32_t IDESC_DQ = idesc_bf16_f32(128, D, true, true);      // dQ
      bool ok = wait(bar(L::KV_FULL), 0, 2);
      for (int it = 0; ok && it < n_it; ++it) {
        const int s = it % L::ST, use = it / L::ST;
        if (!wait(bar(L::Q_FULL + s), use & 1, 3)) break;
        if (L::DQ_COL == L::ST_COL && it > 0 && !wait(bar(L::DQ_FREE), (it - 1) & 1, 4)) break;
        tc_fence_after();
        const uint32_t q_t = base + L::Q_OFF + s * L::TILE, do_t = base + L::DO_OFF + s * L::TILE;
        // S^T = K Q_i^T
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t koff = (ks >> 2) * L::HALF + (ks & 3) * 32;
          mma_ss(tmem + L::ST_COL, sdesc_sw128(base + L::K_OFF + koff, 16, 1024), sdesc_sw128(q_t + koff, 16, 1024),
                 IDESC_SQ, ks > 0 ? 1u : 0u);
        }
        tc_commit(bar(L::S_FULL));
        // dP^T = V dO_i^T
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t koff = (ks >> 2) * L::HALF + (ks & 3) * 32;
          mma_ss(tmem + L::DPT_COL, sdesc_sw128(base + L::V_OFF + koff, 16, 1024), sdesc_sw128(do_t + koff, 16, 1024),
                 IDESC_SQ, ks > 0 ? 1u : 0u);
        }
        tc_commit(bar(L::DP_FULL));
        if (!wait(bar(L::PDS_FULL), it & 1, 5)) break;
        if (L::DQ_COL != L::ST_COL && it > 0 && !wait(bar(L::DQ_FREE), (it - 1) & 1, 6)) break;
        tc_fence_after();
        // dV += P^T dO_i ; dK += dS^T Q_i   (K-dim = queries, 16 per MMA)
#pragma unroll
        for (int ks = 0; ks < L::B / 16; ++ks) {
          mma_ts(tmem + L::DV_COL, tmem + L::ST_COL + 8u * ks, sdesc_sw128(do_t + ks * 2048, L::HALF, 1024), IDESC_KV,
                 (it > 0 || ks > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int ks = 0; ks < L::B / 16; ++ks) {
          mma_ts(tmem + L::DK_COL, tmem + L::DPT_COL + 8u * ks, sdesc_sw128(q_t + ks * 2048, L::HALF, 1024), IDESC_KV,
                 (it > 0 || ks > 0) ? 1u : 0u);
        }
        // dQ_i = dS K   (K-dim = keys, 16 per MMA)
#pragma unroll
        for (int ks = 0; ks < L::B / 16; ++ks) {
          mma_ss(tmem + L::DQ_COL, sdesc_sw128(base + L::DS_OFF + ks * 2048, L::HALF, 1024),
                 sdesc_sw128(base + L::K_OFF + ks * 2048, L::HALF, 1024), IDESC_DQ, ks > 0 ? 1u : 0u);
        }
        tc_commit(bar(L::DQ_FULL));
        tc_commit(bar(L::Q_EMPTY + s));
      }
      tc_commit(bar(L::ACC_DONE));
      tc_commit(bar(L::TEARDOWN));
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------- dQ drain warps
    const int t = threadIdx.x - 128;  // query row within the block == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp - 4) * 32) << 16;
    const float scale = p.scale;
    for (int it = 0; it < n_it; ++it) {
      if (!wait(bar(L::DQ_FULL), it & 1, 7)) break;
      tc_fence_after();
      const int q_row = (i0 + it) * L::B + t;
      float* dst = p.dq_acc + (static_cast<size_t>(bh) * p.N + q_row) * D;
      const bool row_ok = q_row < p.N;
      if (D == 64) {
        uint32_t r0[32], r1[32];
        tmem_ld32x2(tmem + lane_base + L::DQ_COL, tmem + lane_base + L::DQ_COL + 32, r0, r1);
        tc_fence_before();
        mbar_arrive(bar(L::DQ_FREE));
        if (row_ok) {
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            red_add_v4(dst + c, __uint_as_float(r0[c]) * scale, __uint_as_float(r0[c + 1]) * scale,
                       __uint_as_float(r0[c + 2]) * scale, __uint_as_float(r0[c + 3]) * scale);
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            red_add_v4(dst + 32 + c, __uint_as_float(r1[c]) * scale, __uint_as_float(r1[c + 1]) * scale,
                       __uint_as_float(r1[c + 2]) * scale, __uint_as_float(r1[c + 3]) * scale);
        }
      } else {
        uint32_t r0[32], r1[32], r2[32], r3[32];
        tmem_ld32x2(tmem + lane_base + L::DQ_COL, tmem + lane_base + L::DQ_COL + 32, r0, r1);
        tmem_ld32x2(tmem + lane_base + L::DQ_COL + 64, tmem + lane_base + L::DQ_COL + 96, r2, r3);
        tc_fence_before();
        mbar_arrive(bar(L::DQ_FREE));
        if (row_ok) {
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            red_add_v4(dst + c, __uint_as_float(r0[c]) * scale, __uint_as_float(r0[c + 1]) * scale,
                       __uint_as_float(r0[c + 2]) * scale, __uint_as_float(r0[c + 3]) * scale);
            red_add_v4(dst + 32 + c, __uint_as_float(r1[c]) * scale, __uint_as_float(r1[c + 1]) * scale,
                       __uint_as_float(r1[c + 2]) * scale, __uint_as_float(r1[c + 3]) * scale);
            red_add_v4(dst + 64 + c, __uint_as_float(r2[c]) * scale, __uint_as_float(r2[c + 1]) * scale,
                       __uint_as_float(r2[c + 2]) * scale, __uint_as_float(r2[c + 3]) * scale);
            red_add_v4(dst + 96 + c, __uint_as_float(r3[c]) * scale, __uint_as_float(r3[c + 1]) * scale,
                       __uint_as_float(r3[c + 2]) * scale, __uint_as_float(r3[c + 3]) * scale);
          }
        }
      }
    }
  } else {
    // ---------------------------------------------------- softmax/dS warps 0..3
    const int t = threadIdx.x;  // key within the block == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int key = kblk * L::B + t;
    const float scale = p.scale;
    const size_t vrow0 = static_cast<size_t>(bh) * p.N;
    // per-query vectors of the next block, prefetched one step ahead
    auto fetch = [&](int it, float& a, float& b, float& dl) {
      const int q = (i0 + it) * L::B + t;
      if (it < n_it && q < p.N) {
        const float lse = __ldg(p.lse + vrow0 + q);
        dl = __ldg(p.delta + vrow0 + q);
        if (p.mode == 1) {
          const float m = __ldg(p.row_m + vrow0 + q);
          a = m;
          b = 1.f / ex2_approx((lse - m) * kLog2e);
        } else {
          a = lse * kLog2e;
          b = 1.f;
        }
      } else {
        a = INFINITY;  // padded query rows: P = 0
        b = 0.f;
        dl = 0.f;
      }
    };
    float na, nb, nd;
    fetch(0, na, nb, nd);
    // A bounded wait that gives up only clears `ok`; the four warps leave the
    // loop together at the AND vote that opens the next iteration.
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int i = i0 + it;
      // publish this block's vectors (all 128 softmax threads), then prefetch the next
      if (!named_barrier_and(1, 128, ok)) break;
      vec_a[t] = na;
      vec_b[t] = nb;
      vec_d[t] = nd;
      named_barrier_sync_128();
      fetch(it + 1, na, nb, nd);
      // dS smem is free once the previous dQ product has completed
      ok = (it == 0 || wait.warp(bar(L::DQ_FULL), (it - 1) & 1, 8));
      ok = ok && wait.warp(bar(L::S_FULL), it & 1, 9);
      ok = ok && wait.warp(bar(L::DP_FULL), it & 1, 10);
      if (!ok) continue;
      tc_fence_after();
      const bool diag = p.causal && (i == kblk);
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t rs_[32], rd_[32];
        tmem_ld32x2(tmem + lane_base + L::ST_COL + c0, tmem + lane_base + L::DPT_COL + c0, rs_, rd_);
        uint32_t pk[16], dk_[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          float pv[2], dsv[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int qc = c0 + c + e;
            const float s = __uint_as_float(rs_[c + e]) * scale;
            float pe;
            if (p.mode == 1) {
              pe = ex2_approx((s - vec_a[qc]) * kLog2e) * vec_b[qc];
            } else {
              pe = ex2_approx(fmaf(s, kLog2e, -vec_a[qc]));
            }
            if (diag && t > qc) pe = 0.f;  // key after query: masked
            if (vec_b[qc] == 0.f) pe = 0.f;
            pv[e] = pe;
            dsv[e] = pe * (__uint_as_float(rd_[c + e]) - vec_d[qc]);
          }
          pk[c >> 1] = pack_bf16x2(pv[0], pv[1]);
          dk_[c >> 1] = pack_bf16x2(dsv[0], dsv[1]);
        }
        tmem_st16(tmem + lane_base + L::ST_COL + (c0 >> 1), pk);
        tmem_st16(tmem + lane_base + L::DPT_COL + (c0 >> 1), dk_);
        // dS^T row (key t) into the 128B-swizzled [keys][queries] tile:
        // 16-byte chunk j of a 128-byte row r lives at chunk (j ^ (r & 7)).
        const int half = c0 >> 6;
        uint8_t* row_base = smem + L::DS_OFF + half * L::HALF + t * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int chunk = ((c0 & 63) >> 3) + j;
          *reinterpret_cast<uint4*>(row_base + ((chunk ^ (t & 7)) << 4)) =
              make_uint4(dk_[4 * j], dk_[4 * j + 1], dk_[4 * j + 2], dk_[4 * j + 3]);
        }
      }
      fence_proxy_async_smem();
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::PDS_FULL));
    }
    // ------------------------------------------------------------- epilogue
    if (ok && wait.warp(bar(L::ACC_DONE), 0, 11)) {
      tc_fence_after();
      const bool row_ok = key < p.N;
      __nv_bfloat16* dk_row = p.dk + (vrow0 + key) * D;
      __nv_bfloat16* dv_row = p.dv + (vrow0 + key) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t rk[32], rv[32];
        tmem_ld32x2(tmem + lane_base + L::DK_COL + c0, tmem + lane_base + L::DV_COL + c0, rk, rv);
        if (row_ok) {
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            uint4 wk, wv;
            wk.x = pack_bf16x2(__uint_as_float(rk[c + 0]) * scale, __uint_as_float(rk[c + 1]) * scale);
            wk.y = pack_bf16x2(__uint_as_float(rk[c + 2]) * scale, __uint_as_float(rk[c + 3]) * scale);
            wk.z = pack_bf16x2(__uint_as_float(rk[c + 4]) * scale, __uint_as_float(rk[c + 5]) * scale);
            wk.w = pack_bf16x2(__uint_as_float(rk[c + 6]) * scale, __uint_as_float(rk[c + 7]) * scale);
            wv.x = pack_bf16x2(__uint_as_float(rv[c + 0]), __uint_as_float(rv[c + 1]));
            wv.y = pack_bf16x2(__uint_as_float(rv[c + 2]), __uint_as_float(rv[c + 3]));
            wv.z = pack_bf16x2(__uint_as_float(rv[c + 4]), __uint_as_float(rv[c + 5]));
            wv.w = pack_bf16x2(__uint_as_float(rv[c + 6]), __uint_as_float(rv[c + 7]));
            *reinterpret_cast<uint4*>(dk_row + c0 + c) = wk;
            *reinterpret_cast<uint4*>(dv_row + c0 + c) = wv;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    volatile int never = 0;
    const BoundedWait drain{&never, 2u};
    drain(bar(L::TEARDOWN), 0, 30);
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace fa
