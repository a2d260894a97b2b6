// Backward kernels: delta preprocess, dQ convert, and the parameters of the
// dQ/dK/dV main kernels (fa_bwd_pipe.cuh for d = 64, fa_bwd_pipe128.cuh for
// d = 128).
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
//                (the kernels apply 1/l as the exponent offset -log2(l), so
//                P = exp2((S - m) log2(e) - (lse - m) log2(e)): one exp2 per score),
//                with m the row shift the forward selected.
//
// Main kernels: a work item is one (batch, head, 128-key block), looping over
// the 128-query blocks that see those keys.  They work in the transposed
// orientation so that P^T and dS^T (lane = key) feed the dV and dK products
// straight from TMEM.  Products per query block (M = N = 128 unless noted,
// K-dim 16 per MMA):
//   S^T  = K  Q_i^T   (A: K  smem K-major, B: Q_i  smem K-major)
//   dP^T = V  dO_i^T  (A: V  smem K-major, B: dO_i smem K-major)
//   dV  += P^T  dO_i  (A: P^T  TMEM,     B: dO_i smem MN-major, N = d)
//   dK  += dS^T Q_i   (A: dS^T from TMEM, written over dP^T columns the
//                      elementwise warps have read, B: Q_i smem MN-major, N = d)
//   dQ_i = dS   K     (A: dS smem MN-major (written from dS^T), B: K MN-major)
#pragma once

#include "fa_fwd.cuh"

namespace fa {

// ------------------------------------------------------------------ delta
// delta[r] = sum_c dO[r,c] * O[r,c] in fp32; also clears the dQ accumulator
// and the work-item counter behind it.  O is the bf16 output of the
// forward, or (OT = float) its fp32 value before rounding (the
// high-precision O_hp of the pages).
// Memory bound: each row of O and dO is read once with 16-byte loads, LPR
// lanes per row (8 elements of dO per lane); every warp takes U row groups at
// a time and issues all of their loads before using any.  Blocks of 128
// threads at no more than 32 registers fit beside the forward kernel's CTAs
// (two per SM, 80 registers x 384 threads each), so with programmatic
// dependent launch they are resident when the forward ends (measured: g2s
// step 123.0 -> 122.4 us, long 2415 -> 2392 us, against 256-thread blocks).
// The clear does not depend on the forward: the first clear_blocks blocks
// zero one contiguous share of the accumulator each before they wait for the
// forward grid.  When the accumulator is small (a quarter of L2 at most) the
// host makes that one block per SM, the blocks resident beside the forward's
// CTAs, so the whole clear runs while the forward does (g2s step 116.7 ->
// 115.7 us); a larger one is shared by every block, since clearing it beside
// the forward would push the forward's K and V tiles out of L2 (long: 2546
// against 2373 us).  Against clearing each block's rows in the dot loop the
// shared form took the g2s step from 123.1 to 121.3 us and long from 2396 to
// 2373 us.  In the same place each
// block asks for its share of dO to be brought into L2 (neutral on g2s and
// tiestress, long step ~2420 -> ~2375 us over three runs).  The one kernel of this
// library that reads the accumulator, the dQ convert of an earlier call, lets
// its dependents start only after its last read.
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
__global__ void __launch_bounds__(128, 16)
fa_bwd_delta_kernel(const OT* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
                    float* __restrict__ delta, float* __restrict__ dq_acc, long long rows, int clear_blocks) {
  constexpr int LPR = D / 8;               // lanes per row (8 elements per lane)
  constexpr int RPW = 32 / LPR;            // rows per warp per group
  constexpr int U = 2;                     // row groups per warp per pass
  const int lane = threadIdx.x & 31;
  const long long warp_global = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const int sub = lane / LPR, li = lane % LPR;
  if (static_cast<int>(blockIdx.x) < clear_blocks) {
    const long long n4 = rows * (D / 4);
    const long long lo = n4 * blockIdx.x / clear_blocks, hi = n4 * (blockIdx.x + 1) / clear_blocks;
    float4* acc4 = reinterpret_cast<float4*>(dq_acc);
    for (long long i = lo + threadIdx.x; i < hi; i += blockDim.x) acc4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    // the 256-byte block after the accumulator (the d = 128 kernel's work-item counter)
    if (blockIdx.x == 0 && threadIdx.x < 64) reinterpret_cast<unsigned int*>(dq_acc + rows * D)[threadIdx.x] = 0u;
  }
  // and its share of dO into L2 (a prefetch is only a hint, so it is harmless
  // even if the previous grid is still writing dO)
  if (threadIdx.x == 0) {
    const long long nb = rows * D * 2;  // bytes of dO; its base is 16-byte aligned (checked by its tensor map)
    const long long lo = (nb * blockIdx.x / gridDim.x) & ~15ll;
    const long long hi = (blockIdx.x + 1 == gridDim.x) ? nb : ((nb * (blockIdx.x + 1) / gridDim.x) & ~15ll);
    for (long long a = lo; a < hi; a += (1ll << 20)) {
      const long long n = (hi - a < (1ll << 20)) ? (hi - a) : (1ll << 20);
      bulk_prefetch_l2(reinterpret_cast<const char*>(dO) + a, static_cast<uint32_t>(n));
    }
  }
  grid_dependency_wait();  // O comes from the forward grid
  // Dependents launch only now, when every grid before this one in the
  // stream has completed: the d = 64 main kernel therefore reads its inputs
  // without a dependency wait of its own, and only its drain warps (delta,
  // the cleared accumulator) wait for this grid, so its loads and first
  // products overlap this kernel (g2s step 118.2 -> 117.4 us).
  grid_launch_dependents();
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
  // the delta kernel of a later call clears the accumulator before its own
  // dependency wait: let it start only once every read here has been used
  __syncthreads();
  grid_launch_dependents();
}

// --------------------------------------------------------------- main kernel
struct BwdParams {
  const float* lse;    // [BH, N]
  const float* row_m;  // [BH, N], stabilised mode only
  const float* delta;  // [BH, N]
  float* dq_acc;       // [BH, N, D] fp32, zeroed by the delta kernel
  unsigned int* item_ctr;  // d = 128: next unclaimed work item (zeroed by the delta kernel)
  int head_group;          // d = 128: heads per group of the item order
  __nv_bfloat16* dk;   // [BH, N, D]
  __nv_bfloat16* dv;   // [BH, N, D]
  int BH, N, n_blk;
  int causal, mode;
  float scale;
};

}  // namespace fa
