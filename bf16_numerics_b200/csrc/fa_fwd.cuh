// Forward kernel: tiled attention with the stabilised safe softmax.
//
// Method (Qiu & Yao, arXiv 2510.04212; itsolotime.com/archives/23922,
// "mechanism two" and "minimal fix"):
//   S = Q K^T * scale, rm = rowmax(S), rs = rowsum(S == rm),
//   m = beta*rm (rs>1, rm>0) | 0 (rs>1, rm<0) | beta-1 (rs>1, rm==0) | rm,
//   P_bar = exp(S - m), P = P_bar / rowsum(P_bar), O = P V, lse = m + ln(l).
// The row statistics are kept online across key tiles: a later tile with a
// larger maximum resets (rm, rs); an equal maximum adds its tie count; whenever
// the selected shift m changes, the running sum l and the O accumulator are
// rescaled by exp(m_old - m_new) before the tile's P_bar is formed, so every
// P_bar operand is computed against the shift in force for the rows seen so
// far (the final shift once the last tile has been merged).
//
// One CTA computes one 128-row Q tile of one (batch, head):
//   warps 0-3  softmax: thread t owns row t (TMEM lane t); S, P_bar, O
//              rescale and the epilogue;
//   warp  4    TMA producer (Q once, K/V through a 2-stage ring);
//   warp  5    MMA issuer (one thread) and TMEM owner.
// TMEM columns: S0 [0,128) S1 [128,256) P0 [256,320) P1 [320,384)
//               O [384, 384+D).  P_bar is stored back into TMEM as packed
// bf16 pairs and fed to the P V product as the A operand straight from TMEM.
#pragma once

#include "fa_ptx.cuh"

namespace fa {

constexpr float kLog2e = 1.4426950408889634f;

struct FwdParams {
  __nv_bfloat16* o;   // [BH, N, D]
  float* lse;         // [BH, N]
  float* st_rm;       // optional [BH, N]
  int32_t* st_rs;     // optional
  float* st_m;        // optional
  float* st_pbar_max; // optional
  int BH, N, n_qblk;
  int causal, mode;
  float beta, scale;
};

template <int D>
struct FwdLayout {
  static constexpr int BM = 128, BN = 128;
  static constexpr int TILE = BM * D * 2;  // bytes of a 128 x D bf16 tile
  static constexpr int HALF = 128 * 128;   // bytes of one 128-row x 64-col TMA box
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + TILE;
  static constexpr int V_OFF = K_OFF + 2 * TILE;
  static constexpr int BAR_OFF = V_OFF + 2 * TILE;
  // barrier indices
  enum { Q_FULL = 0, K_FULL = 1, V_FULL = 3, KV_EMPTY = 5, S_FULL = 7, S_FREE = 9, P_FULL = 11,
         O_READY = 13, TEARDOWN = 14, NBAR = 15 };
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;  // tmem base (4B), abort flag (4B)
  static constexpr int USED = MISC_OFF + 16;
  // force one CTA per SM: each CTA owns all 512 TMEM columns
  static constexpr int SMEM_BYTES = (USED + 1024 > 120 * 1024 ? USED + 1024 : 120 * 1024);
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL0 = 0, P_COL0 = 256, O_COL = 384;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using L = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;  // 1024-byte aligned for the 128B swizzle
  uint8_t* smem = smem_raw + (base - raw_addr);
  auto bar = [&](int i) { return base + L::BAR_OFF + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  const BoundedWait wait{abort_flag, 1u};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = p.BH;
  const int tile_rev = blockIdx.x / BH;
  const int bh = blockIdx.x - tile_rev * BH;
  const int qblk = p.causal ? (p.n_qblk - 1 - tile_rev) : tile_rev;  // longest causal rows first
  const int n_kblk_all = (p.N + L::BN - 1) / L::BN;
  const int nkv = p.causal ? (qblk + 1) : n_kblk_all;

  if (threadIdx.x == 0) {
    mbar_init(bar(L::Q_FULL), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::K_FULL + s), 1);
      mbar_init(bar(L::V_FULL + s), 1);
      mbar_init(bar(L::KV_EMPTY + s), 1);
      mbar_init(bar(L::S_FULL + s), 1);
      mbar_init(bar(L::S_FREE + s), 128);
      mbar_init(bar(L::P_FULL + s), 128);
    }
    mbar_init(bar(L::O_READY), 1);
    mbar_init(bar(L::TEARDOWN), 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int issued[2] = {-1, -1};
      mbar_expect_tx(bar(L::Q_FULL), L::TILE);
      for (int h = 0; h < D / 64; ++h)
        tma_load_3d(base + L::Q_OFF + h * L::HALF, &tm_q, bar(L::Q_FULL), 64 * h, qblk * L::BM, bh);
      for (int j = 0; j < nkv; ++j) {
        const int s = j & 1;
        if (j >= 2 && !wait(bar(L::KV_EMPTY + s), ((j >> 1) - 1) & 1, 1)) break;
        mbar_expect_tx(bar(L::K_FULL + s), L::TILE);
        for (int h = 0; h < D / 64; ++h)
          tma_load_3d(base + L::K_OFF + s * L::TILE + h * L::HALF, &tm_k, bar(L::K_FULL + s), 64 * h, j * L::BN, bh);
        mbar_expect_tx(bar(L::V_FULL + s), L::TILE);
        for (int h = 0; h < D / 64; ++h)
          tma_load_3d(base + L::V_OFF + s * L::TILE + h * L::HALF, &tm_v, bar(L::V_FULL + s), 64 * h, j * L::BN, bh);
        issued[s] = j;
      }
      // drain: every load issued must have landed before the CTA may exit
      volatile int never = 0;
      const BoundedWait drain{&never, 1u};
      for (int s = 0; s < 2; ++s) {
        if (issued[s] >= 0) {
          drain(bar(L::K_FULL + s), (issued[s] >> 1) & 1, 20);
          drain(bar(L::V_FULL + s), (issued[s] >> 1) & 1, 21);
        }
      }
      drain(bar(L::Q_FULL), 0, 22);
    }
    __syncwarp();
  } else if (warp == 5) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, false, true);
      bool ok = wait(bar(L::Q_FULL), 0, 2);
      for (int j = 0; ok && j <= nkv; ++j) {
        if (j < nkv) {
          const int s = j & 1;
          if (!wait(bar(L::K_FULL + s), (j >> 1) & 1, 3)) break;
          if (j >= 2 && !wait(bar(L::S_FREE + s), ((j >> 1) - 1) & 1, 4)) break;
          tc_fence_after();
          const uint32_t d_tmem = tmem + L::S_COL0 + 128u * s;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t koff = (ks >> 2) * L::HALF + (ks & 3) * 32;
            const uint64_t a = sdesc_sw128(base + L::Q_OFF + koff, 16, 1024);
            const uint64_t b = sdesc_sw128(base + L::K_OFF + s * L::TILE + koff, 16, 1024);
            mma_ss(d_tmem, a, b, IDESC_S, ks > 0 ? 1u : 0u);
          }
          tc_commit(bar(L::S_FULL + s));
        }
        if (j >= 1) {
          const int jj = j - 1, s = jj & 1;
          if (!wait(bar(L::P_FULL + s), (jj >> 1) & 1, 5)) break;
          if (!wait(bar(L::V_FULL + s), (jj >> 1) & 1, 6)) break;
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < L::BN / 16; ++ks) {
            const uint32_t a_tmem = tmem + L::P_COL0 + 64u * s + 8u * ks;
            const uint64_t b = sdesc_sw128(base + L::V_OFF + s * L::TILE + ks * 2048, L::HALF, 1024);
            mma_ts(tmem + L::O_COL, a_tmem, b, IDESC_O, (jj > 0 || ks > 0) ? 1u : 0u);
          }
          tc_commit(bar(L::O_READY));
          tc_commit(bar(L::KV_EMPTY + s));
        }
      }
      tc_commit(bar(L::TEARDOWN));
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------- softmax warps 0..3
    const int t = threadIdx.x;  // row within the tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int q_row = qblk * L::BM + t;
    const float scale = p.scale, beta = p.beta;
    float rm = -INFINITY, m_run = -INFINITY, l = 0.f;
    int rs = 0;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int s = j & 1;
      if (!wait(bar(L::S_FULL + s), (j >> 1) & 1, 7)) { ok = false; break; }
      tc_fence_after();
      float x[128];
      {
        uint32_t r0[32], r1[32];
        const uint32_t sa = tmem + lane_base + L::S_COL0 + 128u * s;
        tmem_ld32x2(sa, sa + 32, r0, r1);
#pragma unroll
        for (int c = 0; c < 32; ++c) { x[c] = __uint_as_float(r0[c]); x[32 + c] = __uint_as_float(r1[c]); }
        tmem_ld32x2(sa + 64, sa + 96, r0, r1);
#pragma unroll
        for (int c = 0; c < 32; ++c) { x[64 + c] = __uint_as_float(r0[c]); x[96 + c] = __uint_as_float(r1[c]); }
      }
      tc_fence_before();
      mbar_arrive(bar(L::S_FREE + s));
      // scores in the S domain, masked entries -inf
      const int kv0 = j * L::BN;
      const bool diag = p.causal && (j == qblk);
      const int lim_causal = diag ? t : (L::BN - 1);
      const int lim_len = p.N - 1 - kv0;
      const int lim = lim_causal < lim_len ? lim_causal : lim_len;
      float tmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        const float v = (c <= lim) ? x[c] * scale : -INFINITY;
        x[c] = v;
        tmax = fmaxf(tmax, v);
      }
      int tcnt = 0;
#pragma unroll
      for (int c = 0; c < 128; ++c) tcnt += (x[c] == tmax) ? 1 : 0;
      if (tmax > rm) { rm = tmax; rs = tcnt; }
      else if (tmax == rm) { rs += tcnt; }
      float m_new = rm;
      if (p.mode == 1 && rs > 1) m_new = (rm > 0.f) ? beta * rm : ((rm < 0.f) ? 0.f : beta - 1.f);
      // O and P[s] are free once the previous P V product has completed
      if (j > 0) {
        if (!wait(bar(L::O_READY), (j - 1) & 1, 8)) { ok = false; break; }
        tc_fence_after();
        const bool changed = (m_new != m_run);
        float alpha = 1.f;
        if (changed) {
          alpha = ex2_approx((m_run - m_new) * kLog2e);
          l *= alpha;
        }
        if (__any_sync(0xffffffffu, changed)) {
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t r[32];
            const uint32_t oa = tmem + lane_base + L::O_COL + c0;
            tmem_ld32(oa, r);
#pragma unroll
            for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * alpha);
            tmem_st32(oa, r);
          }
        }
      }
      m_run = m_new;
      // P_bar = exp(S - m), rowsum in fp32, bf16 operand into TMEM
      float rsum = 0.f;
#pragma unroll
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float e0 = ex2_approx((x[c0 + c] - m_new) * kLog2e);
          const float e1 = ex2_approx((x[c0 + c + 1] - m_new) * kLog2e);
          rsum += e0 + e1;
          pk[c >> 1] = pack_bf16x2(e0, e1);
        }
        tmem_st16(tmem + lane_base + L::P_COL0 + 64u * s + (c0 >> 1), pk);
      }
      l += rsum;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::P_FULL + s));
    }
    // ------------------------------------------------------------- epilogue
    if (ok && wait(bar(L::O_READY), (nkv - 1) & 1, 9)) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool row_ok = q_row < p.N;
      __nv_bfloat16* orow = p.o + (static_cast<size_t>(bh) * p.N + q_row) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + L::O_COL + c0, r);
        if (row_ok) {
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(r[c + 0]) * inv_l, __uint_as_float(r[c + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(r[c + 2]) * inv_l, __uint_as_float(r[c + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(r[c + 4]) * inv_l, __uint_as_float(r[c + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(r[c + 6]) * inv_l, __uint_as_float(r[c + 7]) * inv_l);
            *reinterpret_cast<uint4*>(orow + c0 + c) = w;
          }
        }
      }
      if (row_ok) {
        const size_t ri = static_cast<size_t>(bh) * p.N + q_row;
        p.lse[ri] = m_run + logf(l);
        if (p.st_rm) p.st_rm[ri] = rm;
        if (p.st_rs) p.st_rs[ri] = rs;
        if (p.st_m) p.st_m[ri] = m_run;
        if (p.st_pbar_max) p.st_pbar_max[ri] = ex2_approx((rm - m_run) * kLog2e);
      }
    }
  }

  // ----------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    volatile int never = 0;
    const BoundedWait drain{&never, 1u};
    drain(bar(L::TEARDOWN), 0, 30);  // every MMA of this CTA has completed
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace fa
