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
// TMEM columns: S [0,128)  P_bar [128,192) (bf16 pairs)  O [192, 192+D).
// With d = 64 that is 256 columns and two CTAs share an SM, so eight softmax
// warps hide each other's latency.  S is single-buffered: the softmax warps
// copy it to registers first and release it, so the next tile's Q K^T runs on
// the tensor core while they work; P_bar is fed to the P V product as the A
// operand straight from TMEM.
//
// For d = 64 the scale 1/8 is a power of two, so comparisons (max, ties) are
// taken on the raw fp32 accumulator: x == y <=> x/8 == y/8 and rm = max/8
// exactly.  For d = 128 the scores are scaled first (fp32 multiply), because
// two raw values one ulp apart can round to the same scaled value.
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
  enum { Q_FULL = 0, K_FULL = 1, V_FULL = 3, KV_EMPTY = 5, S_FULL = 7, S_FREE, P_FULL, O_READY, TEARDOWN, NBAR };
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;  // tmem base (4B), abort flag (4B)
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  static constexpr uint32_t S_COL = 0, P_COL = 128, O_COL = 192;
  static constexpr uint32_t TMEM_COLS = (O_COL + D <= 256) ? 256 : 512;
  static constexpr int CTAS_PER_SM = (TMEM_COLS == 256) ? 2 : 1;
};

template <int D>
__global__ void __launch_bounds__(192, FwdLayout<D>::CTAS_PER_SM)
fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
              const FwdParams p) {
  using L = FwdLayout<D>;
  constexpr bool kRawCompare = (D == 64);  // scale is exactly 1/8
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
    FA_TRACE_POINT(0);
    mbar_init(bar(L::Q_FULL), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::K_FULL + s), 1);
      mbar_init(bar(L::V_FULL + s), 1);
      mbar_init(bar(L::KV_EMPTY + s), 1);
    }
    mbar_init(bar(L::S_FULL), 1);
    mbar_init(bar(L::S_FREE), 128);
    mbar_init(bar(L::P_FULL), 128);
    mbar_init(bar(L::O_READY), 1);
    mbar_init(bar(L::TEARDOWN), 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
    tmem_relinquish();
  }
  grid_launch_dependents();
  // inputs (and the outputs' previous contents) belong to the previous grid in
  // the stream until it has completed: everything above overlaps its tail
  grid_dependency_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) FA_TRACE_POINT(1);

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
      auto issue_s = [&](int j) {
        const int s = j & 1;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t koff = (ks >> 2) * L::HALF + (ks & 3) * 32;
          mma_ss(tmem + L::S_COL, sdesc_sw128(base + L::Q_OFF + koff, 16, 1024),
                 sdesc_sw128(base + L::K_OFF + s * L::TILE + koff, 16, 1024), IDESC_S, ks > 0 ? 1u : 0u);
        }
        tc_commit(bar(L::S_FULL));
      };
      bool ok = wait(bar(L::Q_FULL), 0, 2) && wait(bar(L::K_FULL), 0, 3);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      for (int j = 0; ok && j < nkv; ++j) {
        const int s = j & 1;
        // S of the next tile as soon as the softmax warps have copied S_j out
        if (j + 1 < nkv) {
          if (!wait(bar(L::S_FREE), j & 1, 4)) break;
          if (!wait(bar(L::K_FULL + ((j + 1) & 1)), ((j + 1) >> 1) & 1, 3)) break;
          tc_fence_after();
          issue_s(j + 1);
          FA_TRACE_POINT(10);
        }
        if (!wait(bar(L::P_FULL), j & 1, 5)) break;
        if (!wait(bar(L::V_FULL + s), (j >> 1) & 1, 6)) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < L::BN / 16; ++ks) {
          const uint64_t b = sdesc_sw128(base + L::V_OFF + s * L::TILE + ks * 2048, L::HALF, 1024);
          mma_ts(tmem + L::O_COL, tmem + L::P_COL + 8u * ks, b, IDESC_O, (j > 0 || ks > 0) ? 1u : 0u);
        }
        tc_commit(bar(L::O_READY));
        tc_commit(bar(L::KV_EMPTY + s));
        FA_TRACE_POINT(11);
      }
      tc_commit(bar(L::TEARDOWN));
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------- softmax warps 0..3
    const int t = threadIdx.x;  // row within the tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int q_row = qblk * L::BM + t;
    // compare domain: raw accumulator (d = 64) or scaled scores (d = 128)
    const float cmp_scale = kRawCompare ? 1.f : p.scale;        // x = acc * cmp_scale
    const float to_s = kRawCompare ? p.scale : 1.f;             // S = x * to_s (exact)
    const float exp_c = (kRawCompare ? p.scale : 1.f) * kLog2e; // exp2 argument per unit of x
    const uint64_t EXPC2 = f2_pack(exp_c, exp_c);
    const float beta = p.beta;
    float rm_x = -INFINITY;  // running row max, x domain
    float m_run = -INFINITY; // shift in force, S domain
    float l = 0.f;
    int rs = 0;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      if (!wait(bar(L::S_FULL), j & 1, 7)) { ok = false; break; }
      if (t == 0) FA_TRACE_POINT(20);
      tc_fence_after();
      float x[128];
      {
        uint32_t r0[32], r1[32];
        const uint32_t sa = tmem + lane_base + L::S_COL;
        tmem_ld32x2(sa, sa + 32, r0, r1);
#pragma unroll
        for (int c = 0; c < 32; ++c) { x[c] = __uint_as_float(r0[c]); x[32 + c] = __uint_as_float(r1[c]); }
        tmem_ld32x2(sa + 64, sa + 96, r0, r1);
#pragma unroll
        for (int c = 0; c < 32; ++c) { x[64 + c] = __uint_as_float(r0[c]); x[96 + c] = __uint_as_float(r1[c]); }
      }
      tc_fence_before();
      mbar_arrive(bar(L::S_FREE));
      if (t == 0) FA_TRACE_POINT(21);
      // mask (diagonal tile / ragged tail) and tile max, eight partial maxima
      const int kv0 = j * L::BN;
      const bool diag = p.causal && (j == qblk);
      const int lim_causal = diag ? t : (L::BN - 1);
      const int lim_len = p.N - 1 - kv0;
      const int lim = lim_causal < lim_len ? lim_causal : lim_len;
      const bool masked = (lim < L::BN - 1);
      // tile max: three-input max, eight partial maxima
      float pm[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) pm[u] = -INFINITY;
      if (masked) {
#pragma unroll
        for (int c = 0; c < 128; ++c) x[c] = (c <= lim) ? x[c] * cmp_scale : -INFINITY;
      } else if (!kRawCompare) {
#pragma unroll
        for (int c = 0; c < 128; ++c) x[c] *= cmp_scale;
      }
#pragma unroll
      for (int c = 0; c < 128; c += 16) {
#pragma unroll
        for (int u = 0; u < 8; ++u) pm[u] = fmax3(pm[u], x[c + 2 * u], x[c + 2 * u + 1]);
      }
      const float tmax = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
      // tie count: only rows whose tile max reaches the running max need it;
      // set.eq gives 1.0/0.0, summed exactly in fp32 pairs (counts <= 128)
      if (__any_sync(0xffffffffu, tmax >= rm_x)) {
        uint64_t cnt2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int c = 0; c < 128; c += 2)
          cnt2[(c >> 1) & 3] = f2_add(cnt2[(c >> 1) & 3], f2_pack(feq(x[c], tmax), feq(x[c + 1], tmax)));
        float c0, c1, c2, c3, c4, c5, c6, c7;
        f2_unpack(cnt2[0], c0, c1);
        f2_unpack(cnt2[1], c2, c3);
        f2_unpack(cnt2[2], c4, c5);
        f2_unpack(cnt2[3], c6, c7);
        const int tc = static_cast<int>(((c0 + c1) + (c2 + c3)) + ((c4 + c5) + (c6 + c7)));
        if (tmax > rm_x) {
          rm_x = tmax;
          rs = tc;
        } else if (tmax == rm_x) {
          rs += tc;
        }
      }
      const float rm_s = rm_x * to_s;
      float m_new = rm_s;
      if (p.mode == 1 && rs > 1) m_new = (rm_s > 0.f) ? beta * rm_s : ((rm_s < 0.f) ? 0.f : beta - 1.f);
      // P and O are free once the previous P V product has completed
      if (t == 0) FA_TRACE_POINT(22);
      if (j > 0) {
        if (!wait(bar(L::O_READY), (j - 1) & 1, 8)) { ok = false; break; }
        if (t == 0) FA_TRACE_POINT(23);
        tc_fence_after();
        const bool changed = (m_new != m_run);
        float alpha = 1.f;
        if (changed) {
          alpha = ex2_approx((m_run - m_new) * kLog2e);
          l *= alpha;
        }
        if (__any_sync(0xffffffffu, changed)) {
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 16) {
            uint32_t r[16];
            const uint32_t oa = tmem + lane_base + L::O_COL + c0;
            tmem_ld16(oa, r);
            uint32_t w[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) w[c] = __float_as_uint(__uint_as_float(r[c]) * alpha);
            tmem_st16(oa, w);
          }
        }
      }
      m_run = m_new;
      // P_bar = exp2(x * exp_c - m * log2e); row sum in fp32 (four pair accumulators)
      const float nm = -m_new * kLog2e;
      const uint64_t NM2 = f2_pack(nm, nm);
      uint64_t sum2[2] = {0ull, 0ull};
#pragma unroll
      for (int c0 = 0; c0 < 128; c0 += 16) {
        uint32_t pk[8];
#pragma unroll
        for (int c = 0; c < 16; c += 2) {
          const uint64_t y = f2_fma(f2_pack(x[c0 + c], x[c0 + c + 1]), EXPC2, NM2);
          float y0, y1;
          f2_unpack(y, y0, y1);
          const float e0 = ex2_approx(y0), e1 = ex2_approx(y1);
          sum2[(c >> 1) & 1] = f2_add(sum2[(c >> 1) & 1], f2_pack(e0, e1));
          pk[c >> 1] = pack_bf16x2(e0, e1);
        }
        tmem_st8(tmem + lane_base + L::P_COL + (c0 >> 1), pk);
      }
      {
        const uint64_t s01 = f2_add(sum2[0], sum2[1]);
        float a, b;
        f2_unpack(s01, a, b);
        l += a + b;
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::P_FULL));
      if (t == 0) FA_TRACE_POINT(24);
    }
    // ------------------------------------------------------------- epilogue
    if (ok && nkv > 0 && wait(bar(L::O_READY), (nkv - 1) & 1, 9)) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool row_ok = q_row < p.N;
      // O rows -> bf16 in 128B-swizzled 64-column boxes (the K stages, free
      // once the last P V product has completed) -> TMA tensor store
#pragma unroll
      for (int h = 0; h < D / 64; ++h) {
        uint32_t r0[32], r1[32];
        tmem_ld32x2(tmem + lane_base + L::O_COL + 64 * h, tmem + lane_base + L::O_COL + 64 * h + 32, r0, r1);
        uint32_t w[32];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          w[c] = pack_bf16x2(__uint_as_float(r0[2 * c]) * inv_l, __uint_as_float(r0[2 * c + 1]) * inv_l);
          w[16 + c] = pack_bf16x2(__uint_as_float(r1[2 * c]) * inv_l, __uint_as_float(r1[2 * c + 1]) * inv_l);
        }
        sts_row_sw128(base + L::K_OFF + h * L::HALF, t, w);
      }
      fence_proxy_async_smem();
      named_barrier_sync(1, 128);
      if (t == 0) {
        for (int h = 0; h < D / 64; ++h) tma_store_3d(&tm_o, base + L::K_OFF + h * L::HALF, 64 * h, qblk * L::BM, bh);
        bulk_commit();
        bulk_wait_all();
      }
      if (row_ok) {
        const size_t ri = static_cast<size_t>(bh) * p.N + q_row;
        const float rm_s = rm_x * to_s;
        p.lse[ri] = m_run + logf(l);
        if (p.st_rm) p.st_rm[ri] = rm_s;
        if (p.st_rs) p.st_rs[ri] = rs;
        if (p.st_m) p.st_m[ri] = m_run;
        if (p.st_pbar_max) p.st_pbar_max[ri] = ex2_approx((rm_s - m_run) * kLog2e);
      }
    }
  }

  // ----------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) FA_TRACE_POINT(2);
  if (warp == 5) {
    tc_fence_after();
    volatile int never = 0;
    const BoundedWait drain{&never, 1u};
    drain(bar(L::TEARDOWN), 0, 30);  // every MMA of this CTA has completed
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace fa
