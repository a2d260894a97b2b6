// Pipelined backward main kernel for head dimension 64.
//
// Same mathematics as fa_bwd_main_kernel (see fa_bwd.cuh): one CTA per
// (batch, head, 128-key block), looping over the query blocks that see the
// keys, in the transposed orientation (lane = key).  What changes is the
// schedule, so that the tensor core and the elementwise work overlap:
//
//   * S^T is double-buffered in TMEM: the MMA warp issues S^T of query block
//     i+2 while the elementwise warps work on block i, and dP^T of block i+1
//     as soon as block i's dS has been consumed.
//   * Eight elementwise warps (two warpgroups) split the 128 query columns of
//     a key row: warpgroup h takes columns [64h, 64h+64).  Both copy their S^T
//     columns to registers and meet at a named barrier; then warpgroup h
//     writes its bf16 P^T into S^T cols [32h, 32h+32), so P^T occupies
//     [0,64) and [64,128) is free for dQ.  dS^T goes into the first half of
//     the dP^T columns each warpgroup has just read (64h + [0,32)), which
//     needs no barrier.
//   * dQ_i = dS K is one N = 64 product into S^T cols [64,128) of the same
//     buffer, which no later product of the iteration touches.
//   * Four drain warps move the dQ partial from TMEM into a 128B-swizzled
//     fp32 tile in shared memory and add it to the fp32 accumulator in global
//     memory with one TMA tensor reduce-add per 32-column half (rows past N
//     are clipped by the tensor map).  They also prepare the per-query
//     vectors (lse or m, 1/l, delta) two blocks ahead.
//
// TMEM columns: S^T[0] [0,128)  S^T[1] [128,256)  dP^T [256,384)
//               dV [384,448)  dK [448,512)
// Warps: 0-3 and 4-7 elementwise (key t = threadIdx % 128), 8-11 drain
// (query t), 12 TMA producer, 13 MMA issuer / TMEM owner, 14-15 idle.  The
// block is launched with 128 registers per thread; the warpgroups then
// re-balance them: elementwise 176, drain 96, TMA/MMA 56
// (2*176 + 96 + 56 = 504 <= 4*128).
#pragma once

#include "fa_bwd.cuh"

namespace fa {

struct BwdPipeLayout {
  static constexpr int D = 64, B = 128, TILE = 128 * 64 * 2, NST = 3;
  static constexpr int K_OFF = 0, V_OFF = TILE, Q_OFF = 2 * TILE;
  static constexpr int DO_OFF = Q_OFF + NST * TILE;
  static constexpr int DS_OFF = DO_OFF + NST * TILE;  // dS^T [keys][queries], two 64-query halves
  static constexpr int DQS_OFF = DS_OFF + 2 * TILE;   // dQ staging: two [128 rows][32 fp32] swizzled boxes
  static constexpr int VEC_OFF = DQS_OFF + 2 * TILE;  // [2 stages][3][128] fp32
  static constexpr int BAR_OFF = VEC_OFF + 2 * 3 * 128 * 4;
  enum {
    KV_FULL = 0,
    Q_FULL = 1,
    Q_EMPTY = Q_FULL + NST,
    S_FULL = Q_EMPTY + NST,  // [2]
    P_FULL = S_FULL + 2,     // [2]
    DP_FULL = P_FULL + 2,
    DS_FULL,
    DQ_FULL,                 // [2]
    DQ_FREE = DQ_FULL + 2,
    VEC_FULL,                // [2]
    VEC_EMPTY = VEC_FULL + 2,  // [2]
    ACC_DONE = VEC_EMPTY + 2,
    TEARDOWN,
    NBAR
  };
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 512, DPT_COL = 256, DV_COL = 384, DK_COL = 448;
  static constexpr int THREADS = 512;
  static constexpr uint32_t REGS_ELEM = 176, REGS_DRAIN = 96, REGS_CTRL = 56;
};

__device__ __forceinline__ void tma_reduce_add_3d(const void* tmap, uint32_t src, int x, int y, int z) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(tmap)),
      "r"(src), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__global__ void __launch_bounds__(512, 1)
fa_bwd_main_pipe_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                        const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_dk,
                        const __grid_constant__ CUtensorMap tm_dv, const BwdParams p) {
  using L = BwdPipeLayout;
  constexpr int TILE = L::TILE, NST = L::NST;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);
  auto bar = [&](int i) { return base + L::BAR_OFF + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  // per-query vectors at VEC_OFF, [stage][0]: -a, [stage][1]: 1/l, [stage][2]: delta (fp32 x 128)
  const BoundedWait wait{abort_flag, 3u};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = p.BH;
  const int kblk = blockIdx.x / BH;
  const int bh = blockIdx.x - kblk * BH;
  const int i0 = p.causal ? kblk : 0;
  const int n_it = p.n_blk - i0;

  if (threadIdx.x == 0) {
    FA_TRACE_POINT(0);
    mbar_init(bar(L::KV_FULL), 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar(L::Q_FULL + s), 1);
      mbar_init(bar(L::Q_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(L::S_FULL + b), 1);
      mbar_init(bar(L::P_FULL + b), 256);
      mbar_init(bar(L::DQ_FULL + b), 1);
      mbar_init(bar(L::VEC_FULL + b), 128);
      mbar_init(bar(L::VEC_EMPTY + b), 256);
    }
    mbar_init(bar(L::DP_FULL), 1);
    mbar_init(bar(L::DS_FULL), 256);
    mbar_init(bar(L::DQ_FREE), 128);
    mbar_init(bar(L::ACC_DONE), 1);
    mbar_init(bar(L::TEARDOWN), 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 13) {
    tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
    tmem_relinquish();
  }
  grid_launch_dependents();
  grid_dependency_wait();  // delta and the cleared dQ accumulator come from the previous grid
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) FA_TRACE_POINT(1);

  // End of every role: all 16 warps meet on named barrier 15, then warp 13
  // waits for its last MMAs and frees TMEM.  Each role's branch ends on its
  // own (no common tail), so each keeps its own register budget.
  auto teardown = [&]() {
    tc_fence_before();
    named_barrier_sync(15, L::THREADS);
    if (threadIdx.x == 0) FA_TRACE_POINT(2);
    if (warp == 13) {
      tc_fence_after();
      volatile int never = 0;
      const BoundedWait drain{&never, 3u};
      drain(bar(L::TEARDOWN), 0, 30);
      tmem_dealloc(tmem, L::TMEM_COLS);
    }
  };

  if (warp >= 12) {
    warpgroup_reg_dealloc<L::REGS_CTRL>();
  if (warp == 12) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_expect_tx(bar(L::KV_FULL), 2 * TILE);
      tma_load_3d(base + L::K_OFF, &tm_k, bar(L::KV_FULL), 0, kblk * L::B, bh);
      tma_load_3d(base + L::V_OFF, &tm_v, bar(L::KV_FULL), 0, kblk * L::B, bh);
      int issued[NST];
      for (int s = 0; s < NST; ++s) issued[s] = -1;
      for (int i = 0; i < n_it; ++i) {
        const int s = i % NST, use = i / NST;
        if (use > 0 && !wait(bar(L::Q_EMPTY + s), (use - 1) & 1, 1)) break;
        const int row0 = (i0 + i) * L::B;
        mbar_expect_tx(bar(L::Q_FULL + s), 2 * TILE);
        tma_load_3d(base + L::Q_OFF + s * TILE, &tm_q, bar(L::Q_FULL + s), 0, row0, bh);
        tma_load_3d(base + L::DO_OFF + s * TILE, &tm_do, bar(L::Q_FULL + s), 0, row0, bh);
        issued[s] = i;
      }
      volatile int never = 0;
      const BoundedWait drain{&never, 3u};
      drain(bar(L::KV_FULL), 0, 20);
      for (int s = 0; s < NST; ++s)
        if (issued[s] >= 0) drain(bar(L::Q_FULL + s), (issued[s] / NST) & 1, 21);
    }
    __syncwarp();
  } else if (warp == 13) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_SQ = idesc_bf16_f32(128, 128, false, false);  // S^T, dP^T
      constexpr uint32_t IDESC_KV = idesc_bf16_f32(128, 64, false, true);    // dV, dK
      constexpr uint32_t IDESC_DQ = idesc_bf16_f32(128, 64, true, true);     // dQ
      auto q_tile = [&](int i) { return base + L::Q_OFF + (i % NST) * TILE; };
      auto do_tile = [&](int i) { return base + L::DO_OFF + (i % NST) * TILE; };
      auto issue_s = [&](int i) {
        const uint32_t d_tmem = tmem + 128u * (i & 1);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_ss(d_tmem, sdesc_sw128(base + L::K_OFF + ks * 32, 16, 1024), sdesc_sw128(q_tile(i) + ks * 32, 16, 1024),
                 IDESC_SQ, ks > 0 ? 1u : 0u);
        tc_commit(bar(L::S_FULL + (i & 1)));
      };
      auto issue_dp = [&](int i) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_ss(tmem + L::DPT_COL, sdesc_sw128(base + L::V_OFF + ks * 32, 16, 1024),
                 sdesc_sw128(do_tile(i) + ks * 32, 16, 1024), IDESC_SQ, ks > 0 ? 1u : 0u);
        tc_commit(bar(L::DP_FULL));
      };
      bool ok = wait(bar(L::KV_FULL), 0, 2);
      if (ok && n_it > 0) {
        ok = wait(bar(L::Q_FULL + 0), 0, 3);
        if (ok) {
          tc_fence_after();
          issue_s(0);
          issue_dp(0);
        }
      }
      if (ok && n_it > 1) {
        ok = wait(bar(L::Q_FULL + 1), 0, 3);
        if (ok) {
          tc_fence_after();
          issue_s(1);
        }
      }
      for (int i = 0; ok && i < n_it; ++i) {
        const int b = i & 1;
        if (!wait(bar(L::P_FULL + b), (i >> 1) & 1, 4)) break;
        FA_TRACE_POINT(10);
        tc_fence_after();
        // dV += P^T dO_i   (K-dim = queries; P^T at S^T cols [0,64))
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t a = tmem + 128u * b + 8u * ks;
          mma_ts(tmem + L::DV_COL, a, sdesc_sw128(do_tile(i) + ks * 2048, 16384, 1024), IDESC_KV,
                 (i > 0 || ks > 0) ? 1u : 0u);
        }
        if (!wait(bar(L::DS_FULL), i & 1, 5)) break;
        FA_TRACE_POINT(11);
        tc_fence_after();
        // dK += dS^T Q_i
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t a = tmem + L::DPT_COL + (ks < 4 ? 8u * ks : 64u + 8u * (ks - 4));
          mma_ts(tmem + L::DK_COL, a, sdesc_sw128(q_tile(i) + ks * 2048, 16384, 1024), IDESC_KV,
                 (i > 0 || ks > 0) ? 1u : 0u);
        }
        // dQ_i = dS K into S^T cols [64,128) of the same buffer
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss(tmem + 128u * b + 64u, sdesc_sw128(base + L::DS_OFF + ks * 2048, 16384, 1024),
                 sdesc_sw128(base + L::K_OFF + ks * 2048, 16384, 1024), IDESC_DQ, ks > 0 ? 1u : 0u);
        tc_commit(bar(L::DQ_FULL + b));
        tc_commit(bar(L::Q_EMPTY + (i % NST)));
        if (i + 1 < n_it) issue_dp(i + 1);
        FA_TRACE_POINT(12);
        if (i + 2 < n_it) {
          if (!wait(bar(L::DQ_FREE), i & 1, 6)) break;
          FA_TRACE_POINT(13);
          if (!wait(bar(L::Q_FULL + ((i + 2) % NST)), ((i + 2) / NST) & 1, 7)) break;
          tc_fence_after();
          issue_s(i + 2);
        }
      }
      tc_commit(bar(L::ACC_DONE));
      tc_commit(bar(L::TEARDOWN));
    }
    __syncwarp();
  }  // warps 14-15: idle
    teardown();
    return;
  }
  if (warp >= 8) {
    warpgroup_reg_dealloc<L::REGS_DRAIN>();
    // --------------------------------------------------------- drain warps
    const int t = threadIdx.x - 256;  // query within the block == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float scale = p.scale;
    const size_t vrow0 = static_cast<size_t>(bh) * p.N;
    // per-query vectors of block i: global loads first (prefetch), smem later
    struct Vec3 { float lse, m, dl; };
    auto load_vec = [&](int i) {
      Vec3 v{0.f, 0.f, 0.f};
      const int q = (i0 + i) * L::B + t;
      if (i < n_it && q < p.N) {
        v.lse = __ldg(p.lse + vrow0 + q);
        v.dl = __ldg(p.delta + vrow0 + q);
        v.m = (p.mode == 1) ? __ldg(p.row_m + vrow0 + q) : 0.f;
      }
      return v;
    };
    auto publish_vec = [&](int i, const Vec3& v) {
      const int s = i & 1, q = (i0 + i) * L::B + t;
      float na = -INFINITY, bb = 0.f, dl = 0.f;
      if (q < p.N) {
        dl = v.dl;
        if (p.mode == 1) {
          na = -v.m * kLog2e;
          bb = 1.f / ex2_approx((v.lse - v.m) * kLog2e);
        } else {
          na = -v.lse * kLog2e;
          bb = 1.f;
        }
      }
      sts32(base + L::VEC_OFF + ((s * 3 + 0) * 128 + t) * 4, na);
      sts32(base + L::VEC_OFF + ((s * 3 + 1) * 128 + t) * 4, bb);
      sts32(base + L::VEC_OFF + ((s * 3 + 2) * 128 + t) * 4, dl);
      mbar_arrive(bar(L::VEC_FULL + s));
    };
    if (n_it > 0) publish_vec(0, load_vec(0));
    if (n_it > 1) publish_vec(1, load_vec(1));
    Vec3 next = load_vec(2);
    if (t == 0) tma_prefetch_desc(&tm_dq);
    for (int i = 0; i < n_it; ++i) {
      const int b = i & 1;
      if (!wait(bar(L::DQ_FULL + b), (i >> 1) & 1, 13)) break;
      if (t == 0) FA_TRACE_POINT(30);
      tc_fence_after();
      uint32_t r0[32], r1[32];
      tmem_ld32x2(tmem + lane_base + 128u * b + 64u, tmem + lane_base + 128u * b + 96u, r0, r1);
      tc_fence_before();
      mbar_arrive(bar(L::DQ_FREE));
      if (t == 0) bulk_wait_read_all();  // the previous reduce has finished reading the staging tile
      named_barrier_sync(2, 128);
      // row t of each 32-column box, 16-byte chunk c stored at chunk c ^ (t & 7)
      const uint32_t row0 = base + L::DQS_OFF + t * 128;
      const uint32_t row1 = row0 + TILE;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t pc = (c ^ (t & 7)) << 4;
        sts128(row0 + pc, __float_as_uint(__uint_as_float(r0[4 * c]) * scale),
               __float_as_uint(__uint_as_float(r0[4 * c + 1]) * scale),
               __float_as_uint(__uint_as_float(r0[4 * c + 2]) * scale),
               __float_as_uint(__uint_as_float(r0[4 * c + 3]) * scale));
        sts128(row1 + pc, __float_as_uint(__uint_as_float(r1[4 * c]) * scale),
               __float_as_uint(__uint_as_float(r1[4 * c + 1]) * scale),
               __float_as_uint(__uint_as_float(r1[4 * c + 2]) * scale),
               __float_as_uint(__uint_as_float(r1[4 * c + 3]) * scale));
      }
      fence_proxy_async_smem();
      named_barrier_sync(2, 128);
      if (t == 0) {
        const int q0 = (i0 + i) * L::B;
        tma_reduce_add_3d(&tm_dq, base + L::DQS_OFF, 0, q0, bh);
        tma_reduce_add_3d(&tm_dq, base + L::DQS_OFF + TILE, 32, q0, bh);
        bulk_commit();
        FA_TRACE_POINT(31);
      }
      if (i + 2 < n_it) {
        if (!wait(bar(L::VEC_EMPTY + b), (i >> 1) & 1, 14)) break;
        publish_vec(i + 2, next);
        next = load_vec(i + 3);
      }
    }
    if (t == 0) bulk_wait_all();
    teardown();
    return;
  }
  {
    warpgroup_reg_alloc<L::REGS_ELEM>();
    // ----------------------------------------------- elementwise warps 0..7
    const int h = warp >> 2;          // query half
    const int t = threadIdx.x & 127;  // key within the block == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int key = kblk * L::B + t;
    const float scale = p.scale;
    const float c_log2 = scale * kLog2e;
    const uint64_t C2 = f2_pack(c_log2, c_log2);
    const bool mode1 = p.mode == 1;
    bool ok = true;
    for (int i = 0; i < n_it; ++i) {
      const int b = i & 1;
      if (!wait(bar(L::VEC_FULL + b), (i >> 1) & 1, 8)) { ok = false; break; }
      if (!wait(bar(L::S_FULL + b), (i >> 1) & 1, 9)) { ok = false; break; }
      if (threadIdx.x == 0) FA_TRACE_POINT(20);
      tc_fence_after();
      const uint32_t va = base + L::VEC_OFF + ((b * 3 + 0) * 128 + 64 * h) * 4;
      const uint32_t vb = base + L::VEC_OFF + ((b * 3 + 1) * 128 + 64 * h) * 4;
      const uint32_t vd = base + L::VEC_OFF + ((b * 3 + 2) * 128 + 64 * h) * 4;
      const bool diag = p.causal && (i0 + i == kblk);
      const int qoff = 64 * h;
      uint64_t p2[32];  // this row's 64 P values (fp32 pairs)
      {
        uint32_t r0[32], r1[32];
        tmem_ld32x2(tmem + lane_base + 128u * b + 64u * h, tmem + lane_base + 128u * b + 64u * h + 32u, r0, r1);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          p2[e] = f2_pack(__uint_as_float(r0[2 * e]), __uint_as_float(r0[2 * e + 1]));
          p2[16 + e] = f2_pack(__uint_as_float(r1[2 * e]), __uint_as_float(r1[2 * e + 1]));
        }
      }
      if (threadIdx.x == 0) FA_TRACE_POINT(25);
      // both warpgroups hold their S^T columns: P^T may now overwrite [0,64)
      named_barrier_sync(1, 256);
      if (threadIdx.x == 0) FA_TRACE_POINT(26);
      uint32_t pk[32];
#pragma unroll
      for (int pi = 0; pi < 32; pi += 2) {
        const int ql = 2 * pi;
        const float4 na = lds128(va + ql * 4);
        const uint64_t y0 = f2_fma(p2[pi], C2, f2_pack(na.x, na.y));
        const uint64_t y1 = f2_fma(p2[pi + 1], C2, f2_pack(na.z, na.w));
        float a0, a1, a2, a3;
        f2_unpack(y0, a0, a1);
        f2_unpack(y1, a2, a3);
        float p0 = ex2_approx(a0), p1 = ex2_approx(a1), p2v = ex2_approx(a2), p3 = ex2_approx(a3);
        if (mode1) {
          const float4 bb = lds128(vb + ql * 4);
          p0 *= bb.x;
          p1 *= bb.y;
          p2v *= bb.z;
          p3 *= bb.w;
        }
        if (diag) {
          const int qg = qoff + ql;
          if (t > qg) p0 = 0.f;
          if (t > qg + 1) p1 = 0.f;
          if (t > qg + 2) p2v = 0.f;
          if (t > qg + 3) p3 = 0.f;
        }
        p2[pi] = f2_pack(p0, p1);
        p2[pi + 1] = f2_pack(p2v, p3);
        pk[pi] = pack_bf16x2(p0, p1);
        pk[pi + 1] = pack_bf16x2(p2v, p3);
      }
      tmem_st32(tmem + lane_base + 128u * b + 32u * h, pk);
      if (threadIdx.x == 0) FA_TRACE_POINT(27);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::P_FULL + b));
      if (threadIdx.x == 0) FA_TRACE_POINT(21);
      if (!wait(bar(L::DP_FULL), i & 1, 10)) { ok = false; break; }
      if (threadIdx.x == 0) FA_TRACE_POINT(22);
      // the dQ product of the previous block has finished reading the dS tile
      if (i > 0 && !wait(bar(L::DQ_FULL + ((i - 1) & 1)), ((i - 1) >> 1) & 1, 11)) { ok = false; break; }
      tc_fence_after();
      const uint32_t ds_row = base + L::DS_OFF + h * TILE + t * 128;
      uint32_t dpr[64];
      {
        uint32_t (&d0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&dpr[0]);
        uint32_t (&d1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&dpr[32]);
        tmem_ld32x2(tmem + lane_base + L::DPT_COL + 64u * h, tmem + lane_base + L::DPT_COL + 64u * h + 32u, d0, d1);
      }
      uint32_t dk_[32];
#pragma unroll
      for (int pi = 0; pi < 32; pi += 2) {
        const int ql = 2 * pi;
        const float4 dl = lds128(vd + ql * 4);
        const uint64_t ds0 = f2_mul(p2[pi], f2_sub(f2_pack(__uint_as_float(dpr[2 * pi]), __uint_as_float(dpr[2 * pi + 1])),
                                                   f2_pack(dl.x, dl.y)));
        const uint64_t ds1 = f2_mul(p2[pi + 1], f2_sub(f2_pack(__uint_as_float(dpr[2 * pi + 2]), __uint_as_float(dpr[2 * pi + 3])),
                                                       f2_pack(dl.z, dl.w)));
        float d0, d1, d2, d3;
        f2_unpack(ds0, d0, d1);
        f2_unpack(ds1, d2, d3);
        dk_[pi] = pack_bf16x2(d0, d1);
        dk_[pi + 1] = pack_bf16x2(d2, d3);
      }
      // dS^T into the dP^T columns this warpgroup has read: 64h + [0,32)
      tmem_st32(tmem + lane_base + L::DPT_COL + 64u * h, dk_);
      // dS^T row t, queries 64h + [0,64) = the eight 16-byte chunks of the half tile's row
#pragma unroll
      for (int chunk = 0; chunk < 8; ++chunk)
        sts128(ds_row + ((chunk ^ (t & 7)) << 4), dk_[4 * chunk], dk_[4 * chunk + 1], dk_[4 * chunk + 2],
               dk_[4 * chunk + 3]);
      fence_proxy_async_smem();
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::DS_FULL));
      mbar_arrive(bar(L::VEC_EMPTY + b));
      if (threadIdx.x == 0) FA_TRACE_POINT(24);
    }
    // ------------------------------------------------------------- epilogue
    // warpgroup 0 writes dV, warpgroup 1 writes dK * scale: TMEM -> bf16 rows
    // in a 128B-swizzled tile (the dS tile, free once every product is done)
    // -> one TMA tensor store per warpgroup (rows past N are clipped).
    if (ok && wait(bar(L::ACC_DONE), 0, 12)) {
      tc_fence_after();
      const float f = (h == 0) ? 1.f : scale;
      const uint32_t col = (h == 0) ? L::DV_COL : L::DK_COL;
      uint32_t r0[32], r1[32];
      tmem_ld32x2(tmem + lane_base + col, tmem + lane_base + col + 32, r0, r1);
      uint32_t w[32];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        w[c] = pack_bf16x2(__uint_as_float(r0[2 * c]) * f, __uint_as_float(r0[2 * c + 1]) * f);
        w[16 + c] = pack_bf16x2(__uint_as_float(r1[2 * c]) * f, __uint_as_float(r1[2 * c + 1]) * f);
      }
      sts_row_sw128(base + L::DS_OFF + h * TILE, t, w);
      fence_proxy_async_smem();
      named_barrier_sync(3 + h, 128);
      if (t == 0) {
        tma_store_3d(h == 0 ? static_cast<const void*>(&tm_dv) : static_cast<const void*>(&tm_dk),
                     base + L::DS_OFF + h * TILE, 0, kblk * L::B, bh);
        bulk_commit();
        bulk_wait_all();
      }
    }
    (void)key;
    teardown();
  }
}

}  // namespace fa
