// Forward kernel for head dimension 64: tiled attention with the stabilised
// safe softmax, two CTAs per SM with the 128 score columns of a row split
// between two warpgroups.  (Head dimension 128 runs the pair kernel of
// fa_fwd.cuh, which holds the method's formulas and the shared parameter
// block.)
//
// Persistent kernel.  A work item is one 128-row Q tile of one (batch, head);
// items are ordered longest first (causal: the last Q tiles, which see the
// most key tiles) and dealt to the CTAs in snake order (round r gives CTA c
// item r*G + c for even r, r*G + G-1-c for odd r), which balances the causal
// triangle.  Per CTA:
//   warps 0-3, 4-7  softmax: warpgroup h owns columns [64h, 64h+64) of every
//                   row; thread t of each warpgroup owns row t (TMEM lane t);
//   warp  8         TMA producer: Q per item (two buffers), K and V through
//                   2-stage rings with separate "empty" barriers (a K stage is
//                   free once its Q K^T is done, a V stage once its P V is),
//                   and the TMA store of each finished O tile;
//   warp  9         MMA issuer (one thread) and TMEM owner;
//   warps 10-11     idle (they complete the control warpgroup, whose register
//                   budget is handed to the softmax warpgroups with setmaxnreg).
// The two warpgroups keep identical copies of a row's running statistics:
// per tile each half finds its maximum and its tie count at that maximum, the
// pair is exchanged through shared memory, and both combine them the same
// way (row max = the larger half maximum, tie count = the counts of the halves
// that reach it).  Each half rescales and stores its half of O and writes its
// half of P_bar; the row sum is kept per half and added at the end.
// TMEM columns: S [0,128)  P_bar [128,192) (bf16 pairs)  O [192, 192+D).
// With d = 64 that is 256 columns and two CTAs share an SM: sixteen softmax
// warps per SM, which hide the latency of the per-tile dependent chain
// better than the pair kernel's eight (measured on g2s: 43 us here against
// 47-52 us for the pair kernel at d = 64).  S is single-buffered: the softmax
// warps copy it to registers first and release it, so the next tile's Q K^T
// (also across items) runs on the tensor core while they work; P_bar is fed
// to the P V product as the A operand straight from TMEM.  A finished O tile
// is normalised, converted to bf16 and staged (128B-swizzled) in the item's
// own Q buffer, whose last reader -- the item's final Q K^T -- has completed
// by then; the producer stores it before it loads a later item's Q into that
// buffer.  The scale 1/8 is a power of two, so comparisons (max, ties) are
// taken on the raw fp32 accumulator: x == y <=> x/8 == y/8 and rm = max/8
// exactly.
#pragma once

#include "fa_fwd.cuh"

namespace fa {
template <int D, bool HP = false>
struct FwdSplitLayout {
  static constexpr int BM = 128, BN = 128;
  static constexpr int TILE = BM * D * 2;  // bytes of a 128 x D bf16 tile
  static constexpr int HALF = 128 * 128;   // bytes of one 128-row x 64-col TMA box
  static constexpr int Q_OFF = 0;                      // two Q buffers (also the O staging tiles)
  static constexpr int K_OFF = Q_OFF + 2 * TILE;       // two K stages
  static constexpr int V_OFF = K_OFF + 2 * TILE;       // two V stages
  static constexpr int XCHG_OFF = V_OFF + 2 * TILE;    // [3 slots][2 halves][128 rows] x 8 bytes
  static constexpr int BAR_OFF = XCHG_OFF + 3 * 2 * 128 * 8;
  // barrier indices
  enum {
    Q_FULL = 0, O_STAGED = 2, K_FULL = 4, K_EMPTY = 6, V_FULL = 8, V_EMPTY = 10,
    S_FULL = 12, S_FREE, P_FULL, O_READY, TEARDOWN, NBAR
  };
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;  // tmem base (4B), abort flag (4B)
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  // HP (high-precision O requested): P_bar also as a second bf16 part
  // P_lo = bf16(P_bar - P_hi) at PLO_COL, multiplied into its own
  // accumulator O_lo, so that (O + O_lo) / l carries P_bar to ~16 bits
  static constexpr uint32_t S_COL = 0, P_COL = 128, PLO_COL = 192;
  static constexpr uint32_t O_COL = HP ? 256 : 192, OLO_COL = 256 + D;
  static constexpr uint32_t TMEM_COLS = (!HP && O_COL + D <= 256) ? 256 : 512;
  static constexpr int CTAS_PER_SM = (TMEM_COLS == 256) ? 2 : 1;
  static constexpr int THREADS = 384;
  // register budgets after setmaxnreg (two CTAs per SM: 80 per thread at
  // launch, 2 x 128 x 104 + 128 x 32 = 384 x 80)
  static constexpr bool SPLIT_REGS = (CTAS_PER_SM == 2);
  static constexpr uint32_t REGS_SOFT = 104, REGS_CTRL = 32;
};

// setmaxnreg draws on the registers the block was launched with (two CTAs
// per SM: 384 threads x 80): a split above that total would wait forever
static_assert(2 * FwdSplitLayout<64, false>::REGS_SOFT + FwdSplitLayout<64, false>::REGS_CTRL == 3 * 80,
              "register split");
static_assert(2 * FwdSplitLayout<64, false>::SMEM_BYTES <= 228 * 1024, "two CTAs per SM");

// The work items of one CTA, in order (see the file comment).  Only the
// item's coordinates are held; the rest is read from the launch (kernel
// parameters and the grid shape) when needed.
struct FwdSplitCursor {
  int r, qblk, bh, nkv;
  bool valid;
  __device__ __forceinline__ static int item(int r) {
    const int G = gridDim.x, c = blockIdx.x;
    return r * G + ((r & 1) ? (G - 1 - c) : c);
  }
  __device__ __forceinline__ void load(const FwdParams& p) {
    const int w = item(r);
    valid = w < p.n_qblk * p.BH;
    if (valid) {
      const int tile_rev = w / p.BH;
      bh = w - tile_rev * p.BH;
      qblk = p.causal ? (p.n_qblk - 1 - tile_rev) : tile_rev;
      nkv = p.causal ? (qblk + 1) : p.n_qblk;
    }
  }
  __device__ __forceinline__ void start(const FwdParams& p) {
    r = 0;
    load(p);
  }
  __device__ __forceinline__ void next(const FwdParams& p) {
    ++r;
    load(p);
  }
  // whether this CTA has a work item after the current one
  __device__ __forceinline__ bool has_next(const FwdParams& p) const { return item(r + 1) < p.n_qblk * p.BH; }
};

template <int D, bool HP>
__global__ void __launch_bounds__(384, FwdSplitLayout<D, HP>::CTAS_PER_SM)
fa_fwd_split_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
              const FwdParams p) {
  using L = FwdSplitLayout<D, HP>;
  constexpr bool kRawCompare = (D == 64);  // scale is exactly 1/8
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;  // 1024-byte aligned for the 128B swizzle
  uint8_t* smem = smem_raw + (base - raw_addr);
  auto bar = [&](int i) { return base + L::BAR_OFF + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  const uint64_t limit_ns = wait_limit_ns();
  const BoundedWait wait{abort_flag, 1u, limit_ns};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    FA_TRACE_POINT(0);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::Q_FULL + s), 1);
      mbar_init(bar(L::O_STAGED + s), 256);
      mbar_init(bar(L::K_FULL + s), 1);
      mbar_init(bar(L::K_EMPTY + s), 1);
      mbar_init(bar(L::V_FULL + s), 1);
      mbar_init(bar(L::V_EMPTY + s), 1);
    }
    mbar_init(bar(L::S_FULL), 1);
    mbar_init(bar(L::S_FREE), 256);
    mbar_init(bar(L::P_FULL), 256);
    mbar_init(bar(L::O_READY), 1);
    mbar_init(bar(L::TEARDOWN), 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 9) {
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

  // End of every role: all warps meet on named barrier 2, then warp 9 waits
  // for the last MMAs and frees TMEM.  Each role's branch ends on its own (no
  // common tail), so each keeps its own register budget.
  auto teardown = [&]() {
    tc_fence_before();
    named_barrier_sync(2, L::THREADS);
    if (threadIdx.x == 0) FA_TRACE_POINT(2);
    if (warp == 9) {
      tc_fence_after();
      volatile int never = 0;
      const BoundedWait drain{&never, 1u, limit_ns};
      drain(bar(L::TEARDOWN), 0, 30);  // every MMA of this CTA has completed
      tmem_dealloc(tmem, L::TMEM_COLS);
    }
  };

  if (warp >= 8) {
    if constexpr (L::SPLIT_REGS) warpgroup_reg_dealloc<L::REGS_CTRL>();
  }
  if (warp >= 10) {
    teardown();
    return;
  }
  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_o);
      FwdSplitCursor cur;
      cur.start(p);
      // counts of the tiles issued so far, for the drain at exit
      int q_issued = 0, k_issued = 0, v_issued = 0;
      // item m's O is staged in Q buffer m & 1 (its m>>1-th use)
      auto store_staged = [&](int m) -> bool {
        const int qs = m & 1;
        if (!wait(bar(L::O_STAGED + qs), (m >> 1) & 1, 1)) return false;
        FwdSplitCursor it;
        it.r = m;
        it.load(p);
        for (int hh = 0; hh < D / 64; ++hh)
          tma_store_3d(&tm_o, base + L::Q_OFF + qs * L::TILE + hh * L::HALF, 64 * hh, it.qblk * L::BM, it.bh);
        bulk_commit();
        return true;
      };
      // Loads go in the order in which the MMA warp consumes them: K of the
      // next tile (this item's next one, or the next item's first, followed
      // there by the next item's Q) ahead of V of the current tile.  A K load
      // then waits only for the Q K^T two tiles back; loading V(j) before
      // K(j+1) tied each K load to the P V product two tiles back, and the
      // softmax warps waited ~600 cycles per tile for their next S.
      auto load_q = [&](const FwdSplitCursor& c, int m) -> bool {
        const int qs = m & 1;
        if (m >= 2) {
          // item m-2's O is staged in this buffer: store it, and reuse the
          // buffer once the store has read it
          if (!store_staged(m - 2)) return false;
          bulk_wait_read_all();
        }
        mbar_expect_tx(bar(L::Q_FULL + qs), L::TILE);
        for (int hh = 0; hh < D / 64; ++hh)
          tma_load_3d(base + L::Q_OFF + qs * L::TILE + hh * L::HALF, &tm_q, bar(L::Q_FULL + qs), 64 * hh,
                      c.qblk * L::BM, c.bh);
        q_issued = m + 1;
        return true;
      };
      auto load_k = [&](const FwdSplitCursor& c, int j, int g) -> bool {
        const int s = g & 1, u = g >> 1;
        if (u > 0 && !wait(bar(L::K_EMPTY + s), (u - 1) & 1, 2)) return false;
        mbar_expect_tx(bar(L::K_FULL + s), L::TILE);
        for (int hh = 0; hh < D / 64; ++hh)
          tma_load_3d(base + L::K_OFF + s * L::TILE + hh * L::HALF, &tm_k, bar(L::K_FULL + s), 64 * hh,
                      j * L::BN, c.bh);
        k_issued = g + 1;
        return true;
      };
      auto load_v = [&](const FwdSplitCursor& c, int j, int g) -> bool {
        const int s = g & 1, u = g >> 1;
        if (u > 0 && !wait(bar(L::V_EMPTY + s), (u - 1) & 1, 3)) return false;
        mbar_expect_tx(bar(L::V_FULL + s), L::TILE);
        for (int hh = 0; hh < D / 64; ++hh)
          tma_load_3d(base + L::V_OFF + s * L::TILE + hh * L::HALF, &tm_v, bar(L::V_FULL + s), 64 * hh,
                      j * L::BN, c.bh);
        v_issued = g + 1;
        return true;
      };
      int n = 0, gt = 0;
      bool ok = true;
      if (cur.valid) {
        // cold start: let the first Q K^T's operands arrive before the rest
        // of the rings competes with them for DRAM
        ok = load_q(cur, 0) && load_k(cur, 0, 0) && wait(bar(L::Q_FULL), 0, 23) && wait(bar(L::K_FULL), 0, 24);
      }
      for (; ok && cur.valid; cur.next(p), ++n) {
        for (int j = 0; ok && j < cur.nkv; ++j, ++gt) {
          if (j + 1 < cur.nkv) {
            ok = load_k(cur, j + 1, gt + 1);
          } else if (cur.has_next(p)) {
            FwdSplitCursor nx = cur;
            nx.next(p);
            ok = load_k(nx, 0, gt + 1) && load_q(nx, n + 1);
          }
          ok = ok && load_v(cur, j, gt);
        }
      }
      // the O tiles still staged: the last two items
      if (ok) {
        for (int m = (n >= 2 ? n - 2 : 0); m < n; ++m)
          if (!store_staged(m)) break;
      }
      bulk_wait_all();
      // drain: every load issued must have landed before the CTA may exit
      // (the last two uses of each two-slot ring)
      volatile int never = 0;
      const BoundedWait drain{&never, 1u, limit_ns};
      for (int g = q_issued - 2; g < q_issued; ++g)
        if (g >= 0) drain(bar(L::Q_FULL + (g & 1)), (g >> 1) & 1, 20);
      for (int g = k_issued - 2; g < k_issued; ++g)
        if (g >= 0) drain(bar(L::K_FULL + (g & 1)), (g >> 1) & 1, 21);
      for (int g = v_issued - 2; g < v_issued; ++g)
        if (g >= 0) drain(bar(L::V_FULL + (g & 1)), (g >> 1) & 1, 22);
    }
    __syncwarp();
    teardown();
    return;
  }
  if (warp == 9) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, false, true);
      // Shared-memory descriptors, built once: the start-address field holds
      // address >> 4 in its low 14 bits and every operand lies below 256 KB,
      // so a descriptor for (tile + offset) is the tile's descriptor plus
      // offset >> 4 (no carry leaves the field).
      const uint64_t dq0 = sdesc_sw128(base + L::Q_OFF, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(base + L::K_OFF, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(base + L::V_OFF, L::HALF, 1024);
      constexpr uint64_t kTile = L::TILE >> 4;
      // S(g) = Q(buffer qs) K(stage g&1)^T into the single S slot
      auto issue_s = [&](int qs, int g) {
        const int s = g & 1;
        const uint64_t qa = dq0 + kTile * static_cast<uint64_t>(qs), kb = dk0 + kTile * static_cast<uint64_t>(s);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t koff = ((ks >> 2) * L::HALF + (ks & 3) * 32) >> 4;
          mma_ss(tmem + L::S_COL, qa + koff, kb + koff, IDESC_S, ks > 0 ? 1u : 0u);
        }
        tc_commit(bar(L::S_FULL));
        tc_commit(bar(L::K_EMPTY + s));
      };
      FwdSplitCursor cur;
      cur.start(p);
      int n = 0, gt = 0;
      bool ok = cur.valid && wait(bar(L::Q_FULL), 0, 4) && wait(bar(L::K_FULL), 0, 5);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
      }
      for (; ok && cur.valid; cur.next(p), ++n) {
        const int nkv = cur.nkv;
        const bool more = cur.has_next(p);
        for (int j = 0; j < nkv; ++j, ++gt) {
          // S of the next tile (this item's next one, or the next item's
          // first) as soon as the softmax warps have copied S(gt) out
          const bool last = (j + 1 == nkv);
          if (!last || more) {
            const int qs_next = last ? ((n + 1) & 1) : (n & 1);
            if (last && !wait(bar(L::Q_FULL + qs_next), ((n + 1) >> 1) & 1, 4)) { ok = false; break; }
            if (!wait(bar(L::S_FREE), gt & 1, 6)) { ok = false; break; }
            if (!wait(bar(L::K_FULL + ((gt + 1) & 1)), ((gt + 1) >> 1) & 1, 5)) { ok = false; break; }
            tc_fence_after();
            issue_s(qs_next, gt + 1);
            FA_TRACE_POINT(10);
          }
          if (!wait(bar(L::P_FULL), gt & 1, 7)) { ok = false; break; }
          if (!wait(bar(L::V_FULL + (gt & 1)), (gt >> 1) & 1, 8)) { ok = false; break; }
          tc_fence_after();
          const uint64_t vd = dv0 + kTile * static_cast<uint64_t>(gt & 1);
#pragma unroll
          for (int ks = 0; ks < L::BN / 16; ++ks) {
            const uint64_t b = vd + 128u * ks;
            mma_ts(tmem + L::O_COL, tmem + L::P_COL + 8u * ks, b, IDESC_O, (j > 0 || ks > 0) ? 1u : 0u);
          }
          if constexpr (HP) {
#pragma unroll
            for (int ks = 0; ks < L::BN / 16; ++ks) {
              const uint64_t b = vd + 128u * ks;
              mma_ts(tmem + L::OLO_COL, tmem + L::PLO_COL + 8u * ks, b, IDESC_O, (j > 0 || ks > 0) ? 1u : 0u);
            }
          }
          tc_commit(bar(L::O_READY));
          tc_commit(bar(L::V_EMPTY + (gt & 1)));
          FA_TRACE_POINT(11);
        }
      }
      tc_commit(bar(L::TEARDOWN));
    }
    __syncwarp();
    teardown();
    return;
  }
  {
    // ---------------------------------------------- softmax warps 0..7
    if constexpr (L::SPLIT_REGS) warpgroup_reg_alloc<L::REGS_SOFT>();
    const int h = warp >> 2;           // column half
    const int t = threadIdx.x & 127;   // row within the tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    // compare domain: raw accumulator (d = 64) or scaled scores (d = 128)
    const float cmp_scale = kRawCompare ? 1.f : p.scale;        // x = acc * cmp_scale
    const float to_s = kRawCompare ? p.scale : 1.f;             // S = x * to_s (exact)
    const float exp_c = (kRawCompare ? p.scale : 1.f) * kLog2e; // exp2 argument per unit of x
    const uint64_t EXPC2 = f2_pack(exp_c, exp_c);
    const float beta = p.beta;
    constexpr int DH = D / 2;  // O columns per half
    // Error discipline: the two warpgroups meet on named barrier 1 once per
    // tile and once per item.  A bounded wait that gives up only clears `ok`;
    // the meeting that follows is an AND vote, so both warpgroups leave
    // together and neither is left waiting on a barrier the other no longer
    // reaches.
    bool ok = true;
    const bool stall = inject_stall_here(1u);  // test hook (fa_debug_inject_stall)
    FwdSplitCursor cur;
    cur.start(p);
    int gt = 0;
    for (; cur.valid; cur.next(p)) {
      const int qblk = cur.qblk, nkv = cur.nkv;
      float rm_x = -INFINITY;    // running row max, x domain (same in both halves)
      float m_run = -INFINITY;   // shift in force, S domain
      float l = 0.f;             // running sum of this half's P_bar
      int rs = 0;
      bool left = false;
      for (int j = 0; j < nkv; ++j, ++gt) {
        float x[64];
        float hmax = -INFINITY, hcnt = 0.f;
        ok = ok && wait.warp(bar(L::S_FULL), gt & 1, 9);
        // (after a failed wait the loads below read stale TMEM, which is in
        // bounds and harmless; the vote at the exchange then ends the loop)
        {
          if (threadIdx.x == 0) FA_TRACE_POINT(20);
          tc_fence_after();
          {
            uint32_t r0[32], r1[32];
            const uint32_t sa = tmem + lane_base + L::S_COL + 64u * h;
            tmem_ld32x2(sa, sa + 32, r0, r1);
#pragma unroll
            for (int c = 0; c < 32; ++c) { x[c] = __uint_as_float(r0[c]); x[32 + c] = __uint_as_float(r1[c]); }
          }
          tc_fence_before();
          mbar_arrive(bar(L::S_FREE));
          if (threadIdx.x == 0) FA_TRACE_POINT(21);
          // mask (diagonal tile / ragged tail); column index of x[c] is 64h + c
          const int kv0 = j * L::BN;
          const bool diag = p.causal && (j == qblk);
          const int lim_causal = diag ? t : (L::BN - 1);
          const int lim_len = p.N - 1 - kv0;
          const int lim = (lim_causal < lim_len ? lim_causal : lim_len) - 64 * h;  // last visible local column
          if (lim < 63) {
#pragma unroll
            for (int c = 0; c < 64; ++c) x[c] = (c <= lim) ? x[c] * cmp_scale : -INFINITY;
          } else if (!kRawCompare) {
#pragma unroll
            for (int c = 0; c < 64; ++c) x[c] *= cmp_scale;
          }
          // this half's maximum (three-input max, eight partial maxima)
          float pm[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) pm[u] = -INFINITY;
#pragma unroll
          for (int c = 0; c < 64; c += 16) {
#pragma unroll
            for (int u = 0; u < 8; ++u) pm[u] = fmax3(pm[u], x[c + 2 * u], x[c + 2 * u + 1]);
          }
          hmax = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
          // this half's tie count at its maximum (needed only if it can reach the
          // running maximum); set.eq gives 1.0/0.0, summed exactly in fp32 pairs
          if (__any_sync(0xffffffffu, hmax >= rm_x)) {
            uint64_t cnt2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int c = 0; c < 64; c += 2)
              cnt2[(c >> 1) & 3] = f2_add(cnt2[(c >> 1) & 3], f2_pack(feq(x[c], hmax), feq(x[c + 1], hmax)));
            float c0, c1, c2, c3, c4, c5, c6, c7;
            f2_unpack(cnt2[0], c0, c1);
            f2_unpack(cnt2[1], c2, c3);
            f2_unpack(cnt2[2], c4, c5);
            f2_unpack(cnt2[3], c6, c7);
            hcnt = ((c0 + c1) + (c2 + c3)) + ((c4 + c5) + (c6 + c7));
          }
        }
        // exchange with the other half (double-buffered by tile parity)
        {
          const uint32_t xa = base + L::XCHG_OFF + (((gt & 1) * 2 + h) * 128 + t) * 8;
          asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(xa), "f"(hmax), "f"(hcnt) : "memory");
        }
        ok = named_barrier_and(1, 256, ok);
        if (!ok) { left = true; break; }
        float omax, ocnt;
        {
          const uint32_t xa = base + L::XCHG_OFF + (((gt & 1) * 2 + (1 - h)) * 128 + t) * 8;
          asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(omax), "=f"(ocnt) : "r"(xa) : "memory");
        }
        const float tmax = fmaxf(hmax, omax);
        const int tcnt = static_cast<int>(((hmax == tmax) ? hcnt : 0.f) + ((omax == tmax) ? ocnt : 0.f));
        if (tmax > rm_x) {
          rm_x = tmax;
          rs = tcnt;
        } else if (tmax == rm_x) {
          rs += tcnt;
        }
        const float rm_s = rm_x * to_s;
        float m_new = rm_s;
        if (p.mode != 0 && rs > 1) {
          // binary32 operations without contraction, as the rule states them
          m_new = (rm_s > 0.f) ? __fmul_rn(beta, rm_s) : ((rm_s < 0.f) ? 0.f : __fsub_rn(beta, 1.f));
          if (p.mode == 2 && __fsub_rn(m_new, rm_s) < kShiftMargin) m_new = __fadd_rn(rm_s, kShiftMargin);
        }
        if (threadIdx.x == 0) FA_TRACE_POINT(22);
        // P_bar = exp2(x * exp_c - m * log2e) for this half, packed to bf16 pairs
        // in registers (the TMEM P slot is still being read by the previous P V
        // product); row sum in fp32
        const float nm = -m_new * kLog2e;
        const uint64_t NM2 = f2_pack(nm, nm);
        uint64_t sum2[2] = {0ull, 0ull};
        uint32_t pk[32];
        uint32_t plo[HP ? 32 : 1];  // HP: P_bar - bf16(P_bar), rounded to bf16
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const uint64_t y = f2_fma(f2_pack(x[c], x[c + 1]), EXPC2, NM2);
          float e0, e1;
          if ((c >> 1) % kPolyPeriod == kPolyPeriod - 1) {
            // one pair in kPolyPeriod on the FMA pipe (measured: 43.1 us
            // against 45.1 us for all pairs on the MUFU at g2s; the same holds
            // for 1/16 of the pairs, so the gain is the register allocation
            // this gives the loop, which spills less, rather than MUFU relief)
            f2_unpack(exp2_poly_f2(y), e0, e1);
          } else {
            float y0, y1;
            f2_unpack(y, y0, y1);
            e0 = ex2_approx(y0);
            e1 = ex2_approx(y1);
          }
          sum2[(c >> 1) & 1] = f2_add(sum2[(c >> 1) & 1], f2_pack(e0, e1));
          pk[c >> 1] = pack_bf16x2(e0, e1);
          if constexpr (HP) {
            const float h0 = __uint_as_float(pk[c >> 1] << 16), h1 = __uint_as_float(pk[c >> 1] & 0xffff0000u);
            plo[c >> 1] = pack_bf16x2(e0 - h0, e1 - h1);
          }
        }
        float psum;
        {
          const uint64_t s01 = f2_add(sum2[0], sum2[1]);
          float a, b;
          f2_unpack(s01, a, b);
          psum = a + b;
        }
        // P and O are free once the previous P V product has completed (for
        // the item's first tile the previous item's epilogue has waited)
        if (j > 0) {
          ok = wait.warp(bar(L::O_READY), (gt - 1) & 1, 10);
          if (!ok) continue;  // the next meeting takes everyone out
          if (threadIdx.x == 0) FA_TRACE_POINT(23);
          tc_fence_after();
        }
        tmem_st32(tmem + lane_base + L::P_COL + 32u * h, pk);
        if constexpr (HP) tmem_st32(tmem + lane_base + L::PLO_COL + 32u * h, plo);
        if (j > 0) {
          const bool changed = (m_new != m_run);
          float alpha = 1.f;
          if (changed) {
            alpha = ex2_approx((m_run - m_new) * kLog2e);
            l *= alpha;
          }
          if (__any_sync(0xffffffffu, changed)) {
#pragma unroll 1
            for (int c0 = 0; c0 < (HP ? 2 * DH : DH); c0 += 16) {
              uint32_t r[16];
              const uint32_t acc_col = (c0 < DH) ? (L::O_COL + c0) : (L::OLO_COL + c0 - DH);
              const uint32_t oa = tmem + lane_base + acc_col + DH * h;
              tmem_ld16(oa, r);
#pragma unroll
              for (int c = 0; c < 16; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * alpha);
              tmem_st16(oa, r);
            }
          }
        }
        m_run = m_new;
        l += psum;
        tmem_st_wait();
        tc_fence_before();
        if (!(stall && gt == 0)) mbar_arrive(bar(L::P_FULL));
        if (threadIdx.x == 0) FA_TRACE_POINT(24);
      }
      if (left) break;
      // ----------------------------------------------------------- epilogue
      // (gt is one past the item's last tile)
      ok = ok && wait.warp(bar(L::O_READY), (gt - 1) & 1, 11);
      {
        const uint32_t xa = base + L::XCHG_OFF + ((2 * 2 + h) * 128 + t) * 8;
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(xa), "f"(l) : "memory");
      }
      ok = named_barrier_and(1, 256, ok);
      if (!ok) break;
      tc_fence_after();
      float lo;
      {
        const uint32_t xa = base + L::XCHG_OFF + ((2 * 2 + (1 - h)) * 128 + t) * 8;
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(lo) : "r"(xa) : "memory");
      }
      const float lsum = l + lo;
      const float inv_l = 1.f / lsum;
      // this half's O columns -> bf16 -> the item's Q buffer, 128B-swizzled
      // (and, if asked, the same fp32 values to o_hp)
      const uint32_t stage = base + L::Q_OFF + (cur.r & 1) * L::TILE;
      const int q_row = qblk * L::BM + t;
      // o_hp (HP only) = (O + O_lo) / l; the bf16 o is fa_fwd's, from O alone
      float* hp_row = (HP && q_row < p.N) ? p.o_hp + (static_cast<size_t>(cur.bh) * p.N + q_row) * D + DH * h
                                           : nullptr;
      auto write_hp = [&](float* dst, const uint32_t (&o_)[32], uint32_t lo_col) {
        uint32_t lo[32];
        tmem_ld32(lo_col, lo);
        if (dst) {
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<float4*>(dst + c) = make_float4(
                (__uint_as_float(o_[c]) + __uint_as_float(lo[c])) * inv_l,
                (__uint_as_float(o_[c + 1]) + __uint_as_float(lo[c + 1])) * inv_l,
                (__uint_as_float(o_[c + 2]) + __uint_as_float(lo[c + 2])) * inv_l,
                (__uint_as_float(o_[c + 3]) + __uint_as_float(lo[c + 3])) * inv_l);
        }
      };
      if constexpr (D == 64) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + L::O_COL + 32u * h, r);
        if constexpr (HP) write_hp(hp_row, r, tmem + lane_base + L::OLO_COL + 32u * h);
        const uint32_t rp = stage + t * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int chunk = 4 * h + c;  // 8 bf16 = 16 bytes
          sts128(rp + ((chunk ^ (t & 7)) << 4),
                 pack_bf16x2(__uint_as_float(r[8 * c + 0]) * inv_l, __uint_as_float(r[8 * c + 1]) * inv_l),
                 pack_bf16x2(__uint_as_float(r[8 * c + 2]) * inv_l, __uint_as_float(r[8 * c + 3]) * inv_l),
                 pack_bf16x2(__uint_as_float(r[8 * c + 4]) * inv_l, __uint_as_float(r[8 * c + 5]) * inv_l),
                 pack_bf16x2(__uint_as_float(r[8 * c + 6]) * inv_l, __uint_as_float(r[8 * c + 7]) * inv_l));
        }
      } else {
        uint32_t r0[32], r1[32];
        tmem_ld32x2(tmem + lane_base + L::O_COL + 64u * h, tmem + lane_base + L::O_COL + 64u * h + 32, r0, r1);
        if constexpr (HP) {
          write_hp(hp_row, r0, tmem + lane_base + L::OLO_COL + 64u * h);
          write_hp(hp_row ? hp_row + 32 : nullptr, r1, tmem + lane_base + L::OLO_COL + 64u * h + 32);
        }
        uint32_t w[32];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          w[c] = pack_bf16x2(__uint_as_float(r0[2 * c]) * inv_l, __uint_as_float(r0[2 * c + 1]) * inv_l);
          w[16 + c] = pack_bf16x2(__uint_as_float(r1[2 * c]) * inv_l, __uint_as_float(r1[2 * c + 1]) * inv_l);
        }
        sts_row_sw128(stage + h * L::HALF, t, w);
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(L::O_STAGED + (cur.r & 1)));
      if (threadIdx.x == 0) FA_TRACE_POINT(25);
      if (h == 0 && q_row < p.N) {
        const size_t ri = static_cast<size_t>(cur.bh) * p.N + q_row;
        const float rm_s = rm_x * to_s;
        p.lse[ri] = m_run + logf(lsum);
        if (p.st_rm) p.st_rm[ri] = rm_s;
        if (p.st_rs) p.st_rs[ri] = rs;
        if (p.st_m) p.st_m[ri] = m_run;
        if (p.st_pbar_max) p.st_pbar_max[ri] = ex2_approx((rm_s - m_run) * kLog2e);
      }
    }
    teardown();
  }
}

}  // namespace fa
