// Forward kernel: tiled attention with the stabilised safe softmax.
//
// Method (Qiu & Yao, arXiv 2510.04212; itsolotime.com/archives/23922,
// "mechanism two" and "minimal fix"):
//   S = Q K^T * scale, rm = rowmax(S), rs = rowsum(S == rm),
//   m = beta*rm (rs>1, rm>0) | 0 (rs>1, rm<0) | beta-1 (rs>1, rm==0) | rm,
//   and in the margin mode, on tied rows, m = rm + 2^-8 where m - rm < 2^-8,
//   P_bar = exp(S - m), P = P_bar / rowsum(P_bar), O = P V, lse = m + ln(l).
// The row statistics are kept online across key tiles: a later tile with a
// larger maximum resets (rm, rs); an equal maximum adds its tie count; whenever
// the selected shift m changes, the running sum l and the O accumulator are
// rescaled by exp(m_old - m_new) before the tile's P_bar V product, so every
// P_bar operand is computed against the shift in force for the rows seen so
// far (the final shift once the last tile has been merged).
//
// This file holds the method's formulas and parameters for every forward
// kernel, and the pair kernel that runs head dimension 128 (head dimension 64
// runs the column-split kernel of fa_fwd_split.cuh, which hides the latency
// of the per-tile chain better at that size: 43 us against 47 us for this
// kernel on g2s; at d = 128 this one is faster, 658 us against 823 us on the
// long workload).
//
// Pair kernel: persistent, one CTA per SM.  A work item is a pair of 128-row Q tiles
// of one (batch, head) -- tile slot 0 the longer one (causal: query blocks
// n-1-2p and n-2-2p of n) -- which share every K and V tile they both see;
// items are ordered longest first and dealt to the CTAs in snake order (round
// r gives CTA c item r*G + c for even r, r*G + G-1-c for odd r).
// Sixteen warps:
//   warps 0-3, 4-7   softmax, one warpgroup per tile slot; thread t owns row t
//                    of its tile (TMEM lane t) and all 128 scores of that row
//                    per key tile, so the row statistics need no exchange
//                    between warps.  The two warpgroups work on different
//                    tiles and drift apart: while one computes exponentials
//                    the other finds maxima and tie counts, which keeps the
//                    exponential unit busy.
//   warps 8-11       correction: rescales a tile's O accumulator in TMEM when
//                    a row's shift has moved (off the softmax warps' path: the
//                    MMA warp waits for it before the tile's next P_bar V), and
//                    the epilogue of each item (O / l -> bf16 -> staged
//                    128B-swizzled in the item's Q buffer; lse; row stats).
//   warp 12          TMA producer: Q tiles per item, K and V through rings,
//                    the TMA store of each finished O tile.
//   warp 13          MMA issuer (one thread) and TMEM owner.
//   warps 14-15      idle.
// TMEM: S of tile slot t at columns [128t, 128t+128); P_bar (bf16 pairs)
// overwrites the first 64 of them once the softmax warps hold S in
// registers, and the next S of that slot is issued right after the P_bar V
// product that reads it (tcgen05 products from one thread run in issue
// order).  O of slot t follows the S columns.  In the high-precision variant
// (HP) P_bar also goes out as a second bf16 part P_lo = bf16(P_bar - P_hi) in
// S columns [64,128), multiplied into its own accumulator O_lo.
//
// For d = 64 the scale 1/8 is a power of two, so comparisons (max, ties) are
// taken on the raw fp32 accumulator: x == y <=> x/8 == y/8 and rm = max/8
// exactly.  For d = 128 the scores are scaled first (fp32 multiply), because
// two raw values one ulp apart can round to the same scaled value.
#pragma once

#include "fa_ptx.cuh"

namespace fa {

constexpr float kLog2e = 1.4426950408889634f;
// margin mode: minimum m - rm on rows with a tied maximum (2^-8), so that
// bf16(exp(rm - m)) < 1 as well
constexpr float kShiftMargin = 0.00390625f;
// one exp2 pair in kPolyPeriod goes to the FMA pipe instead of the MUFU
constexpr int kPolyPeriod = 8;

struct FwdParams {
  float* lse;         // [BH, N]
  float* o_hp;        // optional fp32 O [BH, N, D] (the normalised accumulator before bf16 rounding)
  float* st_rm;       // optional [BH, N]
  int32_t* st_rs;     // optional
  float* st_m;        // optional
  float* st_pbar_max; // optional
  int BH, N, n_qblk;
  int causal, mode;
  float beta, scale;
};

template <int D, bool HP = false>
struct FwdLayout {
  // Q tiles per work item: two, except where TMEM cannot hold two tiles'
  // S, O and O_lo (d = 128 with the high-precision O)
  static constexpr int NT = (D == 128 && HP) ? 1 : 2;
  static constexpr int QBUF = (D == 128 && NT == 2) ? 1 : 2;  // Q buffers (items in flight)
  static constexpr int KVS = (D == 64) ? 3 : 2;               // K and V ring stages
  static constexpr int BM = 128, BN = 128;
  static constexpr int TILE = BM * D * 2;  // bytes of a 128 x D bf16 tile
  static constexpr int HALF = 128 * 128;   // bytes of one 128-row x 64-col TMA box
  static constexpr int Q_OFF = 0;                          // [QBUF][NT] tiles (also the O staging tiles)
  static constexpr int K_OFF = Q_OFF + QBUF * NT * TILE;   // [KVS] tiles
  static constexpr int V_OFF = K_OFF + KVS * TILE;         // [KVS] tiles
  static constexpr int ALPHA_OFF = V_OFF + KVS * TILE;     // [2 slots][NT][128] fp32 rescale factors
  static constexpr int FIN_OFF = ALPHA_OFF + 2 * NT * 128 * 4; // [2 item slots][NT][4][128]: l, m, rm, rs
  static constexpr int BAR_OFF = FIN_OFF + 2 * NT * 4 * 128 * 4;
  enum {
    Q_FULL = 0,                  // [2] by Q buffer
    O_STAGED = Q_FULL + 2,       // [2] by Q buffer
    K_FULL = O_STAGED + 2,       // [3] by ring stage
    K_EMPTY = K_FULL + 3,        // [3]
    V_FULL = K_EMPTY + 3,        // [3]
    V_EMPTY = V_FULL + 3,        // [3]
    S_FULL = V_EMPTY + 3,        // [2] by tile slot
    P_FULL = S_FULL + 2,         // [2]
    ALPHA_READY = P_FULL + 2,    // [2 factor slots][2 tile slots]
    CORR_DONE = ALPHA_READY + 4, // [2]
    FIN_READY = CORR_DONE + 2,   // [2 item slots][2 tile slots]: one barrier per FIN slot, so
                                 // that a tile's softmax warps two items ahead stay one phase ahead
    O_DONE = FIN_READY + 4,      // [2]
    O_FREE = O_DONE + 2,         // [2]
    TEARDOWN = O_FREE + 2,
    NBAR
  };
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;  // tmem base (4B), abort flag (4B)
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  __host__ __device__ static constexpr uint32_t s_col(int t) { return 128u * t; }
  __host__ __device__ static constexpr uint32_t o_col(int t) { return 128u * NT + D * t; }
  __host__ __device__ static constexpr uint32_t olo_col(int t) { return 128u * NT + D * NT + D * t; }
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int THREADS = 512;
  // register budgets after setmaxnreg (launched with 128 per thread; the
  // four warpgroups' shares add up to 4 x 128: 2 x 176 + 72 + 88, the split
  // at which no role spills at d = 128)
  static constexpr uint32_t REGS_SOFT = 176, REGS_CORR = 72, REGS_CTRL = 88;
  static_assert(2 * REGS_SOFT + REGS_CORR + REGS_CTRL == 4 * 128, "register split");
};
static_assert(FwdLayout<128, false>::SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert(FwdLayout<128, true>::SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert(FwdLayout<128, false>::o_col(1) + 128 <= 512 && FwdLayout<128, true>::olo_col(0) + 128 <= 512,
              "TMEM budget");

// One work item: NT Q tiles of one (batch, head).  Slot 0 always holds a
// tile; slot 1 may be empty (an odd number of Q tiles).  Causal: slot 0 is
// query block n_qblk-1-2p and slot 1 the block below it, so slot 0 sees one
// key tile more; without the mask both see all of them.
template <int NT>
struct FwdItem {
  int bh, qblk[2], nkv[2];
  bool valid1;
  __device__ __forceinline__ int nkv_max() const { return nkv[0]; }
  __device__ __forceinline__ bool has(int t) const { return t == 0 || valid1; }
  __device__ __forceinline__ static int count(const FwdParams& p) { return ((p.n_qblk + NT - 1) / NT) * p.BH; }
  // the r-th item of this CTA; false past the end of the list
  __device__ __forceinline__ bool load(const FwdParams& p, int r) {
    const int G = gridDim.x, c = blockIdx.x;
    const int w = r * G + ((r & 1) ? (G - 1 - c) : c);
    if (w >= count(p)) return false;
    const int pr = w / p.BH;
    bh = w - pr * p.BH;
    qblk[0] = p.n_qblk - 1 - NT * pr;
    qblk[1] = qblk[0] - 1;
    valid1 = NT == 2 && qblk[1] >= 0;
    nkv[0] = p.causal ? qblk[0] + 1 : p.n_qblk;
    nkv[1] = valid1 ? (p.causal ? qblk[1] + 1 : p.n_qblk) : 0;
    return true;
  }
};

template <int D, bool HP>
__global__ void __launch_bounds__(512, 1)
fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
              const FwdParams p) {
  using L = FwdLayout<D, HP>;
  constexpr int NT = L::NT, QBUF = L::QBUF, KVS = L::KVS;
  constexpr bool kRawCompare = (D == 64);  // scale is exactly 1/8
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;  // 1024-byte aligned for the 128B swizzle
  uint8_t* smem = smem_raw + (base - raw_addr);
  auto bar = [&](int i) { return base + L::BAR_OFF + 8u * i; };
  auto q_tile = [&](int b, int t) { return base + L::Q_OFF + (b * NT + t) * L::TILE; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  const uint64_t limit_ns = wait_limit_ns();
  const BoundedWait wait{abort_flag, 1u, limit_ns};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    FA_TRACE_POINT(0);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(L::Q_FULL + b), 1);
      mbar_init(bar(L::O_STAGED + b), 128);
    }
    for (int s = 0; s < 3; ++s) {
      mbar_init(bar(L::K_FULL + s), 1);
      mbar_init(bar(L::K_EMPTY + s), 1);
      mbar_init(bar(L::V_FULL + s), 1);
      mbar_init(bar(L::V_EMPTY + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(L::S_FULL + t), 1);
      mbar_init(bar(L::P_FULL + t), 128);
      mbar_init(bar(L::ALPHA_READY + t), 128);
      mbar_init(bar(L::ALPHA_READY + 2 + t), 128);
      mbar_init(bar(L::CORR_DONE + t), 128);
      mbar_init(bar(L::FIN_READY + t), 128);
      mbar_init(bar(L::FIN_READY + 2 + t), 128);
      mbar_init(bar(L::O_DONE + t), 1);
      mbar_init(bar(L::O_FREE + t), 128);
    }
    mbar_init(bar(L::TEARDOWN), 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 13) {
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

  // End of every role: all warps meet on named barrier 2, then warp 13 waits
  // for the last MMAs and frees TMEM.  Each role's branch ends on its own (no
  // common tail), so each keeps its own register budget.  No role meets
  // another on a named barrier before this point: a role whose bounded wait
  // gave up leaves its loop and comes straight here, and the others follow as
  // their own waits give up.
  auto teardown = [&]() {
    tc_fence_before();
    named_barrier_sync(2, L::THREADS);
    if (threadIdx.x == 0) FA_TRACE_POINT(2);
    if (warp == 13) {
      tc_fence_after();
      volatile int never = 0;
      const BoundedWait drain{&never, 1u, limit_ns};
      drain(bar(L::TEARDOWN), 0, 30);  // every MMA of this CTA has completed
      tmem_dealloc(tmem, L::TMEM_COLS);
    }
  };

  if (warp >= 12) {
    warpgroup_reg_dealloc<L::REGS_CTRL>();
    if (warp == 12 && lane == 0) {
      // ------------------------------------------------------------ TMA producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_o);
      // counts of the loads issued so far, for the drain at exit
      int q_issued = 0, k_issued = 0, v_issued = 0;
      // item m's O tiles are staged in its Q buffer m % QBUF
      auto store_staged = [&](int m) -> bool {
        const int b = m % QBUF;
        if (!wait(bar(L::O_STAGED + b), (m / QBUF) & 1, 1)) return false;
        FwdItem<NT> it;
        it.load(p, m);
        for (int t = 0; t < NT; ++t) {
          if (!it.has(t)) continue;
          for (int hh = 0; hh < D / 64; ++hh)
            tma_store_3d(&tm_o, q_tile(b, t) + hh * L::HALF, 64 * hh, it.qblk[t] * L::BM, it.bh);
        }
        bulk_commit();
        return true;
      };
      FwdItem<NT> it;
      int n = 0, gk = 0;
      bool ok = true;
      for (; ok && it.load(p, n); ++n) {
        const int b = n % QBUF;
        if (n >= QBUF) {
          // item n-QBUF's O is staged in this buffer: store it, and reuse the
          // buffer once the store has read it
          if (!store_staged(n - QBUF)) break;
          bulk_wait_read_all();
        }
        mbar_expect_tx(bar(L::Q_FULL + b), (it.valid1 ? 2 : 1) * L::TILE);
        for (int t = 0; t < NT; ++t) {
          if (!it.has(t)) continue;
          for (int hh = 0; hh < D / 64; ++hh)
            tma_load_3d(q_tile(b, t) + hh * L::HALF, &tm_q, bar(L::Q_FULL + b), 64 * hh, it.qblk[t] * L::BM,
                        it.bh);
        }
        q_issued = n + 1;
        for (int j = 0; j < it.nkv_max(); ++j) {
          const int g = gk + j, s = g % KVS, u = g / KVS;
          if (u > 0 && !wait(bar(L::K_EMPTY + s), (u - 1) & 1, 2)) { ok = false; break; }
          mbar_expect_tx(bar(L::K_FULL + s), L::TILE);
          for (int hh = 0; hh < D / 64; ++hh)
            tma_load_3d(base + L::K_OFF + s * L::TILE + hh * L::HALF, &tm_k, bar(L::K_FULL + s), 64 * hh,
                        j * L::BN, it.bh);
          k_issued = g + 1;
          if (g == 0) {
            // cold start: let the first Q K^T's operands arrive before the
            // rest of the rings competes with them for DRAM
            if (!wait(bar(L::Q_FULL), 0, 23) || !wait(bar(L::K_FULL), 0, 24)) { ok = false; break; }
          }
          if (u > 0 && !wait(bar(L::V_EMPTY + s), (u - 1) & 1, 3)) { ok = false; break; }
          mbar_expect_tx(bar(L::V_FULL + s), L::TILE);
          for (int hh = 0; hh < D / 64; ++hh)
            tma_load_3d(base + L::V_OFF + s * L::TILE + hh * L::HALF, &tm_v, bar(L::V_FULL + s), 64 * hh,
                        j * L::BN, it.bh);
          v_issued = g + 1;
        }
        gk += it.nkv_max();
      }
      // the O tiles still staged: the last QBUF items
      if (ok) {
        for (int m = (n >= QBUF ? n - QBUF : 0); m < n; ++m)
          if (!store_staged(m)) break;
      }
      bulk_wait_all();
      // drain: every load issued must have landed before the CTA may exit
      volatile int never = 0;
      const BoundedWait drain{&never, 1u, limit_ns};
      for (int g = q_issued - QBUF; g < q_issued; ++g)
        if (g >= 0) drain(bar(L::Q_FULL + (g % QBUF)), (g / QBUF) & 1, 20);
      for (int g = k_issued - KVS; g < k_issued; ++g)
        if (g >= 0) drain(bar(L::K_FULL + (g % KVS)), (g / KVS) & 1, 21);
      for (int g = v_issued - KVS; g < v_issued; ++g)
        if (g >= 0) drain(bar(L::V_FULL + (g % KVS)), (g / KVS) & 1, 22);
    } else if (warp == 13 && lane == 0) {
      // -------------------------------------------------------------- MMA issuer
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, false, true);
      // S_t = Q(buffer b, slot t) K(stage s)^T into slot t's S columns
      // descriptor arithmetic: (tile + offset) is the tile's descriptor plus
      // offset >> 4 (the start-address field holds address >> 4 in 14 bits
      // and every operand lies below 256 KB, so no carry leaves the field)
      const uint64_t dk0 = sdesc_sw128(base + L::K_OFF, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(base + L::V_OFF, L::HALF, 1024);
      constexpr uint64_t kTile = L::TILE >> 4;
      auto issue_s = [&](int b, int t, int s) {
        const uint64_t qa = sdesc_sw128(q_tile(b, t), 16, 1024), kb = dk0 + kTile * static_cast<uint64_t>(s);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t koff = ((ks >> 2) * L::HALF + (ks & 3) * 32) >> 4;
          mma_ss(tmem + L::s_col(t), qa + koff, kb + koff, IDESC_S, ks > 0 ? 1u : 0u);
        }
        tc_commit(bar(L::S_FULL + t));
      };
      // O_t (+)= P_bar_t V(stage s)  (and O_lo_t (+)= P_lo_t V)
      auto issue_pv = [&](int t, int s, bool acc) {
        const uint64_t vd = dv0 + kTile * static_cast<uint64_t>(s);
#pragma unroll
        for (int ks = 0; ks < L::BN / 16; ++ks) {
          const uint64_t bdesc = vd + 128u * ks;
          mma_ts(tmem + L::o_col(t), tmem + L::s_col(t) + 8u * ks, bdesc, IDESC_O, (acc || ks > 0) ? 1u : 0u);
        }
        if constexpr (HP) {
#pragma unroll
          for (int ks = 0; ks < L::BN / 16; ++ks) {
            const uint64_t bdesc = vd + 128u * ks;
            mma_ts(tmem + L::olo_col(t), tmem + L::s_col(t) + 64u + 8u * ks, bdesc, IDESC_O,
                   (acc || ks > 0) ? 1u : 0u);
          }
        }
      };
      FwdItem<NT> it;
      int n = 0, gk = 0;
      int gs[2] = {0, 0}, ga[2] = {0, 0}, gi[2] = {0, 0};  // per slot: S steps, rescale steps, items
      bool ok = true;
      for (; ok && it.load(p, n); ++n) {
        const int b = n % QBUF;
        const int nkv = it.nkv_max();
        {
          const int s0 = gk % KVS;
          if (!wait(bar(L::Q_FULL + b), (n / QBUF) & 1, 4)) break;
          if (!wait(bar(L::K_FULL + s0), (gk / KVS) & 1, 5)) break;
          tc_fence_after();
          for (int t = 0; t < NT; ++t)
            if (it.has(t)) issue_s(b, t, s0);
          tc_commit(bar(L::K_EMPTY + s0));
          FA_TRACE_POINT(10);
        }
        for (int j = 0; ok && j < nkv; ++j) {
          const int g = gk + j, sv = g % KVS;
          const bool next = j + 1 < nkv;
          const int sk = (g + 1) % KVS;
          if (!wait(bar(L::V_FULL + sv), (g / KVS) & 1, 8)) { ok = false; break; }
          if (next && !wait(bar(L::K_FULL + sk), ((g + 1) / KVS) & 1, 5)) { ok = false; break; }
          for (int t = 0; t < NT; ++t) {
            if (!it.has(t) || j >= it.nkv[t]) continue;
            if (!wait(bar(L::P_FULL + t), gs[t] & 1, 7)) { ok = false; break; }
            if (j == 0) {
              // the first product of an item overwrites O_t: the previous
              // item's epilogue must have read it
              if (gi[t] > 0 && !wait(bar(L::O_FREE + t), (gi[t] - 1) & 1, 6)) { ok = false; break; }
            } else {
              if (!wait(bar(L::CORR_DONE + t), ga[t] & 1, 9)) { ok = false; break; }
              ++ga[t];
            }
            tc_fence_after();
            issue_pv(t, sv, j > 0);
            ++gs[t];
            if (j + 1 < it.nkv[t]) {
              issue_s(b, t, sk);  // after the product that reads P_bar_t from the same columns
            } else {
              tc_commit(bar(L::O_DONE + t));
              ++gi[t];
            }
            FA_TRACE_POINT(11 + t);
          }
          if (!ok) break;
          tc_commit(bar(L::V_EMPTY + sv));
          if (next) tc_commit(bar(L::K_EMPTY + sk));
        }
        gk += nkv;
      }
      tc_commit(bar(L::TEARDOWN));
    }
    __syncwarp();
    teardown();
    return;
  }

  if (warp >= 8) {
    // ------------------------------------------------- correction warps 8..11
    warpgroup_reg_dealloc<L::REGS_CORR>();
    const int r = threadIdx.x & 127;  // row within a tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    FwdItem<NT> it;
    int n = 0;
    int ga[2] = {0, 0}, gi[2] = {0, 0};
    bool ok = true;
    for (; ok && it.load(p, n); ++n) {
      const int b = n % QBUF;
      // O rescales: one per tile and key step after the first, in the order
      // the MMA warp issues the P_bar V products
      for (int j = 1; ok && j < it.nkv_max(); ++j) {
        for (int t = 0; t < NT; ++t) {
          if (!it.has(t) || j >= it.nkv[t]) continue;
          const int slot = ga[t] & 1;
          ok = wait.warp(bar(L::ALPHA_READY + 2 * slot + t), (ga[t] >> 1) & 1, 15);
          if (!ok) break;
          ++ga[t];
          const float a = lds32(base + L::ALPHA_OFF + ((slot * NT + t) * 128 + r) * 4);
          if (__any_sync(0xffffffffu, a != 1.f)) {
            tc_fence_after();
#pragma unroll 1
            for (int c0 = 0; c0 < (HP ? 2 * D : D); c0 += 32) {
              const uint32_t col = c0 < D ? L::o_col(t) + c0 : L::olo_col(t) + (c0 - D);
              uint32_t v[32];
              tmem_ld32(tmem + lane_base + col, v);
#pragma unroll
              for (int c = 0; c < 32; ++c) v[c] = __float_as_uint(__uint_as_float(v[c]) * a);
              tmem_st32(tmem + lane_base + col, v);
            }
            tmem_st_wait();
          }
          tc_fence_before();
          mbar_arrive(bar(L::CORR_DONE + t));
        }
      }
      if (!ok) break;
      // epilogue of each tile of the item
      for (int t = 0; t < NT; ++t) {
        if (!it.has(t)) continue;
        ok = wait.warp(bar(L::FIN_READY + 2 * (gi[t] & 1) + t), (gi[t] >> 1) & 1, 16) &&
             wait.warp(bar(L::O_DONE + t), gi[t] & 1, 17);
        if (!ok) break;
        tc_fence_after();
        const uint32_t fin = base + L::FIN_OFF + ((((gi[t] & 1) * NT + t) * 4) * 128 + r) * 4;
        const float l = lds32(fin);
        const float m = lds32(fin + 512);
        const float rm_s = lds32(fin + 1024);
        const int rs = __float_as_int(lds32(fin + 1536));
        ++gi[t];
        const float inv_l = 1.f / l;
        const int q_row = it.qblk[t] * L::BM + r;
        const uint32_t stage = q_tile(b, t);
        float* hp_row = (HP && q_row < p.N) ? p.o_hp + (static_cast<size_t>(it.bh) * p.N + q_row) * D : nullptr;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + L::o_col(t) + c0, v);
          if constexpr (HP) {
            uint32_t lo[32];
            tmem_ld32(tmem + lane_base + L::olo_col(t) + c0, lo);
            if (hp_row) {
#pragma unroll
              for (int c = 0; c < 32; c += 4)
                *reinterpret_cast<float4*>(hp_row + c0 + c) =
                    make_float4((__uint_as_float(v[c]) + __uint_as_float(lo[c])) * inv_l,
                                (__uint_as_float(v[c + 1]) + __uint_as_float(lo[c + 1])) * inv_l,
                                (__uint_as_float(v[c + 2]) + __uint_as_float(lo[c + 2])) * inv_l,
                                (__uint_as_float(v[c + 3]) + __uint_as_float(lo[c + 3])) * inv_l);
            }
          }
          // 32 columns = four 16-byte chunks of row r in the 128B-swizzled
          // box of columns [64*(c0/64), +64)
          const uint32_t rowp = stage + (c0 / 64) * L::HALF + r * 128;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int chunk = ((c0 & 63) >> 3) + c;
            sts128(rowp + ((chunk ^ (r & 7)) << 4),
                   pack_bf16x2(__uint_as_float(v[8 * c + 0]) * inv_l, __uint_as_float(v[8 * c + 1]) * inv_l),
                   pack_bf16x2(__uint_as_float(v[8 * c + 2]) * inv_l, __uint_as_float(v[8 * c + 3]) * inv_l),
                   pack_bf16x2(__uint_as_float(v[8 * c + 4]) * inv_l, __uint_as_float(v[8 * c + 5]) * inv_l),
                   pack_bf16x2(__uint_as_float(v[8 * c + 6]) * inv_l, __uint_as_float(v[8 * c + 7]) * inv_l));
          }
        }
        tc_fence_before();
        mbar_arrive(bar(L::O_FREE + t));  // the next item may overwrite O_t
        if (q_row < p.N) {
          const size_t ri = static_cast<size_t>(it.bh) * p.N + q_row;
          p.lse[ri] = m + logf(l);
          if (p.st_rm) p.st_rm[ri] = rm_s;
          if (p.st_rs) p.st_rs[ri] = rs;
          if (p.st_m) p.st_m[ri] = m;
          if (p.st_pbar_max) p.st_pbar_max[ri] = ex2_approx((rm_s - m) * kLog2e);
        }
      }
      if (!ok) break;
      fence_proxy_async_smem();
      mbar_arrive(bar(L::O_STAGED + b));
      if (threadIdx.x == 256) FA_TRACE_POINT(26);
    }
    teardown();
    return;
  }

  {
    // ------------------------------------------------- softmax warps 0..7
    warpgroup_reg_alloc<L::REGS_SOFT>();
    const int t = warp >> 2;           // tile slot
    const int r = threadIdx.x & 127;   // row within the tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + L::s_col(t);
    // compare domain: raw accumulator (d = 64) or scaled scores (d = 128)
    const float cmp_scale = kRawCompare ? 1.f : p.scale;        // x = acc * cmp_scale
    const float to_s = kRawCompare ? p.scale : 1.f;             // S = x * to_s (exact)
    const float exp_c = (kRawCompare ? p.scale : 1.f) * kLog2e; // exp2 argument per unit of x
    const uint64_t EXPC2 = f2_pack(exp_c, exp_c);
    const float beta = p.beta;
    const bool stall = t == 0 && inject_stall_here(1u);  // test hook (fa_debug_inject_stall)
    FwdItem<NT> it;
    int n = 0, gs = 0, gi = 0, na = 0;
    bool ok = true;
    for (; ok && (NT == 2 || t == 0) && it.load(p, n); ++n) {
      if (!it.has(t)) continue;
      const int qblk = it.qblk[t], nkv = it.nkv[t];
      float rm_x = -INFINITY;    // running row max, x domain
      float m_run = -INFINITY;   // shift in force, S domain
      float l = 0.f;             // running sum of P_bar
      int rs = 0;
      for (int j = 0; j < nkv; ++j, ++gs) {
        ok = wait.warp(bar(L::S_FULL + t), gs & 1, 10);
        if (!ok) break;
        if (r == 0) FA_TRACE_POINT(20 + t);
        tc_fence_after();
        float x[128];
        {
          uint32_t raw[128];
          tmem_ld32x4(s_addr, raw);  // four loads, one wait
#pragma unroll
          for (int c = 0; c < 128; ++c) x[c] = __uint_as_float(raw[c]);
        }
        // mask (diagonal tile / ragged tail); x[c] is key j*128 + c
        {
          const int kv0 = j * L::BN;
          const bool diag = p.causal && (j == qblk);
          const int lim_causal = diag ? r : (L::BN - 1);
          const int lim_len = p.N - 1 - kv0;
          const int lim = lim_causal < lim_len ? lim_causal : lim_len;  // last visible column
          if (lim < L::BN - 1) {
#pragma unroll
            for (int c = 0; c < 128; ++c) x[c] = (c <= lim) ? x[c] * cmp_scale : -INFINITY;
          } else if (!kRawCompare) {
#pragma unroll
            for (int c = 0; c < 128; ++c) x[c] *= cmp_scale;
          }
        }
        // tile maximum: eight partial maxima over the 128 columns, three-input max
        float tmax;
        {
          float pm[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) pm[u] = fmaxf(x[2 * u], x[2 * u + 1]);
#pragma unroll
          for (int c = 16; c < 128; c += 16) {
#pragma unroll
            for (int u = 0; u < 8; ++u) pm[u] = fmax3(pm[u], x[c + 2 * u], x[c + 2 * u + 1]);
          }
          tmax = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
        }
        // tie count at the tile maximum, needed only where it can reach the
        // running maximum; set.eq gives 1.0/0.0, summed exactly in fp32 pairs
        int tcnt = 0;
        if (__any_sync(0xffffffffu, tmax >= rm_x)) {
          uint64_t cnt2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
          for (int c = 0; c < 128; c += 2)
            cnt2[(c >> 1) & 3] = f2_add(cnt2[(c >> 1) & 3], f2_pack(feq(x[c], tmax), feq(x[c + 1], tmax)));
          float ca, cb;
          f2_unpack(f2_add(f2_add(cnt2[0], cnt2[1]), f2_add(cnt2[2], cnt2[3])), ca, cb);
          tcnt = static_cast<int>(ca + cb);
        }
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
        if (j > 0) {
          // hand the rescale factor of O to the correction warps (1 if the
          // shift did not move); they rescale O_t while the exponentials run
          float alpha = 1.f;
          if (m_new != m_run) {
            alpha = ex2_approx((m_run - m_new) * kLog2e);
            l *= alpha;
          }
          // two factor slots, used alternately (one slot would also do here:
          // the next factor is written after S of the next step, which needs
          // this step's P_bar V, which needs the correction warps' hand-back)
          const int slot = na & 1;
          sts32(base + L::ALPHA_OFF + ((slot * NT + t) * 128 + r) * 4, alpha);
          tc_fence_before();
          mbar_arrive(bar(L::ALPHA_READY + 2 * slot + t));
          ++na;
        }
        m_run = m_new;
        if (r == 0) FA_TRACE_POINT(22 + t);
        // P_bar = exp2(x * exp_c - m * log2e), packed to bf16 pairs; row sum in fp32
        const float nm = -m_new * kLog2e;
        const uint64_t NM2 = f2_pack(nm, nm);
        uint64_t sum2[2] = {0ull, 0ull};
        uint32_t pk[64];
        uint32_t plo[HP ? 64 : 1];  // HP: P_bar - bf16(P_bar), rounded to bf16
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          const uint64_t y = f2_fma(f2_pack(x[c], x[c + 1]), EXPC2, NM2);
          float e0, e1;
          if ((c >> 1) % kPolyPeriod == kPolyPeriod - 1) {
            // one pair in kPolyPeriod on the FMA pipe (Cody-Waite +
            // polynomial): fewer exponentials queue on the MUFU
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
        {
          float a, bsum;
          f2_unpack(f2_add(sum2[0], sum2[1]), a, bsum);
          l += a + bsum;
        }
        // P_bar over S columns [0,64) (and P_lo over [64,128)): S is in registers
        tmem_st32(s_addr, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
        tmem_st32(s_addr + 32, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
        if constexpr (HP) {
          tmem_st32(s_addr + 64, *reinterpret_cast<const uint32_t(*)[32]>(&plo[0]));
          tmem_st32(s_addr + 96, *reinterpret_cast<const uint32_t(*)[32]>(&plo[32]));
        }
        tmem_st_wait();
        tc_fence_before();
        if (!(stall && gs == 0)) mbar_arrive(bar(L::P_FULL + t));
        if (r == 0) FA_TRACE_POINT(24 + t);
      }
      if (!ok) break;
      // the item's row results for the correction warps' epilogue
      {
        const uint32_t fin = base + L::FIN_OFF + ((((gi & 1) * NT + t) * 4) * 128 + r) * 4;
        sts32(fin, l);
        sts32(fin + 512, m_run);
        sts32(fin + 1024, rm_x * to_s);
        sts32(fin + 1536, __int_as_float(rs));
        mbar_arrive(bar(L::FIN_READY + 2 * (gi & 1) + t));
        ++gi;
      }
    }
    teardown();
  }
}

}  // namespace fa
