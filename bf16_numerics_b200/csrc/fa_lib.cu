// Host side of libfa_b200.so: argument validation, TMA tensor maps, kernel
// launches, the device error word and optional per-kernel event timing.
// The C ABI is declared (and documented) in include/fa_b200.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "fa_b200.h"
#include "fa_bwd_pipe.cuh"
#include "fa_bwd_pipe128.cuh"
#include "fa_fwd_split.cuh"

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// [BH, N, D] bf16 -> 3-D tensor map, box 64 (d) x 128 (rows) x 1, 128B swizzle.
// Rows past N read as zeros.
bool make_map(CUtensorMap* map, const void* ptr, long long BH, long long N, int D) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(N) * D * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// fp32 dQ accumulator [BH, N, D] -> 3-D tensor map, box 32 (d) x 128 (rows) x 1,
// 128B swizzle: the target of the pipelined backward's TMA reduce-add.
bool make_map_dq(CUtensorMap* map, const void* ptr, long long BH, long long N, int D) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 4, static_cast<cuuint64_t>(N) * D * 4};
  cuuint32_t box[3] = {32, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Last CUDA failure seen by this thread's fa_* call: "<what>: <cudaError name>".
thread_local char g_last_error[256] = "";

fa_status cuda_fail(const char* what, cudaError_t e) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", what, cudaGetErrorName(e));
  return FA_ERR_CUDA;
}
fa_status cuda_fail(const char* what) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s", what);
  return FA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// ------------------------------------------------------------ event timing
struct TimingRec {
  int kernel;
  cudaEvent_t start, stop;
};
// The timing records are shared by all host threads (one lock; timing is a
// measurement aid and off by default).
std::atomic<bool> g_timing{false};
std::mutex g_timing_mutex;
std::vector<TimingRec> g_recs;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {  // caller holds g_timing_mutex
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

struct LaunchTimer {
  int kernel;
  cudaStream_t stream;
  cudaEvent_t start = nullptr;
  LaunchTimer(int k, cudaStream_t s) : kernel(k), stream(s) {
    if (g_timing) {
      std::lock_guard<std::mutex> lock(g_timing_mutex);
      start = take_event();
      if (start) cudaEventRecord(start, stream);
    }
  }
  void done() {
    if (g_timing && start) {
      std::lock_guard<std::mutex> lock(g_timing_mutex);
      cudaEvent_t stop = take_event();
      if (stop) {
        cudaEventRecord(stop, stream);
        g_recs.push_back({kernel, start, stop});
      } else {
        g_event_pool.push_back(start);
      }
    }
  }
};

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel in the stream is finishing; every kernel of this
// library executes griddepcontrol.wait before touching data the previous
// grid may still be producing.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename K>
bool set_smem(K kernel, int bytes) {
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) {
    cuda_fail("cudaFuncSetAttribute(max dynamic shared memory)", e);
    return false;
  }
  return true;
}

// The dynamic shared memory limit of a kernel, raised once per device (the
// attribute belongs to the kernel as loaded on the current device).
template <typename K>
bool ensure_smem(K kernel, int bytes, std::atomic<uint64_t>& done_mask) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return set_smem(kernel, bytes);
  const uint64_t bit = uint64_t{1} << dev;
  if (done_mask.load() & bit) return true;
  if (!set_smem(kernel, bytes)) return false;
  done_mask |= bit;
  return true;
}

// Multiprocessor count of the current device (queried once per device).
int sm_count() {
  static std::atomic<int> cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev] = n;
  }
  return cached[dev].load();
}

// L2 size of the current device in bytes (queried once per device; 0 if unknown).
long long l2_bytes() {
  static std::atomic<long long> cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrL2CacheSize, dev) != cudaSuccess) return 0;
    cached[dev] = n;
  }
  return cached[dev].load();
}

// How many delta blocks clear the dQ accumulator (before their dependency
// wait).  A small accumulator, a quarter of L2 at most, goes to one block per
// SM: those blocks sit beside the forward's CTAs and clear it while the
// forward runs.  A larger one is shared by every block, because clearing it
// beside the forward would push the forward's K and V tiles out of L2.
int delta_clear_blocks(int grid, long long acc_bytes) {
  const int n_sm = sm_count();
  const long long l2 = l2_bytes();
  if (n_sm <= 0 || l2 <= 0 || acc_bytes > l2 / 4 || grid <= n_sm) return grid;
  return n_sm;
}

bool shape_ok(int B, int H, int N, int d) {
  if (B < 0 || H < 0 || N < 0) return false;
  const long long BH = static_cast<long long>(B) * H;
  if (BH * N * d >= (1ll << 40)) return false;
  const long long nblk = (static_cast<long long>(N) + 127) / 128;
  if (BH * nblk >= (1ll << 31)) return false;
  return true;
}

template <int D>
fa_status launch_fwd(const void* q, const void* k, const void* v, void* o, float* o_hp, float* lse,
                     const fa_row_stats* st, int BH, int N, int causal, int mode, float beta, cudaStream_t stream) {
  CUtensorMap mq, mk, mv, mo;
  if (!make_map(&mq, q, BH, N, D) || !make_map(&mk, k, BH, N, D) || !make_map(&mv, v, BH, N, D) ||
      !make_map(&mo, o, BH, N, D))
    return cuda_fail("cuTensorMapEncodeTiled (q/k/v/o)");
  fa::FwdParams p{};
  p.lse = lse;
  p.o_hp = o_hp;
  if (st) {
    p.st_rm = st->rm;
    p.st_rs = st->rs;
    p.st_m = st->m;
    p.st_pbar_max = st->pbar_max;
  }
  p.BH = BH;
  p.N = N;
  p.n_qblk = (N + 127) / 128;
  p.causal = causal;
  p.mode = mode;
  p.beta = beta;
  p.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  // persistent grids: at most one CTA per work item
  const int n_sm = sm_count();
  if (n_sm <= 0) return cuda_fail("cudaDeviceGetAttribute(multiprocessor count)");
  // items of nt Q tiles, ctas_per_sm CTAs of `threads` threads per SM
  auto launch = [&](auto kernel, int smem, int nt, int ctas_per_sm, int threads) {
    const long long items = static_cast<long long>((p.n_qblk + nt - 1) / nt) * BH;
    const long long slots = static_cast<long long>(n_sm) * ctas_per_sm;
    const unsigned grid = static_cast<unsigned>(items < slots ? items : slots);
    LaunchTimer tm(FA_KERNEL_FWD, stream);
    const cudaError_t err = launch_pdl(kernel, dim3(grid), dim3(threads), smem, stream, mq, mk, mv, mo, p);
    tm.done();
    return err;
  };
  cudaError_t e;
  if (D == 64) {
    // column-split kernel: one Q tile per item, two CTAs per SM (one with o_hp)
    if (o_hp == nullptr) {
      using L = fa::FwdSplitLayout<64, false>;
      static std::atomic<uint64_t> attr{0};
      if (!ensure_smem(fa::fa_fwd_split_kernel<64, false>, L::SMEM_BYTES, attr)) return FA_ERR_CUDA;
      e = launch(fa::fa_fwd_split_kernel<64, false>, L::SMEM_BYTES, 1, L::CTAS_PER_SM, L::THREADS);
    } else {
      using L = fa::FwdSplitLayout<64, true>;
      static std::atomic<uint64_t> attr{0};
      if (!ensure_smem(fa::fa_fwd_split_kernel<64, true>, L::SMEM_BYTES, attr)) return FA_ERR_CUDA;
      e = launch(fa::fa_fwd_split_kernel<64, true>, L::SMEM_BYTES, 1, L::CTAS_PER_SM, L::THREADS);
    }
  } else {
    // pair kernel: FwdLayout::NT Q tiles per item, one CTA per SM
    if (o_hp == nullptr) {
      using L = fa::FwdLayout<128, false>;
      static std::atomic<uint64_t> attr{0};
      if (!ensure_smem(fa::fa_fwd_kernel<128, false>, L::SMEM_BYTES, attr)) return FA_ERR_CUDA;
      e = launch(fa::fa_fwd_kernel<128, false>, L::SMEM_BYTES, L::NT, 1, L::THREADS);
    } else {
      using L = fa::FwdLayout<128, true>;
      static std::atomic<uint64_t> attr{0};
      if (!ensure_smem(fa::fa_fwd_kernel<128, true>, L::SMEM_BYTES, attr)) return FA_ERR_CUDA;
      e = launch(fa::fa_fwd_kernel<128, true>, L::SMEM_BYTES, L::NT, 1, L::THREADS);
    }
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : cuda_fail("fa_fwd_kernel launch", e);
}

// Grid of a memory-bound kernel: one block per `per_block` units of work,
// at most 16 resident 256-thread blocks per SM (grid-stride loops take the rest).
int grid_for(long long work, int per_block) {
  long long g = (work + per_block - 1) / per_block;
  const long long cap = 16ll * (sm_count() > 0 ? sm_count() : 148);
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

template <int D>
fa_status launch_bwd(const void* q, const void* k, const void* v, const void* o, bool o_is_hp, const void* dO,
                     const float* lse, const float* row_m, void* dq, void* dk, void* dv, uint8_t* ws, int BH, int N,
                     int causal, int mode, cudaStream_t stream) {
  using LP = fa::BwdPipeLayout;
  using LP128 = fa::BwdPipe128Layout;
  static std::atomic<uint64_t> attr{0};
  if (D == 64) {
    if (!ensure_smem(fa::fa_bwd_main_pipe_kernel, LP::SMEM_BYTES, attr)) return FA_ERR_CUDA;
  } else {
    if (!ensure_smem(fa::fa_bwd_main_pipe128_kernel, LP128::SMEM_BYTES, attr)) return FA_ERR_CUDA;
  }
  const long long rows = static_cast<long long>(BH) * N;
  const int n_blk = (N + 127) / 128;
  // workspace: delta | fp32 dQ accumulator | work-item counter (d = 128)
  float* delta = reinterpret_cast<float*>(ws);
  const size_t acc_off = round256(static_cast<size_t>(rows) * 4);
  const size_t acc_bytes = static_cast<size_t>(rows) * D * 4;  // a multiple of 256
  float* dq_acc = reinterpret_cast<float*>(ws + acc_off);
  unsigned int* item_ctr = reinterpret_cast<unsigned int*>(ws + acc_off + acc_bytes);
  CUtensorMap mq, mk, mv, mdo;
  if (!make_map(&mq, q, BH, N, D) || !make_map(&mk, k, BH, N, D) || !make_map(&mv, v, BH, N, D) ||
      !make_map(&mdo, dO, BH, N, D))
    return cuda_fail("cuTensorMapEncodeTiled (q/k/v/dO)");
  {
    constexpr int rows_per_block = 4 * (32 / (D / 8)) * 2;  // 4 warps x rows per group x 2 groups
    LaunchTimer tm(FA_KERNEL_BWD_DELTA, stream);
    const dim3 grid(grid_for(rows, rows_per_block));
    const int clear_blocks = delta_clear_blocks(static_cast<int>(grid.x), static_cast<long long>(acc_bytes));
    cudaError_t e =
        o_is_hp ? launch_pdl(fa::fa_bwd_delta_kernel<D, float>, grid, dim3(128), 0, stream,
                             static_cast<const float*>(o), static_cast<const __nv_bfloat16*>(dO), delta, dq_acc, rows,
                             clear_blocks)
                : launch_pdl(fa::fa_bwd_delta_kernel<D, __nv_bfloat16>, grid, dim3(128), 0, stream,
                             static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), delta,
                             dq_acc, rows, clear_blocks);
    tm.done();
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("fa_bwd_delta_kernel launch", e);
  }
  {
    fa::BwdParams p{};
    p.lse = lse;
    p.row_m = row_m;
    p.delta = delta;
    p.dq_acc = dq_acc;
    p.item_ctr = item_ctr;
    // d = 128 item order: heads in groups whose fp32 dQ rows (N * D * 4 bytes
    // per head) fit in 32 MB, a quarter of L2, so the reduce-adds of the items
    // in flight hit L2
    {
      const long long per_head = static_cast<long long>(N) * D * 4;
      long long hg = (32ll << 20) / (per_head > 0 ? per_head : 1);
      if (hg < 1) hg = 1;
      if (hg > BH) hg = BH;
      p.head_group = static_cast<int>(hg);
    }
    p.dk = static_cast<__nv_bfloat16*>(dk);
    p.dv = static_cast<__nv_bfloat16*>(dv);
    p.BH = BH;
    p.N = N;
    p.n_blk = n_blk;
    p.causal = causal;
    p.mode = mode;
    p.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
    CUtensorMap mdq;
    if (!make_map_dq(&mdq, dq_acc, BH, N, D)) return cuda_fail("cuTensorMapEncodeTiled (dQ accumulator)");
    // persistent: one CTA per SM (at most one per work item)
    const unsigned grid = static_cast<unsigned>(static_cast<long long>(p.n_blk) * BH);
    const int n_sm = sm_count();
    if (n_sm <= 0) return cuda_fail("cudaDeviceGetAttribute(multiprocessor count)");
    const unsigned pgrid = grid < static_cast<unsigned>(n_sm) ? grid : static_cast<unsigned>(n_sm);
    if (D == 64) {
      CUtensorMap mdk, mdv;
      if (!make_map(&mdk, dk, BH, N, D) || !make_map(&mdv, dv, BH, N, D))
        return cuda_fail("cuTensorMapEncodeTiled (dk/dv)");
      LaunchTimer tm(FA_KERNEL_BWD_MAIN, stream);
      cudaError_t e = launch_pdl(fa::fa_bwd_main_pipe_kernel, dim3(pgrid), dim3(LP::THREADS), LP::SMEM_BYTES, stream,
                                 mq, mk, mv, mdo, mdq, mdk, mdv, p);
      tm.done();
      if (e == cudaSuccess) e = cudaGetLastError();
      if (e != cudaSuccess) return cuda_fail("fa_bwd main kernel launch", e);
    } else {
      LaunchTimer tm(FA_KERNEL_BWD_MAIN, stream);
      cudaError_t e = launch_pdl(fa::fa_bwd_main_pipe128_kernel, dim3(pgrid), dim3(LP128::THREADS),
                                 LP128::SMEM_BYTES, stream, mq, mk, mv, mdo, mdq, p);
      tm.done();
      if (e == cudaSuccess) e = cudaGetLastError();
      if (e != cudaSuccess) return cuda_fail("fa_bwd main kernel launch", e);
    }
  }
  {
    const long long n8 = rows * D / 8;
    LaunchTimer tm(FA_KERNEL_BWD_DQ, stream);
    cudaError_t e = launch_pdl(fa::fa_bwd_dq_convert_kernel, dim3(grid_for(n8, 256 * 4)), dim3(256), 0, stream,
                               static_cast<const float*>(dq_acc), static_cast<__nv_bfloat16*>(dq), n8);
    tm.done();
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("fa_bwd_dq_convert_kernel launch", e);
  }
  return FA_OK;
}

}  // namespace

extern "C" {

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported shape or head dimension";
    case FA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case FA_ERR_CUDA: return "CUDA call or kernel launch failed";
    case FA_ERR_TIMEOUT: return "a kernel gave up on a bounded wait";
  }
  return "unknown status";
}

size_t fa_bwd_workspace_delta_offset(int B, int H, int N, int d) {
  (void)B; (void)H; (void)N; (void)d;
  return 0;
}

size_t fa_bwd_workspace_dq_offset(int B, int H, int N, int d) {
  if (!shape_ok(B, H, N, d)) return 0;
  return round256(static_cast<size_t>(B) * H * N * 4);
}

size_t fa_bwd_workspace_bytes(int B, int H, int N, int d) {
  if (!shape_ok(B, H, N, d) || (d != 64 && d != 128)) return 0;
  const size_t rows = static_cast<size_t>(B) * H * N;
  return round256(rows * 4) + round256(rows * static_cast<size_t>(d) * 4) + 256;
}

}  // extern "C"

namespace {

fa_status fwd_impl(const void* q, const void* k, const void* v, void* o, float* o_hp, bool want_hp, float* lse,
                   const fa_row_stats* stats, int B, int H, int N, int d, int causal, int softmax_mode, float beta,
                   void* stream) {
  if (!shape_ok(B, H, N, d)) return FA_ERR_INVALID_ARG;
  if (softmax_mode != FA_SOFTMAX_STANDARD && softmax_mode != FA_SOFTMAX_STABILIZED &&
      softmax_mode != FA_SOFTMAX_STABILIZED_MARGIN)
    return FA_ERR_INVALID_ARG;
  if (softmax_mode != FA_SOFTMAX_STANDARD && !(std::isfinite(beta) && beta > 1.0f)) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * N == 0) return FA_OK;
  if (!q || !k || !v || !o || !lse || (want_hp && !o_hp)) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (want_hp && !aligned16(o_hp)))
    return FA_ERR_INVALID_ARG;
  if (stats) {
    const void* ptrs[4] = {stats->rm, stats->rs, stats->m, stats->pbar_max};
    for (const void* sp : ptrs)
      if (sp && (reinterpret_cast<uintptr_t>(sp) & 3u)) return FA_ERR_INVALID_ARG;
  }
  const int BH = B * H;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 64) return launch_fwd<64>(q, k, v, o, o_hp, lse, stats, BH, N, causal, softmax_mode, beta, s);
  return launch_fwd<128>(q, k, v, o, o_hp, lse, stats, BH, N, causal, softmax_mode, beta, s);
}

fa_status bwd_impl(const void* q, const void* k, const void* v, const void* o, bool o_is_hp, const void* dO,
                   const float* lse, const float* row_m, void* dq, void* dk, void* dv, void* workspace,
                   size_t workspace_bytes, int B, int H, int N, int d, int causal, int softmax_mode, float beta,
                   void* stream) {
  if (!shape_ok(B, H, N, d)) return FA_ERR_INVALID_ARG;
  if (softmax_mode != FA_SOFTMAX_STANDARD && softmax_mode != FA_SOFTMAX_STABILIZED &&
      softmax_mode != FA_SOFTMAX_STABILIZED_MARGIN)
    return FA_ERR_INVALID_ARG;
  if (softmax_mode != FA_SOFTMAX_STANDARD && !(std::isfinite(beta) && beta > 1.0f)) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * N == 0) return FA_OK;
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (softmax_mode != FA_SOFTMAX_STANDARD && !row_m) return FA_ERR_INVALID_ARG;
  const void* a16[8] = {q, k, v, o, dO, dq, dk, dv};
  for (const void* pp : a16)
    if (!aligned16(pp)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) || (row_m && (reinterpret_cast<uintptr_t>(row_m) & 3u)))
    return FA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_bytes < fa_bwd_workspace_bytes(B, H, N, d))
    return FA_ERR_WORKSPACE;
  const int BH = B * H;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  // both stabilised modes recompute P the same way (P = exp(S - m) / l)
  const int bwd_mode = softmax_mode == FA_SOFTMAX_STANDARD ? 0 : 1;
  if (d == 64)
    return launch_bwd<64>(q, k, v, o, o_is_hp, dO, lse, row_m, dq, dk, dv, ws, BH, N, causal, bwd_mode, s);
  return launch_bwd<128>(q, k, v, o, o_is_hp, dO, lse, row_m, dq, dk, dv, ws, BH, N, causal, bwd_mode, s);
}

}  // namespace

extern "C" {

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, const fa_row_stats* stats, int B,
                 int H, int N, int d, int causal, int softmax_mode, float beta, void* stream) {
  return fwd_impl(q, k, v, o, nullptr, false, lse, stats, B, H, N, d, causal, softmax_mode, beta, stream);
}

fa_status fa_fwd_o_hp(const void* q, const void* k, const void* v, void* o, float* o_hp, float* lse,
                      const fa_row_stats* stats, int B, int H, int N, int d, int causal, int softmax_mode, float beta,
                      void* stream) {
  return fwd_impl(q, k, v, o, o_hp, true, lse, stats, B, H, N, d, causal, softmax_mode, beta, stream);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                 const float* row_m, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B,
                 int H, int N, int d, int causal, int softmax_mode, float beta, void* stream) {
  return bwd_impl(q, k, v, o, false, dO, lse, row_m, dq, dk, dv, workspace, workspace_bytes, B, H, N, d, causal,
                  softmax_mode, beta, stream);
}

fa_status fa_bwd_o_hp(const void* q, const void* k, const void* v, const float* o_hp, const void* dO,
                      const float* lse, const float* row_m, void* dq, void* dk, void* dv, void* workspace,
                      size_t workspace_bytes, int B, int H, int N, int d, int causal, int softmax_mode, float beta,
                      void* stream) {
  return bwd_impl(q, k, v, o_hp, true, dO, lse, row_m, dq, dk, dv, workspace, workspace_bytes, B, H, N, d, causal,
                  softmax_mode, beta, stream);
}

const char* fa_last_error_string(void) { return g_last_error; }

fa_status fa_device_error(unsigned int* code) {
  if (cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_fa_error, sizeof(v)) != cudaSuccess) return FA_ERR_CUDA;
  if (code) *code = v;
  if (v != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(fa::g_fa_error, &zero, sizeof(zero)) != cudaSuccess) return FA_ERR_CUDA;
    return FA_ERR_TIMEOUT;
  }
  return FA_OK;
}

fa_status fa_debug_set_wait_limit_ns(unsigned long long ns) {
  const unsigned long long v = ns == 0 ? 2000000000ull : ns;
  if (cudaMemcpyToSymbol(fa::g_fa_wait_limit_ns, &v, sizeof(v)) != cudaSuccess)
    return cuda_fail("cudaMemcpyToSymbol(wait limit)", cudaGetLastError());
  return FA_OK;
}

fa_status fa_debug_inject_stall(unsigned int kernel_id) {
  if (kernel_id != 0 && kernel_id != FA_ERRWORD_FWD && kernel_id != FA_ERRWORD_BWD_D64 &&
      kernel_id != FA_ERRWORD_BWD_D128)
    return FA_ERR_INVALID_ARG;
  if (cudaMemcpyToSymbol(fa::g_fa_inject, &kernel_id, sizeof(kernel_id)) != cudaSuccess)
    return cuda_fail("cudaMemcpyToSymbol(stall injection)", cudaGetLastError());
  return FA_OK;
}

fa_status fa_timing_enable(int enable) {
  g_timing = enable != 0;
  return FA_OK;
}

fa_status fa_timing_read(int* launches, double* total_ms) {
  if (!launches || !total_ms) return FA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_timing_mutex);
  for (int i = 0; i < FA_NUM_KERNELS; ++i) {
    launches[i] = 0;
    total_ms[i] = 0.0;
  }
  fa_status st = FA_OK;
  for (const TimingRec& r : g_recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) {
      st = FA_ERR_CUDA;
    } else if (r.kernel >= 0 && r.kernel < FA_NUM_KERNELS) {
      launches[r.kernel] += 1;
      total_ms[r.kernel] += ms;
    }
    g_event_pool.push_back(r.start);
    g_event_pool.push_back(r.stop);
  }
  g_recs.clear();
  return st;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free backward (declared in fa_b200.h next to fa_bwd).
//
// For callers that cannot allocate device memory (a static memory plan fixed
// at start-up, or a plug-in without an allocator of its own): the backward's
// scratch -- delta followed by the fp32 dQ accumulator, laid out exactly as
// fa_bwd's workspace -- lives in the file-scope array below.  Its name is a
// host-side stand-in in host code, so the device address is looked up once
// per device with cudaGetSymbolAddress (device current) and that address is
// what the kernels receive.  Nothing here allocates.  The delta kernel clears
// the dQ accumulator on every call; delta is overwritten in full.  All calls
// share the array: overlapping calls race.
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 256;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

fa_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return FA_OK;
}

}  // namespace

extern "C" fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                    const float* lse, const float* row_m, void* dq, void* dk, void* dv, int B, int H,
                                    int N, int d, int causal, int softmax_mode, float beta, void* stream) {
  if (!shape_ok(B, H, N, d)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (fa_bwd_workspace_bytes(B, H, N, d) > FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const fa_status st = noalloc_scratch(&scratch);
  if (st != FA_OK) return st;
  return fa_bwd(q, k, v, o, dO, lse, row_m, dq, dk, dv, scratch, FA_NOALLOC_SCRATCH_BYTES, B, H, N, d, causal,
                softmax_mode, beta, stream);
}
