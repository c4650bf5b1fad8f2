// Host side of libcutbce: argument checks, the planner (tile geometry,
// vocabulary splits, workspace layout), TMA descriptors and the launch
// sequence on one stream.  Everything here is plain C++ over the CUDA runtime;
// the library allocates no device memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "cutbce.h"
#include "common.cuh"
#include "prep_finish.cuh"
#include "pair_sort.cuh"
#include "tile_engine.cuh"
#include "probes.cuh"
#include "topk.cuh"

namespace {
using namespace cutbce;

constexpr long long kDefaultTimeoutNs = 2000000000LL;  // 2 s per wait: far above any tile's latency
constexpr int64_t kSplitItemsTarget = 16 * 148;        // about 16 dH work items per SM of a 148-SM part

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Blocks of the finish kernel: one thread per dH element, and at least 256
// blocks so that the loss partials are summed by many blocks.  Depends only on
// T and D, so the summation order never depends on the device.
int64_t finish_grid(int64_t T, int64_t D) { return std::max<int64_t>(256, ceil_div(T * D, kFinishThreads)); }

// Outputs one call computes; the workspace plan holds only what they need.
struct Want {
  bool loss, dE, dH, met;
};
constexpr Want kWantAll{true, true, true, false};
constexpr int kAllOutputs = CUTBCE_OUT_LOSS | CUTBCE_OUT_DH | CUTBCE_OUT_DE | CUTBCE_OUT_METRICS;

Want want_from_mask(int outputs) {
  return Want{(outputs & CUTBCE_OUT_LOSS) != 0, (outputs & CUTBCE_OUT_DE) != 0, (outputs & CUTBCE_OUT_DH) != 0,
              (outputs & CUTBCE_OUT_METRICS) != 0};
}

// Options of one call, validated (see cutbce_options in the header).
struct Opts {
  int32_t* metrics = nullptr;
  const float* weights = nullptr;
  bool grad_bf16 = false, acc_dH = false, acc_dE = false;
  int64_t v_off = 0, V_total = 0;   // V_total resolved: the problem's V when not sharded
  bool one_stream = false;           // everything on the caller's stream (no pooled second stream)
  // A call in parts (the host-buffer entry, tensor-core path): kPhasePrep
  // compacts the rows and orders the pairs (no E read), kPhasePasses runs the
  // two tile passes over item tiles [tile_begin, tile_end) and vocabulary
  // splits [split_begin, split_end), kPhaseFinish sums the sparse correction
  // and the column sums and finishes.  All three in one call is the plain call.
  int phases = 7;
  int tile_begin = 0, tile_end = INT_MAX, split_begin = 0, split_end = INT_MAX;
};
constexpr int kPhasePrep = 1, kPhasePasses = 2, kPhaseFinish = 4;

cutbce_status resolve_opts(const cutbce_problem* p, const cutbce_options* o, Opts& out) {
  out = Opts{};
  out.V_total = p->V;
  if (o == nullptr) return CUTBCE_OK;
  out.metrics = o->metrics;
  out.weights = o->weights;
  if (o->grad_dtype != CUTBCE_GRAD_F32 && o->grad_dtype != CUTBCE_GRAD_BF16) return CUTBCE_ERR_UNSUPPORTED;
  if (o->accumulate < 0 || o->accumulate > (CUTBCE_ACCUMULATE_DH | CUTBCE_ACCUMULATE_DE)) return CUTBCE_ERR_INVALID_ARG;
  out.grad_bf16 = o->grad_dtype == CUTBCE_GRAD_BF16;
  out.acc_dH = (o->accumulate & CUTBCE_ACCUMULATE_DH) != 0;
  out.acc_dE = (o->accumulate & CUTBCE_ACCUMULATE_DE) != 0;
  if (o->V_total == 0) {
    if (o->vocab_offset != 0) return CUTBCE_ERR_INVALID_ARG;
  } else {
    if (o->vocab_offset < 0 || o->V_total < 0 || o->vocab_offset + p->V > o->V_total ||
        o->V_total >= (int64_t(1) << 31))
      return CUTBCE_ERR_INVALID_ARG;
    out.v_off = o->vocab_offset;
    out.V_total = o->V_total;
  }
  if (out.weights != nullptr && (reinterpret_cast<uintptr_t>(out.weights) & 3) != 0) return CUTBCE_ERR_INVALID_ARG;
  if (out.metrics != nullptr && (reinterpret_cast<uintptr_t>(out.metrics) & 15) != 0) return CUTBCE_ERR_INVALID_ARG;
  return CUTBCE_OK;
}

// (group, column slab) combinations of the position-owned pass's epilogue: one
// metrics partial per split and combination.
constexpr int kMetSlotsPerSplit = kNumEpiWarps / 4;

struct Plan {
  int64_t T, V, D, K;
  int dtype, reduction;
  int DP, BN;
  int64_t Tpad, n_vitems, n_gather_blocks;
  int S, tps, n_vtiles_bn;
  int radix_passes, radix_blocks;
  size_t elem;
  size_t o_hdr, o_cidx, o_orig, o_rowcnt, o_rowptr, o_ids, o_pair_t, o_pair_v, o_srt[4], o_ghist, o_cscoff, o_hc,
      o_lpart, o_cpart, o_dhpart, o_fpart, o_metpart, o_wc, o_csum, total;
  int met_slots;
  int csum_nbE, csum_nbH;   // column-sum blocks (loss on the tensor-core path), 0 otherwise
};

cutbce_status check_problem(const cutbce_problem* p, bool need_data) {
  if (p == nullptr) return CUTBCE_ERR_INVALID_ARG;
  if (p->T <= 0 || p->V <= 0 || p->D <= 0 || p->K <= 0) return CUTBCE_ERR_INVALID_ARG;
  if (p->dtype != CUTBCE_BF16 && p->dtype != CUTBCE_F32) return CUTBCE_ERR_UNSUPPORTED;
  if (p->reduction < 0 || p->reduction > 2) return CUTBCE_ERR_INVALID_ARG;
  if (p->K > kMaxK || p->D > kMaxDim) return CUTBCE_ERR_UNSUPPORTED;
  if (p->dtype == CUTBCE_BF16 && (p->D % 8) != 0) return CUTBCE_ERR_UNSUPPORTED;
  if (p->V >= (int64_t(1) << 31) || p->T >= (int64_t(1) << 30) || p->T * p->K >= (int64_t(1) << 31))
    return CUTBCE_ERR_UNSUPPORTED;
  // the item-owned pass packs a compacted position into 24 bits
  if (p->dtype == CUTBCE_BF16 && round_up(p->T, kTileM) >= (int64_t(1) << kPairPosBits)) return CUTBCE_ERR_UNSUPPORTED;
  if (need_data) {
    if (p->H == nullptr || p->E == nullptr || p->targets == nullptr) return CUTBCE_ERR_INVALID_ARG;
    if (p->dtype == CUTBCE_BF16 &&
        ((reinterpret_cast<uintptr_t>(p->H) | reinterpret_cast<uintptr_t>(p->E)) & 15) != 0)
      return CUTBCE_ERR_INVALID_ARG;
  }
  return CUTBCE_OK;
}

// Workspace layout.  The header and the per-position arrays come first, at the
// same offsets for every set of outputs (cutbce_read_status and
// cutbce_read_counts rely on that); the pair-sort buffers (dE only) and the dH
// split partials (dH only) are laid out only when those outputs are wanted.
void make_plan(const cutbce_problem* p, Want w, Plan& pl, bool weighted = false) {
  pl.T = p->T;
  pl.V = p->V;
  pl.D = p->D;
  pl.K = p->K;
  pl.dtype = p->dtype;
  pl.reduction = p->reduction;
  const bool bf16 = p->dtype == CUTBCE_BF16;
  pl.DP = bf16 ? static_cast<int>(round_up(p->D, 64)) : static_cast<int>(p->D);
  pl.BN = (bf16 && pl.DP > 128) ? 64 : 128;
  pl.elem = bf16 ? 2 : 4;
  pl.Tpad = round_up(p->T, kTileM);
  pl.n_vitems = ceil_div(p->V, kTileM);
  pl.n_gather_blocks = ceil_div(pl.Tpad, 8);
  {
    int bits = 0;
    while ((int64_t(1) << bits) < pl.n_vitems) ++bits;
    pl.radix_passes = std::max(1, (bits + 7) / 8);     // 8-bit digits of the item-tile index
    pl.radix_blocks = static_cast<int>(std::max<int64_t>(1, ceil_div(p->T * p->K, kRadixTile)));
  }
  if (bf16) {
    pl.n_vtiles_bn = static_cast<int>(ceil_div(p->V, pl.BN));
    const int64_t nTmax = ceil_div(p->T, kTileM);
    int64_t s0 = ceil_div(kSplitItemsTarget, nTmax);
    s0 = std::max<int64_t>(1, std::min<int64_t>({s0, kMaxSplits, pl.n_vtiles_bn}));
    pl.tps = static_cast<int>(ceil_div(pl.n_vtiles_bn, s0));
    pl.S = static_cast<int>(ceil_div(pl.n_vtiles_bn, pl.tps));  // every split is non-empty
  } else {
    pl.n_vtiles_bn = 0;
    pl.tps = 0;
    pl.S = 1;
  }
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  const size_t TK = static_cast<size_t>(p->T) * p->K;
  pl.o_hdr = take(256);
  pl.o_cidx = take(4 * p->T);
  pl.o_orig = take(4 * p->T);
  pl.o_rowcnt = take(4 * p->T);
  pl.o_rowptr = take(4 * (p->T + 1));
  pl.o_ids = take(4 * TK);
  pl.o_pair_t = take(4 * TK);
  pl.o_pair_v = take(4 * TK);
  pl.o_hc = take(pl.elem * static_cast<size_t>(pl.Tpad) * pl.DP);
  // dense loss partials: per item tile, or (weighted loss on the tensor-core path)
  // per position-owned work item
  const int64_t n_loss_items = (weighted && bf16 && w.loss) ? std::max<int64_t>(pl.n_vitems, int64_t(pl.S) * (pl.Tpad / kTileM))
                                                           : pl.n_vitems;
  pl.o_lpart = take(8 * kNumEpiWarps * static_cast<size_t>(n_loss_items));
  pl.o_wc = weighted ? take(4 * static_cast<size_t>(pl.Tpad)) : 0;
  pl.o_cpart = take(8 * pl.n_gather_blocks);
  pl.o_fpart = take(16 * static_cast<size_t>(finish_grid(p->T, p->D)));
  const bool sort = bf16 && w.dE;
  for (int k = 0; k < 4; ++k) pl.o_srt[k] = sort ? take(4 * TK) : 0;
  pl.o_ghist = sort ? take(4 * 256 * static_cast<size_t>(pl.radix_blocks)) : 0;
  pl.o_cscoff = sort ? take(4 * static_cast<size_t>(pl.n_vitems + 1)) : 0;
  pl.o_dhpart = w.dH ? take(4 * static_cast<size_t>(pl.S) * pl.Tpad * pl.DP) : 0;
  pl.met_slots = bf16 ? pl.S * kMetSlotsPerSplit : 1;
  pl.o_metpart = w.met ? take(8 * static_cast<size_t>(pl.met_slots) * pl.Tpad) : 0;
  // the linear half of the dense loss (tensor-core path): column sums of E and of H_c
  pl.csum_nbE = (bf16 && w.loss) ? kColSumBlocksE : 0;
  pl.csum_nbH = (bf16 && w.loss) ? static_cast<int>(std::min<int64_t>(kColSumBlocksHMax, ceil_div(pl.Tpad, 256))) : 0;
  pl.o_csum = (bf16 && w.loss) ? take(8 * static_cast<size_t>(pl.csum_nbE + pl.csum_nbH) * p->D) : 0;
  pl.total = o;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// ---------------------------------------------------------------- device facts (cached)
struct DeviceFacts {
  int sms = 0, major = 0, minor = 0;
};
DeviceFacts g_dev[64];
std::mutex g_dev_mu;

cutbce_status device_facts(DeviceFacts& out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return CUTBCE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_dev[dev].sms == 0) {
    DeviceFacts f;
    if (cudaDeviceGetAttribute(&f.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&f.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&f.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return CUTBCE_ERR_CUDA;
    g_dev[dev] = f;
  }
  out = g_dev[dev];
  return CUTBCE_OK;
}

// ---------------------------------------------------------------- TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// A row-major bf16 matrix [rows, cols] with row stride `stride_elems`, read in
// boxes of 64 columns (128 bytes, 128-byte swizzle) by `box_rows` rows.
// Columns >= cols and rows >= rows read as zero.
bool make_map(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int64_t stride_elems, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(stride_elems * 2)};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- launch profiling (benchmarks)
struct ProfRecord {
  int kind;
  cudaEvent_t start, end;
};
struct Profiler {
  std::mutex mu;
  bool enabled = false;
  std::vector<cudaEvent_t> pool;
  std::vector<ProfRecord> pending;
  double ms[CUTBCE_NUM_KERNEL_KINDS] = {};
  int64_t launches[CUTBCE_NUM_KERNEL_KINDS] = {};

  cudaEvent_t take() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    return cudaEventCreate(&e) == cudaSuccess ? e : nullptr;
  }
  void drain() {  // caller holds mu
    for (const ProfRecord& r : pending) {
      float t = 0.f;
      if (cudaEventSynchronize(r.end) == cudaSuccess && cudaEventElapsedTime(&t, r.start, r.end) == cudaSuccess) {
        ms[r.kind] += t;
        launches[r.kind] += 1;
      }
      pool.push_back(r.start);
      pool.push_back(r.end);
    }
    pending.clear();
  }
};
Profiler g_prof;

// Brackets one kernel launch with events when profiling is on.
struct LaunchScope {
  int kind;
  cudaStream_t st;
  cudaEvent_t a = nullptr, b = nullptr;
  LaunchScope(int k, cudaStream_t s) : kind(k), st(s) {
    std::lock_guard<std::mutex> lk(g_prof.mu);
    if (!g_prof.enabled) return;
    if (g_prof.pending.size() > 4096) g_prof.drain();
    a = g_prof.take();
    b = g_prof.take();
    if (a && b) cudaEventRecord(a, st);
  }
  ~LaunchScope() {
    if (!(a && b)) return;
    cudaEventRecord(b, st);
    std::lock_guard<std::mutex> lk(g_prof.mu);
    g_prof.pending.push_back(ProfRecord{kind, a, b});
  }
};

// ---------------------------------------------------------------- tile-engine dispatch
template <int DP, bool kLoss, bool kGrad, bool kDH, bool kMet>
cudaError_t launch_tile(int grid, const CUtensorMap& s, const CUtensorMap& x, const TileParams& tp,
                        cudaStream_t st) {
  auto kern = k_tile<DP, kLoss, kGrad, kDH, kMet>;
  constexpr uint32_t smem = TileCfg<DP, epi_groups<kDH>()>::SMEM_BYTES;
  // the attribute belongs to the current device: set it once per device
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const uint64_t bit = uint64_t(1) << dev;
  if ((configured.load(std::memory_order_acquire) & bit) == 0) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit, std::memory_order_acq_rel);
  }
  kern<<<grid, kTileThreads, smem, st>>>(s, x, tp);
  return cudaGetLastError();
}

template <bool kLoss, bool kGrad, bool kDH, bool kMet = false>
cudaError_t launch_tile_dp(int DP, int grid, const CUtensorMap& s, const CUtensorMap& x, const TileParams& tp,
                           cudaStream_t st) {
  switch (DP) {
    case 64: return launch_tile<64, kLoss, kGrad, kDH, kMet>(grid, s, x, tp, st);
    case 128: return launch_tile<128, kLoss, kGrad, kDH, kMet>(grid, s, x, tp, st);
    case 192: return launch_tile<192, kLoss, kGrad, kDH, kMet>(grid, s, x, tp, st);
    case 256: return launch_tile<256, kLoss, kGrad, kDH, kMet>(grid, s, x, tp, st);
    default: return cudaErrorInvalidValue;
  }
}

// ---------------------------------------------------------------- top-k dispatch
template <int DP, int KMAX>
cudaError_t launch_topk(int grid, const CUtensorMap& q, const CUtensorMap& e, const TopkParams& tp,
                        cudaStream_t st) {
  auto kern = k_topk<DP, KMAX>;
  constexpr uint32_t smem = TopkCfg<DP>::SMEM_BYTES;
  static std::atomic<uint64_t> configured{0};   // the attribute belongs to the current device
  int dev = 0;
  cudaError_t e2 = cudaGetDevice(&dev);
  if (e2 != cudaSuccess) return e2;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const uint64_t bit = uint64_t(1) << dev;
  if ((configured.load(std::memory_order_acquire) & bit) == 0) {
    e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e2 != cudaSuccess) return e2;
    configured.fetch_or(bit, std::memory_order_acq_rel);
  }
  kern<<<grid, kTileThreads, smem, st>>>(q, e, tp);
  return cudaGetLastError();
}

template <int KMAX>
cudaError_t launch_topk_dp(int DP, int grid, const CUtensorMap& q, const CUtensorMap& e, const TopkParams& tp,
                           cudaStream_t st) {
  switch (DP) {
    case 64: return launch_topk<64, KMAX>(grid, q, e, tp, st);
    case 128: return launch_topk<128, KMAX>(grid, q, e, tp, st);
    case 192: return launch_topk<192, KMAX>(grid, q, e, tp, st);
    case 256: return launch_topk<256, KMAX>(grid, q, e, tp, st);
    default: return cudaErrorInvalidValue;
  }
}

struct TopkPlan {
  int DP, BN, KMAX, n_qt, n_vtiles, S, tps;
  size_t o_hdr, o_s, o_i, total;
};

cutbce_status topk_plan(int64_t B, int64_t V, int64_t D, int k, int sms, TopkPlan& tp) {
  if (B <= 0 || V <= 0 || D <= 0 || k <= 0) return CUTBCE_ERR_INVALID_ARG;
  if (D % 8 != 0 || D > kMaxDim || k > 16 || V >= (int64_t(1) << 31) || B >= (int64_t(1) << 24))
    return CUTBCE_ERR_UNSUPPORTED;
  tp.DP = static_cast<int>(round_up(D, 64));
  tp.BN = tp.DP <= 128 ? 128 : 64;
  tp.KMAX = k <= 8 ? 8 : 16;
  tp.n_qt = static_cast<int>(ceil_div(B, kTileM));
  tp.n_vtiles = static_cast<int>(ceil_div(V, tp.BN));
  // about one work item per SM of a 148-SM part, every split non-empty; depends
  // only on the sizes, so the merge order never depends on the device
  (void)sms;
  const int64_t s0 = std::max<int64_t>(1, std::min<int64_t>(tp.n_vtiles, ceil_div(148, tp.n_qt)));
  tp.tps = static_cast<int>(ceil_div(tp.n_vtiles, s0));
  tp.S = static_cast<int>(ceil_div(tp.n_vtiles, tp.tps));
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  const size_t n = static_cast<size_t>(tp.n_qt) * tp.S * 4 * kTileM * tp.KMAX;
  tp.o_hdr = take(256);
  tp.o_s = take(4 * n);
  tp.o_i = take(4 * n);
  tp.total = o;
  return CUTBCE_OK;
}

// Second streams: the host-buffer entry copies dE out on one, ordered after the
// item-owned pass by an event, and a call that computes the loss runs the
// column sums of E on one, concurrently with the prep kernels.  Streams and
// events are created once per device and pooled: each call takes what it uses
// for its duration, so concurrent calls never share an event.
struct SideStream {
  int dev;
  cudaStream_t s;
  cudaEvent_t ev, ev2;
};
std::mutex g_side_mu;
std::vector<SideStream> g_side_free;

cutbce_status take_side_stream(SideStream& out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return CUTBCE_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lk(g_side_mu);
    for (size_t i = 0; i < g_side_free.size(); ++i) {
      if (g_side_free[i].dev == dev) {
        out = g_side_free[i];
        g_side_free.erase(g_side_free.begin() + static_cast<std::ptrdiff_t>(i));
        return CUTBCE_OK;
      }
    }
  }
  out.dev = dev;
  if (cudaStreamCreateWithFlags(&out.s, cudaStreamNonBlocking) != cudaSuccess) return CUTBCE_ERR_CUDA;
  if (cudaEventCreateWithFlags(&out.ev, cudaEventDisableTiming) != cudaSuccess) {
    cudaStreamDestroy(out.s);
    return CUTBCE_ERR_CUDA;
  }
  if (cudaEventCreateWithFlags(&out.ev2, cudaEventDisableTiming) != cudaSuccess) {
    cudaEventDestroy(out.ev);
    cudaStreamDestroy(out.s);
    return CUTBCE_ERR_CUDA;
  }
  return CUTBCE_OK;
}

void give_side_stream(const SideStream& s) {
  std::lock_guard<std::mutex> lk(g_side_mu);
  g_side_free.push_back(s);
}

// Gives a taken side stream back when the call returns, on every path.
struct SideStreamLease {
  SideStream s{};
  bool held = false;
  ~SideStreamLease() {
    if (held) give_side_stream(s);
  }
};

int count_launches(const Plan& pl, Want w) {
  const bool bf16 = pl.dtype == CUTBCE_BF16;
  int n = 3;                                            // rows, scan, gather
  if (bf16 && w.dE) n += 1 + 3 * pl.radix_passes + 1;   // sort keys, radix passes, item-tile offsets
  if (bf16 && w.loss) n += 2;                           // column sums of E (second stream) and of H_c
  if (w.loss || w.dE) n += 1;                           // item-owned pass
  if (w.dH || w.met) n += 1;                            // position-owned pass (dH and/or metrics)
  if (w.loss || w.dH || w.met) n += 1;                  // finish
  return n;
}

// after_item: if not null, recorded on `st` right after the item-owned pass,
// the point from which dE is final.
cutbce_status run(const cutbce_problem* p, const float* grad_loss, double* loss, void* dH, void* dE, Want w,
                  void* ws, size_t ws_bytes, cudaStream_t st, cudaEvent_t after_item = nullptr,
                  Opts o = Opts{}) {
  if (o.V_total == 0) o.V_total = p->V;   // not sharded
  cutbce_status s = check_problem(p, true);
  if (s != CUTBCE_OK) return s;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255) != 0) return CUTBCE_ERR_INVALID_ARG;
  if ((w.loss && loss == nullptr) || (w.met && o.metrics == nullptr)) return CUTBCE_ERR_INVALID_ARG;
  const bool weighted = o.weights != nullptr;
  Plan pl;
  make_plan(p, w, pl, weighted);
  if (ws_bytes < pl.total) return CUTBCE_ERR_WORKSPACE;
  DeviceFacts dev;
  if ((s = device_facts(dev)) != CUTBCE_OK) return s;
  const bool bf16 = p->dtype == CUTBCE_BF16;
  if (bf16 && !(dev.major == 10 && dev.minor == 0)) return CUTBCE_ERR_UNSUPPORTED;

  const int T = static_cast<int>(p->T), V = static_cast<int>(p->V), D = static_cast<int>(p->D),
            K = static_cast<int>(p->K);
  WsHeader* hdr = at<WsHeader>(ws, pl.o_hdr);
  int* cidx = at<int>(ws, pl.o_cidx);
  int* orig = at<int>(ws, pl.o_orig);
  int* rowcnt = at<int>(ws, pl.o_rowcnt);
  int* rowptr = at<int>(ws, pl.o_rowptr);
  int* ids = at<int>(ws, pl.o_ids);
  int* pair_t = at<int>(ws, pl.o_pair_t);
  int* pair_v = at<int>(ws, pl.o_pair_v);
  double* lpart = at<double>(ws, pl.o_lpart);
  double* cpart = at<double>(ws, pl.o_cpart);
  int* cscoff = at<int>(ws, pl.o_cscoff);
  int* ghist = at<int>(ws, pl.o_ghist);
  float* dhpart = at<float>(ws, pl.o_dhpart);
  int2* metpart = w.met ? at<int2>(ws, pl.o_metpart) : nullptr;
  float* wc = weighted ? at<float>(ws, pl.o_wc) : nullptr;

#define CUTBCE_CK(x)                           \
  do {                                         \
    if ((x) != cudaSuccess) return CUTBCE_ERR_CUDA; \
  } while (0)

  // the column sums of E depend on E alone: a second stream computes them while
  // the prep kernels run, and the column-sum kernel of H_c waits for it
  // (the fixed-scratch entry keeps to one stream: it runs them in order)
  const bool ph_prep = (o.phases & kPhasePrep) != 0, ph_passes = (o.phases & kPhasePasses) != 0,
             ph_finish = (o.phases & kPhaseFinish) != 0;
  if (!bf16 && o.phases != (kPhasePrep | kPhasePasses | kPhaseFinish)) return CUTBCE_ERR_UNSUPPORTED;
  SideStreamLease side;
  if (bf16 && w.loss && ph_finish) {
    cudaStream_t cs = st;
    if (!o.one_stream && ph_prep) {
      if ((s = take_side_stream(side.s)) != CUTBCE_OK) return s;
      side.held = true;
      CUTBCE_CK(cudaEventRecord(side.s.ev, st));
      CUTBCE_CK(cudaStreamWaitEvent(side.s.s, side.s.ev, 0));
      cs = side.s.s;
    }
    LaunchScope ls(CUTBCE_KERNEL_COL_SUMS, cs);
    k_col_sums<<<static_cast<unsigned>(pl.csum_nbE), kColSumThreads, 0, cs>>>(
        static_cast<const __nv_bfloat16*>(p->E), V, nullptr, nullptr, pl.Tpad, D, pl.DP, pl.csum_nbE, pl.csum_nbH,
        at<double>(ws, pl.o_csum), hdr, 0, 0);
    CUTBCE_CK(cudaGetLastError());
    if (side.held) CUTBCE_CK(cudaEventRecord(side.s.ev2, side.s.s));
  }
  if (ph_prep) {
    CUTBCE_CK(cudaMemsetAsync(hdr, 0, 256, st));
    {
      LaunchScope ls(CUTBCE_KERNEL_PREP_ROWS, st);
      k_prep_rows<<<static_cast<unsigned>(ceil_div(T, 128)), 128, 0, st>>>(p->targets, p->mask, o.weights, T, K, V,
                                                                            o.v_off, o.V_total, ids, rowcnt, hdr);
      CUTBCE_CK(cudaGetLastError());
    }
    {
      LaunchScope ls(CUTBCE_KERNEL_PREP_SCAN, st);
      k_prep_scan<<<1, kScanThreads, 0, st>>>(p->mask, o.weights, rowcnt, T, o.V_total, p->reduction, grad_loss,
                                              cidx, orig, rowptr, hdr);
      CUTBCE_CK(cudaGetLastError());
    }
  }
  // the gather: the rows and pairs with the prep, the sparse correction (which
  // reads E) with the finish; one launch when the call has both
  auto gather = [&](int mode) -> cudaError_t {
    LaunchScope ls(CUTBCE_KERNEL_PREP_GATHER, st);
    if (bf16) {
      k_prep_gather<__nv_bfloat16><<<static_cast<unsigned>(pl.n_gather_blocks), 256, 0, st>>>(
          static_cast<const __nv_bfloat16*>(p->H), static_cast<const __nv_bfloat16*>(p->E), D, pl.DP, K, pl.Tpad,
          orig, ids, rowcnt, rowptr, hdr, o.weights, wc, at<__nv_bfloat16>(ws, pl.o_hc), pair_t, pair_v, cpart, mode);
    } else {
      k_prep_gather<float><<<static_cast<unsigned>(pl.n_gather_blocks), 256, 0, st>>>(
          static_cast<const float*>(p->H), static_cast<const float*>(p->E), D, pl.DP, K, pl.Tpad, orig, ids, rowcnt,
          rowptr, hdr, o.weights, wc, at<float>(ws, pl.o_hc), pair_t, pair_v, cpart, mode);
    }
    return cudaGetLastError();
  };
  if (ph_prep) CUTBCE_CK(gather(kGatherRows | (ph_finish ? kGatherCorrection : 0)));
  else if (ph_finish) CUTBCE_CK(gather(kGatherCorrection));

  // With per-position weights the tensor-core path sums the loss in the
  // position-owned pass (one weight per row there); the item-owned pass then
  // computes dE only.  The fp32 path sums it per item with the column weights.
  if (bf16 && w.loss && ph_finish) {
    if (side.held) CUTBCE_CK(cudaStreamWaitEvent(st, side.s.ev2, 0));
    LaunchScope ls(CUTBCE_KERNEL_COL_SUMS, st);
    k_col_sums<<<static_cast<unsigned>(pl.csum_nbH), kColSumThreads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(p->E), V, at<__nv_bfloat16>(ws, pl.o_hc), wc, pl.Tpad, D, pl.DP,
        pl.csum_nbE, pl.csum_nbH, at<double>(ws, pl.o_csum), hdr, pl.csum_nbE, 1);
    CUTBCE_CK(cudaGetLastError());
  }

  const bool loss_in_pos = bf16 && weighted && w.loss;
  const bool item_loss = w.loss && !loss_in_pos;
  const bool item_pass = item_loss || w.dE;
  const bool pos_pass = w.dH || w.met || loss_in_pos;
  if (bf16) {
    const int* srt_key = pair_v;
    const int* srt_val = pair_t;
    if (w.dE && !ph_prep) {
      // ordered by an earlier part of the call: the last radix pass's output
      srt_val = at<int>(ws, pl.o_srt[2 * ((pl.radix_passes - 1) & 1) + 1]);
    }
    if (w.dE && ph_prep) {
      // pairs grouped by item tile, ascending position inside a group: stable LSD
      // radix sort of (item tile, packed row/position) starting from (position, item) order
      LaunchScope ls(CUTBCE_KERNEL_PAIR_SORT, st);
      int* k0 = at<int>(ws, pl.o_srt[2]);
      int* v0 = at<int>(ws, pl.o_srt[3]);
      const int64_t TK = static_cast<int64_t>(T) * K;
      k_pair_keys<<<static_cast<unsigned>(std::max<int64_t>(1, ceil_div(TK, 256))), 256, 0, st>>>(pair_v, pair_t,
                                                                                                   hdr, k0, v0);
      srt_key = k0;
      srt_val = v0;
      for (int pass = 0; pass < pl.radix_passes; ++pass) {
        int* out_k = at<int>(ws, pl.o_srt[2 * (pass & 1)]);
        int* out_v = at<int>(ws, pl.o_srt[2 * (pass & 1) + 1]);
        k_radix_hist<<<pl.radix_blocks, kRadixThreads, 0, st>>>(srt_key, hdr, 8 * pass, pl.radix_blocks, ghist);
        k_exclusive_scan<<<1, 1024, 0, st>>>(ghist, 256 * pl.radix_blocks);
        k_radix_scatter<<<pl.radix_blocks, kRadixThreads, 0, st>>>(srt_key, srt_val, out_k, out_v, hdr, 8 * pass,
                                                                   pl.radix_blocks, ghist);
        srt_key = out_k;
        srt_val = out_v;
      }
      CUTBCE_CK(cudaGetLastError());
    }
    if (w.dE && ph_prep) {
      LaunchScope ls(CUTBCE_KERNEL_CSC_OFFSETS, st);
      const int nkeys = static_cast<int>(pl.n_vitems);
      k_key_offsets<<<static_cast<unsigned>(ceil_div(nkeys + 1, 256)), 256, 0, st>>>(srt_key, hdr, nkeys, cscoff);
      CUTBCE_CK(cudaGetLastError());
    }
    TileParams tp{};
    tp.V = V;
    tp.D = D;
    tp.Tpad = pl.Tpad;
    tp.hdr = hdr;
    tp.row_ptr = rowptr;
    tp.pair_v = pair_v;
    tp.tile_pair_off = cscoff;
    tp.tile_pairs = srt_val;
    tp.dE = static_cast<float*>(dE);
    tp.de_bf16 = o.grad_bf16 ? 1 : 0;
    tp.de_acc = o.acc_dE ? 1 : 0;
    tp.wc = wc;
    tp.loss_part = lpart;
    tp.dh_part = dhpart;
    tp.met_part = metpart;
    tp.nsplit = pl.S;
    tp.tiles_per_split = pl.tps;
    tp.n_item_tiles_bn = pl.n_vtiles_bn;
    tp.timeout_ns = kDefaultTimeoutNs;
    tp.range_begin = o.tile_begin;
    tp.range_end = o.tile_end;
    const __nv_bfloat16* hc = at<__nv_bfloat16>(ws, pl.o_hc);
    const int64_t tiles_in_range =
        std::max<int64_t>(0, std::min<int64_t>(o.tile_end, pl.n_vitems) - std::min<int64_t>(o.tile_begin, pl.n_vitems));
    const int64_t splits_in_range =
        std::max<int64_t>(0, std::min<int64_t>(o.split_end, pl.S) - std::min<int64_t>(o.split_begin, pl.S));
    if (ph_passes && item_pass && tiles_in_range > 0) {
      CUtensorMap ms, mx;
      if (!make_map(&ms, p->E, D, V, D, kTileM) || !make_map(&mx, hc, pl.DP, pl.Tpad, pl.DP, pl.BN))
        return CUTBCE_ERR_CUDA;
      const int grid = static_cast<int>(std::min<int64_t>({static_cast<int64_t>(dev.sms), tiles_in_range,
                                                           static_cast<int64_t>(kMaxCtas)}));
      cudaError_t e;
      LaunchScope ls(CUTBCE_KERNEL_ITEM_PASS, st);
      if (item_loss && w.dE) e = launch_tile_dp<true, true, false>(pl.DP, grid, ms, mx, tp, st);
      else if (item_loss) e = launch_tile_dp<true, false, false>(pl.DP, grid, ms, mx, tp, st);
      else e = launch_tile_dp<false, true, false>(pl.DP, grid, ms, mx, tp, st);
      CUTBCE_CK(e);
    }
    if (ph_passes && item_pass && after_item != nullptr) CUTBCE_CK(cudaEventRecord(after_item, st));
    tp.range_begin = o.split_begin;
    tp.range_end = o.split_end;
    if (ph_passes && pos_pass && splits_in_range > 0) {
      CUtensorMap ms, mx;
      if (!make_map(&ms, hc, pl.DP, pl.Tpad, pl.DP, kTileM) || !make_map(&mx, p->E, D, V, D, pl.BN))
        return CUTBCE_ERR_CUDA;
      const int64_t items_max = splits_in_range * ceil_div(T, kTileM);
      const int grid = static_cast<int>(
          std::min<int64_t>({static_cast<int64_t>(dev.sms), items_max, static_cast<int64_t>(kMaxCtas)}));
      LaunchScope ls(CUTBCE_KERNEL_POSITION_PASS, st);
      const int kind = (loss_in_pos ? 4 : 0) | (w.dH ? 2 : 0) | (w.met ? 1 : 0);
      cudaError_t e;
      switch (kind) {
        case 1: e = launch_tile_dp<false, false, true, true>(pl.DP, grid, ms, mx, tp, st); break;
        case 2: e = launch_tile_dp<false, true, true, false>(pl.DP, grid, ms, mx, tp, st); break;
        case 3: e = launch_tile_dp<false, true, true, true>(pl.DP, grid, ms, mx, tp, st); break;
        case 4: e = launch_tile_dp<true, false, true, false>(pl.DP, grid, ms, mx, tp, st); break;
        case 5: e = launch_tile_dp<true, false, true, true>(pl.DP, grid, ms, mx, tp, st); break;
        case 6: e = launch_tile_dp<true, true, true, false>(pl.DP, grid, ms, mx, tp, st); break;
        default: e = launch_tile_dp<true, true, true, true>(pl.DP, grid, ms, mx, tp, st); break;
      }
      CUTBCE_CK(e);
    }
  } else {
    const float* hc = at<float>(ws, pl.o_hc);
    if (item_pass) {
      LaunchScope ls(CUTBCE_KERNEL_ITEM_PASS, st);
      k_simt_items<<<dim3(static_cast<unsigned>(pl.n_vitems), static_cast<unsigned>(ceil_div(D, 32))), 128, 0, st>>>(
          hc, static_cast<const float*>(p->E), V, D, rowptr, pair_v, hdr, wc, w.dE ? dE : nullptr,
          o.grad_bf16 ? 1 : 0, o.acc_dE ? 1 : 0, w.loss ? lpart : nullptr);
      CUTBCE_CK(cudaGetLastError());
    }
    if (item_pass && after_item != nullptr) CUTBCE_CK(cudaEventRecord(after_item, st));
    if (w.dH || w.met) {
      LaunchScope ls(CUTBCE_KERNEL_POSITION_PASS, st);
      k_simt_rows<<<dim3(static_cast<unsigned>(ceil_div(pl.Tpad, 128)), static_cast<unsigned>(ceil_div(D, 32))), 128, 0,
                    st>>>(
          hc, static_cast<const float*>(p->E), V, D, rowptr, pair_v, hdr, w.dH ? dhpart : nullptr, metpart);
      CUTBCE_CK(cudaGetLastError());
    }
  }
  if (ph_finish && (w.loss || w.dH || w.met)) {
    const unsigned grid = static_cast<unsigned>(finish_grid(T, D));
    FinishParams fp{};
    fp.T = T;
    fp.D = D;
    fp.DP = pl.DP;
    fp.S = pl.S;
    fp.V = V;
    fp.Tpad = pl.Tpad;
    fp.cidx = cidx;
    fp.dh_part = dhpart;
    fp.dH = w.dH ? dH : nullptr;
    fp.dh_bf16 = o.grad_bf16 ? 1 : 0;
    fp.dh_acc = o.acc_dH ? 1 : 0;
    fp.weights = o.weights;
    fp.loss_part = lpart;
    fp.n_loss_part = static_cast<int>(pl.n_vitems * kNumEpiWarps);
    fp.loss_pos_splits = loss_in_pos ? pl.S : 0;
    fp.corr_part = cpart;
    fp.n_corr_part = static_cast<int>(pl.n_gather_blocks);
    fp.blk_part = at<double>(ws, pl.o_fpart);
    fp.loss = w.loss ? loss : nullptr;
    fp.met_part = metpart;
    fp.met_slots = pl.met_slots;
    fp.metrics = w.met ? o.metrics : nullptr;
    fp.row_cnt = rowcnt;
    fp.use_lin = (bf16 && w.loss) ? 1 : 0;
    fp.hdr = hdr;
    LaunchScope ls(CUTBCE_KERNEL_FINISH, st);
    k_finish<<<grid, kFinishThreads, 0, st>>>(fp);
    CUTBCE_CK(cudaGetLastError());
  }
#undef CUTBCE_CK
  return CUTBCE_OK;
}

// Host-buffer entry: layout of the caller's device buffer.
struct HostLayout {
  size_t o_H, o_E, o_tg, o_mask, o_loss, o_grad, o_dH, o_dE, o_ws, total;
};

// The host-buffer entry runs a large item table in up to kMaxHostShards
// vocabulary shards (whole splits of the position-owned pass, on whole 128-item
// tiles), so that copying shard s + 1 in and shard s - 1's dE out overlap the
// computation of shard s.
constexpr int kMaxHostShards = 4;
constexpr int64_t kHostShardBytes = int64_t(32) << 20;

int host_shards(const cutbce_problem* p) {
  if (p->dtype != CUTBCE_BF16) return 1;
  int64_t n = ceil_div(2 * p->V * p->D, kHostShardBytes);
  n = std::min<int64_t>({n, static_cast<int64_t>(kMaxHostShards), ceil_div(p->V, kTileM)});
  return static_cast<int>(std::max<int64_t>(1, n));
}

// Shard k of n in vocabulary splits of the position-owned pass: splits
// [s0, s1), which cover the items [v0, v1) and, since the boundaries fall on
// whole 128-item tiles, the item tiles [v0 / 128, ceil(v1 / 128)).
void host_shard_splits(const Plan& pl, int n, int k, int& s0, int& s1, int64_t& v0, int64_t& v1) {
  static const int kCum[kMaxHostShards + 1][kMaxHostShards + 1] = {
      {0, 0, 0, 0, 0}, {0, 20, 0, 0, 0}, {0, 10, 20, 0, 0}, {0, 5, 15, 20, 0}, {0, 3, 10, 17, 20}};
  const int64_t rows_per_split = static_cast<int64_t>(pl.tps) * pl.BN;
  s0 = static_cast<int>(int64_t(pl.S) * kCum[n][k] / 20);
  s1 = static_cast<int>(int64_t(pl.S) * kCum[n][k + 1] / 20);
  if (rows_per_split % kTileM != 0) {   // 64-row splits of odd length: boundaries at even splits
    s0 &= ~1;
    s1 &= ~1;
  }
  if (k + 1 == n) s1 = pl.S;
  v0 = std::min<int64_t>(pl.V, s0 * rows_per_split);
  v1 = k + 1 == n ? pl.V : std::min<int64_t>(pl.V, s1 * rows_per_split);
}

void host_layout(const cutbce_problem* p, const Plan& pl, HostLayout& hl) {
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t a = o;
    o = align256(o + bytes);
    return a;
  };
  hl.o_H = take(pl.elem * p->T * p->D);
  hl.o_E = take(pl.elem * p->V * p->D);
  hl.o_tg = take(4 * p->T * p->K);
  hl.o_mask = take(p->T);
  hl.o_loss = take(8);
  hl.o_grad = take(4);
  hl.o_dH = take(4 * p->T * p->D);
  hl.o_dE = take(4 * p->V * p->D);
  hl.o_ws = take(pl.total);
  hl.total = o;
}

// ---------------------------------------------------------------- fixed scratch
// Scratch of cutbce_forward_fixed_scratch: a static device array of the
// library's own module, so that entry needs no caller workspace and allocates
// nothing.  Every call on a device uses the same array: calls on one device
// must not overlap in time (see the header).
constexpr size_t kFixedScratchBytes = CUTBCE_FIXED_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_fixed_scratch[kFixedScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_fixed_mutex;
void* g_fixed_ptr[kMaxDevices] = {};

// Device address of g_fixed_scratch on the current device, looked up once per
// device (with that device current) and cached.
cutbce_status fixed_scratch_ptr(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CUTBCE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_fixed_mutex);
  if (g_fixed_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_fixed_scratch) != cudaSuccess || ptr == nullptr) return CUTBCE_ERR_CUDA;
    g_fixed_ptr[dev] = ptr;
  }
  *out = g_fixed_ptr[dev];
  return CUTBCE_OK;
}

}  // namespace

extern "C" {

cutbce_status cutbce_workspace_size(const cutbce_problem* prob, size_t* bytes) {
  return cutbce_workspace_size_for(prob, CUTBCE_OUT_LOSS | CUTBCE_OUT_DH | CUTBCE_OUT_DE, bytes);
}

cutbce_status cutbce_workspace_size_for(const cutbce_problem* prob, int outputs, size_t* bytes) {
  if (bytes == nullptr || outputs <= 0 || outputs > kAllOutputs) return CUTBCE_ERR_INVALID_ARG;
  const cutbce_status s = check_problem(prob, false);
  if (s != CUTBCE_OK) return s;
  Plan pl;
  make_plan(prob, want_from_mask(outputs), pl);
  *bytes = pl.total;
  return CUTBCE_OK;
}

cutbce_status cutbce_forward(const cutbce_problem* prob, void* ws, size_t ws_bytes, double* loss,
                             cutbce_stream_t stream) {
  if (loss == nullptr) return CUTBCE_ERR_INVALID_ARG;
  return run(prob, nullptr, loss, nullptr, nullptr, Want{true, false, false, false}, ws, ws_bytes,
             reinterpret_cast<cudaStream_t>(stream));
}

cutbce_status cutbce_forward_fixed_scratch(const cutbce_problem* prob, double* loss, cutbce_stream_t stream) {
  if (loss == nullptr) return CUTBCE_ERR_INVALID_ARG;
  cutbce_status s = check_problem(prob, true);
  if (s != CUTBCE_OK) return s;
  Plan pl;
  make_plan(prob, Want{true, false, false, false}, pl);                   // the loss-only layout that run() uses
  if (pl.total > kFixedScratchBytes) return CUTBCE_ERR_WORKSPACE;   // the problem needs more than the fixed array
  void* ws = nullptr;
  if ((s = fixed_scratch_ptr(&ws)) != CUTBCE_OK) return s;
  Opts o{};
  o.one_stream = true;                                              // creates no stream or event either
  return run(prob, nullptr, loss, nullptr, nullptr, Want{true, false, false, false}, ws, kFixedScratchBytes,
             reinterpret_cast<cudaStream_t>(stream), nullptr, o);
}

cutbce_status cutbce_backward(const cutbce_problem* prob, const float* grad_loss, float* dH, float* dE, void* ws,
                              size_t ws_bytes, cutbce_stream_t stream) {
  if (dH == nullptr && dE == nullptr) return CUTBCE_ERR_INVALID_ARG;
  return run(prob, grad_loss, nullptr, dH, dE, Want{false, dE != nullptr, dH != nullptr, false}, ws, ws_bytes,
             reinterpret_cast<cudaStream_t>(stream));
}

cutbce_status cutbce_forward_backward(const cutbce_problem* prob, const float* grad_loss, double* loss, float* dH,
                                      float* dE, void* ws, size_t ws_bytes, cutbce_stream_t stream) {
  if (loss == nullptr && dH == nullptr && dE == nullptr) return CUTBCE_ERR_INVALID_ARG;
  return run(prob, grad_loss, loss, dH, dE, Want{loss != nullptr, dE != nullptr, dH != nullptr, false}, ws, ws_bytes,
             reinterpret_cast<cudaStream_t>(stream));
}

cutbce_status cutbce_forward_backward_ex(const cutbce_problem* prob, const cutbce_options* opts,
                                         const float* grad_loss, double* loss, void* dH, void* dE, void* ws,
                                         size_t ws_bytes, cutbce_stream_t stream) {
  cutbce_status s = check_problem(prob, false);
  if (s != CUTBCE_OK) return s;
  Opts o;
  if ((s = resolve_opts(prob, opts, o)) != CUTBCE_OK) return s;
  if (loss == nullptr && dH == nullptr && dE == nullptr && o.metrics == nullptr) return CUTBCE_ERR_INVALID_ARG;
  return run(prob, grad_loss, loss, dH, dE, Want{loss != nullptr, dE != nullptr, dH != nullptr, o.metrics != nullptr},
             ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream), nullptr, o);
}

cutbce_status cutbce_workspace_size_ex(const cutbce_problem* prob, const cutbce_options* opts, int outputs,
                                       size_t* bytes) {
  if (bytes == nullptr || outputs <= 0 || outputs > kAllOutputs) return CUTBCE_ERR_INVALID_ARG;
  cutbce_status s = check_problem(prob, false);
  if (s != CUTBCE_OK) return s;
  Opts o;
  if ((s = resolve_opts(prob, opts, o)) != CUTBCE_OK) return s;
  Plan pl;
  make_plan(prob, want_from_mask(outputs), pl, o.weights != nullptr);
  *bytes = pl.total;
  return CUTBCE_OK;
}

cutbce_status cutbce_host_buffer_size(const cutbce_problem* prob, size_t* bytes) {
  if (bytes == nullptr) return CUTBCE_ERR_INVALID_ARG;
  const cutbce_status s = check_problem(prob, false);
  if (s != CUTBCE_OK) return s;
  Plan pl;
  make_plan(prob, kWantAll, pl);
  HostLayout hl;
  host_layout(prob, pl, hl);
  *bytes = hl.total;
  return CUTBCE_OK;
}

cutbce_status cutbce_forward_backward_host(const cutbce_problem* prob, float grad_loss, double* loss, float* dH,
                                           float* dE, void* dev_buf, size_t dev_bytes, cutbce_stream_t stream) {
  cutbce_status s = check_problem(prob, true);
  if (s != CUTBCE_OK) return s;
  if (loss == nullptr || dev_buf == nullptr || (reinterpret_cast<uintptr_t>(dev_buf) & 255) != 0)
    return CUTBCE_ERR_INVALID_ARG;
  Plan pl;
  make_plan(prob, kWantAll, pl);     // the largest layout: the buffer size query covers every set of outputs
  HostLayout hl;
  host_layout(prob, pl, hl);
  if (dev_bytes < hl.total) return CUTBCE_ERR_WORKSPACE;
  const Want w{true, dE != nullptr, dH != nullptr, false};
  Plan plw;
  make_plan(prob, w, plw);           // the plan of the call's parts (splits, tile sizes, header offset)
  int nsh = host_shards(prob);
  nsh = std::min(nsh, std::max(1, plw.S / 2));
  // Streams (per-device pool, created on first use): E's shards are copied in on
  // `cin`, the computation runs on `st`, and each shard's dE is copied out on
  // `cout` as soon as its item-owned pass ends (dE is final then), while the
  // dH pass and the next shard run on `st`.
  //
  // With more than one shard the call runs in parts on one workspace: the prep
  // and the pair order once (they read no E), then each shard's two tile
  // passes as soon as its rows of E are in, over the item tiles and the
  // vocabulary splits it covers, then the sparse correction, the column sums
  // and the finish once.  Every tile and split is computed exactly as by the
  // one-call path and the partials are summed by the same finish, so the
  // results are the same bits.
  SideStreamLease cin, cout;
  if (nsh > 1) {
    if ((s = take_side_stream(cin.s)) != CUTBCE_OK) return s;
    cin.held = true;
  }
  if (dE != nullptr) {
    if ((s = take_side_stream(cout.s)) != CUTBCE_OK) return s;
    cout.held = true;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaStream_t in = nsh > 1 ? cin.s.s : st;
  uint8_t* b = static_cast<uint8_t*>(dev_buf);
  const size_t rowE = pl.elem * prob->D;
  bool ok = cudaMemcpyAsync(b + hl.o_H, prob->H, pl.elem * prob->T * prob->D, cudaMemcpyHostToDevice, st) ==
                cudaSuccess &&
            cudaMemcpyAsync(b + hl.o_tg, prob->targets, 4 * prob->T * prob->K, cudaMemcpyHostToDevice, st) ==
                cudaSuccess &&
            (prob->mask == nullptr ||
             cudaMemcpyAsync(b + hl.o_mask, prob->mask, prob->T, cudaMemcpyHostToDevice, st) == cudaSuccess) &&
            cudaMemcpyAsync(b + hl.o_grad, &grad_loss, 4, cudaMemcpyHostToDevice, st) == cudaSuccess;
  cutbce_problem dp = *prob;
  dp.H = b + hl.o_H;
  dp.E = b + hl.o_E;
  dp.targets = reinterpret_cast<const int32_t*>(b + hl.o_tg);
  dp.mask = prob->mask != nullptr ? reinterpret_cast<const uint8_t*>(b + hl.o_mask) : nullptr;
  float* ddH = dH ? reinterpret_cast<float*>(b + hl.o_dH) : nullptr;
  float* ddE = dE ? reinterpret_cast<float*>(b + hl.o_dE) : nullptr;
  double* dloss = reinterpret_cast<double*>(b + hl.o_loss);
  const float* dgrad = reinterpret_cast<const float*>(b + hl.o_grad);
  void* dws = b + hl.o_ws;
  cudaEvent_t after_item = dE != nullptr ? cout.s.ev : nullptr;
  // the rows [v0, v1) of dE are final once the item-owned pass over them has run
  auto copy_dE_out = [&](int64_t v0, int64_t v1) {
    return dE == nullptr ||
           (cudaStreamWaitEvent(cout.s.s, cout.s.ev, 0) == cudaSuccess &&
            cudaMemcpyAsync(dE + v0 * prob->D, ddE + v0 * prob->D, 4 * (v1 - v0) * prob->D, cudaMemcpyDeviceToHost,
                            cout.s.s) == cudaSuccess);
  };
  if (ok && nsh == 1) {
    ok = cudaMemcpyAsync(b + hl.o_E, prob->E, prob->V * rowE, cudaMemcpyHostToDevice, st) == cudaSuccess;
    if (ok) s = run(&dp, dgrad, dloss, ddH, ddE, w, dws, pl.total, st, after_item);
    if (ok && s == CUTBCE_OK) ok = copy_dE_out(0, prob->V);
  } else if (ok) {
    Opts part{};
    part.phases = kPhasePrep;
    s = run(&dp, dgrad, dloss, ddH, ddE, w, dws, pl.total, st, nullptr, part);
    for (int k = 0; k < nsh && ok && s == CUTBCE_OK; ++k) {
      int s0 = 0, s1 = 0;
      int64_t v0 = 0, v1 = 0;
      host_shard_splits(plw, nsh, k, s0, s1, v0, v1);
      if (v1 <= v0) continue;               // an empty shard (few splits): nothing to copy or compute
      ok = cudaMemcpyAsync(b + hl.o_E + v0 * rowE, static_cast<const uint8_t*>(prob->E) + v0 * rowE,
                           (v1 - v0) * rowE, cudaMemcpyHostToDevice, in) == cudaSuccess &&
           cudaEventRecord(cin.s.ev, in) == cudaSuccess && cudaStreamWaitEvent(st, cin.s.ev, 0) == cudaSuccess;
      if (!ok) break;
      part = Opts{};
      part.phases = kPhasePasses;
      part.tile_begin = static_cast<int>(v0 / kTileM);
      part.tile_end = static_cast<int>(ceil_div(v1, kTileM));
      part.split_begin = s0;
      part.split_end = s1;
      s = run(&dp, dgrad, dloss, ddH, ddE, w, dws, pl.total, st, after_item, part);
      if (s == CUTBCE_OK) ok = copy_dE_out(v0, v1);
    }
    if (ok && s == CUTBCE_OK) {
      part = Opts{};
      part.phases = kPhaseFinish;
      s = run(&dp, dgrad, dloss, ddH, ddE, w, dws, pl.total, st, nullptr, part);
    }
  }
  double loss_h = 0.0;
  int32_t status_h = 0;
  if (ok && s == CUTBCE_OK)
    ok = cudaMemcpyAsync(&loss_h, dloss, 8, cudaMemcpyDeviceToHost, st) == cudaSuccess &&
         (!dH || cudaMemcpyAsync(dH, ddH, 4 * prob->T * prob->D, cudaMemcpyDeviceToHost, st) == cudaSuccess) &&
         cudaMemcpyAsync(&status_h, b + hl.o_ws + plw.o_hdr, 4, cudaMemcpyDeviceToHost, st) == cudaSuccess;
  // every stream is drained before returning, also after an error: no copy from
  // or to the caller's host memory may still run on return
  bool sync_ok = cudaStreamSynchronize(st) == cudaSuccess;
  if (nsh > 1) sync_ok = cudaStreamSynchronize(cin.s.s) == cudaSuccess && sync_ok;
  if (dE != nullptr) sync_ok = cudaStreamSynchronize(cout.s.s) == cudaSuccess && sync_ok;
  if (s != CUTBCE_OK) return s;
  if (!ok || !sync_ok) return CUTBCE_ERR_CUDA;
  *loss = loss_h;
  return status_h != 0 ? static_cast<cutbce_status>(status_h) : CUTBCE_OK;
}

cutbce_status cutbce_topk_workspace_size(int64_t B, int64_t V, int64_t D, int k, size_t* bytes) {
  if (bytes == nullptr) return CUTBCE_ERR_INVALID_ARG;
  TopkPlan tp;
  const cutbce_status s = topk_plan(B, V, D, k, 148, tp);
  if (s != CUTBCE_OK) return s;
  *bytes = tp.total;
  return CUTBCE_OK;
}

cutbce_status cutbce_topk(const void* Q, int64_t B, const void* E, int64_t V, int64_t D, int32_t dtype, int k,
                          int32_t* ids, float* scores, void* ws, size_t ws_bytes, cutbce_stream_t stream) {
  if (Q == nullptr || E == nullptr || ids == nullptr || scores == nullptr || ws == nullptr) return CUTBCE_ERR_INVALID_ARG;
  if (dtype != CUTBCE_BF16) return CUTBCE_ERR_UNSUPPORTED;
  if (((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(E)) & 15) != 0 ||
      (reinterpret_cast<uintptr_t>(ws) & 255) != 0)
    return CUTBCE_ERR_INVALID_ARG;
  DeviceFacts dev;
  cutbce_status s = device_facts(dev);
  if (s != CUTBCE_OK) return s;
  TopkPlan pl;
  if ((s = topk_plan(B, V, D, k, dev.sms, pl)) != CUTBCE_OK) return s;
  if (ws_bytes < pl.total) return CUTBCE_ERR_WORKSPACE;
  if (!(dev.major == 10 && dev.minor == 0)) return CUTBCE_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  CUtensorMap mq, me;
  if (!make_map(&mq, Q, D, B, D, kTileM) || !make_map(&me, E, D, V, D, pl.BN)) return CUTBCE_ERR_CUDA;
  TopkParams tp{};
  tp.B = static_cast<int>(B);
  tp.V = static_cast<int>(V);
  tp.n_qt = pl.n_qt;
  tp.nsplit = pl.S;
  tp.tiles_per_split = pl.tps;
  tp.n_vtiles = pl.n_vtiles;
  tp.cand_s = at<float>(ws, pl.o_s);
  tp.cand_i = at<int>(ws, pl.o_i);
  tp.hdr = at<WsHeader>(ws, pl.o_hdr);
  tp.timeout_ns = kDefaultTimeoutNs;
  if (cudaMemsetAsync(tp.hdr, 0, 256, st) != cudaSuccess) return CUTBCE_ERR_CUDA;
  const int grid = static_cast<int>(std::min<int64_t>({static_cast<int64_t>(dev.sms),
                                                       static_cast<int64_t>(pl.n_qt) * pl.S, kMaxCtas}));
  cudaError_t e;
  {
    LaunchScope ls(CUTBCE_KERNEL_TOPK, st);
    e = pl.KMAX == 8 ? launch_topk_dp<8>(pl.DP, grid, mq, me, tp, st)
                     : launch_topk_dp<16>(pl.DP, grid, mq, me, tp, st);
  }
  if (e != cudaSuccess) return CUTBCE_ERR_CUDA;
  const unsigned mgrid = static_cast<unsigned>(ceil_div(B * 32, 256));
  {
    LaunchScope ls(CUTBCE_KERNEL_TOPK_MERGE, st);
    // many lists per query (more than 64): a block per query, else a warp per query
    const bool per_block = pl.S * 4 > 64;
    if (pl.KMAX == 8) {
      if (per_block) k_topk_merge_block<8><<<static_cast<unsigned>(B), 256, 0, st>>>(tp.cand_s, tp.cand_i, tp.B, pl.S, k, ids, scores);
      else k_topk_merge<8><<<mgrid, 256, 0, st>>>(tp.cand_s, tp.cand_i, tp.B, pl.S, k, ids, scores);
    } else {
      if (per_block) k_topk_merge_block<16><<<static_cast<unsigned>(B), 256, 0, st>>>(tp.cand_s, tp.cand_i, tp.B, pl.S, k, ids, scores);
      else k_topk_merge<16><<<mgrid, 256, 0, st>>>(tp.cand_s, tp.cand_i, tp.B, pl.S, k, ids, scores);
    }
  }
  return cudaGetLastError() == cudaSuccess ? CUTBCE_OK : CUTBCE_ERR_CUDA;
}

cutbce_status cutbce_hit_at_k(const int32_t* ids, int64_t B, int k, const int32_t* targets, int64_t L, int32_t* hits,
                              cutbce_stream_t stream) {
  if (ids == nullptr || targets == nullptr || hits == nullptr || B <= 0 || k <= 0 || L <= 0)
    return CUTBCE_ERR_INVALID_ARG;
  if (B >= (int64_t(1) << 31) || L >= (int64_t(1) << 20) || k > 16) return CUTBCE_ERR_UNSUPPORTED;
  k_hit_at_k<<<static_cast<unsigned>(ceil_div(B, 256)), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      ids, static_cast<int>(B), k, targets, static_cast<int>(L), hits);
  return cudaGetLastError() == cudaSuccess ? CUTBCE_OK : CUTBCE_ERR_CUDA;
}

cutbce_status cutbce_read_status(const void* ws, cutbce_stream_t stream) {
  if (ws == nullptr) return CUTBCE_ERR_INVALID_ARG;
  int v = 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess)
    return CUTBCE_ERR_CUDA;
  return static_cast<cutbce_status>(v);
}

cutbce_status cutbce_read_counts(const cutbce_problem* prob, const void* ws, int64_t* n_valid, int64_t* n_pairs,
                                 int32_t* row_counts, cutbce_stream_t stream) {
  const cutbce_status s = check_problem(prob, false);
  if (s != CUTBCE_OK) return s;
  if (ws == nullptr || n_valid == nullptr || n_pairs == nullptr) return CUTBCE_ERR_INVALID_ARG;
  Plan pl;
  make_plan(prob, kWantAll, pl);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  WsHeader h;
  const uint8_t* b = static_cast<const uint8_t*>(ws);
  if (cudaMemcpyAsync(&h, b + pl.o_hdr, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess) return CUTBCE_ERR_CUDA;
  if (row_counts != nullptr &&
      cudaMemcpyAsync(row_counts, b + pl.o_rowcnt, 4 * prob->T, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return CUTBCE_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return CUTBCE_ERR_CUDA;
  *n_valid = h.n_valid;
  *n_pairs = h.n_pairs;
  return CUTBCE_OK;
}

int cutbce_kernel_launches(const cutbce_problem* prob, int entry) {
  if (check_problem(prob, false) != CUTBCE_OK || entry < 0 || entry > 2) return -1;
  Plan pl;
  make_plan(prob, kWantAll, pl);
  const Want w = entry == 0 ? Want{true, false, false, false}
                 : entry == 1 ? Want{false, true, true, false} : Want{true, true, true, false};
  return count_launches(pl, w);
}

cutbce_status cutbce_profile_enable(int enable) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  g_prof.enabled = enable != 0;
  return CUTBCE_OK;
}

cutbce_status cutbce_profile_read(double* ms, int64_t* launches, int reset) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  g_prof.drain();
  for (int k = 0; k < CUTBCE_NUM_KERNEL_KINDS; ++k) {
    if (ms) ms[k] = g_prof.ms[k];
    if (launches) launches[k] = g_prof.launches[k];
    if (reset) {
      g_prof.ms[k] = 0.0;
      g_prof.launches[k] = 0;
    }
  }
  return CUTBCE_OK;
}

size_t cutbce_probe_scratch_bytes(void) { return 16 * kMaxCtas + 4 * kProbeThreads; }

cutbce_status cutbce_probe_pipe_rate(int op, void* scratch, size_t scratch_bytes, double* ops_per_clock_per_sm,
                                     cutbce_stream_t stream) {
  if (op < 0 || op >= kProbeCount || scratch == nullptr || ops_per_clock_per_sm == nullptr ||
      scratch_bytes < cutbce_probe_scratch_bytes())
    return CUTBCE_ERR_INVALID_ARG;
  DeviceFacts dev;
  cutbce_status s = device_facts(dev);
  if (s != CUTBCE_OK) return s;
  const int grid = std::min(dev.sms, kMaxCtas);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto* cycles = static_cast<unsigned long long*>(scratch);
  float* sink = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + 16 * kMaxCtas);
  constexpr int kIters = 2048;
  constexpr int kSmem = 120 * 1024;   // more than half of an SM's shared memory: one CTA per SM
  cudaError_t e = cudaSuccess;
  auto launch = [&](auto kern) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e == cudaSuccess) {
      kern<<<grid, kProbeThreads, kSmem, st>>>(kIters, cycles, sink);
      e = cudaGetLastError();
    }
  };
  switch (op) {
    case kProbeFfma: launch(k_probe<kProbeFfma>); break;
    case kProbeFfma2: launch(k_probe<kProbeFfma2>); break;
    case kProbeEx2: launch(k_probe<kProbeEx2>); break;
    case kProbeRcp: launch(k_probe<kProbeRcp>); break;
    case kProbeTanh: launch(k_probe<kProbeTanh>); break;
    case kProbeLg2: launch(k_probe<kProbeLg2>); break;
    case kProbeCvtBf16x2: launch(k_probe<kProbeCvtBf16x2>); break;
    case kProbeFmax: launch(k_probe<kProbeFmax>); break;
    case kProbeAdd2: launch(k_probe<kProbeAdd2>); break;
    case kProbeIadd: launch(k_probe<kProbeIadd>); break;
    case kProbePrmt: launch(k_probe<kProbePrmt>); break;
    case kProbeEx2F16x2: launch(k_probe<kProbeEx2F16x2>); break;
    case kProbeEx2Bf16x2: launch(k_probe<kProbeEx2Bf16x2>); break;
    case kProbeTanhF16x2: launch(k_probe<kProbeTanhF16x2>); break;
    case kProbeHfma2: launch(k_probe<kProbeHfma2>); break;
    case kProbeCvtF16x2: launch(k_probe<kProbeCvtF16x2>); break;
    case kProbeFfmaSat: launch(k_probe<kProbeFfmaSat>); break;
    case kProbeSelp: launch(k_probe<kProbeSelp>); break;
    case kProbeLop3: launch(k_probe<kProbeLop3>); break;
    default: launch(k_probe<kProbeFmul2>); break;
  }
  if (e != cudaSuccess) return CUTBCE_ERR_CUDA;
  std::vector<unsigned long long> h(grid);
  if (cudaMemcpyAsync(h.data(), cycles, 8 * grid, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return CUTBCE_ERR_CUDA;
  std::sort(h.begin(), h.end());
  const bool two = op == kProbeFfma2 || op == kProbeAdd2 || op == kProbeFmul2;   // fp32x2: two operations each
  const double ops = static_cast<double>(kProbeThreads) * kIters * kProbeChains * (two ? 2 : 1);
  *ops_per_clock_per_sm = h[grid / 2] > 0 ? ops / static_cast<double>(h[grid / 2]) : 0.0;
  return CUTBCE_OK;
}

cutbce_status cutbce_probe_mma(int n, int flags, int64_t iters, void* scratch, size_t scratch_bytes,
                               double* issue_cycles_per_mma, double* cycles_per_mma, cutbce_stream_t stream) {
  if ((n != 64 && n != 128 && n != 256) || iters <= 0 || iters > (1 << 24) || scratch == nullptr ||
      scratch_bytes < cutbce_probe_scratch_bytes() || issue_cycles_per_mma == nullptr || cycles_per_mma == nullptr)
    return CUTBCE_ERR_INVALID_ARG;
  DeviceFacts dev;
  cutbce_status s = device_facts(dev);
  if (s != CUTBCE_OK) return s;
  if (!(dev.major == 10 && dev.minor == 0)) return CUTBCE_ERR_UNSUPPORTED;
  const int grid = std::min(dev.sms, kMaxCtas) & ~1;   // even: whole 2-CTA clusters for the pair probe
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto* out = static_cast<unsigned long long*>(scratch);
  const int smem = 1024 + 16384 + n * 128 + 16 * 2048;
  const int smem_req = std::max(smem, 120 * 1024);   // one CTA per SM: TMEM allocation uncontended
  cudaError_t e = cudaSuccess;
  auto launch = [&](auto kern) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_req);
    if (e == cudaSuccess) {
      kern<<<grid, 128, smem_req, st>>>(static_cast<int>(iters), out);
      e = cudaGetLastError();
    }
  };
  const bool bmn = (flags & 2) != 0;
  const bool at = (flags & 1) != 0;
  const bool pair = (flags & 4) != 0;
  if (pair) {
    if (bmn) return CUTBCE_ERR_INVALID_ARG;
    if (n == 64) at ? launch(k_probe_mma_pair<64, true>) : launch(k_probe_mma_pair<64, false>);
    else if (n == 128) at ? launch(k_probe_mma_pair<128, true>) : launch(k_probe_mma_pair<128, false>);
    else at ? launch(k_probe_mma_pair<256, true>) : launch(k_probe_mma_pair<256, false>);
  } else if (n == 64) {
    if (bmn) at ? launch(k_probe_mma<64, true, true>) : launch(k_probe_mma<64, false, true>);
    else at ? launch(k_probe_mma<64, true, false>) : launch(k_probe_mma<64, false, false>);
  } else if (n == 128) {
    if (bmn) at ? launch(k_probe_mma<128, true, true>) : launch(k_probe_mma<128, false, true>);
    else at ? launch(k_probe_mma<128, true, false>) : launch(k_probe_mma<128, false, false>);
  } else {
    if (bmn) at ? launch(k_probe_mma<256, true, true>) : launch(k_probe_mma<256, false, true>);
    else at ? launch(k_probe_mma<256, true, false>) : launch(k_probe_mma<256, false, false>);
  }
  if (e != cudaSuccess) return CUTBCE_ERR_CUDA;
  std::vector<unsigned long long> h(2 * grid);
  if (cudaMemcpyAsync(h.data(), out, 16 * grid, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return CUTBCE_ERR_CUDA;
  // with SM pairs only the even CTA of each cluster issues and records
  std::vector<unsigned long long> issue, total;
  for (int b = 0; b < grid; b += pair ? 2 : 1) {
    issue.push_back(h[2 * b]);
    total.push_back(h[2 * b + 1]);
  }
  std::sort(issue.begin(), issue.end());
  std::sort(total.begin(), total.end());
  *issue_cycles_per_mma = static_cast<double>(issue[issue.size() / 2]) / static_cast<double>(iters);
  *cycles_per_mma = static_cast<double>(total[total.size() / 2]) / static_cast<double>(iters);
  return CUTBCE_OK;
}

const char* cutbce_status_string(cutbce_status s) {
  switch (s) {
    case CUTBCE_OK: return "ok";
    case CUTBCE_ERR_INVALID_ARG: return "invalid argument";
    case CUTBCE_ERR_UNSUPPORTED: return "unsupported problem or device";
    case CUTBCE_ERR_WORKSPACE: return "workspace too small";
    case CUTBCE_ERR_TARGET_RANGE: return "target id out of range";
    case CUTBCE_ERR_TIMEOUT: return "bounded wait in a kernel ran out";
    case CUTBCE_ERR_CUDA: return "CUDA runtime error";
  }
  return "unknown status";
}

cutbce_status cutbce_selftest_element_math(const float* x, float* out, int64_t n, cutbce_stream_t stream) {
  if (x == nullptr || out == nullptr || n <= 0 || n > (int64_t(1) << 30)) return CUTBCE_ERR_INVALID_ARG;
  k_selftest_element_math<<<static_cast<unsigned>(ceil_div(n, 256)), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      x, out, n);
  return cudaGetLastError() == cudaSuccess ? CUTBCE_OK : CUTBCE_ERR_CUDA;
}

cutbce_status cutbce_selftest_wait_timeout(int64_t limit_ns, int32_t* status_dev, cutbce_stream_t stream) {
  if (status_dev == nullptr || limit_ns <= 0 || limit_ns > 10000000000LL) return CUTBCE_ERR_INVALID_ARG;
  k_selftest_wait<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns, status_dev);
  return cudaGetLastError() == cudaSuccess ? CUTBCE_OK : CUTBCE_ERR_CUDA;
}

}  // extern "C"
