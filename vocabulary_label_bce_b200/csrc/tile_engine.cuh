// The tensor-core engine: one persistent, warp-specialised sm_100a kernel
// template that forms logit tiles on tcgen05 (accumulators in tensor memory),
// applies the BCE element math to them in registers and, for the gradient,
// writes the bf16 tile of G = sigmoid(X) - Y back into tensor memory, where
// the second tcgen05 contraction reads it as its A operand.  No logit or
// gradient tile ever leaves the SM, and G never touches shared memory.
//
// Two instantiations cover the hot path of "Cut Binary Cross Entropy"
// (section III-A Eqs. (2)-(3); section III-B Eq. (4)):
//
//   item-owned pass (kDH = false): a CTA owns a tile of 128 items v (rows of E,
//     the stationary operand) and streams every tile of the compacted H.
//     Z^T = E_v H_t^T  -> softplus sum (loss) and sigmoid -> G^T (bf16, TMEM)
//     dE_v += G^T H_t  (accumulated in TMEM across all t, written once, no atomics)
//
//   position-owned pass (kDH = true): a CTA owns a tile of 128 valid positions
//     (rows of H) and streams the item tiles of one vocabulary split.
//     Z = H_t E_v^T    -> sigmoid -> G (bf16, TMEM)
//     dH_t += G E_v    (partial per split, reduced later in a fixed order)
//
// The sparse targets (y = 1) are applied inside the tile, before G is rounded
// to bf16, so that G = sigmoid(z) - y is rounded once:
//   * position-owned pass: each epilogue thread owns one position row, which
//     has at most K positives; it walks them with a forward-only cursor;
//   * item-owned pass: the pairs are grouped by item tile in ascending
//     position; each warp walks its item tile's pairs 32 at a time, and the
//     lanes holding a pair of the warp's rows and slab set the bit in a
//     per-warp shared-memory word (atomicOr), which the row's lane then takes.
// Chunks holding a positive run a separate copy of the element loop with the
// subtraction, so the common path has no per-element test.  The dense loss
// uses no Y at all (Eq. (2): l(x,y) = l(x,0) - y x); the -y x part is the
// sparse correction summed in the prep kernel.
//
// The compacted H is stored halved (exact in bf16), so the tiles hold z / 2,
// the argument of the element math's tanh; the item-owned accumulator then
// holds G^T (H / 2) and is scaled by twice the gradient scale (exact).  The
// loss tiles sum |z| / 2; the linear half of max(z, 0) = z / 2 + |z| / 2 is one
// dot product of column sums, added by the finish kernel.
//
// Warp roles (576 threads, one CTA per SM):
//   warp 0      TMA producer (stationary tile, ring of NX streamed tiles)
//   warp 1      TMEM allocator and MMA issuer: an event loop over the logit
//               MMAs and the gradient MMAs, issued by one elected lane
//   warps 2-17  epilogue.  Warp w reads TMEM lanes 32*(w%4).. (the quarter its
//               sub-partition may access) and one column slab of the tile.
//               Two groups of 8 take alternate tiles (64-column slabs, or
//               32 with 64-row streamed tiles).
//
// Tensor memory holds NZ = 3 fp32 logit buffers, the gradient accumulator and,
// where it fits, a copy of the stationary tile (the logit MMA's A operand, so
// that only its B operand is read from shared memory).  Each epilogue warp
// writes its bf16 G slab over the first half of its own, already loaded,
// logit columns; the gradient MMA reads G from there, and its completion frees
// the buffer for the logit tile three tiles on.
//
// Every wait is bounded (global timer); on expiry the CTA records
// CUTBCE_ERR_TIMEOUT and where it happened in the workspace header, the other
// roles leave their loops, the producer and the MMA issuer wait (bounded) for
// their own copies and MMAs in flight, and the CTA frees its tensor memory.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>
#include "common.cuh"
#include "ptx_sm100.cuh"
#include "elementwise.cuh"
#include "pair_sort.cuh"

namespace cutbce {

struct TileParams {
  int V;                       // items
  int D;                       // real feature width (<= DP)
  int64_t Tpad;                // rows of H_c (multiple of 128)
  WsHeader* hdr;               // n_valid, grad scale, status
  const int* row_ptr;          // [n_valid + 1] pair offsets of compacted rows (CSR by position)
  const int* pair_v;           // CSR by position: items of each row, ascending
  const int* tile_pair_off;    // [ceil(V/128) + 1] offsets into tile_pairs, one range per item tile
  const int* tile_pairs;       // pairs grouped by item tile, ascending position: (v mod 128) << 24 | t
  float* dE;                   // item-owned pass output [V, D] (fp32, or bf16 with de_bf16; null: no gradient)
  int de_bf16;                 // dE is written as bf16 (round to nearest even)
  int de_acc;                  // dE += the gradient instead of dE = the gradient
  const float* wc;             // [Tpad] per-position weights of the compacted rows (0 past n_valid), or null
  double* loss_part;           // one double per (work item, epilogue warp): item-owned pass without weights,
                               // position-owned pass with weights
  float* dh_part;              // position-owned pass output [S, Tpad, DP]
  int2* met_part;              // position-owned pass with metrics: [S, slabs, Tpad] (count of x > 0, TP)
  int nsplit;                  // position-owned pass: vocabulary splits S
  int tiles_per_split;         // streamed item tiles per split
  int n_item_tiles_bn;         // ceil(V / BN)
  int range_begin, range_end;  // the launch's share of the work: item tiles [begin, end) of the
                               // item-owned pass, vocabulary splits [begin, end) of the position-owned
                               // pass (the whole of it: 0 and INT_MAX)
  long long timeout_ns;
};

struct WaitCtx {
  volatile int* abort_flag;
  WsHeader* hdr;
  long long limit;
};

// Where a wait happens, recorded if it gives up: role (1 producer, 2 MMA,
// 4 epilogue), barrier id, and the role's tile or item counter.
__device__ __forceinline__ int wait_tag(int role, int barrier, uint32_t counter) {
  return (role << 28) | (barrier << 20) | static_cast<int>(counter & 0xFFFFFu);
}

// Bounded wait for phase `parity` of `bar`.  Returns false if the CTA aborted
// or the limit ran out (then it records the timeout, where it happened, and
// raises the abort flag).
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const WaitCtx& w, int tag = 0) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if (*w.abort_flag) {
      // record where each role stood when the CTA gave up (first record per role wins)
      const int role = (tag >> 28) & 7;
      if (tag != 0 && role >= 1) atomicCAS(&w.hdr->role_wait_tag[role - 1], 0, tag);
      return false;
    }
    if (static_cast<long long>(global_timer_ns() - t0) > w.limit) {
      *w.abort_flag = 1;
      if (atomicCAS(&w.hdr->status, 0, kErrTimeout) == 0) {
        w.hdr->wait_tag = tag;
        w.hdr->wait_block = static_cast<int>(blockIdx.x);
      }
      return false;
    }
  }
}
// Bounded wait that ignores the abort flag (used to drain in-flight copies/MMAs).
__device__ __forceinline__ bool wait_bar_drain(uint64_t* bar, uint32_t parity, long long limit) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (static_cast<long long>(global_timer_ns() - t0) > limit) return false;
  }
  return true;
}
// Whole-warp wait.  Fast path: every lane tests the phase itself (one
// shared-memory instruction for the warp, each lane acquiring the phase) and a
// vote, not a shuffle, gathers the answers.  Otherwise lane 0 waits (bounded)
// and the warp then synchronises with it, which orders the other lanes after
// lane 0's acquire of the phase.
__device__ __forceinline__ bool wait_bar_warp(uint64_t* bar, uint32_t parity, const WaitCtx& w, int tag = 0) {
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = wait_bar(bar, parity, w, tag);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

struct ItemInfo {
  int s_row0;     // first stationary row
  int x_tile0;    // first streamed tile (in units of BN rows)
  int n_x;        // streamed tiles
  int split;      // position-owned pass: vocabulary split
};

template <int DP, bool kDH>
__device__ __forceinline__ ItemInfo item_info(int i, int n_valid, const TileParams& p) {
  using Cfg = TileCfg<DP>;
  ItemInfo it;
  if (!kDH) {
    it.s_row0 = i * kTileM;
    it.x_tile0 = 0;
    it.n_x = static_cast<int>(ceil_div(n_valid, Cfg::BN));
    it.split = 0;
  } else {
    const int nT = static_cast<int>(ceil_div(n_valid, kTileM));
    const int s = i / nT, m = i - s * nT;
    it.s_row0 = m * kTileM;
    it.x_tile0 = s * p.tiles_per_split;
    it.n_x = min(p.tiles_per_split, p.n_item_tiles_bn - it.x_tile0);
    it.split = s;
  }
  return it;
}

// Forward-only cursor over one row's ascending positive keys (positions for the
// item-owned pass, items for the position-owned pass).
struct RowCursor {
  int cur, end, nxt;
};

__device__ __forceinline__ void cursor_init(RowCursor& rc, const int* __restrict__ keys, int begin, int end,
                                            int first_key) {
  int c = begin;
  while (c < end && __ldg(keys + c) < first_key) ++c;
  rc.cur = c;
  rc.end = end;
  rc.nxt = c < end ? __ldg(keys + c) : 0x7fffffff;
}

// Bit e set for each positive whose key is lo + e, e in [0, 32); consumes every
// key below lo + 32 (keys below lo belong to columns this thread does not own).
__device__ __forceinline__ uint32_t cursor_take_mask(RowCursor& rc, const int* __restrict__ keys, int lo) {
  uint32_t mask = 0;
  while (rc.nxt < lo + 32) {
    if (rc.nxt >= lo) mask |= 1u << (rc.nxt - lo);
    ++rc.cur;
    rc.nxt = rc.cur < rc.end ? __ldg(keys + rc.cur) : 0x7fffffff;
  }
  return mask;
}

template <int DP, bool kLoss, bool kGrad, bool kDH, bool kMet = false>
__global__ void __launch_bounds__(kTileThreads, 1)
    k_tile(const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmX, TileParams p) {
  using Cfg = TileCfg<DP, epi_groups<kDH>()>;
  constexpr int BN = Cfg::BN;
  constexpr int NKB = Cfg::NKB;
  constexpr int NX = Cfg::NX;
  constexpr int NZ = Cfg::NZ;
  constexpr uint32_t S_BYTES = Cfg::S_BYTES, X_BYTES = Cfg::X_BYTES;
  constexpr int ACC_COL = Cfg::ACC_COL;
  static_assert(kLoss || kGrad || kMet, "nothing to do");
  static_assert(!kMet || kDH, "the metrics are counted in the position-owned pass");
  constexpr float kLn2 = kLn2F;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sS = smem;
  uint8_t* sX = sS + S_BYTES;
  uint32_t* sMask = reinterpret_cast<uint32_t*>(sX + NX * X_BYTES);   // [16 warps][32 rows][MASK_WORDS]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sX + NX * X_BYTES + Cfg::MASK_BYTES);
  uint64_t* bar_sfull = bars + 0;                 // stationary tile landed (TMA)
  uint64_t* bar_sempty = bars + 1;                // stationary tile free (MMA commit)
  uint64_t* bar_xfull = bars + 2;                 // [NX] streamed tile landed
  uint64_t* bar_xempty = bar_xfull + NX;          // [NX] streamed tile free
  uint64_t* bar_zfull = bar_xempty + NX;          // [NZ] logit tile ready in TMEM (MMA commit)
  uint64_t* bar_zfree = bar_zfull + NZ;           // [NZ] buffer free: gradient MMA done (commit), or,
                                                  //      without a gradient, logits loaded (epilogue group)
  uint64_t* bar_gready = bar_zfree + NZ;          // [NZ] G tile written over the logits (epilogue group)
  uint64_t* bar_accfull = bar_gready + NZ;        // gradient accumulator complete
  uint64_t* bar_accempty = bar_accfull + 1;       // gradient accumulator read out
  uint64_t* bar_drain = bar_accempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NUM_BARS);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  WsHeader* hdr = p.hdr;
  // read the header once so every thread takes the same early-exit decision
  __shared__ int s_status, s_nvalid;
  if (threadIdx.x == 0) {
    s_status = *reinterpret_cast<volatile int*>(&hdr->status);
    s_nvalid = hdr->n_valid;
  }
  __syncthreads();
  if (s_status != 0) return;  // an earlier step failed
  const int n_valid = s_nvalid;
  // work items: item tiles (item-owned pass) or (split, position tile) pairs,
  // split-major (position-owned pass); this launch takes [i_lo, n_items)
  const int n_pos_tiles = static_cast<int>(ceil_div(n_valid, kTileM));
  const int i_lo = kDH ? min(p.range_begin, p.nsplit) * n_pos_tiles : min(p.range_begin, static_cast<int>(ceil_div(p.V, kTileM)));
  const int n_items = kDH ? min(p.range_end, p.nsplit) * n_pos_tiles
                          : min(p.range_end, static_cast<int>(ceil_div(p.V, kTileM)));

  if (!kDH && n_valid == 0) {
    // no valid position: dE = 0 and every item's loss is 0
    for (int i = i_lo + static_cast<int>(blockIdx.x); i < n_items; i += gridDim.x) {
      if (kLoss && threadIdx.x < kNumEpiWarps) p.loss_part[static_cast<int64_t>(i) * kNumEpiWarps + threadIdx.x] = 0.0;
      if (kGrad && p.dE != nullptr && !p.de_acc) {
        const int64_t r0 = static_cast<int64_t>(i) * kTileM;
        const int64_t r1 = min(static_cast<int64_t>(p.V), r0 + kTileM);
        for (int64_t k = r0 * p.D + threadIdx.x; k < r1 * p.D; k += blockDim.x) {
          if (p.de_bf16) reinterpret_cast<__nv_bfloat16*>(p.dE)[k] = __float2bfloat16_rn(0.f);
          else p.dE[k] = 0.f;
        }
      }
    }
    return;
  }
  if (i_lo + static_cast<int>(blockIdx.x) >= n_items) return;

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    mbar_init(bar_sfull, 1);
    mbar_init(bar_sempty, 1);
    for (int s = 0; s < NX; ++s) {
      mbar_init(bar_xfull + s, 1);
      mbar_init(bar_xempty + s, 1);
    }
    for (int b = 0; b < NZ; ++b) {
      mbar_init(bar_zfull + b, 1);
      // every lane of the group's warps arrives (after its own tensor-memory wait and fence)
      mbar_init(bar_zfree + b, kGrad ? 1 : Cfg::GROUP_WARPS * 32);
      mbar_init(bar_gready + b, Cfg::GROUP_WARPS * 32);
    }
    mbar_init(bar_accfull, 1);
    mbar_init(bar_accempty, Cfg::GROUP_WARPS);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmS);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtx wc{abort_flag, hdr, p.timeout_ns};

  if (warp == 0) {
    // ============================================================ TMA producer
    if (lane == 0) {
      uint32_t ic = 0, xc = 0;
      for (int i = i_lo + static_cast<int>(blockIdx.x); i < n_items; i += gridDim.x, ++ic) {
        const ItemInfo it = item_info<DP, kDH>(i, n_valid, p);
        if (!wait_bar(bar_sempty, (ic & 1) ^ 1, wc, wait_tag(1, 1, ic))) break;
        mbar_arrive_expect_tx(bar_sfull, S_BYTES);
#pragma unroll
        for (int kb = 0; kb < NKB; ++kb)
          tma_load_2d(sS + kb * (kTileM * 128), &tmS, kb * 64, it.s_row0, bar_sfull);
        bool ok = true;
        for (int j = 0; j < it.n_x; ++j, ++xc) {
          const uint32_t st = xc % NX;
          if (!wait_bar(bar_xempty + st, ((xc / NX) & 1) ^ 1, wc, wait_tag(1, 3, xc))) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar_xfull + st, X_BYTES);
          const int row0 = (it.x_tile0 + j) * BN;
#pragma unroll
          for (int kb = 0; kb < NKB; ++kb)
            tma_load_2d(sX + st * X_BYTES + kb * (BN * 128), &tmX, kb * 64, row0, bar_xfull + st);
        }
        if (!ok) {
          ++ic;
          break;
        }
      }
      // wait (bounded) for every copy this thread issued to land
      const long long lim = p.timeout_ns;
      if (ic > 0) wait_bar_drain(bar_sfull, (ic - 1) & 1, lim);
      for (uint32_t st = 0; st < NX; ++st) {
        const uint32_t issued = xc > st ? (xc - st + NX - 1) / NX : 0;
        if (issued > 0) wait_bar_drain(bar_xfull + st, (issued - 1) & 1, lim);
      }
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    // The whole warp runs this loop; lane 0 tests the barriers and shares the
    // answer, one elected lane issues each tcgen05 instruction.  It is an event
    // loop over two in-order streams: logit tiles Z(c) into buffer c mod NZ
    // (ready once the streamed tile has landed and the buffer is free) and
    // gradient MMAs G(c) (ready once the epilogue group has written the G tile
    // over the logits of buffer c mod NZ).  Whichever is ready is issued.
    //
    // Shared-memory descriptors are built once and advanced by adding the byte
    // offset / 16 to their 14-bit start-address field (it cannot carry out:
    // shared memory is below 256 KB); ring positions are counters that wrap.
    {
      constexpr uint32_t idesc_z = idesc_bf16_f32(kTileM, BN, false, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(kTileM, DP, false, true);
      constexpr uint32_t kXStep = X_BYTES >> 4;                       // one ring stage, in descriptor units
      constexpr int kKsPerSlab = Cfg::ZC / 16;                         // gradient K steps per epilogue slab
      const uint64_t dS = smem_desc_sw128(smem_u32(sS), 16, 1024);     // stationary tile, K-major
      const uint64_t dXk = smem_desc_sw128(smem_u32(sX), 16, 1024);    // streamed tile as K-major B
      const uint64_t dXmn = smem_desc_sw128(smem_u32(sX), BN * 128, 1024);  // streamed tile as MN-major B
      const uint32_t tZ = tmem_base, tAcc = tmem_base + ACC_COL, tS = tmem_base + Cfg::S_COL;
      int zi = i_lo + static_cast<int>(blockIdx.x), zj = 0, gi = zi, gj = 0;
      uint32_t zic = 0, cz = 0, gic = 0, cg = 0;
      uint32_t zst = 0, zph = 0, zoff = 0;        // ring stage of the next logit tile, its phase, its offset
      uint32_t gst = 0, goff = 0;                 // ring stage of the next gradient MMA, its offset
      uint32_t zb = 0, zbph = 0;                  // logit buffer of the next Z, and its use parity
      uint32_t gb = 0, gbph = 0;                  // logit buffer of the next G, and its use parity
      bool s_ready = false;                       // the current item's stationary tile is in place
      ItemInfo zit{}, git{};
      if (zi < n_items) zit = git = item_info<DP, kDH>(zi, n_valid, p);
      uint64_t idle_since = 0;
      bool ok = true;
      while (ok && (zi < n_items || (kGrad && gi < n_items))) {
        bool progressed = false;
        // Poll every barrier the next step may need at once: lane k tests one
        // barrier, a single ballot gathers the answers (one shared-memory round
        // trip per iteration instead of a chain of them).
        const bool want_z = zi < n_items;
        const bool want_g = kGrad && gi < n_items && cg < cz;
        bool mine = false;
        if (lane == 0 && want_z && zj == 0 && !s_ready) mine = mbar_test_wait(bar_sfull, zic & 1);
        if (lane == 1 && want_z) mine = mbar_test_wait(bar_xfull + zst, zph);
        if (lane == 2 && want_z) mine = mbar_test_wait(bar_zfree + zb, zbph ^ 1);
        if (lane == 3 && want_g) mine = mbar_test_wait(bar_gready + gb, gbph);
        if (lane == 4 && want_g && gj == 0) mine = mbar_test_wait(bar_accempty, (gic & 1) ^ 1);
        const uint32_t ready = __ballot_sync(0xffffffffu, mine);
        // ---- logit tile Z(cz) into buffer zb
        if (want_z) {
          if (zj == 0 && !s_ready && (ready & 1u)) {
            tc_fence_after();
            s_ready = true;
            if (Cfg::S_IN_TMEM) {
              // stationary tile -> tensor memory once per item; its shared-memory buffer is then free
              if (elect_one()) {
#pragma unroll
                for (int ks = 0; ks < DP / 16; ++ks)
                  tmem_cp_128x256b(tS + 8 * ks, dS + static_cast<uint32_t>((ks >> 2) * (kTileM * 8) + (ks & 3) * 2));
                umma_commit(bar_sempty);
              }
              __syncwarp();
            }
          }
          if ((zj > 0 || s_ready) && (ready & 6u) == 6u) {
            tc_fence_after();
            const uint64_t dB = dXk + zoff;
            const uint32_t tD = tZ + zb * BN;
            if (elect_one()) {
#pragma unroll
              for (int ks = 0; ks < DP / 16; ++ks) {
                const uint64_t bd = dB + static_cast<uint32_t>((ks >> 2) * (BN * 8) + (ks & 3) * 2);
                if (Cfg::S_IN_TMEM) {
                  umma_bf16_tmem_a(tD, tS + 8 * ks, bd, idesc_z, ks > 0 ? 1u : 0u);
                } else {
                  umma_bf16(tD, dS + static_cast<uint32_t>((ks >> 2) * (kTileM * 8) + (ks & 3) * 2), bd, idesc_z,
                            ks > 0 ? 1u : 0u);
                }
              }
              umma_commit(bar_zfull + zb);
              if (!kGrad) umma_commit(bar_xempty + zst);
              if (!Cfg::S_IN_TMEM && zj + 1 == zit.n_x) umma_commit(bar_sempty);  // stationary tile no longer read
            }
            __syncwarp();
            progressed = true;
            ++cz;
            zoff += kXStep;
            if (++zst == static_cast<uint32_t>(NX)) {
              zst = 0;
              zoff = 0;
              zph ^= 1;
            }
            if (++zb == static_cast<uint32_t>(NZ)) {
              zb = 0;
              zbph ^= 1;
            }
            if (++zj == zit.n_x) {
              zj = 0;
              ++zic;
              s_ready = false;
              zi += gridDim.x;
              if (zi < n_items) zit = item_info<DP, kDH>(zi, n_valid, p);
            }
          }
        }
        // ---- gradient MMA G(cg): ACC += G[gb] * X, G from tensor memory, X MN-major
        if (want_g) {
          if ((ready & 8u) && (gj > 0 || (ready & 16u))) {
            tc_fence_after();
            const uint64_t dB = dXmn + goff;
            const uint32_t tA = tZ + gb * BN;
            const bool last = gj + 1 == git.n_x;
            if (elect_one()) {
#pragma unroll
              for (int ks = 0; ks < BN / 16; ++ks) {
                // slab k of the G tile sits in the first half of the logit columns of slab k
                const uint32_t a_col = (ks / kKsPerSlab) * Cfg::ZC + 8 * (ks % kKsPerSlab);
                umma_bf16_tmem_a(tAcc, tA + a_col, dB + static_cast<uint32_t>(ks * 128), idesc_acc,
                                 (gj > 0 || ks > 0) ? 1u : 0u);
              }
              umma_commit(bar_zfree + gb);
              umma_commit(bar_xempty + gst);
              if (last) umma_commit(bar_accfull);
            }
            __syncwarp();
            progressed = true;
            ++cg;
            goff += kXStep;
            if (++gst == static_cast<uint32_t>(NX)) {
              gst = 0;
              goff = 0;
            }
            if (++gb == static_cast<uint32_t>(NZ)) {
              gb = 0;
              gbph ^= 1;
            }
            if (last) {
              gj = 0;
              ++gic;
              gi += gridDim.x;
              if (gi < n_items) git = item_info<DP, kDH>(gi, n_valid, p);
            } else {
              ++gj;
            }
          }
        }
        // ---- bounded: give up if nothing became ready within the limit
        if (progressed) {
          idle_since = 0;
        } else {
          const uint64_t now = global_timer_ns();
          if (idle_since == 0) idle_since = now;
          int give_up = 0;
          if (lane == 0) {
            if (*abort_flag) {
              give_up = 1;
            } else if (static_cast<long long>(now - idle_since) > p.timeout_ns) {
              *abort_flag = 1;
              if (atomicCAS(&hdr->status, 0, kErrTimeout) == 0) {
                hdr->wait_tag = wait_tag(2, 15, cz);
                hdr->wait_block = static_cast<int>(blockIdx.x);
              }
              give_up = 1;
            }
          }
          if (__shfl_sync(0xffffffffu, give_up, 0)) ok = false;
        }
      }
      // every MMA this warp issued has completed once the drain barrier flips
      if (elect_one()) umma_commit(bar_drain);
      __syncwarp();
      if (lane == 0) wait_bar_drain(bar_drain, 0, p.timeout_ns);
      __syncwarp();
    }
  } else if (warp >= kEpiWarp0) {
    // ============================================================ epilogue
    // Two groups of 8 warps take alternate tiles (group = tile counter & 1), so
    // one group's tensor-memory traffic overlaps the other group's element math.
    // In a group, warp w reads TMEM lanes 32*(w%4).. (its sub-partition's
    // quarter) and one of two column slabs of the tile, and writes the same
    // slab of the G tile.
    constexpr int ZC = Cfg::ZC;                   // Z columns per warp per tile (64 or 32)
    constexpr int CH = ZC < 32 ? ZC : 32;         // columns per TMEM load
    constexpr int AC = DP / Cfg::SLABS;            // accumulator columns per warp (16 .. 128)
    const int ew = warp - kEpiWarp0;
    const uint32_t grp = static_cast<uint32_t>(ew / Cfg::GROUP_WARPS);   // group: takes tiles c with c mod groups = grp
    const int q = warp & 3;                       // TMEM lane quarter
    const int slab = (ew >> 2) % Cfg::SLABS;       // column slab within the group
    const int row = q * 32 + lane;                // stationary row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    // the item-owned accumulator holds G^T (H / 2): its scale is doubled (exact)
    const float gs = hdr->grad_scale * (kDH ? 1.f : 2.f);
    uint32_t* wmask = sMask + ew * 32 * Cfg::MASK_WORDS;   // this warp's positives scratch
#pragma unroll
    for (int k = 0; k < Cfg::MASK_WORDS; ++k) wmask[lane * Cfg::MASK_WORDS + k] = 0u;
    __syncwarp();
    uint32_t cnt = 0, ic = 0;
    bool ok = true;
    for (int i = i_lo + static_cast<int>(blockIdx.x); i < n_items && ok; i += gridDim.x, ++ic) {
      const ItemInfo it = item_info<DP, kDH>(i, n_valid, p);
      const int n = it.n_x;
      double item_acc = 0.0;
      int met_cnt = 0, met_tp = 0;                // position-owned pass: this row's x > 0 count and TP
      // Positives (y = 1).  Position-owned pass: this thread's row (a position)
      // has at most K of them, walked with a forward cursor over its items.
      // Item-owned pass: the item tile's pairs, in ascending position, are
      // walked by the whole warp, 32 at a time, one cursor per warp.
      RowCursor rc{0, 0, 0x7fffffff};
      int seg = 0, seg_end = 0;
      uint32_t win = 0xFFFFFFFFu;                 // item-owned pass: pairs seg .. seg + 31, one per lane
      if (kGrad || kMet) {
        if (kDH) {
          const int r = it.s_row0 + row;
          if (r < n_valid) cursor_init(rc, p.pair_v, __ldg(p.row_ptr + r), __ldg(p.row_ptr + r + 1), it.x_tile0 * BN);
        } else {
          seg = __ldg(p.tile_pair_off + i);
          seg_end = __ldg(p.tile_pair_off + i + 1);
          win = seg + lane < seg_end ? static_cast<uint32_t>(__ldg(p.tile_pairs + seg + lane)) : 0xFFFFFFFFu;
        }
      }
      // this group's tiles of the item: c = cnt + j with c mod groups = grp
      const int j0 = static_cast<int>((grp + Cfg::GROUPS - cnt % Cfg::GROUPS) % Cfg::GROUPS);
      for (int j = j0; j < n; j += Cfg::GROUPS) {
        const uint32_t c = cnt + j, bz = c % NZ;
        constexpr int NCH = ZC / CH;
        uint32_t pmask[NCH];                      // item-owned pass: this row's positives per chunk
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) pmask[ch] = 0u;
        if (kGrad && !kDH) {
          // consume the item tile's pairs with position < end of this tile; keep
          // those in this warp's rows and column slab (done before the logit wait,
          // so the loads overlap it)
          const int t_hi = (j + 1) * BN, t_lo = j * BN + slab * ZC;
          bool any_pair = false;                  // this lane set a bit in the scratch
          // one window of 32 pairs: set this warp's bits, return how many pairs lie below t_hi
          auto take = [&](uint32_t val) -> int {
            const int t = static_cast<int>(val & ((1u << kPairPosBits) - 1u));
            const int rr = static_cast<int>(val >> kPairPosBits);
            const unsigned below = __ballot_sync(0xffffffffu, t < t_hi);   // a prefix: positions ascend
            // each lane holding one of this warp's pairs sets its bit in the row's
            // word in shared memory (the lanes work in parallel)
            if (t < t_hi && t >= t_lo && t < t_lo + ZC && (rr >> 5) == q) {
              const int cc = t - t_lo;
              atomicOr(wmask + (rr & 31) * Cfg::MASK_WORDS + (cc >> 5), 1u << (cc & 31));
              any_pair = true;
            }
            return __popc(below);
          };
          const int seg0 = seg;
          int nb = take(win);
          seg += nb;
          if (nb == 32) {
            // a hot tile (more than one window of pairs): fetch four windows per
            // round trip to memory instead of one
            constexpr int kBatch = 4;
            bool more = true;
            while (more) {
              uint32_t w[kBatch];
#pragma unroll
              for (int k = 0; k < kBatch; ++k) {
                const int pi = seg + 32 * k + lane;
                w[k] = pi < seg_end ? static_cast<uint32_t>(__ldg(p.tile_pairs + pi)) : 0xFFFFFFFFu;
              }
#pragma unroll
              for (int k = 0; k < kBatch; ++k) {
                if (!more) break;
                nb = take(w[k]);
                seg += nb;
                more = nb == 32;
              }
            }
          }
          // the next window: loaded now, first read at this group's next tile
          // (nothing to load while no pair was consumed, the common case)
          if (seg != seg0) {
            const int pi = seg + lane;
            win = pi < seg_end ? static_cast<uint32_t>(__ldg(p.tile_pairs + pi)) : 0xFFFFFFFFu;
          }
          if (__any_sync(0xffffffffu, any_pair)) {
            __syncwarp();
            // this lane's row: take its words and clear them for the next tile
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) {
              pmask[ch] = wmask[lane * Cfg::MASK_WORDS + ch];
              wmask[lane * Cfg::MASK_WORDS + ch] = 0u;
            }
            __syncwarp();
          }
        }
        if (!wait_bar_warp(bar_zfull + bz, (c / NZ) & 1, wc, wait_tag(4, 4, c))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int key0 = kDH ? (it.x_tile0 + j) * BN : j * BN;   // key of the tile's first column
        // loss terms of the whole tile: the product of the w of its NCH * CH / 2
        // logits per component (each in [1, 2], so at most 2^32 per component and
        // 2^64 for both: finite in fp32) and the sum of |z| / 2
        float2 prod = f2(1.f, 1.f), absz = f2(0.f, 0.f);
        float tile_mx = 0.f, tile_l2 = 0.f;
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
          const int col0 = slab * ZC + ch * CH;
          uint32_t r[CH];
          tmem_ld<CH>(tmem_base + lane_base + bz * BN + col0, r);
          tmem_ld_wait();
          if (!kGrad && ch == NCH - 1) {          // no G: the buffer is free once loaded
            tc_fence_before();
            mbar_arrive(bar_zfree + bz);          // each lane, for its own loads
          }
          const uint32_t mask = !(kGrad || kMet) ? 0u
                                : kDH ? cursor_take_mask(rc, p.pair_v, key0 + col0)
                                      : (NCH == 1 || ch == 0) ? pmask[0] : pmask[NCH - 1];
          const bool any_pos = (kGrad || kMet) && __any_sync(0xffffffffu, mask != 0u);
          float2 mcnt = f2(0.f, 0.f);             // metrics: x > 0 in this chunk (two lanes of a sum)
          float mtp = 0.f;                        // metrics: positives with x > 0 in this chunk
          uint32_t pk[CH / 2];
          // the chunk's element math; the y = 1 subtraction is compiled into a
          // separate copy taken only by chunks that hold a positive (rare), so
          // the common path has no per-element branch or bit test
          // column weights (item-owned pass with per-position weights): G = w (sigmoid - y)
          // (per-position weights move the loss to the position-owned pass, so
          // only the gradient-only item-owned pass ever takes them: the pass with
          // the loss carries no weighted copy of the element loop)
          const float* wcol = (!kDH && kGrad && !kLoss) ? p.wc : nullptr;
          const int wcol0 = j * BN + col0;        // compacted position of this chunk's first column
          auto chunk_math = [&](auto with_y, auto with_w) {
#pragma unroll
            for (int e = 0; e < CH; e += 2) {
              const float2 z = f2(__uint_as_float(r[e]), __uint_as_float(r[e + 1]));   // z / 2 (H_c holds H / 2)
              float2 g = f2(0.f, 0.f);
              float2 mpos = f2(0.f, 0.f);
              if (kMet) {
                // [x > 0] on the FMA pipe, from x / 2: saturate(x / 2 * 2^126) is 1 for every
                // normal x / 2 > 0 and 0 for x <= 0 (a subnormal is flushed to 0: not positive)
                mpos = f2(positive_mask(z.x), positive_mask(z.y));
                mcnt = __fadd2_rn(mcnt, mpos);
                if (decltype(with_y)::value) {
                  if (mask & (1u << e)) mtp += mpos.x;
                  if (mask & (1u << (e + 1))) mtp += mpos.y;
                }
              }
              if (!kLoss && !kGrad) {
                // metrics only: no element math beyond the count
              } else if (kLoss && kGrad) {
                g = bce_pair_loss_grad(z, prod, absz);
              } else if (kLoss) {
                bce_pair_loss(z, prod, absz);
              } else if (((e >> 1) * kPolyPairsPerChunk) % 16 < kPolyPairsPerChunk) {
                g = sigmoid_pair_fma(z);            // wholly on the FMA pipe (a few pairs, spread evenly)
              } else {
                g = sigmoid_pair_tanh(z);           // one tanh per logit on the SFU
              }
              if (kGrad) {
                if (decltype(with_y)::value) {                     // y = 1 at the masked columns
                  if (mask & (1u << e)) g.x -= 1.f;                // a predicated add, no conversion
                  if (mask & (1u << (e + 1))) g.y -= 1.f;
                }
                if (decltype(with_w)::value) g = __fmul2_rn(g, __ldg(reinterpret_cast<const float2*>(wcol + wcol0 + e)));
                pk[e >> 1] = pack_bf16x2(g.x, g.y);
              }
            }
          };
          if (wcol != nullptr) {
            if (any_pos) chunk_math(std::true_type{}, std::true_type{});
            else chunk_math(std::false_type{}, std::true_type{});
          } else {
            if (any_pos) chunk_math(std::true_type{}, std::false_type{});
            else chunk_math(std::false_type{}, std::false_type{});
          }
          if (kMet) {
            met_cnt += static_cast<int>(mcnt.x + mcnt.y);     // exact: at most CH
            met_tp += static_cast<int>(mtp);
          }
          // G over the first half of this warp's own (already loaded) logit columns
          if (kGrad) {
            if constexpr (CH == 32) tmem_st16(tmem_base + lane_base + bz * BN + slab * ZC + ch * (CH / 2), pk);
            else tmem_st8(tmem_base + lane_base + bz * BN + slab * ZC + ch * (CH / 2), pk);
          }
        }
        if (kLoss) {
          // tile_l2 collects log2(1 + e^{-|z|}) = 1 - log2 w of each element (w = 2 sigmoid(|z|)),
          // one log for the whole tile
          tile_l2 = static_cast<float>(NCH * CH) - lg2_approx(prod.x * prod.y);
          tile_mx = absz.x + absz.y;
        }
        if (!ok) break;
        if (kGrad) {
          tmem_st_wait();
          tc_fence_before();
          // each lane's part of G is in place: every lane arrives for its own
          // stores (no warp barrier, no single-lane branch)
          mbar_arrive(bar_gready + bz);
        }
        if (kLoss) {
          if (!kDH && j == n - 1) {
            // zero rows of H_c past n_valid give z = 0 exactly: each adds log2(2) = 1 to tile_l2
            const int t0 = j * BN;
            const int lo = slab * ZC, hi = lo + ZC;
            const int pad = hi - max(min(n_valid - t0, hi), lo);
            tile_l2 -= static_cast<float>(pad);
          }
          if (kDH && it.x_tile0 + j == p.n_item_tiles_bn - 1) {
            // item rows past V in the last streamed tile are zero-filled: z = 0, log2(2) = 1 each
            const int v0 = (it.x_tile0 + j) * BN;
            const int lo = slab * ZC, hi = lo + ZC;
            const int pad = hi - max(min(p.V - v0, hi), lo);
            tile_l2 -= static_cast<float>(pad);
          }
          item_acc += static_cast<double>(tile_mx + tile_l2 * kLn2);   // tile_mx sums |z| / 2
        }
      }
      if (!ok) break;
      if (kLoss) {
        // one partial per (item tile, epilogue warp): no cross-warp barrier, fixed summation order
        // item-owned pass: rows past V are padding; position-owned pass: the row's
        // loss times its weight (0 for the compacted rows past n_valid)
        double val = kDH ? item_acc * static_cast<double>(__ldg(p.wc + it.s_row0 + row))
                         : ((it.s_row0 + row < p.V) ? item_acc : 0.0);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) val += __shfl_xor_sync(0xffffffffu, val, off);
        if (lane == 0) p.loss_part[static_cast<int64_t>(i) * kNumEpiWarps + ew] = val;
      }
      if (kMet) {
        // one partial per (split, column slab, row), summed in a fixed order by the finish kernel;
        // every group writes its own slab's counts, so with two groups the slabs of both are summed
        const int slot = (it.split * Cfg::GROUPS + static_cast<int>(grp)) * Cfg::SLABS + slab;
        p.met_part[static_cast<int64_t>(slot) * p.Tpad + it.s_row0 + row] = make_int2(met_cnt, met_tp);
      }
      if (kGrad && (cnt + n - 1) % Cfg::GROUPS == grp) {
        // the group that took the item's last tile reads the accumulator out
        if (!wait_bar_warp(bar_accfull, ic & 1, wc, wait_tag(4, 9, ic))) break;
        tc_fence_after();
#pragma unroll 1
        for (int ch = 0; ch < AC / 16; ++ch) {
          uint32_t r[16];
          const int col0 = slab * AC + ch * 16;
          tmem_ld<16>(tmem_base + lane_base + ACC_COL + col0, r);
          tmem_ld_wait();
          if (!kDH) {
            const int v = it.s_row0 + row;
            if (v < p.V && p.dE != nullptr) {
              const int64_t o = static_cast<int64_t>(v) * p.D + col0;
#pragma unroll
              for (int e = 0; e < 16; e += 4) {
                if (col0 + e < p.D) {
                  // the fp32 gradient, rounded as written without accumulation (no fused multiply-add)
                  float4 g4 = make_float4(__fmul_rn(__uint_as_float(r[e]), gs), __fmul_rn(__uint_as_float(r[e + 1]), gs),
                                          __fmul_rn(__uint_as_float(r[e + 2]), gs), __fmul_rn(__uint_as_float(r[e + 3]), gs));
                  if (p.de_bf16) {
                    uint2* dst = reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p.dE) + o + e);
                    if (p.de_acc) {
                      const uint2 old = *dst;
                      g4.x = __fadd_rn(g4.x, __uint_as_float(old.x << 16));
                      g4.y = __fadd_rn(g4.y, __uint_as_float(old.x & 0xFFFF0000u));
                      g4.z = __fadd_rn(g4.z, __uint_as_float(old.y << 16));
                      g4.w = __fadd_rn(g4.w, __uint_as_float(old.y & 0xFFFF0000u));
                    }
                    *dst = make_uint2(pack_bf16x2(g4.x, g4.y), pack_bf16x2(g4.z, g4.w));
                  } else {
                    float4* dst = reinterpret_cast<float4*>(p.dE + o + e);
                    if (p.de_acc) {
                      const float4 old = *dst;
                      g4.x = __fadd_rn(g4.x, old.x);
                      g4.y = __fadd_rn(g4.y, old.y);
                      g4.z = __fadd_rn(g4.z, old.z);
                      g4.w = __fadd_rn(g4.w, old.w);
                    }
                    *dst = g4;
                  }
                }
              }
            }
          } else {
            float* dst = p.dh_part + (static_cast<int64_t>(it.split) * p.Tpad + it.s_row0 + row) * DP + col0;
#pragma unroll
            for (int e = 0; e < 16; e += 4)
              *reinterpret_cast<float4*>(dst + e) = make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                                                                __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_accempty);
      }
      cnt += n;
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// Element-math self test, for each x: [0] the FMA-pipe 2^x, [1] the SFU 2^x,
// [2] the gradient-only sigmoid of z = x on the FMA pipe, [3] the sigmoid from
// tanh, [4] w = 1 + |tanh(x/2)| as the loss-and-gradient passes form it.  Used
// only by cutbce_selftest_element_math.
__global__ void k_selftest_element_math(const float* __restrict__ x, float* __restrict__ out, int64_t n) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float v = x[i];
  out[i] = exp2_poly3_pair(f2(v, v)).x;
  out[n + i] = ex2_approx(v);
  const float vh = 0.5f * v;                     // the tiles hold z / 2
  out[2 * n + i] = sigmoid_pair_fma(f2(vh, vh)).x;
  out[3 * n + i] = sigmoid_pair_tanh(f2(vh, vh)).x;
  float2 prod = f2(1.f, 1.f), absz = f2(0.f, 0.f);
  bce_pair_loss_grad(f2(vh, vh), prod, absz);
  out[4 * n + i] = prod.x;
}

// A deliberately unsignalled barrier: the bounded wait must give up, record the
// timeout and return.  Used only by cutbce_selftest_wait_timeout.
__global__ void k_selftest_wait(long long limit_ns, int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    *status = 0;
    if (!wait_bar_drain(&bar, 0, limit_ns)) *status = kErrTimeout;
  }
}

}  // namespace cutbce
