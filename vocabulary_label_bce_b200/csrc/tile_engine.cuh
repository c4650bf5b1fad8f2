// The tensor-core engine: one persistent, warp-specialised sm_100a kernel
// template that forms logit tiles on tcgen05 (accumulators in tensor memory),
// applies the BCE element math to them in registers and, for the gradient,
// feeds the bf16 tile of G = sigmoid(X) - Y straight back into a second
// tcgen05 contraction.  No logit or gradient tile ever leaves the SM.
//
// Two instantiations cover the hot path of "Cut Binary Cross Entropy"
// (section III-A Eqs. (2)-(3); section III-B Eq. (4)):
//
//   item-owned pass (kDH = false): a CTA owns a tile of 128 items v (rows of E,
//     the stationary operand) and streams every tile of the compacted H.
//     Z^T = E_v H_t^T  -> softplus sum (loss) and sigmoid -> G^T (bf16, smem)
//     dE_v += G^T H_t  (accumulated in TMEM across all t, written once, no atomics)
//
//   position-owned pass (kDH = true): a CTA owns a tile of 128 valid positions
//     (rows of H) and streams the item tiles of one vocabulary split.
//     Z = H_t E_v^T    -> sigmoid -> G (bf16, smem)
//     dH_t += G E_v    (partial per split, reduced later in a fixed order)
//
// The sparse targets enter in-tile: after the epilogue warps write sigmoid(z)
// for a tile, a fix-up warp subtracts 1 at the (at most a few) positions of the
// tile where y = 1, walking lists of pairs pre-sorted by item.  The dense loss
// term uses no Y at all (Eq. (2): l(x,y) = l(x,0) - y x); the -y x part is the
// separate sparse correction summed in the prep kernel.
//
// Warp roles (640 threads, one CTA per SM):
//   warp 0      TMA producer (stationary tile, ring of streamed tiles)
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warp 2      fix-up warp (Y in-tile)
//   warp 3      idle
//   warps 4-19  epilogue: warp w reads TMEM lanes 32*(w%4).. and one quarter
//               of the tile's columns
//
// Every wait is bounded (global timer); on expiry the CTA records
// CUTBCE_ERR_TIMEOUT in the status word, the other roles leave their loops, the
// producer and the MMA issuer wait (bounded) for their own copies and MMAs in
// flight, and the CTA frees its tensor memory and returns.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include "common.cuh"
#include "ptx_sm100.cuh"

namespace cutbce {

struct TileParams {
  int V;                       // items
  int D;                       // real feature width (<= DP)
  int64_t Tpad;                // rows of H_c (multiple of 128)
  WsHeader* hdr;               // n_valid, grad scale, status
  const int* row_ptr;          // [n_valid + 1] pair offsets of compacted rows
  const int* grp_v;            // position-owned pass: pairs sorted by (item, position) per 128-row group
  const int* grp_t;
  const int* srt_t;            // item-owned pass: pairs sorted by (item tile, position, item)
  const int* srt_v;
  const int* item_start;       // item-owned pass: [n_item_tiles + 1] ranges into srt_*
  float* dE;                   // item-owned pass output [V, D] (may be null when no gradient)
  double* loss_part;           // item-owned pass: one double per (item tile, epilogue warp)
  float* dh_part;              // position-owned pass output [S, Tpad, DP]
  int nsplit;                  // position-owned pass: vocabulary splits S
  int tiles_per_split;         // streamed item tiles per split
  int n_item_tiles_bn;         // ceil(V / BN)
  long long timeout_ns;
};

struct WaitCtx {
  volatile int* abort_flag;
  WsHeader* hdr;
  long long limit;
};

// Where a wait happens, recorded if it gives up: role (1 producer, 2 MMA,
// 3 fix-up, 4 epilogue), barrier id, and the role's tile or item counter.
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
    if (mbar_try_wait(bar, parity)) return true;
    if (*w.abort_flag) {
      // record where each role stood when the CTA gave up (first record per role wins)
      if (tag != 0) atomicCAS(reinterpret_cast<int*>(w.hdr) + 8 + ((tag >> 28) & 7), 0, tag);
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
// Whole-warp wait with a warp-uniform result.
__device__ __forceinline__ bool wait_bar_warp(uint64_t* bar, uint32_t parity, const WaitCtx& w, int tag = 0) {
  const bool ok = wait_bar(bar, parity, w, tag);
  return __all_sync(0xffffffffu, ok);
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

// Forward-only cursor over one sorted pair range, lane-uniform.  `nxt` holds
// the key (position for the item-owned pass, item for the position-owned pass)
// of the next unapplied pair, so a tile without positives costs no memory
// access.  Every pair with key < hi is applied to the bf16 G tile by
// subtracting 1 (y = 1 in G = sigmoid(X) - Y).
struct PairCursor {
  int cur, end, nxt;
};

template <bool kDH>
__device__ __forceinline__ void fixup_apply(PairCursor& c, int hi, int x0, int s0, uint8_t* G,
                                            const int* __restrict__ keys, const int* __restrict__ others,
                                            int lane) {
  while (c.nxt < hi) {
    const int idx = c.cur + lane;
    const int key = idx < c.end ? __ldg(keys + idx) : 0x7fffffff;
    const bool in = key < hi;
    if (in) {
      const int other = __ldg(others + idx);
      // item-owned: rows are items, columns are positions; position-owned: the reverse
      const int row = other - s0;
      const int col = key - x0;
      const uint32_t off = static_cast<uint32_t>(col >> 6) * 16384u + static_cast<uint32_t>(row) * 128u +
                           ((((static_cast<uint32_t>(col) & 63u) >> 3) ^ (static_cast<uint32_t>(row) & 7u)) << 4) +
                           ((static_cast<uint32_t>(col) & 7u) << 1);
      __nv_bfloat16* e = reinterpret_cast<__nv_bfloat16*>(G + off);
      *e = __float2bfloat16_rn(__bfloat162float(*e) - 1.0f);
    }
    const unsigned m = __ballot_sync(0xffffffffu, in);
    const int n = __popc(m);
    c.cur += n;
    if (n < 32) {
      c.nxt = __shfl_sync(0xffffffffu, key, n);
    } else {
      c.nxt = c.cur < c.end ? __ldg(keys + c.cur) : 0x7fffffff;
    }
  }
}

// First index in [lo, hi) of an ascending int array whose value is >= target.
__device__ __forceinline__ int lower_bound_idx(const int* __restrict__ a, int lo, int hi, int target) {
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(a + mid) < target) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

template <int DP, bool kLoss, bool kGrad, bool kDH>
__global__ void __launch_bounds__(kTileThreads, 1)
    k_tile(const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmX, TileParams p) {
  using Cfg = TileCfg<DP>;
  constexpr int BN = Cfg::BN;
  constexpr int NKB = Cfg::NKB;
  constexpr int NX = Cfg::NX;
  constexpr int NZ = Cfg::NZ;
  constexpr int NG = Cfg::NG;
  constexpr uint32_t S_BYTES = Cfg::S_BYTES, X_BYTES = Cfg::X_BYTES, G_BYTES = Cfg::G_BYTES;
  constexpr int ACC_COL = Cfg::ACC_COL;
  static_assert(!kDH || (kGrad && !kLoss), "the position-owned pass computes dH only");
  static_assert(kLoss || kGrad, "nothing to do");
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr float kLn2 = 0.6931471805599453f;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sS = smem;
  uint8_t* sX = sS + S_BYTES;
  uint8_t* sG = sX + NX * X_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sG + NG * G_BYTES);
  uint64_t* bar_sfull = bars + 0;                 // stationary tile landed (TMA)
  uint64_t* bar_sempty = bars + 1;                // stationary tile free (MMA commit)
  uint64_t* bar_xfull = bars + 2;                 // [NX] streamed tile landed
  uint64_t* bar_xempty = bar_xfull + NX;          // [NX] streamed tile free
  uint64_t* bar_zfull = bar_xempty + NX;          // [NZ] logit tile ready in TMEM
  uint64_t* bar_zempty = bar_zfull + NZ;          // [NZ] logit tile read by the epilogue
  uint64_t* bar_gwritten = bar_zempty + NZ;       // [NG] sigmoid tile written by the epilogue
  uint64_t* bar_fixdone = bar_gwritten + NG;      // [NG] target fix-ups of the tile applied
  uint64_t* bar_gempty = bar_fixdone + NG;        // [NG] sigmoid tile consumed by the MMA
  uint64_t* bar_accfull = bar_gempty + NG;        // gradient accumulator complete
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
  const int n_items = kDH ? p.nsplit * static_cast<int>(ceil_div(n_valid, kTileM))
                          : static_cast<int>(ceil_div(p.V, kTileM));

  if (!kDH && n_valid == 0) {
    // no valid position: dE = 0 and every item's loss is 0
    for (int i = blockIdx.x; i < n_items; i += gridDim.x) {
      if (kLoss && threadIdx.x < kNumEpiWarps) p.loss_part[static_cast<int64_t>(i) * kNumEpiWarps + threadIdx.x] = 0.0;
      if (kGrad && p.dE != nullptr) {
        const int64_t r0 = static_cast<int64_t>(i) * kTileM;
        const int64_t r1 = min(static_cast<int64_t>(p.V), r0 + kTileM);
        for (int64_t k = r0 * p.D + threadIdx.x; k < r1 * p.D; k += blockDim.x) p.dE[k] = 0.f;
      }
    }
    return;
  }
  if (static_cast<int>(blockIdx.x) >= n_items) return;

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
      mbar_init(bar_zempty + b, kNumEpiWarps);
    }
    for (int b = 0; b < NG; ++b) {
      mbar_init(bar_gwritten + b, kNumEpiWarps);
      mbar_init(bar_fixdone + b, 1);
      mbar_init(bar_gempty + b, 1);
    }
    mbar_init(bar_accfull, 1);
    mbar_init(bar_accempty, kNumEpiWarps);
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
      for (int i = blockIdx.x; i < n_items; i += gridDim.x, ++ic) {
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
    // One thread.  Logit tiles (Z) run up to NZ tiles ahead of the gradient
    // MMAs, so the epilogue always finds its next tile computed.
    if (lane == 0) {
      constexpr uint32_t idesc_z = idesc_bf16_f32(kTileM, BN, false, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(kTileM, DP, false, true);
      const uint32_t sS_a = smem_u32(sS), sX_a = smem_u32(sX), sG_a = smem_u32(sG);
      int zi = blockIdx.x, zj = 0, gi = blockIdx.x, gj = 0;
      uint32_t zic = 0, cz = 0, gic = 0, cg = 0;
      ItemInfo zit{}, git{};
      if (zi < n_items) zit = git = item_info<DP, kDH>(zi, n_valid, p);
      // Z[cz % NZ] = S * X^T : both operands K-major, 128-byte swizzle
      auto issue_next_z = [&]() -> bool {
        if (zj == 0) {
          if (!wait_bar(bar_sfull, zic & 1, wc, wait_tag(2, 0, zic))) return false;
          tc_fence_after();
        }
        const uint32_t st = cz % NX, b = cz % NZ;
        if (!wait_bar(bar_xfull + st, (cz / NX) & 1, wc, wait_tag(2, 2, cz))) return false;
        if (!wait_bar(bar_zempty + b, ((cz / NZ) & 1) ^ 1, wc, wait_tag(2, 5, cz))) return false;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < DP / 16; ++ks) {
          const uint64_t a = smem_desc_sw128(sS_a + (ks >> 2) * (kTileM * 128) + (ks & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sX_a + st * X_BYTES + (ks >> 2) * (BN * 128) + (ks & 3) * 32, 16, 1024);
          umma_bf16(tmem_base + b * BN, a, bd, idesc_z, ks > 0 ? 1u : 0u);
        }
        umma_commit(bar_zfull + b);
        if (!kGrad) umma_commit(bar_xempty + st);
        ++cz;
        if (++zj == zit.n_x) {
          umma_commit(bar_sempty);                 // the stationary tile is no longer read
          zj = 0;
          ++zic;
          zi += gridDim.x;
          if (zi < n_items) zit = item_info<DP, kDH>(zi, n_valid, p);
        }
        return true;
      };
      bool ok = true;
      if (!kGrad) {
        while (ok && zi < n_items) ok = issue_next_z();
      } else {
        while (ok && gi < n_items) {
          while (ok && zi < n_items && cz < cg + NZ) ok = issue_next_z();
          if (!ok) break;
          const uint32_t b = cg % NG, st = cg % NX;
          if (!wait_bar(bar_gwritten + b, (cg / NG) & 1, wc, wait_tag(2, 6, cg)) ||
              !wait_bar(bar_fixdone + b, (cg / NG) & 1, wc, wait_tag(2, 7, cg)))
            break;
          tc_fence_after();
          if (gj == 0) {
            if (!wait_bar(bar_accempty, (gic & 1) ^ 1, wc, wait_tag(2, 10, gic))) break;
            tc_fence_after();
          }
          // ACC += G[b] * X[st] : G K-major, X read MN-major (its rows are the K index)
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks) {
            const uint64_t a = smem_desc_sw128(sG_a + b * G_BYTES + (ks >> 2) * (kTileM * 128) + (ks & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(sX_a + st * X_BYTES + ks * 2048, BN * 128, 1024);
            umma_bf16(tmem_base + ACC_COL, a, bd, idesc_acc, (gj > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(bar_gempty + b);
          umma_commit(bar_xempty + st);
          ++cg;
          if (++gj == git.n_x) {
            umma_commit(bar_accfull);
            gj = 0;
            ++gic;
            gi += gridDim.x;
            if (gi < n_items) git = item_info<DP, kDH>(gi, n_valid, p);
          }
        }
      }
      // every MMA this thread issued has completed once the drain barrier flips
      umma_commit(bar_drain);
      wait_bar_drain(bar_drain, 0, p.timeout_ns);
    }
  } else if (warp == 2) {
    // ============================================================ Y fix-up warp
    if (kGrad) {
      uint32_t cnt = 0;
      bool ok = true;
      for (int i = blockIdx.x; i < n_items && ok; i += gridDim.x) {
        const ItemInfo it = item_info<DP, kDH>(i, n_valid, p);
        PairCursor pc;
        if (!kDH) {
          // the item tile's pairs, ordered by position
          pc.cur = __ldg(p.item_start + i);
          pc.end = __ldg(p.item_start + i + 1);
          pc.nxt = pc.cur < pc.end ? __ldg(p.srt_t + pc.cur) : 0x7fffffff;
        } else {
          // the 128 stationary positions' pairs, ordered by item, from the split's first item on
          const int g0 = it.s_row0;
          const int gs = __ldg(p.row_ptr + g0);
          const int ge = __ldg(p.row_ptr + min(g0 + kGroupRows, n_valid));
          pc.cur = lower_bound_idx(p.grp_v, gs, ge, it.x_tile0 * BN);
          pc.end = ge;
          pc.nxt = pc.cur < pc.end ? __ldg(p.grp_v + pc.cur) : 0x7fffffff;
        }
        for (int j = 0; j < it.n_x; ++j) {
          const uint32_t c = cnt + j, b = c % NG;
          const int x0 = kDH ? (it.x_tile0 + j) * BN : j * BN;   // first streamed row of the tile
          // The previous use of this buffer (tile c - NG) must be consumed by the MMA first:
          // that keeps this warp at most one phase ahead on gwritten[b] and fixdone[b], so a
          // parity wait can never match a phase two uses ahead.
          if (!wait_bar_warp(bar_gempty + b, ((c / NG) & 1) ^ 1, wc, wait_tag(3, 8, c))) {
            ok = false;
            break;
          }
          if (pc.nxt < x0 + BN) {
            // positives fall in this tile: wait for the epilogue's sigmoid tile, then subtract 1
            if (!wait_bar_warp(bar_gwritten + b, (c / NG) & 1, wc, wait_tag(3, 6, c))) {
              ok = false;
              break;
            }
            uint8_t* G = sG + b * G_BYTES;
            if (!kDH) fixup_apply<false>(pc, x0 + BN, x0, it.s_row0, G, p.srt_t, p.srt_v, lane);
            else fixup_apply<true>(pc, x0 + BN, x0, it.s_row0, G, p.grp_v, p.grp_t, lane);
            fence_proxy_async_smem();
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_fixdone + b);
        }
        cnt += it.n_x;
      }
    }
  } else if (warp >= kEpiWarp0) {
    // ============================================================ epilogue
    // Warp w reads TMEM lanes 32*(w%4).. (its sub-partition's quarter) and one
    // column slab of each tile: 4 warps per quarter keep the sub-partition's
    // MUFU/FMA pipes fed while others wait on tensor-memory loads.
    constexpr int kSlabs = kNumEpiWarps / 4;
    constexpr int ZC = BN / kSlabs;               // Z columns per warp per tile (32 or 16)
    constexpr int AC = DP / kSlabs;               // accumulator columns per warp (16 .. 64)
    const int q = warp & 3;                       // TMEM lane quarter
    const int slab = (warp - kEpiWarp0) >> 2;     // column slab
    const int row = q * 32 + lane;                // stationary row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t sG_a = smem_u32(sG);
    const float gs = hdr->grad_scale;
    uint32_t cnt = 0, ic = 0;
    bool ok = true;
    for (int i = blockIdx.x; i < n_items && ok; i += gridDim.x, ++ic) {
      const ItemInfo it = item_info<DP, kDH>(i, n_valid, p);
      const int n = it.n_x;
      double item_acc = 0.0;
      for (int j = 0; j < n; ++j) {
        const uint32_t c = cnt + j, bz = c % NZ, bg = c % NG;
        if (!wait_bar_warp(bar_zfull + bz, (c / NZ) & 1, wc, wait_tag(4, 4, c))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t r[ZC];
        tmem_ld<ZC>(tmem_base + lane_base + bz * BN + slab * ZC, r);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_zempty + bz);   // this warp's part of Z[bz] is in registers
        uint32_t pk[ZC / 2];
        float prod = 1.f, tile_mx = 0.f;
#pragma unroll
        for (int e = 0; e < ZC; e += 2) {
          float gpair[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const float z = __uint_as_float(r[e + k]);
            if (kLoss) {
              const float u = ex2_approx(-fabsf(z) * kLog2e);   // e^{-|z|}
              const float pz = 1.f + u;
              prod *= pz;                                        // log1p batched: one lg2 per slab
              tile_mx += fmaxf(z, 0.f);
              if (kGrad) {
                const float rp = rcp_approx(pz);                 // 1 / (1 + e^{-|z|})
                gpair[k] = z >= 0.f ? rp : u * rp;               // sigmoid(z)
              }
            } else {
              gpair[k] = fmaf(0.5f, tanh_approx(0.5f * z), 0.5f);  // sigmoid(z)
            }
          }
          if (kGrad) pk[e >> 1] = pack_bf16x2(gpair[0], gpair[1]);
        }
        if (kGrad) {
          if (!wait_bar_warp(bar_gempty + bg, ((c / NG) & 1) ^ 1, wc, wait_tag(4, 8, c))) {
            ok = false;
            break;
          }
          const int col0 = slab * ZC;
          const uint32_t base = sG_a + bg * G_BYTES + (col0 >> 6) * (kTileM * 128) + row * 128;
          const uint32_t j0 = (col0 & 63) >> 3;
#pragma unroll
          for (int k = 0; k < ZC / 8; ++k)
            st_shared_v4(base + (((j0 + k) ^ (row & 7)) << 4), pk[4 * k], pk[4 * k + 1], pk[4 * k + 2],
                         pk[4 * k + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_gwritten + bg);
        }
        if (kLoss) {
          float tile_l2 = lg2_approx(prod);
          if (j == n - 1) {
            // zero rows of H_c past n_valid give z = 0 exactly: each adds log2(2) = 1 to tile_l2
            const int t0 = j * BN;
            const int lo = slab * ZC, hi = lo + ZC;
            const int pad = hi - max(min(n_valid - t0, hi), lo);
            tile_l2 -= static_cast<float>(pad);
          }
          item_acc += static_cast<double>(tile_mx + tile_l2 * kLn2);
        }
      }
      if (!ok) break;
      if (kLoss) {
        // one partial per (item tile, epilogue warp): no cross-warp barrier, fixed summation order
        double val = (it.s_row0 + row < p.V) ? item_acc : 0.0;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) val += __shfl_xor_sync(0xffffffffu, val, off);
        if (lane == 0) p.loss_part[static_cast<int64_t>(i) * kNumEpiWarps + (warp - kEpiWarp0)] = val;
      }
      if (kGrad) {
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
              float* dst = p.dE + static_cast<int64_t>(v) * p.D + col0;
#pragma unroll
              for (int e = 0; e < 16; e += 4)
                if (col0 + e < p.D)
                  *reinterpret_cast<float4*>(dst + e) =
                      make_float4(__uint_as_float(r[e]) * gs, __uint_as_float(r[e + 1]) * gs,
                                  __uint_as_float(r[e + 2]) * gs, __uint_as_float(r[e + 3]) * gs);
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
