// Full-vocabulary top-k ranking on the tensor cores, for the evaluation of
// "Cut Binary Cross Entropy" (section III-E: a query -- the hidden state of a
// sequence's last non-pad position -- is scored against every item, and Hit@8
// asks whether a held-out item is among the 8 best).  No score ever reaches
// device memory: each logit tile lives in tensor memory until the epilogue has
// folded it into per-thread running top-k lists.
//
// One persistent, warp-specialised kernel (576 threads, one CTA per SM):
//   warp 0      TMA producer: the stationary tile of 128 queries, then a ring of
//               NX streamed item tiles of BN rows;
//   warp 1      TMEM allocator and MMA issuer: logit tile c = Q E_c^T into
//               tensor-memory buffer c mod NZ (in tile order, suspended waits);
//   warps 2-17  epilogue: warp w reads TMEM lanes 32*(w%4).. (one query row per
//               thread) and one of four column slabs of every tile, releases the
//               buffer as soon as every warp has loaded its slab, and inserts
//               its scores into a sorted register list of the kmax best.
// A work item is (query tile, vocabulary split); its per-thread lists are
// written out and k_topk_merge reduces the lists of all splits and slabs of a
// query in a fixed order.  Ranking: descending score, equal scores by ascending
// item id (within a thread the items arrive in ascending id, so a strict
// comparison keeps the lower id first).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include "common.cuh"
#include "ptx_sm100.cuh"
#include "tile_engine.cuh"

namespace cutbce {

template <int DP>
struct TopkCfg {
  static constexpr int BN = DP <= 128 ? 128 : 64;           // items per streamed tile (logit columns)
  static constexpr int NKB = DP / 64;                        // 128-byte column blocks per row
  static constexpr int NX = DP == 64 ? 12 : DP == 128 ? 6 : DP == 192 ? 7 : 5;
  static constexpr int NZ = 512 / BN < 4 ? 512 / BN : 4;     // logit buffers in tensor memory
  static constexpr int SLABS = 4;                            // column slabs (16 epilogue warps / 4 lane quarters)
  static constexpr int ZC = BN / SLABS;                      // columns per epilogue warp per tile
  static constexpr uint32_t S_BYTES = kTileM * DP * 2;
  static constexpr uint32_t X_BYTES = BN * DP * 2;
  static constexpr int NUM_BARS = 2 + 2 * NX + 2 * NZ + 1;
  static constexpr uint32_t SMEM_BYTES = 1024 + S_BYTES + NX * X_BYTES + NUM_BARS * 8 + 16;
  static_assert(ZC <= 32, "one tensor-memory load per warp and tile");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(SMEM_BYTES > 232448 / 2, "one CTA per SM keeps the TMEM allocation uncontended");
};

struct TopkParams {
  int B, V;
  int n_qt;                   // query tiles of 128
  int nsplit;                 // vocabulary splits
  int tiles_per_split;        // item tiles per split
  int n_vtiles;               // ceil(V / BN)
  float* cand_s;              // [n_qt, nsplit, 4 slabs, 128 rows, kmax] scores
  int* cand_i;                // same layout, item ids
  WsHeader* hdr;              // status (bounded waits)
  long long timeout_ns;
};

// Insert (s, v) into a list sorted by descending score whose last entry is
// beaten (s > ls[K-1]); equal scores keep the earlier entry first.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

template <int K>
__device__ __forceinline__ void topk_insert(float (&ls)[K], int (&li)[K], float s, int v) {
#pragma unroll
  for (int k = K - 1; k > 0; --k) {
    const bool shift = s > ls[k - 1];             // the new entry goes above position k-1
    const bool here = !shift && s > ls[k];        // ... or exactly at position k
    if (shift) {
      ls[k] = ls[k - 1];
      li[k] = li[k - 1];
    } else if (here) {
      ls[k] = s;
      li[k] = v;
    }
  }
  if (s > ls[0]) {
    ls[0] = s;
    li[0] = v;
  }
}

template <int DP, int KMAX>
__global__ void __launch_bounds__(kTileThreads, 1)
    k_topk(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmE, TopkParams p) {
  using Cfg = TopkCfg<DP>;
  constexpr int BN = Cfg::BN, NKB = Cfg::NKB, NX = Cfg::NX, NZ = Cfg::NZ, ZC = Cfg::ZC;
  constexpr uint32_t S_BYTES = Cfg::S_BYTES, X_BYTES = Cfg::X_BYTES;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sX = sQ + S_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sX + NX * X_BYTES);
  uint64_t* bar_sfull = bars + 0;           // query tile landed (TMA)
  uint64_t* bar_sempty = bars + 1;          // query tile no longer read (MMA commit)
  uint64_t* bar_xfull = bars + 2;           // [NX] item tile landed
  uint64_t* bar_xempty = bar_xfull + NX;    // [NX] item tile free (MMA commit)
  uint64_t* bar_zfull = bar_xempty + NX;    // [NZ] logit tile ready (MMA commit)
  uint64_t* bar_zfree = bar_zfull + NZ;     // [NZ] logit tile loaded by every epilogue warp
  uint64_t* bar_drain = bar_zfree + NZ;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NUM_BARS);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  WsHeader* hdr = p.hdr;
  const int n_items = p.n_qt * p.nsplit;
  if (static_cast<int>(blockIdx.x) >= n_items) return;

  if (threadIdx.x == 0) {
    mbar_init(bar_sfull, 1);
    mbar_init(bar_sempty, 1);
    for (int s = 0; s < NX; ++s) {
      mbar_init(bar_xfull + s, 1);
      mbar_init(bar_xempty + s, 1);
    }
    for (int b = 0; b < NZ; ++b) {
      mbar_init(bar_zfull + b, 1);
      mbar_init(bar_zfree + b, kNumEpiWarps);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmE);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtx wc{abort_flag, hdr, p.timeout_ns};

  // work item i: query tile i / nsplit, vocabulary split i % nsplit
  auto tile_range = [&](int i, int& qt, int& t0, int& nt) {
    qt = i / p.nsplit;
    const int s = i - qt * p.nsplit;
    t0 = s * p.tiles_per_split;
    nt = max(0, min(p.tiles_per_split, p.n_vtiles - t0));
  };

  if (warp == 0) {
    // ============================================================ TMA producer
    if (lane == 0) {
      uint32_t ic = 0, xc = 0;
      bool ok = true;
      for (int i = blockIdx.x; i < n_items && ok; i += gridDim.x, ++ic) {
        int qt, t0, nt;
        tile_range(i, qt, t0, nt);
        if (!wait_bar(bar_sempty, (ic & 1) ^ 1, wc, wait_tag(1, 1, ic))) break;
        mbar_arrive_expect_tx(bar_sfull, S_BYTES);
#pragma unroll
        for (int kb = 0; kb < NKB; ++kb) tma_load_2d(sQ + kb * (kTileM * 128), &tmQ, kb * 64, qt * kTileM, bar_sfull);
        for (int j = 0; j < nt; ++j, ++xc) {
          const uint32_t st = xc % NX;
          if (!wait_bar(bar_xempty + st, ((xc / NX) & 1) ^ 1, wc, wait_tag(1, 3, xc))) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar_xfull + st, X_BYTES);
#pragma unroll
          for (int kb = 0; kb < NKB; ++kb)
            tma_load_2d(sX + st * X_BYTES + kb * (BN * 128), &tmE, kb * 64, (t0 + j) * BN, bar_xfull + st);
        }
        if (!ok) ++ic;
      }
      // wait (bounded) for every copy this thread issued to land
      if (ic > 0) wait_bar_drain(bar_sfull, (ic - 1) & 1, p.timeout_ns);
      for (uint32_t st = 0; st < NX; ++st) {
        const uint32_t issued = xc > st ? (xc - st + NX - 1) / NX : 0;
        if (issued > 0) wait_bar_drain(bar_xfull + st, (issued - 1) & 1, p.timeout_ns);
      }
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(kTileM, BN, false, false);
    const uint64_t dQ = smem_desc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t dX = smem_desc_sw128(smem_u32(sX), 16, 1024);
    uint32_t ic = 0, c = 0;
    bool ok = true;
    for (int i = blockIdx.x; i < n_items && ok; i += gridDim.x, ++ic) {
      int qt, t0, nt;
      tile_range(i, qt, t0, nt);
      if (!wait_bar_warp(bar_sfull, ic & 1, wc, wait_tag(2, 0, ic))) break;
      for (int j = 0; j < nt; ++j, ++c) {
        const uint32_t st = c % NX, zb = c % NZ;
        if (!wait_bar_warp(bar_xfull + st, (c / NX) & 1, wc, wait_tag(2, 1, c)) ||
            !wait_bar_warp(bar_zfree + zb, ((c / NZ) & 1) ^ 1, wc, wait_tag(2, 2, c))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int ks = 0; ks < DP / 16; ++ks) {
            const uint32_t off = static_cast<uint32_t>((ks >> 2) * (kTileM * 8) + (ks & 3) * 2);
            const uint32_t xoff = static_cast<uint32_t>(st * (X_BYTES >> 4) + (ks >> 2) * (BN * 8) + (ks & 3) * 2);
            umma_bf16(tmem_base + zb * BN, dQ + off, dX + xoff, idesc, ks > 0 ? 1u : 0u);
          }
          umma_commit(bar_zfull + zb);
          umma_commit(bar_xempty + st);
          if (j + 1 == nt) umma_commit(bar_sempty);
        }
        __syncwarp();
      }
      if (ok && nt == 0) {
        // an empty split: the query tile is released at once
        if (elect_one()) umma_commit(bar_sempty);
        __syncwarp();
      }
    }
    if (elect_one()) umma_commit(bar_drain);
    __syncwarp();
    if (lane == 0) wait_bar_drain(bar_drain, 0, p.timeout_ns);
    __syncwarp();
  } else if (warp >= kEpiWarp0) {
    // ============================================================ epilogue
    const int ew = warp - kEpiWarp0;
    const int q = warp & 3;
    const int slab = ew >> 2;
    const int row = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    uint32_t c = 0;
    for (int i = blockIdx.x; i < n_items; i += gridDim.x) {
      int qt, t0, nt;
      tile_range(i, qt, t0, nt);
      float ls[KMAX];
      int li[KMAX];
#pragma unroll
      for (int k = 0; k < KMAX; ++k) {
        ls[k] = -INFINITY;
        li[k] = -1;
      }
      bool ok = true;
      for (int j = 0; j < nt; ++j, ++c) {
        const uint32_t zb = c % NZ;
        if (!wait_bar_warp(bar_zfull + zb, (c / NZ) & 1, wc, wait_tag(4, 4, c))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t r[ZC];
        tmem_ld<ZC>(tmem_base + lane_base + zb * BN + slab * ZC, r);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_zfree + zb);
        const int v0 = (t0 + j) * BN + slab * ZC;
        const int valid_cols = min(ZC, p.V - v0);     // item rows past V are zero-filled: excluded
        if (valid_cols < ZC) {
#pragma unroll
          for (int e = 0; e < ZC; ++e)
            if (e >= valid_cols) r[e] = __float_as_uint(-INFINITY);
        }
        // the tile's best score first (three-input max): once the lists have
        // filled, almost no tile holds a score that beats this thread's k-th,
        // and the tile then costs ZC / 2 max operations and one branch
        float m = __uint_as_float(r[0]);
#pragma unroll
        for (int e = 1; e + 1 < ZC; e += 2) m = fmax3(m, __uint_as_float(r[e]), __uint_as_float(r[e + 1]));
        if (ZC % 2 == 0) m = fmaxf(m, __uint_as_float(r[ZC - 1]));
        if (m > ls[KMAX - 1]) {
#pragma unroll
          for (int e = 0; e < ZC; ++e) {
            const float s = __uint_as_float(r[e]);
            if (s > ls[KMAX - 1]) topk_insert<KMAX>(ls, li, s, v0 + e);
          }
        }
      }
      if (!ok) break;
      const int64_t base = ((static_cast<int64_t>(qt) * p.nsplit + (i - qt * p.nsplit)) * 4 + slab) * kTileM + row;
#pragma unroll
      for (int k = 0; k < KMAX; ++k) {
        p.cand_s[base * KMAX + k] = ls[k];
        p.cand_i[base * KMAX + k] = li[k];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// Merge of the candidate lists (each of kmax entries, sorted) of one query, by
// descending score and ascending id.  Lane steps: each lane keeps the best
// kmax of the lists it reads; then k rounds of a warp-wide argmax, the lane
// holding the best head giving it up.  Empty entries (id -1) are never chosen.
template <int KMAX>
__device__ __forceinline__ void lane_take_lists(const float* __restrict__ cand_s, const int* __restrict__ cand_i,
                                                int qt, int row, int nlists, int l0, int lstep, float (&ls)[KMAX],
                                                int (&li)[KMAX]) {
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    ls[j] = -INFINITY;
    li[j] = 0x7fffffff;
  }
  for (int l = l0; l < nlists; l += lstep) {
    const int64_t base = ((static_cast<int64_t>(qt) * nlists + l) * kTileM + row) * KMAX;
    for (int j = 0; j < KMAX; ++j) {
      const int v = cand_i[base + j];
      if (v < 0) break;
      const float sc = cand_s[base + j];
      // insert by (score desc, id asc): a later list may hold a lower id with an equal score
      int pos = KMAX;
      for (int t = KMAX - 1; t >= 0; --t)
        if (sc > ls[t] || (sc == ls[t] && v < li[t])) pos = t;
      if (pos < KMAX) {
        for (int t = KMAX - 1; t > pos; --t) {
          ls[t] = ls[t - 1];
          li[t] = li[t - 1];
        }
        ls[pos] = sc;
        li[pos] = v;
      }
    }
  }
}

// k rounds over the warp's per-lane sorted lists; lane 0 writes round r to
// out_s[r], out_i[r] (id 0x7fffffff: no entry).
template <int KMAX>
__device__ __forceinline__ void warp_best_k(const float (&ls)[KMAX], const int (&li)[KMAX], int k, float* out_s,
                                            int* out_i) {
  const int lane = threadIdx.x & 31;
  int head = 0;
  for (int r = 0; r < k; ++r) {
    float hs = -INFINITY;
    int hi = 0x7fffffff;
#pragma unroll
    for (int t = 0; t < KMAX; ++t)
      if (t == head) {
        hs = ls[t];
        hi = li[t];
      }
    float bs = hs;
    int bi = hi, bl = lane;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, bs, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      const int ol = __shfl_xor_sync(0xffffffffu, bl, off);
      if (os > bs || (os == bs && (oi < bi || (oi == bi && ol < bl)))) {
        bs = os;
        bi = oi;
        bl = ol;
      }
    }
    if (lane == bl && head < KMAX) ++head;
    if (lane == 0) {
      out_s[r] = bs;
      out_i[r] = bi;
    }
  }
}

// One warp per query (few lists per query: many queries).
template <int KMAX>
__global__ void __launch_bounds__(256) k_topk_merge(const float* __restrict__ cand_s, const int* __restrict__ cand_i,
                                                     int B, int nsplit, int k, int32_t* __restrict__ ids,
                                                     float* __restrict__ scores) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= B) return;
  const int qt = warp / kTileM, row = warp - qt * kTileM;
  float ls[KMAX];
  int li[KMAX];
  lane_take_lists<KMAX>(cand_s, cand_i, qt, row, nsplit * 4, lane, 32, ls, li);
  int32_t* oi = ids + static_cast<int64_t>(warp) * k;
  warp_best_k<KMAX>(ls, li, k, scores + static_cast<int64_t>(warp) * k, oi);
  __syncwarp();
  if (lane < k && oi[lane] == 0x7fffffff) oi[lane] = -1;
}

// One block of 8 warps per query (many lists per query: few queries, many
// vocabulary splits): warp w takes lists w * 32 + lane, + 256, ...; warp 0 then
// merges the 8 warps' k best the same way.
template <int KMAX>
__global__ void __launch_bounds__(256) k_topk_merge_block(const float* __restrict__ cand_s,
                                                           const int* __restrict__ cand_i, int B, int nsplit, int k,
                                                           int32_t* __restrict__ ids, float* __restrict__ scores) {
  __shared__ float ws[8][KMAX];
  __shared__ int wi[8][KMAX];
  const int q = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = q / kTileM, row = q - qt * kTileM;
  float ls[KMAX];
  int li[KMAX];
  lane_take_lists<KMAX>(cand_s, cand_i, qt, row, nsplit * 4, warp * 32 + lane, 256, ls, li);
  warp_best_k<KMAX>(ls, li, k, ws[warp], wi[warp]);
  __syncthreads();
  if (warp != 0) return;
#pragma unroll
  for (int t = 0; t < KMAX; ++t) {
    const bool have = lane < 8 && t < k;
    ls[t] = have ? ws[lane < 8 ? lane : 0][t] : -INFINITY;
    li[t] = have ? wi[lane < 8 ? lane : 0][t] : 0x7fffffff;
  }
  int32_t* oi = ids + static_cast<int64_t>(q) * k;
  warp_best_k<KMAX>(ls, li, k, scores + static_cast<int64_t>(q) * k, oi);
  __syncwarp();
  if (lane < k && oi[lane] == 0x7fffffff) oi[lane] = -1;
}

// hits[b] = 1 if a target id (>= 0) of query b is among its k ids.
__global__ void k_hit_at_k(const int32_t* __restrict__ ids, int B, int k, const int32_t* __restrict__ targets, int L,
                           int32_t* __restrict__ hits) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  int hit = 0;
  for (int l = 0; l < L && !hit; ++l) {
    const int t = targets[static_cast<int64_t>(b) * L + l];
    if (t < 0) continue;
    for (int j = 0; j < k; ++j)
      if (ids[static_cast<int64_t>(b) * k + j] == t) hit = 1;
  }
  hits[b] = hit;
}

}  // namespace cutbce
