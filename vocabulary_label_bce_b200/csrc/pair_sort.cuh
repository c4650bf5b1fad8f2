// Order of the (position, item) pairs for the item-owned tensor-core pass:
// grouped by item tile (128 consecutive items, one stationary tile of that
// pass), and within a group in ascending compacted position, so that the
// epilogue warps of a CTA walk their item tile's positives with one forward
// cursor as the position tiles stream by.
//
// The pairs are produced in (position, item) order; a stable LSD radix sort on
// the item-tile index keeps that order inside each group.  The value carried
// along packs the item's row within its tile and the compacted position:
// (v mod 128) << 24 | t.  Every pair is unique, so the order is deterministic.
#pragma once
#include <cstdint>
#include "common.cuh"

namespace cutbce {

constexpr int kRadixThreads = 256;
constexpr int kPairPosBits = 24;                 // compacted positions below 2^24 fit the packed value
constexpr int kRadixTile = 4096;                 // pairs per block
constexpr int kRadixRounds = kRadixTile / kRadixThreads;

__device__ __forceinline__ int item_digit(int v, int shift) { return (v >> shift) & 255; }

// Per-block digit histogram, stored digit-major: ghist[d * nblk + blk].
__global__ void __launch_bounds__(kRadixThreads) k_radix_hist(const int* __restrict__ keys, const WsHeader* hdr,
                                                              int shift, int nblk, int* __restrict__ ghist) {
  __shared__ int h[256];
  h[threadIdx.x] = 0;
  __syncthreads();
  const int n = hdr->n_pairs;
  const int base = blockIdx.x * kRadixTile;
  for (int i = threadIdx.x; i < kRadixTile; i += kRadixThreads) {
    const int idx = base + i;
    if (idx < n) atomicAdd(&h[item_digit(keys[idx], shift)], 1);
  }
  __syncthreads();
  ghist[threadIdx.x * nblk + blockIdx.x] = h[threadIdx.x];
}

// In-place exclusive scan of `total` ints in one block.
__global__ void __launch_bounds__(1024) k_exclusive_scan(int* __restrict__ a, int total) {
  __shared__ int warp_sum[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  constexpr int kItems = 4;
  for (int base = 0; base < total; base += 1024 * kItems) {
    int loc[kItems];
    int s = 0;
#pragma unroll
    for (int i = 0; i < kItems; ++i) {
      const int idx = base + tid * kItems + i;
      loc[i] = idx < total ? a[idx] : 0;
      s += loc[i];
    }
    int inc = s;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += o;
    }
    if (lane == 31) warp_sum[wid] = inc;
    __syncthreads();
    if (wid == 0) {
      const int w = warp_sum[lane];
      int wi = w;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, wi, off);
        if (lane >= off) wi += o;
      }
      warp_sum[lane] = wi - w;
    }
    __syncthreads();
    int run = carry + warp_sum[wid] + inc - s;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kItems; ++i) {
      const int idx = base + tid * kItems + i;
      if (idx < total) a[idx] = run;
      run += loc[i];
    }
    if (tid == 1023) carry = run;
    __syncthreads();
  }
}

// Stable scatter by digit: within a block, rounds of 256 pairs in index order;
// within a round, ranks follow (warp, lane) order.
__global__ void __launch_bounds__(kRadixThreads) k_radix_scatter(const int* __restrict__ keys_in,
                                                                 const int* __restrict__ vals_in,
                                                                 int* __restrict__ keys_out,
                                                                 int* __restrict__ vals_out, const WsHeader* hdr,
                                                                 int shift, int nblk,
                                                                 const int* __restrict__ goff) {
  constexpr int kWarps = kRadixThreads / 32;
  __shared__ int base[256];
  __shared__ int wcnt[kWarps][256];
  __shared__ int wpre[kWarps][256];
  __shared__ int rtot[256];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = hdr->n_pairs;
  base[tid] = goff[tid * nblk + blockIdx.x];
#pragma unroll
  for (int w = 0; w < kWarps; ++w) wcnt[w][tid] = 0;
  __syncthreads();
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int r = 0; r < kRadixRounds; ++r) {
    const int idx = blockIdx.x * kRadixTile + r * kRadixThreads + tid;
    const bool valid = idx < n;
    const int key = valid ? keys_in[idx] : 0;
    const int val = valid ? vals_in[idx] : 0;
    const int d = valid ? item_digit(key, shift) : 256;
    const unsigned peers = __match_any_sync(0xffffffffu, d);
    const int rank = __popc(peers & lt_mask);
    if (valid && rank == 0) wcnt[warp][d] = __popc(peers);
    __syncthreads();
    {
      int run = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const int c = wcnt[w][tid];
        wpre[w][tid] = run;
        run += c;
      }
      rtot[tid] = run;
    }
    __syncthreads();
    if (valid) {
      const int pos = base[d] + wpre[warp][d] + rank;
      keys_out[pos] = key;
      vals_out[pos] = val;
    }
    __syncthreads();
    base[tid] += rtot[tid];
#pragma unroll
    for (int w = 0; w < kWarps; ++w) wcnt[w][tid] = 0;
    __syncthreads();
  }
}

// Sort input: key = item tile v / 128, value = (v mod 128) << 24 | t.
__global__ void k_pair_keys(const int* __restrict__ pair_v, const int* __restrict__ pair_t, const WsHeader* hdr,
                            int* __restrict__ keys, int* __restrict__ vals) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= hdr->n_pairs) return;
  const int v = pair_v[i];
  keys[i] = v >> 7;
  vals[i] = ((v & 127) << kPairPosBits) | pair_t[i];
}

// off[k] = first index of the sorted pairs whose key is >= k, for k in [0, nkeys];
// key k owns [off[k], off[k+1]).
__global__ void k_key_offsets(const int* __restrict__ sorted_v, const WsHeader* hdr, int nkeys,
                              int* __restrict__ csc_off) {
  const int v = blockIdx.x * blockDim.x + threadIdx.x;
  if (v > nkeys) return;
  int lo = 0, hi = hdr->n_pairs;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (sorted_v[mid] < v) lo = mid + 1;
    else hi = mid;
  }
  csc_off[v] = lo;
}

}  // namespace cutbce
