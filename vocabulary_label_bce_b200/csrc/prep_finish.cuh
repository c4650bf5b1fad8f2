// CUDA-core kernels around the tensor-core engine:
//   prep   -- apply the mask and the id rules, compact the valid rows, build the
//             (position, item) pair lists, sum the sparse target correction;
//   finish -- reduce the dH partials in a fixed order, scale, form the loss;
//   simt   -- a plain fp32 path for fp32 inputs (small correctness cases).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "common.cuh"

namespace cutbce {

__device__ __forceinline__ void set_status(int* status, int code) { atomicCAS(status, 0, code); }

// ------------------------------------------------------------------ prep: rows
// A position is valid iff its mask entry is nonzero and its weight (when
// per-position weights are given) is nonzero: a zero weight is padding.
__device__ __forceinline__ bool position_valid(const uint8_t* __restrict__ mask, const float* __restrict__ weights,
                                               int t) {
  return (mask == nullptr || mask[t] != 0) && (weights == nullptr || weights[t] != 0.f);
}

// One thread per position t.  A valid row's ids become its positive set P_t
// (section III-B: sparse [B,N,L] ids, no multi-hot tensor): -1 slots dropped,
// repeats collapsed (y is 0/1), sorted ascending.  Ids of masked rows are
// ignored.  With a vocabulary shard, ids are global: an id in [-1, V_total) but
// outside [v_off, v_off + V) belongs to another shard and is dropped, and the
// kept ids are made shard-local.
__global__ void k_prep_rows(const int32_t* __restrict__ targets, const uint8_t* __restrict__ mask,
                            const float* __restrict__ weights, int T, int K, int V, int64_t v_off, int64_t V_total,
                            int* __restrict__ ids_out, int* __restrict__ row_cnt, WsHeader* hdr) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  if (!position_valid(mask, weights, t)) {
    row_cnt[t] = 0;
    return;
  }
  int buf[kMaxK];
  int n = 0;
  bool bad = false;
  const int32_t* row = targets + static_cast<int64_t>(t) * K;
  for (int k = 0; k < K; ++k) {
    const int gid = row[k];
    if (gid == -1) continue;
    if (gid < -1 || gid >= V_total) {
      bad = true;
      continue;
    }
    if (gid < v_off || gid >= v_off + V) continue;     // another shard's item
    const int id = static_cast<int>(gid - v_off);
    int pos = n;
    while (pos > 0 && buf[pos - 1] > id) --pos;
    if (pos > 0 && buf[pos - 1] == id) continue;
    for (int j = n; j > pos; --j) buf[j] = buf[j - 1];
    buf[pos] = id;
    ++n;
  }
  if (bad) set_status(&hdr->status, kErrTargetRange);
  int* dst = ids_out + static_cast<int64_t>(t) * K;
  for (int j = 0; j < n; ++j) dst[j] = buf[j];
  row_cnt[t] = n;
}

// ------------------------------------------------------------------ prep: scan
// One block.  Exclusive scans over t of valid[t] (compacted row index c) and of
// |P_t| (pair offsets), then the normalisation s and the gradient scale g*s
// (V here is the whole vocabulary, for the per-element mean).
constexpr int kScanThreads = 1024;
constexpr int kScanItems = 8;

__global__ void __launch_bounds__(kScanThreads) k_prep_scan(const uint8_t* __restrict__ mask,
                                                            const float* __restrict__ weights,
                                                            const int* __restrict__ row_cnt, int T, int64_t V,
                                                            int reduction, const float* __restrict__ grad_loss,
                                                            int* __restrict__ cidx, int* __restrict__ orig,
                                                            int* __restrict__ row_ptr, WsHeader* hdr) {
  __shared__ int warp_v[32], warp_c[32];
  __shared__ int carry_v, carry_c;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid == 0) {
    carry_v = 0;
    carry_c = 0;
  }
  __syncthreads();
  for (int base = 0; base < T; base += kScanThreads * kScanItems) {
    int vloc[kScanItems], cloc[kScanItems];
    int vs = 0, cs = 0;
#pragma unroll
    for (int i = 0; i < kScanItems; ++i) {
      const int t = base + tid * kScanItems + i;
      const int v = (t < T && position_valid(mask, weights, t)) ? 1 : 0;
      const int c = (t < T) ? row_cnt[t] : 0;
      vloc[i] = v;
      cloc[i] = c;
      vs += v;
      cs += c;
    }
    int vi = vs, ci = cs;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int nv = __shfl_up_sync(0xffffffffu, vi, off);
      const int nc = __shfl_up_sync(0xffffffffu, ci, off);
      if (lane >= off) {
        vi += nv;
        ci += nc;
      }
    }
    if (lane == 31) {
      warp_v[wid] = vi;
      warp_c[wid] = ci;
    }
    __syncthreads();
    if (wid == 0) {
      int a = warp_v[lane], b = warp_c[lane];
      int ai = a, bi = b;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int na = __shfl_up_sync(0xffffffffu, ai, off);
        const int nb = __shfl_up_sync(0xffffffffu, bi, off);
        if (lane >= off) {
          ai += na;
          bi += nb;
        }
      }
      warp_v[lane] = ai - a;
      warp_c[lane] = bi - b;
    }
    __syncthreads();
    int vex = carry_v + warp_v[wid] + vi - vs;
    int cex = carry_c + warp_c[wid] + ci - cs;
    __syncthreads();  // everyone has read carry_*
#pragma unroll
    for (int i = 0; i < kScanItems; ++i) {
      const int t = base + tid * kScanItems + i;
      if (t < T) {
        if (vloc[i]) {
          cidx[t] = vex;
          orig[vex] = t;
          row_ptr[vex] = cex;
          ++vex;
        } else {
          cidx[t] = -1;
        }
        cex += cloc[i];
      }
    }
    if (tid == kScanThreads - 1) {
      carry_v = vex;
      carry_c = cex;
    }
    __syncthreads();
  }
  if (tid == 0) {
    const int nv = carry_v;
    row_ptr[nv] = carry_c;
    hdr->n_valid = nv;
    hdr->n_pairs = carry_c;
    double s = 0.0;
    if (nv > 0) {
      if (reduction == kMeanValidPositions) s = 1.0 / nv;
      else if (reduction == kSum) s = 1.0;
      else s = 1.0 / (static_cast<double>(nv) * static_cast<double>(V));
    }
    const double g = grad_loss ? static_cast<double>(*grad_loss) : 1.0;
    hdr->loss_scale = s;
    hdr->grad_scale = static_cast<float>(g * s);
  }
}

// ------------------------------------------------------------------ prep: gather
// One warp per compacted row c in [0, Tpad).  Copies h_t into the compacted,
// zero-padded H_c (rows >= n_valid are zero so padded tiles contribute exactly
// nothing to any gradient; with bf16 inputs the row is stored halved, h_t / 2,
// which is exact, so that the tensor-core tiles hold z / 2: the argument of the
// tanh the element math takes), writes the pair lists and, with per-position
// weights, the compacted weights (0 for the padded rows), and sums the sparse
// target correction sum_{v in P_t} w_t h_t . e_v of Eq. (2) in fp32 per pair, in
// a fixed order, into one double per block.
// bf16 H_c (the tensor-core path) holds h / 2; fp32 H_c (the SIMT path) holds h.
// `mode` selects the work: kGatherRows (H_c, the compacted weights and the pair
// lists, which need no E), kGatherCorrection (the correction partials, which
// read E), or both.  Split in two, the same blocks sum the same pairs in the
// same order: the partials are bit-identical to one launch doing both.
template <typename TIn>
constexpr bool kHalveHc = sizeof(TIn) == 2;
constexpr int kGatherRows = 1;
constexpr int kGatherCorrection = 2;

template <typename TIn>
__global__ void __launch_bounds__(256) k_prep_gather(const TIn* __restrict__ H, const TIn* __restrict__ E,
                                                     int D, int DP, int K, int64_t Tpad,
                                                     const int* __restrict__ orig, const int* __restrict__ ids,
                                                     const int* __restrict__ row_cnt,
                                                     const int* __restrict__ row_ptr, const WsHeader* hdr,
                                                     const float* __restrict__ weights, float* __restrict__ wc,
                                                     TIn* __restrict__ Hc, int* __restrict__ pair_t,
                                                     int* __restrict__ pair_v, double* __restrict__ corr_part,
                                                     int mode) {
  const bool rows = (mode & kGatherRows) != 0, corr = (mode & kGatherCorrection) != 0;
  __shared__ double wsum[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t c = static_cast<int64_t>(blockIdx.x) * 8 + warp;
  const int nv = hdr->n_valid;
  double acc = 0.0;
  if (c < Tpad) {
    TIn* dst = Hc + c * DP;
    if (rows && wc != nullptr && lane == 0) wc[c] = c < nv ? weights[orig[c]] : 0.f;
    if (c < nv) {
      const int t = orig[c];
      const double wt = weights != nullptr ? static_cast<double>(weights[t]) : 1.0;
      const TIn* src = H + static_cast<int64_t>(t) * D;
      if (rows)
        for (int d = lane; d < DP; d += 32)
          dst[d] = d < D ? (kHalveHc<TIn> ? TIn(0.5f * static_cast<float>(src[d])) : src[d]) : TIn(0.0f);
      const int p0 = row_ptr[c];
      const int n = row_cnt[t];
      for (int k = 0; k < n; ++k) {
        const int v = ids[static_cast<int64_t>(t) * K + k];
        if (rows && lane == 0) {
          pair_t[p0 + k] = static_cast<int>(c);
          pair_v[p0 + k] = v;
        }
        if (corr) {
          const TIn* e = E + static_cast<int64_t>(v) * D;
          float z = 0.f;
          for (int d = lane; d < D; d += 32) z = fmaf(static_cast<float>(src[d]), static_cast<float>(e[d]), z);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
          acc += wt * static_cast<double>(z);
        }
      }
    } else if (rows) {
      for (int d = lane; d < DP; d += 32) dst[d] = TIn(0.0f);
    }
  }
  if (!corr) return;
  if (lane == 0) wsum[warp] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < 8; ++w) s += wsum[w];
    corr_part[blockIdx.x] = s;
  }
}

// ------------------------------------------------------------------ prep: column sums
// The linear half of the dense loss.  With max(z, 0) = z / 2 + |z| / 2,
//   sum_{t valid} w_t sum_{v < V} max(z_tv, 0)
//     = 1/2 (sum_t w_t h_t) . (sum_v e_v)  +  sum_{t, v} w_t |z_tv| / 2,
// so the tile kernels accumulate only |z / 2| (their tiles hold z / 2), and the
// first term is one dot product of two column sums.  Blocks [0, nbE) sum fixed
// slices of the rows of E, blocks [nbE, nbE + nbH) fixed slices of the
// compacted H (which holds h / 2, rows past n_valid zero) times the compacted
// weights; each block writes one fp64 partial per column.  A launch covers the
// logical blocks [first_block, first_block + gridDim.x); with `final`, the last
// of its blocks to finish (a ticket in the header, which each call clears) sums
// all nbE + nbH partials in a fixed order and writes the dot product to the
// header.  Eight bf16 columns per 16-byte load; D is a multiple of 8.
constexpr int kColSumThreads = 256;
constexpr int kColSumBlocksE = 444;
constexpr int kColSumBlocksHMax = 64;

__global__ void __launch_bounds__(kColSumThreads) k_col_sums(const __nv_bfloat16* __restrict__ E, int64_t V,
                                                              const __nv_bfloat16* __restrict__ Hc,
                                                              const float* __restrict__ wc, int64_t Tpad, int D,
                                                              int DP, int nbE, int nbH, double* __restrict__ part,
                                                              WsHeader* hdr, int first_block, int final) {
  __shared__ double red[kColSumThreads * 8];
  __shared__ int ticket;
  const int b = static_cast<int>(blockIdx.x) + first_block;
  const bool isE = b < nbE;
  const int64_t rows = isE ? V : Tpad;
  const int64_t stride = isE ? D : DP;
  const __nv_bfloat16* src = isE ? E : Hc;
  const int nb = isE ? nbE : nbH;
  const int bb = isE ? b : b - nbE;
  const int64_t per = (rows + nb - 1) / nb;
  const int64_t r0 = static_cast<int64_t>(bb) * per, r1 = min(rows, r0 + per);
  const int tpr = D / 8;                       // threads per row, 8 columns each
  const int rpp = kColSumThreads / tpr;        // rows per pass
  const int cg = threadIdx.x % tpr, rs = threadIdx.x / tpr;
  double acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = 0.0;
  if (rs < rpp) {
#pragma unroll 4
    for (int64_t r = r0 + rs; r < r1; r += rpp) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src + r * stride) + cg);
      const double w = (!isE && wc != nullptr) ? static_cast<double>(__ldg(wc + r)) : 1.0;
      const uint32_t u[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc[2 * k] += w * static_cast<double>(__uint_as_float(u[k] << 16));
        acc[2 * k + 1] += w * static_cast<double>(__uint_as_float(u[k] & 0xFFFF0000u));
      }
    }
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) red[k * kColSumThreads + threadIdx.x] = rs < rpp ? acc[k] : 0.0;
  __syncthreads();
  // column d = 8 cg + k: the rpp row groups in order
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    const int g = d / 8, k = d % 8;
    double sum = 0.0;
    for (int q = 0; q < rpp; ++q) sum += red[k * kColSumThreads + q * tpr + g];
    part[static_cast<int64_t>(b) * D + d] = sum;
  }
  if (!final) return;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) ticket = atomicAdd(&hdr->colsum_count, 1);
  __syncthreads();
  if (ticket != static_cast<int>(gridDim.x) - 1) return;
  __threadfence();
  // the last block: thread (d, j) sums every np-th partial from j on, the np
  // sums of a column are then added in order (np = 256 / D threads per column)
  const int np = kColSumThreads / D;
  const int d = threadIdx.x % D, j = threadIdx.x / D;
  double se = 0.0, sh = 0.0;
  if (j < np) {
#pragma unroll 8
    for (int i = j; i < nbE; i += np) se += __ldcg(part + static_cast<int64_t>(i) * D + d);
#pragma unroll 8
    for (int i = j; i < nbH; i += np) sh += __ldcg(part + static_cast<int64_t>(nbE + i) * D + d);
  }
  red[threadIdx.x] = j < np ? se : 0.0;
  red[kColSumThreads + threadIdx.x] = j < np ? sh : 0.0;
  __syncthreads();
  double prod = 0.0;
  if (threadIdx.x < D) {
    double e = 0.0, h = 0.0;
    for (int q = 0; q < np; ++q) {
      e += red[q * D + threadIdx.x];
      h += red[kColSumThreads + q * D + threadIdx.x];
    }
    prod = e * h;
  }
  __syncthreads();
  // fixed tree over the columns
  red[threadIdx.x] = prod;
  __syncthreads();
  for (int st = kColSumThreads / 2; st > 0; st >>= 1) {
    if (threadIdx.x < st) red[threadIdx.x] += red[threadIdx.x + st];
    __syncthreads();
  }
  if (threadIdx.x == 0) hdr->lin = red[0];
}

// ------------------------------------------------------------------ finish
// dH[t, d] = g*s * sum_{split} partial[split][c(t)][d] in split order (0 for
// masked rows).  The loss = s * (dense - correction) is summed in two levels:
// every block reduces a fixed slice of the partials, and the last block to
// finish (an atomic ticket in the workspace header, which each call clears)
// sums the block results in block order, so the order is fixed.
constexpr int kFinishThreads = 256;

__device__ double block_sum_fixed(double v, double* red) {
  // deterministic: contiguous per-thread values, then a fixed tree
  red[threadIdx.x] = v;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  const double r = red[0];
  __syncthreads();
  return r;
}

struct FinishParams {
  int T, D, DP, S, V;
  int64_t Tpad;
  const int* cidx;            // [T] compacted row of each position, -1 if masked
  const float* dh_part;       // [S, Tpad, DP] dH partials of the vocabulary splits
  void* dH;                   // [T, D] output (fp32, or bf16 with dh_bf16), or null
  int dh_bf16;                // dH is written as bf16 (round to nearest even)
  int dh_acc;                 // dH += the gradient instead of dH = the gradient
  const float* weights;       // [T] per-position weights (row t of dH scaled by w_t), or null
  const double* loss_part;    // dense loss partials
  int n_loss_part;            // their number, or (with loss_pos_splits > 0) computed from n_valid
  int loss_pos_splits;        // > 0: the partials are per position-owned work item, splits x ceil(n_valid/128)
  const double* corr_part;    // sparse correction partials
  int n_corr_part;
  double* blk_part;           // [2 * gridDim.x] per-block loss sums
  double* loss;               // output, or null
  const int2* met_part;       // [met_slots, Tpad] (count of x > 0, TP) partials, or null
  int met_slots;
  int32_t* metrics;           // [T, 4] output TP, FP, FN, TN, or null
  const int* row_cnt;         // [T] distinct positives of each position
  int use_lin;                // add the linear half of the dense loss (hdr->lin, from k_col_sums)
  WsHeader* hdr;
};

__global__ void __launch_bounds__(kFinishThreads) k_finish(const FinishParams f) {
  __shared__ double red[kFinishThreads];
  __shared__ int ticket;
  const float gs = f.hdr->grad_scale;
  const int T = f.T, D = f.D;
  if (f.dH != nullptr) {
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx < static_cast<int64_t>(T) * D) {
      const int t = static_cast<int>(idx / D);
      const int d = static_cast<int>(idx - static_cast<int64_t>(t) * D);
      const int c = f.cidx[t];
      float out = 0.f;
      if (c >= 0) {
        // the partials of the S splits added in split order; their loads are
        // issued eight at a time so that they are in flight together
        const float* src = f.dh_part + static_cast<int64_t>(c) * f.DP + d;
        const int64_t stride = f.Tpad * f.DP;
        float acc = 0.f;
        int s = 0;
        for (; s + 8 <= f.S; s += 8) {
          float v[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) v[k] = __ldg(src + (s + k) * stride);
#pragma unroll
          for (int k = 0; k < 8; ++k) acc += v[k];
        }
        for (; s < f.S; ++s) acc += __ldg(src + s * stride);
        out = __fmul_rn(acc, f.weights != nullptr ? __fmul_rn(gs, f.weights[t]) : gs);
      }
      // accumulation adds the fp32 gradient as it would be written without it
      if (f.dh_bf16) {
        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(f.dH) + idx;
        if (f.dh_acc) out = __fadd_rn(out, __bfloat162float(*o));
        *o = __float2bfloat16_rn(out);
      } else {
        float* o = static_cast<float*>(f.dH) + idx;
        if (f.dh_acc) out = __fadd_rn(out, *o);
        *o = out;
      }
    }
  }
  if (f.metrics != nullptr) {
    // Cut Metrics of each position from the integer partials (exact, any order)
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < T; t += gridDim.x * blockDim.x) {
      const int c = f.cidx[t];
      int4 out = make_int4(0, 0, 0, 0);
      if (c >= 0) {
        int cnt = 0, tp = 0;
        for (int s = 0; s < f.met_slots; ++s) {
          const int2 v = f.met_part[static_cast<int64_t>(s) * f.Tpad + c];
          cnt += v.x;
          tp += v.y;
        }
        const int fn = f.row_cnt[t] - tp;
        out = make_int4(tp, cnt - tp, fn, f.V - cnt - fn);
      }
      reinterpret_cast<int4*>(f.metrics)[t] = out;
    }
  }
  if (f.loss != nullptr) {
    // two levels, both in a fixed order: block b sums slice b of the partials
    // (coalesced, thread-strided, then a fixed tree), the last block to finish
    // sums the block results in block order
    const int nb = static_cast<int>(gridDim.x);
    const int n_loss_part = f.loss_pos_splits > 0
                                ? f.loss_pos_splits * static_cast<int>(ceil_div(f.hdr->n_valid, kTileM)) * kNumEpiWarps
                                : f.n_loss_part;
    const int per_a = (n_loss_part + nb - 1) / nb, per_b = (f.n_corr_part + nb - 1) / nb;
    const int a0 = blockIdx.x * per_a, a1 = min(n_loss_part, a0 + per_a);
    const int b0 = blockIdx.x * per_b, b1 = min(f.n_corr_part, b0 + per_b);
    double a = 0.0, b = 0.0;
    for (int i = a0 + threadIdx.x; i < a1; i += blockDim.x) a += f.loss_part[i];
    for (int i = b0 + threadIdx.x; i < b1; i += blockDim.x) b += f.corr_part[i];
    a = block_sum_fixed(a, red);
    b = block_sum_fixed(b, red);
    if (threadIdx.x == 0) {
      f.blk_part[2 * blockIdx.x] = a;
      f.blk_part[2 * blockIdx.x + 1] = b;
      __threadfence();
      ticket = atomicAdd(&f.hdr->finish_count, 1);
    }
    __syncthreads();
    if (ticket == nb - 1) {
      __threadfence();
      double da = 0.0, db = 0.0;
      for (int i = threadIdx.x; i < nb; i += blockDim.x) {
        da += *reinterpret_cast<volatile double*>(f.blk_part + 2 * i);
        db += *reinterpret_cast<volatile double*>(f.blk_part + 2 * i + 1);
      }
      const double dense = block_sum_fixed(da, red);
      const double corr = block_sum_fixed(db, red);
      // the linear half of the dense term: (sum_c wc_c H_c[c]) . (sum_v e_v), H_c holding h / 2
      const double lin = f.use_lin ? *reinterpret_cast<volatile double*>(&f.hdr->lin) : 0.0;
      if (threadIdx.x == 0) *f.loss = f.hdr->n_valid > 0 ? f.hdr->loss_scale * (dense + lin - corr) : 0.0;
    }
  }
}

// ------------------------------------------------------------------ fp32 CUDA-core path
__device__ __forceinline__ float sigmoid_f32(float z) {
  if (z >= 0.f) return 1.f / (1.f + expf(-z));
  const float e = expf(z);
  return e / (1.f + e);
}

// One thread per item v (blocks of 128 items, matching the tensor-core path's
// item tiles): the dense loss sum over valid positions and dE_v = g s sum_t (s(x)-y) h_t.
__global__ void __launch_bounds__(128) k_simt_items(const float* __restrict__ Hc, const float* __restrict__ E,
                                                    int V, int D, const int* __restrict__ row_ptr,
                                                    const int* __restrict__ pair_v, const WsHeader* hdr,
                                                    const float* __restrict__ wc, void* __restrict__ dE, int de_bf16,
                                                    int de_acc, double* __restrict__ loss_part) {
  // blockIdx.y: the 32 columns of dE this thread accumulates (in registers); the
  // loss is summed by the blocks of column group 0
  __shared__ double red[128];
  const int v = blockIdx.x * 128 + threadIdx.x;
  const int d0 = blockIdx.y * 32;
  const bool lead = blockIdx.y == 0;
  const int nv = hdr->n_valid;
  const float gs = hdr->grad_scale;
  double lsum = 0.0;
  float acc[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) acc[k] = 0.f;
  if (v < V) {
    const float* e = E + static_cast<int64_t>(v) * D;
    for (int c = 0; c < nv; ++c) {
      const float* h = Hc + static_cast<int64_t>(c) * D;
      const float w = wc != nullptr ? wc[c] : 1.f;
      float z = 0.f;
      for (int d = 0; d < D; ++d) z = fmaf(h[d], e[d], z);
      float y = 0.f;
      for (int p = row_ptr[c]; p < row_ptr[c + 1]; ++p) y = pair_v[p] == v ? 1.f : y;
      if (lead) lsum += static_cast<double>(w) * static_cast<double>(fmaxf(z, 0.f) + log1pf(expf(-fabsf(z))));
      if (dE != nullptr) {
        const float g = w * (sigmoid_f32(z) - y);
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (d0 + k < D) acc[k] = fmaf(g, h[d0 + k], acc[k]);
      }
    }
    if (dE != nullptr) {
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        if (d0 + k >= D) break;
        const int64_t o_ = static_cast<int64_t>(v) * D + d0 + k;
        float out = __fmul_rn(acc[k], gs);
        if (de_bf16) {
          __nv_bfloat16* o = static_cast<__nv_bfloat16*>(dE) + o_;
          if (de_acc) out = __fadd_rn(out, __bfloat162float(*o));
          *o = __float2bfloat16_rn(out);
        } else {
          float* o = static_cast<float*>(dE) + o_;
          if (de_acc) out = __fadd_rn(out, *o);
          *o = out;
        }
      }
    }
  }
  if (loss_part != nullptr && lead) {
    // same layout as the tensor-core path: kNumEpiWarps partials per 128-item tile
    const double s = block_sum_fixed(v < V ? lsum : 0.0, red);
    if (threadIdx.x < kNumEpiWarps) loss_part[static_cast<int64_t>(blockIdx.x) * kNumEpiWarps + threadIdx.x] = threadIdx.x == 0 ? s : 0.0;
  }
}

// One thread per compacted row c: dH partial sum_v (s(x)-y) e_v over all items,
// and/or the row's count of x > 0 and of positives with x > 0 (Cut Metrics).
__global__ void __launch_bounds__(128) k_simt_rows(const float* __restrict__ Hc, const float* __restrict__ E,
                                                   int V, int D, const int* __restrict__ row_ptr,
                                                   const int* __restrict__ pair_v, const WsHeader* hdr,
                                                   float* __restrict__ dh_part, int2* __restrict__ met_part) {
  // blockIdx.y: the 32 columns of dH this thread accumulates (in registers); the
  // metrics are counted by the blocks of column group 0
  const int c = blockIdx.x * 128 + threadIdx.x;
  const int d0 = blockIdx.y * 32;
  const bool lead = blockIdx.y == 0;
  if (c >= hdr->n_valid) return;
  float acc[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) acc[k] = 0.f;
  const float* h = Hc + static_cast<int64_t>(c) * D;
  int p = row_ptr[c];
  const int pend = row_ptr[c + 1];
  int cnt = 0, tp = 0;
  // four items at a time: their dot products interleave (four independent load
  // and FMA chains); their contributions are then added in item order
  for (int vb = 0; vb < V; vb += 4) {
    const float* eb = E + static_cast<int64_t>(vb) * D;
    const int nu = min(4, V - vb);
    float z[4] = {0.f, 0.f, 0.f, 0.f};
    for (int d = 0; d < D; ++d) {
      const float hd = h[d];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (u < nu) z[u] = fmaf(hd, eb[u * D + d], z[u]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (u >= nu) break;
      const int v = vb + u;
      const float* e = eb + u * D;
      float y = 0.f;
      if (p < pend && pair_v[p] == v) {
        y = 1.f;
        ++p;
      }
      cnt += z[u] > 0.f ? 1 : 0;
      tp += (z[u] > 0.f && y > 0.f) ? 1 : 0;
      if (dh_part != nullptr) {
        const float g = sigmoid_f32(z[u]) - y;
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (d0 + k < D) acc[k] = fmaf(g, e[d0 + k], acc[k]);
      }
    }
  }
  if (dh_part != nullptr) {
#pragma unroll
    for (int k = 0; k < 32; ++k)
      if (d0 + k < D) dh_part[static_cast<int64_t>(c) * D + d0 + k] = acc[k];
  }
  if (met_part != nullptr && lead) met_part[c] = make_int2(cnt, tp);
}

// Zero a float buffer (used for dE when no position is valid).
__global__ void k_zero_f32(float* __restrict__ p, int64_t n) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = 0.f;
}

}  // namespace cutbce
