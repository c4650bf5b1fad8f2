/*
 * cutbce.h -- C ABI of the exact fused large-vocabulary binary cross-entropy
 * loss and its gradient, for NVIDIA B200 (sm_100a).
 *
 * The operation is the one defined in "Cut Binary Cross Entropy: Efficient
 * Large-Vocabulary Loss and Gradient Kernels for Sequential Recommendation"
 * (Li, Ning, Hammad):
 *
 *   logits      x_tv = h_t . e_v                           (section I-A, X = A E^T)
 *   element     l(x, y) = max(x,0) + log(1 + e^-|x|) - y x  (section III-A, Eq. (2))
 *   loss        s * sum_{valid t} sum_{v < V} l(x_tv, y_tv)   (Eq. (3), averaging of III-B)
 *   gradients   G = sigmoid(X) - Y,  dH = g s G E,  dE = g s G^T H   (section III-B, Eq. (4))
 *
 * where y_tv = 1 iff item v is one of the (distinct) positive ids of
 * position t, s is the normalisation chosen by `reduction`, and g is the
 * upstream gradient.  The [T, V] logits and their gradient are never written
 * to device memory (section III-B, Table I of the paper): every logit tile is
 * formed on chip, in tensor memory, and consumed there.
 *
 * Conventions shared by every entry point:
 *  - T = B * N flattened positions (section III-A, footnote 1), V items,
 *    D feature width, K target slots per position.
 *  - H is [T, D] and E is [V, D], row-major, dense, device memory.  bf16
 *    (CUTBCE_BF16, the fast path) or fp32 (CUTBCE_F32, a plain CUDA-core path
 *    meant for small checks).  For bf16, D must be a multiple of 8 and at most
 *    256, and H, E must be 16-byte aligned.
 *  - targets is int32 [T, K], device memory.  -1 marks an empty slot; an id in
 *    [0, V) is a positive item; repeated ids in one row count once.  Any other
 *    id in a valid row is a data error (CUTBCE_ERR_TARGET_RANGE, reported
 *    through the workspace status word, see cutbce_read_status).
 *  - mask is uint8 [T] (1 = valid position, 0 = padding), device memory, or
 *    NULL for "all valid".  A masked position contributes no loss, receives a
 *    zero dH row and contributes nothing to dE; its ids are ignored entirely.
 *  - Every output and the workspace are owned by the caller.  The library
 *    never allocates or frees device memory and keeps no state between calls
 *    apart from cached device attributes, a per-device pool of second streams
 *    and events (below) and the static scratch array of
 *    cutbce_forward_fixed_scratch.
 *  - All compute calls are asynchronous on `stream`.  A call that computes the
 *    loss runs the column sums of E on a second stream of the library's own
 *    (created once per device, pooled), forked from `stream` and joined back
 *    to it by events, so the work is ordered on `stream` as usual (and is
 *    captured into a CUDA graph with it); cutbce_forward_fixed_scratch uses
 *    `stream` alone.  Errors a host can see
 *    (NULL pointers, sizes <= 0, unsupported D or dtype, a workspace that is
 *    too small, a device that is not sm_100) are returned before anything is
 *    launched.  Data-dependent errors (an id out of range, a bounded wait in a
 *    kernel that ran out) are written to the workspace status word; when it is
 *    nonzero the outputs of that call are unspecified.
 *  - dH and dE are overwritten, not accumulated (cutbce_forward_backward_ex
 *    can accumulate instead).  The loss is double.
 *  - Results are deterministic: no floating-point atomics are used, and every
 *    reduction runs in a fixed order that does not depend on the GPU's SM count.
 */
#ifndef CUTBCE_H
#define CUTBCE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so this header needs no CUDA headers. */
typedef struct CUstream_st* cutbce_stream_t;

typedef enum {
  CUTBCE_OK = 0,
  CUTBCE_ERR_INVALID_ARG = 1,   /* NULL pointer, non-positive size, misaligned pointer */
  CUTBCE_ERR_UNSUPPORTED = 2,   /* D, K or dtype outside the supported set; not an sm_100 device */
  CUTBCE_ERR_WORKSPACE = 3,     /* workspace smaller than cutbce_workspace_size() */
  CUTBCE_ERR_TARGET_RANGE = 4,  /* an id < -1 or >= V in a valid row (device-detected) */
  CUTBCE_ERR_TIMEOUT = 5,       /* a bounded wait inside a kernel ran out (device-detected) */
  CUTBCE_ERR_CUDA = 6           /* a CUDA runtime call failed */
} cutbce_status;

typedef enum { CUTBCE_BF16 = 0, CUTBCE_F32 = 1 } cutbce_dtype;

/* Normalisation s of the summed loss (and of both gradients):
 *  MEAN_VALID_POSITIONS: 1 / n_valid  (positions averaged, padding excluded; section III-B)
 *  SUM:                  1
 *  MEAN_ELEMENTS:        1 / (n_valid * V)  (Eq. (3)'s 1/V and section III-B's 1/BN)
 * With n_valid = 0 the loss and both gradients are 0. */
typedef enum {
  CUTBCE_MEAN_VALID_POSITIONS = 0,
  CUTBCE_SUM = 1,
  CUTBCE_MEAN_ELEMENTS = 2
} cutbce_reduction;

/* Problem statement, after the paper's cut_binary_cross_entropy(activations,
 * embeddings, targets, weights) (section III-C, Listing 1), flattened to T rows. */
typedef struct {
  int64_t T;                 /* positions (B*N), >= 1; < 2^30, and for bf16 < 2^24 - 127
                                (the item-owned pass packs a compacted position into 24 bits) */
  int64_t V;                 /* items, >= 1, < 2^31 */
  int64_t D;                 /* feature width, >= 1 */
  int64_t K;                 /* target slots per position, 1..128 */
  int32_t dtype;             /* cutbce_dtype of H and E */
  int32_t reduction;         /* cutbce_reduction */
  const void* H;             /* [T, D] activations (device) */
  const void* E;             /* [V, D] item embeddings (device) */
  const int32_t* targets;    /* [T, K] positive ids, -1 empty (device) */
  const uint8_t* mask;       /* [T] 1 = valid, or NULL = all valid (device) */
} cutbce_problem;

/* Bytes of device workspace that a compute call on this problem needs, for
 * every set of outputs (loss, dH and dE): enough for any compute call.  The
 * size has no T*V term: it is O(T*K + S*T*D + V) for a split count S <= 64
 * chosen from T.  Host-only; launches nothing.  Returns INVALID_ARG or
 * UNSUPPORTED for a problem the compute calls would reject. */
cutbce_status cutbce_workspace_size(const cutbce_problem* prob, size_t* bytes);

/* Outputs of a compute call, as bits of `outputs` below. */
enum { CUTBCE_OUT_LOSS = 1, CUTBCE_OUT_DH = 2, CUTBCE_OUT_DE = 4, CUTBCE_OUT_METRICS = 8 };

/* Bytes of device workspace for a call that computes only the given outputs
 * (a bitwise or of CUTBCE_OUT_*): cutbce_forward needs CUTBCE_OUT_LOSS;
 * cutbce_backward and cutbce_forward_backward need the bits of the outputs
 * they are given non-NULL; cutbce_forward_backward_ex adds CUTBCE_OUT_METRICS
 * when it is given a metrics output.  The dH split partials (O(S*T*D)) are
 * counted only with CUTBCE_OUT_DH, the metrics partials (O(S*T)) only with
 * CUTBCE_OUT_METRICS, and the pair-sort buffers (O(T*K)) only with
 * CUTBCE_OUT_DE, so a loss-only workspace is O(T*K + T*D + V).  Host-only. */
cutbce_status cutbce_workspace_size_for(const cutbce_problem* prob, int outputs, size_t* bytes);

/* Loss only (section III-A).  loss: device double, written with the
 * normalised loss.  ws: device workspace of ws_bytes bytes
 * (>= cutbce_workspace_size_for(prob, CUTBCE_OUT_LOSS)), 256-byte aligned. */
cutbce_status cutbce_forward(const cutbce_problem* prob, void* ws, size_t ws_bytes,
                             double* loss, cutbce_stream_t stream);

/* Size of the static device scratch array behind cutbce_forward_fixed_scratch
 * (16 MiB, part of the library's device image on every device it runs on). */
#define CUTBCE_FIXED_SCRATCH_BYTES ((size_t)16 << 20)

/* Loss only, like cutbce_forward, but with no workspace argument: the call
 * uses a static scratch array of CUTBCE_FIXED_SCRATCH_BYTES bytes that lives in
 * the library's own device image, so neither the caller nor the library
 * allocates anything.  The paper has no counterpart to this entry; it exists
 * for callers that cannot hand over device memory at the point of the call --
 * for instance code that sized its device memory pool once at start-up and may
 * not grow it, or a host runtime with no device allocator of its own, where a
 * cudaMalloc would also stall the device until pending work drains.
 *
 * Limit: problems with cutbce_workspace_size_for(prob, CUTBCE_OUT_LOSS) >
 * CUTBCE_FIXED_SCRATCH_BYTES are rejected with CUTBCE_ERR_WORKSPACE before
 * anything is launched.  That loss-only workspace is about
 * 16 T K + 2 T D' + 16 * 8 * ceil(V / 128) + 8 D (444 + ceil(T / 256)) bytes
 * (D' = D rounded up to 64; at most 64 in the last ceiling), so
 * for example T = 12,800 positions with K = 16 slots, D = 64 and V = 876,000
 * items (about 6 MB) fits.
 * Setup: the first call on each device, with that device current, looks up
 * the device address of the array (cudaGetSymbolAddress) and caches it; that
 * lookup may load the library's device code on the device, so make the first
 * call on each device before any stream capture begins.  A failed lookup
 * returns CUTBCE_ERR_CUDA.
 * Zeroing: nothing has to start at zero; each call clears the part of the
 * array it needs cleared (the status header) on `stream` itself.
 * Concurrency: all calls on one device share the one array, so two calls whose
 * device work can overlap (different streams, or host threads without
 * ordering between them) race on it and give wrong results; order them, for
 * example by issuing them on one stream.
 * Errors: host-visible errors are returned as for cutbce_forward.  The
 * device status word sits in the static array, which the library does not
 * expose, so a data error (an id out of range) is not reported by this entry
 * (the loss is then unspecified); use cutbce_forward where it must be. */
cutbce_status cutbce_forward_fixed_scratch(const cutbce_problem* prob, double* loss,
                                           cutbce_stream_t stream);

/* Gradients only (section III-B, Eq. (4)), recomputing the logits.
 * grad_loss: device float scalar g, or NULL for g = 1.
 * dH: device float [T, D]; dE: device float [V, D]; either may be NULL to skip it.
 * ws: >= cutbce_workspace_size_for(prob, outputs given) bytes, 256-byte aligned. */
cutbce_status cutbce_backward(const cutbce_problem* prob, const float* grad_loss,
                              float* dH, float* dE, void* ws, size_t ws_bytes,
                              cutbce_stream_t stream);

/* Loss and both gradients in one pass over the logits for the loss and dE and
 * a second pass for dH.  loss may be NULL to skip it; dH or dE may be NULL. */
cutbce_status cutbce_forward_backward(const cutbce_problem* prob, const float* grad_loss,
                                      double* loss, float* dH, float* dE,
                                      void* ws, size_t ws_bytes, cutbce_stream_t stream);

/* dtype of the dH and dE outputs of cutbce_forward_backward_ex. */
enum { CUTBCE_GRAD_F32 = 0, CUTBCE_GRAD_BF16 = 1 };
/* Bits of cutbce_options.accumulate. */
enum { CUTBCE_ACCUMULATE_DH = 1, CUTBCE_ACCUMULATE_DE = 2 };

/* Options of cutbce_forward_backward_ex; a zero-initialised struct gives the
 * behaviour of cutbce_forward_backward. */
typedef struct {
  /* Cut Metrics (section III-D): [T, 4] int32 device output, 16-byte aligned, or
   * NULL.  Row t holds (TP, FP, FN, TN) of position t over the vocabulary of this
   * call, item v counted as predicted positive iff sigmoid(x_tv) > 1/2, i.e.
   * x_tv > 0 as the kernel computes x_tv (fp32 accumulation of the products; a
   * logit of exactly 0, or one below the smallest normal float, is a predicted
   * negative).  TP + FP + FN + TN = V; invalid positions get (0, 0, 0, 0).  The
   * counts are not weighted.  They come from a position-owned pass over the
   * logits: fused into the dH pass when dH is requested, a count-only pass
   * otherwise. */
  int32_t* metrics;
  /* Per-position weights w (the `weights` argument of section III-C, Listing 1):
   * float [T] device array, 4-byte aligned, or NULL for w = 1.  Position t's loss
   * row and its row of G = sigmoid(X) - Y are multiplied by w_t:
   *   loss = s sum_t w_t sum_v l(x_tv, y_tv),  dH_t = g s w_t sum_v (sigmoid - y) e_v,
   *   dE_v = g s sum_t w_t (sigmoid - y) h_t.
   * A position with w_t = 0 is padding, exactly like a masked one: it is not
   * counted in the mean and gets a zero dH row.  With weights the loss is
   * summed in the position-owned pass (one weight per row) and the item-owned
   * pass scales each column of G by its weight. */
  const float* weights;
  /* CUTBCE_GRAD_F32 (default) or CUTBCE_GRAD_BF16: dtype of the dH and dE
   * outputs (bf16 is rounded to nearest even from the fp32 result). */
  int32_t grad_dtype;
  /* Bitwise or of CUTBCE_ACCUMULATE_DH / _DE: add the gradient to what the
   * output already holds instead of overwriting it (the sum is formed in fp32
   * and rounded once; masked rows of dH keep their value). */
  int32_t accumulate;
  /* Vocabulary sharding (section III-C, the vocabulary-parallel split): E holds
   * items [vocab_offset, vocab_offset + V) of a vocabulary of V_total items
   * (V_total = 0 means V, and then vocab_offset must be 0).  Target ids are
   * global: an id in [0, V_total) outside this shard is not a positive of this
   * call (and not an error); an id < -1 or >= V_total in a valid row is
   * CUTBCE_ERR_TARGET_RANGE.  The loss and dH are this shard's shares (the sums
   * over all shards are the unsharded results, with the same normalisation s;
   * MEAN_ELEMENTS uses V_total), dE holds this shard's rows, and the metrics
   * count this shard's items. */
  int64_t vocab_offset;
  int64_t V_total;
} cutbce_options;

/* cutbce_forward_backward with options (see cutbce_options).  dH and dE point
 * to fp32 or bf16 arrays according to opts->grad_dtype.  At least one of loss,
 * dH, dE and opts->metrics must be non-NULL; ws must hold
 * cutbce_workspace_size_ex(prob, opts, the bits of those outputs) bytes. */
cutbce_status cutbce_forward_backward_ex(const cutbce_problem* prob, const cutbce_options* opts,
                                         const float* grad_loss, double* loss, void* dH, void* dE,
                                         void* ws, size_t ws_bytes, cutbce_stream_t stream);

/* Workspace bytes of cutbce_forward_backward_ex for these options and outputs
 * (bits CUTBCE_OUT_*); opts may be NULL.  Host-only. */
cutbce_status cutbce_workspace_size_ex(const cutbce_problem* prob, const cutbce_options* opts, int outputs,
                                       size_t* bytes);

/* Bytes of device memory that cutbce_forward_backward_host needs in dev_buf. */
cutbce_status cutbce_host_buffer_size(const cutbce_problem* prob, size_t* bytes);

/* The fused call for callers whose buffers live in host memory: prob's H, E,
 * targets and mask are HOST pointers (pinned memory makes the copies
 * asynchronous), grad_loss is a host value, and loss / dH / dE are host
 * outputs (dH, dE may be NULL).  dev_buf (>= cutbce_host_buffer_size bytes,
 * 256-byte aligned, caller-owned device memory) holds the device copies and the
 * workspace.  The call copies the inputs in, runs the fused computation,
 * copies the results out and synchronises; on return the host outputs are
 * valid and the returned status includes the device status word.
 * Overlap: with a bf16 item table of more than 32 MiB, the call works in up to
 * four vocabulary shards (whole vocabulary splits of the dH pass, on whole
 * 128-item tiles).  It compacts the rows and orders the pairs once (that reads
 * no E).  Then, as shard s of E lands (copied in on a second stream while shard
 * s - 1 is computed on `stream`), it runs the two tile passes over that shard's
 * item tiles and splits only; the shard's dE rows are copied out on a third
 * stream as soon as its item-owned pass ends.  The sparse correction, the
 * column sums and the finish run once at the end.  Every tile and split is
 * computed exactly as by cutbce_forward_backward and summed by the same finish,
 * so loss, dH and dE are its bits.
 * The streams and events come from a per-device pool, created by the first
 * such calls and kept for the rest of the process; every stream the call used
 * is synchronised before it returns. */
cutbce_status cutbce_forward_backward_host(const cutbce_problem* prob, float grad_loss,
                                           double* loss, float* dH, float* dE,
                                           void* dev_buf, size_t dev_bytes,
                                           cutbce_stream_t stream);

/* Full-vocabulary ranking for evaluation (section III-E: the hidden state of a
 * sequence's last non-pad position is scored against every item; Hit@8 asks
 * whether one of the held-out items is among the 8 best).
 *
 * Q: [B, D] bf16 queries, E: [V, D] bf16 items (device, row-major, 16-byte
 * aligned; D a multiple of 8, at most 256), 1 <= k <= 16.  Writes, for each
 * query b, the k best items by the score x_bv = q_b . e_v (fp32 accumulation of
 * the bf16 products on the tensor cores) in descending score, equal scores in
 * ascending id: ids int32 [B, k] (-1 when V < k), scores float [B, k].  No
 * [B, V] score array is written anywhere: every score tile lives in tensor
 * memory until per-thread running top-k lists have taken it in.  ws: device
 * workspace of cutbce_topk_workspace_size bytes, 256-byte aligned, whose first
 * bytes hold the status word (cutbce_read_status).  dtype must be CUTBCE_BF16.
 * Asynchronous on `stream`. */
cutbce_status cutbce_topk_workspace_size(int64_t B, int64_t V, int64_t D, int k, size_t* bytes);
cutbce_status cutbce_topk(const void* Q, int64_t B, const void* E, int64_t V, int64_t D, int32_t dtype, int k,
                          int32_t* ids, float* scores, void* ws, size_t ws_bytes, cutbce_stream_t stream);

/* Hit@k of ranked ids (e.g. from cutbce_topk): hits[b] = 1 if one of the target
 * ids targets[b, 0..L) (-1 = empty slot) is among ids[b, 0..k), else 0.  All
 * device arrays (ids int32 [B, k], targets int32 [B, L], hits int32 [B]). */
cutbce_status cutbce_hit_at_k(const int32_t* ids, int64_t B, int k, const int32_t* targets, int64_t L, int32_t* hits,
                              cutbce_stream_t stream);

/* Synchronises `stream` and returns the device status word of the last call
 * that used this workspace (CUTBCE_OK, TARGET_RANGE or TIMEOUT). */
cutbce_status cutbce_read_status(const void* ws, cutbce_stream_t stream);

/* Synchronises `stream` and reads the integer side results of the last call on
 * this workspace: the number of valid positions, the number of distinct
 * (position, positive item) pairs, and, if row_counts is not NULL, the number of
 * distinct positive ids of each position (host int32 [T], 0 for masked rows). */
cutbce_status cutbce_read_counts(const cutbce_problem* prob, const void* ws,
                                 int64_t* n_valid, int64_t* n_pairs, int32_t* row_counts,
                                 cutbce_stream_t stream);

/* Number of kernels one call of the given entry (0 forward, 1 backward,
 * 2 forward_backward) launches for this problem (for launch accounting). */
int cutbce_kernel_launches(const cutbce_problem* prob, int entry);

/* Kernel kinds reported by the profiling calls, in launch order. */
enum {
  CUTBCE_KERNEL_PREP_ROWS = 0,      /* mask and id rules per position */
  CUTBCE_KERNEL_PREP_SCAN = 1,      /* row compaction, pair offsets, scales */
  CUTBCE_KERNEL_PREP_GATHER = 2,    /* compacted H, pair lists, sparse correction */
  CUTBCE_KERNEL_CSC_OFFSETS = 3,    /* first pair of every 128-item tile in the sorted pairs */
  CUTBCE_KERNEL_ITEM_PASS = 4,      /* tensor-core pass owning item tiles: loss and dE */
  CUTBCE_KERNEL_POSITION_PASS = 5,  /* tensor-core pass owning position tiles: dH partials */
  CUTBCE_KERNEL_FINISH = 6,         /* fixed-order dH reduction and the loss */
  CUTBCE_KERNEL_PAIR_SORT = 7,      /* pairs grouped by item tile, ascending position: sort keys and all radix passes */
  CUTBCE_KERNEL_TOPK = 8,           /* cutbce_topk: tensor-core scores and per-thread candidate lists */
  CUTBCE_KERNEL_TOPK_MERGE = 9,     /* cutbce_topk: fixed-order merge of the candidate lists */
  CUTBCE_KERNEL_COL_SUMS = 10,      /* column sums of E and of the compacted H: the loss's linear half */
  CUTBCE_NUM_KERNEL_KINDS = 11
};

/* Per-kernel device timing for benchmarks.  While enabled (process-wide),
 * every compute call records a CUDA event on its stream before and after each
 * kernel it launches (the events are created by the library, once, and reused).
 * Always returns CUTBCE_OK; disabling keeps what was already recorded. */
cutbce_status cutbce_profile_enable(int enable);

/* Waits for the recorded events, adds their elapsed times to per-kind totals
 * and writes the totals (milliseconds) to ms[CUTBCE_NUM_KERNEL_KINDS] and the
 * launch counts to launches[CUTBCE_NUM_KERNEL_KINDS]; clears them if reset != 0. */
cutbce_status cutbce_profile_read(double* ms, int64_t* launches, int reset);

/* Operation kinds measured by cutbce_probe_pipe_rate. */
enum {
  CUTBCE_PROBE_FFMA = 0,    /* fma.rn.f32 */
  CUTBCE_PROBE_FFMA2 = 1,   /* fma.rn.f32x2, counted as two operations */
  CUTBCE_PROBE_EX2 = 2,     /* ex2.approx.ftz.f32 */
  CUTBCE_PROBE_RCP = 3,     /* rcp.approx.ftz.f32 */
  CUTBCE_PROBE_TANH = 4,    /* tanh.approx.f32 */
  CUTBCE_PROBE_LG2 = 5,     /* lg2.approx.ftz.f32 */
  CUTBCE_PROBE_CVT_BF16X2 = 6, /* cvt.rn.bf16x2.f32, counted as one instruction */
  CUTBCE_PROBE_FMAX = 7,    /* max.f32 */
  CUTBCE_PROBE_ADD2 = 8,    /* add.rn.f32x2, counted as two operations */
  CUTBCE_PROBE_IADD = 9,    /* add.s32 */
  CUTBCE_PROBE_PRMT = 10,   /* prmt.b32 */
  CUTBCE_PROBE_EX2_F16X2 = 11,   /* ex2.approx.f16x2 (two 16-bit results), counted per instruction */
  CUTBCE_PROBE_EX2_BF16X2 = 12,  /* ex2.approx.ftz.bf16x2, counted per instruction */
  CUTBCE_PROBE_TANH_F16X2 = 13,  /* tanh.approx.f16x2, counted per instruction */
  CUTBCE_PROBE_HFMA2 = 14,       /* fma.rn.f16x2, counted per instruction */
  CUTBCE_PROBE_CVT_F16X2 = 15,   /* cvt.rn.f16x2.f32, counted per instruction */
  CUTBCE_PROBE_FFMA_SAT = 16,    /* fma.rn.sat.f32 */
  CUTBCE_PROBE_SELECT = 17,      /* setp.ge.f32 + selp.f32, counted per select */
  CUTBCE_PROBE_LOP = 18,         /* and.b32 */
  CUTBCE_PROBE_FMUL2 = 19,       /* mul.rn.f32x2, counted as two operations */
  CUTBCE_NUM_PROBES = 20
};

/* Bytes of device scratch cutbce_probe_pipe_rate needs. */
size_t cutbce_probe_scratch_bytes(void);

/* Measures how many operations of one kind an SM retires per clock: one CTA
 * of 1024 threads per SM runs independent dependency chains of the operation
 * and times them with the SM clock.  These rates set the arithmetic roofline
 * of the loss's element math (one exp, a reciprocal and a share of a log per
 * logit).  scratch: caller-owned device memory (cutbce_probe_scratch_bytes).
 * Synchronises `stream`.  Writes the median over SMs to *ops_per_clock_per_sm. */
cutbce_status cutbce_probe_pipe_rate(int op, void* scratch, size_t scratch_bytes, double* ops_per_clock_per_sm,
                                     cutbce_stream_t stream);

/* Tensor-core probe: on every SM one thread issues `iters` bf16 tcgen05.mma
 * instructions of shape 128 x n x 16 (n = 64, 128 or 256; fp32 accumulator in
 * tensor memory) and waits for them.  flags: bit 0, A from tensor memory
 * (else shared memory); bit 1, B MN-major (else K-major); bit 2, SM pairs:
 * 2-CTA clusters whose even CTA issues tcgen05.mma.cta_group::2 of shape
 * 256 x n x 16 (each CTA holds 128 rows of A and half of B; B K-major only).
 * Writes the median over issuing CTAs of the cycles per instruction spent
 * issuing and until completion (the dense ideal on B200 is n/2 cycles per
 * 128 x n x 16 on one SM, the same per 256 x n x 16 on a pair).
 * Synchronises `stream`. */
cutbce_status cutbce_probe_mma(int n, int flags, int64_t iters, void* scratch, size_t scratch_bytes,
                               double* issue_cycles_per_mma, double* cycles_per_mma, cutbce_stream_t stream);

/* Human-readable name of a status code (static storage). */
const char* cutbce_status_string(cutbce_status status);

/* Self-test of the element math the tile kernels run ("Cut Binary Cross
 * Entropy" section III-A Eq. (2) and section III-B Eq. (4)): for each of the n
 * device floats x[i], writes
 *   out[i]      = 2^x[i] by the FMA-pipe polynomial (valid for x in [-100, 100]);
 *   out[n + i]  = 2^x[i] by the SFU (ex2.approx);
 *   out[2n + i] = sigmoid(x[i]) as the gradient-only passes form it on the FMA
 *                 pipe alone (that polynomial, a seed and a cubic reciprocal step);
 *   out[3n + i] = sigmoid(x[i]) from the SFU's tanh, (1 + tanh(x/2)) / 2;
 *   out[4n + i] = w = 1 + |tanh(x[i]/2)| = 2 sigmoid(|x[i]|), the factor whose
 *                 log gives the loss in the passes that form loss and gradient.
 * out: device float [5n].  Asynchronous on `stream`. */
cutbce_status cutbce_selftest_element_math(const float* x, float* out, int64_t n, cutbce_stream_t stream);

/* Self-test of the bounded-wait machinery the kernels use: launches one CTA
 * that waits on a shared-memory barrier nothing will ever signal, with a
 * limit of limit_ns nanoseconds.  The wait gives up, writes CUTBCE_ERR_TIMEOUT
 * to *status_dev (device int32) and the kernel returns normally: the context
 * stays usable.  limit_ns must be in (0, 10^10]. */
cutbce_status cutbce_selftest_wait_timeout(int64_t limit_ns, int32_t* status_dev,
                                           cutbce_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* CUTBCE_H */
