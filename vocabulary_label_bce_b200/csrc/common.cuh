// Shared definitions: status codes, the workspace header, tile geometry.
#pragma once
#include <cstdint>
#include <cstddef>

namespace cutbce {

enum : int {
  kOk = 0,
  kErrInvalidArg = 1,
  kErrUnsupported = 2,
  kErrWorkspace = 3,
  kErrTargetRange = 4,
  kErrTimeout = 5,
  kErrCuda = 6,
};

enum : int { kMeanValidPositions = 0, kSum = 1, kMeanElements = 2 };

constexpr int kMaxK = 128;            // target slots per position
constexpr int kMaxDim = 256;          // feature width
constexpr int kTileM = 128;           // stationary rows per tile = TMEM lanes
constexpr int kMaxCtas = 256;         // upper bound of a persistent grid
constexpr int kMaxSplits = 64;        // dH partial splits over the vocabulary
constexpr int kTileThreads = 576;     // 18 warps: TMA producer, MMA issuer, 16 epilogue
constexpr int kEpiWarp0 = 2;
constexpr int kNumEpiWarps = 16;      // groups x (4 TMEM lane quarters x column slabs)
// Epilogue groups taking tiles in turn: two in both passes, so that one
// group's tile handshakes overlap the other's math and each warp handles a
// 64-column slab (two chunks) per handshake.  (One group of 16 warps on every
// tile, 32 columns each, made the position-owned pass 2% slower: twice the
// handshakes per logit.)
template <bool kDH>
__host__ __device__ constexpr int epi_groups() { return 2; }

// First 256 bytes of the workspace.
struct WsHeader {
  int status;          // first device-detected error, 0 = none
  int n_valid;         // valid positions
  int n_pairs;         // distinct (position, positive item) pairs
  int wait_tag;        // where the first bounded wait gave up: role<<28 | barrier<<20 | counter
  double loss_scale;   // s
  float grad_scale;    // g * s
  int wait_block;      // CTA of that wait
  int finish_count;    // blocks of the finish kernel done with their loss slice
  int role_wait_tag[7];  // [role - 1]: where role 1 (producer), 2 (MMA), 4 (epilogue) stood when its CTA gave up
  int colsum_count;    // blocks of the column-sum kernel done
  double lin;          // (sum_c w_c H_c[c]) . (sum_v e_v): the linear half of the dense loss
};
static_assert(sizeof(WsHeader) <= 256, "the workspace header is 256 bytes");

// Geometry of the tcgen05 tile engine for one padded feature width DP and G
// epilogue groups.
template <int DP, int G = 1>
struct TileCfg {
  static constexpr int GROUPS = G;                           // epilogue groups taking tiles in turn
  static constexpr int GROUP_WARPS = kNumEpiWarps / G;       // warps that take one tile
  static constexpr int SLABS = GROUP_WARPS / 4;              // column slabs of a tile (4 TMEM lane quarters each)
  static_assert(DP % 64 == 0 && DP >= 64 && DP <= 256, "DP must be 64, 128, 192 or 256");
  static constexpr int BN = DP <= 128 ? 128 : 64;          // streamed rows per tile (Z columns)
  static constexpr int NKB = DP / 64;                        // 128-byte column blocks per row
  // stages of the streamed-operand ring: a streamed tile is held from its logit MMA
  // (issued up to NZ-1 tiles early) until its gradient MMA completes, and the ring
  // must still cover the L2 -> shared memory latency of the next loads
  static constexpr int NX = DP == 64 ? 12 : DP == 128 ? 5 : DP == 192 ? 7 : 4;
  // fp32 logit tiles in tensor memory.  The bf16 G tile of a logit tile is
  // written over that tile's own columns (each warp over the slab it loaded),
  // so a buffer holds Z, then G, and is free once the gradient MMA reading G
  // has completed.
  static constexpr int NZ = 3;
  static constexpr uint32_t S_BYTES = kTileM * DP * 2;       // stationary tile
  static constexpr uint32_t X_BYTES = BN * DP * 2;           // streamed tile
  static constexpr int ZC = BN / SLABS;                      // logit columns per epilogue warp (one slab)
  static constexpr int ACC_COL = NZ * BN;                    // TMEM column of the gradient accumulator
  static constexpr int TMEM_COLS = 512;
  // The stationary tile is copied into tensor memory (bf16 pairs, DP/2 columns)
  // when it fits, so the logit MMA reads only its B operand from shared memory.
  static constexpr int S_COL = ACC_COL + DP;
  static constexpr bool S_IN_TMEM = S_COL + DP / 2 <= TMEM_COLS;
  static constexpr int NUM_BARS = 2 + 2 * NX + 3 * NZ + 3;  // see the kernel for the list
  // per epilogue warp: positives of its 32 rows, one word per 32 columns of its slab
  static constexpr int MASK_WORDS = ZC >= 32 ? ZC / 32 : 1;
  static constexpr uint32_t MASK_BYTES = kNumEpiWarps * 32 * MASK_WORDS * 4;
  static constexpr uint32_t SMEM_BYTES = 1024 + S_BYTES + NX * X_BYTES + MASK_BYTES + NUM_BARS * 8 + 16 + 64;
  static_assert(ACC_COL + DP <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(SMEM_BYTES > 232448 / 2, "one CTA per SM keeps the TMEM allocation uncontended");
};

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

}  // namespace cutbce
