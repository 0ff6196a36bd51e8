// Internal layout shared by the host entry points and the kernels of libmla.so.
#pragma once
#include <cstdint>

namespace mla {

constexpr int kBlockSize = 64;     // cache rows per physical block
constexpr int kDLatent = 512;      // c_kv / output width
constexpr int kDRope = 64;         // k_pe / q_pe width
constexpr int kDQK = 576;          // cache row width
constexpr int kRowsPerTile = 128;  // query rows (token-major: row = i * H + h) per CTA pair
constexpr int kRowsPerCta = 64;    // each CTA of the pair owns 64 of them
constexpr int kTileKeys = 256;     // keys per pipeline step (4 cache blocks)
constexpr int kBlocksPerTile = kTileKeys / kBlockSize;

// Packed FP8 cache row (bytes): [0, 512) e4m3 codes of c_kv / scale, [512, 640) k_pe /
// scale as 64 bf16, [640, 644) the fp32 scale, [644, 656) zero.
constexpr int kRowBytes8 = 656;
constexpr int kOffKpe8 = 512;
constexpr int kOffScale8 = 640;

// Split-KV scheduler constants (the same values are stated in the float64 oracle).
constexpr int kSchedOverheadTiles = 1;  // cost of starting a sequence, in 256-key tiles
constexpr int kSchedMinCap = 2;         // smallest partition cost, in tiles
constexpr int kMaxWorkers = 256;         // CTA pairs the metadata can describe

// ---------------------------------------------------------------------------
// Metadata buffer (int32 words), written by mla_get_metadata:
//   [0, kHdrWords)                      header (see kHdr*)
//   part_start [kMaxWorkers][2]         (b, k) of each partition's first block
//   part_end   [kMaxWorkers][2]         exclusive end (next partition's start)
//   nblk[B], first_part[B], num_splits[B], split_prefix[B]
// ---------------------------------------------------------------------------
constexpr int kHdrWords = 16;
enum HdrField : int {
  kHdrMagic = 0,
  kHdrB = 1,
  kHdrSq = 2,
  kHdrH = 3,
  kHdrNumParts = 4,   // P: partitions per row tile
  kHdrNumTiles = 5,   // T: row tiles of 128 query rows
  kHdrCap = 6,        // partition cost cap (256-key tiles)
  kHdrTotalSlots = 7, // sum of num_splits
  kHdrNumWorkers = 8, // CTA pairs available on the device
  kHdrOverhead = 9,
  kHdrTokens = 10,    // token schedule: the call's s_q (query tokens per sequence); 0 otherwise
  kHdrTokCausal = 11, // token schedule: the causal flag the lengths were built with
};
constexpr int32_t kMetaMagic = 0x4D4C4131;  // "MLA1"

// Token schedule: the decode of B sequences with up to `rep` query tokens each (q of
// them real) runs as an s_q = 1 decode of B * rep sequences; sequence u = b * rep + t
// is token t of b.  With the causal mask token t sees the first n - q + t + 1 keys of
// b (all n without it); a padding token (t >= q) sees none.  -1 marks an invalid query
// count or a negative length.  The schedule, the attention kernel and the combine all
// take a token's length from here.
__host__ __device__ inline int token_seq_len(int n, int q, int t, int rep, int causal) {
  if (q < 0 || q > rep || n < 0) return -1;
  if (t >= q) return 0;
  if (!causal) return n;
  const int v = n - q + t + 1;
  return v > 0 ? v : 0;
}

__host__ __device__ inline int64_t meta_words(int B) {
  return kHdrWords + 4LL * kMaxWorkers + 4LL * B;
}
__host__ __device__ inline int off_part_start() { return kHdrWords; }
__host__ __device__ inline int off_part_end() { return kHdrWords + 2 * kMaxWorkers; }
__host__ __device__ inline int off_nblk() { return kHdrWords + 4 * kMaxWorkers; }
__host__ __device__ inline int64_t off_first_part(int B) { return off_nblk() + (int64_t)B; }
__host__ __device__ inline int64_t off_num_splits(int B) { return off_nblk() + 2LL * B; }
__host__ __device__ inline int64_t off_split_prefix(int B) { return off_nblk() + 3LL * B; }

// ---------------------------------------------------------------------------
// Workspace: partial outputs of split sequences.
//   partial_o   fp32 [slots][M_total][512]   (normalised by the piece's own sum)
//   partial_lse fp32 [slots][M_total]
// with slots = B + P*T upper bound (each partition boundary cuts one sequence).
// ---------------------------------------------------------------------------
__host__ __device__ inline int64_t ws_slots(int B, int num_workers) { return (int64_t)B + num_workers; }

// Kernel error bits (mirror MLA_DEVICE_ERR_* of the public header).
constexpr int kErrBlockId = 1;
constexpr int kErrSeqlen = 2;
constexpr int kErrTimeout = 4;
constexpr int kErrMetadata = 8;

}  // namespace mla
