// Split-KV scheduler: one CTA turns cache_seqlens into the partition schedule that
// the decode kernel and the combine kernel follow.  Integer-only; the float64 oracle
// states the same algorithm and the tests compare the two word for word.
//
// Cost model, in key tiles of kBlocksPerTile blocks (256 keys): every tile costs 1
// and every sequence with at least one block costs kSchedOverheadTiles more, placed
// before its first tile.  pre[b] is the cost of the sequences before b, so tile j of
// sequence b sits at position pre[b] + overhead + j.  With P partitions per row tile
// and cap = max(kSchedMinCap, ceil(total / P)), tile (b, j) and its blocks belong to
// partition floor(position / cap): contiguous, near-equal ranges that are cut only
// on tile boundaries, so a split adds no ragged tile.  (Split-K parallelism is named
// in the "DeepSeek speed test / FA3" article, section 2.1; this cost model is ours.)
#include <cuda_runtime.h>
#include <cstdint>
#include "mla_internal.h"

namespace mla {

namespace {

// Block-wide exclusive scan of int64 values held one per thread; returns the
// exclusive prefix for this thread and writes the block total to *total.
template <int kThreads>
__device__ int64_t block_exclusive_scan(int64_t v, int64_t* scratch /*[32]*/, int64_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int64_t w = (lane < (kThreads / 32)) ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    scratch[lane] = w;  // inclusive warp totals
  }
  __syncthreads();
  const int64_t warp_excl = (warp == 0) ? 0 : scratch[warp - 1];
  *total = scratch[kThreads / 32 - 1];
  __syncthreads();
  return warp_excl + x - v;
}

// kThreads = 256 for batches of at most 256 sequences (fewer and cheaper block-wide
// barriers), 1024 otherwise.
// Length of sequence b: seqlens[b], or with a token schedule (rep > 0) the length of
// virtual sequence b = token b % rep of real sequence b / rep (token_seq_len).
struct Lengths {
  const int32_t* seqlens;
  const int32_t* q_lens;  // token schedule: per-sequence query counts, or null (rep each)
  int rep, causal;
  __device__ int operator()(int b) const {
    if (rep == 0) return seqlens[b];
    const int r = b / rep;
    return token_seq_len(seqlens[r], q_lens ? q_lens[r] : rep, b - r * rep, rep, causal);
  }
};

template <int kThreads>
__global__ void __launch_bounds__(kThreads) metadata_kernel(const Lengths len_of, int B,
                                                            int s_q, int H, int num_workers,
                                                            int32_t* __restrict__ meta) {
  __shared__ int64_t scratch[32];
  __shared__ int64_t s_carry, s_total;
  // the attention kernel that follows may start its setup now (it waits for this
  // kernel to complete before reading the schedule)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int tid = threadIdx.x;
  const int M = s_q * H;
  const int T = (M + kRowsPerTile - 1) / kRowsPerTile;
  int P = num_workers / T;
  if (P < 1) P = 1;

  int32_t* part_start = meta + off_part_start();
  int32_t* part_end = meta + off_part_end();
  int32_t* nblk_out = meta + off_nblk();
  int32_t* first_part = meta + off_first_part(B);
  int32_t* num_splits = meta + off_num_splits(B);
  int32_t* split_prefix = meta + off_split_prefix(B);

  // ---- fast path: the whole batch fits one pass of the block ------------------
  // (same arithmetic as the general passes below, with one load of the lengths and
  // one scan of the costs instead of two)
  if (B <= kThreads) {
    const int b = tid;
    const int n = (b < B) ? len_of(b) : 0;
    const int nb = n > 0 ? (n + kBlockSize - 1) / kBlockSize : 0;
    const int64_t nt = (nb + kBlocksPerTile - 1) / kBlocksPerTile;
    const int64_t cost = nb > 0 ? nt + kSchedOverheadTiles : 0;
    int64_t total;
    const int64_t pre = block_exclusive_scan<kThreads>(cost, scratch, &total);
    int64_t cap = (total + P - 1) / P;
    if (cap < kSchedMinCap) cap = kSchedMinCap;
    for (int q = tid; q < kMaxWorkers; q += kThreads) {
      part_start[2 * q] = B;
      part_start[2 * q + 1] = 0;
    }
    __syncthreads();
    int64_t ns = 0;
    if (b < B) {
      nblk_out[b] = nb;
      if (nb > 0) {
        const int64_t first_pos = pre + kSchedOverheadTiles;
        const int64_t p0 = first_pos / cap;
        const int64_t p1 = (first_pos + nt - 1) / cap;
        first_part[b] = (int32_t)p0;
        ns = p1 - p0 + 1;
        const int64_t lo = (pre + cap - 1) / cap;
        const int64_t hi = (pre + cost - 1) / cap;
        for (int64_t q = lo; q <= hi && q < P; ++q) {
          const int64_t j = q * cap - first_pos;  // first tile of partition q
          part_start[2 * q] = b;
          part_start[2 * q + 1] = (int32_t)(j > 0 ? j * kBlocksPerTile : 0);
        }
      } else {
        first_part[b] = 0;
      }
      num_splits[b] = (int32_t)ns;
    }
    int64_t total_slots;
    const int64_t ex = block_exclusive_scan<kThreads>(ns, scratch, &total_slots);
    if (b < B) split_prefix[b] = (int32_t)ex;
    __syncthreads();
    for (int q = tid; q < kMaxWorkers; q += kThreads) {
      if (q + 1 < P) {
        part_end[2 * q] = part_start[2 * (q + 1)];
        part_end[2 * q + 1] = part_start[2 * (q + 1) + 1];
      } else {
        part_end[2 * q] = B;
        part_end[2 * q + 1] = 0;
      }
    }
    if (tid == 0) {
      meta[kHdrMagic] = kMetaMagic;
      meta[kHdrB] = B;
      meta[kHdrSq] = s_q;
      meta[kHdrH] = H;
      meta[kHdrNumParts] = P;
      meta[kHdrNumTiles] = T;
      meta[kHdrCap] = (int32_t)cap;
      meta[kHdrTotalSlots] = (int32_t)total_slots;
      meta[kHdrNumWorkers] = num_workers;
      meta[kHdrOverhead] = kSchedOverheadTiles;
      for (int i = kHdrOverhead + 1; i < kHdrWords; ++i) meta[i] = 0;
      meta[kHdrTokens] = len_of.rep;
      meta[kHdrTokCausal] = len_of.rep ? len_of.causal : 0;
    }
    return;
  }

  // ---- pass 1: total cost -------------------------------------------------
  int64_t total = 0;
  for (int base = 0; base < B; base += kThreads) {
    const int b = base + tid;
    int64_t cost = 0;
    if (b < B) {
      const int n = len_of(b);
      const int nb = n > 0 ? (n + kBlockSize - 1) / kBlockSize : 0;
      nblk_out[b] = nb;
      cost = nb > 0 ? (nb + kBlocksPerTile - 1) / kBlocksPerTile + kSchedOverheadTiles : 0;
    }
    int64_t t;
    block_exclusive_scan<kThreads>(cost, scratch, &t);
    total += t;
  }
  int64_t cap = (total + P - 1) / P;
  if (cap < kSchedMinCap) cap = kSchedMinCap;

  // default partition starts: past the end
  for (int p = tid; p < kMaxWorkers; p += kThreads) {
    part_start[2 * p] = B;
    part_start[2 * p + 1] = 0;
  }
  if (tid == 0) s_carry = 0;
  __syncthreads();

  // ---- pass 2: per-sequence splits and partition starts -------------------
  for (int base = 0; base < B; base += kThreads) {
    const int b = base + tid;
    int64_t cost = 0;
    int nb = 0;
    if (b < B) {
      const int n = len_of(b);
      nb = n > 0 ? (n + kBlockSize - 1) / kBlockSize : 0;
      cost = nb > 0 ? (nb + kBlocksPerTile - 1) / kBlocksPerTile + kSchedOverheadTiles : 0;
    }
    int64_t chunk_total;
    const int64_t pre = s_carry + block_exclusive_scan<kThreads>(cost, scratch, &chunk_total);
    if (b < B) {
      if (nb > 0) {
        const int64_t first_pos = pre + kSchedOverheadTiles;
        const int64_t nt = (nb + kBlocksPerTile - 1) / kBlocksPerTile;
        const int64_t p0 = first_pos / cap;
        const int64_t p1 = (first_pos + nt - 1) / cap;
        first_part[b] = (int32_t)p0;
        num_splits[b] = (int32_t)(p1 - p0 + 1);
        // partitions whose start position falls in [pre, pre + cost)
        const int64_t lo = (pre + cap - 1) / cap;
        const int64_t hi = (pre + cost - 1) / cap;
        for (int64_t p = lo; p <= hi && p < P; ++p) {
          const int64_t j = p * cap - first_pos;  // first tile of partition p
          part_start[2 * p] = b;
          part_start[2 * p + 1] = (int32_t)(j > 0 ? j * kBlocksPerTile : 0);
        }
      } else {
        first_part[b] = 0;
        num_splits[b] = 0;
      }
    }
    __syncthreads();
    if (tid == 0) s_carry += chunk_total;
    __syncthreads();
  }

  // ---- pass 3: split prefix ------------------------------------------------
  if (tid == 0) s_carry = 0;
  __syncthreads();
  for (int base = 0; base < B; base += kThreads) {
    const int b = base + tid;
    const int64_t v = (b < B) ? num_splits[b] : 0;
    int64_t chunk_total;
    const int64_t ex = s_carry + block_exclusive_scan<kThreads>(v, scratch, &chunk_total);
    if (b < B) split_prefix[b] = (int32_t)ex;
    __syncthreads();
    if (tid == 0) s_carry += chunk_total;
    __syncthreads();
  }
  if (tid == 0) s_total = s_carry;
  __syncthreads();

  // ---- partition ends + header ---------------------------------------------
  for (int p = tid; p < kMaxWorkers; p += kThreads) {
    if (p + 1 < P) {
      part_end[2 * p] = part_start[2 * (p + 1)];
      part_end[2 * p + 1] = part_start[2 * (p + 1) + 1];
    } else {
      part_end[2 * p] = B;
      part_end[2 * p + 1] = 0;
    }
  }
  if (tid == 0) {
    meta[kHdrMagic] = kMetaMagic;
    meta[kHdrB] = B;
    meta[kHdrSq] = s_q;
    meta[kHdrH] = H;
    meta[kHdrNumParts] = P;
    meta[kHdrNumTiles] = T;
    meta[kHdrCap] = (int32_t)cap;
    meta[kHdrTotalSlots] = (int32_t)s_total;
    meta[kHdrNumWorkers] = num_workers;
    meta[kHdrOverhead] = kSchedOverheadTiles;
    for (int i = kHdrOverhead + 1; i < kHdrWords; ++i) meta[i] = 0;
    meta[kHdrTokens] = len_of.rep;
    meta[kHdrTokCausal] = len_of.rep ? len_of.causal : 0;
  }
}

}  // namespace

cudaError_t launch_metadata(const int32_t* seqlens, int B, int s_q, int H, int num_workers,
                            int32_t* meta, cudaStream_t stream, const int32_t* q_lens, int rep, int causal) {
  const Lengths len_of{seqlens, q_lens, rep, causal};
  if (B <= 256)
    metadata_kernel<256><<<1, 256, 0, stream>>>(len_of, B, s_q, H, num_workers, meta);
  else
    metadata_kernel<1024><<<1, 1024, 0, stream>>>(len_of, B, s_q, H, num_workers, meta);
  return cudaGetLastError();
}

}  // namespace mla
