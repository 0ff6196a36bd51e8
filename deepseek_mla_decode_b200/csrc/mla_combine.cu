// LSE-combine kernel: merges the normalised partial outputs of split sequences.
//
// A sequence cut into S pieces has, per query row, partial outputs O_s (each already
// divided by its own softmax sum) and their log-sum-exps lse_s.  The exact merge is
//     lse = ln sum_s exp(lse_s),      out = sum_s exp(lse_s - lse) * O_s
// (split-K merge; "DeepSeek speed test / FA3" article, section 2.1 names the split and
// the softmax_lse side output).  HBM-bound: the warps of a query row stream its S
// partial rows with 16-byte loads and write the bf16 row once.  Batches of many
// sequences (few splits each, many rows) take one warp per row with two splits in
// flight; batches of few sequences (long ones, cut into many splits, few rows) take
// four warps per row, each over 128 columns with sixteen splits in flight.
//
// Grid (X, ceil(M * c / 8)), c warps per row.  With more sequences than partitions,
// X = P and block x = p looks at partition p's first block: a split sequence is
// exactly one whose cut opens a partition mid-sequence, and the first such partition
// (first_part + 1) owns its merge, so only blocks with work read more.  With no more
// sequences than partitions, X = B and block x = b takes sequence b if it has two or
// more pieces: no idle partitions' blocks, and one round trip less (b is known).
// Rows of sequences that no partition covers (no visible key, invalid length, a block
// count in the metadata that does not match the length) are written by the attention
// kernel.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>
#include "mla_internal.h"

namespace mla {

namespace {

constexpr int kWarps = 8;
constexpr int kWideBatch = 16;  // batches below this many sequences take four warps per row

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// kColParts warps per query row, each over 512 / kColParts columns; kGroup partial rows
// in flight per lane (32 registers of loads for one warp per row and two splits, 64 for
// four warps per row and sixteen splits); kBySeq: block x is a sequence (else a
// partition)
template <int kColParts, int kGroup, bool kBySeq>
__global__ void __launch_bounds__(kWarps * 32) combine_kernel(
    const int32_t* __restrict__ meta, const int32_t* __restrict__ seqlens, const int32_t* __restrict__ q_lens,
    int max_blocks, int B, int s_q, int M, const float* __restrict__ part_o, const float* __restrict__ part_lse,
    __nv_bfloat16* __restrict__ out, float* __restrict__ lse, int tok_rep, int tok_causal) {
  // launched as a programmatic dependent of the attention kernel: wait for it
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // Dependent round trips to memory: the partition's start (by partition only), then
  // every word of the sequence at once, then the partial lse values together with the
  // first partial rows (the rest of the kernel is arithmetic on registers).
  int b, part = 0;
  if constexpr (kBySeq) {
    b = blockIdx.x;
  } else {
    part = blockIdx.x;
    if (part == 0) return;
    b = meta[off_part_start() + 2 * part];
    const int k0 = meta[off_part_start() + 2 * part + 1];
    if (b >= B || k0 == 0) return;  // partition opens a sequence (or is empty)
  }
  const int fp = meta[off_first_part(B) + b];
  const int nblk = meta[off_nblk() + b];
  const int ns = meta[off_num_splits(B) + b];
  const int slot0 = meta[off_split_prefix(B) + b];
  // with a token schedule, sequence b is one token of real sequence b / tok_rep (its
  // length from token_seq_len, one query token)
  const int r = tok_rep ? b / tok_rep : b;
  const int nr = seqlens[r];
  const int qr = (q_lens != nullptr) ? q_lens[r] : (tok_rep ? tok_rep : s_q);
  const int n = !tok_rep ? nr
                         : ((int64_t)nr > (int64_t)max_blocks * kBlockSize ? -1
                                                                            : token_seq_len(nr, qr, b - r * tok_rep, tok_rep,
                                                                                            tok_causal));
  const int ql = tok_rep ? 1 : qr;
  if constexpr (kBySeq) {
    if (ns < 2) return;  // one piece: its rows were written by the attention kernel
  } else {
    if (fp + 1 != part) return;  // a later cut of the same sequence
  }
  // rows written as NaN already: invalid length, or a schedule built for another length
  if (n < 0 || (int64_t)n > (int64_t)max_blocks * kBlockSize) return;
  if (nblk != (n + kBlockSize - 1) / kBlockSize) return;
  if (ql < 0 || ql > s_q) return;  // invalid query count: NaN rows written already
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wid = blockIdx.y * kWarps + warp;
  const int row = wid / kColParts, part_col = wid % kColParts;
  if (row >= M) return;
  // a row tile holding only padding tokens had no pieces; its rows are written already
  if ((row / kRowsPerTile) * kRowsPerTile >= ql * (M / s_q)) return;
  const float* lse_row = part_lse + (int64_t)slot0 * M + row;  // split s at [s * M]
  constexpr int kF4 = 4 / kColParts;  // float4s per lane and split
  const float4* o_row =
      reinterpret_cast<const float4*>(part_o + ((int64_t)slot0 * M + row) * kDLatent) + part_col * 32 * kF4 + lane;
  const int64_t o_split = (int64_t)M * (kDLatent / 4);  // float4s between splits
  float4 v[kGroup][kF4];
  auto load_group = [&](int s0) {
#pragma unroll
    for (int j = 0; j < kGroup; ++j)
#pragma unroll
      for (int k = 0; k < kF4; ++k)
        v[j][k] = (s0 + j < ns) ? __ldg(o_row + (int64_t)(s0 + j) * o_split + 32 * k) : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  load_group(0);
  // lse of split s is held by lane s % 32 (splits past 32 by further chunks)
  const float l_lane = (lane < ns) ? __ldg(lse_row + (int64_t)lane * M) : -INFINITY;
  float m = l_lane;
  bool any_nan = (l_lane != l_lane);
  for (int c = 32; c < ns; c += 32) {
    const float l = (c + lane < ns) ? __ldg(lse_row + (int64_t)(c + lane) * M) : -INFINITY;
    any_nan |= (l != l);
    m = fmaxf(m, l);
  }
  any_nan = __any_sync(0xffffffffu, any_nan);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float res_lse;
  float4 acc[kF4];
#pragma unroll
  for (int k = 0; k < kF4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (any_nan) {
    res_lse = __int_as_float(0x7fc00000);
#pragma unroll
    for (int k = 0; k < kF4; ++k) acc[k] = make_float4(res_lse, res_lse, res_lse, res_lse);
  } else if (m == -INFINITY) {
    res_lse = -INFINITY;
  } else {
    // z = sum_s exp(lse_s - m), every lane's splits then a butterfly over the lanes
    float z = (lane < ns) ? __expf(l_lane - m) : 0.f;
    for (int c = 32; c < ns; c += 32)
      if (c + lane < ns) z += __expf(__ldg(lse_row + (int64_t)(c + lane) * M) - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    res_lse = m + __logf(z);
    // out = sum_s exp(lse_s - lse) O_s, accumulated in split order
    for (int s0 = 0; s0 < ns; s0 += kGroup) {
      if (s0 > 0) load_group(s0);
#pragma unroll
      for (int j = 0; j < kGroup; ++j) {
        const int s = s0 + j;
        if (s < ns) {  // warp-uniform
          const float l = (s < 32) ? __shfl_sync(0xffffffffu, l_lane, s) : __ldg(lse_row + (int64_t)s * M);
          const float w = __expf(l - res_lse);
#pragma unroll
          for (int k = 0; k < kF4; ++k) {
            acc[k].x += w * v[j][k].x;
            acc[k].y += w * v[j][k].y;
            acc[k].z += w * v[j][k].z;
            acc[k].w += w * v[j][k].w;
          }
        }
      }
    }
  }
  uint2* orow = reinterpret_cast<uint2*>(out + ((int64_t)b * M + row) * kDLatent) + part_col * 32 * kF4;
#pragma unroll
  for (int k = 0; k < kF4; ++k)
    orow[k * 32 + lane] = make_uint2(pack_bf16x2(acc[k].x, acc[k].y), pack_bf16x2(acc[k].z, acc[k].w));
  if (lane == 0 && part_col == 0) lse[(int64_t)b * M + row] = res_lse;
}

}  // namespace

cudaError_t launch_combine(const int32_t* meta, const int32_t* seqlens, const int32_t* q_lens, int max_blocks,
                           int B, int s_q, int M, int P, const float* part_o, const float* part_lse, void* out, float* lse,
                           cudaStream_t stream, int tok_rep, int tok_causal) {
  // few sequences: long ones with many splits and few rows to merge
  const bool wide = B < kWideBatch;
  const bool by_seq = wide || B <= P;
  const int parts = wide ? 4 : 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(by_seq ? B : P, (M * parts + kWarps - 1) / kWarps);
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out);
  if (wide)
    return cudaLaunchKernelEx(&cfg, combine_kernel<4, 16, true>, meta, seqlens, q_lens, max_blocks, B, s_q, M, part_o,
                              part_lse, o, lse, tok_rep, tok_causal);
  if (by_seq)
    return cudaLaunchKernelEx(&cfg, combine_kernel<1, 2, true>, meta, seqlens, q_lens, max_blocks, B, s_q, M, part_o,
                              part_lse, o, lse, tok_rep, tok_causal);
  return cudaLaunchKernelEx(&cfg, combine_kernel<1, 2, false>, meta, seqlens, q_lens, max_blocks, B, s_q, M, part_o,
                            part_lse, o, lse, tok_rep, tok_causal);
}

}  // namespace mla
