// LSE-combine kernel: merges the normalised partial outputs of split sequences.
//
// A sequence cut into S pieces has, per query row, partial outputs O_s (each already
// divided by its own softmax sum) and their log-sum-exps lse_s.  The exact merge is
//     lse = ln sum_s exp(lse_s),      out = sum_s exp(lse_s - lse) * O_s
// (split-K merge; "DeepSeek speed test / FA3" article, section 2.1 names the split and
// the softmax_lse side output).  HBM-bound: one warp per query row streams the S
// partial rows with 16-byte loads and writes the bf16 row once.
//
// Grid (P, ceil(M / 8)): block x = p looks at partition p's first block; a split
// sequence is exactly one whose cut opens a partition mid-sequence, and the first such
// partition (first_part + 1) owns its merge, so only blocks with work touch memory.
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

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __launch_bounds__(kWarps * 32) combine_kernel(
    const int32_t* __restrict__ meta, const int32_t* __restrict__ seqlens, const int32_t* __restrict__ q_lens,
    int max_blocks, int B, int s_q, int M, const float* __restrict__ part_o, const float* __restrict__ part_lse,
    __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  // launched as a programmatic dependent of the attention kernel: wait for it
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int part = blockIdx.x;
  if (part == 0) return;
  const int b = meta[off_part_start() + 2 * part];
  if (b >= B || meta[off_part_start() + 2 * part + 1] == 0) return;  // partition opens a sequence
  if (meta[off_first_part(B) + b] + 1 != part) return;              // a later cut of the same sequence
  const int n = seqlens[b];
  // rows written as NaN already: invalid length, or a schedule built for another length
  if (n < 0 || (int64_t)n > (int64_t)max_blocks * kBlockSize) return;
  if (meta[off_nblk() + b] != (n + kBlockSize - 1) / kBlockSize) return;
  const int ql = q_lens ? q_lens[b] : s_q;
  if (ql < 0 || ql > s_q) return;  // invalid query count: NaN rows written already
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.y * kWarps + warp;
  if (row >= M) return;
  // a row tile holding only padding tokens had no pieces; its rows are written already
  if ((row / kRowsPerTile) * kRowsPerTile >= ql * (M / s_q)) return;
  const int ns = meta[off_num_splits(B) + b];
  uint2* orow = reinterpret_cast<uint2*>(out + ((int64_t)b * M + row) * kDLatent);
  const int64_t slot0 = meta[off_split_prefix(B) + b];
  // pass 1: max and sum over the partial lse values (every lane redundantly)
  float m = -INFINITY;
  bool any_nan = false;
  for (int s = 0; s < ns; ++s) {
    const float l = part_lse[(slot0 + s) * M + row];
    any_nan |= (l != l);
    m = fmaxf(m, l);
  }
  float res_lse;
  float4 acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (any_nan) {
    res_lse = __int_as_float(0x7fc00000);
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] = make_float4(res_lse, res_lse, res_lse, res_lse);
  } else if (m == -INFINITY) {
    res_lse = -INFINITY;
  } else {
    float z = 0.f;
    for (int s = 0; s < ns; ++s) z += __expf(part_lse[(slot0 + s) * M + row] - m);
    res_lse = m + __logf(z);
    for (int s = 0; s < ns; ++s) {
      const float w = __expf(part_lse[(slot0 + s) * M + row] - res_lse);
      const float4* src = reinterpret_cast<const float4*>(part_o + ((slot0 + s) * M + row) * kDLatent);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 v = src[k * 32 + lane];
        acc[k].x += w * v.x;
        acc[k].y += w * v.y;
        acc[k].z += w * v.z;
        acc[k].w += w * v.w;
      }
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k)
    orow[k * 32 + lane] = make_uint2(pack_bf16x2(acc[k].x, acc[k].y), pack_bf16x2(acc[k].z, acc[k].w));
  if (lane == 0) lse[(int64_t)b * M + row] = res_lse;
}

}  // namespace

cudaError_t launch_combine(const int32_t* meta, const int32_t* seqlens, const int32_t* q_lens, int max_blocks,
                           int B, int s_q, int M, int P, const float* part_o, const float* part_lse, void* out, float* lse,
                           cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P, (M + kWarps - 1) / kWarps);
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, combine_kernel, meta, seqlens, q_lens, max_blocks, B, s_q, M, part_o, part_lse,
                            reinterpret_cast<__nv_bfloat16*>(out), lse);
}

}  // namespace mla
