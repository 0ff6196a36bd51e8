// Dynamic quantisation for the quantised prefill attention (sage_attn.cu).
//
// Paddle 3.0 inference upgrade article, long-sequence section: Q and K are quantised
// to INT8 and V to FP8 on the fly.  The granularity is this library's reading of it:
//   Q, K: one fp32 scale per (token, head) over the 192 values, s = max|x| / 127,
//         code = rint(x / s) (IEEE fp32 quotient, ties to even); zero rows: s = 0.
//   V:    one fp32 scale per (head, channel) over all tokens, s = max|v| / 448,
//         code = e4m3(v / s) (fp32 quotient, nearest even, saturating).
// Workspace layout (S_pad = S rounded up to 128; pad tokens hold zero codes / scales):
//   q8  int8  [H][S_pad][192]      k8  int8  [H][S_pad][192]
//   vt8 e4m3  [H][128][S_pad]      (V transposed: each channel's codes over the keys,
//                                   the K-major operand layout of the PV product)
//   sq, sk fp32 [H][S_pad]         sv fp32 [H][128]       vmax uint32 [H][128]
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>
#include "sage_internal.h"

namespace mla {
namespace sage {
namespace {

// One warp per (token, head) row of 192 bf16: lanes 0..23 hold 8 values each.
__global__ void __launch_bounds__(256) quant_rows_kernel(const __nv_bfloat16* __restrict__ x, int8_t* __restrict__ q8,
                                                        float* __restrict__ scale, int S, int S_pad, int H) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);  // = token * H + head over S_pad tokens
  if (row >= (int64_t)S_pad * H) return;
  const int t = (int)(row / H), h = (int)(row % H);
  float v[8];
  bool live = lane < kDQK / 8 && t < S;
  if (live) {
    const uint4 w = reinterpret_cast<const uint4*>(x + ((int64_t)t * H + h) * kDQK)[lane];
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(u[i] << 16);
      v[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.f;
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = __fdiv_rn(amax, 127.0f);
  uint32_t packed[2] = {0u, 0u};
  if (s > 0.f) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int c = __float2int_rn(__fdiv_rn(v[i], s));
      c = max(-127, min(127, c));
      packed[i >> 2] |= (uint32_t)(c & 0xff) << (8 * (i & 3));
    }
  }
  int8_t* dst = q8 + ((int64_t)h * S_pad + t) * kDQK;
  if (lane < kDQK / 8) reinterpret_cast<uint2*>(dst)[lane] = make_uint2(packed[0], packed[1]);
  if (lane == 0) scale[(int64_t)h * S_pad + t] = s;
}

// Channel maxima of V: block (token chunk, head), thread = channel; the maxima of
// non-negative floats order like their bit patterns, so an integer atomicMax suffices.
constexpr int kVChunk = 256;
__global__ void __launch_bounds__(kDV) vmax_kernel(const __nv_bfloat16* __restrict__ v, uint32_t* __restrict__ vmax,
                                                   int S, int H) {
  const int h = blockIdx.y, d = threadIdx.x;
  const int t0 = blockIdx.x * kVChunk, t1 = min(S, t0 + kVChunk);
  float m = 0.f;
  for (int t = t0; t < t1; ++t) m = fmaxf(m, fabsf(__bfloat162float(v[((int64_t)t * H + h) * kDV + d])));
  atomicMax(vmax + h * kDV + d, __float_as_uint(m));
}

__device__ __forceinline__ uint32_t e4m3x2_rn(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// V codes, transposed through shared memory: block (64-token chunk, head) reads 64
// tokens x 128 channels and writes 128 channel rows of 64 codes.
constexpr int kVtTokens = 64;
__global__ void __launch_bounds__(256) vquant_kernel(const __nv_bfloat16* __restrict__ v,
                                                     const uint32_t* __restrict__ vmax, uint8_t* __restrict__ vt8,
                                                     float* __restrict__ sv, int S, int S_pad, int H) {
  __shared__ uint8_t tile[kDV][kVtTokens + 4];
  const int h = blockIdx.y, t0 = blockIdx.x * kVtTokens;
  // each thread: one channel pair for 16 tokens
  const int dp = threadIdx.x & 63;       // channel pair (2 dp, 2 dp + 1)
  const int tq = threadIdx.x >> 6;       // token quarter
  const float s0 = __fdiv_rn(__uint_as_float(vmax[h * kDV + 2 * dp]), 448.0f);
  const float s1 = __fdiv_rn(__uint_as_float(vmax[h * kDV + 2 * dp + 1]), 448.0f);
  for (int i = 0; i < kVtTokens / 4; ++i) {
    const int tl = tq * (kVtTokens / 4) + i, t = t0 + tl;
    uint32_t c = 0;
    if (t < S) {
      const __nv_bfloat162 w = reinterpret_cast<const __nv_bfloat162*>(v + ((int64_t)t * H + h) * kDV)[dp];
      const float a = s0 > 0.f ? __fdiv_rn(__low2float(w), s0) : 0.f;
      const float b = s1 > 0.f ? __fdiv_rn(__high2float(w), s1) : 0.f;
      c = e4m3x2_rn(a, b);
      if (!(s0 > 0.f)) c &= 0xff00u;
      if (!(s1 > 0.f)) c &= 0x00ffu;
    }
    tile[2 * dp][tl] = (uint8_t)(c & 0xff);
    tile[2 * dp + 1][tl] = (uint8_t)(c >> 8);
  }
  __syncthreads();
  // 128 rows x 64 bytes out: thread -> (row, 16-byte quarter); two rows per pass
  for (int r = threadIdx.x >> 2; r < kDV; r += 64) {
    const int qd = threadIdx.x & 3;
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint8_t* p = &tile[r][16 * qd + 4 * j];
      w[j] = (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
    }
    reinterpret_cast<uint4*>(vt8 + ((int64_t)h * kDV + r) * S_pad + t0)[qd] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (blockIdx.x == 0) {
    if (tq == 0) {
      sv[h * kDV + 2 * dp] = s0;
      sv[h * kDV + 2 * dp + 1] = s1;
    }
  }
}

}  // namespace

cudaError_t launch_quantize(const void* q, const void* k, const void* v, int S, int H, const Workspace& ws,
                            cudaStream_t stream) {
  const int S_pad = padded_len(S);
  const int64_t rows = (int64_t)S_pad * H;
  const unsigned grid_rows = (unsigned)((rows + 7) / 8);
  quant_rows_kernel<<<grid_rows, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(q), ws.q8, ws.sq, S, S_pad, H);
  quant_rows_kernel<<<grid_rows, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(k), ws.k8, ws.sk, S, S_pad, H);
  cudaError_t e = cudaMemsetAsync(ws.vmax, 0, (size_t)H * kDV * sizeof(uint32_t), stream);
  if (e != cudaSuccess) return e;
  vmax_kernel<<<dim3((S + kVChunk - 1) / kVChunk, H), kDV, 0, stream>>>(static_cast<const __nv_bfloat16*>(v),
                                                                          ws.vmax, S, H);
  vquant_kernel<<<dim3(S_pad / kVtTokens, H), 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(v), ws.vmax,
                                                                 ws.vt8, ws.sv, S, S_pad, H);
  return cudaGetLastError();
}

}  // namespace sage
}  // namespace mla
