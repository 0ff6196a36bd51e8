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
#include <algorithm>
#include <cstdint>
#include "sage_internal.h"

namespace mla {
namespace sage {
namespace {

// Q / K rows: a warp quantises four (token, head) rows of 192 bf16 at a time, eight
// lanes per row, 24 values (three 16-byte loads) per lane; grid-stride over the rows.
constexpr int kRowLanes = 8, kRowVals = kDQK / kRowLanes;  // 24
__global__ void __launch_bounds__(256) quant_rows_kernel(const __nv_bfloat16* __restrict__ x, int8_t* __restrict__ q8,
                                                        float* __restrict__ scale, int S, int S_pad, int H) {
  const int lane = threadIdx.x & 31, sub = lane & (kRowLanes - 1);
  const int64_t nrows = (int64_t)S_pad * H;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t row = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 4 + (lane >> 3); ;
       row += warps * 4) {
    // the warp's four rows advance together; lanes past the last row idle but stay in
    // the shuffles
    const int64_t row0 = row - (lane >> 3);
    if (row0 >= nrows) break;
    const bool have = row < nrows;
    const int t = have ? (int)(row / H) : 0, h = have ? (int)(row % H) : 0;
    float v[kRowVals];
    if (have && t < S) {
      const uint4* src = reinterpret_cast<const uint4*>(x + ((int64_t)t * H + h) * kDQK + sub * kRowVals);
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        const uint4 w = src[k];
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[8 * k + 2 * i] = __uint_as_float(u[i] << 16);
          v[8 * k + 2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < kRowVals; ++i) v[i] = 0.f;
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < kRowVals; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
    for (int o = kRowLanes / 2; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = __fdiv_rn(amax, 127.0f);
    uint32_t packed[kRowVals / 4] = {0u, 0u, 0u, 0u, 0u, 0u};
    if (s > 0.f) {
#pragma unroll
      for (int i = 0; i < kRowVals; ++i) {
        int c = __float2int_rn(__fdiv_rn(v[i], s));
        c = max(-127, min(127, c));
        packed[i >> 2] |= (uint32_t)(c & 0xff) << (8 * (i & 3));
      }
    }
    if (have) {
      uint2* dst = reinterpret_cast<uint2*>(q8 + ((int64_t)h * S_pad + t) * kDQK + sub * kRowVals);
#pragma unroll
      for (int k = 0; k < 3; ++k) dst[k] = make_uint2(packed[2 * k], packed[2 * k + 1]);
      if (sub == 0) scale[(int64_t)h * S_pad + t] = s;
    }
  }
}

// Channel maxima of V: block (token chunk, head); thread = (token row of 16, group of
// 8 channels), 16-byte loads; the block reduces its maxima in shared memory, then one
// integer atomicMax per channel (the maxima of non-negative floats order like their
// bit patterns).
constexpr int kVChunk = 256;
__global__ void __launch_bounds__(256) vmax_kernel(const __nv_bfloat16* __restrict__ v, uint32_t* __restrict__ vmax,
                                                   int S, int H) {
  __shared__ float red[16][kDV];
  const int h = blockIdx.y, g = threadIdx.x & 15, tr = threadIdx.x >> 4;  // channels 8 g .. 8 g + 7
  const int t0 = blockIdx.x * kVChunk, t1 = min(S, t0 + kVChunk);
  float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int t = t0 + tr; t < t1; t += 16) {
    const uint4 w = reinterpret_cast<const uint4*>(v + ((int64_t)t * H + h) * kDV)[g];
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      m[2 * i] = fmaxf(m[2 * i], fabsf(__uint_as_float(u[i] << 16)));
      m[2 * i + 1] = fmaxf(m[2 * i + 1], fabsf(__uint_as_float(u[i] & 0xffff0000u)));
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) red[tr][8 * g + i] = m[i];
  __syncthreads();
  if (threadIdx.x < kDV) {
    float r = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) r = fmaxf(r, red[k][threadIdx.x]);
    atomicMax(vmax + h * kDV + threadIdx.x, __float_as_uint(r));
  }
}

__device__ __forceinline__ uint32_t e4m3x2_rn(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// V codes, transposed through shared memory: block (64-token chunk, head) reads 64
// tokens x 128 channels with 16-byte loads (thread = token row of 16, group of 8
// channels, four passes) and writes 128 channel rows of 64 codes.
constexpr int kVtTokens = 64;
__global__ void __launch_bounds__(256) vquant_kernel(const __nv_bfloat16* __restrict__ v,
                                                     const uint32_t* __restrict__ vmax, uint8_t* __restrict__ vt8,
                                                     float* __restrict__ sv, int S, int S_pad, int H) {
  __shared__ uint8_t tile[kDV][kVtTokens + 4];
  const int h = blockIdx.y, t0 = blockIdx.x * kVtTokens;
  const int g = threadIdx.x & 15, tr = threadIdx.x >> 4;  // channels 8 g .. 8 g + 7; token row tr of 16
  float sc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) sc[i] = __fdiv_rn(__uint_as_float(vmax[h * kDV + 8 * g + i]), 448.0f);
#pragma unroll
  for (int pass = 0; pass < kVtTokens / 16; ++pass) {
    const int tl = pass * 16 + tr, t = t0 + tl;
    float x[8];
    if (t < S) {
      const uint4 w = reinterpret_cast<const uint4*>(v + ((int64_t)t * H + h) * kDV)[g];
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(u[i] << 16);
        x[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const bool l0 = sc[i] > 0.f && t < S, l1 = sc[i + 1] > 0.f && t < S;
      uint32_t c = e4m3x2_rn(l0 ? __fdiv_rn(x[i], sc[i]) : 0.f, l1 ? __fdiv_rn(x[i + 1], sc[i + 1]) : 0.f);
      if (!l0) c &= 0xff00u;
      if (!l1) c &= 0x00ffu;
      tile[8 * g + i][tl] = (uint8_t)(c & 0xff);
      tile[8 * g + i + 1][tl] = (uint8_t)(c >> 8);
    }
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
  if (blockIdx.x == 0 && tr == 0) {
#pragma unroll
    for (int i = 0; i < 8; ++i) sv[h * kDV + 8 * g + i] = sc[i];
  }
}

}  // namespace

cudaError_t launch_quantize(const void* q, const void* k, const void* v, int S, int H, const Workspace& ws,
                            cudaStream_t stream) {
  const int S_pad = padded_len(S);
  const int64_t rows = (int64_t)S_pad * H;
  // 32 rows per block of 8 warps, at most 16 blocks per SM's worth (grid-stride beyond)
  const unsigned grid_rows = (unsigned)std::min<int64_t>((rows + 31) / 32, 148 * 16);
  quant_rows_kernel<<<grid_rows, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(q), ws.q8, ws.sq, S, S_pad, H);
  quant_rows_kernel<<<grid_rows, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(k), ws.k8, ws.sk, S, S_pad, H);
  cudaError_t e = cudaMemsetAsync(ws.vmax, 0, (size_t)H * kDV * sizeof(uint32_t), stream);
  if (e != cudaSuccess) return e;
  vmax_kernel<<<dim3((S + kVChunk - 1) / kVChunk, H), 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(v),
                                                                          ws.vmax, S, H);
  vquant_kernel<<<dim3(S_pad / kVtTokens, H), 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(v), ws.vmax,
                                                                 ws.vt8, ws.sv, S, S_pad, H);
  return cudaGetLastError();
}

}  // namespace sage
}  // namespace mla
