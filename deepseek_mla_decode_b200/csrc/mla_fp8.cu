// FP8 (e4m3) latent cache: per-token quantisation of bf16 cache rows into the packed
// 656-byte row the FP8 decode reads.
//
// 8-bit KV-cache inference is one of the serving capabilities listed in the Paddle 3.0
// inference upgrade article (closing capabilities list); scaling each token's cached
// vector by its own max-abs value follows the per-token quantised KV cache of the
// "DeepSeek speed test" article, section 3.1.  The row format is this library's own:
//     bytes [0, 512)    e4m3 codes of c_kv / scale     (OCP E4M3FN, no infinities)
//     bytes [512, 640)  k_pe / scale as 64 bf16         (RoPE keys keep 16 bits)
//     bytes [640, 644)  fp32 scale = max|row| / 448     (over all 576 values;
//                                                        448 = largest finite e4m3)
//     bytes [644, 656)  zero
// code_i = e4m3(c_i / scale): the quotient is an IEEE fp32 division, rounded to the
// nearest e4m3 value (ties to even) and saturated to +-448; k_pe'_j = bf16(k_pe_j /
// scale), the fp32 quotient rounded to nearest even.  A row of zeros gets scale 0 and
// stores zeros.  The dequantised row is scale * [e4m3(code) | k_pe'], so one scale
// multiplies the whole score q . k and the whole value row.
//
// One warp per cache row: lane l holds c_kv[16 l, 16 l + 16) and lanes 0-7 also hold
// k_pe[8 l, 8 l + 8); a warp max gives the scale, and each lane writes its 16 codes
// (and its 8 scaled k_pe values) as 16-byte stores.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>
#include "mla_internal.h"
#include "../../include/mla_decode.h"

namespace mla {
namespace {

constexpr int kWarpsPerBlock = 8;

// two fp32 -> two e4m3 (round to nearest even, saturating), lo in the low byte
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__global__ void __launch_bounds__(kWarpsPerBlock * 32) quantize_kernel(const __nv_bfloat16* __restrict__ kv,
                                                                      uint8_t* __restrict__ out, int64_t rows) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  if (row >= rows) return;
  const __nv_bfloat16* src = kv + row * kDQK;
  uint8_t* dst = out + row * kRowBytes8;
  // c_kv[16 lane .. 16 lane + 15]
  const uint4 a = reinterpret_cast<const uint4*>(src)[2 * lane];
  const uint4 b = reinterpret_cast<const uint4*>(src)[2 * lane + 1];
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  float c[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c[2 * i] = __uint_as_float(w[i] << 16);
    c[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
  // k_pe[8 lane .. 8 lane + 7] on lanes 0-7
  float k[8];
  {
    const uint4 e = lane < 8 ? reinterpret_cast<const uint4*>(src + kDLatent)[lane] : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t v[4] = {e.x, e.y, e.z, e.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      k[2 * i] = __uint_as_float(v[i] << 16);
      k[2 * i + 1] = __uint_as_float(v[i] & 0xffff0000u);
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(c[i]));
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(k[i]));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float scale = __fdiv_rn(amax, 448.0f);
  uint32_t q[4] = {0u, 0u, 0u, 0u};
  uint32_t kq[4] = {0u, 0u, 0u, 0u};
  if (scale > 0.f) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = e4m3x2(__fdiv_rn(c[4 * i], scale), __fdiv_rn(c[4 * i + 1], scale));
      const uint32_t hi = e4m3x2(__fdiv_rn(c[4 * i + 2], scale), __fdiv_rn(c[4 * i + 3], scale));
      q[i] = lo | (hi << 16);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(__fdiv_rn(k[2 * i], scale), __fdiv_rn(k[2 * i + 1], scale));
      kq[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
  }
  reinterpret_cast<uint4*>(dst)[lane] = make_uint4(q[0], q[1], q[2], q[3]);
  // scaled k_pe (128 bytes) by lanes 0-7, then the scale and the zero pad by lane 8
  if (lane < 8) {
    reinterpret_cast<uint4*>(dst + kOffKpe8)[lane] = make_uint4(kq[0], kq[1], kq[2], kq[3]);
  } else if (lane == 8) {
    reinterpret_cast<uint4*>(dst + kOffScale8)[0] = make_uint4(__float_as_uint(scale), 0u, 0u, 0u);
  }
}

}  // namespace
}  // namespace mla

extern "C" mla_status_t mla_quantize_kv_fp8(const void* kv_cache, void* kv_fp8, int64_t rows, void* stream) {
  if (!kv_cache || !kv_fp8 || rows < 0) return MLA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(kv_cache) & 15u) || (reinterpret_cast<uintptr_t>(kv_fp8) & 15u))
    return MLA_ERR_INVALID_ARG;
  if (rows == 0) return MLA_OK;
  int sms = 0;
  mla_status_t st = mla_device_sm_count(&sms);
  if (st != MLA_OK) return st;
  const int64_t blocks = (rows + mla::kWarpsPerBlock - 1) / mla::kWarpsPerBlock;
  if (blocks > 0x7fffffffLL) return MLA_ERR_INVALID_ARG;
  mla::quantize_kernel<<<(unsigned)blocks, mla::kWarpsPerBlock * 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(kv_cache), static_cast<uint8_t*>(kv_fp8), rows);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
