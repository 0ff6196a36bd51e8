// Internal layout shared by the quantised prefill attention's host entry points, its
// quantisers (sage_quant.cu) and its attention kernel (sage_attn.cu).
#pragma once
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

namespace mla {
namespace sage {

constexpr int kDQK = 192;     // Q / K head dimension (128 without RoPE + 64 RoPE)
constexpr int kDV = 128;      // V / output head dimension
constexpr int kBlockM = 128;  // query rows per CTA
constexpr int kBlockN = 128;  // keys per pipeline step

inline int padded_len(int S) { return (S + kBlockN - 1) / kBlockN * kBlockN; }

// Views into the caller's workspace (see sage_quant.cu for the layout).
struct Workspace {
  int8_t* q8;
  int8_t* k8;
  uint8_t* vt8;
  float* sq;
  float* sk;
  float* sv;
  uint32_t* vmax;
};

inline size_t workspace_bytes(int S, int H) {
  const size_t sp = (size_t)padded_len(S), h = (size_t)H;
  return 2 * h * sp * kDQK + h * kDV * sp + 2 * h * sp * sizeof(float) + 2 * h * kDV * sizeof(float);
}

inline Workspace carve(void* base, int S, int H) {
  const size_t sp = (size_t)padded_len(S), h = (size_t)H;
  uint8_t* p = static_cast<uint8_t*>(base);
  Workspace w;
  w.q8 = reinterpret_cast<int8_t*>(p);
  p += h * sp * kDQK;
  w.k8 = reinterpret_cast<int8_t*>(p);
  p += h * sp * kDQK;
  w.vt8 = p;
  p += h * kDV * sp;
  w.sq = reinterpret_cast<float*>(p);
  p += h * sp * sizeof(float);
  w.sk = reinterpret_cast<float*>(p);
  p += h * sp * sizeof(float);
  w.sv = reinterpret_cast<float*>(p);
  p += h * kDV * sizeof(float);
  w.vmax = reinterpret_cast<uint32_t*>(p);
  return w;
}

cudaError_t launch_quantize(const void* q, const void* k, const void* v, int S, int H, const Workspace& ws,
                            cudaStream_t stream);

}  // namespace sage
}  // namespace mla
