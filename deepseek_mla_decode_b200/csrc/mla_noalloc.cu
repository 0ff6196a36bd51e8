// mla_decode_noalloc: the decode entry point for callers that cannot allocate device
// memory.
//
// Some callers of this library may not call cudaMalloc at all: a serving engine
// whose memory pool has already reserved the whole device (a new allocation would
// fail or fragment the pool), a plugin that is handed only input and output
// pointers by its host framework, or a latency-critical decode loop where
// cudaMalloc's implicit device synchronisation is not acceptable.  mla_decode needs
// a workspace for split partial results; this variant takes its workspace from a
// fixed-size array compiled into the library instead.
//
// The array is a file-scope __device__ array of kStaticScratchBytes: every GPU that
// loads this library holds it until the process exits.  Host code cannot use the
// array's name as a device address, so on the first call on each device (with that
// device current) the address is looked up once with cudaGetSymbolAddress and cached.
#include <cuda_runtime.h>
#include <cstdint>
#include <mutex>
#include "../../include/mla_decode.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;  // 64 MiB per device
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

mla_status_t static_scratch(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_DEVICE;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return MLA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *ptr = g_scratch_addr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" mla_status_t mla_decode_noalloc(const void* q_nope, const void* q_pe, const void* kv_cache,
                                           int64_t num_blocks, const int32_t* block_table, int max_blocks,
                                           const int32_t* cache_seqlens, int B, int s_q, int H,
                                           float softmax_scale, int causal, const void* metadata,
                                           size_t metadata_bytes, void* out, float* lse, int32_t* status,
                                           void* stream) {
  size_t need = 0;
  mla_status_t st = mla_workspace_size(B, s_q, H, &need);
  if (st != MLA_OK) return st;
  if (need > kStaticScratchBytes) return MLA_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  st = static_scratch(&scratch);
  if (st != MLA_OK) return st;
  return mla_decode(q_nope, q_pe, kv_cache, num_blocks, block_table, max_blocks, cache_seqlens, B, s_q, H,
                    softmax_scale, causal, metadata, metadata_bytes, scratch, kStaticScratchBytes, out, lse,
                    status, stream);
}
