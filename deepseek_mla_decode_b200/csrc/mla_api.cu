// Host side of the C ABI declared in include/mla_decode.h: argument validation,
// TMA tensor-map encoding and the launch sequence (schedule kernel; attention kernel +
// LSE-combine kernel).  No device memory is allocated here.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>
#include "mla_internal.h"
#include "sage_internal.h"
#include "../../include/mla_decode.h"

namespace mla {
// tok_* / q_lens + rep: the token schedule (s_q = 1 over B * rep token sequences; see
// token_seq_len in mla_internal.h); zero / null for the per-sequence schedule.
cudaError_t launch_metadata(const int32_t* seqlens, int B, int s_q, int H, int num_workers, int32_t* meta,
                            cudaStream_t stream, const int32_t* q_lens = nullptr, int rep = 0, int causal = 0);
cudaError_t launch_combine(const int32_t* meta, const int32_t* seqlens, const int32_t* q_lens, int max_blocks,
                           int B, int s_q, int M, int P, const float* part_o, const float* part_lse, void* out,
                           float* lse, cudaStream_t stream, int tok_rep = 0, int tok_causal = 0);
cudaError_t decode_kernel_setup(int device);
namespace sage {
cudaError_t attention_setup();
cudaError_t launch_attention(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                             const Workspace& ws, int S, int H, float softmax_scale, void* out, float* lse,
                             int32_t* status, uint64_t timeout_ns, cudaStream_t stream);
}  // namespace sage
cudaError_t launch_decode(bool fp8, const CUtensorMap& tm_kv, const CUtensorMap& tm_kv2,
                          const CUtensorMap* tm_kpe, const CUtensorMap* tm_scl,
                          const CUtensorMap& tm_qn, const CUtensorMap& tm_qp,
                          const CUtensorMap& tm_out, const CUtensorMap& tm_part,
                          const int32_t* block_table, int max_blocks, const int32_t* seqlens,
                          const int32_t* q_lens, const int32_t* meta, int64_t num_blocks, int B, int s_q,
                          int H, float scale, int causal, void* out, float* lse, float* part_o, float* part_lse,
                          int32_t* status, int num_ctas, uint64_t wait_timeout_ns, int inject_stall,
                          cudaStream_t stream, int tok_rep = 0, int tok_causal = 0,
                          const int32_t* tok_q_lens = nullptr);
}  // namespace mla

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  bool ok = false;
  int sm_count = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
constexpr uint64_t kDefaultWaitTimeoutNs = 1000000000ull;  // 1 s
std::atomic<uint64_t> g_wait_timeout_ns{kDefaultWaitTimeoutNs};
std::atomic<int> g_inject_stall{0};
EncodeTiledFn g_encode = nullptr;

// Per-device one-time setup: SM count, architecture check, kernel attributes.
mla_status_t device_info(int* sm_count) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    d.ready = true;
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MLA_ERR_CUDA;
    if (major != 10 || minor != 0) return MLA_ERR_DEVICE;
    if (mla::decode_kernel_setup(dev) != cudaSuccess) return MLA_ERR_CUDA;
    if (mla::sage::attention_setup() != cudaSuccess) return MLA_ERR_CUDA;
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return MLA_ERR_CUDA;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    d.sm_count = sms;
    d.ok = true;
  }
  if (!d.ok) return MLA_ERR_DEVICE;
  *sm_count = d.sm_count;
  return MLA_OK;
}

bool shape_supported(int B, int s_q, int H) {
  if (B < 1 || B > 65536) return false;
  if (s_q < 1 || s_q > 4) return false;
  return H == 16 || H == 32 || H == 64 || H == 128;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_workers_for(int sm_count) {
  int w = sm_count / 2;
  if (w > mla::kMaxWorkers) w = mla::kMaxWorkers;
  return w < 1 ? 1 : w;
}

int parts_for(int num_workers, int s_q, int H) {
  const int T = (s_q * H + mla::kRowsPerTile - 1) / mla::kRowsPerTile;
  const int P = num_workers / T;
  return P < 1 ? 1 : P;
}

bool encode(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box, CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
            CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  cuuint32_t es[4] = {1, 1, 1, 1};
  return g_encode(m, dt, rank, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

namespace mla {
// bf16 tiled tensor map with the 128-byte swizzle (the device must have been checked
// with device_info first, which resolves the driver entry point)
bool encode_tiled_bf16(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
                       const cuuint32_t* box) {
  return g_encode != nullptr && encode(m, base, rank, dims, strides, box);
}
}  // namespace mla

extern "C" {

const char* mla_status_string(mla_status_t s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_WORKSPACE_TOO_SMALL: return "MLA_ERR_WORKSPACE_TOO_SMALL";
    case MLA_ERR_DEVICE: return "MLA_ERR_DEVICE";
  }
  return "MLA_ERR_UNKNOWN";
}

mla_status_t mla_metadata_size(int B, int s_q, int H, size_t* bytes) {
  if (!bytes) return MLA_ERR_INVALID_ARG;
  if (!shape_supported(B, s_q, H)) return MLA_ERR_UNSUPPORTED;
  *bytes = static_cast<size_t>(mla::meta_words(B)) * sizeof(int32_t);
  return MLA_OK;
}

mla_status_t mla_set_wait_timeout_ns(uint64_t ns) {
  g_wait_timeout_ns.store(ns == 0 ? kDefaultWaitTimeoutNs : ns);
  return MLA_OK;
}

mla_status_t mla_set_stall_injection(int enable) {
  g_inject_stall.store(enable ? 1 : 0);
  return MLA_OK;
}

mla_status_t mla_device_sm_count(int* sm_count) {
  if (!sm_count) return MLA_ERR_INVALID_ARG;
  return device_info(sm_count);
}

mla_status_t mla_workspace_size(int B, int s_q, int H, size_t* bytes) {
  if (!bytes) return MLA_ERR_INVALID_ARG;
  if (!shape_supported(B, s_q, H)) return MLA_ERR_UNSUPPORTED;
  int sms = 0;
  mla_status_t st = device_info(&sms);
  if (st != MLA_OK) return st;
  const int64_t slots = mla::ws_slots(B, num_workers_for(sms));
  const int64_t M = static_cast<int64_t>(s_q) * H;
  *bytes = static_cast<size_t>(slots * M * (mla::kDLatent + 1) * sizeof(float));
  return MLA_OK;
}

mla_status_t mla_get_metadata(const int32_t* cache_seqlens, int B, int s_q, int H, void* metadata,
                              size_t metadata_bytes, void* stream) {
  if (!cache_seqlens || !metadata) return MLA_ERR_INVALID_ARG;
  if (!shape_supported(B, s_q, H)) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(metadata) || (reinterpret_cast<uintptr_t>(cache_seqlens) & 3u)) return MLA_ERR_INVALID_ARG;
  size_t need = 0;
  mla_metadata_size(B, s_q, H, &need);
  if (metadata_bytes < need) return MLA_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  mla_status_t st = device_info(&sms);
  if (st != MLA_OK) return st;
  if (mla::launch_metadata(cache_seqlens, B, s_q, H, num_workers_for(sms), static_cast<int32_t*>(metadata),
                           static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MLA_ERR_CUDA;
  return MLA_OK;
}

}  // extern "C"

namespace {

// Shared validation of the decode arguments; fills the derived launch sizes.
struct DecodeGeom {
  int sms, workers, T, P, M;
  int64_t slots;
};

mla_status_t check_decode_args(const void* q_nope, const void* q_pe, const void* kv_cache, int64_t num_blocks,
                               const int32_t* block_table, int max_blocks, const int32_t* cache_seqlens, int B,
                               int s_q, int H, float softmax_scale, const void* metadata, size_t metadata_bytes,
                               const void* workspace, size_t workspace_bytes, const void* out, const float* lse,
                               const int32_t* status, DecodeGeom* g) {
  if (!q_nope || !q_pe || !kv_cache || !block_table || !cache_seqlens || !metadata || !out || !lse)
    return MLA_ERR_INVALID_ARG;
  if (!shape_supported(B, s_q, H)) return MLA_ERR_UNSUPPORTED;
  if (num_blocks < 1 || num_blocks > (int64_t)INT32_MAX || max_blocks < 1) return MLA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || softmax_scale > 1e30f) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_nope) || !aligned16(q_pe) || !aligned16(kv_cache) || !aligned16(out) || !aligned16(metadata) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(block_table) & 3u) ||
      (reinterpret_cast<uintptr_t>(cache_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(status) & 3u))
    return MLA_ERR_INVALID_ARG;
  size_t need_meta = 0, need_ws = 0;
  mla_metadata_size(B, s_q, H, &need_meta);
  if (metadata_bytes < need_meta) return MLA_ERR_WORKSPACE_TOO_SMALL;
  mla_status_t st = mla_workspace_size(B, s_q, H, &need_ws);
  if (st != MLA_OK) return st;
  if (workspace_bytes < need_ws) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if (!workspace || !aligned16(workspace)) return MLA_ERR_INVALID_ARG;
  st = device_info(&g->sms);
  if (st != MLA_OK) return st;
  g->M = s_q * H;
  g->workers = num_workers_for(g->sms);
  g->T = (g->M + mla::kRowsPerTile - 1) / mla::kRowsPerTile;
  g->P = parts_for(g->workers, s_q, H);
  g->slots = mla::ws_slots(B, g->workers);
  return MLA_OK;
}

// FP8 cache views (rows of kRowBytes8 bytes): code slabs for QK (64 columns, no swizzle)
// and PV (128 columns, 128-byte swizzle), the scaled k_pe as bf16 and the scales as fp32.
bool encode_fp8_cache(const void* kv, int64_t num_blocks, CUtensorMap* tm_q, CUtensorMap* tm_v, CUtensorMap* tm_kpe,
                      CUtensorMap* tm_scl) {
  const cuuint64_t row = mla::kRowBytes8, blk = (cuuint64_t)mla::kRowBytes8 * mla::kBlockSize;
  {
    cuuint64_t dims[3] = {row, (cuuint64_t)mla::kBlockSize, (cuuint64_t)num_blocks};
    cuuint64_t strides[2] = {row, blk};
    cuuint32_t box_q[3] = {64, 64, 1};
    cuuint32_t box_v[3] = {128, 64, 1};
    if (!encode(tm_q, kv, 3, dims, strides, box_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode(tm_v, kv, 3, dims, strides, box_v, CU_TENSOR_MAP_DATA_TYPE_UINT8, CU_TENSOR_MAP_SWIZZLE_128B))
      return false;
  }
  {
    cuuint64_t dims[3] = {row / 2, (cuuint64_t)mla::kBlockSize, (cuuint64_t)num_blocks};
    cuuint64_t strides[2] = {row, blk};
    cuuint32_t box[3] = {64, 64, 1};
    if (!encode(tm_kpe, kv, 3, dims, strides, box)) return false;
  }
  {
    cuuint64_t dims[3] = {row / 4, (cuuint64_t)mla::kBlockSize, (cuuint64_t)num_blocks};
    cuuint64_t strides[2] = {row, blk};
    cuuint32_t box[3] = {4, 64, 1};
    if (!encode(tm_scl, kv, 3, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, CU_TENSOR_MAP_SWIZZLE_NONE))
      return false;
  }
  return true;
}

mla_status_t launch_attention(bool fp8, const void* q_nope, const void* q_pe, const void* kv_cache,
                              int64_t num_blocks, const int32_t* block_table, int max_blocks,
                              const int32_t* cache_seqlens, const int32_t* q_lens, int B, int s_q, int H,
                              float softmax_scale, int causal, const void* metadata, void* workspace, void* out,
                              float* lse, int32_t* status, const DecodeGeom& g, cudaStream_t s, int tok_rep = 0,
                              int tok_causal = 0, const int32_t* tok_q_lens = nullptr) {
  const int64_t rows = static_cast<int64_t>(B) * g.M;
  CUtensorMap tm_kv, tm_kv2, tm_qn, tm_qp, tm_kpe, tm_scl;
  if (fp8) {
    if (!encode_fp8_cache(kv_cache, num_blocks, &tm_kv, &tm_kv2, &tm_kpe, &tm_scl)) return MLA_ERR_INVALID_ARG;
  } else {
    {
    cuuint64_t dims[3] = {(cuuint64_t)mla::kDQK, (cuuint64_t)mla::kBlockSize, (cuuint64_t)num_blocks};
    cuuint64_t strides[2] = {(cuuint64_t)mla::kDQK * 2, (cuuint64_t)mla::kDQK * 2 * mla::kBlockSize};
    cuuint32_t box[3] = {64, 64, 1};
    if (!encode(&tm_kv, kv_cache, 3, dims, strides, box)) return MLA_ERR_INVALID_ARG;
  }
  {
    // The same cache viewed as [block][chunk of 64 columns][row][64]: one box of
    // {64, 64 rows, 2 chunks} lands a 64-row x 128-column slab as two stacked
    // 128-byte-swizzled 64x64 tiles with a single TMA instruction.
    cuuint64_t dims[4] = {64, (cuuint64_t)mla::kBlockSize, (cuuint64_t)(mla::kDQK / 64), (cuuint64_t)num_blocks};
    cuuint64_t strides[3] = {(cuuint64_t)mla::kDQK * 2, 128, (cuuint64_t)mla::kDQK * 2 * mla::kBlockSize};
    cuuint32_t box[4] = {64, 64, 2, 1};
    if (!encode(&tm_kv2, kv_cache, 4, dims, strides, box)) return MLA_ERR_INVALID_ARG;
    }
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)mla::kDLatent, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)mla::kDLatent * 2};
    cuuint32_t box[2] = {64, 64};
    if (!encode(&tm_qn, q_nope, 2, dims, strides, box)) return MLA_ERR_INVALID_ARG;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)mla::kDRope, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)mla::kDRope * 2};
    cuuint32_t box[2] = {64, 64};
    if (!encode(&tm_qp, q_pe, 2, dims, strides, box)) return MLA_ERR_INVALID_ARG;
  }
  float* part_o = static_cast<float*>(workspace);
  float* part_lse = part_o + g.slots * g.M * mla::kDLatent;
  // Output views for the epilogue's TMA stores: rows past M of a sequence are clipped.
  CUtensorMap tm_out, tm_part;
  {
    cuuint64_t dims[3] = {(cuuint64_t)mla::kDLatent, (cuuint64_t)g.M, (cuuint64_t)B};
    cuuint64_t strides[2] = {(cuuint64_t)mla::kDLatent * 2, (cuuint64_t)g.M * mla::kDLatent * 2};
    cuuint32_t box[3] = {64, 64, 1};
    if (!encode(&tm_out, out, 3, dims, strides, box)) return MLA_ERR_INVALID_ARG;
  }
  {
    cuuint64_t dims[3] = {(cuuint64_t)mla::kDLatent, (cuuint64_t)g.M, (cuuint64_t)g.slots};
    cuuint64_t strides[2] = {(cuuint64_t)mla::kDLatent * 4, (cuuint64_t)g.M * mla::kDLatent * 4};
    cuuint32_t box[3] = {32, 64, 1};
    if (!encode(&tm_part, part_o, 3, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_FLOAT32))
      return MLA_ERR_INVALID_ARG;
  }
  if (mla::launch_decode(fp8, tm_kv, tm_kv2, fp8 ? &tm_kpe : nullptr, fp8 ? &tm_scl : nullptr, tm_qn, tm_qp,
                         tm_out, tm_part, block_table, max_blocks, cache_seqlens,
                         q_lens, static_cast<const int32_t*>(metadata), num_blocks, B, s_q, H, softmax_scale,
                         causal != 0,
                         out, lse, part_o, part_lse, status, 2 * g.P * g.T, g_wait_timeout_ns.load(), g_inject_stall.load(), s,
                         tok_rep, tok_causal, tok_q_lens) != cudaSuccess)
    return MLA_ERR_CUDA;
  return MLA_OK;
}

}  // namespace

extern "C" {

mla_status_t mla_decode_attention(const void* q_nope, const void* q_pe, const void* kv_cache, int64_t num_blocks,
                                  const int32_t* block_table, int max_blocks, const int32_t* cache_seqlens, int B,
                                  int s_q, int H, float softmax_scale, int causal, const void* metadata,
                                  size_t metadata_bytes, void* workspace, size_t workspace_bytes, void* out,
                                  float* lse, int32_t* status, void* stream) {
  DecodeGeom g;
  mla_status_t st = check_decode_args(q_nope, q_pe, kv_cache, num_blocks, block_table, max_blocks, cache_seqlens,
                                      B, s_q, H, softmax_scale, metadata, metadata_bytes, workspace,
                                      workspace_bytes, out, lse, status, &g);
  if (st != MLA_OK) return st;
  return launch_attention(false, q_nope, q_pe, kv_cache, num_blocks, block_table, max_blocks, cache_seqlens,
                          nullptr, B, s_q, H, softmax_scale, causal, metadata, workspace, out, lse, status, g,
                          static_cast<cudaStream_t>(stream));
}

mla_status_t mla_decode_combine(const int32_t* cache_seqlens, int max_blocks, int B, int s_q, int H,
                                const void* metadata, size_t metadata_bytes, const void* workspace,
                                size_t workspace_bytes, void* out, float* lse, int32_t* status, void* stream) {
  if (!cache_seqlens || !metadata || !workspace || !out || !lse) return MLA_ERR_INVALID_ARG;
  if (!shape_supported(B, s_q, H)) return MLA_ERR_UNSUPPORTED;
  if (max_blocks < 1) return MLA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(metadata) || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(cache_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(status) & 3u))
    return MLA_ERR_INVALID_ARG;
  size_t need_meta = 0, need_ws = 0;
  mla_metadata_size(B, s_q, H, &need_meta);
  if (metadata_bytes < need_meta) return MLA_ERR_WORKSPACE_TOO_SMALL;
  mla_status_t st = mla_workspace_size(B, s_q, H, &need_ws);
  if (st != MLA_OK) return st;
  if (workspace_bytes < need_ws) return MLA_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  st = device_info(&sms);
  if (st != MLA_OK) return st;
  const int M = s_q * H;
  const int64_t slots = mla::ws_slots(B, num_workers_for(sms));
  const float* part_o = static_cast<const float*>(workspace);
  const float* part_lse = part_o + slots * M * mla::kDLatent;
  (void)status;  // the combine raises no error of its own
  if (mla::launch_combine(static_cast<const int32_t*>(metadata), cache_seqlens, nullptr, max_blocks, B, s_q, M,
                          parts_for(num_workers_for(sms), s_q, H), part_o, part_lse, out, lse,
                          static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MLA_ERR_CUDA;
  return MLA_OK;
}

mla_status_t mla_decode(const void* q_nope, const void* q_pe, const void* kv_cache, int64_t num_blocks,
                        const int32_t* block_table, int max_blocks, const int32_t* cache_seqlens, int B,
                        int s_q, int H, float softmax_scale, int causal, const void* metadata,
                        size_t metadata_bytes, void* workspace, size_t workspace_bytes, void* out, float* lse,
                        int32_t* status, void* stream) {
  return mla_decode_ragged(q_nope, q_pe, kv_cache, num_blocks, block_table, max_blocks, cache_seqlens, nullptr, B,
                           s_q, H, softmax_scale, causal, metadata, metadata_bytes, workspace, workspace_bytes, out,
                           lse, status, stream);
}

}  // extern "C"

namespace {

// Validation, attention and combine launches shared by the bf16 and FP8 entry points.
// tokens: the token schedule, an s_q = 1 decode over B * s_q token sequences (q, out
// and lse are the same memory viewed as [B * s_q, 1, H, ...]); the metadata must come
// from mla_get_metadata_tokens with the same q_lens and causal flag.
mla_status_t decode_any(bool fp8, const void* q_nope, const void* q_pe, const void* kv_cache, int64_t num_blocks,
                        const int32_t* block_table, int max_blocks, const int32_t* cache_seqlens,
                        const int32_t* q_lens, int B, int s_q, int H, float softmax_scale, int causal,
                        const void* metadata, size_t metadata_bytes, void* workspace, size_t workspace_bytes,
                        void* out, float* lse, int32_t* status, void* stream, bool tokens = false) {
  if (q_lens && (reinterpret_cast<uintptr_t>(q_lens) & 3u)) return MLA_ERR_INVALID_ARG;
  if (tokens && !shape_supported(B, s_q, H)) return MLA_ERR_UNSUPPORTED;
  const int Bl = tokens ? B * s_q : B, sl = tokens ? 1 : s_q;  // the launch's batch and query count
  DecodeGeom g;
  mla_status_t st = check_decode_args(q_nope, q_pe, kv_cache, num_blocks, block_table, max_blocks, cache_seqlens,
                                      Bl, sl, H, softmax_scale, metadata, metadata_bytes, workspace,
                                      workspace_bytes, out, lse, status, &g);
  if (st != MLA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (tokens)
    st = launch_attention(fp8, q_nope, q_pe, kv_cache, num_blocks, block_table, max_blocks, cache_seqlens, nullptr,
                          Bl, 1, H, softmax_scale, 0, metadata, workspace, out, lse, status, g, s, s_q,
                          causal != 0, q_lens);
  else
    st = launch_attention(fp8, q_nope, q_pe, kv_cache, num_blocks, block_table, max_blocks, cache_seqlens, q_lens,
                          B, s_q, H, softmax_scale, causal, metadata, workspace, out, lse, status, g, s);
  if (st != MLA_OK) return st;
  const float* part_o = static_cast<const float*>(workspace);
  const float* part_lse = part_o + g.slots * g.M * mla::kDLatent;
  if (mla::launch_combine(static_cast<const int32_t*>(metadata), cache_seqlens, q_lens, max_blocks, Bl, sl, g.M,
                          g.P, part_o, part_lse, out, lse, s, tokens ? s_q : 0, tokens && causal != 0) != cudaSuccess)
    return MLA_ERR_CUDA;
  return MLA_OK;
}

}  // namespace

extern "C" {

mla_status_t mla_decode_ragged(const void* q_nope, const void* q_pe, const void* kv_cache, int64_t num_blocks,
                               const int32_t* block_table, int max_blocks, const int32_t* cache_seqlens,
                               const int32_t* q_lens, int B, int s_q, int H, float softmax_scale, int causal,
                               const void* metadata, size_t metadata_bytes, void* workspace,
                               size_t workspace_bytes, void* out, float* lse, int32_t* status, void* stream) {
  return decode_any(false, q_nope, q_pe, kv_cache, num_blocks, block_table, max_blocks, cache_seqlens, q_lens, B,
                    s_q, H, softmax_scale, causal, metadata, metadata_bytes, workspace, workspace_bytes, out, lse,
                    status, stream);
}

mla_status_t mla_decode_fp8(const void* q_nope, const void* q_pe, const void* kv_fp8, int64_t num_blocks,
                            const int32_t* block_table, int max_blocks, const int32_t* cache_seqlens,
                            const int32_t* q_lens, int B, int s_q, int H, float softmax_scale, int causal,
                            const void* metadata, size_t metadata_bytes, void* workspace, size_t workspace_bytes,
                            void* out, float* lse, int32_t* status, void* stream) {
  return decode_any(true, q_nope, q_pe, kv_fp8, num_blocks, block_table, max_blocks, cache_seqlens, q_lens, B,
                    s_q, H, softmax_scale, causal, metadata, metadata_bytes, workspace, workspace_bytes, out, lse,
                    status, stream);
}

mla_status_t mla_get_metadata_tokens(const int32_t* cache_seqlens, const int32_t* q_lens, int B, int s_q, int H,
                                     int causal, void* metadata, size_t metadata_bytes, void* stream) {
  if (!cache_seqlens || !metadata) return MLA_ERR_INVALID_ARG;
  if (!shape_supported(B, s_q, H) || !shape_supported(B * s_q, 1, H)) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(metadata) || (reinterpret_cast<uintptr_t>(cache_seqlens) & 3u) ||
      (reinterpret_cast<uintptr_t>(q_lens) & 3u))
    return MLA_ERR_INVALID_ARG;
  size_t need = 0;
  mla_metadata_size(B * s_q, 1, H, &need);
  if (metadata_bytes < need) return MLA_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  mla_status_t st = device_info(&sms);
  if (st != MLA_OK) return st;
  if (mla::launch_metadata(cache_seqlens, B * s_q, 1, H, num_workers_for(sms), static_cast<int32_t*>(metadata),
                           static_cast<cudaStream_t>(stream), q_lens, s_q, causal != 0) != cudaSuccess)
    return MLA_ERR_CUDA;
  return MLA_OK;
}

mla_status_t mla_decode_tokens(const void* q_nope, const void* q_pe, const void* kv_cache, int64_t num_blocks,
                               const int32_t* block_table, int max_blocks, const int32_t* cache_seqlens,
                               const int32_t* q_lens, int B, int s_q, int H, float softmax_scale, int causal,
                               const void* metadata, size_t metadata_bytes, void* workspace,
                               size_t workspace_bytes, void* out, float* lse, int32_t* status, void* stream) {
  return decode_any(false, q_nope, q_pe, kv_cache, num_blocks, block_table, max_blocks, cache_seqlens, q_lens, B,
                    s_q, H, softmax_scale, causal, metadata, metadata_bytes, workspace, workspace_bytes, out, lse,
                    status, stream, true);
}

mla_status_t mla_decode_fp8_tokens(const void* q_nope, const void* q_pe, const void* kv_fp8, int64_t num_blocks,
                                   const int32_t* block_table, int max_blocks, const int32_t* cache_seqlens,
                                   const int32_t* q_lens, int B, int s_q, int H, float softmax_scale, int causal,
                                   const void* metadata, size_t metadata_bytes, void* workspace,
                                   size_t workspace_bytes, void* out, float* lse, int32_t* status, void* stream) {
  return decode_any(true, q_nope, q_pe, kv_fp8, num_blocks, block_table, max_blocks, cache_seqlens, q_lens, B,
                    s_q, H, softmax_scale, causal, metadata, metadata_bytes, workspace, workspace_bytes, out, lse,
                    status, stream, true);
}

mla_status_t mla_decode_fp8_attention(const void* q_nope, const void* q_pe, const void* kv_fp8, int64_t num_blocks,
                                      const int32_t* block_table, int max_blocks, const int32_t* cache_seqlens,
                                      const int32_t* q_lens, int B, int s_q, int H, float softmax_scale, int causal,
                                      const void* metadata, size_t metadata_bytes, void* workspace,
                                      size_t workspace_bytes, void* out, float* lse, int32_t* status,
                                      void* stream) {
  if (q_lens && (reinterpret_cast<uintptr_t>(q_lens) & 3u)) return MLA_ERR_INVALID_ARG;
  DecodeGeom g;
  mla_status_t st = check_decode_args(q_nope, q_pe, kv_fp8, num_blocks, block_table, max_blocks, cache_seqlens,
                                      B, s_q, H, softmax_scale, metadata, metadata_bytes, workspace,
                                      workspace_bytes, out, lse, status, &g);
  if (st != MLA_OK) return st;
  return launch_attention(true, q_nope, q_pe, kv_fp8, num_blocks, block_table, max_blocks, cache_seqlens, q_lens,
                          B, s_q, H, softmax_scale, causal, metadata, workspace, out, lse, status, g,
                          static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// quantised prefill attention (SageAttention-style, head dim 192)
// ---------------------------------------------------------------------------
mla_status_t mla_sage_workspace_size(int S, int H, size_t* bytes) {
  if (!bytes || S < 1 || H < 1 || H > 65535) return MLA_ERR_INVALID_ARG;
  if ((int64_t)mla::sage::padded_len(S) / mla::sage::kBlockM * H > 0x7fffffffLL) return MLA_ERR_UNSUPPORTED;
  *bytes = mla::sage::workspace_bytes(S, H);
  return MLA_OK;
}

mla_status_t mla_sage_quantize(const void* q, const void* k, const void* v, int S, int H, void* workspace,
                               size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !workspace) return MLA_ERR_INVALID_ARG;
  size_t need = 0;
  mla_status_t st = mla_sage_workspace_size(S, H, &need);
  if (st != MLA_OK) return st;
  if (workspace_bytes < need) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(workspace)) return MLA_ERR_INVALID_ARG;
  int sms = 0;
  st = device_info(&sms);
  if (st != MLA_OK) return st;
  const mla::sage::Workspace ws = mla::sage::carve(workspace, S, H);
  if (mla::sage::launch_quantize(q, k, v, S, H, ws, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MLA_ERR_CUDA;
  return MLA_OK;
}

mla_status_t mla_sage_attention(int S, int H, float softmax_scale, const void* workspace, size_t workspace_bytes,
                                void* out, float* lse, int32_t* status, void* stream) {
  if (!workspace || !out || !lse) return MLA_ERR_INVALID_ARG;
  size_t need = 0;
  mla_status_t st = mla_sage_workspace_size(S, H, &need);
  if (st != MLA_OK) return st;
  if (workspace_bytes < need) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if (!(softmax_scale > 0.f) || softmax_scale > 1e30f) return MLA_ERR_INVALID_ARG;
  if (!aligned16(workspace) || !aligned16(out) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(status) & 3u))
    return MLA_ERR_INVALID_ARG;
  int sms = 0;
  st = device_info(&sms);
  if (st != MLA_OK) return st;
  const mla::sage::Workspace ws = mla::sage::carve(const_cast<void*>(workspace), S, H);
  const int S_pad = mla::sage::padded_len(S);
  CUtensorMap tm_q, tm_k, tm_v;
  {
    cuuint64_t dims[3] = {(cuuint64_t)mla::sage::kDQK, (cuuint64_t)S_pad, (cuuint64_t)H};
    cuuint64_t strides[2] = {(cuuint64_t)mla::sage::kDQK, (cuuint64_t)mla::sage::kDQK * S_pad};
    cuuint32_t box[3] = {64, (cuuint32_t)mla::sage::kBlockM, 1};
    if (!encode(&tm_q, ws.q8, 3, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_UINT8, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !encode(&tm_k, ws.k8, 3, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_UINT8, CU_TENSOR_MAP_SWIZZLE_64B))
      return MLA_ERR_INVALID_ARG;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)S_pad, (cuuint64_t)mla::sage::kDV * H};
    cuuint64_t strides[1] = {(cuuint64_t)S_pad};
    cuuint32_t box[2] = {(cuuint32_t)mla::sage::kBlockN, (cuuint32_t)mla::sage::kDV};
    if (!encode(&tm_v, ws.vt8, 2, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_UINT8, CU_TENSOR_MAP_SWIZZLE_128B))
      return MLA_ERR_INVALID_ARG;
  }
  if (mla::sage::launch_attention(tm_q, tm_k, tm_v, ws, S, H, softmax_scale, out, lse, status,
                                  g_wait_timeout_ns.load(), static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MLA_ERR_CUDA;
  return MLA_OK;
}

mla_status_t mla_sage_prefill(const void* q, const void* k, const void* v, int S, int H, float softmax_scale,
                              void* workspace, size_t workspace_bytes, void* out, float* lse, int32_t* status,
                              void* stream) {
  mla_status_t st = mla_sage_quantize(q, k, v, S, H, workspace, workspace_bytes, stream);
  if (st != MLA_OK) return st;
  return mla_sage_attention(S, H, softmax_scale, workspace, workspace_bytes, out, lse, status, stream);
}

}  // extern "C"
