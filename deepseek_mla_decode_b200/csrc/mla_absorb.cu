// Weight-absorption GEMMs either side of the MLA decode, for sm_100a.
//
// In decode the per-head key and value up-projections of MLA fold into the query
// and the output (KsanaLLM 0.6.0 release notes, section 2.1, WA-MLA): with
// k_h = W_UK[h] c and v_h = W_UV[h] c for the 512-d latent c,
//     q_nope[r, h, :] = W_UK[h]^T q[r, h, :]     (128 -> 512, before the decode)
//     y[r, h, :]      = W_UV[h] o[r, h, :]        (512 -> 128, after the decode)
// for every query row r (= b * s_q + i) and head h.  Both are batched GEMMs over the
// heads: rows [R, 128] x [128, 512] per head, and rows [R, 512] x [512, 128].
//
// Work items of 128 rows x 128 output columns of one head, with the contraction in
// stages of 128 (the q side's 512 output columns are four items, the out side's
// 512-deep contraction four stages), run by a persistent warp-specialised kernel (one
// CTA per SM; below).  Memory-bound: the weights (16.8 MB per projection for 128
// heads) are read once from HBM, the rows once per row tile and column slice (L2
// serves the repeats); rows past R are zero-filled on load and clipped on store.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>
#include "mla_internal.h"
#include "ptx_sm100.cuh"
#include "../../include/mla_decode.h"

namespace mla {

bool encode_tiled_bf16(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
                       const cuuint32_t* box);

namespace {

using namespace ptx;

constexpr int kRowTile = 128;
constexpr int kBox = 8192;  // 64 rows x 128 bytes

struct AbsorbParams {
  CUtensorMap tm_a;  // rows [R][H][K] bf16, box {64, 1, 128}
  CUtensorMap tm_b;  // weights [H][128][512] bf16: q side box {64 n, 64 k, 1}; out side box {64 k, 128 n, 1}
  CUtensorMap tm_c;  // output [R][H][N] bf16, box {64, 1, 128} (TMA store)
};

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, uint32_t bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma_store_3d(const void* tmap, uint32_t src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void umma_1sm(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void commit_1sm(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// Persistent, warp-specialised kernel.  A work item is (row tile of 128, head, slice
// of 128 output columns); items run head-major, so the CTAs working at one time share
// heads and L2 serves the repeated reads of a head's weights (by its row tiles) and
// of a row tile (by its column slices).  Per CTA:
//   warp 4 (one lane)  TMA loads, one stage per 128-deep contraction phase: the row
//                      tile's [128][128] A and the weight slice's 128 x 128 B (64 KB),
//                      into a two-stage ring;
//   warp 5 (one lane)  tcgen05 MMAs (M = N = 128) into one of two TMEM accumulators,
//                      releasing each stage (commit) and handing over the accumulator
//                      after the item's last phase;
//   warps 0..3         the epilogue: TMEM lanes 32 w .. 32 w + 31 -> bf16 -> one of two
//                      swizzled staging tiles -> TMA stores, so an item's stores overlap
//                      the next item's loads and MMAs.
// Every wait is bounded (1 s); a wait that runs out stops its role, and the CTA drains
// its tensor-core work and in-flight loads before it frees TMEM and exits.
constexpr int kPThreads = 192;
constexpr int kPStages = 2;
constexpr int kPKP = 128;                     // contraction depth per stage
constexpr int kPABytes = 2 * 2 * kBox;        // 128 rows x 128 k bf16 (two 64-wide boxes)
// N output columns per item (64 or 128): the weight slice, the staging tile, the
// shared memory
template <int N>
struct PCfg {
  static constexpr int kBBytes = 2 * (N / 64) * kBox;    // 128 k x N bf16
  static constexpr int kStageBytes = kPABytes + kBBytes;
  static constexpr int kStagingBytes = (N / 64) * 2 * kBox;  // 128 rows x N bf16 (N / 64 boxes)
  static constexpr int kSmem = kPStages * kStageBytes + 2 * kStagingBytes + 1024;
};
constexpr int kPEpiThreads = 128;
constexpr int kPBarEpi = 1;                   // named barrier of the four epilogue warps
constexpr uint64_t kPWaitNs = 1000000000ull;

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// named barrier that also ANDs a predicate over its threads
__device__ __forceinline__ bool named_bar_and(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %3, 0;\n\t"
      "bar.red.and.pred q, %1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(id), "r"(count), "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t deadline = globaltimer_ns() + kPWaitNs;
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() > deadline) {
      *abort = 1;
      return false;
    }
  }
}

template <int N, int K, bool B_MN>
__global__ void __launch_bounds__(kPThreads, 1) absorb_kernel(const __grid_constant__ AbsorbParams p, int R, int H,
                                                              int nslices) {
  static_assert(K % kPKP == 0 && (N == 64 || N == 128), "tile shape");
  using C = PCfg<N>;
  constexpr int kPN = N, kPStageBytes = C::kStageBytes, kPStagingBytes = C::kStagingBytes;
  constexpr int kPhases = K / kPKP;
  constexpr uint32_t kIdesc = make_idesc_bf16(128, kPN, false, B_MN);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[kPStages], empty[kPStages], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sRing = smem_u32(smem), sStaging = sRing + kPStages * kPStageBytes;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nrt = (R + kRowTile - 1) / kRowTile;
  const int items = nrt * H * nslices;

  if (tid == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&acc_full[a]), 1);
      mbar_init(smem_u32(&acc_empty[a]), kPEpiThreads);
    }
    mbar_init(smem_u32(&drain), 1);
    abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&p.tm_a);
    prefetch_tmap(&p.tm_b);
    prefetch_tmap(&p.tm_c);
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base)),
                 "r"(2 * kPN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  // item -> (head, column slice, row tile), head-major
  auto decode_item = [&](int it, int& h, int& n0, int& r0) {
    h = it / (nrt * nslices);
    const int rem = it - h * nrt * nslices;
    n0 = (rem / nrt) * kPN;
    r0 = (rem % nrt) * kRowTile;
  };

  if (warp == 4) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t sc = 0;
      for (int it = blockIdx.x; it < items; it += gridDim.x) {
        int h, n0, r0;
        decode_item(it, h, n0, r0);
        bool ok = true;
        for (int ph = 0; ph < kPhases; ++ph, ++sc) {
          const uint32_t s = sc % kPStages, use = sc / kPStages;
          if (use > 0 && !wait_or_abort(smem_u32(&empty[s]), (use - 1) & 1, &abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full[s]);
          const uint32_t sA = sRing + s * kPStageBytes, sB = sA + kPABytes;
          expect_tx(fb, kPStageBytes);
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int k0 = ph * kPKP + 64 * i;
            tma_load_3d(sA + i * 2 * kBox, &p.tm_a, fb, k0, h, r0);
            if (B_MN) {
#pragma unroll
              for (int j = 0; j < kPN / 64; ++j)
                tma_load_3d(sB + ((kPN / 64) * i + j) * kBox, &p.tm_b, fb, n0 + 64 * j, k0, h);
            } else {
              tma_load_3d(sB + i * (kPN / 64) * kBox, &p.tm_b, fb, k0, n0, h);
            }
          }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t sc = 0, ic = 0;
      for (int it = blockIdx.x; it < items; it += gridDim.x, ++ic) {
        const uint32_t a = ic & 1, ause = ic >> 1;
        if (ause > 0 && !wait_or_abort(smem_u32(&acc_empty[a]), (ause - 1) & 1, &abort_flag)) break;
        tc_fence_after();
        bool ok = true;
        for (int ph = 0; ph < kPhases; ++ph, ++sc) {
          const uint32_t s = sc % kPStages;
          if (!wait_or_abort(smem_u32(&full[s]), (sc / kPStages) & 1, &abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = sRing + s * kPStageBytes, sB = sA + kPABytes;
          // A (rows) K-major: 128-byte rows, 8-row groups 1024 B apart, K step = 32 B.
          // B MN-major: two 64-wide column blocks 8 KB apart (LBO), 8-row k groups 1024 B
          // apart, K step = 16 rows = 2048 B.  B K-major: like A with 128 n rows.
#pragma unroll
          for (int i = 0; i < 2; ++i) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const uint64_t da = make_smem_desc(sA + i * 2 * kBox + 32 * ks, 16, 1024, kSwizzle128B);
              const uint64_t db =
                  B_MN ? make_smem_desc(sB + (kPN / 64) * i * kBox + 2048 * ks, kBox, 1024, kSwizzle128B)
                       : make_smem_desc(sB + i * (kPN / 64) * kBox + 32 * ks, 16, 1024, kSwizzle128B);
              umma_1sm(tmem + a * kPN, da, db, kIdesc, (ph | i | ks) != 0);
            }
          }
          commit_1sm(smem_u32(&empty[s]));
        }
        if (!ok) break;
        commit_1sm(smem_u32(&acc_full[a]));
      }
    }
  } else {
    // ---------------- epilogue (warps 0..3) ----------------
    const int m = tid;  // TMEM lane = row of the tile
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    uint32_t ic = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x, ++ic) {
      int h, n0, r0;
      decode_item(it, h, n0, r0);
      const uint32_t a = ic & 1;
      const bool ok = wait_or_abort(smem_u32(&acc_full[a]), (ic >> 1) & 1, &abort_flag);
      // staging buffer ic & 1 was last stored from two items ago: its reads must be done
      if (tid == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
      if (!named_bar_and(kPBarEpi, kPEpiThreads, ok)) break;
      tc_fence_after();
      const uint32_t sbuf = sStaging + (ic & 1) * kPStagingBytes;
#pragma unroll 1
      for (int j = 0; j < kPN / 64; ++j) {
        uint32_t w[32];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + a * kPN + 64 * j + 32 * hf, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 16; ++k) w[16 * hf + k] = pack2(__uint_as_float(o[2 * k]), __uint_as_float(o[2 * k + 1]));
        }
        const uint32_t row = sbuf + j * 2 * kBox + m * 128;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + ((q ^ (m & 7)) << 4)), "r"(w[4 * q]),
                       "r"(w[4 * q + 1]), "r"(w[4 * q + 2]), "r"(w[4 * q + 3])
                       : "memory");
      }
      // this thread's TMEM reads are done: the accumulator may take the next item
      tc_fence_before();
      mbar_arrive(smem_u32(&acc_empty[a]));
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      named_bar_sync(kPBarEpi, kPEpiThreads);
      if (tid == 0) {
#pragma unroll
        for (int j = 0; j < kPN / 64; ++j) tma_store_3d(&p.tm_c, sbuf + j * 2 * kBox, n0 + 64 * j, h, r0);
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      }
    }
    if (tid == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }

  // ---- teardown: after a wait ran out, drain the tensor-core work and the loads in
  // flight before TMEM and shared memory are released --------------------------
  tc_fence_before();
  __syncthreads();
  if (abort_flag) {
    if (warp == 5 && lane == 0) {
      commit_1sm(smem_u32(&drain));
      const uint64_t dl = globaltimer_ns() + 100000000ull;
      while (!mbar_try_wait(smem_u32(&drain), 0) && globaltimer_ns() < dl) {
      }
    }
    if (tid == 0) {
      const uint64_t until = globaltimer_ns() + 500000ull;
      while (globaltimer_ns() < until) {
      }
    }
    __syncthreads();
  }
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * kPN) : "memory");
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// NT output columns in all (slices of N), contraction K; weights MN-major or K-major
template <int NT, int N, int K, bool B_MN>
mla_status_t launch_absorb(const void* rows, const void* w, void* outp, int R, int H, cudaStream_t stream) {
  static_assert(NT % N == 0, "column slices");
  constexpr int kPN = N;
  if (!rows || !w || !outp) return MLA_ERR_INVALID_ARG;
  if (R < 1 || H < 1 || H > 65535) return MLA_ERR_INVALID_ARG;
  if (!aligned16(rows) || !aligned16(w) || !aligned16(outp)) return MLA_ERR_INVALID_ARG;
  int sms = 0;
  mla_status_t st = mla_device_sm_count(&sms);  // device check and driver entry point
  if (st != MLA_OK) return st;
  AbsorbParams prm;
  {
    const cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)H, (cuuint64_t)R};
    const cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)H * K * 2};
    const cuuint32_t box[3] = {64, 1, kRowTile};
    if (!encode_tiled_bf16(&prm.tm_a, rows, 3, dims, strides, box)) return MLA_ERR_INVALID_ARG;
  }
  if (B_MN) {  // W[h] is [k = 128][n = 512]
    const cuuint64_t dims[3] = {(cuuint64_t)NT, (cuuint64_t)K, (cuuint64_t)H};
    const cuuint64_t strides[2] = {(cuuint64_t)NT * 2, (cuuint64_t)K * NT * 2};
    const cuuint32_t box[3] = {64, 64, 1};
    if (!encode_tiled_bf16(&prm.tm_b, w, 3, dims, strides, box)) return MLA_ERR_INVALID_ARG;
  } else {  // W[h] is [n = 128][k = 512]
    const cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)NT, (cuuint64_t)H};
    const cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)NT * K * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)kPN, 1};
    if (!encode_tiled_bf16(&prm.tm_b, w, 3, dims, strides, box)) return MLA_ERR_INVALID_ARG;
  }
  {
    const cuuint64_t dims[3] = {(cuuint64_t)NT, (cuuint64_t)H, (cuuint64_t)R};
    const cuuint64_t strides[2] = {(cuuint64_t)NT * 2, (cuuint64_t)H * NT * 2};
    const cuuint32_t box[3] = {64, 1, kRowTile};
    if (!encode_tiled_bf16(&prm.tm_c, outp, 3, dims, strides, box)) return MLA_ERR_INVALID_ARG;
  }
  auto kern = absorb_kernel<N, K, B_MN>;
  constexpr int kPSmem = PCfg<N>::kSmem;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmem) != cudaSuccess)
    return MLA_ERR_CUDA;
  const int nslices = NT / kPN;
  const int64_t items = (int64_t)((R + kRowTile - 1) / kRowTile) * H * nslices;
  if (items > (int64_t)1 << 30) return MLA_ERR_INVALID_ARG;
  const int grid = (int)(items < sms ? items : sms);  // persistent: one CTA per SM
  kern<<<grid, kPThreads, kPSmem, stream>>>(prm, R, H, nslices);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace
}  // namespace mla

extern "C" mla_status_t mla_absorb_q(const void* q_heads, const void* w_uk, void* q_nope, int R, int H,
                                     void* stream) {
  return mla::launch_absorb<512, 128, 128, true>(q_heads, w_uk, q_nope, R, H, static_cast<cudaStream_t>(stream));
}

extern "C" mla_status_t mla_absorb_out(const void* o_latent, const void* w_uv, void* y, int R, int H,
                                       void* stream) {
  return mla::launch_absorb<128, 128, 512, false>(o_latent, w_uv, y, R, H, static_cast<cudaStream_t>(stream));
}
