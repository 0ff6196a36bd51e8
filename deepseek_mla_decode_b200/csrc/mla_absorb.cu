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
// One CTA (128 threads) computes 128 rows x 128 output columns of one head: TMA loads
// the row tile and the head's weight slice into shared memory (128-byte swizzle), one
// thread issues 1-CTA tcgen05 MMAs (M = 128, N = 128) into a TMEM accumulator, and the
// four warps move their 32 TMEM lanes (rows) out through a swizzled staging tile and
// TMA stores.  The q side's 512 output columns are four CTAs; the out side's 512-deep
// contraction runs in four phases of 128.  Each CTA holds 64 KB of shared memory, so
// three share an SM and one's loads overlap another's MMAs and stores.  Memory-bound:
// the weights (16.8 MB per projection for 128 heads) are read once from HBM, the rows
// once per row tile and column slice (L2 serves the repeats); rows past R are
// zero-filled on load and clipped on store.
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

constexpr int kAbThreads = 128;
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
// Unbounded waits are not used: every wait gives up after 1 s (a protocol bug then
// leaves a wrong result, not a hung GPU).
__device__ __forceinline__ void wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t deadline = globaltimer_ns() + 1000000000ull;
  while (!mbar_try_wait(bar, parity) && globaltimer_ns() < deadline) {
  }
}

// N output columns per CTA (slice blockIdx.z of the projection's), K contraction,
// weights MN-major (q side: W_UK[h] is [k][n]) or K-major (out side: W_UV[h] is
// [n][k]); the contraction runs in phases of KP.
template <int N, int K, bool B_MN, int KP>
__global__ void __launch_bounds__(kAbThreads) absorb_kernel(const __grid_constant__ AbsorbParams p) {
  static_assert(K % KP == 0 && KP % 64 == 0 && N % 64 == 0, "tile shape");
  constexpr int kKB = KP / 64;                                   // 64-wide k blocks per phase
  constexpr int kABytes = kKB * 2 * kBox;                        // 128 rows x KP
  constexpr int kBBytes = B_MN ? kKB * (N / 64) * kBox : kKB * (N / 64) * kBox;  // KP x N either way
  constexpr int kNMma = N > 256 ? 256 : N;                       // N of one MMA
  constexpr uint32_t kIdesc = make_idesc_bf16(128, kNMma, false, B_MN);
  constexpr uint32_t kCols = N < 32 ? 32 : N;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_load, bar_mma, bar_done;
  __shared__ uint32_t tmem_base;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sA = smem_u32(smem), sB = sA + kABytes;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y, r0 = blockIdx.x * kRowTile, n0 = blockIdx.z * N;

  if (tid == 0) {
    mbar_init(smem_u32(&bar_load), 1);
    mbar_init(smem_u32(&bar_mma), 1);
    mbar_init(smem_u32(&bar_done), 1);
    fence_mbar_init();
    prefetch_tmap(&p.tm_a);
    prefetch_tmap(&p.tm_b);
    prefetch_tmap(&p.tm_c);
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base)),
                 "r"(kCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (tid == 0) {
    const uint32_t bl = smem_u32(&bar_load), bm = smem_u32(&bar_mma);
    for (int ph = 0; ph < K / KP; ++ph) {
      if (ph > 0) wait_bounded(bm, (ph - 1) & 1);  // the previous phase's MMAs have read the tiles
      expect_tx(bl, kABytes + kBBytes);
      for (int i = 0; i < kKB; ++i) {
        const int k0 = ph * KP + 64 * i;
        tma_load_3d(sA + i * 2 * kBox, &p.tm_a, bl, k0, h, r0);
        if (B_MN) {
          for (int j = 0; j < N / 64; ++j)
            tma_load_3d(sB + (i * (N / 64) + j) * kBox, &p.tm_b, bl, n0 + 64 * j, k0, h);
        } else {
          tma_load_3d(sB + i * (N / 64) * kBox, &p.tm_b, bl, k0, n0, h);
        }
      }
      wait_bounded(bl, ph & 1);
      tc_fence_after();
      // A (rows) K-major: 128-byte rows, 8-row groups 1024 B apart, K step = 32 B.
      // B MN-major: 64-wide column blocks 8 KB apart (LBO), 8-row k groups 1024 B apart,
      // K step = 16 rows = 2048 B.  B K-major: like A with N rows.
      for (int i = 0; i < kKB; ++i) {
        for (int s = 0; s < 4; ++s) {
          const uint64_t a = make_smem_desc(sA + i * 2 * kBox + 32 * s, 16, 1024, kSwizzle128B);
          for (int nh = 0; nh < N / kNMma; ++nh) {
            uint64_t b;
            if (B_MN)
              b = make_smem_desc(sB + (i * (N / 64) + nh * (kNMma / 64)) * kBox + 2048 * s, kBox, 1024, kSwizzle128B);
            else
              b = make_smem_desc(sB + i * (N / 64) * kBox + 32 * s, 16, 1024, kSwizzle128B);
            umma_1sm(tmem + nh * kNMma, a, b, kIdesc, (ph | i | s) != 0);
          }
        }
      }
      commit_1sm(bm);
    }
    commit_1sm(smem_u32(&bar_done));  // completes once every MMA above has
  }
  // every thread waits for all MMAs on a barrier with a single phase (a parity wait on
  // bar_mma, which completes once per phase, could alias a later phase)
  wait_bounded(smem_u32(&bar_done), 0);
  tc_fence_after();

  // epilogue: warp w owns TMEM lanes (rows) 32w..32w+31; column block j of 64 goes to
  // staging box j ([128 rows][128 B], 128-byte swizzle), then one thread stores them
  const int m = 32 * warp + lane;
  const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
#pragma unroll 1
  for (int j = 0; j < N / 64; ++j) {
    uint32_t w[32];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      uint32_t o[32];
      tmem_ld32(tmem + lane_off + 64 * j + 32 * hf, o);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 16; ++k) w[16 * hf + k] = pack2(__uint_as_float(o[2 * k]), __uint_as_float(o[2 * k + 1]));
    }
    const uint32_t row = sA + j * 2 * kBox + m * 128;
#pragma unroll
    for (int q = 0; q < 8; ++q)
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + ((q ^ (m & 7)) << 4)), "r"(w[4 * q]),
                   "r"(w[4 * q + 1]), "r"(w[4 * q + 2]), "r"(w[4 * q + 3])
                   : "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    for (int j = 0; j < N / 64; ++j) tma_store_3d(&p.tm_c, sA + j * 2 * kBox, n0 + 64 * j, h, r0);
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols) : "memory");
}

template <int N, int K, bool B_MN, int KP>
constexpr int absorb_smem() {
  return (KP / 64) * 2 * kBox + (KP / 64) * (N / 64) * kBox + 1024;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// NT output columns in all, N per CTA
template <int NT, int N, int K, bool B_MN, int KP>
mla_status_t launch_absorb(const void* rows, const void* w, void* outp, int R, int H, cudaStream_t stream) {
  static_assert(NT % N == 0, "column slices");
  static_assert(2 * (KP / 64) * kBox >= (N / 64) * 2 * kBox, "the epilogue stages the output in the row tile's space");
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
    const cuuint32_t box[3] = {64, (cuuint32_t)N, 1};
    if (!encode_tiled_bf16(&prm.tm_b, w, 3, dims, strides, box)) return MLA_ERR_INVALID_ARG;
  }
  {
    const cuuint64_t dims[3] = {(cuuint64_t)NT, (cuuint64_t)H, (cuuint64_t)R};
    const cuuint64_t strides[2] = {(cuuint64_t)NT * 2, (cuuint64_t)H * NT * 2};
    const cuuint32_t box[3] = {64, 1, kRowTile};
    if (!encode_tiled_bf16(&prm.tm_c, outp, 3, dims, strides, box)) return MLA_ERR_INVALID_ARG;
  }
  constexpr int smem = absorb_smem<N, K, B_MN, KP>();
  auto kern = absorb_kernel<N, K, B_MN, KP>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return MLA_ERR_CUDA;
  dim3 grid((R + kRowTile - 1) / kRowTile, H, NT / N);
  kern<<<grid, kAbThreads, smem, stream>>>(prm);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace
}  // namespace mla

extern "C" mla_status_t mla_absorb_q(const void* q_heads, const void* w_uk, void* q_nope, int R, int H,
                                     void* stream) {
  return mla::launch_absorb<512, 128, 128, true, 128>(q_heads, w_uk, q_nope, R, H,
                                                      static_cast<cudaStream_t>(stream));
}

extern "C" mla_status_t mla_absorb_out(const void* o_latent, const void* w_uv, void* y, int R, int H,
                                       void* stream) {
  return mla::launch_absorb<128, 128, 512, false, 128>(o_latent, w_uv, y, R, H, static_cast<cudaStream_t>(stream));
}
