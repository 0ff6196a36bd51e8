// Quantised causal prefill attention (SageAttention-style) for sm_100a, head dim 192.
//
// Paddle 3.0 inference upgrade article, long-sequence section: Q and K in INT8, the
// INT32 scores converted to FP32 and dequantised, an online softmax, its weights P
// quantised to FP8 and multiplied with the FP8 V, the product dequantised by V's
// scale.  Here (the quantisers are in sage_quant.cu):
//   S_ij   = (Qc_i . Kc_j) * s_q[i] * s_k[j]          tcgen05 kind::i8, int32 in TMEM
//   x_ij   = S_ij * softmax_scale * log2(e),   causal j <= i
//   m      = running row maximum over 128-key blocks (updated at every block)
//   Pc_ij  = e4m3(2^(x_ij - m) * 448)                  P in [0, 1] scaled to e4m3's range
//   O_acc += Pc . Vc  (e4m3 x e4m3)                    tcgen05 kind::f8f6f4, fp32 in TMEM
//   l     += sum of the values of Pc;  O_acc, l scaled by 2^(m_old - m) when m grows
//   out_i  = O_acc * s_v / l,   lse_i = (m + log2(l / 448)) * ln 2
// i.e. the output is normalised by the quantised weights that entered the product.
//
// One CTA = one head x two adjacent 128-row query tiles (rows 256 i .. 256 i + 255),
// longest rows first.  Warp 0 issues the TMA loads (both tiles' Q once; per key block
// its K slab, V slab and the keys' scales, shared by the two tiles), warp 1 the MMAs,
// warps 4..7 the softmax of tile 0 and warps 8..11 that of tile 1 (one thread per
// query row = TMEM lane).  Per key block j the MMA warp issues QK(0, j+1), QK(1, j+1),
// PV(0, j), PV(1, j): the next block's scores need only this block's scores read out
// of TMEM, so they are computed while both tiles' softmax works on block j, and each
// tile's softmax waits for the tensor core only briefly between blocks.
// TMEM: S of tile t in columns [128 t, 128 t + 128), O of tile t in [256 + 128 t, ...).
// Every wait is bounded: a timeout sets MLA_DEVICE_ERR_TIMEOUT, every role stops at its
// next wait, the CTA drains its tensor-core work and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <cstring>
#include "mla_internal.h"
#include "sage_internal.h"
#include "ptx_sm100.cuh"

namespace mla {
namespace sage {

using namespace ptx;

namespace {

constexpr int kThreads = 384;
constexpr int kProducerWarp = 0, kMmaWarp = 1, kSoftmaxWarp0 = 4;  // tile t: warps 4 + 4t .. 7 + 4t
constexpr int kTiles = 2;
constexpr int kStages = 3;
constexpr int kChunk = kBlockN * 64;          // one [128 rows][64 B] SW64 box (8 KB)
constexpr int kQBytes = 3 * kChunk;           // Q of a tile: 128 rows x 192 B
constexpr int kKBytes = 3 * kChunk;           // K slab: 128 keys x 192 B
constexpr int kVBytes = kDV * kBlockN;        // V slab: 128 channels x 128 keys (e4m3)
constexpr int kStageBytes = kKBytes + kVBytes;  // 40 KB, a multiple of 1024
constexpr int kPBytes = kBlockM * kBlockN;    // P of a tile: 128 rows x 128 keys (e4m3)
constexpr int kSmemQ = 0, kSmemP = kSmemQ + kTiles * kQBytes, kSmemStage = kSmemP + kTiles * kPBytes;
constexpr int kSmemScale = kSmemStage + kStages * kStageBytes;
constexpr int kSmemDyn = kSmemScale + kStages * kBlockN * 4;
constexpr uint32_t kTmemS0 = 0, kTmemO = 256, kTmemCols = 512;
constexpr uint64_t kDrainWaitNs = 100000000ull;
constexpr uint64_t kQuiesceNs = 500000ull;
// setmaxnreg split: warps 0..3 (producer, MMA, two idle) give registers to the softmax
// warpgroups; 128 x 56 + 256 x 224 = 384 x 168, the launch allocation.
constexpr int kRegsIssue = 56, kRegsSoftmax = 224;
static_assert(128 * kRegsIssue + 256 * kRegsSoftmax == kThreads * 168, "register split");

// Instruction descriptor (D format, A/B formats, K-major A and B, N, M).
__host__ __device__ constexpr uint32_t make_idesc(uint32_t dfmt, uint32_t afmt, uint32_t bfmt, int M, int N) {
  return (dfmt << 4) | (afmt << 7) | (bfmt << 10) | ((static_cast<uint32_t>(N) >> 3) << 17) |
         ((static_cast<uint32_t>(M) >> 4) << 24);
}
constexpr uint32_t kIdescQK = make_idesc(2 /*s32*/, 1 /*s8*/, 1 /*s8*/, kBlockM, kBlockN);
constexpr uint32_t kIdescPV = make_idesc(1 /*f32*/, 0 /*e4m3*/, 0 /*e4m3*/, kBlockM, kDV);

struct Params {
  CUtensorMap tm_q;  // q8 as [H][S_pad][192] bytes, box {64, 128, 1}, 64-byte swizzle
  CUtensorMap tm_k;  // k8, same
  CUtensorMap tm_v;  // vt8 as [H * 128][S_pad] bytes, box {128, 128}, 128-byte swizzle
  const float* sq;
  const float* sk;
  const float* sv;
  __nv_bfloat16* out;  // [S][H][128]
  float* lse;          // [S][H]
  int32_t* status;
  uint64_t timeout_ns;
  int S, S_pad, H, nqb;
  float scale_log2;
};

struct __align__(8) Ctrl {
  uint64_t full[kStages];   // K, V and scales of a stage landed (count 1 + tx)
  uint64_t empty[kStages];  // both tiles' PV of the stage's block done (commit)
  uint64_t q_full;          // both tiles' Q landed
  uint64_t s_full[kTiles];  // S of a tile written (commit)
  uint64_t s_free[kTiles];  // S of a tile read by its 128 softmax threads
  uint64_t p_full[kTiles];  // P of a tile written and its O rescaled (one arrive)
  uint64_t p_free[kTiles];  // PV of a tile done (commit)
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort;
};

__device__ __forceinline__ void set_status(const Params& p, int bits) {
  if (p.status) atomicOr(p.status, bits);
}

__device__ __forceinline__ bool wait_bar(Ctrl* c, const Params& p, uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t deadline = globaltimer_ns() + p.timeout_ns;
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (c->abort) return false;
    if (globaltimer_ns() > deadline) {
      c->abort = 1;
      set_status(p, kErrTimeout);
      return false;
    }
  }
}

__device__ __forceinline__ void expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void tma_3d(uint32_t dst, const void* tmap, uint32_t bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma_2d(uint32_t dst, const void* tmap, uint32_t bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void mma_i8(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma_f8(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
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
template <int kRegs>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegs));
}
template <int kRegs>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegs));
}
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// two fp32 -> two e4m3 (nearest even, saturating), lo in the low byte
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
// acc + the values of the two e4m3 codes in the low 16 bits of c (exact f16 values,
// added to the fp32 accumulator by the mixed-precision f32 += f16 add)
__device__ __forceinline__ float add_e4m3x2_to(float acc, uint32_t c) {
  float r;
  asm("{\n\t.reg .b16 lo, x, y;\n\t.reg .b32 h2;\n\t.reg .f32 t;\n\tcvt.u16.u32 lo, %1;\n\t"
      "cvt.rn.f16x2.e4m3x2 h2, lo;\n\tmov.b32 {x, y}, h2;\n\t"
      "add.rn.f32.f16 t, x, %2;\n\tadd.rn.f32.f16 %0, y, t;\n\t}"
      : "=f"(r)
      : "r"(c), "f"(acc));
  return r;
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__global__ void __launch_bounds__(kThreads, 1) sage_attn_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ Ctrl ctrl;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + kSmemQ, sP = sbase + kSmemP, sStage = sbase + kSmemStage, sScale = sbase + kSmemScale;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // longest rows first: work item w -> tile pair npair - 1 - w / H, head w % H
  const int npair = (p.nqb + 1) / 2;
  const int pair = npair - 1 - (int)(blockIdx.x / p.H);
  const int h = (int)(blockIdx.x % p.H);
  const int qb0 = 2 * pair;
  // causal: tile t (query block qb0 + t) sees key blocks 0..qb0 + t; a second tile past
  // the last query block (odd block count) does nothing
  const int nk0 = qb0 + 1, nk1 = (qb0 + 1 < p.nqb) ? qb0 + 2 : 0;
  const int nkb = max(nk0, nk1);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&ctrl.full[s]), 1);
      mbar_init(smem_u32(&ctrl.empty[s]), 1);
    }
    mbar_init(smem_u32(&ctrl.q_full), 1);
    for (int t = 0; t < kTiles; ++t) {
      mbar_init(smem_u32(&ctrl.s_full[t]), 1);
      mbar_init(smem_u32(&ctrl.s_free[t]), kBlockM);
      mbar_init(smem_u32(&ctrl.p_full[t]), 1);
      mbar_init(smem_u32(&ctrl.p_free[t]), 1);
    }
    mbar_init(smem_u32(&ctrl.drain), 1);
    ctrl.abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&ctrl.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&p.tm_q);
    prefetch_tmap(&p.tm_k);
    prefetch_tmap(&p.tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl.tmem_base;

  if (warp == kProducerWarp) {
    // =====================================================================
    // TMA producer (lane 0 issues; the warp waits together)
    // =====================================================================
    regs_dec<kRegsIssue>();
    bool ok = true;
    if (lane == 0) {
      const int ntiles = nk1 > 0 ? 2 : 1;
      expect_tx(smem_u32(&ctrl.q_full), ntiles * kQBytes);
      for (int t = 0; t < ntiles; ++t)
        for (int c = 0; c < 3; ++c)
          tma_3d(sQ + t * kQBytes + c * kChunk, &p.tm_q, smem_u32(&ctrl.q_full), 64 * c, (qb0 + t) * kBlockM, h);
    }
    for (int j = 0; j < nkb && ok; ++j) {
      const int st = j % kStages, use = j / kStages;
      if (use > 0) ok = __shfl_sync(0xffffffffu, wait_bar(&ctrl, p, smem_u32(&ctrl.empty[st]), (use - 1) & 1), 0);
      if (!ok) break;
      if (lane == 0) {
        const uint32_t fb = smem_u32(&ctrl.full[st]);
        const uint32_t sk = sStage + st * kStageBytes;
        expect_tx(fb, kStageBytes + kBlockN * 4);
        for (int c = 0; c < 3; ++c) tma_3d(sk + c * kChunk, &p.tm_k, fb, 64 * c, j * kBlockN, h);
        tma_2d(sk + kKBytes, &p.tm_v, fb, j * kBlockN, h * kDV);
        bulk_g2s(sScale + st * kBlockN * 4, p.sk + (int64_t)h * p.S_pad + j * kBlockN, kBlockN * 4, fb);
      }
      __syncwarp();
    }
  } else if (warp == kMmaWarp) {
    // =====================================================================
    // MMA issuer: QK(0, 0), QK(1, 0), then per key block j: QK(0, j + 1), QK(1, j + 1),
    // PV(0, j), PV(1, j), and the block's stage is released
    // =====================================================================
    regs_dec<kRegsIssue>();
    bool ok = wait_bar(&ctrl, p, smem_u32(&ctrl.q_full), 0);
    const bool elected = elect_one();
    // K-major operands: Q / K slabs are three [128 rows][64 B] boxes with the 64-byte
    // swizzle (8-row groups 512 B apart), one K step of 32 int8 = 32 B; P and V are
    // [128 rows][128 B] with the 128-byte swizzle (groups 1024 B apart), one K step of
    // 32 e4m3 = 32 B.  Descriptor start fields count 16-byte units.
    const uint64_t dq0 = make_smem_desc(sQ, 16, 512, kSwizzle64B);
    const uint64_t dk0 = make_smem_desc(sStage, 16, 512, kSwizzle64B);
    const uint64_t dv0 = make_smem_desc(sStage + kKBytes, 16, 1024, kSwizzle128B);
    const uint64_t dp0 = make_smem_desc(sP, 16, 1024, kSwizzle128B);
    constexpr uint64_t kChunkD = kChunk >> 4, kStageD = kStageBytes >> 4, kQD = kQBytes >> 4, kPD = kPBytes >> 4;
    auto qk = [&](int t, int j) {
      const int st = j % kStages;
      ok = ok && wait_bar(&ctrl, p, smem_u32(&ctrl.full[st]), (j / kStages) & 1);
      if (ok && j >= 1) ok = wait_bar(&ctrl, p, smem_u32(&ctrl.s_free[t]), (j - 1) & 1);
      if (!ok) return;
      tc_fence_after();
      if (elected) {
#pragma unroll
        for (int ks = 0; ks < 6; ++ks) {
          const uint64_t off = (ks >> 1) * kChunkD + (ks & 1) * 2;
          mma_i8(tmem + kTmemS0 + 128 * t, dq0 + t * kQD + off, dk0 + st * kStageD + off, kIdescQK, ks > 0);
        }
        commit(smem_u32(&ctrl.s_full[t]));
      }
      __syncwarp();
    };
    auto pv = [&](int t, int j) {
      const int st = j % kStages;
      ok = ok && wait_bar(&ctrl, p, smem_u32(&ctrl.p_full[t]), j & 1);
      if (!ok) return;
      tc_fence_after();
      if (elected) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_f8(tmem + kTmemO + 128 * t, dp0 + t * kPD + ks * 2, dv0 + st * kStageD + ks * 2, kIdescPV,
                 (j > 0 || ks > 0));
        commit(smem_u32(&ctrl.p_free[t]));
      }
      __syncwarp();
    };
    qk(0, 0);
    if (nk1 > 0) qk(1, 0);
    for (int j = 0; j < nkb && ok; ++j) {
      // S of block j+1 needs only S of block j read out (s_free, right after the
      // softmax's TMEM load), so it is computed while the softmax works on block j
#pragma unroll
      for (int t = 0; t < kTiles; ++t)
        if (j + 1 < (t == 0 ? nk0 : nk1)) qk(t, j + 1);
#pragma unroll
      for (int t = 0; t < kTiles; ++t)
        if (j < (t == 0 ? nk0 : nk1)) pv(t, j);
      if (ok && elected) commit(smem_u32(&ctrl.empty[j % kStages]));  // after both tiles' PV of block j
      __syncwarp();
    }
  } else if (warp >= kSoftmaxWarp0) {
    // =====================================================================
    // softmax + epilogue: tile t, thread = query row r of the tile (TMEM lane r)
    // =====================================================================
    regs_inc<kRegsSoftmax>();
    const int t = (warp - kSoftmaxWarp0) >> 2;
    const int r = tid - (kSoftmaxWarp0 + 4 * t) * 32;  // 0..127
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int row = (qb0 + t) * kBlockM + r;
    const int nkt = t == 0 ? nk0 : nk1;
    const bool valid = row < p.S;
    const float cr = valid ? p.sq[(int64_t)h * p.S_pad + row] * p.scale_log2 : 0.f;
    const uint32_t sPt = sP + t * kPBytes;
    const uint32_t tS = tmem + kTmemS0 + 128 * t + lane_off, tO = tmem + kTmemO + 128 * t + lane_off;
    float m = -INFINITY, l = 0.f;
    bool ok = true, go = nkt > 0;
    const float* sc_all = reinterpret_cast<const float*>(smem + kSmemScale);
    for (int j = 0; j < nkt && go; ++j) {
      const int stg = j % kStages;
      ok = wait_bar(&ctrl, p, smem_u32(&ctrl.s_full[t]), j & 1) && ok;
      // the stage's scales landed with its TMA (already complete; this wait makes them
      // visible to these threads)
      ok = wait_bar(&ctrl, p, smem_u32(&ctrl.full[stg]), (j / kStages) & 1) && ok;
      tc_fence_after();
      uint32_t s[128];
      if (ok) {
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * c]));
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&ctrl.s_free[t]));  // S of this tile may be overwritten
      // key-scaled scores x' = S_int * s_k of the visible keys (key j*128 + c <= row); the
      // row factor cr = s_q * scale * log2(e) > 0 (or 0 for a zero or invalid row) keeps
      // their order, so it is applied once to the maximum and inside the exponent's FMA
      const float* sc = sc_all + stg * kBlockN;
      const int vis = valid ? max(0, min(kBlockN, row - j * kBlockN + 1)) : 0;
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int c = 0; c < kBlockN; c += 2) {
        const float x0 = (float)(int)s[c] * sc[c];
        const float x1 = (float)(int)s[c + 1] * sc[c + 1];
        s[c] = __float_as_uint(x0);
        s[c + 1] = __float_as_uint(x1);
        if (c < vis) mx0 = fmaxf(mx0, x0);
        if (c + 1 < vis) mx1 = fmaxf(mx1, x1);
      }
      const float m_new = fmaxf(m, vis > 0 ? cr * fmaxf(mx0, mx1) : -INFINITY);
      const float alpha = (m_new == -INFINITY || m == m_new) ? 1.f : (m == -INFINITY ? 0.f : fast_exp2(m - m_new));
      // P * 448 = 2^(x - (m_new - log2 448)): the scale to e4m3's range rides in the
      // exponent's offset
      const float moff = m_new - 8.8073549220576041f;
      uint32_t pc[32];
      float lsum0 = 0.f, lsum1 = 0.f;
      if (__all_sync(0xffffffffu, vis == kBlockN)) {  // every key of the block visible (warp-uniform)
#pragma unroll
        for (int c = 0; c < kBlockN; c += 4) {
          const uint32_t lo = e4m3x2(fast_exp2(fmaf(__uint_as_float(s[c]), cr, -moff)), fast_exp2(fmaf(__uint_as_float(s[c + 1]), cr, -moff)));
          const uint32_t hi =
              e4m3x2(fast_exp2(fmaf(__uint_as_float(s[c + 2]), cr, -moff)), fast_exp2(fmaf(__uint_as_float(s[c + 3]), cr, -moff)));
          pc[c >> 2] = lo | (hi << 16);
          lsum0 = add_e4m3x2_to(lsum0, lo);
          lsum1 = add_e4m3x2_to(lsum1, hi);
        }
      } else {
#pragma unroll
        for (int c = 0; c < kBlockN; c += 4) {
          const float p0 = (c < vis) ? fast_exp2(fmaf(__uint_as_float(s[c]), cr, -moff)) : 0.f;
          const float p1 = (c + 1 < vis) ? fast_exp2(fmaf(__uint_as_float(s[c + 1]), cr, -moff)) : 0.f;
          const float p2 = (c + 2 < vis) ? fast_exp2(fmaf(__uint_as_float(s[c + 2]), cr, -moff)) : 0.f;
          const float p3 = (c + 3 < vis) ? fast_exp2(fmaf(__uint_as_float(s[c + 3]), cr, -moff)) : 0.f;
          const uint32_t lo = e4m3x2(p0, p1), hi = e4m3x2(p2, p3);
          pc[c >> 2] = lo | (hi << 16);
          lsum0 = add_e4m3x2_to(lsum0, lo);
          lsum1 = add_e4m3x2_to(lsum1, hi);
        }
      }
      l = l * alpha + (lsum0 + lsum1);
      m = m_new;
      // PV of this tile's previous block must be done before P is overwritten or O
      // rescaled
      if (j > 0) ok = wait_bar(&ctrl, p, smem_u32(&ctrl.p_free[t]), (j - 1) & 1) && ok;
      tc_fence_after();
      if (j > 0 && ok && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
        for (int c = 0; c < kDV; c += 32) {
          uint32_t o[32];
          tmem_ld32(tO + c, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tO + c, o);
        }
        tmem_wait_st();
      }
      // P row r: 128 codes, 128-byte swizzle (16-byte granule g at g ^ (r & 7))
      {
        const uint32_t prow = sPt + r * kBlockN;
#pragma unroll
        for (int g = 0; g < 8; ++g)
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow + ((g ^ (r & 7)) << 4)),
                       "r"(pc[4 * g]), "r"(pc[4 * g + 1]), "r"(pc[4 * g + 2]), "r"(pc[4 * g + 3])
                       : "memory");
      }
      fence_proxy_async_smem();
      tc_fence_before();
      go = named_bar_and(1 + t, kBlockM, ok);
      if (go && r == 0) mbar_arrive(smem_u32(&ctrl.p_full[t]));
    }
    // epilogue after the tile's last PV: out = O * s_v / l, lse = (m + log2(l / 448)) ln 2
    if (go) ok = wait_bar(&ctrl, p, smem_u32(&ctrl.p_free[t]), (nkt - 1) & 1) && ok;
    tc_fence_after();
    if (nkt > 0) go = named_bar_and(1 + t, kBlockM, ok && go);
    if (go) {
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      const float* sv = p.sv + h * kDV;
      __nv_bfloat16* orow = p.out + ((int64_t)row * p.H + h) * kDV;
#pragma unroll 1
      for (int c = 0; c < kDV; c += 32) {
        uint32_t o[32];
        tmem_ld32(tO + c, o);
        tmem_wait_ld();
        if (valid) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(o[2 * i]) * inv * sv[c + 2 * i],
                                                            __uint_as_float(o[2 * i + 1]) * inv * sv[c + 2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t*>(&b2);
          }
#pragma unroll
          for (int i = 0; i < 4; ++i)
            reinterpret_cast<uint4*>(orow + c)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      if (valid) p.lse[(int64_t)row * p.H + h] = (m + __log2f(l * (1.f / 448.f))) * 0.69314718055994531f;
    }
  } else {
    regs_dec<kRegsIssue>();  // the idle warps of the first warpgroup
  }

  // ---- teardown ------------------------------------------------------------
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (ctrl.abort) {
    // a wait ran out: let the tensor-core work issued before it finish (a commit
    // arrives once all of it has), and give TMA loads in flight time to land
    if (warp == kMmaWarp) {
      if (elect_one()) commit(smem_u32(&ctrl.drain));
      __syncwarp();
      const uint64_t dl = globaltimer_ns() + kDrainWaitNs;
      while (!mbar_try_wait(smem_u32(&ctrl.drain), 0) && globaltimer_ns() < dl) {
      }
    }
    if (tid == 0) {
      const uint64_t until = globaltimer_ns() + kQuiesceNs;
      while (globaltimer_ns() < until) {
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace

cudaError_t attention_setup() {
  return cudaFuncSetAttribute(sage_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemDyn + 1024);
}

cudaError_t launch_attention(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                             const Workspace& ws, int S, int H, float softmax_scale, void* out, float* lse,
                             int32_t* status, uint64_t timeout_ns, cudaStream_t stream) {
  Params prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.tm_q = tm_q;
  prm.tm_k = tm_k;
  prm.tm_v = tm_v;
  prm.sq = ws.sq;
  prm.sk = ws.sk;
  prm.sv = ws.sv;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.status = status;
  prm.timeout_ns = timeout_ns;
  prm.S = S;
  prm.S_pad = padded_len(S);
  prm.H = H;
  prm.nqb = prm.S_pad / kBlockM;
  prm.scale_log2 = softmax_scale * 1.4426950408889634f;
  const unsigned grid = (unsigned)((prm.nqb + 1) / 2) * (unsigned)H;
  sage_attn_kernel<<<grid, kThreads, kSmemDyn + 1024, stream>>>(prm);
  return cudaGetLastError();
}

}  // namespace sage
}  // namespace mla
