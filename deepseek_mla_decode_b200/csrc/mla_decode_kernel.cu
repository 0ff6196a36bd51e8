// Split-KV weight-absorbed MLA decode kernel for sm_100a.
//
// Math (weight-absorbed MLA: KsanaLLM 0.6.0 release notes, section 2.1; softmax scale
// 1/sqrt(192): Paddle 3.0 inference article, long-sequence section; s_q > 1 draft
// tokens with a causal mask among them: same article, speculative decoding):
//     S = Q K^T,  Q = [q_nope | q_pe] (rows x 576),  K = cache rows (keys x 576)
//     O = softmax(scale * S) V,  V = first 512 columns of the same cache rows
//
// Work unit: a 2-CTA cluster owns 128 query rows (row = token * H + head) of one
// sequence piece (a contiguous block range from the split-KV schedule).  CTA r holds
// rows [64r, 64r + 64) and accumulates their full 512-wide output in its TMEM.
// Both GEMMs are cta_group::2 tcgen05 MMAs with M = 128 (64 rows per CTA), N = 256:
//   QK: per 256-key tile, CTA r stages keys [128r, 128r + 128) of the tile (its half
//       of the B operand) in 64-dim chunks; each CTA receives S for its 64 rows over
//       all 256 keys (TMEM "2x2" layout: lanes 0-63 keys 0..127, lanes 64-127 keys
//       128..255, 128 columns).
//   PV: for each 256-wide half h of the output, CTA r stages V[key block, dims
//       256h + 128r + (0..127)] (its half of N); each CTA receives O for its rows over
//       all 256 dims of that half.
// O uses TMEM columns [0, 256), the two S buffers [256, 384) and [384, 512).
//
// Cache formats: the bf16 cache ([block][64][576] bf16) is staged by TMA straight into
// the ring the MMAs read.  The FP8 cache (656-byte rows: e4m3 codes of c_kv / scale,
// bf16 k_pe / scale, fp32 scale; the row format of mla_fp8.cu) is staged by TMA into a
// separate ring of raw bytes, and converter warps turn each stage into the same bf16
// ring slot the bf16 path would have loaded.  The codes convert to bf16 exactly (their
// values are the e4m3 values); the per-key scale multiplies the scores (S = scale * S')
// and the weights that enter PV (P' = bf16(e * scale)), and the row sums stay in the
// unscaled weights e.
//
// Warp roles, bf16 cache (384 threads): warps 0, 2, 3 = TMA producers (ring stage k is
// issued by producer k % 3; warp 0 also loads Q), warp 1 = MMA issuer (leader CTA only)
// and TMEM owner, warps 4..11 = softmax / correction / epilogue (thread = one row x 64
// keys of S, one row x 128 dims of O).  FP8 cache (512 threads): the same, plus warps
// 12..15 = converters; setmaxnreg moves registers from the producer/MMA and converter
// warpgroups to the softmax warpgroups.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <cstring>
#include "mla_internal.h"
#include "ptx_sm100.cuh"

namespace mla {

using namespace ptx;

namespace {

constexpr int kNumProducers = 3;  // warps 0, 2, 3 (warp 0 also loads Q)
constexpr int kMmaWarp = 1;
constexpr int kSoftmaxWarp0 = 4;   // warps 4..11
constexpr int kNumSoftmaxThreads = 256;
constexpr int kConvWarp0 = 12;     // FP8 cache: warps 12..15 (128 converter threads)
constexpr int kMaxStages = 7;
constexpr int kStageBytes = 16384;  // one bf16 ring slot
constexpr int kChunkBytes = 8192;  // one 64-row x 64-column bf16 SW128 box
constexpr int kQChunks = 9;        // 576 / 64
constexpr int kQBytes = kQChunks * kChunkBytes;
constexpr int kPBytes = 4 * kChunkBytes;  // 64 rows x 256 keys bf16
constexpr int kSmemQ = 0;
constexpr int kSmemP = kSmemQ + kQBytes;
constexpr int kSmemRing = kSmemP + kPBytes;
// The partition's last epilogue stages each of its (up to 4) rounds in its own 32 KB
// from the start of shared memory: Q, P and the ring are contiguous and all idle then.
constexpr int kEpiRoundBytes = 4 * kChunkBytes;
// FP8 cache: raw stages of 8 KB (an e4m3 slab or one block of scaled k_pe) and two
// buffers of per-key scales (4 blocks x 64 rows x 16 bytes, the scale in the first 4)
constexpr int kStgBytes = 8192;
constexpr int kMaxStg = 8;
constexpr int kScaleBufBytes = 4096;
constexpr int kSlabBlockBytes = 64 * 64;           // one block's 64-column slab of codes
constexpr int kScaleBlockBytes = 64 * 16;          // one block's scales (16 bytes per row)
constexpr int kStgPerQk = 8 + 2;                   // raw stages per tile for QK
// FP8 kernel register split (setmaxnreg, per warpgroup): warps 0-3 (producers, MMA),
// 4-11 (softmax), 12-15 (converters); 128 x (issue + conv) + 256 x softmax must equal
// the 512 x 128 registers the block is launched with.
constexpr int kRegsIssue = 88, kRegsConv = 88, kRegsSoftmax = 168;
static_assert(128 * (kRegsIssue + kRegsConv) + 256 * kRegsSoftmax == 512 * 128, "register split");

template <bool kFp8>
struct Cfg {
  static constexpr int kThreads = kFp8 ? 512 : 384;
  static constexpr int kStages = kFp8 ? 3 : 7;  // bf16 ring slots
  static constexpr int kStg = kFp8 ? 7 : 0;     // raw FP8 stages
  static constexpr int kSmemStg = kSmemRing + kStages * kStageBytes;
  static constexpr int kSmemScale = kSmemStg + kStg * kStgBytes;
  static constexpr int kSmemDyn = kSmemScale + (kFp8 ? 2 * kScaleBufBytes : 0);
  static_assert(kStages <= kMaxStages && kStg <= kMaxStg, "ring sizes");
  static_assert(4 * kEpiRoundBytes <= kSmemStg, "the last epilogue's staging stays inside Q, P and the ring");
};
constexpr uint32_t kTmemO = 0, kTmemS0 = 256, kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O is rescaled only when the max grows by > 2^8
constexpr uint32_t kIdescQK = make_idesc_bf16(128, 256, false, false);
constexpr uint32_t kIdescPV = make_idesc_bf16(128, 256, false, true);
constexpr int kBarSoftmax = 1;  // named barrier id for the 256 softmax threads
constexpr int kBarConv = 2;     // named barrier ids 2, 3 for the two converter groups
constexpr uint64_t kDrainWaitNs = 100000000ull;  // bound on the post-abort wait for tensor-core work
constexpr uint64_t kQuiesceNs = 500000ull;       // post-abort wait for TMA loads in flight

struct Params {
  // bf16 cache: tm_kv = [num_blocks][64][576] bf16, box {64, 64, 1}, SW128; tm_kv2 = the
  // same memory as [num_blocks][9][64][64], box {64, 64, 2, 1}, SW128.
  // FP8 cache: tm_kv = the packed rows as bytes [num_blocks][64][656], box {64, 64, 1}
  // (one 64-column slab of codes, no swizzle); tm_kv2 = the same bytes, box {128, 64, 1},
  // SW128 (a 128-column slab for PV).
  CUtensorMap tm_kv;
  CUtensorMap tm_kv2;
  CUtensorMap tm_kpe;   // FP8 cache: rows as [num_blocks][64][328] bf16, box {64, 64, 1} at column 256, SW128
  CUtensorMap tm_scl;   // FP8 cache: rows as [num_blocks][64][164] fp32, box {4, 64, 1} at column 160
  CUtensorMap tm_qn;  // [B*M][512] bf16, box {64, 64}, SW128
  CUtensorMap tm_qp;  // [B*M][64] bf16, box {64, 64}, SW128
  CUtensorMap tm_out;   // out as [B][M][512] bf16, box {64, 64, 1}, SW128 (TMA store)
  CUtensorMap tm_part;  // partial outputs as [slots][M][512] fp32, box {32, 64, 1}, SW128
  const int32_t* block_table;
  const int32_t* seqlens;
  const int32_t* q_lens;  // per-sequence query tokens (<= s_q), or null: s_q for every sequence
  // Token schedule (tok_rep > 0): the launch is an s_q = 1 decode of B = B_real * tok_rep
  // sequences; sequence u is token u % tok_rep of real sequence u / tok_rep, whose
  // length, table row and query count (tok_q_lens, or tok_rep each) it takes.
  const int32_t* tok_q_lens;
  int tok_rep, tok_causal;
  const int32_t* meta;
  __nv_bfloat16* out;
  float* lse;
  float* part_o;
  float* part_lse;
  int32_t* status;
  int64_t num_blocks;
  uint64_t timeout_ns;
  int max_blocks;
  int B, s_q, H, M;
  float scale_log2;
  int causal;
  int inject_stall;  // test hook: the MMA warp first waits on a barrier nothing completes
};

struct __align__(8) Ctrl {
  uint64_t full[kMaxStages];   // leader: stage landed in both CTAs (bf16: count 1 + tx of both
                               // CTAs; FP8: count 2, one converter arrival per CTA)
  uint64_t empty[kMaxStages];  // both: stage consumed by the MMAs (commit)
  uint64_t stg_full[kMaxStg];  // FP8, both: raw stage landed (count 1 + tx)
  uint64_t stg_empty[kMaxStg]; // FP8, both: raw stage read by the converters (count 1)
  uint64_t sc_full[2];         // FP8, both: scales of a tile landed (count 1 + tx)
  uint64_t sc_empty[2];        // FP8, both: scales of a tile used by the softmax (count 1)
  uint64_t q_full;          // leader: Q of both CTAs landed (count 1 + tx)
  uint64_t q_empty;         // both: last QK of the piece done (commit)
  uint64_t s_full[2];       // both: S buffer written (commit)
  uint64_t p_full;          // leader: P written in both CTAs (count 2)
  uint64_t p_free;          // both: PV done (commit)
  uint64_t o_free;          // leader: O read out by both CTAs (count 2)
  uint64_t drain;           // both: every tensor-core op issued before an abort completed (commit)
  uint64_t never;           // nothing arrives: the injected stall of the failure-path test waits on it
  uint32_t tmem_base;
  volatile int abort;
  volatile int peer_abort;  // written by the peer CTA at teardown
  float red_max[2][4][64];
  float red_sum[4][64];   // sum of the bf16-rounded weights (normalises the output)
  float red_sum32[4][64]; // sum of the fp32 weights (gives the lse)
  int bad_piece;
  int block_ids[4][128];  // each producer's window of the current piece's physical block ids
};
constexpr int kIdRing = 128;

struct Piece {
  int b, k_lo, k_hi, split, n, qlen;
};

// Keys of sequence u: its length, or with a token schedule the length of token
// u % tok_rep of its real sequence (token_seq_len; a real length beyond the table makes
// every token of that sequence invalid, as the real sequence would be).
__device__ __forceinline__ int seq_len(const Params& p, int u) {
  if (p.tok_rep == 0) return p.seqlens[u];
  const int r = u / p.tok_rep;
  const int n = p.seqlens[r];
  if ((int64_t)n > (int64_t)p.max_blocks * kBlockSize) return -1;
  return token_seq_len(n, p.tok_q_lens ? p.tok_q_lens[r] : p.tok_rep, u - r * p.tok_rep, p.tok_rep, p.tok_causal);
}
// Block-table row of sequence u.
__device__ __forceinline__ int64_t table_row(const Params& p, int u) {
  return p.tok_rep ? u / p.tok_rep : u;
}

// Block count of a sequence of n keys, or -1 when n is not a valid length for the table.
__device__ __forceinline__ int expected_blocks(const Params& p, int n) {
  if (n < 0 || (int64_t)n > (int64_t)p.max_blocks * kBlockSize) return -1;
  return (n + kBlockSize - 1) / kBlockSize;
}

// Query tokens of sequence b: q_lens[b] when given (must lie in [0, s_q]; -1 marks an
// invalid count), else s_q.
__device__ __forceinline__ int query_len(const Params& p, int b) {
  if (!p.q_lens) return p.s_q;
  const int l = p.q_lens[b];
  return (l < 0 || l > p.s_q) ? -1 : l;
}

// Walks the pieces of one partition.  Pieces of sequences whose length is invalid, or
// whose block count in the metadata is not the one their current length needs (a
// schedule built for other lengths), are skipped consistently by every role (producer
// warp 0 writes their NaN rows).  Piece bounds are clamped to the sequence's blocks, so
// no block-table entry past ceil(n / 64) is ever read.  With per-sequence query counts,
// a row tile that holds only padding tokens of a sequence (rows >= q_lens[b] * H) skips
// that sequence too; producer warp 0 writes those rows (0 / -inf).
struct PieceWalker {
  const Params* p;
  int cb, ck, be, ke;
  const int32_t* nblk;
  const int32_t* first_part;
  int part, row0;
  __device__ PieceWalker(const Params& prm, int part_, int row0_) : p(&prm), part(part_), row0(row0_) {
    const int32_t* m = prm.meta;
    cb = m[off_part_start() + 2 * part];
    ck = m[off_part_start() + 2 * part + 1];
    be = m[off_part_end() + 2 * part];
    ke = m[off_part_end() + 2 * part + 1];
    nblk = m + off_nblk();
    first_part = m + off_first_part(prm.B);
  }
  __device__ bool next(Piece& pc) {
    if (cb < 0) cb = p->B;  // malformed start: no pieces
    while (cb < p->B && (cb < be || (cb == be && ck < ke))) {
      const int nb = nblk[cb];
      const int hi = min((cb == be) ? ke : nb, nb);
      const int b = cb, lo = max(ck, 0);
      cb += 1;
      ck = 0;
      if (lo >= hi) continue;
      const int n = seq_len(*p, b);
      if (expected_blocks(*p, n) != nb) continue;
      const int ql = query_len(*p, b);
      if (ql < 0 || row0 >= ql * p->H) continue;
      pc.b = b;
      pc.k_lo = lo;
      pc.k_hi = hi;
      pc.split = part - first_part[b];
      pc.n = n;
      pc.qlen = ql;
      return true;
    }
    return false;
  }
};

__device__ __forceinline__ int num_tiles(const Piece& pc) {
  return (pc.k_hi - pc.k_lo + kBlocksPerTile - 1) / kBlocksPerTile;
}
__device__ __forceinline__ int blocks_in_tile(const Piece& pc, int t) {
  const int r = pc.k_hi - pc.k_lo - t * kBlocksPerTile;
  return r < kBlocksPerTile ? r : kBlocksPerTile;
}
// valid keys (< n) in block kb of tile t
__device__ __forceinline__ int rows_in_block(const Piece& pc, int t, int kb) {
  const int key0 = (pc.k_lo + t * kBlocksPerTile + kb) * kBlockSize;
  const int r = pc.n - key0;
  return r < kBlockSize ? r : kBlockSize;
}

__device__ __forceinline__ void set_status(const Params& p, int bits) {
  if (p.status) atomicOr(p.status, bits);
}

// Bounded wait that also gives up when another role of this CTA aborted.
__device__ __forceinline__ bool wait_bar(Ctrl* c, const Params& p, uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t deadline = globaltimer_ns() + p.timeout_ns;
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i) {
      if (mbar_try_wait(bar, parity)) return true;
    }
    if (c->abort) return false;
    if (globaltimer_ns() > deadline) {
      c->abort = 1;
      set_status(p, kErrTimeout);
      return false;
    }
  }
}

// Predicated forms: the whole warp executes the instruction and only lanes with
// `on` set issue it, so the issuing warp never diverges around the issue.
__device__ __forceinline__ void umma_2sm_if(bool on, uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                            uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %4, 0;\n\tsetp.ne.b32 q, %5, 0;\n\t"
      "@q tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"((uint32_t)on)
      : "memory");
}
__device__ __forceinline__ void commit_2sm_if(bool on, uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %1, 0;\n\t"
      "@q tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %2;\n\t}" ::"r"(bar),
      "r"((uint32_t)on), "h"((uint16_t)0x3)
      : "memory");
}
__device__ __forceinline__ void expect_tx_if(bool on, uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %2, 0;\n\t"
      "@q mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n\t}" ::"r"(bar),
      "r"(bytes), "r"((uint32_t)on)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_cg2_if(bool on, uint32_t dst, const void* tmap, uint32_t bar_cluster,
                                                   int c0, int c1, int c2) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %6, 0;\n\t"
      "@q cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];\n\t}" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"((uint32_t)on)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d_cg2_if(bool on, uint32_t dst, const void* tmap, uint32_t bar_cluster,
                                                   int c0, int c1) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %5, 0;\n\t"
      "@q cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];\n\t}" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"((uint32_t)on)
      : "memory");
}
__device__ __forceinline__ void tma_load_4d_cg2_if(bool on, uint32_t dst, const void* tmap, uint32_t bar_cluster,
                                                   int c0, int c1, int c2, int c3) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %7, 0;\n\t"
      "@q cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];\n\t}" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"((uint32_t)on)
      : "memory");
}
__device__ __forceinline__ void tma_store_3d(const void* tmap, uint32_t src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Named barrier that also ANDs a predicate over its threads: every thread gets the same
// answer, so a wait that ran out in one thread makes all of them leave together
// instead of leaving the others at the next barrier.
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
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// acc + lo(v) + hi(v) for a packed bf16 pair, with the mixed-precision f32 += bf16 add
__device__ __forceinline__ float add_bf16x2_to(float acc, uint32_t v) {
  float r;
  asm("{\n\t.reg .b16 lo, hi;\n\t.reg .f32 t;\n\tmov.b32 {lo, hi}, %1;\n\t"
      "add.rn.f32.bf16 t, lo, %2;\n\tadd.rn.f32.bf16 %0, hi, t;\n\t}"
      : "=f"(r)
      : "r"(v), "f"(acc));
  return r;
}

// ---- FP8 cache helpers --------------------------------------------------------
// TMA load into this CTA's own shared memory, completing on its own barrier.
__device__ __forceinline__ void tma_load_3d_if(bool on, uint32_t dst, const void* tmap, uint32_t bar, int c0, int c1,
                                               int c2) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %6, 0;\n\t"
      "@q cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];\n\t}" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"((uint32_t)on)
      : "memory");
}
template <int kRegs>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegs));
}
template <int kRegs>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegs));
}
// Two e4m3 codes (bytes b0, b1 of w, or b2, b3 with kHigh) -> two bf16 of the same
// values, exactly.  Per 16-bit lane a byte permute builds [sign of the code replicated |
// code]; shifting left by 4 and masking leaves sign at bit 15, the code's 4 exponent
// bits at 10..7 and its 3 mantissa bits at 6..4: a bf16 pattern whose exponent field is
// the e4m3 exponent field, i.e. the code's value times 2^(7 - 127) for normal codes and,
// through the bf16 subnormal range, for subnormal codes and zero too.  One bf16 multiply
// by 2^120 (exact: every result is a normal bf16) restores the value.
template <bool kHigh>
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t w) {
  uint32_t a;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(a) : "r"(w), "n"(kHigh ? 0xB3A2 : 0x9180));
  const uint32_t t = (a << 4) & 0x87F087F0u;
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(t), "r"(0x7B807B80u));  // 2^120 in both lanes
  return r;
}

__device__ __forceinline__ int clamp_block_id(const Params& p, int32_t id) {
  if (id < 0 || (int64_t)id >= p.num_blocks) {
    set_status(p, kErrBlockId);
    return 0;
  }
  return id;
}

// Rows that no piece of this row tile covers: no visible key (out 0, lse -inf), a row
// tile holding only padding tokens (0 / -inf), an invalid length or query count (NaN and
// MLA_DEVICE_ERR_SEQLEN) or a block count in the metadata that does not match the
// current length (NaN and MLA_DEVICE_ERR_METADATA).  Partition `part` takes the
// sequences b with b % P == part; the 32 lanes of one warp write this CTA's 64 rows
// [y0, y0 + 64) of the row tile that starts at row0.
__device__ __forceinline__ void write_orphan_rows(const Params& p, int part, int P, int row0, int y0, int lane) {
  const int32_t* nblk = p.meta + off_nblk();
  for (int b = part; b < p.B; b += P) {
    const int n = seq_len(p, b);
    const int want = expected_blocks(p, n);
    const int ql = query_len(p, b);
    const bool bad_len = want < 0 || ql < 0;
    const bool stale = !bad_len && nblk[b] != want;
    if (!bad_len && !stale && n > 0 && row0 < ql * p.H) continue;
    const bool bad = bad_len || stale;
    const float v = bad ? __int_as_float(0x7fc00000) : 0.0f;
    const uint32_t pv = pack_bf16x2(v, v);
    for (int i = lane; i < kRowsPerCta * (kDLatent / 8); i += 32) {  // 16-byte units
      const int row = y0 + i / (kDLatent / 8);
      if (row < p.M)
        reinterpret_cast<uint4*>(p.out + ((int64_t)b * p.M + row) * kDLatent)[i % (kDLatent / 8)] =
            make_uint4(pv, pv, pv, pv);
    }
    for (int r = lane; r < kRowsPerCta; r += 32)
      if (y0 + r < p.M) p.lse[(int64_t)b * p.M + y0 + r] = bad ? __int_as_float(0x7fc00000) : -INFINITY;
    if (bad && lane == 0) set_status(p, bad_len ? kErrSeqlen : kErrMetadata);
  }
}

// ===========================================================================
// the kernel
// ===========================================================================
template <bool kFp8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg<kFp8>::kThreads, 1)
    mla_decode_kernel(const __grid_constant__ Params p) {
  using C = Cfg<kFp8>;
  constexpr int kStages = C::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ Ctrl ctrl;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + kSmemQ, sP = sbase + kSmemP, sRing = sbase + kSmemRing;
  const uint32_t sStg = sbase + C::kSmemStg, sScale = sbase + C::kSmemScale;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int worker = blockIdx.x >> 1;

  // ---- setup (reads no input: it overlaps the previous kernel's tail when this one
  // is launched as a programmatic dependent) -----------------------------------
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&ctrl.full[s]), kFp8 ? 2 : 1);
      mbar_init(smem_u32(&ctrl.empty[s]), 1);
    }
    if constexpr (kFp8) {
      for (int s = 0; s < C::kStg; ++s) {
        mbar_init(smem_u32(&ctrl.stg_full[s]), 1);
        mbar_init(smem_u32(&ctrl.stg_empty[s]), 1);
      }
      for (int s = 0; s < 2; ++s) {
        mbar_init(smem_u32(&ctrl.sc_full[s]), 1);
        mbar_init(smem_u32(&ctrl.sc_empty[s]), 1);
      }
    }
    mbar_init(smem_u32(&ctrl.q_full), 1);
    mbar_init(smem_u32(&ctrl.q_empty), 1);
    mbar_init(smem_u32(&ctrl.s_full[0]), 1);
    mbar_init(smem_u32(&ctrl.s_full[1]), 1);
    mbar_init(smem_u32(&ctrl.p_full), 2);
    mbar_init(smem_u32(&ctrl.p_free), 1);
    mbar_init(smem_u32(&ctrl.o_free), 2);
    mbar_init(smem_u32(&ctrl.drain), 1);
    mbar_init(smem_u32(&ctrl.never), 1);
    ctrl.abort = 0;
    ctrl.peer_abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&ctrl.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&p.tm_kv);
    prefetch_tmap(&p.tm_kv2);
    prefetch_tmap(&p.tm_qn);
    prefetch_tmap(&p.tm_qp);
    prefetch_tmap(&p.tm_out);
    prefetch_tmap(&p.tm_part);
    if constexpr (kFp8) {
      prefetch_tmap(&p.tm_kpe);
      prefetch_tmap(&p.tm_scl);
    }
  }
  tc_fence_before();
  __syncthreads();
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  tc_fence_after();
  const uint32_t tmem = ctrl.tmem_base;
  // Inputs may come from the previous kernel in the stream (the schedule): wait for
  // it to complete, then let the next kernel (the LSE combine) start launching.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int P = p.meta[kHdrNumParts];
  int T = p.meta[kHdrNumTiles];
  if (p.meta[kHdrMagic] != kMetaMagic || p.meta[kHdrB] != p.B || p.meta[kHdrSq] != p.s_q ||
      p.meta[kHdrH] != p.H || P * T * 2 != (int)gridDim.x || p.meta[kHdrTokens] != p.tok_rep ||
      (p.tok_rep != 0 && p.meta[kHdrTokCausal] != p.tok_causal)) {
    if (tid == 0 && blockIdx.x == 0) set_status(p, kErrMetadata);
    T = 0;  // every role skips; the CTA still joins the cluster barriers below
  }
  const int tile = worker / P;
  const int part = worker % P;
  const int tile_row0 = tile * kRowsPerTile;

  if (tile < T) {
    // =======================================================================
    // producers: warps 0, 2, 3 own ring stages k % 3 == 0, 1, 2 (one issuing warp
    // sustains only about half the L2 -> SM bandwidth a CTA needs; several warps
    // issuing alternate stages of the same ring lift that limit).  Warp 0 also loads
    // each piece's Q.
    // =======================================================================
    if (warp == 0 || warp == 2 || warp == 3) {
      if constexpr (kFp8) regs_dec<kRegsIssue>();
      const int pi = (warp == 0) ? 0 : warp - 1;
      int32_t* idwin = ctrl.block_ids[pi];
      PieceWalker walk(p, part, tile_row0);
      uint32_t it = 0;
      bool ok = true;
      auto mine = [&]() { return (int)(it % kNumProducers) == pi; };
      // acquire the slot of stage `it` (every lane waits, the warp stays converged): a
      // bf16 ring slot freed by the MMAs, or (FP8 cache) a raw stage freed by the
      // converters
      auto acquire = [&](uint32_t& slot) -> bool {
        constexpr int kSlots = kFp8 ? C::kStg : kStages;
        slot = it % kSlots;
        const uint32_t use = it / kSlots;
        const uint32_t eb = kFp8 ? smem_u32(&ctrl.stg_empty[slot]) : smem_u32(&ctrl.empty[slot]);
        if (use > 0 && !wait_bar(&ctrl, p, eb, (use - 1) & 1)) return false;
        return true;
      };
      uint32_t ntile = 0;  // tiles issued so far (FP8: selects the scale buffer)
      // Physical block ids of the current piece, fetched 32 at a time (one coalesced
      // load per lane) one chunk ahead of use into this warp's 128-entry window, from
      // window offset `cur_base` on; invalid ids are clamped to block 0 here (the
      // epilogue turns that piece's rows into NaN).  The previous piece's ids stay in
      // the window until its last PV stages have been issued.
      Piece cur{};
      int cur_base = 0, id_pending = 0, id_chunks = 0;
      const int32_t* bt = nullptr;
      auto fetch_id = [&](int i) -> int {
        return (i < cur.k_hi - cur.k_lo) ? clamp_block_id(p, bt[cur.k_lo + i]) : 0;
      };
      auto ensure_ids = [&](int last) {  // make relative blocks <= last of `cur` readable
        while (last >= 32 * id_chunks) {
          idwin[(cur_base + 32 * id_chunks + lane) % kIdRing] = id_pending;
          ++id_chunks;
          id_pending = fetch_id(32 * id_chunks + lane);
          __syncwarp();
        }
      };
      // FP8 cache, QK of tile t: this CTA's (up to) two blocks as 8 slabs of 64 code
      // columns (4 KB per block), then its blocks' scaled k_pe (8 KB each, one raw stage
      // per block, present or not); with the first slab, the scales of all the tile's
      // blocks for the softmax.
      auto issue_qk_fp8 = [&](int t) {
        const int nb = blocks_in_tile(cur, t);
        const int own0 = 2 * (int)rank;
        ensure_ids(t * kBlocksPerTile + nb - 1);
        const int own = min(max(nb - own0, 0), 2);
        const int my_id = idwin[(cur_base + t * kBlocksPerTile + own0 + (lane & 1)) % kIdRing];
        for (int st = 0; st < kStgPerQk && ok; ++st) {  // 8 code slabs, then 2 k_pe blocks
          if (!mine()) {
            ++it;
            continue;
          }
          if (st == 0) {  // the tile's scales, into buffer ntile & 1
            const uint32_t sb = ntile & 1, use = ntile >> 1;
            if (use > 0)
              ok = __shfl_sync(0xffffffffu, wait_bar(&ctrl, p, smem_u32(&ctrl.sc_empty[sb]), (use - 1) & 1), 0);
            if (!ok) break;
            const uint32_t fb = smem_u32(&ctrl.sc_full[sb]);
            expect_tx_if(lane == 0, fb, nb * kScaleBlockBytes);
            const int id = idwin[(cur_base + t * kBlocksPerTile + (lane & 3)) % kIdRing];
            tma_load_3d_if(lane < nb, sScale + sb * kScaleBufBytes + lane * kScaleBlockBytes, &p.tm_scl, fb,
                           kOffScale8 / 4, 0, id);
          }
          uint32_t slot;
          ok = __shfl_sync(0xffffffffu, acquire(slot), 0);
          if (!ok) break;
          const uint32_t fb = smem_u32(&ctrl.stg_full[slot]);
          if (st < 8) {
            expect_tx_if(lane == 0, fb, own * kSlabBlockBytes);
            tma_load_3d_if(lane < own, sStg + slot * kStgBytes + lane * kSlabBlockBytes, &p.tm_kv, fb, 64 * st, 0,
                           my_id);
          } else {
            const int kp = st - 8;
            const int id = idwin[(cur_base + t * kBlocksPerTile + own0 + kp) % kIdRing];
            expect_tx_if(lane == 0, fb, kp < own ? kStgBytes : 0);
            tma_load_3d_if(lane == 0 && kp < own, sStg + slot * kStgBytes, &p.tm_kpe, fb, kDLatent / 2, 0, id);
          }
          ++it;
        }
        ++ntile;
      };
      auto issue_qk = [&](int t) {
        const int nb = blocks_in_tile(cur, t);
        const int own0 = 2 * (int)rank;
        ensure_ids(t * kBlocksPerTile + nb - 1);
        // this lane's box (lanes 0 and 1 each issue one of the CTA's two blocks)
        const int own = min(max(nb - own0, 0), 2);
        int my_id = idwin[(cur_base + t * kBlocksPerTile + own0 + (lane & 1)) % kIdRing];
        // Every stage must carry bytes from both CTAs: the leader's full barrier then
        // cannot complete before the peer has issued the stage, which keeps the peer
        // producers within one ring cycle of the MMAs (otherwise its empty-barrier
        // parity could alias).  A peer without keys in this tile loads a copy of the
        // tile's first block; those S columns are masked.
        const int nbox = own > 0 ? own : 1;
        if (own == 0) my_id = idwin[(cur_base + t * kBlocksPerTile) % kIdRing];
        const int peer_boxes = nb > 2 ? nb - 2 : 1;
        const int lead_boxes = nb < 2 ? nb : 2;
        for (int c = 0; c < kQChunks && ok; ++c) {
          if (!mine()) {
            ++it;
            continue;
          }
          uint32_t slot;
          ok = __shfl_sync(0xffffffffu, acquire(slot), 0);
          if (!ok) break;
          // Only the leader arrives (posting both CTAs' bytes); the peer's TMA
          // completes its bytes on the leader's barrier.
          const uint32_t fb = smem_u32(&ctrl.full[slot]);
          expect_tx_if(lane == 0 && leader, fb, kChunkBytes * (lead_boxes + peer_boxes));
          tma_load_3d_cg2_if(lane < nbox, sRing + slot * kStageBytes + (lane & 1) * kChunkBytes, &p.tm_kv,
                             mapa_shared(fb, 0), 64 * c, 0, my_id);
          ++it;
        }
      };
      // V stages of tile t of piece pc (ids at window offset base).  The sequence's
      // last block, with rv < 64 valid keys, is loaded from row rv - 64: the box's
      // first 64 - rv rows fall before the block and are zero-filled by the TMA, the
      // keys land in rows [64 - rv, 64).  No row past the sequence end is read, so
      // the stage needs no zeroing; P of that block is stored shifted to match.
      auto issue_pv = [&](const Piece& pc, int base, int t) {
        const int nb = blocks_in_tile(pc, t);
        for (int h = 0; h < 2 && ok; ++h) {
          for (int kb = 0; kb < nb && ok; ++kb) {
            if (!mine()) {
              ++it;
              continue;
            }
            const int id = idwin[(base + t * kBlocksPerTile + kb) % kIdRing];
            const int rv = rows_in_block(pc, t, kb);
            uint32_t slot;
            ok = __shfl_sync(0xffffffffu, acquire(slot), 0);
            if (!ok) break;
            const int d0 = 256 * h + 128 * (int)rank;
            if constexpr (kFp8) {  // one block's 128-column slab of codes (8 KB)
              const uint32_t fb = smem_u32(&ctrl.stg_full[slot]);
              expect_tx_if(lane == 0, fb, kStgBytes);
              tma_load_3d_if(lane == 0, sStg + slot * kStgBytes, &p.tm_kv2, fb, d0, rv - kBlockSize, id);
            } else {
              const uint32_t fb = smem_u32(&ctrl.full[slot]);
              expect_tx_if(lane == 0 && leader, fb, 2 * kStageBytes);
              tma_load_4d_cg2_if(lane == 0, sRing + slot * kStageBytes, &p.tm_kv2, mapa_shared(fb, 0), 0,
                                 rv - kBlockSize, d0 / 64, id);
            }
            ++it;
          }
        }
      };
      // Q of a piece: the whole warp waits until the previous piece's last QK has
      // completed (its Q buffer is free), then lanes 0..8 each issue one 64-column box.
      const uint32_t q_full_l = mapa_shared(smem_u32(&ctrl.q_full), 0);
      auto load_q = [&](const Piece& pc, int piece_idx) {
        if (piece_idx > 0)
          ok = __shfl_sync(0xffffffffu, wait_bar(&ctrl, p, smem_u32(&ctrl.q_empty), (piece_idx - 1) & 1), 0);
        if (!ok) return;
        const int row_base = pc.b * p.M + tile_row0 + kRowsPerCta * (int)rank;
        expect_tx_if(lane == 0 && leader, smem_u32(&ctrl.q_full), 2 * kQBytes);
        __syncwarp();
        const int c = lane < kQChunks ? lane : 0;
        tma_load_2d_cg2_if(lane < kQChunks, sQ + c * kChunkBytes, c < 8 ? (const void*)&p.tm_qn : (const void*)&p.tm_qp,
                           q_full_l, c < 8 ? 64 * c : 0, row_base);
      };
      // One ring order for the whole partition: the tiles of all its pieces form one
      // sequence, and each tile's QK stages are followed by the PV stages of the tile
      // before it, across piece boundaries too; the last PV ends the ring.  The next
      // piece is looked up one piece ahead and its first 32 block ids are loaded
      // during the current piece's last tile.
      Piece nxt{}, prv{};
      int prv_base = 0, prv_t = -1, npieces = 0;
      bool have = walk.next(cur);
      bool have_nxt = have && walk.next(nxt);
      if (have) {
        bt = p.block_table + table_row(p, cur.b) * p.max_blocks;
        id_pending = fetch_id(lane);
      }
      while (ok && have) {
        id_chunks = 0;
        const int nt = num_tiles(cur);
        int id_next = 0;
        for (int t = 0; t < nt && ok; ++t) {
          if (t == nt - 1 && have_nxt) {
            const int32_t* btn = p.block_table + table_row(p, nxt.b) * p.max_blocks;
            id_next = (lane < nxt.k_hi - nxt.k_lo) ? clamp_block_id(p, btn[nxt.k_lo + lane]) : 0;
          }
          if (t == 0 && pi == 0) load_q(cur, npieces);
          if (ok) {
            if constexpr (kFp8)
              issue_qk_fp8(t);
            else
              issue_qk(t);
          }
          if (ok && prv_t >= 0) issue_pv(prv, prv_base, prv_t);
          prv = cur;
          prv_base = cur_base;
          prv_t = t;
        }
        cur_base = (cur_base + 32 * id_chunks) % kIdRing;
        ++npieces;
        have = have_nxt;
        if (have) {
          cur = nxt;
          bt = p.block_table + table_row(p, cur.b) * p.max_blocks;
          id_pending = id_next;
          have_nxt = walk.next(nxt);
        }
      }
      if (ok && prv_t >= 0) issue_pv(prv, prv_base, prv_t);
      // With its loads issued, producer warp 0 writes the rows that no partition
      // covers while the last tiles are still being computed.
      if (pi == 0) write_orphan_rows(p, part, P, tile_row0, tile_row0 + kRowsPerCta * (int)rank, lane);
    }
    // =======================================================================
    // MMA issuer (leader CTA only)
    // =======================================================================
    else if (warp == kMmaWarp && leader) {
      if constexpr (kFp8) regs_dec<kRegsIssue>();
      // Every lane waits and the elected lane's predicate issues.  No full-warp
      // collective sits inside the loop, so lanes that leave it at different points
      // after a wait ran out cannot deadlock the warp; they meet again at teardown.
      PieceWalker walk(p, part, tile_row0);
      uint32_t slot = 0, phase = 0, qk_count = 0, pv_count = 0;
      int npieces = 0;
      bool ok = true;
      const bool elected = elect_one();
      // Shared-memory descriptors: the 14-bit start field holds address >> 4, so the
      // operand of chunk c / slot s / 16-element K step k is the base plus
      // c * (8192 >> 4) / s * (16384 >> 4) / k * (32 >> 4) (K-major) or k * (2048 >> 4)
      // (V, MN-major: 16 keys = 16 rows of 128 bytes).
      const uint64_t dq0 = make_smem_desc(sQ, 16, 1024, kSwizzle128B);
      const uint64_t dp0 = make_smem_desc(sP, 16, 1024, kSwizzle128B);
      const uint64_t dk0 = make_smem_desc(sRing, 16, 1024, kSwizzle128B);
      const uint64_t dv0 = make_smem_desc(sRing, 8192, 1024, kSwizzle128B);
      constexpr uint64_t kChunkD = kChunkBytes >> 4, kStageD = kStageBytes >> 4;
      auto next_stage = [&]() {
        if (++slot == kStages) {
          slot = 0;
          phase ^= 1;
        }
      };
      auto mma_qk = [&](int nt, int t) {
        const uint32_t buf = qk_count & 1;
        const uint32_t d = tmem + kTmemS0 + 128 * buf;
        for (int c = 0; c < kQChunks && ok; ++c) {
          ok = wait_bar(&ctrl, p, smem_u32(&ctrl.full[slot]), phase);
          if (!ok) break;
          const uint64_t a0 = dq0 + c * kChunkD, b0 = dk0 + slot * kStageD;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) umma_2sm_if(elected, d, a0 + 2 * ks, b0 + 2 * ks, kIdescQK, (c | ks) != 0);
          commit_2sm_if(elected, smem_u32(&ctrl.empty[slot]));
          next_stage();
        }
        if (ok) {
          commit_2sm_if(elected, smem_u32(&ctrl.s_full[buf]));
          if (t == nt - 1) commit_2sm_if(elected, smem_u32(&ctrl.q_empty));
        }
        ++qk_count;
      };
      // PV of tile t of piece pc, the piece_idx-th piece of this partition
      auto mma_pv = [&](const Piece& pc, int piece_idx, int t) {
        if (!ok) return;
        ok = wait_bar(&ctrl, p, smem_u32(&ctrl.p_full), pv_count & 1);
        if (ok && t == 0 && piece_idx > 0) ok = wait_bar(&ctrl, p, smem_u32(&ctrl.o_free), (piece_idx - 1) & 1);
        if (!ok) return;
        tc_fence_after();
        const int nb = blocks_in_tile(pc, t);
        for (int h = 0; h < 2 && ok; ++h) {
          for (int kb = 0; kb < nb && ok; ++kb) {
            ok = wait_bar(&ctrl, p, smem_u32(&ctrl.full[slot]), phase);
            if (!ok) break;
            // the sequence's last block sits in rows [64 - rv, 64): skip whole zero steps
            const int rv = rows_in_block(pc, t, kb);
            const int ks0 = (kBlockSize - rv) >> 4;
            const bool first = (t == 0 && kb == 0);
            const uint64_t a0 = dp0 + kb * kChunkD, b0 = dv0 + slot * kStageD;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              umma_2sm_if(elected && ks >= ks0, tmem + kTmemO + 128 * h, a0 + 2 * ks, b0 + 128 * ks, kIdescPV,
                          !(first && ks == ks0));
            commit_2sm_if(elected, smem_u32(&ctrl.empty[slot]));
            next_stage();
          }
        }
        if (ok) commit_2sm_if(elected, smem_u32(&ctrl.p_free));
        ++pv_count;
      };
      // same ring order as the producers: QK of each tile, then PV of the tile before
      Piece cur, prv{};
      int prv_t = -1, prv_idx = 0;
      if (p.inject_stall) ok = wait_bar(&ctrl, p, smem_u32(&ctrl.never), 0);
      while (ok && walk.next(cur)) {
        ok = wait_bar(&ctrl, p, smem_u32(&ctrl.q_full), npieces & 1);
        const int nt = num_tiles(cur);
        for (int t = 0; t < nt && ok; ++t) {
          mma_qk(nt, t);
          if (prv_t >= 0) mma_pv(prv, prv_idx, prv_t);
          prv = cur;
          prv_t = t;
          prv_idx = npieces;
        }
        ++npieces;
      }
      if (prv_t >= 0) mma_pv(prv, prv_idx, prv_t);
    }
    // =======================================================================
    // softmax / correction / epilogue
    // =======================================================================
    else if (warp >= kSoftmaxWarp0 && warp < kSoftmaxWarp0 + 8) {
      if constexpr (kFp8) regs_inc<kRegsSoftmax>();
      const int st = tid - kSoftmaxWarp0 * 32;  // 0..255
      const int g = st >> 7;                   // column group: keys 64g.. of each half; O half g
      const int L = st & 127;                  // TMEM lane
      const int quad = (warp & 3);             // lane quadrant this warp may access
      const int m = L & 63;                    // row within the CTA
      const int hk = L >> 6;                   // key half (0: keys 0..127, 1: 128..255)
      const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
      const int grow = tile_row0 + kRowsPerCta * (int)rank + m;  // row within the sequence
      const bool row_valid = grow < p.M;
      const int token = row_valid ? grow / p.H : 0;
      const int y0 = tile_row0 + kRowsPerCta * (int)rank;
      const uint32_t p_full_l = mapa_shared(smem_u32(&ctrl.p_full), 0);
      const uint32_t o_free_l = mapa_shared(smem_u32(&ctrl.o_free), 0);
      PieceWalker walk(p, part, tile_row0);
      Piece pc;
      uint32_t qk_count = 0, pv_count = 0;
      // ok: this thread's waits all completed.  go: the same for all 256 threads,
      // refreshed only by named barriers that AND ok, so every loop decision is
      // uniform and no thread leaves the others waiting at a barrier.
      bool ok = true, go = true;
      // Epilogue of a finished piece: it runs once the piece's last PV has completed,
      // inside the next piece's first tile (after that tile's weights are computed),
      // or after the last tile.  out = O / l (bf16) or the normalised fp32 partial,
      // written through TMA stores staged in the P buffer, which is free between a
      // PV and the next P; then O's TMEM is handed back to the MMAs (o_free).  After
      // the partition's last tile (drain) the Q buffer and the ring are idle as well:
      // each round then stages into its own 32 KB from the start of shared memory, and
      // the stores of all rounds go out together after one barrier.
      bool pend = false, pend_direct = true;
      int pend_b = 0, pend_slot = 0;
      float pend_sc = 0.f, pend_lse = 0.f;
      auto epilogue = [&](bool drain) {
        const uint32_t to = tmem + kTmemO + 128 * g + lane_off;
        // per round every thread writes 128 bytes of its row (64 bf16 or 32 fp32 columns)
        // into box 2g + hk, laid out [64 rows][128 B] with the 128-byte swizzle, and one
        // thread stores the four boxes; rows past M are clipped by the tensor map
        const int rounds = pend_direct ? 2 : 4;
        auto stage = [&](int r) -> uint32_t { return drain ? sQ + r * kEpiRoundBytes : sP; };
        auto store_round = [&](int r) {
#pragma unroll
          for (int bx = 0; bx < 4; ++bx) {
            const int gg = bx >> 1, hh = bx & 1;
            if (pend_direct)
              tma_store_3d(&p.tm_out, stage(r) + bx * kChunkBytes, 256 * gg + 128 * hh + 64 * r, y0, pend_b);
            else
              tma_store_3d(&p.tm_part, stage(r) + bx * kChunkBytes, 256 * gg + 128 * hh + 32 * r, y0, pend_slot);
          }
        };
#pragma unroll 1
        for (int r = 0; r < rounds; ++r) {
          const uint32_t srow = stage(r) + (2 * g + hk) * kChunkBytes + m * 128;
          uint32_t w[32];
          if (pend_direct) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              uint32_t o[32];
              tmem_ld32(to + 64 * r + 32 * hf, o);
              tmem_wait_ld();
#pragma unroll
              for (int k = 0; k < 16; ++k)
                w[16 * hf + k] =
                    pack_bf16x2(__uint_as_float(o[2 * k]) * pend_sc, __uint_as_float(o[2 * k + 1]) * pend_sc);
            }
          } else {
            tmem_ld32(to + 32 * r, w);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) w[k] = __float_as_uint(__uint_as_float(w[k]) * pend_sc);
          }
          if (r > 0 && !drain) named_bar_sync(kBarSoftmax, kNumSoftmaxThreads);  // previous round's boxes were read
#pragma unroll
          for (int q = 0; q < 8; ++q)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(srow + ((q ^ (m & 7)) << 4)),
                         "r"(w[4 * q]), "r"(w[4 * q + 1]), "r"(w[4 * q + 2]), "r"(w[4 * q + 3])
                         : "memory");
          fence_proxy_async_smem();
          if (drain) continue;
          if (r == 0) {
            go = named_bar_and(kBarSoftmax, kNumSoftmaxThreads, ok);
            if (!go) return;
          } else {
            named_bar_sync(kBarSoftmax, kNumSoftmaxThreads);
          }
          if (st == 0 && y0 < p.M) {  // a CTA whose 64 rows all lie past M stores nothing
            store_round(r);
            bulk_commit();
            bulk_wait_read_all();
          }
        }
        if (drain) {
          go = named_bar_and(kBarSoftmax, kNumSoftmaxThreads, ok);
          if (!go) return;
          if (st == 0 && y0 < p.M) {  // completion is awaited at teardown
            for (int r = 0; r < rounds; ++r) store_round(r);
            bulk_commit();
          }
        }
        if (row_valid && hk == 0 && g == 0) {
          if (pend_direct)
            p.lse[(int64_t)pend_b * p.M + grow] = pend_lse;
          else
            p.part_lse[(int64_t)pend_slot * p.M + grow] = pend_lse;
        }
        // every O read and the staging reads of the last round are done
        tc_fence_before();
        named_bar_sync(kBarSoftmax, kNumSoftmaxThreads);
        if (st == 0) {
          if (leader)
            mbar_arrive(smem_u32(&ctrl.o_free));
          else
            mbar_arrive_remote(o_free_l);
        }
        pend = false;
      };
      while (go && walk.next(pc)) {
        const int nt = num_tiles(pc);
        const int piece_end = min(pc.n, pc.k_hi * kBlockSize);
        int lim = p.causal ? (pc.n - pc.qlen + token) : (pc.n - 1);
        if (token >= pc.qlen) lim = -1;  // padding token: no visible key (out 0, lse -inf)
        lim = min(lim, piece_end - 1);
        if (!row_valid) lim = -1;
        // l_part: sum of the bf16 weights that enter the PV MMA (output normaliser, so
        // the weights sum to one exactly); l32_part: fp32 weights (the lse).
        float m_used = -INFINITY, l_part = 0.f, l32_part = 0.f;
        // Block-id validity and split layout of the piece (loads issued now, consumed
        // at the piece's end).
        const int nsplit = p.meta[off_num_splits(p.B) + pc.b];
        const int split_base = p.meta[off_split_prefix(p.B) + pc.b];
        int bad_ids = 0;
        {
          const int32_t* bt = p.block_table + table_row(p, pc.b) * p.max_blocks;
          for (int k = pc.k_lo + st; k < pc.k_hi; k += kNumSoftmaxThreads) {
            const int32_t id = bt[k];
            bad_ids |= (id < 0 || (int64_t)id >= p.num_blocks);
          }
        }
        for (int t = 0; t < nt && go; ++t) {
          const uint32_t buf = qk_count & 1;
          // A wait that runs out does not leave the loop here: the thread carries on to
          // the next AND barrier, which makes all 256 threads leave together.
          ok = wait_bar(&ctrl, p, smem_u32(&ctrl.s_full[buf]), (qk_count >> 1) & 1) && ok;
          // FP8 cache: the tile's per-key scales (key 64 j + c of the tile at float
          // 256 j + 4 c of its buffer); this thread's 64 keys are block 2 hk + g
          const float* scb = reinterpret_cast<const float*>(smem + C::kSmemScale + (qk_count & 1) * kScaleBufBytes +
                                                            (2 * hk + g) * kScaleBlockBytes);
          if constexpr (kFp8)
            ok = wait_bar(&ctrl, p, smem_u32(&ctrl.sc_full[qk_count & 1]), (qk_count >> 1) & 1) && ok;
          tc_fence_after();
          uint32_t sr[64];
          {
            uint32_t (&a)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
            uint32_t (&b)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
            const uint32_t ta = tmem + kTmemS0 + 128 * buf + lane_off + 64 * g;
            tmem_ld32(ta, a);
            tmem_ld32(ta + 32, b);
            tmem_wait_ld();
          }
          const int key0 = (pc.k_lo + t * kBlocksPerTile) * kBlockSize + 128 * hk + 64 * g;
          int cnt = lim - key0 + 1;
          cnt = cnt < 0 ? 0 : (cnt > 64 ? 64 : cnt);
          // Tiles with every key visible (all but a sequence's last tile and causal
          // edges) take an unmasked path; the choice is warp-uniform.
          const bool full = __all_sync(0xffffffffu, cnt == kBlockSize);
          // Row maximum of the raw scores (the scale is positive, so it keeps their
          // order), over four independent chains.
          float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
          const float sl2 = p.scale_log2;
          if constexpr (kFp8) {
            // scores in log2 units, x = S' * scale_key * scale_log2, kept in sr
#pragma unroll
            for (int c = 0; c < 64; ++c) {
              const float x = __uint_as_float(sr[c]) * (scb[4 * c] * sl2);
              sr[c] = __float_as_uint(x);
            }
          }
          if (full) {
#pragma unroll
            for (int c = 0; c < 64; c += 4) {
              mx0 = fmaxf(mx0, __uint_as_float(sr[c]));
              mx1 = fmaxf(mx1, __uint_as_float(sr[c + 1]));
              mx2 = fmaxf(mx2, __uint_as_float(sr[c + 2]));
              mx3 = fmaxf(mx3, __uint_as_float(sr[c + 3]));
            }
          } else {
#pragma unroll
            for (int c = 0; c < 64; c += 4) {
              if (c < cnt) mx0 = fmaxf(mx0, __uint_as_float(sr[c]));
              if (c + 1 < cnt) mx1 = fmaxf(mx1, __uint_as_float(sr[c + 1]));
              if (c + 2 < cnt) mx2 = fmaxf(mx2, __uint_as_float(sr[c + 2]));
              if (c + 3 < cnt) mx3 = fmaxf(mx3, __uint_as_float(sr[c + 3]));
            }
          }
          const float lmax = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * (kFp8 ? 1.0f : sl2);
          ctrl.red_max[qk_count & 1][2 * hk + g][m] = lmax;
          go = named_bar_and(kBarSoftmax, kNumSoftmaxThreads, ok);
          if (!go) break;
          float rmax = ctrl.red_max[qk_count & 1][0][m];
          rmax = fmaxf(rmax, ctrl.red_max[qk_count & 1][1][m]);
          rmax = fmaxf(rmax, ctrl.red_max[qk_count & 1][2][m]);
          rmax = fmaxf(rmax, ctrl.red_max[qk_count & 1][3][m]);
          const float m_new = fmaxf(m_used, rmax);
          const bool rescale = m_new > m_used + kRescaleThreshold;
          float alpha = 1.f;
          if (rescale) {
            alpha = (m_used == -INFINITY) ? 0.f : fast_exp2(m_used - m_new);
            m_used = m_new;
            l_part *= alpha;
            l32_part *= alpha;
          }
          const float nref = (m_used == -INFINITY) ? 0.f : -m_used;
          uint32_t pk[32];
          // bf16 cache: weights 2^(s * scale_log2 - m); sums of the bf16-rounded weights
          // (output normaliser) and of the fp32 weights (lse), two chains each
          float ls0 = 0.f, ls1 = 0.f, lf0 = 0.f, lf1 = 0.f;
          if constexpr (kFp8) {
            // weights e = 2^(x - m) (their fp32 sums normalise the output and give the
            // lse); the PV operand is P' = bf16(e * scale_key), since V = scale_key * codes
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
              const bool v0 = full || c < cnt, v1 = full || c + 1 < cnt;
              const float e0 = v0 ? fast_exp2(__uint_as_float(sr[c]) + nref) : 0.f;
              const float e1 = v1 ? fast_exp2(__uint_as_float(sr[c + 1]) + nref) : 0.f;
              const float p0 = v0 ? e0 * scb[4 * c] : 0.f;
              const float p1 = v1 ? e1 * scb[4 * c + 4] : 0.f;
              pk[c >> 1] = pack_bf16x2(p0, p1);
              if (c & 2)
                lf1 += e0 + e1;
              else
                lf0 += e0 + e1;
            }
            ls0 = lf0;
            ls1 = lf1;
          } else {
            if (full) {
#pragma unroll
              for (int c = 0; c < 64; c += 4) {
                const float e0 = fast_exp2(fmaf(__uint_as_float(sr[c]), sl2, nref));
                const float e1 = fast_exp2(fmaf(__uint_as_float(sr[c + 1]), sl2, nref));
                const float e2 = fast_exp2(fmaf(__uint_as_float(sr[c + 2]), sl2, nref));
                const float e3 = fast_exp2(fmaf(__uint_as_float(sr[c + 3]), sl2, nref));
                const uint32_t v0 = pack_bf16x2(e0, e1), v1 = pack_bf16x2(e2, e3);
                pk[c >> 1] = v0;
                pk[(c >> 1) + 1] = v1;
                ls0 = add_bf16x2_to(ls0, v0);
                ls1 = add_bf16x2_to(ls1, v1);
                lf0 += e0 + e1;
                lf1 += e2 + e3;
              }
            } else {
#pragma unroll
              for (int c = 0; c < 64; c += 4) {
                const float e0 = (c < cnt) ? fast_exp2(fmaf(__uint_as_float(sr[c]), sl2, nref)) : 0.f;
                const float e1 = (c + 1 < cnt) ? fast_exp2(fmaf(__uint_as_float(sr[c + 1]), sl2, nref)) : 0.f;
                const float e2 = (c + 2 < cnt) ? fast_exp2(fmaf(__uint_as_float(sr[c + 2]), sl2, nref)) : 0.f;
                const float e3 = (c + 3 < cnt) ? fast_exp2(fmaf(__uint_as_float(sr[c + 3]), sl2, nref)) : 0.f;
                const uint32_t v0 = pack_bf16x2(e0, e1), v1 = pack_bf16x2(e2, e3);
                pk[c >> 1] = v0;
                pk[(c >> 1) + 1] = v1;
                ls0 = add_bf16x2_to(ls0, v0);
                ls1 = add_bf16x2_to(ls1, v1);
                lf0 += e0 + e1;
                lf1 += e2 + e3;
              }
            }
          }
          l_part += ls0 + ls1;
          l32_part += lf0 + lf1;
          // PV of the previous tile (possibly the previous piece's last) must be done
          // before P is overwritten, O is rescaled or the previous piece's O is read.
          if (qk_count >= 1) {
            ok = wait_bar(&ctrl, p, smem_u32(&ctrl.p_free), pv_count & 1) && ok;
            ++pv_count;
            tc_fence_after();
            if (t == 0) {
              if (pend) {
                epilogue(false);
                if (!go) break;
              }
            } else if (__any_sync(0xffffffffu, rescale)) {
              const uint32_t to = tmem + kTmemO + 128 * g + lane_off;
#pragma unroll 1
              for (int c = 0; c < 128; c += 32) {
                uint32_t o[32];
                tmem_ld32(to + c, o);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                asm volatile(
                    "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
                    "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
                    "%29, %30, %31, %32};" ::"r"(to + c),
                    "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3]), "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7]),
                    "r"(o[8]), "r"(o[9]), "r"(o[10]), "r"(o[11]), "r"(o[12]), "r"(o[13]), "r"(o[14]),
                    "r"(o[15]), "r"(o[16]), "r"(o[17]), "r"(o[18]), "r"(o[19]), "r"(o[20]), "r"(o[21]),
                    "r"(o[22]), "r"(o[23]), "r"(o[24]), "r"(o[25]), "r"(o[26]), "r"(o[27]), "r"(o[28]),
                    "r"(o[29]), "r"(o[30]), "r"(o[31])
                    : "memory");
              }
              tmem_wait_st();
            }
          }
          // The sequence's last block (rv < 64 keys) was loaded into rows [64 - rv, 64)
          // of its V stage: shift its P row right by 64 - rv keys to match (the keys
          // shifted out are >= rv, whose weights are 0; zeros are shifted in).
          {
            const int rv = pc.n - key0;
            if (rv > 0 && rv < kBlockSize) {  // warp-uniform: the warp's rows share the block
              const int sh = kBlockSize - rv;
              if (sh & 1) {
#pragma unroll
                for (int w = 31; w >= 1; --w) pk[w] = __byte_perm(pk[w - 1], pk[w], 0x5432);
                pk[0] <<= 16;
              }
              const int ws = sh >> 1;
#pragma unroll
              for (int bit = 0; bit < 5; ++bit) {
                if ((ws >> bit) & 1) {
#pragma unroll
                  for (int w = 31; w >= 0; --w) pk[w] = (w >= (1 << bit)) ? pk[w - (1 << bit)] : 0u;
                }
              }
            }
          }
          // P -> shared memory: chunk (2 hk + g) holds keys 64 (2hk+g) .. of all 64 rows,
          // K-major 128-byte swizzle (16-byte granule j of row m at j ^ (m & 7)).
          {
            const uint32_t prow = sP + (2 * hk + g) * kChunkBytes + m * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const uint32_t a = prow + ((j ^ (m & 7)) << 4);
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(pk[4 * j]), "r"(pk[4 * j + 1]),
                           "r"(pk[4 * j + 2]), "r"(pk[4 * j + 3])
                           : "memory");
            }
          }
          fence_proxy_async_smem();
          tc_fence_before();
          named_bar_sync(kBarSoftmax, kNumSoftmaxThreads);
          if (st == 0) {
            if (leader)
              mbar_arrive(smem_u32(&ctrl.p_full));
            else
              mbar_arrive_remote(p_full_l);
            if constexpr (kFp8) mbar_arrive(smem_u32(&ctrl.sc_empty[qk_count & 1]));  // scales read
          }
          ++qk_count;
        }
        if (!go) break;
        // ---- end of the piece: row sums and the block-id verdict are final; reduce
        // them while its last PV is still running, and keep what its epilogue needs
        ctrl.red_sum[2 * hk + g][m] = l_part;
        ctrl.red_sum32[2 * hk + g][m] = l32_part;
        if (st == 0) ctrl.bad_piece = 0;
        named_bar_sync(kBarSoftmax, kNumSoftmaxThreads);
        if (bad_ids) ctrl.bad_piece = 1;
        const float l_row = ctrl.red_sum[0][m] + ctrl.red_sum[1][m] + ctrl.red_sum[2][m] + ctrl.red_sum[3][m];
        const float l32_row =
            ctrl.red_sum32[0][m] + ctrl.red_sum32[1][m] + ctrl.red_sum32[2][m] + ctrl.red_sum32[3][m];
        named_bar_sync(kBarSoftmax, kNumSoftmaxThreads);
        const bool bad = ctrl.bad_piece != 0;
        const float nanf_ = __int_as_float(0x7fc00000);
        // a bad piece's rows become NaN: scaling by NaN turns every value into NaN
        pend_sc = bad ? nanf_ : ((l_row > 0.f) ? 1.f / l_row : 0.f);
        pend_lse = bad ? nanf_ : ((l32_row > 0.f) ? (m_used + __log2f(l32_row)) * 0.69314718055994531f : -INFINITY);
        pend_direct = (nsplit == 1);
        pend_b = pc.b;
        pend_slot = split_base + pc.split;
        pend = true;
      }
      // the last piece's epilogue, after its last PV (the AND makes the decision uniform)
      go = named_bar_and(kBarSoftmax, kNumSoftmaxThreads, ok && go);
      if (go && pend) {
        ok = wait_bar(&ctrl, p, smem_u32(&ctrl.p_free), pv_count & 1) && ok;
        ++pv_count;
        tc_fence_after();
        epilogue(true);
      }
    }
    // =======================================================================
    // FP8 cache: converters (warps 12..15).  In ring order, each raw stage becomes a
    // bf16 ring slot in exactly the layout the bf16 path's TMA would have produced
    // (64-column K-major boxes for QK, 2 x 64-column boxes for PV, 128-byte swizzle),
    // then both CTAs' converters arrive on the leader's full barrier of that slot.
    // =======================================================================
    else if (warp >= kConvWarp0) {
      if constexpr (kFp8) {
        regs_dec<kRegsConv>();
        constexpr int kStg = C::kStg;
        // two groups of two warps take alternate ring slots, so one group's hand-off
        // overlaps the other group's conversion
        const int grp = (tid - kConvWarp0 * 32) >> 6;  // 0, 1
        const int ct = (tid - kConvWarp0 * 32) & 63;   // 0..63 within the group
        constexpr int kGrpThreads = 64;
        PieceWalker walk(p, part, tile_row0);
        uint32_t js = 0, ir = 0;  // raw stages and ring slots consumed so far
        bool ok = true, go = true;
        auto wait_raw = [&](uint32_t j) {
          ok = wait_bar(&ctrl, p, smem_u32(&ctrl.stg_full[j % kStg]), (j / kStg) & 1) && ok;
        };
        auto wait_slot = [&]() {
          if (ir >= (uint32_t)kStages)
            ok = wait_bar(&ctrl, p, smem_u32(&ctrl.empty[ir % kStages]), ((ir / kStages) - 1) & 1) && ok;
        };
        // Hand slot ir to the MMAs and raw stages [j0, j0 + nraw) back to the
        // producers.  The AND barrier makes a timed-out wait leave all 128 threads
        // together.
        auto publish = [&](uint32_t j0, int nraw) -> bool {
          fence_proxy_async_smem();
          go = named_bar_and(kBarConv + grp, kGrpThreads, ok);
          if (!go) return false;
          if (ct == 0) {
            for (int k = 0; k < nraw; ++k) mbar_arrive(smem_u32(&ctrl.stg_empty[(j0 + k) % kStg]));
            const uint32_t fb = smem_u32(&ctrl.full[ir % kStages]);
            if (leader)
              mbar_arrive(fb);
            else
              mbar_arrive_remote(mapa_shared(fb, 0));
          }
          ++ir;
          return true;
        };
        // QK slab: raw = box b (own block b) as [64 rows][64 codes]; slot = box b as
        // [64 rows][128 B] swizzled.  Unit u = 16 codes: b = u >> 8, row m, granule k.
        // Eight consecutive threads cover two rows x four granules: 128 contiguous raw
        // bytes and eight distinct swizzled granules, so neither side has bank conflicts.
        auto conv_slab = [&](const uint8_t* src, uint8_t* dst, int own) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int u = ct + kGrpThreads * i, b = u >> 8;
            if (b >= own) continue;
            const int m = (u >> 2) & 63, k = u & 3;
            const uint4 v = *reinterpret_cast<const uint4*>(src + b * kSlabBlockBytes + m * 64 + 16 * k);
            uint8_t* row = dst + b * kChunkBytes + m * 128;
            const int g0 = (2 * k) ^ (m & 7);
            *reinterpret_cast<uint4*>(row + (g0 << 4)) =
                make_uint4(e4m3x2_to_bf16x2<false>(v.x), e4m3x2_to_bf16x2<true>(v.x), e4m3x2_to_bf16x2<false>(v.y),
                           e4m3x2_to_bf16x2<true>(v.y));
            *reinterpret_cast<uint4*>(row + ((g0 ^ 1) << 4)) =
                make_uint4(e4m3x2_to_bf16x2<false>(v.z), e4m3x2_to_bf16x2<true>(v.z), e4m3x2_to_bf16x2<false>(v.w),
                           e4m3x2_to_bf16x2<true>(v.w));
          }
        };
        // PV slab: raw = [64 rows][128 codes] swizzled; slot = two [64 rows][128 B]
        // swizzled boxes (columns 0..63, 64..127).  Unit u: row m = u & 63, 16-column
        // granule k = u >> 6; eight consecutive threads take eight rows of one granule.
        auto conv_vslab = [&](const uint8_t* src, uint8_t* dst) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int u = ct + kGrpThreads * i;
            const int m = u & 63, k = u >> 6;
            const uint4 v = *reinterpret_cast<const uint4*>(src + m * 128 + ((k ^ (m & 7)) << 4));
            uint8_t* row = dst + (k >> 2) * kChunkBytes + m * 128;
            const int g0 = (2 * (k & 3)) ^ (m & 7);
            *reinterpret_cast<uint4*>(row + (g0 << 4)) =
                make_uint4(e4m3x2_to_bf16x2<false>(v.x), e4m3x2_to_bf16x2<true>(v.x), e4m3x2_to_bf16x2<false>(v.y),
                           e4m3x2_to_bf16x2<true>(v.y));
            *reinterpret_cast<uint4*>(row + ((g0 ^ 1) << 4)) =
                make_uint4(e4m3x2_to_bf16x2<false>(v.z), e4m3x2_to_bf16x2<true>(v.z), e4m3x2_to_bf16x2<false>(v.w),
                           e4m3x2_to_bf16x2<true>(v.w));
          }
        };
        uint8_t* const ring = smem + kSmemRing;
        const uint8_t* const raw = smem + C::kSmemStg;
        auto conv_qk = [&](const Piece& pc, int t) {
          const int own = min(max(blocks_in_tile(pc, t) - 2 * (int)rank, 0), 2);
          for (int c = 0; c < 8; ++c) {
            if ((int)(ir & 1) != grp) {
              ++ir;
              ++js;
              continue;
            }
            wait_raw(js);
            wait_slot();
            if (ok) conv_slab(raw + (js % kStg) * kStgBytes, ring + (ir % kStages) * kStageBytes, own);
            if (!publish(js, 1)) return;
            ++js;
          }
          // k_pe: the two blocks' raw stages already hold the slot's boxes; copy them
          if ((int)(ir & 1) != grp) {
            ++ir;
            js += 2;
            return;
          }
          wait_raw(js);
          wait_raw(js + 1);
          wait_slot();
          if (ok) {
#pragma unroll
            for (int b = 0; b < 2; ++b) {
              if (b >= own) continue;
              const uint4* src = reinterpret_cast<const uint4*>(raw + ((js + b) % kStg) * kStgBytes);
              uint4* dst = reinterpret_cast<uint4*>(ring + (ir % kStages) * kStageBytes + b * kChunkBytes);
#pragma unroll
              for (int i = 0; i < 8; ++i) dst[ct + kGrpThreads * i] = src[ct + kGrpThreads * i];
            }
          }
          if (!publish(js, 2)) return;
          js += 2;
        };
        auto conv_pv = [&](const Piece& pc, int t) {
          const int nb = blocks_in_tile(pc, t);
          for (int h = 0; h < 2; ++h) {
            for (int kb = 0; kb < nb; ++kb) {
              if ((int)(ir & 1) != grp) {
                ++ir;
                ++js;
                continue;
              }
              wait_raw(js);
              wait_slot();
              if (ok) conv_vslab(raw + (js % kStg) * kStgBytes, ring + (ir % kStages) * kStageBytes);
              if (!publish(js, 1)) return;
              ++js;
            }
          }
        };
        // the producers' and the MMAs' ring order
        Piece cur, prv{};
        int prv_t = -1;
        while (go && walk.next(cur)) {
          const int nt = num_tiles(cur);
          for (int t = 0; t < nt && go; ++t) {
            conv_qk(cur, t);
            if (go && prv_t >= 0) conv_pv(prv, prv_t);
            prv = cur;
            prv_t = t;
          }
        }
        if (go && prv_t >= 0) conv_pv(prv, prv_t);
      }
    }
    // the peer CTA's MMA warp has no role; it joins its warpgroup's register release
    else if (warp == kMmaWarp) {
      if constexpr (kFp8) regs_dec<kRegsIssue>();
    }
  }

  // ---- teardown ------------------------------------------------------------
  if (warp == kSoftmaxWarp0 && lane == 0) bulk_wait_all();  // the epilogue's TMA stores landed
  tc_fence_before();
  __syncthreads();
  // Every role has stopped issuing (all waits are bounded).  Each CTA tells the other
  // whether it aborted; then both drain together or neither does.
  if (tid == 0) st_cluster_u32(mapa_shared(smem_u32((const void*)&ctrl.peer_abort), rank ^ 1u), (uint32_t)ctrl.abort);
  cluster_sync();
  tc_fence_after();
  if (ctrl.abort || ctrl.peer_abort) {
    // A wait ran out somewhere in the pair: asynchronous work issued before it may still
    // be in flight.  Tensor-core work (MMAs) has a completion handle: a commit issued
    // after it arrives on both CTAs' drain barriers once all of it has completed.  TMA
    // loads have none besides the stage barriers that did not complete, so both CTAs
    // also wait out their latency (at most a few microseconds even under full load)
    // with a 500 us margin before the TMEM and the shared memory are released.
    if (warp == kMmaWarp) {
      const bool el = elect_one();
      if (leader) commit_2sm_if(el, smem_u32(&ctrl.drain));
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
    cluster_sync();
    tc_fence_after();
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace

cudaError_t decode_kernel_setup(int device) {
  (void)device;
  cudaError_t e = cudaFuncSetAttribute(mla_decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cfg<false>::kSmemDyn + 1024);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(mla_decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              Cfg<true>::kSmemDyn + 1024);
}

// tm_kpe / tm_scl: FP8 cache only (null for the bf16 cache, which fp8 = false selects).
cudaError_t launch_decode(bool fp8, const CUtensorMap& tm_kv, const CUtensorMap& tm_kv2,
                          const CUtensorMap* tm_kpe, const CUtensorMap* tm_scl,
                          const CUtensorMap& tm_qn, const CUtensorMap& tm_qp,
                          const CUtensorMap& tm_out, const CUtensorMap& tm_part,
                          const int32_t* block_table, int max_blocks, const int32_t* seqlens,
                          const int32_t* q_lens, const int32_t* meta, int64_t num_blocks, int B, int s_q,
                          int H, float scale, int causal, void* out, float* lse, float* part_o, float* part_lse,
                          int32_t* status, int num_ctas, uint64_t wait_timeout_ns, int inject_stall,
                          cudaStream_t stream, int tok_rep, int tok_causal, const int32_t* tok_q_lens) {
  if (fp8 && (!tm_kpe || !tm_scl)) return cudaErrorInvalidValue;
  Params prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.tm_kv = tm_kv;
  prm.tm_kv2 = tm_kv2;
  if (fp8) {
    prm.tm_kpe = *tm_kpe;
    prm.tm_scl = *tm_scl;
  }
  prm.tm_qn = tm_qn;
  prm.tm_qp = tm_qp;
  prm.tm_out = tm_out;
  prm.tm_part = tm_part;
  prm.block_table = block_table;
  prm.seqlens = seqlens;
  prm.q_lens = q_lens;
  prm.tok_q_lens = tok_q_lens;
  prm.tok_rep = tok_rep;
  prm.tok_causal = tok_causal;
  prm.meta = meta;
  prm.out = reinterpret_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.part_o = part_o;
  prm.part_lse = part_lse;
  prm.status = status;
  prm.num_blocks = num_blocks;
  prm.timeout_ns = wait_timeout_ns;
  prm.max_blocks = max_blocks;
  prm.B = B;
  prm.s_q = s_q;
  prm.H = H;
  prm.M = s_q * H;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.causal = causal;
  prm.inject_stall = inject_stall;
  // Programmatic dependent launch: the CTAs start (and run their setup) while the
  // previous kernel in the stream finishes; the kernel waits for it before reading
  // any input.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_ctas);
  cfg.blockDim = dim3(fp8 ? Cfg<true>::kThreads : Cfg<false>::kThreads);
  cfg.dynamicSmemBytes = (fp8 ? Cfg<true>::kSmemDyn : Cfg<false>::kSmemDyn) + 1024;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return fp8 ? cudaLaunchKernelEx(&cfg, mla_decode_kernel<true>, prm)
             : cudaLaunchKernelEx(&cfg, mla_decode_kernel<false>, prm);
}

}  // namespace mla
