/*
 * mla_decode.h -- C ABI of libmla.so: weight-absorbed multi-head latent attention
 * (MLA) decode over a paged latent KV cache, for NVIDIA B200 (sm_100a).
 *
 * What is computed.  For sequence b with n_b = cache_seqlens[b] cached tokens, query
 * token i (0 <= i < s_q) and head h, the cache row of token t is
 *     r_t = kv_cache[block_table[b][t / 64]][t % 64][0:576]  =  [ c_kv (512) | k_pe (64) ]
 * and the key t is visible when t < n_b and, with causal != 0, t <= n_b - s_q + i
 * (the s_q new tokens are the last s_q cache positions).  Over the visible keys:
 *     s_t            = softmax_scale * (q_nope[b,i,h,:] . c_kv_t + q_pe[b,i,h,:] . k_pe_t)
 *     lse[b,i,h]     = ln sum_t exp(s_t)
 *     out[b,i,h,:]   = sum_t exp(s_t - lse) * c_kv_t
 * Rows with no visible key get out = 0 and lse = -inf.
 *
 * Sources (page titles and sections): weight-absorbed MLA in decode, one latent row
 * shared by all heads -- KsanaLLM 0.6.0 release notes, section 2.1 (WA-MLA / DP
 * attention); softmax scale 1/sqrt(192) from DeepSeek's 192-wide attention head --
 * Paddle 3.0 inference upgrade article, long-sequence (SageAttention) section;
 * several draft tokens per sequence in one decode call -- same article, speculative
 * decoding section; softmax_lse side output and split-K (split-KV) parallelism --
 * "DeepSeek speed test / FA3" article, section 2.1; paged cache with a block table --
 * Dewu deployment slides (PagedAttention) and the same FA3 article, section 4.1.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller, contiguous
 *    row-major in the shapes shown, and 16-byte aligned.  The library allocates
 *    no device memory and keeps no state except a per-device cache of the SM count
 *    and of kernel attributes.
 *  - Calls that take a stream are asynchronous on that stream.  Host-detectable
 *    errors are returned before anything is launched; nothing else is written.
 *  - Device-detectable data errors (a block id outside [0, num_blocks) among the
 *    blocks a sequence uses, n_b < 0, n_b > max_blocks * 64, metadata whose block
 *    count for a sequence is not ceil(n_b / 64)) never fault and never read past a
 *    sequence's blocks: the affected sequence's out rows and lse are set to NaN and
 *    a bit is OR-ed into *status (MLA_DEVICE_ERR_*) when status != NULL.  A bounded
 *    wait inside a kernel that runs out (1 s) sets MLA_DEVICE_ERR_TIMEOUT and the
 *    kernel returns.
 *  - No C++ exception crosses this boundary.  Calls are re-entrant given distinct
 *    metadata / workspace buffers.
 */
#ifndef MLA_DECODE_H_
#define MLA_DECODE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,         /* null pointer, negative size, misalignment, ... */
  MLA_ERR_UNSUPPORTED = 2,         /* shape outside the supported set (see below)    */
  MLA_ERR_CUDA = 3,                /* a CUDA runtime / driver call failed            */
  MLA_ERR_WORKSPACE_TOO_SMALL = 4, /* metadata or workspace buffer below its size    */
  MLA_ERR_DEVICE = 5               /* no sm_100 device current                        */
} mla_status_t;

/* Bits OR-ed into the optional device status word by the kernels. */
#define MLA_DEVICE_ERR_BLOCK_ID 1 /* block_table entry outside [0, num_blocks) */
#define MLA_DEVICE_ERR_SEQLEN 2   /* cache_seqlens[b] < 0 or > max_blocks * 64,
                                     or q_lens[b] outside [0, s_q]               */
#define MLA_DEVICE_ERR_TIMEOUT 4  /* an internal bounded wait ran out           */
#define MLA_DEVICE_ERR_METADATA 8 /* metadata not produced for these B, s_q, H, or
                                     for another length of some sequence (its block
                                     count differs; that sequence's rows are NaN)   */

/* Fixed geometry. */
#define MLA_BLOCK_SIZE 64  /* cache rows per physical block   */
#define MLA_D_LATENT 512   /* c_kv width = output width       */
#define MLA_D_ROPE 64      /* k_pe / q_pe width               */
#define MLA_D_QK 576       /* cache row width                 */

/* Supported shapes: H in {16, 32, 64, 128}, s_q in {1, 2, 3, 4}, 1 <= B <= 65536. */

/* Human-readable name of a status code (static string, never NULL). */
const char* mla_status_string(mla_status_t status);

/*
 * Bytes of the schedule buffer mla_get_metadata writes for (B, s_q, H).  Host only,
 * no device call.  *bytes receives the size.  Library convenience: no passage of the
 * source pages corresponds to it.
 */
mla_status_t mla_metadata_size(int B, int s_q, int H, size_t* bytes);

/*
 * Split-KV schedule for one decode step (shared by every layer of that step).
 *
 * The concatenation of all sequences' key tiles (four 64-row blocks, 256 keys) is cut
 * into contiguous ranges of near-equal cost, one per partition, only on tile
 * boundaries; every sequence also costs a fixed overhead of one tile before its
 * first tile.  A sequence cut across partitions is computed as several
 * partial results that mla_decode merges by log-sum-exp (split-K parallelism, "DeepSeek
 * speed test / FA3" article section 2.1; the cost model is this library's own).
 *
 *   cache_seqlens  device int32 [B]   (n_b; negative values count as 0 here)
 *   metadata       device buffer of at least mla_metadata_size(B, s_q, H) bytes,
 *                  written asynchronously on `stream`; opaque to the caller.
 * The schedule depends only on (cache_seqlens, s_q, H, the device's SM count).
 */
mla_status_t mla_get_metadata(const int32_t* cache_seqlens, int B, int s_q, int H,
                              void* metadata, size_t metadata_bytes, void* stream);

/*
 * Upper bound, in bytes, of the fp32 scratch mla_decode needs for split partial
 * results (partial outputs and their lse) for (B, s_q, H) on the current device.
 * The partials are the split-K intermediate results of the "DeepSeek speed test /
 * FA3" article, section 2.1; the size query itself is a library convenience.
 */
mla_status_t mla_workspace_size(int B, int s_q, int H, size_t* bytes);

/*
 * The decode attention itself.
 *
 *   q_nope         bf16 [B, s_q, H, 512]   absorbed latent queries
 *   q_pe           bf16 [B, s_q, H, 64]    RoPE queries
 *   kv_cache       bf16 [num_blocks, 64, 576]
 *   block_table    int32 [B, max_blocks]   physical block of logical block k of b;
 *                                          entries past ceil(n_b / 64) are never read
 *   cache_seqlens  int32 [B]               n_b, counting the s_q new tokens
 *   softmax_scale  scale applied to the scores (1/sqrt(192) for DeepSeek MLA)
 *   causal         nonzero: causal mask among the s_q new tokens (bottom-right)
 *   metadata       from mla_get_metadata for the same cache_seqlens, s_q, H
 *   workspace      >= mla_workspace_size(B, s_q, H) bytes of device scratch
 *   out            bf16 [B, s_q, H, 512]   (written)
 *   lse            fp32 [B, s_q, H]        natural-log log-sum-exp of the scaled scores
 *   status         device int32 (may be NULL): MLA_DEVICE_ERR_* bits are OR-ed in
 *   stream         cudaStream_t (NULL = legacy default stream)
 *
 * Launches the split-KV attention kernel (one 2-CTA cluster per 128 query rows and
 * partition; TMA-fed tcgen05 MMAs with TMEM accumulators) and then the LSE-combine
 * kernel that merges split sequences.
 */
mla_status_t mla_decode(const void* q_nope, const void* q_pe, const void* kv_cache,
                        int64_t num_blocks, const int32_t* block_table, int max_blocks,
                        const int32_t* cache_seqlens, int B, int s_q, int H,
                        float softmax_scale, int causal, const void* metadata,
                        size_t metadata_bytes, void* workspace, size_t workspace_bytes,
                        void* out, float* lse, int32_t* status, void* stream);

/*
 * mla_decode with a per-sequence number of query tokens: sequence b has
 * q_lens[b] <= s_q new tokens (speculative decoding where sequences accept different
 * numbers of draft tokens -- Paddle 3.0 inference upgrade article, speculative
 * decoding section).  Its tokens are the last q_lens[b] cache positions: with causal
 * != 0, token i sees keys 0 .. n_b - q_lens[b] + i.  Tokens i >= q_lens[b] are padding:
 * their out rows are 0 and their lse -inf.  q and out keep the padded
 * [B, s_q, H, ...] layout.
 *
 *   q_lens  device int32 [B], each in [0, s_q]; NULL means s_q for every sequence
 *           (then the call is mla_decode).  A value outside [0, s_q] makes that
 *           sequence's rows NaN and sets MLA_DEVICE_ERR_SEQLEN.
 * Other arguments, the metadata and the workspace are those of mla_decode.  A 128-row
 * tile of query rows that holds only padding tokens of a sequence is not computed.
 */
mla_status_t mla_decode_ragged(const void* q_nope, const void* q_pe, const void* kv_cache,
                               int64_t num_blocks, const int32_t* block_table, int max_blocks,
                               const int32_t* cache_seqlens, const int32_t* q_lens, int B, int s_q,
                               int H, float softmax_scale, int causal, const void* metadata,
                               size_t metadata_bytes, void* workspace, size_t workspace_bytes,
                               void* out, float* lse, int32_t* status, void* stream);

/*
 * Token schedule for ragged query counts.  mla_decode_ragged schedules every 128-row
 * tile of query rows over the same partitions, so when sequences carry different
 * numbers of real tokens the tiles of the later token positions (held only by the
 * sequences that kept that many drafts) leave their partitions' CTAs idle.  The token
 * schedule instead runs the call as an s_q = 1 decode over B * s_q token sequences:
 * sequence u = b * s_q + t is token t of sequence b, with the first n_b - q_lens[b] + t + 1
 * keys of b under the causal mask (all n_b keys without it) and none for a padding
 * token (t >= q_lens[b]).  That is the same result (the causal mask of a token is a
 * shorter visible prefix; speculative-decoding section of the Paddle 3.0 inference
 * upgrade article for the per-sequence draft counts), balanced over all CTAs like an
 * s_q = 1 batch.
 *
 * mla_get_metadata_tokens: the schedule for mla_decode_tokens / mla_decode_fp8_tokens.
 *   q_lens may be NULL (s_q tokens for every sequence); causal must be the flag the
 *   decode will use.  metadata holds mla_metadata_size(B * s_q, 1, H) bytes.
 * mla_decode_tokens, mla_decode_fp8_tokens: arguments and outputs as mla_decode_ragged /
 *   mla_decode_fp8 (q, out, lse in the padded [B, s_q, H, ...] layout); the metadata must
 *   come from mla_get_metadata_tokens with the same cache_seqlens, q_lens and causal flag,
 *   and the workspace holds mla_workspace_size(B * s_q, 1, H) bytes.  Device errors as in
 *   mla_decode_ragged (an invalid length or query count makes all of that sequence's rows
 *   NaN and sets MLA_DEVICE_ERR_SEQLEN; metadata of another shape, schedule kind or causal
 *   flag sets MLA_DEVICE_ERR_METADATA).  Library scheduling, no further passage.
 */
mla_status_t mla_get_metadata_tokens(const int32_t* cache_seqlens, const int32_t* q_lens, int B, int s_q, int H,
                                     int causal, void* metadata, size_t metadata_bytes, void* stream);
mla_status_t mla_decode_tokens(const void* q_nope, const void* q_pe, const void* kv_cache, int64_t num_blocks,
                               const int32_t* block_table, int max_blocks, const int32_t* cache_seqlens,
                               const int32_t* q_lens, int B, int s_q, int H, float softmax_scale, int causal,
                               const void* metadata, size_t metadata_bytes, void* workspace,
                               size_t workspace_bytes, void* out, float* lse, int32_t* status, void* stream);
mla_status_t mla_decode_fp8_tokens(const void* q_nope, const void* q_pe, const void* kv_fp8, int64_t num_blocks,
                                   const int32_t* block_table, int max_blocks, const int32_t* cache_seqlens,
                                   const int32_t* q_lens, int B, int s_q, int H, float softmax_scale, int causal,
                                   const void* metadata, size_t metadata_bytes, void* workspace,
                                   size_t workspace_bytes, void* out, float* lse, int32_t* status, void* stream);

/*
 * The two launches mla_decode performs, exposed separately (same arguments, same
 * semantics; mla_decode == mla_decode_attention followed by mla_decode_combine on
 * the same stream with the same workspace).
 *
 * mla_decode_attention: the split-KV attention kernel (the
 *   weight-absorbed attention of the KsanaLLM 0.6.0 release notes, section 2.1, with
 *   the split-K partials of the "DeepSeek speed test / FA3" article, section 2.1).
 *   Sequences processed in one piece get their out / lse rows written directly;
 *   pieces of split sequences write normalised fp32 partial outputs and their lse into
 *   the workspace.  It also writes the rows of sequences with no visible key
 *   (0 / -inf) and of sequences with an invalid length (NaN, MLA_DEVICE_ERR_SEQLEN)
 *   or a stale block count in the metadata (NaN, MLA_DEVICE_ERR_METADATA).  Exposing
 *   it separately is a library convenience (timing, custom merges).
 * mla_decode_combine: the LSE-combine kernel (split-K merge, "DeepSeek speed test /
 *   FA3" article section 2.1): for every split sequence, lse = ln sum_s exp(lse_s) and
 *   out = sum_s exp(lse_s - lse) O_s.  Only split sequences are touched; `status` is
 *   accepted for symmetry and never written.
 */
mla_status_t mla_decode_attention(const void* q_nope, const void* q_pe, const void* kv_cache,
                                  int64_t num_blocks, const int32_t* block_table, int max_blocks,
                                  const int32_t* cache_seqlens, int B, int s_q, int H,
                                  float softmax_scale, int causal, const void* metadata,
                                  size_t metadata_bytes, void* workspace, size_t workspace_bytes,
                                  void* out, float* lse, int32_t* status, void* stream);
mla_status_t mla_decode_combine(const int32_t* cache_seqlens, int max_blocks, int B, int s_q, int H,
                                const void* metadata, size_t metadata_bytes, const void* workspace,
                                size_t workspace_bytes, void* out, float* lse, int32_t* status,
                                void* stream);

/*
 * mla_decode without a caller-provided workspace, for callers that cannot allocate
 * device memory (an engine whose memory pool already reserved the device, a plugin
 * that only receives input and output pointers, a decode loop that cannot afford
 * cudaMalloc's implicit synchronisation).  There is no counterpart of this call in
 * the source pages; it is a deployment convenience.
 *
 * Same arguments and results as mla_decode minus the workspace.  The split-KV
 * scratch is a 64 MiB array compiled into the library (each GPU that loads the
 * library holds it until the process exits).  The call allocates nothing.
 *  - If mla_workspace_size(B, s_q, H) exceeds 64 MiB it returns
 *    MLA_ERR_WORKSPACE_TOO_SMALL and launches nothing (use mla_decode with your own
 *    workspace for such shapes; for H = 128, s_q = 1 the limit is B <= 181 on a
 *    148-SM B200).
 *  - The first call on each device looks up the array's device address (with that
 *    device current) and caches it; make that first call before any stream capture.
 *  - All calls share the one array and it keeps the last call's contents; every slot
 *    a call reads is written earlier in the same call, so nothing needs clearing.
 *    Calls whose kernels overlap on the GPU (different streams without ordering)
 *    race on the array: serialise them.
 */
mla_status_t mla_decode_noalloc(const void* q_nope, const void* q_pe, const void* kv_cache,
                                int64_t num_blocks, const int32_t* block_table, int max_blocks,
                                const int32_t* cache_seqlens, int B, int s_q, int H,
                                float softmax_scale, int causal, const void* metadata,
                                size_t metadata_bytes, void* out, float* lse, int32_t* status,
                                void* stream);

/*
 * Failure-path test hooks, process-wide, for launches made after the call.  Library
 * conveniences: no passage of the source pages corresponds to them, and production
 * code never needs them.
 *
 * mla_set_wait_timeout_ns: bound on every internal mbarrier wait of the attention
 *   kernel, in nanoseconds (ns = 0 restores the default of 1 s).  A wait that runs
 *   out sets MLA_DEVICE_ERR_TIMEOUT: every role of the kernel stops issuing work, the
 *   CTA pair waits for the tensor-core work and the TMA loads it had in flight, and
 *   the kernel returns with that call's outputs undefined.
 * mla_set_stall_injection: nonzero makes the attention kernel's MMA warp first wait
 *   on a barrier that nothing ever completes, so that wait and then the others run
 *   out -- the way the timeout path is exercised without a faulty kernel.  0 turns
 *   it off.
 */
mla_status_t mla_set_wait_timeout_ns(uint64_t ns);
mla_status_t mla_set_stall_injection(int enable);

/*
 * Weight-absorption GEMMs either side of the decode (KsanaLLM 0.6.0 release notes,
 * section 2.1, WA-MLA).  With per-head up-projections k_h = W_UK[h] c and
 * v_h = W_UV[h] c of the 512-d latent c, and query rows r = b * s_q + i (R rows):
 *
 * mla_absorb_q:   q_nope[r, h, :] = W_UK[h]^T q_heads[r, h, :]
 *   q_heads  bf16 [R, H, 128]   per-head no-RoPE queries
 *   w_uk     bf16 [H, 128, 512] key up-projections (row k of W_UK[h] is 512 wide)
 *   q_nope   bf16 [R, H, 512]   written: the absorbed query mla_decode takes
 * mla_absorb_out: y[r, h, :] = W_UV[h] o[r, h, :]
 *   o_latent bf16 [R, H, 512]   the decode output
 *   w_uv     bf16 [H, 128, 512] value up-projections
 *   y        bf16 [R, H, 128]   written: per-head attention output
 *
 * fp32 accumulation, bf16 results (round to nearest even).  Pointers are device
 * pointers, 16-byte aligned; 1 <= R, 1 <= H <= 65535.  Asynchronous on `stream`;
 * host-detectable errors return before any launch.
 */
mla_status_t mla_absorb_q(const void* q_heads, const void* w_uk, void* q_nope, int R, int H,
                          void* stream);
mla_status_t mla_absorb_out(const void* o_latent, const void* w_uv, void* y, int R, int H,
                            void* stream);

/*
 * FP8 (e4m3) latent cache.  8-bit KV-cache inference is among the serving
 * capabilities of the Paddle 3.0 inference upgrade article (closing list); the
 * per-token max-abs scale follows the quantised KV cache of the "DeepSeek speed test"
 * article, section 3.1.  The packed row (656 bytes, this library's format):
 *   [0, 512)    e4m3 codes of c_kv / scale (OCP E4M3FN)
 *   [512, 640)  k_pe / scale as 64 bf16
 *   [640, 644)  fp32 scale = max|row| / 448 over all 576 values
 *   [644, 656)  zero
 * with code = e4m3(c / scale): IEEE fp32 quotient, rounded to nearest even, saturated
 * to +-448, and k_pe' = bf16(k_pe / scale) rounded to nearest even; a zero row has
 * scale 0 and stores zeros.  The dequantised row is scale * [e4m3(code) | k_pe'].
 *
 * mla_quantize_kv_fp8: quantise `rows` bf16 cache rows [rows, 576] into packed rows
 *   [rows, 656] (for a paged cache, rows = num_blocks * 64).  Device pointers, 16-byte
 *   aligned; asynchronous on `stream`.
 */
mla_status_t mla_quantize_kv_fp8(const void* kv_cache, void* kv_fp8, int64_t rows, void* stream);

/*
 * mla_decode_fp8: mla_decode_ragged over a packed FP8 cache (the format above): the
 * same arguments, with `kv_fp8` = [num_blocks][64][656] bytes (device, 16-byte aligned)
 * in place of the bf16 cache; q_lens may be NULL (s_q tokens for every sequence).  The
 * result is the decode of the dequantised rows scale * [e4m3(code) | k_pe'] (the FP8
 * cache is 8-bit KV-cache inference, Paddle 3.0 inference upgrade article, closing
 * capabilities list).  The schedule, workspace, error statuses and asynchrony are
 * those of mla_decode.
 */
mla_status_t mla_decode_fp8(const void* q_nope, const void* q_pe, const void* kv_fp8, int64_t num_blocks,
                            const int32_t* block_table, int max_blocks, const int32_t* cache_seqlens,
                            const int32_t* q_lens, int B, int s_q, int H, float softmax_scale, int causal,
                            const void* metadata, size_t metadata_bytes, void* workspace, size_t workspace_bytes,
                            void* out, float* lse, int32_t* status, void* stream);

/* mla_decode_fp8_attention: the split-KV attention launch of mla_decode_fp8 alone (its
 * LSE combine is mla_decode_combine, as for mla_decode_attention).  Same arguments and
 * passage as mla_decode_fp8; used to time the attention kernel by itself. */
mla_status_t mla_decode_fp8_attention(const void* q_nope, const void* q_pe, const void* kv_fp8, int64_t num_blocks,
                                      const int32_t* block_table, int max_blocks, const int32_t* cache_seqlens,
                                      const int32_t* q_lens, int B, int s_q, int H, float softmax_scale, int causal,
                                      const void* metadata, size_t metadata_bytes, void* workspace,
                                      size_t workspace_bytes, void* out, float* lse, int32_t* status,
                                      void* stream);

/*
 * Quantised causal prefill attention, head dimension 192 (SageAttention-style: Paddle
 * 3.0 inference upgrade article, long-sequence section -- Q and K dynamically
 * quantised to INT8 and V to FP8, the INT32 scores converted to FP32 and dequantised,
 * an online softmax, P quantised to FP8 and multiplied with the FP8 V, the product
 * dequantised by V's scale; DeepSeek's head dimension 192).
 *
 * Inputs (device, 16-byte aligned, bf16, row-major): q, k [S][H][192] (query i is
 * token i of one sequence; key j is visible to query i when j <= i), v [S][H][128].
 * Outputs: out [S][H][128] bf16, lse [S][H] fp32 (natural log of the sum of the
 * quantised weights, scale included).  Quantisation (this library's reading of the
 * passage): Q and K per (token, head), scale = max|x| / 127, code = rint(x / scale);
 * V per (head, channel) over all tokens, scale = max|v| / 448, code = e4m3(v / scale);
 * P = 2^(x - m) in [0, 1] at the running row maximum m of 128-key blocks, coded as
 * e4m3(P * 448); the output is normalised by the sum of the coded weights.
 *
 * mla_sage_workspace_size: bytes of the workspace for (S, H): the codes and scales,
 *   S_pad = S rounded up to 128: q8, k8 int8 [H][S_pad][192]; vt8 e4m3 [H][128][S_pad]
 *   (V transposed); sq, sk fp32 [H][S_pad]; sv fp32 [H][128]; uint32 [H][128] scratch.
 *   1 <= S, 1 <= H <= 65535.
 * mla_sage_quantize: fill the workspace from q, k, v (asynchronous on `stream`).
 * mla_sage_attention: the attention kernel over a filled workspace.  status (device
 *   int32, may be NULL) gets MLA_DEVICE_ERR_TIMEOUT if a pipeline wait ran out.
 * mla_sage_prefill: mla_sage_quantize then mla_sage_attention.
 * Host-detectable errors return before any launch; the workspace belongs to the caller
 * and must not be shared by concurrent calls.
 */
mla_status_t mla_sage_workspace_size(int S, int H, size_t* bytes);
mla_status_t mla_sage_quantize(const void* q, const void* k, const void* v, int S, int H, void* workspace,
                               size_t workspace_bytes, void* stream);
mla_status_t mla_sage_attention(int S, int H, float softmax_scale, const void* workspace, size_t workspace_bytes,
                                void* out, float* lse, int32_t* status, void* stream);
mla_status_t mla_sage_prefill(const void* q, const void* k, const void* v, int S, int H, float softmax_scale,
                              void* workspace, size_t workspace_bytes, void* out, float* lse, int32_t* status,
                              void* stream);

/* Number of streaming multiprocessors the schedule targets on the current device.
 * Library convenience: no passage of the source pages corresponds to it. */
mla_status_t mla_device_sm_count(int* sm_count);

#ifdef __cplusplus
}
#endif
#endif /* MLA_DECODE_H_ */
