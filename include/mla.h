/*
 * mla.h -- C ABI of libmla_b200: Multi-head Latent Attention (MLA) decoding
 * over a paged latent KV cache on NVIDIA B200 (sm_100a).
 *
 * The method (sources by page title and section):
 *   - every query head attends to ONE shared latent KV head of 576 dims
 *     (512 "nope" dims followed by 64 decoupled-RoPE dims); V is the first
 *     d_v dims of the same latent row
 *       [FlashMLA (AI Wiki), "How does MLA differ from MHA and GQA?"]
 *   - the cache is paged in 64-token blocks reached through a block table,
 *     sequences have variable lengths
 *       [FlashMLA (AI Wiki), "What is FlashMLA?"]
 *   - the call pair get_mla_metadata(cache_seqlens, s_q*h_q/h_kv, h_kv) ->
 *     (tile_scheduler_metadata, num_splits), then per layer
 *     flash_mla_with_kvcache(q, kcache, block_table, cache_seqlens, dv,
 *     metadata, num_splits, causal) -> (o, lse)
 *       [FlashMLA Ampere port README, "Usage"]
 *   - outputs come with their log-sum-exp; token-level sparse decoding takes
 *     indices (b, s_q, topk) of physical slots (block*64 + offset), -1 =
 *     invalid, and ignores the block table
 *       [FlashMLA (AI Wiki), "Interfaces"]
 *   - the fused kernel applies Q RMSNorm, Q-RoPE, attention, conjugate O-RoPE
 *     and the FP8 cast in one pass
 *       [FlashMLA fused norm-RoPE-attention-RoPE-cast kernel card,
 *        "Arithmetic intensity"; deepseek-ai/FlashMLA README, "News"]
 *   - the 656-byte FP8 cache row: 512 E4M3 values with one fp32 scale per 128,
 *     then the 64 RoPE dims in bf16; the V4.1 rows of a 512-dim latent: 528
 *     bytes (512 E4M3 + 16 E8M0 scales, one per 32) or 288 bytes (512 E2M1
 *     packed two per byte + 32 E4M3 scales, one per 16)
 *       [FlashMLA (AI Wiki), "The FP8 and FP4 KV cache"]
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller, unless an
 *     argument says "host".  The library allocates no device memory; scratch
 *     space is the caller's `workspace` (size from the *_size queries),
 *     except for mla_decode_fwd_noalloc, which uses a fixed array of its own.
 *   - Layouts are dense, row-major, innermost dimension last:
 *       q            [batch, s_q, h_q, 576]        bf16 (16-byte aligned)
 *       kcache       [num_blocks, 64, 1, 576]      bf16 (16-byte aligned)
 *       block_table  [batch, max_pages]            int32 (entries past a
 *                                                  sequence's last page are
 *                                                  never read)
 *       cache_seqlens[batch]                       int32
 *       out          [batch, s_q, h_q, d_v]        bf16
 *       lse          [batch, s_q, h_q]             fp32, natural log
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All GPU work is enqueued asynchronously on it.
 *   - Every function returns MLA_OK (0) or a negative status.  Arguments are
 *     validated before anything is launched, so a failed call has enqueued
 *     no work.  mla_last_error() returns a message for the calling thread's
 *     most recent failure.
 *   - An empty row (no visible token) produces O = 0 and LSE = -inf.
 *   - Cache slots that are not visible to a row must still hold finite
 *     values: masked tokens are multiplied by a zero probability.
 */
#ifndef MLA_B200_H_
#define MLA_B200_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_OK 0
#define MLA_ERR_INVALID_ARG (-1) /* null/misaligned pointer, bad size or shape */
#define MLA_ERR_UNSUPPORTED (-2) /* valid request outside what is built (h_kv != 1, ...) */
#define MLA_ERR_CUDA (-3)        /* a CUDA runtime call failed; see mla_last_error() */
#define MLA_ERR_TIMEOUT (-4)     /* a kernel gave up on a bounded wait (mla_device_status) */

/* Message describing the calling thread's most recent failure ("" if none). */
MLA_API const char* mla_last_error(void);

/* Number of streaming multiprocessors of `device` (host out-pointer). */
MLA_API int mla_num_sms(int device, int* num_sms);

/* Scheduler partition count for `device`: num_SMs / ceil(heads_per_kv / 64)
 * / h_kv.  heads_per_kv = s_q * h_q / h_kv is the number of query rows that
 * share one KV head (the second argument of get_mla_metadata in the port
 * README's "Usage").  Result in *num_sm_parts (host). */
MLA_API int mla_num_sm_parts(int device, int heads_per_kv, int h_kv, int* num_sm_parts);

/* Byte sizes of the two scheduler outputs for `batch` sequences and
 * `num_sm_parts` partitions: metadata int32[num_sm_parts][8] and num_splits
 * int32[batch + 1] (host out-pointers). */
MLA_API int mla_metadata_size(int batch, int num_sm_parts, size_t* metadata_bytes,
                      size_t* num_splits_bytes);

/* Split-KV tile scheduler (the metadata call of the port README's "Usage").
 * Deals the 128-token tiles of all sequences to `num_sm_parts` partitions of
 * about equal cost (tiles + a fixed per-segment overhead); each partition
 * covers one contiguous run of (sequence, tile) pairs.
 *   cache_seqlens  int32[batch], device
 *   metadata       int32[num_sm_parts][8], device, written:
 *                  {begin_seq, begin_tile, end_seq, end_tile (exclusive),
 *                   split index of begin_seq's segment, 0, 0, 0}
 *   num_splits     int32[batch + 1], device, written: prefix sums of the
 *                  number of partitions holding tiles of each sequence
 * Runs as one small kernel on `stream`; compute it once per decode step and
 * reuse it for every layer.  heads_per_kv and h_kv are validated only. */
MLA_API int mla_get_metadata(const int32_t* cache_seqlens, int batch, int heads_per_kv, int h_kv,
                     int num_sm_parts, int32_t* metadata, int32_t* num_splits, void* stream);

/* The same planner on the host (all three arrays are host pointers); the
 * result is bit-identical to mla_get_metadata's. */
MLA_API int mla_get_metadata_host(const int32_t* cache_seqlens, int batch, int heads_per_kv, int h_kv,
                          int num_sm_parts, int32_t* metadata, int32_t* num_splits);

/* Workspace bytes for mla_decode_fwd: fp32 partial outputs and LSEs of up
 * to batch + num_sm_parts splits of `rows_per_kv` (= s_q*h_q) rows of d_v
 * values. */
MLA_API int mla_workspace_size(int batch, int rows_per_kv, int d_v, int num_sm_parts, size_t* bytes);

/* Workspace bytes for mla_fused_norm_rope_attn_rope_cast: the split partials
 * of mla_workspace_size(batch, h_q, 576, num_sm_parts), then the normalised,
 * rotated query rows (batch * h_q rows of 576 bf16). */
MLA_API int mla_fused_workspace_size(int batch, int h_q, int num_sm_parts, size_t* bytes);

/* Dense paged MLA decode, bf16 in, bf16 out + fp32 LSE
 * (flash_mla_with_kvcache of the port README's "Usage").
 *   q, kcache, block_table, cache_seqlens, out, lse: see the layouts above.
 *   max_pages       second dimension of block_table
 *   num_blocks      first dimension of kcache (block ids must be < num_blocks)
 *   h_kv            must be 1 (MLA: one latent KV head)
 *   d_v             512 (V = K[:, :512]) or 576
 *   softmax_scale   multiplies q.k before the softmax (typically 1/sqrt(576))
 *   causal          nonzero: query i of s_q sees L - s_q + 1 + i tokens
 *                   (bottom-right alignment); zero: every query sees L tokens
 *   metadata, num_splits, num_sm_parts: from mla_get_metadata for the same
 *                   cache_seqlens and heads_per_kv = s_q*h_q
 *   workspace       device scratch of >= mla_workspace_size() bytes,
 *                   16-byte aligned; contents need no initialisation
 * Launches the decode kernel and the split-combine kernel on `stream`. */
MLA_API int mla_decode_fwd(const void* q, const void* kcache, const int32_t* block_table, int max_pages,
                   int num_blocks, const int32_t* cache_seqlens, int batch, int s_q, int h_q,
                   int h_kv, int d_v, float softmax_scale, int causal, const int32_t* metadata,
                   const int32_t* num_splits, int num_sm_parts, void* workspace,
                   size_t workspace_bytes, void* out, float* lse, void* stream);

/* Fused Q RMSNorm -> Q-RoPE -> attention -> conjugate O-RoPE -> FP8 cast,
 * s_q = 1, d_v = 576 (V is the whole latent row).  Three launches on
 * `stream`: the query prologue (once per row, into the workspace), the
 * attention kernel, and the split combine with the output RoPE and the cast.
 *   q_raw           [batch, 1, h_q, 576] bf16, before normalisation
 *   norm_gain       fp32[576], shared by all heads; eps added to mean(x^2)
 *   rope_base       RoPE base (e.g. 10000); pairs (2k, 2k+1) of dims
 *                   512..575 rotate by theta_k = pos * base^(-2k/64)
 *   positions       int32[batch] query positions, or NULL for L - 1
 *   kcache ...      as in mla_decode_fwd; the cache's RoPE dims are expected
 *                   to be rotated at their own positions already
 *   out_e4m3        [batch, 1, h_q, 576] E4M3 codes (OCP FP8), RNE, saturating
 *   out_scale       fp32[batch, 1, h_q]: absmax(O_row) / 448 (1 for a zero row);
 *                   O ~= code * scale
 *   lse             fp32[batch, 1, h_q]
 *   metadata, num_splits from mla_get_metadata with heads_per_kv = h_q
 *   workspace       >= mla_fused_workspace_size() bytes, 16-byte aligned. */
MLA_API int mla_fused_norm_rope_attn_rope_cast(
    const void* q_raw, const float* norm_gain, float eps, float rope_base,
    const int32_t* positions, const void* kcache, const int32_t* block_table, int max_pages,
    int num_blocks, const int32_t* cache_seqlens, int batch, int h_q, float softmax_scale,
    const int32_t* metadata, const int32_t* num_splits, int num_sm_parts, void* workspace,
    size_t workspace_bytes, uint8_t* out_e4m3, float* out_scale, float* lse, void* stream);

/* Workspace bytes for mla_sparse_decode (scheduler tables + split partials). */
MLA_API int mla_sparse_workspace_size(int batch, int s_q, int h_q, int topk, int d_v, int num_sm_parts,
                              size_t* bytes);

/* Token-level sparse decode over the 656-byte FP8 latent cache.
 *   q             [batch, s_q, h_q, 576] bf16
 *   kcache_fp8    [num_slots, 656] bytes per row: 512 E4M3 codes, 4 fp32
 *                 scales (one per 128 codes, little-endian), 64 bf16 RoPE dims
 *   num_slots     rows of kcache_fp8 (num_blocks * 64)
 *   indices       int32[batch, s_q, topk]: physical slots; -1 (or any value
 *                 outside [0, num_slots)) marks an unused entry
 *   d_v           512
 *   out, lse      [batch, s_q, h_q, d_v] bf16 and [batch, s_q, h_q] fp32
 *   num_sm_parts  from mla_num_sm_parts(device, h_q, 1)
 * The scheduling tables are generated inside this call (into workspace). */
MLA_API int mla_sparse_decode(const void* q, const uint8_t* kcache_fp8, int64_t num_slots,
                      const int32_t* indices, int topk, int batch, int s_q, int h_q, int d_v,
                      float softmax_scale, int num_sm_parts, void* workspace,
                      size_t workspace_bytes, void* out, float* lse, void* stream);

/* Workspace bytes for mla_sparse_decode_v41 and mla_sparse_decode_v41_fp4:
 * those of mla_sparse_decode with d_v = 512, plus room for the query widened
 * to 576 dims (used when h_q <= 64). */
MLA_API int mla_sparse_v41_workspace_size(int batch, int s_q, int h_q, int topk, int num_sm_parts,
                                  size_t* bytes);

/* Token-level sparse decode over the 528-byte V4.1 FP8 latent cache
 * [FlashMLA (AI Wiki), "The FP8 and FP4 KV cache", layout table].
 *   q             [batch, s_q, h_q, 512] bf16: the latent is 512 wide, RoPE
 *                 dims included
 *   kcache_528    [num_slots, 528] bytes per row: 512 E4M3 codes covering all
 *                 512 dims, then 16 E8M0 scales (one per 32 consecutive
 *                 codes); a value is code * 2^(e - 127), e = 0xFF is NaN
 *   num_slots     rows of kcache_528 (num_blocks * 64)
 *   indices       int32[batch, s_q, topk]: physical slots; -1 (or any value
 *                 outside [0, num_slots)) marks an unused entry
 *   out, lse      [batch, s_q, h_q, 512] bf16 (V = the whole latent) and
 *                 [batch, s_q, h_q] fp32
 *   softmax_scale usually 1/sqrt(512)
 *   num_sm_parts  from mla_num_sm_parts(device, h_q, 1)
 * The dequantised rows are written in the 576-dim layout of the dense kernels
 * with zero dims 512..575.  With h_q > 64 the CTA-pair kernel reads the
 * 512-wide query as it is and multiplies 512 dims of each row; otherwise the
 * query is widened with zero dims too, which leaves q . k unchanged.
 * Ownership, alignment (q, the cache and out 16-byte aligned, workspace
 * 256-byte aligned) and errors as in mla_sparse_decode. */
MLA_API int mla_sparse_decode_v41(const void* q, const uint8_t* kcache_528, int64_t num_slots,
                          const int32_t* indices, int topk, int batch, int s_q, int h_q,
                          float softmax_scale, int num_sm_parts, void* workspace,
                          size_t workspace_bytes, void* out, float* lse, void* stream);

/* Token-level sparse decode over the 288-byte V4.1 FP4 latent cache
 * [FlashMLA (AI Wiki), "The FP8 and FP4 KV cache", layout table].
 *   kcache_288    [num_slots, 288] bytes per row: 512 E2M1 codes packed two
 *                 per byte into 256 bytes (code 2i in the low nibble of byte
 *                 i, code 2i + 1 in the high nibble), then 32 E4M3 scales,
 *                 one per 16 consecutive codes; a value is code * scale
 * Every other argument, the layouts, the workspace
 * (mla_sparse_v41_workspace_size), ownership and errors are those of
 * mla_sparse_decode_v41. */
MLA_API int mla_sparse_decode_v41_fp4(const void* q, const uint8_t* kcache_288, int64_t num_slots,
                              const int32_t* indices, int topk, int batch, int s_q, int h_q,
                              float softmax_scale, int num_sm_parts, void* workspace,
                              size_t workspace_bytes, void* out, float* lse, void* stream);

/* Workspace bytes for mla_sparse_prefill_fwd: the clamped lengths and split
 * plan of up to 8192 query tokens, the list of the tokens split over several
 * parts, and their partials (2 * num_sm_parts * h_q rows of 512 fp32). */
MLA_API int mla_sparse_prefill_workspace_size(int s_q, int h_q, int topk, int num_sm_parts,
                                      size_t* bytes);

/* Token-level sparse prefill, with no batch dimension
 * [FlashMLA (AI Wiki), "Interfaces": sparse prefill takes optional
 * attention-sink and per-token top-k-length arguments].
 *   q             [s_q, h_q, 576] bf16, one row per (query token, head)
 *   kv            [s_kv, 576] bf16: the latent KV head, one row per position
 *   indices       int32[s_q, topk]: rows of kv each query token attends to;
 *                 -1 (or a value outside [0, s_kv)) marks an unused entry
 *   topk_length   int32[s_q] or NULL: only the first topk_length[t] entries
 *                 of token t's indices count (clamped to [0, topk])
 *   attn_sink     fp32[h_q] or NULL: a per-head logit that joins the softmax
 *                 normaliser without a value row: LSE' = log(e^LSE + e^sink),
 *                 O' = O e^(LSE - LSE'); a token with no row gets O = 0 and
 *                 LSE = sink
 *   d_v           512 (V = kv[:, :512]); softmax_scale usually 1/sqrt(576)
 *   out, lse      [s_q, h_q, 512] bf16 (16-byte aligned) and [s_q, h_q] fp32
 *   num_sm_parts  from mla_num_sm_parts(device, h_q, 1)
 * Each query token is one unit of the CTA-pair attention kernel, whose loads
 * fetch the token's rows straight from kv (four named rows per TMA copy); a
 * launch covers up to 8192 tokens.  The sinks join each row's normaliser
 * where the row is finished (the attention kernel, or the combine of the
 * tokens split over several parts).  num_sm_parts is capped at the device's
 * SMs / (2 ceil(h_q / 128)) CTA pairs.
 * Ownership and errors as in mla_sparse_decode. */
MLA_API int mla_sparse_prefill_fwd(const void* q, const void* kv, int64_t s_kv,
                           const int32_t* indices, int topk, const int32_t* topk_length,
                           const float* attn_sink, int s_q, int h_q, int d_v,
                           float softmax_scale, int num_sm_parts, void* workspace,
                           size_t workspace_bytes, void* out, float* lse, void* stream);

/* Workspace bytes for mla_sparse_fused_norm_rope_attn_rope_cast. */
MLA_API int mla_sparse_fused_workspace_size(int batch, int h_q, int topk, int num_sm_parts,
                                    size_t* bytes);

/* The fused decode in sparse mode: the steps of
 * mla_fused_norm_rope_attn_rope_cast (Q RMSNorm, Q-RoPE, attention,
 * conjugate O-RoPE, FP8 cast; s_q = 1, d_v = 576) over the valid slots of
 * `indices` in the 656-byte FP8 cache, as mla_sparse_decode selects them
 * [FlashMLA fused norm-RoPE-attention-RoPE-cast kernel card, "Arithmetic
 * intensity", "Workarounds"; FlashMLA (AI Wiki), "Interfaces"].
 *   q_raw, norm_gain, eps, rope_base, out_e4m3, out_scale, lse: as in
 *                 mla_fused_norm_rope_attn_rope_cast
 *   positions     int32[batch] query positions, REQUIRED (the selected slots
 *                 do not give the query's position)
 *   kcache_fp8, num_slots: as in mla_sparse_decode
 *   indices       int32[batch, 1, topk] physical slots, -1 = unused
 *   num_sm_parts  from mla_num_sm_parts(device, h_q, 1)
 * A row with no valid slot gives O = 0 (codes 0, scale 1) and LSE = -inf.
 * Ownership, alignment and errors as in mla_sparse_decode. */
MLA_API int mla_sparse_fused_norm_rope_attn_rope_cast(
    const void* q_raw, const float* norm_gain, float eps, float rope_base,
    const int32_t* positions, const uint8_t* kcache_fp8, int64_t num_slots,
    const int32_t* indices, int topk, int batch, int h_q, float softmax_scale, int num_sm_parts,
    void* workspace, size_t workspace_bytes, uint8_t* out_e4m3, float* out_scale, float* lse,
    void* stream);

/* Dense decode without a caller workspace.  This entry point has no
 * counterpart in the method's published interface; it exists for callers
 * that cannot supply scratch memory at decode time (an embedder whose device
 * memory belongs to another allocator, or a caller that must not allocate at
 * that moment).  Arguments, layouts and results are those of mla_decode_fwd;
 * the split planner runs inside the call.
 *   Scratch   the split tables and fp32 partials live in one fixed array of
 *             mla_noalloc_scratch_bytes() (32 MiB) bytes inside the
 *             library's device image; this call allocates no device memory.
 *   Limit     a problem whose tables + partials exceed that size
 *             ((batch + parts) * s_q*h_q * d_v * 4 bytes dominate, parts =
 *             mla_num_sm_parts(device, s_q*h_q, 1)) returns
 *             MLA_ERR_INVALID_ARG with the bytes it would need.
 *   Device    the current CUDA device; `stream` must belong to it.  The
 *             first call on each device looks up the array's address once;
 *             make that first call outside any stream capture.  The address
 *             is kept for the life of the process, so a cudaDeviceReset
 *             between calls is not supported.
 *   Sharing   every call on a device uses the same array: calls that may
 *             run at the same time on the GPU (unordered streams) race and
 *             give wrong results.  Order them, e.g. on one stream.
 *             Nothing in the array needs to be zeroed first. */
MLA_API size_t mla_noalloc_scratch_bytes(void);
MLA_API int mla_decode_fwd_noalloc(const void* q, const void* kcache, const int32_t* block_table,
                           int max_pages, int num_blocks, const int32_t* cache_seqlens, int batch,
                           int s_q, int h_q, int h_kv, int d_v, float softmax_scale, int causal,
                           void* out, float* lse, void* stream);

/* Profiling aid, with no counterpart in the method's published interface:
 * while set, every decode entry point records `start_event` on its stream
 * right before it launches its attention kernel and `stop_event` right after,
 * so that a caller can time that kernel alone (cudaEventElapsedTime) next to
 * the planner and combine launches of the same call.  Both are cudaEvent_t
 * handles owned by the caller (NULL = do not record).  Inside a stream
 * capture they become event-record nodes of the graph, timed at each replay.
 * The setting belongs to the calling host thread; pass NULL, NULL to clear
 * it. */
MLA_API int mla_set_kernel_events(void* start_event, void* stop_event);

/* Debug aid, with no counterpart in the method's published interface: while
 * set, every decode entry point called from this host thread records which
 * cache rows its kernels read, so that a test can compare the index and
 * block-table handling with the inputs bit for bit.
 *   trace     int32 device array (caller-owned) of `capacity` entries, or
 *             NULL to switch the trace off.  A call writes two planes of N
 *             entries each (plane 1 starts at trace + N):
 *               dense and fused decode: N = batch * max_pages * 64; entry
 *                 b * max_pages * 64 + t holds the physical slot
 *                 (block * 64 + t % 64) that token t of sequence b was loaded
 *                 from, plane 0 for the rows read as K and plane 1 for the
 *                 rows read as V.  Only tokens of pages that hold part of the
 *                 sequence are written (a partial last page in full); an
 *                 out-of-range block id shows as block 0.
 *               sparse decode and fused sparse decode: N = batch * s_q *
 *                 topk; entry p * topk + j holds the slot entry j of query p
 *                 read (-1 if unused or out of range) in plane 0, and the row
 *                 of the compacted buffer it went to (valid entries numbered
 *                 in index order) in plane 1.
 *               sparse prefill: N = s_q * topk; entry t * topk + j holds the
 *                 kv row entry j of token t read in plane 0 and j itself in
 *                 plane 1 (the rows are read in place), both -1 for an entry
 *                 that is unused, out of range or past the token's length.
 *             Entries the call does not write keep their contents.
 *   capacity  entries of `trace`; a call needing more than 2 * N returns
 *             MLA_ERR_INVALID_ARG before any launch.
 * The setting belongs to the calling host thread. */
MLA_API int mla_set_slot_trace(int32_t* trace, int64_t capacity);

/* Reads the device status words that kernels set: 0 = ok, else (code << 16)
 * | site of the first event, code 1 = a bounded wait expired, 2 = an input
 * named nothing in the cache (a block id outside [0, num_blocks), a length
 * above max_pages * 64, a sparse index outside [0, num_slots)).  A code-2
 * fault does not stop any kernel: the block id reads block 0, the length is
 * cut to max_pages * 64 (the default fused query position still follows the
 * length as given), and the index is skipped like -1.  A timeout makes every
 * later bounded wait give up until the words are reset, and it takes
 * precedence in *status.  Synchronises the device; reset != 0 clears both
 * words afterwards.  Returns MLA_ERR_TIMEOUT if a wait expired, else
 * MLA_OK. */
MLA_API int mla_device_status(int* status, int reset);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_H_ */
