/*
 * csa.h -- C ABI of the CSA / HCA hot-path library for NVIDIA B200 (sm_100a).
 *
 * The method (DeepSeek-V4 long-context attention, as described by the
 * "DeepSeek-V4" book, slop-6tp.pages.dev/papers-html-argon/dsv4.html):
 *   1. block-compress the KV sequence into one entry per m tokens by
 *      coordinate-wise softmax pooling        (Ch.5 "How CSA Compresses Memory")
 *   2. score every eligible compressed entry for each query with the lightning
 *      indexer                                 (Ch.6 "The lightning indexer")
 *   3. keep the top-k entries per query        (Ch.6 "Top-k selection ...")
 *   4. softmax attention over the selected entries plus a window of recent raw
 *      tokens; HCA attends densely to every eligible heavily compressed entry
 *                                              (Ch.6 "Shared key-value MQA",
 *                                               Ch.7 "HCA, Local Attention, and Position")
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; every tensor
 *     is row-major with the innermost dimension contiguous and 16-byte aligned.
 *     bf16 tensors are passed as raw bit patterns (csa_bf16).
 *   - Shared-KV layout: one tensor row is both the key and the value of an
 *     entry (Ch.6 "Shared key-value MQA").
 *   - The library allocates no memory and never synchronises, except
 *     csa_workspace_check(), which synchronises its stream.  Work is enqueued
 *     on the given stream (NULL = the legacy default stream).
 *   - Positions are 0-based.  Query position t may read compressed entry s iff
 *     s < floor(t/m) (Ch.5 "Causal availability and the local sliding window").
 *     A query's window holds its raw tokens max(0, t-W+1) .. t, itself
 *     included; duplicates of selected entries are kept (Ch.7 "The 128-token
 *     uncompressed sliding window").
 *   - Every call returns a csa_status_t.  Argument errors are detected on the
 *     host before anything is enqueued.  A kernel that meets a bad index or
 *     page id records CSA_ERR_DEVICE_CHECK in the workspace header (see
 *     csa_workspace_check), skips that row and carries on; nothing traps.
 *   - csa_last_error() returns a thread-local description of the last failure.
 *
 * Supported sizes: attention head dim d in {128, 512} (512, the pages' entry
 * width, runs on an mma.sync kernel whose four warps split the dims; the
 * mixed-precision entries and the fused query prologue / output de-rotation
 * need d = 128); indexer key dim c_I in {64, 128}; indexer heads H_I <= 64;
 * attention heads H <= 128; m >= 1; window <= 1024.
 */
#ifndef CSA_H
#define CSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t csa_bf16;                 /* raw bf16 bit pattern */
typedef struct CUstream_st* csa_stream_t;  /* a cudaStream_t */

typedef enum {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = 1,   /* bad pointer, size or combination; nothing enqueued */
  CSA_ERR_UNSUPPORTED = 2,   /* legal but not built (e.g. d != 128); nothing enqueued */
  CSA_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
  CSA_ERR_DEVICE_CHECK = 4,  /* a kernel recorded a bad index / page id */
  CSA_ERR_WORKSPACE = 5      /* workspace missing or smaller than required */
} csa_status_t;

/*
 * A per-sequence compressed cache (main KV entries or indexer keys).
 *   data        device, rows of `dim` bf16 (dim given by the call)
 *   n_rows      number of physical rows `data` holds (bounds for the checks)
 *   page_table  NULL: contiguous; sequence b's entry s is row b*seq_stride + s.
 *               else device int32 [n_seq, max_pages]: entry s of sequence b is
 *               row page_table[b*max_pages + s/page_size]*page_size + s%page_size
 *               (a paged-attention style block table; the pages note that the
 *               compressed cache is kept apart from the raw-token state cache,
 *               "Decode-time cache state", Ch.5).
 */
typedef struct {
  const void* data;
  int64_t n_rows;
  int64_t seq_stride;
  const int32_t* page_table;
  int32_t page_size;
  int32_t max_pages;
} csa_cache_t;

/* ---- library information ------------------------------------------------ */
const char* csa_version(void);
const char* csa_last_error(void);
/* Number of kernels this library has launched since it was loaded. */
uint64_t csa_launch_count(void);

/*
 * Timing hook: when `ev_begin`/`ev_end` (cudaEvent_t, created by the caller)
 * are non-NULL, the library records them on the call's stream immediately
 * before and after every launch of kernel `kernel_id`.  Pass NULLs to detach.
 * kernel_id: 0 = indexer scoring, 1 = top-k selection, 2 = attention,
 * 3 = split merge, 4 = compression, 5 = 4-bit quantization.
 */
csa_status_t csa_set_timing_events(int32_t kernel_id, void* ev_begin, void* ev_end);

/*
 * Attention kernel choice for csa_sparse_attn_prefill, csa_sparse_attn_decode
 * and hca_attn (process-wide; a library setting with no counterpart in the
 * method).  0 = automatic (default): the tcgen05 tensor-core kernel wherever
 * it supports the call and the call asks for the fused query prologue /
 * output de-rotation, or a query's row list may hold more than 256 rows
 * (top_k, or max_entries for hca_attn, plus window) and the call is not one
 * of at most 16 heads over at least 2048 queries; else the mma.sync kernel
 * (faster on short row lists and on few heads over many queries); 1 = the
 * tcgen05 kernel wherever it supports the
 * call, else the mma.sync kernel; 2 = always the mma.sync kernel.  Both compute the same attention within the same
 * tolerance; the split-KV slicing of a decode call may differ between them
 * (within the same workspace size).  Returns CSA_ERR_INVALID_ARG for any other
 * value.
 */
csa_status_t csa_set_attention_kernel(int32_t choice);

/*
 * Batch-invariant decode (process-wide; off by default).  When on, the split
 * of each query's row list (selected entries, then window rows) for
 * csa_sparse_attn_decode and for decode calls of hca_attn is fixed slices of
 * 512 rows, merged in slice order, whatever the batch: a query's output and
 * log-sum-exp are then bit-identical whether it is decoded alone or in any
 * batch, at some cost in speed for small batches.  The decode and HCA
 * workspace-size queries account for the mode in force when they are called.
 * DeepSeek-V4 infrastructure notes, "batch invariance": split-KV decoding
 * otherwise makes the accumulation order, and so the bits, depend on the
 * batch.  Returns CSA_ERR_INVALID_ARG unless `on` is 0 or 1.
 */
csa_status_t csa_set_batch_invariant(int32_t on);

/*
 * Failure-detection self-test (process-wide, one shot; a library setting with
 * no counterpart in the method).  With on = 1 the next launch of the tcgen05
 * attention kernel never issues its first work item's query-tile copy and
 * waits at most about 1 ms (2^21 cycles) on each pipeline barrier: its
 * bounded waits give up, it records "a bounded pipeline wait timed out" in
 * the workspace header (read it with csa_workspace_check) and returns, and
 * the device stays usable.  No output of that launch is valid.  The setting
 * clears itself at that launch; on = 0 clears it before.  Returns
 * CSA_ERR_INVALID_ARG unless `on` is 0 or 1.
 */
csa_status_t csa_test_attention_timeout(int32_t on);

/* ---- workspace ------------------------------------------------------------ */
/*
 * Calls that take `ws` need a caller-allocated device workspace of at least
 * the size returned by the matching *_workspace_size function (256-byte
 * aligned).  Its first 256 bytes are a header holding the device-check record;
 * initialise it once with csa_workspace_init (or zero the buffer).  Calls that
 * run concurrently on different streams need separate workspaces.
 */
size_t csa_indexer_topk_workspace_size(int64_t T, int64_t max_entries, int32_t top_k);
size_t csa_sparse_attn_decode_workspace_size(int32_t B, int32_t H, int32_t d, int32_t top_k,
                                             int32_t window);
size_t csa_sparse_attn_prefill_workspace_size(int64_t L, int32_t H, int32_t d);
size_t hca_attn_workspace_size(int64_t T, int32_t H, int32_t d, int64_t max_entries,
                               int32_t window);

/* Zero the header of a workspace (enqueued on `stream`). */
csa_status_t csa_workspace_init(void* ws, size_t ws_bytes, csa_stream_t stream);
/*
 * Synchronise `stream`, read the header and return CSA_OK or
 * CSA_ERR_DEVICE_CHECK (details in csa_last_error()).  Clears the record.
 */
csa_status_t csa_workspace_check(void* ws, csa_stream_t stream);

/* ---- step 1: block compression ------------------------------------------- */
/*
 * csa_compress_kv -- coordinate-wise softmax pooling of a token sequence into
 * floor(n_tokens/m) compressed entries.
 *   overlap = 0 (BLOCK, HCA's compressor, Ch.7 "HCA's 128:1 non-overlapping
 *     compressor"): entry i, coordinate r =
 *       sum_{j=mi}^{mi+m-1} softmax_j(Z_a[j,r] + bias[j-mi,r]) * C_a[j,r]
 *   overlap = 1 (CSA's compressor, Ch.5 "Coordinate-wise softmax pooling"):
 *     one softmax over 2m positions: block i with (C_a, Z_a + bias[0]) and
 *     block i-1 with (C_b, Z_b + bias[1]); entry 0 has no previous block, its
 *     b branch contributes nothing (content 0, logits -inf).
 *   C_a, Z_a   [n_tokens, dim] bf16
 *   C_b, Z_b   [n_tokens, dim] bf16, overlap only; NULL -> use C_a / Z_a
 *   bias       fp32 [m, dim] (BLOCK) or [2, m, dim] (OVERLAP, a then b), or NULL
 *   out        [floor(n_tokens/m), dim] bf16; tokens past the last full block
 *              produce nothing (the window covers them)
 *   dim % 8 == 0.  Accumulation in fp32, output rounded to nearest bf16.
 */
csa_status_t csa_compress_kv(const csa_bf16* C_a, const csa_bf16* Z_a, const csa_bf16* C_b,
                             const csa_bf16* Z_b, const float* bias, int64_t n_tokens,
                             int32_t dim, int32_t m, int32_t overlap, csa_bf16* out,
                             csa_stream_t stream);

/*
 * csa_cache_append -- decode-time cache maintenance, one new token per
 * sequence (Book Ch.5 "Decode-time cache state"; Ch.8 "Quantization scales
 * and bounded tail buffers").  For sequence b, with t = pos[b] (the number of
 * tokens before the new one):
 *   - its raw row C_a[b] goes to the window ring: win[b, t mod window]
 *     (the decode attention reads the ring's first min(t+1, window) slots;
 *     their order does not matter to the softmax);
 *   - its a-branch rows (C_a, Z_a) go to the unfinished-block buffers at row
 *     t mod m, and in overlap mode its b-branch rows (C_b, Z_b) to the buffer
 *     of block parity (t / m) mod 2;
 *   - when it completes block i = t / m (t mod m == m - 1), entry i of the
 *     compressed cache is written: the csa_compress_kv pooling of block i
 *     (and of block i-1's b-branch rows in overlap mode), bit for bit the
 *     entry csa_compress_kv gives for the whole sequence.
 * Call once per decode step, in order of t, for every sequence; the buffers
 * are the per-sequence state and must persist between calls.
 *   C_a, Z_a      [B, dim] bf16;  C_b, Z_b [B, dim] bf16 (overlap; NULL -> C_a / Z_a)
 *   bias          fp32 [m, dim] or [2, m, dim] (as csa_compress_kv), or NULL
 *   pos           int64 [B], >= 0
 *   blk_c, blk_z  [B, m, dim] bf16 state
 *   bb_c, bb_z    [B, 2, m, dim] bf16 state (overlap only, else NULL)
 *   win           [B, window, dim] bf16 ring (NULL when window == 0)
 *   cache         compressed entries [.., dim]; sequence b's entry i at its row
 *   max_entries   entries each sequence's cache can hold; a completed block past
 *                 it, or a bad page id, is skipped and recorded in the workspace
 *   ws            device workspace of at least 256 bytes (the device-check header)
 * dim % 8 == 0, dim <= 2048; all buffers 16-byte aligned.
 */
csa_status_t csa_cache_append(const csa_bf16* C_a, const csa_bf16* Z_a, const csa_bf16* C_b,
                              const csa_bf16* Z_b, const float* bias, const int64_t* pos,
                              int32_t B, int32_t dim, int32_t m, int32_t overlap,
                              csa_bf16* blk_c, csa_bf16* blk_z, csa_bf16* bb_c, csa_bf16* bb_z,
                              csa_bf16* win, int32_t window, const csa_cache_t* cache,
                              int64_t max_entries, void* ws, size_t ws_bytes, csa_stream_t stream);

/*
 * csa_norm_rope -- the attention prologue / epilogue on [T, H, dim] bf16
 * vectors (Book Ch.2 "Normalization and rotary position embeddings"; Ch.7
 * "Query and KV RMSNorm", "Partial RoPE and output de-rotation"):
 *   eps >= 0: RMSNorm, x / sqrt(mean(x^2) + eps) * gain (gain [dim] fp32 or
 *             NULL for 1); eps < 0 skips it;
 *   rope_dims > 0: the last rope_dims coordinates are rotated by R_p, pairs
 *             (2j, 2j+1) of that slice by angle p * rope_base^(-2j/rope_dims),
 *             at position p = (pos ? pos[t] : t) * pos_mul; inverse = 1 applies
 *             R_{-p} (the output de-rotation with the query position).
 * Queries: eps, rope at the token position.  Compressed entries: pos_mul = m
 * (entry i at position i*m, the first token of its block; a reading, the
 * pages do not say which token).  Window rows: their token positions.
 * Attention outputs: eps < 0, inverse = 1, the query positions.
 *   out may equal x (in place).  dim in {64, 128, 256}; rope_dims a multiple
 *   of 8 and <= dim; 16-byte aligned buffers.  fp32 arithmetic (angles reduced
 *   modulo 2 pi in fp64), output rounded to nearest bf16.
 */
csa_status_t csa_norm_rope(const csa_bf16* x, csa_bf16* out, int64_t T, int32_t H, int32_t dim,
                           const float* gain, float eps, const int64_t* pos, int64_t pos_mul,
                           int32_t rope_dims, float rope_base, int32_t inverse,
                           csa_stream_t stream);

/* ---- steps 2-3: lightning indexer + top-k ---------------------------------- */
/*
 * csa_indexer_topk -- for every query i at position t_i of sequence b_i:
 *   I[s] = sum_h w[i,h] * ReLU(q_idx[i,h,:] . K[b_i, s, :]),  s < floor(t_i/m)
 * (Ch.6 "The lightning indexer"), then the top_k entries by I (Ch.6 "Top-k
 * selection and asymptotic scaling").  Scores are accumulated and compared in
 * fp32; equal scores go to the lower entry index; with fewer than top_k
 * eligible entries all are taken.  The score matrix is never returned.
 * Up to 2048 queries per call (decode), no score matrix is formed at all: a
 * small pass scores a strided sample of each query's entries and sets a
 * threshold that about 2 top_k of them are expected to reach; the scorer keeps
 * only the (score, entry) pairs at or above it, O(top_k) per query in the
 * workspace; an exact select over those finishes the job whenever at least
 * top_k and at most the workspace's slots reached the threshold, and exact
 * recompute passes over the query's entries handle the other (rare) cases.
 * Larger calls (prefill) keep every score of a chunk of queries in the
 * workspace and select per query.  Results are the same either way.
 * top_k <= 4096; max_entries <= 2^19; c_I in {64, 128}; H_I <= 64.
 *   q_idx      [T, H_I, c_I] bf16
 *   w          [T, H_I] fp32
 *   k_idx      cache of [*, c_I] bf16 indexer keys (host struct)
 *   seq_id     [T] int32 sequence of each query, or NULL (all sequence 0)
 *   q_pos      [T] int64 position of each query, or NULL (query i at position i)
 *   max_entries upper bound of floor(t_i/m) over the queries (workspace layout)
 *   idx_out    [T, top_k] int32: selected entry ids, ascending, padded with -1
 *   count_out  [T] int32: number selected = min(top_k, floor(t_i/m))
 *   score_out  [T, top_k] fp32 score of each selected entry (-inf pad), or NULL
 */
csa_status_t csa_indexer_topk(const csa_bf16* q_idx, const float* w, const csa_cache_t* k_idx,
                              const int32_t* seq_id, const int64_t* q_pos, int64_t T,
                              int32_t H_I, int32_t c_I, int32_t m, int64_t max_entries,
                              int32_t top_k, int32_t* idx_out, int32_t* count_out,
                              float* score_out, void* ws, size_t ws_bytes, csa_stream_t stream);

/*
 * 4-bit indexer storage (Ch.8 "A Cost Model for Long Context": "V4
 * compressed-entry payload" keeps the indexer keys in FP4, half a byte per
 * scalar; "Quantization scales and bounded tail buffers": one 1-byte scale per
 * 32 elements; Ch.6 "Top-k selection and asymptotic scaling": the indexer
 * scan runs in FP4).  The pages fix no encoding; the one used is the OCP
 * Microscaling (MXFP4) format:
 *   element  E2M1 code: bit 3 sign, bits 2..1 exponent (bias 1), bit 0
 *            mantissa; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6
 *   scale    byte b = X + 127 means 2^X; X = floor(log2 amax) - 2 for the
 *            block's largest magnitude amax, clamped to [-127, 127]
 *            (-127 for an all-zero block)
 *   code     x / 2^X rounded to the nearest magnitude, ties to the even code
 *            (mantissa bit 0), saturating at 6; sign bit = sign bit of x
 *   packing  byte i of a vector holds element 2i in its low nibble and
 *            element 2i+1 in its high nibble; scales in their own array
 *
 * csa_quantize_mxfp4 -- quantize n_vectors rows of dim bf16 values:
 *   x       [n_vectors, dim] bf16 (16-byte aligned); dim % 32 == 0
 *   codes   [n_vectors, dim/2] uint8 out (16-byte aligned)
 *   scales  [n_vectors, dim/32] uint8 out
 * Bit-exact; results for non-finite inputs are unspecified.
 */
csa_status_t csa_quantize_mxfp4(const csa_bf16* x, int64_t n_vectors, int32_t dim, uint8_t* codes,
                                uint8_t* scales, csa_stream_t stream);

/*
 * csa_indexer_topk_mxfp4 -- csa_indexer_topk with the indexer keys in 4-bit
 * storage: every query's bf16 heads are quantized to the same format inside
 * the call (codes identical to csa_quantize_mxfp4's), and the score definition
 * is applied to the dequantized queries and keys (each 32-element block's dot
 * product is exact; the blocks are scaled and summed, and the heads weighted
 * and summed, in fp32).  Selection rules, workspace
 * (csa_indexer_topk_workspace_size) and outputs are those of csa_indexer_topk.
 *   q_idx     [T, H_I, c_I] bf16 (16-byte aligned)
 *   k_codes   cache whose rows are c_I/2 code bytes (data 16-byte aligned)
 *   k_scales  [k_codes->n_rows, c_I/32] uint8 (16-byte aligned): the scale bytes
 *             of physical row r of k_codes are row r of k_scales
 * c_I in {64, 128}; H_I <= 64.  Scale bytes 0 and 255 (2^-127 and the
 * E8M0 NaN) are outside the supported range: csa_quantize_mxfp4 produces 0
 * only for blocks whose largest magnitude is below 2^-124.
 */
csa_status_t csa_indexer_topk_mxfp4(const csa_bf16* q_idx, const float* w,
                                    const csa_cache_t* k_codes, const uint8_t* k_scales,
                                    const int32_t* seq_id, const int64_t* q_pos, int64_t T,
                                    int32_t H_I, int32_t c_I, int32_t m, int64_t max_entries,
                                    int32_t top_k, int32_t* idx_out, int32_t* count_out,
                                    float* score_out, void* ws, size_t ws_bytes,
                                    csa_stream_t stream);

/* ---- step 4: attention ---------------------------------------------------- */
/*
 * csa_qrope_t -- the attention layer's query prologue and output epilogue,
 * fused into the attention calls below (Ch.7 "Query and KV RMSNorm", "Partial
 * RoPE and output de-rotation"; Ch.2 "Normalization and rotary position
 * embeddings").  With a non-NULL csa_qrope_t* the call reads the raw queries
 * and, before the dot products, replaces every query head q by
 *   R_t . (q / sqrt(mean(q^2) + q_eps) * q_gain)        (q_eps < 0: no RMSNorm)
 * rounded to bf16, R_t rotating pairs (2j, 2j+1) of the last rope_dims
 * coordinates by t * rope_base^(-2j / rope_dims) (t the query's position); with
 * derotate = 1 each output head's last rope_dims coordinates are rotated by
 * R_{-t} before they are stored.  The compressed entries and window rows are
 * used as given (normalise and rotate them once with csa_norm_rope).
 *   q_gain     [d] fp32 gain, or NULL (gain 1)
 *   rope_dims  a multiple of 8 up to d (0: no rotation); rope_base > 1 when used
 *   pos        [T] int64 position of each query; NULL means the row index for
 *              csa_sparse_attn_prefill and q_pos (else the row index) for
 *              hca_attn; required by csa_sparse_attn_decode
 * Needs the tensor-core attention kernel (CSA_ERR_UNSUPPORTED otherwise).
 */
typedef struct {
  const float* q_gain;
  float q_eps;
  int32_t rope_dims;
  float rope_base;
  int32_t derotate;
  const int64_t* pos;
} csa_qrope_t;

/*
 * csa_sparse_attn_prefill -- CSA attention for the L queries of one sequence,
 * query t at position t:
 *   o[t,h] = sum_j softmax_j(sm_scale * q[t,h] . kv_j) kv_j
 * over j in {kv_comp[idx[t,0..count[t]-1]]} followed by the window rows
 * kv_raw[max(0,t-W+1) .. t], one softmax (Ch.6 "Shared key-value MQA", Ch.7
 * "The 128-token uncompressed sliding window").  With `sink` (fp32 [H]) each
 * head's denominator gains exp(sink[h]) (Ch.7 "Learned attention sinks").
 *   q        [L, H, d] bf16        kv_comp [n_entries, d] bf16
 *   kv_raw   [L, d] bf16           idx [L, top_k] int32, count [L] int32
 *   out      [L, H, d] bf16        lse [L, H] fp32 log of the denominator, or NULL
 *   qrope    query prologue / output epilogue (see csa_qrope_t), or NULL
 */
csa_status_t csa_sparse_attn_prefill(const csa_bf16* q, const csa_bf16* kv_comp,
                                     int64_t n_entries, const csa_bf16* kv_raw,
                                     const int32_t* idx, const int32_t* count, int64_t L,
                                     int32_t H, int32_t d, int32_t top_k, int32_t window,
                                     float sm_scale, const float* sink, csa_bf16* out,
                                     float* lse, void* ws, size_t ws_bytes,
                                     csa_stream_t stream, const csa_qrope_t* qrope);

/*
 * csa_sparse_attn_decode -- one new token per sequence b (query b belongs to
 * sequence b of kv_comp): attention over the selected entries
 * kv_comp[b, idx[b, 0..count[b]-1]] followed by the window buffer rows
 * win[b, 0..win_len[b]-1] (oldest first, the new token last), one softmax.
 * The selected set is split over several CTAs and merged (split-KV, which the
 * DeepSeek-V4 infrastructure video transcript, prism.simon-ai.net, describes
 * as the way decode keeps every SM busy).
 *   q [B, H, d] bf16; win [B, window, d] bf16; win_len [B] int32 (<= window)
 *   idx [B, top_k] int32; count [B] int32; out [B, H, d] bf16; lse [B, H] or NULL
 *   qrope query prologue / output epilogue (csa_qrope_t; its pos is required), or NULL
 */
csa_status_t csa_sparse_attn_decode(const csa_bf16* q, const csa_cache_t* kv_comp,
                                    const csa_bf16* win, const int32_t* win_len,
                                    const int32_t* idx, const int32_t* count, int32_t B,
                                    int32_t H, int32_t d, int32_t top_k, int32_t window,
                                    float sm_scale, const float* sink, csa_bf16* out,
                                    float* lse, void* ws, size_t ws_bytes,
                                    csa_stream_t stream, const csa_qrope_t* qrope);

/*
 * csa_sparse_attn_decode_noalloc -- csa_sparse_attn_decode for callers that
 * cannot allocate device memory (no counterpart in the paper: it only changes
 * where the scratch lives).  Some callers never get to call cudaMalloc: a
 * plugin inside a serving engine that owns all device memory and hands its
 * plugins only a stream, or latency-critical code that must not call
 * cudaMalloc because it can synchronise the device.  This form takes the same
 * arguments minus the workspace and keeps its split-KV partials in a 16 MiB
 * array in the library's own device memory (every GPU that loads the library
 * holds it until exit).  It allocates nothing.
 *   - Calls needing more than 16 MiB of scratch (see
 *     csa_sparse_attn_decode_workspace_size) fail with CSA_ERR_WORKSPACE and
 *     enqueue nothing; e.g. B = 64, H = 64, top_k = 2048, window = 128 needs
 *     about 10.6 MB.
 *   - Argument errors (the same checks as csa_sparse_attn_decode) are returned
 *     before the array is touched; B == 0 returns CSA_OK at once.
 *   - The first call on a device looks up the array's device address with that
 *     device current and keeps it for the life of the process; make that first
 *     call before any stream capture.  A device reset (cudaDeviceReset or
 *     anything else that destroys the primary context) invalidates the kept
 *     address: do not call this form again in that process after one.
 *   - Every call shares the one array, which keeps the last call's contents:
 *     calls that overlap on the GPU (other streams, other host threads) race.
 *     Each call clears the array's device-check header first; that record is
 *     not readable by the caller, so what the kernels record there -- bad entry
 *     indices or page ids (skipped), and a pipeline wait that gave up (output
 *     incomplete) -- is not reported by this form: a call can return CSA_OK
 *     after either.  Callers that need those reports use
 *     csa_sparse_attn_decode with csa_workspace_check.
 */
csa_status_t csa_sparse_attn_decode_noalloc(const csa_bf16* q, const csa_cache_t* kv_comp,
                                            const csa_bf16* win, const int32_t* win_len,
                                            const int32_t* idx, const int32_t* count, int32_t B,
                                            int32_t H, int32_t d, int32_t top_k, int32_t window,
                                            float sm_scale, const float* sink, csa_bf16* out,
                                            float* lse, csa_stream_t stream);

/*
 * Mixed-precision compressed entries (Ch.8 "A Cost Model for Long Context",
 * "V4 compressed-entry payload": the content channels in FP8, the last 64
 * rotary channels in BF16, 576 bytes at c = 512; "Quantization scales and
 * bounded tail buffers": block scale metadata).  The pages fix neither the
 * FP8 variant nor the scale rule; the ones used:
 *   element  E4M3 without infinities (sign, 4 exponent bits with bias 7,
 *            field 0 subnormal, 3 mantissa bits), largest value 448
 *   scale    one byte per 32 content coordinates, b = X + 127 for 2^X,
 *            X = floor(log2 amax) - 8, clamped to [-127, 127] (-127 for an
 *            all-zero block), as in the OCP Microscaling format
 *   code     x / 2^X rounded to the nearest E4M3 value, ties to the even code,
 *            saturating at 448; sign bit = sign bit of x
 *   layout   an entry of dim coordinates, the last rope_dims of them rotary, is
 *            dim - rope_dims code bytes, (dim - rope_dims)/32 scale bytes and
 *            rope_dims bf16 values, in three arrays indexed by the same row
 * Every dequantized value is a bf16 number.
 *
 * csa_quantize_entries_fp8 -- store n entries x [n, dim] bf16:
 *   codes [n, dim - rope_dims] uint8, scales [n, (dim - rope_dims)/32] uint8,
 *   rope [n, rope_dims] bf16 (NULL when rope_dims == 0)
 * dim and rope_dims multiples of 8, rope_dims < dim, (dim - rope_dims) % 32 == 0;
 * x, codes and rope 16-byte aligned.  Bit-exact.
 */
csa_status_t csa_quantize_entries_fp8(const csa_bf16* x, int64_t n, int32_t dim, int32_t rope_dims,
                                      uint8_t* codes, uint8_t* scales, csa_bf16* rope,
                                      csa_stream_t stream);

/*
 * csa_sparse_attn_decode_fp8 -- csa_sparse_attn_decode over mixed-precision
 * entries: the attention of each query over its selected entries
 * (dequantized, exactly bf16) and its bf16 window rows, with the same
 * arguments, workspace (csa_sparse_attn_decode_workspace_size) and outputs.
 *   kv_codes   cache whose rows are 128 - rope_dims code bytes (data 16-byte aligned)
 *   kv_scales  [kv_codes->n_rows, (128 - rope_dims)/32] uint8
 *   kv_rope    [kv_codes->n_rows, rope_dims] bf16 (16-byte aligned), or NULL when
 *              rope_dims == 0; row r of each array belongs to physical row r
 * d = 128; rope_dims a multiple of 8 with 128 - rope_dims a multiple of 32.  The
 * attention kernel follows csa_set_attention_kernel: the tcgen05 kernel's
 * producer warps (or the mma.sync kernel's gather) expand each entry's codes
 * exactly to bf16 in shared memory, so the result equals that kernel's over a
 * bf16 cache holding the dequantized entries, bit for bit.
 */
csa_status_t csa_sparse_attn_decode_fp8(const csa_bf16* q, const csa_cache_t* kv_codes,
                                        const uint8_t* kv_scales, const csa_bf16* kv_rope,
                                        int32_t rope_dims, const csa_bf16* win,
                                        const int32_t* win_len, const int32_t* idx,
                                        const int32_t* count, int32_t B, int32_t H, int32_t d,
                                        int32_t top_k, int32_t window, float sm_scale,
                                        const float* sink, csa_bf16* out, float* lse, void* ws,
                                        size_t ws_bytes, csa_stream_t stream);

/*
 * hca_attn -- dense attention over every eligible heavily compressed entry
 * s < floor(t_i/m) plus the window, one softmax (Ch.7 "Dense attention over
 * heavily compressed history").
 *   Decode (win_len != NULL): query i sits at position q_pos[i] (required) and
 *     its window is kv_win[i, 0..win_len[i]-1] ([T, window, d], oldest first,
 *     itself last); it reads the compressed entries of sequence seq_id[i], or
 *     of sequence i when seq_id is NULL.
 *   Prefill (win_len == NULL), one sequence (seq_id NULL): every query reads
 *     sequence 0; query i sits at position q_pos[i] (or i if q_pos is NULL);
 *     kv_win is that sequence's raw tokens [*, d] and the window is rows
 *     max(0,t-W+1) .. t.
 *   Prefill, packed sequences (seq_id given): the T queries are the tokens of
 *     several sequences laid end to end; query i reads sequence seq_id[i]'s
 *     entries, sits at position q_pos[i] within it (required) and is raw row i
 *     of kv_win [T, d], so its window is rows i-n+1 .. i with
 *     n = min(W, q_pos[i] + 1).  Those rows must belong to the same sequence
 *     (the caller's layout); a window that would start before row 0 is cut
 *     there and recorded in the workspace header.
 *   max_entries bounds floor(t_i/m) (split layout); q [T, H, d]; out [T, H, d];
 *   lse [T, H] or NULL; sink [H] or NULL; seq_id [T] int32 or NULL;
 *   qrope query prologue / output epilogue (csa_qrope_t), or NULL.
 */
csa_status_t hca_attn(const csa_bf16* q, const csa_cache_t* kv_comp, const csa_bf16* kv_win,
                      const int32_t* win_len, const int32_t* seq_id, const int64_t* q_pos,
                      int64_t T, int32_t H, int32_t d, int32_t m, int64_t max_entries,
                      int32_t window, float sm_scale, const float* sink, csa_bf16* out,
                      float* lse, void* ws, size_t ws_bytes, csa_stream_t stream,
                      const csa_qrope_t* qrope);

#ifdef __cplusplus
}
#endif
#endif /* CSA_H */
