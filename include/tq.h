/*
 * tq.h -- C ABI of libtq: TurboQuant KV-cache compression and attention over
 * the compressed cache, on one NVIDIA B200 (sm_100a).
 *
 * The method (turboquant-plus-rs 0.1.0 README, "Architecture" and "Key
 * ideas"): every key/value head vector is rotated by a seeded random
 * rotation (fast Walsh-Hadamard with random signs), scalar-quantized per
 * coordinate against the Lloyd-Max codebook of the post-rotation Gaussian
 * with norm extraction and correction (PolarQuant: b-1 bits for keys, b bits
 * MSE-only for values), and for keys the residual gets a 1-bit QJL sign
 * sketch.  Attention scores are estimated from the packed codes.  The call
 * shapes follow bitpolar 0.3.3 src/kv_cache.rs (KvCacheConfig {head_dim,
 * bits, projections, seed}; KvCacheCompressor::push, attention_scores,
 * decode_values; MultiHeadKvCache with seed + h per head).
 *
 * Conventions for every entry point:
 *  - All tensor arguments are DEVICE pointers owned by the caller, on the
 *    device that was current when the context was created.  The library
 *    never frees or keeps them past the call.  A context owns only its small
 *    device tables (signs, QJL matrix, codebooks) and a status word.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every call enqueues its kernels on that stream and returns
 *    without synchronizing, except tq_get_status and tq_ensure_heads.
 *  - Argument errors are detected on the host before anything is enqueued
 *    and returned as tq_status; nothing runs in that case.
 *  - There is no CPU fallback: if the device is not an sm_100 GPU or the
 *    kernels cannot launch, the call returns TQ_ERR_DEVICE / TQ_ERR_CUDA.
 *  - Threads: different contexts may be used from different host threads at
 *    once.  Calls on one context from several threads must be serialized
 *    by the caller when any of them may build head tables (tq_ensure_heads,
 *    or a call using more heads than built so far).
 *  - d = head_dim, m = projections, b = bits, B_K = b-1, B_V = b.
 *
 * Packed row formats (the pages give no layout; this is the library's):
 *  K row (k_row_bytes = B_K*d/8 + m/8 + 8):
 *    B_K index bit planes of d/8 bytes (plane p holds bit p of the index of
 *    coordinate j at byte j/8, bit j%8), then the m-bit QJL sign plane
 *    (projection i at byte i/8, bit i%8; 1 = non-negative), then n_s
 *    (float32, the corrected norm), then gamma (float32, the residual norm).
 *    With binary16 key norms (tq_create_format, TQ_NORMS_F16) the tail is
 *    one 32-bit word instead: n_s and gamma rounded to binary16 (ties to
 *    even), n_s in the low half; k_row_bytes = B_K*d/8 + m/8 + 4.
 *  V row (v_row_bytes = B_V*d/8 + 4):
 *    B_V-bit index fields, coordinate j at bit B_V*j of a little-endian bit
 *    stream, then n_s (float32).
 *  Indices count the codebook boundaries at or below z = sqrt(d)*Pi*x/|x|.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tq_status {
    TQ_OK = 0,
    TQ_ERR_NULL = 1,          /* a required pointer is NULL */
    TQ_ERR_ZERO_DIM = 2,      /* head_dim == 0 (bitpolar ZeroDimension) */
    TQ_ERR_DIM = 3,           /* head_dim not 64, 128 or 256, or 256 with the Haar rotation
                                 (bitpolar OddDimension, generalized) */
    TQ_ERR_BITS = 4,          /* bits not in 2..5 (bitpolar InvalidBitWidth) */
    TQ_ERR_ZERO_PROJ = 5,     /* projections == 0 (bitpolar ZeroProjections) */
    TQ_ERR_PROJ = 6,          /* projections not a multiple of 32 in [32, 256] ([32, 192] at
                                 head_dim 256) */
    TQ_ERR_EMPTY = 7,         /* zero heads or zero batch (bitpolar EmptyInput) */
    TQ_ERR_DIM_MISMATCH = 8,  /* shapes disagree: H_q % H_kv, tokens beyond capacity,
                                 capacity not a multiple of 16 (bitpolar DimensionMismatch) */
    TQ_ERR_WORKSPACE = 9,     /* workspace NULL or smaller than tq_decode_workspace_bytes */
    TQ_ERR_ALIGN = 10,        /* a pointer or stride breaks the stated alignment */
    TQ_ERR_CUDA = 11,         /* a CUDA runtime call failed (see tq_last_cuda_error) */
    TQ_ERR_DEVICE = 12,       /* current device is not compute capability 10.0 */
    TQ_ERR_LIMIT = 13         /* a count exceeds a documented maximum (segments, heads) */
} tq_status;

typedef enum tq_dtype { TQ_F32 = 0, TQ_F16 = 1, TQ_BF16 = 2 } tq_dtype;
typedef enum tq_which { TQ_KEYS = 0, TQ_VALUES = 1, TQ_BOTH = 2 } tq_which;

/* The random rotation Pi (turboquant-plus-rs README, Architecture and
 * Modules: rotation -- either a Haar-random orthogonal matrix or a fast
 * Walsh-Hadamard transform with random signs). */
/* Storage of the two key-row norms (turboquant-plus-rs README,
 * "Compression formats": turbo4 is 4.25 bits per value, which binary16
 * norms give a key row at b = 4, d = m = 128). */
typedef enum tq_norm_format {
    TQ_NORMS_F32 = 0,      /* n_s, gamma as float32 (8 bytes) */
    TQ_NORMS_F16 = 1       /* n_s, gamma as binary16 in one 32-bit word */
} tq_norm_format;

typedef enum tq_rotation {
    TQ_ROT_HADAMARD = 0,   /* Pi = H D / sqrt(d): Sylvester Walsh-Hadamard, random signs D */
    TQ_ROT_HAAR = 1        /* Pi = Q: orthogonal factor of the QR of a d x d Gaussian matrix,
                              R's diagonal positive (Haar-distributed) */
} tq_rotation;

typedef struct tq_ctx tq_ctx;

/* A packed cache: two device buffers laid out [batch][n_kv_heads][capacity]
 * rows of k_row_bytes / v_row_bytes.  Either pointer may be NULL when the
 * call does not touch it.  capacity must be a multiple of 16 and the
 * buffers 16-byte aligned, so every (batch, head) block starts 16-byte
 * aligned.  Sized by tq_packed_bytes. */
typedef struct tq_codes {
    void *k;
    void *v;
    int32_t batch;
    int32_t n_kv_heads;
    int64_t capacity;
} tq_codes;

/* One segment of compressed keys/values that a contiguous range of
 * sequences attends to (shared prefixes appear once with n_seqs > 1; a
 * sequence's private tail has n_seqs = 1).  Tokens [0, n_tokens) of batch
 * slot `codes_batch` of `codes` are read.  Different segments may use
 * different contexts (bit widths, seeds). */
typedef struct tq_segment {
    const tq_ctx *ctx;
    tq_codes codes;
    int32_t codes_batch;
    int32_t first_seq;
    int32_t n_seqs;
    int32_t reserved;
    int64_t n_tokens;
} tq_segment;

#define TQ_MAX_SEGMENTS 64
#define TQ_MAX_HEADS 1024

/* Create a codec context on the current CUDA device: KvCacheConfig {head_dim,
 * bits, projections, seed} of bitpolar src/kv_cache.rs, where `bits` is the
 * total TurboQuant width b (keys: b-1 PolarQuant bits + 1 QJL bit; values: b
 * MSE bits; turboquant-plus-rs "Architecture").  Builds the Lloyd-Max
 * codebooks on the host and uploads them.  Head tables are built by
 * tq_ensure_heads (or on first use).  head_dim in {64, 128, 256}; bits in
 * 2..5; projections a multiple of 32 in [32, 256], at most 192 when head_dim
 * is 256 (the key encoder's S tile and residual operand share 227 KB of
 * shared memory).  On success *out owns device memory released by
 * tq_destroy.  Synchronous. */
tq_status tq_create(int head_dim, int bits, int projections, uint64_t seed, tq_ctx **out);

/* tq_create with a choice of rotation.  TQ_ROT_HADAMARD is tq_create.
 * TQ_ROT_HAAR: head h's rotation is Q from the QR factorization of a d x d
 * matrix of N(0,1) Box-Muller draws that continue head h's SplitMix64
 * stream (seed + h) after the d sign draws and the m*d (rounded up to even)
 * draws of S; Q's columns are signed so that R has a positive diagonal.  The
 * rows are rotated on the tensor cores: binary16 and bfloat16 rows as they
 * are, against sqrt(d) Q split into 2 binary16 or 3 bfloat16 pieces of the
 * row's own type (the TMA-fed encoder); float32 rows, and bfloat16 keys with
 * more than 136 projections (whose three pieces leave too little shared
 * memory), scaled by a power of two into binary16 range and split hi + lo,
 * against sqrt(d) Q as binary16 hi + lo.  Queries and outputs use fp32 Q.
 * Not available at head_dim 256 (TQ_ERR_DIM: the two binary16 pieces of
 * sqrt(d) Q alone fill 256 KB, above the 227 KB of shared memory a CTA can
 * hold).  Packed formats and every other call are unchanged.  In this mode a
 * row whose largest |x_j| is below 2^-100 is encoded as a zero row, and so is
 * a 16-bit row on the TMA-fed encoder whose d |x|^2 is below the smallest
 * normal float (as under the default rotation).  Returns TQ_ERR_DIM for an
 * unknown rotation. */
tq_status tq_create_ex(int head_dim, int bits, int projections, uint64_t seed, tq_rotation rotation,
                       tq_ctx **out);

/* tq_create_ex with a choice of key-norm storage.  TQ_NORMS_F32 is
 * tq_create_ex.  TQ_NORMS_F16: key rows store n_s and gamma rounded to
 * binary16 (ties to even) in one 32-bit word; indices and sign bits are
 * those of the float32 format, and scores, dequantization and decode read
 * the rounded norms.  A key row whose n_s or gamma rounds to binary16
 * infinity (>= 65520) is stored as a zero row and counted with the
 * non-finite rows (tq_get_status).  Value rows keep their float32 n_s.
 * Returns TQ_ERR_DIM for an unknown rotation or norm format. */
tq_status tq_create_format(int head_dim, int bits, int projections, uint64_t seed, tq_rotation rotation,
                           tq_norm_format key_norms, tq_ctx **out);

/* Release a context and its device tables (synchronizes the device). NULL is a no-op.
 * The counterpart of dropping a bitpolar KvCacheCompressor / MultiHeadKvCache
 * (bitpolar 0.3.3 src/kv_cache.rs): the context owns its codec state, the
 * caller owns the caches it filled. */
void tq_destroy(tq_ctx *ctx);

/* Build and upload the tables of heads 0..n_heads-1 (head h uses seed + h,
 * bitpolar MultiHeadKvCache::new): random signs of the rotation and the
 * m x d QJL matrix (binary16 entries).  Synchronous; idempotent.  Calls that
 * use more heads than built call this themselves, so make the first such
 * call before capturing a CUDA graph.  n_heads <= TQ_MAX_HEADS. */
tq_status tq_ensure_heads(tq_ctx *ctx, int n_heads);

/* Packed bytes per token-head row: K, V, or K+V for TQ_BOTH; 0 if ctx is NULL. */
int64_t tq_row_bytes(const tq_ctx *ctx, tq_which which);

/* Device bytes of a tq_codes buffer pair (or one side) for the given shape
 * (turboquant-plus-rs "Modules": memory footprint). */
size_t tq_packed_bytes(const tq_ctx *ctx, int batch, int n_kv_heads, int64_t capacity, tq_which which);

/* Encode n_tokens keys and/or values per (batch, head) into tokens
 * [token_offset, token_offset + n_tokens) of `codes` (bitpolar
 * KvCacheCompressor::push; MultiHeadKvCache::push_token).
 *  k, v   : device input, element (b, h, t, j) at base[b*stride_b + h*stride_h
 *           + t*stride_t + j] in `dtype`; either may be NULL to skip that side.
 *           Rows must be 16-byte aligned (strides multiples of 16 bytes).
 *  codes  : batch and n_kv_heads must equal the call's; token_offset +
 *           n_tokens <= capacity.  n_tokens == 0 is a no-op (k, v may be NULL).
 * Keys get PolarQuant at b-1 bits plus QJL signs (computed on tcgen05
 * tensor cores); values get PolarQuant at b bits.  Non-finite rows are
 * encoded as zero vectors and counted in the context's status word
 * (bitpolar NonFiniteInput), read with tq_get_status. */
tq_status tq_encode_kv(tq_ctx *ctx, const void *k, const void *v, tq_dtype dtype, int batch,
                       int n_kv_heads, int64_t n_tokens, int64_t stride_b, int64_t stride_h,
                       int64_t stride_t, const tq_codes *codes, int64_t token_offset, void *stream);

/* Pre-softmax scores of every query head against tokens [0, n_tokens) of its
 * kv head, estimated from the packed keys and scaled by 1/sqrt(d) (bitpolar
 * KvCacheCompressor::attention_scores):
 *   s = [n_s <Pi q, C[idx]>/sqrt(d) + sqrt(pi/2)/m gamma <S Pi q, 2 bit - 1>] / sqrt(d).
 *  q      : device float32 [codes->batch][n_q_heads][d].
 *  scores : device float32 [codes->batch][n_q_heads][n_tokens].
 * Query head j reads kv head j / (n_q_heads / n_kv_heads). */
tq_status tq_attention_scores(tq_ctx *ctx, const tq_codes *codes, const float *q, int n_q_heads,
                              int64_t n_tokens, float *scores, void *stream);

/* Reconstruct tokens [0, n_tokens) (bitpolar decode_values):
 *   v_hat = n_s Pi^T C[idx]/sqrt(d),
 *   k_hat = Pi^T (n_s C[idx]/sqrt(d) + sqrt(pi/2)/m gamma S^T (2 bit - 1)).
 *  k_hat, v_hat : device float32 [batch][n_kv_heads][n_tokens][d]; either may be NULL. */
tq_status tq_dequantize(tq_ctx *ctx, const tq_codes *codes, int64_t n_tokens, float *k_hat,
                        float *v_hat, void *stream);

/* Workspace bytes tq_decode_attention needs for this segment list. */
size_t tq_decode_workspace_bytes(const tq_segment *segs, int n_segs, int batch, int n_q_heads,
                                 int n_kv_heads);

/* Number of kernels one tq_decode_attention (or tq_decode_append) call with
 * this segment list launches on the current device: the query preparation,
 * one split-K decode launch per group of segments sharing bits, queries per
 * CTA, m and row length, and the combine step, which is left out when every
 * sequence is covered by exactly one segment holding tokens that the plan
 * does not split (the decode kernel then writes the output itself).  -1 if
 * the arguments are invalid.  Host-only; no device work. */
int tq_decode_launch_count(const tq_segment *segs, int n_segs, int batch, int n_q_heads, int n_kv_heads);

/* One decode step (bitpolar 0.3.3 src/kv_cache.rs: attention_scores gives the
 * pre-softmax scores q.K^T/sqrt(d) of the stored keys and decode_values the
 * stored values; turboquant-plus-rs README, Architecture: the inner product
 * is estimated from the codes; fib-quant README, C Kernels: compressed
 * attention logits followed by the softmax).  For every sequence b and
 * query head j,
 *   out[b][j] = sum_t softmax_t(s_t) v_hat_t
 * over the concatenation of all segments that sequence b attends to, with
 * s_t the score of tq_attention_scores.  Split-K over tokens: each work item
 * stages packed K/V tiles in shared memory, scores them through per-query
 * lookup tables, keeps an online softmax and the value sum in registers,
 * and shares each tile across the query heads of its kv-head group (GQA)
 * and across all sequences of a shared segment; a second kernel merges the
 * partials by log-sum-exp (left out when every sequence has one unsplit
 * segment: the decode kernel then writes the output).  A segment read by 16
 * or more queries per kv head (sequences x query heads of a group), with d
 * and m in {64, 128} and the Walsh-Hadamard rotation, is decoded on the
 * tensor cores instead: the queries are the rows of the score and value
 * MMAs, with q_rot, S q_rot, the centroids and the softmax weights split
 * into bfloat16 hi + lo parts (about 2^-16 relative error per product).
 * The environment variable TQ_DECODE_PATH, read at each call, overrides the
 * choice: "lut" keeps every segment on the lookup tables, "mma" sends every
 * segment that fits to the tensor cores.  The decode and merge kernels are
 * programmatic dependent launches: they may begin while the kernel before
 * them in the stream ends, and wait for it before reading its output.
 *  segs      : HOST array of n_segs (<= TQ_MAX_SEGMENTS) segments; every
 *              sequence in [0, batch) must be covered by at least one.
 *  q         : device [batch][n_q_heads][d] in q_dtype.
 *  out       : device [batch][n_q_heads][d] in out_dtype.
 *  workspace : device, >= tq_decode_workspace_bytes(...), 16-byte aligned;
 *              contents on entry are ignored. */
tq_status tq_decode_attention(const tq_segment *segs, int n_segs, const void *q, tq_dtype q_dtype,
                              int batch, int n_q_heads, int n_kv_heads, void *out,
                              tq_dtype out_dtype, void *workspace, size_t ws_bytes, void *stream);

/* One decode step that first appends the step's new key and value rows
 * (bitpolar MultiHeadKvCache::push_token followed by attention over the
 * cache; fib-quant README, "Streaming KV encoder": a cache built one token
 * at a time).
 * Sequence b's private tail -- the one segment with n_seqs == 1 and
 * first_seq == b -- receives the rows of b as token n_tokens (keys: b-1
 * PolarQuant bits + QJL signs; values: b bits; the same codes tq_encode_kv
 * produces for them, up to decisions within float rounding of a boundary)
 * and is attended over n_tokens + 1 tokens; every other argument and the
 * output are those of tq_decode_attention.  The encode runs inside the
 * step's query-preparation kernel, so the step launches the same kernels as
 * tq_decode_attention.
 *  k_new, v_new : device [batch][n_kv_heads][d] in kv_dtype (contiguous).
 *  Every sequence needs exactly one private tail with n_tokens < capacity
 *  (TQ_ERR_DIM_MISMATCH otherwise); tails must be distinct rows of memory.
 *  The segments are read, not modified: the caller advances each tail's
 *  n_tokens by one after the call.  Non-finite new rows are encoded as zero
 *  vectors and counted in the tail context's status word.
 *  workspace : >= tq_decode_append_workspace_bytes(...) bytes. */
tq_status tq_decode_append(const tq_segment *segs, int n_segs, const void *k_new, const void *v_new,
                           tq_dtype kv_dtype, const void *q, tq_dtype q_dtype, int batch, int n_q_heads,
                           int n_kv_heads, void *out, tq_dtype out_dtype, void *workspace, size_t ws_bytes,
                           void *stream);

/* Workspace bytes tq_decode_append needs (that of tq_decode_attention over
 * the segments with every tail one token longer); 0 on invalid arguments. */
size_t tq_decode_append_workspace_bytes(const tq_segment *segs, int n_segs, int batch, int n_q_heads,
                                        int n_kv_heads);

/* Bytes of the scratch array compiled into the library for
 * tq_decode_attention_static (8 MiB). */
#define TQ_STATIC_SCRATCH_BYTES (8u << 20)

/* Decode attention that allocates nothing.  The paper has no counterpart:
 * this entry point exists for callers that cannot call cudaMalloc -- for
 * example a plug-in living inside a host application that owns all device
 * memory through its own allocator and gives the plug-in no allocation
 * hook, or a serving loop that must not allocate on the decode path because
 * cudaMalloc may synchronize the device.  It computes exactly what
 * tq_decode_attention computes, with the same arguments minus the
 * workspace: the scratch (prepared queries and split-K partials) lives in a
 * fixed array of TQ_STATIC_SCRATCH_BYTES inside the library, which every GPU
 * that loads the library holds until the process exits.
 *  - Returns TQ_ERR_LIMIT if the call needs more scratch than
 *    TQ_STATIC_SCRATCH_BYTES (tq_decode_workspace_bytes gives the need), or
 *    if a segment's context has no tables yet for n_kv_heads heads (building
 *    them allocates; call tq_ensure_heads first).
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current.  The address is kept for the life of the
 *    process, per device number: only the device's primary context (the
 *    one the CUDA runtime uses) is supported, and the address is not looked
 *    up again after cudaDeviceReset.
 *  - Every call on a device shares the one array and it keeps the last
 *    call's contents; nothing in it needs clearing, because the decode writes
 *    every scratch value it later reads.  Calls that overlap on the GPU
 *    (unordered streams) race on the array and must be serialized by the
 *    caller.
 *  - Calls no cudaMalloc, cudaFree or allocating library routine. */
tq_status tq_decode_attention_static(const tq_segment *segs, int n_segs, const void *q, tq_dtype q_dtype,
                                     int batch, int n_q_heads, int n_kv_heads, void *out,
                                     tq_dtype out_dtype, void *stream);

/* Synchronize `stream` and read the context's status word: the number of
 * non-finite rows encoded so far, and device error flags (bit 0: a bounded
 * wait inside a kernel gave up; its outputs for that tile are invalid).
 * bitpolar 0.3.3 src/kv_cache.rs rejects a non-finite input row with
 * NonFiniteInput before it is stored; on the GPU the rows of one call are
 * encoded in parallel, so such rows are stored as zero vectors and counted
 * here instead of failing the call. */
tq_status tq_get_status(tq_ctx *ctx, void *stream, uint64_t *nonfinite_rows, uint32_t *error_flags);

/* Decode attention over an outlier/normal channel-split cache
 * (turboquant-plus-rs README, Modules: outlier -- a fractional bit rate from
 * coding outlier and normal channels at different widths).  A head's channels are split into an
 * outlier group (the first d_o channels, codec ctx_o) and a normal group (the
 * next d_n channels, codec ctx_n); each group is encoded with tq_encode_kv
 * of its own codec (e.g. 64 channels at b+1 bits and 64 at b: b + 1/2 index
 * bits per value), so the caller orders the channels outliers first.  For
 * every sequence b and query head j:
 *   s_t = q . k_hat_t / sqrt(d_o + d_n)  (k_hat_t: both groups' keys),
 *   out[b][j] = sum_t softmax_t(s_t) v_hat_t  (v_hat_t: both groups' values).
 *  codes_o, codes_n : the groups' caches, same batch, kv heads and capacity;
 *                     tokens [0, n_tokens) of batch slot b are sequence b's.
 *  q, out           : device [batch][n_q_heads][d_o + d_n], outliers first.
 *  workspace        : >= tq_decode_split_workspace_bytes(...), 16-byte aligned.
 * Query head j reads kv head j / (n_q_heads / n_kv_heads).  Launches five
 * kernels: the query's groups as fp32, each group's exact scores (the
 * tq_attention_scores kernel), a softmax-and-value kernel over chunks of
 * tokens, and the log-sum-exp merge of the chunks with each group's
 * unrotation. */
size_t tq_decode_split_workspace_bytes(const tq_ctx *ctx_o, const tq_ctx *ctx_n, int batch, int n_q_heads,
                                       int64_t n_tokens);
tq_status tq_decode_attention_split(tq_ctx *ctx_o, const tq_codes *codes_o, tq_ctx *ctx_n, const tq_codes *codes_n,
                                    int64_t n_tokens, const void *q, tq_dtype q_dtype, int batch, int n_q_heads,
                                    void *out, tq_dtype out_dtype, void *workspace, size_t ws_bytes, void *stream);

/* Failure-detection self-test (the paper has no counterpart): enqueue one
 * kernel that waits, bounded by timeout_us of wall time (1..100000), on an
 * mbarrier phase nothing completes, and records the timeout in the
 * context's status word exactly as the library's kernels do when one of
 * their waits runs out.  Afterwards tq_get_status reports error flag bit 0,
 * kernels of this context skip their work (key encode and decode; their
 * outputs are invalid) until tq_reset_status clears the word, and the
 * context is usable again.  No fault, trap or unbounded wait is involved.
 * TQ_ERR_LIMIT for a timeout outside the range. */
tq_status tq_selftest_wait_timeout(tq_ctx *ctx, uint32_t timeout_us, void *stream);

/* Zero the status word (enqueued on `stream`). */
tq_status tq_reset_status(tq_ctx *ctx, void *stream);

/* Human-readable name of a status code (static storage). */
const char *tq_status_string(tq_status s);

/* Message of the last CUDA error seen by this thread's libtq calls (static storage). */
const char *tq_last_cuda_error(void);

#ifdef __cplusplus
}
#endif
#endif /* TQ_H */
