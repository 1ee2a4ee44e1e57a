/*
 * kvq.h -- C ABI of a B200 (sm_100a) library for decode-step attention over a
 * prunable 2-bit KV cache, following "Dual-QK: Sharp Queries and Flat Keys for
 * Prunable 2-bit KV Caches" (§3.1 dual transforms, §3.2 dynamic query-channel
 * pruning, §3.3 INT2 KV quantization and channel-major page layout, §3.4 one
 * global softmax across the cache).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor arguments are DEVICE pointers to caller-owned memory.  The
 *    library allocates nothing and keeps no global state; it is safe to call
 *    from several host threads on different caches or streams.
 *  - Every call is asynchronous on the given stream (NULL = legacy default
 *    stream).  A return of KVQ_OK means the work was validated and enqueued;
 *    results are ready when the stream reaches that point.
 *  - Calls that use the same cache must be ordered on one stream (or by
 *    events): they share its pages, lengths and status counters.
 *  - Argument errors are found on the host before anything is launched and
 *    reported as a negative status; nothing is enqueued then.  Conditions
 *    only the device can see (a sequence that would overflow its capacity)
 *    set a sticky flag in the cache's device status word and leave the data
 *    untouched; read it with kvq_read_status().
 *  - Head dimension d = 128 and quantization groups of 32 or 128 channels
 *    are the supported shapes; other values return KVQ_ERR_SHAPE.
 *  - Tensors are dense, row-major, innermost dimension last, with the
 *    shapes given per argument.  Float inputs are either float32 or bf16
 *    (bit patterns in uint16), chosen by a KVQ_DTYPE_* argument.
 *
 * Cache format (one "page" = 128 tokens of one (sequence, KV head))
 * ------------------------------------------------------------------
 *  rowbytes R = 128 * bits / 8   (32 for INT2, 64 for INT4)
 *  groups per token ng = 128 / group: 4 (groups of 32 channels) or 1 (the
 *  pages' own format, Dual-QK §3.3: one grid per token and KV head)
 *  offset 0        key codes, 128 rows x R bytes, row r = transformed key
 *                  channel r; row 0 is unused and stays zero
 *  offset 128R     value codes, 128 rows x R bytes, row r = value channel r
 *  offset 256R     channel 0 of the transformed key, 128 x bf16
 *  offset 256R+256 key metadata: 128 ng words {fp16 scale (low half), fp16 zero}
 *  +512 ng         value metadata, same shape
 *  Metadata word of token t (0..127), group g (0..ng-1):
 *      128 g + 4 sw(g, t / 4) + t % 4,   sw(g, c) = c XOR ((c / 8) XOR 4 (g % 2))
 *  i.e. each group's 32 chunks of 4 tokens are stored XOR-permuted within
 *  blocks of 8 chunks (a layout that lets the decode kernels read metadata
 *  without shared-memory bank conflicts after a contiguous copy).
 *  page bytes = 256R + 256 + 1024 ng (12544 / 20736 for INT2 / INT4 with
 *  groups of 32; 9472 / 17664 with one grid per token)
 *  Code of token t (0..127) of a page: byte t*bits/8 of its row, bit
 *  (t mod (8/bits))*bits, least significant first.  Key group g is channels
 *  max(1, g group) .. (g+1) group - 1 (channel 0 is kept in bf16 and left out
 *  of the range); value group g is channels g group .. (g+1) group - 1.
 *  With buckets (cache->bucket = w > 0) the key of position n is stored in
 *  the frame of its bucket b = n / w (Dual-QK §3.4): its anchor's rotary
 *  rotation removed, then the key transform, K' = (k T_b) A, where for
 *  i < 64 (channel i paired with channel i + 64, the rotate-half layout)
 *      (k T_b)[i]      = k[i] cos_bi + k[i+64] sin_bi
 *      (k T_b)[i + 64] = k[i+64] cos_bi - k[i] sin_bi
 *  in float64, each product rounded, then the sum or difference.
 *  Pages of one (sequence b, KV head h) are contiguous; unit (b, h) starts at
 *  byte ((b * n_kv_heads + h) * (capacity / 128)) * page_bytes.
 *  Dequantized value = scale * code + zero.
 *
 * Protected BF16 tier (optional; Dual-QK §3.3 keeps the first 64 and the most
 * recent 256 tokens in BF16 for keys and values, with the same query-channel
 * mask, §3.4 one softmax over all tiers)
 * ---------------------------------------------------------------------------
 *  With n_sink + n_recent > 0 the page array is followed, per unit (b, h) in
 *  the same order, by n_sink + n_recent slots of 512 bytes: 128 bf16 values of
 *  the transformed key, then 128 bf16 values of the value (round to nearest
 *  even).  Position p owns slot p if p < n_sink, else slot n_sink + p mod
 *  n_recent (a ring over the recent window).  Every appended token is coded in
 *  the pages as usual; a token is also written to its slot if p < n_sink or
 *  if it is among the last n_recent tokens once the append completes.  For a
 *  sequence of length L, positions [0, min(n_sink, L)) and
 *  [max(min(n_sink, L), L - n_recent), L) are read from their slots and all
 *  others from the codes.
 *  Bytes of token positions at or beyond seq_len are zero in the pages (as
 *  kvq_cache_init leaves them; appends write each position once).
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *kvq_stream_t;   /* same type as cudaStream_t */

/* return codes */
enum {
    KVQ_OK = 0,
    KVQ_ERR_ARG = -1,        /* null pointer, negative count, unknown dtype    */
    KVQ_ERR_SHAPE = -2,      /* unsupported head_dim / group / bits / GQA ratio */
    KVQ_ERR_CAPACITY = -3,   /* request can never fit the cache's capacity      */
    KVQ_ERR_WORKSPACE = -4,  /* workspace pointer null or too small             */
    KVQ_ERR_CUDA = -5,       /* a CUDA runtime call or kernel launch failed     */
    KVQ_ERR_ALIGN = -6       /* a pointer is not aligned as documented          */
};

/* input element types */
enum { KVQ_DTYPE_F32 = 0, KVQ_DTYPE_BF16 = 1 };

/* device status flags (sticky; cleared by kvq_cache_init) */
enum {
    KVQ_DEV_CAPACITY = 1u,   /* an append would have overflowed a sequence           */
    KVQ_DEV_TIMEOUT = 2u,    /* a bounded wait for an asynchronous copy gave up; the
                                result of that call is not valid                    */
    KVQ_DEV_INDEX = 4u       /* a decode got a channel list that is not channel 0
                                followed by ascending channels in 1..127; it read
                                no key rows outside the page and its result is not
                                valid                                               */
};

/* Cache descriptor.  The struct itself is host memory; the pointers in it are
 * device memory owned by the caller. */
typedef struct {
    int32_t batch;        /* sequences B >= 1                                */
    int32_t n_kv_heads;   /* KV heads per sequence >= 1                      */
    int32_t head_dim;     /* must be 128                                     */
    int32_t group;        /* quantization group in channels: 32, or 128 (one
                             grid per token, the pages' format)              */
    int32_t bits;         /* code width: 2 (INT2) or 4 (INT4)                */
    int32_t capacity;     /* tokens per sequence, a positive multiple of 128 */
    void *pages;          /* kvq_cache_bytes() bytes, 256-byte aligned        */
    int32_t *seq_len;     /* [batch] tokens currently stored per sequence    */
    uint32_t *status;     /* kvq_status_words() words, 4-byte aligned: word 0
                             holds the KVQ_DEV_* flags, the rest are
                             completion counters the calls use to finish a
                             step in the same kernel; every call leaves them
                             at zero (kvq_cache_init zeroes them)           */
    int32_t n_sink;       /* protected BF16 tier: first tokens kept, >= 0     */
    int32_t n_recent;     /* and most recent tokens kept, >= 0; together at
                             most KVQ_MAX_PROTECTED (0 and 0: no tier)       */
    const double *v_rot;  /* value rotation (Dual-QK §3.3, App. B.2), or NULL
                             for none: [n_kv_heads][128][128] float64,
                             row-major, 16-byte aligned, orthogonal, device
                             memory.  Appends store V Rv (coded and in the
                             protected slots); decodes aggregate in that basis
                             and return out = o Rv^T                        */
    double v_clip;        /* clipping ratio of the value grids, in (0, 1]
                             (the pages use 0.92 with rotated values); 0 means
                             1, no clipping.  Keys are never clipped.        */
    int32_t bucket;       /* bucket-relative RoPE (Dual-QK §3.4, App. C.4):
                             tokens per bucket w, a positive multiple of 128,
                             or 0 for none.  Bucket b holds positions
                             [b w, (b+1) w) and has the anchor a_b = b w.   */
    const double *rope;   /* with buckets: the anchors' rotary table,
                             [kvq_num_buckets()][64][2] float64 {cos(a_b
                             theta_i), sin(a_b theta_i)} with the model's
                             rotary frequencies theta_i (any scaling such as
                             YaRN included), 16-byte aligned, device memory */
} kvq_cache;

/* Largest n_sink + n_recent. */
#define KVQ_MAX_PROTECTED 1024

/* Buckets of a cache: ceil(capacity / bucket), or 1 without buckets (0 if
 * the descriptor is invalid).  Every channel-selection array has one entry
 * per bucket: idx [batch][n_kv_heads][nb][k], qsel [batch][n_q_heads][nb][k],
 * qgsum [batch][n_q_heads][nb][4]. */
int kvq_num_buckets(const kvq_cache *cache);

/* Words of the cache's status array: 1 + batch + batch * n_kv_heads
 * (0 if an argument is below 1). */
size_t kvq_status_words(int batch, int n_kv_heads);

/* Bytes of one 128-token page for the given code width and group size (0 if
 * unsupported). */
size_t kvq_page_bytes(int bits, int group);

/* Bytes of the whole page array of a cache, protected slots included (0 if
 * the descriptor is invalid). */
size_t kvq_cache_bytes(const kvq_cache *cache);

/* Zero every page, every seq_len entry and the status array (stream-ordered).
 * Returns KVQ_ERR_ARG / KVQ_ERR_SHAPE / KVQ_ERR_ALIGN on a bad descriptor. */
int kvq_cache_init(const kvq_cache *cache, kvq_stream_t stream);

/*
 * kvq_append -- quantize n_new tokens per (sequence, KV head) into the cache
 * at positions seq_len[b] .. seq_len[b]+n_new-1, then advance seq_len[b].
 * Dual-QK §3.1 (keys multiplied by the fixed transform, K' = K A), §3.3
 * (channel 0 of K' kept as bf16 and excluded from the range; the other key
 * channels and all value channels quantized per token with an asymmetric
 * min/max grid, round to nearest; channel-major 128-token pages), App. B.2
 * (values rotated by cache->v_rot and their grids clipped by cache->v_clip),
 * §3.4 (with buckets, K' = (K T_b) A in the frame of the token's bucket).
 *
 *  K, V    [batch][n_kv_heads][n_new][128], dtype KVQ_DTYPE_F32 or _BF16
 *  A       [n_kv_heads][128][128] float64, row-major, 16-byte aligned:
 *          K'[j] = sum_c K[c] A[c][j]
 *          summed c = 0..127 as a chain of fused multiply-adds from 0.0
 *  Arithmetic (defines the stored bits): K' in float64; per token and group
 *  zero = fp16(min), scale = fp16((max-min)/(2^bits-1)) (fp16 rounding to
 *  nearest even from float64), code = clamp(rint((x - zero)/scale), 0,
 *  2^bits-1) in float64, or 0 when scale == 0; channel 0 -> bf16 (nearest
 *  even from float64).  Values: with v_rot, x = (V v_rot)[j] by the same
 *  fma chain as K'; with a clip ratio r the value grids use min' = r*min and
 *  max' = r*max (each product rounded to float64) in place of min and max.
 *  Bits of other tokens sharing a code byte are kept.
 *  Values must stay within the fp16 range after the transform.
 *  A sequence whose seq_len + n_new would exceed capacity is left untouched
 *  and sets KVQ_DEV_CAPACITY.  n_new == 0 is a no-op.
 *  Errors: KVQ_ERR_ARG (null pointer, n_new < 0, bad dtype), KVQ_ERR_SHAPE,
 *  KVQ_ERR_CAPACITY (n_new > capacity), KVQ_ERR_CUDA.
 */
int kvq_append(const kvq_cache *cache, const void *K, const void *V, int dtype,
               int n_new, const double *A, kvq_stream_t stream);

/* k = ceil((1 - sparsity) * head_dim) (with a 1e-9 guard), the number of key
 * channels kept per KV head, channel 0 included.  Returns -1 if sparsity is
 * outside [0, 1) or head_dim < 1.  Dual-QK §4.1 (x% query-channel sparsity). */
int kvq_num_selected(float sparsity, int head_dim);

/*
 * kvq_select_channels -- transform the decode query and choose the key
 * channels to read.  Dual-QK §3.1 (queries multiplied by the paired inverse
 * transpose, q' = q A^{-T}, so q'.K' = q.K), §3.2 Eq. 4 (energy pooled over
 * the g = n_q_heads / n_kv_heads query heads of a KV head, e_j^2 =
 * sum_h q'_{h,j}^2; one mask per KV head); channel 0 is always kept.
 * §3.3 / App. C.2 (diagonal refinement): when Ainvt is a base transform times
 * a positive diagonal D (and A the base key transform times D^{-1}), pass D
 * as delta; the energies are then those of the base queries,
 * u_{h,j} = q'_{h,j} / delta_j (one float64 division), e_j^2 = sum_h u_{h,j}^2,
 * while qsel / qgsum keep q'.  §3.4 (bucket-relative RoPE): with buckets the
 * choice is made per bucket b that holds a token (b = 0, and b w < seq_len),
 * on the query moved into the bucket's frame, q'_b = (q T_b) Ainvt (T_b as
 * for keys), and written to entry b of idx / qsel / qgsum; entries of
 * buckets beyond the length are not written.
 *
 *  q       [batch][n_q_heads][128], dtype F32 or BF16; query head h belongs
 *          to KV head h / g
 *  Ainvt   [n_kv_heads][128][128] float64, row-major, 16-byte aligned:
 *          q'[j] = sum_c q[c] Ainvt[c][j]
 *          (fma chain over c from 0.0), e^2 by an fma chain over h ascending
 *  delta   [n_kv_heads][128] float64 positive finite (NULL: no refinement);
 *          other values give an unspecified but valid channel list
 *  idx     out [batch][n_kv_heads][nb][k] int32 (nb = kvq_num_buckets(), 1
 *          without buckets): channel 0 and the k-1 channels of
 *          1..127 with the largest e^2 (ties to the lower index), ascending
 *  qsel    out [batch][n_q_heads][nb][k] float32: q'[h][idx[i]] rounded to fp32
 *  qgsum   out [batch][n_q_heads][nb][4] float32: per key group, the float64 sum
 *          of q'[h][c] over selected c != 0 of that group (ascending c),
 *          rounded to fp32 (the zero-point term of the dequantized dot); with
 *          one grid per token entry 0 holds the one sum and entries 1..3 are 0
 *  k_out   out (HOST int*, may be NULL): k
 *  Errors: KVQ_ERR_ARG (null, sparsity outside [0,1)), KVQ_ERR_SHAPE
 *  (n_q_heads not a multiple of n_kv_heads, or g > 32), KVQ_ERR_CUDA.
 */
int kvq_select_channels(const kvq_cache *cache, const void *q, int dtype,
                        int n_q_heads, const double *Ainvt, const double *delta, float sparsity,
                        int32_t *idx, float *qsel, float *qgsum, int *k_out,
                        kvq_stream_t stream);

/* Workspace bytes kvq_decode_attn and kvq_decode_step need for this cache on
 * the CURRENT device (the split over the context is sized by the device's SM
 * count): the split partials, and for INT2 with 4 query heads per KV head
 * also the decode step's page plans, one per (sequence, KV head, RoPE
 * bucket).  0 if the arguments are invalid. */
size_t kvq_decode_workspace(const kvq_cache *cache, int n_q_heads, int k);

/*
 * kvq_decode_attn -- attention of one decode query per head over every
 * cached token, reading only the selected key channels.  Dual-QK §3.2 (scores
 * use the retained channels, scaled by 1/sqrt(128) with the full dimension),
 * §3.3 (only key rows holding selected channels are fetched -- in 64-byte
 * chunks of two rows, the unit the memory system fetches; values and
 * metadata are read in full), §3.4 (one softmax over all tokens, then value
 * aggregation).  Realised as a split over the context (flash-decoding): per
 * split a running max, sum and output, then one exact merge.
 *
 *  score_h(t) = [qsel_h0 * ch0(t) + sum_g (scale_g(t) * sum_{c in S_g}
 *               qsel_hc * code_c(t) + zero_g(t) * qgsum_hg)] / sqrt(128)
 *  out     [batch][n_q_heads][128] float32 = sum_t p_h(t) v_hat(t) / sum_t p_h(t)
 *          (zeros for a sequence with no tokens); with cache->v_rot set the
 *          aggregate is rotated back (Dual-QK §3.3), out = o v_rot^T, in
 *          float64 over the 128 channels from the float32 merged sums
 *  idx, qsel, qgsum, k exactly as produced by kvq_select_channels; with
 *          buckets, token t is scored with the entries of its bucket t / w
 *          (one softmax over all buckets and tiers, §3.4)
 *  ws      device workspace of at least kvq_decode_workspace() bytes,
 *          16-byte aligned; contents need no initialisation
 *  Arithmetic: float32 accumulation of tensor-core products of exact small
 *  integers with the query as a float16 hi + lo pair and the softmax weights
 *  as float16 (INT2, 4 query heads per KV head), or of CUDA-core float32
 *  products (other shapes).
 *  Errors: KVQ_ERR_ARG, KVQ_ERR_SHAPE, KVQ_ERR_WORKSPACE, KVQ_ERR_ALIGN,
 *  KVQ_ERR_CUDA.
 */
int kvq_decode_attn(const kvq_cache *cache, int n_q_heads, const int32_t *idx,
                    const float *qsel, const float *qgsum, int k, float *out,
                    void *ws, size_t ws_bytes, kvq_stream_t stream);

/*
 * kvq_decode_attn_wait_bound -- kvq_decode_attn with an explicit bound on each
 * wait of the tensor-core decode for a staged page (INT2, 4 query heads per
 * KV head, the shapes that decode runs on; other shapes return
 * KVQ_ERR_SHAPE).  A fault-handling hook, not part of the method: the pages
 * describe no failure path.  kvq_decode_attn waits up to about a million
 * polls per stage.  With wait_polls = 0 a wait gives up at once unless the
 * page has already landed.  A wait that gives up sets KVQ_DEV_TIMEOUT; its
 * pair of warps then issues no further copy, waits for the copies already in
 * flight to land, and finishes, so the call leaves the cache, the counters
 * and the GPU ready for the next call, but its `out` is not valid.
 * Same arguments and errors as kvq_decode_attn otherwise.
 */
int kvq_decode_attn_wait_bound(const kvq_cache *cache, int n_q_heads, const int32_t *idx,
                               const float *qsel, const float *qgsum, int k, float *out,
                               void *ws, size_t ws_bytes, uint32_t wait_polls, kvq_stream_t stream);

/*
 * kvq_decode_step -- one whole decode step: kvq_append of the n_new new
 * tokens, kvq_select_channels of the query, then kvq_decode_attn over every
 * token including the new ones.  Same arguments, results and errors as those
 * three calls made in that order on `stream` (idx / qsel / qgsum are written
 * too), and the same stored bits.  With INT2 codes, 4 query heads per KV head,
 * n_new <= 4 and no buckets the step is one kernel launch: each CTA repeats
 * the channel choice of its (sequence, KV head) with the same float64
 * arithmetic, and the CTA holding the last page appends the new tokens before
 * reading it.  With buckets it is three launches, each a programmatic
 * dependent of the one before: the append (the length not yet advanced), the
 * channel choice of every bucket with the decode's page plans (written into
 * `ws`), and the decode, which advances the length.
 *
 *  q       [batch][n_q_heads][128]; k_new, v_new [batch][n_kv_heads][n_new][128];
 *          all of dtype KVQ_DTYPE_F32 or _BF16
 *  A, Ainvt, delta  as for kvq_append / kvq_select_channels (16-byte aligned)
 *  idx, qsel, qgsum  outputs as for kvq_select_channels
 *  out, ws, ws_bytes  as for kvq_decode_attn (kvq_decode_workspace() with the
 *          k of `sparsity`)
 *  Errors: the union of the three calls' errors.
 */
int kvq_decode_step(const kvq_cache *cache, const void *q, const void *k_new,
                    const void *v_new, int dtype, int n_q_heads, int n_new,
                    const double *A, const double *Ainvt, const double *delta, float sparsity,
                    int32_t *idx, float *qsel, float *qgsum, float *out,
                    void *ws, size_t ws_bytes, kvq_stream_t stream);

/* Workspace bytes for kvq_bf16_decode_attn on the current device. */
size_t kvq_bf16_decode_workspace(int batch, int n_q_heads, int n_kv_heads, int n_tokens);

/*
 * kvq_bf16_decode_attn -- the unpruned, unquantized comparator: plain
 * softmax(q K^T / sqrt(128)) V per query head over n_tokens bf16 keys and
 * values (what Dual-QK compares against as "unpruned BF16", §4.4).
 *  q       [batch][n_q_heads][128] bf16
 *  K, V    [batch][n_kv_heads][n_tokens][128] bf16 (original coordinates),
 *          16-byte aligned; may be NULL when n_tokens == 0
 *  out     [batch][n_q_heads][128] float32
 *  ws      at least kvq_bf16_decode_workspace() bytes, 16-byte aligned
 * Arithmetic in float32.  Errors as for kvq_decode_attn.
 */
int kvq_bf16_decode_attn(const void *q, const void *K, const void *V, int batch,
                         int n_q_heads, int n_kv_heads, int n_tokens, float *out,
                         void *ws, size_t ws_bytes, kvq_stream_t stream);

/*
 * kvq_decode_attn_static -- kvq_decode_attn for callers that cannot allocate
 * device memory at call time (for example a plugin inside an inference engine
 * that owns all device memory and offers no scratch buffer, or a decode loop
 * that must not call cudaMalloc, which may synchronise the device).  The
 * paper has no counterpart; this is a deployment convenience.
 *
 * Same arguments, arithmetic and result as kvq_decode_attn, without ws /
 * ws_bytes: the split partials live in one static device array of
 * kvq_decode_static_scratch_bytes() bytes (4 MiB) that every GPU loading this
 * library holds until the process exits.  The library allocates nothing.
 *  - The first call on a device, with that device current, looks up the
 *    array's device address (cudaGetSymbolAddress) and caches it; make that
 *    first call before any stream capture.  The cached address is never
 *    refreshed: after cudaDeviceReset() on a device (which unloads the
 *    library's device code there) do not call this entry point again on that
 *    device in the same process.
 *  - All calls share the one array, and it keeps the last call's contents.
 *    Nothing in it needs to start at zero.  Calls whose kernels can overlap
 *    on the GPU (different streams, or different host threads) race on it:
 *    serialise them.
 *  - A request needing more than the maximum (kvq_decode_workspace() >
 *    kvq_decode_static_scratch_bytes()) returns KVQ_ERR_WORKSPACE and
 *    launches nothing.
 * Errors: as kvq_decode_attn, plus KVQ_ERR_CUDA if the address lookup fails.
 */
size_t kvq_decode_static_scratch_bytes(void);
int kvq_decode_attn_static(const kvq_cache *cache, int n_q_heads, const int32_t *idx,
                           const float *qsel, const float *qgsum, int k, float *out,
                           kvq_stream_t stream);

/*
 * kvq_copy_async -- stream-ordered copy of `bytes` bytes between caller
 * buffers, device memory or pinned host memory, the direction taken from the
 * pointers (unified addressing).  For moving a decode step's packed inputs in
 * and its result out as one transfer each; with pinned host buffers the copy
 * can be recorded into a CUDA graph together with the step.  The paper has no
 * counterpart; this is a serving convenience.
 * Errors: KVQ_ERR_ARG (null pointer with bytes > 0), KVQ_ERR_CUDA.
 */
int kvq_copy_async(void *dst, const void *src, size_t bytes, kvq_stream_t stream);

/* Copy the device status flags (word 0) into *flags (synchronises the stream).
 * KVQ_ERR_ARG on null pointers, KVQ_ERR_CUDA on a failed copy. */
int kvq_read_status(const kvq_cache *cache, uint32_t *flags, kvq_stream_t stream);

/* Static description of a status code. */
const char *kvq_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int kvq_version(void);

#ifdef __cplusplus
}
#endif
#endif /* KVQ_H */
