/*
 * kvq.h -- C ABI of libkvq: an asymmetric low-bit KV cache with decode
 * attention that reads the packed cache directly, for NVIDIA B200 (sm_100a).
 *
 * The method (pages cited by title and section):
 *  - "KV cache compression: quantization, eviction and sparse attention"
 *    (arganzheng.life), section 3.2 "KIVI": keys are quantized per channel
 *    with the range taken over a group of G tokens, values per token with the
 *    range taken over the channels; the most recent tokens stay full
 *    precision until a whole group exists; attention over the quantized part
 *    and the window is computed separately and merged.  Section 3.4: with
 *    paged storage every 16-token block carries its own scales and the key
 *    group is aligned to the block.  Section 3.1: FP8 E4M3 with a static
 *    per-head scale, dequantized inside attention.
 *  - "KV Cache lab" (door4ai-lab), experiment 01 and jaedaily.cn "KV cache
 *    compression", formulas section: scale = (max - min)/(2^bits - 1),
 *    zero = min, code = round((x - zero)/scale), x^ = code*scale + zero.
 *
 * Arithmetic of the encoder (fixed so results are reproducible bit for bit):
 *   scale32 = (max - min) / (2^bits - 1)      IEEE fp32 division
 *   s = fp16_rn(scale32); z = fp16_rn(min + 0.0f)
 *   inv = s > 0 ? 1/s : 0                     IEEE fp32, correctly rounded
 *   code = clamp(rint_half_even((x - z) * inv), 0, 2^bits - 1)
 *          (subtract and multiply rounded separately; NaN -> 0)
 * Window bookkeeping per sequence with n tokens:
 *   n_quant = G * floor(max(n - R, 0) / G); tokens [n_quant, n) are held in
 *   bf16 in a ring of R + G slots (slot = token mod (R + G)); a group is
 *   quantized (flushed) when n - n_quant reaches R + G.
 * FP8: one scale per (kv head, K|V) set by the prefill, S = amax/448 (1 when
 *   amax is 0), code = e4m3_rn_satfinite(x * (1/S)); no window.
 * MIXED ("KV cache compression" on the miraclefarms wiki, TriAxialKV: each
 *   class of token is kept at 2 or 4 bits, most at 2): every token carries a
 *   class, 2 or 4, given by the caller; a key group and the values of its G
 *   tokens are stored at the widest class among those tokens (INT4 if any is
 *   4, else INT2), with the INT4 / INT2 arithmetic above.  The window keeps
 *   each token's class until its group is flushed.
 * Pre-RoPE keys (section 3.3 of the arganzheng page, KVQuant: quantize keys
 *   before RoPE, whose rotation spreads an outlier channel over its pair
 *   partner differently at every position, and apply RoPE when reading):
 *   with rope_theta > 0 the cache takes and stores un-rotated keys, and the
 *   decode turns key t (t = its position in the sequence, 0-based) pair by
 *   pair: channels (2i, 2i+1) by the angle t * rope_theta^(-2i/128),
 *   k'_2i = k_2i cos - k_2i+1 sin, k'_2i+1 = k_2i sin + k_2i+1 cos, after
 *   dequantization (window keys alike).  Queries are used as given.
 * Dense-and-sparse ("KV Cache lab", door4ai-lab, after experiment 03:
 *   KVQuant keeps the few extreme values apart in fp16 and quantizes the
 *   rest; experiment 01: one large value stretches a whole set's scale):
 *   with sparse = 1, each key set (a channel of a group) and each value set
 *   (a token's 128 channels) keeps its value of largest magnitude (the first
 *   such; NaN counts below any number) aside, exactly, as its bf16 input
 *   with its index in the set; the set's min/max and codes are taken over
 *   the other values, and the kept value's own code is 0.  The decode uses
 *   the kept values in place of the dense ones.
 * INT8 (section 3.1 of the arganzheng page: the 8-bit cache can also be INT8
 *   per token with a dynamic scale): the encoder above at 8 bits with one
 *   (scale, zero) per token over its 128 channels, for keys and for values,
 *   computed when the token is written; no window (n_quant == seq_len).
 *
 * Ownership: the caller allocates every byte of device memory (sizes from
 * kvq_buffer_bytes / kvq_decode_workspace_bytes); the library allocates
 * nothing.  Its only global state is the fixed device array that
 * kvq_decode_attention_noalloc uses instead of a workspace.  All calls enqueue work on the given
 * stream and return without synchronizing, except kvq_read_error.  Inputs
 * are read-only; the cache buffers are read-write; `out` and the workspace
 * are write-only.  Every device buffer must be 16-byte aligned.
 *
 * Errors: arguments are validated on the host before any launch and give
 * KVQ_ERR_* with nothing enqueued.  A failed launch gives KVQ_ERR_CUDA.
 * Conditions only the device can see set bits in *err_word (KVQ_DEVERR_*)
 * and skip the offending work; kernels never trap.
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *kvq_stream_t;   /* == cudaStream_t; NULL = legacy default stream */

typedef enum {
    KVQ_OK = 0,
    KVQ_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad enum */
    KVQ_ERR_SHAPE = 2,         /* inconsistent shape (H_q % H_kv, capacity % G, ...) */
    KVQ_ERR_UNSUPPORTED = 3,   /* valid but not implemented (head_dim != 128, ...) */
    KVQ_ERR_ALIGNMENT = 4,     /* a device pointer is not 16-byte aligned */
    KVQ_ERR_WORKSPACE = 5,     /* workspace too small */
    KVQ_ERR_CUDA = 6           /* a kernel launch failed (cudaGetLastError) */
} kvq_status;

typedef enum {
    KVQ_FORMAT_INT2 = 2,       /* 2-bit codes, asymmetric min/max, bf16 window */
    KVQ_FORMAT_INT4 = 4,       /* 4-bit codes, asymmetric min/max, bf16 window */
    KVQ_FORMAT_FP8_E4M3 = 8,   /* e4m3 codes, static per-(kv head) scale, no window */
    KVQ_FORMAT_INT8 = 16,      /* 8-bit codes, asymmetric min/max per token for K and V, no window */
    KVQ_FORMAT_MIXED = 6       /* INT4 or INT2 per key/value group by token class, bf16 window */
} kvq_format;

/* Device error bits (OR-ed into *err_word). */
#define KVQ_DEVERR_APPEND_FULL   0x1u   /* append found the capacity or the window full; token dropped */
#define KVQ_DEVERR_PAGE_RANGE    0x2u   /* a page id outside [0, num_pages); that page skipped */
#define KVQ_DEVERR_PREFILL_LEN   0x4u   /* a prefill sequence longer than the capacity; skipped */
#define KVQ_DEVERR_WAIT_TIMEOUT  0x8u   /* reserved: no current kernel waits on another (copies complete in hardware) */
#define KVQ_DEVERR_STATE         0x10u  /* seq_len / n_quant inconsistent; unit skipped */

/* Cache shape.  head_dim must be 128.  INT2/INT4: group % 16 == 0,
 * capacity % group == 0, residual >= 0.  Paged: page_size == 16 == group,
 * capacity is max_pages_per_seq * 16.  FP8 and INT8 (every token quantized
 * when written): group and residual ignored (treated as 16 and 0),
 * capacity % 16 == 0, contiguous only.  num_q_heads % num_kv_heads == 0
 * with at most 8 query heads per kv head.  INT groups are powers of two
 * (16, 32, 64 or 128 tokens). */
typedef struct {
    int32_t format;             /* kvq_format */
    int32_t batch;              /* B sequences */
    int32_t num_q_heads;        /* H_q */
    int32_t num_kv_heads;       /* H_kv */
    int32_t head_dim;           /* D = 128 */
    int32_t group;              /* G, tokens per key group */
    int32_t residual;           /* R, window tokens kept in bf16 */
    int32_t capacity;           /* tokens per sequence (contiguous layout) */
    int32_t page_size;          /* 0 = contiguous, 16 = paged */
    int32_t max_pages_per_seq;  /* paged: page-table row length */
    int32_t num_pages;          /* paged: pages in the pool */
    float rope_theta;           /* 0: keys as given.  > 0 (INT2/INT4, contiguous): keys are stored
                                   before RoPE and rotated by their position when read (below) */
    int32_t sparse;             /* 0, or 1 (INT2/INT4, contiguous, G of 16 or 32): dense-and-sparse,
                                   every key and value set keeps its largest value aside (below) */
} kvq_shape;

/*
 * Cache descriptor: the shape plus the caller's device buffers.
 * Layouts (b = sequence, h = kv head, t = token, c = channel, D = 128,
 * RB = D*bits/8 bytes per packed row, W = R + G):
 *
 *  k_codes  contiguous: u8 [B][H_kv][capacity][RB]    paged: [num_pages][H_kv][16][RB]
 *           row t holds token t's key codes packed along channels:
 *           4-bit: byte j = channel 2j (bits 0-3) | channel 2j+1 (bits 4-7);
 *           2-bit: byte j holds channel 4j+i in bits 2i..2i+1;
 *           FP8:   byte c = e4m3 code of channel c;
 *           INT8:  byte c = code of channel c.
 *  k_meta   INT8: fp16 [B][H_kv][capacity][2], per-token (scale, zero).
 *  k_meta   contiguous: fp16 [B][H_kv][capacity/G][2][D]   paged: [num_pages][H_kv][2][D]
 *           row 0 = per-channel scale, row 1 = per-channel zero of the group,
 *           each row in pair order: with c = 32l + u (l = c / 32),
 *             4-bit: u = 8J + r%2 + 4(r/2) + 2h (r < 4, h < 2) is stored at 32l + 8J + 2r + h;
 *             2-bit: u = 16J + r + 8h (r < 8, h < 2) is stored at 32l + 16J + 2r + h
 *           (adjacent halves hold the channel pair one decode fragment uses).
 *  v_codes  contiguous: u8 [B][H_kv][capacity/16][TB]      paged: [num_pages][H_kv][TB]
 *           one tile of 16 tokens, TB = 16*RB bytes, in the order the decode's
 *           tensor-core fragments consume it.  Code of (token i, channel c)
 *           of a tile, with n = c / 16, j = c % 16, lane = 4n + (i % 8) / 2,
 *           s = (i / 8) (0 or 1), o = i % 2 (first/second token of a pair):
 *             4-bit: word w = j / 2 (0..7), nibble p = (j % 2) + 2*o + 4*s;
 *                    word address = 16*lane + 4*(w % 4) + 512*(w / 4).
 *             2-bit: word w = j / 4 (0..3), position p = (j % 4) + 4*o + 8*s
 *                    (bits 2p..2p+1); word address = 16*lane + 4*w.
 *             FP8 and INT8: byte address = 16*lane + 512*(j / 4) + 4*(j % 4) + 2*s + o.
 *  v_meta   contiguous: fp16 [B][H_kv][capacity][2]       paged: [num_pages][H_kv][16][2]
 *           per-token (scale, zero).  Unused for FP8.
 *  k_res, v_res  bf16 [B][H_kv][W][D]: the window ring, slot = t mod W.
 *           Unused for FP8 and INT8.
 *  seq_len, n_quant  int32 [B]: tokens held / tokens quantized per sequence
 *           (n_quant == seq_len for FP8 and INT8).  Written by prefill,
 *           append, flush.  FP8 and INT8 codes and scales of the tokens of a
 *           sequence's last 16-token tile past seq_len are unspecified (the
 *           decode masks them).
 *  page_table  int32 [B][max_pages_per_seq]: physical page of logical page p
 *           (tokens [16p, 16p+16)).  Paged only.
 *  fp8_scale  float [2][H_kv]: row 0 = K scales, row 1 = V scales.  FP8 only.
 *  fp8_amax   uint32 [2][H_kv]: scratch for the prefill's amax.  FP8 only.
 *  err_word   uint32 [1]: device error bits, cleared by the caller.
 */
typedef struct {
    kvq_shape shape;
    void *k_codes;
    void *k_meta;
    void *v_codes;
    void *v_meta;
    void *k_res;
    void *v_res;
    int32_t *seq_len;
    int32_t *n_quant;
    const int32_t *page_table;
    float *fp8_scale;
    uint32_t *fp8_amax;
    uint32_t *err_word;
    uint8_t *group_bits;        /* MIXED: uint8 [B][capacity/G], 2 or 4 per stored group */
    uint8_t *window_class;      /* MIXED: uint8 [B][W], class of the token in each window slot */
    uint32_t *k_sparse;         /* sparse: [B][H_kv][capacity/G][D], kept key of each channel's set:
                                   bf16 bits | token within the group << 16 */
    uint32_t *v_sparse;         /* sparse: [B][H_kv][capacity], kept value of each token:
                                   bf16 bits | channel << 16 */
} kvq_cache;

typedef enum {
    KVQ_REGION_K_CODES = 0,
    KVQ_REGION_K_META = 1,
    KVQ_REGION_V_CODES = 2,
    KVQ_REGION_V_META = 3,
    KVQ_REGION_K_RES = 4,
    KVQ_REGION_V_RES = 5,
    KVQ_REGION_SEQ_LEN = 6,
    KVQ_REGION_N_QUANT = 7,
    KVQ_REGION_PAGE_TABLE = 8,
    KVQ_REGION_FP8_SCALE = 9,
    KVQ_REGION_FP8_AMAX = 10,
    KVQ_REGION_ERR_WORD = 11,
    KVQ_REGION_GROUP_BITS = 12,
    KVQ_REGION_WINDOW_CLASS = 13,
    KVQ_REGION_K_SPARSE = 14,
    KVQ_REGION_V_SPARSE = 15
} kvq_region;

/* Bytes the caller must allocate for one region of a cache of this shape
 * (0 for regions the format does not use).  Validates the shape. */
kvq_status kvq_buffer_bytes(const kvq_shape *shape, kvq_region region, size_t *bytes);

/*
 * Quantize a prefill into the cache, overwriting its state (section 3.2 of
 * the arganzheng page: per-channel key groups, per-token values, the last
 * tokens kept in the window).
 *  k_bf16, v_bf16: bf16 [T_total][H_kv][D], the B sequences back to back.
 *  cu_seqlens_dev: int32 [B+1] device array, sequence b is rows
 *                  [cu[b], cu[b+1]); lengths may be 0.
 *  max_len:        an upper bound of the lengths (sizes the grid).
 * Sets seq_len[b] = n_b and n_quant[b] = G*floor(max(n_b - R, 0)/G)
 * (n_b for FP8).  FP8 also sets fp8_scale from this prefill's amax over the
 * whole batch.  A sequence longer than the capacity or than max_len sets
 * KVQ_DEVERR_PREFILL_LEN and is left empty (and takes no part in the FP8
 * amax); the other sequences are quantized as if it were not there.
 */
kvq_status kvq_quantize_prefill(kvq_cache *cache, const void *k_bf16, const void *v_bf16,
                                const int32_t *cu_seqlens_dev, int32_t max_len, kvq_stream_t stream);

/*
 * Append one token per sequence (section 3.2 of the arganzheng page: the
 * newest tokens stay in full precision until a whole key group of G tokens
 * exists; jaedaily.cn "KV cache compression", process section: the cache
 * keeps two regions, the recent tokens in 16-bit and the rest quantized).
 *  k_new_bf16, v_new_bf16: bf16 [B][H_kv][D].  INT formats write the window slot seq_len mod (R + G);
 * FP8 encodes the token with the stored scales (saturating).  Then
 * seq_len += 1.  A sequence whose capacity is reached, or whose window
 * already holds R + G tokens (a flush is due), sets KVQ_DEVERR_APPEND_FULL
 * and drops the token.
 */
kvq_status kvq_append_token(kvq_cache *cache, const void *k_new_bf16, const void *v_new_bf16,
                            kvq_stream_t stream);

/*
 * Flush (section 3.2 of the arganzheng page: a group is quantized only once
 * all G of its tokens exist, per channel for keys and per token for values;
 * jaedaily.cn, process section: tokens leave the 16-bit region for the
 * quantized one).  For every sequence whose window holds R + G tokens,
 * quantize its oldest G window tokens as key group n_quant/G (and G value
 * tokens) and advance n_quant by G.  The decision is taken on the device (no host sync).  A
 * no-op for FP8.
 */
kvq_status kvq_flush_group(kvq_cache *cache, kvq_stream_t stream);

/*
 * kvq_append_token followed by kvq_flush_group, in one launch: the same
 * arguments, states, codes and error bits as the two calls in a row.  INT
 * formats with H_kv <= 8 run one cluster of H_kv CTAs per sequence (append,
 * quantize the oldest group if the window is now full, then advance
 * seq_len and n_quant after a cluster barrier); other shapes and FP8 issue
 * the two calls.
 */
kvq_status kvq_append_flush(kvq_cache *cache, const void *k_new_bf16, const void *v_new_bf16,
                            kvq_stream_t stream);

/*
 * The write side of a MIXED cache ("KV cache compression" on the
 * miraclefarms wiki, TriAxialKV: tokens are kept at 2 or 4 bits by their
 * class).  The same as kvq_quantize_prefill / kvq_append_token /
 * kvq_append_flush, plus the tokens' classes, which the calls above cannot
 * take (they return KVQ_ERR_INVALID_ARG on a MIXED cache):
 *  token_class_dev: uint8 device array, 2 or 4 per token (prefill: [T_total]
 *                   in the order of the K/V rows; append: [B]).  A class
 *                   other than 4 counts as 2.
 * A prefill stores every whole group at 4 bits if any of its G tokens is of
 * class 4, else at 2 bits, and records the width in group_bits; the window
 * tokens keep their class in window_class, and kvq_flush_group (which works
 * on every INT format) stores the flushed group at the widest class of its
 * tokens.  Codes are laid out as for INT4 (rows of 64 bytes, 1 KB value
 * tiles); a group stored at 2 bits fills the first half of its slot: its G
 * key rows packed at 32 bytes from the slot's start, each value tile in the
 * first 512 bytes of its 1 KB tile.  Its key scale/zero rows use the 2-bit
 * pair order.  Groups are 32, 64 or 128 tokens; contiguous layout only.
 */
kvq_status kvq_quantize_prefill_mixed(kvq_cache *cache, const void *k_bf16, const void *v_bf16,
                                      const uint8_t *token_class_dev, const int32_t *cu_seqlens_dev,
                                      int32_t max_len, kvq_stream_t stream);
kvq_status kvq_append_token_mixed(kvq_cache *cache, const void *k_new_bf16, const void *v_new_bf16,
                                  const uint8_t *token_class_dev, kvq_stream_t stream);
kvq_status kvq_append_flush_mixed(kvq_cache *cache, const void *k_new_bf16, const void *v_new_bf16,
                                  const uint8_t *token_class_dev, kvq_stream_t stream);

/*
 * Decode attention (split-K, then a combine pass): for each sequence b and
 * query head h, out[b][h][:] = sum_t softmax_t(softmax_scale * q.k^_t) v^_t
 * over all seq_len[b] tokens (quantized part dequantized in registers,
 * window tokens in bf16), kv head = h / (H_q / H_kv).  No mask: the query's
 * own token is expected to be in the cache already (section 3.2 of the
 * arganzheng page: the quantized part and the full-precision window are
 * attended separately and merged).
 *  q_bf16:    bf16 [B][H_q][D]
 *  out:       float [B][H_q][D]
 *  workspace: kvq_decode_workspace_bytes(cache, num_splits, max_len) bytes
 *  num_splits: >= 1, or 0 to let the library choose (the choice depends
 *             only on the shape and max_len).
 *             INT formats: the number of CTAs (4 warps each) that stream
 *             the quantized part; the chunks of all sequences are laid end
 *             to end and cut into 4 * num_splits equal slices, one per warp,
 *             whatever the lengths.  Each (warp, sequence x kv head) slice
 *             writes one partial to the workspace: at most
 *             4 * num_splits + B * H_kv partials of (H_q/H_kv) x 130 floats.
 *             FP8: CTAs per (sequence, kv head); B * H_q * num_splits
 *             partials of 130 floats.
 *  max_len:   an upper bound of seq_len over the batch.
 * A sequence with seq_len 0 gets out = 0.  Two launches are enqueued; for
 * INT formats the second (window + merge) may start before the first ends
 * and waits for it on the device.
 */
kvq_status kvq_decode_attention(const kvq_cache *cache, const void *q_bf16, float *out,
                                float softmax_scale, void *workspace, size_t ws_bytes,
                                int32_t num_splits, int32_t max_len, kvq_stream_t stream);

/* Largest split-partial area kvq_decode_attention_noalloc can use (8 MiB). */
#define KVQ_NOALLOC_SCRATCH_BYTES (8u << 20)

/*
 * kvq_decode_attention for callers that cannot allocate device memory, so
 * cannot hand over a workspace: code running inside a custom device
 * allocator's callbacks, plugins whose host framework owns all device
 * memory, or latency paths that must never enter the driver's allocator.
 * The paper has no counterpart to this entry point; it only changes where
 * the split partials live.  Arguments and results are those of
 * kvq_decode_attention without (workspace, ws_bytes).
 *
 * The partials go to a fixed array of KVQ_NOALLOC_SCRATCH_BYTES in the
 * library's own device memory; every GPU that loads the library keeps it
 * until the process exits.  A shape/split count whose partials do not fit
 * (kvq_decode_workspace_bytes > KVQ_NOALLOC_SCRATCH_BYTES) returns
 * KVQ_ERR_WORKSPACE and enqueues nothing.  The function calls no
 * allocation routine.  All calls on a device share the array and it keeps
 * the last call's contents (nothing in it needs clearing: each partial is
 * written before it is read); calls that overlap on the GPU, e.g. on two
 * streams, race on it.  The first call on each device looks up the array's
 * address with that device current; make it before any stream capture.
 */
kvq_status kvq_decode_attention_noalloc(const kvq_cache *cache, const void *q_bf16, float *out,
                                        float softmax_scale, int32_t num_splits, int32_t max_len,
                                        kvq_stream_t stream);

/*
 * kvq_decode_attention that also returns each row's softmax denominator, so
 * that attentions over disjoint token sets (for instance the shards of one
 * long sequence held by several GPUs) can be merged exactly afterwards by
 * kvq_merge_partials.
 *  lse: float [B][H_q], 16-byte aligned: ln sum_t exp(softmax_scale * q.k^_t)
 *       over the row's seq_len[b] tokens; -inf for a sequence with none.
 * Everything else is as for kvq_decode_attention (the same two launches).
 */
kvq_status kvq_decode_attention_lse(const kvq_cache *cache, const void *q_bf16, float *out, float *lse,
                                    float softmax_scale, void *workspace, size_t ws_bytes,
                                    int32_t num_splits, int32_t max_len, kvq_stream_t stream);

/*
 * Merge `parts` attentions of the same rows over disjoint token sets into
 * the attention over their union (the merge the decode itself applies to
 * its splits and to the quantized part and the window, section 3.2 of the
 * arganzheng page):
 *   out[r] = sum_p exp(lse_p[r] - L[r]) * outs_p[r],  L[r] = ln sum_p exp(lse_p[r]).
 *  outs:    float [parts][rows][D], each part's output (kvq_decode_attention_lse)
 *  lses:    float [parts][rows], each part's lse
 *  out:     float [rows][D]
 *  lse_out: float [rows] receives L, or NULL
 * A part whose lse is -inf has no tokens and contributes nothing; a row
 * with no tokens in any part gets out = 0 and L = -inf.  parts >= 1,
 * 0 <= rows <= 2^31 - 1; every pointer is 16-byte aligned device memory.
 * One launch on `stream` (none for rows = 0).
 */
kvq_status kvq_merge_partials(const float *outs, const float *lses, int32_t parts, int64_t rows,
                              float *out, float *lse_out, kvq_stream_t stream);

/* Workspace bytes kvq_decode_attention needs for this split count (0 = the
 * library's choice for max_len). */
size_t kvq_decode_workspace_bytes(const kvq_cache *cache, int32_t num_splits, int32_t max_len);

/* The split count kvq_decode_attention uses when given 0. */
int32_t kvq_decode_default_splits(const kvq_cache *cache, int32_t max_len);

/* Synchronize `stream` and read *err_word into *flags (blocking). */
kvq_status kvq_read_error(const kvq_cache *cache, uint32_t *flags, kvq_stream_t stream);

/* Static description of a status code. */
const char *kvq_status_string(kvq_status status);

/* Library version, "major.minor.patch". */
const char *kvq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */
