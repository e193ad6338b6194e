/*
 * mqkv.h — C ABI of libmqkv, a B200 (sm_100a) library for a chunk-adaptive
 * mixed-bitwidth KV cache.
 *
 * The library implements one data path, in three calls:
 *
 *   mq_route_chunks  a small router scores every context token against three
 *                    quantisation "experts" {FP16, INT4, INT2}; each fixed-size
 *                    chunk takes the majority choice of its tokens.
 *                    (MoQAE paper notes, 方法详解 › 整体框架 and
 *                     关键设计 › Quantization-Aware Experts.)
 *   mq_similarity_route  alternative chunk map: each chunk's bitwidth from its
 *                    similarity to a per-sequence query vector (Cocktail
 *                    abstract: chunk-level quantization search).
 *   mq_build_layout  chunks of each sequence are regrouped by precision into
 *                    contiguous FP16 → INT4 → INT2 segments before anything is
 *                    quantised (Cocktail abstract on the "Bin Zhang" scholarfeed
 *                    author page: chunk-level KV cache computation).
 *   mq_pack_kv       K and V of one layer are quantised at the chunk's bitwidth
 *                    and written into those segments.
 *   mq_decode_attn   single-query attention for every sequence, read directly
 *                    from the mixed-bitwidth packed cache.
 *   mq_grow_*        decode-time growth: new tokens in an FP16 tail, each full
 *                    chunk routed and appended to its precision segment.
 *   mq_decode_attn_partial / mq_combine_partials
 *                    a sequence split by context across devices: per-shard
 *                    partial results, merged after an all-gather.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Pointers prefixed h_ are HOST memory; every other data pointer is DEVICE
 *   memory on the current CUDA device.  All memory is owned by the caller; the
 *   library never allocates, frees or retains a pointer after a call returns.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   Every call that launches work is asynchronous on that stream and never
 *   synchronises the host, except the two calls documented as synchronising
 *   (mq_packed_bytes, mq_device_status).
 * - Arguments are validated on the host before anything is launched.  A
 *   failing check returns a non-zero mq_status, launches nothing, and leaves a
 *   human-readable reason in mq_last_error() (thread-local).  Validation makes
 *   no CUDA call, so it works on a machine without a GPU.
 * - Device pointers must be 16-byte aligned.
 * - Conditions that can only be seen on the device (for example a packed
 *   buffer smaller than the layout needs) make the kernel skip its writes and
 *   set a bit in a device-side status word, read with mq_device_status().
 *
 * Shapes and notation
 * -------------------
 *   B    = shape.num_seqs          sequences in the batch
 *   Hq   = shape.num_q_heads       query heads
 *   Hkv  = shape.num_kv_heads      key/value heads; Hq % Hkv == 0 (GQA when >1)
 *   d    = shape.head_dim          64 or 128
 *   L    = shape.chunk_len         tokens per routing chunk, a multiple of 32
 *   G    = shape.group_size        quantisation group along head_dim, must be 32
 *   T_b  = h_seq_lens[b]           tokens of sequence b (0 allowed)
 *   n_b  = ceil(T_b / L)           chunks of sequence b; the last one may be short
 *   T    = sum_b T_b,  N = sum_b n_b
 *   expert / segment index s: 0 = FP16 (16 bits), 1 = INT4, 2 = INT2.
 *
 * d_cu_seqlens is a device int64[B+1] with d_cu_seqlens[0] = 0 and
 * d_cu_seqlens[b+1] - d_cu_seqlens[b] = T_b: row r of C, K and V belongs to
 * sequence b when d_cu_seqlens[b] <= r < d_cu_seqlens[b+1].
 *
 * Packed cache format (one buffer per layer; part of this ABI)
 * ------------------------------------------------------------
 * Per sequence b, segments in the order FP16, INT4, INT2.  A segment holds the
 * sequence's chunks of that precision in their ORIGINAL chunk order (stable
 * regrouping), so the short tail chunk, when present, is the last chunk of its
 * segment.  Inside segment s of sequence b there are 2*Hkv regions, K regions
 * for kv-heads 0..Hkv-1 first, then V regions 0..Hkv-1, each of
 * layout.seq[b].region_bytes[s] bytes.  With n = seg_tokens[s] tokens:
 *   FP16 region : codes = n rows of d IEEE binary16 values (2*d bytes a row),
 *                 converted from the input with round-to-nearest-even (a copy
 *                 for fp16 input); no scales.
 *                 region_bytes = align128(n * 2*d).
 *   INT-b region: codes  = n rows of d*b/8 bytes; group k (dims 32k..32k+31)
 *                 fills bytes [4b*k, 4b*(k+1)) of the row.  Inside a group,
 *                 element j sits at bit position b*(j mod (32/b)) of the
 *                 little-endian 32-bit word j / (32/b) (least significant bits
 *                 first).
 *                 scales = n rows of d/32 pairs of binary16 (scale, min), the
 *                 pair for group k at bytes [4k, 4k+4) of the row, scale in the
 *                 low half.  They start at byte layout.seq[b].scale_offset[s]
 *                 = align128(n * d*b/8) of the region.
 *                 region_bytes = scale_offset + align128(n * (d/32) * 4).
 *   Row i of a region is segment token i: token t of the chunk at reordered
 *   position p sits at row (p - seg_chunk_begin[s]) * L + t.
 *   Segment s of sequence b starts at byte layout.seq[b].seg_base[s]; bases
 *   are consecutive in (b, s) order (each segment is 2*Hkv*region_bytes long,
 *   a multiple of 128), and the buffer is layout.header.packed_bytes long.
 *   Padding bytes are unspecified.
 *
 * Quantiser (spec reading; the MoQAE notes leave it open)
 * --------------------------------------------------------------
 * For every (token, kv-head, group of 32) of an INT-b chunk, with x the fp32
 * value of each element (fp16 input widened exactly):
 *   mn = min x, mx = max x                                  (fp32)
 *   s  = (mx - mn) / (2^b - 1)   IEEE fp32 subtract and divide, s = 1 if mx == mn
 *   q  = min(max(rint((x - mn) / s), 0), 2^b - 1)   fp32 subtract and divide,
 *        rint rounds half to even, no FMA contraction, no fast-math
 *   stored: q bit-packed, (half)s and (half)mn rounded to nearest even.
 * Inputs must be finite with |x| < 65504 (undefined otherwise).
 * Dequantised value: xhat = q * (half)s + (half)mn.
 */
#ifndef MQKV_H_
#define MQKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mq_status {
  MQ_OK = 0,
  MQ_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or shape */
  MQ_ERR_UNSUPPORTED = 2,   /* valid in principle, not built (e.g. d = 96) */
  MQ_ERR_WORKSPACE = 3,     /* caller buffer smaller than the call needs */
  MQ_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
  MQ_ERR_DEVICE_CHECK = 5   /* a kernel reported a failed check */
} mq_status;

typedef enum mq_dtype {
  MQ_F32 = 0,               /* IEEE binary32 */
  MQ_F16 = 1                /* IEEE binary16 */
} mq_dtype;

typedef enum mq_expert {
  MQ_EXPERT_FP16 = 0,
  MQ_EXPERT_INT4 = 1,
  MQ_EXPERT_INT2 = 2
} mq_expert;

typedef struct mq_shape {
  int32_t num_seqs;      /* B   >= 1 */
  int32_t num_q_heads;   /* Hq  >= 1 */
  int32_t num_kv_heads;  /* Hkv >= 1, Hq % Hkv == 0, Hq / Hkv <= 8 */
  int32_t head_dim;      /* d: 64 or 128 */
  int32_t chunk_len;     /* L: multiple of 32, 32 <= L <= 4096 */
  int32_t group_size;    /* G: must be 32 */
} mq_shape;

/* Device-side status bits (mq_device_status). */
#define MQ_DEV_PACKED_TOO_SMALL   0x1u  /* packed_bytes < layout packed size */
#define MQ_DEV_WORKSPACE_TOO_SMALL 0x2u /* decode schedule exceeds workspace */
#define MQ_DEV_BAD_LAYOUT         0x4u  /* layout magic/shape mismatch */
#define MQ_DEV_WAIT_TIMEOUT       0x8u  /* a bounded wait on a copy gave up */
#define MQ_DEV_INDEX_RANGE        0x10u /* an index left its valid range */
#define MQ_DEV_CAPACITY           0x20u /* a growth step exceeded a reserved capacity */

/* ---------------------------------------------------------------------------
 * Layout table (device memory written by mq_build_layout; part of this ABI).
 *
 *   [mq_layout_header][mq_seq_layout x B][int32 perm[N] (padded to 16 B)]
 *   [int32 inv[N] (padded to 16 B)]
 *
 * perm[chunk_offset_b + p] = original chunk index of the chunk stored at
 * reordered position p of sequence b; inv is its inverse (original index ->
 * reordered position); both are local to the sequence.
 * Fields marked "schedule" describe how mq_decode_attn splits the work; they
 * are implementation-defined (any split that covers every segment token once
 * is valid) and are not part of the method.
 * ------------------------------------------------------------------------- */
#define MQ_LAYOUT_MAGIC 0x4C4B514Du   /* "MQKL" */
#define MQ_LAYOUT_VERSION 1u

typedef struct mq_layout_header {
  uint32_t magic;           /* MQ_LAYOUT_MAGIC */
  uint32_t version;         /* MQ_LAYOUT_VERSION */
  int32_t  num_seqs;        /* B */
  int32_t  num_kv_heads;    /* Hkv */
  int32_t  head_dim;        /* d */
  int32_t  chunk_len;       /* L */
  int32_t  total_chunks;    /* N */
  int32_t  total_items;     /* schedule: work items per kv-head */
  int64_t  total_tokens;    /* T */
  uint64_t packed_bytes;    /* bytes of one layer's packed buffer */
  int32_t  item_tokens[3];  /* schedule: max tokens of a work item, per segment */
  int32_t  grow_chunks;     /* 0: fixed layout; > 0: growable (mq_grow_*), chunk
                               slots per sequence beyond its built chunks */
} mq_layout_header;         /* 64 bytes */

typedef struct mq_seq_layout {
  int64_t  token_offset;      /* d_cu_seqlens[b] */
  int32_t  num_tokens;        /* T_b */
  int32_t  num_chunks;        /* n_b */
  int32_t  chunk_offset;      /* sum of n_b' for b' < b */
  int32_t  seg_chunks[3];     /* chunks in each segment */
  int32_t  seg_chunk_begin[3];/* first reordered position of each segment */
  int32_t  seg_tokens[3];     /* tokens in each segment */
  uint64_t seg_base[3];       /* byte offset of each segment in packed */
  uint64_t region_bytes[3];   /* bytes of one (K|V, kv-head) region */
  uint64_t scale_offset[3];   /* byte offset of scales inside an INT region (0 for FP16) */
  int32_t  item_begin[3];     /* schedule: first work item of (b, s) */
  int32_t  item_count[3];     /* schedule: work items of (b, s) */
  int32_t  chunk_capacity;    /* growable: chunk slots of b (perm/inv entries
                                 reserved at chunk_offset); fixed: 0 */
  int32_t  grow_state;        /* growable: MQ_GROW_* bits; fixed: 0 */
} mq_seq_layout;              /* 160 bytes */

/* grow_state bits */
#define MQ_GROW_OPEN 0x1  /* the last chunk is the open FP16 tail (not yet routed) */
#define MQ_GROW_FULL 0x2  /* the last growth step found no room for this sequence */

/* ---------------------------------------------------------------------------
 * Status and sizes
 * ------------------------------------------------------------------------- */

/* Static text for a status code. Never NULL. */
const char* mq_status_string(mq_status status);

/* Reason for the last failing call on this thread ("" if none). */
const char* mq_last_error(void);

/* Bytes of the layout table for this shape and these lengths; 0 if the
 * arguments are invalid (see mq_last_error). */
size_t mq_layout_bytes(const mq_shape* shape, const int32_t* h_seq_lens);

/* Bytes of one layer's packed buffer if every chunk were FP16 — an upper bound
 * for any routing map. 0 if the arguments are invalid. */
size_t mq_packed_bytes_upper_bound(const mq_shape* shape, const int32_t* h_seq_lens);

/* Bytes of workspace mq_decode_attn needs for a layout built from this shape
 * and these lengths. 0 if the arguments are invalid. */
size_t mq_decode_workspace_bytes(const mq_shape* shape, const int32_t* h_seq_lens);

/* Reads layout.header.packed_bytes into *h_bytes. SYNCHRONISES `stream`. */
mq_status mq_packed_bytes(const void* layout, size_t* h_bytes, void* stream);

/* Synchronises `stream`, then stores the device status word (MQ_DEV_* bits,
 * OR-ed over every kernel since the last clear) in *h_flags; clears it when
 * `clear` is non-zero. Returns MQ_ERR_DEVICE_CHECK when any bit is set. */
mq_status mq_device_status(uint32_t* h_flags, int32_t clear, void* stream);

/* ---------------------------------------------------------------------------
 * mq_route_chunks — router, per-token argmax, per-chunk vote, routing freezing.
 *
 * MoQAE paper notes, 关键设计 › Quantization-Aware Experts: the router maps a
 * chunk C (rows = tokens, D features) to one score per expert for every token,
 * printed as f(CW1·CW2)W3.  This library reads that as the gated MLP
 *     z_t = (SiLU(C_t W1) ⊙ (C_t W2)) W3 + b3,   SiLU(x) = x / (1 + e^-x)
 * evaluated in fp32.  Every token picks argmax_e z_t[e] (an exact tie goes to
 * the lower index = more bits); every chunk takes the expert most of its
 * tokens picked (a tie in counts goes to the lower index).  With
 * routing_freeze != 0, chunk 0 of every sequence is forced to FP16
 * (路由冻结 / Routing Freezing).  The map is computed once per sequence from
 * the router input C; the caller reuses the resulting layout for every layer
 * (路由共享 / Routing Sharing).
 *
 *   C            device fp32 [T, D] row-major (row r = token r, see d_cu_seqlens)
 *   W1, W2       device fp32 [D, H] row-major
 *   W3           device fp32 [H, 3] row-major
 *   b3           device fp32 [3], or NULL for zero bias
 *   token_expert device uint8 [T]  out: per-token argmax
 *   chunk_expert device uint8 [N]  out: per-chunk expert, chunk (b, c) at
 *                                  index chunk_offset_b + c
 *   logits       device fp32 [T, 3] out, or NULL
 *   workspace    device buffer of at least mq_route_workspace_bytes(shape,
 *                h_seq_lens, D, H) bytes (weights split for the tensor
 *                cores, partial scores); contents on entry are ignored
 * Constraints: 1 <= D, D % 4 == 0; H in {64, 128, 256}.
 * The two projections run on the tensor cores in three bf16 passes
 * (hi*hi + hi*lo + lo*hi of a bf16 high part and the bf16 of the remainder,
 * fp32 accumulation), which keeps each product within about 2^-16 relative;
 * the scores agree with exact arithmetic to about 1e-4 relative, well inside
 * the gap a routing decision needs before rounding can flip it (a token's
 * choice can only change when its two best scores are within twice the
 * error).
 * ------------------------------------------------------------------------- */
size_t mq_route_workspace_bytes(const mq_shape* shape, const int32_t* h_seq_lens,
                                int32_t D, int32_t H);

mq_status mq_route_chunks(const mq_shape* shape, const int32_t* h_seq_lens,
                          const int64_t* d_cu_seqlens,
                          const float* C, int32_t D, int32_t H,
                          const float* W1, const float* W2, const float* W3,
                          const float* b3, int32_t routing_freeze,
                          uint8_t* token_expert, uint8_t* chunk_expert,
                          float* logits, void* workspace, size_t workspace_bytes,
                          void* stream);

/* ---------------------------------------------------------------------------
 * mq_similarity_route — chunk-level quantization search by similarity, an
 * alternative to mq_route_chunks that writes the same chunk_expert map.
 *
 * Cocktail abstract on the "Bin Zhang" scholarfeed author page: the bitwidth
 * of each context chunk follows from how similar the chunk is to the query.
 * The page names neither the similarity nor the cut-offs; this library reads
 * it as the cosine between the chunk's mean router-input row and a per-
 * sequence query vector u_b, cut at two thresholds the caller gives:
 *     m_(b,c) = mean of C_t over the chunk's tokens (a short tail chunk
 *               averages its own tokens),
 *     sim     = <m, u_b> / (|m| |u_b|),   0 when either vector is zero,
 *     expert  = FP16 if sim >= tau_hi, else INT4 if sim >= tau_lo, else INT2.
 * With routing_freeze != 0, chunk 0 of every sequence is FP16 (the same
 * freezing rule as the router's).  Sums and the threshold test are in fp64.
 *
 *   C            device fp32 [T, D] row-major (rows as for mq_route_chunks)
 *   u            device fp32 [B, D] row-major, one query vector per sequence
 *   tau_hi, tau_lo  thresholds (any finite values; tau_hi <= tau_lo makes
 *                INT4 unreachable)
 *   chunk_expert device uint8 [N]  out, chunk (b, c) at chunk_offset_b + c
 *   similarity   device fp64 [N] out, or NULL
 * Constraints: 1 <= D, D % 4 == 0; B <= 65535.  Needs no workspace.  NaN
 * thresholds are rejected (MQ_ERR_INVALID_ARG).  A NaN or infinite value in C
 * or u gives a NaN similarity, which compares false and maps to INT2.
 * ------------------------------------------------------------------------- */
mq_status mq_similarity_route(const mq_shape* shape, const int32_t* h_seq_lens,
                              const int64_t* d_cu_seqlens,
                              const float* C, int32_t D, const float* u,
                              double tau_hi, double tau_lo, int32_t routing_freeze,
                              uint8_t* chunk_expert, double* similarity,
                              void* stream);

/* ---------------------------------------------------------------------------
 * mq_build_layout — Cocktail's chunk regrouping (chunk-level KV cache
 * computation): stable partition of each sequence's chunks by precision into
 * FP16 → INT4 → INT2 segments, with perm/inv tables, segment token counts and
 * byte offsets of the packed format above.
 *
 *   chunk_expert device uint8 [N], values 0..2 (other values: treated as INT2
 *                and MQ_DEV_INDEX_RANGE is set)
 *   layout       device buffer of at least mq_layout_bytes(shape, h_seq_lens)
 * One layout serves every layer (routing sharing) and every decode step.
 * ------------------------------------------------------------------------- */
mq_status mq_build_layout(const mq_shape* shape, const int32_t* h_seq_lens,
                          const int64_t* d_cu_seqlens,
                          const uint8_t* chunk_expert,
                          void* layout, size_t layout_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * mq_pack_kv — quantise one layer's K and V at each chunk's bitwidth (the
 * quantiser above) and write them into the packed format.
 *
 *   K, V         device [T, Hkv, d] row-major, dtype kv_dtype (MQ_F16 or MQ_F32)
 *   packed       device buffer of packed_bytes bytes; must be at least the
 *                layout's packed_bytes (checked on the device: if it is
 *                smaller nothing is written and MQ_DEV_PACKED_TOO_SMALL is set)
 * ------------------------------------------------------------------------- */
mq_status mq_pack_kv(const mq_shape* shape, const int32_t* h_seq_lens,
                     const void* layout, const void* K, const void* V,
                     int32_t kv_dtype, void* packed, size_t packed_bytes,
                     void* stream);

/* ---------------------------------------------------------------------------
 * mq_decode_attn — one decode query per (sequence, query head) attends over
 * every cached token of its sequence (MoQAE notes, 整体框架: ordinary attention
 * after quantisation), reading the packed cache directly:
 *   o[b,h] = sum_t softmax_t(scale * q[b,h] · khat_t) vhat_t
 * with khat/vhat the dequantised K/V of kv-head h / (Hq/Hkv).  Work is split
 * into precision-homogeneous pieces of one segment each; a second pass merges
 * the pieces' (max, sum, accumulator) triples.  The result is repeatable bit
 * for bit: each piece is computed by one warp from a fresh state and the
 * merge takes the pieces in a fixed order, however the warps interleave.
 *
 *   q            device [B, Hq, d], dtype q_dtype (MQ_F16 or MQ_F32)
 *   softmax_scale  <= 0 selects 1/sqrt(d)
 *   out          device fp32 [B, Hq, d]; a sequence with T_b = 0 gets zeros
 *   workspace    device buffer of at least mq_decode_workspace_bytes(shape,
 *                h_seq_lens) bytes; contents on entry are ignored
 * ------------------------------------------------------------------------- */
mq_status mq_decode_attn(const mq_shape* shape, const int32_t* h_seq_lens,
                         const void* layout, const void* packed,
                         const void* q, int32_t q_dtype, float softmax_scale,
                         float* out, void* workspace, size_t workspace_bytes,
                         void* stream);

/* ---------------------------------------------------------------------------
 * mq_decode_attn_noalloc — mq_decode_attn without a caller workspace.
 *
 * The paper has no counterpart to this call; it exists for callers that
 * cannot allocate device memory: for example a serving runtime that reserves
 * nearly all of HBM for its own KV pool at start-up and permits no later
 * cudaMalloc, or a plain C host program with no device allocator of its own.
 * The per-item partial results go to a scratch array of
 * MQ_NOALLOC_SCRATCH_BYTES bytes that is part of the library's module image:
 * every GPU that loads the library holds it until the process exits.
 *
 *   Arguments: as mq_decode_attn, without workspace / workspace_bytes.
 *   Limit: fails with MQ_ERR_WORKSPACE, before anything is launched, when
 *          mq_decode_workspace_bytes(shape, h_seq_lens) exceeds
 *          MQ_NOALLOC_SCRATCH_BYTES; otherwise errors as mq_decode_attn.
 *   Set-up: the first call on each device looks up the array's device
 *          address (cudaGetSymbolAddress) with that device current; make that
 *          first call before any stream capture begins.  The address is kept
 *          for the life of the process: after cudaDeviceReset on a device,
 *          do not call this function on that device again.
 *   Sharing: every call uses the same array, which keeps what the last call
 *          wrote.  Calls whose work overlaps on the GPU (other streams, other
 *          host threads) race on it and corrupt each other's results.
 *          Nothing in it has to start at zero: each entry the merge pass
 *          reads is written earlier in the same call.
 *   Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * ------------------------------------------------------------------------- */
#define MQ_NOALLOC_SCRATCH_BYTES (16u << 20)

mq_status mq_decode_attn_noalloc(const mq_shape* shape, const int32_t* h_seq_lens,
                                 const void* layout, const void* packed,
                                 const void* q, int32_t q_dtype, float softmax_scale,
                                 float* out, void* stream);

/* ---------------------------------------------------------------------------
 * Context split across devices: mq_decode_attn_partial + mq_combine_partials.
 *
 * A long sequence can be split by context: device r holds a contiguous range
 * of whole chunks of every sequence (routed with routing_freeze only on the
 * device holding chunk 0), builds its own layout and packed cache for that
 * range, and computes a partial result for every (sequence, query head).
 * The records of all devices are gathered (an all-gather over NVLink) and
 * merged with mq_combine_partials.  The merge is the usual split softmax
 * (the pages are silent on it): with m_r a reference score of shard r and
 * l_r = sum exp(score - m_r) over its tokens,
 *     M = max_r m_r,  w_r = l_r exp(m_r - M),  o = sum_r w_r o_r / sum_r w_r.
 *
 * Record layout, MQ_PARTIAL_FLOATS(d) floats per (b, h), [B][Hq] order:
 *     [ o_0 .. o_{d-1} (this shard's normalised output), m, l, 0, 0 ]
 * m is not necessarily the largest score: the decode moves its reference only
 * when a score exceeds it by more than 8 ln 2, so the largest score lies in
 * [m, m + 8 ln 2] and l <= 256 * tokens; m + ln l (the log-sum-exp of the
 * shard's scores) is what the record fixes.  An empty shard gives m = -inf,
 * l = 0, o = 0.
 * ------------------------------------------------------------------------- */
#define MQ_PARTIAL_FLOATS(d) ((d) + 4)

/* mq_decode_attn over this device's shard, writing records instead of the
 * output: partial is device fp32 [B, Hq, MQ_PARTIAL_FLOATS(d)].  Other
 * arguments and errors as mq_decode_attn. */
mq_status mq_decode_attn_partial(const mq_shape* shape, const int32_t* h_seq_lens,
                                 const void* layout, const void* packed, const void* q,
                                 int32_t q_dtype, float softmax_scale, float* partial,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* Merges num_parts records per (b, h): partials is device fp32
 * [num_parts][num_seqs][num_q_heads][MQ_PARTIAL_FLOATS(head_dim)] (the
 * gathered records, shard order irrelevant), out is device fp32
 * [num_seqs, num_q_heads, head_dim].  head_dim 64 or 128. */
mq_status mq_combine_partials(int32_t num_parts, int32_t num_seqs, int32_t num_q_heads,
                              int32_t head_dim, const float* partials, float* out,
                              void* stream);

/* ---------------------------------------------------------------------------
 * Cache growth during decoding (mq_grow_*).
 *
 * The pages describe routing and packing of a prefilled context and say
 * nothing about tokens produced while decoding; this library follows the
 * plain reading that new tokens accumulate in an FP16 tail and that a chunk
 * is routed, quantised and appended to its precision segment once it holds L
 * tokens (MoQAE notes, 整体框架: one bitwidth per chunk; Cocktail abstract:
 * chunks grouped by precision).
 *
 * A growable layout reserves, per sequence, room for `grow_tokens` more
 * tokens: ceil(grow_tokens / L) more chunks in every segment (the FP16
 * segment one more, for the open tail) and as many chunk slots in perm/inv.
 * The last chunk of a sequence, when partial, is the OPEN tail: it is kept in
 * FP16 at the end of the FP16 segment whatever chunk_expert says, and it is
 * the only partial chunk.  Each decode step, in this order:
 *
 *   mq_grow_commit(layout, sealed, 1)        once: applies the seals of the
 *                                            previous step, then reserves one
 *                                            token row per sequence
 *   for every layer:
 *     mq_grow_append_kv(layout, K_new, V_new, packed[layer])
 *     mq_decode_attn(h_seq_lens + grow_tokens, layout, packed[layer], q, ...)
 *   if some sequence's open tail now holds L tokens:
 *     route it (mq_route_chunks or mq_similarity_route over its L rows, with
 *     routing_freeze only for a sequence's chunk 0) into sealed[B]
 *     (255 = no seal for that sequence)
 *     for every layer: mq_grow_seal(layout, sealed, packed[layer])
 *
 * mq_grow_seal encodes the full tail from its fp16 rows into the next free
 * rows of segment sealed[b] (1 or 2; 0 leaves it in FP16); the following
 * mq_grow_commit moves the chunk there in the layout (perm, inv, counts,
 * decode schedule).  Every step touches O(L) rows per layer.  The result is
 * the layout and packed bytes that mq_build_layout / mq_pack_kv would give
 * for the grown sequences with the same map, except that (a) regions keep
 * their reserved capacity, and (b) chunks quantised from the tail were
 * quantised from fp16 values (the tail's storage), which matters only for
 * fp32 inputs.  A step that would overflow a reservation is skipped for that
 * sequence, sets MQ_GROW_FULL in its grow_state and MQ_DEV_CAPACITY in the
 * status word.  All calls are asynchronous on `stream`; none synchronises.
 * ------------------------------------------------------------------------- */

/* Sizes for a growable layout: layout table bytes, an upper bound of one
 * layer's packed bytes (every present chunk at FP16 plus all reservations),
 * and the decode workspace for the grown lengths.  Output pointers may be
 * NULL.  Constraints as mq_build_layout, 0 <= grow_tokens and every
 * h_seq_lens[b] + grow_tokens <= 2^23. */
mq_status mq_grow_sizes(const mq_shape* shape, const int32_t* h_seq_lens,
                        int32_t grow_tokens, size_t* layout_bytes,
                        size_t* packed_bytes_upper_bound,
                        size_t* decode_workspace_bytes);

/* mq_build_layout for a growable layout (header.grow_chunks > 0).  The
 * chunk_expert entry of a partial last chunk is ignored (open tail, FP16). */
mq_status mq_grow_build_layout(const mq_shape* shape, const int32_t* h_seq_lens,
                               int32_t grow_tokens, const int64_t* d_cu_seqlens,
                               const uint8_t* chunk_expert, void* layout,
                               size_t layout_bytes, void* stream);

/* mq_pack_kv for a growable layout (same arguments plus grow_tokens, which
 * must be the value the layout was built with); packed must hold
 * header.packed_bytes (mq_packed_bytes). */
mq_status mq_grow_pack_kv(const mq_shape* shape, const int32_t* h_seq_lens,
                          int32_t grow_tokens, const void* layout, const void* K,
                          const void* V, int32_t kv_dtype, void* packed,
                          size_t packed_bytes, void* stream);

/* One step of the layout: with `sealed` (device uint8[B], or NULL for none),
 * every sequence whose open tail holds L tokens and whose sealed[b] is 0, 1
 * or 2 has that chunk moved to segment sealed[b] (255: left open); then, with
 * add_token = 1, one token row is reserved at the end of every sequence's
 * open tail (a new tail is opened after a sealed chunk).  A layout that is
 * not growable sets MQ_DEV_BAD_LAYOUT. */
mq_status mq_grow_commit(const mq_shape* shape, void* layout, const uint8_t* sealed,
                         int32_t add_token, void* stream);

/* Writes the newest token of every sequence: K_new and V_new are device
 * [B, Hkv, d] in kv_dtype (rows stored as fp16, round-to-nearest-even) into
 * the row the last mq_grow_commit reserved in this layer's packed buffer.
 * Sequences whose last commit found no room (MQ_GROW_FULL) are skipped. */
mq_status mq_grow_append_kv(const mq_shape* shape, const void* layout,
                            const void* K_new, const void* V_new, int32_t kv_dtype,
                            void* packed, size_t packed_bytes, void* stream);

/* Encodes every full open tail with sealed[b] in {1, 2} into the next free
 * rows of that segment of this layer's packed buffer (the layout is not
 * changed; the next mq_grow_commit with the same `sealed` moves the chunk). */
mq_status mq_grow_seal(const mq_shape* shape, const void* layout, const uint8_t* sealed,
                       void* packed, size_t packed_bytes, void* stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* MQKV_H_ */
