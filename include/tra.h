/*
 * tra.h -- C ABI of the tile-routed mixed-precision causal attention library
 * for NVIDIA B200 (sm_100a).
 *
 * The method (from the pages this library implements):
 *  - "TriAttention: Unified Sparse Mixed-Precision Attention for Long-Context
 *    LLM Inference", abstract: every query-key (QK) tile goes to skip, 4-bit or
 *    8-bit score computation; a head's policy is two diagonal-distance
 *    boundaries; the boundaries generate precision-grouped traversals for one
 *    fused kernel that skips omitted tiles and combines both QK precisions into
 *    one normalised attention output; the quantised keys/values prepared during
 *    prefill are reused as a compressed KV cache for decoding.
 *  - "TileMix: Tile-Centric Mixed-Precision Attention for LLM Inference
 *    Acceleration", abstract: hardware-aligned score tiles, routing decisions
 *    packed into bitmasks with one bit per group of adjacent key tiles, FP16
 *    (BF16 here) or INT8 score computation, both paths updating one shared
 *    online-softmax state; grouped-query attention, variable-length batches and
 *    INT8 key/value caches.
 *  - "HyQuant Uses Hybrid Precision to Compress LLM Attention", "How HyQuant
 *    works": decode-time dequantisation fused into the attention kernel.
 *
 * Conventions (the pages print no formulas; these are the readings adopted):
 *  - Tiles are TRA_TILE = 64 tokens.  A sequence of T tokens has
 *    nt = ceil(T/64) tiles; tile numbering restarts at every sequence start.
 *    ntiles = sum over sequences of nt (see tra_num_tiles).
 *  - bf16 tensors are passed as uint16_t bit patterns.
 *  - Q [ntok][Hq][d], K and V [ntok][Hkv][d], token-major, ntok = cu_seqlens[B].
 *  - Quantised tensors are tile-major per head:
 *      X8 int8  [H][ntiles][64][d], X4 uint8 [H][ntiles][64][d/2],
 *      scales float [H][ntiles].
 *    One symmetric scale per (head, tile) over the tile's valid rows:
 *      s8 = fl32(amax/127), s4 = fl32(amax/7),
 *      code = clamp(round_half_even(fl32(x / s)), -qmax, qmax)
 *    (IEEE fp32 divide); amax == 0 gives s = 0 and codes 0; rows past the end
 *    of a sequence are code 0.  INT4: two codes per byte, the even channel in
 *    the low nibble, two's complement.
 *  - Boundary policy, dist = qt - kt (tiles): dist < b1 -> INT8,
 *    b1 <= dist < b2 -> INT4, dist >= b2 -> skip; 1 <= b1 <= b2, so the
 *    diagonal tile is always kept in INT8.  Storage 8*Hq bytes at any length.
 *  - Bitmask policy: uint32 [Hq][ntiles][W]; bit g of row (h, q-tile) (word
 *    g/32, bit g%32) covers k-tiles [g*G, g*G+G): 1 -> BF16, 0 -> INT8; no skip.
 *  - Mixed policy: both of the above; the boundaries decide skip / INT4 / INT8
 *    and a set bit promotes a kept tile to BF16 (see TRA_POLICY_MIXED).
 *  - Traversal lists (CSR): prefill rows are (h, global q-tile), h-major;
 *    decode-cache rows are (b, kv-head), b-major.  entry = (prec << 28) | kt,
 *    kt local to the sequence, prec = TRA_PREC_*; a row lists its INT4 tiles
 *    ascending, then INT8 ascending, then BF16 ascending.
 *  - Softmax scale: any positive float; 1/sqrt(d) is the usual choice.
 *  - GQA: query head h reads KV head h / (Hq/Hkv).
 *
 * Memory and streams: every buffer is caller-owned device memory unless a
 * parameter says "host".  The library allocates no device memory (the host-only
 * boundary allocator keeps its tables in host memory), never synchronises the
 * device, and enqueues all work on the given stream (a cudaStream_t passed as
 * void*; NULL = legacy default stream).  Pointers to device buffers must be
 * 16-byte aligned.  Every call validates its arguments on the host before any
 * launch and returns a tra_status; tra_last_error() gives a thread-local text.
 * Errors found on the device (a bounded wait that expired, a full decode tail)
 * are OR-ed into the caller's int32 status word (TRA_DEV_*), which the caller
 * zeroes and reads back when it chooses.
 */
#ifndef TRA_H
#define TRA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TRA_API __attribute__((visibility("default")))
#else
#define TRA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TRA_OK = 0,
  TRA_ERR_INVALID = 1,     /* bad argument (null pointer, bad size, bad policy) */
  TRA_ERR_UNSUPPORTED = 2, /* valid but unsupported (e.g. d not 64 or 128) */
  TRA_ERR_BUFFER = 3,      /* a caller buffer is too small */
  TRA_ERR_CUDA = 4,        /* a CUDA call or launch failed */
  TRA_ERR_TIMEOUT = 5      /* reserved for callers that map TRA_DEV_TIMEOUT */
} tra_status;

#define TRA_TILE 64

#define TRA_PREC_INT4 1
#define TRA_PREC_INT8 2
#define TRA_PREC_BF16 3
/* FP8 (E4M3) score tiles of the optional middle band of a boundary policy (tra_policy.b8):
 * an extension the pages do not describe (an FP8 tier between INT8 and INT4), run on the
 * fp8 tensor-core kind at the INT8 rate.  Listed after the other groups of a row. */
#define TRA_PREC_FP8 4

#define TRA_POLICY_BOUNDARY 0
#define TRA_POLICY_BITMASK 1
/* Both at once (four-way): the boundaries decide skip / INT4 / INT8 by distance
 * and a set bitmask bit of a kept tile's group promotes it to BF16.  Neither page
 * describes the combination; it joins TriAttention's boundary rule (abstract) and
 * TileMix's bitmask (abstract).  Decode caches of a mixed policy follow its
 * boundaries.  The prefill runs one work unit per CTA in this mode (its operand
 * buffers do not fit twice), so it is slower per tile than the other two. */
#define TRA_POLICY_MIXED 2

#define TRA_LISTS_PREFILL 0
#define TRA_LISTS_DECODE_CACHE 1

/* tra_qtiles.formats bits */
#define TRA_FMT_Q8 0x01u
#define TRA_FMT_Q4 0x02u
#define TRA_FMT_K8 0x04u
#define TRA_FMT_K4 0x08u
#define TRA_FMT_V8 0x10u
#define TRA_FMT_V4 0x20u
/* INT4 codes of Q / K expanded to the int8 values 16 x code, row-major [H][ntiles][64][d]:
 * the tensor-core operand form the prefill streams for INT4 tiles (sm_100 has no integer
 * 4-bit MMA, so INT4 tiles run as int8 MMAs on these; the factor 256 of a product is
 * taken out of the INT4 scales exactly).  They share the sq4 / sk4 scales with Q4 / K4.
 * The packed Q4 / K4 formats stay the compact cache for decoding. */
#define TRA_FMT_Q4X 0x40u
#define TRA_FMT_K4X 0x80u
/* FP8 E4M3 codes of Q / K [H][ntiles][64][d] (one byte per value, row-major) with one
 * scale per (head, tile): sf = fl32(amax / 448), code = E4M3 round-to-nearest-even of
 * fl32(x / sf) saturating at +-448 (the sign of a zero kept); amax = 0 gives sf = 0 and
 * codes 0.  Needed by the prefill when a boundary policy has an FP8 band (b8 > b1). */
#define TRA_FMT_Q8F 0x100u
#define TRA_FMT_K8F 0x200u

/* device status word bits */
#define TRA_DEV_TIMEOUT 0x1      /* a bounded pipeline wait expired */
#define TRA_DEV_TAIL_FULL 0x2    /* decode: tail_len reached tail_cap */
#define TRA_DEV_BAD_LIST 0x4     /* prefill: a list entry whose precision has no tiles bound, or whose key tile is past its rows' last causal tile */

#define TRA_MAX_HEADS 256        /* Hq limit (policies travel as launch params) */
#define TRA_MAX_DUMP 64          /* max tiles per integer-accumulator dump */
#define TRA_MAX_DECODE_SPLITS 64

typedef struct {
  int32_t B;                        /* sequences */
  int32_t Hq, Hkv;                  /* query / key-value heads, Hq % Hkv == 0 */
  int32_t d;                        /* head dim: 64 or 128 */
  const int32_t* cu_seqlens_dev;    /* device [B+1], cu[0] = 0, non-decreasing */
  const int32_t* cu_seqlens_host;   /* host copy of the same values */
} tra_shape;

typedef struct {
  int32_t mode;                     /* TRA_POLICY_BOUNDARY, _BITMASK or _MIXED */
  const int32_t* b1;                /* host [Hq] (boundary and mixed modes) */
  const int32_t* b2;                /* host [Hq] (boundary and mixed modes) */
  const uint32_t* bitmask_dev;      /* device [Hq][ntiles][W] (bitmask and mixed modes) */
  int32_t G;                        /* k-tiles per bit (bitmask and mixed modes), >= 1 */
  int32_t W;                        /* words per bitmask row, W*32*G >= max nt */
  /* boundary mode only, optional (NULL: no FP8 band): host [Hq] with b1 <= b8 <= b2;
   * b1 <= dist < b8 -> FP8 instead of INT4.  Decode caches keep a band tile as INT8. */
  const int32_t* b8;
} tra_policy;

typedef struct {
  int8_t* q8;  uint8_t* q4;         /* [Hq][ntiles][64][d] / [..][d/2] */
  int8_t* k8;  uint8_t* k4;         /* [Hkv][ntiles][64][d] / [..][d/2] */
  int8_t* v8;  uint8_t* v4;         /* v4: see the V4 byte order below */
  float* sq8;  float* sq4;          /* [Hq][ntiles] */
  float* sk8;  float* sk4;          /* [Hkv][ntiles] */
  float* sv8;  float* sv4;
  uint32_t formats;                 /* TRA_FMT_* bits: which fields are present */
  int8_t* q4x; int8_t* k4x;         /* [Hq|Hkv][ntiles][64][d]: 16 x INT4 code (TRA_FMT_Q4X/K4X) */
  uint8_t* q8f; uint8_t* k8f;       /* [Hq|Hkv][ntiles][64][d]: FP8 E4M3 codes (TRA_FMT_Q8F/K8F) */
  float* sqf; float* skf;           /* [Hq|Hkv][ntiles]: their scales */
} tra_qtiles;
/* Code layout.  Rows are tokens of a 64-token tile; INT8 rows hold channel c in byte c,
 * as two's complement for Q8 and K8 and offset-binary (code + 128) for V8, which only
 * the decode reads.
 * INT4 rows pack two signed codes (range -7..7) per byte, the even channel in the low
 * nibble.  Q4 and K4 rows are row-major: byte j holds channels 2j and 2j + 1.  V4 rows,
 * read only by the decode, are stored in its MMA fragment order: within each 16-byte
 * group m, byte 2g + e (g = 0..7, e = 0, 1) holds the pair that row-major order keeps at
 * byte 16m + 8e + g, i.e. channels 32m + 16e + 2g and 32m + 16e + 2g + 1. */

/* Thread-local description of the last error returned on this thread. */
TRA_API const char* tra_last_error(void);

/* Library version string. */
TRA_API const char* tra_version(void);

/* Total tiles over the batch (sum of ceil(T_b/64)), from cu_seqlens_host;
 * -1 if the shape is invalid. */
TRA_API int64_t tra_num_tiles(const tra_shape* shape);

/* Bytes of each quantised buffer for `formats` (the sum over present fields,
 * each rounded up to 256 bytes); 0 on an invalid shape. */
TRA_API size_t tra_qtiles_bytes(const tra_shape* shape, uint32_t formats);

/*
 * quantize_qkv_tiles -- per-(head, 64-token tile) symmetric INT8/INT4
 * quantisation of Q, K and V (TriAttention abstract: the prefill prepares
 * quantised keys and values; TileMix abstract: INT8 tiles and K/V caches).
 * q/k/v: device bf16 [ntok][H][d]; a tensor may be NULL when `out->formats`
 * requests none of its formats.  Writes the codes and scales selected by
 * out->formats (layouts above).  Deterministic and bit-exact with the rule in
 * the header comment.
 */
TRA_API tra_status quantize_qkv_tiles(const tra_shape* shape, const uint16_t* q, const uint16_t* k,
                              const uint16_t* v, const tra_qtiles* out, void* stream);

/*
 * tra_tile_lists_size -- exact CSR sizes of the traversal lists (host only,
 * closed form; no device access).  list_kind = TRA_LISTS_PREFILL gives
 * rows = Hq*ntiles; TRA_LISTS_DECODE_CACHE gives rows = B*Hkv.  *row_ptr_len =
 * rows + 1.  Fails with TRA_ERR_INVALID on a bad policy and TRA_ERR_UNSUPPORTED
 * if nnz does not fit in int32.
 */
TRA_API tra_status tra_tile_lists_size(const tra_shape* shape, const tra_policy* policy,
                               int32_t list_kind, int64_t* rows, int64_t* nnz);

/*
 * build_tile_lists -- precision-grouped traversals (TriAttention abstract:
 * each head's two boundaries are turned into traversals grouped by precision;
 * TileMix abstract: routing decisions are packed into bitmasks in which one
 * bit governs several adjacent key tiles).
 * Prefill rows (h, q-tile): boundary mode lists INT4 k-tiles
 * [max(0,qt-b2+1), qt-b1] then INT8 [max(0,qt-b1+1), qt]; bitmask mode lists
 * the INT8 k-tiles <= qt then the BF16 ones.  Decode-cache rows (b, kv-head):
 * a k-tile's precision is the highest any query head of the group gives it at
 * dist = nt-1-kt (boundary mode), INT8 for all tiles in bitmask mode.
 * row_ptr: device int32 [row_ptr_len]; entries: device uint32 [entries_cap];
 * sizes from tra_tile_lists_size, else TRA_ERR_BUFFER.
 */
TRA_API tra_status build_tile_lists(const tra_shape* shape, const tra_policy* policy, int32_t list_kind,
                            int32_t* row_ptr, int64_t row_ptr_len, uint32_t* entries,
                            int64_t entries_cap, void* stream);

/*
 * routed_attention_prefill -- fused causal prefill attention over the
 * precision-grouped traversal: every listed tile's scores come from its
 * precision (INT8 or INT4 codes multiplied exactly in int32 and rescaled by
 * sQ*sK, or BF16 with fp32 accumulation); every path updates one online
 * softmax state per query row; P*V uses bf16 P and the original bf16 V.
 * (TriAttention abstract: one fused kernel skips the omitted tiles and merges
 * the contributions of both QK precisions into a single normalised output;
 * TileMix abstract: the high- and low-precision paths share one online-softmax
 * state.)
 * q/k/v: device bf16 as above; tiles: output of quantize_qkv_tiles (Q8/K8
 * always, Q4X/K4X and the INT4 scales when the policy has INT4 tiles, Q8F/K8F
 * when a boundary policy has an FP8 band: its tiles score on FP8 E4M3 codes with
 * fp32 accumulation, rescaled by sQ*sK); row_ptr/entries: prefill
 * lists; out: device bf16 [ntok][Hq][d]; lse: device float [Hq][ntok] natural-
 * log logsumexp of the scaled scores, or NULL.
 * Integer-accumulator dump (debug; n_dump = 0 disables): dump_coords device
 * int32 [n_dump][4] = (b, h, qt, kt); for each listed INT8/INT4 tile the raw
 * int32 Q-code x K-code^T accumulators go to dump_out [n_dump][64][64]
 * (row = query within the tile, column = key; BF16 and FP8 tiles, whose
 * accumulators are fp32, are not dumped).  n_dump <= TRA_MAX_DUMP.
 * status_dev: device int32, receives TRA_DEV_* bits.  row_ptr must be as
 * build_tile_lists wrote it (entries are read over [row_ptr[r], row_ptr[r+1]));
 * an entry the kernel cannot use (a precision with no tiles bound, a key tile past
 * its rows' last causal tile) sets TRA_DEV_BAD_LIST, no copy is issued for it, and
 * out is then undefined.
 */
TRA_API tra_status routed_attention_prefill(const tra_shape* shape, const tra_policy* policy,
                                    const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                    const tra_qtiles* tiles, const int32_t* row_ptr,
                                    const uint32_t* entries, float softmax_scale, uint16_t* out,
                                    float* lse, const int32_t* dump_coords, int32_t n_dump,
                                    int32_t* dump_out, int32_t* status_dev, void* stream);

/* Workspace bytes routed_attention_decode needs (split-K partials); 0 on bad sizes. */
TRA_API size_t tra_decode_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t d);

/*
 * routed_attention_decode -- one decode step over the compressed KV cache
 * (TriAttention abstract: the K/V quantised during prefill are reused as a
 * compressed KV cache when decoding, so the prompt is not re-read at full
 * precision; HyQuant, "How HyQuant works": dequantisation happens inside the
 * attention kernel).  For each sequence b: the new token's k_new/v_new [b][kvh] is
 * appended at tail position tail_len[b]; every query head attends to the
 * cached tiles listed for (b, kv-head) -- K = sK*code and V = sV*code in the
 * tile's cached format -- plus the bf16 tail tokens [0, tail_len[b]] ; one
 * softmax per head; then tail_len[b] is incremented.
 * prefill_shape: the prefill's shape (cu_seqlens give the cached lengths);
 * policy: the policy the lists were built from (validation only: INT4 cache
 * formats are required when a boundary policy has b1 < b2);
 * q: device bf16 [B][Hq][d]; k_new/v_new: device bf16 [B][Hkv][d];
 * cache: K8/K4/V8/V4 (+scales) from quantize_qkv_tiles;
 * row_ptr/entries: TRA_LISTS_DECODE_CACHE lists;
 * k_tail/v_tail: device bf16 [B][Hkv][tail_cap][d]; tail_len_dev: device
 * int32 [B] (read, then incremented by one); out: device bf16 [B][Hq][d];
 * workspace: device, >= tra_decode_workspace_bytes(B, Hq, Hkv, d), zero-filled
 * before its first use and not written by anything else between calls: it starts
 * with per-(sequence, KV head) arrival counters, which every call leaves at zero
 * (at a fixed place for every shape with B * (Hkv + 1) <= 16384, so one workspace
 * may serve several shapes), followed by the splits' partial results.
 * A sequence whose tail is full sets TRA_DEV_TAIL_FULL and leaves its output
 * and tail untouched.
 */
TRA_API tra_status routed_attention_decode(const tra_shape* prefill_shape, const tra_policy* policy,
                                   const uint16_t* q,
                                   const uint16_t* k_new, const uint16_t* v_new,
                                   const tra_qtiles* cache, const int32_t* row_ptr,
                                   const uint32_t* entries, uint16_t* k_tail, uint16_t* v_tail,
                                   int32_t* tail_len_dev, int32_t tail_cap, float softmax_scale,
                                   uint16_t* out, void* workspace, size_t workspace_bytes,
                                   int32_t* status_dev, void* stream);

/*
 * routed_attention_decode_noalloc -- the same decode step as
 * routed_attention_decode, for callers that cannot allocate device memory.
 * The paper has no counterpart: this is a deployment convenience of this
 * library.  Some callers only ever receive input and output buffers -- a
 * custom operator or plugin inside a host framework that owns every device
 * allocation and hands out no allocator, or a serving loop that reserved all
 * of its device memory up front and must not allocate while it decodes -- so
 * they cannot provide the workspace the regular entry point needs.  This entry
 * point keeps that scratch in a fixed array of TRA_NOALLOC_SCRATCH_BYTES bytes
 * inside the library instead: every GPU that loads the library holds the
 * array until the process exits.  It calls no allocator of any kind.
 * Arguments, layouts, device status bits and validation are those of
 * routed_attention_decode, minus workspace/workspace_bytes.
 * Limits and rules:
 *  - problems needing more than TRA_NOALLOC_SCRATCH_BYTES of scratch
 *    (tra_decode_workspace_bytes(B, Hq, Hkv, d)), or with
 *    B * (Hkv + 1) > TRA_NOALLOC_MAX_COUNTERS, are rejected with
 *    TRA_ERR_UNSUPPORTED;
 *  - the first call on each device looks up the array's device address with
 *    that device current; make that first call before any stream capture;
 *  - all calls on a device share the one array, which keeps whatever the last
 *    call left there; calls whose kernels overlap on the GPU (for example on
 *    two streams at once) race on it and give wrong results, so issue them on
 *    one stream or otherwise order them;
 *  - the array starts zero-filled (static storage).  Its first 64 KiB hold the
 *    decode's per-(sequence, KV head) and per-sequence arrival counters, which
 *    must be zero when a call starts; every call leaves them at zero again, and
 *    for every accepted shape (B * (Hkv + 1) <= TRA_NOALLOC_MAX_COUNTERS) they
 *    stay inside that area, so calls of different shapes may follow one another.
 *    The partial results behind the counters are written before they are read.
 */
#define TRA_NOALLOC_SCRATCH_BYTES (4u << 20)
#define TRA_NOALLOC_MAX_COUNTERS 16384

TRA_API tra_status routed_attention_decode_noalloc(
    const tra_shape* prefill_shape, const tra_policy* policy, const uint16_t* q,
    const uint16_t* k_new, const uint16_t* v_new, const tra_qtiles* cache, const int32_t* row_ptr,
    const uint32_t* entries, uint16_t* k_tail, uint16_t* v_tail, int32_t* tail_len_dev,
    int32_t tail_cap, float softmax_scale, uint16_t* out, int32_t* status_dev, void* stream);

/*
 * Token-level hybrid (HyQuant Uses Hybrid Precision to Compress LLM Attention, "The
 * observation behind the method" and "How HyQuant works": a small set of important
 * key positions and a window of recent tokens keep high precision, the rest of the
 * context is read from quantised storage; selection and the decode kernel run on the
 * GPU).  Reading adopted here: per (sequence, KV head) the n = ceil(frac * T) prefix
 * positions of largest importance (ties to the earlier position) and every key within
 * `window` positions of the query keep bf16 K and V; all other prefix keys and values
 * are read from their tile's INT4 codes (K4 / V4 of quantize_qkv_tiles) times the
 * tile scale; queries stay bf16.  A decode query sits at position T + tail_len,
 * after the prefix and the tail tokens before it.
 * All arrays are caller-owned device memory:
 *   sel_count int32 [B]                 n of each sequence (written by the selection)
 *   sel_pos   int32 [B][Hkv][cap]       selected positions (0 .. T-1), ascending
 *   sel_mask  uint64 [Hkv][ntiles]      bit c of tile kt: token kt*64 + c is selected
 *   k_sel, v_sel bf16 [B][Hkv][cap][d]  K / V rows of the selected positions
 *   k_win, v_win bf16 [B][Hkv][window][d] K / V of prefix tokens T - window .. T - 1
 *                                       (rows before the sequence start are zero)
 * cap >= tra_hybrid_capacity(shape, frac); window >= 0.
 */
typedef struct {
  int32_t window;
  int32_t cap;
  int32_t* sel_count;
  int32_t* sel_pos;
  uint64_t* sel_mask;
  uint16_t* k_sel;
  uint16_t* v_sel;
  uint16_t* k_win;
  uint16_t* v_win;
} tra_hybrid;

/* max over sequences of ceil(frac * T); -1 for an invalid shape or frac outside [0, 1]. */
TRA_API int32_t tra_hybrid_capacity(const tra_shape* shape, double frac);

/*
 * hybrid_select_tokens -- the high-precision side of the hybrid cache.  importance:
 * device float [ntok][Hkv] (finite), one score per key position and KV head (the
 * signal that marks "vertical lines"; synthetic in this library's tests);
 * k, v: device bf16 [ntok][Hkv][d].  Writes every array of *hy (layouts above).
 * TRA_ERR_INVALID for bad pointers, frac outside [0, 1], window < 0;
 * TRA_ERR_BUFFER if hy->cap is below tra_hybrid_capacity.
 */
TRA_API tra_status hybrid_select_tokens(const tra_shape* shape, const float* importance, double frac,
                                        const uint16_t* k, const uint16_t* v, const tra_hybrid* hy,
                                        void* stream);

/*
 * hybrid_attention_decode -- one decode step of the token-level hybrid: every prefix
 * tile of (b, kv-head) is streamed in INT4 (cache: K4 / V4 and their scales) with
 * its selected and in-window keys masked out, those keys are read from the bf16 side
 * arrays of *hy instead, and the bf16 tail (earlier decode tokens and the new one,
 * appended at tail position tail_len[b]) is attended as in routed_attention_decode;
 * one softmax per query head; then tail_len[b] is incremented.  Arguments as
 * routed_attention_decode (same workspace size and rules), with *hy from
 * hybrid_select_tokens on the same shape.  Hq / Hkv <= 8.
 */
TRA_API tra_status hybrid_attention_decode(const tra_shape* prefill_shape, const tra_hybrid* hy,
                                           const uint16_t* q, const uint16_t* k_new,
                                           const uint16_t* v_new, const tra_qtiles* cache,
                                           uint16_t* k_tail, uint16_t* v_tail, int32_t* tail_len_dev,
                                           int32_t tail_cap, float softmax_scale, uint16_t* out,
                                           void* workspace, size_t workspace_bytes,
                                           int32_t* status_dev, void* stream);

/*
 * hybrid_attention_prefill -- causal prefill attention of the token-level hybrid
 * (HyQuant Uses Hybrid Precision to Compress LLM Attention, "How HyQuant works":
 * prefill support with dedicated kernels).  Query i of a sequence reads key j <= i
 * with bf16 K and V when j is selected (hy->sel_mask, from hybrid_select_tokens on
 * the same shape) or i - j < hy->window, and from the INT4 codes of j's tile times
 * the tile scale (K4 and V4 of quantize_qkv_tiles) otherwise; one softmax per row.
 *   q bf16 [ntok][Hq][d]; k, v bf16 [ntok][Hkv][d]; kv: the INT4 scales sk4 and sv4
 *   (formats K4 or K4X, and V4; the codes are not read: they are recomputed from k,
 *   v and those scales exactly as the quantiser computes them);
 *   k_mix, v_mix: caller-owned scratch, bf16 [ntok][Hkv][d], written by this call:
 *   each row is the token's bf16 row when it is selected, else its INT4 codes as
 *   bf16 integers (the operands of the tiles outside the window);
 *   out bf16 [ntok][Hq][d]; lse fp32 [Hq][ntok] (natural log of the row's sum of
 *   exp of scaled scores) or NULL.  Two launches (operand build, attention), no
 *   synchronisation.  Device-side errors (a bounded wait expired) are OR-ed into
 *   *status_dev.  TRA_ERR_INVALID for NULL or misaligned pointers, a missing
 *   scale array, window < 0 or a bad softmax_scale.
 */
TRA_API tra_status hybrid_attention_prefill(const tra_shape* shape, const tra_hybrid* hy,
                                            const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                            const tra_qtiles* kv, uint16_t* k_mix, uint16_t* v_mix,
                                            float softmax_scale, uint16_t* out, float* lse,
                                            int32_t* status_dev, void* stream);

/* Complete-tile counts of one head's boundary pair over a batch (TriAttention
 * abstract: candidate boundary pairs are weighed by complete-tile execution costs):
 * n8 = sum over every sequence's q-tiles qt of min(qt + 1, b1), n4 = the sum of
 * min(qt + 1, b2) minus n8; the cost of the pair is n8 and n4 times the per-tile
 * times of the two precisions.  Host only.  TRA_ERR_INVALID for an invalid shape,
 * NULL outputs, or not 1 <= b1 <= b2. */
TRA_API tra_status tra_boundary_tile_counts(const tra_shape* shape, int32_t b1, int32_t b2,
                                            int64_t* n8, int64_t* n4);

/* Complete-tile cost model of routed_attention_prefill under a boundary policy (TriAttention
 * abstract: candidate boundary pairs are weighed by complete-tile execution costs).  Host
 * only.  The prefill runs one work unit per (query head, sequence, q-tile pair) and two
 * units per CTA; a unit's work is its entries -- the k-tiles either of its two q-tiles
 * lists -- counting dual_weight for an entry the two q-tiles give different precisions
 * (two score products, one P V) and 1 for the others; the two units of a CTA run side by
 * side until the lighter one ends, then the heavier one runs alone, `solo` times as long
 * per entry (it no longer shares the SM): CTA time = min(w0, w1) + solo * |w0 - w1|;
 * CTAs are placed in launch order on n_sm SMs, each on the SM that frees first.
 * *makespan receives the resulting time in entry units and *entries the total entry
 * count, so that a kernel time is predicted as entry_time * makespan + fixed with
 * entry_time, fixed and solo fitted from measured launches.  b1 / b2: host [Hq].
 * TRA_ERR_INVALID for an invalid shape or policy, dual_weight < 1, solo not in (0, 1]
 * or n_sm < 1. */
TRA_API tra_status tra_prefill_cost_model(const tra_shape* shape, const int32_t* b1, const int32_t* b2,
                                          double dual_weight, double solo, int32_t n_sm,
                                          double* makespan, double* entries);

/* Model-wide boundary allocation (TriAttention abstract: an allocator selects each
 * head's boundaries to minimise calibration error under a shared computation budget).
 * Host only.  err [n_heads][n_cand] (finite) and cost [n_heads][n_cand] (>= 0, integer
 * units chosen by the caller, e.g. tile counts times per-tile times, rounded up) describe
 * each head's candidate pairs; choice [n_heads] receives, per head, the index of the
 * candidate that minimises the total error with total cost <= budget.  Exact: candidates
 * beaten on both cost and error are dropped, then a dynamic programme runs over the
 * integer budget (O(n_heads x n_cand x budget) time, one byte per head and budget unit of
 * host memory); ties between equal totals are broken deterministically.
 * total_err / total_cost (nullable) receive the sums.  TRA_ERR_INVALID for bad arguments
 * or when no choice fits the budget; TRA_ERR_UNSUPPORTED when n_heads x (budget + 1)
 * exceeds 2^27 (use coarser cost units).  1 <= n_cand <= 255. */
TRA_API tra_status tra_allocate_boundaries(int32_t n_heads, int32_t n_cand, const double* err,
                                           const int64_t* cost, int64_t budget, int32_t* choice,
                                           double* total_err, int64_t* total_cost);

/*
 * tra_selftest_bounded_wait -- diagnostic; the pages have no counterpart.  Runs
 * one small kernel whose mbarrier wait can never complete, through the same
 * bounded-wait routine every pipeline wait of the prefill and decode kernels
 * uses, with a limit of limit_ns nanoseconds instead of their 2 s.  The wait
 * must give up, OR TRA_DEV_TIMEOUT (0x1) into *status_dev and let the kernel
 * return; a waiter that returns success would OR 0x100 instead.  Nothing is
 * read or written outside the kernel's shared memory and *status_dev.
 * status_dev: device int32 (the caller zeroes it).  limit_ns: 1e3 .. 1e9, else
 * TRA_ERR_INVALID.  stream: cudaStream_t or NULL.  Asynchronous like the other
 * entry points; a launch failure is returned as TRA_ERR_CUDA.
 */
TRA_API tra_status tra_selftest_bounded_wait(int32_t* status_dev, int64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TRA_H */
