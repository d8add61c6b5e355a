/*
 * kvq.h - low-bit KV-cache quantize-append and split-K decode attention for one B200 GPU.
 *
 * C ABI.  Every pointer is a plain device (or host, where stated) pointer; sizes are plain
 * integers; streams are passed as `void*` holding a cudaStream_t (NULL = legacy default stream).
 * No call allocates device memory except kvq_create (a small split-K workspace and nothing
 * else); the cache itself lives in one caller-owned device arena.
 *
 * Sources (web pages, cited by title and section):
 *   [FMKQ]  "Fourier Magnitude KV Cache Quantization" forum thread: post 6 ("Corrected
 *           semantics", "Minimal recipe", "Milestone", "The winning recipe") and the long
 *           reply ("The three controls I would try first", "Fixed-rate magnitude/phase
 *           allocation", "The finite-phase implementation and the physical codec may be
 *           worth separating").
 *   [E21W]  "PROVISIONAL: known 3-bit KV cache methods on the 4B ... (proxy queries)":
 *           "What I tested", "Result".
 *   [E22L]  "Can 4-bit keys and 2-bit values hit a 1M-token memory budget?": "What I
 *           tested", "Result".
 *   [LCPP]  llama.cpp issue #21385 "Per-head adaptive KV cache quantization": "Finding 1".
 *
 * Error behaviour: argument and configuration errors are detected on the host before any
 * launch and returned as a status; launch failures come back as KVQ_ERR_CUDA.  No kernel
 * traps.  A device-side condition the host cannot see in advance (an append past the capacity
 * while a CUDA graph replays, a bad sequence id) skips the offending writes and raises a bit in
 * the cache's error word (kvq_error_flags).  The only wait in any kernel is the decode's poll
 * for a staged tile, bounded (about one second; KVQ_ERRF_WAIT_TIMEOUT when it runs out).  Test
 * hook: with the environment variable KVQ_TEST_STALL_FIRST_WAIT=<cycles> set when a handle is
 * created, the first such wait of every tensor-core decode CTA of that handle polls a barrier
 * that nothing arrives on for that many clock cycles and then takes the give-up path.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = -1,  /* null pointer, out-of-range index or size, inconsistent config */
  KVQ_ERR_UNSUPPORTED = -2,  /* valid but not built (e.g. polar at head_dim != 128) */
  KVQ_ERR_CAPACITY = -3,     /* append past capacity, or more queries than max_queries */
  KVQ_ERR_CUDA = -4,         /* a CUDA runtime call or launch failed */
  KVQ_ERR_ALLOC = -5,        /* arena too small, or the workspace allocation failed */
  KVQ_ERR_STATE = -6         /* call order violated (e.g. channel scale never set) */
} kvq_status;

/* Storage format of one side (K or V). */
enum {
  KVQ_FMT_FP16 = 0,     /* unquantized fp16 rows (the K-only arm's V [E22L]) */
  KVQ_FMT_INT = 1,      /* b-bit integer grid; scale_mode ABSMAX (ggml signed -2^(b-1)..2^(b-1)-1,
                           [E22L] "Result", [LCPP]) or MINMAX (asymmetric, [E21W] variant A) */
  KVQ_FMT_NF4 = 2,      /* 16-level NormalFloat codebook, absmax scale [FMKQ] post 6 "NF4/g64" */
  KVQ_FMT_TERNARY = 3,  /* {-s, 0, +s}, s = group absmax, 5 trits per byte [FMKQ] "Milestone" */
  KVQ_FMT_SIGN = 4,     /* {-s, +s}, s = group mean |x| [FMKQ] "Minimal recipe" */
  KVQ_FMT_POLAR = 5,    /* rFFT magnitude (bits) / phase (bits2) indices [FMKQ] reply */
  KVQ_FMT_CART = 6,     /* rFFT real/imag, signed absmax int-bits, one scale [FMKQ] reply control */
  KVQ_FMT_LLOYD = 7,    /* Gaussian Lloyd-Max levels (bits 2..4) times the group RMS, [E22L] "Result":
                           the value grid named for the next run */
  KVQ_FMT_SORTED = 8    /* sorted groups ([FMKQ] post 6 "The winning recipe" item 1): the row sorted
                           descending (equal values in channel order), consecutive `group` values on
                           the min-max grid at `bits` (2..4), and each channel's rank stored in
                           ceil(log2 head_dim) bits after the codes; fp16 scale and zero per group */
};
/* INT scale modes: ABSMAX = the ggml signed grid; MINMAX = asymmetric; SYMMETRIC = levels
 * (q - (2^b - 1)/2) d, outermost level at the group's largest magnitude ([E22L] "Result": the
 * signed grid has one level fewer on its positive side; a symmetric grid is named as the next
 * value grid to try). */
enum { KVQ_SCALE_ABSMAX = 0, KVQ_SCALE_MINMAX = 1, KVQ_SCALE_SYMMETRIC = 2 };
enum { KVQ_ROT_NONE = 0, KVQ_ROT_H128 = 128, KVQ_ROT_H256 = 256 };
enum { KVQ_ANCHOR_NONE = 0, KVQ_ANCHOR_FIRST_N = 1, KVQ_ANCHOR_WINDOW = 2, KVQ_ANCHOR_ALL = 3 };
enum { KVQ_SIDE_K = 0, KVQ_SIDE_V = 1 };
enum { KVQ_DOMAIN_STORED = 0, KVQ_DOMAIN_ORIGINAL = 1 };
/* Error-word bits.  KVQ_ERRF_WAIT_TIMEOUT: a decode kernel gave up waiting for a staged tile of
 * keys/values (a bounded wait on a shared-memory barrier ran out); its output is not valid. */
enum { KVQ_ERRF_CAPACITY = 1, KVQ_ERRF_SEQ_ID = 2, KVQ_ERRF_WAIT_TIMEOUT = 4 };

typedef struct {
  int32_t format;      /* KVQ_FMT_* */
  int32_t bits;        /* INT: 2..8; CART: 2..8; POLAR: magnitude bits 1..8; else ignored */
  int32_t bits2;       /* POLAR: phase bits 1..8; else ignored */
  int32_t scale_mode;  /* INT: KVQ_SCALE_ABSMAX or KVQ_SCALE_MINMAX; else must be ABSMAX */
  int32_t group;       /* channels per scale: 4, 8, 16, 32, 64 or 128, dividing head_dim
                          (POLAR/CART: ignored, one scale per row; FP16: ignored) */
  int32_t rotation;    /* KVQ_ROT_NONE / H128 / H256: orthonormal Sylvester Walsh-Hadamard over
                          blocks of that many channels (block-diagonal if < head_dim)
                          [E21W] variant B, [E22L] "What I tested".  Not with POLAR/CART. */
  int32_t chan_scale;  /* K only: 1 = divide by a per-(layer, kv-head) fp16 channel scale
                          before the rotation ([E21W] variants C/D); set with
                          kvq_set_chan_scale before the first append. */
  int32_t mean_sub;    /* K only, quantized formats: 1 = subtract the sequence's key mean before
                          everything else and add it back after dequantizing ([LCPP], the later
                          comment on a per-head shared key mean, removed before quantizing and
                          restored afterwards).  The mean of a (sequence,
                          kv-head) is the mean of the rows of the sequence's first append (its
                          length was 0), rounded to fp16 once from the exact sum, and is kept for
                          the rows that follow; anchored rows stay raw. */
} kvq_side;

typedef struct {
  int32_t n_layers;      /* 1..64 */
  int32_t batch;         /* sequences, >= 1 */
  int32_t n_kv_heads;    /* >= 1 */
  int32_t n_q_heads;     /* multiple of n_kv_heads; query head h reads kv-head h / (Hq/Hkv) */
  int32_t head_dim;      /* 64, 128 or 256 */
  int32_t capacity;      /* tokens per sequence per layer, >= 1 */
  int32_t max_queries;   /* largest n_q passed to kvq_decode_attention, >= 1 */
  kvq_side k, v;
  uint64_t anchor_layer_mask;  /* bit l set: layer l keeps fp16 anchor rows */
  int32_t anchor_rule;         /* KVQ_ANCHOR_*; [FMKQ] post 6 "Corrected semantics" */
  int32_t anchor_n;            /* FIRST_N: tokens t < n; WINDOW: the last n tokens */
  float sm_scale;              /* softmax scale; 0 selects 1/sqrt(head_dim) */
  int32_t anchor_bits;         /* anchor precision ([FMKQ] post 6 "The winning recipe" item 4, the
                                  anchor-precision dial): 16 (or 0) keeps anchored rows as fp16;
                                  8 or 4 stores them on the signed absmax grid (largest magnitude at
                                  -2^(b-1)) in groups of 32 channels with an fp16 scale each, in the
                                  original domain.  8/4 need row formats (INT, NF4, TERNARY, SIGN,
                                  LLOYD) on both sides of anchored layers. */
} kvq_config;

/* Byte offsets (into the arena) and geometry of one (layer, side) of a head group.  Rows of one
 * (sequence, kv-head) are contiguous: row r of unit u = (b * n_heads + h - head0) is at
 * codes + (u * row_stride_tokens + r) * row_bytes; scales (fp16) at
 * scales + ((u * row_stride_tokens + r) * n_groups) * 2, zeros likewise (MINMAX only).
 * Anchor rows (fp16, original domain) at anchors + ((u * anchor_rows + slot) * head_dim) * 2,
 * slot = t (FIRST_N, ALL) or t mod anchor_n (WINDOW).  Offsets are -1 when absent. */
typedef struct {
  int64_t codes, scales, zeros, anchors, chan_scale, seq_len;
  int64_t key_mean;  /* K with mean_sub: fp16 [batch * n_kv_heads][head_dim], unit u at u * head_dim */
  int64_t anchor_scales;  /* int anchors: fp16 [units][anchor_rows][head_dim / 32]; anchor rows then hold
                             head_dim * anchor_bits / 8 code bytes each (LSB-first) instead of fp16 */
  int32_t row_bytes, n_groups, row_stride_tokens, anchor_rows;
  int32_t head0, n_heads;  /* the head group these regions hold: kv-heads [head0, head0 + n_heads) of
                              the layer (all of them without per-head formats); unit u = b * n_heads
                              + (h - head0) */
} kvq_layout;

typedef struct kvq_cache kvq_cache;

/* Bytes of device memory the cache arena needs for `cfg` (256-byte aligned base).
 * Returns KVQ_ERR_INVALID_ARG / KVQ_ERR_UNSUPPORTED for a bad config. Host only. */
kvq_status kvq_arena_bytes(const kvq_config* cfg, uint64_t* bytes);

/* Validate `cfg`, bind the caller-owned device arena (>= kvq_arena_bytes, 256-byte aligned;
 * owned by the caller, must outlive the handle), zero its sequence lengths, and allocate the
 * handle plus a split-K workspace on the current device.  Synchronous. */
kvq_status kvq_create(const kvq_config* cfg, void* arena, uint64_t arena_bytes, kvq_cache** out);

/* Per-layer formats ("E21W" "What I tested" and "Result": a per-layer K/V bit allocation
 * under an average budget, e.g. 2-bit K in two layers and 4-bit V in three, 3-bit elsewhere).
 * layer_k / layer_v: host arrays of cfg->n_layers sides, read during the call only; NULL
 * means cfg->k / cfg->v on every layer (and only then is that field read).  Every side is
 * checked as in kvq_create; otherwise identical to kvq_arena_bytes / kvq_create (the same
 * kernels run, each layer with its own format). */
kvq_status kvq_arena_bytes_layers(const kvq_config* cfg, const kvq_side* layer_k, const kvq_side* layer_v,
                                  uint64_t* bytes);
kvq_status kvq_create_layers(const kvq_config* cfg, const kvq_side* layer_k, const kvq_side* layer_v, void* arena,
                             uint64_t arena_bytes, kvq_cache** out);

/* Per-(layer, kv-head) formats (llama.cpp #21385 "Finding 2": per-head bit allocation from the
 * Renyi entropy of each head's attention, b_h = b_avg + 0.25 (H_avg - H_2(h)), with the lowest-
 * entropy ~2% of heads -- the sink heads -- kept unquantized; "Feature Request: Per-Head KV Cache
 * Types": per-head type selection in the cache allocation and per-head dequantization dispatch).
 * head_k / head_v: host arrays of n_layers * n_kv_heads sides, layer-major, read during the call
 * only; NULL means cfg->k / cfg->v everywhere.  Consecutive heads of a layer with equal (K, V)
 * formats form a head group with its own arena regions and launches (kvq_get_layout_head).
 * Every side is checked as in kvq_create; otherwise identical to kvq_arena_bytes / kvq_create.
 * The allocation itself (entropies, rounding, sink heads) is the caller's calibration. */
kvq_status kvq_arena_bytes_heads(const kvq_config* cfg, const kvq_side* head_k, const kvq_side* head_v,
                                 uint64_t* bytes);
kvq_status kvq_create_heads(const kvq_config* cfg, const kvq_side* head_k, const kvq_side* head_v, void* arena,
                            uint64_t arena_bytes, kvq_cache** out);

/* Release the handle and its split-K workspace; the caller-owned arena (the packed cache itself)
 * is left untouched and may be freed by the caller afterwards.  NULL is a no-op.  Synchronous
 * (cudaFree).  The pages manage no handle: their cache memory is what the configuration budgets
 * ([LCPP] "Finding 1": an f16 cache that no longer fits where the q4_0 one does; [E22L] "What I
 * tested": the bytes per token a 1M-token budget allows), and that memory belongs to the caller
 * here. */
void kvq_free(kvq_cache* cache);

/* Geometry of (layer, side) for inspection and tests: the head group holding kv-head `head`
 * (kvq_get_layout: kv-head 0).  Host only. */
kvq_status kvq_get_layout(const kvq_cache* cache, int32_t layer, int32_t side, kvq_layout* out);
kvq_status kvq_get_layout_head(const kvq_cache* cache, int32_t layer, int32_t side, int32_t head, kvq_layout* out);

/* Copy the per-channel K scale c [n_kv_heads][head_dim] (fp16, device) of `layer` into the
 * arena ([E21W] variants C/D: "calibrated offline").  Required before appending to a layer
 * whose K side has chan_scale = 1. */
kvq_status kvq_set_chan_scale(kvq_cache* cache, int32_t layer, const void* c_fp16, void* stream);

/* Set the stored length of every sequence of `layer` (-1: all layers) to `len` (0..capacity).
 * kvq_set_seq_len(cache, -1, 0, s) empties the cache. */
kvq_status kvq_set_seq_len(kvq_cache* cache, int32_t layer, int32_t len, void* stream);

/* Append n_new tokens to n_seqs sequences of `layer`.
 *   seq_ids: int32 device [n_seqs], the sequences that receive rows, distinct, in [0, batch);
 *            or NULL: every sequence in order (then n_seqs must equal batch).
 *   k, v:    fp16 device [n_seqs][n_kv_heads][n_new][head_dim] (16-byte aligned), row s for
 *            sequence seq_ids[s] (or s).
 * Token i of sequence b lands at position seq_len[b] + i (read on the device); every row is
 * quantized (pre-transform, group scales, codes, packing), rows in the anchor set are also
 * kept as fp16, and seq_len[b] += n_new.  Sequences not listed are untouched.  n_new = prompt
 * length is the bulk prefill; n_new = 1 is the decode-time append.
 * Errors: KVQ_ERR_INVALID_ARG for a bad pointer, layer or count; KVQ_ERR_CAPACITY if n_new >
 * capacity or, with seq_ids NULL, if the host-side length bound would pass capacity;
 * KVQ_ERR_STATE if a channel scale is required and was never set.  On the device (so also
 * under graph replay): a listed sequence with no room for all n_new rows gets none of them and
 * keeps its length (KVQ_ERRF_CAPACITY in the error word); an id outside [0, batch) is skipped
 * (KVQ_ERRF_SEQ_ID).  A repeated id is a caller error: its rows race and its length advances
 * once per listing.
 * Sources: [E22L] "What I tested" (keys and values quantized on entry to the cache), [FMKQ]
 * post 6 "Corrected semantics" (every layer quantized, anchors as extra protection). */
kvq_status kvq_quantize_append(kvq_cache* cache, int32_t layer, const void* k_fp16, const void* v_fp16,
                               const int32_t* seq_ids, int32_t n_seqs, int32_t n_new, void* stream);

/* Reconstruct tokens [t0, t0 + nt) of every (sequence, kv-head) of one side of `layer` into
 * out [batch][n_kv_heads][nt][head_dim] (fp32 if out_fp32 else fp16), device, caller-owned.
 * STORED domain: the grid values (code x scale + zero; polar m cos(phi), m sin(phi)
 * slot-interleaved) before any inverse transform, bit-exact by definition.  ORIGINAL domain:
 * inverse DFT, inverse rotation and x channel scale applied, and anchored rows replaced by
 * their fp16 copy.  Rows at or past a sequence's stored length hold whatever the arena held.
 * Errors: KVQ_ERR_INVALID_ARG for a bad layer, side, domain or range (t0 + nt > capacity).
 * Sources: the dequantized cache is what the pages' simulations attend over ([E22L] "What I
 * tested": keys and values quantized, then dequantized, on entry to the cache) and what their
 * K/V error is measured on ([E21W] "What I tested": squared error over signal energy; [E21W]
 * variants C/D: channel scales multiplied back after dequantizing). */
kvq_status kvq_dequantize(const kvq_cache* cache, int32_t layer, int32_t side, int32_t domain,
                          int32_t t0, int32_t nt, void* out, int32_t out_fp32, void* stream);

/* Decode attention for n_q query positions on `layer`.  q: fp16 device [n_q][n_q_heads]
 * [head_dim].  seq_ids: int32 device [n_q] (sequence each query reads) or NULL (query i reads
 * sequence i; needs n_q <= batch); an id outside [0, batch) attends nothing and raises
 * KVQ_ERRF_SEQ_ID in the error word.  kv_len: int32 device [n_q] (keys t < kv_len attended) or
 * NULL (the sequence's stored length).  out: [n_q][n_q_heads][head_dim], fp32 if out_fp32 else
 * fp16.  lse: fp32 device [n_q][n_q_heads] natural-log sum-exp of the scaled logits, or NULL.
 * Split-K over tokens, dequantizing in registers, query pre-transformed once (q' = H(c . q)
 * or the rFFT adjoint), partials merged by a second kernel that also undoes V's transform.
 * An empty key range gives out = 0 and lse = -inf.  Errors: KVQ_ERR_CAPACITY if n_q >
 * max_queries.  The split-K partials go to the handle's one workspace, shared by all layers:
 * decode calls on one handle must not overlap on the GPU (issue them on one stream, or order
 * the streams).  [E21W] "What I tested" (attention output, causal proxy queries). */
kvq_status kvq_decode_attention(kvq_cache* cache, int32_t layer, const void* q_fp16, int32_t n_q,
                                const int32_t* seq_ids, const int32_t* kv_len, void* out,
                                int32_t out_fp32, float* lse, void* stream);

/* kvq_decode_attention without any device allocation behind it.  Same arguments, same results,
 * same errors (KVQ_ERR_CAPACITY for n_q > max_queries included), plus KVQ_ERR_CAPACITY when the
 * split-K partials of this call (n_q x n_q_heads x (splits + 1) x (head_dim + 4) floats) exceed
 * the library's fixed scratch of 2^21 floats (8 MiB), and KVQ_ERR_INVALID_ARG when the current
 * device is not the handle's.  The pages have no counterpart: this is an interface convenience.
 * For callers that cannot call cudaMalloc where they decode: a serving runtime that hands
 * nearly all of HBM to its own pool and budgets every other byte, or a latency-critical decode
 * loop that must not make the implicit device synchronisation a cudaMalloc/cudaFree can cause.
 * The scratch is a file-scope device array that every GPU loading this library holds until the
 * process exits.  The first call on a device looks up that array's device address
 * (cudaGetSymbolAddress, with that device current) and keeps it; make that first call before
 * any stream capture, and do not use the call after a cudaDeviceReset (the kept address is then
 * stale).  All calls share the array, so calls that overlap on the GPU (different streams, or
 * different handles on one device) race; serialize them.  Each call writes every partial it
 * reads, so nothing is cleared between calls.  The handle from kvq_create keeps its own
 * workspace; this call leaves it alone. */
kvq_status kvq_decode_attention_noalloc(kvq_cache* cache, int32_t layer, const void* q_fp16, int32_t n_q,
                                        const int32_t* seq_ids, const int32_t* kv_len, void* out,
                                        int32_t out_fp32, float* lse, void* stream);

/* One decode step of `layer`: append n_new tokens to n_seqs sequences, then decode one query per
 * listed sequence over its whole new length.  Same results as kvq_quantize_append(cache, layer,
 * k, v, seq_ids, n_seqs, n_new) followed by kvq_decode_attention(cache, layer, q, n_seqs,
 * seq_ids, NULL, out, out_fp32, lse): the same codes, lengths and outputs.
 *   k, v, seq_ids, n_seqs, n_new: as kvq_quantize_append (ids distinct).
 *   q: fp16 device [n_seqs][n_q_heads][head_dim], query s for sequence seq_ids[s] (or s).
 *   out, out_fp32, lse: as kvq_decode_attention, one row per listed sequence.
 * Where a register-decode tensor-core kernel serves the layer's formats, the append needs no
 * key mean, int anchors or per-head formats, and the split-K grid fits in one wave of resident
 * CTAs (a latency-bound step), one split-K launch writes the new rows (each by the CTA that
 * reads it, before its tile copies) and decodes, and the merge advances the lengths: two
 * launches per layer instead of three (anchored layers add their anchor pass).  Elsewhere the
 * two calls run in turn.  kvq_last_launch_count tells which.  Errors: those of the two
 * calls (KVQ_ERR_CAPACITY also for n_seqs > max_queries); on the device, a listed sequence
 * without room for its rows gets none of them, keeps its length and is decoded over its old
 * rows (KVQ_ERRF_CAPACITY).  Shares the handle's workspace like kvq_decode_attention.
 * [FMKQ] post 6 "The winning recipe", component 2 (decode anchoring: each generated token is
 * appended, anchored or not, before the step attends over the cache); the single launch is an
 * engineering choice of this library, not the pages'. */
kvq_status kvq_append_decode(kvq_cache* cache, int32_t layer, const void* k_fp16, const void* v_fp16,
                             const int32_t* seq_ids, int32_t n_seqs, int32_t n_new, const void* q_fp16,
                             void* out, int32_t out_fp32, float* lse, void* stream);

/* Read and clear the device error word (KVQ_ERRF_* bits) into *flags.  Synchronizes the
 * device. */
kvq_status kvq_error_flags(kvq_cache* cache, int32_t* flags);

/* The 16 NF4 levels this library stores (fp16-exact values, ascending).  Host only. */
kvq_status kvq_nf4_levels(float out[16]);

/* The 2^bits Gaussian Lloyd-Max levels (bits 2..4) this library stores, in units of the
 * group RMS (fp16-exact values, ascending).  Host only. */
kvq_status kvq_lloyd_levels(int32_t bits, float* out);

/* Kernels launched by the last kvq_decode_attention / kvq_quantize_append call on this
 * handle (for launch accounting).  Host only. */
int32_t kvq_last_launch_count(const kvq_cache* cache);

const char* kvq_status_str(kvq_status s);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
