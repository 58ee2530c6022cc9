/*
 * kv4.h -- C ABI of a paged INT4 KV cache with INT8-protected positions and
 * its decode attention, for NVIDIA B200 (sm_100a).
 *
 * What it computes
 * ----------------
 * New keys/values of each token are rotated by a block-diagonal Hadamard
 * transform and quantized token-wise (one group per token, KV head and K/V)
 * to asymmetric INT4 with an fp16 scale and zero point, then written into the
 * page of a paged cache that the block table names ("SAW-INT4: System-Aware
 * 4-Bit KV-Cache Quantization for Real-World LLM Serving", Abstract).  A
 * bounded set of positions -- the first S tokens (attention sinks) and the
 * W most recent tokens -- is also kept in INT8 and read from there ("KV4-RL:
 * Unlocking Faster Asynchronous Rollouts for RLVR with INT4 KV Cache
 * Quantization", Abstract).  Decode attention rotates the bf16 queries by the
 * same Hadamard transform, attends over the mixed INT4/INT8 cache and rotates
 * the output back.
 *
 * Alternative page format: with page_format = KV4_FORMAT_NVFP4 the pages hold
 * NVFP4 instead of INT4 ("KV Cache Quantization" topic page, item 3: the
 * NVFP4 paged KV cache of SGLang, about 56 % of the FP8 bytes per token):
 * E2M1 codes in blocks of 16 dims sharing one E4M3 scale (per-tensor scale
 * 1), after the same rotation; the INT8 store of the protected positions and
 * every entry point are the same.  With KV4_FORMAT_INT2 they hold 2-bit codes
 * of the same token-wise quantizer ("KV Cache Quantization" topic page, item
 * 2: INT2 KV with the scale and offset folded into the other operand and the
 * partial product, as the attention kernel does for INT4).
 *
 * Conventions
 * -----------
 * - Every function returns KV4_OK (0) or a negative KV4_ERR_* code; nothing
 *   aborts the process.  Kernels run asynchronously on the given stream; a
 *   fault found on the device (bad block-table entry, capacity overflow,
 *   out-of-range input, a wait that gave up) sets a bit in a device status
 *   word and skips the affected write, it never traps.  Read the word with
 *   kv4_get_status().
 * - All device pointers are caller-owned, 16-byte aligned (the cache buffer
 *   and the workspace 256-byte aligned), and must stay valid until the work
 *   queued on the stream has finished.  The library never allocates device
 *   memory.  A cache lives on the device that holds its buffer; every call on
 *   it runs there, whatever device the calling thread has selected, and the
 *   stream must belong to that device.  A call makes that device current only
 *   for its own duration: the calling thread's current device is the same
 *   before and after it.
 * - Calls on one cache handle must be ordered on one stream; a handle is not
 *   thread-safe.  Caches on different handles are independent.
 * - Keys arrive after RoPE, unless the RoPE entry points below (kv4_set_rope,
 *   kv4_rope_rotate_quantize_append, KV4_MODE_ROPE_Q) apply it on the way in.
 * - GQA grouping is contiguous: query head j reads KV head j / (Hq / Hkv).
 * - bf16 arrays are IEEE bfloat16 bit patterns (uint16); the layout of the
 *   cache buffer is defined by this library (16-token tiles whose byte order
 *   follows the tensor-core operand order of the attention kernel).
 */
#ifndef KV4_H
#define KV4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t); NULL means the legacy default stream. */
typedef struct CUstream_st* kv4_stream_t;

/* Return codes. */
enum {
  KV4_OK = 0,
  KV4_ERR_INVALID_ARG = -1,   /* a null pointer, a negative count, a misaligned pointer   */
  KV4_ERR_UNSUPPORTED = -2,   /* a shape the library does not support (see kv4_config)    */
  KV4_ERR_CAPACITY = -3,      /* a buffer smaller than kv4_cache_required_bytes()          */
  KV4_ERR_CUDA = -4,          /* a CUDA runtime call or launch failed                      */
  KV4_ERR_DEVICE_FAULT = -5,  /* kv4_get_status() found device status bits set             */
  KV4_ERR_WORKSPACE = -6,     /* workspace smaller than kv4_attention_workspace_bytes()    */
  KV4_ERR_SCRATCH = -7        /* kv4_decode_attention_noalloc: the call needs more scratch
                                 than KV4_NOALLOC_SCRATCH_BYTES                             */
};

/* Bits of the device status word. */
enum {
  KV4_DEV_BAD_PAGE = 1,       /* block-table entry < 0 or >= num_pages: token not written  */
  KV4_DEV_OVERFLOW = 2,       /* append past max_pages_per_seq * page_size: seq skipped    */
  KV4_DEV_RANGE = 4,          /* a rotated value was non-finite or beyond +-65504: clamped  */
  KV4_DEV_TIMEOUT = 8,        /* a bounded wait inside a kernel gave up (~1 s)              */
  KV4_DEV_BAD_SEQ = 16,       /* a sequence id outside [0, max_seqs): entry skipped        */
  KV4_DEV_WORKSPACE = 32,     /* the attention plan did not fit the workspace              */
  KV4_DEV_ROPE_POS = 64,      /* a position at or past the RoPE table: key not written,
                                 query rotated with the table's last row                    */
  KV4_DEV_BAD_CU = 128        /* append row offsets not 0 = cu[0] <= ... <= cu[n] =
                                 total_new: nothing appended, no length changed              */
};

/* RoPE pair layouts (kv4_set_rope). */
enum {
  KV4_ROPE_NEOX = 0,          /* pairs (i, i + R/2): "rotate half"                          */
  KV4_ROPE_GPTJ = 1           /* pairs (2i, 2i + 1): interleaved                            */
};

/* kv4_decode_attention / kv4_extend_attention mode bits.
 * KV4_MODE_Q_ROTATED and KV4_MODE_OUT_ROTATED let a caller fold the block
 * Hadamard H (normalised, symmetric, its own inverse) into its projections:
 * with W_q' = H W_q the query arrives rotated (q' = H q, bf16), and with
 * o_proj' = o_proj H the attention output can stay in the rotated basis.  The
 * kernels then skip that rotation (the query is used as given, no extra
 * rounding).  The rotated cache is unchanged.  The BF16 baseline cache ignores
 * both bits (it has no rotation). */
enum {
  KV4_MODE_PROTECTED = 0,     /* INT8 for protected positions, INT4 elsewhere (the method) */
  KV4_MODE_INT4_ONLY = 1,     /* read the pages (INT4 or NVFP4) for every position         */
  KV4_MODE_OUT_F32 = 2,       /* write fp32 output instead of bf16 (checking mode)          */
  KV4_MODE_Q_ROTATED = 4,     /* q is already H q: do not rotate it                         */
  KV4_MODE_OUT_ROTATED = 8,   /* write the output in the rotated basis (H o): no inverse    */
  KV4_MODE_ROPE_Q = 16        /* apply the cache's RoPE table to q at its position first    */
};

/* Page formats (kv4_config.page_format). */
enum {
  KV4_FORMAT_INT4 = 0,        /* token-wise asymmetric INT4, fp16 scale and zero point      */
  KV4_FORMAT_NVFP4 = 1,       /* E2M1 codes, one E4M3 scale per 16 dims (values beyond
                                 +-2688 saturate)                                          */
  KV4_FORMAT_INT2 = 2         /* token-wise asymmetric INT2, fp16 scale and zero point      */
};

/* kv4_dequantize_debug views. */
enum {
  KV4_VIEW_EFFECTIVE = 0,     /* what attention reads in KV4_MODE_PROTECTED                 */
  KV4_VIEW_INT4 = 1           /* the page copy (INT4 or NVFP4) of every position            */
};

/*
 * Cache configuration.
 *   num_layers          >= 1   independent per-layer caches sharing one block table
 *   max_seqs            >= 1   sequence ids are 0 .. max_seqs-1
 *   num_q_heads         Hq, a multiple of num_kv_heads with Hq/Hkv <= 8
 *   num_kv_heads        Hkv >= 1
 *   head_dim            D, 64 or 128
 *   page_size           P, a multiple of 16, at most 1024
 *   num_pages           pages in each layer's pool
 *   max_pages_per_seq   columns of the block table
 *   hadamard_block      Bh, a power of two dividing D (1 = no rotation)
 *   sink_tokens         S >= 0
 *   recent_window       W >= 1, S + W <= 4096
 *   page_format         KV4_FORMAT_INT4 (0), KV4_FORMAT_NVFP4 (1) or
 *                       KV4_FORMAT_INT2 (2); the BF16 baseline cache needs 0
 */
typedef struct {
  int32_t num_layers, max_seqs, num_q_heads, num_kv_heads, head_dim;
  int32_t page_size, num_pages, max_pages_per_seq;
  int32_t hadamard_block;
  int32_t sink_tokens, recent_window;
  int32_t page_format;
} kv4_config;

typedef struct kv4_cache kv4_cache;   /* opaque host handle owned by the library */

/* Bytes of device memory a cache with this configuration needs (INT4 pools,
 * INT8 sink/ring stores, sequence lengths and a small state block). */
int kv4_cache_required_bytes(const kv4_config* cfg, size_t* bytes);

/* Create a cache inside the caller's device buffer `dev_buf` (>= required
 * bytes, 256-byte aligned).  `dev_block_table` is caller-owned device memory,
 * int32 [max_seqs][max_pages_per_seq]: entry [s][i] is the page (in every
 * layer's pool) holding positions [i*P, (i+1)*P) of sequence s, -1 when
 * unmapped; the caller may update it between calls.  Sequence lengths and the
 * state block are zeroed on `stream`; pool contents stay undefined. */
int kv4_cache_create(const kv4_config* cfg, void* dev_buf, size_t bytes, int32_t* dev_block_table,
                     kv4_stream_t stream, kv4_cache** out);

/* Free the host handle (the device buffer stays the caller's). */
int kv4_cache_destroy(kv4_cache* cache);

/* Device addresses inside the cache buffer for layer `layer` (any pointer may
 * be NULL): the page pool, uint8 [num_pages][P/16][Hkv][16*D+128] (INT4),
 * [num_pages][P/16][Hkv][18*D] (NVFP4) or [num_pages][P/16][Hkv][8*D+128]
 * (INT2); the INT8 store, uint8 [max_seqs][ceil((S+W)/16)][Hkv][32*D+128];
 * and the sequence lengths int32 [num_layers][max_seqs] (all layers).  KV
 * heads are innermost, so the 16-token tiles of all heads at one page
 * position are contiguous (one bulk copy feeds a group of four heads). */
int kv4_cache_layout(const kv4_cache* cache, int32_t layer, void** dev_pages, void** dev_protected,
                     int32_t** dev_seq_lens);

/* Set the length of sequence `seq_id` to 0 in every layer (its pages can then
 * be reused or remapped). */
int kv4_seq_reset(kv4_cache* cache, int32_t seq_id, kv4_stream_t stream);

/*
 * Fused rotate + quantize + pack + append ("SAW-INT4 ...", Abstract: the
 * fused rotation-quantization kernel writing into the paged layout).
 *   dev_seq_ids  int32 [n_seqs], distinct sequence ids
 *   dev_cu_new   int32 [n_seqs+1], cu_new[0] = 0, non-decreasing; sequence
 *                seq_ids[i] receives rows cu_new[i] .. cu_new[i+1]-1
 *   total_new    = cu_new[n_seqs] (host copy, sizes the launch); offsets that
 *                break either rule set KV4_DEV_BAD_CU and append nothing
 *   k_new, v_new bf16 [total_new][Hkv][D], post-RoPE keys and values
 * Every new position p is INT4-encoded into page block_table[s][p / P], slot
 * p % P; positions p < S and p >= L_new - W are also INT8-encoded into the
 * sequence's protected store (sink slot p, or ring slot S + (p - S) mod W).
 * The sequence length of this layer advances by the number of new rows.
 * At most 3413 sequences per call (KV4_ERR_UNSUPPORTED above).
 */
int kv4_rotate_quantize_append(kv4_cache* cache, int32_t layer, const int32_t* dev_seq_ids,
                               const int32_t* dev_cu_new, int32_t n_seqs, int32_t total_new,
                               const void* k_new, const void* v_new, kv4_stream_t stream);

/*
 * RoPE fused into the append and the query kernel (the step before the
 * rotation: keys are rotated by position after RoPE, cf. the key transform
 * applied after RoPE on the method's pages).  kv4_set_rope registers a table
 * that stays owned by the caller and must outlive its use:
 *   dev_cos_sin  fp32 [max_pos][R]: row p holds cos(theta_{p,i}) for
 *                i = 0 .. R/2-1, then sin(theta_{p,i}) (any angles the model
 *                uses, e.g. theta_{p,i} = p * base^(-2i/R))
 *   rotary_dim   R: a power of two, 32 <= R <= D; dimensions >= R pass through
 *   style        KV4_ROPE_NEOX or KV4_ROPE_GPTJ
 * dev_cos_sin = NULL removes the table.  Pair (a, b) with angle i becomes
 * (a*c - b*s, b*c + a*s), each product and sum rounded to fp32 (no fused
 * multiply-add), on the fp32 value of the bf16 input; the result goes to the
 * Hadamard rotation in fp32 (no bf16 rounding in between).
 * kv4_rope_rotate_quantize_append is kv4_rotate_quantize_append with RoPE
 * applied to each new key at its position in the sequence (values are not
 * rotated); a key at position >= max_pos is not written and sets
 * KV4_DEV_ROPE_POS.  KV4_MODE_ROPE_Q applies RoPE to each query at its
 * position (decode: L - 1; kv4_extend_attention: L - q_len + i); it cannot
 * be combined with KV4_MODE_Q_ROTATED.  Without a table both return
 * KV4_ERR_INVALID_ARG.
 */
int kv4_set_rope(kv4_cache* cache, const float* dev_cos_sin, int32_t max_pos, int32_t rotary_dim, int32_t style);
int kv4_rope_rotate_quantize_append(kv4_cache* cache, int32_t layer, const int32_t* dev_seq_ids,
                                    const int32_t* dev_cu_new, int32_t n_seqs, int32_t total_new,
                                    const void* k_new, const void* v_new, kv4_stream_t stream);

/* Workspace bytes for kv4_decode_attention over up to `n_seqs` sequences of at
 * most `max_ctx` tokens each (max_ctx <= 0: the cache capacity
 * max_pages_per_seq * page_size). */
int kv4_attention_workspace_bytes(const kv4_cache* cache, int32_t n_seqs, int32_t max_ctx, size_t* bytes);

/*
 * Decode attention of one query token per sequence over every cached position
 * 0 .. L-1 of that sequence ("SAW-INT4 ...", Abstract: fused attention over
 * the paged quantized cache; "KV4-RL ...", Abstract: INT8 sinks and recent
 * context).
 *   dev_seq_ids    int32 [n_seqs]
 *   q              bf16 [n_seqs][Hq][D] (not yet rotated)
 *   out            bf16 [n_seqs][Hq][D] (fp32 with KV4_MODE_OUT_F32), in the
 *                  unrotated basis: softmax(scale * q_rot . K^) V^ rotated back
 *   softmax_scale  <= 0 means 1/sqrt(D)
 *   mode           KV4_MODE_* bits
 *   dev_workspace  >= kv4_attention_workspace_bytes(cache, n_seqs, max L, ...)
 * A sequence of length 0 gives an all-zero output row.  n_seqs <= max_seqs
 * (KV4_ERR_INVALID_ARG otherwise).  Calls on one cache must be ordered on one
 * stream (they share the cache's state block), and a workspace must not be
 * shared by calls that can run at the same time.
 * Steps: a query kernel (rotation, integer tensor-core operands), then one
 * persistent attention kernel: every CTA derives the same stream-K split of
 * all (sequence, KV-head group) page stages from the sequence lengths (groups
 * of 4 KV heads; of 2 or 1 when num_kv_heads is not a multiple of 4), streams
 * its stages through shared memory by bulk copies, turns INT4/INT8 codes into
 * operands in registers (online softmax) and stores the rotated-back output
 * of the groups it covers whole; groups split over several CTAs are finished
 * by a merge kernel (log-sum-exp merge of the workspace partials, inverse
 * rotation).  The three kernels are chained as programmatic dependents.
 */
int kv4_decode_attention(kv4_cache* cache, int32_t layer, const int32_t* dev_seq_ids, int32_t n_seqs,
                         const void* q, void* out, float softmax_scale, int32_t mode,
                         void* dev_workspace, size_t ws_bytes, kv4_stream_t stream);

/*
 * Multi-token query (speculative verification, extend): attention of the
 * last q_len cached positions of every sequence, each over the positions up
 * to and including its own.  Query token i (0 = oldest) of a sequence of
 * length L sits at position L - q_len + i and sees positions 0 .. L - q_len + i
 * of the same effective view as kv4_decode_attention (INT8 for the S sinks and
 * the last W positions of L, INT4 elsewhere; KV4_MODE_INT4_ONLY reads INT4 for
 * all).  Append the q_len tokens first.  With q_len = 1 this is
 * kv4_decode_attention.  ("SAW-INT4 ...", Abstract: fused attention over the
 * paged quantized cache; the causal mask over the new tokens is the textbook
 * one.)
 *   q_len          >= 1.  The query tokens and heads of one KV head share one
 *                  8-column tensor-core operand, so one pass over the cache
 *                  serves 8 / (Hq/Hkv) tokens; more tokens run as several
 *                  passes in stream order (q_len * Hq/Hkv <= 8: one pass)
 *   q, out         bf16 [n_seqs][q_len][Hq][D] (out fp32 with KV4_MODE_OUT_F32)
 *   dev_workspace  >= kv4_extend_workspace_bytes(cache, n_seqs, q_len, ...)
 * A query token with no visible position (L < q_len - i) gets an all-zero row.
 * Errors as kv4_decode_attention.  Same kernels as kv4_decode_attention,
 * with the operand columns standing for (query token, query head) pairs.
 */
int kv4_extend_workspace_bytes(const kv4_cache* cache, int32_t n_seqs, int32_t q_len, size_t* bytes);
int kv4_extend_attention(kv4_cache* cache, int32_t layer, const int32_t* dev_seq_ids, int32_t n_seqs, int32_t q_len,
                         const void* q, void* out, float softmax_scale, int32_t mode,
                         void* dev_workspace, size_t ws_bytes, kv4_stream_t stream);

/*
 * One decode step in one call: append one new token to every listed sequence
 * (as kv4_rotate_quantize_append with cu_new = 0, 1, ..., n_seqs), then
 * decode attention of q over the caches including that token (as
 * kv4_decode_attention).  Codes, lengths and outputs are those of the two
 * calls in a row.  With KV4_MODE_ROPE_Q the registered RoPE table is applied
 * to the new keys (as kv4_rope_rotate_quantize_append) and to the queries.
 *   k_new, v_new   bf16 [n_seqs][Hkv][D], the new token of entry i
 *   q, out, mode, softmax_scale, dev_workspace   as kv4_decode_attention
 *                  (the workspace of kv4_attention_workspace_bytes)
 * The sequence ids must be distinct.  Needs num_kv_heads <= 16
 * (KV4_ERR_UNSUPPORTED otherwise; use the two calls then).
 * Kernels: one block per sequence appends its token (two warps per KV head,
 * one for K and one for V) and builds the query operands, then the attention
 * and merge kernels of kv4_decode_attention: three launches instead of four.
 */
int kv4_decode_step(kv4_cache* cache, int32_t layer, const int32_t* dev_seq_ids, int32_t n_seqs,
                    const void* k_new, const void* v_new, const void* q, void* out, float softmax_scale,
                    int32_t mode, void* dev_workspace, size_t ws_bytes, kv4_stream_t stream);

/*
 * kv4_decode_attention_noalloc: kv4_decode_attention without a workspace
 * argument.  Its scratch (query operands and split-K partials) lives in a
 * static device array of this library, KV4_NOALLOC_SCRATCH_BYTES (16 MiB) per
 * device, so the call itself allocates nothing and needs no buffer from the
 * caller.  The method's pages have no counterpart of this call.
 *
 * For callers that cannot allocate device memory when they issue attention:
 * an inference loop that must not call an allocator between steps (a caching
 * allocator may synchronize the device or grow its pool at an arbitrary
 * step), or a caller that holds no device memory of its own for scratch.
 *
 * Arguments, results and errors are those of kv4_decode_attention, plus:
 *   KV4_ERR_SCRATCH when kv4_attention_workspace_bytes(cache, n_seqs, 0) is
 *   above KV4_NOALLOC_SCRATCH_BYTES (that is n_seqs * Hkv * (16*D + 64)
 *   bytes of query operands plus 2 * 3 * SMs * w * G * (D + 4) * 4 bytes of
 *   partials, w = 4, 2 or 1 KV heads per group, e.g. about 8.6 MB for
 *   64 sequences, 32/8 heads, D = 128 on 148 SMs, and 16.2 MB for 512);
 *   nothing is launched then.
 * The scratch is one per device and shared by every cache and stream of the
 * process on that device: calls that can run at the same time (two streams,
 * two host threads) race on it and give wrong results, so order them (one
 * stream, or events).  Nothing in it has to start at zero.  The first call
 * on a device looks the array up (cudaGetSymbolAddress, with the cache's
 * device current) and should come before any stream capture.  The address
 * is kept for the life of the process: do not use this call on a device
 * after cudaDeviceReset() (or any other teardown of its primary context).
 */
#define KV4_NOALLOC_SCRATCH_BYTES (16u << 20)
int kv4_decode_attention_noalloc(kv4_cache* cache, int32_t layer, const int32_t* dev_seq_ids, int32_t n_seqs,
                                 const void* q, void* out, float softmax_scale, int32_t mode,
                                 kv4_stream_t stream);

/* Dequantized keys/values of positions [start, start+count) of one sequence,
 * fp32 [count][Hkv][D], in the rotated basis: x^ = fma(code, s, z) from the
 * INT4 page or the INT8 store as `view` selects (NVFP4 pages: x^ = e2m1(code)
 * * e4m3(scale)).  For inspection and tests.  KV4_ERR_INVALID_ARG when the
 * range passes the sequence's capacity (max_pages_per_seq * page_size),
 * KV4_ERR_UNSUPPORTED when count * Hkv is too large for one launch; nothing
 * is launched then. */
int kv4_dequantize_debug(kv4_cache* cache, int32_t layer, int32_t seq_id, int32_t start, int32_t count,
                         int32_t view, float* dev_k_out, float* dev_v_out, kv4_stream_t stream);

/* Synchronize `stream`, return the device status word in *device_status and
 * clear it.  Returns KV4_ERR_DEVICE_FAULT when any bit was set. */
int kv4_get_status(kv4_cache* cache, kv4_stream_t stream, int32_t* device_status);

/* Timing hook: record the CUDA events `ev_before` and `ev_after` (cudaEvent_t,
 * created by the caller on the cache's device) on the call's stream right
 * before the first and right after the last attention kernel of every later
 * kv4_decode_attention call on this cache.  NULL, NULL turns it off.  The
 * events stay owned by the caller. */
int kv4_set_attention_events(kv4_cache* cache, void* ev_before, void* ev_after);

/* Testing hook for the bounded waits inside the attention kernel: in the
 * next kv4_decode_attention, kv4_decode_step or kv4_extend_attention call on
 * this cache (its first pass), the first CTA of the attention kernel does not
 * fill its stage number `stage` (counted from 0 in that CTA's share of the
 * work; no effect if the share is shorter).  That CTA's waits then give up
 * after about a second: the kernel lets its copies in flight land, sets
 * KV4_DEV_TIMEOUT and returns, the call's output is not valid, and later
 * calls on the cache are unaffected.  The hook applies to one call and then
 * clears itself; stage < 0 clears it.  Not for production use: it exists so
 * that tests can exercise the timeout path without a device fault. */
int kv4_test_stall_next_attention(kv4_cache* cache, int32_t stage);

/* Static text for a return code. */
const char* kv4_status_string(int status);

/* Build identification: "kv4 <version> sm_100a". */
const char* kv4_version(void);

typedef struct kv4bf16_cache kv4bf16_cache;   /* opaque host handle of the BF16 baseline cache */

/*
 * BF16 baseline cache: the same paging, block table, split-K attention and
 * merge, with bf16 keys/values stored as they arrive (no rotation, no
 * quantization, no protected store).  It exists to measure what the INT4
 * format saves; hadamard_block, sink_tokens and recent_window are ignored.
 * Page pool: bf16 [num_pages][P/16][Hkv][16-token tile of 32*D elements].
 * Each kv4bf16_* call takes the arguments of its kv4_* namesake, with the
 * same layouts, ownership and error codes: kv4bf16_append stores k_new and
 * v_new (bf16 [total_new][Hkv][D]) unchanged, with the same row-offset rules
 * and device status bits (KV4_DEV_BAD_PAGE, _OVERFLOW, _BAD_SEQ, _BAD_CU);
 * kv4bf16_decode_attention reads bf16 q [n_seqs][Hq][D] and writes out in
 * the same layout, with a workspace of kv4bf16_attention_workspace_bytes
 * bytes (max_ctx <= 0: the cache capacity).  kv4bf16_cache_layout has no
 * protected store to report.
 */
int kv4bf16_cache_required_bytes(const kv4_config* cfg, size_t* bytes);
int kv4bf16_cache_create(const kv4_config* cfg, void* dev_buf, size_t bytes, int32_t* dev_block_table,
                         kv4_stream_t stream, kv4bf16_cache** out);
int kv4bf16_cache_destroy(kv4bf16_cache* cache);
int kv4bf16_cache_layout(const kv4bf16_cache* cache, int32_t layer, void** dev_pages, int32_t** dev_seq_lens);
int kv4bf16_append(kv4bf16_cache* cache, int32_t layer, const int32_t* dev_seq_ids, const int32_t* dev_cu_new,
                   int32_t n_seqs, int32_t total_new, const void* k_new, const void* v_new, kv4_stream_t stream);
int kv4bf16_attention_workspace_bytes(const kv4bf16_cache* cache, int32_t n_seqs, int32_t max_ctx, size_t* bytes);
/* mode: only KV4_MODE_OUT_F32 is meaningful. */
int kv4bf16_decode_attention(kv4bf16_cache* cache, int32_t layer, const int32_t* dev_seq_ids, int32_t n_seqs,
                             const void* q, void* out, float softmax_scale, int32_t mode,
                             void* dev_workspace, size_t ws_bytes, kv4_stream_t stream);
int kv4bf16_get_status(kv4bf16_cache* cache, kv4_stream_t stream, int32_t* device_status);
int kv4bf16_set_attention_events(kv4bf16_cache* cache, void* ev_before, void* ev_after);

#ifdef __cplusplus
}
#endif

#endif /* KV4_H */
