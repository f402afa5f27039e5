/*
 * kvq.h -- C ABI of the quantized KV-cache library (libkvq.so, sm_100a).
 *
 * What the library computes comes from these web pages on KV-cache
 * quantization (cited by title and section):
 *   [KIVI]  "Quantification du KV-Cache : TurboQuant et l'etat de l'art en
 *           2026", section "KIVI (2024) -- la quantification asymetrique par
 *           canal"; zubnet.ai survey of KV-cache compression techniques,
 *           paragraph "Famille deux, c'est la quantification".
 *   [TQ]    same survey paragraph; "La compression du cache KV est une decision
 *           d'infrastructure, pas un debat sur les modeles", section
 *           "TurboQuant est le choix de portabilite, pas le gagnant universel";
 *           "Quantification du KV-Cache ...", "TurboQuant : les cinq
 *           innovations" items 1-4.
 *   [DEC]   "La compression du cache KV ...", section "... quand la HBM, pas
 *           les FLOPs, est votre plafond" (every decoded token reads the whole
 *           cache); "Quantification du KV-Cache ...", "Le probleme" (the cache
 *           lets each new token look back without recomputation).
 *   [MERGE] "KV-cache compresse et modeles 4-bit : la compression s'impose
 *           comme le premier levier d'inference", section "Minima-KV : la
 *           compression sans eviction" (partial attention states merged by a
 *           globally normalised online softmax).
 *   [MIXED] the same section: recent and protected ("Anchor") pages in FP8,
 *           older pages in TQ3, one attention over both.
 *
 * Conventions for every call:
 *   - Ownership: the caller allocates and frees all device memory (cache
 *     buffer, inputs, outputs, workspace).  The library keeps only a small
 *     host-side handle; it never allocates device memory.
 *   - Pointers marked "device" must point to memory of the current CUDA device
 *     and be 16-byte aligned; 16-bit inputs are bf16 or fp16 bit patterns as
 *     the config says.  `stream` is a cudaStream_t (NULL = legacy default).
 *   - Asynchrony: every call only enqueues kernels on `stream` and returns.
 *     Argument errors are detected on the host and returned before anything is
 *     launched.  Conditions found on the device (non-finite input, a quantizer
 *     parameter that overflows fp16, a bounded wait that ran out) set bits of a
 *     status word inside the cache buffer; kvq_get_status reads it.
 *   - One handle must not be used from two streams at the same time.
 *   - No C++ exception crosses this interface.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer   */
  KVQ_ERR_UNSUPPORTED = 2,   /* config outside the supported shapes         */
  KVQ_ERR_CAPACITY = 3,      /* sequence would exceed max_seq                */
  KVQ_ERR_CUDA = 4,          /* a CUDA runtime call failed                   */
  KVQ_ERR_DEVICE_STATUS = 5  /* kvq_get_status: the device status word is set */
} kvq_status;

enum { KVQ_KIVI = 0, KVQ_TURBO = 1 };
enum { KVQ_BF16 = 0, KVQ_FP16 = 1 };

/* Device status bits (kvq_get_status). */
enum {
  KVQ_DEV_NONFINITE_INPUT = 1u << 0, /* a quantized input was inf or nan       */
  KVQ_DEV_PARAM_OVERFLOW = 1u << 1,  /* a scale or zero-point overflowed fp16  */
  KVQ_DEV_WAIT_TIMEOUT = 1u << 2,    /* a bounded pipeline wait gave up        */
  KVQ_DEV_BAD_PAGE = 1u << 3         /* a page table entry was outside the pool */
};

/*
 * Cache configuration.
 *   scheme        KVQ_KIVI (int2/int4 asymmetric, [KIVI]) or KVQ_TURBO ([TQ]).
 *   bits          KIVI: 2 or 4.  TURBO: 3 (codes per rotated coordinate).
 *   group         KIVI: G, tokens per key quantization group (32 or 64).
 *                 TURBO: tokens flushed from the window at a time (32).
 *   residual      R, tokens always kept unquantized (a multiple of group).
 *   head_dim      d: 64 or 128 (TURBO: 128).
 *   num_kv_heads, num_q_heads  Hkv and Hq; Hq / Hkv in {1, 2, 4, 8}; query
 *                 head h reads kv head h / (Hq / Hkv).
 *   batch         B sequences; all of them have the same length.
 *   max_seq       capacity in tokens per sequence.
 *   dtype         KVQ_BF16 or KVQ_FP16: the 16-bit format of k, v and q.
 *   qjl_dim       TURBO: m, rows of the 1-bit QJL sketch of the key residual
 *                 (128).  KIVI: 0.
 *   page_records  0: each row's records are contiguous in the cache buffer.
 *                 > 0: paged ("TurboQuant : les cinq innovations", item 3:
 *                 block-wise paged decoding stays possible because the
 *                 packing is aligned to token blocks).  The records live in
 *                 a pool of num_pages pages of page_records (a power of
 *                 two) records each
 *                 (a record = G tokens for KIVI, 32 for TURBO), and a block
 *                 table given to kvq_cache_set_page_table maps each row's
 *                 logical pages to pool pages.
 *   num_pages     paged caches: pages in the pool (>= 1); else 0.
 *   fp8_recent    TURBO only, 0 or 1: the mixed-format cache of [MIXED]:
 *                 the residual window and the anchor tokens are stored in
 *                 FP8 E4M3 with one fp16 scale per token vector
 *                 (s = RNE_fp16(max |x| / 448), codes RNE_e4m3(x / s)), and
 *                 window tokens leave for TQ3 from their FP8 values.
 *   anchor_tokens fp8_recent caches: A, a multiple of 32: the first A tokens
 *                 of every sequence (from the prefill, which then needs
 *                 seq_len >= A) stay in FP8 for good.  Else 0.
 */
typedef struct {
  int32_t scheme;
  int32_t bits;
  int32_t group;
  int32_t residual;
  int32_t head_dim;
  int32_t num_kv_heads;
  int32_t num_q_heads;
  int32_t batch;
  int32_t max_seq;
  int32_t dtype;
  int32_t qjl_dim;
  int32_t page_records;
  int32_t num_pages;
  int32_t fp8_recent;
  int32_t anchor_tokens;
} kvq_config;

/*
 * Where things live inside the caller's cache buffer (byte offsets from its
 * start).  For KIVI every (batch, kv head) row holds `groups_per_row` group
 * records of `record_bytes` each; a record packs G tokens: the key codes and
 * value codes of its 32-token blocks (16 INT2 or 8 INT4 codes per 32-bit word,
 * ordered so that a lane's word yields its mma fragments directly; the exact
 * bit order is the packed format v1 the oracle also implements), the fp16
 * (scale, zero) of each
 * key channel, and the fp16 (scale, zero) of each value token.  Each row also
 * owns a ring of `ring_tokens` 16-bit key rows and one of value rows (the
 * residual window).
 */
typedef struct {
  uint64_t total_bytes;      /* == kvq_cache_bytes                           */
  uint64_t records_offset;   /* [B][Hkv][groups_per_row][record_bytes]       */
  uint64_t record_bytes;     /* bytes of one group record (KIVI) or token    */
                             /* record (TURBO)                               */
  uint64_t groups_per_row;   /* record capacity of one row                   */
  uint64_t window_offset;    /* [B][Hkv][2 (k, v)][ring_tokens][d] 16-bit    */
  uint64_t ring_tokens;      /* R + group                                    */
  uint64_t params_offset;    /* TURBO: rotation, sketch and codebook         */
  uint64_t params_bytes;
  uint64_t status_offset;    /* uint32 device status word                    */
  uint64_t pages_per_row;    /* paged: block table entries per row (the pages */
                             /* that groups_per_row records fill); else 0      */
  uint64_t token_row_bytes;  /* bytes of one window token row of K or V: 2 d, */
                             /* or 144 for FP8 rows (128 E4M3 codes, the fp16 */
                             /* scale, 14 zero bytes)                         */
  uint64_t anchor_offset;    /* fp8_recent: [B][Hkv][2][A][token_row_bytes]   */
} kvq_layout;

typedef struct kvq_cache kvq_cache; /* opaque host handle */

/* Device bytes the caller must allocate for a cache of this config; 0 if the
 * config is invalid or unsupported. */
size_t kvq_cache_bytes(const kvq_config* cfg);

/* Device scratch bytes kvq_decode_attention needs: the split-K partial states
 * and, for TURBO, the rotated query of every (batch, kv head) row; 0 if the
 * config is invalid. */
size_t kvq_workspace_bytes(const kvq_config* cfg);

/* Fills *out with the buffer layout of a config. */
kvq_status kvq_get_layout(const kvq_config* cfg, kvq_layout* out);

/*
 * Creates a host handle over the caller's device buffer `dev_buf` (at least
 * kvq_cache_bytes(cfg) bytes, 256-byte aligned) and enqueues the clearing of
 * its status word on `stream`.  The cache starts empty.  On success *out owns
 * only host memory; release it with kvq_cache_destroy.
 */
kvq_status kvq_cache_init(const kvq_config* cfg, void* dev_buf, size_t bytes,
                          void* stream, kvq_cache** out);

/*
 * Paged caches only, after kvq_cache_init and before any call that touches
 * records: the block table, device int32 [B * Hkv][pages_per_row] (row-major,
 * caller-owned, 16-byte aligned).  Entry (row, p) is the pool page holding the
 * row's records p * page_records .. (p + 1) * page_records - 1; only entries
 * of pages a row's quantized tokens reach are read, so the caller may fill
 * them as rows grow (stream-ordered with the calls that use them).  Rows must
 * not share pages.  An entry outside [0, num_pages) is never dereferenced: the
 * access is skipped and KVQ_DEV_BAD_PAGE is set.  May be called again to
 * replace the table pointer.
 * Errors: KVQ_ERR_UNSUPPORTED for a contiguous cache; KVQ_ERR_INVALID_ARG for
 * a null or misaligned pointer.
 */
kvq_status kvq_cache_set_page_table(kvq_cache* cache, const int32_t* table);

/*
 * TURBO only, once after kvq_cache_init and before any prefill.  Derives the
 * deployment constants of [TQ] on the device and stores them in the cache
 * buffer:
 *   rot_gauss  device float32 [d][d]: a seeded N(0,1) draw; the rotation is
 *              the Q factor of its QR decomposition with diag(R) > 0, a random
 *              orthogonal matrix as [TQ] asks for.
 *   qjl_gauss  device float32 [m][d]: the N(0,1) QJL projection S, used as is.
 * The 8-level Lloyd-Max codebook for N(0, 1/d) ("TurboQuant : les cinq
 * innovations", item 2) is computed on the device as well.
 * Errors: KVQ_ERR_UNSUPPORTED for a KIVI cache; KVQ_ERR_INVALID_ARG for null
 * or misaligned pointers or a cache that already holds tokens.
 */
kvq_status kvq_turbo_setup(kvq_cache* cache, const float* rot_gauss, const float* qjl_gauss,
                           void* stream);

/*
 * As kvq_turbo_setup, with the Walsh-Hadamard rotation instead of a random
 * one ("TurboQuant : les cinq innovations", item 1): Pi = H_d / sqrt(d), H_d
 * the Sylvester-order Hadamard matrix (entry (i, j) = (-1)^popcount(i & j)),
 * stored as exactly +-fp32(1 / sqrt(d)).  The quantizer then applies Pi with
 * the fast transform (add/sub butterflies) instead of a d x d product.
 *   qjl_gauss  device float32 [m][d], as for kvq_turbo_setup.
 * Errors: as kvq_turbo_setup.
 */
kvq_status kvq_turbo_setup_wht(kvq_cache* cache, const float* qjl_gauss, void* stream);

/*
 * Prefill ([KIVI] / [TQ]).  k, v: device [B][Hkv][seq_len][d], 16-bit.
 * The cache must be empty.  Quantizes T_q = G * floor(max(0, seq_len - R) / G)
 * tokens per row and keeps the other seq_len - T_q tokens, unchanged, in the
 * residual window ("TurboQuant : les cinq innovations", item 4).
 * Errors: KVQ_ERR_CAPACITY if seq_len > max_seq; KVQ_ERR_INVALID_ARG for a
 * null or misaligned pointer, a negative length or a non-empty cache.
 */
kvq_status kvq_quantize_prefill(kvq_cache* cache, const void* k, const void* v, int32_t seq_len,
                                void* stream);

/*
 * One decode step's new token per row.  k_new, v_new: device [B][Hkv][d],
 * 16-bit.  The token enters the residual window; when the window then holds
 * R + G tokens, its oldest G tokens are quantized (one new key group and G
 * value tokens) and leave it.
 * Errors: KVQ_ERR_CAPACITY if the sequence would exceed max_seq.
 */
kvq_status kvq_append_token(kvq_cache* cache, const void* k_new, const void* v_new, void* stream);

/*
 * Single-token decode attention over the whole cache ([DEC], [MERGE]).
 *   q          device [B][Hq][d], 16-bit.
 *   out        device float32 [B][Hq][d]: softmax(scale * q.k_t) v_t summed
 *              over every cached token t, quantized tokens dequantized on the
 *              fly and window tokens exact.
 *   softmax_scale  usually 1/sqrt(d).
 *   workspace  device scratch of at least kvq_workspace_bytes(cfg) bytes; its
 *              contents need no initialisation and are overwritten.
 * Errors: KVQ_ERR_INVALID_ARG on an empty cache, null pointers or a short
 * workspace.
 */
kvq_status kvq_decode_attention(const kvq_cache* cache, const void* q, float* out, float softmax_scale,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * One whole decode step: kvq_append_token(cache, k_new, v_new) followed by
 * kvq_decode_attention(cache, q, out, ...), with the same results, cache
 * state and errors ([DEC]: the step on either side of the path).  When the
 * appended token does not complete a flush, both run as one kernel launch:
 * the attention reads the new token from k_new / v_new and stores it into the
 * residual window itself.  A step that flushes the window's oldest G tokens
 * quantizes them first, as kvq_append_token does, then attends.
 *   k_new, v_new   device [B][Hkv][d], 16-bit (as for kvq_append_token).
 *   q, out, softmax_scale, workspace, workspace_bytes, stream
 *                  as for kvq_decode_attention.
 * Errors: those of kvq_append_token and kvq_decode_attention, all detected
 * before anything is launched; on an error the cache state is unchanged.
 */
kvq_status kvq_append_decode(kvq_cache* cache, const void* k_new, const void* v_new, const void* q, float* out,
                             float softmax_scale, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Decode attention that allocates nothing and needs no workspace argument.
 * The pages have no counterpart for this call: it exists for callers that
 * cannot allocate device memory -- for example a plugin running inside a
 * serving engine that owns every device allocation and gives its plugins no
 * allocator, or a serving loop that forbids allocator calls once it is
 * running -- and so cannot provide the scratch space kvq_decode_attention
 * takes.  It computes the same result as kvq_decode_attention, using a
 * scratch array of KVQ_STATIC_WORKSPACE_BYTES compiled into this library
 * (every GPU that loads the library holds that array until the process exits).
 *   q, out, softmax_scale, stream  as for kvq_decode_attention.
 * Errors: KVQ_ERR_CAPACITY, before anything is launched, if this cache's
 * configuration needs more scratch than KVQ_STATIC_WORKSPACE_BYTES
 * (kvq_workspace_bytes(cfg) > KVQ_STATIC_WORKSPACE_BYTES); otherwise the
 * errors of kvq_decode_attention.
 * The first call on a device looks up the array's device address for that
 * device (cudaGetSymbolAddress, with that device current); make that first
 * call before any stream capture.  All calls share the one array and it keeps
 * the last call's contents (nothing in it needs to start at zero), so calls
 * whose GPU work overlaps -- on two streams, or on two caches at once -- race
 * and must be serialised by the caller.  No call allocates or frees memory.
 */
#define KVQ_STATIC_WORKSPACE_BYTES ((size_t)4 * 1024 * 1024)
kvq_status kvq_decode_attention_static(const kvq_cache* cache, const void* q, float* out, float softmax_scale,
                                       void* stream);

/*
 * Synchronises `stream`, reads the device status word into *bits (may be
 * NULL) and returns KVQ_ERR_DEVICE_STATUS if any bit is set, else KVQ_OK.
 * `clear` != 0 also zeroes the word and the per-row arrival counters of the
 * decode merge (enqueued on `stream`).
 * After KVQ_DEV_WAIT_TIMEOUT the outputs of the launch that set it are
 * unspecified, and so is the window slot of the new token when that launch
 * was a fused step (kvq_append_decode); the cache's other contents are
 * unchanged, and after a clear the next call computes normally.
 */
kvq_status kvq_get_status(kvq_cache* cache, uint32_t* bits, int32_t clear, void* stream);

/* Host-side counters (no device access). */
int32_t kvq_seq_len(const kvq_cache* cache);        /* tokens per sequence   */
int32_t kvq_quantized_len(const kvq_cache* cache);  /* T_q                   */
int32_t kvq_window_len(const kvq_cache* cache);     /* r = seq_len - T_q     */
int32_t kvq_window_head(const kvq_cache* cache);    /* ring slot of the oldest window token */

/*
 * Checkpoint / resume: sets the counters of a handle whose buffer already
 * holds a cache in the documented layout (e.g. restored by the caller).
 * Requires quantized_len % G == 0, window_head % G == 0, and
 * 0 <= seq_len - quantized_len < R + G.
 */
kvq_status kvq_cache_set_state(kvq_cache* cache, int32_t seq_len, int32_t quantized_len,
                               int32_t window_head);

void kvq_cache_destroy(kvq_cache* cache);

const char* kvq_status_string(kvq_status s);

/* Message of the CUDA error behind the calling thread's last KVQ_ERR_CUDA
 * ("no error" if there was none); a static string, never freed. */
const char* kvq_cuda_error_string(void);

/* Kernels this library has launched since it was loaded (all handles). */
uint64_t kvq_launch_count(void);

/*
 * Test hook for the bounded waits of the decode kernels and of the
 * tensor-core TurboQuant quantizer (no counterpart on the pages).  Every
 * pipeline wait inside such a launch gives up after a bound (default: about
 * 1 s of SM clock cycles); a wait that gives up sets KVQ_DEV_WAIT_TIMEOUT and
 * the launch finishes without writing outputs it cannot trust (a quantizer
 * CTA stops at a tile boundary: its remaining records are unspecified),
 * leaving the GPU context usable.  This call lets a test reach that path
 * without a GPU fault:
 *   wait_cycles           the bound in SM clock cycles for later launches of
 *                         these kernels in this process (0 restores the
 *                         default; values above the default are rejected);
 *   withhold_first_stage  nonzero: CTA 0 of later decode launches does not
 *                         issue the copy of its first pipeline stage, and CTA
 *                         0 of later tensor-core quantizer launches not the
 *                         copy of its operand images, so the waits on them
 *                         run out after `wait_cycles`.
 * Waits for copies already in flight before a CTA exits keep the default
 * bound.  Process-wide, not thread-safe against concurrent launches; for
 * tests only.  Returns KVQ_ERR_INVALID_ARG for a bound above the default.
 */
kvq_status kvq_debug_set_wait_test(uint64_t wait_cycles, int32_t withhold_first_stage);

/* Decode-attention split count the library picks for the current state. */
int32_t kvq_decode_splits(const kvq_cache* cache);

/* The decode work partition for a cache of configuration `cfg` holding
 * `n_groups` quantized groups (KIVI) or 32-token blocks (TURBO) and `r`
 * window tokens per row, on a GPU with `sms` multiprocessors.  A row's work
 * items are its quantized items, then its window chunks of 32 tokens (and, in
 * the mixed TURBO cache, its anchor chunks); *n_items receives their count.
 * CTA c of the decode launch owns the global items item0[c] .. item0[c+1]-1
 * (global item = row x n_items + item); item0[0] = 0, item0[n] = rows x
 * n_items, strictly increasing.  The ranges balance stages (a stage carries
 * up to 12 KIVI groups for G = 32, 6 for G = 64, or 11 TURBO blocks;
 * a window chunk's stage weighs 1.5 of them) and quantized ranges start at a
 * stage boundary of their row.  Fills item0[0 .. n] (caller-owned, `cap`
 * entries) and returns n, or 0 for a null pointer, an unsupported
 * configuration, n_groups < 0, r < 0, sms < 1 or cap < n + 1.  Host only: no
 * CUDA call.  The decode entry points use this partition with the current
 * GPU's multiprocessor count. */
int32_t kvq_decode_partition(const kvq_config* cfg, int64_t n_groups, int32_t r, int32_t sms, int32_t* item0,
                             int32_t cap, int32_t* n_items);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
