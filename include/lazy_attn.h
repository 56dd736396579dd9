/*
 * lazy_attn.h -- C ABI of a B200 (sm_100a) library for LazyAttention's hot
 * path: attention over a shared, paged KV cache whose keys are stored with
 * RoPE at document-local positions, with each request's document offsets
 * applied inside the kernels.
 *
 * Sources (three web pages about arXiv 2606.04302):
 *   [ABS] shd-paper.top, "LazyAttention: Efficient Retrieval-Augmented
 *         Generation with Deferred Positional Encoding" -- English abstract.
 *   [CORE], [PRE], [DEC], [EQV], [CON]: gist.science, same title --
 *         Technical Summary: Core Concept: Deferred Positional Encoding;
 *         Technical Implementation: Prefilling; Technical Implementation:
 *         Decoding; Mathematical Equivalence; Key Contributions.
 *   [RES] gist.science, same title -- Experimental Results (cache hit
 *         ratios under a KV budget).
 *
 * Conventions for every entry point
 *   - Pointers are DEVICE pointers unless marked "host".  bf16 tensors are
 *     passed as uint16_t bit patterns.  `stream` is a cudaStream_t (NULL =
 *     the legacy default stream).  Every launch is asynchronous on it.
 *   - Ownership: the caller allocates and frees every buffer (pools, tables,
 *     outputs, workspaces).  The library allocates no device memory and keeps
 *     no state between calls, except the fixed scratch array that
 *     lazy_decode_attn_noalloc uses (described at its declaration).
 *   - Errors found on the host (bad shapes, null pointers, a workspace too
 *     small) are returned BEFORE anything is launched.  A launch failure
 *     returns LAZY_ECUDA.
 *   - Errors found on the device (a block id >= num_blocks, a slot outside
 *     the pool, a segment that is not block-aligned, a bounded wait that ran
 *     out) are OR-ed into *d_status (a device int, may be NULL) as
 *     LAZY_DSTATUS_* bits; the affected unit of work is skipped (its output
 *     rows are written as zeros, or its pool slot is not written).  Nothing
 *     traps.
 *
 * Data layout
 *   - Pools: k_pool, v_pool are bf16 [num_blocks][Hkv][16][head_dim]; one
 *     16-token block of one KV head is 4 KiB contiguous.  Keys are stored as
 *     RoPE(k, j) at their local index j inside their segment ([CORE]; the
 *     pages leave open what is stored, and the local position is the plainest
 *     reading that lets one relative rotation per segment suffice [PRE]).
 *   - blk_meta: uint32 [num_blocks], one word per physical block:
 *     (j0 / 16) << 8 | n_valid, with j0 the local index of the block's first
 *     token and n_valid (1..16) the number of written slots.  lazy_kv_write
 *     maintains it; the caller zeroes the words of freshly allocated blocks.
 *   - Tables: per request r, table[table_indptr[r] .. table_indptr[r+1]) holds
 *     one 32-bit word per logical block, in logical order:
 *         word = (offset << 17) | block
 *     block = physical block id (17 bits), offset = logical offset of the
 *     block's segment in tokens (15 bits) ([DEC]: the block id and the offset
 *     are packed together into one register word).  Slot s of the block holds local
 *     index j0 + s and sits at logical position offset + j0 + s.  The same
 *     physical block may appear in many requests and several times in one
 *     request at different offsets; gaps between segments are legal.
 *   - Queries: bf16 [tokens][Hq][head_dim], unrotated.  Outputs: bf16, same
 *     shape.  Query head h reads KV head h / (Hq / Hkv) ([CON]: GQA/MQA).
 *   - Causal rule: a key at logical position t is visible to a query at
 *     position p iff t <= p.  A query that sees no key gets a zero row.
 *   - head_dim must be 128 and block_size 16.  Hq / Hkv must be an integer
 *     <= 32.
 */
#ifndef LAZY_ATTN_H
#define LAZY_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct lazy_attn_cfg {
    int num_q_heads;     /* Hq */
    int num_kv_heads;    /* Hkv; Hq % Hkv == 0, Hq / Hkv <= 32 */
    int head_dim;        /* must be 128 */
    int block_size;      /* must be 16 */
    float rope_base;     /* RoPE base, e.g. 500000; theta_i = base^(-2i/d) */
    float softmax_scale; /* <= 0 selects 1/sqrt(head_dim) */
    /* Optional: head_dim/2 RoPE frequencies theta_i (radians per position), in
     * place of base^(-2i/d) -- RoPE variants such as Llama-3.1 frequency
     * scaling.  NULL selects base^(-2i/d).  Read during the call only (the
     * caller keeps ownership); each value must be finite and >= 0, else
     * LAZY_EINVAL.  The deferred rotation is unchanged: every angle is
     * (position difference) x theta_i.  The pages name other relative
     * encodings as within reach of the method but fix no table. */
    const double *rope_theta;
    /* Optional: ALiBi in place of RoPE (ABI version 102).  NULL selects RoPE.
     * Otherwise num_q_heads slopes m_h (num_q_heads <= 128, else
     * LAZY_ESHAPE; each finite, else LAZY_EINVAL), read during the call only.
     * Nothing is rotated: lazy_kv_write stores keys exactly as given, and the
     * score of query head h at position p for the key at o + j gets
     * -m_h * (p - o - j), computed from the table word's offset and the
     * block's local index in the kernel, like the rotation angle of the RoPE
     * path ([CON] lists ALiBi among the encodings the method extends to).
     * The stored keys then carry no position at all, so the materialisation
     * and plain comparison entry points refuse ALiBi (LAZY_EINVAL).  With
     * ALiBi set, rope_base and rope_theta are ignored. */
    const double *alibi_slopes;
} lazy_attn_cfg;

/* Host-side return codes. */
enum {
    LAZY_OK = 0,
    LAZY_EINVAL = -1,     /* null pointer or negative count */
    LAZY_ERANGE = -2,     /* a table field overflows 17/15 bits, or a size is too large */
    LAZY_ESHAPE = -3,     /* head_dim != 128, block_size != 16, bad head counts (ALiBi: Hq > 128) */
    LAZY_EWORKSPACE = -4, /* workspace smaller than the matching *_workspace_bytes() */
    LAZY_ECUDA = -5       /* a CUDA launch or driver call failed */
};

/* Device-side status bits, OR-ed into *d_status. */
enum {
    LAZY_DSTATUS_BAD_BLOCK = 1,   /* a table word names a block >= num_blocks */
    LAZY_DSTATUS_BAD_SLOT = 2,    /* lazy_kv_write: slot outside the pool */
    LAZY_DSTATUS_BAD_ALIGN = 4,   /* lazy_kv_write: local index j and slot differ mod 16 */
    LAZY_DSTATUS_BAD_TABLE = 8,   /* a request has more words than max_words */
    LAZY_DSTATUS_TIMEOUT = 16     /* a bounded pipeline wait ran out (kernel bailed out) */
};

#define LAZY_BLOCK_BITS 17
#define LAZY_OFFSET_BITS 15
#define LAZY_MAX_BLOCKS (1u << LAZY_BLOCK_BITS)
#define LAZY_MAX_OFFSET ((1u << LAZY_OFFSET_BITS) - 1u)

/* Table-word codec, usable from host and device code.  No range check:
 * callers that cannot guarantee block < 2^17 and offset < 2^15 use
 * lazy_pack_words, which checks. */
static inline uint32_t lazy_pack(uint32_t block, uint32_t offset) { return (offset << LAZY_BLOCK_BITS) | block; }
static inline uint32_t lazy_block(uint32_t word) { return word & (LAZY_MAX_BLOCKS - 1u); }
static inline uint32_t lazy_offset(uint32_t word) { return word >> LAZY_BLOCK_BITS; }

/* Packs n (block, offset) pairs into table words.  HOST pointers.
 * Returns LAZY_ERANGE (and stops) at the first field that does not fit. */
int lazy_pack_words(const int32_t *block, const int32_t *offset, int64_t n, uint32_t *words);

/* Writes n_tok tokens' keys and values into the paged pools ([CORE], [ABS]):
 *   k_pool[slot/16][h][slot%16][:] = bf16_rne(RoPE(k_raw[t][h][:], local_j[t]))
 *   v_pool[slot/16][h][slot%16][:] = v_raw[t][h][:]
 *   blk_meta[slot/16] = max(blk_meta[slot/16], (local_j/16) << 8 | (slot%16 + 1))
 * k_raw, v_raw: bf16 [n_tok][Hkv][128], unrotated.  slot, local_j: int32 [n_tok].
 * RoPE is computed in fp32 with angles reduced in fp64.  A slot outside the
 * pool (LAZY_DSTATUS_BAD_SLOT) or with local_j % 16 != slot % 16
 * (LAZY_DSTATUS_BAD_ALIGN) is skipped.  Distinct tokens must use distinct slots. */
int lazy_kv_write(const lazy_attn_cfg *cfg, const uint16_t *k_raw, const uint16_t *v_raw, int n_tok,
                  const int32_t *slot, const int32_t *local_j, uint16_t *k_pool, uint16_t *v_pool,
                  uint32_t *blk_meta, int num_blocks, int *d_status, void *stream);

/* Workspace for lazy_decode_attn: split-K partial results. */
size_t lazy_decode_workspace_bytes(const lazy_attn_cfg *cfg, int num_req, int max_words);

/* One decode step: one query token per request over its table ([DEC]).
 * q_raw: bf16 [num_req][Hq][128]; q_pos: int32 [num_req] (the query's logical
 * position; its own key must already be in the pool, written by
 * lazy_kv_write).  max_words: host upper bound of words per request (sizes the
 * split-K grid and the workspace; a request with more words sets
 * LAZY_DSTATUS_BAD_TABLE).  out: bf16 [num_req][Hq][128].
 * The query is rotated by (q_pos - offset) in registers whenever a warp
 * meets a new segment offset; keys are used as stored, so the kernel reads
 * only K and V ([DEC]: its memory traffic equals that of plain paged attention).
 * Two launches: split-K attention, then a combine over splits. */
int lazy_decode_attn(const lazy_attn_cfg *cfg, const uint16_t *q_raw, const int32_t *q_pos, int num_req,
                     const uint32_t *table, const int32_t *table_indptr, int max_words,
                     const uint32_t *blk_meta, const uint16_t *k_pool, const uint16_t *v_pool,
                     int num_blocks, uint16_t *out, void *workspace, size_t ws_bytes, int *d_status,
                     void *stream);

/* lazy_decode_attn for callers that cannot allocate device memory.  The
 * paper has no counterpart: this is a deployment convenience of this library.
 * Some callers have no allocator to draw a workspace from (a plugin handed
 * only its input and output buffers by a serving engine), or must not call
 * cudaMalloc on their hot path because it synchronises the device.  This
 * variant keeps the split-K partials in a fixed array inside the library's
 * device image (lazy_decode_noalloc_capacity() bytes, 16 MiB, held by every
 * GPU that loads the library until the process exits) and allocates nothing.
 * Arguments and results are those of lazy_decode_attn minus the workspace.
 * Returns LAZY_ERANGE, before launching anything, when the call needs more
 * than the capacity (lazy_decode_workspace_bytes(cfg, num_req, max_words) >
 * capacity).  The first call on each device looks up the array's device
 * address (cudaGetSymbolAddress), so make that first call before any stream
 * capture; the address is looked up again when the device's current context
 * changes (e.g. after cudaDeviceReset).  All calls share the array: calls
 * that can overlap on the GPU (different streams or host threads) race and
 * must be serialised by the caller. */
int lazy_decode_attn_noalloc(const lazy_attn_cfg *cfg, const uint16_t *q_raw, const int32_t *q_pos, int num_req,
                             const uint32_t *table, const int32_t *table_indptr, int max_words,
                             const uint32_t *blk_meta, const uint16_t *k_pool, const uint16_t *v_pool,
                             int num_blocks, uint16_t *out, int *d_status, void *stream);

/* Bytes of the built-in scratch array used by lazy_decode_attn_noalloc. */
size_t lazy_decode_noalloc_capacity(void);

/* Workspace for lazy_prefill_attn on the current device.  The prefill work is
 * one unit per 256 query rows of one KV head of one request, one CTA per SM;
 * when the last wave of units would leave at least half of the SMs idle, each
 * of its units runs as two CTAs over the two halves of the request's table
 * words, and their partial results (fp32 O, running max and sum per row) are
 * merged by a second kernel.  This returns the bytes those partial results
 * need (0 when no unit is split); lazy_prefill_attn balances the last wave
 * only when given at least that much workspace, and runs unsplit otherwise.
 * The result does not depend on the split beyond fp32 rounding order. */
size_t lazy_prefill_workspace_bytes(const lazy_attn_cfg *cfg, int num_req, int total_q, int max_q,
                                    int max_words);

/* Causal prefill of a chunk of query tokens per request over its table ([PRE]).
 * q_raw: bf16 [total_q][Hq][128]; request r owns tokens cu_q[r] .. cu_q[r+1]-1
 * at positions q_pos0[r] + i.  max_q: host upper bound of tokens per request;
 * max_words as for decode.  out: bf16 [total_q][Hq][128].
 * Each CTA (256 query rows of one KV head) rotates its query rows once by
 * (p_i - P0), P0 its first query position, and every key tile once by
 * (o - P0), o the tile's segment offset: one relative rotation per tile, not
 * a reset to position 0 and a re-rotation; scores carry (p_i - o - j).
 * Tensor cores (tcgen05, accumulators in tensor memory); with the workspace
 * of lazy_prefill_workspace_bytes, a second kernel merges split units.
 * Under ALiBi (cfg.alibi_slopes) nothing is rotated and the bias is added to
 * the scores instead. */
int lazy_prefill_attn(const lazy_attn_cfg *cfg, const uint16_t *q_raw, const int32_t *cu_q,
                      const int32_t *q_pos0, int num_req, int total_q, int max_q,
                      const uint32_t *table, const int32_t *table_indptr, int max_words,
                      const uint32_t *blk_meta, const uint16_t *k_pool, const uint16_t *v_pool,
                      int num_blocks, uint16_t *out, void *workspace, size_t ws_bytes, int *d_status,
                      void *stream);

/* ---- one serving step: prefill chunks and decodes in one call ---- */

/* The arguments of lazy_prefill_attn for one batch of prefill chunks. */
typedef struct lazy_prefill_batch {
    const uint16_t *q_raw;
    const int32_t *cu_q;
    const int32_t *q_pos0;
    int num_req, total_q, max_q;
    const uint32_t *table;
    const int32_t *table_indptr;
    int max_words;
    uint16_t *out;
    void *workspace;
    size_t ws_bytes;
} lazy_prefill_batch;

/* The arguments of lazy_decode_attn for one batch of decodes. */
typedef struct lazy_decode_batch {
    const uint16_t *q_raw;
    const int32_t *q_pos;
    int num_req;
    const uint32_t *table;
    const int32_t *table_indptr;
    int max_words;
    uint16_t *out;
    void *workspace;
    size_t ws_bytes;
} lazy_decode_batch;

/* A serving step that holds both prefill chunks and decodes over one pool
 * (the mixed batches of a continuous-batching engine, as in the vLLM setting
 * of [RES]).  The results are exactly those of lazy_prefill_attn(prefill)
 * and lazy_decode_attn(decode) (the same kernels on the same inputs); the
 * difference is scheduling.  Both batches are validated on the host before
 * anything is enqueued, so an error leaves nothing half-launched.  Then
 * the prefill and the decode run in that order on `stream`, so work
 * enqueued on `stream` afterwards sees both outputs.  (Running the two
 * concurrently, the decode on the SMs the prefill's grid leaves idle, was
 * measured 3-5 % slower on B200, with small and large prefill batches.)
 * Either batch may be NULL or empty.  The two workspaces must be distinct
 * buffers (LAZY_EINVAL otherwise).  The call captures into a CUDA graph like
 * the two separate calls. */
int lazy_mixed_attn(const lazy_attn_cfg *cfg, const lazy_prefill_batch *prefill, const lazy_decode_batch *decode,
                    const uint32_t *blk_meta, const uint16_t *k_pool, const uint16_t *v_pool, int num_blocks,
                    int *d_status, void *stream);

/* ---- comparison paths (the position-aware alternative the pages argue against) ---- */

/* Materialises position-adjusted keys ([ABS]: copying keys re-encoded for
 * their positions is the cost the method avoids): for every table word w
 * (global index into table,
 * 0 <= w < total_words) with block b and offset o,
 *   k_mat[w][h][s][:] = bf16_rne(RoPE(k_pool[b][h][s][:], o))   for s < n_valid(b)
 *   k_mat[w][h][s][:] = 0                                        otherwise
 * i.e. keys rotated to their absolute positions o + j.  k_mat: bf16
 * [total_words][Hkv][16][128]. */
int lazy_materialize_k(const lazy_attn_cfg *cfg, const uint32_t *table, int total_words,
                       const uint32_t *blk_meta, const uint16_t *k_pool, int num_blocks,
                       uint16_t *k_mat, int *d_status, void *stream);

/* Plain paged attention over materialised keys: the same kernels with the
 * deferred rotation removed.  Keys come from k_mat (indexed by the word's
 * global table index, as written by lazy_materialize_k), values from v_pool
 * (indexed by the word's block), and the query is rotated once, at its
 * absolute position.  Arguments otherwise as lazy_decode_attn /
 * lazy_prefill_attn, whose workspace sizes apply. */
int lazy_plain_decode_attn(const lazy_attn_cfg *cfg, const uint16_t *q_raw, const int32_t *q_pos,
                           int num_req, const uint32_t *table, const int32_t *table_indptr,
                           int max_words, const uint32_t *blk_meta, const uint16_t *k_mat,
                           int total_words, const uint16_t *v_pool, int num_blocks, uint16_t *out,
                           void *workspace, size_t ws_bytes, int *d_status, void *stream);

int lazy_plain_prefill_attn(const lazy_attn_cfg *cfg, const uint16_t *q_raw, const int32_t *cu_q,
                            const int32_t *q_pos0, int num_req, int total_q, int max_q,
                            const uint32_t *table, const int32_t *table_indptr, int max_words,
                            const uint32_t *blk_meta, const uint16_t *k_mat, int total_words,
                            const uint16_t *v_pool, int num_blocks, uint16_t *out, void *workspace,
                            size_t ws_bytes, int *d_status, void *stream);

/* ---- block cache (host side): what the shared pool holds ---- */

/* A keyed LRU cache over pool blocks 0 .. capacity_blocks-1 ([ABS], [RES]:
 * one physical copy per document, reused at any position; the pages compare
 * its hit ratio with position-aware caching, one copy per (document, offset),
 * and with prefix caching).  The caching policy is the caller's key: the
 * document id (position-agnostic), a hash of (document, offset)
 * (position-aware) or of the whole preceding document sequence (prefix).
 * Host memory only; not thread-safe (one cache per scheduling thread).
 * Returns NULL for capacity_blocks <= 0, > LAZY_MAX_BLOCKS or no memory. */
typedef struct lazy_block_cache lazy_block_cache;
lazy_block_cache *lazy_cache_create(int64_t capacity_blocks);
void lazy_cache_destroy(lazy_block_cache *cache);

/* One use of the entry `key` of n_blocks blocks.  Hit: writes its block ids
 * to blocks[0..n_blocks-1], makes it the most recently used entry, returns 1
 * (LAZY_EINVAL if it was cached with another size).  Miss: evicts least
 * recently used entries until n_blocks are free, allocates them (consecutive
 * when one free extent holds them all), writes their ids and returns 0; the
 * caller then writes the document's keys and values there (lazy_kv_write).
 * An entry larger than the whole cache is counted as a miss and not cached:
 * LAZY_ERANGE. */
int lazy_cache_access(lazy_block_cache *cache, uint64_t key, int32_t n_blocks, int32_t *blocks);

/* 1 if key is cached, 0 if not. */
int lazy_cache_contains(const lazy_block_cache *cache, uint64_t key);

/* stats[8]: hits, misses, hit blocks, miss blocks, evictions, blocks in use,
 * cached entries, free extents. */
int lazy_cache_stats(const lazy_block_cache *cache, int64_t *stats);

/* ---- position-encoding tables (host) ----
 * Tables for lazy_attn_cfg.rope_theta and lazy_attn_cfg.alibi_slopes ([CON]:
 * the deferred encoding carries over to other relative encodings, RoPE
 * variants and ALiBi; the pages fix no table, so each function follows the
 * published rule it names).  All pointers are HOST pointers to caller-owned
 * arrays; nothing is launched.  Each returns LAZY_OK, or LAZY_EINVAL (and
 * writes nothing) for a null pointer or an argument outside its domain. */

/* theta[i] = base^(-2i/head_dim), i < head_dim/2 (head_dim even, base > 1):
 * the table the kernels use when rope_theta is NULL. */
int lazy_rope_theta(double base, int head_dim, double *theta);

/* Llama-3.1 frequency scaling (the "llama3" rope type of the Llama 3.1 model
 * configuration; Llama 3.1 itself uses base 500000, factor 8, low 1, high 4,
 * original context 8192).  With f_i = base^(-2i/head_dim) and wavelength
 * 2 pi / f_i: wavelengths below original_max_position / high_freq_factor keep
 * f_i, those above original_max_position / low_freq_factor get f_i / factor,
 * and in between theta_i = t f_i + (1 - t) f_i / factor with
 * t = (original_max_position / wavelength - low) / (high - low).
 * Needs factor > 0, 0 < low_freq_factor < high_freq_factor,
 * original_max_position > 0.  theta: head_dim/2 doubles. */
int lazy_rope_theta_llama31(double base, int head_dim, double factor, double low_freq_factor,
                            double high_freq_factor, double original_max_position, double *theta);

/* ALiBi head slopes (Press, Smith and Lewis, "Train Short, Test Long", 2022):
 * for a power of two n, slope k = 2^(-8k/n), k = 1..n; otherwise the slopes
 * of the largest power of two p below num_heads, then every second slope
 * (1st, 3rd, ...) of the 2p-head rule, num_heads - p of them.
 * slopes: num_heads doubles (num_heads >= 1). */
int lazy_alibi_slopes(int num_heads, double *slopes);

/* ---- test export ---- */

/* Decodes n_words table words on the device, exactly as the attention kernels
 * do, into per-slot records: out_block[16w+s] = block, out_slot[16w+s] =
 * 16*block + s, out_pos[16w+s] = offset + j0 + s if s < n_valid else -1.
 * A block id >= num_blocks gives -1 records and LAZY_DSTATUS_BAD_BLOCK. */
int lazy_debug_decode_table(const uint32_t *table, int64_t n_words, const uint32_t *blk_meta,
                            int num_blocks, int32_t *out_block, int32_t *out_slot, int32_t *out_pos,
                            int *d_status, void *stream);

/* Exercises the bounded pipeline wait that every warp-specialised kernel of
 * the library uses, without stalling a real pipeline: one CTA arms an
 * mbarrier that nothing completes (complete = 0) and waits on it for at most
 * `polls` polls (1 .. 2^24), as a consumer whose copy never lands would; the
 * wait gives up, ORs LAZY_DSTATUS_TIMEOUT into *d_status and raises the CTA's
 * abort flag, and a second role waiting on another barrier leaves through
 * that flag.  result: device int32[2] -- result[0] = 1 if the first wait ran
 * out, result[1] = 1 if the second role left through the abort flag.  With
 * complete != 0 both barriers complete first: both waits succeed, result is
 * {0, 0} and nothing is reported.  LAZY_EINVAL for a null result or a poll
 * count outside 1 .. 2^24. */
int lazy_debug_bounded_wait(uint32_t polls, int complete, int32_t *result, int *d_status, void *stream);

/* Text for a host return code (static storage). */
const char *lazy_strerror(int code);

/* Library ABI version (major * 100 + minor). */
int lazy_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LAZY_ATTN_H */
