/*
 * pkv - paged KV-cache decode attention for NVIDIA B200 (sm_100a).
 *
 * Plain C interface of libpkv.so.  Every pointer argument marked "device" is
 * caller-owned device memory; the library allocates nothing, frees nothing and
 * never synchronises the stream.  Work is enqueued on `stream` (a
 * cudaStream_t passed as void*, NULL = legacy default stream).  Argument
 * checks run on the host before anything is launched and return a status;
 * nothing is launched when a call returns an error.
 *
 * Layouts (row-major, innermost last):
 *   key / value (new rows)   [num_tokens, n_kv, head_dim]          act dtype
 *   key_cache / value_cache  [num_blocks, block_size, n_kv, head_dim] cache dtype
 *                            (INT4: [..., head_dim / 2] bytes)
 *   query / out              [num_seqs, n_q, head_dim]             act dtype
 *   block_tables             int32 [num_seqs, max_blocks_per_seq]
 *   context_lens             int32 [num_seqs]
 *   slot_mapping             int64 [num_tokens]
 *   k_scale / v_scale        INT8, INT4:     float [num_blocks, block_size, n_kv]
 *                            FP8 E4M3, E5M2: float [n_kv]
 * A physical block holds the K (or V) rows of block_size consecutive tokens
 * for all KV heads: "Chapter 18 - KV-Cache Optimization Strategies", How
 * PagedAttention Works (Physical KV Block figure: [block_size, G, d_k]).
 */
#ifndef PKV_H
#define PKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PKV_F32 = 0,      /* IEEE float32 */
  PKV_BF16 = 1,     /* bfloat16 */
  PKV_INT8 = 2,     /* int8 codes, one float scale per (token, head); cache only */
  PKV_FP8_E4M3 = 3, /* OCP E4M3 bytes, one float scale per KV head; cache only */
  PKV_FP8_E5M2 = 4, /* OCP E5M2 bytes, one float scale per KV head; cache only */
  PKV_INT4 = 5,     /* signed 4-bit codes, two per byte (element 2j in the low
                       nibble of byte j), one float scale per (token, KV head);
                       cache only, pools [num_blocks, block_size, n_kv, head_dim/2] */
  PKV_KIVI2 = 6     /* 2-bit KIVI cache (pkv_kivi_* calls and the block movers):
                       signed 2-bit codes, four per byte (element 4j + m in bits
                       [2m, 2m+1] of byte j), K scaled per (block, KV head,
                       channel), V per (token, KV head); pools [num_blocks, n_kv,
                       block_size, head_dim/4] (layout under pkv_kivi_decode) */
} pkv_dtype;

typedef enum {
  PKV_OK = 0,
  PKV_ERR_INVALID_ARG = 1, /* null pointer, negative size, misaligned pointer, bad combination */
  PKV_ERR_UNSUPPORTED = 2, /* valid but not implemented: head_dim, block_size, dtype pair, group size */
  PKV_ERR_WORKSPACE = 3,   /* workspace missing or smaller than pkv_paged_attention_workspace_size() */
  PKV_ERR_CUDA = 4         /* a CUDA runtime / driver call or a launch failed */
} pkv_status;

/* Bits OR-ed by the kernels into the optional int32 *device_error word.  An
 * offending entry is skipped (never dereferenced); results of the affected
 * sequence are then unspecified.  Kernels never trap. */
#define PKV_DEVERR_SLOT_RANGE 0x1   /* slot < -1 or slot >= num_blocks * block_size */
#define PKV_DEVERR_BLOCK_RANGE 0x2  /* block table entry outside [0, num_blocks) */
#define PKV_DEVERR_CONTEXT_LEN 0x4  /* context_len < 0, > max_context_len or > max_blocks_per_seq * block_size */
#define PKV_DEVERR_TIMEOUT 0x8      /* a bounded wait inside a kernel gave up (~1 s) */
#define PKV_DEVERR_PREFIX 0x10      /* shared-prefix decode: a block table does not begin with
                                       row 0's prefix_blocks entries */

/*
 * Append new tokens' K/V rows into their cache slots (reshape_and_cache).
 *
 * "Chapter 18 - KV-Cache Optimization Strategies", How PagedAttention Works:
 * new tokens fill the current block; the block table maps logical blocks to
 * physical ones (KV-cache overview page t13_4, block-table paragraph).  Row t
 * goes to row slot % block_size of physical block slot / block_size, where
 * slot = slot_mapping[t]; slot -1 skips the row.
 *
 *   key, value          device, [num_tokens, n_kv, head_dim], act_dtype (F32 or BF16)
 *   key_cache, value_cache device, [num_blocks, block_size, n_kv, head_dim], cache_dtype
 *   k_scale, v_scale    INT8 / INT4: device, written, one scale per (slot, head);
 *                       FP8_E4M3 / FP8_E5M2: device, read, one scale per KV head;
 *                       F32/BF16: must be NULL
 *   slot_mapping        device int64 [num_tokens]
 *   device_error        optional device int32 (NULL = not reported)
 *
 * Cache dtype rules: F32 cache needs F32 rows and BF16 cache needs BF16 rows
 * (bit copies).  INT8: per (token, head) absmax quantiser of "KV Cache
 * Engineering for LLM Serving", section 8, at 8 bits in IEEE float32:
 * scale = max|x| / 127, code = clamp(rint(x / scale), -127, 127) (ties to
 * even); an all-zero row stores scale 0 and codes 0.  INT4: the same rule at 4
 * bits, scale = max|x| / 7, codes -7..7 packed two per byte.  FP8_E4M3: code =
 * E4M3(x / scale_h) rounded to nearest-even, saturating at +-448; FP8_E5M2
 * likewise at +-57344; scale_h == 0 stores code 0.  head_dim must be 64, 128
 * or 256; pointers 16-byte aligned.
 * Slots of one call must be distinct, and must not lie in blocks shared by
 * several sequences (copy-on-write is the caller's job: Chapter 18, Prefix
 * Caching).
 */
pkv_status pkv_kv_cache_write(const void* key, const void* value, void* key_cache, void* value_cache, float* k_scale,
                              float* v_scale, const int64_t* slot_mapping, int64_t num_tokens, int n_kv, int head_dim,
                              int block_size, int64_t num_blocks, pkv_dtype act_dtype, pkv_dtype cache_dtype,
                              int32_t* device_error, void* stream);

/*
 * Bytes of device workspace pkv_paged_attention_decode needs for this shape on
 * the current device (0 when it needs none, e.g. an F32 cache).  Returns
 * (size_t)-1 when the shape is unsupported or the device cannot be queried.
 */
size_t pkv_paged_attention_workspace_size(int num_seqs, int n_q, int n_kv, int head_dim, int block_size,
                                          pkv_dtype cache_dtype);

/*
 * Single-token decode attention over a paged KV cache (PagedAttention).
 *
 * For sequence s and query head h (KV head kv = h / (n_q / n_kv), consecutive
 * grouping: "KV Cache Engineering for LLM Serving", section 1), over the
 * L = context_lens[s] cached tokens reached through block_tables[s]
 * (KV-cache overview page t13_4, block-table paragraph):
 *   score_p = sm_scale * <query[s,h,:], K_p[kv,:]>
 *   out[s,h,:] = sum_p softmax(score)_p * V_p[kv,:]
 *   lse_out[s,h] = log(sum_p exp(score_p))             (natural log; optional)
 * K_p / V_p are dequantised for INT8 / INT4 (code * scale[block,row,kv]) and
 * FP8 (value * scale[kv]) caches.  L == 0 gives out = 0, lse = -inf.
 * Entries of block_tables past ceil(L / block_size) are never read, and rows of
 * the last block past L never enter the softmax.
 *
 *   out                device, [num_seqs, n_q, head_dim], act_dtype
 *   query              device, [num_seqs, n_q, head_dim], act_dtype
 *   k_scale, v_scale   as for pkv_kv_cache_write (read only); NULL for F32/BF16
 *   max_context_len    host upper bound of context_lens (sizes the launch; no
 *                      device->host read happens)
 *   lse_out            optional device float [num_seqs, n_q]
 *   workspace          device scratch of workspace_bytes (any contents: every
 *                      byte is written before it is read), 16-byte aligned.
 *                      One workspace serves calls of any shape in stream order;
 *                      calls that may run concurrently need separate ones.
 *
 * A call on a BF16 or quantised cache makes two launches on `stream`: the decode kernel and,
 * queued behind it with programmatic stream serialisation, the merge of
 * sequences whose blocks were split over several CTAs.
 *
 * Supported: block_size 16; act F32 with an F32 cache (head_dim 32..256, a
 * multiple of 32); act BF16 with a BF16 cache (head_dim 64 or 128); act BF16
 * or F32 with an INT8, INT4, FP8_E4M3 or FP8_E5M2 cache (head_dim 128); n_q a
 * multiple of n_kv with n_q / n_kv <= 64.  Pointers 16-byte aligned.
 */
pkv_status pkv_paged_attention_decode(void* out, const void* query, const void* key_cache, const void* value_cache,
                                      const float* k_scale, const float* v_scale, const int32_t* block_tables,
                                      int max_blocks_per_seq, const int32_t* context_lens, int max_context_len,
                                      int num_seqs, int n_q, int n_kv, int head_dim, int block_size, int64_t num_blocks,
                                      float sm_scale, pkv_dtype act_dtype, pkv_dtype cache_dtype, float* lse_out,
                                      void* workspace, size_t workspace_bytes, int32_t* device_error, void* stream);

/*
 * One decode step in one launch: append each sequence's new token, then attend.
 *
 * Same result as pkv_kv_cache_write(key, value, ...) with slot_mapping[s] =
 * the slot of position context_lens[s] - 1 (block_tables[s][(L-1) / 16] * 16 +
 * (L-1) % 16), followed by pkv_paged_attention_decode(...).  New tokens fill
 * the current block ("Chapter 18 - KV-Cache Optimization Strategies", How
 * PagedAttention Works), and the decode then reads them through the block
 * table like every other row.
 *
 *   key, value   device, [num_seqs, n_kv, head_dim], act_dtype: the new
 *                token's rows; sequences with context_lens[s] == 0 append nothing
 *   key_cache, value_cache, k_scale, v_scale   as for pkv_kv_cache_write
 *                (INT8 scales are written, FP8 per-head scales are read)
 * Other arguments, shapes and errors as for pkv_paged_attention_decode.  In the
 * tensor-core path the CTA that reads a sequence's last block writes its new
 * rows first, so no second launch is needed.
 */
pkv_status pkv_paged_decode_step(void* out, const void* query, const void* key, const void* value, void* key_cache,
                                 void* value_cache, float* k_scale, float* v_scale, const int32_t* block_tables,
                                 int max_blocks_per_seq, const int32_t* context_lens, int max_context_len,
                                 int num_seqs, int n_q, int n_kv, int head_dim, int block_size, int64_t num_blocks,
                                 float sm_scale, pkv_dtype act_dtype, pkv_dtype cache_dtype, float* lse_out,
                                 void* workspace, size_t workspace_bytes, int32_t* device_error, void* stream);

/*
 * Decode attention over a sliding window with attention sinks.
 *
 * Like pkv_paged_attention_decode, but sequence s attends only to positions
 * p < min(sinks, L) and p >= L - window (L = context_lens[s]); window == 0
 * attends to every position.  A local layer keeps only its latest `window`
 * positions ("KV Cache Engineering for LLM Serving", section 3, Sliding
 * windows); StreamingLLM keeps the first tokens as attention sinks plus a recent
 * window ("Chapter 18 - KV-Cache Optimization Strategies", Token Eviction and
 * Pruning).  Blocks holding no attended position are never read, so their
 * block-table entries may be -1 once the engine has freed them.
 */
pkv_status pkv_paged_attention_decode_window(void* out, const void* query, const void* key_cache,
                                             const void* value_cache, const float* k_scale, const float* v_scale,
                                             const int32_t* block_tables, int max_blocks_per_seq,
                                             const int32_t* context_lens, int max_context_len, int num_seqs, int n_q,
                                             int n_kv, int head_dim, int block_size, int64_t num_blocks,
                                             float sm_scale, int window, int sinks, pkv_dtype act_dtype,
                                             pkv_dtype cache_dtype, float* lse_out, void* workspace,
                                             size_t workspace_bytes, int32_t* device_error, void* stream);

/* The fused step (append token L-1, then attend) with a sliding window and
 * sinks: the new rows of pkv_paged_decode_step, the attended positions of
 * pkv_paged_attention_decode_window (the appended token is always inside the
 * window).  Same arguments, layouts and rules as those two calls. */
pkv_status pkv_paged_decode_step_window(void* out, const void* query, const void* key, const void* value,
                                        void* key_cache, void* value_cache, float* k_scale, float* v_scale,
                                        const int32_t* block_tables, int max_blocks_per_seq,
                                        const int32_t* context_lens, int max_context_len, int num_seqs, int n_q,
                                        int n_kv, int head_dim, int block_size, int64_t num_blocks, float sm_scale,
                                        int window, int sinks, pkv_dtype act_dtype, pkv_dtype cache_dtype,
                                        float* lse_out, void* workspace, size_t workspace_bytes,
                                        int32_t* device_error, void* stream);

/*
 * Decode for a batch whose sequences all begin with the same physical blocks:
 * a shared prompt prefix stored once ("Chapter 18 - KV-Cache Optimization
 * Strategies", Prefix Caching; "KV Cache Engineering for LLM Serving", section
 * 11).  The first prefix_blocks entries of every block table must name the same
 * blocks (the caller's contract, as for shared blocks in general; row 0's are
 * the ones read, and a row that differs sets PKV_DEVERR_PREFIX).  The prefix is
 * attended once per KV head for the queries of all sequences together (a dense
 * pass on the fifth-generation tensor cores), each sequence's own positions
 * [prefix_blocks * block_size, L) are attended by the paged decode, and the two
 * softmax states are merged exactly, so the result equals
 * pkv_paged_attention_decode's.
 *
 *   key, value        optional new rows [num_seqs, n_kv, head_dim] (act dtype):
 *                     appended as token L-1 first, as in pkv_paged_decode_step;
 *                     NULL for a plain decode
 *   prefix_blocks     >= 1; every context length must exceed prefix_blocks *
 *                     block_size (else PKV_DEVERR_CONTEXT_LEN, and that
 *                     sequence's output is undefined)
 *   workspace         pkv_shared_prefix_workspace_size bytes
 * BF16 cache and activations, head_dim 64 or 128.  Three launches on `stream`:
 * the prefix pass, the decode over each sequence's own blocks, which runs
 * beside the prefix pass (it touches none of the prefix pass's data), and the
 * merge.  The prefix pass waits for the kernel launched before the call; the
 * decode starts only once every CTA of the prefix pass has done so.
 */
size_t pkv_shared_prefix_workspace_size(int num_seqs, int n_q, int n_kv, int head_dim, int block_size,
                                        int prefix_blocks);
pkv_status pkv_paged_attention_decode_shared_prefix(void* out, const void* query, const void* key, const void* value,
                                                    void* key_cache, void* value_cache, const int32_t* block_tables,
                                                    int max_blocks_per_seq, const int32_t* context_lens,
                                                    int max_context_len, int num_seqs, int n_q, int n_kv,
                                                    int head_dim, int block_size, int64_t num_blocks, float sm_scale,
                                                    int prefix_blocks, pkv_dtype act_dtype, pkv_dtype cache_dtype,
                                                    float* lse_out, void* workspace, size_t workspace_bytes,
                                                    int32_t* device_error, void* stream);

/*
 * Quest, query-aware sparse reads ("KV Cache Engineering for LLM Serving",
 * section 7).  A page is one cache block.  Each page keeps the element-wise
 * minimum and maximum of its keys; a query scores a page by
 * sum_i max(q_i * min_i, q_i * max_i) (an upper bound of q . k for every key of
 * the page), and only the best pages are read.  Pages are chosen per
 * (sequence, KV head) by the largest score of that head's query heads; the
 * k best are kept, ties toward the lower page index.  BF16 and F32 caches,
 * head_dim 64 or 128, block_size 16.
 */

/* Page summaries: page_min / page_max [num_blocks, n_kv, head_dim] (device, in
 * the cache dtype) receive, for each listed block of each sequence, the
 * element-wise min / max of its keys (the last page over rows < L only).
 * Blocks shared by several sequences are written with identical values.  With
 * last_page_only nonzero only the page holding token L-1 of each sequence is
 * refreshed: the per-step update after appending one token.  A block table
 * entry outside [0, num_blocks) sets the block-range bit and is skipped; a
 * length outside [0, max_blocks_per_seq * block_size] sets the context bit. */
pkv_status pkv_quest_page_summaries(const void* key_cache, void* page_min, void* page_max,
                                    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                                    int num_seqs, int n_kv, int head_dim, int block_size, int64_t num_blocks,
                                    pkv_dtype cache_dtype, int last_page_only, int32_t* device_error, void* stream);

/* Page selection: selected [num_seqs, n_kv, k_pages] (int32, device) receives
 * each KV head's min(k_pages, ceil(L / block_size)) best logical pages in
 * increasing order, -1 after them.  scores (required, device float
 * [num_seqs, n_kv, ceil(min(max_context_len, max_blocks_per_seq * 16) / 16)])
 * receives every page's score (entries past a sequence's pages are left as
 * they are); the selection reads it back.  query [num_seqs, n_q, head_dim] in
 * act_dtype; page_min / page_max as written by pkv_quest_page_summaries.  Two
 * launches (scoring, then top-k) on `stream`.  A block table entry outside
 * [0, num_blocks) sets the block-range bit and gives its page the score -inf. */
pkv_status pkv_quest_select(const void* query, const void* page_min, const void* page_max,
                            const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                            int max_context_len, int num_seqs, int n_q, int n_kv, int head_dim, int block_size,
                            int64_t num_blocks, pkv_dtype act_dtype, pkv_dtype cache_dtype, int k_pages,
                            int32_t* selected, float* scores, int32_t* device_error, void* stream);

/* Decode attention over listed pages only: KV head kv of sequence s attends
 * to the tokens of the logical pages pages[s][kv][0 .. k_pages) (int32,
 * device, strictly increasing; the list ends at its first -1 and every later
 * entry must be -1 too).  At most min(k_pages, ceil(L / block_size)) entries
 * are read.  A listed page at or past the sequence's page count sets the
 * block-range bit of device_error and the outputs are then undefined.
 * An empty list gives a zero output and lse -inf.  BF16/INT8/FP8/F32 caches as
 * pkv_paged_attention_decode, whose arguments and results this shares; a
 * workspace sized by pkv_paged_attention_workspace_size suffices. */
pkv_status pkv_paged_attention_decode_pages(void* out, const void* query, const void* key_cache,
                                            const void* value_cache, const float* k_scale, const float* v_scale,
                                            const int32_t* block_tables, int max_blocks_per_seq,
                                            const int32_t* context_lens, int max_context_len, int num_seqs, int n_q,
                                            int n_kv, int head_dim, int block_size, int64_t num_blocks,
                                            float sm_scale, const int32_t* pages, int k_pages, pkv_dtype act_dtype,
                                            pkv_dtype cache_dtype, float* lse_out, void* workspace,
                                            size_t workspace_bytes, int32_t* device_error, void* stream);

/*
 * Launch shape overrides for pkv_paged_attention_decode_ex (0 = automatic).
 * num_ctas: persistent CTAs sharing the blocks of all (sequence, KV-head group)
 * pairs; stages: depth of the shared-memory ring of K/V blocks; heads_per_cta:
 * KV heads a CTA streams together (a divisor of n_kv).
 */
typedef struct {
  int num_ctas;
  int stages;
  int heads_per_cta;
  int flags;         /* PKV_TUNE_* bits */
  int prefix_splits; /* shared-prefix decode: splits of the prefix pass along the prefix (0 = automatic) */
  int reserved;      /* must be 0 */
  /* SM clock cycles a bounded wait of the decode kernels may spend before it
   * gives up and sets PKV_DEVERR_TIMEOUT (0 = about one second).  A kernel that
   * gives up still waits, with the full limit, for the copies it has issued, so
   * nothing is in flight when it exits; its outputs are then undefined.  For
   * tests of the timeout path. */
  int64_t wait_limit_cycles;
} pkv_decode_tuning;

/* Launch the decode kernel so that it may start while the kernel launched just
 * before it on the same stream is still finishing (programmatic dependent
 * launch).  Its CTAs then build their schedule from context_lens and
 * block_tables and wait for the earlier kernel before reading anything else
 * (queries, new rows, the cache, the workspace) or writing anything.  Only
 * valid when context_lens and block_tables were not written by the kernel
 * launched immediately before this call. */
#define PKV_TUNE_OVERLAP_PROLOGUE 0x1

/* Shared-prefix decode: run the decode over each sequence's own blocks after
 * the prefix pass instead of beside it. */
#define PKV_TUNE_PREFIX_SERIAL 0x2

/* Workspace bytes for pkv_paged_attention_decode_ex with the given tuning. */
size_t pkv_paged_attention_workspace_size_ex(int num_seqs, int n_q, int n_kv, int head_dim, int block_size,
                                             pkv_dtype cache_dtype, const pkv_decode_tuning* tuning);

/* pkv_paged_decode_step with launch overrides (tuning may be NULL). */
pkv_status pkv_paged_decode_step_ex(void* out, const void* query, const void* key, const void* value, void* key_cache,
                                    void* value_cache, float* k_scale, float* v_scale, const int32_t* block_tables,
                                    int max_blocks_per_seq, const int32_t* context_lens, int max_context_len,
                                    int num_seqs, int n_q, int n_kv, int head_dim, int block_size, int64_t num_blocks,
                                    float sm_scale, pkv_dtype act_dtype, pkv_dtype cache_dtype, float* lse_out,
                                    void* workspace, size_t workspace_bytes, int32_t* device_error,
                                    const pkv_decode_tuning* tuning, void* stream);

/* pkv_paged_attention_decode with explicit launch shape (tuning may be NULL). */
pkv_status pkv_paged_attention_decode_ex(void* out, const void* query, const void* key_cache, const void* value_cache,
                                         const float* k_scale, const float* v_scale, const int32_t* block_tables,
                                         int max_blocks_per_seq, const int32_t* context_lens, int max_context_len,
                                         int num_seqs, int n_q, int n_kv, int head_dim, int block_size,
                                         int64_t num_blocks, float sm_scale, pkv_dtype act_dtype, pkv_dtype cache_dtype,
                                         float* lse_out, void* workspace, size_t workspace_bytes, int32_t* device_error,
                                         const pkv_decode_tuning* tuning, void* stream);

/* Shared-prefix decode with launch overrides (tuning may be NULL): num_ctas,
 * stages and flags apply to the decode over each sequence's own blocks,
 * prefix_splits to the prefix pass, PKV_TUNE_PREFIX_SERIAL orders the two
 * passes.  Size the workspace with pkv_shared_prefix_workspace_size_ex and the
 * same tuning. */
size_t pkv_shared_prefix_workspace_size_ex(int num_seqs, int n_q, int n_kv, int head_dim, int block_size,
                                           int prefix_blocks, const pkv_decode_tuning* tuning);
pkv_status pkv_paged_attention_decode_shared_prefix_ex(void* out, const void* query, const void* key,
                                                       const void* value, void* key_cache, void* value_cache,
                                                       const int32_t* block_tables, int max_blocks_per_seq,
                                                       const int32_t* context_lens, int max_context_len,
                                                       int num_seqs, int n_q, int n_kv, int head_dim, int block_size,
                                                       int64_t num_blocks, float sm_scale, int prefix_blocks,
                                                       pkv_dtype act_dtype, pkv_dtype cache_dtype, float* lse_out,
                                                       void* workspace, size_t workspace_bytes,
                                                       int32_t* device_error, const pkv_decode_tuning* tuning,
                                                       void* stream);

/* pkv_paged_attention_decode_pages with explicit launch shape (tuning may be
 * NULL; heads_per_cta must be 0 or 1: a page list belongs to one KV head).
 * Size the workspace with pkv_paged_attention_workspace_size_ex and the same
 * tuning with heads_per_cta 1. */
pkv_status pkv_paged_attention_decode_pages_ex(void* out, const void* query, const void* key_cache,
                                               const void* value_cache, const float* k_scale, const float* v_scale,
                                               const int32_t* block_tables, int max_blocks_per_seq,
                                               const int32_t* context_lens, int max_context_len, int num_seqs,
                                               int n_q, int n_kv, int head_dim, int block_size, int64_t num_blocks,
                                               float sm_scale, const int32_t* pages, int k_pages,
                                               pkv_dtype act_dtype, pkv_dtype cache_dtype, float* lse_out,
                                               void* workspace, size_t workspace_bytes, int32_t* device_error,
                                               const pkv_decode_tuning* tuning, void* stream);

/*
 * pkv_paged_attention_decode for callers that cannot allocate device memory.
 * This entry point has no counterpart in the paper; it exists for the callers
 * of this library.
 *
 * Some callers cannot give the library a workspace: a library loaded into a
 * host runtime that owns every device allocation and offers plug-ins no
 * allocator, or a serving loop that must never call cudaMalloc because it can
 * synchronise the device.  This call takes the same arguments as
 * pkv_paged_attention_decode minus the workspace and runs the same kernels.
 * Its scratch is a 16 MiB array that is part of libpkv itself.  Every GPU that
 * loads the library holds that array until the process exits.  The call itself
 * allocates nothing.
 *
 *   - Shapes needing more scratch than 16 MiB (see
 *     pkv_paged_attention_workspace_size) are rejected with PKV_ERR_WORKSPACE
 *     before anything is launched; pkv_last_cuda_error() then says how many
 *     bytes the shape needs.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress).  Make that first call before any stream capture
 *     on that device.  The address is kept for the life of the process: after
 *     cudaDeviceReset on a device it no longer names the array, so a process
 *     that resets a device must not call this entry point on it again.
 *   - Every call on a device shares the one array.  Calls whose work can
 *     overlap on the GPU (different streams, no ordering between them) race on
 *     the array and give wrong results; keep such calls in one stream.
 */
pkv_status pkv_paged_attention_decode_static(void* out, const void* query, const void* key_cache,
                                             const void* value_cache, const float* k_scale, const float* v_scale,
                                             const int32_t* block_tables, int max_blocks_per_seq,
                                             const int32_t* context_lens, int max_context_len, int num_seqs, int n_q,
                                             int n_kv, int head_dim, int block_size, int64_t num_blocks,
                                             float sm_scale, pkv_dtype act_dtype, pkv_dtype cache_dtype,
                                             float* lse_out, int32_t* device_error, void* stream);

/*
 * 2-bit KIVI cache ("KV Cache Engineering for LLM Serving", section 8,
 * Quantization: KIVI groups key values by channel and value-cache numbers by
 * token, with a 2-bit cache; "Chapter 18 - KV-Cache Optimization Strategies",
 * KV-Cache Quantization methods table).  Quantiser: the section's symmetric
 * absmax one at 2 bits: scale = max |x| of the group (float), codes
 * rint(x / scale) (ties to even) in {-1, 0, 1}, restored values code * scale;
 * an all-zero group has scale 0 and codes 0.
 *   K group: one channel of one KV head over the 16 tokens of a block
 *   V group: the head_dim values of one token of one KV head
 * A channel group needs its whole block, so only full blocks are quantised.
 * Sequence s of length L keeps positions [0, 16 * floor(L / 16)) in the pool
 * blocks named by its block table and the L % 16 positions of its partial
 * last block, in order, in rows [0, L % 16) of its BF16 residual.
 *
 * Layouts (row-major, innermost last):
 *   key_cache, value_cache  device uint8 [num_blocks, n_kv, 16, head_dim / 4]
 *                           (head-major inside a block: one (block, head) tile
 *                           is 512 contiguous bytes): element 4j + m of a token
 *                           row in bits [2m, 2m+1] of byte j, two's complement
 *   k_scale                 device float [num_blocks, n_kv, head_dim]
 *   v_scale                 device float [num_blocks, n_kv, 16]
 *   residual_k, residual_v  device bf16 [num_seqs, 16, n_kv, head_dim]; row r of
 *                           sequence s holds position 16 * floor(L / 16) + r
 * BF16 activations, head_dim 128, block_size 16, n_q / n_kv <= 64.  All
 * pointers 16-byte aligned.
 */

/* Workspace bytes of pkv_kivi_decode; (size_t)-1 for an unsupported shape. */
size_t pkv_kivi_workspace_size(int num_seqs, int n_q, int n_kv, int head_dim, int block_size);

/*
 * Quantise whole 16-token blocks of K/V rows into the pools (prefill).
 *   key_rows, value_rows  device bf16 [num_src_blocks, 16, n_kv, head_dim]
 *   dst_blocks            device int32 [num_src_blocks]: physical block of
 *                         each source block; -1 skips it, any other id outside
 *                         [0, num_blocks) sets PKV_DEVERR_BLOCK_RANGE and skips it
 * Destinations must be distinct.  One launch on `stream`.
 */
pkv_status pkv_kivi_quantize_blocks(const void* key_rows, const void* value_rows, const int32_t* dst_blocks,
                                    int64_t num_src_blocks, void* key_cache, void* value_cache, float* k_scale,
                                    float* v_scale, int n_kv, int head_dim, int block_size, int64_t num_blocks,
                                    pkv_dtype act_dtype, int32_t* device_error, void* stream);

/*
 * Decode over a KIVI cache, optionally appending the step's token first.
 *
 *   key, value     optional device bf16 [num_seqs, n_kv, head_dim]: token
 *                  L - 1 of each sequence (L = context_lens[s] >= 1, counted
 *                  with it), written to residual row (L - 1) % 16; when that
 *                  row is 15 the block is full and its 16 rows are quantised
 *                  into physical block block_tables[s][(L - 1) / 16].  Both
 *                  NULL for a plain decode.
 *   query, out     device bf16 [num_seqs, n_q, head_dim]
 *   lse_out        optional device float [num_seqs, n_q], natural log
 *   workspace      pkv_kivi_workspace_size bytes (any contents)
 * For each query head: softmax(sm_scale * q.k) over the dequantised keys of
 * the full blocks and the residual rows, weighting the values likewise; a
 * sequence with L == 0 gives out 0 and lse -inf.  Context lengths outside
 * [0, min(max_context_len, max_blocks_per_seq * 16)] set
 * PKV_DEVERR_CONTEXT_LEN; block-table entries outside [0, num_blocks) set
 * PKV_DEVERR_BLOCK_RANGE (the block is skipped).  Three launches on `stream`
 * (residual pass, decode over the full blocks, merge of split units), the
 * last two queued with programmatic serialisation.
 */
pkv_status pkv_kivi_decode(void* out, const void* query, const void* key, const void* value, void* residual_k,
                           void* residual_v, void* key_cache, void* value_cache, float* k_scale, float* v_scale,
                           const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                           int max_context_len, int num_seqs, int n_q, int n_kv, int head_dim, int block_size,
                           int64_t num_blocks, float sm_scale, pkv_dtype act_dtype, float* lse_out, void* workspace,
                           size_t workspace_bytes, int32_t* device_error, void* stream);

/*
 * Copy whole physical blocks inside one pool: copy-on-write of shared blocks.
 *
 * Several block tables may point at one physical block; when a sequence
 * diverges, only the affected block is duplicated ("Chapter 18 - KV-Cache
 * Optimization Strategies", Prefix Caching; KV-cache overview page t13_4,
 * copy-on-write paragraph).  For each pair p: block block_mapping[2p+1] of the
 * K and V pools (and, for INT8 / INT4, of k_scale / v_scale) <- block block_mapping[2p].
 *
 *   key_cache, value_cache  device, [num_blocks, block_size, n_kv, head_dim], cache_dtype
 *   k_scale, v_scale        INT8 / INT4: device [num_blocks, block_size, n_kv]; KIVI2:
 *                           k_scale [num_blocks, n_kv, head_dim], v_scale [num_blocks,
 *                           n_kv, block_size]; NULL otherwise (FP8 per-head scales
 *                           belong to no block)
 *   block_mapping           device (or mapped host) int64 [num_pairs, 2] = (src, dst)
 * Destinations must be distinct and no block may be both a source and a
 * destination in one call (all pairs run in parallel).  Out-of-range block ids
 * set PKV_DEVERR_BLOCK_RANGE and the pair is skipped.  The bytes of one row
 * (n_kv * head_dim * bytes per value, half a byte for INT4, a quarter for
 * KIVI2) must be a multiple of 16.
 */
pkv_status pkv_copy_blocks(void* key_cache, void* value_cache, float* k_scale, float* v_scale,
                           const int64_t* block_mapping, int64_t num_pairs, int n_kv, int head_dim, int block_size,
                           int64_t num_blocks, pkv_dtype cache_dtype, int32_t* device_error, void* stream);

/*
 * Move whole blocks between two pools: offload to host memory and restore.
 *
 * Blocks not needed now move to a larger, slower tier and come back when they
 * are needed again ("KV Cache Engineering for LLM Serving", section 12, Cache
 * Offloading from GPU).  For each pair p: block block_mapping[2p+1] of the dst
 * pools <- block block_mapping[2p] of the src pools (K, V and INT8 / INT4 scales).
 * Either side may be page-locked host memory mapped into the device address
 * space (cudaHostAlloc, or cudaHostRegister with cudaHostRegisterMapped): the
 * kernel reads or writes it directly over the host link.  Same layouts,
 * dtype rules and error handling as pkv_copy_blocks; destinations distinct.
 */
pkv_status pkv_swap_blocks(const void* src_key, const void* src_value, const float* src_k_scale,
                           const float* src_v_scale, int64_t src_num_blocks, void* dst_key, void* dst_value,
                           float* dst_k_scale, float* dst_v_scale, int64_t dst_num_blocks,
                           const int64_t* block_mapping, int64_t num_pairs, int n_kv, int head_dim, int block_size,
                           pkv_dtype cache_dtype, int32_t* device_error, void* stream);

/* Static text for a status code. */
const char* pkv_status_string(pkv_status status);

/* Text describing this thread's last failing CUDA call, or the last scratch-size
 * rejection of pkv_paged_attention_decode_static ("" if none). */
const char* pkv_last_cuda_error(void);

/* Library version: major * 10000 + minor * 100 + patch. */
int pkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H */
