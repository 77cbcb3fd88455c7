/*
 * mla_decode.h -- C ABI of the B200 (sm_100a) MLA paged latent-cache decoder.
 *
 * The operation ("OpenSourceWeek Day 1: FlashMLA", opening paragraph and "Key
 * Highlights"; "FlashMLA: Revolutionizing Efficient Decoding in Large Language
 * Models...", sections 4.1.1 and 4.3.2): multi-head latent attention decoding.
 * Every query head attends over one cached latent row per token, shared by all
 * heads ("How MLA Optimizes Memory Usage": only c_t is cached and both K and V
 * derive from it).  Rows are bf16 and live in 64-token pages reached through a
 * per-sequence block table.  For sequence i, query position j and head h:
 *
 *     s_t   = softmax_scale * <q[i][j][h][0:576], K_t[0:576]>   for visible t
 *     out   = sum_t softmax(s)_t * K_t[0:512]       (the value is the first 512 dims)
 *     lse   = ln sum_t exp(s_t)
 *
 * with K_t = kcache[block_table[i][t / 64]][t % 64].  Visible tokens are
 * t < cache_seqlens[i]; with `causal`, query j (of s_q) sees t <= L - s_q + j
 * (the s_q queries are the last s_q positions).  An empty visible set yields
 * out = 0 and lse = -inf.
 *
 * Conventions for every entry point:
 *   - Device pointers are caller-owned device memory; the library allocates no
 *     device memory and keeps no state beyond a per-device cache of SM counts
 *     and kernel attributes.  Tensors are contiguous and row-major with the
 *     shapes stated.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously; nothing synchronises.
 *   - Arguments are validated on the host before anything is launched; a
 *     failing check returns MLA_ERR_INVALID_ARG or MLA_ERR_UNSUPPORTED and
 *     launches nothing.  CUDA errors at launch return MLA_ERR_CUDA.
 *   - Conditions found on the device (a bounded wait that timed out, and with
 *     device checks enabled, a block-table entry outside the cache) are written
 *     to `device_status` when it is not NULL; the caller reads it after the
 *     stream has completed.  No kernel traps or aborts.
 */
#ifndef MLA_DECODE_H
#define MLA_DECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = 1,    /* null pointer, bad size, misaligned buffer */
    MLA_ERR_UNSUPPORTED = 2,    /* a dimension this build does not implement */
    MLA_ERR_CUDA = 3,           /* a CUDA runtime call failed */
    MLA_ERR_DEVICE_TIMEOUT = 4, /* a device-side wait gave up (device_status only) */
    MLA_ERR_DEVICE_CHECK = 5,   /* a device-side bounds check failed (device_status only) */
    MLA_ERR_SCRATCH_LIMIT = 6,  /* workspace would exceed MLA_STATIC_SCRATCH_BYTES */
    MLA_ERR_NO_FREE_PAGES = 7   /* free-page stack too short for an append, or too
                                   full for a release (device_status only) */
} mla_status;

#define MLA_HEAD_DIM_QK 576     /* 512 latent + 64 rope dims per row */
#define MLA_HEAD_DIM_V 512      /* value = first 512 dims of the same row */
#define MLA_PAGE_SIZE 64        /* tokens per cache page */
#define MLA_MD_STRIDE 8         /* int32 per worker in tile_md */
#define MLA_SPLIT_PIECE_COST_CTA 2   /* per-sequence cost in pages, s_q * h_q <= 64 (partition rule) */
#define MLA_SPLIT_PIECE_COST_PAIR 7  /* per-sequence cost in pages, s_q * h_q > 64 (partition rule) */
#define MLA_ROWS_PER_CTA 64     /* query rows (s_q * h_q, flattened) per decode CTA */
#define MLA_STATIC_SCRATCH_BYTES ((size_t)48 << 20) /* see mla_decode_kvcache_static_scratch */

/*
 * mla_metadata_shape -- sizes for the split-KV metadata.
 *
 * num_workers: how many workers the decode grid uses on the current device.
 *   With s_q * h_q <= 64 query rows per sequence, one worker is one CTA and
 *   num_workers = SMs.  With more rows, one worker is one pair of CTAs (a
 *   cluster of 2) per 128-row block: num_workers = min(SMs / (2 B),
 *   C / B) with B = ceil(s_q * h_q / 128) and C the number of pairs of the
 *   decode kernel the device holds at once, so that every pair of the grid
 *   runs in the first wave.  At least 1.  md_stride: MLA_MD_STRIDE.
 * Returns MLA_OK, MLA_ERR_INVALID_ARG (batch, h_q or s_q < 1, null outputs), or
 * MLA_ERR_CUDA (no current device).
 */
int mla_metadata_shape(int batch, int h_q, int s_q, int* num_workers, int* md_stride);

/*
 * mla_get_metadata -- the length-balanced split-KV tile scheduler.
 *
 * The pages ask for a kernel optimised for variable-length serving ("OpenSourceWeek
 * Day 1: FlashMLA", opening paragraph; "DeepSeek merilis open source FlashMLA",
 * release bullets) and give no partition rule.  The rule used here:
 *   n_i = ceil(L_i / 64) pages; items_i = max(n_i, 1) (an empty sequence owns one
 *   item so that its zero output is written); sequence i costs P + items_i units,
 *   laid end to end from unit start_i, with item j at unit start_i + P + j;
 *   cap = ceil(total / W); the item at unit u goes to worker u / cap.
 *   P = MLA_SPLIT_PIECE_COST_CTA when s_q * h_q <= 64 (one CTA per worker) and
 *   MLA_SPLIT_PIECE_COST_PAIR otherwise (CTA pairs): roughly what starting and
 *   finishing a piece costs that kernel, in page-loop time.  It was set by
 *   measurement: on a CTA pair, a piece boundary stalls the page loop for its
 *   epilogue (fp32 or bf16 output of 128 rows x 512), about 8 pages' time.
 *   Exception (whole sequences): when batch <= W and no sequence costs more than
 *   cap + 2 P units, worker i takes all items of sequence i (i < batch) and the
 *   other workers are idle: a split would save at most about 2 P pages of the
 *   longest worker's time, less than its piece boundaries and the merge cost.
 * Each worker thus owns a contiguous run of items.  A sequence whose items fall
 * to k workers has k pieces (splits), merged by log-sum-exp in the decode call.
 *
 * cache_seqlens: device int32 [batch], each >= 0.
 * tile_md:       device int32 [num_workers * 8], written:
 *                [begin_seq, begin_item, end_seq, end_item (exclusive),
 *                 begin_split (piece index of begin_seq within that sequence),
 *                 num_pieces (0 = idle worker, then all fields are 0), 0, 0]
 * num_splits:    device int32 [batch + 1], written: exclusive prefix sum of the
 *                pieces per sequence (num_splits[0] = 0).
 * num_workers:   >= 1; normally the value from mla_metadata_shape.  The same
 *                value must be passed to mla_decode_kvcache.
 * h_q, s_q:      > 0; s_q * h_q selects P (the decode kernel is chosen the same way).
 * One CTA; integer only; no host synchronisation.  batch <= 65536.
 */
int mla_get_metadata(const int32_t* cache_seqlens, int batch, int h_q, int s_q,
                     int32_t* tile_md, int32_t* num_splits, int num_workers, void* stream);

/*
 * mla_workspace_size -- bytes of scratch mla_decode_kvcache needs for split
 * partials: (batch + num_workers) pieces of s_q * h_q rows, each with dv fp32
 * values plus one fp32 lse, rounded up to 256 bytes.  Returns 0 for invalid
 * arguments.
 */
size_t mla_workspace_size(int batch, int s_q, int h_q, int dv, int num_workers);

/*
 * mla_decode_kvcache -- the decode itself.
 *
 * q:            device bf16 [batch, s_q, h_q, 576], 16-byte aligned.
 * kcache:       device bf16 [num_blocks, 64, 576], 16-byte aligned.
 * num_blocks:   pages in kcache (1 <= num_blocks, num_blocks * 64 < 2^31).
 * block_table:  device int32 [batch, bt_stride]; entries [0, ceil(L_i/64)) of
 *               row i name pages of kcache (the rest are never read).
 * cache_seqlens: device int32 [batch], 0 <= L_i <= bt_stride * 64.
 * d, dv:        must be 576 and 512 (MLA_ERR_UNSUPPORTED otherwise).
 * softmax_scale: multiplies the dot products before the softmax.
 * causal:       0 or 1, see the header comment.
 * tile_md, num_splits, num_workers: from mla_get_metadata on the same
 *               cache_seqlens (the same stream order makes them ready).
 * workspace:    device scratch of at least mla_workspace_size(...) bytes,
 *               256-byte aligned; contents need not be initialised.
 * out:          device bf16 [batch, s_q, h_q, 512], 16-byte aligned, written.
 * lse:          device fp32 [batch, h_q, s_q], written (natural log).
 * device_status: device int32, or NULL; receives MLA_ERR_DEVICE_* on a device
 *               condition (never reset by the library: the caller zeroes it).
 * Requires 1 <= s_q * h_q <= 65536 (MLA_ERR_UNSUPPORTED otherwise).
 * Launches the decode kernel and, when a sequence has more than one piece,
 * the split-combine kernel, on `stream`.
 */
int mla_decode_kvcache(const void* q, const void* kcache, int64_t num_blocks,
                       const int32_t* block_table, int bt_stride,
                       const int32_t* cache_seqlens, int batch, int s_q, int h_q,
                       int d, int dv, float softmax_scale, int causal,
                       const int32_t* tile_md, const int32_t* num_splits, int num_workers,
                       void* workspace, size_t workspace_bytes,
                       void* out, float* lse, int32_t* device_status, void* stream);

/*
 * mla_decode_kvcache_static_scratch -- mla_decode_kvcache for callers that
 * cannot allocate device memory.
 *
 * The pages have no counterpart to this entry point; it exists for library
 * users.  mla_decode_kvcache needs a workspace for the fp32 partial results of
 * sequences split across workers.  Some callers cannot provide one, because
 * they cannot call cudaMalloc: an engine that reserves all device memory up
 * front in its own arena and allows no further allocation, or a
 * latency-critical loop that must not allocate or free (cudaFree synchronises
 * the device).  This call takes the same arguments minus the workspace and
 * uses a fixed array of MLA_STATIC_SCRATCH_BYTES (48 MiB) compiled into the
 * library instead; it calls no allocating routine.
 *
 * Limit: if mla_workspace_size(batch, s_q, h_q, dv, num_workers) exceeds
 * MLA_STATIC_SCRATCH_BYTES it returns MLA_ERR_SCRATCH_LIMIT and launches
 * nothing (fewer workers need less workspace).  Null pointers, d / dv other
 * than 576 / 512 and sizes below 1 are checked before the limit and reported
 * as MLA_ERR_INVALID_ARG / MLA_ERR_UNSUPPORTED.
 * Every GPU that loads this part of the library holds the 48 MiB array until
 * the process exits.  All calls on a device share it and it keeps the last
 * call's contents (nothing in it needs to start at zero); calls that overlap
 * on the GPU race on it, so serialise them.  The first call on each device
 * looks up the array's device address; make that first call before any
 * stream capture.  Otherwise identical to mla_decode_kvcache, including its
 * errors.
 */
int mla_decode_kvcache_static_scratch(const void* q, const void* kcache, int64_t num_blocks,
                                      const int32_t* block_table, int bt_stride,
                                      const int32_t* cache_seqlens, int batch, int s_q, int h_q,
                                      int d, int dv, float softmax_scale, int causal,
                                      const int32_t* tile_md, const int32_t* num_splits,
                                      int num_workers, void* out, float* lse,
                                      int32_t* device_status, void* stream);

/*
 * mla_append_latent -- add s_new tokens' latent rows to every sequence of the
 * paged cache, taking new 64-token pages from a free-page stack.
 *
 * After each decoding step the newest token's cached state joins the cache for
 * later steps ("DeepSeek #OpenSourceWeek Day 1: Launch of FlashMLA", "How KV
 * Caching Works?"); in MLA that state is one latent row per token ("How MLA
 * Optimizes Memory Usage").  Pages are allocated on demand, like OS virtual
 * memory, so a sequence grows in 64-token increments ("FlashMLA:
 * Revolutionizing Efficient Decoding...", section 4.3.2).  The pages give no
 * allocation order; the rule here:
 *   - sequence i with L_i = cache_seqlens[i] tokens holds ceil(L_i / 64) pages;
 *     it needs ceil((L_i + s_new) / 64) - ceil(L_i / 64) new ones;
 *   - free pages are the stack free_pages[0 : *free_count]; pages are popped
 *     from the top, sequence after sequence in batch order, page after page
 *     within a sequence, into block_table[i][ceil(L_i / 64) ...];
 *   - row k of sequence i becomes token L_i + k: it is copied to row
 *     (L_i + k) % 64 of page block_table[i][(L_i + k) / 64];
 *   - then cache_seqlens[i] += s_new and *free_count drops by the pages taken.
 * Call it before the decode of the step that attends to the new tokens.
 *
 * rows:          device bf16 [batch, s_new, 576], 16-byte aligned (read).
 * s_new:         tokens added to every sequence, 1 .. 65536.
 * kcache:        device bf16 [num_blocks, 64, 576], 16-byte aligned (written).
 * block_table:   device int32 [batch, bt_stride] (entries past each sequence's
 *                pages are written as pages are taken).
 * cache_seqlens: device int32 [batch] (read, then grown).
 * free_pages:    device int32 [free_capacity]: the free-page stack (read).
 * free_count:    device int32 [1]: pages on the stack, 0 .. free_capacity
 *                (read, then lowered).
 * device_status: device int32 or NULL, as for mla_decode_kvcache.
 * The request is checked as a whole on the device.  If any L_i is negative,
 * ceil((L_i + s_new) / 64) > bt_stride, a page to be written (a sequence's
 * partly filled last page, or a popped page) lies outside [0, num_blocks), or
 * *free_count is outside [0, free_capacity], it writes MLA_ERR_DEVICE_CHECK to
 * device_status; if the stack holds fewer pages than needed, it writes
 * MLA_ERR_NO_FREE_PAGES.  Either way no length and no free count changes, and
 * no token a reader can see changes (rows may have been copied into free pages
 * or past a sequence's length, and block-table entries past its pages).
 * Host checks (nulls, sizes, alignment) return MLA_ERR_INVALID_ARG.  The
 * caller keeps the state consistent: a page in a block table must not also be
 * on the free stack.  Two launches (a grid that copies rows, one CTA that
 * checks and commits); no host synchronisation.
 */
int mla_append_latent(const void* rows, int s_new, void* kcache, int64_t num_blocks,
                      int32_t* block_table, int bt_stride, int32_t* cache_seqlens, int batch,
                      int32_t* free_pages, int free_capacity, int32_t* free_count,
                      int32_t* device_status, void* stream);

/*
 * mla_append_latent_fp8 -- mla_append_latent for an FP8 latent cache: each new
 * bf16 row is encoded into 576 E4M3 codes and one per-token scale as it is
 * written.
 *
 * The pages name FP8 support as the next way to cut the cache's memory
 * ("FlashMLA: Revolutionizing Efficient Decoding...", section 9 "Future
 * Directions") and give no format.  The format here: E4M3 codes (1 sign, 4
 * exponent bits with bias 7, 3 mantissa bits, largest finite value 448) and a
 * scale 2^k per token, k the smallest integer with max_c |x_c| <= 448 * 2^k
 * (k = 0 for an all-zero row); code_c is x_c / 2^k rounded to the nearest E4M3
 * value, ties to even, sign kept.  The decode uses code * 2^k, which is exact.
 *
 * kcache:  device uint8 [num_blocks, 64, 576] E4M3 codes, 16-byte aligned.
 * kscale:  device fp32 [num_blocks, 64] scales, 16-byte aligned.
 * Everything else (pages, block table, lengths, free stack, checks, status,
 * launches) is as for mla_append_latent.
 */
int mla_append_latent_fp8(const void* rows, int s_new, void* kcache, float* kscale,
                          int64_t num_blocks, int32_t* block_table, int bt_stride,
                          int32_t* cache_seqlens, int batch, int32_t* free_pages,
                          int free_capacity, int32_t* free_count, int32_t* device_status,
                          void* stream);

/*
 * mla_decode_kvcache_fp8 -- the decode over an FP8 latent cache (written by
 * mla_append_latent_fp8): the same operation as mla_decode_kvcache with each
 * cached row K_t = code_t * scale_t.  The cache moves half the bytes of the
 * bf16 cache; each page is widened to bf16 inside the decode kernel, exactly.
 *
 * kcache:  device uint8 [num_blocks, 64, 576] E4M3 codes, 16-byte aligned.
 * kscale:  device fp32 [num_blocks, 64] per-token scales, 16-byte aligned.
 * Rows of a sequence's last page past its length are never read as data (the
 * kernels zero them), so their codes and scales may hold anything.  Widening is exact for scales 2^k with -124 <= k <= 67 (what
 * the quantising append writes for rows whose largest magnitude lies in about
 * [1e-35, 6.6e22]).  Any s_q * h_q up to 65536 (MLA_ERR_UNSUPPORTED above):
 * up to 64 query rows per sequence on single CTAs, more on CTA pairs like
 * mla_decode_kvcache; both widen the codes to code * scale.  Metadata from
 * mla_get_metadata as for mla_decode_kvcache.
 * All other arguments, the workspace, errors and launches are as for
 * mla_decode_kvcache.
 */
int mla_decode_kvcache_fp8(const void* q, const void* kcache, const float* kscale,
                           int64_t num_blocks, const int32_t* block_table, int bt_stride,
                           const int32_t* cache_seqlens, int batch, int s_q, int h_q, int d,
                           int dv, float softmax_scale, int causal, const int32_t* tile_md,
                           const int32_t* num_splits, int num_workers, void* workspace,
                           size_t workspace_bytes, void* out, float* lse,
                           int32_t* device_status, void* stream);

/*
 * mla_release_pages -- give back the pages of finished sequences ("FlashMLA:
 * Revolutionizing Efficient Decoding...", section 4.3.2: unused blocks are
 * easily deallocated).
 *
 * For every i with release_mask[i] != 0 (batch order), pushes
 * block_table[i][0 : ceil(L_i / 64)] onto the free stack in page order and sets
 * cache_seqlens[i] = 0; *free_count grows by the pages pushed.  Block-table
 * rows are not cleared (entries past a sequence's pages are never read).
 * release_mask: device int32 [batch]; the other arguments as for
 * mla_append_latent.  A negative length, ceil(L_i / 64) > bt_stride or a free
 * count outside [0, free_capacity] writes MLA_ERR_DEVICE_CHECK, and pages that
 * would overfill free_pages write MLA_ERR_NO_FREE_PAGES, to device_status; then
 * nothing changes.  One CTA; no host synchronisation.
 */
int mla_release_pages(const int32_t* release_mask, int32_t* block_table, int bt_stride,
                      int32_t* cache_seqlens, int batch, int32_t* free_pages, int free_capacity,
                      int32_t* free_count, int32_t* device_status, void* stream);

/*
 * mla_sparse_workspace_size -- bytes of workspace mla_decode_sparse needs:
 * the cached row of every used index entry (4 bytes per entry and query
 * position), the counts, and the split metadata and partials of the decode
 * over them.  num_workers: mla_metadata_shape(batch * s_q, h_q, 1).  Returns 0
 * for invalid arguments.
 */
size_t mla_sparse_workspace_size(int batch, int s_q, int h_q, int topk, int num_workers);

/*
 * mla_decode_sparse -- sparse (top-k) decode given token indices.
 *
 * Dynamic sparse attention restricts each query to the most relevant cached
 * tokens, reached by gathering them ("Boosting DeepSeek V3.2: Faster LLM
 * Inference With FlashMLA", the paragraph on Dynamic Sparse Attention).  The
 * selection is an input (choosing it needs an indexer with trained weights):
 * indices: device int32 [batch, s_q, topk], logical token positions of
 *          sequence i for query position j, shared by every head.  An entry t
 *          is used when 0 <= t < L_i and, with causal, t <= L_i - s_q + j;
 *          other entries (-1 padding) are skipped.  Each used entry is one
 *          term, so a position listed twice counts twice.
 * Over the used entries the result is mla_decode_kvcache's definition: out
 * [batch, s_q, h_q, 512] bf16 and lse [batch, h_q, s_q] fp32; a query position
 * with no used entry gets out = 0 and lse = -inf.
 * num_workers: mla_metadata_shape(batch * s_q, h_q, 1).  workspace: at least
 * mla_sparse_workspace_size(...) bytes, 256-byte aligned, contents need not
 * be initialised.  The other arguments are as for mla_decode_kvcache.
 * Requires topk <= 65536, batch * s_q <= 65536.  A used entry whose page lies
 * outside the block-table row or the cache is read as a zero row and reported
 * as MLA_ERR_DEVICE_CHECK in device_status.
 * Launches: a compaction kernel (the used entries of each query position, as
 * cached rows, in list order), then the scheduler, decode and combine kernels
 * of mla_decode_kvcache over b * s_q sequences of one query position each,
 * the decode kernel copying the listed rows from the cache itself (each
 * selected row is read once), and (s_q > 1) a kernel that reorders lse.  No
 * host synchronisation.
 */
int mla_decode_sparse(const void* q, const void* kcache, int64_t num_blocks,
                      const int32_t* block_table, int bt_stride, const int32_t* cache_seqlens,
                      int batch, int s_q, int h_q, int d, int dv, const int32_t* indices,
                      int topk, float softmax_scale, int causal, int num_workers,
                      void* workspace, size_t workspace_bytes, void* out, float* lse,
                      int32_t* device_status, void* stream);

/* mla_error_string -- static text for a status code (never NULL). */
const char* mla_error_string(int status);

/*
 * mla_merge_partials -- merge decode results over disjoint parts of each
 * sequence's cache by log-sum-exp: the exchange step of a decode whose cache is
 * sharded across GPUs (each rank decodes the pages it holds, the ranks gather
 * their results, and every rank merges them).
 *
 * The pages describe the cross-device form as partition-then-combine ("TPLA:
 * Tensor Parallel Latent Attention...", abstract: attend per shard, then
 * combine across devices).  Sharding the cached tokens keeps it exact:
 *   lse = ln sum_r exp(lse_r),  out = sum_r exp(lse_r - lse) * out_r,
 * with a part whose lse_r = -inf (no visible token there) weighing nothing, and
 * out = 0, lse = -inf when every part is empty.
 *
 *   outs  [num_parts, batch, s_q, h_q, 512] bf16, device: part r's decode output
 *         (normalised over part r's tokens), parts back to back.  16-B aligned.
 *   lses  [num_parts, batch, h_q, s_q] fp32, device: part r's lse (natural log).
 *   out   [batch, s_q, h_q, 512] bf16, device, 16-B aligned; lse [batch, h_q, s_q]
 *         fp32, device.  May not overlap the inputs.
 * The caller owns every buffer; nothing is allocated.  Asynchronous on `stream`.
 * Returns MLA_OK, MLA_ERR_INVALID_ARG (null, sizes < 1, more than 4096 parts,
 * s_q * h_q > 65536, num_parts * batch * s_q * h_q >= 2^31, misalignment) or
 * MLA_ERR_CUDA (launch failure).
 */
int mla_merge_partials(const void* outs, const float* lses, int num_parts, int batch, int s_q,
                       int h_q, void* out, float* lse, void* stream);

/*
 * mla_set_wait_limit_ns -- limit of each bounded wait inside the decode kernels.
 *
 * Not part of the method (the pages have no counterpart): every wait of a
 * decode kernel on a barrier gives up after this long, stops the CTA, lets the
 * asynchronous copies and MMAs it has already issued finish, and reports
 * MLA_ERR_DEVICE_TIMEOUT through device_status; nothing traps.  The default,
 * 2 s, is far above any legitimate wait.  Lowering it makes the timeout path
 * run on purpose, which is how the tests check it (a wait of a few microseconds
 * cannot see its data arrive).  ns = 0 restores the default; values are
 * clamped to [1000, 2e9].  Applies to decode calls launched after it, from any
 * thread (a process-wide setting).  Returns the previous limit.
 */
uint64_t mla_set_wait_limit_ns(uint64_t ns);

/*
 * mla_debug_set_stall_flag -- test hook of the timeout path.
 *
 * Not part of the method.  With a non-null device pointer to an int32 word, the
 * PV-issuing thread of every decode CTA launched afterwards waits, before its
 * first PV, for that word to become non-zero (a bounded wait like every other:
 * mla_set_wait_limit_ns).  A word that stays zero makes that wait run out while
 * the CTA's TMA copies and QK^T MMAs are in flight, which exercises the drain
 * and the MLA_ERR_DEVICE_TIMEOUT report.  NULL (the default) switches the hook
 * off.  Process-wide; the caller owns the word and keeps it alive while such
 * launches run.  Returns the previous pointer.
 */
const int32_t* mla_debug_set_stall_flag(const int32_t* device_flag);

/* mla_version -- build identification string (never NULL). */
const char* mla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_DECODE_H */
