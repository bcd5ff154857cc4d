/*
 * kv4.h -- C ABI of libkv4: decode-step attention over a KV4-RL compressed KV
 * cache on NVIDIA B200 (sm_100a).
 *
 * The method (cited by page title and section):
 *  [KV4RL] "[Paper review] KV4-RL: Unlocking Faster Asynchronous Rollouts for
 *          RLVR with INT4 KV Cache Quantization", sec. 1 (Selective Protection)
 *          and sec. 3 (Method & Key Results). The full context is stored as
 *          paged INT4 K/V; the first 16 ("attention sink") and the 128 most
 *          recent positions are also held in an INT8 side cache; the INT4 and
 *          INT8 regions are attended independently and their partial
 *          (max, sum, output) triples are joined by an exact softmax merge, so
 *          no full-precision cache is ever rebuilt.
 *  [SMD]   "How to compress the KV cache in RL post-training? Shadow Mask
 *          Distillation" (arXiv 2605.06850), sec. 1 and Figure 1: eviction is
 *          recorded as a binary mask of retained positions and applied inside
 *          attention instead of slicing tensors.
 *  [KVP]   promo of arXiv 2602.10238 ("learning to evict"), core-mechanism
 *          section, and the TTKV promo (arXiv 2604.19769), insight 1: score each
 *          position, rank, truncate at a budget, per attention head; the KVP
 *          promo's engineering-limitations section, third item: in a paged
 *          cache of 16-position blocks the ranking is taken per block.
 *  [KVS]   "KV-streams for Efficient Compaction in Agentic Reinforcement
 *          Learning" (summary page), method details, core idea: a compacted
 *          cache keeps streaming into its surviving pages.
 * Stated readings where the pages are silent: symmetric INT4 codes in [-7, 7]
 * per group of 32 consecutive head_dim elements with one fp16 scale; per-token
 * INT8 codes in [-127, 127] with one fp16 scale; scales are max|x|/qmax rounded
 * toward +inf to fp16; codes are x/scale rounded to nearest-even.
 *
 * Conventions for every call:
 *  - All pointers named *_dev or documented "device" are device memory owned by
 *    the caller; the library never allocates device memory except the 4-byte
 *    error word owned by a kv4_cache (kv4_decode_attn_noalloc's fixed scratch
 *    is a variable of the library's module, reserved when the module loads).
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL =
 *    the legacy default stream) unless stated otherwise.
 *  - Argument errors are detected on the host before any launch and return
 *    KV4_ERR_INVALID / KV4_ERR_UNSUPPORTED with nothing enqueued.
 *  - Data errors found on the device (a page id outside the pool, a length
 *    beyond the page-table capacity, a scale that overflows fp16, a bounded
 *    wait that ran out) set a bit in the cache's device error word; the kernel
 *    skips the offending work and returns normally. kv4_get_error() reports it.
 *  - A failed launch returns KV4_ERR_CUDA.
 */
#ifndef KV4_H
#define KV4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KV4_OK = 0,
  KV4_ERR_INVALID = 1,      /* bad argument (null, misaligned, inconsistent sizes) */
  KV4_ERR_UNSUPPORTED = 2,  /* valid but not built (head_dim, GQA group, sink/recent) */
  KV4_ERR_CAPACITY = 3,     /* a length exceeds the page-table / side-cache capacity */
  KV4_ERR_BOUNDS = 4,       /* a page id outside [0, num_pages) */
  KV4_ERR_RANGE = 5,        /* a K/V value too large for an fp16 scale (|x| > 458,528),
                               or a query component beyond the fp16 range */
  KV4_ERR_TIMEOUT = 6,      /* a bounded device wait ran out */
  KV4_ERR_CUDA = 7          /* a CUDA runtime call failed */
} kv4_status;

/* Geometry of one compressed cache (one attention layer). */
typedef struct {
  int32_t num_kv_heads;  /* Hkv >= 1 */
  int32_t head_dim;      /* D: 64 or 128 */
  int32_t page_tokens;   /* positions per page: must be 16 */
  int32_t group;         /* INT4 group along head_dim: must be 32 */
  int32_t sink;          /* INT8 sink positions: 0..16 (16 in KV4-RL) */
  int32_t recent;        /* INT8 recent window: 0..128, a multiple of 16 (128 in KV4-RL) */
  int32_t max_seqs;      /* sequence slots in the side cache */
  int32_t num_pages;     /* physical pages in the pool */
} kv4_config;

typedef struct kv4_cache kv4_cache;   /* opaque host handle */

/* Human-readable name of a status. Never NULL. */
const char *kv4_status_string(kv4_status s);

/* Text of the last CUDA runtime error behind a KV4_ERR_CUDA returned to the
 * calling thread ("no error" if none); a static string, not to be freed. */
const char *kv4_last_cuda_error(void);

/*
 * kv4_cache_bytes -- sizes of the two caller-owned device buffers.
 *  page_pool_bytes: num_pages pages. One page holds 16 positions of every KV
 *    head: per head a block of 18*D bytes = K codes 8D | V codes 8D |
 *    K scales D | V scales D (INT4 nibbles in the register-fragment order the
 *    decode kernel consumes; fp16 scales [slot][group]).
 *  side_cache_bytes: max_seqs * Hkv INT8 blocks, one per (sequence, KV head).
 *    A block is a sequence of 16-row pages: a sink page when sink > 0 (position
 *    p < sink in row p), then recent/16 ring pages (position p in ring slot
 *    p mod recent). A page is K codes 16*D | K scales 16 x fp16 | V scales
 *    16 x fp16 | V codes 16*D (32*D + 64 bytes), codes in the register-fragment
 *    order of the fp16 decode tiles.
 * [KV4RL] sec. 3 (paged INT4 full context; bounded INT8 side cache).
 * Host only; no CUDA call.
 */
kv4_status kv4_cache_bytes(const kv4_config *cfg, size_t *page_pool_bytes, size_t *side_cache_bytes);

/*
 * kv4_cache_create -- bind caller-owned device buffers into a cache handle.
 *  page_pool, side_cache: device, 256-byte aligned, at least the sizes above.
 *  The handle keeps the pointers (no copy, no ownership) and allocates one
 *  4-byte device error word on the current device. Contents of the buffers
 *  are not touched. Returns KV4_ERR_CUDA if the device query or allocation fails.
 */
kv4_status kv4_cache_create(const kv4_config *cfg, void *page_pool, size_t pool_bytes,
                            void *side_cache, size_t side_bytes, kv4_cache **out);

/* Free the handle and its error word (not the caller's buffers). NULL is a no-op. */
void kv4_cache_destroy(kv4_cache *cache);

/*
 * kv4_append -- quantise new K/V positions into the cache ([KV4RL] sec. 3).
 *  k_new, v_new: device bf16 [T][Hkv][D], the new positions of all sequences
 *    concatenated; sequence b owns rows new_offsets[b] .. new_offsets[b+1]-1.
 *  new_offsets: device int32 [B+1], non-decreasing, new_offsets[0] = 0; or
 *    NULL for the decode-step case of exactly one new position per sequence
 *    (then total_new must equal B and row b belongs to sequence b).
 *  seq_lens_old: device int32 [B], positions already cached (read only; the
 *    caller adds the new counts afterwards).
 *  page_table: device int32 [B][pt_stride]; logical page p/16 of sequence b
 *    must be mapped before position p is appended.
 *  total_new: T, the host-known number of new rows (sizes the launch).
 * Position p = seq_lens_old[b] + j gets INT4 codes in slot p%16 of page
 * page_table[b][p/16]; INT8 codes in sink row p if p < sink; and INT8 codes in
 * ring row p mod recent if p >= (new length) - recent (only the last occupant
 * of a ring row writes, so multi-token appends are race-free).
 */
kv4_status kv4_append(kv4_cache *cache, void *stream, const void *k_new, const void *v_new,
                      const int32_t *new_offsets, const int32_t *seq_lens_old,
                      const int32_t *page_table, int32_t pt_stride, int32_t B, int64_t total_new);

/*
 * kv4_workspace_bytes -- device scratch needed by kv4_decode_attn for B
 * sequences and Hq query heads with `num_workers` parallel workers (0 = the
 * library's default for this device). Queries the current device once per
 * process (kernel attributes and occupancy); enqueues nothing.
 */
kv4_status kv4_workspace_bytes(const kv4_cache *cache, int32_t B, int32_t num_q_heads,
                               int32_t num_workers, size_t *bytes);

/*
 * kv4_decode_attn -- one decode step of attention for every sequence and query
 * head over the compressed cache.
 *  q: device bf16 [B][Hq][D]; query head hq reads KV head hq / (Hq/Hkv).
 *  seq_lens: device int32 [B], lengths after this step's append.
 *  retain_mask: NULL, or device uint32 [B][Hkv][mask_stride]; bit p%32 of word
 *    p/32 set = position p retained ([SMD] Figure 1). Positions with a clear bit
 *    are excluded; pages with no retained position are not read.
 *  softmax_scale: tau, scores are tau * q.k.
 *  num_workers: 0 = default (as many CTAs as are resident at once); otherwise
 *    the number of warps, rounded up to whole CTAs of HB warps (HB = the
 *    largest divisor of Hkv not above 8), among which every (sequence, head)'s
 *    pages are split (results agree within rounding for any value).
 *  workspace: device, >= kv4_workspace_bytes(), 256-byte aligned.
 *  out: device [B][Hq][D], bf16 (out_is_fp32 = 0) or fp32 (1).
 * The INT4 region [sink, L - recent) and the INT8 region (the rest) are
 * attended separately into (max, sum, output) partials and merged exactly
 * ([KV4RL] sec. 3). An empty retained set gives an output of 0.
 * Errors found on the device set bits in the cache's error word
 * (kv4_get_error). After KV4_ERR_TIMEOUT the output is undefined: a CTA whose
 * wait ran out leaves its partials empty, so out holds the attention over the
 * other CTAs' pages only. A query component beyond the fp16 range
 * (|q| > 65504) sets KV4_ERR_RANGE; that query head's output is then
 * undefined.
 */
kv4_status kv4_decode_attn(kv4_cache *cache, void *stream, const void *q, int32_t Hq,
                           const int32_t *seq_lens, const int32_t *page_table, int32_t pt_stride,
                           const uint32_t *retain_mask, int32_t mask_stride, float softmax_scale,
                           int32_t num_workers, void *workspace, size_t ws_bytes, void *out,
                           int32_t out_is_fp32, int32_t B);

/*
 * kv4_decode_partials -- the decode step of kv4_decode_attn over one shard of
 * each sequence's context, returning the exact softmax partial instead of the
 * output, for context-parallel decoding of long sequences across GPUs (the
 * TTKV promo of arXiv 2604.19769, opening section, puts contexts of about a
 * million tokens beyond one GPU). KV4-RL review, sec. 3: partials of disjoint
 * position sets combine exactly (kv4_merge_partials), so each GPU attends the
 * pages it holds and only (m, l, o) crosses the interconnect.
 *  page_begin, page_end: device int32 [B]; the shard attends the INT4 pages
 *    [page_begin[b], page_end[b]) of sequence b (logical page indices, the
 *    INT4 region's pages outside the range are skipped; page-table entries of
 *    skipped pages are never read). Both NULL = every INT4 page.
 *  with_int8: nonzero = the shard also attends the INT8 sink/recent positions
 *    (exactly one shard per sequence must, normally the one holding the side
 *    cache); zero = INT4 positions only.
 *  partials: device fp32 [B][Hq][D+4], 16-byte aligned: per (sequence, query
 *    head) m (the running maximum of the scores in log2 units, i.e. of
 *    softmax_scale * log2(e) * q.k; -inf when nothing was attended), l (the
 *    sum of 2^(s - m) over the attended positions), two unused words, then o
 *    (the attended values' softmax average, D floats; 0 when l = 0).
 *  Other arguments as kv4_decode_attn; the same workspace size applies.
 */
kv4_status kv4_decode_partials(kv4_cache *cache, void *stream, const void *q, int32_t Hq, const int32_t *seq_lens,
                               const int32_t *page_table, int32_t pt_stride, const int32_t *page_begin,
                               const int32_t *page_end, int32_t with_int8, const uint32_t *retain_mask,
                               int32_t mask_stride, float softmax_scale, int32_t num_workers, void *workspace,
                               size_t ws_bytes, float *partials, int32_t B);

/*
 * kv4_masked_workspace_bytes / kv4_decode_attn_masked -- kv4_decode_attn under
 * a retained-position mask, with the INT4 region's reads and work following
 * the retained count. Shadow Mask Distillation, sec. 1 and Figure 1: eviction
 * is a binary mask applied inside attention instead of slicing the cache;
 * KV4-RL review, sec. 3: the INT4 and INT8 regions are attended separately
 * and merged exactly.
 * The retained INT4-region positions of every (sequence, KV head), in position
 * order, are gathered 16 at a time into a page image in shared memory (K rows
 * and scales whole; a V row's bytes from the 16-byte pieces of the V block
 * that hold them) and attended there, so only the retained rows' K codes and
 * scales and the V pieces of their 4-row groups are read, and the work is
 * proportional to the retained rows. The INT8 region's side pages are attended
 * by the same CTAs under the same mask, and the CTAs' partials are merged. The
 * result is the same attention as kv4_decode_attn with retain_mask (within
 * rounding). Each (sequence, head) is gathered by one CTA, page after page, so
 * the call gains on sparse masks (an H2O-style 10% budget: 0.31x the unmasked
 * decode time on the eviction workload) and loses on dense ones (beyond about
 * half of the positions, kv4_decode_attn with retain_mask is faster).
 *  retain_mask: device uint32 [B][Hkv][mask_stride], required; mask_stride *
 *    32 >= pt_stride * 16.
 *  max_retained: bound on the retained INT4-region positions [sink, L - recent)
 *    of any (sequence, head). A row with more sets KV4_ERR_CAPACITY and only
 *    its first max_retained positions are attended.
 *  workspace: device, >= kv4_masked_workspace_bytes(), 256-byte aligned.
 * Other arguments as kv4_decode_attn. Launches on `stream`: a count kernel,
 * the gathering kernel and a partial merge.
 */
kv4_status kv4_masked_workspace_bytes(const kv4_cache *cache, int32_t B, int32_t Hq, int32_t pt_stride,
                                      int32_t max_retained, size_t *bytes);
kv4_status kv4_decode_attn_masked(kv4_cache *cache, void *stream, const void *q, int32_t Hq,
                                  const int32_t *seq_lens, const int32_t *page_table, int32_t pt_stride,
                                  const uint32_t *retain_mask, int32_t mask_stride, int32_t max_retained,
                                  float softmax_scale, void *workspace, size_t ws_bytes, void *out,
                                  int32_t out_is_fp32, int32_t B);

/*
 * kv4_merge_partials -- exact softmax merge of N partials per (sequence, query
 * head), e.g. those of N context shards gathered from N GPUs (KV4-RL review,
 * sec. 3: the exact merge of (max, sum, output) triples): with
 * M = max_s m_s and W_s = l_s 2^(m_s - M), out = sum_s W_s o_s / sum_s W_s;
 * 0 when every l_s = 0.
 *  partials: device fp32 [N][B][Hq][D+4] in the layout of kv4_decode_partials,
 *    16-byte aligned. out: device [B][Hq][D], bf16 (RNE of the fp32 result) or
 *    fp32 (out_is_fp32), 16-byte aligned. D = 64 or 128.
 */
kv4_status kv4_merge_partials(void *stream, const float *partials, int32_t N, int32_t B, int32_t Hq, int32_t D,
                              void *out, int32_t out_is_fp32);

/*
 * kv_topk_retain -- per (sequence, KV head) retained-position mask ([KVP] core
 * mechanism; [SMD] sec. 1).
 *  scores: device fp32 [B][Hkv][score_stride], one score per position.
 *  Forced set F: positions < sink and positions >= L - recent.
 *  k = floor(L * budget_permille / 1000); F plus the max(0, k - |F|) other
 *  positions with the highest scores (ties: lower index first) are retained.
 *  mask_out: device uint32 [B][Hkv][mask_stride]; words 0..ceil(L/32)-1 are
 *    written (bits >= L zero); later words are not touched.
 *  count_out: NULL or device int32 [B][Hkv], the retained count.
 *  max_len: host upper bound on seq_lens (sizes the launch); must be
 *    <= score_stride and <= 32 * mask_stride.
 * Scores must not be NaN; -0 and +0 compare equal.
 */
kv4_status kv_topk_retain(void *stream, const float *scores, int64_t score_stride,
                          const int32_t *seq_lens, int32_t B, int32_t Hkv, int32_t budget_permille,
                          int32_t sink, int32_t recent, uint32_t *mask_out, int32_t mask_stride,
                          int32_t *count_out, int32_t max_len);

/*
 * kv4_evict_pages -- page-granular eviction and compaction of the cache.
 * [KVP] engineering-limitations section, third item: in a paged cache of
 * 16-position blocks the ranking applies per block, on the mean of the block's
 * position scores, and whole blocks leave. "KV-streams for Efficient
 * Compaction in Agentic Reinforcement Learning" (summary page), method
 * details, core idea: the compacted cache keeps streaming; appends continue in
 * the surviving pages.
 *  scores: device fp32 [B][Hkv][score_stride] (4-byte aligned), one score per
 *    position, as for kv_topk_retain; positions [0, L) of each row are read.
 *  budget_permille: 0..1000.
 *  seq_lens: device int32 [B], read and rewritten (L - 16 e).
 *  page_table: device int32 [B][pt_stride], pt_stride <= 16384, read and
 *    rewritten in place.
 *  freed_pages: device int32 [B][pt_stride]; entries 0..e-1 of row b receive
 *    the evicted physical page ids in logical order, later entries are not
 *    touched. freed_count: device int32 [B], receives e.
 * Per sequence with L positions in n = ceil(L/16) pages: the candidates are
 * the full pages holding no position of the INT8 set (p < sink or p >= L -
 * recent); all other pages stay. A candidate's score is the fp64 sum of its
 * 16 * Hkv scores taken head by head, slot by slot (the same order as its
 * mean). k = floor(n * budget_permille / 1000) pages stay: the non-candidates
 * and the max(0, k - non-candidates) best candidates (score descending, then
 * lower page index); the other e are evicted. The row becomes the surviving
 * entries in order, then the entries past logical page n - 1 (mapped ahead for
 * later appends), then e times -1. Positions after an evicted page move down
 * 16 each; the recent window moves down 16 e, and the INT8 ring pages of each
 * (sequence, head) in the side cache are rotated to match. The INT4 pages are
 * not touched; the freed ids belong to the caller's allocator. A length below
 * 0, above 16 * pt_stride or above score_stride sets KV4_ERR_CAPACITY and
 * leaves that sequence unchanged (freed_count 0). Scores must not be NaN.
 */
kv4_status kv4_evict_pages(kv4_cache *cache, void *stream, const float *scores, int64_t score_stride,
                           int32_t budget_permille, int32_t *seq_lens, int32_t *page_table, int32_t pt_stride,
                           int32_t *freed_pages, int32_t *freed_count, int32_t B);

/*
 * smd_masked_attn -- learner-side causal attention under the recorded shadow
 * mask. "How to compress the KV cache in RL post-training? Shadow Mask
 * Distillation" (arXiv 2605.06850), sec. 1 and Figure 1: the rollout records,
 * for the query at every position, a binary mask of the positions its KV
 * eviction kept; the learner applies that mask inside its causal attention so
 * that each row reproduces what the rollout attended to.
 *  q: device bf16 [B][T][Hq][D]; k, v: device bf16 [B][T][Hkv][D]; all 16-byte
 *    aligned. D: 64 or 128; Hq / Hkv: 1, 2 or 4; T <= 65536.
 *  seq_lens: NULL (every sequence has T positions) or device int32 [B]; rows at
 *    or past the length are written as 0 and never attended to. A length
 *    outside [0, T] is clamped and sets KV4_ERR_CAPACITY in *error_word.
 *  mask: NULL (dense causal attention) or device uint32 [B][Hkv][T][mask_stride]
 *    (mask_stride >= ceil(T / 32)): bit p % 32 of word p / 32 of row (b, h, t)
 *    set = the rollout kept position p when it produced the query at position
 *    t. Bits above t are ignored (causality).
 *  Query t of head hq (KV head hq / (Hq/Hkv)) attends to {p <= t : bit p of its
 *    row set} with scores softmax_scale * q.k over the bf16 values; an empty
 *    set gives 0.
 *  out: device [B][T][Hq][D], bf16 (out_is_fp32 = 0) or fp32 (1).
 *  error_word: NULL or a device uint32 receiving status bits (1 << status).
 */
kv4_status smd_masked_attn(void *stream, const void *q, const void *k, const void *v, int32_t B, int32_t T,
                           int32_t Hq, int32_t Hkv, int32_t D, const int32_t *seq_lens, const uint32_t *mask,
                           int32_t mask_stride, float softmax_scale, void *out, int32_t out_is_fp32,
                           uint32_t *error_word);

/*
 * bf16_paged_workspace_bytes / bf16_paged_decode_attn -- the uncompressed
 * comparison ([KV4RL] sec. 3 compares against BF16 rollouts): the same decode
 * attention over bf16 pages. One page holds 16 positions of every KV head: per
 * head a block K[16][D] bf16 then V[16][D] bf16 (64*D bytes).
 *  kv_pages: device, num_pages pages. error_word: NULL or a device uint32 that
 *  receives KV4_ERR_BOUNDS / KV4_ERR_CAPACITY bits (1 << status).
 * Other arguments as kv4_decode_attn.
 */
kv4_status bf16_paged_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t D,
                                      int32_t num_workers, size_t *bytes);
kv4_status bf16_paged_decode_attn(void *stream, const void *q, int32_t Hq, int32_t Hkv, int32_t D,
                                  const void *kv_pages, int32_t num_pages, const int32_t *page_table,
                                  int32_t pt_stride, const int32_t *seq_lens, float softmax_scale,
                                  int32_t num_workers, void *workspace, size_t ws_bytes, void *out,
                                  int32_t out_is_fp32, int32_t B, uint32_t *error_word);

/*
 * kv4_decode_attn_noalloc -- kv4_decode_attn without a caller workspace. The
 * pages describe no such call: it serves callers that cannot allocate device
 * memory for the library, e.g. C code with no access to the application's
 * device allocator, or a serving loop that must not call cudaMalloc/cudaFree
 * (which may synchronise the device) between decode steps.
 *  Scratch: a fixed array of KV4_NOALLOC_SCRATCH_BYTES (16 MiB) per device,
 *    part of the library's loaded module; no call allocates or frees memory.
 *    Nothing in it has to start at zero (the kernels write each word before
 *    reading it).
 *  Limit: returns KV4_ERR_CAPACITY, with nothing enqueued, when
 *    kv4_workspace_bytes() for the same (B, Hq, num_workers) exceeds
 *    KV4_NOALLOC_SCRATCH_BYTES (with Hkv = 8, head_dim = 128, Hq = 32 and the
 *    default 296 CTAs on a 148-SM B200: up to about 350 sequences). A smaller
 *    num_workers lowers the need.
 *  Set-up: the first call on each device looks up the array's address (this
 *    makes the CUDA runtime load the library's module on that device); make
 *    that first call before capturing the stream into a graph. Later calls on
 *    the device reuse the cached address.
 *  Concurrency: all calls on one device share the one array. Two calls whose
 *    kernels may overlap in time (different streams without ordering between
 *    them, or host threads racing on streams) corrupt each other's partials;
 *    order them on one stream or with events.
 * Other arguments, the outputs and the error behaviour are those of
 * kv4_decode_attn (q, out 16-byte aligned; the cache's device error word).
 */
#define KV4_NOALLOC_SCRATCH_BYTES (16u << 20)
kv4_status kv4_decode_attn_noalloc(kv4_cache *cache, void *stream, const void *q, int32_t Hq,
                                   const int32_t *seq_lens, const int32_t *page_table, int32_t pt_stride,
                                   const uint32_t *retain_mask, int32_t mask_stride, float softmax_scale,
                                   int32_t num_workers, void *out, int32_t out_is_fp32, int32_t B);

/*
 * kv4_get_error --synchronise `stream`, then read and clear the cache's device
 * error word. Returns KV4_OK if no device error was recorded, else the most
 * severe recorded status (TIMEOUT > BOUNDS > CAPACITY > RANGE). *bits (optional)
 * receives the raw word: bit (1 << status) per recorded status.
 */
kv4_status kv4_get_error(kv4_cache *cache, void *stream, uint32_t *bits);

/*
 * kv4_debug_set_wait_limit -- test hook for the bounded device waits of this
 * cache's decode calls, in SM clock cycles.
 *   cycles = 0:  the first wait on a page copy gives up at once and records
 *                KV4_ERR_TIMEOUT; the worker then drains the copies it has in
 *                flight (with the default limit) and stops.
 *   cycles > 0:  that limit.
 *   cycles < 0:  the default limit (about 2^32 cycles, ~2 s).
 * Host only.
 */
kv4_status kv4_debug_set_wait_limit(kv4_cache *cache, int64_t cycles);

/*
 * Kernel timing hook (host only). While enabled, every `every`-th
 * kv4_decode_attn and bf16_paged_decode_attn call (counted per kind, the first
 * call included) records a pair of CUDA events on its stream immediately
 * before and after its split-K worker kernel, for up to `max_records` calls per
 * kind. An event between two kernels keeps the second from starting early
 * (programmatic dependent launch), so sampling (every > 1) leaves most calls
 * undisturbed. kv4_timing_read synchronises those events and returns the summed
 * worker-kernel time in milliseconds and the number of recorded calls for
 * `kind` (0 = kv4_decode_attn, 1 = bf16_paged_decode_attn), then clears the
 * records. kv4_timing_disable frees the events. max_records, every >= 1.
 */
kv4_status kv4_timing_enable(int32_t max_records, int32_t every);
kv4_status kv4_timing_read(int32_t kind, double *total_ms, int32_t *count);
/* The same records as kv4_timing_read, one duration per recorded call
 * (milliseconds, oldest first): fills min(cap, count) entries of the host
 * array ms_out, sets *count to the number recorded, and clears them. */
kv4_status kv4_timing_read_each(int32_t kind, float *ms_out, int32_t cap, int32_t *count);
kv4_status kv4_timing_disable(void);

/* Number of multiprocessors and default worker count the library uses. */
kv4_status kv4_device_info(int32_t *num_sms, int32_t *default_workers);

#ifdef __cplusplus
}
#endif
#endif /* KV4_H */
