/*
 * kv4_oracle.h -- plain fp64 CPU oracle for decode attention over a KV4-RL
 * compressed KV cache (paged INT4 + INT8 sink/recent side cache).
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg load this library. It shares no code, header or table with
 * the CUDA library; the only contract between the two is the stated byte
 * layout and the stated quantiser, both written out independently on each side.
 *
 * Sources (web pages, cited by title and section):
 *  [KV4RL]  "[Paper review] KV4-RL: Unlocking Faster Asynchronous Rollouts for
 *           RLVR with INT4 KV Cache Quantization", sec. 1 (Selective Protection)
 *           and sec. 3 (Method & Key Results): full context in paged INT4,
 *           first 16 + most recent 128 positions in an INT8 side cache, the two
 *           regions attended separately and joined by an exact softmax merge.
 *  [SMD]    "How to compress the KV cache in RL post-training? Shadow Mask
 *           Distillation" (arXiv 2605.06850), sec. 1 and Figure 1: the retained
 *           index set is recorded as a binary mask and applied inside attention.
 *  [KVP]    promo of arXiv 2602.10238 ("learning to evict"), core-mechanism
 *           section: score every token, rank, truncate at a 10%..90% budget,
 *           one ranking per attention head; engineering-limitations section,
 *           third item: in a paged (vLLM-style, 16-position block) cache the
 *           ranking is taken per block, on the mean of its positions' scores.
 *  [KVS]    "KV-streams for Efficient Compaction in Agentic Reinforcement
 *           Learning" (summary page), method details, core idea: after a
 *           compaction the cache keeps streaming instead of being flushed.
 * Quantiser details the pages leave open (symmetric INT4 per 32-element group
 * along head_dim with an fp16 scale; per-token INT8 with an fp16 scale;
 * scale rounded toward +inf; codes rounded to nearest-even) are this project's
 * stated readings.
 *
 * What pins each function to something other than itself (tests/test_oracle_*):
 *  fp16 round-up, RNE, fp16/bf16 decoders: exact rational arithmetic over every
 *    positive finite bf16 maximum (both divisors), numpy's fp16 decoder.
 *  kv4o_quant_int4/int8: brute force over all codes with ties to even;
 *    |x - c s| <= s/2; re-quantising c s returns c; overflow flag.
 *  byte layout and kv4o_write_cache: hand-computed offsets, bijection of every
 *    layout, the written image read back through the fragment view.
 *  kv4o_attend_rows, kv4o_merge, kv4o_decode: closed forms (equal scores,
 *    zero query, one dominant key, two keys), merge of random chunkings equal
 *    to one softmax, decode equal to the merge of its INT4 and INT8 partials,
 *    contexts of at most 144 positions independent of the INT4 codes, GQA
 *    head mapping, full / empty / subset masks.
 *  kv4o_topk: subset enumeration on short rows, nested budgets, the forced
 *    set, budget counts from the floor rule, -0 equal to +0.
 *  kv4o_masked_attn: torch float64 softmax attention on small cases, closed
 *    forms (a diagonal-only mask returns v_t, an empty row returns 0), and
 *    row t equal to kv4o_decode over bf16 values at length t + 1 under mask
 *    row t (the learner reproduces the rollout's attention).
 *  kv4o_evict_pages: pairwise order check of kept against evicted pages on
 *    scores whose page sums are exact, hand-worked tables and free lists,
 *    decode of the compacted cache equal to masked decode of the original,
 *    the compacted side image equal to re-appending the surviving positions.
 * Parity unpinned: the size of the error that INT8 protection removes relative
 * to unquantised attention (reported, only its direction is checked).
 */
#ifndef KV4_ORACLE_H
#define KV4_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int32_t B;        /* sequences */
  int32_t Hq;       /* query heads */
  int32_t Hkv;      /* KV heads; Hq % Hkv == 0 */
  int32_t D;        /* head_dim, a multiple of 32 */
  int32_t sink;     /* INT8 sink positions (16 in KV4-RL) */
  int32_t recent;   /* INT8 recent window (128 in KV4-RL) */
} kv4o_shape;

/* ---- number formats ---- */
uint16_t kv4o_fp16_round_up(double y);          /* smallest fp16 >= y (y >= 0); +inf bits if none */
double   kv4o_fp16_to_double(uint16_t bits);
double   kv4o_bf16_to_double(uint16_t bits);
double   kv4o_round_half_even(double x);

/* ---- quantiser ---- */
/* Symmetric INT4 over n elements (a group of 32): s = RU_fp16(max|x|/7),
 * c = RNE(x/s) in [-7,7]. Returns 1 if the scale overflowed fp16 (then
 * s = 0x7BFF and codes are clamped), else 0. */
int kv4o_quant_int4(const uint16_t *x_bf16, int n, uint16_t *scale_bits, int8_t *codes);
/* Symmetric INT8 over n elements (one token row): s = RU_fp16(max|x|/127),
 * c = RNE(x/s) in [-127,127]. Same overflow rule. */
int kv4o_quant_int8(const uint16_t *x_bf16, int n, uint16_t *scale_bits, int8_t *codes);

/* ---- byte layout (offsets inside one head block of one physical page) ---- */
int64_t kv4o_page_head_bytes(int D);                       /* 18*D */
int64_t kv4o_k_code_byte(int D, int r, int d, int *nibble); /* r = slot 0..15 */
int64_t kv4o_v_code_byte(int D, int r, int d, int *nibble);
int64_t kv4o_k_scale_byte(int D, int r, int grp);
int64_t kv4o_v_scale_byte(int D, int r, int grp);
int64_t kv4o_side_head_bytes(int D, int sink, int recent); /* INT8 block per (seq, head) */
int     kv4o_side_pages(int sink, int recent);             /* 16-row pages per block */
int64_t kv4o_side_page_bytes(int D);                       /* 32*D + 64 */
int64_t kv4o_side_k_byte(int D, int row, int d);           /* offsets inside one block */
int64_t kv4o_side_v_byte(int D, int row, int d);
int64_t kv4o_side_ks_byte(int D, int row);
int64_t kv4o_side_vs_byte(int D, int row);

/* Write the byte image that appending positions [0, lens[b]) of every sequence
 * leaves in the page pool and the side cache. k, v: bf16 bits [B][Lmax][Hkv][D].
 * page_table: [B][pt_stride]. Bytes not written are left untouched.
 * Returns the OR of range flags (1 = a scale overflowed). */
int kv4o_write_cache(const kv4o_shape *sh, const uint16_t *k, const uint16_t *v, int Lmax,
                     const int32_t *lens, const int32_t *page_table, int pt_stride,
                     uint8_t *pool, int64_t pool_bytes, uint8_t *side, int64_t side_bytes);

/* Dequantised K and V rows of (sequence b, KV head h) as attention sees them:
 * INT8 values for positions in the protected set, INT4 values elsewhere.
 * khat, vhat: [lens[b]][D] doubles. */
void kv4o_dequant_rows(const kv4o_shape *sh, const uint16_t *k, const uint16_t *v, int Lmax,
                       const int32_t *lens, int b, int h, double *khat, double *vhat);

/* ---- attention ---- */
/* Softmax attention of every query head over the retained positions.
 * q: bf16 bits [B][Hq][D]. mask: NULL or bits [B][Hkv][mask_stride] (bit p of
 * word p/32 set = position p retained). mode 0: KV4 values (INT4 + INT8
 * protection); mode 1: the bf16 values themselves. out: [B][Hq][D]. */
void kv4o_decode(const kv4o_shape *sh, const uint16_t *q, const uint16_t *k, const uint16_t *v,
                 int Lmax, const int32_t *lens, const uint32_t *mask, int mask_stride,
                 float softmax_scale, int mode, double *out);

/* Partial over an arbitrary set of n rows: m = max s, l = sum e^(s-m),
 * o = sum e^(s-m) v / l. Empty set: m = -inf, l = 0, o = 0. */
void kv4o_attend_rows(int D, const double *q, const double *krows, const double *vrows, int n,
                      double scale, double *m, double *l, double *o);
/* Exact merge of C partials: M = max m_c, W_c = l_c e^(m_c - M),
 * out = sum W_c o_c / sum W_c. All empty: out = 0. */
void kv4o_merge(int D, int C, const double *m, const double *l, const double *o, double *out);

/* ---- retained-position selection ---- */
/* Per (b, h): forced set F = first min(sink, L) and last min(recent, L)
 * positions; k = floor(L * permille / 1000); keep F plus the max(0, k - |F|)
 * best other positions by (score descending, index ascending). */
void kv4o_topk(const float *scores, int64_t score_stride, const int32_t *lens, int B, int Hkv,
               int permille, int sink, int recent, uint32_t *mask, int mask_stride, int32_t *count);

/* ---- page-granular eviction and compaction ([KVP], [KVS]) ----
 * Per sequence b with L = lens[b] and n = ceil(L/16) logical pages.
 * Candidates: full pages (16 positions < L) none of whose positions is in the
 * INT8 set (p < sink or p >= L - recent); every other page is kept. Page score:
 * the fp64 sum of its 16 * Hkv scores in (head, slot) order. k = floor(n *
 * permille / 1000); the max(0, k - (n - candidates)) best candidates (score
 * descending, index ascending) are kept, the other e are evicted. Then:
 * lens[b] -= 16 e; page_table row b = surviving entries in order, then entries
 * [n, pt_stride), then e times -1; freed[b][0..e) = evicted ids in logical
 * order (freed is [B][pt_stride]); freed_count[b] = e; in the side cache ring
 * page q of every (b, h) moves to ring page (q - e) mod (recent / 16).
 * scores: [B][Hkv][score_stride]; requires lens[b] <= score_stride and
 * lens[b] <= 16 * pt_stride. */
void kv4o_evict_pages(const float *scores, int64_t score_stride, int32_t *lens, int B, int Hkv, int D,
                      int permille, int sink, int recent, int32_t *page_table, int pt_stride,
                      int32_t *freed, int32_t *freed_count, uint8_t *side);

/* ---- learner-side attention under the shadow mask ([SMD] sec. 1, Figure 1) ----
 * q: bf16 bits [B][T][Hq][D]; k, v: bf16 bits [B][T][Hkv][D]; lens: NULL or [B]
 * (positions >= lens[b] give 0 and are never attended). mask: NULL (dense
 * causal) or bits [B][Hkv][T][mask_stride]: row t of KV head h lists the
 * positions the rollout kept for the query at position t. Query t of head hq
 * (KV head hq / (Hq/Hkv)) attends to {p <= t : bit p of row t set} over the bf16
 * values; an empty set gives 0. out: [B][T][Hq][D]. */
void kv4o_masked_attn(int B, int T, int Hq, int Hkv, int D, const uint16_t *q, const uint16_t *k,
                      const uint16_t *v, const int32_t *lens, const uint32_t *mask, int mask_stride,
                      float softmax_scale, double *out);

#ifdef __cplusplus
}
#endif
#endif
