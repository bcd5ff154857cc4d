/*
 * kv4_oracle.c -- plain fp64 CPU oracle for KV4-RL decode attention.
 *
 * TEST INFRASTRUCTURE ONLY (see kv4_oracle.h). Written to be checked by eye
 * against the pages: no blocking, no fusion, no reordering beyond what the
 * definitions state. Every loop is the definition written out.
 */
#include "kv4_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define PAGE_TOKENS 16
#define GROUP 32

/* ------------------------------------------------------------------ */
/* Number formats (IEEE 754 binary16 / bfloat16 definitions).          */
/* ------------------------------------------------------------------ */

double kv4o_fp16_to_double(uint16_t bits) {
  int sign = (bits >> 15) & 1;
  int e = (bits >> 10) & 0x1F;
  int m = bits & 0x3FF;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -24);               /* subnormal: m * 2^-24 */
  } else if (e == 31) {
    v = m ? NAN : INFINITY;
  } else {
    v = ldexp((double)(1024 + m), e - 25);    /* (1 + m/1024) * 2^(e-15) */
  }
  return sign ? -v : v;
}

double kv4o_bf16_to_double(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Smallest binary16 value >= y, for y >= 0 (round toward +infinity). */
uint16_t kv4o_fp16_round_up(double y) {
  if (y != y) return 0x7E00;
  if (y <= 0.0) return 0x0000;
  if (y > 65504.0) return 0x7C00;
  if (y < ldexp(1.0, -14)) {
    /* subnormal range: multiples of 2^-24 */
    double m = ceil(ldexp(y, 24));
    return (uint16_t)m;                       /* m == 1024 is exactly 2^-14 = 0x0400 */
  }
  int e2;
  frexp(y, &e2);                              /* y in [2^(e2-1), 2^e2) */
  int E = e2 - 1;
  double m = ceil(ldexp(y, 10 - E));          /* significand in units of the ulp: [1024, 2048] */
  if (m >= 2048.0) {
    m = 1024.0;
    E += 1;
  }
  if (E > 15) return 0x7C00;
  return (uint16_t)(((E + 15) << 10) | ((int)m - 1024));
}

/* Round to the nearest integer, ties to the even integer. */
double kv4o_round_half_even(double x) {
  double f = floor(x);
  double d = x - f;
  if (d > 0.5) return f + 1.0;
  if (d < 0.5) return f;
  return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* ------------------------------------------------------------------ */
/* Quantiser: symmetric, scale = RU_fp16(max|x| / qmax), code = RNE(x/s). */
/* ------------------------------------------------------------------ */

static int quant_sym(const uint16_t *x, int n, int qmax, uint16_t *scale_bits, int8_t *codes) {
  double a = 0.0;
  for (int i = 0; i < n; ++i) {
    double v = fabs(kv4o_bf16_to_double(x[i]));
    if (v > a) a = v;
  }
  if (a == 0.0) {
    *scale_bits = 0;
    for (int i = 0; i < n; ++i) codes[i] = 0;
    return 0;
  }
  int overflow = 0;
  uint16_t s = kv4o_fp16_round_up(a / (double)qmax);
  if (s == 0x7C00) {
    s = 0x7BFF;
    overflow = 1;
  }
  double sv = kv4o_fp16_to_double(s);
  for (int i = 0; i < n; ++i) {
    double c = kv4o_round_half_even(kv4o_bf16_to_double(x[i]) / sv);
    if (c > qmax) c = qmax;       /* reachable only on overflow */
    if (c < -qmax) c = -qmax;
    codes[i] = (int8_t)c;
  }
  *scale_bits = s;
  return overflow;
}

int kv4o_quant_int4(const uint16_t *x_bf16, int n, uint16_t *scale_bits, int8_t *codes) {
  return quant_sym(x_bf16, n, 7, scale_bits, codes);
}

int kv4o_quant_int8(const uint16_t *x_bf16, int n, uint16_t *scale_bits, int8_t *codes) {
  return quant_sym(x_bf16, n, 127, scale_bits, codes);
}

/* ------------------------------------------------------------------ */
/* Byte layout of one head block of one physical page (16 slots):      */
/*   [K codes 8D][V codes 8D][K scales D][V scales D]   = 18*D bytes    */
/* K codes: row r at r*D/2; inside a row, chunk t (t = (d%32)/8) at     */
/*   t*D/8, word i (i = d/32) at 4*i inside the chunk, element k = d%8  */
/*   in nibble k of that 32-bit word (little-endian byte k/2, low nibble */
/*   for even k).                                                       */
/* V codes: 32 "lanes" (g, t) with g = d%8 and t = (r%8)/2, stored at  */
/*   position P = 8t + (g XOR 2t), so the four rows {2t, 2t+1, 2t+8,    */
/*   2t+9} own 128 contiguous bytes of each 512-byte block; m = d/16;   */
/*   32-bit word (lane, m) at 4*((m/4)*128 + P*4 + m%4); inside the     */
/*   word byte 2*(r%2) + r/8, nibble (d%16)/8.                          */
/* Scales: fp16, row r group i at 2*(r*D/32 + i).                       */
/* ------------------------------------------------------------------ */

int64_t kv4o_page_head_bytes(int D) { return 18LL * D; }

int64_t kv4o_k_code_byte(int D, int r, int d, int *nibble) {
  int i = d / 32, t = (d % 32) / 8, k = d % 8;
  *nibble = k % 2;
  return (int64_t)r * (D / 2) + (int64_t)t * (D / 8) + 4 * i + k / 2;
}

int64_t kv4o_v_code_byte(int D, int r, int d, int *nibble) {
  int m = d / 16, g = d % 8, hi8 = (d % 16) / 8;
  int t = (r % 8) / 2, rodd = r % 2, r8 = r / 8;
  int pos = 8 * t + (g ^ (2 * t));
  int64_t word = (int64_t)(m / 4) * 128 + pos * 4 + (m % 4);
  *nibble = hi8;
  return 8LL * D + 4 * word + 2 * rodd + r8;
}

int64_t kv4o_k_scale_byte(int D, int r, int grp) { return 16LL * D + 2LL * (r * (D / 32) + grp); }
int64_t kv4o_v_scale_byte(int D, int r, int grp) { return 17LL * D + 2LL * (r * (D / 32) + grp); }

/* INT8 side block per (sequence, KV head): a sequence of 16-row pages. With
 * sink > 0 the first page holds sink rows 0..15 (position p < sink in row p);
 * then recent/16 ring pages hold ring slots 0..recent-1 (position p in slot
 * p mod recent, page 16-slot blocks in slot order). Each page is
 *   [K codes 16*D][K scales 16 x fp16][V scales 16 x fp16][V codes 16*D]
 * and the codes of a page are in register-fragment order:
 *   K row r, element d: t = d / (D/4), j = (d % (D/4)) / 4, e = d % 4,
 *     lane = 4*(r%8) + t, word w = (r/8)*(D/16) + j,
 *     byte = (w/4)*512 + lane*16 + (w%4)*4 + e.
 *   V row r, element d: m = d/16, g = d%8, lane = 4*g + (r%8)/2,
 *     word w = 2*m + r/8, byte = (w/4)*512 + lane*16 + (w%4)*4 + 2*(r%2) + (d%16)/8.
 */
int kv4o_side_pages(int sink, int recent) { return (sink > 0 ? 1 : 0) + recent / 16; }
int64_t kv4o_side_page_bytes(int D) { return 32LL * D + 64; }
int64_t kv4o_side_head_bytes(int D, int sink, int recent) {
  return kv4o_side_pages(sink, recent) * kv4o_side_page_bytes(D);
}

int64_t kv4o_side_k_byte(int D, int row, int d) {
  const int r = row % 16;
  const int t = d / (D / 4), j = (d % (D / 4)) / 4, e = d % 4;
  const int lane = 4 * (r % 8) + t;
  const int w = (r / 8) * (D / 16) + j;
  return (int64_t)(row / 16) * kv4o_side_page_bytes(D) + (w / 4) * 512 + lane * 16 + (w % 4) * 4 + e;
}

int64_t kv4o_side_v_byte(int D, int row, int d) {
  const int r = row % 16;
  const int m = d / 16, g = d % 8;
  const int lane = 4 * g + (r % 8) / 2;
  const int w = 2 * m + r / 8;
  return (int64_t)(row / 16) * kv4o_side_page_bytes(D) + 16LL * D + 64 + (w / 4) * 512 + lane * 16 +
         (w % 4) * 4 + 2 * (r % 2) + (d % 16) / 8;
}

int64_t kv4o_side_ks_byte(int D, int row) {
  return (int64_t)(row / 16) * kv4o_side_page_bytes(D) + 16LL * D + 2 * (row % 16);
}

int64_t kv4o_side_vs_byte(int D, int row) {
  return (int64_t)(row / 16) * kv4o_side_page_bytes(D) + 16LL * D + 32 + 2 * (row % 16);
}

static void put_nibble(uint8_t *p, int nibble, int code) {
  uint8_t v = (uint8_t)(code & 0xF);
  if (nibble) *p = (uint8_t)((*p & 0x0F) | (v << 4));
  else *p = (uint8_t)((*p & 0xF0) | v);
}

static void put_u16(uint8_t *p, uint16_t v) {
  p[0] = (uint8_t)(v & 0xFF);
  p[1] = (uint8_t)(v >> 8);
}

/* The INT8-protected set of [KV4RL] sec. 3: the first `sink` positions and the
 * `recent` most recent cached positions (the new token included). */
static int is_protected(int p, int L, int sink, int recent) {
  return p < sink || p >= L - recent;
}

int kv4o_write_cache(const kv4o_shape *sh, const uint16_t *k, const uint16_t *v, int Lmax,
                     const int32_t *lens, const int32_t *page_table, int pt_stride,
                     uint8_t *pool, int64_t pool_bytes, uint8_t *side, int64_t side_bytes) {
  const int D = sh->D, Hkv = sh->Hkv, S = sh->sink, R = sh->recent;
  const int64_t head_bytes = kv4o_page_head_bytes(D);
  const int64_t page_bytes = head_bytes * Hkv;
  const int64_t side_stride = kv4o_side_head_bytes(D, S, R);
  int flags = 0;
  int8_t codes[1024];
  uint16_t sc;
  (void)pool_bytes;
  (void)side_bytes;
  for (int b = 0; b < sh->B; ++b) {
    const int L = lens[b];
    for (int p = 0; p < L; ++p) {
      const int page = page_table[(int64_t)b * pt_stride + p / PAGE_TOKENS];
      const int r = p % PAGE_TOKENS;
      for (int h = 0; h < Hkv; ++h) {
        const uint16_t *krow = k + (((int64_t)b * Lmax + p) * Hkv + h) * D;
        const uint16_t *vrow = v + (((int64_t)b * Lmax + p) * Hkv + h) * D;
        uint8_t *blk = pool + (int64_t)page * page_bytes + h * head_bytes;
        /* INT4 copy of every position ([KV4RL] sec. 3: the full context is paged INT4). */
        for (int grp = 0; grp < D / GROUP; ++grp) {
          int nib;
          flags |= kv4o_quant_int4(krow + grp * GROUP, GROUP, &sc, codes);
          for (int e = 0; e < GROUP; ++e) {
            int64_t off = kv4o_k_code_byte(D, r, grp * GROUP + e, &nib);
            put_nibble(blk + off, nib, codes[e]);
          }
          put_u16(blk + kv4o_k_scale_byte(D, r, grp), sc);
          flags |= kv4o_quant_int4(vrow + grp * GROUP, GROUP, &sc, codes);
          for (int e = 0; e < GROUP; ++e) {
            int64_t off = kv4o_v_code_byte(D, r, grp * GROUP + e, &nib);
            put_nibble(blk + off, nib, codes[e]);
          }
          put_u16(blk + kv4o_v_scale_byte(D, r, grp), sc);
        }
        /* INT8 side cache: sink row p for p < S; ring slot p mod R for the
         * last R positions. Rows count from the block start: the sink page
         * (16 rows) comes first when S > 0. */
        uint8_t *sb = side + ((int64_t)b * Hkv + h) * side_stride;
        const int ring0 = S > 0 ? 16 : 0;
        int row = -1;
        for (int pass = 0; pass < 2; ++pass) {
          if (pass == 0) row = (p < S) ? p : -1;
          else row = (R > 0 && p >= L - R) ? ring0 + p % R : -1;
          if (row < 0) continue;
          flags |= kv4o_quant_int8(krow, D, &sc, codes);
          for (int d = 0; d < D; ++d) sb[kv4o_side_k_byte(D, row, d)] = (uint8_t)codes[d];
          put_u16(sb + kv4o_side_ks_byte(D, row), sc);
          flags |= kv4o_quant_int8(vrow, D, &sc, codes);
          for (int d = 0; d < D; ++d) sb[kv4o_side_v_byte(D, row, d)] = (uint8_t)codes[d];
          put_u16(sb + kv4o_side_vs_byte(D, row), sc);
        }
      }
    }
  }
  return flags;
}

/* Dequantised row: INT8 values inside the protected set, INT4 values elsewhere. */
static void dequant_row(const uint16_t *row, int D, int protected_, double *out) {
  int8_t codes[1024];
  uint16_t sc;
  if (protected_) {
    kv4o_quant_int8(row, D, &sc, codes);
    double s = kv4o_fp16_to_double(sc);
    for (int d = 0; d < D; ++d) out[d] = codes[d] * s;
  } else {
    for (int grp = 0; grp < D / GROUP; ++grp) {
      kv4o_quant_int4(row + grp * GROUP, GROUP, &sc, codes);
      double s = kv4o_fp16_to_double(sc);
      for (int e = 0; e < GROUP; ++e) out[grp * GROUP + e] = codes[e] * s;
    }
  }
}

void kv4o_dequant_rows(const kv4o_shape *sh, const uint16_t *k, const uint16_t *v, int Lmax,
                       const int32_t *lens, int b, int h, double *khat, double *vhat) {
  const int D = sh->D, Hkv = sh->Hkv, L = lens[b];
  for (int p = 0; p < L; ++p) {
    const int prot = is_protected(p, L, sh->sink, sh->recent);
    dequant_row(k + (((int64_t)b * Lmax + p) * Hkv + h) * D, D, prot, khat + (int64_t)p * D);
    dequant_row(v + (((int64_t)b * Lmax + p) * Hkv + h) * D, D, prot, vhat + (int64_t)p * D);
  }
}

/* ------------------------------------------------------------------ */
/* Attention                                                           */
/* ------------------------------------------------------------------ */

static int mask_bit(const uint32_t *mask, int mask_stride, int b, int Hkv, int h, int p) {
  if (!mask) return 1;
  const uint32_t w = mask[((int64_t)b * Hkv + h) * mask_stride + p / 32];
  return (w >> (p % 32)) & 1u;
}

void kv4o_decode(const kv4o_shape *sh, const uint16_t *q, const uint16_t *k, const uint16_t *v,
                 int Lmax, const int32_t *lens, const uint32_t *mask, int mask_stride,
                 float softmax_scale, int mode, double *out) {
  const int B = sh->B, Hq = sh->Hq, Hkv = sh->Hkv, D = sh->D;
  const int G = Hq / Hkv;
  const double tau = (double)softmax_scale;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int b = 0; b < B; ++b) {
    for (int h = 0; h < Hkv; ++h) {
      const int L = lens[b];
      double *s = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * G);
      double *row = (double *)malloc(sizeof(double) * D);
      double *qd = (double *)malloc(sizeof(double) * (size_t)G * D);
      double *acc = (double *)calloc((size_t)G * D, sizeof(double));
      double m[64], l[64];
      for (int g = 0; g < G; ++g) {
        for (int d = 0; d < D; ++d)
          qd[g * D + d] = kv4o_bf16_to_double(q[((int64_t)b * Hq + h * G + g) * D + d]);
        m[g] = -INFINITY;
        l[g] = 0.0;
      }
      /* scores s_p = tau * (q . K_p) over the retained positions */
      for (int p = 0; p < L; ++p) {
        if (!mask_bit(mask, mask_stride, b, Hkv, h, p)) continue;
        const uint16_t *krow = k + (((int64_t)b * Lmax + p) * Hkv + h) * D;
        if (mode == 0) dequant_row(krow, D, is_protected(p, L, sh->sink, sh->recent), row);
        else for (int d = 0; d < D; ++d) row[d] = kv4o_bf16_to_double(krow[d]);
        for (int g = 0; g < G; ++g) {
          double dot = 0.0;
          for (int d = 0; d < D; ++d) dot += qd[g * D + d] * row[d];
          s[(int64_t)p * G + g] = tau * dot;
          if (tau * dot > m[g]) m[g] = tau * dot;
        }
      }
      /* o = sum_p e^(s_p - m) V_p / sum_p e^(s_p - m) */
      for (int p = 0; p < L; ++p) {
        if (!mask_bit(mask, mask_stride, b, Hkv, h, p)) continue;
        const uint16_t *vrow = v + (((int64_t)b * Lmax + p) * Hkv + h) * D;
        if (mode == 0) dequant_row(vrow, D, is_protected(p, L, sh->sink, sh->recent), row);
        else for (int d = 0; d < D; ++d) row[d] = kv4o_bf16_to_double(vrow[d]);
        for (int g = 0; g < G; ++g) {
          const double w = exp(s[(int64_t)p * G + g] - m[g]);
          l[g] += w;
          for (int d = 0; d < D; ++d) acc[g * D + d] += w * row[d];
        }
      }
      for (int g = 0; g < G; ++g)
        for (int d = 0; d < D; ++d)
          out[((int64_t)b * Hq + h * G + g) * D + d] = (l[g] > 0.0) ? acc[g * D + d] / l[g] : 0.0;
      free(s);
      free(row);
      free(qd);
      free(acc);
    }
  }
}

void kv4o_attend_rows(int D, const double *q, const double *krows, const double *vrows, int n,
                      double scale, double *m, double *l, double *o) {
  double mx = -INFINITY;
  double *s = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  for (int i = 0; i < n; ++i) {
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += q[d] * krows[(int64_t)i * D + d];
    s[i] = scale * dot;
    if (s[i] > mx) mx = s[i];
  }
  double sum = 0.0;
  for (int d = 0; d < D; ++d) o[d] = 0.0;
  for (int i = 0; i < n; ++i) {
    const double w = exp(s[i] - mx);
    sum += w;
    for (int d = 0; d < D; ++d) o[d] += w * vrows[(int64_t)i * D + d];
  }
  for (int d = 0; d < D; ++d) o[d] = (sum > 0.0) ? o[d] / sum : 0.0;
  *m = mx;
  *l = sum;
  free(s);
}

void kv4o_merge(int D, int C, const double *m, const double *l, const double *o, double *out) {
  double M = -INFINITY;
  for (int c = 0; c < C; ++c)
    if (l[c] > 0.0 && m[c] > M) M = m[c];
  double den = 0.0;
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  for (int c = 0; c < C; ++c) {
    if (!(l[c] > 0.0)) continue;
    const double W = l[c] * exp(m[c] - M);
    den += W;
    for (int d = 0; d < D; ++d) out[d] += W * o[(int64_t)c * D + d];
  }
  for (int d = 0; d < D; ++d) out[d] = (den > 0.0) ? out[d] / den : 0.0;
}

/* ------------------------------------------------------------------ */
/* Retained-position selection: score -> rank -> truncate ([KVP]).     */
/* ------------------------------------------------------------------ */

typedef struct {
  double score;
  int idx;
} cand_t;

static int cand_cmp(const void *a, const void *b) {
  const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
  if (x->score > y->score) return -1;   /* higher score first */
  if (x->score < y->score) return 1;
  return (x->idx < y->idx) ? -1 : (x->idx > y->idx);   /* tie: lower index first */
}

void kv4o_topk(const float *scores, int64_t score_stride, const int32_t *lens, int B, int Hkv,
               int permille, int sink, int recent, uint32_t *mask, int mask_stride, int32_t *count) {
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int b = 0; b < B; ++b) {
    for (int h = 0; h < Hkv; ++h) {
      const int L = lens[b];
      const float *row = scores + ((int64_t)b * Hkv + h) * score_stride;
      uint32_t *mrow = mask + ((int64_t)b * Hkv + h) * mask_stride;
      for (int w = 0; w < (L + 31) / 32; ++w) mrow[w] = 0u;
      const int64_t kbud = (int64_t)L * permille / 1000;
      cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (size_t)(L > 0 ? L : 1));
      int nc = 0, nforced = 0;
      for (int p = 0; p < L; ++p) {
        if (is_protected(p, L, sink, recent)) {
          mrow[p / 32] |= 1u << (p % 32);
          ++nforced;
        } else {
          c[nc].score = (double)row[p];
          c[nc].idx = p;
          ++nc;
        }
      }
      qsort(c, (size_t)nc, sizeof(cand_t), cand_cmp);
      int64_t take = kbud - nforced;
      if (take < 0) take = 0;
      if (take > nc) take = nc;
      for (int64_t i = 0; i < take; ++i) mrow[c[i].idx / 32] |= 1u << (c[i].idx % 32);
      if (count) count[(int64_t)b * Hkv + h] = (int32_t)(nforced + take);
      free(c);
    }
  }
}

/* ------------------------------------------------------------------ */
/* Page-granular eviction and compaction.                              */
/* [KVP] engineering-limitations section, third item (vLLM block       */
/* granularity): a paged cache evicts whole 16-position blocks, ranked  */
/* by the mean of their positions' scores. [KVS] method details (core   */
/* idea): the compacted cache keeps streaming -- later appends go on    */
/* into the surviving pages, nothing is flushed or re-prefilled.        */
/* ------------------------------------------------------------------ */

void kv4o_evict_pages(const float *scores, int64_t score_stride, int32_t *lens, int B, int Hkv, int D,
                      int permille, int sink, int recent, int32_t *page_table, int pt_stride,
                      int32_t *freed, int32_t *freed_count, uint8_t *side) {
  const int64_t side_stride = kv4o_side_head_bytes(D, sink, recent);
  const int64_t spb = kv4o_side_page_bytes(D);
  const int ring_pages = recent / PAGE_TOKENS, ring0 = sink > 0 ? 1 : 0;
  for (int b = 0; b < B; ++b) {
    const int L = lens[b];
    const int n = (L + PAGE_TOKENS - 1) / PAGE_TOKENS;
    int32_t *row = page_table + (int64_t)b * pt_stride;
    /* Candidates: full pages that hold no position of the INT8 set. */
    cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (size_t)(n > 0 ? n : 1));
    char *evict = (char *)calloc((size_t)(n > 0 ? n : 1), 1);
    int nc = 0;
    for (int j = 0; j < n; ++j) {
      int cand = (j + 1) * PAGE_TOKENS <= L;
      for (int p = j * PAGE_TOKENS; cand && p < (j + 1) * PAGE_TOKENS; ++p)
        if (is_protected(p, L, sink, recent)) cand = 0;
      if (!cand) continue;
      /* The page's score: its 16 * Hkv position scores added in fp64, head by
       * head and slot by slot. Every candidate holds the same number of
       * scores, so this sum orders pages as their mean does. */
      double s = 0.0;
      for (int h = 0; h < Hkv; ++h)
        for (int r = 0; r < PAGE_TOKENS; ++r)
          s += (double)scores[((int64_t)b * Hkv + h) * score_stride + (int64_t)j * PAGE_TOKENS + r];
      c[nc].score = s;
      c[nc].idx = j;
      ++nc;
    }
    const int64_t kbud = (int64_t)n * permille / 1000;
    int64_t take = kbud - (n - nc);
    if (take < 0) take = 0;
    if (take > nc) take = nc;
    qsort(c, (size_t)nc, sizeof(cand_t), cand_cmp);
    for (int i = (int)take; i < nc; ++i) evict[c[i].idx] = 1;
    const int e = nc - (int)take;

    /* Page table: surviving pages in order, then the entries past the last
     * logical page (mapped ahead for later appends), then -1 for the freed
     * tail. Evicted ids go to the free list in logical order. */
    int32_t *old = (int32_t *)malloc(sizeof(int32_t) * (size_t)pt_stride);
    memcpy(old, row, sizeof(int32_t) * (size_t)pt_stride);
    int w = 0, f = 0;
    for (int j = 0; j < pt_stride; ++j) {
      if (j < n && evict[j]) freed[(int64_t)b * pt_stride + f++] = old[j];
      else row[w++] = old[j];
    }
    while (w < pt_stride) row[w++] = -1;
    freed_count[b] = e;
    lens[b] = L - PAGE_TOKENS * e;

    /* Positions after an evicted page move down by 16 each, so position p of
     * the recent window becomes p - 16e and its ring slot (p - 16e) mod
     * recent: ring page q moves to ring page (q - e) mod (recent / 16). */
    if (ring_pages > 0 && e % ring_pages != 0) {
      uint8_t *tmp = (uint8_t *)malloc((size_t)(ring_pages * spb));
      for (int h = 0; h < Hkv; ++h) {
        uint8_t *ring = side + ((int64_t)b * Hkv + h) * side_stride + ring0 * spb;
        memcpy(tmp, ring, (size_t)(ring_pages * spb));
        for (int q = 0; q < ring_pages; ++q) {
          const int dst = ((q - e) % ring_pages + ring_pages) % ring_pages;
          memcpy(ring + dst * spb, tmp + q * spb, (size_t)spb);
        }
      }
      free(tmp);
    }
    free(old);
    free(evict);
    free(c);
  }
}

/* ------------------------------------------------------------------ */
/* Learner-side attention under the recorded shadow mask ([SMD] sec. 1 */
/* and Figure 1): the rollout records, for the query at each position, */
/* the set of positions its eviction kept; the learner's causal        */
/* attention applies exactly that set, over the full-precision (bf16)  */
/* K and V, so each row reproduces what the rollout attended to.       */
/* ------------------------------------------------------------------ */

void kv4o_masked_attn(int B, int T, int Hq, int Hkv, int D, const uint16_t *q, const uint16_t *k,
                      const uint16_t *v, const int32_t *lens, const uint32_t *mask, int mask_stride,
                      float softmax_scale, double *out) {
  const int G = Hq / Hkv;
  const double tau = (double)softmax_scale;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int b = 0; b < B; ++b) {
    for (int hq = 0; hq < Hq; ++hq) {
      const int h = hq / G;
      const int L = lens ? lens[b] : T;
      double *s = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
      double *qd = (double *)malloc(sizeof(double) * (size_t)D);
      for (int t = 0; t < T; ++t) {
        double *o = out + (((int64_t)b * T + t) * Hq + hq) * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        if (t >= L) continue;
        for (int d = 0; d < D; ++d) qd[d] = kv4o_bf16_to_double(q[(((int64_t)b * T + t) * Hq + hq) * D + d]);
        const uint32_t *mrow = mask ? mask + (((int64_t)b * Hkv + h) * T + t) * mask_stride : NULL;
        /* visible keys: p <= t (causal) whose bit is set in row t */
        double m = -INFINITY;
        for (int p = 0; p <= t; ++p) {
          s[p] = -INFINITY;
          if (mrow && !((mrow[p / 32] >> (p % 32)) & 1u)) continue;
          const uint16_t *kr = k + (((int64_t)b * T + p) * Hkv + h) * D;
          double dot = 0.0;
          for (int d = 0; d < D; ++d) dot += qd[d] * kv4o_bf16_to_double(kr[d]);
          s[p] = tau * dot;
          if (s[p] > m) m = s[p];
        }
        double l = 0.0;
        for (int p = 0; p <= t; ++p) {
          if (s[p] == -INFINITY) continue;
          const double w = exp(s[p] - m);
          const uint16_t *vr = v + (((int64_t)b * T + p) * Hkv + h) * D;
          l += w;
          for (int d = 0; d < D; ++d) o[d] += w * kv4o_bf16_to_double(vr[d]);
        }
        for (int d = 0; d < D; ++d) o[d] = (l > 0.0) ? o[d] / l : 0.0;
      }
      free(s);
      free(qd);
    }
  }
}
