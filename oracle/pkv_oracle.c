/*
 * pkv_oracle.c -- plain FP64 CPU oracle for paged KV-cache decode attention.
 *
 * TEST INFRASTRUCTURE ONLY (see pkv_oracle.h).  Slow and literal on purpose:
 * no blocking, no fusion, no online softmax.  Each function names the passage
 * of the pages it restates.
 */
#include "pkv_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* Shapes of the Llama-3.2-1B attention block ("Construye tu propio motor de
 * inferencia LLM...", section "La arquitectura del modelo: Llama 3.2 1B"):
 * hidden 2048 = 32 query heads x 64; k/v_proj out 512 = 8 kv heads x 64.
 * 16 tokens per page: "Curso gratuito recorre la inferencia de LLM...",
 * section "¿Cómo administra el motor la memoria de la caché KV?". */
#define O_TOKENS_PER_PAGE 16
#define O_Q_HEADS 32
#define O_KV_HEADS 8
#define O_DIM 64
/* "Atención de Consulta Agrupada (GQA)": 4 query heads use one kv head. */
#define O_Q_PER_KV 4

/* Offset (in 16-bit elements) of element d of token slot `slot`, kv head g,
 * K (kv = 0) or V (kv = 1), of physical page `page`.  Layout reading:
 * page[kv][g][slot][d]. */
static int64_t o_offset(int64_t page, int kv, int g, int slot, int d) {
  return ((((page * 2 + kv) * O_KV_HEADS + g) * O_TOKENS_PER_PAGE + slot) *
          O_DIM) + d;
}

/* A BF16 value is the upper half of an IEEE binary32; widening is exact. */
static double o_bf16(uint16_t bits) {
  uint32_t w = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &w, sizeof f);
  return (double)f;
}

/* Physical page holding logical token t of sequence b at `layer`, or -1 when
 * the block table entry is outside the pool. */
static int64_t o_page_of(const int32_t *bt, int32_t batch, int32_t max_blocks,
                         int32_t layer, int32_t b, int64_t t,
                         int32_t num_pages) {
  int64_t j = t / O_TOKENS_PER_PAGE;
  int32_t phys = bt[((int64_t)layer * batch + b) * max_blocks + j];
  if (phys < 0 || phys >= num_pages) return -1;
  return phys;
}

int pkvo_append(uint16_t *pool, int32_t num_pages, const int32_t *block_tables,
                int32_t num_layers, int32_t batch, int32_t max_blocks,
                const int32_t *seq_lens, const uint16_t *k_new,
                const uint16_t *v_new, int32_t layer) {
  /* The decode step adds the new token's K/V to the cache (comrad404 article
   * on samir-vllm, section "Что README говорит о KV-кэше и пакетном
   * декодировании"); it lands in slot (L-1) % 16 of the page the block table
   * names for logical page (L-1) / 16. */
  if (!pool || !block_tables || !seq_lens || !k_new || !v_new) return PKVO_BAD_ARG;
  if (batch < 0 || max_blocks < 0 || num_pages < 0) return PKVO_BAD_ARG;
  if (layer < 0 || layer >= num_layers) return PKVO_BAD_ARG;
  for (int32_t b = 0; b < batch; ++b) {
    int32_t L = seq_lens[b];
    if (L < 1 || (int64_t)L > (int64_t)max_blocks * O_TOKENS_PER_PAGE) return PKVO_BAD_LEN;
    if (o_page_of(block_tables, batch, max_blocks, layer, b, L - 1, num_pages) < 0)
      return PKVO_BAD_PAGE;
  }
  for (int32_t b = 0; b < batch; ++b) {
    int64_t pos = seq_lens[b] - 1;
    int64_t page = o_page_of(block_tables, batch, max_blocks, layer, b, pos, num_pages);
    int slot = (int)(pos % O_TOKENS_PER_PAGE);
    for (int g = 0; g < O_KV_HEADS; ++g) {
      for (int d = 0; d < O_DIM; ++d) {
        int64_t src = ((int64_t)b * O_KV_HEADS + g) * O_DIM + d;
        pool[o_offset(page, 0, g, slot, d)] = k_new[src];
        pool[o_offset(page, 1, g, slot, d)] = v_new[src];
      }
    }
  }
  return PKVO_OK;
}

int pkvo_fill(uint16_t *pool, int32_t num_pages, const int32_t *block_tables,
              int32_t num_layers, int32_t batch, int32_t max_blocks, const int32_t *cu,
              const int32_t *start, const uint16_t *k_src, const uint16_t *v_src,
              int32_t layer) {
  /* Prefill writes a request's tokens into its pages (comrad404 article on
   * samir-vllm, section "Что README говорит о KV-кэше и пакетном
   * декодировании"), token by token through the block table. */
  if (!pool || !block_tables || !cu || !start || !k_src || !v_src) return PKVO_BAD_ARG;
  if (batch < 0 || max_blocks < 0 || num_pages < 0) return PKVO_BAD_ARG;
  if (layer < 0 || layer >= num_layers) return PKVO_BAD_ARG;
  if (batch > 0 && cu[0] != 0) return PKVO_BAD_ARG;
  for (int32_t b = 0; b < batch; ++b) {
    if (cu[b + 1] < cu[b] || start[b] < 0) return PKVO_BAD_ARG;
    int64_t end = (int64_t)start[b] + (cu[b + 1] - cu[b]);
    if (end > (int64_t)max_blocks * O_TOKENS_PER_PAGE) return PKVO_BAD_LEN;
    for (int64_t pos = start[b]; pos < end; ++pos)
      if (o_page_of(block_tables, batch, max_blocks, layer, b, pos, num_pages) < 0)
        return PKVO_BAD_PAGE;
  }
  for (int32_t b = 0; b < batch; ++b) {
    for (int32_t i = 0; i < cu[b + 1] - cu[b]; ++i) {
      int64_t pos = (int64_t)start[b] + i;
      int64_t page = o_page_of(block_tables, batch, max_blocks, layer, b, pos, num_pages);
      int slot = (int)(pos % O_TOKENS_PER_PAGE);
      for (int g = 0; g < O_KV_HEADS; ++g) {
        for (int d = 0; d < O_DIM; ++d) {
          int64_t src = ((int64_t)(cu[b] + i) * O_KV_HEADS + g) * O_DIM + d;
          pool[o_offset(page, 0, g, slot, d)] = k_src[src];
          pool[o_offset(page, 1, g, slot, d)] = v_src[src];
        }
      }
    }
  }
  return PKVO_OK;
}

int pkvo_gather(const uint16_t *pool, int32_t num_pages,
                const int32_t *block_tables, int32_t num_layers, int32_t batch,
                int32_t max_blocks, const int32_t *seq_lens, int32_t layer,
                uint16_t *k_out, uint16_t *v_out, int32_t max_seq_len) {
  /* Logical-to-physical walk of the block table, token by token, as the
   * "Curso gratuito..." page's KV-cache section describes it. */
  if (!pool || !block_tables || !seq_lens || !k_out || !v_out) return PKVO_BAD_ARG;
  if (batch < 0 || max_blocks < 0 || max_seq_len < 0) return PKVO_BAD_ARG;
  if (layer < 0 || layer >= num_layers) return PKVO_BAD_ARG;
  for (int32_t b = 0; b < batch; ++b) {
    int32_t L = seq_lens[b];
    if (L < 0 || L > max_seq_len ||
        (int64_t)L > (int64_t)max_blocks * O_TOKENS_PER_PAGE)
      return PKVO_BAD_LEN;
    for (int64_t t = 0; t < L; ++t)
      if (o_page_of(block_tables, batch, max_blocks, layer, b, t, num_pages) < 0)
        return PKVO_BAD_PAGE;
  }
  for (int32_t b = 0; b < batch; ++b) {
    for (int g = 0; g < O_KV_HEADS; ++g) {
      for (int64_t t = 0; t < seq_lens[b]; ++t) {
        int64_t page = o_page_of(block_tables, batch, max_blocks, layer, b, t, num_pages);
        int slot = (int)(t % O_TOKENS_PER_PAGE);
        for (int d = 0; d < O_DIM; ++d) {
          int64_t dst = (((int64_t)b * O_KV_HEADS + g) * max_seq_len + t) * O_DIM + d;
          k_out[dst] = pool[o_offset(page, 0, g, slot, d)];
          v_out[dst] = pool[o_offset(page, 1, g, slot, d)];
        }
      }
    }
  }
  return PKVO_OK;
}

/* ---------------------------------------------------------------- decode -- */

typedef struct {
  const uint16_t *q, *pool;
  const int32_t *bt, *seq_lens, *rows;
  int32_t num_pages, batch, max_blocks, layer, nrows, first, stride;
  double scale;
  double *out;
} o_job;

/* Attention of the 32 query heads of sequence b over its L cached tokens:
 *   s[t]  = scale * sum_d q[h][d] * K[t][g][d],       g = h / 4
 *   w[t]  = exp(s[t] - max_t s)
 *   out[h][d] = sum_t w[t] * V[t][g][d] / sum_t w[t]
 * This is plain softmax attention; the pages' FP32 online softmax
 * ("Curso gratuito...", KV-cache section) is a way of computing exactly this
 * sum in one pass, so the oracle is the definition itself, in double. */
static void o_decode_one(const o_job *jb, int32_t b, double *s, double *w) {
  int32_t L = jb->seq_lens[b];
  double *o = jb->out + (int64_t)b * O_Q_HEADS * O_DIM;
  for (int h = 0; h < O_Q_HEADS; ++h) {
    int g = h / O_Q_PER_KV;
    const uint16_t *qh = jb->q + ((int64_t)b * O_Q_HEADS + h) * O_DIM;
    double *oh = o + (int64_t)h * O_DIM;
    if (L == 0) {
      for (int d = 0; d < O_DIM; ++d) oh[d] = 0.0;
      continue;
    }
    /* pass 1: scores, page by page through the block table */
    for (int64_t t = 0; t < L; ++t) {
      int64_t page = o_page_of(jb->bt, jb->batch, jb->max_blocks, jb->layer, b, t,
                               jb->num_pages);
      int slot = (int)(t % O_TOKENS_PER_PAGE);
      double acc = 0.0;
      for (int d = 0; d < O_DIM; ++d)
        acc += o_bf16(qh[d]) * o_bf16(jb->pool[o_offset(page, 0, g, slot, d)]);
      s[t] = jb->scale * acc;
    }
    /* pass 2: maximum */
    double m = s[0];
    for (int64_t t = 1; t < L; ++t)
      if (s[t] > m) m = s[t];
    /* pass 3: weights and their sum */
    double l = 0.0;
    for (int64_t t = 0; t < L; ++t) {
      w[t] = exp(s[t] - m);
      l += w[t];
    }
    /* pass 4: normalised weighted sum of values */
    for (int d = 0; d < O_DIM; ++d) oh[d] = 0.0;
    for (int64_t t = 0; t < L; ++t) {
      int64_t page = o_page_of(jb->bt, jb->batch, jb->max_blocks, jb->layer, b, t,
                               jb->num_pages);
      int slot = (int)(t % O_TOKENS_PER_PAGE);
      for (int d = 0; d < O_DIM; ++d)
        oh[d] += w[t] * o_bf16(jb->pool[o_offset(page, 1, g, slot, d)]);
    }
    for (int d = 0; d < O_DIM; ++d) oh[d] /= l;
  }
}

static void *o_decode_worker(void *arg) {
  const o_job *jb = (const o_job *)arg;
  int32_t maxL = 1;
  for (int32_t i = jb->first; i < jb->nrows; i += jb->stride) {
    int32_t b = jb->rows ? jb->rows[i] : i;
    if (jb->seq_lens[b] > maxL) maxL = jb->seq_lens[b];
  }
  double *s = (double *)malloc(sizeof(double) * (size_t)maxL);
  double *w = (double *)malloc(sizeof(double) * (size_t)maxL);
  if (!s || !w) {
    free(s);
    free(w);
    return (void *)1;
  }
  for (int32_t i = jb->first; i < jb->nrows; i += jb->stride) {
    int32_t b = jb->rows ? jb->rows[i] : i;
    o_decode_one(jb, b, s, w);
  }
  free(s);
  free(w);
  return NULL;
}

int pkvo_decode(const uint16_t *q, const uint16_t *pool, int32_t num_pages,
                const int32_t *block_tables, int32_t num_layers, int32_t batch,
                int32_t max_blocks, const int32_t *seq_lens, int32_t layer,
                double scale, double *out, const int32_t *rows, int32_t nrows,
                int32_t nthreads) {
  if (!q || !pool || !block_tables || !seq_lens || !out) return PKVO_BAD_ARG;
  if (batch < 0 || max_blocks < 0 || num_pages < 0) return PKVO_BAD_ARG;
  if (layer < 0 || layer >= num_layers) return PKVO_BAD_ARG;
  if (!rows) nrows = batch;
  if (nrows < 0) return PKVO_BAD_ARG;
  for (int32_t i = 0; i < nrows; ++i) {
    int32_t b = rows ? rows[i] : i;
    if (b < 0 || b >= batch) return PKVO_BAD_ARG;
    int32_t L = seq_lens[b];
    if (L < 0 || (int64_t)L > (int64_t)max_blocks * O_TOKENS_PER_PAGE) return PKVO_BAD_LEN;
    for (int64_t t = 0; t < L; t += O_TOKENS_PER_PAGE)
      if (o_page_of(block_tables, batch, max_blocks, layer, b, t, num_pages) < 0)
        return PKVO_BAD_PAGE;
  }
  if (nthreads < 1) nthreads = 1;
  if (nthreads > nrows) nthreads = nrows > 0 ? nrows : 1;

  o_job *jobs = (o_job *)calloc((size_t)nthreads, sizeof(o_job));
  pthread_t *tids = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
  if (!jobs || !tids) {
    free(jobs);
    free(tids);
    return PKVO_BAD_ARG;
  }
  int rc = PKVO_OK;
  for (int i = 0; i < nthreads; ++i) {
    o_job j = {q, pool, block_tables, seq_lens, rows, num_pages, batch, max_blocks,
               layer, nrows, i, nthreads, scale, out};
    jobs[i] = j;
  }
  if (nthreads == 1) {
    if (o_decode_worker(&jobs[0])) rc = PKVO_BAD_ARG;
  } else {
    for (int i = 0; i < nthreads; ++i)
      pthread_create(&tids[i], NULL, o_decode_worker, &jobs[i]);
    for (int i = 0; i < nthreads; ++i) {
      void *r = NULL;
      pthread_join(tids[i], &r);
      if (r) rc = PKVO_BAD_ARG;
    }
  }
  free(jobs);
  free(tids);
  return rc;
}
