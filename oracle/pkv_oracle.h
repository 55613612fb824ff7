/*
 * pkv_oracle.h -- plain FP64 CPU oracle for paged KV-cache decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library
 * and its Python binding) may include, link or call this code; only the
 * tests, the package's smoke check and the benchmark's CPU-baseline leg use
 * it.  It shares no header, constant or helper with the CUDA sources: every
 * shape constant and index formula below is written out again here from the
 * pages' description of the method.
 *
 * What it models (sources, by page title and section):
 *  - "Curso gratuito recorre la inferencia de LLM con videos, notas y un
 *    motor funcional en C++", section "¿Cómo administra el motor la memoria
 *    de la caché KV?": one shared pool of BF16 pages, each physical page
 *    holding keys and values of 16 tokens; a block table per sequence and
 *    layer; decode reads each sequence's pages in place (no contiguous
 *    prefix is gathered) with an FP32 online softmax.
 *  - the comrad404 article on samir-vllm ("Как устроен путь от текста
 *    запроса до следующего токена в языковой модели?"), section
 *    "Что README говорит о KV-кэше и пакетном декодировании": decode adds the
 *    new token's K/V to the cache.
 *  - "Construye tu propio motor de inferencia LLM de alto rendimiento en C++
 *    y CUDA", section "Atención de Consulta Agrupada (GQA)": four query heads
 *    share one key/value head, kv head = q head / 4; section "La
 *    arquitectura del modelo: Llama 3.2 1B": q_proj 2048->2048 and
 *    k/v_proj 2048->512, i.e. 32 query heads and 8 kv heads of dimension 64.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - page layout: page[kv in {K,V}][kv_head 0..7][slot 0..15][d 0..63] BF16,
 *    so element (page, kv, g, slot, d) sits at
 *    (((page*2 + kv)*8 + g)*16 + slot)*64 + d  (uint16 units);
 *  - block tables are int32 [num_layers][batch][max_blocks], row-major;
 *  - seq_lens hold the context length AFTER this step's append; the new
 *    token sits at position L-1 and decode attends to positions 0..L-1;
 *  - L == 0 gives an all-zero output row;
 *  - the softmax scale is a caller argument multiplying q.k.
 *
 * The decode here is deliberately NOT online: it is the textbook definition
 * (scores, max, exponentials, normalised weighted sum of values) in double
 * precision, walking the block table page by page in logical token order.
 */
#ifndef PKV_ORACLE_H
#define PKV_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  PKVO_OK = 0,
  PKVO_BAD_ARG = 1,   /* null pointer, negative size, layer out of range   */
  PKVO_BAD_LEN = 2,   /* seq_len < 0 (or < 1 for append) or > max_blocks*16 */
  PKVO_BAD_PAGE = 3   /* block-table entry outside [0, num_pages)          */
};

/* Append: for each sequence b, copy k_new[b][g][:] and v_new[b][g][:] (all 8
 * kv heads, bit copies) into slot (L-1) % 16 of the physical page
 * block_tables[layer][b][(L-1)/16], L = seq_lens[b] >= 1.  Checks every
 * sequence before writing anything; returns a PKVO_* code. */
int pkvo_append(uint16_t *pool, int32_t num_pages, const int32_t *block_tables,
                int32_t num_layers, int32_t batch, int32_t max_blocks,
                const int32_t *seq_lens, const uint16_t *k_new,
                const uint16_t *v_new, int32_t layer);

/* Fill (prefill, or chunked prefill): sequence b writes its tokens
 * k_src/v_src[cu[b] + i][g][:], i < cu[b+1] - cu[b], at positions
 * start[b] + i, each into slot pos % 16 of page block_tables[layer][b][pos/16]
 * (the prefill half of "prefill fills the request's pages, decode adds the
 * new token", comrad404 article, KV-cache section).  k_src / v_src are
 * [cu[batch]][8][64].  Checks every token before writing anything. */
int pkvo_fill(uint16_t *pool, int32_t num_pages, const int32_t *block_tables,
              int32_t num_layers, int32_t batch, int32_t max_blocks, const int32_t *cu,
              const int32_t *start, const uint16_t *k_src, const uint16_t *v_src,
              int32_t layer);

/* Gather: k_out[b][g][t][d] = K of token t of sequence b (and likewise V),
 * for t < seq_lens[b]; entries t >= seq_lens[b] are left untouched.
 * k_out / v_out are [batch][8][max_seq_len][64]. */
int pkvo_gather(const uint16_t *pool, int32_t num_pages,
                const int32_t *block_tables, int32_t num_layers, int32_t batch,
                int32_t max_blocks, const int32_t *seq_lens, int32_t layer,
                uint16_t *k_out, uint16_t *v_out, int32_t max_seq_len);

/* Decode: out[b][h][d] (double, [batch][32][64]) = softmax over t < L of
 * scale * q[b][h] . K[t][h/4], weighted sum of V[t][h/4].  Only the
 * sequences listed in rows[0..nrows) are computed (rows == NULL: all);
 * other rows of out are not touched.  nthreads > 1 splits the listed
 * sequences over that many POSIX threads (each sequence is computed by
 * exactly one thread, in the same order, so results do not depend on it). */
int pkvo_decode(const uint16_t *q, const uint16_t *pool, int32_t num_pages,
                const int32_t *block_tables, int32_t num_layers, int32_t batch,
                int32_t max_blocks, const int32_t *seq_lens, int32_t layer,
                double scale, double *out, const int32_t *rows, int32_t nrows,
                int32_t nthreads);

#ifdef __cplusplus
}
#endif

#endif /* PKV_ORACLE_H */
