/*
 * pkv.h -- C ABI of libpkv: paged KV-cache decode attention for B200 (sm_100a).
 *
 * The method (sources, by page title and section):
 *  - "Curso gratuito recorre la inferencia de LLM con videos, notas y un
 *    motor funcional en C++", section "¿Cómo administra el motor la memoria
 *    de la caché KV?": one shared pool of BF16 pages, each physical page
 *    holding the keys and values of 16 tokens, a block table per sequence
 *    and layer, and decode attention that reads each sequence's pages in
 *    place with an FP32 online softmax instead of gathering a contiguous
 *    prefix.
 *  - comrad404 article on samir-vllm ("Как устроен путь от текста запроса
 *    до следующего токена в языковой модели?"), section "Что README говорит
 *    о KV-кэше и пакетном декодировании": each decode step adds the new
 *    token's K/V to the cache.
 *  - "Construye tu propio motor de inferencia LLM de alto rendimiento en C++
 *    y CUDA", sections "La arquitectura del modelo: Llama 3.2 1B" (32 query
 *    heads, 8 kv heads, head dimension 64) and "Atención de Consulta
 *    Agrupada (GQA)" (query head h reads kv head h / 4).
 *
 * Conventions shared by every call:
 *  - Every call returns an int status (pkv_status).  No call aborts, exits
 *    or traps.  Host-visible argument errors are returned at once and
 *    nothing is launched.
 *  - Every device pointer is caller-owned device memory (for instance a
 *    torch tensor's data_ptr()).  The library keeps no pointer to it after
 *    the call returns.
 *  - Every kernel call is asynchronous on the given stream and allocates
 *    nothing.  A NULL stream is the legacy default stream.
 *  - Errors that only the device can see (a block-table entry outside the
 *    pool, a sequence length out of range, a timed-out wait) never fault:
 *    the kernel skips the offending work, leaves the result for that
 *    sequence unspecified, and records the first such error in a sticky
 *    word of the pool, read and cleared by pkv_get_device_error().
 *  - BF16 values are passed as their 16-bit patterns (uint16_t).
 *
 * Layouts (the pages fix none of them; these are this library's readings):
 *  - Pool page p (32768 bytes) = [kv in {K=0, V=1}][kv head g < 8]
 *    [slot s < 16][d < 64] BF16, so element (p, kv, g, s, d) sits at
 *    ((((p*2 + kv)*8 + g)*16 + s)*64 + d) * 2 bytes from the pool base.
 *    Token t of a sequence lives in slot t % 16 of logical page t / 16.
 *  - Block tables: int32 [num_layers][batch][max_blocks], row-major;
 *    entry [layer][b][j] is the physical page of logical page j of
 *    sequence b at that layer.  Entries past a sequence's last page are
 *    never read.
 *  - seq_lens: int32 [batch], the context length AFTER this step's append.
 *    The new token sits at position L-1; decode attends to 0..L-1.
 *  - q: BF16 [batch][32][64]; k_new, v_new: BF16 [batch][8][64];
 *    out: FP32 [batch][32][64].
 */
#ifndef PKV_H
#define PKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

#define PKV_PAGE_TOKENS 16
#define PKV_NUM_KV_HEADS 8
#define PKV_NUM_Q_HEADS 32
#define PKV_HEAD_DIM 64
#define PKV_PAGE_BYTES 32768

/* Same type as cudaStream_t. */
typedef struct CUstream_st *pkv_stream_t;

/* Opaque pool handle; owned by the caller between create and destroy. */
typedef struct pkv_pool pkv_pool;

typedef enum {
  PKV_OK = 0,
  PKV_ERR_INVALID_ARG = -1,    /* null pointer, negative size, layer out of range  */
  PKV_ERR_UNSUPPORTED = -2,    /* shape other than 16 tokens / 8 kv heads / d 64    */
  PKV_ERR_CUDA = -3,           /* a CUDA runtime call failed                        */
  PKV_ERR_OUT_OF_PAGES = -4,   /* page allocator: not enough free pages right now    */
  PKV_ERR_BAD_PAGE = -5,       /* device: block-table entry outside [0, num_pages)  */
  PKV_ERR_WORKSPACE = -6,      /* workspace missing, misaligned or too small        */
  PKV_ERR_DEVICE_TIMEOUT = -7, /* device: a bounded wait on a copy ran out           */
  PKV_ERR_BAD_SEQ_LEN = -8,    /* device: seq_len < 0 (append: < 1) or too long      */
  PKV_ERR_TOO_LARGE = -9,      /* larger than the no-alloc scratch / the whole pool */
  PKV_ERR_APPEND_CONFLICT = -10 /* device, with PKV_LAUNCH_CHECK_APPENDS: appends of
                                   one call race (see pkv_pool_set_launch_flags) */
} pkv_status;

/* Launch flags for pkv_pool_set_launch_flags. */
#define PKV_LAUNCH_PDL 1          /* programmatic dependent launch (see below) */
#define PKV_LAUNCH_EARLY_TABLES 2 /* with PDL: decode reads seq_lens and block
                                     tables before the preceding kernel ends */
#define PKV_LAUNCH_EARLY_PAGES 4  /* with PDL | EARLY_TABLES: decode also starts
                                     its first page loads before then */
#define PKV_LAUNCH_CHECK_APPENDS 8 /* check every append call for racing
                                     appends first (debugging aid, see below) */
#define PKV_LAUNCH_TEST_STALL (1 << 30) /* testing only: decode withholds one
                                     page so its bounded waits run out (~1 s)
                                     and it reports PKV_ERR_DEVICE_TIMEOUT */

/* Decode kernel variants for paged_attention_decode_ex. */
#define PKV_KERNEL_AUTO 0
#define PKV_KERNEL_SIMT 1 /* CUDA-core FP32 dot products, warp-shuffle reductions */
#define PKV_KERNEL_MMA 2  /* tensor-core (mma.sync BF16) QK and PV, FP32 softmax   */

/*
 * Create a pool of num_pages pages on the current CUDA device.
 * page_tokens, num_kv_heads and head_dim must be 16, 8 and 64 (else
 * PKV_ERR_UNSUPPORTED).  device_storage: caller-owned device memory of at
 * least num_pages * PKV_PAGE_BYTES bytes (storage_bytes), 16-byte aligned;
 * or NULL, in which case the library allocates (and later frees) it.  The
 * pool's contents are not initialised.  Also allocates a 4-byte device
 * error word.  The pages' engine sizes its pool with a command-line flag
 * (128 MiB by default), which is what num_pages expresses here.
 */
PKV_API int pkv_pool_create(int32_t num_pages, int32_t page_tokens, int32_t num_kv_heads,
                    int32_t head_dim, void *device_storage, size_t storage_bytes,
                    pkv_pool **out);

/* Free the pool handle and whatever the library allocated for it (not
 * caller-owned storage).  Synchronises the device. NULL is accepted. */
PKV_API int pkv_pool_destroy(pkv_pool *pool);

/* Device pointer to page 0 of the pool (layout above), or NULL. */
PKV_API void *pkv_pool_data(const pkv_pool *pool);

/* Number of pages, or -1 for a NULL pool. */
PKV_API int32_t pkv_pool_num_pages(const pkv_pool *pool);

/*
 * Launch options for every later pkv_append / paged_attention_decode call on
 * this pool.  PKV_LAUNCH_PDL launches the kernels with programmatic stream
 * serialisation: a kernel may be scheduled while the preceding kernel of the
 * stream is still running, and waits for it (griddepcontrol.wait) before it
 * reads or writes any memory, so results are the same as without the flag;
 * only launch latency is hidden.  Also valid under CUDA graph capture.
 * PKV_LAUNCH_EARLY_TABLES (only together with PKV_LAUNCH_PDL) lets decode
 * read seq_lens and the block tables -- never q, the pool or the outputs --
 * before the preceding kernels of the stream have finished, so its set-up
 * overlaps them.  Every kernel of this library lets the next launch start
 * early, so "preceding kernels" means every earlier kernel of the stream
 * that may still be running, not only the one launched just before (the
 * previous decode can still run beside its split-KV merge, for instance).
 * The caller guarantees that none of them writes seq_lens or the block
 * tables (an append or a decode, which only read them, is fine).
 * PKV_LAUNCH_EARLY_PAGES (only together with both) lets decode also start
 * loading the first pages of its range -- the KV of tokens already in the
 * cache -- before those kernels have finished, so their memory latency
 * overlaps them; q, the new token's rows and the outputs still wait.  These
 * early loads never touch a sequence's last two pages: that is where an
 * append or a fused append + decode of the same layer writes the newest
 * tokens (one per step, so the pages of the preceding 16 steps' tokens), so
 * chains of fused calls, or of pkv_append then decode, on one layer are
 * safe, repeated steps of a one-layer model included.  The caller
 * guarantees that no other pool page a decode reads is written by a kernel
 * that may still be running: true for the decodes and merges of other
 * layers and for a projection that writes q; false for a pkv_fill into this
 * layer's pages (its tokens can land in any page) or for a caller kernel
 * that writes pages, unless that kernel completes before decode starts
 * (launch decode without this flag after it).
 * PKV_LAUNCH_CHECK_APPENDS makes pkv_append, pkv_fill and the fused calls
 * (paged_attention_decode_append[_ex], pkv_decode with k_new) first launch a
 * check, on the same stream, that records PKV_ERR_APPEND_CONFLICT when the
 * call's result would be undefined: two sequences append to the same slot,
 * or (fused calls only) a sequence appends to a slot that lies inside a
 * context the call reads -- another sequence's, or its own through a page
 * its table names twice; for pkv_fill, two tokens (of two sequences, or of
 * one whose table names a page twice) are written to the same slot.  A
 * shared page whose slots are only read (a common prefix) is fine.
 * Sequences and tokens that the call itself skips as invalid are left to
 * its own errors.  The check only reports: the write still runs.  It costs
 * batch x (batch, or table entries when fused) comparisons, and for
 * pkv_fill a clear of a slot bitmap (2 bytes per page) plus one atomic per
 * token, so it is meant for debugging, not for the hot path.  Setting the
 * flag allocates that bitmap once (freed with the pool): the only device
 * allocation outside pool creation; PKV_ERR_CUDA if it fails.
 * PKV_LAUNCH_TEST_STALL exists only to test the device-timeout path: the
 * decode kernel never fills one shared-memory stage, every wait on it gives
 * up after about a second, the kernel exits early with garbage output and
 * pkv_get_device_error reports PKV_ERR_DEVICE_TIMEOUT; the context stays
 * usable.
 * flags: 0, PKV_LAUNCH_PDL, PKV_LAUNCH_PDL | PKV_LAUNCH_EARLY_TABLES or
 * PKV_LAUNCH_PDL | PKV_LAUNCH_EARLY_TABLES | PKV_LAUNCH_EARLY_PAGES,
 * each optionally | PKV_LAUNCH_CHECK_APPENDS and | PKV_LAUNCH_TEST_STALL,
 * else PKV_ERR_INVALID_ARG.
 */
PKV_API int pkv_pool_set_launch_flags(pkv_pool *pool, int32_t flags);

/*
 * Append (decode step, one token per sequence): for each b with
 * L = seq_lens[b], copy k_new[b][g][:] and v_new[b][g][:] for all 8 kv
 * heads into slot (L-1) % 16 of page block_tables[layer][b][(L-1)/16].
 * Bit copies.  seq_lens is not modified (the caller advances it).  Two
 * sequences appending into the same page slot is undefined (detected with
 * PKV_LAUNCH_CHECK_APPENDS).  Device errors:
 * L < 1 or L > max_blocks*16 -> PKV_ERR_BAD_SEQ_LEN, page outside the pool
 * -> PKV_ERR_BAD_PAGE; that sequence is skipped.
 */
PKV_API int pkv_append(pkv_pool *pool, const int32_t *block_tables, const int32_t *seq_lens,
               const uint16_t *k_new, const uint16_t *v_new, int32_t layer,
               int32_t num_layers, int32_t batch, int32_t max_blocks, pkv_stream_t stream);

/*
 * Fill (prefill, or chunked prefill): the counterpart of pkv_append for many
 * tokens; prefill is the step that fills a request's pages (comrad404 article
 * on samir-vllm, section "Что README говорит о KV-кэше и пакетном
 * декодировании").  Sequence b writes its tokens k_src/v_src[cu_tokens[b] +
 * i][g][:], i < cu_tokens[b+1] - cu_tokens[b], at positions start_pos[b] + i,
 * each in slot pos % 16 of page block_tables[layer][b][pos / 16].  Bit
 * copies.  k_src, v_src: dev BF16 [total_tokens][8][64], 16-byte aligned
 * (NULL allowed when total_tokens is 0); total_tokens: host int, the row
 * count of k_src and v_src, which sizes the grid (0 launches nothing);
 * cu_tokens: dev int32 [batch+1], from 0, non-decreasing, ending at
 * total_tokens; start_pos: dev int32 [batch].  Device errors
 * (PKV_ERR_BAD_SEQ_LEN): cu_tokens[0] != 0 or cu_tokens[batch] !=
 * total_tokens (nothing written), a decreasing entry (reported; which tokens
 * are written is then unspecified), a negative start or a position beyond
 * max_blocks*16 (that sequence is skipped).  A page outside the pool ->
 * PKV_ERR_BAD_PAGE (that token is skipped).  Whatever the device inputs, no
 * source row outside [0, total_tokens) is read and nothing outside the pool
 * is written.  The positions of different sequences must name different
 * slots (detected with PKV_LAUNCH_CHECK_APPENDS).  Stream ordered; PDL-chained like pkv_append when the pool's PDL
 * flag is set.  max_blocks * 16 must fit in int32.
 */
PKV_API int pkv_fill(pkv_pool *pool, const int32_t *block_tables, const int32_t *cu_tokens,
                     const int32_t *start_pos, const uint16_t *k_src, const uint16_t *v_src,
                     int32_t total_tokens, int32_t layer, int32_t num_layers, int32_t batch,
                     int32_t max_blocks, pkv_stream_t stream);

/*
 * Host page allocator (no GPU work; not thread-safe).  Hands out physical
 * page ids of a pool of num_pages pages from a LIFO free stack (page 0 first
 * on a fresh allocator), all or nothing:
 *  - pkv_allocator_alloc(count): PKV_ERR_TOO_LARGE if count exceeds the whole
 *    pool (such a request can never run: reject it), PKV_ERR_OUT_OF_PAGES if
 *    fewer than count pages are free now (queue the request, first in first
 *    out, and retry when pages are freed); nothing is taken on error.
 *  - pkv_allocator_free(pages, count): returns pages (for instance when a
 *    sequence ends); PKV_ERR_INVALID_ARG, and nothing freed, if a page is out
 *    of range, not allocated, or listed twice.
 */
typedef struct pkv_page_allocator pkv_page_allocator;
PKV_API int pkv_allocator_create(int32_t num_pages, pkv_page_allocator **out);
PKV_API int pkv_allocator_destroy(pkv_page_allocator *alloc);
PKV_API int32_t pkv_allocator_free_count(const pkv_page_allocator *alloc);
PKV_API int pkv_allocator_alloc(pkv_page_allocator *alloc, int32_t count, int32_t *pages_out);
PKV_API int pkv_allocator_free(pkv_page_allocator *alloc, const int32_t *pages, int32_t count);

/*
 * Workspace bytes paged_attention_decode needs for this batch on the pool's
 * device: the split-KV partial results (m, l and the unnormalised output of
 * every piece of a split sequence).  The workspace is caller-owned device
 * memory, 256-byte aligned; its contents need no initialisation (every
 * decode writes what it later reads).  Calls that share one workspace must
 * not overlap in time.
 */
PKV_API int pkv_decode_workspace_bytes(const pkv_pool *pool, int32_t batch, size_t *bytes_out);

/*
 * Decode attention of one new query token per sequence at one layer:
 *   out[b][h][:] = sum_{t<L} softmax_t(scale * q[b][h].K[t][h/4]) V[t][h/4]
 * with K/V read in place from the pages block_tables[layer][b][*], FP32
 * online softmax and FP32 accumulation.  Sequences with L == 0 get an
 * all-zero output.  Long contexts are split across the GPU (split-KV): the
 * decode kernel writes the pieces to the workspace and a second kernel,
 * launched right after it on the same stream, merges them with log-sum-exp
 * weights in a fixed order (results do not depend on timing); above 512
 * sequences the decode kernel also leaves the merge one split-table entry
 * per CTA, so the merge's set-up does not grow with the square of the
 * batch.  Device errors:
 * L < 0 or L > max_blocks*16 -> PKV_ERR_BAD_SEQ_LEN (that row is written as
 * zeros); a page outside the pool -> PKV_ERR_BAD_PAGE (that page is
 * skipped).  Requires 8 * batch * max_blocks < 2^31.  Every CTA keeps the
 * batch's lengths and page-count prefix in shared memory (8 bytes per
 * sequence): above about 4,000 sequences the tensor-core kernel runs one
 * CTA per SM instead of two, and above about 18,000 the call returns
 * PKV_ERR_UNSUPPORTED.
 */
PKV_API int paged_attention_decode(const uint16_t *q, const pkv_pool *pool, const int32_t *block_tables,
                           const int32_t *seq_lens, int32_t layer, float scale, float *out,
                           int32_t num_layers, int32_t batch, int32_t max_blocks,
                           void *workspace, size_t workspace_bytes, pkv_stream_t stream);

/*
 * As paged_attention_decode, with tuning/testing knobs:
 *   kernel:      PKV_KERNEL_AUTO / _SIMT / _MMA;
 *   grid_ctas:   0 = one persistent wave over the device; > 0 = exactly that
 *                many CTAs (the split of long contexts changes with it; the
 *                workspace needed is pkv_decode_workspace_bytes_ex's);
 *   min_chunk:   0 = automatic; > 0 = each CTA takes at least this many
 *                pages.
 */
PKV_API int paged_attention_decode_ex(const uint16_t *q, const pkv_pool *pool,
                              const int32_t *block_tables, const int32_t *seq_lens, int32_t layer,
                              float scale, float *out, int32_t num_layers, int32_t batch,
                              int32_t max_blocks, void *workspace, size_t workspace_bytes,
                              pkv_stream_t stream, int32_t kernel, int32_t grid_ctas,
                              int32_t min_chunk);

/*
 * Fused append + decode: exactly pkv_append(k_new, v_new) followed by
 * paged_attention_decode with the same seq_lens, in one launch (plus the
 * split-KV merge).  Decode adds the new token to the cache and attends to it
 * (comrad404 article on samir-vllm, section "Что README говорит о KV-кэше и
 * пакетном декодировании").  The CTA that reads sequence b's last page
 * writes the new token's rows into slot (L-1) % 16 of that page, both in
 * the pool and in its staged copy, so the page is read once and no append
 * launch is needed.  k_new, v_new: dev BF16 [batch][8][64], 16-byte aligned.
 * Differences from the two calls: a sequence with L = 0 gets no append and
 * a zero output row without an error (an idle batch slot); the appended
 * slot must not lie in another sequence's context in this call (a page that
 * several sequences read is read-only; detected with
 * PKV_LAUNCH_CHECK_APPENDS).  Errors and outputs otherwise as
 * pkv_append and paged_attention_decode; a page outside the pool is neither
 * read nor written.  Workspace: pkv_decode_workspace_bytes[_ex].
 */
PKV_API int paged_attention_decode_append(const uint16_t *q, const uint16_t *k_new,
                                          const uint16_t *v_new, pkv_pool *pool,
                                          const int32_t *block_tables, const int32_t *seq_lens,
                                          int32_t layer, float scale, float *out,
                                          int32_t num_layers, int32_t batch, int32_t max_blocks,
                                          void *workspace, size_t workspace_bytes,
                                          pkv_stream_t stream);

/* As paged_attention_decode_append, with the knobs of paged_attention_decode_ex. */
PKV_API int paged_attention_decode_append_ex(const uint16_t *q, const uint16_t *k_new,
                                             const uint16_t *v_new, pkv_pool *pool,
                                             const int32_t *block_tables, const int32_t *seq_lens,
                                             int32_t layer, float scale, float *out,
                                             int32_t num_layers, int32_t batch, int32_t max_blocks,
                                             void *workspace, size_t workspace_bytes,
                                             pkv_stream_t stream, int32_t kernel,
                                             int32_t grid_ctas, int32_t min_chunk);

/*
 * General decode call: every option of the calls above, plus two that they
 * lack, in one parameter block (future fields are appended; struct_size
 * tells the library which fields the caller knows).
 *
 *  - num_queries = T in 2..8: T queries per sequence, causal among them
 *    (the plainest multi-token decode, as in checking T - 1 drafted tokens):
 *    q and out are [batch][T][32][64]; query i of sequence b attends to
 *    tokens t < seq_lens[b] - T + 1 + i, so query T-1 sees the whole context
 *    and each earlier query one token fewer.  Needs seq_lens[b] = 0 or >= T
 *    (1..T-1 -> PKV_ERR_BAD_SEQ_LEN, zero rows), the tensor-core kernel
 *    (PKV_KERNEL_SIMT -> PKV_ERR_UNSUPPORTED) and no fused append (k_new must
 *    be NULL: write the T tokens with pkv_fill).
 *  - out_dtype = PKV_DTYPE_BF16: the output rows are BF16, rounded to
 *    nearest even from the FP32 result (the pages warn that BF16 rounding
 *    can differ with the batch size: "Curso gratuito recorre la inferencia
 *    de LLM...", the note on batch-dependent BF16 rounding).
 *
 * Fields: q (dev BF16 [batch][num_queries][32][64]); k_new, v_new (NULL, or
 * dev BF16 [batch][8][64]: fused append as paged_attention_decode_append);
 * block_tables, seq_lens, layer, num_layers, batch, max_blocks, scale as in
 * paged_attention_decode; out (dev [batch][num_queries][32][64] of
 * out_dtype, 16-byte aligned); workspace, workspace_bytes (see
 * pkv_decode_params_workspace_bytes); kernel, grid_ctas, min_chunk as in
 * paged_attention_decode_ex.  Errors as paged_attention_decode.
 */
#define PKV_DTYPE_F32 0
#define PKV_DTYPE_BF16 1

typedef struct pkv_decode_params {
  size_t struct_size; /* sizeof(pkv_decode_params) */
  const uint16_t *q;
  const uint16_t *k_new;
  const uint16_t *v_new;
  const int32_t *block_tables;
  const int32_t *seq_lens;
  void *out;
  void *workspace;
  size_t workspace_bytes;
  float scale;
  int32_t layer;
  int32_t num_layers;
  int32_t batch;
  int32_t max_blocks;
  int32_t num_queries; /* 1..8 */
  int32_t out_dtype;   /* PKV_DTYPE_F32 or PKV_DTYPE_BF16 */
  int32_t kernel;
  int32_t grid_ctas;
  int32_t min_chunk;
} pkv_decode_params;

PKV_API int pkv_decode(pkv_pool *pool, const pkv_decode_params *params, pkv_stream_t stream);

/* Workspace bytes pkv_decode needs for these parameters (only batch,
 * num_queries, kernel and grid_ctas are read). */
PKV_API int pkv_decode_params_workspace_bytes(const pkv_pool *pool,
                                              const pkv_decode_params *params,
                                              size_t *bytes_out);

/* Workspace bytes for paged_attention_decode_ex with these knobs. */
PKV_API int pkv_decode_workspace_bytes_ex(const pkv_pool *pool, int32_t batch, int32_t kernel,
                                  int32_t grid_ctas, size_t *bytes_out);

/*
 * Gather (page indexing made visible): k_out[b][g][t][:] and v_out[b][g][t][:]
 * = K and V of token t of sequence b at `layer`, for t < seq_lens[b]; rows
 * t >= seq_lens[b] are not written.  k_out, v_out: BF16 [batch][8]
 * [max_seq_len][64].  Device errors: L < 0, L > max_seq_len or
 * L > max_blocks*16 -> PKV_ERR_BAD_SEQ_LEN; page outside the pool ->
 * PKV_ERR_BAD_PAGE (those rows are not written).
 */
PKV_API int pkv_gather(const pkv_pool *pool, const int32_t *block_tables, const int32_t *seq_lens,
               int32_t layer, uint16_t *k_out, uint16_t *v_out, int32_t num_layers,
               int32_t batch, int32_t max_blocks, int32_t max_seq_len, pkv_stream_t stream);

/*
 * Allocation-free decode (the pages have no counterpart: this entry point
 * exists for callers that cannot allocate device memory where they run
 * attention -- code running inside an allocator or memory-pool callback,
 * runtime plugins that receive only their inputs and outputs, or loops that
 * must never call cudaMalloc/cudaFree because those calls synchronise the
 * device).  Same computation, arguments and device-error behaviour as
 * paged_attention_decode, but instead of a caller workspace it uses a
 * scratch area of PKV_NOALLOC_SCRATCH_BYTES that the library keeps in every
 * GPU's memory from load until process exit.  It allocates nothing.
 *  - Limit: returns PKV_ERR_TOO_LARGE (nothing launched) when the batch
 *    needs more scratch than that, i.e. when pkv_decode_workspace_bytes for
 *    this pool and batch (the exact check) exceeds it.  That size is
 *    (batch + grid) * 8 * 1056 + grid * 8 bytes, grid being the decode
 *    kernel's CTAs (SM count x CTAs per SM: 296 on a B200 while the batch is
 *    small enough for two CTAs per SM), so a B200 takes up to 1,689
 *    sequences.
 *  - The first call on a device looks up the scratch's device address
 *    (cudaGetSymbolAddress, with the pool's device current; nothing is
 *    allocated) and keeps it for the life of the process; make that first
 *    call before any stream capture.  A reset of the device's context
 *    (cudaDeviceReset, or the primary context torn down) invalidates the
 *    kept address: do not call this entry point on that device afterwards.
 *  - All calls on one device share the one scratch area, which keeps the
 *    last call's contents; nothing in it has to start at zero.  Calls whose
 *    kernels overlap on the GPU (different streams, or different threads
 *    without ordering) race on it and give wrong results: serialise them.
 */
#define PKV_NOALLOC_SCRATCH_BYTES (16u << 20)
PKV_API int paged_attention_decode_noalloc(const uint16_t *q, const pkv_pool *pool,
                                           const int32_t *block_tables, const int32_t *seq_lens,
                                           int32_t layer, float scale, float *out,
                                           int32_t num_layers, int32_t batch, int32_t max_blocks,
                                           pkv_stream_t stream);

/* Synchronise `stream`, return in *status_out the first device error
 * recorded since the last call (PKV_OK if none) and clear it. */
PKV_API int pkv_get_device_error(pkv_pool *pool, pkv_stream_t stream, int32_t *status_out);

/* Static English text for a status code. */
PKV_API const char *pkv_status_string(int status);

/* Text naming the CUDA call behind the calling thread's most recent
 * PKV_ERR_CUDA ("" if none); valid until the thread's next failing call. */
PKV_API const char *pkv_last_error_message(void);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H */
