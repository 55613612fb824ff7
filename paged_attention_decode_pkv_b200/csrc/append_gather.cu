// append_gather.cu -- KV-append scatter and block-table page gather.
//
// Append: each decode step adds the new token's K/V to the cache (comrad404
// article on samir-vllm, section "Что README говорит о KV-кэше и пакетном
// декодировании"); the token goes to slot (L-1) % 16 of the page that the
// sequence's block table names for logical page (L-1) / 16 ("Curso gratuito
// recorre la inferencia de LLM...", section on the KV cache).
//
// Gather: the same block-table walk, copying a sequence's tokens out into a
// contiguous [8][max_seq_len][64] layout.  Decode never does this (it reads
// pages in place); the gather exists so that page indexing can be checked
// bit for bit.
//
// Fill: the prefill counterpart of append -- prefill writes a request's
// prompt tokens into its pages (same comrad404 section) -- a ragged batch of
// tokens per sequence, written at consecutive positions from start_pos[b].
//
// All three are pure 16-byte copies: 8 consecutive threads move one 128-byte row
// (one token of one kv head), so every warp access is four full 128-byte
// lines.
#include "fill_map.cuh"
#include "pkv_internal.cuh"

namespace pkv {

// One CTA per sequence, 128 threads = (K|V) x 8 kv heads x 8 chunks of 16 B.
__global__ void __launch_bounds__(128) append_kernel(const uint4* __restrict__ k_new,
                                                     const uint4* __restrict__ v_new,
                                                     uint4* __restrict__ pool,
                                                     const int32_t* __restrict__ bt,
                                                     const int32_t* __restrict__ seq_lens,
                                                     int32_t* __restrict__ err, int32_t max_blocks,
                                                     int32_t num_pages) {
  pdl_wait();   // the pool may be in use by the preceding kernel
  pdl_trigger();
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  const int kv = tid >> 6;
  const int g = (tid >> 3) & 7;
  const int c = tid & 7;
  const int32_t L = seq_lens[b];
  if (L < 1 || static_cast<int64_t>(L) > static_cast<int64_t>(max_blocks) * kTokens) {
    if (tid == 0) record_error(err, kErrBadLen);
    return;
  }
  const int32_t pos = L - 1;
  const int32_t phys = bt[static_cast<int64_t>(b) * max_blocks + pos / kTokens];
  if (phys < 0 || phys >= num_pages) {
    if (tid == 0) record_error(err, kErrBadPage);
    return;
  }
  const int slot = pos % kTokens;
  // source: [B][8][64] BF16 = 8 chunks of 16 B per (b, g)
  const uint4* src = (kv ? v_new : k_new) + (static_cast<int64_t>(b) * kKvHeads + g) * 8 + c;
  // destination row (phys, kv, g, slot): 128 B = 8 chunks
  const int64_t row = (static_cast<int64_t>(phys) * 2 + kv) * (kKvHeads * kTokens) +
                      g * kTokens + slot;
  pool[row * 8 + c] = *src;
}

// Fill: one CTA per kFillRowsPerCta consecutive source rows t (rows
// [0, total) of k_src / v_src).  512 threads = 4 row lanes x (K|V) x 8 kv
// heads x 8 chunks of 16 B; each lane moves kFillRowsPerLane rows, and all
// their loads go out first: they depend on nothing but the row count.
// While they are in flight, one thread per row maps the row to its
// destination -- row t belongs to the last sequence b with cu[b] <= t,
// goes to position start[b] + t - cu[b], so to slot pos % 16 of page
// bt[b][pos / 16] -- and shares it through shared memory, so the index
// loads are issued once per row, not once per 16-byte chunk.  For batches
// of fewer than 512 sequences the CTA first copies cu and start into
// shared memory (one round of loads, beside the data loads) and searches
// there, so a row's destination costs two dependent rounds of memory
// latency (cu and start, then the block-table entry) instead of one per
// step of a binary search in global memory.  The grid follows the row
// count, not (sequence x longest prompt), so a batch of mixed prompt
// lengths launches no empty CTAs.
constexpr int kFillThreads = 512;
constexpr int kFillLanes = kFillThreads / 128;
constexpr int kFillRowsPerLane = 4;
constexpr int kFillRowsPerCta = kFillLanes * kFillRowsPerLane;
constexpr int kFillSmemBatch = kFillThreads - 1;   // largest batch searched in shared memory

__global__ void __launch_bounds__(kFillThreads)
    fill_kernel(const uint4* __restrict__ k_src, const uint4* __restrict__ v_src,
                uint4* __restrict__ pool, const int32_t* __restrict__ bt,
                const int32_t* __restrict__ cu, const int32_t* __restrict__ start,
                int32_t* __restrict__ err, int32_t batch, int32_t max_blocks,
                int32_t num_pages, int32_t total) {
  __shared__ int64_t s_row[kFillRowsPerCta];   // pool row of (page, K, head 0, slot), or -1
  __shared__ int32_t s_cu[kFillSmemBatch + 1];
  __shared__ int32_t s_start[kFillSmemBatch];
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x;
  const int kv = (tid >> 6) & 1;
  const int g = (tid >> 3) & 7;
  const int c = tid & 7;
  const int32_t row0 = blockIdx.x * kFillRowsPerCta;
  const uint4* src = kv ? v_src : k_src;
  uint4 val[kFillRowsPerLane];
#pragma unroll
  for (int j = 0; j < kFillRowsPerLane; ++j) {
    const int32_t t = row0 + (tid >> 7) + kFillLanes * j;
    if (t < total) val[j] = __ldcs(src + (static_cast<int64_t>(t) * kKvHeads + g) * 8 + c);
  }
  const bool staged = batch <= kFillSmemBatch;   // uniform over the grid
  if (staged) {
    for (int i = tid; i <= batch; i += kFillThreads) {
      s_cu[i] = cu[i];
      if (i < batch) s_start[i] = start[i];
    }
  }
  // a decreasing cu makes the row -> sequence map ambiguous: report it
  for (int32_t b = blockIdx.x * blockDim.x + tid; b < batch; b += gridDim.x * blockDim.x)
    if (cu[b + 1] < cu[b]) record_error(err, kErrBadLen);
  __syncthreads();
  const int32_t* cu_s = staged ? s_cu : cu;
  // the rows the caller passed must be exactly the rows cu describes
  if (cu_s[0] != 0 || cu_s[batch] != total) {   // uniform over the grid: nothing is written
    if (blockIdx.x == 0 && tid == 0) record_error(err, kErrBadLen);
    return;
  }
  if (tid < kFillRowsPerCta) {
    const int32_t t = row0 + tid;
    int64_t row = -1;
    if (t < total) {
      const int32_t b = fill_seq_of(cu_s, batch, t);
      const int32_t c0 = cu_s[b], c1 = cu_s[b + 1], s0 = staged ? s_start[b] : start[b];
      if (t < c0 || t >= c1 || s0 < 0 ||
          static_cast<int64_t>(s0) + (c1 - c0) > static_cast<int64_t>(max_blocks) * kTokens) {
        record_error(err, kErrBadLen);
      } else {
        const int32_t pos = s0 + (t - c0);
        const int32_t phys = bt[static_cast<int64_t>(b) * max_blocks + pos / kTokens];
        if (phys < 0 || phys >= num_pages)
          record_error(err, kErrBadPage);
        else
          row = static_cast<int64_t>(phys) * (2 * kKvHeads * kTokens) + pos % kTokens;
      }
    }
    s_row[tid] = row;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kFillRowsPerLane; ++j) {
    const int64_t row = s_row[(tid >> 7) + kFillLanes * j];
    if (row >= 0) pool[(row + (kv * kKvHeads + g) * kTokens) * 8 + c] = val[j];
  }
}

// grid (ceil(max_seq_len / 32), 8 kv heads, batch); 256 threads = 32 tokens
// x 8 chunks of 16 B; each thread copies one K chunk and one V chunk.
__global__ void __launch_bounds__(256) gather_kernel(const uint4* __restrict__ pool,
                                                     const int32_t* __restrict__ bt,
                                                     const int32_t* __restrict__ seq_lens,
                                                     uint4* __restrict__ k_out,
                                                     uint4* __restrict__ v_out,
                                                     int32_t* __restrict__ err, int32_t max_blocks,
                                                     int32_t num_pages, int32_t max_seq_len) {
  const int b = blockIdx.z;
  const int g = blockIdx.y;
  const int t = blockIdx.x * 32 + (threadIdx.x >> 3);
  const int c = threadIdx.x & 7;
  const int32_t L = seq_lens[b];
  if (L < 0 || L > max_seq_len ||
      static_cast<int64_t>(L) > static_cast<int64_t>(max_blocks) * kTokens) {
    if (blockIdx.x == 0 && g == 0 && threadIdx.x == 0) record_error(err, kErrBadLen);
    return;
  }
  if (t >= L) return;
  const int32_t phys = bt[static_cast<int64_t>(b) * max_blocks + t / kTokens];
  if (phys < 0 || phys >= num_pages) {
    if ((t % kTokens) == 0 && c == 0) record_error(err, kErrBadPage);
    return;
  }
  const int64_t krow = (static_cast<int64_t>(phys) * 2) * (kKvHeads * kTokens) + g * kTokens +
                       (t % kTokens);
  const int64_t vrow = krow + kKvHeads * kTokens;
  const int64_t orow = (static_cast<int64_t>(b) * kKvHeads + g) * max_seq_len + t;
  k_out[orow * 8 + c] = pool[krow * 8 + c];
  v_out[orow * 8 + c] = pool[vrow * 8 + c];
}

cudaError_t launch_append(const __nv_bfloat16* k_new, const __nv_bfloat16* v_new,
                          __nv_bfloat16* pool, const int32_t* bt, const int32_t* seq_lens,
                          int32_t* err, int32_t batch, int32_t max_blocks, int32_t num_pages,
                          int flags, cudaStream_t stream) {
  if (batch == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(batch);
  cfg.blockDim = dim3(128);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (flags & kLaunchPdl) ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, append_kernel, reinterpret_cast<const uint4*>(k_new),
                            reinterpret_cast<const uint4*>(v_new), reinterpret_cast<uint4*>(pool),
                            bt, seq_lens, err, max_blocks, num_pages);
}

cudaError_t launch_fill(const __nv_bfloat16* k_src, const __nv_bfloat16* v_src,
                        __nv_bfloat16* pool, const int32_t* bt, const int32_t* cu,
                        const int32_t* start, int32_t* err, int32_t batch, int32_t max_blocks,
                        int32_t num_pages, int32_t total_tokens, int flags, cudaStream_t stream) {
  if (batch == 0 || total_tokens == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((total_tokens + kFillRowsPerCta - 1) / kFillRowsPerCta);
  cfg.blockDim = dim3(kFillThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (flags & kLaunchPdl) ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, fill_kernel, reinterpret_cast<const uint4*>(k_src),
                            reinterpret_cast<const uint4*>(v_src), reinterpret_cast<uint4*>(pool),
                            bt, cu, start, err, batch, max_blocks, num_pages, total_tokens);
}

cudaError_t launch_gather(const __nv_bfloat16* pool, const int32_t* bt, const int32_t* seq_lens,
                          __nv_bfloat16* k_out, __nv_bfloat16* v_out, int32_t* err,
                          int32_t batch, int32_t max_blocks, int32_t num_pages,
                          int32_t max_seq_len, cudaStream_t stream) {
  if (batch == 0 || max_seq_len == 0) return cudaSuccess;
  dim3 grid((max_seq_len + 31) / 32, kKvHeads, batch);
  gather_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(pool), bt, seq_lens,
                                          reinterpret_cast<uint4*>(k_out),
                                          reinterpret_cast<uint4*>(v_out), err, max_blocks,
                                          num_pages, max_seq_len);
  return cudaGetLastError();
}

}  // namespace pkv
