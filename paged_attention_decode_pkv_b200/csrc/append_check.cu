// append_check.cu -- opt-in device check for appends whose result the API
// leaves undefined (PKV_LAUNCH_CHECK_APPENDS).
//
// An append writes one slot: position L_b - 1 of sequence b, which is slot
// (L_b - 1) % 16 of the page its block table names for logical page
// (L_b - 1) / 16 ("Curso gratuito recorre la inferencia de LLM...", section on
// the KV cache).  Two sequences naming the same slot race.  The fused
// append + decode also reads every page of every context while it appends,
// so an appended slot that lies inside some context of the same call -- a
// page shared read-only, such as a reused prompt prefix (the mascipolletti
// article on André Gray's Deeply vLLM, section "Cómo funciona", lists KV-cache
// management with prefix reuse) -- races with that read.
//
// Every thread takes block-table entries (c, j) and compares each with all
// appended slots of the call, staged in shared memory a chunk at a time:
//  - plain append: only c's own append page (j = (L_c - 1) / 16) is taken,
//    and another sequence appending to the same page and slot conflicts;
//  - fused: every j < ceil(L_c / 16) is taken, and a sequence appending to
//    that page at a slot s with 16 j + s < L_c conflicts (the same sequence
//    too, when its table names the page at another logical index).  A
//    shared slot is the case s = (L_c - 1) % 16 of it.
// Sequences whose own append is invalid (length or page out of range) are
// skipped; the append itself reports them.  The cost is entries x batch
// comparisons: a debugging aid, not a hot-path step.
//
// pkv_fill writes many tokens per sequence, so its check marks the written
// slots in a bitmap of the pool (one bit per slot, two bytes per page)
// instead of comparing pairs.
#include "append_check.cuh"
#include "fill_map.cuh"
#include "pkv_internal.cuh"

namespace pkv {

namespace {

constexpr int kCheckThreads = 256;
constexpr int kCheckChunk = 2048;        // appended slots staged per pass
constexpr int kCheckMaxCtas = 148 * 8;
constexpr int32_t kErrAppendConflict = PKV_ERR_APPEND_CONFLICT;

// The slot sequence b appends to, or false when its append is invalid.
__device__ __forceinline__ bool append_slot(const int32_t* __restrict__ bt,
                                            const int32_t* __restrict__ seq_lens, int32_t b,
                                            int32_t max_blocks, int32_t num_pages,
                                            int32_t* page, int32_t* slot) {
  const int32_t L = seq_lens[b];
  if (L < 1 || static_cast<int64_t>(L) > static_cast<int64_t>(max_blocks) * kTokens) return false;
  const int32_t p = bt[static_cast<int64_t>(b) * max_blocks + (L - 1) / kTokens];
  if (p < 0 || p >= num_pages) return false;
  *page = p;
  *slot = (L - 1) % kTokens;
  return true;
}

__global__ void __launch_bounds__(kCheckThreads)
    append_check_kernel(const int32_t* __restrict__ bt, const int32_t* __restrict__ seq_lens,
                        int32_t* __restrict__ err, int32_t batch, int32_t max_blocks,
                        int32_t num_pages, int32_t fused) {
  __shared__ int32_t s_page[kCheckChunk];   // -1: no valid append
  __shared__ int32_t s_slot[kCheckChunk];
  const int64_t entries =
      fused ? static_cast<int64_t>(batch) * max_blocks : static_cast<int64_t>(batch);
  bool conflict = false;
  for (int32_t b0 = 0; b0 < batch; b0 += kCheckChunk) {
    const int32_t n = min(kCheckChunk, batch - b0);
    __syncthreads();   // the previous chunk is no longer read
    for (int32_t i = threadIdx.x; i < n; i += blockDim.x) {
      int32_t page = -1, slot = 0;
      append_slot(bt, seq_lens, b0 + i, max_blocks, num_pages, &page, &slot);
      s_page[i] = page;
      s_slot[i] = slot;
    }
    __syncthreads();
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < entries;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
      const int32_t c = fused ? static_cast<int32_t>(e / max_blocks) : static_cast<int32_t>(e);
      const int32_t Lc = seq_lens[c];
      if (Lc < 1 || static_cast<int64_t>(Lc) > static_cast<int64_t>(max_blocks) * kTokens)
        continue;
      const int32_t jlast = (Lc - 1) / kTokens;
      const int32_t j = fused ? static_cast<int32_t>(e % max_blocks) : jlast;
      if (j > jlast) continue;
      const int32_t page = bt[static_cast<int64_t>(c) * max_blocks + j];
      if (page < 0 || page >= num_pages) continue;
      const int32_t read_end = min(kTokens, Lc - j * kTokens);   // slots [0, read_end) are read
      const int32_t own = (Lc - 1) % kTokens;
      for (int32_t i = 0; i < n; ++i) {
        if (s_page[i] != page) continue;
        const int32_t b = b0 + i;
        if (fused) {
          if ((b != c || j != jlast) && s_slot[i] < read_end) conflict = true;
        } else {
          if (b != c && s_slot[i] == own) conflict = true;
        }
      }
    }
  }
  if (conflict) record_error(err, kErrAppendConflict);
}

// Fill: every valid source row t marks bit (page * 16 + slot) of `bits`
// (zeroed before the launch); a bit that was already set means two rows --
// of two sequences, or of one whose table names a page twice -- write one
// slot.  Rows are mapped exactly as pkv_fill maps them, and rows that
// pkv_fill skips (bad range, page outside the pool) mark nothing.
__global__ void __launch_bounds__(kCheckThreads)
    fill_check_kernel(const int32_t* __restrict__ bt, const int32_t* __restrict__ cu,
                      const int32_t* __restrict__ start, uint32_t* __restrict__ bits,
                      int32_t* __restrict__ err, int32_t batch, int32_t max_blocks,
                      int32_t num_pages, int32_t total) {
  if (cu[0] != 0 || cu[batch] != total) return;   // pkv_fill writes nothing
  bool conflict = false;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int32_t t = static_cast<int32_t>(e);
    const int32_t b = fill_seq_of(cu, batch, t);
    const int32_t c0 = cu[b], c1 = cu[b + 1], s0 = start[b];
    if (t < c0 || t >= c1 || s0 < 0 ||
        static_cast<int64_t>(s0) + (c1 - c0) > static_cast<int64_t>(max_blocks) * kTokens)
      continue;
    const int32_t pos = s0 + (t - c0);
    const int32_t page = bt[static_cast<int64_t>(b) * max_blocks + pos / kTokens];
    if (page < 0 || page >= num_pages) continue;
    const int64_t idx = static_cast<int64_t>(page) * kTokens + pos % kTokens;
    const uint32_t bit = 1u << (idx & 31);
    if (atomicOr(bits + (idx >> 5), bit) & bit) conflict = true;
  }
  if (conflict) record_error(err, kErrAppendConflict);
}

}  // namespace

size_t fill_check_bitmap_bytes(int32_t num_pages) {
  return (static_cast<size_t>(num_pages) * kTokens + 31) / 32 * sizeof(uint32_t);
}

cudaError_t launch_fill_check(const int32_t* bt, const int32_t* cu, const int32_t* start,
                              uint32_t* bits, int32_t* err, int32_t batch, int32_t max_blocks,
                              int32_t num_pages, int32_t total_tokens, cudaStream_t stream) {
  if (batch == 0 || total_tokens == 0) return cudaSuccess;
  cudaError_t e = cudaMemsetAsync(bits, 0, fill_check_bitmap_bytes(num_pages), stream);
  if (e != cudaSuccess) return e;
  const int64_t want = (static_cast<int64_t>(total_tokens) + kCheckThreads - 1) / kCheckThreads;
  const int grid = static_cast<int>(want < kCheckMaxCtas ? want : kCheckMaxCtas);
  fill_check_kernel<<<grid, kCheckThreads, 0, stream>>>(bt, cu, start, bits, err, batch,
                                                        max_blocks, num_pages, total_tokens);
  return cudaGetLastError();
}

cudaError_t launch_append_check(const int32_t* bt, const int32_t* seq_lens, int32_t* err,
                                int32_t batch, int32_t max_blocks, int32_t num_pages,
                                bool fused, cudaStream_t stream) {
  if (batch == 0) return cudaSuccess;
  const int64_t entries =
      fused ? static_cast<int64_t>(batch) * max_blocks : static_cast<int64_t>(batch);
  const int64_t want = (entries + kCheckThreads - 1) / kCheckThreads;
  const int grid = static_cast<int>(want < kCheckMaxCtas ? (want > 0 ? want : 1) : kCheckMaxCtas);
  append_check_kernel<<<grid, kCheckThreads, 0, stream>>>(bt, seq_lens, err, batch, max_blocks,
                                                          num_pages, fused ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace pkv
