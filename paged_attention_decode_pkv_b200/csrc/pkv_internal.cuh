// pkv_internal.cuh -- shared definitions of the sm_100a kernels behind pkv.h.
//
// Shapes: 16-token pages ("Curso gratuito recorre la inferencia de LLM...",
// section on the KV cache), 32 query heads over 8 kv heads of dimension 64
// ("Construye tu propio motor de inferencia LLM...", sections on the
// Llama 3.2 1B architecture and on GQA).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pkv.h"

namespace pkv {

constexpr int kTokens = 16;                       // tokens per page
constexpr int kKvHeads = 8;
constexpr int kQHeads = 32;
constexpr int kDim = 64;
constexpr int kGroup = kQHeads / kKvHeads;        // 4 query heads per kv head
constexpr int kRowBytes = kDim * 2;               // one token of one kv head: 128 B
constexpr int kTileBytes = kTokens * kRowBytes;   // (page, K|V, kv head) tile: 2 KiB
constexpr int kRowsPerPage = 2 * kKvHeads * kTokens;  // 256 rows of 128 B
constexpr int kPartialFloats = 2 * kGroup + kGroup * kDim;  // m[4], l[4], acc[4][64]
constexpr int kMaxQueries = 8;   // queries per sequence in one decode launch

// Sticky device error codes (first one wins).
constexpr int32_t kErrBadPage = PKV_ERR_BAD_PAGE;
constexpr int32_t kErrBadLen = PKV_ERR_BAD_SEQ_LEN;
constexpr int32_t kErrTimeout = PKV_ERR_DEVICE_TIMEOUT;

// Bounded waits give up after this many nanoseconds of global time.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ void record_error(int32_t* err, int32_t code) {
  atomicCAS(err, 0, code);
}

// ------------------------------------------------------------ PTX wrappers --

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for phase `parity` of an mbarrier; false once kWaitLimitNs have
// passed without completion (the caller records kErrTimeout).
static __device__ __noinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
}

// L2 policy for data read exactly once (the KV stream).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 2-D tiled TMA load (no multicast) of box {64 elements, 16 rows} at
// coordinates (x, y) into shared memory, completing on mbarrier `bar`.
__device__ __forceinline__ void tma_load_tile(uint32_t dst, const CUtensorMap* map, int32_t x,
                                              int32_t y, uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}

// L2 prefetch of `bytes` (multiple of 16, 16-byte aligned) of global memory.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)),
               "r"(bytes)
               : "memory");
}

// 1-D bulk copy (no multicast) of `bytes` (multiple of 16, both addresses
// 16-byte aligned) from global to shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Four 8x8 b16 matrices from shared memory; lane i gives the address of row
// i % 8 of matrix i / 8.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D += A (16x16, row) * B (16x8, col); BF16 inputs, FP32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two floats -> BF16 pair (round to nearest even); `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (TMA / bulk copy) accesses to shared memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Byte offset of 16-byte chunk `c` of row `r` inside a TMA tile written with
// the 128-byte swizzle (rows of 128 B; chunk index XOR row % 8).
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return static_cast<uint32_t>(r * kRowBytes + ((c ^ (r & 7)) << 4));
}

// BF16 pair (one 32-bit word, element 0 in the low half) -> two floats.
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// ------------------------------------------------------------ launch glue --

// Work-partition cost of one sequence, in pages, on top of its pages (the
// per-sequence fixed work: query load, softmax finalisation, output).
constexpr int kSeqCost = 1;

// Launch flags (pool-wide).
constexpr int kLaunchPdl = 1;         // programmatic dependent launch
constexpr int kLaunchEarlyTables = 2; // read seq_lens / block tables before waiting
constexpr int kLaunchEarlyPages = PKV_LAUNCH_EARLY_PAGES;  // + first page loads too
constexpr int kLaunchTestStall = PKV_LAUNCH_TEST_STALL;  // testing the timeout path only

struct DecodeArgs {
  const __nv_bfloat16* q;   // [B][32][64]
  const int32_t* bt;        // this layer's block-table slab [B][max_blocks]
  const int32_t* seq_lens;  // [B]
  void* out;                // [B][num_queries][32][64], FP32 or BF16 (out_bf16)
  float* partials;          // [8 kv heads][B + grid][num_queries][kPartialFloats]
  int2* split_table;        // [grid]: (sequence, pieces) of the split sequence whose first
                            // piece each decode CTA holds, or (-1, 0); large batches only
  int32_t* err;             // sticky device error word
  int32_t batch;
  int32_t max_blocks;
  int32_t num_pages;
  int32_t min_chunk;        // minimum pages per CTA range
  float scale_log2;         // scale * log2(e)
  int32_t flags;            // kLaunch* bits
  int32_t num_queries;      // queries per sequence (1 or kMaxQueries), causal among them
  int32_t out_bf16;         // nonzero: out is BF16
  // Fused append (paged_attention_decode_append): the new token's K/V rows
  // [B][8][64] and the page storage they are written into; null otherwise.
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  __nv_bfloat16* pool;
};

// Batches up to this size: each merge CTA finds its split from the lengths
// before its dependency wait (B loads, overlapping decode).  Larger ones:
// decode publishes one split-table entry per CTA and the merge grid has one
// CTA per (kv head, decode CTA), each reading its entry after the wait, so
// the merge set-up no longer grows with the square of the batch.
constexpr int kMergeScanMaxBatch = 512;

// Launch planning shared by the workspace query and the launch.
struct DecodePlan {
  int kernel;        // PKV_KERNEL_SIMT or PKV_KERNEL_MMA
  int num_queries;   // queries per sequence (picks the kernel variant)
  int grid;          // CTAs
  int threads;       // threads per CTA
  size_t smem;       // dynamic shared memory bytes
  size_t records_bytes;  // workspace bytes of the partial records (at its start)
  size_t ws_bytes;   // workspace bytes: the records, then the split table [grid] int2
  int merge_chunk;   // pieces the merge kernel stages in shared memory per round
  size_t merge_smem;  // its dynamic shared memory bytes
};

int plan_decode(int device, int sm_count, int32_t batch, int kernel, int grid_ctas,
                int num_queries, DecodePlan* plan);
cudaError_t launch_decode(const DecodePlan& plan, const CUtensorMap& tmap, const DecodeArgs& a,
                          int flags, cudaStream_t stream);
cudaError_t prepare_decode_kernels(int device);

cudaError_t launch_append(const __nv_bfloat16* k_new, const __nv_bfloat16* v_new,
                          __nv_bfloat16* pool, const int32_t* bt, const int32_t* seq_lens,
                          int32_t* err, int32_t batch, int32_t max_blocks, int32_t num_pages,
                          int flags, cudaStream_t stream);

cudaError_t launch_fill(const __nv_bfloat16* k_src, const __nv_bfloat16* v_src,
                        __nv_bfloat16* pool, const int32_t* bt, const int32_t* cu,
                        const int32_t* start, int32_t* err, int32_t batch, int32_t max_blocks,
                        int32_t num_pages, int32_t total_tokens, int flags,
                        cudaStream_t stream);

cudaError_t launch_gather(const __nv_bfloat16* pool, const int32_t* bt, const int32_t* seq_lens,
                          __nv_bfloat16* k_out, __nv_bfloat16* v_out, int32_t* err,
                          int32_t batch, int32_t max_blocks, int32_t num_pages,
                          int32_t max_seq_len, cudaStream_t stream);

// Programmatic dependent launch: wait for the preceding kernel of the stream
// (no-op when the launch has no programmatic dependency), and allow the next
// kernel to start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace pkv
