// pkv_api.cu -- the C ABI of pkv.h: argument checks, pool handles, launches.
//
// Host-visible argument errors are caught here before anything is launched;
// everything else is the kernels' business (see pkv.h for the contract).
#include <cstdio>
#include <mutex>
#include <new>

#include "append_check.cuh"
#include "pkv_internal.cuh"

struct pkv_pool {
  void* data;
  bool owns_data;
  int32_t num_pages;
  int device;
  int sm_count;
  int32_t* d_err;
  int launch_flags;  // PKV_LAUNCH_* bits applied to this pool's kernel launches
  uint32_t* d_slot_bits;  // pkv_fill's race check: one bit per slot, allocated with the flag
  CUtensorMap tmap;  // 2-D view of the pool: rows of 64 BF16, one 256-row box per page
};

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The pool's device must be current for calls that launch on it.
int check_device(const pkv_pool* pool) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ERR_CUDA;
  return dev == pool->device ? PKV_OK : PKV_ERR_INVALID_ARG;
}

int check_table_args(const pkv_pool* pool, const int32_t* bt, const int32_t* seq_lens,
                     int32_t layer, int32_t num_layers, int32_t batch, int32_t max_blocks) {
  if (!pool || !bt || !seq_lens) return PKV_ERR_INVALID_ARG;
  if (batch < 0 || max_blocks < 1 || num_layers < 1) return PKV_ERR_INVALID_ARG;
  if (layer < 0 || layer >= num_layers) return PKV_ERR_INVALID_ARG;
  if (static_cast<int64_t>(batch) * max_blocks * pkv::kKvHeads >= (int64_t(1) << 31))
    return PKV_ERR_UNSUPPORTED;
  return check_device(pool);
}

const int32_t* layer_slab(const int32_t* bt, int32_t layer, int32_t batch, int32_t max_blocks) {
  return bt + static_cast<int64_t>(layer) * batch * max_blocks;
}

thread_local char g_last_error[256] = "";

void note(const char* where, cudaError_t e) {
  snprintf(g_last_error, sizeof g_last_error, "%s: %s", where, cudaGetErrorString(e));
}

int from_cuda(cudaError_t e, const char* where = "kernel launch") {
  if (e == cudaSuccess) return PKV_OK;
  note(where, e);
  return PKV_ERR_CUDA;
}

}  // namespace

extern "C" {

int pkv_pool_create(int32_t num_pages, int32_t page_tokens, int32_t num_kv_heads,
                    int32_t head_dim, void* device_storage, size_t storage_bytes,
                    pkv_pool** out) {
  if (!out) return PKV_ERR_INVALID_ARG;
  *out = nullptr;
  if (page_tokens != PKV_PAGE_TOKENS || num_kv_heads != PKV_NUM_KV_HEADS ||
      head_dim != PKV_HEAD_DIM)
    return PKV_ERR_UNSUPPORTED;
  if (num_pages < 1) return PKV_ERR_INVALID_ARG;
  // TMA row coordinates (page * 256 + ...) must stay below 2^31.
  if (static_cast<int64_t>(num_pages) * pkv::kRowsPerPage >= (int64_t(1) << 31))
    return PKV_ERR_UNSUPPORTED;
  const size_t need = static_cast<size_t>(num_pages) * PKV_PAGE_BYTES;
  if (device_storage && (storage_bytes < need || !aligned(device_storage, 16)))
    return PKV_ERR_INVALID_ARG;
  EncodeTiledFn encode = encode_tiled_fn();
  if (!encode) {
    snprintf(g_last_error, sizeof g_last_error, "pkv_pool_create: cuTensorMapEncodeTiled not found");
    return PKV_ERR_CUDA;
  }

  pkv_pool* p = new (std::nothrow) pkv_pool();
  if (!p) return PKV_ERR_INVALID_ARG;
  p->num_pages = num_pages;
  p->launch_flags = 0;
  cudaError_t e = cudaGetDevice(&p->device);
  if (e == cudaSuccess)
    e = cudaDeviceGetAttribute(&p->sm_count, cudaDevAttrMultiProcessorCount, p->device);
  if (e != cudaSuccess) {
    delete p;
    return from_cuda(e, "pkv_pool_create: device query");
  }
  e = pkv::prepare_decode_kernels(p->device);
  if (e != cudaSuccess) {
    delete p;
    return from_cuda(e, "pkv_pool_create: kernel attributes");
  }
  if (device_storage) {
    p->data = device_storage;
    p->owns_data = false;
  } else {
    e = cudaMalloc(&p->data, need);
    if (e != cudaSuccess) {
      delete p;
      return from_cuda(e, "pkv_pool_create: cudaMalloc(pool)");
    }
    p->owns_data = true;
  }
  e = cudaMalloc(&p->d_err, sizeof(int32_t));
  if (e == cudaSuccess) e = cudaMemset(p->d_err, 0, sizeof(int32_t));
  if (e != cudaSuccess) {
    if (p->owns_data) cudaFree(p->data);
    delete p;
    return from_cuda(e, "pkv_pool_create: error word");
  }
  const cuuint64_t dims[2] = {PKV_HEAD_DIM,
                              static_cast<cuuint64_t>(num_pages) * pkv::kRowsPerPage};
  const cuuint64_t strides[1] = {pkv::kRowBytes};
  const cuuint32_t box[2] = {PKV_HEAD_DIM, pkv::kRowsPerPage};
  const cuuint32_t elem_strides[2] = {1, 1};
  CUresult r = encode(&p->tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p->data, dims, strides, box,
                      elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_last_error, sizeof g_last_error, "pkv_pool_create: cuTensorMapEncodeTiled: CUresult %d",
             static_cast<int>(r));
    cudaFree(p->d_err);
    if (p->owns_data) cudaFree(p->data);
    delete p;
    return PKV_ERR_CUDA;
  }
  *out = p;
  return PKV_OK;
}

int pkv_pool_destroy(pkv_pool* pool) {
  if (!pool) return PKV_OK;
  int prev = -1;
  cudaGetDevice(&prev);
  cudaSetDevice(pool->device);
  cudaError_t e = cudaDeviceSynchronize();
  cudaFree(pool->d_err);
  cudaFree(pool->d_slot_bits);
  if (pool->owns_data) cudaFree(pool->data);
  if (prev >= 0) cudaSetDevice(prev);
  delete pool;
  return from_cuda(e);
}

void* pkv_pool_data(const pkv_pool* pool) { return pool ? pool->data : nullptr; }

int32_t pkv_pool_num_pages(const pkv_pool* pool) { return pool ? pool->num_pages : -1; }

int pkv_append(pkv_pool* pool, const int32_t* block_tables, const int32_t* seq_lens,
               const uint16_t* k_new, const uint16_t* v_new, int32_t layer, int32_t num_layers,
               int32_t batch, int32_t max_blocks, pkv_stream_t stream) {
  int s = check_table_args(pool, block_tables, seq_lens, layer, num_layers, batch, max_blocks);
  if (s != PKV_OK) return s;
  if (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16)) return PKV_ERR_INVALID_ARG;
  if (batch > 2147483647 / 2) return PKV_ERR_UNSUPPORTED;
  if (pool->launch_flags & PKV_LAUNCH_CHECK_APPENDS) {
    s = from_cuda(pkv::launch_append_check(layer_slab(block_tables, layer, batch, max_blocks),
                                           seq_lens, pool->d_err, batch, max_blocks,
                                           pool->num_pages, false,
                                           reinterpret_cast<cudaStream_t>(stream)));
    if (s != PKV_OK) return s;
  }
  return from_cuda(pkv::launch_append(
      reinterpret_cast<const __nv_bfloat16*>(k_new), reinterpret_cast<const __nv_bfloat16*>(v_new),
      static_cast<__nv_bfloat16*>(pool->data), layer_slab(block_tables, layer, batch, max_blocks),
      seq_lens, pool->d_err, batch, max_blocks, pool->num_pages, pool->launch_flags,
      reinterpret_cast<cudaStream_t>(stream)));
}

int pkv_fill(pkv_pool* pool, const int32_t* block_tables, const int32_t* cu_tokens,
             const int32_t* start_pos, const uint16_t* k_src, const uint16_t* v_src,
             int32_t total_tokens, int32_t layer, int32_t num_layers, int32_t batch,
             int32_t max_blocks, pkv_stream_t stream) {
  int s = check_table_args(pool, block_tables, cu_tokens, layer, num_layers, batch, max_blocks);
  if (s != PKV_OK) return s;
  if (!start_pos || total_tokens < 0) return PKV_ERR_INVALID_ARG;
  // the sources may be NULL only when there is no row to read
  if (total_tokens > 0 && (!k_src || !v_src || !aligned(k_src, 16) || !aligned(v_src, 16)))
    return PKV_ERR_INVALID_ARG;
  // positions are int32 on the device
  if (static_cast<int64_t>(max_blocks) * pkv::kTokens > 2147483647) return PKV_ERR_UNSUPPORTED;
  if (pool->launch_flags & PKV_LAUNCH_CHECK_APPENDS) {
    s = from_cuda(pkv::launch_fill_check(layer_slab(block_tables, layer, batch, max_blocks),
                                         cu_tokens, start_pos, pool->d_slot_bits, pool->d_err,
                                         batch, max_blocks, pool->num_pages, total_tokens,
                                         reinterpret_cast<cudaStream_t>(stream)));
    if (s != PKV_OK) return s;
  }
  return from_cuda(pkv::launch_fill(
      reinterpret_cast<const __nv_bfloat16*>(k_src), reinterpret_cast<const __nv_bfloat16*>(v_src),
      static_cast<__nv_bfloat16*>(pool->data), layer_slab(block_tables, layer, batch, max_blocks),
      cu_tokens, start_pos, pool->d_err, batch, max_blocks, pool->num_pages, total_tokens,
      pool->launch_flags, reinterpret_cast<cudaStream_t>(stream)));
}

int pkv_pool_set_launch_flags(pkv_pool* pool, int32_t flags) {
  if (!pool || (flags & ~(PKV_LAUNCH_PDL | PKV_LAUNCH_EARLY_TABLES | PKV_LAUNCH_EARLY_PAGES |
                          PKV_LAUNCH_CHECK_APPENDS | PKV_LAUNCH_TEST_STALL)))
    return PKV_ERR_INVALID_ARG;
  if ((flags & PKV_LAUNCH_EARLY_TABLES) && !(flags & PKV_LAUNCH_PDL)) return PKV_ERR_INVALID_ARG;
  if ((flags & PKV_LAUNCH_EARLY_PAGES) && !(flags & PKV_LAUNCH_EARLY_TABLES))
    return PKV_ERR_INVALID_ARG;
  if ((flags & PKV_LAUNCH_CHECK_APPENDS) && !pool->d_slot_bits) {
    // pkv_fill's check needs a slot bitmap: allocated once, here, not in the calls
    int prev = -1;
    cudaGetDevice(&prev);
    cudaSetDevice(pool->device);
    void* bits = nullptr;
    const cudaError_t e = cudaMalloc(&bits, pkv::fill_check_bitmap_bytes(pool->num_pages));
    if (prev >= 0) cudaSetDevice(prev);
    if (e != cudaSuccess) return from_cuda(e, "pkv_pool_set_launch_flags: cudaMalloc(slot bitmap)");
    pool->d_slot_bits = static_cast<uint32_t*>(bits);
  }
  pool->launch_flags = flags;
  return PKV_OK;
}

int pkv_decode_workspace_bytes_ex(const pkv_pool* pool, int32_t batch, int32_t kernel,
                                  int32_t grid_ctas, size_t* bytes_out) {
  if (!pool || !bytes_out || batch < 0 || grid_ctas < 0) return PKV_ERR_INVALID_ARG;
  pkv::DecodePlan plan;
  int s = pkv::plan_decode(pool->device, pool->sm_count, batch, kernel, grid_ctas, 1, &plan);
  if (s != PKV_OK) return s;
  *bytes_out = plan.ws_bytes;
  return PKV_OK;
}

int pkv_decode_workspace_bytes(const pkv_pool* pool, int32_t batch, size_t* bytes_out) {
  return pkv_decode_workspace_bytes_ex(pool, batch, PKV_KERNEL_AUTO, 0, bytes_out);
}

}  // extern "C"

namespace {

// Decode, with the fused append when k_new / v_new are given.
int decode_common(const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                  const pkv_pool* pool, const int32_t* block_tables, const int32_t* seq_lens,
                  int32_t layer, float scale, void* out, int32_t out_dtype, int32_t num_queries,
                  int32_t num_layers, int32_t batch, int32_t max_blocks, void* workspace,
                  size_t workspace_bytes, pkv_stream_t stream, int32_t kernel, int32_t grid_ctas,
                  int32_t min_chunk) {
  int s = check_table_args(pool, block_tables, seq_lens, layer, num_layers, batch, max_blocks);
  if (s != PKV_OK) return s;
  if (!q || !out || !aligned(q, 16) || !aligned(out, 16)) return PKV_ERR_INVALID_ARG;
  if (!(scale == scale) || grid_ctas < 0 || min_chunk < 0) return PKV_ERR_INVALID_ARG;
  if (out_dtype != PKV_DTYPE_F32 && out_dtype != PKV_DTYPE_BF16) return PKV_ERR_INVALID_ARG;
  if ((k_new == nullptr) != (v_new == nullptr)) return PKV_ERR_INVALID_ARG;
  if (k_new && (!aligned(k_new, 16) || !aligned(v_new, 16))) return PKV_ERR_INVALID_ARG;
  if (k_new && num_queries != 1) return PKV_ERR_UNSUPPORTED;
  pkv::DecodePlan plan;
  s = pkv::plan_decode(pool->device, pool->sm_count, batch, kernel, grid_ctas, num_queries, &plan);
  if (s != PKV_OK) return s;
  if (batch == 0) return PKV_OK;
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < plan.ws_bytes)
    return PKV_ERR_WORKSPACE;
  pkv::DecodeArgs a;
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.bt = layer_slab(block_tables, layer, batch, max_blocks);
  a.seq_lens = seq_lens;
  a.out = out;
  a.partials = static_cast<float*>(workspace);
  a.split_table = reinterpret_cast<int2*>(static_cast<uint8_t*>(workspace) + plan.records_bytes);
  a.err = pool->d_err;
  a.batch = batch;
  a.max_blocks = max_blocks;
  a.num_pages = pool->num_pages;
  a.min_chunk = min_chunk;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.flags = pool->launch_flags;
  a.num_queries = num_queries;
  a.out_bf16 = out_dtype == PKV_DTYPE_BF16;
  a.k_new = reinterpret_cast<const __nv_bfloat16*>(k_new);
  a.v_new = reinterpret_cast<const __nv_bfloat16*>(v_new);
  a.pool = static_cast<__nv_bfloat16*>(pool->data);
  if (k_new && (pool->launch_flags & PKV_LAUNCH_CHECK_APPENDS)) {
    s = from_cuda(pkv::launch_append_check(a.bt, seq_lens, pool->d_err, batch, max_blocks,
                                           pool->num_pages, true,
                                           reinterpret_cast<cudaStream_t>(stream)));
    if (s != PKV_OK) return s;
  }
  return from_cuda(pkv::launch_decode(plan, pool->tmap, a, pool->launch_flags,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

int paged_attention_decode_ex(const uint16_t* q, const pkv_pool* pool,
                              const int32_t* block_tables, const int32_t* seq_lens, int32_t layer,
                              float scale, float* out, int32_t num_layers, int32_t batch,
                              int32_t max_blocks, void* workspace, size_t workspace_bytes,
                              pkv_stream_t stream, int32_t kernel, int32_t grid_ctas,
                              int32_t min_chunk) {
  return decode_common(q, nullptr, nullptr, pool, block_tables, seq_lens, layer, scale, out,
                       PKV_DTYPE_F32, 1, num_layers, batch, max_blocks, workspace, workspace_bytes,
                       stream, kernel, grid_ctas, min_chunk);
}

int paged_attention_decode_append_ex(const uint16_t* q, const uint16_t* k_new,
                                     const uint16_t* v_new, pkv_pool* pool,
                                     const int32_t* block_tables, const int32_t* seq_lens,
                                     int32_t layer, float scale, float* out, int32_t num_layers,
                                     int32_t batch, int32_t max_blocks, void* workspace,
                                     size_t workspace_bytes, pkv_stream_t stream, int32_t kernel,
                                     int32_t grid_ctas, int32_t min_chunk) {
  if (!k_new || !v_new) return PKV_ERR_INVALID_ARG;
  return decode_common(q, k_new, v_new, pool, block_tables, seq_lens, layer, scale, out,
                       PKV_DTYPE_F32, 1, num_layers, batch, max_blocks, workspace, workspace_bytes,
                       stream, kernel, grid_ctas, min_chunk);
}

int pkv_decode(pkv_pool* pool, const pkv_decode_params* p, pkv_stream_t stream) {
  if (!p || p->struct_size < sizeof(pkv_decode_params)) return PKV_ERR_INVALID_ARG;
  return decode_common(p->q, p->k_new, p->v_new, pool, p->block_tables, p->seq_lens, p->layer,
                       p->scale, p->out, p->out_dtype, p->num_queries, p->num_layers, p->batch,
                       p->max_blocks, p->workspace, p->workspace_bytes, stream, p->kernel,
                       p->grid_ctas, p->min_chunk);
}

int pkv_decode_params_workspace_bytes(const pkv_pool* pool, const pkv_decode_params* p,
                                      size_t* bytes_out) {
  if (!pool || !p || !bytes_out || p->struct_size < sizeof(pkv_decode_params) || p->batch < 0 ||
      p->grid_ctas < 0)
    return PKV_ERR_INVALID_ARG;
  pkv::DecodePlan plan;
  int s = pkv::plan_decode(pool->device, pool->sm_count, p->batch, p->kernel, p->grid_ctas,
                           p->num_queries, &plan);
  if (s != PKV_OK) return s;
  *bytes_out = plan.ws_bytes;
  return PKV_OK;
}

int paged_attention_decode_append(const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                                  pkv_pool* pool, const int32_t* block_tables,
                                  const int32_t* seq_lens, int32_t layer, float scale, float* out,
                                  int32_t num_layers, int32_t batch, int32_t max_blocks,
                                  void* workspace, size_t workspace_bytes, pkv_stream_t stream) {
  return paged_attention_decode_append_ex(q, k_new, v_new, pool, block_tables, seq_lens, layer,
                                          scale, out, num_layers, batch, max_blocks, workspace,
                                          workspace_bytes, stream, PKV_KERNEL_AUTO, 0, 0);
}

int paged_attention_decode(const uint16_t* q, const pkv_pool* pool, const int32_t* block_tables,
                           const int32_t* seq_lens, int32_t layer, float scale, float* out,
                           int32_t num_layers, int32_t batch, int32_t max_blocks,
                           void* workspace, size_t workspace_bytes, pkv_stream_t stream) {
  return paged_attention_decode_ex(q, pool, block_tables, seq_lens, layer, scale, out, num_layers,
                                   batch, max_blocks, workspace, workspace_bytes, stream,
                                   PKV_KERNEL_AUTO, 0, 0);
}

int pkv_gather(const pkv_pool* pool, const int32_t* block_tables, const int32_t* seq_lens,
               int32_t layer, uint16_t* k_out, uint16_t* v_out, int32_t num_layers,
               int32_t batch, int32_t max_blocks, int32_t max_seq_len, pkv_stream_t stream) {
  int s = check_table_args(pool, block_tables, seq_lens, layer, num_layers, batch, max_blocks);
  if (s != PKV_OK) return s;
  if (!k_out || !v_out || !aligned(k_out, 16) || !aligned(v_out, 16) || max_seq_len < 0)
    return PKV_ERR_INVALID_ARG;
  if (batch > 65535) return PKV_ERR_UNSUPPORTED;
  return from_cuda(pkv::launch_gather(
      static_cast<const __nv_bfloat16*>(pool->data),
      layer_slab(block_tables, layer, batch, max_blocks), seq_lens,
      reinterpret_cast<__nv_bfloat16*>(k_out), reinterpret_cast<__nv_bfloat16*>(v_out),
      pool->d_err, batch, max_blocks, pool->num_pages, max_seq_len,
      reinterpret_cast<cudaStream_t>(stream)));
}

int pkv_get_device_error(pkv_pool* pool, pkv_stream_t stream, int32_t* status_out) {
  if (!pool || !status_out) return PKV_ERR_INVALID_ARG;
  int s = check_device(pool);
  if (s != PKV_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t v = 0;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&v, pool->d_err, sizeof v, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(pool->d_err, 0, sizeof(int32_t), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return PKV_ERR_CUDA;
  *status_out = v;
  return PKV_OK;
}

// ---------------------------------------------------------------------------
// Allocation-free decode.
//
// Some callers cannot allocate device memory at the point where they run
// attention: code that executes inside a custom memory-pool or allocator
// callback (where re-entering the allocator deadlocks or corrupts its
// state), plugins for inference runtimes that hand a kernel only its
// inputs and outputs, or real-time loops that must never call
// cudaMalloc/cudaFree because those calls synchronise the device.  For them
// paged_attention_decode_noalloc uses a fixed scratch area that the library
// reserves in device memory when it is loaded, instead of a caller-provided
// workspace.  The area is a file-scope __device__ array (so every GPU that
// loads the library holds it until the process exits); its size bounds the
// batch (pkv.h gives the limit).  The host needs the array's device address,
// which is not the host-side symbol: it is looked up once per device with
// cudaGetSymbolAddress, with that device current, on the first call, and
// kept for the life of the process (a reset of the device's context
// invalidates it; pkv.h says so).
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[PKV_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_scratch_mutex;
void* g_scratch_addr[256];   // per device ordinal; nullptr until looked up

// Device address of this device's scratch array (looked up on first use,
// with `device` current: the caller has checked that it is).
int scratch_for_device(int device, void** out) {
  if (device < 0 || device >= 256) return PKV_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[device]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) return from_cuda(e == cudaSuccess ? cudaErrorInvalidSymbol : e,
                                                 "paged_attention_decode_noalloc: scratch address");
    g_scratch_addr[device] = p;
  }
  *out = g_scratch_addr[device];
  return PKV_OK;
}
}  // namespace

int paged_attention_decode_noalloc(const uint16_t* q, const pkv_pool* pool,
                                   const int32_t* block_tables, const int32_t* seq_lens,
                                   int32_t layer, float scale, float* out, int32_t num_layers,
                                   int32_t batch, int32_t max_blocks, pkv_stream_t stream) {
  // (also checks that the pool's device is the current one, which the
  // address lookup below relies on)
  int s = check_table_args(pool, block_tables, seq_lens, layer, num_layers, batch, max_blocks);
  if (s != PKV_OK) return s;
  size_t need = 0;
  s = pkv_decode_workspace_bytes(pool, batch, &need);
  if (s != PKV_OK) return s;
  if (need > sizeof(g_noalloc_scratch)) {
    snprintf(g_last_error, sizeof g_last_error,
             "paged_attention_decode_noalloc: batch %d needs %zu scratch bytes, the fixed scratch "
             "holds %zu",
             batch, need, sizeof(g_noalloc_scratch));
    return PKV_ERR_TOO_LARGE;
  }
  void* scratch = nullptr;
  s = scratch_for_device(pool->device, &scratch);
  if (s != PKV_OK) return s;
  // Nothing in the workspace has to start at zero (each decode writes the
  // partial records and the split table before reading them), so the shared
  // scratch needs no clearing between calls.
  return paged_attention_decode(q, pool, block_tables, seq_lens, layer, scale, out, num_layers,
                                batch, max_blocks, scratch, sizeof(g_noalloc_scratch), stream);
}

const char* pkv_last_error_message(void) { return g_last_error; }

const char* pkv_status_string(int status) {
  switch (status) {
    case PKV_OK: return "ok";
    case PKV_ERR_INVALID_ARG: return "invalid argument";
    case PKV_ERR_UNSUPPORTED: return "unsupported shape or size";
    case PKV_ERR_CUDA: return "CUDA runtime error";
    case PKV_ERR_OUT_OF_PAGES: return "out of pages";
    case PKV_ERR_BAD_PAGE: return "block-table entry outside the pool";
    case PKV_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case PKV_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case PKV_ERR_BAD_SEQ_LEN: return "sequence length out of range";
    case PKV_ERR_TOO_LARGE: return "request larger than the fixed no-alloc scratch or the whole pool";
    case PKV_ERR_APPEND_CONFLICT: return "appends of one call race (same slot, or a slot another context reads)";
    default: return "unknown status";
  }
}

}  // extern "C"
