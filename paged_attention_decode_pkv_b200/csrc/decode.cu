// decode.cu -- paged decode attention for sm_100a.
//
// What it computes: for every sequence b and query head h,
//   out[b][h] = sum_{t < L_b} softmax_t(scale * q[b][h] . K_t) V_t,
// with K_t / V_t the key / value of token t at kv head h / 4 ("Construye tu
// propio motor de inferencia LLM...", section "Atención de Consulta Agrupada
// (GQA)"), read in place from the 16-token pages that the sequence's block
// table names, with an FP32 online softmax ("Curso gratuito recorre la
// inferencia de LLM...", section "¿Cómo administra el motor la memoria de la
// caché KV?").  Decode is memory-bound (same "Construye..." page, section
// "Prefill vs. Decode"), so the design is about streaming K/V from HBM at
// full bandwidth with as few instructions per byte as possible.
//
// Work decomposition (B200 design, not from the pages).  A unit is one
// (sequence, kv head) pair; its pages form a run of (page, kv head) tiles of
// 4 KiB (2 KiB of K + 2 KiB of V).  All units' tiles are laid end to end in
// (sequence, kv head, page) order and the resulting list is cut into equal
// contiguous ranges, one per warp of a persistent grid (one wave: every SM
// holds the same number of CTAs).  Each warp is an independent pipeline:
// lane 0 issues 2-D TMA loads (128-byte swizzle, L2 evict-first, no
// multicast) of the next tiles into a ring of shared-memory stages guarded
// by mbarriers, while the whole warp computes on the current tile.  No
// __syncthreads in the loop.  The 4 query heads of a kv head share every
// K/V tile load.
//
// A unit that falls inside one warp's range is finished in registers.  A
// unit cut by range boundaries is split-KV: each piece writes (m, l, acc) to
// the workspace and the last piece to arrive (atomic counter per unit)
// merges them in a fixed order with log-sum-exp weights and writes out, so
// the split needs no second launch and the result does not depend on which
// warp finishes last.  Every lane works in log2 units: scores are scaled by
// scale * log2(e) and exponentials are exp2.
#include "pkv_internal.cuh"

namespace pkv {

constexpr int kWarps = 4;                       // warps per CTA
constexpr int kStages = 4;                      // tiles in flight per warp
constexpr int kStageBytes = 2 * kTileBytes;     // K tile + V tile
constexpr unsigned kFull = 0xFFFFFFFFu;

constexpr size_t kTilesBytes = size_t(kWarps) * kStages * kStageBytes;
constexpr size_t kBarsOff = kTilesBytes;
constexpr size_t kLensOff = kBarsOff + size_t(kWarps) * kStages * 8;

static size_t decode_smem_bytes(int32_t batch) {
  // tiles, mbarriers, lengths [B], page-count prefix [B+1], alignment slack
  return kLensOff + size_t(batch) * 4 + size_t(batch + 1) * 4 + 1024;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------------------
// CUDA-core compute: FP32 dot products with packed FFMA2, warp-shuffle
// reductions for the dot products, the max and the sum.
//
// Lane = (token group tg = lane / 8, d chunk c = lane % 8).  For QK the lane
// holds the 8 dims [8c, 8c+8) of q for all 4 heads and reads K rows
// tg, tg+4, tg+8, tg+12 of the page (one 16-byte chunk each), giving 16
// partial dot products; a transposing butterfly over the 8 d-chunk lanes
// (3 steps, 14 shuffles) leaves each lane one full score for one token and
// two heads.  PV uses the same (token group, d chunk) split on V; each lane
// keeps acc[4 heads][8 dims] over its tokens, reduced across token groups
// only when a unit ends.
// ---------------------------------------------------------------------------
struct SimtCompute {
  float2 q2[kGroup][4];   // q[h][8c + 2e], q[h][8c + 2e + 1]
  float2 acc[kGroup][4];  // sum over this lane's tokens of p * v[8c + 2e ..]
  float m[kGroup];        // running max per head (log2 units), warp-uniform
  float lsum[2];          // sum of p over this lane's scores, heads 2*b2 + k

  __device__ __forceinline__ void begin(const __nv_bfloat16* qrows, int lane) {
    const int c = lane & 7;
#pragma unroll
    for (int h = 0; h < kGroup; ++h) {
      const uint4 w = *reinterpret_cast<const uint4*>(qrows + h * kDim + 8 * c);
      q2[h][0] = bf16x2_to_float2(w.x);
      q2[h][1] = bf16x2_to_float2(w.y);
      q2[h][2] = bf16x2_to_float2(w.z);
      q2[h][3] = bf16x2_to_float2(w.w);
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[h][e] = make_float2(0.f, 0.f);
      m[h] = -INFINITY;
    }
    lsum[0] = lsum[1] = 0.f;
  }

  __device__ __forceinline__ void consume(uint32_t ktile, uint32_t vtile, int nvalid,
                                          float scale_log2, int lane) {
    const int c = lane & 7, tg = lane >> 3;
    const int b0 = c & 1, b1 = (c >> 1) & 1, b2 = c >> 2;

    // ---- scores: 4 tokens x 4 heads, partial over this lane's 8 dims
    float s[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = tg + 4 * i;
      const uint4 w = lds128(ktile + swz(t, c));
      const float2 k0 = bf16x2_to_float2(w.x), k1 = bf16x2_to_float2(w.y);
      const float2 k2 = bf16x2_to_float2(w.z), k3 = bf16x2_to_float2(w.w);
#pragma unroll
      for (int h = 0; h < kGroup; ++h) {
        float2 d = __fmul2_rn(q2[h][0], k0);
        d = __ffma2_rn(q2[h][1], k1, d);
        d = __ffma2_rn(q2[h][2], k2, d);
        d = __ffma2_rn(q2[h][3], k3, d);
        s[4 * i + h] = d.x + d.y;
      }
    }
    // ---- transposing butterfly over the 8 d-chunk lanes: 16 -> 8 -> 4 -> 2
    float r1[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float lo = s[k], hi = s[k + 8];
      r1[k] = (b0 ? hi : lo) + __shfl_xor_sync(kFull, b0 ? lo : hi, 1);
    }
    float r2[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float lo = r1[k], hi = r1[k + 4];
      r2[k] = (b1 ? hi : lo) + __shfl_xor_sync(kFull, b1 ? lo : hi, 2);
    }
    float x[2];
    const int tsel = tg + 4 * (b1 + 2 * b0);   // this lane's token
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float lo = r2[k], hi = r2[k + 2];
      const float r3 = (b2 ? hi : lo) + __shfl_xor_sync(kFull, b2 ? lo : hi, 4);
      x[k] = (tsel < nvalid) ? r3 * scale_log2 : -INFINITY;   // head 2*b2 + k
    }
    // ---- page max per head, then running max, rescale factors, weights
    float mx[2] = {x[0], x[1]};
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      mx[k] = fmaxf(mx[k], __shfl_xor_sync(kFull, mx[k], 1));
      mx[k] = fmaxf(mx[k], __shfl_xor_sync(kFull, mx[k], 2));
      mx[k] = fmaxf(mx[k], __shfl_xor_sync(kFull, mx[k], 8));
      mx[k] = fmaxf(mx[k], __shfl_xor_sync(kFull, mx[k], 16));
    }
    const float o0 = __shfl_xor_sync(kFull, mx[0], 4);
    const float o1 = __shfl_xor_sync(kFull, mx[1], 4);
    const float pm[4] = {b2 ? o0 : mx[0], b2 ? o1 : mx[1], b2 ? mx[0] : o0, b2 ? mx[1] : o1};
    float alpha[4];
#pragma unroll
    for (int h = 0; h < kGroup; ++h) {
      const float mn = fmaxf(m[h], pm[h]);
      alpha[h] = fast_exp2(m[h] - mn);
      m[h] = mn;
    }
    float p[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float mh = b2 ? m[2 + k] : m[k];
      const float ah = b2 ? alpha[2 + k] : alpha[k];
      p[k] = fast_exp2(x[k] - mh);
      lsum[k] = fmaf(lsum[k], ah, p[k]);
    }
    // ---- weights of this lane's 4 PV tokens for all 4 heads
    float pv[4][4];
    const int base = tg << 3;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int h = 0; h < kGroup; ++h)
        pv[i][h] = __shfl_sync(kFull, p[h & 1], base | (i >> 1) | ((i & 1) << 1) | ((h >> 1) << 2));
    // ---- rescale and accumulate p * V
#pragma unroll
    for (int h = 0; h < kGroup; ++h) {
      const float2 a2 = make_float2(alpha[h], alpha[h]);
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[h][e] = __fmul2_rn(acc[h][e], a2);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = tg + 4 * i;
      uint4 w = lds128(vtile + swz(t, c));
      if (t >= nvalid) w = make_uint4(0u, 0u, 0u, 0u);   // unused slots may hold NaN
      const float2 v[4] = {bf16x2_to_float2(w.x), bf16x2_to_float2(w.y),
                           bf16x2_to_float2(w.z), bf16x2_to_float2(w.w)};
#pragma unroll
      for (int h = 0; h < kGroup; ++h) {
        const float2 pp = make_float2(pv[i][h], pv[i][h]);
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[h][e] = __ffma2_rn(pp, v[e], acc[h][e]);
      }
    }
  }

  // Sum acc over the 4 token groups: lane (tg, c) ends with head
  // 2*(tg & 1) + (tg >> 1), dims [8c, 8c + 8).
  __device__ __forceinline__ int reduce_acc(float (&r)[8], int lane) const {
    const int tg = lane >> 3, t0 = tg & 1, t1 = tg >> 1;
    float f[32];
#pragma unroll
    for (int h = 0; h < kGroup; ++h)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        f[h * 8 + 2 * e] = acc[h][e].x;
        f[h * 8 + 2 * e + 1] = acc[h][e].y;
      }
    float r1[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float lo = f[k], hi = f[k + 16];
      r1[k] = (t0 ? hi : lo) + __shfl_xor_sync(kFull, t0 ? lo : hi, 8);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float lo = r1[k], hi = r1[k + 8];
      r[k] = (t1 ? hi : lo) + __shfl_xor_sync(kFull, t1 ? lo : hi, 16);
    }
    return 2 * t0 + t1;
  }

  // Softmax denominators of all 4 heads, in every lane.
  __device__ __forceinline__ void reduce_l(float (&l)[4], int lane) const {
    const int b2 = (lane >> 2) & 1;
    float s2[2] = {lsum[0], lsum[1]};
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      s2[k] += __shfl_xor_sync(kFull, s2[k], 1);
      s2[k] += __shfl_xor_sync(kFull, s2[k], 2);
      s2[k] += __shfl_xor_sync(kFull, s2[k], 8);
      s2[k] += __shfl_xor_sync(kFull, s2[k], 16);
    }
    const float o0 = __shfl_xor_sync(kFull, s2[0], 4);
    const float o1 = __shfl_xor_sync(kFull, s2[1], 4);
    l[0] = b2 ? o0 : s2[0];
    l[1] = b2 ? o1 : s2[1];
    l[2] = b2 ? s2[0] : o0;
    l[3] = b2 ? s2[1] : o1;
  }

  __device__ __forceinline__ void finalize(float* out_rows, int lane) const {
    float r[8], l[4];
    const int h = reduce_acc(r, lane);
    reduce_l(l, lane);
    const float lh = h == 0 ? l[0] : h == 1 ? l[1] : h == 2 ? l[2] : l[3];
    const float inv = 1.f / lh;
    float4* dst = reinterpret_cast<float4*>(out_rows + h * kDim + 8 * (lane & 7));
    dst[0] = make_float4(r[0] * inv, r[1] * inv, r[2] * inv, r[3] * inv);
    dst[1] = make_float4(r[4] * inv, r[5] * inv, r[6] * inv, r[7] * inv);
  }

  // Partial record: m[4], l[4], acc[4][64] (unnormalised).
  __device__ __forceinline__ void store_partial(float* P, int lane) const {
    float r[8], l[4];
    const int h = reduce_acc(r, lane);
    reduce_l(l, lane);
    if (lane == 0) {
      reinterpret_cast<float4*>(P)[0] = make_float4(m[0], m[1], m[2], m[3]);
      reinterpret_cast<float4*>(P)[1] = make_float4(l[0], l[1], l[2], l[3]);
    }
    float4* dst = reinterpret_cast<float4*>(P + 2 * kGroup + h * kDim + 8 * (lane & 7));
    dst[0] = make_float4(r[0], r[1], r[2], r[3]);
    dst[1] = make_float4(r[4], r[5], r[6], r[7]);
  }
};

// ---------------------------------------------------------------------------
// Shared pieces of the persistent kernel
// ---------------------------------------------------------------------------

// Lengths of all sequences and the exclusive prefix of their page counts,
// computed by every CTA (B integers from L2; cheaper than a second launch).
// Invalid lengths count as empty sequences and are reported.
__device__ __forceinline__ void cta_lengths(const DecodeArgs& a, int32_t* s_len, int32_t* s_pfx,
                                            int32_t* s_tot) {
  const int B = a.batch, tid = threadIdx.x, nthr = blockDim.x;
  const int per = (B + nthr - 1) / nthr;
  const int b0 = min(B, tid * per), b1 = min(B, b0 + per);
  const int64_t cap = static_cast<int64_t>(a.max_blocks) * kTokens;
  int sum = 0;
  for (int b = b0; b < b1; ++b) {
    int L = a.seq_lens[b];
    if (L < 0 || L > cap) {
      if (blockIdx.x == 0) record_error(a.err, kErrBadLen);
      L = 0;
    }
    s_len[b] = L;
    sum += (L + kTokens - 1) / kTokens;
  }
  const int lane = tid & 31, warp = tid >> 5;
  int x = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_tot[warp] = x;
  __syncthreads();
  int run = x - sum;
  for (int k = 0; k < warp; ++k) run += s_tot[k];
  if (tid == 0) s_pfx[0] = 0;
  for (int b = b0; b < b1; ++b) {
    run += (s_len[b] + kTokens - 1) / kTokens;
    s_pfx[b + 1] = run;
  }
  __syncthreads();
}

// (sequence, kv head, page) of flat tile index f < 8 * s_pfx[B].
__device__ __forceinline__ void locate(const int32_t* s_pfx, int B, int32_t f, int& b, int& g,
                                       int& j) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {   // largest b with 8 * pfx[b] <= f
    const int mid = (lo + hi + 1) >> 1;
    if (kKvHeads * s_pfx[mid] <= f) lo = mid; else hi = mid - 1;
  }
  b = lo;
  const int np = s_pfx[b + 1] - s_pfx[b];
  const int rel = f - kKvHeads * s_pfx[b];
  g = rel / np;
  j = rel - g * np;
}

__device__ __forceinline__ void zero_rows(float* rows, int lane) {
  float4* d = reinterpret_cast<float4*>(rows);
#pragma unroll 4
  for (int i = lane; i < kQHeads * kDim / 4; i += 32) d[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// Fixed-order log-sum-exp merge of `cnt` partial records.  Lane handles dims
// 2*lane, 2*lane+1 of all 4 heads.
__device__ __noinline__ void merge_partials(const float* P, int cnt, float* out_rows, int lane) {
  float M[kGroup], S[kGroup];
  float2 O[kGroup];
#pragma unroll
  for (int h = 0; h < kGroup; ++h) {
    M[h] = -INFINITY;
    S[h] = 0.f;
    O[h] = make_float2(0.f, 0.f);
  }
#pragma unroll 2
  for (int s = 0; s < cnt; ++s) {
    const float* p = P + static_cast<int64_t>(s) * kPartialFloats;
    const float4 m4 = __ldcg(reinterpret_cast<const float4*>(p));
    const float4 l4 = __ldcg(reinterpret_cast<const float4*>(p) + 1);
    const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
    const float ll[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
    for (int h = 0; h < kGroup; ++h) {
      const float2 o = __ldcg(reinterpret_cast<const float2*>(p + 2 * kGroup + h * kDim) + lane);
      const float mn = fmaxf(M[h], mm[h]);
      if (mn == -INFINITY) continue;   // nothing accumulated on either side yet
      const float sa = fast_exp2(M[h] - mn), sb = fast_exp2(mm[h] - mn);
      S[h] = S[h] * sa + ll[h] * sb;
      O[h].x = O[h].x * sa + o.x * sb;
      O[h].y = O[h].y * sa + o.y * sb;
      M[h] = mn;
    }
  }
#pragma unroll
  for (int h = 0; h < kGroup; ++h) {
    const float inv = S[h] > 0.f ? 1.f / S[h] : 0.f;
    reinterpret_cast<float2*>(out_rows + h * kDim)[lane] = make_float2(O[h].x * inv, O[h].y * inv);
  }
}

// End of a unit's piece inside this warp's range: finish it in registers, or
// hand it to the split-KV merge.
template <class C>
__device__ __forceinline__ void flush_unit(const C& cmp, const DecodeArgs& a,
                                           const int32_t* s_pfx, int b, int g, int j0, int j1,
                                           int np, int w, int64_t chunk, int lane) {
  float* out_rows = a.out + (static_cast<int64_t>(b) * kQHeads + g * kGroup) * kDim;
  if (j0 == 0 && j1 == np - 1) {
    cmp.finalize(out_rows, lane);
    return;
  }
  const int u = b * kKvHeads + g;
  const int64_t start = static_cast<int64_t>(kKvHeads) * s_pfx[b] + static_cast<int64_t>(g) * np;
  const int w_first = static_cast<int>(start / chunk);
  const int w_last = static_cast<int>((start + np - 1) / chunk);
  cmp.store_partial(a.partials + static_cast<int64_t>(u + w) * kPartialFloats, lane);
  __threadfence();
  __syncwarp();
  int prev = 0;
  if (lane == 0) prev = atomicAdd(a.counters + u, 1);
  prev = __shfl_sync(kFull, prev, 0);
  if (prev != w_last - w_first) return;   // not the last piece of this unit
  __threadfence();
  merge_partials(a.partials + static_cast<int64_t>(u + w_first) * kPartialFloats,
                 w_last - w_first + 1, out_rows, lane);
  if (lane == 0) a.counters[u] = 0;       // ready for the next launch
}

// Producer-side description of 32 consecutive tiles: lane i -> tile f0 + i.
__device__ __forceinline__ void load_tile_batch(const DecodeArgs& a, const int32_t* s_pfx,
                                                int32_t f, int32_t f_end, int32_t& phys,
                                                int32_t& kvh) {
  phys = -1;
  kvh = 0;
  if (f < f_end) {
    int b, g, j;
    locate(s_pfx, a.batch, f, b, g, j);
    phys = __ldg(a.bt + static_cast<int64_t>(b) * a.max_blocks + j);
    kvh = g;
  }
}

template <class C>
__global__ void __launch_bounds__(kWarps * 32, 3)
    decode_kernel(const __grid_constant__ CUtensorMap tmap, const DecodeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ int32_t s_tot[kWarps];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int B = a.batch;
  int32_t* s_len = reinterpret_cast<int32_t*>(smem + kLensOff);
  int32_t* s_pfx = s_len + B;

  cta_lengths(a, s_len, s_pfx, s_tot);

  const uint32_t tiles = smem_addr(smem) + warp * kStages * kStageBytes;
  const uint32_t bars = smem_addr(smem + kBarsOff) + warp * kStages * 8;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) mbar_init(bars + 8 * s, 1);
    fence_mbar_init();
  }
  __syncwarp();

  const int W = gridDim.x * kWarps;
  const int w = blockIdx.x * kWarps + warp;
  const int32_t P = kKvHeads * s_pfx[B];
  int64_t chunk = (static_cast<int64_t>(P) + W - 1) / W;
  if (chunk < a.min_chunk) chunk = a.min_chunk;
  if (chunk < 1) chunk = 1;

  for (int b = w; b < B; b += W)
    if (s_pfx[b + 1] == s_pfx[b]) zero_rows(a.out + static_cast<int64_t>(b) * kQHeads * kDim, lane);

  const int64_t q0l = static_cast<int64_t>(w) * chunk;
  if (q0l >= P) return;
  const int32_t q0 = static_cast<int32_t>(q0l);
  const int32_t q1 = static_cast<int32_t>(q0l + chunk < P ? q0l + chunk : P);
  const int n = q1 - q0;
  const uint64_t policy = l2_evict_first_policy();

  // producer state: tile descriptions for batches k (cur) and k + 1 (nxt)
  int32_t cur_phys, cur_g, nxt_phys, nxt_g;
  load_tile_batch(a, s_pfx, q0 + lane, q1, cur_phys, cur_g);
  load_tile_batch(a, s_pfx, q0 + 32 + lane, q1, nxt_phys, nxt_g);
  int cur_k = 0;
  uint32_t bad = 0;   // bit s set: stage s holds a skipped (invalid) page
  int prod = 0;

  auto issue = [&](int r) {
    if ((r >> 5) != cur_k) {
      cur_phys = nxt_phys;
      cur_g = nxt_g;
      ++cur_k;
      load_tile_batch(a, s_pfx, q0 + 32 * (cur_k + 1) + lane, q1, nxt_phys, nxt_g);
    }
    const int32_t phys = __shfl_sync(kFull, cur_phys, r & 31);
    const int32_t g = __shfl_sync(kFull, cur_g, r & 31);
    const int st = r % kStages;
    const bool ok = static_cast<uint32_t>(phys) < static_cast<uint32_t>(a.num_pages);
    if (lane == 0) {
      const uint32_t bar = bars + 8 * st;
      if (ok) {
        mbar_arrive_expect_tx(bar, kStageBytes);
        const int32_t y = phys * kRowsPerPage + g * kTokens;
        tma_load_tile(tiles + st * kStageBytes, &tmap, 0, y, bar, policy);
        tma_load_tile(tiles + st * kStageBytes + kTileBytes, &tmap, 0, y + kKvHeads * kTokens, bar,
                      policy);
      } else {
        record_error(a.err, kErrBadPage);
        mbar_arrive(bar);
      }
    }
    bad = ok ? (bad & ~(1u << st)) : (bad | (1u << st));
  };

  // consumer state
  int b, g, j;
  locate(s_pfx, B, q0, b, g, j);
  int np = s_pfx[b + 1] - s_pfx[b];
  int L = s_len[b];
  int j_first = j;
  C cmp;
  cmp.begin(a.q + (static_cast<int64_t>(b) * kQHeads + g * kGroup) * kDim, lane);

  for (; prod < n && prod < kStages; ++prod) issue(prod);

  for (int r = 0; r < n; ++r) {
    const int st = r % kStages;
    const uint32_t parity = static_cast<uint32_t>(r / kStages) & 1u;
    if (!mbar_try_wait(bars + 8 * st, parity) && !mbar_wait_bounded(bars + 8 * st, parity)) {
      // A copy never landed.  Record it, wait (bounded) for the other copies
      // this warp still has in flight, and stop; the workspace counters of
      // this launch are then unreliable and must be zeroed again.
      if (lane == 0) record_error(a.err, kErrTimeout);
      for (int rr = r + 1; rr < prod; ++rr)
        mbar_wait_bounded(bars + 8 * (rr % kStages), static_cast<uint32_t>(rr / kStages) & 1u);
      return;
    }
    if (!((bad >> st) & 1u)) {
      const int nvalid = min(kTokens, L - kTokens * j);
      cmp.consume(tiles + st * kStageBytes, tiles + st * kStageBytes + kTileBytes, nvalid,
                  a.scale_log2, lane);
    }
    __syncwarp();
    if (prod < n) {
      issue(prod);
      ++prod;
    }
    if (j == np - 1 || r == n - 1) {
      flush_unit(cmp, a, s_pfx, b, g, j_first, j, np, w, chunk, lane);
      if (r < n - 1) {
        if (++g == kKvHeads) {
          g = 0;
          do {
            ++b;
          } while (s_pfx[b + 1] == s_pfx[b]);
        }
        j = 0;
        j_first = 0;
        np = s_pfx[b + 1] - s_pfx[b];
        L = s_len[b];
        cmp.begin(a.q + (static_cast<int64_t>(b) * kQHeads + g * kGroup) * kDim, lane);
      }
    } else {
      ++j;
    }
  }
}

// ---------------------------------------------------------------- host side --

template <class C>
static const void* kernel_ptr() {
  return reinterpret_cast<const void*>(&decode_kernel<C>);
}

static const void* kernel_for(int kernel) {
  switch (kernel) {
    case PKV_KERNEL_SIMT: return kernel_ptr<SimtCompute>();
    default: return nullptr;
  }
}

cudaError_t prepare_decode_kernels(int device) {
  int optin = 0;
  cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
  if (e != cudaSuccess) return e;
  for (int k : {PKV_KERNEL_SIMT}) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kernel_for(k));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kernel_for(k), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin - static_cast<int>(fa.sharedSizeBytes));
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

int plan_decode(int device, int sm_count, int32_t batch, int kernel, int grid_ctas,
                DecodePlan* plan) {
  if (kernel == PKV_KERNEL_AUTO) kernel = PKV_KERNEL_SIMT;
  const void* fn = kernel_for(kernel);
  if (!fn) return PKV_ERR_UNSUPPORTED;
  int optin = 0;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) !=
      cudaSuccess)
    return PKV_ERR_CUDA;
  const size_t smem = decode_smem_bytes(batch);
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) return PKV_ERR_CUDA;
  if (smem + fa.sharedSizeBytes > static_cast<size_t>(optin)) return PKV_ERR_UNSUPPORTED;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kWarps * 32, smem) !=
      cudaSuccess)
    return PKV_ERR_CUDA;
  if (per_sm < 1) return PKV_ERR_UNSUPPORTED;
  plan->kernel = kernel;
  plan->warps = kWarps;
  plan->smem = smem;
  plan->grid = grid_ctas > 0 ? grid_ctas : sm_count * per_sm;
  const int64_t units = static_cast<int64_t>(batch) * kKvHeads;
  const int64_t W = static_cast<int64_t>(plan->grid) * kWarps;
  plan->counters_bytes = ((units * 4 + 255) / 256) * 256;
  plan->ws_bytes = plan->counters_bytes +
                   static_cast<size_t>(units + W) * kPartialFloats * sizeof(float);
  return PKV_OK;
}

cudaError_t launch_decode(const DecodePlan& plan, const CUtensorMap& tmap, const DecodeArgs& a,
                          cudaStream_t stream) {
  switch (plan.kernel) {
    case PKV_KERNEL_SIMT:
      decode_kernel<SimtCompute><<<plan.grid, plan.warps * 32, plan.smem, stream>>>(tmap, a);
      break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace pkv
