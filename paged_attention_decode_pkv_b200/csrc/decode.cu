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
// full bandwidth with as few instructions and as little serial latency per
// byte as possible.
//
// Work decomposition (B200 design, not from the pages).  Pages are the unit
// of data movement: a 32 KiB page holds K and V of 16 tokens for all 8 kv
// heads, and one 2-D TMA box of 256 rows x 128 B (128-byte swizzle, L2
// evict-first, no multicast) brings a whole page into shared memory.  A CTA
// has 8 warps, warp g computing kv head g -- the 4 query heads of that group
// share every K/V tile.  The sequences' pages are laid end to end (each
// sequence also costs kSeqCost pages of fixed work) and the total is cut into
// equal contiguous ranges, one per CTA of a persistent grid (one wave, the
// same number of CTAs on every SM).  Lane 0 of warp 0 is the producer: it
// walks the CTA's range, reads each page's block-table entry, and issues the
// page's TMA load -- plus, for a page that starts a sequence, a bulk copy of
// the sequence's 32 query rows -- into a ring of stages, each guarded by a
// "full" mbarrier (TMA transaction bytes) and an "empty" mbarrier (one
// arrival per warp once it is done with the stage).
//
// A sequence whose pages all fall in one CTA is finished in registers.  A
// sequence cut by range boundaries is split-KV: each piece writes (m, l, acc)
// per kv head to the workspace, and merge_kernel, launched right after on the
// same stream, combines the pieces in piece order with log-sum-exp weights,
// so the result does not depend on which CTA finishes first.  Scores are kept
// in log2 units (scaled by scale * log2(e)) and exponentials are exp2.
//
// Fused append (paged_attention_decode_append).  Decode attends to the token
// that the step appends (comrad404 article on samir-vllm, section "Что README
// говорит о KV-кэше и пакетном декодировании": decode adds the new token to
// the cache).  With k_new / v_new given, the producer also bulk-copies the
// new token's K and V rows (2 KiB) into the stage of the sequence's last
// page; once the page has landed, warp g writes its head's two rows into the
// staged page (slot (L-1) % 16) and into the pool, then computes as usual.
// So the append costs no launch, and the page is read from HBM only once.
//
// Two compute variants share this skeleton:
//  - SimtCompute: CUDA-core FP32 dot products (packed FFMA2) with
//    warp-shuffle reductions for the dot products, the max and the sum;
//  - MmaComputeT<n-tiles, one>: the 16-token x 4-head tile on the tensor
//    cores (mma.sync m16n8k16, BF16 in, FP32 accumulate) for both Q.K^T and
//    P.V, with P split into two BF16 terms (hi + lo) so that rounding P to
//    BF16 costs no accuracy; softmax stays FP32 on the CUDA cores.  Each
//    N = 8 tile holds 4 heads of two queries of the same sequence, so up to
//    8 causal queries (each seeing one token more than the one before) share
//    every K/V fragment; a single query leaves 4 columns zero.
//
// With programmatic dependent launch the kernel reads the lengths and block
// tables, and optionally starts its first page loads, before waiting for the
// preceding kernel of the stream (launch flags in pkv.h).
#include <type_traits>

#include "pkv_internal.cuh"

namespace pkv {

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr int kWarps = kKvHeads;                    // one warp per kv head
constexpr int kPageBytes = 2 * kKvHeads * kTileBytes;  // 32 KiB
constexpr int kQRowsBytes = kQHeads * kRowBytes;    // one query's 32 head rows: 4 KiB
constexpr int kNewRowsBytes = 2 * kKvHeads * kRowBytes;  // new token's K and V rows: 2 KiB
// stage = page | query rows (nq queries) | new token rows; a multiple of
// 1024 B, so that every stage keeps the 1024-B alignment the 128-byte
// swizzle needs
template <int nq>
struct StageLayout {
  static constexpr int kQBytes = nq * kQRowsBytes;
  static constexpr int kBytes = kPageBytes + kQBytes + kNewRowsBytes;
  static_assert(kBytes % 1024 == 0, "stage alignment");
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Output rows of one (sequence, kv head) unit: element (query i, head h of
// the group, dim d) is at base + i * qstride + h * 64 + d, FP32 or (kBf16)
// BF16 rounded to nearest even.  Partial records use the same shape in FP32.
template <bool kBf16>
struct OutRowsT {
  void* base;
  int64_t qstride;   // elements

  __device__ __forceinline__ int64_t at(int i, int h, int d) const {
    return i * qstride + h * kDim + d;
  }
  __device__ __forceinline__ void put(int i, int h, int d, float v) const {
    if constexpr (kBf16)
      static_cast<__nv_bfloat16*>(base)[at(i, h, d)] = __float2bfloat16_rn(v);
    else
      static_cast<float*>(base)[at(i, h, d)] = v;
  }
  // dims d, d + 1 (d even)
  __device__ __forceinline__ void put2(int i, int h, int d, float x, float y) const {
    if constexpr (kBf16)
      *reinterpret_cast<uint32_t*>(static_cast<__nv_bfloat16*>(base) + at(i, h, d)) =
          pack_bf16x2(x, y);
    else
      *reinterpret_cast<float2*>(static_cast<float*>(base) + at(i, h, d)) = make_float2(x, y);
  }
  // dims d .. d + 7 (d a multiple of 8)
  __device__ __forceinline__ void put8(int i, int h, int d, const float* v) const {
    if constexpr (kBf16) {
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(base) + at(i, h, d)) =
          make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                     pack_bf16x2(v[6], v[7]));
    } else {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(base) + at(i, h, d));
      dst[0] = make_float4(v[0], v[1], v[2], v[3]);
      dst[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
  }
};

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
  static constexpr int kStages = 3;
  static constexpr int kMinBlocks = 1;
  static constexpr int kMaxQueries = 1;
  static constexpr int kScratch = 512;

  float2 q2[kGroup][4];   // q[h][8c + 2e], q[h][8c + 2e + 1]
  float2 acc[kGroup][4];  // sum over this lane's tokens of p * v[8c + 2e ..]
  float m[kGroup];        // running max per head (log2 units), warp-uniform
  float lsum[2];          // sum of p over this lane's scores, heads 2*b2 + k

  // (one query per sequence: the CUDA-core variant does not take two)
  __device__ __forceinline__ void begin(uint32_t qrows, int warp, int /*nq*/, int lane) {
    const uint32_t qslot = qrows + warp * (kGroup * kRowBytes);
    const int c = lane & 7;
#pragma unroll
    for (int h = 0; h < kGroup; ++h) {
      const uint4 w = lds128(qslot + h * kRowBytes + 16 * c);
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

  __device__ __forceinline__ void consume(uint32_t ktile, uint32_t vtile, uint32_t /*scratch*/,
                                          int rem, float scale_log2, int lane) {
    const int nvalid = min(kTokens, rem);
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

  template <class Out>
  __device__ __forceinline__ void finalize(const Out& out, int lane) const {
    float r[8], l[4];
    const int h = reduce_acc(r, lane);
    reduce_l(l, lane);
    const float lh = h == 0 ? l[0] : h == 1 ? l[1] : h == 2 ? l[2] : l[3];
    const float inv = 1.f / lh;
#pragma unroll
    for (int k = 0; k < 8; ++k) r[k] *= inv;
    out.put8(0, h, 8 * (lane & 7), r);
  }

  // Partial record: m[4], l[4], acc[4][64] (unnormalised).
  __device__ __forceinline__ void store_partial(float* P, int /*nq*/, int lane) const {
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
// Tensor-core compute (mma.sync m16n8k16, BF16 x BF16 -> FP32).
//
// Lane = (r = lane / 4, qd = lane % 4), the mma fragment coordinates.
//  QK:  S^T[t][h] = sum_d K[t][d] Q[h][d]: M = 16 tokens (A = the K tile,
//       ldmatrix from the swizzled stage), N = 8 (4 real heads + 4 zero
//       columns), K = 64 in 4 steps.  Products of BF16 values are exact in
//       FP32, so this is the same arithmetic as the CUDA-core dot product.
//       Lane holds S^T[r][2qd..2qd+1] and S^T[r+8][2qd..2qd+1].
//  softmax: FP32, per head over the 16 tokens (2 per lane x 8 lanes).
//  PV:  O^T[d][h] = sum_t V^T[d][t] P^T[t][h]: M = 64 dims in 4 tiles
//       (A = V^T via ldmatrix.trans), N = 8 heads, K = 16 tokens.  P^T is
//       written to a per-warp scratch in [t][h] order and read back with
//       ldmatrix.trans as the B fragment.  P is split into
//       hi = bf16(p) and lo = bf16(p - hi), two MMAs, so the product keeps
//       ~16 mantissa bits of p.
//  Lane holds O^T[16mt + r (+8)][2qd..2qd+1]: its softmax heads and its
//  accumulator heads are the same, so rescaling needs no data movement.
// ---------------------------------------------------------------------------
// kNt n-tiles of the MMA's N = 8: column n of tile nt is head n % 4 of
// query 2 nt + n / 4, so one K/V stream serves up to 2 kNt queries of a
// sequence.  kOne: exactly one query (tile 0's columns 4..7 stay zero); its
// masks and guards are then compile-time.
template <int kNt, bool kOne>
struct MmaComputeT {
  static constexpr int kStages = 2;
  static constexpr int kMinBlocks = kNt == 1 ? 2 : 1;
  static constexpr int kMaxQueries = kOne ? 1 : 2 * kNt;
  static constexpr int kScratch = kNt * 512;   // per-warp P^T transpose buffers

  uint32_t qb[kNt][4][2];  // B fragments of Q^T, k-steps 0..3 (zero for absent queries)
  float o[kNt][4][4];      // O^T accumulators, m-tiles 0..3
  float m[kNt][2];         // running max of the lane's two columns (log2 units)
  float l[kNt][2];         // this lane's share of the softmax denominators
  int nq;                  // queries of the sequence

  // qrows: the staged query rows ([query][32 heads][64]).
  __device__ __forceinline__ void begin(uint32_t qrows, int warp, int nq_, int lane) {
    nq = kOne ? 1 : nq_;
    const int r = lane >> 2, qd = lane & 3;
#pragma unroll
    for (int nt = 0; nt < kNt; ++nt) {
      const int qi = 2 * nt + r / kGroup;
      const uint32_t row = qrows + (qi * kQHeads + warp * kGroup + r % kGroup) * kRowBytes;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        if (qi < nq) {
          const uint32_t a = row + (16 * ks + 2 * qd) * 2;
          qb[nt][ks][0] = lds32(a);
          qb[nt][ks][1] = lds32(a + 16);
        } else {
          qb[nt][ks][0] = qb[nt][ks][1] = 0u;
        }
      }
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) o[nt][mt][i] = 0.f;
      m[nt][0] = m[nt][1] = -INFINITY;
      l[nt][0] = l[nt][1] = 0.f;
    }
  }

  // rem: tokens from this page's first slot to the end of the context (of the
  // last query); query q of nq sees nq - 1 - q tokens fewer, possibly none
  // of this page.
  __device__ __forceinline__ void consume(uint32_t ktile, uint32_t vtile, uint32_t scratch,
                                          int rem, float scale_log2, int lane) {
    const int r = lane >> 2, qd = lane & 3;
    const int nvalid = min(kTokens, rem);
    // ---- S^T = K Q^T, each K fragment used by every n-tile
    float s[kNt][4];
#pragma unroll
    for (int nt = 0; nt < kNt; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t a[4];
      ldsm_x4(a, ktile + swz(lane & 15, 2 * ks + (lane >> 4)));
#pragma unroll
      for (int nt = 0; nt < kNt; ++nt) mma_bf16_16816(s[nt], a, qb[nt][ks][0], qb[nt][ks][1]);
    }
    uint32_t pb[kNt][4];   // per tile: hi b0, b1; lo b0, b1
    float a0[kNt], a1[kNt];
#pragma unroll
    for (int nt = 0; nt < kNt; ++nt) {
      // ---- FP32 online softmax; tokens r and r + 8, columns 2qd and 2qd + 1
      // (query 2 nt + qd / 2)
      const int nv = kOne ? nvalid : min(kTokens, rem - (nq - 1 - (2 * nt + (qd >> 1))));
      const bool v0 = r < nv, v1 = r + 8 < nv;
      const float x0 = v0 ? s[nt][0] * scale_log2 : -INFINITY;
      const float x1 = v0 ? s[nt][1] * scale_log2 : -INFINITY;
      const float x2 = v1 ? s[nt][2] * scale_log2 : -INFINITY;
      const float x3 = v1 ? s[nt][3] * scale_log2 : -INFINITY;
      float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, off));
      }
      const float mn0 = fmaxf(m[nt][0], mx0), mn1 = fmaxf(m[nt][1], mx1);
      // a column with no valid score yet (an earlier query's context can end
      // a page early) keeps m = -inf: subtract 0 there, so that -inf - -inf
      // never appears; its p and the rescale factor are then 0
      const float r0 = (!kOne && mn0 == -INFINITY) ? 0.f : mn0;
      const float r1 = (!kOne && mn1 == -INFINITY) ? 0.f : mn1;
      a0[nt] = fast_exp2(m[nt][0] - r0);
      a1[nt] = fast_exp2(m[nt][1] - r1);
      m[nt][0] = mn0;
      m[nt][1] = mn1;
      const float p0 = fast_exp2(x0 - r0), p1 = fast_exp2(x1 - r1);
      const float p2 = fast_exp2(x2 - r0), p3 = fast_exp2(x3 - r1);
      l[nt][0] = fmaf(l[nt][0], a0[nt], p0 + p2);
      l[nt][1] = fmaf(l[nt][1], a1[nt], p1 + p3);
      // ---- P^T, split into BF16 hi + lo, through the tile's scratch ([t][8])
      const uint32_t h01 = pack_bf16x2(p0, p1), h23 = pack_bf16x2(p2, p3);
      const uint32_t l01 = pack_bf16x2(p0 - __uint_as_float(h01 << 16),
                                       p1 - __uint_as_float(h01 & 0xFFFF0000u));
      const uint32_t l23 = pack_bf16x2(p2 - __uint_as_float(h23 << 16),
                                       p3 - __uint_as_float(h23 & 0xFFFF0000u));
      const uint32_t sc = scratch + nt * 512;
      if (nt == 0) __syncwarp();   // previous page's scratch reads are done
      const uint32_t w0 = sc + r * 16 + qd * 4;
      sts32(w0, h01);
      sts32(w0 + 128, h23);
      sts32(w0 + 256, l01);
      sts32(w0 + 384, l23);
    }
    __syncwarp();
#pragma unroll
    for (int nt = 0; nt < kNt; ++nt)
      ldsm_x4_trans(pb[nt], scratch + nt * 512 + (lane >> 3) * 128 + (lane & 7) * 16);
    // ---- rescale and O^T += V^T P^T (hi, lo), each V fragment used by every tile
    uint32_t mlo = kFull, mhi = kFull;
    if (nvalid < kTokens) {   // zero V rows past the context: 0 * NaN would be NaN
      const int t = 2 * qd;
      mlo = (t < nvalid ? 0x0000FFFFu : 0u) | (t + 1 < nvalid ? 0xFFFF0000u : 0u);
      mhi = (t + 8 < nvalid ? 0x0000FFFFu : 0u) | (t + 9 < nvalid ? 0xFFFF0000u : 0u);
    }
    const int vrow = (lane & 7) + ((lane >> 4) << 3);
    const int vchunk = (lane >> 3) & 1;
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      uint32_t a[4];
      ldsm_x4_trans(a, vtile + swz(vrow, 2 * mt + vchunk));
      a[0] &= mlo;
      a[1] &= mlo;
      a[2] &= mhi;
      a[3] &= mhi;
#pragma unroll
      for (int nt = 0; nt < kNt; ++nt) {
        o[nt][mt][0] *= a0[nt];
        o[nt][mt][1] *= a1[nt];
        o[nt][mt][2] *= a0[nt];
        o[nt][mt][3] *= a1[nt];
        mma_bf16_16816(o[nt][mt], a, pb[nt][0], pb[nt][1]);
        mma_bf16_16816(o[nt][mt], a, pb[nt][2], pb[nt][3]);
      }
    }
  }

  // Full softmax denominators of tile nt's columns 2qd, 2qd + 1.
  __device__ __forceinline__ void reduce_l(int nt, float& l0, float& l1) const {
    l0 = l[nt][0];
    l1 = l[nt][1];
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(kFull, l0, off);
      l1 += __shfl_xor_sync(kFull, l1, off);
    }
  }

  // Tile nt's O^T columns 2qd, 2qd + 1 = query 2 nt + qd / 2, heads
  // 2(qd % 2) and 2(qd % 2) + 1, scaled by s0, s1; absent queries write nothing.
  template <class Out>
  __device__ __forceinline__ void write_rows(const Out& out, int nt, int lane, float s0,
                                             float s1) const {
    const int r = lane >> 2, qd = lane & 3;
    const int qi = 2 * nt + (qd >> 1), h = 2 * (qd & 1);
    if (qi < nq) {
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        out.put(qi, h, 16 * mt + r, o[nt][mt][0] * s0);
        out.put(qi, h + 1, 16 * mt + r, o[nt][mt][1] * s1);
        out.put(qi, h, 16 * mt + r + 8, o[nt][mt][2] * s0);
        out.put(qi, h + 1, 16 * mt + r + 8, o[nt][mt][3] * s1);
      }
    }
  }

  template <class Out>
  __device__ __forceinline__ void finalize(const Out& out, int lane) const {
#pragma unroll
    for (int nt = 0; nt < kNt; ++nt) {
      float l0, l1;
      reduce_l(nt, l0, l1);
      write_rows(out, nt, lane, 1.f / l0, 1.f / l1);
    }
  }

  // Partial records, one per query: P + i * kPartialFloats = m[4], l[4],
  // acc[4][64] of query i (unnormalised).
  __device__ __forceinline__ void store_partial(float* P, int /*nq*/, int lane) const {
#pragma unroll
    for (int nt = 0; nt < kNt; ++nt) {
      float l0, l1;
      reduce_l(nt, l0, l1);
      const int qd = lane & 3, qi = 2 * nt + (qd >> 1), h = 2 * (qd & 1);
      if (lane < 4 && qi < nq) {   // r == 0
        float* rec = P + qi * kPartialFloats;
        rec[h] = m[nt][0];
        rec[h + 1] = m[nt][1];
        rec[kGroup + h] = l0;
        rec[kGroup + h + 1] = l1;
      }
      write_rows(OutRowsT<false>{P + 2 * kGroup, kPartialFloats}, nt, lane, 1.f, 1.f);
    }
  }
};

// ---------------------------------------------------------------------------
// Shared pieces of the persistent kernel
// ---------------------------------------------------------------------------

// Lengths of all sequences and the prefix of their page counts, computed by
// every CTA (B integers from L2; cheaper than a second launch).  Invalid
// lengths count as empty sequences and are reported.
__device__ __forceinline__ void cta_lengths(const DecodeArgs& a, int32_t* s_len, int32_t* s_pfx,
                                            int32_t* s_tot) {
  const int B = a.batch, tid = threadIdx.x, nthr = blockDim.x;
  const int per = (B + nthr - 1) / nthr;
  const int b0 = min(B, tid * per), b1 = min(B, b0 + per);
  const int64_t cap = static_cast<int64_t>(a.max_blocks) * kTokens;
  int sum = 0;
  for (int b = b0; b < b1; ++b) {
    int L = a.seq_lens[b];
    if (L < 0 || L > cap || (L > 0 && L < a.num_queries)) {   // every query needs a token
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
}

// Cost position where sequence b starts: every sequence costs its pages plus
// kSeqCost.  Page j of sequence b sits at seq_cost(b) + kSeqCost + j.
__device__ __forceinline__ int64_t seq_cost(const int32_t* s_pfx, int b) {
  return static_cast<int64_t>(s_pfx[b]) + static_cast<int64_t>(kSeqCost) * b;
}

// Number of pages whose cost position is below x.
__device__ __forceinline__ int32_t pages_below(const int32_t* s_pfx, int B, int64_t x) {
  if (x >= seq_cost(s_pfx, B)) return s_pfx[B];
  int lo = 0, hi = B - 1;
  while (lo < hi) {   // largest b with seq_cost(b) <= x
    const int mid = (lo + hi + 1) >> 1;
    if (seq_cost(s_pfx, mid) <= x) lo = mid; else hi = mid - 1;
  }
  const int64_t off = x - seq_cost(s_pfx, lo) - kSeqCost;
  return s_pfx[lo] + static_cast<int32_t>(off < 0 ? 0 : off);
}

// (sequence, page) of flat page index f < s_pfx[B].
__device__ __forceinline__ void locate(const int32_t* s_pfx, int B, int32_t f, int& b, int& j) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {   // largest b with pfx[b] <= f
    const int mid = (lo + hi + 1) >> 1;
    if (s_pfx[mid] <= f) lo = mid; else hi = mid - 1;
  }
  b = lo;
  j = f - s_pfx[b];
}

// Zero the output rows of sequence b (all its queries), one warp.
__device__ __forceinline__ void zero_rows(const DecodeArgs& a, int b, int lane) {
  const int64_t bytes =
      static_cast<int64_t>(a.num_queries) * kQHeads * kDim * (a.out_bf16 ? 2 : 4);
  float4* d = reinterpret_cast<float4*>(static_cast<uint8_t*>(a.out) + b * bytes);
#pragma unroll 4
  for (int i = lane; i < bytes / 16; i += 32) d[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// Output rows of (sequence b, kv head g).
template <bool kBf16>
__device__ __forceinline__ OutRowsT<kBf16> out_rows(const DecodeArgs& a, int b, int g) {
  const int64_t e = (static_cast<int64_t>(b) * a.num_queries * kQHeads + g * kGroup) * kDim;
  using T = typename std::conditional<kBf16, __nv_bfloat16, float>::type;
  return OutRowsT<kBf16>{static_cast<T*>(a.out) + e, kQHeads * kDim};
}

// Split-KV merge staging: the merge kernel copies the records of a
// (sequence, kv head) unit from the workspace into shared memory with
// cp.async (L2 only: the records were written by the decode grid just
// before), all of them in one round when they fit, so that the merge waits
// for a single L2 round trip instead of one per batch of register loads.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Split-KV bookkeeping of sequence b: the CTA range of its first page and
// its number of pieces (CTAs its pages span).  Partial records live at
// [g][b + cta], so the pieces of one (sequence, kv head) unit are the
// consecutive slots S0 .. S0 + K - 1 with S0 = g * (B + grid) + b + c_first
// (b + cta is distinct for every piece of head g because both only grow
// along the page order).
__device__ __forceinline__ int2 split_of(int64_t pages_before, int b, int np, int64_t chunk) {
  if (np == 0) return make_int2(0, 0);
  const int64_t first = pages_before + static_cast<int64_t>(kSeqCost) * b + kSeqCost;
  const int c_first = static_cast<int>(first / chunk);
  return make_int2(c_first, static_cast<int>((first + np - 1) / chunk) - c_first + 1);
}

// Pages per CTA range: every sequence costs its pages plus kSeqCost, the
// total is cut into `grid` equal ranges (at least min_chunk pages).
__device__ __forceinline__ int64_t range_chunk(int64_t total_pages, int batch, int grid,
                                               int min_chunk) {
  const int64_t total = total_pages + static_cast<int64_t>(kSeqCost) * batch;
  int64_t chunk = (total + grid - 1) / grid;
  if (chunk < min_chunk) chunk = min_chunk;
  return chunk < 1 ? 1 : chunk;
}

// End of a sequence's piece inside this CTA's range, for kv head g (= this
// warp): finish it in registers when the CTA holds the whole sequence, else
// store the piece for the merge kernel that follows.
template <class C>
__device__ __forceinline__ void flush_unit(const C& cmp, const DecodeArgs& a,
                                           const int32_t* s_pfx, int b, int g, int j0, int j1,
                                           int np, int64_t chunk, int lane) {
  if (j0 == 0 && j1 == np - 1) {
    if (a.out_bf16)
      cmp.finalize(out_rows<true>(a, b, g), lane);
    else
      cmp.finalize(out_rows<false>(a, b, g), lane);
    return;
  }
  const int64_t slot = static_cast<int64_t>(g) * (a.batch + gridDim.x) + b + blockIdx.x;
  cmp.store_partial(a.partials + slot * a.num_queries * kPartialFloats, a.num_queries, lane);
}

// Producer-side description of page f (this lane's slot of a 32-page batch):
// physical page, and (sequence << kInfoSeqShift) | kInfoRecent (one of the
// sequence's last two pages) | kInfoLast (its last page) | kInfoStart
// (starts a sequence in this range).
// A range of at most kS + kShortRest pages prefetches, once its dependency
// wait is over, all its pages beyond the stages into L2.
constexpr int kShortRest = 4;

constexpr int32_t kInfoStart = 1, kInfoLast = 2, kInfoRecent = 4;
constexpr int kInfoSeqShift = 3;

__device__ __forceinline__ void load_page_batch(const DecodeArgs& a, const int32_t* s_pfx,
                                                int32_t f, int32_t f_begin, int32_t f_end,
                                                int32_t& phys, int32_t& info) {
  phys = -1;
  info = 0;
  if (f < f_end) {
    int b, j;
    locate(s_pfx, a.batch, f, b, j);
    phys = __ldg(a.bt + static_cast<int64_t>(b) * a.max_blocks + j);
    const int np = s_pfx[b + 1] - s_pfx[b];
    info = (b << kInfoSeqShift) | (j >= np - 2 ? kInfoRecent : 0) |
           (j == np - 1 ? kInfoLast : 0) | ((j == 0 || f == f_begin) ? kInfoStart : 0);
  }
}

template <class C>
struct SmemPlan {
  static constexpr int S = C::kStages;
  static constexpr size_t stages = 0;   // [S][page 32 KiB | query rows 4 KiB]
  static constexpr int kStageBytes = StageLayout<C::kMaxQueries>::kBytes;
  static constexpr size_t scratch = stages + size_t(S) * kStageBytes;
  static constexpr size_t full = scratch + size_t(kWarps) * C::kScratch;
  static constexpr size_t empty = full + size_t(S) * 8;
  static constexpr size_t flags = empty + size_t(S) * 8;   // [S] bad page, [1] abort
  static constexpr size_t phys = flags + size_t(S + 1) * 4;  // [S] physical page of the stage
  static constexpr size_t tot = phys + size_t(S) * 4;        // [kWarps] scan totals
  static constexpr size_t lens = tot + size_t(kWarps) * 4;
  static size_t bytes(int32_t batch) {
    // lengths [B] and page-count prefix [B+1], plus 1024 B of alignment slack
    return lens + size_t(batch) * 4 + size_t(batch + 1) * 4 + 1024;
  }
};

// kTable: the batch is above kMergeScanMaxBatch, so the merge kernel reads
// its splits from a table this kernel writes (a separate instantiation, so
// that smaller batches run exactly the code without it).
template <class C, bool kTable>
__device__ __forceinline__ void decode_body(const CUtensorMap& tmap, const DecodeArgs& a) {
  constexpr int kS = C::kStages;
  using L = SmemPlan<C>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int B = a.batch;
  volatile int32_t* s_flags = reinterpret_cast<int32_t*>(smem + L::flags);
  volatile int32_t* s_phys = reinterpret_cast<int32_t*>(smem + L::phys);
  const bool fused = a.k_new != nullptr;
  const int nq = a.num_queries;   // <= C::kMaxQueries (the host picks the variant)
  int32_t* s_len = reinterpret_cast<int32_t*>(smem + L::lens);
  int32_t* s_pfx = s_len + B;
  const uint32_t base = smem_addr(smem);
  const uint32_t full = base + L::full, empty = base + L::empty;
  const uint32_t scratch = base + L::scratch + warp * C::kScratch;

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < kS; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, kWarps);
      s_flags[s] = 0;
    }
    s_flags[kS] = 0;
    fence_mbar_init();
  }
  // With kLaunchEarlyTables the lengths and block tables are read before the
  // preceding kernels of the stream have finished (the caller guarantees
  // they do not write them); q, the pool and the outputs only after.  With
  // kLaunchEarlyPages as well, the loads of the first kS pages go out before
  // then too, except for pages among a sequence's last two (see below; the
  // caller guarantees nothing still running writes the others); their query
  // rows and new-token rows only after.
  const bool early = (a.flags & kLaunchEarlyTables) != 0;
  const bool early_pages = early && (a.flags & kLaunchEarlyPages) != 0;
  if (!early) pdl_wait();
  pdl_trigger();
  cta_lengths(a, s_len, s_pfx, reinterpret_cast<int32_t*>(smem + L::tot));
  __syncthreads();

  const int G = gridDim.x;
  const int64_t total = seq_cost(s_pfx, B);
  const int64_t chunk = range_chunk(s_pfx[B], B, G, a.min_chunk);
  const int64_t x0 = static_cast<int64_t>(blockIdx.x) * chunk;
  const int32_t p0 = x0 < total ? pages_below(s_pfx, B, x0) : 0;
  const int32_t p1 = x0 < total ? pages_below(s_pfx, B, x0 + chunk) : 0;
  const int n = p1 - p0;

  // ---- producer (warp 0): page descriptions for batches k (cur), k+1 (nxt)
  int32_t cur_phys = -1, cur_info = 0, nxt_phys = -1, nxt_info = 0;
  int cur_k = 0;
  uint64_t policy = 0;
  if (warp == 0 && n > 0) {
    policy = l2_evict_first_policy();
    load_page_batch(a, s_pfx, p0 + lane, p0, p1, cur_phys, cur_info);
    load_page_batch(a, s_pfx, p0 + 32 + lane, p0, p1, nxt_phys, nxt_info);
  }
  // Issue page r into stage r % kS (warp 0 only; stage known to be free):
  // kIssuePage arms the stage's full barrier with all its bytes and starts
  // the page's TMA load; kIssueRows starts the bulk copies of the query rows
  // (first page of a sequence in this range) and of the new token's rows
  // (fused append, last page of a sequence).  A first-batch page (r < 32)
  // may take the two parts at different times.
  // Test-only: leave page 0's full barrier unarmed, so the consumers' bounded
  // waits run out and the launch reports PKV_ERR_DEVICE_TIMEOUT.
  constexpr int kIssuePage = 1, kIssueRows = 2;
  const bool stall = (a.flags & kLaunchTestStall) != 0;
  int issued = 0;   // pages issued so far (warp 0)
  auto issue = [&](int r, int part) {
    if (part & kIssuePage) {
      ++issued;
      if ((r >> 5) != cur_k) {
        cur_phys = nxt_phys;
        cur_info = nxt_info;
        ++cur_k;
        load_page_batch(a, s_pfx, p0 + 32 * (cur_k + 1) + lane, p0, p1, nxt_phys, nxt_info);
      }
    }
    const int32_t phys = __shfl_sync(kFull, cur_phys, r & 31);
    const int32_t info = __shfl_sync(kFull, cur_info, r & 31);
    if (lane == 0 && !(stall && r == 0)) {
      const int st = r % kS;
      const uint32_t bar = full + 8 * st;
      const uint32_t dst = base + L::stages + st * L::kStageBytes;
      const bool ok = static_cast<uint32_t>(phys) < static_cast<uint32_t>(a.num_pages);
      const bool start = info & kInfoStart;
      const bool append = fused && (info & kInfoLast);
      const int64_t seq = info >> kInfoSeqShift;
      const uint32_t rows = (start ? nq * kQRowsBytes : 0) + (append ? kNewRowsBytes : 0);
      if (part & kIssuePage) {
        s_flags[st] = ok ? 0 : 1;
        s_phys[st] = phys;
        if (!ok) record_error(a.err, kErrBadPage);
        const uint32_t bytes = (ok ? kPageBytes : 0) + rows;
        if (bytes) {
          mbar_arrive_expect_tx(bar, bytes);
          if (ok) tma_load_tile(dst, &tmap, 0, phys * kRowsPerPage, bar, policy);
        } else {
          mbar_arrive(bar);
        }
      }
      if (part & kIssueRows) {
        if (start)
          bulk_load(dst + kPageBytes, a.q + seq * nq * kQHeads * kDim, nq * kQRowsBytes, bar);
        if (append) {
          const uint32_t nd = dst + kPageBytes + nq * kQRowsBytes;
          bulk_load(nd, a.k_new + seq * kKvHeads * kDim, kNewRowsBytes / 2, bar);
          bulk_load(nd + kNewRowsBytes / 2, a.v_new + seq * kKvHeads * kDim, kNewRowsBytes / 2,
                    bar);
        }
      }
    }
  };
  // Early loads skip a sequence's last two pages: a kernel still running
  // before this one may write the newest tokens there (a fused decode or an
  // append of this layer at an earlier step: one token per step, so the
  // last 16 steps' tokens lie in those two pages).  early_mask: pages r < kS
  // whose page part went out early.
  uint32_t early_mask = 0;
  if (warp == 0 && early_pages)
    for (int r = 0; r < n && r < kS; ++r)
      if (!(__shfl_sync(kFull, cur_info, r & 31) & kInfoRecent)) {
        issue(r, kIssuePage);
        early_mask |= 1u << r;
      }
  if (early) pdl_wait();

  // Large batches: publish the split sequence whose first piece this CTA
  // holds -- the range's last sequence, if it starts in the range and
  // continues past it -- for the merge kernel (after the wait: the previous
  // merge on this workspace reads the table until then).
  if (kTable && threadIdx.x == 0) {
    int2 e = make_int2(-1, 0);
    if (n > 0) {
      int bl, jl;
      locate(s_pfx, B, p1 - 1, bl, jl);
      if (s_pfx[bl] >= p0 && s_pfx[bl + 1] > p1)
        e = make_int2(bl, split_of(s_pfx[bl], bl, s_pfx[bl + 1] - s_pfx[bl], chunk).y);
    }
    a.split_table[blockIdx.x] = e;
  }

  // empty (or invalid) sequences: zero output rows, once across the grid
  for (int b = blockIdx.x * kWarps + warp; b < B; b += G * kWarps)
    if (s_pfx[b + 1] == s_pfx[b]) zero_rows(a, b, lane);
  if (n <= 0) return;
  if (warp == 0) {
    for (int r = 0; r < n && r < kS; ++r)
      issue(r, (early_mask >> r) & 1u ? kIssueRows : kIssuePage | kIssueRows);
    // A short range spends most of its time starting up: its pages beyond
    // the stages would each wait for a stage to free before their load even
    // starts.  So they all go to L2 now, and the stage loads that follow hit
    // there.  Longer ranges reach the steady state of the two-stage pipeline,
    // where extra requests only delay other CTAs' loads (measured: prefetching
    // ahead on every range is much slower on short-context batches).
    if (n <= kS + kShortRest)
      for (int r = kS; r < n; ++r) {   // r < 32: a first-batch page
        const int32_t phys = __shfl_sync(kFull, cur_phys, r);
        if (lane == 0 && static_cast<uint32_t>(phys) < static_cast<uint32_t>(a.num_pages))
          bulk_prefetch_l2(a.pool + static_cast<int64_t>(phys) * (kPageBytes / 2), kPageBytes);
      }
  }
  // After a timed-out wait: wait (bounded) for the copies still in flight
  // into this CTA's stages, pages k0 .. issued-1, before the CTA exits.
  auto drain = [&](int k0) {
    if (warp != 0) return;
    for (int k = k0; k < issued; ++k)
      if (!(stall && k == 0))
        mbar_wait_bounded(full + 8 * (k % kS), static_cast<uint32_t>(k / kS) & 1u);
  };

  // ---- consumers (all 8 warps; warp g computes kv head g)
  int b, j;
  locate(s_pfx, B, p0, b, j);
  int np = s_pfx[b + 1] - s_pfx[b];
  int Lb = s_len[b];
  int j_first = j;
  bool need_q = true;
  C cmp;

  for (int r = 0; r < n; ++r) {
    const int st = r % kS;
    if (warp == 0 && r >= 1 && r - 1 + kS < n) {
      // refill the stage that page r - 1 used, once every warp released it
      const int rr = r - 1;
      const uint32_t eb = empty + 8 * (rr % kS);
      const uint32_t par = static_cast<uint32_t>(rr / kS) & 1u;
      if (!mbar_try_wait(eb, par) && !mbar_wait_bounded(eb, par)) {
        if (lane == 0) record_error(a.err, kErrTimeout);
        s_flags[kS] = 1;
        drain(r);
        return;
      }
      issue(rr + kS, kIssuePage | kIssueRows);
    }
    const uint32_t fb = full + 8 * st;
    const uint32_t par = static_cast<uint32_t>(r / kS) & 1u;
    if (!mbar_try_wait(fb, par) && !mbar_wait_bounded(fb, par)) {
      if (lane == 0) record_error(a.err, kErrTimeout);
      s_flags[kS] = 1;
      drain(r + 1);
      return;
    }
    if (s_flags[kS]) {   // another warp gave up; results are void
      drain(r + 1);
      return;
    }
    const uint32_t stage = base + L::stages + st * L::kStageBytes;
    if (need_q) {
      cmp.begin(stage + kPageBytes, warp, nq, lane);
      need_q = false;
    }
    if (fused && j == np - 1) {
      // the appended token: slot (Lb - 1) % 16 of this, the sequence's last
      // page; lanes 0..7 move the K row of head `warp`, lanes 8..15 its V row
      if (lane < 16) {
        const int kv = lane >> 3, c = lane & 7;
        const int slot = (Lb - 1) % kTokens;
        const uint4 v = lds128(stage + kPageBytes + nq * kQRowsBytes + kv * (kNewRowsBytes / 2) +
                               warp * kRowBytes + c * 16);
        const int row = kv * (kKvHeads * kTokens) + warp * kTokens + slot;
        sts128(stage + swz(row, c), v);
        if (!s_flags[st]) {
          const int64_t prow = static_cast<int64_t>(s_phys[st]) * kRowsPerPage + row;
          reinterpret_cast<uint4*>(a.pool)[prow * (kRowBytes / 16) + c] = v;
        }
        // the stage is refilled by TMA (async proxy) after this generic write
        fence_proxy_async_smem();
      }
      __syncwarp();
    }
    if (!s_flags[st]) {
      // tokens from this page's first slot to the end of the (last query's) context
      const int rem = Lb - kTokens * j;
      const uint32_t ktile = stage + warp * kTileBytes;
      cmp.consume(ktile, ktile + kKvHeads * kTileBytes, scratch, rem, a.scale_log2, lane);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + 8 * st);
    if (j == np - 1 || r == n - 1) {
      flush_unit(cmp, a, s_pfx, b, warp, j_first, j, np, chunk, lane);
      if (r < n - 1) {
        do {
          ++b;
        } while (s_pfx[b + 1] == s_pfx[b]);
        j = 0;
        j_first = 0;
        np = s_pfx[b + 1] - s_pfx[b];
        Lb = s_len[b];
        need_q = true;
      }
    } else {
      ++j;
    }
  }
}

template <class C, bool kTable>
__global__ void __launch_bounds__(kWarps * 32, C::kMinBlocks)
    decode_kernel(const __grid_constant__ CUtensorMap tmap, const DecodeArgs a) {
  decode_body<C, kTable>(tmap, a);
}

// The one-query tensor-core variant needs no more than 88 registers per
// thread without spilling.  Capped there, its two CTAs per SM leave 20,480
// of the SM's 65,536 registers free: room for one merge CTA (256 threads at
// up to 80 registers) beside them.  A merge CTA waiting for its decode
// grid then no longer keeps the next layer's decode CTAs off its SM, so
// that decode's first page loads (PKV_LAUNCH_EARLY_PAGES) overlap the merge.
constexpr int kQ1Regs = 88;

template <bool kTable>
__global__ void __maxnreg__(kQ1Regs)
    decode_kernel_q1(const __grid_constant__ CUtensorMap tmap, const DecodeArgs a) {
  decode_body<MmaComputeT<1, true>, kTable>(tmap, a);
}

// ---------------------------------------------------------------------------
// Split-KV merge: one CTA per (kv head g, unit) for the (sequence, kv head)
// units that decode split into K > 1 pieces.  Up to kMergeScanMaxBatch
// sequences the grid is (8, batch) and each CTA recomputes its sequence's
// split from the lengths (an input that nothing in the launch writes),
// before waiting for the decode grid, so that with programmatic dependent
// launch only the partial records are read after decode ends.  Above, the
// grid is (8, decode CTAs) and CTA (g, c) reads, after the wait, the split
// table entry decode CTA c wrote: the set-up no longer reads every length in
// every one of 8 x batch CTAs.
//
// The merge itself is the fixed-order log-sum-exp combination of the unit's
// pieces s = 0 .. K-1 (in piece order), per head h of the group:
//   M[h] = max_s m_s[h],  w_s[h] = exp2(m_s[h] - M[h]) (0 where m_s = -inf),
//   S[h] = sum_s w_s[h] l_s[h],  out[h][d] = (sum_s w_s[h] acc_s[h][d]) / S[h]
// (zero where S == 0).  The records are staged in shared memory `chunk` at a
// time (one round for every unit of up to `chunk` pieces; a running max
// rescales between rounds).  Per round, warp h < 4 computes head h's weights
// (lane s holds pieces s and s + 32) and the round's share of S; then each of
// the 256 threads accumulates one output element (h, d) over the round's
// pieces in order.
// ---------------------------------------------------------------------------
constexpr int kMergeThreads = kGroup * kDim;   // one output element per thread
constexpr int kMergeWarps = kMergeThreads / 32;
constexpr int kMergeMaxChunk = 64;             // pieces per round: at most two per lane
constexpr int kMergeMinChunk = 8;
constexpr int kRec16 = kPartialFloats * 4 / 16;   // 16-byte copies per record
// shared memory per staged piece: its record and its kGroup weights
constexpr int kMergePieceSmem = (kPartialFloats + kGroup) * 4;
static_assert(kMergeThreads == 256 && kPartialFloats % 4 == 0, "merge layout");

// Three CTAs' worth of registers per SM (at most 85 per thread): one merge
// CTA fits beside two one-query decode CTAs (see decode_kernel_q1), and the
// host sizes `chunk` so that its shared memory fits there too.
// kNq: queries per sequence, 0 = read from the arguments; kTable: splits
// from decode's table (batches above kMergeScanMaxBatch), else from the
// lengths.
template <int kNq, bool kBf16, bool kTable>
__global__ void __launch_bounds__(kMergeThreads, 3)
    merge_kernel(const DecodeArgs a, int32_t decode_grid, int32_t chunk) {
  extern __shared__ __align__(16) float s_rec[];   // [chunk][kPartialFloats], then [chunk][kGroup]
  __shared__ int32_t s_sum[2][kMergeWarps];
  __shared__ float s_scale[kGroup], s_inv[kGroup];
  pdl_trigger();
  const int g = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int b, K, c_first;
  if constexpr (!kTable) {
    // CTA (g, b): sequence b's split, from the lengths
    b = blockIdx.y;
    const int64_t cap = static_cast<int64_t>(a.max_blocks) * kTokens;
    int before = 0, all = 0;
    for (int i = threadIdx.x; i < a.batch; i += blockDim.x) {
      int L = a.seq_lens[i];
      if (L < 0 || L > cap || (L > 0 && L < a.num_queries)) L = 0;
      const int np = (L + kTokens - 1) / kTokens;
      all += np;
      before += (i < b) ? np : 0;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      before += __shfl_xor_sync(kFull, before, off);
      all += __shfl_xor_sync(kFull, all, off);
    }
    if (lane == 0) {
      s_sum[0][warp] = before;
      s_sum[1][warp] = all;
    }
    __syncthreads();
    int64_t pages_before = 0, pages_all = 0;
#pragma unroll
    for (int k = 0; k < kMergeWarps; ++k) {
      pages_before += s_sum[0][k];
      pages_all += s_sum[1][k];
    }
    int Lb = a.seq_lens[b];
    if (Lb < 0 || Lb > cap || (Lb > 0 && Lb < a.num_queries)) Lb = 0;
    const int64_t range = range_chunk(pages_all, a.batch, decode_grid, a.min_chunk);
    const int2 sp = split_of(pages_before, b, (Lb + kTokens - 1) / kTokens, range);
    K = sp.y;
    c_first = sp.x;
    // This grid's completion is what the next programmatically dependent
    // launch waits for, so it must imply decode's: CTA (0, 0) always waits
    // for the decode grid; the other CTAs without work leave at once,
    // freeing their SM slot for the next launch.
    if (K <= 1 && (g | b) != 0) return;
    pdl_wait();   // the pieces are written by the decode grid
  } else {
    // CTA (g, c): the split sequence whose first piece decode CTA c holds,
    // from the table decode wrote (every CTA waits: the table comes from
    // the decode grid)
    pdl_wait();
    c_first = blockIdx.y;
    const int2 e = __ldcg(&a.split_table[c_first]);
    b = e.x;
    K = e.y;
    if (b < 0) return;
  }
  if (K <= 1) return;
  const int nq = kNq > 0 ? kNq : a.num_queries;   // kNq == 0: any count
  const int64_t S0 = static_cast<int64_t>(g) * (a.batch + decode_grid) + b + c_first;
  const OutRowsT<kBf16> out = out_rows<kBf16>(a, b, g);
  float* s_w = s_rec + static_cast<size_t>(chunk) * kPartialFloats;
  const int h = threadIdx.x / kDim, d = threadIdx.x % kDim;   // this thread's output element
  for (int qi = 0; qi < nq; ++qi) {   // a piece's record of query qi: slot * nq + qi
    float M = -INFINITY, S = 0.f;     // warp h < kGroup: head h's running max and sum
    float O = 0.f;
    for (int c0 = 0; c0 < K; c0 += chunk) {
      const int n = min(chunk, K - c0);
      const float* src = a.partials + ((S0 + c0) * nq + qi) * kPartialFloats;
      for (int i = threadIdx.x; i < n * kRec16; i += kMergeThreads) {
        const int s = i / kRec16, o = 4 * (i - s * kRec16);
        cp_async16(smem_addr(s_rec + s * kPartialFloats + o),
                   src + static_cast<int64_t>(s) * nq * kPartialFloats + o);
      }
      cp_async_wait_all();
      __syncthreads();
      if (warp < kGroup) {   // head `warp`: weights of this round's pieces, rescale, sum
        const bool has0 = lane < n, has1 = lane + 32 < n;
        const float* r0 = s_rec + lane * kPartialFloats + warp;
        const float* r1 = s_rec + (lane + 32) * kPartialFloats + warp;
        const float m0 = has0 ? r0[0] : -INFINITY, m1 = has1 ? r1[0] : -INFINITY;
        float mc = fmaxf(m0, m1);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mc = fmaxf(mc, __shfl_xor_sync(kFull, mc, off));
        const float mn = fmaxf(M, mc);
        // a piece whose pages were all skipped has m = -inf and weight 0
        const float scale = (mn == -INFINITY) ? 1.f : fast_exp2(M - mn);
        const float w0 = (m0 == -INFINITY) ? 0.f : fast_exp2(m0 - mn);
        const float w1 = (m1 == -INFINITY) ? 0.f : fast_exp2(m1 - mn);
        if (has0) s_w[lane * kGroup + warp] = w0;
        if (has1) s_w[(lane + 32) * kGroup + warp] = w1;
        float sc = fmaf(w1, has1 ? r1[kGroup] : 0.f, w0 * (has0 ? r0[kGroup] : 0.f));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sc += __shfl_xor_sync(kFull, sc, off);
        S = fmaf(S, scale, sc);
        M = mn;
        if (lane == 0) s_scale[warp] = scale;
      }
      __syncthreads();
      O *= s_scale[h];
      const float* acc = s_rec + 2 * kGroup + h * kDim + d;
#pragma unroll 4
      for (int s = 0; s < n; ++s) O = fmaf(s_w[s * kGroup + h], acc[s * kPartialFloats], O);
      __syncthreads();   // the next round (or query) restages s_rec, s_w and s_scale
    }
    if (warp < kGroup && lane == 0) s_inv[warp] = S > 0.f ? 1.f / S : 0.f;
    __syncthreads();
    out.put(qi, h, d, O * s_inv[h]);
  }
}

// ---------------------------------------------------------------- host side --

using MergeFn = void (*)(const DecodeArgs, int32_t, int32_t);

// The merge kernel for (queries per sequence, BF16 output, split table).
static MergeFn merge_fn(int nq, bool bf16, bool table) {
  if (table)
    return nq == 1 ? (bf16 ? merge_kernel<1, true, true> : merge_kernel<1, false, true>)
                   : (bf16 ? merge_kernel<0, true, true> : merge_kernel<0, false, true>);
  return nq == 1 ? (bf16 ? merge_kernel<1, true, false> : merge_kernel<1, false, false>)
                 : (bf16 ? merge_kernel<0, true, false> : merge_kernel<0, false, false>);
}

// The kernel that runs compute type C.
template <class C, bool kTable>
static auto decode_fn() {
  if constexpr (std::is_same_v<C, MmaComputeT<1, true>>)
    return &decode_kernel_q1<kTable>;
  else
    return &decode_kernel<C, kTable>;
}

template <class C, bool kTable = false>
static const void* kernel_ptr() {
  return reinterpret_cast<const void*>(decode_fn<C, kTable>());
}

// Tensor-core variants by queries per sequence: 1 (its own, fastest),
// 2 (one n-tile), 3-4, 5-6, 7-8 (two to four n-tiles).
using MmaQ1 = MmaComputeT<1, true>;
using MmaQ2 = MmaComputeT<1, false>;
using MmaQ4 = MmaComputeT<2, false>;
using MmaQ6 = MmaComputeT<3, false>;
using MmaQ8 = MmaComputeT<4, false>;

// Calls f with a value of the compute type that serves (kernel, nq); false
// if there is none.
template <class F>
static bool with_compute(int kernel, int nq, F&& f) {
  if (kernel == PKV_KERNEL_SIMT) {
    if (nq != 1) return false;
    f(SimtCompute{});
    return true;
  }
  if (kernel != PKV_KERNEL_MMA || nq < 1 || nq > kMaxQueries) return false;
  if (nq == 1) f(MmaQ1{});
  else if (nq == 2) f(MmaQ2{});
  else if (nq <= 4) f(MmaQ4{});
  else if (nq <= 6) f(MmaQ6{});
  else f(MmaQ8{});
  return true;
}

static const void* kernel_for(int kernel, int nq, bool table = false) {
  const void* fn = nullptr;
  with_compute(kernel, nq, [&](auto c) {
    fn = table ? kernel_ptr<decltype(c), true>() : kernel_ptr<decltype(c), false>();
  });
  return fn;
}

static size_t smem_for(int kernel, int nq, int32_t batch) {
  size_t bytes = 0;
  with_compute(kernel, nq, [&](auto c) { bytes = SmemPlan<decltype(c)>::bytes(batch); });
  return bytes;
}

cudaError_t prepare_decode_kernels(int device) {
  int optin = 0;
  cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
  if (e != cudaSuccess) return e;
  for (const void* fn : {kernel_for(PKV_KERNEL_SIMT, 1), kernel_for(PKV_KERNEL_MMA, 1),
                          kernel_for(PKV_KERNEL_MMA, 2), kernel_for(PKV_KERNEL_MMA, 4),
                          kernel_for(PKV_KERNEL_MMA, 6), kernel_for(PKV_KERNEL_MMA, 8),
                          kernel_for(PKV_KERNEL_SIMT, 1, true), kernel_for(PKV_KERNEL_MMA, 1, true),
                          kernel_for(PKV_KERNEL_MMA, 2, true), kernel_for(PKV_KERNEL_MMA, 4, true),
                          kernel_for(PKV_KERNEL_MMA, 6, true), kernel_for(PKV_KERNEL_MMA, 8, true)}) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, fn);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin - static_cast<int>(fa.sharedSizeBytes));
    if (e != cudaSuccess) return e;
    // all of the SM's unified memory as shared memory, for decode and merge
    // CTAs side by side (the decode kernels read nothing through L1 that
    // needs more than what is left)
    e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
  }
  for (int nq : {1, 2})
    for (bool bf16 : {false, true})
      for (bool table : {false, true}) {
        const void* fn = reinterpret_cast<const void*>(merge_fn(nq, bf16, table));
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kMergeMaxChunk * kMergePieceSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
      }
  return cudaSuccess;
}

int plan_decode(int device, int sm_count, int32_t batch, int kernel, int grid_ctas,
                int num_queries, DecodePlan* plan) {
  if (num_queries < 1 || num_queries > kMaxQueries) return PKV_ERR_UNSUPPORTED;
  if (kernel == PKV_KERNEL_AUTO) kernel = PKV_KERNEL_MMA;
  const void* fn = kernel_for(kernel, num_queries, batch > kMergeScanMaxBatch);
  if (!fn) return PKV_ERR_UNSUPPORTED;
  int optin = 0;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) !=
      cudaSuccess)
    return PKV_ERR_CUDA;
  const size_t smem = smem_for(kernel, num_queries, batch);
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) return PKV_ERR_CUDA;
  if (smem + fa.sharedSizeBytes > static_cast<size_t>(optin)) return PKV_ERR_UNSUPPORTED;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kWarps * 32, smem) != cudaSuccess)
    return PKV_ERR_CUDA;
  if (per_sm < 1) return PKV_ERR_UNSUPPORTED;
  plan->kernel = kernel;
  plan->num_queries = num_queries;
  plan->threads = kWarps * 32;
  plan->smem = smem;
  plan->grid = grid_ctas > 0 ? grid_ctas : sm_count * per_sm;
  const int64_t slots = static_cast<int64_t>(kKvHeads) * (batch + plan->grid);
  plan->records_bytes = static_cast<size_t>(slots) * num_queries * kPartialFloats * sizeof(float);
  plan->ws_bytes = plan->records_bytes + static_cast<size_t>(plan->grid) * sizeof(int2);
  // Merge rounds: as many pieces as fit in the shared memory an SM has left
  // beside its decode CTAs (so that a merge CTA can wait there while decode
  // runs), within [kMergeMinChunk, kMergeMaxChunk].
  int sm_smem = 0, reserved = 0;
  if (cudaDeviceGetAttribute(&sm_smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor, device) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, device) !=
          cudaSuccess)
    return PKV_ERR_CUDA;
  cudaFuncAttributes mfa;
  if (cudaFuncGetAttributes(&mfa, reinterpret_cast<const void*>(merge_fn(1, false, false))) !=
      cudaSuccess)
    return PKV_ERR_CUDA;
  const int64_t left = static_cast<int64_t>(sm_smem) -
                       static_cast<int64_t>(per_sm) * (smem + fa.sharedSizeBytes + reserved) -
                       reserved - static_cast<int64_t>(mfa.sharedSizeBytes);
  const int64_t fit = left / kMergePieceSmem;
  plan->merge_chunk = static_cast<int>(fit < kMergeMinChunk   ? kMergeMinChunk
                                       : fit > kMergeMaxChunk ? kMergeMaxChunk
                                                              : fit);
  plan->merge_smem = static_cast<size_t>(plan->merge_chunk) * kMergePieceSmem;
  return PKV_OK;
}

template <class C>
static cudaError_t launch_one(const DecodePlan& plan, const CUtensorMap& tmap, const DecodeArgs& a,
                              int flags, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.grid);
  cfg.blockDim = dim3(plan.threads);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (flags & kLaunchPdl) ? 1 : 0;
  return a.batch > kMergeScanMaxBatch ? cudaLaunchKernelEx(&cfg, decode_fn<C, true>(), tmap, a)
                                      : cudaLaunchKernelEx(&cfg, decode_fn<C, false>(), tmap, a);
}

cudaError_t launch_decode(const DecodePlan& plan, const CUtensorMap& tmap, const DecodeArgs& a,
                          int flags, cudaStream_t stream) {
  cudaError_t e = cudaErrorInvalidValue;
  with_compute(plan.kernel, plan.num_queries,
               [&](auto c) { e = launch_one<decltype(c)>(plan, tmap, a, flags, stream); });
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kKvHeads, a.batch <= kMergeScanMaxBatch ? a.batch : plan.grid);
  cfg.blockDim = dim3(kMergeThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (flags & kLaunchPdl) ? 1 : 0;
  cfg.dynamicSmemBytes = plan.merge_smem;
  return cudaLaunchKernelEx(&cfg, merge_fn(a.num_queries, a.out_bf16, a.batch > kMergeScanMaxBatch),
                            a, static_cast<int32_t>(plan.grid),
                            static_cast<int32_t>(plan.merge_chunk));
}

}  // namespace pkv
