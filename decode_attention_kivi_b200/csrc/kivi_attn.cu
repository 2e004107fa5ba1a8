// kivi_attn.cu - fused single-token decode attention over the packed KIVI cache.
//
// For query head h of sequence b (kv head h / (Hq/Hkv)), over all S cached tokens:
//   s_t = sm_scale * <q, k_t>,  out = sum_t softmax(s)_t v_t,
// where k_t, v_t are the dequantized codes (scale_h * code + min_h) of the
// NG(S)*32 grouped tokens and the bf16 residual ring for the rest (record
// "kv-efficiency/kivi-2bit-llama3-8b-gqa-8k", "KV bytes basis": the most recent
// R tokens stay full precision).  Grouped history and residual share one
// online softmax.
//
// Work: one persistent CTA per SM.  The work of a (sequence, kv head) pair is a
// list of items: pairs of group records (64 tokens), a last single record, and
// residual items of 8 ring tokens.  The items of all pairs, in order, are split
// into one contiguous range per CTA, balanced by their bytes.  Inside a CTA the
// items of one pair form a segment; each segment gets its own group of warps
// (sized by the segment's cost), and the warps of a group claim its items from
// the segment's counter, so warps that run ahead take more.  Each warp streams
// its items into its own two-item shared-memory ring with cp.async.bulk on
// mbarriers and keeps one online-softmax state.  A warp that has to move to
// another pair (only when a CTA holds more segments than warps; then every pair
// of the CTA belongs to one warp) finishes the pair it leaves from its
// registers.  At the end the last warp of each segment's group to finish merges
// the group's final states on its own (no CTA-wide barrier, so it overlaps the
// other groups' items).
// A pair held whole goes to the output; for a pair shared with other CTAs the
// CTA writes a partial, and the last CTA to arrive (a ticket per pair) merges
// the partials into the output.
//
// Group records, on the tensor cores (mma.sync m16n8k16, fp16 operands, fp32
// accumulation):
//   scores  C[token][head] = sum_d code[token][d] * (q''[head][d] * kscale[d])
//                          + sum_d kmin[d] * q''[head][d]
//           with q'' * kscale carried as an fp16 pair hi + lo (the two halves of
//           the exact product of two fp16 numbers) in adjacent columns;
//   P.V     C[chan][head] += sum_t code[t][chan] * (p[head][t] * vscale[t][j])
//                          + sum_t vmin[t][j] * p[head][t]
//           with p * vscale carried as hi + lo as well: p is split into fp16
//           hi + lo, and for up to four heads per kv head the lo parts use the
//           four columns the heads leave free.
// The codes turn into exact fp16 operands with the sm_100a conversions of
// packed small floats: one mask spreads eight 2-bit codes into nibbles, and one
// conversion turns a byte of two nibbles into two fp16 values c/2 (4-bit codes:
// a byte holds one code, the value is c/8).  The scale and the min fold into
// the other operand, so nothing is dequantized element by element; the
// constant factor 1/2 (1/8) is undone in fp32.  q'' = q * 2^-e_h (exact) keeps
// |q''| < 1 so q'' * kscale stays in fp16 range; scores are rescaled by
// 2^e_h * sm_scale * log2(e) in fp32.
//
// Residual items: 8 bf16 ring tokens on the tensor cores in bf16 (exact
// products): scores with q itself, P.V with p as a bf16 hi + lo pair in the two
// halves of the k dimension.
//
// Every wait is bounded: a wait on an mbarrier that runs out sets the device
// status word and the warp stops issuing work; the CTA still finishes its
// bookkeeping so that no other CTA waits on it.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kivi_kernels.h"
#include "kivi_launch.cuh"
#include "kivi_ptx.cuh"
#include "kivi_layout.cuh"

namespace kivi {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kStatusWaitTimeout = 1u;
constexpr uint32_t kStatusBadSplit = 4u;
constexpr uint32_t kStatusBounds = 8u;  // debug build: an index outside its buffer (access skipped)

#ifdef KIVI_DEBUG_BUILD
// Debug build only: bytes added to every expected copy size, so that a test can
// make the bounded waits run out while every issued copy still lands whole.
__device__ unsigned g_kivi_debug_overstate = 0u;
__device__ __forceinline__ uint32_t debug_overstate() { return g_kivi_debug_overstate; }
#else
__device__ __forceinline__ uint32_t debug_overstate() { return 0u; }
#endif
constexpr int kResTok = 8;             // residual tokens per item
constexpr int kPRow = 2 * 32 + 8;      // p tile row (fp16 entries): 64 tokens + 8 padding
constexpr int kGridBase = 256;         // CTAs at most, before the pair-slot bound
constexpr int kSmemBudget = 227 * 1024;
#ifndef KIVI_ITEM_SLOTS
#define KIVI_ITEM_SLOTS 2
#endif
#ifndef KIVI_MAX_WARPS
#define KIVI_MAX_WARPS 12  // measured: 12 warps per SM beat 16 (and 14, 11, 10)
#endif

// ---------------------------------------------------------------------------
// Codes -> exact fp16 operands
// ---------------------------------------------------------------------------

// Byte K of x holds two e2m1 values (2-bit codes in the low bits of its
// nibbles): fp16x2 (low nibble / 2, high nibble / 2).
template <int K>
__device__ __forceinline__ uint32_t e2m1_byte(uint32_t x) {
  uint32_t d;
  if constexpr (K == 0)
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t}" : "=r"(d) : "r"(x));
  else if constexpr (K == 1)
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b1;\n\t}" : "=r"(d) : "r"(x));
  else if constexpr (K == 2)
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b2;\n\t}" : "=r"(d) : "r"(x));
  else
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b3;\n\t}" : "=r"(d) : "r"(x));
  return d;
}

// Half-word K of x holds two e2m3 values (4-bit codes in the low nibbles of its
// bytes): fp16x2 (low byte / 8, high byte / 8).
template <int K>
__device__ __forceinline__ uint32_t e2m3_half(uint32_t x) {
  uint32_t d;
  if constexpr (K == 0)
    asm("{\n\t.reg .b16 h0, h1;\n\tmov.b32 {h0, h1}, %1;\n\t"
        "cvt.rn.f16x2.e2m3x2 %0, h0;\n\t}" : "=r"(d) : "r"(x));
  else
    asm("{\n\t.reg .b16 h0, h1;\n\tmov.b32 {h0, h1}, %1;\n\t"
        "cvt.rn.f16x2.e2m3x2 %0, h1;\n\t}" : "=r"(d) : "r"(x));
  return d;
}

// A operands of k-step SL of a K-code word pair (rows g and g + 8): a0..a3,
// from the words already masked into nibbles (2 bits: m0 = w & 0x33333333 and
// m2 = (w >> 2) & 0x33333333; 4 bits: m0 = w & 0x0F0F0F0F, m2 = (w >> 4) & ...).
template <int BITS, int SL>
__device__ __forceinline__ void key_operands(uint32_t m0, uint32_t m2, uint32_t n0, uint32_t n2,
                                             uint32_t (&a)[4]) {
  if constexpr (BITS == 2) {
    // byte SL: codes j = 0 (bits 0-1), 1 (4-5) -> a0; j = 2 (2-3), 3 (6-7) -> a2
    a[0] = e2m1_byte<SL>(m0);
    a[2] = e2m1_byte<SL>(m2);
    a[1] = e2m1_byte<SL>(n0);
    a[3] = e2m1_byte<SL>(n2);
  } else {
    // nibble SL of every byte j: half-word 0 -> (j0, j1) = a0, half-word 1 -> a2
    const uint32_t x = SL == 0 ? m0 : m2, y = SL == 0 ? n0 : n2;
    a[0] = e2m3_half<0>(x);
    a[2] = e2m3_half<1>(x);
    a[1] = e2m3_half<0>(y);
    a[3] = e2m3_half<1>(y);
  }
}

template <int BITS>
__device__ __forceinline__ void key_masks(uint32_t w, uint32_t& m0, uint32_t& m2) {
  if constexpr (BITS == 2) {
    m0 = w & 0x33333333u;
    m2 = (w >> 2) & 0x33333333u;
  } else {
    m0 = w & 0x0F0F0F0Fu;
    m2 = (w >> 4) & 0x0F0F0F0Fu;
  }
}

// A operands (a0..a3) of k-step kk of V-code m-tile: 2 bits from lane word x
// (both k-steps), 4 bits from the k-step's own word.
template <int BITS>
__device__ __forceinline__ void value_operands(uint32_t x, int kk, uint32_t (&a)[4]) {
  if constexpr (BITS == 2) {
    const uint32_t y = (x >> (2 * kk)) & 0x33333333u;  // byte r + 2 hf
    a[0] = e2m1_byte<0>(y);
    a[1] = e2m1_byte<1>(y);
    a[2] = e2m1_byte<2>(y);
    a[3] = e2m1_byte<3>(y);
  } else {
    const uint32_t lo = x & 0x0F0F0F0Fu, hi = (x >> 4) & 0x0F0F0F0Fu;  // r = 0, 1
    a[0] = e2m3_half<0>(lo);
    a[2] = e2m3_half<1>(lo);
    a[1] = e2m3_half<0>(hi);
    a[3] = e2m3_half<1>(hi);
  }
}

// ---------------------------------------------------------------------------
// Configuration and shared-memory plan
// ---------------------------------------------------------------------------

__host__ __device__ constexpr int round_up(int x, int m) { return (x + m - 1) / m * m; }
__host__ __device__ constexpr int cmin_i(int a, int b) { return a < b ? a : b; }

template <int D, int BITS, int HPK>
struct Cfg {
  static constexpr RecordGeom geo{D, BITS};
  static constexpr int kRec = (int)geo.bytes();          // multiple of 128
  static constexpr int kItemBytes = 2 * kRec;             // two records, or 8 K + 8 V rows
  static constexpr int kItemSlots = KIVI_ITEM_SLOTS;        // items in a warp's ring
  static constexpr int kResRow = 2 * D + 16;              // padded residual row (bank spread)
  static_assert(kResTok * kResRow <= kRec, "residual rows must fit in one record's space");
  static constexpr int kChunks = HPK > 4 ? 2 : 1;         // score column chunks of 4 heads
  static constexpr bool kLoCols = HPK <= 4;               // P.V lo parts in the free columns
  static constexpr int kCodeShift = BITS == 2 ? 1 : 3;    // operands are code / 2^shift
  // p tile rows: heads' p_hi, then -p_lo (<= 4 heads) or p_lo (8 heads), then a zero row
  static constexpr int kPRows = 2 * HPK + (kLoCols ? 1 : 0);
  static constexpr int kZeroRow = 2 * HPK;
  static constexpr int kWarpBytes = round_up(kItemSlots * kItemBytes + kPRows * kPRow * 2, 128);
  static constexpr int kSlotBytes = HPK * D * 2;          // a pair's q (bf16)
  static constexpr int kStateFloats = HPK * (D + 2);      // m[HPK], l[HPK], acc[HPK][D]
  static_assert(kStateFloats * 4 <= kItemSlots * kItemBytes, "a warp's final state fits its item slots");
  static constexpr int kMinSlots = 4;
  static constexpr int kFixed = 2048;                     // mbarriers, counters, masks
  // warps per CTA: a multiple of 4, so that the four schedulers of an SM hold
  // the same number of warps
  static constexpr int kNW =
      cmin_i(HPK > 4 ? cmin_i(8, KIVI_MAX_WARPS) : KIVI_MAX_WARPS,
             (kSmemBudget - kFixed - kMinSlots * kSlotBytes) / kWarpBytes) / 4 * 4;
  static constexpr int kThreads = kNW * 32;
  static constexpr int kSlots =
      cmin_i(64, (kSmemBudget - kFixed - kNW * kWarpBytes) / kSlotBytes);
  static_assert(kNW >= 4 && kNW <= 32 && kSlots >= kMinSlots, "shared-memory plan");
  static_assert(8 * kItemSlots * kNW + 16 + 8 * kNW + 20 * kSlots <= kFixed, "fixed area");
  static constexpr int kOffSlots = kNW * kWarpBytes;
  static constexpr int kOffFixed = kOffSlots + kSlots * kSlotBytes;
  static constexpr int kBytes = kOffFixed + kFixed;
  // item costs for the split between CTAs: bytes read / 512 + 1
  static constexpr int kCostG2 = 2 * kRec / 512 + 1;
  static constexpr int kCostG1 = kRec / 512 + 1;
  static constexpr int kCostR = kResTok * D * 4 / 512 + 1;
};

// ---------------------------------------------------------------------------
// The split of the items between CTAs
// ---------------------------------------------------------------------------

// Items of one pair: n2 record pairs, n1 (0 or 1) single record, nr residual
// items; costs c2, c1, cr.  The CTA ranges cut the concatenated cost axis of
// all pairs into n equal parts: CTA c owns [lo(c), lo(c+1)) with
// lo(c) = c*q + min(c, rem), and the items whose cost interval starts there.
struct Split {
  int pairs, ipp, n2, n1, nr, NG;
  int c2, c1, cr, pc;  // item costs, cost per pair
  int n, q, rem;       // CTAs and the division of pairs*pc among them
  unsigned long long ipp_inv;  // ceil(2^64 / ipp) for ipp >= 2: x / ipp = umulhi64(x, ipp_inv)
};

// Pair of global item `it` (0 <= it < 2^31): one 64-bit high multiply instead of
// a division by the runtime value ipp.
__device__ __forceinline__ int pair_of(const Split& s, int it) {
  return s.ipp == 1 ? it : (int)__umul64hi((unsigned long long)it, s.ipp_inv);
}

__host__ __device__ inline int cost_lo(const Split& s, int c) {
  return c * s.q + (c < s.rem ? c : s.rem);
}

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// First item whose cost interval starts at or after cost x (global item index).
__host__ __device__ inline int first_item_at(const Split& s, int x) {
  const int p = x / s.pc, w = x % s.pc;
  int k;
  if (w <= s.n2 * s.c2) {
    k = ceil_div(w, s.c2);
  } else if (w <= s.n2 * s.c2 + s.n1 * s.c1) {
    k = s.n2 + ceil_div(w - s.n2 * s.c2, s.c1);
  } else {
    k = s.n2 + s.n1 + ceil_div(w - s.n2 * s.c2 - s.n1 * s.c1, s.cr);
  }
  return p * s.ipp + k;  // k == ipp is item 0 of pair p + 1
}

__host__ __device__ inline int cta_first_item(const Split& s, int c) {
  return first_item_at(s, cost_lo(s, c));
}

// Start of global item `it` (it <= pairs * ipp) on the cost axis.
__host__ __device__ inline int item_cost_start(const Split& s, int it) {
  const int p = it / s.ipp, k = it % s.ipp;
  int cs = p * s.pc;
  if (k <= s.n2) cs += k * s.c2;
  else if (k <= s.n2 + s.n1) cs += s.n2 * s.c2 + (k - s.n2) * s.c1;
  else cs += s.n2 * s.c2 + s.n1 * s.c1 + (k - s.n2 - s.n1) * s.cr;
  return cs;
}

// The CTA that owns global item `it`.
__host__ __device__ inline int cta_of_item(const Split& s, int it) {
  const int cs = item_cost_start(s, it);
  const int big = s.rem * (s.q + 1);
  return cs < big ? cs / (s.q + 1) : s.rem + (cs - big) / s.q;
}

// ---------------------------------------------------------------------------
// The decode kernel
// ---------------------------------------------------------------------------

template <int D, int BITS, int HPK>
struct Warp;  // per-warp state and item processing (below)

template <int D, int BITS, int HPK>
struct Warp {
  using C = Cfg<D, BITS, HPK>;
  static constexpr RecordGeom geo = C::geo;
  static constexpr int kChunks = C::kChunks;
  static constexpr int kKSteps = D / 16;             // score k-steps (16 channels each)
  static constexpr int kMTiles = D / 16;             // P.V m-tiles (16 channels each)
  static constexpr int kBlocks = D / 32;             // value channel blocks j
  static constexpr int kLaneWordsK = D * BITS / 128;  // K-code words of one quad lane per row
  static constexpr int kStepsPerWord = 8 / BITS;
  static constexpr int kVWords = kMTiles * BITS / 2;  // V-code words of one lane per record

  const DecodeArgs& a;
  const int lane, g, tig;
  // online softmax state of the current pair: heads 4c + tig
  float m_run[kChunks], l_run[kChunks];
  float acc[kMTiles][4];  // (channel 16mt + g (+8), column 2tig + e)
  float vmacc[4];         // value-min term: (row g -> block g % kBlocks, column 2tig + e)
  // score B operands of the current pair: q'' split so that one fma gives hi or lo
  uint32_t qa[kChunks][kKSteps][2], qb[kChunks][kKSteps][2];
  float ch[kChunks];      // log2 score scale of head 4c + tig
  float qscale;           // sm_scale * log2(e)
  const __nv_bfloat16* q_pair;  // the pair's q (HPK x D, global memory)
  unsigned char* p_tile;  // this warp's p tile
  int rowA, rowX, rowR;   // p tile rows this lane reads (byte offsets)
  uint32_t maskY, signY, maskHi;

  __device__ Warp(const DecodeArgs& args, int lane_, float qs)
      : a(args), lane(lane_), g(lane_ >> 2), tig(lane_ & 3), qscale(qs) {}

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      m_run[c] = -INFINITY;
      l_run[c] = 0.f;
    }
#pragma unroll
    for (int mt = 0; mt < kMTiles; ++mt)
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[mt][r] = 0.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) vmacc[r] = 0.f;
  }

  // The pair's q (bf16 in shared memory): the score B operands and scales.
  __device__ __forceinline__ void load_pair(const __nv_bfloat16* qs) {
    q_pair = qs;
    // per-head exponent e_h with max |q_h| 2^-e_h in [0.5, 1): lanes of head hs
    // (g = 2hs', 2hs'+1 in chunk c) each scan the head's D/4 channels of quad lane tig
    int e_h[kChunks];
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      const int hs = 4 * c + g / 2;
      float mx = 0.f;
      if (hs < HPK) {
#pragma unroll
        for (int s = 0; s < kKSteps; ++s) {
          const uint2 v = *reinterpret_cast<const uint2*>(qs + hs * D + 16 * s + 4 * tig);
          const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.x));
          const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.y));
          mx = fmaxf(mx, fmaxf(fmaxf(fabsf(f0.x), fabsf(f0.y)), fmaxf(fabsf(f1.x), fabsf(f1.y))));
        }
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      int e = 0;
      if (mx > 0.f) frexpf(mx, &e);
      e_h[c] = e;
      const float sc = ldexpf(1.f, -e);
      const bool lo = (g & 1) != 0;
#pragma unroll
      for (int s = 0; s < kKSteps; ++s) {
        uint32_t qq0 = 0u, qq1 = 0u;
        if (hs < HPK) {
          const uint2 v = *reinterpret_cast<const uint2*>(qs + hs * D + 16 * s + 4 * tig);
          const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.x));
          const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.y));
          qq0 = pack_half2(f0.x * sc, f0.y * sc);
          qq1 = pack_half2(f1.x * sc, f1.y * sc);
        }
        // hi column: qa = 0, qb = q''  -> fma(0, ks, RN(q'' ks)) = hi
        // lo column: qa = q'', qb = -q'' -> fma(q'', ks, -RN(q'' ks)) = lo
        qa[c][s][0] = lo ? qq0 : 0u;
        qa[c][s][1] = lo ? qq1 : 0u;
        qb[c][s][0] = lo ? (qq0 ^ 0x80008000u) : qq0;
        qb[c][s][1] = lo ? (qq1 ^ 0x80008000u) : qq1;
      }
    }
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      // exponent of head 4c + tig: held by the lanes with g = 2 tig
      const int e = __shfl_sync(0xffffffffu, e_h[c], 8 * tig);
      ch[c] = 4 * c + tig < HPK ? ldexpf(qscale, e + C::kCodeShift) : 1.f;
    }
  }

  // Shares of alpha for the accumulator columns 2tig + e of this lane.
  __device__ __forceinline__ void col_factors(const float (&f)[kChunks], float (&out)[2]) const {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int col = 2 * tig + e;
      const int h = C::kLoCols ? (col & 3) : col;
      const int src = (lane & ~3) | (h & 3);
      float v = __shfl_sync(0xffffffffu, f[0], src);
      if constexpr (kChunks == 2) {
        const float v1 = __shfl_sync(0xffffffffu, f[kChunks - 1], src);
        v = h >= 4 ? v1 : v;
      }
      out[e] = v;
    }
  }

  __device__ __forceinline__ void rescale(const float (&alpha)[kChunks]) {
    bool same = true;
#pragma unroll
    for (int c = 0; c < kChunks; ++c) same = same && alpha[c] == 1.f;
    if (__all_sync(0xffffffffu, same)) return;
    float al[2];
    col_factors(alpha, al);
#pragma unroll
    for (int mt = 0; mt < kMTiles; ++mt) {
      acc[mt][0] *= al[0];
      acc[mt][1] *= al[1];
      acc[mt][2] *= al[0];
      acc[mt][3] *= al[1];
    }
    vmacc[0] *= al[0];
    vmacc[1] *= al[1];
    vmacc[2] *= al[0];
    vmacc[3] *= al[1];
  }

  // Stores p (fp32, head 4c + tig, column col of the tile) as fp16 hi and
  // (negated for <= 4 heads) lo.
  __device__ __forceinline__ void store_p(int c, int col, float p) {
    const int h = 4 * c + tig;
    if (h >= HPK) return;
    const __half hi = __float2half_rn(p);
    const float r = C::kLoCols ? __half2float(hi) - p : p - __half2float(hi);
    __half* t = reinterpret_cast<__half*>(p_tile) + col;
    t[h * kPRow] = hi;
    t[(HPK + h) * kPRow] = __float2half_rn(r);
  }

  __device__ __forceinline__ uint32_t lds32(const unsigned char* p) const {
    return *reinterpret_cast<const uint32_t*>(p);
  }

  // MMAs of the k-steps SL.. of one K-code word pair into acc
  template <int SL>
  __device__ __forceinline__ void score_steps(uint32_t m0, uint32_t m2, uint32_t n0, uint32_t n2,
                                              const uint32_t (&bq)[kChunks][kStepsPerWord][2],
                                              float (&acc_)[kChunks][4]) {
    if constexpr (SL < kStepsPerWord) {
      uint32_t ka[4];
      key_operands<BITS, SL>(m0, m2, n0, n2, ka);
#pragma unroll
      for (int c = 0; c < kChunks; ++c)
        mma_f16(acc_[c], ka[0], ka[1], ka[2], ka[3], bq[c][SL][0], bq[c][SL][1]);
      score_steps<SL + 1>(m0, m2, n0, n2, bq, acc_);
    }
  }

  // ---- one item of one or two group records ----
  __device__ __forceinline__ void groups(const unsigned char* rec0, bool has_b) {
    const unsigned char* recs[2] = {rec0, has_b ? rec0 + C::kRec : rec0};

    // key-min term of both groups: rows g <- group A, rows g+8 <- group B
    float cmin[kChunks][4];
#pragma unroll
    for (int c = 0; c < kChunks; ++c)
#pragma unroll
      for (int r = 0; r < 4; ++r) cmin[c][r] = 0.f;
    {
      const __half* kmA = reinterpret_cast<const __half*>(recs[0] + geo.k_min_off());
      const __half* kmB = reinterpret_cast<const __half*>(recs[1] + geo.k_min_off());
#pragma unroll
      for (int s = 0; s < kKSteps; ++s) {
        const int c0 = 16 * s + 4 * tig;
        const uint2 x = *reinterpret_cast<const uint2*>(kmA + c0);
        const uint2 y = *reinterpret_cast<const uint2*>(kmB + c0);
#pragma unroll
        for (int c = 0; c < kChunks; ++c) mma_f16(cmin[c], x.x, y.x, x.y, y.y, qb[c][s][0], qb[c][s][1]);
      }
    }
    // scores in units of 2^-kCodeShift: sc[grp][c][mt][row half]
    constexpr float kInv = 1.f / (1 << C::kCodeShift);
    float sc[2][kChunks][2][2];
#pragma unroll
    for (int grp = 0; grp < 2; ++grp) {
      const unsigned char* rec = recs[grp];
      const __half* kscale = reinterpret_cast<const __half*>(rec + geo.k_scale_off());
      float cacc[2][kChunks][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          // a missing second group scores -inf: p = 0, the max is unchanged
          cacc[mt][c][0] = cacc[mt][c][2] = (grp == 1 && !has_b) ? -INFINITY : cmin[c][2 * grp] * kInv;
          cacc[mt][c][1] = cacc[mt][c][3] = 0.f;
        }
#pragma unroll
      for (int w = 0; w < kLaneWordsK; ++w) {
        uint32_t bq[kChunks][kStepsPerWord][2];
#pragma unroll
        for (int sl = 0; sl < kStepsPerWord; ++sl) {
          const int s = w * kStepsPerWord + sl;
          const uint2 ks = *reinterpret_cast<const uint2*>(kscale + 16 * s + 4 * tig);
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
            bq[c][sl][0] = hfma2(qa[c][s][0], ks.x, hmul2(qb[c][s][0], ks.x));
            bq[c][sl][1] = hfma2(qa[c][s][1], ks.y, hmul2(qb[c][s][1], ks.y));
          }
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const uint32_t* row = reinterpret_cast<const uint32_t*>(rec) +
                                (16 * mt + g) * geo.k_row_words() + tig * kLaneWordsK + w;
          uint32_t m0, m2, n0, n2;
          key_masks<BITS>(row[0], m0, m2);
          key_masks<BITS>(row[8 * geo.k_row_words()], n0, n2);
          score_steps<0>(m0, m2, n0, n2, bq, cacc[mt]);
        }
      }
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          sc[grp][c][mt][0] = cacc[mt][c][0] + cacc[mt][c][1];  // token 16mt + g, head 4c + tig
          sc[grp][c][mt][1] = cacc[mt][c][2] + cacc[mt][c][3];  // token 16mt + g + 8
        }
    }

    // ---- online softmax over the 64 tokens, head 4c + tig (log2 units) ----
    float alpha[kChunks];
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      // max of the raw MMA scores (ch > 0 keeps the order), then log2 units
      float mx = fmaxf(fmaxf(fmaxf(sc[0][c][0][0], sc[0][c][0][1]),
                             fmaxf(sc[0][c][1][0], sc[0][c][1][1])),
                       fmaxf(fmaxf(sc[1][c][0][0], sc[1][c][0][1]),
                             fmaxf(sc[1][c][1][0], sc[1][c][1][1])));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float m_new = fmaxf(m_run[c], mx * ch[c]);
      alpha[c] = fast_exp2(m_run[c] - m_new);
      m_run[c] = m_new;
      float sum = 0.f;
#pragma unroll
      for (int grp = 0; grp < 2; ++grp)
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int hr = 0; hr < 2; ++hr) {
            const float pv = fast_exp2(fmaf(sc[grp][c][mt][hr], ch[c], -m_new));
            sum += pv;
            store_p(c, grp * kGroup + 16 * mt + 8 * hr + g, pv);
          }
      l_run[c] = l_run[c] * alpha[c] + sum;
    }
    __syncwarp();
    rescale(alpha);

    // ---- P.V of both groups ----
#pragma unroll
    for (int grp = 0; grp < 2; ++grp) {
      const unsigned char* rec = recs[grp];
      const __half* vscale = reinterpret_cast<const __half*>(rec + geo.v_scale_off());
      const __half* vmin = reinterpret_cast<const __half*>(rec + geo.v_min_off());
      // p of tokens (16kk + 8hf + 2tig, +1) for this lane's B column
      uint32_t pa[2][2], px[2][2];
#pragma unroll
      for (int kk = 0; kk < 2; ++kk)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const uint32_t col = (uint32_t)(grp * kGroup + 16 * kk + 8 * hf + 2 * tig) * 2;
          pa[kk][hf] = lds32(p_tile + rowA + col);
          px[kk][hf] = lds32(p_tile + rowX + col);
        }
      // this lane's V-code words
      const uint32_t* vw = reinterpret_cast<const uint32_t*>(rec + geo.v_codes_off()) + lane * 4;
      uint32_t vwords[kVWords];
#pragma unroll
      for (int q4 = 0; q4 < kVWords / 4; ++q4) {
        const uint4 x = *reinterpret_cast<const uint4*>(vw + q4 * 128);
        vwords[4 * q4] = x.x;
        vwords[4 * q4 + 1] = x.y;
        vwords[4 * q4 + 2] = x.z;
        vwords[4 * q4 + 3] = x.w;
      }
      // value-min term: rows g -> block g % kBlocks
      {
        const uint4 vm = *reinterpret_cast<const uint4*>(vmin + 32 * (g % kBlocks) + 8 * tig);
        if constexpr (C::kLoCols) {
          // hi columns: p_hi; lo columns: -p_lo
          mma_f16(vmacc, vm.x, vm.x, vm.y, vm.y, and_or(pa[0][0], maskHi, px[0][0]),
                  and_or(pa[0][1], maskHi, px[0][1]));
          mma_f16(vmacc, vm.z, vm.z, vm.w, vm.w, and_or(pa[1][0], maskHi, px[1][0]),
                  and_or(pa[1][1], maskHi, px[1][1]));
        } else {
          mma_f16(vmacc, vm.x, vm.x, vm.y, vm.y, pa[0][0], pa[0][1]);
          mma_f16(vmacc, vm.z, vm.z, vm.w, vm.w, pa[1][0], pa[1][1]);
          mma_f16(vmacc, vm.x, vm.x, vm.y, vm.y, px[0][0], px[0][1]);
          mma_f16(vmacc, vm.z, vm.z, vm.w, vm.w, px[1][0], px[1][1]);
        }
      }
#pragma unroll
      for (int j = 0; j < kBlocks; ++j) {
        const uint4 vs4 = *reinterpret_cast<const uint4*>(vscale + 32 * j + 8 * tig);
        const uint32_t vs[2][2] = {{vs4.x, vs4.y}, {vs4.z, vs4.w}};
        uint32_t pt[2][2], pl[2][2];
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            if constexpr (C::kLoCols) {
              // hi columns: RN(p_hi vs); lo columns: -RN(p_lo vs + (p_hi vs - hi))
              const uint32_t y = and_xor(pa[kk][hf], maskY, signY);
              pt[kk][hf] = hfma2(px[kk][hf], vs[kk][hf],
                                 hfma2(y, vs[kk][hf], hmul2(pa[kk][hf], vs[kk][hf])));
            } else {
              const uint32_t nhi = hmul2(pa[kk][hf] ^ 0x80008000u, vs[kk][hf]);
              pl[kk][hf] = hfma2(px[kk][hf], vs[kk][hf], hfma2(pa[kk][hf], vs[kk][hf], nhi));
              pt[kk][hf] = nhi ^ 0x80008000u;
            }
          }
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
          const int mt = 2 * j + mi;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            uint32_t va[4];
            value_operands<BITS>(BITS == 2 ? vwords[mt] : vwords[2 * mt + kk], kk, va);
            mma_f16(acc[mt], va[0], va[1], va[2], va[3], pt[kk][0], pt[kk][1]);
            if constexpr (!C::kLoCols)
              mma_f16(acc[mt], va[0], va[1], va[2], va[3], pl[kk][0], pl[kk][1]);
          }
        }
      }
    }
  }

  // ---- one residual item: n (1..8) ring tokens, K rows then V rows (padded) ----
  __device__ __forceinline__ void residual(unsigned char* base, int n) {
    const uint32_t kbase = smem_addr(base), vbase = smem_addr(base + C::kRec);
    if (n < kResTok) {  // rows past the last token: zero V (0 * stale data must stay 0)
      constexpr int kVec = 2 * D / 16;
      for (int i = lane; i < (kResTok - n) * kVec; i += 32) {
        const int t = n + i / kVec, c = i % kVec;
        *reinterpret_cast<uint4*>(base + C::kRec + t * C::kResRow + 16 * c) =
            make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async();  // the slot's next bulk copy comes after these writes
      __syncwarp();
    }
    // scores: rows = tokens (0..7), columns 2h = head 4c + h (q in bf16), 2h+1 = 0
    float sacc[kChunks][4];
#pragma unroll
    for (int c = 0; c < kChunks; ++c)
#pragma unroll
      for (int r = 0; r < 4; ++r) sacc[c][r] = 0.f;
    const int mrow = lane & 7, mat = lane >> 3;
#pragma unroll
    for (int s = 0; s < kKSteps; s += 2) {
      uint32_t kf[4];  // (s: a0, a2), (s+1: a0, a2)
      ldsm_x4(kf, kbase + mrow * C::kResRow + (16 * (s + mat / 2) + 8 * (mat % 2)) * 2);
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
        const int h = 4 * c + g / 2;
        const bool live = (g % 2) == 0 && h < HPK;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int ch0 = 16 * (s + u) + 2 * tig;
          const uint32_t b0 = live ? *reinterpret_cast<const uint32_t*>(q_pair + h * D + ch0) : 0u;
          const uint32_t b1 =
              live ? *reinterpret_cast<const uint32_t*>(q_pair + h * D + ch0 + 8) : 0u;
          mma_bf16(sacc[c], kf[2 * u], 0u, kf[2 * u + 1], 0u, b0, b1);
        }
      }
    }
    // online softmax: one token (g) per lane, head 4c + tig
    float alpha[kChunks];
    constexpr float kInv = 1.f / (1 << C::kCodeShift);
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      const float x = g < n ? sacc[c][0] * qscale : -INFINITY;
      float mx = x;
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float m_new = fmaxf(m_run[c], mx);
      alpha[c] = fast_exp2(m_run[c] - m_new);
      m_run[c] = m_new;
      const float pv = fast_exp2(x - m_new);
      l_run[c] = l_run[c] * alpha[c] + pv;
      // p / 2^shift as bf16 hi (tile columns 0..7) + lo (8..15): the accumulators
      // hold the group terms in units of 2^-shift as well
      const int h = 4 * c + tig;
      if (h < HPK) {
        const float ps = pv * kInv;
        const __nv_bfloat16 hi = __float2bfloat16_rn(ps);
        const __nv_bfloat16 lo = __float2bfloat16_rn(ps - __bfloat162float(hi));
        __nv_bfloat16* row = reinterpret_cast<__nv_bfloat16*>(p_tile) + h * kPRow;
        row[g] = hi;
        row[8 + g] = lo;
      }
    }
    __syncwarp();
    rescale(alpha);
    // P.V: A = V^T (channels x tokens) from ldmatrix.trans; k = 0..7 with p_hi,
    // k = 8..15 the same tokens with p_lo
    const uint32_t b0 = lds32(p_tile + rowR + 2 * tig * 2);
    const uint32_t b1 = lds32(p_tile + rowR + (8 + 2 * tig) * 2);
#pragma unroll
    for (int mt = 0; mt < kMTiles; mt += 2) {
      uint32_t vf[4];  // (mt: a0, a1), (mt+1: a0, a1)
      ldsm_x4_trans(vf, vbase + mrow * C::kResRow + (16 * (mt + mat / 2) + 8 * (mat % 2)) * 2);
      mma_bf16(acc[mt], vf[0], vf[1], vf[0], vf[1], b0, b1);
      mma_bf16(acc[mt + 1], vf[2], vf[3], vf[2], vf[3], b0, b1);
    }
  }
};

// RAGGED: a length per sequence (args.lens); otherwise every pair has the split's
// shape and the per-pair checks compile away.
template <int D, int BITS, int HPK, bool RAGGED>
__global__ void __launch_bounds__(Cfg<D, BITS, HPK>::kThreads, 1)
decode_kernel(DecodeArgs args, Split sp) {
  using C = Cfg<D, BITS, HPK>;
  using W = Warp<D, BITS, HPK>;
  extern __shared__ __align__(128) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;

  const int it_begin = cta_first_item(sp, cta), it_end = cta_first_item(sp, cta + 1);
  const int p_first = it_begin / sp.ipp, p_last = (it_end - 1) / sp.ipp;
  const int n_pairs = p_last - p_first + 1;
  unsigned char* wbase = smem + warp * C::kWarpBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffFixed) + C::kItemSlots * warp;
  int* s_ctr = reinterpret_cast<int*>(smem + C::kOffFixed + 8 * C::kItemSlots * C::kNW);
  int* s_final = s_ctr + 4;                          // [kNW] pair (local) of each warp's final state
  int* s_seg_next = s_final + C::kNW;                                  // [kSlots] claim counters
  int* s_seg_end = s_seg_next + C::kSlots;                             // [kSlots] end items
  int* s_gsize = s_seg_end + C::kSlots + C::kNW;  // [kSlots] warps of each segment (after s_warp_seg)
  int* s_done = s_gsize + C::kSlots;              // [kSlots] warps of each segment that finished
  if (it_end <= it_begin || n_pairs > C::kSlots) {  // the host's split rules exclude both
    if (threadIdx.x == 0) atomicOr(args.status, kStatusBadSplit);
    return;
  }

  // ---- set-up: p tiles, mbarriers, masks, the claim counter ----
  {
    uint32_t* pt = reinterpret_cast<uint32_t*>(wbase + C::kItemSlots * C::kItemBytes);
    for (int i = lane; i < C::kPRows * kPRow / 2; i += 32) pt[i] = 0u;
    if (lane == 0) {
      for (int k = 0; k < C::kItemSlots; ++k) mbar_init(&bars[k], 1);
      fence_mbar_init();
      s_final[warp] = -1;
    }
    for (int k = threadIdx.x; k < n_pairs; k += C::kThreads) {
      s_done[k] = 0;
      s_seg_next[k] = max(it_begin, (p_first + k) * sp.ipp);
      s_seg_end[k] = min(it_end, (p_first + k + 1) * sp.ipp);
    }
  }
  // Segments: the items of one pair inside this CTA's range.  With at most kNW
  // segments every segment gets its own group of warps, sized by its cost, so a
  // warp never leaves its pair; with more, each warp sweeps a run of segments.
  // Thread 0 writes each warp's segment range [lo, hi) to s_warp_seg.
  int* s_warp_seg = s_seg_end + C::kSlots;  // [kNW]: lo | hi << 16
  if (threadIdx.x == 0) {
    if (n_pairs <= C::kNW) {
      int cost[C::kNW], wk[C::kNW];
      for (int k = 0; k < n_pairs; ++k) {
        const int a = max(it_begin, (p_first + k) * sp.ipp);
        const int b = min(it_end, (p_first + k + 1) * sp.ipp);
        cost[k] = item_cost_start(sp, b) - item_cost_start(sp, a);
        wk[k] = 1;
      }
      for (int extra = C::kNW - n_pairs; extra > 0; --extra) {  // largest cost per warp first
        int best = 0;
        for (int k = 1; k < n_pairs; ++k)
          if ((long)cost[k] * wk[best] > (long)cost[best] * wk[k]) best = k;
        ++wk[best];
      }
      int ww = 0;
      for (int k = 0; k < n_pairs; ++k) {
        s_gsize[k] = wk[k];
        for (int j = 0; j < wk[k]; ++j, ++ww) s_warp_seg[ww] = k | ((k + 1) << 16);
      }
    } else {
      for (int ww = 0; ww < C::kNW; ++ww)
        s_warp_seg[ww] = (ww * n_pairs / C::kNW) | (((ww + 1) * n_pairs / C::kNW) << 16);
    }
  }
  int seg_cur = 0, seg_hi = 0;  // this warp's segments, read after the barrier below
  const long rec_stride = C::kRec;
  // the items of one pair: n2 record pairs, n1 single records, nr residual items
  // of its own length S_b (the split is laid out for the longest sequence; the
  // items of a shorter one past its own count are empty)
  struct PairShape { int S, NG, n2, n1, nr; };
  auto pair_shape = [&](int pair) -> PairShape {
    if constexpr (!RAGGED) return PairShape{args.S, sp.NG, sp.n2, sp.n1, sp.nr};
    PairShape p;
    p.S = __ldg(args.lens + pair / args.Hkv) + args.steps;
    p.NG = num_groups(p.S);
    p.n2 = p.NG / 2;
    p.n1 = p.NG % 2;
    p.nr = (p.S - p.NG * kGroup + kResTok - 1) / kResTok;
    return p;
  };
  // claims the next item of this warp's segments (warp-uniform; -1 when done)
  auto claim = [&]() -> int {
    while (seg_cur < seg_hi) {
      int it = 0;
      if (lane == 0) it = atomicAdd(&s_seg_next[seg_cur], 1);
      it = __shfl_sync(0xffffffffu, it, 0);
      if (it < s_seg_end[seg_cur]) return it;
      ++seg_cur;
    }
    return -1;
  };
  // starts the copies of item `it` into item slot k: records from lane 0, the
  // rows of a residual item from one lane each (row t of K: lane t, of V: lane 8 + t)
  auto issue = [&](int it, int k) {
    if (it < 0) return;
    unsigned char* dst = wbase + k * C::kItemBytes;
    const int pair = pair_of(sp, it), kk = it - pair * sp.ipp;
    const PairShape ps = pair_shape(pair);
    if (RAGGED && kk >= ps.n2 + ps.n1 + ps.nr) {  // past this sequence's items: nothing to copy
      if (lane == 0) mbar_arrive(&bars[k]);
      return;
    }
    if (kk < ps.n2 + ps.n1) {
      if (lane == 0) {
        const int g0 = 2 * kk;
        const int n_rec = kk < ps.n2 ? 2 : 1;
        const uint32_t bytes = n_rec * C::kRec;
#ifdef KIVI_DEBUG_BOUNDS
        if (pair >= sp.pairs || g0 + n_rec > min(ps.NG, args.ngcap)) {
          atomicOr(args.status, kStatusBounds);
          return;
        }
#endif
        mbar_expect_tx(&bars[k], bytes + debug_overstate());
        bulk_load(dst, args.records + ((long)pair * args.ngcap + g0) * rec_stride, bytes, &bars[k]);
      }
    } else {
      const int t0 = ps.NG * kGroup + kResTok * (kk - ps.n2 - ps.n1);
      const int n = min(kResTok, ps.S - t0);
      const long row0 = (long)pair * kRingSlots + t0 % kRingSlots;
#ifdef KIVI_DEBUG_BOUNDS
      if (pair >= sp.pairs || n < 1 || t0 % kRingSlots + n > kRingSlots) {
        if (lane == 0) atomicOr(args.status, kStatusBounds);
        return;
      }
#endif
      if (lane == 0) mbar_expect_tx(&bars[k], 2u * n * D * 2 + debug_overstate());
      __syncwarp();
      const int t = lane & 7;
      if (lane < 16 && t < n) {
        const bool v = lane >= 8;
        bulk_load(dst + (v ? C::kRec : 0) + t * C::kResRow,
                  (v ? args.ring_v : args.ring_k) + (row0 + t) * D, D * 2, &bars[k]);
      }
    }
  };

  wait_for_predecessor();  // q, the records and the rings may come from the previous kernel
  __syncthreads();         // counters, segment table and mbarriers are set up
  seg_cur = s_warp_seg[warp] & 0xffff;
  seg_hi = s_warp_seg[warp] >> 16;
  int itm[C::kItemSlots];
#pragma unroll
  for (int k = 0; k < C::kItemSlots; ++k) {
    itm[k] = claim();
    issue(itm[k], k);
  }

  const float qscale = (args.sm_scale > 0.f ? args.sm_scale : rsqrtf((float)D)) * kLog2e;
  W w(args, lane, qscale);
  w.p_tile = wbase + C::kItemSlots * C::kItemBytes;
  {
    const int hcol = w.g & 3;
    const bool lo_lane = C::kLoCols && w.g >= 4;
    constexpr int kRowBytes = kPRow * 2;
    if constexpr (C::kLoCols) {
      w.rowA = (hcol < HPK ? hcol : C::kZeroRow) * kRowBytes;
      w.rowX = (lo_lane && hcol < HPK ? HPK + hcol : C::kZeroRow) * kRowBytes;
      w.rowR = (!lo_lane && hcol < HPK ? hcol : C::kZeroRow) * kRowBytes;
    } else {
      w.rowA = w.g * kRowBytes;
      w.rowX = (HPK + w.g) * kRowBytes;
      w.rowR = w.g * kRowBytes;
    }
    w.maskY = lo_lane ? 0xffffffffu : 0u;
    w.signY = lo_lane ? 0x80008000u : 0u;
    w.maskHi = lo_lane ? 0u : 0xffffffffu;
  }
  w.reset();

  // The partial of CTA ct for `pair`: side 0 if the pair is ct's first pair.
  auto partial_of = [&](int ct, int pair) -> float* {
    return args.partials + ((long)ct * 2 + (pair == cta_first_item(sp, ct) / sp.ipp ? 0 : 1)) *
                               (long)(HPK * (D + 2));
  };
  // Merges, with this warp alone, the final states of segment `seg`'s warps (all
  // of them have counted themselves done) and writes the pair's output, or this
  // CTA's partial and the pair's ticket; the CTA that takes the last ticket of a
  // shared pair merges the pair's partials.
  // After this warp wrote its CTA's partial of a shared pair: takes the pair's
  // ticket, and if this CTA is the last of the pair's CTAs to arrive, merges the
  // partials (online, CTA by CTA, all of a lane's elements in flight) into out.
  auto ticket_and_combine = [&](int pair, int fc, int lc, float* out) {
    constexpr int kEl = HPK * D / 32;
    __threadfence();  // the partial before the ticket
    __syncwarp();
    int is_last = 0;
    if (lane == 0) is_last = atomicAdd(&args.tickets[pair], 1) == lc - fc;
    is_last = __shfl_sync(0xffffffffu, is_last, 0);
    if (!is_last) return;
    __threadfence();
    float A[kEl];
    // the pair's partials, CTA by CTA (online), all of a lane's elements at once
    float Mh[HPK], Lh[HPK];
#pragma unroll
    for (int h = 0; h < HPK; ++h) {
      Mh[h] = -INFINITY;
      Lh[h] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < kEl; ++i) A[i] = 0.f;
    for (int ct = fc; ct <= lc; ++ct) {
      const float* pp = partial_of(ct, pair);
      float a[kEl], fo[HPK], fn[HPK];
#pragma unroll
      for (int i = 0; i < kEl; ++i) a[i] = __ldcg(pp + 2 * HPK + lane + 32 * i);
#pragma unroll
      for (int h = 0; h < HPK; ++h) {
        const float m = __ldcg(pp + h), l = __ldcg(pp + HPK + h);
        const float Mn = fmaxf(Mh[h], m);
        fo[h] = Mh[h] == -INFINITY ? 0.f : exp2f(Mh[h] - Mn);
        fn[h] = m == -INFINITY ? 0.f : exp2f(m - Mn);  // a partial without tokens
        Lh[h] = Lh[h] * fo[h] + l * fn[h];
        Mh[h] = Mn;
      }
#pragma unroll
      for (int i = 0; i < kEl; ++i) {
        const int h = (lane + 32 * i) / D;
        A[i] = A[i] * fo[h] + a[i] * fn[h];
      }
    }
#pragma unroll
    for (int i = 0; i < kEl; ++i) out[lane + 32 * i] = A[i] / Lh[(lane + 32 * i) / D];
    if (lane == 0) args.tickets[pair] = 0;  // ready for the next call
  };
  auto merge_segment = [&](int seg) {
    constexpr int kEl = HPK * D / 32;  // elements of a state per lane: e = lane + 32 i
    const int pair = p_first + seg;
    float* tab = reinterpret_cast<float*>(wbase + C::kItemSlots * C::kItemBytes);  // own p tile
    float* s_M = tab + C::kNW * HPK;  // [HPK] merged max, then [HPK] merged sum
    // lane ww < kNW: warp ww's factors 2^(m - M) per head (0 when not in the group)
    const int wl = min(lane, C::kNW - 1);
    const bool member = lane < C::kNW && (s_warp_seg[wl] & 0xffff) == seg && s_final[wl] == seg;
    const unsigned members = __ballot_sync(0xffffffffu, member);
    const float* st = reinterpret_cast<const float*>(smem + wl * C::kWarpBytes);
#pragma unroll
    for (int h = 0; h < HPK; ++h) {
      const float m = member ? st[h] : -INFINITY;
      float M = m;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      // (a segment may hold only empty items of a short sequence: m = M = -inf)
      const float f = member && m != -INFINITY ? exp2f(m - M) : 0.f;
      float L = member ? f * st[HPK + h] : 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
      if (lane < C::kNW) tab[lane * HPK + h] = f;
      if (lane == 0) {
        s_M[h] = M;
        s_M[HPK + h] = L;
      }
    }
    __syncwarp();
    // acc: the member warps one after another, all of a lane's elements at once
    float A[kEl];
#pragma unroll
    for (int i = 0; i < kEl; ++i) A[i] = 0.f;
    for (unsigned mm = members; mm; mm &= mm - 1) {
      const int ww = __ffs(mm) - 1;
      const float* src = reinterpret_cast<const float*>(smem + ww * C::kWarpBytes) + 2 * HPK;
#pragma unroll
      for (int i = 0; i < kEl; ++i) A[i] = fmaf(tab[ww * HPK + (lane + 32 * i) / D], src[lane + 32 * i], A[i]);
    }
    const int fc = cta_of_item(sp, pair * sp.ipp), lc = cta_of_item(sp, pair * sp.ipp + sp.ipp - 1);
    const int b = pair / args.Hkv, kvh = pair % args.Hkv;
    float* out = args.out + ((long)b * args.Hq + (long)kvh * HPK) * D;
    if (fc == lc) {  // held whole by this CTA
#pragma unroll
      for (int i = 0; i < kEl; ++i) out[lane + 32 * i] = A[i] / s_M[HPK + (lane + 32 * i) / D];
      return;
    }
    if (cta >= args.max_ctas) {  // the host's split rules exclude this
      if (lane == 0) atomicOr(args.status, kStatusBadSplit);
      return;
    }
    float* part = partial_of(cta, pair);
#pragma unroll
    for (int i = 0; i < kEl; ++i) part[2 * HPK + lane + 32 * i] = A[i];
    if (lane < HPK) {
      part[lane] = s_M[lane];
      part[HPK + lane] = s_M[HPK + lane];
    }
    ticket_and_combine(pair, fc, lc, out);
  };

  // this warp's state as m[HPK], l[HPK], acc[HPK][D] (fp32) at dst
  auto export_state = [&](float* dst) {
    float lw[C::kChunks];
#pragma unroll
    for (int c = 0; c < C::kChunks; ++c) {
      float l = w.l_run[c];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      lw[c] = l;
    }
    // accumulators: (hi - lo') for <= 4 heads, times 2^shift, plus the value-min term
    float vm[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) vm[r] = w.vmacc[r];
    if constexpr (C::kLoCols) {
#pragma unroll
      for (int r = 0; r < 4; ++r) vm[r] -= __shfl_xor_sync(0xffffffffu, vm[r], 2);
    }
    float vb[W::kBlocks][2];  // value-min term of block j, columns 2tig + e: lane 4j + tig
#pragma unroll
    for (int j = 0; j < W::kBlocks; ++j) {
      vb[j][0] = __shfl_sync(0xffffffffu, vm[0], 4 * j + w.tig);
      vb[j][1] = __shfl_sync(0xffffffffu, vm[1], 4 * j + w.tig);
    }
    const bool valid_lane = C::kLoCols ? w.tig < 2 : true;
#pragma unroll
    for (int mt = 0; mt < W::kMTiles; ++mt) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        float x = w.acc[mt][r];
        if constexpr (C::kLoCols) x -= __shfl_xor_sync(0xffffffffu, x, 2);
        x = x * (float)(1 << C::kCodeShift) + vb[mt / 2][r & 1];
        const int h = 2 * w.tig + (r & 1);
        if (valid_lane && h < HPK) dst[2 * HPK + h * D + 16 * mt + w.g + 8 * (r >> 1)] = x;
      }
    }
#pragma unroll
    for (int c = 0; c < C::kChunks; ++c) {
      const int h = 4 * c + w.tig;
      if (w.g == 0 && h < HPK) {
        dst[h] = w.m_run[c];
        dst[HPK + h] = lw[c];
      }
    }
  };

  // out = acc / l of this warp's state for the HPK heads of a pair (out: the
  // pair's first head, HPK x D fp32), the same elements as export_state
  auto export_output = [&](float* out) {
    float lw[C::kChunks];
#pragma unroll
    for (int c = 0; c < C::kChunks; ++c) {
      float l = w.l_run[c];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      lw[c] = l;  // head 4c + tig
    }
    float inv[2];  // 1 / l of heads 2tig + e (lanes tig < 2 only, for <= 4 heads)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = (2 * w.tig + e) & 7;
      const int src = (lane & ~3) | (h & 3);
      float l = __shfl_sync(0xffffffffu, lw[0], src);
      if constexpr (C::kChunks == 2) {
        const float l1 = __shfl_sync(0xffffffffu, lw[C::kChunks - 1], src);
        l = h >= 4 ? l1 : l;
      }
      inv[e] = 1.f / l;
    }
    float vm[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) vm[r] = w.vmacc[r];
    if constexpr (C::kLoCols) {
#pragma unroll
      for (int r = 0; r < 4; ++r) vm[r] -= __shfl_xor_sync(0xffffffffu, vm[r], 2);
    }
    float vb[W::kBlocks][2];
#pragma unroll
    for (int j = 0; j < W::kBlocks; ++j) {
      vb[j][0] = __shfl_sync(0xffffffffu, vm[0], 4 * j + w.tig);
      vb[j][1] = __shfl_sync(0xffffffffu, vm[1], 4 * j + w.tig);
    }
    const bool valid_lane = C::kLoCols ? w.tig < 2 : true;
#pragma unroll
    for (int mt = 0; mt < W::kMTiles; ++mt) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        float x = w.acc[mt][r];
        if constexpr (C::kLoCols) x -= __shfl_xor_sync(0xffffffffu, x, 2);
        x = x * (float)(1 << C::kCodeShift) + vb[mt / 2][r & 1];
        const int h = 2 * w.tig + (r & 1);
        if (valid_lane && h < HPK) out[h * D + 16 * mt + w.g + 8 * (r >> 1)] = x * inv[r & 1];
      }
    }
  };

  // With more segments than warps every pair of the CTA belongs to one warp:
  // when the warp leaves it, its state is the CTA's whole result for the pair.
  // A pair held whole goes straight to out (acc / l from the registers); the
  // CTA's first or last pair, when shared, goes to the CTA's partial and its
  // ticket.
  auto finish_pair = [&](int pair) {
    const int fc = cta_of_item(sp, pair * sp.ipp), lc = cta_of_item(sp, pair * sp.ipp + sp.ipp - 1);
    const int b = pair / args.Hkv, kvh = pair % args.Hkv;
    float* out = args.out + ((long)b * args.Hq + (long)kvh * HPK) * D;
    if (fc != lc) {
      if (cta >= args.max_ctas) {  // the host's split rules exclude this
        if (lane == 0) atomicOr(args.status, kStatusBadSplit);
        return;
      }
      export_state(partial_of(cta, pair));
      ticket_and_combine(pair, fc, lc, out);
      return;
    }
    export_output(out);
  };

  int cur_pair = -1;
  PairShape cur{};
  bool timed_out = false;
  int i_stop = 0;

  for (int i = 0;; ++i) {
    const int k = i % C::kItemSlots;
    const int it = itm[k];
    if (it < 0) break;
    const int pair = pair_of(sp, it), kk = it - pair * sp.ipp;
    if (pair != cur_pair) {
      if (cur_pair >= 0) {  // (only with more segments than warps)
        finish_pair(cur_pair);
        w.reset();
      }
      // the pair's q (global, HPK x D bf16), read by the warp itself before it
      // waits for the item, so that the two latencies overlap
      w.load_pair(args.q + ((long)(pair / args.Hkv) * args.Hq + (long)(pair % args.Hkv) * HPK) * D);
      cur_pair = pair;
      cur = pair_shape(pair);
    }
    // the next item, claimed now: the counter's latency hides under the item
    const int next = claim();
    const bool arrived = mbar_wait_bounded(&bars[k], (uint32_t)(i / C::kItemSlots) & 1u);
    if (!__all_sync(0xffffffffu, arrived)) {
      timed_out = true;
      i_stop = i;
      break;
    }
    unsigned char* base = wbase + k * C::kItemBytes;
    if (kk < cur.n2 + cur.n1) {
      w.groups(base, kk < cur.n2);
    } else if (!RAGGED || kk < cur.n2 + cur.n1 + cur.nr) {
      const int t0 = cur.NG * kGroup + kResTok * (kk - cur.n2 - cur.n1);
      w.residual(base, min(kResTok, cur.S - t0));
    }  // else: an empty item of a shorter sequence
    // release the item slot and start the next item's copies into it (the only
    // generic writes to a slot, residual rows zeroed, are fenced where they happen)
    __syncwarp();
    itm[k] = next;
    issue(next, k);
  }
  if (timed_out) {
    // record the failure, then give the copies still in flight a bounded chance
    // to land before this CTA's shared memory is reused
    if (lane == 0) {
      atomicOr(args.status, kStatusWaitTimeout);
      for (int j = i_stop; j < i_stop + C::kItemSlots; ++j)
        if (itm[j % C::kItemSlots] >= 0)
          (void)mbar_wait_bounded(&bars[j % C::kItemSlots], (uint32_t)(j / C::kItemSlots) & 1u);
    }
    __syncwarp();
  }
  if (n_pairs <= C::kNW) {
    // the final state goes to this warp's own item slots (no copy is in flight any more)
    if (cur_pair >= 0) {
      export_state(reinterpret_cast<float*>(wbase));
      if (lane == 0) s_final[warp] = cur_pair - p_first;
    }
    // ---- every segment is merged by the last warp of its group to finish: no
    // CTA-wide barrier, so a group's merge overlaps the other groups' items ----
    const int seg = s_warp_seg[warp] & 0xffff;
    __syncwarp();
    __threadfence_block();  // this warp's state and s_final before its count
    int last = 0;
    if (lane == 0) last = atomicAdd(&s_done[seg], 1) == s_gsize[seg] - 1;
    last = __shfl_sync(0xffffffffu, last, 0);
    allow_successor();
    if (!last) return;
    __threadfence_block();
    merge_segment(seg);
    return;
  }
  allow_successor();
  if (cur_pair >= 0) finish_pair(cur_pair);  // the warp's last pair (more segments than warps)
}

// ---------------------------------------------------------------------------
// Launch
// ---------------------------------------------------------------------------

template <int D, int BITS, int HPK>
Split make_split(int pairs, int S, int num_sms) {
  using C = Cfg<D, BITS, HPK>;
  Split s{};
  s.pairs = pairs;
  s.NG = num_groups(S);
  const int r = S - s.NG * kGroup;
  s.n2 = s.NG / 2;
  s.n1 = s.NG % 2;
  s.nr = (r + kResTok - 1) / kResTok;
  s.ipp = s.n2 + s.n1 + s.nr;
  // ceil(2^64 / ipp) = floor((2^64 - 1) / ipp) + 1 for ipp >= 2
  if (s.ipp >= 2) s.ipp_inv = ~0ULL / (unsigned long long)s.ipp + 1;
  s.c2 = C::kCostG2;
  s.c1 = C::kCostG1;
  s.cr = C::kCostR;
  s.pc = s.n2 * s.c2 + s.n1 * s.c1 + s.nr * s.cr;
  const long T = (long)pairs * s.pc;
  // every CTA range must start an item: length >= the largest item cost present
  const int cmax = max(max(s.n2 > 0 ? s.c2 : 0, s.n1 > 0 ? s.c1 : 0), s.nr > 0 ? s.cr : 0);
  const long most = T / cmax > 0 ? T / cmax : 1;
  int n = (int)(most < (long)min(num_sms, kGridBase) ? most : min(num_sms, kGridBase));
  // and span at most kSlots pairs; beyond one wave, whole waves
  const int need = (pairs + C::kSlots - 2) / (C::kSlots - 1);
  if (need > n) n = num_sms > 0 ? (need + num_sms - 1) / num_sms * num_sms : need;
  s.n = max(n, 1);
  s.q = (int)(T / s.n);
  s.rem = (int)(T % s.n);
  return s;
}

template <int D, int BITS, int HPK, bool RAGGED>
cudaError_t launch_decode_r(const DecodeArgs& a, cudaStream_t stream) {
  using C = Cfg<D, BITS, HPK>;
  int unused = 0;
  cudaError_t e = per_device_setup(a.device, &unused, [](int* v) {
    *v = 1;
    cudaError_t r = cudaFuncSetAttribute(decode_kernel<D, BITS, HPK, RAGGED>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kBytes);
    if (r != cudaSuccess) return r;
    return cudaFuncSetAttribute(decode_kernel<D, BITS, HPK, RAGGED>,
                                cudaFuncAttributePreferredSharedMemoryCarveout,
                                (int)cudaSharedmemCarveoutMaxShared);
  });
  if (e != cudaSuccess) return e;
  const long pairs = (long)a.B * a.Hkv;
  if (pairs > (1L << 30) / 4096) return cudaErrorInvalidValue;  // keeps the cost axis in int
  const Split sp = make_split<D, BITS, HPK>((int)pairs, a.S, a.num_sms);
  if ((long)sp.pairs * sp.pc >= (1L << 31) || sp.n > a.max_ctas) return cudaErrorInvalidValue;
  e = launch_pdl(decode_kernel<D, BITS, HPK, RAGGED>, dim3(sp.n), dim3(C::kThreads), C::kBytes,
                 stream, a, sp);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D, int BITS, int HPK>
cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t stream) {
  return a.lens != nullptr ? launch_decode_r<D, BITS, HPK, true>(a, stream)
                           : launch_decode_r<D, BITS, HPK, false>(a, stream);
}

template <int D, int BITS>
cudaError_t launch_decode_d(const DecodeArgs& a, cudaStream_t stream) {
  switch (a.Hq / a.Hkv) {
    case 1: return launch_decode_t<D, BITS, 1>(a, stream);
    case 2: return launch_decode_t<D, BITS, 2>(a, stream);
    case 4: return launch_decode_t<D, BITS, 4>(a, stream);
    case 8: return launch_decode_t<D, BITS, 8>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <int D, int BITS>
int slots_d(int hpk) {
  switch (hpk) {
    case 1: return Cfg<D, BITS, 1>::kSlots;
    case 2: return Cfg<D, BITS, 2>::kSlots;
    case 4: return Cfg<D, BITS, 4>::kSlots;
    case 8: return Cfg<D, BITS, 8>::kSlots;
    default: return 0;
  }
}

template <int D, int BITS>
int grid_d(int hpk, int pairs, int S, int num_sms) {
  switch (hpk) {
    case 1: return make_split<D, BITS, 1>(pairs, S, num_sms).n;
    case 2: return make_split<D, BITS, 2>(pairs, S, num_sms).n;
    case 4: return make_split<D, BITS, 4>(pairs, S, num_sms).n;
    case 8: return make_split<D, BITS, 8>(pairs, S, num_sms).n;
    default: return 0;
  }
}

int pair_slots(int D, int bits, int hpk) {
  if (D == 128 && bits == 2) return slots_d<128, 2>(hpk);
  if (D == 128 && bits == 4) return slots_d<128, 4>(hpk);
  if (D == 64 && bits == 2) return slots_d<64, 2>(hpk);
  if (D == 64 && bits == 4) return slots_d<64, 4>(hpk);
  return 0;
}

}  // namespace

int decode_items(int S) {
  const int NG = num_groups(S);
  return NG / 2 + NG % 2 + (S - NG * kGroup + kResTok - 1) / kResTok;
}

cudaError_t debug_overstate_copies(unsigned bytes) {
#ifdef KIVI_DEBUG_BUILD
  return cudaMemcpyToSymbol(g_kivi_debug_overstate, &bytes, sizeof bytes);
#else
  (void)bytes;
  return cudaErrorNotSupported;
#endif
}

int decode_max_ctas(int D, int bits, int hpk, long pairs) {
  const int slots = pair_slots(D, bits, hpk);
  if (slots < 2) return 0;
  // make_split rounds a grid above one wave up to whole waves: below 2 * need
  const long need = (pairs + slots - 2) / (slots - 1);
  return (int)(2 * need > kGridBase ? 2 * need : kGridBase);
}

int decode_grid_ctas(int D, int bits, int hpk, long pairs, int S, int num_sms) {
  if (pairs < 1 || pairs > (1L << 30) / 4096 || S < 1) return 0;
  if (D == 128 && bits == 2) return grid_d<128, 2>(hpk, (int)pairs, S, num_sms);
  if (D == 128 && bits == 4) return grid_d<128, 4>(hpk, (int)pairs, S, num_sms);
  if (D == 64 && bits == 2) return grid_d<64, 2>(hpk, (int)pairs, S, num_sms);
  if (D == 64 && bits == 4) return grid_d<64, 4>(hpk, (int)pairs, S, num_sms);
  return 0;
}

long decode_partial_bytes(int D, int hpk) { return 2L * hpk * (D + 2) * (long)sizeof(float); }

long decode_workspace_bytes(int D, int bits, int hpk, long pairs) {
  const long ctas = decode_max_ctas(D, bits, hpk, pairs);
  return kWsHeader + ws_tickets_bytes(pairs) + ctas * decode_partial_bytes(D, hpk);
}

cudaError_t launch_decode(int D, int bits, const DecodeArgs& a, cudaStream_t stream) {
  if (D == 128 && bits == 2) return launch_decode_d<128, 2>(a, stream);
  if (D == 128 && bits == 4) return launch_decode_d<128, 4>(a, stream);
  if (D == 64 && bits == 2) return launch_decode_d<64, 2>(a, stream);
  if (D == 64 && bits == 4) return launch_decode_d<64, 4>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace kivi
