// kivi_quant.cuh - the KIVI group quantizer as device code shared by the
// quantize kernels and the prefill-attention epilogue.
//
// The quantizer ("KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV
// Cache"; "asymmetric" also on "KV cache quantization squeezes 5GB down to fit
// longer LLM generations"): zero point = group min, scale = (max - min) /
// (2^b - 1) in IEEE fp32, code = round-half-even((x - min) / scale) clamped to
// [0, 2^b - 1], all codes 0 when scale == 0; the record keeps {fp16 scale,
// fp16 min} rounded to nearest even.  Keys: one group per channel over 32
// tokens.  Values: one group per token over 32 channels.  Explicit _rn
// intrinsics keep every step IEEE round-to-nearest so the codes are
// reproducible bit for bit.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kivi_layout.cuh"

namespace kivi {
namespace quant {

// The value rows are padded by 16 bytes: the per-token parameter loop, whose
// threads read four channel blocks of eight tokens at once, then meets 4-way
// bank conflicts instead of 16-way.
template <int D>
struct QuantSmem {
  static constexpr int kVRow = D + 8;
  __nv_bfloat16 k[kGroup][D];
  __nv_bfloat16 v[kGroup][kVRow];
  uint8_t kc[kGroup][D];
  uint8_t vc[kGroup][D];
};

__device__ __forceinline__ unsigned short to_f16_bits(float x) {
  return __half_as_ushort(__float2half_rn(x));
}

// Codes of one group of values already reduced to (mn, scale):
// round-half-even(fl(fl(x - mn) / scale)), the quotient rounded to fp32 first.
template <int BITS>
__device__ __forceinline__ uint8_t quant_code(float x, float mn, float scale) {
  constexpr int kQmax = (1 << BITS) - 1;
  if (!(scale > 0.0f)) return 0;
  int c = __float2int_rn(__fdiv_rn(__fsub_rn(x, mn), scale));
  return (uint8_t)min(max(c, 0), kQmax);
}

// The same code with one multiply instead of the division, given inv =
// fl(1 / scale).  With d = fl(x - mn) in [0, max - min], the quotient
// Q = d / scale is at most 2^b - 1 (to within 2^-22), t = fl(d * inv) is within
// 2^-19 of Q and fl(Q) within 2^-20 of Q.  So when t is more than 2^-12 away
// from the nearest half-integer, fl(Q) lies on the same side of it and rounds
// to the same integer as t; the rare rest (and a non-finite t, from an inverse
// that overflows or is unusable) takes the division.
template <int BITS>
__device__ __forceinline__ uint8_t quant_code_inv(float x, float mn, float scale, float inv) {
  constexpr int kQmax = (1 << BITS) - 1;
  if (!(scale > 0.0f)) return 0;
  const float d = __fsub_rn(x, mn);
  float q = __fmul_rn(d, inv);
  const float frac = q - floorf(q);  // NaN for a non-finite q: the test below fails
  if (!(fabsf(frac - 0.5f) > 0x1p-12f)) q = __fdiv_rn(d, scale);
  const int c = __float2int_rn(q);
  return (uint8_t)min(max(c, 0), kQmax);
}

// fl(1 / scale) for quant_code_inv (unused when scale is 0); NaN, which sends
// every code to the division, when the inverse would be subnormal and lose its
// relative accuracy.
__device__ __forceinline__ float quant_inverse(float scale) {
  if (!(scale > 0.0f)) return 0.0f;
  const float r = __fdiv_rn(1.0f, scale);
  return r >= 0x1p-126f ? r : __int_as_float(0x7fffffff);
}

// Loads 32 token rows of D bf16 (row stride `ld` elements) into a smem tile,
// with NT threads (tid in [0, NT)).
template <int D, int NT, int ROW>
__device__ __forceinline__ void load_tile(__nv_bfloat16 (*dst)[ROW], const __nv_bfloat16* src,
                                          long ld, int tid) {
  static_assert(ROW >= D && ROW * 2 % 16 == 0, "rows of whole 16-byte vectors");
  constexpr int kVecPerRow = D * 2 / 16;
  for (int i = tid; i < kGroup * kVecPerRow; i += NT) {
    const int t = i / kVecPerRow, c = i % kVecPerRow;
    reinterpret_cast<uint4*>(&dst[t][0])[c] =
        reinterpret_cast<const uint4*>(src + (long)t * ld)[c];
  }
}

// (min, scale) of the n values x[0], x[stride], ...: exact min and max, then
// scale = (max - min) / (2^b - 1) rounded to nearest.
template <int BITS>
__device__ __forceinline__ void group_params(const __nv_bfloat16* x, int n, int stride, float& mn,
                                             float& scale) {
  constexpr int kQmax = (1 << BITS) - 1;
  mn = __bfloat162float(x[0]);
  float mx = mn;
#pragma unroll 8
  for (int i = 1; i < n; ++i) {
    const float v = __bfloat162float(x[i * stride]);
    mn = v < mn ? v : mn;  // strict comparisons, first occurrence wins (signed zeros)
    mx = v > mx ? v : mx;
  }
  scale = __fdiv_rn(__fsub_rn(mx, mn), (float)kQmax);
}

// Quantizes the K and V tiles in smem into one group record at `rec`, with NT
// threads (tid in [0, NT)); `sync()` is a barrier over exactly those threads.
template <int D, int BITS, int NT, typename Sync>
__device__ void quantize_tiles_to_record(QuantSmem<D>& sm, uint32_t* __restrict__ rec, int tid,
                                         Sync sync) {
  constexpr RecordGeom geo{D, BITS};
  unsigned short* rec16 = reinterpret_cast<unsigned short*>(rec);
  unsigned short* kscale = rec16 + geo.k_scale_off() / 2;
  unsigned short* kmin = rec16 + geo.k_min_off() / 2;
  unsigned short* vscale = rec16 + geo.v_scale_off() / 2;
  unsigned short* vmin = rec16 + geo.v_min_off() / 2;
  // Keys: per channel d over the 32 tokens.
  for (int d = tid; d < D; d += NT) {
    float mn, scale;
    group_params<BITS>(&sm.k[0][d], kGroup, D, mn, scale);
    const float inv = quant_inverse(scale);
#pragma unroll 8
    for (int t = 0; t < kGroup; ++t)
      sm.kc[t][d] = quant_code_inv<BITS>(__bfloat162float(sm.k[t][d]), mn, scale, inv);
    kscale[d] = to_f16_bits(scale);
    kmin[d] = to_f16_bits(mn);
  }
  // Values: per token t over channel block j.
  constexpr int kBlocks = D / 32;
  for (int p = tid; p < kGroup * kBlocks; p += NT) {
    const int t = p / kBlocks, j = p % kBlocks;
    float mn, scale;
    group_params<BITS>(&sm.v[t][32 * j], 32, 1, mn, scale);
    const float inv = quant_inverse(scale);
#pragma unroll 8
    for (int c = 0; c < 32; ++c)
      sm.vc[t][32 * j + c] =
          quant_code_inv<BITS>(__bfloat162float(sm.v[t][32 * j + c]), mn, scale, inv);
    vscale[v_meta_index(t, j)] = to_f16_bits(scale);
    vmin[v_meta_index(t, j)] = to_f16_bits(mn);
  }
  sync();
  // Pack the K codes: word w of token row t.  The word belongs to quad lane
  // tq = w / (D*b/128) and covers k-steps s = (32/(4b)) * (w % (D*b/128)) + sl;
  // code j of k-step s is channel 16s + 4tq + j (see kivi_layout.cuh).
  constexpr int kLaneWords = D * BITS / 128;  // words of one quad lane in a row
  constexpr int kStepsPerWord = 8 / BITS;
  for (int wi = tid; wi < geo.code_words(); wi += NT) {
    const int t = wi / geo.k_row_words(), w = wi % geo.k_row_words();
    const int tq = w / kLaneWords, s0 = kStepsPerWord * (w % kLaneWords);
    uint32_t word = 0;
#pragma unroll
    for (int sl = 0; sl < kStepsPerWord; ++sl)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int d = 16 * (s0 + sl) + 4 * tq + j;
        word |= (uint32_t)sm.kc[t][d] << k_code_bit(d, BITS);
      }
    rec[wi] = word;
  }
  // Pack the V codes: stored word wi holds lane word w of lane L = 4g + tig
  // (inverse of v_code_word); its codes are channels 16mt + g + 8r of tokens
  // 16kk + 8hf + 2tig + e.
  for (int wi = tid; wi < geo.code_words(); wi += NT) {
    const int L = (wi % 128) / 4, w = (wi / 128) * 4 + wi % 4;
    const int g = L / 4, tig = L % 4;
    uint32_t word = 0;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int mt = BITS == 2 ? w : w / 2;
            if (BITS == 4 && kk != w % 2) continue;
            const int d = 16 * mt + g + 8 * r, i = 16 * kk + 8 * hf + 2 * tig + e;
            word |= (uint32_t)sm.vc[i][d] << v_code_bit(i, d, BITS);
          }
    rec[geo.v_codes_off() / 4 + wi] = word;
  }
}

}  // namespace quant
}  // namespace kivi
