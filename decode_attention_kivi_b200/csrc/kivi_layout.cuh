// kivi_layout.cuh - geometry of the packed KIVI cache as the kernels see it.
//
// One group record per (layer, sequence, kv head, group of 32 tokens):
//   K codes  [32 tokens][D*b/32 words]: channel d = code d % (32/b) of word
//            d/(32/b); code n of a word sits at bit (n % 2)*16 + (n/2)*b (even
//            codes in the low half, odd codes in the high half).
//   V codes  D*32*b/32 words in the order the decode warps consume them: the
//            word of (row group g, lane-in-quad tig, 16-channel tile mt) holds,
//            for channels 16mt+g and 16mt+g+8, the tokens 2tig+{0,1}+{0,8}+{0,16}
//            as (even token low half, odd token high half) pairs.  See
//            v_code_word / v_code_bit below.
//   K scale  [D] fp16, K min [D] fp16
//   V scale  [D/32][32] fp16 with the token pairs in thread order (v_meta_index),
//   V min    the same.
// Keys are quantized per channel over 32 tokens and values per token over 32
// channels ("KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache");
// group size 32 and residual 128 follow the record
// "kv-efficiency/kivi-2bit-llama3-8b-gqa-8k", field "Methodology".
#pragma once

#include <cstdint>

namespace kivi {

constexpr int kGroup = 32;                 // G
constexpr int kResidual = 128;             // R
constexpr int kRingSlots = kResidual + kGroup;  // ring slots per (layer, seq, kv head)
constexpr int kMaxHeadsPerKv = 8;
constexpr int kMaxSplitsCap = 64;
constexpr int kTargetCtas = 2048;          // split-K sizing target (independent of the device)

// Bit offset of code n inside its 32-bit word.
__host__ __device__ constexpr int code_bit(int n, int bits) {
  return (n % 2) * 16 + ((n % (32 / bits)) / 2) * bits;
}

// V code of token i (0..31), channel d: word index and bit offset.
__host__ __device__ constexpr int v_code_idx(int i, int d) {
  return 4 * (i / 16) + 2 * ((i % 16) / 8) + (d % 16) / 8;  // 4 kk + 2 hf + r
}
__host__ __device__ constexpr int v_code_word(int i, int d, int D, int bits) {
  return ((4 * (d % 8) + (i % 8) / 2) * (D / 16) + d / 16) * (bits / 2) +
         v_code_idx(i, d) / (16 / bits);
}
__host__ __device__ constexpr int v_code_bit(int i, int d, int bits) {
  return 16 * (i % 2) + (v_code_idx(i, d) % (16 / bits)) * bits;
}
// fp16 index of the V scale / min of token i, channel block j.
__host__ __device__ constexpr int v_meta_index(int i, int j) {
  return 32 * j + 2 * (4 * ((i % 8) / 2) + 2 * (i / 16) + (i % 16) / 8) + i % 2;
}

__host__ __device__ constexpr int num_groups(int S) {
  return S < kResidual ? 0 : (S - kResidual) / kGroup;
}

struct RecordGeom {
  int D, bits;
  __host__ __device__ constexpr int codes_per_word() const { return 32 / bits; }
  __host__ __device__ constexpr int k_row_words() const { return D * bits / 32; }
  __host__ __device__ constexpr int v_row_words() const { return kGroup * bits / 32; }
  __host__ __device__ constexpr int code_words() const { return kGroup * D * bits / 32; }
  __host__ __device__ constexpr long k_codes_off() const { return 0; }
  __host__ __device__ constexpr long v_codes_off() const { return 4L * code_words(); }
  __host__ __device__ constexpr long k_scale_off() const { return 8L * code_words(); }
  __host__ __device__ constexpr long k_min_off() const { return k_scale_off() + 2L * D; }
  __host__ __device__ constexpr long v_scale_off() const { return k_min_off() + 2L * D; }
  __host__ __device__ constexpr long v_min_off() const { return v_scale_off() + 2L * D; }
  __host__ __device__ constexpr long bytes() const { return v_min_off() + 2L * D; }
};

// Split-K partials per (sequence, query head) the workspace is sized for: at
// least one split over the quantized groups plus one per residual chunk of up
// to 32 tokens (the residual holds fewer than R + G = 160 tokens: 5 chunks).
constexpr int kMinSplits = 1 + (kRingSlots + kGroup - 1) / kGroup;
__host__ __device__ constexpr int max_splits(int batch, int kv_heads) {
  int pairs = batch * kv_heads;
  int s = (kTargetCtas + pairs - 1) / pairs;
  return s < kMinSplits ? kMinSplits : (s > kMaxSplitsCap ? kMaxSplitsCap : s);
}

// Workspace: [0, 256) device status word and padding; then per (b, q head,
// split) the running max m and sum l (two floats), then acc[D] floats.
constexpr long kWsHeader = 256;

}  // namespace kivi
