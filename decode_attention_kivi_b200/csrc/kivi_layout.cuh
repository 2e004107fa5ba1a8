// kivi_layout.cuh - geometry of the packed KIVI cache as the kernels see it.
//
// One group record per (layer, sequence, kv head, group of 32 tokens), in order:
//   K codes  [32 token rows][D*b/32 words]
//   V codes  D*32*b/32 words in the order the decode warps read them
//   K scale  [D] fp16, K min [D] fp16
//   V scale  [D/32][32] fp16 with the token pairs in thread order (v_meta_index),
//   V min    the same.
// Keys are quantized per channel over 32 tokens and values per token over 32
// channels ("KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache");
// group size 32 and residual 128 follow the record
// "kv-efficiency/kivi-2bit-llama3-8b-gqa-8k", field "Methodology".
//
// Code placement.  The decode kernel turns codes into tensor-core operands with
// the sm_100a conversions of packed small floats: a 2-bit code c sitting in the
// low two bits of a 4-bit field is the e2m1 value c/2, and a 4-bit code c
// sitting in the low four bits of a byte is the e2m3 value c/8, both exact.  So
// the 2-bit layouts put codes in the low two bits of nibbles (one mask spreads
// eight codes into nibbles, a shifted mask the other eight), and the 4-bit
// layouts put one code in each nibble.
//
//   K codes, 2 bits: channel d = 16s + 4t + j (k-step s, quad lane t, j < 4) of
//     a token row is in word t*(D/64) + s/4 of the row, at bit
//     8*(s%4) + 2*(j/2) + 4*(j%2).
//   K codes, 4 bits: the same channel is in word t*(D/32) + s/2, at bit
//     4*(s%2) + 8*j.
//   V codes: token i, channel d of lane L = 4*(d%8) + (i%8)/2 are in lane word w
//     (2 bits: w = d/16; 4 bits: w = 2*(d/16) + i/16), stored at word
//     ((w/4)*32 + L)*4 + w%4, so one 16-byte load per lane and four lane words
//     reads 512 contiguous bytes per warp.  With r = (d%16)/8, kk = i/16,
//     hf = (i%16)/8, e = i%2 the bit is
//       2 bits: 8*(r + 2*hf) + 2*kk + 4*e,
//       4 bits: 8*(2*hf + e) + 4*r.
#pragma once

#include <cstdint>

namespace kivi {

constexpr int kGroup = 32;                 // G
constexpr int kResidual = 128;             // R
constexpr int kRingSlots = kResidual + kGroup;  // ring slots per (layer, seq, kv head)
constexpr int kMaxHeadsPerKv = 8;

// K code of channel d in a token row: word index within the row and bit offset.
__host__ __device__ constexpr int k_code_word(int d, int D, int bits) {
  return bits == 2 ? ((d % 16) / 4) * (D / 64) + (d / 16) / 4
                   : ((d % 16) / 4) * (D / 32) + (d / 16) / 2;
}
__host__ __device__ constexpr int k_code_bit(int d, int bits) {
  return bits == 2 ? 8 * ((d / 16) % 4) + 2 * ((d % 4) / 2) + 4 * (d % 2)
                   : 4 * ((d / 16) % 2) + 8 * (d % 4);
}

// V code of token i (0..31), channel d: word index and bit offset.
__host__ __device__ constexpr int v_lane_word(int i, int d, int bits) {
  return bits == 2 ? d / 16 : 2 * (d / 16) + i / 16;
}
__host__ __device__ constexpr int v_code_word(int i, int d, int bits) {
  return ((v_lane_word(i, d, bits) / 4) * 32 + 4 * (d % 8) + (i % 8) / 2) * 4 +
         v_lane_word(i, d, bits) % 4;
}
__host__ __device__ constexpr int v_code_bit(int i, int d, int bits) {
  return bits == 2 ? 8 * ((d % 16) / 8 + 2 * ((i % 16) / 8)) + 2 * (i / 16) + 4 * (i % 2)
                   : 8 * (2 * ((i % 16) / 8) + i % 2) + 4 * ((d % 16) / 8);
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
  __host__ __device__ constexpr int k_row_words() const { return D * bits / 32; }
  __host__ __device__ constexpr int code_words() const { return kGroup * D * bits / 32; }
  __host__ __device__ constexpr long k_codes_off() const { return 0; }
  __host__ __device__ constexpr long v_codes_off() const { return 4L * code_words(); }
  __host__ __device__ constexpr long k_scale_off() const { return 8L * code_words(); }
  __host__ __device__ constexpr long k_min_off() const { return k_scale_off() + 2L * D; }
  __host__ __device__ constexpr long v_scale_off() const { return k_min_off() + 2L * D; }
  __host__ __device__ constexpr long v_min_off() const { return v_scale_off() + 2L * D; }
  __host__ __device__ constexpr long bytes() const { return v_min_off() + 2L * D; }
};

// Workspace of a handle (and of the static scratch array): [0, 256) the device
// status word and padding; then one int ticket per (sequence, kv head), rounded
// up to 256 bytes; then the split partials of the decode kernel.
constexpr long kWsHeader = 256;
__host__ __device__ constexpr long ws_tickets_bytes(long pairs) {
  return (4 * pairs + 255) / 256 * 256;
}

}  // namespace kivi
