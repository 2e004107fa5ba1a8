// kivi_layout.cuh - geometry of the packed KIVI cache as the kernels see it.
//
// One group record per (layer, sequence, kv head, group of 32 tokens):
//   K codes  [32 tokens][D*b/32 words]   channel d at bit (d % (32/b))*b of word d/(32/b)
//   V codes  [D channels][32*b/32 words] token i at bit (i % (32/b))*b of word i/(32/b)
//   K meta   [D] x {fp16 scale, fp16 min}
//   V meta   [32 tokens][D/32] x {fp16 scale, fp16 min}
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
  __host__ __device__ constexpr long k_meta_off() const { return 8L * code_words(); }
  __host__ __device__ constexpr long v_meta_off() const { return k_meta_off() + 4L * D; }
  __host__ __device__ constexpr long bytes() const { return v_meta_off() + 4L * kGroup * (D / 32); }
};

// Split-K count the workspace is sized for.
__host__ __device__ constexpr int max_splits(int batch, int kv_heads) {
  int pairs = batch * kv_heads;
  int s = (kTargetCtas + pairs - 1) / pairs;
  return s < 1 ? 1 : (s > kMaxSplitsCap ? kMaxSplitsCap : s);
}

// Workspace: [0, 256) device status word and padding; then per (b, q head,
// split) the running max m and sum l (two floats), then acc[D] floats.
constexpr long kWsHeader = 256;

}  // namespace kivi
