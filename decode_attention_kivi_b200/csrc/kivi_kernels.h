// kivi_kernels.h - launchers of the KIVI kernels, called by the C ABI in kivi_api.cu.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace kivi {

struct PrefillArgs {
  const __nv_bfloat16* k;  // [B][Hkv][S][D] (S: the row stride, the longest sequence)
  const __nv_bfloat16* v;
  const int* lens;         // device [B] tokens per sequence, or null: S for every sequence
  int B, Hkv, S, ng, ngcap;  // ng = NG(S)
  uint8_t* records;        // layer base [B][Hkv][ngcap] records
  __nv_bfloat16* ring_k;   // layer base [B][Hkv][R+G][D]
  __nv_bfloat16* ring_v;
};

struct AppendArgs {
  const __nv_bfloat16* k_new;  // [B][Hkv][D]
  const __nv_bfloat16* v_new;
  const int* lens;             // device [B] prompt lengths, or null: S for every sequence
  int steps;                   // appends since the prompt (with lens): S_b = lens[b] + steps
  int B, Hkv, S, ngcap;
  __nv_bfloat16* ring_k;
  __nv_bfloat16* ring_v;
  uint8_t* records;
};

struct DecodeArgs {
  const uint8_t* records;        // layer base: [B][Hkv][ngcap] group records
  const __nv_bfloat16* ring_k;   // layer base: [B][Hkv][R+G][D]
  const __nv_bfloat16* ring_v;
  const __nv_bfloat16* q;        // [B][Hq][D]
  float* out;                    // [B][Hq][D]
  uint32_t* status;              // device status word
  int* tickets;                  // one per (sequence, kv head); zero between calls
  float* partials;               // [max_ctas][2][Hq/Hkv][D + 2] split partials
  int max_ctas;                  // capacity of `partials` in CTAs
  const int* lens;               // device [B] prompt lengths, or null: S for every sequence
  int steps;                     // appends since the prompt: S_b = lens[b] + steps
  int B, Hkv, Hq, S, ngcap;      // S: every sequence's length, or with lens the length
                                 // whose decode_items the split gives each pair
  float sm_scale;                // <= 0: 1/sqrt(D)
  int num_sms;
  int device;                    // the CUDA device the buffers live on (current at launch)
};

// Workspace of the decode kernel for `pairs` (sequence, kv head) pairs, in
// order: status header, tickets, then the
// per-CTA partials (partial_bytes each) of the largest grid it uses
// (decode_max_ctas).  Host-only arithmetic; no device is queried.
int decode_max_ctas(int D, int bits, int hpk, long pairs);
long decode_partial_bytes(int D, int hpk);
// CTAs the decode kernel launches for this shape on a device with num_sms SMs
// (0 for an unsupported shape).
int decode_grid_ctas(int D, int bits, int hpk, long pairs, int S, int num_sms);
long decode_workspace_bytes(int D, int bits, int hpk, long pairs);

// Debug build only (KIVI_DEBUG_BUILD): bytes added to every expected copy size
// of the decode kernel; cudaErrorNotSupported in a regular build.
cudaError_t debug_overstate_copies(unsigned bytes);

// Decode attention over an unquantized bf16 cache [B][Hkv][Smax][D] (tokens
// 0..S-1): the 16-bit baseline.  Workspace: status header, tickets, then
// bf16_partial_bytes of split partials.
struct Bf16DecodeArgs {
  const __nv_bfloat16 *k, *v;  // one layer's cache
  const __nv_bfloat16* q;      // [B][Hq][D]
  float* out;                  // [B][Hq][D]
  uint32_t* status;            // workspace header
  int* tickets;                // [B * Hkv], zero between calls
  float* partials;
  int B, Hkv, Hq, D, Smax, S;
  float sm_scale;              // <= 0: 1/sqrt(D)
  int num_sms;
  int device;
};
long bf16_partial_bytes(int D, int hpk);
cudaError_t launch_bf16_decode(const Bf16DecodeArgs& a, cudaStream_t stream);

// Key-granularity ablation: quantize-dequantize keys [rows][D] (rows a multiple
// of 32) per channel or per token into fp32 k_hat.
cudaError_t launch_fake_quant_keys(int D, int bits, const __nv_bfloat16* k, long rows,
                                   float* k_hat, int per_token, cudaStream_t stream);

// Causal prefill attention on the tcgen05 tensor cores; with `records` set, the
// CTAs of the first query head of every kv head also quantize their diagonal
// key/value tile into the cache (groups below NG(S)) and its ring (the rest).
struct PrefillAttnArgs {
  const __nv_bfloat16* q;        // [B][Hq][S][D]
  const __nv_bfloat16* k;        // [B][Hkv][S][D]
  const __nv_bfloat16* v;        // [B][Hkv][S][D]
  float* out;                    // [B][Hq][S][D]
  uint32_t* status;              // device status word, or null
  int B, Hkv, Hq, S;
  float sm_scale;                // <= 0: 1/sqrt(D)
  uint8_t* records;              // this layer's records, or null: attention only
  __nv_bfloat16* ring_k;         // this layer's rings [B][Hkv][R+G][D]
  __nv_bfloat16* ring_v;
  int ngcap;
  int device;
};

cudaError_t launch_prefill_attention(int D, int bits, const PrefillAttnArgs& a,
                                     cudaStream_t stream);

cudaError_t launch_prefill(int D, int bits, const PrefillArgs& a, cudaStream_t stream);
cudaError_t launch_append(int D, int bits, const AppendArgs& a, cudaStream_t stream);
cudaError_t launch_decode(int D, int bits, const DecodeArgs& a, cudaStream_t stream);

// Work items the decode split gives one (sequence, kv head) pair of S tokens:
// record pairs, a lone record, and residual rows of 8 tokens.  Not monotonic in
// S: just before a flush the residual holds R + G - 1 tokens.
int decode_items(int S);

}  // namespace kivi
