// kivi_kernels.h - launchers of the KIVI kernels, called by the C ABI in kivi_api.cu.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace kivi {

struct PrefillArgs {
  const __nv_bfloat16* k;  // [B][Hkv][S][D]
  const __nv_bfloat16* v;
  int B, Hkv, S, ng, ngcap;
  uint8_t* records;        // layer base [B][Hkv][ngcap] records
  __nv_bfloat16* ring_k;   // layer base [B][Hkv][R+G][D]
  __nv_bfloat16* ring_v;
};

struct AppendArgs {
  const __nv_bfloat16* k_new;  // [B][Hkv][D]
  const __nv_bfloat16* v_new;
  int B, Hkv, S, ngcap;
  int flush, ng;               // flush ring tokens [ng*G, ng*G+G) into record ng
  __nv_bfloat16* ring_k;
  __nv_bfloat16* ring_v;
  uint8_t* records;
};

struct DecodeArgs {
  const uint8_t* records;        // layer base
  const __nv_bfloat16* ring_k;   // layer base
  const __nv_bfloat16* ring_v;
  const __nv_bfloat16* q;        // [B][Hq][D]
  float* out;                    // [B][Hq][D]
  float* ws_ml;                  // [B][Hq][splits] x {m, l}
  float* ws_acc;                 // [B][Hq][splits][D]
  uint32_t* status;              // device status word
  int B, Hkv, Hq, S, ngcap;
  float sm_scale;
  int max_splits;                // the workspace's capacity in splits
  int num_sms;
};

cudaError_t launch_prefill(int D, int bits, const PrefillArgs& a, cudaStream_t stream);
cudaError_t launch_append(int D, int bits, const AppendArgs& a, cudaStream_t stream);
cudaError_t launch_decode(int D, int bits, const DecodeArgs& a, cudaStream_t stream);

}  // namespace kivi
