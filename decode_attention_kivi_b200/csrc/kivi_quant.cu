// kivi_quant.cu - KIVI group quantization: prefill, residual copy, append with flush.
//
// The quantizer itself (rounding rules, record packing) is in kivi_quant.cuh.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kivi_kernels.h"
#include "kivi_launch.cuh"
#include "kivi_layout.cuh"
#include "kivi_quant.cuh"

namespace kivi {
namespace {

using quant::group_params;
using quant::quant_code;
using quant::QuantSmem;

constexpr int kQuantThreads = 128;

template <int D, int ROW>
__device__ __forceinline__ void load_tile(__nv_bfloat16 (*dst)[ROW], const __nv_bfloat16* src,
                                          long ld) {
  quant::load_tile<D, kQuantThreads>(dst, src, ld, threadIdx.x);
}

template <int D, int BITS>
__device__ __forceinline__ void quantize_tiles_to_record(QuantSmem<D>& sm, uint32_t* rec) {
  quant::quantize_tiles_to_record<D, BITS, kQuantThreads>(sm, rec, threadIdx.x, [] { __syncthreads(); });
}

// Prefill: one CTA per (group, kv head, sequence).  Input rows have stride
// Smax tokens; sequence b holds lens[b] tokens (all Smax when lens is null).
template <int D, int BITS>
__global__ void __launch_bounds__(kQuantThreads)
prefill_groups_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                      int Smax, const int* __restrict__ lens, int Hkv, int ngcap,
                      uint8_t* __restrict__ records) {
  __shared__ __align__(16) QuantSmem<D> sm;
  constexpr RecordGeom geo{D, BITS};
  const int g = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  if (lens != nullptr && g >= num_groups(lens[b])) return;  // beyond this sequence's groups
  const long seq = (long)b * Hkv + h;
  const long src = (seq * Smax + (long)g * kGroup) * D;
  load_tile<D>(sm.k, k + src, D);
  load_tile<D>(sm.v, v + src, D);
  __syncthreads();
  uint8_t* rec = records + (seq * ngcap + g) * geo.bytes();
  quantize_tiles_to_record<D, BITS>(sm, reinterpret_cast<uint32_t*>(rec));
}

// Copies prompt tokens [NG(S_b)*G, S_b) of every (sequence, kv head) into ring
// slots t mod (R+G); S_b = lens[b], or Smax for every sequence when lens is null.
template <int D>
__global__ void __launch_bounds__(kQuantThreads)
copy_residual_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                     int Smax, const int* __restrict__ lens, int Hkv,
                     __nv_bfloat16* __restrict__ ring_k, __nv_bfloat16* __restrict__ ring_v) {
  constexpr int kVecPerRow = D * 2 / 16;
  const int h = blockIdx.x, b = blockIdx.y;
  const long seq = (long)b * Hkv + h;
  const int S = lens != nullptr ? lens[b] : Smax;
  const int first = num_groups(S) * kGroup;
  const int n = S - first;
  for (int i = threadIdx.x; i < n * kVecPerRow; i += kQuantThreads) {
    const int t = first + i / kVecPerRow, c = i % kVecPerRow;
    const long src = (seq * Smax + t) * D;
    const long dst = (seq * kRingSlots + t % kRingSlots) * D;
    reinterpret_cast<uint4*>(ring_k + dst)[c] = reinterpret_cast<const uint4*>(k + src)[c];
    reinterpret_cast<uint4*>(ring_v + dst)[c] = reinterpret_cast<const uint4*>(v + src)[c];
  }
}

// Append token S_b to every (sequence, kv head), S_b = lens[b] + steps (or S
// for every sequence when lens is null); when the residual would reach R + G,
// quantize the ring tokens [NG*G, NG*G + 32) of that sequence into record NG.
template <int D, int BITS>
__global__ void __launch_bounds__(kQuantThreads)
append_kernel(const __nv_bfloat16* __restrict__ k_new, const __nv_bfloat16* __restrict__ v_new,
              int S_all, const int* __restrict__ lens, int steps, int Hkv, int ngcap,
              __nv_bfloat16* __restrict__ ring_k, __nv_bfloat16* __restrict__ ring_v,
              uint8_t* __restrict__ records) {
  __shared__ __align__(16) QuantSmem<D> sm;
  constexpr RecordGeom geo{D, BITS};
  constexpr int kVecPerRow = D * 2 / 16;
  wait_for_predecessor();  // the previous kernel may still read this layer's ring
  allow_successor();
  const int h = blockIdx.x, b = blockIdx.y;
  const int S = lens != nullptr ? lens[b] + steps : S_all;
  const int ng = num_groups(S);
  const bool flush = S + 1 - ng * kGroup == kRingSlots;
  const long seq = (long)b * Hkv + h;
  __nv_bfloat16* rk = ring_k + seq * kRingSlots * D;
  __nv_bfloat16* rv = ring_v + seq * kRingSlots * D;
  if (flush) {
    const int first = (ng * kGroup) % kRingSlots;  // a group never wraps the ring
    load_tile<D>(sm.k, rk + (long)first * D, D);
    load_tile<D>(sm.v, rv + (long)first * D, D);
  }
  // The new token's slot is not one of the flushed group's 32 slots.
  const int slot = S % kRingSlots;
  for (int c = threadIdx.x; c < kVecPerRow; c += kQuantThreads) {
    reinterpret_cast<uint4*>(rk + (long)slot * D)[c] =
        reinterpret_cast<const uint4*>(k_new + seq * D)[c];
    reinterpret_cast<uint4*>(rv + (long)slot * D)[c] =
        reinterpret_cast<const uint4*>(v_new + seq * D)[c];
  }
  if (flush) {
    __syncthreads();
    uint8_t* rec = records + (seq * ngcap + ng) * geo.bytes();
    quantize_tiles_to_record<D, BITS>(sm, reinterpret_cast<uint32_t*>(rec));
  }
}

// Key-granularity ablation: quantize-dequantize the keys of one 32-token group,
// per channel (KIVI's rule for keys) or per token over 32-channel blocks (the
// values' rule), with the record's quantizer and fp16 metadata;
// k_hat = RN(fp16(scale) * code + fp16(min)) in fp32 (one rounding).
template <int D, int BITS>
__global__ void __launch_bounds__(kQuantThreads)
fake_quant_keys_kernel(const __nv_bfloat16* __restrict__ k, float* __restrict__ k_hat,
                       int per_token) {
  __shared__ __align__(16) __nv_bfloat16 tile[kGroup][D];
  const long row0 = (long)blockIdx.x * kGroup;
  wait_for_predecessor();
  load_tile<D>(tile, k + row0 * D, D);
  __syncthreads();
  allow_successor();
  const int n_groups = per_token ? kGroup * (D / 32) : D;
  for (int u = threadIdx.x; u < n_groups; u += kQuantThreads) {
    // group u: channel u of the 32 tokens, or token u / (D/32), channels 32 (u % (D/32)) + i
    const int t0 = per_token ? u / (D / 32) : 0, d0 = per_token ? 32 * (u % (D / 32)) : u;
    const int stride = per_token ? 1 : D;
    const __nv_bfloat16* x = &tile[t0][d0];
    float mn, scale;
    group_params<BITS>(x, 32, stride, mn, scale);
    const float sh = __half2float(__float2half_rn(scale)), mh = __half2float(__float2half_rn(mn));
    for (int i = 0; i < 32; ++i) {
      const int c = quant_code<BITS>(__bfloat162float(x[i * stride]), mn, scale);
      k_hat[(row0 + t0) * D + d0 + (long)i * stride] = __fmaf_rn(sh, (float)c, mh);
    }
  }
}

template <int D, int BITS>
cudaError_t launch_fake_quant_t(const __nv_bfloat16* k, long rows, float* k_hat, int per_token,
                                cudaStream_t stream) {
  if (rows % kGroup != 0 || rows / kGroup > 0x7fffffffL) return cudaErrorInvalidValue;
  cudaError_t e = launch_pdl(fake_quant_keys_kernel<D, BITS>, dim3((unsigned)(rows / kGroup)),
                             dim3(kQuantThreads), 0, stream, k, k_hat, per_token);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int D, int BITS>
cudaError_t launch_prefill_t(const PrefillArgs& a, cudaStream_t stream) {
  if (a.ng > 0) {  // groups of the longest sequence; shorter ones skip the rest
    dim3 grid(a.ng, a.Hkv, a.B);
    prefill_groups_kernel<D, BITS><<<grid, kQuantThreads, 0, stream>>>(a.k, a.v, a.S, a.lens,
                                                                      a.Hkv, a.ngcap, a.records);
  }
  if (a.lens != nullptr || a.S > a.ng * kGroup) {
    dim3 grid(a.Hkv, a.B);
    copy_residual_kernel<D><<<grid, kQuantThreads, 0, stream>>>(a.k, a.v, a.S, a.lens, a.Hkv,
                                                               a.ring_k, a.ring_v);
  }
  return cudaGetLastError();
}

template <int D, int BITS>
cudaError_t launch_append_t(const AppendArgs& a, cudaStream_t stream) {
  dim3 grid(a.Hkv, a.B);
  cudaError_t e = launch_pdl(append_kernel<D, BITS>, grid, dim3(kQuantThreads), 0, stream,
                             a.k_new, a.v_new, a.S, a.lens, a.steps, a.Hkv, a.ngcap, a.ring_k,
                             a.ring_v, a.records);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fake_quant_keys(int D, int bits, const __nv_bfloat16* k, long rows,
                                   float* k_hat, int per_token, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  if (D == 128 && bits == 2) return launch_fake_quant_t<128, 2>(k, rows, k_hat, per_token, stream);
  if (D == 128 && bits == 4) return launch_fake_quant_t<128, 4>(k, rows, k_hat, per_token, stream);
  if (D == 64 && bits == 2) return launch_fake_quant_t<64, 2>(k, rows, k_hat, per_token, stream);
  if (D == 64 && bits == 4) return launch_fake_quant_t<64, 4>(k, rows, k_hat, per_token, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_prefill(int D, int bits, const PrefillArgs& a, cudaStream_t stream) {
  if (D == 128 && bits == 2) return launch_prefill_t<128, 2>(a, stream);
  if (D == 128 && bits == 4) return launch_prefill_t<128, 4>(a, stream);
  if (D == 64 && bits == 2) return launch_prefill_t<64, 2>(a, stream);
  if (D == 64 && bits == 4) return launch_prefill_t<64, 4>(a, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_append(int D, int bits, const AppendArgs& a, cudaStream_t stream) {
  if (D == 128 && bits == 2) return launch_append_t<128, 2>(a, stream);
  if (D == 128 && bits == 4) return launch_append_t<128, 4>(a, stream);
  if (D == 64 && bits == 2) return launch_append_t<64, 2>(a, stream);
  if (D == 64 && bits == 4) return launch_append_t<64, 4>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace kivi
