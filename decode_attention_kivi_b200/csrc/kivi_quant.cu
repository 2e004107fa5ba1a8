// kivi_quant.cu - KIVI group quantization: prefill, residual copy, append with flush.
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
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kivi_kernels.h"
#include "kivi_launch.cuh"
#include "kivi_layout.cuh"

namespace kivi {
namespace {

constexpr int kQuantThreads = 128;

template <int D>
struct QuantSmem {
  __nv_bfloat16 k[kGroup][D];
  __nv_bfloat16 v[kGroup][D];
  uint8_t kc[kGroup][D];
  uint8_t vc[kGroup][D];
};

__device__ __forceinline__ unsigned short to_f16_bits(float x) {
  return __half_as_ushort(__float2half_rn(x));
}

// Codes of one group of values already reduced to (mn, scale).
template <int BITS>
__device__ __forceinline__ uint8_t quant_code(float x, float mn, float scale) {
  constexpr int kQmax = (1 << BITS) - 1;
  if (!(scale > 0.0f)) return 0;
  int c = __float2int_rn(__fdiv_rn(__fsub_rn(x, mn), scale));
  return (uint8_t)min(max(c, 0), kQmax);
}

// Loads 32 token rows of D bf16 (row stride `ld` elements) into a smem tile.
template <int D>
__device__ __forceinline__ void load_tile(__nv_bfloat16 (*dst)[D], const __nv_bfloat16* src,
                                          long ld) {
  constexpr int kVecPerRow = D * 2 / 16;
  for (int i = threadIdx.x; i < kGroup * kVecPerRow; i += kQuantThreads) {
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

// Quantizes the K and V tiles in smem into one group record at `rec`.
template <int D, int BITS>
__device__ void quantize_tiles_to_record(QuantSmem<D>& sm, uint32_t* __restrict__ rec) {
  constexpr RecordGeom geo{D, BITS};
  unsigned short* rec16 = reinterpret_cast<unsigned short*>(rec);
  unsigned short* kscale = rec16 + geo.k_scale_off() / 2;
  unsigned short* kmin = rec16 + geo.k_min_off() / 2;
  unsigned short* vscale = rec16 + geo.v_scale_off() / 2;
  unsigned short* vmin = rec16 + geo.v_min_off() / 2;
  // Keys: per channel d over the 32 tokens.
  for (int d = threadIdx.x; d < D; d += kQuantThreads) {
    float mn, scale;
    group_params<BITS>(&sm.k[0][d], kGroup, D, mn, scale);
#pragma unroll 8
    for (int t = 0; t < kGroup; ++t) sm.kc[t][d] = quant_code<BITS>(__bfloat162float(sm.k[t][d]), mn, scale);
    kscale[d] = to_f16_bits(scale);
    kmin[d] = to_f16_bits(mn);
  }
  // Values: per token t over channel block j.
  constexpr int kBlocks = D / 32;
  for (int p = threadIdx.x; p < kGroup * kBlocks; p += kQuantThreads) {
    const int t = p / kBlocks, j = p % kBlocks;
    float mn, scale;
    group_params<BITS>(&sm.v[t][32 * j], 32, 1, mn, scale);
#pragma unroll 8
    for (int c = 0; c < 32; ++c)
      sm.vc[t][32 * j + c] = quant_code<BITS>(__bfloat162float(sm.v[t][32 * j + c]), mn, scale);
    vscale[v_meta_index(t, j)] = to_f16_bits(scale);
    vmin[v_meta_index(t, j)] = to_f16_bits(mn);
  }
  __syncthreads();
  // Pack the K codes: word w of token row t.  The word belongs to quad lane
  // tq = w / (D*b/128) and covers k-steps s = (32/(4b)) * (w % (D*b/128)) + sl;
  // code j of k-step s is channel 16s + 4tq + j (see kivi_layout.cuh).
  constexpr int kLaneWords = D * BITS / 128;  // words of one quad lane in a row
  constexpr int kStepsPerWord = 8 / BITS;
  for (int wi = threadIdx.x; wi < geo.code_words(); wi += kQuantThreads) {
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
  for (int wi = threadIdx.x; wi < geo.code_words(); wi += kQuantThreads) {
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

// Prefill: one CTA per (group, kv head, sequence).
template <int D, int BITS>
__global__ void __launch_bounds__(kQuantThreads)
prefill_groups_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                      int S, int Hkv, int ngcap, uint8_t* __restrict__ records) {
  __shared__ __align__(16) QuantSmem<D> sm;
  constexpr RecordGeom geo{D, BITS};
  const int g = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const long seq = (long)b * Hkv + h;
  const long src = (seq * S + (long)g * kGroup) * D;
  load_tile<D>(sm.k, k + src, D);
  load_tile<D>(sm.v, v + src, D);
  __syncthreads();
  uint8_t* rec = records + (seq * ngcap + g) * geo.bytes();
  quantize_tiles_to_record<D, BITS>(sm, reinterpret_cast<uint32_t*>(rec));
}

// Copies prompt tokens [first, S) of every (sequence, kv head) into ring slots t mod (R+G).
template <int D>
__global__ void __launch_bounds__(kQuantThreads)
copy_residual_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                     int S, int first, int Hkv, __nv_bfloat16* __restrict__ ring_k,
                     __nv_bfloat16* __restrict__ ring_v) {
  constexpr int kVecPerRow = D * 2 / 16;
  const int h = blockIdx.x, b = blockIdx.y;
  const long seq = (long)b * Hkv + h;
  const int n = S - first;
  for (int i = threadIdx.x; i < n * kVecPerRow; i += kQuantThreads) {
    const int t = first + i / kVecPerRow, c = i % kVecPerRow;
    const long src = (seq * S + t) * D;
    const long dst = (seq * kRingSlots + t % kRingSlots) * D;
    reinterpret_cast<uint4*>(ring_k + dst)[c] = reinterpret_cast<const uint4*>(k + src)[c];
    reinterpret_cast<uint4*>(ring_v + dst)[c] = reinterpret_cast<const uint4*>(v + src)[c];
  }
}

// Append token S to every (sequence, kv head); with `flush`, quantize ring
// tokens [first, first + 32) into record `ng`.
template <int D, int BITS>
__global__ void __launch_bounds__(kQuantThreads)
append_kernel(const __nv_bfloat16* __restrict__ k_new, const __nv_bfloat16* __restrict__ v_new,
              int S, int Hkv, int ngcap, int flush, int ng, __nv_bfloat16* __restrict__ ring_k,
              __nv_bfloat16* __restrict__ ring_v, uint8_t* __restrict__ records) {
  __shared__ __align__(16) QuantSmem<D> sm;
  constexpr RecordGeom geo{D, BITS};
  constexpr int kVecPerRow = D * 2 / 16;
  wait_for_predecessor();  // the previous kernel may still read this layer's ring
  allow_successor();
  const int h = blockIdx.x, b = blockIdx.y;
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
  if (a.ng > 0) {
    dim3 grid(a.ng, a.Hkv, a.B);
    prefill_groups_kernel<D, BITS><<<grid, kQuantThreads, 0, stream>>>(a.k, a.v, a.S, a.Hkv,
                                                                      a.ngcap, a.records);
  }
  if (a.S > a.ng * kGroup) {
    dim3 grid(a.Hkv, a.B);
    copy_residual_kernel<D><<<grid, kQuantThreads, 0, stream>>>(a.k, a.v, a.S, a.ng * kGroup,
                                                               a.Hkv, a.ring_k, a.ring_v);
  }
  return cudaGetLastError();
}

template <int D, int BITS>
cudaError_t launch_append_t(const AppendArgs& a, cudaStream_t stream) {
  dim3 grid(a.Hkv, a.B);
  cudaError_t e = launch_pdl(append_kernel<D, BITS>, grid, dim3(kQuantThreads), 0, stream,
                             a.k_new, a.v_new, a.S, a.Hkv, a.ngcap, a.flush, a.ng, a.ring_k,
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
