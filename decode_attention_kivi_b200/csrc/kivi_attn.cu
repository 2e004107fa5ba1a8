// kivi_attn.cu - fused single-token decode attention over the packed KIVI cache.
//
// For query head h of sequence b (kv head h / (Hq/Hkv)), over all S cached tokens:
//   s_t = sm_scale * <q, k_t>,  out = sum_t softmax(s)_t v_t,
// where k_t, v_t are dequantized in registers (scale_h * code + min_h) for the
// NG(S)*32 grouped tokens and read as bf16 from the residual ring for the rest
// (record "kv-efficiency/kivi-2bit-llama3-8b-gqa-8k", "KV bytes basis": the
// most recent R tokens stay full precision).  Quantized history and residual
// share one online softmax.
//
// Dequantization is folded into the dot products: per key group with channel
// scales s_d and mins m_d, <q, k_t> = sum_d (q_d s_d) c_td + sum_d q_d m_d; per
// value token with block scale s_tj and min m_tj, sum_t p_t v_td = sum_t (p_t s_tj)
// c_td + sum_t p_t m_tj.  Scores are kept in log2 units (q pre-scaled by
// sm_scale * log2 e) so the softmax uses exp2.
//
// Work split: grid (splits, Hkv, B); the units of one (b, kv head) are its
// quantized groups followed by its residual chunks of up to 32 tokens; split s
// takes a contiguous range of units and its 4 warps take the units round-robin.
// Each warp keeps its own (m, l, acc) per query head; the CTA merges its warps
// and writes one partial per (b, q head, split); a second kernel merges splits.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cfloat>

#include "kivi_kernels.h"
#include "kivi_layout.cuh"

namespace kivi {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float2 unpack_meta(uint32_t m) {
  return make_float2(__half2float(__ushort_as_half((unsigned short)(m & 0xffffu))),
                     __half2float(__ushort_as_half((unsigned short)(m >> 16))));
}

template <int D, int HPK>
struct AttnSmem {
  float q[HPK][D];                    // q * sm_scale * log2 e
  float qt[kWarps][HPK][D];           // per warp: q * key channel scale (current group)
  float a[kWarps][HPK][kGroup][D / 32];  // per warp: p * value block scale
  float wm[kWarps][HPK];
  float wl[kWarps][HPK];
};

template <int D, int BITS, int HPK>
__global__ void __launch_bounds__(kThreads)
decode_split_kernel(DecodeArgs args, int splits, int units_per_split, float qscale) {
  constexpr RecordGeom geo{D, BITS};
  constexpr int kQmax = (1 << BITS) - 1;
  constexpr int kCpw = geo.codes_per_word();
  constexpr int kKRow = geo.k_row_words();
  constexpr int kVRow = geo.v_row_words();
  constexpr int kCh = D / 32;  // channels per lane (lane + 32 i), also value blocks
  __shared__ __align__(16) AttnSmem<D, HPK> sm;

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int Hkv = args.Hkv, Hq = args.Hq, S = args.S;
  const long seq = (long)b * Hkv + kvh;
  const int NG = num_groups(S);
  const int n_units = NG + (S - NG * kGroup + kGroup - 1) / kGroup;
  const int u_begin = split * units_per_split;
  const int u_end = min(n_units, u_begin + units_per_split);

  for (int i = threadIdx.x; i < HPK * D; i += kThreads) {
    const int hh = i / D, d = i % D;
    sm.q[hh][d] = __bfloat162float(args.q[((long)b * Hq + kvh * HPK + hh) * D + d]) * qscale;
  }
  __syncthreads();

  float m[HPK], l[HPK], acc[HPK][kCh];
#pragma unroll
  for (int hh = 0; hh < HPK; ++hh) {
    m[hh] = -INFINITY;
    l[hh] = 0.f;
#pragma unroll
    for (int i = 0; i < kCh; ++i) acc[hh][i] = 0.f;
  }

  const uint8_t* seq_records = args.records + seq * args.ngcap * geo.bytes();
  const __nv_bfloat16* rk = args.ring_k + seq * kRingSlots * D;
  const __nv_bfloat16* rv = args.ring_v + seq * kRingSlots * D;

  for (int u = u_begin + warp; u < u_end; u += kWarps) {
    float s[HPK];
    if (u < NG) {
      const uint8_t* rec = seq_records + (long)u * geo.bytes();
      const uint32_t* kmeta = reinterpret_cast<const uint32_t*>(rec + geo.k_meta_off());
      // q~ = q * key scale per channel, and sum_d q_d m_d per head.
      float qm[HPK];
#pragma unroll
      for (int hh = 0; hh < HPK; ++hh) qm[hh] = 0.f;
#pragma unroll
      for (int i = 0; i < kCh; ++i) {
        const int d = lane + 32 * i;
        const float2 sc = unpack_meta(kmeta[d]);
#pragma unroll
        for (int hh = 0; hh < HPK; ++hh) {
          sm.qt[warp][hh][d] = sm.q[hh][d] * sc.x;
          qm[hh] += sm.q[hh][d] * sc.y;
        }
      }
#pragma unroll
      for (int hh = 0; hh < HPK; ++hh) s[hh] = warp_sum(qm[hh]);
      __syncwarp();
      // Scores: lane = token of the group.
      const uint32_t* krow = reinterpret_cast<const uint32_t*>(rec) + lane * kKRow;
#pragma unroll
      for (int w = 0; w < kKRow; ++w) {
        const uint32_t word = krow[w];
#pragma unroll
        for (int i = 0; i < kCpw; ++i) {
          const float c = (float)((word >> (i * BITS)) & kQmax);
          const int d = w * kCpw + i;
#pragma unroll
          for (int hh = 0; hh < HPK; ++hh) s[hh] += c * sm.qt[warp][hh][d];
        }
      }
    } else {
      const int t = NG * kGroup + (u - NG) * kGroup + lane;
      if (t < S) {
        const __nv_bfloat16* kr = rk + (long)(t % kRingSlots) * D;
#pragma unroll
        for (int hh = 0; hh < HPK; ++hh) s[hh] = 0.f;
        for (int d = 0; d < D; ++d) {
          const float kv = __bfloat162float(kr[d]);
#pragma unroll
          for (int hh = 0; hh < HPK; ++hh) s[hh] += kv * sm.q[hh][d];
        }
      } else {
#pragma unroll
        for (int hh = 0; hh < HPK; ++hh) s[hh] = -INFINITY;
      }
    }
    // Online softmax update (log2 domain).
    float p[HPK];
#pragma unroll
    for (int hh = 0; hh < HPK; ++hh) {
      const float m_new = fmaxf(m[hh], warp_max(s[hh]));
      const float alpha = exp2f(m[hh] - m_new);
      p[hh] = exp2f(s[hh] - m_new);
      l[hh] = l[hh] * alpha + warp_sum(p[hh]);
      m[hh] = m_new;
#pragma unroll
      for (int i = 0; i < kCh; ++i) acc[hh][i] *= alpha;
    }
    if (u < NG) {
      const uint8_t* rec = seq_records + (long)u * geo.bytes();
      const uint32_t* vmeta = reinterpret_cast<const uint32_t*>(rec + geo.v_meta_off());
      // a = p * value block scale (lane = token); sum_t p_t m_tj per block.
      float pm[HPK][kCh];
#pragma unroll
      for (int j = 0; j < kCh; ++j) {
        const float2 sc = unpack_meta(vmeta[lane * kCh + j]);
#pragma unroll
        for (int hh = 0; hh < HPK; ++hh) {
          sm.a[warp][hh][lane][j] = p[hh] * sc.x;
          pm[hh][j] = p[hh] * sc.y;
        }
      }
#pragma unroll
      for (int hh = 0; hh < HPK; ++hh)
#pragma unroll
        for (int j = 0; j < kCh; ++j) pm[hh][j] = warp_sum(pm[hh][j]);
      __syncwarp();
      // P.V: lane owns channels lane + 32 i (value block i).
      const uint32_t* vcodes = reinterpret_cast<const uint32_t*>(rec + geo.v_codes_off());
#pragma unroll
      for (int i = 0; i < kCh; ++i) {
        const uint32_t* vrow = vcodes + (lane + 32 * i) * kVRow;
        uint32_t words[kVRow];
#pragma unroll
        for (int w = 0; w < kVRow; ++w) words[w] = vrow[w];
#pragma unroll
        for (int t = 0; t < kGroup; ++t) {
          const float c = (float)((words[t / kCpw] >> ((t % kCpw) * BITS)) & kQmax);
#pragma unroll
          for (int hh = 0; hh < HPK; ++hh) acc[hh][i] += sm.a[warp][hh][t][i] * c;
        }
#pragma unroll
        for (int hh = 0; hh < HPK; ++hh) acc[hh][i] += pm[hh][i];
      }
    } else {
      // Residual chunk: broadcast p through smem, lane owns channels.
#pragma unroll
      for (int hh = 0; hh < HPK; ++hh) sm.a[warp][hh][lane][0] = p[hh];
      __syncwarp();
      const int t0 = NG * kGroup + (u - NG) * kGroup;
      const int n = min(kGroup, S - t0);
      for (int t = 0; t < n; ++t) {
        const __nv_bfloat16* vr = rv + (long)((t0 + t) % kRingSlots) * D;
#pragma unroll
        for (int i = 0; i < kCh; ++i) {
          const float vv = __bfloat162float(vr[lane + 32 * i]);
#pragma unroll
          for (int hh = 0; hh < HPK; ++hh) acc[hh][i] += sm.a[warp][hh][t][0] * vv;
        }
      }
    }
    __syncwarp();
  }

  // Merge the warps of this CTA.
  if (lane == 0) {
#pragma unroll
    for (int hh = 0; hh < HPK; ++hh) {
      sm.wm[warp][hh] = m[hh];
      sm.wl[warp][hh] = l[hh];
    }
  }
  __syncthreads();
  float* wacc = &sm.qt[0][0][0];  // reuse: [kWarps][HPK][D]
#pragma unroll
  for (int hh = 0; hh < HPK; ++hh) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm.wm[w][hh]);
    const float f = (m[hh] == -INFINITY) ? 0.f : exp2f(m[hh] - M);
#pragma unroll
    for (int i = 0; i < kCh; ++i) wacc[(warp * HPK + hh) * D + lane + 32 * i] = acc[hh][i] * f;
  }
  __syncthreads();
  const long part0 = ((long)b * Hq + kvh * HPK) * splits + split;
  for (int i = threadIdx.x; i < HPK * D; i += kThreads) {
    const int hh = i / D, d = i % D;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) sum += wacc[(w * HPK + hh) * D + d];
    args.ws_acc[(part0 + (long)hh * splits) * D + d] = sum;
  }
  if (threadIdx.x < HPK) {
    const int hh = threadIdx.x;
    float M = -INFINITY, L = 0.f;
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm.wm[w][hh]);
    for (int w = 0; w < kWarps; ++w)
      if (sm.wm[w][hh] != -INFINITY) L += sm.wl[w][hh] * exp2f(sm.wm[w][hh] - M);
    args.ws_ml[2 * (part0 + (long)hh * splits)] = M;
    args.ws_ml[2 * (part0 + (long)hh * splits) + 1] = L;
  }
}

// out[b][h] = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s.
template <int D>
__global__ void __launch_bounds__(D) combine_kernel(DecodeArgs args, int splits) {
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const long part0 = ((long)b * args.Hq + h) * splits;
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, args.ws_ml[2 * (part0 + s)]);
  float L = 0.f, o = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float ms = args.ws_ml[2 * (part0 + s)];
    if (ms == -INFINITY) continue;
    const float f = exp2f(ms - M);
    L += f * args.ws_ml[2 * (part0 + s) + 1];
    o += f * args.ws_acc[(part0 + s) * D + d];
  }
  args.out[((long)b * args.Hq + h) * D + d] = o / L;
}

template <int D, int BITS, int HPK>
cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t stream) {
  const int NG = num_groups(a.S);
  const int n_units = NG + (a.S - NG * kGroup + kGroup - 1) / kGroup;
  const int pairs = a.B * a.Hkv;
  int splits = (2 * a.num_sms * 4 + pairs - 1) / pairs;  // aim for ~8 CTAs per SM
  splits = max(1, min(splits, min(a.max_splits, n_units)));
  const int ups = (n_units + splits - 1) / splits;
  splits = (n_units + ups - 1) / ups;  // every split non-empty
  const float qscale = (a.sm_scale > 0.f ? a.sm_scale : rsqrtf((float)D)) * kLog2e;
  dim3 grid(splits, a.Hkv, a.B);
  decode_split_kernel<D, BITS, HPK><<<grid, kThreads, 0, stream>>>(a, splits, ups, qscale);
  dim3 cgrid(a.Hq, a.B);
  combine_kernel<D><<<cgrid, D, 0, stream>>>(a, splits);
  return cudaGetLastError();
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

}  // namespace

cudaError_t launch_decode(int D, int bits, const DecodeArgs& a, cudaStream_t stream) {
  if (D == 128 && bits == 2) return launch_decode_d<128, 2>(a, stream);
  if (D == 128 && bits == 4) return launch_decode_d<128, 4>(a, stream);
  if (D == 64 && bits == 2) return launch_decode_d<64, 2>(a, stream);
  if (D == 64 && bits == 4) return launch_decode_d<64, 4>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace kivi
