// kivi_bf16_attn.cu - single-token decode attention over an unquantized bf16
// KV cache: the 16-bit baseline that the KIVI page and the HF news page set the
// 2-bit cache against (the same attention, s_t = sm_scale * <q, k_t>,
// out = sum_t softmax(s)_t v_t, over bf16 keys and values).
//
// The cache is [B][Hkv][Smax][D] bf16 per layer; tokens 0..S-1 are attended.
// Work: the tiles of 64 tokens of all (sequence, kv head) pairs, in order, are
// cut into one contiguous, equal-length range per CTA (one persistent CTA per
// SM).  Each CTA runs a producer warp that streams K and V tiles with 2D tensor
// copies (128-byte swizzle) into a ring of stages, and four consumer warps that
// take 16 tokens of every tile each.  On the tensor cores (mma.sync m16n8k16,
// bf16 operands, fp32 accumulation):
//   scores  C[token][head] = sum_d K[token][d] q[head][d]      (exact products)
//   P.V     C[chan][col]  += sum_t V[t][chan] p[col][t]
// with p carried as a bf16 pair hi + lo; for up to four heads per kv head the
// lo parts take the four columns the heads leave free.  The four warps merge
// their online-softmax states whenever the pair changes; a pair held whole is
// written to the output directly, a pair shared with other CTAs as a partial,
// and the last CTA to arrive at a pair (a ticket per pair) merges its partials.
// Every wait is bounded; a wait that runs out sets the status word.
#include <cuda_bf16.h>

#include "kivi_kernels.h"
#include "kivi_launch.cuh"
#include "kivi_layout.cuh"
#include "kivi_ptx.cuh"
#include "kivi_tmap.cuh"

namespace kivi {
namespace {

constexpr float kLog2eB = 1.4426950408889634f;
constexpr uint32_t kStatusWaitTimeoutB = 1u;
constexpr int kTile = 64;          // tokens per tile
constexpr int kCW = 4;             // consumer warps, 16 tokens of each tile
constexpr int kBoxCols = 64;       // channels per tensor-copy box: 128 bytes, the swizzle span
constexpr int kBoxBytes = kTile * kBoxCols * 2;
constexpr int kPCols = 16;         // p tile columns: hi parts, lo parts
constexpr int kPStride = 24;       // p tile row (bf16): 16 tokens + 8 padding
constexpr int kMaxGridB = 256;     // CTAs at most

template <int D, int HPK>
struct BCfg {
  static constexpr int kBoxes = D / kBoxCols;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;  // one K (or V) tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStages = (192 * 1024) / kStageBytes < 12 ? (192 * 1024) / kStageBytes : 12;
  static constexpr bool kLoCols = HPK <= 4;  // lo parts in the free columns
  static constexpr int kState = HPK * (D + 2);  // m[HPK], l[HPK], acc[HPK][D]
  static constexpr int kOffP = kStages * kStageBytes;
  static constexpr int kOffMerge = kOffP + kCW * kPCols * kPStride * 2;
  static constexpr int kOffBars = kOffMerge + kCW * kState * 4;
  static constexpr int kBytes = kOffBars + 2 * kStages * 8 + 16 + 1024;  // + alignment slack
  static constexpr int kThreads = (kCW + 1) * 32;
  static_assert(kOffP % 1024 == 0, "stages keep the 1024-byte alignment of the swizzle");
  static_assert(kBytes <= 227 * 1024, "shared-memory plan");
};

struct BSplit {
  int pairs, nt, S, Smax;  // nt: tiles per pair
  int n, q, rem;           // CTAs; tiles pairs*nt = n*q + rem
};

__host__ __device__ inline long b_lo(const BSplit& s, int c) {
  return (long)c * s.q + (c < s.rem ? c : s.rem);
}
__host__ __device__ inline int b_cta_of(const BSplit& s, long tile) {
  const long big = (long)s.rem * (s.q + 1);
  return (int)(tile < big ? tile / (s.q + 1) : s.rem + (tile - big) / s.q);
}

struct Bf16Args {
  const __nv_bfloat16* q;
  float* out;
  uint32_t* status;
  int* tickets;
  float* partials;  // [kMaxGridB][2][HPK][D + 2]
  int Hq, Hkv;
  float sm_scale;
};

// The partial slot of CTA c for pair p: 0 for its first pair, 1 for its last.
template <int D, int HPK>
__device__ __forceinline__ float* b_slot(const Bf16Args& a, const BSplit& sp, int c, int p) {
  const int first = (int)(b_lo(sp, c) / sp.nt);
  return a.partials + ((long)c * 2 + (p == first ? 0 : 1)) * BCfg<D, HPK>::kState;
}

template <int D, int HPK>
__global__ void __launch_bounds__(BCfg<D, HPK>::kThreads, 1)
bf16_decode_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                   Bf16Args a, BSplit sp) {
  using C = BCfg<D, HPK>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* empty = full + C::kStages;
  int* s_flag = reinterpret_cast<int*>(empty + C::kStages);  // the ticket's verdict
  volatile int* s_abort = s_flag + 1;   // a wait of this CTA ran out: stop streaming
  volatile int* s_issued = s_flag + 2;  // tiles the producer issued
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const long t_begin = b_lo(sp, cta), t_end = b_lo(sp, cta + 1);
  const int n_tiles = (int)(t_end - t_begin);

  if (threadIdx.x == 0) {
    *s_abort = 0;
    *s_issued = 0;
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    fence_mbar_init();
  }
  {  // p tiles start at zero: columns of absent heads stay zero
    uint32_t* pt = reinterpret_cast<uint32_t*>(smem + C::kOffP);
    for (int i = threadIdx.x; i < kCW * kPCols * kPStride / 2; i += C::kThreads) pt[i] = 0u;
  }
  __syncthreads();
  wait_for_predecessor();  // q may come from the previous kernel

  if (warp == kCW) {
    // ---- producer: one lane streams the CTA's tiles through the stages ----
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % C::kStages;
        if (*s_abort) break;
        if (i >= C::kStages &&
            !mbar_wait_bounded(&empty[s], (uint32_t)((i / C::kStages) - 1) & 1u)) {
          atomicOr(a.status, kStatusWaitTimeoutB);
          *s_abort = 1;
          break;
        }
        const long tile = t_begin + i;
        const int pair = (int)(tile / sp.nt), j = (int)(tile % sp.nt);
        const int y = pair * sp.Smax + j * kTile;
        unsigned char* st = smem + s * C::kStageBytes;
        mbar_expect_tx(&full[s], C::kStageBytes);
#pragma unroll
        for (int b = 0; b < C::kBoxes; ++b) {
          tma_load_2d(st + b * kBoxBytes, &tk, b * kBoxCols, y, &full[s]);
          tma_load_2d(st + C::kTileBytes + b * kBoxBytes, &tv, b * kBoxCols, y, &full[s]);
        }
        issued = i + 1;
      }
      *s_issued = issued;
    }
    __syncwarp();
    named_sync(2, C::kThreads);  // the consumers read s_issued after this
    return;
  }

  // ---- consumers: warp w takes tokens 16w .. 16w+15 of every tile ----
  const int g = lane >> 2, tig = lane & 3;
  const int r0 = 16 * warp;
  const float qscale = (a.sm_scale > 0.f ? a.sm_scale : rsqrtf((float)D)) * kLog2eB;
  __nv_bfloat16* p_tile = reinterpret_cast<__nv_bfloat16*>(smem + C::kOffP) + warp * kPCols * kPStride;
  float* merge = reinterpret_cast<float*>(smem + C::kOffMerge);
  constexpr int kKS = D / 16, kMT = D / 16;
  constexpr int kNB = C::kLoCols ? 1 : 2;  // P.V column blocks (hi+lo, or hi and lo)

  uint32_t qf[kKS][2];     // score B operand: q[head g][16s + 2tig ..], [16s + 8 + 2tig ..]
  float m_run[2], l_part[2];  // heads 2tig, 2tig+1 (score columns)
  float acc[kNB][kMT][4];
  int cur_pair = -1;
  bool dead = false;  // this warp stopped consuming (a wait ran out somewhere in the CTA)
  int i_dead = n_tiles;

  auto reset = [&]() {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      m_run[e] = -INFINITY;
      l_part[e] = 0.f;
    }
#pragma unroll
    for (int nb = 0; nb < kNB; ++nb)
#pragma unroll
      for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
        for (int r = 0; r < 4; ++r) acc[nb][mt][r] = 0.f;
  };

  // Merges the four warps' states of `pair` and writes its output or partial;
  // the last CTA of a shared pair merges the partials.
  auto flush = [&](int pair) {
    // l over this warp's 16 tokens, per score column
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      l_part[e] += __shfl_xor_sync(0xffffffffu, l_part[e], 4);
      l_part[e] += __shfl_xor_sync(0xffffffffu, l_part[e], 8);
      l_part[e] += __shfl_xor_sync(0xffffffffu, l_part[e], 16);
    }
    float* mine = merge + warp * C::kState;
    if (g == 0) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int h = 2 * tig + e;
        if (h < HPK) {
          mine[h] = m_run[e];
          mine[HPK + h] = l_part[e];
        }
      }
    }
    // acc column -> head: hi + lo of the same head
#pragma unroll
    for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        float v = acc[0][mt][r];
        if constexpr (C::kLoCols) {
          v += __shfl_xor_sync(0xffffffffu, v, 2);  // columns 4 + h sit two lanes over
        } else {
          v += acc[1][mt][r];
        }
        const int h = 2 * tig + (r & 1);
        const int d = 16 * mt + g + 8 * (r >> 1);
        if ((C::kLoCols ? tig < 2 : true) && h < HPK) mine[2 * HPK + h * D + d] = v;
      }
    named_sync(1, kCW * 32);
    const int b = pair / a.Hkv, kvh = pair % a.Hkv;
    const long first_tile = (long)pair * sp.nt, last_tile = first_tile + sp.nt - 1;
    const bool whole = first_tile >= t_begin && last_tile < t_end;
    float* part = whole ? nullptr : b_slot<D, HPK>(a, sp, cta, pair);
    for (int idx = threadIdx.x; idx < HPK * (D + 1); idx += kCW * 32) {
      const int h = idx / (D + 1), d = idx % (D + 1);  // d == D: the (m, l) entry
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kCW; ++w) M = fmaxf(M, merge[w * C::kState + h]);
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kCW; ++w) {
        const float* src = merge + w * C::kState;
        const float f = src[h] == -INFINITY ? 0.f : fast_exp2(src[h] - M);
        sum += f * (d == D ? src[HPK + h] : src[2 * HPK + h * D + d]);
      }
      if (whole) {
        if (d < D) {
          float L = 0.f;
#pragma unroll
          for (int w = 0; w < kCW; ++w) {
            const float* src = merge + w * C::kState;
            L += src[h] == -INFINITY ? 0.f : fast_exp2(src[h] - M) * src[HPK + h];
          }
          a.out[((long)b * a.Hq + (long)kvh * HPK + h) * D + d] = sum / L;
        }
      } else if (d == D) {
        part[h] = M;
        part[HPK + h] = sum;
      } else {
        part[2 * HPK + h * D + d] = sum;
      }
    }
    named_sync(1, kCW * 32);  // the merge area is free again
    if (whole) return;
    // ---- ticket: the last CTA of the pair merges the partials ----
    __threadfence();
    named_sync(1, kCW * 32);
    const int c_first = b_cta_of(sp, first_tile), c_last = b_cta_of(sp, last_tile);
    if (threadIdx.x == 0) {
      const int old = atomicAdd(&a.tickets[pair], 1);
      *s_flag = old == c_last - c_first;
    }
    named_sync(1, kCW * 32);
    if (!*s_flag) return;
    __threadfence();
    for (int idx = threadIdx.x; idx < HPK * D; idx += kCW * 32) {
      const int h = idx / D, d = idx % D;
      float M = -INFINITY;
      for (int c = c_first; c <= c_last; ++c) M = fmaxf(M, __ldcg(b_slot<D, HPK>(a, sp, c, pair) + h));
      float L = 0.f, sum = 0.f;
      for (int c = c_first; c <= c_last; ++c) {
        const float* src = b_slot<D, HPK>(a, sp, c, pair);
        const float m = __ldcg(src + h);
        const float f = m == -INFINITY ? 0.f : fast_exp2(m - M);
        L += f * __ldcg(src + HPK + h);
        sum += f * __ldcg(src + 2 * HPK + h * D + d);
      }
      a.out[((long)b * a.Hq + (long)kvh * HPK + h) * D + d] = sum / L;
    }
    named_sync(1, kCW * 32);
    if (threadIdx.x == 0) a.tickets[pair] = 0;  // ready for the next call
  };

  reset();
  for (int i = 0; i < n_tiles; ++i) {
    const long tile = t_begin + i;
    const int pair = (int)(tile / sp.nt), j = (int)(tile % sp.nt);
    if (pair != cur_pair) {
      if (cur_pair >= 0) {
        flush(cur_pair);
        reset();
      }
      cur_pair = pair;
      // q of head g of this kv head (zero for absent heads)
      const __nv_bfloat16* qh =
          a.q + ((long)(pair / a.Hkv) * a.Hq + (long)(pair % a.Hkv) * HPK + g) * D;
#pragma unroll
      for (int s = 0; s < kKS; ++s) {
        qf[s][0] = g < HPK ? *reinterpret_cast<const uint32_t*>(qh + 16 * s + 2 * tig) : 0u;
        qf[s][1] = g < HPK ? *reinterpret_cast<const uint32_t*>(qh + 16 * s + 8 + 2 * tig) : 0u;
      }
    }
    // after a wait ran out, the warps keep to the same pair switches (their
    // merges meet on a named barrier) but consume nothing more
    const int s = i % C::kStages;
    if (!dead && __any_sync(0xffffffffu, *s_abort != 0)) {
      dead = true;
      i_dead = i;
    }
    if (!dead && !__all_sync(0xffffffffu,
                             mbar_wait_bounded(&full[s], (uint32_t)(i / C::kStages) & 1u))) {
      dead = true;
      i_dead = i;
      if (lane == 0) {
        atomicOr(a.status, kStatusWaitTimeoutB);
        *s_abort = 1;
      }
    }
    if (dead) continue;
    const int nv = min(16, sp.S - j * kTile - r0);  // valid tokens of this warp (may be <= 0)
    unsigned char* st = smem + s * C::kStageBytes;
    if (nv > 0) {
      const uint32_t kb = smem_addr(st), vb = smem_addr(st + C::kTileBytes);
      if (nv < 16) {  // rows past the last token: zero V (0 * stale data must stay 0)
        for (int x = lane; x < (16 - nv) * C::kBoxes * 8; x += 32) {
          const int row = r0 + nv + x / (C::kBoxes * 8), rest = x % (C::kBoxes * 8);
          *reinterpret_cast<uint4*>(st + C::kTileBytes + (rest / 8) * kBoxBytes + row * 128 +
                                    16 * (rest % 8)) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async();  // the stage's next tensor copy comes after these writes
        __syncwarp();
      }
      // ---- scores: rows = tokens r0 + (g, g + 8), columns = heads ----
      float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      const int lrow = r0 + (lane & 15);
#pragma unroll
      for (int ks = 0; ks < kKS; ++ks) {
        // matrices: (rows 0-7 | 8-15) x (channels 16ks + 0-7 | 8-15)
        const int ch = 16 * ks + 8 * (lane >> 4);
        const uint32_t addr = kb + (ch / kBoxCols) * kBoxBytes + lrow * 128 +
                              ((((ch % kBoxCols) >> 3) ^ (lrow & 7)) << 4);
        uint32_t kf[4];
        ldsm_x4(kf, addr);
        mma_bf16(sacc[ks & 1], kf[0], kf[1], kf[2], kf[3], qf[ks][0], qf[ks][1]);
      }
      // ---- online softmax, heads 2tig + e, tokens g and g + 8 ----
      float alpha[2], pr[2][2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float x0 = (sacc[0][e] + sacc[1][e]) * qscale;
        float x1 = (sacc[0][2 + e] + sacc[1][2 + e]) * qscale;
        if (g >= nv) x0 = -INFINITY;
        if (g + 8 >= nv) x1 = -INFINITY;
        float mx = fmaxf(x0, x1);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m_run[e], mx);  // finite: token r0 of the tile is valid
        alpha[e] = fast_exp2(m_run[e] - m_new);
        m_run[e] = m_new;
        pr[e][0] = fast_exp2(x0 - m_new);
        pr[e][1] = fast_exp2(x1 - m_new);
        l_part[e] = l_part[e] * alpha[e] + pr[e][0] + pr[e][1];
      }
      // p tile [column][token]: hi parts in columns h, lo parts in 4 + h (8 + h)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int h = 2 * tig + e;
        if (h < HPK) {
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const __nv_bfloat16 hi = __float2bfloat16_rn(pr[e][u]);
            const __nv_bfloat16 lo = __float2bfloat16_rn(pr[e][u] - __bfloat162float(hi));
            p_tile[h * kPStride + g + 8 * u] = hi;
            p_tile[((C::kLoCols ? 4 : 8) + h) * kPStride + g + 8 * u] = lo;
          }
        }
      }
      // rescale: accumulator columns 2tig + e hold head (2tig + e) & 3 (<= 4 heads) or 2tig + e
      float al[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        al[e] = C::kLoCols ? __shfl_sync(0xffffffffu, alpha[e], (lane & ~3) | (tig & 1)) : alpha[e];
      }
#pragma unroll
      for (int nb = 0; nb < kNB; ++nb)
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt) {
          acc[nb][mt][0] *= al[0];
          acc[nb][mt][1] *= al[1];
          acc[nb][mt][2] *= al[0];
          acc[nb][mt][3] *= al[1];
        }
      __syncwarp();
      // ---- P.V: A = V^T (channels x tokens) by ldmatrix.trans, B = p ----
      uint32_t pb[kNB][2];
#pragma unroll
      for (int nb = 0; nb < kNB; ++nb) {
        const __nv_bfloat16* col = p_tile + (8 * nb + g) * kPStride;
        pb[nb][0] = *reinterpret_cast<const uint32_t*>(col + 2 * tig);
        pb[nb][1] = *reinterpret_cast<const uint32_t*>(col + 8 + 2 * tig);
      }
      const int vrow = r0 + (lane & 7) + 8 * (lane >> 4);
#pragma unroll
      for (int mt = 0; mt < kMT; ++mt) {
        // matrices: (tokens 0-7 | 8-15) x (channels 16mt + 0-7 | 8-15)
        const int ch = 16 * mt + 8 * ((lane >> 3) & 1);
        const uint32_t addr = vb + (ch / kBoxCols) * kBoxBytes + vrow * 128 +
                              ((((ch % kBoxCols) >> 3) ^ (vrow & 7)) << 4);
        uint32_t vf[4];
        ldsm_x4_trans(vf, addr);
#pragma unroll
        for (int nb = 0; nb < kNB; ++nb)
          mma_bf16(acc[nb][mt], vf[0], vf[1], vf[2], vf[3], pb[nb][0], pb[nb][1]);
      }
    }
    // release the stage
    __syncwarp();
    if (lane == 0) {
      fence_proxy_async();
      mbar_arrive(&empty[s]);
    }
  }
  named_sync(2, C::kThreads);  // the producer is done issuing
  if (dead) {
    // the copies this warp did not see land (at most one per stage) get a
    // bounded chance to do so before the CTA's shared memory is released
    const int issued = *s_issued;
    for (int i = i_dead; i < issued; ++i)
      (void)mbar_wait_bounded(&full[i % C::kStages], (uint32_t)(i / C::kStages) & 1u);
  }
  allow_successor();
  if (cur_pair >= 0) flush(cur_pair);
}

BSplit make_bsplit(int pairs, int S, int Smax, int num_sms) {
  BSplit s{};
  s.pairs = pairs;
  s.S = S;
  s.Smax = Smax;
  s.nt = (S + kTile - 1) / kTile;
  const long T = (long)pairs * s.nt;
  long n = num_sms < kMaxGridB ? num_sms : kMaxGridB;
  if (n > T) n = T;
  s.n = (int)(n > 0 ? n : 1);
  s.q = (int)(T / s.n);
  s.rem = (int)(T % s.n);
  return s;
}

template <int D, int HPK>
cudaError_t launch_bf16_t(const Bf16DecodeArgs& x, cudaStream_t stream) {
  using C = BCfg<D, HPK>;
  int unused = 0;
  cudaError_t e = per_device_setup(x.device, &unused, [](int* v) {
    *v = 1;
    return cudaFuncSetAttribute(bf16_decode_kernel<D, HPK>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, C::kBytes);
  });
  if (e != cudaSuccess) return e;
  const long rows = (long)x.B * x.Hkv * x.Smax;
  CUtensorMap tk, tv;
  if (!encode_bf16_map(&tk, x.k, rows, D, kTile) || !encode_bf16_map(&tv, x.v, rows, D, kTile))
    return cudaErrorInvalidValue;
  const BSplit sp = make_bsplit(x.B * x.Hkv, x.S, x.Smax, x.num_sms);
  Bf16Args a{};
  a.q = x.q;
  a.out = x.out;
  a.status = x.status;
  a.tickets = x.tickets;
  a.partials = x.partials;
  a.Hq = x.Hq;
  a.Hkv = x.Hkv;
  a.sm_scale = x.sm_scale;
  e = launch_pdl(bf16_decode_kernel<D, HPK>, dim3(sp.n), dim3(C::kThreads), C::kBytes, stream,
                 tk, tv, a, sp);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_bf16_d(const Bf16DecodeArgs& x, cudaStream_t stream) {
  switch (x.Hq / x.Hkv) {
    case 1: return launch_bf16_t<D, 1>(x, stream);
    case 2: return launch_bf16_t<D, 2>(x, stream);
    case 4: return launch_bf16_t<D, 4>(x, stream);
    case 8: return launch_bf16_t<D, 8>(x, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

long bf16_partial_bytes(int D, int hpk) { return (long)kMaxGridB * 2 * hpk * (D + 2) * 4; }

cudaError_t launch_bf16_decode(const Bf16DecodeArgs& x, cudaStream_t stream) {
  if (x.S < 1 || x.S > x.Smax || (long)x.B * x.Hkv * x.Smax >= (1L << 31)) return cudaErrorInvalidValue;
  if (x.D == 128) return launch_bf16_d<128>(x, stream);
  if (x.D == 64) return launch_bf16_d<64>(x, stream);
  return cudaErrorInvalidValue;
}

}  // namespace kivi
