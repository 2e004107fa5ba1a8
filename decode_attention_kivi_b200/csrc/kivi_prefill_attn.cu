// kivi_prefill_attn.cu - causal attention of a prompt over its own keys and
// values on the fifth-generation tensor cores, with the KIVI quantize of the
// prompt fused into its epilogue.
//
// Prefill is the step on the other side of the decode path: the prompt's keys
// and values are attended once in full precision, and the history then lives
// in the cache as quantized groups while the newest tokens stay in bf16 (the
// "KIVI-2bit on Llama-3-8B (GQA)" record, "KV bytes basis"; "KIVI: A
// Tuning-Free Asymmetric 2bit Quantization for KV Cache": groups of 32, a
// residual of 128).
// For query head h of sequence b (kv head h / (Hq / Hkv)) and position i,
//   out[b][h][i] = sum_{j <= i} softmax_j(sm_scale * <q_i, k_j>) v_j.
//
// One CTA per (query tile of 128 positions, sequence, query head), the tiles
// with the most key tiles first.  Eight warps:
//   warp 4 (producer)  2D tensor copies of Q once and of K and V tiles of 128
//                      keys into two-stage rings (128-byte swizzle), the
//                      diagonal tile first, then towards key 0; a K stage is
//                      refilled once its scores are computed, a V stage once
//                      its product is;
//   warp 5 (MMA)       one thread issues S_j = Q K_j^T (M = N = 128, K = D) into
//                      one of two TMEM score buffers, and O += P_j V_j (M = 128,
//                      N = D, K = 128) into the TMEM output, each followed by a
//                      commit to an mbarrier;
//   warps 0-3          one query row per thread (its TMEM lane): the row of S_j
//                      from TMEM, the causal mask on the diagonal tile, the
//                      online softmax in base 2 with the weights computed while
//                      the tensor cores finish P_{j-1} V_{j-1}, then P_j as bf16
//                      into shared memory in the operand layout of the second
//                      MMA.  The output is rescaled in TMEM only when a row
//                      maximum grew by more than 2^8 (up to then the stale
//                      maximum is kept: the weights stay below 2^8 and O / l is
//                      unchanged);
//   warps 6-7          with the quantize on, in the CTAs of the longer half of
//                      the query tiles: this CTA's share of the groups of key
//                      tiles qt and nqt - 1 - qt (query head j < 4 of a kv head
//                      takes groups j, j + min(HPK, 4), ...): group records
//                      below NG(S), ring rows for tokens NG(S)*G .. S-1, with the
//                      quantizer of the quantize kernels, bit for bit, while the
//                      other warps run the attention.
// S_{j+1} is computed while the softmax works on S_j.
//
// TMEM: 512 columns (one CTA per SM): scores at columns 0 and 128, O at 256.
// Every mbarrier wait is bounded; a wait that runs out sets the status word,
// and every role drains what it issued before TMEM is released.
#include <cuda_bf16.h>

#include <cmath>

#include "kivi_kernels.h"
#include "kivi_launch.cuh"
#include "kivi_layout.cuh"
#include "kivi_ptx.cuh"
#include "kivi_quant.cuh"
#include "kivi_tcgen05.cuh"
#include "kivi_tmap.cuh"

namespace kivi {
namespace {

constexpr int kTileM = 128;                   // query rows per CTA = TMEM lanes
constexpr int kTileN = 128;                   // keys per tile
constexpr int kSoftWarps = 4;
constexpr int kProducerWarp = kSoftWarps;
constexpr int kMmaWarp = kSoftWarps + 1;
constexpr int kQuantWarp0 = kSoftWarps + 2;   // two warps that quantize the prompt
constexpr int kQuantThreadsPA = 64;           // (eight warps in all, two per SM sub-partition:
                                              // up to 255 registers per thread)
constexpr int kThreadsPA = (kSoftWarps + 2) * 32 + kQuantThreadsPA;
constexpr int kSlabBytes = 128 * 128;         // 64 bf16 columns of 128 rows
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kStatusWaitTimeoutPA = 1u;
constexpr float kLog2ePA = 1.4426950408889634f;
constexpr float kRescaleSlack = 8.f;          // log2 growth of a row max before O is rescaled
constexpr int kQuantBarrier = 1;              // named barrier of the quantize warps

template <int D>
struct PACfg {
  static constexpr int kSlabs = D / 64;
  static constexpr int kTileBytes = kSlabs * kSlabBytes;  // a Q, K or V tile
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = kOffQ + kTileBytes;       // stage s: K at 2s, V at 2s + 1
  static constexpr int kOffP = kOffKV + 4 * kTileBytes;
  static constexpr int kOffQuant = kOffP + 2 * kSlabBytes; // P: 128 rows x 128 keys
  static constexpr int kOffBars = kOffQuant + (int)sizeof(quant::QuantSmem<D>);
  static constexpr int kUsed = kOffBars + 256;
  // more than half of the SM's shared memory: one CTA per SM, which holds all
  // 512 TMEM columns
  static constexpr int kBytes = kUsed + 1024 > 120 * 1024 ? kUsed + 1024 : 120 * 1024;
  static constexpr uint32_t kColS = 0, kColO = 2 * kTileN;
  static_assert(kColO + D <= kTmemCols, "TMEM plan");
  static_assert(sizeof(quant::QuantSmem<D>) % 16 == 0, "barriers stay aligned");
  static_assert(kBytes <= 227 * 1024, "shared-memory plan");
};

struct PAParams {
  const __nv_bfloat16* k;  // the prompt's keys and values, read by the quantize warps
  const __nv_bfloat16* v;
  float* out;
  uint32_t* status;
  int B, Hkv, Hq, S, nqt, NG, ngcap;
  float scale_log2;
  uint8_t* records;
  __nv_bfloat16* ring_k;
  __nv_bfloat16* ring_v;
};

// Byte offset of (row, 8-column chunk c8) in a swizzled tile of 128 rows.
__device__ __forceinline__ int sw128_offset(int row, int c8) {
  return (c8 >> 3) * kSlabBytes + row * 128 + (((c8 & 7) ^ (row & 7)) << 4);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <int D, int BITS>
__global__ void __launch_bounds__(kThreadsPA, 1)
prefill_attention_kernel(const __grid_constant__ CUtensorMap tq,
                         const __grid_constant__ CUtensorMap tk,
                         const __grid_constant__ CUtensorMap tv, PAParams a) {
  using C = PACfg<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // K and V stages have their own barriers: a K stage is free once its scores
  // are computed, long before the V stage of the same tile.
  uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* k_full = q_full + 1;    // [2]
  uint64_t* k_empty = q_full + 3;   // [2]
  uint64_t* v_full = q_full + 5;    // [2]
  uint64_t* v_empty = q_full + 7;   // [2]
  uint64_t* s_full = q_full + 9;    // [2]
  uint64_t* p_full = q_full + 11;
  uint64_t* o_done = q_full + 12;
  uint64_t* drained = q_full + 13;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(q_full + 14);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = a.B * a.Hq;
  const int qt = a.nqt - 1 - (int)(blockIdx.x / BH);  // the longest rows first
  const int bh = (int)(blockIdx.x % BH);
  const int b = bh / a.Hq, hq = bh % a.Hq;
  const int hpk = a.Hq / a.Hkv, kvh = hq / hpk;
  const int nt = qt + 1;  // key tiles 0..qt
  const int q_row0 = bh * a.S + qt * kTileM;
  const int kv_row0 = (b * a.Hkv + kvh) * a.S;

  if (threadIdx.x == 0) {
    *s_abort = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
    }
    mbar_init(p_full, kSoftWarps * 32);
    mbar_init(o_done, 1);
    mbar_init(drained, 1);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tc::alloc(s_tmem, kTmemCols);
    tc::relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *s_tmem;
  auto fail = [&]() {
    *s_abort = 1;
    if (a.status != nullptr) atomicOr(a.status, kStatusWaitTimeoutPA);
  };

  if (warp == kProducerWarp) {
    if (lane == 0) {
      mbar_expect_tx(q_full, C::kTileBytes);
      for (int sl = 0; sl < C::kSlabs; ++sl)
        tma_load_2d(smem + C::kOffQ + sl * kSlabBytes, &tq, 64 * sl, q_row0, q_full);
      // tile j (the diagonal tile first, then towards key 0) goes to stage j mod 2;
      // K(j + 1) is issued before V(j): it is needed first and freed first
      auto issue = [&](int j, bool is_k) -> bool {
        const int st = j & 1;
        uint64_t* empty = is_k ? &k_empty[st] : &v_empty[st];
        if (j >= 2 && !mbar_wait_bounded(empty, ((j >> 1) - 1) & 1)) return false;
        if (*s_abort) return false;
        uint64_t* full = is_k ? &k_full[st] : &v_full[st];
        unsigned char* dst = smem + C::kOffKV + (2 * st + (is_k ? 0 : 1)) * C::kTileBytes;
        const int row = kv_row0 + (qt - j) * kTileN;
        mbar_expect_tx(full, C::kTileBytes);
        for (int sl = 0; sl < C::kSlabs; ++sl)
          tma_load_2d(dst + sl * kSlabBytes, is_k ? &tk : &tv, 64 * sl, row, full);
        return true;
      };
      int issued_k = 0, issued_v = 0;
      bool ok = issue(0, true);
      if (ok) issued_k = 1;
      for (int j = 0; ok && j < nt; ++j) {
        if (j + 1 < nt) {
          if (!(ok = issue(j + 1, true))) break;
          issued_k = j + 2;
        }
        if (!(ok = issue(j, false))) break;
        issued_v = j + 1;
      }
      if (!ok) fail();
      // every copy issued lands before the CTA may exit
      if (!mbar_wait_bounded(q_full, 0)) fail();
      for (int j = issued_k > 2 ? issued_k - 2 : 0; j < issued_k; ++j)
        if (!mbar_wait_bounded(&k_full[j & 1], (j >> 1) & 1)) fail();
      for (int j = issued_v > 2 ? issued_v - 2 : 0; j < issued_v; ++j)
        if (!mbar_wait_bounded(&v_full[j & 1], (j >> 1) & 1)) fail();
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t id_s = tc::idesc_bf16(kTileM, kTileN, false);
      constexpr uint32_t id_o = tc::idesc_bf16(kTileM, D, true);
      const uint32_t q_base = smem_addr(smem + C::kOffQ);
      const uint32_t p_base = smem_addr(smem + C::kOffP);
      auto issue_scores = [&](int j) {
        const int st = j & 1;
        const uint32_t k_base = smem_addr(smem + C::kOffKV + 2 * st * C::kTileBytes);
#pragma unroll
        for (int s = 0; s < D / 16; ++s) {  // k-steps over the head dimension
          const uint32_t off = (s >> 2) * kSlabBytes + (s & 3) * 32;
          tc::mma_bf16(tmem + C::kColS + st * kTileN, tc::desc_sw128(q_base + off, 16, 1024),
                       tc::desc_sw128(k_base + off, 16, 1024), id_s, s > 0);
        }
        tc::commit(&s_full[st]);
        tc::commit(&k_empty[st]);
      };
      bool ok = mbar_wait_bounded(q_full, 0) && mbar_wait_bounded(&k_full[0], 0);
      if (ok) {
        tc::fence_after();
        issue_scores(0);
      }
      for (int j = 0; ok && j < nt; ++j) {
        if (j + 1 < nt) {
          if (!mbar_wait_bounded(&k_full[(j + 1) & 1], ((j + 1) >> 1) & 1)) {
            ok = false;
            break;
          }
          tc::fence_after();
          issue_scores(j + 1);  // its buffer was read by the softmax of tile j - 1
        }
        if (!mbar_wait_bounded(p_full, j & 1) || !mbar_wait_bounded(&v_full[j & 1], (j >> 1) & 1) ||
            *s_abort) {
          ok = false;
          break;
        }
        tc::fence_after();
        const uint32_t v_base =
            smem_addr(smem + C::kOffKV + (2 * (j & 1) + 1) * C::kTileBytes);
#pragma unroll
        for (int s = 0; s < kTileN / 16; ++s) {  // k-steps over the keys
          const uint32_t a_off = (s >> 2) * kSlabBytes + (s & 3) * 32;
          tc::mma_bf16(tmem + C::kColO, tc::desc_sw128(p_base + a_off, 16, 1024),
                       tc::desc_sw128(v_base + s * 16 * 128, kSlabBytes, 1024), id_o,
                       j > 0 || s > 0);
        }
        tc::commit(&v_empty[j & 1]);
        tc::commit(o_done);
      }
      if (!ok) fail();
      // all MMAs issued have completed before TMEM is released
      tc::commit(drained);
      if (!mbar_wait_bounded(drained, 0)) fail();
    }
  } else if (warp < kSoftWarps) {
    // Softmax warps: thread r owns query row r of the tile (TMEM lane r).
    const int r = threadIdx.x;
    const int qpos = qt * kTileM + r;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    unsigned char* prow = smem + C::kOffP;
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) {
      const bool w = mbar_wait_bounded(bar, parity);
      return __all_sync(0xffffffffu, w && !*s_abort);
    };
    const float sl2 = a.scale_log2;
    float m = -INFINITY, l = 0.f;  // running max (log2 units) and sum of the row's weights
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int st = j & 1;
      if (!wait_warp(&s_full[st], (j >> 1) & 1)) {
        ok = false;
        break;
      }
      tc::fence_after();
      float s[kTileN];
      tc::ld_x128(lane_base + C::kColS + st * kTileN, s);
      if (j == 0) {  // the diagonal tile: keys after the query are masked
#pragma unroll
        for (int c = 0; c < kTileN; ++c) s[c] = c <= r ? s[c] : -INFINITY;
      }
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = s[i];
#pragma unroll
      for (int c = 8; c < kTileN; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], s[c]);
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      // scores scaled into log2 units inside the exponent's FMA (sl2 > 0 keeps the max)
      const float m_new = fmaxf(m, mx * sl2);
      const bool grow = m_new > m + kRescaleSlack;  // always at the first tile (m = -inf)
      const float m_use = grow ? m_new : m;
      const float alpha = fast_exp2(m - m_use);     // 1 when kept, 0 at the first tile
      // the weights of this tile while the tensor cores still work on the last one
      uint32_t pk[kTileN / 2];
      float sum4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < kTileN; c += 2) {
        const float p0 = fast_exp2(fmaf(s[c], sl2, -m_use));
        const float p1 = fast_exp2(fmaf(s[c + 1], sl2, -m_use));
        sum4[(c >> 1) & 3] += p0 + p1;
        pk[c >> 1] = pack_bf16x2(p0, p1);
      }
      if (j > 0) {
        // O holds P_{j-1} V_{j-1}, and the P buffer is free again
        if (!wait_warp(o_done, (j - 1) & 1)) {
          ok = false;
          break;
        }
        tc::fence_after();
        if (__any_sync(0xffffffffu, grow)) {  // TMEM loads and stores are warp-wide
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            float o[32];
            tc::ld_x32(lane_base + C::kColO + c0, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tc::st_x32(lane_base + C::kColO + c0, o);
          }
          tc::wait_st();
        }
      }
#pragma unroll
      for (int c8 = 0; c8 < kTileN / 8; ++c8)
        *reinterpret_cast<uint4*>(prow + sw128_offset(r, c8)) =
            make_uint4(pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]);
      l = l * alpha + ((sum4[0] + sum4[1]) + (sum4[2] + sum4[3]));
      m = m_use;
      fence_proxy_async();  // P is read by the tensor cores
      tc::fence_before();
      mbar_arrive(p_full);
    }
    if (ok) ok = wait_warp(o_done, (nt - 1) & 1);
    if (ok) {
      tc::fence_after();
      const float inv = 1.f / l;
      float* orow = a.out + ((long)bh * a.S + qpos) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        float o[32];
        tc::ld_x32(lane_base + C::kColO + c0, o);
        if (qpos < a.S) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(orow + c0 + i) =
                make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv);
        }
      }
    } else {
      fail();
    }
  } else {
    // Quantize warps, running beside the attention: the CTAs of query tile qt
    // with qt >= nqt - 1 - qt (the longer half) quantize key tile qt and its
    // partner tile nqt - 1 - qt, so the work hides under their longer attention
    // and every tile is taken once.  Query head j < 4 of a kv head takes groups
    // j, j + min(HPK, 4), ... of a tile's four.  Rows are read from global
    // memory (tile qt right behind the producer's copy; low tiles are read by
    // every CTA of the kv head and stay in L2).
    const int hi = hq % hpk, nq = hpk < 4 ? hpk : 4;
    const int partner = a.nqt - 1 - qt;
    if (a.records != nullptr && hi < 4 && qt >= partner) {
      constexpr RecordGeom geo{D, BITS};
      const int qtid = threadIdx.x - kQuantWarp0 * 32;
      auto& qs = *reinterpret_cast<quant::QuantSmem<D>*>(smem + C::kOffQuant);
      const long seq = (long)b * a.Hkv + kvh;
      const __nv_bfloat16* ks = a.k + seq * a.S * D;
      const __nv_bfloat16* vs = a.v + seq * a.S * D;
      auto sync = [] { named_sync(kQuantBarrier, kQuantThreadsPA); };
      for (int u = 0; u < (partner == qt ? 1 : 2); ++u) {
        const int tile = u == 0 ? qt : partner;
        for (int gi = hi; gi < kTileN / kGroup; gi += nq) {
          const int t0 = tile * kTileN + gi * kGroup;  // the group's first token
          if (t0 >= a.S) break;
          const int g = t0 / kGroup;
          if (g < a.NG) {
            quant::load_tile<D, kQuantThreadsPA>(qs.k, ks + (long)t0 * D, D, qtid);
            quant::load_tile<D, kQuantThreadsPA>(qs.v, vs + (long)t0 * D, D, qtid);
            sync();
            uint8_t* rec = a.records + (seq * a.ngcap + g) * geo.bytes();
            quant::quantize_tiles_to_record<D, BITS, kQuantThreadsPA>(
                qs, reinterpret_cast<uint32_t*>(rec), qtid, sync);
            sync();  // the tiles are refilled by the next group
          } else {
            // residual tokens t0 .. min(t0 + G, S) - 1 to ring slots t mod (R + G)
            const int n = (t0 + kGroup < a.S ? t0 + kGroup : a.S) - t0;
            for (int i = qtid; i < n * (D / 8); i += kQuantThreadsPA) {
              const int t = t0 + i / (D / 8), c = i % (D / 8);
              const long dst = (seq * kRingSlots + t % kRingSlots) * D;
              reinterpret_cast<uint4*>(a.ring_k + dst)[c] =
                  reinterpret_cast<const uint4*>(ks + (long)t * D)[c];
              reinterpret_cast<uint4*>(a.ring_v + dst)[c] =
                  reinterpret_cast<const uint4*>(vs + (long)t * D)[c];
            }
          }
        }
      }
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc::fence_after();
    tc::dealloc(tmem, kTmemCols);
  }
}

template <int D, int BITS>
cudaError_t launch_pa_t(const PrefillAttnArgs& x, cudaStream_t stream) {
  using C = PACfg<D>;
  int unused = 0;
  cudaError_t e = per_device_setup(x.device, &unused, [](int* v) {
    *v = 1;
    return cudaFuncSetAttribute(prefill_attention_kernel<D, BITS>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, C::kBytes);
  });
  if (e != cudaSuccess) return e;
  CUtensorMap tq, tk, tv;
  if (!encode_bf16_map(&tq, x.q, (long)x.B * x.Hq * x.S, D, kTileM) ||
      !encode_bf16_map(&tk, x.k, (long)x.B * x.Hkv * x.S, D, kTileN) ||
      !encode_bf16_map(&tv, x.v, (long)x.B * x.Hkv * x.S, D, kTileN))
    return cudaErrorInvalidValue;
  PAParams p{};
  p.k = x.k;
  p.v = x.v;
  p.out = x.out;
  p.status = x.status;
  p.B = x.B;
  p.Hkv = x.Hkv;
  p.Hq = x.Hq;
  p.S = x.S;
  p.nqt = (x.S + kTileM - 1) / kTileM;
  p.NG = num_groups(x.S);
  p.ngcap = x.ngcap;
  const float scale = x.sm_scale > 0.f ? x.sm_scale : 1.f / std::sqrt((float)D);
  p.scale_log2 = scale * kLog2ePA;
  p.records = x.records;
  p.ring_k = x.ring_k;
  p.ring_v = x.ring_v;
  const long grid = (long)p.nqt * x.B * x.Hq;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreadsPA);
  cfg.dynamicSmemBytes = C::kBytes;
  cfg.stream = stream;
  e = cudaLaunchKernelEx(&cfg, prefill_attention_kernel<D, BITS>, tq, tk, tv, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_attention(int D, int bits, const PrefillAttnArgs& x,
                                     cudaStream_t stream) {
  if (x.S < 1 || x.B < 1 || x.Hkv < 1 || x.Hq < x.Hkv || x.Hq % x.Hkv != 0)
    return cudaErrorInvalidValue;
  // tensor-copy row coordinates and the grid stay in int
  if ((long)x.B * x.Hq * (x.S + kTileM) >= (1L << 31)) return cudaErrorInvalidValue;
  if (D == 128 && bits == 2) return launch_pa_t<128, 2>(x, stream);
  if (D == 128 && bits == 4) return launch_pa_t<128, 4>(x, stream);
  if (D == 64 && bits == 2) return launch_pa_t<64, 2>(x, stream);
  if (D == 64 && bits == 4) return launch_pa_t<64, 4>(x, stream);
  return cudaErrorInvalidValue;
}

}  // namespace kivi
