// kivi_attn.cu - fused single-token decode attention over the packed KIVI cache.
//
// For query head h of sequence b (kv head h / (Hq/Hkv)), over all S cached tokens:
//   s_t = sm_scale * <q, k_t>,  out = sum_t softmax(s)_t v_t,
// where k_t, v_t are the dequantized codes (scale_h * code + min_h) for the
// NG(S)*32 grouped tokens and the bf16 residual ring for the rest (record
// "kv-efficiency/kivi-2bit-llama3-8b-gqa-8k", "KV bytes basis": the most recent
// R tokens stay full precision).  Grouped history and residual share one
// online softmax.
//
// Group CTAs (split < splits_g of each sequence and kv head; one wave of 4 CTAs
// per SM): each warp streams whole 32-token group
// records (one contiguous block each) into its own shared-memory ring with
// cp.async.bulk on mbarriers, and does both contractions on the tensor cores
// (mma.sync m16n8k16, fp16 operands, fp32 accumulation):
//   scores  C[token][head] = sum_d code[token][d] * (q''[head][d] * kscale[d])
//                          + sum_d kmin[d] * q''[head][d]
//           with q'' * kscale carried as an fp16 pair hi + lo (two MMAs sharing
//           the code operand) so the scores keep about 22 significant bits
//   P.V     C[chan][head] += sum_t code[t][chan] * (p[head][t] * vscale[t][j])
//                          + sum_t vmin[t][j] * p[head][t]
// The codes become exact fp16 small integers with one three-input logic op and
// one add per pair (the packing puts adjacent codes in the two halves of a word); the
// scale and the min fold into the other operand, so nothing is dequantized
// element by element.  The min terms are MMAs whose A rows all repeat the min
// vector.  q'' = q * 2^-e_h (exact) keeps |q''| < 1 so q'' * kscale stays in
// fp16 range; scores are rescaled by 2^e_h * sm_scale * log2(e) in fp32.
//
// Residual-chunk CTAs (after the group CTAs in the grid; they fill the SMs the
// group CTAs leave free): 32 bf16 ring tokens each, on CUDA cores.
// Every CTA writes one (m, l, acc) partial per query head; combine_kernel
// merges the partials.  Every wait on an mbarrier is bounded; a wait that runs
// out sets the device status word and the CTA stops issuing work.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kivi_kernels.h"
#include "kivi_launch.cuh"
#include "kivi_layout.cuh"

namespace kivi {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 4;
// Row stride (fp16 entries) of a warp's p tile [8 heads][64 tokens]: 64 plus 8 of
// padding, so that the eight rows a P.V operand load touches fall in distinct
// banks (a 64-entry row is 128 bytes: every row would start in bank 0).
constexpr int kPRow = 2 * 32 + 8;
constexpr float kLog2e = 1.4426950408889634f;
constexpr long long kWaitBudgetCycles = 4000000000LL;  // about 2 s at 1.9 GHz
constexpr uint32_t kStatusWaitTimeout = 1u;
constexpr int kMaxResidualChunks = (kRingSlots + kGroup - 1) / kGroup;  // residual < R + G tokens

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// Bulk copy global -> this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// One test of the phase; the warp is suspended in hardware (not spinning) for
// up to kSuspendHintNs while the phase is incomplete.
constexpr uint32_t kSuspendHintNs = 1000000u;
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return done != 0;
}

// Waits for phase `parity` of `bar` for at most kWaitBudgetCycles.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitBudgetCycles) return false;
  }
  return true;
}

__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// ---------------------------------------------------------------------------
// Codes -> exact fp16 pairs
// ---------------------------------------------------------------------------

// The two codes at bit offset P of each 16-bit half of w, as fp16x2 (c_lo, c_hi).
// OR-ing the masked bits under the fp16 exponent of 2^(10-P) puts the code bits
// at weight 1: the half is 2^(10-P) + c exactly (P + BITS <= 10), and one add
// of -2^(10-P) leaves c.  The magic constants live in registers (CodeConsts).
template <int BITS>
struct CodeConsts {
  static constexpr int kNumP = BITS == 2 ? 5 : 2;  // offsets P = 0, b, 2b, ... below 10
  uint32_t magic[kNumP];                           // fp16x2 2^(10-P)
  uint32_t neg[kNumP];                             // fp16x2 -2^(10-P)
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int i = 0; i < kNumP; ++i) {
      const uint32_t e = (uint32_t)(25 - i * BITS) << 10;
      magic[i] = e | (e << 16);
      neg[i] = magic[i] | 0x80008000u;
      // opaque to the compiler: keep the constants in registers instead of
      // rematerializing them at every use
      asm volatile("" : "+r"(magic[i]), "+r"(neg[i]));
    }
  }
};

__device__ __forceinline__ uint32_t hadd2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// (w & mask) | magic as one three-input logic op (LUT 0xEA = (a & b) | c); the
// two-operator C form costs two instructions.
template <uint32_t MASK>
__device__ __forceinline__ uint32_t and_or(uint32_t w, uint32_t magic) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(w), "n"(MASK), "r"(magic));
  return d;
}

template <int BITS, int P>
__device__ __forceinline__ uint32_t code_pair(uint32_t w, const CodeConsts<BITS>& k) {
  static_assert(P + BITS <= 10 && P % BITS == 0, "code bits must lie inside the fp16 mantissa");
  constexpr uint32_t m = ((1u << BITS) - 1u) << P;
  return hadd2(and_or<m | (m << 16)>(w, k.magic[P / BITS]), k.neg[P / BITS]);
}

// Pair K (codes 2K and 2K+1) of a word; pairs past the fp16 mantissa come from
// the word shifted right by kHiShift.
template <int BITS>
struct CodeWord {
  static constexpr int kHiShift = BITS == 2 ? 10 : 8;
  template <int K>
  static __device__ __forceinline__ uint32_t pair(uint32_t w, uint32_t w_hi,
                                                  const CodeConsts<BITS>& k) {
    constexpr int off = K * BITS;
    if constexpr (off + BITS <= 10) {
      return code_pair<BITS, off>(w, k);
    } else {
      return code_pair<BITS, off - kHiShift>(w_hi, k);
    }
  }
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------------------
// Shared memory plan (dynamic)
// ---------------------------------------------------------------------------

template <int D, int BITS, int HPK>
struct Plan {
  static constexpr RecordGeom geo{D, BITS};
  static constexpr int kRec = (int)geo.bytes();             // bytes, multiple of 128
  static constexpr int kStageBytes = kWarps * kStages * kRec;
  static constexpr int kPBytes = kWarps * 8 * kPRow * 2;  // per warp p[8 heads][kPRow] fp16
  static constexpr int kQBytes = HPK * D * 4;               // q (fp32) of this kv head
  static constexpr int kMergeBytes = kWarps * HPK * D * 4;  // aliases the stages
  static_assert(kMergeBytes <= kStageBytes, "merge area must fit in the stage area");
  static constexpr int kResidPBytes = kWarps * HPK * kGroup * 4;  // residual p, aliases stages
  static_assert(kResidPBytes <= kStageBytes, "residual scratch must fit in the stage area");
  static constexpr int kOffP = kStageBytes;
  static constexpr int kOffQ = kOffP + kPBytes;
  static constexpr int kOffML = kOffQ + kQBytes;               // wm, wl [kWarps][8] each
  static constexpr int kOffBar = kOffML + 2 * kWarps * 8 * 4;  // [kWarps][kStages] mbarriers
  static constexpr int kBytes = kOffBar + kWarps * kStages * 8;
};

// ---------------------------------------------------------------------------
// The decode kernel
// ---------------------------------------------------------------------------

template <int D, int BITS, int HPK>
__global__ void __launch_bounds__(kThreads, HPK <= 4 ? 4 : 2)
decode_kernel(DecodeArgs args, int splits_g, int n_res, int groups_per_cta, float qscale) {
  // Linear grid: B*Hkv*splits_g group CTAs (split fastest), then B*Hkv*n_res
  // residual-chunk CTAs, which take the slots the group CTAs leave free.
  using P = Plan<D, BITS, HPK>;
  using CW = CodeWord<BITS>;
  constexpr RecordGeom geo = P::geo;
  constexpr int kKSteps = D / 16;            // score k-steps (16 channels each)
  constexpr int kMTiles = D / 16;            // P.V m-tiles (16 channels each)
  constexpr int kBlocks = D / 32;            // value channel blocks j
  constexpr int kThrWords = D * BITS / 128;  // K-code words one thread reads per token row
  constexpr int kChunks = HPK > 4 ? 2 : 1;   // score column chunks of 4 heads x {hi, lo}
  constexpr int kVWords = kMTiles * BITS / 2;  // V-code words one thread reads per group

  extern __shared__ __align__(128) unsigned char smem[];
  float* q_s = reinterpret_cast<float*>(smem + P::kOffQ);
  float* wm = reinterpret_cast<float*>(smem + P::kOffML);
  float* wl = wm + kWarps * 8;

  const int n_group_ctas = splits_g * args.Hkv * args.B;
  int split, kvh, b;
  if ((int)blockIdx.x < n_group_ctas) {
    split = blockIdx.x % splits_g;
    kvh = (blockIdx.x / splits_g) % args.Hkv;
    b = blockIdx.x / (splits_g * args.Hkv);
  } else {
    const int r = blockIdx.x - n_group_ctas;
    split = splits_g + r % n_res;
    kvh = (r / n_res) % args.Hkv;
    b = r / (n_res * args.Hkv);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hq = args.Hq, S = args.S;
  const long seq = (long)b * args.Hkv + kvh;
  const int NG = num_groups(S);

  const bool group_cta = split < splits_g;
  const int g = lane >> 2, tig = lane & 3;
  float* merge_acc = reinterpret_cast<float*>(smem);  // [kWarps][HPK][D], used after the loop
  // Group-CTA geometry: this warp's groups are first + warp, first + warp + kWarps, ...
  unsigned char* stage0 = smem + warp * kStages * P::kRec;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P::kOffBar) + warp * kStages;
  __half* p_s = reinterpret_cast<__half*>(smem + P::kOffP) + warp * 8 * kPRow;
  const int first = split * groups_per_cta;
  const int last = min(NG, first + groups_per_cta);
  const int n_mine =
      group_cta && first + warp < last ? (last - first - warp + kWarps - 1) / kWarps : 0;
  const uint8_t* seq_rec = args.records + seq * args.ngcap * (long)P::kRec;
  if (group_cta) {
    for (int i = lane; i < 8 * kPRow / 2; i += 32)
      reinterpret_cast<uint32_t*>(p_s)[i] = 0u;  // heads without a query stay finite
    if (lane == 0) {
      for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
      fence_mbar_init();
    }
  }

  wait_for_predecessor();  // q, the records and the rings may come from the previous kernel
  // q of this kv head's query heads (16-byte pieces): the loads go out before
  // the record stream so that they do not queue behind it
  constexpr int kQPieces = HPK * D / 8;
  static_assert(kQPieces <= kThreads, "one 16-byte piece of q per thread");
  uint4 qv = make_uint4(0u, 0u, 0u, 0u);
  if (threadIdx.x < kQPieces)  // the heads of kv head kvh are contiguous
    qv = reinterpret_cast<const uint4*>(args.q + ((long)b * Hq + kvh * HPK) * D)[threadIdx.x];
  if (group_cta && lane == 0) {
    for (int i = 0; i < kStages && i < n_mine; ++i) {
      mbar_expect_tx(&bars[i], P::kRec);
      bulk_load(stage0 + i * P::kRec, seq_rec + (long)(first + warp + i * kWarps) * P::kRec,
                P::kRec, &bars[i]);
    }
  }
  if (threadIdx.x < kQPieces) {  // q as fp32 in smem
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&qv);
    float4* dst = reinterpret_cast<float4*>(q_s + threadIdx.x * 8);
    const float2 f0 = __bfloat1622float2(h2[0]), f1 = __bfloat1622float2(h2[1]);
    const float2 f2 = __bfloat1622float2(h2[2]), f3 = __bfloat1622float2(h2[3]);
    dst[0] = make_float4(f0.x, f0.y, f1.x, f1.y);
    dst[1] = make_float4(f2.x, f2.y, f3.x, f3.y);
  }
  __syncthreads();

  if (group_cta) {
    // ===================== group CTA: tensor-core path =====================
    CodeConsts<BITS> kc;
    kc.init();

    // Score B operand: column n = g is head 4c + g/2 of chunk c, hi part for even
    // g and lo part for odd g.  qq = q''[head][channels c0..c0+3] per k-step,
    // c0 = tig*D/4 + 4s.  negm = -1 (odd g) or 0 (even g) in fp16x2.
    // Per-head exponent e_h with max |q_h| 2^-e_h in [0.5, 1), computed by every
    // warp: lanes [h L, (h+1) L) take head h (L = 32 / HPK lanes, D / L values each).
    int ex[HPK];
    {
      constexpr int kLanesPerHead = 32 / HPK;
      constexpr int kPerLane = D / kLanesPerHead;
      const float* qh = q_s + (lane / kLanesPerHead) * D + (lane % kLanesPerHead) * kPerLane;
      float mx = 0.f;
#pragma unroll
      for (int i = 0; i < kPerLane; ++i) mx = fmaxf(mx, fabsf(qh[i]));
#pragma unroll
      for (int o = 1; o < kLanesPerHead; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      int e = 0;
      if (mx > 0.f) frexpf(mx, &e);
#pragma unroll
      for (int hh = 0; hh < HPK; ++hh) ex[hh] = __shfl_sync(0xffffffffu, e, hh * kLanesPerHead);
    }
    uint32_t qq[kChunks][kKSteps][2];
    const uint32_t negm = (g & 1) ? 0xBC00BC00u : 0u;
    float ch[kChunks];  // log2 score scale of head 4c + tig
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      const int hs = 4 * c + g / 2;
      int es = 0, et = 0;
#pragma unroll
      for (int hh = 0; hh < HPK; ++hh) {
        es = hh == hs ? ex[hh] : es;
        et = hh == 4 * c + tig ? ex[hh] : et;
      }
#pragma unroll
      for (int s = 0; s < kKSteps; ++s) {
        const int c0 = tig * (D / 4) + 4 * s;
        if (hs < HPK) {
          const float sc = ldexpf(1.f, -es);
          const float* qr = q_s + hs * D + c0;
          qq[c][s][0] = pack_half2(qr[0] * sc, qr[1] * sc);
          qq[c][s][1] = pack_half2(qr[2] * sc, qr[3] * sc);
        } else {
          qq[c][s][0] = qq[c][s][1] = 0u;
        }
      }
      const int hh = 4 * c + tig;
      ch[c] = hh < HPK ? ldexpf(qscale, et) : 1.f;  // > 0 keeps -inf scores at p = 0
    }

    float acc[kMTiles][4];
    float vmacc[4] = {0.f, 0.f, 0.f, 0.f};  // sum_t vmin[t][j] p[h][t], row g -> block g % kBlocks
#pragma unroll
    for (int mt = 0; mt < kMTiles; ++mt)
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[mt][r] = 0.f;
    float m_run[kChunks], l_run[kChunks];
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      m_run[c] = -INFINITY;
      l_run[c] = 0.f;
    }

    bool timed_out = false;
    int i_stop = n_mine;
    for (int i = 0; i < n_mine; i += 2) {
      const bool has_b = i + 1 < n_mine;
      bool arrived = mbar_wait_bounded(&bars[i % kStages], (uint32_t)(i / kStages) & 1u);
      if (has_b)
        arrived = arrived && mbar_wait_bounded(&bars[(i + 1) % kStages],
                                               (uint32_t)((i + 1) / kStages) & 1u);
      if (!__all_sync(0xffffffffu, arrived)) {  // warp-uniform decision
        timed_out = true;
        i_stop = i;
        break;
      }
      const unsigned char* recs[2] = {stage0 + (i % kStages) * P::kRec,
                                      stage0 + ((has_b ? i + 1 : i) % kStages) * P::kRec};

      // ---- key-min term of both groups: rows g <- group A, rows g+8 <- group B ----
      float cmin[kChunks][4];
#pragma unroll
      for (int c = 0; c < kChunks; ++c)
#pragma unroll
        for (int r = 0; r < 4; ++r) cmin[c][r] = 0.f;
      {
        const __half* kmA = reinterpret_cast<const __half*>(recs[0] + geo.k_min_off());
        const __half* kmB = reinterpret_cast<const __half*>(recs[1] + geo.k_min_off());
#pragma unroll
        for (int s = 0; s < kKSteps; ++s) {
          const int c0 = tig * (D / 4) + 4 * s;
          const uint2 a = *reinterpret_cast<const uint2*>(kmA + c0);
          const uint2 bb = *reinterpret_cast<const uint2*>(kmB + c0);
#pragma unroll
          for (int c = 0; c < kChunks; ++c) mma_f16(cmin[c], a.x, bb.x, a.y, bb.y, qq[c][s][0], qq[c][s][1]);
        }
      }

      // ---- scores: sc[grp][c][mt][row half] ----
      float sc[2][kChunks][2][2];
#pragma unroll
      for (int grp = 0; grp < 2; ++grp) {
        const unsigned char* rec = recs[grp];
        const __half* kscale = reinterpret_cast<const __half*>(rec + geo.k_scale_off());
        uint32_t bq[kChunks][kKSteps][2];
#pragma unroll
        for (int s = 0; s < kKSteps; ++s) {
          const int c0 = tig * (D / 4) + 4 * s;
          const uint2 ks = *reinterpret_cast<const uint2*>(kscale + c0);
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
            // hi = RN(q'' s) for even g; lo = RN(q'' s - hi) for odd g
            bq[c][s][0] = hfma2(qq[c][s][0], ks.x, hmul2(hmul2(qq[c][s][0], ks.x), negm));
            bq[c][s][1] = hfma2(qq[c][s][1], ks.y, hmul2(hmul2(qq[c][s][1], ks.y), negm));
          }
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          float cacc[kChunks][4];
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
            // a missing second group scores -inf: p = 0, the max is unchanged
            cacc[c][0] = cacc[c][2] = (grp == 1 && !has_b) ? -INFINITY : cmin[c][2 * grp];
            cacc[c][1] = cacc[c][3] = 0.f;
          }
          const uint32_t* row0 = reinterpret_cast<const uint32_t*>(rec) +
                                 (16 * mt + g) * geo.k_row_words() + tig * kThrWords;
          const uint32_t* row1 = row0 + 8 * geo.k_row_words();
          uint32_t w0[kThrWords], w1[kThrWords];
          if constexpr (kThrWords == 4) {
            const uint4 x0 = *reinterpret_cast<const uint4*>(row0);
            const uint4 x1 = *reinterpret_cast<const uint4*>(row1);
            w0[0] = x0.x; w0[1] = x0.y; w0[2] = x0.z; w0[3] = x0.w;
            w1[0] = x1.x; w1[1] = x1.y; w1[2] = x1.z; w1[3] = x1.w;
          } else if constexpr (kThrWords == 2) {
            const uint2 x0 = *reinterpret_cast<const uint2*>(row0);
            const uint2 x1 = *reinterpret_cast<const uint2*>(row1);
            w0[0] = x0.x; w0[1] = x0.y;
            w1[0] = x1.x; w1[1] = x1.y;
          } else {
            w0[0] = row0[0];
            w1[0] = row1[0];
          }
#pragma unroll
          for (int w = 0; w < kThrWords; ++w) {
            const uint32_t h0 = w0[w] >> CW::kHiShift;
            const uint32_t h1 = w1[w] >> CW::kHiShift;
            constexpr int kStepsPerWord = 8 / BITS;
#pragma unroll
            for (int sw = 0; sw < kStepsPerWord; ++sw) {
              const int s = w * kStepsPerWord + sw;
              uint32_t a0, a1, a2, a3;
              if (sw == 0) {
                a0 = CW::template pair<0>(w0[w], h0, kc); a1 = CW::template pair<0>(w1[w], h1, kc);
                a2 = CW::template pair<1>(w0[w], h0, kc); a3 = CW::template pair<1>(w1[w], h1, kc);
              } else if (sw == 1) {
                a0 = CW::template pair<2>(w0[w], h0, kc); a1 = CW::template pair<2>(w1[w], h1, kc);
                a2 = CW::template pair<3>(w0[w], h0, kc); a3 = CW::template pair<3>(w1[w], h1, kc);
              } else if (sw == 2) {
                a0 = CW::template pair<4 % (16 / BITS)>(w0[w], h0, kc);
                a1 = CW::template pair<4 % (16 / BITS)>(w1[w], h1, kc);
                a2 = CW::template pair<5 % (16 / BITS)>(w0[w], h0, kc);
                a3 = CW::template pair<5 % (16 / BITS)>(w1[w], h1, kc);
              } else {
                a0 = CW::template pair<6 % (16 / BITS)>(w0[w], h0, kc);
                a1 = CW::template pair<6 % (16 / BITS)>(w1[w], h1, kc);
                a2 = CW::template pair<7 % (16 / BITS)>(w0[w], h0, kc);
                a3 = CW::template pair<7 % (16 / BITS)>(w1[w], h1, kc);
              }
#pragma unroll
              for (int c = 0; c < kChunks; ++c)
                mma_f16(cacc[c], a0, a1, a2, a3, bq[c][s][0], bq[c][s][1]);
            }
          }
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
            sc[grp][c][mt][0] = cacc[c][0] + cacc[c][1];  // token 16mt + g, head 4c + tig
            sc[grp][c][mt][1] = cacc[c][2] + cacc[c][3];  // token 16mt + g + 8
          }
        }
      }

      // ---- online softmax over the 64 tokens, head 4c + tig (log2 units) ----
      float alpha[kChunks];
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
        // max of the raw MMA scores (ch > 0 keeps the order), then log2 units
        float mx = fmaxf(fmaxf(fmaxf(sc[0][c][0][0], sc[0][c][0][1]),
                               fmaxf(sc[0][c][1][0], sc[0][c][1][1])),
                         fmaxf(fmaxf(sc[1][c][0][0], sc[1][c][0][1]),
                               fmaxf(sc[1][c][1][0], sc[1][c][1][1])));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m_run[c], mx * ch[c]);
        alpha[c] = fast_exp2(m_run[c] - m_new);
        m_run[c] = m_new;
        float sum = 0.f;
        __half* prow = p_s + (4 * c + tig) * kPRow;
#pragma unroll
        for (int grp = 0; grp < 2; ++grp)
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
              const float pv = fast_exp2(fmaf(sc[grp][c][mt][hr], ch[c], -m_new));
              sum += pv;
              prow[grp * kGroup + 16 * mt + 8 * hr + g] = __float2half_rn(pv);
            }
        l_run[c] = l_run[c] * alpha[c] + sum;
      }
      __syncwarp();

      // ---- rescale the P.V accumulators (columns = heads 2tig, 2tig+1) ----
      bool same = true;
#pragma unroll
      for (int c = 0; c < kChunks; ++c) same = same && alpha[c] == 1.f;
      if (!__all_sync(0xffffffffu, same)) {
        float al[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int h = 2 * tig + e;
          const int src = 4 * g + (h & 3);
          float v0 = __shfl_sync(0xffffffffu, alpha[0], src);
          if constexpr (kChunks == 2) {
            const float v1 = __shfl_sync(0xffffffffu, alpha[kChunks - 1], src);
            v0 = h >= 4 ? v1 : v0;
          }
          al[e] = v0;
        }
#pragma unroll
        for (int mt = 0; mt < kMTiles; ++mt) {
          acc[mt][0] *= al[0];
          acc[mt][1] *= al[1];
          acc[mt][2] *= al[0];
          acc[mt][3] *= al[1];
        }
        vmacc[0] *= al[0];
        vmacc[1] *= al[1];
        vmacc[2] *= al[0];
        vmacc[3] *= al[1];
      }

      // ---- P.V of both groups ----
#pragma unroll
      for (int grp = 0; grp < 2; ++grp) {
        const unsigned char* rec = recs[grp];
        const __half* vscale = reinterpret_cast<const __half*>(rec + geo.v_scale_off());
        const __half* vmin = reinterpret_cast<const __half*>(rec + geo.v_min_off());
        // B: p of head g, tokens (16kk + 8hf + 2tig, +1)
        uint32_t pb[2][2];
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
            pb[kk][hf] = *reinterpret_cast<const uint32_t*>(p_s + g * kPRow + grp * kGroup +
                                                            16 * kk + 8 * hf + 2 * tig);
        // value-min term, deferred: rows g -> block g % kBlocks
        {
          const uint4 vm = *reinterpret_cast<const uint4*>(vmin + 32 * (g % kBlocks) + 8 * tig);
          mma_f16(vmacc, vm.x, vm.x, vm.y, vm.y, pb[0][0], pb[0][1]);
          mma_f16(vmacc, vm.z, vm.z, vm.w, vm.w, pb[1][0], pb[1][1]);
        }
        // this thread's V-code words: (4g + tig) * kVWords ... + kVWords - 1
        const uint32_t* vw = reinterpret_cast<const uint32_t*>(rec + geo.v_codes_off()) +
                             (4 * g + tig) * kVWords;
        uint32_t vwords[kVWords];
#pragma unroll
        for (int q4 = 0; q4 < kVWords / 4; ++q4) {
          const uint4 x = *reinterpret_cast<const uint4*>(vw + 4 * q4);
          vwords[4 * q4] = x.x; vwords[4 * q4 + 1] = x.y;
          vwords[4 * q4 + 2] = x.z; vwords[4 * q4 + 3] = x.w;
        }
#pragma unroll
        for (int j = 0; j < kBlocks; ++j) {
          const uint4 vs = *reinterpret_cast<const uint4*>(vscale + 32 * j + 8 * tig);
          const uint32_t pt00 = hmul2(pb[0][0], vs.x), pt01 = hmul2(pb[0][1], vs.y);
          const uint32_t pt10 = hmul2(pb[1][0], vs.z), pt11 = hmul2(pb[1][1], vs.w);
#pragma unroll
          for (int mi = 0; mi < 2; ++mi) {
            const int mt = 2 * j + mi;
            if constexpr (BITS == 2) {
              const uint32_t x = vwords[mt], xh = x >> CW::kHiShift;
              // pairs idx = 4kk + 2hf + r: a0 (r0,hf0), a1 (r1,hf0), a2 (r0,hf1), a3 (r1,hf1)
              mma_f16(acc[mt], CW::template pair<0>(x, xh, kc), CW::template pair<1>(x, xh, kc),
                      CW::template pair<2>(x, xh, kc), CW::template pair<3>(x, xh, kc), pt00, pt01);
              mma_f16(acc[mt], CW::template pair<4>(x, xh, kc), CW::template pair<5>(x, xh, kc),
                      CW::template pair<6>(x, xh, kc), CW::template pair<7>(x, xh, kc), pt10, pt11);
            } else {
              const uint32_t x0 = vwords[2 * mt], x0h = x0 >> CW::kHiShift;
              const uint32_t x1 = vwords[2 * mt + 1], x1h = x1 >> CW::kHiShift;
              mma_f16(acc[mt], CW::template pair<0>(x0, x0h, kc), CW::template pair<1>(x0, x0h, kc),
                      CW::template pair<2>(x0, x0h, kc), CW::template pair<3>(x0, x0h, kc), pt00, pt01);
              mma_f16(acc[mt], CW::template pair<0>(x1, x1h, kc), CW::template pair<1>(x1, x1h, kc),
                      CW::template pair<2>(x1, x1h, kc), CW::template pair<3>(x1, x1h, kc), pt10, pt11);
            }
          }
        }
      }

      // release both stages and refill them with groups i + kStages, i + 1 + kStages
      __syncwarp();
      if (lane == 0) {
        fence_proxy_async();
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int k = i + e + kStages;
          if (i + e < n_mine && k < n_mine) {
            const int st = (i + e) % kStages;
            mbar_expect_tx(&bars[st], P::kRec);
            bulk_load(stage0 + st * P::kRec,
                      seq_rec + (long)(first + warp + k * kWarps) * P::kRec, P::kRec, &bars[st]);
          }
        }
      }
    }

    if (timed_out && lane == 0) {
      // record the failure, then give the copies already issued (local groups
      // i_stop .. i_stop + kStages - 1) a bounded chance to land before this
      // CTA's shared memory is reused
      atomicOr(args.status, kStatusWaitTimeout);
      for (int k = i_stop; k < n_mine && k < i_stop + kStages; ++k)
        (void)mbar_wait_bounded(&bars[k % kStages], (uint32_t)(k / kStages) & 1u);
    }
    // row sums over the 8 token lanes of each head
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      l_run[c] += __shfl_xor_sync(0xffffffffu, l_run[c], 4);
      l_run[c] += __shfl_xor_sync(0xffffffffu, l_run[c], 8);
      l_run[c] += __shfl_xor_sync(0xffffffffu, l_run[c], 16);
    }
    // add the deferred value-min term: block j of head 2tig+e sits in lane 4j + tig
#pragma unroll
    for (int j = 0; j < kBlocks; ++j) {
      const float v0 = __shfl_sync(0xffffffffu, vmacc[0], 4 * j + tig);
      const float v1 = __shfl_sync(0xffffffffu, vmacc[1], 4 * j + tig);
#pragma unroll
      for (int mi = 0; mi < 2; ++mi) {
        acc[2 * j + mi][0] += v0;
        acc[2 * j + mi][2] += v0;
        acc[2 * j + mi][1] += v1;
        acc[2 * j + mi][3] += v1;
      }
    }
    __syncthreads();  // every warp is done with its stages: the merge area may alias them
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      const int hh = 4 * c + tig;
      if (hh < HPK && g == 0) {
        wm[warp * 8 + hh] = n_mine > 0 ? m_run[c] : -INFINITY;
        wl[warp * 8 + hh] = n_mine > 0 ? l_run[c] : 0.f;
      }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int hh = 2 * tig + e;
      if (hh < HPK) {
#pragma unroll
        for (int mt = 0; mt < kMTiles; ++mt) {
          merge_acc[(warp * HPK + hh) * D + 16 * mt + g] = acc[mt][e];
          merge_acc[(warp * HPK + hh) * D + 16 * mt + g + 8] = acc[mt][e + 2];
        }
      }
    }
  } else {
    // ============ residual CTA: one chunk of <= 32 bf16 ring tokens, CUDA cores ============
    // The chunk's K and V rows are staged in shared memory (one coalesced pass;
    // a chunk starts at a multiple of 32 tokens, so its ring slots are
    // contiguous), then scores, the chunk softmax and P.V read shared memory.
    // This CTA writes its partial directly and returns.
    allow_successor();
    const int chunk = split - splits_g;
    const int t0 = NG * kGroup + chunk * kGroup;
    const int n = min(kGroup, S - t0);
    const int slot0 = t0 % kRingSlots;
    __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(smem);  // [32][D]
    __nv_bfloat16* vc = kc + kGroup * D;                          // [32][D]
    float* s_res = reinterpret_cast<float*>(vc + kGroup * D);     // [HPK][32]
    static_assert(2 * kGroup * D * 2 + HPK * kGroup * 4 <= P::kStageBytes,
                  "residual chunk must fit in the stage area");
    {
      // every load of the chunk is issued before the first store: one round trip
      const uint4* gk = reinterpret_cast<const uint4*>(args.ring_k + (seq * kRingSlots + slot0) * D);
      const uint4* gv = reinterpret_cast<const uint4*>(args.ring_v + (seq * kRingSlots + slot0) * D);
      const int n16 = n * D * 2 / 16;
      constexpr int kPer = (kGroup * D * 2 / 16 + kThreads - 1) / kThreads;
      uint4 rk[kPer], rv[kPer];
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int i = threadIdx.x + k * kThreads;
        if (i < n16) {
          rk[k] = gk[i];
          rv[k] = gv[i];
        }
      }
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int i = threadIdx.x + k * kThreads;
        if (i < n16) {
          reinterpret_cast<uint4*>(kc)[i] = rk[k];
          reinterpret_cast<uint4*>(vc)[i] = rv[k];
        }
      }
    }
    __syncthreads();
    // scores: one (token, head) pair per thread step; each thread walks the
    // channel pairs starting at an offset set by its token (spreads the banks)
    for (int pidx = threadIdx.x; pidx < kGroup * HPK; pidx += kThreads) {
      const int t = pidx / HPK, hh = pidx % HPK;
      float sum = -INFINITY;
      if (t < n) {
        sum = 0.f;
        const __nv_bfloat162* kr = reinterpret_cast<const __nv_bfloat162*>(kc + t * D);
        const float2* qr = reinterpret_cast<const float2*>(q_s + hh * D);
#pragma unroll 8
        for (int w = 0; w < D / 2; ++w) {
          const int ww = (w + t) & (D / 2 - 1);
          const float2 kf = __bfloat1622float2(kr[ww]);
          const float2 qf = qr[ww];
          sum = fmaf(kf.x, qf.x, fmaf(kf.y, qf.y, sum));
        }
        sum *= qscale;
      }
      s_res[hh * kGroup + t] = sum;
    }
    __syncthreads();
    // chunk softmax per head: warp w takes heads w, w + 4, ...
    for (int hh = warp; hh < HPK; hh += kWarps) {
      const float x = s_res[hh * kGroup + lane];
      float mx = x;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float pv = exp2f(x - mx);
      float l = pv;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      s_res[hh * kGroup + lane] = pv;
      if (lane == 0) {
        wm[hh] = mx;
        wl[hh] = l;
      }
    }
    __syncthreads();
    const int splits_total = splits_g + n_res;
    const long part0 = ((long)b * Hq + kvh * HPK) * splits_total + split;
    for (int i = threadIdx.x; i < HPK * D; i += kThreads) {
      const int hh = i / D, d = i % D;
      float o = 0.f;
      for (int t = 0; t < n; ++t)
        o = fmaf(s_res[hh * kGroup + t], __bfloat162float(vc[t * D + d]), o);
      args.ws_acc[(part0 + (long)hh * splits_total) * D + d] = o;
    }
    if (threadIdx.x < HPK) {
      const int hh = threadIdx.x;
      args.ws_ml[2 * (part0 + (long)hh * splits_total)] = wm[hh];
      args.ws_ml[2 * (part0 + (long)hh * splits_total) + 1] = wl[hh];
    }
    return;
  }

  allow_successor();
  // ===================== merge the warps, write this CTA's partial =====================
  __syncthreads();
  const int splits_total = splits_g + n_res;
  const long part0 = ((long)b * Hq + kvh * HPK) * splits_total + split;
  for (int i = threadIdx.x; i < HPK * D; i += kThreads) {
    const int hh = i / D, d = i % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, wm[w * 8 + hh]);
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float mw = wm[w * 8 + hh];
      if (mw != -INFINITY) o += exp2f(mw - M) * merge_acc[(w * HPK + hh) * D + d];
    }
    args.ws_acc[(part0 + (long)hh * splits_total) * D + d] = o;
  }
  if (threadIdx.x < HPK) {
    const int hh = threadIdx.x;
    float M = -INFINITY, L = 0.f;
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, wm[w * 8 + hh]);
    for (int w = 0; w < kWarps; ++w)
      if (wm[w * 8 + hh] != -INFINITY) L += wl[w * 8 + hh] * exp2f(wm[w * 8 + hh] - M);
    args.ws_ml[2 * (part0 + (long)hh * splits_total)] = M;
    args.ws_ml[2 * (part0 + (long)hh * splits_total) + 1] = L;
  }
}

// out[b][h] = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s.
// Warp 0 reads every split's (m, l) at once (two per lane, splits <= 64) and
// reduces them with shuffles; then every thread sums its channel over the
// splits with independent loads.
template <int D>
__global__ void __launch_bounds__(D) combine_kernel(DecodeArgs args, int splits) {
  static_assert(D >= 64, "warp 0 and the split weights need D >= 64 threads");
  __shared__ float f_s[kMaxSplitsCap];
  __shared__ float inv_l;
  wait_for_predecessor();  // every split's partial is written
  allow_successor();
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const long part0 = ((long)b * args.Hq + h) * splits;
  if (d < 32) {
    float m[2], l[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int s = d + 32 * k;
      m[k] = s < splits ? args.ws_ml[2 * (part0 + s)] : -INFINITY;
      l[k] = s < splits ? args.ws_ml[2 * (part0 + s) + 1] : 0.f;
    }
    float M = fmaxf(m[0], m[1]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float f = m[k] == -INFINITY ? 0.f : exp2f(m[k] - M);
      if (d + 32 * k < splits) f_s[d + 32 * k] = f;
      L += f * l[k];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (d == 0) inv_l = 1.f / L;
  }
  __syncthreads();
  const float* acc = args.ws_acc + part0 * D + d;
  float o0 = 0.f, o1 = 0.f;
  int s = 0;
#pragma unroll 4
  for (; s + 1 < splits; s += 2) {
    o0 = fmaf(f_s[s], acc[(long)s * D], o0);
    o1 = fmaf(f_s[s + 1], acc[(long)(s + 1) * D], o1);
  }
  if (s < splits) o0 = fmaf(f_s[s], acc[(long)s * D], o0);
  args.out[((long)b * args.Hq + h) * D + d] = (o0 + o1) * inv_l;
}

template <int D, int BITS, int HPK>
cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t stream) {
  using P = Plan<D, BITS, HPK>;
  // Per process (every device of a process is the same part): the largest
  // shared-memory carveout, and the CTAs per SM that the kernel really gets.
  static int ctas_per_sm = 0;
  if (ctas_per_sm == 0) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, BITS, HPK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, P::kBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(decode_kernel<D, BITS, HPK>,
                             cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_kernel<D, BITS, HPK>, kThreads,
                                                      P::kBytes);
    if (e != cudaSuccess) return e;
    ctas_per_sm = max(1, n);
  }
  const int NG = num_groups(a.S);
  const int pairs = a.B * a.Hkv;
  int splits_g = 0, gpc = 1;
  if (NG > 0) {
    const int want = max(1, (a.num_sms * ctas_per_sm) / pairs);   // one wave of group CTAs
    const int by_work = max(1, NG / (2 * kWarps));                 // >= 2 groups per warp
    splits_g = max(1, min(min(want, by_work), a.max_splits - kMaxResidualChunks));
    gpc = (NG + splits_g - 1) / splits_g;
    splits_g = (NG + gpc - 1) / gpc;  // every group split non-empty
  }
  const float qscale = (a.sm_scale > 0.f ? a.sm_scale : rsqrtf((float)D)) * kLog2e;
  const int r = a.S - NG * kGroup;                      // residual tokens, >= 1
  const int n_res = (r + kGroup - 1) / kGroup;           // residual chunks, <= 5
  const int n_ctas = (splits_g + n_res) * a.Hkv * a.B;
  cudaError_t e = launch_pdl(decode_kernel<D, BITS, HPK>, dim3(n_ctas), dim3(kThreads), P::kBytes,
                             stream, a, splits_g, n_res, gpc, qscale);
  if (e != cudaSuccess) return e;
  e = launch_pdl(combine_kernel<D>, dim3(a.Hq, a.B), dim3(D), 0, stream, a, splits_g + n_res);
  if (e != cudaSuccess) return e;
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
  if (a.max_splits < kMaxResidualChunks + 1) return cudaErrorInvalidValue;
  if (D == 128 && bits == 2) return launch_decode_d<128, 2>(a, stream);
  if (D == 128 && bits == 4) return launch_decode_d<128, 4>(a, stream);
  if (D == 64 && bits == 2) return launch_decode_d<64, 2>(a, stream);
  if (D == 64 && bits == 4) return launch_decode_d<64, 4>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace kivi
