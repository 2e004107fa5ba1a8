/*
 * kivi_oracle.c - plain, slow, CPU reference of the KIVI cache and decode
 * attention.  TEST INFRASTRUCTURE ONLY: the tests, the package's smoke check
 * and the benchmark's CPU-baseline leg may call it; the library path never
 * does.  It shares no code, header or table with the CUDA library: the packed
 * layout below is written here again from its definition.
 *
 * Sources (page title and section):
 *   [KIVI page]   "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache":
 *                 keys quantized per channel, values per token, asymmetric.
 *   [HF page]     "KV cache quantization squeezes 5GB down to fit longer LLM
 *                 generations": keys per channel, values per token; quantization
 *                 rounds values.
 *   [Llama-3 rec] "kv-efficiency/kivi-2bit-llama3-8b-gqa-8k", fields "Model",
 *                 "KV bytes basis", "Methodology": group size 32, residual 128,
 *                 the most recent R tokens kept in full precision, the grouped
 *                 term covering S - R tokens.
 *
 * Readings where the pages are silent (each one is a choice, listed in the
 * design notes): zero point = group min and scale = (max - min)/(2^b - 1) in
 * IEEE fp32; codes round half to even and are clamped to [0, 2^b - 1]; a
 * constant group has scale 0 and codes 0; metadata stored as fp16
 * round-to-nearest-even; the residual slides (it always holds the newest
 * r in [R, R + G) tokens once S >= R); softmax scale 1/sqrt(D) unless given.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC.
 * Float expressions are evaluated in single precision (SSE, FLT_EVAL_METHOD 0).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Number formats                                                           */
/* ------------------------------------------------------------------------ */

/* bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32 bits. */
static float bf16_bits_to_float(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* Round half to even of a non-negative double r (exactly representable). */
static double round_half_even_nonneg(double r) {
  double f = floor(r);
  double diff = r - f;
  if (diff > 0.5) return f + 1.0;
  if (diff < 0.5) return f;
  return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* fp32 -> IEEE binary16 bits, round to nearest, ties to even.  Binary16 has an
 * 11-bit significand for |v| >= 2^-14 and a fixed quantum of 2^-24 below it;
 * values that round to 65520 or more overflow to infinity. */
uint16_t oracle_f32_to_f16_bits(float x) {
  uint16_t sign = signbit(x) ? 0x8000u : 0u;
  double a = fabs((double)x);
  if (isnan(x)) return (uint16_t)(sign | 0x7e00u);
  if (isinf(x)) return (uint16_t)(sign | 0x7c00u);
  if (a == 0.0) return sign;
  int e2;
  frexp(a, &e2);          /* a = m * 2^e2, m in [0.5, 1) -> floor(log2 a) = e2 - 1 */
  int e = e2 - 1;
  if (e < -14) e = -14;   /* subnormal range shares the quantum of the lowest binade */
  double quantum = ldexp(1.0, e - 10);
  double n = round_half_even_nonneg(a / quantum); /* a / quantum is exact */
  double v = n * quantum;
  if (v >= 65520.0) return (uint16_t)(sign | 0x7c00u);
  if (v < ldexp(1.0, -14)) {
    return (uint16_t)(sign | (uint16_t)(v / ldexp(1.0, -24)));
  }
  frexp(v, &e2);
  int ev = e2 - 1;                                  /* v may have moved up a binade */
  uint32_t mant = (uint32_t)(v / ldexp(1.0, ev - 10)) - 1024u;
  return (uint16_t)(sign | (uint16_t)((ev + 15) << 10) | (uint16_t)mant);
}

/* IEEE binary16 bits -> double (exact). */
double oracle_f16_bits_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int exp = (h >> 10) & 0x1f;
  int mant = h & 0x3ff;
  double v;
  if (exp == 0) v = ldexp((double)mant, -24);
  else if (exp == 31) v = mant ? NAN : INFINITY;
  else v = ldexp((double)(1024 + mant), exp - 25);
  return sign ? -v : v;
}

/* ------------------------------------------------------------------------ */
/* The asymmetric quantizer ([KIVI page] title, [HF page]: "asymmetric")    */
/* ------------------------------------------------------------------------ */

/* Quantizes n values x[0], x[stride], ... with b bits.  Outputs the fp32 scale
 * and zero point and one code per value. */
void oracle_quantize_group(const float* x, int n, int stride, int bits,
                           float* scale_out, float* mn_out, uint8_t* codes) {
  float mn = x[0], mx = x[0];
  for (int i = 1; i < n; ++i) {
    float v = x[(size_t)i * stride];
    if (v < mn) mn = v;
    if (v > mx) mx = v;
  }
  const int qmax = (1 << bits) - 1;
  float scale = (mx - mn) / (float)qmax;
  for (int i = 0; i < n; ++i) {
    int c = 0;
    if (scale > 0.0f) {
      float t = (x[(size_t)i * stride] - mn) / scale;
      c = (int)round_half_even_nonneg((double)t); /* t >= 0, exact in double */
      if (c > qmax) c = qmax;
    }
    codes[i] = (uint8_t)c;
  }
  *scale_out = scale;
  *mn_out = mn;
}

/* ------------------------------------------------------------------------ */
/* Packed group record (layout definition of the library's header)          */
/* ------------------------------------------------------------------------ */

enum { ORACLE_G = 32, ORACLE_R = 128 };

long oracle_record_bytes(int D, int bits) {
  return (long)ORACLE_G * D * bits / 4 + 8L * D;
}

/* Number of quantized groups for S tokens: NG(S) = max(0, floor((S-R)/G))
 * ([Llama-3 rec] "KV bytes basis": the grouped term covers S - R tokens). */
int oracle_num_groups(int S) {
  if (S < ORACLE_R) return 0;
  return (S - ORACLE_R) / ORACLE_G;
}

/* Key codes of one token row: D*b/32 little-endian 32-bit words.  The decode
 * kernel walks the channels in k-steps of 16 and hands channel
 * d = 16 s + 4 t + j (k-step s, quad lane t = 0..3, j = 0..3) to quad lane t,
 * which owns the W = D*b/128 words t*W .. t*W + W - 1 of the row; each of those
 * words covers 8/b consecutive k-steps, the k-step s being number
 * s mod (8/b) inside its word.
 *   2 bits: byte (s mod 4) of the word holds the four codes of k-step s: j = 0
 *           in bits 0-1, j = 1 in bits 4-5, j = 2 in bits 2-3, j = 3 in bits
 *           6-7 (each code in the low half of a nibble).
 *   4 bits: byte j of the word holds code j of the word's first k-step in its
 *           low nibble and of its second k-step in its high nibble. */
static void k_code_position(int d, int D, int bits, int* word_in_row, int* bit) {
  const int s = d / 16, t = (d % 16) / 4, j = d % 4;
  const int per_word = 8 / bits; /* k-steps per word */
  *word_in_row = t * (D * bits / 128) + s / per_word;
  if (bits == 2) {
    static const int nibble_offset[4] = {0, 4, 2, 6};
    *bit = 8 * (s % per_word) + nibble_offset[j];
  } else {
    *bit = 8 * j + 4 * (s % per_word);
  }
}

static void put_key_code(uint32_t* row_words, int d, int D, int bits, int code) {
  int w, b;
  k_code_position(d, D, bits, &w, &b);
  row_words[w] |= (uint32_t)code << b;
}

/* Value codes are stored in the order the decode kernel's threads read them.
 * Token i (0..31), channel d of a group record belong to lane
 * L = 4 (d mod 8) + (i mod 8) / 2 and to that lane's word
 *   lw = d / 16            (2 bits),
 *   lw = 2 (d / 16) + i/16 (4 bits);
 * lane words are interleaved four at a time over the 32 lanes:
 *   word = ((lw / 4) * 32 + L) * 4 + lw mod 4.
 * Inside the word, with r = (d mod 16) / 8, kk = i / 16, hf = (i mod 16) / 8,
 * e = i mod 2:
 *   2 bits: bit 8 (r + 2 hf) + 2 kk + 4 e (nibble pairs: even token low, odd
 *           token high),
 *   4 bits: bit 8 (2 hf + e) + 4 r (one code per nibble). */
static void v_code_position(int i, int d, int D, int bits, long* word, int* bit) {
  (void)D;
  const int mt = d / 16, g = d % 8, r = (d % 16) / 8;
  const int kk = i / 16, hf = (i % 16) / 8, tig = (i % 8) / 2, e = i % 2;
  const int lane = 4 * g + tig;
  const int lw = bits == 2 ? mt : 2 * mt + kk;
  *word = ((long)(lw / 4) * 32 + lane) * 4 + lw % 4;
  *bit = bits == 2 ? 8 * (r + 2 * hf) + 2 * kk + 4 * e : 8 * (2 * hf + e) + 4 * r;
}

/* fp16 index of the value scale (and min) of token i, channel block j: each
 * block holds 16 token pairs, pair q = 4 tig + 2 kk + hf at indices 2q, 2q+1
 * (with tig, kk, hf, e of token i as above). */
static long v_meta_index(int i, int j) {
  const int kk = i / 16, hf = (i % 16) / 8, tig = (i % 8) / 2, e = i % 2;
  return (long)j * 32 + 2 * (4 * tig + 2 * kk + hf) + e;
}

static void put_u16(uint8_t* p, uint16_t v) {
  p[0] = (uint8_t)(v & 0xff);
  p[1] = (uint8_t)(v >> 8);
}

/* Builds one group record from a key tile and a value tile of G tokens,
 * each token a row of D bf16 values (row stride `ld` elements).
 *   keys: one quantization group per channel over the G tokens ([KIVI page]
 *         "KEYS ... PER-CHANNEL");
 *   values: one group per token over each block of 32 channels ([KIVI page]
 *         "VALUES ... PER-TOKEN"; group size 32 per [Llama-3 rec] "Methodology"). */
void oracle_make_record(const uint16_t* k, const uint16_t* v, long ld, int D,
                        int bits, uint8_t* record) {
  const int G = ORACLE_G;
  const long kc_words = (long)G * D * bits / 32;
  memset(record, 0, (size_t)oracle_record_bytes(D, bits));
  uint32_t* kcodes = (uint32_t*)malloc(sizeof(uint32_t) * kc_words);
  uint32_t* vcodes = (uint32_t*)malloc(sizeof(uint32_t) * kc_words);
  memset(kcodes, 0, sizeof(uint32_t) * kc_words);
  memset(vcodes, 0, sizeof(uint32_t) * kc_words);
  /* K meta: D fp16 scales, then D fp16 mins.  V meta: (D/32) x 32 fp16 scales
   * (block j, then token i), then the same for the mins. */
  uint8_t* kscale = record + 8L * kc_words;
  uint8_t* kmin = kscale + 2L * D;
  uint8_t* vscale = kmin + 2L * D;
  uint8_t* vmin = vscale + 2L * D;

  float col[ORACLE_G];
  uint8_t codes[ORACLE_G];
  /* Keys, per channel d over tokens 0..G-1. */
  for (int d = 0; d < D; ++d) {
    for (int i = 0; i < G; ++i) col[i] = bf16_bits_to_float(k[(long)i * ld + d]);
    float scale, mn;
    oracle_quantize_group(col, G, 1, bits, &scale, &mn, codes);
    /* token-major rows of D*b/32 words: channel d of token i */
    for (int i = 0; i < G; ++i) put_key_code(kcodes + (long)i * D * bits / 32, d, D, bits, codes[i]);
    put_u16(kscale + 2L * d, oracle_f32_to_f16_bits(scale));
    put_u16(kmin + 2L * d, oracle_f32_to_f16_bits(mn));
  }
  /* Values, per token i over channel block j. */
  float row[32];
  for (int i = 0; i < G; ++i) {
    for (int j = 0; j < D / 32; ++j) {
      for (int c = 0; c < 32; ++c) row[c] = bf16_bits_to_float(v[(long)i * ld + 32 * j + c]);
      float scale, mn;
      oracle_quantize_group(row, 32, 1, bits, &scale, &mn, codes);
      for (int c = 0; c < 32; ++c) {
        long word;
        int bit;
        v_code_position(i, 32 * j + c, D, bits, &word, &bit);
        vcodes[word] |= (uint32_t)codes[c] << bit;
      }
      const long e = v_meta_index(i, j);
      put_u16(vscale + 2 * e, oracle_f32_to_f16_bits(scale));
      put_u16(vmin + 2 * e, oracle_f32_to_f16_bits(mn));
    }
  }
  for (long w = 0; w < kc_words; ++w) {
    for (int byte = 0; byte < 4; ++byte) {
      record[4 * w + byte] = (uint8_t)(kcodes[w] >> (8 * byte));
      record[4 * kc_words + 4 * w + byte] = (uint8_t)(vcodes[w] >> (8 * byte));
    }
  }
  free(kcodes);
  free(vcodes);
}

/* Reads the key code of channel d from a packed little-endian token row. */
static int get_key_code(const uint8_t* row, int d, int D, int bits) {
  int w, b;
  k_code_position(d, D, bits, &w, &b);
  const uint8_t* p = row + 4L * w;
  uint32_t word = (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) |
                  ((uint32_t)p[3] << 24);
  return (int)((word >> b) & ((1u << bits) - 1u));
}

static uint16_t get_u16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }

/* Dequantizes a record into key and value tiles [G][D] of doubles:
 * x_hat = scale_h * code + min_h with the stored fp16 parameters. */
void oracle_dequant_record(const uint8_t* record, int D, int bits, double* k_hat,
                           double* v_hat) {
  const int G = ORACLE_G;
  const long row_words_k = (long)D * bits / 32;
  const long kc_bytes = 4L * G * row_words_k;
  const uint8_t* kscale = record + 2 * kc_bytes;
  const uint8_t* kmin = kscale + 2L * D;
  const uint8_t* vscale = kmin + 2L * D;
  const uint8_t* vmin = vscale + 2L * D;
  for (int i = 0; i < G; ++i) {
    for (int d = 0; d < D; ++d) {
      int ck = get_key_code(record + 4L * row_words_k * i, d, D, bits);
      double sk = oracle_f16_bits_to_double(get_u16(kscale + 2L * d));
      double mk = oracle_f16_bits_to_double(get_u16(kmin + 2L * d));
      k_hat[(long)i * D + d] = sk * ck + mk;
      long vw;
      int vb;
      v_code_position(i, d, D, bits, &vw, &vb);
      const uint8_t* wp = record + kc_bytes + 4 * vw;
      const uint32_t vword = (uint32_t)wp[0] | ((uint32_t)wp[1] << 8) |
                             ((uint32_t)wp[2] << 16) | ((uint32_t)wp[3] << 24);
      int cv = (int)((vword >> vb) & ((1u << bits) - 1u));
      long e = v_meta_index(i, d / 32);
      double sv = oracle_f16_bits_to_double(get_u16(vscale + 2 * e));
      double mv = oracle_f16_bits_to_double(get_u16(vmin + 2 * e));
      v_hat[(long)i * D + d] = sv * cv + mv;
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Cache state of one layer                                                 */
/*   records [B][Hkv][NGcap][record bytes]; rings [B][Hkv][R+G][D] bf16      */
/* ------------------------------------------------------------------------ */

/* Prefill with S tokens: k, v are [B][Hkv][S][D] bf16. */
void oracle_prefill(const uint16_t* k, const uint16_t* v, int B, int Hkv, int S, int D,
                    int bits, int NGcap, uint8_t* records, uint16_t* ring_k,
                    uint16_t* ring_v) {
  const int G = ORACLE_G, slots = ORACLE_R + ORACLE_G;
  const int NG = oracle_num_groups(S);
  const long rb = oracle_record_bytes(D, bits);
  for (int b = 0; b < B; ++b) {
    for (int h = 0; h < Hkv; ++h) {
      const long seq = (long)b * Hkv + h;
      const uint16_t* kseq = k + seq * S * D;
      const uint16_t* vseq = v + seq * S * D;
      for (int g = 0; g < NG; ++g)
        oracle_make_record(kseq + (long)g * G * D, vseq + (long)g * G * D, D, D, bits,
                           records + (seq * NGcap + g) * rb);
      for (int t = NG * G; t < S; ++t) {
        memcpy(ring_k + (seq * slots + t % slots) * D, kseq + (long)t * D, 2L * D);
        memcpy(ring_v + (seq * slots + t % slots) * D, vseq + (long)t * D, 2L * D);
      }
    }
  }
}

/* Appends token S (k_new, v_new are [B][Hkv][D] bf16) to a layer holding S
 * tokens; flushes the oldest G residual tokens into group NG(S) when the
 * residual reaches R + G tokens.  Returns the new token count S + 1. */
int oracle_append(const uint16_t* k_new, const uint16_t* v_new, int B, int Hkv, int S,
                  int D, int bits, int NGcap, uint8_t* records, uint16_t* ring_k,
                  uint16_t* ring_v) {
  const int G = ORACLE_G, slots = ORACLE_R + ORACLE_G;
  const int NG = oracle_num_groups(S);
  const long rb = oracle_record_bytes(D, bits);
  const int flush = (S + 1 - NG * G == slots);
  for (int b = 0; b < B; ++b) {
    for (int h = 0; h < Hkv; ++h) {
      const long seq = (long)b * Hkv + h;
      memcpy(ring_k + (seq * slots + S % slots) * D, k_new + seq * D, 2L * D);
      memcpy(ring_v + (seq * slots + S % slots) * D, v_new + seq * D, 2L * D);
      if (flush) {
        const long first = (long)(NG * G) % slots; /* a whole group never wraps */
        oracle_make_record(ring_k + (seq * slots + first) * D,
                           ring_v + (seq * slots + first) * D, D, D, bits,
                           records + (seq * NGcap + NG) * rb);
      }
    }
  }
  return S + 1;
}

/* Softmax attention of one query row over S dense (K, V) rows [S][D] in
 * double: s_t = sm_scale * <q, k_t>, out = sum_t softmax(s)_t v_t. */
static void attend_dense(const double* K, const double* V, const uint16_t* q, int S, int D,
                         double sm_scale, double* out) {
  double* s = (double*)malloc(sizeof(double) * (size_t)(S > 0 ? S : 1));
  double m = -INFINITY;
  for (int t = 0; t < S; ++t) {
    double acc = 0.0;
    for (int d = 0; d < D; ++d) acc += (double)bf16_bits_to_float(q[d]) * K[(long)t * D + d];
    s[t] = sm_scale * acc;
    if (s[t] > m) m = s[t];
  }
  double denom = 0.0;
  for (int t = 0; t < S; ++t) {
    s[t] = exp(s[t] - m);
    denom += s[t];
  }
  for (int d = 0; d < D; ++d) {
    double acc = 0.0;
    for (int t = 0; t < S; ++t) acc += s[t] * V[(long)t * D + d];
    out[d] = acc / denom;
  }
  free(s);
}

/* Decode attention of one query head over one kv head holding S tokens:
 * scores s_t = sm_scale * <q, k_hat_t>, out = sum_t softmax(s)_t v_hat_t, in
 * double.  k_hat/v_hat are the dequantized groups for t < NG*G and the bf16
 * residual otherwise. */
void oracle_attend_one(const uint8_t* seq_records, const uint16_t* seq_ring_k,
                       const uint16_t* seq_ring_v, const uint16_t* q, int S, int D,
                       int bits, double sm_scale, double* out) {
  const int G = ORACLE_G, slots = ORACLE_R + ORACLE_G;
  const int NG = oracle_num_groups(S);
  const long rb = oracle_record_bytes(D, bits);
  double* K = (double*)malloc(sizeof(double) * (size_t)(S > 0 ? S : 1) * D);
  double* V = (double*)malloc(sizeof(double) * (size_t)(S > 0 ? S : 1) * D);
  for (int g = 0; g < NG; ++g)
    oracle_dequant_record(seq_records + g * rb, D, bits, K + (long)g * G * D,
                          V + (long)g * G * D);
  for (int t = NG * G; t < S; ++t) {
    for (int d = 0; d < D; ++d) {
      K[(long)t * D + d] = bf16_bits_to_float(seq_ring_k[(long)(t % slots) * D + d]);
      V[(long)t * D + d] = bf16_bits_to_float(seq_ring_v[(long)(t % slots) * D + d]);
    }
  }
  attend_dense(K, V, q, S, D, sm_scale, out);
  free(K);
  free(V);
}

/* Decode attention of a whole layer: q [B][Hq][D] bf16 -> out [B][Hq][D]
 * double.  Query head h reads kv head h / (Hq / Hkv). */
void oracle_attention(const uint8_t* records, const uint16_t* ring_k,
                      const uint16_t* ring_v, const uint16_t* q, int B, int Hkv, int Hq,
                      int S, int D, int bits, int NGcap, double sm_scale, double* out) {
  const int slots = ORACLE_R + ORACLE_G;
  const long rb = oracle_record_bytes(D, bits);
  const int per_kv = Hq / Hkv;
  for (int b = 0; b < B; ++b) {
    for (int h = 0; h < Hq; ++h) {
      const long seq = (long)b * Hkv + h / per_kv;
      oracle_attend_one(records + seq * NGcap * rb, ring_k + seq * slots * D,
                        ring_v + seq * slots * D, q + ((long)b * Hq + h) * D, S, D, bits,
                        sm_scale, out + ((long)b * Hq + h) * D);
    }
  }
}

/* ------------------------------------------------------------------------ */
/* The full-precision baseline: attention over an unquantized bf16 cache    */
/* ------------------------------------------------------------------------ */

/* Decode attention over a bf16 cache, the 16-bit baseline the [HF page] and
 * the [KIVI page] compare the quantized cache with.  k, v: bf16 bits
 * [B][Hkv][Smax][D], tokens 0..S-1 of each (sequence, kv head) used; q: bf16
 * bits [B][Hq][D]; out: [B][Hq][D] double.  Query head h reads kv head
 * h / (Hq / Hkv). */
void oracle_attention_bf16(const uint16_t* k, const uint16_t* v, const uint16_t* q, int B,
                           int Hkv, int Hq, int S, int Smax, int D, double sm_scale,
                           double* out) {
  const int per_kv = Hq / Hkv;
  double* K = (double*)malloc(sizeof(double) * (size_t)(S > 0 ? S : 1) * D);
  double* V = (double*)malloc(sizeof(double) * (size_t)(S > 0 ? S : 1) * D);
  for (int b = 0; b < B; ++b) {
    for (int kvh = 0; kvh < Hkv; ++kvh) {
      const long base = ((long)b * Hkv + kvh) * Smax * D;
      for (long i = 0; i < (long)S * D; ++i) {
        K[i] = bf16_bits_to_float(k[base + i]);
        V[i] = bf16_bits_to_float(v[base + i]);
      }
      for (int j = 0; j < per_kv; ++j) {
        const long row = (long)b * Hq + (long)kvh * per_kv + j;
        attend_dense(K, V, q + row * D, S, D, sm_scale, out + row * D);
      }
    }
  }
  free(K);
  free(V);
}

/* ------------------------------------------------------------------------ */
/* Key-granularity ablation: fake quantization of a key tile                */
/* ------------------------------------------------------------------------ */

/* Quantizes and dequantizes keys k (bf16 bits [T][D], T a multiple of G) with
 * b bits, returning k_hat [T][D] in double:
 *   per_token == 0: KIVI's key quantization ([KIVI page], [HF page]): each
 *     channel of each G-token group is one group (the group record's keys);
 *   per_token != 0: the granularity the pages argue against for keys: each
 *     token's channels in blocks of G form one group (the values' rule).
 * Parameters and codes follow the same quantizer and fp16 metadata as the
 * record; k_hat = f16(scale) * code + f16(min). */
void oracle_fake_quant_keys(const uint16_t* k, int T, int D, int bits, int per_token,
                            double* k_hat) {
  const int G = ORACLE_G;
  /* group n (n_groups of G elements each): element i sits at k[first + i * step] */
  const long n_groups = per_token ? (long)T * (D / G) : (long)(T / G) * D;
  for (long n = 0; n < n_groups; ++n) {
    long first, step;
    if (per_token) {  /* token n / (D/G), channels G * (n % (D/G)) .. + G-1 */
      first = (n / (D / G)) * D + (long)G * (n % (D / G));
      step = 1;
    } else {          /* channel n % D of tokens G * (n / D) .. + G-1 */
      first = (n / D) * G * D + n % D;
      step = D;
    }
    float x[ORACLE_G];
    uint8_t codes[ORACLE_G];
    for (int i = 0; i < G; ++i) x[i] = bf16_bits_to_float(k[first + i * step]);
    float scale, mn;
    oracle_quantize_group(x, G, 1, bits, &scale, &mn, codes);
    const double sh = oracle_f16_bits_to_double(oracle_f32_to_f16_bits(scale));
    const double mh = oracle_f16_bits_to_double(oracle_f32_to_f16_bits(mn));
    for (int i = 0; i < G; ++i) k_hat[first + i * step] = sh * codes[i] + mh;
  }
}

/* ------------------------------------------------------------------------ */
/* Prefill attention over the prompt (causal), the step before the cache     */
/* ------------------------------------------------------------------------ */

/* Causal attention of a prompt over its own bf16 keys and values, the step whose
 * epilogue quantizes the prompt into the cache ([Llama-3 rec] "KV bytes basis":
 * the history is quantized, the newest tokens stay in full precision).  For
 * query head h of sequence b (kv head h / (Hq / Hkv)) and position i:
 *   out[b][h][i] = sum_{j <= i} softmax_j(sm_scale * <q_i, k_j>) v_j,  in double.
 * q: bf16 bits [B][Hq][S][D]; k, v: [B][Hkv][S][D]; out: [B][Hq][S][D]. */
void oracle_prefill_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B,
                              int Hkv, int Hq, int S, int D, double sm_scale, double* out) {
  const int per_kv = Hq / Hkv;
  double* K = (double*)malloc(sizeof(double) * (size_t)(S > 0 ? S : 1) * D);
  double* V = (double*)malloc(sizeof(double) * (size_t)(S > 0 ? S : 1) * D);
  for (int b = 0; b < B; ++b) {
    for (int kvh = 0; kvh < Hkv; ++kvh) {
      const long base = ((long)b * Hkv + kvh) * S * D;
      for (long i = 0; i < (long)S * D; ++i) {
        K[i] = bf16_bits_to_float(k[base + i]);
        V[i] = bf16_bits_to_float(v[base + i]);
      }
      for (int j = 0; j < per_kv; ++j) {
        const long head = (long)b * Hq + (long)kvh * per_kv + j;
        for (int i = 0; i < S; ++i)  /* position i sees tokens 0..i */
          attend_dense(K, V, q + (head * S + i) * D, i + 1, D, sm_scale,
                       out + (head * S + i) * D);
      }
    }
  }
  free(K);
  free(V);
}
