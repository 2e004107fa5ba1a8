/*
 * kivi.h - C ABI of the KIVI packed KV cache and its fused decode attention
 * (libkivi.so, built for sm_100a).
 *
 * Method sources (cited by page title and section):
 *   [KIVI page]   "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache"
 *                 (inference-research papers/kivi summary page): keys are
 *                 quantized per channel, values per token, asymmetric 2-bit.
 *   [HF page]     "KV cache quantization squeezes 5GB down to fit longer LLM
 *                 generations": the cache grows with every generated token;
 *                 quantization rounds values; keys per channel, values per token.
 *   [Llama-3 rec] record "kv-efficiency/kivi-2bit-llama3-8b-gqa-8k", fields
 *                 "Model" (32 layers, 8 kv heads, 32 query heads, head_dim 128),
 *                 "KV bytes basis" (grouped history plus a full-precision
 *                 residual of the most recent R tokens; the grouped term covers
 *                 S-R tokens), "Methodology" (group size 32, residual length 128
 *                 for both KIVI-2 and KIVI-4) and "notes" (4-bit byte count).
 *
 * Quantizer (one group of 32 values x, b bits): zero point mn = min(x),
 * scale = (max(x) - mn) / (2^b - 1) in IEEE fp32, code = round-half-even(
 * (x - mn) / scale) clamped to [0, 2^b - 1] (all codes 0 when scale == 0).
 * The stored metadata is {fp16(scale), fp16(mn)}, both round-to-nearest-even;
 * dequantized value = scale_h * code + mn_h.  Keys: one group per channel over
 * 32 consecutive tokens.  Values: one group per token over 32 consecutive
 * channels.
 *
 * Cache state of one layer holding S tokens (uniform over the batch):
 *   NG(S) = max(0, floor((S - R) / G)) quantized groups cover tokens
 *   [0, NG*G); tokens [NG*G, S) stay bf16 in a ring of R + G slots, token t at
 *   slot t mod (R + G).  Appending token S flushes the oldest G ring tokens into
 *   group NG exactly when S + 1 - NG*G == R + G, so NG after the append is
 *   NG(S + 1).  G = 32 and R = 128 here.
 *
 * Packed layout (all little-endian, 32-bit code words):
 *   records  [L][B][Hkv][NGcap] group records, NGcap = NG(max_tokens),
 *            record bytes = G*D*b/4 + 8*D (3072 at D=128 b=2, 5120 at b=4,
 *            1536 at D=64 b=2).  One record, in order:
 *     K codes  G rows (token i of the group) x D*b/32 words; channel d is code
 *              n = d mod (32/b) of word d/(32/b), at bit (n mod 2)*16 + (n/2)*b
 *              (even codes in the low 16 bits, odd codes in the high 16 bits).
 *     V codes  G*D*b/32 words in the order the decode kernel's threads consume
 *              them.  Token i, channel d: with mt = d/16, g = d mod 8,
 *              r = (d mod 16)/8, kk = i/16, hf = (i mod 16)/8, tig = (i mod 8)/2,
 *              e = i mod 2, idx = 4kk + 2hf + r and p = 16/b:
 *                word = ((4g + tig)*(D/16) + mt)*(b/2) + idx/p,
 *                bit  = 16e + (idx mod p)*b.
 *     K scale  D fp16 (channel d), then K min: D fp16.
 *     V scale  (D/32) blocks of G fp16; token i of block j at index
 *              32j + 2(4tig + 2kk + hf) + e (tig, kk, hf, e of i as above);
 *              then V min in the same layout.
 *              Each array puts the operands one thread reads next to each
 *              other, so the kernel turns a pair of codes into an fp16x2
 *              register with one mask-and-or.
 *   resid_k, resid_v  bf16 [L][B][Hkv][R + G][D].
 *
 * Conventions for every call below:
 *   - Ownership: the caller allocates and frees every device buffer; the
 *     library never allocates device memory.  The handle owns host state only
 *     (config, pointers, token count S per layer).
 *   - Device pointers are plain CUDA device addresses, contiguous row-major,
 *     16-byte aligned.  `stream` is a cudaStream_t passed as void* (NULL =
 *     legacy default stream).
 *   - Calls are asynchronous on `stream`: they validate on the host, launch and
 *     return.  KIVI_ERR_CUDA reports a launch error; device faults surface at
 *     the caller's next synchronisation.  No exception crosses the ABI and the
 *     library never exits the process.
 *   - Inputs must be finite with |x| <= 65504 (fp16 metadata range); this is a
 *     documented precondition, not checked on the device.
 *   - One handle must not be used from two host threads at once; calls that
 *     share a handle's workspace must be ordered on one stream.
 */
#ifndef KIVI_H
#define KIVI_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KIVI_OK = 0,
  KIVI_ERR_INVALID_ARG = 1,      /* null pointer, negative size, bad layer index */
  KIVI_ERR_UNSUPPORTED = 2,      /* config outside the supported set (below) */
  KIVI_ERR_BUFFER_TOO_SMALL = 3, /* a kivi_buffers size is below kivi_required_bytes */
  KIVI_ERR_CAPACITY = 4,         /* the call would exceed max_tokens */
  KIVI_ERR_STATE = 5,            /* prefill on a non-empty layer, append/attend on an empty one */
  KIVI_ERR_CUDA = 6,             /* a CUDA runtime call or launch failed */
  KIVI_ERR_DEVICE = 7,           /* a kernel reported a failure in the device status word */
  KIVI_ERR_SCRATCH_LIMIT = 8     /* the call needs more than the library's static scratch array */
} kivi_status;

/* Size of the file-scope device array used by
 * kivi_decode_attention_static_scratch (every GPU that loads the library holds
 * it until the process exits). */
#define KIVI_STATIC_SCRATCH_BYTES (8u << 20)

/* Cache geometry.  Supported: bits in {2, 4}, group_size == 32,
 * residual == 128, head_dim in {64, 128}, num_q_heads / num_kv_heads in
 * {1, 2, 4, 8} (exact multiple), all counts >= 1, max_tokens >= 1.  Query
 * head h reads kv head h / (num_q_heads / num_kv_heads) (consecutive grouping,
 * the usual repeat-KV convention; [Llama-3 rec] "Model" gives 32 query heads
 * over 8 kv heads). */
typedef struct {
  int32_t batch;
  int32_t num_layers;
  int32_t num_kv_heads;
  int32_t num_q_heads;
  int32_t head_dim;
  int32_t bits;
  int32_t group_size;
  int32_t residual;
  int32_t max_tokens;
} kivi_config;

typedef struct {
  size_t records_bytes;   /* group records of all layers */
  size_t resid_k_bytes;   /* bf16 key ring of all layers */
  size_t resid_v_bytes;   /* bf16 value ring of all layers */
  size_t workspace_bytes; /* split-K partials and the device status word */
} kivi_sizes;

typedef struct {
  void* records;
  void* resid_k;
  void* resid_v;
  void* workspace;
  kivi_sizes sizes;       /* the sizes the caller actually allocated */
} kivi_buffers;

typedef struct kivi_cache kivi_cache; /* opaque host handle */

/* Device bytes each buffer needs for `cfg`.  Host only.
 * Errors: INVALID_ARG (null), UNSUPPORTED (config outside the supported set). */
kivi_status kivi_required_bytes(const kivi_config* cfg, kivi_sizes* out);

/* Geometry of the records buffer for `cfg`, host only: the bytes of one group
 * record (G*D*b/4 + 8*D: codes plus fp16 metadata) and the records each
 * (layer, sequence, kv head) has room for, NGcap = NG(max_tokens) (zero when
 * max_tokens < R).  Records are ordered [layer][sequence][kv head][NGcap].
 * Either output may be NULL.  Errors: INVALID_ARG (null cfg), UNSUPPORTED. */
kivi_status kivi_record_layout(const kivi_config* cfg, size_t* record_bytes,
                               int32_t* records_per_seq);

/* Creates a handle over caller-owned buffers; every layer starts empty (S = 0).
 * Zeroes the device status word in `workspace` with a synchronous cudaMemset.
 * Errors: INVALID_ARG, UNSUPPORTED, BUFFER_TOO_SMALL, CUDA. */
kivi_status kivi_cache_create(const kivi_config* cfg, const kivi_buffers* bufs,
                              kivi_cache** out);

/* Frees the host handle (not the caller's device buffers).  NULL is a no-op. */
void kivi_cache_destroy(kivi_cache* cache);

/* Token count S and quantized-group count NG(S) of `layer`.  Host only. */
kivi_status kivi_cache_length(const kivi_cache* cache, int32_t layer,
                              int32_t* S, int32_t* NG);

/* Marks `layer` empty again (S = 0).  Host only; device contents are left as
 * they are and are overwritten by the next prefill. */
kivi_status kivi_cache_reset(kivi_cache* cache, int32_t layer);

/* Prefill of one layer with S prompt tokens ([HF page]: the history that is
 * quantized; [Llama-3 rec] "KV bytes basis": grouped history plus residual).
 * k, v: device bf16 [B][Hkv][S][D].  Quantizes NG(S) groups of keys (per
 * channel) and values (per token) into records 0..NG-1 and copies tokens
 * [NG*G, S) into the rings.  S may be 0..max_tokens.
 * Errors: INVALID_ARG, STATE (layer not empty), CAPACITY (S > max_tokens), CUDA. */
kivi_status kivi_quantize_prefill(kivi_cache* cache, int32_t layer,
                                  const void* k, const void* v, int32_t S,
                                  void* stream);

/* Prefill with a prompt length per sequence (a ragged batch, as in the serving
 * setting of the [Llama-3 rec] "Methodology", which batches prompts of
 * different lengths).  k, v: bf16 [batch][num_kv_heads][S_max][head_dim] on the device;
 * sequence b uses its first lengths[b] tokens (0 <= lengths[b] <= S_max <=
 * max_tokens), quantized in groups aligned to its own token 0, the rest of its
 * residual in its ring.  lengths: host array [batch], read before the call
 * returns (the call synchronises `stream` once to place them in the workspace).
 * Every later kivi_append_token adds one token to every sequence (each flushes
 * on its own schedule), and kivi_decode_attention attends each sequence's own
 * tokens; kivi_cache_length reports the longest sequence.  The layer must be
 * empty.  Errors: INVALID_ARG, STATE, CAPACITY (S_max > max_tokens), CUDA. */
kivi_status kivi_quantize_prefill_ragged(kivi_cache* cache, int32_t layer, const void* k,
                                         const void* v, int32_t S_max,
                                         const int32_t* lengths, void* stream);

/* Causal prefill attention with the prompt quantized into `layer` in its
 * epilogue: the step before decoding ([Llama-3 rec] "KV bytes basis": the
 * prompt's history is kept as quantized groups, its newest tokens in bf16).
 * For query head h of sequence b (kv head h / (num_q_heads / num_kv_heads))
 * and prompt position i,
 *   out[b][h][i] = sum_{j<=i} softmax_j(sm_scale * <q[b][h][i], k[b][kvh][j]>) v[b][kvh][j],
 * computed on the tensor cores with bf16 operands, fp32 scores and accumulation,
 * and the softmax weights rounded to bf16 for the second product.  The layer
 * then holds exactly what kivi_quantize_prefill(k, v, S) writes (records of the
 * NG(S) groups, tokens [NG*G, S) in the rings).
 *   q: bf16 [batch][num_q_heads][S][head_dim]; k, v: bf16 [batch][num_kv_heads]
 *      [S][head_dim]; out: fp32 [batch][num_q_heads][S][head_dim], written.  All
 *      device, 16-byte aligned, owned by the caller.
 *   sm_scale <= 0 means 1/sqrt(head_dim).  S >= 1.
 * A wait that runs out sets the cache's device status word
 * (kivi_check_device_status).  Asynchronous on `stream`.
 * Errors: INVALID_ARG (NULL or unaligned pointers, S < 1, batch * num_q_heads *
 * (S + 128) >= 2^31, sm_scale not finite), STATE (layer not empty), CAPACITY
 * (S > max_tokens), CUDA. */
kivi_status kivi_prefill_attention(kivi_cache* cache, int32_t layer, const void* q,
                                   const void* k, const void* v, int32_t S, float* out,
                                   float sm_scale, void* stream);

/* The same causal attention without a cache (for comparisons and for models
 * that quantize elsewhere).  Arguments as in kivi_prefill_attention, with the
 * shape given explicitly; head_dim 64 or 128, num_q_heads a multiple of
 * num_kv_heads.  status: NULL, or a zeroed device uint32 (4-byte aligned) that
 * a wait that ran out sets to a non-zero code.
 * Errors: INVALID_ARG, UNSUPPORTED (head_dim, head ratio), CUDA. */
kivi_status kivi_causal_attention(const void* q, const void* k, const void* v, int32_t batch,
                                  int32_t num_kv_heads, int32_t num_q_heads, int32_t head_dim,
                                  int32_t S, float* out, float sm_scale, uint32_t* status,
                                  void* stream);

/* Token count of every sequence of `layer` (host array S_out[batch]): the
 * ragged lengths, or the layer's common length.  Errors: INVALID_ARG. */
kivi_status kivi_cache_lengths(const kivi_cache* cache, int32_t layer, int32_t* S_out);

/* Appends one generated token per sequence to `layer` ([HF page]: the cache
 * grows with every generated token).  k_new, v_new: device bf16 [B][Hkv][D],
 * written to ring slot S mod (R+G).  When S + 1 - NG*G == R + G the same launch
 * quantizes ring tokens [NG*G, NG*G + G) into record NG (the residual flush).
 * The layer need not have been prefilled (S may be 0).
 * Errors: INVALID_ARG, CAPACITY (S + 1 > max_tokens), CUDA. */
kivi_status kivi_append_token(kivi_cache* cache, int32_t layer,
                              const void* k_new, const void* v_new, void* stream);

/* Single-token decode attention of `layer` over all S cached tokens:
 * quantized groups dequantized in registers and the bf16 residual, merged under
 * one softmax ([KIVI page]: the per-channel/per-token split follows how the
 * attention kernel reads memory).  q: device bf16 [B][Hq][D]; out: device fp32
 * [B][Hq][D], out[b][h] = sum_t softmax_t(sm_scale * <q[b][h], k_t>) v_t over the
 * dequantized keys/values of kv head h / (Hq/Hkv).  sm_scale <= 0 selects
 * 1/sqrt(D).  Uses the handle's workspace (split-K partials).
 * Errors: INVALID_ARG, STATE (S == 0), CUDA. */
kivi_status kivi_decode_attention(const kivi_cache* cache, int32_t layer,
                                  const void* q, float* out, float sm_scale,
                                  void* stream);

/* Decode attention that allocates nothing and needs neither a handle nor a
 * workspace buffer.  The pages have no counterpart: this entry point is for
 * callers that cannot allocate device memory - for example an inference engine
 * that loads this library as a plugin and owns all device memory through its
 * own pool allocator (a cudaMalloc behind its back would fail or break its
 * accounting), or a process whose device memory is already reserved by such an
 * allocator.  The caller passes only inputs and outputs: the cache buffers of
 * `cfg` in the layout above (records may be NULL when NG(max_tokens) == 0),
 * the layer, its token count S (for example from kivi_cache_length), q and
 * out exactly as for kivi_decode_attention, whose result this call reproduces.
 * Scratch: the split-K partials go to one file-scope device array of
 * KIVI_STATIC_SCRATCH_BYTES.  The first call on a device looks up the array's
 * address with cudaGetSymbolAddress and clears its header on `stream`; make
 * that first call before any stream capture.  All calls on a device share the
 * array and leave their contents in it: calls whose kernels may overlap on the
 * GPU (other streams, other host threads) race on it and must be serialised by
 * the caller.  The call picks at most as many splits as fit the array.
 * Errors: INVALID_ARG, UNSUPPORTED, STATE (S == 0), CAPACITY (S > max_tokens),
 * SCRATCH_LIMIT (the partials of the fewest splits a call uses - one over the
 * quantized groups and one per residual chunk of 32 tokens, 6 in all -
 * 256 + 6*B*Hq*(D+2)*4 bytes, exceed the array), CUDA. */
kivi_status kivi_decode_attention_static_scratch(const kivi_config* cfg, const void* records,
                                                 const void* resid_k, const void* resid_v,
                                                 int32_t layer, int32_t S, const void* q,
                                                 float* out, float sm_scale, void* stream);

/* The device status word of kivi_decode_attention_static_scratch on the current
 * device (that call keeps it in the static scratch array, not in a workspace):
 * synchronises `stream`, reads the word through the array's device address
 * and clears it.  Returns KIVI_ERR_DEVICE if one of those calls recorded a
 * failure (a bounded wait that ran out) since the last query, KIVI_ERR_CUDA if
 * a CUDA call failed, else KIVI_OK.  `code_out` (may be NULL) receives the raw
 * word.  Allocates nothing; like the attention call, its first use on a device
 * looks up the array's address.  The pages have no counterpart. */
kivi_status kivi_static_scratch_status(void* stream, uint32_t* code_out);

/* Synchronises `stream`, then reads and clears the device status word.
 * Returns KIVI_ERR_DEVICE if a kernel recorded a failure (a bounded wait that
 * ran out), KIVI_ERR_CUDA if the synchronisation failed, else KIVI_OK.
 * `code_out` (may be NULL) receives the raw status word. */
kivi_status kivi_check_device_status(kivi_cache* cache, void* stream,
                                     uint32_t* code_out);

/* KV-cache bytes per token of one sequence of `cfg` holding S >= 1 tokens, all
 * layers, host only ([Llama-3 rec] "KV bytes basis" and "notes").
 *   stored:     what this layout keeps: NG(S) group records (codes plus fp16
 *               metadata) and r = S - NG(S)*G bf16 residual tokens, over S.
 *   codes_only: the record's "exact stored amount": codes of the NG(S)*G grouped
 *               tokens plus the r bf16 residual tokens, no metadata, over S
 *               (18,176 B/token for the Llama-3-8B skeleton at 2 bits, S=8192).
 *   convention: the record's convention: grouped codes counted over all S tokens
 *               plus R residual tokens amortised over S (16,384 + 2,048 =
 *               18,432 B/token for the same skeleton; 34,816 at 4 bits).
 * Any output pointer may be NULL.  Errors: INVALID_ARG (S < 1), UNSUPPORTED. */
kivi_status kivi_cache_bytes(const kivi_config* cfg, int32_t S, double* stored,
                             double* codes_only, double* convention);

/* ------------------------------------------------------------------------ */
/* The 16-bit baseline: decode attention over an unquantized bf16 cache      */
/* ------------------------------------------------------------------------ */

/* Workspace bytes of kivi_bf16_decode_attention for `batch` sequences of
 * `num_kv_heads` kv heads and `num_q_heads` query heads of `head_dim`: a status
 * header (256 B), one ticket per (sequence, kv head) rounded up to 256 B, and
 * the split partials of up to 256 CTAs.  Host only.  The buffer must be
 * zero-filled before its first use; every call leaves it zeroed again except
 * for the status word after a failure (cleared by kivi_bf16_status).
 * Errors: INVALID_ARG, UNSUPPORTED (head_dim not 64/128, num_q_heads /
 * num_kv_heads not 1, 2, 4 or 8). */
kivi_status kivi_bf16_workspace_bytes(int32_t batch, int32_t num_kv_heads,
                                      int32_t num_q_heads, int32_t head_dim,
                                      size_t* bytes);

/* Decode attention over an unquantized bf16 KV cache: the full-precision
 * baseline the [KIVI page] and the [HF page] compare the 2-bit cache with.
 * For query head h of sequence b (kv head h / (num_q_heads / num_kv_heads)),
 *   out[b][h] = sum_{t<S} softmax_t(sm_scale * <q[b][h], k[b][kvh][t]>) v[b][kvh][t].
 *   k_cache, v_cache: bf16 [batch][num_kv_heads][max_tokens][head_dim] (one
 *       layer), device, 16-byte aligned, owned by the caller; tokens S and
 *       beyond are never read into the result (they may hold anything).
 *   q: bf16 [batch][num_q_heads][head_dim]; out: fp32, same shape.
 *   sm_scale <= 0 means 1/sqrt(head_dim).
 *   workspace: kivi_bf16_workspace_bytes bytes (see there).
 * Asynchronous on `stream`; allocates nothing.  Calls that share a workspace
 * must not overlap on the GPU.
 * Errors: INVALID_ARG (NULL or unaligned pointers, S < 1 or S > max_tokens,
 * batch * num_kv_heads * max_tokens >= 2^31, workspace too small, sm_scale not
 * finite), UNSUPPORTED, CUDA. */
kivi_status kivi_bf16_decode_attention(const void* k_cache, const void* v_cache,
                                       int32_t batch, int32_t num_kv_heads,
                                       int32_t num_q_heads, int32_t head_dim,
                                       int32_t max_tokens, int32_t S, const void* q,
                                       float* out, float sm_scale, void* workspace,
                                       size_t workspace_bytes, void* stream);

/* Synchronises `stream`, reads the status word of a kivi_bf16_decode_attention
 * workspace and, if it is not zero, clears the header and the tickets of
 * `batch` x `num_kv_heads` pairs.  KIVI_ERR_DEVICE if a bounded wait ran out,
 * KIVI_ERR_CUDA if a CUDA call failed, else KIVI_OK; `code_out` may be NULL. */
kivi_status kivi_bf16_status(void* workspace, int32_t batch, int32_t num_kv_heads,
                             void* stream, uint32_t* code_out);

/* ------------------------------------------------------------------------ */
/* Key-granularity ablation                                                  */
/* ------------------------------------------------------------------------ */

/* Quantizes and dequantizes keys with `bits` bits at one of two granularities,
 * to measure the claim of the [KIVI page] and the [HF page] that keys, whose
 * magnitudes concentrate in a few outlier channels, must be quantized per
 * channel and not per token:
 *   per_token == 0: KIVI's key rule, one group per channel of every 32
 *       consecutive rows (tokens), as in the group record;
 *   per_token != 0: one group per row over each block of 32 channels (the
 *       values' rule applied to keys).
 * The quantizer is the record's (min/max zero point, fp32 scale, codes round
 * half to even, fp16 metadata); k_hat = fp16(scale) * code + fp16(min) rounded
 * once to fp32.
 *   k: bf16 [rows][head_dim], device, 16-byte aligned; rows a multiple of 32
 *      (rows of several sequences may be stacked: groups never straddle 32).
 *   k_hat: fp32 [rows][head_dim], device, written.
 * Asynchronous on `stream`.  Errors: INVALID_ARG (NULL or unaligned pointers,
 * rows < 0 or not a multiple of 32), UNSUPPORTED (bits not 2/4, head_dim not
 * 64/128), CUDA. */
kivi_status kivi_fake_quant_keys(const void* k, int64_t rows, int32_t head_dim, int32_t bits,
                                 int32_t per_token, float* k_hat, void* stream);

/* Static text for a status code; never NULL. */
const char* kivi_status_string(kivi_status status);

#ifdef __cplusplus
}
#endif

#endif /* KIVI_H */
