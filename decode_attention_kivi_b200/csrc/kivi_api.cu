// kivi_api.cu - the C ABI declared in include/kivi.h: validation, cache state
// bookkeeping on the host, and kernel launches.  No device memory is allocated
// here; the caller owns every buffer.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/kivi.h"
#include "kivi_kernels.h"
#include "kivi_launch.cuh"
#include "kivi_layout.cuh"

struct kivi_cache {
  kivi_config cfg;
  kivi_buffers bufs;
  std::vector<int32_t> S;      // token count per layer (the longest sequence's)
  std::vector<char> ragged;    // layer prefilled with a length per sequence
  std::vector<std::vector<int32_t>> Sb;  // ragged layers: token count per sequence
  std::vector<int32_t> steps;  // ragged layers: appends since the prefill
  int ngcap;
  long rec_bytes;
  int num_sms;
  int device;
};

namespace {

using kivi::kGroup;
using kivi::kResidual;
using kivi::kRingSlots;

kivi_status validate_config(const kivi_config* c) {
  if (!c) return KIVI_ERR_INVALID_ARG;
  if (c->batch < 1 || c->num_layers < 1 || c->num_kv_heads < 1 || c->num_q_heads < 1 ||
      c->max_tokens < 1 || c->head_dim < 1)
    return KIVI_ERR_INVALID_ARG;
  if (c->bits != 2 && c->bits != 4) return KIVI_ERR_UNSUPPORTED;
  if (c->group_size != kGroup || c->residual != kResidual) return KIVI_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return KIVI_ERR_UNSUPPORTED;
  if (c->num_q_heads % c->num_kv_heads != 0) return KIVI_ERR_UNSUPPORTED;
  const int hpk = c->num_q_heads / c->num_kv_heads;
  if (hpk != 1 && hpk != 2 && hpk != 4 && hpk != 8) return KIVI_ERR_UNSUPPORTED;
  return KIVI_OK;
}

// Per-layer prompt lengths of ragged layers ([L][B] int32) at the end of a
// handle's workspace, after the part the decode kernel uses.
size_t lens_bytes(const kivi_config* c) {
  return ((size_t)c->num_layers * c->batch * 4 + 255) / 256 * 256;
}
size_t decode_part_bytes(const kivi_config* c) {
  return (size_t)kivi::decode_workspace_bytes(c->head_dim, c->bits,
                                              c->num_q_heads / c->num_kv_heads,
                                              (long)c->batch * c->num_kv_heads);
}

long record_bytes(const kivi_config* c) {
  return kivi::RecordGeom{c->head_dim, c->bits}.bytes();
}

kivi_sizes sizes_of(const kivi_config* c) {
  kivi_sizes s;
  const size_t seqs = (size_t)c->num_layers * c->batch * c->num_kv_heads;
  const size_t ngcap = (size_t)kivi::num_groups(c->max_tokens);
  s.records_bytes = seqs * ngcap * (size_t)record_bytes(c);
  s.resid_k_bytes = seqs * kRingSlots * (size_t)c->head_dim * 2;
  s.resid_v_bytes = s.resid_k_bytes;
  s.workspace_bytes = (size_t)kivi::decode_workspace_bytes(
      c->head_dim, c->bits, c->num_q_heads / c->num_kv_heads,
      (long)c->batch * c->num_kv_heads) + lens_bytes(c);
  return s;
}

long partial_bytes(const kivi_config* c) {
  return kivi::decode_partial_bytes(c->head_dim, c->num_q_heads / c->num_kv_heads);
}

// Bytes before the partials: status header, tickets.
long fixed_workspace_bytes(const kivi_config* c) {
  const long pairs = (long)c->batch * c->num_kv_heads;
  return kivi::kWsHeader + kivi::ws_tickets_bytes(pairs);
}

// Points the decode arguments at a workspace of `bytes` bytes: status header,
// tickets, then as many CTAs' partials as fit.
void bind_workspace(kivi::DecodeArgs& a, const kivi_config* c, void* ws, size_t bytes) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  const long fixed = fixed_workspace_bytes(c);
  a.status = reinterpret_cast<uint32_t*>(base);
  a.tickets = reinterpret_cast<int*>(base + kivi::kWsHeader);
  a.partials = reinterpret_cast<float*>(base + fixed);
  const long room = (long)bytes - fixed;
  a.max_ctas = room > 0 ? (int)(room / partial_bytes(c)) : 0;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

kivi_status check_layer(const kivi_cache* h, int32_t layer) {
  if (!h) return KIVI_ERR_INVALID_ARG;
  if (layer < 0 || layer >= h->cfg.num_layers) return KIVI_ERR_INVALID_ARG;
  return KIVI_OK;
}

size_t layer_seqs(const kivi_cache* h) {
  return (size_t)h->cfg.batch * h->cfg.num_kv_heads;
}

uint8_t* layer_records(const kivi_cache* h, int32_t layer) {
  return static_cast<uint8_t*>(h->bufs.records) +
         (size_t)layer * layer_seqs(h) * h->ngcap * h->rec_bytes;
}

__nv_bfloat16* layer_ring(const kivi_cache* h, void* base, int32_t layer) {
  return static_cast<__nv_bfloat16*>(base) +
         (size_t)layer * layer_seqs(h) * kRingSlots * h->cfg.head_dim;
}

kivi_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KIVI_OK : KIVI_ERR_CUDA; }

const int* layer_lens(const kivi_cache* h, int32_t layer) {
  return reinterpret_cast<const int*>(static_cast<const uint8_t*>(h->bufs.workspace) +
                                      decode_part_bytes(&h->cfg)) +
         (size_t)layer * h->cfg.batch;
}

// The length whose shape the decode split gives every pair.  A ragged layer's
// pairs take the items of the length with the most items, which need not be the
// longest: a sequence just short of a flush has more residual rows than a longer
// one that has just flushed.  Each pair skips the items past its own.
int32_t decode_shape_len(const kivi_cache* h, int32_t layer) {
  if (!h->ragged[layer]) return h->S[layer];
  int32_t best = 0;
  int best_items = -1;
  for (const int32_t s : h->Sb[layer]) {
    const int items = kivi::decode_items(s);
    if (items > best_items || (items == best_items && s > best)) {
      best = s;
      best_items = items;
    }
  }
  return best;
}

}  // namespace

extern "C" {

kivi_status kivi_required_bytes(const kivi_config* cfg, kivi_sizes* out) {
  if (!out) return KIVI_ERR_INVALID_ARG;
  kivi_status st = validate_config(cfg);
  if (st != KIVI_OK) return st;
  *out = sizes_of(cfg);
  return KIVI_OK;
}

kivi_status kivi_record_layout(const kivi_config* cfg, size_t* rec_bytes,
                               int32_t* records_per_seq) {
  const kivi_status st = validate_config(cfg);
  if (st != KIVI_OK) return st;
  if (rec_bytes) *rec_bytes = (size_t)record_bytes(cfg);
  if (records_per_seq) *records_per_seq = kivi::num_groups(cfg->max_tokens);
  return KIVI_OK;
}

kivi_status kivi_cache_create(const kivi_config* cfg, const kivi_buffers* bufs,
                              kivi_cache** out) {
  if (!out || !bufs) return KIVI_ERR_INVALID_ARG;
  *out = nullptr;
  kivi_status st = validate_config(cfg);
  if (st != KIVI_OK) return st;
  const kivi_sizes need = sizes_of(cfg);
  if ((need.records_bytes && !bufs->records) || !bufs->resid_k || !bufs->resid_v ||
      !bufs->workspace)
    return KIVI_ERR_INVALID_ARG;
  if ((bufs->records && !aligned16(bufs->records)) || !aligned16(bufs->resid_k) ||
      !aligned16(bufs->resid_v) || !aligned16(bufs->workspace))
    return KIVI_ERR_INVALID_ARG;
  if (bufs->sizes.records_bytes < need.records_bytes ||
      bufs->sizes.resid_k_bytes < need.resid_k_bytes ||
      bufs->sizes.resid_v_bytes < need.resid_v_bytes ||
      bufs->sizes.workspace_bytes < need.workspace_bytes)
    return KIVI_ERR_BUFFER_TOO_SMALL;
  int device = 0, sms = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return KIVI_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
    return KIVI_ERR_CUDA;
  // status word and tickets start at zero (the decode kernel leaves the tickets at zero)
  const size_t clear = kivi::kWsHeader +
                       kivi::ws_tickets_bytes((long)cfg->batch * cfg->num_kv_heads);
  if (cudaMemset(bufs->workspace, 0, clear) != cudaSuccess) return KIVI_ERR_CUDA;
  kivi_cache* h = new (std::nothrow) kivi_cache();
  if (!h) return KIVI_ERR_INVALID_ARG;
  h->cfg = *cfg;
  h->bufs = *bufs;
  h->S.assign(cfg->num_layers, 0);
  h->ragged.assign(cfg->num_layers, 0);
  h->Sb.assign(cfg->num_layers, std::vector<int32_t>());
  h->steps.assign(cfg->num_layers, 0);
  h->ngcap = kivi::num_groups(cfg->max_tokens);
  h->rec_bytes = record_bytes(cfg);
  h->num_sms = sms;
  h->device = device;
  *out = h;
  return KIVI_OK;
}

void kivi_cache_destroy(kivi_cache* cache) { delete cache; }

kivi_status kivi_cache_length(const kivi_cache* cache, int32_t layer, int32_t* S,
                              int32_t* NG) {
  kivi_status st = check_layer(cache, layer);
  if (st != KIVI_OK) return st;
  if (S) *S = cache->S[layer];
  if (NG) *NG = kivi::num_groups(cache->S[layer]);
  return KIVI_OK;
}

kivi_status kivi_cache_reset(kivi_cache* cache, int32_t layer) {
  kivi_status st = check_layer(cache, layer);
  if (st != KIVI_OK) return st;
  cache->S[layer] = 0;
  cache->ragged[layer] = 0;
  cache->Sb[layer].clear();
  cache->steps[layer] = 0;
  return KIVI_OK;
}

kivi_status kivi_quantize_prefill(kivi_cache* cache, int32_t layer, const void* k,
                                  const void* v, int32_t S, void* stream) {
  kivi_status st = check_layer(cache, layer);
  if (st != KIVI_OK) return st;
  if (S < 0) return KIVI_ERR_INVALID_ARG;
  if (S > 0 && (!k || !v || !aligned16(k) || !aligned16(v))) return KIVI_ERR_INVALID_ARG;
  if (cache->S[layer] != 0) return KIVI_ERR_STATE;
  if (S > cache->cfg.max_tokens) return KIVI_ERR_CAPACITY;
  if (S > 0) {
    kivi::PrefillArgs a{};
    a.k = static_cast<const __nv_bfloat16*>(k);
    a.v = static_cast<const __nv_bfloat16*>(v);
    a.B = cache->cfg.batch;
    a.Hkv = cache->cfg.num_kv_heads;
    a.lens = nullptr;
    a.S = S;
    a.ng = kivi::num_groups(S);
    a.ngcap = cache->ngcap;
    a.records = layer_records(cache, layer);
    a.ring_k = layer_ring(cache, cache->bufs.resid_k, layer);
    a.ring_v = layer_ring(cache, cache->bufs.resid_v, layer);
    st = from_cuda(kivi::launch_prefill(cache->cfg.head_dim, cache->cfg.bits, a,
                                        static_cast<cudaStream_t>(stream)));
    if (st != KIVI_OK) return st;
  }
  cache->S[layer] = S;
  cache->ragged[layer] = 0;
  cache->Sb[layer].clear();
  cache->steps[layer] = 0;
  return KIVI_OK;
}

namespace {
kivi_status prefill_attn_shape(int32_t batch, int32_t hkv, int32_t hq, int32_t D, int32_t S) {
  if (batch < 1 || hkv < 1 || hq < 1 || S < 1) return KIVI_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return KIVI_ERR_UNSUPPORTED;
  if (hq % hkv != 0) return KIVI_ERR_UNSUPPORTED;
  if ((long)batch * hq * ((long)S + 128) >= (1L << 31)) return KIVI_ERR_INVALID_ARG;
  return KIVI_OK;
}
bool prefill_ptrs_ok(const void* q, const void* k, const void* v, const void* out) {
  return q && k && v && out && aligned16(q) && aligned16(k) && aligned16(v) && aligned16(out);
}
}  // namespace

kivi_status kivi_prefill_attention(kivi_cache* cache, int32_t layer, const void* q,
                                   const void* k, const void* v, int32_t S, float* out,
                                   float sm_scale, void* stream) {
  kivi_status st = check_layer(cache, layer);
  if (st != KIVI_OK) return st;
  const kivi_config& c = cache->cfg;
  st = prefill_attn_shape(c.batch, c.num_kv_heads, c.num_q_heads, c.head_dim, S);
  if (st != KIVI_OK) return st;
  if (!prefill_ptrs_ok(q, k, v, out) || !std::isfinite(sm_scale)) return KIVI_ERR_INVALID_ARG;
  if (cache->S[layer] != 0) return KIVI_ERR_STATE;
  if (S > c.max_tokens) return KIVI_ERR_CAPACITY;
  kivi::PrefillAttnArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.out = out;
  a.status = static_cast<uint32_t*>(cache->bufs.workspace);
  a.B = c.batch;
  a.Hkv = c.num_kv_heads;
  a.Hq = c.num_q_heads;
  a.S = S;
  a.sm_scale = sm_scale;
  a.records = layer_records(cache, layer);
  a.ring_k = layer_ring(cache, cache->bufs.resid_k, layer);
  a.ring_v = layer_ring(cache, cache->bufs.resid_v, layer);
  a.ngcap = cache->ngcap;
  a.device = cache->device;
  st = from_cuda(kivi::launch_prefill_attention(c.head_dim, c.bits, a,
                                                static_cast<cudaStream_t>(stream)));
  if (st != KIVI_OK) return st;
  cache->S[layer] = S;
  cache->ragged[layer] = 0;
  cache->Sb[layer].clear();
  cache->steps[layer] = 0;
  return KIVI_OK;
}

kivi_status kivi_causal_attention(const void* q, const void* k, const void* v, int32_t batch,
                                  int32_t num_kv_heads, int32_t num_q_heads, int32_t head_dim,
                                  int32_t S, float* out, float sm_scale, uint32_t* status,
                                  void* stream) {
  kivi_status st = prefill_attn_shape(batch, num_kv_heads, num_q_heads, head_dim, S);
  if (st != KIVI_OK) return st;
  if (!prefill_ptrs_ok(q, k, v, out) || !std::isfinite(sm_scale)) return KIVI_ERR_INVALID_ARG;
  if (status != nullptr && ((uintptr_t)status & 3u) != 0) return KIVI_ERR_INVALID_ARG;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return KIVI_ERR_CUDA;
  kivi::PrefillAttnArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.out = out;
  a.status = status;
  a.B = batch;
  a.Hkv = num_kv_heads;
  a.Hq = num_q_heads;
  a.S = S;
  a.sm_scale = sm_scale;
  a.device = device;
  return from_cuda(kivi::launch_prefill_attention(head_dim, 2, a,
                                                  static_cast<cudaStream_t>(stream)));
}

kivi_status kivi_quantize_prefill_ragged(kivi_cache* cache, int32_t layer, const void* k,
                                         const void* v, int32_t S_max, const int32_t* lengths,
                                         void* stream) {
  kivi_status st = check_layer(cache, layer);
  if (st != KIVI_OK) return st;
  if (!lengths || S_max < 0) return KIVI_ERR_INVALID_ARG;
  const int B = cache->cfg.batch;
  int longest = 0;
  for (int b = 0; b < B; ++b) {
    if (lengths[b] < 0 || lengths[b] > S_max) return KIVI_ERR_INVALID_ARG;
    longest = std::max(longest, (int)lengths[b]);
  }
  if (longest > 0 && (!k || !v || !aligned16(k) || !aligned16(v))) return KIVI_ERR_INVALID_ARG;
  if (cache->S[layer] != 0) return KIVI_ERR_STATE;
  if (S_max > cache->cfg.max_tokens) return KIVI_ERR_CAPACITY;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* lens = const_cast<int*>(layer_lens(cache, layer));
  // the lengths go to the workspace once; the kernels derive S_b = lens[b] + steps
  if (cudaMemcpyAsync(lens, lengths, sizeof(int32_t) * B, cudaMemcpyHostToDevice, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return KIVI_ERR_CUDA;
  if (longest > 0) {
    kivi::PrefillArgs a{};
    a.k = static_cast<const __nv_bfloat16*>(k);
    a.v = static_cast<const __nv_bfloat16*>(v);
    a.lens = lens;
    a.B = B;
    a.Hkv = cache->cfg.num_kv_heads;
    a.S = S_max;  // the row stride of k and v
    a.ng = kivi::num_groups(longest);
    a.ngcap = cache->ngcap;
    a.records = layer_records(cache, layer);
    a.ring_k = layer_ring(cache, cache->bufs.resid_k, layer);
    a.ring_v = layer_ring(cache, cache->bufs.resid_v, layer);
    st = from_cuda(kivi::launch_prefill(cache->cfg.head_dim, cache->cfg.bits, a, s));
    if (st != KIVI_OK) return st;
  }
  cache->S[layer] = longest;
  cache->ragged[layer] = 1;
  cache->Sb[layer].assign(lengths, lengths + B);
  cache->steps[layer] = 0;
  return KIVI_OK;
}

kivi_status kivi_cache_lengths(const kivi_cache* cache, int32_t layer, int32_t* S_out) {
  kivi_status st = check_layer(cache, layer);
  if (st != KIVI_OK) return st;
  if (!S_out) return KIVI_ERR_INVALID_ARG;
  for (int b = 0; b < cache->cfg.batch; ++b)
    S_out[b] = cache->ragged[layer] ? cache->Sb[layer][b] : cache->S[layer];
  return KIVI_OK;
}

kivi_status kivi_append_token(kivi_cache* cache, int32_t layer, const void* k_new,
                              const void* v_new, void* stream) {
  kivi_status st = check_layer(cache, layer);
  if (st != KIVI_OK) return st;
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return KIVI_ERR_INVALID_ARG;
  const int S = cache->S[layer];  // the longest sequence's
  if (S + 1 > cache->cfg.max_tokens) return KIVI_ERR_CAPACITY;
  kivi::AppendArgs a{};
  a.k_new = static_cast<const __nv_bfloat16*>(k_new);
  a.v_new = static_cast<const __nv_bfloat16*>(v_new);
  a.lens = cache->ragged[layer] ? layer_lens(cache, layer) : nullptr;
  a.steps = cache->steps[layer];
  a.B = cache->cfg.batch;
  a.Hkv = cache->cfg.num_kv_heads;
  a.S = S;
  a.ngcap = cache->ngcap;
  a.ring_k = layer_ring(cache, cache->bufs.resid_k, layer);
  a.ring_v = layer_ring(cache, cache->bufs.resid_v, layer);
  a.records = layer_records(cache, layer);
  st = from_cuda(kivi::launch_append(cache->cfg.head_dim, cache->cfg.bits, a,
                                     static_cast<cudaStream_t>(stream)));
  if (st != KIVI_OK) return st;
  cache->S[layer] = S + 1;
  if (cache->ragged[layer]) {
    ++cache->steps[layer];
    for (int32_t& x : cache->Sb[layer]) ++x;
  }
  return KIVI_OK;
}

kivi_status kivi_decode_attention(const kivi_cache* cache, int32_t layer, const void* q,
                                  float* out, float sm_scale, void* stream) {
  kivi_status st = check_layer(cache, layer);
  if (st != KIVI_OK) return st;
  if (!q || !out || !aligned16(q) || !aligned16(out)) return KIVI_ERR_INVALID_ARG;
  if (!std::isfinite(sm_scale)) return KIVI_ERR_INVALID_ARG;
  if (cache->S[layer] == 0) return KIVI_ERR_STATE;
  if (cache->ragged[layer] &&
      *std::min_element(cache->Sb[layer].begin(), cache->Sb[layer].end()) == 0)
    return KIVI_ERR_STATE;  // a sequence without tokens has no attention
  kivi::DecodeArgs a{};
  a.records = layer_records(cache, layer);
  a.ring_k = layer_ring(cache, cache->bufs.resid_k, layer);
  a.ring_v = layer_ring(cache, cache->bufs.resid_v, layer);
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.out = out;
  bind_workspace(a, &cache->cfg, cache->bufs.workspace, decode_part_bytes(&cache->cfg));
  a.lens = cache->ragged[layer] ? layer_lens(cache, layer) : nullptr;
  a.steps = cache->steps[layer];
  a.B = cache->cfg.batch;
  a.Hkv = cache->cfg.num_kv_heads;
  a.Hq = cache->cfg.num_q_heads;
  a.S = decode_shape_len(cache, layer);
  a.ngcap = cache->ngcap;
  a.sm_scale = sm_scale;
  a.num_sms = cache->num_sms;
  a.device = cache->device;
  return from_cuda(kivi::launch_decode(cache->cfg.head_dim, cache->cfg.bits, a,
                                       static_cast<cudaStream_t>(stream)));
}

kivi_status kivi_check_device_status(kivi_cache* cache, void* stream, uint32_t* code_out) {
  if (!cache) return KIVI_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return KIVI_ERR_CUDA;
  uint32_t code = 0;
  if (cudaMemcpy(&code, cache->bufs.workspace, sizeof code, cudaMemcpyDeviceToHost) !=
      cudaSuccess)
    return KIVI_ERR_CUDA;
  // after a failure the tickets may be left counting: clear them with the word
  const size_t clear =
      kivi::kWsHeader +
      kivi::ws_tickets_bytes((long)cache->cfg.batch * cache->cfg.num_kv_heads);
  if (code != 0 && cudaMemset(cache->bufs.workspace, 0, clear) != cudaSuccess)
    return KIVI_ERR_CUDA;
  if (code_out) *code_out = code;
  return code ? KIVI_ERR_DEVICE : KIVI_OK;
}

// ---- the 16-bit baseline ----

namespace {
kivi_status bf16_shape(int32_t batch, int32_t hkv, int32_t hq, int32_t D) {
  if (batch < 1 || hkv < 1 || hq < 1) return KIVI_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return KIVI_ERR_UNSUPPORTED;
  if (hq % hkv != 0) return KIVI_ERR_UNSUPPORTED;
  const int hpk = hq / hkv;
  if (hpk != 1 && hpk != 2 && hpk != 4 && hpk != 8) return KIVI_ERR_UNSUPPORTED;
  return KIVI_OK;
}
size_t bf16_fixed_bytes(int32_t batch, int32_t hkv) {
  return kivi::kWsHeader + kivi::ws_tickets_bytes((long)batch * hkv);
}
}  // namespace

kivi_status kivi_bf16_workspace_bytes(int32_t batch, int32_t num_kv_heads, int32_t num_q_heads,
                                      int32_t head_dim, size_t* bytes) {
  if (!bytes) return KIVI_ERR_INVALID_ARG;
  const kivi_status st = bf16_shape(batch, num_kv_heads, num_q_heads, head_dim);
  if (st != KIVI_OK) return st;
  *bytes = bf16_fixed_bytes(batch, num_kv_heads) +
           kivi::bf16_partial_bytes(head_dim, num_q_heads / num_kv_heads);
  return KIVI_OK;
}

kivi_status kivi_bf16_decode_attention(const void* k_cache, const void* v_cache, int32_t batch,
                                       int32_t num_kv_heads, int32_t num_q_heads,
                                       int32_t head_dim, int32_t max_tokens, int32_t S,
                                       const void* q, float* out, float sm_scale,
                                       void* workspace, size_t workspace_bytes, void* stream) {
  size_t need = 0;
  const kivi_status st =
      kivi_bf16_workspace_bytes(batch, num_kv_heads, num_q_heads, head_dim, &need);
  if (st != KIVI_OK) return st;
  if (!k_cache || !v_cache || !q || !out || !workspace) return KIVI_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(q) || !aligned16(out) ||
      !aligned16(workspace))
    return KIVI_ERR_INVALID_ARG;
  if (S < 1 || S > max_tokens || workspace_bytes < need || !std::isfinite(sm_scale))
    return KIVI_ERR_INVALID_ARG;
  if ((long)batch * num_kv_heads * max_tokens >= (1L << 31)) return KIVI_ERR_INVALID_ARG;
  int device = 0, sms = 0;
  if (cudaGetDevice(&device) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
    return KIVI_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  kivi::Bf16DecodeArgs a{};
  a.k = static_cast<const __nv_bfloat16*>(k_cache);
  a.v = static_cast<const __nv_bfloat16*>(v_cache);
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.out = out;
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.tickets = reinterpret_cast<int*>(ws + kivi::kWsHeader);
  a.partials = reinterpret_cast<float*>(ws + bf16_fixed_bytes(batch, num_kv_heads));
  a.B = batch;
  a.Hkv = num_kv_heads;
  a.Hq = num_q_heads;
  a.D = head_dim;
  a.Smax = max_tokens;
  a.S = S;
  a.sm_scale = sm_scale;
  a.num_sms = sms;
  a.device = device;
  return from_cuda(kivi::launch_bf16_decode(a, static_cast<cudaStream_t>(stream)));
}

kivi_status kivi_bf16_status(void* workspace, int32_t batch, int32_t num_kv_heads, void* stream,
                             uint32_t* code_out) {
  if (!workspace || batch < 1 || num_kv_heads < 1) return KIVI_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KIVI_ERR_CUDA;
  uint32_t code = 0;
  if (cudaMemcpy(&code, workspace, sizeof code, cudaMemcpyDeviceToHost) != cudaSuccess)
    return KIVI_ERR_CUDA;
  if (code != 0 &&
      cudaMemset(workspace, 0, bf16_fixed_bytes(batch, num_kv_heads)) != cudaSuccess)
    return KIVI_ERR_CUDA;
  if (code_out) *code_out = code;
  return code ? KIVI_ERR_DEVICE : KIVI_OK;
}

// ---- key-granularity ablation ----

kivi_status kivi_fake_quant_keys(const void* k, int64_t rows, int32_t head_dim, int32_t bits,
                                 int32_t per_token, float* k_hat, void* stream) {
  if (bits != 2 && bits != 4) return KIVI_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return KIVI_ERR_UNSUPPORTED;
  if (rows < 0 || rows % kGroup != 0) return KIVI_ERR_INVALID_ARG;
  if (rows == 0) return KIVI_OK;
  if (!k || !k_hat || !aligned16(k) || !aligned16(k_hat)) return KIVI_ERR_INVALID_ARG;
  return from_cuda(kivi::launch_fake_quant_keys(head_dim, bits,
                                                static_cast<const __nv_bfloat16*>(k), rows,
                                                k_hat, per_token ? 1 : 0,
                                                static_cast<cudaStream_t>(stream)));
}

kivi_status kivi_cache_bytes(const kivi_config* cfg, int32_t S, double* stored,
                             double* codes_only, double* convention) {
  kivi_status st = validate_config(cfg);
  if (st != KIVI_OK) return st;
  if (S < 1) return KIVI_ERR_INVALID_ARG;
  const double lh = (double)cfg->num_layers * cfg->num_kv_heads;
  const double codes_per_tok = lh * cfg->head_dim * 2.0 * cfg->bits / 8.0;
  const double bf16_per_tok = lh * cfg->head_dim * 2.0 * 2.0;
  const int ng = kivi::num_groups(S);
  const int r = S - ng * kGroup;
  if (stored) *stored = (ng * lh * (double)record_bytes(cfg) + r * bf16_per_tok) / S;
  if (codes_only) *codes_only = ((double)ng * kGroup * codes_per_tok + r * bf16_per_tok) / S;
  if (convention) *convention = codes_per_tok + kResidual * bf16_per_tok / S;
  return KIVI_OK;
}

const char* kivi_status_string(kivi_status status) {
  switch (status) {
    case KIVI_OK: return "ok";
    case KIVI_ERR_INVALID_ARG: return "invalid argument";
    case KIVI_ERR_UNSUPPORTED: return "unsupported configuration";
    case KIVI_ERR_BUFFER_TOO_SMALL: return "buffer smaller than kivi_required_bytes";
    case KIVI_ERR_CAPACITY: return "cache capacity (max_tokens) exceeded";
    case KIVI_ERR_STATE: return "call not valid in the layer's current state";
    case KIVI_ERR_CUDA: return "CUDA runtime error";
    case KIVI_ERR_DEVICE: return "a kernel reported a failure in the device status word";
    case KIVI_ERR_SCRATCH_LIMIT:
      return "call needs more split-K scratch than KIVI_STATIC_SCRATCH_BYTES";
  }
  return "unknown status";
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode attention with a static scratch array, for callers that cannot
// allocate device memory (see kivi_decode_attention_static_scratch in kivi.h).
// ---------------------------------------------------------------------------

// The split-K partials of kivi_decode_attention_static_scratch: the same layout
// as a handle's workspace (header with the status word, then m/l, then acc).
// In host code this name is only a stand-in for the device array; its device
// address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_kivi_static_scratch[KIVI_STATIC_SCRATCH_BYTES];

namespace {

using kivi::kMaxDevices;

struct StaticScratchSlot {
  void* ptr = nullptr;  // device address of g_kivi_static_scratch on this device
  int num_sms = 0;
  int device = 0;
};

std::mutex g_static_mu;
StaticScratchSlot g_static_slots[kMaxDevices];

// Once per device, with that device current: look up the array's address and
// clear the whole array on `stream` (the status word and the tickets of any
// shape must start at zero; the decode kernel leaves the tickets at zero).
kivi_status static_scratch_slot(cudaStream_t stream, StaticScratchSlot* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KIVI_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_mu);
  StaticScratchSlot& slot = g_static_slots[dev];
  if (slot.ptr == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_kivi_static_scratch) != cudaSuccess || p == nullptr)
      return KIVI_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return KIVI_ERR_CUDA;
    if (cudaMemsetAsync(p, 0, KIVI_STATIC_SCRATCH_BYTES, stream) != cudaSuccess)
      return KIVI_ERR_CUDA;
    slot.ptr = p;
    slot.num_sms = sms;
    slot.device = dev;
  }
  *out = slot;
  return KIVI_OK;
}

}  // namespace

extern "C" kivi_status kivi_decode_attention_static_scratch(
    const kivi_config* cfg, const void* records, const void* resid_k, const void* resid_v,
    int32_t layer, int32_t S, const void* q, float* out, float sm_scale, void* stream) {
  kivi_status st = validate_config(cfg);
  if (st != KIVI_OK) return st;
  const int ngcap = kivi::num_groups(cfg->max_tokens);
  if (layer < 0 || layer >= cfg->num_layers) return KIVI_ERR_INVALID_ARG;
  if ((ngcap > 0 && !records) || !resid_k || !resid_v || !q || !out)
    return KIVI_ERR_INVALID_ARG;
  if ((records && !aligned16(records)) || !aligned16(resid_k) || !aligned16(resid_v) ||
      !aligned16(q) || !aligned16(out))
    return KIVI_ERR_INVALID_ARG;
  if (!std::isfinite(sm_scale)) return KIVI_ERR_INVALID_ARG;
  if (S < 0) return KIVI_ERR_INVALID_ARG;
  if (S == 0) return KIVI_ERR_STATE;
  if (S > cfg->max_tokens) return KIVI_ERR_CAPACITY;
  const long pairs = (long)cfg->batch * cfg->num_kv_heads;
  const int hpk = cfg->num_q_heads / cfg->num_kv_heads;

  // the fixed part (status word, tickets) must fit before any device work
  const long fixed = fixed_workspace_bytes(cfg);
  if (fixed + partial_bytes(cfg) > (long)KIVI_STATIC_SCRATCH_BYTES) return KIVI_ERR_SCRATCH_LIMIT;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  StaticScratchSlot slot;
  st = static_scratch_slot(s, &slot);
  if (st != KIVI_OK) return st;
  const int grid = kivi::decode_grid_ctas(cfg->head_dim, cfg->bits, hpk, pairs, S, slot.num_sms);
  if (grid < 1) return KIVI_ERR_UNSUPPORTED;
  if (fixed + grid * partial_bytes(cfg) > (long)KIVI_STATIC_SCRATCH_BYTES)
    return KIVI_ERR_SCRATCH_LIMIT;

  const size_t seqs = (size_t)pairs;
  const long rb = record_bytes(cfg);
  kivi::DecodeArgs a{};
  a.records = static_cast<const uint8_t*>(records) + (size_t)layer * seqs * ngcap * rb;
  a.ring_k = static_cast<const __nv_bfloat16*>(resid_k) +
             (size_t)layer * seqs * kRingSlots * cfg->head_dim;
  a.ring_v = static_cast<const __nv_bfloat16*>(resid_v) +
             (size_t)layer * seqs * kRingSlots * cfg->head_dim;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.out = out;
  bind_workspace(a, cfg, slot.ptr, KIVI_STATIC_SCRATCH_BYTES);
  a.B = cfg->batch;
  a.Hkv = cfg->num_kv_heads;
  a.Hq = cfg->num_q_heads;
  a.S = S;
  a.ngcap = ngcap;
  a.sm_scale = sm_scale;
  a.num_sms = slot.num_sms;
  a.device = slot.device;
  return from_cuda(kivi::launch_decode(cfg->head_dim, cfg->bits, a, s));
}

extern "C" kivi_status kivi_static_scratch_status(void* stream, uint32_t* code_out) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  StaticScratchSlot slot;
  kivi_status st = static_scratch_slot(s, &slot);
  if (st != KIVI_OK) return st;
  if (cudaStreamSynchronize(s) != cudaSuccess) return KIVI_ERR_CUDA;
  uint32_t code = 0;
  if (cudaMemcpy(&code, slot.ptr, sizeof code, cudaMemcpyDeviceToHost) != cudaSuccess)
    return KIVI_ERR_CUDA;
  // after a failure the tickets may be left counting: clear the whole array
  if (code != 0 && cudaMemset(slot.ptr, 0, KIVI_STATIC_SCRATCH_BYTES) != cudaSuccess)
    return KIVI_ERR_CUDA;
  if (code_out) *code_out = code;
  return code ? KIVI_ERR_DEVICE : KIVI_OK;
}

#ifdef KIVI_DEBUG_BUILD
#include "../../include/kivi_debug.h"

extern "C" kivi_status kivi_debug_overstate_copies(uint32_t bytes) {
  return from_cuda(kivi::debug_overstate_copies(bytes));
}
#endif
