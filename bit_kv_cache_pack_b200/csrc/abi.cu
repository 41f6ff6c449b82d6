// C ABI of the OmniKVQuant kernels: argument validation and launches.
// Every check runs on the host before any launch; see include/omnikv.h.
#include <cuda_runtime.h>

#include "../../include/omnikv_testing.h"
#include "abi_internal.h"
#include "common.cuh"
#include "kernels.h"

using namespace omnikv;

namespace {

bool aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

// the kernels' key metadata format of a validated omnikv_config.key_meta_format
int meta_of(int32_t key_meta_format) {
  return key_meta_format == OMNIKV_META_MXFP4 ? kMetaMx : key_meta_format == OMNIKV_META_TURBO ? kMetaTurbo : kMetaFp16;
}

omnikv_status check_config(const omnikv_config* cfg) {
  if (!cfg) return OMNIKV_ERR_INVALID_ARG;
  if (cfg->head_dim != kHeadDim || cfg->window != kWindow) return OMNIKV_ERR_UNSUPPORTED;
  if ((cfg->key_bits != 2 && cfg->key_bits != 4) || (cfg->value_bits != 2 && cfg->value_bits != 4))
    return OMNIKV_ERR_UNSUPPORTED;
  if (cfg->num_kv_heads < 1 || cfg->num_q_heads < 1 || cfg->num_q_heads % cfg->num_kv_heads)
    return OMNIKV_ERR_INVALID_ARG;
  if (cfg->num_q_heads / cfg->num_kv_heads > kMaxGroup) return OMNIKV_ERR_UNSUPPORTED;
  if (!cfg->key_codebook || !cfg->value_codebook || !cfg->key_signs || !cfg->value_rot)
    return OMNIKV_ERR_INVALID_ARG;
  if (!aligned(cfg->key_signs, 16) || !aligned(cfg->value_rot, 16)) return OMNIKV_ERR_INVALID_ARG;
  if (cfg->key_meta_format != OMNIKV_META_FP16 && cfg->key_meta_format != OMNIKV_META_MXFP4 &&
      cfg->key_meta_format != OMNIKV_META_TURBO)
    return OMNIKV_ERR_UNSUPPORTED;
  return OMNIKV_OK;
}

omnikv_status check_cache(const omnikv_cache* c) {
  if (!c || !c->records || !c->key_tail || !c->modality || !c->seq_lens) return OMNIKV_ERR_INVALID_ARG;
  if (c->batch < 1 || c->cap_tokens < kWindow || c->cap_tokens % kWindow) return OMNIKV_ERR_INVALID_ARG;
  if (c->max_seq_len < 0 || c->max_seq_len > c->cap_tokens) return OMNIKV_ERR_INVALID_ARG;
  if (!aligned(c->records, 16) || !aligned(c->key_tail, 16) || !aligned(c->modality, 16) ||
      !aligned(c->seq_lens, 4) || (c->error_word && !aligned(c->error_word, 4)))
    return OMNIKV_ERR_INVALID_ARG;
  return OMNIKV_OK;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

}  // namespace

namespace omnikv {

namespace {

// Splits for one full wave of `per_sm` resident decode CTAs per SM over the whole
// batch (a second, partial wave would double the time), with at least 4 windows
// (one per warp) per split.
int32_t wave_splits(long long units, int per_sm, int nw) {
  const long long target = (long long)per_sm * sm_count();
  long long s = target / units;
  // a large batch leaves little split parallelism, and its lengths may differ
  // (fixed-size splits of short sequences are empty): at least 8 splits (on the
  // ragged 64-sequence workload 8 splits measured 1.7x faster than 2, and faster
  // than 9 or 16)
  if (4 * units >= target && s < 8) s = 8;
  const long long max_s = (nw + 3) / 4;
  if (s > max_s) s = max_s;
  if (s < 1) s = 1;
  if (s > kMaxSplits) s = kMaxSplits;
  return (int32_t)s;
}

int split_windows_of(const omnikv_cache* c, int32_t S) {
  const int nw = (c->max_seq_len + kWindow - 1) / kWindow;
  return nw > 0 ? (nw + S - 1) / S : 1;
}

}  // namespace

// The library's split count: one wave of the body that will run it. For 2-bit
// caches the cooperative body takes the split if its wave leaves at most
// kCoopMaxWindows windows per split, else the per-warp body sizes it.
int32_t resolve_splits(const omnikv_config* cfg, const omnikv_cache* c, int32_t requested) {
  if (requested > 0) return requested;
  const int nw = (c->max_seq_len + kWindow - 1) / kWindow;
  if (nw <= 0) return 1;
  const long long units = (long long)c->batch * cfg->num_kv_heads;
  if (cfg->key_bits != 2 || cfg->value_bits != 2)
    return wave_splits(units, decode_ctas_per_sm(decode_body(cfg->key_bits, cfg->value_bits, meta_of(cfg->key_meta_format), 0)), nw);
  const int32_t s = wave_splits(units, decode_ctas_per_sm(kBodyCoop), nw);
  if (split_windows_of(c, s) <= kCoopMaxWindows) return s;
  return wave_splits(units, decode_ctas_per_sm(kBodyWarp), nw);
}

// Resident CTAs of a decode-step launch with S splits (the residency of its body).
long long step_residency(const omnikv_config* cfg, const omnikv_cache* c, int32_t S) {
  const int body = decode_body(cfg->key_bits, cfg->value_bits, meta_of(cfg->key_meta_format), split_windows_of(c, S));
  return (long long)decode_ctas_per_sm(body) * sm_count();
}

omnikv_status prepare_decode(const omnikv_config* cfg, const omnikv_cache* cache, const void* q, void* partials,
                             int32_t num_splits, DecodeParams* p) {
  omnikv_status st = check_config(cfg);
  if (st != OMNIKV_OK) return st;
  if ((st = check_cache(cache)) != OMNIKV_OK) return st;
  if (!q || !partials || num_splits < 0) return OMNIKV_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(partials, 16)) return OMNIKV_ERR_INVALID_ARG;
  p->key_cb = cfg->key_codebook;
  p->val_cb = cfg->value_codebook;
  p->key_signs = cfg->key_signs;
  p->value_rot = cfg->value_rot;
  p->key_bits = cfg->key_bits;
  p->value_bits = cfg->value_bits;
  p->key_meta = meta_of(cfg->key_meta_format);
  p->num_kv_heads = cfg->num_kv_heads;
  p->group = cfg->num_q_heads / cfg->num_kv_heads;
  p->records = static_cast<const uint8_t*>(cache->records);
  p->modality = cache->modality;
  p->seq_lens = cache->seq_lens;
  p->cap_tokens = cache->cap_tokens;
  p->cap_windows = cache->cap_tokens / kWindow;
  p->q = static_cast<const __half*>(q);
  p->partials = static_cast<Partial*>(partials);
  p->num_splits = resolve_splits(cfg, cache, num_splits);
  if (p->num_splits > kMaxSplits) return OMNIKV_ERR_UNSUPPORTED;
  const int nw = (cache->max_seq_len + kWindow - 1) / kWindow;
  p->split_windows = nw > 0 ? (nw + p->num_splits - 1) / p->num_splits : 1;
  p->error_word = cache->error_word;
  p->batch = cache->batch;
  p->len_add = 0;
  p->step_flags = nullptr;
  p->append_ctas = 0;
  p->stream = 0;
  p->flag_wait_ns = kFlagWaitNs;
  return OMNIKV_OK;
}

omnikv_status prepare_combine(const omnikv_config* cfg, const omnikv_cache* cache, const void* partials,
                              int32_t num_splits, float* out, CombineParams* p) {
  omnikv_status st = check_config(cfg);
  if (st != OMNIKV_OK) return st;
  if ((st = check_cache(cache)) != OMNIKV_OK) return st;
  if (!partials || !out || num_splits < 0) return OMNIKV_ERR_INVALID_ARG;
  if (!aligned(partials, 16) || !aligned(out, 16)) return OMNIKV_ERR_INVALID_ARG;
  p->value_rot = cfg->value_rot;
  p->num_kv_heads = cfg->num_kv_heads;
  p->group = cfg->num_q_heads / cfg->num_kv_heads;
  p->partials = static_cast<const Partial*>(partials);
  p->num_splits = resolve_splits(cfg, cache, num_splits);
  if (p->num_splits > kMaxSplits) return OMNIKV_ERR_UNSUPPORTED;
  p->out = out;
  p->seq_lens = cache->seq_lens;
  p->len_add = 0;
  p->cap_tokens = cache->cap_tokens;
  return OMNIKV_OK;
}

omnikv_status validate_config_cache(const omnikv_config* cfg, const omnikv_cache* cache) {
  omnikv_status st = check_config(cfg);
  if (st != OMNIKV_OK) return st;
  return check_cache(cache);
}

}  // namespace omnikv

extern "C" {

size_t omnikv_record_bytes(int32_t key_bits, int32_t value_bits) {
  if ((key_bits != 2 && key_bits != 4) || (value_bits != 2 && value_bits != 4)) return 0;
  return (size_t)RecordLayout(key_bits, value_bits).bytes;
}

size_t omnikv_record_bytes_meta(int32_t key_bits, int32_t value_bits, int32_t key_meta_format) {
  if ((key_bits != 2 && key_bits != 4) || (value_bits != 2 && value_bits != 4)) return 0;
  if (key_meta_format != OMNIKV_META_FP16 && key_meta_format != OMNIKV_META_MXFP4 &&
      key_meta_format != OMNIKV_META_TURBO)
    return 0;
  return (size_t)RecordLayout(key_bits, value_bits, meta_of(key_meta_format)).bytes;
}

size_t omnikv_partials_bytes(int32_t batch, int32_t num_q_heads, int32_t num_splits) {
  if (batch < 1 || num_q_heads < 1 || num_splits < 1) return 0;
  return (size_t)batch * num_q_heads * num_splits * sizeof(Partial);
}

int32_t omnikv_default_splits(const omnikv_config* cfg, const omnikv_cache* cache) {
  if (check_config(cfg) != OMNIKV_OK || check_cache(cache) != OMNIKV_OK) return 0;
  return resolve_splits(cfg, cache, 0);
}

namespace {

void fill_write_params(const omnikv_config* cfg, const omnikv_cache* cache, const void* k_new, const void* v_new,
                       const uint8_t* modality_new, int32_t n_new, WriteParams* p) {
  p->key_cb = cfg->key_codebook;
  p->val_cb = cfg->value_codebook;
  p->key_signs = cfg->key_signs;
  p->value_rot = cfg->value_rot;
  p->key_bits = cfg->key_bits;
  p->value_bits = cfg->value_bits;
  p->key_meta = meta_of(cfg->key_meta_format);
  p->num_kv_heads = cfg->num_kv_heads;
  p->records = static_cast<uint8_t*>(cache->records);
  p->key_tail = static_cast<__half*>(cache->key_tail);
  p->modality = cache->modality;
  p->seq_lens = cache->seq_lens;
  p->error_word = cache->error_word;
  p->cap_tokens = cache->cap_tokens;
  p->cap_windows = cache->cap_tokens / kWindow;
  p->k_new = static_cast<const __half*>(k_new);
  p->v_new = static_cast<const __half*>(v_new);
  p->mod_new = modality_new;
  p->n_new = n_new;
  p->tc_values = 0;
  p->step_flags = nullptr;
  p->vrot_dump = nullptr;
}

}  // namespace

omnikv_status omnikv_write_cache(const omnikv_config* cfg, omnikv_cache* cache, const void* k_new,
                                 const void* v_new, const uint8_t* modality_new, int32_t n_new,
                                 void* stream) {
  omnikv_status st = check_config(cfg);
  if (st != OMNIKV_OK) return st;
  if ((st = check_cache(cache)) != OMNIKV_OK) return st;
  if (n_new < 1 || !k_new || !v_new || !modality_new) return OMNIKV_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16)) return OMNIKV_ERR_INVALID_ARG;
  if ((long long)cache->max_seq_len + n_new > cache->cap_tokens) return OMNIKV_ERR_CAPACITY;
  WriteParams p;
  fill_write_params(cfg, cache, k_new, v_new, modality_new, n_new, &p);
  if (launch_write(p, cache->batch, static_cast<cudaStream_t>(stream)) != cudaSuccess) return OMNIKV_ERR_CUDA;
  cache->max_seq_len += n_new;
  return OMNIKV_OK;
}

omnikv_status omnikv_write_cache_rotations(const omnikv_config* cfg, omnikv_cache* cache, const void* k_new,
                                           const void* v_new, const uint8_t* modality_new, int32_t n_new,
                                           float* v_rot, void* stream) {
  omnikv_status st = check_config(cfg);
  if (st != OMNIKV_OK) return st;
  if ((st = check_cache(cache)) != OMNIKV_OK) return st;
  if (n_new < 1 || !k_new || !v_new || !modality_new || !v_rot) return OMNIKV_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(v_rot, 16)) return OMNIKV_ERR_INVALID_ARG;
  if ((long long)cache->max_seq_len + n_new > cache->cap_tokens) return OMNIKV_ERR_CAPACITY;
  WriteParams p;
  fill_write_params(cfg, cache, k_new, v_new, modality_new, n_new, &p);
  p.vrot_dump = v_rot;
  if (launch_write(p, cache->batch, static_cast<cudaStream_t>(stream)) != cudaSuccess) return OMNIKV_ERR_CUDA;
  cache->max_seq_len += n_new;
  return OMNIKV_OK;
}

omnikv_status omnikv_decode_attention(const omnikv_config* cfg, const omnikv_cache* cache, const void* q,
                                      void* partials, int32_t num_splits, void* stream) {
  DecodeParams p;
  const omnikv_status st = prepare_decode(cfg, cache, q, partials, num_splits, &p);
  if (st != OMNIKV_OK) return st;
  if (launch_decode(p, cache->batch, static_cast<cudaStream_t>(stream)) != cudaSuccess) return OMNIKV_ERR_CUDA;
  return OMNIKV_OK;
}

omnikv_status omnikv_combine(const omnikv_config* cfg, const omnikv_cache* cache, const void* partials,
                             int32_t num_splits, float* out, void* stream) {
  CombineParams p;
  const omnikv_status st = prepare_combine(cfg, cache, partials, num_splits, out, &p);
  if (st != OMNIKV_OK) return st;
  if (launch_combine(p, cache->batch, static_cast<cudaStream_t>(stream)) != cudaSuccess) return OMNIKV_ERR_CUDA;
  return OMNIKV_OK;
}

}  // extern "C"

namespace {

// The split count of a decode step, whether its append runs inside the decode
// launch and with how many append CTAs, for the cache as the step sees it
// (max_seq_len already counting the appended token). Fused only when every CTA of
// that launch is resident at once, so a waiting warp never waits on an
// unscheduled CTA. The append CTAs fill the slots the decode CTAs leave, each
// appending for at most kMaxAppendsPerCta (sequence, kv head) units in turn (its
// flags are read only by the last window of each split); with num_splits = 0 the
// default split count is lowered (by at most half) when even that does not fit.
constexpr long long kMaxAppendsPerCta = 4;

void plan_step(const omnikv_config* cfg, const omnikv_cache* after, int32_t num_splits, int32_t* S, bool* fused,
               int32_t* append_ctas = nullptr) {
  const long long units = (long long)after->batch * cfg->num_kv_heads;
  const long long min_append = (units + kMaxAppendsPerCta - 1) / kMaxAppendsPerCta;
  *S = resolve_splits(cfg, after, num_splits);
  const long long resident = step_residency(cfg, after, *S);
  long long A = units;
  *fused = units * (long long)*S + min_append <= resident;
  if (*fused) {
    A = resident - units * (long long)*S;
    if (A > units) A = units;
  } else if (num_splits == 0) {
    const long long s_res = resident / units - 1;
    if (s_res >= 1 && 2 * s_res >= *S && units * (1 + s_res) <= step_residency(cfg, after, (int32_t)s_res)) {
      *S = (int32_t)s_res;
      *fused = true;
      A = units;
    }
  }
  if (append_ctas) *append_ctas = (int32_t)A;
}

}  // namespace

extern "C" {

omnikv_status omnikv_test_decode_pending(const omnikv_config* cfg, const omnikv_cache* cache, const void* q,
                                         void* partials, int32_t num_splits, uint64_t flag_wait_ns, void* stream) {
  omnikv_status st = check_config(cfg);
  if (st != OMNIKV_OK) return st;
  if ((st = check_cache(cache)) != OMNIKV_OK) return st;
  if (!cache->step_flags || !aligned(cache->step_flags, 4)) return OMNIKV_ERR_INVALID_ARG;
  if ((long long)cache->max_seq_len + 1 > cache->cap_tokens) return OMNIKV_ERR_CAPACITY;
  omnikv_cache after = *cache;  // the decode reads the cache as if the token were appended
  after.max_seq_len += 1;
  DecodeParams dp;
  if ((st = prepare_decode(cfg, &after, q, partials, num_splits, &dp)) != OMNIKV_OK) return st;
  dp.len_add = 1;
  dp.step_flags = cache->step_flags;
  dp.flag_wait_ns = flag_wait_ns;
  if (launch_decode(dp, cache->batch, static_cast<cudaStream_t>(stream)) != cudaSuccess) return OMNIKV_ERR_CUDA;
  return OMNIKV_OK;
}

int32_t omnikv_step_splits(const omnikv_config* cfg, const omnikv_cache* cache, int32_t num_splits, int32_t* fused) {
  if (check_config(cfg) != OMNIKV_OK || check_cache(cache) != OMNIKV_OK || num_splits < 0) return 0;
  omnikv_cache after = *cache;
  after.max_seq_len = cache->max_seq_len < cache->cap_tokens ? cache->max_seq_len + 1 : cache->max_seq_len;
  int32_t S;
  bool f;
  plan_step(cfg, &after, num_splits, &S, &f);
  if (fused) *fused = f ? 1 : 0;
  return S;
}

omnikv_status omnikv_append_decode(const omnikv_config* cfg, omnikv_cache* cache, const void* q, const void* k_new,
                                   const void* v_new, const uint8_t* modality_new, void* partials,
                                   int32_t num_splits, void* stream) {
  omnikv_status st = check_config(cfg);
  if (st != OMNIKV_OK) return st;
  if ((st = check_cache(cache)) != OMNIKV_OK) return st;
  if (!cache->step_flags || !q || !k_new || !v_new || !modality_new || !partials || num_splits < 0)
    return OMNIKV_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(cache->step_flags, 4)) return OMNIKV_ERR_INVALID_ARG;
  if ((long long)cache->max_seq_len + 1 > cache->cap_tokens) return OMNIKV_ERR_CAPACITY;
  omnikv_cache after = *cache;  // the decode sees the appended token
  after.max_seq_len += 1;
  int32_t S, A;
  bool fused;
  plan_step(cfg, &after, num_splits, &S, &fused, &A);
  DecodeParams dp;
  if ((st = prepare_decode(cfg, &after, q, partials, S, &dp)) != OMNIKV_OK) return st;
  WriteParams wp;
  fill_write_params(cfg, cache, k_new, v_new, modality_new, 1, &wp);
  wp.step_flags = cache->step_flags;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (fused) {
    dp.len_add = 1;
    dp.step_flags = cache->step_flags;
    dp.append_ctas = A;
    if (launch_decode_step(dp, wp, s) != cudaSuccess) return OMNIKV_ERR_CUDA;
  } else {
    if (launch_write(wp, cache->batch, s) != cudaSuccess) return OMNIKV_ERR_CUDA;
    if (launch_decode(dp, cache->batch, s) != cudaSuccess) return OMNIKV_ERR_CUDA;
  }
  cache->max_seq_len += 1;
  return OMNIKV_OK;
}

omnikv_status omnikv_combine_step(const omnikv_config* cfg, omnikv_cache* cache, const void* partials,
                                  int32_t num_splits, float* out, void* stream) {
  omnikv_status st = check_config(cfg);
  if (st != OMNIKV_OK) return st;
  if ((st = check_cache(cache)) != OMNIKV_OK) return st;
  if (!partials || !out || num_splits < 0) return OMNIKV_ERR_INVALID_ARG;
  int32_t S;
  bool fused;
  plan_step(cfg, cache, num_splits, &S, &fused);  // the same plan as omnikv_append_decode made
  CombineParams cp;
  if ((st = prepare_combine(cfg, cache, partials, S, out, &cp)) != OMNIKV_OK) return st;
  cp.len_add = fused ? 1 : 0;  // the fused append leaves the length to this launch
  if (launch_combine(cp, cache->batch, static_cast<cudaStream_t>(stream)) != cudaSuccess) return OMNIKV_ERR_CUDA;
  return OMNIKV_OK;
}

omnikv_status omnikv_decode_step(const omnikv_config* cfg, omnikv_cache* cache, const void* q, const void* k_new,
                                 const void* v_new, const uint8_t* modality_new, void* partials, int32_t num_splits,
                                 float* out, void* stream) {
  if (!out) return OMNIKV_ERR_INVALID_ARG;
  omnikv_status st = omnikv_append_decode(cfg, cache, q, k_new, v_new, modality_new, partials, num_splits, stream);
  if (st != OMNIKV_OK) return st;
  return omnikv_combine_step(cfg, cache, partials, num_splits, out, stream);
}

size_t omnikv_dense_partials_bytes(int32_t batch, int32_t num_q_heads, int32_t num_splits) {
  if (batch < 1 || num_q_heads < 1 || num_splits < 1) return 0;
  return (size_t)batch * num_q_heads * num_splits * kDensePartialFloats * sizeof(float);
}

omnikv_status omnikv_dense_decode_bf16(const void* k_cache, const void* v_cache, const int32_t* seq_lens, int32_t batch,
                                       int32_t num_q_heads, int32_t num_kv_heads, int32_t cap_tokens,
                                       int32_t max_seq_len, const void* q, void* partials, int32_t num_splits,
                                       float* out, int32_t* error_word, void* stream) {
  if (!k_cache || !v_cache || !seq_lens || !q || !partials || !out) return OMNIKV_ERR_INVALID_ARG;
  if (batch < 1 || num_kv_heads < 1 || num_q_heads < 1 || num_q_heads % num_kv_heads) return OMNIKV_ERR_INVALID_ARG;
  if (num_q_heads / num_kv_heads > kMaxGroup) return OMNIKV_ERR_UNSUPPORTED;
  if (cap_tokens < 1 || max_seq_len < 0 || max_seq_len > cap_tokens || num_splits < 0) return OMNIKV_ERR_INVALID_ARG;
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(q, 4) || !aligned(partials, 16) || !aligned(out, 16))
    return OMNIKV_ERR_INVALID_ARG;
  DenseParams p;
  p.k = static_cast<const __nv_bfloat16*>(k_cache);
  p.v = static_cast<const __nv_bfloat16*>(v_cache);
  p.seq_lens = seq_lens;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.partials = static_cast<float*>(partials);
  p.out = out;
  p.error_word = error_word;
  p.num_kv_heads = num_kv_heads;
  p.group = num_q_heads / num_kv_heads;
  p.cap_tokens = cap_tokens;
  const int nc = (max_seq_len + 31) / 32;
  int S = num_splits;
  if (S == 0) {
    const long long units = (long long)batch * num_kv_heads;
    long long s = sm_count() / units;
    if (s > (nc + 7) / 8) s = (nc + 7) / 8;
    S = (int)(s < 1 ? 1 : s);
  }
  if (S > kMaxSplits) return OMNIKV_ERR_UNSUPPORTED;
  p.num_splits = S;
  p.split_chunks = nc > 0 ? (nc + S - 1) / S : 1;
  if (launch_dense(p, batch, static_cast<cudaStream_t>(stream)) != cudaSuccess) return OMNIKV_ERR_CUDA;
  return OMNIKV_OK;
}

omnikv_status omnikv_stream_write_cache(const omnikv_config* cfg, omnikv_cache* cache, void* ring_k, void* ring_v,
                                        const void* k_new, const void* v_new, const uint8_t* modality_new,
                                        int32_t n_new, void* stream) {
  omnikv_status st = check_config(cfg);
  if (st != OMNIKV_OK) return st;
  if ((st = check_cache(cache)) != OMNIKV_OK) return st;
  if (n_new < 1 || !k_new || !v_new || !modality_new || !ring_k || !ring_v) return OMNIKV_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(ring_k, 16) || !aligned(ring_v, 16))
    return OMNIKV_ERR_INVALID_ARG;
  if ((long long)cache->max_seq_len + n_new > cache->cap_tokens) return OMNIKV_ERR_CAPACITY;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the raw inputs into their ring slots first (positions from the lengths before the write)
  if (launch_stream_push(static_cast<const __half*>(k_new), static_cast<const __half*>(v_new), cache->seq_lens,
                         static_cast<__half*>(ring_k), static_cast<__half*>(ring_v), cache->batch, cfg->num_kv_heads,
                         n_new, s) != cudaSuccess)
    return OMNIKV_ERR_CUDA;
  return omnikv_write_cache(cfg, cache, k_new, v_new, modality_new, n_new, stream);
}

omnikv_status omnikv_stream_decode(const omnikv_config* cfg, const omnikv_cache* cache, const void* ring_k,
                                   const void* ring_v, const void* q, void* partials, int32_t num_splits, float* out,
                                   void* stream) {
  if (!ring_k || !ring_v || !out) return OMNIKV_ERR_INVALID_ARG;
  if (!aligned(ring_k, 16) || !aligned(ring_v, 16) || !aligned(out, 16)) return OMNIKV_ERR_INVALID_ARG;
  DecodeParams dp;
  omnikv_status st = prepare_decode(cfg, cache, q, partials, num_splits, &dp);
  if (st != OMNIKV_OK) return st;
  // body splits 0 .. S-1, tail splits S .. S+3 (the body's empty splits there are overwritten)
  const int S = dp.num_splits;
  if (S + kStreamTailSplits > kMaxSplits) return OMNIKV_ERR_UNSUPPORTED;
  dp.num_splits = S + kStreamTailSplits;  // partials stride
  dp.stream = 1;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (launch_decode(dp, cache->batch, s) != cudaSuccess) return OMNIKV_ERR_CUDA;
  if (launch_stream_tail(dp, static_cast<const __half*>(ring_k), static_cast<const __half*>(ring_v), S, s) !=
      cudaSuccess)
    return OMNIKV_ERR_CUDA;
  CombineParams cp;
  if ((st = prepare_combine(cfg, cache, partials, S + kStreamTailSplits, out, &cp)) != OMNIKV_OK) return st;
  if (launch_combine(cp, cache->batch, s) != cudaSuccess) return OMNIKV_ERR_CUDA;
  return OMNIKV_OK;
}

size_t omnikv_calibrate_workspace_bytes(int32_t num_tokens) { return calibrate_workspace_bytes(num_tokens); }

omnikv_status omnikv_calibrate_bases(const void* values, const uint8_t* modality, const float* weights,
                                     int32_t num_tokens, void* workspace, size_t workspace_bytes, float* bases,
                                     double* eigenvalues, void* stream) {
  if (!values || !modality || !weights || !workspace || !bases || num_tokens < 1) return OMNIKV_ERR_INVALID_ARG;
  if (!aligned(values, 16) || !aligned(weights, 4) || !aligned(workspace, 16) || !aligned(bases, 4) ||
      (eigenvalues && !aligned(eigenvalues, 8)))
    return OMNIKV_ERR_INVALID_ARG;
  if (workspace_bytes < calibrate_workspace_bytes(num_tokens)) return OMNIKV_ERR_CAPACITY;
  if (launch_calibrate(static_cast<const __half*>(values), modality, weights, num_tokens, workspace, bases, eigenvalues,
                       static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return OMNIKV_ERR_CUDA;
  return OMNIKV_OK;
}

const char* omnikv_status_string(omnikv_status s) {
  switch (s) {
    case OMNIKV_OK: return "ok";
    case OMNIKV_ERR_INVALID_ARG: return "invalid argument";
    case OMNIKV_ERR_UNSUPPORTED: return "unsupported configuration";
    case OMNIKV_ERR_CAPACITY: return "cache capacity exceeded";
    case OMNIKV_ERR_CUDA: return "CUDA launch failed";
    case OMNIKV_ERR_DEVICE_CHECK: return "device-side check failed";
  }
  return "unknown status";
}

int32_t omnikv_abi_version(void) { return OMNIKV_ABI_VERSION; }

}  // extern "C"
