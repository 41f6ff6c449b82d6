/*
 * omnikv.h -- C ABI of the OmniKVQuant 2-bit KV-cache write and fused decode
 * attention for NVIDIA B200 (sm_100a).
 *
 * Method: "OmniKVQuant: KV Cache Quantization for Omni-LLMs" (arXiv:2609.11582).
 *   - keys: sign-flip Hadamard rotation (the TurboQuant rotation kept for keys,
 *     paperpeel.com section 2.2 "Temporal key drift"), then a per-channel
 *     min-max range over each 32-token group (section 3.1 "Implementation
 *     details"), stored as fp16 minimum m_gc and scale s_gc (section 3.3 "Error
 *     comparison"), mapped onto a fixed codebook (pchao.org "方法概览").
 *   - values: rotated with the orthogonal basis U_m of the token's modality
 *     m in {V, A, L} (section 2.3 "Modality-aware value rotation"), then coded
 *     on the same kind of fixed codebook with one fp16 scale per token.
 *   - decode: the query is rotated once per head instead of inverse-rotating
 *     every cached key, the 2-bit cache is unpacked inside attention in
 *     FlashAttention order, and the inverse value rotations are batched across
 *     head outputs, so no dense fp16 cache is built (section 1, last paragraph;
 *     abstract on arxiv / thelatestinai.com).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, except the
 *     configuration and cache structs themselves, which live in host memory.
 *     The library allocates nothing, frees nothing and never synchronises the
 *     device. It keeps no global state, with one exception: omnikv_decode_static
 *     (below) keeps its split partials in a fixed device array of the library.
 *   - `stream` is a cudaStream_t (passed as void*); NULL means the legacy
 *     default stream. All work is stream-ordered on it.
 *   - Host-side validation runs before any launch; a failed check returns an
 *     error status and launches nothing. A launch failure returns
 *     OMNIKV_ERR_CUDA. Conditions only the device can see (a sequence whose
 *     length would pass cap_tokens) skip that sequence's work and set a bit in
 *     the optional device error word (see omnikv_cache.error_word); they never
 *     fault.
 *   - fp16 tensors are IEEE binary16 (passed as void*), row-major, contiguous.
 *
 * Window record (one per sequence, kv head and 32-token window; all fields
 * little-endian; bits = key_bits or value_bits; cpw = 32 / bits codes per u32):
 *   K codes [32 tokens][128 / cpw] u32  token-major: channel c of token t is
 *           in word (t, c / cpw) at bits [bits * (c % cpw), +bits)
 *   meta    key metadata of the window, in the config's key_meta_format:
 *           OMNIKV_META_FP16 (512 B): [128] { fp16 m_gc, fp16 s_gc };
 *           OMNIKV_META_MXFP4 (144 B; the pages' default metadata, section 3.1):
 *           E2M1 codes (sign << 3 | magnitude index, magnitudes 0, 0.5, 1, 1.5,
 *           2, 3, 4, 6) of the 128 minima, two per byte (even channel in the low
 *           nibble), then of the 128 scales; then the E8M0 exponents (e + 127) of
 *           the 4 blocks of 32 channels of the minima, then of the scales; 8 zero
 *           bytes. m_gc = E2M1(m code) 2^e_m, s_gc = E2M1(s code) 2^e_s;
 *           OMNIKV_META_TURBO (64 B; the TurboQuant key codec the pages compare
 *           against, pchao.org related work / paperpeel.com section 2.2): [32]
 *           fp16 key scales, one per token (0 for padded slots).
 *   V codes [32 / cpw][128] u32         channel-major: token t, channel c is in
 *           word (t / cpw, c) at bits [bits * (t % cpw), +bits)
 *   sigma   [32] fp16 (per-token value scale)
 * Size (omnikv_record_bytes_meta): 2624 bytes for K2/V2 and 4672 for K4/V4 with
 * fp16 metadata; 2256 and 4304 with MXFP4 metadata; 2176 and 4224 with TurboQuant
 * keys.
 * Dequantised rotated-space cache: k'_tc = m_gc + s_gc (c_j - c_0) for key code
 * j (window metadata) or k'_tc = ksigma_t c_j (TurboQuant keys); v'_tc = sigma_t
 * c_j for value code j. Padded slots of a partial window hold code 0 and sigma 0.
 */
#ifndef OMNIKV_H_
#define OMNIKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define OMNIKV_API __attribute__((visibility("default")))
#else
#define OMNIKV_API
#endif

#define OMNIKV_ABI_VERSION 3
#define OMNIKV_HEAD_DIM 128
#define OMNIKV_WINDOW 32
#define OMNIKV_NUM_MODALITIES 3 /* 0 = text (L), 1 = audio (A), 2 = video (V) */
#define OMNIKV_META_FP16 0      /* key window metadata: fp16 minimum and scale per channel */
#define OMNIKV_META_MXFP4 1     /* key window metadata: MXFP4 (E2M1 values, one E8M0 exponent per 32 channels) */
#define OMNIKV_META_TURBO 2     /* TurboQuant key codec: one fp16 scale per token, no window statistics */

typedef enum {
  OMNIKV_OK = 0,
  OMNIKV_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer */
  OMNIKV_ERR_UNSUPPORTED = 2,  /* head_dim != 128, window != 32, bits not 2/4, GQA group > 8 */
  OMNIKV_ERR_CAPACITY = 3,     /* max_seq_len + n_new > cap_tokens */
  OMNIKV_ERR_CUDA = 4,         /* a CUDA launch failed (cudaGetLastError) */
  OMNIKV_ERR_DEVICE_CHECK = 5  /* reserved for device-side checks read back by the caller */
} omnikv_status;

/* Device error word bits (omnikv_cache.error_word). */
#define OMNIKV_DEVERR_CAPACITY 0x1 /* a write would have passed cap_tokens; that sequence was skipped */
#define OMNIKV_DEVERR_MODALITY 0x2 /* a modality id was > 2; it was stored and used as 2 (video) */
#define OMNIKV_DEVERR_BOUND 0x8    /* a sequence was longer than cache->max_seq_len promised; windows past
                                      num_splits * ceil(ceil(max_seq_len / 32) / num_splits) were skipped */
#define OMNIKV_DEVERR_TIMEOUT 0x4  /* a staged copy did not complete within its wait limit; outputs of that
                                      CTA are zero (never expected; the kernel returns instead of hanging) */
#define OMNIKV_DEVERR_RANGE 0x10   /* a decode split produced a non-finite partial and was written empty
                                      (weight 0 in the combine): inputs outside the range of the fp16
                                      tensor-core operands of 2-bit decoding -- key window scales s_gc
                                      above 32752, value scales sigma of 565 or more -- or non-finite
                                      queries or cache entries. Queries of any finite size are supported. */

/* Per-layer constants. All pointers are device pointers. */
typedef struct {
  int32_t head_dim;             /* must be 128 */
  int32_t num_q_heads;          /* multiple of num_kv_heads; group size G = num_q_heads / num_kv_heads in 1..8 */
  int32_t num_kv_heads;         /* >= 1 */
  int32_t window;               /* must be 32 (the 32-token group g of section 3.1) */
  int32_t key_bits;             /* 2 or 4 */
  int32_t value_bits;           /* 2 or 4 */
  const float* key_codebook;    /* [2^key_bits] fp32, strictly ascending (fixed codebook) */
  const float* value_codebook;  /* [2^value_bits] fp32, strictly ascending */
  const float* key_signs;       /* [128] fp32, each +1 or -1 (sign flip before the Hadamard transform) */
  const float* value_rot;       /* [num_kv_heads][3][128][128] fp32: U_m row-major, its COLUMNS are the
                                   basis: v' = U_m^T v, v = U_m v'. Must be orthogonal. */
  int32_t key_meta_format;      /* OMNIKV_META_FP16 (0) or OMNIKV_META_MXFP4 (1): how a window's key minima and
                                   scales are stored (section 3.1 "Implementation details": MXFP4 by default;
                                   section 3.3: fp16). With MXFP4, per block of 32 channels the shared exponent
                                   is the smallest e in [-127, 127] with max |x| <= 6 2^e (-127 for a zero
                                   block); the minimum rounds to the nearest E2M1 value times 2^e (ties to the
                                   even code), then the scale it needs, fp32((max - m^) / (c_last - c_0)) (0 if
                                   negative), on its block's grid the same way. Codes as with fp16 metadata.
                                   OMNIKV_META_TURBO (2): the TurboQuant key codec, per token: ksigma =
                                   fp16(sqrt(sum_c k_c^2 / 128)) of the unrotated fp16 key (the value scale's
                                   rule) and code = #{j : k'_c / ksigma > t_j} (0 where ksigma == 0); the
                                   values are unchanged (TurboQuant proper passes the transposed key rotation
                                   R^T as every modality's value basis: one shared rotation). */
} omnikv_config;

/* One layer's cache for a batch. Device memory is owned by the caller and must be
 * zero-filled before the first write (records, modality, seq_lens). A view of
 * one sequence (batch = 1, pointers advanced by its index) is itself a valid cache. */
typedef struct {
  void* records;        /* [batch][num_kv_heads][cap_tokens / 32] window records, 16-byte aligned */
  void* key_tail;       /* [batch][num_kv_heads][32][128] fp16: raw keys of each partial last window */
  uint8_t* modality;    /* [batch][cap_tokens] modality id of every cached token */
  int32_t* seq_lens;    /* [batch] tokens cached per sequence; advanced by omnikv_write_cache */
  int32_t* error_word;  /* optional [1] int32: OMNIKV_DEVERR_* bits are OR-ed in; may be NULL */
  int32_t batch;        /* >= 1 */
  int32_t cap_tokens;   /* capacity per sequence, a positive multiple of 32 */
  int32_t max_seq_len;  /* HOST-side upper bound on every seq_lens[b]; sizes grids and checks capacity.
                           omnikv_write_cache adds n_new to it on success. */
  int32_t* step_flags;  /* optional [batch][num_kv_heads] int32, zero-filled with the cache; used (and
                           required) only by omnikv_decode_step, which stores the new length there once
                           the appended token's window record is written; may be NULL otherwise */
} omnikv_cache;

/* Bytes of one window record with fp16 key metadata: 2624 for K2/V2, 4672 for K4/V4; 0 for
 * unsupported bits. */
OMNIKV_API size_t omnikv_record_bytes(int32_t key_bits, int32_t value_bits);

/* Bytes of one window record in a key metadata format (OMNIKV_META_FP16: as omnikv_record_bytes;
 * OMNIKV_META_MXFP4: 2256 for K2/V2, 4304 for K4/V4; OMNIKV_META_TURBO: 2176 for K2/V2, 4224 for
 * K4/V4); 0 for unsupported arguments. The cache's
 * records array holds [batch][num_kv_heads][cap_tokens / 32] records of this size. */
OMNIKV_API size_t omnikv_record_bytes_meta(int32_t key_bits, int32_t value_bits, int32_t key_meta_format);

/* Bytes of the split-K partials buffer for omnikv_decode_attention / omnikv_combine:
 * [batch][num_q_heads][num_splits] entries of { fp32 acc[3][128], fp32 m, fp32 l, 2 x fp32 padding }
 * (1552 B each, 16-byte aligned). num_splits is at most 4096 (OMNIKV_ERR_UNSUPPORTED above). */
OMNIKV_API size_t omnikv_partials_bytes(int32_t batch, int32_t num_q_heads, int32_t num_splits);

/* The split count used when omnikv_decode_attention is given num_splits = 0 (depends on the
 * batch, the kv heads, max_seq_len, the bit widths and the device's SM count): one wave of resident
 * decode CTAs over batch x kv heads, at most one split per 4 windows, at least 8 splits for large
 * batches. The decode kernel body depends on the split length (2-bit caches: splits of at most 16
 * windows run a body with more resident CTAs per SM), and the wave is sized for that body.
 * Returns >= 1, or 0 on bad arguments. */
OMNIKV_API int32_t omnikv_default_splits(const omnikv_config* cfg, const omnikv_cache* cache);

/* Cache write (kv_quant_pack). Appends n_new tokens to EVERY sequence of the batch, at position
 * seq_lens[b] (read on the device), then advances seq_lens[b] and cache->max_seq_len by n_new.
 *   k_new, v_new : [batch][num_kv_heads][n_new][128] fp16, 16-byte aligned
 *   modality_new : [batch][n_new] u8, each 0, 1 or 2 (larger ids: OMNIKV_DEVERR_MODALITY)
 * Keys: every 32-token window touched by the new positions is (re)quantised over all its valid
 * tokens: rotation k' = fp32(2^-3.5) H (s . k) (butterflies h = 1..64, fp32), per-channel
 * m = fp16(min), s = fp16((max - min) / (c_last - c_0)), code = #{j : (k' - m) / s + c_0 > t_j},
 * t_j = fp32((c_j + c_{j+1}) * 0.5), code 0 where s == 0. A window left partial keeps its raw keys in
 * key_tail. Values: sigma = fp16(sqrt(pairwise-tree sum of v_c^2 / 128)) of the unrotated fp16 value,
 * v' = U_m^T v (windows the write fills completely: tcgen05 tensor cores, fp16 values times U split into
 * fp16 high + low parts, fp32 accumulation; other tokens: fp32 FMA), code = #{j : v'_c / sigma > t_j},
 * 0 where sigma == 0.
 * Key codes and metadata are bit-exact with a scalar fp32 evaluation in this order; value codes
 * depend on the fp32-accumulated rotation and may differ from an fp64 rotation only where v'/sigma
 * lies within rounding of a threshold.
 * Errors: OMNIKV_ERR_CAPACITY if cache->max_seq_len + n_new > cap_tokens (nothing launched);
 * OMNIKV_ERR_INVALID_ARG for n_new < 1 or a null / misaligned pointer. */
OMNIKV_API omnikv_status omnikv_write_cache(const omnikv_config* cfg, omnikv_cache* cache,
                                 const void* k_new, const void* v_new, const uint8_t* modality_new,
                                 int32_t n_new, void* stream);

/* omnikv_write_cache that also returns the rotated values v' = U_m^T v the kernels computed for the
 * written tokens (section 2.3 "Modality-aware value rotation"; the value codes are decided from exactly
 * these fp32 numbers), so a caller can check the value codes against v' / sigma bit for bit and v' against
 * an exact rotation. Arguments as omnikv_write_cache, plus
 *   v_rot : [batch][num_kv_heads][n_new][128] fp32, 16-byte aligned; every entry is written.
 * Slower than omnikv_write_cache (an extra 512 B written per token and kv head); meant for tests. */
OMNIKV_API omnikv_status omnikv_write_cache_rotations(const omnikv_config* cfg, omnikv_cache* cache,
                                                      const void* k_new, const void* v_new,
                                                      const uint8_t* modality_new, int32_t n_new, float* v_rot,
                                                      void* stream);

/* Fused split-K decode attention over the packed cache (decode_split_k). For every sequence b,
 * query head i (kv head i / G) and split s, over the windows [s C, min((s+1) C, W)) of the
 * W = ceil(seq_lens[b] / 32) windows, C = ceil(ceil(cache->max_seq_len / 32) / S):
 * q' = fp32(2^-3.5) H (s . q_i); score_t = q' . k'_t /
 * sqrt(128); a running max m and sum l of exp(score - m), and one rotated-space accumulator per
 * modality acc_m = sum_{t of modality m} exp(score_t - m) v'_t. Written to `partials`.
 *   q          : [batch][num_q_heads][128] fp16, 16-byte aligned
 *   partials   : device buffer of omnikv_partials_bytes(batch, num_q_heads, S) bytes, 16-byte aligned
 *   num_splits : 1 <= S <= 4096, or 0 for omnikv_default_splits(cfg, cache)
 * Empty splits write m = -inf and l = 0 only (their accumulators are not written; the combine gives
 * them weight 0). */
OMNIKV_API omnikv_status omnikv_decode_attention(const omnikv_config* cfg, const omnikv_cache* cache,
                                      const void* q, void* partials, int32_t num_splits, void* stream);

/* Split-K combine and batched inverse value rotation (combine_inverse_rotate):
 * M = max_s m_s, l = sum_s l_s e^(m_s - M), acc_m = sum_s acc_{s,m} e^(m_s - M),
 * out = sum_m U_m acc_m / l (fp32). A sequence with no tokens yields zeros.
 *   partials   : as written by omnikv_decode_attention with the same num_splits (0 resolves the same way)
 *   out        : [batch][num_q_heads][128] fp32 */
OMNIKV_API omnikv_status omnikv_combine(const omnikv_config* cfg, const omnikv_cache* cache,
                             const void* partials, int32_t num_splits, float* out, void* stream);

/* One decode step: append ONE token to every sequence (as omnikv_write_cache with n_new = 1), then
 * decode attention over the cache including it and combine (as omnikv_decode_attention +
 * omnikv_combine), in two launches instead of four: the append runs in CTAs of the decode launch,
 * concurrently with the decode of the other windows; only the warp that decodes a sequence's last
 * window waits (bounded, OMNIKV_DEVERR_TIMEOUT on expiry) until cache->step_flags[b][h] holds the
 * new length, and the combine launch advances seq_lens[b]. Results are identical to the four calls.
 *   q                     : [batch][num_q_heads][128] fp16 (the step's queries)
 *   k_new, v_new          : [batch][num_kv_heads][1][128] fp16; modality_new: [batch] u8
 *   partials, num_splits  : as for omnikv_decode_attention (num_splits = 0: the default, lowered if
 *                           needed so that every CTA of the launch is resident at once)
 *   out                   : [batch][num_q_heads][128] fp32
 * Requires cache->step_flags (OMNIKV_ERR_INVALID_ARG without it);
 * OMNIKV_ERR_CAPACITY if cache->max_seq_len + 1 > cap_tokens; advances cache->max_seq_len by 1. */
OMNIKV_API omnikv_status omnikv_decode_step(const omnikv_config* cfg, omnikv_cache* cache, const void* q,
                                            const void* k_new, const void* v_new, const uint8_t* modality_new,
                                            void* partials, int32_t num_splits, float* out, void* stream);

/* The split count the next omnikv_decode_step (or omnikv_append_decode) uses with this num_splits
 * (0: default) for the cache as it is now (partials must hold that many splits), and in *fused whether
 * its append runs inside the decode launch (1; 2 launches per step) or before it (0; 3 launches).
 * Returns 0 on bad arguments. */
OMNIKV_API int32_t omnikv_step_splits(const omnikv_config* cfg, const omnikv_cache* cache, int32_t num_splits,
                                      int32_t* fused);

/* The two launches of omnikv_decode_step as separate calls (omnikv_decode_step = this pair), e.g. to
 * time them apart or to schedule other work between them. omnikv_append_decode appends the token and
 * writes the split partials (arguments as above) and advances cache->max_seq_len by 1;
 * omnikv_combine_step must follow it on the same stream with the same cache, partials and
 * num_splits: it merges them into out and advances seq_lens where the append left that to it. */
OMNIKV_API omnikv_status omnikv_append_decode(const omnikv_config* cfg, omnikv_cache* cache, const void* q,
                                              const void* k_new, const void* v_new, const uint8_t* modality_new,
                                              void* partials, int32_t num_splits, void* stream);
OMNIKV_API omnikv_status omnikv_combine_step(const omnikv_config* cfg, omnikv_cache* cache, const void* partials,
                                             int32_t num_splits, float* out, void* stream);

/* Decode attention and combine in one call, with the split-K partials in a fixed device array of
 * OMNIKV_DECODE_STATIC_SCRATCH_BYTES owned by this library; the caller passes only inputs (q) and
 * outputs (out), as for omnikv_decode_attention + omnikv_combine, and nothing is allocated.
 * The paper has no counterpart: this entry point serves callers that cannot allocate device memory
 * while decoding -- engines that reserved nearly all device memory for their own pool at start-up
 * (a further cudaMalloc fails or fragments it), plug-ins whose host framework owns every allocation,
 * and latency-critical loops that cannot pay for cudaMalloc / cudaFree, which may synchronise the
 * device.
 *   q, out, num_splits : as for omnikv_decode_attention / omnikv_combine; num_splits = 0 takes the
 *                        default, lowered until batch * num_q_heads * num_splits partials (1552 B each)
 *                        fit in the array
 * Errors: OMNIKV_ERR_CAPACITY if the partials do not fit (an explicit num_splits too large, or
 * batch * num_q_heads above 5405); OMNIKV_ERR_CUDA if the array's device address cannot be obtained.
 * Every GPU that loads the library holds the array until the process exits. Its device address is
 * looked up (cudaGetSymbolAddress) by the first call made on each device, and again by the first
 * call made in a new context of that device (after cudaDeviceReset, for example); make that first
 * call before any stream capture. All calls share the array, which keeps the last call's contents (no
 * part of it needs to start at zero); calls that overlap on the GPU race on it, so run them on one
 * stream or otherwise ordered. */
#define OMNIKV_DECODE_STATIC_SCRATCH_BYTES (8u << 20)
OMNIKV_API omnikv_status omnikv_decode_static(const omnikv_config* cfg, const omnikv_cache* cache, const void* q,
                                              float* out, int32_t num_splits, void* stream);

/* Dense bf16 split-K decode attention over an unquantised cache: the comparison baseline for the
 * packed kernels (the same attention read at 512 B per token and kv head). Not part of the method.
 *   k_cache, v_cache : [batch][num_kv_heads][cap_tokens][128] bf16, 16-byte aligned
 *   seq_lens         : [batch] device; max_seq_len a host bound on them
 *   q                : [batch][num_q_heads][128] bf16; scores q.k / sqrt(128)
 *   partials         : device buffer of omnikv_dense_partials_bytes(batch, num_q_heads, S) bytes
 *   num_splits       : S >= 1, or 0 for a default; out: [batch][num_q_heads][128] fp32
 *   error_word       : optional device int32 (OMNIKV_DEVERR_TIMEOUT) */
OMNIKV_API size_t omnikv_dense_partials_bytes(int32_t batch, int32_t num_q_heads, int32_t num_splits);
OMNIKV_API omnikv_status omnikv_dense_decode_bf16(const void* k_cache, const void* v_cache, const int32_t* seq_lens,
                                                  int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                                  int32_t cap_tokens, int32_t max_seq_len, const void* q,
                                                  void* partials, int32_t num_splits, float* out,
                                                  int32_t* error_word, void* stream);

/* Streaming / captioning cache policy (paperpeel.com section 3.1, "Implementation details": keys are
 * quantised every 128 tokens in groups of 32, values keep a 128-token fp16 sliding window before
 * quantisation). With T tokens cached, the decode reads the keys of positions [0, KB) quantised,
 * KB = 128 floor(T / 128) (blocks aligned at absolute positions), and the values of positions
 * [0, VB) quantised, VB = max(0, T - 128); every other key and value enters attention as its raw
 * fp16 input (original basis). Records are written for every token as by omnikv_write_cache (a
 * quantised entry is exactly the ordinary write's); the raw inputs of the newest 256 positions are
 * kept in caller-owned rings:
 *   ring_k, ring_v : [batch][num_kv_heads][256][128] fp16 each, 16-byte aligned; position p of a
 *                    sequence in slot p mod 256 (no initialisation needed).
 * omnikv_stream_write_cache: omnikv_write_cache plus the copy of the last min(n_new, 256) tokens of
 *   the write into the rings (at the positions the write gives them); the same arguments and errors.
 * omnikv_stream_decode: decode + combine under the policy, three stream-ordered launches: the
 *   ordinary decode over the windows before 32 floor(VB / 32) (splits 0 .. S-1), a tail kernel over
 *   the remaining (at most 159) positions in 4 chunks (splits S .. S+3; its raw values' sums are
 *   carried in modality 0's rotated basis), and the combine over S + 4 splits.
 *   num_splits: S, or 0 for omnikv_default_splits; partials: omnikv_partials_bytes(batch,
 *   num_q_heads, S + OMNIKV_STREAM_TAIL_SPLITS) bytes; out: [batch][num_q_heads][128] fp32. Errors as
 *   omnikv_decode_attention and omnikv_combine. */
#define OMNIKV_STREAM_TAIL_SPLITS 4
OMNIKV_API omnikv_status omnikv_stream_write_cache(const omnikv_config* cfg, omnikv_cache* cache, void* ring_k,
                                                   void* ring_v, const void* k_new, const void* v_new,
                                                   const uint8_t* modality_new, int32_t n_new, void* stream);
OMNIKV_API omnikv_status omnikv_stream_decode(const omnikv_config* cfg, const omnikv_cache* cache,
                                              const void* ring_k, const void* ring_v, const void* q, void* partials,
                                              int32_t num_splits, float* out, void* stream);

/* Calibration of the per-modality value bases U_m of one (layer, kv head) from calibration values
 * (paperpeel.com section 2.3 "Modality-aware value rotation": one basis per modality, calibrated
 * once per model on calibration clips, section 3.1; pchao.org 方法概览: an attention-contribution-
 * weighted covariance per modality and its eigendecomposition). For each modality m (ids 0, 1, 2;
 * tokens with another id, or with a weight that is not positive, are ignored):
 *   C_m = sum_t a_t (v_t - mu_m)(v_t - mu_m)^T / sum_t a_t, mu_m = sum_t a_t v_t / sum_t a_t (fp64);
 *   E_m = the eigenvectors of C_m as columns, eigenvalues descending, each column's entry of
 *         largest magnitude positive (the first on ties);
 *   U_m = E_m H, H = 2^-3.5 H_128 (Sylvester; "a modality-aware correction of the Hadamard
 *         rotation", paperpeel.com section 2.2); a modality without weight gets U_m = H.
 *   values     : [num_tokens][128] fp16, device, 16-byte aligned
 *   modality   : [num_tokens] u8, device;  weights: [num_tokens] fp32 a_t, device
 *   workspace  : device scratch of at least omnikv_calibrate_workspace_bytes(num_tokens) bytes,
 *                16-byte aligned, owned by the caller (contents undefined afterwards)
 *   bases      : [3][128][128] fp32 out, device: U_m row-major, columns the basis (the layout of
 *                omnikv_config.value_rot for one kv head)
 *   eigenvalues: [3][128] fp64 out, device, descending (zeros for a modality without weight), or NULL
 * Four stream-ordered launches (fp64 weighted Gram sums per token run, their reduction, a cyclic
 * parallel Jacobi eigensolver per modality with at most 40 sweeps, sorting and the product with H).
 * A modality with fewer than 129 weighted tokens has a singular covariance: its null-space
 * eigenvectors are not unique (any orthonormal basis of the null space is returned).
 * OMNIKV_ERR_INVALID_ARG: a null pointer, num_tokens < 1 or a misaligned pointer;
 * OMNIKV_ERR_CAPACITY: workspace_bytes too small; OMNIKV_ERR_CUDA: a launch failed. */
OMNIKV_API size_t omnikv_calibrate_workspace_bytes(int32_t num_tokens);
OMNIKV_API omnikv_status omnikv_calibrate_bases(const void* values, const uint8_t* modality, const float* weights,
                                                int32_t num_tokens, void* workspace, size_t workspace_bytes,
                                                float* bases, double* eigenvalues, void* stream);

/* Static text for a status code. */
OMNIKV_API const char* omnikv_status_string(omnikv_status status);

/* OMNIKV_ABI_VERSION of the loaded library. */
OMNIKV_API int32_t omnikv_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* OMNIKV_H_ */
