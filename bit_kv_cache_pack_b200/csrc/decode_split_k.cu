// decode_split_k: fused decode attention over the packed OmniKVQuant cache.
//
// paperpeel.com section 1 (last paragraph): the query is rotated once per head
// instead of inverse-rotating every cached key, the cache is unpacked inside
// attention in FlashAttention order (refs [4], [5]), and no dense fp16 cache is
// built. One CTA of 4 warps per (split of the context, kv head, sequence); all
// query heads of the kv head (the GQA group, up to 8) are served by every load
// of a window record.
//
// Tensor-core path (2-bit keys and values, symmetric codebook):
//   * scores use mma.sync m16n8k16 with the 8 query heads as N. With a
//     symmetric codebook c_j - c_0 = (c_1 - c_0) b0 + (c_2 - c_0) b1 for the
//     code's bits b0, b1, so k'_tc - m_gc = s_gc ((c_1 - c_0) b0 + (c_2 - c_0) b1).
//     The A operand (16 tokens x 16 channels) holds s_gc * 2^-7 * b0 and
//     s_gc * 2 * b1, both exact in fp16: one shift and one AND put a code bit on
//     fp16 bit 13 (2^-7) or 14 (2), and one HMUL2 by the window's fp16 scales.
//     The B operand is q'_c (c_1 - c_0) * 128 and q'_c (c_2 - c_0) / 2, split
//     into an fp16 high and low part (so the product keeps ~22 bits), built
//     once per CTA in shared memory; the window minimum enters as the per-head
//     offset sum_c q'_c m_gc;
//   * online softmax (running max with exact rescale when it grows, per-lane
//     partial sums reduced once at the end);
//   * P (times the token's value scale sigma and the plane constants, split
//     into fp16 high + low parts) becomes the B operand of the value product
//     through movmatrix; values are stored channel-major so the A operand (16
//     channels x 16 tokens) again needs one shift and one AND per register; one
//     fp32 accumulator set per modality (values of different modalities live in
//     different rotated bases); the c_0 term is c_0 * sum_t p_t sigma_t per
//     modality, added at the end.
// Two bodies run this arithmetic; the host picks by the split length:
//   * per-warp body (long splits): each warp streams its own contiguous run of
//     the split's windows through a 3-stage ring of 1-D bulk async copies (record
//     + the window's 32 modality ids) and owns all 128 channels of the value
//     product; the active modality's accumulator is in registers, the others are
//     parked in the warp's tensor-memory lanes (tcgen05.st / tcgen05.ld) with the
//     running max they were parked at; the 4 warps merge at the end (common max,
//     shared-memory reduction, one modality at a time). ~240 registers, 2 CTAs
//     per SM;
//   * cooperative body (splits of at most 16 windows): the CTA takes 4 windows
//     at a time (one 2-stage ring of group copies); warp w scores window w, the
//     CTA shares one running max, warp w writes its window's value-product B
//     operand to shared memory, and every warp then runs the value product of
//     the whole group for its own 32 channels (all three modality accumulators
//     in registers, no merge). ~168 registers, 3 CTAs per SM; the shorter
//     critical path wins when a split has few windows (decode steps at small
//     batch), the per-warp body when it streams many.
// Token order inside a 16-token tile: fragment row / k-slot r holds token
// tau(r) = r/2 + 8 (r%2) for r < 8 and 4 + (r-8)/2 + 8 (r%2) for r >= 8, so the
// two tokens of every value-operand register (k-slots 2t, 2t+1 -> tokens t,
// t+8) sit 16 bits apart in one channel-major code word.
//
// 4-bit codes (every key format): the per-warp table body, mma.sync operands
// looked up per code byte in shared-memory codeword tables.
//
// CUDA-core path (mixed bit widths, or a 2-bit codebook that is not symmetric):
// the CTA decodes a window at a time (four threads per token for the scores, a
// thread per channel for the values), built into its own kernel for mixed bit
// widths (more CTAs per SM, no tensor memory).
//
// Decode step (decode_step_kernel): the first batch x kv-head CTAs of the launch
// append one token per (sequence, kv head) and publish the new length in a flag;
// the decode CTAs read the cache at that length, and only the copy of the window
// that receives the token waits (bounded) for the flag.
//
// Launches use programmatic dependent launch: everything that does not depend on
// the cache (query rotation, score operand, L2 prefetch of the value bases for the
// combine) runs before griddepcontrol.wait.
//
// Operand range: the score operand carries a per-CTA power of two, so queries of
// any finite magnitude are exact to ~22 bits; key scales s_gc up to 32752 (the
// A operand holds s_gc * 2) and value scales sigma below 565 (the value operand
// holds p sigma (c_1 - c_0) 128 with p <= 1) stay inside fp16. Beyond them a
// split's partial is not finite: it is written empty (weight 0 in the combine) and
// OMNIKV_DEVERR_RANGE is set. Key scales below 2^-7 lose relative precision in the
// s_gc * 2^-7 plane (fp16 subnormals); realistic key ranges are far above.
#include <atomic>
#include <cstddef>

#include "decode_common.cuh"

namespace omnikv {

namespace {

constexpr int kStages = 3;                      // per-warp body: windows in flight per warp
constexpr int kRec22 = 2624;                    // K2/V2 record bytes with fp16 key metadata (the largest)
constexpr int kStageBytes = kRec22 + kWindow;   // record + modality ids

// Offsets of a K2/V2 record with key metadata format kMeta.
template <int kMeta>
struct Rec22 {
  static constexpr int meta = 1024;
  static constexpr int v = meta + meta_bytes_of(kMeta);
  static constexpr int sigma = v + 1024;
  static constexpr int bytes = sigma + 64;
};
constexpr int kCoop = kWarps;                   // cooperative body: windows per group (one per warp for the scores)
constexpr int kCoopStages = 2;                  // cooperative body: window groups in flight per CTA
constexpr int kGroupBytes = kCoop * kStageBytes;  // kCoop records, then their modality ids
constexpr uint32_t kTmemCols = 128;  // per-warp body, per CTA: 3 parked accumulators x 32 columns in each warp's lanes

struct __align__(16) DecodeSmem {
  union {
    struct {
      uint8_t stage[kWarps][kStages][kStageBytes];  // per-warp rings; also the final merge buffer
    } w;
    struct {
      uint8_t stage[kCoopStages][kGroupBytes];     // window groups
      uint4 pfrag[kCoop][2][2][32];                 // value B operand per (window, tile, plane, lane): {hi b0, hi b1, lo b0, lo b1}
    } c;
  } u;                                            // also the generic path's buffers
  uint4 btab[8][2][32];                           // score B operand per (chunk, plane, lane): {hi, hi, lo, lo}
  uint64_t bar[kWarps][kStages];
  uint64_t cbar[kCoopStages];
  float q[kMaxGroup][kHeadDim];                   // rotated queries, times the softmax scale
  float mw[kWarps][kMaxGroup];                    // per-warp running max (per-warp body merge; cooperative body: window max)
  float lw[kWarps][kMaxGroup];                    // per-warp softmax denominators, for the merge
  float red[kWarps][1 + kMods][kMaxGroup];        // cooperative body: per-warp sums of p and of p sigma per modality
  uint32_t tmask[kCoop][2];                       // cooperative body: modality bits of each tile of the group (0: no window)
  uint32_t tmem_base;                             // per-warp body: TMEM columns of the parked accumulators
  alignas(16) uint32_t mxpairs[kWarps][kHeadDim]; // MXFP4 caches: a warp's window metadata as fp16 (m, s) pairs
                                                  // (read as 16-byte vectors)
  float qoff[kMaxGroup];                          // TurboQuant keys: c_0 sum_c q'_c per head
  uint32_t bad_heads;                             // bit h: head h's partial is not finite (written empty)
  int abort;                                      // cooperative body: a step flag never arrived
  int wabort[kWarps];                             // per-warp body: a step flag of warp w never arrived
};
static_assert(sizeof(DecodeSmem) <= 48 * 1024, "static shared memory");
// fields read or written as 16-byte / 8-byte vectors, and mbarriers
static_assert(offsetof(DecodeSmem, btab) % 16 == 0 && offsetof(DecodeSmem, q) % 16 == 0 &&
                  offsetof(DecodeSmem, mxpairs) % 16 == 0, "16-byte vector fields");
static_assert(offsetof(DecodeSmem, mw) % 8 == 0 && offsetof(DecodeSmem, bar) % 8 == 0 &&
                  offsetof(DecodeSmem, cbar) % 8 == 0, "8-byte fields");
static_assert(sizeof(GenSmem) <= sizeof(DecodeSmem::u), "CUDA-core path shared memory");

// ---------------------------------------------------------------------------
// tensor-core path (K2/V2, symmetric codebooks)
// ---------------------------------------------------------------------------
__device__ __forceinline__ int tile_token(int r) {  // tau(r), r in 0..15
  return r < 8 ? (r >> 1) + 8 * (r & 1) : 4 + ((r - 8) >> 1) + 8 * (r & 1);
}

constexpr uint32_t kPlane0 = 0x20002000u;  // bit 13 of each half: 2^-7
constexpr uint32_t kPlane1 = 0x40004000u;  // bit 14 of each half: 2

__device__ __forceinline__ uint32_t rotl(uint32_t x, int n) { return __funnelshift_l(x, x, n); }


// (lo, hi) -> fp16 pair h = fp16(x) and l = fp16(x - h), each transposed to the
// B-fragment layout with movmatrix.
__device__ __forceinline__ void split_pair_t(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 f = __half22float2(h);
  const __half2 l = __floats2half2_rn(x0 - f.x, x1 - f.y);
  hi = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&h));
  lo = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&l));
}

// The window's key metadata as fp16 (m_c, s_c) pairs, channel c at index c: the
// record's own for fp16 metadata; for MXFP4 the warp converts its window's E2M1
// values (exact in fp16 for block exponents in [-16, 12]; a scale beyond makes the
// split non-finite, reported as OMNIKV_DEVERR_RANGE) into its buffer.
__device__ __forceinline__ void mx_window_pairs(const uint8_t* meta, uint32_t* out, int lane) {
  __syncwarp();  // the previous window's readers are done
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int c = lane + 32 * k;
    const float2 ms = mx_meta_channel(meta, c);
    const __half2 h = __floats2half2_rn(ms.x, ms.y);
    out[c] = *reinterpret_cast<const uint32_t*>(&h);
  }
  __syncwarp();
}

template <int kMeta>
__device__ __forceinline__ const __half2* window_meta_pairs(DecodeSmem& sm, const uint8_t* rec, int warp, int lane) {
  if (kMeta != kMetaMx) return reinterpret_cast<const __half2*>(rec + Rec22<kMeta>::meta);
  mx_window_pairs(rec + Rec22<kMeta>::meta, sm.mxpairs[warp], lane);
  return reinterpret_cast<const __half2*>(sm.mxpairs[warp]);
}

// The split's maximum and denominator of head h; a split whose partial is not
// finite (inputs outside the fp16 range of the operands) is reported and written
// empty, so the combine gives it weight 0 and never reads its accumulators.
template <class Smem>
__device__ __forceinline__ void write_split_ml(const DecodeParams& p, const Smem& sm, int b, int kvh, int h,
                                               int split, float m, float l) {
  Partial* out = p.partials + ((size_t)b * p.num_kv_heads * p.group + kvh * p.group + h) * p.num_splits + split;
  const bool bad = ((sm.bad_heads >> h) & 1u) || !isfinite(l) || isnan(m) || m == INFINITY;
  if (bad) set_error(p.error_word, OMNIKV_DEVERR_RANGE);
  out->m = bad ? -INFINITY : m;
  out->l = bad ? 0.0f : l;
}

// Per-warp decode state. Only the accumulator of the active modality lives in
// registers; the others are parked in this warp's TMEM lanes (columns 32 m ..
// 32 m + 31 for modality m), each with the running max it was parked at, and are
// rescaled to the current max when they are brought back.
struct WarpState {
  float m[2];              // running max for heads 2t, 2t+1 (warp-uniform per column)
  float l[2];              // per-lane partial sum of p for heads 2t, 2t+1
  float S[kMods][2];       // per-lane partial sum of p * sigma per modality (kept at the running max)
  float mref[kMods][2];    // running max at which a parked accumulator was stored
  float acc[8][4];         // accumulator of the active modality
  int cur;                 // active modality, -1 if none (warp-uniform)
  uint32_t parked;         // bit m set: modality m's accumulator is parked in TMEM (warp-uniform)
};

__device__ __forceinline__ uint32_t slot_addr(uint32_t tbase, int warp, int m) {
  return tbase + ((uint32_t)(32 * warp) << 16) + 32u * (uint32_t)m;
}

__device__ __forceinline__ void park_active(WarpState& st, uint32_t tbase, int warp) {
  tmem_st32(slot_addr(tbase, warp, st.cur), reinterpret_cast<const uint32_t*>(&st.acc[0][0]));
#pragma unroll
  for (int mm = 0; mm < kMods; ++mm)
    if (mm == st.cur) {
      st.mref[mm][0] = st.m[0];
      st.mref[mm][1] = st.m[1];
    }
  st.parked |= 1u << st.cur;
}

// Load modality m's parked accumulator into acc, scaled by 2^((mref - target) log2 e)
// per column, or zeros if it was never parked. Warp-collective.
__device__ __forceinline__ void unpark(WarpState& st, int m, uint32_t tbase, int warp, float tgt0, float tgt1) {
  if (st.parked & (1u << m)) {
    tmem_ld32(slot_addr(tbase, warp, m), reinterpret_cast<uint32_t*>(&st.acc[0][0]));
    float r0 = 0.f, r1 = 0.f;
#pragma unroll
    for (int mm = 0; mm < kMods; ++mm)
      if (mm == m) {
        r0 = st.mref[mm][0];
        r1 = st.mref[mm][1];
      }
    const float f0 = fast_exp2((r0 - tgt0) * kLog2e), f1 = fast_exp2((r1 - tgt1) * kLog2e);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      st.acc[mt][0] *= f0;
      st.acc[mt][1] *= f1;
      st.acc[mt][2] *= f0;
      st.acc[mt][3] *= f1;
    }
  } else {
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int r = 0; r < 4; ++r) st.acc[mt][r] = 0.0f;
  }
}

// Make modality m the active one (warp-uniform m).
__device__ __forceinline__ void activate(WarpState& st, int m, uint32_t tbase, int warp) {
  if (m == st.cur) return;
  if (st.cur >= 0) park_active(st, tbase, warp);
  unpark(st, m, tbase, warp, st.m[0], st.m[1]);
  st.cur = m;
}

// Warp `warp` of the CTA decodes the contiguous windows [*a, *e) of [w0, w1).
__device__ __forceinline__ void warp_windows(int w0, int w1, int warp, int& a, int& e) {
  const int per = (w1 - w0 + kWarps - 1) / kWarps;
  a = min(w0 + warp * per, w1);
  e = min(a + per, w1);
}

template <int kMeta>
__device__ __forceinline__ void issue_window(const DecodeParams& p, DecodeSmem& sm, int warp, int stage,
                                             const uint8_t* rec_base, int b, int kvh, int wi, int wait_win,
                                             int wait_val) {
  uint64_t* bar = &sm.bar[warp][stage];
  if (wi == wait_win &&
      !wait_flag(p.step_flags + (size_t)b * p.num_kv_heads + kvh, wait_val, p.flag_wait_ns)) {
    // the appended token's record never became ready: no copy of a stale record;
    // the warp's split is written empty
    set_error(p.error_word, OMNIKV_DEVERR_TIMEOUT);
    sm.wabort[warp] = 1;
    mbar_arrive_expect_tx(bar, 0);
    return;
  }
  uint8_t* dst = &sm.u.w.stage[warp][stage][0];
  constexpr int rb = Rec22<kMeta>::bytes;
  mbar_arrive_expect_tx(bar, rb + kWindow);
  bulk_copy_g2s(dst, rec_base + (size_t)wi * rb, rb, bar);
  bulk_copy_g2s(dst + rb, p.modality + (size_t)b * p.cap_tokens + (size_t)wi * kWindow, kWindow, bar);
}

// Each warp's first kStages windows: barrier set-up and bulk copies (lane 0).
template <int kMeta>
__device__ __forceinline__ void prime_pipeline(const DecodeParams& p, DecodeSmem& sm, int b, int kvh, int w0, int w1) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint8_t* rec_base =
      p.records + ((size_t)(b * p.num_kv_heads + kvh) * p.cap_windows) * Rec22<kMeta>::bytes;
  int wa, we, wait_win, wait_val;
  warp_windows(w0, w1, warp, wa, we);
  step_window(p, b, wait_win, wait_val);
  if (lane == 0) {
    sm.wabort[warp] = 0;
#pragma unroll
    for (int s = 0; s < kStages; ++s) mbar_init(&sm.bar[warp][s], 1);
    fence_barrier_init();
    for (int i = 0; i < kStages && wa + i < we; ++i)
      issue_window<kMeta>(p, sm, warp, i, rec_base, b, kvh, wa + i, wait_win, wait_val);
  }
  __syncwarp();
}

template <int kMeta>
__device__ void decode_mma(const DecodeParams& p, DecodeSmem& sm, int b, int kvh, int split, float kV0, float kV1,
                           float vc0, uint32_t tbase, float escale) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int G = p.group;
  const int Hq = p.num_kv_heads * G;
  int T, w0, w1;
  split_range(p, b, split, T, w0, w1);
  const uint8_t* rec_base =
      p.records + ((size_t)(b * p.num_kv_heads + kvh) * p.cap_windows) * Rec22<kMeta>::bytes;
  int wa, we, wait_win, wait_val;
  warp_windows(w0, w1, warp, wa, we);
  step_window(p, b, wait_win, wait_val);
  const int nmine = we - wa;

  WarpState st;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    st.m[j] = -INFINITY;
    st.l[j] = 0.0f;
#pragma unroll
    for (int m = 0; m < kMods; ++m) {
      st.S[m][j] = 0.0f;
      st.mref[m][j] = -INFINITY;
    }
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int r = 0; r < 4; ++r) st.acc[mt][r] = 0.0f;
  st.cur = -1;
  st.parked = 0;

  int failed_at = -1;
  for (int i = 0; i < nmine; ++i) {
    const int s = i % kStages;
    const int wi = wa + i;
    // the warp leaves together: a lane whose wait ran out, or lane 0 (the lane
    // that issues the copies) having given up on a step flag, stops every lane
    const bool ok = mbar_wait_bounded(&sm.bar[warp][s], (i / kStages) & 1, kWaitLimitNs) &&
                    *reinterpret_cast<volatile int*>(&sm.wabort[warp]) == 0;
    if (!__all_sync(0xffffffffu, ok)) {
      failed_at = i;
      break;
    }
    const uint8_t* stg = &sm.u.w.stage[warp][s][0];
    const uint32_t* kw = reinterpret_cast<const uint32_t*>(stg);
    using L = Rec22<kMeta>;
    const __half2* meta = window_meta_pairs<kMeta>(sm, stg, warp, lane);
    const __half* ksig = reinterpret_cast<const __half*>(stg + L::meta);  // TurboQuant keys: per-token scales
    const uint32_t* vw = reinterpret_cast<const uint32_t*>(stg + L::v);
    const __half* sig = reinterpret_cast<const __half*>(stg + L::sigma);
    const uint8_t* mods = stg + L::bytes;

    // ---- per-window: fp16 scale pairs for the A operand, offset sum_c q'_c m_gc
    // lane (g, t) covers channels 32t .. 32t+31 (k-slot pairs (c, c+8))
    uint32_t sp[8][2];
    float off = 0.0f;
    if constexpr (kMeta == kMetaTurbo) {
#pragma unroll
      for (int kc = 0; kc < 8; ++kc) sp[kc][0] = sp[kc][1] = 0u;  // no window scales
    } else {
      const float* qrow = &sm.q[g][32 * t];
      const int qsw = (4 * (g & 1) + t) & 7;
      const uint4* mv4 = reinterpret_cast<const uint4*>(meta + 32 * t);
      uint32_t mv[32];
#pragma unroll
      for (int i4 = 0; i4 < 8; ++i4) {
        const uint4 mm = mv4[i4];
        mv[4 * i4 + 0] = mm.x;
        mv[4 * i4 + 1] = mm.y;
        mv[4 * i4 + 2] = mm.z;
        mv[4 * i4 + 3] = mm.w;
      }
      off = 0.0f;
#pragma unroll
      for (int i4 = 0; i4 < 8; ++i4) {
        const float4 qq = *reinterpret_cast<const float4*>(qrow + 4 * (i4 ^ qsw));
        const float qa[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          off = fmaf(qa[j], __low2float(*reinterpret_cast<const __half2*>(&mv[4 * i4 + j])), off);
      }
#pragma unroll
      for (int kc = 0; kc < 8; ++kc) {  // high halves (the scales) of channels (c, c+8)
        sp[kc][0] = __byte_perm(mv[kc], mv[kc + 8], 0x7632);
        sp[kc][1] = __byte_perm(mv[kc + 16], mv[kc + 24], 0x7632);
      }
      off += __shfl_xor_sync(0xffffffffu, off, 1);
      off += __shfl_xor_sync(0xffffffffu, off, 2);
    }
    // TurboQuant keys: the window-independent c_0 sum_c q'_c of heads 2t, 2t+1
    const float off0 = kMeta == kMetaTurbo ? sm.qoff[2 * t] : __shfl_sync(0xffffffffu, off, 8 * t);
    const float off1 = kMeta == kMetaTurbo ? sm.qoff[2 * t + 1] : __shfl_sync(0xffffffffu, off, 8 * t + 4);

    // ---- scores for the two 16-token tiles, issued interleaved per chunk (4
    // independent accumulator chains)
    float sc[2][4];
    int tokA[2], tokB[2];
    uint2 kA[2], kB[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      tokA[h] = 16 * h + tile_token(g);
      tokB[h] = 16 * h + tile_token(g + 8);
      kA[h] = *reinterpret_cast<const uint2*>(kw + tokA[h] * 8 + 2 * t);
      kB[h] = *reinterpret_cast<const uint2*>(kw + tokB[h] * 8 + 2 * t);
    }
    {
      float d0[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      float d1[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int kc = 0; kc < 8; ++kc) {
        const uint32_t s0 = sp[kc][0], s1 = sp[kc][1];
        const uint4 bp0 = sm.btab[kc][0][lane], bp1 = sm.btab[kc][1][lane];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t r[4];
          if (kc < 7) {
            r[0] = kA[h].x << (13 - 2 * kc);
            r[1] = kB[h].x << (13 - 2 * kc);
            r[2] = kA[h].y << (13 - 2 * kc);
            r[3] = kB[h].y << (13 - 2 * kc);
          } else {
            r[0] = kA[h].x >> 1;
            r[1] = kB[h].x >> 1;
            r[2] = kA[h].y >> 1;
            r[3] = kB[h].y >> 1;
          }
          uint32_t a0[4], a1[4];
          if constexpr (kMeta == kMetaTurbo) {  // the code planes alone (the scale is per token)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              a0[k] = r[k] & kPlane0;
              a1[k] = r[k] & kPlane1;
            }
          } else {
            a0[0] = hmul2_u32(s0, r[0] & kPlane0), a0[1] = hmul2_u32(s0, r[1] & kPlane0);
            a0[2] = hmul2_u32(s1, r[2] & kPlane0), a0[3] = hmul2_u32(s1, r[3] & kPlane0);
            a1[0] = hmul2_u32(s0, r[0] & kPlane1), a1[1] = hmul2_u32(s0, r[1] & kPlane1);
            a1[2] = hmul2_u32(s1, r[2] & kPlane1), a1[3] = hmul2_u32(s1, r[3] & kPlane1);
          }
          mma_f16_16816(d0[h], a0, bp0.x, bp0.y);
          mma_f16_16816(d1[h], a1, bp1.x, bp1.y);
          mma_f16_16816(d0[h], a0, bp0.z, bp0.w);
          mma_f16_16816(d1[h], a1, bp1.z, bp1.w);
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int posA = wi * kWindow + tokA[h], posB = wi * kWindow + tokB[h];
        // TurboQuant keys: k'_tc = ksigma_t c_j, so the score is ksigma_t times the sum
        const float kgA = kMeta == kMetaTurbo ? __half2float(ksig[tokA[h]]) : 1.0f;
        const float kgB = kMeta == kMetaTurbo ? __half2float(ksig[tokB[h]]) : 1.0f;
        sc[h][0] = posA < T ? kgA * fmaf(d0[h][0] + d1[h][0], escale, off0) : -INFINITY;
        sc[h][1] = posA < T ? kgA * fmaf(d0[h][1] + d1[h][1], escale, off1) : -INFINITY;
        sc[h][2] = posB < T ? kgB * fmaf(d0[h][2] + d1[h][2], escale, off0) : -INFINITY;
        sc[h][3] = posB < T ? kgB * fmaf(d0[h][3] + d1[h][3], escale, off1) : -INFINITY;
      }
    }

    // ---- online softmax over the window (parked accumulators keep their own
    // reference max and are rescaled when brought back)
    float mx0 = fmaxf(fmaxf(sc[0][0], sc[0][2]), fmaxf(sc[1][0], sc[1][2]));
    float mx1 = fmaxf(fmaxf(sc[0][1], sc[0][3]), fmaxf(sc[1][1], sc[1][3]));
#pragma unroll
    for (int o = 4; o <= 16; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const float mn0 = fmaxf(st.m[0], mx0), mn1 = fmaxf(st.m[1], mx1);
    if (__any_sync(0xffffffffu, mn0 > st.m[0] || mn1 > st.m[1])) {
      const float a0 = fast_exp2((st.m[0] - mn0) * kLog2e), a1 = fast_exp2((st.m[1] - mn1) * kLog2e);
      st.l[0] *= a0;
      st.l[1] *= a1;
#pragma unroll
      for (int m = 0; m < kMods; ++m) {
        st.S[m][0] *= a0;
        st.S[m][1] *= a1;
      }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        st.acc[mt][0] *= a0;
        st.acc[mt][1] *= a1;
        st.acc[mt][2] *= a0;
        st.acc[mt][3] *= a1;
      }
      st.m[0] = mn0;
      st.m[1] = mn1;
    }
    const float ms0 = st.m[0] * kLog2e, ms1 = st.m[1] * kLog2e;

    // ---- value product per tile (a rolled loop: half the code, fewer instruction
    // fetch stalls; 2.6 % faster on the 8 x 65,536-token layer than unrolled)
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
      const float p0 = fast_exp2(fmaf(h ? sc[1][0] : sc[0][0], kLog2e, -ms0));
      const float p1 = fast_exp2(fmaf(h ? sc[1][1] : sc[0][1], kLog2e, -ms1));
      const float p2 = fast_exp2(fmaf(h ? sc[1][2] : sc[0][2], kLog2e, -ms0));
      const float p3 = fast_exp2(fmaf(h ? sc[1][3] : sc[0][3], kLog2e, -ms1));
      st.l[0] += p0 + p2;
      st.l[1] += p1 + p3;
      const int tA = h ? tokA[1] : tokA[0], tB = h ? tokB[1] : tokB[0];
      const float sgA = __half2float(sig[tA]), sgB = __half2float(sig[tB]);
      const float w0v = p0 * sgA, w1v = p1 * sgA, w2v = p2 * sgB, w3v = p3 * sgB;
      // value-product B operand per plane, as fp16 high + low parts
      uint32_t bv0[4], bv1[4];  // {hi(row g), hi(row g+8), lo(row g), lo(row g+8)}, transposed
      split_pair_t(w0v * kV0, w1v * kV0, bv0[0], bv0[2]);
      split_pair_t(w2v * kV0, w3v * kV0, bv0[1], bv0[3]);
      split_pair_t(w0v * kV1, w1v * kV1, bv1[0], bv1[2]);
      split_pair_t(w2v * kV1, w3v * kV1, bv1[1], bv1[3]);
      // modalities of this tile (warp-uniform mask) and of this lane's tokens
      const int mA = min((int)mods[tA], 2), mB = min((int)mods[tB], 2);
      const uint32_t mbits = __reduce_or_sync(0xffffffffu, (1u << mA) | (1u << mB));
      // k-slots of this lane's B registers: 2t, 2t+1 -> tokens t, t+8; 2t+8, 2t+9 -> t+4, t+12
      const int base = 16 * h;
      const int mk0 = min((int)mods[base + t], 2), mk1 = min((int)mods[base + t + 8], 2);
      const int mk2 = min((int)mods[base + t + 4], 2), mk3 = min((int)mods[base + t + 12], 2);
      const int rlo = 13 - 2 * t, rhi = (5 - 2 * t) & 31;
      const uint4* vsrc = reinterpret_cast<const uint4*>(vw + h * kHeadDim + 16 * g);
      // one (masked) product per modality present, the active one first
      uint32_t todo = mbits;
      int mm = (st.cur >= 0 && ((todo >> st.cur) & 1u)) ? st.cur : __ffs(todo) - 1;
#pragma unroll 1
      while (true) {
        activate(st, mm, tbase, warp);
        const bool single = mbits == (1u << mm);
        const uint32_t msk01 = single ? 0xFFFFFFFFu : ((mk0 == mm ? 0x0000FFFFu : 0u) | (mk1 == mm ? 0xFFFF0000u : 0u));
        const uint32_t msk23 = single ? 0xFFFFFFFFu : ((mk2 == mm ? 0x0000FFFFu : 0u) | (mk3 == mm ? 0xFFFF0000u : 0u));
        const uint32_t b00 = bv0[0] & msk01, b01 = bv0[1] & msk23;
        const uint32_t b10 = bv1[0] & msk01, b11 = bv1[1] & msk23;
        const uint32_t c00 = bv0[2] & msk01, c01 = bv0[3] & msk23;
        const uint32_t c10 = bv1[2] & msk01, c11 = bv1[3] & msk23;
        const float u0 = (mA == mm ? w0v : 0.0f) + (mB == mm ? w2v : 0.0f);
        const float u1 = (mA == mm ? w1v : 0.0f) + (mB == mm ? w3v : 0.0f);
#pragma unroll
        for (int k = 0; k < kMods; ++k)
          if (k == mm) {
            st.S[k][0] += u0;
            st.S[k][1] += u1;
          }
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint4 u = vsrc[q4];  // V words of channels 16g + 4 q4 .. + 3
          const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int mt = 2 * q4 + e;
            const uint32_t wg = wv[2 * e], wg8 = wv[2 * e + 1];
            const uint32_t r[4] = {rotl(wg, rlo), rotl(wg8, rlo), rotl(wg, rhi), rotl(wg8, rhi)};
            const uint32_t a0[4] = {r[0] & kPlane0, r[1] & kPlane0, r[2] & kPlane0, r[3] & kPlane0};
            const uint32_t a1[4] = {r[0] & kPlane1, r[1] & kPlane1, r[2] & kPlane1, r[3] & kPlane1};
            mma_f16_16816(st.acc[mt], a0, b00, b01);
            mma_f16_16816(st.acc[mt], a1, b10, b11);
            mma_f16_16816(st.acc[mt], a0, c00, c01);
            mma_f16_16816(st.acc[mt], a1, c10, c11);
          }
        }
        todo &= ~(1u << mm);
        if (!todo) break;
        mm = __ffs(todo) - 1;
      }
    }
    __syncwarp();
    if (lane == 0 && i + kStages < nmine) {
      fence_proxy_async_smem();
      issue_window<kMeta>(p, sm, warp, s, rec_base, b, kvh, wa + i + kStages, wait_win, wait_val);
    }
  }

  if (__any_sync(0xffffffffu, failed_at >= 0)) {
    // a copy did not complete in time: report it, wait (bounded) for the copies
    // still in flight (windows failed_at .. failed_at + kStages - 1), give up
    const int f = __shfl_sync(0xffffffffu, failed_at, 0);
    if (lane == 0) set_error(p.error_word, OMNIKV_DEVERR_TIMEOUT);
    for (int j = f; j < nmine && j < f + kStages; ++j)
      mbar_wait_bounded(&sm.bar[warp][j % kStages], (j / kStages) & 1, kWaitLimitNs);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      st.m[j] = -INFINITY;
      st.l[j] = 0.0f;
#pragma unroll
      for (int m = 0; m < kMods; ++m) st.S[m][j] = 0.0f;
    }
    st.cur = -1;
    st.parked = 0;
  }
  if (st.cur >= 0) park_active(st, tbase, warp);

  // ---- reduce the per-lane partial sums over the 8 lanes sharing a column
#pragma unroll
  for (int o = 4; o <= 16; o <<= 1) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      st.l[j] += __shfl_xor_sync(0xffffffffu, st.l[j], o);
#pragma unroll
      for (int m = 0; m < kMods; ++m) st.S[m][j] += __shfl_xor_sync(0xffffffffu, st.S[m][j], o);
    }
  }

  // ---- merge the 4 warps at their common max, one modality at a time ------
  if (g == 0) {
    sm.mw[warp][2 * t] = st.m[0];
    sm.mw[warp][2 * t + 1] = st.m[1];
  }
  __syncthreads();  // also: all warps are done with their stage buffers
  float M[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) mm = fmaxf(mm, sm.mw[w][2 * t + j]);
    M[j] = mm;
    const float f = (st.m[j] == -INFINITY) ? 0.0f : fast_exp2((st.m[j] - mm) * kLog2e);
    st.l[j] *= f;
#pragma unroll
    for (int m = 0; m < kMods; ++m) st.S[m][j] *= f;
  }
  if (g == 0) {
    sm.lw[warp][2 * t] = st.l[0];
    sm.lw[warp][2 * t + 1] = st.l[1];
  }
  float* xbuf = reinterpret_cast<float*>(&sm.u.w.stage[0][0][0]);  // [warp][32 registers][32 lanes]
  static_assert(kWarps * 32 * 32 * 4 <= kWarps * kStages * kStageBytes, "merge buffer");
#pragma unroll
  for (int m = 0; m < kMods; ++m) {
    unpark(st, m, tbase, warp, M[0], M[1]);  // zeros if this warp never saw modality m
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int r = 0; r < 4; ++r)
        xbuf[(warp * 32 + mt * 4 + r) * 32 + lane] = st.acc[mt][r] + vc0 * st.S[m][r & 1];
    __syncthreads();
    // warp w sums registers of m-tiles 2w, 2w+1 over the 4 warps and writes them
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int mt = 2 * warp + e;
      float v[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        float x = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) x += xbuf[(w * 32 + mt * 4 + r) * 32 + lane];
        v[r] = x;
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int hh = 2 * t + j;
        if (hh >= G) continue;
        Partial* out = p.partials + ((size_t)b * Hq + kvh * G + hh) * p.num_splits + split;
        *reinterpret_cast<float2*>(&out->acc[m][16 * g + 2 * mt]) = make_float2(v[j], v[j + 2]);
        if (!isfinite(v[j]) || !isfinite(v[j + 2])) atomicOr(&sm.bad_heads, 1u << hh);
      }
    }
    __syncthreads();
  }
  if (warp == 0 && g == 0) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int hh = 2 * t + j;
      if (hh >= G) continue;
      float l = 0.0f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) l += sm.lw[w][hh];
      write_split_ml(p, sm, b, kvh, hh, split, M[j], l);
    }
  }
}

// Value-product accumulators of one warp: the warp owns channels 32 w + 4 g + 2 mt
// (fragment row g) and + 1 (row g + 8) for m-tiles mt = 0, 1, and the query
// heads 2t, 2t+1 as columns. The active modality accumulates in act (one chain
// per m-tile and code plane); the totals of the other modalities wait in st, and
// are exchanged when a tile of another modality comes (rare: modality runs are
// long).
struct PvAcc {
  float act[2][2][4];      // [m-tile][plane][fragment] of the active modality
  float st[kMods][2][4];   // [modality][m-tile][fragment], inactive modalities
  int cur;                 // active modality, -1 before the first tile (warp-uniform)
};

__device__ __forceinline__ void pv_activate(PvAcc& a, int k) {
  if (k == a.cur) return;
#pragma unroll
  for (int kk = 0; kk < kMods; ++kk)
    if (kk == a.cur) {
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int r = 0; r < 4; ++r) a.st[kk][mt][r] = a.act[mt][0][r] + a.act[mt][1][r];
    }
#pragma unroll
  for (int kk = 0; kk < kMods; ++kk)
    if (kk == k) {
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          a.act[mt][0][r] = a.st[kk][mt][r];
          a.act[mt][1][r] = 0.0f;
        }
    }
  a.cur = k;
}

// 8 MMAs of one 16-token tile into the active accumulator: B = {hi b0, hi b1,
// lo b0, lo b1} per plane, k-slot halves masked with m01 (b0) and m23 (b1).
__device__ __forceinline__ void pv_tile(PvAcc& a, const uint32_t (&a0)[2][4], const uint32_t (&a1)[2][4],
                                        const uint4& f0, const uint4& f1, uint32_t m01, uint32_t m23) {
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    mma_f16_16816(a.act[mt][0], a0[mt], f0.x & m01, f0.y & m23);
    mma_f16_16816(a.act[mt][1], a1[mt], f1.x & m01, f1.y & m23);
  }
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    mma_f16_16816(a.act[mt][0], a0[mt], f0.z & m01, f0.w & m23);
    mma_f16_16816(a.act[mt][1], a1[mt], f1.z & m01, f1.w & m23);
  }
}

__device__ __forceinline__ void pv_scale(PvAcc& a, float f0, float f1) {
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int P = 0; P < 2; ++P) {
      a.act[mt][P][0] *= f0;
      a.act[mt][P][1] *= f1;
      a.act[mt][P][2] *= f0;
      a.act[mt][P][3] *= f1;
    }
#pragma unroll
  for (int k = 0; k < kMods; ++k)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      a.st[k][mt][0] *= f0;
      a.st[k][mt][1] *= f1;
      a.st[k][mt][2] *= f0;
      a.st[k][mt][3] *= f1;
    }
}

// Copies of window group `gi` (windows wfirst .. wfirst + nwin - 1): the records
// (contiguous in the cache) and then their modality ids, completing on the
// stage's mbarrier. In a decode step the window that receives the new token is
// copied only after its flag shows the append (bounded wait); the records before
// it go first. Thread 0.
template <int kMeta>
__device__ __forceinline__ void issue_group(const DecodeParams& p, DecodeSmem& sm, int stage, const uint8_t* rec_base,
                                            int b, int kvh, int wfirst, int nwin, int wait_win, int wait_val) {
  uint64_t* bar = &sm.cbar[stage];
  uint8_t* dst = &sm.u.c.stage[stage][0];
  constexpr int rb = Rec22<kMeta>::bytes;
  int nfree = nwin;  // records that need no wait
  if (wait_win >= wfirst && wait_win < wfirst + nwin) nfree = wait_win - wfirst;
  if (nfree == nwin) {
    mbar_arrive_expect_tx(bar, (uint32_t)nwin * (rb + kWindow));
    bulk_copy_g2s(dst, rec_base + (size_t)wfirst * rb, (uint32_t)nwin * rb, bar);
    bulk_copy_g2s(dst + kCoop * rb, p.modality + (size_t)b * p.cap_tokens + (size_t)wfirst * kWindow,
                  (uint32_t)nwin * kWindow, bar);
    return;
  }
  // the records that need no wait are copied first; the phase cannot complete
  // before the arrive below. The modality ids (the appended token's is written by
  // its append CTA before the flag) and the waited-for records follow the flag.
  if (nfree > 0) {
    mbar_expect_tx(bar, (uint32_t)nfree * rb);
    bulk_copy_g2s(dst, rec_base + (size_t)wfirst * rb, (uint32_t)nfree * rb, bar);
  }
  if (!wait_flag(p.step_flags + (size_t)b * p.num_kv_heads + kvh, wait_val, p.flag_wait_ns)) {
    // the appended token's record never became ready: no copy of a stale record;
    // the split is written empty
    set_error(p.error_word, OMNIKV_DEVERR_TIMEOUT);
    sm.abort = 1;
    mbar_arrive_expect_tx(bar, 0);
    return;
  }
  mbar_arrive_expect_tx(bar, (uint32_t)(nwin - nfree) * rb + (uint32_t)nwin * kWindow);
  bulk_copy_g2s(dst + nfree * rb, rec_base + (size_t)(wfirst + nfree) * rb, (uint32_t)(nwin - nfree) * rb, bar);
  bulk_copy_g2s(dst + kCoop * rb, p.modality + (size_t)b * p.cap_tokens + (size_t)wfirst * kWindow,
                (uint32_t)nwin * kWindow, bar);
}

// The tensor-core decode of one split. Windows are taken kCoop at a time (a
// group, one shared-memory stage): warp w scores window w of the group (both
// 16-token tiles), the CTA takes the common running max, warp w turns its
// probabilities into the value-product B operand in shared memory, and then every
// warp runs the value product of the whole group for its own 32 channels.
template <int kMeta>
__device__ void decode_coop(const DecodeParams& p, DecodeSmem& sm, int b, int kvh, int split, float kV0, float kV1,
                            float vc0, float escale) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int G = p.group;
  const int Hq = p.num_kv_heads * G;
  int T, w0, w1;
  split_range(p, b, split, T, w0, w1);
  const uint8_t* rec_base =
      p.records + ((size_t)(b * p.num_kv_heads + kvh) * p.cap_windows) * Rec22<kMeta>::bytes;
  int wait_win, wait_val;
  step_window(p, b, wait_win, wait_val);
  const int ngroups = (w1 - w0 + kCoop - 1) / kCoop;
  int issued = 0;  // groups whose copies were issued (meaningful in thread 0)
  if (threadIdx.x == 0) {
    sm.abort = 0;
#pragma unroll
    for (int s = 0; s < kCoopStages; ++s) mbar_init(&sm.cbar[s], 1);
    fence_barrier_init();
    for (; issued < kCoopStages && issued < ngroups; ++issued)
      issue_group<kMeta>(p, sm, issued, rec_base, b, kvh, w0 + kCoop * issued, min(kCoop, w1 - w0 - kCoop * issued),
                  wait_win, wait_val);
  }
  __syncthreads();  // barrier initialisation (and the score operand) visible to every thread

  float m_run[2] = {-INFINITY, -INFINITY};  // running max of heads 2t, 2t+1 (the same in every warp)
  float l_part[2] = {0.0f, 0.0f};           // per-lane partial sums of p over this warp's windows
  float S_part[kMods][2];                   // per-lane partial sums of p * sigma per modality
#pragma unroll
  for (int k = 0; k < kMods; ++k) S_part[k][0] = S_part[k][1] = 0.0f;
  PvAcc pv;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      pv.act[mt][0][r] = pv.act[mt][1][r] = 0.0f;
#pragma unroll
      for (int k = 0; k < kMods; ++k) pv.st[k][mt][r] = 0.0f;
    }
  pv.cur = -1;
  const int rlo = 13 - 2 * t, rhi = (5 - 2 * t) & 31;

  int failed_at = -1;
  for (int it = 0; it < ngroups; ++it) {
    const int s = it % kCoopStages;
    const int wi = w0 + kCoop * it + warp;  // this warp's window for the scores
    const bool have = wi < w1;              // warp-uniform
    const uint8_t* stg = &sm.u.c.stage[s][0];
    const bool ok = mbar_wait_bounded(&sm.cbar[s], (it / kCoopStages) & 1, kWaitLimitNs) &&
                    *reinterpret_cast<volatile int*>(&sm.abort) == 0;
    const bool wok = __all_sync(0xffffffffu, ok);

    // ---- scores of this warp's window (both tiles) -------------------------
    using L = Rec22<kMeta>;
    const uint8_t* rec = stg + warp * L::bytes;
    const uint8_t* mods = stg + kCoop * L::bytes + warp * kWindow;
    float sc[2][4];
    int tokA[2], tokB[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      tokA[h] = 16 * h + tile_token(g);
      tokB[h] = 16 * h + tile_token(g + 8);
#pragma unroll
      for (int r = 0; r < 4; ++r) sc[h][r] = -INFINITY;
    }
    if (have && wok) {
      const uint32_t* kw = reinterpret_cast<const uint32_t*>(rec);
      const __half2* meta = window_meta_pairs<kMeta>(sm, rec, warp, lane);
      const __half* ksig = reinterpret_cast<const __half*>(rec + L::meta);  // TurboQuant keys: per-token scales
      // fp16 scale pairs of the A operand and the offset sum_c q'_c m_gc; lane
      // (g, t) covers channels 32t .. 32t+31 (k-slot pairs (c, c+8))
      uint32_t sp[8][2];
      float off = 0.0f;
      if constexpr (kMeta == kMetaTurbo) {
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) sp[kc][0] = sp[kc][1] = 0u;  // no window scales
      } else {
        const float* qrow = &sm.q[g][32 * t];
        const int qsw = (4 * (g & 1) + t) & 7;
        const uint4* mv4 = reinterpret_cast<const uint4*>(meta + 32 * t);
        uint32_t mv[32];
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const uint4 mm = mv4[i4];
          mv[4 * i4 + 0] = mm.x;
          mv[4 * i4 + 1] = mm.y;
          mv[4 * i4 + 2] = mm.z;
          mv[4 * i4 + 3] = mm.w;
        }
        off = 0.0f;
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 qq = *reinterpret_cast<const float4*>(qrow + 4 * (i4 ^ qsw));
          const float qa[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            off = fmaf(qa[j], __low2float(*reinterpret_cast<const __half2*>(&mv[4 * i4 + j])), off);
        }
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {  // high halves (the scales) of channels (c, c+8)
          sp[kc][0] = __byte_perm(mv[kc], mv[kc + 8], 0x7632);
          sp[kc][1] = __byte_perm(mv[kc + 16], mv[kc + 24], 0x7632);
        }
        off += __shfl_xor_sync(0xffffffffu, off, 1);
        off += __shfl_xor_sync(0xffffffffu, off, 2);
      }
      // TurboQuant keys: the window-independent c_0 sum_c q'_c of heads 2t, 2t+1
      const float off0 = kMeta == kMetaTurbo ? sm.qoff[2 * t] : __shfl_sync(0xffffffffu, off, 8 * t);
      const float off1 = kMeta == kMetaTurbo ? sm.qoff[2 * t + 1] : __shfl_sync(0xffffffffu, off, 8 * t + 4);
      uint2 kA[2], kB[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        kA[h] = *reinterpret_cast<const uint2*>(kw + tokA[h] * 8 + 2 * t);
        kB[h] = *reinterpret_cast<const uint2*>(kw + tokB[h] * 8 + 2 * t);
      }
      float d0[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      float d1[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int kc = 0; kc < 8; ++kc) {
        const uint32_t s0 = sp[kc][0], s1 = sp[kc][1];
        const uint4 bp0 = sm.btab[kc][0][lane], bp1 = sm.btab[kc][1][lane];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t r[4];
          if (kc < 7) {
            r[0] = kA[h].x << (13 - 2 * kc);
            r[1] = kB[h].x << (13 - 2 * kc);
            r[2] = kA[h].y << (13 - 2 * kc);
            r[3] = kB[h].y << (13 - 2 * kc);
          } else {
            r[0] = kA[h].x >> 1;
            r[1] = kB[h].x >> 1;
            r[2] = kA[h].y >> 1;
            r[3] = kB[h].y >> 1;
          }
          uint32_t a0[4], a1[4];
          if constexpr (kMeta == kMetaTurbo) {  // the code planes alone (the scale is per token)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              a0[k] = r[k] & kPlane0;
              a1[k] = r[k] & kPlane1;
            }
          } else {
            a0[0] = hmul2_u32(s0, r[0] & kPlane0), a0[1] = hmul2_u32(s0, r[1] & kPlane0);
            a0[2] = hmul2_u32(s1, r[2] & kPlane0), a0[3] = hmul2_u32(s1, r[3] & kPlane0);
            a1[0] = hmul2_u32(s0, r[0] & kPlane1), a1[1] = hmul2_u32(s0, r[1] & kPlane1);
            a1[2] = hmul2_u32(s1, r[2] & kPlane1), a1[3] = hmul2_u32(s1, r[3] & kPlane1);
          }
          mma_f16_16816(d0[h], a0, bp0.x, bp0.y);
          mma_f16_16816(d1[h], a1, bp1.x, bp1.y);
          mma_f16_16816(d0[h], a0, bp0.z, bp0.w);
          mma_f16_16816(d1[h], a1, bp1.z, bp1.w);
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int posA = wi * kWindow + tokA[h], posB = wi * kWindow + tokB[h];
        // TurboQuant keys: k'_tc = ksigma_t c_j, so the score is ksigma_t times the sum
        const float kgA = kMeta == kMetaTurbo ? __half2float(ksig[tokA[h]]) : 1.0f;
        const float kgB = kMeta == kMetaTurbo ? __half2float(ksig[tokB[h]]) : 1.0f;
        sc[h][0] = posA < T ? kgA * fmaf(d0[h][0] + d1[h][0], escale, off0) : -INFINITY;
        sc[h][1] = posA < T ? kgA * fmaf(d0[h][1] + d1[h][1], escale, off1) : -INFINITY;
        sc[h][2] = posB < T ? kgB * fmaf(d0[h][2] + d1[h][2], escale, off0) : -INFINITY;
        sc[h][3] = posB < T ? kgB * fmaf(d0[h][3] + d1[h][3], escale, off1) : -INFINITY;
      }
    }
    {
      float mx0 = fmaxf(fmaxf(sc[0][0], sc[0][2]), fmaxf(sc[1][0], sc[1][2]));
      float mx1 = fmaxf(fmaxf(sc[0][1], sc[0][3]), fmaxf(sc[1][1], sc[1][3]));
#pragma unroll
      for (int o = 4; o <= 16; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      if (g == 0) *reinterpret_cast<float2*>(&sm.mw[warp][2 * t]) = make_float2(mx0, mx1);
    }
    if (__syncthreads_or(!ok)) {  // a copy did not complete in time (the whole CTA stops here)
      failed_at = it;
      break;
    }
    // every warp is past the value product of group it - 1: its stage may be refilled
    if (threadIdx.x == 0 && issued < ngroups && issued == it + kCoopStages - 1) {
      fence_proxy_async_smem();
      issue_group<kMeta>(p, sm, issued % kCoopStages, rec_base, b, kvh, w0 + kCoop * issued,
                  min(kCoop, w1 - w0 - kCoop * issued), wait_win, wait_val);
      ++issued;
    }

    // ---- common running max; rescale when it grows ------------------------
    {
      float mn0 = m_run[0], mn1 = m_run[1];
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float2 x = *reinterpret_cast<const float2*>(&sm.mw[w][2 * t]);
        mn0 = fmaxf(mn0, x.x);
        mn1 = fmaxf(mn1, x.y);
      }
      if (__any_sync(0xffffffffu, mn0 > m_run[0] || mn1 > m_run[1])) {
        const float a0 = fast_exp2((m_run[0] - mn0) * kLog2e), a1 = fast_exp2((m_run[1] - mn1) * kLog2e);
        l_part[0] *= a0;
        l_part[1] *= a1;
#pragma unroll
        for (int k = 0; k < kMods; ++k) {
          S_part[k][0] *= a0;
          S_part[k][1] *= a1;
        }
        pv_scale(pv, a0, a1);
        m_run[0] = mn0;
        m_run[1] = mn1;
      }
    }
    const float ms0 = m_run[0] * kLog2e, ms1 = m_run[1] * kLog2e;

    // ---- this warp's window: p, the sums, the value-product B operand --------
    if (have) {
      const __half* sig = reinterpret_cast<const __half*>(rec + L::sigma);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float p0 = fast_exp2(fmaf(sc[h][0], kLog2e, -ms0));
        const float p1 = fast_exp2(fmaf(sc[h][1], kLog2e, -ms1));
        const float p2 = fast_exp2(fmaf(sc[h][2], kLog2e, -ms0));
        const float p3 = fast_exp2(fmaf(sc[h][3], kLog2e, -ms1));
        l_part[0] += p0 + p2;
        l_part[1] += p1 + p3;
        const float sgA = __half2float(sig[tokA[h]]), sgB = __half2float(sig[tokB[h]]);
        const float w0v = p0 * sgA, w1v = p1 * sgA, w2v = p2 * sgB, w3v = p3 * sgB;
        uint32_t bv0[4], bv1[4];  // per plane {hi b0, hi b1, lo b0, lo b1}, transposed
        split_pair_t(w0v * kV0, w1v * kV0, bv0[0], bv0[2]);
        split_pair_t(w2v * kV0, w3v * kV0, bv0[1], bv0[3]);
        split_pair_t(w0v * kV1, w1v * kV1, bv1[0], bv1[2]);
        split_pair_t(w2v * kV1, w3v * kV1, bv1[1], bv1[3]);
        sm.u.c.pfrag[warp][h][0][lane] = make_uint4(bv0[0], bv0[1], bv0[2], bv0[3]);
        sm.u.c.pfrag[warp][h][1][lane] = make_uint4(bv1[0], bv1[1], bv1[2], bv1[3]);
        const int mA = min((int)mods[tokA[h]], kMods - 1), mB = min((int)mods[tokB[h]], kMods - 1);
#pragma unroll
        for (int k = 0; k < kMods; ++k) {
          S_part[k][0] += (mA == k ? w0v : 0.0f) + (mB == k ? w2v : 0.0f);
          S_part[k][1] += (mA == k ? w1v : 0.0f) + (mB == k ? w3v : 0.0f);
        }
        const uint32_t tm = __reduce_or_sync(0xffffffffu, (1u << mA) | (1u << mB));
        if (lane == 0) sm.tmask[warp][h] = tm;
      }
    } else if (lane == 0) {
      sm.tmask[warp][0] = 0u;
      sm.tmask[warp][1] = 0u;
    }
    __syncthreads();

    // ---- value product of the group for this warp's 32 channels -------------
#pragma unroll 1
    for (int ww = 0; ww < kCoop; ++ww) {
      const uint8_t* rv = stg + ww * L::bytes + L::v;
#pragma unroll 1  // rolled: half the code (3 % faster at batch 1 and 2 than unrolled)
      for (int h = 0; h < 2; ++h) {
        const uint32_t tm = sm.tmask[ww][h];
        if (tm == 0u) continue;  // no window (the group's tail)
        const uint4 u = *reinterpret_cast<const uint4*>(rv + 4 * (h * kHeadDim + 32 * warp + 4 * g));
        const uint4 f0 = sm.u.c.pfrag[ww][h][0][lane], f1 = sm.u.c.pfrag[ww][h][1][lane];
        uint32_t a0[2][4], a1[2][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const uint32_t wg = mt ? u.z : u.x, wg8 = mt ? u.w : u.y;
          const uint32_t r[4] = {rotl(wg, rlo), rotl(wg8, rlo), rotl(wg, rhi), rotl(wg8, rhi)};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            a0[mt][j] = r[j] & kPlane0;
            a1[mt][j] = r[j] & kPlane1;
          }
        }
        if ((tm & (tm - 1u)) == 0u) {  // one modality (the common case)
          pv_activate(pv, __ffs(tm) - 1);
          pv_tile(pv, a0, a1, f0, f1, 0xFFFFFFFFu, 0xFFFFFFFFu);
        } else {  // masked products, one per modality present, the active one first
          const uint8_t* md = stg + kCoop * L::bytes + ww * kWindow + 16 * h;
          // k-slots of this lane's B registers: 2t, 2t+1 -> tokens t, t+8; 2t+8, 2t+9 -> t+4, t+12
          const int mk0 = min((int)md[t], kMods - 1), mk1 = min((int)md[t + 8], kMods - 1);
          const int mk2 = min((int)md[t + 4], kMods - 1), mk3 = min((int)md[t + 12], kMods - 1);
          uint32_t todo = tm;
          int mm = (pv.cur >= 0 && ((todo >> pv.cur) & 1u)) ? pv.cur : __ffs(todo) - 1;
#pragma unroll 1
          while (true) {
            pv_activate(pv, mm);
            const uint32_t m01 = (mk0 == mm ? 0x0000FFFFu : 0u) | (mk1 == mm ? 0xFFFF0000u : 0u);
            const uint32_t m23 = (mk2 == mm ? 0x0000FFFFu : 0u) | (mk3 == mm ? 0xFFFF0000u : 0u);
            pv_tile(pv, a0, a1, f0, f1, m01, m23);
            todo &= ~(1u << mm);
            if (!todo) break;
            mm = __ffs(todo) - 1;
          }
        }
      }
    }
  }

  if (failed_at >= 0) {
    // a copy did not complete in time: report it, wait (bounded) for the copies
    // still in flight, and leave an empty split
    if (threadIdx.x == 0) {
      set_error(p.error_word, OMNIKV_DEVERR_TIMEOUT);
      for (int j = failed_at; j < issued; ++j) mbar_wait_bounded(&sm.cbar[j % kCoopStages], (j / kCoopStages) & 1, kWaitLimitNs);
    }
    m_run[0] = m_run[1] = -INFINITY;
    l_part[0] = l_part[1] = 0.0f;
#pragma unroll
    for (int k = 0; k < kMods; ++k) S_part[k][0] = S_part[k][1] = 0.0f;
    pv_scale(pv, 0.0f, 0.0f);
  }
  pv_activate(pv, kMods);  // parks the active modality (index kMods: none)

  // ---- sums over the 8 lanes of a column, then over the warps ---------------
#pragma unroll
  for (int o = 4; o <= 16; o <<= 1) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      l_part[j] += __shfl_xor_sync(0xffffffffu, l_part[j], o);
#pragma unroll
      for (int k = 0; k < kMods; ++k) S_part[k][j] += __shfl_xor_sync(0xffffffffu, S_part[k][j], o);
    }
  }
  if (g == 0) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      sm.red[warp][0][2 * t + j] = l_part[j];
#pragma unroll
      for (int k = 0; k < kMods; ++k) sm.red[warp][1 + k][2 * t + j] = S_part[k][j];
    }
  }
  __syncthreads();
  float Lsum[2], Ssum[kMods][2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    Lsum[j] = 0.0f;
#pragma unroll
    for (int k = 0; k < kMods; ++k) Ssum[k][j] = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      Lsum[j] += sm.red[w][0][2 * t + j];
#pragma unroll
      for (int k = 0; k < kMods; ++k) Ssum[k][j] += sm.red[w][1 + k][2 * t + j];
    }
  }
  // ---- this warp's channels of the split partial, per query head ------------
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int hh = 2 * t + j;
    if (hh >= G) continue;
    Partial* out = p.partials + ((size_t)b * Hq + kvh * G + hh) * p.num_splits + split;
    bool fin = true;
#pragma unroll
    for (int k = 0; k < kMods; ++k)
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const float c0 = vc0 * Ssum[k][j];
        const float2 v = make_float2(pv.st[k][mt][j] + c0, pv.st[k][mt][j + 2] + c0);
        *reinterpret_cast<float2*>(&out->acc[k][32 * warp + 4 * g + 2 * mt]) = v;
        fin = fin && isfinite(v.x) && isfinite(v.y);
      }
    if (!fin) atomicOr(&sm.bad_heads, 1u << hh);
  }
  __syncthreads();
  if (warp == 0 && g == 0) {
#pragma unroll
    for (int j = 0; j < 2; ++j)
      if (2 * t + j < G) write_split_ml(p, sm, b, kvh, 2 * t + j, split, m_run[j], Lsum[j]);
  }
}

// Score B operand for lane (g, t), chunk kc, plane P: k-slots 2t, 2t+1 hold
// channels 32t + kc and 32t + kc + 8, k-slots 2t+8, 2t+9 hold 32t + 16 + kc and
// 32t + 24 + kc; column g is query head g. Entry {hi(slots 2t..), hi(slots
// 2t+8..), lo(..), lo(..)} with lo = fp16(y - hi).
__device__ __forceinline__ void build_score_operand(DecodeSmem& sm, float k0scale, float k1scale) {
  const float* qflat = &sm.q[0][0];
  for (int e = threadIdx.x; e < 8 * 2 * 32; e += kThreads) {
    const int lane = e & 31, P = (e >> 5) & 1, kc = e >> 6;
    const int g = lane >> 2, t = lane & 3;
    const float sc = P == 0 ? k0scale : k1scale;
    float y[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) y[j] = qflat[qpos(g, 32 * t + kc + 8 * j)] * sc;
    const __half2 h01 = __floats2half2_rn(y[0], y[1]);
    const __half2 h23 = __floats2half2_rn(y[2], y[3]);
    const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
    const __half2 l01 = __floats2half2_rn(y[0] - f01.x, y[1] - f01.y);
    const __half2 l23 = __floats2half2_rn(y[2] - f23.x, y[3] - f23.y);
    sm.btab[kc][P][lane] = make_uint4(*reinterpret_cast<const uint32_t*>(&h01), *reinterpret_cast<const uint32_t*>(&h23),
                                      *reinterpret_cast<const uint32_t*>(&l01), *reinterpret_cast<const uint32_t*>(&l23));
  }
}

// ---------------------------------------------------------------------------
// tensor-core path for 4-bit caches over codeword tables: the per-warp table body
// ---------------------------------------------------------------------------
// A 16-level codebook is not linear in its code bits, so the codewords come from
// shared-memory tables, and the codebook needs no symmetry: each codeword is held
// as an fp16 high and low part, hi = fp16(x), lo = fp16(x - hi), which carry x to
// ~22 bits (keys: c_j - c_0, values: c_j). The window's key scales move from the A
// to the B operand of the scores: B = q'_c s_gc 2^-E_w, with a per-window power of
// two keeping it inside fp16, also as a high + low pair. Each product is
// A_hi B_hi + A_hi B_lo + A_lo B_hi (A_lo B_lo is below 2^-22 of it), accumulated in
// fp32: 3 MMAs per 16 x 16 x 8 tile; a register's two k-slots come from one code
// byte. Tokens are in natural order within a 16-token tile (score row r = value
// k-slot r = token r), channels in natural order within a 16-channel chunk.
// (The same tables serve 2-bit codes in a register per code nibble, but there the
// bit-plane bodies above are faster: 235.5 against 200.7 us per layer on the
// 8 x 65,536-token decode.)
constexpr int kLutRing = 9408;  // per-warp record ring: 2 windows of K4/V4 with fp16 metadata

template <int kMeta>
struct RecLut {
  static constexpr int meta = 2048;                       // key codes: 32 tokens x 128 channels x 4 bits
  static constexpr int v = meta + meta_bytes_of(kMeta);
  static constexpr int sigma = v + 2048;                  // value codes
  static constexpr int bytes = sigma + 64;
  static constexpr int stage = bytes + kWindow;           // record + modality ids
  static constexpr int stages = kLutRing / stage;
  static_assert(stage % 16 == 0 && stages >= 2, "ring of 16-byte aligned stages");
};

struct __align__(16) DecodeSmemLut {
  uint8_t ring[kWarps][kLutRing];  // per-warp record rings; also the final merge buffer
  float qlane[32][36];  // lane (g, t): q' of head g at channels 16kc + 2t + {0, 1, 8, 9}, kc-major (rows padded)
  float q[kMaxGroup][kHeadDim];                   // rotated queries (qpos layout), softmax scale folded in
  uint32_t klut[16], vlut[16];                    // tables: fp16 hi | lo << 16 of each codeword
  uint64_t bar[kWarps][2];
  float mw[kWarps][kMaxGroup];
  float lw[kWarps][kMaxGroup];
  alignas(16) uint32_t mxpairs[kWarps][kHeadDim]; // MXFP4 caches: a warp's window metadata as fp16 (m, s) pairs
  float qmax;                                     // max |q'| over the CTA's heads
  uint32_t tmem_base;
  uint32_t bad_heads;
  int wabort[kWarps];
};
static_assert(offsetof(DecodeSmemLut, qlane) % 16 == 0 && offsetof(DecodeSmemLut, mxpairs) % 16 == 0 &&
                  offsetof(DecodeSmemLut, bar) % 8 == 0 && kLutRing % 16 == 0, "aligned fields");
static_assert(kWarps * 32 * 32 * 4 <= kWarps * kLutRing, "merge buffer");
static_assert(sizeof(WindowSmem) <= sizeof(DecodeSmemLut), "append uses the decode shared memory");
static_assert(RecLut<kMetaFp16>::stages == 2 && RecLut<kMetaMx>::stages == 2 && RecLut<kMetaTurbo>::stages == 2,
              "barriers per warp");

// The A operand registers of byte `t` of a code word (two codes: the even k-slot in
// the low nibble): hi and lo parts from the table.
__device__ __forceinline__ void lut4_a(const uint32_t* lut, uint32_t w, int t, uint32_t& hi, uint32_t& lo) {
  const uint32_t byte = (w >> (8 * t)) & 0xFFu;
  const uint32_t e0 = lut[byte & 15u], e1 = lut[byte >> 4];
  hi = __byte_perm(e0, e1, 0x5410);
  lo = __byte_perm(e0, e1, 0x7632);
}

template <int kMeta>
__device__ __forceinline__ void issue_window_lut(const DecodeParams& p, DecodeSmemLut& sm, int warp, int stage,
                                                 const uint8_t* rec_base, int b, int kvh, int wi, int wait_win,
                                                 int wait_val) {
  using L = RecLut<kMeta>;
  uint64_t* bar = &sm.bar[warp][stage];
  if (wi == wait_win &&
      !wait_flag(p.step_flags + (size_t)b * p.num_kv_heads + kvh, wait_val, p.flag_wait_ns)) {
    set_error(p.error_word, OMNIKV_DEVERR_TIMEOUT);  // no copy of a stale record; the split is written empty
    sm.wabort[warp] = 1;
    mbar_arrive_expect_tx(bar, 0);
    return;
  }
  uint8_t* dst = &sm.ring[warp][stage * L::stage];
  mbar_arrive_expect_tx(bar, L::bytes + kWindow);
  bulk_copy_g2s(dst, rec_base + (size_t)wi * L::bytes, L::bytes, bar);
  bulk_copy_g2s(dst + L::bytes, p.modality + (size_t)b * p.cap_tokens + (size_t)wi * kWindow, kWindow, bar);
}

template <int kMeta>
__device__ void decode_mma_lut(const DecodeParams& p, DecodeSmemLut& sm, int b, int kvh, int split, uint32_t tbase) {
  using L = RecLut<kMeta>;
  constexpr int kSt = L::stages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int G = p.group;
  const int Hq = p.num_kv_heads * G;
  int T, w0, w1;
  split_range(p, b, split, T, w0, w1);
  const uint8_t* rec_base = p.records + ((size_t)(b * p.num_kv_heads + kvh) * p.cap_windows) * L::bytes;
  int wa, we, wait_win, wait_val;
  warp_windows(w0, w1, warp, wa, we);
  step_window(p, b, wait_win, wait_val);
  const int nmine = we - wa;
  if (lane == 0) {
    sm.wabort[warp] = 0;
#pragma unroll
    for (int s = 0; s < kSt; ++s) mbar_init(&sm.bar[warp][s], 1);
    fence_barrier_init();
    for (int i = 0; i < kSt && i < nmine; ++i)
      issue_window_lut<kMeta>(p, sm, warp, i, rec_base, b, kvh, wa + i, wait_win, wait_val);
  }
  __syncwarp();

  WarpState st;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    st.m[j] = -INFINITY;
    st.l[j] = 0.0f;
#pragma unroll
    for (int m = 0; m < kMods; ++m) st.mref[m][j] = -INFINITY;
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int r = 0; r < 4; ++r) st.acc[mt][r] = 0.0f;
  st.cur = -1;
  st.parked = 0;
  const float qmax = sm.qmax;
  // TurboQuant keys (k'_tc = ksigma_t c_j): the score operand is q' alone, the same
  // for every window, built here once; each score is its token's ksigma times the sum
  uint32_t bqt[8][4];
  float esct = 1.0f;
  if constexpr (kMeta == kMetaTurbo) {
    int E = 0;
    if (qmax > 0.0f && isfinite(qmax)) E = max(-100, min(100, (int)ceilf(log2f(qmax / 16384.0f))));
    const float bscale = ldexpf(1.0f, -E);
    esct = ldexpf(1.0f, E);
    const float4* ql = reinterpret_cast<const float4*>(&sm.qlane[lane][0]);
#pragma unroll
    for (int kc = 0; kc < 8; ++kc) {
      const float4 q4 = ql[kc];
      const float x0 = q4.x * bscale, x1 = q4.y * bscale, x2 = q4.z * bscale, x3 = q4.w * bscale;
      const __half2 h01 = __floats2half2_rn(x0, x1), h23 = __floats2half2_rn(x2, x3);
      const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
      const __half2 l01 = __floats2half2_rn(x0 - f01.x, x1 - f01.y), l23 = __floats2half2_rn(x2 - f23.x, x3 - f23.y);
      bqt[kc][0] = *reinterpret_cast<const uint32_t*>(&h01);
      bqt[kc][1] = *reinterpret_cast<const uint32_t*>(&h23);
      bqt[kc][2] = *reinterpret_cast<const uint32_t*>(&l01);
      bqt[kc][3] = *reinterpret_cast<const uint32_t*>(&l23);
    }
  }

  int failed_at = -1;
  for (int i = 0; i < nmine; ++i) {
    const int s = i % kSt;
    const int wi = wa + i;
    const bool ok = mbar_wait_bounded(&sm.bar[warp][s], (i / kSt) & 1, kWaitLimitNs) &&
                    *reinterpret_cast<volatile int*>(&sm.wabort[warp]) == 0;
    if (!__all_sync(0xffffffffu, ok)) {
      failed_at = i;
      break;
    }
    const uint8_t* stg = &sm.ring[warp][s * L::stage];
    const uint32_t* kw = reinterpret_cast<const uint32_t*>(stg);
    const uint32_t* vw = reinterpret_cast<const uint32_t*>(stg + L::v);
    const __half* sig = reinterpret_cast<const __half*>(stg + L::sigma);
    const uint8_t* mods = stg + L::bytes;
    const __half* ksig = reinterpret_cast<const __half*>(stg + L::meta);  // TurboQuant keys: per-token scales
    uint32_t bq[8][4];  // per chunk: {hi (2t, 2t+1), hi (8+2t, 9+2t), lo (2t, 2t+1), lo (8+2t, 9+2t)}
    float off0 = 0.0f, off1 = 0.0f, escale = esct;
    if constexpr (kMeta == kMetaTurbo) {
#pragma unroll
      for (int kc = 0; kc < 8; ++kc)
#pragma unroll
        for (int r = 0; r < 4; ++r) bq[kc][r] = bqt[kc][r];
    } else {
      const __half2* meta;
      if constexpr (kMeta == kMetaMx) {
        mx_window_pairs(stg + L::meta, sm.mxpairs[warp], lane);
        meta = reinterpret_cast<const __half2*>(sm.mxpairs[warp]);
      } else {
        meta = reinterpret_cast<const __half2*>(stg + L::meta);
      }

      // ---- the window's score operand: q'_c s_c 2^-E (hi, lo) at this lane's
      // B-fragment channels 16kc + 2t + {0, 1, 8, 9}, and the offset sum_c q'_c m_c
      float qs[32];
      float off = 0.0f, smax = 0.0f;
      {
        const float4* ql = reinterpret_cast<const float4*>(&sm.qlane[lane][0]);
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {
          const float4 q4 = ql[kc];
          const uint2 ma = *reinterpret_cast<const uint2*>(meta + 16 * kc + 2 * t);      // channels 2t, 2t+1
          const uint2 mb = *reinterpret_cast<const uint2*>(meta + 16 * kc + 8 + 2 * t);  // channels 8+2t, 9+2t
          const float2 p0 = __half22float2(*reinterpret_cast<const __half2*>(&ma.x));
          const float2 p1 = __half22float2(*reinterpret_cast<const __half2*>(&ma.y));
          const float2 p2 = __half22float2(*reinterpret_cast<const __half2*>(&mb.x));
          const float2 p3 = __half22float2(*reinterpret_cast<const __half2*>(&mb.y));
          off = fmaf(q4.x, p0.x, off);
          off = fmaf(q4.y, p1.x, off);
          off = fmaf(q4.z, p2.x, off);
          off = fmaf(q4.w, p3.x, off);
          smax = fmaxf(smax, fmaxf(fmaxf(fabsf(p0.y), fabsf(p1.y)), fmaxf(fabsf(p2.y), fabsf(p3.y))));
          qs[4 * kc + 0] = q4.x * p0.y;
          qs[4 * kc + 1] = q4.y * p1.y;
          qs[4 * kc + 2] = q4.z * p2.y;
          qs[4 * kc + 3] = q4.w * p3.y;
        }
        off += __shfl_xor_sync(0xffffffffu, off, 1);
        off += __shfl_xor_sync(0xffffffffu, off, 2);
        smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, 1));
        smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, 2));
      }
      off0 = __shfl_sync(0xffffffffu, off, 8 * t);      // head 2t
      off1 = __shfl_sync(0xffffffffu, off, 8 * t + 4);  // head 2t + 1
      // the largest |B| entry at most 2^14
      const float bmax = qmax * smax;
      int E = 0;
      if (bmax > 0.0f && isfinite(bmax)) E = max(-100, min(100, (int)ceilf(log2f(bmax / 16384.0f))));
      const float bscale = ldexpf(1.0f, -E);
      escale = ldexpf(1.0f, E);
#pragma unroll
      for (int kc = 0; kc < 8; ++kc) {
        const float x0 = qs[4 * kc] * bscale, x1 = qs[4 * kc + 1] * bscale;
        const float x2 = qs[4 * kc + 2] * bscale, x3 = qs[4 * kc + 3] * bscale;
        const __half2 h01 = __floats2half2_rn(x0, x1), h23 = __floats2half2_rn(x2, x3);
        const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
        const __half2 l01 = __floats2half2_rn(x0 - f01.x, x1 - f01.y), l23 = __floats2half2_rn(x2 - f23.x, x3 - f23.y);
        bq[kc][0] = *reinterpret_cast<const uint32_t*>(&h01);
        bq[kc][1] = *reinterpret_cast<const uint32_t*>(&h23);
        bq[kc][2] = *reinterpret_cast<const uint32_t*>(&l01);
        bq[kc][3] = *reinterpret_cast<const uint32_t*>(&l23);
      }
    }

    // ---- scores of the two 16-token tiles: rows g, g + 8 = tokens 16h + g, 16h + g + 8
    // (the tile loops stay rolled: unrolled, the window's code outgrows the
    // instruction cache -- 10 % slower, instruction-fetch stalls 0.89 per issue)
    float sc[2][4];
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
      const int tokA = 16 * h + g, tokB = tokA + 8;
      float d[4] = {0.f, 0.f, 0.f, 0.f}, e[4] = {0.f, 0.f, 0.f, 0.f};
      const uint4* ka = reinterpret_cast<const uint4*>(kw + tokA * 16);
      const uint4* kb = reinterpret_cast<const uint4*>(kw + tokB * 16);
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const uint4 wa4 = ka[q4], wb4 = kb[q4];  // words 4 q4 .. 4 q4 + 3: chunks 2 q4, 2 q4 + 1
        const uint32_t wa[4] = {wa4.x, wa4.y, wa4.z, wa4.w}, wb[4] = {wb4.x, wb4.y, wb4.z, wb4.w};
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int kc = 2 * q4 + half;
          uint32_t ahi[4], alo[4];
          lut4_a(sm.klut, wa[2 * half], t, ahi[0], alo[0]);      // row g, k-slots 2t, 2t+1
          lut4_a(sm.klut, wb[2 * half], t, ahi[1], alo[1]);      // row g + 8
          lut4_a(sm.klut, wa[2 * half + 1], t, ahi[2], alo[2]);  // row g, k-slots 2t+8, 2t+9
          lut4_a(sm.klut, wb[2 * half + 1], t, ahi[3], alo[3]);  // row g + 8
          mma_f16_16816(d, ahi, bq[kc][0], bq[kc][1]);
          mma_f16_16816(e, ahi, bq[kc][2], bq[kc][3]);
          mma_f16_16816(e, alo, bq[kc][0], bq[kc][1]);
        }
      }
      const int posA = wi * kWindow + tokA, posB = wi * kWindow + tokB;
      const float kgA = kMeta == kMetaTurbo ? __half2float(ksig[tokA]) : 1.0f;
      const float kgB = kMeta == kMetaTurbo ? __half2float(ksig[tokB]) : 1.0f;
      const float r0 = posA < T ? kgA * fmaf(d[0] + e[0], escale, off0) : -INFINITY;
      const float r1 = posA < T ? kgA * fmaf(d[1] + e[1], escale, off1) : -INFINITY;
      const float r2 = posB < T ? kgB * fmaf(d[2] + e[2], escale, off0) : -INFINITY;
      const float r3 = posB < T ? kgB * fmaf(d[3] + e[3], escale, off1) : -INFINITY;
      if (h == 0) {
        sc[0][0] = r0; sc[0][1] = r1; sc[0][2] = r2; sc[0][3] = r3;
      } else {
        sc[1][0] = r0; sc[1][1] = r1; sc[1][2] = r2; sc[1][3] = r3;
      }
    }

    // ---- online softmax over the window
    float mx0 = fmaxf(fmaxf(sc[0][0], sc[0][2]), fmaxf(sc[1][0], sc[1][2]));
    float mx1 = fmaxf(fmaxf(sc[0][1], sc[0][3]), fmaxf(sc[1][1], sc[1][3]));
#pragma unroll
    for (int o = 4; o <= 16; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const float mn0 = fmaxf(st.m[0], mx0), mn1 = fmaxf(st.m[1], mx1);
    if (__any_sync(0xffffffffu, mn0 > st.m[0] || mn1 > st.m[1])) {
      const float a0 = fast_exp2((st.m[0] - mn0) * kLog2e), a1 = fast_exp2((st.m[1] - mn1) * kLog2e);
      st.l[0] *= a0;
      st.l[1] *= a1;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        st.acc[mt][0] *= a0;
        st.acc[mt][1] *= a1;
        st.acc[mt][2] *= a0;
        st.acc[mt][3] *= a1;
      }
      st.m[0] = mn0;
      st.m[1] = mn1;
    }
    const float ms0 = st.m[0] * kLog2e, ms1 = st.m[1] * kLog2e;

    // ---- value product per tile: rows g, g + 8 of m-tile mt = channels 16g + 2mt,
    // 16g + 2mt + 1; k-slots 2t, 2t+1 (2t+8, 2t+9) = tokens 16h + 2t, +1 (+8)
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
      const int tokA = 16 * h + g, tokB = tokA + 8;
      const float p0 = fast_exp2(fmaf(h ? sc[1][0] : sc[0][0], kLog2e, -ms0));
      const float p1 = fast_exp2(fmaf(h ? sc[1][1] : sc[0][1], kLog2e, -ms1));
      const float p2 = fast_exp2(fmaf(h ? sc[1][2] : sc[0][2], kLog2e, -ms0));
      const float p3 = fast_exp2(fmaf(h ? sc[1][3] : sc[0][3], kLog2e, -ms1));
      st.l[0] += p0 + p2;
      st.l[1] += p1 + p3;
      const float sgA = __half2float(sig[tokA]), sgB = __half2float(sig[tokB]);
      uint32_t bv[4];  // {hi (k 0..7), hi (k 8..15), lo (k 0..7), lo (k 8..15)}, transposed
      split_pair_t(p0 * sgA, p1 * sgA, bv[0], bv[2]);
      split_pair_t(p2 * sgB, p3 * sgB, bv[1], bv[3]);
      const int mA = min((int)mods[tokA], 2), mB = min((int)mods[tokB], 2);
      const uint32_t mbits = __reduce_or_sync(0xffffffffu, (1u << mA) | (1u << mB));
      const int base = 16 * h;
      const int mk0 = min((int)mods[base + 2 * t], 2), mk1 = min((int)mods[base + 2 * t + 1], 2);
      const int mk2 = min((int)mods[base + 8 + 2 * t], 2), mk3 = min((int)mods[base + 9 + 2 * t], 2);
      uint32_t todo = mbits;
      int mm = (st.cur >= 0 && ((todo >> st.cur) & 1u)) ? st.cur : __ffs(todo) - 1;
#pragma unroll 1
      while (true) {
        activate(st, mm, tbase, warp);
        const bool single = mbits == (1u << mm);
        const uint32_t msk01 = single ? 0xFFFFFFFFu : ((mk0 == mm ? 0x0000FFFFu : 0u) | (mk1 == mm ? 0xFFFF0000u : 0u));
        const uint32_t msk23 = single ? 0xFFFFFFFFu : ((mk2 == mm ? 0x0000FFFFu : 0u) | (mk3 == mm ? 0xFFFF0000u : 0u));
        const uint32_t bh0 = bv[0] & msk01, bh1 = bv[1] & msk23, bl0 = bv[2] & msk01, bl1 = bv[3] & msk23;
        const uint4* r0 = reinterpret_cast<const uint4*>(vw + (2 * h) * kHeadDim + 16 * g);      // tokens 16h .. +7
        const uint4* r1 = reinterpret_cast<const uint4*>(vw + (2 * h + 1) * kHeadDim + 16 * g);  // tokens 16h+8 .. +15
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint4 u0w = r0[q4], u1w = r1[q4];  // channels 16g + 4 q4 .. + 3
          const uint32_t x0[4] = {u0w.x, u0w.y, u0w.z, u0w.w}, x1[4] = {u1w.x, u1w.y, u1w.z, u1w.w};
#pragma unroll
          for (int e2 = 0; e2 < 2; ++e2) {
            const int mt = 2 * q4 + e2;
            uint32_t ahi[4], alo[4];
            lut4_a(sm.vlut, x0[2 * e2], t, ahi[0], alo[0]);      // channel 16g + 2mt, tokens 2t, 2t+1
            lut4_a(sm.vlut, x0[2 * e2 + 1], t, ahi[1], alo[1]);  // channel 16g + 2mt + 1
            lut4_a(sm.vlut, x1[2 * e2], t, ahi[2], alo[2]);      // channel 16g + 2mt, tokens 8+2t, 9+2t
            lut4_a(sm.vlut, x1[2 * e2 + 1], t, ahi[3], alo[3]);
            mma_f16_16816(st.acc[mt], ahi, bh0, bh1);
            mma_f16_16816(st.acc[mt], ahi, bl0, bl1);
            mma_f16_16816(st.acc[mt], alo, bh0, bh1);
          }
        }
        todo &= ~(1u << mm);
        if (!todo) break;
        mm = __ffs(todo) - 1;
      }
    }
    __syncwarp();
    if (lane == 0 && i + kSt < nmine) {
      fence_proxy_async_smem();
      issue_window_lut<kMeta>(p, sm, warp, s, rec_base, b, kvh, wa + i + kSt, wait_win, wait_val);
    }
  }

  if (__any_sync(0xffffffffu, failed_at >= 0)) {
    const int f = __shfl_sync(0xffffffffu, failed_at, 0);
    if (lane == 0) set_error(p.error_word, OMNIKV_DEVERR_TIMEOUT);
    for (int j = f; j < nmine && j < f + kSt; ++j)
      mbar_wait_bounded(&sm.bar[warp][j % kSt], (j / kSt) & 1, kWaitLimitNs);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      st.m[j] = -INFINITY;
      st.l[j] = 0.0f;
    }
    st.cur = -1;
    st.parked = 0;
  }
  if (st.cur >= 0) park_active(st, tbase, warp);

  // ---- reduce the per-lane denominators over the 8 lanes sharing a column
#pragma unroll
  for (int o = 4; o <= 16; o <<= 1) {
#pragma unroll
    for (int j = 0; j < 2; ++j) st.l[j] += __shfl_xor_sync(0xffffffffu, st.l[j], o);
  }
  // ---- merge the 4 warps at their common max, one modality at a time
  if (g == 0) {
    sm.mw[warp][2 * t] = st.m[0];
    sm.mw[warp][2 * t + 1] = st.m[1];
  }
  __syncthreads();  // also: all warps are done with their rings
  float M[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) mm = fmaxf(mm, sm.mw[w][2 * t + j]);
    M[j] = mm;
    const float f = (st.m[j] == -INFINITY) ? 0.0f : fast_exp2((st.m[j] - mm) * kLog2e);
    st.l[j] *= f;
  }
  if (g == 0) {
    sm.lw[warp][2 * t] = st.l[0];
    sm.lw[warp][2 * t + 1] = st.l[1];
  }
  float* xbuf = reinterpret_cast<float*>(&sm.ring[0][0]);  // [warp][32 registers][32 lanes]
#pragma unroll
  for (int m = 0; m < kMods; ++m) {
    unpark(st, m, tbase, warp, M[0], M[1]);  // zeros if this warp never saw modality m
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int r = 0; r < 4; ++r) xbuf[(warp * 32 + mt * 4 + r) * 32 + lane] = st.acc[mt][r];
    __syncthreads();
#pragma unroll
    for (int e2 = 0; e2 < 2; ++e2) {
      const int mt = 2 * warp + e2;
      float v[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        float x = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) x += xbuf[(w * 32 + mt * 4 + r) * 32 + lane];
        v[r] = x;
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int hh = 2 * t + j;
        if (hh >= G) continue;
        Partial* out = p.partials + ((size_t)b * Hq + kvh * G + hh) * p.num_splits + split;
        *reinterpret_cast<float2*>(&out->acc[m][16 * g + 2 * mt]) = make_float2(v[j], v[j + 2]);
        if (!isfinite(v[j]) || !isfinite(v[j + 2])) atomicOr(&sm.bad_heads, 1u << hh);
      }
    }
    __syncthreads();
  }
  if (warp == 0 && g == 0) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int hh = 2 * t + j;
      if (hh >= G) continue;
      float l = 0.0f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) l += sm.lw[w][hh];
      write_split_ml(p, sm, b, kvh, hh, split, M[j], l);
    }
  }
}

__device__ __forceinline__ uint32_t half_pair_bits(float x, uint32_t& lo) {
  const __half h = __float2half_rn(x);
  lo = __half_as_ushort(__float2half_rn(x - __half2float(h)));
  return __half_as_ushort(h);
}

// One decode CTA of the table body.
template <int kMeta>
__device__ __forceinline__ void decode_cta_lut(const DecodeParams& p, DecodeSmemLut& sm, int b, int kvh, int split) {
  {
    const size_t ubytes = (size_t)kMods * kHeadDim * kHeadDim * sizeof(float);
    const size_t share = (ubytes + p.num_splits - 1) / p.num_splits;
    const char* ub = reinterpret_cast<const char*>(p.value_rot) + (size_t)kvh * ubytes;
    for (size_t off = (size_t)split * share + 128 * threadIdx.x; off < min(ubytes, (size_t)(split + 1) * share);
         off += 128 * kThreads)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(ub + off));
  }
  rotate_queries(p, b, kvh, &sm.q[0][0]);
  if (threadIdx.x < 16) {  // codeword tables: c_j - c_0 (keys; c_j for TurboQuant keys), c_j (values)
    const int j = threadIdx.x;
    uint32_t lk, lv;
    const uint32_t hk = half_pair_bits(kMeta == kMetaTurbo ? p.key_cb[j] : p.key_cb[j] - p.key_cb[0], lk);
    const uint32_t hv = half_pair_bits(p.val_cb[j], lv);
    sm.klut[j] = hk | (lk << 16);
    sm.vlut[j] = hv | (lv << 16);
  }
  if (threadIdx.x == 0) sm.bad_heads = 0u;
  __syncthreads();  // every warp's rotated queries are written
  {
    float qm = 0.0f;
    for (int e = threadIdx.x; e < kMaxGroup * kHeadDim; e += kThreads) qm = fmaxf(qm, fabsf((&sm.q[0][0])[e]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) qm = fmaxf(qm, __shfl_xor_sync(0xffffffffu, qm, o));
    if ((threadIdx.x & 31) == 0) sm.lw[threadIdx.x >> 5][0] = qm;
    // the lanes' B-fragment copy of the queries: lane (g, t), chunk kc: channels
    // 16kc + 2t, 16kc + 2t + 1, 16kc + 8 + 2t, 16kc + 9 + 2t of head g
    for (int e = threadIdx.x; e < 32 * 32; e += kThreads) {
      const int ln = e >> 5, j = e & 31;
      const int gg = ln >> 2, tt = ln & 3, kc = j >> 2, r = j & 3;
      sm.qlane[ln][j] = sm.q[0][qpos(gg, 16 * kc + 2 * tt + (r & 1) + 8 * (r >> 1))];
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) sm.qmax = fmaxf(fmaxf(sm.lw[0][0], sm.lw[1][0]), fmaxf(sm.lw[2][0], sm.lw[3][0]));
  __syncthreads();

  griddep_wait();  // lengths and records may come from the previous launch
  int T, w0, w1;
  split_range(p, b, split, T, w0, w1);
  if (w0 == w1) {
    if (threadIdx.x < p.group) {
      Partial* out = p.partials + ((size_t)b * p.num_kv_heads * p.group + kvh * p.group + threadIdx.x) * p.num_splits + split;
      out->m = -INFINITY;
      out->l = 0.0f;
    }
    return;
  }
  if (threadIdx.x < 32) tmem_alloc(&sm.tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;
  decode_mma_lut<kMeta>(p, sm, b, kvh, split, tbase);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x < 32) tmem_dealloc(tbase, kTmemCols);
}

template <int kMeta>
__global__ void __launch_bounds__(kThreads, 2) decode_split_lut_kernel(const DecodeParams p) {
  extern __shared__ __align__(16) uint8_t lut_smem[];
  DecodeSmemLut& sm = *reinterpret_cast<DecodeSmemLut*>(lut_smem);
  griddep_launch_dependents();
  decode_cta_lut<kMeta>(p, sm, blockIdx.z, blockIdx.y, blockIdx.x);
}

template <int kMeta>
__global__ void __launch_bounds__(kThreads, 2) decode_step_lut_kernel(const DecodeParams p, const WriteParams w) {
  extern __shared__ __align__(16) uint8_t lut_smem[];
  DecodeSmemLut& sm = *reinterpret_cast<DecodeSmemLut*>(lut_smem);
  griddep_launch_dependents();
  const int H = p.num_kv_heads;
  const int nappend = p.append_ctas;
  if ((int)blockIdx.x < nappend) {
    griddep_wait();
    for (int u = blockIdx.x; u < p.batch * H; u += nappend) {
      const int b = u / H, h = u % H;
      const int L0 = w.seq_lens[b];
      const int L1 = L0 + 1;
      if (L0 >= 0 && L1 <= w.cap_tokens) {
        quantize_window<kMeta>(w, b, h, L0 / kWindow, L0, L1, *reinterpret_cast<WindowSmem*>(&sm), threadIdx.x, 1,
                               true);
        if (h > 0 && threadIdx.x == 0) {  // the decode of head h reads the token's modality after h's flag
          const int m = w.mod_new[b];
          w.modality[(size_t)b * w.cap_tokens + L0] = (uint8_t)(m >= kMods ? kMods - 1 : m);
        }
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0)
          asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(w.step_flags + (size_t)b * H + h), "r"(L1)
                       : "memory");
      } else if (threadIdx.x == 0 && h == 0) {
        set_error(w.error_word, OMNIKV_DEVERR_CAPACITY);
      }
      __syncthreads();  // the shared memory is the next unit's
    }
    return;
  }
  const int r = blockIdx.x - nappend;
  decode_cta_lut<kMeta>(p, sm, r / (p.num_splits * H), (r / p.num_splits) % H, r % p.num_splits);
}

// One decode CTA: split `split` of kv head kvh of sequence b. kBody: the 4-bit
// build (CUDA-core path only, no TMEM, more CTAs per SM), or a tensor-core build
// (per-warp or cooperative body), whose kernels fall back to the CUDA-core path for
// 2-bit codebooks that are not symmetric. kMeta: the key metadata format the
// tensor-core builds are compiled for (the CUDA-core path reads it at run time).
template <int kBody, int kMeta>
__device__ __forceinline__ void decode_cta(const DecodeParams& p, DecodeSmem& sm, int b, int kvh, int split) {
  constexpr bool kGen = kBody == kBodyGeneric;
  // ---- independent of the cache (overlaps the previous launch of the stream):
  // query rotation, score operand, L2 prefetch of this split's share of the
  // value bases (read by the combine)
  bool fast = false;
  float k0 = 0.f, k1 = 0.f, k2 = 0.f, v0 = 0.f, v1 = 0.f, v2 = 0.f;
  if (!kGen && p.key_bits == 2 && p.value_bits == 2) {
    k0 = p.key_cb[0], k1 = p.key_cb[1], k2 = p.key_cb[2];
    const float k3 = p.key_cb[3];
    v0 = p.val_cb[0], v1 = p.val_cb[1], v2 = p.val_cb[2];
    const float v3 = p.val_cb[3];
    fast = (k0 == -k3) && (k1 == -k2) && (v0 == -v3) && (v1 == -v2);
  }
  {
    const size_t ubytes = (size_t)kMods * kHeadDim * kHeadDim * sizeof(float);
    const size_t share = (ubytes + p.num_splits - 1) / p.num_splits;
    const char* ub = reinterpret_cast<const char*>(p.value_rot) + (size_t)kvh * ubytes;
    for (size_t off = (size_t)split * share + 128 * threadIdx.x; off < min(ubytes, (size_t)(split + 1) * share);
         off += 128 * kThreads)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(ub + off));
  }
  rotate_queries(p, b, kvh, &sm.q[0][0]);
  if (threadIdx.x == 0) sm.bad_heads = 0u;
  __syncthreads();  // every warp's rotated queries are written before they are scanned
  // the score operand carries a power of two 2^-E that keeps its largest entry at
  // most 2^14 (so large queries stay inside the fp16 range); scores are scaled back
  // by 2^E in fp32
  {
    float qm = 0.0f;
    for (int i = threadIdx.x; i < kMaxGroup * kHeadDim; i += kThreads) qm = fmaxf(qm, fabsf((&sm.q[0][0])[i]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) qm = fmaxf(qm, __shfl_xor_sync(0xffffffffu, qm, o));
    if ((threadIdx.x & 31) == 0) sm.lw[threadIdx.x >> 5][0] = qm;
  }
  if constexpr (kMeta == kMetaTurbo) {
    // c_0 sum_c q'_c per head: the codebook's c_0 term of every score (warp w sums
    // the rows of heads w and w + 4, in any channel order)
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    for (int g = w; g < kMaxGroup; g += kWarps) {
      float x = 0.0f;
#pragma unroll
      for (int c = l; c < kHeadDim; c += 32) x += sm.q[g][c];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      if (l == 0) sm.qoff[g] = p.key_cb[0] * x;
    }
  }
  __syncthreads();
  float escale = 1.0f;
  if (fast) {
    const float c0k = (k1 - k0) * 128.0f, c1k = (k2 - k0) * 0.5f;
    const float xmax = fmaxf(fmaxf(sm.lw[0][0], sm.lw[1][0]), fmaxf(sm.lw[2][0], sm.lw[3][0])) *
                       fmaxf(fabsf(c0k), fabsf(c1k));
    int E = 0;
    if (xmax > 0.0f && isfinite(xmax)) E = max(-24, min(100, (int)ceilf(log2f(xmax / 16384.0f))));
    escale = ldexpf(1.0f, E);
    build_score_operand(sm, c0k * ldexpf(1.0f, -E), c1k * ldexpf(1.0f, -E));
  }

  // ---- the cache: lengths and records may come from the previous launch
  griddep_wait();
  int T, w0, w1;
  split_range(p, b, split, T, w0, w1);
  if (w0 == w1) {  // empty split (short sequence): only m and l are read by the combine
    if (threadIdx.x < p.group) {
      Partial* out = p.partials + ((size_t)b * p.num_kv_heads * p.group + kvh * p.group + threadIdx.x) * p.num_splits + split;
      out->m = -INFINITY;
      out->l = 0.0f;
    }
    return;
  }
  if (kBody == kBodyCoop && fast) {
    decode_coop<kMeta>(p, sm, b, kvh, split, (v1 - v0) * 128.0f, (v2 - v0) * 0.5f, v0, escale);
    return;
  }
  if (kBody == kBodyWarp && fast) {
    prime_pipeline<kMeta>(p, sm, b, kvh, w0, w1);
    if (threadIdx.x < 32) tmem_alloc(&sm.tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sm.tmem_base;
    decode_mma<kMeta>(p, sm, b, kvh, split, (v1 - v0) * 128.0f, (v2 - v0) * 0.5f, v0, tbase, escale);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x < 32) tmem_dealloc(tbase, kTmemCols);
    return;
  }
  decode_generic<kGen, SyncCta>(p, *reinterpret_cast<GenSmem*>(&sm.u), &sm.q[0][0], b, kvh, split);
}

// Registers for this many resident CTAs per SM: per-warp body 2 (its accumulators
// need ~240 registers), cooperative body 3, CUDA-core build 4.
__host__ __device__ constexpr int body_ctas_per_sm(int body) {
  return body == kBodyWarp ? 2 : body == kBodyCoop ? 3 : 4;
}

template <int kBody, int kMeta>
__global__ void __launch_bounds__(kThreads, body_ctas_per_sm(kBody)) decode_split_k_kernel(const DecodeParams p) {
  __shared__ DecodeSmem sm;
  griddep_launch_dependents();
  decode_cta<kBody, kMeta>(p, sm, blockIdx.z, blockIdx.y, blockIdx.x);
}

// Decode step: CTAs [0, batch * H) append one token to (sequence, kv head) and
// then publish the new length in the step flag; the others are decode CTAs
// (split fastest, then kv head, then sequence). Only the copy of the window that
// receives the token waits for the flag.
template <int kBody, int kMeta>
__global__ void __launch_bounds__(kThreads, body_ctas_per_sm(kBody))
    decode_step_kernel(const DecodeParams p, const WriteParams w) {
  __shared__ DecodeSmem sm;
  static_assert(sizeof(WindowSmem) <= sizeof(DecodeSmem), "append uses the decode shared memory");
  griddep_launch_dependents();
  const int H = p.num_kv_heads;
  const int nappend = p.append_ctas;
  if ((int)blockIdx.x < nappend) {
    griddep_wait();
    for (int u = blockIdx.x; u < p.batch * H; u += nappend) {
      const int b = u / H, h = u % H;
      const int L0 = w.seq_lens[b];
      const int L1 = L0 + 1;
      if (L0 >= 0 && L1 <= w.cap_tokens) {
        if constexpr (kBody == kBodyGeneric)  // one instance serves every key format
          quantize_window_any(w, b, h, L0 / kWindow, L0, L1, *reinterpret_cast<WindowSmem*>(&sm), threadIdx.x, 1, true);
        else
          quantize_window<kMeta>(w, b, h, L0 / kWindow, L0, L1, *reinterpret_cast<WindowSmem*>(&sm), threadIdx.x, 1,
                                 true);
        if (h > 0 && threadIdx.x == 0) {  // the decode of head h reads the token's modality after h's flag
          const int m = w.mod_new[b];
          w.modality[(size_t)b * w.cap_tokens + L0] = (uint8_t)(m >= kMods ? kMods - 1 : m);
        }
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0)
          asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(w.step_flags + (size_t)b * H + h), "r"(L1)
                       : "memory");
      } else if (threadIdx.x == 0 && h == 0) {
        set_error(w.error_word, OMNIKV_DEVERR_CAPACITY);
      }
      __syncthreads();  // the shared memory is the next unit's
    }
    return;
  }
  const int r = blockIdx.x - nappend;
  decode_cta<kBody, kMeta>(p, sm, r / (p.num_splits * H), (r / p.num_splits) % H, r % p.num_splits);
}

// Several decode CTAs share an SM only if the SM's unified L1 / shared memory is
// split in favour of shared memory; without a preference the runtime may pick a
// split that holds one CTA. Set once per device and kernel (bit d of a mask).
template <typename Kernel>
cudaError_t prefer_shared_carveout(Kernel kernel, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

std::atomic<uint64_t> g_carveout[2][kNumBodies][3];  // [decode, step][body][key metadata format]

// The table body's kernels take their shared memory dynamically (above the 48 KB
// static limit): the attribute and the carveout, set once per device.
template <typename Kernel>
cudaError_t prepare_dynamic(Kernel kernel, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(DecodeSmemLut));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

template <int kMeta>
cudaError_t prepare_lut() {
  const cudaError_t e = prepare_dynamic(decode_split_lut_kernel<kMeta>, g_carveout[0][kBodyLut][kMeta]);
  if (e != cudaSuccess) return e;
  return prepare_dynamic(decode_step_lut_kernel<kMeta>, g_carveout[1][kBodyLut][kMeta]);
}

template <int kBody, int kMeta>
cudaError_t prepare_body() {
  const cudaError_t e = prefer_shared_carveout(decode_split_k_kernel<kBody, kMeta>, g_carveout[0][kBody][kMeta]);
  if (e != cudaSuccess) return e;
  return prefer_shared_carveout(decode_step_kernel<kBody, kMeta>, g_carveout[1][kBody][kMeta]);
}

// The CUDA-core build reads the metadata format at run time: one instance.
cudaError_t prepare_kernels(int body, int meta) {
  if (body == kBodyGeneric) return prepare_body<kBodyGeneric, kMetaFp16>();
  if (body == kBodyLut)
    return meta == kMetaMx ? prepare_lut<kMetaMx>() : meta == kMetaTurbo ? prepare_lut<kMetaTurbo>() : prepare_lut<kMetaFp16>();
  if (meta == kMetaMx) return body == kBodyWarp ? prepare_body<kBodyWarp, kMetaMx>() : prepare_body<kBodyCoop, kMetaMx>();
  if (meta == kMetaTurbo)
    return body == kBodyWarp ? prepare_body<kBodyWarp, kMetaTurbo>() : prepare_body<kBodyCoop, kMetaTurbo>();
  return body == kBodyWarp ? prepare_body<kBodyWarp, kMetaFp16>() : prepare_body<kBodyCoop, kMetaFp16>();
}

template <int kBody, int kMeta>
cudaError_t body_attributes_of(cudaFuncAttributes* a) {
  cudaError_t e = cudaFuncGetAttributes(a, decode_step_kernel<kBody, kMeta>);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes a2;
  e = cudaFuncGetAttributes(&a2, decode_split_k_kernel<kBody, kMeta>);
  if (e != cudaSuccess) return e;
  // size both kernels of the body by the larger register count
  if (a2.numRegs > a->numRegs) a->numRegs = a2.numRegs;
  if (a2.sharedSizeBytes > a->sharedSizeBytes) a->sharedSizeBytes = a2.sharedSizeBytes;
  return cudaSuccess;
}

// Attributes of a body, over every key metadata format (the residency of the largest).
template <int kBody>
cudaError_t body_attributes(cudaFuncAttributes* a) {
  cudaError_t e = body_attributes_of<kBody, kMetaFp16>(a);
  if (e != cudaSuccess || kBody == kBodyGeneric) return e;
  cudaFuncAttributes a2;
  if ((e = body_attributes_of<kBody, kMetaMx>(&a2)) != cudaSuccess) return e;
  if (a2.numRegs > a->numRegs) a->numRegs = a2.numRegs;
  if (a2.sharedSizeBytes > a->sharedSizeBytes) a->sharedSizeBytes = a2.sharedSizeBytes;
  if ((e = body_attributes_of<kBody, kMetaTurbo>(&a2)) != cudaSuccess) return e;
  if (a2.numRegs > a->numRegs) a->numRegs = a2.numRegs;
  if (a2.sharedSizeBytes > a->sharedSizeBytes) a->sharedSizeBytes = a2.sharedSizeBytes;
  return cudaSuccess;
}

template <int kMeta>
cudaError_t lut_attributes_of(cudaFuncAttributes* a) {
  cudaError_t e = cudaFuncGetAttributes(a, decode_step_lut_kernel<kMeta>);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes a2;
  if ((e = cudaFuncGetAttributes(&a2, decode_split_lut_kernel<kMeta>)) != cudaSuccess) return e;
  if (a2.numRegs > a->numRegs) a->numRegs = a2.numRegs;
  if (a2.sharedSizeBytes > a->sharedSizeBytes) a->sharedSizeBytes = a2.sharedSizeBytes;
  a->sharedSizeBytes += sizeof(DecodeSmemLut);
  return cudaSuccess;
}

// Attributes of the table body over every key metadata format.
cudaError_t lut_attributes(cudaFuncAttributes* a) {
  cudaError_t e = lut_attributes_of<kMetaFp16>(a);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes a2;
  if ((e = lut_attributes_of<kMetaMx>(&a2)) != cudaSuccess) return e;
  if (a2.numRegs > a->numRegs) a->numRegs = a2.numRegs;
  if (a2.sharedSizeBytes > a->sharedSizeBytes) a->sharedSizeBytes = a2.sharedSizeBytes;
  if ((e = lut_attributes_of<kMetaTurbo>(&a2)) != cudaSuccess) return e;
  if (a2.numRegs > a->numRegs) a->numRegs = a2.numRegs;
  if (a2.sharedSizeBytes > a->sharedSizeBytes) a->sharedSizeBytes = a2.sharedSizeBytes;
  return cudaSuccess;
}

}  // namespace

int decode_body(int key_bits, int value_bits, int key_meta, int split_windows) {
  if (key_bits == 4 && value_bits == 4) return kBodyLut;
  if (key_bits != 2 || value_bits != 2) return kBodyGeneric;
  return split_windows <= kCoopMaxWindows ? kBodyCoop : kBodyWarp;
}

// Resident decode CTAs per SM of a body, from its kernels' registers and shared
// memory and the TMEM columns each CTA allocates (computed from the attributes
// rather than the runtime occupancy query, which does not report the residency
// seen on sm_100a for these kernels). Cached per device and body.
int decode_ctas_per_sm(int body) {
  static std::atomic<int> cached[kNumBodies][64];
  if (body < 0 || body >= kNumBodies) body = kBodyGeneric;
  const int fallback = body_ctas_per_sm(body);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fallback;
  if (dev < 64) {
    const int c = cached[body][dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  cudaFuncAttributes a;
  int regs_sm = 0, smem_sm = 0, smem_rsv = 0;
  const cudaError_t ea = body == kBodyWarp ? body_attributes<kBodyWarp>(&a)
                       : body == kBodyCoop ? body_attributes<kBodyCoop>(&a)
                       : body == kBodyLut  ? lut_attributes(&a)
                                           : body_attributes<kBodyGeneric>(&a);
  if (prepare_kernels(body, kMetaFp16) != cudaSuccess ||
      (body != kBodyGeneric && prepare_kernels(body, kMetaMx) != cudaSuccess) ||
      (body != kBodyGeneric && prepare_kernels(body, kMetaTurbo) != cudaSuccess) ||
      ea != cudaSuccess ||
      cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_rsv, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
    return fallback;
  const int warp_regs = ((a.numRegs * 32 + 255) / 256) * 256;  // allocated per warp in units of 256
  const int by_regs = regs_sm / (warp_regs * kWarps);
  const int by_smem = smem_sm / ((int)a.sharedSizeBytes + smem_rsv);
  const int by_tmem = (body == kBodyWarp || body == kBodyLut) ? 512 / (int)kTmemCols : 64;  // per-warp bodies hold tensor memory
  const int n = max(1, min(by_regs, min(by_smem, by_tmem)));
  if (dev < 64) cached[body][dev].store(n, std::memory_order_relaxed);
  return n;
}

cudaError_t launch_decode_step(const DecodeParams& p, const WriteParams& w, cudaStream_t stream) {
  const int meta = p.key_meta;
  const int body = decode_body(p.key_bits, p.value_bits, meta, p.split_windows);
  const cudaError_t e = prepare_kernels(body, meta);
  if (e != cudaSuccess) return e;
  const dim3 grid(p.append_ctas + p.batch * p.num_kv_heads * p.num_splits);
  const dim3 block(kThreads);
  constexpr size_t lsm = sizeof(DecodeSmemLut);
  if (body == kBodyLut)
    return meta == kMetaMx      ? launch_pdl(decode_step_lut_kernel<kMetaMx>, grid, block, lsm, stream, p, w)
           : meta == kMetaTurbo ? launch_pdl(decode_step_lut_kernel<kMetaTurbo>, grid, block, lsm, stream, p, w)
                                : launch_pdl(decode_step_lut_kernel<kMetaFp16>, grid, block, lsm, stream, p, w);
  if (body == kBodyGeneric) return launch_pdl(decode_step_kernel<kBodyGeneric, kMetaFp16>, grid, block, 0, stream, p, w);
  if (meta == kMetaMx)
    return body == kBodyWarp ? launch_pdl(decode_step_kernel<kBodyWarp, kMetaMx>, grid, block, 0, stream, p, w)
                             : launch_pdl(decode_step_kernel<kBodyCoop, kMetaMx>, grid, block, 0, stream, p, w);
  if (meta == kMetaTurbo)
    return body == kBodyWarp ? launch_pdl(decode_step_kernel<kBodyWarp, kMetaTurbo>, grid, block, 0, stream, p, w)
                             : launch_pdl(decode_step_kernel<kBodyCoop, kMetaTurbo>, grid, block, 0, stream, p, w);
  return body == kBodyWarp ? launch_pdl(decode_step_kernel<kBodyWarp, kMetaFp16>, grid, block, 0, stream, p, w)
                           : launch_pdl(decode_step_kernel<kBodyCoop, kMetaFp16>, grid, block, 0, stream, p, w);
}

cudaError_t launch_decode(const DecodeParams& p, int batch, cudaStream_t stream) {
  const int meta = p.key_meta;
  const int body = decode_body(p.key_bits, p.value_bits, meta, p.split_windows);
  const cudaError_t e = prepare_kernels(body, meta);
  if (e != cudaSuccess) return e;
  const dim3 grid(p.num_splits, p.num_kv_heads, batch);
  const dim3 block(kThreads);
  constexpr size_t lsm = sizeof(DecodeSmemLut);
  if (body == kBodyLut)
    return meta == kMetaMx      ? launch_pdl(decode_split_lut_kernel<kMetaMx>, grid, block, lsm, stream, p)
           : meta == kMetaTurbo ? launch_pdl(decode_split_lut_kernel<kMetaTurbo>, grid, block, lsm, stream, p)
                                : launch_pdl(decode_split_lut_kernel<kMetaFp16>, grid, block, lsm, stream, p);
  if (body == kBodyGeneric) return launch_pdl(decode_split_k_kernel<kBodyGeneric, kMetaFp16>, grid, block, 0, stream, p);
  if (meta == kMetaMx)
    return body == kBodyWarp ? launch_pdl(decode_split_k_kernel<kBodyWarp, kMetaMx>, grid, block, 0, stream, p)
                             : launch_pdl(decode_split_k_kernel<kBodyCoop, kMetaMx>, grid, block, 0, stream, p);
  if (meta == kMetaTurbo)
    return body == kBodyWarp ? launch_pdl(decode_split_k_kernel<kBodyWarp, kMetaTurbo>, grid, block, 0, stream, p)
                             : launch_pdl(decode_split_k_kernel<kBodyCoop, kMetaTurbo>, grid, block, 0, stream, p);
  return body == kBodyWarp ? launch_pdl(decode_split_k_kernel<kBodyWarp, kMetaFp16>, grid, block, 0, stream, p)
                           : launch_pdl(decode_split_k_kernel<kBodyCoop, kMetaFp16>, grid, block, 0, stream, p);
}

}  // namespace omnikv
