// The per-window body of the OmniKVQuant cache write, shared by the write
// kernels (kv_quant_pack.cu) and the decode-step kernel (decode_split_k.cu).
// See kv_quant_pack.cu for the method and its sources.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace omnikv {
namespace {

constexpr int kWriteThreads = 128;  // one group of 128 threads per (window, kv head)

struct __align__(16) WindowSmem {  // 16-byte multiple: per-group copies stay float4-aligned
  float kp[kWindow][kHeadDim];  // rotated keys, then reused for fp32 values
  float s_min[kHeadDim], s_scale[kHeadDim];
  float s_sigma[kWindow];
  CodeBound bk[15], bv[15];  // code decision bounds (keys: after + c_0; values: none added)
  float tb[kWindow][15];     // TurboQuant keys: each token's bounds scaled by its key scale
  uint8_t codes[kWindow][kHeadDim];  // key codes (token, channel) before packing
};

static_assert(sizeof(WindowSmem) % 16 == 0, "per-group shared memory must keep 16-byte alignment");

// Barrier over the 128 threads of one group (id 0 is __syncthreads).
__device__ __forceinline__ void group_sync(int id) { asm volatile("bar.sync %0, 128;\n" ::"r"(id) : "memory"); }

// Column of channel c of token t in the rotated-key buffer: the 4-float chunks
// of each 32-channel block are XOR-permuted by (t % 2, block), so that the 8
// threads of a quarter warp storing one chunk each (2 tokens x 4 blocks) hit 8
// different bank groups. Readers of a whole row see a permutation of it.
__device__ __forceinline__ int kp_col(int t, int c) {
  const int q = c >> 5, j = (c >> 2) & 7;
  return 32 * q + 4 * (j ^ ((t & 1) | (q << 1))) + (c & 3);
}

// Key codes of the window's valid tokens, code = #{j : (k' - m) / s + c_0 > t_j}
// (0 where s == 0) with window metadata, or code = #{j : k' / ksigma_t > t_j} (0
// where ksigma_t == 0) for TurboQuant keys (scales in s_scale[0..31], bounds built
// without c_0): thread c decides channel c for every token, then the codes are
// packed 32 / BITS per token-major word.
template <int BITS, bool kTurbo>
__device__ __forceinline__ void key_code_words(WindowSmem& sm, uint8_t* kout, int nvalid, int tid, int bar_id) {
  constexpr int NB = (1 << BITS) - 1, cpw = 32 / BITS, wpt = kHeadDim / cpw;
  if constexpr (!kTurbo) {
    const int c = tid;
    const float s = sm.s_scale[c], m = sm.s_min[c];
    const ScaledBounds<NB> sb = scale_bounds(load_bounds<NB>(sm.bk), s);
    const int col0 = kp_col(0, c), col1 = kp_col(1, c);  // the column depends on the token's parity only
#pragma unroll 4
    for (int t = 0; t < kWindow; ++t)
      sm.codes[t][c] = (uint8_t)((t < nvalid && s != 0.0f)
                                     ? code_from_scaled(sb, __fsub_rn(sm.kp[t][(t & 1) ? col1 : col0], m))
                                     : 0u);
  } else {
    if (tid < kWindow) {  // thread t: token t's bounds, once
      const ScaledBounds<NB> sb = scale_bounds(load_bounds<NB>(sm.bk), sm.s_scale[tid]);
#pragma unroll
      for (int j = 0; j < NB; ++j) sm.tb[tid][j] = sb.b[j];
    }
    group_sync(bar_id);
    const int c = tid;
    const int col0 = kp_col(0, c), col1 = kp_col(1, c);
#pragma unroll 2
    for (int t = 0; t < kWindow; ++t) {
      const float s = sm.s_scale[t];
      ScaledBounds<NB> sb;
#pragma unroll
      for (int j = 0; j < NB; ++j) sb.b[j] = sm.tb[t][j];
      sm.codes[t][c] = (uint8_t)((t < nvalid && s != 0.0f) ? code_from_scaled(sb, sm.kp[t][(t & 1) ? col1 : col0]) : 0u);
    }
  }
  group_sync(bar_id);
  uint32_t* kw = reinterpret_cast<uint32_t*>(kout);
  for (int wi = tid; wi < kWindow * wpt; wi += kWriteThreads) {
    const int t = wi / wpt;
    const int word = wi - t * wpt;
    // cpw code bytes, 4 per u32, compacted to BITS-bit fields (bytes hold codes < 2^BITS)
    const uint32_t* src = reinterpret_cast<const uint32_t*>(&sm.codes[t][word * cpw]);
    uint32_t bits = 0;
#pragma unroll
    for (int q = 0; q < cpw / 4; ++q) {
      const uint32_t x = src[q];
      const uint32_t f = (x & 0xFFu) | ((x >> (8 - BITS)) & (0xFFu << BITS)) | ((x >> (16 - 2 * BITS)) & (0xFFu << (2 * BITS))) |
                         ((x >> (24 - 3 * BITS)) & (0xFFu << (3 * BITS)));
      bits |= (f & ((1u << (4 * BITS)) - 1u)) << (4 * BITS * q);
    }
    kw[wi] = bits;
  }
}

// Re-quantise window w of (sequence b, kv head h) after the append of
// positions [L0, L1), by the 128 threads of one group (tid 0..127, barrier
// bar_id). tail_any: this group also handles every other window the append
// touches, in order, so a partial window always keeps its new raw keys in the
// tail (otherwise only the first touched window does, and finish_write_kernel
// copies those of a distinct partial last window).
// kMeta: the key metadata format (kMetaFp16, kMetaMx, kMetaTurbo), a compile-time
// choice so that each kernel carries only its format's code.
template <int kMeta>
__device__ void quantize_window(const WriteParams& p, int b, int h, int w, int L0, int L1, WindowSmem& sm, int tid,
                                int bar_id, bool tail_any) {
  const int H = p.num_kv_heads;
  const int p0 = w * kWindow;
  const int p1 = min(p0 + kWindow, L1);
  const int nvalid = p1 - p0;
  const int inew0 = max(L0 - p0, 0);  // first slot of this window holding a new token

  const RecordLayout lay(p.key_bits, p.value_bits, kMeta);
  uint8_t* rec = p.records + ((size_t)(b * H + h) * p.cap_windows + w) * lay.bytes;
  const size_t seq_head = (size_t)b * H + h;
  __half* tail = p.key_tail + seq_head * kWindow * kHeadDim;
  const __half* knew = p.k_new + seq_head * p.n_new * kHeadDim;
  const __half* vnew = p.v_new + seq_head * p.n_new * kHeadDim;
  const uint8_t* mnew = p.mod_new + (size_t)b * p.n_new;

  float (*kp)[kHeadDim] = sm.kp;
  float* s_min = sm.s_min;
  float* s_scale = sm.s_scale;
  float* s_sigma = sm.s_sigma;

  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int LK = 1 << p.key_bits;
  const int LV = 1 << p.value_bits;
  constexpr bool turbo = kMeta == kMetaTurbo;
  const float kc0 = p.key_cb[0];
  if (tid < LK - 1)
    sm.bk[tid] = make_code_bound(__fmul_rn(__fadd_rn(p.key_cb[tid], p.key_cb[tid + 1]), 0.5f), turbo ? 0.0f : kc0);
  if (tid >= 32 && tid - 32 < LV - 1) {
    const int j = tid - 32;
    sm.bv[j] = make_code_bound(__fmul_rn(__fadd_rn(p.val_cb[j], p.val_cb[j + 1]), 0.5f), 0.0f);
  }
  const float kspan = __fsub_rn(p.key_cb[LK - 1], kc0);

  // ---- issue every raw-key load of the window first (one memory round trip),
  // and prefetch the value basis of the first new token into L2 so that the
  // value rotation below reads it from L2. Four threads per token: thread
  // (i = tid / 4, q = tid % 4) holds channels 32 q .. 32 q + 31 of token i.
  const int ti = tid >> 2, tq = tid & 3;
  uint4 raw[4] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u),
                  make_uint4(0u, 0u, 0u, 0u)};
  if (ti < nvalid) {
    const int pos = p0 + ti;
    const __half* src = (pos < L0 ? tail + ti * kHeadDim : knew + (size_t)(pos - L0) * kHeadDim) + 32 * tq;
#pragma unroll
    for (int j = 0; j < 4; ++j) raw[j] = reinterpret_cast<const uint4*>(src)[j];
  }
  // the value of this warp's first new token (used after the keys, loaded now)
  __half vfirst[4] = {__float2half(0.f), __float2half(0.f), __float2half(0.f), __float2half(0.f)};
  if (!(p.tc_values && p0 >= L0 && nvalid == kWindow) && inew0 + warp < nvalid) {
    const __half* src = vnew + (size_t)(p0 + inew0 + warp - L0) * kHeadDim;
#pragma unroll
    for (int j = 0; j < 4; ++j) vfirst[j] = src[lane + 32 * j];
  }
  if (!(p.tc_values && p0 >= L0 && nvalid == kWindow)) {
    int m0 = mnew[p0 + inew0 - L0];
    m0 = m0 >= kMods ? kMods - 1 : m0;
    const float* U = p.value_rot + ((size_t)(h * kMods + m0) * kHeadDim + tid) * kHeadDim;  // row tid
#pragma unroll
    for (int q = 0; q < 4; ++q) asm volatile("prefetch.global.L2 [%0];" ::"l"(U + 32 * q));
  }

  // ---- keys: rotate every valid token of the window: sign flip, butterflies
  // h = 1 .. 16 inside the thread's 32 channels, h = 32 and 64 with the threads
  // of the same token holding channels c + h (the lower index of a pair becomes
  // a + b, the upper a - b, as in the scalar order), then the scale 2^-3.5.
  if (ti < nvalid) {
    const int pos = p0 + ti;
    // the tail keeps the new raw keys of a window left partial (see tail_any)
    if (nvalid < kWindow && pos >= L0 && (tail_any || w == L0 / kWindow)) {
#pragma unroll
      for (int j = 0; j < 4; ++j) reinterpret_cast<uint4*>(tail + ti * kHeadDim + 32 * tq)[j] = raw[j];
    }
  }
  {
    float x[32];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __half2* hp = reinterpret_cast<const __half2*>(&raw[j]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(hp[e]);
        x[8 * j + 2 * e] = f.x;
        x[8 * j + 2 * e + 1] = f.y;
      }
    }
    const float4* sgn = reinterpret_cast<const float4*>(p.key_signs + 32 * tq);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 g = sgn[j];
      x[4 * j] = __fmul_rn(x[4 * j], g.x);
      x[4 * j + 1] = __fmul_rn(x[4 * j + 1], g.y);
      x[4 * j + 2] = __fmul_rn(x[4 * j + 2], g.z);
      x[4 * j + 3] = __fmul_rn(x[4 * j + 3], g.w);
    }
#pragma unroll
    for (int hh = 1; hh < 32; hh <<= 1)
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (!(c & hh)) {
          const float a = x[c], b = x[c + hh];
          x[c] = __fadd_rn(a, b);
          x[c + hh] = __fsub_rn(a, b);
        }
#pragma unroll
    for (int d = 1; d <= 2; d <<= 1) {  // h = 32 (partner q ^ 1), h = 64 (partner q ^ 2)
      const bool upper = (tq & d) != 0;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float other = __shfl_xor_sync(0xffffffffu, x[c], d);
        x[c] = upper ? __fsub_rn(other, x[c]) : __fadd_rn(x[c], other);
      }
    }
    const float sc = inv_sqrt_d();
    if (ti < nvalid) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<float4*>(&kp[ti][kp_col(ti, 32 * tq + 4 * j)]) =
            make_float4(__fmul_rn(x[4 * j], sc), __fmul_rn(x[4 * j + 1], sc), __fmul_rn(x[4 * j + 2], sc),
                        __fmul_rn(x[4 * j + 3], sc));
    }
  }
  group_sync(bar_id);

  // ---- TurboQuant keys: one scale per token from the unrotated fp16 key, the
  // pairwise tree of the value scale (h = 64 across threads q ^ 2, h = 32 across
  // q ^ 1, then h = 16 .. 1 inside the thread's 32 channels)
  if constexpr (turbo) {
    float x[32];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __half2* hp = reinterpret_cast<const __half2*>(&raw[j]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(hp[e]);
        x[8 * j + 2 * e] = __fmul_rn(f.x, f.x);  // exact: an fp16 square fits in fp32
        x[8 * j + 2 * e + 1] = __fmul_rn(f.y, f.y);
      }
    }
#pragma unroll
    for (int c = 0; c < 32; ++c) x[c] = __fadd_rn(x[c], __shfl_xor_sync(0xffffffffu, x[c], 2));
#pragma unroll
    for (int c = 0; c < 32; ++c) x[c] = __fadd_rn(x[c], __shfl_xor_sync(0xffffffffu, x[c], 1));
#pragma unroll
    for (int hh = 16; hh >= 1; hh >>= 1)
#pragma unroll
      for (int c = 0; c < hh; ++c) x[c] = __fadd_rn(x[c], x[c + hh]);
    if (tq == 0 && ti < kWindow) {
      const __half s16 = ti < nvalid ? __float2half_rn(__fsqrt_rn(__fmul_rn(x[0], 0.0078125f))) : __float2half(0.0f);
      reinterpret_cast<__half*>(rec + lay.meta_off)[ti] = s16;
      s_scale[ti] = __half2float(s16);
    }
  } else {
  // ---- window range per channel -> fp16 metadata -----------------------------
  {
    const int c = tid;
    const int col0 = kp_col(0, c), col1 = kp_col(1, c);  // the column depends on the token's parity only
    float mn = kp[0][col0], mx = mn;
    for (int i = 1; i < nvalid; ++i) {
      const float v = kp[i][(i & 1) ? col1 : col0];
      mn = fminf(mn, v);
      mx = fmaxf(mx, v);
    }
    if constexpr (kMeta == kMetaMx) {
      // MXFP4: the warp's 32 channels form one block. The minimum is rounded to
      // the nearest E2M1 value of its block's exponent, then the scale it needs,
      // fp32((max - m^) / (c_last - c_0)) (0 if negative), on the scale block's grid.
      uint8_t* meta = rec + lay.meta_off;
      float am = fabsf(mn);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      const int em = mx_block_exp(am);
      uint32_t mcode, scode;
      const float mhat = mx_round_nearest(mn, em, &mcode);
      const float sreq = fmaxf(__fdiv_rn(__fsub_rn(mx, mhat), kspan), 0.0f);
      float as = sreq;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) as = fmaxf(as, __shfl_xor_sync(0xffffffffu, as, o));
      const int es = mx_block_exp(as);
      const float shat = mx_round_nearest(sreq, es, &scode);
      const uint32_t mnext = __shfl_down_sync(0xffffffffu, mcode, 1);
      const uint32_t snext = __shfl_down_sync(0xffffffffu, scode, 1);
      if (!(c & 1)) {  // byte c / 2: channel c in the low nibble, c + 1 in the high one
        meta[c >> 1] = (uint8_t)(mcode | (mnext << 4));
        meta[64 + (c >> 1)] = (uint8_t)(scode | (snext << 4));
      }
      if ((c & 31) == 0) {
        meta[128 + (c >> 5)] = (uint8_t)(em + 127);
        meta[132 + (c >> 5)] = (uint8_t)(es + 127);
      }
      if (c < 8) meta[136 + c] = 0;
      s_min[c] = mhat;
      s_scale[c] = shat;
    } else {
      const __half m16 = __float2half_rn(mn);
      const __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), kspan));
      reinterpret_cast<__half2*>(rec + lay.meta_off)[c] = __halves2half2(m16, s16);
      s_min[c] = __half2float(m16);
      s_scale[c] = __half2float(s16);
    }
  }
  }
  group_sync(bar_id);

  // ---- key codes, token-major words -----------------------------------------
  if (p.key_bits == 2)
    key_code_words<2, turbo>(sm, rec + lay.k_off, nvalid, tid, bar_id);
  else
    key_code_words<4, turbo>(sm, rec + lay.k_off, nvalid, tid, bar_id);
  group_sync(bar_id);  // kp is reused for values below

  // windows filled completely by this write get their values from vrot_tc
  const bool tc_window = p.tc_values && p0 >= L0 && nvalid == kWindow;
  if (tc_window) {
    if (h == 0 && tid < kWindow) {
      const int m = mnew[p0 + tid - L0];
      if (m >= kMods) set_error(p.error_word, OMNIKV_DEVERR_MODALITY);
      p.modality[(size_t)b * p.cap_tokens + p0 + tid] = (uint8_t)(m >= kMods ? kMods - 1 : m);
    }
    return;
  }

  // ---- values: per-token scale (pairwise tree in a warp) ----------------------
  for (int i = inew0 + warp; i < nvalid; i += kWriteThreads / 32) {
    float x[4];
    if (i == inew0 + warp) {  // the warp's first new value was loaded at the start
#pragma unroll
      for (int j = 0; j < 4; ++j) x[j] = __half2float(vfirst[j]);
    } else {
      const __half* src = vnew + (size_t)(p0 + i - L0) * kHeadDim;
#pragma unroll
      for (int j = 0; j < 4; ++j) x[j] = __half2float(src[lane + 32 * j]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) kp[i][lane + 32 * j] = x[j];
    // tree: h = 64 pairs j with j + 2, h = 32 pairs the two results, then lanes
    const float a = __fadd_rn(__fmul_rn(x[0], x[0]), __fmul_rn(x[2], x[2]));
    const float c = __fadd_rn(__fmul_rn(x[1], x[1]), __fmul_rn(x[3], x[3]));
    float z = __fadd_rn(a, c);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) z = __fadd_rn(z, __shfl_xor_sync(0xffffffffu, z, o));
    if (lane == 0) s_sigma[i] = __half2float(__float2half_rn(__fsqrt_rn(__fmul_rn(z, 0.0078125f))));
  }
  group_sync(bar_id);

  // ---- values: rotation, codes, channel-major packing --------------------------
  {
    const int j = tid;  // output channel
    const int cpw = 32 / p.value_bits;
    const int ngroups = kWindow / cpw;
    const uint32_t mask = (1u << p.value_bits) - 1u;
    uint32_t* vw = reinterpret_cast<uint32_t*>(rec + lay.v_off);
    uint32_t words[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) words[g] = g < ngroups ? vw[g * kHeadDim + j] : 0u;
    for (int i = inew0; i < nvalid; ++i) {
      int m = mnew[p0 + i - L0];
      if (m >= kMods) m = kMods - 1;  // out-of-range ids are flagged below and read as video
      const float* U = p.value_rot + ((size_t)(h * kMods + m) * kHeadDim) * kHeadDim + j;
      // column j of U_m against the value: independent loads, 8 partial sums
      float part[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll  // every load of the column issued before the first FMA needs it
      for (int c = 0; c < kHeadDim; ++c) part[c & 7] = fmaf(U[(size_t)c * kHeadDim], kp[i][c], part[c & 7]);
      const float acc = ((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7]));
      if (p.vrot_dump) p.vrot_dump[((size_t)(b * H + h) * p.n_new + (p0 + i - L0)) * kHeadDim + j] = acc;
      const float s = s_sigma[i];
      uint32_t code = 0;  // #{j : v' / sigma > t_j}, 0 where sigma == 0
      if (s != 0.0f)
        code = p.value_bits == 2 ? code_from_scaled(scale_bounds(load_bounds<3>(sm.bv), s), acc)
                                 : code_from_scaled(scale_bounds(load_bounds<15>(sm.bv), s), acc);
      const int g = i / cpw;
      const int sh = p.value_bits * (i - g * cpw);
#pragma unroll
      for (int gg = 0; gg < 4; ++gg)
        if (gg == g) words[gg] = (words[gg] & ~(mask << sh)) | (code << sh);
    }
#pragma unroll
    for (int g = 0; g < 4; ++g)
      if (g < ngroups) vw[g * kHeadDim + j] = words[g];
  }
  if (tid >= inew0 && tid < nvalid) {
    reinterpret_cast<__half*>(rec + lay.sigma_off)[tid] = __float2half_rn(s_sigma[tid]);
    if (h == 0) {
      const int m = mnew[p0 + tid - L0];
      if (m >= kMods) set_error(p.error_word, OMNIKV_DEVERR_MODALITY);
      p.modality[(size_t)b * p.cap_tokens + p0 + tid] = (uint8_t)(m >= kMods ? kMods - 1 : m);
    }
  }
}


// quantize_window for the format in p.key_meta (a kernel that serves every format).
__device__ __forceinline__ void quantize_window_any(const WriteParams& p, int b, int h, int w, int L0, int L1,
                                                    WindowSmem& sm, int tid, int bar_id, bool tail_any) {
  if (p.key_meta == kMetaMx)
    quantize_window<kMetaMx>(p, b, h, w, L0, L1, sm, tid, bar_id, tail_any);
  else if (p.key_meta == kMetaTurbo)
    quantize_window<kMetaTurbo>(p, b, h, w, L0, L1, sm, tid, bar_id, tail_any);
  else
    quantize_window<kMetaFp16>(p, b, h, w, L0, L1, sm, tid, bar_id, tail_any);
}

}  // namespace
}  // namespace omnikv
