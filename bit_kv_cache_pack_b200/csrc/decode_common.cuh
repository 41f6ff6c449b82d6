// Device helpers shared by the decode kernels (decode_split_k.cu, stream.cu):
// rotated-query layout, split ranges, decode-step flags, and the CUDA-core decode
// path (mixed bit widths, 2-bit codebooks that are not symmetric).
#pragma once

#include <cstddef>

#include "append.cuh"
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace omnikv {

namespace {

constexpr int kWarps = 4;                         // warps of the CUDA-core path (and of the mma.sync bodies)
constexpr int kThreads = 32 * kWarps;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: a copy or flag that takes longer is an error
constexpr float kLog2e = 1.4426950408889634f;

// Barrier policy of the CUDA-core path: the whole CTA (its kernels' CTAs are the
// 4 warps of the decode).
struct SyncCta {
  __device__ __forceinline__ static void sync() { __syncthreads(); }
  __device__ __forceinline__ static bool sync_or(bool p) { return __syncthreads_or(p); }
};

// Position of channel c of head g in the rotated-query buffer. Chunks of 4
// channels inside each group of 32 are XOR-swizzled so that the 8 lanes of a
// quarter warp (heads g, g+1 x channel groups t = 0..3) reading chunk i read 8
// different bank groups.
__device__ __forceinline__ int qpos(int g, int c) {
  const int t = c >> 5, i4 = (c >> 2) & 7;
  return g * kHeadDim + 32 * t + 4 * (i4 ^ ((4 * (g & 1) + t) & 7)) + (c & 3);
}

// q' = fp32(2^-3.5) H (s . q) for every head of the group, times 2^-3.5 more
// (the softmax scale 1/sqrt(128)); heads >= G are zero. Stored at qpos(g, c).
template <int kNumWarps = kWarps>
__device__ __forceinline__ void rotate_queries(const DecodeParams& p, int b, int kvh, float* qflat) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.group;
  const int Hq = p.num_kv_heads * G;
  float sg[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) sg[r] = p.key_signs[4 * lane + r];
  for (int g = warp; g < kMaxGroup && warp < kNumWarps; g += kNumWarps) {
    if (g < G) {
      const __half* q = p.q + ((size_t)b * Hq + kvh * G + g) * kHeadDim;
      const uint2 raw = *reinterpret_cast<const uint2*>(q + 4 * lane);
      const __half2 lo = *reinterpret_cast<const __half2*>(&raw.x);
      const __half2 hi = *reinterpret_cast<const __half2*>(&raw.y);
      float x[4] = {__low2float(lo), __high2float(lo), __low2float(hi), __high2float(hi)};
      warp_hadamard_rotate(x, sg);
#pragma unroll
      for (int r = 0; r < 4; ++r) qflat[qpos(g, 4 * lane + r)] = x[r] * inv_sqrt_d();
    } else {
#pragma unroll
      for (int r = 0; r < 4; ++r) qflat[qpos(g, 4 * lane + r)] = 0.0f;
    }
  }
}

// Split s covers windows [s C, min((s+1) C, W_b)) of sequence b, with C =
// p.split_windows chosen on the host from the length bound, so a short sequence
// leaves its last splits empty and every non-empty split has the same size.
__device__ __forceinline__ void split_range(const DecodeParams& p, int b, int split, int& T, int& w0, int& w1) {
  const int L = p.seq_lens[b];
  const int La = L + p.len_add;  // a decode step's append happens only within the capacity
  T = max(0, min(La <= p.cap_tokens ? La : L, p.cap_tokens));
  if (p.stream) T = kWindow * (max(0, T - 128) / kWindow);  // streaming policy: the packed body only
  const int nw = (T + kWindow - 1) / kWindow;
  w0 = min(split * p.split_windows, nw);
  w1 = min(w0 + p.split_windows, nw);
  if (split == p.num_splits - 1 && threadIdx.x == 0 && nw > p.num_splits * p.split_windows)
    set_error(p.error_word, OMNIKV_DEVERR_BOUND);
}

// Decode step: the window that receives the appended token, and the flag value
// that marks its record as written (window -1: nothing to wait for).
__device__ __forceinline__ void step_window(const DecodeParams& p, int b, int& win, int& val) {
  win = -1;
  val = 0;
  if (p.len_add > 0 && p.step_flags != nullptr) {
    const int L = p.seq_lens[b];
    if (L >= 0 && L + p.len_add <= p.cap_tokens) {
      val = L + p.len_add;
      win = (val - 1) / kWindow;
    }
  }
}

// Bounded acquire-spin until *flag == val (written with release by the append
// CTA of the same launch); false after about `limit_ns`.
__device__ __forceinline__ bool wait_flag(const int32_t* flag, int val, uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 0;; ++it) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v == val) break;
    if ((it & 63u) == 63u && global_timer_ns() - t0 > limit_ns) return false;
    __nanosleep(64);
  }
  // the record is then read through the async proxy (bulk copy)
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return true;
}

// 2^x with the hardware approximation (relative error below 2^-22); -inf -> 0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------------------
// CUDA-core path (mixed bit widths, or a 2-bit codebook that is not symmetric):
// the CTA decodes the split's windows one at a time from a double-buffered ring of bulk
// copies. Scores: four threads per token, thread q of token t holding channels
// 4 j + q (j = 0..31), each dequantised once, k'_tc = m_c + s_c (c_code - c_0),
// and used for the 8 query heads; two shuffles complete the dot products.
// Values: thread c owns channel c and one fp32 accumulator per (modality, head).
// ---------------------------------------------------------------------------
constexpr int kGenStages = 2;

struct GenSmem {                 // laid over the calling body's staging buffers
  uint8_t rec[kGenStages][4704];  // window record + 32 modality ids (largest record: 4672 B)
  float qT[kHeadDim][kMaxGroup];  // rotated queries, channel-major
  float pw[kWindow][kMaxGroup];   // p_ht * sigma_t of the current window
  float dk[16], dv[16];           // c_j - c_0 (keys), c_j (values)
  float wmax[kWarps][kMaxGroup];
  float2 mxm[kHeadDim];            // MXFP4 caches: (m^, s^) of every channel of the current window
  uint64_t bar[kGenStages];
  uint32_t runs;                  // bit t: token t of the current window starts a run of one modality
  int abort;                      // a step flag never arrived: the split is written empty
};

static_assert(offsetof(GenSmem, qT) % 16 == 0 && offsetof(GenSmem, pw) % 16 == 0, "16-byte vector fields");
static_assert(offsetof(GenSmem, mxm) % 8 == 0 && offsetof(GenSmem, bar) % 8 == 0, "8-byte fields");

// (m^, s^) of channel c from a window's MXFP4 key metadata: E2M1 codes two per
// byte (even channel in the low nibble), minima then scales, then the E8M0
// exponents (e + 127) of the 4 minimum blocks and the 4 scale blocks.
// E2M1 code (sign << 3 | magnitude index i) times 2^(eb - 127) for a block exponent
// byte eb, without branches: the magnitude's fp32 bits (0, 0.5, or (1 + (i & 1)/2) *
// 2^(i/2 - 1) for i >= 2) times the fp32 power of two (2^-127 is subnormal; eb = 255
// is taken as 2^127 * 2). Exact, and the same value as mx_value(code, eb - 127).
__device__ __forceinline__ float mx_decode(uint32_t code, uint32_t eb) {
  const uint32_t i = code & 7u;
  const uint32_t mag = i >= 2u ? (i << 22) + 0x3F000000u : (i != 0u ? 0x3F000000u : 0u);
  const float p2 = __uint_as_float(eb == 0u ? 0x00400000u : (eb == 255u ? 254u << 23 : eb << 23));
  const float v = __uint_as_float(mag | ((code & 8u) << 28)) * p2;
  return eb == 255u ? v * 2.0f : v;
}

__device__ __forceinline__ float2 mx_meta_channel(const uint8_t* meta, int c) {
  const uint32_t mb = meta[c >> 1], sb = meta[64 + (c >> 1)];
  const uint32_t mc = (c & 1) ? (mb >> 4) : (mb & 15u), sc = (c & 1) ? (sb >> 4) : (sb & 15u);
  return make_float2(mx_decode(mc, meta[128 + (c >> 5)]), mx_decode(sc, meta[132 + (c >> 5)]));
}

__device__ __forceinline__ void gen_issue(const DecodeParams& p, GenSmem& g, int stage, const uint8_t* rec_base,
                                          int rec_bytes, int b, int kvh, int wi, int wait_win, int wait_val) {
  if (wi == wait_win &&
      !wait_flag(p.step_flags + (size_t)b * p.num_kv_heads + kvh, wait_val, p.flag_wait_ns)) {
    // the appended token's record never became ready: no copy of a stale record
    set_error(p.error_word, OMNIKV_DEVERR_TIMEOUT);
    g.abort = 1;
    mbar_arrive_expect_tx(&g.bar[stage], 0);
    return;
  }
  mbar_arrive_expect_tx(&g.bar[stage], rec_bytes + kWindow);
  bulk_copy_g2s(g.rec[stage], rec_base + (size_t)wi * rec_bytes, rec_bytes, &g.bar[stage]);
  bulk_copy_g2s(g.rec[stage] + rec_bytes, p.modality + (size_t)b * p.cap_tokens + (size_t)wi * kWindow, kWindow,
                &g.bar[stage]);
}

template <int KB, int VB, class Sync>
__device__ void decode_generic_t(const DecodeParams& p, GenSmem& g, const float* qflat, int b, int kvh, int split) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.group;
  const int Hq = p.num_kv_heads * G;
  int T, w0, w1;
  split_range(p, b, split, T, w0, w1);
  int wait_win, wait_val;
  step_window(p, b, wait_win, wait_val);
  const RecordLayout lay(p.key_bits, p.value_bits, p.key_meta);
  const uint8_t* rec_base = p.records + ((size_t)(b * p.num_kv_heads + kvh) * p.cap_windows) * lay.bytes;
  const int nwin = w1 - w0;
  if (tid == 0) {
    g.abort = 0;
    for (int s = 0; s < kGenStages; ++s) mbar_init(&g.bar[s], 1);
    fence_barrier_init();
    for (int s = 0; s < kGenStages && s < nwin; ++s) gen_issue(p, g, s, rec_base, lay.bytes, b, kvh, w0 + s, wait_win, wait_val);
  }
  const int LK = 1 << p.key_bits, LV = 1 << p.value_bits;
  const bool tqfmt = p.key_meta == kMetaTurbo;  // TurboQuant keys: k'_tc = ksigma_t c_j
  if (tid < LK) g.dk[tid] = tqfmt ? p.key_cb[tid] : p.key_cb[tid] - p.key_cb[0];
  if (tid >= 32 && tid - 32 < LV) g.dv[tid - 32] = p.val_cb[tid - 32];
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) g.qT[tid][h] = qflat[qpos(h, tid)];
  Sync::sync();

  // score threads: token t = tid / 4, channel phase q = tid % 4
  const int st = tid >> 2, sq = tid & 3;
  constexpr uint32_t kmask = (1u << KB) - 1u, vmask = (1u << VB) - 1u;
  constexpr int kcpw = 32 / KB, kwpt = kHeadDim / kcpw, vcpw = 32 / VB;
  float m_run[kMaxGroup], l_part[kMaxGroup];  // running max (CTA-uniform), per-thread partial sums of p
  float acc[kMods][kMaxGroup];               // thread c = tid: channel c
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    m_run[h] = -INFINITY;
    l_part[h] = 0.0f;
#pragma unroll
    for (int m = 0; m < kMods; ++m) acc[m][h] = 0.0f;
  }

  int failed_at = -1;
  for (int i = 0; i < nwin; ++i) {
    const int s = i % kGenStages;
    const int wi = w0 + i;
    const bool ok = mbar_wait_bounded(&g.bar[s], (i / kGenStages) & 1, kWaitLimitNs) &&
                    *reinterpret_cast<volatile int*>(&g.abort) == 0;
    if (Sync::sync_or(!ok)) {
      failed_at = i;
      break;
    }
    const uint8_t* rec = g.rec[s];
    const uint32_t* kw = reinterpret_cast<const uint32_t*>(rec + lay.k_off);
    const __half2* meta = reinterpret_cast<const __half2*>(rec + lay.meta_off);
    const uint32_t* vw = reinterpret_cast<const uint32_t*>(rec + lay.v_off);
    const __half* sig = reinterpret_cast<const __half*>(rec + lay.sigma_off);
    const uint8_t* mods = rec + lay.bytes;
    const bool mxfmt = p.key_meta == kMetaMx;
    if (mxfmt) {  // the window's (m^, s^) in fp32, one channel per thread
      g.mxm[tid] = mx_meta_channel(rec + lay.meta_off, tid);
      Sync::sync();
    }

    // ---- scores of token st for the 8 heads over channels 4 j + sq
    float sc[kMaxGroup];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) sc[h] = 0.0f;
    {
      uint32_t row[kwpt];  // this token's key words (every channel 4 j + sq of word j * 4 / kcpw)
#pragma unroll
      for (int k4 = 0; k4 < kwpt / 4; ++k4) {
        const uint4 u = reinterpret_cast<const uint4*>(kw + st * kwpt)[k4];
        row[4 * k4] = u.x;
        row[4 * k4 + 1] = u.y;
        row[4 * k4 + 2] = u.z;
        row[4 * k4 + 3] = u.w;
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int c = 4 * j + sq;
        const uint32_t code = (row[(4 * j) / kcpw] >> (KB * (c % kcpw))) & kmask;
        const float2 ms = mxfmt ? g.mxm[c] : tqfmt ? make_float2(0.0f, 1.0f) : __half22float2(meta[c]);
        const float kv = fmaf(ms.y, g.dk[code], ms.x);
        const float4 qa = *reinterpret_cast<const float4*>(&g.qT[c][0]);
        const float4 qb = *reinterpret_cast<const float4*>(&g.qT[c][4]);
        sc[0] = fmaf(qa.x, kv, sc[0]);
        sc[1] = fmaf(qa.y, kv, sc[1]);
        sc[2] = fmaf(qa.z, kv, sc[2]);
        sc[3] = fmaf(qa.w, kv, sc[3]);
        sc[4] = fmaf(qb.x, kv, sc[4]);
        sc[5] = fmaf(qb.y, kv, sc[5]);
        sc[6] = fmaf(qb.z, kv, sc[6]);
        sc[7] = fmaf(qb.w, kv, sc[7]);
      }
    }
    const float ksg = tqfmt ? __half2float(reinterpret_cast<const __half*>(rec + lay.meta_off)[st]) : 1.0f;
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
      sc[h] += __shfl_xor_sync(0xffffffffu, sc[h], 1);
      sc[h] += __shfl_xor_sync(0xffffffffu, sc[h], 2);
      sc[h] *= ksg;
      if (wi * kWindow + st >= T || h >= G) sc[h] = -INFINITY;
    }
    // ---- window max per head: lanes of a warp (8 tokens), then the 4 warps
    float mx[kMaxGroup];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
      float v = sc[h];
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
      mx[h] = v;
    }
    if (lane == 0) {
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) g.wmax[warp][h] = mx[h];
    }
    Sync::sync();
    float alpha[kMaxGroup];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
      float v = fmaxf(fmaxf(g.wmax[0][h], g.wmax[1][h]), fmaxf(g.wmax[2][h], g.wmax[3][h]));
      const float mn = fmaxf(m_run[h], v);
      alpha[h] = (mn == -INFINITY) ? 1.0f : fast_exp2((m_run[h] - mn) * kLog2e);
      m_run[h] = mn;
    }
    // ---- where the window's modality runs start (warp 0; read after the barrier)
    if (warp == 0) {
      const int mt = min((int)mods[lane], kMods - 1);
      const int mp = lane > 0 ? min((int)mods[lane - 1], kMods - 1) : -1;
      const uint32_t starts = __ballot_sync(0xffffffffu, mt != mp);
      if (lane == 0) g.runs = starts;
    }
    // ---- p = exp(score - max); thread (st, sq) stores heads 2 sq, 2 sq + 1 of token st
    {
      const float sgm = __half2float(sig[st]);
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) {
        const float pp = (sc[h] == -INFINITY) ? 0.0f : fast_exp2((sc[h] - m_run[h]) * kLog2e);
        l_part[h] = l_part[h] * alpha[h] + (sq == 0 ? pp : 0.0f);
        if ((h >> 1) == sq) g.pw[st][h] = pp * sgm;
      }
    }
    Sync::sync();
    // ---- values: channel c = tid over the window's valid tokens, taken in runs
    // of one modality (one accumulator set per run, no per-token selection)
    {
      bool grew = false;
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) grew |= alpha[h] != 1.0f;
      if (grew) {  // the same decision in every thread
#pragma unroll
        for (int m = 0; m < kMods; ++m)
#pragma unroll
          for (int h = 0; h < kMaxGroup; ++h) acc[m][h] *= alpha[h];
      }
      const int nvalid = min(kWindow, T - wi * kWindow);
      const uint32_t starts = g.runs;
      for (int t = 0; t < nvalid;) {
        const int mod = min((int)mods[t], kMods - 1);  // the same for every thread
        const uint32_t later = starts & ~((2u << t) - 1u);  // runs starting after token t
        const int e = later ? min(nvalid, __ffs(later) - 1) : nvalid;
        float a[kMaxGroup];
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) a[h] = 0.0f;
#pragma unroll
        for (int m = 0; m < kMods; ++m)
          if (m == mod) {
#pragma unroll
            for (int h = 0; h < kMaxGroup; ++h) a[h] = acc[m][h];
          }
#pragma unroll 4
        for (int tt = t; tt < e; ++tt) {
          const uint32_t code = (vw[(tt / vcpw) * kHeadDim + tid] >> (VB * (tt % vcpw))) & vmask;
          const float d = g.dv[code];
          const float4 pa = *reinterpret_cast<const float4*>(&g.pw[tt][0]);
          const float4 pb = *reinterpret_cast<const float4*>(&g.pw[tt][4]);
          a[0] = fmaf(pa.x, d, a[0]);
          a[1] = fmaf(pa.y, d, a[1]);
          a[2] = fmaf(pa.z, d, a[2]);
          a[3] = fmaf(pa.w, d, a[3]);
          a[4] = fmaf(pb.x, d, a[4]);
          a[5] = fmaf(pb.y, d, a[5]);
          a[6] = fmaf(pb.z, d, a[6]);
          a[7] = fmaf(pb.w, d, a[7]);
        }
#pragma unroll
        for (int m = 0; m < kMods; ++m)
          if (m == mod) {
#pragma unroll
            for (int h = 0; h < kMaxGroup; ++h) acc[m][h] = a[h];
          }
        t = e;
      }
    }
    Sync::sync();  // stage s and pw are free again
    if (tid == 0 && i + kGenStages < nwin) {
      fence_proxy_async_smem();
      gen_issue(p, g, s, rec_base, lay.bytes, b, kvh, w0 + i + kGenStages, wait_win, wait_val);
    }
  }
  if (failed_at >= 0) {
    if (tid == 0) set_error(p.error_word, OMNIKV_DEVERR_TIMEOUT);
    // the copies still in flight (windows failed_at, failed_at + 1) land before
    // this CTA's shared memory is released
    for (int j = failed_at; j < nwin && j < failed_at + kGenStages; ++j)
      mbar_wait_bounded(&g.bar[j % kGenStages], (j / kGenStages) & 1, kWaitLimitNs);
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
      m_run[h] = -INFINITY;
      l_part[h] = 0.0f;
#pragma unroll
      for (int m = 0; m < kMods; ++m) acc[m][h] = 0.0f;
    }
  }

  // ---- l per head: thread sums over the tokens it owns (sq == 0), CTA reduction
  {
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
      float v = l_part[h];
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      l_part[h] = v;
    }
    Sync::sync();
    if (lane == 0) {
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) g.wmax[warp][h] = l_part[h];
    }
    Sync::sync();
  }
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    if (h >= G) continue;
    Partial* out = p.partials + ((size_t)b * Hq + kvh * G + h) * p.num_splits + split;
#pragma unroll
    for (int m = 0; m < kMods; ++m) out->acc[m][tid] = acc[m][h];
    if (tid == 0) {
      out->m = m_run[h];
      out->l = g.wmax[0][h] + g.wmax[1][h] + g.wmax[2][h] + g.wmax[3][h];
    }
  }
}

// The 2-bit builds reach the CUDA-core path only for a codebook that is not
// symmetric: out of line there, so that the tensor-core paths stay compact in
// the instruction cache. The CUDA-core build inlines its three instances.
template <class Sync>
__device__ __noinline__ void decode_generic_asym(const DecodeParams& p, GenSmem& g, const float* qflat, int b,
                                                 int kvh, int split) {
  decode_generic_t<2, 2, Sync>(p, g, qflat, b, kvh, split);
}

template <bool kGen, class Sync>
__device__ __forceinline__ void decode_generic(const DecodeParams& p, GenSmem& g, const float* qflat, int b, int kvh,
                                               int split) {
  if (!kGen)
    decode_generic_asym<Sync>(p, g, qflat, b, kvh, split);
  else if (p.key_bits == 2)
    decode_generic_t<2, 4, Sync>(p, g, qflat, b, kvh, split);
  else if (p.value_bits == 2)
    decode_generic_t<4, 2, Sync>(p, g, qflat, b, kvh, split);
  else
    decode_generic_t<4, 4, Sync>(p, g, qflat, b, kvh, split);
}

}  // namespace

}  // namespace omnikv
