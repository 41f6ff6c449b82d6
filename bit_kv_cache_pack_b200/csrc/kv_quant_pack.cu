// kv_quant_pack: the OmniKVQuant cache write.
//
// One CTA per (window touched by the new positions, kv head, sequence).
// Keys (paperpeel.com section 2.2 "Temporal key drift", 3.1 "32-token groups g",
// 3.3 "FP16 minimum m_gc and scale s_gc"): every touched window is re-quantised
// over all its valid tokens -- sign flip + Hadamard butterflies in a warp
// (4 channels per lane), per-channel min / max over the window, fp16 metadata,
// codes on the fixed codebook, 16 (or 8) codes per u32. A window left partial
// keeps its raw fp16 keys in the tail so a later append can re-quantise it.
// Values (section 2.3 "Modality-aware value rotation"): per token, the fp16
// scale sigma (pairwise-tree sum of squares in a warp), the rotation
// v' = U_m^T v, and codes v'/sigma on the fixed codebook, packed channel-major
// (16 tokens of one channel per u32 for 2-bit codes).
#include "common.cuh"
#include "kernels.h"

namespace omnikv {

namespace {

constexpr int kWriteThreads = 128;

__global__ void __launch_bounds__(kWriteThreads)
kv_quant_pack_kernel(const WriteParams p) {
  const int b = blockIdx.z;
  const int h = blockIdx.y;
  const int H = p.num_kv_heads;
  const int L0 = p.seq_lens[b];
  const int L1 = L0 + p.n_new;
  if (L0 < 0 || L1 > p.cap_tokens) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && h == 0) set_error(p.error_word, OMNIKV_DEVERR_CAPACITY);
    return;
  }
  const int w = L0 / kWindow + blockIdx.x;
  const int p0 = w * kWindow;
  if (p0 >= L1) return;
  const int p1 = min(p0 + kWindow, L1);
  const int nvalid = p1 - p0;
  const int inew0 = max(L0 - p0, 0);  // first slot of this window holding a new token

  const RecordLayout lay(p.key_bits, p.value_bits);
  uint8_t* rec = p.records + ((size_t)(b * H + h) * p.cap_windows + w) * lay.bytes;
  const size_t seq_head = (size_t)b * H + h;
  __half* tail = p.key_tail + seq_head * kWindow * kHeadDim;
  const __half* knew = p.k_new + seq_head * p.n_new * kHeadDim;
  const __half* vnew = p.v_new + seq_head * p.n_new * kHeadDim;
  const uint8_t* mnew = p.mod_new + (size_t)b * p.n_new;

  __shared__ float kp[kWindow][kHeadDim];   // rotated keys, then reused for fp32 values
  __shared__ float s_min[kHeadDim], s_scale[kHeadDim];
  __shared__ float s_sigma[kWindow];
  __shared__ float thr_k[15], thr_v[15];

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int LK = 1 << p.key_bits;
  const int LV = 1 << p.value_bits;
  if (tid < LK - 1) thr_k[tid] = __fmul_rn(__fadd_rn(p.key_cb[tid], p.key_cb[tid + 1]), 0.5f);
  if (tid < LV - 1) thr_v[tid] = __fmul_rn(__fadd_rn(p.val_cb[tid], p.val_cb[tid + 1]), 0.5f);
  const float kc0 = p.key_cb[0];
  const float kspan = __fsub_rn(p.key_cb[LK - 1], kc0);

  // ---- issue every raw-key load of the window first (one memory round trip),
  // and prefetch the value basis of the first new token into L2 so that the
  // value rotation below reads it from L2
  constexpr int kPerWarp = kWindow / (kWriteThreads / 32);
  uint2 raws[kPerWarp];
#pragma unroll
  for (int k = 0; k < kPerWarp; ++k) {
    const int i = warp + (kWriteThreads / 32) * k;
    if (i < nvalid) {
      const int pos = p0 + i;
      const __half* src = pos < L0 ? tail + i * kHeadDim : knew + (size_t)(pos - L0) * kHeadDim;
      raws[k] = *reinterpret_cast<const uint2*>(src + 4 * lane);
    }
  }
  if (!(p.tc_values && p0 >= L0 && nvalid == kWindow)) {
    int m0 = mnew[p0 + inew0 - L0];
    m0 = m0 >= kMods ? kMods - 1 : m0;
    const float* U = p.value_rot + ((size_t)(h * kMods + m0) * kHeadDim + tid) * kHeadDim;  // row tid
#pragma unroll
    for (int q = 0; q < 4; ++q) asm volatile("prefetch.global.L2 [%0];" ::"l"(U + 32 * q));
  }

  // ---- keys: rotate every valid token of the window -------------------------
  float sg[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) sg[r] = p.key_signs[4 * lane + r];
#pragma unroll
  for (int k = 0; k < kPerWarp; ++k) {
    const int i = warp + (kWriteThreads / 32) * k;
    if (i >= nvalid) break;
    const int pos = p0 + i;
    const uint2 raw = raws[k];
    // the tail is written here only when this window is also the first one
    // touched (it reads old slots < L0 - p0 and writes new ones); a distinct
    // partial last window is copied by finish_write_kernel after this kernel.
    if (nvalid < kWindow && pos >= L0 && w == L0 / kWindow)
      *reinterpret_cast<uint2*>(tail + i * kHeadDim + 4 * lane) = raw;
    const __half2 lo = *reinterpret_cast<const __half2*>(&raw.x);
    const __half2 hi = *reinterpret_cast<const __half2*>(&raw.y);
    float x[4] = {__low2float(lo), __high2float(lo), __low2float(hi), __high2float(hi)};
    warp_hadamard_rotate(x, sg);
    *reinterpret_cast<float4*>(&kp[i][4 * lane]) = make_float4(x[0], x[1], x[2], x[3]);
  }
  __syncthreads();

  // ---- window range per channel -> fp16 metadata -----------------------------
  {
    const int c = tid;
    float mn = kp[0][c], mx = kp[0][c];
    for (int i = 1; i < nvalid; ++i) {
      mn = fminf(mn, kp[i][c]);
      mx = fmaxf(mx, kp[i][c]);
    }
    const __half m16 = __float2half_rn(mn);
    const __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), kspan));
    reinterpret_cast<__half2*>(rec + lay.meta_off)[c] = __halves2half2(m16, s16);
    s_min[c] = __half2float(m16);
    s_scale[c] = __half2float(s16);
  }
  __syncthreads();

  // ---- key codes, token-major words -----------------------------------------
  {
    const int cpw = 32 / p.key_bits;
    const int wpt = kHeadDim / cpw;
    uint32_t* kw = reinterpret_cast<uint32_t*>(rec + lay.k_off);
    for (int wi = tid; wi < kWindow * wpt; wi += kWriteThreads) {
      const int t = wi / wpt;
      const int word = wi - t * wpt;
      uint32_t bits = 0;
      if (t < nvalid) {
        for (int k = 0; k < cpw; ++k) {
          const int ch = word * cpw + k;
          const float s = s_scale[ch];
          uint32_t code = 0;
          if (s != 0.0f) {
            const float z = __fadd_rn(__fdiv_rn(__fsub_rn(kp[t][ch], s_min[ch]), s), kc0);
            code = count_above(z, thr_k, LK - 1);
          }
          bits |= code << (p.key_bits * k);
        }
      }
      kw[wi] = bits;
    }
  }
  __syncthreads();  // kp is reused for values below

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
    const __half* src = vnew + (size_t)(p0 + i - L0) * kHeadDim;
    float x[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      x[j] = __half2float(src[lane + 32 * j]);
      kp[i][lane + 32 * j] = x[j];
    }
    // tree: h = 64 pairs j with j + 2, h = 32 pairs the two results, then lanes
    const float a = __fadd_rn(__fmul_rn(x[0], x[0]), __fmul_rn(x[2], x[2]));
    const float c = __fadd_rn(__fmul_rn(x[1], x[1]), __fmul_rn(x[3], x[3]));
    float z = __fadd_rn(a, c);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) z = __fadd_rn(z, __shfl_xor_sync(0xffffffffu, z, o));
    if (lane == 0) s_sigma[i] = __half2float(__float2half_rn(__fsqrt_rn(__fmul_rn(z, 0.0078125f))));
  }
  __syncthreads();

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
#pragma unroll 32
      for (int c = 0; c < kHeadDim; ++c) part[c & 7] = fmaf(U[(size_t)c * kHeadDim], kp[i][c], part[c & 7]);
      const float acc = ((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7]));
      const float s = s_sigma[i];
      uint32_t code = 0;
      if (s != 0.0f) code = count_above(__fdiv_rn(acc, s), thr_v, LV - 1);
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

// One CTA per sequence: copies the raw keys of a partial last window that is
// not the first window touched into the tail, then advances the length.
__global__ void finish_write_kernel(const WriteParams p) {
  const int b = blockIdx.x;
  const int L0 = p.seq_lens[b];
  const int L1 = L0 + p.n_new;
  if (L0 < 0 || L1 > p.cap_tokens) return;
  const int wl = L1 / kWindow;             // window holding position L1 (partial if L1 % 32)
  const int r = L1 - wl * kWindow;
  if (r > 0 && wl != L0 / kWindow) {
    for (int h = 0; h < p.num_kv_heads; ++h) {
      const size_t seq_head = (size_t)b * p.num_kv_heads + h;
      __half* tail = p.key_tail + seq_head * kWindow * kHeadDim;
      const __half* knew = p.k_new + (seq_head * p.n_new + (wl * kWindow - L0)) * kHeadDim;
      for (int e = threadIdx.x; e < r * kHeadDim / 4; e += blockDim.x)
        reinterpret_cast<uint2*>(tail)[e] = reinterpret_cast<const uint2*>(knew)[e];
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) p.seq_lens[b] = L1;
}

}  // namespace

cudaError_t launch_write(const WriteParams& p_in, int batch, cudaStream_t stream) {
  WriteParams p = p_in;
  p.tc_values = p.n_new >= kWindow ? 1 : 0;  // a write this long can fill whole windows
  const int slots = (p.n_new + kWindow - 1) / kWindow + 1;
  dim3 grid(slots, p.num_kv_heads, batch);
  kv_quant_pack_kernel<<<grid, kWriteThreads, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (p.tc_values) {
    e = launch_vrot_tc(p, batch, stream);
    if (e != cudaSuccess) return e;
  }
  finish_write_kernel<<<batch, 128, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace omnikv
