// decode_split_k: fused decode attention over the packed OmniKVQuant cache.
//
// paperpeel.com section 1 (last paragraph): the query is rotated once per head
// instead of inverse-rotating every cached key, the cache is unpacked inside
// attention in FlashAttention order (refs [4], [5]), and no dense fp16 cache
// is built. One CTA per (split of the context, kv head, sequence); warp g owns
// query head kvh * G + g and shares each staged window record with the other
// query heads of its group (GQA). Per window: scores from the packed key codes
// and the window's fp16 min / scale, an online softmax (running max and sum),
// and one rotated-space accumulator per modality (values are stored in the
// basis of their modality, so they are summed per modality and mapped back by
// the combine kernel).
#include "common.cuh"
#include "kernels.h"

namespace omnikv {

namespace {

constexpr int kMaxRecordBytes = 4672;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(32 * kMaxGroup)
decode_split_k_simt_kernel(const DecodeParams p) {
  const int b = blockIdx.z;
  const int kvh = blockIdx.y;
  const int split = blockIdx.x;
  const int G = p.group;
  const int g = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int Hq = p.num_kv_heads * G;
  const int qh = kvh * G + g;

  const int T = max(0, min(p.seq_lens[b], p.cap_tokens));
  const int nw = (T + kWindow - 1) / kWindow;
  const int w0 = (int)(((long long)split * nw) / p.num_splits);
  const int w1 = (int)(((long long)(split + 1) * nw) / p.num_splits);

  const RecordLayout lay(p.key_bits, p.value_bits);
  __shared__ __align__(16) uint8_t rec[kMaxRecordBytes];
  __shared__ __align__(16) uint8_t mods[kWindow];
  __shared__ float qs[kMaxGroup][kHeadDim];
  __shared__ float cbk[16], cbv[16];

  if (threadIdx.x < (1 << p.key_bits)) cbk[threadIdx.x] = p.key_cb[threadIdx.x];
  if (threadIdx.x < (1 << p.value_bits)) cbv[threadIdx.x] = p.val_cb[threadIdx.x];

  // q' = fp32(2^-3.5) H (s . q), then the softmax scale 1/sqrt(128)
  {
    const __half* q = p.q + ((size_t)b * Hq + qh) * kHeadDim;
    const uint2 raw = *reinterpret_cast<const uint2*>(q + 4 * lane);
    const __half2 lo = *reinterpret_cast<const __half2*>(&raw.x);
    const __half2 hi = *reinterpret_cast<const __half2*>(&raw.y);
    float x[4] = {__low2float(lo), __high2float(lo), __low2float(hi), __high2float(hi)};
    float sg[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) sg[r] = p.key_signs[4 * lane + r];
    warp_hadamard_rotate(x, sg);
#pragma unroll
    for (int r = 0; r < 4; ++r) qs[g][4 * lane + r] = x[r] * inv_sqrt_d();
  }

  const int kcpw = 32 / p.key_bits, kwpt = kHeadDim / kcpw;
  const uint32_t kmask = (1u << p.key_bits) - 1u;
  const int vcpw = 32 / p.value_bits;
  const uint32_t vmask = (1u << p.value_bits) - 1u;

  float m_run = -INFINITY, l_run = 0.0f;
  float acc[kMods][4];
#pragma unroll
  for (int m = 0; m < kMods; ++m)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[m][j] = 0.0f;

  const uint8_t* rec_base = p.records + ((size_t)(b * p.num_kv_heads + kvh) * p.cap_windows) * lay.bytes;
  for (int w = w0; w < w1; ++w) {
    __syncthreads();
    {
      const uint4* src = reinterpret_cast<const uint4*>(rec_base + (size_t)w * lay.bytes);
      uint4* dst = reinterpret_cast<uint4*>(rec);
      for (int i = threadIdx.x; i < lay.bytes / 16; i += blockDim.x) dst[i] = src[i];
      if (threadIdx.x < 2)
        reinterpret_cast<uint4*>(mods)[threadIdx.x] =
            reinterpret_cast<const uint4*>(p.modality + (size_t)b * p.cap_tokens + w * kWindow)[threadIdx.x];
    }
    __syncthreads();

    const int nvalid = min(kWindow, T - w * kWindow);
    const uint32_t* kw = reinterpret_cast<const uint32_t*>(rec + lay.k_off);
    const __half2* meta = reinterpret_cast<const __half2*>(rec + lay.meta_off);
    const uint32_t* vw = reinterpret_cast<const uint32_t*>(rec + lay.v_off);
    const __half* sig = reinterpret_cast<const __half*>(rec + lay.sigma_off);

    // scores: lane = token of the window
    float sc = 0.0f;
    const float c0 = cbk[0];
    for (int c = 0; c < kHeadDim; ++c) {
      const uint32_t code = (kw[lane * kwpt + c / kcpw] >> (p.key_bits * (c % kcpw))) & kmask;
      const float2 ms = __half22float2(meta[c]);
      const float kval = ms.x + ms.y * (cbk[code] - c0);
      sc = fmaf(qs[g][c], kval, sc);
    }
    if (lane >= nvalid) sc = -INFINITY;
    const float m_new = fmaxf(m_run, warp_max(sc));
    const float alpha = expf(m_run - m_new);
    const float pt = lane < nvalid ? expf(sc - m_new) : 0.0f;
    l_run = l_run * alpha + warp_sum(pt);
#pragma unroll
    for (int m = 0; m < kMods; ++m)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[m][j] *= alpha;
    m_run = m_new;

    // per-modality rotated-space values: lane = channels lane + 32 j
    for (int t = 0; t < nvalid; ++t) {
      const float wt = __shfl_sync(0xffffffffu, pt, t) * __half2float(sig[t]);
      const int mod = mods[t];
      const uint32_t* vrow = vw + (t / vcpw) * kHeadDim;
      const int sh = p.value_bits * (t % vcpw);
      float val[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) val[j] = wt * cbv[(vrow[lane + 32 * j] >> sh) & vmask];
      if (mod == 0) {
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[0][j] += val[j];
      } else if (mod == 1) {
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[1][j] += val[j];
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[2][j] += val[j];
      }
    }
  }
  Partial* out = p.partials + ((size_t)b * Hq + qh) * p.num_splits + split;
#pragma unroll
  for (int m = 0; m < kMods; ++m)
#pragma unroll
    for (int j = 0; j < 4; ++j) out->acc[m][lane + 32 * j] = acc[m][j];
  if (lane == 0) {
    out->m = m_run;
    out->l = l_run;
  }
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, int batch, cudaStream_t stream) {
  dim3 grid(p.num_splits, p.num_kv_heads, batch);
  decode_split_k_simt_kernel<<<grid, 32 * p.group, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace omnikv
