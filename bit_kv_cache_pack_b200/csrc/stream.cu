// stream: the streaming / captioning cache policy (paperpeel.com section 3.1,
// "Implementation details": for captioning, keys are quantised every 128 tokens
// in groups of 32 while values keep a 128-token fp16 sliding window before
// quantisation). Readings: key blocks are aligned at absolute positions, so the
// keys of positions [0, KB) are read quantised, KB = 128 floor(T / 128); a value is
// read quantised once it has left the newest 128 tokens, positions [0, VB), VB =
// max(0, T - 128); a quantised key or value is exactly the ordinary write's; the
// others enter attention as the raw fp16 inputs (original basis).
//
// The library writes every record eagerly (omnikv_write_cache, unchanged) and keeps
// the raw fp16 keys and values of the newest 256 positions in a ring (slot
// position mod 256, stream_push_kernel); the policy decides what the decode reads:
//   * the packed body, windows [0, T0 / 32) with T0 = 32 floor(VB / 32), in which
//     every key and value is read quantised: the ordinary decode kernels with their
//     lengths cut to T0 (DecodeParams::stream), splits 0 .. S-1;
//   * the tail, positions [T0, T) (at most 159): stream_tail_kernel, one CTA per
//     (sequence, kv head), CUDA cores: keys before KB dequantised from their
//     records (any key format), the others rotated from the ring; values before VB
//     dequantised per modality (rotated bases), the others summed in the original
//     basis and mapped into modality 0's rotated basis (U_0^T a, so that the
//     combine's U_0 brings them back); written as split S;
//   * the ordinary combine over S + 1 splits.
#include "decode_common.cuh"

namespace omnikv {
namespace {

constexpr int kRing = 256;     // raw positions kept: slot = position mod 256
constexpr int kTailMax = 160;  // tail tokens: T - 32 floor(max(0, T - 128) / 32) <= 159

// Block (i, h, b), 32 threads: token n_new - n_copy + i of the write goes to its
// ring slot (16 threads the key's 256 bytes, 16 the value's).
__global__ void stream_push_kernel(const __half* __restrict__ k_new, const __half* __restrict__ v_new,
                                   const int32_t* __restrict__ seq_lens, __half* __restrict__ ring_k,
                                   __half* __restrict__ ring_v, int n_new, int n_copy) {
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z, H = gridDim.y;
  const int L0 = seq_lens[b];
  if (L0 < 0) return;
  const int j = n_new - n_copy + i;
  const int pos = L0 + j;
  const size_t src = (((size_t)b * H + h) * n_new + j) * kHeadDim;
  const size_t dst = (((size_t)b * H + h) * kRing + (pos % kRing)) * kHeadDim;
  const int lane = threadIdx.x;
  if (lane < 16)
    reinterpret_cast<uint4*>(ring_k + dst)[lane] = reinterpret_cast<const uint4*>(k_new + src)[lane];
  else
    reinterpret_cast<uint4*>(ring_v + dst)[lane - 16] = reinterpret_cast<const uint4*>(v_new + src)[lane - 16];
}

struct TailSmem {
  float q[kMaxGroup * kHeadDim];     // rotated queries (qpos layout), softmax scale folded in
  float s[kTailMax][kMaxGroup];      // scores, then p = exp(score - max)
  float orig[kMaxGroup][kHeadDim];   // raw values' weighted sums, original basis
  float m[kMaxGroup], l[kMaxGroup];
  float cbk[16], cbv[16];
};

__global__ void __launch_bounds__(kThreads) stream_tail_kernel(const DecodeParams p, const __half* __restrict__ ring_k,
                                                              const __half* __restrict__ ring_v, int tail_split) {
  __shared__ TailSmem sm;
  const int kvh = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.group, H = p.num_kv_heads, Hq = H * G;
  rotate_queries(p, b, kvh, sm.q);
  if (tid < 16) {
    sm.cbk[tid] = tid < (1 << p.key_bits) ? p.key_cb[tid] : 0.0f;
    sm.cbv[tid] = tid < (1 << p.value_bits) ? p.val_cb[tid] : 0.0f;
  }
  __syncthreads();
  const int T = max(0, min(p.seq_lens[b], p.cap_tokens));
  const int KB = 128 * (T / 128), VB = max(0, T - 128), T0 = kWindow * (VB / kWindow);
  const int n = T - T0;  // <= 159
  const RecordLayout lay(p.key_bits, p.value_bits, p.key_meta);
  const uint8_t* rec_base = p.records + ((size_t)(b * H + kvh) * p.cap_windows) * lay.bytes;
  const __half* rk = ring_k + (size_t)(b * H + kvh) * kRing * kHeadDim;
  const __half* rv = ring_v + (size_t)(b * H + kvh) * kRing * kHeadDim;
  const int kcpw = 32 / p.key_bits, vcpw = 32 / p.value_bits;
  const uint32_t kmask = (1u << p.key_bits) - 1u, vmask = (1u << p.value_bits) - 1u;

  // ---- scores: warp w takes tokens w, w + 4, ...; lane l holds channels 4l .. 4l+3
  for (int i = warp; i < n; i += kWarps) {
    const int t = T0 + i;
    float x[4];
    if (t < KB) {  // the quantised key, dequantised in the rotated basis
      const uint8_t* rec = rec_base + (size_t)(t / kWindow) * lay.bytes;
      const int slot = t % kWindow;
      const uint32_t* kw = reinterpret_cast<const uint32_t*>(rec + lay.k_off) + slot * (kHeadDim / kcpw);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int c = 4 * lane + r;
        const uint32_t code = (kw[c / kcpw] >> (p.key_bits * (c % kcpw))) & kmask;
        if (p.key_meta == kMetaTurbo) {
          x[r] = __half2float(reinterpret_cast<const __half*>(rec + lay.meta_off)[slot]) * sm.cbk[code];
        } else {
          const float2 ms = p.key_meta == kMetaMx
                                ? mx_meta_channel(rec + lay.meta_off, c)
                                : __half22float2(reinterpret_cast<const __half2*>(rec + lay.meta_off)[c]);
          x[r] = fmaf(ms.y, sm.cbk[code] - sm.cbk[0], ms.x);
        }
      }
    } else {  // the raw key, rotated as the cache's keys are
      const uint2 raw = *reinterpret_cast<const uint2*>(rk + (size_t)(t % kRing) * kHeadDim + 4 * lane);
      const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
      const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
      x[0] = lo.x, x[1] = lo.y, x[2] = hi.x, x[3] = hi.y;
      float sg[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) sg[r] = p.key_signs[4 * lane + r];
      warp_hadamard_rotate(x, sg);
    }
    float d[kMaxGroup];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
      float a = 0.0f;
#pragma unroll
      for (int r = 0; r < 4; ++r) a = fmaf(sm.q[qpos(h, 4 * lane + r)], x[r], a);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      d[h] = a;
    }
    if (lane == 0) {
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) sm.s[i][h] = h < G ? d[h] : -INFINITY;
    }
  }
  __syncthreads();
  // ---- softmax over the tail, per head
  if (tid < kMaxGroup) {
    float mx = -INFINITY;
    for (int i = 0; i < n; ++i) mx = fmaxf(mx, sm.s[i][tid]);
    float l = 0.0f;
    for (int i = 0; i < n; ++i) {
      const float e = (mx == -INFINITY) ? 0.0f : exp2f((sm.s[i][tid] - mx) * kLog2e);
      sm.s[i][tid] = e;
      l += e;
    }
    sm.m[tid] = mx;
    sm.l[tid] = l;
  }
  __syncthreads();
  // ---- values: thread c = channel c
  const int c = tid;
  float acc[kMods][kMaxGroup], org[kMaxGroup];
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    org[h] = 0.0f;
#pragma unroll
    for (int m = 0; m < kMods; ++m) acc[m][h] = 0.0f;
  }
  for (int i = 0; i < n; ++i) {
    const int t = T0 + i;
    if (t < VB) {  // quantised: sigma_t c_code in the rotated basis of the token's modality
      const uint8_t* rec = rec_base + (size_t)(t / kWindow) * lay.bytes;
      const int slot = t % kWindow;
      const uint32_t w = reinterpret_cast<const uint32_t*>(rec + lay.v_off)[(slot / vcpw) * kHeadDim + c];
      const uint32_t code = (w >> (p.value_bits * (slot % vcpw))) & vmask;
      const float v = __half2float(reinterpret_cast<const __half*>(rec + lay.sigma_off)[slot]) * sm.cbv[code];
      const int md = min((int)p.modality[(size_t)b * p.cap_tokens + t], kMods - 1);
#pragma unroll
      for (int m = 0; m < kMods; ++m)
        if (m == md) {
#pragma unroll
          for (int h = 0; h < kMaxGroup; ++h) acc[m][h] = fmaf(sm.s[i][h], v, acc[m][h]);
        }
    } else {  // raw, original basis
      const float v = __half2float(rv[(size_t)(t % kRing) * kHeadDim + c]);
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) org[h] = fmaf(sm.s[i][h], v, org[h]);
    }
  }
  // ---- raw values into modality 0's rotated basis: acc_0 += U_0^T org (U_0 row-major,
  // columns the basis: v' = U^T v)
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) sm.orig[h][c] = org[h];
  __syncthreads();
  const float* U0 = p.value_rot + (size_t)kvh * kMods * kHeadDim * kHeadDim;
  for (int r = 0; r < kHeadDim; ++r) {
    const float u = U0[(size_t)r * kHeadDim + c];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) acc[0][h] = fmaf(u, sm.orig[h][r], acc[0][h]);
  }
  // ---- the tail's partial, split tail_split
  for (int h = 0; h < G; ++h) {
    Partial* out = p.partials + ((size_t)b * Hq + kvh * G + h) * p.num_splits + tail_split;
#pragma unroll
    for (int m = 0; m < kMods; ++m) {
      float a = 0.0f;
#pragma unroll
      for (int hh = 0; hh < kMaxGroup; ++hh)
        if (hh == h) a = acc[m][hh];
      out->acc[m][c] = a;
    }
    if (c == 0) {
      out->m = n > 0 ? sm.m[h] : -INFINITY;
      out->l = n > 0 ? sm.l[h] : 0.0f;
    }
  }
}

}  // namespace

cudaError_t launch_stream_push(const __half* k_new, const __half* v_new, const int32_t* seq_lens, __half* ring_k,
                               __half* ring_v, int batch, int num_kv_heads, int n_new, cudaStream_t stream) {
  const int n_copy = min(n_new, kRing);
  stream_push_kernel<<<dim3(n_copy, num_kv_heads, batch), 32, 0, stream>>>(k_new, v_new, seq_lens, ring_k, ring_v,
                                                                         n_new, n_copy);
  return cudaGetLastError();
}

cudaError_t launch_stream_tail(const DecodeParams& p, const __half* ring_k, const __half* ring_v, int tail_split,
                               cudaStream_t stream) {
  stream_tail_kernel<<<dim3(p.num_kv_heads, p.batch), kThreads, 0, stream>>>(p, ring_k, ring_v, tail_split);
  return cudaGetLastError();
}

}  // namespace omnikv
