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
//   * the tail, positions [T0, T) (at most 159): stream_tail_kernel, four CTAs of 8
//     warps per (sequence, kv head), each a chunk of up to 40 positions and its own
//     split, CUDA cores: the tail's keys and values are
//     first staged in shared memory as fp32 in one pass (keys before KB
//     dequantised from their records in the rotated basis, any key format, the
//     others raw in the original basis and scored against the unrotated query;
//     values before VB dequantised per modality in the rotated bases, the others
//     raw), then scored, softmaxed and summed; the raw values' sums are mapped
//     into modality 0's rotated basis (U_0^T a, so that the combine's U_0 brings
//     them back); written as splits S .. S+3;
//   * the ordinary combine over S + 4 splits.
#include "decode_common.cuh"

namespace omnikv {
namespace {

constexpr int kRing = 256;     // raw positions kept: slot = position mod 256
constexpr int kTailChunks = kStreamTailSplits;  // tail CTAs per (sequence, kv head), each its own split
constexpr int kTailMax = 40;    // tail tokens per CTA: the tail, T - 32 floor(max(0, T - 128) / 32) <= 159, in 4 chunks

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

constexpr int kTailThreads = 256;
constexpr int kRowPad = kHeadDim + 1;  // padded rows: threads reading different rows hit different banks

// A chunk of the tail in shared memory (dynamic, ~77 KB): its keys and values as
// fp32 (keys rotated where quantised, original basis where raw; the scores pick the
// matching query), loaded in one pass so the global reads are all in flight.
struct TailSmem {
  float kx[kTailMax][kRowPad];
  float vx[kTailMax][kHeadDim];
  float qr[kMaxGroup][kRowPad];  // rotated queries q' (natural channel order), softmax scale folded in
  float qo[kMaxGroup][kRowPad];  // original-basis queries times the softmax scale
  float s[kTailMax][kMaxGroup];  // scores, then p = exp(score - max)
  float orig[kMaxGroup][kHeadDim];
  float part[kMods + 1][kMaxGroup][kHeadDim];  // the second half of the tokens' value sums
  float qtmp[kMaxGroup * kHeadDim];
  float m[kMaxGroup], l[kMaxGroup];
  float cbk[16], cbv[16];
  int mods[kTailMax];
};

__global__ void __launch_bounds__(kTailThreads) stream_tail_kernel(const DecodeParams p,
                                                                  const __half* __restrict__ ring_k,
                                                                  const __half* __restrict__ ring_v, int tail_split) {
  extern __shared__ __align__(16) uint8_t tail_smem_raw[];
  TailSmem& sm = *reinterpret_cast<TailSmem*>(tail_smem_raw);
  const int kvh = blockIdx.x, b = blockIdx.y, chunk = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.group, H = p.num_kv_heads, Hq = H * G;
  rotate_queries<kTailThreads / 32>(p, b, kvh, sm.qtmp);
  if (tid < 16) {
    sm.cbk[tid] = tid < (1 << p.key_bits) ? p.key_cb[tid] : 0.0f;
    sm.cbv[tid] = tid < (1 << p.value_bits) ? p.val_cb[tid] : 0.0f;
  }
  const int T = max(0, min(p.seq_lens[b], p.cap_tokens));
  const int KB = 128 * (T / 128), VB = max(0, T - 128);
  // this CTA's chunk of the tail: positions [T0, T0 + n)
  const int Tt = kWindow * (VB / kWindow);
  const int T0 = min(T, Tt + kTailMax * chunk);
  const int n = min(kTailMax, T - T0);
  const RecordLayout lay(p.key_bits, p.value_bits, p.key_meta);
  const uint8_t* rec_base = p.records + ((size_t)(b * H + kvh) * p.cap_windows) * lay.bytes;
  const __half* rk = ring_k + (size_t)(b * H + kvh) * kRing * kHeadDim;
  const __half* rv = ring_v + (size_t)(b * H + kvh) * kRing * kHeadDim;
  const int kcpw = 32 / p.key_bits, vcpw = 32 / p.value_bits;
  const uint32_t kmask = (1u << p.key_bits) - 1u, vmask = (1u << p.value_bits) - 1u;
  for (int e = tid; e < kMaxGroup * kHeadDim; e += kTailThreads) {  // original-basis queries
    const int h = e / kHeadDim, c = e % kHeadDim;
    sm.qo[h][c] = h < G ? __half2float(p.q[((size_t)b * Hq + kvh * G + h) * kHeadDim + c]) * inv_sqrt_d() : 0.0f;
  }
  if (tid < n) sm.mods[tid] = min((int)p.modality[(size_t)b * p.cap_tokens + T0 + tid], kMods - 1);
  __syncthreads();
  for (int e = tid; e < kMaxGroup * kHeadDim; e += kTailThreads) {  // rotated queries in natural order
    const int h = e / kHeadDim, c = e % kHeadDim;
    sm.qr[h][c] = sm.qtmp[qpos(h, c)];
  }
  // ---- every key and value of the tail as fp32, thread (token i, channel c); one
  // branch-free loop per region so that the loads of many elements are in flight
  const int nkq = min(n, max(0, KB - T0)), nvq = min(n, max(0, VB - T0));  // quantised prefixes
#pragma unroll 8
  for (int e = nkq * kHeadDim + tid; e < n * kHeadDim; e += kTailThreads) {  // raw keys
    const int i = e / kHeadDim, c = e % kHeadDim;
    sm.kx[i][c] = __half2float(rk[(size_t)((T0 + i) % kRing) * kHeadDim + c]);
  }
#pragma unroll 8
  for (int e = nvq * kHeadDim + tid; e < n * kHeadDim; e += kTailThreads) {  // raw values
    const int i = e / kHeadDim, c = e % kHeadDim;
    sm.vx[i][c] = __half2float(rv[(size_t)((T0 + i) % kRing) * kHeadDim + c]);
  }
  if (p.key_meta == kMetaTurbo) {  // quantised keys, rotated basis: ksigma_t c_code
#pragma unroll 4
    for (int e = tid; e < nkq * kHeadDim; e += kTailThreads) {
      const int i = e / kHeadDim, c = e % kHeadDim, t = T0 + i, slot = t % kWindow;
      const uint8_t* rec = rec_base + (size_t)(t / kWindow) * lay.bytes;
      const uint32_t w = reinterpret_cast<const uint32_t*>(rec + lay.k_off)[slot * (kHeadDim / kcpw) + c / kcpw];
      const float sg = __half2float(reinterpret_cast<const __half*>(rec + lay.meta_off)[slot]);
      sm.kx[i][c] = sg * sm.cbk[(w >> (p.key_bits * (c % kcpw))) & kmask];
    }
  } else if (p.key_meta == kMetaMx) {  // quantised keys: m + s (c_code - c_0), MXFP4 metadata
#pragma unroll 4
    for (int e = tid; e < nkq * kHeadDim; e += kTailThreads) {
      const int i = e / kHeadDim, c = e % kHeadDim, t = T0 + i, slot = t % kWindow;
      const uint8_t* rec = rec_base + (size_t)(t / kWindow) * lay.bytes;
      const uint32_t w = reinterpret_cast<const uint32_t*>(rec + lay.k_off)[slot * (kHeadDim / kcpw) + c / kcpw];
      const float2 ms = mx_meta_channel(rec + lay.meta_off, c);
      sm.kx[i][c] = fmaf(ms.y, sm.cbk[(w >> (p.key_bits * (c % kcpw))) & kmask] - sm.cbk[0], ms.x);
    }
  } else {  // quantised keys: m + s (c_code - c_0), fp16 metadata
#pragma unroll 4
    for (int e = tid; e < nkq * kHeadDim; e += kTailThreads) {
      const int i = e / kHeadDim, c = e % kHeadDim, t = T0 + i, slot = t % kWindow;
      const uint8_t* rec = rec_base + (size_t)(t / kWindow) * lay.bytes;
      const uint32_t w = reinterpret_cast<const uint32_t*>(rec + lay.k_off)[slot * (kHeadDim / kcpw) + c / kcpw];
      const float2 ms = __half22float2(reinterpret_cast<const __half2*>(rec + lay.meta_off)[c]);
      sm.kx[i][c] = fmaf(ms.y, sm.cbk[(w >> (p.key_bits * (c % kcpw))) & kmask] - sm.cbk[0], ms.x);
    }
  }
#pragma unroll 4
  for (int e = tid; e < nvq * kHeadDim; e += kTailThreads) {  // quantised values: sigma_t c_code
    const int i = e / kHeadDim, c = e % kHeadDim, t = T0 + i, slot = t % kWindow;
    const uint8_t* rec = rec_base + (size_t)(t / kWindow) * lay.bytes;
    const uint32_t w = reinterpret_cast<const uint32_t*>(rec + lay.v_off)[(slot / vcpw) * kHeadDim + c];
    const float sg = __half2float(reinterpret_cast<const __half*>(rec + lay.sigma_off)[slot]);
    sm.vx[i][c] = sg * sm.cbv[(w >> (p.value_bits * (slot % vcpw))) & vmask];
  }
  __syncthreads();
  // ---- scores: pair (token i, head h); the query in the key's basis
  for (int e = tid; e < n * kMaxGroup; e += kTailThreads) {
    const int i = e / kMaxGroup, h = e % kMaxGroup;
    const float* qv = (T0 + i < KB) ? sm.qr[h] : sm.qo[h];
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
    for (int c = 0; c < kHeadDim; c += 4) {
      a0 = fmaf(qv[c], sm.kx[i][c], a0);
      a1 = fmaf(qv[c + 1], sm.kx[i][c + 1], a1);
      a2 = fmaf(qv[c + 2], sm.kx[i][c + 2], a2);
      a3 = fmaf(qv[c + 3], sm.kx[i][c + 3], a3);
    }
    sm.s[i][h] = h < G ? (a0 + a1) + (a2 + a3) : -INFINITY;
  }
  __syncthreads();
  // ---- softmax over the tail: warp h, lanes over the tokens
  {
    const int h = warp;
    float mx = -INFINITY;
    for (int i = lane; i < n; i += 32) mx = fmaxf(mx, sm.s[i][h]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float l = 0.0f;
    for (int i = lane; i < n; i += 32) {
      const float e = (mx == -INFINITY) ? 0.0f : exp2f((sm.s[i][h] - mx) * kLog2e);
      sm.s[i][h] = e;
      l += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      sm.m[h] = mx;
      sm.l[h] = l;
    }
  }
  __syncthreads();
  // ---- values: channel c, tokens of parity `half` (the two halves summed below)
  const int c = tid % kHeadDim, half = tid / kHeadDim;
  float acc[kMods][kMaxGroup], org[kMaxGroup];
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    org[h] = 0.0f;
#pragma unroll
    for (int m = 0; m < kMods; ++m) acc[m][h] = 0.0f;
  }
  for (int i = half; i < n; i += 2) {
    const float v = sm.vx[i][c];
    if (T0 + i < VB) {
      const int md = sm.mods[i];
#pragma unroll
      for (int m = 0; m < kMods; ++m)
        if (m == md) {
#pragma unroll
          for (int h = 0; h < kMaxGroup; ++h) acc[m][h] = fmaf(sm.s[i][h], v, acc[m][h]);
        }
    } else {
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) org[h] = fmaf(sm.s[i][h], v, org[h]);
    }
  }
  if (half == 1) {
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
#pragma unroll
      for (int m = 0; m < kMods; ++m) sm.part[m][h][c] = acc[m][h];
      sm.part[kMods][h][c] = org[h];
    }
  }
  __syncthreads();
  if (half == 0) {
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
#pragma unroll
      for (int m = 0; m < kMods; ++m) acc[m][h] += sm.part[m][h][c];
      sm.orig[h][c] = org[h] + sm.part[kMods][h][c];
    }
  }
  __syncthreads();
  if (half != 0) return;
  // ---- raw values into modality 0's rotated basis: acc_0 += U_0^T orig (U_0 row-major,
  // columns the basis: v' = U^T v)
  const float* U0 = p.value_rot + (size_t)kvh * kMods * kHeadDim * kHeadDim;
#pragma unroll 8
  for (int r = 0; r < kHeadDim; ++r) {
    const float u = U0[(size_t)r * kHeadDim + c];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) acc[0][h] = fmaf(u, sm.orig[h][r], acc[0][h]);
  }
  // ---- the chunk's partial, split tail_split + chunk
  for (int h = 0; h < G; ++h) {
    Partial* out = p.partials + ((size_t)b * Hq + kvh * G + h) * p.num_splits + tail_split + chunk;
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
  const int smem = (int)sizeof(TailSmem);
  const cudaError_t e = cudaFuncSetAttribute(stream_tail_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  stream_tail_kernel<<<dim3(p.num_kv_heads, p.batch, kTailChunks), kTailThreads, smem, stream>>>(p, ring_k, ring_v,
                                                                                                 tail_split);
  return cudaGetLastError();
}

}  // namespace omnikv
