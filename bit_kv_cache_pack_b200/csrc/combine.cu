// combine_inverse_rotate: merges the split-K partials of decode_split_k and
// applies the inverse value rotations (paperpeel.com section 1: inverse value
// rotations are applied to head outputs instead of to every cached value).
//
// One CTA per (query head, block of output rows, kv head, sequence), the rows
// split in 4 blocks of 32 when the heads alone would not fill the GPU, else one
// block of 128:
//   0. before waiting on the decode launch: this warp's 4 rows of U_m for the 3
//      modalities go into registers (they do not depend on the decode);
//   1. warp 0: M = max_s m_s, weights e_s = exp(m_s - M), l = sum_s l_s e_s,
//      each lane's (m, l) pairs loaded together;
//   2. a_m[c] = sum_s acc_{s,m}[c] e_s / l, the splits read as 16-byte vectors,
//      two threads per vector column, 16 loads in flight per thread, splits of
//      weight 0 not read;
//   3. out[j] = sum_m sum_c U_m[j][c] a_m[c] for the block's rows: one warp per 4
//      rows, lanes over c, warp reduction.
// The row blocks of a head merge the same partials (read from L2); splitting the
// rows keeps every step one memory round trip deep when there are few heads.
// A sequence without tokens (all m_s = -inf) yields zeros.
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace omnikv {

namespace {

constexpr int kCombineThreads = 256;
constexpr int kWarpsC = kCombineThreads / 32;
constexpr int kMaxSplitsSmem = 4096;

template <int kRowBlocks>
__global__ void __launch_bounds__(kCombineThreads)
combine_inverse_rotate_kernel(const CombineParams p) {
  constexpr int kRowsPerWarp = kHeadDim / kRowBlocks / kWarpsC;  // 4 or 16
  const int g = blockIdx.x / kRowBlocks;  // query head within the group
  const int rb = blockIdx.x % kRowBlocks;
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int G = p.group;
  const int Hq = p.num_kv_heads * G;
  const int S = p.num_splits;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qh = kvh * G + g;

  __shared__ float w[kMaxSplitsSmem];   // split maxima, then weights
  __shared__ float wl[kMaxSplitsSmem];  // split denominators
  __shared__ __align__(16) float4 red[2][96];
  __shared__ __align__(16) float a[kMods * kHeadDim];
  __shared__ float s_l;

  griddep_launch_dependents();
  // ---- 0. value-basis rows (constant input): this warp's rows j0 .., lanes over
  // c; with 4 row blocks all of them (4 rows x 3 modalities) are loaded before
  // the wait, with one block the first 4
  const int j0 = rb * (kHeadDim / kRowBlocks) + warp * kRowsPerWarp;
  const float* Ubase = p.value_rot + (size_t)kvh * kMods * kHeadDim * kHeadDim;
  constexpr int kPre = 4;
  float4 u[kPre][kMods];
#pragma unroll
  for (int r = 0; r < kPre; ++r)
#pragma unroll
    for (int m = 0; m < kMods; ++m)
      u[r][m] = reinterpret_cast<const float4*>(Ubase + ((size_t)m * kHeadDim + j0 + r) * kHeadDim)[lane];

  griddep_wait();  // the partials come from the decode launch just before
  const Partial* part = p.partials + ((size_t)b * Hq + qh) * S;
  if (p.len_add > 0 && blockIdx.x == 0 && kvh == 0 && tid == 0) {  // decode step: advance the length
    const int L = p.seq_lens[b];
    if (L >= 0 && L + p.len_add <= p.cap_tokens) p.seq_lens[b] = L + p.len_add;
  }

  // ---- 1. split weights (warp 0): every lane loads (m, l) of all its splits at
  // once (one memory round trip for up to 128 splits), then the max, the weights
  // e_s and l = sum_s l_s e_s
  if (warp == 0) {
    constexpr int kPer = 4;  // splits per lane per pass
    float M = -INFINITY;
    for (int base = 0; base < S; base += 32 * kPer) {
      float2 ml[kPer];
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int s = base + 32 * i + lane;
        ml[i] = s < S ? *reinterpret_cast<const float2*>(&part[s].m) : make_float2(-INFINITY, 0.0f);
      }
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int s = base + 32 * i + lane;
        if (s < S) {
          w[s] = ml[i].x;
          wl[s] = ml[i].y;
        }
        M = fmaxf(M, ml[i].x);
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float l = 0.0f;
    for (int s = lane; s < S; s += 32) {
      const float ms = w[s];
      const float e = (ms == -INFINITY) ? 0.0f : expf(ms - M);
      w[s] = e;
      if (e != 0.0f) l += wl[s] * e;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) s_l = l;
  }
  __syncthreads();

  // ---- 2. weighted sum over splits: column c4 (of 96 float4), half h of the
  // splits, kU loads in flight per thread (splits of weight 0 are not read)
  {
    const int c4 = tid & 127, h = tid >> 7;
    if (c4 < 96) {
      constexpr int kU = 16;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s0 = h; s0 < S; s0 += 2 * kU) {
        float4 v[kU];
        float e[kU];
#pragma unroll
        for (int i = 0; i < kU; ++i) {
          const int s = s0 + 2 * i;
          e[i] = s < S ? w[s] : 0.0f;
          v[i] = e[i] != 0.0f ? reinterpret_cast<const float4*>(part[s].acc)[c4] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int i = 0; i < kU; ++i) {
          acc.x = fmaf(v[i].x, e[i], acc.x);
          acc.y = fmaf(v[i].y, e[i], acc.y);
          acc.z = fmaf(v[i].z, e[i], acc.z);
          acc.w = fmaf(v[i].w, e[i], acc.w);
        }
      }
      red[h][c4] = acc;
    }
  }
  __syncthreads();
  if (tid < 96) {
    const float inv = s_l > 0.0f ? 1.0f / s_l : 0.0f;
    const float4 x = red[0][tid], y = red[1][tid];
    reinterpret_cast<float4*>(a)[tid] =
        make_float4((x.x + y.x) * inv, (x.y + y.y) * inv, (x.z + y.z) * inv, (x.w + y.w) * inv);
  }
  __syncthreads();

  // ---- 3. out[j] = sum_m U_m[j][:] . a_m for this warp's rows, 4 at a time
  float* out = p.out + ((size_t)b * Hq + qh) * kHeadDim;
  float4 xa[kMods];
#pragma unroll
  for (int m = 0; m < kMods; ++m) xa[m] = reinterpret_cast<const float4*>(a + m * kHeadDim)[lane];
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; rr += kPre) {
    if (rr > 0) {
#pragma unroll
      for (int r = 0; r < kPre; ++r)
#pragma unroll
        for (int m = 0; m < kMods; ++m)
          u[r][m] = reinterpret_cast<const float4*>(Ubase + ((size_t)m * kHeadDim + j0 + rr + r) * kHeadDim)[lane];
    }
#pragma unroll
    for (int r = 0; r < kPre; ++r) {
      float v = 0.0f;
#pragma unroll
      for (int m = 0; m < kMods; ++m) {
        v = fmaf(u[r][m].x, xa[m].x, v);
        v = fmaf(u[r][m].y, xa[m].y, v);
        v = fmaf(u[r][m].z, xa[m].z, v);
        v = fmaf(u[r][m].w, xa[m].w, v);
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) out[j0 + rr + r] = v;
    }
  }
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, int batch, cudaStream_t stream) {
  if (p.num_splits > kMaxSplitsSmem) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long heads = (long long)batch * p.num_kv_heads * p.group;
  if (heads >= sms) {  // enough heads to fill the GPU: one CTA per head
    dim3 grid(p.group, p.num_kv_heads, batch);
    return launch_pdl(combine_inverse_rotate_kernel<1>, grid, dim3(kCombineThreads), 0, stream, p);
  }
  dim3 grid(p.group * 4, p.num_kv_heads, batch);
  return launch_pdl(combine_inverse_rotate_kernel<4>, grid, dim3(kCombineThreads), 0, stream, p);
}

}  // namespace omnikv
