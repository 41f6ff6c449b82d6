// combine_inverse_rotate: merges the split-K partials of decode_split_k and
// applies the inverse value rotations (paperpeel.com section 1: inverse value
// rotations are applied to head outputs instead of to every cached value).
//
// One CTA per (query head, block of output rows, kv head, sequence), the rows
// split in 4 blocks of 32 when the heads alone would not fill the GPU, else one
// block of 128:
//   0. before waiting on the decode launch: this warp's 4 rows of U_m for the 3
//      modalities go into registers (they do not depend on the decode);
//   1. warp w merges the splits s = w, w + 8, ... as they arrive: a split's (m, l)
//      and its 384 accumulators (three 16-byte vectors per lane) are loaded
//      together, kBatch splits at a time, and folded in with a running maximum
//      (the running sums rescaled when it grows; splits with m = -inf skipped);
//   2. the 8 warps' (max, sum, accumulators) merge through shared memory at their
//      common maximum M: a_m[c] = sum_s acc_{s,m}[c] e^(m_s - M) / l with
//      l = sum_s l_s e^(m_s - M);
//   3. out[j] = sum_m sum_c U_m[j][c] a_m[c] for the block's rows: one warp per 4
//      rows, lanes over c, warp reduction.
// The merge needs no maximum before the first accumulator load, so up to 8 kBatch
// splits are one memory round trip deep. The row blocks of a head merge the same
// partials (read from L2); splitting the rows keeps every step short when there
// are few heads.
// A sequence without tokens (all m_s = -inf) yields zeros.
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace omnikv {

namespace {

constexpr int kCombineThreads = 256;
constexpr int kWarpsC = kCombineThreads / 32;
constexpr int kMaxSplitsSmem = 4096;  // the library's split limit
constexpr int kBatch = 3;             // splits per warp in flight

template <int kRowBlocks>
__global__ void __launch_bounds__(kCombineThreads, 2)
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

  __shared__ __align__(16) float4 wacc[kWarpsC][96];  // each warp's accumulators, at its own max
  __shared__ float wmax[kWarpsC], wsum[kWarpsC];
  __shared__ __align__(16) float a[kMods * kHeadDim];

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

  // ---- 1. each warp folds in its splits as they arrive (running maximum)
  {
    float mw = -INFINITY, lw = 0.0f;
    float4 aw[3] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f),
                    make_float4(0.f, 0.f, 0.f, 0.f)};
    for (int s0 = warp; s0 < S; s0 += kWarpsC * kBatch) {
      float2 ml[kBatch];
      float4 v[kBatch][3];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const int sp = s0 + kWarpsC * i;
        ml[i] = sp < S ? *reinterpret_cast<const float2*>(&part[sp].m) : make_float2(-INFINITY, 0.0f);
        // the accumulators of an empty split (m = -inf) are never written: loaded
        // (the memory is the split's own) but not used
        const float4* src = reinterpret_cast<const float4*>(part[sp < S ? sp : s0].acc);
#pragma unroll
        for (int j = 0; j < 3; ++j) v[i][j] = src[lane + 32 * j];
      }
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        if (ml[i].x == -INFINITY) continue;  // warp-uniform
        const float mn = fmaxf(mw, ml[i].x);
        const float fo = mw == -INFINITY ? 0.0f : expf(mw - mn);
        const float fn = expf(ml[i].x - mn);
        lw = lw * fo + ml[i].y * fn;
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          aw[j].x = fmaf(v[i][j].x, fn, aw[j].x * fo);
          aw[j].y = fmaf(v[i][j].y, fn, aw[j].y * fo);
          aw[j].z = fmaf(v[i][j].z, fn, aw[j].z * fo);
          aw[j].w = fmaf(v[i][j].w, fn, aw[j].w * fo);
        }
        mw = mn;
      }
    }
#pragma unroll
    for (int j = 0; j < 3; ++j) wacc[warp][lane + 32 * j] = aw[j];
    if (lane == 0) {
      wmax[warp] = mw;
      wsum[warp] = lw;
    }
  }
  __syncthreads();

  // ---- 2. the warps' partial merges at their common maximum
  if (tid < 96) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarpsC; ++w) M = fmaxf(M, wmax[w]);
    float l = 0.0f;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kWarpsC; ++w) {
      if (wmax[w] == -INFINITY) continue;
      const float e = expf(wmax[w] - M);
      l = fmaf(wsum[w], e, l);
      const float4 y = wacc[w][tid];
      x.x = fmaf(y.x, e, x.x);
      x.y = fmaf(y.y, e, x.y);
      x.z = fmaf(y.z, e, x.z);
      x.w = fmaf(y.w, e, x.w);
    }
    const float inv = l > 0.0f ? 1.0f / l : 0.0f;
    reinterpret_cast<float4*>(a)[tid] = make_float4(x.x * inv, x.y * inv, x.z * inv, x.w * inv);
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
