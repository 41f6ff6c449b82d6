// combine_inverse_rotate: merges the split-K partials of decode_split_k and
// applies the inverse value rotations, batched across the query heads of a kv
// head (paperpeel.com section 1: inverse value rotations are batched across
// head outputs instead of applied per cached value).
//
// Per (sequence, kv head): M = max_s m_s, l = sum_s l_s e^(m_s - M),
// a_m = sum_s acc_{s,m} e^(m_s - M) / l, then out = sum_m U_m a_m for the G
// query heads at once, i.e. the [G x 384] x [384 x 128] product with the
// stacked bases.
#include "common.cuh"
#include "kernels.h"

namespace omnikv {

namespace {

constexpr int kCombineThreads = 128;

__global__ void __launch_bounds__(kCombineThreads)
combine_inverse_rotate_kernel(const CombineParams p) {
  const int b = blockIdx.y;
  const int kvh = blockIdx.x;
  const int G = p.group;
  const int Hq = p.num_kv_heads * G;
  const int S = p.num_splits;
  const int tid = threadIdx.x;

  __shared__ float a[kMaxGroup][kMods][kHeadDim];

  // merge splits; thread = rotated-space channel
  for (int g = 0; g < G; ++g) {
    const Partial* part = p.partials + ((size_t)b * Hq + kvh * G + g) * S;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, part[s].m);
    float l = 0.0f, acc[kMods] = {0.0f, 0.0f, 0.0f};
    if (M != -INFINITY) {
      for (int s = 0; s < S; ++s) {
        const float ms = part[s].m;
        if (ms == -INFINITY) continue;
        const float e = expf(ms - M);
        l += part[s].l * e;
#pragma unroll
        for (int m = 0; m < kMods; ++m) acc[m] += part[s].acc[m][tid] * e;
      }
    }
    const float inv = l > 0.0f ? 1.0f / l : 0.0f;
#pragma unroll
    for (int m = 0; m < kMods; ++m) a[g][m][tid] = acc[m] * inv;
  }
  __syncthreads();

  // out[g][j] = sum_m sum_c U_m[j][c] a[g][m][c]; warp per output row j,
  // lanes over c (coalesced reads of U_m rows)
  const int warp = tid >> 5, lane = tid & 31;
  const float* Ubase = p.value_rot + (size_t)kvh * kMods * kHeadDim * kHeadDim;
  for (int j = warp; j < kHeadDim; j += kCombineThreads / 32) {
    float part[kMaxGroup];
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g) part[g] = 0.0f;
#pragma unroll
    for (int m = 0; m < kMods; ++m) {
      const float* row = Ubase + ((size_t)m * kHeadDim + j) * kHeadDim;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = lane + 32 * k;
        const float u = row[c];
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g)
          if (g < G) part[g] = fmaf(u, a[g][m][c], part[g]);
      }
    }
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g) {
      if (g >= G) break;
      float v = part[g];
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) p.out[((size_t)b * Hq + kvh * G + g) * kHeadDim + j] = v;
    }
  }
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, int batch, cudaStream_t stream) {
  dim3 grid(p.num_kv_heads, batch);
  combine_inverse_rotate_kernel<<<grid, kCombineThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace omnikv
