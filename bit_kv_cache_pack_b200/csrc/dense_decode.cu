// dense_decode_bf16: split-K decode attention over an ordinary (unquantised)
// bf16 KV cache -- the reference point the 2-bit kernels are measured against
// (the same context read at 512 B per token and kv head instead of 82 B). Not
// part of the OmniKVQuant method.
//
// One CTA of 4 warps per (split, kv head, sequence); split s covers the
// 32-token chunks [s C, (s+1) C). Warp w streams chunks w, w+4, ... of its split
// through a 2-stage ring of 1-D bulk copies (K and V rows of the chunk); per
// 16-token tile: scores with mma.sync m16n8k16 bf16 (A = K rows via ldmatrix,
// B = the 8 query heads of the group, bf16), online softmax, P (bf16) times V
// (A = V^T via ldmatrix.trans). The warps merge, one partial per query head;
// a second kernel merges the splits (log-sum-exp) into fp32 outputs.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace omnikv {

namespace {

constexpr int kDWarps = 4;
constexpr int kDThreads = 32 * kDWarps;
constexpr int kDStages = 2;
constexpr int kChunk = 32;                                 // tokens per bulk copy
constexpr int kRowBytes = kHeadDim * 2;                    // 256 B per token row
constexpr int kDStageBytes = 2 * kChunk * kRowBytes;       // K + V rows: 16 KB
constexpr uint64_t kDWaitNs = 2000000000ull;
constexpr float kDLog2e = 1.4426950408889634f;

struct __align__(128) DenseSmem {
  uint8_t stage[kDWarps][kDStages][kDStageBytes];  // 128 KB
  uint64_t bar[kDWarps][kDStages];
  float mw[kDWarps][kMaxGroup];
  float merge[kMaxGroup][kHeadDim + 1];
  float lsum[kMaxGroup];
};

__device__ __forceinline__ void ldmatrix_x4(uint32_t r[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t r[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

__device__ __forceinline__ void mma_bf16_16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf162(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// XOR swizzle of the 16-byte chunks of a 256-byte token row, so that ldmatrix
// (8 rows x 16 B per matrix) reads 8 different bank groups.
__device__ __forceinline__ int rowchunk(int row, int chunk) { return row * kRowBytes + ((chunk ^ (row & 7)) << 4); }

__global__ void __launch_bounds__(kDThreads, 1) dense_split_kernel(const DenseParams p) {
  extern __shared__ uint8_t dsm_raw[];
  DenseSmem& sm = *reinterpret_cast<DenseSmem*>((reinterpret_cast<uintptr_t>(dsm_raw) + 127) & ~uintptr_t(127));
  const int b = blockIdx.z, kvh = blockIdx.y, split = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int G = p.group, Hq = p.num_kv_heads * G;
  const int T = max(0, min(p.seq_lens[b], p.cap_tokens));
  const int nc = (T + kChunk - 1) / kChunk;
  const int c0 = min(split * p.split_chunks, nc), c1 = min(c0 + p.split_chunks, nc);
  const int nmine = (c1 - c0 > warp) ? (c1 - c0 - warp + kDWarps - 1) / kDWarps : 0;
  const size_t head_off = ((size_t)b * p.num_kv_heads + kvh) * p.cap_tokens * kHeadDim;
  const __nv_bfloat16* kbase = p.k + head_off;
  const __nv_bfloat16* vbase = p.v + head_off;

  // query fragments (B operand): head g, channels 16 kc + {2t, 2t+1, 2t+8, 2t+9}, times 1/sqrt(128)
  uint32_t qf[8][2];
  {
    const __nv_bfloat16* q = p.q + ((size_t)b * Hq + kvh * G + min(g, G - 1)) * kHeadDim;
    const float sc = g < G ? 0.08838834764831845f : 0.0f;
#pragma unroll
    for (int kc = 0; kc < 8; ++kc) {
      const float x0 = __bfloat162float(q[16 * kc + 2 * t]) * sc, x1 = __bfloat162float(q[16 * kc + 2 * t + 1]) * sc;
      const float x2 = __bfloat162float(q[16 * kc + 2 * t + 8]) * sc, x3 = __bfloat162float(q[16 * kc + 2 * t + 9]) * sc;
      qf[kc][0] = pack_bf162(x0, x1);
      qf[kc][1] = pack_bf162(x2, x3);
    }
  }

  // ring: chunk i of this warp -> stage i % 2; rows are swizzled after arrival
  auto issue = [&](int i) {
    const int ch = c0 + warp + kDWarps * i;
    uint64_t* bar = &sm.bar[warp][i % kDStages];
    uint8_t* dst = &sm.stage[warp][i % kDStages][0];
    const int ntok = min(kChunk, T - ch * kChunk);
    const uint32_t bytes = (uint32_t)ntok * kRowBytes;
    mbar_arrive_expect_tx(bar, 2 * bytes);
    bulk_copy_g2s(dst, kbase + (size_t)ch * kChunk * kHeadDim, bytes, bar);
    bulk_copy_g2s(dst + kChunk * kRowBytes, vbase + (size_t)ch * kChunk * kHeadDim, bytes, bar);
  };
  if (lane == 0) {
    for (int s = 0; s < kDStages; ++s) mbar_init(&sm.bar[warp][s], 1);
    fence_barrier_init();
    for (int i = 0; i < kDStages && i < nmine; ++i) issue(i);
  }
  __syncwarp();

  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float acc[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[mt][r] = 0.f;
  int failed_at = -1;

  for (int i = 0; i < nmine; ++i) {
    const int s = i % kDStages;
    const int ch = c0 + warp + kDWarps * i;
    if (!mbar_wait_bounded(&sm.bar[warp][s], (i / kDStages) & 1, kDWaitNs)) {
      failed_at = i;
      break;
    }
    uint8_t* kst = &sm.stage[warp][s][0];
    uint8_t* vst = kst + kChunk * kRowBytes;
    const int ntok = min(kChunk, T - ch * kChunk);
    // swizzle rows in place: each lane permutes one row's chunks (lane = row);
    // rows past the chunk's tokens (never copied) become zero
    {
      uint4 tmp[16];
      const uint4* kr = reinterpret_cast<const uint4*>(kst + lane * kRowBytes);
      const uint4* vr = reinterpret_cast<const uint4*>(vst + lane * kRowBytes);
      const bool live = lane < ntok;
#pragma unroll
      for (int c = 0; c < 16; ++c) tmp[c] = live ? kr[c] : make_uint4(0u, 0u, 0u, 0u);
      __syncwarp();
#pragma unroll
      for (int c = 0; c < 16; ++c) *reinterpret_cast<uint4*>(kst + rowchunk(lane, c)) = tmp[c];
#pragma unroll
      for (int c = 0; c < 16; ++c) tmp[c] = live ? vr[c] : make_uint4(0u, 0u, 0u, 0u);
      __syncwarp();
#pragma unroll
      for (int c = 0; c < 16; ++c) *reinterpret_cast<uint4*>(vst + rowchunk(lane, c)) = tmp[c];
      __syncwarp();
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      // scores: A = K rows 16h .. 16h+15 (ldmatrix: matrices = rows 0-7 / 8-15 x chunk 2kc / 2kc+1)
      float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kc = 0; kc < 8; ++kc) {
        uint32_t a[4];
        const int row = 16 * h + (lane & 15);
        const int chunk = 2 * kc + (lane >> 4);
        ldmatrix_x4(a, kst + rowchunk(row, chunk));
        mma_bf16_16816(d, a, qf[kc][0], qf[kc][1]);
      }
      const int tA = 16 * h + g, tB = tA + 8;
      float sc[4] = {tA < ntok ? d[0] : -INFINITY, tA < ntok ? d[1] : -INFINITY, tB < ntok ? d[2] : -INFINITY,
                     tB < ntok ? d[3] : -INFINITY};
      float mx0 = fmaxf(sc[0], sc[2]), mx1 = fmaxf(sc[1], sc[3]);
#pragma unroll
      for (int o = 4; o <= 16; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
      const float a0 = exp2f((m_run[0] - mn0) * kDLog2e), a1 = exp2f((m_run[1] - mn1) * kDLog2e);
      m_run[0] = mn0;
      m_run[1] = mn1;
      l_run[0] *= a0;
      l_run[1] *= a1;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        acc[mt][0] *= a0;
        acc[mt][1] *= a1;
        acc[mt][2] *= a0;
        acc[mt][3] *= a1;
      }
      const float p0 = exp2f((sc[0] - mn0) * kDLog2e), p1 = exp2f((sc[1] - mn1) * kDLog2e);
      const float p2 = exp2f((sc[2] - mn0) * kDLog2e), p3 = exp2f((sc[3] - mn1) * kDLog2e);
      l_run[0] += p0 + p2;
      l_run[1] += p1 + p3;
      const uint32_t b0 = movmatrix_trans(pack_bf162(p0, p1)), b1 = movmatrix_trans(pack_bf162(p2, p3));
      // values: A = V^T (channels 16 mt .. x tokens 16h ..) via ldmatrix.trans
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        uint32_t a[4];
        // matrices: (tok 0-7, ch 0-7), (tok 0-7, ch 8-15), (tok 8-15, ch 0-7), (tok 8-15, ch 8-15) of the tile,
        // transposed -> A rows = channels, columns = tokens
        const int row = 16 * h + (lane & 7) + ((lane >> 4) << 3);
        const int chunk = 2 * mt + ((lane >> 3) & 1);
        ldmatrix_x4_trans(a, vst + rowchunk(row, chunk));
        mma_bf16_16816(acc[mt], a, b0, b1);
      }
    }
    __syncwarp();
    if (lane == 0 && i + kDStages < nmine) {
      fence_proxy_async_smem();
      issue(i + kDStages);
    }
  }
  if (__any_sync(0xffffffffu, failed_at >= 0)) {
    const int f = __shfl_sync(0xffffffffu, failed_at, 0);
    if (lane == 0) set_error(p.error_word, OMNIKV_DEVERR_TIMEOUT);
    for (int j = f; j < nmine && j < f + kDStages; ++j)
      mbar_wait_bounded(&sm.bar[warp][j % kDStages], (j / kDStages) & 1, kDWaitNs);
    m_run[0] = m_run[1] = -INFINITY;
    l_run[0] = l_run[1] = 0.f;
  }
#pragma unroll
  for (int o = 4; o <= 16; o <<= 1) {
    l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], o);
    l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], o);
  }
  // ---- merge the warps (shared-memory reduction, one warp at a time)
  if (g == 0) {
    sm.mw[warp][2 * t] = m_run[0];
    sm.mw[warp][2 * t + 1] = m_run[1];
  }
  for (int i = threadIdx.x; i < kMaxGroup * (kHeadDim + 1); i += kDThreads) (&sm.merge[0][0])[i] = 0.f;
  if (threadIdx.x < kMaxGroup) sm.lsum[threadIdx.x] = 0.f;
  __syncthreads();
  float M[2], f[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    M[j] = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDWarps; ++w) M[j] = fmaxf(M[j], sm.mw[w][2 * t + j]);
    f[j] = m_run[j] == -INFINITY ? 0.f : exp2f((m_run[j] - M[j]) * kDLog2e);
  }
  for (int w = 0; w < kDWarps; ++w) {
    if (warp == w) {
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        // acc[mt]: (channel 16 mt + g, heads 2t, 2t+1), (channel 16 mt + g + 8, ...)
        sm.merge[2 * t][16 * mt + g] += acc[mt][0] * f[0];
        sm.merge[2 * t + 1][16 * mt + g] += acc[mt][1] * f[1];
        sm.merge[2 * t][16 * mt + g + 8] += acc[mt][2] * f[0];
        sm.merge[2 * t + 1][16 * mt + g + 8] += acc[mt][3] * f[1];
      }
      if (g == 0) {
        sm.lsum[2 * t] += l_run[0] * f[0];
        sm.lsum[2 * t + 1] += l_run[1] * f[1];
      }
    }
    __syncthreads();
  }
  for (int hh = warp; hh < G; hh += kDWarps) {
    float* out = p.partials + (((size_t)b * Hq + kvh * G + hh) * p.num_splits + split) * kDensePartialFloats;
#pragma unroll
    for (int j = 0; j < 4; ++j) out[lane + 32 * j] = sm.merge[hh][lane + 32 * j];
    if (lane == 0) {
      float mm = -INFINITY;
#pragma unroll
      for (int w = 0; w < kDWarps; ++w) mm = fmaxf(mm, sm.mw[w][hh]);
      out[kHeadDim] = mm;
      out[kHeadDim + 1] = sm.lsum[hh];
    }
  }
}

__global__ void dense_combine_kernel(const DenseParams p) {
  const int qh = blockIdx.x, b = blockIdx.y;
  const int Hq = p.num_kv_heads * p.group, S = p.num_splits;
  const float* part = p.partials + ((size_t)b * Hq + qh) * S * kDensePartialFloats;
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, part[s * kDensePartialFloats + kHeadDim]);
  float l = 0.f, acc = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < S; ++s) {
      const float ms = part[s * kDensePartialFloats + kHeadDim];
      if (ms == -INFINITY) continue;
      const float e = expf(ms - M);
      l += part[s * kDensePartialFloats + kHeadDim + 1] * e;
      acc += part[s * kDensePartialFloats + threadIdx.x] * e;
    }
  }
  p.out[((size_t)b * Hq + qh) * kHeadDim + threadIdx.x] = l > 0.f ? acc / l : 0.f;
}

}  // namespace

size_t dense_smem_bytes() { return sizeof(DenseSmem) + 128; }

cudaError_t launch_dense(const DenseParams& p, int batch, cudaStream_t stream) {
  const int smem = (int)dense_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(dense_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dense_split_kernel<<<dim3(p.num_splits, p.num_kv_heads, batch), kDThreads, smem, stream>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  dense_combine_kernel<<<dim3(p.num_kv_heads * p.group, batch), kHeadDim, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace omnikv
