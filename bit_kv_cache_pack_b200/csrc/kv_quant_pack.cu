// kv_quant_pack: the OmniKVQuant cache write.
//
// One CTA per (window touched by the new positions, kv head, sequence), or for
// a short append one CTA per sequence (one 128-thread group per kv head).
// Keys (paperpeel.com section 2.2 "Temporal key drift", 3.1 "32-token groups g",
// 3.3 "FP16 minimum m_gc and scale s_gc"): every touched window is re-quantised
// over all its valid tokens -- sign flip + Hadamard butterflies (four threads
// per token), per-channel min / max over the window, fp16 metadata, codes on the
// fixed codebook (decided exactly without the division, see common.cuh), 16 (or
// 8) codes per u32. A window left partial keeps its raw fp16 keys in the tail so
// a later append can re-quantise it. The per-window body is quantize_window
// (append.cuh); values of windows a long write fills completely go to vrot_tc.
// Values (section 2.3 "Modality-aware value rotation"): per token, the fp16
// scale sigma (pairwise-tree sum of squares in a warp), the rotation
// v' = U_m^T v, and codes v'/sigma on the fixed codebook, packed channel-major
// (16 tokens of one channel per u32 for 2-bit codes).
#include "append.cuh"
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace omnikv {

namespace {

constexpr int kMaxAppendHeads = 4;  // kv heads of one sequence in one append CTA (512 threads: up to 128
                                    // registers, so the window body does not spill)

// One CTA per (window touched by the new positions, kv head, sequence); one
// instance per key metadata format.
template <int kMeta>
__global__ void __launch_bounds__(kWriteThreads) kv_quant_pack_kernel(const WriteParams p) {
  __shared__ WindowSmem sm;
  griddep_launch_dependents();
  griddep_wait();  // lengths, records and tail may come from the launch just before
  const int b = blockIdx.z, h = blockIdx.y;
  const int L0 = p.seq_lens[b];
  const int L1 = L0 + p.n_new;
  if (L0 < 0 || L1 > p.cap_tokens) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && h == 0) set_error(p.error_word, OMNIKV_DEVERR_CAPACITY);
    return;
  }
  const int w = L0 / kWindow + blockIdx.x;
  if (w * kWindow >= L1) return;
  quantize_window<kMeta>(p, b, h, w, L0, L1, sm, threadIdx.x, 1, false);
}

// Short appends (n_new < 32): one CTA per sequence, one group of 128 threads
// per kv head; each group re-quantises the (one or two) touched windows in
// order, and the CTA advances the length itself, so no second launch is needed.
template <int kMeta>
__global__ void __launch_bounds__(kWriteThreads * kMaxAppendHeads) kv_append_kernel(const WriteParams p) {
  extern __shared__ __align__(16) uint8_t append_smem[];
  griddep_launch_dependents();
  griddep_wait();
  const int b = blockIdx.x;
  const int grp = threadIdx.x / kWriteThreads, tid = threadIdx.x % kWriteThreads;
  WindowSmem& sm = reinterpret_cast<WindowSmem*>(append_smem)[grp];
  const int L0 = p.seq_lens[b];
  const int L1 = L0 + p.n_new;
  if (L0 < 0 || L1 > p.cap_tokens) {
    if (threadIdx.x == 0) set_error(p.error_word, OMNIKV_DEVERR_CAPACITY);
    return;
  }
  for (int w = L0 / kWindow; w * kWindow < L1; ++w) {
    quantize_window<kMeta>(p, b, grp, w, L0, L1, sm, tid, 1 + grp, true);
    group_sync(1 + grp);  // this window's tail reads are done before the next one writes it
  }
  __syncthreads();  // every group has read the old length
  if (threadIdx.x == 0) p.seq_lens[b] = L1;
}

// One CTA per sequence: copies the raw keys of a partial last window that is
// not the first window touched into the tail, then advances the length.
__global__ void finish_write_kernel(const WriteParams p) {
  griddep_launch_dependents();
  griddep_wait();
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
  if (p.n_new < kWindow && p.num_kv_heads <= kMaxAppendHeads) {
    p.tc_values = 0;
    const size_t smem = sizeof(WindowSmem) * p.num_kv_heads;
    auto kern = p.key_meta == kMetaMx ? kv_append_kernel<kMetaMx>
              : p.key_meta == kMetaTurbo ? kv_append_kernel<kMetaTurbo> : kv_append_kernel<kMetaFp16>;
    if (smem > 48 * 1024) {
      const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    return launch_pdl(kern, dim3(batch), dim3(kWriteThreads * p.num_kv_heads), smem, stream, p);
  }
  p.tc_values = p.n_new >= kWindow ? 1 : 0;  // a write this long can fill whole windows
  const int slots = (p.n_new + kWindow - 1) / kWindow + 1;
  dim3 grid(slots, p.num_kv_heads, batch);
  auto pack = p.key_meta == kMetaMx ? kv_quant_pack_kernel<kMetaMx>
            : p.key_meta == kMetaTurbo ? kv_quant_pack_kernel<kMetaTurbo> : kv_quant_pack_kernel<kMetaFp16>;
  cudaError_t e = launch_pdl(pack, grid, dim3(kWriteThreads), 0, stream, p);
  if (e != cudaSuccess) return e;
  if (p.tc_values) {
    e = launch_vrot_tc(p, batch, stream);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(finish_write_kernel, dim3(batch), dim3(128), 0, stream, p);
}

}  // namespace omnikv
