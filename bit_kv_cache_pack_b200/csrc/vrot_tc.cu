// vrot_tc: the per-modality value rotation of the cache write on 5th-generation
// tensor cores (tcgen05 / TMEM), for every 32-token window that a write fills
// completely (paperpeel.com section 2.3 "Modality-aware value rotation": each
// value is rotated by the basis U_m of its modality m before quantisation).
//
// One CTA (4 warps) per tile of 128 tokens (4 whole windows) of one (sequence,
// kv head):
//   * A = the tile's fp16 values, [128 tokens x 128 channels], exact;
//     B = U_m^T split into fp16 high and low parts (U = hi + lo to ~22 bits);
//     both in shared memory in the K-major 128-byte-swizzled layout, written with
//     16-byte stores whose chunk index is XOR-ed with the row (conflict free);
//   * one elected thread issues tcgen05.mma kind::f16 (M = N = 128, K = 16,
//     8 k-steps x {hi, lo}) into a 128-column fp32 accumulator in TMEM and
//     commits to an mbarrier (bounded wait);
//   * one pass per modality present in the tile: warp w reads TMEM lanes
//     32w .. 32w+31 (= window w of the tile, one token per thread) with
//     tcgen05.ld, and the tokens of that modality compute their codes
//     code = #{j : v'_c / sigma16 > t_j} (sigma from the unrotated fp16 value,
//     pairwise tree in fp32, as in the per-token path);
//   * codes are transposed through shared memory into the channel-major value
//     words (16 tokens of one channel per u32) and written with sigma.
// The key half of these windows, partial windows and one-token appends are
// handled by kv_quant_pack.
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace omnikv {

namespace {

constexpr int kTile = 128;                 // tokens per tile = MMA M
constexpr int kVThreads = 128;
constexpr uint32_t kTmemCols = 128;        // one fp32 accumulator of N = 128 columns
constexpr uint64_t kMmaWaitNs = 2000000000ull;

// operand: [2 k-atoms][128 rows][128 B], 16-byte chunks XOR-swizzled by row % 8
constexpr int kOperandBytes = 2 * 128 * 128;   // 32 KB of fp16

struct __align__(1024) VrotSmem {
  uint8_t a[kOperandBytes];        // values (A)
  uint8_t bhi[kOperandBytes];      // U_m^T high part (B)
  uint8_t blo[kOperandBytes];      // U_m^T low part (B)
  uint8_t codes[kHeadDim][kTile + 4];  // code of (channel, token); rows padded against bank conflicts
  float sigma[kTile];
  uint8_t mods[kTile];
  float thr[15];
  uint64_t mma_bar;
  uint32_t tmem_base;
  int nmods;
  int mod_list[kMods];
};

__device__ __forceinline__ uint32_t swz_offset(int row, int k16) {  // k16: 16-byte chunk index 0..15 along K
  const int katom = k16 >> 3, chunk = k16 & 7;
  return (uint32_t)(katom * (128 * 128) + row * 128 + ((chunk ^ (row & 7)) << 4));
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 B apart (SBO), version 1.
__device__ __forceinline__ uint64_t make_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);        // start address
  d |= (uint64_t)1u << 16;                          // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32;                // stride byte offset
  d |= (uint64_t)1u << 46;                          // descriptor version
  d |= (uint64_t)2u << 61;                          // SWIZZLE_128B
  return d;
}

// kind::f16 instruction descriptor: fp32 accumulator, fp16 A and B, both
// K-major, N = 128, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n"
      "}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_u32(bar))
               : "memory");
}

__global__ void __launch_bounds__(kVThreads, 1) vrot_tc_kernel(const WriteParams p) {
  extern __shared__ uint8_t dyn_smem[];
  VrotSmem& sm = *reinterpret_cast<VrotSmem*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  griddep_launch_dependents();
  griddep_wait();  // kv_quant_pack (just before) writes the records' key parts
  const int b = blockIdx.z, h = blockIdx.y;
  const int H = p.num_kv_heads;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int L0 = p.seq_lens[b];
  const int L1 = L0 + p.n_new;
  if (L0 < 0 || L1 > p.cap_tokens) return;  // reported by kv_quant_pack
  const int wf = (L0 + kWindow - 1) / kWindow;  // first window made only of new tokens
  const int wl = L1 / kWindow;                  // one past the last such window
  const int wt0 = wf + 4 * blockIdx.x;          // first window of this tile
  if (wt0 >= wl) return;
  const int nwin = min(4, wl - wt0);
  const int ntok = nwin * kWindow;
  const size_t seq_head = (size_t)b * H + h;
  const __half* vnew = p.v_new + seq_head * p.n_new * kHeadDim;
  const uint8_t* mnew = p.mod_new + (size_t)b * p.n_new;
  const int LV = 1 << p.value_bits;
  const RecordLayout lay(p.key_bits, p.value_bits);

  // ---- values -> A (rows >= ntok are zero), modality ids, thresholds ----------
  for (int it = 0; it < 16; ++it) {
    const int id = it * kVThreads + tid;
    const int r = id >> 4, k16 = id & 15;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (r < ntok) val = *reinterpret_cast<const uint4*>(vnew + (size_t)(wt0 * kWindow + r - L0) * kHeadDim + 8 * k16);
    *reinterpret_cast<uint4*>(sm.a + swz_offset(r, k16)) = val;
  }
  if (tid < kTile) {
    int m = tid < ntok ? mnew[wt0 * kWindow + tid - L0] : 0;
    sm.mods[tid] = (uint8_t)(m >= kMods ? kMods - 1 : m);
  }
  if (tid < LV - 1) sm.thr[tid] = __fmul_rn(__fadd_rn(p.val_cb[tid], p.val_cb[tid + 1]), 0.5f);
  if (warp == 0) tmem_alloc(&sm.tmem_base, kTmemCols);
  if (tid == 0) {
    mbar_init(&sm.mma_bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    int present = 0;
    for (int r = 0; r < ntok; ++r) present |= 1 << sm.mods[r];
    int n = 0;
    for (int m = 0; m < kMods; ++m)
      if (present & (1 << m)) sm.mod_list[n++] = m;
    sm.nmods = n;
  }

  // ---- sigma of each token from the unrotated fp16 value (pairwise tree:
  // x_c + x_{c+64} first, then halving) -----------------------------------------
  {
    const int r = tid;  // token row
    float y[64];
#pragma unroll
    for (int k16 = 0; k16 < 8; ++k16) {
      const uint4 u0 = *reinterpret_cast<const uint4*>(sm.a + swz_offset(r, k16));      // channels 8 k16 ..
      const uint4 u1 = *reinterpret_cast<const uint4*>(sm.a + swz_offset(r, k16 + 8));  // channels 64 + 8 k16 ..
      const __half2* h0 = reinterpret_cast<const __half2*>(&u0);
      const __half2* h1 = reinterpret_cast<const __half2*>(&u1);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f0 = __half22float2(h0[e]), f1 = __half22float2(h1[e]);
        y[8 * k16 + 2 * e] = __fadd_rn(__fmul_rn(f0.x, f0.x), __fmul_rn(f1.x, f1.x));
        y[8 * k16 + 2 * e + 1] = __fadd_rn(__fmul_rn(f0.y, f0.y), __fmul_rn(f1.y, f1.y));
      }
    }
#pragma unroll
    for (int hh = 32; hh >= 1; hh >>= 1)
#pragma unroll
      for (int c = 0; c < hh; ++c) y[c] = __fadd_rn(y[c], y[c + hh]);
    sm.sigma[r] = __half2float(__float2half_rn(__fsqrt_rn(__fmul_rn(y[0], 0.0078125f))));
  }
  __syncthreads();
  const uint32_t tmem = sm.tmem_base;
  const int nmods = sm.nmods;
  bool timed_out = false;

  for (int mi = 0; mi < nmods; ++mi) {
    const int m = sm.mod_list[mi];
    // ---- U_m^T -> B (high, low), thread = output channel j = B row
    {
      const int j = tid;
      const float* U = p.value_rot + ((size_t)(h * kMods + m) * kHeadDim) * kHeadDim + j;
      for (int k16 = 0; k16 < 16; ++k16) {
        float u[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) u[e] = U[(size_t)(8 * k16 + e) * kHeadDim];
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __half2 hv = __floats2half2_rn(u[2 * e], u[2 * e + 1]);
          const float2 hf = __half22float2(hv);
          const __half2 lv = __floats2half2_rn(u[2 * e] - hf.x, u[2 * e + 1] - hf.y);
          hi[e] = *reinterpret_cast<const uint32_t*>(&hv);
          lo[e] = *reinterpret_cast<const uint32_t*>(&lv);
        }
        *reinterpret_cast<uint4*>(sm.bhi + swz_offset(j, k16)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(sm.blo + swz_offset(j, k16)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
    fence_proxy_async_smem();  // generic-proxy operand writes -> visible to the tensor core
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      const uint32_t a0 = smem_u32(sm.a), bh0 = smem_u32(sm.bhi), bl0 = smem_u32(sm.blo);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t off = (uint32_t)((ks >> 2) * (128 * 128) + (ks & 3) * 32);
        umma_f16(tmem, make_desc_sw128(a0 + off), make_desc_sw128(bh0 + off), kIdesc, ks > 0 ? 1u : 0u);
        umma_f16(tmem, make_desc_sw128(a0 + off), make_desc_sw128(bl0 + off), kIdesc, 1u);
      }
      umma_commit(&sm.mma_bar);
    }
    const bool ok = mbar_wait_bounded(&sm.mma_bar, mi & 1, kMmaWaitNs);
    tc_fence_after();
    if (__syncthreads_or(!ok)) {
      timed_out = true;
      break;
    }
    // ---- epilogue: this thread's token (TMEM lane 32 warp + lane)
    {
      const int r = tid;
      const bool mine = r < ntok && sm.mods[r] == m;
      const float s = sm.sigma[r];
      const uint32_t row_addr = tmem + ((uint32_t)(32 * warp) << 16);
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) {
        uint32_t v[32];
        tmem_ld32(row_addr + 32 * cb, v);  // warp-collective: every lane loads
        if (mine) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            uint32_t code = 0;
            if (s != 0.0f) code = count_above(__fdiv_rn(__uint_as_float(v[i]), s), sm.thr, LV - 1);
            sm.codes[32 * cb + i][r] = (uint8_t)code;
          }
        }
      }
    }
    tc_fence_before();
    __syncthreads();  // the accumulator and B are reused by the next modality
    tc_fence_after();
  }

  if (!timed_out) {
    // ---- channel-major words: warp w packs window w of the tile
    if (warp < nwin) {
      const int w = wt0 + warp;
      uint8_t* rec = p.records + (seq_head * p.cap_windows + w) * lay.bytes;
      uint32_t* vw = reinterpret_cast<uint32_t*>(rec + lay.v_off);
      const int cpw = 32 / p.value_bits;
      const int ngroups = kWindow / cpw;
      for (int e = lane; e < ngroups * kHeadDim; e += 32) {
        const int grp = e / kHeadDim, c = e - grp * kHeadDim;
        const uint8_t* src = &sm.codes[c][32 * warp + grp * cpw];
        uint32_t word = 0;
        for (int i = 0; i < cpw; ++i) word |= (uint32_t)src[i] << (p.value_bits * i);
        vw[grp * kHeadDim + c] = word;
      }
      reinterpret_cast<__half*>(rec + lay.sigma_off)[lane] = __float2half_rn(sm.sigma[32 * warp + lane]);
    }
  } else if (tid == 0) {
    set_error(p.error_word, OMNIKV_DEVERR_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

size_t vrot_tc_smem_bytes() { return sizeof(VrotSmem) + 1024; }

cudaError_t launch_vrot_tc(const WriteParams& p, int batch, cudaStream_t stream) {
  static_assert(sizeof(VrotSmem) + 1024 <= 227 * 1024, "shared memory");
  const int smem = (int)vrot_tc_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(vrot_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int tiles = (p.n_new / kWindow + 1 + 3) / 4;  // full windows <= n_new / 32 (+1 for alignment)
  dim3 grid(tiles, p.num_kv_heads, batch);
  return launch_pdl(vrot_tc_kernel, grid, dim3(kVThreads), (size_t)smem, stream, p);
}

}  // namespace omnikv
