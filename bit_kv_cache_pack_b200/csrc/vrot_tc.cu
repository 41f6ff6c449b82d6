// vrot_tc: the per-modality value rotation of the cache write on 5th-generation
// tensor cores (tcgen05 / TMEM), for every 32-token window that a write fills
// completely (paperpeel.com section 2.3 "Modality-aware value rotation": each
// value is rotated by the basis U_m of its modality m before quantisation).
//
// A persistent kernel: one CTA (4 warps) per SM walks a contiguous run of tiles
// of 128 tokens (4 whole windows) of one or a few (sequence, kv head) pairs:
//   * A = the tile's fp16 values, [128 tokens x 128 channels], exact, in a
//     double buffer: the next tile's loads are issued before this tile's tensor
//     work and stored into the other buffer after it;
//     B = U_m^T split into fp16 high and low parts (U = hi + lo to ~22 bits);
//     both in shared memory in the K-major 128-byte-swizzled layout, written with
//     16-byte stores whose chunk index is XOR-ed with the row (conflict free);
//     two converted bases stay resident (slots tagged with modality and kv head,
//     least recently used replaced), so a stream that alternates two modalities
//     (audio and video blocks) converts each basis once; a missing basis is read
//     from global memory (coalesced over the output channel) and converted;
//   * one elected thread issues tcgen05.mma kind::f16 (M = N = 128, K = 16,
//     8 k-steps x {hi, lo}) into a 128-column fp32 accumulator in TMEM and
//     commits to an mbarrier (bounded wait);
//   * one pass per modality present in the tile (the one already in B first):
//     warp w reads TMEM lanes 32w .. 32w+31 (= window w of the tile, one token
//     per thread) with tcgen05.ld, and the tokens of that modality compute their
//     codes code = #{j : v'_c / sigma16 > t_j} (exact, division-free; sigma from
//     the unrotated fp16 value, pairwise tree in fp32, as in the per-token path);
//   * codes are transposed through shared memory into the channel-major value
//     words (16 tokens of one channel per u32) and written with sigma.
// The key half of these windows, partial windows and short appends are handled
// by kv_quant_pack.
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace omnikv {

namespace {

constexpr int kTile = 128;                 // tokens per tile = MMA M
constexpr int kVThreads = 512;             // 16 warps: 4 per TMEM lane quarter
constexpr uint32_t kTmemCols = 128;        // one fp32 accumulator of N = 128 columns
constexpr uint64_t kMmaWaitNs = 2000000000ull;

// operand: [2 k-atoms][128 rows][128 B], 16-byte chunks XOR-swizzled by row % 8
constexpr int kOperandBytes = 2 * 128 * 128;   // 32 KB of fp16

constexpr int kSlots = 2;  // converted bases resident in shared memory

struct __align__(1024) VrotSmem {
  uint8_t a[2][kOperandBytes];          // values (A), double buffer
  uint8_t b[kSlots][2][kOperandBytes];  // U_m^T per slot: high, low part (B)
  uint8_t codes[kHeadDim][kTile + 4];   // code of (channel, token); rows padded against bank conflicts
  float sigma[kTile];
  uint8_t mods[kTile];
  CodeBound bv[15];                     // value code decision bounds
  uint64_t mma_bar;
  uint32_t tmem_base;
  int present;                          // modality bits of the current tile
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

// One tile of 128 tokens of (sequence b, kv head h): windows [wt0, wt0 + nwin).
struct TileItem {
  int b, h, L0, wt0, nwin;
  bool valid;
};

// (lb, lL0): the last sequence whose length was read and that length (the
// lengths do not change during the launch), so that consecutive tiles of one
// sequence wait on no global load.
__device__ __forceinline__ TileItem tile_item(const WriteParams& p, int i, int tiles_per_seq, int& lb, int& lL0) {
  TileItem t;
  const int H = p.num_kv_heads;
  const int bh = i / tiles_per_seq, tile = i - bh * tiles_per_seq;
  t.b = bh / H;
  t.h = bh - t.b * H;
  if (t.b != lb) {
    lL0 = p.seq_lens[t.b];
    lb = t.b;
  }
  t.L0 = lL0;
  t.wt0 = 0;
  t.nwin = 0;
  t.valid = false;
  const int L1 = t.L0 + p.n_new;
  if (t.L0 < 0 || L1 > p.cap_tokens) return t;  // reported by kv_quant_pack
  const int wf = (t.L0 + kWindow - 1) / kWindow;  // first window made only of new tokens
  const int wl = L1 / kWindow;                    // one past the last such window
  t.wt0 = wf + 4 * tile;
  if (t.wt0 >= wl) return t;
  t.nwin = min(4, wl - t.wt0);
  t.valid = true;
  return t;
}

constexpr int kChunks = kTile * 16 / kVThreads;  // 16-byte chunks of A per thread

// This thread's chunks of the tile's values (rows >= the tile's tokens are zero)
// and, for threads < 128, the modality id of token row `tid`.
__device__ __forceinline__ void load_tile(const WriteParams& p, const TileItem& t, int tid, uint4 (&v)[kChunks],
                                          int& mod) {
  const int ntok = t.nwin * kWindow;
  const __half* vnew = p.v_new + ((size_t)t.b * p.num_kv_heads + t.h) * p.n_new * kHeadDim;
#pragma unroll
  for (int it = 0; it < kChunks; ++it) {
    const int id = it * kVThreads + tid;
    const int r = id >> 4, k16 = id & 15;
    v[it] = make_uint4(0u, 0u, 0u, 0u);
    if (t.valid && r < ntok)
      v[it] = *reinterpret_cast<const uint4*>(vnew + (size_t)(t.wt0 * kWindow + r - t.L0) * kHeadDim + 8 * k16);
  }
  mod = -1;
  if (t.valid && tid < ntok) {
    const int m = p.mod_new[(size_t)t.b * p.n_new + t.wt0 * kWindow + tid - t.L0];
    mod = m >= kMods ? kMods - 1 : m;
  }
}

__device__ __forceinline__ void store_tile(uint8_t* a, int tid, const uint4 (&v)[kChunks]) {
#pragma unroll
  for (int it = 0; it < kChunks; ++it) {
    const int id = it * kVThreads + tid;
    *reinterpret_cast<uint4*>(a + swz_offset(id >> 4, id & 15)) = v[it];
  }
}

// OR of the modality bits of the CTA's threads into *dst (warp reduction, one
// shared atomic per warp).
__device__ __forceinline__ void gather_present(int* dst, int mod) {
  const unsigned bits = __reduce_or_sync(0xffffffffu, mod >= 0 ? (1u << mod) : 0u);
  if ((threadIdx.x & 31) == 0 && bits) atomicOr(dst, (int)bits);
}

// U^T (U: one basis, fp32 row-major, global memory) -> slot `slot` of B as fp16
// high and low parts: thread = output channel j = B row, 16-byte chunks 4 q ..
// 4 q + 3 along K; the 32 loads of a thread are in flight together.
__device__ __forceinline__ void convert_basis(VrotSmem& sm, int slot, const float* U, int tid) {
  const int j = tid & (kHeadDim - 1), q = tid >> 7;
  float u[4][8];
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
#pragma unroll
    for (int e = 0; e < 8; ++e) u[kk][e] = U[(size_t)(8 * (4 * q + kk) + e) * kHeadDim + j];
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const int k16 = 4 * q + kk;
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __half2 hv = __floats2half2_rn(u[kk][2 * e], u[kk][2 * e + 1]);
      const float2 hf = __half22float2(hv);
      const __half2 lv = __floats2half2_rn(u[kk][2 * e] - hf.x, u[kk][2 * e + 1] - hf.y);
      hi[e] = *reinterpret_cast<const uint32_t*>(&hv);
      lo[e] = *reinterpret_cast<const uint32_t*>(&lv);
    }
    *reinterpret_cast<uint4*>(sm.b[slot][0] + swz_offset(j, k16)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(sm.b[slot][1] + swz_offset(j, k16)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

// Epilogue of one modality pass: warp w reads TMEM lanes 32 (w % 4) .. + 31
// (token rows) and columns 32 (w / 4) .. + 31 (channels); each lane computes its
// token's codes code = #{j : v' / sigma > t_j} (0 where sigma == 0) for the
// tokens of modality m.
template <int BITS>
__device__ __forceinline__ void epilogue_codes(VrotSmem& sm, uint32_t tmem, int warp, int lane, int ntok, int m,
                                               float* dump) {
  const CodeBounds<(1 << BITS) - 1> bv = load_bounds<(1 << BITS) - 1>(sm.bv);
  const int r = 32 * (warp & 3) + lane, cb = warp >> 2;
  const bool mine = r < ntok && sm.mods[r] == m;
  const float sg = sm.sigma[r];
  const ScaledBounds<(1 << BITS) - 1> sb = scale_bounds(bv, sg);
  uint32_t v[32];
  tmem_ld32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + 32 * cb, v);  // warp-collective
  if (mine) {
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const uint32_t code = code_from_scaled(sb, __uint_as_float(v[c]));
      sm.codes[32 * cb + c][r] = (uint8_t)(sg != 0.0f ? code : 0u);
    }
    if (dump) {  // test hook: this token's v' for channels 32 cb .. 32 cb + 31
      float4* d = reinterpret_cast<float4*>(dump + 32 * cb);
#pragma unroll
      for (int c4 = 0; c4 < 8; ++c4)
        d[c4] = make_float4(__uint_as_float(v[4 * c4]), __uint_as_float(v[4 * c4 + 1]), __uint_as_float(v[4 * c4 + 2]),
                            __uint_as_float(v[4 * c4 + 3]));
    }
  }
}

__global__ void __launch_bounds__(kVThreads, 1) vrot_tc_kernel(const WriteParams p, int tiles_per_seq, int batch) {
  extern __shared__ __align__(16) uint8_t dyn_smem[];
  // 1024-byte aligned (the swizzled operands), by an offset on the shared array
  // itself so that accesses stay shared-memory instructions
  VrotSmem& sm = *reinterpret_cast<VrotSmem*>(dyn_smem + ((1024u - (smem_u32(dyn_smem) & 1023u)) & 1023u));
  griddep_launch_dependents();
  griddep_wait();  // kv_quant_pack (just before) writes the records' key parts
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_items = p.num_kv_heads * tiles_per_seq * batch;
  const int per = (n_items + gridDim.x - 1) / gridDim.x;
  const int i0 = blockIdx.x * per, i1 = min(i0 + per, n_items);
  if (i0 >= i1) return;
  const int LV = 1 << p.value_bits;
  const RecordLayout lay(p.key_bits, p.value_bits, p.key_meta);

  if (tid < LV - 1) sm.bv[tid] = make_code_bound(__fmul_rn(__fadd_rn(p.val_cb[tid], p.val_cb[tid + 1]), 0.5f), 0.0f);
  if (warp == 0) tmem_alloc(&sm.tmem_base, kTmemCols);
  if (tid == 0) {
    mbar_init(&sm.mma_bar, 1);
    fence_barrier_init();
    sm.present = 0;
  }
  // the first tile's values
  int i = i0;
  int last_b = -1, last_L0 = 0;
  TileItem cur = tile_item(p, i, tiles_per_seq, last_b, last_L0);
  uint4 regs[kChunks];
  int mod_tok;
  load_tile(p, cur, tid, regs, mod_tok);
  store_tile(sm.a[0], tid, regs);
  fence_proxy_async_smem();
  __syncthreads();
  gather_present(&sm.present, mod_tok);
  if (tid < kTile) sm.mods[tid] = (uint8_t)(mod_tok < 0 ? 0 : mod_tok);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  int buf = 0;
  int slot_m[kSlots], slot_h[kSlots], slot_use[kSlots];  // basis held by each slot (every thread: the same)
#pragma unroll
  for (int sl = 0; sl < kSlots; ++sl) {
    slot_m[sl] = -1;
    slot_h[sl] = -1;
    slot_use[sl] = -1;
  }
  int npass = 0;  // modality passes so far (slot recency)
  uint32_t mma_phase = 0;
  bool timed_out = false;

  while (true) {
    // ---- the next tile's loads are issued now and land during this tile's work
    int inext = i + 1;
    TileItem nxt = tile_item(p, inext < i1 ? inext : i, tiles_per_seq, last_b, last_L0);
    if (inext >= i1) nxt.valid = false;
    int mod_next;
    load_tile(p, nxt, tid, regs, mod_next);

    if (cur.valid) {
      const int ntok = cur.nwin * kWindow;
      // ---- sigma of each token from the unrotated fp16 value (pairwise tree:
      // x_c + x_{c+64} first, then halving): 4 threads per token, thread k of a
      // token holding the partial sums y_c with c % 4 == k through the h = 4
      // level, the last two levels across the 4 threads (same order)
      {
        const int r = tid >> 2, k = tid & 3;
        float y[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c = 4 * i + k;  // c and c + 64
          const __half* row0 = reinterpret_cast<const __half*>(sm.a[buf] + swz_offset(r, c >> 3)) + (c & 7);
          const __half* row1 = reinterpret_cast<const __half*>(sm.a[buf] + swz_offset(r, (c + 64) >> 3)) + (c & 7);
          const float f0 = __half2float(*row0), f1 = __half2float(*row1);
          y[i] = __fadd_rn(__fmul_rn(f0, f0), __fmul_rn(f1, f1));
        }
#pragma unroll
        for (int hh = 8; hh >= 1; hh >>= 1)  // h = 32, 16, 8, 4 (index step hh = h / 4)
#pragma unroll
          for (int i = 0; i < hh; ++i) y[i] = __fadd_rn(y[i], y[i + hh]);
        float z = y[0];  // y_k after the h = 4 level
        const float z2 = __shfl_down_sync(0xffffffffu, z, 2);  // h = 2: y_k += y_{k+2}
        if (k < 2) z = __fadd_rn(z, z2);
        const float z1 = __shfl_down_sync(0xffffffffu, z, 1);  // h = 1: y_0 += y_1
        if (k == 0) sm.sigma[r] = __half2float(__float2half_rn(__fsqrt_rn(__fmul_rn(__fadd_rn(z, z1), 0.0078125f))));
      }
      __syncthreads();
      const int present = sm.present;

      // ---- one pass per modality present, those whose basis is resident first
      int todo = present;
      while (todo) {
        int m = -1, slot = -1;
#pragma unroll
        for (int sl = 0; sl < kSlots; ++sl)
          if (m < 0 && slot_h[sl] == cur.h && slot_m[sl] >= 0 && ((todo >> slot_m[sl]) & 1)) {
            m = slot_m[sl];
            slot = sl;
          }
        if (m < 0) {  // convert the basis into the least recently used slot
          m = __ffs(todo) - 1;
          slot = slot_use[0] <= slot_use[1] ? 0 : 1;
          convert_basis(sm, slot, p.value_rot + ((size_t)cur.h * kMods + m) * kHeadDim * kHeadDim, tid);
          slot_m[slot] = m;
          slot_h[slot] = cur.h;
          fence_proxy_async_smem();  // generic-proxy operand writes -> visible to the tensor core
          __syncthreads();
        }
        slot_use[slot] = npass++;
        tc_fence_after();
        if (tid == 0) {
          const uint32_t a0 = smem_u32(sm.a[buf]), bh0 = smem_u32(sm.b[slot][0]), bl0 = smem_u32(sm.b[slot][1]);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t off = (uint32_t)((ks >> 2) * (128 * 128) + (ks & 3) * 32);
            umma_f16(tmem, make_desc_sw128(a0 + off), make_desc_sw128(bh0 + off), kIdesc, ks > 0 ? 1u : 0u);
            umma_f16(tmem, make_desc_sw128(a0 + off), make_desc_sw128(bl0 + off), kIdesc, 1u);
          }
          umma_commit(&sm.mma_bar);
        }
        const bool ok = mbar_wait_bounded(&sm.mma_bar, mma_phase, kMmaWaitNs);
        mma_phase ^= 1u;
        tc_fence_after();
        if (__syncthreads_or(!ok)) {
          timed_out = true;
          break;
        }
        // ---- epilogue: this thread's token (TMEM lane 32 warp + lane)
        float* dump = nullptr;  // test hook: where this thread's token's v' goes
        if (p.vrot_dump) {
          const int tok = cur.wt0 * kWindow + 32 * (warp & 3) + lane - cur.L0;
          dump = p.vrot_dump + (((size_t)cur.b * p.num_kv_heads + cur.h) * p.n_new + tok) * kHeadDim;
        }
        if (p.value_bits == 2)
          epilogue_codes<2>(sm, tmem, warp, lane, ntok, m, dump);
        else
          epilogue_codes<4>(sm, tmem, warp, lane, ntok, m, dump);
        tc_fence_before();
        __syncthreads();  // the accumulator is reused by the next pass (and B may be replaced)
        todo &= ~(1 << m);
      }
      if (timed_out) break;

      // ---- channel-major words: warps 4 w .. 4 w + 3 pack window w of the tile
      {
        const int w = warp >> 2, part = warp & 3;
        if (w < cur.nwin) {
          const size_t seq_head = (size_t)cur.b * p.num_kv_heads + cur.h;
          uint8_t* rec = p.records + (seq_head * p.cap_windows + cur.wt0 + w) * lay.bytes;
          uint32_t* vw = reinterpret_cast<uint32_t*>(rec + lay.v_off);
          const int cpw = 32 / p.value_bits;
          const int ngroups = kWindow / cpw;
          for (int e = 32 * part + lane; e < ngroups * kHeadDim; e += 128) {
            const int grp = e / kHeadDim, c = e - grp * kHeadDim;
            const uint8_t* src = &sm.codes[c][32 * w + grp * cpw];
            uint32_t word = 0;
            for (int k = 0; k < cpw; ++k) word |= (uint32_t)src[k] << (p.value_bits * k);
            vw[grp * kHeadDim + c] = word;
          }
          if (part == 0) reinterpret_cast<__half*>(rec + lay.sigma_off)[lane] = __float2half_rn(sm.sigma[32 * w + lane]);
        }
      }
    }
    if (inext >= i1) break;  // (an invalid item -- past a sequence's windows -- is skipped, not an end)
    // ---- the next tile: values into the other buffer (its last MMA has completed)
    buf ^= 1;
    store_tile(sm.a[buf], tid, regs);
    fence_proxy_async_smem();
    if (tid == 0) sm.present = 0;
    __syncthreads();  // packing reads of codes / mods are done before they are rewritten
    gather_present(&sm.present, mod_next);
    if (tid < kTile) sm.mods[tid] = (uint8_t)(mod_next < 0 ? 0 : mod_next);
    __syncthreads();
    cur = nxt;
    i = inext;
  }

  if (timed_out && tid == 0) set_error(p.error_word, OMNIKV_DEVERR_TIMEOUT);
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
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int tiles_per_seq = (p.n_new / kWindow + 1 + 3) / 4;  // full windows <= n_new / 32 (+1 for alignment)
  const int n_items = tiles_per_seq * p.num_kv_heads * batch;
  const int ctas = min(n_items, max(1, sms));  // persistent: one CTA per SM
  return launch_pdl(vrot_tc_kernel, dim3(ctas), dim3(kVThreads), (size_t)smem, stream, p, tiles_per_seq, batch);
}

}  // namespace omnikv
