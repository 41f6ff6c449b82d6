// Shared device helpers for the OmniKVQuant kernels (sm_100a).
//
// Arithmetic that decides a stored bit (key rotation, window range, codes,
// value scale) uses explicitly rounded intrinsics (__fadd_rn, __fsub_rn,
// __fmul_rn, __fdiv_rn, __fsqrt_rn) so that the compiler never contracts a
// multiply and an add into an FMA: the result is the IEEE value of each step.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/omnikv.h"

namespace omnikv {

constexpr int kHeadDim = 128;
constexpr int kWindow = 32;
constexpr int kMods = 3;
constexpr int kMaxGroup = 8;  // query heads per kv head handled by one CTA

// fp32(2^-3.5) = fp32(1/sqrt(128)), bit pattern 0x3DB504F3
__device__ __forceinline__ float inv_sqrt_d() { return __int_as_float(0x3DB504F3); }

// Key metadata formats of a window: fp16 (m, s) pairs per channel (512 B), or
// MXFP4 -- E2M1 elements sharing an E8M0 exponent per 32 channels (144 B).
// key metadata formats: fp16 (m, s) per window channel; MXFP4 blocks of them; the
// TurboQuant key codec (one fp16 scale per token, no window statistics)
constexpr int kMetaFp16 = 0, kMetaMx = 1, kMetaTurbo = 2;
constexpr int kMetaFp16Bytes = 512, kMetaMxBytes = 144, kMetaTurboBytes = 64;

__host__ __device__ constexpr int meta_bytes_of(int key_meta) {
  return key_meta == kMetaMx ? kMetaMxBytes : key_meta == kMetaTurbo ? kMetaTurboBytes : kMetaFp16Bytes;
}

struct RecordLayout {
  int k_off, meta_off, v_off, sigma_off, bytes;
  int key_bits, value_bits;
  __host__ __device__ RecordLayout(int kb, int vb, int key_meta = kMetaFp16) : key_bits(kb), value_bits(vb) {
    const int kbytes = kWindow * kHeadDim * kb / 8;
    const int vbytes = kWindow * kHeadDim * vb / 8;
    k_off = 0;
    meta_off = kbytes;
    v_off = meta_off + meta_bytes_of(key_meta);
    sigma_off = v_off + vbytes;
    bytes = sigma_off + kWindow * 2;
  }
};

// ---- MXFP4 key metadata (E2M1 elements, one E8M0 exponent per 32 channels) ----
// The shared exponent of a block: the smallest e in [-127, 127] with
// amax <= 6 * 2^e (no element saturates); -127 for an all-zero block.
__device__ __forceinline__ int mx_block_exp(float amax) {
  if (!(amax > 0.0f)) return -127;
  const int f = ilogbf(amax);  // 2^f <= amax < 2^(f + 1)
  int e = (amax <= ldexpf(1.5f, f)) ? f - 2 : f - 1;  // 6 * 2^(f-2) = 1.5 * 2^f
  return max(-127, min(127, e));
}

// Value of an E2M1 code (sign << 3 | magnitude index; magnitudes 0, 0.5, 1, 1.5,
// 2, 3, 4, 6) times 2^e, exact in fp32 (subnormal results included).
__device__ __forceinline__ float mx_value(uint32_t code, int e) {
  const uint32_t idx = code & 7u;
  float v = 0.0f;
  if (idx != 0u) {
    const int ex = (idx >= 2u ? (int)(idx >> 1) - 1 : -1) + e;  // 2^ex * (1 or 1.5)
    const bool half_up = idx >= 2u && (idx & 1u);
    if (ex > 127)
      v = INFINITY;
    else if (ex >= -126)
      v = __uint_as_float(((uint32_t)(ex + 127) << 23) | (half_up ? (1u << 22) : 0u));
    else
      v = ldexpf(half_up ? 1.5f : 1.0f, ex);
  }
  return (code & 8u) ? -v : v;
}

// Nearest E2M1 grid value g * 2^e to x (|x| <= 6 * 2^e), ties to the even code;
// a zero is coded +0. Returns the value; *code receives the E2M1 code.
__device__ __forceinline__ float mx_round_nearest(float x, int e, uint32_t* code) {
  const float a = fabsf(ldexpf(x, -e));  // exact scaling by a power of two
  // midpoints 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5: a tie goes to the even index
  uint32_t idx = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) + (a >= 3.5f) + (a > 5.0f);
  const uint32_t c = idx | ((idx != 0u && x < 0.0f) ? 8u : 0u);
  *code = c;
  return mx_value(c, e);
}

// One entry of the split-K partials buffer.
struct __align__(16) Partial {
  float acc[kMods][kHeadDim];
  float m;
  float l;
  float pad[2];
};
static_assert(sizeof(Partial) == 1552, "partials entry is 1552 bytes");

constexpr int kMaxSplits = 4096;

// Sign flip, Sylvester-Hadamard butterflies with h = 1, 2, ..., 64, then the
// fp32 scale 2^-3.5, on a 128-vector spread over a warp: lane L holds channels
// 4L + r, r = 0..3, in x[r]. Stages h = 1, 2 stay inside the thread; stage h >= 4
// pairs lane L with lane L ^ (h / 4). The lower index of a pair becomes a + b
// and the upper a - b (a the lower, b the upper), exactly as the scalar order.
__device__ __forceinline__ void warp_hadamard_rotate(float x[4], const float sign[4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int r = 0; r < 4; ++r) x[r] = __fmul_rn(x[r], sign[r]);
  {  // h = 1
    const float a0 = x[0], b0 = x[1], a1 = x[2], b1 = x[3];
    x[0] = __fadd_rn(a0, b0);
    x[1] = __fsub_rn(a0, b0);
    x[2] = __fadd_rn(a1, b1);
    x[3] = __fsub_rn(a1, b1);
  }
  {  // h = 2
    const float a0 = x[0], b0 = x[2], a1 = x[1], b1 = x[3];
    x[0] = __fadd_rn(a0, b0);
    x[2] = __fsub_rn(a0, b0);
    x[1] = __fadd_rn(a1, b1);
    x[3] = __fsub_rn(a1, b1);
  }
#pragma unroll
  for (int hl = 1; hl < 32; hl <<= 1) {  // h = 4 * hl
    const bool upper = (lane & hl) != 0;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float other = __shfl_xor_sync(0xffffffffu, x[r], hl);
      x[r] = upper ? __fsub_rn(other, x[r]) : __fadd_rn(x[r], other);
    }
  }
  const float s = inv_sqrt_d();
#pragma unroll
  for (int r = 0; r < 4; ++r) x[r] = __fmul_rn(x[r], s);
}

// Division-free, exact form of the code decision  fl(fl(a / s) + c) > t  for
// s > 0 (fl: fp32 round to nearest even). y -> fl(y + c) is monotone, so the
// decision is  fl(a / s) >= F  for F the smallest float with fl(F + c) > t; and
// fl(x) >= F  iff  x > mid  or  (x == mid and F has an even significand), mid
// the midpoint of F and its predecessor (the rounding boundary). The sign of
// a - mid * s is exact in one fp64 FMA: mid has at most 25 significant bits,
// s (an fp16 value) 11 and a (fp32) 24, so mid * s is exact and the FMA rounds
// only its exact result. s = +inf gives the decision for a / s = 0.
struct CodeBound {
  double mid;
  int tie_up;  // 1: a / s == mid rounds up to F
};

__device__ inline CodeBound make_code_bound(float t, float c) {
  float y = __fsub_rn(t, c);
  for (int i = 0; i < 64 && __fadd_rn(y, c) > t; ++i) y = nextafterf(y, -INFINITY);
  for (int i = 0; i < 64 && !(__fadd_rn(y, c) > t); ++i) y = nextafterf(y, INFINITY);
  const float prev = nextafterf(y, -INFINITY);
  CodeBound b;
  b.mid = 0.5 * ((double)prev + (double)y);
  b.tie_up = (__float_as_uint(y) & 1u) == 0u;
  return b;
}

// The NB = 2^bits - 1 bounds of one code, in registers.
template <int NB>
struct CodeBounds {
  double mid[NB];
  uint32_t tie_up;  // bit j: a / s == mid[j] rounds up past threshold j
};

template <int NB>
__device__ __forceinline__ CodeBounds<NB> load_bounds(const CodeBound* bd) {
  CodeBounds<NB> r;
  r.tie_up = 0;
#pragma unroll
  for (int j = 0; j < NB; ++j) {
    r.mid[j] = bd[j].mid;
    r.tie_up |= (uint32_t)bd[j].tie_up << j;
  }
  return r;
}

// The decisions for one scale s > 0 as fp32 bounds: decision j  <=>  a > b[j].
// With T = mid_j * s (exact in fp64), a > T or (a == T and ties round up):
// for T not an fp32 value, a > T <=> a > RD(T) (a is fp32); for T an fp32
// value, a >= T <=> a > pred(T). s = +inf maps to +-inf bounds, the decisions
// for a / s = 0.
template <int NB>
struct ScaledBounds {
  float b[NB];
};

template <int NB>
__device__ __forceinline__ ScaledBounds<NB> scale_bounds(const CodeBounds<NB>& cb, float s) {
  ScaledBounds<NB> r;
  const double sd = (double)s;
#pragma unroll
  for (int j = 0; j < NB; ++j) {
    const double T = cb.mid[j] * sd;
    float B = __double2float_rd(T);
    if ((double)B == T && ((cb.tie_up >> j) & 1u)) B = nextafterf(B, -INFINITY);
    r.b[j] = B;
  }
  return r;
}

// #{ j : fl(fl(a / s) + c) > t_j } for the ascending thresholds behind `sb`.
template <int NB>
__device__ __forceinline__ uint32_t code_from_scaled(const ScaledBounds<NB>& sb, float a) {
  uint32_t code = 0;
#pragma unroll
  for (int j = 0; j < NB; ++j) code += (a > sb.b[j]) ? 1u : 0u;
  return code;
}

__device__ __forceinline__ void set_error(int32_t* word, int32_t bits) {
  if (word) atomicOr(word, bits);
}

}  // namespace omnikv
