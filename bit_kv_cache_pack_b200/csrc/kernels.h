// Launch parameters and launchers of the OmniKVQuant kernels (internal).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace omnikv {

struct Partial;

struct WriteParams {
  const float* key_cb;
  const float* val_cb;
  const float* key_signs;
  const float* value_rot;
  int key_bits, value_bits, num_kv_heads;
  int key_meta;  // kMetaFp16, kMetaMx or kMetaTurbo
  uint8_t* records;
  __half* key_tail;
  uint8_t* modality;
  int32_t* seq_lens;
  int32_t* error_word;
  int cap_tokens, cap_windows;
  const __half* k_new;
  const __half* v_new;
  const uint8_t* mod_new;
  int n_new;
  int tc_values;  // 1: values of windows filled completely by this write are done by vrot_tc
  int32_t* step_flags;  // decode step only: [batch][kv heads], set to the new length once written
  float* vrot_dump;     // optional: [batch][kv heads][n_new][128] fp32 rotated values v' of the written tokens
};

constexpr uint64_t kFlagWaitNs = 2000000000ull;  // default limit of a decode step's flag wait (2 s)

struct DecodeParams {
  const float* key_cb;
  const float* val_cb;
  const float* key_signs;
  const float* value_rot;  // only prefetched into L2 (for the combine)
  int key_bits, value_bits, num_kv_heads, group;
  int key_meta;  // kMetaFp16, kMetaMx or kMetaTurbo
  const uint8_t* records;
  const uint8_t* modality;
  const int32_t* seq_lens;
  int cap_tokens, cap_windows;
  const __half* q;
  Partial* partials;
  int num_splits;
  int split_windows;  // windows per split (C)
  int32_t* error_word;
  int batch;
  // decode step only: the length seen is seq_lens[b] + len_add, and the window
  // holding the appended position is read once step_flags[b][h] == that length
  int len_add;
  const int32_t* step_flags;
  uint64_t flag_wait_ns;  // how long a copy waits for its step flag before giving up (OMNIKV_DEVERR_TIMEOUT)
  // decode step only: the append CTAs in front of the decode CTAs; append CTA a
  // appends for (sequence, kv head) units a, a + append_ctas, ... in turn
  int append_ctas;
  // streaming policy: the decode covers only the packed body, the windows before
  // 32 floor(max(0, T - 128) / 32) (the tail is stream_tail_kernel's)
  int stream;
};

struct CombineParams {
  const float* value_rot;
  int num_kv_heads, group;
  const Partial* partials;
  int num_splits;
  float* out;
  // decode step only: seq_lens[b] += len_add (when within cap_tokens) after the merge
  int32_t* seq_lens;
  int len_add, cap_tokens;
};

// Dense bf16 decode (comparison baseline).
constexpr int kDensePartialFloats = 132;  // acc[128], m, l, 2 pad
struct DenseParams {
  const __nv_bfloat16* k;  // [B][H_kv][cap][128]
  const __nv_bfloat16* v;
  const int32_t* seq_lens;
  const __nv_bfloat16* q;  // [B][H_q][128]
  float* partials;         // [B][H_q][S][132]
  float* out;              // [B][H_q][128]
  int32_t* error_word;
  int num_kv_heads, group, cap_tokens, num_splits, split_chunks;
};
cudaError_t launch_dense(const DenseParams& p, int batch, cudaStream_t stream);

// Launch with programmatic stream serialisation: the kernel may start while
// the previous kernel of the stream is still running; it calls griddep_wait()
// before touching anything that kernel may write, and griddep_launch_dependents()
// to let its own successor start early.
template <typename Kernel, typename... Args>
cudaError_t launch_pdl(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, const Args&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

cudaError_t launch_write(const WriteParams& p, int batch, cudaStream_t stream);
cudaError_t launch_vrot_tc(const WriteParams& p, int batch, cudaStream_t stream);
cudaError_t launch_decode(const DecodeParams& p, int batch, cudaStream_t stream);
// The decode launch of a decode step: batch * kv heads append CTAs (one token per
// sequence, described by w) followed by the decode CTAs of p.
cudaError_t launch_decode_step(const DecodeParams& p, const WriteParams& w, cudaStream_t stream);

// Decode kernel bodies. 2-bit caches: the per-warp body (each warp streams its own
// run of windows; registers for 2 CTAs per SM) for long splits, the cooperative
// body (the CTA takes 4 windows at a time; 3 CTAs per SM) for splits of at most
// kCoopMaxWindows windows; 4-bit keys and values (every key format): the per-warp
// tensor-core body over codeword tables; other bit mixes: the CUDA-core build.
enum DecodeBody { kBodyWarp = 0, kBodyCoop = 1, kBodyGeneric = 2, kBodyLut = 3, kNumBodies = 4 };
constexpr int kCoopMaxWindows = 16;
int decode_body(int key_bits, int value_bits, int key_meta, int split_windows);
int decode_ctas_per_sm(int body);  // resident decode CTAs per SM of a body on the current device
cudaError_t launch_combine(const CombineParams& p, int batch, cudaStream_t stream);
cudaError_t launch_stream_push(const __half* k_new, const __half* v_new, const int32_t* seq_lens, __half* ring_k,
                               __half* ring_v, int batch, int num_kv_heads, int n_new, cudaStream_t stream);
constexpr int kStreamTailSplits = 4;  // splits the streaming decode's tail adds after the body's
cudaError_t launch_stream_tail(const DecodeParams& p, const __half* ring_k, const __half* ring_v, int tail_split,
                               cudaStream_t stream);
size_t calibrate_workspace_bytes(int num_tokens);  // 0 for num_tokens < 1
cudaError_t launch_calibrate(const __half* values, const uint8_t* modality, const float* weights, int num_tokens,
                             void* workspace, float* bases, double* eigenvalues, cudaStream_t stream);

}  // namespace omnikv
