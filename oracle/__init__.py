"""CPU oracle for the OmniKVQuant 2-bit KV-cache write and decode attention.

TEST INFRASTRUCTURE ONLY. This package is the plain, slow, obviously correct
reference that the CUDA path is checked against. Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it; the product path (``bit_kv_cache_pack_b200``) never does, and shares no code
with it.

Sources: "OmniKVQuant: KV Cache Quantization for Omni-LLMs" (arXiv:2609.11582),
as extracted on paperpeel.com (sections 1, 2.2, 2.3, 3.1, 3.3) and summarised on
pchao.org ("方法概览", "关联工作"). The pages print no formula; where they are
silent the oracle takes the plainest reading and each function says which.

Modules:
  codebook  -- Lloyd-Max scalar quantiser for N(0,1) (the fixed codebook)
  codec     -- key rotation, window range, codes, packing, value rotation, the
               cache-write state machine (fp32, op-for-op)
  attention -- dequantisation and decode attention in fp64, two ways (dense in
               the original basis; fused rotated-space split-K per modality)
  mxmeta    -- MXFP4 key metadata (the pages' default format): E2M1 minima and
               scales with shared E8M0 exponents, codes and byte layout
  codec_error -- key reconstruction MSE, attention KL and output MSE of the
               codecs (fp16 / MXFP4 metadata, TurboQuant) on synthetic inputs
  calibration -- per-modality value bases from attention-weighted covariances
               (eigenbasis composed with the Hadamard rotation)

Parity status: every function is pinned by ``tests/test_oracle_*.py`` against
closed forms, textbook values, brute force or invariants, except the claims the
pages make about model accuracy, which need models and datasets that are not
here (parity unpinned, and not part of the path).
"""
