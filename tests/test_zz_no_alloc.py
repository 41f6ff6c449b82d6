"""The allocation-free decode entry point (omnikv_decode_static).

It exists for callers that cannot allocate device memory while decoding: an
engine that reserved nearly all device memory for its own pool, a plug-in whose
host framework owns every allocation, a latency-critical loop that cannot pay for
cudaMalloc. It keeps the split partials in the library's fixed device array, so
its results must equal those of omnikv_decode_attention + omnikv_combine with a
caller-allocated partials buffer, call after call, even though the array still
holds the previous call's contents.

This file is collected last so that a stop-at-first-failure run has already run
every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_kv_cache_pack_b200 import _abi
from bit_kv_cache_pack_b200._abi import OmniKVCache, OmniKVConfig
from synth.workloads import WORKLOADS, key_drift, prefill_inputs, seq_lengths

from helpers import check_decode, make_layer, seeded_randn


def test_static_scratch_rejects_what_does_not_fit():
    """Host-side size check (no GPU work): batch * heads * splits partials of
    1552 B must fit in the 8 MiB array."""
    fake = 0x10000
    cfg = OmniKVConfig(128, 16, 2, 32, 2, 2, fake, fake, fake, fake)
    lib = _abi.load()
    big = OmniKVCache(fake, fake, fake, fake, 0, 400, 2048, 2048, 0)     # 400 * 16 = 6400 entries > 5405
    assert lib.omnikv_decode_static(ctypes.byref(cfg), ctypes.byref(big), fake, fake, 1, 0) == \
        _abi.OMNIKV_ERR_CAPACITY
    small = OmniKVCache(fake, fake, fake, fake, 0, 1, 2048, 2048, 0)     # 16 entries per split
    assert lib.omnikv_decode_static(ctypes.byref(cfg), ctypes.byref(small), fake, fake, 400, 0) == \
        _abi.OMNIKV_ERR_CAPACITY                                      # 6400 entries again
    assert lib.omnikv_decode_static(ctypes.byref(cfg), ctypes.byref(small), None, fake, 1, 0) == \
        _abi.OMNIKV_ERR_INVALID_ARG


@pytest.mark.gpu
def test_static_scratch_matches_allocated_partials(cuda_device):
    import bit_kv_cache_pack_b200 as m
    spec, seed = WORKLOADS["tiny"], 21
    params, consts, _ = make_layer(spec, seed, 0, cuda_device)
    L = seq_lengths(spec, seed)
    drift = key_drift(spec, seed, 0, 65, cuda_device)
    k, v, mod = prefill_inputs(spec, seed, 0, params, drift, L, cuda_device)
    cache = m.KVCache(1, spec.num_kv_heads, 2080, 2, 2, cuda_device)
    m.omnikv_write_cache(consts.struct, cache.struct, k, v, mod, int(L[0]))

    def with_allocated_partials(q, S):
        S = S or m.omnikv_default_splits(consts.struct, cache.struct)
        part = m.partials_tensor(1, spec.num_q_heads, S, cuda_device)
        out = torch.empty(1, spec.num_q_heads, 128, dtype=torch.float32, device=cuda_device)
        m.omnikv_decode_attention(consts.struct, cache.struct, q, part, S)
        m.omnikv_combine(consts.struct, cache.struct, part, S, out)
        torch.cuda.synchronize()
        return out.cpu().numpy().astype(np.float64)

    # two calls in a row, different queries and split counts: the second call
    # runs over the first call's leftover scratch contents
    for call, (qseed, S) in enumerate([(1, 7), (2, 0)]):
        q = seeded_randn((1, spec.num_q_heads, 128), cuda_device, qseed).half()
        ref = with_allocated_partials(q, S)
        out = torch.full((1, spec.num_q_heads, 128), float("nan"), dtype=torch.float32, device=cuda_device)
        m.omnikv_decode_static(consts.struct, cache.struct, q, out, S)
        torch.cuda.synchronize()
        check_decode(out.cpu().numpy(), ref, "static scratch, call %d" % (call + 1))
    assert int(cache.error_word.item()) == 0
