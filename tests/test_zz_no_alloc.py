"""The allocation-free decode entry point (omnikv_decode_static).

It exists for callers that cannot allocate device memory while decoding: an
engine that reserved nearly all device memory for its own pool, a plug-in whose
host framework owns every allocation, a latency-critical loop that cannot pay for
cudaMalloc. It keeps the split partials in the library's fixed device array, so
its results must equal -- bit for bit, at the same split count -- those of
omnikv_decode_attention + omnikv_combine with a caller-allocated partials buffer,
call after call, even though the array still holds the previous call's contents;
and, like them, the oracle's fp64 attention over the same dequantised cache within
the decode tolerance.

This file is collected last so that a stop-at-first-failure run has already run
every other test.
"""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

from bit_kv_cache_pack_b200 import _abi
from bit_kv_cache_pack_b200._abi import OmniKVCache, OmniKVConfig
from oracle import codec
from oracle.attention import decode_dense
from synth.workloads import WORKLOADS, key_drift, prefill_inputs, seq_lengths

from helpers import check_decode, make_layer, seeded_randn, upload_oracle_cache

SCRATCH_BYTES = 8 << 20   # OMNIKV_DECODE_STATIC_SCRATCH_BYTES
PARTIAL_BYTES = 1552      # one split-K partials entry


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


def _oracle_cache(spec, seed, ocfg, params):
    """The oracle's own cache of the workload's prefill (never the GPU's), and its
    capacity in tokens."""
    L = seq_lengths(spec, seed)
    cap = int(-(-int(L.max()) // 32) * 32) + 32
    drift = key_drift(spec, seed, 0, cap // 32, "cpu")
    k, v, mod = prefill_inputs(spec, seed, 0, params, drift, L, "cpu")
    oc = codec.OracleCache(spec.batch, spec.num_kv_heads, cap, spec.key_bits, spec.value_bits)
    codec.write_cache(ocfg, oc, k.numpy(), v.numpy(), mod.numpy())
    return oc


def _allocated(m, consts, cache, q, S):
    B, Hq = q.shape[:2]
    part = m.partials_tensor(B, Hq, S, q.device)
    out = torch.empty(B, Hq, 128, dtype=torch.float32, device=q.device)
    m.omnikv_decode_attention(consts.struct, cache.struct, q, part, S)
    m.omnikv_combine(consts.struct, cache.struct, part, S, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _static(m, consts, cache, q, S):
    B, Hq = q.shape[:2]
    out = torch.full((B, Hq, 128), float("nan"), dtype=torch.float32, device=q.device)
    m.omnikv_decode_static(consts.struct, cache.struct, q, out, S)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.gpu
def test_static_scratch_matches_allocated_partials(cuda_device):
    """Two calls in a row (different queries and split counts; the second runs
    over the first's leftover scratch contents): bit-identical to the allocating
    entry points at the same split count, and within tolerance of the oracle."""
    import bit_kv_cache_pack_b200 as m
    spec, seed = WORKLOADS["tiny"], 21
    params, consts, ocfg = make_layer(spec, seed, 0, cuda_device)
    oc = _oracle_cache(spec, seed, ocfg, params)
    cache = upload_oracle_cache(oc, cuda_device)
    for call, (qseed, S) in enumerate([(1, 7), (2, 0)]):
        q = seeded_randn((1, spec.num_q_heads, 128), cuda_device, qseed).half()
        S_used = S or m.omnikv_default_splits(consts.struct, cache.struct)
        got = _static(m, consts, cache, q, S)
        assert np.array_equal(got, _allocated(m, consts, cache, q, S_used)), "call %d" % (call + 1)
        check_decode(got, decode_dense(ocfg, oc, q.cpu().numpy()), "static scratch, call %d" % (call + 1))
    assert int(cache.error_word.item()) == 0


@pytest.mark.gpu
def test_static_scratch_matches_allocated_partials_4bit(cuda_device):
    """The same with 4-bit codes (the table body, which takes its shared memory
    dynamically): bit-identical to the allocating path, within tolerance of the
    oracle."""
    import bit_kv_cache_pack_b200 as m
    from synth.workloads import with_bits
    spec, seed = with_bits(WORKLOADS["tiny"], 4, 4), 22
    params, consts, ocfg = make_layer(spec, seed, 0, cuda_device)
    oc = _oracle_cache(spec, seed, ocfg, params)
    cache = upload_oracle_cache(oc, cuda_device)
    for call, (qseed, S) in enumerate([(3, 5), (4, 0)]):
        q = seeded_randn((1, spec.num_q_heads, 128), cuda_device, qseed).half()
        S_used = S or m.omnikv_default_splits(consts.struct, cache.struct)
        got = _static(m, consts, cache, q, S)
        assert np.array_equal(got, _allocated(m, consts, cache, q, S_used)), "K4 call %d" % (call + 1)
        check_decode(got, decode_dense(ocfg, oc, q.cpu().numpy()), "static scratch K4, call %d" % (call + 1))
    assert int(cache.error_word.item()) == 0


@pytest.mark.gpu
def test_static_scratch_lowers_the_default_split_count(cuda_device):
    """Batch 64 x 16 query heads: the default split count does not fit the array
    (5405 entries hold 5 splits), so the call lowers it to 5 -- which also moves the
    decode to longer splits -- and must equal the allocating path at 5 splits."""
    import bit_kv_cache_pack_b200 as m
    spec = dataclasses.replace(WORKLOADS["tiny"], batch=64)
    seed = 23
    params, consts, ocfg = make_layer(spec, seed, 0, cuda_device)
    oc = _oracle_cache(spec, seed, ocfg, params)
    cache = upload_oracle_cache(oc, cuda_device)
    fit = SCRATCH_BYTES // (spec.batch * spec.num_q_heads * PARTIAL_BYTES)
    assert fit == 5
    default = m.omnikv_default_splits(consts.struct, cache.struct)
    assert default > fit
    for call in range(2):
        q = seeded_randn((spec.batch, spec.num_q_heads, 128), cuda_device, 40 + call).half()
        got = _static(m, consts, cache, q, 0)
        assert np.array_equal(got, _allocated(m, consts, cache, q, fit)), "call %d" % (call + 1)
        check_decode(got, decode_dense(ocfg, oc, q.cpu().numpy()), "static scratch, batch 64, call %d" % (call + 1))
    assert int(cache.error_word.item()) == 0
