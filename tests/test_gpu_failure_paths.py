"""Error paths of the decode on a GPU, without faulting or hanging it.

* A decode step's flag that never arrives: the copy of the window receiving the
  appended token waits (bounded), gives up after the limit, copies no stale
  record and writes its split empty; the error word reports
  OMNIKV_DEVERR_TIMEOUT and the combined output stays finite. Run for each decode
  body: the cooperative body (short splits), the per-warp body (long splits), the
  4-bit table body and the CUDA-core build (mixed bit widths).
* Operand range: queries far larger than the fp16 score operand could hold
  unscaled decode within the tolerance (the operand carries a power of two);
  2-bit value scales beyond the fp16 range of the value operand (sigma >= 565)
  are reported as OMNIKV_DEVERR_RANGE with a finite output; the 4-bit table body
  takes them.
"""
import time

import numpy as np
import pytest
import torch

from oracle import codec
from oracle.attention import decode_dense
from synth.workloads import WORKLOADS, key_drift, prefill_inputs, with_bits

from helpers import check_decode, make_layer, seeded_randn, upload_oracle_cache

pytestmark = pytest.mark.gpu

TIMEOUT_BIT = 0x4
RANGE_BIT = 0x10


def _oracle_cache(spec, seed, ocfg, params, L, cap, value_scale=1.0):
    drift = key_drift(spec, seed, 0, cap // 32, "cpu")
    k, v, mod = prefill_inputs(spec, seed, 0, params, drift, L, "cpu")
    if value_scale != 1.0:
        v = (v.float() * value_scale).half()
    oc = codec.OracleCache(len(L), spec.num_kv_heads, cap, spec.key_bits, spec.value_bits)
    codec.write_cache(ocfg, oc, k.numpy(), v.numpy(), mod.numpy())
    return oc


@pytest.mark.parametrize("kb,vb,splits,body", [(2, 2, 8, "cooperative"), (2, 2, 1, "per-warp"),
                                               (4, 4, 2, "4-bit tables"), (2, 4, 2, "CUDA-core")])
def test_step_flag_that_never_arrives(cuda_device, kb, vb, splits, body):
    import bit_kv_cache_pack_b200 as m
    spec = with_bits(WORKLOADS["tiny"], kb, vb)
    seed = 41
    params, consts, ocfg = make_layer(spec, seed, 0, cuda_device)
    L = np.array([1000], np.int32)                     # the appended token lands in window 31 (partial)
    oc = _oracle_cache(spec, seed, ocfg, params, L, 1024)
    cache = upload_oracle_cache(oc, cuda_device)       # step flags zero: never set by anyone
    q = seeded_randn((1, spec.num_q_heads, 128), cuda_device, 5).half()
    part = m.partials_tensor(1, spec.num_q_heads, splits, cuda_device)
    out = torch.full((1, spec.num_q_heads, 128), float("nan"), device=cuda_device)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    m.omnikv_test_decode_pending(consts.struct, cache.struct, q, part, splits, 1_000_000)  # 1 ms
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert elapsed < 1.0, "the wait ran past its limit (%.3f s)" % elapsed
    assert int(cache.error_word.item()) & TIMEOUT_BIT, body
    # the combine reads the cache as the step would (one more token)
    cache.struct.max_seq_len = int(L[0]) + 1
    m.omnikv_combine(consts.struct, cache.struct, part, splits, out)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all(), body
    assert int(cache.seq_lens[0].item()) == int(L[0])  # the cache is unchanged


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("splits", [0, 1])
def test_large_queries_decode_within_tolerance(cuda_device, splits, bits):
    """Queries x 4096: the largest score-operand entry would be ~10x the fp16
    maximum without the operand's power of two. 2-bit: default splits run the
    cooperative body, one split the per-warp body; 4-bit: the table body."""
    import bit_kv_cache_pack_b200 as m
    spec, seed = with_bits(WORKLOADS["tiny"], bits, bits), 43
    params, consts, ocfg = make_layer(spec, seed, 0, cuda_device)
    L = np.array([2048], np.int32)
    oc = _oracle_cache(spec, seed, ocfg, params, L, 2080)
    cache = upload_oracle_cache(oc, cuda_device)
    q = (seeded_randn((1, spec.num_q_heads, 128), cuda_device, 7) * 4096.0).half()
    assert torch.isfinite(q).all()
    S = splits or m.omnikv_default_splits(consts.struct, cache.struct)
    part = m.partials_tensor(1, spec.num_q_heads, S, cuda_device)
    out = torch.empty(1, spec.num_q_heads, 128, device=cuda_device)
    m.omnikv_decode_attention(consts.struct, cache.struct, q, part, S)
    m.omnikv_combine(consts.struct, cache.struct, part, S, out)
    torch.cuda.synchronize()
    assert int(cache.error_word.item()) == 0
    check_decode(out.cpu().numpy(), decode_dense(ocfg, oc, q.cpu().numpy()), "queries x 4096, K%d S=%d" % (bits, S))


@pytest.mark.parametrize("splits", [0, 1])
def test_value_scales_out_of_range_are_reported(cuda_device, splits):
    """Values x 1024 (sigma of several thousand): the 2-bit value operand cannot
    hold them; the split is written empty, RANGE is set, the output is finite."""
    import bit_kv_cache_pack_b200 as m
    spec, seed = WORKLOADS["tiny"], 47
    params, consts, ocfg = make_layer(spec, seed, 0, cuda_device)
    L = np.array([2048], np.int32)
    oc = _oracle_cache(spec, seed, ocfg, params, L, 2080, value_scale=1024.0)
    sig = oc.records[0, :, :, oc.off["sigma"]:].copy().view(np.float16).astype(np.float32)
    assert sig.max() >= 565.0
    cache = upload_oracle_cache(oc, cuda_device)
    q = seeded_randn((1, spec.num_q_heads, 128), cuda_device, 9).half()
    S = splits or m.omnikv_default_splits(consts.struct, cache.struct)
    part = m.partials_tensor(1, spec.num_q_heads, S, cuda_device)
    out = torch.empty(1, spec.num_q_heads, 128, device=cuda_device)
    m.omnikv_decode_attention(consts.struct, cache.struct, q, part, S)
    m.omnikv_combine(consts.struct, cache.struct, part, S, out)
    torch.cuda.synchronize()
    assert int(cache.error_word.item()) & RANGE_BIT
    assert torch.isfinite(out).all()


@pytest.mark.parametrize("splits", [0, 1])
def test_4bit_large_value_scales_decode(cuda_device, splits):
    """Values x 1024 on a 4-bit cache: the table body's value operand is the
    softmax weight times sigma (at most 65504), so scales of several thousand
    decode without a range report and within the tolerance relative to their size."""
    import bit_kv_cache_pack_b200 as m
    spec, seed = with_bits(WORKLOADS["tiny"], 4, 4), 47
    params, consts, ocfg = make_layer(spec, seed, 0, cuda_device)
    L = np.array([2048], np.int32)
    oc = _oracle_cache(spec, seed, ocfg, params, L, 2080, value_scale=1024.0)
    sig = oc.records[0, :, :, oc.off["sigma"]:].copy().view(np.float16).astype(np.float32)
    assert sig.max() >= 565.0 and np.isfinite(sig).all()
    cache = upload_oracle_cache(oc, cuda_device)
    q = seeded_randn((1, spec.num_q_heads, 128), cuda_device, 9).half()
    S = splits or m.omnikv_default_splits(consts.struct, cache.struct)
    part = m.partials_tensor(1, spec.num_q_heads, S, cuda_device)
    out = torch.empty(1, spec.num_q_heads, 128, device=cuda_device)
    m.omnikv_decode_attention(consts.struct, cache.struct, q, part, S)
    m.omnikv_combine(consts.struct, cache.struct, part, S, out)
    torch.cuda.synchronize()
    assert int(cache.error_word.item()) == 0
    check_decode(out.cpu().numpy() / 1024.0, decode_dense(ocfg, oc, q.cpu().numpy()) / 1024.0,
                 "K4 values x 1024, S=%d" % S)
