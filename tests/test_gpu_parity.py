"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Cache write: key codes, window metadata, value scales, modality ids, lengths
and the key tail bit-exact; value codes equal except adjacent codes at a
threshold (the rotation is accumulated in a different order). Decode: the
GPU's decode + combine over the ORACLE-written cache against the oracle's fp64
attention over the same dequantised cache: max abs <= 2e-3, rel L2 <= 1e-3.
"""
import numpy as np
import pytest
import torch

from oracle import codec
from oracle.attention import decode_dense
from synth.workloads import WORKLOADS, decode_inputs, key_drift, prefill_inputs, seq_lengths, with_bits

from helpers import check_decode, compare_records, make_layer, seeded_randn, upload_oracle_cache

pytestmark = pytest.mark.gpu


def _abi():
    import bit_kv_cache_pack_b200 as m
    return m


def gpu_decode(consts, cache, q, num_splits=0):
    m = _abi()
    B, Hq, _ = q.shape
    S = num_splits or m.omnikv_default_splits(consts.struct, cache.struct)
    part = m.partials_tensor(B, Hq, S, q.device)
    out = torch.empty(B, Hq, 128, dtype=torch.float32, device=q.device)
    m.omnikv_decode_attention(consts.struct, cache.struct, q, part, S)
    m.omnikv_combine(consts.struct, cache.struct, part, S, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _write_both(consts, ocfg, gcache, ocache, k, v, mod):
    m = _abi()
    n = k.shape[2]
    m.omnikv_write_cache(consts.struct, gcache.struct, k.contiguous(), v.contiguous(), mod.contiguous(), n)
    codec.write_cache(ocfg, ocache, k.cpu().numpy(), v.cpu().numpy(), mod.cpu().numpy())
    torch.cuda.synchronize()


def _check_state(ocfg, ocache, gcache, v_all, mod_all):
    grec = gcache.records.cpu().numpy()
    assert np.array_equal(gcache.seq_lens.cpu().numpy(), ocache.seq_lens)
    assert int(gcache.error_word.item()) == 0
    B, H = grec.shape[:2]
    mism = 0
    for b in range(B):
        T = int(ocache.seq_lens[b])
        assert np.array_equal(gcache.modality[b, :T].cpu().numpy(), ocache.modality[b, :T])
        r = T % 32
        if r:
            assert np.array_equal(gcache.key_tail[b, :, :r].cpu().numpy(), ocache.key_tail[b, :, :r])
        for h in range(H):
            mism += compare_records(ocfg, ocache, grec, b, h, range((T + 31) // 32), v_all[b, h], mod_all[b])
    return mism


def test_config0_write_append_decode(cuda_device):
    """The tiny configuration end to end: 2048-token prefill, one appended text
    token, one decode step."""
    m = _abi()
    spec, seed = WORKLOADS["tiny"], 0
    params, consts, ocfg = make_layer(spec, seed, 0, cuda_device)
    L = seq_lengths(spec, seed)
    cap = 2048 + 32
    drift = key_drift(spec, seed, 0, cap // 32, cuda_device)
    k, v, mod = prefill_inputs(spec, seed, 0, params, drift, L, cuda_device)
    gc = m.KVCache(spec.batch, spec.num_kv_heads, cap, 2, 2, cuda_device)
    oc = codec.OracleCache(spec.batch, spec.num_kv_heads, cap, 2, 2)
    _write_both(consts, ocfg, gc, oc, k, v, mod)
    q, kn, vn, mn = decode_inputs(spec, seed, 0, 0, params, drift, L, cuda_device)
    _write_both(consts, ocfg, gc, oc, kn, vn, mn)
    v_all = torch.cat([v, vn], dim=2).cpu().numpy()
    mod_all = torch.cat([mod, mn], dim=1).cpu().numpy()
    mism = _check_state(ocfg, oc, gc, v_all, mod_all)
    assert mism <= 1e-4 * v_all.size
    ref = decode_dense(ocfg, oc, q.cpu().numpy())
    out = gpu_decode(consts, upload_oracle_cache(oc, cuda_device), q)
    check_decode(out, ref, "oracle cache")
    out2 = gpu_decode(consts, gc, q)  # the GPU-written cache end to end
    check_decode(out2, ref, "gpu cache")


@pytest.mark.parametrize("bits", [2, 4])
def test_chunked_writes_and_tail(cuda_device, bits):
    """Prefill in ragged chunks (1, 2, 31, 33, ... tokens), per-head value bases:
    every partial-window path of the write."""
    m = _abi()
    spec = with_bits(WORKLOADS["tiny"], bits, bits)
    seed = 3
    params, consts, ocfg = make_layer(spec, seed, 0, cuda_device, per_head=True)
    L = np.array([300], np.int32)
    drift = key_drift(spec, seed, 0, 16, cuda_device)
    k, v, mod = prefill_inputs(spec, seed, 0, params, drift, L, cuda_device)
    gc = m.KVCache(1, 2, 320, bits, bits, cuda_device)
    oc = codec.OracleCache(1, 2, 320, bits, bits)
    cuts = [0, 1, 3, 34, 67, 96, 97, 160, 191, 255, 300]
    for a, b_ in zip(cuts[:-1], cuts[1:]):
        _write_both(consts, ocfg, gc, oc, k[:, :, a:b_], v[:, :, a:b_], mod[:, a:b_])
        _check_state(ocfg, oc, gc, v.cpu().numpy(), mod.cpu().numpy())
    q = seeded_randn((1, 16, 128), cuda_device, 11).half()
    ref = decode_dense(ocfg, oc, q.cpu().numpy())
    check_decode(gpu_decode(consts, upload_oracle_cache(oc, cuda_device), q), ref, "bits=%d" % bits)


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("splits", [1, 2, 3, 5, 7, 64, 200])
def test_decode_split_counts(cuda_device, splits, bits):
    """1,000 tokens (32 windows). 2-bit: one split of 32 windows runs the per-warp
    body; 16, 11, 7, 5 and 1 windows per split run the cooperative body (whole and
    partial window groups). 4-bit: the per-warp table body at every split length
    (one to four windows per warp, warps without windows)."""
    m = _abi()
    spec, seed = with_bits(WORKLOADS["tiny"], bits, bits), 5
    params, consts, ocfg = make_layer(spec, seed, 0, cuda_device)
    L = np.array([1000], np.int32)
    drift = key_drift(spec, seed, 0, 32, cuda_device)
    k, v, mod = prefill_inputs(spec, seed, 0, params, drift, L, cuda_device)
    oc = codec.OracleCache(1, 2, 1024, bits, bits)
    codec.write_cache(ocfg, oc, k.cpu().numpy(), v.cpu().numpy(), mod.cpu().numpy())
    for scale in (1.0, 3.0):  # 3x sharpens the attention (larger error amplification)
        g = torch.Generator(device=cuda_device).manual_seed(splits)
        q = (scale * torch.randn(1, 16, 128, device=cuda_device, generator=g)).half()
        ref = decode_dense(ocfg, oc, q.cpu().numpy())
        check_decode(gpu_decode(consts, upload_oracle_cache(oc, cuda_device), q, splits), ref,
                     "K%d S=%d scale=%g" % (bits, splits, scale))


@pytest.mark.parametrize("bits", [2, 4])
def test_decode_edge_cases(cuda_device, bits):
    """Batch of four: an empty sequence (zeros), a single token, a zero query
    (mean of the values) and a one-window sequence."""
    m = _abi()
    spec, seed = with_bits(WORKLOADS["tiny"], bits, bits), 6
    params, consts, ocfg = make_layer(spec, seed, 0, cuda_device)
    drift = key_drift(spec, seed, 0, 4, cuda_device)
    oc = codec.OracleCache(4, 2, 96, bits, bits)
    gc = m.KVCache(4, 2, 96, bits, bits, cuda_device)
    for b, n in [(1, 1), (2, 70), (3, 32)]:
        k, v, mod = prefill_inputs(spec, seed + b, 0, params, drift, np.array([n]), cuda_device)
        view = gc.sequence_view(b)
        m.omnikv_write_cache(consts.struct, view, k.contiguous(), v.contiguous(), mod.contiguous(), n)
        sub = codec.OracleCache(1, 2, 96, bits, bits)
        codec.write_cache(ocfg, sub, k.cpu().numpy(), v.cpu().numpy(), mod.cpu().numpy())
        oc.records[b], oc.key_tail[b], oc.modality[b], oc.seq_lens[b] = (
            sub.records[0], sub.key_tail[0], sub.modality[0], sub.seq_lens[0])
    gc.struct.max_seq_len = 70
    torch.cuda.synchronize()
    assert np.array_equal(gc.seq_lens.cpu().numpy(), [0, 1, 70, 32])
    q = seeded_randn((4, 16, 128), cuda_device, 12).half()
    q[2] = 0
    ref = decode_dense(ocfg, oc, q.cpu().numpy())
    out = gpu_decode(consts, upload_oracle_cache(oc, cuda_device), q)
    assert np.all(out[0] == 0)
    check_decode(out, ref, "edge cases K%d" % bits)


def test_device_capacity_check_sets_error_word(cuda_device):
    """A host bound that understates the device length: the kernel skips the
    write and reports it in the error word, without faulting."""
    m = _abi()
    spec, seed = WORKLOADS["tiny"], 7
    params, consts, ocfg = make_layer(spec, seed, 0, cuda_device)
    gc = m.KVCache(1, 2, 64, 2, 2, cuda_device)
    gc.seq_lens.fill_(60)
    k = seeded_randn((1, 2, 8, 128), cuda_device, 13).half()
    mod = torch.zeros(1, 8, dtype=torch.uint8, device=cuda_device)
    m.omnikv_write_cache(consts.struct, gc.struct, k, k.clone(), mod, 8)
    torch.cuda.synchronize()
    assert int(gc.error_word.item()) & m.OMNIKV_DEVERR_CAPACITY
    assert int(gc.seq_lens.item()) == 60
    assert int(gc.records.sum().item()) == 0


def test_asymmetric_codebook_uses_generic_path(cuda_device):
    """A 2-bit codebook that is not symmetric takes the CUDA-core path inside
    the same kernel; results still match the oracle."""
    import dataclasses
    m = _abi()
    spec, seed = WORKLOADS["tiny"], 8
    params, consts, ocfg = make_layer(spec, seed, 0, cuda_device)
    cb = np.array([-1.2, -0.3, 0.5, 1.7], np.float32)
    consts = m.LayerConstants(cb, cb, params["key_signs"], params["value_rot"], spec.num_q_heads, cuda_device)
    ocfg = dataclasses.replace(ocfg, key_codebook=cb, value_codebook=cb)
    L = np.array([500], np.int32)
    drift = key_drift(spec, seed, 0, 16, cuda_device)
    k, v, mod = prefill_inputs(spec, seed, 0, params, drift, L, cuda_device)
    gc = m.KVCache(1, 2, 512, 2, 2, cuda_device)
    oc = codec.OracleCache(1, 2, 512, 2, 2)
    _write_both(consts, ocfg, gc, oc, k, v, mod)
    _check_state(ocfg, oc, gc, v.cpu().numpy(), mod.cpu().numpy())
    q = seeded_randn((1, 16, 128), cuda_device, 11).half()
    ref = decode_dense(ocfg, oc, q.cpu().numpy())
    check_decode(gpu_decode(consts, upload_oracle_cache(oc, cuda_device), q, 3), ref, "asymmetric")


@pytest.mark.parametrize("splits", [1, 3])
def test_4bit_codebook_with_full_fp32_mantissas(cuda_device, splits):
    """The 4-bit tensor-core body holds each codeword as an fp16 high + low pair:
    an asymmetric 16-level codebook whose entries use the whole fp32 mantissa (no
    entry exact in fp16) still matches the oracle, keys and values."""
    import dataclasses
    m = _abi()
    spec, seed = with_bits(WORKLOADS["tiny"], 4, 4), 10
    params, consts, ocfg = make_layer(spec, seed, 0, cuda_device)
    rng = np.random.default_rng(10)
    kb = np.sort(rng.normal(0.3, 1.1, 16)).astype(np.float32)
    vb = np.sort(rng.normal(-0.2, 0.9, 16)).astype(np.float32)
    assert np.all(np.diff(kb) > 0) and np.all(np.diff(vb) > 0)
    assert not np.any(kb.astype(np.float16).astype(np.float32) == kb)
    consts = m.LayerConstants(kb, vb, params["key_signs"], params["value_rot"], spec.num_q_heads, cuda_device)
    ocfg = dataclasses.replace(ocfg, key_codebook=kb, value_codebook=vb)
    L = np.array([700], np.int32)
    drift = key_drift(spec, seed, 0, 22, cuda_device)
    k, v, mod = prefill_inputs(spec, seed, 0, params, drift, L, cuda_device)
    oc = codec.OracleCache(1, 2, 704, 4, 4)
    codec.write_cache(ocfg, oc, k.cpu().numpy(), v.cpu().numpy(), mod.cpu().numpy())
    for scale in (1.0, 3.0):
        q = (scale * seeded_randn((1, 16, 128), cuda_device, 15)).half()
        ref = decode_dense(ocfg, oc, q.cpu().numpy())
        check_decode(gpu_decode(consts, upload_oracle_cache(oc, cuda_device), q, splits), ref,
                     "K4 fp32 codebook S=%d scale=%g" % (splits, scale))


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("G,hkv", [(1, 4), (4, 2), (8, 1)])
def test_group_sizes(cuda_device, G, hkv, bits):
    """GQA groups smaller than 8 leave tensor-core columns unused; every group
    size up to 8 must match the oracle, with both 2-bit decode bodies (600 tokens:
    one split of 19 windows runs the per-warp body, 4 splits the cooperative one)
    and the 4-bit table body."""
    import dataclasses
    m = _abi()
    spec = dataclasses.replace(with_bits(WORKLOADS["tiny"], bits, bits), num_q_heads=G * hkv, num_kv_heads=hkv)
    seed = 9
    params, consts, ocfg = make_layer(spec, seed, 0, cuda_device, per_head=True)
    L = np.array([600, 70], np.int32)
    spec2 = dataclasses.replace(spec, batch=2)
    drift = key_drift(spec2, seed, 0, 20, cuda_device)
    k, v, mod = prefill_inputs(spec2, seed, 0, params, drift, np.array([600, 600]), cuda_device)
    oc = codec.OracleCache(2, hkv, 640, bits, bits)
    for b in range(2):
        sub = codec.OracleCache(1, hkv, 640, bits, bits)
        n = int(L[b])
        codec.write_cache(ocfg, sub, k[b:b + 1, :, :n].cpu().numpy(), v[b:b + 1, :, :n].cpu().numpy(),
                          mod[b:b + 1, :n].cpu().numpy())
        oc.records[b], oc.key_tail[b], oc.modality[b], oc.seq_lens[b] = (
            sub.records[0], sub.key_tail[0], sub.modality[0], sub.seq_lens[0])
    q = seeded_randn((2, G * hkv, 128), cuda_device, 14 + G).half()
    ref = decode_dense(ocfg, oc, q.cpu().numpy())
    for S in (1, 4):
        check_decode(gpu_decode(consts, upload_oracle_cache(oc, cuda_device), q, S), ref, "K%d G=%d S=%d" % (bits, G, S))
