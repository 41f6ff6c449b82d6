"""MXFP4 key metadata on the GPU (paperpeel.com section 3.1, "Implementation
details": MXFP4 metadata by default), against the oracle's reading of the format
(oracle/mxmeta.py: E2M1 minima and scales, one E8M0 exponent per 32 channels, the
smallest non-saturating exponent, nearest rounding with ties to the even code, the
scale derived from the rounded minimum).

Cache write: key codes and the 144 metadata bytes of every window bit-exact, value
scales bit-exact, value codes as for the fp16 format (at a threshold within the
rotation's error bound); the records are 2,256 bytes for K2/V2. Decode: the GPU's
decode + combine over the oracle-written MXFP4 cache against the oracle's fp64
attention over the same dequantised cache, on both 2-bit decode bodies and the
4-bit build.
"""
import numpy as np
import pytest
import torch

from oracle import codec
from oracle.attention import decode_dense
from synth.workloads import WORKLOADS, decode_inputs, key_drift, prefill_inputs, seq_lengths, with_bits

from helpers import check_decode, compare_records, make_layer, seeded_randn, upload_oracle_cache

pytestmark = pytest.mark.gpu

MX = 1


def _write_both(m, consts, ocfg, gc, oc, k, v, mod):
    n = k.shape[2]
    m.omnikv_write_cache(consts.struct, gc.struct, k.contiguous(), v.contiguous(), mod.contiguous(), n)
    codec.write_cache(ocfg, oc, k.cpu().numpy(), v.cpu().numpy(), mod.cpu().numpy())
    torch.cuda.synchronize()


def _check(ocfg, oc, gc, v_all, mod_all):
    grec = gc.records.cpu().numpy()
    assert grec.shape[-1] == oc.records.shape[-1]
    assert np.array_equal(gc.seq_lens.cpu().numpy(), oc.seq_lens)
    assert int(gc.error_word.item()) == 0
    mism = 0
    for b in range(grec.shape[0]):
        T = int(oc.seq_lens[b])
        for h in range(grec.shape[1]):
            mism += compare_records(ocfg, oc, grec, b, h, range((T + 31) // 32), v_all[b, h], mod_all[b])
    return mism


@pytest.mark.parametrize("bits", [2, 4])
def test_mx_chunked_writes_bit_exact(cuda_device, bits):
    import bit_kv_cache_pack_b200 as m
    spec = with_bits(WORKLOADS["tiny"], bits, bits)
    seed = 51
    params, consts, ocfg = make_layer(spec, seed, 0, cuda_device, per_head=True, key_meta_format=MX)
    assert m.omnikv_record_bytes_meta(bits, bits, MX) == (2256 if bits == 2 else 4304)
    L = np.array([300], np.int32)
    drift = key_drift(spec, seed, 0, 16, cuda_device)
    k, v, mod = prefill_inputs(spec, seed, 0, params, drift, L, cuda_device)
    gc = m.KVCache(1, 2, 320, bits, bits, cuda_device, key_meta_format=MX)
    oc = codec.OracleCache(1, 2, 320, bits, bits, meta_format="mx")
    cuts = [0, 1, 3, 34, 67, 96, 97, 160, 191, 255, 300]
    for a, b_ in zip(cuts[:-1], cuts[1:]):
        _write_both(m, consts, ocfg, gc, oc, k[:, :, a:b_], v[:, :, a:b_], mod[:, a:b_])
        _check(ocfg, oc, gc, v.cpu().numpy(), mod.cpu().numpy())
    q = seeded_randn((1, 16, 128), cuda_device, 13).half()
    ref = decode_dense(ocfg, oc, q.cpu().numpy())
    for S in (1, 3, 0):
        S = S or m.omnikv_default_splits(consts.struct, gc.struct)
        part = m.partials_tensor(1, 16, S, cuda_device)
        out = torch.empty(1, 16, 128, device=cuda_device)
        cache = upload_oracle_cache(oc, cuda_device)
        m.omnikv_decode_attention(consts.struct, cache.struct, q, part, S)
        m.omnikv_combine(consts.struct, cache.struct, part, S, out)
        torch.cuda.synchronize()
        assert int(cache.error_word.item()) == 0
        check_decode(out.cpu().numpy(), ref, "mx bits=%d S=%d" % (bits, S))


def test_mx_prefill_append_decode(cuda_device):
    """The tiny workload's 2,048-token prefill and one appended token in MXFP4
    format; decode over the oracle's cache and over the GPU-written one, with the
    default split count (cooperative body) and one split (per-warp body), and
    through the fused decode step."""
    import bit_kv_cache_pack_b200 as m
    spec, seed = WORKLOADS["tiny"], 53
    params, consts, ocfg = make_layer(spec, seed, 0, cuda_device, key_meta_format=MX)
    L = seq_lengths(spec, seed)
    cap = 2048 + 64
    drift = key_drift(spec, seed, 0, cap // 32, cuda_device)
    k, v, mod = prefill_inputs(spec, seed, 0, params, drift, L, cuda_device)
    gc = m.KVCache(1, 2, cap, 2, 2, cuda_device, key_meta_format=MX)
    oc = codec.OracleCache(1, 2, cap, 2, 2, meta_format="mx")
    _write_both(m, consts, ocfg, gc, oc, k, v, mod)
    q, kn, vn, mn = decode_inputs(spec, seed, 0, 0, params, drift, L, cuda_device)
    _write_both(m, consts, ocfg, gc, oc, kn, vn, mn)
    v_all = torch.cat([v, vn], dim=2).cpu().numpy()
    mod_all = torch.cat([mod, mn], dim=1).cpu().numpy()
    mism = _check(ocfg, oc, gc, v_all, mod_all)
    assert mism <= 1e-4 * v_all.size
    ref = decode_dense(ocfg, oc, q.cpu().numpy())
    for cache, what in ((upload_oracle_cache(oc, cuda_device), "oracle cache"), (gc, "gpu cache")):
        for S in (0, 1):
            S = S or m.omnikv_default_splits(consts.struct, cache.struct)
            part = m.partials_tensor(1, 16, S, cuda_device)
            out = torch.empty(1, 16, 128, device=cuda_device)
            m.omnikv_decode_attention(consts.struct, cache.struct, q, part, S)
            m.omnikv_combine(consts.struct, cache.struct, part, S, out)
            torch.cuda.synchronize()
            check_decode(out.cpu().numpy(), ref, "mx %s S=%d" % (what, S))
    # the fused step (append + decode) on an MXFP4 cache, against the oracle
    q2, kn2, vn2, mn2 = decode_inputs(spec, seed, 0, 1, params, drift, L + 1, cuda_device)
    S, fused = m.omnikv_step_splits(consts.struct, gc.struct, 0)
    part = m.partials_tensor(1, 16, S, cuda_device)
    out = torch.empty(1, 16, 128, device=cuda_device)
    m.omnikv_decode_step(consts.struct, gc.struct, q2, kn2, vn2, mn2, part, 0, out)
    codec.write_cache(ocfg, oc, kn2.cpu().numpy(), vn2.cpu().numpy(), mn2.cpu().numpy())
    torch.cuda.synchronize()
    assert int(gc.error_word.item()) == 0
    check_decode(out.cpu().numpy(), decode_dense(ocfg, oc, q2.cpu().numpy()), "mx decode step (fused=%d)" % fused)
