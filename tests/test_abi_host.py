"""CPU-only checks of the C-ABI library: it loads, exports every function that
include/omnikv.h declares, reports sizes, and rejects bad arguments on the host
before launching anything (every call below fails validation, so no CUDA work
is ever issued)."""
import ctypes
import os
import re

import pytest

from bit_kv_cache_pack_b200 import _abi
from bit_kv_cache_pack_b200._abi import OmniKVCache, OmniKVConfig

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"OMNIKV_API\s+[\w\s\*]+?\b(omnikv_\w+)\s*\(", text)
    return names


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 8
    lib = ctypes.CDLL(_abi._LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) >= set(_abi.EXPORTED)


def test_package_exports_every_binding():
    import bit_kv_cache_pack_b200 as pkg
    for n in _abi.EXPORTED:
        if n not in ("omnikv_status_string",):
            assert hasattr(pkg, n), n


def test_sizes_and_version():
    assert _abi.omnikv_abi_version() == 3
    assert _abi.omnikv_record_bytes(2, 2) == 2624
    assert _abi.omnikv_record_bytes(4, 4) == 4672
    assert _abi.omnikv_record_bytes(2, 4) == 1024 + 512 + 2048 + 64
    assert _abi.omnikv_record_bytes(3, 2) == 0
    assert _abi.omnikv_record_bytes_meta(2, 2, _abi.OMNIKV_META_FP16) == 2624
    assert _abi.omnikv_record_bytes_meta(2, 2, _abi.OMNIKV_META_MXFP4) == 2256   # 1024 + 144 + 1024 + 64
    assert _abi.omnikv_record_bytes_meta(4, 4, _abi.OMNIKV_META_MXFP4) == 4304
    assert _abi.omnikv_record_bytes_meta(2, 2, _abi.OMNIKV_META_TURBO) == 2176   # 1024 + 64 + 1024 + 64
    assert _abi.omnikv_record_bytes_meta(4, 4, _abi.OMNIKV_META_TURBO) == 4224
    assert _abi.omnikv_record_bytes_meta(2, 2, 3) == 0
    assert _abi.omnikv_partials_bytes(2, 16, 5) == 2 * 16 * 5 * 1552
    assert _abi.omnikv_partials_bytes(0, 16, 5) == 0
    assert _abi.status_string(_abi.OMNIKV_ERR_CAPACITY) == "cache capacity exceeded"


FAKE = 0x10000  # 64 KiB-aligned fake device address; never dereferenced


def _cfg(**kw):
    c = OmniKVConfig(128, 16, 2, 32, 2, 2, FAKE, FAKE, FAKE, FAKE)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def _cache(**kw):
    c = OmniKVCache(FAKE, FAKE, FAKE, FAKE, 0, 1, 2048, 0, FAKE)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def _write_status(cfg, cache, n_new=1, k=FAKE, v=FAKE, mod=FAKE):
    lib = _abi.load()
    return lib.omnikv_write_cache(ctypes.byref(cfg), ctypes.byref(cache), k, v, mod, n_new, 0)


@pytest.mark.parametrize("kw,want", [
    (dict(head_dim=64), _abi.OMNIKV_ERR_UNSUPPORTED),
    (dict(window=16), _abi.OMNIKV_ERR_UNSUPPORTED),
    (dict(key_bits=3), _abi.OMNIKV_ERR_UNSUPPORTED),
    (dict(value_bits=8), _abi.OMNIKV_ERR_UNSUPPORTED),
    (dict(num_q_heads=15), _abi.OMNIKV_ERR_INVALID_ARG),
    (dict(num_q_heads=32, num_kv_heads=2), _abi.OMNIKV_ERR_UNSUPPORTED),
    (dict(num_kv_heads=0), _abi.OMNIKV_ERR_INVALID_ARG),
    (dict(key_codebook=None), _abi.OMNIKV_ERR_INVALID_ARG),
    (dict(value_rot=FAKE + 4), _abi.OMNIKV_ERR_INVALID_ARG),
    (dict(key_meta_format=3), _abi.OMNIKV_ERR_UNSUPPORTED),
])
def test_config_rejected(kw, want):
    assert _write_status(_cfg(**kw), _cache()) == want


@pytest.mark.parametrize("kw,want", [
    (dict(records=None), _abi.OMNIKV_ERR_INVALID_ARG),
    (dict(records=FAKE + 8), _abi.OMNIKV_ERR_INVALID_ARG),
    (dict(cap_tokens=100), _abi.OMNIKV_ERR_INVALID_ARG),
    (dict(batch=0), _abi.OMNIKV_ERR_INVALID_ARG),
    (dict(max_seq_len=4096), _abi.OMNIKV_ERR_INVALID_ARG),
    (dict(max_seq_len=2048), _abi.OMNIKV_ERR_CAPACITY),
    (dict(max_seq_len=2040), None),
])
def test_cache_rejected(kw, want):
    if want is None:  # 2040 + 9 > 2048
        assert _write_status(_cfg(), _cache(**kw), n_new=9) == _abi.OMNIKV_ERR_CAPACITY
    else:
        assert _write_status(_cfg(), _cache(**kw)) == want


def test_write_arguments_rejected():
    assert _write_status(_cfg(), _cache(), n_new=0) == _abi.OMNIKV_ERR_INVALID_ARG
    assert _write_status(_cfg(), _cache(), k=None) == _abi.OMNIKV_ERR_INVALID_ARG
    assert _write_status(_cfg(), _cache(), v=FAKE + 2) == _abi.OMNIKV_ERR_INVALID_ARG
    assert _write_status(_cfg(), _cache(), mod=None) == _abi.OMNIKV_ERR_INVALID_ARG


def test_decode_and_combine_arguments_rejected():
    lib = _abi.load()
    cfg, cache = _cfg(), _cache()
    assert lib.omnikv_decode_attention(ctypes.byref(cfg), ctypes.byref(cache), None, FAKE, 0, 0) == \
        _abi.OMNIKV_ERR_INVALID_ARG
    assert lib.omnikv_decode_attention(ctypes.byref(cfg), ctypes.byref(cache), FAKE, FAKE + 4, 0, 0) == \
        _abi.OMNIKV_ERR_INVALID_ARG
    assert lib.omnikv_decode_attention(ctypes.byref(cfg), ctypes.byref(cache), FAKE, FAKE, -1, 0) == \
        _abi.OMNIKV_ERR_INVALID_ARG
    assert lib.omnikv_combine(ctypes.byref(cfg), ctypes.byref(cache), FAKE, 1, None, 0) == \
        _abi.OMNIKV_ERR_INVALID_ARG
    bad = _cfg(head_dim=256)
    assert lib.omnikv_combine(ctypes.byref(bad), ctypes.byref(cache), FAKE, 1, FAKE, 0) == \
        _abi.OMNIKV_ERR_UNSUPPORTED
    assert lib.omnikv_default_splits(ctypes.byref(bad), ctypes.byref(cache)) == 0
    with pytest.raises(_abi.OmniKVError):
        _abi.omnikv_decode_attention(cfg, cache, None, FAKE)


def test_binding_rejects_non_contiguous_tensors():
    import torch
    t = torch.zeros(4, 8).t()
    with pytest.raises(ValueError):
        _abi._ptr(t)
    assert _abi._ptr(torch.zeros(3)) != 0


def _step_status(cfg, cache, q=FAKE, k=FAKE, v=FAKE, mod=FAKE, part=FAKE, out=FAKE):
    lib = _abi.load()
    return lib.omnikv_decode_step(ctypes.byref(cfg), ctypes.byref(cache), q, k, v, mod, part, 0, out, 0)


def test_decode_step_arguments_rejected():
    """The fused step needs the cache's step flags and every buffer, and checks
    the capacity for its one appended token, all before any launch."""
    assert _step_status(_cfg(), _cache(step_flags=None)) == _abi.OMNIKV_ERR_INVALID_ARG
    assert _step_status(_cfg(), _cache(step_flags=FAKE + 2)) == _abi.OMNIKV_ERR_INVALID_ARG
    for kw in ("q", "k", "v", "mod", "part", "out"):
        assert _step_status(_cfg(), _cache(), **{kw: None}) == _abi.OMNIKV_ERR_INVALID_ARG, kw
    assert _step_status(_cfg(), _cache(), k=FAKE + 8) == _abi.OMNIKV_ERR_INVALID_ARG
    assert _step_status(_cfg(), _cache(max_seq_len=2048)) == _abi.OMNIKV_ERR_CAPACITY
    assert _step_status(_cfg(key_bits=3), _cache()) == _abi.OMNIKV_ERR_UNSUPPORTED


def test_step_splits_and_two_phase_arguments_rejected():
    lib = _abi.load()
    f = ctypes.c_int32(7)
    assert lib.omnikv_step_splits(ctypes.byref(_cfg(key_bits=3)), ctypes.byref(_cache()), 0, ctypes.byref(f)) == 0
    assert lib.omnikv_step_splits(ctypes.byref(_cfg()), ctypes.byref(_cache()), -1, ctypes.byref(f)) == 0
    cfg, cache = _cfg(), _cache(step_flags=None)
    assert lib.omnikv_append_decode(ctypes.byref(cfg), ctypes.byref(cache), FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0) == \
        _abi.OMNIKV_ERR_INVALID_ARG
    cache = _cache(max_seq_len=2048)
    assert lib.omnikv_append_decode(ctypes.byref(cfg), ctypes.byref(cache), FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0) == \
        _abi.OMNIKV_ERR_CAPACITY
    assert lib.omnikv_combine_step(ctypes.byref(cfg), ctypes.byref(_cache()), FAKE, 0, None, 0) == \
        _abi.OMNIKV_ERR_INVALID_ARG


# The library's split counts on the host without a GPU: residency falls back to
# each decode body's register budget (per-warp body 2 CTAs per SM, cooperative
# body 3, 4-bit build 4) on 148 SMs. The expected counts are the ones the B200
# runs use (same SM count and residencies there).
@pytest.mark.parametrize("batch,tokens,bits,want", [
    (1, 10240, 2, 80),    # 2 units: cooperative wave 222, capped at one window per warp (4 per split)
    (2, 32768, 2, 111),   # cooperative wave, 10 windows per split (<= 16)
    (4, 32768, 2, 37),    # cooperative wave would give 19 windows per split: per-warp wave 296 / 8
    (16, 32768, 2, 9),    # per-warp wave 296 / 32
    (64, 32768, 2, 8),    # large batch: at least 8 splits
    (16, 32768, 4, 18),   # 4-bit build: 592 / 32
])
def test_default_split_rule(batch, tokens, bits, want):
    lib = _abi.load()
    cfg = _cfg(key_bits=bits, value_bits=bits)
    cache = _cache(batch=batch, cap_tokens=65536, max_seq_len=tokens)
    assert lib.omnikv_default_splits(ctypes.byref(cfg), ctypes.byref(cache)) == want


@pytest.mark.parametrize("batch,tokens,want_s,want_fused", [
    (1, 10240, 81, 1),    # 10,241 tokens after the append: 81 splits of 4 windows, 164 CTAs fit
    (16, 32768, 9, 1),    # 32 units x 9 per-warp splits = 288 CTAs + 8 append CTAs of 4 units each = 296
    (64, 32768, 8, 0),    # 128 units x 9 CTAs do not fit: append launch, then decode launch
])
def test_step_split_rule(batch, tokens, want_s, want_fused):
    lib = _abi.load()
    f = ctypes.c_int32(-1)
    cache = _cache(batch=batch, cap_tokens=65536, max_seq_len=tokens)
    assert lib.omnikv_step_splits(ctypes.byref(_cfg()), ctypes.byref(cache), 0, ctypes.byref(f)) == want_s
    assert f.value == want_fused


def test_calibration_arguments_rejected():
    """Host checks of omnikv_calibrate_bases run before any launch (fake device
    addresses are never dereferenced)."""
    lib = _abi.load()
    need = _abi.omnikv_calibrate_workspace_bytes(4096)
    assert need > 0 and _abi.omnikv_calibrate_workspace_bytes(0) == 0
    assert _abi.omnikv_calibrate_workspace_bytes(8192) >= need
    A = 1 << 20  # an aligned fake address
    ok = dict(values=A, modality=A, weights=A, num_tokens=4096, workspace=A, workspace_bytes=need, bases=A,
              eigenvalues=0)

    def call(**kw):
        a = dict(ok, **kw)
        return lib.omnikv_calibrate_bases(a["values"], a["modality"], a["weights"], a["num_tokens"], a["workspace"],
                                          a["workspace_bytes"], a["bases"], a["eigenvalues"], None)
    assert call(values=0) == _abi.OMNIKV_ERR_INVALID_ARG
    assert call(workspace=0) == _abi.OMNIKV_ERR_INVALID_ARG
    assert call(num_tokens=0) == _abi.OMNIKV_ERR_INVALID_ARG
    assert call(values=A + 8) == _abi.OMNIKV_ERR_INVALID_ARG       # values: 16-byte aligned
    assert call(eigenvalues=A + 4) == _abi.OMNIKV_ERR_INVALID_ARG  # eigenvalues: 8-byte aligned
    assert call(workspace_bytes=need - 1) == _abi.OMNIKV_ERR_CAPACITY


def test_streaming_arguments_rejected():
    """Host checks of the streaming entry points run before any launch."""
    lib = _abi.load()
    cfg, cache = _cfg(), _cache()

    def write(ring_k=FAKE, ring_v=FAKE, k=FAKE, v=FAKE, mod=FAKE, n=1, c=None):
        return lib.omnikv_stream_write_cache(ctypes.byref(cfg), ctypes.byref(c or cache), ring_k, ring_v, k, v, mod,
                                             n, None)

    def decode(ring_k=FAKE, ring_v=FAKE, q=FAKE, part=FAKE, S=0, out=FAKE):
        return lib.omnikv_stream_decode(ctypes.byref(cfg), ctypes.byref(cache), ring_k, ring_v, q, part, S, out, None)
    assert write(ring_k=0) == _abi.OMNIKV_ERR_INVALID_ARG
    assert write(ring_v=FAKE + 8) == _abi.OMNIKV_ERR_INVALID_ARG        # rings: 16-byte aligned
    assert write(n=0) == _abi.OMNIKV_ERR_INVALID_ARG
    assert write(n=4096) == _abi.OMNIKV_ERR_CAPACITY                     # past cap_tokens
    assert decode(ring_v=0) == _abi.OMNIKV_ERR_INVALID_ARG
    assert decode(out=0) == _abi.OMNIKV_ERR_INVALID_ARG
    assert decode(q=0) == _abi.OMNIKV_ERR_INVALID_ARG
    assert decode(S=-1) == _abi.OMNIKV_ERR_INVALID_ARG
    assert decode(S=4096) == _abi.OMNIKV_ERR_UNSUPPORTED  # 4096 body splits + 4 tail splits: past the 4096 limit
