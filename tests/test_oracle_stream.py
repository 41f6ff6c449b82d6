"""Pins of the streaming / captioning policy oracle (oracle/attention.py
decode_dense_stream; paperpeel.com section 3.1 "Implementation details": keys
quantised every 128 tokens in groups of 32, values in a 128-token fp16 sliding
window): the boundaries in closed form, a context shorter than one key block
reduces to textbook attention over the raw fp16 cache (torch SDPA, fp64), a
context whose every token is quantised reduces to the ordinary decode, the
position of each boundary (moving a single token's raw key or value changes the
output exactly when the policy reads it raw), and the two-part split used by the
kernels (the quantised body and the raw tail, merged by log-sum-exp)."""
import numpy as np
import pytest
import torch

from oracle import codec
from oracle.attention import (decode_dense, decode_dense_stream, dequantize, key_rotation_matrix,
                              stream_boundaries)

from test_oracle_codec import _cfg, _inputs

F16 = np.float16
F64 = np.float64


def _cache(cfg, k, v, mod, cap=None):
    B, H, n, _ = k.shape
    c = codec.OracleCache(B, H, cap or -(-n // 32) * 32, cfg.key_bits, cfg.value_bits)
    codec.write_cache(cfg, c, k, v, mod)
    return c


def test_boundaries():
    assert stream_boundaries(0) == (0, 0)
    assert stream_boundaries(127) == (0, 0)
    assert stream_boundaries(128) == (128, 0)
    assert stream_boundaries(129) == (128, 1)
    assert stream_boundaries(300) == (256, 172)
    assert stream_boundaries(4096) == (4096, 3968)


def test_short_context_is_plain_attention_over_raw():
    rng = np.random.default_rng(1)
    cfg = _cfg(rng)
    k, v, mod = _inputs(rng, 1, 2, 100)
    c = _cache(cfg, k, v, mod)
    q = rng.normal(size=(1, 16, 128)).astype(F16)
    d = decode_dense_stream(cfg, c, k, v, q)
    for h in range(2):
        qq = torch.from_numpy(q[0, 8 * h:8 * h + 8].astype(F64))[:, None, :]
        kk = torch.from_numpy(k[0, h].astype(F64))[None].expand(8, -1, -1)
        vv = torch.from_numpy(v[0, h].astype(F64))[None].expand(8, -1, -1)
        ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv)[:, 0].numpy()
        assert np.abs(d[0, 8 * h:8 * h + 8] - ref).max() < 1e-12


def test_all_quantised_is_the_ordinary_decode():
    # with the raw inputs replaced by the dequantised cache, every reading agrees
    rng = np.random.default_rng(2)
    cfg = _cfg(rng)
    k, v, mod = _inputs(rng, 2, 2, 300)
    c = _cache(cfg, k, v, mod)
    q = rng.normal(size=(2, 16, 128)).astype(F16)
    R = key_rotation_matrix(cfg.key_signs)
    kd = np.zeros(k.shape, F64)
    vd = np.zeros(v.shape, F64)
    for b in range(2):
        for h in range(2):
            kq, vq, md = dequantize(cfg, c, b, h)
            kd[b, h] = kq @ R
            vd[b, h] = np.stack([cfg.value_rot[h, md[t]].astype(F64) @ vq[t] for t in range(300)])
    # the stream oracle reads raw inputs through fp16; feed it values exactly representable
    kd16, vd16 = kd.astype(F16), vd.astype(F16)
    d_stream = decode_dense_stream(cfg, c, kd16, vd16, q)
    d_plain = decode_dense(cfg, c, q)
    assert np.abs(d_stream - d_plain).max() < 5e-3  # only the fp16 rounding of the recent tokens differs


@pytest.mark.parametrize("T", [129, 200, 300])
def test_each_boundary_is_where_the_policy_says(T):
    rng = np.random.default_rng(3)
    cfg = _cfg(rng)
    k, v, mod = _inputs(rng, 1, 2, T)
    c = _cache(cfg, k, v, mod)
    q = (rng.normal(size=(1, 16, 128)) * 2).astype(F16)
    KB, VB = stream_boundaries(T)
    base = decode_dense_stream(cfg, c, k, v, q)
    for t in (KB - 1, KB, VB - 1, VB):
        if t < 0 or t >= T:
            continue
        key_raw, val_raw = t >= KB, t >= VB
        k2 = k.copy()
        k2[0, :, t] = (k2[0, :, t].astype(np.float32) * 3).astype(F16)
        assert (np.abs(decode_dense_stream(cfg, c, k2, v, q) - base).max() > 0) == key_raw, ("key", t)
        v2 = v.copy()
        v2[0, :, t] = (v2[0, :, t].astype(np.float32) * 3).astype(F16)
        assert (np.abs(decode_dense_stream(cfg, c, k, v2, q) - base).max() > 0) == val_raw, ("value", t)


def test_body_and_tail_merge_by_log_sum_exp():
    # the kernels' split: the windows before 32 floor(VB / 32) from the cache alone,
    # the rest (at most 159 tokens, raw where the policy says) on its own, merged
    rng = np.random.default_rng(4)
    cfg = _cfg(rng)
    T = 333
    k, v, mod = _inputs(rng, 1, 2, T)
    c = _cache(cfg, k, v, mod)
    q = rng.normal(size=(1, 16, 128)).astype(F16)
    KB, VB = stream_boundaries(T)
    T_body = 32 * (VB // 32)
    assert T - T_body <= 159
    R = key_rotation_matrix(cfg.key_signs)
    full = decode_dense_stream(cfg, c, k, v, q)
    for h in range(2):
        kq, vq, md = dequantize(cfg, c, 0, h)
        kk = kq @ R
        vv = np.stack([cfg.value_rot[h, md[t]].astype(F64) @ vq[t] for t in range(T)])
        kk[KB:] = k[0, h, KB:].astype(F64)
        vv[VB:] = v[0, h, VB:].astype(F64)
        for g in range(8):
            s = kk @ q[0, 8 * h + g].astype(F64) / np.sqrt(128)
            parts = []
            for a, b_ in ((0, T_body), (T_body, T)):
                m = s[a:b_].max()
                p = np.exp(s[a:b_] - m)
                parts.append((m, p.sum(), p @ vv[a:b_]))
            M = max(x[0] for x in parts)
            l = sum(x[1] * np.exp(x[0] - M) for x in parts)
            o = sum(x[2] * np.exp(x[0] - M) for x in parts) / l
            assert np.abs(o - full[0, 8 * h + g]).max() < 1e-12
