"""Pins for the oracle's decode attention (fp64)."""
import numpy as np
import pytest
import torch

from oracle import codec
from oracle.attention import decode_dense, decode_fused, dequantize, key_rotation_matrix

from test_oracle_codec import _cfg, _inputs

F16 = np.float16


def _filled(rng, B=2, H=2, n=(150,), kbits=2, vbits=2, per_head=False, cap=256):
    cfg = _cfg(rng, kbits, vbits, H, per_head)
    c = codec.OracleCache(B, H, cap, kbits, vbits)
    for m in n:
        k, v, mod = _inputs(rng, B, H, m)
        codec.write_cache(cfg, c, k, v, mod)
    return cfg, c


def _original_basis(cfg, c, b, h):
    kq, vq, mod = dequantize(cfg, c, b, h)
    R = key_rotation_matrix(cfg.key_signs)
    k = kq @ R
    v = np.stack([cfg.value_rot[h, mod[t]].astype(np.float64) @ vq[t] for t in range(len(mod))])
    return k, v


@pytest.mark.parametrize("splits", [1, 2, 3, 7, 100])
@pytest.mark.parametrize("per_head", [False, True])
def test_fused_equals_dense(splits, per_head):
    rng = np.random.default_rng(11)
    cfg, c = _filled(rng, per_head=per_head)
    q = (rng.normal(size=(2, 16, 128)) * 1.5).astype(F16)
    d = decode_dense(cfg, c, q)
    f = decode_fused(cfg, c, q, num_splits=splits)
    assert np.abs(d - f).max() < 1e-10


def test_dense_matches_library_attention():
    # torch's scaled_dot_product_attention in fp64 over the original-basis cache
    rng = np.random.default_rng(12)
    cfg, c = _filled(rng, B=1, n=(77,))
    q = rng.normal(size=(1, 16, 128)).astype(F16)
    d = decode_dense(cfg, c, q)
    for h in range(2):
        k, v = _original_basis(cfg, c, 0, h)
        qq = torch.from_numpy(q[0, 8 * h:8 * h + 8].astype(np.float64))[:, None, :]
        out = torch.nn.functional.scaled_dot_product_attention(
            qq, torch.from_numpy(k)[None].expand(8, -1, -1), torch.from_numpy(v)[None].expand(8, -1, -1))
        assert np.abs(out[:, 0].numpy() - d[0, 8 * h:8 * h + 8]).max() < 1e-12


def test_single_token_context_returns_its_value():
    rng = np.random.default_rng(13)
    cfg, c = _filled(rng, B=1, n=(1,))
    q = rng.normal(size=(1, 16, 128)).astype(F16)
    d = decode_dense(cfg, c, q)
    for h in range(2):
        _, v = _original_basis(cfg, c, 0, h)
        assert np.abs(d[0, 8 * h:8 * h + 8] - v[0][None]).max() < 1e-12
    assert np.abs(decode_fused(cfg, c, q, 1) - d).max() < 1e-12


def test_zero_query_gives_mean_value():
    rng = np.random.default_rng(14)
    cfg, c = _filled(rng, B=1, n=(70,))
    q = np.zeros((1, 16, 128), F16)
    d = decode_fused(cfg, c, q, 3)
    for h in range(2):
        _, v = _original_basis(cfg, c, 0, h)
        assert np.abs(d[0, 8 * h:8 * h + 8] - v.mean(axis=0)[None]).max() < 1e-12


def test_brute_force_loops_tiny():
    # pure-Python dequantisation from raw record bytes and a loop softmax
    rng = np.random.default_rng(15)
    cfg, c = _filled(rng, B=1, H=2, n=(37,), cap=64)
    q = rng.normal(size=(1, 16, 128)).astype(F16)
    d = decode_dense(cfg, c, q)
    R = key_rotation_matrix(cfg.key_signs)
    off = c.off
    for h in range(2):
        ks, vs = [], []
        for t in range(37):
            w, i = divmod(t, 32)
            rec = c.records[0, h, w]
            kp, vp = [], []
            for ch in range(128):
                kword = int.from_bytes(rec[off["k"] + 4 * (i * 8 + ch // 16):][:4].tobytes(), "little")
                j = (kword >> (2 * (ch % 16))) & 3
                m16 = rec[off["meta"] + 4 * ch:][:2].view(F16)[0]
                s16 = rec[off["meta"] + 4 * ch + 2:][:2].view(F16)[0]
                kp.append(float(m16) + float(s16) * (float(cfg.key_codebook[j]) - float(cfg.key_codebook[0])))
                vword = int.from_bytes(rec[off["v"] + 4 * ((i // 16) * 128 + ch):][:4].tobytes(), "little")
                jv = (vword >> (2 * (i % 16))) & 3
                sg = rec[off["sigma"] + 2 * i:][:2].view(F16)[0]
                vp.append(float(sg) * float(cfg.value_codebook[jv]))
            ks.append(R.T @ np.array(kp))
            vs.append(cfg.value_rot[h, c.modality[0, t]].astype(np.float64) @ np.array(vp))
        for g in range(8):
            qi = q[0, 8 * h + g].astype(np.float64)
            sc = [float(qi @ k) / np.sqrt(128.0) for k in ks]
            mx = max(sc)
            p = [np.exp(s - mx) for s in sc]
            o = sum(pi * vi for pi, vi in zip(p, vs)) / sum(p)
            assert np.abs(o - d[0, 8 * h + g]).max() < 1e-12


def test_empty_sequence_gives_zero():
    rng = np.random.default_rng(16)
    cfg, c = _filled(rng, B=2, n=(40,))
    c.seq_lens[1] = 0
    q = rng.normal(size=(2, 16, 128)).astype(F16)
    assert np.all(decode_dense(cfg, c, q)[1] == 0)
    assert np.all(decode_fused(cfg, c, q, 2)[1] == 0)


def test_planted_transpose_is_caught():
    # a plausible mistake (U instead of U^T in the value rotation) must break
    # agreement with an independent computation of the decoded values
    rng = np.random.default_rng(17)
    cfg, c = _filled(rng, B=1, n=(33,))
    good = decode_dense(cfg, c, np.zeros((1, 16, 128), F16))
    orig = codec.rotate_values
    try:
        codec.rotate_values = lambda v, U: orig(v, np.asarray(U).T)
        cfg2, c2 = _filled(np.random.default_rng(17), B=1, n=(33,))
        bad = decode_dense(cfg2, c2, np.zeros((1, 16, 128), F16))
    finally:
        codec.rotate_values = orig
    # with q = 0 the output is the mean decoded value; the true mean of the
    # inputs is a (noisy) target the correct rotation approaches far better
    rng2 = np.random.default_rng(17)
    _cfg(rng2)
    k, v, mod = _inputs(rng2, 1, 2, 33)
    true_mean = v[0].astype(np.float64).mean(axis=1)      # [H][128]
    e_good = np.abs(good[0, ::8] - true_mean).mean()
    e_bad = np.abs(bad[0, ::8] - true_mean).mean()
    assert e_good < 0.5 * e_bad
