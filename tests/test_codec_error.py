"""Pins of the codec-error comparison (oracle/codec_error.py): the metrics against
closed forms and brute force, the codecs' round trips against invariants that a
wrong rotation, scale or metadata would break."""
import numpy as np
import pytest

from oracle import codec, codec_error
from oracle.attention import key_rotation_matrix

from test_oracle_codec import _cfg, _inputs


def test_kl_closed_form_and_sign():
    p, q = 0.3, 0.6
    want = p * np.log(p / q) + (1 - p) * np.log((1 - p) / (1 - q))
    got = codec_error.kl_divergence(np.array([[p, 1 - p]]), np.array([[q, 1 - q]]))[0]
    assert abs(got - want) < 1e-15
    rng = np.random.default_rng(0)
    a = rng.dirichlet(np.ones(9), 20)
    b = rng.dirichlet(np.ones(9), 20)
    assert np.all(codec_error.kl_divergence(a, b) >= 0)
    assert np.all(np.abs(codec_error.kl_divergence(a, a)) < 1e-15)
    # zero-probability terms contribute nothing
    assert codec_error.kl_divergence(np.array([[1.0, 0.0]]), np.array([[0.5, 0.5]]))[0] == np.log(2.0)


def test_metrics_brute_force_two_tokens():
    q = np.zeros((1, 128))
    q[0, 0] = np.sqrt(128.0)                  # score_t = k_t[0]
    k = np.zeros((2, 128))
    k[:, 0] = [0.0, np.log(3.0)]              # p = (1/4, 3/4)
    k_hat = k.copy()
    k_hat[1, 0] = 0.0                         # p^ = (1/2, 1/2)
    v = np.zeros((2, 128))
    v[:, 1] = [1.0, 5.0]                      # o_1 = 4
    v_hat = v.copy()                          # o^_1 = 3
    recon, kl, out = codec_error.attention_metrics(q, k, v, k_hat, v_hat)
    assert abs(recon - np.log(3.0) ** 2 / 256) < 1e-15
    assert abs(kl - (0.25 * np.log(0.5) + 0.75 * np.log(1.5))) < 1e-15
    assert abs(out - 1.0 / 128) < 1e-15


def test_identity_codec_has_no_error():
    rng = np.random.default_rng(1)
    q, k, v = rng.normal(size=(8, 128)), rng.normal(size=(50, 128)), rng.normal(size=(50, 128))
    assert codec_error.attention_metrics(q, k, v, k, v) == (0.0, 0.0, 0.0)


@pytest.mark.parametrize("bits", [2, 4])
def test_turbo_round_trip_invariants(bits):
    """x^ = R^T (sigma16 c_codes): rotated forward it lies on the scaled codebook, and
    every coordinate took its nearest codeword (a wrong rotation, scale or
    threshold breaks one of the two)."""
    rng = np.random.default_rng(2)
    cfg = _cfg(rng, bits, bits)
    x = (rng.normal(size=(40, 128)) * 2.0).astype(np.float16)
    xh = codec_error.turbo_dequantized(cfg, x, cfg.key_codebook)
    sg = codec.value_sigma(x).astype(np.float64)
    fwd = xh @ key_rotation_matrix(cfg.key_signs).T      # back to the rotated space
    cb = np.asarray(cfg.key_codebook, np.float32).astype(np.float64)
    on_grid = np.min(np.abs(fwd[:, :, None] / sg[:, None, None] - cb[None, None, :]), axis=2)
    assert on_grid.max() < 1e-9
    # every rotated coordinate took the nearest codeword (thresholds at the midpoints)
    z = codec.rotate_keys(x, cfg.key_signs).astype(np.float64) / sg[:, None]
    took = np.abs(z - fwd / sg[:, None])
    nearest = np.min(np.abs(z[:, :, None] - cb[None, None, :]), axis=2)
    assert np.all(took <= nearest + 1e-6)


@pytest.mark.parametrize("fmt", ["fp16", "mx"])
def test_omni_round_trip_stays_in_window_ranges(fmt):
    """Rotated forward, the dequantised keys of every window lie in its stored range
    [m, m + s (c_last - c_0)] (checks the inverse rotation and the metadata)."""
    rng = np.random.default_rng(3)
    cfg = _cfg(rng)
    k, v, mod = _inputs(rng, 1, 2, 70)
    kh, vh = codec_error.omni_dequantized(cfg, k[0], v[0], mod[0], fmt)
    c = codec.OracleCache(1, 2, 96, 2, 2, meta_format=fmt)
    codec.write_cache(cfg, c, k, v, mod)
    R = key_rotation_matrix(cfg.key_signs)
    span = float(cfg.key_codebook[-1]) - float(cfg.key_codebook[0])
    for h in range(2):
        kr = kh[h] @ R.T
        for w in range(3):
            m, s = (x.astype(np.float64) for x in c.key_meta_f32(0, h, w))
            blk = kr[32 * w:min(32 * w + 32, 70)]
            assert np.all(blk >= m - 1e-9) and np.all(blk <= m + s * span + 1e-9)


def test_more_bits_and_window_ranges_help_on_drifting_keys():
    """On keys whose offset drifts from window to window (the data model of the
    workloads), every codec improves from 2 to 4 bits, and the per-window key range
    reconstructs keys better than a per-token scale."""
    rng = np.random.default_rng(4)
    n, H = 256, 2
    drift = np.repeat(rng.normal(size=(H, n // 32, 128)) * 2.0, 32, axis=1)
    k = (rng.normal(size=(H, n, 128)) + drift).astype(np.float16)
    v = (rng.normal(size=(H, n, 128))).astype(np.float16)
    mod = rng.integers(0, 3, n).astype(np.uint8)
    q = rng.normal(size=(8 * H, 128)).astype(np.float16)
    res = {}
    for bits in (2, 4):
        res[bits] = codec_error.compare(_cfg(np.random.default_rng(5), bits, bits), k, v, mod, q)
    for name in codec_error.CODECS:
        assert res[4][name][0] < res[2][name][0]
    assert res[2]["omni-fp16"][0] < res[2]["turbo"][0]
