"""Pins of the oracle's TurboQuant key codec (codec.quantize_key_window_turbo, the
"turbo" record format) against what the codec's definition fixes: the per-token
scale ||k|| / sqrt(128) (fp64 within fp16 rounding; exact on integers), codes that
are the nearest codeword of k' / sigma (brute force), a closed-form case (one-hot
keys: every rotated entry is +-sigma up to rounding, so every code is the top or
bottom level by the sign of the Hadamard row), per-token independence (any chunking of a write, and
any other token in the window, leaves a token's codes and scale unchanged), the
record layout, and the decode over a turbo cache (fused order == dense definition,
zero query == mean value, one token == its value)."""
import numpy as np
import pytest

from oracle import codec
from oracle.attention import decode_dense, decode_fused, dequantize, key_rotation_matrix

from test_oracle_codec import _cfg, _inputs

F16 = np.float16
F64 = np.float64


def _turbo_cache(cfg, k, v, mod, cap=None):
    B, H, n, _ = k.shape
    c = codec.OracleCache(B, H, cap or -(-n // 32) * 32, cfg.key_bits, cfg.value_bits, meta_format="turbo")
    codec.write_cache(cfg, c, k, v, mod)
    return c


def test_record_layout():
    assert codec.record_bytes(2, 2, "turbo") == 1024 + 64 + 1024 + 64
    assert codec.record_bytes(4, 4, "turbo") == 2048 + 64 + 2048 + 64
    off = codec.record_offsets(2, 2, "turbo")
    assert (off["meta"], off["v"], off["sigma"]) == (1024, 1088, 2112)


@pytest.mark.parametrize("bits", [2, 4])
def test_scale_is_the_token_norm(bits):
    rng = np.random.default_rng(1)
    cfg = _cfg(rng, bits, bits)
    k, v, mod = _inputs(rng, 1, 2, 70)
    k *= F16(3.0)
    c = _turbo_cache(cfg, k, v, mod)
    for h in range(2):
        sg = np.concatenate([c.key_sigma(0, h, w) for w in range(3)])[:70].astype(F64)
        want = np.sqrt((k[0, h].astype(F64) ** 2).mean(axis=1))
        # fp16 rounding of an fp32 pairwise sum: within one fp16 ulp
        assert np.all(np.abs(sg - want) <= np.spacing(want.astype(F16)).astype(F64))
        assert np.all(c.key_sigma(0, h, 2)[70 - 64:] == 0)  # padded rows


def test_scale_exact_on_integers():
    # integer keys: the sum of squares is exact in fp32, so sigma16 = fp16(sqrt(S / 128))
    rng = np.random.default_rng(2)
    cfg = _cfg(rng)
    k = rng.integers(-20, 21, size=(1, 2, 40, 128)).astype(F16)
    _, v, mod = _inputs(rng, 1, 2, 40)
    c = _turbo_cache(cfg, k, v, mod, cap=64)
    S = (k[0].astype(np.int64) ** 2).sum(axis=2)
    want = np.sqrt(S / 128.0).astype(np.float32).astype(F16)
    got = np.stack([np.concatenate([c.key_sigma(0, h, 0), c.key_sigma(0, h, 1)])[:40] for h in range(2)])
    np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("bits", [2, 4])
def test_codes_are_the_nearest_codeword(bits):
    rng = np.random.default_rng(3)
    cfg = _cfg(rng, bits, bits)
    k, v, mod = _inputs(rng, 1, 2, 64)
    c = _turbo_cache(cfg, k, v, mod)
    cb = np.asarray(cfg.key_codebook, np.float32).astype(F64)
    for h in range(2):
        kp = codec.rotate_keys(k[0, h], cfg.key_signs)
        for w in range(2):
            codes = codec.unpack_key_codes(c.k_words(0, h, w), bits)
            sg = c.key_sigma(0, h, w).astype(np.float32)
            z = (kp[32 * w:32 * w + 32] / sg[:, None]).astype(F64)   # the fp32 quotient the rule reads
            nearest = np.argmin(np.abs(z[:, :, None] - cb[None, None, :]), axis=2)
            np.testing.assert_array_equal(codes, nearest)


def test_one_hot_keys_closed_form():
    # k = a e_i: k' = R k has every entry +-fp32(a 2^-3.5) and sigma16 = fp16 of the
    # correctly rounded fp32 sqrt(a^2 / 128), so z = +-1 within fp16 rounding and the
    # 2-bit codes are the top (z ~ 1 > t_2 = 0.98) or bottom level
    rng = np.random.default_rng(4)
    cfg = _cfg(rng)
    n = 32
    k = np.zeros((1, 2, n, 128), F16)
    amp = np.array([0.5, 1.0, 2.0, 3.0, 6.0, 12.0, 0.25, 48.0] * 4, F16)
    for t in range(n):
        k[0, :, t, (5 * t) % 128] = amp[t] * (1 if t % 3 else -1)
    _, v, mod = _inputs(rng, 1, 2, n)
    c = _turbo_cache(cfg, k, v, mod)
    R = key_rotation_matrix(cfg.key_signs)
    for h in range(2):
        codes = codec.unpack_key_codes(c.k_words(0, h, 0), 2)
        sg = c.key_sigma(0, h, 0).astype(F64)
        a32 = amp.astype(np.float32)
        np.testing.assert_array_equal(sg, np.sqrt(a32 * a32 * np.float32(1.0 / 128)).astype(F16).astype(F64))
        for t in range(n):
            i = (5 * t) % 128
            sign = np.sign(R[:, i] * float(k[0, h, t, i]))
            np.testing.assert_array_equal(codes[t], np.where(sign > 0, 3, 0))


def test_tokens_are_independent_and_chunking_is_invisible():
    rng = np.random.default_rng(5)
    cfg = _cfg(rng, 2, 2)
    B, H, n = 2, 2, 101
    k, v, mod = _inputs(rng, B, H, n)
    one = _turbo_cache(cfg, k, v, mod, cap=128)
    many = codec.OracleCache(B, H, 128, 2, 2, meta_format="turbo")
    cuts = [0, 1, 2, 31, 33, 64, 65, 90, 100, 101]
    for a, b_ in zip(cuts[:-1], cuts[1:]):
        codec.write_cache(cfg, many, k[:, :, a:b_], v[:, :, a:b_], mod[:, a:b_])
    assert np.array_equal(one.records, many.records)
    # a token's key codes and scale do not depend on the other tokens of its window
    k2 = k.copy()
    k2[:, :, 40:64] = (k2[:, :, 40:64].astype(np.float32) * 7.0).astype(F16)
    other = _turbo_cache(cfg, k2, v, mod, cap=128)
    for b in range(B):
        for h in range(H):
            a = codec.unpack_key_codes(one.k_words(b, h, 1), 2)[:8]
            o = codec.unpack_key_codes(other.k_words(b, h, 1), 2)[:8]
            np.testing.assert_array_equal(a, o)
            np.testing.assert_array_equal(one.key_sigma(b, h, 1)[:8], other.key_sigma(b, h, 1)[:8])


def test_dequantised_keys_match_the_codec_error_formula():
    # the record round trip equals the direct TurboQuant formula of the codec-error
    # comparison (rotate, per-token scale, codes, sigma16 c_j, back to the original basis)
    from oracle.codec_error import turbo_dequantized
    rng = np.random.default_rng(6)
    cfg = _cfg(rng)
    k, v, mod = _inputs(rng, 1, 2, 77)
    c = _turbo_cache(cfg, k, v, mod)
    R = key_rotation_matrix(cfg.key_signs)
    for h in range(2):
        kq, _, _ = dequantize(cfg, c, 0, h)
        np.testing.assert_allclose(kq @ R, turbo_dequantized(cfg, k[0, h], cfg.key_codebook), rtol=0, atol=1e-12)


@pytest.mark.parametrize("splits", [1, 3, 100])
def test_decode_fused_equals_dense(splits):
    rng = np.random.default_rng(7)
    cfg = _cfg(rng)
    k, v, mod = _inputs(rng, 2, 2, 150)
    c = _turbo_cache(cfg, k, v, mod, cap=160)
    q = (rng.normal(size=(2, 16, 128)) * 1.5).astype(F16)
    assert np.abs(decode_dense(cfg, c, q) - decode_fused(cfg, c, q, num_splits=splits)).max() < 1e-10


def test_decode_special_cases():
    rng = np.random.default_rng(8)
    cfg = _cfg(rng)
    k, v, mod = _inputs(rng, 1, 2, 1)
    c = _turbo_cache(cfg, k, v, mod)
    q = rng.normal(size=(1, 16, 128)).astype(F16)
    d = decode_dense(cfg, c, q)
    for h in range(2):
        _, vq, md = dequantize(cfg, c, 0, h)
        v0 = cfg.value_rot[h, md[0]].astype(F64) @ vq[0]
        assert np.abs(d[0, 8 * h:8 * h + 8] - v0[None]).max() < 1e-12
    k, v, mod = _inputs(rng, 1, 2, 45)
    c = _turbo_cache(cfg, k, v, mod)
    d = decode_dense(cfg, c, np.zeros((1, 16, 128), F16))
    for h in range(2):
        _, vq, md = dequantize(cfg, c, 0, h)
        vo = np.stack([cfg.value_rot[h, md[t]].astype(F64) @ vq[t] for t in range(45)])
        assert np.abs(d[0, 8 * h] - vo.mean(axis=0)).max() < 1e-12
