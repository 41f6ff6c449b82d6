"""Pins of the MXFP4 key-metadata oracle (oracle/mxmeta.py) against what the format
and the readings fix: the E2M1 value table, the minimal shared exponent (closed
form), the rounding directions (brute force over every grid point), coverage of
each channel's range, the reconstruction error bound, exact recovery of keys that
lie on the grid, and the byte layout."""
import itertools

import numpy as np
import pytest

from oracle import codec, mxmeta
from synth.workloads import codebook

F32 = np.float32


def _codebook(bits):
    return np.asarray(codebook(bits), dtype=F32)


def test_e2m1_table():
    # sign-magnitude with 2 exponent bits (bias 1) and 1 mantissa bit: subnormal
    # 0, 0.5; normals 2^(E-1) (1 + M/2)
    want = []
    for code in range(16):
        s, e, m = code >> 3, (code >> 1) & 3, code & 1
        mag = 0.5 * m if e == 0 else 2.0 ** (e - 1) * (1 + 0.5 * m)
        want.append(-mag if s else mag)
    np.testing.assert_array_equal(mxmeta.e2m1_decode(np.arange(16)), np.asarray(want))


@pytest.mark.parametrize("seed", range(6))
def test_block_exponent_is_the_smallest_without_saturation(seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal(32) * 10.0 ** rng.uniform(-6, 6)).astype(F32)
    x[rng.integers(0, 32, 5)] = 0.0
    e = mxmeta.block_exponent(x)
    amax = float(np.max(np.abs(x.astype(np.float64))))
    assert amax <= 6.0 * 2.0 ** e
    assert amax > 6.0 * 2.0 ** (e - 1)


def test_block_exponent_edges():
    assert mxmeta.block_exponent(np.zeros(32, F32)) == -127
    assert mxmeta.block_exponent(np.full(32, 6.0, F32)) == 0      # 6 = 6 * 2^0 exactly
    assert mxmeta.block_exponent(np.full(32, 6.000001, F32)) == 1
    assert mxmeta.block_exponent(np.full(32, -3.0, F32)) == -1    # 3 = 6 * 2^-1


def _grid_values(e):
    return sorted(set(v * 2.0 ** e for v in mxmeta.e2m1_decode(np.arange(16))))


@pytest.mark.parametrize("seed", range(4))
def test_rounding_directions_by_enumeration(seed):
    rng = np.random.default_rng(100 + seed)
    for _ in range(200):
        e = int(rng.integers(-20, 20))
        x = float(F32(rng.uniform(-6.0, 6.0) * 2.0 ** e))
        vals = _grid_values(e)
        cd, vd = mxmeta.round_down(x, e)
        cu, vu = mxmeta.round_up(x, e)
        cn, vn = mxmeta.round_nearest(x, e)
        assert vd == max(v for v in vals if v <= x)
        assert vu == min(v for v in vals if v >= x)
        best = min(abs(v - x) for v in vals)
        assert abs(vn - x) == best
        assert mxmeta.e2m1_decode(cd) * 2.0 ** e == vd
        assert mxmeta.e2m1_decode(cu) * 2.0 ** e == vu
        assert mxmeta.e2m1_decode(cn) * 2.0 ** e == vn


def test_nearest_ties_go_to_the_even_code():
    # midpoints of the E2M1 grid: 0.25 0.75 1.25 1.75 2.5 3.5 5 -> 0 1 1 2 2 4 4
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    want = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    for e in (-3, 0, 2):
        for x, w in zip(mids, want):
            for sgn in (1.0, -1.0):
                code, val = mxmeta.round_nearest(sgn * x * 2.0 ** e, e)
                assert val == sgn * w * 2.0 ** e and code % 2 == 0


def test_zero_is_positive_code():
    assert mxmeta.round_down(-0.0, 3)[0] == 0
    assert mxmeta.round_up(0.0, 3)[0] == 0


def _synthetic_window(seed, n=32, outliers=4):
    """Rotated keys of one window shaped like the workloads' (drift per channel,
    a few scaled outlier channels)."""
    rng = np.random.default_rng(seed)
    raw = rng.standard_normal((n, 128)) + 0.5 * rng.standard_normal(128)[None, :]
    raw[:, rng.choice(128, outliers, replace=False)] *= 8.0
    signs = np.where(rng.random(128) < 0.5, -1.0, 1.0).astype(F32)
    return codec.rotate_keys(raw.astype(np.float16), signs)


@pytest.mark.parametrize("rounding", ["nearest", "cover"])
@pytest.mark.parametrize("bits,seed", [(2, 0), (2, 1), (2, 2), (4, 3), (4, 4)])
def test_window_metadata_and_error_bounds(bits, seed, rounding):
    cb = _codebook(bits)
    kp = _synthetic_window(seed, n=32 if seed % 2 == 0 else 17)
    m_codes, m_exps, s_codes, s_exps, m_hat, s_hat = mxmeta.window_meta_mx(kp, cb, rounding)
    mn, mx = kp.min(axis=0).astype(np.float64), kp.max(axis=0).astype(np.float64)
    m64, s64 = m_hat.astype(np.float64), s_hat.astype(np.float64)
    span = float(cb[-1]) - float(cb[0])
    top = m64 + s64 * span
    em = np.repeat(m_exps, 32).astype(np.float64)
    if rounding == "cover":
        # the rounded minimum never exceeds the true one; the range reaches the
        # maximum (up to the fp32 rounding of the required scale)
        assert np.all(m64 <= mn)
        assert np.all(top >= mx - 1e-6 * np.abs(mx))
    else:
        # within half the widest grid gap (2 * 2^e between 4 and 6) of the minimum
        assert np.all(np.abs(m64 - mn) <= 2.0 ** em)
    # reconstruction: half a codebook gap times the scale inside the stored range,
    # plus the distance by which a key lies outside it (end codes), plus the fp32
    # rounding of z
    codes = mxmeta.key_codes_mx(kp, m_hat, s_hat, cb)
    rec = mxmeta.dequantize_keys_mx(codes, m_hat, s_hat, cb)
    k64 = kp.astype(np.float64)
    gap = float(np.max(np.diff(cb.astype(np.float64))))
    outside = np.maximum(m64[None, :] - k64, 0) + np.maximum(k64 - top[None, :], 0)
    bound = s64 * (gap / 2.0) * (1 + 1e-5) + outside + 1e-6 * (np.abs(k64) + 1)
    assert np.all(np.abs(rec - k64) <= bound)
    assert codes.max() < (1 << bits)


def _codes_every_level(rng, levels):
    """[32 tokens][128 channels] codes, every level present in every channel."""
    return np.stack([rng.permutation(np.resize(np.arange(levels), 32)) for _ in range(128)], axis=1)


def test_grid_minimum_is_reproduced():
    """Minima on the E2M1 grid of their block (the block maximum sets the
    exponent): the code-0 key of each channel is exactly its minimum, so m^ = m."""
    cb = _codebook(2)
    rng = np.random.default_rng(7)
    mags = np.asarray(mxmeta.E2M1_MAGNITUDES[1:])
    m = np.zeros(128, F32)
    for b in range(4):
        em = int(rng.integers(-3, 3))
        mm = rng.choice(np.concatenate([mags, -mags]), 32) * 2.0 ** em
        mm[0] = -6.0 * 2.0 ** em
        m[32 * b:32 * b + 32] = mm
    s = (rng.uniform(0.1, 2.0, 128)).astype(F32)
    j = _codes_every_level(rng, 4)
    kp = (m[None, :].astype(np.float64) + s[None, :].astype(np.float64)
          * (cb[j].astype(np.float64) - float(cb[0]))).astype(F32)
    assert np.array_equal(kp.min(axis=0), m)
    for rounding in ("nearest", "cover"):
        m_hat = mxmeta.window_meta_mx(kp, cb, rounding)[4]
        assert np.array_equal(m_hat, m)


def test_power_of_two_scales_recover_scale_and_codes():
    """Zero minima and scales 2^k (a power of two per channel, several exponents
    per block): the keys s (c_j - c_0) and the scale each channel needs,
    max / (c_{L-1} - c_0) = s, are exact in fp32, so s^ = s and the codes return j."""
    for bits in (2, 4):
        cb = _codebook(bits)
        rng = np.random.default_rng(8 + bits)
        s = np.zeros(128, F32)
        for b in range(4):
            es = int(rng.integers(-6, 3))
            s[32 * b:32 * b + 32] = 2.0 ** (es + rng.integers(-1, 3, 32))   # 0.5 .. 4 times 2^es
        j = _codes_every_level(rng, 1 << bits)
        kp = (s[None, :].astype(np.float64) * (cb[j].astype(np.float64) - float(cb[0]))).astype(F32)
        for rounding in ("nearest", "cover"):
            m_codes, m_exps, s_codes, s_exps, m_hat, s_hat = mxmeta.window_meta_mx(kp, cb, rounding)
            assert not m_hat.any()
            assert np.array_equal(s_hat, s)
            np.testing.assert_array_equal(mxmeta.key_codes_mx(kp, m_hat, s_hat, cb), j)


def test_constant_channels():
    """A constant channel on the grid keeps s^ = 0 and codes 0 (reading r5), with
    either rounding; off the grid, the covering rounding takes the minimum down and
    a nonzero scale that reaches the value."""
    cb = _codebook(2)
    kp = _synthetic_window(11)
    rng = np.random.default_rng(12)
    grid = np.asarray([-6.0, -3.0, -1.5, -0.5, 0.0, 1.0, 2.0, 4.0], F32)
    vals = rng.choice(grid, 32).astype(F32)
    vals[0] = F32(-6.0)                     # block 0 exponent 0: every value on its grid
    kp[:, 0:32] = vals[None, :]
    kp[:, 40] = F32(1.25)                   # off the grid of block 1
    for rounding in ("nearest", "cover"):
        m_codes, m_exps, s_codes, s_exps, m_hat, s_hat = mxmeta.window_meta_mx(kp, cb, rounding)
        codes = mxmeta.key_codes_mx(kp, m_hat, s_hat, cb)
        assert m_exps[0] == 0 and s_exps[0] == -127
        assert np.array_equal(m_hat[0:32], vals) and not s_hat[0:32].any() and not codes[:, 0:32].any()
        if rounding == "cover":
            assert m_hat[40] < 1.25 < m_hat[40] + s_hat[40] * (float(cb[-1]) - float(cb[0]))
            rec = mxmeta.dequantize_keys_mx(codes, m_hat, s_hat, cb)[:, 40]
            assert np.all(np.abs(rec - 1.25) <= s_hat[40] * float(np.max(np.diff(cb))) / 2 * (1 + 1e-5))


def test_meta_bytes_round_trip_and_record_size():
    cb = _codebook(2)
    kp = _synthetic_window(21)
    meta = mxmeta.window_meta_mx(kp, cb)
    packed = mxmeta.pack_meta_mx(*meta[:4])
    assert packed.shape == (144,) and not packed[136:].any()
    back = mxmeta.unpack_meta_mx(packed)
    for a, b in itertools.zip_longest(meta, back):
        np.testing.assert_array_equal(np.asarray(a), np.asarray(b))
    assert mxmeta.record_bytes_mx(2, 2) == 2256 and mxmeta.record_bytes_mx(2, 2) % 16 == 0
    assert mxmeta.record_bytes_mx(4, 4) == 4304 and mxmeta.record_bytes_mx(4, 4) % 16 == 0
    # 70.5 B per token and kv head instead of the fp16 format's 82
    assert mxmeta.record_bytes_mx(2, 2) / 32 == 70.5 and codec.record_bytes(2, 2) / 32 == 82


def test_meta_byte_layout():
    """Channel c's element in byte c // 2 (low nibble for even c), minima first,
    then scales, then the exponent bytes e + 127 (minima, then scales)."""
    m_codes = np.arange(128) % 16
    s_codes = (np.arange(128) * 7) % 16
    packed = mxmeta.pack_meta_mx(m_codes, np.array([-127, -1, 0, 127]), s_codes, np.array([3, 2, 1, 0]))
    assert packed[0] == (0 | 1 << 4) and packed[1] == (2 | 3 << 4) and packed[63] == (14 | 15 << 4)
    assert packed[64] == (0 | 7 << 4) and packed[65] == (14 | 5 << 4)
    assert list(packed[128:136]) == [0, 126, 127, 254, 130, 129, 128, 127]


# ---- the MXFP4 format inside the oracle's cache state machine ---------------------
def _cache_cfg(rng, bits):
    from test_oracle_codec import _cfg
    return _cfg(rng, bits, bits)


@pytest.mark.parametrize("bits", [2, 4])
def test_mx_cache_chunked_writes_equal_one_shot(bits):
    """Appends in pieces re-quantise partial windows from the fp16 tail and give the
    records a single prefill writes, with MXFP4 metadata too."""
    from test_oracle_codec import _inputs
    rng = np.random.default_rng(31)
    cfg = _cache_cfg(rng, bits)
    B, H, n = 2, 2, 101
    k, v, mod = _inputs(rng, B, H, n)
    one = codec.OracleCache(B, H, 128, bits, bits, meta_format="mx")
    codec.write_cache(cfg, one, k, v, mod)
    many = codec.OracleCache(B, H, 128, bits, bits, meta_format="mx")
    cuts = [0, 1, 2, 31, 33, 64, 65, 90, 100, 101]
    for a, b_ in zip(cuts[:-1], cuts[1:]):
        codec.write_cache(cfg, many, k[:, :, a:b_], v[:, :, a:b_], mod[:, a:b_])
    assert one.records.shape[-1] == mxmeta.record_bytes_mx(bits, bits)
    assert np.array_equal(one.records, many.records)


def test_mx_cache_records_follow_the_window_functions():
    """Each stored window holds pack(codes) and pack(metadata) of its valid keys,
    and its value fields are those of the fp16-metadata cache (same values path)."""
    from test_oracle_codec import _inputs
    rng = np.random.default_rng(32)
    cfg = _cache_cfg(rng, 2)
    k, v, mod = _inputs(rng, 1, 2, 77)
    mx = codec.OracleCache(1, 2, 96, 2, 2, meta_format="mx")
    fp = codec.OracleCache(1, 2, 96, 2, 2)
    codec.write_cache(cfg, mx, k, v, mod)
    codec.write_cache(cfg, fp, k, v, mod)
    for h in range(2):
        for w, (p0, p1) in enumerate([(0, 32), (32, 64), (64, 77)]):
            kp = codec.rotate_keys(k[0, h, p0:p1], cfg.key_signs)
            meta = mxmeta.window_meta_mx(kp, cfg.key_codebook)
            codes = np.zeros((32, 128), np.uint32)
            codes[:p1 - p0] = mxmeta.key_codes_mx(kp, meta[4], meta[5], cfg.key_codebook)
            assert np.array_equal(mx.k_words(0, h, w), codec.pack_key_codes(codes, 2))
            assert np.array_equal(mx.meta_bytes(0, h, w), mxmeta.pack_meta_mx(*meta[:4]))
            assert np.array_equal(mx.v_words(0, h, w), fp.v_words(0, h, w))
            assert np.array_equal(mx.sigma(0, h, w), fp.sigma(0, h, w))


def test_mx_cache_decode_fused_equals_dense():
    from test_oracle_codec import _inputs
    from oracle.attention import decode_dense, decode_fused
    rng = np.random.default_rng(33)
    cfg = _cache_cfg(rng, 2)
    c = codec.OracleCache(2, 2, 256, 2, 2, meta_format="mx")
    k, v, mod = _inputs(rng, 2, 2, 150)
    codec.write_cache(cfg, c, k, v, mod)
    q = (rng.normal(size=(2, 16, 128)) * 1.5).astype(np.float16)
    d = decode_dense(cfg, c, q)
    for splits in (1, 3, 7):
        assert np.abs(d - decode_fused(cfg, c, q, num_splits=splits)).max() < 1e-10
