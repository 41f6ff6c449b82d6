"""Pins for the oracle's cache write: rotation, window range, codes, packing,
value scale, and the cache-write state machine."""
import numpy as np
import pytest
import scipy.linalg

from oracle import codec
from oracle.attention import key_rotation_matrix
from oracle.codebook import lloyd_max_gaussian
from synth.workloads import codebook

F16, F32 = np.float16, np.float32
RNG = np.random.default_rng(1234)


def _signs(rng):
    return np.where(rng.random(128) < 0.5, -1.0, 1.0).astype(F32)


# --- rotation -----------------------------------------------------------------
def test_fwht_equals_library_hadamard_on_integers():
    # integer inputs keep every fp32 butterfly exact, so the result must equal
    # the product with scipy's Sylvester-ordered Hadamard matrix exactly
    H = scipy.linalg.hadamard(128).astype(np.float64)
    x = RNG.integers(-1000, 1000, size=(16, 128)).astype(F32)
    got = codec.fwht_f32(x).astype(np.float64)
    assert np.array_equal(got, x.astype(np.float64) @ H.T)


def test_rotation_matrix_orthogonal_and_sylvester():
    s = _signs(RNG)
    R = key_rotation_matrix(s)
    assert np.abs(R @ R.T - np.eye(128)).max() < 1e-12
    H = scipy.linalg.hadamard(128).astype(np.float64)
    assert np.abs(R - 2.0 ** -3.5 * H * s[None, :]).max() == 0.0
    e = np.zeros(128)
    e[37] = 1.0
    assert np.allclose(np.abs(R @ e), 2.0 ** -3.5, rtol=0, atol=1e-15)


def test_rotate_keys_close_to_fp64():
    s = _signs(RNG)
    k = RNG.normal(size=(64, 128)).astype(F16)
    got = codec.rotate_keys(k, s).astype(np.float64)
    ref = k.astype(np.float64) @ key_rotation_matrix(s).T
    # 7 butterfly stages + one scaling, each with relative rounding 2^-24
    bound = 8 * 2.0 ** -24 * np.abs(k.astype(np.float64)).sum(axis=1, keepdims=True) * 2.0 ** -3.5
    assert np.all(np.abs(got - ref) <= bound + 1e-30)
    # norm preserved up to fp32 rounding
    assert np.allclose(np.linalg.norm(got, axis=1), np.linalg.norm(k.astype(np.float64), axis=1), rtol=1e-5)


# --- key range and codes ------------------------------------------------------
@pytest.mark.parametrize("bits", [2, 4])
def test_key_exact_grid_recovers_codes(bits):
    cb = codebook(bits)
    L = len(cb)
    m = F16(-1.75)
    s = F16(0.625)
    j = RNG.integers(0, L, size=(32, 128))
    j[0, :] = 0
    j[1, :] = L - 1          # both extremes present in every channel
    x = (F32(m) + F32(s) * (cb[j] - cb[0])).astype(F32)
    m16, s16 = codec.key_window_meta(x, cb)
    assert np.all(m16 == m) and np.all(s16 == s)
    codes = codec.key_codes(x, m16, s16, cb)
    assert np.array_equal(codes, j)
    xhat = F32(m) + F32(s) * (cb[codes] - cb[0])
    assert np.all(np.abs(xhat - x) <= np.spacing(np.abs(x).astype(F32)))


@pytest.mark.parametrize("bits", [2, 4])
def test_key_codes_are_nearest_codeword(bits):
    cb = codebook(bits)
    x = (RNG.normal(size=(32, 128)) * 3 + RNG.normal(size=128)).astype(F32)
    m16, s16 = codec.key_window_meta(x, cb)
    codes = codec.key_codes(x, m16, s16, cb)
    assert codes.min() >= 0 and codes.max() < len(cb)
    z = (x.astype(np.float64) - m16.astype(np.float64)) / s16.astype(np.float64) + cb[0]
    dist = np.abs(z[..., None] - cb.astype(np.float64))
    brute = dist.argmin(axis=-1)
    # brute force nearest level; differences allowed only on exact-tie fp noise
    gap = np.sort(dist, axis=-1)
    clear = (gap[..., 1] - gap[..., 0]) > 1e-5
    assert np.array_equal(codes[clear], brute[clear])
    # error bound: half the widest cell plus the fp16 rounding of m and s
    xhat = m16.astype(np.float64) + s16.astype(np.float64) * (cb[codes] - cb[0])
    mn, mx = x.min(0).astype(np.float64), x.max(0).astype(np.float64)
    span = float(cb[-1]) - float(cb[0])
    slack = np.abs(mn - m16) + span * np.abs((mx - mn) / span - s16.astype(np.float64))
    maxgap = np.max(np.diff(cb.astype(np.float64)))
    assert np.all(np.abs(x - xhat) <= s16.astype(np.float64) * maxgap / 2 + 2 * slack + 1e-5)


def test_midpoint_goes_to_lower_level_and_constant_channel():
    cb = codebook(2)
    t = codec.thresholds(cb)
    z = np.array([t[0], t[1], t[2], np.nextafter(t[1], F32(10))], F32)
    assert list(codec.count_above(z, t)) == [0, 1, 2, 2]
    x = np.full((32, 128), 0.3, F32)
    m16, s16 = codec.key_window_meta(x, cb)
    assert np.all(s16 == 0)
    assert np.all(codec.key_codes(x, m16, s16, cb) == 0)


# --- packing ------------------------------------------------------------------
@pytest.mark.parametrize("bits", [2, 4])
def test_pack_bit_layout_brute_force(bits):
    L = 1 << bits
    cpw = 32 // bits
    codes = RNG.integers(0, L, size=(32, 128)).astype(np.uint32)
    kw = codec.pack_key_codes(codes, bits)
    vw = codec.pack_value_codes(codes, bits)
    for t in range(0, 32, 5):
        for c in range(0, 128, 7):
            assert (int(kw[t, c // cpw]) >> (bits * (c % cpw))) & (L - 1) == codes[t, c]
            assert (int(vw[t // cpw, c]) >> (bits * (t % cpw))) & (L - 1) == codes[t, c]
    assert np.array_equal(codec.unpack_key_codes(kw, bits), codes)
    assert np.array_equal(codec.unpack_value_codes(vw, bits), codes)


def test_record_sizes():
    assert codec.record_bytes(2, 2) == 2624
    assert codec.record_bytes(4, 4) == 4672


# --- values -------------------------------------------------------------------
def test_value_sigma_exact_on_integers():
    v = RNG.integers(-40, 40, size=(50, 128)).astype(F16)
    ref = np.sqrt((v.astype(np.float64) ** 2).sum(axis=1) / 128.0)
    got = codec.value_sigma(v)
    # sums of small integer squares are exact in fp32; one sqrt, one fp16 rounding
    assert np.array_equal(got, ref.astype(F32).astype(F16))


def test_value_sigma_close_on_normals():
    v = (RNG.normal(size=(200, 128)) * 3).astype(F16)
    ref = np.sqrt((v.astype(np.float64) ** 2).mean(axis=1))
    got = codec.value_sigma(v).astype(np.float64)
    assert np.all(np.abs(got - ref) <= np.spacing(ref.astype(F16)).astype(np.float64) * 0.5 + 1e-6 * ref)


def test_value_rotation_identity_and_permutation():
    cb = codebook(2)
    v = (RNG.normal(size=(40, 128)) * 2).astype(F16)
    sg = codec.value_sigma(v)
    # U = I: v' = v; codes are the brute-force nearest level of v / sigma16
    vp = codec.rotate_values(v, np.eye(128, dtype=F32))
    assert np.array_equal(vp, v.astype(F32))
    codes = codec.value_codes(vp, sg, cb)
    z = v.astype(np.float64) / sg.astype(np.float64)[:, None]
    d = np.abs(z[..., None] - cb.astype(np.float64))
    srt = np.sort(d, axis=-1)
    clear = srt[..., 1] - srt[..., 0] > 1e-5
    assert np.array_equal(codes[clear], d.argmin(-1)[clear])
    # U = permutation matrix P (columns e_{pi(j)}): v'_j = v_{pi(j)}
    pi = RNG.permutation(128)
    P = np.zeros((128, 128), F32)
    P[pi, np.arange(128)] = 1.0
    vp2 = codec.rotate_values(v, P)
    assert np.array_equal(vp2, v.astype(F32)[:, pi])
    assert np.array_equal(codec.value_codes(vp2, sg, cb), codes[:, pi])


def test_value_rotation_preserves_norm():
    from synth.workloads import _gen, _orthogonal
    U = _orthogonal(_gen("cpu", 5, 1)).numpy()
    assert np.abs(U.astype(np.float64) @ U.T.astype(np.float64) - np.eye(128)).max() < 1e-6
    v = (RNG.normal(size=(30, 128))).astype(F16)
    vp = codec.rotate_values(v, U).astype(np.float64)
    assert np.allclose(np.linalg.norm(vp, axis=1), np.linalg.norm(v.astype(np.float64), axis=1), rtol=1e-6)


# --- the cache-write state machine --------------------------------------------
def _cfg(rng, kbits=2, vbits=2, H=2, per_head=False):
    from synth.workloads import _gen, _orthogonal
    rot = np.stack([np.stack([_orthogonal(_gen("cpu", 9, h if per_head else 0, m)).numpy()
                              for m in range(3)]) for h in range(H)])
    return codec.OracleConfig(codebook(kbits), codebook(vbits), _signs(rng), rot, 8 * H, H)


def _inputs(rng, B, H, n):
    k = (rng.normal(size=(B, H, n, 128)) + rng.normal(size=(B, H, 1, 128))).astype(F16)
    v = (rng.normal(size=(B, H, n, 128)) * 1.5 + 0.3).astype(F16)
    mod = rng.integers(0, 3, size=(B, n)).astype(np.uint8)
    return k, v, mod


@pytest.mark.parametrize("bits", [2, 4])
def test_chunked_writes_equal_one_shot(bits):
    rng = np.random.default_rng(7)
    cfg = _cfg(rng, bits, bits)
    B, H, n = 2, 2, 101
    k, v, mod = _inputs(rng, B, H, n)
    one = codec.OracleCache(B, H, 128, bits, bits)
    codec.write_cache(cfg, one, k, v, mod)
    many = codec.OracleCache(B, H, 128, bits, bits)
    cuts = [0, 1, 2, 31, 33, 64, 65, 90, 100, 101]
    for a, b_ in zip(cuts[:-1], cuts[1:]):
        codec.write_cache(cfg, many, k[:, :, a:b_], v[:, :, a:b_], mod[:, a:b_])
    assert np.array_equal(one.records, many.records)
    assert np.array_equal(one.seq_lens, many.seq_lens)
    r = n % 32
    assert np.array_equal(one.key_tail[:, :, :r], many.key_tail[:, :, :r])
    assert np.array_equal(one.key_tail[:, :, :r], k[:, :, n - r:])


def test_partial_window_statistics_over_valid_tokens():
    rng = np.random.default_rng(8)
    cfg = _cfg(rng)
    k, v, mod = _inputs(rng, 1, 2, 45)
    c = codec.OracleCache(1, 2, 64, 2, 2)
    codec.write_cache(cfg, c, k, v, mod)
    # window 1 holds 13 valid tokens; its range is their min / max
    kp = codec.rotate_keys(k[0, 1, 32:45], cfg.key_signs)
    m16, s16 = codec.key_window_meta(kp, cfg.key_codebook)
    assert np.array_equal(c.meta(0, 1, 1)[:, 0], m16)
    assert np.array_equal(c.meta(0, 1, 1)[:, 1], s16)
    kc = codec.unpack_key_codes(c.k_words(0, 1, 1), 2)
    assert np.all(kc[13:] == 0)
    vc = codec.unpack_value_codes(c.v_words(0, 1, 1), 2)
    assert np.all(vc[13:] == 0)
    assert np.all(c.sigma(0, 1, 1)[13:] == 0)
    assert np.array_equal(c.modality[0, :45], mod[0])


def test_capacity_exceeded_raises():
    rng = np.random.default_rng(9)
    cfg = _cfg(rng)
    k, v, mod = _inputs(rng, 1, 2, 40)
    c = codec.OracleCache(1, 2, 32, 2, 2)
    with pytest.raises(ValueError):
        codec.write_cache(cfg, c, k, v, mod)
