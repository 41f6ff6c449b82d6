"""Pins of the value-basis calibration oracle (oracle/calibration.py): exact
recovery of a known eigenbasis from a sample set whose weighted covariance is known
in closed form, the Hadamard composition, orthogonality, the role of the weights,
sorting and the sign rule, and the quantisation error of the candidate bases."""
import numpy as np
import pytest

from oracle import calibration


def _orthogonal(rng, n=128):
    q, r = np.linalg.qr(rng.normal(size=(n, n)))
    return q * np.sign(np.diag(r))[None, :]


def _symmetric_samples(B, lam, mu, weight=1.0):
    """Tokens mu +- s_i b_i with s_i = sqrt(128 lam_i) and equal weights: the mean
    is mu and the weighted covariance is exactly B diag(lam) B^T."""
    s = np.sqrt(B.shape[0] * lam)
    v = np.concatenate([mu[None, :] + (s[:, None] * B.T), mu[None, :] - (s[:, None] * B.T)])
    return v, np.full(len(v), weight)


def test_covariance_closed_form():
    rng = np.random.default_rng(0)
    B = _orthogonal(rng)
    lam = np.exp(rng.uniform(-3, 3, 128))
    mu = rng.normal(size=128)
    v, a = _symmetric_samples(B, lam, mu)
    C = calibration.weighted_covariance(v, a)
    np.testing.assert_allclose(C, (B * lam[None, :]) @ B.T, atol=1e-10 * lam.max())


@pytest.mark.parametrize("seed", [1, 2])
def test_known_basis_is_recovered(seed):
    rng = np.random.default_rng(seed)
    B = _orthogonal(rng)
    lam = np.sort(np.exp(rng.uniform(-3, 3, 128)))[::-1] * (1 + 1e-3 * np.arange(128)[::-1])  # distinct
    mu = rng.normal(size=128)
    v, a = _symmetric_samples(B, lam, mu)
    mod = np.zeros(len(v), np.uint8)
    U = calibration.calibrate_bases(v, mod, a)[0].astype(np.float64)
    np.testing.assert_allclose(U.T @ U, np.eye(128), atol=1e-6)
    # U = E H with H symmetric orthogonal: E = U H; its columns equal B's up to
    # sign, in the order of descending eigenvalues
    H = calibration.hadamard_normalised()
    np.testing.assert_allclose(H @ H, np.eye(128), atol=1e-12)
    E = U @ H
    np.testing.assert_allclose(np.abs(np.diag(E.T @ B)), 1.0, atol=1e-6)
    # the sign rule: every column's largest-magnitude entry is positive
    idx = np.argmax(np.abs(E), axis=0)
    assert np.all(E[idx, np.arange(128)] > 0)
    # after U^T the coordinates have equal variance (the mean eigenvalue)
    var = np.diag(U.T @ ((B * lam[None, :]) @ B.T) @ U)
    np.testing.assert_allclose(var, lam.mean(), rtol=1e-5)


def test_weights_zero_tokens_and_scale():
    rng = np.random.default_rng(3)
    v = rng.normal(size=(300, 128)) * np.exp(rng.uniform(-1, 1, 128))[None, :]
    a = rng.uniform(0.1, 2.0, 300)
    mod = np.zeros(300, np.uint8)
    U0 = calibration.calibrate_bases(v, mod, a)[0]
    # scaling every weight leaves the basis unchanged
    np.testing.assert_allclose(calibration.calibrate_bases(v, mod, 7.5 * a)[0], U0, atol=1e-6)
    # tokens of weight zero do not count, whatever their values
    v2 = np.concatenate([v, 1e3 * rng.normal(size=(50, 128))])
    a2 = np.concatenate([a, np.zeros(50)])
    np.testing.assert_allclose(calibration.calibrate_bases(v2, np.zeros(350, np.uint8), a2)[0], U0, atol=1e-6)
    # the weights matter: uniform weights give another basis
    assert np.abs(calibration.calibrate_bases(v, mod, np.ones(300))[0] - U0).max() > 1e-3


def test_modalities_are_calibrated_separately():
    rng = np.random.default_rng(4)
    B = [_orthogonal(rng) for _ in range(2)]
    lam = np.sort(np.exp(rng.uniform(-2, 2, 128)))[::-1] * (1 + 1e-3 * np.arange(128)[::-1])
    parts = [_symmetric_samples(B[m], lam, rng.normal(size=128)) for m in range(2)]
    v = np.concatenate([p[0] for p in parts])
    a = np.concatenate([p[1] for p in parts])
    mod = np.concatenate([np.full(len(p[0]), m, np.uint8) for m, p in enumerate(parts)])
    U = calibration.calibrate_bases(v, mod, a).astype(np.float64)
    H = calibration.hadamard_normalised()
    for m in range(2):
        np.testing.assert_allclose(np.abs(np.diag((U[m] @ H).T @ B[m])), 1.0, atol=1e-6)
    np.testing.assert_allclose(U[2], H, atol=1e-7)   # no video tokens: the plain Hadamard (c4)


def test_per_modality_bases_beat_a_pooled_basis():
    """Values whose modalities have different covariance structure (a different
    random basis and spectrum each): bases calibrated per modality (E_m H) quantise
    them with less error than one basis calibrated on the pooled tokens, which beats
    the identity (the direction of the pages' value-rotation analysis); the
    eigenbasis alone (no Hadamard) is the worst (reading c3)."""
    from synth.workloads import codebook
    rng = np.random.default_rng(5)
    n = 600
    vs, mods = [], []
    for m in range(3):
        B = _orthogonal(rng)
        lam = np.exp(rng.uniform(-4, 2, 128))
        vs.append((rng.normal(size=(n, 128)) * np.sqrt(lam)[None, :]) @ B.T + 0.2 * rng.normal(size=128)[None, :])
        mods.append(np.full(n, m, np.uint8))
    v = np.concatenate(vs).astype(np.float16)
    mod = np.concatenate(mods)
    a = np.ones(len(v))
    cb = codebook(2)
    own = calibration.calibrate_bases(v.astype(np.float64), mod, a)
    pooled = np.repeat(calibration.calibrate_bases(v.astype(np.float64), np.zeros(len(v), np.uint8), a)[:1], 3, axis=0)
    ident = np.repeat(np.eye(128, dtype=np.float32)[None], 3, axis=0)
    H = calibration.hadamard_normalised()
    eig_only = np.stack([own[m].astype(np.float64) @ H for m in range(3)]).astype(np.float32)   # E_m alone
    e_own = calibration.value_quant_mse(v, mod, own, cb)
    e_pool = calibration.value_quant_mse(v, mod, pooled, cb)
    e_id = calibration.value_quant_mse(v, mod, ident, cb)
    e_eig = calibration.value_quant_mse(v, mod, eig_only, cb)
    assert e_own < e_pool < e_id < e_eig
