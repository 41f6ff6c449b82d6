"""Calibration of the value bases U_m on the GPU (paperpeel.com section 2.3; pchao.org
方法概览: attention-contribution-weighted covariance per modality, its
eigendecomposition, U_m = E_m H) against the oracle (oracle/calibration.py, fp64
with LAPACK's symmetric eigensolver): eigenvalues to 1e-9 of the largest, bases to
2e-6 per entry (fp32 storage), orthogonality, the plain Hadamard rotation for a
modality without weight, and invariance to tokens with zero weight or a foreign id.
A modality with fewer weighted tokens than 129 has a singular covariance whose null
space has no unique eigenbasis: there the eigenpairs with distinct nonzero
eigenvalues are compared, and the rest are checked as eigenvectors (residual).

Inputs: one (layer, kv head) of a workload's synthetic values (per-modality means
and variances, the workload's modality layout) and, as the attention contribution
a_t, the attention weight each token receives from the kv head's query heads for a
few synthetic decode queries (softmax over the raw keys), as reading c1 defines it.
"""
import dataclasses

import numpy as np
import pytest
import torch

from oracle.calibration import calibrate_bases, eigenbasis, hadamard_normalised, weighted_covariance
from synth.workloads import WORKLOADS, decode_inputs, key_drift, layer_params, prefill_inputs

pytestmark = pytest.mark.gpu


def _calibration_set(name, T, seed, head=0, n_queries=4):
    spec = dataclasses.replace(WORKLOADS[name], batch=1)
    params = layer_params(spec, seed, 0)
    drift = key_drift(spec, seed, 0, T // 32 + 1, "cpu")
    k, v, mod = prefill_inputs(spec, seed, 0, params, drift, np.array([T]), "cpu")
    G = spec.num_q_heads // spec.num_kv_heads
    kh = k[0, head].double().numpy()
    a = np.zeros(T)
    for step in range(n_queries):
        q = decode_inputs(spec, seed, 0, step, params, drift, np.array([T]), "cpu")[0][0].double().numpy()
        s = q[head * G:(head + 1) * G] @ kh.T / np.sqrt(128.0)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        a += (p / p.sum(axis=1, keepdims=True)).sum(axis=0)
    return v[0, head].numpy(), mod[0].numpy(), a.astype(np.float32)


def _gpu(values, mod, a, dev):
    import bit_kv_cache_pack_b200 as m
    T = values.shape[0]
    vt = torch.from_numpy(values).to(dev).contiguous()
    mt = torch.from_numpy(mod).to(dev).contiguous()
    at = torch.from_numpy(a).to(dev).contiguous()
    ws = torch.empty(m.omnikv_calibrate_workspace_bytes(T) // 8 + 1, dtype=torch.float64, device=dev)
    bases = torch.empty(3, 128, 128, dtype=torch.float32, device=dev)
    lam = torch.empty(3, 128, dtype=torch.float64, device=dev)
    m.omnikv_calibrate_bases(vt, mt, at, T, ws, bases, lam)
    torch.cuda.synchronize()
    return bases.cpu().numpy(), lam.cpu().numpy()


def _oracle_eigenvalues(values, mod, a):
    out = np.zeros((3, 128))
    for mm in range(3):
        sel = (mod == mm) & (a > 0)
        if sel.any():
            out[mm] = eigenbasis(weighted_covariance(values[sel], a[sel]))[1]
    return out


@pytest.mark.parametrize("name,T", [("omni30b-b8", 2048), ("omni30b-b8", 8192)])
def test_bases_match_the_oracle(cuda_device, name, T):
    values, mod, a = _calibration_set(name, T, seed=5)
    assert min(np.bincount(mod[a > 0], minlength=3)) >= 256  # full-rank covariances
    bases, lam = _gpu(values, mod, a, cuda_device)
    ref = calibrate_bases(values, mod, a)
    ref_lam = _oracle_eigenvalues(values, mod, a)
    for mm in range(3):
        assert np.all(np.abs(lam[mm] - ref_lam[mm]) <= 1e-9 * np.abs(ref_lam[mm]).max()), mm
        err = np.abs(bases[mm].astype(np.float64) - ref[mm].astype(np.float64)).max()
        assert err <= 2e-6, (mm, err)
        U = bases[mm].astype(np.float64)
        assert np.abs(U.T @ U - np.eye(128)).max() < 1e-5


def test_modality_without_weight_keeps_the_hadamard_rotation(cuda_device):
    values, mod, a = _calibration_set("omni30b-b8", 2048, seed=7)
    a = a.copy()
    a[mod == 1] = 0.0                  # audio: no weight at all
    mod = mod.copy()
    mod[:64] = 7                       # ids outside 0..2 are ignored
    bases, lam = _gpu(values, mod, a, cuda_device)
    np.testing.assert_array_equal(bases[1], hadamard_normalised().astype(np.float32))
    assert np.all(lam[1] == 0.0)
    ref = calibrate_bases(values, mod, a)
    for mm in (0, 2):
        assert np.abs(bases[mm].astype(np.float64) - ref[mm].astype(np.float64)).max() <= 2e-6


def test_zero_weight_tokens_do_not_count(cuda_device):
    values, mod, a = _calibration_set("omni30b-b8", 3000, seed=9)
    base, lam = _gpu(values, mod, a, cuda_device)
    # the same set with extra tokens of zero weight (random values) interleaved
    rng = np.random.default_rng(1)
    extra = (rng.normal(size=(500, 128)) * 5).astype(np.float16)
    v2 = np.concatenate([values, extra])
    m2 = np.concatenate([mod, rng.integers(0, 3, 500).astype(np.uint8)])
    a2 = np.concatenate([a, np.zeros(500, np.float32)])
    perm = rng.permutation(len(a2))
    b2, lam2 = _gpu(v2[perm], m2[perm], a2[perm], cuda_device)
    assert np.abs(lam2 - lam).max() <= 1e-9 * np.abs(lam).max()
    assert np.abs(b2.astype(np.float64) - base.astype(np.float64)).max() <= 2e-6


def test_singular_covariance_gives_valid_eigenpairs(cuda_device):
    """omni3b's layout has 96 text tokens in 4,096: the text covariance has rank 95.
    The eigenpairs with distinct nonzero eigenvalues match the oracle's; every
    column is an eigenvector of C (residual) and the basis stays orthogonal."""
    values, mod, a = _calibration_set("omni3b-b16", 4096, seed=5)
    bases, lam = _gpu(values, mod, a, cuda_device)
    ref = calibrate_bases(values, mod, a)
    H = hadamard_normalised()
    sel = (mod == 0) & (a > 0)
    C = weighted_covariance(values[sel], a[sel])
    ref_lam = _oracle_eigenvalues(values, mod, a)[0]
    top = np.abs(ref_lam).max()
    E = bases[0].astype(np.float64) @ H          # U = E H, H symmetric and orthogonal
    E_ref = ref[0].astype(np.float64) @ H
    assert np.abs(E.T @ E - np.eye(128)).max() < 1e-5
    assert np.all(np.abs(lam[0] - ref_lam) <= 1e-9 * top)
    gaps = np.minimum(np.abs(np.diff(ref_lam, prepend=np.inf)), np.abs(np.diff(ref_lam, append=-np.inf)))
    distinct = (np.abs(ref_lam) > 1e-9 * top) & (gaps > 1e-6 * top)
    assert distinct.sum() >= 90
    assert np.abs(E[:, distinct] - E_ref[:, distinct]).max() <= 2e-5
    resid = C @ E - E * lam[0][None, :]
    assert np.abs(resid).max() <= 1e-5 * top
    for mm in (1, 2):  # full-rank modalities
        assert np.abs(bases[mm].astype(np.float64) - ref[mm].astype(np.float64)).max() <= 2e-6
