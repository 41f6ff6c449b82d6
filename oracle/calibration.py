"""Oracle for the calibration of the per-modality value bases U_m. TEST
INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

paperpeel.com section 2.3 ("Modality-aware value rotation"): a separate basis U_m
is calibrated for each modality m in {V, A, L}; section 3.1: once per model, on
calibration clips. pchao.org "方法概览": the rotation of each modality comes from
an attention-contribution-weighted covariance matrix and its eigendecomposition.
Reading (c1..c4):
  c1  inputs: calibration values v_t [T][128] of one (layer, kv head), their
      modality ids, and a non-negative attention contribution a_t per token (the
      attention weight the token receives, summed over the queries that read it).
  c2  C_m = sum_{t of m} a_t (v_t - mu_m)(v_t - mu_m)^T / sum_{t of m} a_t with the
      weighted mean mu_m = sum a_t v_t / sum a_t, in fp64.
  c3  E_m = the eigenvectors of C_m as columns, sorted by descending eigenvalue,
      each column's sign making its entry of largest magnitude positive (first
      such entry on ties); U_m = E_m H with H = 2^-3.5 H_128 (Sylvester): the
      pages call the method "a modality-aware correction of the Hadamard
      rotation" (paperpeel section 2.2), and v' = U_m^T v = H (E_m^T v)
      decorrelates the value in its modality's eigenbasis and then spreads the
      variance equally over the coordinates (each gets the mean eigenvalue), as
      the per-token scale and the fixed Gaussian codebook want. Taken alone, the
      eigenbasis concentrates the variance in a few coordinates and quantises
      worse than any of the rotations above (tests/test_oracle_calibration.py).
  c4  a modality without weight keeps the plain Hadamard rotation H; U_m is
      stored fp32, row-major, columns the basis (reading r11: v' = U_m^T v).
"""
from __future__ import annotations

import numpy as np

from .codec import HEAD_DIM, NUM_MODALITIES

F64 = np.float64


def weighted_covariance(v, a):
    """C = sum a_t (v_t - mu)(v_t - mu)^T / sum a_t, mu = sum a_t v_t / sum a_t (c2)."""
    v = np.asarray(v, F64)
    a = np.asarray(a, F64)
    w = a.sum()
    mu = (a[:, None] * v).sum(axis=0) / w
    d = v - mu[None, :]
    return (a[:, None] * d).T @ d / w


def hadamard_normalised():
    """H = 2^-3.5 H_128, H_ij = (-1)^popcount(i & j) (symmetric, orthogonal)."""
    i = np.arange(HEAD_DIM)
    pc = np.array([[bin(x & y).count("1") for y in i] for x in i])
    return np.where(pc % 2 == 0, 1.0, -1.0) * 2.0 ** -3.5


def eigenbasis(C):
    """Eigenvectors of the symmetric C as columns, descending eigenvalues, the sign
    rule of c3. Returns (E [128][128] fp64, eigenvalues descending)."""
    lam, U = np.linalg.eigh(np.asarray(C, F64))
    order = np.argsort(-lam, kind="stable")
    lam, U = lam[order], U[:, order]
    for j in range(U.shape[1]):
        i = int(np.argmax(np.abs(U[:, j])))
        if U[i, j] < 0:
            U[:, j] = -U[:, j]
    return U, lam


def calibrate_bases(v, modality, a):
    """U_m = E_m H for m = 0, 1, 2 from one (layer, kv head)'s calibration values
    (c1-c4). Returns [3][128][128] fp32."""
    v = np.asarray(v, F64)
    modality = np.asarray(modality)
    a = np.asarray(a, F64)
    H = hadamard_normalised()
    out = np.zeros((NUM_MODALITIES, HEAD_DIM, HEAD_DIM), np.float32)
    for m in range(NUM_MODALITIES):
        sel = (modality == m) & (a > 0)
        if not sel.any():
            out[m] = H.astype(np.float32)
            continue
        E, _ = eigenbasis(weighted_covariance(v[sel], a[sel]))
        out[m] = (E @ H).astype(np.float32)
    return out


def value_quant_mse(v_fp16, modality, bases, codebook):
    """Mean squared error per element of the value codec with the given bases (the
    per-token scale and codes of oracle/codec.py): v^ = U_m (sigma16 c_codes).
    v: [T][128] fp16, modality [T], bases [3][128][128]."""
    from . import codec
    v_fp16 = np.asarray(v_fp16, np.float16)
    modality = np.asarray(modality)
    cb = np.asarray(codebook, np.float32).astype(F64)
    err = 0.0
    for m in range(NUM_MODALITIES):
        sel = modality == m
        if not sel.any():
            continue
        codes, sg = codec.encode_values_with_basis(v_fp16[sel], bases[m], codebook)
        vq = (sg.astype(F64)[:, None] * cb[codes]) @ np.asarray(bases[m], np.float32).astype(F64).T
        err += float(((vq - v_fp16[sel].astype(F64)) ** 2).sum())
    return err / v_fp16.size
