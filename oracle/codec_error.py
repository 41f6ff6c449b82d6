"""Codec-error comparison of KV-cache codecs on synthetic inputs: the analogue of
the pages' error comparison (paperpeel.com section 3.3 "Error comparison", Table 3:
key reconstruction MSE, attention KL divergence, attention-output MSE at a matched
bit rate). TEST INFRASTRUCTURE / ANALYSIS ONLY (see ``oracle/__init__.py``); the
printed values of the pages are for real models and data and are context only.

Codecs (keys; values), every quantiser on the fixed Lloyd-Max codebook:
  omni-fp16 -- OmniKVQuant (oracle/codec.py): sign-flip Hadamard keys with a
               per-channel min-max range per 32-token window, fp16 metadata;
               values rotated by the basis U_m of their modality, per-token scale.
  omni-mx   -- the same with MXFP4 window metadata (oracle/mxmeta.py, its default
               nearest rounding).
  turbo     -- TurboQuant as the pages describe it (pchao.org 关联工作; paperpeel
               section 2.2 "Temporal key drift", section 2.3): one random rotation
               (the same sign-flip Hadamard) for keys and values, and a per-token
               scale sigma = ||x|| / sqrt(128) for both (no windows, no modality
               bases): x^' = sigma16 c_j.
Metrics for one (sequence, kv head) and its query heads, in fp64 and the original
basis (k = R^T k', v = U_m v' or R^T v'):
  recon_mse = mean_{t,c} (k^_tc - k_tc)^2
  attn_kl   = mean_queries KL(p || p^), p = softmax_t(q . k_t / sqrt(128)),
              p^ the same over k^
  out_mse   = mean_{queries,c} (o^_c - o_c)^2, o = sum_t p_t v_t, o^ = sum_t p^_t v^_t
"""
from __future__ import annotations

import numpy as np

from . import codec
from .attention import dequantize, key_rotation_matrix

F64 = np.float64
CODECS = ("omni-fp16", "omni-mx", "turbo")


def _softmax(x):
    x = x - x.max(axis=-1, keepdims=True)
    e = np.exp(x)
    return e / e.sum(axis=-1, keepdims=True)


def kl_divergence(p, q):
    """sum_t p_t log(p_t / q_t) per row (terms with p_t = 0 contribute 0)."""
    p = np.asarray(p, F64)
    q = np.asarray(q, F64)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(p > 0, p * (np.log(p) - np.log(q)), 0.0)
    return t.sum(axis=-1)


def attention_metrics(q, k, v, k_hat, v_hat):
    """(recon_mse, attn_kl, out_mse) of one head group: q [G][128], k, v, k_hat,
    v_hat [T][128] (original basis)."""
    q, k, v, k_hat, v_hat = (np.asarray(x, F64) for x in (q, k, v, k_hat, v_hat))
    scale = 1.0 / np.sqrt(k.shape[1])
    p = _softmax(q @ k.T * scale)
    p_hat = _softmax(q @ k_hat.T * scale)
    o = p @ v
    o_hat = p_hat @ v_hat
    return (float(np.mean((k_hat - k) ** 2)), float(np.mean(kl_divergence(p, p_hat))),
            float(np.mean((o_hat - o) ** 2)))


def omni_dequantized(cfg: codec.OracleConfig, k_fp16, v_fp16, modality, meta_format):
    """OmniKVQuant round trip of one sequence [H][T][128] through the oracle's
    cache: dequantised keys and values in the original basis, [H][T][128]."""
    H, T, _ = k_fp16.shape
    cap = -(-T // codec.WINDOW) * codec.WINDOW
    c = codec.OracleCache(1, H, cap, cfg.key_bits, cfg.value_bits, meta_format=meta_format)
    codec.write_cache(cfg, c, k_fp16[None], v_fp16[None], np.asarray(modality)[None])
    R = key_rotation_matrix(cfg.key_signs)
    ks, vs = [], []
    for h in range(H):
        kq, vq, mod = dequantize(cfg, c, 0, h)
        ks.append(kq @ R)
        vs.append(np.stack([cfg.value_rot[h, mod[t]].astype(F64) @ vq[t] for t in range(T)]))
    return np.stack(ks), np.stack(vs)


def turbo_dequantized(cfg: codec.OracleConfig, x_fp16, bits_codebook):
    """TurboQuant round trip of [T][128] fp16 vectors: Hadamard rotation, per-token
    scale sigma16 (the same pairwise-tree rule as the value scale), codes, back to
    the original basis."""
    xp = codec.rotate_keys(x_fp16, cfg.key_signs)
    sg = codec.value_sigma(x_fp16)
    codes = codec.value_codes(xp, sg, bits_codebook)
    cb = np.asarray(bits_codebook, np.float32).astype(F64)
    xq = sg.astype(F64)[:, None] * cb[codes]
    return xq @ key_rotation_matrix(cfg.key_signs)


def compare(cfg: codec.OracleConfig, k_fp16, v_fp16, modality, q_fp16):
    """Metrics of every codec for one sequence: k, v [H][T][128] fp16, modality [T],
    q [H * G][128] fp16 (query head i reads kv head i // G). Returns
    {codec: (recon_mse, attn_kl, out_mse)}, each the mean over kv heads."""
    H = k_fp16.shape[0]
    G = q_fp16.shape[0] // H
    k = np.asarray(k_fp16, np.float16).astype(F64)
    v = np.asarray(v_fp16, np.float16).astype(F64)
    q = np.asarray(q_fp16, np.float16).astype(F64)
    out = {}
    for name in CODECS:
        if name == "turbo":
            kh = np.stack([turbo_dequantized(cfg, k_fp16[h], cfg.key_codebook) for h in range(H)])
            vh = np.stack([turbo_dequantized(cfg, v_fp16[h], cfg.value_codebook) for h in range(H)])
        else:
            kh, vh = omni_dequantized(cfg, k_fp16, v_fp16, modality, "fp16" if name == "omni-fp16" else "mx")
        per_head = [attention_metrics(q[h * G:(h + 1) * G], k[h], v[h], kh[h], vh[h]) for h in range(H)]
        out[name] = tuple(float(np.mean([m[i] for m in per_head])) for i in range(3))
    return out


def _workload_case(name, bits, tokens, seed=3):
    """One sequence of a workload's synthetic inputs (its shape, key drift and
    outliers, value statistics and modality layout), truncated to `tokens`."""
    import dataclasses

    from synth.workloads import WORKLOADS, codebook, decode_inputs, key_drift, layer_params, prefill_inputs, with_bits
    spec = dataclasses.replace(with_bits(WORKLOADS[name], bits, bits), batch=1)
    params = layer_params(spec, seed, 0)
    cfg = codec.OracleConfig(codebook(bits), codebook(bits), params["key_signs"].numpy(),
                             params["value_rot"].numpy(), spec.num_q_heads, spec.num_kv_heads)
    drift = key_drift(spec, seed, 0, tokens // codec.WINDOW + 1, "cpu")
    k, v, mod = prefill_inputs(spec, seed, 0, params, drift, np.array([tokens]), "cpu")
    q = decode_inputs(spec, seed, 0, 0, params, drift, np.array([tokens]), "cpu")[0]
    return cfg, k[0].numpy(), v[0].numpy(), mod[0].numpy(), q[0].numpy()


if __name__ == "__main__":
    # python -m oracle.codec_error: the comparison on two workload shapes (one
    # sequence of 2,048 tokens each), as recorded in the design notes
    for name in ("omni3b-b16", "omni30b-b8"):
        for bits in (2, 4):
            res = compare(*_workload_case(name, bits, 2048))
            for codec_name, (rm, kl, om) in res.items():
                print("%-11s K%dV%d %-9s recon_mse %.4e  attn_kl %.4e  out_mse %.4e" % (name, bits, bits, codec_name, rm, kl, om))
