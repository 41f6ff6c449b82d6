"""Test helpers: build one layer's constants for both sides and compare the
GPU's packed records with the oracle's."""
from __future__ import annotations

import numpy as np
import torch

from oracle import codec
from synth.workloads import codebook, layer_params

MAX_ABS = 2e-3     # decode output tolerance (absolute)
MAX_REL_L2 = 1e-3  # decode output tolerance (relative L2)
Z_TOL = 5e-5       # value-code disagreement allowed only this close to a threshold


def seeded_randn(shape, device, seed):
    g = torch.Generator(device=device).manual_seed(seed)
    return torch.randn(*shape, device=device, generator=g)


def make_layer(spec, seed, layer, device, per_head=False):
    from bit_kv_cache_pack_b200 import LayerConstants
    params = layer_params(spec, seed, layer, per_head)
    kb, vb = codebook(spec.key_bits), codebook(spec.value_bits)
    consts = LayerConstants(kb, vb, params["key_signs"], params["value_rot"], spec.num_q_heads, device)
    ocfg = codec.OracleConfig(kb, vb, params["key_signs"].numpy(), params["value_rot"].numpy(),
                              spec.num_q_heads, spec.num_kv_heads)
    return params, consts, ocfg


def upload_oracle_cache(oc: codec.OracleCache, device):
    """A GPU KVCache holding exactly the oracle's records (decode parity input)."""
    from bit_kv_cache_pack_b200 import KVCache
    B, H, _, _ = oc.records.shape
    c = KVCache(B, H, oc.cap_tokens, oc.key_bits, oc.value_bits, device)
    c.records.copy_(torch.from_numpy(oc.records))
    c.key_tail.copy_(torch.from_numpy(oc.key_tail))
    c.modality.copy_(torch.from_numpy(oc.modality))
    c.seq_lens.copy_(torch.from_numpy(oc.seq_lens))
    c.struct.max_seq_len = int(oc.seq_lens.max())
    return c


def check_decode(out_gpu: np.ndarray, ref: np.ndarray, where=""):
    out = np.asarray(out_gpu, np.float64)
    err = np.abs(out - ref)
    rel = np.linalg.norm(out - ref) / max(np.linalg.norm(ref), 1e-30)
    assert np.all(np.isfinite(out)), where
    assert err.max() <= MAX_ABS, "%s max abs %.3g" % (where, err.max())
    assert rel <= MAX_REL_L2, "%s rel L2 %.3g" % (where, rel)
    return float(err.max()), float(rel)


def compare_records(ocfg, oc: codec.OracleCache, grec: np.ndarray, b: int, h: int, windows, v_raw, mod_raw):
    """Key codes, metadata and sigma bit-exact; value codes equal except adjacent
    codes whose oracle z = v'/sigma16 lies within Z_TOL of the threshold between
    them. v_raw / mod_raw: fp16 values [T][128] and modality ids [T] of sequence b,
    head h, indexed by position. Returns the number of value-code mismatches."""
    off = oc.off
    thr = codec.thresholds(ocfg.value_codebook)
    mism = 0
    for w in windows:
        o = oc.records[b, h, w]
        g = grec[b, h, w]
        assert np.array_equal(o[off["k"]:off["meta"]], g[off["k"]:off["meta"]]), "key codes w=%d" % w
        assert np.array_equal(o[off["meta"]:off["v"]], g[off["meta"]:off["v"]]), "key meta w=%d" % w
        assert np.array_equal(o[off["sigma"]:], g[off["sigma"]:]), "sigma w=%d" % w
        oc_codes = codec.unpack_value_codes(o[off["v"]:off["sigma"]].view(np.uint32), oc.value_bits)
        g_codes = codec.unpack_value_codes(g[off["v"]:off["sigma"]].view(np.uint32), oc.value_bits)
        bad = np.argwhere(oc_codes != g_codes)
        for t, c in bad:
            pos = w * 32 + t
            d = int(g_codes[t, c]) - int(oc_codes[t, c])
            assert abs(d) == 1, "value code off by %d at pos %d ch %d" % (d, pos, c)
            sg = codec.value_sigma(v_raw[pos][None])[0]
            vp = codec.rotate_values(v_raw[pos][None], ocfg.value_rot[h, mod_raw[pos]])[0]
            z = np.float32(vp[c]) / np.float32(sg)
            tj = thr[min(oc_codes[t, c], g_codes[t, c])]
            assert abs(float(z) - float(tj)) <= Z_TOL * (1 + abs(float(z))), \
                "value code mismatch away from a threshold at pos %d ch %d (z=%r t=%r)" % (pos, c, z, tj)
            mism += 1
    return mism
