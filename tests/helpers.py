"""Test helpers: build one layer's constants for both sides and compare the
GPU's packed records with the oracle's."""
from __future__ import annotations

import numpy as np
import torch

from oracle import codec
from synth.workloads import codebook, layer_params

MAX_ABS = 2e-3     # decode output tolerance (absolute)
MAX_REL_L2 = 1e-3  # decode output tolerance (relative L2)
# A value code may differ from the oracle's only where the oracle's z = v'/sigma16
# lies within the a-priori error of the GPU's rotation of a threshold. U is taken
# as fp16 high + low parts (tensor cores; the low part may be subnormal) or fp32
# (CUDA cores), times the exact fp16 value, accumulated in fp32 over 128 products
# (allowing twice round-to-nearest's error per addition, as tensor-core adders need
# not round to nearest):
#   |v'_gpu_c - v'_c| <= (260 u + 2^-22) sum_k |U_kc v_k| + 2^-25 sum_k |v_k|, u = 2^-24.
ROT_ERR = 260 * 2.0 ** -24 + 2.0 ** -22
ROT_ERR_ABS = 2.0 ** -25


def rotation_error_bound(v_fp16, U, c=None):
    """The bound above for channel c (or every channel) of the rotation of one value."""
    v = np.abs(np.asarray(v_fp16, np.float64))
    Ua = np.abs(np.asarray(U, np.float64))
    rel = v @ (Ua[:, c] if c is not None else Ua)
    return ROT_ERR * rel + ROT_ERR_ABS * float(v.sum())


def seeded_randn(shape, device, seed):
    g = torch.Generator(device=device).manual_seed(seed)
    return torch.randn(*shape, device=device, generator=g)


def make_layer(spec, seed, layer, device, per_head=False, key_meta_format=0):
    from bit_kv_cache_pack_b200 import LayerConstants
    params = layer_params(spec, seed, layer, per_head)
    kb, vb = codebook(spec.key_bits), codebook(spec.value_bits)
    consts = LayerConstants(kb, vb, params["key_signs"], params["value_rot"], spec.num_q_heads, device,
                            key_meta_format=key_meta_format)
    ocfg = codec.OracleConfig(kb, vb, params["key_signs"].numpy(), params["value_rot"].numpy(),
                              spec.num_q_heads, spec.num_kv_heads)
    return params, consts, ocfg


def upload_oracle_cache(oc: codec.OracleCache, device):
    """A GPU KVCache holding exactly the oracle's records (decode parity input)."""
    from bit_kv_cache_pack_b200 import KVCache
    B, H, _, _ = oc.records.shape
    c = KVCache(B, H, oc.cap_tokens, oc.key_bits, oc.value_bits, device,
                key_meta_format={"fp16": 0, "mx": 1, "turbo": 2}[oc.meta_format])
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
    codes whose oracle z = v'/sigma16 lies within the rotation's error bound
    (ROT_ERR, over sigma16) of the threshold between them. v_raw / mod_raw: fp16
    values [T][128] and modality ids [T] of sequence b, head h, indexed by
    position. Returns the number of value-code mismatches."""
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
            U = ocfg.value_rot[h, mod_raw[pos]]
            sg = codec.value_sigma(v_raw[pos][None])[0]
            vp = codec.rotate_values(v_raw[pos][None], U)[0]
            z = np.float32(vp[c]) / np.float32(sg)
            tj = thr[min(oc_codes[t, c], g_codes[t, c])]
            slack = float(rotation_error_bound(v_raw[pos], U, c)) / float(sg) + 2.0 * float(np.spacing(np.abs(z)))
            assert abs(float(z) - float(tj)) <= slack, \
                "value code mismatch away from a threshold at pos %d ch %d (z=%r t=%r slack=%.3g)" % (
                    pos, c, z, tj, slack)
            mism += 1
    return mism
