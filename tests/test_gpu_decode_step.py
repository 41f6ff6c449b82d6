"""The fused decode step (omnikv_decode_step: one-token append inside the decode
launch, length advanced by the combine) against the same step done as four
calls (omnikv_write_cache + omnikv_decode_attention + omnikv_combine) on an
identical cache, and against the oracle.

Both paths of the step are covered: the fused launch (the whole grid resident)
and the fallback that an explicit, too large split count forces. The cache state
after every step (records, key tail, modality ids, lengths) must equal the
four-call cache byte for byte, and the outputs must be identical (the decode CTAs
run the same code on the same bytes); the final outputs are also checked
against the oracle's fp64 attention over its own cache (the decode tolerance).
"""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import codec
from oracle.attention import decode_dense
from synth.workloads import WORKLOADS, key_drift, prefill_inputs, with_bits

from helpers import check_decode, make_layer, seeded_randn

pytestmark = pytest.mark.gpu


def _prefill(m, consts, cache, spec, params, drift, lengths, dev, seed):
    """Per-sequence prefill (lengths may differ) through sequence views."""
    kept = []
    H = spec.num_kv_heads
    for b, n in enumerate(lengths):
        if n == 0:
            kept.append((np.zeros((H, 0, 128), np.float16), np.zeros((H, 0, 128), np.float16), np.zeros(0, np.uint8)))
            continue
        k, v, mod = prefill_inputs(spec, seed, 0, params, drift, np.array(lengths, np.int32), dev, batch_index=[b])
        k, v, mod = k[:, :, :n].contiguous(), v[:, :, :n].contiguous(), mod[:, :n].contiguous()
        m.omnikv_write_cache(consts.struct, cache.sequence_view(b), k, v, mod, n)
        kept.append((k[0].cpu().numpy(), v[0].cpu().numpy(), mod[0].cpu().numpy()))
    cache.struct.max_seq_len = int(max(lengths))
    return kept


CASES = [
    # (kv heads, group, lengths, steps, explicit splits: 0 = default (fused), bits)
    (2, 8, [93], 5, 0, 2),                 # crosses the window boundary at 96
    (2, 8, [31, 64, 0], 3, 0, 2),           # a full window, a fresh window, an empty sequence
    (4, 8, [200, 17], 4, 0, 2),             # 4 kv heads, 32 query heads
    (2, 8, [93, 40], 4, 200, 2),            # 2 x (1 + 200) CTAs: beyond residency -> four-call fallback
    (2, 8, [93, 250], 4, 0, 4),             # K4V4: the table body with the fused append
    (2, 8, [700], 3, 1, 2),                 # one split of 22 windows: the per-warp body in the fused launch
    # 16 x 2 units x 9 per-warp splits = 288 decode CTAs: the 8 append CTAs left
    # in a 296-CTA wave append for 4 (sequence, kv head) units each
    (2, 8, [4700 + 13 * i for i in range(16)], 2, 0, 2),
    (2, 8, [700, 333], 3, 1, 4),            # K4V4, one split per (sequence, kv head): long table-body splits
    (2, 8, [2300 + 13 * i for i in range(16)], 2, 0, 4),  # K4V4 with shared append CTAs (2 CTAs per SM)
    (2, 8, [93, 40], 4, 200, 4),            # K4V4 beyond residency -> four-call fallback
]


@pytest.mark.parametrize("hkv,G,lengths,steps,splits,bits", CASES,
                         ids=["b1-boundary", "ragged-b3", "h4", "fallback", "k4", "per-warp", "shared-append-ctas",
                              "k4-one-split", "k4-shared-append-ctas", "k4-fallback"])
def test_decode_step_matches_four_calls_and_oracle(cuda_device, hkv, G, lengths, steps, splits, bits):
    import bit_kv_cache_pack_b200 as m
    dev = cuda_device
    seed = 21 + hkv + len(lengths)
    spec = dataclasses.replace(with_bits(WORKLOADS["tiny"], bits, bits), num_kv_heads=hkv, num_q_heads=hkv * G,
                               batch=len(lengths))
    params, consts, ocfg = make_layer(spec, seed, 0, dev)
    B = len(lengths)
    cap = max(320, -(-(max(lengths) + steps) // 32) * 32)
    drift = key_drift(spec, seed, 0, cap // 32, dev)
    fused = m.KVCache(B, hkv, cap, bits, bits, dev)
    plain = m.KVCache(B, hkv, cap, bits, bits, dev)
    kept = _prefill(m, consts, fused, spec, params, drift, lengths, dev, seed)
    _prefill(m, consts, plain, spec, params, drift, lengths, dev, seed)
    torch.cuda.synchronize()

    Hq = hkv * G
    S_alloc = max(splits, 64)
    part_f = m.partials_tensor(B, Hq, S_alloc, dev)
    part_p = m.partials_tensor(B, Hq, S_alloc, dev)
    newk, newv, newm = [], [], []
    for s in range(steps):
        q = seeded_randn((B, Hq, 128), dev, 100 + s).half()
        kn = seeded_randn((B, hkv, 1, 128), dev, 200 + s).half()
        vn = (2.0 * seeded_randn((B, hkv, 1, 128), dev, 300 + s)).half()
        mn = torch.tensor([(s + b) % 3 for b in range(B)], dtype=torch.uint8, device=dev)
        out_f = torch.full((B, Hq, 128), float("nan"), device=dev)
        out_p = torch.full((B, Hq, 128), float("nan"), device=dev)
        if s % 2:  # the same step as its two launches
            m.omnikv_append_decode(consts.struct, fused.struct, q, kn, vn, mn, part_f, splits)
            m.omnikv_combine_step(consts.struct, fused.struct, part_f, splits, out_f)
        else:
            m.omnikv_decode_step(consts.struct, fused.struct, q, kn, vn, mn, part_f, splits, out_f)
        m.omnikv_write_cache(consts.struct, plain.struct, kn, vn, mn, 1)
        Sp = splits or m.omnikv_default_splits(consts.struct, plain.struct)
        m.omnikv_decode_attention(consts.struct, plain.struct, q, part_p, Sp)
        m.omnikv_combine(consts.struct, plain.struct, part_p, Sp, out_p)
        torch.cuda.synchronize()
        assert int(fused.error_word.item()) == 0 and int(plain.error_word.item()) == 0
        assert fused.max_seq_len == plain.max_seq_len
        assert torch.equal(fused.seq_lens, plain.seq_lens)
        assert torch.equal(fused.records, plain.records)
        assert torch.equal(fused.key_tail, plain.key_tail)
        assert torch.equal(fused.modality, plain.modality)
        of, op = out_f.cpu().numpy(), out_p.cpu().numpy()
        assert np.all(np.isfinite(of))
        np.testing.assert_array_equal(of, op)  # the same decode code over the same bytes and splits
        newk.append(kn.cpu().numpy()), newv.append(vn.cpu().numpy()), newm.append(mn.cpu().numpy())
    assert np.array_equal(fused.seq_lens.cpu().numpy(), np.array(lengths) + steps)

    assert int(fused.struct.max_seq_len) == max(lengths) + steps
    # the oracle, writing the same prefill and appends, decodes the last step's query
    ref_all = []
    for b in range(B):
        oc = codec.OracleCache(1, hkv, cap, bits, bits)
        kb, vb, mb = kept[b]
        if lengths[b]:
            codec.write_cache(ocfg, oc, kb[None], vb[None], mb[None])
        for s in range(steps):
            codec.write_cache(ocfg, oc, newk[s][b:b + 1], newv[s][b:b + 1], newm[s][b:b + 1, None])
        ref_all.append(decode_dense(ocfg, oc, q[b:b + 1].cpu().numpy()))
    check_decode(of, np.concatenate(ref_all), "fused step")
