"""The streaming / captioning cache policy on the GPU (paperpeel.com section 3.1,
"Implementation details": keys quantised every 128 tokens in groups of 32,
values in a 128-token fp16 sliding window) against the oracle
(oracle/attention.py decode_dense_stream: the cache written for every token,
keys before KB = 128 floor(T/128) and values before VB = T - 128 read quantised,
the rest raw).

Each case prefills (per sequence, so lengths differ) and then appends one token at
a time through omnikv_stream_write_cache (records checked against the oracle's),
decoding after every append with omnikv_stream_decode over the oracle's records; the lengths cross the policy's boundaries (a context shorter
than one key block, the first key block, a block boundary with the ring wrapped,
long contexts whose body runs on either decode body), for every key format and
the 4-bit build.
"""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import codec
from oracle.attention import decode_dense_stream
from synth.workloads import WORKLOADS, key_drift, prefill_inputs, with_bits

from helpers import check_decode, compare_records, make_layer, seeded_randn

pytestmark = pytest.mark.gpu

FMT = {"fp16": 0, "mx": 1, "turbo": 2}

CASES = [
    # (bits, key format, prefill lengths, appended steps, explicit splits: 0 = default)
    (2, "fp16", [100, 120], 12, 0),        # < 128 raw, then the first key block and the first quantised values
    (2, "fp16", [250, 253], 6, 0),         # the second key block boundary
    (2, "fp16", [2043, 1500], 3, 0),       # long contexts, the ring wrapped; cooperative body
    (2, "fp16", [2043, 1500], 2, 1),       # one split: the per-warp body
    (2, "mx", [250, 2043], 6, 0),
    (2, "turbo", [250, 2043], 6, 0),
    (4, "fp16", [250, 700], 6, 0),         # the 4-bit build
]


@pytest.mark.parametrize("bits,fmt,lengths,steps,splits", CASES,
                         ids=["first-block", "block-boundary", "long", "long-per-warp", "mx", "turbo", "k4"])
def test_stream_decode_matches_the_oracle(cuda_device, bits, fmt, lengths, steps, splits):
    import bit_kv_cache_pack_b200 as m
    dev = cuda_device
    spec = dataclasses.replace(with_bits(WORKLOADS["tiny"], bits, bits), batch=len(lengths))
    seed = 71 + bits
    params, consts, ocfg = make_layer(spec, seed, 0, dev, key_meta_format=FMT[fmt])
    B, H, Hq = len(lengths), spec.num_kv_heads, spec.num_q_heads
    cap = -(-(max(lengths) + steps) // 32) * 32 + 32
    drift = key_drift(spec, seed, 0, cap // 32, dev)
    cache = m.KVCache(B, H, cap, bits, bits, dev, key_meta_format=FMT[fmt])
    ring_k, ring_v = m.stream_rings(B, H, dev)
    oc = codec.OracleCache(B, H, cap, bits, bits, meta_format=fmt)
    k_all = [[[] for _ in range(H)] for _ in range(B)]
    v_all = [[[] for _ in range(H)] for _ in range(B)]
    for b, n in enumerate(lengths):
        k, v, mod = prefill_inputs(spec, seed, 0, params, drift, np.array(lengths, np.int32), dev, batch_index=[b])
        k, v, mod = k[:, :, :n].contiguous(), v[:, :, :n].contiguous(), mod[:, :n].contiguous()
        view = cache.sequence_view(b)
        m.omnikv_stream_write_cache(consts.struct, view, ring_k[b:b + 1], ring_v[b:b + 1], k, v, mod, n)
        ob = codec.OracleCache(1, H, cap, bits, bits, meta_format=fmt)
        codec.write_cache(ocfg, ob, k.cpu().numpy(), v.cpu().numpy(), mod.cpu().numpy())
        oc.records[b], oc.key_tail[b], oc.modality[b], oc.seq_lens[b] = ob.records[0], ob.key_tail[0], ob.modality[0], n
        for h in range(H):
            k_all[b][h].append(k[0, h].cpu().numpy())
            v_all[b][h].append(v[0, h].cpu().numpy())
    cache.struct.max_seq_len = int(max(lengths))
    for s in range(steps):
        kn = seeded_randn((B, H, 1, 128), dev, 500 + s).half()
        vn = (2.0 * seeded_randn((B, H, 1, 128), dev, 600 + s)).half()
        mn = torch.tensor([[(s + b) % 3] for b in range(B)], dtype=torch.uint8, device=dev)
        q = seeded_randn((B, Hq, 128), dev, 700 + s).half()
        m.omnikv_stream_write_cache(consts.struct, cache.struct, ring_k, ring_v, kn, vn, mn, 1)
        codec.write_cache(ocfg, oc, kn.cpu().numpy(), vn.cpu().numpy(), mn.cpu().numpy())
        for b in range(B):
            for h in range(H):
                k_all[b][h].append(kn[b, h].cpu().numpy())
                v_all[b][h].append(vn[b, h].cpu().numpy())
        # the GPU's records equal the oracle's except value codes at a threshold (the
        # rotation's rounding); the decode is compared over the oracle's records so
        # that such a code in a heavily weighted recent token does not blur the check
        grec = cache.records.cpu().numpy()
        for b in range(B):
            T = int(oc.seq_lens[b])
            vr_b = [np.concatenate(v_all[b][h]) for h in range(H)]
            for h in range(H):
                compare_records(ocfg, oc, grec, b, h, range((T + 31) // 32), vr_b[h], oc.modality[b])
        cache.records.copy_(torch.from_numpy(oc.records))
        S = splits or m.omnikv_default_splits(consts.struct, cache.struct)
        part = m.partials_tensor(B, Hq, S + m._abi.OMNIKV_STREAM_TAIL_SPLITS, dev)
        out = torch.full((B, Hq, 128), float("nan"), device=dev)
        m.omnikv_stream_decode(consts.struct, cache.struct, ring_k, ring_v, q, part, S, out)
        torch.cuda.synchronize()
        assert int(cache.error_word.item()) == 0
        assert np.array_equal(cache.seq_lens.cpu().numpy(), oc.seq_lens)
        kr = [[np.concatenate(k_all[b][h]) for h in range(H)] for b in range(B)]
        vr = [[np.concatenate(v_all[b][h]) for h in range(H)] for b in range(B)]
        ref = decode_dense_stream(ocfg, oc, kr, vr, q.cpu().numpy())
        check_decode(out.cpu().numpy(), ref, "%s bits=%d step %d (lengths %s)" % (fmt, bits, s, list(oc.seq_lens)))
