"""GPU parity at the full sizes of every workload (one layer each), in the
launch configuration the benchmark uses (default split count).

For each workload: prefill every sequence through omnikv_write_cache, append
one text token per sequence, then
  * for sampled sequences, the oracle encodes the same inputs and the GPU's
    window records are compared with it: key codes, window metadata and value
    scales bit-exact, value codes equal except adjacent codes at a threshold;
  * the sampled sequences' GPU records are replaced by the oracle's, the batch is
    decoded on the GPU (decode + combine), and the sampled outputs are compared
    with the oracle's fp64 attention over that same cache (max abs <= 2e-3, rel
    L2 <= 1e-3); the other sequences must be finite.
"""
import numpy as np
import pytest
import torch

from oracle import codec
from oracle.attention import decode_dense
from synth.workloads import WORKLOADS, decode_inputs, key_drift, prefill_inputs, seq_lengths, with_bits

from helpers import check_decode, compare_records, make_layer

pytestmark = pytest.mark.gpu

CASES = [
    ("omni3b-b1", 2, 1),
    ("omni3b-b16", 2, 16),
    ("omni3b-b16", 4, 16),
    ("omni30b-b8", 2, 30),
    ("ragged-b64", 2, 64),
]


@pytest.mark.parametrize("name,bits,seed", CASES, ids=["%s-K%d" % (c[0], c[1]) for c in CASES])
def test_full_size_layer(cuda_device, name, bits, seed):
    import bit_kv_cache_pack_b200 as m
    spec = with_bits(WORKLOADS[name], bits, bits)
    dev = cuda_device
    B, H = spec.batch, spec.num_kv_heads
    params, consts, ocfg = make_layer(spec, seed, 0, dev)
    L = seq_lengths(spec, seed)
    cap = int(-(-(int(L.max()) + 1) // 32) * 32)
    drift = key_drift(spec, seed, 0, cap // 32, dev)
    gc = m.KVCache(B, H, cap, bits, bits, dev)
    samples = [B - 1] if not spec.ragged else [int(np.argmin(L)), int(np.argmax(L))]

    # ---- prefill, exactly as the benchmark writes it
    kept = {}
    if spec.ragged:
        for b in range(B):
            k, v, mod = prefill_inputs(spec, seed, 0, params, drift, L, dev, batch_index=[b])
            n = int(L[b])
            k, v, mod = k[:, :, :n].contiguous(), v[:, :, :n].contiguous(), mod[:, :n].contiguous()
            m.omnikv_write_cache(consts.struct, gc.sequence_view(b), k, v, mod, n)
            if b in samples:
                kept[b] = (k[0].cpu().numpy(), v[0].cpu().numpy(), mod[0].cpu().numpy())
            del k, v, mod
        gc.struct.max_seq_len = int(L.max())
    else:
        k, v, mod = prefill_inputs(spec, seed, 0, params, drift, L, dev)
        m.omnikv_write_cache(consts.struct, gc.struct, k, v, mod, int(L[0]))
        for b in samples:
            kept[b] = (k[b].cpu().numpy(), v[b].cpu().numpy(), mod[b].cpu().numpy())
        del k, v, mod
    q, kn, vn, mn = decode_inputs(spec, seed, 0, 0, params, drift, L, dev)
    m.omnikv_write_cache(consts.struct, gc.struct, kn, vn, mn, 1)
    torch.cuda.synchronize()
    assert int(gc.error_word.item()) == 0
    assert np.array_equal(gc.seq_lens.cpu().numpy(), L + 1)

    # ---- sampled sequences: oracle encode, compare records, substitute
    oracles = {}
    grec = {b: gc.records[b].cpu().numpy()[None] for b in samples}
    for b in samples:
        kb, vb, modb = kept[b]
        oc = codec.OracleCache(1, H, cap, bits, bits)
        codec.write_cache(ocfg, oc, kb[None], vb[None], modb[None])
        codec.write_cache(ocfg, oc, kn[b:b + 1].cpu().numpy(), vn[b:b + 1].cpu().numpy(), mn[b:b + 1].cpu().numpy())
        T = int(L[b]) + 1
        nw = (T + 31) // 32
        v_all = np.concatenate([vb, vn[b].cpu().numpy()], axis=1)       # [H][T][128]
        mod_all = np.concatenate([modb, mn[b].cpu().numpy()])
        assert np.array_equal(gc.modality[b, :T].cpu().numpy(), mod_all)
        mism = 0
        for h in range(H):
            mism += compare_records(ocfg, oc, grec[b], 0, h, range(nw), v_all[h], mod_all)
        assert mism <= 1e-4 * v_all.size, "too many value-code disagreements: %d" % mism
        r = T % 32
        if r:
            assert np.array_equal(gc.key_tail[b, :, :r].cpu().numpy(), oc.key_tail[0, :, :r])
        gc.records[b].copy_(torch.from_numpy(oc.records[0]))
        oracles[b] = oc

    # ---- decode the whole batch with the default split count
    S = m.omnikv_default_splits(consts.struct, gc.struct)
    part = m.partials_tensor(B, spec.num_q_heads, S, dev)
    out = torch.empty(B, spec.num_q_heads, 128, dtype=torch.float32, device=dev)
    m.omnikv_decode_attention(consts.struct, gc.struct, q, part, S)
    m.omnikv_combine(consts.struct, gc.struct, part, S, out)
    torch.cuda.synchronize()
    assert int(gc.error_word.item()) == 0
    out = out.cpu().numpy()
    assert np.all(np.isfinite(out))
    for b in samples:
        ref = decode_dense(ocfg, oracles[b], q[b:b + 1].cpu().numpy())
        check_decode(out[b:b + 1], ref, "%s b=%d" % (spec.name, b))
