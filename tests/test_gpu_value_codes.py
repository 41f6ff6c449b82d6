"""Value codes, pinned exactly: the write's value codes are a function of the
rotated values v' = U_m^T v the kernels compute (tensor cores for windows a write
fills completely, CUDA cores for the rest; paperpeel.com section 2.3), so

  1. the oracle's code decision (z = v' / sigma16 in fp32, code = #{j : z > t_j})
     applied to the GPU's own v' must reproduce the GPU's value codes bit for bit;
  2. the GPU's v' must agree with the exact rotation (fp64) within the a-priori
     error bound of its arithmetic (helpers.rotation_error_bound: U as an fp16
     high + low pair or fp32, times the fp16 value, accumulated in fp32 over 128
     products);
  3. end to end, every value code that differs from the oracle's own (fp64
     rotation) is explained by (2): the oracle's z lies within that bound (over
     sigma16) of the threshold between the two codes. The number of such codes is
     reported.
"""
import numpy as np
import pytest
import torch

from oracle import codec
from synth.workloads import WORKLOADS, key_drift, prefill_inputs, seq_lengths, with_bits

from helpers import make_layer, rotation_error_bound

pytestmark = pytest.mark.gpu


def _gpu_value_codes(records, b, h, pos, bits):
    rec = records[b, h, pos // 32]
    off = codec.record_offsets(bits, bits)
    codes = codec.unpack_value_codes(rec[off["v"]:off["sigma"]].view(np.uint32), bits)
    sig = rec[off["sigma"]:off["sigma"] + 64].view(np.float16)
    return codes[pos % 32], sig[pos % 32]


def _check_write(ocfg, gc, v_new, mod_new, v_rot, L0, bits):
    """Checks 1-3 for the tokens [L0, L0 + n) of every sequence and kv head that
    one write added. Returns (tokens, end-to-end mismatches, max |err| / bound)."""
    B, H, n, _ = v_new.shape
    thr = codec.thresholds(ocfg.value_codebook)
    records = gc.records.cpu().numpy()
    mism, worst, tokens = 0, 0.0, 0
    for b in range(B):
        for h in range(H):
            for i in range(n):
                pos = int(L0[b]) + i
                v = v_new[b, h, i]
                m = min(int(mod_new[b, i]), 2)
                U = ocfg.value_rot[h, m]
                g_codes, g_sig = _gpu_value_codes(records, b, h, pos, bits)
                sig = codec.value_sigma(v[None])[0]
                assert g_sig == sig, "sigma b=%d h=%d pos=%d" % (b, h, pos)
                vp_gpu = v_rot[b, h, i]
                # 1. the oracle's decision on the GPU's v' is the GPU's code, bit for bit
                np.testing.assert_array_equal(codec.value_codes(vp_gpu[None], sig[None], ocfg.value_codebook)[0],
                                              g_codes, err_msg="b=%d h=%d pos=%d" % (b, h, pos))
                # 2. v' against the exact rotation, within the arithmetic's bound
                exact = v.astype(np.float64) @ U.astype(np.float64)
                bound = rotation_error_bound(v, U)
                err = np.abs(vp_gpu.astype(np.float64) - exact)
                assert np.all(err <= bound + 1e-30), "v' b=%d h=%d pos=%d: max err / bound %.3g" % (
                    b, h, pos, float(np.max(err / np.maximum(bound, 1e-30))))
                worst = max(worst, float(np.max(err / np.maximum(bound, 1e-30))))
                # 3. end to end: a differing code has the oracle's z within the bound of (2)
                # (divided by sigma) of the threshold between the two codes
                vp_exact = exact.astype(np.float32)
                o_codes = codec.value_codes(vp_exact[None], sig[None], ocfg.value_codebook)[0]
                for c in np.nonzero(o_codes != g_codes)[0]:
                    lo, hi = sorted((int(o_codes[c]), int(g_codes[c])))
                    assert hi == lo + 1, "non-adjacent codes"
                    z_o = np.float32(vp_exact[c] / np.float32(sig))
                    slack = bound[c] / float(sig) + 2.0 * float(np.spacing(np.abs(z_o)))
                    assert abs(float(z_o) - float(thr[lo])) <= slack, \
                        "code differs away from the threshold (z %r, t %r, slack %.3g)" % (z_o, thr[lo], slack)
                    mism += 1
                tokens += 1
    return tokens, mism, worst


@pytest.mark.parametrize("bits", [2, 4])
def test_value_codes_are_the_decision_on_the_gpu_rotation(cuda_device, bits):
    """Chunked writes (every partial-window path and whole windows on the tensor
    cores) of one 300-token sequence with per-head value bases, then the tiny
    workload's full 2,048-token prefill."""
    import bit_kv_cache_pack_b200 as m
    spec = with_bits(WORKLOADS["tiny"], bits, bits)
    seed = 31
    params, consts, ocfg = make_layer(spec, seed, 0, cuda_device, per_head=True)
    total_tokens, total_mism, worst = 0, 0, 0.0

    L = np.array([300], np.int32)
    drift = key_drift(spec, seed, 0, 16, cuda_device)
    k, v, mod = prefill_inputs(spec, seed, 0, params, drift, L, cuda_device)
    gc = m.KVCache(1, 2, 320, bits, bits, cuda_device)
    cuts = [0, 1, 3, 34, 67, 96, 97, 160, 191, 255, 300]
    for a, b_ in zip(cuts[:-1], cuts[1:]):
        n = b_ - a
        v_rot = torch.empty(1, 2, n, 128, dtype=torch.float32, device=cuda_device)
        L0 = gc.seq_lens.cpu().numpy().copy()
        m.omnikv_write_cache_rotations(consts.struct, gc.struct, k[:, :, a:b_].contiguous(),
                                       v[:, :, a:b_].contiguous(), mod[:, a:b_].contiguous(), n, v_rot)
        torch.cuda.synchronize()
        t, mm, w = _check_write(ocfg, gc, v[:, :, a:b_].cpu().numpy(), mod[:, a:b_].cpu().numpy(),
                                v_rot.cpu().numpy(), L0, bits)
        total_tokens, total_mism, worst = total_tokens + t, total_mism + mm, max(worst, w)

    L = seq_lengths(spec, seed)
    drift = key_drift(spec, seed, 0, 65, cuda_device)
    k, v, mod = prefill_inputs(spec, seed, 0, params, drift, L, cuda_device)
    gc = m.KVCache(1, 2, 2080, bits, bits, cuda_device)
    n = int(L[0])
    v_rot = torch.empty(1, 2, n, 128, dtype=torch.float32, device=cuda_device)
    m.omnikv_write_cache_rotations(consts.struct, gc.struct, k, v, mod, n, v_rot)
    torch.cuda.synchronize()
    t, mm, w = _check_write(ocfg, gc, v.cpu().numpy(), mod.cpu().numpy(), v_rot.cpu().numpy(),
                            np.zeros(1, np.int32), bits)
    total_tokens, total_mism, worst = total_tokens + t, total_mism + mm, max(worst, w)
    assert int(gc.error_word.item()) == 0
    print("value codes (%d bits): %d token-heads, %d codes differ from the fp64 rotation's (all at a "
          "threshold), worst |v' error| / bound = %.3g" % (bits, total_tokens, total_mism, worst))
