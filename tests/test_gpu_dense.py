"""The dense bf16 decode kernel (the comparison baseline for the packed cache)
against a plain fp32 PyTorch reference of the same attention. bf16 rounding of
the scaled query and of the probabilities bounds the agreement at about 1e-2."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _reference(k, v, q, lens, G):
    B, H, _, D = k.shape
    out = torch.zeros(B, H * G, D, dtype=torch.float64)
    for b in range(B):
        T = int(lens[b])
        if T == 0:
            continue
        for i in range(H * G):
            h = i // G
            kk = k[b, h, :T].double().cpu()
            vv = v[b, h, :T].double().cpu()
            s = (kk @ q[b, i].double().cpu()) / np.sqrt(D)
            out[b, i] = torch.softmax(s, 0) @ vv
    return out.numpy()


@pytest.mark.parametrize("S", [0, 1, 3, 17])
def test_dense_bf16_decode(cuda_device, S):
    import bit_kv_cache_pack_b200 as m
    g = torch.Generator(device=cuda_device).manual_seed(5)
    B, H, G, cap = 3, 2, 8, 1024
    lens = torch.tensor([1000, 37, 0], dtype=torch.int32, device=cuda_device)
    k = torch.randn(B, H, cap, 128, generator=g, device=cuda_device).to(torch.bfloat16)
    v = (1.5 * torch.randn(B, H, cap, 128, generator=g, device=cuda_device) + 0.5).to(torch.bfloat16)
    q = torch.randn(B, H * G, 128, generator=g, device=cuda_device).to(torch.bfloat16)
    Sr = S or 4
    part = torch.empty(m.omnikv_dense_partials_bytes(B, H * G, max(S, 64)) // 4, device=cuda_device)
    out = torch.full((B, H * G, 128), float("nan"), device=cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    m.omnikv_dense_decode_bf16(k, v, lens, B, H * G, H, cap, 1000, q, part, S, out, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = _reference(k, v, q, lens.cpu().numpy(), G)
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(got[2] == 0)
    assert np.abs(got - ref).max() < 5e-2
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-2
