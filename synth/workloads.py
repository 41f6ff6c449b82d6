"""Workload recipes: shapes, modality layouts and seeded random tensors.

Five workloads (WORKLOADS) with the shapes of the models the OmniKVQuant pages evaluate
(Qwen2.5-Omni-3B: 36 layers, 16 query / 2 KV heads, head dim 128; Qwen3-Omni-
30B-A3B: 48 layers, 32 / 4 heads), about 10k tokens per minute of audio-visual
input (paperpeel.com section 1), 32-token windows (section 3.1). The pages
measure on real models and benchmarks that are not available here; these
synthetic tensors stand in for them:

keys    k[t][c] = z + d[w(t)][c], z ~ N(0,1), a drift d ~ N(0, drift_std^2) drawn
        per (sequence, head, 32-token window, channel); a few outlier channels per
        (layer, head) are multiplied by outlier_scale. Stored fp16.
values  v[t] = mu_m + sqrt(lam_m) * e, e ~ N(0, I), with a mean mu_m ~ N(0, I) and a
        diagonal variance lam_m log-uniform on [0.1, 10] per (layer, head,
        modality m). Stored fp16.
queries N(0,1) per channel, fp16.
key signs        Rademacher, one vector of 128 per layer.
value bases U_m  Q diag(sign(diag R)) from the QR factorisation of a 128x128 N(0,1)
                 matrix in fp64, stored fp32; one per (layer, modality), replicated
                 over kv heads unless per_head_bases is set.
codebooks        Lloyd-Max levels for N(0,1) from tests/golden/lloyd_max_n01.txt.

Modality ids: 0 = text, 1 = audio, 2 = video. Small parameters are drawn on the
CPU (identical on every machine); the large K/V/Q tensors are drawn on the
device they are requested on.
"""
from __future__ import annotations

import os
import struct
from dataclasses import dataclass, field

import numpy as np
import torch

TEXT, AUDIO, VIDEO = 0, 1, 2
HEAD_DIM = 128
WINDOW = 32
_GOLDEN = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                       "tests", "golden", "lloyd_max_n01.txt")


@dataclass(frozen=True)
class WorkloadSpec:
    name: str
    layers: int
    batch: int
    num_q_heads: int
    num_kv_heads: int
    context: int                 # tokens per sequence before decoding (0: ragged)
    layout: str                  # see modality_layout
    drift_std: float = 0.5
    n_outliers: int = 4
    outlier_scale: float = 8.0
    key_bits: int = 2
    value_bits: int = 2
    decode_steps: int = 1
    ragged: tuple = field(default=())   # (lo, hi) for ragged lengths


WORKLOADS = {
    # 1 layer, batch 1, 2,048 tokens: text 128 | audio 640 | video 1152 | text 128
    "tiny": WorkloadSpec("tiny-1L-b1-16q2kv-ctx2048", 1, 1, 16, 2, 2048, "tavt", decode_steps=1),
    # Qwen2.5-Omni-3B shape, batch 1, 10,240 tokens, 128 one-token decode steps
    "omni3b-b1": WorkloadSpec("qwen2.5-omni-3b-36L-b1-ctx10240", 36, 1, 16, 2, 10240, "interleaved",
                              decode_steps=128),
    # same shape, batch 16, 32,768 tokens per sequence, 64 decode steps
    "omni3b-b16": WorkloadSpec("qwen2.5-omni-3b-36L-b16-ctx32768", 36, 16, 16, 2, 32768, "interleaved",
                               decode_steps=64),
    # Qwen3-Omni-30B-A3B shape, batch 8, 65,536 tokens per sequence, audio-heavy, 32 decode steps
    "omni30b-b8": WorkloadSpec("qwen3-omni-30b-48L-b8-ctx65536", 48, 8, 32, 4, 65536, "audio_heavy",
                               drift_std=1.0, n_outliers=8, outlier_scale=16.0, decode_steps=32),
    # ragged serving mix, batch 64, lengths uniform in [1024, 32768] (never a multiple of 32)
    "ragged-b64": WorkloadSpec("ragged-36L-b64-ctx1024..32768", 36, 64, 16, 2, 0, "mixed",
                               decode_steps=1, ragged=(1024, 32768)),
}


def with_bits(spec: WorkloadSpec, key_bits: int, value_bits: int) -> WorkloadSpec:
    d = dict(spec.__dict__)
    d.update(key_bits=key_bits, value_bits=value_bits, name=spec.name + "-K%dV%d" % (key_bits, value_bits))
    return WorkloadSpec(**d)


# ----------------------------------------------------------------------------
# seeds
# ----------------------------------------------------------------------------
def _mix(*parts) -> int:
    """splitmix64 over the parts -> a 63-bit seed."""
    x = 0x9E3779B97F4A7C15
    for p in parts:
        x = (x + (int(p) & 0xFFFFFFFFFFFFFFFF) + 0x9E3779B97F4A7C15) & 0xFFFFFFFFFFFFFFFF
        z = x
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & 0xFFFFFFFFFFFFFFFF
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & 0xFFFFFFFFFFFFFFFF
        x = z ^ (z >> 31)
    return x & 0x7FFFFFFFFFFFFFFF


def _gen(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_mix(*parts))
    return g


_P_SIGNS, _P_BASIS, _P_OUTL, _P_VSTAT, _P_DRIFT, _P_K, _P_V, _P_Q, _P_LEN, _P_LAYOUT = range(10)


# ----------------------------------------------------------------------------
# codebooks
# ----------------------------------------------------------------------------
def codebook(bits: int) -> np.ndarray:
    """Ascending fp32 levels of the 2^bits-level Lloyd-Max quantiser of N(0,1)."""
    want = 1 << bits
    levels, cur = {}, None
    with open(_GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("levels"):
                cur = int(line.split()[1])
                levels[cur] = []
            else:
                levels[cur].append(struct.unpack("<f", struct.pack("<I", int(line.split()[0], 16)))[0])
    return np.array(levels[want], dtype=np.float32)


# ----------------------------------------------------------------------------
# lengths and modality layouts
# ----------------------------------------------------------------------------
def seq_lengths(spec: WorkloadSpec, seed: int) -> np.ndarray:
    """Context length of every sequence before decoding. Ragged workloads draw
    T_b uniformly from [lo, hi] and redraw any multiple of 32, so every sequence
    ends in a partial window."""
    if not spec.ragged:
        return np.full(spec.batch, spec.context, np.int32)
    rng = np.random.Generator(np.random.PCG64(_mix(seed, _P_LEN)))
    lo, hi = spec.ragged
    out = np.zeros(spec.batch, np.int32)
    for b in range(spec.batch):
        while True:
            t = int(rng.integers(lo, hi + 1))
            if t % WINDOW:
                break
        out[b] = t
    return out


def _fill(T, head_text, tail_text, block):
    """text head, then the block pattern repeated and truncated in order, then text tail."""
    ids = np.zeros(T, np.uint8)
    body = T - head_text - tail_text
    if body < 0:
        raise ValueError("context shorter than its text framing")
    pos = head_text
    while pos < head_text + body:
        for mod, n in block:
            n = min(n, head_text + body - pos)
            ids[pos:pos + n] = mod
            pos += n
            if pos >= head_text + body:
                break
    return ids


def modality_layout(spec: WorkloadSpec, seed: int, b: int, T: int) -> np.ndarray:
    """Modality id of each of the first T positions of sequence b."""
    if spec.layout == "tavt":          # text 128 | audio 640 | video 1152 | text 128
        ids = np.zeros(T, np.uint8)
        ids[128:768] = AUDIO
        ids[768:1920] = VIDEO
        return ids
    if spec.layout == "interleaved":   # text 64, (50 audio + 144 video)*, text 32
        return _fill(T, 64, 32, [(AUDIO, 50), (VIDEO, 144)])
    if spec.layout == "audio_heavy":   # text 256, (100 audio + 64 video)*, text 256
        return _fill(T, 256, 256, [(AUDIO, 100), (VIDEO, 64)])
    if spec.layout == "mixed":         # one of four layouts per sequence
        rng = np.random.Generator(np.random.PCG64(_mix(seed, _P_LAYOUT, b)))
        kind = int(rng.integers(0, 4))
        block = [[(TEXT, 1)], [(AUDIO, 1)], [(VIDEO, 1)], [(AUDIO, 50), (VIDEO, 144)]][kind]
        return _fill(T, 64, 32, block)
    raise ValueError(spec.layout)


# ----------------------------------------------------------------------------
# per-layer parameters (CPU, small)
# ----------------------------------------------------------------------------
def _orthogonal(g: torch.Generator) -> torch.Tensor:
    a = torch.randn(HEAD_DIM, HEAD_DIM, generator=g, dtype=torch.float64)
    q, r = torch.linalg.qr(a)
    return (q * torch.sign(torch.diagonal(r))[None, :]).to(torch.float32)


def layer_params(spec: WorkloadSpec, seed: int, layer: int, per_head_bases: bool = False):
    """key_signs [128] f32 (+-1); value_rot [H_kv][3][128][128] f32; outlier channel
    ids [H_kv][n_out]; value means mu [H_kv][3][128] and variances lam [H_kv][3][128]."""
    H = spec.num_kv_heads
    g = _gen("cpu", seed, _P_SIGNS, layer)
    signs = torch.where(torch.rand(HEAD_DIM, generator=g) < 0.5, -1.0, 1.0).to(torch.float32)
    rot = torch.empty(H, 3, HEAD_DIM, HEAD_DIM, dtype=torch.float32)
    for h in range(H):
        for m in range(3):
            g = _gen("cpu", seed, _P_BASIS, layer, h if per_head_bases else 0, m)
            rot[h, m] = _orthogonal(g)
    outl = torch.empty(H, spec.n_outliers, dtype=torch.int64)
    for h in range(H):
        g = _gen("cpu", seed, _P_OUTL, layer, h)
        outl[h] = torch.randperm(HEAD_DIM, generator=g)[:spec.n_outliers]
    g = _gen("cpu", seed, _P_VSTAT, layer)
    mu = torch.randn(H, 3, HEAD_DIM, generator=g)
    lam = torch.exp(torch.empty(H, 3, HEAD_DIM).uniform_(np.log(0.1), np.log(10.0), generator=g))
    return {"key_signs": signs, "value_rot": rot, "outliers": outl, "mu": mu, "lam": lam}


def key_drift(spec: WorkloadSpec, seed: int, layer: int, cap_windows: int, device) -> torch.Tensor:
    """d [B][H_kv][cap_windows][128] f32 on device."""
    g = _gen(device, seed, _P_DRIFT, layer)
    return spec.drift_std * torch.randn(spec.batch, spec.num_kv_heads, cap_windows, HEAD_DIM,
                                        generator=g, device=device)


def _outlier_scale(spec, params, device):
    sc = torch.ones(spec.num_kv_heads, HEAD_DIM, device=device)
    for h in range(spec.num_kv_heads):
        sc[h, params["outliers"][h].to(device)] = spec.outlier_scale
    return sc


def prefill_inputs(spec: WorkloadSpec, seed: int, layer: int, params, drift, lengths, device,
                   batch_index=None):
    """Prefill K, V [B][H_kv][T_max][128] fp16 and modality [B][T_max] u8 on device.
    Positions >= lengths[b] are zero. batch_index restricts to a subset of sequences."""
    bidx = list(range(spec.batch)) if batch_index is None else list(batch_index)
    T = int(max(lengths[b] for b in bidx))
    H = spec.num_kv_heads
    g = _gen(device, seed, _P_K, layer, bidx[0] if batch_index is not None else -1)
    k = torch.randn(len(bidx), H, T, HEAD_DIM, generator=g, device=device)
    win = torch.arange(T, device=device) // WINDOW
    k += drift[bidx][:, :, win, :]
    k *= _outlier_scale(spec, params, device)[None, :, None, :]
    mod = torch.zeros(len(bidx), T, dtype=torch.uint8)
    for i, b in enumerate(bidx):
        mod[i, :lengths[b]] = torch.from_numpy(modality_layout(spec, seed, b, int(lengths[b])))
    mod = mod.to(device)
    g = _gen(device, seed, _P_V, layer, bidx[0] if batch_index is not None else -1)
    e = torch.randn(len(bidx), H, T, HEAD_DIM, generator=g, device=device)
    mu = params["mu"].to(device)        # [H][3][128]
    sd = params["lam"].to(device).sqrt()
    mi = mod.long()                     # [B][T]
    mu_t = mu[:, mi].permute(1, 0, 2, 3)  # [B][H][T][128]
    sd_t = sd[:, mi].permute(1, 0, 2, 3)
    v = mu_t + sd_t * e
    valid = (torch.arange(T, device=device)[None, :] < torch.as_tensor(
        [int(lengths[b]) for b in bidx], device=device)[:, None])
    k = (k * valid[:, None, :, None]).to(torch.float16).contiguous()
    v = (v * valid[:, None, :, None]).to(torch.float16).contiguous()
    return k, v, mod.contiguous()


def decode_inputs(spec: WorkloadSpec, seed: int, layer: int, step: int, params, drift, positions, device):
    """One decode step: q [B][H_q][128] fp16; the appended text token's k, v
    [B][H_kv][1][128] fp16 (its key drift is that of its window); modality [B][1]."""
    B, H = spec.batch, spec.num_kv_heads
    g = _gen(device, seed, _P_Q, layer, step)
    q = torch.randn(B, spec.num_q_heads, HEAD_DIM, generator=g, device=device).to(torch.float16)
    z = torch.randn(B, H, 1, HEAD_DIM, generator=g, device=device)
    w = torch.as_tensor(np.asarray(positions) // WINDOW, device=device, dtype=torch.long)
    d = drift[torch.arange(B, device=device), :, w, :][:, :, None, :]
    k = ((z + d) * _outlier_scale(spec, params, device)[None, :, None, :]).to(torch.float16)
    e = torch.randn(B, H, 1, HEAD_DIM, generator=g, device=device)
    mu = params["mu"].to(device)[:, TEXT]
    sd = params["lam"].to(device)[:, TEXT].sqrt()
    v = (mu[None, :, None, :] + sd[None, :, None, :] * e).to(torch.float16).contiguous()
    mod = torch.zeros(B, 1, dtype=torch.uint8, device=device)
    return q.contiguous(), k.contiguous(), v, mod
