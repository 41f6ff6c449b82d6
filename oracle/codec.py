"""Oracle for the OmniKVQuant cache write: keys and values into packed window records.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``). Plain numpy, fp32 where
the encoding takes decisions (so that the integer codes it produces are defined
to the bit), written step by step in the order below. No blocking, fusion or
reordering beyond what each step states.

Method (arXiv:2609.11582; paperpeel.com sections 1, 2.2, 2.3, 3.1, 3.3;
pchao.org "方法概览"):
  keys   -- rotate with the sign-flip Hadamard transform (the TurboQuant rotation
            the method keeps for keys, section 2.2 "Temporal key drift"), then
            take a min-max range per channel over each 32-token group g
            (section 3.1, "32-token groups g"), stored as an fp16 minimum m_gc
            and an fp16 scale s_gc (section 3.3, "Error comparison"), and map each
            coordinate onto the fixed codebook (pchao.org: min-max scaling per
            short window, codebook kept fixed).
  values -- rotate each value with the orthogonal basis U_m of its modality
            m in {V, A, L} (section 2.3, "Modality-aware value rotation"), then
            quantise on the fixed codebook with a per-token scale (reading r6).

Readings where the pages are silent (the same readings the kernels implement):
  r1  affine map of [min, max] onto [c_0, c_{L-1}]:  x_hat = m + s (c_j - c_0),
      s = (max - min) / (c_{L-1} - c_0).
  r3  m and s are rounded to fp16 (round to nearest even) BEFORE codes are
      chosen, so encoder and decoder use the same numbers.
  r4  code = #{ j : z > t_j },  t_j = fp32((c_j + c_{j+1}) * 0.5); a value exactly
      on a midpoint takes the lower index.
  r5  s16 == 0 (constant channel in the window): every code is 0, x_hat = m.
  r6  value scale sigma_t = sqrt(sum_c v_c^2 / 128) over the UNROTATED fp16 value
      (it equals the rotated norm since U_m is orthogonal), summed as a pairwise
      tree x_c <- x_c + x_{c+h} for h = 64, 32, ..., 1; stored fp16;
      z = v'_c / sigma16, same code rule; v_hat' = sigma16 * c_j.
  r7  windows are positions [32w, 32w+32) of each sequence; a partial last
      window is quantised over its valid tokens only and its raw fp16 keys are
      kept in a 32-slot tail so the window can be re-quantised when a token is
      appended. Padded slots hold code 0 and scale 0.
  r8  k' = fp32(2^-3.5) * H_128 (s . k): sign flip first, Sylvester H
      (H_ij = (-1)^popcount(i & j)) applied as butterflies with h = 1, 2, ..., 64,
      each replacing (a, b) = (x_i, x_{i+h}) by (a + b, a - b), in fp32.
  r11 v' = U_m^T v (the columns of U_m are the basis); inverse v = U_m v'.
  r16 modality ids: 0 = text (L), 1 = audio (A), 2 = video (V).

Storage layout of one window record (little-endian), per (sequence, kv head,
window); bits = 2 or 4, cpw = 32 / bits codes per uint32 word:
  K codes  [32 tokens][128 / cpw] u32  token-major: channel c of token t sits in
           word (t, c // cpw), bits [bits * (c % cpw), +bits)
  meta     [128] {fp16 m_gc, fp16 s_gc}
  V codes  [32 / cpw][128] u32         channel-major: token t, channel c sits in
           word (t // cpw, c), bits [bits * (t % cpw), +bits)
  sigma    [32] fp16
Sizes: 1024 + 512 + 1024 + 64 = 2624 B (K2/V2); 2048 + 512 + 2048 + 64 = 4672 B (K4/V4).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

HEAD_DIM = 128
WINDOW = 32
NUM_MODALITIES = 3
F32 = np.float32
F16 = np.float16
INV_SQRT_D_F32 = np.float32(2.0 ** -3.5)  # fp32(1/sqrt(128))


# ----------------------------------------------------------------------------
# record layout
# ----------------------------------------------------------------------------
def codes_per_word(bits: int) -> int:
    return 32 // bits


# key metadata: fp16 (m, s) pairs per window channel, MXFP4 (oracle/mxmeta.py), or the
# TurboQuant key codec ("turbo": one fp16 scale per token, no window statistics)
META_FORMATS = ("fp16", "mx", "turbo")
META_BYTES = {"fp16": HEAD_DIM * 4, "mx": 144, "turbo": WINDOW * 2}


def record_offsets(key_bits: int, value_bits: int, meta_format: str = "fp16"):
    if meta_format not in META_FORMATS:
        raise ValueError(meta_format)
    k_bytes = WINDOW * HEAD_DIM * key_bits // 8
    v_bytes = WINDOW * HEAD_DIM * value_bits // 8
    meta = k_bytes
    v = meta + META_BYTES[meta_format]
    sig = v + v_bytes
    total = sig + WINDOW * 2
    return {"k": 0, "meta": meta, "v": v, "sigma": sig, "total": total,
            "k_bytes": k_bytes, "v_bytes": v_bytes}


def record_bytes(key_bits: int, value_bits: int, meta_format: str = "fp16") -> int:
    return record_offsets(key_bits, value_bits, meta_format)["total"]


# ----------------------------------------------------------------------------
# a1 / a8: sign-flip Hadamard rotation (fp32 butterflies)
# ----------------------------------------------------------------------------
def fwht_f32(x):
    """Unnormalised Walsh-Hadamard transform on the last axis in fp32, butterfly
    stages h = 1, 2, 4, ..., n/2; each stage maps (x_i, x_{i+h}) -> (x_i + x_{i+h},
    x_i - x_{i+h}) for every i with bit h of i clear."""
    x = np.asarray(x, dtype=F32)
    n = x.shape[-1]
    lead = x.shape[:-1]
    h = 1
    while h < n:
        y = x.reshape(lead + (n // (2 * h), 2, h))
        a = y[..., 0, :]
        b = y[..., 1, :]
        x = np.stack([a + b, a - b], axis=-2).reshape(lead + (n,))
        h *= 2
    return x


def rotate_keys(k_fp16, signs):
    """k' = fp32(2^-3.5) * H (s . k) in fp32 (reading r8). k: [..., 128] fp16,
    signs: [128] of +-1."""
    s = np.asarray(signs, dtype=F32)
    x = np.asarray(k_fp16, dtype=F16).astype(F32) * s
    return fwht_f32(x) * INV_SQRT_D_F32


def thresholds(codebook):
    """t_j = fp32((c_j + c_{j+1}) * 0.5) for j = 0..L-2 (reading r4)."""
    c = np.asarray(codebook, dtype=F32)
    return ((c[:-1] + c[1:]) * F32(0.5)).astype(F32)


def count_above(z, thr):
    """code = #{j : z > t_j} (strict; a midpoint goes to the lower level)."""
    z = np.asarray(z, dtype=F32)
    code = np.zeros(z.shape, dtype=np.uint32)
    for t in thr:
        code += (z > t).astype(np.uint32)
    return code


# ----------------------------------------------------------------------------
# a2 / a3: window range and key codes
# ----------------------------------------------------------------------------
def key_window_meta(kp_valid, codebook):
    """Per-channel min and scale of the rotated keys of one window (valid tokens
    only). Returns fp16 (m16, s16), each [128] (readings r1, r3)."""
    kp = np.asarray(kp_valid, dtype=F32)
    c = np.asarray(codebook, dtype=F32)
    mn = kp.min(axis=0)
    mx = kp.max(axis=0)
    span = c[-1] - c[0]
    with np.errstate(over="ignore"):
        s = (mx - mn) / span
    return mn.astype(F16), s.astype(F16)


def key_codes(kp, m16, s16, codebook):
    """z = (k' - m16) / s16 + c_0 in fp32, code = #{j : z > t_j}; s16 == 0 -> 0."""
    kp = np.asarray(kp, dtype=F32)
    c = np.asarray(codebook, dtype=F32)
    m = m16.astype(F32)
    s = s16.astype(F32)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        z = (kp - m) / s + c[0]
    code = count_above(z, thresholds(codebook))
    code = np.where(s == F32(0.0), np.uint32(0), code)
    return code.astype(np.uint32)


# ----------------------------------------------------------------------------
# a5 / a6: value rotation, scale and codes
# ----------------------------------------------------------------------------
def value_sigma(v_fp16):
    """sigma16 = fp16(sqrt(S / 128)) with S the pairwise-tree sum of v_c^2 in fp32
    (reading r6). v: [..., 128] fp16."""
    x = np.asarray(v_fp16, dtype=F16).astype(F32)
    x = x * x  # exact: an fp16 square fits in fp32
    h = HEAD_DIM // 2
    while h >= 1:
        x = x[..., :h] + x[..., h:2 * h]
        h //= 2
    ms = x[..., 0] * F32(1.0 / HEAD_DIM)  # exact power-of-two scaling
    return np.sqrt(ms).astype(F32).astype(F16)


def rotate_values(v_fp16, basis):
    """v' = U^T v, computed in fp64 from the fp16 value and the fp32 basis, then
    rounded once to fp32 (reading r11). v: [n, 128]; basis: [128, 128] (row-major,
    columns are the basis vectors)."""
    v = np.asarray(v_fp16, dtype=F16).astype(np.float64)
    U = np.asarray(basis, dtype=F32).astype(np.float64)
    return (v @ U).astype(F32)


def value_codes(vp, sigma16, codebook):
    """z = v'_c / sigma16 in fp32, code = #{j : z > t_j}; sigma16 == 0 -> 0."""
    vp = np.asarray(vp, dtype=F32)
    sg = np.asarray(sigma16, dtype=F16).astype(F32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        z = vp / sg
    code = count_above(z, thresholds(codebook))
    code = np.where(sg == F32(0.0), np.uint32(0), code)
    return code.astype(np.uint32)


# ----------------------------------------------------------------------------
# a4: packing
# ----------------------------------------------------------------------------
def pack_key_codes(codes, bits):
    """[32][128] codes -> [32][128/cpw] u32, token-major."""
    cpw = codes_per_word(bits)
    c = np.asarray(codes, dtype=np.uint32).reshape(WINDOW, HEAD_DIM // cpw, cpw)
    w = np.zeros((WINDOW, HEAD_DIM // cpw), dtype=np.uint32)
    for i in range(cpw):
        w |= c[:, :, i] << np.uint32(bits * i)
    return w


def pack_value_codes(codes, bits):
    """[32][128] codes -> [32/cpw][128] u32, channel-major."""
    cpw = codes_per_word(bits)
    c = np.asarray(codes, dtype=np.uint32).reshape(WINDOW // cpw, cpw, HEAD_DIM)
    w = np.zeros((WINDOW // cpw, HEAD_DIM), dtype=np.uint32)
    for i in range(cpw):
        w |= c[:, i, :] << np.uint32(bits * i)
    return w


def unpack_key_codes(words, bits):
    """[32][128/cpw] u32 -> [32][128] codes (inverse of pack_key_codes)."""
    cpw = codes_per_word(bits)
    w = np.asarray(words, dtype=np.uint32).reshape(WINDOW, HEAD_DIM // cpw)
    c = np.arange(HEAD_DIM)
    shifts = (bits * (c % cpw)).astype(np.uint32)
    return (w[:, c // cpw] >> shifts[None, :]) & np.uint32((1 << bits) - 1)


def unpack_value_codes(words, bits):
    """[32/cpw][128] u32 -> [32][128] codes (inverse of pack_value_codes)."""
    cpw = codes_per_word(bits)
    w = np.asarray(words, dtype=np.uint32).reshape(WINDOW // cpw, HEAD_DIM)
    t = np.arange(WINDOW)
    shifts = (bits * (t % cpw)).astype(np.uint32)
    return (w[t // cpw, :] >> shifts[:, None]) & np.uint32((1 << bits) - 1)


# ----------------------------------------------------------------------------
# configuration and cache state
# ----------------------------------------------------------------------------
@dataclass
class OracleConfig:
    """Per-layer constants (mirrors the library's configuration)."""
    key_codebook: np.ndarray     # [2^key_bits] fp32, ascending
    value_codebook: np.ndarray   # [2^value_bits] fp32, ascending
    key_signs: np.ndarray        # [128] fp32, each +-1
    value_rot: np.ndarray        # [num_kv_heads][3][128][128] fp32, U_m row-major
    num_q_heads: int
    num_kv_heads: int

    @property
    def key_bits(self) -> int:
        return int(np.log2(len(self.key_codebook)))

    @property
    def value_bits(self) -> int:
        return int(np.log2(len(self.value_codebook)))


class OracleCache:
    """Window records, fp16 key tail, modality ids and lengths of a batch."""

    def __init__(self, batch, num_kv_heads, cap_tokens, key_bits, value_bits, meta_format="fp16"):
        if cap_tokens % WINDOW:
            raise ValueError("cap_tokens must be a multiple of 32")
        self.off = record_offsets(key_bits, value_bits, meta_format)
        self.meta_format = meta_format
        self.key_bits, self.value_bits = key_bits, value_bits
        self.records = np.zeros((batch, num_kv_heads, cap_tokens // WINDOW, self.off["total"]), np.uint8)
        self.key_tail = np.zeros((batch, num_kv_heads, WINDOW, HEAD_DIM), F16)
        self.modality = np.zeros((batch, cap_tokens), np.uint8)
        self.seq_lens = np.zeros(batch, np.int32)
        self.cap_tokens = cap_tokens

    # field views of one record ------------------------------------------------
    def k_words(self, b, h, w):
        o = self.off
        return self.records[b, h, w, o["k"]:o["meta"]].view(np.uint32).reshape(WINDOW, -1)

    def meta(self, b, h, w):
        """fp16 format: the [128] {m16, s16} pairs of the record."""
        o = self.off
        if self.meta_format != "fp16":
            raise ValueError("the record holds MXFP4 metadata")
        return self.records[b, h, w, o["meta"]:o["v"]].view(F16).reshape(HEAD_DIM, 2)

    def key_sigma(self, b, h, w):
        """turbo format: the [32] fp16 key scales of the record's tokens."""
        o = self.off
        if self.meta_format != "turbo":
            raise ValueError("the record holds window metadata")
        return self.records[b, h, w, o["meta"]:o["v"]].view(F16)

    def meta_bytes(self, b, h, w):
        o = self.off
        return self.records[b, h, w, o["meta"]:o["v"]]

    def key_meta_f32(self, b, h, w):
        """The window's decoded minimum and scale per channel, (m, s) fp32 [128]."""
        if self.meta_format == "fp16":
            mt = self.meta(b, h, w)
            return mt[:, 0].astype(F32), mt[:, 1].astype(F32)
        if self.meta_format == "turbo":
            raise ValueError("turbo records have per-token key scales, not window metadata")
        from . import mxmeta
        unpacked = mxmeta.unpack_meta_mx(self.meta_bytes(b, h, w))
        return unpacked[4], unpacked[5]

    def v_words(self, b, h, w):
        o = self.off
        return self.records[b, h, w, o["v"]:o["sigma"]].view(np.uint32).reshape(-1, HEAD_DIM)

    def sigma(self, b, h, w):
        o = self.off
        return self.records[b, h, w, o["sigma"]:o["total"]].view(F16)


# ----------------------------------------------------------------------------
# a1-a7: the cache write
# ----------------------------------------------------------------------------
def quantize_key_window(cfg: OracleConfig, raw_keys_fp16):
    """One window of raw fp16 keys (n_valid <= 32 rows) -> (packed words, m16, s16).
    Padded rows get code 0."""
    n = raw_keys_fp16.shape[0]
    kp = rotate_keys(raw_keys_fp16, cfg.key_signs)
    m16, s16 = key_window_meta(kp, cfg.key_codebook)
    codes = np.zeros((WINDOW, HEAD_DIM), np.uint32)
    codes[:n] = key_codes(kp, m16, s16, cfg.key_codebook)
    return pack_key_codes(codes, cfg.key_bits), m16, s16


def quantize_key_window_mx(cfg: OracleConfig, raw_keys_fp16):
    """The same window with MXFP4 metadata (oracle/mxmeta.py) -> (packed words,
    the 144 metadata bytes)."""
    from . import mxmeta
    n = raw_keys_fp16.shape[0]
    kp = rotate_keys(raw_keys_fp16, cfg.key_signs)
    m_codes, m_exps, s_codes, s_exps, m_hat, s_hat = mxmeta.window_meta_mx(kp, cfg.key_codebook)
    codes = np.zeros((WINDOW, HEAD_DIM), np.uint32)
    codes[:n] = mxmeta.key_codes_mx(kp, m_hat, s_hat, cfg.key_codebook)
    return pack_key_codes(codes, cfg.key_bits), mxmeta.pack_meta_mx(m_codes, m_exps, s_codes, s_exps)


def quantize_key_window_turbo(cfg: OracleConfig, raw_keys_fp16):
    """The TurboQuant key codec on one window of raw fp16 keys (pchao.org 关联工作;
    paperpeel.com section 2.2 "Temporal key drift": one random rotation and a
    per-token scale, no window statistics). Each token on its own: k' = R k (a1),
    sigma16 = fp16(||k|| / sqrt(128)) from the unrotated key (the value scale's
    rule, reading r6), code = #{j : k'_c / sigma16 > t_j} (the value code's rule).
    Returns (packed words, sigma16 [32]); padded rows get code 0 and scale 0."""
    n = raw_keys_fp16.shape[0]
    kp = rotate_keys(raw_keys_fp16, cfg.key_signs)
    sg = np.zeros(WINDOW, F16)
    codes = np.zeros((WINDOW, HEAD_DIM), np.uint32)
    if n:
        sg[:n] = value_sigma(raw_keys_fp16)
        codes[:n] = value_codes(kp, sg[:n], cfg.key_codebook)
    return pack_key_codes(codes, cfg.key_bits), sg


def encode_values_with_basis(v_fp16, basis, codebook):
    """Values of one modality rotated by `basis` -> (codes [n][128], sigma16 [n])."""
    v = np.asarray(v_fp16, dtype=F16)
    sg = value_sigma(v)
    return value_codes(rotate_values(v, basis), sg, codebook), sg


def encode_values(cfg: OracleConfig, head: int, v_fp16, modality):
    """Values of n tokens of one kv head -> (codes [n][128], sigma16 [n])."""
    v = np.asarray(v_fp16, dtype=F16)
    sg = value_sigma(v)
    codes = np.zeros(v.shape, np.uint32)
    for m in range(NUM_MODALITIES):
        sel = np.asarray(modality) == m
        if not sel.any():
            continue
        vp = rotate_values(v[sel], cfg.value_rot[head, m])
        codes[sel] = value_codes(vp, sg[sel], cfg.value_codebook)
    return codes, sg


def write_cache(cfg: OracleConfig, cache: OracleCache, k_new, v_new, modality_new, n_new=None):
    """Append n_new tokens to every sequence of the batch (step a7 for n_new = 1,
    prefill for larger n_new). k_new, v_new: [B][H_kv][n_new][128] fp16;
    modality_new: [B][n_new] u8."""
    k_new = np.asarray(k_new, dtype=F16)
    v_new = np.asarray(v_new, dtype=F16)
    modality_new = np.asarray(modality_new, dtype=np.uint8)
    B, H, n, _ = k_new.shape
    if n_new is not None and n_new != n:
        raise ValueError("n_new does not match k_new")
    vcpw = codes_per_word(cfg.value_bits)
    vmask = np.uint32((1 << cfg.value_bits) - 1)
    for b in range(B):
        L0 = int(cache.seq_lens[b])
        L1 = L0 + n
        if L1 > cache.cap_tokens:
            raise ValueError("capacity exceeded")
        cache.modality[b, L0:L1] = modality_new[b]
        for h in range(H):
            # keys: every window touched by [L0, L1)
            for w in range(L0 // WINDOW, (L1 - 1) // WINDOW + 1):
                p0, p1 = w * WINDOW, min(w * WINDOW + WINDOW, L1)
                raw = np.zeros((p1 - p0, HEAD_DIM), F16)
                for p in range(p0, p1):
                    raw[p - p0] = cache.key_tail[b, h, p - p0] if p < L0 else k_new[b, h, p - L0]
                if cache.meta_format == "fp16":
                    words, m16, s16 = quantize_key_window(cfg, raw)
                    meta = cache.meta(b, h, w)
                    meta[:, 0] = m16
                    meta[:, 1] = s16
                elif cache.meta_format == "turbo":
                    words, ksg = quantize_key_window_turbo(cfg, raw)
                    cache.key_sigma(b, h, w)[:] = ksg
                else:
                    words, mbytes = quantize_key_window_mx(cfg, raw)
                    cache.meta_bytes(b, h, w)[:] = mbytes
                cache.k_words(b, h, w)[:] = words
                if p1 - p0 < WINDOW:  # partial window: keep its raw keys
                    cache.key_tail[b, h, :p1 - p0] = raw
            # values: per token
            codes, sg = encode_values(cfg, h, v_new[b, h], modality_new[b])
            for i in range(n):
                p = L0 + i
                w, t = divmod(p, WINDOW)
                vw = cache.v_words(b, h, w)
                sh = np.uint32(cfg.value_bits * (t % vcpw))
                col = vw[t // vcpw]
                col &= ~(vmask << sh)
                col |= codes[i].astype(np.uint32) << sh
                cache.sigma(b, h, w)[t] = sg[i]
        cache.seq_lens[b] = L1
