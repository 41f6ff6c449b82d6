"""Oracle for MXFP4 key metadata, the pages' default metadata format for the key
window ranges. TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

paperpeel.com section 3.1 ("Implementation details"): keys use 32-token groups
for the range estimate "with MXFP4 metadata by default"; section 3.3 ("Error
comparison"): the fp16 minimum and scale variant (``oracle/codec.py``) costs one
bit per element. The pages give nothing more, so this module takes the plainest
reading of "MXFP4" (the microscaling FP4 format: E2M1 elements sharing one
power-of-two E8M0 scale per block of 32) and states each choice:

  x1  elements: E2M1 -- sign, 2 exponent bits, 1 mantissa bit; magnitudes
      0, 0.5, 1, 1.5, 2, 3, 4, 6. Code = (sign << 3) | index of the magnitude.
      A zero is stored as +0 (code 0).
  x2  blocks run along the channels: channels 32 b .. 32 b + 31 of one window
      share one exponent; the minima and the scales have their own blocks
      (4 + 4 exponents per window of 128 channels).
  x3  the shared exponent e (stored as the E8M0 byte e + 127) is the smallest
      integer in [-127, 127] with max_c |x_c| <= 6 * 2^e over the block, so no
      element saturates; an all-zero block takes e = -127.
  x4  rounding on the grid {+-magnitude * 2^e}: the minimum first (from the fp32
      minimum), then the scale that minimum needs, s_req = fp32(fp32(max - m^) /
      (c_{L-1} - c_0)) (0 if negative). Default ("nearest", the MX conversion rule):
      both round to the nearest grid value, ties to the even code; keys outside
      [m^, m^ + s^ (c_{L-1} - c_0)] take the end codes. Option ("cover"): the
      minimum rounds toward -inf and the scale toward +inf, so the range covers
      every key of the channel. On the workloads' synthetic keys with 2-bit codes
      the covering option roughly doubles the errors of the fp16 format while the
      nearest one stays within ~10 % of it (oracle/codec_error.py; with 4-bit codes
      the covering one is the closer), and the pages report MXFP4 as their accurate
      default at the 2-bit budget, hence the default.
  x5  codes as in the fp16 format with (m^, s^) in place of (m16, s16):
      z = (k' - m^) / s^ + c_0 in fp32, code = #{j : z > t_j}; s^ == 0 -> 0;
      reconstruction k^' = m^ + s^ (c_j - c_0).
  x6  metadata bytes of a window (144 B, a multiple of 16 so records stay
      16-byte aligned): [m elements: 64 B, channel c in byte c // 2, low nibble
      for even c][s elements: 64 B, same order][m exponents: 4 B, block b at
      byte b][s exponents: 4 B][8 zero bytes]. A K2/V2 record is then
      1024 + 144 + 1024 + 64 = 2256 B (70.5 B per token and kv head instead of 82).
"""
from __future__ import annotations

import numpy as np

from .codec import HEAD_DIM, WINDOW, count_above, thresholds

F32 = np.float32
F64 = np.float64

E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)   # x1
E2M1_MAX = 6.0
BLOCK = 32                                                     # x2
BLOCKS = HEAD_DIM // BLOCK
EXP_MIN, EXP_MAX = -127, 127                                   # x3
META_BYTES = 144                                               # x6


def e2m1_decode(code):
    """E2M1 code(s) -> value (fp64): (-1)^(code >> 3) * magnitude[code & 7] (x1)."""
    code = np.asarray(code, dtype=np.int64)
    mag = np.asarray(E2M1_MAGNITUDES, dtype=F64)[code & 7]
    return np.where((code >> 3) & 1, -mag, mag)


def block_exponent(x_block):
    """Smallest e in [-127, 127] with max |x| <= 6 * 2^e; -127 for an all-zero
    block (x3). x_block: fp32 values."""
    amax = float(np.max(np.abs(np.asarray(x_block, dtype=F64))))
    if amax == 0.0:
        return EXP_MIN
    e = EXP_MIN
    while e < EXP_MAX and E2M1_MAX * 2.0 ** e < amax:
        e += 1
    return e


def _signed_grid():
    g = sorted(set([m for m in E2M1_MAGNITUDES] + [-m for m in E2M1_MAGNITUDES]))
    return np.asarray(g, dtype=F64)   # -6 .. 6, one zero


def _code_of(value):
    """E2M1 code of a grid value (+0 for zero)."""
    mag = abs(value)
    idx = E2M1_MAGNITUDES.index(mag)
    return (8 if value < 0 else 0) | idx


def round_down(x, e):
    """Largest grid value g * 2^e <= x (x4, for the minimum). Returns (code, value)."""
    q = float(x) / 2.0 ** e          # exact: scaling by a power of two
    grid = _signed_grid()
    below = grid[grid <= q]
    g = float(below.max())
    return _code_of(g), g * 2.0 ** e


def round_nearest(x, e):
    """Nearest grid value g * 2^e to x, ties to the even code (x4, default).
    Returns (code, value)."""
    q = float(x) / 2.0 ** e
    grid = _signed_grid()
    d = np.abs(grid - q)
    best = np.flatnonzero(d == d.min())
    if len(best) > 1:   # a tie between two neighbours: the even code
        best = [i for i in best if _code_of(float(grid[i])) % 2 == 0]
    g = float(grid[best[0]])
    return _code_of(g), g * 2.0 ** e


def round_up(x, e):
    """Smallest grid value g * 2^e >= x (x4, for the scale). Returns (code, value)."""
    q = float(x) / 2.0 ** e
    grid = _signed_grid()
    above = grid[grid >= q]
    g = float(above.min())
    return _code_of(g), g * 2.0 ** e


def window_meta_mx(kp_valid, codebook, rounding="nearest"):
    """MXFP4 metadata of one window from its rotated fp32 keys (valid tokens only):
    per channel the minimum, then the scale it needs, each rounded on its block's
    grid (x3, x4; rounding "nearest" or "cover"). Returns (m_codes [128], m_exps [4],
    s_codes [128], s_exps [4], m_hat [128], s_hat [128]); m_hat and s_hat are exact
    in fp32."""
    if rounding not in ("nearest", "cover"):
        raise ValueError(rounding)
    rnd_m = round_nearest if rounding == "nearest" else round_down
    rnd_s = round_nearest if rounding == "nearest" else round_up
    kp = np.asarray(kp_valid, dtype=F32)
    c = np.asarray(codebook, dtype=F32)
    mn = kp.min(axis=0)
    mx = kp.max(axis=0)
    span = c[-1] - c[0]
    m_codes = np.zeros(HEAD_DIM, np.uint8)
    s_codes = np.zeros(HEAD_DIM, np.uint8)
    m_hat = np.zeros(HEAD_DIM, F64)
    s_hat = np.zeros(HEAD_DIM, F64)
    m_exps = np.zeros(BLOCKS, np.int32)
    s_exps = np.zeros(BLOCKS, np.int32)
    for b in range(BLOCKS):
        ch = slice(BLOCK * b, BLOCK * (b + 1))
        e = block_exponent(mn[ch])
        m_exps[b] = e
        for cc in range(BLOCK * b, BLOCK * (b + 1)):
            m_codes[cc], m_hat[cc] = rnd_m(mn[cc], e)
    # the scale each channel needs with its rounded minimum, in fp32
    with np.errstate(over="ignore"):
        s_req = ((mx - m_hat.astype(F32)) / span).astype(F32)
    s_req = np.maximum(s_req, F32(0.0))   # a minimum rounded above the maximum: no range
    for b in range(BLOCKS):
        ch = slice(BLOCK * b, BLOCK * (b + 1))
        e = block_exponent(s_req[ch])
        s_exps[b] = e
        for cc in range(BLOCK * b, BLOCK * (b + 1)):
            s_codes[cc], s_hat[cc] = rnd_s(s_req[cc], e)
    return m_codes, m_exps, s_codes, s_exps, m_hat.astype(F32), s_hat.astype(F32)


def key_codes_mx(kp, m_hat, s_hat, codebook):
    """z = (k' - m^) / s^ + c_0 in fp32, code = #{j : z > t_j}; s^ == 0 -> 0 (x5)."""
    kp = np.asarray(kp, dtype=F32)
    c = np.asarray(codebook, dtype=F32)
    m = np.asarray(m_hat, dtype=F32)
    s = np.asarray(s_hat, dtype=F32)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        z = (kp - m) / s + c[0]
    code = count_above(z, thresholds(codebook))
    return np.where(s == F32(0.0), np.uint32(0), code).astype(np.uint32)


def dequantize_keys_mx(codes, m_hat, s_hat, codebook):
    """k^' = m^ + s^ (c_j - c_0) in fp64 (x5)."""
    c = np.asarray(codebook, dtype=F32).astype(F64)
    return (np.asarray(m_hat, F64)[None, :]
            + np.asarray(s_hat, F64)[None, :] * (c[np.asarray(codes)] - c[0]))


def pack_meta_mx(m_codes, m_exps, s_codes, s_exps):
    """The 144 metadata bytes of a window (x6)."""
    out = np.zeros(META_BYTES, np.uint8)
    mc = np.asarray(m_codes, np.uint8)
    sc = np.asarray(s_codes, np.uint8)
    out[0:64] = mc[0::2] | (mc[1::2] << 4)
    out[64:128] = sc[0::2] | (sc[1::2] << 4)
    out[128:132] = (np.asarray(m_exps, np.int32) + 127).astype(np.uint8)
    out[132:136] = (np.asarray(s_exps, np.int32) + 127).astype(np.uint8)
    return out


def unpack_meta_mx(meta):
    """Inverse of pack_meta_mx: (m_codes, m_exps, s_codes, s_exps, m_hat, s_hat)."""
    meta = np.asarray(meta, np.uint8)
    m_codes = np.zeros(HEAD_DIM, np.uint8)
    s_codes = np.zeros(HEAD_DIM, np.uint8)
    m_codes[0::2], m_codes[1::2] = meta[0:64] & 15, meta[0:64] >> 4
    s_codes[0::2], s_codes[1::2] = meta[64:128] & 15, meta[64:128] >> 4
    m_exps = meta[128:132].astype(np.int32) - 127
    s_exps = meta[132:136].astype(np.int32) - 127
    blk = np.arange(HEAD_DIM) // BLOCK
    m_hat = (e2m1_decode(m_codes) * np.exp2(m_exps[blk].astype(F64))).astype(F32)
    s_hat = (e2m1_decode(s_codes) * np.exp2(s_exps[blk].astype(F64))).astype(F32)
    return m_codes, m_exps, s_codes, s_exps, m_hat, s_hat


def record_bytes_mx(key_bits: int, value_bits: int) -> int:
    """Window record with MXFP4 key metadata: key codes, 144 B metadata, value
    codes, 32 fp16 value scales (x6)."""
    return WINDOW * HEAD_DIM * key_bits // 8 + META_BYTES + WINDOW * HEAD_DIM * value_bits // 8 + 2 * WINDOW
