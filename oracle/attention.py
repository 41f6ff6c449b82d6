"""Oracle for decode attention over the packed OmniKVQuant cache, in fp64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The method attends over the quantised cache exactly (the fused kernel of
paperpeel.com section 1 changes where the rotations are applied, not what is
computed), so the reference is plain softmax attention over the dequantised
cache. It is written two ways that must agree:

``decode_dense``  -- the definition: dequantise every cached token back to the
    ORIGINAL basis (k = R^T k_hat', v = U_m v_hat') and run textbook softmax
    attention with the unrotated query, scale 1/sqrt(128) (reading r14).
``decode_fused``  -- the fused kernel's order (paperpeel.com section 1: rotate
    one query per head instead of inverse-rotating every key, FlashAttention
    order [refs 4, 5], inverse value rotations batched across head outputs):
    q' = R q; the context is split into contiguous runs of windows; each run
    keeps a running max, a running sum and one rotated-space accumulator per
    modality; runs are merged by log-sum-exp rescaling; the merged accumulators
    are mapped back with sum_m U_m acc_m / l.

GQA: query head i reads kv head i // (num_q_heads / num_kv_heads).
A sequence of length 0 yields an all-zero output (nothing to attend to).
"""
from __future__ import annotations

import numpy as np

from .codec import (HEAD_DIM, NUM_MODALITIES, WINDOW, OracleCache, OracleConfig,
                    codes_per_word, unpack_key_codes, unpack_value_codes)

F64 = np.float64


def key_rotation_matrix(signs):
    """R = 2^-3.5 H diag(s) in fp64, Sylvester H_ij = (-1)^popcount(i & j)."""
    n = HEAD_DIM
    i = np.arange(n)
    pc = np.array([[bin(a & b).count("1") for b in i] for a in i])
    H = np.where(pc % 2 == 0, 1.0, -1.0)
    return (2.0 ** -3.5) * H * np.asarray(signs, dtype=F64)[None, :]


def dequantize(cfg: OracleConfig, cache: OracleCache, b: int, h: int):
    """Rotated-space dequantised cache of one (sequence, kv head):
    k_hat'[t][c] = m + s (c_j - c_0) with the record's decoded metadata (fp16 m16, s16, or
    MXFP4 m^, s^), or k_hat'[t][c] = sigma16_t c_j for the TurboQuant key codec (one
    scale per token); v_hat'[t][c] = sigma16 c_j  (fp64),
    and the modality id of every token. Returns (kq [T][128], vq [T][128], mod [T])."""
    T = int(cache.seq_lens[b])
    ck = np.asarray(cfg.key_codebook, dtype=np.float32).astype(F64)
    cv = np.asarray(cfg.value_codebook, dtype=np.float32).astype(F64)
    nw = (T + WINDOW - 1) // WINDOW
    kq = np.zeros((nw * WINDOW, HEAD_DIM), F64)
    vq = np.zeros((nw * WINDOW, HEAD_DIM), F64)
    for w in range(nw):
        kc = unpack_key_codes(cache.k_words(b, h, w), cache.key_bits)
        if cache.meta_format == "turbo":
            kq[w * WINDOW:(w + 1) * WINDOW] = cache.key_sigma(b, h, w).astype(F64)[:, None] * ck[kc]
        else:
            m, s = (x.astype(F64) for x in cache.key_meta_f32(b, h, w))
            kq[w * WINDOW:(w + 1) * WINDOW] = m[None, :] + s[None, :] * (ck[kc] - ck[0])
        vc = unpack_value_codes(cache.v_words(b, h, w), cache.value_bits)
        sg = cache.sigma(b, h, w).astype(F64)
        vq[w * WINDOW:(w + 1) * WINDOW] = sg[:, None] * cv[vc]
    return kq[:T], vq[:T], cache.modality[b, :T].copy()


def decode_dense(cfg: OracleConfig, cache: OracleCache, q_fp16):
    """out[b][i] = sum_t softmax_t(q . k_t / sqrt(128)) v_t over the dequantised
    cache in the original basis. q: [B][H_q][128] fp16. Returns fp64 [B][H_q][128]."""
    q = np.asarray(q_fp16, dtype=np.float16).astype(F64)
    B, Hq, _ = q.shape
    G = cfg.num_q_heads // cfg.num_kv_heads
    R = key_rotation_matrix(cfg.key_signs)
    out = np.zeros((B, Hq, HEAD_DIM), F64)
    for b in range(B):
        if cache.seq_lens[b] == 0:
            continue
        for h in range(cfg.num_kv_heads):
            kq, vq, mod = dequantize(cfg, cache, b, h)
            k = kq @ R                      # rows: k_t = R^T k_hat'_t
            v = np.zeros_like(vq)
            for m in range(NUM_MODALITIES):
                U = np.asarray(cfg.value_rot[h, m], dtype=np.float32).astype(F64)
                sel = mod == m
                v[sel] = vq[sel] @ U.T      # rows: v_t = U_m v_hat'_t
            for g in range(G):
                i = h * G + g
                s = (k @ q[b, i]) / np.sqrt(HEAD_DIM)
                p = np.exp(s - s.max())
                out[b, i] = (p[:, None] * v).sum(axis=0) / p.sum()
    return out


def split_ranges(num_windows: int, num_splits: int):
    """Split i covers windows [floor(i n / S), floor((i+1) n / S))."""
    return [((i * num_windows) // num_splits, ((i + 1) * num_windows) // num_splits)
            for i in range(num_splits)]


def decode_fused(cfg: OracleConfig, cache: OracleCache, q_fp16, num_splits: int = 1):
    """The fused order: rotated query, per-split online softmax with per-modality
    rotated-space accumulators, log-sum-exp merge, batched inverse rotation."""
    q = np.asarray(q_fp16, dtype=np.float16).astype(F64)
    B, Hq, _ = q.shape
    G = cfg.num_q_heads // cfg.num_kv_heads
    R = key_rotation_matrix(cfg.key_signs)
    out = np.zeros((B, Hq, HEAD_DIM), F64)
    for b in range(B):
        T = int(cache.seq_lens[b])
        if T == 0:
            continue
        nw = (T + WINDOW - 1) // WINDOW
        for h in range(cfg.num_kv_heads):
            kq, vq, mod = dequantize(cfg, cache, b, h)
            qr = q[b, h * G:(h + 1) * G] @ R.T            # q'_g = R q_g
            parts = []
            for w0, w1 in split_ranges(nw, num_splits):
                m_run = np.full(G, -np.inf)
                l_run = np.zeros(G)
                acc = np.zeros((G, NUM_MODALITIES, HEAD_DIM))
                for w in range(w0, w1):                    # FlashAttention order
                    t0, t1 = w * WINDOW, min(w * WINDOW + WINDOW, T)
                    s = (qr @ kq[t0:t1].T) / np.sqrt(HEAD_DIM)   # [G][n]
                    m_new = np.maximum(m_run, s.max(axis=1))
                    alpha = np.exp(m_run - m_new)
                    p = np.exp(s - m_new[:, None])
                    l_run = l_run * alpha + p.sum(axis=1)
                    acc *= alpha[:, None, None]
                    for m in range(NUM_MODALITIES):
                        sel = mod[t0:t1] == m
                        acc[:, m] += p[:, sel] @ vq[t0:t1][sel]
                    m_run = m_new
                parts.append((m_run, l_run, acc))
            M = np.max([p[0] for p in parts], axis=0)
            l = np.zeros(G)
            acc = np.zeros((G, NUM_MODALITIES, HEAD_DIM))
            for m_s, l_s, a_s in parts:
                e = np.where(np.isfinite(m_s), np.exp(m_s - M), 0.0)
                l += l_s * e
                acc += a_s * e[:, None, None]
            o = np.zeros((G, HEAD_DIM))
            for m in range(NUM_MODALITIES):
                U = np.asarray(cfg.value_rot[h, m], dtype=np.float32).astype(F64)
                o += (acc[:, m] / l[:, None]) @ U.T
            out[b, h * G:(h + 1) * G] = o
    return out


# ----------------------------------------------------------------------------
# streaming / captioning cache policy
# ----------------------------------------------------------------------------
STREAM_KEY_BLOCK = 128     # keys are quantised every 128 tokens (in 32-token windows)
STREAM_VALUE_WINDOW = 128  # values keep a 128-token fp16 sliding window


def stream_boundaries(T: int):
    """The streaming policy of paperpeel.com section 3.1 ("Implementation details",
    captioning: keys quantised every 128 tokens in groups of 32, values in a
    128-token fp16 sliding window before quantisation). Readings:
      s1  key blocks are aligned at absolute positions: the keys of positions
          [0, KB) are read quantised, KB = 128 floor(T / 128); the others fp16;
      s2  a value is quantised when it leaves the window of the newest 128
          tokens: positions [0, VB) are read quantised, VB = max(0, T - 128);
      s3  a quantised key or value is exactly what the ordinary cache write
          produces (the key windows of a complete block are full; the value
          codec is per token);
      s4  fp16 keys and values enter attention as they are (original basis).
    Returns (KB, VB)."""
    return STREAM_KEY_BLOCK * (T // STREAM_KEY_BLOCK), max(0, T - STREAM_VALUE_WINDOW)


def decode_dense_stream(cfg: OracleConfig, cache: OracleCache, k_raw, v_raw, q_fp16):
    """decode_dense under the streaming policy: the cache holds every token's
    record (written by the ordinary write); token t's key is the dequantised one
    for t < KB and the raw fp16 key otherwise, its value the dequantised one for
    t < VB and the raw fp16 value otherwise. k_raw, v_raw: [B][H][>= T_b][128] fp16
    (the raw inputs of every cached position); q: [B][H_q][128]. fp64 result."""
    q = np.asarray(q_fp16, dtype=np.float16).astype(F64)
    B, Hq, _ = q.shape
    G = cfg.num_q_heads // cfg.num_kv_heads
    R = key_rotation_matrix(cfg.key_signs)
    out = np.zeros((B, Hq, HEAD_DIM), F64)
    for b in range(B):
        T = int(cache.seq_lens[b])
        if T == 0:
            continue
        KB, VB = stream_boundaries(T)
        for h in range(cfg.num_kv_heads):
            kq, vq, mod = dequantize(cfg, cache, b, h)
            k = kq @ R
            v = np.zeros_like(vq)
            for m in range(NUM_MODALITIES):
                U = np.asarray(cfg.value_rot[h, m], dtype=np.float32).astype(F64)
                sel = mod == m
                v[sel] = vq[sel] @ U.T
            k[KB:T] = np.asarray(k_raw[b][h][KB:T], np.float16).astype(F64)
            v[VB:T] = np.asarray(v_raw[b][h][VB:T], np.float16).astype(F64)
            for g in range(G):
                i = h * G + g
                s = (k @ q[b, i]) / np.sqrt(HEAD_DIM)
                p = np.exp(s - s.max())
                out[b, i] = (p[:, None] * v).sum(axis=0) / p.sum()
    return out
