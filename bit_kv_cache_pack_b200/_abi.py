"""ctypes binding of libomnikv.so: the C ABI declared in include/omnikv.h.

Argument marshalling only: every step of the cache write and decode runs in the
library's CUDA kernels. Functions keep the C names; tensors may be passed as
torch tensors (their data_ptr() is used) or as integer device addresses.
A non-OK status raises OmniKVError. Loading fails loudly if the library has not
been built (python -m bit_kv_cache_pack_b200.build).
"""
from __future__ import annotations

import ctypes
import os

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libomnikv.so")

OMNIKV_OK = 0
OMNIKV_ERR_INVALID_ARG = 1
OMNIKV_ERR_UNSUPPORTED = 2
OMNIKV_ERR_CAPACITY = 3
OMNIKV_ERR_CUDA = 4
OMNIKV_ERR_DEVICE_CHECK = 5
OMNIKV_DEVERR_CAPACITY = 0x1
OMNIKV_DEVERR_MODALITY = 0x2
OMNIKV_DEVERR_TIMEOUT = 0x4
OMNIKV_DEVERR_BOUND = 0x8
OMNIKV_DEVERR_RANGE = 0x10
OMNIKV_META_FP16 = 0
OMNIKV_META_MXFP4 = 1
OMNIKV_META_TURBO = 2
OMNIKV_STREAM_TAIL_SPLITS = 4  # partials of omnikv_stream_decode: S + this many splits

EXPORTED = (
    "omnikv_record_bytes", "omnikv_partials_bytes", "omnikv_default_splits",
    "omnikv_write_cache", "omnikv_decode_attention", "omnikv_combine",
    "omnikv_status_string", "omnikv_abi_version", "omnikv_decode_static",
    "omnikv_dense_partials_bytes", "omnikv_dense_decode_bf16", "omnikv_decode_step",
    "omnikv_append_decode", "omnikv_combine_step", "omnikv_step_splits", "omnikv_write_cache_rotations",
    "omnikv_test_decode_pending", "omnikv_record_bytes_meta", "omnikv_calibrate_workspace_bytes",
    "omnikv_calibrate_bases", "omnikv_stream_write_cache", "omnikv_stream_decode",
)
OMNIKV_DECODE_STATIC_SCRATCH_BYTES = 8 << 20


class OmniKVError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s (status %d)" % (where, status_string(status), status))


class OmniKVConfig(ctypes.Structure):
    _fields_ = [
        ("head_dim", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("key_bits", ctypes.c_int32),
        ("value_bits", ctypes.c_int32),
        ("key_codebook", ctypes.c_void_p),
        ("value_codebook", ctypes.c_void_p),
        ("key_signs", ctypes.c_void_p),
        ("value_rot", ctypes.c_void_p),
        ("key_meta_format", ctypes.c_int32),
    ]


class OmniKVCache(ctypes.Structure):
    _fields_ = [
        ("records", ctypes.c_void_p),
        ("key_tail", ctypes.c_void_p),
        ("modality", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p),
        ("error_word", ctypes.c_void_p),
        ("batch", ctypes.c_int32),
        ("cap_tokens", ctypes.c_int32),
        ("max_seq_len", ctypes.c_int32),
        ("step_flags", ctypes.c_void_p),
    ]


_lib = None


def load() -> ctypes.CDLL:
    """The loaded library; raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError("libomnikv.so is not built (%s); run python -m bit_kv_cache_pack_b200.build"
                          % _LIB_PATH)
    lib = ctypes.CDLL(_LIB_PATH)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    cfgp, cachep = ctypes.POINTER(OmniKVConfig), ctypes.POINTER(OmniKVCache)
    lib.omnikv_record_bytes.argtypes, lib.omnikv_record_bytes.restype = [I32, I32], SZ
    lib.omnikv_record_bytes_meta.argtypes, lib.omnikv_record_bytes_meta.restype = [I32, I32, I32], SZ
    lib.omnikv_partials_bytes.argtypes, lib.omnikv_partials_bytes.restype = [I32, I32, I32], SZ
    lib.omnikv_default_splits.argtypes, lib.omnikv_default_splits.restype = [cfgp, cachep], I32
    lib.omnikv_write_cache.argtypes = [cfgp, cachep, P, P, P, I32, P]
    lib.omnikv_write_cache.restype = ctypes.c_int
    lib.omnikv_write_cache_rotations.argtypes = [cfgp, cachep, P, P, P, I32, P, P]
    lib.omnikv_write_cache_rotations.restype = ctypes.c_int
    lib.omnikv_test_decode_pending.argtypes = [cfgp, cachep, P, P, I32, ctypes.c_uint64, P]
    lib.omnikv_test_decode_pending.restype = ctypes.c_int
    lib.omnikv_decode_attention.argtypes = [cfgp, cachep, P, P, I32, P]
    lib.omnikv_decode_attention.restype = ctypes.c_int
    lib.omnikv_combine.argtypes = [cfgp, cachep, P, I32, P, P]
    lib.omnikv_combine.restype = ctypes.c_int
    lib.omnikv_dense_partials_bytes.argtypes, lib.omnikv_dense_partials_bytes.restype = [I32, I32, I32], SZ
    lib.omnikv_dense_decode_bf16.argtypes = [P, P, P, I32, I32, I32, I32, I32, P, P, I32, P, P, P]
    lib.omnikv_calibrate_workspace_bytes.argtypes, lib.omnikv_calibrate_workspace_bytes.restype = [I32], SZ
    lib.omnikv_stream_write_cache.argtypes = [cfgp, cachep, P, P, P, P, P, I32, P]
    lib.omnikv_stream_write_cache.restype = ctypes.c_int
    lib.omnikv_stream_decode.argtypes = [cfgp, cachep, P, P, P, P, I32, P, P]
    lib.omnikv_stream_decode.restype = ctypes.c_int
    lib.omnikv_calibrate_bases.argtypes = [P, P, P, I32, P, SZ, P, P, P]
    lib.omnikv_calibrate_bases.restype = ctypes.c_int
    lib.omnikv_dense_decode_bf16.restype = ctypes.c_int
    lib.omnikv_decode_step.argtypes = [cfgp, cachep, P, P, P, P, P, I32, P, P]
    lib.omnikv_decode_step.restype = ctypes.c_int
    lib.omnikv_step_splits.argtypes = [cfgp, cachep, I32, ctypes.POINTER(I32)]
    lib.omnikv_step_splits.restype = I32
    lib.omnikv_append_decode.argtypes = [cfgp, cachep, P, P, P, P, P, I32, P]
    lib.omnikv_append_decode.restype = ctypes.c_int
    lib.omnikv_combine_step.argtypes = [cfgp, cachep, P, I32, P, P]
    lib.omnikv_combine_step.restype = ctypes.c_int
    lib.omnikv_decode_static.argtypes = [cfgp, cachep, P, P, I32, P]
    lib.omnikv_decode_static.restype = ctypes.c_int
    lib.omnikv_status_string.argtypes, lib.omnikv_status_string.restype = [ctypes.c_int], ctypes.c_char_p
    lib.omnikv_abi_version.argtypes, lib.omnikv_abi_version.restype = [], I32
    _lib = lib
    return lib


def _ptr(x) -> int:
    """Device address of a tensor (which must be contiguous: the C ABI takes
    row-major dense arrays) or an integer address passed through."""
    if x is None:
        return 0
    if isinstance(x, int):
        return x
    if hasattr(x, "is_contiguous") and not x.is_contiguous():
        raise ValueError("tensor arguments of the C ABI must be contiguous (got strides %s)" % (x.stride(),))
    return int(x.data_ptr())


def _stream(s) -> int:
    if s is None:
        return 0
    if isinstance(s, int):
        return s
    return int(s.cuda_stream)


def _check(status: int, where: str) -> None:
    if status != OMNIKV_OK:
        raise OmniKVError(status, where)


def status_string(status: int) -> str:
    return load().omnikv_status_string(status).decode()


def omnikv_abi_version() -> int:
    return int(load().omnikv_abi_version())


def omnikv_record_bytes(key_bits: int, value_bits: int) -> int:
    return int(load().omnikv_record_bytes(key_bits, value_bits))


def omnikv_record_bytes_meta(key_bits: int, value_bits: int, key_meta_format: int) -> int:
    return int(load().omnikv_record_bytes_meta(key_bits, value_bits, key_meta_format))


def omnikv_partials_bytes(batch: int, num_q_heads: int, num_splits: int) -> int:
    return int(load().omnikv_partials_bytes(batch, num_q_heads, num_splits))


def omnikv_default_splits(cfg: OmniKVConfig, cache: OmniKVCache) -> int:
    return int(load().omnikv_default_splits(ctypes.byref(cfg), ctypes.byref(cache)))


def omnikv_write_cache(cfg: OmniKVConfig, cache: OmniKVCache, k_new, v_new, modality_new, n_new: int,
                       stream=None) -> None:
    st = load().omnikv_write_cache(ctypes.byref(cfg), ctypes.byref(cache), _ptr(k_new), _ptr(v_new),
                                   _ptr(modality_new), int(n_new), _stream(stream))
    _check(st, "omnikv_write_cache")


def omnikv_write_cache_rotations(cfg: OmniKVConfig, cache: OmniKVCache, k_new, v_new, modality_new, n_new: int,
                                 v_rot, stream=None) -> None:
    st = load().omnikv_write_cache_rotations(ctypes.byref(cfg), ctypes.byref(cache), _ptr(k_new), _ptr(v_new),
                                             _ptr(modality_new), int(n_new), _ptr(v_rot), _stream(stream))
    _check(st, "omnikv_write_cache_rotations")


def omnikv_test_decode_pending(cfg: OmniKVConfig, cache: OmniKVCache, q, partials, num_splits: int,
                               flag_wait_ns: int, stream=None) -> None:
    st = load().omnikv_test_decode_pending(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q), _ptr(partials),
                                           int(num_splits), int(flag_wait_ns), _stream(stream))
    _check(st, "omnikv_test_decode_pending")


def omnikv_decode_attention(cfg: OmniKVConfig, cache: OmniKVCache, q, partials, num_splits: int = 0,
                            stream=None) -> None:
    st = load().omnikv_decode_attention(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q), _ptr(partials),
                                        int(num_splits), _stream(stream))
    _check(st, "omnikv_decode_attention")


def omnikv_combine(cfg: OmniKVConfig, cache: OmniKVCache, partials, num_splits: int, out, stream=None) -> None:
    st = load().omnikv_combine(ctypes.byref(cfg), ctypes.byref(cache), _ptr(partials), int(num_splits),
                               _ptr(out), _stream(stream))
    _check(st, "omnikv_combine")


def omnikv_decode_step(cfg: OmniKVConfig, cache: OmniKVCache, q, k_new, v_new, modality_new, partials,
                       num_splits: int, out, stream=None) -> None:
    """Append one token per sequence, decode and combine (see include/omnikv.h);
    the cache needs its step_flags array."""
    st = load().omnikv_decode_step(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q), _ptr(k_new), _ptr(v_new),
                                   _ptr(modality_new), _ptr(partials), int(num_splits), _ptr(out), _stream(stream))
    _check(st, "omnikv_decode_step")


def omnikv_step_splits(cfg: OmniKVConfig, cache: OmniKVCache, num_splits: int = 0):
    """(split count, fused) of the next decode step; see include/omnikv.h."""
    f = ctypes.c_int32(0)
    S = int(load().omnikv_step_splits(ctypes.byref(cfg), ctypes.byref(cache), int(num_splits), ctypes.byref(f)))
    return S, bool(f.value)


def omnikv_append_decode(cfg: OmniKVConfig, cache: OmniKVCache, q, k_new, v_new, modality_new, partials,
                         num_splits: int, stream=None) -> None:
    """First launch of omnikv_decode_step (append + decode into the partials)."""
    st = load().omnikv_append_decode(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q), _ptr(k_new), _ptr(v_new),
                                     _ptr(modality_new), _ptr(partials), int(num_splits), _stream(stream))
    _check(st, "omnikv_append_decode")


def omnikv_combine_step(cfg: OmniKVConfig, cache: OmniKVCache, partials, num_splits: int, out, stream=None) -> None:
    """Second launch of omnikv_decode_step (combine + length advance)."""
    st = load().omnikv_combine_step(ctypes.byref(cfg), ctypes.byref(cache), _ptr(partials), int(num_splits),
                                    _ptr(out), _stream(stream))
    _check(st, "omnikv_combine_step")


def omnikv_decode_static(cfg: OmniKVConfig, cache: OmniKVCache, q, out, num_splits: int = 0, stream=None) -> None:
    """Decode + combine with the split partials in the library's fixed device
    array (no allocation by the caller or the library); see include/omnikv.h."""
    st = load().omnikv_decode_static(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q), _ptr(out), int(num_splits),
                                     _stream(stream))
    _check(st, "omnikv_decode_static")


def omnikv_dense_partials_bytes(batch: int, num_q_heads: int, num_splits: int) -> int:
    return int(load().omnikv_dense_partials_bytes(batch, num_q_heads, num_splits))


def omnikv_stream_write_cache(cfg: OmniKVConfig, cache: OmniKVCache, ring_k, ring_v, k_new, v_new, modality_new,
                              n_new: int, stream=None) -> None:
    """omnikv_write_cache plus the raw-input rings of the streaming policy; see include/omnikv.h."""
    st = load().omnikv_stream_write_cache(ctypes.byref(cfg), ctypes.byref(cache), _ptr(ring_k), _ptr(ring_v),
                                          _ptr(k_new), _ptr(v_new), _ptr(modality_new), int(n_new), _stream(stream))
    _check(st, "omnikv_stream_write_cache")


def omnikv_stream_decode(cfg: OmniKVConfig, cache: OmniKVCache, ring_k, ring_v, q, partials, num_splits: int, out,
                         stream=None) -> None:
    """Decode + combine under the streaming policy; see include/omnikv.h."""
    st = load().omnikv_stream_decode(ctypes.byref(cfg), ctypes.byref(cache), _ptr(ring_k), _ptr(ring_v), _ptr(q),
                                     _ptr(partials), int(num_splits), _ptr(out), _stream(stream))
    _check(st, "omnikv_stream_decode")


def omnikv_calibrate_workspace_bytes(num_tokens: int) -> int:
    return int(load().omnikv_calibrate_workspace_bytes(int(num_tokens)))


def omnikv_calibrate_bases(values, modality, weights, num_tokens: int, workspace, bases, eigenvalues=None,
                           stream=None) -> None:
    """Value bases U_m of one (layer, kv head) from calibration values; see include/omnikv.h."""
    st = load().omnikv_calibrate_bases(_ptr(values), _ptr(modality), _ptr(weights), int(num_tokens), _ptr(workspace),
                                       int(workspace.numel() * workspace.element_size()), _ptr(bases),
                                       _ptr(eigenvalues), _stream(stream))
    _check(st, "omnikv_calibrate_bases")


def omnikv_dense_decode_bf16(k_cache, v_cache, seq_lens, batch: int, num_q_heads: int, num_kv_heads: int,
                             cap_tokens: int, max_seq_len: int, q, partials, num_splits: int, out,
                             error_word=None, stream=None) -> None:
    """Dense bf16 split-K decode (comparison baseline); see include/omnikv.h."""
    st = load().omnikv_dense_decode_bf16(_ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), int(batch), int(num_q_heads),
                                         int(num_kv_heads), int(cap_tokens), int(max_seq_len), _ptr(q), _ptr(partials),
                                         int(num_splits), _ptr(out), _ptr(error_word), _stream(stream))
    _check(st, "omnikv_dense_decode_bf16")
