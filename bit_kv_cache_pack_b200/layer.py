"""Device-memory plumbing around the C ABI: PyTorch allocates, the library computes.

LayerConstants holds one layer's codebooks, key signs and value bases on the
device and the matching omnikv_config; KVCache allocates one layer's packed
cache for a batch (zero-filled, as the ABI requires) and the matching
omnikv_cache. Nothing here computes any step of the method.
"""
from __future__ import annotations

import torch

from . import _abi
from ._abi import OmniKVCache, OmniKVConfig

HEAD_DIM = 128
WINDOW = 32


class LayerConstants:
    def __init__(self, key_codebook, value_codebook, key_signs, value_rot, num_q_heads: int,
                 device="cuda", key_meta_format: int = _abi.OMNIKV_META_FP16):
        dev = torch.device(device)
        f32 = dict(dtype=torch.float32, device=dev)
        self.key_codebook = torch.as_tensor(key_codebook, **f32).contiguous()
        self.value_codebook = torch.as_tensor(value_codebook, **f32).contiguous()
        self.key_signs = torch.as_tensor(key_signs, **f32).contiguous()
        self.value_rot = torch.as_tensor(value_rot, **f32).contiguous()
        self.num_kv_heads = int(self.value_rot.shape[0])
        self.num_q_heads = int(num_q_heads)
        self.key_bits = int(self.key_codebook.numel()).bit_length() - 1
        self.value_bits = int(self.value_codebook.numel()).bit_length() - 1
        self.key_meta_format = int(key_meta_format)
        self.struct = OmniKVConfig(
            HEAD_DIM, self.num_q_heads, self.num_kv_heads, WINDOW, self.key_bits, self.value_bits,
            self.key_codebook.data_ptr(), self.value_codebook.data_ptr(), self.key_signs.data_ptr(),
            self.value_rot.data_ptr(), self.key_meta_format)


class KVCache:
    def __init__(self, batch: int, num_kv_heads: int, cap_tokens: int, key_bits: int = 2,
                 value_bits: int = 2, device="cuda", key_meta_format: int = _abi.OMNIKV_META_FP16):
        dev = torch.device(device)
        if cap_tokens % WINDOW:
            raise ValueError("cap_tokens must be a multiple of 32")
        self.record_bytes = _abi.omnikv_record_bytes_meta(key_bits, value_bits, key_meta_format)
        self.batch, self.num_kv_heads, self.cap_tokens = batch, num_kv_heads, cap_tokens
        self.key_bits, self.value_bits = key_bits, value_bits
        self.records = torch.zeros(batch, num_kv_heads, cap_tokens // WINDOW, self.record_bytes,
                                   dtype=torch.uint8, device=dev)
        self.key_tail = torch.zeros(batch, num_kv_heads, WINDOW, HEAD_DIM, dtype=torch.float16, device=dev)
        self.modality = torch.zeros(batch, cap_tokens, dtype=torch.uint8, device=dev)
        self.seq_lens = torch.zeros(batch, dtype=torch.int32, device=dev)
        self.error_word = torch.zeros(1, dtype=torch.int32, device=dev)
        self.step_flags = torch.zeros(batch, num_kv_heads, dtype=torch.int32, device=dev)
        self.struct = OmniKVCache(self.records.data_ptr(), self.key_tail.data_ptr(), self.modality.data_ptr(),
                                  self.seq_lens.data_ptr(), self.error_word.data_ptr(), batch, cap_tokens, 0,
                                  self.step_flags.data_ptr())

    @property
    def max_seq_len(self) -> int:
        return int(self.struct.max_seq_len)

    def sequence_view(self, b: int) -> OmniKVCache:
        """An omnikv_cache covering sequence b alone (batch = 1); its max_seq_len
        is the batch-wide bound."""
        return OmniKVCache(self.records[b].data_ptr(), self.key_tail[b].data_ptr(), self.modality[b].data_ptr(),
                           self.seq_lens[b:].data_ptr(), self.error_word.data_ptr(), 1, self.cap_tokens,
                           self.struct.max_seq_len, self.step_flags[b].data_ptr())


def stream_rings(batch: int, num_kv_heads: int, device="cuda"):
    """The raw fp16 key and value rings of the streaming policy, [B][H_kv][256][128] each."""
    shape = (batch, num_kv_heads, 256, HEAD_DIM)
    return (torch.zeros(shape, dtype=torch.float16, device=device),
            torch.zeros(shape, dtype=torch.float16, device=device))


def partials_tensor(batch: int, num_q_heads: int, num_splits: int, device="cuda") -> torch.Tensor:
    n = _abi.omnikv_partials_bytes(batch, num_q_heads, num_splits)
    return torch.empty(n // 4, dtype=torch.float32, device=device)
