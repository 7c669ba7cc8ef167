"""The Python binding rejects malformed tensors before it calls the library
(argument marshalling only: no computation, no fallback). CPU tensors serve
as stand-ins; every case below fails before any device work."""
import pytest
import torch

import bit_quantized_flashattention_b200 as H


def _packed(B=1, Hq=2, Hkv=1, Nq=128, Nkv=256, D=64):
    sizes = H.packed_bytes(B, Hq, Hkv, Nq, Nkv, D)
    bufs = [torch.empty(n, dtype=torch.uint8) for n in sizes]
    return H.PackedQKV(*bufs, B, Hq, Hkv, Nq, Nkv, D)


def test_inputs_must_be_device_tensors():
    x = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        H.quantize_qkv(x, x[:, :1], x[:, :1])
    with pytest.raises(ValueError, match="CUDA"):
        H.q_mean(x)
    with pytest.raises(ValueError, match="CUDA"):
        H.quantize_q(x, _packed())


def test_rope_tables_and_positions_are_checked():
    cos = torch.zeros(16, 32, dtype=torch.float64)
    with pytest.raises(ValueError):
        H.api._prequant(rope=H.Rope(cos, cos))
    cos32 = torch.zeros(16, 32, dtype=torch.float32)
    with pytest.raises(ValueError):
        H.api._prequant(rope=H.Rope(cos32, cos32))          # host tables are not device tensors


def test_tile_stats_shape_is_checked():
    with pytest.raises(ValueError):
        H.tile_stats(torch.zeros(1, 2, 128, 2, 2))              # host tensor
    with pytest.raises(ValueError):
        H.tile_stats(torch.zeros(1, 2, 128, 2))                 # wrong rank


def test_library_size_queries_through_the_binding():
    sizes = H.packed_bytes(1, 32, 8, 4096, 4096, 128)
    assert sizes[0] == 32 * 4096 * 64 and sizes[4] == 8 * 4096 * 64
    assert H.workspace_bytes(1, 32, 8, 4096, 4096, 128) == 256
    assert H.attention_splits(64, 32, 8, 16, 8192, 128, split_kv=True) == 4
    assert H.attention_splits(64, 32, 8, 16, 8192, 128, split_kv=False) == 1
    assert H.attention_splits(1, 32, 8, 4096, 4096, 128, split_kv=True) == 1   # prefill: one pass
    assert H.attention_splits(1, 32, 8, 16, 384, 128, split_kv=True) == 1      # fewer tiles than ranges
    with pytest.raises(H.HiFA4Error):
        H.packed_bytes(1, 3, 2, 16, 128, 128)
