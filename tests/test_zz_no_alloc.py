"""hifa4_attention_fwd_noalloc: the attention call for callers that cannot
allocate device memory (a plugin inside a runtime that owns all device memory
and offers no allocator, or a path that cannot afford cudaMalloc's implicit
device synchronisation). Its scratch is the library's own fixed device array.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W
from tests import hifa4_testutil as U

pytestmark = pytest.mark.gpu

O_MAX_ABS = 5e-3     # the tolerances of the parity tests
O_ROW_REL = 1e-3


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    import bit_quantized_flashattention_b200 as H
    from bit_quantized_flashattention_b200 import _lib as L
    lib = L.load()
    B, Hq, Hkv, Nq, Nkv, D = 1, 4, 2, 256, 384, 128
    rng = np.random.default_rng(21)
    q = W.round_to_dtype(rng.standard_normal((B, Hq, Nq, D)).astype(np.float32), "bf16")
    k = W.round_to_dtype(rng.standard_normal((B, Hkv, Nkv, D)).astype(np.float32), "bf16")
    v = W.round_to_dtype(rng.standard_normal((B, Hkv, Nkv, D)).astype(np.float32), "bf16")
    pk = H.quantize_qkv(U.to_device(q, "bf16"), U.to_device(k, "bf16"), U.to_device(v, "bf16"))
    o_ref, lse_ref = H.attention_fwd(pk, causal=True, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = o_ref.double().cpu().numpy().reshape(-1, D)
    st = pk.struct()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        status = lib.hifa4_attention_fwd_noalloc(ctypes.byref(st), B, Hq, Hkv, Nq, Nkv, D, 1.0 / np.sqrt(D),
                                                 L.CAUSAL, L.NORM_P_REORDER, ctypes.c_void_p(o.data_ptr()), L.F32,
                                                 ctypes.c_void_p(lse.data_ptr()), stream)
        assert status == L.OK, f"call {call}: {L.status_string(status)}"
        torch.cuda.synchronize()
        max_abs, rel = U.row_errors(o.cpu().numpy().reshape(-1, D), ref)
        assert max_abs <= O_MAX_ABS and rel.max() <= O_ROW_REL, (call, max_abs, rel.max())
        assert float((lse - lse_ref).abs().max()) <= 1e-3
