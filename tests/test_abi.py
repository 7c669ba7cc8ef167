"""The C-ABI library loads on a machine without a GPU, exports every function
include/hifa4.h declares, and rejects bad arguments on the host before any
CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from bit_quantized_flashattention_b200 import _build, _lib
    _build.build()
    return _lib.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "hifa4.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hifa4_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_hot_path_calls():
    names = declared_functions()
    for n in ("hifa4_calibrate_smooth", "hifa4_quantize_qkv", "hifa4_attention_fwd", "hifa4_packed_bytes",
              "hifa4_workspace_bytes", "hifa4_get_status"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from bit_quantized_flashattention_b200 import _lib
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), n
        assert n in _lib.EXPORTS, n


def test_size_queries(lib):
    out = (ctypes.c_size_t * 6)()
    total = lib.hifa4_packed_bytes(1, 32, 8, 4096, 4096, 128, out)
    # codes: 0.5 B per element; scales: 1/16 B per element (no padding at this shape)
    assert list(out) == [32 * 4096 * 64, 32 * 4096 * 8, 8 * 4096 * 64, 8 * 4096 * 8, 8 * 128 * 2048, 8 * 4096 * 8]
    assert total == sum(out)
    # G*Nq = 48 rows per group: one 128-row tile of scale atoms per group
    lib.hifa4_packed_bytes(1, 6, 2, 16, 128, 128, out)
    assert out[1] == 2 * 1 * 2 * 512
    assert lib.hifa4_packed_bytes(1, 3, 2, 16, 128, 128, out) == 0        # Hq % Hkv != 0
    assert lib.hifa4_packed_bytes(1, 2, 2, 16, 100, 128, out) == 0        # Nkv % 128 != 0
    assert lib.hifa4_packed_bytes(1, 2, 2, 16, 128, 96, out) == 0         # D not in {64,128,256}
    assert lib.hifa4_workspace_bytes(1, 32, 8, 4096, 4096, 128) >= 8


def test_host_validation_rejects_before_launch(lib):
    from bit_quantized_flashattention_b200 import _lib as L
    fake = ctypes.c_void_p(1 << 20)                       # 16-byte aligned, never dereferenced
    pk = L.Packed(*([fake] * 6))
    args = dict(B=1, Hq=2, Hkv=1, Nq=128, Nkv=128, D=128)

    def attn(**kw):
        a = {**args, **kw}
        return lib.hifa4_attention_fwd(ctypes.byref(pk), a["B"], a["Hq"], a["Hkv"], a["Nq"], a["Nkv"], a["D"],
                                       ctypes.c_float(a.get("scale", 0.1)), a.get("flags", 0), a.get("norm", 0),
                                       fake, a.get("odt", L.F32), None, a.get("ws", fake), None)

    assert attn(Nkv=100) == L.ERR_UNSUPPORTED
    assert attn(D=96) == L.ERR_UNSUPPORTED
    assert attn(Nq=8) == L.ERR_UNSUPPORTED
    assert attn(Hq=3, Hkv=2) == L.ERR_UNSUPPORTED
    assert attn(Nq=256, flags=L.CAUSAL) == L.ERR_UNSUPPORTED             # causal needs Nq <= Nkv
    assert attn(scale=0.0) == L.ERR_INVALID_ARG
    assert attn(scale=float("inf")) == L.ERR_INVALID_ARG
    assert attn(flags=8) == L.ERR_INVALID_ARG
    assert attn(norm=5) == L.ERR_INVALID_ARG
    assert attn(odt=7) == L.ERR_INVALID_ARG
    assert attn(ws=None) == L.ERR_INVALID_ARG
    bad = L.Packed(*([fake] * 5 + [ctypes.c_void_p((1 << 20) + 4)]))  # misaligned scale pointer
    assert lib.hifa4_attention_fwd(ctypes.byref(bad), 1, 2, 1, 128, 128, 128, ctypes.c_float(0.1), 0, 0, fake,
                                   L.F32, None, fake, None) == L.ERR_INVALID_ARG
    assert lib.hifa4_quantize_qkv(fake, fake, fake, L.BF16, 1, 2, 1, 128, 100, 128, None, None,
                                  ctypes.byref(pk), None) == L.ERR_UNSUPPORTED
    assert lib.hifa4_quantize_qkv(fake, fake, fake, L.BF16, 1, 2, 1, 128, 128, 128, fake, None,
                                  ctypes.byref(pk), None) == L.ERR_INVALID_ARG      # s without s_inv
    assert lib.hifa4_quantize_qkv(fake, fake, fake, L.F32, 1, 2, 1, 128, 128, 128, None, None,
                                  ctypes.byref(pk), None) == L.ERR_INVALID_ARG      # fp32 inputs
    assert lib.hifa4_calibrate_smooth(fake, fake, L.BF16, 1, 2, 1, 64, 128, ctypes.c_float(0.0), fake, fake,
                                      None) == L.ERR_INVALID_ARG                     # alpha outside (0, 1]
    assert lib.hifa4_calibrate_smooth(None, fake, L.BF16, 1, 2, 1, 64, 128, ctypes.c_float(0.5), fake, fake,
                                      None) == L.ERR_INVALID_ARG
    assert lib.hifa4_status_string(4) == b"bounded wait expired inside a kernel"
    assert lib.hifa4_version() >= 100


def test_noalloc_checks_arguments_before_any_cuda_call(lib):
    """The no-allocation entry point rejects bad arguments on the host before it
    looks up its scratch array or queues the memset (on a machine without a GPU
    a CUDA call would fail, so these statuses prove the order)."""
    from bit_quantized_flashattention_b200 import _lib as L
    fake = ctypes.c_void_p(1 << 20)
    pk = L.Packed(*([fake] * 6))

    def call(Nkv=128, scale=0.1, flags=0, o=fake):
        return lib.hifa4_attention_fwd_noalloc(ctypes.byref(pk), 1, 2, 1, 128, Nkv, 128, ctypes.c_float(scale), flags,
                                               0, o, L.F32, None, None)

    assert call(Nkv=100) == L.ERR_UNSUPPORTED
    assert call(scale=0.0) == L.ERR_INVALID_ARG
    assert call(flags=8) == L.ERR_INVALID_ARG
    assert call(o=None) == L.ERR_INVALID_ARG
