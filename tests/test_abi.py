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


def declared_prototypes():
    """{name: (return type, [parameter declarations])} of every function in the header."""
    text = open(os.path.join(ROOT, "include", "hifa4.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"^\s*#.*$", "", text, flags=re.M)
    protos = {}
    for ret, name, params in re.findall(r"([A-Za-z_][\w ]*?\**)\s*\b(hifa4_[a-z0-9_]+)\s*\(([^;{}]*?)\)\s*;", text, flags=re.S):
        plist = [p.strip() for p in params.split(",") if p.strip()]
        if plist == ["void"]:
            plist = []
        protos[name] = (" ".join(ret.split()), plist)
    return protos


def _ctype_kind(t):
    if t in (ctypes.c_void_p, ctypes.c_char_p) or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return "pointer"
    return {ctypes.c_int: "int", ctypes.c_uint: "unsigned", ctypes.c_float: "float",
            ctypes.c_size_t: "size_t", ctypes.c_longlong: "long long"}.get(t, repr(t))


def _c_kind(decl):
    d = " ".join(decl.split())
    if "*" in d or "[" in d or d.startswith("hifa4_stream_t") or d.startswith("const hifa4_stream_t"):
        return "pointer"
    for k in ("size_t", "long long", "unsigned", "float"):
        if d.startswith(k) or d.startswith("const " + k):
            return k
    # int and the library's enums (status, dtype, norm mode) travel as int
    return "int"


def test_binding_signatures_match_the_header(lib):
    """The thin ctypes binding declares, for every exported call, the same
    number of parameters with the same kinds (pointer / int / unsigned /
    float / size_t / long long) and the same return kind as the header."""
    from bit_quantized_flashattention_b200 import _lib
    protos = declared_prototypes()
    assert set(protos) == set(declared_functions())
    for name, (ret, params) in protos.items():
        fn = getattr(lib, name)
        assert fn.argtypes is not None, name
        got = [_ctype_kind(t) for t in fn.argtypes]
        want = [_c_kind(p) for p in params]
        assert got == want, (name, got, want)
        want_ret = "pointer" if ("*" in ret) else _c_kind(ret)
        assert _ctype_kind(fn.restype) == want_ret, (name, fn.restype, ret)


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


def test_extension_calls_validate_on_the_host(lib):
    """RoPE / Q-Mean / Q-only / append / extras / tile-statistics calls reject bad
    arguments before any CUDA call (a CUDA call would fail without a GPU)."""
    from bit_quantized_flashattention_b200 import _lib as L
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 4)
    pk = L.Packed(*([fake] * 6))

    def pre(**kw):
        p = L.Prequant()
        for k, v in kw.items():
            setattr(p, k, v)
        return ctypes.byref(p)

    def qx(p):
        return lib.hifa4_quantize_qkv_ex(fake, fake, fake, L.BF16, 1, 2, 1, 128, 128, 128, p, ctypes.byref(pk), None)

    assert qx(pre(s=fake)) == L.ERR_INVALID_ARG                            # s without s_inv
    assert qx(pre(rope_cos=fake)) == L.ERR_INVALID_ARG                     # cos without sin
    assert qx(pre(rope_cos=fake, rope_sin=fake, n_pos=8, k_pos=fake)) == L.ERR_INVALID_ARG   # no q_pos
    assert qx(pre(rope_cos=fake, rope_sin=fake, n_pos=0, q_pos=fake, k_pos=fake)) == L.ERR_INVALID_ARG
    assert qx(pre(rope_cos=odd, rope_sin=fake, n_pos=8, q_pos=fake, k_pos=fake)) == L.ERR_INVALID_ARG
    assert qx(pre(q_mean=fake)) == L.ERR_INVALID_ARG                       # q_mean without s_bias
    assert qx(pre(q_mean=fake, s_bias=odd)) == L.ERR_INVALID_ARG

    def qo(p=None, dtype=L.BF16, Hq=2, Hkv=1, Nq=128, D=128, q=fake, packed=pk):
        return lib.hifa4_quantize_q(q, dtype, 1, Hq, Hkv, Nq, D, p, ctypes.byref(packed), None)

    assert qo(pre(s_bias=fake)) == L.ERR_INVALID_ARG                       # the bias belongs to the K pass
    assert qo(pre(q_mean=odd)) == L.ERR_INVALID_ARG
    assert qo(pre(s=odd)) == L.ERR_INVALID_ARG
    assert qo(pre(rope_cos=fake, rope_sin=fake, n_pos=8)) == L.ERR_INVALID_ARG      # no q_pos
    assert qo(dtype=L.F32) == L.ERR_INVALID_ARG
    assert qo(D=96) == L.ERR_UNSUPPORTED
    assert qo(Hq=3, Hkv=2) == L.ERR_UNSUPPORTED
    assert qo(Nq=8) == L.ERR_UNSUPPORTED
    assert qo(q=None) == L.ERR_INVALID_ARG
    assert qo(packed=L.Packed(fake, None, None, None, None, None)) == L.ERR_INVALID_ARG   # no qs

    def app(n_new=16, start=0, cap=128, p=None):
        return lib.hifa4_append_kv(fake, fake, L.BF16, 1, 1, n_new, 128, p, ctypes.byref(pk), cap, start, None)

    assert app(n_new=8) == L.ERR_INVALID_ARG                               # not a multiple of 16
    assert app(start=8) == L.ERR_INVALID_ARG
    assert app(start=120) == L.ERR_INVALID_ARG                             # past the end of the cache
    assert app(n_new=0) == L.ERR_INVALID_ARG
    assert app(cap=100) == L.ERR_UNSUPPORTED
    assert app(p=pre(q_mean=fake, s_bias=fake)) == L.ERR_INVALID_ARG       # no Q-Mean on an append
    assert app(p=pre(rope_cos=fake, rope_sin=fake, n_pos=4)) == L.ERR_INVALID_ARG   # no k_pos

    assert lib.hifa4_q_mean(fake, L.BF16, 1, 2, 1, 128, 96, None, fake, None) == L.ERR_UNSUPPORTED
    assert lib.hifa4_q_mean(fake, L.BF16, 1, 3, 2, 128, 128, None, fake, None) == L.ERR_INVALID_ARG
    assert lib.hifa4_q_mean(fake, L.BF16, 1, 2, 1, 128, 128, None, odd, None) == L.ERR_INVALID_ARG

    def ax(ex):
        return lib.hifa4_attention_fwd_ex(ctypes.byref(pk), 1, 2, 1, 128, 128, 128, ctypes.c_float(0.1), 0, 0, fake,
                                          L.F32, None, ex, fake, None)

    assert ax(ctypes.byref(L.AttentionExtras(None, fake, None, None))) == L.ERR_INVALID_ARG   # codes, no scales
    assert ax(ctypes.byref(L.AttentionExtras(odd, None, None, None))) == L.ERR_INVALID_ARG
    assert ax(ctypes.byref(L.AttentionExtras(None, None, None, odd))) == L.ERR_INVALID_ARG
    assert lib.hifa4_tile_stats(fake, 1, 2, 128, 100, fake, None) == L.ERR_INVALID_ARG
    assert lib.hifa4_tile_stats(None, 1, 2, 128, 128, fake, None) == L.ERR_INVALID_ARG


def test_in_kernel_q_entry_point_validates_on_the_host(lib):
    from bit_quantized_flashattention_b200 import _lib as L
    fake = ctypes.c_void_p(1 << 20)
    pk = L.Packed(*([fake] * 6))

    def call(q=fake, dt=None, D=128, Nq=128, Nkv=256, flags=0, Hq=2, Hkv=1, B=1):
        return lib.hifa4_attention_fwd_q(q, L.BF16 if dt is None else dt, None, ctypes.byref(pk), B, Hq, Hkv, Nq, Nkv,
                                         D, ctypes.c_float(0.1), flags, 0, fake, L.F32, None, fake, None)

    assert call(q=None) == L.ERR_INVALID_ARG
    assert call(dt=L.F32) == L.ERR_INVALID_ARG
    assert call(q=ctypes.c_void_p((1 << 20) + 8)) == L.ERR_INVALID_ARG
    assert call(D=64) == L.ERR_UNSUPPORTED                                  # D = 128 only
    assert call(Nkv=100) == L.ERR_UNSUPPORTED
    assert call(Hq=8, Hkv=2, Nq=16, Nkv=512, flags=L.SPLIT_KV) == L.ERR_UNSUPPORTED   # would take the decode mode
