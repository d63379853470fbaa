"""C ABI checks that need no GPU: the library builds and loads, exports every
entry point include/nsnq.h declares, and rejects bad arguments on the host
before anything is launched."""
import ctypes
import os
import re

import pytest

import attention_decode_b200 as nsnq
from attention_decode_b200 import build as nbuild
from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "nsnq.h")
FAKE = 0x10000  # a 16-byte aligned non-null address: validation never dereferences it


@pytest.fixture(scope="module")
def lib():
    nbuild.build()
    return nsnq.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nsnq_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_exported_set(lib):
    decl = declared_functions()
    assert set(decl) == set(nsnq.EXPORTED), decl
    for name in decl:
        assert hasattr(lib, name), name


def test_symbols_in_dynamic_table(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", nsnq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    for name in declared_functions():
        assert re.search(rf"\bT {name}\b", out), name


def test_status_strings(lib):
    assert lib.nsnq_status_string(0) == b"NSNQ_OK"
    assert lib.nsnq_status_string(3) == b"NSNQ_ERR_WORKSPACE"


def _cb(sub=4, n=256, ptr=FAKE, index=FAKE):
    return nsnq._Codebook(ptr, n, sub, index)


def _cache(cap=100):
    return nsnq._Cache(FAKE, FAKE, FAKE, cap)


def _encode(lib, **kw):
    a = dict(x=FAKE, dt=nsnq.NSNQ_BF16, B=1, H=1, T=10, D=128, sb=128 * 10, sh=128 * 10, st=128,
             off=0, mode=0, flags=0, cb=_cb(), cache=_cache(), ws=FAKE, wsb=1 << 20, stream=None)
    a.update(kw)
    return lib.nsnq_encode(a["x"], a["dt"], a["B"], a["H"], a["T"], a["D"], a["sb"], a["sh"],
                           a["st"], a["off"], a["mode"], a["flags"], a["cb"], a["cache"], a["ws"],
                           a["wsb"], a["stream"])


def test_encode_validation(lib):
    assert _encode(lib, D=64) == nsnq.NSNQ_ERR_UNSUPPORTED
    assert _encode(lib, cb=_cb(sub=5)) == nsnq.NSNQ_ERR_UNSUPPORTED
    assert _encode(lib, cb=_cb(n=128)) == nsnq.NSNQ_ERR_UNSUPPORTED
    assert _encode(lib, cb=_cb(ptr=None)) == nsnq.NSNQ_ERR_INVALID_ARG
    assert _encode(lib, x=None) == nsnq.NSNQ_ERR_INVALID_ARG
    assert _encode(lib, x=FAKE + 2) == nsnq.NSNQ_ERR_INVALID_ARG        # misaligned
    assert _encode(lib, st=100) == nsnq.NSNQ_ERR_INVALID_ARG            # stride_t < D
    assert _encode(lib, off=95) == nsnq.NSNQ_ERR_INVALID_ARG            # past capacity
    assert _encode(lib, T=-1) == nsnq.NSNQ_ERR_INVALID_ARG
    assert _encode(lib, mode=7) == nsnq.NSNQ_ERR_INVALID_ARG
    assert _encode(lib, flags=8) == nsnq.NSNQ_ERR_INVALID_ARG            # unknown flag bit
    assert _encode(lib, flags=2) == nsnq.NSNQ_ERR_INVALID_ARG  # double quantization needs s1_grid
    assert _encode(lib, ws=None) == nsnq.NSNQ_ERR_WORKSPACE
    assert _encode(lib, cb=_cb(index=None)) == nsnq.NSNQ_ERR_INVALID_ARG     # 2-bit needs its index
    assert b"nsnq_codebook_index_build" in lib.nsnq_last_error()
    assert _encode(lib, cb=_cb(sub=8, index=None), T=0) == nsnq.NSNQ_OK
    # the tensor-core search needs no index: the index check passes and the
    # workspace check (later) fails; without the flag the index check fails
    assert _encode(lib, cb=_cb(index=None), wsb=16) == nsnq.NSNQ_ERR_INVALID_ARG
    assert _encode(lib, cb=_cb(index=None), flags=nsnq.ENCODE_TC_SEARCH, wsb=16) == nsnq.NSNQ_ERR_WORKSPACE
    need = lib.nsnq_encode_workspace(1, 1, 10, 128)
    assert need > 0
    assert _encode(lib, wsb=need - 1) == nsnq.NSNQ_ERR_WORKSPACE
    assert b"workspace" in lib.nsnq_last_error()
    assert _encode(lib, T=0) == nsnq.NSNQ_OK                            # no-op, no launch
    assert lib.nsnq_last_error() == b""


def _cache_v(cap=100):  # buffers distinct from _cache()'s
    return nsnq._Cache(0x20000, 0x21000, 0x22000, cap)


def _encode_kv(lib, **kw):
    a = dict(xk=FAKE, xv=FAKE + 0x1000, dt=nsnq.NSNQ_BF16, B=1, H=1, T=10, D=128, sb=128 * 10,
             sh=128 * 10, st=128, off=0, mode=0, flags=0, cb=_cb(), ck=_cache(), cv=_cache_v(),
             ws=FAKE, wsb=1 << 20, stream=None)
    a.update(kw)
    return lib.nsnq_encode_kv(a["xk"], a["xv"], a["dt"], a["B"], a["H"], a["T"], a["D"], a["sb"],
                              a["sh"], a["st"], a["off"], a["mode"], a["flags"], a["cb"], a["ck"],
                              a["cv"], a["ws"], a["wsb"], a["stream"])


def test_encode_kv_validation(lib):
    assert _encode_kv(lib, D=64) == nsnq.NSNQ_ERR_UNSUPPORTED
    assert _encode_kv(lib, xv=None) == nsnq.NSNQ_ERR_INVALID_ARG
    assert _encode_kv(lib, xv=FAKE + 2) == nsnq.NSNQ_ERR_INVALID_ARG     # misaligned
    assert _encode_kv(lib, cv=_cache_v(cap=99)) == nsnq.NSNQ_ERR_INVALID_ARG  # caps differ
    assert b"cap" in lib.nsnq_last_error()
    assert _encode_kv(lib, cv=nsnq._Cache(FAKE, None, FAKE, 100)) == nsnq.NSNQ_ERR_INVALID_ARG
    assert b"cache_v" in lib.nsnq_last_error()
    packed = nsnq._Cache(FAKE, FAKE, FAKE, 100, FAKE, FAKE)
    plain_dq = nsnq._Cache(0x20000, 0x21000, 0x22000, 100, 0x23000, None)
    assert _encode_kv(lib, ck=packed, cv=plain_dq, flags=nsnq.ENCODE_DOUBLE_QUANT) == \
        nsnq.NSNQ_ERR_INVALID_ARG                                       # one packed, one not
    assert b"packed" in lib.nsnq_last_error()
    assert _encode_kv(lib, B=32768) == nsnq.NSNQ_ERR_UNSUPPORTED          # grid batch 2B
    same = _cache()
    assert _encode_kv(lib, ck=same, cv=same) == nsnq.NSNQ_ERR_INVALID_ARG  # one cache for both
    assert b"share" in lib.nsnq_last_error()
    assert _encode_kv(lib, B=1 << 14, H=1 << 10, T=1 << 6) == nsnq.NSNQ_ERR_UNSUPPORTED  # 2^31
    # the workspace is that of a 2B-batch encode
    need = lib.nsnq_encode_kv_workspace(1, 1, 10, 128)
    assert need == lib.nsnq_encode_workspace(2, 1, 10, 128) > 0
    assert lib.nsnq_encode_kv_workspace(8, 8, 4096, 128) == lib.nsnq_encode_workspace(16, 8, 4096, 128)
    assert lib.nsnq_encode_kv_workspace(32768, 1, 10, 128) == 0
    assert _encode_kv(lib, wsb=need - 1) == nsnq.NSNQ_ERR_WORKSPACE
    assert _encode_kv(lib, T=0) == nsnq.NSNQ_OK                          # no-op, no launch
    assert lib.nsnq_last_error() == b""


def test_binding_encode_kv_checks_the_pair_layout():
    """The binding rejects keys and values of different shape, dtype or
    strides before it touches the library (the C ABI takes one layout)."""
    import torch
    k = torch.empty(1, 2, 10, 128, dtype=torch.bfloat16)
    for v in (torch.empty(1, 2, 11, 128, dtype=torch.bfloat16),
              torch.empty(1, 2, 10, 128, dtype=torch.float32),
              torch.empty(1, 2, 10, 256, dtype=torch.bfloat16)[..., :128]):
        with pytest.raises(ValueError):
            nsnq.nsnq_encode_kv(k, v, None, None, None)


def test_index_build_validation(lib):
    assert lib.nsnq_codebook_index_bytes(4) > 0 and lib.nsnq_codebook_index_bytes(8) == 0
    need = lib.nsnq_codebook_index_bytes(4)
    assert lib.nsnq_codebook_index_build(_cb(sub=8), FAKE, need, None) == nsnq.NSNQ_ERR_UNSUPPORTED
    assert lib.nsnq_codebook_index_build(_cb(), None, need, None) == nsnq.NSNQ_ERR_INVALID_ARG
    assert lib.nsnq_codebook_index_build(_cb(), FAKE, need - 1, None) == nsnq.NSNQ_ERR_WORKSPACE


def test_encode_workspace_is_bounded(lib):
    # pass 1 uses at most one wave of chunks: the workspace stops growing with T
    a = lib.nsnq_encode_workspace(8, 8, 256, 128)
    b = lib.nsnq_encode_workspace(8, 8, 4096, 128)
    c = lib.nsnq_encode_workspace(8, 8, 1 << 20, 128)
    assert 0 < a <= b == c and a % 256 == 0
    assert lib.nsnq_encode_workspace(1, 1, 10, 128) > 0
    assert lib.nsnq_encode_workspace(8, 8, 4096, 64) == 0


def test_dequant_validation(lib):
    f = lambda **kw: lib.nsnq_dequant(kw.get("cache", _cache()), kw.get("cb", _cb()), 1, 1,
                                      kw.get("t0", 0), kw.get("T", 10), kw.get("D", 128),
                                      kw.get("out", FAKE), None)
    assert f(D=256) == nsnq.NSNQ_ERR_UNSUPPORTED
    assert f(t0=95) == nsnq.NSNQ_ERR_INVALID_ARG
    assert f(out=None) == nsnq.NSNQ_ERR_INVALID_ARG
    assert f(out=FAKE + 4) == nsnq.NSNQ_ERR_INVALID_ARG
    assert f(cache=nsnq._Cache(None, FAKE, FAKE, 100)) == nsnq.NSNQ_ERR_INVALID_ARG
    assert f(T=0) == nsnq.NSNQ_OK


def _attn(lib, **kw):
    a = dict(q=FAKE, qdt=nsnq.NSNQ_BF16, kc=_cache(), vc=_cache(), kcb=_cb(4), vcb=_cb(8),
             lens=FAKE, max_len=100, B=2, Hq=8, Hkv=2, D=128, scale=0.0, out=FAKE,
             odt=nsnq.NSNQ_BF16, ws=FAKE, wsb=1 << 24)
    a.update(kw)
    return lib.nsnq_attn_decode(a["q"], a["qdt"], a["kc"], a["vc"], a["kcb"], a["vcb"], a["lens"],
                                a["max_len"], a["B"], a["Hq"], a["Hkv"], a["D"], a["scale"],
                                a["out"], a["odt"], a["ws"], a["wsb"], None)


def test_attention_validation(lib):
    assert _attn(lib, Hq=6, Hkv=4) == nsnq.NSNQ_ERR_INVALID_ARG
    assert _attn(lib, max_len=101) == nsnq.NSNQ_ERR_INVALID_ARG
    assert _attn(lib, vc=_cache(cap=50)) == nsnq.NSNQ_ERR_INVALID_ARG
    assert _attn(lib, lens=None) == nsnq.NSNQ_ERR_INVALID_ARG
    assert _attn(lib, qdt=9) == nsnq.NSNQ_ERR_UNSUPPORTED
    assert _attn(lib, vcb=_cb(3)) == nsnq.NSNQ_ERR_UNSUPPORTED
    assert _attn(lib, scale=float("nan")) == nsnq.NSNQ_ERR_INVALID_ARG
    assert _attn(lib, wsb=16) == nsnq.NSNQ_ERR_WORKSPACE
    assert _attn(lib, B=0) == nsnq.NSNQ_OK
    need = lib.nsnq_attn_workspace(2, 8, 2, 128, 100)
    assert need > 0 and need % 256 == 0
    assert lib.nsnq_attn_workspace(2, 8, 3, 128, 100) == 0


def _attn_res(lib, res, **kw):
    a = dict(q=FAKE, qdt=nsnq.NSNQ_BF16, kc=_cache(), vc=_cache(), kcb=_cb(4), vcb=_cb(8),
             lens=FAKE, max_len=100, B=2, Hq=8, Hkv=2, D=128, scale=0.0, out=FAKE,
             odt=nsnq.NSNQ_BF16, ws=FAKE, wsb=1 << 24)
    a.update(kw)
    return lib.nsnq_attn_decode_res(a["q"], a["qdt"], a["kc"], a["vc"], a["kcb"], a["vcb"],
                                    a["lens"], a["max_len"], res, a["B"], a["Hq"], a["Hkv"],
                                    a["D"], a["scale"], a["out"], a["odt"], a["ws"], a["wsb"],
                                    None)


def test_residual_attention_validation(lib):
    R = lambda k=FAKE, v=FAKE, dt=nsnq.NSNQ_BF16, lens=FAKE, cap=16: nsnq._Residual(k, v, dt, lens, cap)
    assert _attn_res(lib, R(cap=-1)) == nsnq.NSNQ_ERR_INVALID_ARG
    assert _attn_res(lib, R(k=None)) == nsnq.NSNQ_ERR_INVALID_ARG
    assert _attn_res(lib, R(lens=None)) == nsnq.NSNQ_ERR_INVALID_ARG
    assert _attn_res(lib, R(v=FAKE + 8)) == nsnq.NSNQ_ERR_INVALID_ARG
    assert _attn_res(lib, R(dt=7)) == nsnq.NSNQ_ERR_UNSUPPORTED
    assert _attn_res(lib, R(), Hq=6, Hkv=4) == nsnq.NSNQ_ERR_INVALID_ARG
    assert _attn_res(lib, R(), wsb=16) == nsnq.NSNQ_ERR_WORKSPACE
    assert _attn_res(lib, R(), B=0) == nsnq.NSNQ_OK
    # no window: NULL pointers are accepted (the call is nsnq_attn_decode)
    assert _attn_res(lib, R(k=None, v=None, lens=None, cap=0), B=0) == nsnq.NSNQ_OK


def test_rope_attention_validation(lib):
    def f(base=10000.0, **kw):
        a = dict(q=FAKE, qdt=nsnq.NSNQ_BF16, kc=_cache(), vc=_cache(), kcb=_cb(4), vcb=_cb(8),
                 lens=FAKE, max_len=100, B=2, Hq=8, Hkv=2, D=128, scale=0.0, out=FAKE,
                 odt=nsnq.NSNQ_BF16, ws=FAKE, wsb=1 << 24)
        a.update(kw)
        return lib.nsnq_attn_decode_rope(a["q"], a["qdt"], a["kc"], a["vc"], a["kcb"], a["vcb"],
                                         a["lens"], a["max_len"], base, a["B"], a["Hq"], a["Hkv"],
                                         a["D"], a["scale"], a["out"], a["odt"], a["ws"], a["wsb"],
                                         None)
    assert f(base=float("nan")) == nsnq.NSNQ_ERR_INVALID_ARG
    assert f(base=1.0) == nsnq.NSNQ_ERR_INVALID_ARG
    assert f(Hq=6, Hkv=4) == nsnq.NSNQ_ERR_INVALID_ARG
    assert f(wsb=16) == nsnq.NSNQ_ERR_WORKSPACE
    assert f(qdt=9) == nsnq.NSNQ_ERR_UNSUPPORTED
    assert f(B=0) == nsnq.NSNQ_OK


def test_residual_write_validation(lib):
    def f(**kw):
        a = dict(x=FAKE, dt=nsnq.NSNQ_BF16, B=2, H=2, T=1, D=128, sb=512, sh=256, st=128, off=3,
                 buf=FAKE, bdt=nsnq.NSNQ_BF16, cap=4)
        a.update(kw)
        return lib.nsnq_residual_write(a["x"], a["dt"], a["B"], a["H"], a["T"], a["D"], a["sb"],
                                       a["sh"], a["st"], a["off"], a["buf"], a["bdt"], a["cap"],
                                       None)
    assert f(off=4) == nsnq.NSNQ_ERR_INVALID_ARG
    assert f(T=2) == nsnq.NSNQ_ERR_INVALID_ARG
    assert f(off=-1) == nsnq.NSNQ_ERR_INVALID_ARG
    assert f(D=64) == nsnq.NSNQ_ERR_UNSUPPORTED
    assert f(bdt=5) == nsnq.NSNQ_ERR_UNSUPPORTED
    assert f(x=None) == nsnq.NSNQ_ERR_INVALID_ARG
    assert f(buf=FAKE + 2) == nsnq.NSNQ_ERR_INVALID_ARG
    assert f(st=100) == nsnq.NSNQ_ERR_INVALID_ARG
    assert f(sh=12) == nsnq.NSNQ_ERR_INVALID_ARG
    assert f(T=0) == nsnq.NSNQ_OK


def test_codebook_quantize4_validation(lib):
    q = lib.nsnq_codebook_quantize4
    assert q(FAKE, FAKE, None, None, 128, 4, None) == nsnq.NSNQ_ERR_UNSUPPORTED
    assert q(FAKE, FAKE, None, None, 256, 5, None) == nsnq.NSNQ_ERR_UNSUPPORTED
    assert q(None, FAKE, None, None, 256, 4, None) == nsnq.NSNQ_ERR_INVALID_ARG
    assert q(FAKE, None, None, None, 256, 8, None) == nsnq.NSNQ_ERR_INVALID_ARG
    assert q(FAKE + 2, FAKE, None, None, 256, 8, None) == nsnq.NSNQ_ERR_INVALID_ARG
    assert q(FAKE, FAKE, None, FAKE + 4, 256, 8, None) == nsnq.NSNQ_ERR_INVALID_ARG


def test_packed_cache_validation(lib):
    packed = nsnq._Cache(FAKE, FAKE, FAKE, 100, FAKE, FAKE)
    no_grid = nsnq._Cache(FAKE, FAKE, FAKE, 100, None, FAKE)
    # a packed cache takes double-quantized s1 only, and needs its grid
    assert _encode(lib, cache=packed, flags=0) == nsnq.NSNQ_ERR_INVALID_ARG
    assert _encode(lib, cache=no_grid, flags=2) == nsnq.NSNQ_ERR_INVALID_ARG
    assert _encode(lib, cache=nsnq._Cache(FAKE, FAKE, FAKE, 100, FAKE, FAKE + 2),
                   flags=2) == nsnq.NSNQ_ERR_INVALID_ARG
    assert lib.nsnq_dequant(no_grid, _cb(), 1, 1, 0, 10, 128, FAKE, None) == nsnq.NSNQ_ERR_INVALID_ARG


def test_binding_has_no_fallback(tmp_path):
    """The binding raises when the library file is absent; it never computes on the CPU."""
    import importlib
    mod = importlib.reload(nsnq)
    mod._lib = None
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        mod.load(str(tmp_path / "missing.so"))
    mod._lib = None
    mod.load()
