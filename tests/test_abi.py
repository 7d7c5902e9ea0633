"""The C-ABI library loads without a GPU, exports every entry point include/ck.h declares,
and rejects invalid calls on the host before any CUDA work (no device needed)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest
import torch

from rotated_w4a4_quantized_group_b200 import build as ck_build
from rotated_w4a4_quantized_group_b200 import ck

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ck.h")


@pytest.fixture(scope="module")
def L():
    ck_build.build()
    return ck.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ck_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("ck_rotate_quant", "ck_w4a4_linear", "ck_unpack_w4"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(ck.SIGNATURES), "binding signatures must cover the header exactly"


def test_status_strings(L):
    for s in range(7):
        assert ck.status_string(s)
    assert "overflow" in ck.status_string(ck.CK_ERR_OVERFLOW).lower()


def test_workspace_sizes(L):
    M, N, K = 8192, 3840, 3840
    P = ck.workspace_codes_pitch(K)
    assert P == 3840 and ck.workspace_codes_pitch(48) == 48 and ck.workspace_codes_pitch(40) == 48
    off = ck.workspace_scales_offset(M, K)
    assert off >= M * P and off % 256 == 0
    assert ck.workspace_bytes(M, N, K, K // 2) >= off + 4 * M
    # an unaligned weight pitch adds room for a 16-byte-pitched weight copy
    assert ck.workspace_bytes(7, 5, 48, 24) >= ck.workspace_bytes(7, 5, 48, 32) + 5 * 32
    assert ck.workspace_bytes(7, 5, 47, 24) == 0          # odd K is invalid


NULL = None


def rq(L, **kw):
    a = dict(x=1 << 20, dt=ck.CK_BF16, M=4, K=64, sm=64, sk=1, R=1 << 20, g=16, scale_in=NULL,
             codes=1 << 20, ldq=64, scales=1 << 20, dev_status=NULL, stream=NULL)
    a.update(kw)
    return L.ck_rotate_quant(a["x"], a["dt"], a["M"], a["K"], a["sm"], a["sk"], a["R"], a["g"],
                             a["scale_in"], a["codes"], a["ldq"], a["scales"], a["dev_status"],
                             a["stream"])


@pytest.mark.parametrize("bad", [dict(g=32), dict(g=0), dict(K=48, g=64), dict(K=0), dict(M=-1),
                                 dict(ldq=63), dict(dt=ck.CK_I8), dict(dt=9), dict(x=NULL),
                                 dict(R=NULL), dict(codes=NULL), dict(scales=NULL),
                                 dict(R=(1 << 20) + 2)])
def test_rotate_quant_rejects_on_host(L, bad):
    assert rq(L, **bad) == ck.CK_ERR_INVALID_ARG


def test_rotate_quant_empty_rows_is_a_noop(L):
    assert rq(L, M=0, x=NULL, codes=NULL, scales=NULL) == ck.CK_OK


def lin(L, **kw):
    a = dict(x=1 << 20, dt=ck.CK_BF16, M=4, K=64, sm=64, sk=1, R=1 << 20, g=16, a_scale=NULL,
             w=1 << 20, N=8, w_ld=32, w_scale=1 << 20, sdt=ck.CK_BF16, bias=NULL, out=1 << 20,
             odt=ck.CK_BF16, ldo=8, ws=1 << 20, ws_bytes=1 << 20, dev_status=NULL, stream=NULL)
    a.update(kw)
    return L.ck_w4a4_linear(a["x"], a["dt"], a["M"], a["K"], a["sm"], a["sk"], a["R"], a["g"],
                            a["a_scale"], a["w"], a["N"], a["w_ld"], a["w_scale"], a["sdt"],
                            a["bias"], a["out"], a["odt"], a["ldo"], a["ws"], a["ws_bytes"],
                            a["dev_status"], a["stream"])


@pytest.mark.parametrize("bad", [dict(K=63), dict(K=48, g=64), dict(g=8), dict(w_ld=31),
                                 dict(ldo=7), dict(sdt=ck.CK_I8), dict(odt=ck.CK_I8), dict(dt=7),
                                 dict(M=-2), dict(N=-1), dict(x=NULL), dict(w=NULL),
                                 dict(w_scale=NULL), dict(out=NULL), dict(R=NULL),
                                 dict(dt=ck.CK_I8, sk=2), dict(dt=ck.CK_I8, sm=32),
                                 dict(dt=ck.CK_I8, a_scale=NULL)])
def test_linear_rejects_on_host(L, bad):
    assert lin(L, **bad) == ck.CK_ERR_INVALID_ARG


def test_linear_overflow_guard(L):
    K = (2 ** 31 - 1) // 64 + 1
    K += K % 2
    assert lin(L, dt=ck.CK_I8, K=K, sm=K, w_ld=K // 2, a_scale=1 << 20) == ck.CK_ERR_OVERFLOW
    # the largest even K under the bound passes the guard (and then fails on the fake
    # null workspace, still on the host)
    Kfit = (2 ** 31 - 1) // 64 // 2 * 2
    assert lin(L, K=Kfit, g=16, sm=Kfit, w_ld=Kfit // 2, ws=NULL, ws_bytes=0) in (
        ck.CK_ERR_INVALID_ARG, ck.CK_ERR_WORKSPACE)


def test_linear_missing_workspace(L):
    assert lin(L, ws=NULL, ws_bytes=0) == ck.CK_ERR_WORKSPACE
    assert lin(L, ws_bytes=10) == ck.CK_ERR_WORKSPACE
    assert lin(L, ws=(1 << 20) + 16) == ck.CK_ERR_WORKSPACE     # not 256-byte aligned


def test_linear_empty_is_a_noop(L):
    assert lin(L, M=0, x=NULL, out=NULL, ws=NULL, ws_bytes=0) == ck.CK_OK
    assert lin(L, N=0, ldo=0, x=NULL, out=NULL, ws=NULL, ws_bytes=0) == ck.CK_OK


@pytest.mark.parametrize("bad", [dict(K=7), dict(K=0), dict(N=-1), dict(ldp=3), dict(ldo=15),
                                 dict(p=NULL), dict(o=NULL)])
def test_unpack_rejects_on_host(L, bad):
    a = dict(p=1 << 20, N=4, K=16, ldp=8, o=1 << 20, ldo=16)
    a.update(bad)
    assert L.ck_unpack_w4(a["p"], a["N"], a["K"], a["ldp"], a["o"], a["ldo"], None) == \
        ck.CK_ERR_INVALID_ARG


def test_product_path_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(ck, "_lib", None)
    monkeypatch.setattr(ck, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        ck.lib()


def test_binding_refuses_host_tensors(L):
    """A CPU tensor never reaches the library: its address would be read by the device."""
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    R = torch.eye(64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA device"):
        ck.ck_rotate_quant(x, R, 64)
    with pytest.raises(ValueError, match="CUDA device"):
        ck.ck_unpack_w4(torch.zeros(4, 32, dtype=torch.int8), 64)


def grouped(L, **kw):
    a = dict(x=1 << 20, dt=ck.CK_BF16, M=4, K=64, sm=64, sk=1, R=1 << 20, g=16, a_scale=NULL,
             w=1 << 20, w_ld=32, w_scale=1 << 20, sdt=ck.CK_BF16, bias=NULL, G=2,
             gn=[8, 8], outs=[1 << 20, 1 << 21], ldos=[8, 8], odt=ck.CK_BF16, ws=1 << 20,
             ws_bytes=1 << 20)
    a.update(kw)
    G = len(a["gn"])
    gn = (ctypes.c_int64 * max(G, 1))(*a["gn"])
    outs = (ctypes.c_void_p * max(G, 1))(*a["outs"])
    ldos = (ctypes.c_int64 * max(G, 1))(*a["ldos"])
    return L.ck_w4a4_grouped_linear(a["x"], a["dt"], a["M"], a["K"], a["sm"], a["sk"], a["R"],
                                    a["g"], a["a_scale"], a["w"], a["w_ld"], a["w_scale"], a["sdt"],
                                    a["bias"], a["G"], gn, outs, ldos, a["odt"], a["ws"],
                                    a["ws_bytes"], None, None)


@pytest.mark.parametrize("bad", [dict(G=0), dict(G=9, gn=[1] * 9, outs=[1 << 20] * 9, ldos=[1] * 9),
                                 dict(gn=[8, -1]), dict(ldos=[8, 7]), dict(outs=[1 << 20, None]),
                                 dict(K=63), dict(g=8), dict(w_ld=31), dict(sdt=ck.CK_I8)])
def test_grouped_linear_rejects_on_host(L, bad):
    assert grouped(L, **bad) == ck.CK_ERR_INVALID_ARG


def test_grouped_linear_empty_group_and_empty_rows(L):
    # an empty group needs no output pointer; M = 0 is a no-op
    assert grouped(L, M=0, x=NULL, outs=[None, None], ws=NULL, ws_bytes=0) == ck.CK_OK
    assert grouped(L, gn=[0, 0], outs=[None, None], ldos=[0, 0], ws=NULL, ws_bytes=0) == ck.CK_OK


def test_grouped_linear_missing_workspace(L):
    assert grouped(L, ws=NULL, ws_bytes=0) == ck.CK_ERR_WORKSPACE


def w8(L, **kw):
    a = dict(x=1 << 20, dt=ck.CK_BF16, M=4, K=64, sm=64, sk=1, R=1 << 20, g=16, a_scale=NULL,
             w=1 << 20, N=8, w_ld=64, w_scale=1 << 20, sdt=ck.CK_BF16, bias=NULL, out=1 << 20,
             odt=ck.CK_BF16, ldo=8, ws=1 << 20, ws_bytes=1 << 20)
    a.update(kw)
    return L.ck_w8a8_linear(a["x"], a["dt"], a["M"], a["K"], a["sm"], a["sk"], a["R"], a["g"],
                            a["a_scale"], a["w"], a["N"], a["w_ld"], a["w_scale"], a["sdt"],
                            a["bias"], a["out"], a["odt"], a["ldo"], a["ws"], a["ws_bytes"],
                            None, None)


@pytest.mark.parametrize("bad", [dict(w_ld=63), dict(K=63), dict(g=8), dict(ldo=7), dict(out=NULL),
                                 dict(dt=ck.CK_I8, a_scale=NULL), dict(sdt=ck.CK_I8)])
def test_w8a8_linear_rejects_on_host(L, bad):
    assert w8(L, **bad) == ck.CK_ERR_INVALID_ARG


def test_w8a8_overflow_guard_is_the_int8_bound(L):
    """|acc| <= 128 * 128 * K: K = 131071 passes the guard, 131072 does not."""
    K = 131072
    assert w8(L, dt=ck.CK_I8, K=K, sm=K, w_ld=K, a_scale=1 << 20) == ck.CK_ERR_OVERFLOW
    assert w8(L, dt=ck.CK_I8, K=K - 2, sm=K, w_ld=K, a_scale=1 << 20, ws=NULL,
              ws_bytes=0) != ck.CK_ERR_OVERFLOW


def test_w8a8_workspace_sizes(L):
    assert L.ck_w8a8_linear_workspace_bytes(8192, 3840, 3840, 3840) == \
        ck.workspace_bytes(8192, 3840, 3840, 1920)
    # an unaligned INT8 weight pitch needs room for a 16-byte-pitched (N, K) copy
    assert L.ck_w8a8_linear_workspace_bytes(7, 5, 48, 50) >= \
        L.ck_w8a8_linear_workspace_bytes(7, 5, 48, 48) + 5 * 48
    assert L.ck_w8a8_linear_workspace_bytes(7, 5, 48, 47) == 0


def test_rotate_quant_int8_rejects_like_stage_1(L):
    assert L.ck_rotate_quant_int8(1 << 20, ck.CK_BF16, 4, 64, 64, 1, 1 << 20, 32, None, 1 << 20,
                                  64, 1 << 20, None, None) == ck.CK_ERR_INVALID_ARG


@pytest.mark.parametrize("bad", [dict(K=62, g=2), dict(K=63), dict(g=32), dict(ldp=31), dict(sr=2),
                                 dict(x=NULL), dict(p=NULL), dict(s=NULL), dict(dt=ck.CK_I8)])
def test_packed_quantizer_rejects_on_host(L, bad):
    a = dict(x=1 << 20, dt=ck.CK_BF16, M=4, K=64, g=16, sr=1, p=1 << 20, ldp=32, s=1 << 20)
    a.update(bad)
    assert L.ck_rotate_quant_packed(a["x"], a["dt"], a["M"], a["K"], a["K"], 1, 1 << 20, a["g"],
                                    None, a["sr"], 7, 0, a["p"], a["ldp"], a["s"], None) == \
        ck.CK_ERR_INVALID_ARG
