"""C-ABI contract of libfa.so, on the host only.

The library must load, export every function that include/fa.h declares, and reject bad
arguments synchronously, before any CUDA call (these tests run without a GPU and hand the
library fake, never-dereferenced pointers only on paths that are rejected on the host).
"""
import ctypes
import os
import re

import pytest

from io_aware_exact_22_b200 import fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")

OK, INVALID, UNSUPPORTED = 0, 1, 2
A16 = 0x10000  # a 16-byte aligned fake address (never dereferenced: every call below is rejected)


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    return fa.lib()


def test_library_exports_every_declared_function(L):
    names = declared_functions()
    assert set(names) == set(fa.EXPORTS)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code, name in fa.STATUS.items():
        assert fa.fa_status_string(code) == name
    assert fa.fa_status_string(99) == "FA_ERR_UNKNOWN"
    assert fa.fa_version() >= 100


def test_workspace_size():
    B, H, N, d = 2, 3, 100, 128
    rows = B * H * N
    tiles = B * H * ((N + 63) // 64)
    # per-tile statistics (rounded up to 256 bytes), the fp32 dQ accumulator, the work counter block
    assert fa.fa_bwd_workspace_bytes(B, H, N, d) == ((tiles * 512 + 255) // 256) * 256 + rows * d * 4 + 256
    assert fa.fa_bwd_workspace_bytes(0, 3, 100, 128) == 0
    assert fa.fa_bwd_workspace_bytes(1, 1, -1, 128) == 0


def _fwd(**kw):
    args = dict(q=A16, k=A16, v=A16, o=A16, lse=A16, B=1, H=1, N=128, d=64, scale=0.125,
                causal=0, stream=0)
    args.update(kw)
    return fa.fa_fwd(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"],
                     args["H"], args["N"], args["d"], args["scale"], args["causal"], args["stream"])


def _bwd(**kw):
    args = dict(q=A16, k=A16, v=A16, o=A16, dO=A16, lse=A16, dq=A16, dk=A16, dv=A16, ws=A16,
                wsb=1 << 40, B=1, H=1, N=128, d=128, scale=0.125, causal=1, stream=0)
    args.update(kw)
    return fa.fa_bwd(args["q"], args["k"], args["v"], args["o"], args["dO"], args["lse"],
                     args["dq"], args["dk"], args["dv"], args["ws"], args["wsb"], args["B"],
                     args["H"], args["N"], args["d"], args["scale"], args["causal"], args["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), INVALID), (dict(k=0), INVALID), (dict(v=0), INVALID), (dict(o=0), INVALID),
    (dict(lse=0), INVALID),
    (dict(q=A16 + 8), INVALID), (dict(v=A16 + 2), INVALID), (dict(o=A16 + 4), INVALID),
    (dict(lse=A16 + 2), INVALID),
    (dict(N=-1), INVALID), (dict(B=-2), INVALID), (dict(H=-1), INVALID),
    (dict(d=32), UNSUPPORTED), (dict(d=96), UNSUPPORTED), (dict(d=256), UNSUPPORTED),
    (dict(scale=0.0), INVALID), (dict(scale=-1.0), INVALID), (dict(scale=float("nan")), INVALID),
    (dict(scale=float("inf")), INVALID), (dict(causal=2), INVALID), (dict(causal=-1), INVALID),
    (dict(B=1 << 16, H=1 << 16), INVALID),
    (dict(B=1 << 15, H=1 << 15, N=1 << 20, d=128), INVALID),
])
def test_forward_rejects_bad_arguments(kw, code):
    assert _fwd(**kw) == code


@pytest.mark.parametrize("kw", [dict(N=0), dict(B=0), dict(H=0),
                                dict(N=0, q=0, k=0, v=0, o=0, lse=0)])
def test_forward_empty_problem_is_a_no_op(kw):
    assert _fwd(**kw) == OK


@pytest.mark.parametrize("kw,code", [
    (dict(dO=0), INVALID), (dict(ws=0), INVALID), (dict(dq=0), INVALID), (dict(lse=0), INVALID),
    (dict(ws=A16 + 16), INVALID), (dict(dk=A16 + 8), INVALID), (dict(dO=A16 + 2), INVALID),
    (dict(wsb=10), INVALID), (dict(d=32), UNSUPPORTED), (dict(d=80), UNSUPPORTED),
    (dict(d=256), UNSUPPORTED),
    (dict(N=-5), INVALID), (dict(scale=-0.1), INVALID), (dict(causal=3), INVALID),
])
def test_backward_rejects_bad_arguments(kw, code):
    assert _bwd(**kw) == code


def test_backward_workspace_must_cover_requirement():
    need = fa.fa_bwd_workspace_bytes(1, 1, 128, 128)
    assert _bwd(wsb=need - 1) == INVALID


@pytest.mark.parametrize("kw", [dict(N=0), dict(B=0, H=7)])
def test_backward_empty_problem_is_a_no_op(kw):
    assert _bwd(**kw) == OK


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(fa, "_lib", None)
    monkeypatch.setattr(fa, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        fa.lib()


def test_library_is_the_in_tree_build():
    path = fa.LIB_PATH
    assert os.path.dirname(os.path.abspath(path)) == os.path.join(ROOT, "io_aware_exact_22_b200")
    assert isinstance(fa.lib(), ctypes.CDLL)


def _bwd_main(**kw):
    args = dict(q=A16, k=A16, v=A16, dO=A16, ws=A16, wsb=1 << 40, dk=A16, dv=A16, B=1, H=1, N=128,
                d=128, scale=0.125, causal=1, stream=0)
    args.update(kw)
    return fa.fa_bwd_main(args["q"], args["k"], args["v"], args["dO"], args["ws"], args["wsb"],
                          args["dk"], args["dv"], args["B"], args["H"], args["N"], args["d"],
                          args["scale"], args["causal"], args["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), INVALID), (dict(dO=0), INVALID), (dict(ws=0), INVALID), (dict(dv=0), INVALID),
    (dict(ws=A16 + 16), INVALID), (dict(dk=A16 + 8), INVALID), (dict(wsb=10), INVALID),
    (dict(d=32), UNSUPPORTED), (dict(d=96), UNSUPPORTED), (dict(N=-1), INVALID),
    (dict(scale=0.0), INVALID), (dict(causal=2), INVALID),
])
def test_backward_main_rejects_bad_arguments(kw, code):
    assert _bwd_main(**kw) == code


@pytest.mark.parametrize("args,code", [
    ((0, 1 << 40, A16, 1, 1, 128, 128, 0.1), INVALID),
    ((A16, 1 << 40, 0, 1, 1, 128, 128, 0.1), INVALID),
    ((A16 + 16, 1 << 40, A16, 1, 1, 128, 128, 0.1), INVALID),
    ((A16, 1 << 40, A16 + 4, 1, 1, 128, 128, 0.1), INVALID),
    ((A16, 100, A16, 1, 1, 128, 128, 0.1), INVALID),
    ((A16, 1 << 40, A16, 1, 1, 128, 96, 0.1), UNSUPPORTED),
    ((A16, 1 << 40, A16, 1, 1, 128, 128, -1.0), INVALID),
    ((A16, 1 << 40, A16, 1, 1, 0, 128, 0.1), OK),
])
def test_backward_dq_post_rejects_bad_arguments(args, code):
    assert fa.fa_bwd_dq_post(*args, 0) == code


@pytest.mark.parametrize("kw,code", [
    (dict(flags=4), INVALID), (dict(flags=-1), INVALID), (dict(q=0), INVALID), (dict(o_part=0), INVALID),
    (dict(o=0), INVALID), (dict(lse=0), INVALID), (dict(o_part=A16 + 8), INVALID), (dict(o=A16 + 2), INVALID),
    (dict(d=96), UNSUPPORTED), (dict(N=-1), INVALID), (dict(scale=0.0), INVALID), (dict(N=0), OK),
])
def test_carry_rejects_bad_arguments(kw, code):
    args = dict(q=A16, k=A16, v=A16, o_part=A16, lse_part=A16, o=A16, lse=A16, B=1, H=1, N=128, d=128,
                scale=0.125, causal=0, flags=fa.FA_CARRY_IN | fa.FA_CARRY_FINAL)
    args.update(kw)
    assert fa.fa_fwd_carry(args["q"], args["k"], args["v"], args["o_part"], args["lse_part"], args["o"],
                           args["lse"], args["B"], args["H"], args["N"], args["d"], args["scale"], args["causal"],
                           args["flags"], 0) == code

