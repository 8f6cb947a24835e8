"""CPU-only checks of the C ABI boundary: the library loads, exports every entry point the
header declares, and rejects invalid arguments before touching the GPU."""

from __future__ import annotations

import ctypes
import os
import re

import pytest

import exact_attention_111_b200 as fa
from exact_attention_111_b200 import build as fabuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


@pytest.fixture(scope="module")
def L():
    fabuild.build()
    return fa.lib()


def declared_functions():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(fa_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("fa_fwd", "fa_bwd", "fa_fwd_ex", "fa_bwd_ex", "fa_bwd_workspace_bytes",
              "fa_check_status", "fa_status_string", "fa_last_launch_count"):
        assert n in names, n


def test_library_exports_every_declared_symbol(L):
    for n in declared_functions():
        assert hasattr(L, n), f"libfa.so does not export {n}"


def test_status_strings(L):
    assert fa.fa_status_string(0) == "FA_OK"
    assert fa.fa_status_string(2) == "FA_ERR_UNSUPPORTED"
    assert fa.fa_status_string(99) == "FA_ERR_UNKNOWN"


def test_workspace_formula(L):
    # fp32 dQ accumulator + two fp32 vectors padded to whole 128-row tiles, 256-B aligned.
    def expect(B, H, N, d):
        a = lambda x: (x + 255) // 256 * 256
        Np = (N + 127) // 128 * 128
        return a(B * H * N * d * 4) + 2 * a(B * H * Np * 4)
    for shape in ((1, 1, 128, 64), (64, 16, 1024, 64), (1, 32, 16384, 128), (2, 3, 1000, 128), (1, 1, 1, 64)):
        assert fa.fa_bwd_workspace_bytes(*shape) == expect(*shape)
    assert fa.fa_bwd_workspace_bytes(1, 1, 128, 96) == 0
    assert fa.fa_bwd_workspace_bytes(0, 1, 128, 64) == 0


FAKE = 0x10000  # 16-byte aligned, never dereferenced: argument errors return first


def _fwd(L, **kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, H=1, N=128, d=64, scale=0.125,
                causal=0, mask=None, stream=None)
    args.update(kw)
    return L.fa_fwd(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"], args["H"],
                    args["N"], args["d"], args["scale"], args["causal"], args["mask"], args["stream"])


def test_fwd_argument_errors(L):
    assert _fwd(L, d=96) == fa.FA_ERR_UNSUPPORTED
    assert _fwd(L, d=256) == fa.FA_ERR_UNSUPPORTED
    assert _fwd(L, N=0) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, B=0) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, H=-1) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, q=None) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, lse=None) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, k=FAKE + 8) == fa.FA_ERR_INVALID_ARG       # not 16-byte aligned
    assert _fwd(L, scale=0.0) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, scale=float("nan")) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, N=2048 * 128 + 1) == fa.FA_ERR_UNSUPPORTED


def test_fwd_ex_dtype_error(L):
    a = fa.FwdArgs(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0.125, 0, None, 7, 0, None, None)
    assert L.fa_fwd_ex(ctypes.byref(a)) == fa.FA_ERR_UNSUPPORTED
    assert L.fa_fwd_ex(None) == fa.FA_ERR_INVALID_ARG


def test_bwd_argument_errors(L):
    ws = fa.fa_bwd_workspace_bytes(1, 1, 128, 64)

    def call(**kw):
        a = dict(ptr=FAKE, d=64, N=128, ws=0x100000, wsb=ws)
        a.update(kw)
        p = a["ptr"]
        return L.fa_bwd(p, p, p, p, p, p, p, p, p, 1, 1, a["N"], a["d"], 0.125, 0, None,
                        a["ws"], a["wsb"], None)
    assert call(d=80) == fa.FA_ERR_UNSUPPORTED
    assert call(N=0) == fa.FA_ERR_INVALID_ARG
    assert call(ptr=None) == fa.FA_ERR_INVALID_ARG
    assert call(wsb=ws - 1) == fa.FA_ERR_WORKSPACE
    assert call(ws=None) == fa.FA_ERR_WORKSPACE
    assert call(ws=0x100000 + 16) == fa.FA_ERR_WORKSPACE     # not 256-byte aligned


def test_valid_call_without_gpu_reports_cuda_error(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _fwd(L) == fa.FA_ERR_CUDA


def test_python_binding_raises(L):
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 96, 0.125, False, None, stream=0)
    assert e.value.code == fa.FA_ERR_UNSUPPORTED
