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


# ----------------------------------------------------------------------------------------
# Split-KV forward, forward over a key slice, LSE merge
# ----------------------------------------------------------------------------------------

def test_splitkv_symbols_declared():
    names = declared_functions()
    for n in ("fa_fwd_partial", "fa_lse_merge", "fa_fwd_splitkv", "fa_fwd_splitkv_workspace_bytes",
              "fa_splitkv_choose"):
        assert n in names, n


def test_splitkv_workspace_formula(L):
    a = lambda x: (x + 255) // 256 * 256
    for B, H, N, d, S in ((1, 1, 16384, 128, 2), (2, 3, 1000, 64, 5), (1, 1, 1, 64, 1), (4, 2, 777, 128, 64)):
        rows = B * H * N
        assert fa.fa_fwd_splitkv_workspace_bytes(B, H, N, d, S) == S * (a(rows * d * 4) + a(rows * 4))
    assert fa.fa_fwd_splitkv_workspace_bytes(1, 1, 128, 64, 0) == 0
    assert fa.fa_fwd_splitkv_workspace_bytes(1, 1, 128, 64, 65) == 0
    assert fa.fa_fwd_splitkv_workspace_bytes(1, 1, 128, 96, 2) == 0


def _choose_model(B, H, N, causal, sms):
    """The documented rule, restated: minimise waves x (tiles per range + 2), causal CTAs
    counting half, ranges of >= 4 tiles, a larger count winning only by 10 %."""
    T = -(-N // 128)
    units = B * H * -(-T // 2)
    best, best_cost = 1, None
    for S in range(1, 65):
        sp = -(-T // S)
        if S > 1 and sp < 4:
            break
        s_eff = -(-T // sp)
        if s_eff < S:
            continue
        load = units * s_eff // (2 if causal else 1)
        cost = max(1, -(-load // sms)) * (sp + 2)
        if best_cost is None or 10 * cost < 9 * best_cost:
            best, best_cost = S, cost
    return best


def test_splitkv_choose(L):
    # one head of 16k keys leaves most SMs idle: two ranges; a full GPU takes none
    assert fa.fa_splitkv_choose(1, 1, 16384, False, 148) == 2
    assert fa.fa_splitkv_choose(64, 16, 1024, False, 148) == 1
    assert fa.fa_splitkv_choose(4, 32, 4096, True, 148) == 1
    for B, H, N, causal in ((1, 1, 4096, False), (1, 1, 16384, True), (2, 1, 8192, False),
                            (1, 3, 30000, True), (1, 2, 16384, False), (3, 5, 300, False)):
        for sms in (148, 132, 20):
            got = fa.fa_splitkv_choose(B, H, N, causal, sms)
            assert got == _choose_model(B, H, N, causal, sms), (B, H, N, causal, sms)
            T = -(-N // 128)
            assert 1 <= got <= 64 and (got == 1 or -(-T // got) >= 4)
    assert fa.fa_splitkv_choose(0, 1, 128, False, 148) == 0
    assert fa.fa_splitkv_choose(1, 1, 128, False, 0) == 0


def test_splitkv_argument_errors(L):
    ws = fa.fa_fwd_splitkv_workspace_bytes(1, 1, 1024, 64, 4)

    def call(S=4, wsp=0x100000, wsb=ws, d=64, ptr=FAKE):
        return L.fa_fwd_splitkv(ptr, ptr, ptr, ptr, ptr, 1, 1, 1024, d, 0.125, 0, None, S, wsp, wsb, None)
    assert call(S=0) == fa.FA_ERR_INVALID_ARG
    assert call(S=65) == fa.FA_ERR_INVALID_ARG
    assert call(d=96) == fa.FA_ERR_UNSUPPORTED
    assert call(ptr=None) == fa.FA_ERR_INVALID_ARG
    assert call(wsb=ws - 1) == fa.FA_ERR_WORKSPACE
    assert call(wsp=None) == fa.FA_ERR_WORKSPACE
    assert call(wsp=0x100000 + 64) == fa.FA_ERR_WORKSPACE


def test_partial_argument_errors(L):
    def call(**kw):
        a = dict(N=1024, Nk=256, key_offset=256, causal=0, mask=None, d=64, dtype=fa.FA_BF16, k=FAKE)
        a.update(kw)
        args = fa.PartialArgs(FAKE, a["k"], FAKE, FAKE, FAKE, 1, 1, a["N"], a["Nk"], a["d"], a["key_offset"],
                              0.125, a["causal"], a["mask"], a["dtype"], None)
        return L.fa_fwd_partial(ctypes.byref(args))
    assert call(key_offset=100) == fa.FA_ERR_INVALID_ARG        # not a multiple of 128
    assert call(key_offset=-128) == fa.FA_ERR_INVALID_ARG
    assert call(Nk=0) == fa.FA_ERR_INVALID_ARG
    assert call(causal=1, key_offset=896) == fa.FA_ERR_INVALID_ARG   # keys past the sequence
    assert call(mask=FAKE, key_offset=896) == fa.FA_ERR_INVALID_ARG
    assert call(d=80) == fa.FA_ERR_UNSUPPORTED
    assert call(dtype=2) == fa.FA_ERR_UNSUPPORTED                # fp32 inputs are not accepted
    assert call(k=FAKE + 4) == fa.FA_ERR_INVALID_ARG
    assert call(Nk=2048 * 128 + 1) == fa.FA_ERR_UNSUPPORTED
    assert L.fa_fwd_partial(None) == fa.FA_ERR_INVALID_ARG


def test_merge_argument_errors(L):
    def call(n=2, d=64, out=fa.FA_BF16, parts=None, o=FAKE):
        ps = parts if parts is not None else [FAKE] * max(n, 1)
        arr = (ctypes.c_void_p * len(ps))(*ps)
        return L.fa_lse_merge(arr, arr, n, o, FAKE, 1, 1, 128, d, out, None)
    assert call(n=0) == fa.FA_ERR_INVALID_ARG
    assert call(n=65, parts=[FAKE] * 65) == fa.FA_ERR_INVALID_ARG
    assert call(d=96) == fa.FA_ERR_UNSUPPORTED
    assert call(out=3) == fa.FA_ERR_UNSUPPORTED
    assert call(parts=[FAKE, None]) == fa.FA_ERR_INVALID_ARG
    assert call(parts=[FAKE, FAKE + 4]) == fa.FA_ERR_INVALID_ARG   # O part not 16-byte aligned
    assert call(o=None) == fa.FA_ERR_INVALID_ARG


def test_deterministic_workspace_formula(L):
    # int64 accumulator over whole 128-row tiles, then the two fp32 row vectors
    a = lambda x: (x + 255) // 256 * 256
    for B, H, N, d in ((1, 1, 128, 64), (64, 16, 1024, 64), (2, 3, 1000, 128), (1, 1, 1, 64)):
        Np = (N + 127) // 128 * 128
        assert fa.fa_bwd_workspace_bytes_ex(B, H, N, d, True) == a(B * H * Np * d * 8) + 2 * a(B * H * Np * 4)
        assert fa.fa_bwd_workspace_bytes_ex(B, H, N, d, False) == fa.fa_bwd_workspace_bytes(B, H, N, d)
    assert fa.fa_bwd_workspace_bytes_ex(1, 1, 128, 96, True) == 0


def test_deterministic_needs_its_workspace(L):
    import ctypes as ct
    ws_det = fa.fa_bwd_workspace_bytes_ex(1, 1, 1000, 64, True)
    ws = fa.fa_bwd_workspace_bytes(1, 1, 1000, 64)
    p = FAKE
    a = fa.BwdArgs(p, p, p, p, p, p, p, p, p, 1, 1, 1000, 64, 0.125, 0, None, fa.FA_BF16, None,
                   0x100000, ws_det - 1, None, None, None, 1)
    assert L.fa_bwd_ex(ct.byref(a)) == fa.FA_ERR_WORKSPACE
    assert ws < ws_det
    assert fa.fa_status_string(fa.FA_ERR_RANGE) == "FA_ERR_RANGE"


def test_dropout_argument_errors(L):
    import ctypes as ct
    for p in (1.0, -0.1, float("nan"), 2.0):
        a = fa.FwdArgs(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0.125, 0, None, fa.FA_BF16, 0, None, None, p, 1)
        assert L.fa_fwd_ex(ct.byref(a)) == fa.FA_ERR_INVALID_ARG, p
        ws = fa.fa_bwd_workspace_bytes(1, 1, 128, 64)
        b = fa.BwdArgs(*([FAKE] * 9), 1, 1, 128, 64, 0.125, 0, None, fa.FA_BF16, None, 0x100000, ws, None, None, None,
                       0, p, 1)
        assert L.fa_bwd_ex(ct.byref(b)) == fa.FA_ERR_INVALID_ARG, p


def test_fp8_workspace_and_argument_errors(L):
    import ctypes as ct
    for B, H, N in ((1, 1, 128), (2, 3, 1000), (1, 1, 1)):
        Np = (N + 127) // 128 * 128
        assert fa.fa_fwd_fp8_workspace_bytes(B, H, N, 128) == (B * H * 128 * Np + 255) // 256 * 256
    assert fa.fa_fwd_fp8_workspace_bytes(1, 1, 128, 64) == 0
    ws = fa.fa_fwd_fp8_workspace_bytes(1, 1, 256, 128)

    def call(**kw):
        a = dict(d=128, dq=0.5, dk=0.5, dv=0.5, q=FAKE, ws=0x100000, wsb=ws, N=256)
        a.update(kw)
        args = fa.Fp8Args(a["q"], FAKE, FAKE, a["dq"], a["dk"], a["dv"], FAKE, FAKE, 1, 1, a["N"], a["d"], 0.088,
                          0, None, 0, a["ws"], a["wsb"], None)
        return L.fa_fwd_fp8(ct.byref(args))
    assert call(d=64) == fa.FA_ERR_UNSUPPORTED
    assert call(dq=0.0) == fa.FA_ERR_INVALID_ARG
    assert call(dv=float("inf")) == fa.FA_ERR_INVALID_ARG
    assert call(dk=float("nan")) == fa.FA_ERR_INVALID_ARG
    assert call(q=FAKE + 8) == fa.FA_ERR_INVALID_ARG
    assert call(wsb=ws - 1) == fa.FA_ERR_WORKSPACE
    assert call(ws=0x100000 + 128) == fa.FA_ERR_WORKSPACE
    assert L.fa_fwd_fp8(None) == fa.FA_ERR_INVALID_ARG


def test_selftest_argument_errors(L):
    assert L.fa_selftest_wait_timeout(0, None, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_selftest_wait_timeout(1000001, None, None) == fa.FA_ERR_INVALID_ARG


def test_noalloc_argument_errors_come_first(L):
    """fa_bwd_noalloc reports fa_bwd's argument errors before any CUDA call (so also on a
    host with no GPU), and refuses shapes whose workspace exceeds its fixed array."""
    def call(ptr=FAKE, B=1, H=1, N=128, d=64, scale=0.125, lse=None):
        p = ptr
        return L.fa_bwd_noalloc(p, p, p, p, p if lse is None else lse, p, p, p, p, B, H, N, d,
                                ctypes.c_float(scale), 0, None, None)
    assert call(ptr=None) == fa.FA_ERR_INVALID_ARG
    assert call(ptr=FAKE + 8) == fa.FA_ERR_INVALID_ARG
    assert call(N=0) == fa.FA_ERR_INVALID_ARG
    assert call(scale=0.0) == fa.FA_ERR_INVALID_ARG
    assert call(d=96) == fa.FA_ERR_UNSUPPORTED
    # an oversized shape with NULL pointers is an argument error, as in fa_bwd
    assert call(ptr=None, B=64, H=16, N=16384, d=128) == fa.FA_ERR_INVALID_ARG
    # valid pointers but a workspace beyond the 64 MiB array: refused, nothing launched
    assert fa.fa_bwd_workspace_bytes(64, 16, 16384, 128) > 64 << 20
    assert call(B=64, H=16, N=16384, d=128) == fa.FA_ERR_WORKSPACE


def test_device_status_codes_are_disjoint_from_public_codes():
    """The kernels' status-word codes (csrc/fa_internal.h) share no value with the public
    fa_status codes (include/fa.h), and fa_check_status translates each one by name."""
    hdr = open(os.path.join(ROOT, "include", "fa.h")).read()
    public = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(FA_(?:OK|ERR_\w+))\s*=\s*(\d+)", hdr)}
    assert public["FA_ERR_RANGE"] == 6 and public["FA_ERR_TIMEOUT"] == 4
    internal = open(os.path.join(ROOT, "exact_attention_111_b200", "csrc", "fa_internal.h")).read()
    m = re.search(r"enum\s*:\s*int\s*\{([^}]*kDevTimeout[^}]*)\}", internal)
    dev = {k: int(v, 0) for k, v in re.findall(r"(kDev\w+)\s*=\s*(0x[0-9a-fA-F]+|\d+)", m.group(1))}
    assert dev["kDevOk"] == 0
    nonzero = {k: v for k, v in dev.items() if k != "kDevOk"}
    assert not set(nonzero.values()) & set(public.values())
    host = open(os.path.join(ROOT, "exact_attention_111_b200", "csrc", "fa_host.cu")).read()
    body = re.search(r"int status_from_device_word\(int v\) \{(.*?)\n\}", host, flags=re.S).group(1)
    assert "case kDevTimeout: return FA_ERR_TIMEOUT;" in body
    assert "case kDevRange: return FA_ERR_RANGE;" in body
    assert "default: return FA_ERR_CUDA;" in body          # kDevBadState and anything else
    assert "return status_from_device_word(v);" in host


def test_split_backward_workspace_and_arguments(L):
    """Query-range splits: the workspace adds two fp32 [B, H, N, d] accumulators; S <= 1 is the
    plain layout; S outside [0, 64] and S >= 2 with the deterministic mode are refused."""
    a = lambda x: (x + 255) // 256 * 256
    for B, H, N, d in ((1, 1, 16384, 128), (2, 3, 1000, 64)):
        base = fa.fa_bwd_workspace_bytes(B, H, N, d)
        assert fa.fa_bwd_workspace_bytes_split(B, H, N, d, 0) == base
        assert fa.fa_bwd_workspace_bytes_split(B, H, N, d, 1) == base
        assert fa.fa_bwd_workspace_bytes_split(B, H, N, d, 3) == base + 2 * a(B * H * N * d * 4)
    assert fa.fa_bwd_workspace_bytes_split(1, 1, 128, 64, 65) == 0
    ws = fa.fa_bwd_workspace_bytes_split(1, 1, 128, 64, 2)

    def call(splits, det=0, wsb=ws):
        b = fa.BwdArgs(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0.125, 0, None,
                       fa.FA_BF16, None, 0x100000, wsb, None, None, None, det, 0.0, 0, splits)
        return L.fa_bwd_ex(ctypes.byref(b))
    assert call(-1) == fa.FA_ERR_INVALID_ARG
    assert call(65) == fa.FA_ERR_INVALID_ARG
    assert call(2, det=1, wsb=1 << 30) == fa.FA_ERR_UNSUPPORTED
    assert call(2, wsb=ws - 1) == fa.FA_ERR_WORKSPACE


def splitq_choose_reference(B, H, N, causal, sms):
    """The choice restated: minimise the finishing time (whole waves of equal ranges without a
    causal mask, else max(longest range, average tile pairs per SM)) + 2 per wave of non-empty
    CTAs over S = 1 .. 64 with at least 4 steps per range; a larger S must win by 10 %."""
    T = -(-N // 128)
    total = B * H * (T * (T + 1) // 2 if causal else T * T)
    avg = -(-total // sms)
    best, best_cost = 1, None
    for S in range(1, 65):
        chunk = -(-T // S)
        if S > 1 and chunk < 4:
            break
        s_eff = -(-T // chunk)
        if s_eff < S:
            continue
        ctas = B * H * sum((T - s * chunk) if causal else T for s in range(s_eff))
        waves = -(-ctas // sms)
        cost = (max(chunk, avg) if causal else waves * chunk) + 2 * waves
        if best_cost is None or 10 * cost < 9 * best_cost:
            best, best_cost = S, cost
    return best


def test_split_backward_choice(L):
    assert fa.fa_bwd_splitq_choose(1, 1, 16384, True, 148) == 3
    assert fa.fa_bwd_splitq_choose(1, 1, 16384, False, 148) == 1     # 128 equal CTAs: one wave already
    assert fa.fa_bwd_splitq_choose(1, 32, 16384, True, 148) == 1     # the long-context batch fills the GPU
    assert fa.fa_bwd_splitq_choose(64, 16, 1024, False, 148) == 1
    assert fa.fa_bwd_splitq_choose(0, 1, 128, False, 148) == 0
    for B, H, N, causal in ((1, 1, 16384, True), (1, 2, 8192, True), (2, 1, 4096, False), (1, 1, 1000, True),
                            (1, 4, 32768, True), (3, 5, 777, False)):
        assert fa.fa_bwd_splitq_choose(B, H, N, causal, 148) == splitq_choose_reference(B, H, N, causal, 148)
