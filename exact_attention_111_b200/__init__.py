"""Fused exact attention for B200 (sm_100a): the Python binding of libfa.so.

The binding marshals arguments only; every step of the computation runs in the CUDA
kernels behind the C ABI of ``include/fa.h``.  The C entry points are mirrored one to one
(``fa_fwd``, ``fa_bwd``, ``fa_fwd_ex``, ``fa_bwd_ex``, ``fa_bwd_workspace_bytes``,
``fa_bwd_workspace_bytes_ex``, ``fa_bwd_workspace_bytes_split``, ``fa_bwd_splitq_choose``, ``fa_bwd_noalloc``, ``fa_fwd_partial``, ``fa_lse_merge``, ``fa_fwd_splitkv``,
``fa_fwd_splitkv_workspace_bytes``, ``fa_splitkv_choose``, ``fa_fwd_fp8``, ``fa_fwd_fp8_workspace_bytes``, ``fa_selftest_wait_timeout``, ``fa_selftest_exp2_poly``, ``fa_check_status``,
``fa_status_string``, ``fa_last_launch_count``); they take torch tensors (or raw device
addresses as ints).  ``attention_forward`` / ``attention_backward`` /
``attention_forward_splitkv`` / ``attention_forward_partial`` / ``lse_merge`` and
``FlashAttention`` add output allocation with torch on top.

There is no fallback: if ``libfa.so`` is missing or a call fails, an exception is raised.
"""

from __future__ import annotations

import ctypes
import os

__all__ = [
    "FAError", "fa_fwd", "fa_bwd", "fa_fwd_ex", "fa_bwd_ex", "fa_bwd_workspace_bytes",
    "fa_check_status", "fa_status_string", "fa_last_launch_count", "fa_bwd_noalloc", "lib", "library_path",
    "attention_forward", "attention_backward", "FlashAttention", "FA_BF16", "FA_FP16", "FA_FP32",
    "fa_fwd_partial", "fa_lse_merge", "fa_fwd_splitkv", "fa_fwd_splitkv_workspace_bytes",
    "fa_splitkv_choose", "attention_forward_splitkv", "attention_forward_partial", "lse_merge",
    "FA_MAX_PARTS", "fa_bwd_workspace_bytes_ex", "fa_bwd_workspace_bytes_split", "fa_bwd_splitq_choose", "FA_ERR_RANGE", "fa_fwd_fp8", "fa_fwd_fp8_workspace_bytes",
    "attention_forward_fp8", "fa_selftest_wait_timeout", "fa_selftest_exp2_poly",
]

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT, FA_ERR_WORKSPACE, FA_ERR_RANGE = range(7)
FA_BF16, FA_FP16, FA_FP32 = 0, 1, 2
TILE = 128
FA_MAX_PARTS = 64

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libfa.so")
_lib = None

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float


class FwdArgs(ctypes.Structure):
    """Mirror of fa_fwd_args."""
    _fields_ = [("q", _vp), ("k", _vp), ("v", _vp), ("o", _vp), ("lse", _vp),
                ("B", _i), ("H", _i), ("N", _i), ("d", _i), ("scale", _f), ("causal", _i),
                ("blockmask", _vp), ("dtype", _i), ("o_fp32", _i), ("visit_log", _vp),
                ("stream", _vp), ("dropout_p", _f), ("dropout_seed", ctypes.c_ulonglong)]


class BwdArgs(ctypes.Structure):
    """Mirror of fa_bwd_args."""
    _fields_ = [("q", _vp), ("k", _vp), ("v", _vp), ("o", _vp), ("lse", _vp), ("dout", _vp),
                ("dq", _vp), ("dk", _vp), ("dv", _vp),
                ("B", _i), ("H", _i), ("N", _i), ("d", _i), ("scale", _f), ("causal", _i),
                ("blockmask", _vp), ("dtype", _i), ("visit_log", _vp),
                ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t), ("stream", _vp),
                ("main_start_event", _vp), ("main_stop_event", _vp), ("deterministic", _i),
                ("dropout_p", _f), ("dropout_seed", ctypes.c_ulonglong), ("query_splits", _i)]


class PartialArgs(ctypes.Structure):
    """Mirror of fa_fwd_partial_args."""
    _fields_ = [("q", _vp), ("k", _vp), ("v", _vp), ("o_part", _vp), ("lse_part", _vp),
                ("B", _i), ("H", _i), ("N", _i), ("Nk", _i), ("d", _i), ("key_offset", _i),
                ("scale", _f), ("causal", _i), ("blockmask", _vp), ("dtype", _i), ("stream", _vp)]


class Fp8Args(ctypes.Structure):
    """Mirror of fa_fwd_fp8_args."""
    _fields_ = [("q", _vp), ("k", _vp), ("v", _vp), ("descale_q", _f), ("descale_k", _f), ("descale_v", _f),
                ("o", _vp), ("lse", _vp), ("B", _i), ("H", _i), ("N", _i), ("d", _i), ("scale", _f),
                ("causal", _i), ("blockmask", _vp), ("o_fp32", _i), ("workspace", _vp),
                ("workspace_bytes", ctypes.c_size_t), ("stream", _vp)]


class FAError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {fa_status_string(code)} ({code})")
        self.code = code


def lib() -> ctypes.CDLL:
    """Load libfa.so (built in-tree by exact_attention_111_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise RuntimeError(f"{library_path} is not built; run `python -m exact_attention_111_b200.build`")
    L = ctypes.CDLL(library_path)
    L.fa_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _vp]
    L.fa_fwd.restype = _i
    L.fa_bwd.argtypes = [_vp] * 9 + [_i, _i, _i, _i, _f, _i, _vp, _vp, ctypes.c_size_t, _vp]
    L.fa_bwd.restype = _i
    L.fa_fwd_ex.argtypes = [ctypes.POINTER(FwdArgs)]
    L.fa_fwd_ex.restype = _i
    L.fa_bwd_ex.argtypes = [ctypes.POINTER(BwdArgs)]
    L.fa_bwd_ex.restype = _i
    L.fa_bwd_workspace_bytes.argtypes = [_i, _i, _i, _i]
    L.fa_bwd_workspace_bytes.restype = ctypes.c_size_t
    L.fa_bwd_workspace_bytes_ex.argtypes = [_i, _i, _i, _i, _i]
    L.fa_bwd_workspace_bytes_ex.restype = ctypes.c_size_t
    L.fa_bwd_workspace_bytes_split.argtypes = [_i, _i, _i, _i, _i]
    L.fa_bwd_workspace_bytes_split.restype = ctypes.c_size_t
    L.fa_bwd_splitq_choose.argtypes = [_i, _i, _i, _i, _i]
    L.fa_bwd_splitq_choose.restype = _i
    L.fa_check_status.argtypes = [_vp]
    L.fa_check_status.restype = _i
    L.fa_status_string.argtypes = [_i]
    L.fa_status_string.restype = ctypes.c_char_p
    L.fa_bwd_noalloc.argtypes = [_vp] * 9 + [_i, _i, _i, _i, _f, _i, _vp, _vp]
    L.fa_bwd_noalloc.restype = _i
    L.fa_last_launch_count.argtypes = []
    L.fa_last_launch_count.restype = _i
    L.fa_fwd_partial.argtypes = [ctypes.POINTER(PartialArgs)]
    L.fa_fwd_partial.restype = _i
    L.fa_lse_merge.argtypes = [ctypes.POINTER(_vp), ctypes.POINTER(_vp), _i, _vp, _vp, _i, _i, _i, _i, _i, _vp]
    L.fa_lse_merge.restype = _i
    L.fa_fwd_splitkv.argtypes = [_vp] * 5 + [_i, _i, _i, _i, _f, _i, _vp, _i, _vp, ctypes.c_size_t, _vp]
    L.fa_fwd_splitkv.restype = _i
    L.fa_fwd_splitkv_workspace_bytes.argtypes = [_i, _i, _i, _i, _i]
    L.fa_fwd_splitkv_workspace_bytes.restype = ctypes.c_size_t
    L.fa_splitkv_choose.argtypes = [_i, _i, _i, _i, _i]
    L.fa_splitkv_choose.restype = _i
    L.fa_fwd_fp8.argtypes = [ctypes.POINTER(Fp8Args)]
    L.fa_fwd_fp8.restype = _i
    L.fa_fwd_fp8_workspace_bytes.argtypes = [_i, _i, _i, _i]
    L.fa_fwd_fp8_workspace_bytes.restype = ctypes.c_size_t
    L.fa_selftest_wait_timeout.argtypes = [ctypes.c_uint, _vp, _vp]
    L.fa_selftest_wait_timeout.restype = _i
    L.fa_selftest_exp2_poly.argtypes = [_vp, _vp, _i, _vp]
    L.fa_selftest_exp2_poly.restype = _i
    _lib = L
    return L


def _ptr(x):
    """Device address of a tensor (or None / int passed through)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, what: str):
    if rc != FA_OK:
        raise FAError(rc, what)


def fa_status_string(code: int) -> str:
    return lib().fa_status_string(code).decode()


def fa_last_launch_count() -> int:
    return lib().fa_last_launch_count()


def fa_bwd_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return lib().fa_bwd_workspace_bytes(B, H, N, d)


def fa_bwd_workspace_bytes_ex(B: int, H: int, N: int, d: int, deterministic: bool) -> int:
    return lib().fa_bwd_workspace_bytes_ex(B, H, N, d, int(bool(deterministic)))


def fa_bwd_workspace_bytes_split(B: int, H: int, N: int, d: int, query_splits: int) -> int:
    return lib().fa_bwd_workspace_bytes_split(B, H, N, d, int(query_splits))


def fa_bwd_splitq_choose(B: int, H: int, N: int, causal: bool, num_sms: int) -> int:
    return lib().fa_bwd_splitq_choose(B, H, N, int(bool(causal)), num_sms)


def fa_check_status(stream=None):
    _check(lib().fa_check_status(_stream(stream)), "fa_check_status")


def fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, blockmask, stream=None):
    _check(lib().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, scale,
                        int(bool(causal)), _ptr(blockmask), _stream(stream)), "fa_fwd")


def fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, blockmask,
           workspace, workspace_bytes, stream=None):
    _check(lib().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq),
                        _ptr(dk), _ptr(dv), B, H, N, d, scale, int(bool(causal)), _ptr(blockmask),
                        _ptr(workspace), workspace_bytes, _stream(stream)), "fa_bwd")


def fa_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, blockmask,
                   stream=None):
    """fa_bwd without a workspace argument, for callers that cannot allocate device memory
    at call time; uses the library's fixed 64 MiB per-device scratch (see include/fa.h)."""
    _check(lib().fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq),
                                _ptr(dk), _ptr(dv), B, H, N, d, scale, int(bool(causal)),
                                _ptr(blockmask), _stream(stream)), "fa_bwd_noalloc")


def fa_fwd_ex(q, k, v, o, lse, B, H, N, d, scale, causal=False, blockmask=None, dtype=FA_BF16,
              o_fp32=False, visit_log=None, stream=None, dropout_p=0.0, dropout_seed=0):
    a = FwdArgs(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, scale, int(bool(causal)),
                _ptr(blockmask), dtype, int(bool(o_fp32)), _ptr(visit_log), _stream(stream),
                float(dropout_p), int(dropout_seed))
    _check(lib().fa_fwd_ex(ctypes.byref(a)), "fa_fwd_ex")


def fa_fwd_partial(q, k, v, o_part, lse_part, B, H, N, Nk, d, key_offset, scale, causal=False,
                   blockmask=None, dtype=FA_BF16, stream=None):
    a = PartialArgs(_ptr(q), _ptr(k), _ptr(v), _ptr(o_part), _ptr(lse_part), B, H, N, Nk, d, key_offset,
                    scale, int(bool(causal)), _ptr(blockmask), dtype, _stream(stream))
    _check(lib().fa_fwd_partial(ctypes.byref(a)), "fa_fwd_partial")


def fa_lse_merge(o_parts, lse_parts, o, lse, B, H, N, d, out_dtype=FA_BF16, stream=None):
    """o_parts / lse_parts: sequences of device tensors (or addresses), one per part."""
    n = len(o_parts)
    if len(lse_parts) != n:
        raise ValueError("o_parts and lse_parts differ in length")
    po = (_vp * max(n, 1))(*[_ptr(x) for x in o_parts])
    pl = (_vp * max(n, 1))(*[_ptr(x) for x in lse_parts])
    _check(lib().fa_lse_merge(po, pl, n, _ptr(o), _ptr(lse), B, H, N, d, out_dtype, _stream(stream)),
           "fa_lse_merge")


def fa_fwd_splitkv_workspace_bytes(B: int, H: int, N: int, d: int, num_splits: int) -> int:
    return lib().fa_fwd_splitkv_workspace_bytes(B, H, N, d, num_splits)


def fa_splitkv_choose(B: int, H: int, N: int, causal: bool, num_sms: int) -> int:
    return lib().fa_splitkv_choose(B, H, N, int(bool(causal)), num_sms)


def fa_fwd_splitkv(q, k, v, o, lse, B, H, N, d, scale, causal, blockmask, num_splits, workspace,
                   workspace_bytes, stream=None):
    _check(lib().fa_fwd_splitkv(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, scale,
                                int(bool(causal)), _ptr(blockmask), num_splits, _ptr(workspace),
                                workspace_bytes, _stream(stream)), "fa_fwd_splitkv")


def fa_selftest_wait_timeout(limit_us: int, waited_ok=None, stream=None):
    """Runs the bounded-wait diagnostic (include/fa.h); fa_check_status then reports
    FA_ERR_TIMEOUT."""
    _check(lib().fa_selftest_wait_timeout(int(limit_us), _ptr(waited_ok), _stream(stream)), "fa_selftest_wait_timeout")


def fa_selftest_exp2_poly(x, y, n: int, stream=None):
    """y[:n] = 2^x[:n] by the kernels' FMA-pipe polynomial (the diagnostic of include/fa.h)."""
    _check(lib().fa_selftest_exp2_poly(_ptr(x), _ptr(y), int(n), _stream(stream)), "fa_selftest_exp2_poly")


def fa_fwd_fp8_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return lib().fa_fwd_fp8_workspace_bytes(B, H, N, d)


def fa_fwd_fp8(q8, k8, v8, descale_q, descale_k, descale_v, o, lse, B, H, N, d, scale, causal=False,
               blockmask=None, o_fp32=False, workspace=None, workspace_bytes=0, stream=None):
    a = Fp8Args(_ptr(q8), _ptr(k8), _ptr(v8), float(descale_q), float(descale_k), float(descale_v), _ptr(o),
                _ptr(lse), B, H, N, d, scale, int(bool(causal)), _ptr(blockmask), int(bool(o_fp32)),
                _ptr(workspace), workspace_bytes, _stream(stream))
    _check(lib().fa_fwd_fp8(ctypes.byref(a)), "fa_fwd_fp8")


def _event(e):
    if e is None or isinstance(e, int):
        return e
    return e.cuda_event  # torch.cuda.Event (created lazily by torch on first use)


def fa_bwd_ex(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal=False, blockmask=None,
              dtype=FA_BF16, visit_log=None, workspace=None, workspace_bytes=0, stream=None,
              main_start_event=None, main_stop_event=None, deterministic=False, dropout_p=0.0, dropout_seed=0,
              query_splits=0):
    a = BwdArgs(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                _ptr(dv), B, H, N, d, scale, int(bool(causal)), _ptr(blockmask), dtype,
                _ptr(visit_log), _ptr(workspace), workspace_bytes, _stream(stream),
                _event(main_start_event), _event(main_stop_event), int(bool(deterministic)),
                float(dropout_p), int(dropout_seed), int(query_splits))
    _check(lib().fa_bwd_ex(ctypes.byref(a)), "fa_bwd_ex")


# ----------------------------------------------------------------------------------------
# torch conveniences (allocation only; the arithmetic is in the kernels)
# ----------------------------------------------------------------------------------------

def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return FA_BF16
    if t.dtype == torch.float16:
        return FA_FP16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _check_qkv(*ts):
    for t in ts:
        if not (t.is_cuda and t.is_contiguous() and t.dim() == 4):
            raise ValueError("expected contiguous CUDA tensors of shape [B, H, N, d]")


def attention_forward(q, k, v, causal=False, blockmask=None, scale=None, o_fp32=False,
                      visit_log=None, stream=None, dropout_p=0.0, dropout_seed=0):
    """Returns (O, LSE) for [B, H, N, d] CUDA tensors (bf16 or fp16).  ``dropout_p`` > 0 drops
    probabilities with the Philox mask of ``dropout_seed`` (include/fa.h)."""
    import torch
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    scale = (1.0 / d ** 0.5) if scale is None else scale
    o = torch.empty(q.shape, dtype=torch.float32 if o_fp32 else q.dtype, device=q.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    fa_fwd_ex(q, k, v, o, lse, B, H, N, d, scale, causal, blockmask, _dtype_code(q), o_fp32,
              visit_log, stream, dropout_p=dropout_p, dropout_seed=dropout_seed)
    return o, lse


def attention_forward_splitkv(q, k, v, causal=False, blockmask=None, scale=None, num_splits=None,
                              workspace=None, stream=None):
    """fa_fwd_splitkv on bf16 [B, H, N, d] tensors.  ``num_splits=None`` takes
    fa_splitkv_choose for this GPU's SM count.  Returns (O, LSE, num_splits)."""
    import torch
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    scale = (1.0 / d ** 0.5) if scale is None else scale
    if num_splits is None:
        sms = torch.cuda.get_device_properties(q.device).multi_processor_count
        num_splits = fa_splitkv_choose(B, H, N, causal, sms)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    nbytes = fa_fwd_splitkv_workspace_bytes(B, H, N, d, num_splits)
    if workspace is None and num_splits > 1:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    fa_fwd_splitkv(q, k, v, o, lse, B, H, N, d, scale, causal, blockmask, num_splits, workspace,
                   0 if workspace is None else workspace.numel(), stream)
    return o, lse, num_splits


def attention_forward_partial(q, k, v, key_offset=0, causal=False, blockmask=None, scale=None,
                              stream=None):
    """Attention of all query rows of q [B, H, N, d] over the keys k, v [B, H, Nk, d] that sit
    at query-sequence positions key_offset.. (fa_fwd_partial).  Returns fp32 (O_part, LSE_part)."""
    import torch
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    Nk = k.shape[2]
    scale = (1.0 / d ** 0.5) if scale is None else scale
    o = torch.empty((B, H, N, d), dtype=torch.float32, device=q.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    fa_fwd_partial(q, k, v, o, lse, B, H, N, Nk, d, key_offset, scale, causal, blockmask,
                   _dtype_code(q), stream)
    return o, lse


def lse_merge(o_parts, lse_parts, out_dtype=None, stream=None):
    """Merge fp32 partial results [B, H, N, d] / [B, H, N] over disjoint key slices
    (fa_lse_merge).  ``out_dtype``: torch dtype of O (bf16 default, fp16 or fp32)."""
    import torch
    B, H, N, d = o_parts[0].shape
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    code = {torch.bfloat16: FA_BF16, torch.float16: FA_FP16, torch.float32: FA_FP32}[out_dtype]
    for t in list(o_parts) + list(lse_parts):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == torch.float32):
            raise ValueError("parts must be contiguous fp32 CUDA tensors")
    o = torch.empty((B, H, N, d), dtype=out_dtype, device=o_parts[0].device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=o_parts[0].device)
    fa_lse_merge(list(o_parts), list(lse_parts), o, lse, B, H, N, d, code, stream)
    return o, lse


def attention_forward_fp8(q8, k8, v8, descale_q, descale_k, descale_v, causal=False, blockmask=None, scale=None,
                          o_fp32=False, workspace=None, stream=None):
    """FP8 forward on E4M3 tensors [B, H, N, 128] (torch.float8_e4m3fn or uint8 codes) with
    per-tensor dequantisation factors.  Returns (O bf16 or fp32, LSE)."""
    import torch
    for t in (q8, k8, v8):
        if not (t.is_cuda and t.is_contiguous() and t.dim() == 4 and t.element_size() == 1):
            raise ValueError("expected contiguous 8-bit CUDA tensors of shape [B, H, N, 128]")
    B, H, N, d = q8.shape
    scale = (1.0 / d ** 0.5) if scale is None else scale
    o = torch.empty((B, H, N, d), dtype=torch.float32 if o_fp32 else torch.bfloat16, device=q8.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device)
    if workspace is None:
        workspace = torch.empty(max(fa_fwd_fp8_workspace_bytes(B, H, N, d), 1), dtype=torch.uint8, device=q8.device)
    fa_fwd_fp8(q8, k8, v8, descale_q, descale_k, descale_v, o, lse, B, H, N, d, scale, causal, blockmask, o_fp32,
               workspace, workspace.numel(), stream)
    return o, lse


def attention_backward(q, k, v, o, lse, dout, causal=False, blockmask=None, scale=None,
                       workspace=None, visit_log=None, stream=None, deterministic=False, dropout_p=0.0,
                       dropout_seed=0, query_splits=0):
    """Returns (dQ, dK, dV) for the gradient ``dout`` of O.  ``deterministic``: bitwise
    repeatable dQ through the int64 fixed-point accumulator; ``query_splits`` S >= 2: each key
    tile's query range cut into S ranges (include/fa.h)."""
    import torch
    _check_qkv(q, k, v, o, dout)
    B, H, N, d = q.shape
    scale = (1.0 / d ** 0.5) if scale is None else scale
    nbytes = (fa_bwd_workspace_bytes_split(B, H, N, d, query_splits) if query_splits > 1
              else fa_bwd_workspace_bytes_ex(B, H, N, d, deterministic))
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    fa_bwd_ex(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, blockmask,
              _dtype_code(q), visit_log, workspace, workspace.numel(), stream, deterministic=deterministic,
              dropout_p=dropout_p, dropout_seed=dropout_seed, query_splits=query_splits)
    return dq, dk, dv


def _make_autograd():
    import torch

    class FlashAttention(torch.autograd.Function):
        """autograd glue: forward saves (q, k, v, O, LSE); backward calls fa_bwd."""

        @staticmethod
        def forward(ctx, q, k, v, causal=False, blockmask=None, scale=None):
            o, lse = attention_forward(q, k, v, causal, blockmask, scale)
            ctx.save_for_backward(q, k, v, o, lse)
            ctx.causal, ctx.blockmask, ctx.scale = causal, blockmask, scale
            return o

        @staticmethod
        def backward(ctx, do):
            q, k, v, o, lse = ctx.saved_tensors
            dq, dk, dv = attention_backward(q, k, v, o, lse, do.contiguous(), ctx.causal,
                                            ctx.blockmask, ctx.scale)
            return dq, dk, dv, None, None, None

    return FlashAttention


def __getattr__(name):
    if name == "FlashAttention":
        fn = _make_autograd()
        globals()["FlashAttention"] = fn
        return fn
    raise AttributeError(name)
