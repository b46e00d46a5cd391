"""io_aware_exact_32_b200: exact IO-aware fused attention for NVIDIA B200 (sm_100a).

The compute lives in a C-ABI shared library (``libfa_sm100.so``, declared in
``include/fa.h``).  This module only marshals arguments: it checks shapes,
dtypes and devices, passes raw device pointers and the current CUDA stream,
and raises on a non-zero status.  PyTorch provides device memory and streams.

C-ABI mirrors (same names, torch tensors in place of pointers):
    fa_fwd, fa_bwd, fa_bwd_deterministic, fa_bwd_workspace_size, fa_decode_splitkv, fa_decode_num_splits,
    fa_decode_partials, fa_decode_merge,
    fa_decode_workspace_size, fa_decode_splitkv_noalloc, fa_quantize_fp8, fa_fwd_fp8, fa_fwd_ext,
    fa_bwd_ext, fa_get_device_error, fa_debug_set_wait_limit, fa_status_string, fa_version
Convenience wrappers that allocate outputs:
    attention_forward, attention_backward, decode_splitkv, quantize_fp8, attention_forward_fp8
"""
from __future__ import annotations

import ctypes
import math
import os

__all__ = [
    "FAError", "lib", "lib_path",
    "fa_fwd", "fa_bwd", "fa_bwd_deterministic", "fa_bwd_workspace_size", "fa_decode_splitkv",
    "fa_decode_workspace_size", "fa_decode_num_splits", "fa_decode_partials", "fa_decode_merge",
    "fa_decode_splitkv_noalloc", "fa_quantize_fp8", "fa_fwd_fp8", "fa_fwd_ext", "fa_bwd_ext",
    "fa_get_device_error", "fa_debug_set_wait_limit", "fa_status_string",
    "fa_version", "attention_forward", "attention_backward", "decode_splitkv", "quantize_fp8",
    "attention_forward_fp8",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libfa_sm100.so")

FA_OK = 0
_STATUS_NAMES = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_MISALIGNED",
                 4: "FA_ERR_WORKSPACE", 5: "FA_ERR_CUDA", 6: "FA_ERR_TIMEOUT"}


class FAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {_STATUS_NAMES.get(code, code)} ({fa_status_string(code)})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C-ABI library; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(lib_path):
        raise ImportError(f"{lib_path} is missing: build it with `python -m io_aware_exact_32_b200.build`")
    L = ctypes.CDLL(lib_path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
    L.fa_fwd.restype = i
    L.fa_bwd_workspace_size.argtypes = [i, i, i, i]
    L.fa_bwd_workspace_size.restype = sz
    L.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, f, i, vp]
    L.fa_bwd.restype = i
    L.fa_bwd_deterministic.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, f, i, vp]
    L.fa_bwd_deterministic.restype = i
    L.fa_decode_workspace_size.argtypes = [i, i, i, i, i]
    L.fa_decode_workspace_size.restype = sz
    L.fa_decode_splitkv.argtypes = [vp, vp, vp, vp, i, vp, vp, i, i, i, f, i, vp, sz, vp]
    L.fa_decode_splitkv.restype = i
    L.fa_decode_splitkv_noalloc.argtypes = [vp, vp, vp, vp, i, vp, vp, i, i, i, f, i, vp]
    L.fa_decode_splitkv_noalloc.restype = i
    L.fa_decode_num_splits.argtypes = [i, i]
    L.fa_decode_num_splits.restype = i
    L.fa_decode_partials.argtypes = [vp, vp, vp, vp, i, vp, vp, i, i, i, f, i, vp]
    L.fa_decode_partials.restype = i
    L.fa_decode_merge.argtypes = [vp, vp, i, i, vp, vp, i, i, i, vp]
    L.fa_decode_merge.restype = i
    L.fa_quantize_fp8.argtypes = [vp, vp, vp, vp, i, i, i, i, i, vp]
    L.fa_quantize_fp8.restype = i
    L.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
    L.fa_fwd_fp8.restype = i
    u64, u32 = ctypes.c_ulonglong, ctypes.c_uint
    L.fa_fwd_ext.argtypes = [vp, vp, vp, vp, i, i, vp, vp, i, i, i, i, i, f, i, f, u64, u32, vp]
    L.fa_fwd_ext.restype = i
    L.fa_bwd_ext.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, vp, vp, vp, vp, sz, i, i, i, i, i, f, i, f, u64, u32,
                             vp]
    L.fa_bwd_ext.restype = i
    L.fa_debug_set_wait_limit.argtypes = [ctypes.c_ulonglong]
    L.fa_debug_set_wait_limit.restype = i
    L.fa_get_device_error.argtypes = [vp]
    L.fa_get_device_error.restype = i
    L.fa_status_string.argtypes = [i]
    L.fa_status_string.restype = ctypes.c_char_p
    L.fa_version.argtypes = []
    L.fa_version.restype = i
    _lib = L
    return L


def fa_status_string(code: int) -> str:
    return lib().fa_status_string(int(code)).decode()


def fa_version() -> int:
    return lib().fa_version()


def _stream_ptr(stream, device=None):
    """The cudaStream_t to launch on: ``stream`` (a torch.cuda.Stream or a raw handle), else the current
    stream of ``device``.  A torch stream that belongs to another device than the tensors is refused."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    sdev = getattr(stream, "device", None)
    if device is not None and sdev is not None and torch.device(sdev) != torch.device(device):
        raise ValueError(f"stream is on {sdev}, the tensors on {device}")
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _on_device(device):
    """Context that makes ``device`` current for one C-ABI call.  The library resolves the SM count,
    the shared-memory opt-in and its per-device scratch from the current device, and the default
    stream is the current device's, so the tensors' device must be current while it runs."""
    import torch
    return torch.cuda.device(device)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _check(code: int, where: str):
    if code != FA_OK:
        raise FAError(code, where)


def _need(t, name, dtype, device, shape=None):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device.type != "cuda":
        # The kernels take device pointers: a host tensor must never reach them.
        raise ValueError(f"{name} must be a CUDA tensor, got {t.device}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _scale(scale, d):
    return float(1.0 / math.sqrt(d) if scale is None else scale)


# ------------------------------------------------------------------------------ C-ABI mirrors
def fa_fwd(q, k, v, o, lse, causal: bool, scale=None, stream=None) -> None:
    """O, LSE of exact attention (see include/fa.h: fa_fwd).  q/o [B,H,Nq,d], k/v [B,H,Nk,d] bf16, lse [B,H,Nq] fp32."""
    import torch
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    dev = q.device
    _need(q, "q", torch.bfloat16, dev)
    _need(k, "k", torch.bfloat16, dev, (B, H, Nk, d))
    _need(v, "v", torch.bfloat16, dev, (B, H, Nk, d))
    _need(o, "o", torch.bfloat16, dev, (B, H, Nq, d))
    _need(lse, "lse", torch.float32, dev, (B, H, Nq))
    with _on_device(dev):
        _check(lib().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk, d,
                            _scale(scale, d), int(bool(causal)), _stream_ptr(stream, dev)), "fa_fwd")


def fa_bwd_workspace_size(B: int, H: int, Nq: int, d: int) -> int:
    return int(lib().fa_bwd_workspace_size(B, H, Nq, d))


def fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, workspace, causal: bool, scale=None, stream=None,
           deterministic: bool = False) -> None:
    """dQ, dK, dV by recomputation (see include/fa.h: fa_bwd, and fa_bwd_deterministic when
    deterministic is set).  workspace: uint8 device tensor."""
    import torch
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    dev = q.device
    for t, n, shp in ((q, "q", (B, H, Nq, d)), (o, "o", (B, H, Nq, d)), (dO, "dO", (B, H, Nq, d)),
                      (dq, "dq", (B, H, Nq, d)), (k, "k", (B, H, Nk, d)), (v, "v", (B, H, Nk, d)),
                      (dk, "dk", (B, H, Nk, d)), (dv, "dv", (B, H, Nk, d))):
        _need(t, n, torch.bfloat16, dev, shp)
    _need(lse, "lse", torch.float32, dev, (B, H, Nq))
    _need(workspace, "workspace", torch.uint8, dev)
    fn, name = (lib().fa_bwd_deterministic, "fa_bwd_deterministic") if deterministic else (lib().fa_bwd, "fa_bwd")
    with _on_device(dev):
        _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                  _ptr(workspace), workspace.numel(), B, H, Nq, Nk, d, _scale(scale, d),
                  int(bool(causal)), _stream_ptr(stream, dev)), name)


def fa_bwd_deterministic(q, k, v, o, dO, lse, dq, dk, dv, workspace, causal: bool, scale=None, stream=None) -> None:
    """fa_bwd with bitwise reproducible dQ (see include/fa.h: fa_bwd_deterministic)."""
    fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, workspace, causal, scale, stream, deterministic=True)


def fa_decode_workspace_size(B: int, H: int, Lmax: int, d: int, num_splits: int = 0) -> int:
    return int(lib().fa_decode_workspace_size(B, H, Lmax, d, num_splits))


def fa_decode_splitkv(q, k_cache, v_cache, seqlens, o, lse, workspace, scale=None, num_splits: int = 0,
                      stream=None) -> None:
    """Split-KV decode (see include/fa.h: fa_decode_splitkv).  q/o [B,H,1,d], caches [B,H,Lmax,d], seqlens int32 [B]."""
    import torch
    B, H, one, d = q.shape
    if one != 1:
        raise ValueError("decode takes one query per (batch, head)")
    Lmax = k_cache.shape[2]
    dev = q.device
    _need(q, "q", torch.bfloat16, dev)
    _need(k_cache, "k_cache", torch.bfloat16, dev, (B, H, Lmax, d))
    _need(v_cache, "v_cache", torch.bfloat16, dev, (B, H, Lmax, d))
    _need(seqlens, "seqlens", torch.int32, dev, (B,))
    _need(o, "o", torch.bfloat16, dev, (B, H, 1, d))
    if lse is not None:
        _need(lse, "lse", torch.float32, dev, (B, H))
    _need(workspace, "workspace", torch.uint8, dev)
    with _on_device(dev):
        _check(lib().fa_decode_splitkv(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), Lmax, _ptr(o), _ptr(lse),
                                       B, H, d, _scale(scale, d), int(num_splits), _ptr(workspace), workspace.numel(),
                                       _stream_ptr(stream, dev)), "fa_decode_splitkv")


def fa_decode_splitkv_noalloc(q, k_cache, v_cache, seqlens, o, lse, scale=None, num_splits: int = 0,
                              stream=None) -> None:
    """Split-KV decode with no workspace (see include/fa.h: fa_decode_splitkv_noalloc).

    For callers that cannot allocate device memory: the partials live in the
    library's own fixed-size device scratch, shared by every call (calls that
    overlap on the GPU race on it)."""
    import torch
    B, H, one, d = q.shape
    if one != 1:
        raise ValueError("decode takes one query per (batch, head)")
    Lmax = k_cache.shape[2]
    dev = q.device
    _need(q, "q", torch.bfloat16, dev)
    _need(k_cache, "k_cache", torch.bfloat16, dev, (B, H, Lmax, d))
    _need(v_cache, "v_cache", torch.bfloat16, dev, (B, H, Lmax, d))
    _need(seqlens, "seqlens", torch.int32, dev, (B,))
    _need(o, "o", torch.bfloat16, dev, (B, H, 1, d))
    if lse is not None:
        _need(lse, "lse", torch.float32, dev, (B, H))
    with _on_device(dev):
        _check(lib().fa_decode_splitkv_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), Lmax, _ptr(o),
                                               _ptr(lse), B, H, d, _scale(scale, d), int(num_splits),
                                               _stream_ptr(stream, dev)), "fa_decode_splitkv_noalloc")


def fa_decode_num_splits(Lmax: int, num_splits: int = 0) -> int:
    return int(lib().fa_decode_num_splits(Lmax, num_splits))


def fa_decode_partials(q, k_cache, v_cache, seqlens, part_o, part_ml, scale=None, num_splits: int = 0,
                       stream=None) -> None:
    """Unmerged split-KV partials for a KV slice (see include/fa.h: fa_decode_partials).
    part_o [B, H, S, d] fp32, part_ml [B, H, S, 2] fp32 with S = fa_decode_num_splits(Lmax, num_splits)."""
    import torch
    B, H, one, d = q.shape
    if one != 1:
        raise ValueError("decode takes one query per (batch, head)")
    Lmax = k_cache.shape[2]
    S = fa_decode_num_splits(Lmax, num_splits)
    dev = q.device
    _need(q, "q", torch.bfloat16, dev)
    _need(k_cache, "k_cache", torch.bfloat16, dev, (B, H, Lmax, d))
    _need(v_cache, "v_cache", torch.bfloat16, dev, (B, H, Lmax, d))
    _need(seqlens, "seqlens", torch.int32, dev, (B,))
    _need(part_o, "part_o", torch.float32, dev, (B, H, S, d))
    _need(part_ml, "part_ml", torch.float32, dev, (B, H, S, 2))
    with _on_device(dev):
        _check(lib().fa_decode_partials(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), Lmax, _ptr(part_o),
                                        _ptr(part_ml), B, H, d, _scale(scale, d), int(num_splits), _stream_ptr(stream, dev)),
               "fa_decode_partials")


def fa_decode_merge(part_o, part_ml, o, lse=None, stream=None) -> None:
    """Merge R groups of S partials, part_o [R, B, H, S, d] and part_ml [R, B, H, S, 2] fp32, into o [B, H, 1, d]
    bf16 and lse [B, H] (see include/fa.h: fa_decode_merge)."""
    import torch
    R, B, H, S, d = part_o.shape
    dev = part_o.device
    _need(part_o, "part_o", torch.float32, dev)
    _need(part_ml, "part_ml", torch.float32, dev, (R, B, H, S, 2))
    _need(o, "o", torch.bfloat16, dev, (B, H, 1, d))
    if lse is not None:
        _need(lse, "lse", torch.float32, dev, (B, H))
    with _on_device(dev):
        _check(lib().fa_decode_merge(_ptr(part_o), _ptr(part_ml), R, S, _ptr(o), _ptr(lse), B, H, d,
                                     _stream_ptr(stream, dev)), "fa_decode_merge")


def _bias_dims(bias, B, H, Nq, Nk, device):
    import torch
    if bias is None:
        return 1, 1
    if not isinstance(bias, torch.Tensor):
        raise TypeError("bias must be a torch.Tensor")
    if bias.dim() != 4 or tuple(bias.shape[2:]) != (Nq, Nk) or bias.shape[0] not in (1, B) or \
            bias.shape[1] not in (1, H):
        raise ValueError(f"bias has shape {tuple(bias.shape)}, expected [1 or {B}, 1 or {H}, {Nq}, {Nk}]")
    _need(bias, "bias", torch.bfloat16, device)
    return int(bias.shape[0]), int(bias.shape[1])


def fa_fwd_ext(q, k, v, o, lse, bias=None, causal: bool = False, scale=None, dropout_p: float = 0.0, seed: int = 0,
               offset: int = 0, stream=None) -> None:
    """Forward with an additive bias and dropout (see include/fa.h: fa_fwd_ext).  bias [1|B, 1|H, Nq, Nk] bf16
    or None."""
    import torch
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    dev = q.device
    _need(q, "q", torch.bfloat16, dev)
    _need(k, "k", torch.bfloat16, dev, (B, H, Nk, d))
    _need(v, "v", torch.bfloat16, dev, (B, H, Nk, d))
    _need(o, "o", torch.bfloat16, dev, (B, H, Nq, d))
    _need(lse, "lse", torch.float32, dev, (B, H, Nq))
    bB, bH = _bias_dims(bias, B, H, Nq, Nk, dev)
    with _on_device(dev):
        _check(lib().fa_fwd_ext(_ptr(q), _ptr(k), _ptr(v), _ptr(bias), bB, bH, _ptr(o), _ptr(lse), B, H, Nq, Nk, d,
                                _scale(scale, d), int(bool(causal)), float(dropout_p), int(seed) & (2 ** 64 - 1),
                                int(offset) & 0xFFFFFFFF, _stream_ptr(stream, dev)), "fa_fwd_ext")


def fa_bwd_ext(q, k, v, o, dO, lse, dq, dk, dv, workspace, bias=None, causal: bool = False, scale=None,
               dropout_p: float = 0.0, seed: int = 0, offset: int = 0, stream=None) -> None:
    """Backward of fa_fwd_ext with the same bias, dropout_p, seed and offset (see include/fa.h: fa_bwd_ext)."""
    import torch
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    dev = q.device
    for t, n, shp in ((q, "q", (B, H, Nq, d)), (o, "o", (B, H, Nq, d)), (dO, "dO", (B, H, Nq, d)),
                      (dq, "dq", (B, H, Nq, d)), (k, "k", (B, H, Nk, d)), (v, "v", (B, H, Nk, d)),
                      (dk, "dk", (B, H, Nk, d)), (dv, "dv", (B, H, Nk, d))):
        _need(t, n, torch.bfloat16, dev, shp)
    _need(lse, "lse", torch.float32, dev, (B, H, Nq))
    _need(workspace, "workspace", torch.uint8, dev)
    bB, bH = _bias_dims(bias, B, H, Nq, Nk, dev)
    with _on_device(dev):
        _check(lib().fa_bwd_ext(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse), _ptr(bias), bB, bH, _ptr(dq),
                                _ptr(dk), _ptr(dv), _ptr(workspace), workspace.numel(), B, H, Nq, Nk, d, _scale(scale, d),
                                int(bool(causal)), float(dropout_p), int(seed) & (2 ** 64 - 1), int(offset) & 0xFFFFFFFF,
                                _stream_ptr(stream, dev)), "fa_bwd_ext")


def _need_e4m3(t, name, device, shape=None):
    """E4M3 codes: a torch.uint8 or torch.float8_e4m3fn tensor."""
    import torch
    dtype = t.dtype if isinstance(t, torch.Tensor) and t.dtype in (torch.uint8, torch.float8_e4m3fn) else torch.uint8
    _need(t, name, dtype, device, shape)


def fa_quantize_fp8(x, signs, x8, descale, hadamard: bool = True, stream=None) -> None:
    """Per-head E4M3 quantisation with optional incoherent processing (see include/fa.h: fa_quantize_fp8).
    x [B,H,N,d] bf16, signs [d] fp32 (+-1) or None, x8 [B,H,N,d] uint8 / float8_e4m3fn, descale [B,H] fp32."""
    import torch
    B, H, N, d = x.shape
    dev = x.device
    _need(x, "x", torch.bfloat16, dev)
    if signs is not None:
        _need(signs, "signs", torch.float32, dev, (d,))
    _need_e4m3(x8, "x8", dev, (B, H, N, d))
    _need(descale, "descale", torch.float32, dev, (B, H))
    with _on_device(dev):
        _check(lib().fa_quantize_fp8(_ptr(x), _ptr(signs), _ptr(x8), _ptr(descale), B, H, N, d, int(bool(hadamard)),
                                     _stream_ptr(stream, dev)), "fa_quantize_fp8")


def fa_fwd_fp8(q8, k8, v8, descale_q, descale_k, descale_v, o, lse, causal: bool, scale=None, stream=None) -> None:
    """Forward on E4M3 operands (see include/fa.h: fa_fwd_fp8).  q8 [B,H,Nq,d], k8/v8 [B,H,Nk,d] uint8 or
    float8_e4m3fn codes; descale_* [B,H] fp32; o [B,H,Nq,d] bf16, lse [B,H,Nq] fp32."""
    import torch
    B, H, Nq, d = q8.shape
    Nk = k8.shape[2]
    dev = q8.device
    _need_e4m3(q8, "q8", dev)
    _need_e4m3(k8, "k8", dev, (B, H, Nk, d))
    _need_e4m3(v8, "v8", dev, (B, H, Nk, d))
    for t, n in ((descale_q, "descale_q"), (descale_k, "descale_k"), (descale_v, "descale_v")):
        _need(t, n, torch.float32, dev, (B, H))
    _need(o, "o", torch.bfloat16, dev, (B, H, Nq, d))
    _need(lse, "lse", torch.float32, dev, (B, H, Nq))
    with _on_device(dev):
        _check(lib().fa_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(descale_q), _ptr(descale_k), _ptr(descale_v),
                                _ptr(o), _ptr(lse), B, H, Nq, Nk, d, _scale(scale, d), int(bool(causal)),
                                _stream_ptr(stream, dev)), "fa_fwd_fp8")


def fa_debug_set_wait_limit(limit_ns: int, device=None) -> None:
    """Test hook (see include/fa.h: fa_debug_set_wait_limit): the limit of every pipeline wait on
    ``device`` (default: current), 0 restoring the default 2 s."""
    with _on_device(device):
        _check(lib().fa_debug_set_wait_limit(int(limit_ns)), "fa_debug_set_wait_limit")


def fa_get_device_error(stream=None, device=None) -> int:
    """Synchronise the stream and read and clear the device status word (see include/fa.h: fa_get_device_error)
    of ``device`` (default: the stream's device, else the current device)."""
    dev = device if device is not None else getattr(stream, "device", None)
    with _on_device(dev):
        return int(lib().fa_get_device_error(_stream_ptr(stream, dev)))


# ------------------------------------------------------------------------------ conveniences
def _workspace(nbytes: int, device):
    import torch
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def attention_forward(q, k, v, causal: bool = False, scale=None, stream=None):
    """Allocate O and LSE and run fa_fwd; returns (o, lse)."""
    import torch
    B, H, Nq, d = q.shape
    o = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    fa_fwd(q, k, v, o, lse, causal, scale, stream)
    return o, lse


def attention_backward(q, k, v, o, lse, dO, causal: bool = False, scale=None, stream=None, workspace=None,
                       deterministic: bool = False):
    """Allocate dQ, dK, dV (and the workspace unless given) and run fa_bwd (fa_bwd_deterministic when
    deterministic is set); returns (dq, dk, dv)."""
    import torch
    B, H, Nq, d = q.shape
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    if workspace is None:
        workspace = _workspace(fa_bwd_workspace_size(B, H, Nq, d), q.device)
    fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, workspace, causal, scale, stream, deterministic=deterministic)
    return dq, dk, dv


def decode_splitkv(q, k_cache, v_cache, seqlens, scale=None, num_splits: int = 0, stream=None, workspace=None):
    """Allocate O, LSE (and the workspace unless given) and run fa_decode_splitkv; returns (o, lse)."""
    import torch
    B, H, _, d = q.shape
    o = torch.empty((B, H, 1, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = _workspace(fa_decode_workspace_size(B, H, k_cache.shape[2], d, num_splits), q.device)
    fa_decode_splitkv(q, k_cache, v_cache, seqlens, o, lse, workspace, scale, num_splits, stream)
    return o, lse


def quantize_fp8(x, signs=None, hadamard: bool = True, stream=None):
    """Allocate the codes and scales and run fa_quantize_fp8; returns (x8 uint8, descale fp32 [B, H])."""
    import torch
    B, H, N, d = x.shape
    x8 = torch.empty((B, H, N, d), dtype=torch.uint8, device=x.device)
    descale = torch.empty((B, H), dtype=torch.float32, device=x.device)
    fa_quantize_fp8(x, signs, x8, descale, hadamard, stream)
    return x8, descale


def attention_forward_fp8(q, k, v, causal: bool = False, scale=None, signs=None, hadamard: bool = True, stream=None):
    """FP8 forward from bf16 Q, K, V: Q and K are rotated (random-sign Hadamard, the same signs for both)
    and quantised, V is quantised, then fa_fwd_fp8 runs.  Returns (o bf16, lse fp32)."""
    import torch
    B, H, Nq, d = q.shape
    q8, dq = quantize_fp8(q, signs, hadamard, stream)
    k8, dk = quantize_fp8(k, signs, hadamard, stream)
    v8, dv = quantize_fp8(v, None, False, stream)
    o = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    fa_fwd_fp8(q8, k8, v8, dq, dk, dv, o, lse, causal, scale, stream)
    return o, lse
