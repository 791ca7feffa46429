"""Thin Python binding over the C ABI (include/fa.h), same names.

Argument marshalling only: torch tensors (device memory) are turned into
pointers and sizes and passed to libfa.so on the current CUDA stream.  Every
computation runs in the library's kernels.
"""
from __future__ import annotations

import ctypes
import math

import torch

from . import _lib
from ._lib import check

_BF16 = torch.bfloat16


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _shape(q: torch.Tensor):
    if q.dim() != 4:
        raise ValueError("expected a [B, H, N, d] tensor")
    return tuple(int(x) for x in q.shape)


def _need(t: torch.Tensor, name: str, dtype, shape):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous() or not t.is_cuda:
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} contiguous={t.is_contiguous()} cuda={t.is_cuda}")
    _on_current_device(t, name)


def _on_current_device(t: torch.Tensor, name: str):
    # the library launches on the current device; a pointer into another GPU's memory must not reach it
    if t.device.index is not None and t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name}: on {t.device}, but the current device is cuda:{torch.cuda.current_device()}")


def _need_workspace(ws: torch.Tensor, nbytes: int):
    if not ws.is_cuda or not ws.is_contiguous():
        raise ValueError("workspace: expected a contiguous CUDA tensor")
    _on_current_device(ws, "workspace")
    if ws.numel() * ws.element_size() < nbytes:
        raise ValueError(f"workspace: {ws.numel() * ws.element_size()} bytes, {nbytes} needed")


def fa_fwd(q, k, v, scale: float | None = None, causal: bool = False, out=None, lse=None, stream=None):
    """O, LSE = attention(q, k, v); q/k/v bf16 [B, H, N, d] on the GPU."""
    B, H, N, d = _shape(q)
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, nm, _BF16, (B, H, N, d))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _need(out, "out", _BF16, (B, H, N, d))
    _need(lse, "lse", torch.float32, (B, H, N))
    check(_lib.lib().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, d, scale,
                            int(bool(causal)), _stream(stream)), "fa_fwd")
    return out, lse


def fa_bwd_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(_lib.lib().fa_bwd_workspace_size(B, H, N, d))


def fa_bwd(q, k, v, o, do, lse, scale: float | None = None, causal: bool = False,
           dq=None, dk=None, dv=None, workspace=None, stream=None):
    """dQ, dK, dV of attention given the forward's O and LSE and the upstream dO."""
    B, H, N, d = _shape(q)
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (do, "do")):
        _need(t, nm, _BF16, (B, H, N, d))
    _need(lse, "lse", torch.float32, (B, H, N))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    ws_bytes = fa_bwd_workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    _need_workspace(workspace, ws_bytes)
    for t, nm in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _need(t, nm, _BF16, (B, H, N, d))
    check(_lib.lib().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk),
                            _ptr(dv), _ptr(workspace), workspace.numel() * workspace.element_size(),
                            B, H, N, d, scale, int(bool(causal)), _stream(stream)), "fa_bwd")
    return dq, dk, dv


def fa_bwd_noalloc(q, k, v, o, do, lse, scale: float | None = None, causal: bool = False,
                   dq=None, dk=None, dv=None, stream=None):
    """fa_bwd on the library's fixed scratch array (no workspace; see include/fa.h for the size limit)."""
    B, H, N, d = _shape(q)
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (do, "do")):
        _need(t, nm, _BF16, (B, H, N, d))
    _need(lse, "lse", torch.float32, (B, H, N))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    check(_lib.lib().fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk),
                                    _ptr(dv), B, H, N, d, scale, int(bool(causal)), _stream(stream)),
          "fa_bwd_noalloc")
    return dq, dk, dv


def _shape_qk(q, k):
    B, Hq, Nq, d = _shape(q)
    Bk, Hkv, Nk, dk = _shape(k)
    if Bk != B or dk != d:
        raise ValueError("q and k must agree in batch and head dimension")
    return B, Hq, Hkv, Nq, Nk, d


def fa_fwd_qk(q, k, v, scale: float | None = None, causal: bool = False, out=None, lse=None, stream=None):
    """O, LSE of grouped-query attention with Nq queries over Nk keys: q bf16 [B, Hq, Nq, d],
    k/v bf16 [B, Hkv, Nk, d] (Hq a multiple of Hkv; causal aligns the last query with the last key)."""
    B, Hq, Hkv, Nq, Nk, d = _shape_qk(q, k)
    _need(q, "q", _BF16, (B, Hq, Nq, d))
    for t, nm in ((k, "k"), (v, "v")):
        _need(t, nm, _BF16, (B, Hkv, Nk, d))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    _need(out, "out", _BF16, (B, Hq, Nq, d))
    _need(lse, "lse", torch.float32, (B, Hq, Nq))
    check(_lib.lib().fa_fwd_qk(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Nq, Nk, d, scale,
                               int(bool(causal)), _stream(stream)), "fa_fwd_qk")
    return out, lse


def fa_bwd_qk_workspace_size(B: int, Hq: int, Nq: int, d: int) -> int:
    return int(_lib.lib().fa_bwd_qk_workspace_size(B, Hq, Nq, d))


def fa_bwd_qk(q, k, v, o, do, lse, scale: float | None = None, causal: bool = False,
              dq=None, dk=None, dv=None, workspace=None, stream=None):
    """dQ [B, Hq, Nq, d] and dK, dV [B, Hkv, Nk, d] (summed over each key/value head's query heads)."""
    B, Hq, Hkv, Nq, Nk, d = _shape_qk(q, k)
    for t, nm in ((q, "q"), (o, "o"), (do, "do")):
        _need(t, nm, _BF16, (B, Hq, Nq, d))
    for t, nm in ((k, "k"), (v, "v")):
        _need(t, nm, _BF16, (B, Hkv, Nk, d))
    _need(lse, "lse", torch.float32, (B, Hq, Nq))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(k) if dv is None else dv
    ws_bytes = fa_bwd_qk_workspace_size(B, Hq, Nq, d)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    _need_workspace(workspace, ws_bytes)
    _need(dq, "dq", _BF16, (B, Hq, Nq, d))
    for t, nm in ((dk, "dk"), (dv, "dv")):
        _need(t, nm, _BF16, (B, Hkv, Nk, d))
    check(_lib.lib().fa_bwd_qk(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk),
                               _ptr(dv), _ptr(workspace), workspace.numel() * workspace.element_size(),
                               B, Hq, Hkv, Nq, Nk, d, scale, int(bool(causal)), _stream(stream)), "fa_bwd_qk")
    return dq, dk, dv


def fa_fwd_accumulate(q, k, v, o_acc, lse_acc, scale: float | None = None, causal: bool = False,
                      first: bool = False, stream=None) -> None:
    """Fold attention of q over one key block (k, v) into fp32 accumulators o_acc [B, Hq, Nq, d],
    lse_acc [B, Hq, Nq] by their log-sum-exp (first: initialise them)."""
    B, Hq, Hkv, Nq, Nk, d = _shape_qk(q, k)
    _need(q, "q", _BF16, (B, Hq, Nq, d))
    for t, nm in ((k, "k"), (v, "v")):
        _need(t, nm, _BF16, (B, Hkv, Nk, d))
    _need(o_acc, "o_acc", torch.float32, (B, Hq, Nq, d))
    _need(lse_acc, "lse_acc", torch.float32, (B, Hq, Nq))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    check(_lib.lib().fa_fwd_accumulate(_ptr(q), _ptr(k), _ptr(v), _ptr(o_acc), _ptr(lse_acc), B, Hq, Hkv, Nq, Nk,
                                       d, scale, int(bool(causal)), int(bool(first)), _stream(stream)),
          "fa_fwd_accumulate")


def fa_bwd_prepare(o, do, lse, workspace=None, stream=None):
    """D and LSE*log2(e) of a query block into a (new or given) workspace, dQ accumulator zeroed;
    o, do bf16 [B, Hq, Nq, d], lse fp32 [B, Hq, Nq].  Returns the workspace."""
    B, Hq, Nq, d = _shape(o)
    for t, nm in ((o, "o"), (do, "do")):
        _need(t, nm, _BF16, (B, Hq, Nq, d))
    _need(lse, "lse", torch.float32, (B, Hq, Nq))
    ws_bytes = fa_bwd_qk_workspace_size(B, Hq, Nq, d)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=o.device)
    _need_workspace(workspace, ws_bytes)
    check(_lib.lib().fa_bwd_prepare(_ptr(o), _ptr(do), _ptr(lse), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), B, Hq, Nq, d, _stream(stream)),
          "fa_bwd_prepare")
    return workspace


def fa_bwd_accumulate(q, k, v, do, workspace, dk_acc, dv_acc, scale: float | None = None, causal: bool = False,
                      first: bool = False, stream=None) -> None:
    """Gradients of one key block: dQ added into the workspace, dK (scaled) and dV stored (first) or
    added into the fp32 accumulators dk_acc, dv_acc [B, Hkv, Nk, d]."""
    B, Hq, Hkv, Nq, Nk, d = _shape_qk(q, k)
    for t, nm in ((q, "q"), (do, "do")):
        _need(t, nm, _BF16, (B, Hq, Nq, d))
    for t, nm in ((k, "k"), (v, "v")):
        _need(t, nm, _BF16, (B, Hkv, Nk, d))
    for t, nm in ((dk_acc, "dk_acc"), (dv_acc, "dv_acc")):
        _need(t, nm, torch.float32, (B, Hkv, Nk, d))
    _need_workspace(workspace, fa_bwd_qk_workspace_size(B, Hq, Nq, d))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    check(_lib.lib().fa_bwd_accumulate(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _ptr(dk_acc), _ptr(dv_acc),
                                       B, Hq, Hkv, Nq, Nk, d, scale, int(bool(causal)), int(bool(first)),
                                       _stream(stream)), "fa_bwd_accumulate")


def fa_bwd_finish(workspace, B: int, Hq: int, Nq: int, d: int, scale: float | None = None, out=None, stream=None):
    """dQ (bf16 [B, Hq, Nq, d]) from the workspace's accumulator."""
    _need_workspace(workspace, fa_bwd_qk_workspace_size(B, Hq, Nq, d))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty((B, Hq, Nq, d), dtype=_BF16, device=workspace.device) if out is None else out
    _need(out, "out", _BF16, (B, Hq, Nq, d))
    check(_lib.lib().fa_bwd_finish(_ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(out), B, Hq,
                                   Nq, d, scale, _stream(stream)), "fa_bwd_finish")
    return out


def fa_lse_merge(o_part, lse_part, o_acc, lse_acc, first: bool = False, stream=None) -> None:
    """Fold a partial (O bf16 [..., d], LSE fp32 [...]) over one key set into an fp32 accumulator."""
    d = int(o_part.shape[-1])
    rows = o_part.numel() // d
    _need(o_part, "o_part", _BF16, tuple(o_part.shape))
    _need(o_acc, "o_acc", torch.float32, tuple(o_part.shape))
    _need(lse_part, "lse_part", torch.float32, tuple(o_part.shape[:-1]))
    _need(lse_acc, "lse_acc", torch.float32, tuple(o_part.shape[:-1]))
    check(_lib.lib().fa_lse_merge(_ptr(o_part), _ptr(lse_part), _ptr(o_acc), _ptr(lse_acc), rows, d,
                                  int(bool(first)), _stream(stream)), "fa_lse_merge")


def fa_accumulate_bf16(acc, x, first: bool = False, stream=None) -> None:
    """acc (fp32) = (0 if first else acc) + x (bf16), elementwise."""
    _need(acc, "acc", torch.float32, tuple(x.shape))
    _need(x, "x", _BF16, tuple(x.shape))
    check(_lib.lib().fa_accumulate_bf16(_ptr(acc), _ptr(x), x.numel(), int(bool(first)), _stream(stream)),
          "fa_accumulate_bf16")


def fa_accumulate_f32(acc, x, stream=None) -> None:
    """acc (fp32) += x (fp32), elementwise."""
    _need(acc, "acc", torch.float32, tuple(x.shape))
    _need(x, "x", torch.float32, tuple(x.shape))
    check(_lib.lib().fa_accumulate_f32(_ptr(acc), _ptr(x), x.numel(), _stream(stream)), "fa_accumulate_f32")


def fa_convert_f32_bf16(x, out=None, stream=None):
    """bf16 copy of an fp32 tensor (round to nearest even)."""
    out = torch.empty(x.shape, dtype=_BF16, device=x.device) if out is None else out
    _need(x, "x", torch.float32, tuple(x.shape))
    _need(out, "out", _BF16, tuple(x.shape))
    check(_lib.lib().fa_convert_f32_bf16(_ptr(x), _ptr(out), x.numel(), _stream(stream)), "fa_convert_f32_bf16")
    return out


def fa_last_device_status(stream=None) -> tuple[int, int]:
    """(status, detail) after synchronising the stream; see include/fa.h."""
    detail = ctypes.c_int(0)
    rc = _lib.lib().fa_last_device_status(_stream(stream), ctypes.byref(detail))
    return int(rc), int(detail.value)


def fa_set_softmax_options(tau: float = 8.0, poly: int = -1) -> None:
    """Rescale threshold and cubic-exp2 share (pairs per 16; -1 = per-head-dim default)."""
    check(_lib.lib().fa_set_softmax_options(float(tau), int(poly)), "fa_set_softmax_options")


def fa_set_forward_variant(cluster_pair: int = 0) -> None:
    check(_lib.lib().fa_set_forward_variant(int(cluster_pair)), "fa_set_forward_variant")


def fa_set_backward_variant(cluster_pair: int = 0) -> None:
    check(_lib.lib().fa_set_backward_variant(int(cluster_pair)), "fa_set_backward_variant")


def fa_exp2_eval(x: torch.Tensor, mode: int = 0, stream=None) -> torch.Tensor:
    """2^x on the device: mode 0 = cubic software exp2, 1 = SFU ex2."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA float32 tensor")
    _on_current_device(x, "x")
    y = torch.empty_like(x)
    check(_lib.lib().fa_exp2_eval(_ptr(x), _ptr(y), x.numel(), int(mode), _stream(stream)), "fa_exp2_eval")
    return y


def fa_profile_next(which: int, start, stop) -> None:
    """Have the next fa_fwd (0) / fa_bwd (1) record torch.cuda.Events around its main kernel."""
    h = lambda e: None if e is None else ctypes.c_void_p(e.cuda_event)
    check(_lib.lib().fa_profile_next(int(which), h(start), h(stop)), "fa_profile_next")


def fa_sm_clock_probe(out: torch.Tensor | None = None, stream=None):
    """Effective SM clock, measured on the device by a ~20 us probe kernel queued on `stream`
    behind whatever work is already queued there.  With `out` (a CUDA int64 tensor of 2 elements)
    it only queues the probe, which writes [cycles, nanoseconds] there (no synchronisation, so
    the GPU keeps the clock of the surrounding work); without, it synchronises and returns MHz."""
    own = out is None
    if own:
        out = torch.zeros(2, dtype=torch.int64, device="cuda")
    elif out.dtype != torch.int64 or not out.is_cuda or out.numel() != 2 or not out.is_contiguous():
        raise ValueError("out must be a contiguous CUDA int64 tensor of 2 elements")
    else:
        _on_current_device(out, "out")
    check(_lib.lib().fa_sm_clock_probe(_ptr(out), _stream(stream)), "fa_sm_clock_probe")
    if not own:
        return None
    torch.cuda.synchronize()
    cycles, ns = out.tolist()
    return 1000.0 * cycles / ns if ns > 0 else 0.0


def fa_strerror(code: int) -> str:
    return _lib.lib().fa_strerror(int(code)).decode()


def fa_version() -> int:
    return int(_lib.lib().fa_version())
