"""ctypes binding of libra.so (argument marshalling only).

Every call forwards torch tensors' device pointers and sizes to the C ABI declared in
include/ra.h and launches on torch's current CUDA stream. PyTorch provides device memory
and streams; all arithmetic of the path runs in the library's CUDA kernels. There is no
CPU fallback: a missing library raises on first use.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
library_path = os.environ.get("RA_LIBRARY", os.path.join(_PKG, "libra.so"))

RA_OK, RA_ERR_INVALID_ARG, RA_ERR_UNSUPPORTED, RA_ERR_CUDA, RA_ERR_TIMEOUT, RA_ERR_DEVICE_BOUNDS = range(6)
RA_F32, RA_BF16 = 0, 1
LAYOUTS = {"contiguous": 0, "striped": 1, "zigzag": 2}
ABI_VERSION = 4  # the ABI these signatures describe (ra_abi_version() of a matching library)

# name -> (restype, argtypes) of every symbol include/ra.h declares
_i64, _i32, _f32, _vp = ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_void_p
SIGNATURES = {
    "ra_partial": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i64, _i64, _i32, _f32, _i32,
                          _i64, _i64, _i64, _i64, _vp, _vp, _vp]),
    "ra_partial_fold": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i64, _i64, _i32, _f32, _i32,
                               _i64, _i64, _i64, _i64, _vp, _vp, _vp, _vp]),
    "ra_key_norm_max": (_i32, [_vp, _i32, _i32, _i32, _i64, _i32, _vp, _vp]),
    "ra_merge": (_i32, [_vp, _vp, _i32, _i64, _i32, _vp, _i32, _vp, _vp]),
    "ra_ring_forward": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i64, _i32, _f32, _i32, _i32,
                               _i32, _vp, _vp, _vp]),
    "ra_backward_delta": (_i32, [_vp, _vp, _i32, _i64, _i32, _vp, _vp]),
    "ra_partial_backward": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i64, _i64, _i32, _f32, _i32,
                                   _i64, _i64, _i64, _i64, _vp, _vp, _vp, _vp]),
    "ra_ring_backward_workspace_bytes": (_i64, [_i32, _i32, _i32, _i64, _i32]),
    "ra_ring_backward": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i64, _i32, _f32, _i32, _i32,
                                _i32, _vp, _vp, _vp, _vp, _i64, _vp]),
    "ra_ring_backward_noalloc": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i64, _i32, _f32, _i32,
                                        _i32, _i32, _vp, _vp, _vp, _vp]),
    "ra_status_string": (ctypes.c_char_p, [_i32]),
    "ra_get_device_error": (_i32, [_vp]),
    "ra_selftest_wait_timeout": (_i32, [_i64, _vp]),
    "ra_abi_version": (_i32, []),
}

_lock = threading.Lock()
_handle = None


class RaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


def load():
    """Load libra.so once and declare the C signatures. Raises if the library is missing."""
    global _handle
    with _lock:
        if _handle is None:
            if not os.path.exists(library_path):
                raise RuntimeError(
                    f"libra.so not found at {library_path}: build it with "
                    "`python -m sequence_softmax_b200.build` (there is no CPU fallback)")
            lib = ctypes.CDLL(library_path)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            if lib.ra_abi_version() != ABI_VERSION:
                raise RuntimeError(f"{library_path} implements ABI {lib.ra_abi_version()}, this binding "
                                   f"ABI {ABI_VERSION}: rebuild with `python -m sequence_softmax_b200.build`")
            _handle = lib
    return _handle


def status_string(status: int) -> str:
    return load().ra_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != RA_OK:
        raise RaError(status, what)


def _stream_ptr(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return RA_F32
    if t.dtype == torch.bfloat16:
        return RA_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _dev(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def get_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status code."""
    return load().ra_get_device_error(_stream_ptr(stream))


def selftest_wait_timeout(limit_ns: int = 50_000_000, stream=None, read: bool = True) -> int:
    """Launch the failure-detection self-test (a bounded wait that must run out); returns the
    device error status read afterwards (RA_ERR_TIMEOUT when detection works), or RA_OK
    without reading when ``read`` is False."""
    _check(load().ra_selftest_wait_timeout(int(limit_ns), _stream_ptr(stream)), "ra_selftest_wait_timeout")
    return get_device_error(stream) if read else RA_OK


def partial(q, k, v, causal: bool = False, scale: float | None = None,
            q_tok0: int = 0, q_tok_stride: int = 1, k_tok0: int = 0, k_tok_stride: int = 1,
            out=None, lse=None, stream=None):
    """One query block against one KV chunk -> (O_partial fp32 [B,H,Lq,d], lse fp32 [B,H,Lq])."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    if k.shape != (B, H, Lk, d) or v.shape != k.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("k and v must be [B, H, Lk, d] with q's B, H, d and dtype")
    scale = d ** -0.5 if scale is None else float(scale)
    out = torch.empty(B, H, Lq, d, device=q.device, dtype=torch.float32) if out is None else out
    lse = torch.empty(B, H, Lq, device=q.device, dtype=torch.float32) if lse is None else lse
    _dev(out, "out")
    _dev(lse, "lse")
    st = load().ra_partial(q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q), B, H, Lq, Lk, d, scale,
                           int(bool(causal)), q_tok0, q_tok_stride, k_tok0, k_tok_stride,
                           out.data_ptr(), lse.data_ptr(), _stream_ptr(stream))
    _check(st, "ra_partial")
    return out, lse


def partial_fold(q, k, v, o_state, lse_state, causal: bool = False, scale: float | None = None,
                 q_tok0: int = 0, q_tok_stride: int = 1, k_tok0: int = 0, k_tok_stride: int = 1,
                 k_norm_max=None, stream=None):
    """One query block against one KV chunk, merged in place into the running state
    (o_state fp32 [B,H,Lq,d], lse_state fp32 [B,H,Lq]); returns them. ``k_norm_max``
    (fp32 [B,H] from ``key_norm_max(k)``, or None) enables the row-max skip."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o_state, "o_state"), (lse_state, "lse_state")):
        _dev(t, n)
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    if k.shape != (B, H, Lk, d) or v.shape != k.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("k and v must be [B, H, Lk, d] with q's B, H, d and dtype")
    if o_state.shape != (B, H, Lq, d) or lse_state.shape != (B, H, Lq) or o_state.dtype != torch.float32 \
            or lse_state.dtype != torch.float32:
        raise ValueError("the state is o_state fp32 [B, H, Lq, d] and lse_state fp32 [B, H, Lq]")
    scale = d ** -0.5 if scale is None else float(scale)
    kmax_ptr = None
    if k_norm_max is not None:
        _dev(k_norm_max, "k_norm_max")
        if k_norm_max.shape != (B, H) or k_norm_max.dtype != torch.float32 or not k_norm_max.is_contiguous():
            raise ValueError("k_norm_max is a contiguous fp32 [B, H] tensor")
        kmax_ptr = k_norm_max.data_ptr()
    st = load().ra_partial_fold(q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q), B, H, Lq, Lk, d, scale,
                                int(bool(causal)), q_tok0, q_tok_stride, k_tok0, k_tok_stride,
                                o_state.data_ptr(), lse_state.data_ptr(), kmax_ptr, _stream_ptr(stream))
    _check(st, "ra_partial_fold")
    return o_state, lse_state


def key_norm_max(k, out=None, stream=None):
    """The largest L2 norm of each head's keys: k bf16 [B, H, Lk, d] -> fp32 [B, H]."""
    _dev(k, "k")
    B, H, Lk, d = k.shape
    out = torch.empty(B, H, device=k.device, dtype=torch.float32) if out is None else out
    _dev(out, "out")
    if out.shape != (B, H) or out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError("out is a contiguous fp32 [B, H] tensor")
    st = load().ra_key_norm_max(k.data_ptr(), _dtype_code(k), B, H, Lk, d, out.data_ptr(), _stream_ptr(stream))
    _check(st, "ra_key_norm_max")
    return out


def merge(o_parts, lse_parts, out_dtype=torch.bfloat16, with_lse: bool = True, out=None, lse=None,
          stream=None):
    """lse-weighted combination of n partial states.

    o_parts [n, ..., d] fp32, lse_parts [n, ...] fp32 -> (O [..., d] out_dtype, L [...] fp32 or None).
    """
    _dev(o_parts, "o_parts")
    _dev(lse_parts, "lse_parts")
    if o_parts.dtype != torch.float32 or lse_parts.dtype != torch.float32:
        raise TypeError("partial states are float32")
    n, d = o_parts.shape[0], o_parts.shape[-1]
    lead = tuple(o_parts.shape[1:-1])
    if tuple(lse_parts.shape) != (n, *lead):
        raise ValueError("lse_parts must be [n, ...] matching o_parts [n, ..., d]")
    rows = 1
    for x in lead:
        rows *= x
    out = torch.empty(*lead, d, device=o_parts.device, dtype=out_dtype) if out is None else out
    if with_lse and lse is None:
        lse = torch.empty(*lead, device=o_parts.device, dtype=torch.float32)
    _dev(out, "out")
    st = load().ra_merge(o_parts.data_ptr(), lse_parts.data_ptr(), n, rows, d, out.data_ptr(),
                         _dtype_code(out), lse.data_ptr() if with_lse else None, _stream_ptr(stream))
    _check(st, "ra_merge")
    return out, (lse if with_lse else None)


HOST_PIPELINE_GROUPS = 4


def _pipeline_bounds(BH: int, G: int) -> list[int]:
    """Group boundaries over BH (batch, head) rows for the host pipeline. Only the first
    group's input copy and the last group's output copy are not hidden behind a kernel, so
    those two groups get half the weight of the others (8 rows in 4 groups: 1, 3, 3, 1)."""
    if G <= 2:
        return [BH * g // G for g in range(G + 1)]
    w = [0.5] + [1.0] * (G - 2) + [0.5]
    tot, acc, bounds = sum(w), 0.0, [0]
    for x in w:
        acc += x
        bounds.append(min(BH, max(bounds[-1] + 1, round(BH * acc / tot))))
    bounds[-1] = BH
    return bounds


def _ring_forward_host(q, k, v, n_chunks, causal, layout, scale, return_lse, out, lse, stream):
    """ring_forward for host tensors: the (batch, head) rows are processed in up to
    HOST_PIPELINE_GROUPS groups, one library call each, so that the copy of group g + 1's
    inputs to the device and of group g - 1's outputs back to the host (on two copy streams)
    overlap group g's kernel. Heads are independent, so the result equals one call over all
    heads. With pinned host tensors the copies are asynchronous; otherwise they serialise."""
    for t, n in ((k, "k"), (v, "v")):
        if t.is_cuda or t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError(f"{n} must be a host tensor shaped and typed like q")
    if not all(t.is_contiguous() for t in (q, k, v)):
        raise ValueError("host q, k, v must be contiguous")
    dev = torch.device("cuda", torch.cuda.current_device())
    B, H, N, d = q.shape
    BH = B * H
    pin = q.is_pinned() and k.is_pinned() and v.is_pinned()
    o_h = torch.empty(q.shape, dtype=q.dtype, pin_memory=pin) if out is None else out
    l_h = None
    if return_lse:
        l_h = torch.empty(B, H, N, dtype=torch.float32, pin_memory=pin) if lse is None else lse
    if BH == 0 or N == 0:
        return o_h, l_h
    qf, kf, vf, of = (t.view(BH, N, d) for t in (q, k, v, o_h))
    lf = l_h.view(BH, N) if return_lse else None
    qd, kd, vd, od = (torch.empty(BH, N, d, dtype=q.dtype, device=dev) for _ in range(4))
    ld = torch.empty(BH, N, dtype=torch.float32, device=dev) if return_lse else None
    compute = torch.cuda.current_stream() if stream is None else stream
    h2d, d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    G = max(1, min(HOST_PIPELINE_GROUPS, BH))
    bounds = _pipeline_bounds(BH, G)
    for g in range(G):
        a, b = bounds[g], bounds[g + 1]
        if a == b:
            continue
        with torch.cuda.stream(h2d):
            for dst, src in ((qd, qf), (kd, kf), (vd, vf)):
                dst[a:b].copy_(src[a:b], non_blocking=pin)
            loaded = torch.cuda.Event()
            loaded.record(h2d)
        compute.wait_event(loaded)
        view = lambda t: t[a:b].view(1, b - a, N, d)  # noqa: E731
        ring_forward(view(qd), view(kd), view(vd), n_chunks, causal, layout, scale, return_lse, out=view(od),
                     lse=ld[a:b].view(1, b - a, N) if return_lse else None, stream=compute)
        done = torch.cuda.Event()
        done.record(compute)
        d2h.wait_event(done)
        with torch.cuda.stream(d2h):
            of[a:b].copy_(od[a:b], non_blocking=pin)
            if return_lse:
                lf[a:b].copy_(ld[a:b], non_blocking=pin)
    d2h.synchronize()
    compute.synchronize()
    return o_h, l_h


def ring_forward(q, k, v, n_chunks: int, causal: bool = False, layout: str = "contiguous",
                 scale: float | None = None, return_lse: bool = True, out=None, lse=None, stream=None):
    """Exact attention by the ordered ring over ``n_chunks`` virtual positions.

    q, k, v [B, H, N, d] (bf16 with d in {64, 128}, or fp32 with d <= 128), natural token order.
    Returns (O [B,H,N,d] in q's dtype, lse [B,H,N] fp32 or None). Host (CPU) tensors are
    accepted: they are copied to the current device group of heads by group, overlapped with
    the computation of the previous group, and the results are copied back to host memory
    before returning.
    """
    if not q.is_cuda:
        return _ring_forward_host(q, k, v, n_chunks, causal, layout, scale, return_lse, out, lse, stream)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
    B, H, N, d = q.shape
    if k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share shape [B, H, N, d] and dtype")
    if layout not in LAYOUTS:
        raise ValueError(f"layout must be one of {sorted(LAYOUTS)}")
    scale = d ** -0.5 if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    if return_lse and lse is None:
        lse = torch.empty(B, H, N, device=q.device, dtype=torch.float32)
    _dev(out, "out")
    st = load().ra_ring_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q), B, H, N, d, scale,
                                int(n_chunks), int(bool(causal)), LAYOUTS[layout], out.data_ptr(),
                                lse.data_ptr() if return_lse else None, _stream_ptr(stream))
    _check(st, "ra_ring_forward")
    return out, (lse if return_lse else None)


def backward_delta(o, d_o, out=None, stream=None):
    """D = rowsum(dO * O) -> fp32 [...] for o, d_o [..., d]."""
    _dev(o, "o")
    _dev(d_o, "d_o")
    if d_o.shape != o.shape or d_o.dtype != o.dtype:
        raise ValueError("o and d_o must share shape and dtype")
    d = o.shape[-1]
    rows = o.numel() // d if d else 0
    out = torch.empty(o.shape[:-1], device=o.device, dtype=torch.float32) if out is None else out
    _dev(out, "out")
    st = load().ra_backward_delta(o.data_ptr(), d_o.data_ptr(), _dtype_code(o), rows, d, out.data_ptr(),
                                  _stream_ptr(stream))
    _check(st, "ra_backward_delta")
    return out


def partial_backward(q, k, v, d_o, lse, delta, dq_acc, dk_acc, dv_acc, causal: bool = False,
                     scale: float | None = None, q_tok0: int = 0, q_tok_stride: int = 1, k_tok0: int = 0,
                     k_tok_stride: int = 1, stream=None):
    """Adds one (query block, KV chunk) pair's gradients to fp32 accumulators (in place).

    q, d_o [B,H,Lq,d]; k, v [B,H,Lk,d]; lse, delta [B,H,Lq] fp32 (final lse of the forward and
    D = rowsum(dO * O)); dq_acc [B,H,Lq,d], dk_acc / dv_acc [B,H,Lk,d] fp32.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (d_o, "d_o"), (lse, "lse"), (delta, "delta"),
                 (dq_acc, "dq_acc"), (dk_acc, "dk_acc"), (dv_acc, "dv_acc")):
        _dev(t, n)
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    if k.shape != (B, H, Lk, d) or v.shape != k.shape or d_o.shape != q.shape:
        raise ValueError("k, v must be [B, H, Lk, d] and d_o [B, H, Lq, d]")
    if any(t.dtype != q.dtype for t in (k, v, d_o)):
        raise ValueError("q, k, v, d_o must share a dtype")
    if any(t.dtype != torch.float32 for t in (lse, delta, dq_acc, dk_acc, dv_acc)):
        raise TypeError("lse, delta and the accumulators are float32")
    if dq_acc.shape != q.shape or dk_acc.shape != k.shape or dv_acc.shape != k.shape:
        raise ValueError("accumulators must match q / k shapes")
    scale = d ** -0.5 if scale is None else float(scale)
    st = load().ra_partial_backward(q.data_ptr(), k.data_ptr(), v.data_ptr(), d_o.data_ptr(), lse.data_ptr(),
                                    delta.data_ptr(), _dtype_code(q), B, H, Lq, Lk, d, scale, int(bool(causal)),
                                    q_tok0, q_tok_stride, k_tok0, k_tok_stride, dq_acc.data_ptr(),
                                    dk_acc.data_ptr(), dv_acc.data_ptr(), _stream_ptr(stream))
    _check(st, "ra_partial_backward")
    return dq_acc, dk_acc, dv_acc


def ring_backward_workspace_bytes(dtype, B: int, H: int, N: int, d: int) -> int:
    code = RA_BF16 if dtype == torch.bfloat16 else RA_F32
    return int(load().ra_ring_backward_workspace_bytes(code, B, H, N, d))


def ring_backward(q, k, v, o, d_o, lse, n_chunks: int, causal: bool = False, layout: str = "contiguous",
                  scale: float | None = None, workspace=None, out=None, stream=None):
    """Gradients (dQ, dK, dV) of ``ring_forward``'s output for upstream gradient d_o.

    q, k, v, o, d_o [B,H,N,d] in one dtype, lse [B,H,N] fp32 from ring_forward. ``workspace``
    (a uint8 CUDA tensor of at least ring_backward_workspace_bytes bytes) is allocated when
    not given; ``out`` may be a (dq, dk, dv) tuple of preallocated tensors.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (d_o, "d_o"), (lse, "lse")):
        _dev(t, n)
    B, H, N, d = q.shape
    if any(t.shape != q.shape or t.dtype != q.dtype for t in (k, v, o, d_o)):
        raise ValueError("q, k, v, o, d_o must share shape [B, H, N, d] and dtype")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N):
        raise ValueError("lse must be float32 [B, H, N]")
    if layout not in LAYOUTS:
        raise ValueError(f"layout must be one of {sorted(LAYOUTS)}")
    scale = d ** -0.5 if scale is None else float(scale)
    need = ring_backward_workspace_bytes(q.dtype, B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=q.device, dtype=torch.uint8)
    _dev(workspace, "workspace")
    dq, dk, dv = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)) if out is None else out
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _dev(t, n)
    st = load().ra_ring_backward(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), d_o.data_ptr(),
                                 lse.data_ptr(), _dtype_code(q), B, H, N, d, scale, int(n_chunks),
                                 int(bool(causal)), LAYOUTS[layout], dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                 workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                 _stream_ptr(stream))
    _check(st, "ra_ring_backward")
    return dq, dk, dv


def ring_backward_noalloc(q, k, v, o, d_o, lse, n_chunks: int, causal: bool = False, layout: str = "contiguous",
                          scale: float | None = None, out=None, stream=None):
    """``ring_backward`` through the entry point that allocates nothing on the device.

    For callers that cannot allocate device memory: the library's static scratch array
    replaces the workspace (4 bytes per query row, up to 2^24 rows). Pass ``out`` = (dq, dk, dv) preallocated tensors to allocate
    nothing here either. Calls on one device must not overlap on the GPU (they share the
    scratch); problems larger than the array raise RaError(RA_ERR_UNSUPPORTED).
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (d_o, "d_o"), (lse, "lse")):
        _dev(t, n)
    B, H, N, d = q.shape
    if any(t.shape != q.shape or t.dtype != q.dtype for t in (k, v, o, d_o)):
        raise ValueError("q, k, v, o, d_o must share shape [B, H, N, d] and dtype")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N):
        raise ValueError("lse must be float32 [B, H, N]")
    if layout not in LAYOUTS:
        raise ValueError(f"layout must be one of {sorted(LAYOUTS)}")
    scale = d ** -0.5 if scale is None else float(scale)
    dq, dk, dv = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)) if out is None else out
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _dev(t, n)
    st = load().ra_ring_backward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), d_o.data_ptr(),
                                         lse.data_ptr(), _dtype_code(q), B, H, N, d, scale, int(n_chunks),
                                         int(bool(causal)), LAYOUTS[layout], dq.data_ptr(), dk.data_ptr(),
                                         dv.data_ptr(), _stream_ptr(stream))
    _check(st, "ra_ring_backward_noalloc")
    return dq, dk, dv
