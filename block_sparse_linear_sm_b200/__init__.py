"""Python binding of the sparse+linear attention C ABI (include/sla.h).

Argument marshalling only: every step of the layer runs in the CUDA kernels of
libsla.so. The functions keep the C names; tensors are torch CUDA tensors (or
raw device addresses as int), the stream is torch's current stream unless one
is given. A missing library raises instead of falling back to anything.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

from . import workloads  # noqa: F401  (seeded inputs; no layer arithmetic)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsla.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "sla.h")

SLA_OK = 0
SLA_ERR_INVALID_ARG = 1
SLA_ERR_UNSUPPORTED = 2
SLA_ERR_WORKSPACE = 3
SLA_ERR_CUDA = 4
SLA_ERR_DEVICE_TIMEOUT = 5
SLA_ERR_DEVICE_CHECK = 6

SLA_MODE_THREEWAY = 0
SLA_MODE_TOPN_WINDOW = 1


class sla_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "H", "H_kv", "N", "N_valid", "d", "block", "mode", "k_h", "k_l", "top_n",
                 "window", "causal", "has_proj", "proj_per_head", "has_gate", "smooth_k",
                 "linear_all", "cos_filter")] + [("scale", ctypes.c_float), ("cos_theta", ctypes.c_float)] + \
        [(n, ctypes.c_int32) for n in ("nsa_branches", "cmp_block", "cmp_stride")]


class SlaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C-ABI library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m block_sparse_linear_sm_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, S, I32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
        C = ctypes.POINTER(sla_config)
        L.sla_validate_config.argtypes = [C]
        L.sla_validate_config.restype = ctypes.c_int
        L.sla_workspace_bytes.argtypes = [C]
        L.sla_workspace_bytes.restype = S
        L.sla_route.argtypes = [P, P, C, P, P, P, P, S, P]
        L.sla_route.restype = ctypes.c_int
        L.sla_forward.argtypes = [P, P, P, P, P, C, P, P, P, S, P]
        L.sla_forward.restype = ctypes.c_int
        L.sla_forward_blocks.argtypes = [P, P, P, P, P, C, I32, I32, P, P, P, S, P]
        L.sla_forward_blocks.restype = ctypes.c_int
        L.sla_forward_timed.argtypes = [P, P, P, P, P, C, P, P, P, S, P,
                                        ctypes.POINTER(ctypes.c_void_p), I32]
        L.sla_forward_timed.restype = ctypes.c_int
        L.sla_num_stages.argtypes = [C]
        L.sla_num_stages.restype = I32
        L.sla_stage_name.argtypes = [C, I32]
        L.sla_stage_name.restype = ctypes.c_char_p
        L.sla_check_device_status.argtypes = [P, P, ctypes.POINTER(I32)]
        L.sla_check_device_status.restype = ctypes.c_int
        L.sla_hilbert_order.argtypes = [I32, I32, I32, ctypes.POINTER(I32)]
        L.sla_hilbert_order.restype = ctypes.c_int
        L.sla_permute_tokens.argtypes = [P, P, P, I32, I32, I32, I32, I32, P]
        L.sla_permute_tokens.restype = ctypes.c_int
        L.sla_selftest_wait_timeout.argtypes = [P, S, ctypes.c_int64, P]
        L.sla_selftest_wait_timeout.restype = ctypes.c_int
        L.sla_backward_workspace_bytes.argtypes = [C]
        L.sla_backward_workspace_bytes.restype = S
        bwd = [P, P, P, P, P, C, P, P, P, P, P, P, P, P, S, P, S, P]
        L.sla_backward.argtypes = bwd
        L.sla_backward.restype = ctypes.c_int
        L.sla_backward_timed.argtypes = bwd + [ctypes.POINTER(ctypes.c_void_p), I32]
        L.sla_backward_timed.restype = ctypes.c_int
        L.sla_backward_num_stages.argtypes = [C]
        L.sla_backward_num_stages.restype = I32
        L.sla_backward_stage_name.argtypes = [C, I32]
        L.sla_backward_stage_name.restype = ctypes.c_char_p
        L.sla_status_string.argtypes = [ctypes.c_int]
        L.sla_status_string.restype = ctypes.c_char_p
        L.sla_version.argtypes = []
        L.sla_version.restype = ctypes.c_char_p
        L.sla_forward_host_device_bytes.argtypes = [C, I32]
        L.sla_forward_host_device_bytes.restype = S
        L.sla_forward_host.argtypes = [P, P, P, P, P, C, P, I32, P, S, P, P, P]
        L.sla_forward_host.restype = ctypes.c_int
        L.sla_route_noalloc.argtypes = [P, P, C, P, P, P, P]
        L.sla_route_noalloc.restype = ctypes.c_int
        L.sla_route_noalloc_status.argtypes = [P, ctypes.POINTER(I32)]
        L.sla_route_noalloc_status.restype = ctypes.c_int
        _lib = L
    return _lib


def make_config(c) -> sla_config:
    """sla_config from any object with the same field names (e.g. workloads.LayerConfig)."""
    cfg = sla_config()
    for name, _ in sla_config._fields_:
        setattr(cfg, name, getattr(c, name))
    return cfg


def _cfg(c) -> sla_config:
    return c if isinstance(c, sla_config) else make_config(c)


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not x.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not x.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != SLA_OK:
        raise SlaError(status, where)


def status_string(status: int) -> str:
    return lib().sla_status_string(status).decode()


def sla_status_string(status: int) -> str:
    return status_string(status)


def sla_validate_config(c) -> int:
    return lib().sla_validate_config(ctypes.byref(_cfg(c)))


def sla_workspace_bytes(c) -> int:
    return int(lib().sla_workspace_bytes(ctypes.byref(_cfg(c))))


def sla_num_stages(c) -> int:
    return int(lib().sla_num_stages(ctypes.byref(_cfg(c))))


def sla_stage_names(c) -> list:
    cfg = _cfg(c)
    n = lib().sla_num_stages(ctypes.byref(cfg))
    return [lib().sla_stage_name(ctypes.byref(cfg), i).decode() for i in range(max(n, 0))]


def sla_route(q, k, c, mask_out, crit_idx, neg_idx, ws, stream=None) -> None:
    cfg = _cfg(c)
    ws_bytes = ws.numel() * ws.element_size() if hasattr(ws, "numel") else int(ws[1])
    ws_ptr = _ptr(ws) if hasattr(ws, "numel") else ws[0]
    _check(lib().sla_route(_ptr(q), _ptr(k), ctypes.byref(cfg), _ptr(mask_out), _ptr(crit_idx),
                           _ptr(neg_idx), ws_ptr, ws_bytes, _stream(stream)), "sla_route")


def sla_forward(q, k, v, w_p, w_g, c, out, mask_out, ws, stream=None) -> None:
    cfg = _cfg(c)
    ws_bytes = ws.numel() * ws.element_size()
    _check(lib().sla_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(w_p), _ptr(w_g), ctypes.byref(cfg),
                             _ptr(out), _ptr(mask_out), _ptr(ws), ws_bytes, _stream(stream)),
           "sla_forward")


def sla_forward_blocks(q, k, v, w_p, w_g, c, qb_begin, qb_end, out, mask_out, ws, stream=None) -> None:
    """sla_forward writing only the output rows of query blocks [qb_begin, qb_end)."""
    cfg = _cfg(c)
    ws_bytes = ws.numel() * ws.element_size()
    _check(lib().sla_forward_blocks(_ptr(q), _ptr(k), _ptr(v), _ptr(w_p), _ptr(w_g), ctypes.byref(cfg),
                                    int(qb_begin), int(qb_end), _ptr(out), _ptr(mask_out), _ptr(ws), ws_bytes,
                                    _stream(stream)), "sla_forward_blocks")


def sla_forward_timed(q, k, v, w_p, w_g, c, out, mask_out, ws, events, stream=None) -> None:
    """events: torch.cuda.Event(enable_timing=True) list of length sla_num_stages(c) + 1."""
    cfg = _cfg(c)
    for e in events:
        if e.cuda_event == 0:  # torch creates the CUDA event on first record
            e.record()
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    ws_bytes = ws.numel() * ws.element_size()
    _check(lib().sla_forward_timed(_ptr(q), _ptr(k), _ptr(v), _ptr(w_p), _ptr(w_g),
                                   ctypes.byref(cfg), _ptr(out), _ptr(mask_out), _ptr(ws),
                                   ws_bytes, _stream(stream), arr, len(events)),
           "sla_forward_timed")


def _host_ptr(x) -> Optional[int]:
    if isinstance(x, int):
        return x
    if x.is_cuda:
        raise ValueError("tensor must live in host memory")
    if not x.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return x.data_ptr()


def sla_forward_host_device_bytes(c, n_chunks: int) -> int:
    cfg = _cfg(c)
    return int(lib().sla_forward_host_device_bytes(ctypes.byref(cfg), n_chunks))


def sla_forward_host(q_host, k_host, v_host, w_p, w_g, c, out_host, n_chunks, dev, stream=None,
                     h2d_stream=None, d2h_stream=None) -> None:
    """The layer on host tensors (q/k/v/out in host memory, ideally pinned; w_p, w_g and the
    arena ``dev`` of sla_forward_host_device_bytes(c, n_chunks) bytes on the device)."""
    cfg = _cfg(c)
    dev_bytes = dev.numel() * dev.element_size()
    s = _stream(stream)
    _check(lib().sla_forward_host(_host_ptr(q_host), _host_ptr(k_host), _host_ptr(v_host), _ptr(w_p),
                                  _ptr(w_g), ctypes.byref(cfg), _host_ptr(out_host), n_chunks, _ptr(dev),
                                  dev_bytes, s, s if h2d_stream is None else _stream(h2d_stream),
                                  s if d2h_stream is None else _stream(d2h_stream)),
           "sla_forward_host")


def sla_backward_workspace_bytes(c) -> int:
    cfg = _cfg(c)
    return int(lib().sla_backward_workspace_bytes(ctypes.byref(cfg)))


def sla_backward_num_stages(c) -> int:
    cfg = _cfg(c)
    return int(lib().sla_backward_num_stages(ctypes.byref(cfg)))


def sla_backward_stage_names(c) -> list:
    cfg = _cfg(c)
    n = lib().sla_backward_num_stages(ctypes.byref(cfg))
    return [lib().sla_backward_stage_name(ctypes.byref(cfg), i).decode() for i in range(max(n, 0))]


def _bwd_args(q, k, v, w_p, w_g, c, out, dout, dq, dk, dv, dw_p, dw_g, ws, bws, stream):
    return (_ptr(q), _ptr(k), _ptr(v), _ptr(w_p), _ptr(w_g), ctypes.byref(_cfg(c)), _ptr(out), _ptr(dout),
            _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dw_p), _ptr(dw_g), _ptr(ws), ws.numel() * ws.element_size(),
            _ptr(bws), bws.numel() * bws.element_size(), _stream(stream))


def sla_backward(q, k, v, w_p, w_g, c, out, dout, dq, dk, dv, dw_p, dw_g, ws, bws, stream=None) -> None:
    """Gradients of sum(out * dout); ws is the matching sla_forward call's workspace."""
    _check(lib().sla_backward(*_bwd_args(q, k, v, w_p, w_g, c, out, dout, dq, dk, dv, dw_p, dw_g, ws, bws,
                                         stream)), "sla_backward")


def sla_backward_timed(q, k, v, w_p, w_g, c, out, dout, dq, dk, dv, dw_p, dw_g, ws, bws, events,
                       stream=None) -> None:
    """events: torch.cuda.Event(enable_timing=True) list of length sla_backward_num_stages(c) + 1."""
    for e in events:
        if e.cuda_event == 0:
            e.record()
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    _check(lib().sla_backward_timed(*_bwd_args(q, k, v, w_p, w_g, c, out, dout, dq, dk, dv, dw_p, dw_g, ws,
                                               bws, stream), arr, len(events)), "sla_backward_timed")


def sla_route_noalloc(q, k, c, mask_out, crit_idx, neg_idx, stream=None) -> None:
    """sla_route without a workspace: its scratch is the library's static device array."""
    cfg = _cfg(c)
    _check(lib().sla_route_noalloc(_ptr(q), _ptr(k), ctypes.byref(cfg), _ptr(mask_out), _ptr(crit_idx),
                                   _ptr(neg_idx), _stream(stream)), "sla_route_noalloc")


def sla_route_noalloc_status(stream=None) -> tuple:
    """(status, detail) of the last sla_route_noalloc on this device, after synchronising the
    stream; clears the status word."""
    detail = ctypes.c_int32(0)
    st = lib().sla_route_noalloc_status(_stream(stream), ctypes.byref(detail))
    return int(st), int(detail.value)


def sla_check_device_status(ws, stream=None) -> tuple:
    """(status, detail) after synchronising the stream; clears the device status word."""
    detail = ctypes.c_int32(0)
    st = lib().sla_check_device_status(_ptr(ws), _stream(stream), ctypes.byref(detail))
    return int(st), int(detail.value)


def sla_selftest_wait_timeout(ws, limit_ns: int, stream=None) -> None:
    """Enqueue the failure-detection self-test: a bounded wait that runs out and is
    recorded in ws's status word (read it with sla_check_device_status)."""
    nbytes = ws.numel() * ws.element_size() if hasattr(ws, "numel") else 256
    _check(lib().sla_selftest_wait_timeout(_ptr(ws), nbytes, int(limit_ns), _stream(stream)),
           "sla_selftest_wait_timeout")


def sla_hilbert_order(t: int, h: int, w: int):
    """Raster indices of the (t, h, w) grid's tokens in Hilbert-curve order (numpy int32)."""
    import numpy as np
    out = np.empty(t * h * w, dtype=np.int32)
    _check(lib().sla_hilbert_order(t, h, w, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))),
           "sla_hilbert_order")
    return out


def sla_permute_tokens(x, y, order, inverse: bool = False, stream=None) -> None:
    """y[..., n, :] = x[..., order[n], :] for n < len(order) (inverse: the scatter back);
    x, y: bf16 [..., n_tok, d] CUDA tensors, order: int32 CUDA tensor."""
    n_tok, d = x.shape[-2], x.shape[-1]
    rows = x.numel() // (n_tok * d)
    _check(lib().sla_permute_tokens(_ptr(x), _ptr(y), _ptr(order), order.numel(), rows, n_tok, d,
                                    1 if inverse else 0, _stream(stream)), "sla_permute_tokens")


def sla_version() -> str:
    return lib().sla_version().decode()
