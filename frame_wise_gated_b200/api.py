"""Python binding of libgdnscan.so: argument marshalling only.

Every step of the frame scan runs in the library's CUDA kernels; this module
checks tensor dtypes/devices, allocates outputs and scratch with torch (device
memory and streams are all torch provides here) and passes raw pointers
through the C ABI declared in include/gdn.h. There is no CPU fallback: if the
library is missing, loading it raises.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgdnscan.so")

GDN_OK = 0
GDN_ERR_INVALID = -1
GDN_ERR_UNSUPPORTED = -2
GDN_ERR_CUDA = -3
GDN_ERR_TIMEOUT = -4
GDN_ERR_WORKSPACE = -5

BF16 = 0x1
REVERSE = 0x2
BLOCK_RESET = 0x4
SEQUENTIAL = 0x8
FUSED_PROLOGUE = 0x10
KEYS_SCALED = 0x20
FORCE_SIMT = 0x40
BIDIR = 0x80
FUSED_REPLAY = 0x1000000
CHUNKED = 0x2000000
NO_OVERLAP = 0x4000000
SAVE_FOR_BACKWARD = 0x10000000
UCPE = 0x20000000
REV_STATE_IN = 0x8000000


def make_block(n: int) -> int:
    return (n & 0xFF) << 8


def make_chunk(n: int) -> int:
    return (n & 0xFF) << 16


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: status {status} ({detail})")
        self.status = status


class GdnParams(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("beta", ctypes.c_void_p), ("gamma", ctypes.c_void_p), ("state_in", ctypes.c_void_p),
        ("out", ctypes.c_void_p), ("state_out", ctypes.c_void_p),
        ("out_rev", ctypes.c_void_p), ("state_out_rev", ctypes.c_void_p),
        ("w_q", ctypes.c_void_p), ("w_k", ctypes.c_void_p),
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int), ("S", ctypes.c_int),
        ("D", ctypes.c_int), ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int),
        ("eps", ctypes.c_float), ("rope_base", ctypes.c_float), ("flags", ctypes.c_uint),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("state_in_rev", ctypes.c_void_p),
        ("ucpe_q", ctypes.c_void_p),
        ("ucpe_k", ctypes.c_void_p),
    ]


class GdnBwdParams(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("beta", ctypes.c_void_p), ("gamma", ctypes.c_void_p), ("state_in", ctypes.c_void_p),
        ("d_out", ctypes.c_void_p), ("d_state_out", ctypes.c_void_p),
        ("dq", ctypes.c_void_p), ("dk", ctypes.c_void_p), ("dv", ctypes.c_void_p),
        ("dbeta", ctypes.c_void_p), ("dgamma", ctypes.c_void_p), ("d_state_in", ctypes.c_void_p),
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int), ("S", ctypes.c_int),
        ("D", ctypes.c_int), ("flags", ctypes.c_uint),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("saved_workspace", ctypes.c_void_p),
    ]


_P = ctypes.c_void_p
_I = ctypes.c_int
_U = ctypes.c_uint
_F = ctypes.c_float

# name -> (restype, argtypes); one entry per function declared in include/gdn.h
SIGNATURES = {
    "gdn_frame_scan_fwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _U, _P]),
    "gdn_qk_prologue": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _F, _U, _P]),
    "gdn_qk_prologue_ucpe": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _F,
                                  _U, _P]),
    "gdn_frame_scan_fwd_ex": (_I, [ctypes.POINTER(GdnParams), _P]),
    "gdn_frame_scan_fwd_static": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _U, _P]),
    "gdn_frame_scan_fwd_host": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _U, _I,
                                     _P]),
    "gdn_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _U]),
    "gdn_frame_scan_bwd": (_I, [ctypes.POINTER(GdnBwdParams), _P]),
    "gdn_cp_shard_composite": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _U, _P,
                                    ctypes.c_size_t, _P]),
    "gdn_cp_prefix": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "gdn_bwd_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _U]),
    "gdn_frame_contract": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _U, _P]),
    "gdn_chunk_composites": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _U, _P]),
    "gdn_check_device_status": (_I, [_P]),
    "gdn_selftest_wait": (_I, [_I, ctypes.c_longlong, _P]),
    "gdn_status_string": (ctypes.c_char_p, [_I]),
    "gdn_last_error": (ctypes.c_char_p, []),
    "gdn_launch_count": (ctypes.c_longlong, [_I]),
    "gdn_version": (_I, []),
    "gdn_profile_enable": (_I, [_I]),
    "gdn_fault_inject": (_I, [_I]),
    "gdn_rope_eval": (_I, [_I, _I, _F, _I, _P, _P]),
    "gdn_profile_read": (_I, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong), _I]),
}

PHASES = ("prologue", "contract", "compose", "prefix", "scan", "readout", "scan_readout",
          "contract_scan", "bwd_recompute", "bwd_w", "bwd_adjoint", "bwd_frame", "bwd_tokens",
          "bwd_dq")

_lib = None


def lib() -> ctypes.CDLL:
    """Loads libgdnscan.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise OSError(f"libgdnscan.so not built at {_LIB_PATH}; run "
                          "python -m frame_wise_gated_b200.build")
        L = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int, where: str) -> None:
    if status != GDN_OK:
        L = lib()
        detail = L.gdn_last_error().decode() or L.gdn_status_string(status).decode()
        raise GdnError(status, where, detail)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _want(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _want_states_outputs(q, state_in, out, state_out):
    """Checks caller-supplied state_in / out / state_out against q's sizes:
    a wrong dtype or size would make the kernels read or write past them."""
    B, H, T, S, D = q.shape
    if state_in is not None:
        _want(state_in, "state_in", torch.float32, (B, H, D, D))
    if out is not None:
        _want(out, "out", q.dtype, (B, H, T, S, D))
    if state_out is not None:
        _want(state_out, "state_out", torch.float32, (B, H, D, D))


def scan_flags(*, bf16: bool, reverse=False, block_reset=False, block=3, chunk=8,
               sequential=False, keys_scaled=False, force_simt=False, prologue=False,
               bidir=False, fused_replay=False, chunked=False, overlap=True,
               save_for_backward=False) -> int:
    """Flag word of the C ABI. Plan: sequential=True forces one chain per head,
    chunked=True the span-composed plan, neither lets the library choose;
    overlap=False keeps the chains out of the contraction's launch."""
    f = (BF16 if bf16 else 0) | make_block(block) | make_chunk(chunk)
    f |= CHUNKED if chunked else 0
    f |= 0 if overlap else NO_OVERLAP
    f |= FUSED_REPLAY if fused_replay else 0
    f |= REVERSE if reverse else 0
    f |= BLOCK_RESET if block_reset else 0
    f |= SEQUENTIAL if sequential else 0
    f |= KEYS_SCALED if keys_scaled else 0
    f |= FORCE_SIMT if force_simt else 0
    f |= FUSED_PROLOGUE if prologue else 0
    f |= BIDIR if bidir else 0
    f |= SAVE_FOR_BACKWARD if save_for_backward else 0
    return f


def workspace_bytes(B, H, T, S, D, flags) -> int:
    return int(lib().gdn_workspace_bytes(B, H, T, S, D, flags))


def frame_scan_fwd_ex(q, k, v, beta, gamma, state_in=None, *, reverse=False, block_reset=False,
                      block=3, chunk=8, sequential=False, keys_scaled=False, force_simt=False,
                      prologue=None, bidir=False, fused_replay=False, chunked=False,
                      overlap=True, out=None, state_out=None, out_rev=None, state_out_rev=None,
                      workspace=None, stream=None, state_in_rev=..., save_for_backward=False):
    """The frame scan through gdn_frame_scan_fwd_ex.

    q, k, v [B,H,T,S,D] (bf16 or fp32); beta [B,H,T,S] fp32; gamma [B,H,T]
    fp32; state_in [B,H,D,D] fp32 or None. prologue = dict(w_q, w_k, grid_h,
    grid_w[, eps, rope_base, ucpe_q, ucpe_k]) applies the fused
    RMSNorm/ReLU/key-scale/RoPE to raw q, k; with ucpe_q and ucpe_k
    ([B,T,S,4,4] fp32: D^T and D^-1 per token) the camera encoding takes
    channels [0, D/2) and the RoPE the rest (GDN_UCPE). Returns (out, state_out) or, with bidir, (out, state_out,
    out_rev, state_out_rev). With bidir, state_in_rev (a tensor or None)
    gives the reverse scan its own start state (GDN_REV_STATE_IN); left out,
    state_in seeds both directions. save_for_backward keeps what a later
    frame_scan_bwd(saved_workspace=workspace) reads (GDN_SAVE_FOR_BACKWARD)."""
    B, H, T, S, D = q.shape
    bf16 = q.dtype == torch.bfloat16
    if q.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("q must be bf16 or fp32")
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _want(t, n, q.dtype, (B, H, T, S, D))
    _want(beta, "beta", torch.float32, (B, H, T, S))
    _want(gamma, "gamma", torch.float32, (B, H, T))
    _want_states_outputs(q, state_in, out, state_out)
    if out_rev is not None:
        _want(out_rev, "out_rev", q.dtype, (B, H, T, S, D))
    if state_out_rev is not None:
        _want(state_out_rev, "state_out_rev", torch.float32, (B, H, D, D))
    flags = scan_flags(bf16=bf16, reverse=reverse, block_reset=block_reset, block=block,
                       chunk=chunk, sequential=sequential, keys_scaled=keys_scaled,
                       force_simt=force_simt, prologue=prologue is not None, bidir=bidir,
                       fused_replay=fused_replay, chunked=chunked, overlap=overlap,
                       save_for_backward=save_for_backward)
    out = torch.empty_like(q) if out is None else out
    state_out = torch.empty((B, H, D, D), device=q.device, dtype=torch.float32) \
        if state_out is None else state_out
    if bidir:
        out_rev = torch.empty_like(q) if out_rev is None else out_rev
        state_out_rev = torch.empty_like(state_out) if state_out_rev is None else state_out_rev
    need = workspace_bytes(B, H, T, S, D, flags)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=q.device, dtype=torch.uint8)
    p = GdnParams()
    p.q, p.k, p.v = _ptr(q), _ptr(k), _ptr(v)
    p.beta, p.gamma, p.state_in = _ptr(beta), _ptr(gamma), _ptr(state_in)
    p.out, p.state_out = _ptr(out), _ptr(state_out)
    p.out_rev, p.state_out_rev = _ptr(out_rev), _ptr(state_out_rev)
    if bidir and state_in_rev is not ...:
        if state_in_rev is not None:
            _want(state_in_rev, "state_in_rev", torch.float32, (B, H, D, D))
        p.state_in_rev = _ptr(state_in_rev)
        flags |= REV_STATE_IN
    if prologue is not None:
        _want(prologue["w_q"], "w_q", torch.float32, (D,))
        _want(prologue["w_k"], "w_k", torch.float32, (D,))
        p.w_q, p.w_k = _ptr(prologue["w_q"]), _ptr(prologue["w_k"])
        p.grid_h, p.grid_w = int(prologue["grid_h"]), int(prologue["grid_w"])
        if prologue.get("ucpe_q") is not None or prologue.get("ucpe_k") is not None:
            for n in ("ucpe_q", "ucpe_k"):
                _want(prologue[n], n, torch.float32, (B, T, S, 4, 4))
            p.ucpe_q, p.ucpe_k = _ptr(prologue["ucpe_q"]), _ptr(prologue["ucpe_k"])
            flags |= UCPE
        p.eps = float(prologue.get("eps", 1e-6))
        p.rope_base = float(prologue.get("rope_base", 10000.0))
    p.B, p.H, p.T, p.S, p.D = B, H, T, S, D
    p.flags = flags
    p.workspace = workspace.data_ptr()
    p.workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib().gdn_frame_scan_fwd_ex(ctypes.byref(p), _stream(stream)), "gdn_frame_scan_fwd_ex")
    if bidir:
        return out, state_out, out_rev, state_out_rev
    return out, state_out


def frame_scan_fwd(q, k, v, beta, gamma, state_in=None, *, reverse=False, block_reset=False,
                   block=3, chunk=8, sequential=False, keys_scaled=False, force_simt=False,
                   chunked=False, overlap=True, out=None, state_out=None, stream=None):
    """The frame scan through gdn_frame_scan_fwd (scratch allocated by the
    library, stream-ordered). Returns (out, state_out)."""
    B, H, T, S, D = q.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _want(t, n, q.dtype, (B, H, T, S, D))
    _want(beta, "beta", torch.float32, (B, H, T, S))
    _want(gamma, "gamma", torch.float32, (B, H, T))
    _want_states_outputs(q, state_in, out, state_out)
    flags = scan_flags(bf16=q.dtype == torch.bfloat16, reverse=reverse, block_reset=block_reset,
                       block=block, chunk=chunk, sequential=sequential,
                       keys_scaled=keys_scaled, force_simt=force_simt, chunked=chunked,
                       overlap=overlap)
    out = torch.empty_like(q) if out is None else out
    state_out = torch.empty((B, H, D, D), device=q.device, dtype=torch.float32) \
        if state_out is None else state_out
    _check(lib().gdn_frame_scan_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(gamma),
                                    _ptr(state_in), _ptr(out), _ptr(state_out),
                                    B, H, T, S, D, flags, _stream(stream)), "gdn_frame_scan_fwd")
    return out, state_out


def frame_scan_fwd_host(q, k, v, beta, gamma, state_in=None, *, out=None, state_out=None,
                        heads_per_chunk=2, device=None, **plan):
    """The scan over HOST tensors through gdn_frame_scan_fwd_host: the library
    streams the heads through the GPU in chunks (copies in, scans and copies
    out overlapping on three streams; pinned memory for full overlap) and
    returns once the results are in host memory.

    q, k, v [B,H,T,S,D] bf16 or fp32; beta [B,H,T,S], gamma [B,H,T],
    state_in [B,H,D,D] (or None), all contiguous host tensors. plan: the
    scan-plan keywords of frame_scan_fwd (reverse, block_reset, block, chunk,
    sequential, chunked, overlap, keys_scaled, force_simt). Returns host
    (out, state_out)."""
    B, H, T, S, D = q.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if t.is_cuda or t.shape != q.shape or t.dtype != q.dtype or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous host tensor shaped and typed like q")
    shapes = [(beta, "beta", (B, H, T, S)), (gamma, "gamma", (B, H, T))]
    if state_in is not None:
        shapes.append((state_in, "state_in", (B, H, D, D)))
    out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True) if out is None else out
    state_out = torch.empty((B, H, D, D), dtype=torch.float32, pin_memory=True) \
        if state_out is None else state_out
    shapes.append((state_out, "state_out", (B, H, D, D)))
    for t, n, shp in shapes:
        if t.is_cuda or tuple(t.shape) != shp or t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous fp32 host tensor of shape {shp}")
    if out.is_cuda or out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous():
        raise ValueError("out must be a contiguous host tensor shaped and typed like q")
    flags = scan_flags(bf16=q.dtype == torch.bfloat16, **plan)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _check(lib().gdn_frame_scan_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(gamma),
                                             _ptr(state_in), _ptr(out), _ptr(state_out),
                                             B, H, T, S, D, flags, int(heads_per_chunk),
                                             _stream(torch.cuda.current_stream(dev))),
               "gdn_frame_scan_fwd_host")
    return out, state_out

def frame_scan_bwd(q, k, v, beta, gamma, state_in, d_out, d_state_out=None, *, reverse=False,
                   block_reset=False, block=3, keys_scaled=False, want_state_in_grad=True,
                   force_simt=False, saved_workspace=None, workspace=None, grads=None,
                   stream=None):
    """Gradients through the frame scan (gdn_frame_scan_bwd): given
    d_out = dL/dO [B,H,T,S,D] and d_state_out = dL/d(state_out) [B,H,D,D]
    (or None), returns (dq, dk, dv, dbeta, dgamma, d_state_in) for the scan
    with the same flags (d_state_in None unless want_state_in_grad).
    saved_workspace: the workspace tensor of a frame_scan_fwd_ex call on the
    same inputs and flags (bf16, D = 128), reused instead of recomputing.
    grads: optional dict of caller-owned output tensors (dq, dk, dv, dbeta,
    dgamma, d_state_in) to write into instead of allocating."""
    B, H, T, S, D = q.shape
    bf16 = q.dtype == torch.bfloat16
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (d_out, "d_out")):
        _want(t, n, q.dtype, (B, H, T, S, D))
    _want(beta, "beta", torch.float32, (B, H, T, S))
    _want(gamma, "gamma", torch.float32, (B, H, T))
    if state_in is not None:
        _want(state_in, "state_in", torch.float32, (B, H, D, D))
    if d_state_out is not None:
        _want(d_state_out, "d_state_out", torch.float32, (B, H, D, D))
    flags = scan_flags(bf16=bf16, reverse=reverse, block_reset=block_reset, block=block,
                       keys_scaled=keys_scaled, force_simt=force_simt)
    flags &= ~(CHUNKED | NO_OVERLAP | 0xFF0000)  # plan bits do not apply to the backward
    g = dict(grads or {})
    dq = g.get("dq", None)
    dq = torch.empty_like(q) if dq is None else dq
    dk = g.get("dk", None)
    dk = torch.empty_like(k) if dk is None else dk
    dv = g.get("dv", None)
    dv = torch.empty_like(v) if dv is None else dv
    dbeta = g.get("dbeta", None)
    dbeta = torch.empty_like(beta) if dbeta is None else dbeta
    dgamma = g.get("dgamma", None)
    dgamma = torch.empty_like(gamma) if dgamma is None else dgamma
    ds0 = g.get("d_state_in", None)
    if ds0 is None and want_state_in_grad:
        ds0 = torch.empty((B, H, D, D), device=q.device, dtype=torch.float32)
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _want(t, n, q.dtype, (B, H, T, S, D))
    _want(dbeta, "dbeta", torch.float32, (B, H, T, S))
    _want(dgamma, "dgamma", torch.float32, (B, H, T))
    if ds0 is not None:
        _want(ds0, "d_state_in", torch.float32, (B, H, D, D))
    need = int(lib().gdn_bwd_workspace_bytes(B, H, T, S, D, flags))
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=q.device, dtype=torch.uint8)
    p = GdnBwdParams()
    p.q, p.k, p.v = _ptr(q), _ptr(k), _ptr(v)
    p.beta, p.gamma, p.state_in = _ptr(beta), _ptr(gamma), _ptr(state_in)
    p.d_out, p.d_state_out = _ptr(d_out), _ptr(d_state_out)
    p.dq, p.dk, p.dv = _ptr(dq), _ptr(dk), _ptr(dv)
    p.dbeta, p.dgamma, p.d_state_in = _ptr(dbeta), _ptr(dgamma), _ptr(ds0)
    p.B, p.H, p.T, p.S, p.D = B, H, T, S, D
    p.flags = flags
    p.workspace = workspace.data_ptr()
    p.workspace_bytes = workspace.numel() * workspace.element_size()
    p.saved_workspace = _ptr(saved_workspace)
    _check(lib().gdn_frame_scan_bwd(ctypes.byref(p), _stream(stream)), "gdn_frame_scan_bwd")
    return dq, dk, dv, dbeta, dgamma, ds0


def cp_shard_composite(k, v, beta, gamma, *, keys_scaled=False, force_simt=False,
                       workspace=None, stream=None):
    """This rank's frames as one affine map per head (gdn_cp_shard_composite):
    returns E, H [B,H,D,D] and g [B,H] with S_end = g (S_start - S_start E) + H."""
    B, H, T, S, D = k.shape
    _want(v, "v", k.dtype, (B, H, T, S, D))
    _want(beta, "beta", torch.float32, (B, H, T, S))
    _want(gamma, "gamma", torch.float32, (B, H, T))
    flags = scan_flags(bf16=k.dtype == torch.bfloat16, keys_scaled=keys_scaled,
                       force_simt=force_simt)
    E = torch.empty((B, H, D, D), device=k.device, dtype=torch.float32)
    Hm = torch.empty_like(E)
    g = torch.empty((B, H), device=k.device, dtype=torch.float32)
    need = workspace_bytes(B, H, T, S, D, flags)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=k.device, dtype=torch.uint8)
    _check(lib().gdn_cp_shard_composite(_ptr(k), _ptr(v), _ptr(beta), _ptr(gamma), _ptr(E),
                                        _ptr(Hm), _ptr(g), B, H, T, S, D, flags,
                                        workspace.data_ptr(),
                                        workspace.numel() * workspace.element_size(),
                                        _stream(stream)), "gdn_cp_shard_composite")
    return E, Hm, g


def cp_prefix(E_all, H_all, g_all, state_in, r, *, stream=None):
    """Start state of rank r (gdn_cp_prefix) from the gathered maps
    E_all, H_all [R,B,H,D,D], g_all [R,B,H]; state_in [B,H,D,D] or None."""
    R, B, H, D = E_all.shape[0], E_all.shape[1], E_all.shape[2], E_all.shape[3]
    _want(E_all, "E_all", torch.float32, (R, B, H, D, D))
    _want(H_all, "H_all", torch.float32, (R, B, H, D, D))
    _want(g_all, "g_all", torch.float32, (R, B, H))
    if state_in is not None:
        _want(state_in, "state_in", torch.float32, (B, H, D, D))
    out = torch.empty((B, H, D, D), device=E_all.device, dtype=torch.float32)
    _check(lib().gdn_cp_prefix(_ptr(E_all), _ptr(H_all), _ptr(g_all), _ptr(state_in), _ptr(out),
                               R, int(r), B * H, D, _stream(stream)), "gdn_cp_prefix")
    return out


STATIC_SCRATCH_BYTES = 32 << 20


def frame_scan_fwd_static(q, k, v, beta, gamma, state_in=None, *, reverse=False,
                          block_reset=False, block=3, chunk=8, sequential=False,
                          keys_scaled=False, force_simt=False, chunked=False, overlap=True,
                          out=None, state_out=None, stream=None):
    """The frame scan through gdn_frame_scan_fwd_static: for callers that must
    not allocate device memory per call (e.g. a streaming loop running one
    short block of frames at a time). Scratch is the library's fixed 32 MiB
    device array; outputs are allocated here only when not passed in.
    Returns (out, state_out)."""
    B, H, T, S, D = q.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _want(t, n, q.dtype, (B, H, T, S, D))
    _want(beta, "beta", torch.float32, (B, H, T, S))
    _want(gamma, "gamma", torch.float32, (B, H, T))
    _want_states_outputs(q, state_in, out, state_out)
    flags = scan_flags(bf16=q.dtype == torch.bfloat16, reverse=reverse, block_reset=block_reset,
                       block=block, chunk=chunk, sequential=sequential,
                       keys_scaled=keys_scaled, force_simt=force_simt, chunked=chunked,
                       overlap=overlap)
    out = torch.empty_like(q) if out is None else out
    state_out = torch.empty((B, H, D, D), device=q.device, dtype=torch.float32) \
        if state_out is None else state_out
    _check(lib().gdn_frame_scan_fwd_static(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(gamma),
                                           _ptr(state_in), _ptr(out), _ptr(state_out),
                                           B, H, T, S, D, flags, _stream(stream)),
           "gdn_frame_scan_fwd_static")
    return out, state_out


def qk_prologue(q_raw, k_raw, w_q, w_k, grid_h, grid_w, *, eps=1e-6, rope_base=10000.0,
                ucpe=None, stream=None):
    """RMSNorm -> ReLU -> key scale -> 2-D RoPE on raw q, k [B,H,T,S,D];
    with ucpe = (ucpe_q, ucpe_k) ([B,T,S,4,4] fp32) the camera encoding takes
    channels [0, D/2) and the RoPE the rest (gdn_qk_prologue_ucpe)."""
    B, H, T, S, D = q_raw.shape
    _want(q_raw, "q_raw", None, (B, H, T, S, D))
    _want(k_raw, "k_raw", q_raw.dtype, (B, H, T, S, D))
    _want(w_q, "w_q", torch.float32, (D,))
    _want(w_k, "w_k", torch.float32, (D,))
    q_out, k_out = torch.empty_like(q_raw), torch.empty_like(k_raw)
    flags = BF16 if q_raw.dtype == torch.bfloat16 else 0
    if ucpe is None:
        _check(lib().gdn_qk_prologue(_ptr(q_raw), _ptr(k_raw), _ptr(w_q), _ptr(w_k),
                                     _ptr(q_out), _ptr(k_out), B, H, T, grid_h, grid_w, D, eps,
                                     rope_base, flags, _stream(stream)), "gdn_qk_prologue")
        return q_out, k_out
    for t, n in zip(ucpe, ("ucpe_q", "ucpe_k")):
        _want(t, n, torch.float32, (B, T, S, 4, 4))
    _check(lib().gdn_qk_prologue_ucpe(_ptr(q_raw), _ptr(k_raw), _ptr(w_q), _ptr(w_k),
                                      _ptr(ucpe[0]), _ptr(ucpe[1]), _ptr(q_out), _ptr(k_out),
                                      B, H, T, grid_h, grid_w, D, eps, rope_base, flags,
                                      _stream(stream)), "gdn_qk_prologue_ucpe")
    return q_out, k_out


def frame_contract(k, v, beta, *, keys_scaled=False, force_simt=False, stream=None):
    """Step a2 alone: A, U [N,D,D] fp32 from k, v [N,S,D] and beta [N,S]."""
    N, S, D = k.shape
    _want(k, "k", None, (N, S, D))
    _want(v, "v", k.dtype, (N, S, D))
    _want(beta, "beta", torch.float32, (N, S))
    A = torch.empty((N, D, D), device=k.device, dtype=torch.float32)
    U = torch.empty_like(A)
    flags = (BF16 if k.dtype == torch.bfloat16 else 0) | (KEYS_SCALED if keys_scaled else 0) | \
        (FORCE_SIMT if force_simt else 0)
    _check(lib().gdn_frame_contract(_ptr(k), _ptr(v), _ptr(beta), _ptr(A), _ptr(U), N, S, D,
                                    flags, _stream(stream)), "gdn_frame_contract")
    return A, U


def chunk_composites(A, U, gamma, L, *, force_simt=False, stream=None):
    """Step a3 alone: per span of L frames, E, H [N,D,D] and g [N]."""
    NL, D, _ = A.shape
    N = NL // L
    _want(A, "A", torch.float32, (N * L, D, D))
    _want(U, "U", torch.float32, (N * L, D, D))
    _want(gamma, "gamma", torch.float32, (N * L,))
    E = torch.empty((N, D, D), device=A.device, dtype=torch.float32)
    Hc = torch.empty_like(E)
    g = torch.empty((N,), device=A.device, dtype=torch.float32)
    _check(lib().gdn_chunk_composites(_ptr(A), _ptr(U), _ptr(gamma), _ptr(E), _ptr(Hc), _ptr(g),
                                      N, L, D, FORCE_SIMT if force_simt else 0, _stream(stream)),
           "gdn_chunk_composites")
    return E, Hc, g


def check_device_status(stream=None) -> None:
    _check(lib().gdn_check_device_status(_stream(stream)), "gdn_check_device_status")


def fault_inject(n: int) -> int:
    """Arms host-side fault injection: the next n scan calls on this thread
    fail with GDN_ERR_CUDA before launching. Returns the previous pending count."""
    return int(lib().gdn_fault_inject(int(n)))


def launch_count(reset: bool = False) -> int:
    return int(lib().gdn_launch_count(1 if reset else 0))


def profile_enable(on: bool) -> None:
    lib().gdn_profile_enable(1 if on else 0)


def profile_read() -> dict:
    """Per-phase kernel time (ms) and launch count recorded since profile_enable(True)."""
    n = len(PHASES)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_longlong * n)()
    r = lib().gdn_profile_read(ms, cnt, n)
    if r < 0:
        _check(r, "gdn_profile_read")
    return {PHASES[i]: (ms[i], cnt[i]) for i in range(r)}


def selftest_wait(arrive: bool, limit_ns: int = 1_000_000, stream=None) -> None:
    """Launches the bounded-wait self test (see gdn_selftest_wait)."""
    _check(lib().gdn_selftest_wait(1 if arrive else 0, int(limit_ns), _stream(stream)),
           "gdn_selftest_wait")
