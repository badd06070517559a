"""Thin ctypes binding of libsla2.so (the C ABI in include/sla2.h).

Argument marshalling only: every step of the forward pass runs in the CUDA
kernels of the library. PyTorch provides device memory and streams. There is
no CPU fallback: if the library or a CUDA device is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsla2.so")

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "workspace", 4: "CUDA error",
          5: "device wait timed out"}


class Sla2Error(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: status {code} ({STATUS.get(code, '?')})")
        self.code = code


class Desc(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int),
        ("quantize", ctypes.c_int), ("out_dtype", ctypes.c_int),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("status", ctypes.c_void_p),
        ("dbg_scores", ctypes.c_void_p), ("dbg_os", ctypes.c_void_p), ("dbg_ol", ctypes.c_void_p),
        ("dbg_qhat", ctypes.c_void_p), ("dbg_khat", ctypes.c_void_p), ("dbg_vhat", ctypes.c_void_p),
        ("dbg_qscale", ctypes.c_void_p), ("dbg_kscale", ctypes.c_void_p), ("dbg_vscale", ctypes.c_void_p),
        ("dbg_mask", ctypes.c_void_p), ("dbg_idx", ctypes.c_void_p),
        ("stage_events", ctypes.c_void_p),
    ]

STAGE_EVENTS = 5   # [start, router done, linear state done, sparse done, end]


# The exported symbols and their C signatures (checked by the CPU tests).
SIGNATURES = {
    "sla2_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "sla2_topk_count": (ctypes.c_int, [ctypes.c_int, ctypes.c_float]),
    "sla2_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(Desc), ctypes.c_float]),
    "sla2_router": (ctypes.c_int, [ctypes.POINTER(Desc)] + [ctypes.c_void_p] * 4 + [ctypes.c_float]
                    + [ctypes.c_void_p] * 4),
    "sla2_router_soft": (ctypes.c_int, [ctypes.POINTER(Desc)] + [ctypes.c_void_p] * 4
                         + [ctypes.c_float, ctypes.c_float] + [ctypes.c_void_p] * 3),
    "sla2_linear_state": (ctypes.c_int, [ctypes.POINTER(Desc)] + [ctypes.c_void_p] * 8),
    "sla2_forward": (ctypes.c_int, [ctypes.POINTER(Desc)] + [ctypes.c_void_p] * 6 + [ctypes.c_float]
                     + [ctypes.c_void_p] * 2),
    "sla2_workspace_size_heads": (ctypes.c_size_t, [ctypes.POINTER(Desc), ctypes.c_int, ctypes.c_float]),
    "sla2_backward_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(Desc), ctypes.c_float]),
    "sla2_backward": (ctypes.c_int, [ctypes.POINTER(Desc)] + [ctypes.c_void_p] * 6 + [ctypes.c_float]
                      + [ctypes.c_void_p] * 6),
    "sla2_forward_heads": (ctypes.c_int, [ctypes.POINTER(Desc), ctypes.c_int, ctypes.c_int] + [ctypes.c_void_p] * 6
                           + [ctypes.c_float] + [ctypes.c_void_p] * 2),
    "sla2_forward_host_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(Desc), ctypes.c_int, ctypes.c_float]),
    "sla2_forward_host": (ctypes.c_int, [ctypes.POINTER(Desc), ctypes.c_int] + [ctypes.c_void_p] * 6
                          + [ctypes.c_float] + [ctypes.c_void_p] * 2),
}

_lib = None


def load_library(path: str = LIB_PATH):
    """Load libsla2.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libsla2.so not built ({path}); run python -m block_sparse_linear_router_b200.build")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    lib.sla2_set_wait_budget_ns.restype = None
    lib.sla2_set_wait_budget_ns.argtypes = [ctypes.c_ulonglong]
    _lib = lib
    return lib


def topk_count(nk: int, frac: float) -> int:
    return load_library().sla2_topk_count(nk, frac)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check_qkv(*ts):
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device (no CPU path)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def make_desc(B, H, N, d, quantize=1, out_dtype=0) -> Desc:
    return Desc(B=B, H=H, N=N, d=d, quantize=quantize, out_dtype=out_dtype)


def workspace_size(B, H, N, d, frac, quantize=1) -> int:
    desc = make_desc(B, H, N, d, quantize)
    return load_library().sla2_workspace_size(ctypes.byref(desc), frac)


def set_wait_budget_ns(ns: int) -> None:
    load_library().sla2_set_wait_budget_ns(int(ns))


@dataclass
class Workspace:
    buf: torch.Tensor

    @staticmethod
    def for_shape(B, H, N, d, frac, quantize=1, device="cuda") -> "Workspace":
        n = workspace_size(B, H, N, d, frac, quantize)
        if n == 0:
            raise Sla2Error(1, "sla2_workspace_size")
        return Workspace(torch.empty(n, dtype=torch.uint8, device=device))


def router(q, k, proj_q, proj_k, frac, workspace: Optional[Workspace] = None, scores=False, stream=None):
    """Mask M_c (uint8 [B,H,nq,nk]), idx (int32 [B,H,nq,k]), colmean (fp32 [B,H,d]) and optionally the fp32 logits."""
    lib = load_library()
    _check_qkv(q, k, proj_q, proj_k)
    B, H, N, d = q.shape
    nq, nk = N // 128, N // 64
    kk = lib.sla2_topk_count(nk, frac)
    ws = workspace or Workspace.for_shape(B, H, N, d, frac, 0, q.device)
    desc = make_desc(B, H, N, d, 0)
    desc.workspace, desc.workspace_bytes = ws.buf.data_ptr(), ws.buf.numel()
    mask = torch.empty(B, H, nq, nk, dtype=torch.uint8, device=q.device)
    idx = torch.empty(B, H, nq, max(kk, 1), dtype=torch.int32, device=q.device)
    cm = torch.empty(B, H, d, dtype=torch.float32, device=q.device)
    sc = torch.empty(B, H, nq, nk, dtype=torch.float32, device=q.device) if scores else None
    if sc is not None:
        desc.dbg_scores = sc.data_ptr()
    r = lib.sla2_router(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(proj_q), _ptr(proj_k), frac,
                        _ptr(mask), _ptr(idx), _ptr(cm), _stream(stream))
    if r != 0:
        raise Sla2Error(r, "sla2_router")
    out = {"mask": mask, "idx": idx, "colmean": cm}
    if sc is not None:
        out["scores"] = sc
    return out


def router_soft(q, k, proj_q, proj_k, frac, tau=0.1, workspace: Optional[Workspace] = None, scores=False,
                stream=None):
    """SoftTop-k mask sigmoid(P_c / tau + lambda) (fp32 [B,H,nq,nk], rows summing to k) and lambda
    (fp32 [B,H,nq]); optionally the fp32 logits."""
    lib = load_library()
    _check_qkv(q, k, proj_q, proj_k)
    B, H, N, d = q.shape
    nq, nk = N // 128, N // 64
    ws = workspace or Workspace.for_shape(B, H, N, d, frac, 0, q.device)
    desc = make_desc(B, H, N, d, 0)
    desc.workspace, desc.workspace_bytes = ws.buf.data_ptr(), ws.buf.numel()
    soft = torch.empty(B, H, nq, nk, dtype=torch.float32, device=q.device)
    lam = torch.empty(B, H, nq, dtype=torch.float32, device=q.device)
    sc = torch.empty(B, H, nq, nk, dtype=torch.float32, device=q.device) if scores else None
    if sc is not None:
        desc.dbg_scores = sc.data_ptr()
    r = lib.sla2_router_soft(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(proj_q), _ptr(proj_k), frac, tau,
                             _ptr(soft), _ptr(lam), _stream(stream))
    if r != 0:
        raise Sla2Error(r, "sla2_router_soft")
    out = {"soft": soft, "lambda": lam}
    if sc is not None:
        out["scores"] = sc
    return out


def linear_state(k, v, colmean, workspace: Optional[Workspace] = None, stream=None):
    """Per key block h_j^T (fp32 [B,H,nk,d(c),d(e)]), z_j, and their sums H_total^T, Z_total, for the
    smoothed keys K - colmean."""
    lib = load_library()
    _check_qkv(k, v, colmean)
    B, H, N, d = k.shape
    nk = N // 64
    ws = workspace or Workspace.for_shape(B, H, N, d, 1.0, 0, k.device)
    desc = make_desc(B, H, N, d, 0)
    desc.workspace, desc.workspace_bytes = ws.buf.data_ptr(), ws.buf.numel()
    dev = k.device
    h = torch.empty(B, H, nk, d, d, dtype=torch.float32, device=dev)
    z = torch.empty(B, H, nk, d, dtype=torch.float32, device=dev)
    Ht = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
    Zt = torch.empty(B, H, d, dtype=torch.float32, device=dev)
    r = lib.sla2_linear_state(ctypes.byref(desc), _ptr(k), _ptr(v), _ptr(colmean), _ptr(h), _ptr(z), _ptr(Ht),
                              _ptr(Zt), _stream(stream))
    if r != 0:
        raise Sla2Error(r, "sla2_linear_state")
    return {"h": h, "z": z, "Htot": Ht, "Ztot": Zt}


def forward(q, k, v, proj_q, proj_k, alpha, frac, quantize=1, out_dtype=torch.bfloat16,
            workspace: Optional[Workspace] = None, out: Optional[torch.Tensor] = None, debug=False,
            status: Optional[torch.Tensor] = None, stream=None, stage_events=None):
    """The SLA2 forward pass: returns out [B,H,N,d] (and a dict of debug exports when debug=True)."""
    lib = load_library()
    _check_qkv(q, k, v, proj_q, proj_k, alpha)
    B, H, N, d = q.shape
    nq, nk = N // 128, N // 64
    f32 = out_dtype == torch.float32
    ws = workspace or Workspace.for_shape(B, H, N, d, frac, quantize, q.device)
    desc = make_desc(B, H, N, d, quantize, 1 if f32 else 0)
    desc.workspace, desc.workspace_bytes = ws.buf.data_ptr(), ws.buf.numel()
    if out is None:
        out = torch.empty(B, H, N, d, dtype=torch.float32 if f32 else torch.bfloat16, device=q.device)
    if status is not None:
        desc.status = status.data_ptr()
    if stage_events is not None:
        # a ctypes array of STAGE_EVENTS raw cudaEvent_t handles (kept alive by the caller)
        desc.stage_events = ctypes.cast(stage_events, ctypes.c_void_p)
    dbg = {}
    if debug:
        dev = q.device
        kk = lib.sla2_topk_count(nk, frac)
        dbg = {
            "scores": torch.empty(B, H, nq, nk, dtype=torch.float32, device=dev),
            "O_s": torch.empty(B, H, N, d, dtype=torch.float32, device=dev),
            "O_l": torch.empty(B, H, N, d, dtype=torch.float32, device=dev),
            "mask": torch.empty(B, H, nq, nk, dtype=torch.uint8, device=dev),
            "idx": torch.empty(B, H, nq, kk, dtype=torch.int32, device=dev),
        }
        desc.dbg_scores, desc.dbg_os, desc.dbg_ol = (dbg[n].data_ptr() for n in ("scores", "O_s", "O_l"))
        desc.dbg_mask, desc.dbg_idx = dbg["mask"].data_ptr(), dbg["idx"].data_ptr()
        if quantize:
            dbg.update({
                "qhat": torch.empty(B, H, N, d, dtype=torch.int8, device=dev),
                "khat": torch.empty(B, H, N, d, dtype=torch.int8, device=dev),
                "vhatT": torch.empty(B, H, nk, d, 64, dtype=torch.uint8, device=dev),
                "sq": torch.empty(B, H, nq, dtype=torch.float32, device=dev),
                "sk": torch.empty(B, H, nk, dtype=torch.float32, device=dev),
                "sv": torch.empty(B, H, d, dtype=torch.float32, device=dev),
            })
            desc.dbg_qhat, desc.dbg_khat, desc.dbg_vhat = (dbg[n].data_ptr() for n in ("qhat", "khat", "vhatT"))
            desc.dbg_qscale, desc.dbg_kscale, desc.dbg_vscale = (dbg[n].data_ptr() for n in ("sq", "sk", "sv"))
    r = lib.sla2_forward(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(proj_q), _ptr(proj_k), _ptr(alpha),
                         frac, _ptr(out), _stream(stream))
    if r != 0:
        raise Sla2Error(r, "sla2_forward")
    return (out, dbg) if debug else out


def shard_heads(H: int, world_size: int, rank: int):
    """Contiguous head range (h_begin, h_count) of `rank` when H heads are split
    over `world_size` ranks as evenly as possible (the first H % world_size
    ranks take one head more). A rank may get h_count = 0 when world_size > H."""
    if world_size < 1 or not (0 <= rank < world_size) or H < 0:
        raise ValueError("bad head sharding arguments")
    base, extra = divmod(H, world_size)
    h_begin = rank * base + min(rank, extra)
    return h_begin, base + (1 if rank < extra else 0)


def workspace_size_heads(B, H, N, d, h_count, frac, quantize=1) -> int:
    desc = make_desc(B, H, N, d, quantize)
    return load_library().sla2_workspace_size_heads(ctypes.byref(desc), h_count, frac)


def forward_heads(q, k, v, proj_q, proj_k, alpha, frac, h_begin, h_count, out, quantize=1,
                  workspace: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None, stream=None):
    """Heads [h_begin, h_begin + h_count) of the forward pass, written into the full
    output tensor `out` [B,H,N,d] (bf16 or fp32); nothing else of `out` is touched.
    Bit-identical to those heads of forward() on the same full inputs."""
    lib = load_library()
    _check_qkv(q, k, v, proj_q, proj_k, alpha, out)
    B, H, N, d = q.shape
    if out.dtype not in (torch.bfloat16, torch.float32) or tuple(out.shape) != (B, H, N, d):
        raise ValueError("out must be a bf16 or fp32 [B,H,N,d] tensor")
    n = lib.sla2_workspace_size_heads(ctypes.byref(make_desc(B, H, N, d, quantize)), h_count, frac)
    if n == 0:
        raise Sla2Error(1, "sla2_workspace_size_heads")
    ws = workspace if workspace is not None else torch.empty(n, dtype=torch.uint8, device=q.device)
    desc = make_desc(B, H, N, d, quantize, 1 if out.dtype == torch.float32 else 0)
    desc.workspace, desc.workspace_bytes = ws.data_ptr(), ws.numel()
    if status is not None:
        desc.status = status.data_ptr()
    r = lib.sla2_forward_heads(ctypes.byref(desc), h_begin, h_count, _ptr(q), _ptr(k), _ptr(v), _ptr(proj_q),
                               _ptr(proj_k), _ptr(alpha), frac, _ptr(out), _stream(stream))
    if r != 0:
        raise Sla2Error(r, "sla2_forward_heads")
    return out


def forward_host_workspace_size(B, H, N, d, frac, heads_per_group, quantize=1, out_dtype=torch.bfloat16) -> int:
    desc = make_desc(B, H, N, d, quantize, 1 if out_dtype == torch.float32 else 0)
    return load_library().sla2_forward_host_workspace_size(ctypes.byref(desc), heads_per_group, frac)


def forward_host(q, k, v, proj_q, proj_k, alpha, frac, out, heads_per_group=2, quantize=1,
                 workspace: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None, stream=None):
    """The forward pass from HOST tensors to the HOST tensor `out` (bf16 or fp32 [B,H,N,d]),
    with the copies overlapped with the computation head group by head group; the
    workspace is device memory. Returns once enqueued: `out` is complete when `stream`
    (default: the current stream) is, and the host tensors must live until then
    (page-locked tensors let the copies run asynchronously)."""
    lib = load_library()
    for t in (q, k, v, proj_q, proj_k, alpha, out):
        if t.is_cuda:
            raise ValueError("forward_host takes host tensors")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    B, H, N, d = q.shape
    if out.dtype not in (torch.bfloat16, torch.float32) or tuple(out.shape) != (B, H, N, d):
        raise ValueError("out must be a bf16 or fp32 [B,H,N,d] tensor")
    f32 = 1 if out.dtype == torch.float32 else 0
    desc = make_desc(B, H, N, d, quantize, f32)
    n = lib.sla2_forward_host_workspace_size(ctypes.byref(desc), heads_per_group, frac)
    if n == 0:
        raise Sla2Error(1, "sla2_forward_host_workspace_size")
    ws = workspace if workspace is not None else torch.empty(n, dtype=torch.uint8, device="cuda")
    if not ws.is_cuda:
        raise ValueError("the workspace is device memory")
    desc.workspace, desc.workspace_bytes = ws.data_ptr(), ws.numel()
    if status is not None:
        desc.status = status.data_ptr()
    r = lib.sla2_forward_host(ctypes.byref(desc), heads_per_group, _ptr(q), _ptr(k), _ptr(v), _ptr(proj_q),
                              _ptr(proj_k), _ptr(alpha), frac, _ptr(out), _stream(stream))
    if r != 0:
        raise Sla2Error(r, "sla2_forward_host")
    return out


def backward(q, k, v, proj_q, proj_k, alpha, frac, dout, workspace: Optional[torch.Tensor] = None,
             status: Optional[torch.Tensor] = None, stream=None):
    """Gradients of the unquantised forward for the router's mask: (dq, dk, dv) fp32
    [B,H,N,d] and dalpha fp32 [H,nq] (summed over the batch), for dL/dO = dout (fp32)."""
    lib = load_library()
    _check_qkv(q, k, v, proj_q, proj_k, alpha, dout)
    if dout.dtype != torch.float32 or tuple(dout.shape) != tuple(q.shape):
        raise ValueError("dout must be fp32 with the shape of q")
    B, H, N, d = q.shape
    desc = make_desc(B, H, N, d, 0)
    n = lib.sla2_backward_workspace_size(ctypes.byref(desc), frac)
    if n == 0:
        raise Sla2Error(1, "sla2_backward_workspace_size")
    ws = workspace if workspace is not None else torch.empty(n, dtype=torch.uint8, device=q.device)
    desc.workspace, desc.workspace_bytes = ws.data_ptr(), ws.numel()
    if status is not None:
        desc.status = status.data_ptr()
    dq, dk, dv = (torch.empty(B, H, N, d, dtype=torch.float32, device=q.device) for _ in range(3))
    dalpha = torch.empty(H, N // 128, dtype=torch.float32, device=q.device)
    r = lib.sla2_backward(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(proj_q), _ptr(proj_k), _ptr(alpha),
                          frac, _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dalpha), _stream(stream))
    if r != 0:
        raise Sla2Error(r, "sla2_backward")
    return dq, dk, dv, dalpha
