"""Python binding of the C ABI in ``include/attn_jvp.h``.

Argument marshalling only: torch supplies device memory and the stream, the
library does all of the work.  There is no CPU or library fallback; if the
CUDA library is missing the call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

from .build import LIB_PATH

ATTN_JVP_OK = 0
ATTN_JVP_ERR_NULL = -1
ATTN_JVP_ERR_SHAPE = -2
ATTN_JVP_ERR_HEADDIM = -3
ATTN_JVP_ERR_ALIGN = -4
ATTN_JVP_ERR_LAUNCH = -5
ATTN_JVP_ERR_TIMEOUT = -6
ATTN_JVP_ERR_VALUE = -7
ATTN_JVP_ERR_SCRATCH = -8
ATTN_JVP_DEBUG_STARVE_Q = 1

EXPORTED = ("attn_jvp_fwd", "attn_jvp_fwd_ex", "attn_jvp_fwd_ws", "attn_jvp_workspace_bytes",
            "attn_jvp_fwd_noalloc",
            "attn_jvp_fwd_debug", "attn_jvp_fwd_trace", "attn_jvp_check", "attn_jvp_status_string", "attn_jvp_version", "scm_tangent_loss",
            "qkv_rmsnorm_jvp", "qkv_prologue_check")
TRACE_EVENTS = 11  # stamps per key tile of attn_jvp_fwd_trace

_lock = threading.Lock()
_lib = None


class AttnJvpError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = attn_jvp_status_string(status)
        super().__init__(f"{what}: {msg} (status {status})" if what else f"{msg} (status {status})")


def library_path() -> str:
    return LIB_PATH


def load_library():
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"CUDA library {LIB_PATH} is not built; run "
                    "`python -m attention_jvp_fwd_b200.build` (nvcc, sm_100a)")
            lib = ctypes.CDLL(LIB_PATH)
            vp, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
            lib.attn_jvp_fwd.restype = i32
            lib.attn_jvp_fwd.argtypes = [vp] * 9 + [i32] * 5 + [f32, vp, vp]
            lib.qkv_rmsnorm_jvp.restype = i32
            lib.qkv_rmsnorm_jvp.argtypes = [vp] * 11 + [i32] * 5 + [f32, vp]
            lib.qkv_prologue_check.restype = i32
            lib.qkv_prologue_check.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
            lib.scm_tangent_loss.restype = i32
            lib.scm_tangent_loss.argtypes = [vp] * 5 + [i32, ctypes.c_longlong, f32, vp]
            lib.attn_jvp_fwd_ex.restype = i32
            lib.attn_jvp_fwd_ex.argtypes = [vp] * 10 + [i32] * 5 + [f32, vp, vp]
            lib.attn_jvp_fwd_ws.restype = i32
            lib.attn_jvp_fwd_ws.argtypes = [vp] * 10 + [i32] * 5 + [f32, vp, vp, ctypes.c_size_t, vp]
            lib.attn_jvp_fwd_noalloc.restype = i32
            lib.attn_jvp_fwd_noalloc.argtypes = [vp] * 10 + [i32] * 5 + [f32, vp, vp]
            lib.attn_jvp_workspace_bytes.restype = ctypes.c_size_t
            lib.attn_jvp_workspace_bytes.argtypes = [i32] * 5
            lib.attn_jvp_fwd_debug.restype = i32
            lib.attn_jvp_fwd_debug.argtypes = [vp] * 9 + [i32] * 5 + [f32, vp, vp,
                                                                     ctypes.c_uint64, i32]
            lib.attn_jvp_fwd_trace.restype = i32
            lib.attn_jvp_fwd_trace.argtypes = [vp] * 9 + [i32] * 5 + [f32, vp, vp, vp, i32, i32]
            lib.attn_jvp_check.restype = i32
            lib.attn_jvp_check.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
            lib.attn_jvp_status_string.restype = ctypes.c_char_p
            lib.attn_jvp_status_string.argtypes = [i32]
            lib.attn_jvp_version.restype = i32
            lib.attn_jvp_version.argtypes = []
            _lib = lib
    return _lib


def attn_jvp_status_string(status: int) -> str:
    return load_library().attn_jvp_status_string(int(status)).decode()


def _check_inputs(q, k, v, q_dot, k_dot, v_dot):
    if (k_dot is None) != (v_dot is None):
        raise ValueError("k_dot and v_dot must both be tensors or both be None (K' = V' = 0)")
    for name, t in (("q", q), ("k", k), ("v", v), ("q_dot", q_dot), ("k_dot", k_dot),
                    ("v_dot", v_dot)):
        if t is None and name in ("k_dot", "v_dot"):
            continue
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous [B, H, L, d]")
        if t.dim() != 4:
            raise ValueError(f"{name} must be 4-D [B, H, L, d]")
        if t.device != q.device:
            raise ValueError("all tensors must be on one device")
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    for name, t, L in (("k", k, Lk), ("v", v, Lk), ("q_dot", q_dot, Lq), ("k_dot", k_dot, Lk),
                       ("v_dot", v_dot, Lk)):
        if t is not None and tuple(t.shape) != (B, H, L, d):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {(B, H, L, d)}")
    return B, H, Lq, Lk, d


def _stream_handle(device, stream):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(int(stream.cuda_stream))


def attn_jvp_workspace_bytes(B: int, H: int, Lq: int, Lk: int, d: int, device=None) -> int:
    """Workspace bytes the split call needs for this shape on `device` (0: no
    split for this shape)."""
    device = device if device is not None else torch.cuda.current_device()
    with torch.cuda.device(device):
        return int(load_library().attn_jvp_workspace_bytes(int(B), int(H), int(Lq), int(Lk), int(d)))


def attn_jvp_fwd(q, k, v, q_dot, k_dot, v_dot, scale: float | None = None, kv_len=None,
                 out=None, stream=None, *, lse_dot: bool = False, split: bool = True,
                 workspace: torch.Tensor | None = None,
                 _debug_timeout_ns: int | None = None, _debug_flags: int = 0):
    """O = softmax(scale Q K^T) V, its tangent O' along (Q', K', V'), and lse.

    q, q_dot: bf16 [B, H, Lq, d]; k, v, k_dot, v_dot: bf16 [B, H, Lk, d];
    d in {64, 128}; kv_len: optional int32 [B] on the same device (keys
    j >= kv_len[b] are masked).  scale defaults to 1/sqrt(d).  ``k_dot`` and
    ``v_dot`` may both be None, meaning K' = V' = 0 (a cheaper kernel).  With
    ``lse_dot=True`` the tangent of lse (sum_j P S') is returned as well.
    ``out`` may supply (o, o_dot, lse[, lse_dot]) buffers.  Queued on
    ``stream`` (default: the current stream).  Returns (o, o_dot, lse) or
    (o, o_dot, lse, lse_dot), lse and lse_dot fp32 [B, H, Lq].

    ``split`` (default) cuts the last wave of query tiles into key ranges
    (attn_jvp_fwd_ws); its workspace is ``workspace`` (a uint8 CUDA tensor of
    at least attn_jvp_workspace_bytes bytes) or, if None, allocated here.
    ``split=False`` walks every query tile whole and needs no workspace.
    """
    B, H, Lq, Lk, d = _check_inputs(q, k, v, q_dot, k_dot, v_dot)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    kv_ptr = None
    if kv_len is not None:
        if (not isinstance(kv_len, torch.Tensor) or kv_len.dtype != torch.int32
                or kv_len.device != q.device or tuple(kv_len.shape) != (B,)
                or not kv_len.is_contiguous()):
            raise ValueError("kv_len must be a contiguous int32 [B] tensor on q's device")
        kv_ptr = kv_len.data_ptr()
    ld = None
    if out is None:
        o = torch.empty_like(q)
        od = torch.empty_like(q)
        lse = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
        if lse_dot:
            ld = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
    else:
        if len(out) != (4 if lse_dot else 3):
            raise ValueError("out must hold (o, o_dot, lse) or, with lse_dot, four buffers")
        o, od, lse = out[:3]
        if lse_dot:
            ld = out[3]
    for name, t in (("o", o), ("o_dot", od)):
        if (t.dtype != torch.bfloat16 or t.device != q.device or not t.is_contiguous()
                or tuple(t.shape) != (B, H, Lq, d)):
            raise ValueError(f"{name} must be a contiguous bf16 [B, H, Lq, d] tensor on q's device")
    for name, t in (("lse", lse), ("lse_dot", ld)):
        if t is not None and (t.dtype != torch.float32 or t.device != q.device
                              or not t.is_contiguous() or tuple(t.shape) != (B, H, Lq)):
            raise ValueError(f"{name} must be a contiguous fp32 [B, H, Lq] tensor on q's device")
    lib = load_library()
    ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    ptrs = [ptr(t) for t in (q, k, v, q_dot, k_dot, v_dot, o, od, lse)]
    sh = _stream_handle(q.device, stream)
    with torch.cuda.device(q.device):
        if _debug_timeout_ns is not None or _debug_flags:
            if k_dot is None or lse_dot:
                raise ValueError("the debug entry point takes all six inputs and no lse_dot")
            rc = lib.attn_jvp_fwd_debug(*ptrs, B, H, Lq, Lk, d, float(scale), kv_ptr, sh,
                                        int(_debug_timeout_ns or 0), int(_debug_flags))
        elif split:
            need = int(lib.attn_jvp_workspace_bytes(B, H, Lq, Lk, d))
            ws = workspace
            if need and ws is None:
                ws = torch.empty(need, dtype=torch.uint8, device=q.device)
                if stream is not None:
                    ws.record_stream(stream)  # alive until the kernel on `stream` is done
            if ws is not None and (ws.dtype != torch.uint8 or ws.device != q.device
                                   or not ws.is_contiguous()):
                raise ValueError("workspace must be a contiguous uint8 tensor on q's device")
            rc = lib.attn_jvp_fwd_ws(*ptrs, ptr(ld), B, H, Lq, Lk, d, float(scale), kv_ptr,
                                     ptr(ws), 0 if ws is None else ws.numel(), sh)
        elif k_dot is None or lse_dot:
            rc = lib.attn_jvp_fwd_ex(*ptrs, ptr(ld), B, H, Lq, Lk, d, float(scale), kv_ptr, sh)
        else:
            rc = lib.attn_jvp_fwd(*ptrs, B, H, Lq, Lk, d, float(scale), kv_ptr, sh)
    if rc != ATTN_JVP_OK:
        raise AttnJvpError(rc, "attn_jvp_fwd")
    return (o, od, lse, ld) if lse_dot else (o, od, lse)


def attn_jvp_fwd_trace(q, k, v, q_dot, k_dot, v_dot, scale: float | None = None, kv_len=None,
                       tiles: int = 64, ctas: int | None = None, stream=None):
    """attn_jvp_fwd in the trace build: returns (o, o_dot, lse, trace), where
    trace is int64 [ctas, tiles, TRACE_EVENTS] of SM clock stamps of each
    CTA's first ``tiles`` key tiles (0 where no stamp was taken); ``ctas``
    defaults to the SM count.  The outputs equal attn_jvp_fwd's bit for bit.
    See attention_jvp_fwd_b200.trace for the event list and a summary."""
    B, H, Lq, Lk, d = _check_inputs(q, k, v, q_dot, k_dot, v_dot)
    if k_dot is None:
        raise ValueError("the trace build takes all six inputs")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    kv_ptr = None
    if kv_len is not None:
        if (not isinstance(kv_len, torch.Tensor) or kv_len.dtype != torch.int32
                or kv_len.device != q.device or tuple(kv_len.shape) != (B,)
                or not kv_len.is_contiguous()):
            raise ValueError("kv_len must be a contiguous int32 [B] tensor on q's device")
        kv_ptr = kv_len.data_ptr()
    if ctas is None:
        ctas = torch.cuda.get_device_properties(q.device).multi_processor_count
    o = torch.empty_like(q)
    od = torch.empty_like(q)
    lse = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
    trace = torch.zeros((ctas, tiles, TRACE_EVENTS), dtype=torch.int64, device=q.device)
    lib = load_library()
    ptrs = [t.data_ptr() for t in (q, k, v, q_dot, k_dot, v_dot, o, od, lse)]
    with torch.cuda.device(q.device):
        rc = lib.attn_jvp_fwd_trace(*ptrs, B, H, Lq, Lk, d, float(scale), kv_ptr,
                                    _stream_handle(q.device, stream), trace.data_ptr(), int(tiles),
                                    int(ctas))
    if rc != ATTN_JVP_OK:
        raise AttnJvpError(rc, "attn_jvp_fwd_trace")
    return o, od, lse, trace


def attn_jvp_check(stream=None, device=None) -> tuple[int, int]:
    """Synchronise the stream and read/clear the device status word.
    Returns (status, site)."""
    lib = load_library()
    device = device if device is not None else torch.cuda.current_device()
    site = ctypes.c_int(0)
    with torch.cuda.device(device):
        rc = lib.attn_jvp_check(_stream_handle(device, stream), ctypes.byref(site))
    return rc, site.value


def scm_tangent_loss(f, f_ema, g, c: float = 0.1, grad: bool = True, out=None, stream=None):
    """Tangent-normalised sCM loss per sample: r = F - F_ema - g / (|g|^2 + c),
    loss = |r|^2 and (if ``grad``) d loss / dF = 2 r.

    f, f_ema, g: contiguous bf16 CUDA tensors of one shape [B, ...] (each
    sample flattened to N elements).  Returns ``(loss, grad)``: fp32 [B] and
    bf16 of f's shape (None when ``grad`` is False).  ``out`` may supply
    ``(loss, grad)`` buffers.
    """
    for name, t in (("f", f), ("f_ema", f_ema), ("g", g)):
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
        if t.shape != f.shape or t.device != f.device:
            raise ValueError("f, f_ema and g must share one shape and device")
    if f.dim() < 1 or f.numel() == 0:
        raise ValueError("f must be [B, ...] with B >= 1 and at least one element per sample")
    B = f.shape[0]
    N = f.numel() // B
    if out is None:
        loss = torch.empty(B, dtype=torch.float32, device=f.device)
        gr = torch.empty_like(f) if grad else None
    else:
        loss, gr = out
    if loss.dtype != torch.float32 or tuple(loss.shape) != (B,) or loss.device != f.device:
        raise ValueError("loss must be fp32 [B] on f's device")
    if gr is not None and (gr.dtype != torch.bfloat16 or gr.shape != f.shape
                           or not gr.is_contiguous() or gr.device != f.device):
        raise ValueError("grad must be a contiguous bf16 tensor of f's shape")
    lib = load_library()
    with torch.cuda.device(f.device):
        rc = lib.scm_tangent_loss(f.data_ptr(), f_ema.data_ptr(), g.data_ptr(), loss.data_ptr(),
                                  None if gr is None else gr.data_ptr(), B, N, float(c),
                                  _stream_handle(f.device, stream))
    if rc != ATTN_JVP_OK:
        raise AttnJvpError(rc, "scm_tangent_loss")
    return loss, gr


def qkv_rmsnorm_jvp(x, x_dot, w_qkv, gamma_q, gamma_k, B: int, L: int, H: int, eps: float = 1e-6,
                    out=None, stream=None):
    """QKV projection + per-head RMSNorm of tokens x and its tangent along x'.

    x, x_dot: bf16 [B*L, D]; w_qkv: bf16 [3*H*d, D] (q, k, v heads stacked, as
    a linear layer stores its weight); gamma_q, gamma_k: fp32 [d].  Returns
    (q, k, v, q_dot, k_dot, v_dot), bf16 [B, H, L, d] each: the inputs of
    attn_jvp_fwd.  ``out`` may supply the six buffers.
    """
    for name, t in (("x", x), ("x_dot", x_dot), ("w_qkv", w_qkv)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be a bfloat16 torch.Tensor")
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 2:
            raise ValueError(f"{name} must be a contiguous 2-D CUDA tensor")
    for name, t in (("gamma_q", gamma_q), ("gamma_k", gamma_k)):
        if (not isinstance(t, torch.Tensor) or t.dtype != torch.float32 or not t.is_cuda
                or not t.is_contiguous() or t.dim() != 1):
            raise ValueError(f"{name} must be a contiguous fp32 1-D CUDA tensor")
    T, D = x.shape
    d = gamma_q.shape[0]
    if T != B * L or x_dot.shape != x.shape or tuple(w_qkv.shape) != (3 * H * d, D) \
            or gamma_k.shape != gamma_q.shape:
        raise ValueError("shapes: x, x_dot [B*L, D], w_qkv [3*H*d, D], gamma_q, gamma_k [d]")
    if out is None:
        out = tuple(torch.empty((B, H, L, d), dtype=torch.bfloat16, device=x.device) for _ in range(6))
    if len(out) != 6 or any(o.dtype != torch.bfloat16 or tuple(o.shape) != (B, H, L, d)
                            or not o.is_contiguous() or o.device != x.device for o in out):
        raise ValueError("out must be six contiguous bf16 [B, H, L, d] tensors on x's device")
    lib = load_library()
    with torch.cuda.device(x.device):
        rc = lib.qkv_rmsnorm_jvp(x.data_ptr(), x_dot.data_ptr(), w_qkv.data_ptr(), gamma_q.data_ptr(),
                                 gamma_k.data_ptr(), *[o.data_ptr() for o in out], B, L, H, D, d,
                                 float(eps), _stream_handle(x.device, stream))
    if rc != ATTN_JVP_OK:
        raise AttnJvpError(rc, "qkv_rmsnorm_jvp")
    return tuple(out)


def qkv_prologue_check(stream=None, device=None) -> tuple[int, int]:
    """Synchronise and read/clear the prologue kernel's status word: (status, site)."""
    lib = load_library()
    device = device if device is not None else torch.cuda.current_device()
    site = ctypes.c_int(0)
    with torch.cuda.device(device):
        rc = lib.qkv_prologue_check(_stream_handle(device, stream), ctypes.byref(site))
    return rc, site.value
