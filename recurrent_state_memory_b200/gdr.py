"""Thin ctypes binding over libgdr.so (C ABI in include/gdr.h).

Argument marshalling only: every step of the recurrence runs in the library's
CUDA kernels.  torch is used for device memory and streams.  There is no CPU
fallback: if the library is missing or a call fails, an exception is raised.

Layouts follow include/gdr.h: q, k [B,T,H,dk]; v, o [B,T,H,dv]; g [B,T,H,dk]
([B,T,H,dk/2] with rotation); beta [B,T,H]; theta [B,T,H,dk/2]; S [B,H,dv,dk].
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdr.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "gdr.h")

(GDR_OK, GDR_ERR_INVALID_ARG, GDR_ERR_UNSUPPORTED, GDR_ERR_CUDA, GDR_ERR_TIMEOUT, GDR_ERR_WORKSPACE,
 GDR_ERR_RANGE, GDR_ERR_BOUNDS) = range(8)
GDR_F32, GDR_BF16 = 0, 1
GATE_LOGDECAY, GATE_NEG_SOFTPLUS = 0, 1
ALGOS = {"auto": 0, "simt": 1, "tcgen05": 2, "tcgen05_split": 3, "tcgen05_waves": 4, "tcgen05_segments": 5,
         "tcgen05_chains": 6}
ALGO_NAMES = {v: k for k, v in ALGOS.items()}


class FwdDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("chunk", ctypes.c_int),
                ("qkv_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
                ("gate_mode", ctypes.c_int), ("rotation", ctypes.c_int),
                ("scale", ctypes.c_float), ("algo", ctypes.c_int), ("qk_l2norm", ctypes.c_int),
                ("segments", ctypes.c_int)]


class DecDesc(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int), ("H", ctypes.c_int), ("dk", ctypes.c_int), ("dv", ctypes.c_int),
                ("qkv_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
                ("gate_mode", ctypes.c_int), ("rotation", ctypes.c_int), ("scale", ctypes.c_float),
                ("qk_l2norm", ctypes.c_int)]


class RavenDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int), ("d", ctypes.c_int),
                ("slots", ctypes.c_int), ("topk", ctypes.c_int), ("qkv_dtype", ctypes.c_int),
                ("out_dtype", ctypes.c_int), ("gate_mode", ctypes.c_int), ("scale", ctypes.c_float),
                ("segments", ctypes.c_int)]


class GdrError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: {status_string(status)} ({detail})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load libgdr.so; raise if it has not been built (no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m recurrent_state_memory_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, fp, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t
        L.gdr_abi_version.restype = ctypes.c_int
        L.gdr_status_string.restype = ctypes.c_char_p
        L.gdr_status_string.argtypes = [ctypes.c_int]
        L.gdr_last_error_detail.restype = ctypes.c_char_p
        L.gdr_chunk_fwd_workspace_bytes.restype = sz
        L.gdr_chunk_fwd_workspace_bytes.argtypes = [ctypes.POINTER(FwdDesc)]
        L.gdr_chunk_fwd.restype = ctypes.c_int
        L.gdr_chunk_fwd.argtypes = [ctypes.POINTER(FwdDesc), vp, vp, vp, fp, fp, fp, fp, vp, fp, vp, sz, vp]
        L.gdr_decode_step.restype = ctypes.c_int
        L.gdr_decode_step.argtypes = [ctypes.POINTER(DecDesc), vp, vp, vp, fp, fp, fp, fp, vp, vp]
        L.gdr_chunk_fwd_untied.restype = ctypes.c_int
        L.gdr_chunk_fwd_untied.argtypes = [ctypes.POINTER(FwdDesc), vp, vp, vp, fp, fp, fp, fp, fp, vp, fp, vp, sz, vp]
        L.gdr_chunk_fwd_ex.restype = ctypes.c_int
        L.gdr_chunk_fwd_ex.argtypes = [ctypes.POINTER(FwdDesc), vp, vp, vp, fp, fp, fp, fp, fp, vp, fp, fp, vp, sz, vp]
        L.gdr_chunk_fwd_host.restype = ctypes.c_int
        L.gdr_chunk_fwd_host.argtypes = [ctypes.POINTER(FwdDesc), vp, vp, vp, fp, fp, fp, fp, fp, vp, fp, fp, vp, sz, vp]
        L.gdr_chunk_fwd_host_workspace_bytes.restype = sz
        L.gdr_chunk_fwd_host_workspace_bytes.argtypes = [ctypes.POINTER(FwdDesc)] + [ctypes.c_int] * 4
        L.gdr_decode_step_untied.restype = ctypes.c_int
        L.gdr_decode_step_untied.argtypes = [ctypes.POINTER(DecDesc), vp, vp, vp, fp, fp, fp, fp, fp, vp, vp]
        L.gdr_query_device_status.restype = ctypes.c_int
        L.gdr_query_device_status.argtypes = [vp]
        L.gdr_chunk_fwd_algo.restype = ctypes.c_int
        L.gdr_chunk_fwd_algo.argtypes = [ctypes.POINTER(FwdDesc)]
        L.gdr_chunk_fwd_kernel_launches.restype = ctypes.c_int
        L.gdr_chunk_fwd_kernel_launches.argtypes = [ctypes.POINTER(FwdDesc)]
        L.gdr_debug_bounds_site.restype = ctypes.c_int
        L.gdr_debug_bounds_site.argtypes = []
        L.gdr_chunk_bwd_workspace_bytes.restype = ctypes.c_size_t
        L.gdr_chunk_bwd_workspace_bytes.argtypes = [ctypes.POINTER(FwdDesc)]
        L.gdr_chunk_bwd.restype = ctypes.c_int
        L.gdr_chunk_bwd.argtypes = [ctypes.POINTER(FwdDesc), vp, vp, vp, fp, fp, fp, fp, fp, vp, fp,
                                    fp, fp, fp, fp, fp, fp, fp, fp, vp, ctypes.c_size_t, vp]
        L.gdr_raven_fwd_segments.restype = ctypes.c_int
        L.gdr_raven_fwd_segments.argtypes = [ctypes.POINTER(RavenDesc)]
        L.gdr_raven_fwd_workspace_bytes.restype = ctypes.c_size_t
        L.gdr_raven_fwd_workspace_bytes.argtypes = [ctypes.POINTER(RavenDesc)]
        L.gdr_raven_fwd.restype = ctypes.c_int
        L.gdr_raven_fwd.argtypes = [ctypes.POINTER(RavenDesc), vp, vp, vp, fp, fp, fp, fp, vp, fp, fp, vp,
                                    ctypes.c_size_t, vp]
        L.gdr_chunk_fwd_noalloc.restype = ctypes.c_int
        L.gdr_chunk_fwd_noalloc.argtypes = [ctypes.POINTER(FwdDesc), vp, vp, vp, fp, fp, fp, fp, vp, fp, vp]
        L.gdr_debug_set_tc_fault.restype = None
        L.gdr_debug_set_tc_fault.argtypes = [ctypes.c_int, ctypes.c_ulonglong]
        if L.gdr_abi_version() != 5:
            raise RuntimeError("libgdr.so ABI version mismatch")
        _lib = L
    return _lib


def header_symbols() -> list:
    """Names of the entry points include/gdr.h declares."""
    text = open(HEADER_PATH).read()
    return re.findall(r"GDR_API\s+[\w\s\*]+?\b(gdr_\w+)\s*\(", text)


def status_string(s: int) -> str:
    return lib().gdr_status_string(int(s)).decode()


def _check(status: int, where: str):
    if status != GDR_OK:
        raise GdrError(status, where, lib().gdr_last_error_detail().decode())


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return GDR_BF16
    if t == torch.float32:
        return GDR_F32
    raise TypeError(f"unsupported dtype {t} (bf16 or fp32)")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream: Optional[torch.cuda.Stream], device) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype=None, device=None):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def fwd_desc(B, H, T, dk, dv, qkv_dtype, out_dtype, gate_mode=GATE_NEG_SOFTPLUS, rotation=False,
             scale=1.0, algo="auto", chunk=64, qk_l2norm=False, segments=0) -> FwdDesc:
    return FwdDesc(B, H, T, dk, dv, chunk, _dtype_code(qkv_dtype), _dtype_code(out_dtype),
                   int(gate_mode), int(bool(rotation)), float(scale), ALGOS[algo], int(bool(qk_l2norm)),
                   int(segments))


def resolved_algo(desc: FwdDesc) -> str:
    """Name of the kernel a descriptor runs with ("simt" or "tcgen05")."""
    a = int(lib().gdr_chunk_fwd_algo(ctypes.byref(desc)))
    if a < 0:
        raise ValueError("invalid descriptor")
    return ALGO_NAMES[a]


def kernel_launches(desc: FwdDesc) -> int:
    """How many kernels one forward call with this descriptor launches."""
    n = int(lib().gdr_chunk_fwd_kernel_launches(ctypes.byref(desc)))
    if n < 0:
        raise ValueError("invalid descriptor")
    return n


def use_library(path: str) -> None:
    """Load the library from `path` from now on (the debug build with index checks,
    libgdr_debug.so, for example); the next call loads it."""
    global LIB_PATH, _lib
    LIB_PATH = path
    _lib = None


def debug_bounds_site() -> int:
    """First failing index check of the debug build (0: none), cleared; -1 in the default build."""
    return int(lib().gdr_debug_bounds_site())


def debug_set_tc_fault(skip_first_commit: bool, wait_limit_ns: int = 0):
    """Test hook: make the tensor-core kernel's first MMA wait run out (see gdr.h)."""
    lib().gdr_debug_set_tc_fault(int(bool(skip_first_commit)), int(wait_limit_ns))


def workspace_bytes(desc: FwdDesc) -> int:
    return int(lib().gdr_chunk_fwd_workspace_bytes(ctypes.byref(desc)))


def host_workspace_bytes(desc: FwdDesc, w=False, S0=False, S_T=False, chunk_mean=False) -> int:
    """Device workspace of gdr_chunk_fwd_host for this descriptor and these optional arguments."""
    return int(lib().gdr_chunk_fwd_host_workspace_bytes(ctypes.byref(desc), int(bool(w)), int(bool(S0)),
                                                        int(bool(S_T)), int(bool(chunk_mean))))


def chunk_fwd(q, k, v, g, beta, theta=None, S0=None, *, gate_mode=GATE_NEG_SOFTPLUS, scale=1.0,
              algo="auto", out_dtype=None, want_state=True, o=None, S_T=None, workspace=None,
              stream=None, chunk=64, w=None, qk_l2norm=False, want_chunk_mean=False,
              chunk_mean=None, segments=0):
    """Chunk-parallel forward.  Returns (o, S_T), or (o, S_T, chunk_mean) when
    want_chunk_mean is set or a chunk_mean tensor is passed.

    algo "tcgen05_segments" cuts each sequence into `segments` pieces that run as separate
    chains and are combined exactly (0: the library chooses the number).

    beta is the erase strength; w [B,T,H] (fp32) a separate write strength, or None for
    the tied rule (w = beta).  chunk_mean [B, ceil(T/64), H, dv] (fp32) receives the mean
    of o over each chunk.  With CUDA tensors the call is asynchronous on `stream`
    (default: the current stream).  With host tensors it is one gdr_chunk_fwd_host call
    (copies and kernels pipelined over batch slices inside the library; asynchronous copies
    need page-locked tensors) on the current device, and it returns once the host outputs
    are written; outputs it allocates are page-locked when q (or, for T = 0, S0) is.
    """
    host = not q.is_cuda
    dev = q.device
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    rotation = theta is not None
    out_dtype = out_dtype or q.dtype
    _need(q, "q", device=dev)
    _need(k, "k", q.dtype, dev)
    _need(v, "v", q.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    if tuple(k.shape) != (B, T, H, dk) or tuple(v.shape) != (B, T, H, dv):
        raise ValueError("q, k, v shapes disagree")
    if tuple(g.shape) != (B, T, H, dk // 2 if rotation else dk) or tuple(beta.shape) != (B, T, H):
        raise ValueError("g or beta has the wrong shape")
    if w is not None:
        _need(w, "w", torch.float32, dev)
        if tuple(w.shape) != (B, T, H):
            raise ValueError("w has the wrong shape")
    if theta is not None:
        _need(theta, "theta", torch.float32, dev)
        if tuple(theta.shape) != (B, T, H, dk // 2):
            raise ValueError("theta has the wrong shape")
    if S0 is not None:
        _need(S0, "S0", torch.float32, dev)
        if tuple(S0.shape) != (B, H, dv, dk):
            raise ValueError("S0 has the wrong shape")
    # outputs it allocates are page-locked when the inputs are (asynchronous copies)
    pin = host and any(t.is_pinned() for t in (q, S0) if t is not None and t.numel() > 0)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=out_dtype, device=dev, pin_memory=pin)
    _need(o, "o", out_dtype, dev)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev, pin_memory=pin)
    if S_T is not None:
        _need(S_T, "S_T", torch.float32, dev)
    with_mean = want_chunk_mean or chunk_mean is not None
    if with_mean:
        nc = (T + chunk - 1) // chunk
        if chunk_mean is None:
            chunk_mean = torch.empty((B, nc, H, dv), dtype=torch.float32, device=dev, pin_memory=pin)
        _need(chunk_mean, "chunk_mean", torch.float32, dev)
        if tuple(chunk_mean.shape) != (B, nc, H, dv):
            raise ValueError("chunk_mean has the wrong shape")
    desc = fwd_desc(B, H, T, dk, dv, q.dtype, out_dtype, gate_mode, rotation, scale, algo, chunk, qk_l2norm,
                    segments)
    out = (o, S_T, chunk_mean) if with_mean else (o, S_T)
    if host:
        cdev = torch.device("cuda", torch.cuda.current_device())
        need = host_workspace_bytes(desc, w is not None, S0 is not None, S_T is not None, with_mean)
        if workspace is None and need:
            workspace = torch.empty(need, dtype=torch.uint8, device=cdev)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = lib().gdr_chunk_fwd_host(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                      _ptr(w), _ptr(theta), _ptr(S0), _ptr(o), _ptr(S_T), _ptr(chunk_mean),
                                      _ptr(workspace), ws_bytes, _stream_handle(stream, cdev))
        _check(st, "gdr_chunk_fwd_host")
        (stream if stream is not None else torch.cuda.current_stream(cdev)).synchronize()
        return out
    need = workspace_bytes(desc)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if with_mean:
        st = lib().gdr_chunk_fwd_ex(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                    _ptr(w), _ptr(theta), _ptr(S0), _ptr(o), _ptr(S_T), _ptr(chunk_mean),
                                    _ptr(workspace), ws_bytes, _stream_handle(stream, dev))
        _check(st, "gdr_chunk_fwd_ex")
    elif w is None:
        st = lib().gdr_chunk_fwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                 _ptr(theta), _ptr(S0), _ptr(o), _ptr(S_T), _ptr(workspace), ws_bytes,
                                 _stream_handle(stream, dev))
        _check(st, "gdr_chunk_fwd")
    else:
        st = lib().gdr_chunk_fwd_untied(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                        _ptr(w), _ptr(theta), _ptr(S0), _ptr(o), _ptr(S_T), _ptr(workspace),
                                        ws_bytes, _stream_handle(stream, dev))
        _check(st, "gdr_chunk_fwd_untied")
    return out


def bwd_workspace_bytes(desc: FwdDesc) -> int:
    return int(lib().gdr_chunk_bwd_workspace_bytes(ctypes.byref(desc)))


def chunk_bwd(q, k, v, g, beta, S0=None, dO=None, dS_T=None, *, gate_mode=GATE_NEG_SOFTPLUS, scale=1.0,
              w=None, theta=None, qk_l2norm=False, out_dtype=None, want_dS0=True, workspace=None, stream=None,
              chunk=64):
    """Backward of ``chunk_fwd`` (dk = dv): the gradients of every input given dO (like o, dtype
    out_dtype, default q's) and dS_T (fp32 like S_T); either may be None (zero).  theta (rotation)
    and qk_l2norm as in the forward.  Returns a dict of fp32 tensors "q", "k", "v", "g", "beta",
    "w" (None without w), "theta" (None without rotation) and "S0" (None unless want_dS0).
    Asynchronous on `stream` (default: the current stream)."""
    dev = q.device
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    rotation = theta is not None
    ng = dk // 2 if rotation else dk
    out_dtype = out_dtype or (dO.dtype if dO is not None else q.dtype)
    _need(q, "q", device=dev)
    _need(k, "k", q.dtype, dev)
    _need(v, "v", q.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    if tuple(k.shape) != (B, T, H, dk) or tuple(v.shape) != (B, T, H, dv) or tuple(g.shape) != (B, T, H, ng):
        raise ValueError("q, k, v, g shapes disagree")
    for t, n, shp in ((w, "w", (B, T, H)), (S0, "S0", (B, H, dv, dk)), (dS_T, "dS_T", (B, H, dv, dk)),
                      (theta, "theta", (B, T, H, dk // 2))):
        if t is not None:
            _need(t, n, torch.float32, dev)
            if tuple(t.shape) != shp:
                raise ValueError(f"{n} has the wrong shape")
    if dO is not None:
        _need(dO, "dO", out_dtype, dev)
        if tuple(dO.shape) != (B, T, H, dv):
            raise ValueError("dO has the wrong shape")
    f32 = dict(dtype=torch.float32, device=dev)
    grads = {"q": torch.empty((B, T, H, dk), **f32), "k": torch.empty((B, T, H, dk), **f32),
             "v": torch.empty((B, T, H, dv), **f32), "g": torch.empty((B, T, H, ng), **f32),
             "beta": torch.empty((B, T, H), **f32), "w": None if w is None else torch.empty((B, T, H), **f32),
             "theta": torch.empty((B, T, H, dk // 2), **f32) if rotation else None,
             "S0": torch.empty((B, H, dv, dk), **f32) if want_dS0 else None}
    desc = fwd_desc(B, H, T, dk, dv, q.dtype, out_dtype, gate_mode, rotation, scale, "auto", chunk,
                    qk_l2norm=qk_l2norm)
    need = bwd_workspace_bytes(desc)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().gdr_chunk_bwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(w),
                             _ptr(theta), _ptr(S0), _ptr(dO), _ptr(dS_T), _ptr(grads["q"]), _ptr(grads["k"]),
                             _ptr(grads["v"]), _ptr(grads["g"]), _ptr(grads["beta"]), _ptr(grads["w"]),
                             _ptr(grads["theta"]), _ptr(grads["S0"]), _ptr(workspace), ws_bytes,
                             _stream_handle(stream, dev))
    _check(st, "gdr_chunk_bwd")
    return grads


def raven_desc(B, H, T, d, topk, out_dtype=torch.bfloat16, gate_mode=GATE_NEG_SOFTPLUS, scale=1.0, segments=0,
               slots=64) -> RavenDesc:
    return RavenDesc(B, H, T, d, slots, topk, _dtype_code(torch.bfloat16), _dtype_code(out_dtype), int(gate_mode),
                     float(scale), int(segments))


def raven_segments(desc: RavenDesc) -> int:
    n = int(lib().gdr_raven_fwd_segments(ctypes.byref(desc)))
    if n < 0:
        raise ValueError("invalid Raven descriptor")
    return n


def raven_workspace_bytes(desc: RavenDesc) -> int:
    return int(lib().gdr_raven_fwd_workspace_bytes(ctypes.byref(desc)))


def raven_fwd(q, k, v, z, g, S0k=None, S0v=None, *, topk, gate_mode=GATE_NEG_SOFTPLUS, scale=1.0,
              out_dtype=None, segments=0, want_state=True, workspace=None, stream=None):
    """Raven's routed slot memory forward (``gdr_raven_fwd``): q, k, v [B,T,H,d] bf16, router
    logits z [B,T,H,64] fp32, decay gate g [B,T,H] fp32, optional start states S0k, S0v
    [B,H,64,d] fp32.  Returns (o [B,T,H,d], Sk_T, Sv_T) (the states None unless want_state)."""
    dev = q.device
    B, T, H, d = q.shape
    out_dtype = out_dtype or q.dtype
    _need(q, "q", torch.bfloat16, dev)
    _need(k, "k", torch.bfloat16, dev)
    _need(v, "v", torch.bfloat16, dev)
    _need(z, "z", torch.float32, dev)
    _need(g, "g", torch.float32, dev)
    if tuple(k.shape) != (B, T, H, d) or tuple(v.shape) != (B, T, H, d) or tuple(z.shape) != (B, T, H, 64) \
            or tuple(g.shape) != (B, T, H):
        raise ValueError("q, k, v, z, g shapes disagree")
    for t, n in ((S0k, "S0k"), (S0v, "S0v")):
        if t is not None:
            _need(t, n, torch.float32, dev)
            if tuple(t.shape) != (B, H, 64, d):
                raise ValueError(f"{n} has the wrong shape")
    o = torch.empty((B, T, H, d), dtype=out_dtype, device=dev)
    SkT = torch.empty((B, H, 64, d), dtype=torch.float32, device=dev) if want_state else None
    SvT = torch.empty((B, H, 64, d), dtype=torch.float32, device=dev) if want_state else None
    desc = raven_desc(B, H, T, d, topk, out_dtype, gate_mode, scale, segments)
    need = raven_workspace_bytes(desc)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().gdr_raven_fwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(g), _ptr(S0k), _ptr(S0v),
                             _ptr(o), _ptr(SkT), _ptr(SvT), _ptr(workspace), ws_bytes, _stream_handle(stream, dev))
    _check(st, "gdr_raven_fwd")
    return o, SkT, SvT


def decode_step(q, k, v, g, beta, S, theta=None, *, gate_mode=GATE_NEG_SOFTPLUS, scale=1.0,
                out_dtype=None, o=None, stream=None, w=None, qk_l2norm=False) -> torch.Tensor:
    """One decode step; S [N,H,dv,dk] (fp32) is updated in place.  Returns o [N,H,dv].
    beta erases; w [N,H] (fp32) is a separate write strength, or None for w = beta."""
    dev = S.device
    N, H, dk = q.shape
    dv = v.shape[-1]
    rotation = theta is not None
    out_dtype = out_dtype or q.dtype
    _need(q, "q", device=dev)
    _need(k, "k", q.dtype, dev)
    _need(v, "v", q.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(S, "S", torch.float32, dev)
    if tuple(S.shape) != (N, H, dv, dk) or tuple(g.shape) != (N, H, dk // 2 if rotation else dk):
        raise ValueError("S or g has the wrong shape")
    if theta is not None:
        _need(theta, "theta", torch.float32, dev)
    if o is None:
        o = torch.empty((N, H, dv), dtype=out_dtype, device=dev)
    desc = DecDesc(N, H, dk, dv, _dtype_code(q.dtype), _dtype_code(out_dtype), int(gate_mode),
                   int(rotation), float(scale), int(bool(qk_l2norm)))
    if w is not None:
        _need(w, "w", torch.float32, dev)
        if tuple(w.shape) != (N, H):
            raise ValueError("w has the wrong shape")
    st = lib().gdr_decode_step_untied(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                      _ptr(w), _ptr(theta), _ptr(S), _ptr(o), _stream_handle(stream, dev))
    _check(st, "gdr_decode_step")
    return o


def query_device_status(stream=None) -> int:
    """Synchronise and read/clear the device status word (GDR_OK or GDR_ERR_TIMEOUT)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    return int(lib().gdr_query_device_status(_stream_handle(stream, dev)))
