"""ctypes binding of libgdn.so (include/gdn.h).

Argument marshalling only: every step of the operator runs in the library's
CUDA kernels.  The functions named like the C entry points take torch tensors
(device memory allocated by the caller), pass their data pointers and the
current CUDA stream through the C ABI and turn a non-OK status into
:class:`GdnError`.  If libgdn.so has not been built, every call raises --
there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_WORKSPACE, GDN_ERR_CUDA, \
    GDN_ERR_TIMEOUT = range(6)
GDN_BF16, GDN_F32 = 0, 1
GDN_GATE_NONE, GDN_GATE_SCALAR, GDN_GATE_PER_DIM = 0, 1, 2

EXPORTED = ("gdn_chunk_fwd", "gdn_chunk_fwd_workspace_bytes", "gdn_chunk_fwd_workspace_min_bytes",
            "gdn_decode_step",
            "gdn_read_device_status", "gdn_status_string", "gdn_abi_version",
            "gdn_kernel_launch_count", "gdn_chunk_fwd_kernel_name", "gdn_chunk_fwd_noalloc",
            "gdn_chunk_fwd_noalloc_scratch_bytes", "gdn_osdn_precondition", "gdn_chunk_fwd_wk",
            "gdn_chunk_fwd_plan", "gdn_chunk_bwd", "gdn_chunk_bwd_workspace_bytes",
            "gdn_osdn_precondition_workspace_bytes")

_lib = None


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def load() -> ctypes.CDLL:
    """Load libgdn.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libgdn.so is not built ({LIB_PATH}); run "
                           "`python -m gated_delta_rule_94_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.gdn_chunk_fwd.argtypes = [vp, vp, vp, vp, vp, i, vp, vp, vp, i, i, i, i, i, i, i, vp, sz, vp]
    lib.gdn_chunk_fwd.restype = i
    lib.gdn_chunk_fwd_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i]
    lib.gdn_chunk_fwd_workspace_bytes.restype = sz
    lib.gdn_chunk_fwd_workspace_min_bytes.argtypes = [i, i, i, i, i, i, i, i]
    lib.gdn_chunk_fwd_workspace_min_bytes.restype = sz
    lib.gdn_decode_step.argtypes = [vp, vp, vp, vp, vp, i, vp, vp, i, i, i, i, i, vp]
    lib.gdn_decode_step.restype = i
    lib.gdn_read_device_status.argtypes = [vp]
    lib.gdn_read_device_status.restype = i
    lib.gdn_status_string.argtypes = [i]
    lib.gdn_status_string.restype = ctypes.c_char_p
    lib.gdn_abi_version.argtypes = []
    lib.gdn_abi_version.restype = i
    lib.gdn_kernel_launch_count.argtypes = []
    lib.gdn_kernel_launch_count.restype = ctypes.c_ulonglong
    lib.gdn_chunk_fwd_kernel_name.argtypes = [i, i, i, i]
    lib.gdn_chunk_fwd_kernel_name.restype = ctypes.c_char_p
    lib.gdn_chunk_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, i, vp, vp, vp, i, i, i, i, i, i, i, vp]
    lib.gdn_chunk_fwd_noalloc.restype = i
    lib.gdn_chunk_fwd_noalloc_scratch_bytes.argtypes = []
    lib.gdn_chunk_fwd_noalloc_scratch_bytes.restype = sz
    lib.gdn_osdn_precondition.argtypes = [vp, vp, vp, ctypes.c_float, vp, vp, vp, i, i, i, i, i,
                                          vp, sz, vp]
    lib.gdn_osdn_precondition.restype = i
    lib.gdn_osdn_precondition_workspace_bytes.argtypes = [i, i, i, i]
    lib.gdn_osdn_precondition_workspace_bytes.restype = sz
    lib.gdn_chunk_fwd_wk.argtypes = [vp, vp, vp, vp, vp, vp, i, vp, vp, vp, i, i, i, i, i, i, i, vp,
                                     sz, vp]
    lib.gdn_chunk_fwd_wk.restype = i
    ip = ctypes.POINTER(ctypes.c_int)
    lib.gdn_chunk_fwd_plan.argtypes = [i, i, i, i, i, i, i, i, sz, ip, ip, ip]
    lib.gdn_chunk_fwd_plan.restype = i
    lib.gdn_chunk_bwd.argtypes = [vp, vp, vp, vp, vp, i, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i,
                                  i, i, i, i, i, vp, sz, vp]
    lib.gdn_chunk_bwd.restype = i
    lib.gdn_chunk_bwd_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i]
    lib.gdn_chunk_bwd_workspace_bytes.restype = sz
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().gdn_status_string(int(status)).decode()


def gdn_status_string(status: int) -> str:
    return status_string(status)


def gdn_abi_version() -> int:
    return load().gdn_abi_version()


def gdn_kernel_launch_count() -> int:
    return int(load().gdn_kernel_launch_count())


def gdn_chunk_fwd_kernel_name(Dk, Dv, gate_kind, dtype=torch.bfloat16):
    name = load().gdn_chunk_fwd_kernel_name(Dk, Dv, int(gate_kind), _dtype_code(dtype))
    return None if name is None else name.decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return GDN_BF16
    if dt == torch.float32:
        return GDN_F32
    raise TypeError(f"unsupported dtype {dt}; use bfloat16 or float32")


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check_contig(**tensors):
    for name, t in tensors.items():
        if t is not None and not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")


def gdn_chunk_fwd_workspace_bytes(B, T, H, Dk, Dv, chunk=64, dtype=torch.bfloat16,
                                  gate_kind=GDN_GATE_SCALAR) -> int:
    n = load().gdn_chunk_fwd_workspace_bytes(B, T, H, Dk, Dv, chunk, _dtype_code(dtype),
                                             int(gate_kind))
    if n == ctypes.c_size_t(-1).value:
        raise GdnError(GDN_ERR_UNSUPPORTED, "gdn_chunk_fwd_workspace_bytes")
    return n


def gdn_chunk_fwd_workspace_min_bytes(B, T, H, Dk, Dv, chunk=64, dtype=torch.bfloat16,
                                      gate_kind=GDN_GATE_SCALAR) -> int:
    n = load().gdn_chunk_fwd_workspace_min_bytes(B, T, H, Dk, Dv, chunk, _dtype_code(dtype),
                                                 int(gate_kind))
    if n == ctypes.c_size_t(-1).value:
        raise GdnError(GDN_ERR_UNSUPPORTED, "gdn_chunk_fwd_workspace_min_bytes")
    return n


def gdn_chunk_fwd_plan(B, T, H, Dk, Dv, chunk=64, dtype=torch.bfloat16, gate_kind=GDN_GATE_SCALAR,
                       workspace_bytes=None) -> dict:
    """Waves, chunks per wave and segments per wave the forward uses with
    `workspace_bytes` (default: the full-speed size)."""
    if workspace_bytes is None:
        workspace_bytes = gdn_chunk_fwd_workspace_bytes(B, T, H, Dk, Dv, chunk, dtype, gate_kind)
    w, c, s = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    st = load().gdn_chunk_fwd_plan(B, T, H, Dk, Dv, chunk, _dtype_code(dtype), int(gate_kind),
                                   workspace_bytes, ctypes.byref(w), ctypes.byref(c),
                                   ctypes.byref(s))
    if st != GDN_OK:
        raise GdnError(st, "gdn_chunk_fwd_plan")
    return {"waves": w.value, "chunks_per_wave": c.value, "segments": s.value}


def gdn_chunk_fwd(q, k, v, beta, g, gate_kind, initial_state, o, final_state, *, chunk=64,
                  workspace=None, stream=None) -> None:
    """Enqueue the chunk forward on `stream` (default: torch's current stream).
    Shapes: q, k [B,T,H,Dk]; v, o [B,T,H,Dv]; beta [B,T,H]; g [B,T,H] or
    [B,T,H,Dk] or None; states [B,H,Dk,Dv] fp32 or None."""
    _check_contig(q=q, k=k, v=v, beta=beta, g=g, initial_state=initial_state, o=o,
                  final_state=final_state)
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dtype_code(q.dtype)
    for name, t in (("k", k), ("v", v), ("beta", beta), ("g", g), ("o", o)):
        if t is not None and t.dtype != q.dtype:
            raise TypeError(f"{name} must have dtype {q.dtype}")
    for name, t in (("initial_state", initial_state), ("final_state", final_state)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"{name} must be float32")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load().gdn_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), int(gate_kind),
                              _ptr(initial_state), _ptr(o), _ptr(final_state), B, T, H, Dk, Dv,
                              chunk, dt, _ptr(workspace), ws_bytes, _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_chunk_fwd")


def gdn_chunk_fwd_wk(q, k, k_write, v, beta, g, gate_kind, initial_state, o, final_state, *,
                     chunk=64, workspace=None, stream=None) -> None:
    """gdn_chunk_fwd with a separate write key k_write [B,T,H,Dk] (or None)."""
    _check_contig(q=q, k=k, k_write=k_write, v=v, beta=beta, g=g, initial_state=initial_state,
                  o=o, final_state=final_state)
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dtype_code(q.dtype)
    for name, t in (("k", k), ("k_write", k_write), ("v", v), ("beta", beta), ("g", g), ("o", o)):
        if t is not None and t.dtype != q.dtype:
            raise TypeError(f"{name} must have dtype {q.dtype}")
    for name, t in (("initial_state", initial_state), ("final_state", final_state)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"{name} must be float32")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load().gdn_chunk_fwd_wk(_ptr(q), _ptr(k), _ptr(k_write), _ptr(v), _ptr(beta), _ptr(g),
                                 int(gate_kind), _ptr(initial_state), _ptr(o), _ptr(final_state),
                                 B, T, H, Dk, Dv, chunk, dt, _ptr(workspace), ws_bytes,
                                 _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_chunk_fwd_wk")


def gdn_osdn_precondition_workspace_bytes(B, T, H, Dk) -> int:
    n = load().gdn_osdn_precondition_workspace_bytes(B, T, H, Dk)
    if n == ctypes.c_size_t(-1).value:
        raise GdnError(GDN_ERR_INVALID_ARG, "gdn_osdn_precondition_workspace_bytes")
    return n


def gdn_osdn_precondition(k, beta, r, eta, d0, k_write, d_final, *, workspace=None,
                          stream=None) -> None:
    """Phase 1 of the preconditioned delta rule: write keys k_write = d (.) k.
    k, k_write [B,T,H,Dk]; beta, r [B,T,H] (r may be None); d0, d_final
    [B,H,Dk] fp32 or None; workspace a uint8 device tensor (allocated here
    with torch when None)."""
    _check_contig(k=k, beta=beta, r=r, d0=d0, k_write=k_write, d_final=d_final)
    B, T, H, Dk = k.shape
    dt = _dtype_code(k.dtype)
    for name, t in (("beta", beta), ("r", r), ("k_write", k_write)):
        if t is not None and t.dtype != k.dtype:
            raise TypeError(f"{name} must have dtype {k.dtype}")
    for name, t in (("d0", d0), ("d_final", d_final)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"{name} must be float32")
    if workspace is None:
        n = gdn_osdn_precondition_workspace_bytes(B, T, H, Dk)
        workspace = torch.empty(n, dtype=torch.uint8, device=k.device) if n else None
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load().gdn_osdn_precondition(_ptr(k), _ptr(beta), _ptr(r), float(eta), _ptr(d0),
                                      _ptr(k_write), _ptr(d_final), B, T, H, Dk, dt,
                                      _ptr(workspace), ws_bytes, _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_osdn_precondition")


def gdn_chunk_bwd_workspace_bytes(B, T, H, Dk, Dv, chunk=64, dtype=torch.bfloat16,
                                  gate_kind=GDN_GATE_SCALAR) -> int:
    n = load().gdn_chunk_bwd_workspace_bytes(B, T, H, Dk, Dv, chunk, _dtype_code(dtype),
                                             int(gate_kind))
    if n == ctypes.c_size_t(-1).value:
        raise GdnError(GDN_ERR_UNSUPPORTED, "gdn_chunk_bwd_workspace_bytes")
    return n


def gdn_chunk_bwd(q, k, v, beta, g, gate_kind, initial_state, d_o, d_final_state, dq, dk, dv,
                  dbeta, dg, d_initial_state, *, chunk=64, workspace=None, stream=None) -> None:
    """Enqueue the backward of the chunk forward: fp32 gradients dq, dk [B,T,H,Dk],
    dv [B,T,H,Dv], dbeta, dg [B,T,H] (dg None without a gate), d_initial_state
    [B,H,Dk,Dv] or None, from d_o [B,T,H,Dv] (dtype of q) and d_final_state."""
    _check_contig(q=q, k=k, v=v, beta=beta, g=g, initial_state=initial_state, d_o=d_o,
                  d_final_state=d_final_state, dq=dq, dk=dk, dv=dv, dbeta=dbeta, dg=dg,
                  d_initial_state=d_initial_state)
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv), ("dbeta", dbeta), ("dg", dg),
                    ("d_initial_state", d_initial_state), ("d_final_state", d_final_state),
                    ("initial_state", initial_state)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"{name} must be float32")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load().gdn_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), int(gate_kind),
                              _ptr(initial_state), _ptr(d_o), _ptr(d_final_state), _ptr(dq),
                              _ptr(dk), _ptr(dv), _ptr(dbeta), _ptr(dg), _ptr(d_initial_state),
                              B, T, H, Dk, Dv, chunk, _dtype_code(q.dtype), _ptr(workspace),
                              ws_bytes, _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_chunk_bwd")


def chunk_bwd(q, k, v, beta, g, initial_state, d_o, d_final_state=None, *, chunk=64,
              stream=None):
    """Allocate the gradients and the workspace with torch and run gdn_chunk_bwd.
    Returns dict dq, dk, dv, dbeta, dg (None without a gate), d_initial_state."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    gate = GDN_GATE_NONE if g is None else GDN_GATE_SCALAR
    dev = q.device
    out = {"dq": torch.empty(B, T, H, Dk, device=dev), "dk": torch.empty(B, T, H, Dk, device=dev),
           "dv": torch.empty(B, T, H, Dv, device=dev), "dbeta": torch.empty(B, T, H, device=dev),
           "dg": None if g is None else torch.empty(B, T, H, device=dev),
           "d_initial_state": torch.empty(B, H, Dk, Dv, device=dev)}
    n = gdn_chunk_bwd_workspace_bytes(B, T, H, Dk, Dv, chunk, q.dtype, gate)
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
    gdn_chunk_bwd(q, k, v, beta, g, gate, initial_state, d_o, d_final_state, out["dq"], out["dk"],
                  out["dv"], out["dbeta"], out["dg"], out["d_initial_state"], chunk=chunk,
                  workspace=ws, stream=stream)
    return out


def gdn_decode_step(q, k, v, beta, g, gate_kind, state, o, *, stream=None) -> None:
    """Enqueue one decode step.  q, k [N,H,Dk]; v, o [N,H,Dv]; beta [N,H];
    g [N,H] or [N,H,Dk] or None; state [N,H,Dk,Dv] fp32, updated in place."""
    _check_contig(q=q, k=k, v=v, beta=beta, g=g, state=state, o=o)
    N, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dtype_code(q.dtype)
    if state.dtype != torch.float32:
        raise TypeError("state must be float32")
    st = load().gdn_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), int(gate_kind),
                                _ptr(state), _ptr(o), N, H, Dk, Dv, dt, _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_decode_step")


def gdn_read_device_status(stream=None) -> int:
    return load().gdn_read_device_status(_stream(stream))


# ----------------------------------------------------------------- convenience
def chunk_fwd(q, k, v, beta, g=None, initial_state=None, *, output_final_state=True,
              chunk=64, stream=None):
    """Allocate o (and the final state) with torch and run gdn_chunk_fwd.
    The gate kind follows g: None -> none, [B,T,H] -> scalar, [B,T,H,Dk] ->
    per-dimension.  Returns (o, final_state or None)."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    gate = GDN_GATE_NONE if g is None else (GDN_GATE_SCALAR if g.dim() == 3 else GDN_GATE_PER_DIM)
    o = torch.empty((B, T, H, Dv), dtype=q.dtype, device=q.device)
    S = (torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=q.device)
         if output_final_state else None)
    ws_n = gdn_chunk_fwd_workspace_bytes(B, T, H, Dk, Dv, chunk, q.dtype, gate)
    ws = torch.empty(ws_n, dtype=torch.uint8, device=q.device) if ws_n else None
    gdn_chunk_fwd(q, k, v, beta, g, gate, initial_state, o, S, chunk=chunk, workspace=ws,
                  stream=stream)
    return o, S


def osdn_chunk_fwd(q, k, v, beta, g=None, initial_state=None, *, eta, r=None, d0=None,
                   output_final_state=True, chunk=64, stream=None):
    """The preconditioned delta rule, both phases: write keys from the
    preconditioner scan, then the chunk forward with them.  Returns
    (o, final_state or None, d_final)."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    gate = GDN_GATE_NONE if g is None else (GDN_GATE_SCALAR if g.dim() == 3 else GDN_GATE_PER_DIM)
    kw = torch.empty_like(k)
    d_final = torch.empty((B, H, Dk), dtype=torch.float32, device=q.device)
    gdn_osdn_precondition(k, beta, r, eta, d0, kw, d_final, stream=stream)
    o = torch.empty((B, T, H, Dv), dtype=q.dtype, device=q.device)
    S = (torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=q.device)
         if output_final_state else None)
    ws_n = gdn_chunk_fwd_workspace_bytes(B, T, H, Dk, Dv, chunk, q.dtype, gate)
    ws = torch.empty(ws_n, dtype=torch.uint8, device=q.device) if ws_n else None
    gdn_chunk_fwd_wk(q, k, kw, v, beta, g, gate, initial_state, o, S, chunk=chunk, workspace=ws,
                     stream=stream)
    return o, S, d_final


def decode_step(q, k, v, beta, g, state, *, stream=None):
    """One decode step; updates `state` in place and returns o."""
    N, H, Dk = q.shape
    gate = GDN_GATE_NONE if g is None else (GDN_GATE_SCALAR if g.dim() == 2 else GDN_GATE_PER_DIM)
    o = torch.empty((N, H, v.shape[-1]), dtype=q.dtype, device=q.device)
    gdn_decode_step(q, k, v, beta, g, gate, state, o, stream=stream)
    return o
