"""B200 (sm_100a) Gated DeltaNet chunked prefill: Python binding of the C ABI.

Argument marshalling only. Every step of the operator runs in the CUDA kernels
of the in-tree library libgdn.so (see include/gdn.h); PyTorch provides device
memory and streams. There is no CPU path: if the library is missing, importing
works but every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = ["lib", "GdnError", "gdn_chunk_fwd", "gdn_chunk_fwd_noalloc", "gdn_chunk_bwd", "fwd_workspace_size",
           "bwd_workspace_size", "chunk_states", "read_device_status", "check_device_error", "Options",
           "LIB_PATH", "KernelTrace", "launch_count", "gdn_recurrent_step", "chunk_gated_delta_rule",
           "gdn_chunk_host", "host_scratch_size", "HOST_MODES"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgdn.so")

GDN_F32, GDN_BF16 = 0, 1
HOST_MODES = {"fwd": 1, "bwd": 2, "fwdbwd": 3}     # gdn_host_mode
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "workspace",
          4: "CUDA runtime error", 5: "device timeout", 6: "inconsistent device input",
          7: "unusable kernel launch"}


def _check_default() -> bool:
    """Whether calls read back the device status word by default (environment GDN_CHECK_STATUS=1)."""
    return os.environ.get("GDN_CHECK_STATUS", "0") not in ("", "0")


class GdnError(RuntimeError):
    def __init__(self, code: int, where: str):
        detail = ""
        if code in (3, 4) and _lib is not None:
            text = _lib.gdn_last_error().decode(errors="replace")
            if text:
                detail = " -- " + text
        super().__init__(f"{where}: {STATUS.get(code, code)} (status {code}){detail}")
        self.code = code


class Options(ctypes.Structure):
    """Mirror of gdn_options (include/gdn.h)."""
    _fields_ = [("cp_mode", ctypes.c_int), ("deterministic", ctypes.c_int),
                ("cp_segment_chunks", ctypes.c_int), ("cp_exact", ctypes.c_int),
                ("states", ctypes.c_void_p), ("qk_l2norm", ctypes.c_int), ("test_stall", ctypes.c_int),
                ("reserved", ctypes.c_int * 2)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C-ABI library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libgdn.so not built ({LIB_PATH}); run "
                               "`python -m gated_deltanet_chunked_prefill_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        dims = [i] * 7
        L.gdn_chunk_fwd_workspace_size.argtypes = dims + [vp]
        L.gdn_chunk_fwd_workspace_size.restype = sz
        L.gdn_chunk_bwd_workspace_size.argtypes = dims + [vp]
        L.gdn_chunk_bwd_workspace_size.restype = sz
        L.gdn_chunk_states_size.argtypes = dims
        L.gdn_chunk_states_size.restype = sz
        L.gdn_chunk_fwd.argtypes = [i] + [i] * 6 + [vp, vp, vp, vp, vp, f, vp, vp, i, vp, vp, vp, sz,
                                                    vp, vp]
        L.gdn_chunk_fwd.restype = i
        L.gdn_chunk_bwd.argtypes = [i] + [i] * 6 + [vp, vp, vp, vp, vp, f, vp, vp, i, vp, vp,
                                                    vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]
        L.gdn_chunk_bwd.restype = i
        L.gdn_chunk_fwd_noalloc.argtypes = [i] + [i] * 6 + [vp, vp, vp, vp, vp, f, vp, vp, i, vp, vp,
                                                            vp, vp]
        L.gdn_chunk_fwd_noalloc.restype = i
        L.gdn_chunk_host_scratch_size.argtypes = [i, i] + dims + [vp]
        L.gdn_chunk_host_scratch_size.restype = sz
        L.gdn_chunk_host.argtypes = ([i, i] + [i] * 6 + [vp, vp, vp, vp, vp, f, vp, vp, i, vp, vp, vp, vp,
                                     vp, vp, vp, vp, vp, vp, vp, sz, vp, vp, vp, vp])
        L.gdn_chunk_host.restype = i
        L.gdn_recurrent_step.argtypes = [i] * 6 + [vp, vp, vp, vp, vp, f, vp, vp, vp]
        L.gdn_recurrent_step.restype = i
        L.gdn_read_device_status.argtypes = [vp, vp]
        L.gdn_read_device_status.restype = i
        L.gdn_check_device_error.argtypes = [vp]
        L.gdn_check_device_error.restype = i
        L.gdn_status_string.argtypes = [i]
        L.gdn_status_string.restype = ctypes.c_char_p
        L.gdn_last_error.argtypes = []
        L.gdn_last_error.restype = ctypes.c_char_p
        L.gdn_trace_begin.argtypes = [i]
        L.gdn_trace_begin.restype = i
        L.gdn_trace_end.argtypes = [vp, vp]
        L.gdn_trace_end.restype = i
        L.gdn_kernel_name.argtypes = [i]
        L.gdn_kernel_name.restype = ctypes.c_char_p
        L.gdn_launch_count.argtypes = []
        L.gdn_launch_count.restype = ctypes.c_longlong
        L.gdn_version.argtypes = []
        L.gdn_version.restype = i
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise TypeError(f"unsupported I/O dtype {t.dtype}")


def _opts(cp_segment_chunks: int = 0, cp_exact: bool = False, states=None, cp_mode: int = 0,
          qk_l2norm: bool = False, deterministic: bool = False, test_stall: bool = False):
    o = Options()
    o.cp_mode = int(cp_mode)
    o.deterministic = int(bool(deterministic))
    o.cp_segment_chunks = int(cp_segment_chunks)
    o.cp_exact = int(cp_exact)       # 0 automatic, 1 exact stitch, 2 gate-driven restart (bool accepted)
    o.qk_l2norm = int(bool(qk_l2norm))
    o.test_stall = int(bool(test_stall))
    if states is not None:
        if states.dtype != torch.bfloat16 or not states.is_cuda or not states.is_contiguous():
            raise ValueError("states: a contiguous bf16 CUDA tensor from chunk_states()")
        o.states = states.data_ptr()
    return o


def _check_states(states, q, v, cu_seqlens):
    """The C ABI takes the chunk-state cache as a bare pointer: refuse one that is too small for
    these sizes or lives on another device before the kernels write or read it."""
    if states is None:
        return
    if states.device != q.device:
        raise ValueError(f"states is on device {states.device}, the inputs on {q.device}")
    B, T, Hqk, Hv, dk, dv, N = _dims(q, v, cu_seqlens)
    need = int(lib().gdn_chunk_states_size(B, T, Hqk, Hv, dk, dv, N))
    if states.numel() * states.element_size() < need:
        raise ValueError(f"states holds {states.numel() * states.element_size()} bytes; these sizes need {need} "
                         "(make it with chunk_states() on the same inputs)")


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dims(q, v, cu_seqlens):
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    N = B if cu_seqlens is None else cu_seqlens.numel() - 1
    return B, T, Hqk, Hv, dk, dv, N


def fwd_workspace_size(B, T, Hqk, Hv, dk, dv, N, cp_segment_chunks=0, cp_exact=False, cp_mode=0) -> int:
    o = _opts(cp_segment_chunks, cp_exact, cp_mode=cp_mode)
    return int(lib().gdn_chunk_fwd_workspace_size(B, T, Hqk, Hv, dk, dv, N, ctypes.byref(o)))


def bwd_workspace_size(B, T, Hqk, Hv, dk, dv, N, cp_segment_chunks=0, cp_exact=False, states=None,
                       cp_mode=0) -> int:
    o = _opts(cp_segment_chunks, cp_exact, states, cp_mode=cp_mode)
    return int(lib().gdn_chunk_bwd_workspace_size(B, T, Hqk, Hv, dk, dv, N, ctypes.byref(o)))


def chunk_states(q, v, cu_seqlens=None):
    """A chunk-start-state cache (gdn_options.states) for these inputs: pass it as
    `states=` to gdn_chunk_fwd, then to gdn_chunk_bwd, which then skips its forward pass."""
    B, T, Hqk, Hv, dk, dv, N = _dims(q, v, cu_seqlens)
    nbytes = int(lib().gdn_chunk_states_size(B, T, Hqk, Hv, dk, dv, N))
    return torch.empty(max(nbytes // 2, 1), dtype=torch.bfloat16, device=q.device)


def _check_shapes(q, k, v, g, beta, h0=None, cu_seqlens=None, dO=None, dhT=None, o=None, hT=None):
    """The C ABI takes its sizes from q and v and trusts every other array to match them, so a
    mismatch is refused here, on the host, before anything reaches the GPU (tensor shapes only)."""
    if q.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k must be [B,T,Hqk,dk] and v [B,T,Hv,dv]")
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    if tuple(k.shape) != tuple(q.shape):
        raise ValueError(f"k must have q's shape {tuple(q.shape)}, got {tuple(k.shape)}")
    if tuple(v.shape[:2]) != (B, T):
        raise ValueError(f"v must be [{B},{T},Hv,dv], got {tuple(v.shape)}")
    for t, n in ((g, "g"), (beta, "beta")):
        if tuple(t.shape) != (B, T, Hv):
            raise ValueError(f"{n} must be [{B},{T},{Hv}], got {tuple(t.shape)}")
    if cu_seqlens is not None and (cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1):
        raise ValueError("cu_seqlens must be 1-D [N+1]")
    N = B if cu_seqlens is None else cu_seqlens.numel() - 1
    for t, n in ((h0, "h0"), (dhT, "dhT"), (hT, "hT")):
        if t is not None and tuple(t.shape) != (N, Hv, dk, dv):
            raise ValueError(f"{n} must be [{N},{Hv},{dk},{dv}], got {tuple(t.shape)}")
    for t, n in ((dO, "dO"), (o, "o")):
        if t is not None and tuple(t.shape) != tuple(v.shape):
            raise ValueError(f"{n} must have v's shape {tuple(v.shape)}, got {tuple(t.shape)}")


def _check(t, name, dtype=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _workspace(nbytes, workspace, device):
    if workspace is None:
        return torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
    if workspace.numel() < nbytes:
        raise ValueError(f"workspace too small: {workspace.numel()} < {nbytes}")
    return workspace


def _status_after(ws, stream, where):
    """Synchronise and raise if the call's kernels recorded a device-side finding in `ws`."""
    code = read_device_status(ws, stream)
    if code != 0:
        raise GdnError(code, where + " (device status)")


def gdn_chunk_fwd(q, k, v, g, beta, scale=None, h0=None, cu_seqlens=None,
                  output_final_state=True, cp_segment_chunks=0, cp_exact=False, workspace=None,
                  o=None, hT=None, stream=None, states=None, cp_mode=0, qk_l2norm=False,
                  deterministic=False, check_status=None, test_stall=False):
    """Forward through the C ABI. Returns (o, hT or None). With `states` (from
    chunk_states()) it also writes every chunk's start state for a later backward.

    Device-side findings (inconsistent cu_seqlens, a timed-out wait) leave o / hT unspecified and
    are only visible through the workspace's status word: with check_status=True (default: the
    environment variable GDN_CHECK_STATUS=1) the call synchronises, reads it and raises GdnError.
    Otherwise read it with read_device_status(workspace) or check_device_error()."""
    _check_shapes(q, k, v, g, beta, h0, cu_seqlens, o=o, hT=hT)
    io = q.dtype
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (beta, "beta")):
        _check(t, n, io)
    _check(g, "g", torch.float32)
    _check(h0, "h0", torch.float32)
    _check(cu_seqlens, "cu_seqlens", torch.int32)
    _check_states(states, q, v, cu_seqlens)
    B, T, Hqk, Hv, dk, dv, N = _dims(q, v, cu_seqlens)
    scale = dk ** -0.5 if scale is None else float(scale)
    if o is None:
        o = torch.empty((B, T, Hv, dv), dtype=io, device=q.device)
    if hT is None and output_final_state:
        hT = torch.empty((N, Hv, dk, dv), dtype=torch.float32, device=q.device)
    ws_bytes = fwd_workspace_size(B, T, Hqk, Hv, dk, dv, N, cp_segment_chunks, cp_exact, cp_mode)
    ws = _workspace(ws_bytes, workspace, q.device)
    opt = _opts(cp_segment_chunks, cp_exact, states, cp_mode, qk_l2norm, deterministic, test_stall)
    st = lib().gdn_chunk_fwd(_dtype_code(q), B, T, Hqk, Hv, dk, dv, _ptr(q), _ptr(k), _ptr(v),
                             _ptr(g), _ptr(beta), scale, _ptr(h0), _ptr(cu_seqlens), N, _ptr(o),
                             _ptr(hT), _ptr(ws), ws.numel(), ctypes.byref(opt), _stream(stream))
    if st != 0:
        raise GdnError(st, "gdn_chunk_fwd")
    if _check_default() if check_status is None else check_status:
        _status_after(ws, stream, "gdn_chunk_fwd")
    return o, hT


def gdn_chunk_fwd_noalloc(q, k, v, g, beta, scale=None, h0=None, cu_seqlens=None,
                          output_final_state=True, cp_segment_chunks=0, o=None, hT=None, stream=None,
                          cp_mode=0, check_status=None):
    """Forward through the allocation-free entry point (library-held 1 MiB scratch; see gdn.h).
    With check_status (as in gdn_chunk_fwd) the device-side findings are read through
    check_device_error(), the per-device status word."""
    _check_shapes(q, k, v, g, beta, h0, cu_seqlens, o=o, hT=hT)
    io = q.dtype
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (beta, "beta")):
        _check(t, n, io)
    _check(g, "g", torch.float32)
    _check(h0, "h0", torch.float32)
    _check(cu_seqlens, "cu_seqlens", torch.int32)
    B, T, Hqk, Hv, dk, dv, N = _dims(q, v, cu_seqlens)
    scale = dk ** -0.5 if scale is None else float(scale)
    if o is None:
        o = torch.empty((B, T, Hv, dv), dtype=io, device=q.device)
    if hT is None and output_final_state:
        hT = torch.empty((N, Hv, dk, dv), dtype=torch.float32, device=q.device)
    opt = _opts(cp_segment_chunks, cp_mode=cp_mode)
    st = lib().gdn_chunk_fwd_noalloc(_dtype_code(q), B, T, Hqk, Hv, dk, dv, _ptr(q), _ptr(k), _ptr(v),
                                     _ptr(g), _ptr(beta), scale, _ptr(h0), _ptr(cu_seqlens), N,
                                     _ptr(o), _ptr(hT), ctypes.byref(opt), _stream(stream))
    if st != 0:
        raise GdnError(st, "gdn_chunk_fwd_noalloc")
    if _check_default() if check_status is None else check_status:
        code = check_device_error(stream)
        if code != 0:
            raise GdnError(code, "gdn_chunk_fwd_noalloc (device status)")
    return o, hT


def gdn_chunk_bwd(q, k, v, g, beta, dO, scale=None, h0=None, dhT=None, cu_seqlens=None,
                  cp_segment_chunks=0, cp_exact=False, workspace=None, want_dh0=True, stream=None,
                  states=None, cp_mode=0, qk_l2norm=False, deterministic=False, check_status=None):
    """Backward through the C ABI. Returns dict dq, dk, dv, dg, dbeta, dh0. With `states`
    written by the matching gdn_chunk_fwd call, the forward pass is not recomputed.
    check_status: as in gdn_chunk_fwd (device-side findings otherwise leave the gradients
    unspecified without an exception)."""
    _check_shapes(q, k, v, g, beta, h0, cu_seqlens, dO=dO, dhT=dhT)
    io = q.dtype
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (beta, "beta"), (dO, "dO")):
        _check(t, n, io)
    _check(g, "g", torch.float32)
    _check(h0, "h0", torch.float32)
    _check(dhT, "dhT", torch.float32)
    _check(cu_seqlens, "cu_seqlens", torch.int32)
    _check_states(states, q, v, cu_seqlens)
    B, T, Hqk, Hv, dk, dv, N = _dims(q, v, cu_seqlens)
    scale = dk ** -0.5 if scale is None else float(scale)
    dq = torch.empty_like(q)
    dkk = torch.empty_like(k)
    dvv = torch.empty_like(v)
    dg = torch.empty_like(g)
    db = torch.empty_like(beta)
    dh0 = torch.empty((N, Hv, dk, dv), dtype=torch.float32, device=q.device) if want_dh0 else None
    ws_bytes = bwd_workspace_size(B, T, Hqk, Hv, dk, dv, N, cp_segment_chunks, cp_exact, states, cp_mode)
    ws = _workspace(ws_bytes, workspace, q.device)
    opt = _opts(cp_segment_chunks, cp_exact, states, cp_mode, qk_l2norm, deterministic)
    st = lib().gdn_chunk_bwd(_dtype_code(q), B, T, Hqk, Hv, dk, dv, _ptr(q), _ptr(k), _ptr(v),
                             _ptr(g), _ptr(beta), scale, _ptr(h0), _ptr(cu_seqlens), N, _ptr(dO),
                             _ptr(dhT), _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dg), _ptr(db),
                             _ptr(dh0), _ptr(ws), ws.numel(), ctypes.byref(opt), _stream(stream))
    if st != 0:
        raise GdnError(st, "gdn_chunk_bwd")
    if _check_default() if check_status is None else check_status:
        _status_after(ws, stream, "gdn_chunk_bwd")
    return dict(dq=dq, dk=dkk, dv=dvv, dg=dg, dbeta=db, dh0=dh0)


def host_scratch_size(mode, dtype, B, T, Hqk, Hv, dk, dv, N, cp_segment_chunks=0, cp_exact=False, cp_mode=0,
                      qk_l2norm=False) -> int:
    """Bytes of device scratch gdn_chunk_host needs (mode "fwd", "bwd" or "fwdbwd")."""
    o = _opts(cp_segment_chunks, cp_exact, cp_mode=cp_mode, qk_l2norm=qk_l2norm)
    code = GDN_BF16 if dtype == torch.bfloat16 else GDN_F32
    return int(lib().gdn_chunk_host_scratch_size(HOST_MODES[mode], code, B, T, Hqk, Hv, dk, dv, N, ctypes.byref(o)))


def _check_host(t, name, dtype=None):
    if t is None:
        return
    if t.is_cuda:
        raise ValueError(f"{name} must be a CPU tensor (host-buffer call)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def gdn_chunk_host(q, k, v, g, beta, scale=None, h0=None, cu_seqlens=None, dO=None, dhT=None, mode=None,
                   scratch=None, outputs=None, output_final_state=True, want_dh0=True, stream=None,
                   h2d_stream=None, d2h_stream=None, device=None, cp_segment_chunks=0, cp_exact=False, cp_mode=0,
                   qk_l2norm=False, synchronize=True):
    """Host-buffer call through the C ABI (gdn_chunk_host): CPU tensors in, CPU tensors out; the copies
    and the kernels run on the current (or given) CUDA device. mode "fwd" (default without dO),
    "bwd" (forward pass recomputed) or "fwdbwd" (default with dO). Page-locked inputs and outputs
    (Tensor.pin_memory()) let the copies overlap; `outputs` (a dict from an earlier call) reuses
    output buffers, `scratch` a device buffer of host_scratch_size() bytes. With synchronize=False
    the call returns once everything is enqueued: the outputs are valid after d2h_stream (or stream)
    synchronises. Returns a dict of the outputs (o, hT; dq, dk, dv, dg, dbeta, dh0)."""
    mode = mode or ("fwd" if dO is None else "fwdbwd")
    if mode not in HOST_MODES:
        raise ValueError(f"mode must be one of {sorted(HOST_MODES)}")
    fw, bw = mode in ("fwd", "fwdbwd"), mode in ("bwd", "fwdbwd")
    if bw and dO is None:
        raise ValueError(f"mode {mode!r} needs dO")
    _check_shapes(q, k, v, g, beta, h0, cu_seqlens, dO=dO if bw else None, dhT=dhT if bw else None)
    io = q.dtype
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (beta, "beta")):
        _check_host(t, n, io)
    _check_host(g, "g", torch.float32)
    _check_host(h0, "h0", torch.float32)
    _check_host(cu_seqlens, "cu_seqlens", torch.int32)
    if bw:
        _check_host(dO, "dO", io)
        _check_host(dhT, "dhT", torch.float32)
    B, T, Hqk, Hv, dk, dv, N = _dims(q, v, cu_seqlens)
    scale = dk ** -0.5 if scale is None else float(scale)
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    pin = q.is_pinned()
    out = dict(outputs) if outputs is not None else {}

    def buf(name, shape, dtype, want=True):
        if not want:
            return None
        t = out.get(name)
        if t is None:
            t = torch.empty(shape, dtype=dtype, pin_memory=pin)
            out[name] = t
        _check_host(t, name, dtype)
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} must be {tuple(shape)}, got {tuple(t.shape)}")
        return t

    o = buf("o", (B, T, Hv, dv), io, fw)
    hT = buf("hT", (N, Hv, dk, dv), torch.float32, fw and output_final_state)
    dq = buf("dq", tuple(q.shape), io, bw)
    dkk = buf("dk", tuple(k.shape), io, bw)
    dvv = buf("dv", tuple(v.shape), io, bw)
    dg = buf("dg", tuple(g.shape), torch.float32, bw)
    db = buf("dbeta", tuple(beta.shape), io, bw)
    dh0 = buf("dh0", (N, Hv, dk, dv), torch.float32, bw and want_dh0)
    need = host_scratch_size(mode, io, B, T, Hqk, Hv, dk, dv, N, cp_segment_chunks, cp_exact, cp_mode, qk_l2norm)
    if scratch is None:
        scratch = torch.empty(max(need, 256), dtype=torch.uint8, device=device)
    elif not scratch.is_cuda or scratch.numel() * scratch.element_size() < need:
        raise ValueError(f"scratch must be a CUDA tensor of at least {need} bytes")
    opt = _opts(cp_segment_chunks, cp_exact, cp_mode=cp_mode, qk_l2norm=qk_l2norm)
    st_main = torch.cuda.current_stream(device) if stream is None else stream
    with torch.cuda.device(device):
        st = lib().gdn_chunk_host(HOST_MODES[mode], _dtype_code(q), B, T, Hqk, Hv, dk, dv, _ptr(q), _ptr(k),
                                  _ptr(v), _ptr(g), _ptr(beta), scale, _ptr(h0), _ptr(cu_seqlens), N,
                                  _ptr(dO if bw else None), _ptr(dhT if bw else None), _ptr(o), _ptr(hT),
                                  _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dg), _ptr(db), _ptr(dh0), _ptr(scratch),
                                  scratch.numel() * scratch.element_size(), ctypes.byref(opt),
                                  ctypes.c_void_p(st_main.cuda_stream),
                                  ctypes.c_void_p(h2d_stream.cuda_stream if h2d_stream is not None else 0),
                                  ctypes.c_void_p(d2h_stream.cuda_stream if d2h_stream is not None else 0))
    if st != 0:
        raise GdnError(st, "gdn_chunk_host")
    if synchronize:
        (d2h_stream if d2h_stream is not None else st_main).synchronize()
    return out


def gdn_recurrent_step(q, k, v, g, beta, state, scale=None, o=None, stream=None):
    """One decode step through the C ABI: q, k [N,Hqk,dk], v [N,Hv,dv], beta [N,Hv] (one dtype),
    g [N,Hv] fp32; `state` [N,Hv,dk,dv] fp32 (e.g. a prefill's hT) is advanced in place.
    Returns o [N,Hv,dv]."""
    if q.dim() != 3 or v.dim() != 3:
        raise ValueError("q, k must be [N,Hqk,dk] and v [N,Hv,dv]")
    N, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    if tuple(k.shape) != tuple(q.shape) or v.shape[0] != N:
        raise ValueError(f"k must have q's shape {tuple(q.shape)} and v must be [{N},Hv,dv]")
    for t, n in ((g, "g"), (beta, "beta")):
        if tuple(t.shape) != (N, Hv):
            raise ValueError(f"{n} must be [{N},{Hv}], got {tuple(t.shape)}")
    if tuple(state.shape) != (N, Hv, dk, dv):
        raise ValueError(f"state must be [{N},{Hv},{dk},{dv}], got {tuple(state.shape)}")
    if o is not None and tuple(o.shape) != (N, Hv, dv):
        raise ValueError(f"o must be [{N},{Hv},{dv}], got {tuple(o.shape)}")
    io = q.dtype
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (beta, "beta")):
        _check(t, n, io)
    _check(g, "g", torch.float32)
    _check(state, "state", torch.float32)
    _check(o, "o", io)
    scale = dk ** -0.5 if scale is None else float(scale)
    if o is None:
        o = torch.empty((N, Hv, dv), dtype=io, device=q.device)
    st = lib().gdn_recurrent_step(_dtype_code(q), N, Hqk, Hv, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                  _ptr(beta), scale, _ptr(state), _ptr(o), _stream(stream))
    if st != 0:
        raise GdnError(st, "gdn_recurrent_step")
    return o


class KernelTrace:
    """Context manager: device time of every kernel the library launches inside it.

    After exit, `launches` holds (kernel name, milliseconds) per launch, in order.
    The library records the CUDA events itself, on each kernel's launch stream.
    """

    def __init__(self, capacity: int = 256):
        self.capacity = capacity
        self.launches = []

    def __enter__(self):
        st = lib().gdn_trace_begin(self.capacity)
        if st != 0:
            raise GdnError(st, "gdn_trace_begin")
        return self

    def __exit__(self, *exc):
        ms = (ctypes.c_float * self.capacity)()
        ids = (ctypes.c_int * self.capacity)()
        n = lib().gdn_trace_end(ms, ids)
        if n < 0:
            raise GdnError(4, "gdn_trace_end")
        self.launches = [(lib().gdn_kernel_name(ids[i]).decode(), float(ms[i])) for i in range(n)]
        return False


def launch_count() -> int:
    """Kernels launched by the library from this host thread so far."""
    return int(lib().gdn_launch_count())


def read_device_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise and return (and clear) the workspace's device status word."""
    return int(lib().gdn_read_device_status(_ptr(workspace), _stream(stream)))


def check_device_error(stream=None) -> int:
    """Synchronise `stream` and return (and clear) the library's per-device status word: the first
    device-side finding of any call on the current device since the last check (0 = none)."""
    return int(lib().gdn_check_device_error(_stream(stream)))


from .autograd import chunk_gated_delta_rule  # noqa: E402  (uses the functions above)
