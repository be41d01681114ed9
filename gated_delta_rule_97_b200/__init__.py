"""B200 (sm_100a) gated delta-rule library: thin Python binding of libgdn.so.

The compute lives in ``libgdn.so`` (CUDA kernels behind the C ABI declared in
``include/gdn.h``).  This module only marshals arguments: it checks tensor
shapes and dtypes, passes raw device pointers and the current CUDA stream to
the C entry points, and raises ``GDNError`` on a non-zero return code.  There
is no fallback: if the library is not built, every call raises.

    import gated_delta_rule_97_b200 as gdn
    o, S_T = gdn.chunk_fwd(q, k, v, g, beta, S0, update="delta", gate="scalar")
    o = gdn.decode_step(q1, k1, v1, g1, beta1, S, update="delta", gate="scalar")
"""
from __future__ import annotations

import ctypes
import os

__all__ = ["GDNError", "chunk_fwd", "decode_step", "device_status", "strerror", "version", "load",
           "lib_path", "Desc", "UPDATES", "GATES", "build", "device_diag", "product_fwd", "chunk_fwd_segmented",
           "segmented_workspace_bytes", "segment_maps", "compose_segments", "chunk_fwd_host",
           "host_workspace_bytes", "chunk_bwd", "bwd_workspace_bytes"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libgdn.so")

UPDATES = {"additive": 0, "decay": 1, "delta": 2}
GATES = {"none": 0, "scalar": 1, "channel": 2}
ALGOS = {"auto": 0, "simt": 1, "tc": 2}
F32, BF16 = 0, 1

DECODE_MAX_T = 16  # GDN_DECODE_MAX_T
PRODUCT_MAX_NH = 16  # GDN_PRODUCT_MAX_NH
CHUNK = 64  # chunk length of the saved states (gdn_chunk_fwd_states)
GDN_OK = 0
ERRORS = {-1: "GDN_ERR_ARG", -2: "GDN_ERR_ALIGN", -3: "GDN_ERR_UNSUPPORTED", -4: "GDN_ERR_CUDA",
          -5: "GDN_ERR_TIMEOUT", -6: "GDN_ERR_RANGE"}


class GDNError(RuntimeError):
    def __init__(self, code, what=""):
        self.code = code
        super().__init__("%s: %s (%d)%s" % (ERRORS.get(code, "?"), strerror(code) if _lib else "", code,
                                            (" in " + what) if what else ""))


class Desc(ctypes.Structure):
    """Mirror of gdn_desc_t."""
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int), ("dk", ctypes.c_int),
                ("dv", ctypes.c_int), ("update", ctypes.c_int), ("gate", ctypes.c_int),
                ("dtype", ctypes.c_int), ("out_dtype", ctypes.c_int), ("chunk", ctypes.c_int),
                ("algo", ctypes.c_int), ("prologue", ctypes.c_int)]


_lib = None


def lib_path() -> str:
    return _LIB_PATH


def build(verbose: bool = False, force: bool = False) -> str:
    """Compiles libgdn.so in-tree (nvcc, sm_100a)."""
    from .builder import build as _build

    return _build(verbose=verbose, force=force)


def load():
    """Loads libgdn.so; raises if it is missing (there is no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError("libgdn.so is not built (%s); run gated_delta_rule_97_b200.build()" % _LIB_PATH)
    lib = ctypes.CDLL(_LIB_PATH)
    vp = ctypes.c_void_p
    dp = ctypes.POINTER(Desc)
    lib.gdn_chunk_fwd.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.gdn_chunk_fwd.restype = ctypes.c_int
    lib.gdn_decode_step.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.gdn_decode_step.restype = ctypes.c_int
    lib.gdn_product_fwd.argtypes = [dp, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.gdn_product_fwd.restype = ctypes.c_int
    lib.gdn_segmented_workspace_bytes.argtypes = [dp, ctypes.c_int]
    lib.gdn_segmented_workspace_bytes.restype = ctypes.c_size_t
    lib.gdn_chunk_fwd_segmented.argtypes = [dp, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.gdn_chunk_fwd_segmented.restype = ctypes.c_int
    lib.gdn_noalloc_scratch_bytes.argtypes = []
    lib.gdn_noalloc_scratch_bytes.restype = ctypes.c_size_t
    lib.gdn_chunk_fwd_segmented_noalloc.argtypes = [dp, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.gdn_chunk_fwd_segmented_noalloc.restype = ctypes.c_int
    lib.gdn_host_workspace_bytes.argtypes = [dp, ctypes.c_int]
    lib.gdn_host_workspace_bytes.restype = ctypes.c_size_t
    lib.gdn_chunk_fwd_host.argtypes = [dp, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.gdn_chunk_fwd_host.restype = ctypes.c_int
    lib.gdn_segment_maps.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.gdn_segment_maps.restype = ctypes.c_int
    lib.gdn_compose_segments.argtypes = [ctypes.c_int] * 4 + [vp] * 6
    lib.gdn_compose_segments.restype = ctypes.c_int
    lib.gdn_bwd_workspace_bytes.argtypes = [dp]
    lib.gdn_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.gdn_chunk_bwd.argtypes = [dp] + [vp] * 15 + [ctypes.c_size_t, vp]
    lib.gdn_chunk_bwd.restype = ctypes.c_int
    lib.gdn_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    lib.gdn_set_wait_limit_ns.restype = ctypes.c_int
    lib.gdn_chunk_fwd_states.argtypes = [dp] + [vp] * 10
    lib.gdn_chunk_fwd_states.restype = ctypes.c_int
    lib.gdn_chunk_bwd_states.argtypes = [dp] + [vp] * 15
    lib.gdn_chunk_bwd_states.restype = ctypes.c_int
    lib.gdn_chunk_fwd_checked.argtypes = [dp] + [vp] * 9
    lib.gdn_chunk_fwd_checked.restype = ctypes.c_int
    lib.gdn_bwd_tc_workspace_bytes.argtypes = [dp]
    lib.gdn_bwd_tc_workspace_bytes.restype = ctypes.c_size_t
    lib.gdn_chunk_bwd_tc.argtypes = [dp] + [vp] * 15 + [ctypes.c_size_t, vp]
    lib.gdn_chunk_bwd_tc.restype = ctypes.c_int
    lib.gdn_strerror.argtypes = [ctypes.c_int]
    lib.gdn_strerror.restype = ctypes.c_char_p
    lib.gdn_device_status.argtypes = [ctypes.c_int]
    lib.gdn_device_status.restype = ctypes.c_int
    lib.gdn_version.restype = ctypes.c_int
    lib.gdn_device_diag.restype = ctypes.c_int
    _lib = lib
    return lib


def strerror(code: int) -> str:
    return load().gdn_strerror(int(code)).decode()


def version() -> int:
    return int(load().gdn_version())


def device_status(clear: bool = True) -> int:
    """The library's device status word (synchronises the device)."""
    return int(load().gdn_device_status(1 if clear else 0))


def device_diag() -> int:
    """Where the first recorded kernel timeout happened (0 if none)."""
    return int(load().gdn_device_diag())


def set_wait_limit_ns(ns: int) -> None:
    """Bound of the kernels' hand-off waits in ns (0 = the default, 1 s): a test
    hook for the timeout path (gdn_set_wait_limit_ns)."""
    load().gdn_set_wait_limit_ns(ctypes.c_ulonglong(int(ns)))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, t):
    """The stream to launch on: ``stream``, else the current stream of the
    device that holds ``t``."""
    import torch

    s = torch.cuda.current_stream(t.device) if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _on_device(t):
    """Makes the device that holds ``t`` current for the call: the library
    launches on, and takes its status word and scratch from, the calling
    thread's current device."""
    import torch

    return torch.cuda.device(t.device)


def _dtype_code(dt):
    import torch

    if dt == torch.bfloat16:
        return BF16
    if dt == torch.float32:
        return F32
    raise TypeError("q, k, v, o must be bfloat16 or float32, got %s" % dt)


# Input prologue bits (GDN_PRO_*): maps applied in-kernel to the raw inputs
PRO_QK_ELU1, PRO_QK_L2, PRO_BETA_SIGMOID, PRO_G_NEG_SOFTPLUS = 1, 2, 4, 8


def make_desc(B, H, T, dk, dv, update, gate, dtype, out_dtype, algo="auto", chunk=64, prologue=0) -> Desc:
    return Desc(B, H, T, dk, dv, UPDATES[update], GATES[gate], dtype, out_dtype, chunk, ALGOS[algo], prologue)


def _check(t, name, shape, dtype=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))


def chunk_fwd(q, k, v, g=None, beta=None, S0=None, *, update, gate, out_dtype=None, o=None, S_T=None,
              return_state=True, algo="auto", prologue=0, states=None, checked=False, stream=None):
    """Prefill over T tokens (gdn_chunk_fwd).  Returns (o, S_T).

    ``states``: a CUDA float32 tensor [B,H,ceil(T/64),dv,dk] that receives the
    state entering every chunk (gdn_chunk_fwd_states, for chunk_bwd(states=...)).
    ``checked``: gdn_chunk_fwd_checked (synchronous; an fp16 operand overflow
    of a tensor-core kernel runs the request again on the fp32 kernel); returns
    (o, S_T, reran) then.

    q, k [B,H,T,dk]; v [B,H,T,dv] (bf16 or fp32, same dtype); g [B,H,T] or
    [B,H,T,dk] fp32 (log of the gate) or None; beta [B,H,T] fp32 (delta);
    S0 [B,H,dv,dk] fp32 or None.  o defaults to fp32; S_T may be S0 (in place).
    """
    import torch

    B, H, T, dk = q.shape
    dv = v.shape[-1]
    _check(q, "q", (B, H, T, dk))
    _check(k, "k", (B, H, T, dk), q.dtype)
    _check(v, "v", (B, H, T, dv), q.dtype)
    if gate == "scalar":
        _check(g, "g", (B, H, T), torch.float32)
    elif gate == "channel":
        _check(g, "g", (B, H, T, dk), torch.float32)
    _check(beta, "beta", (B, H, T), torch.float32)
    _check(S0, "S0", (B, H, dv, dk), torch.float32)
    if out_dtype is None:
        out_dtype = o.dtype if o is not None else torch.float32
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=out_dtype, device=q.device)
    _check(o, "o", (B, H, T, dv), out_dtype)
    if S_T is None and return_state:
        S_T = torch.empty((B, H, dv, dk), dtype=torch.float32, device=q.device)
    _check(S_T, "S_T", (B, H, dv, dk), torch.float32)
    d = make_desc(B, H, T, dk, dv, update, gate, _dtype_code(q.dtype), _dtype_code(out_dtype), algo,
                  prologue=prologue)
    if states is not None:
        _check(states, "states", (B, H, (T + CHUNK - 1) // CHUNK, dv, dk), torch.float32)
        with _on_device(q):
            rc = load().gdn_chunk_fwd_states(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                             _ptr(S0), _ptr(o), _ptr(S_T), _ptr(states), _stream(stream, q))
        if rc != GDN_OK:
            raise GDNError(rc, "gdn_chunk_fwd_states")
        return o, S_T
    if checked:
        with _on_device(q):
            rc = load().gdn_chunk_fwd_checked(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                              _ptr(S0), _ptr(o), _ptr(S_T), _stream(stream, q))
        if rc not in (GDN_OK, 1):
            raise GDNError(rc, "gdn_chunk_fwd_checked")
        return o, S_T, rc == 1
    with _on_device(q):
        rc = load().gdn_chunk_fwd(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                                  _ptr(o), _ptr(S_T), _stream(stream, q))
    if rc != GDN_OK:
        raise GDNError(rc, "gdn_chunk_fwd")
    return o, S_T


def _check_host(t, name, shape, dtype=None):
    if t is None:
        return
    if t.is_cuda:
        raise ValueError("%s must be a host (CPU) tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))


def host_workspace_bytes(B, H, T, dk, dv, update, gate, dtype, out_dtype=F32, n_slices=8) -> int:
    d = make_desc(B, H, T, dk, dv, update, gate, dtype, out_dtype)
    return int(load().gdn_host_workspace_bytes(ctypes.byref(d), int(n_slices)))


def chunk_fwd_host(q, k, v, g=None, beta=None, S0=None, *, update, gate, n_slices=8, out_dtype=None, o=None,
                   S_T=None, return_state=True, algo="auto", prologue=0, workspace=None, device=None, stream=None):
    """gdn_chunk_fwd_host: the prefill on host tensors (pin them for overlap),
    streamed to the GPU in ``n_slices`` head slices.  ``workspace``: a CUDA
    uint8 tensor of host_workspace_bytes(...) bytes (allocated here when None).
    Returns host (o, S_T), complete once ``stream`` (default: the current
    stream) has synchronised."""
    import torch

    B, H, T, dk = q.shape
    dv = v.shape[-1]
    _check_host(q, "q", (B, H, T, dk))
    _check_host(k, "k", (B, H, T, dk), q.dtype)
    _check_host(v, "v", (B, H, T, dv), q.dtype)
    if gate == "scalar":
        _check_host(g, "g", (B, H, T), torch.float32)
    elif gate == "channel":
        _check_host(g, "g", (B, H, T, dk), torch.float32)
    _check_host(beta, "beta", (B, H, T), torch.float32)
    _check_host(S0, "S0", (B, H, dv, dk), torch.float32)
    if out_dtype is None:
        out_dtype = o.dtype if o is not None else torch.float32
    pin = q.is_pinned()
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=out_dtype, pin_memory=pin)
    _check_host(o, "o", (B, H, T, dv), out_dtype)
    if S_T is None and return_state:
        S_T = torch.empty((B, H, dv, dk), dtype=torch.float32, pin_memory=pin)
    _check_host(S_T, "S_T", (B, H, dv, dk), torch.float32)
    d = make_desc(B, H, T, dk, dv, update, gate, _dtype_code(q.dtype), _dtype_code(out_dtype), algo,
                  prologue=prologue)
    need = int(load().gdn_host_workspace_bytes(ctypes.byref(d), int(n_slices)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8,
                                device=device if device is not None else torch.cuda.current_device())
    if not workspace.is_cuda or not workspace.is_contiguous() or workspace.numel() < need:
        raise ValueError("workspace needs %d contiguous CUDA bytes" % need)
    with _on_device(workspace):
        rc = load().gdn_chunk_fwd_host(ctypes.byref(d), int(n_slices), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                       _ptr(S0), _ptr(o), _ptr(S_T), _ptr(workspace), ctypes.c_size_t(workspace.numel()),
                                       _stream(stream, workspace))
    if rc != GDN_OK:
        raise GDNError(rc, "gdn_chunk_fwd_host")
    return o, S_T


def product_fwd(q, k, v, g=None, beta=None, S0=None, *, gate, out_dtype=None, o=None, S_T=None,
                return_state=True, algo="auto", prologue=0, stream=None):
    """Gated DeltaProduct prefill (gdn_product_fwd): nh = k.shape[-2] delta-rule
    substeps per token.  Returns (o, S_T).

    q [B,H,T,dk]; k [B,H,T,nh,dk]; v [B,H,T,nh,dv] (same dtype); beta [B,H,T,nh]
    fp32; g [B,H,T] or [B,H,T,dk] fp32 or None; S0 [B,H,dv,dk] fp32 or None.
    """
    import torch

    B, H, T, dk = q.shape
    nh, dv = k.shape[-2], v.shape[-1]
    if not 1 <= nh <= PRODUCT_MAX_NH:
        raise ValueError("1..%d substeps per token" % PRODUCT_MAX_NH)
    _check(q, "q", (B, H, T, dk))
    _check(k, "k", (B, H, T, nh, dk), q.dtype)
    _check(v, "v", (B, H, T, nh, dv), q.dtype)
    if gate == "scalar":
        _check(g, "g", (B, H, T), torch.float32)
    elif gate == "channel":
        _check(g, "g", (B, H, T, dk), torch.float32)
    _check(beta, "beta", (B, H, T, nh), torch.float32)
    _check(S0, "S0", (B, H, dv, dk), torch.float32)
    if out_dtype is None:
        out_dtype = o.dtype if o is not None else torch.float32
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=out_dtype, device=q.device)
    _check(o, "o", (B, H, T, dv), out_dtype)
    if S_T is None and return_state:
        S_T = torch.empty((B, H, dv, dk), dtype=torch.float32, device=q.device)
    _check(S_T, "S_T", (B, H, dv, dk), torch.float32)
    d = make_desc(B, H, T, dk, dv, "delta", gate, _dtype_code(q.dtype), _dtype_code(out_dtype), algo,
                  prologue=prologue)
    with _on_device(q):
        rc = load().gdn_product_fwd(ctypes.byref(d), ctypes.c_int(nh), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                    _ptr(beta), _ptr(S0), _ptr(o), _ptr(S_T), _stream(stream, q))
    if rc != GDN_OK:
        raise GDNError(rc, "gdn_product_fwd")
    return o, S_T


def chunk_fwd_segmented(q, k, v, g=None, beta=None, S0=None, *, update, gate, nseg, out_dtype=None, o=None,
                        S_T=None, return_state=True, algo="auto", prologue=0, workspace=None, stream=None):
    """gdn_chunk_fwd_segmented: the prefill with each sequence cut into ``nseg``
    segments that run in parallel.  Same tensors as chunk_fwd; ``workspace`` is a
    CUDA uint8 tensor of at least segmented_workspace_bytes(...) bytes (allocated
    here through PyTorch when None).  Returns (o, S_T)."""
    import torch

    B, H, T, dk = q.shape
    dv = v.shape[-1]
    _check(q, "q", (B, H, T, dk))
    _check(k, "k", (B, H, T, dk), q.dtype)
    _check(v, "v", (B, H, T, dv), q.dtype)
    if gate == "scalar":
        _check(g, "g", (B, H, T), torch.float32)
    elif gate == "channel":
        _check(g, "g", (B, H, T, dk), torch.float32)
    _check(beta, "beta", (B, H, T), torch.float32)
    _check(S0, "S0", (B, H, dv, dk), torch.float32)
    if out_dtype is None:
        out_dtype = o.dtype if o is not None else torch.float32
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=out_dtype, device=q.device)
    _check(o, "o", (B, H, T, dv), out_dtype)
    if S_T is None and return_state:
        S_T = torch.empty((B, H, dv, dk), dtype=torch.float32, device=q.device)
    _check(S_T, "S_T", (B, H, dv, dk), torch.float32)
    d = make_desc(B, H, T, dk, dv, update, gate, _dtype_code(q.dtype), _dtype_code(out_dtype), algo,
                  prologue=prologue)
    need = load().gdn_segmented_workspace_bytes(ctypes.byref(d), int(nseg))
    if workspace is None:
        workspace = torch.empty(max(int(need), 16), dtype=torch.uint8, device=q.device)
    if not workspace.is_cuda or not workspace.is_contiguous() or workspace.numel() * workspace.element_size() < need:
        raise ValueError("workspace needs %d contiguous CUDA bytes" % need)
    with _on_device(q):
        rc = load().gdn_chunk_fwd_segmented(ctypes.byref(d), int(nseg), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                            _ptr(beta), _ptr(S0), _ptr(o), _ptr(S_T), _ptr(workspace),
                                            ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                                            _stream(stream, q))
    if rc != GDN_OK:
        raise GDNError(rc, "gdn_chunk_fwd_segmented")
    return o, S_T


def chunk_fwd_segmented_noalloc(q, k, v, g=None, beta=None, S0=None, *, update, gate, nseg, out_dtype=None,
                                o=None, S_T=None, return_state=True, algo="auto", prologue=0, stream=None):
    """gdn_chunk_fwd_segmented_noalloc: chunk_fwd_segmented with its scratch
    in the library's fixed device array (noalloc_scratch_bytes()); nothing is
    allocated when o (and S_T, or return_state=False) are given.  Returns (o, S_T)."""
    import torch

    B, H, T, dk = q.shape
    dv = v.shape[-1]
    _check(q, "q", (B, H, T, dk))
    _check(k, "k", (B, H, T, dk), q.dtype)
    _check(v, "v", (B, H, T, dv), q.dtype)
    if gate == "scalar":
        _check(g, "g", (B, H, T), torch.float32)
    elif gate == "channel":
        _check(g, "g", (B, H, T, dk), torch.float32)
    _check(beta, "beta", (B, H, T), torch.float32)
    _check(S0, "S0", (B, H, dv, dk), torch.float32)
    if out_dtype is None:
        out_dtype = o.dtype if o is not None else torch.float32
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=out_dtype, device=q.device)
    _check(o, "o", (B, H, T, dv), out_dtype)
    if S_T is None and return_state:
        S_T = torch.empty((B, H, dv, dk), dtype=torch.float32, device=q.device)
    _check(S_T, "S_T", (B, H, dv, dk), torch.float32)
    d = make_desc(B, H, T, dk, dv, update, gate, _dtype_code(q.dtype), _dtype_code(out_dtype), algo,
                  prologue=prologue)
    with _on_device(q):
        rc = load().gdn_chunk_fwd_segmented_noalloc(ctypes.byref(d), int(nseg), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                                    _ptr(beta), _ptr(S0), _ptr(o), _ptr(S_T), _stream(stream, q))
    if rc != GDN_OK:
        raise GDNError(rc, "gdn_chunk_fwd_segmented_noalloc")
    return o, S_T


def noalloc_scratch_bytes() -> int:
    return int(load().gdn_noalloc_scratch_bytes())


def segmented_workspace_bytes(B, H, T, dk, dv, nseg) -> int:
    d = make_desc(B, H, T, dk, dv, "delta", "scalar", BF16, F32)
    return int(load().gdn_segmented_workspace_bytes(ctypes.byref(d), int(nseg)))


def segment_maps(q, k, v, g=None, beta=None, *, update, gate, H=None, Lam=None, algo="auto", prologue=0,
                 stream=None):
    """gdn_segment_maps: the affine map S_in -> S_in Lam + H of the T tokens of
    every head.  Same inputs as chunk_fwd; returns (H [B,H,dv,dk],
    Lam [B,H,dk,dk]), both fp32."""
    import torch

    B, Hh, T, dk = q.shape
    dv = v.shape[-1]
    _check(q, "q", (B, Hh, T, dk))
    _check(k, "k", (B, Hh, T, dk), q.dtype)
    _check(v, "v", (B, Hh, T, dv), q.dtype)
    if gate == "scalar":
        _check(g, "g", (B, Hh, T), torch.float32)
    elif gate == "channel":
        _check(g, "g", (B, Hh, T, dk), torch.float32)
    _check(beta, "beta", (B, Hh, T), torch.float32)
    if H is None:
        H = torch.empty((B, Hh, dv, dk), dtype=torch.float32, device=q.device)
    if Lam is None:
        Lam = torch.empty((B, Hh, dk, dk), dtype=torch.float32, device=q.device)
    _check(H, "H", (B, Hh, dv, dk), torch.float32)
    _check(Lam, "Lam", (B, Hh, dk, dk), torch.float32)
    d = make_desc(B, Hh, T, dk, dv, update, gate, _dtype_code(q.dtype), F32, algo, prologue=prologue)
    with _on_device(q):
        rc = load().gdn_segment_maps(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(H),
                                     _ptr(Lam), _stream(stream, q))
    if rc != GDN_OK:
        raise GDNError(rc, "gdn_segment_maps")
    return H, Lam


def compose_segments(H, Lam=None, S0=None, *, S_in=None, S_T=None, want_inputs=True, stream=None):
    """gdn_compose_segments: H [nseg,B,H,dv,dk], Lam [nseg,B,H,dk,dk] or None
    (identity transitions), S0 [B,H,dv,dk] or None.  Returns (S_in
    [nseg,B,H,dv,dk], the state entering each segment, or None when
    ``want_inputs`` is false; S_T [B,H,dv,dk], the final state)."""
    import torch

    nseg, B, Hh, dv, dk = H.shape
    _check(H, "H", (nseg, B, Hh, dv, dk), torch.float32)
    _check(Lam, "Lam", (nseg, B, Hh, dk, dk), torch.float32)
    _check(S0, "S0", (B, Hh, dv, dk), torch.float32)
    if S_in is None and want_inputs:
        S_in = torch.empty_like(H)
    _check(S_in, "S_in", (nseg, B, Hh, dv, dk), torch.float32)
    if S_T is None:
        S_T = torch.empty((B, Hh, dv, dk), dtype=torch.float32, device=H.device)
    _check(S_T, "S_T", (B, Hh, dv, dk), torch.float32)
    with _on_device(H):
        rc = load().gdn_compose_segments(B * Hh, nseg, dk, dv, _ptr(S0), _ptr(H), _ptr(Lam), _ptr(S_in), _ptr(S_T),
                                         _stream(stream, H))
    if rc != GDN_OK:
        raise GDNError(rc, "gdn_compose_segments")
    return S_in, S_T


def decode_step(q, k, v, g, beta, S, *, update, gate, out_dtype=None, o=None, prologue=0, stream=None):
    """T decode steps (gdn_decode_step, 1 <= T <= DECODE_MAX_T, usually 1); S
    [B,H,dv,dk] is updated in place and read / written once for the T tokens.

    q, k [B,H,T,dk]; v [B,H,T,dv]; g [B,H,T] or [B,H,T,dk] or None; beta [B,H,T].
    Returns o [B,H,T,dv].
    """
    import torch

    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if not 1 <= T <= DECODE_MAX_T:
        raise ValueError("decode_step takes 1..%d tokens (gdn_chunk_fwd for longer runs)" % DECODE_MAX_T)
    _check(q, "q", (B, H, T, dk))
    _check(k, "k", (B, H, T, dk), q.dtype)
    _check(v, "v", (B, H, T, dv), q.dtype)
    if gate == "scalar":
        _check(g, "g", (B, H, T), torch.float32)
    elif gate == "channel":
        _check(g, "g", (B, H, T, dk), torch.float32)
    _check(beta, "beta", (B, H, T), torch.float32)
    _check(S, "S", (B, H, dv, dk), torch.float32)
    if out_dtype is None:
        out_dtype = o.dtype if o is not None else torch.float32
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=out_dtype, device=q.device)
    _check(o, "o", (B, H, T, dv), out_dtype)
    d = make_desc(B, H, T, dk, dv, update, gate, _dtype_code(q.dtype), _dtype_code(out_dtype), prologue=prologue)
    with _on_device(q):
        rc = load().gdn_decode_step(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S),
                                    _ptr(o), _stream(stream, q))
    if rc != GDN_OK:
        raise GDNError(rc, "gdn_decode_step")
    return o


def bwd_workspace_bytes(B, H, T, dk, dv, update="delta", gate="scalar", prologue=0, algo="auto") -> int:
    d = make_desc(B, H, T, dk, dv, update, gate, BF16, F32, algo, prologue=prologue)
    return int(load().gdn_bwd_workspace_bytes(ctypes.byref(d)))


def bwd_tc_workspace_bytes(B, H, T, dk, dv, update="delta", gate="scalar") -> int:
    """Workspace of gdn_chunk_bwd_tc (0 for a request it does not serve)."""
    d = make_desc(B, H, T, dk, dv, update, gate, BF16, F32)
    return int(load().gdn_bwd_tc_workspace_bytes(ctypes.byref(d)))


def chunk_bwd(q, k, v, g=None, beta=None, S0=None, dO=None, dS_T=None, *, update, gate, workspace=None,
              want_dS0=True, states=None, prologue=0, algo="token", stream=None):
    """gdn_chunk_bwd: gradients of chunk_fwd for upstream gradients dO [B,H,T,dv]
    and dS_T [B,H,dv,dk] (fp32; None = 0).  Returns (dq, dk, dv, dg, dbeta, dS0),
    fp32, dg / dbeta None when the mode has no gate / write strength, dS0 None
    when ``want_dS0`` is false.  ``workspace``: a CUDA uint8 tensor of
    bwd_workspace_bytes(...) bytes (allocated here when None).  With ``states``
    (written by chunk_fwd(states=...)) the call is gdn_chunk_bwd_states: S0 and
    the workspace are not used.  ``prologue``: the GDN_PRO_* maps the forward
    applied to the raw q, k, beta, g; the gradients are then with respect to
    those raw inputs.  ``algo="tc"``: the chunkwise tensor-core backward, from
    ``states`` (gdn_chunk_bwd_tc; ``workspace`` of bwd_tc_workspace_bytes(...)
    bytes) or, without them, gdn_chunk_bwd with GDN_ALGO_TC (the tensor-core
    forward writes the states into the workspace first; bwd_workspace_bytes(...,
    algo="tc") bytes)."""
    import torch

    B, H, T, dk = q.shape
    dv = v.shape[-1]
    _check(q, "q", (B, H, T, dk))
    _check(k, "k", (B, H, T, dk), q.dtype)
    _check(v, "v", (B, H, T, dv), q.dtype)
    if gate == "scalar":
        _check(g, "g", (B, H, T), torch.float32)
    elif gate == "channel":
        _check(g, "g", (B, H, T, dk), torch.float32)
    _check(beta, "beta", (B, H, T), torch.float32)
    _check(S0, "S0", (B, H, dv, dk), torch.float32)
    _check(dO, "dO", (B, H, T, dv), torch.float32)
    _check(dS_T, "dS_T", (B, H, dv, dk), torch.float32)
    f32 = dict(dtype=torch.float32, device=q.device)
    gq, gk, gv = torch.empty((B, H, T, dk), **f32), torch.empty((B, H, T, dk), **f32), torch.empty((B, H, T, dv), **f32)
    gg = None if gate == "none" else torch.empty(tuple(g.shape), **f32)
    gb = torch.empty((B, H, T), **f32) if update == "delta" else None
    gS0 = torch.empty((B, H, dv, dk), **f32) if want_dS0 else None
    d = make_desc(B, H, T, dk, dv, update, gate, _dtype_code(q.dtype), F32, prologue=prologue)
    if algo == "tc" and states is None:
        d = make_desc(B, H, T, dk, dv, update, gate, _dtype_code(q.dtype), F32, "tc", prologue=prologue)
        need = int(load().gdn_bwd_workspace_bytes(ctypes.byref(d)))
        if workspace is None:
            workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
        if not workspace.is_cuda or not workspace.is_contiguous() or workspace.numel() < need:
            raise ValueError("workspace needs %d contiguous CUDA bytes" % need)
        with _on_device(q):
            rc = load().gdn_chunk_bwd(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                                      _ptr(dO), _ptr(dS_T), _ptr(gq), _ptr(gk), _ptr(gv), _ptr(gg), _ptr(gb),
                                      _ptr(gS0), _ptr(workspace), ctypes.c_size_t(workspace.numel()),
                                      _stream(stream, q))
        if rc != GDN_OK:
            raise GDNError(rc, "gdn_chunk_bwd")
        return gq, gk, gv, gg, gb, gS0
    if algo == "tc":
        _check(states, "states", (B, H, (T + CHUNK - 1) // CHUNK, dv, dk), torch.float32)
        need = int(load().gdn_bwd_tc_workspace_bytes(ctypes.byref(d)))
        if workspace is None:
            workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
        if not workspace.is_cuda or not workspace.is_contiguous() or workspace.numel() < need:
            raise ValueError("workspace needs %d contiguous CUDA bytes" % need)
        with _on_device(q):
            rc = load().gdn_chunk_bwd_tc(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                         _ptr(states), _ptr(dO), _ptr(dS_T), _ptr(gq), _ptr(gk), _ptr(gv), _ptr(gg),
                                         _ptr(gb), _ptr(gS0), _ptr(workspace), ctypes.c_size_t(workspace.numel()),
                                         _stream(stream, q))
        if rc != GDN_OK:
            raise GDNError(rc, "gdn_chunk_bwd_tc")
        return gq, gk, gv, gg, gb, gS0
    if algo != "token":
        raise ValueError("algo is 'token' or 'tc'")
    if states is not None:
        _check(states, "states", (B, H, (T + CHUNK - 1) // CHUNK, dv, dk), torch.float32)
        with _on_device(q):
            rc = load().gdn_chunk_bwd_states(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                             _ptr(states), _ptr(dO), _ptr(dS_T), _ptr(gq), _ptr(gk), _ptr(gv),
                                             _ptr(gg), _ptr(gb), _ptr(gS0), _stream(stream, q))
        if rc != GDN_OK:
            raise GDNError(rc, "gdn_chunk_bwd_states")
        return gq, gk, gv, gg, gb, gS0
    need = int(load().gdn_bwd_workspace_bytes(ctypes.byref(d)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if not workspace.is_cuda or not workspace.is_contiguous() or workspace.numel() < need:
        raise ValueError("workspace needs %d contiguous CUDA bytes" % need)
    with _on_device(q):
        rc = load().gdn_chunk_bwd(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                                  _ptr(dO), _ptr(dS_T), _ptr(gq), _ptr(gk), _ptr(gv), _ptr(gg), _ptr(gb), _ptr(gS0),
                                  _ptr(workspace), ctypes.c_size_t(workspace.numel()), _stream(stream, q))
    if rc != GDN_OK:
        raise GDNError(rc, "gdn_chunk_bwd")
    return gq, gk, gv, gg, gb, gS0
