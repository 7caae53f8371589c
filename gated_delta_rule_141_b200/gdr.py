"""Thin ctypes binding of libgdr.so (C ABI in include/gdr.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libgdr.so.  PyTorch supplies device memory and streams.  There is
no fallback: if the library is missing or the request is rejected, the call
raises.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libgdr.so")

# gdr_status
OK, ERR_ARG, ERR_SHAPE, ERR_DTYPE, ERR_ALIGN, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, \
    ERR_NONFINITE, ERR_WORKSPACE, ERR_SCRATCH_LIMIT = range(11)

# size of the fixed device array gdr_chunk_fwd_static uses as its workspace
STATIC_SCRATCH_BYTES = 64 * 1024 * 1024
# gdr_dtype
F32, BF16 = 0, 1
# gdr_gate_mode
GATE_SCALAR, GATE_GROUP64, GATE_CHANNEL = 0, 1, 2
# gdr_inverse_mode
INV_EXACT, INV_NEUMANN, INV_NEUMANN1 = 0, 1, 2
# gdr_kernel
KERNEL_AUTO, KERNEL_SIMT, KERNEL_TC, KERNEL_TC2, KERNEL_SIMT2, KERNEL_TC2W = 0, 1, 2, 3, 4, 5

_KERNELS = {"auto": KERNEL_AUTO, "simt": KERNEL_SIMT, "tc": KERNEL_TC, "tc2": KERNEL_TC2,
            "simt2": KERNEL_SIMT2, "tc2w": KERNEL_TC2W}
KERNEL_NAMES = {KERNEL_SIMT: "simt", KERNEL_TC: "tc", KERNEL_TC2: "tc2", KERNEL_SIMT2: "simt2",
                KERNEL_TC2W: "tc2w"}

# bytes of one chunk record written by gdr_chunk_prepare (T then L, 64 x 64 bf16 each)
PREP_CHUNK_BYTES = 16384
# bytes of one workspace record of the two-pass kernel: scalar gate, grouped / per-channel gates
TC2_SCALAR_RECORD_BYTES = 33296
TC2_EXT_RECORD_BYTES = 66048
_INVERSES = {"exact": INV_EXACT, "neumann": INV_NEUMANN, "neumann1": INV_NEUMANN1}

# Every symbol include/gdr.h declares.
EXPORTS = ("gdr_chunk_fwd", "gdr_chunk_fwd_momentum", "gdr_chunk_bwd", "gdr_bwd_workspace_bytes",
           "gdr_workspace_bytes", "gdr_chunk_prepare", "gdr_chunk_fwd_host",
           "gdr_chunk_fwd_static",
           "gdr_output_gate_rmsnorm",
           "gdr_select_kernel", "gdr_kernel_chunk", "gdr_state_segments", "gdr_device_status",
           "gdr_selftest_bounded_wait",
           "gdr_status_string",
           "gdr_version")


class GdrShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("Hk", ctypes.c_int),
                ("Hv", ctypes.c_int), ("dk", ctypes.c_int), ("dv", ctypes.c_int),
                ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
                ("neumann_order", ctypes.c_int), ("neumann_residual_steps", ctypes.c_int),
                ("kernel", ctypes.c_int)]


class GdrIO(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("g", ctypes.c_void_p), ("beta", ctypes.c_void_p), ("S0", ctypes.c_void_p),
                ("o", ctypes.c_void_p), ("S_final", ctypes.c_void_p)]


class GdrError(RuntimeError):
    def __init__(self, status: int, what: str = "gdr_chunk_fwd"):
        self.status = status
        super().__init__("%s: %s (status %d)" % (what, status_string(status), status))


_lib = None


def load(path: str = LIB_PATH):
    """Load libgdr.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError("libgdr.so not found at %s; build it with "
                           "`python -m gated_delta_rule_141_b200.build`" % path)
    lib = ctypes.CDLL(path)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.gdr_chunk_fwd.argtypes = [ctypes.POINTER(GdrShape), vp, vp, vp, vp, vp, vp, i, i, i,
                                  vp, vp, vp, sz, vp]
    lib.gdr_chunk_fwd.restype = i
    lib.gdr_chunk_fwd_momentum.argtypes = [ctypes.POINTER(GdrShape), vp, vp, vp, vp, vp, vp, i, i,
                                           i, ctypes.c_float, vp, vp, vp, vp, sz, vp]
    lib.gdr_chunk_fwd_momentum.restype = i
    lib.gdr_chunk_bwd.argtypes = [ctypes.POINTER(GdrShape)] + [vp] * 8 + [i, i] + [vp] * 7 + [sz, vp]
    lib.gdr_chunk_bwd.restype = i
    lib.gdr_bwd_workspace_bytes.argtypes = [ctypes.POINTER(GdrShape), i, i, ctypes.POINTER(sz)]
    lib.gdr_bwd_workspace_bytes.restype = i
    lib.gdr_chunk_fwd_static.argtypes = [ctypes.POINTER(GdrShape), vp, vp, vp, vp, vp, vp, i, i,
                                         i, vp, vp, vp]
    lib.gdr_chunk_fwd_static.restype = i
    lib.gdr_workspace_bytes.argtypes = [ctypes.POINTER(GdrShape), i, i, i, ctypes.POINTER(sz)]
    lib.gdr_workspace_bytes.restype = i
    lib.gdr_chunk_prepare.argtypes = [ctypes.POINTER(GdrShape), vp, vp, vp, vp, i, i, i, vp, sz,
                                      vp]
    lib.gdr_chunk_prepare.restype = i
    lib.gdr_chunk_fwd_host.argtypes = [ctypes.POINTER(GdrShape), ctypes.POINTER(GdrIO),
                                       ctypes.POINTER(GdrIO), i, i, i, vp, sz, vp]
    lib.gdr_chunk_fwd_host.restype = i
    lib.gdr_select_kernel.argtypes = [ctypes.POINTER(GdrShape), i, i, i]
    lib.gdr_select_kernel.restype = i
    lib.gdr_kernel_chunk.argtypes = [ctypes.POINTER(GdrShape), i, i, i]
    lib.gdr_kernel_chunk.restype = i
    lib.gdr_state_segments.argtypes = [ctypes.POINTER(GdrShape), i, i, i]
    lib.gdr_state_segments.restype = i
    lib.gdr_output_gate_rmsnorm.argtypes = [ctypes.POINTER(GdrShape), vp, vp, vp, ctypes.c_float, vp]
    lib.gdr_output_gate_rmsnorm.restype = i
    lib.gdr_device_status.argtypes = [vp]
    lib.gdr_device_status.restype = i
    lib.gdr_selftest_bounded_wait.argtypes = [ctypes.c_uint64, vp]
    lib.gdr_selftest_bounded_wait.restype = i
    lib.gdr_status_string.argtypes = [i]
    lib.gdr_status_string.restype = ctypes.c_char_p
    lib.gdr_version.argtypes = []
    lib.gdr_version.restype = i
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().gdr_status_string(int(status)).decode()


def version() -> int:
    return int(load().gdr_version())


def make_shape(B, T, Hk, Hv, dk, dv, in_dtype=BF16, out_dtype=BF16, neumann_order=4,
               neumann_residual_steps=1, kernel="auto") -> GdrShape:
    return GdrShape(int(B), int(T), int(Hk), int(Hv), int(dk), int(dv), int(in_dtype),
                    int(out_dtype), int(neumann_order), int(neumann_residual_steps),
                    _KERNELS[kernel] if isinstance(kernel, str) else int(kernel))


def gate_mode_for(G: int, dk: int) -> int:
    if G == 1:
        return GATE_SCALAR
    if G == dk:
        return GATE_CHANNEL
    if dk % 64 == 0 and G == dk // 64:
        return GATE_GROUP64
    raise ValueError("no gate mode has G=%d for dk=%d" % (G, dk))


def select_kernel(shape: GdrShape, chunk: int, gate_mode: int, inverse: str = "exact") -> int:
    return int(load().gdr_select_kernel(ctypes.byref(shape), int(chunk), int(gate_mode),
                                        _INVERSES[inverse]))


def kernel_chunk(shape: GdrShape, chunk: int, gate_mode: int, inverse: str = "exact") -> int:
    """Chunk length the selected kernel blocks by (negative status if rejected)."""
    return int(load().gdr_kernel_chunk(ctypes.byref(shape), int(chunk), int(gate_mode),
                                       _INVERSES[inverse]))


def state_segments(shape: GdrShape, chunk: int, gate_mode: int, inverse: str = "exact") -> int:
    """Segments per sequence of the two-pass path's state pass (1: sequential,
    n > 1: segment-parallel, 0: another kernel; negative status if rejected)."""
    return int(load().gdr_state_segments(ctypes.byref(shape), int(chunk), int(gate_mode),
                                         _INVERSES[inverse]))


def workspace_bytes(shape: GdrShape, chunk: int, gate_mode: int, inverse: str = "exact") -> int:
    """Device workspace gdr_chunk_fwd needs for this request (raises if rejected)."""
    n = ctypes.c_size_t(0)
    st = load().gdr_workspace_bytes(ctypes.byref(shape), int(chunk), int(gate_mode),
                                    _INVERSES[inverse], ctypes.byref(n))
    if st != OK:
        raise GdrError(st, "gdr_workspace_bytes")
    return int(n.value)


def device_status(stream=None) -> int:
    return int(load().gdr_device_status(_stream_handle(stream)))


def selftest_bounded_wait(limit_ns: int, stream=None) -> int:
    """Launch the library's bounded-wait self-test (a wait nothing ends, given up
    after limit_ns); its status shows in device_status()."""
    return int(load().gdr_selftest_bounded_wait(int(limit_ns), _stream_handle(stream)))


def _stream_handle(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(int(getattr(stream, "cuda_stream", stream)))


def _dtype_code(t):
    import torch
    if t == torch.bfloat16:
        return BF16
    if t == torch.float32:
        return F32
    raise TypeError("unsupported dtype %s (bf16 or fp32)" % t)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def chunk_fwd(q, k, v, g, beta, S0=None, chunk=64, gate_mode=None, inverse="exact",
              neumann_order=4, neumann_residual_steps=1, out_dtype=None, o=None,
              S_final=None, want_state=True, kernel="auto", workspace=None, stream=None):
    """Chunkwise gated delta-rule forward on the current CUDA device.

    q, k [B,Hk,T,dk] and v [B,Hv,T,dv] (bf16 or fp32, same dtype); g [B,Hk,T,G] and
    beta [B,Hk,T] fp32; S0 [B,Hv,dk,dv] fp32 or None.  Returns (o, S_final);
    S_final is None when want_state is False.  Outputs and the workspace the selected
    kernel needs are allocated with torch unless passed in.  Runs asynchronously on
    `stream` (default: torch's current).
    """
    import torch
    B, Hk, T, dk = q.shape
    Hv, dv = v.shape[1], v.shape[3]
    G = g.shape[-1]
    if gate_mode is None:
        gate_mode = gate_mode_for(G, dk)
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta), ("S0", S0)):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("%s must be a contiguous CUDA tensor" % name)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    out_dtype = q.dtype if out_dtype is None else out_dtype
    if o is None:
        o = torch.empty((B, Hv, T, dv), dtype=out_dtype, device=q.device)
    if S_final is None and want_state:
        S_final = torch.empty((B, Hv, dk, dv), dtype=torch.float32, device=q.device)
    shape = make_shape(B, T, Hk, Hv, dk, dv, _dtype_code(q.dtype), _dtype_code(o.dtype),
                       neumann_order, neumann_residual_steps, kernel)
    if workspace is None:
        nbytes = workspace_bytes(shape, chunk, gate_mode, inverse)
        workspace = (torch.empty(nbytes, dtype=torch.uint8, device=q.device) if nbytes else None)
    st = load().gdr_chunk_fwd(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                              _ptr(beta), _ptr(S0), int(chunk), int(gate_mode),
                              _INVERSES[inverse], _ptr(o), _ptr(S_final), _ptr(workspace),
                              0 if workspace is None else workspace.numel(),
                              _stream_handle(stream))
    if st != OK:
        raise GdrError(st)
    return o, S_final


def chunk_fwd_momentum(q, k, v, g, beta, S0=None, mu=0.0, kappa=None, chunk=64, gate_mode=None,
                       inverse="exact", neumann_order=4, neumann_residual_steps=1,
                       out_dtype=None, o=None, S_final=None, want_state=True, kernel="auto",
                       workspace=None, stream=None):
    """chunk_fwd with chunk-boundary momentum: each chunk's state update is blended
    with a velocity Z (zero at the start), Z <- mu kappa_c Z + (S~_c - F_c S), S <-
    F_c S + Z.  kappa: int32 [B, ceil(T / chunk)] CUDA tensor of per-chunk gates on
    the carried velocity, or None for ones.  Other arguments as chunk_fwd; the
    workspace (allocated here unless passed in) lets the two-pass tensor-core path
    run it."""
    import torch
    B, Hk, T, dk = q.shape
    Hv, dv = v.shape[1], v.shape[3]
    G = g.shape[-1]
    if gate_mode is None:
        gate_mode = gate_mode_for(G, dk)
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta), ("S0", S0),
                    ("kappa", kappa)):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("%s must be a contiguous CUDA tensor" % name)
    if kappa is not None and (kappa.dtype != torch.int32 or
                              tuple(kappa.shape) != (B, (T + int(chunk) - 1) // int(chunk))):
        raise ValueError("kappa must be an int32 [B, ceil(T / chunk)] tensor")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    out_dtype = q.dtype if out_dtype is None else out_dtype
    if o is None:
        o = torch.empty((B, Hv, T, dv), dtype=out_dtype, device=q.device)
    if S_final is None and want_state:
        S_final = torch.empty((B, Hv, dk, dv), dtype=torch.float32, device=q.device)
    shape = make_shape(B, T, Hk, Hv, dk, dv, _dtype_code(q.dtype), _dtype_code(o.dtype),
                       neumann_order, neumann_residual_steps, kernel)
    if workspace is None and kernel != "simt":
        try:
            nbytes = workspace_bytes(shape, chunk, gate_mode, inverse)
        except GdrError:
            nbytes = 0
        workspace = (torch.empty(nbytes, dtype=torch.uint8, device=q.device) if nbytes else None)
    st = load().gdr_chunk_fwd_momentum(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                       _ptr(beta), _ptr(S0), int(chunk), int(gate_mode),
                                       _INVERSES[inverse], float(mu), _ptr(kappa), _ptr(o),
                                       _ptr(S_final), _ptr(workspace),
                                       0 if workspace is None else workspace.numel(),
                                       _stream_handle(stream))
    if st != OK:
        raise GdrError(st, "gdr_chunk_fwd_momentum")
    return o, S_final


def bwd_workspace_bytes(shape: GdrShape, chunk: int, gate_mode: int) -> int:
    """Workspace bytes gdr_chunk_bwd needs (the fp32 state at every chunk start)."""
    out = ctypes.c_size_t(0)
    st = load().gdr_bwd_workspace_bytes(ctypes.byref(shape), int(chunk), int(gate_mode),
                                        ctypes.byref(out))
    if st != OK:
        raise GdrError(st, "gdr_bwd_workspace_bytes")
    return out.value


def chunk_bwd(q, k, v, g, beta, S0, dO, dS_final=None, chunk=64, gate_mode=None, kernel="auto",
              workspace=None, want_dS0=True, stream=None):
    """Gradients of sum(dO * o) + sum(dS_final * S_final) of the chunkwise forward
    (exact inverse) with respect to q, k, v, g, beta and S0.  Inputs as chunk_fwd;
    dO [B,Hv,T,dv] and dS_final [B,Hv,dk,dv] (or None) fp32 CUDA tensors.  Returns a
    dict of fp32 tensors with keys q, k, v, g, beta, S0 (None unless want_dS0)."""
    import torch
    B, Hk, T, dk = q.shape
    Hv, dv = v.shape[1], v.shape[3]
    G = g.shape[-1]
    if gate_mode is None:
        gate_mode = gate_mode_for(G, dk)
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta), ("S0", S0),
                    ("dO", dO), ("dS_final", dS_final)):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("%s must be a contiguous CUDA tensor" % name)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    if dO.dtype != torch.float32 or tuple(dO.shape) != (B, Hv, T, dv):
        raise ValueError("dO must be an fp32 [B, Hv, T, dv] tensor")
    if dS_final is not None and (dS_final.dtype != torch.float32 or
                                 tuple(dS_final.shape) != (B, Hv, dk, dv)):
        raise ValueError("dS_final must be an fp32 [B, Hv, dk, dv] tensor")
    f32 = dict(dtype=torch.float32, device=q.device)
    grads = {"q": torch.empty((B, Hk, T, dk), **f32), "k": torch.empty((B, Hk, T, dk), **f32),
             "v": torch.empty((B, Hv, T, dv), **f32), "g": torch.empty((B, Hk, T, G), **f32),
             "beta": torch.empty((B, Hk, T), **f32),
             "S0": torch.empty((B, Hv, dk, dv), **f32) if want_dS0 else None}
    shape = make_shape(B, T, Hk, Hv, dk, dv, _dtype_code(q.dtype), F32, kernel=kernel)
    if workspace is None:
        nbytes = bwd_workspace_bytes(shape, chunk, gate_mode)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device) if nbytes else None
    st = load().gdr_chunk_bwd(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                              _ptr(S0), _ptr(dO), _ptr(dS_final), int(chunk), int(gate_mode),
                              _ptr(grads["q"]), _ptr(grads["k"]), _ptr(grads["v"]),
                              _ptr(grads["g"]), _ptr(grads["beta"]), _ptr(grads["S0"]),
                              _ptr(workspace), 0 if workspace is None else workspace.numel(),
                              _stream_handle(stream))
    if st != OK:
        raise GdrError(st, "gdr_chunk_bwd")
    return grads


def output_gate_rmsnorm(o, z, weight=None, eps=1e-6, stream=None):
    """In place: o <- sigmoid(z) * RMSNorm(o) * weight over the last axis of o
    [B, Hv, T, dv] (the readout epilogue); z like o, weight [dv] fp32 or None."""
    B, Hv, T, dv = o.shape
    if tuple(z.shape) != tuple(o.shape) or z.dtype != o.dtype:
        raise ValueError("z must match o in shape and dtype")
    if not (o.is_contiguous() and z.is_contiguous()):
        raise ValueError("o and z must be contiguous")
    if weight is not None and (tuple(weight.shape) != (dv,) or not weight.is_contiguous()):
        raise ValueError("weight must be a contiguous [dv] fp32 tensor")
    shape = make_shape(B, T, 1, Hv, 1, dv, out_dtype=_dtype_code(o.dtype))
    st = load().gdr_output_gate_rmsnorm(ctypes.byref(shape), _ptr(o), _ptr(z), _ptr(weight),
                                        float(eps), _stream_handle(stream))
    if st != OK:
        raise GdrError(st, "gdr_output_gate_rmsnorm")
    return o


def chunk_prepare(q, k, g, beta, chunk=64, gate_mode=None, inverse="exact", neumann_order=4,
                  neumann_residual_steps=1, factors=None, stream=None):
    """gdr_chunk_prepare: the chunk factors T = diag(beta) (I + M)^{-1} and L of every
    chunk.  Returns a uint8 device tensor [B, Hk, ceil(T/64), 16384] of tile images
    (see include/gdr.h for the byte layout)."""
    import torch
    B, Hk, T, dk = q.shape
    if gate_mode is None:
        gate_mode = gate_mode_for(g.shape[-1], dk)
    nch = (T + 63) // 64
    if factors is None:
        factors = torch.empty((B, Hk, nch, PREP_CHUNK_BYTES), dtype=torch.uint8, device=q.device)
    shape = make_shape(B, T, Hk, Hk, dk, dk, _dtype_code(q.dtype), BF16, neumann_order,
                       neumann_residual_steps)
    st = load().gdr_chunk_prepare(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(g), _ptr(beta),
                                  int(chunk), int(gate_mode), _INVERSES[inverse], _ptr(factors),
                                  factors.numel(), _stream_handle(stream))
    if st != OK:
        raise GdrError(st, "gdr_chunk_prepare")
    return factors


def chunk_fwd_host(host: dict, dev: dict, shape: GdrShape, chunk: int, gate_mode: int,
                   inverse: str = "exact", workspace=None, stream=None):
    """gdr_chunk_fwd_host: inputs/outputs in (pinned) host tensors, device buffers
    supplied by the caller.  Both dicts map q, k, v, g, beta, S0, o, S_final to
    tensors (S0 / S_final may be None)."""
    names = ("q", "k", "v", "g", "beta", "S0", "o", "S_final")
    h = GdrIO(*[_ptr(host.get(n)) for n in names])
    d = GdrIO(*[_ptr(dev.get(n)) for n in names])
    st = load().gdr_chunk_fwd_host(ctypes.byref(shape), ctypes.byref(h), ctypes.byref(d),
                                   int(chunk), int(gate_mode), _INVERSES[inverse],
                                   _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                   _stream_handle(stream))
    if st != OK:
        raise GdrError(st, "gdr_chunk_fwd_host")
