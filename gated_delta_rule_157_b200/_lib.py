"""ctypes binding of libkda_b200.so (the C ABI in include/kda.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, outputs are allocated with torch when the caller passes none, and
raw device pointers plus the current CUDA stream are handed to the library.
Every step of the computation runs in the library's CUDA kernels; there is no
CPU path.  If the shared object is missing it is built with nvcc; if that
fails, the import fails.
"""
import ctypes
import os

import torch

from . import build as _build

KDA_OK = 0
STATUS_NAMES = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED",
                3: "KDA_ERR_ALIGNMENT", 4: "KDA_ERR_ALIAS", 5: "KDA_ERR_CUDA",
                6: "KDA_ERR_TIMEOUT", 7: "KDA_ERR_RANGE"}
DT_F32, DT_BF16 = 0, 1
ALGOS = {"auto": 0, "simt": 1, "tc": 2}


class KdaError(RuntimeError):
    """A non-OK kda_status returned by the library."""

    def __init__(self, fn, status):
        self.status = int(status)
        super().__init__("%s returned %s" % (fn, STATUS_NAMES.get(self.status, self.status)))


class ChunkArgs(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int), ("HV", ctypes.c_int),
        ("Dk", ctypes.c_int), ("Dv", ctypes.c_int), ("chunk", ctypes.c_int),
        ("dtype", ctypes.c_int), ("algo", ctypes.c_int),
        ("g_min", ctypes.c_float), ("scale", ctypes.c_float), ("l2_eps", ctypes.c_float),
        ("qk_l2norm_in_kernel", ctypes.c_int), ("beta_sigmoid_in_kernel", ctypes.c_int),
        ("gate_in_kernel", ctypes.c_int),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("g", ctypes.c_void_p), ("beta", ctypes.c_void_p),
        ("A_log", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p), ("S0", ctypes.c_void_p),
        ("o", ctypes.c_void_p), ("S_T", ctypes.c_void_p), ("M_T", ctypes.c_void_p),
        ("S_chunks", ctypes.c_void_p), ("g_per_head", ctypes.c_int),
    ]


class ChunkBwdArgs(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int), ("HV", ctypes.c_int),
        ("Dk", ctypes.c_int), ("Dv", ctypes.c_int), ("chunk", ctypes.c_int),
        ("dtype", ctypes.c_int), ("algo", ctypes.c_int),
        ("g_min", ctypes.c_float), ("scale", ctypes.c_float), ("l2_eps", ctypes.c_float),
        ("qk_l2norm_in_kernel", ctypes.c_int), ("beta_sigmoid_in_kernel", ctypes.c_int),
        ("gate_in_kernel", ctypes.c_int),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("g", ctypes.c_void_p), ("beta", ctypes.c_void_p),
        ("A_log", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p), ("S_chunks", ctypes.c_void_p),
        ("dout", ctypes.c_void_p), ("dS_T", ctypes.c_void_p),
        ("dq", ctypes.c_void_p), ("dk", ctypes.c_void_p), ("dv", ctypes.c_void_p),
        ("dg", ctypes.c_void_p), ("dbeta", ctypes.c_void_p), ("dS0", ctypes.c_void_p),
        ("dA_log", ctypes.c_void_p), ("ddt_bias", ctypes.c_void_p), ("g_per_head", ctypes.c_int),
    ]


class StepArgs(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("HV", ctypes.c_int),
        ("Dk", ctypes.c_int), ("Dv", ctypes.c_int), ("dtype", ctypes.c_int),
        ("g_min", ctypes.c_float), ("scale", ctypes.c_float), ("l2_eps", ctypes.c_float),
        ("qk_l2norm_in_kernel", ctypes.c_int), ("beta_sigmoid_in_kernel", ctypes.c_int),
        ("gate_in_kernel", ctypes.c_int),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("g", ctypes.c_void_p), ("beta", ctypes.c_void_p),
        ("A_log", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p),
        ("S", ctypes.c_void_p), ("o", ctypes.c_void_p), ("g_per_head", ctypes.c_int),
    ]


class ConvArgs(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("T", ctypes.c_int), ("C", ctypes.c_int), ("K", ctypes.c_int),
        ("head_dim", ctypes.c_int), ("silu", ctypes.c_int), ("l2_eps", ctypes.c_float),
        ("x", ctypes.c_void_p), ("w", ctypes.c_void_p), ("bias", ctypes.c_void_p),
        ("state_in", ctypes.c_void_p), ("y", ctypes.c_void_p), ("state_out", ctypes.c_void_p),
    ]


class GateArgs(ctypes.Structure):
    _fields_ = [
        ("N", ctypes.c_int), ("HV", ctypes.c_int), ("D", ctypes.c_int), ("eps", ctypes.c_float),
        ("o", ctypes.c_void_p), ("gate", ctypes.c_void_p), ("weight", ctypes.c_void_p),
        ("y", ctypes.c_void_p),
    ]


EXPORTS = ["kda_chunk_fwd", "kda_chunk_bwd", "kda_step", "kda_compose", "kda_device_status",
           "kda_status_string", "kda_version", "kda_debug_chunk_stall",
           "kda_short_conv", "kda_output_gate"]

_lib = None


def library_path() -> str:
    return _build.LIB


def load():
    """Load (building first if needed) the CUDA library; raises if unavailable."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.build()
    if not os.path.exists(path):
        raise ImportError("libkda_b200.so is missing and could not be built")
    lib = ctypes.CDLL(path)
    lib.kda_chunk_fwd.argtypes = [ctypes.POINTER(ChunkArgs), ctypes.c_void_p]
    lib.kda_chunk_fwd.restype = ctypes.c_int
    lib.kda_chunk_bwd.argtypes = [ctypes.POINTER(ChunkBwdArgs), ctypes.c_void_p]
    lib.kda_chunk_bwd.restype = ctypes.c_int
    lib.kda_debug_chunk_stall.argtypes = [ctypes.POINTER(ChunkArgs), ctypes.c_void_p]
    lib.kda_debug_chunk_stall.restype = ctypes.c_int
    lib.kda_short_conv.argtypes = [ctypes.POINTER(ConvArgs), ctypes.c_void_p]
    lib.kda_short_conv.restype = ctypes.c_int
    lib.kda_output_gate.argtypes = [ctypes.POINTER(GateArgs), ctypes.c_void_p]
    lib.kda_output_gate.restype = ctypes.c_int
    lib.kda_step.argtypes = [ctypes.POINTER(StepArgs), ctypes.c_void_p]
    lib.kda_step.restype = ctypes.c_int
    lib.kda_compose.argtypes = [ctypes.c_int] * 4 + [ctypes.c_void_p] * 5
    lib.kda_compose.restype = ctypes.c_int
    lib.kda_device_status.argtypes = [ctypes.c_void_p]
    lib.kda_device_status.restype = ctypes.c_int
    lib.kda_status_string.argtypes = [ctypes.c_int]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_version.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr()).value


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.float32:
        return DT_F32
    if t.dtype == torch.bfloat16:
        return DT_BF16
    raise ValueError("activations must be float32 or bfloat16, got %s" % t.dtype)


def _check(t, name, shape, dtype, device):
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s has dtype %s, expected %s" % (name, t.dtype, dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


GATES = {"bounded": 1, "softplus": 2}


def _gate_code(gate_in_kernel):
    """True / "bounded" -> 1 (bounded sigmoid gate), "softplus" -> 2, False -> 0."""
    if isinstance(gate_in_kernel, str):
        return GATES[gate_in_kernel]
    return 1 if gate_in_kernel else 0


def _raise(fn, status):
    if status != KDA_OK:
        raise KdaError(fn, status)


def _call(name, dev, cfn, *args):
    """Call library entry point `cfn` with `dev` as the current device: the
    library launches on the current device (and keeps its per-device state
    there), so tensors on another device would otherwise be handed to kernels
    on the wrong GPU.  Raises KdaError on a non-OK status."""
    with torch.cuda.device(dev):
        _raise(name, cfn(*args))


def kda_chunk_fwd(q, k, v, g, beta, *, A_log=None, dt_bias=None, S0=None, chunk=64,
                  g_min=-5.0, scale=1.0, l2_eps=1e-6, qk_l2norm_in_kernel=True,
                  beta_sigmoid_in_kernel=True, gate_in_kernel=True,
                  output_final_state=True, output_transition=False, algo="auto",
                  o=None, S_T=None, M_T=None, S_chunks=None, g_per_head=False, stream=None,
                  output_o=True, _withhold_ready=False):
    """Chunk-parallel KDA forward.  Returns (o or None, S_T or None, M_T or None).

    output_o=False (with o=None) skips the output rows: only the states are
    computed (the first pass of a segmented run).

    (_withhold_ready routes to kda_debug_chunk_stall, the failure-path test hook.)

    q, k [B,T,H,Dk]; v [B,T,HV,Dv]; g (log-decay or raw z) [B,T,HV,Dk];
    beta (or logits) [B,T,HV] -- all float32 or all bfloat16, on one CUDA device.
    A_log [HV], dt_bias [HV,Dk], S0 [B,HV,Dk,Dv]: float32.
    S_chunks: optional float32 [B,HV,ceil(T/chunk),Dk,Dv] that receives the
    state entering every chunk (the input of kda_chunk_bwd).
    gate_in_kernel: True or "bounded" (g_min sigmoid gate), "softplus"
    (-exp(A_log) softplus gate, SIMT only) or False.  g_per_head: g [B,T,HV]
    and dt_bias [HV], one decay per (token, value head).
    """
    lib = load()
    if not isinstance(q, torch.Tensor) or not q.is_cuda:
        raise ValueError("q must be a CUDA tensor")
    dev = q.device
    B, T, H, Dk = q.shape
    HV, Dv = v.shape[2], v.shape[3]
    dt = q.dtype
    _check(q, "q", (B, T, H, Dk), dt, dev)
    _check(k, "k", (B, T, H, Dk), dt, dev)
    _check(v, "v", (B, T, HV, Dv), dt, dev)
    gk = () if g_per_head else (Dk,)
    _check(g, "g", (B, T, HV) + gk, dt, dev)
    _check(beta, "beta", (B, T, HV), dt, dev)
    _check(A_log, "A_log", (HV,), torch.float32, dev)
    _check(dt_bias, "dt_bias", (HV,) + gk, torch.float32, dev)
    _check(S0, "S0", (B, HV, Dk, Dv), torch.float32, dev)
    if o is None and output_o:
        o = torch.empty((B, T, HV, Dv), dtype=dt, device=dev)
    _check(o, "o", (B, T, HV, Dv), dt, dev)
    if S_T is None and output_final_state:
        S_T = torch.empty((B, HV, Dk, Dv), dtype=torch.float32, device=dev)
    _check(S_T, "S_T", (B, HV, Dk, Dv), torch.float32, dev)
    if M_T is None and output_transition:
        M_T = torch.empty((B, HV, Dk, Dk), dtype=torch.float32, device=dev)
    _check(M_T, "M_T", (B, HV, Dk, Dk), torch.float32, dev)
    _check(S_chunks, "S_chunks", (B, HV, -(-T // int(chunk)), Dk, Dv), torch.float32, dev)
    a = ChunkArgs()
    a.B, a.T, a.H, a.HV, a.Dk, a.Dv, a.chunk = B, T, H, HV, Dk, Dv, int(chunk)
    a.dtype, a.algo = _dtype_code(q), ALGOS[algo]
    a.g_min, a.scale, a.l2_eps = float(g_min), float(scale), float(l2_eps)
    a.qk_l2norm_in_kernel = int(bool(qk_l2norm_in_kernel))
    a.beta_sigmoid_in_kernel = int(bool(beta_sigmoid_in_kernel))
    a.gate_in_kernel = _gate_code(gate_in_kernel)
    a.g_per_head = int(bool(g_per_head))
    a.q, a.k, a.v, a.g, a.beta = map(_ptr, (q, k, v, g, beta))
    a.A_log, a.dt_bias, a.S0 = _ptr(A_log), _ptr(dt_bias), _ptr(S0)
    a.o, a.S_T, a.M_T, a.S_chunks = _ptr(o), _ptr(S_T), _ptr(M_T), _ptr(S_chunks)
    if _withhold_ready:
        _call("kda_debug_chunk_stall", dev, lib.kda_debug_chunk_stall, ctypes.byref(a), _stream(stream, dev))
    else:
        _call("kda_chunk_fwd", dev, lib.kda_chunk_fwd, ctypes.byref(a), _stream(stream, dev))
    return o, S_T, M_T


def kda_chunk_bwd(q, k, v, g, beta, S_chunks, dout, dS_T=None, *, A_log=None, dt_bias=None,
                  chunk=64, g_min=-5.0, scale=1.0, l2_eps=1e-6, qk_l2norm_in_kernel=True,
                  beta_sigmoid_in_kernel=True, gate_in_kernel=True, want_dS0=True, algo="auto",
                  g_per_head=False, stream=None):
    """Gradient of <dout, o> + <dS_T, S_T> for a kda_chunk_fwd call with the
    same arguments, from the per-chunk states S_chunks that call wrote.

    Returns a dict of float32 tensors: dq, dk [B,T,H,Dk]; dv [B,T,HV,Dv];
    dg [B,T,HV,Dk] ([B,T,HV] with g_per_head; w.r.t. g, or z with the
    in-kernel gate); dbeta [B,T,HV] (w.r.t. beta, or its logit); dS0
    [B,HV,Dk,Dv] (if want_dS0); dA_log [HV] and ddt_bias [HV,Dk] ([HV] with
    g_per_head) with the in-kernel gate (ddt_bias only if dt_bias is given).
    """
    lib = load()
    if not isinstance(q, torch.Tensor) or not q.is_cuda:
        raise ValueError("q must be a CUDA tensor")
    dev = q.device
    B, T, H, Dk = q.shape
    HV, Dv = v.shape[2], v.shape[3]
    dt = q.dtype
    NC = -(-T // int(chunk))
    _check(q, "q", (B, T, H, Dk), dt, dev)
    _check(k, "k", (B, T, H, Dk), dt, dev)
    _check(v, "v", (B, T, HV, Dv), dt, dev)
    gk = () if g_per_head else (Dk,)
    _check(g, "g", (B, T, HV) + gk, dt, dev)
    _check(beta, "beta", (B, T, HV), dt, dev)
    _check(dout, "dout", (B, T, HV, Dv), dt, dev)
    _check(A_log, "A_log", (HV,), torch.float32, dev)
    _check(dt_bias, "dt_bias", (HV,) + gk, torch.float32, dev)
    _check(S_chunks, "S_chunks", (B, HV, NC, Dk, Dv), torch.float32, dev)
    _check(dS_T, "dS_T", (B, HV, Dk, Dv), torch.float32, dev)
    f32 = dict(dtype=torch.float32, device=dev)
    out = {"dq": torch.empty((B, T, H, Dk), **f32), "dk": torch.empty((B, T, H, Dk), **f32),
           "dv": torch.empty((B, T, HV, Dv), **f32), "dg": torch.empty((B, T, HV) + gk, **f32),
           "dbeta": torch.empty((B, T, HV), **f32),
           "dS0": torch.empty((B, HV, Dk, Dv), **f32) if want_dS0 else None,
           "dA_log": torch.empty((HV,), **f32) if gate_in_kernel else None,
           "ddt_bias": torch.empty((HV,) + gk, **f32) if (gate_in_kernel and dt_bias is not None) else None}
    a = ChunkBwdArgs()
    a.B, a.T, a.H, a.HV, a.Dk, a.Dv, a.chunk = B, T, H, HV, Dk, Dv, int(chunk)
    a.dtype, a.algo = _dtype_code(q), ALGOS[algo]
    a.g_min, a.scale, a.l2_eps = float(g_min), float(scale), float(l2_eps)
    a.qk_l2norm_in_kernel = int(bool(qk_l2norm_in_kernel))
    a.beta_sigmoid_in_kernel = int(bool(beta_sigmoid_in_kernel))
    a.gate_in_kernel = _gate_code(gate_in_kernel)
    a.g_per_head = int(bool(g_per_head))
    a.q, a.k, a.v, a.g, a.beta = map(_ptr, (q, k, v, g, beta))
    a.A_log, a.dt_bias, a.S_chunks = _ptr(A_log), _ptr(dt_bias), _ptr(S_chunks)
    a.dout, a.dS_T = _ptr(dout), _ptr(dS_T)
    for name in ("dq", "dk", "dv", "dg", "dbeta", "dS0", "dA_log", "ddt_bias"):
        setattr(a, name, _ptr(out[name]))
    _call("kda_chunk_bwd", dev, lib.kda_chunk_bwd, ctypes.byref(a), _stream(stream, dev))
    return out


def kda_step(S, q, k, v, g, beta, *, A_log=None, dt_bias=None, g_min=-5.0, scale=1.0,
             l2_eps=1e-6, qk_l2norm_in_kernel=True, beta_sigmoid_in_kernel=True,
             gate_in_kernel=True, g_per_head=False, o=None, stream=None):
    """One decode step; S [B,HV,Dk,Dv] float32 is updated in place.  Returns o [B,HV,Dv].

    q, k [B,H,Dk]; v [B,HV,Dv]; g [B,HV,Dk] ([B,HV] with g_per_head);
    beta [B,HV] (float32 or bfloat16).  gate_in_kernel as kda_chunk_fwd.
    """
    lib = load()
    if not isinstance(S, torch.Tensor) or not S.is_cuda:
        raise ValueError("S must be a CUDA tensor")
    dev = S.device
    B, HV, Dk, Dv = S.shape
    H = q.shape[1]
    dt = q.dtype
    _check(S, "S", (B, HV, Dk, Dv), torch.float32, dev)
    _check(q, "q", (B, H, Dk), dt, dev)
    _check(k, "k", (B, H, Dk), dt, dev)
    _check(v, "v", (B, HV, Dv), dt, dev)
    gk = () if g_per_head else (Dk,)
    _check(g, "g", (B, HV) + gk, dt, dev)
    _check(beta, "beta", (B, HV), dt, dev)
    _check(A_log, "A_log", (HV,), torch.float32, dev)
    _check(dt_bias, "dt_bias", (HV,) + gk, torch.float32, dev)
    if o is None:
        o = torch.empty((B, HV, Dv), dtype=dt, device=dev)
    _check(o, "o", (B, HV, Dv), dt, dev)
    a = StepArgs()
    a.B, a.H, a.HV, a.Dk, a.Dv = B, H, HV, Dk, Dv
    a.dtype = _dtype_code(q)
    a.g_min, a.scale, a.l2_eps = float(g_min), float(scale), float(l2_eps)
    a.qk_l2norm_in_kernel = int(bool(qk_l2norm_in_kernel))
    a.beta_sigmoid_in_kernel = int(bool(beta_sigmoid_in_kernel))
    a.gate_in_kernel = _gate_code(gate_in_kernel)
    a.g_per_head = int(bool(g_per_head))
    a.q, a.k, a.v, a.g, a.beta = map(_ptr, (q, k, v, g, beta))
    a.A_log, a.dt_bias, a.S, a.o = _ptr(A_log), _ptr(dt_bias), _ptr(S), _ptr(o)
    _call("kda_step", dev, lib.kda_step, ctypes.byref(a), _stream(stream, dev))
    return o


def kda_compose(M, S_seg, S_init=None, S_in=None, stream=None):
    """Segment prefix combine.  M [n,BH,Dk,Dk], S_seg [n,BH,Dk,Dv], S_init [BH,Dk,Dv]
    (float32, CUDA).  Returns S_in [n+1,BH,Dk,Dv] with S_in[s] the state entering
    segment s and S_in[n] the final state."""
    lib = load()
    dev = S_seg.device
    n, BH, Dk, Dv = S_seg.shape
    _check(M, "M", (n, BH, Dk, Dk), torch.float32, dev)
    _check(S_seg, "S_seg", (n, BH, Dk, Dv), torch.float32, dev)
    _check(S_init, "S_init", (BH, Dk, Dv), torch.float32, dev)
    if S_in is None:
        S_in = torch.empty((n + 1, BH, Dk, Dv), dtype=torch.float32, device=dev)
    _check(S_in, "S_in", (n + 1, BH, Dk, Dv), torch.float32, dev)
    _call("kda_compose", dev, lib.kda_compose, n, BH, Dk, Dv, _ptr(M), _ptr(S_seg), _ptr(S_init),
          _ptr(S_in), _stream(stream, dev))
    return S_in


def kda_short_conv(x, w, bias=None, *, head_dim=0, silu=True, l2_eps=1e-6, state_in=None,
                   y=None, state_out=None, want_state=False, stream=None):
    """Layer prologue: causal depthwise short convolution (K = w.shape[1] taps,
    tap K-1 on the current token), then SiLU and per-128-channel L2 norm when
    asked.  x [B,T,C] bf16 (C % 128 == 0); w [C,K], bias [C] float32;
    state_in [B,K-1,C] bf16 (tokens before x, oldest first) or None.
    Returns y [B,T,C] bf16, or (y, state_out) with want_state."""
    lib = load()
    if not isinstance(x, torch.Tensor) or not x.is_cuda:
        raise ValueError("x must be a CUDA tensor")
    dev = x.device
    B, T, C = x.shape
    K = w.shape[1]
    _check(x, "x", (B, T, C), torch.bfloat16, dev)
    _check(w, "w", (C, K), torch.float32, dev)
    _check(bias, "bias", (C,), torch.float32, dev)
    _check(state_in, "state_in", (B, K - 1, C), torch.bfloat16, dev)
    if y is None:
        y = torch.empty_like(x)
    _check(y, "y", (B, T, C), torch.bfloat16, dev)
    if state_out is None and want_state:
        state_out = torch.empty((B, K - 1, C), dtype=torch.bfloat16, device=dev)
    _check(state_out, "state_out", (B, K - 1, C), torch.bfloat16, dev)
    a = ConvArgs()
    a.B, a.T, a.C, a.K = B, T, C, K
    a.head_dim, a.silu, a.l2_eps = int(head_dim), int(bool(silu)), float(l2_eps)
    a.x, a.w, a.bias, a.state_in = _ptr(x), _ptr(w), _ptr(bias), _ptr(state_in)
    a.y, a.state_out = _ptr(y), _ptr(state_out)
    _call("kda_short_conv", dev, lib.kda_short_conv, ctypes.byref(a), _stream(stream, dev))
    return (y, state_out) if want_state else y


def kda_output_gate(o, gate, weight=None, *, eps=1e-6, y=None, stream=None):
    """Layer epilogue: sigmoid(gate) * weight * RMSNorm over each head's D = 128
    channels of o.  o, gate [..., HV, D] bf16; weight [D] float32 or None."""
    lib = load()
    if not isinstance(o, torch.Tensor) or not o.is_cuda:
        raise ValueError("o must be a CUDA tensor")
    dev = o.device
    HV, D = o.shape[-2], o.shape[-1]
    N = o.numel() // (HV * D)
    _check(o, "o", tuple(o.shape), torch.bfloat16, dev)
    _check(gate, "gate", tuple(o.shape), torch.bfloat16, dev)
    _check(weight, "weight", (D,), torch.float32, dev)
    if y is None:
        y = torch.empty_like(o)
    _check(y, "y", tuple(o.shape), torch.bfloat16, dev)
    a = GateArgs()
    a.N, a.HV, a.D, a.eps = N, HV, D, float(eps)
    a.o, a.gate, a.weight, a.y = _ptr(o), _ptr(gate), _ptr(weight), _ptr(y)
    _call("kda_output_gate", dev, lib.kda_output_gate, ctypes.byref(a), _stream(stream, dev))
    return y


def kda_device_status(stream=None, device=None):
    """Synchronise and read/clear the device error word; raises KdaError if set."""
    lib = load()
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    _call("kda_device_status", dev, lib.kda_device_status, _stream(stream, dev))


def kda_status_string(status: int) -> str:
    return load().kda_status_string(int(status)).decode()


def kda_version() -> int:
    return int(load().kda_version())
