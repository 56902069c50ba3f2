"""Thin Python binding of libkda.so (ctypes).

Argument marshalling only: tensors are passed to the C ABI as device
pointers, the stream is torch's current stream, and every step of the KDA
forward pass runs in the library's CUDA kernels.  Nothing here computes on the
host, and there is no fallback: if ``libkda.so`` is missing or fails to load,
every call raises ``KdaLibraryError``.

Names follow the C ABI in ``include/kda.h``: ``prefill``, ``prologue``,
``recurrence``, ``decode_step``, ``prefill_workspace_size``, ``status_string``.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkda.so")
_lib = None

KDA_OK, KDA_ERR_INVALID_ARGUMENT, KDA_ERR_UNSUPPORTED = 0, 1, 2
KDA_ERR_WORKSPACE, KDA_ERR_CUDA, KDA_ERR_TIMEOUT = 3, 4, 5
KDA_BF16, KDA_FP32 = 0, 1

EXPORTED = ["kda_prefill_workspace_size", "kda_prefill", "kda_prefill_status", "kda_prologue",
            "kda_recurrence", "kda_recurrence_workspace_size", "kda_decode_step",
            "kda_status_string", "kda_version", "kda_prefill_noalloc", "kda_kernel_timing",
            "kda_kernel_times", "kda_prefill_gated", "kda_decode_step_gated", "kda_prefill_ex",
            "kda_decode_multi", "kda_decode_ex", "kda_device_status"]


class KdaLibraryError(RuntimeError):
    """libkda.so is missing or could not be loaded."""


class KdaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__("%s failed: %s" % (what, status_string(status)))
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("seq_len", ctypes.c_int32),
                ("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("lower_bound", ctypes.c_float), ("l2norm_eps", ctypes.c_float),
                ("scale", ctypes.c_float), ("io_dtype", ctypes.c_int32), ("flags", ctypes.c_uint32)]


KDA_FLAG_NEGATIVE_EIGENVALUES = 0x1
KDA_FLAG_TOKEN_RECURRENCE = 0x2           # off the tensor-core path: the token loop (include/kda.h)
KDA_FLAG_TEST_EXPIRE_WAITS = 0x80000000   # failure-path tests only (include/kda.h)
KDA_STATUS_BAD_CU_SEQLENS, KDA_STATUS_TIMEOUT_PREP = 0x1, 0x2
KDA_STATUS_TIMEOUT_STATE, KDA_STATUS_TIMEOUT_DECODE = 0x4, 0x8


class OutputGate(ctypes.Structure):
    """kda_output_gate: o <- o / sqrt(mean o^2 + eps) * weight * sigmoid(gate)."""
    _fields_ = [("gate", ctypes.c_void_p), ("weight", ctypes.c_void_p), ("eps", ctypes.c_float)]


class PrefillArgs(ctypes.Structure):
    """kda_prefill_args: every pointer of a kda_prefill_ex call."""
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("q", "k", "v", "conv_w", "alpha", "b", "A_log", "dt_bias", "initial_state",
                 "initial_conv_state", "cu_seqlens", "o", "final_state", "final_conv_state",
                 "out_gate", "snapshots")] + [("snapshot_every", ctypes.c_int32),
                                              ("snapshot_capacity", ctypes.c_int32),
                                              ("side_stream", ctypes.c_void_p)]


class DecodeArgs(ctypes.Structure):
    """kda_decode_args: every pointer of a kda_decode_ex call (status: device int32 or None)."""
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("q", "k", "v", "alpha", "b", "conv_w", "A_log", "dt_bias", "out_gate", "state",
                 "conv_state", "o", "step_states", "status")]


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libkda.so (build it first with ``gated_delta_rule_70_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise KdaLibraryError("libkda.so not found at %s; run `python -m gated_delta_rule_70_b200.build`"
                              % _LIB_PATH)
    try:
        lib = ctypes.CDLL(_LIB_PATH)
    except OSError as e:
        raise KdaLibraryError("cannot load %s: %s" % (_LIB_PATH, e)) from e
    P, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    SP = ctypes.POINTER(Shape)
    lib.kda_prefill_workspace_size.argtypes = [SP, i32]
    lib.kda_prefill_workspace_size.restype = sz
    lib.kda_prefill.argtypes = [SP] + [P] * 14 + [P, sz, P]
    lib.kda_prefill.restype = i32
    lib.kda_prefill_status.argtypes = [P, P]
    lib.kda_prefill_status.restype = i32
    lib.kda_prologue.argtypes = [SP] + [P] * 16 + [P]
    lib.kda_prologue.restype = i32
    lib.kda_recurrence.argtypes = [SP] + [P] * 9 + [P, sz, P]
    lib.kda_recurrence.restype = i32
    lib.kda_recurrence_workspace_size.argtypes = [SP, i32]
    lib.kda_recurrence_workspace_size.restype = sz
    lib.kda_decode_step.argtypes = [SP] + [P] * 11 + [P]
    lib.kda_decode_step.restype = i32
    OG = ctypes.POINTER(OutputGate)
    lib.kda_prefill_gated.argtypes = [SP] + [P] * 11 + [OG] + [P] * 3 + [P, sz, P]
    lib.kda_prefill_gated.restype = i32
    lib.kda_decode_step_gated.argtypes = [SP] + [P] * 8 + [OG] + [P] * 3 + [P]
    lib.kda_decode_step_gated.restype = i32
    lib.kda_prefill_ex.argtypes = [SP, ctypes.POINTER(PrefillArgs), P, sz, P]
    lib.kda_prefill_ex.restype = i32
    lib.kda_decode_multi.argtypes = [SP] + [P] * 8 + [OG] + [P] * 4 + [P]
    lib.kda_decode_multi.restype = i32
    lib.kda_decode_ex.argtypes = [SP, ctypes.POINTER(DecodeArgs), P]
    lib.kda_decode_ex.restype = i32
    lib.kda_device_status.argtypes = [P, P]
    lib.kda_device_status.restype = i32
    lib.kda_status_string.argtypes = [i32]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_version.argtypes = []
    lib.kda_version.restype = i32
    lib.kda_kernel_timing.argtypes = [i32]
    lib.kda_kernel_timing.restype = i32
    lib.kda_kernel_times.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float)]
    lib.kda_kernel_times.restype = i32
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().kda_status_string(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("KDA tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("KDA tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return KDA_BF16
    if dt == torch.float32:
        return KDA_FP32
    raise ValueError("io dtype must be bfloat16 or float32, got %s" % dt)


def make_shape(num_seqs: int, seq_len: int, num_heads: int, head_dim: int, io_dtype: torch.dtype,
               lower_bound: float = -5.0, l2norm_eps: float = 1e-6, scale: float = 1.0,
               negative_eigenvalues: bool = False, flags: int = 0) -> Shape:
    """A kda_shape; ``flags`` adds raw KDA_FLAG_* bits (e.g. the failure-path test flag)."""
    return Shape(num_seqs, seq_len, num_heads, head_dim, lower_bound, l2norm_eps, scale,
                 _dtype_code(io_dtype),
                 (KDA_FLAG_NEGATIVE_EIGENVALUES if negative_eigenvalues else 0) | int(flags))


_side_streams = {}


def side_stream(device: torch.device) -> torch.cuda.Stream:
    """A high-priority stream per device, handed to kda_prefill_ex as its side stream
    (the time-segmented schedule of few long sequences runs its state passes there)."""
    key = torch.device(device).index if torch.device(device).index is not None else \
        torch.cuda.current_device()
    if key not in _side_streams:
        _side_streams[key] = torch.cuda.Stream(device=torch.device("cuda", key), priority=-100)
    return _side_streams[key]


def device_status(word: torch.Tensor) -> int:
    """Synchronise the current stream and read a device status word (kda_device_status)."""
    return int(load_library().kda_device_status(_ptr(word), _stream(word.device)))


def prefill_workspace_size(shape: Shape, varlen: bool) -> int:
    return int(load_library().kda_prefill_workspace_size(ctypes.byref(shape), int(varlen)))


def _check(status: int, what: str):
    if status != KDA_OK:
        raise KdaError(status, what)


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, conv_w: torch.Tensor,
            alpha: torch.Tensor, b: torch.Tensor, A_log: torch.Tensor, dt_bias: torch.Tensor,
            initial_state: Optional[torch.Tensor] = None, cu_seqlens: Optional[torch.Tensor] = None,
            initial_conv_state: Optional[torch.Tensor] = None, *, num_seqs: Optional[int] = None,
            lower_bound: float = -5.0, l2norm_eps: float = 1e-6,
            scale: float = 1.0, negative_eigenvalues: bool = False,
            out_gate: Optional[torch.Tensor] = None, o_norm_weight: Optional[torch.Tensor] = None,
            o_norm_eps: float = 1e-5, snapshots: Optional[torch.Tensor] = None,
            snapshot_every: int = 1,
            want_conv_state: bool = True, out: Optional[torch.Tensor] = None,
            final_state: Optional[torch.Tensor] = None,
            final_conv_state: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
            check: bool = False, segments: bool = True,
            flags: int = 0) -> Tuple[torch.Tensor, torch.Tensor, Optional[torch.Tensor]]:
    """KDA prefill.  q, k, v: [T_total, H*d] (or [B, T, H*d] dense); alpha: [.., H, d];
    b: [.., H].  Returns (o [T_total, H, d], final_state [N, H, d, d], final_conv_state
    [N, 3, 3*H*d] or None).  ``negative_eigenvalues``: beta = 2 sigmoid(b).  ``out_gate``
    [.., H, d] with ``o_norm_weight`` [d] fp32: the output epilogue o <- o / sqrt(mean o^2 +
    o_norm_eps) * weight * sigmoid(out_gate).  ``snapshots`` [N, C, H, d, d] fp32: snapshot j
    of sequence n (j < C) is the state after its first (j + 1) * 64 * snapshot_every tokens.
    The call is asynchronous on the current stream.  ``check=True`` then synchronises that
    stream and raises on a device-side error (bad cu_seqlens, a bounded wait that gave up);
    leave it off on hot paths.  ``segments``: hand the library this device's high-priority
    side stream, so few long sequences run in overlapped time segments.  ``flags``: raw
    KDA_FLAG_* bits added to the shape."""
    lib = load_library()
    H, d = alpha.shape[-2], alpha.shape[-1]
    if cu_seqlens is not None:
        N = cu_seqlens.numel() - 1
        T_total = q.numel() // (H * d)
        shape = make_shape(N, T_total, H, d, q.dtype, lower_bound, l2norm_eps, scale,
                           negative_eigenvalues, flags)
    else:
        if q.dim() == 3:
            N, T = q.shape[0], q.shape[1]
        else:
            N = 1 if num_seqs is None else num_seqs
            T = q.numel() // (H * d) // N
        T_total = N * T
        shape = make_shape(N, T, H, d, q.dtype, lower_bound, l2norm_eps, scale, negative_eigenvalues,
                           flags)
    dev = q.device
    o = out if out is not None else torch.empty((T_total, H, d), dtype=q.dtype, device=dev)
    fs = final_state if final_state is not None else torch.empty((N, H, d, d), dtype=torch.float32,
                                                                 device=dev)
    fc = final_conv_state
    if fc is None and want_conv_state:
        fc = torch.empty((N, 3, 3 * H * d), dtype=q.dtype, device=dev)
    ws_bytes = prefill_workspace_size(shape, cu_seqlens is not None)
    ws = workspace
    if ws is None or ws.numel() < ws_bytes:
        ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    og = _output_gate(out_gate, o_norm_weight, o_norm_eps)
    og_struct = og._obj if og is not None else None
    pa = PrefillArgs(*[_ptr(t) for t in (q, k, v, conv_w, alpha, b, A_log, dt_bias, initial_state,
                                         initial_conv_state, cu_seqlens, o, fs, fc)],
                     ctypes.cast(ctypes.pointer(og_struct), ctypes.c_void_p) if og_struct is not None
                     else None,
                     _ptr(snapshots), int(snapshot_every),
                     int(snapshots.shape[1]) if snapshots is not None else 0,
                     ctypes.c_void_p(side_stream(dev).cuda_stream) if segments else None)
    st = lib.kda_prefill_ex(ctypes.byref(shape), ctypes.byref(pa), _ptr(ws),
                            ctypes.c_size_t(ws.numel()), _stream(dev))
    _check(st, "kda_prefill")
    if check:
        _check(lib.kda_prefill_status(_ptr(ws), _stream(dev)), "kda_prefill (device)")
    return o, fs, fc


def _output_gate(gate, weight, eps):
    """A kda_output_gate for the call, or None (no epilogue)."""
    if gate is None and weight is None:
        return None
    if gate is None or weight is None:
        raise ValueError("out_gate and o_norm_weight go together")
    return ctypes.byref(OutputGate(_ptr(gate), _ptr(weight), float(eps)))


def _prefill_shape(q, alpha, cu_seqlens, num_seqs, lower_bound, l2norm_eps, scale,
                   negative_eigenvalues=False):
    H, d = alpha.shape[-2], alpha.shape[-1]
    T_total = q.numel() // (H * d)
    if cu_seqlens is not None:
        return make_shape(cu_seqlens.numel() - 1, T_total, H, d, q.dtype, lower_bound, l2norm_eps,
                          scale, negative_eigenvalues), T_total
    N = (q.shape[0] if q.dim() == 3 else 1) if num_seqs is None else num_seqs
    return make_shape(N, T_total // max(N, 1), H, d, q.dtype, lower_bound, l2norm_eps, scale,
                      negative_eigenvalues), T_total


def prologue(q, k, v, conv_w, alpha, b, A_log, dt_bias, cu_seqlens=None, initial_conv_state=None,
             *, num_seqs: Optional[int] = None, lower_bound: float = -5.0, l2norm_eps: float = 1e-6,
             negative_eigenvalues: bool = False, want_conv_state: bool = False, out=None):
    """The prologue alone: returns (qn, kn, vc [T,H,d] io dtype, g [T,H,d] fp32, beta [T,H] fp32,
    final_conv_state [N,3,3*H*d] or None).  ``out`` may pass those six buffers preallocated."""
    lib = load_library()
    shape, T_total = _prefill_shape(q, alpha, cu_seqlens, num_seqs, lower_bound, l2norm_eps, 1.0,
                                    negative_eigenvalues)
    H, d, N = shape.num_heads, shape.head_dim, shape.num_seqs
    dev = q.device
    if out is None:
        qn, kn, vc = (torch.empty((T_total, H, d), dtype=q.dtype, device=dev) for _ in range(3))
        g = torch.empty((T_total, H, d), dtype=torch.float32, device=dev)
        beta = torch.empty((T_total, H), dtype=torch.float32, device=dev)
        fc = torch.empty((N, 3, 3 * H * d), dtype=q.dtype, device=dev) if want_conv_state else None
    else:
        qn, kn, vc, g, beta, fc = out
    st = lib.kda_prologue(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(conv_w), _ptr(alpha),
                          _ptr(b), _ptr(A_log), _ptr(dt_bias), _ptr(initial_conv_state),
                          _ptr(cu_seqlens), _ptr(qn), _ptr(kn), _ptr(vc), _ptr(g), _ptr(beta),
                          _ptr(fc), _stream(dev))
    _check(st, "kda_prologue")
    return qn, kn, vc, g, beta, fc


def recurrence_workspace_size(shape: Shape, varlen: bool) -> int:
    return int(load_library().kda_recurrence_workspace_size(ctypes.byref(shape), int(varlen)))


def recurrence(qn, kn, vc, g, beta, initial_state=None, cu_seqlens=None, *,
               num_seqs: Optional[int] = None, scale: float = 1.0, out=None, final_state=None,
               workspace: Optional[torch.Tensor] = None):
    """The recurrence on prepared inputs (what ``prologue`` returns): (o [T,H,d], final_state)."""
    lib = load_library()
    T_total, H, d = qn.shape
    if cu_seqlens is not None:
        shape = make_shape(cu_seqlens.numel() - 1, T_total, H, d, qn.dtype, scale=scale)
    else:
        N = 1 if num_seqs is None else num_seqs
        shape = make_shape(N, T_total // max(N, 1), H, d, qn.dtype, scale=scale)
    dev = qn.device
    o = out if out is not None else torch.empty((T_total, H, d), dtype=qn.dtype, device=dev)
    fs = final_state if final_state is not None else torch.empty(
        (shape.num_seqs, H, d, d), dtype=torch.float32, device=dev)
    ws_bytes = recurrence_workspace_size(shape, cu_seqlens is not None)
    ws = workspace
    if ws is None or ws.numel() < ws_bytes:
        ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    st = lib.kda_recurrence(ctypes.byref(shape), _ptr(qn), _ptr(kn), _ptr(vc), _ptr(g), _ptr(beta),
                            _ptr(initial_state), _ptr(cu_seqlens), _ptr(o), _ptr(fs), _ptr(ws),
                            ctypes.c_size_t(ws.numel()), _stream(dev))
    _check(st, "kda_recurrence")
    return o, fs


def decode_step(q, k, v, alpha, b, conv_w, A_log, dt_bias, state: torch.Tensor,
                conv_state: torch.Tensor, *, lower_bound: float = -5.0, l2norm_eps: float = 1e-6,
                scale: float = 1.0, negative_eigenvalues: bool = False,
                out_gate: Optional[torch.Tensor] = None, o_norm_weight: Optional[torch.Tensor] = None,
                o_norm_eps: float = 1e-5, out: Optional[torch.Tensor] = None,
                status: Optional[torch.Tensor] = None, flags: int = 0) -> torch.Tensor:
    """One token per sequence; updates ``state`` [N,H,d,d] and ``conv_state`` [N,3,3*H*d] in
    place and returns o [N, H, d].  ``status``: a device int32 the call zeroes and sets on a
    device-side failure (read it with ``device_status``)."""
    lib = load_library()
    N, H, d = state.shape[0], state.shape[1], state.shape[2]
    shape = make_shape(N, 1, H, d, q.dtype, lower_bound, l2norm_eps, scale, negative_eigenvalues,
                       flags)
    o = out if out is not None else torch.empty((N, H, d), dtype=q.dtype, device=q.device)
    if status is None:
        og = _output_gate(out_gate, o_norm_weight, o_norm_eps)
        st = lib.kda_decode_step_gated(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                       _ptr(b), _ptr(conv_w), _ptr(A_log), _ptr(dt_bias), og,
                                       _ptr(state), _ptr(conv_state), _ptr(o), _stream(q.device))
    else:
        st = _decode_ex(lib, shape, q, k, v, alpha, b, conv_w, A_log, dt_bias, out_gate,
                        o_norm_weight, o_norm_eps, state, conv_state, o, None, status)
    _check(st, "kda_decode_step")
    return o


def _decode_ex(lib, shape, q, k, v, alpha, b, conv_w, A_log, dt_bias, out_gate, o_norm_weight,
               o_norm_eps, state, conv_state, o, step_states, status):
    og = None
    if out_gate is not None or o_norm_weight is not None:
        if out_gate is None or o_norm_weight is None:
            raise ValueError("out_gate and o_norm_weight go together")
        og = OutputGate(_ptr(out_gate), _ptr(o_norm_weight), float(o_norm_eps))
    da = DecodeArgs(*[_ptr(t) for t in (q, k, v, alpha, b, conv_w, A_log, dt_bias)],
                    ctypes.cast(ctypes.pointer(og), ctypes.c_void_p) if og is not None else None,
                    *[_ptr(t) for t in (state, conv_state, o, step_states, status)])
    return lib.kda_decode_ex(ctypes.byref(shape), ctypes.byref(da), _stream(q.device))


def kernel_timing(enable: bool) -> None:
    """Start (True) or stop (False) per-kernel event timing of the chunk path."""
    load_library().kda_kernel_timing(1 if enable else 0)


def kernel_times() -> Tuple[int, float, float]:
    """(calls, mean chunk_prep ms, mean state-pass ms) over the calls timed since the last read."""
    a, b = ctypes.c_float(0.0), ctypes.c_float(0.0)
    n = load_library().kda_kernel_times(ctypes.byref(a), ctypes.byref(b))
    if n < 0:
        raise KdaError(KDA_ERR_CUDA, "kda_kernel_times")
    return n, float(a.value), float(b.value)


def decode_multi(q, k, v, alpha, b, conv_w, A_log, dt_bias, state: torch.Tensor,
                 conv_state: torch.Tensor, *, lower_bound: float = -5.0, l2norm_eps: float = 1e-6,
                 scale: float = 1.0, negative_eigenvalues: bool = False,
                 out_gate: Optional[torch.Tensor] = None, o_norm_weight: Optional[torch.Tensor] = None,
                 o_norm_eps: float = 1e-5, step_states: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                 flags: int = 0) -> torch.Tensor:
    """T new tokens per sequence (q, k, v [N, T, H*d]; alpha [N, T, H, d]; b [N, T, H]) in one
    call; updates ``state`` and ``conv_state`` in place, fills ``step_states`` [N, T, H, d, d]
    (the state after each token) when given, and returns o [N, T, H, d].  ``status`` as in
    ``decode_step``."""
    lib = load_library()
    N, H, d = state.shape[0], state.shape[1], state.shape[2]
    T = alpha.shape[1]
    shape = make_shape(N, T, H, d, q.dtype, lower_bound, l2norm_eps, scale, negative_eigenvalues,
                       flags)
    o = out if out is not None else torch.empty((N, T, H, d), dtype=q.dtype, device=q.device)
    st = _decode_ex(lib, shape, q, k, v, alpha, b, conv_w, A_log, dt_bias, out_gate,
                    o_norm_weight, o_norm_eps, state, conv_state, o, step_states, status)
    _check(st, "kda_decode_multi")
    return o
