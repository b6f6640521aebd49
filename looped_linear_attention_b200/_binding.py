"""ctypes binding of libgdn.so: argument marshalling only.

Every compute step runs in the library's CUDA kernels; this module checks
tensor dtypes/shapes/devices, allocates outputs with torch when the caller does
not pass them, and forwards raw device pointers and the current CUDA stream.
If the library is missing the import of any entry point raises -- there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")

GDN_OK = 0
GDN_ERR_INVALID = 1
GDN_ERR_UNSUPPORTED = 2
GDN_ERR_CUDA = 3
GDN_ERR_TIMEOUT = 4
GDN_ERR_WORKSPACE = 5

GDN_F32 = 0
GDN_BF16 = 1

GDN_QK_L2NORM = 0x1
GDN_PRECISE = 0x2
GDN_SINGLE_PASS = 0x4
GDN_CHANNEL_GATE = 0x8
GDN_TEST_WAIT_TIMEOUT = 0x40000000

_DTYPES = {torch.float32: GDN_F32, torch.bfloat16: GDN_BF16}


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class gdn_fwd_params(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("a", ctypes.c_void_p), ("b", ctypes.c_void_p), ("S0", ctypes.c_void_p),
        ("o", ctypes.c_void_p), ("S_T", ctypes.c_void_p), ("cu_seqlens", ctypes.c_void_p),
        ("n_seq", ctypes.c_int), ("seq_len", ctypes.c_int), ("total_tokens", ctypes.c_int),
        ("H", ctypes.c_int), ("dk", ctypes.c_int), ("dv", ctypes.c_int),
        ("io_dtype", ctypes.c_int), ("scale", ctypes.c_float), ("flags", ctypes.c_uint),
        ("gate", ctypes.c_void_p), ("h_prev", ctypes.c_void_p), ("rho", ctypes.c_void_p),
    ]


class gdn_bwd_params(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("a", ctypes.c_void_p), ("b", ctypes.c_void_p), ("S0", ctypes.c_void_p),
        ("grad_o", ctypes.c_void_p), ("grad_S_T", ctypes.c_void_p),
        ("grad_q", ctypes.c_void_p), ("grad_k", ctypes.c_void_p), ("grad_v", ctypes.c_void_p),
        ("grad_a", ctypes.c_void_p), ("grad_b", ctypes.c_void_p), ("grad_S0", ctypes.c_void_p),
        ("cu_seqlens", ctypes.c_void_p),
        ("n_seq", ctypes.c_int), ("seq_len", ctypes.c_int), ("total_tokens", ctypes.c_int),
        ("H", ctypes.c_int), ("dk", ctypes.c_int), ("dv", ctypes.c_int),
        ("io_dtype", ctypes.c_int), ("scale", ctypes.c_float), ("flags", ctypes.c_uint),
    ]


class swa_params(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("o", ctypes.c_void_p),
        ("cu_seqlens", ctypes.c_void_p),
        ("n_seq", ctypes.c_int), ("seq_len", ctypes.c_int), ("max_seq_len", ctypes.c_int),
        ("total_tokens", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int), ("dv", ctypes.c_int),
        ("window", ctypes.c_int), ("io_dtype", ctypes.c_int), ("scale", ctypes.c_float),
    ]


_lib = None


def library() -> ctypes.CDLL:
    """The loaded libgdn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"CUDA library {LIB_PATH} is missing; build it with "
                "`python -m looped_linear_attention_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(LIB_PATH)
        vp, i32, u32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_float
        lib.gdn_chunk_fwd_workspace.argtypes = [ctypes.POINTER(gdn_fwd_params)]
        lib.gdn_chunk_fwd_workspace.restype = ctypes.c_size_t
        lib.gdn_chunk_fwd_schedule.argtypes = [ctypes.POINTER(gdn_fwd_params)] + [
            ctypes.POINTER(ctypes.c_int)] * 5
        lib.gdn_chunk_fwd_schedule.restype = i32
        lib.gdn_chunk_bwd_workspace.argtypes = [ctypes.POINTER(gdn_bwd_params)]
        lib.gdn_chunk_bwd_workspace.restype = ctypes.c_size_t
        lib.gdn_chunk_bwd.argtypes = [ctypes.POINTER(gdn_bwd_params), vp, ctypes.c_size_t, vp]
        lib.gdn_chunk_bwd.restype = i32
        lib.gdn_chunk_fwd.argtypes = [ctypes.POINTER(gdn_fwd_params), vp, ctypes.c_size_t, vp]
        lib.gdn_chunk_fwd.restype = i32
        lib.gdn_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                        f32, u32, vp]
        lib.gdn_decode_step.restype = i32
        lib.gdn_decode_step_looped.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32,
                                               i32, i32, f32, u32, vp]
        lib.gdn_decode_step_looped.restype = i32
        lib.loop_residual.argtypes = [vp, vp, vp, vp, ctypes.c_int64, i32, i32, vp]
        lib.loop_residual.restype = i32
        lib.swa_fwd.argtypes = [ctypes.POINTER(swa_params), vp]
        lib.swa_fwd.restype = i32
        lib.gdn_status_string.argtypes = [i32]
        lib.gdn_status_string.restype = ctypes.c_char_p
        lib.gdn_get_device_status.argtypes = [vp]
        lib.gdn_get_device_status.restype = i32
        lib.gdn_version.argtypes = []
        lib.gdn_version.restype = i32
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return library().gdn_status_string(int(status)).decode()


def _stream_ptr(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _check_epilogue(gate, h_prev, rho, T, H, dv, dtype):
    if gate is not None:
        _check(gate, "gate", torch.float32, (T, H))
    if (h_prev is None) != (rho is None):
        raise ValueError("h_prev and rho come together (the loop residual)")
    if h_prev is not None:
        _check(h_prev, "h_prev", dtype)
        if h_prev.numel() != T * H * dv:
            raise ValueError(f"h_prev must hold {T} x {H * dv} elements")
        _check(rho, "rho", torch.float32, (H * dv,))


def gdn_chunk_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, a: torch.Tensor,
                  b: torch.Tensor, S0: Optional[torch.Tensor] = None,
                  cu_seqlens: Optional[torch.Tensor] = None, *, n_seq: Optional[int] = None,
                  scale: float = 1.0, flags: int = 0, o: Optional[torch.Tensor] = None,
                  S_T: Optional[torch.Tensor] = None, return_state: bool = True,
                  gate: Optional[torch.Tensor] = None, h_prev: Optional[torch.Tensor] = None,
                  rho: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None):
    """Chunkwise prefill (see gdn_chunk_fwd in include/gdn.h).

    q, k: [T, H, dk]; v: [T, H, dv] (fp32 or bf16); a, b: [T, H] fp32;
    S0: [n_seq, H, dk, dv] fp32 or None; cu_seqlens: int32 [n_seq+1] on the device,
    or None with n_seq sequences of T // n_seq tokens (n_seq defaults to 1).
    Looped-block epilogue: gate [T, H] fp32 output-gate logits; h_prev (T x H*dv,
    io dtype) with rho [H*dv] fp32 adds the loop residual (o may be h_prev's storage).
    Returns (o, S_T) (S_T is None when return_state is False)."""
    if q.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {q.dtype}")
    T, H, dk = q.shape
    dv = v.shape[2]
    _check(q, "q", q.dtype)
    _check(k, "k", q.dtype, (T, H, dk))
    _check(v, "v", q.dtype, (T, H, dv))
    _check(a, "a", torch.float32, (T, H, dk) if flags & GDN_CHANNEL_GATE else (T, H))
    _check(b, "b", torch.float32, (T, H))
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32)
        ns = cu_seqlens.numel() - 1
        seq_len = 0
    else:
        ns = 1 if n_seq is None else int(n_seq)
        if ns <= 0 or T % ns != 0:
            raise ValueError("without cu_seqlens, the token count must be n_seq * seq_len")
        seq_len = T // ns
    if S0 is not None:
        _check(S0, "S0", torch.float32, (ns, H, dk, dv))
    _check_epilogue(gate, h_prev, rho, T, H, dv, q.dtype)
    if o is None:
        o = torch.empty(T, H, dv, dtype=q.dtype, device=q.device)
    else:
        _check(o, "o", q.dtype)
        if o.numel() != T * H * dv:
            raise ValueError(f"o must hold {T} x {H} x {dv} elements")
    if S_T is None and return_state:
        S_T = torch.empty(ns, H, dk, dv, dtype=torch.float32, device=q.device)
    elif S_T is not None:
        _check(S_T, "S_T", torch.float32, (ns, H, dk, dv))
    p = gdn_fwd_params(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(S0), _ptr(o),
                       _ptr(S_T), _ptr(cu_seqlens), ns, seq_len, T, H, dk, dv,
                       _DTYPES[q.dtype], float(scale), int(flags), _ptr(gate), _ptr(h_prev),
                       _ptr(rho))
    lib = library()
    ws = lib.gdn_chunk_fwd_workspace(ctypes.byref(p))
    if ws == ctypes.c_size_t(-1).value:
        raise GdnError(GDN_ERR_INVALID, "gdn_chunk_fwd")
    work = torch.empty(ws, dtype=torch.uint8, device=q.device) if ws else None
    if work is not None and stream is not None:
        work.record_stream(stream)
    st = lib.gdn_chunk_fwd(ctypes.byref(p), _ptr(work), ctypes.c_size_t(ws), _stream_ptr(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_chunk_fwd")
    return o, S_T


def gdn_chunk_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, a: torch.Tensor,
                  b: torch.Tensor, grad_o: torch.Tensor, S0: Optional[torch.Tensor] = None,
                  grad_S_T: Optional[torch.Tensor] = None, cu_seqlens: Optional[torch.Tensor] = None,
                  *, n_seq: Optional[int] = None, scale: float = 1.0, want_grad_S0: bool = True,
                  flags: int = 0, stream: Optional[torch.cuda.Stream] = None) -> dict:
    """Reverse mode of gdn_chunk_fwd (see gdn_chunk_bwd in include/gdn.h).

    Inputs as gdn_chunk_fwd plus grad_o [T, H, dv] (io dtype) and grad_S_T
    [n_seq, H, dk, dv] fp32 (or None).  Returns fp32 gradients
    {"q", "k", "v", "a", "b", "S0"} ("S0" None unless want_grad_S0).
    flags: 0 (the chunkwise path) or GDN_PRECISE (token by token)."""
    if q.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {q.dtype}")
    T, H, dk = q.shape
    dv = v.shape[2]
    _check(q, "q", q.dtype)
    _check(k, "k", q.dtype, (T, H, dk))
    _check(v, "v", q.dtype, (T, H, dv))
    _check(grad_o, "grad_o", q.dtype, (T, H, dv))
    _check(a, "a", torch.float32, (T, H))
    _check(b, "b", torch.float32, (T, H))
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32)
        ns, seq_len = cu_seqlens.numel() - 1, 0
    else:
        ns = 1 if n_seq is None else int(n_seq)
        if ns <= 0 or T % ns != 0:
            raise ValueError("without cu_seqlens, the token count must be n_seq * seq_len")
        seq_len = T // ns
    if S0 is not None:
        _check(S0, "S0", torch.float32, (ns, H, dk, dv))
    if grad_S_T is not None:
        _check(grad_S_T, "grad_S_T", torch.float32, (ns, H, dk, dv))
    f32 = dict(dtype=torch.float32, device=q.device)
    g = {"q": torch.empty(T, H, dk, **f32), "k": torch.empty(T, H, dk, **f32),
         "v": torch.empty(T, H, dv, **f32), "a": torch.empty(T, H, **f32), "b": torch.empty(T, H, **f32),
         "S0": torch.empty(ns, H, dk, dv, **f32) if want_grad_S0 else None}
    p = gdn_bwd_params(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(S0), _ptr(grad_o),
                       _ptr(grad_S_T), _ptr(g["q"]), _ptr(g["k"]), _ptr(g["v"]), _ptr(g["a"]),
                       _ptr(g["b"]), _ptr(g["S0"]), _ptr(cu_seqlens), ns, seq_len, T, H, dk, dv,
                       _DTYPES[q.dtype], float(scale), int(flags))
    lib = library()
    ws = lib.gdn_chunk_bwd_workspace(ctypes.byref(p))
    if ws == ctypes.c_size_t(-1).value:
        raise GdnError(GDN_ERR_INVALID, "gdn_chunk_bwd")
    work = torch.empty(ws, dtype=torch.uint8, device=q.device) if ws else None
    if work is not None and stream is not None:
        work.record_stream(stream)
    st = lib.gdn_chunk_bwd(ctypes.byref(p), _ptr(work), ctypes.c_size_t(ws), _stream_ptr(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_chunk_bwd")
    return g


def _shape_params(n_seq, seq_len, H, dk, dv, dtype, flags, varlen):
    T = n_seq * seq_len
    fake = 1 << 40          # aligned placeholders: the queries only read shapes and flags
    return gdn_fwd_params(fake, fake + (1 << 36), fake + (2 << 36), fake + (3 << 36),
                          fake + (4 << 36), None, fake + (5 << 36), None,
                          fake + (6 << 36) if varlen else None, n_seq, 0 if varlen else seq_len, T,
                          H, dk, dv, _DTYPES[dtype], 1.0, int(flags))


def prefill_workspace_bytes(n_seq: int, seq_len: int, H: int, dk: int, dv: int,
                            dtype: torch.dtype = torch.bfloat16, flags: int = 0,
                            varlen: bool = False) -> int:
    """gdn_chunk_fwd_workspace for a call of this shape (no device memory is
    touched).  Non-zero means the segmented schedule."""
    p = _shape_params(n_seq, seq_len, H, dk, dv, dtype, flags, varlen)
    ws = library().gdn_chunk_fwd_workspace(ctypes.byref(p))
    if ws == ctypes.c_size_t(-1).value:
        raise GdnError(GDN_ERR_INVALID, "gdn_chunk_fwd_workspace")
    return int(ws)


def prefill_schedule(n_seq: int, seq_len: int, H: int, dk: int, dv: int,
                     dtype: torch.dtype = torch.bfloat16, flags: int = 0,
                     varlen: bool = False, with_state: bool = True,
                     residual_in_place: bool = False) -> dict:
    """gdn_chunk_fwd_schedule for a call of this shape, given its workspace:
    {"n_segs", "seg0_tok", "seg_tok", "launches", "corrected"} (n_segs = 1: one
    pass per chain).  with_state: the call writes S_T; residual_in_place: o is
    the loop residual's h_prev itself."""
    p = _shape_params(n_seq, seq_len, H, dk, dv, dtype, flags, varlen)
    if with_state:
        p.S_T = (1 << 40) + (8 << 36)
    if residual_in_place:
        p.h_prev, p.rho = p.o, (1 << 40) + (9 << 36)
    n, tok0, tok, launches, corr = (ctypes.c_int() for _ in range(5))
    st = library().gdn_chunk_fwd_schedule(ctypes.byref(p), ctypes.byref(n), ctypes.byref(tok0),
                                          ctypes.byref(tok), ctypes.byref(launches), ctypes.byref(corr))
    if st != GDN_OK:
        raise GdnError(st, "gdn_chunk_fwd_schedule")
    return {"n_segs": n.value, "seg0_tok": tok0.value, "seg_tok": tok.value,
            "launches": launches.value, "corrected": corr.value}


def gdn_decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, a: torch.Tensor,
                    b: torch.Tensor, S: torch.Tensor, *, scale: float = 1.0, flags: int = 0,
                    o: Optional[torch.Tensor] = None, gate: Optional[torch.Tensor] = None,
                    h_prev: Optional[torch.Tensor] = None, rho: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """One token per slot; S [N, H, dk, dv] fp32 is updated in place. Returns o [N, H, dv].
    gate / h_prev / rho: the looped-block epilogue (gdn_decode_step_looped)."""
    if q.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {q.dtype}")
    N, H, dk = q.shape
    dv = v.shape[2]
    _check(q, "q", q.dtype)
    _check(k, "k", q.dtype, (N, H, dk))
    _check(v, "v", q.dtype, (N, H, dv))
    _check(a, "a", torch.float32, (N, H, dk) if flags & GDN_CHANNEL_GATE else (N, H))
    _check(b, "b", torch.float32, (N, H))
    _check(S, "S", torch.float32, (N, H, dk, dv))
    _check_epilogue(gate, h_prev, rho, N, H, dv, q.dtype)
    if o is None:
        o = torch.empty(N, H, dv, dtype=q.dtype, device=q.device)
    else:
        _check(o, "o", q.dtype)
        if o.numel() != N * H * dv:
            raise ValueError(f"o must hold {N} x {H} x {dv} elements")
    if gate is None and h_prev is None:
        st = library().gdn_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(S), _ptr(o),
                                       N, H, dk, dv, _DTYPES[q.dtype], float(scale), int(flags),
                                       _stream_ptr(stream))
    else:
        st = library().gdn_decode_step_looped(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(S),
                                              _ptr(o), _ptr(gate), _ptr(h_prev), _ptr(rho), N, H, dk,
                                              dv, _DTYPES[q.dtype], float(scale), int(flags),
                                              _stream_ptr(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_decode_step")
    return o


def loop_residual(h_tilde: torch.Tensor, h_prev: torch.Tensor, rho: torch.Tensor,
                  out: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """h = h_tilde + rho (.) h_prev over the last dimension; out may alias an input."""
    if h_tilde.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {h_tilde.dtype}")
    d = h_tilde.shape[-1]
    rows = h_tilde.numel() // d if d else 0
    _check(h_tilde, "h_tilde", h_tilde.dtype)
    _check(h_prev, "h_prev", h_tilde.dtype, h_tilde.shape)
    _check(rho, "rho", torch.float32, (d,))
    if out is None:
        out = torch.empty_like(h_tilde)
    else:
        _check(out, "out", h_tilde.dtype, h_tilde.shape)
    st = library().loop_residual(_ptr(h_tilde), _ptr(h_prev), _ptr(rho), _ptr(out), rows, d,
                                 _DTYPES[h_tilde.dtype], _stream_ptr(stream))
    if st != GDN_OK:
        raise GdnError(st, "loop_residual")
    return out


def swa_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, window: int,
            cu_seqlens: Optional[torch.Tensor] = None, *, n_seq: Optional[int] = None,
            max_seq_len: Optional[int] = None, scale: Optional[float] = None,
            o: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Sliding-window causal softmax attention (see swa_fwd in include/gdn.h).

    q, k: [T, H, d]; v: [T, H, dv] bf16; cu_seqlens int32 [n_seq+1] on the
    device with max_seq_len (defaults to T), or None with n_seq sequences of
    T // n_seq tokens; scale defaults to 1/sqrt(d). Returns o [T, H, dv]."""
    T, H, d = q.shape
    dv = v.shape[2]
    _check(q, "q", torch.bfloat16)
    _check(k, "k", torch.bfloat16, (T, H, d))
    _check(v, "v", torch.bfloat16, (T, H, dv))
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32)
        ns, seq_len = cu_seqlens.numel() - 1, 0
        msl = T if max_seq_len is None else int(max_seq_len)
    else:
        ns = 1 if n_seq is None else int(n_seq)
        if ns <= 0 or T % ns != 0:
            raise ValueError("without cu_seqlens, the token count must be n_seq * seq_len")
        seq_len, msl = T // ns, T // ns
    if o is None:
        o = torch.empty(T, H, dv, dtype=q.dtype, device=q.device)
    else:
        _check(o, "o", q.dtype, (T, H, dv))
    sc = float(d) ** -0.5 if scale is None else float(scale)
    p = swa_params(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(cu_seqlens), ns, seq_len, msl, T, H, d, dv,
                   int(window), GDN_BF16, sc)
    st = library().swa_fwd(ctypes.byref(p), _stream_ptr(stream))
    if st != GDN_OK:
        raise GdnError(st, "swa_fwd")
    return o


def gdn_get_device_status(stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronises the stream and returns/clears the device status word."""
    return int(library().gdn_get_device_status(_stream_ptr(stream)))


def version() -> int:
    return int(library().gdn_version())
