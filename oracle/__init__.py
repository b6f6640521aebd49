"""Plain CPU oracle for the looped gated delta-rule (GDN) mixer.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  The library
package never imports it, and it imports nothing from the library: the two
share no code.

Every function works in float64 on host arrays and follows the definition on
the page, not any kernel's blocking:

* ``gdn_bwd`` -- reverse mode of ``gdn_fwd`` (gradients through the outputs
  and the final states), token by token backwards over stored forward states.
* ``gdn_fwd`` / ``gdn_decode`` -- the gated delta rule, token by token
  ("LT2: Linear-Time Looped Transformers", §2, "LT2." paragraph: state
  S_t in R^{dk x dv}; the mixer is Gated DeltaNet, Appendix C).  The per-token
  loop is the C routine in ``gdn_oracle.c``.
* ``kda_fwd`` / ``kda_decode`` -- the per-channel (diagonal) gate variant, the
  KDA mixer of the LT2 mixer list (Appendix C), token by token.
* ``swa_fwd`` -- sliding-window causal softmax attention, the window mixer
  of the hybrid loops (§2, Appendix C), one query at a time.
* ``output_gate`` -- the head-wise sigmoid output gate (§3, gated-attention
  paragraph).
* ``loop_residual`` -- h = h_tilde + rho (.) h_prev (same paragraph).
* ``qk_l2norm`` -- per-head L2 normalisation of q and k, x / sqrt(sum x^2 + eps),
  the input recipe of the looped workloads (the pages do not print it; eps is
  this library's choice, 1e-6).
* ``looped_forward`` -- T applications of projection -> GDN -> loop residual
  for the looped-prefill workload, with bf16 rounding only where that
  workload's tensors are bf16 (projection outputs, mixer output, loop state).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

QK_NORM_EPS = 1e-6


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into liboracle.so next to it (gcc, OpenMP, IEEE)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
               "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        lib.oracle_gdn_fwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, ip,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_double]
        lib.oracle_gdn_fwd.restype = ctypes.c_int
        lib.oracle_gdn_bwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, ip,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_double,
                                       dp, dp, dp, dp, dp, dp]
        lib.oracle_gdn_bwd.restype = ctypes.c_int
        lib.oracle_gdn_decode.argtypes = [dp, dp, dp, dp, dp, dp, dp,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_double]
        lib.oracle_gdn_decode.restype = ctypes.c_int
        lib.oracle_kda_fwd.argtypes = lib.oracle_gdn_fwd.argtypes
        lib.oracle_kda_fwd.restype = ctypes.c_int
        lib.oracle_kda_decode.argtypes = lib.oracle_gdn_decode.argtypes
        lib.oracle_kda_decode.restype = ctypes.c_int
        lib.oracle_swa_fwd.argtypes = [dp, dp, dp, dp, ip, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double]
        lib.oracle_swa_fwd.restype = ctypes.c_int
        lib.oracle_loop_residual.argtypes = [dp, dp, dp, dp, ctypes.c_long, ctypes.c_int]
        lib.oracle_loop_residual.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Host float64 copy of a numpy array or a CPU torch tensor (any float dtype)."""
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(x: np.ndarray, ctype=ctypes.c_double):
    return x.ctypes.data_as(ctypes.POINTER(ctype))


def num_threads() -> int:
    """OpenMP threads the oracle runs with (the CPU-baseline core count)."""
    return int(_load().oracle_num_threads())


def sigmoid(z):
    """1 / (1 + e^-z) in float64, computed from e^-|z| so that no step overflows."""
    z = _f64(z)
    e = np.exp(-np.abs(z))
    return np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def output_gate(o, gate):
    """Head-wise sigmoid output gate ("LT2: Linear-Time Looped Transformers",
    §3, the gated-attention paragraph: a head-specific sigmoid gate after the
    mixer).  o [n_tok, H, dv] times sigmoid(gate) [n_tok, H], one factor per
    token and head; the recurrence's state is not touched."""
    return _f64(o) * sigmoid(gate)[..., None]


def gdn_fwd(q, k, v, a, b, S0=None, cu_seqlens=None, scale: float = 1.0, gate=None):
    """Gated delta rule over packed sequences.

    q, k: [n_tok, H, dk]; v: [n_tok, H, dv]; a, b: [n_tok, H];
    S0: [n_seq, H, dk, dv] or None (zeros); cu_seqlens: int [n_seq+1] or None
    (one sequence of n_tok tokens); gate: [n_tok, H] logits of the head-wise
    output gate, or None.  Returns (o [n_tok, H, dv], S_T [n_seq, H, dk, dv]).
    """
    q, k, v, a, b = (_f64(t) for t in (q, k, v, a, b))
    n_tok, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is None:
        cu = np.array([0, n_tok], dtype=np.int32)
    else:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
            dtype=np.int32))
    n_seq = cu.shape[0] - 1
    if int(cu[-1]) > n_tok or int(cu[0]) < 0:
        raise ValueError("cu_seqlens out of range")
    s0 = None if S0 is None else _f64(S0)
    o = np.zeros((n_tok, H, dv))
    ST = np.zeros((n_seq, H, dk, dv))
    rc = _load().oracle_gdn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b),
        None if s0 is None else _ptr(s0), _ptr(o), _ptr(ST),
        _ptr(cu, ctypes.c_int32), n_seq, H, dk, dv, float(scale))
    if rc != 0:
        raise ValueError("oracle_gdn_fwd rejected its arguments")
    if gate is not None:
        o = output_gate(o, gate)
    return o, ST


def gdn_bwd(q, k, v, a, b, dO, S0=None, dST=None, cu_seqlens=None, scale: float = 1.0):
    """Reverse mode of ``gdn_fwd``: gradients of a loss through its outputs
    (dO [n_tok, H, dv]) and final states (dST [n_seq, H, dk, dv] or None).
    Returns a dict of float64 arrays dq, dk, dv, da, db, dS0 (the gradient
    with respect to the start states, zeros-start included)."""
    q, k, v, a, b, dO = (_f64(t) for t in (q, k, v, a, b, dO))
    n_tok, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is None:
        cu = np.array([0, n_tok], dtype=np.int32)
    else:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
            dtype=np.int32))
    n_seq = cu.shape[0] - 1
    if int(cu[-1]) > n_tok or int(cu[0]) < 0:
        raise ValueError("cu_seqlens out of range")
    s0 = None if S0 is None else _f64(S0)
    dst = None if dST is None else _f64(dST)
    out = dict(dq=np.zeros((n_tok, H, dk)), dk=np.zeros((n_tok, H, dk)), dv=np.zeros((n_tok, H, dv)),
               da=np.zeros((n_tok, H)), db=np.zeros((n_tok, H)), dS0=np.zeros((n_seq, H, dk, dv)))
    rc = _load().oracle_gdn_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), None if s0 is None else _ptr(s0),
        _ptr(dO), None if dst is None else _ptr(dst), _ptr(cu, ctypes.c_int32),
        n_seq, H, dk, dv, float(scale),
        _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["da"]), _ptr(out["db"]),
        _ptr(out["dS0"]))
    if rc != 0:
        raise ValueError("oracle_gdn_bwd rejected its arguments")
    return out


def gdn_decode(q, k, v, a, b, S, scale: float = 1.0, gate=None):
    """One token per slot.  q, k: [N, H, dk]; v: [N, H, dv]; a, b: [N, H];
    S: [N, H, dk, dv]; gate: [N, H] output-gate logits or None.
    Returns (o [N, H, dv], S_new); the input is not modified."""
    q, k, v, a, b = (_f64(t) for t in (q, k, v, a, b))
    S = _f64(S).copy()
    N, H, dk = q.shape
    dv = v.shape[2]
    o = np.zeros((N, H, dv))
    rc = _load().oracle_gdn_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b),
                                   _ptr(S), _ptr(o), N, H, dk, dv, float(scale))
    if rc != 0:
        raise ValueError("oracle_gdn_decode rejected its arguments")
    if gate is not None:
        o = output_gate(o, gate)
    return o, S


def kda_fwd(q, k, v, a, b, S0=None, cu_seqlens=None, scale: float = 1.0, gate=None):
    """Per-channel (diagonal) gate variant, the KDA mixer of the LT2 mixer list
    ("LT2: Linear-Time Looped Transformers", Appendix C; the pages print no
    update rule, the reading is written out in ``gdn_oracle.c``):
    Sigma_t = (I - b_t k_t k_t^T) Diag(a_t) Sigma_{t-1} + b_t k_t v_t^T,
    o_t = scale Sigma_t^T q_t.  As ``gdn_fwd``, with a [n_tok, H, dk]."""
    q, k, v, a, b = (_f64(t) for t in (q, k, v, a, b))
    n_tok, H, dk = q.shape
    dv = v.shape[2]
    if a.shape != (n_tok, H, dk):
        raise ValueError("a must be [n_tok, H, dk]")
    if cu_seqlens is None:
        cu = np.array([0, n_tok], dtype=np.int32)
    else:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
            dtype=np.int32))
    n_seq = cu.shape[0] - 1
    if int(cu[-1]) > n_tok or int(cu[0]) < 0:
        raise ValueError("cu_seqlens out of range")
    s0 = None if S0 is None else _f64(S0)
    o = np.zeros((n_tok, H, dv))
    ST = np.zeros((n_seq, H, dk, dv))
    rc = _load().oracle_kda_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b),
        None if s0 is None else _ptr(s0), _ptr(o), _ptr(ST),
        _ptr(cu, ctypes.c_int32), n_seq, H, dk, dv, float(scale))
    if rc != 0:
        raise ValueError("oracle_kda_fwd rejected its arguments")
    if gate is not None:
        o = output_gate(o, gate)
    return o, ST


def kda_decode(q, k, v, a, b, S, scale: float = 1.0, gate=None):
    """One token per slot of the per-channel gate variant (a [N, H, dk]).
    Returns (o [N, H, dv], S_new); the input is not modified."""
    q, k, v, a, b = (_f64(t) for t in (q, k, v, a, b))
    S = _f64(S).copy()
    N, H, dk = q.shape
    dv = v.shape[2]
    if a.shape != (N, H, dk):
        raise ValueError("a must be [N, H, dk]")
    o = np.zeros((N, H, dv))
    rc = _load().oracle_kda_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b),
                                   _ptr(S), _ptr(o), N, H, dk, dv, float(scale))
    if rc != 0:
        raise ValueError("oracle_kda_decode rejected its arguments")
    if gate is not None:
        o = output_gate(o, gate)
    return o, S


def swa_fwd(q, k, v, window: int, cu_seqlens=None, scale=None):
    """Sliding-window causal softmax attention ("LT2: Linear-Time Looped
    Transformers", §2 and Appendix C): query t attends to the keys
    [t - window + 1, t] of its own sequence.  q, k [n_tok, H, d], v [n_tok, H, dv];
    scale defaults to 1 / sqrt(d).  Returns o [n_tok, H, dv]."""
    q, k, v = (_f64(t) for t in (q, k, v))
    n_tok, H, d = q.shape
    dv = v.shape[2]
    if cu_seqlens is None:
        cu = np.array([0, n_tok], dtype=np.int32)
    else:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
            dtype=np.int32))
    if int(cu[-1]) > n_tok or int(cu[0]) < 0:
        raise ValueError("cu_seqlens out of range")
    sc = 1.0 / np.sqrt(d) if scale is None else float(scale)
    o = np.zeros((n_tok, H, dv))
    rc = _load().oracle_swa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(cu, ctypes.c_int32),
                                cu.shape[0] - 1, H, d, dv, int(window), sc)
    if rc != 0:
        raise ValueError("oracle_swa_fwd rejected its arguments")
    return o


def loop_residual(h_tilde, h_prev, rho):
    """h = h_tilde + rho (.) h_prev in float64; h_* [rows, d], rho [d]."""
    ht, hp, r = _f64(h_tilde), _f64(h_prev), _f64(rho)
    rows, d = ht.shape
    out = np.empty_like(ht)
    rc = _load().oracle_loop_residual(_ptr(ht), _ptr(hp), _ptr(r), _ptr(out), rows, d)
    if rc != 0:
        raise ValueError("oracle_loop_residual rejected its arguments")
    return out


def qk_l2norm(x, eps: float = QK_NORM_EPS):
    """x / sqrt(sum(x^2) + eps) over the last axis (one head's vector)."""
    x = _f64(x)
    return x / np.sqrt((x * x).sum(axis=-1, keepdims=True) + eps)


def round_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), back to float64."""
    import torch
    t = torch.from_numpy(_f64(x))
    return t.to(torch.bfloat16).double().numpy()


def looped_forward(h0, Wq, Wk, Wv, a, b, rho, H: int, dk: int, dv: int,
                   scale: float = 1.0, return_all: bool = False, Wg=None):
    """T loops of the looped-prefill workload on one sequence.

    Per loop tau ("LT2: Linear-Time Looped Transformers", §2, "LT2." paragraph):
    q, k, v = h^(tau-1) W_{q,k,v} (rounded to bf16, the workload's tensor type);
    q, k L2-normalised per head; o = GDN(q, k, v, a_tau, b_tau) from a zero
    state; with the gated variant (§3, gated-attention paragraph) o is scaled
    per head by sigmoid(h^(tau-1) W_g), W_g [d, H], the logits taken in fp32
    from the bf16 state; h~^(tau) = o as [L, H*dv] (rounded to bf16);
    h^(tau) = h~^(tau) + rho_tau (.) h^(tau-1) (rounded to bf16).
    a, b: [T, L, H]; rho: [T, H*dv].  Returns h^(T) (and every h^(tau) if asked).
    """
    h = _f64(h0)
    Wq, Wk, Wv = _f64(Wq), _f64(Wk), _f64(Wv)
    a, b, rho = _f64(a), _f64(b), _f64(rho)
    L = h.shape[0]
    outs = []
    for tau in range(a.shape[0]):
        q = round_bf16(h @ Wq).reshape(L, H, dk)
        k = round_bf16(h @ Wk).reshape(L, H, dk)
        v = round_bf16(h @ Wv).reshape(L, H, dv)
        q, k = qk_l2norm(q), qk_l2norm(k)
        z = None if Wg is None else (h @ _f64(Wg)).astype(np.float32).astype(np.float64)
        o, _ = gdn_fwd(q, k, v, a[tau], b[tau], None, None, scale, gate=z)
        h_tilde = round_bf16(o.reshape(L, H * dv))
        h = round_bf16(loop_residual(h_tilde, h, rho[tau]))
        outs.append(h)
    return outs if return_all else h
