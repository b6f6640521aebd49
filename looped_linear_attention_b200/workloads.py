"""Seeded synthetic inputs for the looped GDN mixer.

This module holds shapes, distributions and seeds only -- none of the mixer's
arithmetic -- so that the test suite's oracle side and the CUDA side can draw
the very same inputs.  It imports nothing else from this package.

Workloads (the shapes of the LT2 efficiency sweep, "LT2: Linear-Time Looped
Transformers", §3.2: 1k-32k tokens, batch 1-8, T = 4 loops; d = 2048 with 16
heads at the 1.3B scale, Appendix C; seed 42 for initialisation, Appendix C):

  tiny            B=1, H=2, L=256, dk=dv=64, T=1, fp32
  looped_prefill  B=1, H=16, L=4096, dk=dv=128, T=4, h [4096, 2048] bf16,
                  W_q, W_k, W_v [2048, 2048] ~ N(0, variance 1/2048) in bf16,
                  rho_tau ~ U(0, 0.5) per channel, fresh a, b per loop
  long_prefill    B=8, H=16, L=16384, dk=dv=128, bf16, zero S0, T=4
  decode          24576 slots (256 sequences x 24 layers x 4 loops), H=16,
                  dk=dv=128, fp32 state ~ N(0, std 0.02), one bf16 token per slot
  varlen          64 sequences, lengths ~ U[512, 32768], H=16, dk=128, dv=256,
                  bf16, per-sequence S0 ~ N(0, std 0.02), T=4

Gates: a = exp(-softplus(x)), x ~ N(-3, 1) (a in (0, 1)); b = sigmoid(N(0, 1)).
q and k are N(0, 1) and, where the workload says so, L2-normalised per head
(x / sqrt(sum x^2 + 1e-6), in fp32) before the cast to the io dtype.
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import Optional

import numpy as np
import torch

BASE_SEED = 42
QK_NORM_EPS = 1e-6


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n_seq: int
    H: int
    seq_len: int            # fixed length (0 for varlen)
    dk: int
    dv: int
    loops: int
    dtype: torch.dtype
    normalize_qk: bool
    random_s0: bool
    varlen: bool = False
    min_len: int = 0
    max_len: int = 0


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 256, 64, 64, 1, torch.float32, True, False),
    "looped_prefill": Workload("looped_prefill", 1, 16, 4096, 128, 128, 4,
                               torch.bfloat16, True, False),
    "long_prefill": Workload("long_prefill", 8, 16, 16384, 128, 128, 4,
                             torch.bfloat16, True, False),
    "decode": Workload("decode", 256 * 24 * 4, 16, 1, 128, 128, 1,
                       torch.bfloat16, True, True),
    "varlen": Workload("varlen", 64, 16, 0, 128, 256, 4, torch.bfloat16, True, True,
                       varlen=True, min_len=512, max_len=32768),
}

MODEL_DIM = 2048          # d of the looped-prefill workload (16 heads x 128)


def seed_for(*parts) -> int:
    """Stable 63-bit seed from the base seed and any labels (workload, loop,
    sequence, tensor name ...)."""
    key = "/".join(str(p) for p in (BASE_SEED,) + parts).encode()
    return (zlib.crc32(key) << 31 ^ zlib.adler32(key)) & ((1 << 63) - 1)


def _gen(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed_for(*parts))
    return g


def varlen_lengths(wl: Workload, n_seq: Optional[int] = None) -> np.ndarray:
    """Sequence lengths ~ U[min_len, max_len] (integers, inclusive), seeded."""
    n = wl.n_seq if n_seq is None else n_seq
    rng = np.random.default_rng(seed_for(wl.name, "lengths"))
    return rng.integers(wl.min_len, wl.max_len + 1, size=n).astype(np.int64)


def cu_seqlens_from_lengths(lengths) -> np.ndarray:
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu


def _l2norm(x: torch.Tensor) -> torch.Tensor:
    return x / torch.sqrt((x * x).sum(-1, keepdim=True) + QK_NORM_EPS)


def gates(n_tok: int, H: int, device, *parts, dtype=torch.float32):
    """a = exp(-softplus(N(-3, 1))), b = sigmoid(N(0, 1)), both [n_tok, H] fp32."""
    g = _gen(device, *parts, "gates")
    x = torch.randn(n_tok, H, generator=g, device=device, dtype=torch.float32) - 3.0
    # stable softplus: max(x, 0) + log1p(exp(-|x|))
    sp = torch.clamp(x, min=0) + torch.log1p(torch.exp(-x.abs()))
    a = torch.exp(-sp)
    b = torch.sigmoid(torch.randn(n_tok, H, generator=g, device=device,
                                  dtype=torch.float32))
    return a.to(dtype), b.to(dtype)


def channel_gates(n_tok: int, H: int, dk: int, device, *parts):
    """Per-channel decay a [n_tok, H, dk] = exp(-softplus(N(-3, 1))) drawn for
    every channel (the scalar gate's distribution, one draw per channel) and
    b = sigmoid(N(0, 1)) [n_tok, H], for the per-channel (KDA) variant."""
    g = _gen(device, *parts, "channel-gates")
    x = torch.randn(n_tok, H, dk, generator=g, device=device, dtype=torch.float32) - 3.0
    sp = torch.clamp(x, min=0) + torch.log1p(torch.exp(-x.abs()))
    a = torch.exp(-sp)
    b = torch.sigmoid(torch.randn(n_tok, H, generator=g, device=device, dtype=torch.float32))
    return a, b


def qkv(n_tok: int, H: int, dk: int, dv: int, dtype, normalize: bool, device,
        *parts, chunk_tokens: int = 1 << 16):
    """q, k [n_tok, H, dk] and v [n_tok, H, dv] in `dtype` (drawn in fp32,
    normalised if asked, then cast).  Drawn in token blocks to bound memory."""
    q = torch.empty(n_tok, H, dk, dtype=dtype, device=device)
    k = torch.empty(n_tok, H, dk, dtype=dtype, device=device)
    v = torch.empty(n_tok, H, dv, dtype=dtype, device=device)
    g = _gen(device, *parts, "qkv")
    for t0 in range(0, n_tok, chunk_tokens):
        t1 = min(n_tok, t0 + chunk_tokens)
        n = t1 - t0
        qq = torch.randn(n, H, dk, generator=g, device=device, dtype=torch.float32)
        kk = torch.randn(n, H, dk, generator=g, device=device, dtype=torch.float32)
        vv = torch.randn(n, H, dv, generator=g, device=device, dtype=torch.float32)
        if normalize:
            qq, kk = _l2norm(qq), _l2norm(kk)
        q[t0:t1] = qq.to(dtype)
        k[t0:t1] = kk.to(dtype)
        v[t0:t1] = vv.to(dtype)
    return q, k, v


def state(n: int, H: int, dk: int, dv: int, device, *parts, std: float = 0.02):
    """fp32 state [n, H, dk, dv] ~ N(0, std^2)."""
    g = _gen(device, *parts, "state")
    out = torch.empty(n, H, dk, dv, dtype=torch.float32, device=device)
    step = max(1, (1 << 26) // (H * dk * dv))
    for i in range(0, n, step):
        j = min(n, i + step)
        out[i:j] = torch.randn(j - i, H, dk, dv, generator=g, device=device,
                               dtype=torch.float32) * std
    return out


def prefill_inputs(wl: Workload, device="cpu", loop: int = 0, n_seq=None,
                   seq_len=None, lengths=None):
    """Inputs of one prefill call of workload `wl` (optionally resized).

    Returns a dict with q, k, v, a, b, S0 (or None), cu_seqlens (host int32 numpy
    array, or None for fixed-length), n_seq, seq_len, total_tokens."""
    n_seq = wl.n_seq if n_seq is None else n_seq
    if wl.varlen or lengths is not None:
        lens = varlen_lengths(wl, n_seq) if lengths is None else np.asarray(lengths)
        cu = cu_seqlens_from_lengths(lens)
        n_seq = len(lens)
        total = int(cu[-1])
        L = 0
    else:
        L = wl.seq_len if seq_len is None else seq_len
        cu = None
        total = n_seq * L
    q, k, v = qkv(total, wl.H, wl.dk, wl.dv, wl.dtype, wl.normalize_qk, device,
                  wl.name, loop)
    a, b = gates(total, wl.H, device, wl.name, loop)
    S0 = state(n_seq, wl.H, wl.dk, wl.dv, device, wl.name, loop) if wl.random_s0 else None
    return dict(q=q, k=k, v=v, a=a, b=b, S0=S0, cu_seqlens=cu, n_seq=n_seq,
                seq_len=L, total_tokens=total)


def decode_inputs(wl: Workload, device="cpu", n_slots=None, step: int = 0):
    """One decode step: q, k, v [N, H, d*] (io dtype), a, b [N, H], S [N, H, dk, dv]."""
    N = wl.n_seq if n_slots is None else n_slots
    q, k, v = qkv(N, wl.H, wl.dk, wl.dv, wl.dtype, wl.normalize_qk, device,
                  wl.name, "step", step)
    a, b = gates(N, wl.H, device, wl.name, "step", step)
    S = state(N, wl.H, wl.dk, wl.dv, device, wl.name)
    return dict(q=q, k=k, v=v, a=a, b=b, S=S, N=N)


def looped_inputs(wl: Workload, device="cpu", seq_len=None, d_model=None):
    """Looped-prefill workload: h0 [L, d] bf16, W_q/W_k/W_v [d, d] bf16 with
    N(0, variance 1/d) entries (the three planes of one [3, d, d] tensor), and
    per loop tau: a, b [T, L, H] fp32 and rho [T, d] ~ U(0, 0.5) fp32."""
    L = wl.seq_len if seq_len is None else seq_len
    d = (wl.H * wl.dk) if d_model is None else d_model
    g = _gen(device, wl.name, "h0")
    h0 = torch.randn(L, d, generator=g, device=device, dtype=torch.float32).to(wl.dtype)
    Ws = torch.empty(3, d, d, device=device, dtype=wl.dtype)   # W_q, W_k, W_v as planes
    for i, name in enumerate(("Wq", "Wk", "Wv")):
        gw = _gen(device, wl.name, name)
        Ws[i] = (torch.randn(d, d, generator=gw, device=device, dtype=torch.float32)
                 / float(np.sqrt(d))).to(wl.dtype)
    a = torch.empty(wl.loops, L, wl.H, device=device)
    b = torch.empty(wl.loops, L, wl.H, device=device)
    rho = torch.empty(wl.loops, d, device=device)
    for tau in range(wl.loops):
        a[tau], b[tau] = gates(L, wl.H, device, wl.name, "loop", tau)
        gr = _gen(device, wl.name, "rho", tau)
        rho[tau] = torch.rand(d, generator=gr, device=device) * 0.5
    return dict(h0=h0, Wq=Ws[0], Wk=Ws[1], Wv=Ws[2], a=a, b=b, rho=rho, L=L, d=d)
