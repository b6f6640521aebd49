"""The looped-prefill step: T iterations of (q/k/v projection -> GDN mixer ->
per-loop residual) on one sequence.

"LT2: Linear-Time Looped Transformers", §2, "LT2." paragraph: the shared block
stack is applied T times, and the loop state is
h^(tau) = h~^(tau) + rho_tau (.) h^(tau-1).  In this workload the block output
h~^(tau) is the GDN output itself, reshaped [L, H*dv] = [L, d] (d = H*dv), from
a zero initial state each loop; q and k are L2-normalised per head inside the
mixer kernel.  The projections are plain torch GEMMs (outside the mixer's hot
path); the mixer and the residual run in this library's kernels.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _binding as B


class LoopedPrefill:
    """Pre-allocated buffers for repeated looped-prefill steps (graph-capturable)."""

    def __init__(self, L: int, H: int, dk: int, dv: int, loops: int, device,
                 dtype=torch.bfloat16, time_mixer: bool = False):
        d_in = H * dk
        # optional CUDA-event pairs around every mixer launch (for per-kernel timing)
        self.time_mixer = time_mixer
        self.mixer_events = []
        self.L, self.H, self.dk, self.dv, self.loops = L, H, dk, dv, loops
        self.q = torch.empty(L, H, dk, dtype=dtype, device=device)
        self.k = torch.empty(L, H, dk, dtype=dtype, device=device)
        self.v = torch.empty(L, H, dv, dtype=dtype, device=device)
        self.o = torch.empty(L, H, dv, dtype=dtype, device=device)
        self.h = [torch.empty(L, H * dv, dtype=dtype, device=device) for _ in range(2)]
        assert d_in == H * dv, "the loop state feeds the next projection: H*dk must equal H*dv"

    def run(self, h0: torch.Tensor, Wq: torch.Tensor, Wk: torch.Tensor, Wv: torch.Tensor,
            a: torch.Tensor, b: torch.Tensor, rho: torch.Tensor, scale: float = 1.0,
            out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """h0 [L, d]; W* [d, d]; a, b [T, L, H] fp32; rho [T, d] fp32. Returns h^(T)."""
        L, H, dk, dv = self.L, self.H, self.dk, self.dv
        h_prev = h0
        for tau in range(self.loops):
            torch.matmul(h_prev, Wq, out=self.q.view(L, H * dk))
            torch.matmul(h_prev, Wk, out=self.k.view(L, H * dk))
            torch.matmul(h_prev, Wv, out=self.v.view(L, H * dv))
            if self.time_mixer:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
            B.gdn_chunk_fwd(self.q, self.k, self.v, a[tau], b[tau], None, scale=scale,
                            flags=B.GDN_QK_L2NORM, o=self.o, return_state=False)
            if self.time_mixer:
                e1.record()
                self.mixer_events.append((e0, e1))
            last = tau == self.loops - 1
            h_next = out if (last and out is not None) else self.h[tau % 2]
            B.loop_residual(self.o.view(L, H * dv), h_prev, rho[tau], out=h_next)
            h_prev = h_next
        return h_prev
