"""The looped-prefill step: T iterations of (q/k/v projection -> GDN mixer ->
per-loop residual) on one sequence.

"LT2: Linear-Time Looped Transformers", §2, "LT2." paragraph: the shared block
stack is applied T times, and the loop state is
h^(tau) = h~^(tau) + rho_tau (.) h^(tau-1).  In this workload the block output
h~^(tau) is the GDN output itself, reshaped [L, H*dv] = [L, d] (d = H*dv), from
a zero initial state each loop; q and k are L2-normalised per head inside the
mixer kernel.  The three projections are one batched torch GEMM over the
stacked weights [W_q; W_k; W_v] (outside the mixer's hot path); the mixer and
the residual run in this library's kernels: by default the residual is fused
into the mixer's output epilogue (one launch fewer per loop, and the mixer
output never makes a round trip through HBM), or it runs as loop_residual.
The gated variant (§3, gated-attention paragraph) adds a head-wise sigmoid
output gate whose logits h^(tau-1) W_g (W_g [d, H] fp32) are one more torch
GEMM per loop; the gate itself is applied in the mixer's epilogue.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _binding as B


class LoopedPrefill:
    """Pre-allocated buffers for repeated looped-prefill steps (graph-capturable)."""

    def __init__(self, L: int, H: int, dk: int, dv: int, loops: int, device,
                 dtype=torch.bfloat16, time_mixer: bool = False, fused_residual: bool = True):
        d_in = H * dk
        self.fused_residual = fused_residual
        # optional CUDA-event pairs around every mixer launch (for per-kernel timing)
        self.time_mixer = time_mixer
        self.mixer_events = []
        self.L, self.H, self.dk, self.dv, self.loops = L, H, dk, dv, loops
        assert d_in == H * dv, "the loop state feeds the next projection: H*dk must equal H*dv"
        # q, k, v as the three planes of one [3, L, d] buffer (one batched GEMM)
        self.qkv = torch.empty(3, L, d_in, dtype=dtype, device=device)
        self.q = self.qkv[0].view(L, H, dk)
        self.k = self.qkv[1].view(L, H, dk)
        self.v = self.qkv[2].view(L, H, dv)
        self.o = torch.empty(L, H, dv, dtype=dtype, device=device)
        self.z = torch.empty(L, H, dtype=torch.float32, device=device)     # output-gate logits
        self.h = [torch.empty(L, H * dv, dtype=dtype, device=device) for _ in range(2)]

    def launches_per_loop(self) -> int:
        """This library's kernel launches per loop: the mixer's (its schedule)
        plus the loop residual when it is not fused."""
        sched = B.prefill_schedule(1, self.L, self.H, self.dk, self.dv, flags=B.GDN_QK_L2NORM,
                                   with_state=False)
        return sched["launches"] + (0 if self.fused_residual else 1)

    def run(self, h0: torch.Tensor, Wq: torch.Tensor, Wk: torch.Tensor, Wv: torch.Tensor,
            a: torch.Tensor, b: torch.Tensor, rho: torch.Tensor, scale: float = 1.0,
            out: Optional[torch.Tensor] = None, Wg: Optional[torch.Tensor] = None) -> torch.Tensor:
        """h0 [L, d]; W* [d, d]; a, b [T, L, H] fp32; rho [T, d] fp32; Wg [d, H]
        fp32 output-gate weights or None. Returns h^(T).

        Wq, Wk, Wv given as the three planes of one [3, d, d] tensor (see
        `stack_weights`) are used in place; otherwise they are stacked into a
        new tensor on every call."""
        L, H, dv = self.L, self.H, self.dv
        W3 = stacked_view(Wq, Wk, Wv)
        if W3 is None:
            W3 = torch.stack((Wq, Wk, Wv))
        h_prev = h0
        for tau in range(self.loops):
            torch.matmul(h_prev.unsqueeze(0), W3, out=self.qkv)
            z = None
            if Wg is not None:
                torch.matmul(h_prev.float(), Wg, out=self.z)
                z = self.z
            last = tau == self.loops - 1
            h_next = out if (last and out is not None) else self.h[tau % 2]
            if self.time_mixer:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
            if self.fused_residual:
                B.gdn_chunk_fwd(self.q, self.k, self.v, a[tau], b[tau], None, scale=scale,
                                flags=B.GDN_QK_L2NORM, o=h_next, return_state=False, gate=z,
                                h_prev=h_prev, rho=rho[tau])
            else:
                B.gdn_chunk_fwd(self.q, self.k, self.v, a[tau], b[tau], None, scale=scale,
                                flags=B.GDN_QK_L2NORM, o=self.o, return_state=False, gate=z)
            if self.time_mixer:
                e1.record()
                self.mixer_events.append((e0, e1))
            if not self.fused_residual:
                B.loop_residual(self.o.view(L, H * dv), h_prev, rho[tau], out=h_next)
            h_prev = h_next
        return h_prev

    def capture(self, h0: torch.Tensor, Wq: torch.Tensor, Wk: torch.Tensor, Wv: torch.Tensor,
                a: torch.Tensor, b: torch.Tensor, rho: torch.Tensor, scale: float = 1.0,
                out: Optional[torch.Tensor] = None, Wg: Optional[torch.Tensor] = None):
        """Records one `run` on these tensors into a CUDA graph.

        Returns (graph, h): each graph.replay() repeats the whole T-loop step
        (projections, mixer launches, residuals; no host work) on the same
        buffers and leaves h^(T) in h.  The tensors' contents may change between
        replays, their storage may not.  One eager run on a side stream first
        sets up the library's lazy state (launch attributes, the status word)
        outside the capture."""
        dev = self.qkv.device
        timing, self.time_mixer = self.time_mixer, False
        try:
            side = torch.cuda.Stream(dev)
            side.wait_stream(torch.cuda.current_stream(dev))
            with torch.cuda.stream(side):
                self.run(h0, Wq, Wk, Wv, a, b, rho, scale=scale, out=out, Wg=Wg)
            torch.cuda.current_stream(dev).wait_stream(side)
            graph = torch.cuda.CUDAGraph()
            # thread-local capture: CUDA calls of other threads (a process
            # group's watchdog, for one) do not invalidate it
            with torch.cuda.graph(graph, capture_error_mode="thread_local"):
                h = self.run(h0, Wq, Wk, Wv, a, b, rho, scale=scale, out=out, Wg=Wg)
        finally:
            self.time_mixer = timing
        return graph, h


def stack_weights(Wq: torch.Tensor, Wk: torch.Tensor, Wv: torch.Tensor):
    """One [3, d, d] tensor holding W_q, W_k, W_v, and its three planes (pass
    those to `LoopedPrefill.run` to avoid a copy per call)."""
    W3 = torch.stack((Wq, Wk, Wv)).contiguous()
    return W3, W3[0], W3[1], W3[2]


def stacked_view(Wq: torch.Tensor, Wk: torch.Tensor, Wv: torch.Tensor) -> Optional[torch.Tensor]:
    """[3, d, d] view of W_q, W_k, W_v when they are consecutive planes of one
    contiguous allocation, else None."""
    ws = (Wq, Wk, Wv)
    if Wq.dim() != 2 or any(w.shape != Wq.shape or w.dtype != Wq.dtype or w.device != Wq.device
                            or not w.is_contiguous() for w in ws):
        return None
    n = Wq.numel()
    base = Wq.untyped_storage().data_ptr()
    if any(w.untyped_storage().data_ptr() != base for w in ws):
        return None
    if Wk.storage_offset() != Wq.storage_offset() + n or Wv.storage_offset() != Wq.storage_offset() + 2 * n:
        return None
    return Wq.as_strided((3,) + tuple(Wq.shape), (n,) + tuple(Wq.stride()))


class HostPipeline:
    """Looped-prefill steps whose inputs and results live in pinned host memory.

    Each `submit` copies one step's h0, a, b to the device, runs the step on the
    caller's current stream and copies h^(T) back, all asynchronously.  Two
    device buffer sets and two copy streams (host-to-device, device-to-host)
    let the copies of one step overlap the compute of its neighbours; events
    keep a buffer set from being refilled before the step that used it is done.
    With `graphs` (the default) the compute of a step is a CUDA-graph replay:
    one graph per buffer set, captured on first use (and again when the
    weights, rho or scale change).  The host buffers of a step must stay
    untouched until the event that `submit` returns has completed (its
    copy-out is then finished)."""

    def __init__(self, runner: LoopedPrefill, device, graphs: bool = True):
        L, d, T = runner.L, runner.H * runner.dv, runner.loops
        self.runner = runner
        self.dev = torch.device(device)
        self.h = [torch.empty(L, d, dtype=torch.bfloat16, device=self.dev) for _ in range(2)]
        self.a = [torch.empty(T, L, runner.H, dtype=torch.float32, device=self.dev) for _ in range(2)]
        self.b = [torch.empty(T, L, runner.H, dtype=torch.float32, device=self.dev) for _ in range(2)]
        self.out = [torch.empty(L, d, dtype=torch.bfloat16, device=self.dev) for _ in range(2)]
        self.s_in = torch.cuda.Stream(self.dev)
        self.s_out = torch.cuda.Stream(self.dev)
        self.inputs_free = [None, None]     # compute of the last step that read buffer set k
        self.output_free = [None, None]     # copy-out of the last step that wrote out[k]
        self.n = 0
        self.graphs = graphs
        self.graph = [None, None]           # (key, CUDA graph) per buffer set

    def submit(self, h_host, a_host, b_host, out_host, Wq, Wk, Wv, rho, scale: float = 1.0):
        compute = torch.cuda.current_stream(self.dev)
        k = self.n % 2
        self.n += 1
        with torch.cuda.stream(self.s_in):
            if self.inputs_free[k] is not None:
                self.s_in.wait_event(self.inputs_free[k])
            self.h[k].copy_(h_host, non_blocking=True)
            self.a[k].copy_(a_host, non_blocking=True)
            self.b[k].copy_(b_host, non_blocking=True)
            loaded = torch.cuda.Event()
            loaded.record(self.s_in)
        compute.wait_event(loaded)
        if self.output_free[k] is not None:
            compute.wait_event(self.output_free[k])
        self._compute(k, Wq, Wk, Wv, rho, scale)
        done = torch.cuda.Event()
        done.record(compute)
        self.inputs_free[k] = done
        with torch.cuda.stream(self.s_out):
            self.s_out.wait_event(done)
            out_host.copy_(self.out[k], non_blocking=True)
            copied = torch.cuda.Event()
            copied.record(self.s_out)
        self.output_free[k] = copied
        return copied

    def _compute(self, k, Wq, Wk, Wv, rho, scale):
        args = (self.h[k], Wq, Wk, Wv, self.a[k], self.b[k], rho)
        if not self.graphs:
            self.runner.run(*args, scale=scale, out=self.out[k])
            return
        # a replay reads whatever the captured addresses hold, so the key is
        # the operands' storage, not their values
        key = (Wq.data_ptr(), Wk.data_ptr(), Wv.data_ptr(), rho.data_ptr(), float(scale))
        if self.graph[k] is None or self.graph[k][0] != key:
            graph, _ = self.runner.capture(*args, scale=scale, out=self.out[k])
            self.graph[k] = (key, graph)
        self.graph[k][1].replay()

    def join(self, stream=None):
        """Makes `stream` (default: the current one) wait for every copy submitted so far."""
        stream = torch.cuda.current_stream(self.dev) if stream is None else stream
        stream.wait_stream(self.s_in)
        stream.wait_stream(self.s_out)

    def start_after(self, stream=None):
        """Makes the copy streams wait for work already queued on `stream`."""
        stream = torch.cuda.current_stream(self.dev) if stream is None else stream
        self.s_in.wait_stream(stream)
        self.s_out.wait_stream(stream)
