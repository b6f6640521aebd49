"""GPU parity of the looped block's output epilogue against the oracle.

The head-wise sigmoid output gate ("LT2: Linear-Time Looped Transformers", §3,
gated-attention paragraph) and the per-loop residual h = h~ + rho (.) h_prev
(§2, "LT2." paragraph) applied in the mixer's output epilogue: on the
tensor-core prefill (one pass, segmented, varlen, in place over h_prev), the
precise prefill, both decode kernels, and the looped step, where the fused
residual must equal the separate loop_residual launch bit for bit (same
arithmetic: the output rounded to bf16, then rho * h_prev + o in fp32, rounded).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import looped_linear_attention_b200 as lla
from looped_linear_attention_b200 import workloads as W
from gpu_util import TOL_BF16_O, TOL_F32, check_prefill, host, rel_l2, seq_bounds

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    from looped_linear_attention_b200 import build
    build.build()
    lla.library()
    torch.cuda.init()
    yield
    assert lla.gdn_get_device_status() == lla.GDN_OK


def _status_ok():
    st = lla.gdn_get_device_status()
    assert st == lla.GDN_OK, lla.status_string(st)


def _wl(name, **kw):
    return dataclasses.replace(W.WORKLOADS[name], **kw)


def _epilogue_inputs(n_tok, H, dv, dtype, label):
    """Gate logits ~ N(0, 2) [n_tok, H]; h_prev ~ N(0, 1) [n_tok, H*dv] (io
    dtype); rho ~ U(0, 0.5) [H*dv]."""
    g = torch.Generator().manual_seed(W.seed_for("test", "epilogue", label))
    z = 2.0 * torch.randn(n_tok, H, generator=g)
    hp = torch.randn(n_tok, H * dv, generator=g).to(dtype)
    rho = 0.5 * torch.rand(H * dv, generator=g)
    return z, hp, rho


def _ref_epilogue(o_gated, hp, rho, dtype):
    """The oracle's order: round the gated output to the io dtype, add
    rho (.) h_prev, round again."""
    n_tok, H, dv = o_gated.shape
    rnd = oracle.round_bf16 if dtype == torch.bfloat16 else (lambda x: x.astype(np.float32).astype(np.float64))
    ht = rnd(o_gated).reshape(n_tok, H * dv)
    return rnd(oracle.loop_residual(ht, hp, rho)).reshape(n_tok, H, dv)


def _run(inp, z, hp, rho, scale=1.0, flags=0, in_place=False):
    q, k, v, a, b = (inp[n].cuda() for n in ("q", "k", "v", "a", "b"))
    s0 = None if inp["S0"] is None else inp["S0"].cuda()
    cu = None if inp["cu_seqlens"] is None else torch.from_numpy(inp["cu_seqlens"]).cuda()
    hp_d = hp.cuda()
    o = hp_d if in_place else None
    o, ST = lla.gdn_chunk_fwd(q, k, v, a, b, s0, cu, n_seq=inp["n_seq"], scale=scale, flags=flags,
                              o=o, gate=z.cuda(), h_prev=hp_d, rho=rho.cuda())
    torch.cuda.synchronize()
    _status_ok()
    return host(o).reshape(inp["total_tokens"], -1, inp["v"].shape[2]), host(ST)


def _oracle(inp, z, scale=1.0, normalize=False):
    q, k = inp["q"], inp["k"]
    if normalize:
        q, k = oracle.qk_l2norm(q), oracle.qk_l2norm(k)
    cu = inp["cu_seqlens"]
    if cu is None:
        cu = np.arange(inp["n_seq"] + 1, dtype=np.int32) * inp["seq_len"]
    return oracle.gdn_fwd(q, k, inp["v"], inp["a"], inp["b"], inp["S0"], cu, scale, gate=z)


@pytest.mark.parametrize("case", ["one_pass", "segmented", "segmented_in_place", "varlen_l2norm"])
def test_prefill_tc_gate_and_residual(case):
    if case == "varlen_l2norm":
        wl = _wl("varlen", H=2, normalize_qk=False)
        inp = W.prefill_inputs(wl, "cpu", lengths=[0, 1, 63, 64, 65, 129, 700])
        flags, scale, norm = lla.GDN_QK_L2NORM, 0.125, True
    else:
        L = 333 if case == "one_pass" else 1500
        wl = _wl("long_prefill", n_seq=1 if case != "one_pass" else 2, H=2, seq_len=L, random_s0=True)
        inp = W.prefill_inputs(wl, "cpu")
        flags, scale, norm = (lla.GDN_SINGLE_PASS if case == "one_pass" else 0), 1.0, False
        if case != "one_pass":
            assert lla.prefill_schedule(1, L, 2, 128, 128)["n_segs"] > 1
    z, hp, rho = _epilogue_inputs(inp["total_tokens"], wl.H, wl.dv, torch.bfloat16, case)
    o, ST = _run(inp, z, hp, rho, scale=scale, flags=flags, in_place=case.endswith("in_place"))
    o_g, S_ref = _oracle(inp, z, scale=scale, normalize=norm)
    ref = _ref_epilogue(o_g, hp, rho, torch.bfloat16)
    check_prefill(o, ST, ref, S_ref, seq_bounds(inp), fp32=False)


def test_prefill_precise_gate_and_residual_fp32():
    wl = _wl("tiny", n_seq=2, H=2, seq_len=150, random_s0=True)
    inp = W.prefill_inputs(wl, "cpu")
    z, hp, rho = _epilogue_inputs(inp["total_tokens"], wl.H, wl.dv, torch.float32, "precise")
    o, ST = _run(inp, z, hp, rho, scale=0.5)
    o_g, S_ref = _oracle(inp, z, scale=0.5)
    ref = _ref_epilogue(o_g, hp, rho, torch.float32)
    check_prefill(o, ST, ref, S_ref, seq_bounds(inp), fp32=True)


@pytest.mark.parametrize("dk,dv,dtype,in_place", [(128, 128, torch.bfloat16, False),
                                                  (128, 128, torch.bfloat16, True),
                                                  (64, 192, torch.float32, False)])
def test_decode_gate_and_residual(dk, dv, dtype, in_place):
    """The streaming kernel (dk = dv = 128, bf16) and the register kernel."""
    wl = _wl("decode", dk=dk, dv=dv, dtype=dtype, H=3)
    inp = W.decode_inputs(wl, "cpu", n_slots=37)
    z, hp, rho = _epilogue_inputs(37, 3, dv, dtype, f"decode-{dk}-{dv}-{in_place}")
    S = inp["S"].cuda()
    hp_d = hp.cuda()
    o = lla.gdn_decode_step(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), inp["a"].cuda(),
                            inp["b"].cuda(), S, scale=0.75, gate=z.cuda(), h_prev=hp_d, rho=rho.cuda(),
                            o=hp_d if in_place else None)
    torch.cuda.synchronize()
    _status_ok()
    o_g, S_ref = oracle.gdn_decode(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["S"], 0.75,
                                   gate=z)
    ref = _ref_epilogue(o_g, hp, rho, dtype)
    tol_o = TOL_F32 if dtype == torch.float32 else 4e-3   # bf16 output rounding
    assert rel_l2(host(o).reshape(ref.shape), ref) < tol_o
    assert rel_l2(host(S), S_ref) < TOL_F32


def test_looped_step_fused_residual_equals_separate_launch():
    """The looped step with the residual in the mixer's epilogue gives the
    same h^(T) bit for bit as the mixer followed by loop_residual."""
    wl = dataclasses.replace(W.WORKLOADS["looped_prefill"], seq_len=1024)
    inp = W.looped_inputs(wl, "cuda")
    args = (inp["h0"], inp["Wq"], inp["Wk"], inp["Wv"], inp["a"], inp["b"], inp["rho"])
    fused = lla.LoopedPrefill(inp["L"], wl.H, wl.dk, wl.dv, wl.loops, "cuda")
    separate = lla.LoopedPrefill(inp["L"], wl.H, wl.dk, wl.dv, wl.loops, "cuda", fused_residual=False)
    assert fused.launches_per_loop() + 1 == separate.launches_per_loop()
    h_f = fused.run(*args).clone()
    h_s = separate.run(*args).clone()
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(h_f, h_s)


def test_looped_step_with_output_gate_matches_oracle():
    """The gated looped variant (W_g [d, H]) on a 512-token sequence, T = 4,
    against the oracle's own chain, also as a CUDA-graph replay."""
    wl = dataclasses.replace(W.WORKLOADS["looped_prefill"], seq_len=512)
    inp = W.looped_inputs(wl, "cpu")
    d = inp["d"]
    g = torch.Generator().manual_seed(W.seed_for("test", "looped-gate"))
    Wg = torch.randn(d, wl.H, generator=g) / float(np.sqrt(d))
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    runner = lla.LoopedPrefill(inp["L"], wl.H, wl.dk, wl.dv, wl.loops, "cuda")
    args = (dev["h0"], dev["Wq"], dev["Wk"], dev["Wv"], dev["a"], dev["b"], dev["rho"])
    hT = runner.run(*args, Wg=Wg.cuda()).clone()
    torch.cuda.synchronize()
    _status_ok()
    ref = oracle.looped_forward(inp["h0"], inp["Wq"], inp["Wk"], inp["Wv"], inp["a"], inp["b"],
                                inp["rho"], wl.H, wl.dk, wl.dv, Wg=Wg)
    assert rel_l2(host(hT), ref) < TOL_BF16_O
    out = torch.empty_like(hT)
    graph, _ = runner.capture(*args, out=out, Wg=Wg.cuda())
    graph.replay()
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(out, hT)
