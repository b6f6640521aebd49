"""GPU parity of the per-channel (diagonal) gate variant, KDA, against the oracle.

Sigma_t = (I - b_t k_t k_t^T) Diag(a_t) Sigma_{t-1} + b_t k_t v_t^T with
a_t in (0, 1]^{dk} (GDN_CHANNEL_GATE; the KDA mixer of the LT2 mixer list,
"LT2: Linear-Time Looped Transformers", Appendix C).  The prefill runs the
fp32 KDA chunk kernel, decode both decode kernels.  Bars: relative L2 1e-4 on
fp32 work; with bf16 inputs the kernels still compute in fp32, so the state
keeps the 1e-4 bar and the outputs carry only their bf16 rounding (1e-2 bar,
about 2e-3 measured), plus the per-sequence and worst-chunk bars of gpu_util.
"""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import looped_linear_attention_b200 as lla
from looped_linear_attention_b200 import workloads as W
from gpu_util import TOL_BF16_O, TOL_F32, check_prefill, host, rel_l2, seq_bounds

pytestmark = pytest.mark.gpu
CG = lla.GDN_CHANNEL_GATE


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


def _inputs(label, dtype, H, dk, dv, lengths=None, n_seq=2, seq_len=200, random_s0=True):
    wl = dataclasses.replace(W.WORKLOADS["varlen"], name=f"kda-{label}", H=H, dk=dk, dv=dv, dtype=dtype,
                             random_s0=random_s0, varlen=lengths is not None)
    inp = W.prefill_inputs(wl, "cpu", lengths=lengths, n_seq=n_seq, seq_len=seq_len)
    inp["a"], inp["b"] = W.channel_gates(inp["total_tokens"], H, dk, "cpu", wl.name)
    return inp


SCHEDULES = ("two_launch", "one_launch")


def _run(inp, scale=1.0, flags=0, schedule="two_launch", **kw):
    """The prefill through the binding, which passes the workspace (two
    launches: the chunks' operands, then the chains), or through the C entry
    point with no workspace (the one-launch kernel)."""
    q, k, v, a, b = (inp[n].cuda() for n in ("q", "k", "v", "a", "b"))
    s0 = None if inp["S0"] is None else inp["S0"].cuda()
    cu = None if inp["cu_seqlens"] is None else torch.from_numpy(inp["cu_seqlens"]).cuda()
    epi = {n: t.cuda() for n, t in kw.items()}
    if schedule == "two_launch":
        o, ST = lla.gdn_chunk_fwd(q, k, v, a, b, s0, cu, n_seq=inp["n_seq"], scale=scale, flags=flags | CG,
                                  **epi)
    else:
        from looped_linear_attention_b200 import _binding as B
        T, H, dk = q.shape
        dv = v.shape[2]
        ns = inp["n_seq"]
        o = torch.full((T, H, dv), float("nan"), dtype=q.dtype, device=q.device)
        ST = torch.full((ns, H, dk, dv), float("nan"), device=q.device)
        ptr = lambda t: 0 if t is None else t.data_ptr()
        p = B.gdn_fwd_params(ptr(q), ptr(k), ptr(v), ptr(a), ptr(b), ptr(s0), ptr(o), ptr(ST), ptr(cu), ns,
                             0 if cu is not None else T // ns, T, H, dk, dv,
                             B.GDN_BF16 if q.dtype == torch.bfloat16 else B.GDN_F32, float(scale),
                             int(flags | CG), ptr(epi.get("gate")), ptr(epi.get("h_prev")), ptr(epi.get("rho")))
        assert lla.library().gdn_chunk_fwd(ctypes.byref(p), None, 0, None) == lla.GDN_OK
    torch.cuda.synchronize()
    _status_ok()
    return host(o), host(ST)


def _ref(inp, scale=1.0, normalize=False, gate=None):
    q, k = inp["q"], inp["k"]
    if normalize:   # the precise kernels round the normalised vectors to the io dtype
        q = torch.from_numpy(oracle.qk_l2norm(q)).to(inp["q"].dtype)
        k = torch.from_numpy(oracle.qk_l2norm(k)).to(inp["k"].dtype)
    cu = inp["cu_seqlens"]
    if cu is None:
        cu = np.arange(inp["n_seq"] + 1, dtype=np.int32) * inp["seq_len"]
    return oracle.kda_fwd(q, k, inp["v"], inp["a"], inp["b"], inp["S0"], cu, scale, gate=gate)


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_kda_prefill_fp32_ragged(schedule):
    inp = _inputs("fp32", torch.float32, 2, 64, 64)
    o, ST = _run(inp, scale=0.5, schedule=schedule)
    o_ref, S_ref = _ref(inp, scale=0.5)
    check_prefill(o, ST, o_ref, S_ref, seq_bounds(inp), fp32=True)


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_kda_prefill_bf16_varlen_l2norm_dv256(schedule):
    inp = _inputs("bf16", torch.bfloat16, 2, 128, 256, lengths=[0, 1, 63, 64, 65, 129, 300])
    o, ST = _run(inp, scale=0.125, flags=lla.GDN_QK_L2NORM, schedule=schedule)
    o_ref, S_ref = _ref(inp, scale=0.125, normalize=True)
    err = check_prefill(o, ST, o_ref, S_ref, seq_bounds(inp), fp32=False)
    assert err["S"] < TOL_F32, err
    np.testing.assert_array_equal(ST[0].numpy(), inp["S0"][0].numpy())   # empty sequence


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_kda_prefill_hard_and_exact_channel_decays(schedule):
    """Channels that reset (a = 1e-20), never decay (a = 1) or decay hard
    (a = 0.05) side by side, over several chunks: every decay factor is an
    exponential of a non-positive number, so nothing overflows."""
    inp = _inputs("hard", torch.float32, 2, 64, 64, n_seq=1, seq_len=333)
    a = inp["a"].clone()
    a[:, :, 0:8] = 1e-20
    a[:, :, 8:16] = 1.0
    a[:, :, 16:24] = 0.05
    a[::7, 1, :] = 1e-20          # whole-token resets on head 1
    inp["a"] = a
    o, ST = _run(inp, schedule=schedule)
    assert torch.isfinite(o).all() and torch.isfinite(ST).all()
    o_ref, S_ref = _ref(inp)
    check_prefill(o, ST, o_ref, S_ref, seq_bounds(inp), fp32=True)


def test_kda_with_equal_channels_equals_gated_delta_rule():
    """The same decay in every channel: the KDA kernel agrees with the fp32
    gated delta-rule kernel (GDN_PRECISE) to fp32 rounding."""
    inp = _inputs("scalar", torch.float32, 2, 128, 128)
    alpha = inp["a"][:, :, 0].contiguous()
    inp["a"] = alpha[:, :, None].expand(-1, -1, 128).contiguous()
    o1, S1 = _run(inp)
    q, k, v, b = (inp[n].cuda() for n in ("q", "k", "v", "b"))
    o2, S2 = lla.gdn_chunk_fwd(q, k, v, alpha.cuda(), b, inp["S0"].cuda(), n_seq=2, flags=lla.GDN_PRECISE)
    torch.cuda.synchronize()
    assert rel_l2(o1, host(o2)) < 1e-5 and rel_l2(S1, host(S2)) < 1e-5


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_kda_prefill_gate_and_residual(schedule):
    inp = _inputs("epi", torch.bfloat16, 2, 128, 128)
    g = torch.Generator().manual_seed(W.seed_for("test", "kda-epilogue"))
    z = 2.0 * torch.randn(inp["total_tokens"], 2, generator=g)
    hp = torch.randn(inp["total_tokens"], 2 * 128, generator=g).bfloat16()
    rho = 0.5 * torch.rand(2 * 128, generator=g)
    o, ST = _run(inp, gate=z, h_prev=hp, rho=rho, schedule=schedule)
    o_g, S_ref = _ref(inp, gate=z)
    ref = oracle.round_bf16(oracle.loop_residual(oracle.round_bf16(o_g).reshape(-1, 256), hp, rho))
    check_prefill(o.reshape(ref.shape[0], 2, 128), ST, ref.reshape(-1, 2, 128), S_ref, seq_bounds(inp),
                  fp32=False)


def test_kda_full_size_both_schedules():
    """The timed KDA workload in full (one sequence of 4096 tokens, 16 heads,
    dk = dv = 128, bf16, in-kernel q/k norm): both schedules against the
    oracle on every output and state, and against each other."""
    wl = dataclasses.replace(W.WORKLOADS["looped_prefill"], name="kda")
    inp = W.prefill_inputs(wl, "cpu")
    inp["a"], inp["b"] = W.channel_gates(inp["total_tokens"], wl.H, wl.dk, "cpu", "bench", "kda")
    o2, S2 = _run(inp, flags=lla.GDN_QK_L2NORM, schedule="two_launch")
    o1, S1 = _run(inp, flags=lla.GDN_QK_L2NORM, schedule="one_launch")
    o_ref, S_ref = _ref(inp, normalize=True)
    err = check_prefill(o2, S2, o_ref, S_ref, seq_bounds(inp), fp32=False)
    assert err["S"] < TOL_F32, err
    check_prefill(o1, S1, o_ref, S_ref, seq_bounds(inp), fp32=False)
    assert rel_l2(S1, S2) < 1e-5 and rel_l2(o1, o2) < TOL_BF16_O


@pytest.mark.parametrize("dk,dv,dtype", [(128, 128, torch.bfloat16), (64, 192, torch.float32)])
def test_kda_decode(dk, dv, dtype):
    """The streaming kernel (dk = dv = 128, bf16; the decay vector rides in
    the bulk-copy ring) and the register kernel."""
    wl = dataclasses.replace(W.WORKLOADS["decode"], dk=dk, dv=dv, dtype=dtype, H=3)
    inp = W.decode_inputs(wl, "cpu", n_slots=41)
    inp["a"], inp["b"] = W.channel_gates(41, 3, dk, "cpu", "kda-decode", dk, dv)
    S = inp["S"].cuda()
    o = lla.gdn_decode_step(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), inp["a"].cuda(),
                            inp["b"].cuda(), S, scale=0.75, flags=CG)
    torch.cuda.synchronize()
    _status_ok()
    o_ref, S_ref = oracle.kda_decode(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["S"], 0.75)
    tol_o = TOL_F32 if dtype == torch.float32 else 4e-3   # bf16 output rounding
    assert rel_l2(host(o), o_ref) < tol_o
    assert rel_l2(host(S), S_ref) < TOL_F32


def test_kda_decode_continues_prefill():
    inp = _inputs("cont", torch.bfloat16, 2, 128, 128, n_seq=1, seq_len=201)
    L = 200
    pre = {k: (v[:L] if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    pre.update(seq_len=L, total_tokens=L)
    _, S_L = _run(pre)
    S = S_L.cuda()
    o_d = lla.gdn_decode_step(*(inp[n][L:].cuda() for n in ("q", "k", "v", "a", "b")), S, flags=CG)
    torch.cuda.synchronize()
    _status_ok()
    o_ref, S_ref = _ref(inp)
    assert rel_l2(host(o_d)[0], o_ref[L]) < TOL_BF16_O
    assert rel_l2(host(S), S_ref) < TOL_F32
