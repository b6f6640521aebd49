"""Parity of the CUDA kernels (through the C ABI) with the CPU oracle.

Small cases span several 64-token chunks with ragged tails and every edge case
the ABI admits; the full-size workloads run on the GPU exactly as the benchmark
launches them and are checked on sampled (sequence, head) chains that the
oracle recomputes one by one.  Bars: relative L2 error 1e-4 for fp32 inputs,
1e-2 on outputs and 5e-3 on final states for bf16 inputs; the loop residual
within one bf16 ulp element-wise.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import looped_linear_attention_b200 as lla
from looped_linear_attention_b200 import workloads as W
from gpu_util import (TOL_BF16_O, TOL_BF16_S, TOL_F32, bf16_ulp, check_prefill, host, rel_l2,
                      seq_bounds)

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


def _gpu_prefill(inp, scale=1.0, flags=0, S0="inp", alias=False):
    q, k, v, a, b = (inp[n].cuda() for n in ("q", "k", "v", "a", "b"))
    s0 = inp["S0"] if S0 == "inp" else S0
    s0 = None if s0 is None else s0.cuda()
    cu = None if inp["cu_seqlens"] is None else torch.from_numpy(inp["cu_seqlens"]).cuda()
    kw = {}
    if alias:
        assert s0 is not None
        kw["S_T"] = s0
    o, ST = lla.gdn_chunk_fwd(q, k, v, a, b, s0, cu, n_seq=inp["n_seq"], scale=scale,
                              flags=flags, **kw)
    torch.cuda.synchronize()
    return host(o), host(ST)


def _oracle_prefill(inp, scale=1.0, normalize=False, S0="inp"):
    q, k = inp["q"], inp["k"]
    if normalize:
        q, k = oracle.qk_l2norm(q), oracle.qk_l2norm(k)
    s0 = inp["S0"] if S0 == "inp" else S0
    cu = inp["cu_seqlens"]
    if cu is None:
        L = inp["seq_len"]
        cu = np.arange(inp["n_seq"] + 1, dtype=np.int32) * L
    return oracle.gdn_fwd(q, k, inp["v"], inp["a"], inp["b"], s0, cu, scale)


def _check(o, ST, o_ref, S_ref, fp32, inp=None, bounds=None):
    """Whole-tensor, per-sequence and worst-chunk bars (gpu_util.check_prefill)."""
    if bounds is None:
        bounds = seq_bounds(inp)
    return check_prefill(o, ST, o_ref, S_ref, bounds, fp32)


# ------------------------------------------------------------------ residual
@pytest.mark.parametrize("alias", [False, True])
def test_loop_residual_bf16_within_one_ulp(alias):
    g = torch.Generator().manual_seed(W.seed_for("test", "residual"))
    rows, d = 4099, 2048
    ht = torch.randn(rows, d, generator=g).bfloat16()
    hp = torch.randn(rows, d, generator=g).bfloat16()
    rho = torch.rand(d, generator=g) * 0.5
    ht_d, hp_d = ht.cuda(), hp.cuda()
    out = lla.loop_residual(ht_d, hp_d, rho.cuda(), out=hp_d if alias else None)
    torch.cuda.synchronize()
    ref = oracle.loop_residual(ht, hp, rho)
    got = host(out).double().numpy()
    err = np.abs(got - ref)
    assert np.all(err <= bf16_ulp(ref) + 1e-30)
    assert np.mean(got == oracle.round_bf16(ref)) > 0.99
    _status_ok()


def test_loop_residual_f32():
    g = torch.Generator().manual_seed(W.seed_for("test", "residual32"))
    ht, hp = torch.randn(37, 24, generator=g), torch.randn(37, 24, generator=g)
    rho = torch.rand(24, generator=g)
    out = lla.loop_residual(ht.cuda(), hp.cuda(), rho.cuda())
    np.testing.assert_allclose(host(out).double().numpy(), oracle.loop_residual(ht, hp, rho),
                               rtol=1e-6, atol=1e-6)


# ------------------------------------------------------------------ decode
@pytest.mark.parametrize("dk,dv,dtype,flags", [
    (128, 128, torch.bfloat16, lla.GDN_QK_L2NORM),
    (128, 128, torch.bfloat16, 0),
    (64, 64, torch.float32, 0),
    (128, 192, torch.bfloat16, 0),
    (64, 256, torch.float32, lla.GDN_QK_L2NORM),
])
def test_decode_step(dk, dv, dtype, flags):
    wl = _wl("decode", dk=dk, dv=dv, dtype=dtype, H=3, normalize_qk=not flags)
    inp = W.decode_inputs(wl, "cpu", n_slots=37)
    S = inp["S"].cuda()
    o = lla.gdn_decode_step(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), inp["a"].cuda(),
                            inp["b"].cuda(), S, scale=0.75, flags=flags)
    torch.cuda.synchronize()
    q, k = inp["q"], inp["k"]
    if flags & lla.GDN_QK_L2NORM:
        q, k = oracle.qk_l2norm(q), oracle.qk_l2norm(k)
    o_ref, S_ref = oracle.gdn_decode(q, k, inp["v"], inp["a"], inp["b"], inp["S"], 0.75)
    tol_o = TOL_F32 if dtype == torch.float32 else 4e-3   # bf16 output rounding
    assert rel_l2(host(o), o_ref) < tol_o
    assert rel_l2(host(S), S_ref) < TOL_F32
    _status_ok()


# ------------------------------------------------------------------ prefill, precise path
def test_prefill_tiny_workload_fp32():
    """B=1, H=2, L=256, dk=dv=64, fp32, zero initial state."""
    inp = W.prefill_inputs(W.WORKLOADS["tiny"], "cpu")
    o, ST = _gpu_prefill(inp)
    o_ref, S_ref = _oracle_prefill(inp)
    _check(o, ST, o_ref, S_ref, fp32=True, inp=inp)
    _status_ok()


@pytest.mark.parametrize("dk,dv", [(128, 192), (64, 64)])
def test_prefill_precise_varlen_edges(dk, dv):
    """Empty, 1-token, 63/64/65-token and longer sequences, random S0, q/k
    normalised in-kernel, scale != 1."""
    wl = _wl("varlen", dk=dk, dv=dv, H=3, dtype=torch.float32, normalize_qk=False)
    inp = W.prefill_inputs(wl, "cpu", lengths=[0, 1, 63, 64, 65, 200])
    o, ST = _gpu_prefill(inp, scale=0.5, flags=lla.GDN_QK_L2NORM)
    o_ref, S_ref = _oracle_prefill(inp, scale=0.5, normalize=True)
    _check(o, ST, o_ref, S_ref, fp32=True, inp=inp)
    np.testing.assert_allclose(ST[0].numpy(), inp["S0"][0].numpy(), rtol=0, atol=0)
    _status_ok()


# ------------------------------------------------------------------ prefill, tensor-core path
def test_prefill_tc_fixed_length_ragged():
    wl = _wl("long_prefill", n_seq=2, H=3, seq_len=300, random_s0=True)
    inp = W.prefill_inputs(wl, "cpu")
    o, ST = _gpu_prefill(inp)
    o_ref, S_ref = _oracle_prefill(inp)
    _check(o, ST, o_ref, S_ref, fp32=False, inp=inp)
    _status_ok()


def test_prefill_tc_strong_and_mixed_decay():
    """Chunks whose decay spans more than 2^64 inside 64 tokens take the
    per-entry exponential path of the decay matrix; the others use its
    row x column factorisation.  Head 0 decays hard everywhere (a = 0.05), head 1
    alternates hard and mild chunks, head 2 mixes the workload's gates with
    near-resets (a = 1e-20) and exact a = 1."""
    wl = _wl("long_prefill", n_seq=2, H=3, seq_len=333, random_s0=True)
    inp = W.prefill_inputs(wl, "cpu")
    a = inp["a"].clone()
    tok = torch.arange(a.shape[0])
    pos = tok % 333
    a[:, 0] = 0.05
    a[:, 1] = torch.where((pos // 64) % 2 == 0, torch.tensor(0.3), torch.tensor(0.98))
    a[pos % 37 == 5, 2] = 1e-20
    a[pos % 11 == 3, 2] = 1.0
    inp["a"] = a
    o, ST = _gpu_prefill(inp)
    o_ref, S_ref = _oracle_prefill(inp)
    _check(o, ST, o_ref, S_ref, fp32=False, inp=inp)
    _status_ok()


def test_prefill_tc_segmented_equals_single_pass_and_oracle():
    """Few long chains take the segmented schedule (segment 0 in full from S0;
    later segments' contributions from a zero state and dk x dk transitions,
    chained in fp32, then segments 1 .. P-1 from their start states); two
    sequences, so every per-sequence slot of the workspace is used.
    GDN_SINGLE_PASS runs the same inputs as one pass per chain."""
    wl = _wl("long_prefill", n_seq=2, H=2, seq_len=1000, random_s0=True)
    assert lla.prefill_workspace_bytes(2, 1000, 2, 128, 128) > 0
    inp = W.prefill_inputs(wl, "cpu")
    o_s, S_s = _gpu_prefill(inp)
    o_1, S_1 = _gpu_prefill(inp, flags=lla.GDN_SINGLE_PASS)
    o_ref, S_ref = _oracle_prefill(inp)
    _check(o_s, S_s, o_ref, S_ref, fp32=False, inp=inp)
    _check(o_1, S_1, o_ref, S_ref, fp32=False, inp=inp)
    assert rel_l2(o_s, o_1) < TOL_BF16_O and rel_l2(S_s, S_1) < TOL_BF16_S
    _status_ok()


def test_prefill_tc_corrected_schedule_with_and_without_final_state():
    """The corrected segmented schedule (zero-start outputs of segments 1 .. P-1
    plus qhat^T S_p from their chained start states): with a final state the
    combine also chains S_T; without one it stops at S_{P-1}.  Both give the
    oracle's outputs, and the same outputs bit for bit (the correction does
    not depend on the last combine step)."""
    wl = _wl("long_prefill", n_seq=2, H=2, seq_len=1000, random_s0=True)
    sched = lla.prefill_schedule(2, 1000, 2, 128, 128)
    assert sched["corrected"] == 1 and sched["n_segs"] > 2
    assert lla.prefill_schedule(2, 1000, 2, 128, 128, with_state=False)["launches"] == 3
    inp = W.prefill_inputs(wl, "cpu")
    q, k, v, a, b, s0 = (inp[n].cuda() for n in ("q", "k", "v", "a", "b", "S0"))
    o1, ST = lla.gdn_chunk_fwd(q, k, v, a, b, s0, n_seq=2)
    o2, none = lla.gdn_chunk_fwd(q, k, v, a, b, s0, n_seq=2, return_state=False)
    torch.cuda.synchronize()
    _status_ok()
    assert none is None and torch.equal(o1, o2)
    o_ref, S_ref = _oracle_prefill(inp)
    _check(host(o1), host(ST), o_ref, S_ref, fp32=False, inp=inp)


def test_prefill_tc_segmented_dv256_l2norm_scale():
    """Segmented schedule with two dv slices per head (plus the transition
    slice), in-kernel L2 norm and an output scale."""
    wl = dataclasses.replace(W.WORKLOADS["varlen"], name="seg256", varlen=False, n_seq=1, H=2,
                             seq_len=777, normalize_qk=False)
    assert lla.prefill_workspace_bytes(1, 777, 2, 128, 256) > 0
    inp = W.prefill_inputs(wl, "cpu")
    o, ST = _gpu_prefill(inp, scale=0.125, flags=lla.GDN_QK_L2NORM)
    o_ref, S_ref = _oracle_prefill(inp, scale=0.125, normalize=True)
    _check(o, ST, o_ref, S_ref, fp32=False, inp=inp)
    _status_ok()


def test_prefill_tc_segmented_strong_decay_in_place():
    """Segment transitions under hard decay (a = 0.05: the transition is nearly
    zero) and mild decay (a = 0.999), with S_T written over S0."""
    wl = _wl("long_prefill", n_seq=1, H=2, seq_len=2000, random_s0=True)
    inp = W.prefill_inputs(wl, "cpu")
    a = inp["a"].clone()
    a[:, 0] = 0.05
    a[:, 1] = 0.999
    inp["a"] = a
    o, ST = _gpu_prefill(inp, alias=True)
    o_ref, S_ref = _oracle_prefill(inp)
    _check(o, ST, o_ref, S_ref, fp32=False, inp=inp)
    _status_ok()


def test_bounded_wait_runs_out_and_context_stays_usable():
    """Failure detection on the device: GDN_TEST_WAIT_TIMEOUT makes one wait of
    the tensor-core prefill wait on a barrier that nothing arrives.  The wait
    gives up after about 2 s, the block aborts every other wait, drains its
    copies and frees tensor memory; the host reads GDN_ERR_TIMEOUT, and the next
    call on the same context runs and matches the oracle."""
    wl = _wl("long_prefill", n_seq=1, H=1, seq_len=200, random_s0=True)
    inp = W.prefill_inputs(wl, "cpu")
    q, k, v, a, b = (inp[n].cuda() for n in ("q", "k", "v", "a", "b"))
    lla.gdn_chunk_fwd(q, k, v, a, b, inp["S0"].cuda(), n_seq=1, flags=lla.GDN_TEST_WAIT_TIMEOUT)
    torch.cuda.synchronize()
    assert lla.gdn_get_device_status() == lla.GDN_ERR_TIMEOUT
    assert lla.gdn_get_device_status() == lla.GDN_OK          # reading clears the word
    o, ST = _gpu_prefill(inp)
    o_ref, S_ref = _oracle_prefill(inp)
    _check(o, ST, o_ref, S_ref, fp32=False, inp=inp)
    _status_ok()


def test_prefill_tc_zero_initial_state():
    wl = _wl("long_prefill", n_seq=1, H=2, seq_len=192)
    inp = W.prefill_inputs(wl, "cpu")
    o, ST = _gpu_prefill(inp)
    o_ref, S_ref = _oracle_prefill(inp)
    _check(o, ST, o_ref, S_ref, fp32=False, inp=inp)


def test_prefill_tc_varlen_dv256_l2norm():
    wl = _wl("varlen", H=2, normalize_qk=False)
    inp = W.prefill_inputs(wl, "cpu", lengths=[0, 1, 63, 64, 65, 129, 700])
    o, ST = _gpu_prefill(inp, scale=0.125, flags=lla.GDN_QK_L2NORM)
    o_ref, S_ref = _oracle_prefill(inp, scale=0.125, normalize=True)
    _check(o, ST, o_ref, S_ref, fp32=False, inp=inp)
    np.testing.assert_array_equal(ST[0].numpy(), inp["S0"][0].numpy())
    _status_ok()


def test_varlen_longest_first_order_matches_natural_order():
    """With more blocks than one wave a varlen call launches its sequences
    longest first (an order sorted on the device into the workspace).  Each
    chain's arithmetic does not depend on where it runs, so the outputs equal
    those of the natural order (no workspace) bit for bit; lengths include 0,
    1, a full chunk and ties; both agree with the oracle."""
    import ctypes
    from looped_linear_attention_b200 import _binding as B
    lengths = [0, 1, 64, 65, 700, 300, 300, 129, 5, 640] * 4       # 40 sequences
    wl = _wl("varlen", H=4, dv=128, random_s0=True)                 # 40 x 4 = 160 blocks
    inp = W.prefill_inputs(wl, "cpu", lengths=lengths)
    assert lla.prefill_schedule(len(lengths), 100, 4, 128, 128, varlen=True)["launches"] == 2
    o_lpt, S_lpt = _gpu_prefill(inp)                                 # the binding passes the workspace
    q, k, v, a, b, s0 = (inp[n].cuda() for n in ("q", "k", "v", "a", "b", "S0"))
    cu = torch.from_numpy(inp["cu_seqlens"]).cuda()
    o = torch.full_like(q[:, :, :128], float("nan"))
    S_T = torch.full_like(s0, float("nan"))
    p = B.gdn_fwd_params(q.data_ptr(), k.data_ptr(), v.data_ptr(), a.data_ptr(), b.data_ptr(),
                         s0.data_ptr(), o.data_ptr(), S_T.data_ptr(), cu.data_ptr(), len(lengths), 0,
                         inp["total_tokens"], 4, 128, 128, B.GDN_BF16, 1.0, 0)
    assert lla.library().gdn_chunk_fwd(ctypes.byref(p), None, 0, None) == lla.GDN_OK
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(host(o), o_lpt) and torch.equal(host(S_T), S_lpt)
    o_ref, S_ref = _oracle_prefill(inp)
    _check(o_lpt, S_lpt, o_ref, S_ref, fp32=False, inp=inp)


def test_varlen_longest_first_in_place_state_and_graph_capture():
    """A multi-wave varlen call (length sort, then the prefill in that order)
    with S_T written over S0, against the oracle; the same call captured in a
    CUDA graph and replayed gives the eager call's outputs bit for bit."""
    lengths = [700, 0, 64, 1, 300, 129, 65, 640, 300, 5] * 4
    wl = _wl("varlen", H=4, dv=128, random_s0=True)
    inp = W.prefill_inputs(wl, "cpu", lengths=lengths)
    o, ST = _gpu_prefill(inp, alias=True)
    o_ref, S_ref = _oracle_prefill(inp)
    _check(o, ST, o_ref, S_ref, fp32=False, inp=inp)
    q, k, v, a, b = (inp[n].cuda() for n in ("q", "k", "v", "a", "b"))
    s0 = inp["S0"].cuda()
    cu = torch.from_numpy(inp["cu_seqlens"]).cuda()
    o_e, S_e = lla.gdn_chunk_fwd(q, k, v, a, b, s0, cu)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        o_g, S_g = lla.gdn_chunk_fwd(q, k, v, a, b, s0, cu)
    o_g.zero_()
    S_g.zero_()
    graph.replay()
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(o_g, o_e) and torch.equal(S_g, S_e)


def _bwd_case(wl, lengths=None, n_seq=None, seq_len=None, grad_ST=True):
    inp = W.prefill_inputs(wl, "cpu", lengths=lengths, n_seq=n_seq, seq_len=seq_len)
    g = torch.Generator().manual_seed(W.seed_for("test", "bwd", wl.name, inp["total_tokens"]))
    go = torch.randn(inp["v"].shape, generator=g).to(inp["v"].dtype)
    gST = (torch.randn(inp["n_seq"], wl.H, wl.dk, wl.dv, generator=g) if grad_ST else None)
    return inp, go, gST


BWD_PATHS = {"chunkwise": 0, "token": lla.GDN_PRECISE}


def _bwd_check(inp, go, gST, scale, flags=0):
    """Every gradient against the oracle's reverse mode: relative L2 below 1e-4
    over the whole tensor and, for the per-token gradients, per sequence."""
    dev = lambda t: None if t is None else t.cuda()
    cu = None if inp["cu_seqlens"] is None else torch.from_numpy(inp["cu_seqlens"]).cuda()
    grads = lla.gdn_chunk_bwd(*(inp[n].cuda() for n in ("q", "k", "v", "a", "b")), go.cuda(),
                              dev(inp["S0"]), dev(gST), cu, n_seq=inp["n_seq"], scale=scale, flags=flags)
    torch.cuda.synchronize()
    _status_ok()
    cu_h = inp["cu_seqlens"]
    if cu_h is None:
        cu_h = np.arange(inp["n_seq"] + 1, dtype=np.int32) * inp["seq_len"]
    ref = oracle.gdn_bwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], go, inp["S0"], gST, cu_h, scale)
    for name, rname in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("a", "da"), ("b", "db"), ("S0", "dS0")):
        got = host(grads[name])
        err = rel_l2(got, ref[rname])
        assert err < TOL_F32, (name, err)
        if name != "S0":
            for s in range(len(cu_h) - 1):
                t0, t1 = int(cu_h[s]), int(cu_h[s + 1])
                if t1 > t0 and np.linalg.norm(ref[rname][t0:t1]) > 0:
                    e = rel_l2(got[t0:t1], ref[rname][t0:t1])
                    assert e < TOL_F32, (name, s, e)
    return grads


@pytest.mark.parametrize("path", list(BWD_PATHS))
def test_backward_fp32_fixed_length_matches_oracle(path):
    """Reverse mode on the GPU (chunks of 64 tokens, ragged last chunk) against
    the oracle's: two sequences of 150 tokens, random S0 and final-state
    gradient, scale 0.5, fp32 inputs; relative L2 per gradient below 1e-4."""
    wl = _wl("tiny", H=2, dk=64, dv=64, random_s0=True, normalize_qk=True)
    inp, go, gST = _bwd_case(wl, n_seq=2, seq_len=150)
    _bwd_check(inp, go, gST, 0.5, BWD_PATHS[path])


@pytest.mark.parametrize("path", list(BWD_PATHS))
def test_backward_bf16_varlen_matches_oracle(path):
    """bf16 inputs (compared on their exact values), varlen lengths 0, 1, 64,
    65, 200, dk = dv = 128."""
    wl = _wl("varlen", H=2, dv=128, random_s0=True)
    inp, go, gST = _bwd_case(wl, lengths=[0, 1, 64, 65, 200])
    _bwd_check(inp, go, gST, 1.0, BWD_PATHS[path])


@pytest.mark.parametrize("path", list(BWD_PATHS))
def test_backward_dv256_without_start_state_or_state_gradient(path):
    wl = _wl("long_prefill", n_seq=1, H=1, dv=256, random_s0=False)
    inp, go, gST = _bwd_case(wl, n_seq=1, seq_len=100, grad_ST=False)
    _bwd_check(inp, go, gST, 1.0, BWD_PATHS[path])


def test_backward_chunkwise_long_chain_matches_oracle():
    """One 1024-token chain of the timed backward workload's shape (16 chunks,
    so the chunk start states and end-state gradients are chained 15 times),
    2 heads, bf16, random S0 and final-state gradient."""
    wl = _wl("long_prefill", n_seq=1, H=2, random_s0=True)
    inp, go, gST = _bwd_case(wl, n_seq=1, seq_len=1024)
    _bwd_check(inp, go, gST, 1.0)


def test_backward_chunkwise_equals_token_path_at_full_size():
    """At the timed backward workload's full size (8 x 1024 tokens, 16 heads,
    dk = dv = 128, bf16) the chunkwise path and the token-by-token path (two
    independent kernels) agree within 1e-4 on every gradient."""
    wl = _wl("long_prefill", n_seq=8, random_s0=True)
    inp = W.prefill_inputs(wl, "cuda", n_seq=8, seq_len=1024)
    g = torch.Generator(device="cuda").manual_seed(W.seed_for("test", "bwd-full"))
    go = torch.randn(inp["v"].shape, generator=g, device="cuda").to(wl.dtype)
    gST = torch.randn(8, wl.H, wl.dk, wl.dv, generator=g, device="cuda")
    args = ([inp[n] for n in ("q", "k", "v", "a", "b")] + [go, inp["S0"], gST])
    ch = lla.gdn_chunk_bwd(*args, n_seq=8)
    tk = lla.gdn_chunk_bwd(*args, n_seq=8, flags=lla.GDN_PRECISE)
    torch.cuda.synchronize()
    _status_ok()
    for name in ("q", "k", "v", "a", "b", "S0"):
        err = float(torch.linalg.vector_norm(ch[name] - tk[name]) / torch.linalg.vector_norm(tk[name]))
        assert err < TOL_F32, (name, err)


def test_prefill_tc_in_place_state():
    wl = _wl("long_prefill", n_seq=2, H=2, seq_len=130, random_s0=True)
    inp = W.prefill_inputs(wl, "cpu")
    o, ST = _gpu_prefill(inp, alias=True)
    o_ref, S_ref = _oracle_prefill(inp)
    _check(o, ST, o_ref, S_ref, fp32=False, inp=inp)


def test_prefill_tc_matches_precise_path_and_oracle():
    wl = _wl("long_prefill", n_seq=1, H=2, seq_len=640, random_s0=True)
    inp = W.prefill_inputs(wl, "cpu")
    o_tc, S_tc = _gpu_prefill(inp)
    o_pr, S_pr = _gpu_prefill(inp, flags=lla.GDN_PRECISE)
    o_ref, S_ref = _oracle_prefill(inp)
    _check(o_tc, S_tc, o_ref, S_ref, fp32=False, inp=inp)
    # the fp32 path only sees bf16 rounding of its outputs
    assert rel_l2(o_pr, o_ref) < 4e-3 and rel_l2(S_pr, S_ref) < TOL_F32


def test_prefill_tc_is_deterministic():
    wl = _wl("long_prefill", n_seq=2, H=2, seq_len=257, random_s0=True)
    inp = W.prefill_inputs(wl, "cpu")
    o1, S1 = _gpu_prefill(inp)
    o2, S2 = _gpu_prefill(inp)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_prefill_split_and_resume():
    """[0, m) then [m, L) with the state carried equals one pass (m not a
    multiple of the chunk)."""
    wl = _wl("long_prefill", n_seq=1, H=2, seq_len=1000)
    inp = W.prefill_inputs(wl, "cpu")
    m = 333
    first = {k: (v[:m] if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    first.update(seq_len=m, total_tokens=m)
    second = {k: (v[m:] if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    second.update(seq_len=1000 - m, total_tokens=1000 - m)
    o1, S1 = _gpu_prefill(first)
    o2, S2 = _gpu_prefill(second, S0=S1)
    o_ref, S_ref = _oracle_prefill(inp)
    _check(torch.cat([o1, o2]), S2, o_ref, S_ref, fp32=False, inp=inp)


def test_decode_continues_prefill():
    wl = _wl("long_prefill", n_seq=1, H=2, seq_len=201)
    inp = W.prefill_inputs(wl, "cpu")
    L = 200
    pre = {k: (v[:L] if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    pre.update(seq_len=L, total_tokens=L)
    _, S_L = _gpu_prefill(pre)
    S = S_L.cuda()
    o_d = lla.gdn_decode_step(*(inp[n][L:].cuda() for n in ("q", "k", "v", "a", "b")), S)
    torch.cuda.synchronize()
    o_ref, S_ref = _oracle_prefill(inp)
    assert rel_l2(host(o_d)[0], o_ref[L]) < TOL_BF16_O
    assert rel_l2(host(S), S_ref) < TOL_BF16_S


# ------------------------------------------------------------------ full-size workloads, sampled
def _sample_chain_check(inp, o, ST, chains):
    cu = inp["cu_seqlens"]
    for s, h in chains:
        if cu is None:
            t0, t1 = s * inp["seq_len"], (s + 1) * inp["seq_len"]
        else:
            t0, t1 = int(cu[s]), int(cu[s + 1])
        sl = slice(t0, t1)
        s0 = None if inp["S0"] is None else host(inp["S0"][s:s + 1, h:h + 1])
        o_ref, S_ref = oracle.gdn_fwd(host(inp["q"][sl, h:h + 1]), host(inp["k"][sl, h:h + 1]),
                                      host(inp["v"][sl, h:h + 1]), host(inp["a"][sl, h:h + 1]),
                                      host(inp["b"][sl, h:h + 1]), s0)
        _check(host(o[sl, h:h + 1]), host(ST[s:s + 1, h:h + 1]), o_ref, S_ref, fp32=False,
               bounds=[(0, t1 - t0)])


def test_full_long_prefill_sampled():
    """B=8, H=16, L=16384, dk=dv=128 bf16, one loop launched as the benchmark does."""
    wl = W.WORKLOADS["long_prefill"]
    inp = W.prefill_inputs(wl, "cuda")
    o, ST = lla.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], None, None,
                              n_seq=wl.n_seq)
    torch.cuda.synchronize()
    _status_ok()
    _sample_chain_check(inp, o, ST, [(0, 0), (7, 15), (3, 9)])


def test_full_looped_shape_segmented_sampled():
    """The looped workload's mixer shape (one 4096-token sequence x 16 heads)
    runs the segmented schedule, as in the benchmark; sampled heads against the
    oracle, outputs and final states."""
    wl = W.WORKLOADS["looped_prefill"]
    assert lla.prefill_workspace_bytes(1, wl.seq_len, wl.H, wl.dk, wl.dv) > 0
    inp = W.prefill_inputs(wl, "cuda")
    o, ST = lla.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], None, None,
                              n_seq=1)
    torch.cuda.synchronize()
    _status_ok()
    _sample_chain_check(inp, o, ST, [(0, 0), (0, 7), (0, 15)])


def test_full_varlen_sampled():
    """64 sequences, lengths U[512, 32768], H=16, dk=128, dv=256, random S0."""
    wl = W.WORKLOADS["varlen"]
    inp = W.prefill_inputs(wl, "cuda")
    cu = torch.from_numpy(inp["cu_seqlens"]).cuda()
    o, ST = lla.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["S0"], cu)
    torch.cuda.synchronize()
    _status_ok()
    lens = np.diff(inp["cu_seqlens"])
    chains = [(int(np.argmin(lens)), 0), (int(np.argmax(lens)), 5), (17, 11)]
    _sample_chain_check(inp, o, ST, chains)
    del inp, o, ST
    torch.cuda.empty_cache()


def test_full_decode_sampled():
    """24576 slots x 16 heads, 128 x 128 fp32 states, in place."""
    wl = W.WORKLOADS["decode"]
    inp = W.decode_inputs(wl, "cuda")
    rng = np.random.default_rng(0)
    slots = np.sort(rng.choice(wl.n_seq, 24, replace=False))
    S_before = host(inp["S"][slots])
    o = lla.gdn_decode_step(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["S"])
    torch.cuda.synchronize()
    _status_ok()
    o_ref, S_ref = oracle.gdn_decode(host(inp["q"][slots]), host(inp["k"][slots]),
                                     host(inp["v"][slots]), host(inp["a"][slots]),
                                     host(inp["b"][slots]), S_before)
    assert rel_l2(host(o[slots]), o_ref) < 4e-3
    assert rel_l2(host(inp["S"][slots]), S_ref) < TOL_F32
    del inp
    torch.cuda.empty_cache()


def test_looped_prefill_end_to_end():
    """B=1, L=4096, d=2048 (16 heads x 128), T=4 loops of projection -> GDN
    (q, k normalised in-kernel) -> loop residual, against the oracle's own chain."""
    wl = W.WORKLOADS["looped_prefill"]
    inp = W.looped_inputs(wl, "cpu")
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    runner = lla.LoopedPrefill(inp["L"], wl.H, wl.dk, wl.dv, wl.loops, "cuda")
    hT = runner.run(dev["h0"], dev["Wq"], dev["Wk"], dev["Wv"], dev["a"], dev["b"], dev["rho"])
    torch.cuda.synchronize()
    _status_ok()
    ref = oracle.looped_forward(inp["h0"], inp["Wq"], inp["Wk"], inp["Wv"], inp["a"], inp["b"],
                                inp["rho"], wl.H, wl.dk, wl.dv)
    assert rel_l2(host(hT), ref) < TOL_BF16_O
    # first loop's mixer on identical projections
    L, d = inp["L"], inp["d"]
    q = (dev["h0"] @ dev["Wq"]).view(L, wl.H, wl.dk)
    k = (dev["h0"] @ dev["Wk"]).view(L, wl.H, wl.dk)
    v = (dev["h0"] @ dev["Wv"]).view(L, wl.H, wl.dv)
    o, _ = lla.gdn_chunk_fwd(q, k, v, dev["a"][0].contiguous(), dev["b"][0].contiguous(),
                             flags=lla.GDN_QK_L2NORM)
    o_ref, _ = oracle.gdn_fwd(oracle.qk_l2norm(host(q)), oracle.qk_l2norm(host(k)), host(v),
                              inp["a"][0], inp["b"][0])
    assert rel_l2(host(o), o_ref) < TOL_BF16_O


def test_looped_step_same_with_stacked_or_separate_weights():
    """The batched q/k/v projection gives the same h^(T) whether the weights
    come as planes of one [3, d, d] tensor (used in place) or as three separate
    tensors (stacked by the runner)."""
    wl = dataclasses.replace(W.WORKLOADS["looped_prefill"], seq_len=256)
    inp = W.looped_inputs(wl, "cuda")
    runner = lla.LoopedPrefill(inp["L"], wl.H, wl.dk, wl.dv, wl.loops, "cuda")
    args = (inp["a"], inp["b"], inp["rho"])
    h_view = runner.run(inp["h0"], inp["Wq"], inp["Wk"], inp["Wv"], *args).clone()
    h_sep = runner.run(inp["h0"], inp["Wq"].clone(), inp["Wk"].clone(), inp["Wv"].clone(), *args)
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(h_view, h_sep)


def test_looped_step_graph_replay_equals_stream_run():
    """The looped step captured in a CUDA graph (the segmented mixer's
    dependent launches included) gives the stream-launched step's h^(T) bit for
    bit, and again after its inputs are overwritten in place."""
    wl = dataclasses.replace(W.WORKLOADS["looped_prefill"], seq_len=1024)
    inp = W.looped_inputs(wl, "cuda")
    assert lla.prefill_schedule(1, 1024, wl.H, wl.dk, wl.dv)["n_segs"] > 1
    runner = lla.LoopedPrefill(inp["L"], wl.H, wl.dk, wl.dv, wl.loops, "cuda")
    W3 = (inp["Wq"], inp["Wk"], inp["Wv"])
    out = torch.empty(inp["L"], inp["d"], dtype=torch.bfloat16, device="cuda")
    graph, h = runner.capture(inp["h0"], *W3, inp["a"], inp["b"], inp["rho"], out=out)
    assert h.data_ptr() == out.data_ptr()
    for i in range(2):
        if i:
            g = torch.Generator(device="cuda").manual_seed(W.seed_for("test", "graph", i))
            inp["h0"].copy_(torch.randn(inp["h0"].shape, generator=g, device="cuda"))
            inp["a"].pow_(1.05)
        graph.replay()
        torch.cuda.synchronize()
        got = out.clone()
        ref = runner.run(inp["h0"], *W3, inp["a"], inp["b"], inp["rho"]).clone()
        torch.cuda.synchronize()
        _status_ok()
        assert torch.equal(got, ref)


def test_host_pipeline_matches_device_steps():
    """HostPipeline (pinned host inputs and results, copies overlapped with the
    neighbouring steps' compute) gives the same h^(T) as LoopedPrefill.run on
    device inputs, step by step, for three different inputs in a row."""
    wl = dataclasses.replace(W.WORKLOADS["looped_prefill"], seq_len=512)
    base = W.looped_inputs(wl, "cpu")
    L, d = base["L"], base["d"]
    runner = lla.LoopedPrefill(L, wl.H, wl.dk, wl.dv, wl.loops, "cuda")
    pipe = lla.HostPipeline(runner, "cuda")
    W_dev = [base[n].cuda() for n in ("Wq", "Wk", "Wv")]
    rho = base["rho"].cuda()
    g = torch.Generator().manual_seed(W.seed_for("test", "host-pipeline"))
    steps = []
    for i in range(3):
        h0 = torch.randn(L, d, generator=g).bfloat16().pin_memory()
        a = (base["a"] ** (1.0 + 0.1 * i)).contiguous().pin_memory()
        b = base["b"].clone().pin_memory()
        out = torch.empty(L, d, dtype=torch.bfloat16).pin_memory()
        steps.append((h0, a, b, out))
        pipe.submit(h0, a, b, out, *W_dev, rho)
    pipe.join()
    torch.cuda.synchronize()
    _status_ok()
    for h0, a, b, out in steps:
        ref = runner.run(h0.cuda(), *W_dev, a.cuda(), b.cuda(), rho)
        torch.cuda.synchronize()
        assert torch.equal(out, host(ref))
