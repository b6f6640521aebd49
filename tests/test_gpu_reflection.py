"""GPU parity in the reflection regime of the update, write strength b in (1, 2].

With unit keys, I - b k k^T has spectral norm <= 1 for every b in [0, 2]; at
b = 2 it is the Householder reflection through k, and products of such
factors realise the permutations of the state's rows (S_n prefix products) and,
by Cartan-Dieudonne, any orthogonal map ("LT2: Linear-Time Looped
Transformers", §2 and Appendix B.1).  This is where the chunk's (I + A) has
its largest off-diagonal entries, so every kernel is checked here against the
oracle at the usual bars (relative L2 1e-2 on bf16 outputs, 5e-3 on states,
1e-4 for fp32 work), with the per-sequence and worst-chunk bars of gpu_util:
  * b ~ U(1, 2) on the tensor-core prefill (one pass, segmented, varlen with
    the in-kernel q/k norm), the precise prefill, decode (streaming and
    register kernels) and the reverse mode;
  * a chain of exact transpositions of a 128-row state (a = 1, b = 2, v = 0,
    keys e_i - e_j normalised in the kernel, and the same swaps written as
    I - k k^T with b = 1 on raw keys);
  * a chain of 128 Householder reflections (random unit keys, b = 2) that
    realises a random orthogonal map of a 128 x 128 state.
The exact-reflection chains (a = 1 throughout, every chunk a full rotation of
the state) are the one regime where the bf16 operands of the tensor-core path
(the state, W, U and T, each rounded once per chunk) add up past the 5e-3
state bar: about 6.3e-3 after one to five chunks, reproduced by a CPU
emulation of those roundings.  There the fp32 chunk kernel (GDN_PRECISE) is
the path that meets the bars; the tensor-core error is still checked, against
1e-2, as a regression guard and not as a parity claim.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import looped_linear_attention_b200 as lla
from looped_linear_attention_b200 import workloads as W
from gpu_util import TOL_BF16_O, TOL_BF16_S, TOL_F32, check_prefill, host, rel_l2, seq_bounds

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


def _reflective_b(inp, label, lo=1.0, hi=2.0):
    """Replaces b by U(lo, hi) draws (seeded), in place of the workload's sigmoid gate."""
    g = torch.Generator().manual_seed(W.seed_for("test", "reflection", label))
    inp["b"] = lo + (hi - lo) * torch.rand(inp["b"].shape, generator=g)
    return inp


def _run(inp, scale=1.0, flags=0):
    q, k, v, a, b = (inp[n].cuda() for n in ("q", "k", "v", "a", "b"))
    s0 = None if inp["S0"] is None else inp["S0"].cuda()
    cu = None if inp["cu_seqlens"] is None else torch.from_numpy(inp["cu_seqlens"]).cuda()
    o, ST = lla.gdn_chunk_fwd(q, k, v, a, b, s0, cu, n_seq=inp["n_seq"], scale=scale, flags=flags)
    torch.cuda.synchronize()
    _status_ok()
    return host(o), host(ST)


def _ref(inp, scale=1.0, normalize=False):
    q, k = inp["q"], inp["k"]
    if normalize:
        q, k = oracle.qk_l2norm(q), oracle.qk_l2norm(k)
    cu = inp["cu_seqlens"]
    if cu is None:
        cu = np.arange(inp["n_seq"] + 1, dtype=np.int32) * inp["seq_len"]
    return oracle.gdn_fwd(q, k, inp["v"], inp["a"], inp["b"], inp["S0"], cu, scale)


# ------------------------------------------------------------------ b ~ U(1, 2)
def test_prefill_tc_one_pass_b_in_1_2():
    wl = _wl("long_prefill", n_seq=2, H=3, seq_len=333, random_s0=True)
    inp = _reflective_b(W.prefill_inputs(wl, "cpu"), "one-pass")
    o, ST = _run(inp, flags=lla.GDN_SINGLE_PASS)
    o_ref, S_ref = _ref(inp)
    check_prefill(o, ST, o_ref, S_ref, seq_bounds(inp), fp32=False)


def test_prefill_tc_segmented_b_in_1_2_mixed_decay():
    """Segmented schedule (segment transitions chained in fp32) with b ~ U(1, 2);
    head 1 decays hard (a = 0.05) so that the exponential path of the decay
    matrix is taken too."""
    wl = _wl("long_prefill", n_seq=1, H=2, seq_len=2000, random_s0=True)
    assert lla.prefill_schedule(1, 2000, 2, 128, 128)["n_segs"] > 1
    inp = _reflective_b(W.prefill_inputs(wl, "cpu"), "segmented")
    inp["a"][:, 1] = 0.05
    o, ST = _run(inp)
    o_ref, S_ref = _ref(inp)
    check_prefill(o, ST, o_ref, S_ref, seq_bounds(inp), fp32=False)


def test_prefill_tc_varlen_dv256_b_in_1_2_l2norm():
    wl = _wl("varlen", H=2, normalize_qk=False)
    inp = _reflective_b(W.prefill_inputs(wl, "cpu", lengths=[0, 1, 63, 64, 65, 129, 700]), "varlen")
    o, ST = _run(inp, scale=0.125, flags=lla.GDN_QK_L2NORM)
    o_ref, S_ref = _ref(inp, scale=0.125, normalize=True)
    check_prefill(o, ST, o_ref, S_ref, seq_bounds(inp), fp32=False)


def test_prefill_precise_b_in_1_2():
    """fp32 inputs on the fp32 chunk kernel: the 1e-4 bar."""
    wl = _wl("tiny", n_seq=2, H=2, seq_len=200, random_s0=True)
    inp = _reflective_b(W.prefill_inputs(wl, "cpu"), "precise")
    o, ST = _run(inp, scale=0.5)
    o_ref, S_ref = _ref(inp, scale=0.5)
    check_prefill(o, ST, o_ref, S_ref, seq_bounds(inp), fp32=True)


@pytest.mark.parametrize("dk,dv,dtype", [(128, 128, torch.bfloat16), (64, 192, torch.float32)])
def test_decode_b_in_1_2(dk, dv, dtype):
    """The streaming kernel (dk = dv = 128, bf16) and the register kernel."""
    wl = _wl("decode", dk=dk, dv=dv, dtype=dtype, H=3)
    inp = W.decode_inputs(wl, "cpu", n_slots=41)
    _reflective_b(inp, f"decode-{dk}-{dv}")
    S = inp["S"].cuda()
    o = lla.gdn_decode_step(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), inp["a"].cuda(),
                            inp["b"].cuda(), S, scale=0.75)
    torch.cuda.synchronize()
    _status_ok()
    o_ref, S_ref = oracle.gdn_decode(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["S"], 0.75)
    tol_o = TOL_F32 if dtype == torch.float32 else 4e-3   # bf16 output rounding
    assert rel_l2(host(o), o_ref) < tol_o
    assert rel_l2(host(S), S_ref) < TOL_F32


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_backward_b_in_1_2(dtype):
    """Reverse mode with b ~ U(1, 2): every gradient within 1e-4 of the oracle's."""
    wl = _wl("long_prefill", n_seq=2, H=2, seq_len=150, dk=64 if dtype == torch.float32 else 128,
             dv=64 if dtype == torch.float32 else 128, dtype=dtype, random_s0=True)
    inp = _reflective_b(W.prefill_inputs(wl, "cpu"), f"bwd-{dtype}")
    g = torch.Generator().manual_seed(W.seed_for("test", "reflection", "bwd", str(dtype)))
    go = torch.randn(inp["v"].shape, generator=g).to(dtype)
    gST = torch.randn(2, wl.H, wl.dk, wl.dv, generator=g)
    grads = lla.gdn_chunk_bwd(*(inp[n].cuda() for n in ("q", "k", "v", "a", "b")), go.cuda(),
                              inp["S0"].cuda(), gST.cuda(), n_seq=2, scale=0.5)
    torch.cuda.synchronize()
    _status_ok()
    cu = np.arange(3, dtype=np.int32) * 150
    ref = oracle.gdn_bwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], go, inp["S0"], gST, cu, 0.5)
    for name, rname in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("a", "da"), ("b", "db"), ("S0", "dS0")):
        assert rel_l2(host(grads[name]), ref[rname]) < TOL_F32, name


# ------------------------------------------------------------------ exact reflections
def _swap_chain(L, H, n, label):
    """L random transpositions (i j) per head: keys e_i - e_j, plus the pairs."""
    rng = np.random.default_rng(W.seed_for("test", "swaps", label) % (1 << 32))
    k = np.zeros((L, H, n), dtype=np.float32)
    pairs = np.zeros((L, H, 2), dtype=np.int64)
    for t in range(L):
        for h in range(H):
            i, j = rng.choice(n, 2, replace=False)
            k[t, h, i], k[t, h, j] = 1.0, -1.0
            pairs[t, h] = (i, j)
    return k, pairs


def _permuted(S0, pairs):
    """S0 [H, n, dv] with rows i and j swapped for every pair in order."""
    S = S0.copy()
    for t in range(pairs.shape[0]):
        for h in range(pairs.shape[1]):
            i, j = pairs[t, h]
            S[h, [i, j]] = S[h, [j, i]]
    return S


@pytest.mark.parametrize("normalised", [True, False])
def test_transposition_chain_permutes_state_rows(normalised):
    """a = 1, v = 0 and keys e_i - e_j: with the in-kernel norm and b = 2 every
    token is the reflection through the unit key (e_i - e_j)/sqrt(2); without
    it, b = 1 on the raw key gives I - k k^T, the same swap.  300 tokens
    (several chunks and a ragged one) over a 128 x 128 state: the oracle's
    final state is S0 with its rows permuted, and the tensor-core prefill
    matches the oracle."""
    L, H, n = 300, 2, 128
    k_np, pairs = _swap_chain(L, H, n, f"perm-{normalised}")
    g = torch.Generator().manual_seed(W.seed_for("test", "swaps", "q", normalised))
    q = W._l2norm(torch.randn(L, H, n, generator=g)).bfloat16()
    S0 = torch.randn(1, H, n, n, generator=g)
    inp = dict(q=q, k=torch.from_numpy(k_np).bfloat16(), v=torch.zeros(L, H, n, dtype=torch.bfloat16),
               a=torch.ones(L, H), b=torch.full((L, H), 2.0 if normalised else 1.0), S0=S0,
               cu_seqlens=None, n_seq=1, seq_len=L, total_tokens=L)
    flags = lla.GDN_QK_L2NORM if normalised else 0
    o_ref, S_ref = _ref(inp, normalize=normalised)
    perm = _permuted(S0[0].numpy().astype(np.float64), pairs)
    # the oracle realises the permutation (up to the norm's eps with the flag)
    assert rel_l2(S_ref[0], perm) < (1e-4 if normalised else 1e-12)
    _exact_reflection_checks(inp, flags, o_ref, S_ref, L)


def _exact_reflection_checks(inp, flags, o_ref, S_ref, L):
    """GDN_PRECISE meets the bars (fp32 state error, bf16 output rounding);
    the tensor-core path stays within its measured envelope.  With the q/k
    norm the precise path works on the normalised vectors rounded to the io
    dtype (its documented contract), so its state is compared with the
    oracle's on those same vectors."""
    o, ST = _run(inp, flags=flags | lla.GDN_PRECISE)
    if flags & lla.GDN_QK_L2NORM:
        rq = torch.from_numpy(oracle.qk_l2norm(inp["q"])).to(inp["q"].dtype)
        rk = torch.from_numpy(oracle.qk_l2norm(inp["k"])).to(inp["k"].dtype)
        o_p, S_p = _ref(dict(inp, q=rq, k=rk))
    else:
        o_p, S_p = o_ref, S_ref
    err = check_prefill(o, ST, o_p, S_p, [(0, L)], fp32=False)
    assert err["S"] < TOL_F32, err
    o, ST = _run(inp, flags=flags)
    assert rel_l2(o, o_ref) < TOL_BF16_O and rel_l2(ST, S_ref) < 2 * TOL_BF16_S


def test_householder_chain_realises_orthogonal_map():
    """128 random unit keys with a = 1, b = 2 and v = 0: the state ends as
    H(k_128) ... H(k_1) S0, a random orthogonal map of the 128 x 128 state
    (Cartan-Dieudonne).  The keys are normalised in fp32 and rounded to bf16,
    so the oracle is compared with the explicit product of the factors
    I - 2 k k^T of those exact keys, and the GPU with the oracle."""
    L, H, n = 128, 2, 128
    g = torch.Generator().manual_seed(W.seed_for("test", "householder"))
    k = W._l2norm(torch.randn(L, H, n, generator=g)).bfloat16()
    q = W._l2norm(torch.randn(L, H, n, generator=g)).bfloat16()
    S0 = torch.randn(1, H, n, n, generator=g)
    inp = dict(q=q, k=k, v=torch.zeros(L, H, n, dtype=torch.bfloat16), a=torch.ones(L, H),
               b=torch.full((L, H), 2.0), S0=S0, cu_seqlens=None, n_seq=1, seq_len=L, total_tokens=L)
    o_ref, S_ref = _ref(inp)
    kd = k.double().numpy()
    for h in range(H):
        P = np.eye(n)
        for t in range(L):
            P = (np.eye(n) - 2.0 * np.outer(kd[t, h], kd[t, h])) @ P
        np.testing.assert_allclose(S_ref[0, h], P @ S0[0, h].double().numpy(), atol=1e-10)
    _exact_reflection_checks(inp, 0, o_ref, S_ref, L)
