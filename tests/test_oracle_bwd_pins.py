"""Pins of the oracle's reverse mode (``oracle.gdn_bwd``) against constructions
that do not re-type its backward loop: central finite differences of the
forward oracle, the closed form of a run with no write and no decay, linearity
in the cotangents, and packed-equals-separate sequences.  A dropped term, a
wrong sign or a state taken one token off fails at least one of them."""
import numpy as np
import pytest

import oracle


def _case(rng, lens, H, dk, dv, s0=True):
    n = int(sum(lens))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q = rng.standard_normal((n, H, dk))
    k = rng.standard_normal((n, H, dk)) / np.sqrt(dk)
    v = rng.standard_normal((n, H, dv))
    a = rng.uniform(0.3, 1.0, (n, H))
    b = rng.uniform(0.0, 2.0, (n, H))
    S0 = rng.standard_normal((len(lens), H, dk, dv)) if s0 else None
    dO = rng.standard_normal((n, H, dv))
    dST = rng.standard_normal((len(lens), H, dk, dv))
    return dict(q=q, k=k, v=v, a=a, b=b, S0=S0, dO=dO, dST=dST, cu=cu)


def _loss(c, scale, **over):
    x = dict(c, **over)
    o, ST = oracle.gdn_fwd(x["q"], x["k"], x["v"], x["a"], x["b"], x["S0"], x["cu"], scale)
    return float((o * c["dO"]).sum() + (ST * c["dST"]).sum())


@pytest.mark.parametrize("lens,scale", [([6], 1.0), ([4, 3], 0.7)])
def test_gradients_match_central_differences(lens, scale):
    rng = np.random.default_rng(sum(lens))
    c = _case(rng, lens, H=2, dk=3, dv=2)
    g = oracle.gdn_bwd(c["q"], c["k"], c["v"], c["a"], c["b"], c["dO"], c["S0"], c["dST"], c["cu"], scale)
    eps = 1e-6
    names = {"q": "dq", "k": "dk", "v": "dv", "a": "da", "b": "db", "S0": "dS0"}
    for name, gname in names.items():
        base = c[name]
        fd = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus, minus = base.copy(), base.copy()
            plus[idx] += eps
            minus[idx] -= eps
            fd[idx] = (_loss(c, scale, **{name: plus}) - _loss(c, scale, **{name: minus})) / (2 * eps)
        np.testing.assert_allclose(g[gname], fd, rtol=1e-6, atol=1e-7, err_msg=name)


def test_no_write_no_decay_closed_form():
    """a = 1, b = 0: every state is S0, so G_t = dS_T + scale sum_{s>=t} q_s dO_s^T,
    dq_t = scale S0 dO_t, dk = dv = 0, da_t = <G_t, S0>,
    db_t = k_t^T G_t (v_t - S0^T k_t) and dS0 = G_1."""
    rng = np.random.default_rng(7)
    c = _case(rng, [5], H=1, dk=4, dv=3)
    L, scale = 5, 0.5
    a, b = np.ones((L, 1)), np.zeros((L, 1))
    g = oracle.gdn_bwd(c["q"], c["k"], c["v"], a, b, c["dO"], c["S0"], c["dST"], None, scale)
    S0, dST = c["S0"][0, 0], c["dST"][0, 0]
    q, k, v, dO = c["q"][:, 0], c["k"][:, 0], c["v"][:, 0], c["dO"][:, 0]
    Gs = [dST + scale * sum(np.outer(q[s], dO[s]) for s in range(t, L)) for t in range(L)]
    np.testing.assert_allclose(g["dq"][:, 0], scale * dO @ S0.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dk"], 0.0, atol=1e-12)
    np.testing.assert_allclose(g["dv"], 0.0, atol=1e-12)
    np.testing.assert_allclose(g["da"][:, 0], [np.sum(G * S0) for G in Gs], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["db"][:, 0], [k[t] @ Gs[t] @ (v[t] - S0.T @ k[t]) for t in range(L)],
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dS0"][0, 0], Gs[0], rtol=1e-12, atol=1e-12)


def test_linear_in_the_cotangents():
    rng = np.random.default_rng(11)
    c = _case(rng, [9], H=2, dk=4, dv=3)
    args = (c["q"], c["k"], c["v"], c["a"], c["b"])
    g1 = oracle.gdn_bwd(*args, c["dO"], c["S0"], c["dST"], None)
    dO2, dST2 = rng.standard_normal(c["dO"].shape), rng.standard_normal(c["dST"].shape)
    g2 = oracle.gdn_bwd(*args, dO2, c["S0"], dST2, None)
    g12 = oracle.gdn_bwd(*args, c["dO"] + 2 * dO2, c["S0"], c["dST"] + 2 * dST2, None)
    for n in g1:
        np.testing.assert_allclose(g12[n], g1[n] + 2 * g2[n], rtol=1e-10, atol=1e-10, err_msg=n)


def test_packed_sequences_equal_separate_calls():
    rng = np.random.default_rng(13)
    lens = [3, 0, 7, 1]
    c = _case(rng, lens, H=2, dk=3, dv=4)
    g = oracle.gdn_bwd(c["q"], c["k"], c["v"], c["a"], c["b"], c["dO"], c["S0"], c["dST"], c["cu"])
    cu = c["cu"]
    for s in range(len(lens)):
        sl = slice(cu[s], cu[s + 1])
        gs = oracle.gdn_bwd(c["q"][sl], c["k"][sl], c["v"][sl], c["a"][sl], c["b"][sl], c["dO"][sl],
                            c["S0"][s:s + 1], c["dST"][s:s + 1], None)
        for n in ("dq", "dk", "dv", "da", "db"):
            np.testing.assert_array_equal(g[n][sl], gs[n])
        np.testing.assert_array_equal(g["dS0"][s], gs["dS0"][0])
    np.testing.assert_array_equal(g["dS0"][1], c["dST"][1])    # an empty sequence passes dS_T through
