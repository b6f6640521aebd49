"""Pins of the oracle's per-channel (diagonal) gate variant, KDA.

The reading (the pages name KDA among the LT2 mixers, "LT2: Linear-Time Looped
Transformers", Appendix C, and treat the DPLR block in its general diagonal
form in §2 and Appendix B.1, but print no update rule):
    Sigma_t = (I - b_t k_t k_t^T) Diag(a_t) Sigma_{t-1} + b_t k_t v_t^T,
    o_t = scale Sigma_t^T q_t,  a_t in (0, 1]^{dk}.
Each pin compares the oracle with a different construction: explicit products
of the dk x dk factors, the scalar gate as a special case (the gated delta
rule), the no-write closed form per channel, and the invariances the kernels
rely on (split and resume, packed sequences, decode after prefill).  A decay
applied after the delta step, on the value side, or per token instead of per
channel fails at least one of them.
"""
import numpy as np
import pytest

import oracle


def _case(rng, L, H, dk, dv, b_hi=2.0):
    q = rng.standard_normal((L, H, dk))
    k = rng.standard_normal((L, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((L, H, dv))
    a = rng.uniform(0.2, 1.0, (L, H, dk))
    b = rng.uniform(0.0, b_hi, (L, H))
    return q, k, v, a, b


def _brute(q, k, v, a, b, S0, scale):
    """S_t = F_t ... F_1 S0 + sum_s F_t ... F_{s+1} b_s k_s v_s^T with
    F_t = (I - b_t k_t k_t^T) Diag(a_t), each S_t from scratch."""
    L, dk = k.shape
    I = np.eye(dk)
    F = [(I - b[t] * np.outer(k[t], k[t])) @ np.diag(a[t]) for t in range(L)]
    o = np.zeros((L, v.shape[1]))
    S = S0
    for t in range(L):
        P = I.copy()
        for s in range(t, -1, -1):
            P = P @ F[s]
        S = P @ S0
        for s in range(t + 1):
            Pr = I.copy()
            for r in range(t, s, -1):
                Pr = Pr @ F[r]
            S = S + Pr @ (b[s] * np.outer(k[s], v[s]))
        o[t] = scale * S.T @ q[t]
    return o, S


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_kda_brute_force_products(seed):
    rng = np.random.default_rng(400 + seed)
    L, H, dk, dv = 11, 2, 5, 3
    q, k, v, a, b = _case(rng, L, H, dk, dv)
    S0 = rng.standard_normal((1, H, dk, dv))
    o, ST = oracle.kda_fwd(q, k, v, a, b, S0, None, 0.7)
    for h in range(H):
        ob, Sb = _brute(q[:, h], k[:, h], v[:, h], a[:, h], b[:, h], S0[0, h], 0.7)
        np.testing.assert_allclose(o[:, h], ob, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(ST[0, h], Sb, rtol=1e-12, atol=1e-12)


def test_kda_scalar_gate_is_the_gated_delta_rule():
    """Equal entries a_t = alpha_t 1 give the gated delta rule (to rounding)."""
    rng = np.random.default_rng(410)
    L, H, dk, dv = 40, 3, 6, 4
    q, k, v, a, b = _case(rng, L, H, dk, dv)
    alpha = a[:, :, 0]
    S0 = rng.standard_normal((1, H, dk, dv))
    o1, S1 = oracle.kda_fwd(q, k, v, np.repeat(alpha[:, :, None], dk, axis=2), b, S0)
    o2, S2 = oracle.gdn_fwd(q, k, v, alpha, b, S0)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S1, S2, rtol=1e-12, atol=1e-12)


def test_kda_no_write_decays_each_channel():
    """b = 0: row i of the state decays by the product of a_{t,i} alone, and
    o_t reads the decayed state."""
    rng = np.random.default_rng(420)
    L, H, dk, dv = 9, 2, 5, 3
    q, k, v, a, _ = _case(rng, L, H, dk, dv)
    S0 = rng.standard_normal((1, H, dk, dv))
    o, ST = oracle.kda_fwd(q, k, v, a, np.zeros((L, H)), S0)
    cum = np.cumprod(a, axis=0)                               # [L, H, dk]
    np.testing.assert_allclose(ST[0], cum[-1][:, :, None] * S0[0], rtol=1e-13)
    for t in range(L):
        St = cum[t][:, :, None] * S0[0]
        np.testing.assert_allclose(o[t], np.einsum("hkv,hk->hv", St, q[t]), rtol=1e-12, atol=1e-13)


def test_kda_first_token_reads_its_own_write():
    """From a zero state, o_1 = scale b_1 (k_1 . q_1) v_1 whatever a_1 is."""
    rng = np.random.default_rng(430)
    q, k, v, a, b = _case(rng, 1, 2, 4, 3)
    o, _ = oracle.kda_fwd(q, k, v, a, b, None, None, 0.5)
    for h in range(2):
        np.testing.assert_allclose(o[0, h], 0.5 * b[0, h] * (k[0, h] @ q[0, h]) * v[0, h], rtol=1e-13)


def test_kda_split_resume_varlen_and_decode():
    rng = np.random.default_rng(440)
    L, H, dk, dv = 30, 2, 4, 5
    q, k, v, a, b = _case(rng, L, H, dk, dv)
    S0 = rng.standard_normal((1, H, dk, dv))
    o, ST = oracle.kda_fwd(q, k, v, a, b, S0)
    m = 13
    o1, S1 = oracle.kda_fwd(q[:m], k[:m], v[:m], a[:m], b[:m], S0)
    o2, S2 = oracle.kda_fwd(q[m:], k[m:], v[m:], a[m:], b[m:], S1)
    np.testing.assert_array_equal(np.concatenate([o1, o2]), o)
    np.testing.assert_array_equal(S2, ST)
    # the same tokens as two packed sequences equal the two runs
    S0b = np.concatenate([S0, S1])
    ov, Sv = oracle.kda_fwd(q, k, v, a, b, S0b, np.array([0, m, L], dtype=np.int32))
    np.testing.assert_array_equal(ov, o)
    np.testing.assert_array_equal(Sv[1], ST[0])
    # decode of token L-1 after prefill of L-1 tokens
    _, SL = oracle.kda_fwd(q[:-1], k[:-1], v[:-1], a[:-1], b[:-1], S0)
    od, Sd = oracle.kda_decode(q[-1:], k[-1:], v[-1:], a[-1:], b[-1:], SL)
    np.testing.assert_array_equal(od[0], o[-1])
    np.testing.assert_array_equal(Sd, ST)
