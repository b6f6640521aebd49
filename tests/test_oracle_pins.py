"""Pins of the CPU oracle against facts fixed by the mathematics and the pages.

None of these re-types the oracle's own loop: each compares it with a different
construction (explicit products of the dk x dk factors, closed forms, exact
reflections and permutations, a hand-worked example) chosen so that a dropped
term, a wrong sign or index, or a transposed operand fails at least one.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_case(rng, L, H, dk, dv, unit_keys=False, b_range=(0.0, 1.0)):
    q = rng.standard_normal((L, H, dk))
    k = rng.standard_normal((L, H, dk))
    if unit_keys:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((L, H, dv))
    a = rng.uniform(0.3, 1.0, (L, H))
    b = rng.uniform(*b_range, (L, H))
    return q, k, v, a, b


# ---------------------------------------------------------------- brute force
def _brute_force(q, k, v, a, b, S0, scale):
    """Unrolled closed form with explicit dk x dk transition matrices
    A_t = a_t (I - b_t k_t k_t^T):
        S_t = A_t ... A_1 S_0 + sum_{s<=t} A_t ... A_{s+1} b_s k_s v_s^T,
    evaluated independently for every t (O(L^2) matrix products)."""
    L, dk = k.shape
    I = np.eye(dk)
    A = [a[t] * (I - b[t] * np.outer(k[t], k[t])) for t in range(L)]
    o = np.zeros((L, v.shape[1]))
    S = None
    for t in range(L):
        P = I.copy()
        for s in range(t, -1, -1):
            P = P @ A[s]            # P = A_t ... A_s
        S = P @ S0
        for s in range(t + 1):
            Pr = I.copy()
            for r in range(t, s, -1):
                Pr = Pr @ A[r]      # A_t ... A_{s+1}
            S = S + Pr @ (b[s] * np.outer(k[s], v[s]))
        o[t] = scale * S.T @ q[t]
    return o, S


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_products(seed):
    rng = np.random.default_rng(seed)
    L, H, dk, dv = 11, 2, 5, 3
    q, k, v, a, b = _rand_case(rng, L, H, dk, dv, b_range=(0.0, 2.0))
    S0 = rng.standard_normal((1, H, dk, dv))
    scale = 0.7
    o, ST = oracle.gdn_fwd(q, k, v, a, b, S0, None, scale)
    for h in range(H):
        o_ref, S_ref = _brute_force(q[:, h], k[:, h], v[:, h], a[:, h], b[:, h], S0[0, h], scale)
        np.testing.assert_allclose(o[:, h], o_ref, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(ST[0, h], S_ref, rtol=1e-11, atol=1e-12)


def test_hand_worked_example():
    with open(os.path.join(GOLDEN, "hand_worked_2x2.json")) as f:
        g = json.load(f)
    inp = {n: np.array(x, dtype=np.float64) for n, x in g["inputs"].items()}
    o, ST = oracle.gdn_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"])
    np.testing.assert_allclose(o, np.array(g["expected"]["o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(ST, np.array(g["expected"]["S_T"]), rtol=0, atol=1e-14)


# ---------------------------------------------------------------- closed forms
def test_identity_when_no_write_and_no_decay():
    rng = np.random.default_rng(3)
    q, k, v, a, b = _rand_case(rng, 9, 3, 6, 4)
    a[:] = 1.0
    b[:] = 0.0
    S0 = rng.standard_normal((1, 3, 6, 4))
    o, ST = oracle.gdn_fwd(q, k, v, a, b, S0, None, 1.5)
    np.testing.assert_array_equal(ST, S0)
    np.testing.assert_allclose(o, 1.5 * np.einsum("thi,hij->thj", q, S0[0]), rtol=1e-14)


def test_pure_decay_closed_form():
    rng = np.random.default_rng(4)
    q, k, v, a, b = _rand_case(rng, 13, 2, 4, 5)
    b[:] = 0.0
    S0 = rng.standard_normal((1, 2, 4, 5))
    o, ST = oracle.gdn_fwd(q, k, v, a, b, S0)
    decay = np.cumprod(a, axis=0)                        # prod_{s<=t} a_s
    np.testing.assert_allclose(ST[0], decay[-1][:, None, None] * S0[0], rtol=1e-13)
    expect_o = decay[:, :, None] * np.einsum("thi,hij->thj", q, S0[0])
    np.testing.assert_allclose(o, expect_o, rtol=1e-12)


def test_retrieval_with_orthonormal_keys():
    """a = b = 1, S0 = 0, orthonormal keys: reading key j returns value j."""
    rng = np.random.default_rng(5)
    dk, dv, n = 8, 3, 6
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm[:, :n].T                                   # n orthonormal rows
    vals = rng.standard_normal((n, dv))
    k = keys[:, None, :]
    v = vals[:, None, :]
    q = keys[:, None, :]
    a = np.ones((n, 1))
    b = np.ones((n, 1))
    _, ST = oracle.gdn_fwd(q, k, v, a, b)
    np.testing.assert_allclose(ST[0, 0].T @ keys.T, vals.T, atol=1e-13)


def test_overwrite_same_key():
    """Writing (k, v1) then (k, v2) with a = b = 1 and a unit key leaves S^T k = v2."""
    rng = np.random.default_rng(6)
    dk, dv = 5, 4
    kk = rng.standard_normal(dk)
    kk /= np.linalg.norm(kk)
    v1, v2 = rng.standard_normal(dv), rng.standard_normal(dv)
    S0 = rng.standard_normal((1, 1, dk, dv))
    k = np.stack([kk, kk])[:, None, :]
    v = np.stack([v1, v2])[:, None, :]
    o, ST = oracle.gdn_fwd(k, k, v, np.ones((2, 1)), np.ones((2, 1)), S0)
    np.testing.assert_allclose(ST[0, 0].T @ kk, v2, atol=1e-13)
    np.testing.assert_allclose(o[1, 0], v2, atol=1e-13)     # q = k reads the value back


def test_first_token_from_zero_state():
    """S_1 = b k v^T from S_0 = 0, so o_1 = b (k . q) v."""
    rng = np.random.default_rng(7)
    q, k, v, a, b = _rand_case(rng, 1, 4, 6, 7)
    o, ST = oracle.gdn_fwd(q, k, v, a, b)
    for h in range(4):
        np.testing.assert_allclose(ST[0, h], b[0, h] * np.outer(k[0, h], v[0, h]), rtol=1e-14)
        np.testing.assert_allclose(o[0, h], b[0, h] * (k[0, h] @ q[0, h]) * v[0, h], rtol=1e-13)


# ------------------------------------------------- the pages' structural claims
def test_transpositions_permute_state_rows():
    """A swap (i j) is I - k k^T with k = e_i - e_j (b = 1), i.e. the reflection
    with the unit key (e_i - e_j)/sqrt(2) and b = 2; n-1 of them realise any
    permutation of n coordinates (S_n prefix products, Appendix B.1).  Equal up
    to the rounding of x - (x - y) = y."""
    rng = np.random.default_rng(8)
    n, dv = 6, 3
    perm = rng.permutation(n)
    # decompose perm into transpositions (selection sort on the target order)
    cur = list(range(n))
    swaps = []
    for i in range(n):
        j = cur.index(perm[i])
        if j != i:
            swaps.append((i, j))
            cur[i], cur[j] = cur[j], cur[i]
    assert len(swaps) <= n - 1
    keys = []
    for i, j in swaps:
        e = np.zeros(n)
        e[i], e[j] = 1.0, -1.0
        keys.append(e)
    T = len(keys)
    k = np.array(keys)[:, None, :]
    S0 = rng.standard_normal((1, 1, n, dv))
    _, ST = oracle.gdn_fwd(np.zeros((T, 1, n)), k, np.zeros((T, 1, dv)),
                           np.ones((T, 1)), np.ones((T, 1)), S0)
    np.testing.assert_allclose(ST[0, 0], S0[0, 0][perm], rtol=0, atol=1e-14)
    # same swaps as unit keys with b = 2
    ku = k / np.sqrt(2.0)
    _, ST2 = oracle.gdn_fwd(np.zeros((T, 1, n)), ku, np.zeros((T, 1, dv)),
                            np.ones((T, 1)), 2.0 * np.ones((T, 1)), S0)
    np.testing.assert_allclose(ST2[0, 0], S0[0, 0][perm], atol=1e-14)


def _householder_factors(Q):
    """Unit vectors u_1..u_m (m <= n) with H(u_m)...H(u_1) Q = I, H(u) = I - 2uu^T."""
    n = Q.shape[0]
    M = Q.copy()
    us = []
    for i in range(n):
        x = M[:, i]
        e = np.zeros(n)
        e[i] = 1.0
        d = x - e
        nd = np.linalg.norm(d)
        if nd > 1e-12:
            u = d / nd
            M = M - 2.0 * np.outer(u, u @ M)
            us.append(u)
    np.testing.assert_allclose(M, np.eye(n), atol=1e-12)
    return us


@pytest.mark.parametrize("seed", [0, 1])
def test_cartan_dieudonne_orthogonal_map(seed):
    """At most dk reflections (a = 1, b = 2, v = 0, unit keys) realise any
    orthogonal map of the state (Appendix B.1)."""
    rng = np.random.default_rng(100 + seed)
    n, dv = 4, 3
    Q, _ = np.linalg.qr(rng.standard_normal((n, n)))
    us = _householder_factors(Q)
    assert len(us) <= n
    k = np.array(us[::-1])[:, None, :]       # feed u_m first: S_T = H(u_1)...H(u_m) S_0 = Q S_0
    T = k.shape[0]
    S0 = rng.standard_normal((1, 1, n, dv))
    _, ST = oracle.gdn_fwd(np.zeros((T, 1, n)), k, np.zeros((T, 1, dv)),
                           np.ones((T, 1)), 2.0 * np.ones((T, 1)), S0)
    np.testing.assert_allclose(ST[0, 0], Q @ S0[0, 0], atol=1e-13)


@pytest.mark.parametrize("T", [1, 2, 4, 6])
def test_rank_T_update_and_spectral_bound(T):
    """T rank-1 DPLR steps compose into I - prod(I - b k k^T) of rank exactly T
    (generic keys), and the product has spectral norm <= 1 for unit keys and
    b in [0, 2] (§2 and Appendix B.1)."""
    rng = np.random.default_rng(200 + T)
    dk = 8
    k = rng.standard_normal((T, 1, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    b = rng.uniform(0.05, 1.95, (T, 1))
    S0 = np.eye(dk)[None, None]              # dv = dk: the state becomes the product itself
    _, ST = oracle.gdn_fwd(np.zeros((T, 1, dk)), k, np.zeros((T, 1, dk)),
                           np.ones((T, 1)), b, S0)
    P = ST[0, 0]
    sv = np.linalg.svd(np.eye(dk) - P, compute_uv=False)
    assert sv[T - 1] > 1e-6                  # rank at least T
    if T < dk:
        assert sv[T] < 1e-12 * sv[0]         # rank at most T
    assert np.linalg.norm(P, 2) <= 1.0 + 1e-12


# ------------------------------------------------------------- invariances
def test_split_and_resume_is_bitwise_identical():
    rng = np.random.default_rng(9)
    L, H, dk, dv = 40, 2, 4, 6
    q, k, v, a, b = _rand_case(rng, L, H, dk, dv)
    S0 = rng.standard_normal((1, H, dk, dv))
    o, ST = oracle.gdn_fwd(q, k, v, a, b, S0)
    for m in (1, 17, 39):
        o1, S1 = oracle.gdn_fwd(q[:m], k[:m], v[:m], a[:m], b[:m], S0)
        o2, S2 = oracle.gdn_fwd(q[m:], k[m:], v[m:], a[m:], b[m:], S1)
        np.testing.assert_array_equal(np.concatenate([o1, o2]), o)
        np.testing.assert_array_equal(S2, ST)


def test_varlen_equals_separate_sequences():
    rng = np.random.default_rng(10)
    lens = [5, 0, 12, 1, 7]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    H, dk, dv = 2, 4, 3
    q, k, v, a, b = _rand_case(rng, int(cu[-1]), H, dk, dv)
    S0 = rng.standard_normal((len(lens), H, dk, dv))
    o, ST = oracle.gdn_fwd(q, k, v, a, b, S0, cu)
    for s, (t0, t1) in enumerate(zip(cu[:-1], cu[1:])):
        os_, Ss = oracle.gdn_fwd(q[t0:t1], k[t0:t1], v[t0:t1], a[t0:t1], b[t0:t1], S0[s:s + 1])
        np.testing.assert_array_equal(o[t0:t1], os_)
        np.testing.assert_array_equal(ST[s], Ss[0])
    np.testing.assert_array_equal(ST[1], S0[1])   # empty sequence keeps its state


def test_decode_continues_prefill():
    rng = np.random.default_rng(11)
    L, H, dk, dv = 10, 3, 4, 5
    q, k, v, a, b = _rand_case(rng, L + 1, H, dk, dv)
    o_full, S_full = oracle.gdn_fwd(q, k, v, a, b, None, None, 0.5)
    _, S_L = oracle.gdn_fwd(q[:L], k[:L], v[:L], a[:L], b[:L], None, None, 0.5)
    o_d, S_d = oracle.gdn_decode(q[L:], k[L:], v[L:], a[L:], b[L:], S_L, 0.5)
    np.testing.assert_array_equal(o_d[0], o_full[L])
    np.testing.assert_array_equal(S_d, S_full)


def test_oracle_rejects_bad_offsets():
    q = np.zeros((4, 1, 2))
    with pytest.raises(ValueError):
        oracle.gdn_fwd(q, q, q, np.ones((4, 1)), np.ones((4, 1)), None,
                       np.array([0, 3, 2, 4], dtype=np.int32))


# --------------------------------------------------------------- residual etc.
def test_loop_residual_closed_forms():
    rng = np.random.default_rng(12)
    ht = rng.standard_normal((5, 8))
    hp = rng.standard_normal((5, 8))
    np.testing.assert_array_equal(oracle.loop_residual(ht, hp, np.zeros(8)), ht)
    np.testing.assert_array_equal(oracle.loop_residual(np.zeros((5, 8)), hp, np.ones(8)), hp)
    rho = np.arange(8) / 8.0                  # per-channel: column c scales by c/8
    out = oracle.loop_residual(np.zeros((5, 8)), np.ones((5, 8)), rho)
    np.testing.assert_array_equal(out, np.tile(rho, (5, 1)))


def test_qk_l2norm_and_bf16_rounding():
    x = np.array([[3.0, 4.0]])
    np.testing.assert_allclose(oracle.qk_l2norm(x), x / np.sqrt(25.0 + 1e-6), rtol=1e-15)
    # bf16 has 8 significant bits: 1 + 2^-8 is a tie and rounds to even (1.0);
    # 1 + 3*2^-8 rounds up to 1 + 2^-6; 257 rounds to 256.
    r = oracle.round_bf16(np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 257.0, -1.5]))
    np.testing.assert_array_equal(r, [1.0, 1 + 2.0 ** -6, 256.0, -1.5])


def test_looped_forward_reduces_to_gate_products():
    """With W = I, a = 1, b = 0 the mixer writes nothing (o = 0), so each loop is
    h^(tau) = rho_tau (.) h^(tau-1); after T loops h^(T) = (prod rho) (.) h^(0)
    up to the bf16 rounding of every loop state."""
    rng = np.random.default_rng(13)
    L, H, dk = 6, 2, 4
    d = H * dk
    h0 = oracle.round_bf16(rng.standard_normal((L, d)))
    T = 3
    rho = np.array([[0.5] * d, [0.25] * d, [2.0] * d])
    a = np.ones((T, L, H))
    b = np.zeros((T, L, H))
    hT = oracle.looped_forward(h0, np.eye(d), np.eye(d), np.eye(d), a, b, rho, H, dk, dk)
    np.testing.assert_array_equal(hT, 0.25 * h0)   # powers of two: exact in bf16


def test_looped_forward_single_token_reads_back_value():
    """W = I, L = 1, a = b = 1, rho = 0: q = k = h/||h|| per head and v = h, so
    S_1 = k v^T and o = (k . q) v = (||h||^2 / (||h||^2 + eps)) h per head."""
    rng = np.random.default_rng(14)
    H, dk = 2, 4
    d = H * dk
    h0 = oracle.round_bf16(rng.standard_normal((1, d)))
    a = np.ones((1, 1, H))
    b = np.ones((1, 1, H))
    out = oracle.looped_forward(h0, np.eye(d), np.eye(d), np.eye(d), a, b,
                                np.zeros((1, d)), H, dk, dk)
    hh = h0.reshape(H, dk)
    n2 = (hh * hh).sum(-1, keepdims=True)
    expect = oracle.round_bf16((n2 / (n2 + 1e-6) * hh).reshape(1, d))
    np.testing.assert_array_equal(out, expect)


@pytest.mark.parametrize("seed", [0, 1])
def test_segment_state_update_is_affine_in_its_start_state(seed):
    """The state a segment ends in is M S_start + B: B is the end state from a
    zero start, and M (dk x dk) is the end state of a run with v = 0 from the
    identity (columns of the identity as dv = dk values).  The segmented
    schedule relies on exactly this; the oracle must satisfy it for any start
    state, and chaining the segments' (M, B) must give the one-pass end state."""
    rng = np.random.default_rng(300 + seed)
    L, H, dk, dv = 37, 2, 5, 3
    q, k, v, a, b = _rand_case(rng, L, H, dk, dv, b_range=(0.0, 2.0))
    S_start = rng.standard_normal((1, H, dk, dv))
    _, S_direct = oracle.gdn_fwd(q, k, v, a, b, S_start)
    _, B = oracle.gdn_fwd(q, k, v, a, b, None)
    eye = np.broadcast_to(np.eye(dk), (1, H, dk, dk)).copy()
    _, M = oracle.gdn_fwd(q[:, :, :], k, np.zeros((L, H, dk)), a, b, eye)
    np.testing.assert_allclose(S_direct[0], np.einsum("hij,hjk->hik", M[0], S_start[0]) + B[0],
                               rtol=1e-12, atol=1e-12)
    # three segments chained through their (M, B) pairs equal one pass
    cuts = [0, 11, 24, L]
    S = S_start[0]
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        sl = slice(lo, hi)
        _, Bp = oracle.gdn_fwd(q[sl], k[sl], v[sl], a[sl], b[sl], None)
        _, Mp = oracle.gdn_fwd(q[sl], k[sl], np.zeros((hi - lo, H, dk)), a[sl], b[sl], eye)
        S = np.einsum("hij,hjk->hik", Mp[0], S) + Bp[0]
    np.testing.assert_allclose(S, S_direct[0], rtol=1e-11, atol=1e-11)


# ------------------------------------------------------------ output gate
def test_output_gate_closed_forms():
    """Head-wise sigmoid output gate (§3, gated-attention paragraph): sigmoid of
    ln 3 is exactly 3/4 and of -ln 3 exactly 1/4 (a sign slip swaps them), a
    logit of 0 halves the output, a large logit leaves it as it is, and the
    factor belongs to its own (token, head) (a transposed index moves the
    3/4 to another head).  The state is never gated."""
    rng = np.random.default_rng(15)
    L, H, dk, dv = 9, 3, 4, 5
    q, k, v, a, b = _rand_case(rng, L, H, dk, dv)
    S0 = rng.standard_normal((1, H, dk, dv))
    o, S = oracle.gdn_fwd(q, k, v, a, b, S0)
    z = np.zeros((L, H))
    z[:, 0] = np.log(3.0)
    z[:, 1] = -np.log(3.0)
    z[::2, 2] = 60.0
    og, Sg = oracle.gdn_fwd(q, k, v, a, b, S0, gate=z)
    np.testing.assert_array_equal(Sg, S)
    np.testing.assert_allclose(og[:, 0], 0.75 * o[:, 0], rtol=1e-15)
    np.testing.assert_allclose(og[:, 1], 0.25 * o[:, 1], rtol=1e-15)
    np.testing.assert_allclose(og[::2, 2], o[::2, 2], rtol=1e-15)
    np.testing.assert_array_equal(og[1::2, 2], 0.5 * o[1::2, 2])
    np.testing.assert_allclose(oracle.sigmoid(np.array([-800.0, 800.0])), [0.0, 1.0], atol=0)
    # the same factor in decode
    od, _ = oracle.gdn_decode(q[:1], k[:1], v[:1], a[:1], b[:1], S0, gate=z[:1])
    o1, _ = oracle.gdn_decode(q[:1], k[:1], v[:1], a[:1], b[:1], S0)
    np.testing.assert_allclose(od[0, 0], 0.75 * o1[0, 0], rtol=1e-15)


def test_looped_forward_gate_single_token():
    """One token, W = I, a = b = 1, rho = 0 and the gate weights W_g chosen so
    that head h's logit is ln 3 (head 0) or 0 (head 1): the read-back value
    (||h||^2 / (||h||^2 + eps)) h of each head is scaled by 3/4 and by 1/2."""
    H, dk = 2, 4
    d = H * dk
    h0 = oracle.round_bf16(np.array([[1.0, -2.0, 0.5, 3.0, 0.25, 1.5, -1.0, 2.0]]))
    Wg = np.zeros((d, H))
    Wg[0, 0] = np.log(3.0) / h0[0, 0]        # logit of head 0: h0[0] * Wg[0, 0]
    a = np.ones((1, 1, H))
    b = np.ones((1, 1, H))
    out = oracle.looped_forward(h0, np.eye(d), np.eye(d), np.eye(d), a, b, np.zeros((1, d)),
                                H, dk, dk, Wg=Wg)
    hh = h0.reshape(H, dk)
    n2 = (hh * hh).sum(-1, keepdims=True)
    z = np.array([[float(np.float32(np.log(3.0)))], [0.0]])
    expect = oracle.round_bf16((oracle.sigmoid(z) * n2 / (n2 + 1e-6) * hh).reshape(1, d))
    np.testing.assert_array_equal(out, expect)
