"""The C-ABI library builds, loads without a GPU, exports every entry point its
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

import looped_linear_attention_b200 as lla
from looped_linear_attention_b200 import _binding as B
from looped_linear_attention_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.library()


def _declared_functions():
    names = []
    for fname in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not fname.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fname)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s+\**\s*([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                             text, flags=re.M):
            names.append(m.group(1))
    return names


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("gdn_chunk_fwd", "gdn_chunk_fwd_workspace", "gdn_decode_step",
                     "loop_residual", "gdn_status_string", "gdn_get_device_status"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), f"libgdn.so does not export {name}"


def test_version_and_status_strings(lib):
    assert lla.version() >= 100
    assert lla.status_string(B.GDN_OK) == "ok"
    assert "invalid" in lla.status_string(B.GDN_ERR_INVALID)
    assert "timed out" in lla.status_string(B.GDN_ERR_TIMEOUT)
    assert lla.status_string(99) == "unknown status"


def _params(**kw):
    p = B.gdn_fwd_params()
    base = dict(q=16, k=32, v=48, a=64, b=80, o=1 << 28, n_seq=1, seq_len=64, total_tokens=64,
                H=2, dk=128, dv=128, io_dtype=B.GDN_BF16, scale=1.0, flags=0)
    base.update(kw)
    for f, val in base.items():
        setattr(p, f, val)
    return p


@pytest.mark.parametrize("bad,expect", [
    (dict(dk=96), B.GDN_ERR_UNSUPPORTED),
    (dict(dv=100), B.GDN_ERR_UNSUPPORTED),
    (dict(dv=1024), B.GDN_ERR_UNSUPPORTED),
    (dict(H=0), B.GDN_ERR_INVALID),
    (dict(io_dtype=7), B.GDN_ERR_INVALID),
    (dict(flags=0x100), B.GDN_ERR_INVALID),
    (dict(total_tokens=65), B.GDN_ERR_INVALID),          # != n_seq * seq_len
    (dict(q=8), B.GDN_ERR_INVALID),                      # misaligned
    (dict(q=0), B.GDN_ERR_INVALID),                      # null input with tokens
    (dict(S0=1 << 20, S_T=(1 << 20) + 64), B.GDN_ERR_INVALID),   # partial state overlap
    (dict(o=16), B.GDN_ERR_INVALID),                     # output overlaps q
    (dict(S0=(1 << 28) + 4096), B.GDN_ERR_INVALID),      # output overlaps S0
    (dict(S_T=(1 << 28) - 4096), B.GDN_ERR_INVALID),     # output overlaps S_T
])
def test_prefill_rejects_bad_arguments_on_host(lib, bad, expect):
    p = _params(**bad)
    assert lib.gdn_chunk_fwd(ctypes.byref(p), None, 0, None) == expect
    assert lib.gdn_chunk_fwd_workspace(ctypes.byref(p)) == ctypes.c_size_t(-1).value


def test_prefill_null_params(lib):
    assert lib.gdn_chunk_fwd(None, None, 0, None) == B.GDN_ERR_INVALID


def test_workspace_query_is_zero_for_valid_shapes(lib):
    p = _params(S0=1 << 20, S_T=1 << 20)     # exact aliasing is allowed
    assert lib.gdn_chunk_fwd_workspace(ctypes.byref(p)) == 0


def _state_set(H, dk, dv):
    return H * dk * dv * 4


def _schedule(lib, p):
    n, tok0, tok, launches, corr = (ctypes.c_int() for _ in range(5))
    assert lib.gdn_chunk_fwd_schedule(ctypes.byref(p), ctypes.byref(n), ctypes.byref(tok0),
                                      ctypes.byref(tok), ctypes.byref(launches),
                                      ctypes.byref(corr)) == B.GDN_OK
    return n.value, tok0.value, tok.value, launches.value, corr.value


def _segmented_need(n_seq, L, H, dv, P, corrected):
    """Workspace of a segmented schedule: B and M for segments 1 .. P-2 (output
    pass) or 1 .. P-1 (corrected), start states for segments 1 .. P-1, and in
    the corrected schedule qhat [tokens][H][dk] bf16 and the start states in
    bf16; each 256-byte aligned."""
    align = lambda x: (x + 255) // 256 * 256
    sd, md = H * 128 * dv * 4, H * 128 * 128 * 4
    n_part = P - 1 if corrected else P - 2
    return (align(n_seq * n_part * sd) + align(n_seq * n_part * md) + align(n_seq * (P - 1) * sd)
            + (align(n_seq * L * H * 128 * 2) + align(n_seq * (P - 1) * sd // 2) if corrected else 0))


def test_workspace_segmented_schedule_for_few_long_chains(lib):
    """One 4096-token sequence x 16 heads fills 16 of 148 SMs in one pass: the
    query asks for the corrected segmented schedule's buffers, and the schedule
    query reports its segments and launches (state pass, combine, correction).
    With o = h_prev (the loop residual in place) the output-pass schedule is
    taken instead."""
    p = _params(n_seq=1, seq_len=4096, total_tokens=4096, H=16, S_T=1 << 36)
    need = lib.gdn_chunk_fwd_workspace(ctypes.byref(p))
    P, tok0, tok, launches, corr = _schedule(lib, p)
    assert corr == 1 and P >= 2 and launches == 3
    assert need == _segmented_need(1, 4096, 16, 128, P, True)
    assert tok % 64 == 0 and tok0 % 64 == 0 and 0 < tok0 <= tok
    assert tok0 + (P - 2) * tok < 4096 <= tok0 + (P - 1) * tok
    p_in_place = _params(n_seq=1, seq_len=4096, total_tokens=4096, H=16, h_prev=1 << 28, rho=1 << 24)
    P2, _, _, launches2, corr2 = _schedule(lib, p_in_place)
    assert corr2 == 0 and P2 >= 2 and launches2 == (3 if P2 > 2 else 2)
    assert lib.gdn_chunk_fwd_workspace(ctypes.byref(p_in_place)) == _segmented_need(1, 4096, 16, 128, P2, False)


@pytest.mark.parametrize("kw", [
    dict(flags=B.GDN_SINGLE_PASS),                                     # forced one pass
    dict(n_seq=8, seq_len=16384, total_tokens=8 * 16384, H=16, o=1 << 40),   # enough chains
    dict(n_seq=1, seq_len=4096, total_tokens=4096, H=16, io_dtype=B.GDN_F32),   # fp32 kernel
    dict(n_seq=1, seq_len=4096, total_tokens=4096, H=16, flags=B.GDN_PRECISE),
    dict(n_seq=1, seq_len=64, total_tokens=64, H=16),                  # a single chunk
])
def test_workspace_zero_for_one_pass_schedules(lib, kw):
    kw.setdefault("n_seq", 1)
    kw.setdefault("seq_len", 4096)
    kw.setdefault("total_tokens", kw["n_seq"] * kw["seq_len"])
    p = _params(**kw)
    assert lib.gdn_chunk_fwd_workspace(ctypes.byref(p)) == 0
    assert _schedule(lib, p) == (1, 0, 0, 1, 0)


def test_schedule_query_rejects_what_the_call_rejects(lib):
    p = _params(dk=96)                                    # dk outside {64, 128}
    bad = lib.gdn_chunk_fwd_workspace(ctypes.byref(p))
    assert bad == ctypes.c_size_t(-1).value
    assert lib.gdn_chunk_fwd_schedule(ctypes.byref(p), None, None, None, None, None) != B.GDN_OK
    empty = _params(n_seq=0, seq_len=64, total_tokens=0)
    launches = ctypes.c_int(-1)
    assert lib.gdn_chunk_fwd_schedule(ctypes.byref(empty), None, None, None,
                                      ctypes.byref(launches), None) == B.GDN_OK
    assert launches.value == 0


def test_varlen_workspace_holds_the_longest_first_order(lib):
    """Varlen calls run one pass.  With more blocks than one wave they ask for
    one int32 per sequence (the device-sorted longest-first order of the
    sequences) and take two launches; one wave, a single sequence, the precise
    path and more sequences than the sort handles need none."""
    def query(**kw):
        p = _params(seq_len=0, cu_seqlens=1 << 32, o=1 << 40, **kw)
        n, launches = ctypes.c_int(), ctypes.c_int()
        assert lib.gdn_chunk_fwd_schedule(ctypes.byref(p), ctypes.byref(n), None, None,
                                          ctypes.byref(launches), None) == B.GDN_OK
        return lib.gdn_chunk_fwd_workspace(ctypes.byref(p)), n.value, launches.value
    assert query(n_seq=64, total_tokens=64 * 1000, H=16, dv=256) == (256, 1, 2)
    assert query(n_seq=1000, total_tokens=1000 * 100, H=16) == (4096, 1, 2)
    assert query(n_seq=1, total_tokens=4096, H=16) == (0, 1, 1)
    assert query(n_seq=4, total_tokens=4000, H=2) == (0, 1, 1)
    assert query(n_seq=64, total_tokens=64 * 1000, H=16, dv=256, flags=B.GDN_PRECISE) == (0, 1, 1)
    assert query(n_seq=5000, total_tokens=5000 * 10, H=16) == (0, 1, 1)


def test_prefill_rejects_short_or_misaligned_workspace_on_host(lib):
    p = _params(n_seq=1, seq_len=4096, total_tokens=4096, H=16)
    need = lib.gdn_chunk_fwd_workspace(ctypes.byref(p))
    assert need > 0
    assert lib.gdn_chunk_fwd(ctypes.byref(p), ctypes.c_void_p(1 << 34), need - 256,
                             None) == B.GDN_ERR_WORKSPACE
    assert lib.gdn_chunk_fwd(ctypes.byref(p), None, need, None) == B.GDN_ERR_WORKSPACE
    assert lib.gdn_chunk_fwd(ctypes.byref(p), ctypes.c_void_p((1 << 34) + 16), need,
                             None) == B.GDN_ERR_INVALID


def test_python_workspace_query_matches_c(lib):
    import looped_linear_attention_b200 as lla
    p = _params(n_seq=1, seq_len=4096, total_tokens=4096, H=16)
    assert lla.prefill_workspace_bytes(1, 4096, 16, 128, 128) == lib.gdn_chunk_fwd_workspace(
        ctypes.byref(p))
    assert lla.prefill_workspace_bytes(1, 4096, 16, 128, 128, flags=B.GDN_SINGLE_PASS) == 0
    assert lla.prefill_workspace_bytes(64, 1000, 16, 128, 256, varlen=True) == 256   # the order
    assert lla.prefill_workspace_bytes(4, 1000, 2, 128, 128, varlen=True) == 0       # one wave


@pytest.mark.parametrize("args,expect", [
    (dict(dk=96), B.GDN_ERR_UNSUPPORTED),
    (dict(dv=40), B.GDN_ERR_UNSUPPORTED),
    (dict(N=-1), B.GDN_ERR_INVALID),
    (dict(flags=B.GDN_PRECISE), B.GDN_ERR_INVALID),
    (dict(q=8), B.GDN_ERR_INVALID),
    (dict(o=1 << 20), B.GDN_ERR_INVALID),                # output inside the state
    (dict(o=16), B.GDN_ERR_INVALID),                     # output over q
    (dict(o=1 << 24, v=(1 << 24) + 512), B.GDN_ERR_INVALID),   # output over v
    (dict(o=1 << 24, a=(1 << 24) + 16), B.GDN_ERR_INVALID),    # output over a
])
def test_decode_rejects_bad_arguments_on_host(lib, args, expect):
    base = dict(q=16, k=32, v=48, a=64, b=80, S=1 << 20, o=1 << 30, N=4, H=2, dk=128, dv=128,
                dt=B.GDN_BF16, scale=1.0, flags=0)
    base.update(args)
    st = lib.gdn_decode_step(base["q"], base["k"], base["v"], base["a"], base["b"], base["S"],
                             base["o"], base["N"], base["H"], base["dk"], base["dv"], base["dt"],
                             base["scale"], base["flags"], None)
    assert st == expect


@pytest.mark.parametrize("args,expect", [
    (dict(d=7), B.GDN_ERR_INVALID),
    (dict(rows=-1), B.GDN_ERR_INVALID),
    (dict(h_tilde=0), B.GDN_ERR_INVALID),
    (dict(rho=4), B.GDN_ERR_INVALID),
    (dict(dt=5), B.GDN_ERR_INVALID),
])
def test_residual_rejects_bad_arguments_on_host(lib, args, expect):
    base = dict(h_tilde=16, h_prev=32, rho=48, out=64, rows=4, d=16, dt=B.GDN_BF16)
    base.update(args)
    st = lib.loop_residual(base["h_tilde"], base["h_prev"], base["rho"], base["out"],
                           base["rows"], base["d"], base["dt"], None)
    assert st == expect


def test_empty_work_is_a_no_op(lib):
    assert lib.loop_residual(None, None, None, None, 0, 16, B.GDN_BF16, None) == B.GDN_OK
    assert lib.gdn_decode_step(None, None, None, None, None, None, None, 0, 2, 128, 128,
                               B.GDN_BF16, 1.0, 0, None) == B.GDN_OK
    p = _params(n_seq=0, seq_len=0, total_tokens=0)
    assert lib.gdn_chunk_fwd(ctypes.byref(p), None, 0, None) == B.GDN_OK


def test_stacked_projection_weights_are_used_in_place():
    """The looped step runs q, k, v as one batched GEMM over [W_q; W_k; W_v]:
    weights that are consecutive planes of one allocation (as the workload
    generator and stack_weights give them) are viewed, not copied; any other
    arrangement is recognised as such (and stacked by the runner)."""
    import dataclasses
    import torch
    from looped_linear_attention_b200 import workloads as W
    from looped_linear_attention_b200.looped import stack_weights, stacked_view
    inp = W.looped_inputs(dataclasses.replace(W.WORKLOADS["looped_prefill"], seq_len=64), "cpu")
    Wq, Wk, Wv = inp["Wq"], inp["Wk"], inp["Wv"]
    v = stacked_view(Wq, Wk, Wv)
    assert v is not None and v.data_ptr() == Wq.data_ptr()
    assert all(torch.equal(v[i], w) for i, w in enumerate((Wq, Wk, Wv)))
    assert stacked_view(Wq.clone(), Wk.clone(), Wv.clone()) is None
    assert stacked_view(Wk, Wq, Wv) is None
    assert stacked_view(Wq, Wk, Wv[:, :-1]) is None
    W3, q, k, w = stack_weights(Wq.clone(), Wk.clone(), Wv.clone())
    assert stacked_view(q, k, w).data_ptr() == W3.data_ptr()


@pytest.mark.parametrize("n_seq,L,H,dv", [(1, 4096, 16, 128), (1, 8192, 16, 128), (2, 4096, 16, 128),
                                         (1, 16384, 16, 128), (1, 4096, 8, 128), (1, 2048, 16, 128),
                                         (1, 1024, 16, 128), (2, 1000, 2, 128), (1, 777, 2, 256),
                                         (1, 2000, 2, 128), (3, 3000, 4, 256), (1, 130, 1, 128)])
def test_segment_plan_covers_the_sequence(lib, n_seq, L, H, dv):
    """The planner's segments tile each sequence exactly: segment 0 of seg0_tok
    tokens, then segments of seg_tok (whole chunks of 64, segment 0 no longer
    than the others), the last one ragged but not empty; the workspace the
    query asks for is exactly that schedule's buffers; and the launch count
    matches it (with and without a final state)."""
    for st in (None, 1 << 36):
        p = _params(n_seq=n_seq, seq_len=L, total_tokens=n_seq * L, H=H, dv=dv, o=1 << 40, S_T=st)
        P, tok0, tok, launches, corr = _schedule(lib, p)
        need = lib.gdn_chunk_fwd_workspace(ctypes.byref(p))
        if P == 1:
            assert (tok0, tok, launches, need, corr) == (0, 0, 1, 0, 0)
            continue
        assert tok % 64 == 0 and tok0 % 64 == 0 and 0 < tok0 <= tok
        assert tok0 + (P - 2) * tok < L <= tok0 + (P - 1) * tok
        if corr:
            assert tok0 == tok
            assert launches == (3 if (P > 2 or st) else 2)
        else:
            assert launches == (3 if P > 2 else 2)
        assert need == _segmented_need(n_seq, L, H, dv, P, corr)


def _bwd_params(**kw):
    p = B.gdn_bwd_params()
    base = dict(q=1 << 32, k=2 << 32, v=3 << 32, a=4 << 32, b=5 << 32, grad_o=6 << 32,
                grad_q=7 << 32, grad_k=8 << 32, grad_v=9 << 32, grad_a=10 << 32, grad_b=11 << 32,
                n_seq=2, seq_len=100, total_tokens=200, H=2, dk=128, dv=128,
                io_dtype=B.GDN_BF16, scale=1.0, flags=0)
    base.update(kw)
    for name, val in base.items():
        setattr(p, name, val)
    return p


def test_backward_validation_and_workspace(lib):
    """gdn_chunk_bwd: host-side rejections before any launch, and the
    workspaces.  Both paths use one chunk slot per 64 tokens (plus two per
    sequence and one) per head.  Chunkwise (default): W, Qh, W^T, diag(r) K and
    its transpose (C x dk each), U~ [C][dv], g [C], start state and end-state
    gradient [dk][dv] per slot.  Token by
    token (GDN_PRECISE): one checkpoint per slot, one chunk of 65 states and
    the running gradient per chain."""
    p = _bwd_params()
    need = lib.gdn_chunk_bwd_workspace(ctypes.byref(p))
    sd = 128 * 128 * 4
    align = lambda x: (x + 255) // 256 * 256
    slots = 200 // 64 + 2 * 2 + 1
    sh = slots * 2
    assert need == (5 * align(sh * 64 * 128 * 4) + align(sh * 64 * 128 * 4) + align(sh * 64 * 4)
                    + 2 * align(sh * sd))
    tok = _bwd_params(flags=B.GDN_PRECISE)
    assert lib.gdn_chunk_bwd_workspace(ctypes.byref(tok)) == align(2 * slots * sd) + align(4 * 65 * sd) + align(4 * sd)
    bad = ctypes.c_size_t(-1).value
    for kw, status in [(dict(dk=96), B.GDN_ERR_UNSUPPORTED), (dict(dv=300), B.GDN_ERR_UNSUPPORTED),
                       (dict(dv=48), B.GDN_ERR_UNSUPPORTED), (dict(flags=B.GDN_QK_L2NORM), B.GDN_ERR_UNSUPPORTED),
                       (dict(H=0), B.GDN_ERR_INVALID), (dict(total_tokens=199), B.GDN_ERR_INVALID),
                       (dict(grad_o=None), B.GDN_ERR_INVALID), (dict(q=(1 << 32) + 8), B.GDN_ERR_INVALID)]:
        q = _bwd_params(**kw)
        assert lib.gdn_chunk_bwd_workspace(ctypes.byref(q)) == bad, kw
        assert lib.gdn_chunk_bwd(ctypes.byref(q), ctypes.c_void_p(1 << 40), 1 << 40, None) == status, kw
    assert lib.gdn_chunk_bwd(ctypes.byref(p), None, 0, None) == B.GDN_ERR_WORKSPACE
    assert lib.gdn_chunk_bwd(ctypes.byref(p), ctypes.c_void_p(1 << 40), need - 256, None) == B.GDN_ERR_WORKSPACE
    assert lib.gdn_chunk_bwd(ctypes.byref(p), ctypes.c_void_p((1 << 40) + 16), need, None) == B.GDN_ERR_INVALID
    empty = _bwd_params(n_seq=0, seq_len=0, total_tokens=0)
    assert lib.gdn_chunk_bwd_workspace(ctypes.byref(empty)) == 0
    assert lib.gdn_chunk_bwd(ctypes.byref(empty), None, 0, None) == B.GDN_OK


def test_backward_checkpoint_slots_never_overlap():
    """The reverse-mode kernel keeps chain (s, h)'s checkpoints in slots
    t0 / 64 + 2 s .. + ceil(len / 64) - 1 of head h, with total / 64 + 2 n + 1
    slots per head in the workspace: over random length mixes (zeros, single
    tokens, exact multiples of 64) no two sequences share a slot and every slot
    is inside the allocation."""
    import numpy as np
    rng = np.random.default_rng(0)
    for trial in range(300):
        n = int(rng.integers(1, 40))
        lens = rng.choice([0, 1, 63, 64, 65, 128, 129, int(rng.integers(0, 700))], size=n)
        cu = np.concatenate([[0], np.cumsum(lens)])
        total = int(cu[-1])
        slots = total // 64 + 2 * n + 1
        used = set()
        for s in range(n):
            base = int(cu[s]) // 64 + 2 * s
            for c in range((int(lens[s]) + 63) // 64):
                slot = base + c
                assert 0 <= slot < slots and slot not in used, (trial, s, c)
                used.add(slot)


def test_backward_binding_refuses_host_tensors():
    """The Python entry point of the reverse mode takes device tensors only and
    refuses host ones before any library call (no CPU fallback)."""
    import torch
    T, H, dk, dv = 8, 2, 64, 64
    q = torch.zeros(T, H, dk, dtype=torch.bfloat16)
    a = torch.zeros(T, H)
    v = torch.zeros(T, H, dv, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        lla.gdn_chunk_bwd(q, q, v, a, a, v)


def test_prefill_epilogue_validation(lib):
    """The looped-block epilogue: h_prev and rho come together, o may be
    h_prev exactly but overlap it no other way, and may not overlap the gate."""
    ok = _params(h_prev=1 << 28, rho=1 << 24, gate=1 << 26)          # o == h_prev
    assert lib.gdn_chunk_fwd_workspace(ctypes.byref(ok)) != ctypes.c_size_t(-1).value
    for bad in (dict(h_prev=1 << 30),                                # no rho
                dict(rho=1 << 24),                                   # no h_prev
                dict(h_prev=(1 << 28) + 256, rho=1 << 24),           # partial overlap with o
                dict(gate=(1 << 28) + 64),                           # gate inside o
                dict(gate=(1 << 26) + 8)):                           # misaligned
        p = _params(**bad)
        assert lib.gdn_chunk_fwd_workspace(ctypes.byref(p)) == ctypes.c_size_t(-1).value, bad
        assert lib.gdn_chunk_fwd(ctypes.byref(p), None, 0, None) == B.GDN_ERR_INVALID, bad


@pytest.mark.parametrize("args", [
    dict(h_prev=1 << 24),                                            # no rho
    dict(rho=1 << 24),                                               # no h_prev
    dict(gate=(1 << 26) + 4),                                        # misaligned gate
    dict(h_prev=(1 << 30) + 512, rho=1 << 24),                       # partial overlap with o
    dict(gate=1 << 30),                                              # gate inside o
])
def test_decode_looped_rejects_bad_epilogue_on_host(lib, args):
    base = dict(q=16, k=32, v=48, a=64, b=80, S=1 << 20, o=1 << 30, gate=None, h_prev=None,
                rho=None, N=4, H=2, dk=128, dv=128, dt=B.GDN_BF16, scale=1.0, flags=0)
    base.update(args)
    st = lib.gdn_decode_step_looped(base["q"], base["k"], base["v"], base["a"], base["b"], base["S"],
                                    base["o"], base["gate"], base["h_prev"], base["rho"], base["N"],
                                    base["H"], base["dk"], base["dv"], base["dt"], base["scale"],
                                    base["flags"], None)
    assert st == B.GDN_ERR_INVALID


def test_channel_gate_flag_validation(lib):
    """GDN_CHANNEL_GATE (per-channel decay, a [tokens][H][dk]) is accepted by
    prefill and decode; the output may not overlap any of a's dk-wide rows.
    The prefill takes two launches with a workspace (one slot per chunk:
    floor(total / 64) + n_seq + 1 slots per head, each holding three
    64 x dk and two 64 x dv fp32 arrays and dk decays) and one without."""
    p = _params(n_seq=1, seq_len=4096, total_tokens=4096, H=16, flags=B.GDN_CHANNEL_GATE)

    def al(x):
        return (x + 255) // 256 * 256

    for dk, dv in ((128, 128), (64, 256)):
        p.dk, p.dv = dk, dv
        sh = (4096 // 64 + 1 + 1) * 16
        need = 3 * al(sh * 64 * dk * 4) + 2 * al(sh * 64 * dv * 4) + al(sh * dk * 4)
        assert lib.gdn_chunk_fwd_workspace(ctypes.byref(p)) == need
    assert _schedule(lib, p) == (1, 0, 0, 2, 0)
    # a workspace smaller than the need, or a size without one, is refused on the host
    assert lib.gdn_chunk_fwd(ctypes.byref(p), ctypes.c_void_p(1 << 30), 256, None) == B.GDN_ERR_WORKSPACE
    assert lib.gdn_chunk_fwd(ctypes.byref(p), None, 256, None) == B.GDN_ERR_WORKSPACE
    # a of 64 tokens x 2 heads x 128 channels x 4 B = 64 KiB: an output 32 KiB past it overlaps
    bad = _params(a=1 << 20, o=(1 << 20) + (32 << 10), flags=B.GDN_CHANNEL_GATE)
    assert lib.gdn_chunk_fwd(ctypes.byref(bad), None, 0, None) == B.GDN_ERR_INVALID
    ok = _params(a=1 << 20, o=(1 << 20) + (32 << 10))               # scalar a: 512 B, no overlap
    assert lib.gdn_chunk_fwd_workspace(ctypes.byref(ok)) != ctypes.c_size_t(-1).value
    st = lib.gdn_decode_step(16, 32, 48, 1 << 20, 80, 1 << 24, (1 << 20) + 2048, 4, 2, 128, 128,
                             B.GDN_BF16, 1.0, B.GDN_CHANNEL_GATE, None)
    assert st == B.GDN_ERR_INVALID                                 # o inside a's 4 KiB
