"""gdn_chunk_fwd_noalloc: prefill for callers that cannot allocate device memory
(a plugin whose host engine owns every device allocation through its own pool,
or a path that must not call cudaMalloc because it can synchronise the device).
Its segmented schedule runs out of a 32 MiB scratch array compiled into the
library instead of a caller-provided workspace.

Called through the C ABI twice in a row, on different inputs (stale scratch
contents from the first call would show in the second), and compared with
gdn_chunk_fwd, the allocating entry point, on the same inputs (bit for bit:
both run the same deterministic schedule).  This file is
collected last so that a failure here does not hide the other tests.
"""
import ctypes
import dataclasses

import pytest
import torch

import looped_linear_attention_b200 as lla
from looped_linear_attention_b200 import _binding as B
from looped_linear_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20        # the compiled-in scratch, as stated in include/gdn.h


@pytest.fixture(scope="module")
def lib():
    from looped_linear_attention_b200 import build
    build.build()
    handle = lla.library()
    handle.gdn_chunk_fwd_noalloc.argtypes = [ctypes.POINTER(B.gdn_fwd_params), ctypes.c_void_p]
    handle.gdn_chunk_fwd_noalloc.restype = ctypes.c_int
    torch.cuda.init()
    yield handle
    assert lla.gdn_get_device_status() == lla.GDN_OK


def _inputs(label, n_seq, H, L):
    wl = dataclasses.replace(W.WORKLOADS["long_prefill"], name=label, n_seq=n_seq, H=H,
                             seq_len=L, random_s0=True)
    return W.prefill_inputs(wl, "cuda")


def _params(inp, o, S_T):
    T, H, dk = inp["q"].shape
    return B.gdn_fwd_params(inp["q"].data_ptr(), inp["k"].data_ptr(), inp["v"].data_ptr(),
                            inp["a"].data_ptr(), inp["b"].data_ptr(), inp["S0"].data_ptr(),
                            o.data_ptr(), S_T.data_ptr(), None, inp["n_seq"], inp["seq_len"], T,
                            H, dk, inp["v"].shape[2], B.GDN_BF16, 1.0, 0)


def test_noalloc_matches_gdn_chunk_fwd_on_two_calls(lib):
    """One 4096-token sequence x 16 heads: the segmented schedule, whose
    scratch fits the 32 MiB array."""
    n_seq, H, L = 1, 16, 4096
    need = lla.prefill_workspace_bytes(n_seq, L, H, 128, 128)
    assert 0 < need <= SCRATCH_BYTES
    # three launches: the combine kernel runs, so every region of the scratch is used
    assert lla.prefill_schedule(n_seq, L, H, 128, 128)["launches"] == 3
    cases = []
    for call in range(2):
        inp = _inputs(f"noalloc-{call}", n_seq, H, L)
        o_ref, S_ref = lla.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"],
                                         inp["S0"], n_seq=n_seq)
        o = torch.full_like(o_ref, float("nan"))
        S_T = torch.full_like(S_ref, float("nan"))
        cases.append((inp, o_ref, S_ref, o, S_T))
    torch.cuda.synchronize()
    for inp, _, _, o, S_T in cases:            # the two calls, back to back
        p = _params(inp, o, S_T)
        assert lib.gdn_chunk_fwd_noalloc(ctypes.byref(p), None) == B.GDN_OK
    torch.cuda.synchronize()
    assert lla.gdn_get_device_status() == lla.GDN_OK
    # the same deterministic schedule on the same shape: equal bit for bit
    for _, o_ref, S_ref, o, S_T in cases:
        assert torch.equal(o, o_ref) and torch.equal(S_T, S_ref)


def test_noalloc_varlen_longest_first(lib):
    """A multi-wave varlen call keeps its length-sorted order in the scratch
    array; outputs equal those of gdn_chunk_fwd."""
    lengths = [640, 3, 64, 300, 0, 129] * 8                  # 48 sequences x 4 heads
    wl = dataclasses.replace(W.WORKLOADS["varlen"], name="noalloc-varlen", H=4, dv=128,
                             random_s0=True)
    inp = W.prefill_inputs(wl, "cuda", lengths=lengths)
    cu = torch.from_numpy(inp["cu_seqlens"]).cuda()
    assert lla.prefill_workspace_bytes(len(lengths), 200, 4, 128, 128, varlen=True) > 0
    o_ref, S_ref = lla.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["S0"], cu)
    o = torch.full_like(o_ref, float("nan"))
    S_T = torch.full_like(S_ref, float("nan"))
    p = B.gdn_fwd_params(inp["q"].data_ptr(), inp["k"].data_ptr(), inp["v"].data_ptr(),
                         inp["a"].data_ptr(), inp["b"].data_ptr(), inp["S0"].data_ptr(),
                         o.data_ptr(), S_T.data_ptr(), cu.data_ptr(), len(lengths), 0,
                         inp["total_tokens"], 4, 128, 128, B.GDN_BF16, 1.0, 0)
    assert lib.gdn_chunk_fwd_noalloc(ctypes.byref(p), None) == B.GDN_OK
    torch.cuda.synchronize()
    assert lla.gdn_get_device_status() == lla.GDN_OK
    assert torch.equal(o, o_ref) and torch.equal(S_T, S_ref)


def test_noalloc_rejects_shapes_beyond_the_scratch(lib):
    """A call whose segmented schedule would need more than the 32 MiB array
    (here 3 heads of one 131072-token sequence with dv = 256) returns
    GDN_ERR_WORKSPACE before it launches anything, so placeholder pointers
    suffice."""
    n_seq, H, L, dv = 1, 3, 131072, 256
    need = lla.prefill_workspace_bytes(n_seq, L, H, 128, dv)
    assert need > SCRATCH_BYTES
    base = 1 << 40
    p = B.gdn_fwd_params(base, base + (1 << 36), base + (2 << 36), base + (3 << 36),
                         base + (4 << 36), None, base + (5 << 36), None, None, n_seq, L,
                         n_seq * L, H, 128, dv, B.GDN_BF16, 1.0, 0)
    assert lib.gdn_chunk_fwd_noalloc(ctypes.byref(p), None) == B.GDN_ERR_WORKSPACE


def _kda_case(label, L, H):
    wl = dataclasses.replace(W.WORKLOADS["looped_prefill"], name=label, H=H, seq_len=L)
    inp = W.prefill_inputs(wl, "cuda")
    inp["a"], inp["b"] = W.channel_gates(L, H, 128, "cuda", label)
    o = torch.full((L, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    S_T = torch.full((1, H, 128, 128), float("nan"), device="cuda")
    p = B.gdn_fwd_params(inp["q"].data_ptr(), inp["k"].data_ptr(), inp["v"].data_ptr(),
                         inp["a"].data_ptr(), inp["b"].data_ptr(), None, o.data_ptr(), S_T.data_ptr(),
                         None, 1, L, L, H, 128, 128, B.GDN_BF16, 1.0,
                         B.GDN_CHANNEL_GATE | B.GDN_QK_L2NORM)
    return inp, p, o, S_T


def test_noalloc_channel_gate_schedules(lib):
    """The per-channel gate prefill: a call whose two-launch workspace fits
    the array runs the two launches out of it (equal bit for bit to
    gdn_chunk_fwd with a workspace); one whose workspace does not (4096
    tokens x 16 heads) runs the one-launch kernel (equal bit for bit to
    gdn_chunk_fwd without one)."""
    inp, p, o, S_T = _kda_case("noalloc-kda-small", 512, 2)
    need = lib.gdn_chunk_fwd_workspace(ctypes.byref(p))
    assert 0 < need <= SCRATCH_BYTES
    fl = B.GDN_CHANNEL_GATE | B.GDN_QK_L2NORM
    o_ref, S_ref = lla.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], flags=fl)
    assert lib.gdn_chunk_fwd_noalloc(ctypes.byref(p), None) == B.GDN_OK
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(S_T, S_ref)

    inp, p, o, S_T = _kda_case("noalloc-kda-large", 4096, 16)
    assert lib.gdn_chunk_fwd_workspace(ctypes.byref(p)) > SCRATCH_BYTES
    o1 = torch.full_like(o, float("nan"))
    S1 = torch.full_like(S_T, float("nan"))
    p1 = B.gdn_fwd_params(*(getattr(p, f) for f, _ in B.gdn_fwd_params._fields_))
    p1.o, p1.S_T = o1.data_ptr(), S1.data_ptr()
    assert lib.gdn_chunk_fwd(ctypes.byref(p1), None, 0, None) == B.GDN_OK
    assert lib.gdn_chunk_fwd_noalloc(ctypes.byref(p), None) == B.GDN_OK
    torch.cuda.synchronize()
    assert lla.gdn_get_device_status() == lla.GDN_OK
    assert torch.isfinite(S1).all()
    assert torch.equal(o, o1) and torch.equal(S_T, S1)
