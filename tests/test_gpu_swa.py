"""GPU parity of the sliding-window causal softmax attention against the oracle.

The window mixer of the hybrid LT2 loops ("LT2: Linear-Time Looped
Transformers", §2 and Appendix C: windows of w = 256 at 0.6B and w = 2048 at
1.3B, the token itself and the w - 1 before it).  bf16 inputs and outputs,
fp32 accumulation, P rounded to bf16 for the second product: the bar is the
bf16 output bar, relative L2 1e-2, over the whole tensor, every sequence, and
every 64-row chunk of every (sequence, head) within twice that.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import looped_linear_attention_b200 as lla
from looped_linear_attention_b200 import workloads as W
from gpu_util import CHUNK_FACTOR, TOL_BF16_O, host, rel_l2, worst_chunk_error

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


def _qkv(label, T, H):
    q, k, v = W.qkv(T, H, 128, 128, torch.bfloat16, False, "cpu", "test", "swa", label)
    return q, k, v


def _bounds(lengths):
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return cu, [(int(cu[i]), int(cu[i + 1])) for i in range(len(lengths))]


def _check(o, ref, bounds):
    x, r = host(o).double().numpy(), np.asarray(ref)
    err = {"o": rel_l2(x, r)}
    seq = [rel_l2(x[a:b], r[a:b]) for a, b in bounds if b > a]
    err["seq_o"] = max(seq) if seq else 0.0
    err["chunk_o"] = worst_chunk_error(x, r, bounds)
    print("parity errors:", {k: f"{v:.3g}" for k, v in err.items()})
    assert err["o"] < TOL_BF16_O and err["seq_o"] < TOL_BF16_O, err
    assert err["chunk_o"] < CHUNK_FACTOR * TOL_BF16_O, err
    return err


def _run(q, k, v, window, lengths=None, n_seq=1, scale=None):
    if lengths is not None:
        cu, _ = _bounds(lengths)
        o = lla.swa_fwd(q.cuda(), k.cuda(), v.cuda(), window, torch.from_numpy(cu).cuda(),
                        max_seq_len=max(lengths), scale=scale)
    else:
        o = lla.swa_fwd(q.cuda(), k.cuda(), v.cuda(), window, n_seq=n_seq, scale=scale)
    torch.cuda.synchronize()
    _status_ok()
    return o


@pytest.mark.parametrize("window", [256, 100, 1000])
def test_swa_fixed_length_ragged(window):
    """Two sequences of 700 tokens (a ragged last query tile), windows that
    start mid-tile (100), span several key tiles (256) or most of the sequence."""
    q, k, v = _qkv(f"fixed-{window}", 1400, 2)
    o = _run(q, k, v, window, n_seq=2)
    ref = oracle.swa_fwd(q, k, v, window, np.array([0, 700, 1400], dtype=np.int32))
    _check(o, ref, [(0, 700), (700, 1400)])


def test_swa_varlen_edges():
    lengths = [0, 1, 127, 128, 129, 300, 1000]
    q, k, v = _qkv("varlen", sum(lengths), 2)
    o = _run(q, k, v, 256, lengths=lengths)
    cu, bounds = _bounds(lengths)
    _check(o, oracle.swa_fwd(q, k, v, 256, cu), bounds)


def test_swa_window_of_one_returns_values_exactly():
    q, k, v = _qkv("w1", 300, 2)
    o = _run(q, k, v, 1)
    assert torch.equal(host(o), v)


def test_swa_window_beyond_the_sequence_is_causal_attention():
    q, k, v = _qkv("full", 333, 2)
    o = _run(q, k, v, 1 << 20, scale=0.2)
    ref = oracle.swa_fwd(q, k, v, 1 << 20, scale=0.2)
    _check(o, ref, [(0, 333)])


def test_swa_equal_scores_average_the_window():
    """Zero keys: o_t is the mean of v over the window (up to bf16 rounding)."""
    q, _, v = _qkv("mean", 500, 1)
    k = torch.zeros_like(q)
    o = _run(q, k, v, 64)
    ref = np.stack([v[max(0, t - 63):t + 1].double().mean(0).numpy() for t in range(500)])
    _check(o, ref, [(0, 500)])


def test_swa_growing_scores_rescale_the_running_sums():
    """Scores that grow along the keys (q . k_j increasing with j, large
    scale): the running maximum rises in every key tile, so the rows' O and l
    are rescaled in tensor memory repeatedly."""
    T = 1024
    q, _, v = _qkv("grow", T, 1)
    q = torch.ones(T, 1, 128).bfloat16()
    k = (torch.linspace(0.0, 1.0, T)[:, None, None] * torch.ones(T, 1, 128)).bfloat16()
    o = _run(q, k, v, 700, scale=0.5)
    ref = oracle.swa_fwd(q, k, v, 700, scale=0.5)
    _check(o, ref, [(0, T)])


def test_swa_window_2048_on_4096_tokens():
    """The 1.3B setting: w = 2048 on a 4096-token sequence (16 key tiles per
    query tile at most), two heads."""
    q, k, v = _qkv("w2048", 4096, 2)
    o = _run(q, k, v, 2048)
    _check(o, oracle.swa_fwd(q, k, v, 2048), [(0, 4096)])
