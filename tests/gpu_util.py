"""Helpers shared by the GPU parity tests (comparison metrics, host copies)."""
import numpy as np
import torch

# Parity bars: relative L2 error over a whole tensor.
TOL_F32 = 1e-4                 # fp32 inputs
TOL_BF16_O = 1e-2              # bf16 inputs: outputs
TOL_BF16_S = 5e-3              # bf16 inputs: final fp32 state
# Finer-grained bars checked beside the whole-tensor ones: every sequence's
# outputs (all heads) and final states at the same bars as the whole tensor,
# and every 64-row chunk of one (sequence, head) chain's outputs within
# CHUNK_FACTOR times the output bar.  One wrong row in a chunk moves that
# chunk's error by about 1/8 (the row's share of the chunk's norm), so a
# wrong row or a wrong short sequence cannot hide under a long one.
CHUNK_ROWS = 64
CHUNK_FACTOR = 2.0


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def rel_l2(x, ref) -> float:
    x, ref = _f64(x), _f64(ref)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(x - ref)
    return float(num / den) if den > 0 else float(num)


def seq_bounds(inp) -> list:
    """(first, end) token of every sequence of a prefill input dict."""
    cu = inp.get("cu_seqlens")
    if cu is None:
        L = inp["seq_len"]
        return [(s * L, (s + 1) * L) for s in range(inp["n_seq"])]
    cu = np.asarray(cu)
    return [(int(cu[s]), int(cu[s + 1])) for s in range(len(cu) - 1)]


def worst_chunk_error(o, o_ref, bounds) -> float:
    """Largest relative L2 error over the 64-row chunks (counted from each
    sequence's first token) of every (sequence, head) chain of o [tokens, H, dv].
    A chunk's denominator is floored at 1e-3 of its chain's RMS row norm, so a
    chunk whose reference is nearly zero does not divide by nothing."""
    x, r = _f64(o), _f64(o_ref)
    worst = 0.0
    for t0, t1 in bounds:
        n = t1 - t0
        if n <= 0:
            continue
        d = x[t0:t1] - r[t0:t1]                          # [n, H, dv]
        pad = (-n) % CHUNK_ROWS
        d2 = np.pad((d * d).sum(-1), ((0, pad), (0, 0)))  # [n + pad, H]
        r2 = np.pad((r[t0:t1] ** 2).sum(-1), ((0, pad), (0, 0)))
        num = d2.reshape(-1, CHUNK_ROWS, d2.shape[1]).sum(1)
        den = r2.reshape(-1, CHUNK_ROWS, r2.shape[1]).sum(1)
        rows = np.minimum(CHUNK_ROWS, n - CHUNK_ROWS * np.arange(num.shape[0]))[:, None]
        floor = 1e-6 * (r2.sum(0, keepdims=True) / n) * rows
        worst = max(worst, float(np.sqrt(num / np.maximum(den, floor + 1e-300)).max()))
    return worst


def check_prefill(o, ST, o_ref, S_ref, bounds, fp32: bool) -> dict:
    """Whole-tensor bars, then per-sequence and worst-chunk bars (see above).
    ST / S_ref are [n_seq, H, dk, dv]; sequences of length 0 have no outputs.
    Returns the measured errors."""
    bar_o = TOL_F32 if fp32 else TOL_BF16_O
    bar_s = TOL_F32 if fp32 else TOL_BF16_S
    x, r = _f64(o), _f64(o_ref)
    sx, sr = _f64(ST), _f64(S_ref)
    err = {"o": rel_l2(x, r), "S": rel_l2(sx, sr)}
    seq_o = [rel_l2(x[t0:t1], r[t0:t1]) for t0, t1 in bounds if t1 > t0]
    seq_s = [rel_l2(sx[s], sr[s]) for s in range(len(bounds))]
    err["seq_o"] = max(seq_o) if seq_o else 0.0
    err["seq_S"] = max(seq_s) if seq_s else 0.0
    err["chunk_o"] = worst_chunk_error(x, r, bounds)
    print("parity errors:", {k: f"{v:.3g}" for k, v in err.items()})
    assert err["o"] < bar_o and err["S"] < bar_s, err
    assert err["seq_o"] < bar_o and err["seq_S"] < bar_s, err
    assert err["chunk_o"] < CHUNK_FACTOR * bar_o, err
    return err


def host(t: torch.Tensor) -> torch.Tensor:
    return t.detach().cpu()


def to_dev(d: dict, device="cuda") -> dict:
    out = {}
    for k, v in d.items():
        out[k] = v.to(device) if isinstance(v, torch.Tensor) else v
    return out


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    e = np.floor(np.log2(ax))
    return 2.0 ** (e - 7)
