"""Helpers shared by the GPU parity tests (comparison metrics, host copies)."""
import numpy as np
import torch

# Parity bars: relative L2 error over a whole tensor.
TOL_F32 = 1e-4                 # fp32 inputs
TOL_BF16_O = 1e-2              # bf16 inputs: outputs
TOL_BF16_S = 5e-3              # bf16 inputs: final fp32 state


def rel_l2(x, ref) -> float:
    x = np.asarray(x.detach().cpu().double().numpy() if hasattr(x, "detach") else x, dtype=np.float64)
    if hasattr(ref, "detach"):
        ref = ref.detach().cpu().double().numpy()
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(x - ref)
    return float(num / den) if den > 0 else float(num)


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
