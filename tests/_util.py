"""Helpers shared by the tests: move synth cases to the GPU, compare."""
import numpy as np

from synth.torch_io import to_dev  # noqa: F401


def rel_l2(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def from_dev(t) -> np.ndarray:
    import torch
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.float().numpy().astype(np.float64)
    return t.numpy().astype(np.float64)


def ffn_to_dev(c, device="cuda"):
    kind = "bf16" if c.dtype == "bf16" else "f32"
    return (to_dev(c.x, kind, device), to_dev(c.w_gate, kind, device), to_dev(c.w_up, kind, device),
            to_dev(c.w_down, kind, device), to_dev(c.mask_words, "mask", device))
