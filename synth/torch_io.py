"""numpy -> torch device tensors for synth arrays (bf16 bit patterns become
torch.bfloat16, packed uint32 mask words become int32 bit patterns)."""
import numpy as np


def to_dev(a: np.ndarray, kind: str, device="cuda"):
    import torch
    a = np.ascontiguousarray(a)
    if kind == "bf16":
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    if kind == "f32":
        return torch.from_numpy(a.astype(np.float32)).to(device)
    if kind == "mask":
        return torch.from_numpy(a.astype(np.uint32).view(np.int32)).to(device)
    raise ValueError(kind)
