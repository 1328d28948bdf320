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


def layer_to_dev(lc, cap_extra: int = 1, device="cuda"):
    """A LayerCase on the device: (x, weights dict, k_cache, v_cache,
    head mask words, FFN mask words, cache capacity).  The caches hold the
    case's past positions and room for cap_extra new positions per token."""
    import torch
    a, f = lc.attn, lc.ffn
    w = {"gamma1": to_dev(a.gamma1, "bf16", device), "wq": to_dev(a.wq, "bf16", device),
         "wk": to_dev(a.wk, "bf16", device), "wv": to_dev(a.wv, "bf16", device),
         "wo": to_dev(a.wo, "bf16", device), "gamma2": to_dev(lc.gamma2, "bf16", device),
         "w_gate": to_dev(f.w_gate, "bf16", device), "w_up": to_dev(f.w_up, "bf16", device),
         "w_down": to_dev(f.w_down, "bf16", device)}
    cap = a.cache_len + a.seq_len + cap_extra - 1
    kc = torch.zeros((a.n_seq, a.n_kv, cap, a.hd), dtype=torch.bfloat16, device=device)
    vc = torch.zeros_like(kc)
    if a.cache_len > 0:
        kc[:, :, :a.cache_len] = to_dev(a.k_cache, "bf16", device)
        vc[:, :, :a.cache_len] = to_dev(a.v_cache, "bf16", device)
    x = to_dev(a.x, "bf16", device)
    hm = to_dev(a.mask_words, "mask", device)
    fm = to_dev(f.mask_words, "mask", device)
    return x, w, kc, vc, hm, fm, cap
