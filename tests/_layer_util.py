"""Moving a synth LayerCase to the GPU and running the library's layer."""
import numpy as np

from synth.torch_io import to_dev


def layer_to_dev(lc, cap_extra: int = 1, device="cuda"):
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


def layer_dims(lc, cap):
    import token_level_dynamic_b200 as wl
    a, f = lc.attn, lc.ffn
    return wl.wide_layer_dims(a.n_seq, a.seq_len, a.cache_len, cap, a.H, f.I, f.gs, a.n_q,
                              a.n_kv, a.hd, a.theta, a.eps)
