"""Moving a synth LayerCase to the GPU and describing it to the library."""
from synth.torch_io import layer_to_dev  # noqa: F401


def layer_dims(lc, cap):
    import token_level_dynamic_b200 as wl
    a, f = lc.attn, lc.ffn
    return wl.wide_layer_dims(a.n_seq, a.seq_len, a.cache_len, cap, a.H, f.I, f.gs, a.n_q,
                              a.n_kv, a.hd, a.theta, a.eps)
