"""Planted mistakes in the oracle (CPU only).

Each mutant below is a plausible error in one oracle function: a dropped
term, a wrong sign, a transposed operand, a wrong index or axis, a wrong
comparison.  The test swaps it in for the real function (in the oracle
module and in the pin module that imported it) and checks that at least
one of the pins written for that function fails, and that all of them pass
with the real function.  This is what makes the pins evidence: a pin that
no plausible mistake can fail would prove nothing.
"""
import numpy as np
import pytest

import oracle.attention as A
import oracle.ffn as F
import oracle.router as R
import tests.test_oracle_attention as TA
import tests.test_oracle_ffn as TF
import tests.test_oracle_router as TR


def _failing(pins):
    failed = []
    for name, fn in pins:
        try:
            fn()
        except Exception:          # an assertion, or a shape error from the mutant
            failed.append(name)
    return failed


def _swap(monkeypatch, name, fn, modules):
    for m in modules:
        if hasattr(m, name):
            monkeypatch.setattr(m, name, fn)


# ------------------------------------------------------------------ router

ROUTER_PINS = [
    ("worked example, bias", lambda: TR.test_worked_example("definition", True)),
    ("worked example, no bias", lambda: TR.test_worked_example("definition", False)),
    ("zero logit skips", TR.test_zero_logit_skips),
    ("torch layers relu", lambda: TR.test_equals_torch_layers("relu", 0.05)),
    ("torch layers silu", lambda: TR.test_equals_torch_layers("silu", 0.05)),
    ("sign flip", TR.test_sign_flip_inverts_decisions),
    ("forced by bias", TR.test_group_forced_by_bias),
    ("packing", TR.test_packing_layout),
]

_real_logits = R.route_logits


def _logits_mutant(kind):
    def f(x, w_r1, w_r2, b_r2=None, act="relu"):
        X = F.widen(x, "bf16")
        W1, W2 = F.widen(w_r1, "bf16"), F.widen(w_r2, "bf16")
        pre = X @ W1.T
        if kind == "no_activation":
            z = pre
        elif kind == "act_swapped":
            z = F.silu(pre) if act == "relu" else np.maximum(pre, 0.0)
        else:
            z = np.maximum(pre, 0.0) if act == "relu" else F.silu(pre)
        lg = z @ W2 if kind == "w2_transposed" else z @ W2.T
        if b_r2 is not None and kind != "no_bias":
            b = np.asarray(b_r2, dtype=np.float32).astype(np.float64)[None, :]
            lg = lg - b if kind == "bias_sign" else lg + b
        return lg
    return f


@pytest.mark.parametrize("kind", ["no_bias", "bias_sign", "w2_transposed", "no_activation",
                                  "act_swapped"])
def test_router_logit_mutants_are_caught(monkeypatch, kind):
    _swap(monkeypatch, "route_logits", _logits_mutant(kind), (R, TR))
    assert _failing(ROUTER_PINS), kind


def test_router_decision_and_packing_mutants_are_caught(monkeypatch):
    with monkeypatch.context() as m:
        _swap(m, "decide", lambda lg: np.asarray(lg) >= 0.0, (R, TR))
        assert _failing(ROUTER_PINS), "decide >= 0"

    def pack_reversed(keep):
        keep = np.asarray(keep, dtype=bool)
        T, G = keep.shape
        out = np.zeros((T, (G + 31) // 32), dtype=np.uint32)
        for g in range(G):
            out[:, g // 32] |= keep[:, g].astype(np.uint32) << np.uint32(31 - g % 32)
        return out

    with monkeypatch.context() as m:
        _swap(m, "pack", pack_reversed, (R, TR))
        assert _failing(ROUTER_PINS), "bit order reversed"


def test_router_pins_pass_unmutated():
    assert R.route_logits is _real_logits
    assert _failing(ROUTER_PINS) == []


# --------------------------------------------------------------------- FFN

FFN_PINS = [
    ("worked example", lambda: TF.test_worked_example("definition")),
    ("equals C token loop", lambda: TF.test_definition_equals_token_loop("bf16", (7, 64, 256, 32))),
    ("all ones = torch dense", TF.test_all_ones_equals_library_dense),
    ("all zeros = 0", TF.test_all_zero_mask_is_exactly_zero),
    ("one group's term", TF.test_removing_one_group_removes_exactly_its_term),
]


def _ffn_mutant(kind):
    def f(X, Wg, Wu, Wd, m, gs):
        if kind == "gate_up_swapped":
            h = F.silu(X @ Wu.T) * (X @ Wg.T)
        elif kind == "no_silu":
            h = (X @ Wg.T) * (X @ Wu.T)
        else:
            h = F.silu(X @ Wg.T) * (X @ Wu.T)
        if kind == "mask_tiled":
            h = h * np.tile(m, (1, gs))          # group of channel c taken as c % G
        elif kind != "mask_ignored":
            h = h * np.repeat(m, gs, axis=1)
        return h @ Wd.T
    return f


@pytest.mark.parametrize("kind", ["gate_up_swapped", "no_silu", "mask_tiled", "mask_ignored"])
def test_ffn_mutants_are_caught(monkeypatch, kind):
    _swap(monkeypatch, "ffn_masked_f64", _ffn_mutant(kind), (F,))
    assert _failing(FFN_PINS), kind


def test_ffn_pins_pass_unmutated():
    assert _failing(FFN_PINS) == []


# --------------------------------------------------------------- attention

ATTN_PINS = [
    ("rmsnorm closed form", TA.test_rmsnorm_closed_form),
    ("rope closed forms", TA.test_rope_closed_forms_and_identity_at_zero),
    ("rope relative phase", TA.test_rope_is_a_rotation_with_relative_phase),
    ("torch sdpa, prefill",
     lambda: TA.test_all_groups_kept_equals_library_attention("prefill", dict(n_seq=2, seq_len=24))),
    ("torch sdpa, decode",
     lambda: TA.test_all_groups_kept_equals_library_attention("decode", dict(n_seq=3, cache_len=40))),
    ("q = 0 averages V", TA.test_zero_queries_average_visible_values),
]


def _rope_sign(v, pos, theta):
    hd = v.shape[-1]
    half = hd // 2
    inv = theta ** (-(2.0 * np.arange(half, dtype=np.float64)) / hd)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = v[..., :half], v[..., half:]
    return np.concatenate([a * c + b * s, b * c - a * s], axis=-1)


def _rope_adjacent_pairs(v, pos, theta):
    hd = v.shape[-1]
    inv = theta ** (-(2.0 * np.arange(hd // 2, dtype=np.float64)) / hd)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = v[..., 0::2], v[..., 1::2]
    out = np.empty_like(v)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = b * c + a * s
    return out


MUTANTS_ATTN = {
    "rope_sign": ("rope", _rope_sign),
    "rope_adjacent_pairs": ("rope", _rope_adjacent_pairs),
    "rmsnorm_no_gamma": ("rmsnorm", lambda x, gamma, eps: x / np.sqrt(
        np.mean(x * x, axis=-1, keepdims=True) + eps)),
    "rmsnorm_no_sqrt": ("rmsnorm", lambda x, gamma, eps: x / (
        np.mean(x * x, axis=-1, keepdims=True) + eps) * gamma),
    "softmax_wrong_axis": ("softmax_rows", lambda s: np.exp(s - np.max(s, axis=0, keepdims=True))
                           / np.sum(np.exp(s - np.max(s, axis=0, keepdims=True)), axis=0,
                                    keepdims=True)),
}


@pytest.mark.parametrize("kind", sorted(MUTANTS_ATTN))
def test_attention_mutants_are_caught(monkeypatch, kind):
    name, fn = MUTANTS_ATTN[kind]
    with np.errstate(all="ignore"):
        _swap(monkeypatch, name, fn, (A, TA))
        assert _failing(ATTN_PINS), kind


def test_attention_pins_pass_unmutated():
    assert _failing(ATTN_PINS) == []
