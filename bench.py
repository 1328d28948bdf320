#!/usr/bin/env python
"""Benchmark of the masked WIDE layer on B200; prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode_ffn_3b|prefill_ffn_8b|decode_layer_8b|
                                prefill_layer_8b [--keep K]]

Workloads (seeded synthetic inputs with the shapes the pages name):
  decode_ffn_3b (default)  Llama-3.2-3B-shaped masked SwiGLU FFN in decode:
      hidden 3072, intermediate 8192 in 64 groups of 128, bf16, Bernoulli(0.5)
      masks.  One step = the three batch sizes of the configuration (1, 8
      and 32 tokens, each with its own x and mask): 41 tokens.  HBM-bound;
      the roofline is union-of-groups weight bytes over measured HBM GB/s.
  decode_layer_8b  Llama-3.1-8B-shaped masked decode layer, batch 16 with a
      2048-entry KV cache: attention (QKV+RoPE, GQA over the cache, o_proj)
      with head groups kept at 0.34 and the FFN with groups kept at 0.72.
      HBM-bound; the roofline is union weight bytes + kept KV bytes.
  prefill_layer_8b  Llama-3.1-8B-shaped masked prefill layer, 4 sequences
      x 2048 tokens, head and FFN groups from 16 prototypes at keep 0.5 (0.25,
      0.75, 1.0 with --keep) + 0.1 flips.  Tensor bound on kept FLOPs.
  prefill_ffn_8b  Llama-3.1-8B-shaped masked SwiGLU FFN in prefill: 4096
      tokens, hidden 4096, intermediate 14336 in 112 groups of 128, 8
      prototype masks (56 groups each) with 0.1 bit flips.  One step = one
      call (mask reordering, zero fill, tcgen05 gate/up and down).  Tensor
      bound; the roofline is kept FLOPs over the measured bf16 tensor peak.

Timing: W untimed warm-up steps, then exactly K steps between a barrier and a
device synchronise on both sides.  Each call is timed with CUDA events on the
launch stream after an L2 flush (a 256 MiB write, then a read of it so that
L2 holds clean lines) that sits outside the events; ms_per_step is the sum
of the call times, maximised over ranks.  Kernel times for the roofline come
from the library's own per-launch begin/end events (wide_profile_*),
recorded on the launch stream in a second pass of the same K steps right
after the timed one (those events cost a few us per call, so the timed pass
runs without them).  SM clocks and throttle reasons are sampled through NVML
during the timed steps.

Multi-GPU: every rank runs the same workload on its own GPU (replicas, weak
scaling); value = all ranks' tokens / the slowest rank's time.

``--impl reference`` times the fp64 CPU oracle (oracle/, the per-token loop
over kept groups) on the host cores, one bounded token sample per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "masked-layer tok/s @50% sparsity; HBM GB/s (decode), TFLOPS (prefill)"
FLUSH_BYTES = 256 << 20


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def _nvml_handle(nv, cuda_index: int):
    """NVML handle of CUDA device `cuda_index`, honouring CUDA_VISIBLE_DEVICES."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").strip()
    if vis:
        ent = vis.split(",")[cuda_index].strip()
        if ent.startswith("GPU-") or ent.startswith("MIG-"):
            return nv.nvmlDeviceGetHandleByUUID(ent)
        return nv.nvmlDeviceGetHandleByIndex(int(ent))
    return nv.nvmlDeviceGetHandleByIndex(cuda_index)


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML (read-only)."""

    def __init__(self, index: int, period: float = 0.01):
        self.index, self.period = index, period
        self.samples, self.reasons = [], set()
        self._stop = threading.Event()
        self._t = None
        self.max_mhz = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self._nv = nv
            self._h = _nvml_handle(nv, self.index)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self._h, nv.NVML_CLOCK_SM)
            self.ok = True
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception:
            self.ok = False
        return self

    def _run(self):
        nv = self._nv
        names = {
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for k, bit in names.items():
                    if r & bit:
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join(timeout=2)

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples), "source": "nvml" if self.ok else "unavailable"}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


def _traffic_record(kernel: str, workload: str):
    """DRAM bytes per step from the committed ncu summary, if the kernel
    source it was taken on is unchanged."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[workload][kernel]
        src = os.path.join(ROOT, rec["source"])
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if digest != rec["source_sha256_16"]:
            return None
        return rec
    except Exception:
        return None


# --------------------------------------------------------------- workloads
# A workload builds its seeded cases, states the algorithmic units of every
# library kernel it launches, runs the oracle on a bounded sample, and sets
# up device buffers with the calls that the timing loop makes.

class FFNDevice:
    """Device buffers and calls of a masked-FFN workload (one call per case)."""

    def __init__(self, wl, cases, dev, stream):
        import torch
        import token_level_dynamic_b200 as w
        from synth.torch_io import to_dev
        self.w, self.stream, self.cases = w, stream, cases
        base = cases[0]
        self.Wg = to_dev(base.w_gate, "bf16", dev)
        self.Wu = to_dev(base.w_up, "bf16", dev)
        self.Wd = to_dev(base.w_down, "bf16", dev)
        self.xs = [to_dev(c.x, "bf16", dev) for c in cases]
        self.ms = [to_dev(c.mask_words, "mask", dev) for c in cases]
        self.outs = [torch.empty_like(x) for x in self.xs]
        self.path = getattr(w, wl.path_name)
        ws_bytes = max(w.wide_ffn_workspace_bytes(c.T, c.H, c.I, c.gs, path=self.path)
                       for c in cases)
        self.ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        self.ones = [_all_ones(m, base.I // base.gs) for m in self.ms]
        self.ncalls = len(cases)
        # decode: the weights' packed copy, made once like loading the weights
        # (outside every timed region); each call then hands the library
        # both copies and it picks the kernel per launch
        self.packed = (w.wide_ffn_pack(self.Wg, self.Wu, self.Wd)
                       if self.path == w.WIDE_PATH_DECODE else None)
        # e2e: pinned host copies of each call's inputs and output
        self.xh = [x.cpu().pin_memory() for x in self.xs]
        self.mh = [m.cpu().pin_memory() for m in self.ms]
        self.oh = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in self.outs]
        self.h2d_bytes = int(sum(x.numel() * 2 + m.numel() * 4 for x, m in zip(self.xh, self.mh)))
        self.d2h_bytes = int(sum(o.numel() * 2 for o in self.oh))

    def call(self, i, all_kept=False):
        m = self.ones[i] if all_kept else self.ms[i]
        if self.packed is not None:
            self.w.wide_ffn_masked_packed(self.xs[i], self.packed, m, self.cases[i].gs,
                                          self.cases[i].I, out=self.outs[i], workspace=self.ws,
                                          stream=self.stream, weights=(self.Wg, self.Wu, self.Wd))
            return
        self.w.wide_ffn_masked(self.xs[i], self.Wg, self.Wu, self.Wd, m, self.cases[i].gs,
                               out=self.outs[i], workspace=self.ws, path=self.path,
                               stream=self.stream)

    def e2e_call(self, i):
        self.xs[i].copy_(self.xh[i], non_blocking=True)
        self.ms[i].copy_(self.mh[i], non_blocking=True)
        self.call(i)
        self.oh[i].copy_(self.outs[i], non_blocking=True)

    def naive_gather_scatter(self, i):
        """The naive masked FFN the pages compare against: for each group, copy
        out the rows of the tokens that keep it (index_select, whose size
        needs a device-to-host sync), run the three matmuls on that copy, and
        scatter-add the result back (index_add).  torch ops only."""
        import torch
        import torch.nn.functional as F
        c, x, m = self.cases[i], self.xs[i], self.ms[i]
        gs, G = c.gs, c.I // c.gs
        sh = torch.arange(32, device=m.device, dtype=torch.int32)
        bits = ((m.unsqueeze(-1) >> sh) & 1).reshape(m.shape[0], -1)[:, :G].bool()
        acc = torch.zeros(x.shape, dtype=torch.float32, device=x.device)
        for g in range(G):
            idx = bits[:, g].nonzero().squeeze(1)
            if idx.numel() == 0:
                continue
            xg = x.index_select(0, idx)
            sl = slice(g * gs, (g + 1) * gs)
            h = F.silu(xg @ self.Wg[sl].T) * (xg @ self.Wu[sl].T)
            acc.index_add_(0, idx, (h @ self.Wd[:, sl].T).float())
        self.outs[i].copy_(acc)

    def dense_torch(self, i):
        import torch.nn.functional as F
        x = self.xs[i]
        self.outs[i].copy_(F.linear(F.silu(F.linear(x, self.Wg)) * F.linear(x, self.Wu), self.Wd))


def _all_ones(m, G):
    import torch
    o = torch.full_like(m, -1)
    if G % 32:
        o[:, -1] = (1 << (G % 32)) - 1
    return o


class DecodeFFN3B:
    name = "decode_ffn_3b"
    desc = ("decode_ffn_3b: Llama-3.2-3B-shaped masked SwiGLU FFN decode, hidden 3072, "
            "intermediate 8192 = 64 groups x 128, bf16, Bernoulli(0.5) masks; one step = "
            "batches 1, 8 and 32 (41 tokens); weights also packed once (wide_ffn_pack, outside "
            "timing) and passed with the nn.Linear copy, so the library picks the kernel per "
            "launch")
    bound = "hbm"
    dominant = None          # the kernel with the largest share of the step
    path_name = "WIDE_PATH_DECODE"
    device = FFNDevice

    def make_cases(self):
        import synth
        base = synth.decode_ffn(1)
        cases = [base]
        for b in (8, 32):
            c = synth.decode_ffn(b, weights=False)
            c.w_gate, c.w_up, c.w_down = base.w_gate, base.w_up, base.w_down
            cases.append(c)
        return cases

    @staticmethod
    def units(case):
        """Algorithmic bytes per call and kernel: every weight byte (gate, up,
        down) of the batch's union of groups once, plus activations."""
        return _ffn_decode_bytes(case)

    def reference_sample(self, cases):
        # one call of n tokens (the oracle's token loop runs one token per
        # OpenMP thread, so n = the host threads, at most the batch of 32)
        c = cases[-1]
        n = max(1, min(c.T, _host_cores()))
        s = type(c)(**{**c.__dict__})
        s.x, s.mask, s.T = c.x[:n], c.mask[:n], n
        return [s], f"per step: the first {n} tokens of the batch-32 call, in one oracle call"

    reference_step = staticmethod(lambda samples: _ffn_oracle_step(samples))


def _split_decode_used(T, H, I, gs, sms=148):
    """Mirror of the library's limits of the channel-split decode kernel
    (plan_split in ffn_decode_split.cu): launches of up to 16 tokens,
    H % 256 == 0, the group size a multiple of 8 in 8..256 dividing I, at
    most 1024 groups (at most 8 whole groups per CTA)."""
    T1 = min(T, 16)
    if not (T1 >= 1 and H % 256 == 0 and gs % 8 == 0 and 8 <= gs <= 256 and I % gs == 0):
        return False
    G = I // gs
    return not (G > 1024 or T1 * (-(-G // 32)) > 1024 or -(-G // sms) > 8)


def _tc_decode_used(T, H, I, gs, sms=148):
    """Mirror of the tensor-core decode kernel's limits (plan_tc in
    ffn_decode_tc.cu): launches of up to 32 tokens, H % 128 == 0, group size
    a multiple of 16 up to 256, at most 1024 groups and 16 chunks of 16
    channels per CTA."""
    G = I // gs if gs else 0
    return (H % 128 == 0 and gs % 16 == 0 and 16 <= gs <= 256 and I % gs == 0 and G <= 1024 and
            -(-(I // 16) // sms) <= 16)


def _ffn_decode_bytes(case, res_bytes=0, x_bytes=None):
    """Algorithmic bytes per kernel of one decode FFN call, following the
    library's choice per launch (AUTO): the channel-split kernel for up to 8
    tokens, the tensor-core kernel (launches of up to 32 tokens) above.  Per
    launch, every weight byte of that launch's union of groups once, plus
    activations in and out; the fp32 accumulators are not counted (they live
    in L2).  The GEMV path (neither kernel applies): h goes through memory."""
    B, H, I, gs = case.T, case.H, case.I, case.gs
    U = int(case.mask.any(axis=0).sum())
    m = case.mask_words.nbytes
    xb = B * H * 2 if x_bytes is None else x_bytes
    io = xb + m + B * H * 2 + res_bytes
    split_ok, tc_ok = _split_decode_used(B, H, I, gs), _tc_decode_used(B, H, I, gs)
    if not (split_ok or tc_ok):
        pairs = int(case.mask.sum())
        h = pairs * gs * 4
        gateup = 2 * U * gs * H * 2 + xb + m + h
        down = H * U * gs * 2 + h + m + B * H * 2 + res_bytes
        return {"decode_gateup_gemv": gateup, "decode_down_gemv": down,
                "total": gateup + down, "union_groups": U}
    out, t0 = {}, 0
    while t0 < B:
        rem = B - t0
        if split_ok and (rem <= 8 or not tc_ok):
            name, per = "decode_ffn_split_gemv", 16
        else:
            name, per = "decode_ffn_tcgen05", 32
        n = min(rem, per)
        u = int(case.mask[t0:t0 + n].any(axis=0).sum())
        out[name] = out.get(name, 0) + 3 * u * gs * H * 2
        t0 += n
    # activations: on the kernel of the first launch
    first = next(iter(out))
    out[first] += io
    out["total"] = sum(out.values())
    out["union_groups"] = U
    return out


def _ffn_oracle_step(samples):
    import oracle
    for c in samples:
        oracle.ffn.ffn_token_loop(c.x, c.w_gate, c.w_up, c.w_down, c.mask_words, c.gs, "bf16")
    return sum(c.T for c in samples)


class PrefillFFN8B:
    name = "prefill_ffn_8b"
    desc = ("prefill_ffn_8b: Llama-3.1-8B-shaped masked SwiGLU FFN prefill, 4096 tokens, hidden "
            "4096, intermediate 14336 = 112 groups x 128, bf16, 8 prototype masks (56 groups) + "
            "0.1 flips; one step = one call")
    bound = "tensor"
    dominant = "prefill_gateup_tcgen05"
    path_name = "WIDE_PATH_PREFILL"
    device = FFNDevice

    def make_cases(self):
        import synth
        return [synth.prefill_ffn()]

    @staticmethod
    def units(case):
        """Kept FLOPs per call: 2 flops per multiply-add, only (token, kept
        group) work; gate and up in the first kernel, down in the second."""
        H, gs = case.H, case.gs
        pairs = int(case.mask.sum())
        gateup = 2 * 2 * H * gs * pairs
        down = 2 * H * gs * pairs
        return {"prefill_gateup_tcgen05": gateup, "prefill_down_tcgen05": down,
                "total": gateup + down, "pairs": pairs,
                "dense_flops": 6 * case.T * H * case.I}

    def reference_sample(self, cases):
        c = cases[0]
        n = max(8, min(32, _host_cores()))
        s = type(c)(**{**c.__dict__})
        s.x, s.mask, s.T = c.x[:n], c.mask[:n], n
        return [s], f"per step: the first {n} tokens of the 4096-token batch, in one oracle call"

    reference_step = staticmethod(lambda samples: _ffn_oracle_step(samples))


class LayerDevice:
    """Device buffers and calls of a masked-layer workload (one call)."""

    def __init__(self, wl, cases, dev, stream):
        import torch
        import token_level_dynamic_b200 as w
        from synth.torch_io import layer_to_dev
        self.w, self.stream = w, stream
        lc = cases[0]
        self.lc = lc
        self.x, self.wts, self.kc, self.vc, self.hm, self.fm, cap = layer_to_dev(lc, device=dev)
        a, f = lc.attn, lc.ffn
        if a.seq_len == 1:
            # decode: the FFN weights' packed copy, made once (outside timing)
            self.wts = dict(self.wts)
            self.wts["ffn_packed"] = w.wide_ffn_pack(self.wts["w_gate"], self.wts["w_up"],
                                                     self.wts["w_down"])
        self.d = w.wide_layer_dims(a.n_seq, a.seq_len, a.cache_len, cap, a.H, f.I, f.gs, a.n_q,
                                   a.n_kv, a.hd, a.theta, a.eps)
        self.out = torch.empty_like(self.x)
        self.ws = torch.empty(max(256, w.wide_layer_workspace_bytes(self.d)), dtype=torch.uint8,
                              device=dev)
        self.hm1 = _all_ones(self.hm, lc.attn.n_kv)
        self.fm1 = _all_ones(self.fm, lc.ffn.I // lc.ffn.gs)
        self.ncalls = 1
        self.xh = self.x.cpu().pin_memory()
        self.hmh = self.hm.cpu().pin_memory()
        self.fmh = self.fm.cpu().pin_memory()
        self.oh = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        self.h2d_bytes = int(self.x.numel() * 2 + self.hm.numel() * 4 + self.fm.numel() * 4)
        self.d2h_bytes = int(self.out.numel() * 2)

    def call(self, i, all_kept=False):
        self.w.wide_layer_masked(self.x, self.wts, self.kc, self.vc,
                                 self.hm1 if all_kept else self.hm,
                                 self.fm1 if all_kept else self.fm, self.d, out=self.out,
                                 workspace=self.ws, stream=self.stream)

    def e2e_call(self, i):
        self.x.copy_(self.xh, non_blocking=True)
        self.hm.copy_(self.hmh, non_blocking=True)
        self.fm.copy_(self.fmh, non_blocking=True)
        self.call(i)
        self.oh.copy_(self.out, non_blocking=True)

    def dense_torch(self, i):
        """The same layer unmasked with torch/cuBLAS ops (bf16)."""
        import torch
        import torch.nn.functional as F
        a = self.lc.attn
        W = self.wts
        x = self.x
        B, S, nq, nkv, hd = a.n_seq, a.seq_len, a.n_q, a.n_kv, a.hd
        L = a.cache_len
        xf = x.float()
        xn = (xf * torch.rsqrt(xf.pow(2).mean(-1, keepdim=True) + a.eps)).to(x.dtype) * W["gamma1"]
        q = F.linear(xn, W["wq"]).view(B, S, nq, hd).transpose(1, 2)
        k = F.linear(xn, W["wk"]).view(B, S, nkv, hd).transpose(1, 2)
        v = F.linear(xn, W["wv"]).view(B, S, nkv, hd).transpose(1, 2)
        pos = torch.arange(L, L + S, device=x.device, dtype=torch.float32)
        inv = a.theta ** (-torch.arange(0, hd, 2, device=x.device, dtype=torch.float32) / hd)
        ang = pos[:, None] * inv[None, :]
        cos, sin = torch.cos(ang).to(x.dtype), torch.sin(ang).to(x.dtype)

        def rope(t):
            t1, t2 = t[..., :hd // 2], t[..., hd // 2:]
            return torch.cat([t1 * cos - t2 * sin, t2 * cos + t1 * sin], -1)

        q, k = rope(q), rope(k)
        self.kc[:, :, L:L + S] = k
        self.vc[:, :, L:L + S] = v
        if S == 1:
            o = F.scaled_dot_product_attention(q, self.kc[:, :, :L + 1], self.vc[:, :, :L + 1],
                                               enable_gqa=True)
        else:
            o = F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True)
        h1 = x + F.linear(o.transpose(1, 2).reshape(B * S, nq * hd), W["wo"])
        hf = h1.float()
        xn2 = (hf * torch.rsqrt(hf.pow(2).mean(-1, keepdim=True) + a.eps)).to(x.dtype) * W["gamma2"]
        f = F.linear(F.silu(F.linear(xn2, W["w_gate"])) * F.linear(xn2, W["w_up"]), W["w_down"])
        self.out.copy_(h1 + f)


class DecodeLayer8B:
    name = "decode_layer_8b"
    desc = ("decode_layer_8b: Llama-3.1-8B-shaped masked decode layer (RMSNorm, QKV with 32 "
            "query / 8 KV heads of 128, RoPE theta 5e5, GQA attention over a 2048-entry KV "
            "cache, o_proj, RMSNorm, SwiGLU FFN 14336 = 112 groups x 128), batch 16, head "
            "groups Bernoulli(0.34), FFN groups Bernoulli(0.72); one step = one call; FFN "
            "weights also packed once (wide_ffn_pack, outside timing) for the decode FFN")
    bound = "hbm"
    dominant = None          # the kernel with the largest share of the step
    device = LayerDevice

    def make_cases(self):
        import synth
        return [synth.decode_layer()]

    @staticmethod
    def units(lc):
        """Algorithmic bytes per call, per kernel: union-of-groups weight
        bytes (each byte once per call), dense Wk/Wv, the kept K/V cache
        bytes, and the activations each kernel must read or write."""
        a, f = lc.attn, lc.ffn
        T, H, hd, nq, nkv = a.T, a.H, a.hd, a.n_q, a.n_kv
        rep = nq // nkv
        Ua = int(a.mask.any(axis=0).sum())
        kept_pairs = int(a.mask.sum())
        keys = a.cache_len + 1
        qkv = (Ua * rep * hd * H * 2 + 2 * nkv * hd * H * 2 + T * H * 2 + H * 2
               + kept_pairs * rep * hd * 4 + 2 * T * nkv * hd * 2)
        attn = kept_pairs * 2 * keys * hd * 2 + kept_pairs * rep * hd * 4 * 2
        oproj = H * Ua * rep * hd * 2 + kept_pairs * rep * hd * 4 + T * H * 2 * 2 + T * H * 4
        out = {"decode_qkv_rope_gemv": qkv, "decode_attention": attn}
        ffn = _ffn_decode_bytes(f, res_bytes=T * H * 4 + T * H * 2)
        if "decode_down_gemv" not in ffn:
            # FFN input norm (h1 fp32 in, bf16 out), then one persistent FFN
            # kernel: bf16 x and h1 in (residual), ffn_out and out back
            out["rmsnorm"] = T * H * 4 + T * H * 2 + H * 2
            out["decode_down_gemv"] = oproj
        else:
            norm = T * H * 4 + T * H * 2 + H * 2
            out["rmsnorm"] = norm
            out["decode_down_gemv"] = oproj + ffn.pop("decode_down_gemv")
        for k, v in ffn.items():
            if k not in ("total", "union_groups"):
                out[k] = v
        out["total"] = sum(v for k, v in out.items())
        out["union_groups"] = ffn["union_groups"]
        return out

    def reference_sample(self, cases):
        import copy
        lc = copy.deepcopy(cases[0])
        a = lc.attn
        keep = 2
        a.n_seq, a.x, a.mask = keep, a.x[:keep], a.mask[:keep]
        a.k_cache, a.v_cache = a.k_cache[:keep], a.v_cache[:keep]
        lc.ffn.mask, lc.ffn.T, lc.ffn.x = lc.ffn.mask[:keep], keep, lc.ffn.x[:keep]
        return [lc], "per step: sequences 0 and 1 of the 16 (2 tokens), fp64 definition form"

    @staticmethod
    def reference_step(samples):
        import oracle
        for lc in samples:
            oracle.attention.layer_masked(lc)
        return sum(lc.attn.T for lc in samples)


class PrefillLayer8B:
    name = "prefill_layer_8b"
    bound = "tensor"
    dominant = "prefill_gateup_tcgen05"
    device = LayerDevice

    def __init__(self, keep: float = 0.5):
        self.keep = keep
        self.desc = ("prefill_layer_8b: Llama-3.1-8B-shaped masked prefill layer, 4 sequences x "
                     "2048 tokens (RMSNorm, QKV with 32 query / 8 KV heads of 128, RoPE theta "
                     "5e5, causal GQA attention, o_proj, RMSNorm, SwiGLU FFN 14336 = 112 groups "
                     f"x 128), 16 prototype masks at keep {keep} + 0.1 flips; one step = one call")

    def make_cases(self):
        import synth
        return [synth.prefill_layer(keep=self.keep)]

    @staticmethod
    def units(lc):
        """Kept FLOPs per call, per kernel (2 per multiply-add): Q only for
        kept (token, head group) pairs; K/V for every token; attention for
        kept pairs over their causal keys; o_proj for kept pairs; the FFN
        for kept (token, channel group) pairs."""
        import numpy as np
        a, f = lc.attn, lc.ffn
        T, H, hd, nq, nkv = a.T, a.H, a.hd, a.n_q, a.n_kv
        rep = nq // nkv
        pairs_a = int(a.mask.sum())
        pos = np.tile(np.arange(a.seq_len), a.n_seq) + a.cache_len
        keys = int((a.mask * (pos[:, None] + 1)).sum())
        q = 2 * H * rep * hd * pairs_a
        kv = 2 * H * 2 * nkv * hd * T
        att = 4 * rep * hd * keys
        oproj = 2 * H * rep * hd * pairs_a
        pairs_f = int(f.mask.sum())
        gateup = 4 * H * f.gs * pairs_f
        down = 2 * H * f.gs * pairs_f
        dense = (2 * H * (nq + 2 * nkv) * hd * T + 4 * nq * hd * int((pos + 1).sum())
                 + 2 * H * nq * hd * T + 6 * H * f.I * T)
        total = q + kv + att + oproj + gateup + down
        return {"prefill_q_rope_tcgen05": q, "prefill_kv_rope_tcgen05": kv,
                "prefill_attention_tcgen05": att, "prefill_oproj_tcgen05": oproj,
                "prefill_gateup_tcgen05": gateup, "prefill_down_tcgen05": down,
                "total": total, "dense_flops": dense}

    def reference_sample(self, cases):
        import copy
        lc = copy.deepcopy(cases[0])
        a, f = lc.attn, lc.ffn
        n = 32
        a.n_seq, a.seq_len = 1, n
        a.x, a.mask = a.x[:n], a.mask[:n]
        f.x, f.mask, f.T = f.x[:n], f.mask[:n], n
        return [lc], ("per step: the first 32 tokens of sequence 0 (causal, so their outputs "
                      "equal the full problem's), fp64 definition form")

    @staticmethod
    def reference_step(samples):
        import oracle
        for lc in samples:
            oracle.attention.layer_masked(lc)
        return sum(lc.attn.T for lc in samples)


class RouterDevice:
    """Device state of the router workload: x of each call, W_r1, W_r2 and
    the packed mask words each call writes."""

    def __init__(self, wl, cases, dev, stream):
        import torch
        import token_level_dynamic_b200 as w
        from synth.torch_io import to_dev
        self.w, self.stream, self.cases = w, stream, cases
        base = cases[0]
        self.W1 = to_dev(base.w_r1, "bf16", dev)
        self.W2 = to_dev(base.w_r2, "bf16", dev)
        self.xs = [to_dev(c.x, "bf16", dev) for c in cases]
        self.ms = [torch.empty((c.T, (c.G + 31) // 32), dtype=torch.int32, device=dev)
                   for c in cases]
        self.ncalls = len(cases)
        self.xh = [x.cpu().pin_memory() for x in self.xs]
        self.mh = [torch.empty(m.shape, dtype=m.dtype).pin_memory() for m in self.ms]
        self.h2d_bytes = int(sum(x.numel() * 2 for x in self.xh))
        self.d2h_bytes = int(sum(m.numel() * 4 for m in self.mh))
        self.ws = torch.empty(0, dtype=torch.uint8, device=dev)

    def call(self, i, all_kept=False):
        # all_kept has no meaning for the router (it produces the masks)
        self.w.wide_route(self.xs[i], self.W1, self.W2, None, self.w.WIDE_ACT_RELU,
                          mask_words=self.ms[i], stream=self.stream)

    def e2e_call(self, i):
        self.xs[i].copy_(self.xh[i], non_blocking=True)
        self.call(i)
        self.mh[i].copy_(self.ms[i], non_blocking=True)

    def dense_torch(self, i):
        """torch/cuBLAS: bf16 logits, then a dense bool [T][G] decision tensor."""
        import torch.nn.functional as F
        lg = F.linear(F.relu(F.linear(self.xs[i], self.W1)), self.W2)
        self.dense_keep = lg > 0


class Router8B:
    name = "router_8b"
    desc = ("router_8b: bottleneck router of the Llama-3.1-8B-shaped FFN (hidden 4096 -> "
            "bottleneck 128, ReLU -> 112 group logits, execute iff > 0), random bf16 weights "
            "N(0, 0.02), x ~ N(0,1); one step = 8192 tokens (the prefill layer's 4 x 2048) "
            "plus a 16-token decode batch, packed mask words out")
    bound = "hbm"
    dominant = "router_tcgen05"
    device = RouterDevice

    def make_cases(self):
        import synth
        out = []
        for T in (8192, 16):
            c = synth.router_case(T, 4096, 128, 112, seed=0)
            c.name = f"router_8b_t{T}"
            out.append(c)
        return out

    @staticmethod
    def units(case):
        """Algorithmic bytes per call: x, W_r1 and W_r2 read once, the mask
        words written once."""
        b = (case.T * case.H * 2 + case.R * case.H * 2 + case.G * case.R * 2
             + case.T * ((case.G + 31) // 32) * 4)
        kernel = "router_small_gemv" if case.T <= 32 else "router_tcgen05"
        return {kernel: b, "total": b}

    def reference_sample(self, cases):
        out = []
        for c in cases:
            s = type(c)(**{**c.__dict__})
            s.x, s.T = c.x[:64], min(64, c.T)
            out.append(s)
        return out, "per step: the first 64 tokens of the 8192-token call and 16 of the decode call"

    @staticmethod
    def reference_step(samples):
        import oracle
        for c in samples:
            oracle.router.route_mask(c.x, c.w_r1, c.w_r2, c.b_r2, c.act)
        return sum(c.T for c in samples)


WORKLOADS = {w.name: w for w in (DecodeFFN3B(), PrefillFFN8B(), DecodeLayer8B(),
                                 PrefillLayer8B(), Router8B())}


# ------------------------------------------------------------ CPU oracle

def cpu_oracle_baseline(wl, samples, seconds: float, threads=None):
    """Times the oracle, repeating the sample until `seconds` have passed.
    `threads` caps the OpenMP and BLAS thread pools the oracle runs on
    (None: every host thread).  Returns (tokens/s, threads used, reps, s)."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=threads):
        used = _host_cores()
        tokens, t0, reps = 0, time.perf_counter(), 0
        while True:
            tokens += wl.reference_step(samples)
            reps += 1
            el = time.perf_counter() - t0
            if el >= seconds:
                break
    return tokens / el, used, reps, el


def _host_cores():
    """OpenMP threads the oracle's C loops run on (BLAS uses as many)."""
    from oracle import _clib
    return int(_clib.lib().oracle_num_threads())


def cpu_baseline_record(wl, cases, seconds: float):
    """The oracle on every host thread and on one, same sample."""
    samples, what = wl.reference_sample(cases)
    v, cores, reps, el = cpu_oracle_baseline(wl, samples, seconds)
    v1, _, reps1, el1 = cpu_oracle_baseline(wl, samples, seconds, threads=1)
    return {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{what}; repeated {reps}x over {el:.1f} s (fp64 oracle)",
            "one_core": {"value": v1, "unit": "tokens/s", "cores": 1,
                         "sample": f"the same; repeated {reps1}x over {el1:.1f} s"}}


def max_over_ranks(x: float, device) -> float:
    """The largest x over all ranks (the slowest rank's time); x itself
    when no process group is up."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, tokens_per_step: int, steps: int, total_ms: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_step * steps / (total_ms / 1e3)


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    samples, what = wl.reference_sample(wl.make_cases())
    for _ in range(args.warmup):
        wl.reference_step(samples)
    t0 = time.perf_counter()
    tok = 0
    for _ in range(args.steps):
        tok += wl.reference_step(samples)
    el = time.perf_counter() - t0
    v = tok / el
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl.desc, "parallelism": "host cores"},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": _host_cores(), "kind": "oracle",
                         "sample": what},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------- ours

EXTRA_WORKLOADS = ("prefill_layer_8b", "decode_layer_8b")


def run_ours(args, wl):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(dev)

    line = measure(args, wl, dev, world, rank, args.steps,
                   cpu_leg=rank == 0 and world == 1 and not args.no_cpu_baseline)
    # The default run also times the two whole-layer workloads (prefill at
    # keep 0.5, decode), one GPU only, without a CPU leg; each entry carries
    # the same fields as the main line.
    extra = {}
    if world == 1 and args.workload == "decode_ffn_3b" and not args.no_extra_workloads:
        for name in EXTRA_WORKLOADS:
            torch.cuda.empty_cache()
            ewl = PrefillLayer8B(0.5) if name == "prefill_layer_8b" else WORKLOADS[name]
            e = measure(args, ewl, dev, world, rank, min(args.steps, 50), cpu_leg=False)
            for k in ("n_gpus", "warmup", "higher_is_better", "scaling", "vs_baseline", "dtype",
                      "data", "kernel_timing", "cpu_baseline"):
                e.pop(k, None)
            extra[name] = e

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    if extra:
        line["extra_workloads"] = extra
    print(json.dumps(line), flush=True)
    return 0


def measure(args, wl, dev, world, rank, steps, cpu_leg):
    """Times `steps` steps of workload `wl` on `dev` (after args.warmup
    untimed ones) and returns the bench line's fields as a dict."""
    import numpy as np
    import torch
    import torch.distributed as dist
    import token_level_dynamic_b200 as w

    cases = wl.make_cases()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_sink = torch.empty((), dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream(dev)
    D = wl.device(wl, cases, dev, stream)
    units = [wl.units(c) for c in cases]
    ncalls = D.ncalls
    tokens_per_step = sum(c.T for c in cases)
    call = D.call

    def timed_step(fn):
        evs = []
        for i in range(ncalls):
            # flush L2: write a buffer larger than L2, then read it back so
            # the lines left behind are clean (a timed kernel should not pay
            # for writing back the flush's own dirty lines)
            flush.zero_()
            flush_sink.copy_(flush.view(torch.int64).sum())
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn(i)
            e1.record(stream)
            evs.append((e0, e1))
        return evs

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def ms_of(evs_list):
        return np.array([[a.elapsed_time(b) for a, b in evs] for evs in evs_list])

    w.wide_clear_device_status(stream)
    for _ in range(args.warmup):
        timed_step(call)
    torch.cuda.synchronize(dev)
    if w.wide_get_device_status(stream) != 0:
        raise RuntimeError("device status set during warm-up")

    # ---- timed region (no per-launch events inside the calls)
    n0 = w.wide_launch_count()
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        barrier()
        all_evs = [timed_step(call) for _ in range(steps)]
        barrier()
    launches = w.wide_launch_count() - n0
    if w.wide_get_device_status(stream) != 0:
        raise RuntimeError("device status set during the timed steps")
    per_call = ms_of(all_evs)                       # [K][ncalls] ms

    # ---- kernel pass: the same K steps again, with the library's begin/end
    # events around every launch (they add a few us per call, so the timed
    # region above runs without them)
    w.wide_profile_start(65536)
    barrier()
    for _ in range(steps):
        timed_step(call)
    barrier()
    w.wide_profile_stop()
    recs = w.wide_profile_read()
    total_ms = max_over_ranks(float(per_call.sum()), dev)
    step_ms = total_ms / steps
    value = job_tokens_per_s(world, tokens_per_step, steps, total_ms)

    # ---- per-kernel figures from the library's launch events
    peaks = _peaks()
    kern = {}
    for name, t in recs:
        kern.setdefault(name, []).append(t)
    kernels = {}
    for name, ts in kern.items():
        t_step = sum(ts) / steps
        entry = {"launches": len(ts), "avg_us": 1e3 * statistics.mean(ts),
                 "us_per_step": 1e3 * t_step}
        if any(name in u for u in units):
            u_step = sum(u.get(name, 0) for u in units)
            if wl.bound == "hbm":
                a = u_step / (t_step / 1e3) / 1e9
                entry.update({"algorithmic_bytes_per_step": u_step, "achieved_gbs": a,
                              "frac_of_hbm": a / peaks["hbm_gbs"]})
            else:
                a = u_step / (t_step / 1e3) / 1e12
                entry.update({"kept_flops_per_step": u_step, "achieved_tflops": a,
                              "frac_of_bf16_peak": a / peaks["bf16_tflops"],
                              "frac_of_bf16_sustained": a / peaks["bf16_tflops_sustained"]})
        kernels[name] = entry
    tot_k = sum(k["us_per_step"] for k in kernels.values())
    for k in kernels.values():
        k["share_of_library_time"] = k["us_per_step"] / tot_k if tot_k else None

    dominant = wl.dominant or max(
        (k for k in kernels if any(k in u for u in units)),
        key=lambda k: kernels[k]["us_per_step"], default=None)
    dk = kernels.get(dominant, {})
    traffic = _traffic_record(dominant, wl.name)
    if wl.bound == "hbm":
        roofline = {"kernel": dominant, "bound": "hbm", "achieved": dk.get("achieved_gbs"),
                    "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": dk.get("frac_of_hbm"),
                    "peak_source": f"{peaks['source']} hbm_gbs (MEASURED_PEAKS.json)"}
    else:
        roofline = {"kernel": dominant, "bound": "tensor", "achieved": dk.get("achieved_tflops"),
                    "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": dk.get("frac_of_bf16_peak"),
                    "frac_of_sustained": dk.get("frac_of_bf16_sustained"),
                    "peak_source": f"{peaks['source']} bf16_tflops burst (MEASURED_PEAKS.json)"}
    roofline["traffic"] = traffic["dram_bytes_per_step"] if traffic else None
    roofline["traffic_unit"] = "DRAM bytes per step of the dominant kernel (ncu)"

    per_call_out = {}
    for i, c in enumerate(cases):
        if not hasattr(c, "mask"):
            t = float(per_call[:, i].mean())
            d = {"tokens": c.T, "us_per_call": 1e3 * t, "tokens_per_s": c.T / (t / 1e3)}
            if wl.bound == "hbm":
                d.update({"algorithmic_bytes": units[i]["total"],
                          "achieved_gbs": units[i]["total"] / (t / 1e3) / 1e9,
                          "frac_of_hbm": units[i]["total"] / (t / 1e3) / 1e9 / peaks["hbm_gbs"]})
            else:
                d.update({"kept_flops": units[i]["total"],
                          "achieved_tflops_whole_call": units[i]["total"] / (t / 1e3) / 1e12,
                          "frac_of_bf16_peak_whole_call":
                              units[i]["total"] / (t / 1e3) / 1e12 / peaks["bf16_tflops"],
                          "kept_fraction_of_dense": units[i]["total"] / units[i]["dense_flops"]})
            per_call_out[getattr(c, "name", wl.name)] = d
            continue
        t = float(per_call[:, i].mean())
        d = {"tokens": c.T, "us_per_call": 1e3 * t, "tokens_per_s": c.T / (t / 1e3)}
        if wl.bound == "hbm":
            d.update({"union_groups": units[i]["union_groups"],
                      "algorithmic_bytes": units[i]["total"],
                      "achieved_gbs": units[i]["total"] / (t / 1e3) / 1e9})
            d["frac_of_hbm"] = d["achieved_gbs"] / peaks["hbm_gbs"]
        else:
            d.update({"kept_flops": units[i]["total"],
                      "achieved_tflops_whole_call": units[i]["total"] / (t / 1e3) / 1e12,
                      "kept_fraction_of_dense": units[i]["total"] / units[i]["dense_flops"]})
        per_call_out[c.name] = d

    # ---- dense baselines: torch/cuBLAS bf16 and our kernels with every group kept
    dense = {}
    nd = max(3, min(steps, 20))
    for name, fn in (("torch_cublas_bf16", D.dense_torch),
                     ("ours_all_groups_kept", lambda i: D.call(i, all_kept=True))):
        for _ in range(3):
            timed_step(fn)
        evs = [timed_step(fn) for _ in range(nd)]
        torch.cuda.synchronize(dev)
        pc = ms_of(evs)
        dense[name] = {"ms_per_step": float(pc.sum(axis=1).mean()),
                       "tokens_per_s": tokens_per_step / (float(pc.sum(axis=1).mean()) / 1e3)}
    dense["masked_speedup_vs_torch_dense"] = dense["torch_cublas_bf16"]["ms_per_step"] / step_ms
    dense["masked_speedup_vs_ours_all_kept"] = dense["ours_all_groups_kept"]["ms_per_step"] / step_ms
    if hasattr(D, "naive_gather_scatter"):
        # the pages' naive comparator: time, and peak device memory it adds
        # per call next to ours (our only extra memory is the workspace)
        ng = D.naive_gather_scatter
        timed_step(ng)
        torch.cuda.synchronize(dev)
        peak = 0
        for i in range(ncalls):
            base_mem = torch.cuda.memory_allocated(dev)
            torch.cuda.reset_peak_memory_stats(dev)
            ng(i)
            torch.cuda.synchronize(dev)
            peak = max(peak, torch.cuda.max_memory_allocated(dev) - base_mem)
        evs = [timed_step(ng) for _ in range(3)]
        torch.cuda.synchronize(dev)
        pc = ms_of(evs)
        ng_ms = float(pc.sum(axis=1).mean())
        dense["naive_gather_scatter_torch"] = {
            "ms_per_step": ng_ms, "tokens_per_s": tokens_per_step / (ng_ms / 1e3),
            "peak_extra_device_bytes_per_call": int(peak),
            "ours_workspace_bytes": int(D.ws.numel()),
            "masked_speedup_vs_naive": ng_ms / step_ms}

    # ---- end to end through the public API with host buffers
    for _ in range(3):
        timed_step(D.e2e_call)
    barrier()
    e_evs = [timed_step(D.e2e_call) for _ in range(steps)]
    barrier()
    e_ms = max_over_ranks(float(ms_of(e_evs).sum()), dev)
    e2e = {"value": job_tokens_per_s(world, tokens_per_step, steps, e_ms), "unit": "tokens/s",
           "h2d_bytes_per_step": D.h2d_bytes, "d2h_bytes_per_step": D.d2h_bytes,
           "ms_per_step": e_ms / steps}

    cpu = cpu_baseline_record(wl, cases, args.cpu_seconds) if cpu_leg else None

    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; shapes of the pages' Llama workloads)",
        "config": {"workload": wl.desc, "global_batch": world * tokens_per_step,
                   "l2": "flushed before every timed call (256 MiB write, then read back)",
                   "parallelism": f"replicas x{world} (no collective on the data path)"},
        "roofline": roofline, "kernels": kernels,
        "kernel_timing": ("library begin/end CUDA events on the launch stream around every "
                          "launch, over a second pass of the K timed steps (same inputs, L2 "
                          "flushed the same way); the timed pass runs without them"),
        "per_call": per_call_out,
        "dense_baseline": dense, "e2e": e2e, "cpu_baseline": cpu,
        "gpu_launches": int(launches), "clocks": clk.summary(),
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="decode_ffn_3b")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-workloads", action="store_true",
                    help="time only --workload (the default run also times "
                         "prefill_layer_8b at keep 0.5 and decode_layer_8b)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--keep", type=float, default=0.5,
                    help="keep rate of the prefill_layer_8b masks (0.25, 0.5, 0.75, 1.0)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = WORKLOADS[args.workload]
    if args.workload == "prefill_layer_8b":
        wl = PrefillLayer8B(args.keep)
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_ours(args, wl)


if __name__ == "__main__":
    sys.exit(main())
