"""bench.py's host side on CPU: the reference arm's JSON line, the CPU
leg, the clock record, and the algorithmic units (bytes or kept FLOPs) that
the workloads divide by, against independent counts (no GPU needed)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("workload", ["decode_ffn_3b", "router_8b"])
def test_reference_arm_line(workload):
    """Rank 0 of the reference arm times the oracle on the host cores and
    prints one JSON line with the contract's keys."""
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", workload, "--steps", "1", "--warmup", "3"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["steps"] == 1 and d["warmup"] == 3
    assert d["config"]["workload"].startswith(workload)
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_cpu_baseline_on_all_threads_and_on_one():
    """The CPU leg times the oracle twice on the same sample: with every
    host thread (the decode sample is one oracle call of as many tokens as
    threads, so the token loop has work for each) and capped at one."""
    sys.path.insert(0, ROOT)
    import bench
    wl = bench.WORKLOADS["decode_ffn_3b"]
    cases = wl.make_cases()
    samples, _ = wl.reference_sample(cases)
    assert len(samples) == 1 and samples[0].T == min(32, bench._host_cores())
    rec = bench.cpu_baseline_record(wl, cases, 0.01)
    assert rec["kind"] == "oracle" and rec["cores"] == bench._host_cores() and rec["value"] > 0
    assert rec["one_core"]["cores"] == 1 and rec["one_core"]["value"] > 0
    # the cap is lifted again afterwards
    assert bench._host_cores() == rec["cores"]


def test_router_units():
    """Algorithmic bytes of one router call: x, W_r1 and W_r2 read once,
    the packed mask words written once; the kernel name follows the size
    split of the library (cluster kernel up to 32 tokens, tcgen05 above)."""
    sys.path.insert(0, ROOT)
    import bench
    wl = bench.WORKLOADS["router_8b"]
    cases = wl.make_cases()
    assert [c.T for c in cases] == [8192, 16]
    u_big, u_small = (wl.units(c) for c in cases)
    assert u_big == {"router_tcgen05": 8192 * 4096 * 2 + 128 * 4096 * 2 + 112 * 128 * 2
                     + 8192 * 4 * 4, "total": u_big["total"]}
    assert u_small == {"router_small_gemv": 16 * 4096 * 2 + 128 * 4096 * 2 + 112 * 128 * 2
                       + 16 * 4 * 4, "total": u_small["total"]}
    assert u_big["total"] == u_big["router_tcgen05"]


def test_clock_sampler_against_a_fake_nvml(monkeypatch):
    """The clock record: median SM clock, max clock and the throttle reasons
    seen while sampling, read through NVML (a fake one here; read-only)."""
    import time
    import types
    sys.path.insert(0, ROOT)
    import bench
    calls = {"n": 0}
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=1,
        nvmlClocksEventReasonSwPowerCap=0x4, nvmlClocksEventReasonHwSlowdown=0x8,
        nvmlClocksEventReasonSwThermalSlowdown=0x20,
        nvmlClocksEventReasonHwThermalSlowdown=0x40,
        nvmlClocksEventReasonHwPowerBrakeSlowdown=0x80,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByIndex=lambda i: ("dev", i),
        nvmlDeviceGetHandleByUUID=lambda u: ("dev", u),
        nvmlDeviceGetMaxClockInfo=lambda h, k: 1965,
    )

    def clock(h, k):
        calls["n"] += 1
        return (1965, 1800, 1965)[calls["n"] % 3]
    fake.nvmlDeviceGetClockInfo = clock
    fake.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x4 if calls["n"] % 2 else 0
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES", raising=False)
    with bench.ClockSampler(0, period=0.001) as c:
        time.sleep(0.05)
    s = c.summary()
    assert s["source"] == "nvml" and s["sm_max_mhz"] == 1965
    assert s["samples"] >= 5 and s["sm_mhz"] in (1800, 1965)
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_sampler_without_nvml(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setitem(sys.modules, "pynvml", None)      # import fails
    with bench.ClockSampler(0) as c:
        pass
    assert c.summary()["source"] == "unavailable"


def test_decode_bytes_follow_the_per_launch_kernel_choice():
    """The decode FFN's algorithmic bytes are booked on the kernel each
    launch runs: the channel-split kernel up to 8 tokens, the tensor-core
    kernel for 32-token launches, and a 40-token batch as one 32-token
    tensor-core launch plus an 8-token split launch, each streaming the
    union of its own tokens' groups."""
    sys.path.insert(0, ROOT)
    import bench
    import synth
    H, I, gs = 3072, 8192, 128
    for T, names in ((1, {"decode_ffn_split_gemv"}), (8, {"decode_ffn_split_gemv"}),
                     (32, {"decode_ffn_tcgen05"}),
                     (40, {"decode_ffn_tcgen05", "decode_ffn_split_gemv"})):
        c = synth.ffn_case(T, H, I, gs, seed=T, keep=0.5)
        b = bench._ffn_decode_bytes(c)
        kern = set(b) - {"total", "union_groups"}
        assert kern == names, (T, kern)
        assert b["total"] == sum(b[k] for k in kern)
        io = T * H * 2 + c.mask_words.nbytes + T * H * 2
        w = 0
        for t0, n in ((0, 32), (32, 8)) if T == 40 else ((0, T),):
            u = int(c.mask[t0:t0 + n].any(axis=0).sum())
            w += 3 * u * gs * H * 2
        assert b["total"] == w + io


def _prefill_flops_by_loops(lc, all_kept=False):
    """Multiply-adds of the masked prefill layer counted one (token, group,
    head) at a time, 2 FLOPs each: Q and o_proj per kept (token, head
    group) pair and query head, attention over the query's causal keys
    (QK^T and PV), K and V for every token, gate/up and down per kept
    (token, channel group) pair."""
    a, f = lc.attn, lc.ffn
    rep = a.n_q // a.n_kv
    n = {"q": 0, "kv": 0, "att": 0, "oproj": 0, "gateup": 0, "down": 0}
    for t in range(a.T):
        pos = t % a.seq_len + a.cache_len
        n["kv"] += 2 * (2 * a.n_kv * a.hd) * a.H
        for g in range(a.n_kv):
            if all_kept or a.mask[t, g]:
                for _ in range(rep):
                    n["q"] += 2 * a.hd * a.H
                    n["att"] += 2 * a.hd * (pos + 1) + 2 * (pos + 1) * a.hd
                    n["oproj"] += 2 * a.hd * a.H
        for g in range(f.I // f.gs):
            if all_kept or f.mask[t, g]:
                n["gateup"] += 2 * (2 * f.gs) * a.H
                n["down"] += 2 * a.H * f.gs
    return n


def test_prefill_layer_kept_flops():
    """The kept FLOPs that the prefill-layer line divides by, against a
    per-pair count on a small layer; the dense figure is the same count
    with every group kept."""
    sys.path.insert(0, ROOT)
    import bench
    import synth
    lc = synth.small_layer("prefill", seed=3, n_seq=2, seq_len=37, H=256, n_q=8, n_kv=2, hd=128,
                           I=512, gs=64, keep_a=0.5, keep_f=0.5)
    u = bench.WORKLOADS["prefill_layer_8b"].units(lc)
    n = _prefill_flops_by_loops(lc)
    assert (u["prefill_q_rope_tcgen05"], u["prefill_kv_rope_tcgen05"],
            u["prefill_attention_tcgen05"], u["prefill_oproj_tcgen05"],
            u["prefill_gateup_tcgen05"], u["prefill_down_tcgen05"]) == \
        (n["q"], n["kv"], n["att"], n["oproj"], n["gateup"], n["down"])
    assert u["total"] == sum(n.values())
    assert u["dense_flops"] == sum(_prefill_flops_by_loops(lc, all_kept=True).values())
    assert 0 < u["total"] < u["dense_flops"]


def test_prefill_ffn_kept_flops():
    """The prefill FFN line's kept FLOPs equal the per-pair count of the
    layer test above (its FFN part) on a small masked FFN."""
    sys.path.insert(0, ROOT)
    import bench
    import synth
    c = synth.ffn_case(T=29, H=256, I=512, gs=64, seed=5, keep=0.5)
    u = bench.WORKLOADS["prefill_ffn_8b"].units(c)
    gateup = down = 0
    for t in range(c.T):
        for g in range(c.I // c.gs):
            if c.mask[t, g]:
                gateup += 2 * (2 * c.gs) * c.H
                down += 2 * c.H * c.gs
    assert (u["prefill_gateup_tcgen05"], u["prefill_down_tcgen05"]) == (gateup, down)
    assert u["total"] == gateup + down and u["pairs"] == int(c.mask.sum())
    assert u["dense_flops"] == 3 * 2 * c.T * c.H * c.I
