"""Host-side accounting of bench.py on small shapes: the causal pair count
behind the effective FLOPs (brute force), the backward's executed (64-row
tile, 128-key block) pairs behind its roofline (against the pairs that
contribute, and the kernel's rule one pair at a time), the static
block-sparse pattern, and the traffic records keyed by kernel source."""
import os

import numpy as np
import pytest

import bench
import synth


@pytest.mark.parametrize("Lq,Lkv", [(1, 1), (5, 5), (7, 19), (130, 300), (256, 256)])
def test_causal_pairs_brute_force(Lq, Lkv):
    off = Lkv - Lq
    n = sum(1 for i in range(Lq) for j in range(Lkv) if j <= i + off)
    assert bench.causal_pairs(Lq, Lkv) == n
    w = synth.CONFIGS["prefill_32k"].replace(B=2, Hq=3, Hkv=1, Lq=Lq, Lkv=Lkv, d=64)
    assert bench.effective_flops(w) == 4.0 * 2 * 3 * 64 * n
    wn = w.replace(causal=False)
    assert bench.effective_flops(wn) == 4.0 * 2 * 3 * 64 * Lq * Lkv


def _effective_pairs(w, mask):
    """(64-row tile, 128-key block) pairs holding at least one causally
    visible (row, key) whose forward tile was computed (mask 0): the pairs
    whose product contributes anything."""
    n = 0
    for b in range(w.B):
        for h in range(w.Hq):
            for t in range(-(-w.Lq // 64)):
                for kb in range(-(-w.Lkv // 128)):
                    hit = False
                    for r in range(64 * t, min(64 * t + 64, w.Lq)):
                        for c in range(128 * kb, min(128 * kb + 128, w.Lkv)):
                            if w.causal and c > r + (w.Lkv - w.Lq):
                                continue
                            if mask[b, h, r // w.Br, c // w.Bc] == 0:
                                hit = True
                                break
                        if hit:
                            break
                    n += hit
    return n


def _kernel_rule_pairs(w, mask):
    """The backward kernel's rule, one pair at a time: tile t reaches block
    kb causally (its last row sees key 128 kb) and the forward computed some
    Bc-key block inside [128 kb, 128 kb + 128) for t's forward tile."""
    n = 0
    off = w.Lkv - w.Lq
    nKt = mask.shape[-1]
    for b in range(w.B):
        for h in range(w.Hq):
            for t in range(-(-w.Lq // 64)):
                qf = (64 * t) // w.Br
                for kb in range(-(-w.Lkv // 128)):
                    if w.causal and 128 * kb > 64 * t + 63 + off:
                        continue
                    blocks = [kb] if w.Bc == 128 else [k for k in (2 * kb, 2 * kb + 1) if k < nKt]
                    n += any(mask[b, h, qf, k] == 0 for k in blocks)
    return n


def _forward_like_mask(w, seed):
    """A skip mask shaped like the forward's: 2 outside a tile's causal
    range, else 0 (computed) or 1 (skipped) at random, block 0 computed."""
    rng = np.random.default_rng(seed)
    nQt, nKt = -(-w.Lq // w.Br), -(-w.Lkv // w.Bc)
    m = (rng.random((w.B, w.Hq, nQt, nKt)) < 0.5).astype(np.uint8)
    m[..., 0] = 0
    off = w.Lkv - w.Lq
    for qt in range(nQt):
        last_row = min(qt * w.Br + w.Br, w.Lq) - 1
        if w.causal:
            m[:, :, qt, (last_row + off) // w.Bc + 1:] = 2
    return m


PAIR_CASES = [dict(Lq=300, Lkv=300, Br=128, Bc=128),
              dict(Lq=300, Lkv=300, Br=64, Bc=64),
              dict(Lq=200, Lkv=450, Br=128, Bc=64),
              dict(Lq=256, Lkv=256, Br=64, Bc=128),
              dict(Lq=333, Lkv=333, Br=64, Bc=128),
              dict(Lq=190, Lkv=333, Br=128, Bc=128, causal=False)]


@pytest.mark.parametrize("over", PAIR_CASES)
def test_backward_pairs_follow_the_kernel_rule(over):
    """bench.backward_pairs counts the pairs the kernel executes: never fewer
    than the pairs that contribute, the same number when the forward tile is
    the backward pair's shape (64 x 128), and the kernel's rule pair by pair."""
    w = synth.CONFIGS["prefill_32k"].replace(B=1, Hq=2, Hkv=1, **over)
    for seed in range(3):
        m = _forward_like_mask(w, seed)
        got = bench.backward_pairs(w, m)
        eff = _effective_pairs(w, m)
        assert got >= eff, (over, seed)
        if w.Br == 64 and w.Bc == 128:
            assert got == eff, (over, seed)
        assert got == _kernel_rule_pairs(w, m), (over, seed)


def test_block_sparse_pattern_properties():
    w = synth.CONFIGS["prefill_32k"].replace(Hq=2, Hkv=1, Lq=4096, Lkv=4096)
    m = bench.block_sparse_pattern(w, sink_blocks=1, band_blocks=8, random_frac=0.1, seed=0)
    nQt, nKt = 4096 // 128, 4096 // 128
    assert m.shape == (1, 2, nQt, nKt) and m.dtype == np.uint8
    assert set(np.unique(m)) <= {0, 1}
    assert np.all(m[..., 0] == 0)                       # the sink block
    for qt in range(nQt):                               # the band ending at the diagonal
        assert np.all(m[:, :, qt, max(0, qt - 7):qt + 1] == 0)
    assert np.array_equal(m, bench.block_sparse_pattern(w, seed=0))
    rest = np.ones((nQt, nKt), dtype=bool)
    rest[:, 0] = False
    for qt in range(nQt):
        rest[qt, max(0, qt - 7):qt + 1] = False
    frac = float((m[:, :, rest] == 0).mean())
    assert 0.07 < frac < 0.13                           # ~10 % of the other blocks


def test_traffic_records_follow_the_kernel_sources(tmp_path, monkeypatch):
    key = "prefill_32k"
    h = bench.kernel_source_hash(key)
    assert len(h) == 16 and h == bench.kernel_source_hash(key)
    (tmp_path / "profiles").mkdir()
    rec = tmp_path / "profiles" / "traffic.txt"
    rec.write_text(f"# comment\n{key} {h} 123456\ndecode_64k 0000000000000000 7\n")
    # the lookup reads profiles/ under the repository root; kernels under csrc
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    os.symlink(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "dynamic_block_sparse_tiled_b200"),
               tmp_path / "dynamic_block_sparse_tiled_b200")
    assert bench.profiled_traffic(key) == 123456.0
    assert bench.profiled_traffic("decode_64k") is None  # recorded for other sources
    other = h[:-1] + ("1" if h[-1] != "1" else "2")  # a record of other sources
    rec.write_text(f"{key} {other} 99\n")
    assert bench.profiled_traffic(key) is None


def test_reference_arm_json_line(monkeypatch, capsys):
    """The reference arm (the oracle on the host cores) prints one JSON line
    with the benchmark's keys, impl = reference, its own cpu_baseline and an
    e2e of the line's value with no device copies (the oracle sample and the
    input generation are stubbed: this checks the line, not the timing)."""
    import argparse
    import json

    calls = []

    def fake_sample(w, lam, budget, seed=0, inputs=None):
        calls.append((w.name, lam, budget, seed))
        return dict(value=0.05 + 0.01 * seed, unit=bench.UNIT, cores=16, kind="oracle",
                    sample=f"{seed} of 8192 query tiles", seconds=2.0 + seed)

    monkeypatch.setattr(synth, "generate", lambda w: None)
    monkeypatch.setattr(bench, "oracle_sample", fake_sample)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    args = argparse.Namespace(gpus=1, steps=2, warmup=3, cpu_budget=15.0)
    assert bench.run_reference(args) == 0
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["steps"] == 2 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["config"]["workload"] == bench.WORKLOAD
    assert abs(d["value"] - 0.055) < 1e-12                # mean over the 2 timed samples
    assert abs(d["ms_per_step"] - 2500.0) < 1e-9
    assert d["cpu_baseline"]["value"] == d["value"] and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"] == dict(value=d["value"], unit=d["unit"], h2d_bytes_per_step=0,
                            d2h_bytes_per_step=0)
    assert len(calls) == 5                                # 3 warm-up samples, then 2 timed
    assert [c[3] for c in calls[3:]] == [0, 1]            # one seed per timed step
    assert all(c[2] < calls[3][2] for c in calls[:3])     # warm-up samples are smaller


def test_clock_samples_are_selected_by_window():
    lines = [
        "2026/12/02 10:00:00.000, 1900, 1965, 700.1, Not Active, Not Active, Not Active, Not Active",
        "2026/12/02 10:00:00.050, 1700, 1965, 990.3, Not Active, Not Active, Not Active, Active",
        "2026/12/02 10:00:00.100, 1800, 1965, 900.0, Not Active, Not Active, Not Active, Active",
        "garbage line",
    ]
    clk = bench.ClockSampler(0)
    for ln in lines:
        s = bench.ClockSampler.parse(ln, 0.0)
        if s is not None:
            clk.samples.append(s)
    assert len(clk.samples) == 3
    t0 = clk.samples[0][0]
    full = clk.summary()
    assert full["sm_mhz"] == 1800 and full["sm_max_mhz"] == 1965
    assert full["reasons"] == ["sw_power_cap"] and full["samples"] == 3
    first = clk.summary([(t0 - 0.001, t0 + 0.001)])
    assert first["sm_mhz"] == 1900 and first["reasons"] == [] and first["samples"] == 1
    two = clk.summary([(t0 + 0.04, t0 + 0.06), (t0 + 0.09, t0 + 0.11)])
    assert two["sm_mhz"] == 1750 and two["samples"] == 2
    assert clk.summary([(t0 + 5, t0 + 6)])["sm_mhz"] is None


def test_interleaved_rounds_alternate_the_arm_order(monkeypatch):
    import torch
    calls = []

    def fake_time_calls(fn, steps, warmup, stream, flush_buf):
        for _ in range(warmup):
            fn()
        out = []
        for _ in range(steps):
            out.append(float(fn()))
        return out

    monkeypatch.setattr(bench, "time_calls", fake_time_calls)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)

    def arm(name, ms):
        def fn():
            calls.append(name)
            return ms
        return fn

    t = bench.time_interleaved([("a", arm("a", 2.0)), ("b", arm("b", 1.0))], rounds=4, per=2,
                               warmup=1, stream=None, flush_buf=None)
    assert calls == ["a", "b"] + ["a", "a", "b", "b", "b", "b", "a", "a"] * 2
    assert t["a"]["block_ms"] == [2.0] * 4 and t["b"]["block_ms"] == [1.0] * 4
    assert len(t["a"]["windows"]) == 4

    class Clk:
        def summary(self, windows):
            return dict(sm_mhz=1000.0 if windows is t["a"]["windows"] else 2000.0, reasons=[])

    res = {0.0: bench.arm_summary(t["a"], Clk()), 1e-3: bench.arm_summary(t["b"], Clk())}
    bench.speedups(res, 0.0)
    assert res[1e-3]["speedup_vs_lambda0"] == 2.0
    # same cycles on both arms: the clock-normalised speedup is 1
    assert res[1e-3]["speedup_clk"] == 1.0 and res[0.0]["speedup_clk"] == 1.0


def test_summary_line_legs_stay_compact():
    def arm(skip, x, **kw):
        return dict(skip_frac=skip, speedup_vs_lambda0=x, speedup_clk=x * 0.99123, frac=0.61234,
                    ms=9.1234567, **kw)
    diffuse = dict(skip_frac_structured=0.91234, skip_frac_diffuse=0.00123)
    legs = {"p32k": {0.0: arm(0.0, 1.0), 1e-3: arm(0.0, 1.0123)},
            "p32k_a12": {0.0: arm(0.0, 1.0), 1e-3: arm(0.95312, 1.62345)}}
    for k in ("p128k", "p128k_a12"):
        legs[k] = {lam: arm(0.75123, 1.45123) for lam in (0.0, 1e-4, 1e-3, 1e-2)}
    for k in ("p256k", "p256k_a12"):
        legs[k] = {lam: arm(0.51234, 1.31234, **diffuse) for lam in (0.0, 1e-3)}
    for k in ("dec", "dec_a12"):
        d = dict(ms=0.69123, gbs=6300.123, frac=0.96234, speedup_vs_lambda0=1.00123,
                 speedup_clk=1.00234, skip_frac=0.51234, v_fetch_frac=0.41234,
                 bytes_saved=1.23456e9)
        legs[k] = {0.0: d, 1e-3: d}
    legs["mla"] = {"decode_mla_64k": {"roofline": dict(bound="hbm", frac=0.39123,
                                                       tensor_frac=0.35123),
                                      str(1e-3): dict(ms=0.24981)}}
    legs["bwd"] = dict(ms=25.5123, roofline=dict(frac=0.52123, traffic=12.45e9),
                       a12=dict(speedup_vs_lambda0=7.5123))
    legs["sel"] = {"prefill_32k": dict(selector_ms=0.19234, roofline=dict(frac=0.84123))}
    legs["static"] = dict(speedup_vs_no_mask=3.2123)
    c = bench.compact_legs(legs)
    assert set(c) == set(legs)
    assert c["p256k"]["skip_s"] == 0.912 and c["p256k"]["skip_d"] == 0.00123
    assert c["p128k"]["0.001"] == [0.751, 1.45, 1.44]
    assert c["dec_a12"]["saved_gb"] == 1.23
    import json
    assert len(json.dumps(c, separators=(",", ":"))) < 1200


def test_kernel_hash_ignores_comments():
    """A traffic record stays valid across comment edits, not code edits."""
    a = "int f(int x) {  // one\n  /* two\n three */ return x + 1;\n}\n"
    b = "// header\nint f(int x) {\n\n  return x + 1;   // other\n}\n"
    c = "int f(int x) {\n  return x + 2;\n}\n"
    assert bench.code_only(a) == bench.code_only(b)
    assert bench.code_only(a) != bench.code_only(c)
