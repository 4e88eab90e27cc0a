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
