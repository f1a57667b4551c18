"""CPU checks of bench.py's reference arm: the CPU oracle timed on a bounded sample.

The arm prints exactly one JSON line on rank 0 with the benchmark's keys (its own
config, the oracle as the CPU baseline, an e2e entry with no host-device copies) and
prints nothing on the other ranks.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CMD = [sys.executable, "bench.py", "--impl", "reference", "--workload", "prefill_t4096_k256",
       "--steps", "1", "--warmup", "1"]
KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "impl")


def _run(env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run(CMD, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_line_on_rank_0():
    r = _run({})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in KEYS:
        assert k in d, k
    assert d["impl"] == "reference"
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["config"]["workload"] == "prefill_t4096_k256"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_is_silent_on_other_ranks():
    r = _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_stage_report_rooflines():
    """bench.stage_report: each stage against the resource that bounds it -- the indexer's
    flops against the sustained bf16 peak, the Top-K bytes of the path that ran (fused rows
    counted by the library, materialised otherwise, both in a mixed batch) against HBM, the
    attention's algorithmic bytes against the measured L2 gather ceiling -- and an 'hbm'
    fraction above 1 is refused."""
    import pytest

    sys.path.insert(0, ROOT)
    import bench
    import dsa_synth as S

    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    gather = {"l2": {"gbs": 20000.0}}
    w = S.workload("prefill_t32768_k2048")
    a = bench.algorithmic(w)
    st = bench.stage_report(w, [1.0, 1.0, 8.0], [3, 3, 1], peaks, gather, fused_rows=w.total_q)
    assert st[0]["achieved"] == pytest.approx(a["idx_flops"] / 1e-3 / 1e12)
    assert st[0]["frac"] == pytest.approx(st[0]["achieved"] / 1400.0)
    # fused: the bytes the fused selection moves are the primary figure, the scope table's
    # definition is the equivalent rate beside it
    assert st[1]["achieved"] == pytest.approx(a["topk_bytes_fused_moved"] / 1e-3 / 1e9)
    assert st[1]["scope_equivalent_gbs"] == pytest.approx(a["topk_bytes"] / 1e-3 / 1e9)
    assert a["topk_bytes_fused_moved"] < a["topk_bytes"]
    assert st[2]["bound"] == "l2" and st[2]["peak"] == 20000.0
    assert st[2]["frac"] == pytest.approx(a["attn_bytes"] / 8e-3 / 1e9 / 20000.0)
    # materialised: the scope table's bytes are what the path moves
    st = bench.stage_report(w, [1.0, 1.0, 8.0], [8, 8, 1], peaks, gather, fused_rows=0)
    assert st[1]["achieved"] == pytest.approx(a["topk_bytes"] / 1e-3 / 1e9)
    assert st[1]["scope_equivalent_gbs"] is None
    # an 'hbm' rate above the copy peak is not an HBM rate
    with pytest.raises(AssertionError):
        bench.stage_report(w, [1.0, 0.1, 8.0], [8, 8, 1], peaks, gather, fused_rows=0)
    # mixed batch: the long query groups fused, the decode rows materialised
    m = S.workload("mixed_serving", scale_down=64)
    long_rows = sum(q for q in m.q_lens if q >= 128)
    st = bench.stage_report(m, [1.0, 1.0, 8.0], [4, 4, 1], peaks, gather, fused_rows=long_rows)
    lw = bench._sub_workload(m, [b for b, q in enumerate(m.q_lens) if q >= 128])
    sw = bench._sub_workload(m, [b for b, q in enumerate(m.q_lens) if q < 128])
    moved = bench.algorithmic(lw)["topk_bytes_fused_moved"] + bench.algorithmic(sw)["topk_bytes"]
    assert st[1]["achieved"] == pytest.approx(moved / 1e-3 / 1e9)


def test_committed_attention_traffic_and_reduced_cases():
    """Each committed attention capture parses to a full-launch DRAM traffic keyed to the
    current kernel source; a reduced case (--seq-stride) never borrows the full launch's
    figure, and its workload keeps every N-th sequence."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    import dsa_synth as S
    for name in ("prefill_t32768_k2048", "prefill_t131072_needles", "mixed_serving"):
        t = b.attn_traffic(name)
        assert t is not None and t > 1e9, name
        assert b.attn_traffic(name, 8) is None
    w = S.workload("mixed_serving")
    sw = b._sub_workload(w, [i for i in range(w.batch) if i % 8 == 0])
    assert sw.batch == 33 and sw.q_lens[0] == 8192 and all(q == 1 for q in sw.q_lens[1:])
    assert abs(b.algorithmic(w)["attn_bytes"] / b.algorithmic(sw)["attn_bytes"] - 8.0) < 0.05
