"""The reference arm of bench.py (the fp64 oracle timed on the host cores)
prints one JSON line whose metric, unit and direction are the GPU arm's, so
that the two lines compare.  The oracle sample is replaced by a stub here;
its own arithmetic is pinned by the oracle tests."""
import json
import types

import bench


def _run(monkeypatch, capsys, rank):
    calls = []

    def fake_inputs(heads=bench.HEADS):
        calls.append(("inputs", heads))
        return heads

    def fake_sample(inputs):
        calls.append(("sample", inputs))
        return bench.ATTN_FLOPS * inputs // bench.HEADS, 2.0, 7

    monkeypatch.setattr(bench, "oracle_inputs", fake_inputs)
    monkeypatch.setattr(bench, "oracle_sample", fake_sample)
    args = types.SimpleNamespace(gpus=1, steps=2, warmup=3)
    bench.run_reference(args, rank)
    return calls, capsys.readouterr().out.strip().splitlines()


def test_reference_line_matches_the_gpu_arm(monkeypatch, capsys):
    calls, lines = _run(monkeypatch, capsys, rank=0)
    # inputs drawn once, then warm-up + timed samples of 2 heads; one line
    assert calls == [("inputs", 2)] + [("sample", 2)] * 5 and len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["config"]["workload"] == bench.WORKLOAD
    want = bench.ATTN_FLOPS * 2 // bench.HEADS / 2.0 / 1e12
    assert abs(d["value"] - want) <= 1e-12 * want
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] == 7
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert (d["steps"], d["warmup"]) == (2, 3)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    calls, lines = _run(monkeypatch, capsys, rank=1)
    assert calls == [] and lines == []
