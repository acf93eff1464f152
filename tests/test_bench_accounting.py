"""The benchmark's work accounting, pinned on CPU.

The roofline fractions bench.py reports divide these counts by measured
times, so they are checked here against independent statements of the same
quantities: the oracle's FLOP count of the iteration, and the per-element
byte counts of each pass written out by hand for the GPT-2-small set.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from oracle import muon as oracle  # noqa: E402

SHAPES = bench.gpt2_shapes()


def test_the_set_is_gpt2_small_hidden_matrices():
    assert len(SHAPES) == 72
    assert sorted(set(SHAPES)) == [(768, 768), (768, 3072), (3072, 768)]
    assert SHAPES.count((768, 768)) == 48


def test_step_flops_match_the_oracle_count():
    assert bench.nominal_flops(SHAPES) == sum(oracle.ns_flops(r, c) for r, c in SHAPES)
    # worked by hand: 5 (4 + 2) 768^3 = 13.59e9; 5 (4 * 4 + 2) 768^3 = 40.77e9
    assert oracle.ns_flops(768, 768) == pytest.approx(13.59e9, rel=1e-3)
    assert oracle.ns_flops(768, 3072) == pytest.approx(40.77e9, rel=1e-3)


def test_per_launch_work():
    w = bench.stage_work(SHAPES)
    elems = 48 * 768 * 768 + 24 * 768 * 3072          # 84,934,656
    gram = 48 * 2 * 768 ** 3 + 24 * 2 * 768 ** 2 * 3072  # X X^T per launch
    assert w["gram"] == ("tensor", gram)
    assert w["bx"] == ("tensor", gram)                 # B X has the X X^T count
    assert w["poly"] == ("tensor", 72 * 2 * 768 ** 3)  # A A, every A is 768 x 768
    assert w["prep"] == ("hbm", 13 * elems)
    assert w["out"] == ("hbm", 11 * elems)
    # fused last BX + apply: pair 3 B + W 8 B per element, B (72 x 768^2 bf16)
    assert w["bx_apply"] == ("hbm", 11 * elems + 72 * 2 * 768 ** 2)
    assert w["bx_apply"][1] == pytest.approx(1019.3e6, rel=1e-4)
    # a step is 5 gram + 5 poly + 5 BX-like launches: the nominal step FLOPs
    assert 5 * (w["gram"][1] + w["poly"][1] + w["bx"][1]) == bench.nominal_flops(SHAPES)


def test_reference_arm_line(capsys, monkeypatch):
    """`bench.py --impl reference` on rank 0: one JSON line with the arm's own
    cpu_baseline and an e2e that moves no bytes (the oracle runs on the host)."""
    import json
    monkeypatch.delenv("RANK", raising=False)

    class A:
        steps, warmup, gpus = 1, 1, 1

    bench.run_reference(A())
    out = capsys.readouterr().out.strip().splitlines()
    assert len(out) == 1
    line = json.loads(out[0])
    assert line["impl"] == "reference"
    assert (line["metric"], line["unit"]) == (bench.METRIC, bench.UNIT)
    assert line["higher_is_better"] is True and line["value"] > 0
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["workload"] == bench.WORKLOAD


def test_executed_flops_of_the_pair_tiles():
    """Executed work counts whole 256 x 256 pair tiles: for m = 768 (3 x 3
    tiles) the symmetric products run 6 of 9 tiles, B X all 9, so a step
    executes (2/3 * 2 m^2 n + 2/3 * 2 m^3 + 2 m^2 n); worked by hand."""
    m, n = 768, 3072
    want = 5 * (2 / 3 * 2 * m * m * n + 2 / 3 * 2 * m ** 3 + 2 * m * m * n)
    assert bench.executed_flops([(m, n)]) == pytest.approx(want, rel=1e-12)
    assert bench.executed_flops([(n, m)]) == bench.executed_flops([(m, n)])
    # one ragged 200 x 328 matrix: 1 pair tile row (padded to 256), 2 tile columns,
    # K padded to 64: 328 -> 384, 200 -> 256
    t = 2 * 256 * 256
    assert bench.executed_flops([(200, 328)], steps=1) == t * (1 * 384 + 1 * 256 + 2 * 256)
    # for large m the symmetric share tends to one half of the nominal work
    big = bench.executed_flops([(4096, 4096)], steps=1)
    assert big / bench.nominal_flops([(4096, 4096)], steps=1) == pytest.approx((136 / 256 * 4 + 2) / 6)
