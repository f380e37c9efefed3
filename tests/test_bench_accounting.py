"""The benchmark's accounting, checked on the CPU against counts derived by hand: the set's
shapes and parameter count, the symmetry-aware Newton-Schulz FLOPs (from the three products'
shapes), the composition of the oracle's per-set time from per-shape times, and the recorded
DRAM traffic lookup, which must only answer for the kernel sources it was captured on."""
import hashlib
import json
import os

import pytest

import bench


def test_llama_set_shapes_and_parameter_count():
    shapes = bench.set_shapes()
    assert len(shapes) == 224
    per_layer = 4 * 4096 * 4096 + 2 * 4096 * 11008 + 11008 * 4096
    assert sum(r * c for r, c in shapes) == 32 * per_layer == 6_476_005_376
    assert bench.layer_counts() == {(4096, 4096): 4, (4096, 11008): 2, (11008, 4096): 1}
    cfg = bench.workload_config(shapes)
    assert cfg["workload"] == "llama7b_muon_step" and cfg["matrices"] == 224 and cfg["params"] == 6_476_005_376


def _product_flops(m, n, k, sym):
    # a product of an m x k by a k x n matrix; a symmetric output is computed as its triangle
    return (1 if sym else 2) * m * n * k


@pytest.mark.parametrize("rows,cols", [(4096, 4096), (4096, 11008), (11008, 4096), (768, 2304), (1024, 1024)])
def test_ns_flops_follow_the_three_products(rows, cols):
    r, s = min(rows, cols), max(rows, cols)
    per_iter = (_product_flops(r, r, s, True)        # A = X X^T (or X^T X): symmetric r x r over s
                + _product_flops(r, r, r, True)      # A A: symmetric r x r over r
                + _product_flops(r, s, r, False))    # B X (or X B): r x s over r
    assert bench.ns_flops_algorithmic(rows, cols) == 5 * per_iter
    assert bench.ns_flops_algorithmic(rows, cols, iters=1) == per_iter


def test_set_flops_total():
    want = 32 * (4 * bench.ns_flops_algorithmic(4096, 4096) + 2 * bench.ns_flops_algorithmic(4096, 11008)
                 + bench.ns_flops_algorithmic(11008, 4096))
    assert bench.set_flops() == want == 474_851_584_245_760


def test_oracle_set_time_is_composed_from_one_matrix_per_shape():
    t = {(4096, 4096): 3.0, (4096, 11008): 6.0, (11008, 4096): 11.0}
    assert bench.oracle_set_ms(t) == pytest.approx(1e3 * 32 * (4 * 3.0 + 2 * 6.0 + 11.0))
    obj = bench.cpu_baseline_object(t)
    assert obj["value"] == pytest.approx(bench.oracle_set_ms(t)) and obj["unit"] == "ms" and obj["kind"] == "oracle"
    assert "4 x t(4096x4096)" in obj["sample"] and "x32 layers" in obj["sample"]


def test_recorded_traffic_answers_only_for_the_captured_sources(tmp_path, monkeypatch):
    path = os.path.join(bench.ROOT, "profiles", "tc_gemm_traffic.json")
    rec = json.load(open(path))
    for key in ("kernel", "workload", "metric", "kernel_sources", "kernel_source_sha256_16",
                "traffic_bytes_per_launch_one_layer"):
        assert key in rec
    h = hashlib.sha256()
    for f in rec["kernel_sources"]:
        h.update(open(os.path.join(bench.ROOT, f), "rb").read())
    got = bench.recorded_traffic(4)
    if rec["kernel_source_sha256_16"] == h.hexdigest()[:16]:
        assert got == int(rec["traffic_bytes_per_launch_one_layer"] * 4)
    else:
        assert got is None
    # the same record against different kernel sources reads as no measurement
    root = tmp_path / "repo"
    (root / "profiles").mkdir(parents=True)
    stale = dict(rec, kernel_source_sha256_16="0" * 16)
    (root / "profiles" / "tc_gemm_traffic.json").write_text(json.dumps(stale))
    for f in rec["kernel_sources"]:
        dst = root / f
        dst.parent.mkdir(parents=True, exist_ok=True)
        dst.write_bytes(open(os.path.join(bench.ROOT, f), "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.recorded_traffic(4) is None
