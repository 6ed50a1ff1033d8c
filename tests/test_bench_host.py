"""Host-side logic of bench.py (CPU): the work model behind `roofline` and the source hash
that decides whether the committed ncu traffic still applies."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from newton_schulz_11_b200 import inputs  # noqa: E402


def test_code_only_strips_comments_not_literals():
    src = 'int a = 1; // note\n/* block\n comment */ const char* s = "x//y/*z*/";\n  char q = \'"\';\treturn;'
    assert bench._code_only(src) == 'int a = 1; const char* s = "x//y/*z*/"; char q = \'"\'; return;'
    # an escaped quote does not end the literal, so the // after it stays
    assert bench._code_only('asm("mov \\"a\\" // b"); // c') == 'asm("mov \\"a\\" // b");'
    assert bench._code_only("a   b\n\n c") == "a b c"


def test_source_hash_ignores_comments_only(tmp_path, monkeypatch):
    csrc = tmp_path / "newton_schulz_11_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("__global__ void k() { int x = 1; }  // v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    (csrc / "k.cu").write_text("// a new header comment\n__global__ void k() {\n  int x = 1;  /* v2 */\n}\n")
    assert bench.kernel_source_hash() == h0
    (csrc / "k.cu").write_text("__global__ void k() { int x = 2; }\n")
    assert bench.kernel_source_hash() != h0


def test_work_model_matches_the_gpt2_124m_counts():
    w = inputs.WORKLOADS["gpt2-124m-72-matrices"]
    n = sum(r * c for r, c in w.shapes)
    assert n == 84_934_656
    # elementwise: read g, m (8 B), write m (4 B), hi (2 B), lo (1 B)
    assert bench.kind_bytes(w, "momentum") == 15 * n
    # apply: read hi, lo (3 B) and B, write hi, lo (3 B)
    m2 = sum(min(r, c) ** 2 for r, c in w.shapes)
    assert bench.kind_bytes(w, "apply") == 6 * n + 2 * m2
    # last apply with bf16 W: read hi, lo, B; W read and written
    assert bench.kind_bytes(w, "apply_last") == 7 * n + 2 * m2
    alg, dense = bench.step_flops(w)
    # 5 iterations of 3 m^2 n + m^3 (algorithmic) and 4 m^2 n + 2 m^3 (dense)
    assert alg == pytest.approx(1.142e12, rel=1e-3)
    assert dense == pytest.approx(1.631e12, rel=1e-3)


def test_work_model_is_orientation_free():
    assert bench.matrix_work(768, 3072) == bench.matrix_work(3072, 768)
    mw = bench.matrix_work(256, 1024)
    assert mw["gram"] == 256 * 256 * 1024 and mw["poly"] == 256 ** 3 and mw["apply"] == 2 * 256 * 256 * 1024


def test_roofline_takes_the_bound_with_the_longer_floor_and_fixed_denominators():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1200.0}
    # 0.75 TFLOP and 6 GB in 1 ms: 750 TF/s (0.5 of the tensor peak), 6000 GB/s (1.0 of HBM)
    r = bench.roofline_of(0.75e12, 6e9, 1.0, peaks, "measured")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["frac"] == pytest.approx(1.0) and r["frac_hbm"] == pytest.approx(1.0)
    assert r["frac_tensor"] == pytest.approx(0.5)
    assert r["frac_tensor_of_sustained"] == pytest.approx(0.625)
    assert r["frac_nominal"]["tensor"] == pytest.approx(750 / bench.NOMINAL_PEAKS["bf16_tflops"], abs=1e-4)
    # the same kernel with a tenth of the bytes is tensor-bound, against the burst peak whatever the clocks
    r = bench.roofline_of(0.75e12, 0.6e9, 1.0, peaks, "measured")
    assert r["bound"] == "tensor" and r["peak"] == 1500.0 and r["frac"] == pytest.approx(0.5)
    # no flops: HBM
    assert bench.roofline_of(0, 3e9, 1.0, peaks, "measured")["bound"] == "hbm"


def test_both_arms_print_the_same_config():
    w = inputs.WORKLOADS["gpt2-124m-72-matrices"]
    import types

    args = types.SimpleNamespace(steps=20, warmup=5, parallel="auto")
    for world in (1, 2, 8):
        mode = bench.parallel_mode(args, world)
        assert mode == ("single" if world == 1 else "sharded")
        line = bench.base_line(w, world, mode, 1.0, args)
        assert line["config"] == bench.config_of(w, world, mode)
        assert line["scaling"] == "strong"
    args.parallel = "replicas"
    assert bench.base_line(w, 4, bench.parallel_mode(args, 4), 1.0, args)["scaling"] == "weak"


def test_oracle_plan_takes_full_steps_within_budget_and_windows_beyond(monkeypatch):
    w = inputs.scaled_workload(inputs.WORKLOADS["gpt2-124m-72-matrices"], [(32, 32), (32, 64), (64, 32)] * 2)
    ow = bench.OracleWorkload(w)
    monkeypatch.setattr(ow, "run", lambda idx: 0.01 * len(idx))  # 10 ms per matrix, no oracle run
    plans, total, sample = ow.plan(5, 10.0)
    assert all(p == list(range(6)) for p in plans) and "full step" in sample
    plans, total, sample = ow.plan(5, 0.1)  # 20 ms per run: windows of matrices, taken cyclically
    assert all(1 <= len(p) < 6 for p in plans)
    assert plans[1][0] == (plans[0][-1] + 1) % 6
    assert total == sum(ow.work(i) for i in range(6))
