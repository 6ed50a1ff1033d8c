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
