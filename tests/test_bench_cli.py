"""bench.py's command line and entry points (no GPU needed)."""
import importlib.util
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load():
    spec = importlib.util.spec_from_file_location("bench_cli_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_bench_modes_exist():
    b = _load()
    for name in ("run_ours", "run_reference", "run_e2e", "run_profile", "run_rows", "cpu_baseline"):
        assert callable(getattr(b, name)), name


def test_bench_arguments(monkeypatch):
    b = _load()
    monkeypatch.setattr(sys, "argv", ["bench.py", "--steps", "5", "--warmup", "3", "--profile"])
    a = b.parse()
    assert a.steps == 5 and a.warmup == 3 and a.profile and not a.rows and a.impl == "ours"
    monkeypatch.setattr(sys, "argv", ["bench.py", "--rows"])
    assert b.parse().rows


def test_algorithmic_bytes():
    b = _load()
    from csa_workloads import CFG2
    # per sequence: 512 entries x (224 codes + 16 scales + 128 rope + 4 id) + 128 KB window + q + out + lse
    assert b.attention_bytes(CFG2, 1) == 512 * 372 + 128 * 1024 + 2 * 64 * 1024 + 64 * 4
    assert b.score_kernel_bytes(CFG2, 1) == 32768 * 72 + 8 * 128 * 2 + 8 * 4
