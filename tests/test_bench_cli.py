"""bench.py's command line and entry points (no GPU needed)."""
import importlib.util
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load():
    spec = importlib.util.spec_from_file_location("bench_cli_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_bench_modes_exist():
    b = _load()
    for name in ("run_ours", "run_reference", "run_e2e", "run_profile", "run_rows", "run_flops", "run_spec", "cpu_baseline"):
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
    # on-chip index + top-k: 68 B per key read (64 codes + 4 scales), q_I and w in, 512 ids out
    assert b.index_topk_bytes(CFG2, 1) == 32768 * 68 + 8 * 128 * 2 + 8 * 4 + 512 * 4


def test_decode_flop_curve():
    """Closed forms of the weighted decode-FLOP model at the cfg2 layer shape (H=64, d=512, 8x128
    indexer, top-512, window 128, r=4)."""
    b = _load()
    from csa_workloads import CFG2
    s = CFG2
    full = b.decode_flops(131072, s, "full")
    n = 131072 // 4
    assert full["entries"] == n and full["keys"] == 512 + 128
    assert full["parts"]["indexer"] == 0.25 * 2 * 8 * 128 * n + 2 * 8 * n
    assert full["parts"]["attention"] == 4 * 64 * 512 * 640
    assert full["parts"]["compressor_k_I"] == 2 * 512 * 128 / 4
    # below k entries every entry is attended; the window is capped by the context
    small = b.decode_flops(1024, s, "full")
    assert small["keys"] == 256 + 128
    # Reuse runs no indexer: constant in the context once k entries exist; Reindex is constant once the
    # context outgrows its pool; Full grows linearly with the entries; HCA attends over T/128 entries
    assert b.decode_flops(4096, s, "reuse")["total"] == b.decode_flops(1 << 20, s, "reuse")["total"]
    assert b.decode_flops(1 << 18, s, "reindex")["total"] == b.decode_flops(1 << 20, s, "reindex")["total"]
    f4, f1m = b.decode_flops(4096, s, "full")["total"], b.decode_flops(1 << 20, s, "full")["total"]
    assert abs((f1m - f4) - (0.25 * 2048 + 16) * ((1 << 18) - 1024)) < 1e-3 * f1m
    assert b.decode_flops(1 << 20, s, "hca")["parts"]["attention"] == 4 * 64 * 512 * (8192 + 128)


@pytest.mark.parametrize("steps,warmup", [(20, 5), (16, 8), (3, 3), (20000, 64)])
def test_no_graph_capture_inside_the_timed_region(steps, warmup):
    """bench.py's timed loop only replays graphs: every capture happens in prepare(), before t0.  With
    the driver's --steps 20 --warmup 5 the loop needs the 8-step and the 4-step graphs, which a warm-up
    of 5 steps alone would not have built."""
    import contextlib

    bench = _load()
    log = []

    class FakeGraph:
        def replay(self):
            log.append("replay")

    def capture(g):
        log.append("capture")
        return contextlib.nullcontext()

    sg = bench.StepGraphs(lambda n, marks: log.append(("launch", n, marks)), lambda flag: None, None, bench.LAYERS,
                          graph_cls=FakeGraph, capture=capture)
    # the same calls, in the same order, as run_ours before its timing events
    sg.prepare(max(warmup, 3), steps)
    sg.prepare(bench.LAYERS, with_marks=True)
    sg.freeze()
    sg.run(max(warmup, 3))
    log.clear()                                   # t0.record(stream)
    sg.run(steps)                                 # the timed region
    assert "capture" not in log and not any(isinstance(e, tuple) for e in log)
    assert log.count("replay") == steps // bench.LAYERS + (1 if steps % bench.LAYERS else 0)
    log.clear()                                   # the stage replay after t1
    sg.run(bench.LAYERS, with_marks=True)
    assert log == ["replay"]
    prepared = {n for n, m in sg.graphs if not m}
    missing = next(n for n in range(1, bench.LAYERS) if n not in prepared)
    with pytest.raises(RuntimeError):             # an unprepared count is refused once frozen
        sg.run(missing)


def test_prefill_work_closed_forms():
    """The prefill FLOP counts: projection 4 T d_m d; the causal indexer scores sum_t floor((t+1)/r)
    entries = 2 (T/r)(T/r - 1) + ... (closed form for T a multiple of r); attention keys by a plain loop."""
    b = _load()
    from csa_workloads import CFG3 as s
    w = b.prefill_work(s)
    assert w["projection"] == 4 * s.T * s.d_m * s.d
    m = s.T // s.r
    scored = s.r * m * (m - 1) // 2 + m                      # sum_{u=1}^{T} floor(u / r)
    assert w["index"] == scored * s.H_I * s.d_I * 2
    keys = sum(min(s.k, (t + 1) // s.r) + min(s.W, t + 1) for t in range(s.T))
    assert w["attention"] == keys * s.H * s.d * 4
