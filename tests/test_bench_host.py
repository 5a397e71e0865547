"""Host logic of bench.py that needs no GPU: the CPU oracle's proportional slices and the
reference (oracle) arm's JSON line."""
import contextlib
import importlib.util
import io
import json
import os
import types

import pytest

from reduced_cross_entropy_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_host_under_test",
                                                  os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


@pytest.mark.parametrize("name", ["sasrec", "large", "very_large", "lm"])
def test_oracle_slice_keeps_chunks_windows_and_per_row_work(name):
    b = _bench()
    w = synth.WORKLOADS[name]
    ws, f = b.oracle_slice(w, seconds=1.0, rate=1e10)
    assert f >= 1 and (f & (f - 1)) == 0
    assert (ws.N * f, ws.C * f, ws.n_c * f) == (w.N, w.C, w.n_c)
    assert ws.N / ws.n_c == w.N / w.n_c and ws.C / ws.n_c == w.C / w.n_c
    assert (ws.d, ws.n_b, ws.k, ws.n_ec, ws.n_r, ws.dtype) == (w.d, w.n_b, w.k, w.n_ec,
                                                               w.n_r, w.dtype)
    if f > 1:
        assert ws.n_c >= 8
        # interior rows see the whole window of 1 + 2 n_ec chunks, as in the workload
        assert b.mean_window(ws) <= b.mean_window(w)
        assert b.mean_window(ws) >= 0.7 * b.mean_window(w)
    # a budget that fits leaves the workload whole
    whole, f1 = b.oracle_slice(w, seconds=1e9, rate=1e12)
    assert f1 == 1 and whole == w


def test_reference_arm_line_is_self_consistent():
    b = _bench()
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        b.run_reference(types.SimpleNamespace(workload="tiny", warmup=1, steps=2, gpus=1,
                                              flags=0))
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "rows/s"
    # value = rows of one (slice) step x steps / the steps' time: ms_per_step is real time
    assert line["value"] == pytest.approx(line["rows_per_step"] / (line["ms_per_step"] / 1e3))
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["method"] == "full" and cb["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
