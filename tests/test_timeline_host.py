"""Host side of the task-timeline profiler ("Mirage Persistent Kernel: Fusing
Multi-GPU LLM Inference into One Kernel Launch", "Getting Started": profiling
visualises the task timeline): the Chrome-trace writer and the per-operation
summary of bench.py on a synthetic record array (no GPU)."""
import json
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from synth import qwen3 as sq  # noqa: E402


def _entry(it, op, task):
    return (it << 32) | (op << 16) | task


def _records(iters=3, ops=(0, 1, 2), tasks=4, t0=1_000_000):
    """One record per (iteration, op, task): popped, ready, end, prologue, first
    data, first issue, stage wait, last data, rows done (ns)."""
    rows = []
    t = t0
    for it in range(iters):
        for op in ops:
            for k in range(tasks):
                pop = t + 100 * k
                ready = pop + 50
                pro = ready + 200
                data = pro + 10
                last = data + 300
                loop = last + 20
                end = loop + 30
                rows.append([_entry(it, op, k), k, pop, ready, end, pro, data, pop - 40, 7, last, loop])
            t += 2000
    return torch.tensor(rows, dtype=torch.int64)


def test_chrome_trace_has_one_event_per_record(tmp_path):
    tl = _records()
    path = tmp_path / "trace.json"
    bench.write_chrome_trace(tl, None, str(path))
    ev = json.load(open(path))["traceEvents"]
    assert len(ev) == tl.shape[0]
    t_min = int(tl[:, 2].min())
    for e, rec in zip(ev, tl.tolist()):
        it, op, task = (rec[0] >> 32) & 0xFFFFFFFF, (rec[0] >> 16) & 0xFFFF, rec[0] & 0xFFFF
        assert e["ph"] == "X" and e["name"] == f"op{op}" and e["tid"] == rec[1]
        assert e["args"]["iter"] == it and e["args"]["task"] == task
        assert abs(e["ts"] - (rec[2] - t_min) / 1e3) < 1e-9
        assert abs(e["dur"] - (rec[4] - rec[2]) / 1e3) < 1e-9
        assert abs(e["args"]["wait_us"] - 0.05) < 1e-9      # ready - popped
        assert abs(e["args"]["pro_us"] - 0.2) < 1e-9        # prologue - ready
        assert abs(e["args"]["rows_done_us"] - 0.53) < 1e-9  # rows done - ready


def test_chrome_trace_of_an_empty_timeline_writes_nothing(tmp_path):
    path = tmp_path / "none.json"
    bench.write_chrome_trace(torch.zeros((0, 11), dtype=torch.int64), None, str(path))
    assert not path.exists()


def test_timeline_summary_means_and_spans():
    shape = sq.Qwen3Shape("t", 1, 256, 4, 2, 64, 768, 1024, False)
    bench.op_kind.per_layer = 1  # embed, one op per layer, LM head: 3 ops
    out = bench.timeline_summary(_records(), shape)
    assert out["records"] == 3 * 3 * 4
    for kind in ("embed", "lmhead_argmax"):
        k = out[kind]
        assert abs(k["wait"] - 0.05) < 1e-9 and abs(k["pro"] - 0.2) < 1e-9
        assert abs(k["work"] - (0.2 + 0.01 + 0.3 + 0.02 + 0.03)) < 1e-9
        # span: first ready -> last end within one (iteration, op): tasks start 0.1 us apart
        assert abs(k["span"] - (0.3 + 0.56)) < 1e-9
    assert "iteration_us" in out and abs(out["iteration_us"] - 6.0) < 1e-9
    bench.op_kind.per_layer = 5
