"""bench.py's roofline accounting, on the CPU.

The algorithmic bytes of each stage are the bytes of the tensors the stage must
read and write once; here they are rebuilt from the tensors themselves (the
workload's inputs as drawn, and the intermediate buffers' shapes), so a wrong
factor or a dropped operand in the bench's formulas fails. The flops are
rebuilt from the matmul shapes each stage performs. The DRAM traffic of the
dominant kernel comes from a committed ncu summary and must disappear once the
kernel's sources change.
"""
import json
import os

import pytest
import torch

import bench
from mixture_experts_ffn_sigmoid_b200.inputs import CONFIGS, make_inputs


def nbytes(*ts):
    return sum(t.numel() * t.element_size() for t in ts if t is not None)


@pytest.mark.parametrize("shared", [False, True])
def test_stage_bytes_are_the_operands_touched_once(shared):
    cfg = CONFIGS["deepseek_v3"].with_(T=24, d=64, E=8, k=2, f=32, f_shared=48 if shared else 0,
                                       n_groups=1, topk_groups=1)
    inp = make_inputs(cfg, "cpu", seed=3)
    counts = torch.tensor([5, 0, 9, 0, 0, 20, 14, 0])
    assert int(counts.sum()) == cfg.T * cfg.k
    work, touched = bench.stage_work(cfg, counts)
    assert touched == 4
    used = counts > 0
    rows, T = cfg.T * cfg.k, cfg.T
    dt = cfg.torch_dtype
    x_perm = torch.empty((rows, cfg.d), dtype=dt)
    h = torch.empty((rows, cfg.f), dtype=dt)
    y_perm = torch.empty((rows, cfg.d), dtype=dt)
    h_s = torch.empty((T, cfg.f_shared), dtype=dt) if shared else None
    y_s = torch.empty((T, cfg.d), dtype=dt) if shared else None
    y = torch.empty((T, cfg.d), dtype=dt)
    idx32 = torch.empty((T, cfg.k), dtype=torch.int32)
    gate32 = torch.empty((T, cfg.k), dtype=torch.float32)
    logits = torch.empty((T, cfg.E), dtype=torch.float32)

    # gate/up: W1 and W3 of the experts that received tokens, the shared pair,
    # the packed rows and x (shared expert input), the activations written.
    gate_up = nbytes(inp["w1"][used], inp["w3"][used], inp["ws1"], inp["ws3"], x_perm,
                     inp["x"] if shared else None, h, h_s)
    assert work["gate_up"]["bytes"] == gate_up
    down = nbytes(inp["w2"][used], inp["ws2"], h, h_s, y_perm, y_s)
    assert work["down"]["bytes"] == down
    # permute: x read once, packed rows written, plus the two int32 row maps
    # (packed row -> token and token slot -> packed row) and the int32 indices read.
    assert work["permute"]["bytes"] == nbytes(inp["x"], x_perm) + 2 * rows * 4 + nbytes(idx32)
    # combine: packed rows and shared rows read, y written, int32 row map and fp32 gates read.
    assert work["combine"]["bytes"] == nbytes(y_perm, y_s, y) + nbytes(idx32, gate32)
    # route: x and the router read, the summed fp32 logits written once, indices and gates written.
    assert work["route"]["bytes"] == nbytes(inp["x"], inp["w_router"], logits, idx32, gate32)

    # flops: 2 per multiply-add of each matmul the stage performs.
    def mm(m, n, kk):
        return 2.0 * m * n * kk
    assert work["gate_up"]["flops"] == 2 * mm(rows, cfg.f, cfg.d) + (2 * mm(T, cfg.f_shared, cfg.d) if shared else 0)
    assert work["down"]["flops"] == mm(rows, cfg.d, cfg.f) + (mm(T, cfg.d, cfg.f_shared) if shared else 0)
    assert work["route"]["flops"] == mm(T, cfg.E, cfg.d)


def test_traffic_is_reported_only_for_the_profiled_sources(monkeypatch):
    path = os.path.join(bench.ROOT, "profiles", "dram_traffic.json")
    table = json.load(open(path))
    for workload, stages in table.items():
        if workload.startswith("_"):
            continue
        for stage, entry in stages.items():
            # a committed figure is reported while the kernel's sources are the
            # ones it was captured on, and withheld (null) once they change
            srcs = [os.path.join(bench.ROOT, x) for x in entry["sources"]]
            current = bench.source_sha(srcs) == entry["source_sha256_16"]
            assert bench.traffic_for(workload, stage) == (entry["bytes_per_launch"] if current else None)
            # and they are within a few percent of the algorithmic bytes they were taken against
            assert 0.97 < entry["traffic_over_algorithmic"] < 1.10
    assert bench.traffic_for("no_such_workload", "gate_up") is None
    monkeypatch.setattr(bench, "source_sha", lambda paths: "0" * 16)
    assert bench.traffic_for("deepseek_v3", "gate_up") is None


def test_source_sha_covers_every_listed_file(tmp_path):
    a, b = tmp_path / "a.cu", tmp_path / "b.cuh"
    a.write_text("kernel A")
    b.write_text("helpers B")
    one = bench.source_sha([str(a), str(b)])
    b.write_text("helpers B, changed")
    assert bench.source_sha([str(a), str(b)]) != one
    assert bench.source_sha(str(a)) == bench.source_sha([str(a)])
