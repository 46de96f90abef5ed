"""Host logic of bench.py's multi-GPU path, run as two gloo ranks on the CPU.

Every rank times its own replicas; the step time is the maximum over ranks,
`value` counts the bytes of all ranks, and only rank 0 prints the JSON line.
"""
import json
import os
import socket
import sys
import types

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r is slower on one timer and faster on another
        mine = [1.0 + rank, 2.0 - rank, 0.5 + 0.25 * rank]
        got = bench.max_over_ranks(dist, mine)
        args = types.SimpleNamespace(steps=10, warmup=3, tokens=16, layers=4, gpus=world, model="llama3-8b")
        line = bench.decode_line(args, world, got[0], got[1], got[2], step_bytes=1e9, gemv_bytes=5e8,
                                 n_calls=16, hbm_peak=6454.9, peak_kind="measured", h2d=1, d2h=2,
                                 per_proj={}, n_launch=320, clocks={})
        printed = bench.emit(line, rank)
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump({"got": got, "line": line, "printed": printed}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_single_line(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["got"] == [2.0, 2.0, 0.75]                 # element-wise max over ranks
    assert [r["printed"] for r in res] == [True, False]     # one JSON line, from rank 0
    line = res[0]["line"]
    assert line["n_gpus"] == 2 and line["scaling"] == "weak"
    assert line["value"] == pytest.approx(1e9 * 10 * 2 / 2.0 / 1e9)   # all ranks' bytes / slowest time
    assert line["ms_per_step"] == pytest.approx(1e3 * 2.0 / 10)
    assert line["roofline"]["achieved"] == pytest.approx(5e8 * 10 / 0.75 / 1e9)   # per-rank kernel rate
    assert line["e2e"]["value"] == pytest.approx(1e9 * 10 * 2 / 2.0 / 1e9)


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(None, [3, 1.5]) == [3.0, 1.5]


def test_decode_line_carries_every_contract_key():
    sys.path.insert(0, ROOT)
    import bench
    args = types.SimpleNamespace(steps=10, warmup=3, tokens=16, layers=4, gpus=1, model="llama3-8b")
    line = bench.decode_line(args, 1, 2.0, 3.0, 1.0, step_bytes=1e9, gemv_bytes=5e8, n_calls=16,
                             hbm_peak=6454.9, peak_kind="measured", h2d=1, d2h=2, per_proj={},
                             n_launch=320, clocks={"sm_mhz": 1965.0})
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert k in line, k
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in line["roofline"], k
    for k in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"):
        assert k in line["e2e"], k
    # the captured traffic belongs to one kernel source: reported only while
    # gemv.cu is that file
    want = bench.GEMV_TRAFFIC_PER_LAUNCH_T16 if bench.gemv_source_sha() == bench.GEMV_TRAFFIC_SOURCE else None
    assert line["roofline"]["traffic"] == want
    assert line["e2e"]["value"] == pytest.approx(1e9 * 10 / 3.0 / 1e9)
    json.dumps(line)
    # the measured traffic belongs to one workload: no figure for another one
    other = types.SimpleNamespace(**{**vars(args), "model": "qwen3-4b"})
    assert bench.decode_line(other, 1, 2.0, 3.0, 1.0, 1e9, 5e8, 16, 6454.9, "measured", 1, 2, {}, 320,
                             {})["roofline"]["traffic"] is None


def test_traffic_figure_follows_the_kernel_source(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setattr(bench, "GEMV_TRAFFIC_SOURCE", bench.gemv_source_sha())
    assert bench.gemv_traffic(16, "llama3-8b") == bench.GEMV_TRAFFIC_PER_LAUNCH_T16
    assert bench.gemv_traffic(4, "llama3-8b") is None
    monkeypatch.setattr(bench, "GEMV_TRAFFIC_SOURCE", "0" * 16)
    assert bench.gemv_traffic(16, "llama3-8b") is None


def test_algorithmic_bytes_per_weight(monkeypatch):
    """The bench's byte counts: 4-bit codes plus one fp16 scale and one
    4-bit zero per group (0.5195 B per weight at group 128), the rotation's
    parameters as the pages give them (per pair an fp32 cos/sin pair and
    two channel bytes, 1/alpha per channel), and X read plus Y written."""
    sys.path.insert(0, ROOT)
    import bench
    n_in, n_out = 4096, 4096
    for g, per_weight in [(128, 0.5 + 2 / 128 + 0.5 / 128), (64, 0.5 + 2 / 64 + 0.5 / 64),
                          (256, 0.5 + 2 / 256 + 0.5 / 256)]:
        assert bench.weight_bytes(n_in, n_out, group=g) == n_in * n_out * per_weight
    monkeypatch.setattr(bench, "GROUP", 128)
    assert bench.rot_param_bytes(n_in, K=8, P=64) == 8 * 32 * 64 * 10 + 4 * 4096
    assert bench.call_bytes(16, n_in, n_out) == (bench.weight_bytes(n_in, n_out) + 2 * 16 * (n_in + n_out)
                                                 + bench.rot_param_bytes(n_in))
