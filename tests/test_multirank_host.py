"""Host logic of the multi-rank benchmark on two gloo ranks (CPU): every
rank gets the slowest rank's time, ranks process distinct images, and the
job's throughput counts all ranks' tokens over that time."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from linear_compressed_attention_b200.inputs import WORKLOADS, make_inputs  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        per_rank_ms = [12.5, 20.0][rank]
        mx = bench.reduce_max(per_rank_ms, world)
        cfg = bench.rank_config(dict(WORKLOADS["tiny_fp32"]), rank)
        x = torch.from_numpy(make_inputs(**cfg)["x"])
        gathered = [torch.zeros_like(x) for _ in range(world)]
        dist.all_gather(gathered, x)
        same = bool(torch.equal(gathered[0], gathered[1]))
        torch.save({"max": mx, "seed": cfg["seed"], "same_images": same}, os.path.join(out, f"r{rank}.pt"))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [torch.load(os.path.join(tmp_path, f"r{r}.pt")) for r in range(world)]
    assert [r["max"] for r in res] == [20.0, 20.0]
    assert [r["seed"] for r in res] == [WORKLOADS["tiny_fp32"]["seed"], WORKLOADS["tiny_fp32"]["seed"] + 1]
    assert not res[0]["same_images"]


def test_single_rank_and_throughput():
    assert bench.reduce_max(3.25, 1) == 3.25
    assert bench.rank_config(dict(seed=3, H=8), 0) == dict(seed=3, H=8)
    # 2 ranks x 1 image x 65,536 tokens x 10 steps in 9.4 ms (slowest rank)
    assert abs(bench.job_tokens_per_s(2, 1, 65536, 10, 9.4) - 2 * 65536 * 10 / 0.0094) < 1e-3


def test_lib_option_rejects_a_missing_build(monkeypatch):
    import pytest

    monkeypatch.setattr(sys, "argv", ["bench.py", "--lib", os.path.join(ROOT, "no-such-dir", "libedit_attn.so")])
    with pytest.raises(SystemExit) as e:
        bench.main()
    assert "no such file" in str(e.value)
