"""The multi-rank host logic of bench.py with two CPU ranks over gloo: every
rank takes the same collective steps; the step time is the maximum over ranks;
the reported value counts the work of all ranks (replicas: no data-path
collective); the reference arm runs on rank 0 only."""
import json
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from causal_flash_attention_packed_b200 import workloads as W

        dev = torch.device("cpu")
        local_ms = [3.0, 5.0][rank]  # rank 1 is the slower one
        bench.barrier(world)
        got = bench.max_over_ranks(local_ms, world, dev)
        w = W.config(1, 0)
        peaks = {"bf16_tflops": 1000.0, "bf16_tflops_sustained": 900.0, "hbm_gbs": 6000.0, "sm_max_mhz": 2000.0,
                 "source": "measured"}
        clk = {"sm_mhz": 1500.0}
        rep = bench.path_report(w, "bf16", got, {n: 1.0 for n in bench.KERNELS["bf16"][0] + bench.KERNELS["bf16"][1]},
                                9, world, peaks, clk, config=1)
        # the tensor denominator is the burst peak scaled to the sampled clock
        assert abs(rep["roofline"]["peak"] - 750.0) < 1e-9
        bench.barrier(world)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max_ms": got, "value": rep["value"], "flops": w.flops()}, f)
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.timeout(240)
def test_two_gloo_ranks_time_is_max_and_value_counts_both(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.loads((tmp_path / f"rank{r}.json").read_text()) for r in range(world)]
    assert res[0]["max_ms"] == res[1]["max_ms"] == 5.0
    # value = the work of all ranks / the slowest rank's time
    want = res[0]["flops"] * world / (5.0e-3) / 1e12
    assert abs(res[0]["value"] - want) <= 1e-9 * want
    assert res[0]["value"] == res[1]["value"]


def _ref_main(rank, world, port, out_dir):
    import datetime
    import contextlib
    import io

    sys.path.insert(0, ROOT)
    torch.distributed.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                         world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench

        class A:
            steps, warmup, ref_seconds = 1, 0, 0.01

        from causal_flash_attention_packed_b200 import workloads as W

        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            bench.run_reference(A, W.config(1, 0), world, rank)
        with open(os.path.join(out_dir, f"ref{rank}.txt"), "w") as f:
            f.write(buf.getvalue())
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.timeout(240)
def test_reference_arm_prints_on_rank0_only(tmp_path):
    world = 2
    mp.start_processes(_ref_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    out0 = (tmp_path / "ref0.txt").read_text().strip().splitlines()
    out1 = (tmp_path / "ref1.txt").read_text()
    assert out1 == ""
    line = json.loads(out0[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == world and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
