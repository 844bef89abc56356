"""The N > 1 host logic of bench.py on two gloo ranks (CPU only).

bench.py runs one independent replica per GPU (weak scaling); the only
cross-rank steps are the timing barrier, the max-over-ranks reduction of the
timed region and of each kernel's time, and the gathering of clock samples.
"""
from __future__ import annotations

import json
import os
import socket
import sys
from pathlib import Path

import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parent.parent


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, str(ROOT))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench

    ms = 100.0 + 10 * rank
    per = {"fwd": 1.0 + rank, "bwd_main": 5.0 - rank}
    clocks = {"sm_mhz": 1900.0 - 100 * rank, "sm_max_mhz": 1965.0,
              "reasons": ["sw_power_cap"] if rank == 1 else []}
    dist.barrier()
    ms2, per2, clk2 = bench.combine_ranks(ms, per, clocks, "cpu")
    value = bench.job_tflops(world, 7.0e12, ms2 / 10)
    dist.barrier()
    dist.destroy_process_group()
    Path(out_dir, "r%d.json" % rank).write_text(json.dumps({"ms": ms2, "per": per2, "clocks": clk2, "value": value}))


def test_two_rank_max_reduction_and_aggregate(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.loads((tmp_path / ("r%d.json" % r)).read_text()) for r in range(world)]
    for r in res:
        assert r["ms"] == 110.0                      # max of 100, 110
        assert r["per"] == {"fwd": 2.0, "bwd_main": 5.0}
        assert r["clocks"]["reasons"] == ["sw_power_cap"]
        assert r["clocks"]["sm_mhz"] == 1850.0       # median of the two ranks' medians
        # 2 ranks x 7e12 FLOPs over the slowest rank's 11 ms per step
        assert abs(r["value"] - 2 * 7.0e12 / 11e-3 / 1e12) < 1e-9


def _bench(args, env_extra=None):
    import subprocess

    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, str(ROOT / "bench.py"), *args], capture_output=True, text=True,
                          env=env, timeout=600, cwd=str(ROOT))


def test_reference_arm_prints_the_contract_line():
    # the reference arm times the float64 oracle on the host; no GPU involved
    r = _bench(["--impl", "reference", "--steps", "2", "--warmup", "0", "--workload", "small_n1024_g256"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert d["steps"] == 2 and d["warmup"] >= 3 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "small_n1024_g256" and d["dtype"] == "f64"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert set(d["cpu_baseline"]["seconds"]) == {"fwd", "bwd", "total"} and d["cpu_baseline"]["cpu_model"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_prints_nothing_on_other_ranks():
    r = _bench(["--impl", "reference", "--steps", "1", "--workload", "small_n1024_g256"],
               {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_sp_layout_cuts_g_aligned_shards_with_padding_on_the_last():
    # bench.py --sp: rank r holds [rL, rL + L); only the last rank may hold padding
    import bench

    assert bench.sp_layout(32768, 8192, 32768, 1) == (32768, [32768])
    assert bench.sp_layout(32768, 8192, 32768, 4) == (8192, [8192] * 4)
    assert bench.sp_layout(106496, 8192, 100000, 13) == (8192, [8192] * 12 + [100000 - 12 * 8192])
    assert bench.sp_layout(12288, 1536, 12288, 8) == (1536, [1536] * 8)
    import pytest

    with pytest.raises(ValueError):
        bench.sp_layout(32768, 8192, 32768, 8)  # shards of 4096 < G
    with pytest.raises(ValueError):
        bench.sp_layout(4096, 1024, 2000, 4)  # padding on ranks 1..3
