"""The multi-GPU branch of bench.py without a GPU.

`python bench.py --gpus N` starts N ranks itself (torchrun on the loopback
address) and refuses clearly when fewer GPUs are visible. The multi-rank
step, timing and JSON line (bench.sharded_line) run here on two gloo ranks
with an oracle-backed stand-in for the per-rank handle: the line must report
both ranks' rows (n_gpus, global_rows, e2e byte counts, a summed roofline)
and the statistics of all rows exactly as the single-process oracle gives
them."""
import json
import math
import os
import subprocess
import sys
import types

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
from logit_kl_divergence_b200 import synth
from logit_kl_divergence_b200.sharded import ShardedKLDStats

from test_sharded_gloo import OracleStats, _free_port, _same

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
N_PER_RANK, V = 24, 1999


class TimedOracleStats(OracleStats):
    """OracleStats with the handle's timing and host-memory calls."""

    def set_timing(self, enable):
        self.timing_on = enable

    def timing(self):
        return 0.5, 0.01  # fixed stand-in durations (ms)

    def run_rows_host(self, base, quant, token_ids=None, out=None):
        return self.run_rows(base, quant, token_ids, out)


def _shard(rank):
    return synth.make_recipe("ctx", n=N_PER_RANK, v=V, dtype=synth.F32, seed=40 + rank)


def _worker(rank, world, port, q):
    try:
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                world_size=world)
        w = _shard(rank)
        sk = ShardedKLDStats(max_rows_per_rank=N_PER_RANK, stats=TimedOracleStats(oracle.F32))
        args = types.SimpleNamespace(warmup=1, steps=2, e2e_steps=1, no_cpu_baseline=False)
        fake_cpu = lambda name: ({"value": 1.0, "unit": "rows/s", "cores": 1, "kind": "oracle",  # noqa: E731
                                  "sample": name}, None)
        line = bench.sharded_line(args, rank, world, torch.device("cpu"), sk,
                                  (w.base, w.quant, w.token_ids), bench.HostClock(), 1000.0,
                                  "measured", cpu_fn=fake_cpu)
        if rank == 0:
            q.put(json.dumps(line))
        else:
            assert line is None
        dist.barrier()
        dist.destroy_process_group()
    except BaseException as e:
        q.put(f"ERROR rank {rank}: {type(e).__name__}: {e}")
        raise


def test_sharded_bench_line_on_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    mp.start_processes(_worker, args=(world, _free_port(), q), nprocs=world, join=True,
                       start_method="spawn")
    msg = q.get()
    assert not msg.startswith("ERROR"), msg
    line = json.loads(msg)
    assert line["n_gpus"] == world and line["scaling"] == "weak"
    assert line["config"]["global_rows"] == world * N_PER_RANK
    assert line["config"]["rows_per_gpu"] == N_PER_RANK
    assert line["value"] > 0 and line["ms_per_step"] > 0
    in_bytes = 2 * N_PER_RANK * V * 4
    assert line["e2e"]["h2d_bytes_per_step"] == world * (in_bytes + 4 * N_PER_RANK)
    assert line["e2e"]["d2h_bytes_per_step"] == world * bench.RESULT_BYTES
    # achieved bandwidth summed over the ranks' row passes (0.5 ms each)
    assert math.isclose(line["roofline"]["achieved"], world * in_bytes / 0.5e-3 / 1e9)
    assert line["roofline"]["peak"] == world * 1000.0
    assert line["cpu_baseline"]["kind"] == "oracle"
    # the statistics of all ranks' rows, as the single-process oracle gives them
    shards = [_shard(r) for r in range(world)]
    base = torch.cat([s.base for s in shards])
    quant = torch.cat([s.quant for s in shards])
    tok = torch.cat([s.token_ids for s in shards])
    _, ref = oracle.run(base, quant, tok, oracle.F32)
    for k in ("mean_kld", "median_kld", "p99_kld", "max_kld", "top1_agree_pct", "ppl", "ppl_base",
              "rms_dp", "mean_dp"):
        assert line[k] == ref[k], (k, line[k], ref[k])


def test_torchrun_command_for_n_ranks():
    cmd = bench.torchrun_argv(4, 29511, "/x/bench.py", ["--gpus", "4", "--steps", "5"])
    assert cmd[:3] == [sys.executable, "-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--nnodes=1" in cmd
    i = cmd.index("--master-addr")
    assert cmd[i + 1] == "127.0.0.1" and cmd[cmd.index("--master-port") + 1] == "29511"
    assert cmd[-5:] == ["/x/bench.py", "--gpus", "4", "--steps", "5"]


def test_more_gpus_than_visible_is_refused_clearly():
    if torch.cuda.device_count() >= 2:
        import pytest

        pytest.skip("two GPUs are visible here")
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--steps", "1"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 2
    assert "2 GPUs requested" in r.stderr and r.stdout == ""
