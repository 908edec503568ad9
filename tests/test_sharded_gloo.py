"""Row sharding across processes (the multi-GPU path's host logic), run as
gloo ranks on the CPU: shard bounds, the rank-ordered all-gather of 40-byte
records (equal and unequal row counts), and the orchestration of
ShardedKLDStats with the per-rank row pass and reduction supplied by the
oracle, so the statistics of the gathered shards must equal the oracle's
statistics of all rows exactly."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from logit_kl_divergence_b200 import rows_view, synth
from logit_kl_divergence_b200.sharded import ShardedKLDStats, gather_records, shard_bounds

RECORD = np.dtype([("kld", "<f8"), ("nll", "<f8"), ("nll_base", "<f8"), ("amax_b", "<i4"),
                   ("amax_q", "<i4"), ("flags", "<u4"), ("dp", "<f4")])
assert RECORD.itemsize == 40


def _pack(r: dict) -> np.ndarray:
    a = np.zeros(r["kld"].shape[0], dtype=RECORD)
    for k in ("kld", "nll", "nll_base", "amax_b", "amax_q", "flags"):
        a[k] = r[k]
    a["dp"] = np.exp(-r["nll"]) - np.exp(-r["nll_base"])
    return a.view(np.uint8).reshape(-1, 40)


class OracleStats:
    """Per-rank stand-in for the GPU handle: the oracle's row pass writes
    records in the library's layout, its reduction reads them back."""

    def __init__(self, dtype):
        self.dtype = dtype
        self.res = None

    def run_rows(self, base, quant, token_ids=None, out=None):
        if base.shape[0] < 1:  # as the library: a row pass needs at least one row
            raise ValueError("kld_stats_run_rows: N must be >= 1")
        r = oracle.rows(base, quant, token_ids, self.dtype)
        out.copy_(torch.from_numpy(_pack(r)))
        return out

    def reduce(self, records, n_rows, has_nll):
        v = rows_view(records[:n_rows])
        r = {k: t.numpy().copy() for k, t in v.items()}
        r["flags"] = r["flags"].astype(np.uint32)
        self.res = oracle.reduce(r, has_nll)

    def result(self):
        return self.res


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _same(a, b):
    assert a.keys() == b.keys()
    for k in a:
        x, y = a[k], b[k]
        if isinstance(x, float) and math.isnan(x):
            assert isinstance(y, float) and math.isnan(y), k
        else:
            assert x == y, (k, x, y)


def _worker(rank, world, port, n_rows, with_tokens, errq):
    try:
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                world_size=world)
        w = synth.make_recipe("edge", n=n_rows, v=3001, dtype=synth.F32, seed=7)
        tok = w.token_ids if with_tokens else None
        lo, hi = shard_bounds(n_rows, world, rank)
        # rank-ordered gather of raw records
        mine = torch.full((hi - lo, 40), rank, dtype=torch.uint8)
        got = gather_records(mine)
        expect = torch.cat([torch.full((b - a, 40), r, dtype=torch.uint8)
                            for r, (a, b) in enumerate(shard_bounds(n_rows, world, q) for q in range(world))])
        assert torch.equal(got, expect)
        # 64-byte vocabulary-slice partials: every rank holds all rows, so
        # the gather is [world][n] in rank order
        slc = torch.full((n_rows, 64), 100 + rank, dtype=torch.uint8)
        allp = gather_records(slc, counts=[n_rows] * world).view(world, n_rows, 64)
        assert all(torch.all(allp[r] == 100 + r) for r in range(world))
        # the whole orchestration, oracle-backed
        sk = ShardedKLDStats(max_rows_per_rank=hi - lo + 1, stats=OracleStats(oracle.F32))
        res = sk.run(w.base[lo:hi].contiguous(), w.quant[lo:hi].contiguous(),
                     None if tok is None else tok[lo:hi].contiguous())
        _, full = oracle.run(w.base, w.quant, tok, oracle.F32)
        _same(res, full)
        assert res["n_rows"] == n_rows
        dist.barrier()
        dist.destroy_process_group()
    except BaseException as e:  # reported to the parent
        errq.put(f"rank {rank}: {type(e).__name__}: {e}")
        raise


def _spawn(world, n_rows, with_tokens):
    ctx = mp.get_context("spawn")
    errq = ctx.SimpleQueue()
    mp.start_processes(_worker, args=(world, _free_port(), n_rows, with_tokens, errq), nprocs=world,
                       join=True, start_method="spawn")
    assert errq.empty(), errq.get()


def test_shard_bounds_cover_all_rows_in_order():
    for n in (0, 1, 7, 8, 37, 8192):
        for world in (1, 2, 3, 8):
            b = [shard_bounds(n, world, r) for r in range(world)]
            assert b[0][0] == 0 and b[-1][1] == n
            assert all(b[i][1] == b[i + 1][0] for i in range(world - 1))
            sizes = [hi - lo for lo, hi in b]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    with pytest.raises(ValueError):
        shard_bounds(4, 2, 2)


@pytest.mark.parametrize("world,n_rows,with_tokens", [(2, 64, True), (2, 37, False), (3, 37, True),
                                                     (3, 2, True)])  # the last rank holds no rows
def test_sharded_statistics_equal_single_process_oracle(world, n_rows, with_tokens):
    _spawn(world, n_rows, with_tokens)


# ---- failure detection on the host: a failing or vanished rank ----------

class FailingStats(OracleStats):
    """OracleStats whose row pass fails with a library-style error on the
    listed steps (the fake of an error status from the failing call)."""

    def __init__(self, dtype, fail_steps):
        super().__init__(dtype)
        self.fail_steps = set(fail_steps)
        self.step = 0

    def run_rows(self, base, quant, token_ids=None, out=None):
        step, self.step = self.step, self.step + 1
        if step in self.fail_steps:
            raise RuntimeError("kld_stats_run: KLD_ERR_CUDA (fake)")
        return super().run_rows(base, quant, token_ids, out)


class SliceStats:
    """Stand-in for the vocabulary-slice handle: each rank's partials are
    bytes that name the rank and row; the merge records what it was given."""

    def __init__(self, rank, fail_steps):
        self.rank, self.fail_steps, self.step, self.merged = rank, set(fail_steps), 0, None

    def run_partials(self, base, quant, token_ids, col_offset, v_total):
        step, self.step = self.step, self.step + 1
        if step in self.fail_steps:
            raise RuntimeError("kld_stats_run_partials: KLD_ERR_OOM (fake)")
        n = base.shape[0]
        p = torch.zeros((n, 64), dtype=torch.uint8)
        p[:, 0] = self.rank
        p[:, 1] = torch.arange(n, dtype=torch.uint8)
        return p

    def merge_partials(self, parts, token_ids, v_total):
        self.merged = parts.clone()

    def result(self):
        return {"merged": self.merged}


def _fail_worker(rank, world, port, mode, errq):
    import datetime
    import time

    from logit_kl_divergence_b200.sharded import ShardFailure, VocabShardedKLDStats
    try:
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                world_size=world, timeout=datetime.timedelta(seconds=5))
        w = synth.make_recipe("ctx", n=24, v=1999, dtype=synth.F32, seed=11)
        lo, hi = shard_bounds(24, world, rank)
        b, q, t = w.base[lo:hi].contiguous(), w.quant[lo:hi].contiguous(), w.token_ids[lo:hi].contiguous()
        if mode == "status":
            # step 0 fails on the last rank only: every rank must raise the
            # same ShardFailure; step 1 then runs normally on the same group
            fails = [0] if rank == world - 1 else []
            sk = ShardedKLDStats(max_rows_per_rank=hi - lo, stats=FailingStats(oracle.F32, fails))
            with pytest.raises(ShardFailure) as ei:
                sk.run(b, q, t)
            assert ei.value.ranks == [world - 1]
            assert (ei.value.cause is not None) == (rank == world - 1)
            res = sk.run(b, q, t)
            _, full = oracle.run(w.base, w.quant, w.token_ids, oracle.F32)
            _same(res, full)
        elif mode == "status_counts":
            # the same with the row counts given by the caller: the status
            # travels in a collective enqueued with the gather and is read
            # after the result; every rank still raises, and the next step
            # on the same group is normal
            counts = [b - a for a, b in (shard_bounds(24, world, r) for r in range(world))]
            fails = [1] if rank == 0 else []
            sk = ShardedKLDStats(max_rows_per_rank=hi - lo, stats=FailingStats(oracle.F32, fails))
            _, full = oracle.run(w.base, w.quant, w.token_ids, oracle.F32)
            _same(sk.run(b, q, t, counts=counts), full)
            with pytest.raises(ShardFailure) as ei:
                sk.run(b, q, t, counts=counts)
            assert ei.value.ranks == [0]
            _same(sk.run(b, q, t, counts=counts), full)
            with pytest.raises(ValueError, match="counts"):
                sk.run(b, q, t, counts=counts[::-1] if len(set(counts)) > 1 else [c + 1 for c in counts])
        elif mode == "vocab":
            fails = [0] if rank == 0 else []
            vs = VocabShardedKLDStats(5, stats=SliceStats(rank, fails))
            x = torch.zeros((5, 10))
            with pytest.raises(ShardFailure) as ei:
                vs.run(x, x, None, 10 * rank, 10 * world)
            assert ei.value.ranks == [0]
            got = vs.run(x, x, None, 10 * rank, 10 * world)["merged"]
            assert got.shape == (world, 5, 64)
            for r in range(world):
                assert torch.all(got[r, :, 0] == r) and torch.equal(got[r, :, 1], torch.arange(5, dtype=torch.uint8))
        elif mode == "zero":
            # every rank passes an empty shard: all raise the same clear
            # error after the same collective steps, and the group stays
            # usable for a normal step
            sk = ShardedKLDStats(max_rows_per_rank=hi - lo, stats=OracleStats(oracle.F32))
            with pytest.raises(ValueError, match="zero rows"):
                sk.run(b[:0], q[:0], t[:0])
            res = sk.run(b, q, t)
            _, full = oracle.run(w.base, w.quant, w.token_ids, oracle.F32)
            _same(res, full)
        elif mode == "exit":
            # the last rank leaves between steps without telling anyone; the
            # others' next collective must end with an error, not hang
            if rank == world - 1:
                dist.barrier()
                os._exit(0)
            sk = ShardedKLDStats(max_rows_per_rank=hi - lo, stats=OracleStats(oracle.F32))
            dist.barrier()
            t0 = time.monotonic()
            try:
                sk.run(b, q, t)
            except Exception:
                dt = time.monotonic() - t0
                assert dt < 60, dt
            else:
                raise AssertionError("run completed without the vanished rank")
            os._exit(0)  # the group cannot be torn down cleanly without its peer
        dist.barrier()
        dist.destroy_process_group()
    except BaseException as e:  # reported to the parent
        errq.put(f"rank {rank}: {type(e).__name__}: {e}")
        raise


@pytest.mark.parametrize("world,mode", [(2, "status"), (3, "status"), (2, "status_counts"),
                                        (3, "status_counts"), (2, "vocab"), (3, "vocab"),
                                        (2, "zero"), (2, "exit")])
def test_rank_failure_is_seen_by_every_rank(world, mode):
    ctx = mp.get_context("spawn")
    errq = ctx.SimpleQueue()
    mp.start_processes(_fail_worker, args=(world, _free_port(), mode, errq), nprocs=world, join=True,
                       start_method="spawn")
    assert errq.empty(), errq.get()
