"""Row-sharded statistics over several processes, one GPU each.

Rows are independent, so N rows split across ranks with no exchange in the
row pass. The one real exchange is for the order statistics: every rank
all-gathers the 40-byte per-row records in rank order (NCCL over NVLink on
GPUs; any torch.distributed backend carries the gather) and reduces the full
set, so the percentiles stay exact and every rank holds the same result.

    >>> sk = ShardedKLDStats(max_rows_per_rank=8192, device=dev)   # after init_process_group
    >>> res = sk.run(base_shard, quant_shard, token_shard)          # same dict on every rank

Failure detection is on the host. A rank whose own pass fails (the library
returned an error status, a bad argument) still takes the step's one small
collective, the all-gather of row counts, with a count of -1; every rank
then raises :class:`ShardFailure` naming the failed ranks, and the group
stays usable for the next step. A rank that dies or never arrives ends its
peers' next collective with an error after the process group's timeout
(give the group a short one).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

ROW_RECORD_BYTES = 40  # sizeof(kld_row_t)


def shard_bounds(n_rows: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous [start, stop) rows of `rank` when n_rows are split over
    `world` ranks; the first n_rows % world ranks take one row more."""
    if world < 1 or not 0 <= rank < world or n_rows < 0:
        raise ValueError("need world >= 1, 0 <= rank < world, n_rows >= 0")
    base, extra = divmod(n_rows, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


class ShardFailure(RuntimeError):
    """Raised on every rank when the pass failed on one or more ranks;
    `ranks` lists them, `cause` is this rank's own exception (or None)."""

    def __init__(self, ranks: list[int], cause: BaseException | None):
        super().__init__(f"sharded pass failed on rank(s) {ranks}"
                         + (f": {type(cause).__name__}: {cause}" if cause is not None else ""))
        self.ranks = ranks
        self.cause = cause


def gather_counts(n: int, device, group=None) -> list[int]:
    """All-gather one int64 per rank (a row count, or -1 for a failed pass)."""
    t = torch.tensor([n], dtype=torch.int64, device=device)
    sizes = [torch.zeros_like(t) for _ in range(dist.get_world_size(group))]
    dist.all_gather(sizes, t, group=group)
    return [int(c.item()) for c in sizes]


def _checked_counts(n: int, err: BaseException | None, device, group) -> list[int]:
    counts = gather_counts(-1 if err is not None else n, device, group)
    failed = [r for r, c in enumerate(counts) if c < 0]
    if failed:
        raise ShardFailure(failed, err) from err
    return counts


def gather_records(records: torch.Tensor, group=None, counts: list[int] | None = None) -> torch.Tensor:
    """All-gather every rank's [n_r, w] uint8 rows (40-byte records, 64-byte
    vocabulary-slice partials), concatenated in rank order (ranks may hold
    different row counts). Collective: every rank of `group` calls it with
    its own rows, in the same order of calls. `counts`: every rank's row
    count when the caller knows them (skips one small all-gather)."""
    if records.dtype != torch.uint8 or records.dim() != 2:
        raise ValueError("records must be a [n, w] uint8 tensor")
    width = records.shape[1]
    world = dist.get_world_size(group)
    if counts is None:
        counts = gather_counts(records.shape[0], records.device, group)
    elif len(counts) != world or counts[dist.get_rank(group)] != records.shape[0]:
        raise ValueError("counts must list every rank's row count")
    m = max(counts)
    padded = records
    if records.shape[0] != m:
        padded = records.new_zeros((m, width))
        padded[:records.shape[0]] = records
    padded = padded.contiguous()
    if dist.get_backend(group) == "nccl":
        out = records.new_empty((m * world, width))
        dist.all_gather_into_tensor(out, padded, group=group)
        parts = list(out.view(world, m, width))
    else:
        parts = [torch.empty_like(padded) for _ in range(world)]
        dist.all_gather(parts, padded, group=group)
    if all(c == m for c in counts):
        return torch.cat(parts) if len(parts) > 1 else parts[0]
    return torch.cat([p[:c] for p, c in zip(parts, counts)])


class ShardedKLDStats:
    """The statistic over rows sharded across the ranks of `group`: each rank
    runs the row pass on its own rows, the records are gathered, and each rank
    runs the reduction on all of them. `stats` is the per-rank handle (a
    :class:`KLDStats` on this rank's GPU by default)."""

    def __init__(self, max_rows_per_rank: int, device=None, group=None, stats=None):
        if stats is None:
            from . import KLDStats

            stats = KLDStats(max_rows=max_rows_per_rank, device=device)
        self.stats = stats
        self.group = group
        self.max_rows_per_rank = int(max_rows_per_rank)
        self._records = None

    def run(self, base: torch.Tensor, quant: torch.Tensor, token_ids: torch.Tensor | None = None,
            counts: list[int] | None = None) -> dict:
        """Collective. Every rank passes its own [n_r, V] rows (same V, dtype
        and token-id presence on every rank); returns the statistics of all
        ranks' rows. The ranks together must hold at least one row: with
        none, every rank raises ValueError after the same collective steps.

        counts: every rank's row count in rank order, when the caller knows
        them (equal shards, say; the same list on every rank). The step then
        waits on the host once, for the result, instead of also waiting for
        the exchange of row counts before it can enqueue the gather: each
        rank's status travels in a collective enqueued with the gather and is
        read after the result, so a failed rank still makes every rank raise
        ShardFailure (the statistics of that step are discarded)."""
        return self._run(base, quant, token_ids, base.device, host=False, counts=counts)

    def run_host(self, base: torch.Tensor, quant: torch.Tensor, token_ids: torch.Tensor | None = None,
                 device=None, counts: list[int] | None = None) -> dict:
        """As :meth:`run` for a shard held in host memory (pinned for full
        copy bandwidth): the library copies it to `device` (the handle's
        GPU by default) in chunks overlapped with the row pass."""
        if device is None:
            device = getattr(self.stats, "device", base.device)
        return self._run(base, quant, token_ids, torch.device(device), host=True, counts=counts)

    def _run(self, base, quant, token_ids, device, host: bool, counts=None) -> dict:
        n = base.shape[0]
        if n > self.max_rows_per_rank:
            raise ValueError("more rows than max_rows_per_rank")
        world = dist.get_world_size(self.group)
        if counts is not None:
            counts = [int(c) for c in counts]
            if len(counts) != world or counts[dist.get_rank(self.group)] != n or min(counts) < 0:
                raise ValueError("counts must list every rank's row count, this rank's included")
        if self._records is None or self._records.device != device:
            self._records = torch.empty((self.max_rows_per_rank, ROW_RECORD_BYTES), dtype=torch.uint8,
                                        device=device)
        records = self._records[:n]
        err = None
        if n > 0:  # an uneven split can leave a rank without rows; it still gathers and reduces
            try:
                if host:
                    self.stats.run_rows_host(base, quant, token_ids, out=records)
                else:
                    self.stats.run_rows(base, quant, token_ids, out=records)
            except Exception as e:  # reported to every rank below
                err = e
        if counts is None:
            counts = _checked_counts(n, err, device, self.group)
            statuses = None
        else:
            # the status exchange is enqueued, not waited for
            mine = torch.tensor([-1 if err is not None else n], dtype=torch.int64, device=device)
            statuses = [torch.zeros_like(mine) for _ in range(world)]
            dist.all_gather(statuses, mine, group=self.group)
        if sum(counts) == 0:  # every rank sees the same counts: all raise together
            raise ValueError("sharded statistic over zero rows: every rank passed an empty shard")
        gathered = gather_records(records, self.group, counts=counts)
        res = None
        try:
            self.stats.reduce(gathered, gathered.shape[0], token_ids is not None)
            res = self.stats.result()
        except Exception as e:
            if statuses is None or err is None:
                raise
        if statuses is not None:
            got = [int(t.item()) for t in statuses]
            failed = [r for r, c in enumerate(got) if c < 0]
            if failed:
                raise ShardFailure(failed, err) from err
        return res

    def close(self):
        close = getattr(self.stats, "close", None)
        if close is not None:
            close()


class VocabShardedKLDStats:
    """The statistic over vocabulary-sharded logits (tensor-parallel lm_head):
    every rank of `group` holds all N rows but only its column slice
    [col_offset, col_offset + V_r) of a V_total-wide vocabulary, ranks in
    column order. Each rank computes one 64-byte partial per row for its
    slice, the partials are all-gathered (N*64 bytes per rank), and every
    rank merges the G partials of each row and reduces: the same statistics
    on every rank as for the full rows on one GPU. At most 32 ranks."""

    def __init__(self, n_rows: int, device=None, group=None, stats=None):
        if stats is None:
            from . import KLDStats

            stats = KLDStats(max_rows=n_rows, device=device)
        self.stats = stats
        self.group = group

    def run(self, base: torch.Tensor, quant: torch.Tensor, token_ids: torch.Tensor | None,
            col_offset: int, v_total: int) -> dict:
        """Collective. `token_ids` are the full-vocabulary ids (the same on
        every rank, or None on every rank)."""
        n = base.shape[0]
        err = parts = None
        try:
            parts = self.stats.run_partials(base, quant, token_ids, col_offset, v_total)
        except Exception as e:  # reported to every rank below
            err = e
        counts = _checked_counts(n, err, base.device, self.group)
        if any(c != n for c in counts):
            raise ValueError(f"every rank must hold the same rows, got counts {counts}")
        world = len(counts)
        gathered = gather_records(parts, self.group, counts=counts)
        self.stats.merge_partials(gathered.view(world, n, -1), token_ids, v_total)
        return self.stats.result()

    def close(self):
        close = getattr(self.stats, "close", None)
        if close is not None:
            close()
