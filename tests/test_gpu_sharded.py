"""The row-sharded path on a real GPU through NCCL: a one-rank NCCL group
(every GPU run here has one GPU) exercises the all_gather_into_tensor branch
of gather_records and ShardedKLDStats end to end; the result must equal the
single-handle run bit for bit, since the rows and their order are the same.
The multi-rank logic is covered by the gloo tests on the CPU."""
import datetime
import math
import socket

import pytest
import torch
import torch.distributed as dist

from logit_kl_divergence_b200 import KLDStats, synth
from logit_kl_divergence_b200.sharded import ShardedKLDStats, gather_records

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture
def nccl_group():
    torch.cuda.set_device(DEV)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=DEV)
    yield
    dist.destroy_process_group()


def test_sharded_run_equals_single_handle_run(nccl_group):
    w = synth.make_recipe("ctx", n=300, v=32001, dtype=synth.BF16, seed=31, device=DEV)
    rec = torch.arange(5 * 40, dtype=torch.uint8, device=DEV).view(5, 40)
    assert torch.equal(gather_records(rec), rec)
    assert torch.equal(gather_records(rec, counts=[5]), rec)
    sk = ShardedKLDStats(max_rows_per_rank=300, device=DEV)
    sk.stats.set_timing(True)
    a = sk.run(w.base, w.quant, w.token_ids)
    # the row pass and the gather + reduction of a sharded step are timed
    # through the handle (kld_stats_run_rows then kld_stats_reduce)
    row_ms, red_ms = sk.stats.timing()
    assert 0.0 < row_ms < 100.0 and 0.0 < red_ms < 100.0
    # the same shard from pinned host memory (kld_stats_run_rows_host)
    hb, hq, ht = (t.cpu().pin_memory() for t in (w.base, w.quant, w.token_ids))
    c = sk.run_host(hb, hq, ht)
    sk.close()
    st = KLDStats(max_rows=300, device=DEV)
    st.run(w.base, w.quant, w.token_ids)
    b = st.result()
    st.close()
    for res in (a, c):
        for k in b:
            x, y = res[k], b[k]
            assert x == y or (isinstance(x, float) and math.isnan(x) and math.isnan(y)), k
