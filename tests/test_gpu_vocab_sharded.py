"""Vocabulary-sharded rows (a tensor-parallel lm_head leaves each GPU with a
column slice of the logits): the full rows are cut into G column slices,
each slice's partials come from kld_stats_run_partials, the [G][N]
partials are merged by kld_stats_merge_partials, and the records and
statistics must match the fp64 oracle on the full rows (the same bar as the
whole-row path; argmax indices bit-exact across slice boundaries). Slices
run one after another on one GPU here; the multi-process gather is the
gather the row-sharded path uses, also run through a one-rank NCCL group."""
import datetime
import math
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from logit_kl_divergence_b200 import KLDStats, rows_view, synth
from logit_kl_divergence_b200.sharded import VocabShardedKLDStats

from gpu_helpers import ODT, assert_rows_match, assert_stats_match

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _bounds(v, g, ragged):
    if not ragged:
        return [(v * k // g, v * (k + 1) // g) for k in range(g)]
    cuts = sorted(set([0, v] + [int(v * (k + 0.37) / g) + (k % 3) for k in range(1, g)]))
    return list(zip(cuts[:-1], cuts[1:]))


def _sharded(b, q, tok, bounds):
    n, v = b.shape
    st = KLDStats(max_rows=n, device=DEV)
    parts = torch.empty((len(bounds), n, 64), dtype=torch.uint8, device=DEV)
    bd, qd = b.to(DEV), q.to(DEV)
    td = None if tok is None else tok.to(DEV)
    for g, (c0, c1) in enumerate(bounds):
        st.run_partials(bd[:, c0:c1].contiguous(), qd[:, c0:c1].contiguous(), td, c0, v, out=parts[g])
    st.merge_partials(parts, td, v)
    res = st.result()
    rec = {k: t.cpu().numpy() for k, t in rows_view(st.records()).items()}
    rec["flags"] = rec["flags"].astype(np.uint32)
    st.close()
    return rec, res


def _parity(b, q, tok, dt, bounds):
    g_rows, gres = _sharded(b, q, tok, bounds)
    o_rows, ores = oracle.run(b, q, tok, ODT[dt])
    assert_rows_match(g_rows, o_rows)
    assert_stats_match(gres, ores)
    return g_rows


@pytest.mark.parametrize("dt", [synth.F32, synth.BF16])
@pytest.mark.parametrize("G,ragged", [(1, False), (2, False), (3, True), (4, False), (8, True), (32, True)])
def test_vocab_slices_match_full_rows(G, ragged, dt):
    w = synth.make_recipe("ctx", n=160, v=151936, dtype=dt, seed=60 + G)
    _parity(w.base, w.quant, w.token_ids, dt, _bounds(151936, G, ragged))


def test_vocab_slices_edge_rows_and_small_n():
    # near-one-hot rows, ties (lowest global index wins across slices),
    # padding masks that fill the last slice, constant shifts; 5 rows
    for n in (5, 300):
        w = synth.make_recipe("edge", n=n, v=131072, dtype=synth.F32, seed=n)
        _parity(w.base, w.quant, w.token_ids, synth.F32, _bounds(131072, 5, True) if n == 5 else
                [(0, 65536), (65536, 130048), (130048, 131072)])


def test_vocab_slices_special_values_and_token_placement():
    n, v = 8, 40000
    g = torch.Generator().manual_seed(13)
    b = torch.randn((n, v), generator=g)
    q = b + 0.2 * torch.randn((n, v), generator=g)
    b[0, 35000] = math.nan                 # NaN in the last slice only
    b[1, :20000] = -math.inf               # first slices hold no base mass
    q[2, 30001] = -math.inf                # KL = +inf from a later slice
    b[3, [10000, 30000]] = 50.0            # tie across slices: lowest index
    q[4, :] = -math.inf
    q[4, 39999] = 1.0                      # one finite quant entry, last column
    tok = torch.tensor([1, 5, 30001, 10000, 39999, 19999, 20000, 40000], dtype=torch.int32)
    bounds = [(0, 10000), (10000, 20000), (20000, 30001), (30001, 40000)]
    rows = _parity(b.contiguous(), q.contiguous(), tok, synth.F32, bounds)
    assert rows["amax_b"][3] == 10000 and rows["amax_q"][4] == 39999
    assert rows["flags"][7] & oracle.ROW_BAD_TOKEN


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_vocab_sharded_class_through_a_one_rank_nccl_group():
    torch.cuda.set_device(DEV)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=DEV)
    try:
        w = synth.make_recipe("ctx", n=64, v=32000, dtype=synth.BF16, seed=3, device=DEV)
        vs = VocabShardedKLDStats(64, device=DEV)
        a = vs.run(w.base, w.quant, w.token_ids, 0, 32000)
        vs.close()
        st = KLDStats(max_rows=64, device=DEV)
        st.run(w.base, w.quant, w.token_ids)
        b = st.result()
        st.close()
        for k in ("n_valid", "top1_agree", "n_nll", "flags_or"):
            assert a[k] == b[k], k
        # whole-row partials against the split-row launch kld_stats_run uses
        # at 64 rows: the same rows summed in another order
        for k in ("mean_kld", "median_kld", "max_kld", "mean_nll", "rms_dp"):
            assert abs(a[k] - b[k]) <= 1e-6 * abs(b[k]) + 1e-12, (k, a[k], b[k])
    finally:
        dist.destroy_process_group()
