"""Failure detection on the GPU without a fault: every device wait of the
kernels (ring-slot barriers, cluster barriers, split-row tickets) is bounded
and reports a timeout in the launch's error word instead of hanging. The
self-test kernel waits on an mbarrier that nothing ever completes; the wait
must run out after its short limit (or end on the abort flag a second warp
raises), the call must return KLD_ERR_TIMEOUT, and the context must still
compute correct statistics afterwards."""
import pytest
import torch

import oracle
from logit_kl_divergence_b200 import KLDStats, _lib, selftest_bounded_wait, synth

from gpu_helpers import ODT, assert_stats_match

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _healthy_run():
    w = synth.make_recipe("ctx", n=64, v=32000, dtype=synth.F32, seed=77)
    with KLDStats(max_rows=64, device=DEV) as st:
        st.run(w.base.to(DEV), w.quant.to(DEV), w.token_ids.to(DEV))
        res = st.result()
    _, ores = oracle.run(w.base, w.quant, w.token_ids, ODT[synth.F32])
    assert_stats_match(res, ores)


@pytest.mark.parametrize("limit_ns", [1_000_000, 20_000_000])
def test_unsatisfied_wait_times_out_and_context_survives(limit_ns):
    st, waited = selftest_bounded_wait(0, limit_ns)
    assert st == _lib.KLD_ERR_TIMEOUT
    # gave up no earlier than the limit and well before the 2 s default
    assert limit_ns <= waited < limit_ns + 200_000_000, waited
    _healthy_run()


def test_abort_flag_ends_the_wait_early():
    st, waited = selftest_bounded_wait(0, 1_000_000_000, use_abort=True)
    assert st == _lib.KLD_ERR_TIMEOUT
    assert 1_000_000 <= waited < 100_000_000, waited
    _healthy_run()


def test_selftest_argument_checks():
    with pytest.raises(_lib.KLDError):
        selftest_bounded_wait(0, 10)               # below the 1 us floor
    with pytest.raises(_lib.KLDError):
        selftest_bounded_wait(-1, 1_000_000)
