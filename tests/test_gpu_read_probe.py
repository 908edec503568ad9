"""kld_stats_read_probe, the read-bandwidth probe the benchmark sets beside
the row pass: it streams two device buffers into shared memory with the row
pass's bulk copies, completes without a device error (its waits are bounded
and would report one), covers sizes that end in a partial tile, and rejects
sizes and addresses the bulk copies cannot take."""
import pytest
import torch

from logit_kl_divergence_b200 import KLDStats, _lib, synth

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def test_probe_streams_buffers_and_leaves_no_device_error():
    st = KLDStats(max_rows=64, device=DEV)
    try:
        a = torch.zeros(256 << 20, dtype=torch.uint8, device=DEV)
        b = torch.ones(256 << 20, dtype=torch.uint8, device=DEV)
        stream = torch.cuda.current_stream(DEV)
        for _ in range(2):
            st.read_probe(a, b)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        st.read_probe(a, b)
        e1.record(stream)
        stream.synchronize()
        ms = e0.elapsed_time(e1)
        gbs = 2 * a.numel() / (ms / 1000.0) / 1e9
        assert 100.0 < gbs < 20000.0, gbs  # plausible for a B200, and not skipped work
        # sizes ending in a partial tile, and the smallest one
        for nbytes in (16 * 12345, 32 * 1024 + 16, 16):
            st.read_probe(a[:nbytes], b[:nbytes])
        # a normal run afterwards: no device error left behind by the probe
        w = synth.make_recipe("small", n=8, v=4096, dtype=synth.F32, seed=3)
        st.run(w.base.to(DEV), w.quant.to(DEV), w.token_ids.to(DEV))
        res = st.result()
        assert res["device_error"] == 0 and res["status"] == _lib.KLD_OK
        with pytest.raises(_lib.KLDError):
            st.read_probe(a[:100], b[:100])   # not a multiple of 16 bytes
        with pytest.raises(_lib.KLDError):
            st.read_probe(a[1:1 + 1024], b[:1024])   # misaligned start
        with pytest.raises(ValueError):
            st.read_probe(a[:1024], b[:2048])   # different sizes
    finally:
        st.close()
