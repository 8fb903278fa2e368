"""GPU parity at the full benchmark sizes, in the launch configuration bench.py times.

The library runs every head of the real workloads (ABot relative RoPE 24 x 2640 x 18480,
LingBot 480P 40 x 6240 x 28080, 720p 40 x 14400 x 64800); the oracle recomputes three
sampled heads (first, middle, last) on sampled query rows (random rows plus every
128-row tile edge and the ragged tail). Checked: the first read and the commit of the
chunk where evictions start and of the last chunk (ring wrapped), and the cache bytes
and slot map of the sampled heads after every chunk from the first eviction on.
"""
import numpy as np
import pytest

from oracle.layer import OracleLayer
from rollout import Config, SampledRollout, sample_rows

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

ABS, REL, SLOTS = OracleLayer.ABSOLUTE, OracleLayer.RELATIVE, OracleLayer.RELATIVE_SLOTS

FULL = [
    # five reference frames become the sinks; evictions start at chunk 5; chunk 6 wraps the ring
    (Config("abot", 20, H=24, grid_h=22, grid_w=40, C=3, W=21, S=5, rope_mode=REL, refs=5, chunks=7, reads=1), (5, 6)),
    # chunk 1 straddles the sink boundary; evictions start at chunk 4
    (Config("480p", 21, H=40, grid_h=30, grid_w=52, C=4, W=18, S=6, rope_mode=ABS, chunks=6, reads=1), (1, 4, 5)),
    # the ABot shape with slot-order relative ids (the five reference sinks keep ids 0..4)
    (Config("abot-slots", 23, H=24, grid_h=22, grid_w=40, C=3, W=21, S=5, rope_mode=SLOTS, refs=5, chunks=7, reads=1), (6,)),
    # 16 heads x 10 query blocks = 160 CTAs, more than the 148 SMs: a second, partial wave
    (Config("many-units", 24, H=16, grid_h=32, grid_w=40, C=2, W=5, S=1, rope_mode=ABS, chunks=5, reads=1), (1, 2, 4)),
    (Config("720p", 22, H=40, grid_h=45, grid_w=80, C=4, W=18, S=6, rope_mode=ABS, chunks=5, reads=1), (4,)),
]


@pytest.mark.parametrize("cfg,checked", FULL, ids=[c.name for c, _ in FULL])
def test_full_size_sampled(cfg, checked):
    heads = [0, cfg.H // 2, cfg.H - 1]
    ro = SampledRollout(cfg, torch, heads)
    rows = sample_rows(cfg.Lq, seed=cfg.cfg_id)
    stats = []
    for chunk in range(cfg.chunks):
        ro.run_chunk(chunk, rows=rows if chunk in checked else None, stats=stats)
        if chunk >= min(checked):
            torch.cuda.synchronize()
            ro.check_cache()
    assert len(stats) == 2 * len(checked)
    assert ro.h.poll_device_status() == 0
    ro.h.close()
