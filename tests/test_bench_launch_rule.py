"""Host-side check of bench.py's launch accounting: which workloads run the partial last wave
of the long-stream attention kernel split by keys (one combine launch more per call), for a
148-SM B200. 720p: 2280 units = 15 waves + 60, split; 480P: 1000 = 6 waves + 112 and ABot:
264 = 1 wave + 116, tails above half the SMs, not split; short windows (<= 32 key tiles) and
grids of at most one wave never split."""
import importlib.util
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    sys.path.insert(0, ROOT)
    spec = importlib.util.spec_from_file_location("bench_rule", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_split_rule_at_the_benchmark_workloads():
    b = _bench()
    steady = 200
    assert b.attention_launches(b.CONFIGS["720p"], steady, steady, 148) == 2
    assert b.attention_launches(b.CONFIGS["480p"], steady, steady, 148) == 1
    assert b.attention_launches(b.CONFIGS["abot"], steady, steady, 148) == 1
    # the first 720p chunk sees only its own 4 frames (113 tiles): still split
    assert b.attention_launches(b.CONFIGS["720p"], 0, 0, 148) == 2
    # one wave or less: nothing to split
    assert b.attention_launches(b.CONFIGS["720p"], steady, steady, 4096) == 1


def test_split_rule_short_window():
    b = _bench()
    cfg = dict(b.CONFIGS["720p"], gh=4, gw=8, W=6, S=1, C=2)  # 64-token chunks, 192-key window
    # 40 units on 32 SMs leave a tail of 8 (would split), but the window has only 2 key tiles
    assert b.attention_launches(cfg, 10, 10, 32) == 1
