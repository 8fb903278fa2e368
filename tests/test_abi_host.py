"""The C-ABI library on the host, without a GPU.

* librkv.so loads and exports every function include/rkv.h declares;
* the host planner (rkv_plan_window) names exactly the frames the oracle's
  literal shift-left cache holds, in the same logical order, in ring slots that
  follow slot(f) = f (f < S), S + (f - S) mod (W - S), in at most four segments;
* argument, order and capacity errors come back as codes before any device work.
"""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

rkv = pytest.importorskip("rolling_kv_chunked_b200")
from oracle.cache import RollingCache  # noqa: E402


def _declared():
    text = open(os.path.join(ROOT, "include", "rkv.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rkv_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 16
    lib = ctypes.CDLL(rkv.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(rkv.EXPORTED)


def test_synth_twin_library_loads():
    lib = ctypes.CDLL(os.path.join(ROOT, "synth", "libsynth.so"))
    assert hasattr(lib, "synth_fill_normal_bf16")


def _frames_from_plan(segs, W, S):
    R = W - S
    frames = []
    for src, first, n, f0 in segs:
        for i in range(n):
            f = f0 + i
            if src == 0:
                slot = first + i
                assert slot == (f if f < S else S + (f - S) % R), (f, slot)
            else:
                assert first + i == f - segs[-1][3]
            frames.append(f)
    return frames


@pytest.mark.parametrize("W,S,C,refs", [(6, 2, 2, 0), (21, 5, 3, 5), (18, 6, 4, 0), (5, 0, 1, 0),
                                        (7, 3, 4, 0), (18, 6, 4, 2), (9, 1, 8, 0), (256, 6, 4, 0)])
def test_planner_matches_oracle_cache(W, S, C, refs):
    cache = RollingCache(W, S)
    committed = 0
    if refs:
        cache.append(list(range(refs)))
        committed = refs
    for _ in range(200 if W < 100 else 80):
        segs = rkv.plan_window(W, S, committed, C, committed)
        assert 1 <= len(segs) <= 4
        assert segs[-1][0] == 1 and segs[-1][2] == C and segs[-1][3] == committed
        assert _frames_from_plan(segs, W, S) == cache.after_append(list(range(committed, committed + C)))
        cache.append(list(range(committed, committed + C)))
        committed += C


def test_planner_matches_oracle_cache_mixed_chunk_sizes():
    """Random windows and random sequences of chunk sizes (every size the window takes), the
    plan of each chunk against the oracle's literal cache (hypothesis, derandomized)."""
    hypothesis = pytest.importorskip("hypothesis")
    st = hypothesis.strategies

    @hypothesis.settings(max_examples=300, deadline=None, derandomize=True)
    @hypothesis.given(st.integers(1, 40).flatmap(
        lambda W: st.tuples(st.just(W), st.integers(0, W - 1)).flatmap(
            lambda ws: st.tuples(st.just(ws[0]), st.just(ws[1]),
                                 st.lists(st.integers(1, ws[0] - ws[1]), min_size=1, max_size=40)))))
    def check(args):
        W, S, sizes = args
        cache = RollingCache(W, S)
        committed = 0
        for C in sizes:
            segs = rkv.plan_window(W, S, committed, C, committed)
            assert 1 <= len(segs) <= 4
            assert segs[-1][0] == 1 and segs[-1][2] == C and segs[-1][3] == committed
            assert _frames_from_plan(segs, W, S) == cache.after_append(list(range(committed, committed + C)))
            cache.append(list(range(committed, committed + C)))
            committed += C

    check()


def test_planner_errors():
    with pytest.raises(rkv.RkvError) as e:
        rkv.plan_window(6, 2, 4, 2, 3)
    assert e.value.code == rkv.ERR_ORDER
    with pytest.raises(rkv.RkvError) as e:
        rkv.plan_window(6, 2, 0, 5, 0)
    assert e.value.code == rkv.ERR_CAPACITY
    for bad in [(0, 0, 0, 1, 0), (6, 6, 0, 1, 0), (6, 2, 0, 0, 0), (6, -1, 0, 1, 0)]:
        with pytest.raises(rkv.RkvError) as e:
            rkv.plan_window(*bad)
        assert e.value.code == rkv.ERR_ARG


def test_create_rejects_bad_arguments_before_touching_the_device():
    lib = ctypes.CDLL(rkv.LIB_PATH)
    lib.rkv_create.argtypes = [ctypes.c_int] * 7 + [ctypes.POINTER(ctypes.c_void_p)]
    h = ctypes.c_void_p()
    assert lib.rkv_create(1, 2, 64, 16, 6, 2, 0, ctypes.byref(h)) == rkv.ERR_UNSUPPORTED   # d != 128
    assert lib.rkv_create(1, 2, 128, 16, 257, 2, 0, ctypes.byref(h)) == rkv.ERR_UNSUPPORTED
    assert lib.rkv_create(1, 2, 128, 16, 6, 6, 0, ctypes.byref(h)) == rkv.ERR_ARG           # sink >= window
    assert lib.rkv_create(0, 2, 128, 16, 6, 2, 0, ctypes.byref(h)) == rkv.ERR_ARG
    assert lib.rkv_create(1, 2, 128, 16, 6, 2, 7, ctypes.byref(h)) == rkv.ERR_ARG           # rope mode
    assert lib.rkv_create(1, 2, 128, 16, 6, 2, 3, ctypes.byref(h)) == rkv.ERR_ARG
    assert lib.rkv_create(1, 2, 128, 16, 6, 2, -1, ctypes.byref(h)) == rkv.ERR_ARG
    assert lib.rkv_create(1, 2, 128, 16, 6, 2, 0, None) == rkv.ERR_ARG
    assert h.value is None


def test_flow_rejects_misaligned_pointers():
    lib = ctypes.CDLL(rkv.LIB_PATH)
    f = lib.rkv_flow_x0_renoise
    f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_double] * 2 + [ctypes.c_void_p] * 2 + [ctypes.c_longlong,
                                                                                         ctypes.c_void_p]
    assert f(None, None, None, 1.0, 0.5, None, None, 0, None) == rkv.OK          # nothing to do
    assert f(0x1000, 0x1002, 0x1000, 1.0, 0.5, 0x1000, 0x1000, 8, None) == rkv.ERR_ARG
    assert f(0x1000, 0x1000, None, 1.0, 0.5, 0x1000, 0x1000, 8, None) == rkv.ERR_ARG   # eps needed
    assert f(None, None, None, 1.0, 0.5, None, None, -1, None) == rkv.ERR_ARG


def test_status_strings():
    for code in range(8):
        assert rkv.status_string(code)
    assert "unknown" in rkv.status_string(99)
