"""Work-unit schedule of the two-problem GEMM launch (dgrad and wgrad of a
layer in one launch), through the host-only entry point
puro_fp8_test_schedule (no GPU needed).

Longest-processing-time list scheduling: units sorted by cost (K blocks + 2),
longest first, each to the least-loaded cluster.  Checks: every unit is
scheduled exactly once; each cluster runs its units longest first; the final
loads differ by at most one unit's cost (the defining property of greedy list
scheduling on sorted jobs); a small case matches a schedule worked by hand;
bad arguments are refused."""
import numpy as np
import pytest


@pytest.fixture(scope="module")
def lib():
    from fp8_block_scaled_13_b200 import build, _lib
    build.build()
    return _lib


def _schedule(lib, u0, k0, u1, k1, clusters):
    off = np.zeros(clusters + 1, dtype=np.int32)
    units = np.zeros(max(u0 + u1, 1), dtype=np.int32)
    st = lib.puro_fp8_test_schedule(u0, k0, u1, k1, clusters, off.ctypes.data, units.ctypes.data)
    assert st == 0, st
    assert off[0] == 0 and off[clusters] == u0 + u1
    return [units[off[c]:off[c + 1]].tolist() for c in range(clusters)]


@pytest.mark.parametrize("u0,k0,u1,k1,clusters", [
    (256, 24, 96, 64, 74),      # QKV backward: dgrad 32x8 tiles (K = 3072), wgrad 12x8 tiles (K = 8192)
    (256, 16, 64, 64, 74),      # O-projection backward: dgrad (K = 2048), wgrad 8x8 tiles (K = 8192)
    (10, 3, 0, 0, 4),           # one problem empty
    (0, 0, 5, 7, 3),
    (1, 1, 1, 1, 74),           # fewer units than clusters
    (2041, 2, 7, 100, 128),     # the largest schedule
])
def test_schedule_invariants(lib, u0, k0, u1, k1, clusters):
    lists = _schedule(lib, u0, k0, u1, k1, clusters)

    def cost(u):
        return (k0 if u < u0 else k1) + 2

    assert sorted(u for l in lists for u in l) == list(range(u0 + u1))
    for l in lists:
        c = [cost(u) for u in l]
        assert c == sorted(c, reverse=True)
    loads = [sum(cost(u) for u in l) for l in lists]
    if u0 + u1:
        assert max(loads) - min(loads) <= max(cost(u) for u in range(u0 + u1))


def test_schedule_worked_example(lib):
    # units 0-2 cost 4 + 2 = 6, units 3-4 cost 10 + 2 = 12, two clusters:
    # 3 -> c0, 4 -> c1, 0 -> c0 (tie at 12: lower index), 1 -> c1, 2 -> c0 (tie at 18)
    assert _schedule(lib, 3, 4, 2, 10, 2) == [[3, 0, 2], [4, 1]]


def test_schedule_argument_errors(lib):
    off = np.zeros(200, dtype=np.int32)
    units = np.zeros(4096, dtype=np.int32)
    f = lib.puro_fp8_test_schedule
    assert f(4, 1, 4, 1, 2, None, units.ctypes.data) == -1
    assert f(4, 1, 4, 1, 0, off.ctypes.data, units.ctypes.data) == -3
    assert f(4, 1, 4, 1, 129, off.ctypes.data, units.ctypes.data) == -3
    assert f(2048, 1, 1, 1, 8, off.ctypes.data, units.ctypes.data) == -3
    assert f(-1, 1, 4, 1, 8, off.ctypes.data, units.ctypes.data) == -3


def test_schedule_invariants_random(lib):
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=300, deadline=None)
    @given(u0=st.integers(0, 1024), k0=st.integers(0, 200), u1=st.integers(0, 1024),
           k1=st.integers(0, 200), clusters=st.integers(1, 128))
    def check(u0, k0, u1, k1, clusters):
        test_schedule_invariants(lib, u0, k0, u1, k1, clusters)

    check()
