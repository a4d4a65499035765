"""Property test of the C ABI's configuration contract (host only, no device needed): the library
accepts exactly the layer configs and token counts that include/beam_moe.h documents as valid."""
import ctypes
import shutil

import pytest

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import given, settings, strategies as st  # noqa: E402

import group_limited_routing_router_b200 as bm  # noqa: E402
from group_limited_routing_router_b200 import build as bm_build  # noqa: E402

_L = None


def lib():
    """The library, built on first use; the test skips where neither it nor nvcc is available."""
    global _L
    if _L is None:
        import os
        if not os.path.exists(bm_build.LIB) and shutil.which(bm_build.nvcc()) is None:
            pytest.skip("libbeam_moe.so is not built and nvcc is not available")
        bm_build.build()
        _L = bm.lib()
    return _L


def documented_valid(H, I, E, G, kg, k, gn, scale) -> bool:
    if not (64 <= H <= 65536 and H % 64 == 0 and 64 <= I <= 65536 and I % 64 == 0):
        return False
    if not (1 <= E <= 256 and 1 <= G <= 32 and E % G == 0):
        return False
    per = E // G
    return 1 <= kg <= G and 1 <= k <= min(16, kg * per) and 1 <= gn <= min(8, per) and scale == scale


def documented_valid_T(T, k) -> bool:
    return 0 <= T <= (1 << 24) and T * k < (1 << 31)


near = lambda lo, hi: st.integers(lo - 3, hi + 3)  # noqa: E731  ranges straddling the limits


@settings(max_examples=400, deadline=None)
@given(H=st.sampled_from([0, 32, 63, 64, 96, 128, 320, 5120, 65536, 65600]),
       I=st.sampled_from([0, 64, 100, 192, 2560, 65536, 70000]),
       E=near(1, 256), G=st.sampled_from([1, 2, 3, 4, 8, 16, 32, 33, 64]),
       kg=near(1, 32), k=near(1, 16), gn=near(1, 8),
       scale=st.sampled_from([2.5, 1.0, 0.0, float("nan")]),
       T=st.sampled_from([-1, 0, 1, 77, 4096, 1 << 24, (1 << 24) + 1]))
def test_workspace_size_and_route_follow_the_documented_ranges(H, I, E, G, kg, k, gn, scale, T):
    c = bm.BeamMoeConfig(H, I, E, G, kg, k, gn, scale)
    valid = documented_valid(H, I, E, G, kg, k, gn, scale)
    L = lib()
    size = L.beam_moe_workspace_size(ctypes.byref(c), T, bm.WS_FORWARD)
    if not valid or not documented_valid_T(T, k):
        assert size == 0
    elif T > 0:
        assert size > 0
    # beam_moe_route only where it returns before any device work (an invalid config or T, or T = 0):
    # the placeholder pointers are never dereferenced, and nothing is launched on any machine
    p = ctypes.c_void_p(4096)
    if not valid:
        assert L.beam_moe_route(ctypes.byref(c), T, p, p, None, p, p, None) == bm.ERR_INVALID_CONFIG
    elif not documented_valid_T(T, k):
        assert L.beam_moe_route(ctypes.byref(c), T, p, p, None, p, p, None) == bm.ERR_INVALID_ARG
    elif T == 0:
        assert L.beam_moe_route(ctypes.byref(c), T, p, p, None, p, p, None) == bm.OK
