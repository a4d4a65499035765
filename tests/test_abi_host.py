"""C-ABI checks that need no GPU: the library loads, exports every entry point the header declares,
and rejects bad arguments on the host before any CUDA call."""
import ctypes

import pytest

import group_limited_routing_router_b200 as bm
from group_limited_routing_router_b200 import build as bm_build


@pytest.fixture(scope="module")
def L():
    bm_build.build()
    return bm.lib()


def test_exports_every_declared_symbol(L):
    names = bm.declared_symbols()
    assert set(names) >= {"beam_moe_route", "beam_moe_permute", "beam_moe_experts", "beam_moe_forward",
                          "beam_moe_workspace_size", "beam_moe_device_status", "beam_moe_strerror",
                          "beam_moe_selftest_timeout"}
    for n in names:
        assert hasattr(L, n), n


def test_strerror_covers_codes(L):
    for code in range(0, 10):
        s = bm.strerror(code)
        assert s and s != "unknown error code"
    assert bm.strerror(12345) == "unknown error code"


def _cfg(**kw):
    d = dict(hidden=5120, inter=2560, n_experts=256, n_groups=8, topk_groups=4, topk=8, group_topn=2,
             routed_scale=2.5)
    d.update(kw)
    return bm.LayerConfig(**d).c()


def test_workspace_sizes(L):
    c = _cfg()
    assert bm.workspace_size(c, 0, bm.WS_ROUTE) == 0
    f = [bm.workspace_size(c, T, bm.WS_FORWARD) for T in (1, 256, 4096, 65536)]
    assert all(b > a for a, b in zip(f, f[1:]))
    # forward holds h (bf16) and the fp32 expert outputs for all T*k rows
    T = 4096
    R = T * 8
    assert f[2] >= R * 2560 * 2 + R * 5120 * 4
    assert bm.workspace_size(c, T, bm.WS_EXPERTS) < f[2]
    assert bm.workspace_size(c, T, bm.WS_PERMUTE) >= 16 * 256 * 4
    assert bm.workspace_size(c, -1, bm.WS_FORWARD) == 0
    assert bm.workspace_size(c, 1 << 25, bm.WS_FORWARD) == 0
    assert bm.workspace_size(c, 4, 99) == 0
    assert bm.workspace_size(_cfg(hidden=100), 4, bm.WS_FORWARD) == 0


def test_screened_route_workspace(L):
    """The screened router's scratch: none below 2048 tokens (the direct router runs); from 2048 the
    three bf16 planes of W_r, the split partial projections, the exact-path list and its projections,
    the per-expert buckets of the screened picks and their exact projections; the forward workspace
    holds it."""
    c = _cfg()
    E, H = 256, 5120
    assert bm.workspace_size(c, 2047, bm.WS_ROUTE_SCREENED) == 0
    for T in (2048, 4096, 65536):
        n = bm.workspace_size(c, T, bm.WS_ROUTE_SCREENED)
        # planes + >= one split + the listed tokens' projections + the list + the per-expert buckets of
        # the screened picks + their exact projections
        assert n >= 3 * E * H * 2 + T * E * 4 * 2 + T * 4 + T * E * 4 + T * 8 * 4
        assert bm.workspace_size(c, T, bm.WS_FORWARD) > n
    assert bm.workspace_size(_cfg(topk=9, topk_groups=8), 4096, bm.WS_ROUTE_SCREENED) == 0  # k > 8: direct


@pytest.mark.parametrize("bad", [dict(hidden=96), dict(inter=0), dict(n_experts=257), dict(n_groups=3),
                                 dict(topk_groups=9), dict(topk=17), dict(topk=0), dict(group_topn=0),
                                 dict(group_topn=9), dict(n_groups=64, n_experts=256),
                                 dict(routed_scale=float("nan"))])
def test_invalid_config_rejected_on_host(L, bad):
    c = _cfg(**bad)
    p = ctypes.c_void_p(4096)  # never dereferenced: validation fails first
    assert L.beam_moe_route(ctypes.byref(c), 4, p, p, None, p, p, None) == bm.ERR_INVALID_CONFIG
    assert L.beam_moe_forward(ctypes.byref(c), 4, p, p, None, p, p, p, p, None, None, p, 1 << 40, None) == \
        bm.ERR_INVALID_CONFIG
    assert L.beam_moe_experts(ctypes.byref(c), 4, p, p, p, p, p, p, p, p, 1 << 40, None) == bm.ERR_INVALID_CONFIG


def test_argument_errors_on_host(L):
    c = _cfg()
    p = ctypes.c_void_p(4096)
    mis = ctypes.c_void_p(4104)
    assert L.beam_moe_route(None, 4, p, p, None, p, p, None) == bm.ERR_NULL
    assert L.beam_moe_route(ctypes.byref(c), 4, None, p, None, p, p, None) == bm.ERR_NULL
    assert L.beam_moe_route(ctypes.byref(c), 4, mis, p, None, p, p, None) == bm.ERR_MISALIGNED
    assert L.beam_moe_route(ctypes.byref(c), -1, p, p, None, p, p, None) == bm.ERR_INVALID_ARG
    assert L.beam_moe_route(ctypes.byref(c), 0, p, p, None, p, p, None) == bm.OK  # T = 0: nothing to do
    need = bm.workspace_size(c, 64, bm.WS_FORWARD)
    assert L.beam_moe_forward(ctypes.byref(c), 64, p, p, None, p, p, p, p, None, None, p, need - 1, None) == \
        bm.ERR_WORKSPACE_TOO_SMALL
    assert L.beam_moe_forward(ctypes.byref(c), 64, p, p, None, p, p, mis, p, None, None, p, need, None) == \
        bm.ERR_MISALIGNED
    assert L.beam_moe_forward(ctypes.byref(c), 64, p, p, None, p, p, p, p, None, None, None, need, None) == \
        bm.ERR_NULL
    assert L.beam_moe_forward(ctypes.byref(c), 0, p, p, None, p, p, p, p, None, None, None, 0, None) == bm.OK
    need_e = bm.workspace_size(c, 64, bm.WS_EXPERTS)
    assert L.beam_moe_experts(ctypes.byref(c), 64, p, p, p, p, p, p, p, p, need_e - 256, None) == \
        bm.ERR_WORKSPACE_TOO_SMALL
    need_p = bm.workspace_size(c, 64, bm.WS_PERMUTE)
    assert L.beam_moe_permute(ctypes.byref(c), 64, p, p, p, p, p, p, need_p - 1, None) == \
        bm.ERR_WORKSPACE_TOO_SMALL
    assert L.beam_moe_selftest_timeout(0, None) == bm.ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors(L):
    import torch
    x = torch.zeros(4, 5120, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        bm.route(bm.BEAM_LAYER, x, torch.zeros(256, 5120))


def test_block_rejects_bad_sublayer_on_host(L):
    c = _cfg()
    p = ctypes.c_void_p(4096)
    for step, eps, hidden in ((1, 1e-6, 5120), (7, -1.0, 5120), (7, float("nan"), 5120), (7, 1e-6, 65536)):
        cc = _cfg(hidden=hidden)
        sub = bm.BeamMoeSublayer(4096, 4096, eps, step)
        assert L.beam_moe_block_forward(ctypes.byref(cc), ctypes.byref(sub), 4, p, p, None, p, p, p, p, None, None,
                                        None, p, 1 << 40, None) == bm.ERR_INVALID_CONFIG
    assert L.beam_moe_block_forward(ctypes.byref(c), None, 4, p, p, None, p, p, p, p, None, None, None, p, 1 << 40,
                                    None) == bm.ERR_NULL
    assert bm.workspace_size(c, 4096, bm.WS_BLOCK) == bm.workspace_size(c, 4096, bm.WS_FORWARD) + 4096 * 5120 * 2


def test_fp8_entry_points_check_arguments_on_host(L):
    c = _cfg()
    p, mis = 4096, 4104
    need = bm.workspace_size(c, 64, bm.WS_FORWARD)
    good = bm.BeamMoeFp8Experts(p, p, p, p, p, p)
    q = ctypes.c_void_p(p)
    assert L.beam_moe_forward_fp8(ctypes.byref(c), 64, q, q, None, None, q, None, None, q, need, None, None) == \
        bm.ERR_NULL
    assert L.beam_moe_experts_fp8(ctypes.byref(c), 64, q, q, q, None, q, q, need, None) == bm.ERR_NULL
    for i in range(6):  # each of the six weight / scale pointers
        vals = [p] * 6
        vals[i] = 0
        w8 = bm.BeamMoeFp8Experts(*vals)
        assert L.beam_moe_forward_fp8(ctypes.byref(c), 64, q, q, None, ctypes.byref(w8), q, None, None, q, need,
                                      None, None) == bm.ERR_NULL
        vals[i] = mis
        w8 = bm.BeamMoeFp8Experts(*vals)
        assert L.beam_moe_forward_fp8(ctypes.byref(c), 64, q, q, None, ctypes.byref(w8), q, None, None, q, need,
                                      None, None) == bm.ERR_MISALIGNED
        assert L.beam_moe_experts_fp8(ctypes.byref(c), 64, q, q, q, ctypes.byref(w8), q, q, need, None) == \
            bm.ERR_MISALIGNED
    assert L.beam_moe_forward_fp8(ctypes.byref(c), 64, q, q, None, ctypes.byref(good), q, None, None, q, need - 1,
                                  None, None) == bm.ERR_WORKSPACE_TOO_SMALL
    bad = _cfg(hidden=96)
    assert L.beam_moe_experts_fp8(ctypes.byref(bad), 64, q, q, q, ctypes.byref(good), q, q, need, None) == \
        bm.ERR_INVALID_CONFIG
    # events: NULL (no profiling) or 7 valid handles
    ev = (ctypes.c_void_p * 7)()
    assert L.beam_moe_forward_fp8(ctypes.byref(c), 64, q, q, None, ctypes.byref(good), q, None, None, q, need,
                                  None, ev) == bm.ERR_NULL
    assert L.beam_moe_forward_fp8(ctypes.byref(c), 0, q, q, None, ctypes.byref(good), q, None, None, None, 0,
                                  None, None) == bm.OK


def test_fp8_binding_refuses_bad_inputs_on_host(L):
    import torch
    x = torch.zeros(4, 5120, dtype=torch.bfloat16)
    with pytest.raises(KeyError):
        bm._fp8_experts(bm.BEAM_LAYER.c(), {"q_gate": None})
    with pytest.raises(TypeError):
        bm.forward_fp8(bm.BEAM_LAYER, x, torch.zeros(256, 5120), None, {})
    with pytest.raises(TypeError):
        bm.experts_fp8(bm.BEAM_LAYER, x, torch.zeros(4, 8, dtype=torch.int32), torch.zeros(4, 8), {})


def test_nvfp4_entry_points_check_arguments_on_host(L):
    c = _cfg()
    p, mis = 4096, 4104
    need = bm.workspace_size(c, 64, bm.WS_FORWARD)
    q = ctypes.c_void_p(p)
    good = bm.BeamMoeNvfp4Experts(*([p] * 9))
    assert L.beam_moe_forward_nvfp4(ctypes.byref(c), 64, q, q, None, None, q, None, None, q, need, None, None) == \
        bm.ERR_NULL
    assert L.beam_moe_experts_nvfp4(ctypes.byref(c), 64, q, q, q, None, q, q, need, None) == bm.ERR_NULL
    for i in range(9):  # each code, scale and per-matrix-scale pointer
        vals = [p] * 9
        vals[i] = 0
        w4 = bm.BeamMoeNvfp4Experts(*vals)
        assert L.beam_moe_forward_nvfp4(ctypes.byref(c), 64, q, q, None, ctypes.byref(w4), q, None, None, q, need,
                                        None, None) == bm.ERR_NULL
        vals[i] = mis + (2 if i % 3 == 2 else 0)  # codes / scale codes: 16-byte rule; per-matrix scales: 4-byte
        w4 = bm.BeamMoeNvfp4Experts(*vals)
        assert L.beam_moe_experts_nvfp4(ctypes.byref(c), 64, q, q, q, ctypes.byref(w4), q, q, need, None) == \
            bm.ERR_MISALIGNED
    assert L.beam_moe_forward_nvfp4(ctypes.byref(c), 64, q, q, None, ctypes.byref(good), q, None, None, q, need - 1,
                                    None, None) == bm.ERR_WORKSPACE_TOO_SMALL
    assert L.beam_moe_forward_nvfp4(ctypes.byref(c), 0, q, q, None, ctypes.byref(good), q, None, None, None, 0,
                                    None, None) == bm.OK
    with pytest.raises(KeyError):
        bm._nvfp4_experts(bm.BEAM_LAYER.c(), {"q_gate": None})


def test_mxfp8_entry_points_check_arguments_on_host(L):
    """The native FP8 path needs hidden and inter in multiples of 128 and checks its own workspace size."""
    p = ctypes.c_void_p(4096)
    good = bm.BeamMoeFp8Experts(4096, 4096, 4096, 4096, 4096, 4096)
    for bad in (dict(hidden=320), dict(inter=192)):
        c = _cfg(**bad)
        assert bm.workspace_size(c, 64, bm.WS_MXFP8) == 0
        assert L.beam_moe_forward_mxfp8(ctypes.byref(c), 64, p, p, None, ctypes.byref(good), p, None, None, p,
                                        1 << 40, None, None) == bm.ERR_INVALID_CONFIG
        assert L.beam_moe_experts_mxfp8(ctypes.byref(c), 64, p, p, p, ctypes.byref(good), p, p, 1 << 40, None) == \
            bm.ERR_INVALID_CONFIG
    c = _cfg()
    need = bm.workspace_size(c, 64, bm.WS_MXFP8)
    assert need > 0 and bm.workspace_size(c, 4096, bm.WS_MXFP8) < bm.workspace_size(c, 4096, bm.WS_FORWARD)
    assert L.beam_moe_forward_mxfp8(ctypes.byref(c), 64, p, p, None, ctypes.byref(good), p, None, None, p, need - 1,
                                    None, None) == bm.ERR_WORKSPACE_TOO_SMALL
    assert L.beam_moe_forward_mxfp8(ctypes.byref(c), 64, p, p, None, None, p, None, None, p, need, None, None) == \
        bm.ERR_NULL
    assert L.beam_moe_experts_mxfp8(ctypes.byref(c), 0, p, p, p, ctypes.byref(good), p, p, 0, None) == bm.OK
