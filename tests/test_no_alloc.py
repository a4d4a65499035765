"""beam_moe_permute_noalloc: the dispatch for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc when they enqueue work: a plugin inside an inference server
whose host framework owns all device memory, or a latency-critical loop where an allocation could
synchronise the device.  For them the library offers a dispatch entry point whose scratch is a fixed
array inside the library (256 KiB per device, enough for 65,536 tokens at 256 experts).  These tests
call it through the C ABI and require outputs identical to the workspace entry point's, on
consecutive calls that reuse the shared array with different sizes.  Its tests carry the `last`
marker, which the collection hook in conftest.py moves behind every other test whatever the file's
name, so a run that stops at the first failure has run everything else first.
"""
import ctypes

import numpy as np
import pytest
import torch

import group_limited_routing_router_b200 as bm


def _fn():
    f = bm.lib().beam_moe_permute_noalloc
    vp = ctypes.c_void_p
    f.argtypes = [ctypes.POINTER(bm.BeamMoeConfig), ctypes.c_int64, vp, vp, vp, vp, vp, vp]
    f.restype = ctypes.c_int
    return f


def _layer(E, k, G=8):
    return bm.LayerConfig(hidden=64, inter=64, n_experts=E, n_groups=G, topk_groups=G, topk=k, group_topn=1,
                          routed_scale=1.0)


def _ids(T, E, k, seed):
    rng = np.random.default_rng(seed)
    return np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)  # k distinct experts per token


def _noalloc(layer, ids_dev):
    T = ids_dev.shape[0]
    c = layer.c()
    dev = ids_dev.device
    out = dict(counts=torch.full((c.n_experts,), -7, dtype=torch.int32, device=dev),
               offsets=torch.full((c.n_experts + 1,), -7, dtype=torch.int64, device=dev),
               row_src=torch.full((T * c.topk,), -7, dtype=torch.int32, device=dev),
               dest_row=torch.full((T * c.topk,), -7, dtype=torch.int32, device=dev))
    rc = _fn()(ctypes.byref(c), T, ctypes.c_void_p(ids_dev.data_ptr()), ctypes.c_void_p(out["counts"].data_ptr()),
               ctypes.c_void_p(out["offsets"].data_ptr()), ctypes.c_void_p(out["row_src"].data_ptr()),
               ctypes.c_void_p(out["dest_row"].data_ptr()),
               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == bm.OK, bm.strerror(rc)
    return out


@pytest.mark.gpu
@pytest.mark.last
def test_noalloc_permute_matches_workspace_permute_on_consecutive_calls():
    cases = [(_layer(256, 8), _ids(4096, 256, 8, 1)),     # Beam prefill shape
             (_layer(64, 6), _ids(777, 64, 6, 2)),        # smaller call: the array keeps stale entries
             (_layer(256, 8), _ids(4096, 256, 8, 3)),     # big again, over the stale contents
             (_layer(256, 8), _ids(65536, 256, 8, 4))]    # the largest size the fixed array allows
    for layer, ids_np in cases:
        ids = torch.from_numpy(ids_np).cuda()
        ref = bm.permute(layer, ids)            # the existing entry point, caller workspace
        got = _noalloc(layer, ids)
        torch.cuda.synchronize()
        assert bm.device_status() == bm.OK
        for key in ("counts", "offsets", "row_src", "dest_row"):
            assert torch.equal(got[key], ref[key]), key


@pytest.mark.last
def test_noalloc_permute_rejects_sizes_beyond_its_array():
    layer = _layer(256, 8)
    p = ctypes.c_void_p(4096)  # never dereferenced: the size check fails first
    rc = _fn()(ctypes.byref(layer.c()), 65536 + 1, p, p, p, p, p, None)
    assert rc == bm.ERR_INVALID_ARG
