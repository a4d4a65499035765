"""Pins of the oracle's MXFP8 activations (block-scaled FP8 path), checked against torch's float8
E4M3 cast (round to nearest even) and the OCP MXFP8 scale rule, none of it the oracle's own code.

Reading (the pages give no FP8 recipe): activations are quantised per row in blocks of 32 along the
reduction axis, with one UE8M0 scale per block, the smallest power of two that brings the block's
largest magnitude to at most 448 (E4M3's largest finite value).
"""
import numpy as np
import torch

import oracle


def _torch_quant_rows(v: np.ndarray) -> np.ndarray:
    """Independent restatement in torch: scale = 2^e, e the smallest integer with amax <= 448 * 2^e
    (searched exactly over powers of two), elements cast with torch's float8_e4m3fn (RNE)."""
    t = torch.from_numpy(v).double()
    rows, K = t.shape
    blk = t.reshape(rows, K // 32, 32)
    amax = blk.abs().amax(-1)
    e = torch.zeros_like(amax)
    nz = amax > 0
    e[nz] = torch.floor(torch.log2(amax[nz])) - 10
    for _ in range(4):  # walk up to the smallest power of two that fits (log2 only seeds the search)
        e = torch.where(nz & (amax > 448.0 * torch.exp2(e)), e + 1, e)
    scale = torch.exp2(e).unsqueeze(-1)
    q = (blk / scale).to(torch.float8_e4m3fn).double() * scale
    return torch.where(nz.unsqueeze(-1), q, torch.zeros_like(q)).reshape(rows, K).numpy()


def _random_rows(seed, rows=16, K=256):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((rows, K)) * np.exp(rng.standard_normal((rows, 1)) * 4)
    v[0, :32] = 0.0                                              # an all-zero block
    v[1, 32:64] = rng.standard_normal(32) * 1e-3                 # small values: subnormal codes
    v[2, 64:96] *= 1e-6
    return v


def test_quantised_rows_match_torch_e4m3_cast_and_scale_rule():
    for seed in range(5):
        v = _random_rows(seed)
        q, sc, deq = oracle.quant_mxfp8_rows(v)
        np.testing.assert_array_equal(deq, _torch_quant_rows(v))
        # codes decode (torch) times the block scale to the dequantised values
        codes = torch.from_numpy(q.view(np.int8)).view(torch.float8_e4m3fn).double().numpy()
        scale = np.exp2(sc.astype(np.float64) - 127).repeat(32, axis=1)
        nzb = np.abs(v).reshape(v.shape[0], -1, 32).max(-1) > 0
        nz = nzb.repeat(32, axis=1)
        np.testing.assert_array_equal(np.where(nz, codes * scale, 0.0), deq)
        # the largest scaled magnitude of every nonzero block lies in (224, 448]
        top = np.abs(v).reshape(v.shape[0], -1, 32).max(-1) / np.exp2(sc.astype(np.float64) - 127)
        assert np.all(top[nzb] <= 448.0) and np.all(top[nzb] > 224.0)
        assert np.all(sc[~nzb] == 0)


def test_ties_round_to_even_code():
    """Midpoints between neighbouring E4M3 values (normal and subnormal) go to the even code."""
    grid = torch.arange(0, 127, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    grid = np.unique(grid[np.isfinite(grid)])
    mids = (grid[:-1] + grid[1:]) / 2
    blk = np.concatenate([mids, grid])
    v = np.zeros((1, 32 * int(np.ceil(len(blk) / 31))))
    for i in range(0, len(blk), 31):  # 448 in every block fixes the scale at 2^0
        v[0, (i // 31) * 32:(i // 31) * 32 + 32] = np.concatenate([[448.0], blk[i:i + 31], np.zeros(31 - len(blk[i:i + 31]))])
    q, sc, deq = oracle.quant_mxfp8_rows(v)
    assert np.all(sc == 127)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(deq, ref)


def test_expert_mx8_matches_torch_float64_composition():
    rng = np.random.default_rng(7)
    n, H, I = 9, 256, 192
    x = torch.from_numpy(rng.standard_normal((n, H))).to(torch.bfloat16)
    wg, wu = (torch.from_numpy(rng.standard_normal((I, H)) / 16).to(torch.bfloat16) for _ in range(2))
    wd = torch.from_numpy(rng.standard_normal((H, I)) / 14).to(torch.bfloat16)
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    got = oracle.expert_mlp_mx8(bits(x), bits(wg), bits(wu), bits(wd))
    xq = torch.from_numpy(_torch_quant_rows(x.double().numpy()))
    g = xq @ wg.double().T
    u = xq @ wu.double().T
    h = torch.nn.functional.silu(g) * u
    hq = torch.from_numpy(_torch_quant_rows(h.numpy()))
    ref = (hq @ wd.double().T).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
