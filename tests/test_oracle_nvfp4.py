"""Pins of the oracle's NVFP4 dequantisation (E2M1 elements, E4M3 scale per 16 K, FP32 per-matrix
scale) and of its SwiGLU expert with FP64 weights."""
import numpy as np
import pytest
import torch

import beam_synth as bs
import oracle

# The eight E2M1 magnitudes in code order, as NVIDIA's FP4 format lists them.
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
E4M3_ONE = 0x38


def _pack(codes: np.ndarray) -> np.ndarray:
    """codes [rows, K] (0..15) -> bytes [rows, K/2], even k in the low nibble."""
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def test_e2m1_decoder_all_codes_both_nibbles():
    codes = np.arange(16, dtype=np.uint8)
    want = np.array(E2M1_TABLE + [-v for v in E2M1_TABLE])
    row = np.concatenate([codes, codes[::-1]]).reshape(1, 32)       # every code in both nibble positions
    got = oracle.dequant_nvfp4(_pack(row), np.full((2, 1), E4M3_ONE, np.uint8), 1.0)[0]
    np.testing.assert_array_equal(got[:16], want)
    np.testing.assert_array_equal(got[16:], want[::-1])


def test_even_element_is_the_low_nibble():
    q = np.zeros((1, 8), np.uint8)
    q[0, 0] = 0x21                                                   # element 0: code 1, element 1: code 2
    got = oracle.dequant_nvfp4(q, np.full((1, 1), E4M3_ONE, np.uint8), 1.0)[0]
    assert got[0] == 0.5 and got[1] == 1.0 and not got[2:].any()


def test_block_scale_per_16_and_global_scale():
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 16, size=(3, 48), dtype=np.uint8)
    q = _pack(codes)
    base = oracle.dequant_nvfp4(q, np.full((3, 3), E4M3_ONE, np.uint8), 1.0)
    sc = rng.integers(0x08, 0x7E, size=(3, 3), dtype=np.uint8)      # finite positive E4M3 codes [K/16, rows]
    sval = torch.from_numpy(sc).view(torch.float8_e4m3fn).double().numpy()
    g = 0.3712890625
    got = oracle.dequant_nvfp4(q, sc, g)
    for r in range(3):
        for kb in range(3):
            np.testing.assert_allclose(got[r, 16 * kb:16 * (kb + 1)], base[r, 16 * kb:16 * (kb + 1)] * sval[kb, r] * g,
                                       rtol=1e-15, atol=0)


def test_bad_scale_codes_rejected():
    q = np.zeros((1, 8), np.uint8)
    for bad in (0x7F, 0xB8):                                         # NaN, sign bit set
        with pytest.raises(ValueError):
            oracle.dequant_nvfp4(q, np.full((1, 1), bad, np.uint8), 1.0)


def test_expert_mlp_f64_matches_torch_float64():
    rng = np.random.default_rng(7)
    n, H, I = 5, 64, 48
    x = torch.randn(n, H, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    wg, wu = rng.normal(0, 0.2, (I, H)), rng.normal(0, 0.2, (I, H))
    wd = rng.normal(0, 0.2, (H, I))
    got = oracle.expert_mlp_f64(oracle.bf16_bits(x), wg, wu, wd)
    xd = x.double()
    g = xd @ torch.from_numpy(wg).T
    want = (torch.nn.functional.silu(g) * (xd @ torch.from_numpy(wu).T)) @ torch.from_numpy(wd).T
    np.testing.assert_allclose(got, want.numpy(), rtol=1e-12, atol=1e-12)


def test_expert_mlp_f64_equals_bf16_version_on_bf16_weights():
    wl = bs.get("tiny")
    x = bs.make_x(wl)[:7]
    wg, wu, wd = (w[3] for w in bs.make_experts(wl))
    a = oracle.expert_mlp(oracle.bf16_bits(x), oracle.bf16_bits(wg), oracle.bf16_bits(wu), oracle.bf16_bits(wd))
    b = oracle.expert_mlp_f64(oracle.bf16_bits(x), wg.double().numpy(), wu.double().numpy(), wd.double().numpy())
    np.testing.assert_array_equal(a, b)


def test_synthetic_nvfp4_round_trip():
    """The input quantiser keeps every element within half an E2M1 step of the weight (steps 0.5, 1,
    2 on [0, 2], [2, 4], [4, 6] in units of the block's scale x global), and maps each block's
    largest magnitude to at most 6 units."""
    wl = bs.get("mid_a")
    w = bs.make_expert(wl, 2, "cpu")[0].unsqueeze(0)                  # [1, I, H]
    q, sc, g = bs.quantize_nvfp4(w)
    deq = oracle.dequant_nvfp4(q[0].numpy(), sc[0].numpy(), float(g[0]))
    wd = w[0].double().numpy()
    unit = np.repeat(torch.from_numpy(sc[0].numpy().T.copy()).view(torch.float8_e4m3fn).double().numpy(), 16,
                     axis=1) * float(g[0])                            # [I, H]: scale x global per element
    a = np.abs(wd) / unit
    step = np.where(a <= 2, 0.5, np.where(a <= 4, 1.0, 2.0))
    err = np.abs(deq - wd) / unit
    assert np.all(err <= step / 2 + 1e-6)
    assert np.all(np.abs(deq) / unit <= 6 + 1e-12)
