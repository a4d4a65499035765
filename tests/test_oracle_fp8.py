"""Pins of the oracle's MXFP8 dequantisation (E4M3 elements, power-of-two UE8M0 scale per 32 K)."""
import numpy as np
import pytest
import torch

import beam_synth as bs
import oracle


def test_e4m3_decoder_matches_torch_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    finite = ~np.isin(codes, [0x7F, 0xFF])
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    q = codes[finite].reshape(1, -1)[:, :224]            # 254 finite codes; use a multiple of 32
    scale = np.full((q.shape[1] // 32, 1), 127, dtype=np.uint8)  # 2^0
    got = oracle.bf16_bits_to_f64(oracle.dequant_mxfp8(q, scale))[0]
    np.testing.assert_array_equal(got, ref[finite][:224])
    rest = codes[finite][224:]
    q2 = np.concatenate([rest, np.zeros(32 - rest.size % 32, np.uint8)]).reshape(1, -1)
    got2 = oracle.bf16_bits_to_f64(oracle.dequant_mxfp8(q2, np.full((q2.shape[1] // 32, 1), 127, np.uint8)))[0]
    np.testing.assert_array_equal(got2[:rest.size], ref[finite][224:])


def test_scale_is_a_power_of_two_per_32_block():
    rng = np.random.default_rng(0)
    q = rng.integers(0, 0x7E, size=(3, 64), dtype=np.uint8)   # finite positive codes
    base = oracle.bf16_bits_to_f64(oracle.dequant_mxfp8(q, np.full((2, 3), 127, np.uint8)))
    sc = np.array([[120, 127, 130], [135, 110, 127]], dtype=np.uint8)   # [K/32, rows]
    got = oracle.bf16_bits_to_f64(oracle.dequant_mxfp8(q, sc))
    for r in range(3):
        for kb in range(2):
            np.testing.assert_array_equal(got[r, 32 * kb:32 * (kb + 1)],
                                          base[r, 32 * kb:32 * (kb + 1)] * 2.0 ** (int(sc[kb, r]) - 127))


def test_nan_codes_rejected():
    q = np.zeros((1, 32), dtype=np.uint8)
    q[0, 5] = 0x7F
    with pytest.raises(ValueError):
        oracle.dequant_mxfp8(q, np.full((1, 1), 127, np.uint8))
    with pytest.raises(ValueError):
        oracle.dequant_mxfp8(np.zeros((1, 32), np.uint8), np.full((1, 1), 255, np.uint8))


def test_synthetic_checkpoint_round_trip():
    """The input quantiser keeps every element within E4M3's half-ulp (2^-4 relative) of the bf16
    weight, and each block's largest element in [224, 448] before scaling."""
    wl = bs.get("mid_a")
    wg = bs.make_expert(wl, 2, "cpu")[0]              # [I, H] bf16
    q, sc = bs.quantize_mxfp8(wg)
    deq = oracle.bf16_bits_to_f64(oracle.dequant_mxfp8(q.numpy(), sc.numpy()))
    w = wg.double().numpy()
    blk = np.abs(w).reshape(w.shape[0], -1, 32).max(-1)                      # [I, H/32]
    scale = 2.0 ** (sc.numpy().astype(np.float64).T - 127)                   # [I, H/32]
    assert np.all((blk / scale >= 224) & (blk / scale <= 448))
    err = np.abs(deq - w)
    bound = np.maximum(np.abs(w) * 2.0 ** -4, np.repeat(scale, 32, axis=1) * 2.0 ** -10)
    assert np.all(err <= bound * (1 + 1e-12))
