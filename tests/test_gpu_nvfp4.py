"""NVFP4 expert weights (E2M1 codes, E4M3 scale per 16 K, FP32 per-matrix scale) on the GPU vs the
oracle run on the dequantised FP64 weights.

The kernels rebuild e2m1 x scale x 2^-9 as exact bf16 values, run the bf16 tensor-core path and
apply the per-matrix scale (times 2^9) to the FP32 accumulators, so the protocol is the bf16 one:
routing bit-exact outside near-ties, outputs within 2e-2 * RMS plus half a bf16 ulp of the oracle's.
The oracle's weights come from oracle.dequant_nvfp4 of the same codes the GPU reads (made by
beam_synth.quantize_nvfp4); nothing is taken from the GPU path.
"""
import numpy as np
import pytest
import torch

import beam_synth as bs
import group_limited_routing_router_b200 as bm
import oracle
from tests import fullsize, parity

pytestmark = pytest.mark.gpu

SMALL = ["tiny", "mid_a", "mid_b", "mid_c", "mid_skew", "mid_big_expert", "beam_small_T"]


class Nvfp4Case(parity.Case):
    """parity.Case whose experts are NVFP4; the oracle dequantises one expert to FP64 on the host."""

    def __init__(self, wl, T=None, weights=None, w4=None):
        super().__init__(wl, T=T, weights=weights)
        self.w4 = bs.quantize_experts_nvfp4(self.wg, self.wu, self.wd) if w4 is None else w4

    def fetch64(self, e: int):
        out = []
        for name in ("gate", "up", "down"):
            q = self.w4["q_" + name][e].cpu().numpy()
            s = self.w4["s_" + name][e].cpu().numpy()
            g = float(self.w4["g_" + name][e].cpu())
            out.append(oracle.dequant_nvfp4(q, s, g))
        return tuple(out)

    def oracle_y(self, ids, w, tokens):
        return oracle.experts_tokens_f64(np.ascontiguousarray(self.x_bits[tokens]), ids[tokens], w[tokens],
                                         self.fetch64, self.layer["n_experts"], self.layer["routed_scale"])


def _case(name, beam_weights, beam_weights_nvfp4):
    wl = bs.get(name)
    if wl.expert_device == "cuda":
        return Nvfp4Case(wl, weights=beam_weights, w4=beam_weights_nvfp4)
    return Nvfp4Case(wl)


def _experts(case, ids_np, w_np):
    ids = torch.from_numpy(np.ascontiguousarray(ids_np, dtype=np.int32)).cuda()
    w = torch.from_numpy(np.ascontiguousarray(w_np, dtype=np.float32)).cuda()
    y = bm.experts_nvfp4(case.layer, case.x, ids, w, case.w4)
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    return y.float().cpu().numpy()


@pytest.mark.parametrize("name", SMALL)
def test_nvfp4_experts_small(name, beam_weights, beam_weights_nvfp4):
    case = _case(name, beam_weights, beam_weights_nvfp4)
    r = case.oracle_route()
    y = _experts(case, r["ids"], r["weight"])
    st = parity.compare_y(y, case.oracle_y(r["ids"], r["weight"], np.arange(case.T)), name)
    print(f"{name}: {st}")


@pytest.mark.parametrize("name", list(fullsize.SAMPLE_LOWP))
def test_nvfp4_experts_full_size(name, bank):
    """The expert half with the shared layer's NVFP4 checkpoint on the oracle's routing; outputs on
    every decode token and on 256 seeded prefill tokens."""
    case = bank.case(name)
    r = case.oracle_route()
    ids = torch.from_numpy(np.ascontiguousarray(r["ids"], dtype=np.int32)).cuda()
    w = torch.from_numpy(np.ascontiguousarray(r["weight"], dtype=np.float32)).cuda()
    y = bm.experts_nvfp4(case.layer, case.x, ids, w, bank.nvfp4())
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    y = y.float().cpu().numpy()
    assert np.isfinite(y).all()
    tok = fullsize.sample(name, "nvfp4")
    st = parity.compare_y(y[tok], bank.oracle_y("nvfp4", name), name)
    print(f"{name}: {len(tok)} tokens: {st}")


@pytest.mark.parametrize("name", ["mid_b", "beam_small_T"])
def test_nvfp4_forward_small(name, beam_weights, beam_weights_nvfp4):
    case = _case(name, beam_weights, beam_weights_nvfp4)
    y, ids, w = bm.forward_nvfp4(case.layer, case.x, case.w_router, case.bias, case.w4, return_routing=True)
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    y, ids, w = y.float().cpu().numpy(), ids.cpu().numpy(), w.cpu().numpy()
    r = case.oracle_route()
    st = parity.compare_routing(r, case.layer, ids, w, case.bias_np)
    tok = np.arange(case.T)
    yo = parity.oracle_y_checked(r, st, ids, tok, case.oracle_y(r["ids"], r["weight"], tok), case.oracle_y)
    sy = parity.compare_y(y[tok], yo, name)
    print(f"{name}: excluded {st['n_excluded']}: {sy}")


@pytest.mark.parametrize("name", list(fullsize.SAMPLE_LOWP))
def test_nvfp4_forward_full_size(name, bank):
    case = bank.case(name)
    y, ids, w = bm.forward_nvfp4(case.layer, case.x, case.w_router, case.bias, bank.nvfp4(),
                           return_routing=True)
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    y, ids, w = y.float().cpu().numpy(), ids.cpu().numpy(), w.cpu().numpy()
    r = case.oracle_route()
    st = parity.compare_routing(r, case.layer, ids, w, case.bias_np)
    tok = fullsize.sample(name, "nvfp4")
    yo = parity.oracle_y_checked(r, st, ids, tok, bank.oracle_y("nvfp4", name), bank.y_of("nvfp4", name))
    sy = parity.compare_y(y[tok], yo, name)
    print(f"{name}: {len(tok)} tokens, excluded {st['n_excluded']}: {sy}")


@pytest.mark.parametrize("codes", ["all", "subnormal_only"])
def test_nvfp4_every_code_and_scale_range(codes):
    """Code coverage with well-conditioned layers.  'all': random bytes over all 256 E2M1 code
    pairs, E4M3 scale codes from 0.5 to 4 (one per weight row), per-matrix scales in [1, 2).
    'subnormal_only': only the E2M1 codes 0 and +-0.5 (exponent 0) with the subnormal E4M3 scale
    codes m * 2^-9 (m = 1..7), per-matrix scales in [2^8, 2^9): a path that flushed either kind of
    subnormal would return zeros or wrong magnitudes.  Both: some all-zero blocks with scale code 0,
    ragged T and row tiles.  The ranges are kept narrow so that the oracle comparison measures the
    decoding, not the conditioning of the layer; the whole scale-code range (subnormal scales up to
    448) is covered by test_nvfp4_matches_bf16_path_on_dequantised_weights, which compares the NVFP4
    path with the bf16 path on the same dequantised weights bit for bit."""
    wl = bs.Workload("nvfp4_codes", T=77, hidden=192, inter=320, n_experts=8, n_groups=2, topk_groups=1, topk=2,
                     seed=4343)
    case = Nvfp4Case(wl)
    g = torch.Generator().manual_seed(98)
    E, H, I = wl.n_experts, wl.hidden, wl.inter
    w4 = {}
    for name, rows, K in (("gate", I, H), ("up", I, H), ("down", H, I)):
        q = torch.randint(0, 256, (E, rows, K // 2), generator=g, dtype=torch.int32)
        if codes == "subnormal_only":
            q = q & 0x99                                             # each nibble: sign + mantissa bit only
            lo, hi, gexp = 0x01, 0x08, 8                             # E4M3 subnormal scales m * 2^-9
        else:
            lo, hi, gexp = 0x30, 0x49, 0                             # E4M3 scales 0.5 .. 4
        s = torch.randint(lo, hi, (E, 1, rows), generator=g, dtype=torch.int32).expand(E, K // 16, rows)
        zero = torch.rand(E, K // 16, rows, generator=g) < 0.05
        s = torch.where(zero, torch.zeros_like(s), s)
        q = torch.where(zero.transpose(1, 2).repeat_interleave(8, dim=2), torch.zeros_like(q), q)
        glob = 2.0 ** gexp * (1 + torch.rand(E, generator=g))
        w4["q_" + name] = q.to(torch.uint8).cuda()
        w4["s_" + name] = s.to(torch.uint8).contiguous().cuda()
        w4["g_" + name] = glob.float().cuda()
    case.w4 = w4
    r = case.oracle_route()
    y = _experts(case, r["ids"], r["weight"])
    st = parity.compare_y(y, case.oracle_y(r["ids"], r["weight"], np.arange(wl.T)), "nvfp4_codes")
    assert st["rms"] > 0
    print(st)


@pytest.mark.parametrize("gexp", [-12, -20])
def test_nvfp4_matches_bf16_path_on_dequantised_weights(gexp):
    """Decode check over the whole scale range, separate from accumulation error.  Random code bytes
    over all 256 E2M1 pairs, one E4M3 scale code per 16 K elements drawn over every non-negative
    finite code (0x00..0x7e: zero, the subnormals m * 2^-9 and 2^-6 .. 448), a power-of-two
    per-matrix scale 2^gexp.  Every dequantised weight e2m1 * e4m3 * 2^gexp has at most 6 significant
    bits, so it is a bf16 value: the bf16 entry point on those weights must return the same bits as
    the NVFP4 entry point, whose rebuilt tiles hold e2m1 * e4m3 * 2^-9 and whose accumulators are
    scaled by 2^(gexp + 9), an exact power of two.  A self-consistency check of the product (not a
    parity claim); the oracle's error on these wide-range weights is printed beside it."""
    wl = bs.Workload("nvfp4_wide", T=333, hidden=512, inter=384, n_experts=16, n_groups=4, topk_groups=2, topk=4,
                     seed=4545)
    case = Nvfp4Case(wl)
    g = torch.Generator().manual_seed(97 + gexp)
    E, H, I = wl.n_experts, wl.hidden, wl.inter
    w4, deq = {}, []
    for name, rows, K in (("gate", I, H), ("up", I, H), ("down", H, I)):
        q = torch.randint(0, 256, (E, rows, K // 2), generator=g, dtype=torch.int32).to(torch.uint8)
        s = torch.randint(0x00, 0x7f, (E, K // 16, rows), generator=g, dtype=torch.int32).to(torch.uint8)
        glob = torch.full((E,), 2.0 ** gexp, dtype=torch.float32)
        w4["q_" + name], w4["s_" + name], w4["g_" + name] = q.cuda(), s.contiguous().cuda(), glob.cuda()
        d = np.stack([oracle.dequant_nvfp4(q[e].numpy(), s[e].numpy(), float(glob[e])) for e in range(E)])
        bits = oracle.f64_to_bf16_bits(d)
        assert np.array_equal(oracle.bf16_bits_to_f64(bits), d), "a dequantised weight is not a bf16 value"
        deq.append(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda())
    case.w4 = w4
    r = case.oracle_route()
    y4 = _experts(case, r["ids"], r["weight"])
    ids = torch.from_numpy(np.ascontiguousarray(r["ids"], dtype=np.int32)).cuda()
    w = torch.from_numpy(np.ascontiguousarray(r["weight"], dtype=np.float32)).cuda()
    y16 = bm.experts(case.layer, case.x, ids, w, *deq)
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    y16 = y16.float().cpu().numpy()
    assert np.isfinite(y4).all() and np.abs(y4).max() > 0
    assert np.array_equal(y4.view(np.uint32), y16.view(np.uint32))
    yo = case.oracle_y(r["ids"], r["weight"], np.arange(wl.T))
    err = np.abs(y16 - yo)
    print(f"2^{gexp}: NVFP4 == bf16 path bit for bit; both vs the oracle: max|err|/RMS "
          f"{err.max() / np.sqrt((yo ** 2).mean()):.4f}")


def test_nvfp4_forward_profiled_events(bank):
    case = bank.case("prefill")
    case.w4 = bank.nvfp4()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(7)]
    y = bm.forward_nvfp4(case.layer, case.x, case.w_router, case.bias, case.w4, events=ev)
    torch.cuda.synchronize()
    assert bm.device_status() == bm.OK
    ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(6)]
    assert all(m >= 0 for m in ms) and ms[3] > 0
    y2 = bm.forward_nvfp4(case.layer, case.x, case.w_router, case.bias, case.w4)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
