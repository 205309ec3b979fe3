"""Pins for the oracle's OCP E4M3fn codec and its 1x128 / 128x128 quantisation.

The codec is checked against torch's own float8_e4m3fn conversion (an
independent implementation) and against brute-force nearest-code search over
all 256 codes; the quantisers against invariants that hold by definition.
"""
import pytest
import torch

from oracle import fp8moe_oracle as O

pytestmark = pytest.mark.filterwarnings("ignore")


def test_decode_matches_torch_float8_for_all_codes():
    codes = torch.arange(256, dtype=torch.int64).to(torch.uint8)
    ours = O.e4m3_decode(codes)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64)
    nan = torch.isnan(ref)
    assert torch.equal(torch.isnan(ours), nan)
    assert nan.sum() == 2                                  # 0x7F and 0xFF only
    assert torch.equal(ours[~nan], ref[~nan])


def test_decode_format_facts():
    d = O.e4m3_decode(torch.tensor([0x7E, 0x08, 0x01, 0x00, 0x80, 0xFE, 0x38], dtype=torch.uint8))
    assert d.tolist()[:4] == [448.0, 2.0 ** -6, 2.0 ** -9, 0.0]
    assert d[5] == -448.0 and d[6] == 1.0


def _nearest_code_bruteforce(v):
    """RNE to the E4M3fn grid by trying every finite code; ties go to the even code."""
    codes = torch.tensor([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=torch.int64)
    vals = O.e4m3_decode(codes.to(torch.uint8))
    out = []
    for x in v.to(torch.float64).tolist():
        if abs(x) > 448.0:
            out.append(0x7E | (0x80 if x < 0 else 0))
            continue
        d = (vals - x).abs()
        best = d.min()
        cand = codes[d == best].tolist()
        # among equidistant codes of the right sign, prefer an even mantissa
        cand = [c for c in cand if ((c >> 7) == (1 if (x < 0 or (x == 0 and str(x)[0] == "-")) else 0))] or cand
        even = [c for c in cand if (c & 1) == 0]
        out.append((even or cand)[0])
    return torch.tensor(out, dtype=torch.int64)


def test_encode_matches_bruteforce_on_grid_midpoints_and_random():
    g = torch.Generator().manual_seed(1)
    vals = O.e4m3_decode(torch.arange(0, 0x7F, dtype=torch.int64).to(torch.uint8))
    mids = (vals[1:] + vals[:-1]) / 2                       # exact ties
    near = torch.cat([mids * (1 + 2.0 ** -20), mids * (1 - 2.0 ** -20)])
    rnd = torch.cat([torch.rand(300, generator=g) * 460, torch.rand(200, generator=g) * 2.0 ** -5,
                     torch.tensor([464.0, 463.99, 448.0, 449.0, 1e9, 2.0 ** -10, 3 * 2.0 ** -11])])
    x = torch.cat([vals, mids, near, rnd]).to(torch.float32)
    x = torch.cat([x, -x])
    ours = O.e4m3_encode(x).to(torch.int64)
    ref = _nearest_code_bruteforce(x)
    assert torch.equal(ours, ref)


def test_encode_matches_torch_cast_in_range():
    g = torch.Generator().manual_seed(2)
    x = torch.cat([torch.randn(200000, generator=g) * 100, torch.randn(100000, generator=g) * 1e-2,
                   torch.randn(50000, generator=g) * 1e-4]).to(torch.float32)
    x = x[x.abs() <= 464.0]                                  # torch's cast is not saturating above
    ours = O.e4m3_encode(x)
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(ours, ref)


def test_encode_saturates():
    x = torch.tensor([465.0, 480.0, 1e30, float("inf"), -500.0, -float("inf")], dtype=torch.float32)
    assert O.e4m3_encode(x).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    assert O.e4m3_encode(torch.tensor([float("nan")])).tolist() == [0x7F]


def test_quant_1x128_invariants():
    g = torch.Generator().manual_seed(3)
    x = (torch.randn(7, 3 * 128 + 40, generator=g) * torch.logspace(-3, 2, 7)[:, None]).to(torch.bfloat16)
    x[2, 128:256] = 0                                        # an all-zero group
    q, s = O.quant_1x128(x)
    assert q.shape == x.shape and s.shape == (7, 4)
    assert s[2, 1] == 0 and (q[2, 128:256] == 0).all()
    xf = x.float()
    for kb in range(4):
        cols = slice(kb * 128, min(x.shape[1], kb * 128 + 128))
        amax = xf[:, cols].abs().amax(1)
        assert torch.equal(s[:, kb], amax / torch.tensor(448.0))
        # the largest element of each non-zero group lands on +-448
        nz = amax > 0
        arg = xf[:, cols].abs().argmax(1)
        top = q[:, cols].gather(1, arg[:, None])[:, 0].to(torch.int64) & 0x7F
        assert (top[nz] == 0x7E).all()
    # dequantised values are within half an E4M3 step of the input (relative 2^-4, or 2^-10 * scale)
    deq = O.e4m3_decode(q) * s.to(torch.float64).repeat_interleave(128, 1)[:, : x.shape[1]]
    err = (deq - xf.double()).abs()
    bound = torch.maximum(xf.double().abs() * 2.0 ** -4, s.double().repeat_interleave(128, 1)[:, : x.shape[1]] * 2.0 ** -10)
    assert (err <= bound * 1.0000001).all()


def test_quant_128x128_blocks_and_edges():
    g = torch.Generator().manual_seed(4)
    w = torch.randn(300, 260, generator=g) * 0.02
    w[128:256, 0:128] *= 1000                               # a block with its own scale
    q, s = O.quant_128x128(w)
    assert q.shape == (300, 260) and s.shape == (3, 3)
    for nb in range(3):
        for kb in range(3):
            blk = w[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            assert s[nb, kb] == blk.abs().max() / torch.tensor(448.0)
            # each block equals the 1x128 recipe applied with that block's scale
            qb = q[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            ref = O.e4m3_encode(blk / s[nb, kb])
            assert torch.equal(qb, ref)


def test_bf16_round_matches_torch_on_fp32_values():
    g = torch.Generator().manual_seed(5)
    x = torch.cat([torch.randn(100000, generator=g) * 10, torch.randn(1000, generator=g) * 1e-39])
    x32 = x.to(torch.float32)
    ours = O.bf16_round(x32.double())
    ref = x32.to(torch.bfloat16).double()                   # fp32 -> bf16 is a single rounding
    assert torch.equal(ours, ref)
