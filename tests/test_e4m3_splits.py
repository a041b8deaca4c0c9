"""The exactness arguments behind the FP8 tensor-core path, checked on the host with
torch's float8_e4m3fn cast (round to nearest even) as the encoder.

The kernels feed E4M3 operands to kind::f8f6f4 MMAs:
  * a bf16 query, scaled by one power of two so that its largest |q| lies in [128, 256),
    is written as Q_hi + Q_lo / 16 with Q_hi = E4M3(y), Q_lo = E4M3(16 (y - Q_hi));
  * a probability rounded to f16 (|y| <= 448) is written as P_hi + P_lo / 16 + P_lo2 / 256,
    each term the E4M3 rounding of the scaled remainder, the remainders taken in f16.
These tests show the sums equal the inputs where E4M3 is in its normal range, and bound
the error below it (no GPU needed)."""
import numpy as np
import torch


def e4m3(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.float8_e4m3fn).to(torch.float32)


def test_two_e4m3_terms_hold_a_scaled_bf16_query_exactly():
    g = torch.Generator().manual_seed(0)
    q = (torch.randn(4096, 128, generator=g) * torch.exp(torch.randn(4096, 1, generator=g)))
    q = q.to(torch.bfloat16).to(torch.float32)
    for row in q:
        m = row.abs().max().item()
        e = 8 - int(np.frexp(m)[1])          # largest |y| in [128, 256)
        y = row * 2.0 ** e
        hi = e4m3(y)
        lo = e4m3((y - hi) * 16)
        rec = hi + lo / 16
        big = y.abs() >= 2.0 ** -6            # every bf16 element at or above 2^-6 (scaled)
        assert torch.equal(rec[big], y[big])
        # smaller elements: within 2^-14 absolute (half of E4M3's subnormal step, / 16)
        if (~big).any():
            assert (rec[~big] - y[~big]).abs().max().item() <= 2.0 ** -14


def test_three_e4m3_terms_hold_an_f16_value_exactly():
    g = torch.Generator().manual_seed(1)
    p = torch.rand(200000, generator=g) * torch.exp2(torch.rand(200000, generator=g) * -24 + 8)
    y = p.clamp(max=448.0).to(torch.float16)    # p * v_scale * 2^-ev rounded to f16
    y32 = y.to(torch.float32)
    hi = e4m3(y32)
    r = ((y.to(torch.float32) - hi).to(torch.float16).to(torch.float32) * 16)
    lo = e4m3(r)
    r2 = ((r - lo).to(torch.float16).to(torch.float32) * 16)
    lo2 = e4m3(r2)
    # the f16 remainders are exact (no rounding in the two subtractions)
    assert torch.equal((y32 - hi) * 16, r)
    assert torch.equal((r - lo) * 16, r2)
    rec = hi + lo / 16 + lo2 / 256
    # exact wherever E4M3 is in its normal range (|y| >= 2^-6); below, the subnormal
    # steps of the three terms (2^-9, 2^-13, 2^-17) leave at most 2^-18 absolute, which
    # is 2^-26 of the largest scaled probability (256)
    normal = y32 >= 2.0 ** -6
    assert torch.equal(rec[normal], y32[normal])
    assert (rec[~normal] - y32[~normal]).abs().max().item() <= 2.0 ** -18
