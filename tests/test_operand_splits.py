"""The error bounds of the tcgen05 kernels' operand splits, checked on the CPU.

bf16 kernels: an MMA's two operands share one type, and V is bf16, so the fp32
softmax weights go in as two bf16 pieces, p = p_hi + p_lo with p_hi = bf16(p)
and p_lo = bf16(p - p_hi), in separate MMA columns summed in fp32.  The
verify-step and prefill kernels take both pieces by truncation instead (the
upper halves of the fp32 bits), which keeps 2^-14 relative.

fp8 kernel:

The kernel multiplies e4m3 cache codes on the tensor cores against q and against
the softmax weights, each represented as three e4m3 pieces scaled 1, 1/16 and
1/256 (x = x1 + x2 / 16 + x3 / 256), after a power-of-two scaling that puts the
largest magnitude in [64, 128) for q and below 2^6 for the weights.  This file
restates that split with torch's float8_e4m3fn rounding (round to nearest even)
and checks the bounds the kernel's design relies on:

* q (bf16): exact for elements down to 2^-6 of the row's largest, and within
  2^-18 of the largest element everywhere;
* weights in (0, 2^6]: relative error below 2^-13 for weights >= 2^-3, and an
  absolute error below 2^-17 for the smaller ones, where the third piece reaches
  e4m3's subnormal step 2^-9 (weights are in the kernel's scaled domain, whose
  largest value is at most 2^6).
"""
import math

import torch

E4M3 = torch.float8_e4m3fn


def e4m3(x: torch.Tensor) -> torch.Tensor:
    return x.to(E4M3).to(torch.float64)


def split3(x: torch.Tensor):
    """Three e4m3 pieces, each holding 16x the rounding error of the one before."""
    p1 = e4m3(x)
    r = (x - p1) * 16
    p2 = e4m3(r)
    r = (r - p2) * 16
    p3 = e4m3(r)
    return p1, p2, p3


def recombine(p1, p2, p3):
    return p1 + p2 / 16 + p3 / 256


def test_q_split_exact_for_bf16_rows():
    g = torch.Generator().manual_seed(0)
    for _ in range(20):
        q = (torch.randn(512, generator=g, dtype=torch.float64)
             * torch.exp2(torch.randint(-8, 9, (1,), generator=g).double()))
        q = q.to(torch.bfloat16).to(torch.float64)
        amax = q.abs().max().item()
        a = 6 - math.floor(math.log2(amax))  # largest |q| 2^a in [64, 128)
        qs = q * 2.0 ** a
        assert 64 <= qs.abs().max().item() < 128
        err = (recombine(*split3(qs)) - qs).abs()
        big = qs.abs() >= 2.0 ** -6 * qs.abs().max()
        assert err[big].max().item() == 0.0, "q split not exact for elements >= 2^-6 of the max"
        assert err.max().item() <= 2.0 ** -18 * qs.abs().max().item()


def test_weight_split_bounds():
    g = torch.Generator().manual_seed(1)
    # weights p * s_v * 2^-e: spread over many octaves below the bound 2^6
    w = torch.exp2(torch.rand(200000, generator=g, dtype=torch.float64) * 30 - 24)
    w = w[w <= 2.0 ** 6]
    err = (recombine(*split3(w)) - w).abs()
    big = w >= 2.0 ** -3
    assert (err[big] / w[big]).max().item() < 2.0 ** -13
    assert err[~big].max().item() < 2.0 ** -17  # the floor below 2^-3


def test_pieces_stay_inside_e4m3_range():
    """No piece saturates: every piece of a value up to 2^7 is below 448."""
    x = torch.linspace(-128, 128, 100001, dtype=torch.float64)
    for p in split3(x):
        assert p.abs().max().item() <= 448
        assert torch.isfinite(p).all()


def test_bf16_hi_lo_weight_split():
    """Two bf16 pieces keep an fp32 weight to 2^-17 relative; one piece keeps 2^-8."""
    g = torch.Generator().manual_seed(2)
    p = torch.exp2(torch.rand(1_000_000, generator=g, dtype=torch.float64) * 40 - 32).float()
    hi = p.to(torch.bfloat16).float()
    lo = (p - hi).to(torch.bfloat16).float()
    rel = ((hi.double() + lo.double()) - p.double()).abs() / p.double()
    assert rel.max().item() <= 2.0 ** -17
    one = (hi.double() - p.double()).abs() / p.double()
    assert 2.0 ** -9 < one.max().item() <= 2.0 ** -8  # what a single piece would keep


def truncate_bf16(x: torch.Tensor) -> torch.Tensor:
    """The upper 16 bits of an fp32 value, as an fp32 value (round toward zero)."""
    bits = x.float().contiguous().view(torch.int32) & ~0xFFFF
    return bits.view(torch.float32)


def test_bf16_truncation_weight_split():
    """The verify-step and prefill kernels split a weight by truncation: hi = the
    upper half of its fp32 bits, lo = the upper half of p - hi (exact in fp32).
    Two truncated pieces keep a positive weight to 2^-14 relative, never above it."""
    g = torch.Generator().manual_seed(3)
    p = torch.exp2(torch.rand(1_000_000, generator=g, dtype=torch.float64) * 40 - 32).float()
    hi = truncate_bf16(p)
    r = p - hi
    assert torch.equal(r.double(), p.double() - hi.double())  # the remainder is exact
    lo = truncate_bf16(r)
    assert torch.equal(hi.to(torch.bfloat16).float(), hi)  # both pieces are bf16 numbers
    assert torch.equal(lo.to(torch.bfloat16).float(), lo)
    total = hi.double() + lo.double()
    assert (total <= p.double()).all()
    rel = (p.double() - total) / p.double()
    assert 2.0 ** -16 < rel.max().item() < 2.0 ** -14
