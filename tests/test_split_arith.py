"""The arithmetic behind fp32 scoring on the tensor cores, checked on the
CPU: every fp32 x splits into three bf16 values hi + mid + lo = x exactly
(round to nearest even at each step, each remainder exact in fp32), with
|mid| <= 2^-8 |x| and |lo| <= 2^-16 |x|, so a dot product summed from the six
part products of order at most two misses at most 2^-23 |q| |k|.  (The
kernels do the same split on the GPU; the GPU parity tests check their
scores against the fp64 oracle.)"""
import numpy as np
import torch


def _split(x: torch.Tensor):
    hi = x.to(torch.bfloat16).float()
    r1 = x - hi
    mid = r1.to(torch.bfloat16).float()
    r2 = r1 - mid
    lo = r2.to(torch.bfloat16).float()
    return hi, mid, lo, r2


def test_three_bf16_parts_sum_to_the_fp32_value_exactly():
    g = torch.Generator().manual_seed(1)
    x = torch.cat([torch.randn(200000, generator=g),
                   torch.randn(20000, generator=g) * 1e-20,
                   torch.randn(20000, generator=g) * 1e20,
                   torch.tensor([0.0, -0.0, 1.0, -1.0, 3.0, 1.0 / 3.0, 65504.0, 2.0 ** -100])]).float()
    hi, mid, lo, r2 = _split(x)
    assert torch.equal(lo, r2)   # the last remainder fits in bf16
    total = hi.double() + mid.double() + lo.double()
    assert torch.equal(total, x.double())
    ax = x.double().abs()
    assert bool((mid.double().abs() <= ax * 2.0 ** -8).all())
    assert bool((lo.double().abs() <= ax * 2.0 ** -16).all())


def test_six_part_products_bound_the_dot_product_error():
    g = torch.Generator().manual_seed(2)
    for _ in range(20):
        q = torch.randn(64, generator=g).float()
        k = torch.randn(64, generator=g).float()
        qh, qm, ql, _ = (t.double() for t in _split(q))
        kh, km, kl, _ = (t.double() for t in _split(k))
        six = (qm * km + qh * kl + ql * kh + qh * km + qm * kh + qh * kh).sum()
        exact = (q.double() * k.double()).sum()
        bound = 2.0 ** -23 * float(np.linalg.norm(q.double()) * np.linalg.norm(k.double()))
        assert abs(float(six - exact)) <= bound
        # a single bf16 product would miss by far more than the 1e-5 margin allows
        one = (q.to(torch.bfloat16).double() * k.to(torch.bfloat16).double()).sum()
        assert abs(float(one - exact)) > 1e3 * abs(float(six - exact)) or abs(float(six - exact)) == 0.0
