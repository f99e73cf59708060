"""The FMA-pipe 2^x approximation the softmax loops can use for part of their
exponentials, checked against CUDA's exp2 (torch.exp2 on the device) and its
stated relative error bound."""
import pytest
import torch

from exact_attention_108_b200 import binding

pytestmark = pytest.mark.gpu


def test_exp2_poly_error_bound():
    x = torch.linspace(-64.0, 16.0, 1 << 22, device="cuda", dtype=torch.float32)
    y = binding.exp2_poly(x)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref) / ref).abs()
    assert rel.max().item() <= 1.1e-4, rel.max().item()


def test_exp2_poly_exact_at_integers_and_clamped_below():
    x = torch.arange(-64, 17, device="cuda", dtype=torch.float32)
    assert torch.equal(binding.exp2_poly(x), torch.exp2(x))
    lo = torch.tensor([-70.0, -1e4, float("-inf")], device="cuda")
    assert torch.equal(binding.exp2_poly(lo), torch.full_like(lo, 2.0 ** -64))
