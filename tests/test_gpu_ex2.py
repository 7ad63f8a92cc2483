"""The prefill's FMA-pipe exponential on the GPU (duo_testing_ex2 runs the
kernel's ex2_poly2) against the exact 2^x: relative error below 1e-4 over
the softmax's range (the polynomial's bound is 7.5e-5; the CPU test
tests/test_ex2_poly.py derives it), and about 2^-125 for masked (-inf) scores."""
import pytest
import torch

import kv_cache_reduction_b200 as duo

pytestmark = pytest.mark.gpu


def test_ex2_poly_against_exact(cuda_device):
    x = torch.cat([torch.linspace(-125.0, 8.0, 1_000_003),
                   torch.arange(-125, 9).float(), torch.arange(-125, 8).float() + 0.5,
                   torch.arange(-124, 9).float() - 0.5]).cuda()
    y = duo.duo_testing_ex2(x)
    torch.cuda.synchronize()
    want = torch.exp2(x.double())
    rel = (y.double() / want - 1.0).abs()
    assert rel.max().item() < 1e-4
    # compared with the MUFU exp2 the torch kernels use
    assert ((y.double() - torch.exp2(x).double()).abs() / want).max().item() < 1e-4


def test_ex2_poly_masked_inputs(cuda_device):
    x = torch.tensor([-float("inf"), -1e30, -300.0, -126.0], device="cuda")
    y = duo.duo_testing_ex2(x).double()
    assert torch.all(y > 0) and torch.all(y <= 2.0 ** -124)


def test_ex2_poly_odd_length(cuda_device):
    x = torch.linspace(-3.0, 3.0, 7, device="cuda")
    y = duo.duo_testing_ex2(x)
    assert ((y.double() / torch.exp2(x.double()) - 1).abs()).max().item() < 1e-4
