"""Tensor-core (tcgen05) and TMA building blocks of the fused forward pass, against torch fp64.

Each case runs one product through the same shared-memory layouts and descriptors the fused
kernel uses (see csrc/lfa_selftest.cu) and compares with a float64 reference.
"""
import pytest
import torch

from laplacian_nystr_attention_avg_b200 import lfa

pytestmark = pytest.mark.gpu


def _bf16(x):
    return x.to(torch.bfloat16).double()


def _rand(*shape, seed=0):
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float32)


def test_bf16_kmajor_a_kmajor_b():
    A, Bt = _rand(128, 64, seed=1), _rand(64, 64, seed=2)
    D = lfa.selftest(0, A.cuda(), Bt.cuda()).double().cpu()
    ref = _bf16(A) @ _bf16(Bt).T
    assert torch.allclose(D, ref, rtol=1e-5, atol=1e-4)


def test_bf16_mnmajor_pass1_product_m64():
    Cs, Vs = _rand(128, 64, seed=3), _rand(128, 64, seed=4)     # [K = tokens][M], [K][N]
    D = lfa.selftest(1, Cs.cuda(), Vs.cuda()).double().cpu()
    ref = _bf16(Cs).T @ _bf16(Vs)
    assert torch.allclose(D[:64], ref, rtol=1e-5, atol=1e-4)


@pytest.mark.parametrize("shift", [0, 8, 56, 64])
def test_bf16_kmajor_a_at_row_offset(shift):
    A, Bt = _rand(192, 64, seed=6), _rand(64, 64, seed=7)
    D = lfa.selftest(3, A.cuda(), Bt.cuda(), param=shift).double().cpu()
    ref = _bf16(A[shift:shift + 128]) @ _bf16(Bt).T
    assert torch.allclose(D, ref, rtol=1e-5, atol=1e-4)


@pytest.mark.parametrize("row0", [0, 5, -9, 40])
def test_tma_swizzle_and_zero_fill(row0):
    src = _rand(100, 64, seed=8).to(torch.bfloat16)
    D = lfa.selftest(4, None, None, param=row0, tma_src=src.cuda()).cpu()
    ref = torch.zeros(128, 64)
    lo, hi = max(row0, 0), min(row0 + 128, 100)
    ref[lo - row0:hi - row0] = src[lo:hi].float()
    assert torch.equal(D, ref)



def test_tf32x1_kmajor_b():
    A, Bt = _rand(128, 64, seed=9), _rand(64, 64, seed=10)
    D = lfa.selftest(5, A.cuda(), Bt.cuda()).double().cpu()
    ref = A.double() @ Bt.double().T
    err = (D - ref).abs().max() / ref.abs().max()
    assert err < 3e-3, float(err)



def test_tf32x3_kmajor_b_from_bottom_rows():
    A = _rand(128, 64, seed=12)
    D = lfa.selftest(7, A.cuda(), A.cuda()).double().cpu()
    ref = A.double() @ A.double()[64:128].T
    err = (D - ref).abs().max() / ref.abs().max()
    assert err < 2e-6, float(err)

