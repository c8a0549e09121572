"""The element-wise arithmetic inside the tensor-core kernels, checked
against float64 references: the FMA-pipe exponential (error bound of its
fitted polynomial), the MUFU exponential, and the integer bf16 packing
(equal to round-to-nearest-even except on exact ties)."""
import numpy as np
import pytest
import torch

from block_sparse_full_b200 import ssa

pytestmark = pytest.mark.gpu


def _run(x):
    n = x.numel()
    xp = x.cuda()
    ep = torch.empty(n, dtype=torch.float32, device="cuda")
    em = torch.empty(n, dtype=torch.float32, device="cuda")
    bf = torch.empty(n, dtype=torch.int16, device="cuda")
    st = ssa.ssa_selftest_math(xp.data_ptr(), n, ep.data_ptr(), em.data_ptr(), bf.data_ptr(),
                               torch.cuda.current_stream().cuda_stream)
    assert st == 0, ssa.ssa_last_error()
    torch.cuda.synchronize()
    return ep.cpu().numpy(), em.cpu().numpy(), bf.cpu()


def test_exp2_polynomial_error_bound():
    # the kernels feed x = s*sigma*log2(e) - max: at most +8 (lazy rescale), down to large negatives
    x = torch.cat([torch.linspace(-125.0, 8.0, 400001), torch.tensor([0.0, -0.5, 0.5, 7.99, -124.9])])
    ep, em, _ = _run(x.float())
    ref = np.exp2(x.double().numpy())
    rel_poly = np.abs(ep / ref - 1)
    rel_mufu = np.abs(em / ref - 1)
    assert rel_poly.max() < 1.0e-4, rel_poly.max()   # fitted bound 7.5e-5
    assert rel_mufu.max() < 1.0e-5
    assert np.all(ep > 0) and np.all(np.isfinite(ep))


def test_exp2_polynomial_clamps_below_range():
    ep, em, _ = _run(torch.tensor([-200.0, -1e30, -np.inf], dtype=torch.float32))
    assert np.all(ep <= 2.0 ** -124) and np.all(ep >= 0)
    assert np.all(em == 0)  # the MUFU path gives exact zeros for masked keys


def test_alu_bf16_pack_matches_round_to_nearest_even_off_ties():
    g = torch.Generator().manual_seed(0)
    x = torch.cat([torch.randn(200000, generator=g) * 10.0 ** torch.randint(-20, 20, (200000,), generator=g),
                   torch.tensor([0.0, -0.0, 1.0, -1.0, 256.0, 3.0e38])]).float()
    _, _, bf = _run(x)
    rne = x.to(torch.bfloat16).view(torch.int16)
    bits = x.view(torch.int32)
    tie = (bits & 0xFFFF) == 0x8000
    assert torch.equal(bf[~tie], rne[~tie])
    # on a tie the magnitude rounds up (one bf16 ulp away from the even choice at most)
    diff = (bf[tie].int() - rne[tie].int()).abs()
    assert (diff <= 1).all()
