"""GPU block selection against the fp64 oracle on integer-valued data.

With small integers in Q and K every block mean is a dyadic rational and
every block score is exact in float64 on both sides, whatever the summation
order.  Key blocks are drawn from a few templates, so equal scores are
common: the tie rule (higher score first, then the lower block index) and the
forced blocks decide many rows, and no row is excused for a small score gap.
"""
import numpy as np
import pytest
import torch

from block_sparse_full_b200 import ssa
from oracle import ssa_oracle as O

from gpu_parity_util import DEV, assert_selection

pytestmark = pytest.mark.gpu

CASES = [
    # dtype, D, block, n blocks, topk, force_sink
    ("bf16", 128, 64, 70, 1, False),
    ("bf16", 128, 64, 70, 5, False),
    ("bf16", 128, 64, 70, 16, True),
    ("bf16", 64, 64, 97, 33, False),
    ("bf16", 64, 128, 40, 12, True),
    ("f32", 128, 128, 45, 7, False),
    ("f32", 64, 64, 130, 64, True),
    ("f32", 64, 128, 33, 5, False),
    ("bf16", 64, 64, 1100, 16, False),   # rows longer than 1024 blocks: the per-row kernel
    ("bf16", 128, 64, 1030, 7, True),
    ("bf16", 128, 64, 1024, 9, True),    # the longest rows of the 8-row kernel
]


def _data(dtype, D, block, n, seed, templates=3, B=1, H=None):
    H = H or (1 if n > 512 else 2)
    rng = np.random.default_rng(seed)
    T = n * block
    q = rng.integers(-2, 3, size=(B, H, T, D)).astype(np.float64)
    tmpl = rng.integers(-1, 2, size=(B, H, templates, block, D)).astype(np.float64)
    pick = rng.integers(0, templates, size=n)
    k = np.concatenate([tmpl[:, :, t] for t in pick], axis=2)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    return q, k, (torch.from_numpy(q).to(tdt).to(DEV), torch.from_numpy(k).to(tdt).to(DEV))


@pytest.mark.parametrize("dtype,D,block,n,topk,sink", CASES)
def test_selection_exact_ties(dtype, D, block, n, topk, sink):
    q, k, (dq, dk) = _data(dtype, D, block, n, seed=n * 7 + topk)
    flags = ssa.SSA_FLAG_FORCE_SINK if sink else 0
    p = ssa.params_for(dq, block, topk, flags=flags)
    got = ssa.select_blocks(p, dq, dk)
    want = O.select_blocks(q, k, block, topk, force_sink=sink)
    torch.cuda.synchronize()
    ssa.device_status()
    assert assert_selection(got, want, margin_tol=-1.0) == 0
    if topk > 1:  # ties really occur: some row has a zero gap at its budget boundary
        assert (want[3] == 0).any()


def test_selection_all_keys_equal_takes_lowest_indices():
    dtype, D, block, n, topk = "bf16", 128, 64, 50, 6
    q, k, (dq, dk) = _data(dtype, D, block, n, seed=3, templates=1)
    p = ssa.params_for(dq, block, topk)
    idx, cnt, _ = (t.cpu().numpy() for t in ssa.select_blocks(p, dq, dk))
    for i in range(n):
        want = list(range(min(i, topk - 1))) + [i]
        assert cnt[0, 0, i] == len(want)
        assert idx[0, 0, i, : len(want)].tolist() == want


@pytest.mark.parametrize("D,block,n,topk,B,H", [(128, 64, 70, 16, 2, 8), (64, 128, 40, 12, 2, 16),
                                                (128, 128, 36, 8, 4, 8)])
def test_selection_many_heads(D, block, n, topk, B, H):
    # more blocks than the pooling grid holds CTAs: every CTA streams several
    # blocks through its ring of stages
    q, k, (dq, dk) = _data("bf16", D, block, n, seed=n + H, B=B, H=H)
    p = ssa.params_for(dq, block, topk)
    got = ssa.select_blocks(p, dq, dk)
    want = O.select_blocks(q, k, block, topk)
    torch.cuda.synchronize()
    ssa.device_status()
    assert assert_selection(got, want, margin_tol=-1.0) == 0


@pytest.mark.parametrize("D,block", [(128, 64), (64, 128)])
def test_pooled_means_exact_over_the_bf16_range(D, block):
    # the float64 block means the selection ranks by are exact: values spread
    # over 36 binades with zeros and both signs (block sums still exact in
    # float64, so any summation order gives the oracle's value), and a block of
    # bf16 subnormals, pool to the oracle's means bit for bit.  The workspace
    # holds Qbar then Kbar, float64 [B, H, n, D] each, at 256-byte aligned offsets.
    B, H, n = 1, 3, 9
    T = n * block
    rng = np.random.default_rng(D + block)
    shape = (2, B, H, T, D)
    x = rng.choice([-1.0, 1.0], size=shape) * rng.integers(1, 256, size=shape) * 2.0 ** rng.integers(-18, 19, size=shape)
    x[rng.random(shape) < 0.05] = 0.0
    sub = slice(2 * block, 3 * block)  # block 2: subnormals and zeros only
    x[..., sub, :] = rng.integers(-127, 128, size=x[..., sub, :].shape) * 2.0 ** -133
    t = torch.from_numpy(x).to(torch.bfloat16)
    back = t.to(torch.float64).numpy()  # the values the GPU sees
    assert np.array_equal(back, x)
    dq, dk = t[0].to(DEV), t[1].to(DEV)
    p = ssa.params_for(dq, block, 4)
    ws = ssa.workspace(p, ssa.SSA_WS_SELECT, DEV)
    ssa.select_blocks(p, dq, dk, ws=ws)
    torch.cuda.synchronize()
    ssa.device_status()
    m = B * H * n * D
    half = (m * 8 + 255) // 256 * 256
    qbar = ws[: m * 8].view(torch.float64).cpu().numpy().reshape(B, H, n, D)
    kbar = ws[half: half + m * 8].view(torch.float64).cpu().numpy().reshape(B, H, n, D)
    for b in range(B):
        for h in range(H):
            np.testing.assert_array_equal(qbar[b, h], O.pool_blocks(back[0, b, h], block))
            np.testing.assert_array_equal(kbar[b, h], O.pool_blocks(back[1, b, h], block))
