"""ssa_select_blocks_noalloc: selection for callers that cannot allocate
device memory (it uses the library's own fixed scratch array instead of a
caller workspace).  Its results must equal ssa_select_blocks' bit for bit,
on consecutive calls that reuse the shared scratch with different shapes.
This file is collected last on purpose."""
import ctypes

import pytest
import torch

from block_sparse_full_b200 import ssa
from block_sparse_full_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _run_both(w):
    inp = make_inputs(w)
    q, k = inp["q"].to(DEV), inp["k"].to(DEV)
    p = ssa.params_for(q, w.block, w.topk, w.sm_scale, w.flags)
    ref = ssa.select_blocks(p, q, k)  # caller-allocated workspace
    n, words = w.n_blocks, (w.n_blocks + 31) // 32
    idx = torch.full((w.B, w.H, n, w.topk), 7, dtype=torch.int32, device=DEV)
    cnt = torch.full((w.B, w.H, n), 7, dtype=torch.int32, device=DEV)
    mask = torch.full((w.B, w.H, n, words), 7, dtype=torch.int32, device=DEV)
    st = ssa.ssa_select_blocks_noalloc(p, q.data_ptr(), k.data_ptr(), idx.data_ptr(),
                                       cnt.data_ptr(), mask.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
    assert st == ssa.SSA_OK, ssa.ssa_last_error()
    torch.cuda.synchronize()
    for got, want in zip((idx, cnt, mask), ref):
        assert torch.equal(got, want)


def test_noalloc_selection_matches_workspace_entry_point_twice():
    # two calls in a row on different shapes share (and overwrite) the scratch
    _run_both(Workload("na_a", B=2, H=4, T=4096, D=128, block=64, topk=8, dtype="bf16",
                       plant="hot", seed=21))
    _run_both(Workload("na_b", B=1, H=3, T=2048, D=64, block=128, topk=3, dtype="f32",
                       scale_data=False, flags=ssa.SSA_FLAG_FORCE_SINK, seed=22))
    ssa.device_status()


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # B*H*(T/block)*D = 2 * 1,048,576 > the 16 MiB scratch limit
    p = ssa.make_params(2, 16, 65536, 128, 64, 4, ssa.SSA_BF16)
    a = 1 << 20  # never dereferenced: rejected before any launch
    st = ssa.ssa_select_blocks_noalloc(p, a, a, a, a, a, None)
    assert st == ssa.SSA_ERR_UNSUPPORTED
    assert "scratch" in ssa.ssa_last_error()
