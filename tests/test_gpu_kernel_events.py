"""The measurement hook that brackets the backward's kernels with caller
events (used by the benchmark to time the dK/dV kernel on its own)."""
import ctypes

import pytest
import torch

from block_sparse_full_b200 import ssa
from block_sparse_full_b200.inputs import WORKLOADS, make_inputs, upstream_grads

pytestmark = pytest.mark.gpu


def test_kernel_events_bracket_the_backward_kernels():
    w = WORKLOADS["bf16_T8192_H16_hot"]
    inp, g = make_inputs(w), upstream_grads(w)
    q, k, v = (inp[n][:, :2].contiguous().cuda() for n in "qkv")  # two heads
    p = ssa.params_for(q, w.block, w.topk)
    assert ssa.ssa_kernel_path(p) == 1
    idx, cnt, mask = ssa.select_blocks(p, q, k)
    out = ssa.attn_fwd_dual(p, q, k, v, mask)
    dhf, dhs = (g[n][:, :2].contiguous().cuda() for n in ("dh_full", "dh_sparse"))
    stream = torch.cuda.current_stream()
    outer = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for e in ev:
        e.record(stream)
    handles = (ctypes.c_void_p * 4)(*[e.cuda_event for e in ev])
    assert ssa.ssa_debug_set_kernel_events(handles, 3) == ssa.SSA_ERR_INVALID_ARG
    assert ssa.ssa_debug_set_kernel_events(handles, 4) == 0
    try:
        outer[0].record(stream)
        ssa.attn_bwd(p, q, k, v, mask, out, dhf, dhs, 1.0, 1.0)
        outer[1].record(stream)
    finally:
        assert ssa.ssa_debug_set_kernel_events(None, 0) == 0
    torch.cuda.synchronize()
    parts = [ev[i].elapsed_time(ev[i + 1]) for i in range(3)]
    total = outer[0].elapsed_time(outer[1])
    assert all(t > 0 for t in parts), parts
    assert sum(parts) <= total * 1.01 + 0.01, (parts, total)
    assert parts[1] > parts[0]  # the dK/dV kernel outweighs the row preprocess
