"""Failure detection without a GPU fault.

Every mbarrier wait inside the tensor-core kernels is bounded.  The
primitive itself is tested on a flag that nothing sets: a self-test kernel
waits on an mbarrier no one arrives at and must give up, leaving a record
that the host reads as SSA_ERR_TIMEOUT.  The kernels' own limit can be
shortened; whichever way their waits then end, the context must stay usable
and later results must be exact."""
import time

import numpy as np
import pytest
import torch

from block_sparse_full_b200 import ssa
from block_sparse_full_b200.inputs import Workload, make_inputs, upstream_grads
from oracle import ssa_oracle as O

pytestmark = pytest.mark.gpu


def _stream():
    return torch.cuda.current_stream().cuda_stream


def test_bounded_wait_on_a_flag_nothing_sets():
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert ssa.ssa_device_status(_stream()) == ssa.SSA_OK
    t0 = time.perf_counter()
    assert ssa.ssa_selftest_wait_timeout(2_000_000, flag.data_ptr(), _stream()) == ssa.SSA_OK
    st = ssa.ssa_device_status(_stream())  # synchronises
    elapsed = time.perf_counter() - t0
    assert st == ssa.SSA_ERR_TIMEOUT
    assert "expired" in ssa.ssa_last_error()
    assert flag.item() == 1
    assert 0.002 <= elapsed < 5.0  # it waited its 2 ms and no more than the guard
    assert ssa.ssa_device_status(_stream()) == ssa.SSA_OK  # the record was cleared


def test_short_kernel_wait_limit_keeps_context_usable():
    w = Workload("fail_bf16_T1216", B=1, H=2, T=1216, D=128, block=64, topk=4, dtype="bf16",
                 plant="hot", seed=31)
    inp = make_inputs(w)
    g = upstream_grads(w)
    q, k, v = (inp[n].cuda() for n in "qkv")
    p = ssa.params_for(q, w.block, w.topk, w.sm_scale)
    assert ssa.ssa_kernel_path(p) == 1
    idx, cnt, mask = ssa.select_blocks(p, q, k)
    good = ssa.attn_fwd_dual(p, q, k, v, mask)
    torch.cuda.synchronize()
    assert ssa.ssa_device_status(_stream()) == ssa.SSA_OK
    ssa.ssa_debug_set_wait_limit_ns(100)
    try:
        ssa.attn_fwd_dual(p, q, k, v, mask)
        assert ssa.ssa_device_status(_stream()) in (ssa.SSA_OK, ssa.SSA_ERR_TIMEOUT)
        ssa.attn_bwd(p, q, k, v, mask, good, g["dh_full"].cuda(), g["dh_sparse"].cuda(), 1.0, 1.0)
        assert ssa.ssa_device_status(_stream()) in (ssa.SSA_OK, ssa.SSA_ERR_TIMEOUT)
    finally:
        ssa.ssa_debug_set_wait_limit_ns(0)
    out = ssa.attn_fwd_dual(p, q, k, v, mask)
    torch.cuda.synchronize()
    assert ssa.ssa_device_status(_stream()) == ssa.SSA_OK
    for name in good:
        assert torch.equal(out[name], good[name])
    o_idx, o_cnt, _, _ = O.select_blocks(inp["q"], inp["k"], w.block, w.topk)
    ref = O.attn_fwd_dual(inp["q"], inp["k"], inp["v"], o_idx, o_cnt, w.block, w.sm_scale)
    for name in ("h_full", "h_sparse"):
        err = np.abs(out[name].float().cpu().numpy() - ref[name]).max()
        assert err <= 1e-2 * np.abs(ref[name]).max()


def test_short_wait_limit_in_the_decode_step():
    # The decode step's waits (its copies, and the leader's wait for the other
    # CTAs' partials) expire under a 100 ns limit; the leader then waits for
    # the partials that are still being written into its shared memory before
    # it leaves.  The context stays usable and the next step is exact.
    w = Workload("fail_bf16_decode", B=1, H=4, T=8192, D=128, block=64, topk=16, dtype="bf16",
                 plant="hot", seed=32)
    inp = make_inputs(w)
    p = ssa.params_for(inp["q"].cuda(), w.block, w.topk, w.sm_scale)
    cache = ssa.DecodeCache(p, "cuda", inp["k"].dtype)
    cache.k.copy_(inp["k"].cuda())
    cache.v.copy_(inp["v"].cuda())
    t = w.T - 1
    q_t = inp["q"][:, :, t].contiguous()
    good = cache.step(t, q_t.cuda())
    good = {n: x.clone() for n, x in good.items()}
    torch.cuda.synchronize()
    assert ssa.ssa_device_status(_stream()) == ssa.SSA_OK
    ssa.ssa_debug_set_wait_limit_ns(100)
    try:
        cache.step(t, q_t.cuda())
        assert ssa.ssa_device_status(_stream()) in (ssa.SSA_OK, ssa.SSA_ERR_TIMEOUT)
    finally:
        ssa.ssa_debug_set_wait_limit_ns(0)
    out = cache.step(t, q_t.cuda())
    torch.cuda.synchronize()
    assert ssa.ssa_device_status(_stream()) == ssa.SSA_OK
    for name in good:
        assert torch.equal(out[name], good[name]), name
    ref = O.decode_step(q_t, inp["k"], inp["v"], t, w.block, w.topk, w.sm_scale)
    np.testing.assert_array_equal(out["idx"].cpu().numpy(), ref["idx"])
    err = np.abs(out["h"].float().cpu().numpy() - ref["h"]).max()
    assert err <= 1e-2 * np.abs(ref["h"]).max()
