"""The tensor-core backward in several head groups.

Its dS workspace holds the dS blocks of a bounded number of heads; longer
sequences or more heads run as consecutive groups that share the buffer.
The full stream carries gradient to every key ("Sintesi Tecnica: SSA",
section 2, full attention stream), so dq, dk and dv of every group are held
to the oracle: a small problem forced into many groups through the budget
hook (every element), and a real grouped shape (T = 32768, five heads in two
groups) on the rows the oracle can take one by one: dq of sampled query rows
(dq_t depends on row t alone) and dk, dv of the last keys (only the last
query rows see them)."""
import numpy as np
import pytest
import torch

from block_sparse_full_b200 import ssa
from block_sparse_full_b200.inputs import Workload, make_inputs, upstream_grads
from oracle import ssa_oracle as O

from gpu_parity_util import (DEV, assert_selection, compare_grads, dq_rounding_budget,
                             oracle_select, params, sample_rows, to_dev)

pytestmark = pytest.mark.gpu


def _ds_bytes_per_head(T):
    ntk = (T + 127) // 128
    return (ntk * (T // 64) - ntk * (ntk - 1)) * 128 * 64 * 2


def _run(w, budget_heads=None, align=False):
    inp = make_inputs(w)
    g = upstream_grads(w)
    d = to_dev(inp)
    p = params(w, d["q"])
    o_sel = oracle_select(w, inp)
    g_sel = ssa.select_blocks(p, d["q"], d["k"])
    assert_selection(g_sel, o_sel)
    N = w.B * w.H * w.T * w.D
    ws_ = wc_ = float(N) if align else 0.0
    if budget_heads is not None:
        ssa.ssa_debug_set_ds_budget_bytes(int(budget_heads * _ds_bytes_per_head(w.T)))
    try:
        hc = ssa.ssa_bwd_heads_per_group(p)
        fwd = ssa.attn_fwd_dual(p, d["q"], d["k"], d["v"], g_sel[2])
        got = ssa.attn_bwd(p, d["q"], d["k"], d["v"], g_sel[2], fwd, g["dh_full"].to(DEV),
                           g["dh_sparse"].to(DEV), ws_, wc_)
        torch.cuda.synchronize()
        ssa.device_status()
    finally:
        ssa.ssa_debug_set_ds_budget_bytes(0)
    return inp, g, o_sel, hc, got, ws_, wc_


SMALL = Workload("bf16_B2_H3_T1216_groups", B=2, H=3, T=1216, D=128, block=64, topk=4,
                 dtype="bf16", plant="hot", seed=41)


@pytest.mark.parametrize("budget_heads,groups", [(1.0, 6), (2.5, 3), (4.0, 2)])
def test_small_problem_in_head_groups(budget_heads, groups):
    w = SMALL
    inp, g, o_sel, hc, got, ws_, wc_ = _run(w, budget_heads, align=budget_heads == 2.5)
    assert hc == int(budget_heads)
    assert -(-w.B * w.H // hc) == groups
    args = (inp["q"], inp["k"], inp["v"], o_sel[0], o_sel[1], w.block, w.sm_scale,
            g["dh_full"], g["dh_sparse"], ws_, wc_)
    want = O.attn_bwd(*args, n_total=inp["q"].numel())
    budget = dq_rounding_budget(*(O.f64(a) if isinstance(a, torch.Tensor) else a for a in args),
                                n_total=inp["q"].numel())
    compare_grads(f"bwd_groups/{groups}", "bf16", got, want, dq_budget=budget)


def test_grouped_results_equal_one_group():
    w = SMALL
    _, _, _, hc1, one, _, _ = _run(w, None)
    _, _, _, hc2, many, _, _ = _run(w, 1.0)
    assert hc1 == w.B * w.H and hc2 == 1
    for a, b in zip(one, many):  # per-head work is identical, so the bits are
        assert torch.equal(a, b)


def test_real_grouped_shape_T32768():
    w = Workload("bf16_H5_T32768_groups", B=1, H=5, T=32768, D=128, block=64, topk=16,
                 dtype="bf16", plant="hot", seed=42)
    inp, g, o_sel, hc, got, ws_, wc_ = _run(w)
    assert hc == (4 << 30) // _ds_bytes_per_head(w.T) == 3  # groups of 3 and 2 heads
    heads = [0, 4]  # one head of each group
    sub = lambda t: t[:, heads]
    args = (sub(inp["q"]), sub(inp["k"]), sub(inp["v"]), o_sel[0][:, heads], o_sel[1][:, heads],
            w.block, w.sm_scale, sub(g["dh_full"]), sub(g["dh_sparse"]), ws_, wc_)
    n = inp["q"].numel()
    rows = sample_rows(w.T, 4096, 6, seed=43)
    dq, _, _ = O.attn_bwd(*args, n_total=n, rows=rows)
    budget = dq_rounding_budget(*(O.f64(a) if isinstance(a, torch.Tensor) else a for a in args),
                                n_total=n, rows=rows)
    compare_grads("bwd_groups/T32768/dq_rows", "bf16", [sub(got[0])[:, :, rows]],
                  [dq[:, :, rows]], dq_budget=budget, names=("dq",))
    tail = np.arange(w.T - 256, w.T)  # keys that only the last 256 query rows see
    _, dk, dv = O.attn_bwd(*args, n_total=n, rows=tail)
    compare_grads("bwd_groups/T32768/dkdv_tail", "bf16",
                  [sub(got[1])[:, :, tail], sub(got[2])[:, :, tail]],
                  [dk[:, :, tail], dv[:, :, tail]], names=("dk", "dv"))
