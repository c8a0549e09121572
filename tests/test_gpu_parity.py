"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs.  Small cases compare every row; full-size workloads
compare sampled rows and properties that hold at any size."""
import numpy as np
import pytest
import torch

from block_sparse_full_b200 import ssa
from block_sparse_full_b200.inputs import WORKLOADS, Workload, make_inputs, upstream_grads
from oracle import ssa_oracle as O

from gpu_parity_util import (DEV, TOL, assert_selection, compare_fwd, compare_grads,
                             compare_loss, dq_rounding_budget, log, oracle_fwd, oracle_loss_rows,
                             oracle_mask_to_dev, oracle_select, params, sample_rows, to_dev)

pytestmark = pytest.mark.gpu

SIMT = ssa.SSA_FLAG_FORCE_SIMT
SINK = ssa.SSA_FLAG_FORCE_SINK

# small cases the oracle finishes in seconds: several 128-row tiles, ragged tails
SMALL = {
    "bf16_T1216_b64": Workload("bf16_T1216_b64", B=1, H=2, T=1216, D=128, block=64, topk=4,
                               dtype="bf16", plant="hot", seed=11),
    "bf16_B2_T640_b128_sink": Workload("bf16_B2_T640_b128_sink", B=2, H=2, T=640, D=128,
                                       block=128, topk=3, dtype="bf16", plant="sink", seed=12),
    "bf16_T448_d64": Workload("bf16_T448_d64", B=1, H=3, T=448, D=64, block=64, topk=2,
                              dtype="bf16", plant="hot", seed=13),
    "f32_T320_d128": Workload("f32_T320_d128", B=2, H=1, T=320, D=128, block=64, topk=2,
                              dtype="f32", scale_data=False, seed=14),
    "bf16_T64_single_block": Workload("bf16_T64_single_block", B=1, H=2, T=64, D=128,
                                      block=64, topk=1, dtype="bf16", seed=15),
}


def _fwd_case(w, flags=0, topk=None, rows=None):
    inp = make_inputs(w)
    o_sel = oracle_select(w, inp, topk, flags)
    d = to_dev(inp)
    p = params(w, d["q"], topk, flags)
    tc_expected = w.dtype == "bf16" and w.D in (64, 128) and not (flags & SIMT)
    assert ssa.ssa_kernel_path(p) == (1 if tc_expected else 0)
    g_sel = ssa.select_blocks(p, d["q"], d["k"])
    excused = assert_selection(g_sel, o_sel)
    mask = oracle_mask_to_dev(o_sel[2])
    out = ssa.attn_fwd_dual(p, d["q"], d["k"], d["v"], mask)
    ref, ref_abs = oracle_fwd(inp["q"], inp["k"], inp["v"], o_sel[0], o_sel[1], w.block,
                              w.sm_scale, rows=rows)
    torch.cuda.synchronize()
    ssa.device_status()
    return inp, d, p, o_sel, out, (ref, ref_abs), excused


# ------------------------------------------------------------------ selection + fwd

@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("flags", [0, SIMT])
def test_fwd_small(name, flags):
    w = SMALL[name]
    _, _, p, _, out, (ref, ref_abs), _ = _fwd_case(w, flags)
    compare_fwd(f"{name}/flags{flags}", w.dtype, out, ref, ref_abs=ref_abs)


def test_fwd_block128_force_sink_flag():
    w = SMALL["bf16_B2_T640_b128_sink"]
    _, _, _, o_sel, out, (ref, ref_abs), _ = _fwd_case(w, SINK)
    assert (o_sel[0][..., 1:, 0] == 0).all()  # block 0 first in every S_i, i > 0
    compare_fwd("b128/force_sink", w.dtype, out, ref, ref_abs=ref_abs)


def test_f32_T1024_workload():
    w = WORKLOADS["f32_T1024_d64"]
    inp, d, p, o_sel, out, (ref, ref_abs), _ = _fwd_case(w)
    compare_fwd(w.name, "f32", out, ref, ref_abs=ref_abs)
    loss = ssa.align_loss(p, out["sqdiff"], 1.0, 0.5).cpu().numpy()
    ls, lc = O.align_loss(ref["h_full"], ref["h_sparse"], 1.0, 0.5)
    assert abs(loss[0] - ls) <= TOL["f32"]["loss_rel"] * ls
    assert abs(loss[1] - lc) <= TOL["f32"]["loss_rel"] * lc
    log(w.name + "/loss", rel=abs(loss[0] - ls) / ls)


def test_T8192_workload_sampled_rows():
    w = WORKLOADS["bf16_T8192_H16_hot"]
    rows = sample_rows(w.T, w.block, 4, seed=1)
    inp, d, p, o_sel, out, (ref, ref_abs), excused = _fwd_case(w, rows=rows)
    assert ssa.ssa_kernel_path(p) == 1
    compare_fwd(w.name, "bf16", out, ref, rows=rows, ref_abs=ref_abs)
    # planted hot blocks are picked by every later query block
    hot = inp["hot_blocks"].numpy()
    sel = O.block_selection_matrix(o_sel[0], o_sel[1])
    n = w.n_blocks
    for h in range(w.H):
        for j in np.flatnonzero(hot[0, h]):
            assert sel[0, h, j + 1:, j].all()
    # loss: GPU reduction vs fp64 sum of the GPU rows
    loss = ssa.align_loss(p, out["sqdiff"], 2.0, 3.0).cpu().numpy()
    host = out["sqdiff"].double().sum().item() / (w.B * w.H * w.T * w.D)
    assert abs(loss[0] - 2.0 * host) <= 1e-6 * 2.0 * host
    assert abs(loss[1] - 3.0 * host) <= 1e-6 * 3.0 * host
    # every row of all 16 heads against the oracle, and the loss against the oracle's
    ref_loss, ref_sq, budget = oracle_loss_rows(inp["q"], inp["k"], inp["v"], o_sel[0], o_sel[1],
                                                w.block, w.sm_scale, "bf16")
    compare_loss(w.name, p, out["sqdiff"], ref_loss, ref_sq, budget, w.B * w.H * w.T * w.D)


def test_T16384_budget_sweep():
    w = WORKLOADS["bf16_T16384_H16_sweep"]
    inp = make_inputs(w)
    d = to_dev(inp)
    rows = sample_rows(w.T, w.block, 2, seed=3)
    heads = [0, 7]
    prev_delta = None
    for k in w.sweep:
        o_sel = oracle_select(w, inp, k)
        p = params(w, d["q"], k)
        assert_selection(ssa.select_blocks(p, d["q"], d["k"]), o_sel)
        out = ssa.attn_fwd_dual(p, d["q"], d["k"], d["v"], oracle_mask_to_dev(o_sel[2]))
        loss = ssa.align_loss(p, out["sqdiff"]).cpu().numpy()
        sub = {n: inp[n][:, heads] for n in "qkv"}
        ref, ref_abs = oracle_fwd(sub["q"], sub["k"], sub["v"], o_sel[0][:, heads],
                                  o_sel[1][:, heads], w.block, w.sm_scale, rows=rows)
        gsub = {n: t[:, heads] for n, t in out.items()}
        compare_fwd(f"{w.name}/k{k}", "bf16", gsub, ref, rows=rows, ref_abs=ref_abs)
        delta = out["delta"].cpu().numpy()
        assert (delta >= -1e-6).all() and (delta <= 1 + 1e-6).all()
        if prev_delta is not None:  # nested budgets: discarded mass cannot grow
            assert (delta <= prev_delta + TOL["bf16"]["delta"]).all()
            assert delta.mean() <= prev_delta.mean()
        prev_delta = delta
        log(f"{w.name}/k{k}", delta_mean=delta.mean(), loss=loss[0])
    # k = all causal blocks: both streams coincide, nothing is discarded
    assert w.sweep[-1] == w.n_blocks
    assert (prev_delta == 0).all()
    torch.testing.assert_close(out["h_sparse"], out["h_full"], rtol=0, atol=0)
    assert loss[0] == 0.0


def test_T65536_sink_workload():
    w = WORKLOADS["bf16_T65536_H8_sink"]
    inp = make_inputs(w)
    d = to_dev(inp)
    o_sel = oracle_select(w, inp)
    p = params(w, d["q"])
    assert_selection(ssa.select_blocks(p, d["q"], d["k"]), o_sel)
    assert (o_sel[0][..., 1:, 0] == 0).all()  # the heavy sink wins for every query block
    # with the sink forced, the selection is identical
    p_sink = params(w, d["q"], flags=SINK)
    g2 = ssa.select_blocks(p_sink, d["q"], d["k"])
    assert (g2[0].cpu().numpy() == o_sel[0]).all()
    out = ssa.attn_fwd_dual(p, d["q"], d["k"], d["v"], oracle_mask_to_dev(o_sel[2]))
    rows = np.unique(np.concatenate([sample_rows(w.T, 4096, 8, seed=5), [w.T - 1]]))
    heads = [0, 5]
    ref, ref_abs = oracle_fwd(inp["q"][:, heads], inp["k"][:, heads], inp["v"][:, heads],
                              o_sel[0][:, heads], o_sel[1][:, heads], w.block, w.sm_scale,
                              rows=rows)
    compare_fwd(w.name, "bf16", {n: t[:, heads] for n, t in out.items()}, ref, rows=rows,
                ref_abs=ref_abs)


# ------------------------------------------------------------------ backward

def _bwd_case(case, w, flags, ws_, wc_, heads=None):
    """GPU selection (checked bit-exact against the oracle) -> forward ->
    backward, and dq, dk, dv of ``heads`` against the oracle.
    dq of bf16 inputs also gets the budget for the bf16 rounding of the
    forward outputs that the backward reads (``dq_rounding_budget``); its
    error against the plain 2e-2 x max|dq| bound is logged beside it."""
    inp = make_inputs(w)
    g = upstream_grads(w) if ws_ == 0 and wc_ == 0 else None
    d = to_dev(inp)
    o_sel = oracle_select(w, inp)
    p = params(w, d["q"], flags=flags)
    g_sel = ssa.select_blocks(p, d["q"], d["k"])
    assert_selection(g_sel, o_sel)
    mask = g_sel[2]
    fwd = ssa.attn_fwd_dual(p, d["q"], d["k"], d["v"], mask)
    dhf = g["dh_full"].to(DEV) if g else None
    dhs = g["dh_sparse"].to(DEV) if g else None
    got = ssa.attn_bwd(p, d["q"], d["k"], d["v"], mask, fwd, dhf, dhs, ws_, wc_)
    torch.cuda.synchronize()
    ssa.device_status()
    hs = slice(None) if heads is None else heads
    zeros = np.zeros(inp["q"][:, hs].shape)
    args = (inp["q"][:, hs], inp["k"][:, hs], inp["v"][:, hs], o_sel[0][:, hs], o_sel[1][:, hs],
            w.block, w.sm_scale, g["dh_full"][:, hs] if g else zeros,
            g["dh_sparse"][:, hs] if g else zeros, ws_, wc_)
    want = O.attn_bwd(*args, n_total=inp["q"].numel())
    budget = dq_rounding_budget(*(O.f64(a) if isinstance(a, torch.Tensor) else a for a in args),
                                n_total=inp["q"].numel()) if w.dtype == "bf16" else None
    compare_grads(case, w.dtype, [t[:, hs] for t in got], want, dq_budget=budget)


@pytest.mark.parametrize("name", ["bf16_T1216_b64", "f32_T320_d128", "bf16_T448_d64",
                                  "bf16_B2_T640_b128_sink"])
@pytest.mark.parametrize("flags", [0, SIMT])
def test_bwd_small_upstream(name, flags):
    _bwd_case(f"bwd/{name}/flags{flags}", SMALL[name], flags, 0.0, 0.0)


@pytest.mark.parametrize("name", ["bf16_T1216_b64", "f32_T320_d128"])
def test_bwd_small_alignment_only(name):
    w = SMALL[name]
    N = w.B * w.H * w.T * w.D
    _bwd_case(f"bwd_align/{name}", w, 0, float(N), float(N))


@pytest.mark.parametrize("mode", ["upstream", "alignment_only"])
def test_train_workload_bwd_head0(mode):
    w = WORKLOADS["bf16_B4_H32_T4096_train"]
    N = w.B * w.H * w.T * w.D
    ws_ = wc_ = 0.0 if mode == "upstream" else float(N)
    _bwd_case(f"{w.name}/{mode}", w, 0, ws_, wc_, heads=[0])


def test_train_workload_selection_fwd_and_loss():
    """The training workload (B4 H32 T4096): selection of all 128 heads bit
    exact, the forward outputs of head 0 of every batch on every row, the
    per-row squared difference of every row and the loss against the
    oracle's."""
    w = WORKLOADS["bf16_B4_H32_T4096_train"]
    inp = make_inputs(w)
    d = to_dev(inp)
    o_sel = oracle_select(w, inp)
    p = params(w, d["q"])
    assert ssa.ssa_kernel_path(p) == 1
    g_sel = ssa.select_blocks(p, d["q"], d["k"])
    assert_selection(g_sel, o_sel)
    out = ssa.attn_fwd_dual(p, d["q"], d["k"], d["v"], g_sel[2])
    torch.cuda.synchronize()
    ssa.device_status()
    heads = [0]
    ref, ref_abs = oracle_fwd(inp["q"][:, heads], inp["k"][:, heads], inp["v"][:, heads],
                              o_sel[0][:, heads], o_sel[1][:, heads], w.block, w.sm_scale)
    compare_fwd(w.name + "/head0", "bf16", {n: t[:, heads] for n, t in out.items()}, ref,
                ref_abs=ref_abs)
    ref_loss, ref_sq, budget = oracle_loss_rows(inp["q"], inp["k"], inp["v"], o_sel[0], o_sel[1],
                                                w.block, w.sm_scale, "bf16")
    compare_loss(w.name, p, out["sqdiff"], ref_loss, ref_sq, budget, w.B * w.H * w.T * w.D)


# head dim 64 (Llama-3.2-1B-sized heads) on the tensor-core path
D64 = Workload("bf16_H8_T4096_d64", B=1, H=8, T=4096, D=64, block=64, topk=16, dtype="bf16",
               plant="hot", grads=True, seed=16)


def test_d64_heads_fwd_sampled_rows_and_bwd():
    w = D64
    rows = sample_rows(w.T, w.block, 3, seed=17)
    inp, d, p, o_sel, out, (ref, ref_abs), _ = _fwd_case(w, rows=rows)
    assert ssa.ssa_kernel_path(p) == 1
    compare_fwd(w.name, "bf16", out, ref, rows=rows, ref_abs=ref_abs)
    _bwd_case(w.name + "/bwd", w, 0, 0.0, 0.0, heads=[0, 5])


# ------------------------------------------------------------------ robustness

def test_fwd_bitwise_repeatable_and_in_bounds():
    w = SMALL["bf16_T1216_b64"]
    inp = make_inputs(w)
    d = to_dev(inp)
    p = params(w, d["q"])
    idx, cnt, mask = ssa.select_blocks(p, d["q"], d["k"])
    # outputs live inside larger buffers filled with a canary; the tails must survive
    CAN = 12345.0
    def canary(shape, dtype):
        n = int(np.prod(shape))
        buf = torch.full((n + 4096,), CAN, dtype=dtype, device=DEV)
        return buf, buf[:n].view(shape)
    bufs = {}
    out = {}
    for nm in ("h_full", "h_sparse"):
        bufs[nm], out[nm] = canary(d["q"].shape, d["q"].dtype)
    for nm in ("delta", "lse_full", "lse_sparse", "sqdiff"):
        bufs[nm], out[nm] = canary((w.B, w.H, w.T), torch.float32)
    ssa.attn_fwd_dual(p, d["q"], d["k"], d["v"], mask, out=out)
    first = {k: v.clone() for k, v in out.items()}
    ssa.attn_fwd_dual(p, d["q"], d["k"], d["v"], mask, out=out)
    torch.cuda.synchronize()
    for nm in out:
        assert torch.equal(first[nm], out[nm]), nm
        n = out[nm].numel()
        can = torch.tensor(CAN, dtype=bufs[nm].dtype, device=DEV)  # as stored (bf16 rounds it)
        assert (bufs[nm][n:] == can).all(), f"{nm} written out of bounds"
    l1 = ssa.align_loss(p, out["sqdiff"]).cpu()
    l2 = ssa.align_loss(p, out["sqdiff"]).cpu()
    assert torch.equal(l1, l2)
    ssa.device_status()


def test_selection_repeatable_and_consistent():
    w = WORKLOADS["bf16_T8192_H16_hot"].with_(H=4)
    d = to_dev(make_inputs(w))
    p = params(w, d["q"])
    a = ssa.select_blocks(p, d["q"], d["k"])
    b = ssa.select_blocks(p, d["q"], d["k"])
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    idx, cnt, mask = (t.cpu().numpy() for t in a)
    m = mask.view(np.uint32)
    n = w.n_blocks
    assert (cnt == np.minimum(np.arange(n) + 1, w.topk)).all()
    for i in range(0, n, 17):
        row = idx[0, 0, i]
        c = cnt[0, 0, i]
        assert (np.diff(row[:c]) > 0).all() and (row[c:] == -1).all() and row[c - 1] == i
        bits = [j for j in range(n) if (m[0, 0, i, j // 32] >> (j % 32)) & 1]
        assert bits == row[:c].tolist()
