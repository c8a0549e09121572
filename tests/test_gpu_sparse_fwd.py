"""GPU parity of the sparse-only forward (inference mode: only the selected
key blocks are visited) against the fp64 oracle's gathered-key sparse
attention, on the same seeded inputs and selections."""
import numpy as np
import pytest
import torch

from block_sparse_full_b200 import ssa
from block_sparse_full_b200.inputs import WORKLOADS, Workload, make_inputs
from oracle import ssa_oracle as O

from gpu_parity_util import (DEV, TOL, log, oracle_mask_to_dev, oracle_select, params,
                             sample_rows, to_dev)
from test_gpu_parity import SIMT, SINK, SMALL

pytestmark = pytest.mark.gpu


def compare_sparse(case, dtype, gpu, ref, rows=None):
    tol = TOL[dtype]
    sl = (slice(None), slice(None), rows) if rows is not None else (slice(None),) * 3
    g = gpu["h_sparse"][sl].float().cpu().numpy()
    e = float(np.abs(g - ref["h"]).max())
    scale = float(np.abs(ref["h"]).max())
    assert np.isfinite(g).all()
    assert e <= tol["h"], f"{case} h: max-abs {e:.3e}"
    assert e <= tol["h_rel"] * max(scale, 1.0 if dtype == "f32" else scale), f"{case} h: {e:.3e}"
    el = float(np.abs(gpu["lse_sparse"][sl].cpu().numpy() - ref["lse"]).max())
    assert el <= tol["lse"], f"{case} lse: {el:.3e}"
    log(case, h=e, h_rel=e / max(scale, 1e-30), lse=el)


def _case(w, flags=0, topk=None, rows=None, heads=None):
    inp = make_inputs(w)
    o_sel = oracle_select(w, inp, topk, flags)
    d = to_dev(inp)
    p = params(w, d["q"], topk, flags)
    mask = oracle_mask_to_dev(o_sel[2])
    out = ssa.attn_fwd_sparse(p, d["q"], d["k"], d["v"], mask)
    torch.cuda.synchronize()
    ssa.device_status()
    hs = slice(None) if heads is None else heads
    ref = O.attn_fwd_sparse(inp["q"][:, hs], inp["k"][:, hs], inp["v"][:, hs], o_sel[0][:, hs],
                            o_sel[1][:, hs], w.block, w.sm_scale, rows=rows)
    got = {n: t[:, hs] for n, t in out.items()}
    return inp, d, p, mask, got, ref


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("flags", [0, SIMT])
def test_sparse_fwd_small(name, flags):
    w = SMALL[name]
    _, _, p, _, out, ref = _case(w, flags)
    tc = w.dtype == "bf16" and w.D in (64, 128) and not (flags & SIMT)
    assert ssa.ssa_kernel_path(p) == (1 if tc else 0)
    compare_sparse(f"sparse/{name}/flags{flags}", w.dtype, out, ref)


def test_sparse_fwd_force_sink_and_full_budget():
    w = SMALL["bf16_B2_T640_b128_sink"]
    _, _, _, _, out, ref = _case(w, SINK)
    compare_sparse("sparse/b128/force_sink", "bf16", out, ref)
    # every causal block selected: the sparse stream is full causal attention
    n = w.T // w.block
    inp, d, p, mask, out, ref = _case(w, topk=n)
    dual = ssa.attn_fwd_dual(p, d["q"], d["k"], d["v"], mask)
    compare_sparse("sparse/b128/full_budget", "bf16", out, ref)
    e = float((out["h_sparse"].float() - dual["h_full"].float()).abs().max())
    assert e <= TOL["bf16"]["h"], e


def test_sparse_fwd_T8192_matches_dual_and_oracle():
    w = WORKLOADS["bf16_T8192_H16_hot"]
    rows = sample_rows(w.T, w.block, 4, seed=21)
    heads = [0, 9]
    inp, d, p, mask, out, ref = _case(w, rows=rows, heads=heads)
    assert ssa.ssa_kernel_path(p) == 1
    compare_sparse(w.name + "/sparse", "bf16", out, ref, rows=rows)
    # same quantities as the dual forward's sparse stream (every head, every row)
    full = ssa.attn_fwd_sparse(p, d["q"], d["k"], d["v"], mask)
    dual = ssa.attn_fwd_dual(p, d["q"], d["k"], d["v"], mask)
    torch.cuda.synchronize()
    e = float((full["h_sparse"].float() - dual["h_sparse"].float()).abs().max())
    el = float((full["lse_sparse"] - dual["lse_sparse"]).abs().max())
    assert e <= TOL["bf16"]["h"] and el <= TOL["bf16"]["lse"], (e, el)
    log(w.name + "/sparse_vs_dual", h=e, lse=el)


def test_sparse_fwd_T65536_sink_sampled_rows():
    w = WORKLOADS["bf16_T65536_H8_sink"]
    rows = np.unique(np.concatenate([sample_rows(w.T, 4096, 8, seed=23), [w.T - 1]]))
    _, _, p, _, out, ref = _case(w, rows=rows, heads=[2, 7])
    compare_sparse(w.name + "/sparse", "bf16", out, ref, rows=rows)


def test_sparse_fwd_T131072_sampled_rows():
    # 1024 key tiles per head at the last query tile: the CTA's list of
    # selected tiles is compacted over several 384-tile chunks
    w = Workload("bf16_T131072_H2_sink", B=1, H=2, T=131072, D=128, block=128, topk=16,
                 dtype="bf16", plant="sink", seed=47)
    rows = np.unique(np.concatenate([sample_rows(w.T, 16384, 6, seed=29), [w.T - 1]]))
    _, _, p, _, out, ref = _case(w, rows=rows)
    assert ssa.ssa_kernel_path(p) == 1
    compare_sparse(w.name + "/sparse", "bf16", out, ref, rows=rows)


def test_sparse_fwd_repeatable():
    w = SMALL["bf16_T1216_b64"]
    inp, d, p, mask, out, _ = _case(w, rows=[0])
    again = ssa.attn_fwd_sparse(p, d["q"], d["k"], d["v"], mask)
    torch.cuda.synchronize()
    assert torch.equal(out["h_sparse"], again["h_sparse"])
    assert torch.equal(out["lse_sparse"], again["lse_sparse"])
