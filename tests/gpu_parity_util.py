"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare with the fp64 oracle on the same seeded inputs."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

from block_sparse_full_b200 import ssa
from oracle import ssa_oracle as O

DEV = "cuda:0"
LOG = os.environ.get("SSA_PARITY_LOG")  # optional JSONL of measured errors

# Tolerances.  fp32 inputs: exact-fp32 SIMT arithmetic, 1e-4 on outputs.
# bf16 inputs: fp32 accumulate; the outputs are rounded to bf16 (relative
# 2^-9) and the tensor-core path rounds the softmax weights P to bf16 before
# the PV product (relative 2^-9 each, averaging out over keys).  The bound
# used is the 2e-2 max-abs ceiling and, tighter, 1e-2 of the largest output
# magnitude (about five bf16 ulps at that magnitude).
TOL = {
    "f32": dict(h=1e-4, h_rel=1e-4, delta=1e-5, lse=1e-4, loss_rel=1e-4, grad_rel=1e-4),
    "bf16": dict(h=2e-2, h_rel=1e-2, delta=2e-3, lse=2e-3, loss_rel=2e-2, grad_rel=2e-2),
}


def log(case: str, **vals):
    if LOG:
        with open(LOG, "a") as f:
            f.write(json.dumps({"case": case, **{k: float(v) for k, v in vals.items()}}) + "\n")


def to_dev(inp):
    return {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def params(w, q, topk=None, flags=0):
    return ssa.params_for(q, w.block, topk if topk is not None else w.topk, w.sm_scale,
                          flags | w.flags)


def mask_u32(mask: torch.Tensor) -> np.ndarray:
    return mask.cpu().numpy().view(np.uint32)


def assert_selection(gpu, ref, margin_tol=1e-12):
    """idx/cnt/mask bit-exact; a row may differ only where the oracle's
    last-selected/first-rejected score gap is below margin_tol."""
    g_idx, g_cnt, g_mask = gpu
    o_idx, o_cnt, o_mask, margin = ref
    gi, gc, gm = g_idx.cpu().numpy(), g_cnt.cpu().numpy(), mask_u32(g_mask)
    bad = (gi != o_idx).any(-1) | (gc != o_cnt) | (gm != o_mask).any(-1)
    excused = bad & (margin <= margin_tol)
    assert not (bad & ~excused).any(), \
        f"{int((bad & ~excused).sum())} selection rows differ (first at {np.argwhere(bad & ~excused)[0]})"
    return int(excused.sum())


def oracle_mask_to_dev(o_mask):
    return torch.from_numpy(o_mask.view(np.int32).copy()).to(DEV)


def compare_fwd(case, dtype, gpu, ref, rows=None):
    """Compare GPU forward outputs (all rows) with oracle outputs (``rows``)."""
    tol = TOL[dtype]
    sl = (slice(None), slice(None), rows) if rows is not None else (slice(None),) * 3
    errs = {}
    for name in ("h_full", "h_sparse"):
        g = gpu[name][sl].float().cpu().numpy()
        r = ref[name]
        e = float(np.abs(g - r).max())
        scale = float(np.abs(r).max())
        errs[name] = e
        errs[name + "_rel"] = e / max(scale, 1e-30)
        assert np.isfinite(g).all(), name
        assert e <= tol["h"], f"{case} {name}: max-abs {e:.3e} > {tol['h']}"
        assert e <= tol["h_rel"] * max(scale, 1.0 if dtype == "f32" else scale), \
            f"{case} {name}: max-abs {e:.3e} > {tol['h_rel']} x max|ref| {scale:.3e}"
    g = gpu["delta"][sl].cpu().numpy()
    errs["delta"] = float(np.abs(g - ref["delta"]).max())
    assert errs["delta"] <= tol["delta"], f"{case} delta {errs['delta']:.3e}"
    for name in ("lse_full", "lse_sparse"):
        g = gpu[name][sl].cpu().numpy()
        errs[name] = float(np.abs(g - ref[name]).max())
        assert errs[name] <= tol["lse"], f"{case} {name} {errs[name]:.3e}"
    g = gpu["sqdiff"][sl].cpu().numpy().astype(np.float64)
    errs["sqdiff_rel"] = float(np.abs(g - ref["sqdiff"]).sum() / max(ref["sqdiff"].sum(), 1e-30))
    log(case, **errs)
    return errs


def dq_rounding_budget(q, k, v, idx, cnt, block, scale, dh_full, dh_sparse, w_s, w_c, n_total):
    """Elementwise bound on the dq deviation that rounding the forward outputs
    to bf16 alone causes.  The backward takes D_f = G_f . h_full and
    D_s = G_s . h_sparse from the stored (bf16) outputs; a perturbation dD
    of D enters dq_t as -sigma * dD(t) * sum_s P(t,s) k_s, and that
    softmax-weighted mean key is the attention output with v := k.  All
    values come from the oracle; the bf16 rounding is torch's on the host."""
    ref = O.attn_fwd_dual(q, k, v, idx, cnt, block, scale)
    kbar = O.attn_fwd_dual(q, k, k, idx, cnt, block, scale)
    hf, hs = ref["h_full"], ref["h_sparse"]
    r16 = lambda a: torch.from_numpy(a).to(torch.bfloat16).double().numpy()
    g_f, g_s = O.alignment_upstream(hf, hs, dh_full, dh_sparse, w_s, w_c, n_total)
    dDf = (np.abs(g_f) * np.abs(hf - r16(hf))).sum(-1, keepdims=True)
    dDs = (np.abs(g_s) * np.abs(hs - r16(hs))).sum(-1, keepdims=True)
    return scale * (dDf * np.abs(kbar["h_full"]) + dDs * np.abs(kbar["h_sparse"]))


def compare_grads(case, dtype, got, want, dq_budget=None):
    """max |g - ref| <= tol * max|ref| per tensor; for dq also allow the
    (elementwise) deviation caused by the bf16 rounding of the forward
    outputs, ``dq_budget`` from ``dq_rounding_budget``."""
    tol = TOL[dtype]["grad_rel"]
    errs = {}
    for name, g, r in zip(("dq", "dk", "dv"), got, want):
        g = g.float().cpu().numpy()
        diff = np.abs(g - r)
        scale = float(np.abs(r).max())
        errs[name + "_rel"] = float(diff.max()) / scale
        assert np.isfinite(g).all(), name
        allowed = tol * scale
        if name == "dq" and dq_budget is not None:
            allowed = allowed + 1.25 * dq_budget
            errs["dq_budget_ratio"] = float((diff / allowed).max())
        ok = diff <= allowed
        assert ok.all(), (f"{case} {name}: max err {diff.max():.3e} (tol {tol} x {scale:.3e}); "
                          f"worst at {np.unravel_index(np.argmax(diff - allowed), diff.shape)}")
    log(case, **errs)
    return errs


def oracle_select(w, inp, topk=None, flags=0):
    f = flags | w.flags
    return O.select_blocks(inp["q"], inp["k"], w.block, topk if topk is not None else w.topk,
                           force_sink=bool(f & ssa.SSA_FLAG_FORCE_SINK))


def sample_rows(T, block, per_block, seed=0):
    """First and last row of every block plus seeded extras."""
    r = np.random.default_rng(seed)
    rows = set()
    for b0 in range(0, T, block):
        rows.update((b0, b0 + block - 1))
        rows.update(int(x) for x in r.integers(b0, b0 + block, max(per_block - 2, 0)))
    return np.array(sorted(rows))
