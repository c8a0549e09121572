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


def compare_fwd(case, dtype, gpu, ref, rows=None, ref_abs=None):
    """Compare GPU forward outputs (all rows) with oracle outputs (``rows``).
    With ``ref_abs`` (the oracle forward on |v|, same rows) the per-row squared
    difference is also held to ``sqdiff_budget``."""
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
    if ref_abs is not None:
        g = gpu["sqdiff"][sl].cpu().numpy().astype(np.float64)
        r = ref["sqdiff"]
        dev = np.abs(g - r)
        budget = sqdiff_budget(dtype, ref, ref_abs)
        assert np.isfinite(g).all(), "sqdiff"
        worst = np.unravel_index(np.argmax(dev - budget), dev.shape)
        assert (dev <= budget).all(), (f"{case} sqdiff: |gpu - oracle| {dev[worst]:.3e} > budget "
                                       f"{budget[worst]:.3e} (oracle {r[worst]:.3e}) at {worst}")
        # and the losses' relative tolerance, row by row (float32 resolution as the floor)
        rel = tol["loss_rel"] * r + 1e-12 * max(float(r.max()), 1e-30)
        assert (dev <= rel).all(), f"{case} sqdiff: relative error above {tol['loss_rel']}"
        errs["sqdiff_budget_ratio"] = float((dev / budget).max())
        errs["sqdiff_rel_max"] = float((dev / np.maximum(r, 1e-30)).max(initial=0.0,
                                                                        where=r > 0))
    log(case, **errs)
    return errs


def sqdiff_budget(dtype, ref, ref_abs):
    """Per-row bound on |r_gpu(t) - r_oracle(t)|, r(t) = sum_c (h_full - h_sparse)_c^2,
    derived from the kernels' arithmetic (both kernels keep O_sel, O_uns and
    l_sel, l_uns and form h_full = (O_sel + O_uns) / (l_sel + l_uns),
    h_sparse = O_sel / l_sel, r from the float32 values before rounding).

    The tensor-core path rounds each softmax weight p to bf16 (relative error
    <= u = 2^-8) before the P.V products but sums l_sel, l_uns from the
    unrounded weights.  With d = h_full - h_sparse, errors e_sel in O_sel and
    e_uns in O_uns move d_c by  e_sel,c (1/l - 1/l_sel) + e_uns,c / l,  and
    since 1/l - 1/l_sel = -delta / l_sel and |e_x,c| <= u sum_x p |v_c|,
    |dd_c| <= u delta (A_sel,c + A_uns,c), A the softmax-weighted means of |v_c|
    over the selected / unselected keys (the oracle run on |v|).  An
    approximate exponential (relative error <= 7.5e-5 < 2^-12) perturbs a
    weight in O and l alike, which moves d_c by at most
    2^-12 (delta (A + |h_full| + |h_sparse|) + 2 |d_c|).  The two separate
    float32 reciprocals and products add 2^-22 (|h_full| + |h_sparse|).  With
    E_c the sum of these terms, |r_gpu - r| <= sum_c (2 |d_c| E_c + E_c^2).
    float32 inputs (no weight rounding, float32 sums over at most 2^10 keys
    per row in the tests) take u = 2^-14 for both terms."""
    d = np.abs(ref["h_full"] - ref["h_sparse"])
    A = ref_abs["h_sparse"] + ref_abs["h_unsel"]
    Hm = np.abs(ref["h_full"]) + np.abs(ref["h_sparse"])
    delta = ref["delta"][..., None]
    u, eta = (2.0 ** -8, 2.0 ** -12) if dtype == "bf16" else (2.0 ** -14, 2.0 ** -14)
    E = delta * (u * A + eta * (A + Hm)) + 2 * eta * d + 2.0 ** -22 * Hm
    return (2 * d * E + E * E).sum(-1) + 1e-6 * ref["sqdiff"] + 1e-30


def oracle_fwd(q, k, v, idx, cnt, block, scale, rows=None, with_abs=True, threads=None):
    """The oracle forward for every (batch, head) of q, k, v, one (b, h) per
    task on a thread pool (numpy releases the GIL in its array loops), and,
    with ``with_abs``, the same forward on |v| (the weighted means of |v| that
    ``sqdiff_budget`` takes).  Returns (ref, ref_abs)."""
    from concurrent.futures import ThreadPoolExecutor

    qn, kn, vn = (O.f64(x) for x in (q, k, v))
    B, H = qn.shape[:2]
    jobs = [(b, h) for b in range(B) for h in range(H)]
    vs = [vn] + ([np.abs(vn)] if with_abs else [])

    def one(args):
        which, (b, h) = args
        sl = (slice(b, b + 1), slice(h, h + 1))
        return O.attn_fwd_dual(qn[sl], kn[sl], vs[which][sl], idx[sl], cnt[sl], block, scale,
                               rows=rows)

    tasks = [(wi, j) for wi in range(len(vs)) for j in jobs]
    nthr = threads or min(len(tasks), os.cpu_count() or 1, 16)
    with ThreadPoolExecutor(max_workers=nthr) as ex:
        res = list(ex.map(one, tasks))
    outs = []
    for wi in range(len(vs)):
        part = res[wi * len(jobs):(wi + 1) * len(jobs)]
        merged = {}
        for name in part[0]:
            arr = np.zeros((B, H) + part[0][name].shape[2:])
            for (b, h), r in zip(jobs, part):
                arr[b, h] = r[name][0, 0]
            merged[name] = arr
        outs.append(merged)
    return outs[0], (outs[1] if with_abs else None)


def oracle_loss_rows(q, k, v, idx, cnt, block, scale, dtype, threads=None):
    """Per (batch, head) and on every row: the oracle's alignment loss term
    (``O.align_loss`` of that head's outputs, a mean over its T x d
    elements), its per-row squared difference and the ``sqdiff_budget`` of
    each row.  Heads run on a thread pool and only row vectors are kept, so
    that whole workloads fit in host memory.  Returns (loss, sqdiff, budget):
    the mean over heads of the per-head losses (heads have equal sizes, so it
    is the loss over all B*H*T*d elements) and two [B, H, T] arrays."""
    from concurrent.futures import ThreadPoolExecutor

    qn, kn, vn = (O.f64(x) for x in (q, k, v))
    B, H, T = qn.shape[:3]
    jobs = [(b, h) for b in range(B) for h in range(H)]

    def one(bh):
        b, h = bh
        sl = (slice(b, b + 1), slice(h, h + 1))
        ref = O.attn_fwd_dual(qn[sl], kn[sl], vn[sl], idx[sl], cnt[sl], block, scale)
        ref_abs = O.attn_fwd_dual(qn[sl], kn[sl], np.abs(vn[sl]), idx[sl], cnt[sl], block, scale)
        ls, _ = O.align_loss(ref["h_full"], ref["h_sparse"])
        return ls, ref["sqdiff"][0, 0], sqdiff_budget(dtype, ref, ref_abs)[0, 0]

    nthr = threads or min(len(jobs), os.cpu_count() or 1, 16)
    with ThreadPoolExecutor(max_workers=nthr) as ex:
        res = list(ex.map(one, jobs))
    sq = np.zeros((B, H, T))
    bud = np.zeros((B, H, T))
    for (b, h), (_, r, bb) in zip(jobs, res):
        sq[b, h], bud[b, h] = r, bb
    return float(np.mean([x[0] for x in res])), sq, bud


def compare_loss(case, p, gpu_sqdiff, ref_loss, ref_sq, budget, n_total, w_s=2.0, w_c=3.0):
    """GPU per-row squared differences (every row) against the oracle's within
    ``budget``, and the GPU loss kernel against the oracle's loss: within the
    summed row budgets and within relative 2e-2."""
    g = gpu_sqdiff.cpu().numpy().astype(np.float64)
    dev = np.abs(g - ref_sq)
    worst = np.unravel_index(np.argmax(dev - budget), dev.shape)
    assert (dev <= budget).all(), (f"{case} sqdiff: {dev[worst]:.3e} > budget {budget[worst]:.3e} "
                                   f"(oracle {ref_sq[worst]:.3e}) at {worst}")
    rel = TOL["bf16"]["loss_rel"] * ref_sq + 1e-12 * max(float(ref_sq.max()), 1e-30)
    assert (dev <= rel).all(), f"{case} sqdiff: relative error above {TOL['bf16']['loss_rel']}"
    loss = ssa.align_loss(p, gpu_sqdiff, w_s, w_c).cpu().numpy().astype(np.float64)
    allowed = min(budget.sum() / n_total, TOL["bf16"]["loss_rel"] * ref_loss)
    errs = {}
    for i, wgt in enumerate((w_s, w_c)):
        e = abs(loss[i] / wgt - ref_loss)
        errs[f"loss{i}_rel"] = e / ref_loss
        assert e <= allowed, f"{case} loss[{i}]: |{loss[i] / wgt:.6e} - {ref_loss:.6e}| > {allowed:.3e}"
    errs["sqdiff_budget_ratio"] = float((dev / budget).max())
    errs["loss_budget"] = budget.sum() / n_total / ref_loss
    log(case + "/loss", **errs)
    return errs


def dq_rounding_budget(q, k, v, idx, cnt, block, scale, dh_full, dh_sparse, w_s, w_c, n_total,
                       rows=None):
    """Elementwise bound on the dq deviation that rounding the forward outputs
    to bf16 alone causes.  The backward takes D_f = G_f . h_full and
    D_s = G_s . h_sparse from the stored (bf16) outputs; a perturbation dD
    of D enters dq_t as -sigma * dD(t) * sum_s P(t,s) k_s, and that
    softmax-weighted mean key is the attention output with v := k.  All
    values come from the oracle; the bf16 rounding is torch's on the host.
    ``rows`` restricts it to those query rows (each row's bound is its own)."""
    ref = O.attn_fwd_dual(q, k, v, idx, cnt, block, scale, rows=rows)
    kbar = O.attn_fwd_dual(q, k, k, idx, cnt, block, scale, rows=rows)
    hf, hs = ref["h_full"], ref["h_sparse"]
    r16 = lambda a: torch.from_numpy(a).to(torch.bfloat16).double().numpy()
    if rows is not None:
        dh_full, dh_sparse = dh_full[:, :, rows], dh_sparse[:, :, rows]
    g_f, g_s = O.alignment_upstream(hf, hs, dh_full, dh_sparse, w_s, w_c, n_total)
    dDf = (np.abs(g_f) * np.abs(hf - r16(hf))).sum(-1, keepdims=True)
    dDs = (np.abs(g_s) * np.abs(hs - r16(hs))).sum(-1, keepdims=True)
    return scale * (dDf * np.abs(kbar["h_full"]) + dDs * np.abs(kbar["h_sparse"]))


def compare_grads(case, dtype, got, want, dq_budget=None, names=("dq", "dk", "dv")):
    """max |g - ref| <= tol * max|ref| per tensor; for dq, if given, also allow
    the (elementwise) deviation caused by the bf16 rounding of the forward
    outputs, ``dq_budget`` from ``dq_rounding_budget``."""
    tol = TOL[dtype]["grad_rel"]
    errs = {}
    for name, g, r in zip(names, got, want):
        g = g.float().cpu().numpy()
        diff = np.abs(g - r)
        scale = float(np.abs(r).max())
        errs[name + "_rel"] = float(diff.max()) / scale
        assert np.isfinite(g).all(), name
        allowed = tol * scale
        if name == "dq" and dq_budget is not None:
            allowed = allowed + 1.25 * dq_budget
            errs["dq_budget_ratio"] = float((diff / allowed).max())
            errs["dq_plain_ratio"] = float(diff.max() / (tol * scale))  # against 2e-2 x max alone
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
