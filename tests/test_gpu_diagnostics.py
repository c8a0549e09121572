"""GPU parity of the attention diagnostics (sink mass on block 0, per-head
means of delta and of the sink mass) against the fp64 oracle, fed the same
forward outputs."""
import numpy as np
import pytest
import torch

from block_sparse_full_b200 import ssa
from block_sparse_full_b200.inputs import WORKLOADS, make_inputs
from oracle import ssa_oracle as O

from gpu_parity_util import log, oracle_mask_to_dev, oracle_select, params, to_dev
from test_gpu_parity import SIMT, SMALL

pytestmark = pytest.mark.gpu


def _check(case, w, flags=0, heads=None):
    inp = make_inputs(w)
    o_sel = oracle_select(w, inp)
    d = to_dev(inp)
    p = params(w, d["q"], flags=flags)
    fwd = ssa.attn_fwd_dual(p, d["q"], d["k"], d["v"], oracle_mask_to_dev(o_sel[2]))
    dg = ssa.diagnostics(p, d["q"], d["k"], fwd)
    torch.cuda.synchronize()
    ssa.device_status()
    hs = slice(None) if heads is None else heads
    # the oracle is fed the GPU's own lse_full / delta: this checks the diagnostics alone
    ref = O.diagnostics(inp["q"][:, hs], inp["k"][:, hs], fwd["lse_full"][:, hs].cpu().numpy(),
                        fwd["delta"][:, hs].cpu().numpy(), w.block, w.sm_scale)
    sink = dg["sink"][:, hs].cpu().numpy()
    stats = dg["head_stats"][:, hs].cpu().numpy()
    es = float(np.abs(sink - ref["sink"]).max())
    ed = float(np.abs(stats[..., 0] - ref["mean_delta"]).max())
    ek = float(np.abs(stats[..., 1] - ref["mean_sink"]).max())
    tol = 1e-5 if w.dtype == "f32" else 1e-3   # bf16 logits sharpen exp errors slightly
    assert es <= tol and ed <= 1e-6 and ek <= tol, (case, es, ed, ek)
    log(case, sink=es, mean_delta=ed, mean_sink=ek)
    return sink, stats


@pytest.mark.parametrize("name", ["bf16_T1216_b64", "bf16_B2_T640_b128_sink", "f32_T320_d128",
                                  "bf16_T448_d64"])
def test_diagnostics_small(name):
    _check("diag/" + name, SMALL[name])


def test_diagnostics_sink_workload_sees_the_planted_sink():
    w = WORKLOADS["bf16_T65536_H8_sink"]
    sink, stats = _check("diag/" + w.name, w, heads=[0, 3])
    # every head of the sink workload puts most of its mass on block 0
    assert (stats[..., 1] > 0.5).all(), stats


def test_diagnostics_repeatable():
    w = SMALL["bf16_T1216_b64"]
    inp = make_inputs(w)
    d = to_dev(inp)
    p = params(w, d["q"])
    o_sel = oracle_select(w, inp)
    fwd = ssa.attn_fwd_dual(p, d["q"], d["k"], d["v"], oracle_mask_to_dev(o_sel[2]))
    a = ssa.diagnostics(p, d["q"], d["k"], fwd)
    b = ssa.diagnostics(p, d["q"], d["k"], fwd)
    torch.cuda.synchronize()
    assert torch.equal(a["sink"], b["sink"]) and torch.equal(a["head_stats"], b["head_stats"])


def _check_fused(case, w, heads=None):
    """ssa_attn_fwd_dual_diag: the forward outputs equal those of
    ssa_attn_fwd_dual bit for bit, and the sink mass the forward kernel
    accumulates matches the oracle's, fed the same lse_full and delta."""
    inp = make_inputs(w)
    o_sel = oracle_select(w, inp)
    d = to_dev(inp)
    p = params(w, d["q"])
    mask = oracle_mask_to_dev(o_sel[2])
    plain = ssa.attn_fwd_dual(p, d["q"], d["k"], d["v"], mask)
    fused = ssa.attn_fwd_dual_diag(p, d["q"], d["k"], d["v"], mask)
    torch.cuda.synchronize()
    ssa.device_status()
    for name in plain:
        assert torch.equal(plain[name], fused[name]), name
    hs = slice(None) if heads is None else heads
    ref = O.diagnostics(inp["q"][:, hs], inp["k"][:, hs], fused["lse_full"][:, hs].cpu().numpy(),
                        fused["delta"][:, hs].cpu().numpy(), w.block, w.sm_scale)
    sink = fused["sink"][:, hs].cpu().numpy()
    stats = fused["head_stats"][:, hs].cpu().numpy()
    es = float(np.abs(sink - ref["sink"]).max())
    ed = float(np.abs(stats[..., 0] - ref["mean_delta"]).max())
    ek = float(np.abs(stats[..., 1] - ref["mean_sink"]).max())
    tol = 1e-5 if w.dtype == "f32" else 1e-3
    assert es <= tol and ed <= 1e-6 and ek <= tol, (case, es, ed, ek)
    log(case, sink=es, mean_delta=ed, mean_sink=ek)
    return stats


@pytest.mark.parametrize("name", ["bf16_T1216_b64", "bf16_B2_T640_b128_sink", "f32_T320_d128",
                                  "bf16_T448_d64", "bf16_T64_single_block"])
def test_fused_diagnostics_small(name):
    _check_fused("diag_fused/" + name, SMALL[name])


def test_fused_diagnostics_sink_workload():
    w = WORKLOADS["bf16_T65536_H8_sink"]
    stats = _check_fused("diag_fused/" + w.name, w, heads=[0, 3])
    assert (stats[..., 1] > 0.5).all(), stats
