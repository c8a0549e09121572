"""GPU parity of the decode step over a key/value cache (the sparse stream at
generation time, MoBA's inference rule) against the fp64 oracle."""
import numpy as np
import pytest
import torch

from block_sparse_full_b200 import ssa
from block_sparse_full_b200.inputs import WORKLOADS, Workload, make_inputs
from oracle import ssa_oracle as O

from gpu_parity_util import DEV, TOL, log, params
from test_gpu_parity import SINK, SMALL

pytestmark = pytest.mark.gpu


def _decode(w, ts, flags=0, heads=None, topk=None):
    inp = make_inputs(w)
    p = params(w, inp["q"].to(DEV), topk, flags)
    cache = ssa.DecodeCache(p, DEV, inp["k"].dtype)
    cache.k.copy_(inp["k"].to(DEV))
    cache.v.copy_(inp["v"].to(DEV))
    hs = slice(None) if heads is None else heads
    tol = TOL[w.dtype]
    k_eff = topk if topk is not None else w.topk
    for t in ts:
        q_t = inp["q"][:, :, t].contiguous()
        got = cache.step(t, q_t.to(DEV))
        torch.cuda.synchronize()
        ssa.device_status()
        ref = O.decode_step(q_t[:, hs], inp["k"][:, hs], inp["v"][:, hs], t, w.block, k_eff,
                            w.sm_scale, force_sink=bool(flags & SINK))
        np.testing.assert_array_equal(got["idx"][:, hs].cpu().numpy(), ref["idx"])
        h = got["h"][:, hs].float().cpu().numpy()
        e = float(np.abs(h - ref["h"]).max())
        scale = float(np.abs(ref["h"]).max())
        el = float(np.abs(got["lse"][:, hs].cpu().numpy() - ref["lse"]).max())
        assert e <= tol["h"] and e <= tol["h_rel"] * max(scale, 1.0 if w.dtype == "f32" else scale), (t, e)
        assert el <= tol["lse"], (t, el)
        log(f"decode/{w.name}/t{t}", h=e, lse=el)
    # the pooled keys are exact float64 block means
    n = cache.pooled
    want = O.decode_pool(inp["k"], w.block, n)
    np.testing.assert_array_equal(cache.kbar[:, :, :n].cpu().numpy(), want)


@pytest.mark.parametrize("name", ["bf16_T1216_b64", "bf16_T448_d64", "f32_T320_d128",
                                  "bf16_B2_T640_b128_sink"])
def test_decode_small(name):
    w = SMALL[name]
    T, b = w.T, w.block
    ts = sorted({0, b - 1, b, 2 * b + 5, T // 2, T - b, T - 1})
    _decode(w, ts)


def test_decode_force_sink_and_full_budget():
    w = SMALL["bf16_B2_T640_b128_sink"]
    _decode(w, [130, 383, 639], flags=SINK)
    _decode(w, [200, 639], topk=w.T // w.block)


def test_decode_T65536_sink_last_token():
    w = WORKLOADS["bf16_T65536_H8_sink"]
    _decode(w, [w.T - 1, w.T // 2 + 17], heads=[1, 6])


def test_decode_f32_d64_workload():
    w = WORKLOADS["f32_T1024_d64"]
    _decode(w, [0, 63, 64, 500, w.T - 1])


def test_decode_more_than_1024_completed_blocks():
    # 1100 blocks of 64: the selection bitmask spans 35 words, so the ascending
    # list is assembled over more than one warp-wide chunk of mask words
    w = Workload("bf16_T70400_d64_decode", B=1, H=1, T=64 * 1100, D=64, block=64, topk=12,
                 dtype="bf16", plant="hot", seed=41)
    _decode(w, [w.T - 1, 64 * 1030 + 3])


def test_decode_topk64_d128_many_heads():
    # the largest budget the decode step takes (64 places) at d = 128: its
    # shared memory passes the default 48 KB per CTA, and with 16 heads the
    # clusters of 4 CTAs take several selected blocks per half of a CTA
    w = Workload("bf16_H16_T16384_k64_decode", B=1, H=16, T=16384, D=128, block=64, topk=64,
                 dtype="bf16", plant="hot", seed=43)
    _decode(w, [w.T - 1, 64 * 70 + 9], heads=[0, 9])


def test_decode_few_heads_cluster_of_eight():
    # eight heads or fewer: clusters of 8 CTAs per head
    w = Workload("bf16_H4_T8192_decode", B=2, H=2, T=8192, D=128, block=128, topk=16,
                 dtype="bf16", plant="sink", seed=44)
    _decode(w, [w.T - 1, 4000])


def test_decode_f32_block128_several_passes():
    # float32 blocks of 128 keys at d = 128 take 128 KB of keys and values each:
    # one fits in a CTA's shared memory, so the two selected blocks of each CTA
    # of a 4-CTA cluster (12 heads) stream in one pass after the other
    w = Workload("f32_H12_T2048_b128_decode", B=1, H=12, T=2048, D=128, block=128, topk=8,
                 dtype="f32", plant="hot", seed=45)
    _decode(w, [w.T - 1, 128 * 9 + 100, 128 * 3 + 1], heads=[0, 5, 11])


def test_decode_step_is_repeatable():
    # the same step twice gives the same bits (fixed reduction orders)
    w = SMALL["bf16_T1216_b64"]
    inp = make_inputs(w)
    p = params(w, inp["q"].to(DEV))
    cache = ssa.DecodeCache(p, DEV, inp["k"].dtype)
    cache.k.copy_(inp["k"].to(DEV))
    cache.v.copy_(inp["v"].to(DEV))
    t = w.T - 1
    q_t = inp["q"][:, :, t].contiguous().to(DEV)
    a = cache.step(t, q_t)
    a = {n: x.clone() for n, x in a.items()}
    b = cache.step(t, q_t)
    torch.cuda.synchronize()
    ssa.device_status()
    for n in a:
        assert torch.equal(a[n], b[n]), n


def test_decode_sixteen_heads_clusters_of_eight_small_ctas():
    # 16 heads at top-k 16: clusters of 8 CTAs of 256 threads
    w = WORKLOADS["bf16_T8192_H16_hot"]
    _decode(w, [w.T - 1, 3000], heads=[0, 7, 15])


def test_decode_many_heads_small_ctas():
    # 128 heads: clusters of 4 CTAs of 256 threads
    w = WORKLOADS["bf16_B4_H32_T4096_train"]
    _decode(w, [w.T - 1, 1500], heads=[0, 31])
