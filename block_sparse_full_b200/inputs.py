"""Seeded synthetic inputs for the SSA dual-stream attention layer.

This module only draws random numbers and lays them out; it holds none of the
attention, selection or loss arithmetic.  Both the CUDA path (tests, bench) and
the CPU oracle (tests) take their inputs from here, so the two sides always see
identical bits.

Workloads stand in for the long-context layers the SSA pages train and run
(a Llama-3.2-1B-scale model, 8k pre-training, 32k continual training and 128k
inference; "SSA: Sparse Sparse Attention", gist.science technical summary,
section 4).  Their activations are not available, so each workload draws
Q, K, V from N(0, 1) (scaled by 1/sqrt(d) for the bf16 workloads) and, where
stated, plants structure that block selection must find:

* ``plant="hot"``: per head, ``n_hot`` key blocks (chosen without replacement)
  and a unit direction u_h; every key of a hot block and every query gets
  ``a * u_h`` added with ``a = sqrt(boost) * d**0.25``.  The expected extra
  logit ``sm_scale * a**2`` is then ``boost`` (default 8) for every
  (query, hot-key) pair.
* ``plant="sink"``: the same with block 0 as the single hot block, a heavy
  "sink" block that should win the block scoring for every query block.

Values are generated in float32, the planted offset added in float32, and the
result rounded to the workload dtype (round-to-nearest-even for bf16).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional

import torch

FORCE_SINK = 1  # same bit as SSA_FLAG_FORCE_SINK in include/ssa.h


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    D: int
    block: int
    topk: int
    dtype: str  # "f32" | "bf16"
    plant: Optional[str] = None  # None | "hot" | "sink"
    n_hot: int = 4
    boost: float = 8.0
    scale_data: bool = True  # divide the N(0,1) draws by sqrt(D)
    grads: bool = False  # also draw upstream gradients dh_full, dh_sparse
    flags: int = 0
    seed: int = 0
    sweep: tuple = field(default_factory=tuple)  # extra top-k budgets

    @property
    def n_blocks(self) -> int:
        return self.T // self.block

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads named by the benchmark spec, by what they are.
WORKLOADS = {
    "f32_T1024_d64": Workload("f32_T1024_d64", B=1, H=1, T=1024, D=64, block=64,
                              topk=4, dtype="f32", scale_data=False, seed=0),
    "bf16_T8192_H16_hot": Workload("bf16_T8192_H16_hot", B=1, H=16, T=8192, D=128,
                                   block=64, topk=16, dtype="bf16", plant="hot",
                                   seed=2),
    "bf16_T16384_H16_sweep": Workload("bf16_T16384_H16_sweep", B=1, H=16, T=16384,
                                      D=128, block=64, topk=16, dtype="bf16",
                                      plant="hot", seed=3,
                                      sweep=(4, 8, 16, 32, 64, 256)),
    "bf16_T65536_H8_sink": Workload("bf16_T65536_H8_sink", B=1, H=8, T=65536, D=128,
                                    block=128, topk=16, dtype="bf16", plant="sink",
                                    seed=4),
    "bf16_B4_H32_T4096_train": Workload("bf16_B4_H32_T4096_train", B=4, H=32,
                                        T=4096, D=128, block=64, topk=8,
                                        dtype="bf16", grads=True, seed=5),
}


def _gen(seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    # distinct, reproducible stream per (seed, tensor)
    g.manual_seed((seed * 1_000_003 + stream * 7919) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _normal(shape, seed: int, stream: int) -> torch.Tensor:
    return torch.randn(shape, generator=_gen(seed, stream), dtype=torch.float32)


def make_inputs(w: Workload) -> dict:
    """Draw q, k, v (and dh_full, dh_sparse if ``w.grads``) as CPU tensors
    of shape [B, H, T, D] in the workload dtype, contiguous."""
    shape = (w.B, w.H, w.T, w.D)
    q = _normal(shape, w.seed, 0)
    k = _normal(shape, w.seed, 1)
    v = _normal(shape, w.seed, 2)
    if w.scale_data:
        s = 1.0 / math.sqrt(w.D)
        q.mul_(s), k.mul_(s), v.mul_(s)
    hot = None
    if w.plant is not None:
        a = math.sqrt(w.boost) * w.D ** 0.25
        u = _normal((w.B, w.H, w.D), w.seed, 3)
        u = u / u.norm(dim=-1, keepdim=True)
        n = w.n_blocks
        hot = torch.zeros((w.B, w.H, n), dtype=torch.bool)
        g = _gen(w.seed, 4)
        for b in range(w.B):
            for h in range(w.H):
                if w.plant == "sink":
                    hot[b, h, 0] = True
                else:
                    blocks = torch.randperm(n, generator=g)[: min(w.n_hot, n)]
                    hot[b, h, blocks] = True
        tok_hot = hot.repeat_interleave(w.block, dim=2)  # [B,H,T]
        off = (a * u)[:, :, None, :]  # [B,H,1,D]
        q.add_(off)
        k.add_(off * tok_hot[..., None].to(torch.float32))
    out = {
        "q": q.to(w.torch_dtype).contiguous(),
        "k": k.to(w.torch_dtype).contiguous(),
        "v": v.to(w.torch_dtype).contiguous(),
        "hot_blocks": hot,
    }
    if w.grads:
        out["dh_full"] = _normal(shape, w.seed, 5).to(w.torch_dtype).contiguous()
        out["dh_sparse"] = _normal(shape, w.seed, 6).to(w.torch_dtype).contiguous()
    return out


def upstream_grads(w: Workload, seed_offset: int = 0) -> dict:
    """N(0,1) upstream gradients for the two outputs, in the workload dtype."""
    shape = (w.B, w.H, w.T, w.D)
    return {
        "dh_full": _normal(shape, w.seed + seed_offset, 5).to(w.torch_dtype).contiguous(),
        "dh_sparse": _normal(shape, w.seed + seed_offset, 6).to(w.torch_dtype).contiguous(),
    }
