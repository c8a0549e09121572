"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each test checks the oracle against one of: a hand-derived closed form
(tests/golden), a library routine that the method reduces to in a special
case (torch's scaled-dot-product attention, logsumexp, mse_loss, autograd),
brute force on tiny inputs, a mathematical identity or bound the SSA pages
state (error linear in the discarded attention mass), or central finite
differences.  CPU only.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import ssa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def rand(*shape):
    return rng.standard_normal(shape)


def sdpa(q, k, v, mask, scale):
    """torch fp64 attention with a boolean mask (True = attend)."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    return F.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=t(mask),
                                          scale=scale).numpy()


def token_masks(idx, cnt, block, T):
    """Causal, selected and unselected token masks [B,H,T,T] built from the
    selection sets (test-side, for the library calls)."""
    sel = O.block_selection_matrix(idx, cnt)
    t = np.arange(T)
    causal = t[None, :] <= t[:, None]
    insel = sel[..., t[:, None] // block, t[None, :] // block]
    return causal, causal & insel, causal & ~insel


# ---------------------------------------------------------------- worked example

def test_worked_example_closed_form():
    g = json.load(open(os.path.join(GOLDEN, "worked_example_T4.json")))
    w, v, e = np.array(g["w"]), np.array(g["v"]), g["expected"]
    q = np.ones((1, 1, 4, 1))
    k = np.log(w).reshape(1, 1, 4, 1)
    vv = v.reshape(1, 1, 4, 1)
    idx, cnt, _, _ = O.select_blocks(q, k, 1, g["topk"])
    assert idx[0, 0].tolist() == e["idx"]
    assert cnt[0, 0].tolist() == e["cnt"]
    out = O.attn_fwd_dual(q, k, vv, idx, cnt, 1, 1.0)
    for name in ("h_full", "h_sparse"):
        np.testing.assert_allclose(out[name][0, 0, :, 0], e[name], rtol=0, atol=1e-14)
    for name in ("delta", "lse_full", "lse_sparse"):
        np.testing.assert_allclose(out[name][0, 0], e[name], rtol=0, atol=1e-14)
    ls, lc = O.align_loss(out["h_full"], out["h_sparse"])
    assert abs(ls - e["loss"]) < 1e-15 and ls == lc


def test_worked_example_sink_flag():
    g = json.load(open(os.path.join(GOLDEN, "worked_example_T4.json")))["sink_variant"]
    q = np.ones((1, 1, 4, 1))
    k = np.log(np.array(g["w"])).reshape(1, 1, 4, 1)
    idx, _, _, _ = O.select_blocks(q, k, 1, 2)
    assert idx[0, 0].tolist() == g["idx_default"]
    idx, _, _, _ = O.select_blocks(q, k, 1, 2, force_sink=True)
    assert idx[0, 0].tolist() == g["idx_force_sink"]


# ---------------------------------------------------------------- selection

def test_pooling_closed_forms():
    # arithmetic ramp: the mean of a block of consecutive integers is the
    # midpoint of its first and last value
    T, block = 48, 8
    x = np.arange(T, dtype=np.float64)[:, None] * np.array([[1.0, -2.0, 0.5]])
    pooled = O.pool_blocks(x, block)
    mids = np.array([(i * block + i * block + block - 1) / 2 for i in range(T // block)])
    np.testing.assert_array_equal(pooled, mids[:, None] * np.array([[1.0, -2.0, 0.5]]))
    # constant blocks pool to their constant (float32 values: block sums are
    # exact in float64, as for every bf16/f32 input the layer takes)
    c = rand(T // block, 5).astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(O.pool_blocks(np.repeat(c, block, axis=0), block), c)


def test_scores_are_mean_of_per_query_scores():
    # two readings of "score a key block for a query block" coincide
    q, k = rand(32, 6), rand(32, 6)
    s = O.block_scores(q, k, 4)
    kbar = k.reshape(8, 4, 6).mean(axis=1)
    per_query = (q @ kbar.T).reshape(8, 4, 8).mean(axis=1)
    np.testing.assert_allclose(s, per_query, rtol=1e-13, atol=1e-13)


# sink forcing needs a budget of at least 2 (the sink and the current block)
@pytest.mark.parametrize("topk,force_sink", [(1, False), (2, False), (3, False), (5, False),
                                             (2, True), (3, True), (5, True)])
def test_topk_against_exhaustive_search(topk, force_sink):
    B, H, block, n, d = 1, 2, 2, 9, 4
    q, k = rand(B, H, n * block, d), rand(B, H, n * block, d)
    idx, cnt, mask, _ = O.select_blocks(q, k, block, topk, force_sink)
    for h in range(H):
        s = O.block_scores(q[0, h], k[0, h], block)
        for i in range(n):
            forced = {i} | ({0} if force_sink and i > 0 else set())
            cand = [j for j in range(i) if j not in forced]
            r = min(max(topk - len(forced), 0), len(cand))
            best = max(itertools.combinations(cand, r),
                       key=lambda c: sum(s[i, j] for j in c))
            want = sorted(forced | set(best))
            assert idx[0, h, i, :cnt[0, h, i]].tolist() == want
            assert all(x == -1 for x in idx[0, h, i, cnt[0, h, i]:])
            bits = [j for j in range(n) if (int(mask[0, h, i, j // 32]) >> (j % 32)) & 1]
            assert bits == want


def test_selection_margin_is_zero_exactly_where_the_best_set_is_not_unique():
    """The margin the GPU tests use to excuse near-ties: with integer-valued
    data every block score is exact, so an exhaustive search over the r-subsets
    of the candidates tells whether the best set is unique; the margin must be
    0 exactly where it is not, positive where it is, and inf where nothing
    was rejected."""
    r = np.random.default_rng(23)
    B, H, block, n, d = 1, 3, 2, 10, 3
    q = r.integers(-2, 3, size=(B, H, n * block, d)).astype(np.float64)
    k = r.integers(-1, 2, size=(B, H, n * block, d)).astype(np.float64)
    seen_tie = seen_unique = False
    for topk in (2, 3, 4):
        _, _, _, margin = O.select_blocks(q, k, block, topk)
        for h in range(H):
            s = O.block_scores(q[0, h], k[0, h], block)
            for i in range(n):
                cand = list(range(i))
                rr = topk - 1
                if rr == 0 or rr >= len(cand):
                    assert margin[0, h, i] == np.inf
                    continue
                sums = [sum(s[i, j] for j in c) for c in itertools.combinations(cand, rr)]
                best = max(sums)
                unique = sum(1 for x in sums if x == best) == 1
                if unique:
                    assert margin[0, h, i] > 0
                    seen_unique = True
                else:
                    assert margin[0, h, i] == 0
                    seen_tie = True
    assert seen_tie and seen_unique


def test_topk_ties_go_to_lower_block_index():
    # block = token, q = 1: scores are the key values; blocks 1, 2, 4 tie
    k = np.array([0.0, 5.0, 5.0, 1.0, 5.0, 0.0, 0.0]).reshape(1, 1, 7, 1)
    q = np.ones_like(k)
    idx, cnt, _, margin = O.select_blocks(q, k, 1, 3)
    # t=6: forced {6}, two slots among {0..5}: ties at 5.0 for 1, 2, 4 -> {1, 2}
    assert idx[0, 0, 6].tolist() == [1, 2, 6]
    assert margin[0, 0, 6] == 0.0
    # t=5: two slots among {0..4} -> {1, 2}
    assert idx[0, 0, 5].tolist() == [1, 2, 5]


def test_mask_words_beyond_32_blocks():
    n, block = 70, 1
    q = np.ones((1, 1, n, 1))
    k = np.arange(n, dtype=np.float64).reshape(1, 1, n, 1)  # later blocks score higher
    idx, cnt, mask, _ = O.select_blocks(q, k, block, 4)
    assert mask.shape[-1] == 3
    # i = 69: forced 69, top 3 of 0..68 by score -> 66, 67, 68
    assert idx[0, 0, 69].tolist() == [66, 67, 68, 69]
    assert int(mask[0, 0, 69, 2]) == (1 << 2) | (1 << 3) | (1 << 4) | (1 << 5)
    assert int(mask[0, 0, 69, 0]) == 0 and int(mask[0, 0, 69, 1]) == 0


# ---------------------------------------------------------------- forward

def _case(B=1, H=2, T=96, d=8, block=8, topk=3, seed=0):
    r = np.random.default_rng(seed)
    q, k, v = (r.standard_normal((B, H, T, d)) for _ in range(3))
    idx, cnt, _, _ = O.select_blocks(q, k, block, topk)
    return q, k, v, idx, cnt


def test_full_budget_reduces_to_causal_attention():
    B, H, T, d, block = 1, 2, 96, 8, 8
    q, k, v, idx, cnt = _case(B, H, T, d, block, topk=T // block)
    out = O.attn_fwd_dual(q, k, v, idx, cnt, block, 0.37)
    ref = sdpa(q, k, v, np.tril(np.ones((T, T), dtype=bool)), 0.37)
    np.testing.assert_allclose(out["h_full"], ref, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(out["h_sparse"], out["h_full"])
    assert np.all(out["delta"] == 0.0)
    assert O.align_loss(out["h_full"], out["h_sparse"]) == (0.0, 0.0)


def test_streams_match_library_attention_with_masks():
    B, H, T, d, block = 1, 3, 128, 8, 8
    q, k, v, idx, cnt = _case(B, H, T, d, block, topk=4, seed=3)
    out = O.attn_fwd_dual(q, k, v, idx, cnt, block, 0.5)
    causal, sel, uns = token_masks(idx, cnt, block, T)
    np.testing.assert_allclose(out["h_full"], sdpa(q, k, v, causal[None, None], 0.5),
                               rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["h_sparse"], sdpa(q, k, v, sel, 0.5), rtol=0, atol=1e-12)
    # the identity h_full = (1 - delta) h_sparse + delta h_unsel, with h_unsel
    # from the library on the complementary mask, pins delta
    has_uns = uns.any(axis=-1)
    h_uns = sdpa(q, k, v, uns | ~has_uns[..., None], 0.5)
    dlt = out["delta"][..., None]
    mix = (1 - dlt) * out["h_sparse"] + dlt * np.where(has_uns[..., None], h_uns, 0.0)
    np.testing.assert_allclose(out["h_full"], mix, rtol=0, atol=1e-12)
    assert np.all(out["delta"][~has_uns] == 0.0)
    assert np.all(out["delta"][has_uns] > 0.0)


def test_sqdiff_rows_from_library_attention():
    """sqdiff(t) = sum_c (h_full - h_sparse)_c^2, with both outputs from library
    attention under the causal and the selection masks; its mean over the
    B*H*T*d elements is the alignment loss."""
    B, H, T, d, block = 1, 2, 96, 8, 8
    q, k, v, idx, cnt = _case(B, H, T, d, block, topk=3, seed=17)
    out = O.attn_fwd_dual(q, k, v, idx, cnt, block, 0.6)
    causal, sel, _ = token_masks(idx, cnt, block, T)
    hf = sdpa(q, k, v, causal[None, None], 0.6)
    hs = sdpa(q, k, v, sel, 0.6)
    np.testing.assert_allclose(out["sqdiff"], ((hf - hs) ** 2).sum(axis=-1), rtol=1e-10, atol=1e-14)
    assert np.all(out["sqdiff"][..., :block] == 0.0)  # the first query block sees only itself
    L, _ = O.align_loss(out["h_full"], out["h_sparse"])
    assert L == pytest.approx(out["sqdiff"].sum() / (B * H * T * d), rel=1e-12)


def test_lse_against_library_logsumexp():
    B, H, T, d, block = 1, 2, 64, 8, 8
    q, k, v, idx, cnt = _case(B, H, T, d, block, topk=2, seed=5)
    out = O.attn_fwd_dual(q, k, v, idx, cnt, block, 0.7)
    causal, sel, _ = token_masks(idx, cnt, block, T)
    x = torch.from_numpy(0.7 * np.einsum("bhtd,bhsd->bhts", q, k))
    lf = torch.logsumexp(x.masked_fill(~torch.from_numpy(causal), -math.inf), -1).numpy()
    ls = torch.logsumexp(x.masked_fill(~torch.from_numpy(sel), -math.inf), -1).numpy()
    np.testing.assert_allclose(out["lse_full"], lf, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["lse_sparse"], ls, rtol=0, atol=1e-12)
    # sparse-stream mass: exp(lse_sparse - lse_full) = 1 - delta
    np.testing.assert_allclose(np.exp(out["lse_sparse"] - out["lse_full"]),
                               1 - out["delta"], rtol=0, atol=1e-12)


def test_error_linear_in_discarded_mass():
    # |h_full - h_sparse|_c <= delta(t) * (max_s v_sc - min_s v_sc) over s <= t
    B, H, T, d, block = 1, 4, 256, 16, 16
    q, k, v, idx, cnt = _case(B, H, T, d, block, topk=3, seed=7)
    q *= 3.0  # sharper attention, wider spread of delta
    out = O.attn_fwd_dual(q, k, v, idx, cnt, block, 0.25)
    vmax = np.maximum.accumulate(v, axis=2)
    vmin = np.minimum.accumulate(v, axis=2)
    err = np.abs(out["h_full"] - out["h_sparse"])
    bound = out["delta"][..., None] * (vmax - vmin)
    assert np.all(err <= bound + 1e-12)
    assert np.all(out["delta"] >= 0) and np.all(out["delta"] <= 1)


def test_delta_non_increasing_in_budget():
    B, H, T, d, block = 1, 3, 256, 8, 16
    q, k, v, _, _ = _case(B, H, T, d, block, topk=1, seed=11)
    prev = None
    for topk in (1, 2, 4, 8, 16):
        idx, cnt, _, _ = O.select_blocks(q, k, block, topk)
        out = O.attn_fwd_dual(q, k, v, idx, cnt, block, 0.35)
        n_blocks_seen = np.arange(T) // block + 1
        assert np.all(out["delta"][..., n_blocks_seen <= topk] == 0.0)
        if prev is not None:
            assert np.all(out["delta"] <= prev + 1e-15)
        prev = out["delta"]
    assert np.all(prev == 0.0)  # 16 blocks = everything


def test_softmax_rows_sum_to_one():
    # weights implied by the outputs: with v = identity rows (d = T), h_full
    # and h_sparse are the softmax rows themselves
    T, block = 32, 4
    r = np.random.default_rng(2)
    q, k = r.standard_normal((1, 1, T, 5)), r.standard_normal((1, 1, T, 5))
    v = np.eye(T)[None, None]
    idx, cnt, _, _ = O.select_blocks(q, k, block, 2)
    out = O.attn_fwd_dual(q, k, v, idx, cnt, block, 1.0)
    np.testing.assert_allclose(out["h_full"].sum(-1), 1.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["h_sparse"].sum(-1), 1.0, rtol=0, atol=1e-12)
    assert np.all(np.triu(out["h_full"][0, 0], 1) == 0)  # causal
    # sparse weights vanish exactly on unselected keys; their full mass is delta
    _, sel, uns = token_masks(idx, cnt, block, T)
    assert np.all(out["h_sparse"][~sel] == 0)
    np.testing.assert_allclose((out["h_full"] * uns).sum(-1), out["delta"], atol=1e-12)


def test_row_sampling_matches_all_rows():
    q, k, v, idx, cnt = _case(1, 2, 96, 8, 8, topk=3, seed=9)
    full = O.attn_fwd_dual(q, k, v, idx, cnt, 8, 0.5)
    rows = [0, 7, 8, 50, 95]
    part = O.attn_fwd_dual(q, k, v, idx, cnt, 8, 0.5, rows=rows)
    for name in full:
        np.testing.assert_allclose(part[name], full[name][:, :, rows], rtol=0, atol=1e-13)


# ---------------------------------------------------------------- losses

def test_align_loss_is_library_mse():
    a, b = rand(2, 3, 40, 8), rand(2, 3, 40, 8)
    ls, lc = O.align_loss(a, b, 0.3, 2.0)
    mse = F.mse_loss(torch.from_numpy(a), torch.from_numpy(b)).item()
    assert abs(ls - 0.3 * mse) < 1e-15 and abs(lc - 2.0 * mse) < 1e-14


# ---------------------------------------------------------------- backward

def _objective(q, k, v, idx, cnt, block, scale, Rf, Rs, ws, wc, c_s, c_f, N):
    out = O.attn_fwd_dual(q, k, v, idx, cnt, block, scale)
    hf, hs = out["h_full"], out["h_sparse"]
    return (np.sum(Rf * hf) + np.sum(Rs * hs)
            + ws / N * np.sum((hf - c_s) ** 2) + wc / N * np.sum((hs - c_f) ** 2))


@pytest.mark.parametrize("ws,wc", [(0.0, 0.0), (40.0, 25.0)])
def test_bwd_central_finite_differences(ws, wc):
    B, H, T, d, block, topk, scale = 1, 2, 24, 3, 4, 2, 0.8
    r = np.random.default_rng(21)
    q, k, v = (r.standard_normal((B, H, T, d)) for _ in range(3))
    Rf, Rs = r.standard_normal((B, H, T, d)), r.standard_normal((B, H, T, d))
    idx, cnt, _, _ = O.select_blocks(q, k, block, topk)
    N = q.size
    base = O.attn_fwd_dual(q, k, v, idx, cnt, block, scale)
    c_s, c_f = base["h_sparse"], base["h_full"]  # stop-gradient targets, frozen
    dq, dk, dv = O.attn_bwd(q, k, v, idx, cnt, block, scale, Rf, Rs, ws, wc)
    eps = 1e-6
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        args = {"q": q, "k": k, "v": v}
        for pos in [(0, 0, 0, 0), (0, 1, 5, 2), (0, 0, 13, 1), (0, 1, 23, 0), (0, 0, 17, 2)]:
            plus = {a: x.copy() for a, x in args.items()}
            minus = {a: x.copy() for a, x in args.items()}
            plus[name][pos] += eps
            minus[name][pos] -= eps
            fp = _objective(plus["q"], plus["k"], plus["v"], idx, cnt, block, scale,
                            Rf, Rs, ws, wc, c_s, c_f, N)
            fm = _objective(minus["q"], minus["k"], minus["v"], idx, cnt, block, scale,
                            Rf, Rs, ws, wc, c_s, c_f, N)
            fd = (fp - fm) / (2 * eps)
            assert abs(fd - grad[pos]) < 1e-7 * max(1.0, abs(fd)), (name, pos, fd, grad[pos])


def test_bwd_matches_library_autograd():
    B, H, T, d, block, topk, scale = 1, 2, 96, 8, 8, 3, 0.45
    r = np.random.default_rng(33)
    q, k, v = (r.standard_normal((B, H, T, d)) for _ in range(3))
    Rf, Rs = r.standard_normal((B, H, T, d)), r.standard_normal((B, H, T, d))
    idx, cnt, _, _ = O.select_blocks(q, k, block, topk)
    ws, wc = 300.0, 700.0
    dq, dk, dv = O.attn_bwd(q, k, v, idx, cnt, block, scale, Rf, Rs, ws, wc)
    # library: autograd through torch attention for each stream, upstream =
    # caller gradient + alignment gradient (stop-gradient on the other stream)
    causal, sel, _ = token_masks(idx, cnt, block, T)
    tq, tk, tv = (torch.from_numpy(x).requires_grad_() for x in (q, k, v))
    hf = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(causal), scale=scale)
    hs = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(sel), scale=scale)
    loss = (hf * torch.from_numpy(Rf)).sum() + (hs * torch.from_numpy(Rs)).sum() \
        + ws * F.mse_loss(hf, hs.detach()) + wc * F.mse_loss(hs, hf.detach())
    loss.backward()
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=0, atol=1e-11)


def test_bwd_full_budget_is_textbook_attention_backward():
    B, H, T, d, block, scale = 1, 1, 64, 8, 8, 0.6
    r = np.random.default_rng(44)
    q, k, v = (r.standard_normal((B, H, T, d)) for _ in range(3))
    Rf, Rs = r.standard_normal((B, H, T, d)), r.standard_normal((B, H, T, d))
    idx, cnt, _, _ = O.select_blocks(q, k, block, T // block)
    dq, dk, dv = O.attn_bwd(q, k, v, idx, cnt, block, scale, Rf, Rs)
    tq, tk, tv = (torch.from_numpy(x).requires_grad_() for x in (q, k, v))
    h = F.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=scale)
    (h * torch.from_numpy(Rf + Rs)).sum().backward()
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=0, atol=1e-11)


# ---------------------------------------------------------------- sparse-only forward (inference)

def test_sparse_only_matches_library_attention_on_selected_keys():
    # the gathered-key sparse stream equals library attention restricted to
    # the selected causal keys, for several budgets including the diagonal only
    B, H, T, d, block = 1, 2, 128, 8, 16
    for topk, seed in ((1, 7), (3, 8), (T // block, 9)):
        q, k, v, idx, cnt = _case(B, H, T, d, block, topk=topk, seed=seed)
        out = O.attn_fwd_sparse(q, k, v, idx, cnt, block, 0.45)
        _, sel, _ = token_masks(idx, cnt, block, T)
        np.testing.assert_allclose(out["h"], sdpa(q, k, v, sel, 0.45), rtol=0, atol=1e-12)
        x = torch.from_numpy(0.45 * np.einsum("bhtd,bhsd->bhts", q, k))
        ls = torch.logsumexp(x.masked_fill(~torch.from_numpy(sel), -math.inf), -1).numpy()
        np.testing.assert_allclose(out["lse"], ls, rtol=0, atol=1e-12)


def test_sparse_only_diagonal_budget_is_blockwise_causal_attention():
    # top-1 keeps only the current block: per-block causal attention (library)
    B, H, T, d, block = 1, 1, 64, 4, 16
    q, k, v, idx, cnt = _case(B, H, T, d, block, topk=1, seed=11)
    assert np.all(cnt == 1) and np.all(idx[..., 0] == np.arange(T // block))
    out = O.attn_fwd_sparse(q, k, v, idx, cnt, block, 0.9)
    for i in range(T // block):
        sl = slice(i * block, (i + 1) * block)
        ref = sdpa(q[..., sl, :], k[..., sl, :], v[..., sl, :],
                   np.tril(np.ones((block, block), dtype=bool)), 0.9)
        np.testing.assert_allclose(out["h"][..., sl, :], ref, rtol=0, atol=1e-12)


def test_sparse_only_equals_the_dual_forwards_sparse_stream():
    B, H, T, d, block = 2, 2, 96, 8, 8
    q, k, v, idx, cnt = _case(B, H, T, d, block, topk=3, seed=13)
    dual = O.attn_fwd_dual(q, k, v, idx, cnt, block, 0.6)
    rows = [0, 5, 8, 40, 95]
    sp = O.attn_fwd_sparse(q, k, v, idx, cnt, block, 0.6, rows=rows)
    np.testing.assert_allclose(sp["h"], dual["h_sparse"][:, :, rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(sp["lse"], dual["lse_sparse"][:, :, rows], rtol=0, atol=1e-12)


def test_sparse_only_brute_force_tiny():
    # T = 4, block 2, one head: keys listed by hand
    q = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0], [0.5, -1.0]])[None, None]
    k = np.array([[0.2, 0.1], [0.0, 0.3], [1.0, -1.0], [0.4, 0.4]])[None, None]
    v = np.array([[1.0, 2.0], [3.0, 4.0], [5.0, 6.0], [7.0, 8.0]])[None, None]
    idx = np.array([[[[0, -1], [1, -1]]]])  # block 1 selects only itself
    cnt = np.array([[[1, 1]]])
    out = O.attn_fwd_sparse(q, k, v, idx, cnt, 2, 1.0)
    # row 3 sees keys 2 and 3 only: weights e^{q3.k2}, e^{q3.k3}
    x2, x3 = 0.5 * 1.0 + (-1.0) * (-1.0), 0.5 * 0.4 + (-1.0) * 0.4
    w2, w3 = math.exp(x2), math.exp(x3)
    np.testing.assert_allclose(out["h"][0, 0, 3], (w2 * v[0, 0, 2] + w3 * v[0, 0, 3]) / (w2 + w3),
                               rtol=0, atol=1e-14)
    np.testing.assert_allclose(out["lse"][0, 0, 3], math.log(w2 + w3), rtol=0, atol=1e-14)
    # row 0 sees only key 0
    np.testing.assert_allclose(out["h"][0, 0, 0], v[0, 0, 0], rtol=0, atol=1e-15)


# ---------------------------------------------------------------- diagnostics

def test_sink_mass_is_library_softmax_on_block_zero():
    B, H, T, d, block = 1, 2, 96, 8, 16
    q, k, v, idx, cnt = _case(B, H, T, d, block, topk=2, seed=17)
    fwd = O.attn_fwd_dual(q, k, v, idx, cnt, block, 0.8)
    dg = O.diagnostics(q, k, fwd["lse_full"], fwd["delta"], block, 0.8)
    x = torch.from_numpy(0.8 * np.einsum("bhtd,bhsd->bhts", q, k))
    causal = torch.from_numpy(np.tril(np.ones((T, T), dtype=bool)))
    p = torch.softmax(x.masked_fill(~causal, -math.inf), dim=-1).numpy()
    np.testing.assert_allclose(dg["sink"], p[..., :block].sum(-1), rtol=0, atol=1e-12)
    # rows inside block 0 put all their mass there
    np.testing.assert_allclose(dg["sink"][..., :block], 1.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dg["mean_sink"], dg["sink"].mean(-1), rtol=0, atol=0)
    np.testing.assert_allclose(dg["mean_delta"], fwd["delta"].mean(-1), rtol=0, atol=0)


def test_sink_mass_rises_with_a_planted_sink():
    # a large logit boost on block 0 moves almost all mass there
    B, H, T, d, block = 1, 1, 64, 8, 16
    q, k, v, idx, cnt = _case(B, H, T, d, block, topk=2, seed=19)
    base = O.attn_fwd_dual(q, k, v, idx, cnt, block, 1.0)
    s0 = O.diagnostics(q, k, base["lse_full"], base["delta"], block, 1.0)["sink"]
    u = np.ones(d) / math.sqrt(d)
    q2, k2 = q + 3.0 * u, k.copy()
    k2[..., :block, :] += 3.0 * u
    fwd = O.attn_fwd_dual(q2, k2, v, idx, cnt, block, 1.0)
    s1 = O.diagnostics(q2, k2, fwd["lse_full"], fwd["delta"], block, 1.0)["sink"]
    assert s1[..., block:].mean() > 0.9 > s0[..., block:].mean()


# ---------------------------------------------------------------- decode over a KV cache

def test_decode_pool_is_block_mean():
    r = np.random.default_rng(31)
    k = r.standard_normal((1, 2, 40, 3))
    kb = O.decode_pool(k, 8, 4)
    np.testing.assert_allclose(kb[0, 1, 2], k[0, 1, 16:24].mean(axis=0), rtol=0, atol=1e-15)
    assert kb.shape == (1, 2, 4, 3)


def test_decode_full_budget_is_causal_attention_row():
    # every block selected: the step is the last row of causal attention (library)
    r = np.random.default_rng(33)
    B, H, Tcap, d, block = 1, 2, 80, 8, 16
    K, V = r.standard_normal((B, H, Tcap, d)), r.standard_normal((B, H, Tcap, d))
    for t in (0, 15, 16, 47, 79):
        q = r.standard_normal((B, H, d))
        out = O.decode_step(q, K, V, t, block, topk=Tcap // block, sm_scale=0.3)
        ref = sdpa(q[:, :, None], K[:, :, : t + 1], V[:, :, : t + 1],
                   np.ones((1, t + 1), dtype=bool), 0.3)[:, :, 0]
        np.testing.assert_allclose(out["h"], ref, rtol=0, atol=1e-12)
        x = torch.from_numpy(0.3 * np.einsum("bhd,bhsd->bhs", q, K[:, :, : t + 1]))
        np.testing.assert_allclose(out["lse"], torch.logsumexp(x, -1).numpy(), rtol=0, atol=1e-12)
        assert (out["idx"][..., : t // block + 1] == np.arange(t // block + 1)).all()


def test_decode_selection_brute_force():
    # the chosen set maximises the summed score among sets holding the current
    # block (with distinct scores the top-(k-1) completed blocks are that set)
    r = np.random.default_rng(35)
    B, H, Tcap, d, block, topk = 1, 3, 96, 4, 8, 4
    K, V = r.standard_normal((B, H, Tcap, d)), r.standard_normal((B, H, Tcap, d))
    t = 90
    q = r.standard_normal((B, H, d))
    out = O.decode_step(q, K, V, t, block, topk, 1.0)
    i = t // block
    kbar = K[:, :, : i * block].reshape(B, H, i, block, d).mean(axis=3)
    for h in range(H):
        s = kbar[0, h] @ q[0, h]
        best = max(itertools.combinations(range(i), topk - 1), key=lambda c: sum(s[list(c)]))
        assert out["idx"][0, h].tolist() == sorted(list(best) + [i])
        # attention restricted to those blocks' keys (library)
        keys = np.concatenate([np.arange(j * block, min((j + 1) * block, t + 1))
                               for j in out["idx"][0, h]])
        ref = sdpa(q[0, h][None, None, None], K[0, h][keys][None, None], V[0, h][keys][None, None],
                   np.ones((1, len(keys)), dtype=bool), 1.0)[0, 0, 0]
        np.testing.assert_allclose(out["h"][0, h], ref, rtol=0, atol=1e-12)


def test_decode_ties_sink_and_first_block():
    B, H, Tcap, d, block = 1, 1, 48, 2, 8
    K = np.zeros((B, H, Tcap, d))
    V = np.arange(Tcap * d, dtype=float).reshape(1, 1, Tcap, d)
    q = np.array([[[1.0, 0.0]]])
    # all completed blocks score 0: ties go to the lowest indices
    out = O.decode_step(q, K, V, 44, block, topk=3, sm_scale=1.0)
    assert out["idx"][0, 0].tolist() == [0, 1, 5]
    # block 0 forced by the sink flag even when another block scores higher
    K2 = K.copy()
    K2[0, 0, 24:32, 0] = 5.0
    out = O.decode_step(q, K2, V, 44, block, topk=2, sm_scale=1.0, force_sink=True)
    assert out["idx"][0, 0].tolist() == [0, 5]
    out = O.decode_step(q, K2, V, 44, block, topk=2, sm_scale=1.0)
    assert out["idx"][0, 0].tolist() == [3, 5]
    # t inside block 0: only the current block's causal keys
    out = O.decode_step(q, K, V, 3, block, topk=4, sm_scale=1.0)
    assert out["idx"][0, 0].tolist() == [0, -1, -1, -1]
    np.testing.assert_allclose(out["h"][0, 0], V[0, 0, :4].mean(axis=0), rtol=0, atol=1e-14)
