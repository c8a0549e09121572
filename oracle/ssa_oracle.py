"""Plain fp64 CPU oracle of SSA dual-stream attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference legs of ``bench.py`` may import this module.  It
shares no code with the CUDA path (``block_sparse_full_b200``) and never
imports it; its inputs come from ``block_sparse_full_b200.inputs`` (random
draws only) or from hand-written fixtures.

Everything here is the plain definition of what one SSA attention layer
computes, written out in float64 with numpy (a matmul is the only library
primitive used).  No blocking, online softmax or fusion: each quantity is
formed directly from its definition so it can be checked by eye against the
method as the SSA pages describe it.

Sources (page title, section):

* "Sintesi Tecnica: SSA (Sparse Sparse Attention)", gist.science (Italian
  technical summary), section 2 "Metodologia": the sparse-attention stream is
  block-sparse attention, the full-attention stream is ordinary (causal)
  softmax attention that gives gradient to every token; the counterpart
  output of the opposite mode is computed only for alignment; the alignment
  loss has two parts, L_sparsity (full output imitates sparse output, which
  lowers the discarded attention mass delta(t)) and L_commit (sparse output
  stays near the full output); the total objective adds alpha * L_align.
* Same page, section 1 "Definizione del Problema": sparse training normalises
  only over the selected subset; the approximation error grows linearly with
  the discarded attention mass (weight on tokens the sparse rule did not
  select).
* Same page, section 4 "Risultati Sperimentali", "Efficienza": at inference SSA
  runs the same operations as MoBA (mean-pooled key blocks scored against the
  query block, top-k blocks, the current block always attended).
* "Résumé technique : SSA", gist.science (French), sections 1, 2 and 4: the
  same statements.

Readings where the pages are silent (each restated in the design doc):

* pooling: mean of the keys of a block and mean of the queries of a query
  block; score s_ij = Qbar_i . Kbar_j (equal to the mean over the block's
  queries of q_t . Kbar_j, by linearity);
* query-block size equals key-block size; selection is per query block;
* the diagonal (current) block is always selected and counts inside the
  budget k; block 0 is forced only with ``force_sink`` (also inside k);
* candidates rank by (score descending, block index ascending); with fewer
  causal blocks than k all are taken; indices are emitted ascending, padded
  with -1;
* L_sparsity = L_commit = mean over all B*H*T*d elements of
  (h_full - h_sparse)^2; L_sparsity sends gradient only to h_full, L_commit
  only to h_sparse (stop-gradient on the opposite stream); the weights
  w_s, w_c absorb alpha;
* no gradient flows through block selection or through delta(t).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "f64", "pool_blocks", "block_scores", "select_blocks", "block_selection_matrix",
    "attn_fwd_dual", "attn_fwd_sparse", "diagnostics", "decode_pool", "decode_step",
    "align_loss", "alignment_upstream", "attn_bwd",
]


def f64(x) -> np.ndarray:
    """Exact float64 copy of a torch tensor or array (bf16/f32 -> f64 is exact)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------
# Block selection (sparse-attention stream's block-sparse rule)
# --------------------------------------------------------------------------

def pool_blocks(x: np.ndarray, block: int) -> np.ndarray:
    """Mean of each run of ``block`` consecutive rows of x [T, d] -> [T/block, d].

    MoBA-identical block representation ("Efficienza", section 4).  With
    bf16/f32 inputs the block sums are exact in float64, and division by a
    power-of-two block is exact too, so this value is the same whatever the
    summation order.
    """
    T, d = x.shape
    n = T // block
    return x[: n * block].reshape(n, block, d).sum(axis=1) / float(block)


def block_scores(q: np.ndarray, k: np.ndarray, block: int) -> np.ndarray:
    """s[i, j] = Qbar_i . Kbar_j for one (batch, head); q, k are [T, d]."""
    return pool_blocks(q, block) @ pool_blocks(k, block).T


def select_blocks(q, k, block: int, topk: int, force_sink: bool = False):
    """Per query block i: the set S_i of key blocks the sparse stream attends.

    S_i = forced_i  u  top-(k - |forced_i|) of the remaining causal blocks
    j < i by (score descending, j ascending), all of them if fewer remain.
    forced_i = {i}, plus {0} when ``force_sink`` and i > 0.

    q, k: [B, H, T, d].  Returns
      idx    int32  [B, H, n, topk]  ascending block indices, -1 padded
      cnt    int32  [B, H, n]        |S_i|
      mask   uint32 [B, H, n, ceil(n/32)]  bit j of S_i
      margin float64 [B, H, n]  score gap between the last selected and the
             first rejected candidate (inf when nothing was rejected); a GPU
             selection may only differ from this one where it is ~0.
    """
    q, k = f64(q), f64(k)
    B, H, T, _ = q.shape
    n = T // block
    words = (n + 31) // 32
    idx = np.full((B, H, n, topk), -1, dtype=np.int32)
    cnt = np.zeros((B, H, n), dtype=np.int32)
    mask = np.zeros((B, H, n, words), dtype=np.uint32)
    margin = np.full((B, H, n), np.inf)
    for b in range(B):
        for h in range(H):
            s = block_scores(q[b, h], k[b, h], block)
            for i in range(n):
                forced = [i] + ([0] if (force_sink and i > 0) else [])
                cand = [j for j in range(i) if j not in forced]
                r = max(topk - len(forced), 0)
                ranked = sorted(cand, key=lambda j: (-s[i, j], j))
                chosen = sorted(set(forced) | set(ranked[:r]))
                if 0 < r < len(ranked):
                    margin[b, h, i] = s[i, ranked[r - 1]] - s[i, ranked[r]]
                cnt[b, h, i] = len(chosen)
                idx[b, h, i, : len(chosen)] = chosen
                for j in chosen:
                    mask[b, h, i, j // 32] |= np.uint32(1 << (j % 32))
    return idx, cnt, mask, margin


def block_selection_matrix(idx: np.ndarray, cnt: np.ndarray) -> np.ndarray:
    """Boolean [.., n, n] with [i, j] = (j in S_i), from idx/cnt [.., n, k]."""
    lead = idx.shape[:-2]
    n = idx.shape[-2]
    sel = np.zeros(lead + (n, n), dtype=bool)
    for pos in np.ndindex(*lead, n):
        c = int(cnt[pos])
        sel[pos][idx[pos][:c]] = True
    return sel


# --------------------------------------------------------------------------
# Forward: both streams, discarded mass, log-sum-exps
# --------------------------------------------------------------------------

def _fwd_rows(q, k, v, blocksel, block, sm_scale, rows):
    """Both attention outputs for query rows ``rows`` of one (batch, head)."""
    tmax = int(rows.max()) + 1
    s = np.arange(tmax)
    x = sm_scale * (q[rows] @ k[:tmax].T)                 # logits  [r, tmax]
    causal = s[None, :] <= rows[:, None]
    in_sel = blocksel[rows // block][:, s // block]        # s's block in S_i
    sel = causal & in_sel
    uns = causal & ~in_sel
    m = np.where(causal, x, -np.inf).max(axis=1)
    p = np.where(causal, np.exp(x - m[:, None]), 0.0)     # unnormalised weights
    p_sel = np.where(sel, p, 0.0)
    p_uns = np.where(uns, p, 0.0)
    l_sel = p_sel.sum(axis=1)
    l_uns = p_uns.sum(axis=1)
    o_sel = p_sel @ v[:tmax]
    o_uns = p_uns @ v[:tmax]
    l_all = l_sel + l_uns
    h_full = (o_sel + o_uns) / l_all[:, None]             # softmax over all s <= t
    h_sparse = o_sel / l_sel[:, None]                     # softmax over selected s only
    with np.errstate(invalid="ignore", divide="ignore"):
        h_unsel = np.where(l_uns[:, None] > 0, o_uns / l_uns[:, None], 0.0)
    return {
        "h_full": h_full,
        "h_sparse": h_sparse,
        "h_unsel": h_unsel,
        "delta": l_uns / l_all,
        "lse_full": m + np.log(l_all),
        "lse_sparse": m + np.log(l_sel),
        "sqdiff": ((h_full - h_sparse) ** 2).sum(axis=1),
    }


def attn_fwd_dual(q, k, v, idx, cnt, block: int, sm_scale: float, rows=None,
                  max_elems: int = 1 << 23):
    """Full-attention and block-sparse outputs of the same Q, K, V.

    For query t (block i) and every key s <= t, with x = sm_scale * q_t . k_s:
      h_full(t)   = sum_s softmax_{s<=t}(x) v_s
      h_sparse(t) = sum_{s: block(s) in S_i} softmax over those s of x, times v_s
      delta(t)    = full-softmax mass on keys whose block is not in S_i
      lse_full    = log sum_{s<=t} e^x,  lse_sparse = log sum_{selected} e^x
      sqdiff(t)   = sum_c (h_full - h_sparse)_c^2
    (sections 1 and 2 of the technical summaries; the sparse stream
    normalises over the selected subset only).

    q, k, v: [B, H, T, d]; idx, cnt from ``select_blocks``.  ``rows``
    optionally restricts the query rows (same rows for every batch/head);
    outputs then have T' = len(rows) rows.  Extra output ``h_unsel`` is the
    softmax average of v over the unselected keys (0 where there are none).
    """
    q, k, v = f64(q), f64(k), f64(v)
    B, H, T, d = q.shape
    rows = np.arange(T) if rows is None else np.asarray(sorted(rows), dtype=np.int64)
    R = len(rows)
    blocksel = block_selection_matrix(idx, cnt)
    dv = v.shape[-1]  # value width (equal to d in the layer; tests may widen it)
    out = {name: np.zeros((B, H, R, dv)) for name in ("h_full", "h_sparse", "h_unsel")}
    for name in ("delta", "lse_full", "lse_sparse", "sqdiff"):
        out[name] = np.zeros((B, H, R))
    for b in range(B):
        for h in range(H):
            step = max(1, max_elems // T)
            for start in range(0, R, step):
                chunk = rows[start:start + step]
                res = _fwd_rows(q[b, h], k[b, h], v[b, h], blocksel[b, h], block,
                                sm_scale, chunk)
                for name, val in res.items():
                    out[name][b, h, start:start + step] = val
    return out


def attn_fwd_sparse(q, k, v, idx, cnt, block: int, sm_scale: float, rows=None):
    """The sparse stream alone, as run at inference (section 4 of the technical
    summaries, "Efficienza": the same operations as MoBA).

    For query t in block i, the keys are gathered explicitly: every key s <= t
    of every block listed in idx[i, :cnt[i]] (S_i, which always holds block i
    itself); with x = sm_scale * q_t . k_s over those keys only,
      h(t) = sum_s softmax(x)_s v_s,   lse(t) = log sum_s e^x.
    Same quantities as h_sparse / lse_sparse of ``attn_fwd_dual``, formed from
    the index lists instead of a mask over all causal keys.

    q, k, v: [B, H, T, d]; idx, cnt: [B, H, n, k] / [B, H, n].  ``rows``
    optionally restricts the query rows.  Returns dict(h, lse).
    """
    q, k, v = f64(q), f64(k), f64(v)
    idx, cnt = np.asarray(idx), np.asarray(cnt)
    B, H, T, d = q.shape
    rows = np.arange(T) if rows is None else np.asarray(sorted(rows), dtype=np.int64)
    h_out = np.zeros((B, H, len(rows), v.shape[-1]))
    lse_out = np.zeros((B, H, len(rows)))
    for b in range(B):
        for h in range(H):
            for i in np.unique(rows // block):
                sel = np.flatnonzero(rows // block == i)
                ts = rows[sel]
                blocks = np.sort(idx[b, h, i, :cnt[b, h, i]])
                keys = np.concatenate([np.arange(j * block, (j + 1) * block) for j in blocks])
                x = sm_scale * (q[b, h, ts] @ k[b, h, keys].T)       # [rows of block i, keys]
                x = np.where(keys[None, :] <= ts[:, None], x, -np.inf)
                m = x.max(axis=1, keepdims=True)
                e = np.exp(x - m)
                l = e.sum(axis=1)
                h_out[b, h, sel] = (e @ v[b, h, keys]) / l[:, None]
                lse_out[b, h, sel] = m[:, 0] + np.log(l)
    return {"h": h_out, "lse": lse_out}


def diagnostics(q, k, lse_full, delta, block: int, sm_scale: float):
    """Attention diagnostics the pages discuss: the approximation error grows
    with the discarded mass delta (section 1 of the technical summaries);
    extrapolation suffers when too much attention goes to sink areas, here
    the first block (the paper's abstract, on the chatpaper.ai summary and the
    arXiv 2511.20102 listing); how sparse learned attention is (same abstract):

      sink(t)        = full-softmax mass on the keys of block 0:
                       sum_{s <= t, s < block} exp(sm_scale q_t . k_s - lse_full(t))
      mean_delta[h]  = mean over t of delta(t)
      mean_sink[h]   = mean over t of sink(t)

    q, k: [B, H, T, d]; lse_full, delta: [B, H, T] (the forward's outputs).
    Returns dict(sink [B,H,T], mean_delta [B,H], mean_sink [B,H]).
    """
    q, k = f64(q), f64(k)
    lse, dl = f64(lse_full), f64(delta)
    B, H, T, d = q.shape
    sink = np.zeros((B, H, T))
    keys = np.arange(min(block, T))
    for b in range(B):
        for h in range(H):
            x = sm_scale * (q[b, h] @ k[b, h, keys].T)                    # [T, block]
            w = np.where(keys[None, :] <= np.arange(T)[:, None], np.exp(x - lse[b, h][:, None]), 0.0)
            sink[b, h] = w.sum(axis=1)
    return {"sink": sink, "mean_delta": dl.mean(axis=2), "mean_sink": sink.mean(axis=2)}


def decode_pool(k_cache, block: int, n_done: int) -> np.ndarray:
    """Pooled keys of the first ``n_done`` completed blocks of a key cache
    [B, H, Tcap, d]: Kbar_j = mean of the keys of block j (float64)."""
    k = f64(k_cache)
    B, H, _, d = k.shape
    return k[:, :, : n_done * block].reshape(B, H, n_done, block, d).mean(axis=3)


def decode_step(q_t, k_cache, v_cache, t: int, block: int, topk: int, sm_scale: float,
                force_sink: bool = False):
    """One generation step of the sparse stream over a key/value cache (the
    summaries' section 4: at inference SSA runs MoBA's operations; decoding
    at long context).  The pages do not describe decoding itself; the reading
    used here is MoBA's inference rule: the current query token q_t (not a
    query-block mean, whose later members do not exist yet) is scored against
    the pooled keys of the completed blocks, Kbar_j for j < i = t // block;
    the current block i is always attended (its keys 0..t) and counts inside
    the budget k; block 0 is forced only with ``force_sink``; the remaining
    places go to the best-scoring completed blocks (score descending, index
    ascending).  Then softmax attention over every key of the selected
    blocks that is <= t.

    q_t: [B, H, d]; k_cache, v_cache: [B, H, Tcap, d] holding keys 0..t.
    Returns dict(h [B,H,d], lse [B,H], idx [B,H,k] ascending, -1 padded).
    """
    q, K, V = f64(q_t), f64(k_cache), f64(v_cache)
    B, H, d = q.shape
    i = t // block
    kbar = decode_pool(k_cache, block, i)                          # [B, H, i, d]
    h_out = np.zeros((B, H, V.shape[-1]))
    lse_out = np.zeros((B, H))
    idx_out = np.full((B, H, topk), -1, dtype=np.int64)
    for b in range(B):
        for h in range(H):
            forced = [i] + ([0] if force_sink and i > 0 else [])
            cand = [j for j in range(i) if j not in forced]
            score = {j: float(q[b, h] @ kbar[b, h, j]) for j in cand}
            ranked = sorted(cand, key=lambda j: (-score[j], j))
            sel = sorted(forced + ranked[: max(topk - len(forced), 0)])
            idx_out[b, h, : len(sel)] = sel
            keys = np.concatenate([np.arange(j * block, min((j + 1) * block, t + 1)) for j in sel])
            x = sm_scale * (K[b, h, keys] @ q[b, h])
            m = x.max()
            e = np.exp(x - m)
            h_out[b, h] = (e @ V[b, h, keys]) / e.sum()
            lse_out[b, h] = m + np.log(e.sum())
    return {"h": h_out, "lse": lse_out, "idx": idx_out}


def align_loss(h_full, h_sparse, w_sparsity: float = 1.0, w_commit: float = 1.0):
    """(w_s * L_sparsity, w_c * L_commit), both the mean squared difference of
    the two outputs over all elements (section 2, "Allineamento
    Bidirezionale"; the distance is the reading stated in the module header)."""
    hf, hs = f64(h_full), f64(h_sparse)
    L = float(np.mean((hf - hs) ** 2))
    return w_sparsity * L, w_commit * L


def alignment_upstream(h_full, h_sparse, dh_full, dh_sparse, w_s, w_c, n_total):
    """Gradients reaching each output: the caller's upstream plus the
    alignment terms with stop-gradient on the opposite stream.

    d(w_s L_sparsity)/d h_full   = w_s * 2/N * (h_full - h_sparse)   (h_sparse held fixed)
    d(w_c L_commit)/d h_sparse   = w_c * 2/N * (h_sparse - h_full)   (h_full held fixed)
    """
    hf, hs = f64(h_full), f64(h_sparse)
    g_full = f64(dh_full) + w_s * (2.0 / n_total) * (hf - hs)
    g_sparse = f64(dh_sparse) + w_c * (2.0 / n_total) * (hs - hf)
    return g_full, g_sparse


# --------------------------------------------------------------------------
# Backward through both streams
# --------------------------------------------------------------------------

def _bwd_head(q, k, v, blocksel, block, sm_scale, g_full, g_sparse, max_elems=1 << 23,
              rows=None):
    """dq, dk, dv of  sum(g_full * h_full) + sum(g_sparse * h_sparse)  for one
    (batch, head), selection held fixed.  Written with the explicit softmax
    Jacobian: for P = softmax(x) over a key set and upstream dP = g v^T,
    dx = P * (dP - rowsum(P * dP)).  Query rows are independent, so they are
    taken a slice at a time; dk and dv sum the slices' contributions."""
    T = q.shape[0]
    s = np.arange(T)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)

    def softmax_over(x, allowed):
        xm = np.where(allowed, x, -np.inf)
        m = xm.max(axis=1, keepdims=True)
        e = np.where(allowed, np.exp(xm - m), 0.0)
        return e / e.sum(axis=1, keepdims=True)

    rows = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    step = max(1, max_elems // T)
    for c0 in range(0, len(rows), step):
        t = rows[c0:c0 + step]
        x = sm_scale * (q[t] @ k.T)
        causal = s[None, :] <= t[:, None]
        sel = causal & blocksel[t // block][:, s // block]
        p_full = softmax_over(x, causal)    # full-attention stream: every s <= t
        p_sparse = softmax_over(x, sel)     # sparse stream: selected blocks only
        dv += p_full.T @ g_full[t] + p_sparse.T @ g_sparse[t]
        dp_full = g_full[t] @ v.T
        dp_sparse = g_sparse[t] @ v.T
        dx = p_full * (dp_full - (p_full * dp_full).sum(axis=1, keepdims=True))
        dx += p_sparse * (dp_sparse - (p_sparse * dp_sparse).sum(axis=1, keepdims=True))
        dq[t] = sm_scale * dx @ k
        dk += sm_scale * dx.T @ q[t]
    return dq, dk, dv


def attn_bwd(q, k, v, idx, cnt, block: int, sm_scale: float, dh_full, dh_sparse,
             w_sparsity: float = 0.0, w_commit: float = 0.0, n_total=None, rows=None):
    """Gradients of  <dh_full, h_full> + <dh_sparse, h_sparse>
    + w_s * L_sparsity + w_c * L_commit  with respect to q, k, v.

    The full stream carries gradient to every causal key (section 2, "Full
    Attention Stream"); the sparse stream only to selected keys; the
    alignment terms follow ``alignment_upstream``.  ``n_total`` is the
    element count N of the whole layer output (defaults to q.size) so that a
    caller may pass a slice of heads.  ``rows`` optionally keeps only the
    terms of those query rows (dq of other rows is then 0 and dk, dv hold
    those rows' share); used to time a bounded slice.  Returns (dq, dk, dv)
    float64.
    """
    q, k, v = f64(q), f64(k), f64(v)
    B, H, T, d = q.shape
    n_total = q.size if n_total is None else n_total
    sel_rows = None if rows is None else np.asarray(sorted(rows), dtype=np.int64)
    fw = attn_fwd_dual(q, k, v, idx, cnt, block, sm_scale, rows=sel_rows)
    dhf, dhs = f64(dh_full), f64(dh_sparse)
    if sel_rows is not None:
        dhf, dhs = dhf[:, :, sel_rows], dhs[:, :, sel_rows]
    g_rows = alignment_upstream(fw["h_full"], fw["h_sparse"], dhf, dhs, w_sparsity,
                                w_commit, n_total)
    if sel_rows is None:
        g_full, g_sparse = g_rows
    else:  # scatter the listed rows' upstream into full-length arrays
        g_full, g_sparse = np.zeros_like(q), np.zeros_like(q)
        g_full[:, :, sel_rows], g_sparse[:, :, sel_rows] = g_rows
    blocksel = block_selection_matrix(idx, cnt)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            dq[b, h], dk[b, h], dv[b, h] = _bwd_head(
                q[b, h], k[b, h], v[b, h], blocksel[b, h], block, sm_scale,
                g_full[b, h], g_sparse[b, h], rows=sel_rows)
    return dq, dk, dv
