"""Plain float64 CPU oracle for FlashPrefill-style block-sparse causal prefill attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this package: only
the tests, the smoke check and the benchmark's CPU-baseline/reference leg do. It
shares no code with the CUDA path.

The method, as the FlashPrefill pages describe it, is an approximation that
deliberately differs from dense attention. So this oracle takes the algorithm's
steps in the pages' order and computes each one exactly in float64:

1. Block pooling -- "FlashPrefill: Near-Zero-Cost Sparsity Discovery for
   Ultra-Fast Long-Context Prefilling" (zhichai.net summary), Method,
   "1. Instantaneous Pattern Discovery": each block of B tokens is represented
   by the mean of its queries / keys ("mean-proxy"), and pooled queries are
   scored against pooled keys, so discovery moves (L/B)^2 instead of L*L/B.
2. Dynamic threshold -- same page, Method, "2. Dynamic Threshold Pruning": a
   block is kept when its score reaches alpha times the row maximum (one
   max-reduction, no sort, no accumulation); attention-sink blocks and
   local-window blocks are always kept ("safety net").
3. Index compaction -- same page, Method, "3. Index Compaction -> Physical
   Jumps": the kept block indices of a row become one contiguous list, and the
   attention visits only those blocks.
4. Sparse attention with PackGQA, paged KV cache and continuous batching --
   "FlashPrefill V2: Block-Sparse Prefill Attention for Long-Context LLM
   Serving", abstract: all query heads of a KV group share the K/V tiles it
   visits (so there is one list per KV group), and K/V may live in a paged
   cache addressed per request.

Readings taken where the pages are silent, garbled or ambiguous:

* Score = softmax_scale * qbar_h,i . kbar_g,j (softmax_scale defaults to
  1/sqrt(d)). The "global reweighting" of the pooled map is read as a per-row
  softmax; a per-row positive renormalisation cancels in the ratio test below,
  so the mask only needs p = exp(s - rowmax).
* Threshold per query head and per row: keep_h(i, j) iff
  exp(s_h(i,j) - max_{j'<=i} s_h(i,j')) >= alpha, with ">=" (ties at the
  maximum are kept; alpha = 0 keeps everything). alpha must be finite, >= 0;
  alpha > 1 keeps only the forced blocks.
* PackGQA needs one list per KV group: the group mask is the union (OR) over
  the group's G query heads, each head thresholded against its own row max.
  Query head h belongs to KV group h // G.
* Causal at block level: candidates j <= i. Token-level causality is applied
  inside the attention.
* Sink / window are given in tokens and converted to blocks:
  Sb = ceil(sink/B) leading blocks; Wb = max(1, ceil(window/B)) blocks ending
  at and including the diagonal block (so the diagonal block is always kept
  and no row is empty).
* Pooling of a ragged last block averages its valid tokens only.
* Lists are strictly ascending block indices.
* Paged / varlen: full prefill (query length = KV length per request); block
  and page boundaries start at each request's first token; the page table
  maps request page p to a pool page.
* FP8: the oracle consumes the exactly dequantised values (e4m3 value times
  its per-head scale, in float64). The kernels' own choice of rounding P to
  e4m3 is not mimicked; the FP8 tolerance covers it.

The V2 "mean correction term" is not defined on the pages and is not part of
this oracle.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "num_blocks", "forced_blocks", "pool_blocks", "pooled_scores", "head_keep",
    "block_mask", "head_masks", "per_head_attention", "discover_row", "compact", "attention_rows", "block_sparse_attention",
    "flashprefill", "gather_pages", "flashprefill_paged", "flashprefill_chunk", "row_borderline",
]


def num_blocks(L: int, B: int) -> int:
    return (L + B - 1) // B


def forced_blocks(sink_tokens: int, window_tokens: int, B: int):
    """(Sb, Wb): sink tokens and window tokens expressed in whole blocks."""
    Sb = (sink_tokens + B - 1) // B
    Wb = max(1, (window_tokens + B - 1) // B)
    return Sb, Wb


def pool_blocks(X: np.ndarray, B: int) -> np.ndarray:
    """Block means (Method 1, mean-proxy). X [L, H, d] -> [N, H, d], over valid tokens."""
    L = X.shape[0]
    N = num_blocks(L, B)
    out = np.empty((N,) + X.shape[1:], dtype=np.float64)
    for i in range(N):
        lo, hi = i * B, min((i + 1) * B, L)
        out[i] = X[lo:hi].sum(axis=0, dtype=np.float64) / (hi - lo)
    return out


def pooled_scores(qbar: np.ndarray, kbar: np.ndarray, scale: float) -> np.ndarray:
    """Pooled block scores s[h, i, j] = scale * qbar[i, h] . kbar[j, h // G] (all i, j)."""
    N, Hq, _ = qbar.shape
    Hkv = kbar.shape[1]
    G = Hq // Hkv
    s = np.empty((Hq, N, kbar.shape[0]), dtype=np.float64)
    for h in range(Hq):
        s[h] = scale * (qbar[:, h, :] @ kbar[:, h // G, :].T)
    return s


def head_keep(s_h: np.ndarray, alpha: float) -> np.ndarray:
    """One query head's dynamic threshold (Method 2): keep[i, j] for j <= i iff
    exp(s[i, j] - max_{j'<=i} s[i, j']) >= alpha."""
    N = s_h.shape[0]
    keep = np.zeros((N, s_h.shape[1]), dtype=bool)
    for i in range(N):
        row = s_h[i, : i + 1]
        p = np.exp(row - row.max())
        keep[i, : i + 1] = p >= alpha
    return keep


def block_mask(qbar, kbar, scale: float, alpha: float, Sb: int, Wb: int) -> np.ndarray:
    """Kept-block mask per KV group, mask[g, i, j] (False above the diagonal):
    union over the group's query heads of each head's threshold, plus the
    sink blocks j < Sb and the window blocks i - Wb < j <= i."""
    if not (math.isfinite(alpha) and alpha >= 0):
        raise ValueError("alpha must be finite and >= 0")
    N, Hq, _ = qbar.shape
    Hkv = kbar.shape[1]
    G = Hq // Hkv
    s = pooled_scores(qbar, kbar, scale)
    mask = np.zeros((Hkv, N, N), dtype=bool)
    for h in range(Hq):
        mask[h // G] |= head_keep(s[h], alpha)
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    forced = (j <= i) & ((j < Sb) | (i - j < Wb))
    mask |= forced[None]
    return mask


def head_masks(qbar, kbar, scale: float, alpha: float, Sb: int, Wb: int) -> np.ndarray:
    """Per-query-head selection (the per-head reading of the threshold under
    PackGQA): keep[h, i, j] = head h's own threshold (against its own row max)
    or j a sink / window block; False above the diagonal. The group mask of
    ``block_mask`` is the OR of these over the group's heads."""
    if not (math.isfinite(alpha) and alpha >= 0):
        raise ValueError("alpha must be finite and >= 0")
    N, Hq, _ = qbar.shape
    s = pooled_scores(qbar, kbar, scale)
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    forced = (j <= i) & ((j < Sb) | (i - j < Wb))
    keep = np.zeros((Hq, N, N), dtype=bool)
    for h in range(Hq):
        keep[h] = head_keep(s[h], alpha) | forced
    return keep


def per_head_attention(Q, K, V, keep, B: int, scale: float):
    """Attention in which query head h sees only the blocks of its own selection
    keep[h] (keys <= query). Returns O [L, Hq, d], lse [Hq, L]."""
    L, Hq, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    N = num_blocks(L, B)
    O = np.empty((L, Hq, d), dtype=np.float64)
    lse = np.empty((Hq, L), dtype=np.float64)
    for h in range(Hq):
        g = h // G
        for i in range(N):
            blocks = [j for j in range(i + 1) if keep[h, i, j]]
            (o, l), = attention_rows(Q, K, V, g, i, blocks, B, scale, heads=[h]).values()
            lo, hi = i * B, min((i + 1) * B, L)
            O[lo:hi, h] = o
            lse[h, lo:hi] = l
    return O, lse


def discover_row(qbar_i: np.ndarray, kbar_g: np.ndarray, i: int, scale: float, alpha: float,
                 Sb: int, Wb: int) -> np.ndarray:
    """Kept blocks of one (KV group, query block i) row, computed on its own:
    qbar_i [G, d] are the pooled queries of the group's heads at block i,
    kbar_g [N, d] the group's pooled keys. Same steps as ``block_mask`` (per-head
    threshold against the head's row max, union, sink/window), then the
    ascending list of kept j."""
    s = scale * (qbar_i @ kbar_g[: i + 1].T)  # [G, i+1]
    keep = np.zeros(i + 1, dtype=bool)
    for h in range(s.shape[0]):
        keep |= np.exp(s[h] - s[h].max()) >= alpha
    j = np.arange(i + 1)
    keep |= (j < Sb) | (i - j < Wb)
    return np.flatnonzero(keep)


def compact(mask: np.ndarray):
    """Index compaction (Method 3): per (g, i) row, the ascending list of kept j.
    Returns (lists, cnt) with lists[g][i] an int array and cnt [Hkv, N]."""
    Hkv, N, _ = mask.shape
    lists = []
    cnt = np.zeros((Hkv, N), dtype=np.int64)
    for g in range(Hkv):
        rows = []
        for i in range(N):
            kept = [j for j in range(i + 1) if mask[g, i, j]]
            rows.append(np.array(kept, dtype=np.int64))
            cnt[g, i] = len(kept)
        lists.append(rows)
    return lists, cnt


def attention_rows(Q, K, V, g: int, i: int, blocks, B: int, scale: float, heads=None):
    """Exact masked-softmax attention for the query tokens of block i and the
    query heads of group g, over the keys of the listed blocks with key <= query.
    Q [L, Hq, d], K/V [L, Hkv, d]. Returns {h: (O [n_i, d], lse [n_i])}."""
    L, Hq, _ = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    rows = np.arange(i * B, min((i + 1) * B, L))
    keys = np.concatenate([np.arange(j * B, min((j + 1) * B, L)) for j in blocks])
    allowed = keys[None, :] <= rows[:, None]
    Kg = K[keys, g]
    Vg = V[keys, g]
    out = {}
    for h in (heads if heads is not None else range(g * G, (g + 1) * G)):
        logits = scale * (Q[rows, h] @ Kg.T)
        logits = np.where(allowed, logits, -np.inf)
        m = logits.max(axis=1, keepdims=True)
        e = np.exp(logits - m)
        z = e.sum(axis=1, keepdims=True)
        out[h] = ((e / z) @ Vg, (m + np.log(z))[:, 0])
    return out


def block_sparse_attention(Q, K, V, lists, B: int, scale: float):
    """Attention of every query over its row's kept blocks. Returns O [L, Hq, d], lse [Hq, L]."""
    L, Hq, d = Q.shape
    Hkv = K.shape[1]
    N = num_blocks(L, B)
    O = np.empty((L, Hq, d), dtype=np.float64)
    lse = np.empty((Hq, L), dtype=np.float64)
    for g in range(Hkv):
        for i in range(N):
            res = attention_rows(Q, K, V, g, i, lists[g][i], B, scale)
            lo, hi = i * B, min((i + 1) * B, L)
            for h, (o, l) in res.items():
                O[lo:hi, h] = o
                lse[h, lo:hi] = l
    return O, lse


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def flashprefill(Q, K, V, B: int, alpha: float, sink_tokens: int, window_tokens: int,
                 scale: float | None = None, attention: bool = True):
    """The whole path for one sequence: Q [L, Hq, d], K/V [L, Hkv, d] float64.
    Returns dict(qbar, kbar, mask, lists, cnt, O, lse)."""
    d = Q.shape[-1]
    scale = default_scale(d) if scale is None else scale
    Sb, Wb = forced_blocks(sink_tokens, window_tokens, B)
    qbar = pool_blocks(Q, B)
    kbar = pool_blocks(K, B)
    mask = block_mask(qbar, kbar, scale, alpha, Sb, Wb)
    lists, cnt = compact(mask)
    res = dict(qbar=qbar, kbar=kbar, mask=mask, lists=lists, cnt=cnt, scale=scale)
    if attention:
        res["O"], res["lse"] = block_sparse_attention(Q, K, V, lists, B, scale)
    return res


def gather_pages(pool: np.ndarray, table_row, L: int, page_size: int) -> np.ndarray:
    """Tokens 0..L-1 of one request from a paged pool [num_pages, page, H, d]."""
    t = np.arange(L)
    pages = np.asarray(table_row)[t // page_size]
    return pool[pages, t % page_size]


def flashprefill_paged(Q, k_pool, v_pool, cu_seqlens, page_table, page_size: int, B: int,
                       alpha: float, sink_tokens: int, window_tokens: int,
                       scale: float | None = None, attention: bool = True):
    """Continuous batching over a paged KV cache: the path applied to each request
    on its own tokens. Q [T, Hq, d] packed by cu_seqlens. Returns a list of
    per-request result dicts (as ``flashprefill``) plus the packed O/lse."""
    cu = [int(x) for x in cu_seqlens]
    out = []
    for r in range(len(cu) - 1):
        L = cu[r + 1] - cu[r]
        Kr = gather_pages(k_pool, page_table[r], L, page_size)
        Vr = gather_pages(v_pool, page_table[r], L, page_size)
        out.append(flashprefill(Q[cu[r]:cu[r + 1]], Kr, Vr, B, alpha, sink_tokens,
                                window_tokens, scale, attention))
    return out


def flashprefill_chunk(Qc, K, V, B: int, alpha: float, sink_tokens: int, window_tokens: int,
                       scale: float | None = None, attention: bool = True):
    """Prefill of a request's last queries against its whole KV (chunked prefill
    with a cached prefix): K/V [kv_len, Hkv, d] hold every token of the
    request, Qc [q_len, Hq, d] the queries of its last q_len tokens, which sit
    at positions p0 = kv_len - q_len .. kv_len - 1.

    Same steps as ``flashprefill`` on the block grid of the KV positions
    (blocks start at the request's first token): a query block is pooled over
    the queries it holds (blocks wholly before p0 hold none and get an empty
    list), key blocks over their tokens; scores, threshold, union and sink /
    window forcing as before; each query attends to the keys of its row's kept
    blocks at positions <= its own. With q_len = kv_len this is ``flashprefill``.
    Returns dict(qbar (None rows for empty blocks), kbar, mask, lists, cnt, O
    [q_len, Hq, d], lse [Hq, q_len], p0)."""
    d = Qc.shape[-1]
    scale = default_scale(d) if scale is None else scale
    if not (math.isfinite(alpha) and alpha >= 0):
        raise ValueError("alpha must be finite and >= 0")
    kv_len, q_len = K.shape[0], Qc.shape[0]
    if q_len > kv_len:
        raise ValueError("more queries than keys")
    p0 = kv_len - q_len
    N = num_blocks(kv_len, B)
    Hq, Hkv = Qc.shape[1], K.shape[1]
    G = Hq // Hkv
    Sb, Wb = forced_blocks(sink_tokens, window_tokens, B)
    kbar = pool_blocks(K, B)
    mask = np.zeros((Hkv, N, N), dtype=bool)
    qbar = [None] * N
    for i in range(N):
        lo, hi = max(i * B, p0), min((i + 1) * B, kv_len)
        if lo >= hi:
            continue
        qbar[i] = Qc[lo - p0: hi - p0].sum(axis=0, dtype=np.float64) / (hi - lo)
    # the keep rule per row, with the same steps as block_mask
    for i in range(N):
        if qbar[i] is None:
            continue
        for g in range(Hkv):
            keep = np.zeros(i + 1, dtype=bool)
            for h in range(g * G, (g + 1) * G):
                s = scale * (kbar[: i + 1, g, :] @ qbar[i][h])
                keep |= np.exp(s - s.max()) >= alpha
            j = np.arange(i + 1)
            keep |= (j < Sb) | (i - j < Wb)
            mask[g, i, : i + 1] = keep
    lists, cnt = compact(mask)
    res = dict(qbar=qbar, kbar=kbar, mask=mask, lists=lists, cnt=cnt, scale=scale, p0=p0)
    if attention:
        O = np.zeros((q_len, Hq, d))
        lse = np.full((Hq, q_len), -np.inf)
        for g in range(Hkv):
            for i in range(N):
                lo, hi = max(i * B, p0), min((i + 1) * B, kv_len)
                if lo >= hi:
                    continue
                rows = np.arange(lo, hi)
                keys = np.concatenate([np.arange(j * B, min((j + 1) * B, kv_len)) for j in lists[g][i]])
                allowed = keys[None, :] <= rows[:, None]
                for h in range(g * G, (g + 1) * G):
                    logits = scale * (Qc[rows - p0, h] @ K[keys, g].T)
                    logits = np.where(allowed, logits, -np.inf)
                    m = logits.max(axis=1, keepdims=True)
                    e = np.exp(logits - m)
                    z = e.sum(axis=1, keepdims=True)
                    O[rows - p0, h] = (e / z) @ V[keys, g]
                    lse[h, rows - p0] = (m + np.log(z))[:, 0]
        res["O"], res["lse"] = O, lse
    return res


def row_borderline(qbar, kbar, scale: float, alpha: float, g: int, i: int, rel: float = 1e-5):
    """Blocks j <= i of row (g, i) whose probability p = exp(s - rowmax) lies within
    ``rel * alpha`` of alpha for some head of the group: where a float32 kernel may
    decide the other way. Returns a set of j."""
    if alpha <= 0:
        return set()
    Hq = qbar.shape[1]
    Hkv = kbar.shape[1]
    G = Hq // Hkv
    out = set()
    for h in range(g * G, (g + 1) * G):
        s = scale * (kbar[: i + 1, g, :] @ qbar[i, h, :])
        p = np.exp(s - s.max())
        out |= set(np.flatnonzero(np.abs(p - alpha) <= rel * alpha).tolist())
    return out
