"""Pins for the CPU oracle: each check ties it to something other than itself.

* a hand-derived worked example (tests/golden/hand_example.json),
* library routines that reduce to special cases (torch avg_pool1d for block
  means, torch scaled_dot_product_attention in float64 for dense causal and
  boolean-masked attention, numpy flatnonzero for compaction),
* closed forms (alpha = 0 keeps every causal block, alpha > 1 only the forced
  ones, alpha = 1 only the row maxima, constant blocks pool to the constant,
  Q = 0 gives the mean of V over the allowed keys, rows of P sum to one),
* an independent per-element brute force on tiny inputs,
* mutation checks: mistakes planted in the oracle (on the CPU) must fail a pin.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import flashprefill_oracle as fo

GOLD = os.path.join(os.path.dirname(__file__), "golden", "hand_example.json")


def _hand():
    with open(GOLD) as f:
        return json.load(f)


def _arr(x):
    return np.array(x, dtype=np.float64)


def _eval(expr):
    return eval(expr, {"e": math.e, "exp": math.exp, "log": math.log, "__builtins__": {}})


def _lists(res):
    return [[list(map(int, l)) for l in rows] for rows in res["lists"]]


# ----------------------------------------------------------------------------- golden
@pytest.mark.parametrize("case", [c["name"] for c in _hand()["cases"]])
def test_hand_example_lists(case):
    f = _hand()
    c = next(c for c in f["cases"] if c["name"] == case)
    Q, K, V = _arr(f["Q"]), _arr(f["K"]), _arr(f["V"])
    res = oracle.flashprefill(Q, K, V, f["B"], c["alpha"], c["sink_tokens"], c["window_tokens"],
                              scale=c["scale"])
    assert _lists(res) == c["lists"]
    np.testing.assert_array_equal(res["qbar"], _arr(f["pooled"]["qbar"]))
    np.testing.assert_array_equal(res["kbar"], _arr(f["pooled"]["kbar"]))
    assert res["cnt"].tolist() == [[len(l) for l in rows] for rows in c["lists"]]


def test_hand_example_attention():
    f = _hand()
    Q, K, V = _arr(f["Q"]), _arr(f["K"]), _arr(f["V"])
    for a in f["attention"]:
        c = next(c for c in f["cases"] if c["name"] == a["case"])
        res = oracle.flashprefill(Q, K, V, f["B"], c["alpha"], c["sink_tokens"],
                                  c["window_tokens"], scale=c["scale"])
        want = [_eval(x) for x in a["O"]]
        np.testing.assert_allclose(res["O"][a["t"], a["h"]], want, rtol=0, atol=1e-13)
        assert abs(res["lse"][a["h"], a["t"]] - _eval(a["lse"])) < 1e-13


# ----------------------------------------------------------------------------- helpers
def _rand(L, hq, hkv, d, seed, amp=0.0):
    g = np.random.default_rng(seed)
    Q = g.standard_normal((L, hq, d))
    K = g.standard_normal((L, hkv, d))
    V = g.standard_normal((L, hkv, d))
    if amp:
        u = g.standard_normal(d)
        u /= np.linalg.norm(u)
        Q += amp * u
        heavy = g.choice(-(-L // 4), size=2, replace=False)
        for j in heavy:
            K[4 * j: 4 * j + 4] += amp * u
    return Q, K, V


def _token_mask(mask_g, L, B):
    """Token-level boolean mask [L, L] from a block mask: block kept and key <= query."""
    t = np.arange(L)
    m = mask_g[t[:, None] // B, t[None, :] // B] & (t[None, :] <= t[:, None])
    return m


def _sdpa(Q, K, V, token_masks, G, scale):
    """torch scaled_dot_product_attention in float64; token_masks [Hkv, L, L] or None (causal)."""
    q = torch.from_numpy(Q).permute(1, 0, 2)[None]
    k = torch.from_numpy(K).permute(1, 0, 2)[None]
    v = torch.from_numpy(V).permute(1, 0, 2)[None]
    if token_masks is None:
        o = F.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale, enable_gqa=True)
    else:
        m = torch.from_numpy(np.repeat(token_masks, G, axis=0))[None]
        o = F.scaled_dot_product_attention(q, k, v, attn_mask=m, scale=scale, enable_gqa=True)
    return o[0].permute(1, 0, 2).numpy()


# ----------------------------------------------------------------------------- pooling
@pytest.mark.parametrize("L,B", [(7, 2), (64, 16), (70, 16), (33, 32), (5, 8)])
def test_pool_matches_avg_pool1d(L, B):
    X = np.random.default_rng(L * B).standard_normal((L, 3, 5))
    got = oracle.pool_blocks(X, B)
    x = torch.from_numpy(X).permute(1, 2, 0).reshape(1, 15, L)
    want = F.avg_pool1d(x, B, B, ceil_mode=True).reshape(3, 5, -1).permute(2, 0, 1).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-14, atol=1e-14)


def test_pool_constant_blocks():
    B, N = 8, 5
    vals = np.random.default_rng(0).standard_normal((N, 2, 4))
    X = np.repeat(vals, B, axis=0)[: N * B - 3]  # ragged tail of 5 tokens
    np.testing.assert_allclose(oracle.pool_blocks(X, B), vals, rtol=0, atol=1e-15)


# ----------------------------------------------------------------------------- threshold
def test_alpha_zero_keeps_all_causal():
    Q, K, V = _rand(40, 4, 2, 8, 1, amp=3.0)
    r = oracle.flashprefill(Q, K, V, 4, 0.0, 0, 0, attention=False)
    N = 10
    assert (r["mask"] == np.tril(np.ones((N, N), bool))[None]).all()


def test_alpha_above_one_keeps_forced_only():
    Q, K, V = _rand(40, 4, 2, 8, 2, amp=3.0)
    B, sink, win = 4, 5, 9  # Sb = 2, Wb = 3
    r = oracle.flashprefill(Q, K, V, B, 1.5, sink, win, attention=False)
    N = 10
    i, j = np.meshgrid(np.arange(N), np.arange(N), indexing="ij")
    want = (j <= i) & ((j < 2) | (i - j < 3))
    assert (r["mask"] == want[None]).all()


def test_alpha_one_keeps_row_maxima():
    Q, K, V = _rand(48, 6, 2, 8, 3, amp=2.0)
    B = 4
    r = oracle.flashprefill(Q, K, V, B, 1.0, 0, 0, attention=False)
    s = oracle.pooled_scores(r["qbar"], r["kbar"], r["scale"])
    N, G = 12, 3
    for g in range(2):
        for i in range(N):
            want = {i}  # window of one block
            for h in range(g * G, (g + 1) * G):
                want.add(int(np.argmax(s[h, i, : i + 1])))
            assert set(np.flatnonzero(r["mask"][g, i]).tolist()) == want


def test_mask_monotone_in_alpha_and_union_superset():
    Q, K, V = _rand(64, 4, 1, 8, 4, amp=2.5)
    B = 4
    prev = None
    for a in [0.0, 1e-3, 0.05, 0.1, 0.3, 0.7, 1.0, 2.0]:
        r = oracle.flashprefill(Q, K, V, B, a, 4, 4, attention=False)
        if prev is not None:
            assert (prev | r["mask"] == prev).all()  # larger alpha keeps a subset
        prev = r["mask"]
        s = oracle.pooled_scores(r["qbar"], r["kbar"], r["scale"])
        for h in range(4):
            assert (r["mask"][0] | oracle.head_keep(s[h], a) == r["mask"][0]).all()


def test_invalid_alpha_rejected():
    Q, K, V = _rand(8, 2, 1, 4, 5)
    for a in [-0.1, float("nan"), float("inf")]:
        with pytest.raises(ValueError):
            oracle.flashprefill(Q, K, V, 4, a, 0, 0)


def test_forced_blocks_conversion():
    assert oracle.forced_blocks(256, 512, 128) == (2, 4)
    assert oracle.forced_blocks(64, 128, 64) == (1, 2)
    assert oracle.forced_blocks(0, 0, 128) == (0, 1)
    assert oracle.forced_blocks(1, 129, 128) == (1, 2)


# ----------------------------------------------------------------------------- compaction
def test_compact_is_flatnonzero():
    rng = np.random.default_rng(6)
    N = 37
    mask = np.tril(rng.random((3, N, N)) < 0.3)
    lists, cnt = oracle.compact(mask)
    for g in range(3):
        for i in range(N):
            np.testing.assert_array_equal(lists[g][i], np.flatnonzero(mask[g, i]))
            assert cnt[g, i] == np.count_nonzero(mask[g, i])


# ----------------------------------------------------------------------------- attention
@pytest.mark.parametrize("L,B,hq,hkv", [(64, 8, 4, 2), (70, 16, 6, 2), (33, 32, 2, 1), (96, 16, 8, 1)])
def test_alpha_zero_equals_dense_causal_sdpa(L, B, hq, hkv):
    d = 16
    Q, K, V = _rand(L, hq, hkv, d, L + B, amp=2.0)
    r = oracle.flashprefill(Q, K, V, B, 0.0, 0, 0)
    want = _sdpa(Q, K, V, None, hq // hkv, 1 / math.sqrt(d))
    np.testing.assert_allclose(r["O"], want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("alpha", [0.05, 0.3, 1.0, 3.0])
def test_masked_attention_equals_masked_sdpa(alpha):
    L, B, hq, hkv, d = 80, 8, 4, 2, 16
    Q, K, V = _rand(L, hq, hkv, d, 11, amp=4.0)
    r = oracle.flashprefill(Q, K, V, B, alpha, 8, 8)
    tm = np.stack([_token_mask(r["mask"][g], L, B) for g in range(hkv)])
    want = _sdpa(Q, K, V, tm, hq // hkv, 1 / math.sqrt(d))
    np.testing.assert_allclose(r["O"], want, rtol=1e-12, atol=1e-12)


def test_lse_and_row_sums():
    L, B, hq, hkv, d = 48, 8, 4, 2, 8
    Q, K, V = _rand(L, hq, hkv, d, 12, amp=3.0)
    r = oracle.flashprefill(Q, K, V, B, 0.2, 8, 8)
    scale = r["scale"]
    for g in range(hkv):
        for i in range(L // B):
            keys = np.concatenate([np.arange(j * B, (j + 1) * B) for j in r["lists"][g][i]])
            for h in range(g * 2, g * 2 + 2):
                for t in range(i * B, (i + 1) * B):
                    ks = keys[keys <= t]
                    p = np.exp(scale * (K[ks, g] @ Q[t, h]) - r["lse"][h, t])
                    assert abs(p.sum() - 1.0) < 1e-12
    Vones = np.ones_like(V)
    r1 = oracle.flashprefill(Q, K, Vones, B, 0.2, 8, 8)
    np.testing.assert_allclose(r1["O"], 1.0, rtol=0, atol=1e-13)


def test_zero_queries_average_allowed_values():
    L, B, hq, hkv, d = 40, 8, 2, 1, 8
    Q, K, V = _rand(L, hq, hkv, d, 13)
    Q0 = np.zeros_like(Q)
    # With Q = 0 all pooled scores tie, so every causal block is kept for any alpha <= 1;
    # the output is the plain mean of V over keys 0..t.
    r = oracle.flashprefill(Q0, K, V, B, 0.5, 0, 0)
    for t in range(L):
        np.testing.assert_allclose(r["O"][t, 0], V[: t + 1, 0].mean(axis=0), atol=1e-13)
    # alpha > 1 keeps only the diagonal block: mean over its keys <= t.
    r = oracle.flashprefill(Q0, K, V, B, 2.0, 0, 0)
    for t in range(L):
        lo = (t // B) * B
        np.testing.assert_allclose(r["O"][t, 1], V[lo: t + 1, 0].mean(axis=0), atol=1e-13)


# ----------------------------------------------------------------------------- brute force
@pytest.mark.parametrize("L,B,hq,hkv,d,alpha,sink,win", [
    (16, 4, 2, 1, 4, 0.3, 0, 0),
    (23, 4, 4, 2, 3, 0.1, 4, 8),
    (20, 8, 3, 1, 5, 1.0, 0, 9),
    (18, 2, 2, 2, 2, 0.6, 3, 2),
    (12, 16, 2, 1, 4, 0.2, 0, 0),
])
def test_oracle_matches_brute_force(L, B, hq, hkv, d, alpha, sink, win):
    Q, K, V = _rand(L, hq, hkv, d, L * 7 + B, amp=3.0)
    r = oracle.flashprefill(Q, K, V, B, alpha, sink, win)
    bf = oracle.brute_force(Q.tolist(), K.tolist(), V.tolist(), B, alpha, sink, win)
    assert _lists(r) == bf["lists"]
    np.testing.assert_allclose(r["O"], np.array(bf["O"]), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["lse"], np.array(bf["lse"]), rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- paged / varlen
def _paged_case(lens, P, hq, hkv, d, seed, perm=True):
    rng = np.random.default_rng(seed)
    seqs = [(rng.standard_normal((L, hq, d)), rng.standard_normal((L, hkv, d)),
             rng.standard_normal((L, hkv, d))) for L in lens]
    npages = [-(-L // P) for L in lens]
    total = sum(npages)
    order = rng.permutation(total) if perm else np.arange(total)
    kp = np.zeros((total, P, hkv, d))
    vp = np.zeros((total, P, hkv, d))
    table = -np.ones((len(lens), max(npages)), dtype=np.int64)
    off = 0
    for r, (L, (q, k, v)) in enumerate(zip(lens, seqs)):
        for p in range(npages[r]):
            pg = order[off + p]
            table[r, p] = pg
            n = min(P, L - p * P)
            kp[pg, :n] = k[p * P: p * P + n]
            vp[pg, :n] = v[p * P: p * P + n]
        off += npages[r]
    Q = np.concatenate([s[0] for s in seqs])
    cu = np.concatenate([[0], np.cumsum(lens)])
    return seqs, Q, kp, vp, table, cu


@pytest.mark.parametrize("perm", [False, True])
def test_paged_equals_per_request_contiguous(perm):
    lens, P, B = [37, 16, 50], 4, 8
    seqs, Q, kp, vp, table, cu = _paged_case(lens, P, 4, 2, 8, 21, perm)
    res = oracle.flashprefill_paged(Q, kp, vp, cu, table, P, B, 0.2, 8, 8)
    for r, (q, k, v) in enumerate(seqs):
        ref = oracle.flashprefill(q, k, v, B, 0.2, 8, 8)
        assert _lists(res[r]) == _lists(ref)
        np.testing.assert_array_equal(res[r]["O"], ref["O"])


def test_gather_pages_identity_and_permutation():
    rng = np.random.default_rng(3)
    P, L = 4, 13
    pool = rng.standard_normal((6, P, 2, 3))
    table = np.array([5, 0, 3, 1])
    got = oracle.gather_pages(pool, table, L, P)
    for t in range(L):
        np.testing.assert_array_equal(got[t], pool[table[t // P], t % P])


# ----------------------------------------------------------------------------- mutations
def _pins_pass():
    """Run the golden and library pins once; True if all of them hold."""
    try:
        for c in _hand()["cases"]:
            test_hand_example_lists(c["name"])
        test_hand_example_attention()
        test_alpha_one_keeps_row_maxima()
        test_masked_attention_equals_masked_sdpa(0.3)
        test_pool_matches_avg_pool1d(70, 16)
        test_alpha_zero_equals_dense_causal_sdpa(64, 8, 4, 2)
    except AssertionError:
        return False
    return True


def _mut_strict_threshold(s_h, alpha):
    N = s_h.shape[0]
    keep = np.zeros((N, s_h.shape[1]), dtype=bool)
    for i in range(N):
        row = s_h[i, : i + 1]
        keep[i, : i + 1] = np.exp(row - row.max()) > alpha
    return keep


def _mut_global_max(s_h, alpha):
    N = s_h.shape[0]
    tri = np.tril(np.ones((N, N), bool))
    m = s_h[tri].max()
    return tri & (np.exp(s_h - m) >= alpha)


def _mut_sum_pool(X, B):
    L = X.shape[0]
    N = -(-L // B)
    return np.stack([X[i * B: (i + 1) * B].sum(axis=0) for i in range(N)])


def _mut_full_block_pool(X, B):
    L = X.shape[0]
    N = -(-L // B)
    return np.stack([X[i * B: (i + 1) * B].sum(axis=0) / B for i in range(N)])


def _mut_transposed_scores(qbar, kbar, scale):
    s = fo.__dict__["_orig_pooled_scores"](qbar, kbar, scale)
    return np.swapaxes(s, 1, 2).copy()


def _mut_unscaled_scores(qbar, kbar, scale):
    return fo.__dict__["_orig_pooled_scores"](qbar, kbar, 1.0)


def _mut_forced_window_off_by_one(sink, win, B):
    Sb, Wb = fo.__dict__["_orig_forced_blocks"](sink, win, B)
    return Sb, Wb + 1


def _mut_attention_strict_causal(Q, K, V, g, i, blocks, B, scale, heads=None):
    L, Hq, _ = Q.shape
    G = Hq // K.shape[1]
    rows = np.arange(i * B, min((i + 1) * B, L))
    keys = np.concatenate([np.arange(j * B, min((j + 1) * B, L)) for j in blocks])
    allowed = (keys[None, :] < rows[:, None]) | (rows[:, None] == 0)
    out = {}
    for h in (heads if heads is not None else range(g * G, (g + 1) * G)):
        lg = np.where(allowed, scale * (Q[rows, h] @ K[keys, g].T), -np.inf)
        m = lg.max(axis=1, keepdims=True)
        e = np.exp(lg - m)
        z = e.sum(axis=1, keepdims=True)
        out[h] = ((e / z) @ V[keys, g], (m + np.log(z))[:, 0])
    return out


@pytest.mark.parametrize("name,func", [
    ("head_keep", _mut_strict_threshold),
    ("head_keep", _mut_global_max),
    ("pool_blocks", _mut_sum_pool),
    ("pool_blocks", _mut_full_block_pool),
    ("pooled_scores", _mut_transposed_scores),
    ("pooled_scores", _mut_unscaled_scores),
    ("forced_blocks", _mut_forced_window_off_by_one),
    ("attention_rows", _mut_attention_strict_causal),
])
def test_planted_mistake_fails_a_pin(monkeypatch, name, func):
    assert _pins_pass()
    monkeypatch.setitem(fo.__dict__, "_orig_pooled_scores", fo.pooled_scores)
    monkeypatch.setitem(fo.__dict__, "_orig_forced_blocks", fo.forced_blocks)
    monkeypatch.setattr(fo, name, func)
    monkeypatch.setattr(oracle, name, func, raising=False)
    assert not _pins_pass(), f"mutation of {name} ({func.__name__}) went unnoticed"


def test_discover_row_agrees_with_block_mask():
    """The per-row entry point (used to time bounded samples) takes the same steps."""
    Q, K, V = _rand(96, 8, 2, 8, 31, amp=3.0)
    B, a, sink, win = 8, 0.2, 8, 16
    r = oracle.flashprefill(Q, K, V, B, a, sink, win, attention=False)
    Sb, Wb = oracle.forced_blocks(sink, win, B)
    for g in range(2):
        for i in range(12):
            got = oracle.discover_row(r["qbar"][i, 4 * g: 4 * g + 4], r["kbar"][:, g], i, r["scale"], a, Sb, Wb)
            np.testing.assert_array_equal(got, np.flatnonzero(r["mask"][g, i]))


# ----------------------------------------------------------------------------- chunked prefill
def _chunk_case(kv_len, hq=4, hkv=2, d=8, seed=77):
    Q, K, V = _rand(kv_len, hq, hkv, d, seed, amp=3.0)
    return Q, K, V


def test_chunk_with_all_queries_is_full_prefill():
    Q, K, V = _chunk_case(70)
    full = oracle.flashprefill(Q, K, V, 8, 0.2, 8, 16)
    ch = oracle.flashprefill_chunk(Q, K, V, 8, 0.2, 8, 16)
    assert _lists(ch) == _lists(full)
    np.testing.assert_array_equal(ch["O"], full["O"])
    np.testing.assert_array_equal(ch["lse"], full["lse"])


def test_block_aligned_chunk_equals_full_prefill_rows():
    """With the chunk boundary on a block boundary every query block holds the
    same queries as in full prefill, so lists and outputs coincide."""
    kv_len, B, p0 = 90, 8, 40
    Q, K, V = _chunk_case(kv_len)
    full = oracle.flashprefill(Q, K, V, B, 0.2, 8, 16)
    ch = oracle.flashprefill_chunk(Q[p0:], K, V, B, 0.2, 8, 16)
    for g in range(2):
        for i in range(p0 // B):
            assert len(ch["lists"][g][i]) == 0
        for i in range(p0 // B, len(full["lists"][g])):
            assert ch["lists"][g][i].tolist() == full["lists"][g][i].tolist()
    np.testing.assert_allclose(ch["O"], full["O"][p0:], rtol=0, atol=1e-13)


def test_chunk_partial_first_block_pools_present_queries():
    kv_len, B, p0 = 50, 8, 21  # block 2 holds queries at positions 21..23 only
    Q, K, V = _chunk_case(kv_len)
    ch = oracle.flashprefill_chunk(Q[p0:], K, V, B, 0.2, 0, 0, attention=False)
    assert ch["qbar"][0] is None and ch["qbar"][1] is None
    np.testing.assert_allclose(ch["qbar"][2], Q[21:24].mean(axis=0), atol=1e-15)
    np.testing.assert_allclose(ch["qbar"][3], Q[24:32].mean(axis=0), atol=1e-15)


@pytest.mark.parametrize("kv_len,p0,alpha", [(64, 13, 0.1), (77, 40, 1.0), (40, 39, 0.0), (33, 0, 3.0)])
def test_chunk_attention_equals_masked_sdpa(kv_len, p0, alpha):
    B, hq, hkv, d = 8, 4, 2, 8
    Q, K, V = _chunk_case(kv_len, hq, hkv, d, seed=kv_len + p0)
    ch = oracle.flashprefill_chunk(Q[p0:], K, V, B, alpha, 8, 8)
    # token mask: query position t (p0..kv_len-1) sees key k iff block(k) is kept in row block(t) and k <= t
    t = np.arange(p0, kv_len)
    kk = np.arange(kv_len)
    tm = np.stack([ch["mask"][g][t[:, None] // B, kk[None, :] // B] & (kk[None, :] <= t[:, None])
                   for g in range(hkv)])
    q = torch.from_numpy(Q[p0:]).permute(1, 0, 2)[None]
    k = torch.from_numpy(K).permute(1, 0, 2)[None]
    v = torch.from_numpy(V).permute(1, 0, 2)[None]
    m = torch.from_numpy(np.repeat(tm, hq // hkv, axis=0))[None]
    want = F.scaled_dot_product_attention(q, k, v, attn_mask=m, scale=1 / math.sqrt(d), enable_gqa=True)
    np.testing.assert_allclose(ch["O"], want[0].permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)


def test_chunk_rejects_bad_arguments():
    Q, K, V = _chunk_case(20)
    with pytest.raises(ValueError):
        oracle.flashprefill_chunk(Q, K[:10], V[:10], 8, 0.1, 0, 0)
    with pytest.raises(ValueError):
        oracle.flashprefill_chunk(Q[5:], K, V, 8, -1.0, 0, 0)


# ----------------------------------------------------------------------------- per-head masks
def test_head_masks_union_is_group_mask_and_single_head_group_agrees():
    Q, K, V = _rand(96, 8, 2, 8, 5, amp=3.0)
    r = oracle.flashprefill(Q, K, V, 8, 0.2, 8, 16, attention=False)
    Sb, Wb = oracle.forced_blocks(8, 16, 8)
    hm = oracle.head_masks(r["qbar"], r["kbar"], r["scale"], 0.2, Sb, Wb)
    for g in range(2):
        np.testing.assert_array_equal(hm[4 * g: 4 * g + 4].any(axis=0), r["mask"][g])
    # with one query head per group the per-head and group selections coincide
    Q1, K1, V1 = _rand(64, 2, 2, 8, 6, amp=3.0)
    r1 = oracle.flashprefill(Q1, K1, V1, 8, 0.2, 8, 8)
    hm1 = oracle.head_masks(r1["qbar"], r1["kbar"], r1["scale"], 0.2, *oracle.forced_blocks(8, 8, 8))
    np.testing.assert_array_equal(hm1, r1["mask"])
    O1, l1 = oracle.per_head_attention(Q1, K1, V1, hm1, 8, r1["scale"])
    np.testing.assert_allclose(O1, r1["O"], rtol=0, atol=1e-13)


@pytest.mark.parametrize("alpha", [0.05, 0.5, 1.0])
def test_per_head_attention_equals_per_head_masked_sdpa(alpha):
    L, B, hq, hkv, d = 72, 8, 4, 2, 8
    Q, K, V = _rand(L, hq, hkv, d, 21, amp=4.0)
    r = oracle.flashprefill(Q, K, V, B, alpha, 8, 8, attention=False)
    hm = oracle.head_masks(r["qbar"], r["kbar"], r["scale"], alpha, *oracle.forced_blocks(8, 8, B))
    O, lse = oracle.per_head_attention(Q, K, V, hm, B, r["scale"])
    t = np.arange(L)
    tm = np.stack([hm[h][t[:, None] // B, t[None, :] // B] & (t[None, :] <= t[:, None]) for h in range(hq)])
    q = torch.from_numpy(Q).permute(1, 0, 2)[None]
    k = torch.from_numpy(np.repeat(K, hq // hkv, axis=1)).permute(1, 0, 2)[None]
    v = torch.from_numpy(np.repeat(V, hq // hkv, axis=1)).permute(1, 0, 2)[None]
    want = F.scaled_dot_product_attention(q, k, v, attn_mask=torch.from_numpy(tm)[None], scale=r["scale"])
    np.testing.assert_allclose(O, want[0].permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)


def test_row_borderline_finds_blocks_at_alpha():
    """Pooled vectors built so that block 1 has exactly probability alpha in
    head 0's row and block 2 sits well above it: only block 1 is borderline,
    and a perturbation beyond the band takes it out."""
    alpha, scale, d = 0.1, 1.0, 4
    kbar = np.zeros((3, 1, d))
    kbar[0, 0, 0] = 1.0                    # s0 = 1 (row max)
    kbar[1, 0, 0] = 1.0 + math.log(alpha)  # s1 - s0 = ln(alpha): p1 = alpha exactly
    kbar[2, 0, 0] = 0.9                    # p2 = exp(-0.1), far from alpha
    qbar = np.zeros((3, 1, d))
    qbar[2, 0, 0] = 1.0
    assert fo.row_borderline(qbar, kbar, scale, alpha, 0, 2) == {1}
    kbar[1, 0, 0] += 1e-3                  # p1 = alpha * e^1e-3: outside 1e-5 relative
    assert fo.row_borderline(qbar, kbar, scale, alpha, 0, 2) == set()
    assert fo.row_borderline(qbar, kbar, scale, 0.0, 0, 2) == set()  # alpha = 0 has no boundary


# ----------------------------------------------------------------------------- randomised
from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=40, deadline=None, derandomize=True)
@given(L=st.integers(1, 40), B=st.sampled_from([4, 8, 16]), hkv=st.integers(1, 2), G=st.integers(1, 3),
       alpha=st.sampled_from([0.0, 1e-3, 0.1, 0.5, 1.0, 2.0]), sink=st.integers(0, 12), win=st.integers(0, 20),
       seed=st.integers(0, 10_000))
def test_oracle_matches_brute_force_random_shapes(L, B, hkv, G, alpha, sink, win, seed):
    """The vectorised oracle against the per-element brute force on random tiny
    shapes (ragged tails, every group size up to 3, sink/window in tokens)."""
    Q, K, V = _rand(L, hkv * G, hkv, 4, seed, amp=2.0 if L > 4 else 0.0)  # (heavy blocks need L > 4)
    r = oracle.flashprefill(Q, K, V, B, alpha, sink, win)
    bf = oracle.brute_force(Q.tolist(), K.tolist(), V.tolist(), B, alpha, sink, win)
    assert _lists(r) == bf["lists"]
    np.testing.assert_allclose(r["O"], np.array(bf["O"]), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(r["lse"], np.array(bf["lse"]), rtol=1e-10, atol=1e-12)
