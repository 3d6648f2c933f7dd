"""GPU parity of the CUDA path (through the C ABI) against the float64 oracle.

Discovery + compaction: kept-block lists bit-exact except borderline blocks
(exact probability within 1e-5 relative of alpha). Attention: run on the
oracle's own lists; BF16 max |err| <= 2e-2, mean <= 2e-3; FP8 max <= 6e-2.
Small cases span several tiles and a ragged tail; the full-size workloads are
checked on sampled query blocks.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_blocks_b200 import workloads as wl
from tests import _helpers as H

pytestmark = pytest.mark.gpu

W = wl.workloads()


def _case(name, L=None, **kw):
    w = W[name]
    if L is not None:
        w = wl.small_case(w, L)
    return w.with_(**kw) if kw else w


def _inputs(w, fp8=False):
    inp = wl.make_inputs(w)
    return wl.to_fp8(inp) if fp8 else inp


def _mask_matches_lists(dev):
    m = dev.mask()
    lists = dev.lists()
    for r in range(dev.cfg.batch):
        for g in range(dev.cfg.hkv):
            for i in range(dev.cfg.nmax):
                assert np.flatnonzero(m[r, g, i]).tolist() == lists[r][g][i]


# ----------------------------------------------------------------------------- discovery
DISCOVERY_CASES = [
    ("tiny2k", None, None),
    ("qwen7b_32k", 4096, 0.0),
    ("qwen7b_32k", 4096, 0.05),
    ("qwen7b_32k", 5000, 0.2),
    ("qwen30b_128k", 8192, None),
    ("qwen30b_128k", 3000, 1.0),
    ("extreme_256k", 8192, None),
    ("extreme_256k", 1000, 3.0),
]


@pytest.mark.parametrize("name,L,alpha", DISCOVERY_CASES)
@pytest.mark.parametrize("fused", [True, False])
def test_discovery_matches_oracle(name, L, alpha, fused):
    w = _case(name, L)
    inp = _inputs(w)
    dev = H.Device(w, inp, alpha)
    dev.discover(fused=fused)
    assert dev.status() == 0
    orc = H.oracle_discovery(w, inp, alpha)
    H.compare_lists(orc, dev.lists())
    _mask_matches_lists(dev)


# Cases spanning several 128-block column tiles of the scoring kernel (ragged
# last tile) and the group sizes it specialises.
TILE_CASES = [
    ("qwen30b_128k", 40000, {}),                     # G=8, Nmax=313: three column tiles
    ("tiny2k", 10000, {}),                           # B=64, G=4, Nmax=157
    ("qwen7b_32k", 20000, {}),                       # G=7: 18 query blocks x 7 heads per tile
    ("qwen30b_128k", 9000, {"hkv": 2}),              # G=16
    ("qwen30b_128k", 9000, {"hq": 4}),               # G=1: 128 query blocks per tile
    ("qwen30b_128k", 20000, {"hq": 6, "hkv": 2}),    # G=3
]


@pytest.mark.parametrize("name,L,kw", TILE_CASES)
def test_discovery_column_tiles_and_groups(name, L, kw):
    w = _case(name, L, **kw)
    inp = _inputs(w)
    dev = H.Device(w, inp)
    dev.discover()
    assert dev.status() == 0
    H.compare_lists(H.oracle_discovery(w, inp), dev.lists())
    _mask_matches_lists(dev)


@pytest.mark.parametrize("name,L", [("tiny2k", None), ("qwen30b_128k", 4096)])
def test_discovery_fp8_matches_oracle(name, L):
    w = _case(name, L)
    inp = _inputs(w, fp8=True)
    dev = H.Device(w, inp)
    dev.discover()
    assert dev.status() == 0
    H.compare_lists(H.oracle_discovery(w, inp), dev.lists())


def test_discovery_alpha_zero_and_above_one():
    w = _case("qwen30b_128k", 2000)
    inp = _inputs(w)
    for alpha, expect in [(0.0, "all"), (1.5, "forced")]:
        dev = H.Device(w, inp, alpha)
        dev.discover()
        lists = dev.lists()[0]
        N = dev.cfg.nmax
        Sb, Wb = oracle.forced_blocks(w.sink_tokens, w.window_tokens, w.block)
        for g in range(w.hkv):
            for i in range(N):
                want = list(range(i + 1)) if expect == "all" else \
                    [j for j in range(i + 1) if j < Sb or i - j < Wb]
                assert lists[g][i] == want


# ----------------------------------------------------------------------------- attention
ATTN_CASES = [
    ("tiny2k", None, None),              # B=64, G=4, full size
    ("qwen7b_32k", 2048, 0.0),           # G=7 (112-row M-tiles), alpha=0: dense causal
    ("qwen30b_128k", 3000, None),        # G=8, ragged tail
    ("qwen30b_128k", 4096, 0.3),
    ("extreme_256k", 2500, None),
    ("qwen30b_128k", 100, None),         # one partial block
]


@pytest.mark.parametrize("name,L,alpha", ATTN_CASES)
@pytest.mark.parametrize("fp8", [False, True])
def test_attention_on_oracle_lists(name, L, alpha, fp8):
    w = _case(name, L)
    inp = _inputs(w, fp8)
    dev = H.Device(w, inp, alpha)
    orc = H.oracle_discovery(w, inp, alpha)
    idx, cnt = H.upload_lists(dev.cfg, [o["lists"] for o in orc])
    dev.attend(idx, cnt)
    assert dev.status() == 0
    H.check_attention(dev, H.oracle_attention(w, inp, orc), fp8)


# PackGQA M-tile shapes beyond G = 4, 7, 8: G = 1 (64 tokens x 1 head, one
# M-tile pair per block), G = 3 (32 x 3 = 96 rows), G = 16 (8 x 16 = 128 rows,
# eight pairs per block), and G = 2 at block 64 (32 x 2).
GROUP_CASES = [
    ("qwen30b_128k", 2600, {"hq": 4}),
    ("qwen30b_128k", 2600, {"hq": 6, "hkv": 2}),
    ("qwen30b_128k", 2600, {"hkv": 2}),
    ("tiny2k", 1500, {"hq": 2}),
]


@pytest.mark.parametrize("name,L,kw", GROUP_CASES)
@pytest.mark.parametrize("fp8", [False, True])
def test_attention_group_shapes(name, L, kw, fp8):
    w = _case(name, L, **kw)
    inp = _inputs(w, fp8)
    dev = H.Device(w, inp)
    orc = H.oracle_discovery(w, inp)
    idx, cnt = H.upload_lists(dev.cfg, [o["lists"] for o in orc])
    dev.attend(idx, cnt)
    assert dev.status() == 0
    H.check_attention(dev, H.oracle_attention(w, inp, orc), fp8)


@pytest.mark.parametrize("fp8", [False, True])
def test_full_path_tiny(fp8):
    """Discovery -> compaction -> attention on the GPU; lists equal the oracle's."""
    w = _case("tiny2k")
    inp = _inputs(w, fp8)
    dev = H.Device(w, inp)
    dev.discover()
    orc = H.oracle_discovery(w, inp)
    assert H.compare_lists(orc, dev.lists()) == 0
    dev.attend()
    assert dev.status() == 0
    H.check_attention(dev, H.oracle_attention(w, inp, orc), fp8)


def test_values_ones_and_zero_queries():
    """V = 1 gives O = 1; Q = 0 gives, for every head and every channel, the mean
    of the group's V over the keys up to the query (alpha = 0)."""
    w = _case("qwen30b_128k", 1000)
    inp = _inputs(w)
    inp.v = torch.ones_like(inp.v)
    dev = H.Device(w, inp, 0.0)
    dev.discover()
    dev.attend()
    o = dev.bufs.o.float()
    assert (o - 1).abs().max().item() <= 1e-2
    inp2 = _inputs(w)
    inp2.q = torch.zeros_like(inp2.q)
    dev2 = H.Device(w, inp2, 0.0)
    dev2.discover()
    dev2.attend()
    n = torch.arange(1, inp2.v.shape[1] + 1, dtype=torch.float64)[:, None]
    got = dev2.bufs.o[0].double().cpu()
    worst = 0.0
    for g in range(w.hkv):
        ref = torch.cumsum(inp2.v[0, :, g].double(), 0) / n  # [L, d]
        for h in range(g * w.group, (g + 1) * w.group):
            e = (got[:, h] - ref).abs()
            worst = max(worst, e.max().item())
            assert e.max().item() <= 2e-2 and e.mean().item() <= 2e-3, (h, e.max().item())
    print("Q = 0 closed form, all heads: max abs", worst)


def test_empty_rows_give_zero_output():
    w = _case("qwen30b_128k", 512)
    inp = _inputs(w)
    dev = H.Device(w, inp)
    N = dev.cfg.nmax
    lists = [[[list(range(i + 1)) if i != 2 else [] for i in range(N)] for _ in range(w.hkv)]]
    idx, cnt = H.upload_lists(dev.cfg, lists)
    dev.attend(idx, cnt)
    o = dev.bufs.o[0].float()
    assert o[256:384].abs().max().item() == 0.0
    assert torch.isinf(dev.bufs.lse[:, 256:384]).all()
    assert torch.isfinite(o).all()


# ----------------------------------------------------------------------------- paged / varlen
@pytest.mark.parametrize("fp8", [False, True])
def test_paged_varlen_matches_oracle(fp8):
    w = W["paged_varlen"].with_(seqlens=(700, 1290, 64, 2048))
    inp = _inputs(w, fp8)
    dev = H.Device(w, inp)
    dev.discover()
    assert dev.status() == 0
    orc = H.oracle_discovery(w, inp)
    H.compare_lists(orc, dev.lists())
    dev.attend()
    assert dev.status() == 0
    H.check_attention(dev, H.oracle_attention(w, inp, orc), fp8)


def test_paged_identity_table_equals_permuted():
    """Permuting the pool and the table together leaves every output bit unchanged."""
    w = W["paged_varlen"].with_(seqlens=(1000, 333, 1500))
    inp = _inputs(w)
    dev = H.Device(w, inp)
    dev.discover()
    dev.attend()
    o1, l1 = dev.bufs.o.clone(), dev.bufs.lse.clone()
    n = inp.k_pool.shape[0]
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(9))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(n)
    inp2 = wl.Inputs(w, inp.q, cu_seqlens=inp.cu_seqlens, k_pool=inp.k_pool[inv], v_pool=inp.v_pool[inv],
                     page_table=torch.where(inp.page_table >= 0, perm[inp.page_table.long().clamp(min=0)].int(),
                                            inp.page_table))
    dev2 = H.Device(w, inp2)
    dev2.discover()
    dev2.attend()
    assert torch.equal(o1, dev2.bufs.o) and torch.equal(l1, dev2.bufs.lse)
    assert torch.equal(dev.bufs.cnt, dev2.bufs.cnt)


def test_single_request_paged_equals_contiguous():
    L = 1500
    wc = _case("qwen30b_128k", L)
    inc = _inputs(wc)
    dc = H.Device(wc, inc)
    dc.discover()
    dc.attend()
    wp = W["paged_varlen"].with_(seqlens=(L,), hkv=4, seed=wc.seed, seed_stride=0, heavy_frac=wc.heavy_frac,
                                  n_slash=wc.n_slash, amp_scale=wc.amp_scale)
    inpp = _inputs(wp)
    assert torch.equal(inpp.q, inc.q[0])
    dp = H.Device(wp, inpp)
    dp.discover()
    dp.attend()
    assert torch.equal(dc.bufs.cnt, dp.bufs.cnt)
    assert torch.equal(dc.bufs.o[0], dp.bufs.o)


# ----------------------------------------------------------------------------- device checks
def test_bad_page_and_list_entries_are_reported():
    w = W["paged_varlen"].with_(seqlens=(600, 300))
    inp = _inputs(w)
    inp.page_table = inp.page_table.clone()
    inp.page_table[0, 3] = 10_000  # outside the pool
    dev = H.Device(w, inp)
    dev.discover()
    assert dev.status() & 4  # FP_DEV_BAD_PAGE
    dev.attend()
    assert dev.status() & 4
    w2 = _case("qwen30b_128k", 512)
    dev2 = H.Device(w2, _inputs(w2))
    N = dev2.cfg.nmax
    lists = [[[[i + 1] if i == 1 else list(range(i + 1)) for i in range(N)] for _ in range(w2.hkv)]]
    idx, cnt = H.upload_lists(dev2.cfg, lists)
    dev2.attend(idx, cnt)
    assert dev2.status() & 8  # FP_DEV_BAD_LIST
    assert dev2.status() == 0  # cleared by the read


def test_bad_cu_seqlens_reported():
    w = W["paged_varlen"].with_(seqlens=(600, 300))
    inp = _inputs(w)
    inp.cu_seqlens = torch.tensor([0, 600, 500], dtype=torch.int32)  # decreasing
    dev = H.Device(w, inp)
    dev.discover()
    assert dev.status() & 2  # FP_DEV_BAD_SEQLENS


# ----------------------------------------------------------------------------- chunked prefill
def _chunk_oracle(w, inp):
    """Oracle result per request of a chunked input (float64 of the exact inputs)."""
    res = []
    for r, (qc, k, v, row0) in enumerate(H.chunk_requests(inp)):
        qs = inp.q_scale
        Qc = H.f64(qc, qs)
        K = H.f64(k, inp.k_scale)
        V = H.f64(v, inp.v_scale)
        res.append((oracle.flashprefill_chunk(Qc, K, V, w.block, w.alpha, w.sink_tokens, w.window_tokens), row0))
    return res


def _check_chunk_lists(dev, w, orc):
    """GPU lists of a chunked input equal the oracle's up to borderline blocks;
    returns the number of rows with a borderline difference."""
    gl = dev.lists()
    border = 0
    for r, (o, _) in enumerate(orc):
        N = o["mask"].shape[1]
        for g in range(w.hkv):
            for i in range(dev.cfg.nmax):
                want = o["lists"][g][i].tolist() if i < N else []
                if gl[r][g][i] != want:
                    qb = np.stack([x if x is not None else np.zeros_like(o["kbar"][0, :1].repeat(w.hq, 0))
                                   for x in o["qbar"]])
                    b = oracle.row_borderline(qb, o["kbar"], o["scale"], w.alpha, g, i, H.BORDER_REL)
                    assert set(gl[r][g][i]) ^ set(want) <= b, (r, g, i)
                    border += 1
    return border


def _check_chunk_attention(dev, orc, fp8, label):
    O = dev.bufs.o.double().cpu().numpy()
    L = dev.bufs.lse.double().cpu().numpy()
    errs, tot, n, lse_err = [], 0.0, 0, 0.0
    for o, row0 in orc:
        q_len = o["O"].shape[0]
        e = np.abs(O[row0: row0 + q_len] - o["O"])
        errs.append(e.max())
        tot += e.sum()
        n += e.size
        lse_err = max(lse_err, float(np.abs(L[:, row0: row0 + q_len] - o["lse"]).max()))
    mx, mean = max(errs), tot / n
    print(label, "fp8" if fp8 else "bf16", dict(max_abs=mx, mean_abs=mean, lse=lse_err))
    if fp8:
        assert mx <= H.FP8_MAX
    else:
        assert mx <= H.BF16_MAX and mean <= H.BF16_MEAN
    assert lse_err <= (2e-3 if fp8 else 5e-3)


@pytest.mark.parametrize("fp8", [False, True])
def test_chunked_prefill_matches_oracle(fp8):
    w = W["paged_varlen"]
    kv = (1500, 700, 2049, 640, 300)
    ql = (300, 700, 1000, 1, 173)  # ragged first query block, full, one query, ...
    inp = wl.make_chunked_inputs(w, kv, ql)
    if fp8:
        inp = wl.to_fp8(inp)
    dev = H.Device(w, inp)
    dev.discover()
    assert dev.status() == 0
    orc = _chunk_oracle(w, inp)
    border = _check_chunk_lists(dev, w, orc)
    print("chunked borderline rows:", border)
    dev.attend()
    assert dev.status() == 0
    _check_chunk_attention(dev, orc, fp8, "chunked")


def test_block_aligned_chunk_equals_full_prefill_on_gpu():
    """A chunk that starts on a block boundary sees the same pooled blocks as full
    prefill, so its lists and outputs are bit-identical to full prefill's."""
    w = W["paged_varlen"]
    kv, q = (1024, 1536), (512, 768)
    full = wl.make_inputs(w.with_(seqlens=kv))
    df = H.Device(w, full)
    df.discover()
    df.attend()
    ch = wl.make_chunked_inputs(w, kv, q)
    dc = H.Device(w, ch)
    dc.discover()
    dc.attend()
    assert dc.status() == 0
    lf, lc = df.lists(), dc.lists()
    for r in range(2):
        p0 = kv[r] - q[r]
        for g in range(w.hkv):
            for i in range(p0 // w.block, kv[r] // w.block):
                assert lc[r][g][i] == lf[r][g][i]
    cf = full.cu_seqlens.tolist()
    cc = ch.cu_seqlens.tolist()
    for r in range(2):
        assert torch.equal(dc.bufs.o[cc[r]:cc[r + 1]], df.bufs.o[cf[r + 1] - q[r]:cf[r + 1]])


# ----------------------------------------------------------------------------- per-head selection
@pytest.mark.parametrize("name,L,fp8", [("qwen30b_128k", 3000, False), ("qwen30b_128k", 3000, True),
                                        ("tiny2k", None, False)])
def test_per_head_selection_matches_oracle(name, L, fp8):
    w = _case(name, L)
    inp = _inputs(w, fp8)
    dev = H.Device(w, inp, per_head=True)
    dev.discover()
    assert dev.status() == 0
    orc = H.oracle_discovery(w, inp)
    H.compare_lists(orc, dev.lists())
    Sb, Wb = oracle.forced_blocks(w.sink_tokens, w.window_tokens, w.block)
    keep = [oracle.head_masks(o["qbar"], o["kbar"], o["scale"], w.alpha, Sb, Wb) for o in orc]
    want = H.head_bits_array(dev.cfg, [o["lists"] for o in orc], keep, w.group)
    got = dev.head_bits.cpu().numpy()
    gl = dev.lists()
    N = dev.cfg.nmax
    tri = N * (N + 1) // 2
    for g in range(w.hkv):
        for i in range(N):
            base = g * tri + i * (i + 1) // 2
            if gl[0][g][i] != [int(x) for x in orc[0]["lists"][g][i]]:
                continue  # borderline rows (already checked by compare_lists)
            n = len(gl[0][g][i])
            if not np.array_equal(got[base:base + n], want[base:base + n]):
                b = oracle.row_borderline(orc[0]["qbar"], orc[0]["kbar"], orc[0]["scale"], w.alpha, g, i,
                                          H.BORDER_REL)
                bad = [gl[0][g][i][k] for k in range(n) if got[base + k] != want[base + k]]
                assert set(bad) <= b, (g, i, bad)
    # attention on the oracle's lists and head bits against per-head attention
    idx, cnt = H.upload_lists(dev.cfg, [o["lists"] for o in orc])
    dev.head_bits.copy_(torch.from_numpy(want))
    dev.attend(idx, cnt)
    assert dev.status() == 0
    q, k, v = H.request_views(inp)[0]
    O, lse = oracle.per_head_attention(H.f64(q, inp.q_scale), H.f64(k, inp.k_scale), H.f64(v, inp.v_scale),
                                       keep[0], w.block, oracle.default_scale(w.head_dim))
    go = dev.bufs.o[0].double().cpu().numpy()
    e = np.abs(go - O)
    gl_ = dev.bufs.lse.double().cpu().numpy()
    print("per-head", name, "fp8" if fp8 else "bf16", dict(max_abs=e.max(), mean_abs=e.mean(),
                                                             lse=np.abs(gl_ - lse).max()))
    if fp8:
        assert e.max() <= H.FP8_MAX
    else:
        assert e.max() <= H.BF16_MAX and e.mean() <= H.BF16_MEAN
    assert np.abs(gl_ - lse).max() <= (2e-3 if fp8 else 5e-3)


def _check_head_bits(dev, w, orc):
    """Device head bits equal the oracle's per-head keep bits on every list entry
    the two lists share exactly (borderline rows are left to compare_lists)."""
    Sb, Wb = oracle.forced_blocks(w.sink_tokens, w.window_tokens, w.block)
    keep = [oracle.head_masks(o["qbar"], o["kbar"], o["scale"], w.alpha, Sb, Wb) for o in orc]
    want = H.head_bits_array(dev.cfg, [o["lists"] for o in orc], keep, w.group)
    got = dev.head_bits.cpu().numpy()
    gl = dev.lists()
    N = dev.cfg.nmax
    tri = N * (N + 1) // 2
    for g in range(w.hkv):
        for i in range(N):
            if gl[0][g][i] != [int(x) for x in orc[0]["lists"][g][i]]:
                continue
            base = g * tri + i * (i + 1) // 2
            n = len(gl[0][g][i])
            if not np.array_equal(got[base:base + n], want[base:base + n]):
                b = oracle.row_borderline(orc[0]["qbar"], orc[0]["kbar"], orc[0]["scale"], w.alpha, g, i,
                                          H.BORDER_REL)
                bad = [gl[0][g][i][k] for k in range(n) if got[base + k] != want[base + k]]
                assert set(bad) <= b, (g, i, bad)


def test_per_head_bits_span_column_tiles():
    w = _case("qwen30b_128k", 40000)
    inp = _inputs(w)
    dev = H.Device(w, inp, per_head=True)
    dev.discover()
    assert dev.status() == 0
    orc = H.oracle_discovery(w, inp)
    H.compare_lists(orc, dev.lists())
    _check_head_bits(dev, w, orc)


def test_per_head_with_every_head_selecting_equals_group_mode():
    """At alpha = 0 every head keeps every causal block: per-head mode must
    reproduce group (union) mode bit for bit."""
    w = _case("qwen30b_128k", 1500)
    inp = _inputs(w)
    d1 = H.Device(w, inp, 0.0)
    d1.discover()
    d1.attend()
    d2 = H.Device(w, inp, 0.0, per_head=True)
    d2.discover()
    d2.attend()
    assert torch.equal(d1.bufs.cnt, d2.bufs.cnt)
    assert torch.equal(d1.bufs.o, d2.bufs.o) and torch.equal(d1.bufs.lse, d2.bufs.lse)


# ----------------------------------------------------------------------------- single-call path
def _prefill_case(case):
    if case == "contig":
        w = _case("qwen30b_128k", 4000)
        return w, _inputs(w), False
    if case == "fp8":
        w = _case("qwen30b_128k", 3000)
        return w, _inputs(w, True), False
    if case == "paged":
        w = W["paged_varlen"].with_(seqlens=(900, 2100, 64))
        return w, _inputs(w), False
    if case == "chunked":
        w = W["paged_varlen"]
        return w, wl.make_chunked_inputs(w, (1500, 700), (600, 700)), False
    w = _case("tiny2k")
    return w, _inputs(w), True


@pytest.mark.parametrize("case", ["contig", "fp8", "paged", "chunked", "per_head"])
def test_prefill_single_call_equals_separate_calls(case):
    """fp_prefill (device work queue, dependent launch) gives exactly the outputs
    of fp_discover_compact followed by the attention call."""
    from block_sparse_long_blocks_b200 import binding as fb
    w, inp, per_head = _prefill_case(case)
    a = H.Device(w, inp, per_head=per_head)
    a.discover()
    a.attend()
    b = H.Device(w, inp, per_head=per_head)
    b.bufs.o.zero_()
    b.bufs.lse.fill_(float("nan"))
    fb.fp_prefill(b.p, b.q, b.k, b.v, b.bufs.mask, b.bufs.idx, b.bufs.cnt, b.bufs.o, b.bufs.workspace, b.bufs.lse)
    torch.cuda.synchronize()
    assert b.status() == 0
    assert torch.equal(a.bufs.cnt, b.bufs.cnt) and torch.equal(a.bufs.mask, b.bufs.mask)
    assert a.lists() == b.lists()
    if per_head:
        assert torch.equal(a.head_bits, b.head_bits)
    assert torch.equal(a.bufs.o, b.bufs.o)
    assert torch.equal(torch.nan_to_num(a.bufs.lse, nan=7.0), torch.nan_to_num(b.bufs.lse, nan=7.0))


def _run_prefill(w, inp, per_head):
    from block_sparse_long_blocks_b200 import binding as fb
    d = H.Device(w, inp, per_head=per_head)
    d.bufs.o.zero_()
    d.bufs.lse.fill_(float("nan"))
    fb.fp_prefill(d.p, d.q, d.k, d.v, d.bufs.mask, d.bufs.idx, d.bufs.cnt, d.bufs.o, d.bufs.workspace, d.bufs.lse)
    torch.cuda.synchronize()
    assert d.status() == 0
    return d


def _keep_from_gpu(dev, w):
    """Per-head selection [Hq, N, N] that the GPU's lists and head bits encode
    (request 0), for the oracle's per-head attention."""
    gl = dev.lists()[0]
    bits = dev.head_bits.cpu().numpy()
    N = dev.cfg.nmax
    tri = N * (N + 1) // 2
    keep = np.zeros((w.hq, N, N), dtype=bool)
    for g in range(w.hkv):
        for i in range(N):
            base = g * tri + i * (i + 1) // 2
            for n, j in enumerate(gl[g][i]):
                for hh in range(w.group):
                    keep[g * w.group + hh, i, j] = bool((bits[base + n] >> hh) & 1)
    return keep


@pytest.mark.parametrize("case", ["contig", "fp8", "paged", "chunked", "per_head"])
def test_prefill_single_call_matches_oracle(case):
    """fp_prefill (discovery, compaction, claim-order sort and attention in one
    call) against the float64 oracle: lists bit-exact up to borderline blocks,
    outputs within the bars. The oracle's attention runs on the lists the GPU
    chose (each already checked against the oracle's own), so a borderline
    block decided the other way cannot fail the output check."""
    w, inp, per_head = _prefill_case(case)
    fp8 = inp.dtype == "e4m3"
    d = _run_prefill(w, inp, per_head)
    if case == "chunked":
        orc = _chunk_oracle(w, inp)
        assert _check_chunk_lists(d, w, orc) == 0  # no borderline rows in this case: same lists
        _check_chunk_attention(d, orc, fp8, "fp_prefill chunked")
        return
    orc = H.oracle_discovery(w, inp)
    rep = {}
    H.compare_lists(orc, d.lists(), rep)
    gl = d.lists()
    for r, o in enumerate(orc):
        o["lists"] = [[np.asarray(gl[r][g][i], dtype=np.int64) for i in range(len(o["lists"][g]))]
                      for g in range(w.hkv)]
    if per_head:
        _check_head_bits(d, w, H.oracle_discovery(w, inp))
        q, k, v = H.request_views(inp)[0]
        O, lse = oracle.per_head_attention(H.f64(q, inp.q_scale), H.f64(k, inp.k_scale), H.f64(v, inp.v_scale),
                                           _keep_from_gpu(d, w), w.block, oracle.default_scale(w.head_dim))
        e = np.abs(d.bufs.o[0].double().cpu().numpy() - O)
        le = np.abs(d.bufs.lse.double().cpu().numpy() - lse).max()
        print("fp_prefill per-head", dict(max_abs=e.max(), mean_abs=e.mean(), lse=le, **rep))
        assert e.max() <= H.BF16_MAX and e.mean() <= H.BF16_MEAN and le <= 5e-3
        return
    H.check_attention(d, H.oracle_attention(w, inp, orc), fp8, rep)
    print("fp_prefill", case, rep)
