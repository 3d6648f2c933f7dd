"""GPU parity at the workloads' stated sizes (through the C ABI, against the float64 oracle).

* 32K prefill, Qwen2.5-7B-like attention (Hq=28, Hkv=4, block 128) at alpha in
  {0, 0.05, 0.2}: full-length kept-block lists; at alpha = 0 every causal block
  is kept and the attention equals dense causal attention (written out here,
  independently of the oracle) on sampled query blocks.
* 256K extreme-sparsity prefill (Hq=32, Hkv=4, alpha 0.3): all 2048 x 4 lists,
  the long-list case of index compaction; attention on sampled query blocks.
* Paged KV + continuous batching, 8 requests of 4K-64K tokens (Hq=32, Hkv=8,
  page 64), bf16 and e4m3: every request's full lists; attention on sampled
  query blocks of every request.
* 128K prefill (Hq=32, Hkv=4), bf16 and e4m3: full lists, attention on every
  KV group of the first, middle, last and densest query blocks plus random rows.

Lists must be bit-exact except blocks whose exact probability lies within
1e-5 relative of alpha; attention runs on the oracle's own lists with the
bars BF16 max |err| <= 2e-2, mean <= 2e-3; FP8 max <= 6e-2.
"""
import numpy as np
import pytest
import torch

from block_sparse_long_blocks_b200 import workloads as wl
from tests import _helpers as H

pytestmark = pytest.mark.gpu

W = wl.workloads()


def sample_rows(orc, w, r=0, k=6, seed=0):
    """(r, g, i) rows to check: every KV group of the first, middle, last and
    densest query blocks of request r, plus k random (group, block) rows."""
    N = orc[r]["mask"].shape[1]
    dens = orc[r]["cnt"].sum(axis=0)
    rng = np.random.default_rng(seed + r)
    key = {0, N - 1, N // 2, int(np.argmax(dens))}
    rows = {(r, g, i) for i in key for g in range(w.hkv)}
    for i in rng.integers(0, N, k).tolist():
        rows.add((r, int(rng.integers(0, w.hkv)), int(i)))
    return rows


def run_full(w, inp, alpha=None, fp8=False, rows_per_request=6):
    """Discovery on the GPU vs the oracle (all rows), then the attention on the
    oracle's lists vs the oracle on sampled rows of every request."""
    dev = H.Device(w, inp, alpha)
    dev.discover()
    assert dev.status() == 0
    orc = H.oracle_discovery(w, inp, alpha)
    rep = {}
    H.compare_lists(orc, dev.lists(), rep)
    gpu_lists = dev.lists()
    idx, cnt = H.upload_lists(dev.cfg, [o["lists"] for o in orc])
    dev.attend(idx, cnt)
    assert dev.status() == 0
    rows = set()
    for r in range(len(orc)):
        rows |= sample_rows(orc, w, r, rows_per_request)
    H.check_attention(dev, H.oracle_attention(w, inp, orc, rows), fp8, rep)
    rep["rows_checked"] = len(rows)
    rep["kept_blocks"] = int(sum(int(o["cnt"].sum()) for o in orc))
    return dev, orc, gpu_lists, rows, rep


def dense_causal_rows(inp, g, i, B, G, scale):
    """Dense causal attention (every key <= query) for the query tokens of block
    i and the heads of group g, in float64: softmax(scale * q K^T) V."""
    q, k, v = inp.q[0], inp.k[0], inp.v[0]
    lo, hi = i * B, min((i + 1) * B, q.shape[0])
    K = k[:hi, g].double()
    V = v[:hi, g].double()
    t = torch.arange(lo, hi)[:, None]
    allowed = torch.arange(hi)[None, :] <= t
    out = {}
    for h in range(g * G, (g + 1) * G):
        logits = scale * (q[lo:hi, h].double() @ K.T)
        logits = logits.masked_fill(~allowed, float("-inf"))
        out[h] = torch.softmax(logits, dim=1) @ V
    return out


@pytest.mark.parametrize("alpha", [0.0, 0.05, 0.2])
def test_qwen7b_32k_at_full_length(alpha):
    w = W["qwen7b_32k"]
    inp = wl.make_inputs(w)
    dev, orc, gl, rows, rep = run_full(w, inp, alpha)
    print(f"32K alpha={alpha}:", rep)
    if alpha == 0.0:
        N = dev.cfg.nmax
        for g in range(w.hkv):
            for i in range(N):
                assert gl[0][g][i] == list(range(i + 1)), (g, i)
        # the sampled rows against dense causal attention written out directly
        scale = 1.0 / np.sqrt(w.head_dim)
        worst = 0.0
        for (_, g, i) in sorted(rows):
            ref = dense_causal_rows(inp, g, i, w.block, w.group, scale)
            for h, o in ref.items():
                got, _ = H.gpu_rows(dev, 0, i, h)
                e = np.abs(got - o.numpy())
                worst = max(worst, float(e.max()))
                assert e.max() <= H.BF16_MAX and e.mean() <= H.BF16_MEAN, (g, i, h, e.max(), e.mean())
        print("32K alpha=0 vs dense causal: max abs", worst)


def test_extreme_256k_at_full_length():
    w = W["extreme_256k"]
    inp = wl.make_inputs(w)
    dev, orc, gl, rows, rep = run_full(w, inp)
    longest = max(len(x) for g in gl[0] for x in g)
    rep["longest_list"] = longest
    print("256K:", rep)
    assert longest > 64  # the long-list case the workload exists for


@pytest.mark.parametrize("fp8", [False, True])
def test_paged_varlen_eight_requests_at_full_length(fp8):
    w = W["paged_varlen"]
    assert len(w.seqlens) == 8 and min(w.seqlens) >= 4096 and max(w.seqlens) <= 65536
    inp = wl.make_inputs(w)
    if fp8:
        inp = wl.to_fp8(inp)
    dev, orc, gl, rows, rep = run_full(w, inp, fp8=fp8, rows_per_request=3)
    print("paged varlen", "e4m3" if fp8 else "bf16", rep)
    assert {r for (r, _, _) in rows} == set(range(8))


@pytest.mark.parametrize("fp8", [False, True])
def test_qwen30b_128k_at_full_length(fp8):
    w = W["qwen30b_128k"]
    inp = wl.make_inputs(w)
    if fp8:
        inp = wl.to_fp8(inp)
    dev, orc, gl, rows, rep = run_full(w, inp, fp8=fp8)
    print("128K", "e4m3" if fp8 else "bf16", rep)
