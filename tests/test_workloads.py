"""Host-side checks of the seeded input generator (no GPU)."""
import numpy as np
import torch

from block_sparse_long_blocks_b200 import workloads as wl


def test_registry_shapes():
    w = wl.workloads()
    assert set(w) == {"tiny2k", "qwen7b_32k", "qwen30b_128k", "extreme_256k", "paged_varlen"}
    assert w["tiny2k"].group == 4 and w["qwen7b_32k"].group == 7 and w["qwen30b_128k"].group == 8
    pv = w["paged_varlen"]
    assert len(pv.seqlens) == 8 and all(4096 <= L <= 65536 for L in pv.seqlens)
    assert pv.paged and pv.page_size == 64 and pv.group == 4


def test_generation_is_deterministic_and_structured():
    w = wl.small_case(wl.workloads()["qwen30b_128k"], 1024)
    a = wl.make_inputs(w)
    b = wl.make_inputs(w)
    assert torch.equal(a.q, b.q) and torch.equal(a.k, b.k) and torch.equal(a.v, b.v)
    assert a.q.shape == (1, 1024, 32, 128) and a.k.shape == (1, 1024, 4, 128)
    assert a.q.dtype == torch.bfloat16
    heavy = a.plants[0]["heavy_blocks"]
    assert len(heavy) == 1  # 1% of 8 blocks rounds up to one
    # without slash terms, the heavy key block carries the shared direction and
    # its pooled norm stands out
    c = wl.make_inputs(w.with_(n_slash=0))
    kb = c.k[0, :, 0].float().view(8, 128, 128).mean(1).norm(dim=-1)
    assert int(kb.argmax()) == c.plants[0]["heavy_blocks"][0]


def test_paged_layout_roundtrip():
    w = wl.workloads()["paged_varlen"].with_(seqlens=(300, 129, 64))
    inp = wl.make_inputs(w)
    P = w.page_size
    cu = inp.cu_seqlens.tolist()
    assert cu == [0, 300, 429, 493]
    used = inp.page_table[inp.page_table >= 0].tolist()
    assert sorted(used) == list(range(inp.k_pool.shape[0]))  # a permutation of the pool
    ref = wl.make_inputs(w.with_(paged=False, seqlens=(300,)))
    for t in range(300):
        pg = int(inp.page_table[0, t // P])
        assert torch.equal(inp.k_pool[pg, t % P], ref.k[0, t])
    assert torch.equal(inp.q[:300], ref.q[0])


def test_fp8_quantisation_bounds():
    w = wl.small_case(wl.workloads()["qwen30b_128k"], 256)
    inp = wl.make_inputs(w)
    f8 = wl.to_fp8(inp)
    assert f8.q.dtype == torch.float8_e4m3fn and f8.q_scale.shape == (32,)
    x = f8.q.float()
    assert torch.isfinite(x).all() and x.abs().max() <= 448
    deq = wl.dequantize(f8.q, f8.q_scale)
    err = (deq - inp.q.double()).abs().max().item()
    assert err <= 0.07 * inp.q.float().abs().max().item()
    # the per-head absmax lands exactly on the e4m3 maximum
    amax = x.abs().amax(dim=(0, 1, 3))
    assert torch.all(amax == 448)


def test_chunked_inputs_take_the_last_tokens_as_queries():
    w = wl.workloads()["paged_varlen"]
    ch = wl.make_chunked_inputs(w, kv_lens=(300, 200), q_lens=(100, 200))
    full = wl.make_inputs(w.with_(seqlens=(300, 200)))
    assert ch.cu_seqlens.tolist() == [0, 100, 300]
    assert ch.kv_lens.tolist() == [300, 200]
    assert torch.equal(ch.q[:100], full.q[200:300])
    assert torch.equal(ch.q[100:], full.q[300:500])
    assert torch.equal(ch.k_pool, full.k_pool) and torch.equal(ch.page_table, full.page_table)
