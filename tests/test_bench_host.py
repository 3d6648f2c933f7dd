"""Host-side arithmetic of bench.py that needs no GPU: the CPU-baseline
extrapolation from a sampled set of rows to the whole layer."""
import bench
from block_sparse_long_blocks_b200 import workloads as wl


def test_full_sample_extrapolates_to_itself():
    w = wl.small_case(wl.workloads()["qwen30b_128k"], 4096)
    N = -(-4096 // w.block)
    rows = N * w.hkv
    s = dict(t_kpool=0.5, t_disc=2.0, t_attn=3.0, rows=rows, score_work=w.hkv * N * (N + 1) // 2,
             visits=1000, N=N, wall=5.5)
    assert abs(bench.extrapolate(s, w, total_visits=1000) - 5.5) < 1e-12


def test_extrapolation_scales_with_the_unsampled_work():
    w = wl.small_case(wl.workloads()["qwen30b_128k"], 4096)
    N = -(-4096 // w.block)
    rows = N * w.hkv
    half = dict(t_kpool=0.5, t_disc=1.0, t_attn=1.5, rows=rows // 2, score_work=w.hkv * N * (N + 1) // 4,
                visits=500, N=N, wall=3.0)
    # half the rows, half the scoring work and half the visits: twice the row work
    assert abs(bench.extrapolate(half, w, total_visits=1000) - (0.5 + 2.0 + 3.0)) < 1e-12
