#!/usr/bin/env python
"""Benchmark of the block-sparse prefill hot path on B200.

One step = one layer of the workload through the whole path: block pattern
discovery + index compaction (fused launch) and block-sparse attention, on
inputs already resident in HBM. Default workload: 128K-token prefill with
Qwen3-30B-A3B-like attention (Hq=32, Hkv=4, d=128, block 128, alpha 0.1,
sink 256, window 512, ~5% of causal blocks kept), bf16.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                       [--workload NAME] [--dtype bf16|e4m3]
Multi-GPU (weak scaling, every rank runs its own layer, no data-path collective):
  python -m torch.distributed.run --nproc-per-node N --master-addr 127.0.0.1 bench.py --gpus N

Prints one JSON line (rank 0). value = dense-equivalent TFLOP/s of the step
(4*d*Hq*sum L(L+1)/2 per layer) over all ranks; ms_per_step = ms per layer.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from block_sparse_long_blocks_b200 import workloads as wl  # noqa: E402

METRIC = "sparse prefill attn ms/layer & dense-equiv TFLOPS @128K; % of TC peak"
UNIT = "TFLOPS (dense-equivalent)"
FP8_OVER_BF16 = 2.0  # nominal dense fp8 / bf16 tensor-core ratio (4.5 / 2.25 PFLOP/s)


def recorded_traffic(workload: str, dtype: str):
    """DRAM bytes per attention launch from the committed ncu record, if it was taken
    on the current kernel sources (else None)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)
        h = hashlib.sha256()
        for src in rec["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != rec["source_sha256"]:
            return None
        e = rec["entries"].get(f"{workload}/{dtype}")
        return None if e is None else e["dram_read_bytes"] + e["dram_write_bytes"]
    except (OSError, KeyError, ValueError):
        return None


def blas_threads() -> int:
    """Threads the oracle's numpy BLAS uses (what the CPU baseline actually ran on)."""
    try:
        from threadpoolctl import threadpool_info
        n = [d["num_threads"] for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


FP8_PEAK_PATH = os.path.join(ROOT, "profiles", "fp8_peak.json")


def peaks():
    """Roofline denominators: HBM copy bandwidth and dense bf16 tensor throughput
    from MEASURED_PEAKS.json; dense e4m3 (and f16) tensor throughput from
    profiles/fp8_peak.json (measured by ``--measure-peaks``), else None."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        out = dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                   bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), source="measured")
    except (OSError, KeyError, ValueError):
        out = dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")
    out["fp8"] = out["f16"] = None
    try:
        with open(FP8_PEAK_PATH) as f:
            d = json.load(f)
        out["fp8"] = float(d["e4m3_tflops"])
        out["f16"] = float(d["f16_tflops"])
    except (OSError, KeyError, ValueError):
        pass
    return out


def measure_peaks(seconds: float = 4.0):
    """Dense tensor-core throughput on this GPU, measured like the bf16 figure of
    MEASURED_PEAKS.json: an 8192^3 product, best of 10 (CUDA events), for e4m3
    (torch._scaled_mm, bf16 output, unit scales) and f16 (torch.matmul); the e4m3
    one also back to back for a few seconds (sustained). Writes profiles/fp8_peak.json."""
    n = 8192
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(0)
    a16 = torch.randn(n, n, device=dev, generator=g, dtype=torch.float16)
    b16 = torch.randn(n, n, device=dev, generator=g, dtype=torch.float16)
    a8 = a16.to(torch.float8_e4m3fn)
    b8 = b16.to(torch.float8_e4m3fn).t().contiguous().t()  # column-major second operand
    one = torch.ones((), device=dev, dtype=torch.float32)
    fp8 = lambda: torch._scaled_mm(a8, b8, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)  # noqa: E731
    f16 = lambda: torch.matmul(a16, b16)  # noqa: E731

    def best(fn, reps=10):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return 2.0 * n ** 3 / (min(ts) * 1e-3) / 1e12

    def sustained(fn):
        clocks = ClockSampler(torch.cuda.current_device())
        clocks.start()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        k, t0 = 0, time.time()
        e0.record()
        while time.time() - t0 < seconds:
            for _ in range(20):
                fn()
            k += 20
            torch.cuda.synchronize()
        e1.record()
        torch.cuda.synchronize()
        clk = clocks.stop()
        return 2.0 * n ** 3 * k / (e0.elapsed_time(e1) * 1e-3) / 1e12, clk

    fp8_best, f16_best = best(fp8), best(f16)
    fp8_sus, clk = sustained(fp8)
    rec = {"e4m3_tflops": fp8_best, "e4m3_tflops_sustained": fp8_sus, "f16_tflops": f16_best,
           "gpu_name": torch.cuda.get_device_name(), "torch": torch.__version__,
           "when": time.strftime("%Y-%m-%dT%H:%M:%SZ", time.gmtime()),
           "how": "8192^3 products (2*N^3 flops): torch._scaled_mm e4m3 x e4m3 -> bf16 with unit scales and "
                  "torch.matmul f16, best of 10 with CUDA events; e4m3 also back to back for a few seconds "
                  "(sustained)",
           "clocks_sustained": clk}
    os.makedirs(os.path.dirname(FP8_PEAK_PATH), exist_ok=True)
    with open(FP8_PEAK_PATH, "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")
    print(json.dumps(rec), flush=True)


def fp8_peaks(pk):
    """Tensor-core bounds of the e4m3 attention: every visited flop at the dense
    e4m3 rate ("fp8"), and the kernel's own mix ("design"): S = Q K^T (half the
    flops) on e4m3 operands, O += P V (the other half) on 16-bit f16 operands,
    whose dense rate is the bf16/f16 one (the larger of the two measured)."""
    p8 = pk["fp8"] if pk["fp8"] else pk["bf16"] * FP8_OVER_BF16
    p16 = max(pk["bf16"], pk["f16"] or 0.0)
    return {"fp8": p8, "fp8_source": "measured e4m3 burst" if pk["fp8"] else "bf16 measured x2 (nominal ratio)",
            "design": 2.0 / (1.0 / p8 + 1.0 / p16), "f16": p16}


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        try:
            props = torch.cuda.get_device_properties(device_index)
            self.sel = "GPU-" + str(props.uuid)
        except Exception:
            self.sel = str(device_index)

    @staticmethod
    def _rows(path):
        rows = []
        with open(path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        return rows

    def start(self):
        """Starts sampling every 100 ms and returns once the first sample is in
        (nvidia-smi takes a moment to start), so the timed region is covered."""
        self.skip = 0
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
            return
        t0 = time.time()
        while time.time() - t0 < 5.0 and self.proc.poll() is None:
            n = len(self._rows(self.path))
            if n:
                self.skip = n  # samples taken before the timed region
                return
            time.sleep(0.02)

    def stop(self):
        """Samples taken from the start of the timed region (at least one)."""
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = self._rows(self.path)
        os.unlink(self.path)
        rows = rows[self.skip:] if len(rows) > self.skip else rows[-1:]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- oracle baseline
def oracle_sample(w: wl.Workload, inp: wl.Inputs, budget_s: float, max_rows: int, seed: int = 0):
    """Time the CPU oracle on a bounded sample of (KV group, query block) rows of
    the first request and extrapolate to the whole layer by work counts."""
    import oracle
    from tests import _helpers as H

    q, k, v = H.request_views(inp)[0]
    B, G = w.block, w.group
    scale = oracle.default_scale(w.head_dim)
    Sb, Wb = oracle.forced_blocks(w.sink_tokens, w.window_tokens, B)
    L = q.shape[0]
    N = -(-L // B)
    t0 = time.perf_counter()
    kbar = H.pooled_f64(k, B, inp.k_scale)  # all key blocks (every row needs them)
    t_kpool = time.perf_counter() - t0
    Qv, Kv, Vv = H.Lazy64(q, inp.q_scale), H.Lazy64(k, inp.k_scale), H.Lazy64(v, inp.v_scale)
    rng = np.random.default_rng(seed)
    order = rng.permutation(N * w.hkv)
    t_disc = t_attn = 0.0
    rows = 0
    score_work = 0        # sum over sampled rows of (i + 1)
    visits = 0
    for u in order[:max_rows]:
        g, i = int(u % w.hkv), int(u // w.hkv)
        t1 = time.perf_counter()
        lo, hi = i * B, min((i + 1) * B, L)
        qs = None if inp.q_scale is None else inp.q_scale[g * G:(g + 1) * G]
        qbar_i = oracle.pool_blocks(H.f64(q[lo:hi, g * G:(g + 1) * G], qs), B)[0]
        lst = oracle.discover_row(qbar_i, kbar[:, g], i, scale, w.alpha, Sb, Wb)
        t2 = time.perf_counter()
        oracle.attention_rows(Qv, Kv, Vv, g, i, lst, B, scale)
        t3 = time.perf_counter()
        t_disc += t2 - t1
        t_attn += t3 - t2
        rows += 1
        score_work += i + 1
        visits += len(lst)
        if t_kpool + t_disc + t_attn > budget_s:
            break
    return dict(t_kpool=t_kpool, t_disc=t_disc, t_attn=t_attn, rows=rows, score_work=score_work,
                visits=visits, N=N, wall=t_kpool + t_disc + t_attn)


def extrapolate(s: dict, w: wl.Workload, total_visits: int) -> float:
    """Seconds the oracle would take for the whole layer, from a sample's rates."""
    N, rows = s["N"], max(1, s["rows"])
    total_rows = N * w.hkv
    total_score = w.hkv * N * (N + 1) / 2
    # discovery per row = q-block pooling (constant) + scoring (proportional to i + 1)
    disc = s["t_disc"] * 0.5 * (total_rows / rows + total_score / max(1, s["score_work"]))
    attn = s["t_attn"] * total_visits / max(1, s["visits"])
    return s["t_kpool"] + disc + attn


# ----------------------------------------------------------------------------- multi-rank
def max_over_ranks(values, dist, device):
    """Element-wise max of per-rank timings (the job is as slow as its slowest rank)."""
    if dist is None:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def weak_value(world: int, flops_per_rank: float, ms: float) -> float:
    """Whole-job throughput in TFLOP/s when every rank processes its own layer."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="qwen30b_128k")
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "e4m3"])
    ap.add_argument("--path", default="fused", choices=["fused", "unfused", "single"],
                    help="fused: fp_discover_compact + attention (default); unfused: fp_discover + fp_compact + "
                         "attention; single: fp_prefill (one call, device work queue)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-fp8-extra", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the 256K / paged / chunked measurements")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--measure-peaks", action="store_true",
                    help="measure the dense e4m3 / f16 tensor-core peaks and write profiles/fp8_peak.json")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="run a shorter sequence of the same workload (profiling small cases)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "native":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)

    if args.measure_peaks:
        measure_peaks()
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist_mod
        dist = dist_mod
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))

    w = wl.workloads()[args.workload]
    if args.seq_len:
        w = wl.small_case(w, args.seq_len)
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, w, world)
        if dist is not None:
            dist.destroy_process_group()
        return
    line = run_native(args, w, world, rank, local, dist)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args, w, world):
    inp = wl.make_inputs(w)
    if args.dtype == "e4m3":
        inp = wl.to_fp8(inp)
    # the oracle's own lists give the visited-block count used for extrapolation
    from tests import _helpers as H
    orc = H.oracle_discovery(w, inp)
    total_visits = int(sum(int(o["cnt"].sum()) for o in orc))
    times, walls = [], []
    per_step_budget = max(2.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    last = None
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        smp = oracle_sample(w, inp, per_step_budget, max_rows=64, seed=s)
        if s >= args.warmup:
            walls.append(time.perf_counter() - t0)
            times.append(extrapolate(smp, w, total_visits))
        last = smp
    t = statistics.mean(times)
    flops = w.dense_equiv_flops()
    val = flops / t / 1e12
    # ms_per_step is what each step took on this machine's clock: a bounded
    # sample of the layer; the whole layer's time is extrapolated from it.
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(walls) * 1e3,
            "extrapolated_ms_per_layer": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "seq_len": w.seqlens[0], "hq": w.hq, "hkv": w.hkv, "block": w.block,
                       "alpha": w.alpha, "input_dtype": args.dtype},
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": f"per step {last['rows']} (KV group, query block) rows of the layer "
                                       f"(discovery + attention) plus full key pooling, timed "
                                       f"({statistics.mean(walls):.1f} s per step) and extrapolated by work "
                                       f"counts to all {last['N'] * w.hkv} rows / {total_visits} visited blocks "
                                       f"(value = dense-equivalent flops / extrapolated_ms_per_layer)"},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_native(args, w, world, rank, local, dist):
    from block_sparse_long_blocks_b200 import binding as fb

    fb.load()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pk = peaks()
    inp_host = wl.make_inputs(w)
    fp8 = args.dtype == "e4m3"
    if fp8:
        inp_host = wl.to_fp8(inp_host)

    def setup(inp, per_head=False):
        cfg = fb.config_for(inp.workload, inp)
        t = lambda x: None if x is None else x.to(dev).contiguous()  # noqa: E731
        paged = inp.page_table is not None
        d = dict(q=t(inp.q), k=t(inp.k if not paged else inp.k_pool), v=t(inp.v if not paged else inp.v_pool),
                 cu=t(inp.cu_seqlens), table=t(inp.page_table), qs=t(inp.q_scale), ks=t(inp.k_scale),
                 vs=t(inp.v_scale), kv=t(getattr(inp, "kv_lens", None)), paged=paged, cfg=cfg)
        d["p"] = fb.make_params(cfg, d["qs"], d["ks"], d["vs"], d["cu"], d["table"], d["kv"])
        if per_head:  # per-query-head selection inside the PackGQA tiles
            d["hb"] = torch.zeros(fb.sizes(d["p"])["list_capacity"], dtype=torch.uint8, device=dev)
            d["p"] = fb.make_params(cfg, d["qs"], d["ks"], d["vs"], d["cu"], d["table"], d["kv"], d["hb"])
        d["bufs"] = fb.Buffers(d["p"], device=dev, o_shape=tuple(inp.q.shape))
        return d

    D = setup(inp_host)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        if args.path == "single":  # one call: discovery, claim-order sort, attention (no split)
            fb.fp_prefill(D["p"], D["q"], D["k"], D["v"], None, D["bufs"].idx, D["bufs"].cnt, D["bufs"].o,
                          D["bufs"].workspace)
            if ev is not None:
                ev[1].record(stream)
                ev[2].record(stream)
            return
        if args.path == "unfused":
            fb.fp_discover(D["p"], D["q"], D["k"], D["bufs"].mask, D["bufs"].workspace)
            fb.fp_compact(D["p"], D["bufs"].mask, D["bufs"].idx, D["bufs"].cnt)
        else:
            fb.fp_discover_compact(D["p"], D["q"], D["k"], None, D["bufs"].idx, D["bufs"].cnt, D["bufs"].workspace)
        if ev is not None:
            ev[1].record(stream)
        if D["paged"]:
            fb.fp_paged_sparse_prefill(D["p"], D["q"], D["k"], D["v"], D["bufs"].idx, D["bufs"].cnt, D["bufs"].o)
        else:
            fb.fp_sparse_prefill(D["p"], D["q"], D["k"], D["v"], D["bufs"].idx, D["bufs"].cnt, D["bufs"].o)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = fb.fp_get_device_status()
    if status:
        raise RuntimeError(f"device status {status:#x} after warm-up")

    # timed region (inputs > L2: Q alone is 1 GiB, so no flush between steps)
    clocks = ClockSampler(local)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    start.record(stream)
    for s in range(args.steps):
        step(evs[s])
    end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if dist is not None:
        dist.barrier()
    ms = start.elapsed_time(end)
    disc_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    attn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    if args.path == "single":  # no event between the kernels of one call: the step is the attention's bound
        disc_ms, attn_ms = float("nan"), statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    ms, disc_ms, attn_ms = max_over_ranks([ms, disc_ms, attn_ms], dist, dev)
    ms_step = ms / args.steps

    # work counts from the lists of the last step
    cfg = D["cfg"]
    cnt = D["bufs"].cnt.long()
    visits = int(cnt.sum().item())
    B, d, G = w.block, w.head_dim, w.group
    visited_flops = visits * 4.0 * B * B * d * G
    dense = w.dense_equiv_flops()
    causal_pairs = w.hkv * sum((-(-L // B)) * ((-(-L // B)) + 1) // 2 for L in w.seqlens)
    es = 1 if fp8 else 2
    qk_bytes = (inp_host.q.numel() + (inp_host.k.numel() if inp_host.k is not None else inp_host.k_pool.numel())) * es
    disc_bytes = qk_bytes + 4 * visits + 4 * cnt.numel()
    fpk = fp8_peaks(pk)
    peak_tc = fpk["design"] if fp8 else pk["bf16"]
    achieved = visited_flops / (attn_ms * 1e-3) / 1e12
    value = weak_value(world, dense, ms_step)

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": args.dtype, "data": "synthetic (seeded Gaussian Q/K/V with heavy key "
            "blocks and slash diagonals; no model weights)",
            "config": {"workload": w.name, "seq_len": w.seqlens[0] if len(w.seqlens) == 1 else list(w.seqlens),
                       "global_batch": world * len(w.seqlens), "hq": w.hq, "hkv": w.hkv, "head_dim": d,
                       "block": B, "alpha": w.alpha, "sink_tokens": w.sink_tokens,
                       "window_tokens": w.window_tokens, "parallelism": f"replicas{world} (one layer per rank)",
                       "l2": "inputs larger than L2 (Q alone 1 GiB); no flush", "call_path": args.path,
                       "density": visits / causal_pairs},
            "ms_per_layer": ms_step, "discover_compact_ms": disc_ms, "attention_ms": attn_ms,
            "visited_tile_tflops": achieved,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_tc, "unit": "TFLOP/s",
                         "frac": achieved / peak_tc, "traffic": recorded_traffic(w.name, args.dtype),
                         "traffic_unit": "bytes per launch (ncu dram read+write)",
                         "kernel": "sparse_attention_kernel",
                         "peak_source": (f"{pk['source']} bf16 burst" if not fp8 else
                                         "QK on e4m3 at the measured e4m3 burst peak, PV on f16 at the measured "
                                         "16-bit burst peak (harmonic mean over equal flops)"),
                         **({"frac_of_fp8_peak": achieved / fpk["fp8"], "fp8_peak": fpk["fp8"]} if fp8 else {})},
            "discovery_roofline": {"bound": "hbm", "achieved": disc_bytes / (disc_ms * 1e-3) / 1e9,
                                   "peak": pk["hbm"], "unit": "GB/s",
                                   "frac": disc_bytes / (disc_ms * 1e-3) / 1e9 / pk["hbm"],
                                   "algorithmic_bytes": disc_bytes},
            "gpu_launches": (3 if args.path == "fused" else 4) * args.steps,
            "clocks": clk}

    if args.path == "single":
        line["discover_compact_ms"] = None
        line["discovery_roofline"] = None
    # end to end through the C ABI with host buffers (pinned), copies inside the timed region
    if not args.no_e2e:
        line["e2e"] = e2e(args, D, inp_host, dev, stream, dense, world, dist)
    if fp8 is False and not args.no_fp8_extra:
        line["fp8"] = fp8_extra(args, w, inp_host, dev, stream, pk, setup, dist)
    if not args.no_extras:
        del D
        torch.cuda.empty_cache()
        line["other_workloads"] = extra_workloads(args, setup, stream, pk, fp8)
        if not fp8:
            line["other_workloads"]["short_4k"] = short_context(setup, stream)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        smp = oracle_sample(w, inp_host, args.cpu_budget, max_rows=10_000)
        t = extrapolate(smp, w, visits)
        line["cpu_baseline"] = {"value": dense / t / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                                "sample": f"{smp['rows']} (KV group, query block) rows of the layer (discovery + "
                                          f"attention, {smp['wall']:.1f} s) plus full key pooling, extrapolated by "
                                          f"work counts to {smp['N'] * w.hkv} rows / {visits} visited blocks",
                                "extrapolated_s_per_layer": t}
    return line


def chunk_dense_flops(w, kv_lens, q_lens) -> float:
    """Dense causal attention flops of queries at positions kv-q..kv-1 over keys <= position."""
    tot = 0.0
    for kv, q in zip(kv_lens, q_lens):
        p0 = kv - q
        tot += (kv * (kv + 1) - p0 * (p0 + 1)) / 2
    return 4.0 * w.head_dim * w.hq * tot


def extra_workloads(args, setup, stream, pk, fp8):
    """Per-layer time of the other workload shapes (the 256K extreme-sparsity
    case, the paged/varlen batch and a chunked prefill over the same batch)."""
    from block_sparse_long_blocks_b200 import binding as fb
    W = wl.workloads()
    pv = W["paged_varlen"]
    kv = pv.seqlens
    ql = tuple(max(1, L // 4) for L in kv)
    cases = [("qwen30b_128k_per_head_selection", W["qwen30b_128k"], lambda: wl.make_inputs(W["qwen30b_128k"]),
              None),
             ("extreme_256k", W["extreme_256k"], lambda: wl.make_inputs(W["extreme_256k"]), None),
             ("paged_varlen", pv, lambda: wl.make_inputs(pv), None),
             ("chunked_prefill_last_quarter", pv, lambda: wl.make_chunked_inputs(pv, kv, ql),
              chunk_dense_flops(pv, kv, ql))]
    out = {}
    for name, w, make, dense in cases:
        inp = make()
        if fp8:
            inp = wl.to_fp8(inp)
        D = setup(inp, per_head=name.endswith("per_head_selection"))
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        disc, attn, tot = [], [], []
        for s in range(3 + 5):
            ev[0].record(stream)
            fb.fp_discover_compact(D["p"], D["q"], D["k"], None, D["bufs"].idx, D["bufs"].cnt, D["bufs"].workspace)
            ev[1].record(stream)
            if D["paged"]:
                fb.fp_paged_sparse_prefill(D["p"], D["q"], D["k"], D["v"], D["bufs"].idx, D["bufs"].cnt, D["bufs"].o)
            else:
                fb.fp_sparse_prefill(D["p"], D["q"], D["k"], D["v"], D["bufs"].idx, D["bufs"].cnt, D["bufs"].o)
            ev[2].record(stream)
            torch.cuda.synchronize()
            if s >= 3:
                disc.append(ev[0].elapsed_time(ev[1]))
                attn.append(ev[1].elapsed_time(ev[2]))
                tot.append(ev[0].elapsed_time(ev[2]))
        single = None
        if name in ("paged_varlen", "chunked_prefill_last_quarter"):
            # the same layer through fp_prefill: one call, longest lists claimed first
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            st = []
            for s in range(3 + 5):
                e0.record(stream)
                fb.fp_prefill(D["p"], D["q"], D["k"], D["v"], None, D["bufs"].idx, D["bufs"].cnt, D["bufs"].o,
                              D["bufs"].workspace)
                e1.record(stream)
                torch.cuda.synchronize()
                if s >= 3:
                    st.append(e0.elapsed_time(e1))
            single = statistics.mean(st)
        cnt = D["bufs"].cnt.long()
        visits = int(cnt.sum().item())
        flops = visits * 4.0 * w.block * w.block * w.head_dim * w.group
        a = statistics.mean(attn)
        t = statistics.mean(tot)
        dbytes = (D["q"].numel() + D["k"].numel()) * D["q"].element_size() + 4 * visits + 4 * cnt.numel()
        dm = statistics.mean(disc)
        dense = w.dense_equiv_flops() if dense is None else dense
        peak = fp8_peaks(pk)["design"] if fp8 else pk["bf16"]
        out[name] = {"ms_per_layer": t, "discover_compact_ms": dm, "attention_ms": a,
                     "discovery_frac_of_hbm": dbytes / (dm * 1e-3) / 1e9 / pk["hbm"],
                     "dense_equiv_tflops": dense / (t * 1e-3) / 1e12,
                     "visited_tile_tflops": flops / (a * 1e-3) / 1e12, "frac_of_peak": flops / (a * 1e-3) / 1e12 / peak,
                     "visited_blocks": visits, "tokens": int(inp.q.shape[0] * (inp.q.shape[1] if inp.q.dim() == 4 else 1))}
        if single is not None:
            out[name]["single_call_ms_per_layer"] = single
        del D, inp
        torch.cuda.empty_cache()
    return out


def short_context(setup, stream):
    """4K-token prefill (128K workload's shapes and generator): per-layer time of
    the separate calls, of the single fp_prefill call, and of a CUDA-graph
    replay of fp_prefill (launch overheads matter at this size)."""
    from block_sparse_long_blocks_b200 import binding as fb
    w = wl.small_case(wl.workloads()["qwen30b_128k"], 4096)
    D = setup(wl.make_inputs(w))
    b = D["bufs"]

    def separate():
        fb.fp_discover_compact(D["p"], D["q"], D["k"], None, b.idx, b.cnt, b.workspace)
        fb.fp_sparse_prefill(D["p"], D["q"], D["k"], D["v"], b.idx, b.cnt, b.o)

    def single():
        fb.fp_prefill(D["p"], D["q"], D["k"], D["v"], None, b.idx, b.cnt, b.o, b.workspace)

    def timed(fn, n=50):
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    out = {"tokens": 4096, "separate_calls_ms": timed(separate), "fp_prefill_ms": timed(single)}
    try:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            single()
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=side):
                single()
        out["fp_prefill_graph_ms"] = timed(g.replay)
    except RuntimeError as e:  # graph capture unavailable: report, do not fail the bench
        out["fp_prefill_graph_error"] = str(e)[:200]
    dense = w.dense_equiv_flops()
    out["dense_equiv_tflops_fp_prefill"] = dense / (out["fp_prefill_ms"] * 1e-3) / 1e12
    return out


def e2e(args, D, inp_host, dev, stream, dense, world, dist):
    """The metric end to end through the C ABI: every step copies its Q/K/V in
    from pinned host memory, runs discovery + compaction + attention and
    copies O back. Steps are pipelined over two device buffer sets on three
    streams (inputs of step n+1 and the output of step n-1 cross PCIe while
    step n computes), as a serving loop would; the timed region runs from the
    first input copy to the last output copy."""
    from block_sparse_long_blocks_b200 import binding as fb
    paged = D["paged"]
    hq = inp_host.q.pin_memory()
    hk = (inp_host.k if not paged else inp_host.k_pool).pin_memory()
    hv = (inp_host.v if not paged else inp_host.v_pool).pin_memory()
    ho = torch.empty(tuple(inp_host.q.shape), dtype=torch.bfloat16).pin_memory()
    h2d = hq.numel() * hq.element_size() + hk.numel() * hk.element_size() + hv.numel() * hv.element_size()
    d2h = ho.numel() * ho.element_size()
    # as many steps as the device-timed region (at least 3, at most 50): the
    # first step's copy in and the last step's copy out overlap nothing, and
    # over more steps they weigh less, as in a serving loop
    steps = max(3, min(args.steps, 50))
    sets = [dict(q=D["q"], k=D["k"], v=D["v"], o=D["bufs"].o, ws=D["bufs"].workspace, idx=D["bufs"].idx,
                 cnt=D["bufs"].cnt)]
    sets.append({n: torch.empty_like(t) for n, t in sets[0].items()})
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    h2d_done, cmp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for e in cmp_done + d2h_done:
        e.record(stream)

    def one(n):
        b = sets[n % 2]
        with torch.cuda.stream(s_in):
            s_in.wait_event(cmp_done[n % 2])  # step n-2 is done reading this set
            b["q"].copy_(hq, non_blocking=True)
            b["k"].copy_(hk, non_blocking=True)
            b["v"].copy_(hv, non_blocking=True)
            h2d_done[n % 2].record(s_in)
        stream.wait_event(h2d_done[n % 2])
        stream.wait_event(d2h_done[n % 2])  # step n-2's output has left this set
        fb.fp_discover_compact(D["p"], b["q"], b["k"], None, b["idx"], b["cnt"], b["ws"])
        if paged:
            fb.fp_paged_sparse_prefill(D["p"], b["q"], b["k"], b["v"], b["idx"], b["cnt"], b["o"])
        else:
            fb.fp_sparse_prefill(D["p"], b["q"], b["k"], b["v"], b["idx"], b["cnt"], b["o"])
        cmp_done[n % 2].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(cmp_done[n % 2])
            ho.copy_(b["o"], non_blocking=True)
            d2h_done[n % 2].record(s_out)

    one(0)
    one(1)
    torch.cuda.synchronize()

    # the parts on their own (device clocks), to show how much the pipeline overlaps
    def timed_on(st, fn, reps=3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(st)
        with torch.cuda.stream(st):
            for _ in range(reps):
                fn()
        e1.record(st)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    b0 = sets[0]
    h2d_ms = timed_on(s_in, lambda: (b0["q"].copy_(hq, non_blocking=True), b0["k"].copy_(hk, non_blocking=True),
                                     b0["v"].copy_(hv, non_blocking=True)))
    d2h_ms = timed_on(s_out, lambda: ho.copy_(b0["o"], non_blocking=True))
    b1 = sets[1]
    e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    torch.cuda.synchronize()
    e0.record(s_in)
    s_out.wait_event(e0)
    with torch.cuda.stream(s_in):
        for _ in range(3):
            b1["q"].copy_(hq, non_blocking=True)
            b1["k"].copy_(hk, non_blocking=True)
            b1["v"].copy_(hv, non_blocking=True)
    e1.record(s_in)
    with torch.cuda.stream(s_out):
        for _ in range(3):
            ho.copy_(b0["o"], non_blocking=True)
    e2.record(s_out)
    torch.cuda.synchronize()
    both_ms = max(e0.elapsed_time(e1), e0.elapsed_time(e2)) / 3
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    a.record(s_in)
    for n in range(steps):
        one(n)
    b.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks([a.elapsed_time(b) / steps], dist, dev)[0]
    return {"value": weak_value(world, dense, ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": steps,
            "pipelined": "two buffer sets, inputs / compute / output on three streams",
            "parts_ms": {"h2d_alone": h2d_ms, "d2h_alone": d2h_ms, "h2d_with_d2h_concurrent": both_ms,
                         "h2d_GBps": h2d / (h2d_ms * 1e-3) / 1e9, "d2h_GBps": d2h / (d2h_ms * 1e-3) / 1e9}}


def fp8_extra(args, w, inp_host, dev, stream, pk, setup, dist):
    """Same step with FP8-e4m3 inputs (per-head absmax scales): ms/layer and fractions."""
    from block_sparse_long_blocks_b200 import binding as fb
    inp8 = wl.to_fp8(inp_host)
    D = setup(inp8)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    disc, attn, tot = [], [], []
    for s in range(args.warmup + args.steps):
        ev[0].record(stream)
        fb.fp_discover_compact(D["p"], D["q"], D["k"], None, D["bufs"].idx, D["bufs"].cnt, D["bufs"].workspace)
        ev[1].record(stream)
        fb.fp_sparse_prefill(D["p"], D["q"], D["k"], D["v"], D["bufs"].idx, D["bufs"].cnt, D["bufs"].o)
        ev[2].record(stream)
        torch.cuda.synchronize()
        if s >= args.warmup:
            disc.append(ev[0].elapsed_time(ev[1]))
            attn.append(ev[1].elapsed_time(ev[2]))
            tot.append(ev[0].elapsed_time(ev[2]))
    visits = int(D["bufs"].cnt.long().sum().item())
    flops = visits * 4.0 * w.block * w.block * w.head_dim * w.group
    a = statistics.mean(attn)
    fpk = fp8_peaks(pk)
    es = D["q"].element_size()
    qk_bytes = (D["q"].numel() + D["k"].numel()) * es
    dbytes = qk_bytes + 4 * visits + 4 * D["bufs"].cnt.numel()
    dm = statistics.mean(disc)
    del D
    ach = flops / (a * 1e-3) / 1e12
    return {"ms_per_layer": statistics.mean(tot), "discover_compact_ms": dm, "attention_ms": a,
            "dense_equiv_tflops": w.dense_equiv_flops() / (statistics.mean(tot) * 1e-3) / 1e12,
            "visited_tile_tflops": ach,
            "frac_of_fp8_peak": ach / fpk["fp8"], "fp8_peak": fpk["fp8"], "fp8_peak_source": fpk["fp8_source"],
            "frac_of_design_peak": ach / fpk["design"], "design_peak": fpk["design"],
            "design_peak_note": "QK (half the flops) at the e4m3 peak, PV at the 16-bit peak",
            "discovery_frac_of_hbm": dbytes / (dm * 1e-3) / 1e9 / pk["hbm"]}


if __name__ == "__main__":
    main()
