"""Shared helpers of the parity tests: run the CUDA path through the C ABI and the
oracle on the same seeded inputs, and compare them by the stated bars.

Bars (from the method's contract):
* kept-block lists bit-exact, except blocks whose exact probability lies within
  1e-5 relative of alpha (reported, not failed);
* BF16 output: max |err| <= 2e-2 and mean |err| <= 2e-3 against the float64
  oracle on the oracle's own lists; FP8 output: max |err| <= 6e-2.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from block_sparse_long_blocks_b200 import binding as fb
from block_sparse_long_blocks_b200 import workloads as wl

BF16_MAX, BF16_MEAN, FP8_MAX = 2e-2, 2e-3, 6e-2
BORDER_REL = 1e-5


def f64(t: torch.Tensor, scale: torch.Tensor | None = None) -> np.ndarray:
    """Exact float64 value of a bf16 tensor, or of an e4m3 tensor times its per-head scale."""
    if scale is None:
        return t.to(torch.float64).numpy()
    return wl.dequantize(t, scale).numpy()


class Lazy64:
    """Read-only float64 view of a [L, H, d] bf16 / e4m3 tensor: indexing with
    (token indices, head) converts just those rows (dequantising e4m3 by the
    head's scale), so the oracle can take sampled rows of a long sequence."""

    def __init__(self, t: torch.Tensor, scale: torch.Tensor | None = None):
        self.t, self.scale = t, scale
        self.shape = tuple(t.shape)

    def __getitem__(self, key):
        rows, h = key
        x = self.t[torch.as_tensor(np.asarray(rows)), int(h)].to(torch.float64)
        if self.scale is not None:
            x = x * float(self.scale[int(h)])
        return x.numpy()


def pooled_f64(t: torch.Tensor, B: int, scale: torch.Tensor | None = None, chunk: int = 4) -> np.ndarray:
    """Oracle block means of a [L, H, d] tensor, a few heads at a time (bounded memory)."""
    parts = []
    for h0 in range(0, t.shape[1], chunk):
        sl = t[:, h0:h0 + chunk]
        parts.append(oracle.pool_blocks(f64(sl, None if scale is None else scale[h0:h0 + chunk]), B))
    return np.concatenate(parts, axis=1)


def config_for(w: wl.Workload, inp: wl.Inputs, alpha: float | None = None) -> fb.Config:
    return fb.config_for(w, inp, alpha)


class Device:
    """The inputs of one case on the GPU plus the library parameters."""

    def __init__(self, w: wl.Workload, inp: wl.Inputs, alpha: float | None = None, lse: bool = True,
                 per_head: bool = False):
        self.w, self.inp = w, inp
        self.cfg = config_for(w, inp, alpha)
        dev = "cuda"
        up = lambda t: None if t is None else t.to(dev).contiguous()  # noqa: E731
        self.q = up(inp.q)
        self.paged = inp.page_table is not None
        self.k = up(inp.k if not self.paged else inp.k_pool)
        self.v = up(inp.v if not self.paged else inp.v_pool)
        self.cu = up(inp.cu_seqlens)
        self.table = up(inp.page_table)
        self.qs, self.ks, self.vs = up(inp.q_scale), up(inp.k_scale), up(inp.v_scale)
        self.kv_lens = up(getattr(inp, "kv_lens", None))
        self.head_bits = None
        if per_head:
            p0 = fb.make_params(self.cfg, self.qs, self.ks, self.vs, self.cu, self.table, self.kv_lens)
            self.head_bits = torch.zeros(fb.sizes(p0)["list_capacity"], dtype=torch.uint8, device=dev)
        self.p = fb.make_params(self.cfg, self.qs, self.ks, self.vs, self.cu, self.table, self.kv_lens,
                                self.head_bits)
        T = inp.q.shape[0] * inp.q.shape[1] if inp.cu_seqlens is None else inp.q.shape[0]
        self.T = T
        self.bufs = fb.Buffers(self.p, lse_rows=T if lse else 0, o_shape=tuple(inp.q.shape), hq=self.cfg.hq)

    def discover(self, fused: bool = True):
        if fused:
            fb.fp_discover_compact(self.p, self.q, self.k, self.bufs.mask, self.bufs.idx, self.bufs.cnt,
                                   self.bufs.workspace)
        else:
            fb.fp_discover(self.p, self.q, self.k, self.bufs.mask, self.bufs.workspace)
            fb.fp_compact(self.p, self.bufs.mask, self.bufs.idx, self.bufs.cnt)
        torch.cuda.synchronize()

    def attend(self, idx=None, cnt=None):
        idx = self.bufs.idx if idx is None else idx
        cnt = self.bufs.cnt if cnt is None else cnt
        self.bufs.o.zero_()
        if self.bufs.lse is not None:
            self.bufs.lse.fill_(float("nan"))
        if self.paged:
            fb.fp_paged_sparse_prefill(self.p, self.q, self.k, self.v, idx, cnt, self.bufs.o, self.bufs.lse)
        else:
            fb.fp_sparse_prefill(self.p, self.q, self.k, self.v, idx, cnt, self.bufs.o, self.bufs.lse)
        torch.cuda.synchronize()

    def status(self) -> int:
        return fb.fp_get_device_status()

    def lists(self):
        return fb.lists_from_device(self.cfg, self.bufs.idx, self.bufs.cnt)

    def mask(self):
        return fb.mask_from_device(self.cfg, self.bufs.mask)


def request_views(inp: wl.Inputs):
    """Per-request (q, k, v) CPU tensors [L, H, d] (gathering paged K/V through the table)."""
    out = []
    if inp.cu_seqlens is None:
        for r in range(inp.q.shape[0]):
            out.append((inp.q[r], inp.k[r], inp.v[r]))
        return out
    cu = inp.cu_seqlens.tolist()
    P = inp.workload.page_size
    for r in range(len(cu) - 1):
        L = cu[r + 1] - cu[r]
        q = inp.q[cu[r]:cu[r + 1]]
        if inp.page_table is None:
            out.append((q, inp.k[cu[r]:cu[r + 1]], inp.v[cu[r]:cu[r + 1]]))
        else:
            t = torch.arange(L)
            pages = inp.page_table[r][t // P].long()
            out.append((q, inp.k_pool[pages, t % P], inp.v_pool[pages, t % P]))
    return out


def oracle_discovery(w: wl.Workload, inp: wl.Inputs, alpha: float | None = None):
    """Per request: dict(qbar, kbar, mask, lists, cnt, scale) from the oracle."""
    a = w.alpha if alpha is None else alpha
    res = []
    scale = oracle.default_scale(w.head_dim)
    Sb, Wb = oracle.forced_blocks(w.sink_tokens, w.window_tokens, w.block)
    for q, k, _ in request_views(inp):
        qbar = pooled_f64(q, w.block, inp.q_scale)
        kbar = pooled_f64(k, w.block, inp.k_scale)
        mask = oracle.block_mask(qbar, kbar, scale, a, Sb, Wb)
        lists, cnt = oracle.compact(mask)
        res.append(dict(qbar=qbar, kbar=kbar, mask=mask, lists=lists, cnt=cnt, scale=scale, alpha=a))
    return res


def compare_lists(orc, gpu_lists, report: dict | None = None):
    """Assert GPU lists equal the oracle's except for borderline blocks; return the count of those."""
    n_border = 0
    for r, o in enumerate(orc):
        for g, rows in enumerate(o["lists"]):
            for i, ol in enumerate(rows):
                gl = gpu_lists[r][g][i]
                assert gl == sorted(set(gl)), f"row {(r, g, i)} not strictly ascending: {gl}"
                if list(ol) == gl:
                    continue
                diff = set(ol.tolist()) ^ set(gl)
                border = oracle.row_borderline(o["qbar"], o["kbar"], o["scale"], o["alpha"], g, i, BORDER_REL)
                assert diff <= border, f"row {(r, g, i)}: blocks {sorted(diff - border)} differ beyond the band"
                n_border += len(diff)
    if report is not None:
        report["borderline_blocks"] = n_border
    for r in range(len(gpu_lists)):
        for g in range(len(gpu_lists[r])):
            for i in range(len(orc[r]["lists"][g]) if r < len(orc) else 0, len(gpu_lists[r][g])):
                assert gpu_lists[r][g][i] == [], f"row {(r, g, i)} past the request must be empty"
    return n_border


def upload_lists(cfg: fb.Config, per_request_lists):
    """Device idx/cnt in the library's triangular layout from lists[r][g][i]."""
    N = cfg.nmax
    tri = N * (N + 1) // 2
    idx = np.zeros(cfg.batch * cfg.hkv * tri, dtype=np.int32)
    cnt = np.zeros(cfg.batch * cfg.hkv * N, dtype=np.int32)
    for r, lists in enumerate(per_request_lists):
        for g, rows in enumerate(lists):
            for i, l in enumerate(rows):
                base = (r * cfg.hkv + g) * tri + i * (i + 1) // 2
                idx[base: base + len(l)] = np.asarray(l, dtype=np.int32)
                cnt[(r * cfg.hkv + g) * N + i] = len(l)
    return torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()


def oracle_attention(w: wl.Workload, inp: wl.Inputs, orc, rows=None):
    """Oracle O/lse per request. rows: None (all) or a set of (r, g, i) to compute only those."""
    scale = oracle.default_scale(w.head_dim)
    out = {}
    for r, (q, k, v) in enumerate(request_views(inp)):
        Q, K, V = Lazy64(q, inp.q_scale), Lazy64(k, inp.k_scale), Lazy64(v, inp.v_scale)
        N = orc[r]["mask"].shape[1]
        for g in range(w.hkv):
            for i in range(N):
                if rows is not None and (r, g, i) not in rows:
                    continue
                res = oracle.attention_rows(Q, K, V, g, i, orc[r]["lists"][g][i], w.block, scale)
                for h, (o, l) in res.items():
                    out[(r, g, i, h)] = (o, l)
    return out


def gpu_rows(dev: Device, r: int, i: int, h: int):
    """GPU O rows (float64) and lse of request r, query block i, head h."""
    B = dev.w.block
    if dev.inp.cu_seqlens is None:
        L = dev.inp.q.shape[1]
        lo, hi = i * B, min((i + 1) * B, L)
        o = dev.bufs.o[r, lo:hi, h]
        t0 = r * L
    else:
        cu = dev.inp.cu_seqlens.tolist()
        lo, hi = cu[r] + i * B, min(cu[r] + (i + 1) * B, cu[r + 1])
        o = dev.bufs.o[lo:hi, h]
        t0, lo, hi = 0, lo, hi
        lse = dev.bufs.lse[h, lo:hi] if dev.bufs.lse is not None else None
        return o.double().cpu().numpy(), None if lse is None else lse.double().cpu().numpy()
    lse = dev.bufs.lse[h, t0 + lo:t0 + hi] if dev.bufs.lse is not None else None
    return o.double().cpu().numpy(), None if lse is None else lse.double().cpu().numpy()


def check_attention(dev: Device, orc_out: dict, fp8: bool, report: dict | None = None):
    errs, means = [], []
    lse_err = 0.0
    tot, n = 0.0, 0
    for (r, g, i, h), (o, l) in orc_out.items():
        go, gl = gpu_rows(dev, r, i, h)
        e = np.abs(go - o)
        errs.append(e.max())
        tot += e.sum()
        n += e.size
        if gl is not None:
            lse_err = max(lse_err, float(np.abs(gl - l).max()))
    mx = max(errs)
    mean = tot / n
    print(f"attention {'e4m3' if fp8 else 'bf16'}: max abs {mx:.3e}, mean abs {mean:.3e}, lse {lse_err:.3e}")
    if report is not None:
        report.update(max_abs=mx, mean_abs=mean, lse_max_abs=lse_err)
    if fp8:
        assert mx <= FP8_MAX, f"fp8 max abs err {mx}"
    else:
        assert mx <= BF16_MAX, f"bf16 max abs err {mx}"
        assert mean <= BF16_MEAN, f"bf16 mean abs err {mean}"
    # bf16: lse is the log of the sum of the bf16-rounded weights (<= 2^-8 relative)
    lse_tol = 2e-3 if fp8 else 5e-3
    assert lse_err <= lse_tol, f"lse max abs err {lse_err}"
    return mx, mean


def chunk_requests(inp: wl.Inputs):
    """Per request of a chunked input: (queries [q_len, Hq, d], K [kv_len, Hkv, d],
    V, first query row) as CPU tensors."""
    cu = inp.cu_seqlens.tolist()
    P = inp.workload.page_size
    out = []
    for r, kv in enumerate(inp.kv_lens.tolist()):
        t = torch.arange(kv)
        pages = inp.page_table[r][t // P].long()
        out.append((inp.q[cu[r]:cu[r + 1]], inp.k_pool[pages, t % P], inp.v_pool[pages, t % P], cu[r]))
    return out


def head_bits_array(cfg: fb.Config, per_request_lists, per_request_masks, G: int) -> np.ndarray:
    """Per-head bits in the library's list layout from lists[r][g][i] and the
    per-head selections keep[r] [Hq, N, N]."""
    N = cfg.nmax
    tri = N * (N + 1) // 2
    out = np.zeros(cfg.batch * cfg.hkv * tri, dtype=np.uint8)
    for r, (lists, keep) in enumerate(zip(per_request_lists, per_request_masks)):
        for g, rows in enumerate(lists):
            for i, l in enumerate(rows):
                base = (r * cfg.hkv + g) * tri + i * (i + 1) // 2
                for n, j in enumerate(l):
                    out[base + n] = sum(int(keep[g * G + hh, i, j]) << hh for hh in range(G))
    return out
