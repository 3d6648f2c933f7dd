"""Seeded synthetic inputs for block-sparse causal prefill attention.

This module only draws random tensors and lays them out; it performs no step of
the method (no pooling, scoring, thresholding, compaction or attention), so the
CUDA path and the CPU oracle can both consume what it produces.

The structure it plants follows the pattern kinds that the FlashPrefill abstract
("FlashPrefill: Instantaneous Pattern Discovery and Thresholding for Ultra-Fast
Long-Context Prefilling", abstract) says the discovery step finds at once:
vertical stripes (a few "heavy" key blocks every query attends to), slash
diagonals (keys that resemble the query a fixed distance later) and the
block-sparse remainder.

Recipe for one sequence of L tokens (seeded ``torch.Generator`` on the CPU):

* ``u``: one random unit vector in R^d shared by all heads.
* ``Q = Q0 + a_q*u`` with ``Q0 ~ N(0, 1)`` per ``[L, Hq, d]``.
* ``K = K0 ~ N(0, 1)`` per ``[L, Hkv, d]``; every token of each heavy key block
  gets ``+a_h*u``; for each slash offset ``delta``,
  ``K[t, g] += a_s * Q0[t + delta, g*G]`` (``t + delta < L``), i.e. key ``t``
  resembles the Gaussian part of the query ``delta`` tokens later, which lies
  below the causal diagonal.
* ``V ~ N(0, 1)`` per ``[L, Hkv, d]``.
* All three amplitudes are multiplied by ``amp_scale``.

Tensors are produced in float32 and rounded once to bfloat16. FP8 inputs are
derived from the bfloat16 tensors by per-head absmax scaling (scale =
absmax / 448) and round-to-nearest-even conversion to e4m3 (torch's cast),
clamped to +-448.

The public benchmark suites the pages measure on (RULER, InfiniteBench,
Needle-in-a-Haystack) and the model weights are not available here; these
seeded tensors with the attention shapes of the models the pages name stand in
for them.
"""
from __future__ import annotations

import json
import math
import os
from dataclasses import dataclass, field, replace
from typing import Optional

import torch

E4M3_MAX = 448.0


@dataclass(frozen=True)
class Workload:
    """One synthetic prefill workload (shapes, method parameters, generator knobs)."""

    name: str
    seqlens: tuple            # one entry per request (batch element)
    hq: int
    hkv: int
    head_dim: int
    block: int
    alpha: float
    sink_tokens: int
    window_tokens: int
    seed: int                 # request r uses seed + r*seed_stride
    seed_stride: int = 0
    a_q: float = 4.0
    a_h: float = 4.0
    a_s: float = 2.0
    heavy_frac: Optional[float] = None   # fraction of key blocks made heavy
    n_heavy: Optional[int] = None        # or an explicit count
    n_slash: int = 1
    slash_offsets: Optional[tuple] = None  # explicit offsets (tokens) or drawn
    amp_scale: float = 1.0
    paged: bool = False
    page_size: int = 0
    page_seed: int = 0
    description: str = ""

    @property
    def group(self) -> int:
        return self.hq // self.hkv

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    def heavy_count(self, L: int) -> int:
        n = -(-L // self.block)
        if self.n_heavy is not None:
            return min(self.n_heavy, n)
        return max(1, int(round(self.heavy_frac * n)))

    def dense_equiv_flops(self) -> float:
        """4*d*Hq*sum L(L+1)/2: the flops of dense causal attention on these shapes."""
        return 4.0 * self.head_dim * self.hq * sum(L * (L + 1) / 2 for L in self.seqlens)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


_CAL_PATH = os.path.join(os.path.dirname(__file__), "workloads_calibration.json")


def _calibrated(name: str, default: float) -> float:
    """Amplitude factor stored by the calibration script (see that JSON's header)."""
    try:
        with open(_CAL_PATH) as f:
            data = json.load(f)
        return float(data["amp_scale"].get(name, default))
    except (OSError, KeyError, ValueError):
        return default


def _varlen_lengths(seed: int, n: int, lo: int, hi: int) -> tuple:
    g = torch.Generator().manual_seed(seed)
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g))


def workloads() -> dict:
    """The five shape configurations of the FlashPrefill workloads (2K..256K)."""
    w = {}
    w["tiny2k"] = Workload(
        name="tiny2k", seqlens=(2048,), hq=4, hkv=1, head_dim=128, block=64,
        alpha=0.1, sink_tokens=64, window_tokens=128, seed=1,
        n_heavy=6, slash_offsets=(256,),
        description="batch 1, seq 2048, Hq=4, Hkv=1, d=128, bf16, block 64, alpha 0.1, "
                    "sink 1 block, window 2 blocks")
    w["qwen7b_32k"] = Workload(
        name="qwen7b_32k", seqlens=(32768,), hq=28, hkv=4, head_dim=128, block=128,
        alpha=0.05, sink_tokens=256, window_tokens=512, seed=2,
        heavy_frac=0.01, n_slash=3,
        description="32K prefill, Qwen2.5-7B-like attention (Hq=28, Hkv=4, d=128), "
                    "block 128, alpha in {0, 0.05, 0.2}")
    w["qwen30b_128k"] = Workload(
        name="qwen30b_128k", seqlens=(131072,), hq=32, hkv=4, head_dim=128, block=128,
        alpha=0.1, sink_tokens=256, window_tokens=512, seed=3,
        heavy_frac=0.01, n_slash=3, amp_scale=_calibrated("qwen30b_128k", 1.0),
        description="128K prefill, Qwen3-30B-A3B-like attention (Hq=32, Hkv=4, d=128), "
                    "block 128, sink 256, window 512, ~5% of causal blocks kept")
    w["extreme_256k"] = Workload(
        name="extreme_256k", seqlens=(262144,), hq=32, hkv=4, head_dim=128, block=128,
        alpha=0.3, sink_tokens=256, window_tokens=512, seed=4,
        heavy_frac=0.005, n_slash=1, amp_scale=_calibrated("extreme_256k", 1.0),
        description="256K extreme-sparsity prefill, Hq=32, Hkv=4, d=128, block 128, alpha 0.3")
    w["paged_varlen"] = Workload(
        name="paged_varlen", seqlens=_varlen_lengths(5, 8, 4096, 65536), hq=32, hkv=8,
        head_dim=128, block=128, alpha=0.1, sink_tokens=256, window_tokens=512,
        seed=50, seed_stride=1, heavy_frac=0.01, n_slash=3,
        amp_scale=_calibrated("qwen30b_128k", 1.0), paged=True, page_size=64, page_seed=5,
        description="paged KV + continuous batching: 8 requests of 4K-64K tokens, Hq=32, "
                    "Hkv=8, d=128, page 64")
    return w


# ----------------------------------------------------------------------------
# tensor generation
# ----------------------------------------------------------------------------

def _sequence(w: Workload, L: int, seed: int):
    """Q [L,Hq,d], K [L,Hkv,d], V [L,Hkv,d] in bfloat16 plus a description of the plant."""
    g = torch.Generator().manual_seed(seed)
    d, B, G = w.head_dim, w.block, w.group
    c = w.amp_scale
    u = torch.randn(d, generator=g, dtype=torch.float32)
    u = u / u.norm()
    nblk = -(-L // B)
    heavy = torch.randperm(nblk, generator=g)[: w.heavy_count(L)].sort().values.tolist()
    if w.slash_offsets is not None:
        offsets = [int(x) for x in w.slash_offsets]
    else:
        hi = max(B + 1, L // 2 + 1)
        offsets = sorted(int(x) for x in torch.randint(B, hi, (w.n_slash,), generator=g))
    q = torch.empty(L, w.hq, d, dtype=torch.bfloat16)
    k = torch.empty(L, w.hkv, d, dtype=torch.bfloat16)
    v = torch.empty(L, w.hkv, d, dtype=torch.bfloat16)
    q0_first = {}
    for h in range(w.hq):
        x = torch.randn(L, d, generator=g, dtype=torch.float32)
        if h % G == 0:
            q0_first[h // G] = x.clone()
        x += (c * w.a_q) * u
        q[:, h] = x.to(torch.bfloat16)
    for kv in range(w.hkv):
        x = torch.randn(L, d, generator=g, dtype=torch.float32)
        for j in heavy:
            x[j * B:(j + 1) * B] += (c * w.a_h) * u
        for delta in offsets:
            if delta < L:
                x[: L - delta] += (c * w.a_s) * q0_first[kv][delta:]
        k[:, kv] = x.to(torch.bfloat16)
    del q0_first
    for kv in range(w.hkv):
        v[:, kv] = torch.randn(L, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
    return q, k, v, {"heavy_blocks": heavy, "slash_offsets": offsets}


def quantize_e4m3(x: torch.Tensor, head_dim_axis: int = -1, head_axis: int = -2):
    """Per-head absmax e4m3 quantisation. Returns (x8, scale[H] float32)."""
    xf = x.float()
    dims = [a for a in range(xf.dim()) if a != (head_axis % xf.dim())]
    amax = xf.abs().amax(dim=dims)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    shape = [1] * xf.dim()
    shape[head_axis % xf.dim()] = -1
    x8 = (xf / scale.view(shape)).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return x8, scale.float().contiguous()


@dataclass
class Inputs:
    """Generated tensors (CPU). Contiguous layout: q [batch, L, Hq, d]; k, v [batch, L, Hkv, d].
    Varlen layout: q [T, Hq, d] with cu_seqlens; paged: k_pool/v_pool
    [num_pages, page, Hkv, d] with page_table [R, max_pages] (-1 padded)."""

    workload: Workload
    q: torch.Tensor
    k: Optional[torch.Tensor] = None
    v: Optional[torch.Tensor] = None
    cu_seqlens: Optional[torch.Tensor] = None
    k_pool: Optional[torch.Tensor] = None
    v_pool: Optional[torch.Tensor] = None
    page_table: Optional[torch.Tensor] = None
    plants: list = field(default_factory=list)
    kv_lens: Optional[torch.Tensor] = None   # chunked prefill: KV length per request
    # fp8 variants (filled by to_fp8)
    q_scale: Optional[torch.Tensor] = None
    k_scale: Optional[torch.Tensor] = None
    v_scale: Optional[torch.Tensor] = None
    dtype: str = "bf16"


def make_inputs(w: Workload, seqlens: Optional[tuple] = None) -> Inputs:
    """Generate a workload's tensors. ``seqlens`` overrides the workload's lengths
    (used for small parity cases of the same structure)."""
    lens = tuple(seqlens) if seqlens is not None else tuple(w.seqlens)
    seqs = [_sequence(w, L, w.seed + r * w.seed_stride) for r, L in enumerate(lens)]
    plants = [s[3] for s in seqs]
    if not w.paged:
        if len(set(lens)) != 1:
            raise ValueError("a contiguous batch needs equal lengths")
        q = torch.stack([s[0] for s in seqs])
        k = torch.stack([s[1] for s in seqs])
        v = torch.stack([s[2] for s in seqs])
        return Inputs(w, q, k, v, plants=plants)
    P = w.page_size
    npages = [-(-L // P) for L in lens]
    total_pages = sum(npages)
    gperm = torch.Generator().manual_seed(w.page_seed)
    perm = torch.randperm(total_pages, generator=gperm)
    maxp = max(npages)
    table = torch.full((len(lens), maxp), -1, dtype=torch.int32)
    k_pool = torch.zeros(total_pages, P, w.hkv, w.head_dim, dtype=torch.bfloat16)
    v_pool = torch.zeros_like(k_pool)
    off = 0
    for r, (L, (qs, ks, vs, _)) in enumerate(zip(lens, seqs)):
        pages = perm[off: off + npages[r]]
        off += npages[r]
        table[r, : npages[r]] = pages.to(torch.int32)
        for p in range(npages[r]):
            lo, hi = p * P, min((p + 1) * P, L)
            k_pool[pages[p], : hi - lo] = ks[lo:hi]
            v_pool[pages[p], : hi - lo] = vs[lo:hi]
    q = torch.cat([s[0] for s in seqs])
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lens, dtype=torch.int64), 0).to(torch.int32)
    return Inputs(w, q, cu_seqlens=cu, k_pool=k_pool, v_pool=v_pool, page_table=table,
                  plants=plants)


def make_chunked_inputs(w: Workload, kv_lens: tuple, q_lens: tuple) -> Inputs:
    """Chunked prefill with a cached prefix: request r has kv_lens[r] tokens in
    the paged KV pool and its last q_lens[r] tokens are the queries (packed by
    cu_seqlens). The tokens are generated exactly as for full prefill."""
    if len(kv_lens) != len(q_lens) or any(q > k for q, k in zip(q_lens, kv_lens)):
        raise ValueError("need one q_len <= kv_len per request")
    full = make_inputs(w.with_(paged=True, page_size=w.page_size or 64), seqlens=tuple(kv_lens))
    cu = full.cu_seqlens.tolist()
    q = torch.cat([full.q[cu[r + 1] - q_lens[r]: cu[r + 1]] for r in range(len(kv_lens))])
    cuq = torch.zeros(len(q_lens) + 1, dtype=torch.int32)
    cuq[1:] = torch.cumsum(torch.tensor(q_lens, dtype=torch.int64), 0).to(torch.int32)
    return Inputs(full.workload, q, cu_seqlens=cuq, k_pool=full.k_pool, v_pool=full.v_pool,
                  page_table=full.page_table, plants=full.plants,
                  kv_lens=torch.tensor(kv_lens, dtype=torch.int32))


def to_fp8(inp: Inputs) -> Inputs:
    """FP8-e4m3 copy of ``inp`` with per-head absmax scales (over the whole sequence or pool)."""
    out = Inputs(inp.workload, None, cu_seqlens=inp.cu_seqlens, page_table=inp.page_table,
                 plants=inp.plants, dtype="e4m3", kv_lens=inp.kv_lens)
    out.q, out.q_scale = quantize_e4m3(inp.q)
    if inp.k is not None:
        out.k, out.k_scale = quantize_e4m3(inp.k)
        out.v, out.v_scale = quantize_e4m3(inp.v)
    else:
        out.k_pool, out.k_scale = quantize_e4m3(inp.k_pool)
        out.v_pool, out.v_scale = quantize_e4m3(inp.v_pool)
    return out


def dequantize(x8: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
    """Exact float64 value of an e4m3 tensor times its per-head (axis -2) scale."""
    return x8.to(torch.float64) * scale.to(torch.float64).view(-1, 1)


def small_case(w: Workload, L: int, **kw) -> Workload:
    """Same structure at a reduced length (for parity cases the oracle finishes quickly)."""
    return replace(w, seqlens=(L,), **kw)
