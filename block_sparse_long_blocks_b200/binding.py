"""ctypes binding of ``libflashprefill.so`` (argument marshalling only).

Every computation happens in the library's CUDA kernels; this module converts
torch tensors into pointers/sizes, fills ``fp_params_t`` and raises on a
non-zero status. torch supplies device memory and the current CUDA stream.
The function names mirror the C ABI in ``include/flashprefill.h``.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libflashprefill.so")

FP_BF16, FP_E4M3 = 0, 1
STATUS = {0: "FP_OK", -1: "FP_ERR_INVALID_ARG", -2: "FP_ERR_UNSUPPORTED", -3: "FP_ERR_ALIGNMENT",
          -4: "FP_ERR_WORKSPACE", -5: "FP_ERR_CUDA", -6: "FP_ERR_DEVICE"}
DEV_TIMEOUT, DEV_BAD_SEQLENS, DEV_BAD_PAGE, DEV_BAD_LIST = 1, 2, 4, 8


class FPError(RuntimeError):
    def __init__(self, fn: str, code: int):
        detail = ""
        if code == -5 and _lib is not None:
            detail = " (" + (_lib.fp_last_error() or b"").decode(errors="replace") + ")"
        super().__init__(f"{fn} returned {STATUS.get(code, code)}{detail}")
        self.code = code


class Params(ctypes.Structure):
    """Mirror of ``fp_params_t``."""

    _fields_ = [
        ("dtype", ctypes.c_int),
        ("batch", ctypes.c_int),
        ("max_seqlen", ctypes.c_int),
        ("hq", ctypes.c_int),
        ("hkv", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("block", ctypes.c_int),
        ("alpha", ctypes.c_float),
        ("sink_tokens", ctypes.c_int),
        ("window_tokens", ctypes.c_int),
        ("softmax_scale", ctypes.c_float),
        ("q_scale", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p),
        ("v_scale", ctypes.c_void_p),
        ("cu_seqlens", ctypes.c_void_p),
        ("total_tokens", ctypes.c_int),
        ("page_table", ctypes.c_void_p),
        ("page_size", ctypes.c_int),
        ("max_pages_per_req", ctypes.c_int),
        ("num_pages", ctypes.c_int),
        ("kv_lens", ctypes.c_void_p),
        ("head_bits", ctypes.c_void_p),
    ]


_lib = None


def load_library(path: str) -> ctypes.CDLL:
    """A handle on a build of the library at ``path`` with every entry point's
    signature declared (not cached: build variants load side by side)."""
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m block_sparse_long_blocks_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(Params)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    sig = {
        "fp_workspace_size": (sz, [P]),
        "fp_mask_words": (sz, [P]),
        "fp_list_capacity": (sz, [P]),
        "fp_count_entries": (sz, [P]),
        "fp_discover": (ctypes.c_int, [P, vp, vp, vp, vp, sz, vp]),
        "fp_compact": (ctypes.c_int, [P, vp, vp, vp, vp]),
        "fp_discover_compact": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, sz, vp]),
        "fp_sparse_prefill": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, vp]),
        "fp_paged_sparse_prefill": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, vp]),
        "fp_get_device_status": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), vp]),
        "fp_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "fp_last_error": (ctypes.c_char_p, []),
        "fp_discover_compact_static": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp]),
        "fp_prefill": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "fp_static_scratch_bytes": (sz, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the in-tree library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        _lib = load_library(path)
    return _lib


@dataclass
class Config:
    """Method and shape parameters of one call (see ``fp_params_t``)."""

    batch: int
    max_seqlen: int
    hq: int
    hkv: int
    block: int
    alpha: float
    sink_tokens: int = 0
    window_tokens: int = 0
    head_dim: int = 128
    softmax_scale: float = 0.0
    fp8: bool = False
    total_tokens: int = 0
    page_size: int = 0
    max_pages_per_req: int = 0
    num_pages: int = 0

    @property
    def nmax(self) -> int:
        return -(-self.max_seqlen // self.block)

    @property
    def wmax(self) -> int:
        return -(-self.nmax // 32)

    @property
    def scale(self) -> float:
        return self.softmax_scale if self.softmax_scale > 0 else 1.0 / math.sqrt(self.head_dim)


def config_for(w, inp, alpha: Optional[float] = None) -> Config:
    """Library parameters of a generated workload (``workloads.Workload`` + ``Inputs``)."""
    a = w.alpha if alpha is None else alpha
    fp8 = inp.dtype == "e4m3"
    if inp.cu_seqlens is None:
        return Config(batch=inp.q.shape[0], max_seqlen=inp.q.shape[1], hq=w.hq, hkv=w.hkv, block=w.block,
                      alpha=a, sink_tokens=w.sink_tokens, window_tokens=w.window_tokens, fp8=fp8,
                      head_dim=w.head_dim)
    lens = (inp.cu_seqlens[1:] - inp.cu_seqlens[:-1]).tolist()
    if getattr(inp, "kv_lens", None) is not None:
        lens = inp.kv_lens.tolist()
    paged = inp.page_table is not None
    return Config(batch=len(lens), max_seqlen=max(lens), hq=w.hq, hkv=w.hkv, block=w.block, alpha=a,
                  sink_tokens=w.sink_tokens, window_tokens=w.window_tokens, fp8=fp8, head_dim=w.head_dim,
                  total_tokens=int(inp.cu_seqlens[-1]), page_size=w.page_size if paged else 0,
                  max_pages_per_req=inp.page_table.shape[1] if paged else 0,
                  num_pages=inp.k_pool.shape[0] if paged else 0)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def make_params(cfg: Config, q_scale=None, k_scale=None, v_scale=None, cu_seqlens=None,
                page_table=None, kv_lens=None, head_bits=None) -> Params:
    p = Params()
    p.dtype = FP_E4M3 if cfg.fp8 else FP_BF16
    p.batch, p.max_seqlen, p.hq, p.hkv = cfg.batch, cfg.max_seqlen, cfg.hq, cfg.hkv
    p.head_dim, p.block, p.alpha = cfg.head_dim, cfg.block, cfg.alpha
    p.sink_tokens, p.window_tokens, p.softmax_scale = cfg.sink_tokens, cfg.window_tokens, cfg.softmax_scale
    p.q_scale, p.k_scale, p.v_scale = _ptr(q_scale), _ptr(k_scale), _ptr(v_scale)
    p.cu_seqlens = _ptr(cu_seqlens)
    p.total_tokens = cfg.total_tokens
    p.page_table = _ptr(page_table)
    p.page_size, p.max_pages_per_req, p.num_pages = cfg.page_size, cfg.max_pages_per_req, cfg.num_pages
    p.kv_lens = _ptr(kv_lens)
    p.head_bits = _ptr(head_bits)
    return p


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check(fn: str, code: int):
    if code != 0:
        raise FPError(fn, code)


def sizes(p: Params) -> dict:
    lib = load()
    return dict(workspace=lib.fp_workspace_size(ctypes.byref(p)), mask_words=lib.fp_mask_words(ctypes.byref(p)),
                list_capacity=lib.fp_list_capacity(ctypes.byref(p)),
                count_entries=lib.fp_count_entries(ctypes.byref(p)))


class Buffers:
    """Device outputs and scratch of one configuration (allocated by torch)."""

    def __init__(self, p: Params, device="cuda", lse_rows: int = 0, o_shape=None, hq: int = 0):
        s = sizes(p)
        if s["workspace"] == 0:
            raise FPError("fp_workspace_size", -1)
        self.workspace = torch.empty(s["workspace"], dtype=torch.uint8, device=device)
        self.mask = torch.empty(s["mask_words"], dtype=torch.int32, device=device)
        self.idx = torch.empty(s["list_capacity"], dtype=torch.int32, device=device)
        self.cnt = torch.empty(s["count_entries"], dtype=torch.int32, device=device)
        self.o = torch.empty(o_shape, dtype=torch.bfloat16, device=device) if o_shape is not None else None
        self.lse = torch.empty(hq, lse_rows, dtype=torch.float32, device=device) if lse_rows else None


def fp_discover(p: Params, q, k, mask, workspace, stream=None):
    lib = load()
    _check("fp_discover", lib.fp_discover(ctypes.byref(p), q.data_ptr(), k.data_ptr(), mask.data_ptr(),
                                          workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                          _stream(stream)))


def fp_compact(p: Params, mask, idx, cnt, stream=None):
    lib = load()
    _check("fp_compact", lib.fp_compact(ctypes.byref(p), mask.data_ptr(), idx.data_ptr(), cnt.data_ptr(),
                                        _stream(stream)))


def fp_discover_compact(p: Params, q, k, mask, idx, cnt, workspace, stream=None):
    lib = load()
    _check("fp_discover_compact",
           lib.fp_discover_compact(ctypes.byref(p), q.data_ptr(), k.data_ptr(), _ptr(mask), idx.data_ptr(),
                                   cnt.data_ptr(), workspace.data_ptr(),
                                   workspace.numel() * workspace.element_size(), _stream(stream)))


def fp_discover_compact_static(p: Params, q, k, mask, idx, cnt, stream=None):
    """fp_discover_compact with the library's fixed scratch array (no workspace)."""
    lib = load()
    _check("fp_discover_compact_static",
           lib.fp_discover_compact_static(ctypes.byref(p), q.data_ptr(), k.data_ptr(), _ptr(mask), idx.data_ptr(),
                                          cnt.data_ptr(), _stream(stream)))


def fp_sparse_prefill(p: Params, q, k, v, idx, cnt, o, lse=None, stream=None):
    lib = load()
    _check("fp_sparse_prefill",
           lib.fp_sparse_prefill(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(),
                                 cnt.data_ptr(), o.data_ptr(), _ptr(lse), _stream(stream)))


def fp_paged_sparse_prefill(p: Params, q, k_pool, v_pool, idx, cnt, o, lse=None, stream=None):
    lib = load()
    _check("fp_paged_sparse_prefill",
           lib.fp_paged_sparse_prefill(ctypes.byref(p), q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(),
                                       idx.data_ptr(), cnt.data_ptr(), o.data_ptr(), _ptr(lse),
                                       _stream(stream)))


def fp_prefill(p: Params, q, k, v, mask, idx, cnt, o, workspace, lse=None, stream=None):
    """The whole path in one call (discovery + compaction + attention, device work queue)."""
    lib = load()
    _check("fp_prefill",
           lib.fp_prefill(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), _ptr(mask), idx.data_ptr(),
                          cnt.data_ptr(), o.data_ptr(), _ptr(lse), workspace.data_ptr(),
                          workspace.numel() * workspace.element_size(), _stream(stream)))


def fp_get_device_status(stream=None) -> int:
    """Synchronises and returns (then clears) the device status bits."""
    lib = load()
    bits = ctypes.c_uint32(0)
    code = lib.fp_get_device_status(ctypes.byref(bits), _stream(stream))
    if code not in (0, -6):
        raise FPError("fp_get_device_status", code)
    return int(bits.value)


def run_path(p: Params, q, k, v, bufs: Buffers, paged: bool = False, fused: bool = True, stream=None):
    """One pass of the hot path: discovery (+ compaction) then sparse attention."""
    if fused:
        fp_discover_compact(p, q, k, bufs.mask, bufs.idx, bufs.cnt, bufs.workspace, stream)
    else:
        fp_discover(p, q, k, bufs.mask, bufs.workspace, stream)
        fp_compact(p, bufs.mask, bufs.idx, bufs.cnt, stream)
    if paged:
        fp_paged_sparse_prefill(p, q, k, v, bufs.idx, bufs.cnt, bufs.o, bufs.lse, stream)
    else:
        fp_sparse_prefill(p, q, k, v, bufs.idx, bufs.cnt, bufs.o, bufs.lse, stream)


def lists_from_device(cfg: Config, idx: torch.Tensor, cnt: torch.Tensor):
    """Host view of the triangular list layout: lists[r][g][i] (python lists of ints)."""
    N = cfg.nmax
    idx = idx.cpu().tolist()
    cnt = cnt.cpu().view(cfg.batch, cfg.hkv, N).tolist()
    tri = N * (N + 1) // 2
    out = []
    for r in range(cfg.batch):
        rg = []
        for g in range(cfg.hkv):
            base = (r * cfg.hkv + g) * tri
            rg.append([idx[base + i * (i + 1) // 2: base + i * (i + 1) // 2 + cnt[r][g][i]] for i in range(N)])
        out.append(rg)
    return out


def mask_from_device(cfg: Config, mask: torch.Tensor):
    """Boolean [R, Hkv, Nmax, Nmax] view of the bit mask (host)."""
    N, W = cfg.nmax, cfg.wmax
    words = mask.cpu().view(torch.int32).numpy().astype("uint32").reshape(cfg.batch, cfg.hkv, N, W)
    import numpy as np
    bits = np.unpackbits(words.view(np.uint8).reshape(cfg.batch, cfg.hkv, N, W, 4), axis=-1,
                         bitorder="little").reshape(cfg.batch, cfg.hkv, N, W * 32)
    return bits[..., :N].astype(bool)
