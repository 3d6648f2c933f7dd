"""C-ABI boundary checks that need no GPU: the library builds for sm_100a,
loads, exports every function include/flashprefill.h declares, sizes its
buffers by the documented formulas, and rejects invalid arguments before any
CUDA call."""
import ctypes
import math
import os
import re

import pytest

from block_sparse_long_blocks_b200 import binding as fb
from block_sparse_long_blocks_b200 import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "flashprefill.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return fb.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fp_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert {"fp_discover", "fp_compact", "fp_sparse_prefill", "fp_paged_sparse_prefill"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def _cfg(**kw):
    base = dict(batch=1, max_seqlen=131072, hq=32, hkv=4, block=128, alpha=0.1, sink_tokens=256,
                window_tokens=512)
    base.update(kw)
    return fb.Config(**base)


def test_buffer_sizes(lib):
    p = fb.make_params(_cfg())
    s = fb.sizes(p)
    N = 1024
    assert s["mask_words"] == 4 * N * 32
    assert s["list_capacity"] == 4 * N * (N + 1) // 2
    assert s["count_entries"] == 4 * N
    assert s["workspace"] >= (N * 32 * 128 + 4 * 128 * N) * 4
    p = fb.make_params(_cfg(max_seqlen=1000, block=64, batch=3))
    s = fb.sizes(p)
    N = math.ceil(1000 / 64)
    assert s["mask_words"] == 3 * 4 * N * 1 and s["count_entries"] == 3 * 4 * N


def _pad256(n):
    return (n + 255) // 256 * 256


@pytest.mark.parametrize("kw,pairs", [({}, 4), (dict(hq=4), 1), (dict(hkv=2), 8), (dict(hq=6, hkv=2), 2)])
def test_workspace_layout(lib, kw, pairs):
    """Pooled query and key planes (three bf16 parts each, d values per row),
    the work-queue counter and the claim order of the attention's work units:
    M-tile pairs per query block = B / (2 Tm), Tm the largest power of two with
    Tm G <= 128 and Tm <= B / 2."""
    for d in (128, 64):
        cfg = _cfg(head_dim=d, **kw)
        p = fb.make_params(cfg)
        N, R, Hq, Hkv = cfg.nmax, cfg.batch, cfg.hq, cfg.hkv
        q_planes = _pad256(3 * 2 * R * N * Hq * d)
        k_planes = _pad256(3 * 2 * R * Hkv * N * d)
        order = _pad256(4 * N * R * Hkv * pairs)
        assert fb.sizes(p)["workspace"] == q_planes + k_planes + 256 + order


def test_single_call_argument_checks(lib):
    p = fb.make_params(_cfg())
    ok = 1 << 20  # never dereferenced: validation fails first
    ws = lib.fp_workspace_size(ctypes.byref(p))
    f = lib.fp_prefill
    assert f(ctypes.byref(p), ok, ok, ok, None, None, ok, ok, None, ok, ws, None) == -1   # idx missing
    assert f(ctypes.byref(p), ok, ok, ok, None, ok, None, ok, None, ok, ws, None) == -1   # cnt missing
    assert f(ctypes.byref(p), ok, ok, None, None, ok, ok, ok, None, ok, ws, None) == -1   # v missing
    assert f(ctypes.byref(p), ok, ok, ok, None, ok, ok, ok + 8, None, ok, ws, None) == -3  # o misaligned
    assert f(ctypes.byref(p), ok, ok, ok, None, ok, ok, ok, None, ok, ws - 1, None) == -4  # workspace short


@pytest.mark.parametrize("bad,code", [
    (dict(head_dim=96), -2), (dict(head_dim=256), -2), (dict(head_dim=64, fp8=True), -2), (dict(block=32), -2), (dict(alpha=-0.5), -1), (dict(alpha=float("nan")), -1),
    (dict(alpha=float("inf")), -1), (dict(hq=30, hkv=4), -1), (dict(batch=0), -1), (dict(max_seqlen=0), -1),
    (dict(sink_tokens=-1), -1), (dict(hq=36, hkv=4), -2), (dict(max_seqlen=128 * 8193), -2),
])
def test_invalid_arguments_rejected_before_launch(lib, bad, code):
    p = fb.make_params(_cfg(**bad))
    assert lib.fp_workspace_size(ctypes.byref(p)) == 0
    fake = 1 << 20  # never dereferenced: validation fails first
    rc = lib.fp_discover(ctypes.byref(p), fake, fake, fake, fake, 1 << 30, None)
    assert rc == code
    rc = lib.fp_sparse_prefill(ctypes.byref(p), fake, fake, fake, fake, fake, fake, None, None)
    assert rc == code


def test_alignment_workspace_and_pointer_checks(lib):
    p = fb.make_params(_cfg())
    ok = 1 << 20
    assert lib.fp_discover(ctypes.byref(p), ok + 2, ok, ok, ok, 1 << 30, None) == -3
    assert lib.fp_discover(ctypes.byref(p), ok, ok, ok, None, 1 << 30, None) == -4
    assert lib.fp_discover(ctypes.byref(p), ok, ok, ok, ok, 16, None) == -4
    assert lib.fp_discover(ctypes.byref(p), ok, ok, None, ok, 1 << 30, None) == -1
    assert lib.fp_sparse_prefill(ctypes.byref(p), ok, ok, ok, ok, ok, None, None, None) == -1
    # paged call without a page table, and a page table without cu_seqlens
    assert lib.fp_paged_sparse_prefill(ctypes.byref(p), ok, ok, ok, ok, ok, ok, None, None) == -1
    p.page_table = ok
    p.page_size, p.max_pages_per_req, p.num_pages = 64, 2048, 10
    assert lib.fp_sparse_prefill(ctypes.byref(p), ok, ok, ok, ok, ok, ok, None, None) == -1
    # fp8 without scales
    p = fb.make_params(_cfg(fp8=True))
    assert lib.fp_discover(ctypes.byref(p), ok, ok, ok, ok, 1 << 30, None) == -1


def test_status_strings(lib):
    for code, name in fb.STATUS.items():
        assert lib.fp_status_string(code).decode() == name


def test_short_wait_variant_builds_and_exports_the_same_symbols():
    """The test build with a 500 ns pipeline-wait limit (abort-path test) is the
    same library: same sources, same entry points."""
    path = build.build_variant("short_wait")
    short = fb.load_library(path)
    for n in declared_functions():
        assert hasattr(short, n), n
    assert short.fp_static_scratch_bytes() == fb.load().fp_static_scratch_bytes()
