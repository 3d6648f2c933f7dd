"""The workspace-free discovery entry point, fp_discover_compact_static.

It serves callers that cannot allocate device memory (a plugin inside an
engine that owns all device memory, or a path that must not call cudaMalloc
because it can synchronise the device): its scratch is a fixed array inside
the library. Its outputs must equal those of fp_discover_compact, which takes
a caller-allocated workspace, on consecutive calls that reuse the array.
This file is collected last so that a failure here never hides another test.
"""
import ctypes

import pytest
import torch

from block_sparse_long_blocks_b200 import binding as fb
from block_sparse_long_blocks_b200 import build
from block_sparse_long_blocks_b200 import workloads as wl


@pytest.mark.gpu
def test_static_scratch_matches_workspace_entry_on_consecutive_calls():
    lib = fb.load()
    cases = [wl.small_case(wl.workloads()["qwen30b_128k"], 8192),
             wl.workloads()["tiny2k"],
             wl.small_case(wl.workloads()["extreme_256k"], 5000),
             wl.workloads()["qwen30b_128k"]]  # the full 128K sequence the size limit is stated for
    for w in cases:
        inp = wl.make_inputs(w)
        cfg = fb.config_for(w, inp)
        p = fb.make_params(cfg)
        assert lib.fp_workspace_size(ctypes.byref(p)) <= lib.fp_static_scratch_bytes()
        q, k = inp.q.cuda(), inp.k.cuda()
        ref = fb.Buffers(p)
        fb.fp_discover_compact(p, q, k, ref.mask, ref.idx, ref.cnt, ref.workspace)
        out = fb.Buffers(p)
        for t in (out.mask, out.idx, out.cnt):
            t.fill_(-7)
        fb.fp_discover_compact_static(p, q, k, out.mask, out.idx, out.cnt)
        torch.cuda.synchronize()
        assert fb.fp_get_device_status() == 0
        assert torch.equal(ref.cnt, out.cnt)
        assert torch.equal(ref.mask, out.mask)
        lists_ref = fb.lists_from_device(cfg, ref.idx, ref.cnt)
        lists_out = fb.lists_from_device(cfg, out.idx, out.cnt)
        assert lists_ref == lists_out


def test_static_scratch_rejects_problems_beyond_its_size():
    build.build()
    lib = fb.load()
    limit = lib.fp_static_scratch_bytes()
    cfg = fb.Config(batch=1, max_seqlen=262144, hq=32, hkv=4, block=128, alpha=0.3, sink_tokens=256,
                    window_tokens=512)
    p = fb.make_params(cfg)
    assert lib.fp_workspace_size(ctypes.byref(p)) > limit
    fake = 1 << 20  # never dereferenced: the size check comes first
    rc = lib.fp_discover_compact_static(ctypes.byref(p), fake, fake, fake, fake, fake, None)
    assert rc == -4  # FP_ERR_WORKSPACE
    assert b"static array holds" in lib.fp_last_error()
