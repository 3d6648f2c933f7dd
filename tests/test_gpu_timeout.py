"""The kernels' abort path, driven without any fault.

Every pipeline wait in the kernels gives up after a time limit (2 s in the
library), records FP_DEV_TIMEOUT in the device status word, lets the CTA's own
TMA copies and MMAs land (those drain waits keep the 2 s limit), frees its
tensor memory and returns. A build of the library with a 500 ns pipeline limit
(``libflashprefill_short_wait.so``) makes ordinary waits run out, so every
launch takes that path: the calls must return, report the timeout and clear it
on the read, and leave the device usable -- the normal library's results
afterwards are bit-identical to those before.
"""
import ctypes

import pytest
import torch

from block_sparse_long_blocks_b200 import binding as fb
from block_sparse_long_blocks_b200 import build
from block_sparse_long_blocks_b200 import workloads as wl
from tests import _helpers as H

pytestmark = pytest.mark.gpu


def _status(lib) -> int:
    bits = ctypes.c_uint32(0)
    rc = lib.fp_get_device_status(ctypes.byref(bits), torch.cuda.current_stream().cuda_stream)
    assert rc in (0, -6), rc  # FP_OK or FP_ERR_DEVICE
    return int(bits.value)


@pytest.mark.parametrize("name,L,fp8", [("qwen30b_128k", 4096, False), ("qwen30b_128k", 4096, True),
                                        ("paged_varlen", None, False)])
def test_short_wait_limit_aborts_cleanly_then_normal_calls_are_exact(name, L, fp8):
    short = fb.load_library(build.build_variant("short_wait"))
    w = wl.workloads()[name]
    w = wl.small_case(w, L) if L else w.with_(seqlens=(1500, 700, 2100))
    inp = wl.make_inputs(w)
    if fp8:
        inp = wl.to_fp8(inp)
    ref = H.Device(w, inp)
    ref.discover()
    ref.attend()
    assert ref.status() == 0
    o_ref, lse_ref, cnt_ref = ref.bufs.o.clone(), ref.bufs.lse.clone(), ref.bufs.cnt.clone()

    s = torch.cuda.current_stream().cuda_stream
    d = H.Device(w, inp)
    p = ctypes.byref(d.p)
    ws = d.bufs.workspace
    attend = short.fp_paged_sparse_prefill if d.paged else short.fp_sparse_prefill

    # discovery + compaction (scoring kernel waits)
    d.bufs.cnt.zero_()
    assert short.fp_discover_compact(p, d.q.data_ptr(), d.k.data_ptr(), d.bufs.mask.data_ptr(),
                                     d.bufs.idx.data_ptr(), d.bufs.cnt.data_ptr(), ws.data_ptr(), ws.numel(), s) == 0
    assert _status(short) == fb.DEV_TIMEOUT
    assert _status(short) == 0  # cleared by the read

    # attention on valid lists (producer / MMA / softmax waits)
    assert attend(p, d.q.data_ptr(), d.k.data_ptr(), d.v.data_ptr(), ref.bufs.idx.data_ptr(),
                  ref.bufs.cnt.data_ptr(), d.bufs.o.data_ptr(), d.bufs.lse.data_ptr(), s) == 0
    assert _status(short) == fb.DEV_TIMEOUT
    assert _status(short) == 0

    # the single call: discovery, claim-order sort, attention as a dependent launch on the device queue
    d.bufs.idx.zero_()
    d.bufs.cnt.zero_()
    assert short.fp_prefill(p, d.q.data_ptr(), d.k.data_ptr(), d.v.data_ptr(), None, d.bufs.idx.data_ptr(),
                            d.bufs.cnt.data_ptr(), d.bufs.o.data_ptr(), d.bufs.lse.data_ptr(), ws.data_ptr(),
                            ws.numel(), s) == 0
    assert _status(short) & fb.DEV_TIMEOUT
    assert _status(short) == 0

    # the normal library's status word is its own and was never touched
    assert ref.status() == 0
    again = H.Device(w, inp)
    again.discover()
    again.attend()
    assert again.status() == 0
    assert torch.equal(again.bufs.cnt, cnt_ref)
    assert torch.equal(again.bufs.o, o_ref)
    assert torch.equal(torch.nan_to_num(again.bufs.lse, nan=7.0), torch.nan_to_num(lse_ref, nan=7.0))
