"""The forward entry point that allocates nothing (fapk_attn_fwd_noalloc),
for callers that cannot obtain device memory where they run the forward (a
plugin handed its buffers by a host framework, a runtime that has reserved all
device memory).  Its output must agree with the regular fapk_attn_fwd on two
calls in a row (the second reuses the library's scratch array as the first left
it), the second call must not change the device's free memory or torch's
allocation, and its device status word is read with fapk_noalloc_status.  This
file is collected last so that a run stopping at the first failure has already
run every other test."""
import ctypes

import numpy as np
import pytest
import torch

from causal_flash_attention_packed_b200 import fapk, workloads as W
from gpu_util import LSE_ABS, check_close, f64, require_gpu, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(P, qd, kd, vd, o, lse, ctx):
    L = fapk.lib()
    fn = L.fapk_attn_fwd_noalloc
    fn.argtypes = [ctypes.POINTER(fapk.Problem)] + [ctypes.c_void_p] * 7
    fn.restype = ctypes.c_int
    return fn(ctypes.byref(P), qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(), lse.data_ptr(),
              ctx.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_noalloc_forward_matches_regular_forward_twice():
    dev = require_gpu()
    w = W.custom([1, 300, 700, 129, 2048], Hq=4, Hkv=2, d=128, seed=51)
    (_, _, _, _), (qd, kd, vd, _) = to_dev(w, dev, with_dout=False)
    seq = fapk.Seqlens(w.cu, dev)
    P = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale)
    o_ref, lse_ref, _ = fapk.attn_fwd(P, qd, kd, vd)
    bufs = [(torch.full_like(o_ref, float("nan")), torch.full_like(lse_ref, float("nan")),
             torch.empty(max(fapk.ctx_size(P), 256), dtype=torch.uint8, device=dev)) for _ in range(2)]
    for call, (o, lse, ctx) in enumerate(bufs):
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info(dev)
        alloc0 = torch.cuda.memory_allocated(dev)
        assert _noalloc(P, qd, kd, vd, o, lse, ctx) == fapk.OK, f"call {call}"
        assert fapk.noalloc_status() == fapk.OK, f"call {call}"
        torch.cuda.synchronize()
        if call == 1:
            # the first call may load the library's module (and its array) on
            # this device; the second must take no device memory at all
            assert torch.cuda.mem_get_info(dev)[0] == free0
            assert torch.cuda.memory_allocated(dev) == alloc0
        check_close(f"O (call {call})", f64(o), f64(o_ref))
        assert float(np.max(np.abs(f64(lse) - f64(lse_ref)))) <= LSE_ABS


def test_noalloc_status_reports_a_device_side_error():
    """Without the host copy of cu_seqlens the library cannot validate on the
    host; a document longer than max_seqlen is caught by the device scheduler,
    skipped, and reported through the no-allocation status word.  The next
    valid call clears it."""
    dev = require_gpu()
    w = W.custom([100, 700], Hq=2, Hkv=2, d=64, seed=42)
    (_, _, _, _), (qd, kd, vd, _) = to_dev(w, dev, with_dout=False)
    seq = fapk.Seqlens(w.cu, dev)
    bad = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale, validate_host=False)
    bad.max_seqlen = 256
    o = torch.empty_like(qd)
    lse = torch.empty((w.Hq, w.T), dtype=torch.float32, device=dev)
    ctx = torch.empty(max(fapk.ctx_size(bad), 256), dtype=torch.uint8, device=dev)
    assert _noalloc(bad, qd, kd, vd, o, lse, ctx) == fapk.OK
    assert fapk.noalloc_status() == fapk.ERR_BAD_SEQLENS
    good = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale)
    ctx = torch.empty(max(fapk.ctx_size(good), 256), dtype=torch.uint8, device=dev)
    assert _noalloc(good, qd, kd, vd, o, lse, ctx) == fapk.OK
    assert fapk.noalloc_status() == fapk.OK


def test_noalloc_rejects_problems_beyond_its_scratch():
    dev = require_gpu()
    # 200000 one-token documents need a work list larger than the 1 MiB array
    lengths = [1] * 200000
    seq = fapk.Seqlens(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32), dev)
    P = fapk.make_problem(seq, 1, 1, 64, 0.125)
    x = torch.zeros((seq.T, 1, 64), dtype=torch.bfloat16, device=dev)
    o = torch.empty_like(x)
    lse = torch.empty((1, seq.T), dtype=torch.float32, device=dev)
    ctx = torch.empty(max(fapk.ctx_size(P), 256), dtype=torch.uint8, device=dev)
    assert _noalloc(P, x, x, x, o, lse, ctx) == fapk.ERR_WORKSPACE_TOO_SMALL
