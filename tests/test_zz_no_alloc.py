"""The forward entry point that allocates nothing (fapk_attn_fwd_noalloc),
for callers that cannot obtain device memory where they run the forward.  Its
output must agree with the regular fapk_attn_fwd on two calls in a row (the
second reuses the library's scratch array as the first left it).  This file is
collected last so that a run stopping at the first failure has already run
every other test."""
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
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        ctx = torch.empty(max(fapk.ctx_size(P), 256), dtype=torch.uint8, device=dev)
        assert _noalloc(P, qd, kd, vd, o, lse, ctx) == fapk.OK, f"call {call}"
        torch.cuda.synchronize()
        check_close(f"O (call {call})", f64(o), f64(o_ref))
        assert float(np.max(np.abs(f64(lse) - f64(lse_ref)))) <= LSE_ABS


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
