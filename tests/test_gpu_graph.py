"""The attention step captured into a CUDA graph: the library allocates
nothing and makes only stream-ordered calls, so a whole fwd + bwd step of each
path can be captured once and replayed; replays give results bit-identical to
the eager calls (the schedule kernel runs inside the graph and resets the work
counters every replay)."""
import pytest
import torch

from causal_flash_attention_packed_b200 import fapk, workloads as W
from gpu_util import require_gpu, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("prec", [fapk.BF16, fapk.MXFP8, fapk.NVFP4_MIXED])
def test_fwd_bwd_step_replays_bit_identically(prec):
    dev = require_gpu()
    w = W.custom([1, 129, 300, 700, 64], Hq=4, Hkv=2, d=128, seed=101)
    (_, _, _, _), (qd, kd, vd, dod) = to_dev(w, dev)
    seq = fapk.Seqlens(w.cu, dev)
    P = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale, prec=prec)
    ws_f = fapk.workspace(P, fapk.FWD, dev)
    ws_b = fapk.workspace(P, fapk.BWD, dev)
    ctx = torch.empty(fapk.ctx_size(P), dtype=torch.uint8, device=dev)
    o = torch.empty((w.T, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.Hq, w.T), dtype=torch.float32, device=dev)
    dq = torch.empty((w.T, w.Hq, w.d), dtype=torch.float32, device=dev)
    dk = torch.empty((w.T, w.Hkv, w.d), dtype=torch.float32, device=dev)
    dv = torch.empty((w.T, w.Hkv, w.d), dtype=torch.float32, device=dev)

    def step(stream):
        fapk.attn_fwd(P, qd, kd, vd, o=o, lse=lse, ctx=ctx, ws=ws_f, stream=stream)
        fapk.attn_bwd(P, qd, kd, vd, o, lse, dod, ctx=ctx, dq=dq, dk=dk, dv=dv, ws=ws_b, stream=stream)

    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        step(s)  # eager, on the side stream the graph will use
    torch.cuda.synchronize(dev)
    ref = [t.clone() for t in (o, lse, dq, dk, dv)]
    assert fapk.status(ws_f) == fapk.OK and fapk.status(ws_b) == fapk.OK
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(s)
    for t in (o, lse, dq, dk, dv):
        t.zero_()
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize(dev)
        for a, b in zip(ref, (o, lse, dq, dk, dv)):
            assert torch.equal(a, b)
    assert fapk.status(ws_f) == fapk.OK and fapk.status(ws_b) == fapk.OK
