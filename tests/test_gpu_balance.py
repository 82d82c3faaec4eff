"""Scheduler balance records (FAPK_FLAG_CTA_TIMES): every CTA of the
persistent kernels reports a (start, end) %globaltimer pair, and recording
changes no output bit."""
import numpy as np
import pytest
import torch

from causal_flash_attention_packed_b200 import fapk, workloads as W
from gpu_util import require_gpu, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("prec", [fapk.BF16, fapk.MXFP8])
def test_cta_times_recorded_and_outputs_unchanged(prec):
    dev = require_gpu()
    w = W.custom([900, 2048, 77, 3000], Hq=4, Hkv=2, d=128, seed=91)
    (q, k, v, do), (qd, kd, vd, dod) = to_dev(w, dev)
    seq = fapk.Seqlens(w.cu, dev)
    outs = []
    for flags in (0, fapk.FLAG_CTA_TIMES):
        P = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale, prec=prec, flags=flags)
        ws_f = fapk.workspace(P, fapk.FWD, dev)
        ws_b = fapk.workspace(P, fapk.BWD, dev)
        o, lse, ctx = fapk.attn_fwd(P, qd, kd, vd, ws=ws_f)
        dq, dk, dv = fapk.attn_bwd(P, qd, kd, vd, o, lse, dod, ctx=ctx, ws=ws_b)
        assert fapk.status(ws_f) == fapk.OK and fapk.status(ws_b) == fapk.OK
        outs.append((o, lse, dq, dk, dv))
        if flags:
            sms = torch.cuda.get_device_properties(dev).multi_processor_count
            for which, kernel, ws in ((fapk.FWD, 0, ws_f), (fapk.BWD, 0, ws_b), (fapk.BWD, 1, ws_b)):
                t = fapk.cta_times(P, which, kernel, ws)
                assert 1 <= len(t) <= sms
                assert np.all(t[:, 0] > 0) and np.all(t[:, 1] >= t[:, 0])
                # all CTAs of one launch run within one second of each other
                assert t[:, 1].max() - t[:, 0].min() < 1_000_000_000
    for a, b in zip(*outs):
        assert torch.equal(a, b)
