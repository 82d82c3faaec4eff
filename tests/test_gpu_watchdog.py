"""Failure detection without a GPU fault: the forward's load warp drops one
K/V copy (host-requested fault injection), the consumer's bounded wait runs
out after `timeout_ms`, the kernel records FAPK_ERR_DEVICE_TIMEOUT in the
workspace status word and every warp leaves its loop; the context stays
usable and the next call is correct."""
import numpy as np
import pytest
import torch

import oracle
from causal_flash_attention_packed_b200 import fapk, workloads as W
from gpu_util import check_close, f64, require_gpu, to_dev

pytestmark = pytest.mark.gpu


def test_dropped_load_reports_timeout_and_context_survives():
    dev = require_gpu()
    w = W.custom([2048, 300], Hq=2, Hkv=2, d=128, seed=41)
    (q, k, v, _), (qd, kd, vd, _) = to_dev(w, dev, with_dout=False)
    seq = fapk.Seqlens(w.cu, dev)
    bad = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale, flags=fapk.FLAG_INJECT_DROP_LOAD,
                            timeout_ms=50)
    ws = fapk.workspace(bad, fapk.FWD, dev)
    fapk.attn_fwd(bad, qd, kd, vd, ws=ws)
    assert fapk.status(ws) == fapk.ERR_DEVICE_TIMEOUT
    # same workspace, normal call: the status word is cleared and results are right
    good = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale)
    o, lse, _ = fapk.attn_fwd(good, qd, kd, vd, ws=ws)
    assert fapk.status(ws) == fapk.OK
    ro, _ = oracle.attn_fwd(q.double().numpy(), k.double().numpy(), v.double().numpy(), w.cu, w.scale)
    check_close("O", f64(o), ro)


def test_document_longer_than_max_seqlen_is_reported():
    """Without the host copy of cu_seqlens the library cannot validate on the
    host; a document longer than max_seqlen is then caught by the device
    scheduler, skipped, and reported as FAPK_ERR_BAD_SEQLENS."""
    dev = require_gpu()
    w = W.custom([100, 700], Hq=2, Hkv=2, d=64, seed=42)
    (_, _, _, _), (qd, kd, vd, _) = to_dev(w, dev, with_dout=False)
    seq = fapk.Seqlens(w.cu, dev)
    P = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale, validate_host=False)
    P.max_seqlen = 256
    ws = fapk.workspace(P, fapk.FWD, dev)
    fapk.attn_fwd(P, qd, kd, vd, ws=ws)
    assert fapk.status(ws) == fapk.ERR_BAD_SEQLENS
