"""bf16 forward on the GPU against the exact fp64 oracle (O, LSE)."""
import math

import numpy as np
import pytest
import torch

import oracle
from causal_flash_attention_packed_b200 import fapk, workloads as W
from gpu_util import LSE_ABS, check_close, f64, require_gpu, to_dev

pytestmark = pytest.mark.gpu


def run_fwd(w, dev, o_fill=float("nan")):
    (q, k, v, _), (qd, kd, vd, _) = to_dev(w, dev, with_dout=False)
    seq = fapk.Seqlens(w.cu, dev)
    P = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale)
    o = torch.full((w.T, w.Hq, w.d), o_fill, dtype=torch.bfloat16, device=dev)
    lse = torch.full((w.Hq, w.T), o_fill, dtype=torch.float32, device=dev)
    ws = fapk.workspace(P, fapk.FWD, dev)
    fapk.attn_fwd(P, qd, kd, vd, o=o, lse=lse, ws=ws)
    assert fapk.status(ws) == fapk.OK
    return (q, k, v), o, lse


def _check_against_oracle(w, dev):
    (q, k, v), o, lse = run_fwd(w, dev)
    ro, rlse = oracle.attn_fwd(q.double().numpy(), k.double().numpy(), v.double().numpy(), w.cu, w.scale)
    check_close("O", f64(o), ro)
    err = float(np.max(np.abs(f64(lse) - rlse)))
    assert err <= LSE_ABS, f"LSE max_abs={err:.3e}"


def test_single_document_d64():
    """One 256-token document, Hq = Hkv = 2, d = 64 (the small bf16 case)."""
    _check_against_oracle(W.config(1, 0), require_gpu())


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [1, 2])
def test_ragged_documents(d, G):
    """Lengths around every tile boundary (127/128/129, 255/256/257), a
    one-token document, a zero-length document and a long tail."""
    lengths = [1, 127, 128, 0, 129, 255, 256, 257, 300, 1000, 5]
    w = W.custom(lengths, Hq=2 * G, Hkv=2, d=d, seed=11)
    _check_against_oracle(w, require_gpu())


def test_packed_8k_full():
    """8192 packed tokens, U{128..2048} lengths, 16 heads, d = 128, full oracle."""
    _check_against_oracle(W.config(2, 0), require_gpu())


def test_deterministic():
    """Same inputs, same bits."""
    dev = require_gpu()
    w = W.custom([700, 33, 1200], Hq=4, Hkv=2, d=128, seed=5)
    _, o1, l1 = run_fwd(w, dev)
    _, o2, l2 = run_fwd(w, dev)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_later_documents_do_not_leak():
    """T1: randomising every later document leaves O and LSE of the earlier
    documents bit-identical."""
    dev = require_gpu()
    lengths = [300, 513, 200]
    w = W.custom(lengths, Hq=2, Hkv=2, d=128, seed=6)
    (q, k, v, _), (qd, kd, vd, _) = to_dev(w, dev, with_dout=False)
    seq = fapk.Seqlens(w.cu, dev)
    P = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale)
    o1, l1, _ = fapk.attn_fwd(P, qd, kd, vd)
    t = 300 + 100  # perturb everything after token t (rest of doc 1 and doc 2)
    g = torch.Generator(device="cpu").manual_seed(99)
    for x in (qd, kd, vd):
        x[t + 1:] = torch.randn(x[t + 1:].shape, generator=g).to(x.dtype).to(dev)
    o2, l2, _ = fapk.attn_fwd(P, qd, kd, vd)
    torch.cuda.synchronize()
    assert torch.equal(o1[: t + 1], o2[: t + 1])
    assert torch.equal(l1[:, : t + 1], l2[:, : t + 1])
