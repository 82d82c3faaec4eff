"""Randomised parity cases: seeded document layouts (lengths from 0 to 700,
including zero-length and one-token documents and lengths next to the 16-,
32- and 128-token boundaries), head counts (MHA, GQA, MQA) and head dims
(64, 128), each run forward and backward through all three paths and checked
against the oracle: bf16 against exact fp64 (max-abs 2e-2, relative Frobenius
5e-3), MXFP8 and mixed NVFP4/FP8 against the oracle's emulation (relative
Frobenius 1e-2), LSE within 1e-3, every output finite."""
import numpy as np
import pytest
import torch

import oracle
from causal_flash_attention_packed_b200 import fapk, workloads as W
from gpu_util import check_close, f64, rel_frob, require_gpu, to_dev

pytestmark = pytest.mark.gpu

_EDGE = [0, 1, 2, 15, 16, 17, 31, 32, 33, 127, 128, 129]


def _case(seed):
    rng = np.random.default_rng(1000 + seed)
    n = int(rng.integers(1, 9))
    lengths = [int(rng.choice(_EDGE)) if rng.random() < 0.5 else int(rng.integers(0, 701)) for _ in range(n)]
    if sum(lengths) == 0:
        lengths.append(int(rng.integers(1, 300)))
    Hkv = int(rng.choice([1, 2]))
    G = int(rng.choice([1, 2, 4]))
    d = int(rng.choice([64, 128]))
    return W.custom(lengths, Hq=Hkv * G, Hkv=Hkv, d=d, seed=seed)


def _run(w, dev, prec):
    (q, k, v, do), (qd, kd, vd, dod) = to_dev(w, dev)
    seq = fapk.Seqlens(w.cu, dev)
    P = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale, prec=prec)
    o, lse, ctx = fapk.attn_fwd(P, qd, kd, vd)
    ws = fapk.workspace(P, fapk.BWD, dev)
    dq, dk, dv = fapk.attn_bwd(P, qd, kd, vd, o, lse, dod, ctx=ctx, ws=ws)
    torch.cuda.synchronize()
    assert fapk.status(ws) == fapk.OK
    return [t.double().numpy() for t in (q, k, v, do)], dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv)


@pytest.mark.parametrize("seed", range(32))
def test_random_layouts_all_paths(seed):
    dev = require_gpu()
    w = _case(seed)
    args, got = _run(w, dev, fapk.BF16)
    ex = oracle.attn_bwd(*args, w.cu, w.scale)
    for name in ("o", "dq", "dk", "dv"):
        check_close(f"bf16 {name}", f64(got[name]), ex[name])
    assert float(np.max(np.abs(f64(got["lse"]) - ex["lse"]))) <= 1e-3
    for prec, emu in ((fapk.MXFP8, oracle.mx_attn_bwd), (fapk.NVFP4_MIXED, oracle.nvmx_attn_bwd)):
        args, got = _run(w, dev, prec)
        em = emu(*args, w.cu, w.scale)
        for name in ("o", "dq", "dk", "dv"):
            g = f64(got[name])
            assert np.all(np.isfinite(g)), (prec, name)
            rf = rel_frob(g, em[name])
            assert rf <= 1e-2, f"{prec} {name}: rel_frob {rf:.3e} (lengths {np.diff(w.cu).tolist()})"
        assert float(np.max(np.abs(f64(got["lse"]) - em["lse"]))) <= 1e-3
