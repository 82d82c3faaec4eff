"""bf16 backward on the GPU against the exact fp64 oracle (dQ, dK, dV), the
leak tests T1-T3 and bitwise determinism."""
import numpy as np
import pytest
import torch

import oracle
from causal_flash_attention_packed_b200 import fapk, workloads as W
from gpu_util import check_close, f64, require_gpu, to_dev

pytestmark = pytest.mark.gpu


def run_fwd_bwd(w, dev, grad_dtype=fapk.GRAD_F32, tensors=None):
    if tensors is None:
        (q, k, v, do), (qd, kd, vd, dod) = to_dev(w, dev)
    else:
        q, k, v, do = tensors
        qd, kd, vd, dod = (t.to(dev) for t in tensors)
    seq = fapk.Seqlens(w.cu, dev)
    P = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale, grad_dtype=grad_dtype)
    o, lse, ctx = fapk.attn_fwd(P, qd, kd, vd)
    ws = fapk.workspace(P, fapk.BWD, dev)
    gdt = torch.float32 if grad_dtype == fapk.GRAD_F32 else torch.bfloat16
    dq = torch.full((w.T, w.Hq, w.d), float("nan"), dtype=gdt, device=dev)
    dk = torch.full((w.T, w.Hkv, w.d), float("nan"), dtype=gdt, device=dev)
    dv = torch.full((w.T, w.Hkv, w.d), float("nan"), dtype=gdt, device=dev)
    fapk.attn_bwd(P, qd, kd, vd, o, lse, dod, ctx=ctx, dq=dq, dk=dk, dv=dv, ws=ws)
    assert fapk.status(ws) == fapk.OK
    return (q, k, v, do), (o, lse, dq, dk, dv)


def _full_check(w, dev, grad_dtype=fapk.GRAD_F32):
    (q, k, v, do), (o, lse, dq, dk, dv) = run_fwd_bwd(w, dev, grad_dtype)
    ref = oracle.attn_bwd(*(t.double().numpy() for t in (q, k, v, do)), w.cu, w.scale)
    out = {}
    if grad_dtype == fapk.GRAD_F32:
        for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
            out[name] = check_close(name, f64(got), ref[name])
    else:
        # bf16 gradients: rounding to bf16 alone costs up to half an ulp,
        # 2^-9 relative; the relative-Frobenius bar still applies
        for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
            g = f64(got)
            out[name] = check_close(name, g, ref[name], max_abs=2e-2 + 2.0 ** -8 * np.abs(ref[name]).max())
    return out


def test_single_document_d64():
    _full_check(W.config(1, 0), require_gpu())


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [1, 4])
def test_ragged_documents(d, G):
    lengths = [1, 127, 128, 0, 129, 255, 256, 257, 300, 700, 5]
    _full_check(W.custom(lengths, Hq=2 * G, Hkv=2, d=d, seed=21), require_gpu())


def test_bf16_gradients():
    _full_check(W.custom([200, 513, 64], Hq=4, Hkv=2, d=128, seed=22), require_gpu(), fapk.GRAD_BF16)


def test_packed_8k_full():
    """8192 packed tokens, 16 heads, d = 128, every output against the full
    oracle."""
    _full_check(W.config(2, 0), require_gpu())


def _sampled_check(w, dev, n_rows=96, n_cols=24, seed=0, long_doc=None):
    """Full-size workload in the launch configuration the benchmark uses;
    the oracle computes sampled rows (O, LSE, dQ) and sampled keys (dK, dV) one
    by one.  Keys are drawn near document ends, where the exact dK/dV needs few
    query rows, and, with `long_doc` = (document, KV head, doc-local key
    positions), at the start of a long document, where every later query of
    every query head of the group adds to them (the longest accumulations)."""
    (q, k, v, do), (o, lse, dq, dk, dv) = run_fwd_bwd(w, dev)
    if long_doc is not None:
        _long_doc_keys(w, (q, k, v, do), dk, dv, *long_doc)
    rng = np.random.default_rng(seed)
    cu = w.cu
    tok = rng.integers(0, w.T, n_rows)
    head = rng.integers(0, w.Hq, n_rows)
    qn, kn, vn, don = (t.double().numpy() for t in (q, k, v, do))
    ro, rl, rdq = oracle.attn_rows(qn, kn, vn, don, cu, w.scale, tok, head)
    check_close("O", f64(o)[tok, head], ro)
    assert np.max(np.abs(f64(lse)[head, tok] - rl)) <= 1e-3
    check_close("dQ", f64(dq)[tok, head], rdq)
    docs = rng.integers(0, w.n_docs, n_cols)
    docs = docs[np.diff(cu)[docs] > 0]
    ends = cu[docs + 1]
    ktok = ends - 1 - rng.integers(0, 48, len(docs))
    ktok = np.maximum(ktok, cu[docs])
    kvh = rng.integers(0, w.Hkv, len(docs))
    rdk, rdv = oracle.attn_kv_cols(qn, kn, vn, don, cu, w.scale, ktok, kvh)
    check_close("dK", f64(dk)[ktok, kvh], rdk)
    check_close("dV", f64(dv)[ktok, kvh], rdv)


def _long_doc_keys(w, tensors, dk, dv, doc, kv_head, key_locals):
    """dK, dV of keys of one document and KV head against the oracle: the
    exact forward rows (O, LSE) of every query of the document for the group's
    query heads, then each key's sums over all queries after it."""
    q, k, v, do = tensors
    s, e = int(w.cu[doc]), int(w.cu[doc + 1])
    G = w.Hq // w.Hkv
    hq = slice(kv_head * G, (kv_head + 1) * G)
    qs, dos = (x[s:e, hq].double().numpy() for x in (q, do))
    ks, vs = (x[s:e, kv_head:kv_head + 1].double().numpy() for x in (k, v))
    cu_s = np.array([0, e - s], np.int32)
    o_s = np.zeros_like(qs)
    lse_s = np.zeros((G, e - s))
    for h in range(G):
        o_s[:, h], lse_s[h] = oracle.attn_fwd_doc(qs, ks, vs, cu_s, w.scale, 0, h)
    tok = np.asarray(key_locals, dtype=np.int32)
    rdk, rdv = oracle.attn_kv_cols_from_rows(qs, ks, vs, dos, o_s, lse_s, cu_s, w.scale, tok,
                                             np.zeros_like(tok))
    check_close("dK (long document)", f64(dk)[s + tok, kv_head], rdk)
    check_close("dV (long document)", f64(dv)[s + tok, kv_head], rdv)


def test_full_size_packed_32k_sampled():
    """32768 tokens, log-normal lengths, 32 heads (the benchmark workload);
    plus 16 keys in the first 256 tokens of its longest document (7545
    tokens), KV head 5."""
    w = W.config(4, 0)
    doc = int(np.argmax(np.diff(w.cu)))
    keys = np.random.default_rng(3).choice(256, 16, replace=False)
    _sampled_check(w, require_gpu(), long_doc=(doc, 5, keys))


def test_full_size_gqa_128k_sampled():
    """131072 tokens with a 65536-token document, 32 query heads on 8 KV heads;
    plus 3 keys at the start of the 65536-token document (KV head 1, so the
    sums run over 4 query heads x up to 65536 queries)."""
    _sampled_check(W.config(5, 0), require_gpu(), n_rows=48, n_cols=12, long_doc=(0, 1, [0, 37, 300]))


def test_deterministic():
    dev = require_gpu()
    w = W.custom([700, 33, 1200], Hq=4, Hkv=2, d=128, seed=5)
    _, a = run_fwd_bwd(w, dev)
    _, b = run_fwd_bwd(w, dev)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def _perturbed(tensors, t, seed, keep_dout_zero=False):
    g = torch.Generator().manual_seed(seed)
    out = []
    for idx, x in enumerate(tensors):
        y = x.clone()
        if idx == 3 and keep_dout_zero:
            y[t + 1:] = 0
        else:
            y[t + 1:] = torch.randn(y[t + 1:].shape, generator=g).to(y.dtype)
        out.append(y)
    return out


@pytest.mark.parametrize("t_rel", [0, 13, 127, 128, 200, 385])
def test_leak_T1_T2(t_rel):
    """Randomising Q, K, V, dO at every position after t (the rest of t's
    document and all later documents) leaves O, LSE and dQ at positions <= t
    bit-identical; at t = the end of a document, dK and dV of earlier documents
    are bit-identical too (T1)."""
    dev = require_gpu()
    lengths = [300, 513, 200]
    w = W.custom(lengths, Hq=4, Hkv=2, d=128, seed=31)
    base = w.tensors()
    t = 300 + t_rel
    _, a = run_fwd_bwd(w, dev, tensors=base)
    _, b = run_fwd_bwd(w, dev, tensors=_perturbed(base, t, 7))
    o1, l1, dq1, dk1, dv1 = a
    o2, l2, dq2, dk2, dv2 = b
    assert torch.equal(o1[: t + 1], o2[: t + 1])
    assert torch.equal(l1[:, : t + 1], l2[:, : t + 1])
    assert torch.equal(dq1[: t + 1], dq2[: t + 1])
    assert torch.equal(dk1[:300], dk2[:300]) and torch.equal(dv1[:300], dv2[:300])


@pytest.mark.parametrize("t_rel", [0, 13, 127, 128, 200, 385, 512])
def test_leak_T3(t_rel):
    """With dO = 0 after t in both runs, randomising Q, K, V after t leaves dK
    and dV at positions <= t bit-identical (bf16 path: any t)."""
    dev = require_gpu()
    w = W.custom([300, 513, 200], Hq=4, Hkv=2, d=128, seed=32)
    base = list(w.tensors())
    t = 300 + t_rel
    base[3][t + 1:] = 0
    _, a = run_fwd_bwd(w, dev, tensors=base)
    _, b = run_fwd_bwd(w, dev, tensors=_perturbed(base, t, 8, keep_dout_zero=True))
    assert torch.equal(a[3][: t + 1], b[3][: t + 1])
    assert torch.equal(a[4][: t + 1], b[4][: t + 1])


@pytest.mark.parametrize("d", [64, 128])
def test_multi_query_attention(d):
    """MQA: every query head reads the one KV head (Hkv = 1), so dK and dV sum
    over all eight query heads; full outputs against the oracle."""
    _full_check(W.custom([1, 129, 300, 700, 64], Hq=8, Hkv=1, d=d, seed=23), require_gpu())
