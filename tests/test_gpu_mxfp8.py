"""MXFP8 path on the GPU against the oracle's MXFP8 emulation (relative
Frobenius <= 1e-2 for O), the cosine to exact fp64 next to the emulation's
own, and the leak tests.  The cosine >= 0.999 bar against exact fp64 is not
reachable by the quantisation rule itself on these inputs (the emulation
stays below it), so the test requires the kernel to be no further from exact
than the emulation plus a small margin."""
import numpy as np
import pytest
import torch

import oracle
from causal_flash_attention_packed_b200 import fapk, workloads as W
from gpu_util import f64, rel_frob, require_gpu, to_dev

pytestmark = pytest.mark.gpu

MX_REL_FROB = 1e-2
LSE_ABS = 1e-3


def _cos(a, b):
    a, b = a.reshape(-1), b.reshape(-1)
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def mx_fwd(w, dev, tensors=None, rule=fapk.SCALE_RCEIL):
    if tensors is None:
        (q, k, v, _), (qd, kd, vd, _) = to_dev(w, dev, with_dout=False)
    else:
        q, k, v = tensors[:3]
        qd, kd, vd = (t.to(dev) for t in (q, k, v))
    seq = fapk.Seqlens(w.cu, dev)
    P = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale, prec=fapk.MXFP8, scale_rule=rule)
    ws = fapk.workspace(P, fapk.FWD, dev)
    o = torch.full((w.T, w.Hq, w.d), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((w.Hq, w.T), float("nan"), dtype=torch.float32, device=dev)
    o, lse, ctx = fapk.attn_fwd(P, qd, kd, vd, o=o, lse=lse, ws=ws)
    assert fapk.status(ws) == fapk.OK
    return (q, k, v), o, lse


def _check(w, dev, rule=fapk.SCALE_RCEIL):
    (q, k, v), o, lse = mx_fwd(w, dev, rule=rule)
    qn, kn, vn = (t.double().numpy() for t in (q, k, v))
    flags = oracle.MX_QUANT_P | (oracle.MX_RULE_OCP if rule == fapk.SCALE_OCP else 0)
    eo, else_ = oracle.mx_attn_fwd(qn, kn, vn, w.cu, w.scale, flags=flags)
    go, gl = f64(o), f64(lse)
    assert np.all(np.isfinite(go)) and np.all(np.isfinite(gl))
    rf = rel_frob(go, eo)
    assert rf <= MX_REL_FROB, f"O rel_frob vs emulation {rf:.3e}"
    assert float(np.max(np.abs(gl - else_))) <= LSE_ABS
    xo, _ = oracle.attn_fwd(qn, kn, vn, w.cu, w.scale)
    c_gpu, c_emu = _cos(go, xo), _cos(eo, xo)
    assert c_gpu >= c_emu - 1e-3, f"cosine to exact: kernel {c_gpu:.5f}, emulation {c_emu:.5f}"
    return rf, c_gpu, c_emu


def test_single_tile_and_ragged_documents():
    """Lengths around the 32-token block and 128-token tile boundaries."""
    w = W.custom([1, 31, 32, 33, 127, 128, 129, 300, 700], Hq=2, Hkv=2, d=128, seed=61)
    _check(w, require_gpu())


def test_gqa():
    w = W.custom([513, 64, 1000], Hq=4, Hkv=2, d=128, seed=62)
    _check(w, require_gpu())


@pytest.mark.parametrize("G", [1, 2])
def test_head_dim_64_ragged_documents(G):
    """d = 64: the MX forms keep 128 codes per row with a zero upper half, which
    changes no real block's scale; against the emulation at d = 64."""
    w = W.custom([1, 31, 32, 33, 127, 128, 129, 300, 700], Hq=2 * G, Hkv=2, d=64, seed=64)
    _check(w, require_gpu())


def test_outlier_channels_16k_full():
    """The 16384-token MXFP8 workload (x20 outlier channels), full size."""
    _check(W.config(3, 0), require_gpu())


@pytest.mark.parametrize("t_rel", [0, 13, 31, 100, 200])
def test_forward_leak_free(t_rel):
    """T1/T2 on the MXFP8 forward: randomising Q, K, V after t leaves O and LSE
    at positions <= t bit-identical, at block-aligned and unaligned t."""
    dev = require_gpu()
    w = W.custom([300, 513, 200], Hq=2, Hkv=2, d=128, seed=63)
    q, k, v, _ = w.tensors(with_dout=False)
    t = 300 + t_rel
    _, o1, l1 = mx_fwd(w, dev, tensors=(q, k, v))
    g = torch.Generator().manual_seed(5)
    q2, k2, v2 = (x.clone() for x in (q, k, v))
    for x in (q2, k2, v2):
        x[t + 1:] = (torch.randn(x[t + 1:].shape, generator=g) * 30).to(x.dtype)
    _, o2, l2 = mx_fwd(w, dev, tensors=(q2, k2, v2))
    assert torch.equal(o1[: t + 1], o2[: t + 1])
    assert torch.equal(l1[:, : t + 1], l2[:, : t + 1])


def mx_fwd_bwd(w, dev, tensors=None, rule=fapk.SCALE_RCEIL):
    if tensors is None:
        (q, k, v, do), (qd, kd, vd, dod) = to_dev(w, dev)
    else:
        q, k, v, do = tensors
        qd, kd, vd, dod = (t.to(dev) for t in tensors)
    seq = fapk.Seqlens(w.cu, dev)
    P = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale, prec=fapk.MXFP8, scale_rule=rule)
    o, lse, ctx = fapk.attn_fwd(P, qd, kd, vd)
    ws = fapk.workspace(P, fapk.BWD, dev)
    dq = torch.full((w.T, w.Hq, w.d), float("nan"), dtype=torch.float32, device=dev)
    dk = torch.full((w.T, w.Hkv, w.d), float("nan"), dtype=torch.float32, device=dev)
    dv = torch.full((w.T, w.Hkv, w.d), float("nan"), dtype=torch.float32, device=dev)
    fapk.attn_bwd(P, qd, kd, vd, o, lse, dod, ctx=ctx, dq=dq, dk=dk, dv=dv, ws=ws)
    assert fapk.status(ws) == fapk.OK
    return (q, k, v, do), (o, lse, dq, dk, dv)


def _check_bwd(w, dev):
    (q, k, v, do), (o, lse, dq, dk, dv) = mx_fwd_bwd(w, dev)
    bar = MX_REL_FROB
    args = [t.double().numpy() for t in (q, k, v, do)]
    em = oracle.mx_attn_bwd(*args, w.cu, w.scale, flags=oracle.MX_QUANT_P)
    ex = oracle.attn_bwd(*args, w.cu, w.scale)
    out = {}
    for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
        g = f64(got)
        assert np.all(np.isfinite(g)), name
        rf = rel_frob(g, em[name])
        c_gpu, c_emu = _cos(g, ex[name]), _cos(em[name], ex[name])
        out[name] = (rf, c_gpu, c_emu)
        assert rf <= bar, f"{name} rel_frob vs emulation {rf:.3e}"
        assert c_gpu >= c_emu - 2e-3, f"{name} cosine to exact: kernel {c_gpu:.5f}, emulation {c_emu:.5f}"
    return out


def test_bwd_ragged_documents():
    w = W.custom([1, 31, 32, 33, 127, 128, 129, 300, 700], Hq=2, Hkv=2, d=128, seed=71)
    _check_bwd(w, require_gpu())


def test_bwd_gqa():
    w = W.custom([513, 64, 1000], Hq=4, Hkv=2, d=128, seed=72)
    _check_bwd(w, require_gpu())


@pytest.mark.parametrize("G", [1, 2])
def test_bwd_head_dim_64_ragged_documents(G):
    w = W.custom([1, 31, 32, 33, 127, 128, 129, 300, 700], Hq=2 * G, Hkv=2, d=64, seed=75)
    _check_bwd(w, require_gpu())


@pytest.mark.parametrize("t_rel", [13, 31, 200])
def test_head_dim_64_leak_free(t_rel):
    """T1/T2 at d = 64: O, LSE and dQ at positions <= t are bit-identical when
    everything after t is randomised."""
    dev = require_gpu()
    w = W.custom([300, 513, 200], Hq=2, Hkv=2, d=64, seed=76)
    base = w.tensors()
    t = 300 + t_rel
    _, a = mx_fwd_bwd(w, dev, tensors=base)
    _, b = mx_fwd_bwd(w, dev, tensors=_perturb(base, t, 11))
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x[: t + 1] if x.dim() == 3 else x[:, : t + 1], y[: t + 1] if y.dim() == 3 else y[:, : t + 1])


def test_bwd_outlier_channels_16k_full():
    """The 16384-token MXFP8 workload, full size, every gradient element."""
    _check_bwd(W.config(3, 0), require_gpu())


def _perturb(tensors, t, seed, zero_dout=False):
    g = torch.Generator().manual_seed(seed)
    out = []
    for idx, x in enumerate(tensors):
        y = x.clone()
        if idx == 3 and zero_dout:
            y[t + 1:] = 0
        else:
            y[t + 1:] = (torch.randn(y[t + 1:].shape, generator=g) * 30).to(y.dtype)
        out.append(y)
    return out


@pytest.mark.parametrize("t_rel", [0, 13, 31, 100, 200])
def test_bwd_dq_leak_free(t_rel):
    """T1/T2: randomising Q, K, V, dO after t leaves dQ at positions <= t
    bit-identical (any t), and dK, dV of earlier documents too."""
    dev = require_gpu()
    w = W.custom([300, 513, 200], Hq=2, Hkv=2, d=128, seed=73)
    base = w.tensors()
    t = 300 + t_rel
    _, a = mx_fwd_bwd(w, dev, tensors=base)
    _, b = mx_fwd_bwd(w, dev, tensors=_perturb(base, t, 9))
    assert torch.equal(a[2][: t + 1], b[2][: t + 1])
    assert torch.equal(a[3][:300], b[3][:300]) and torch.equal(a[4][:300], b[4][:300])


@pytest.mark.parametrize("t_rel", [31, 127, 255, 512])
def test_bwd_dkdv_leak_free_at_block_aligned_t(t_rel):
    """T3 at block-aligned t (t - s = 31 mod 32, or the document's last
    token): with dO = 0 after t in both runs, randomising Q, K, V after t
    leaves dK and dV at positions <= t bit-identical."""
    dev = require_gpu()
    w = W.custom([300, 513, 200], Hq=2, Hkv=2, d=128, seed=74)
    base = list(w.tensors())
    t = 300 + t_rel
    base[3][t + 1:] = 0
    _, a = mx_fwd_bwd(w, dev, tensors=base)
    _, b = mx_fwd_bwd(w, dev, tensors=_perturb(base, t, 10, zero_dout=True))
    assert torch.equal(a[3][: t + 1], b[3][: t + 1])
    assert torch.equal(a[4][: t + 1], b[4][: t + 1])


def _mx_sampled_docs(w, dev, max_tokens=6000, first_doc=0, kv_group=0):
    """Full-size workload in the launch configuration the benchmark uses; the
    oracle's MXFP8 emulation reruns whole documents (the scales are
    document-local, so a document's outputs depend on its own tokens only)
    for the query heads of one KV group: O, LSE, dQ, dK, dV of those
    documents and heads against the emulation."""
    (q, k, v, do), (o, lse, dq, dk, dv) = mx_fwd_bwd(w, dev)
    cu = w.cu
    lengths = np.diff(cu)
    k0 = first_doc
    k1 = k0
    while k1 < w.n_docs and cu[k1 + 1] - cu[k0] <= max_tokens:
        k1 += 1
    if k1 == k0:  # the first candidate alone is longer than the budget
        k1 = k0 + 1
    t0, t1 = int(cu[k0]), int(cu[k1])
    assert t1 > t0 and lengths[k0:k1].min() >= 0
    G = w.Hq // w.Hkv
    hs = list(range(kv_group * G, (kv_group + 1) * G))
    cu_s = (cu[k0:k1 + 1] - t0).astype(np.int32)
    sub_q = lambda x: x[t0:t1, hs].double().numpy()
    sub_k = lambda x: x[t0:t1, kv_group:kv_group + 1].double().numpy()
    em_o, em_l = oracle.mx_attn_fwd(sub_q(q), sub_k(k), sub_k(v), cu_s, w.scale, flags=oracle.MX_QUANT_P)
    em = oracle.mx_attn_bwd(sub_q(q), sub_k(k), sub_k(v), sub_q(do), cu_s, w.scale, flags=oracle.MX_QUANT_P)
    res = {
        "o": rel_frob(f64(o)[t0:t1, hs], em_o),
        "dq": rel_frob(f64(dq)[t0:t1, hs], em["dq"]),
        "dk": rel_frob(f64(dk)[t0:t1, kv_group:kv_group + 1], em["dk"]),
        "dv": rel_frob(f64(dv)[t0:t1, kv_group:kv_group + 1], em["dv"]),
    }
    for name, rf in res.items():
        assert rf <= MX_REL_FROB, f"{name} rel_frob vs emulation {rf:.3e} (documents {k0}..{k1 - 1})"
    assert float(np.max(np.abs(f64(lse)[hs, t0:t1] - em_l))) <= LSE_ABS
    return res


@pytest.mark.parametrize("first_doc,max_tokens,kv_group", [(0, 6000, 0), (6, 13000, 9)])
def test_full_size_packed_32k_documents_vs_emulation(first_doc, max_tokens, kv_group):
    """The 32768-token benchmark workload (32 heads, 1% x8 outlier tokens):
    its first two documents (2322 and 1795 tokens), and its two longest
    (7545 and 5280 tokens, documents 6 and 7)."""
    _mx_sampled_docs(W.config(4, 0), require_gpu(), max_tokens=max_tokens, first_doc=first_doc,
                     kv_group=kv_group)


def test_full_size_gqa_128k_documents_vs_emulation():
    """131072 tokens with a 65536-token first document, 32 query heads on 8 KV
    heads; two documents after the long one, KV group 3."""
    _mx_sampled_docs(W.config(5, 0), require_gpu(), first_doc=4, kv_group=3)


@pytest.mark.parametrize("t_rel", [13, 100, 200])
def test_bwd_dkdv_at_unaligned_t_measured(t_rel):
    """T3 at a t that is not the end of a 32-token block (the reading of the
    leak test that the quantisation rule cannot meet bit for bit): the query
    block holding t shares one Q~tb scale (and one P~T / dS~T scale per key)
    with the randomised queries after t, so dK and dV at positions <= t may
    move by range effects (values that turn subnormal or flush).  The oracle's
    emulation measures 40 to 2347 of 0.8e5 to 1.9e5 dK elements moving, by at
    most 7.4e-4 of the RMS of dK, and no dV element.  The kernel must stay
    within 2e-3 of the RMS; the counts are printed."""
    dev = require_gpu()
    w = W.custom([300, 513, 200], Hq=2, Hkv=2, d=128, seed=74)
    base = list(w.tensors())
    t = 300 + t_rel
    base[3][t + 1:] = 0
    _, a = mx_fwd_bwd(w, dev, tensors=base)
    _, b = mx_fwd_bwd(w, dev, tensors=_perturb(base, t, 10, zero_dout=True))
    for name, x, y in (("dk", a[3], b[3]), ("dv", a[4], b[4])):
        x, y = f64(x[: t + 1]), f64(y[: t + 1])
        n = int(np.count_nonzero(x != y))
        rel = float(np.max(np.abs(x - y)) / np.sqrt(np.mean(x * x)))
        print(f"T3 t_rel={t_rel} {name}: {n} of {x.size} elements differ, max diff {rel:.2e} of RMS")
        assert rel <= 2e-3, (name, n, rel)


def test_forward_from_quantised_kv_matches_the_mxfp8_forward():
    """fapk_attn_fwd_quantized_kv: K and V quantised once by fapk_quantize_mxfp8
    (as a quantised KV cache would hold them) and reused by two calls with
    different Q; each call's O and LSE are bit-identical to the MXFP8 forward
    on the bf16 K and V, and within the bar of the oracle's emulation."""
    dev = require_gpu()
    w = W.custom([1, 31, 33, 127, 129, 300, 700], Hq=4, Hkv=2, d=128, seed=77)
    (q, k, v, _), (qd, kd, vd, _) = to_dev(w, dev, with_dout=False)
    seq = fapk.Seqlens(w.cu, dev)
    P = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale, prec=fapk.MXFP8)
    kf = fapk.quantize_mxfp8(kd, seq)
    vf = fapk.quantize_mxfp8(vd, seq)
    g = torch.Generator().manual_seed(78)
    q2 = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    for qq in (q, q2):
        qqd = qq.to(dev)
        o1, l1 = fapk.attn_fwd_quantized_kv(P, qqd, kf, vf)
        o2, l2, _ = fapk.attn_fwd(P, qqd, kd, vd)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
        eo, _ = oracle.mx_attn_fwd(qq.double().numpy(), k.double().numpy(), v.double().numpy(), w.cu, w.scale)
        assert rel_frob(f64(o1), eo) <= MX_REL_FROB


def test_multi_query_attention_fwd_bwd():
    """MQA in the MXFP8 path (Hkv = 1, eight query heads)."""
    w = W.custom([1, 129, 300, 700, 64], Hq=8, Hkv=1, d=128, seed=79)
    _check(w, require_gpu())
    _check_bwd(w, require_gpu())


def test_zero_length_and_one_token_documents():
    """Zero-length documents produce nothing and one-token documents attend to
    themselves only (O = their own V~): forward and backward against the
    emulation, with every other output finite."""
    w = W.custom([0, 1, 40, 0, 0, 1, 257, 1, 0], Hq=2, Hkv=1, d=128, seed=80)
    _check(w, require_gpu())
    _check_bwd(w, require_gpu())


def test_bf16_gradient_output():
    """grad_dtype = bf16 in the MXFP8 path: the gradients are the fp32 ones
    rounded to bf16 (within half a bf16 ulp of the fp32-output run)."""
    dev = require_gpu()
    w = W.custom([200, 513, 64], Hq=4, Hkv=2, d=128, seed=81)
    (q, k, v, do), (qd, kd, vd, dod) = to_dev(w, dev)
    seq = fapk.Seqlens(w.cu, dev)
    outs = []
    for gdt in (fapk.GRAD_F32, fapk.GRAD_BF16):
        P = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale, prec=fapk.MXFP8, grad_dtype=gdt)
        o, lse, ctx = fapk.attn_fwd(P, qd, kd, vd)
        outs.append(fapk.attn_bwd(P, qd, kd, vd, o, lse, dod, ctx=ctx))
    torch.cuda.synchronize()
    for a, b in zip(*outs):
        assert b.dtype == torch.bfloat16
        assert torch.equal(a.to(torch.bfloat16), b)
