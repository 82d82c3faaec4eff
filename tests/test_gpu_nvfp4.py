"""Mixed NVFP4/FP8 path on the GPU (FLAMIA page, sec. "FLAMIA Mimarisi ve
Temel Tasarim Ilkeleri": mixed NVFP4/FP8 training paths; forward/backward
consistency; leak guards).

The scores take Q and K in NVFP4 in the forward and in the backward's
recomputation; everything else is the MXFP8 path.  Checks: the NVFP4
quantiser bit-exact against the oracle over every finite bf16 value; O, LSE,
dQ, dK, dV against the oracle's mixed emulation (relative Frobenius <= 1e-2,
the MXFP8 path's bar), with the cosine to exact fp64 no worse than the
emulation's by more than a small margin; and the leak tests T1/T2."""
import numpy as np
import pytest
import torch

import oracle
from causal_flash_attention_packed_b200 import fapk, workloads as W
from gpu_util import f64, rel_frob, require_gpu, to_dev

pytestmark = pytest.mark.gpu

NV_REL_FROB = 1e-2
LSE_ABS = 1e-3


def _cos(a, b):
    a, b = a.reshape(-1), b.reshape(-1)
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def _problem(w, dev, gq, gk):
    """(problem, seqlens): the caller keeps the Seqlens, which owns the device
    cu_seqlens the problem points to, alive while the problem is used."""
    seq = fapk.Seqlens(w.cu, dev)
    return fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale, prec=fapk.NVFP4_MIXED, nv_scale_q=gq,
                             nv_scale_k=gk), seq


def nv_fwd(w, dev, tensors=None, gq=1.0, gk=1.0):
    if tensors is None:
        (q, k, v, _), (qd, kd, vd, _) = to_dev(w, dev, with_dout=False)
    else:
        q, k, v = tensors[:3]
        qd, kd, vd = (t.to(dev) for t in (q, k, v))
    P, seq = _problem(w, dev, gq, gk)
    ws = fapk.workspace(P, fapk.FWD, dev)
    o = torch.full((w.T, w.Hq, w.d), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((w.Hq, w.T), float("nan"), dtype=torch.float32, device=dev)
    o, lse, ctx = fapk.attn_fwd(P, qd, kd, vd, o=o, lse=lse, ws=ws)
    assert fapk.status(ws) == fapk.OK
    return (q, k, v), o, lse


def nv_fwd_bwd(w, dev, tensors=None, gq=1.0, gk=1.0):
    if tensors is None:
        (q, k, v, do), (qd, kd, vd, dod) = to_dev(w, dev)
    else:
        q, k, v, do = tensors
        qd, kd, vd, dod = (t.to(dev) for t in tensors)
    P, seq = _problem(w, dev, gq, gk)
    o, lse, ctx = fapk.attn_fwd(P, qd, kd, vd)
    ws = fapk.workspace(P, fapk.BWD, dev)
    dq = torch.full((w.T, w.Hq, w.d), float("nan"), dtype=torch.float32, device=dev)
    dk = torch.full((w.T, w.Hkv, w.d), float("nan"), dtype=torch.float32, device=dev)
    dv = torch.full((w.T, w.Hkv, w.d), float("nan"), dtype=torch.float32, device=dev)
    fapk.attn_bwd(P, qd, kd, vd, o, lse, dod, ctx=ctx, dq=dq, dk=dk, dv=dv, ws=ws)
    assert fapk.status(ws) == fapk.OK
    return (q, k, v, do), (o, lse, dq, dk, dv)


# ---------------------------------------------------------------------------
# quantiser
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("g", [1.0, 0.37, 2.0 ** -20, 3.0e5])
def test_quantize_nvfp4_every_bf16_value(g):
    """Every finite bf16 bit pattern (infinities and NaNs replaced by zero), as
    a [512, 1, 128] tensor, and a random tensor with all-zero, tiny and loud
    blocks: codes and scale bytes bit-exact against the oracle."""
    dev = require_gpu()
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    x = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).reshape(512, 1, 128)
    x = torch.where(torch.isfinite(x.float()), x, torch.zeros_like(x))
    rng = np.random.default_rng(7)
    r = rng.standard_normal((96, 3, 128)) * np.exp(rng.uniform(-30, 30, (96, 3, 1)))
    r[5, 1, :16] = 0.0
    r[6, 2, 16:32] = -0.0
    r[7, 0, 32:48] = 1e-38
    y = torch.from_numpy(r).to(torch.bfloat16)
    for t in (x, y):
        codes, scales = fapk.quantize_nvfp4(t.to(dev), g)
        ec, es = oracle.quantize_nvfp4(t.double().numpy(), g)
        np.testing.assert_array_equal(codes.cpu().numpy(), ec)
        np.testing.assert_array_equal(scales.cpu().numpy(), es)


# ---------------------------------------------------------------------------
# forward
# ---------------------------------------------------------------------------

def _check(w, dev, gq=1.0, gk=1.0):
    (q, k, v), o, lse = nv_fwd(w, dev, gq=gq, gk=gk)
    qn, kn, vn = (t.double().numpy() for t in (q, k, v))
    eo, el = oracle.nvmx_attn_fwd(qn, kn, vn, w.cu, w.scale, gq=gq, gk=gk)
    go, gl = f64(o), f64(lse)
    assert np.all(np.isfinite(go)) and np.all(np.isfinite(gl))
    rf = rel_frob(go, eo)
    assert rf <= NV_REL_FROB, f"O rel_frob vs emulation {rf:.3e}"
    assert float(np.max(np.abs(gl - el))) <= LSE_ABS
    xo, _ = oracle.attn_fwd(qn, kn, vn, w.cu, w.scale)
    c_gpu, c_emu = _cos(go, xo), _cos(eo, xo)
    print(f"O: rel_frob vs emulation {rf:.2e}; cosine to exact: kernel {c_gpu:.5f}, emulation {c_emu:.5f}")
    assert c_gpu >= c_emu - 1e-3, f"cosine to exact: kernel {c_gpu:.5f}, emulation {c_emu:.5f}"


def test_single_tile_and_ragged_documents():
    """Lengths around the 16/32-token blocks and 128-token tile boundaries."""
    w = W.custom([1, 15, 16, 17, 31, 32, 33, 127, 128, 129, 300, 700], Hq=2, Hkv=2, d=128, seed=81)
    _check(w, require_gpu())


def test_gqa_and_decode_scales():
    """GQA (G = 2) with decode scales gq = 0.37, gk = 3.5 (applied to the
    scores in the softmax, not by the MMA)."""
    w = W.custom([513, 64, 1000], Hq=4, Hkv=2, d=128, seed=82)
    _check(w, require_gpu(), gq=0.37, gk=3.5)


@pytest.mark.parametrize("G", [1, 2])
def test_head_dim_64_ragged_documents(G):
    """d = 64: the NVFP4 rows keep 128 channels with a zero upper half (scale
    0), which adds nothing to the scores; against the emulation at d = 64."""
    w = W.custom([1, 15, 16, 17, 31, 32, 33, 127, 128, 129, 300, 700], Hq=2 * G, Hkv=2, d=64, seed=84)
    _check(w, require_gpu())


def test_outlier_channels_16k_full():
    """The 16384-token workload with x20 outlier channels, full size."""
    _check(W.config(3, 0), require_gpu())


@pytest.mark.parametrize("t_rel", [0, 13, 31, 100, 200])
def test_forward_leak_free(t_rel):
    """T1/T2: randomising Q, K, V after t leaves O and LSE at positions <= t
    bit-identical, at block-aligned and unaligned t."""
    dev = require_gpu()
    w = W.custom([300, 513, 200], Hq=2, Hkv=2, d=128, seed=83)
    q, k, v, _ = w.tensors(with_dout=False)
    t = 300 + t_rel
    _, o1, l1 = nv_fwd(w, dev, tensors=(q, k, v))
    g = torch.Generator().manual_seed(5)
    q2, k2, v2 = (x.clone() for x in (q, k, v))
    for x in (q2, k2, v2):
        x[t + 1:] = (torch.randn(x[t + 1:].shape, generator=g) * 30).to(x.dtype)
    _, o2, l2 = nv_fwd(w, dev, tensors=(q2, k2, v2))
    assert torch.equal(o1[: t + 1], o2[: t + 1])
    assert torch.equal(l1[:, : t + 1], l2[:, : t + 1])


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------

def _check_bwd(w, dev, gq=1.0, gk=1.0):
    (q, k, v, do), (o, lse, dq, dk, dv) = nv_fwd_bwd(w, dev, gq=gq, gk=gk)
    args = [t.double().numpy() for t in (q, k, v, do)]
    em = oracle.nvmx_attn_bwd(*args, w.cu, w.scale, gq=gq, gk=gk)
    ex = oracle.attn_bwd(*args, w.cu, w.scale)
    for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
        g = f64(got)
        assert np.all(np.isfinite(g)), name
        rf = rel_frob(g, em[name])
        c_gpu, c_emu = _cos(g, ex[name]), _cos(em[name], ex[name])
        print(f"{name}: rel_frob vs emulation {rf:.2e}; cosine to exact: kernel {c_gpu:.5f}, emulation {c_emu:.5f}")
        assert rf <= NV_REL_FROB, f"{name} rel_frob vs emulation {rf:.3e}"
        assert c_gpu >= c_emu - 2e-3, f"{name} cosine to exact: kernel {c_gpu:.5f}, emulation {c_emu:.5f}"


def test_bwd_ragged_documents():
    w = W.custom([1, 15, 16, 17, 31, 32, 33, 127, 128, 129, 300, 700], Hq=2, Hkv=2, d=128, seed=91)
    _check_bwd(w, require_gpu())


def test_bwd_gqa_and_decode_scales():
    w = W.custom([513, 64, 1000], Hq=4, Hkv=2, d=128, seed=92)
    _check_bwd(w, require_gpu(), gq=2.0, gk=0.3)


@pytest.mark.parametrize("G", [1, 2])
def test_bwd_head_dim_64_ragged_documents(G):
    w = W.custom([1, 15, 16, 17, 31, 32, 33, 127, 128, 129, 300, 700], Hq=2 * G, Hkv=2, d=64, seed=95)
    _check_bwd(w, require_gpu())


def test_bwd_outlier_channels_16k_full():
    _check_bwd(W.config(3, 0), require_gpu())


def _perturb(tensors, t, seed, zero_dout=False):
    """Q, K, V (and dO unless zero_dout) replaced by large random values after t."""
    g = torch.Generator().manual_seed(seed)
    out = [x.clone() for x in tensors]
    for i, x in enumerate(out):
        if i == 3 and zero_dout:
            x[t + 1:] = 0
        else:
            x[t + 1:] = (torch.randn(x[t + 1:].shape, generator=g) * 30).to(x.dtype)
    return tuple(out)


@pytest.mark.parametrize("t_rel", [0, 13, 31, 100, 200])
def test_bwd_dq_leak_free(t_rel):
    """T1/T2: randomising Q, K, V, dO after t leaves dQ at positions <= t
    bit-identical (any t), and dK, dV of earlier documents too."""
    dev = require_gpu()
    w = W.custom([300, 513, 200], Hq=2, Hkv=2, d=128, seed=93)
    base = w.tensors()
    t = 300 + t_rel
    _, a = nv_fwd_bwd(w, dev, tensors=base)
    _, b = nv_fwd_bwd(w, dev, tensors=_perturb(base, t, 9))
    assert torch.equal(a[2][: t + 1], b[2][: t + 1])
    assert torch.equal(a[3][:300], b[3][:300]) and torch.equal(a[4][:300], b[4][:300])


@pytest.mark.parametrize("t_rel", [31, 127, 255, 512])
def test_bwd_dkdv_leak_free_at_block_aligned_t(t_rel):
    """T3 at block-aligned t (t - s = 31 mod 32, or the document's last
    token): with dO = 0 after t in both runs, randomising Q, K, V after t
    leaves dK and dV at positions <= t bit-identical."""
    dev = require_gpu()
    w = W.custom([300, 513, 200], Hq=2, Hkv=2, d=128, seed=94)
    base = list(w.tensors())
    t = 300 + t_rel
    base[3][t + 1:] = 0
    _, a = nv_fwd_bwd(w, dev, tensors=tuple(base))
    _, b = nv_fwd_bwd(w, dev, tensors=_perturb(base, t, 10, zero_dout=True))
    assert torch.equal(a[3][: t + 1], b[3][: t + 1])
    assert torch.equal(a[4][: t + 1], b[4][: t + 1])


def _nv_sampled_docs(w, dev, max_tokens=6000, first_doc=0, kv_group=0):
    """Full-size workload in the launch configuration the benchmark uses; the
    oracle's mixed emulation reruns whole documents (every scale is per token
    or document-local, so a document's outputs depend on its own tokens only)
    for the query heads of one KV group: O, LSE, dQ, dK, dV of those documents
    and heads against the emulation."""
    (q, k, v, do), (o, lse, dq, dk, dv) = nv_fwd_bwd(w, dev)
    cu = w.cu
    k0 = k1 = first_doc
    while k1 < w.n_docs and cu[k1 + 1] - cu[k0] <= max_tokens:
        k1 += 1
    if k1 == k0:  # the first candidate alone is longer than the budget
        k1 = k0 + 1
    t0, t1 = int(cu[k0]), int(cu[k1])
    G = w.Hq // w.Hkv
    hs = list(range(kv_group * G, (kv_group + 1) * G))
    cu_s = (cu[k0:k1 + 1] - t0).astype(np.int32)
    sub_q = lambda x: x[t0:t1, hs].double().numpy()  # noqa: E731
    sub_k = lambda x: x[t0:t1, kv_group:kv_group + 1].double().numpy()  # noqa: E731
    em = oracle.nvmx_attn_bwd(sub_q(q), sub_k(k), sub_k(v), sub_q(do), cu_s, w.scale)
    res = {
        "o": rel_frob(f64(o)[t0:t1, hs], em["o"]),
        "dq": rel_frob(f64(dq)[t0:t1, hs], em["dq"]),
        "dk": rel_frob(f64(dk)[t0:t1, kv_group:kv_group + 1], em["dk"]),
        "dv": rel_frob(f64(dv)[t0:t1, kv_group:kv_group + 1], em["dv"]),
    }
    print(f"documents {k0}..{k1 - 1} ({t1 - t0} tokens), KV group {kv_group}: " +
          ", ".join(f"{n} {r:.2e}" for n, r in res.items()))
    for name, rf in res.items():
        assert rf <= NV_REL_FROB, f"{name} rel_frob vs emulation {rf:.3e} (documents {k0}..{k1 - 1})"
    assert float(np.max(np.abs(f64(lse)[hs, t0:t1] - em["lse"]))) <= LSE_ABS


@pytest.mark.parametrize("first_doc,max_tokens,kv_group", [(0, 6000, 0), (6, 13000, 9)])
def test_full_size_packed_32k_documents_vs_emulation(first_doc, max_tokens, kv_group):
    """The 32768-token benchmark workload (32 heads, 1% x8 outlier tokens):
    its first two documents (2322 and 1795 tokens), and its two longest
    (7545 and 5280 tokens, documents 6 and 7)."""
    _nv_sampled_docs(W.config(4, 0), require_gpu(), max_tokens=max_tokens, first_doc=first_doc,
                     kv_group=kv_group)


def test_full_size_gqa_128k_documents_vs_emulation():
    """131072 tokens with a 65536-token first document, 32 query heads on 8 KV
    heads; two documents after the long one, KV group 3."""
    _nv_sampled_docs(W.config(5, 0), require_gpu(), first_doc=4, kv_group=3)


def test_zero_length_and_one_token_documents():
    """Empty documents between others and one-token documents: the empty ones
    own no tile, the one-token ones are a single visible key."""
    w = W.custom([0, 1, 0, 0, 37, 1, 0, 200, 1, 0], Hq=2, Hkv=1, d=128, seed=96)
    _check_bwd(w, require_gpu())


def test_multi_query_attention_fwd_bwd():
    """MQA in the mixed path (Hkv = 1, eight query heads)."""
    w = W.custom([1, 129, 300, 700, 64], Hq=8, Hkv=1, d=128, seed=97)
    _check(w, require_gpu())
    _check_bwd(w, require_gpu())


def test_bf16_gradient_output():
    """grad_dtype = bf16 in the mixed path: the gradients are the fp32 ones
    rounded to bf16 (bit for bit)."""
    dev = require_gpu()
    w = W.custom([200, 513, 64], Hq=4, Hkv=2, d=128, seed=98)
    (q, k, v, do), (qd, kd, vd, dod) = to_dev(w, dev)
    seq = fapk.Seqlens(w.cu, dev)
    outs = []
    for gdt in (fapk.GRAD_F32, fapk.GRAD_BF16):
        P = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale, prec=fapk.NVFP4_MIXED, grad_dtype=gdt)
        o, lse, ctx = fapk.attn_fwd(P, qd, kd, vd)
        outs.append(fapk.attn_bwd(P, qd, kd, vd, o, lse, dod, ctx=ctx))
    torch.cuda.synchronize()
    for a, b in zip(*outs):
        assert b.dtype == torch.bfloat16
        assert torch.equal(a.to(torch.bfloat16), b)


def test_forward_from_quantised_kv_matches_the_mixed_forward():
    """fapk_attn_fwd_quantized_kv_nvfp4 over K quantised by fapk_quantize_nvfp4
    and V by fapk_quantize_mxfp8 (as a cache would hold them) gives O and LSE
    bit-identical to the mixed forward, twice over the same forms."""
    dev = require_gpu()
    w = W.custom([1, 129, 300, 700, 64], Hq=4, Hkv=2, d=128, seed=99)
    (q, k, v, _), (qd, kd, vd, _) = to_dev(w, dev, with_dout=False)
    P, seq = _problem(w, dev, 0.7, 1.3)
    kn = fapk.quantize_nvfp4(kd, 1.3)
    vf = fapk.quantize_mxfp8(vd, seq)
    o_ref, l_ref, _ = fapk.attn_fwd(P, qd, kd, vd)
    for _ in range(2):
        o, lse = fapk.attn_fwd_quantized_kv_nvfp4(P, qd, kn, vf)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
