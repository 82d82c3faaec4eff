"""Fused QKV projection with MXFP8 quantisation of K and V in its epilogue
(fapk_qkv_proj_mxfp8) against the oracle: the bf16 outputs within the
rounding of an fp32 product to bf16, K's and V's MX forms bit-exact against
the oracle's quantiser applied to the kernel's own bf16 K and V (a quantised
code is decided on the bf16 value on both sides), and the attention forward
over those forms bit-identical to the MXFP8 forward over the bf16 K and V."""
import numpy as np
import pytest
import torch

import oracle
from causal_flash_attention_packed_b200 import fapk, workloads as W
from gpu_util import f64, require_gpu

pytestmark = pytest.mark.gpu


def _inputs(lengths, d_model, Hq, Hkv, seed):
    g = torch.Generator().manual_seed(seed)
    T = int(sum(lengths))
    x = torch.randn((T, d_model), generator=g).to(torch.bfloat16)
    w = (torch.randn(((Hq + 2 * Hkv) * 128, d_model), generator=g) / d_model ** 0.5).to(torch.bfloat16)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return x, w, cu


@pytest.mark.parametrize("lengths,d_model", [([1, 31, 33, 127, 129, 300, 700], 512), ([200, 77, 1025], 200)])
def test_projection_and_forms(lengths, d_model):
    dev = require_gpu()
    Hq, Hkv = 4, 2
    x, w, cu = _inputs(lengths, d_model, Hq, Hkv, seed=90)
    seq = fapk.Seqlens(cu, dev)
    P = fapk.make_problem(seq, Hq, Hkv, 128, 128 ** -0.5, prec=fapk.MXFP8)
    ws = fapk.workspace(P, fapk.FWD, dev)
    q, k, v, kf, vf = fapk.qkv_proj_mxfp8(P, x.to(dev), w.to(dev), ws=ws)
    assert fapk.status(ws) == fapk.OK
    rq, rk, rv = oracle.qkv_proj(x.double().numpy(), w.double().numpy(), Hq, Hkv, 128)
    for name, got, ref in (("q", q, rq), ("k", k, rk), ("v", v, rv)):
        g = f64(got)
        # round to nearest of an fp32 sum: half a bf16 ulp (2^-9 relative),
        # plus the fp32 accumulation error of d_model products
        bound = 2.0 ** -8 * np.abs(ref) + 1e-4
        assert np.all(np.abs(g - ref) <= bound), f"{name}: worst excess {np.max(np.abs(g - ref) - bound):.3e}"
    n_slots = oracle.tb_slots(seq.T, seq.n_docs)
    slots = np.zeros(n_slots, bool)
    for kd in range(len(cu) - 1):
        s, e = cu[kd], cu[kd + 1]
        for m in range(0, e - s, 32):
            slots[s // 32 + kd + m // 32] = True
    for name, got_t, got_f in (("k", k, kf), ("v", v, vf)):
        ref = oracle.quantize_mxfp8(f64(got_t), cu)
        for key in ("val_tb", "val_pt", "scale_pt"):
            assert np.array_equal(got_f[key].cpu().numpy(), ref[key]), (name, key)
        assert np.array_equal(got_f["scale_tb"].cpu().numpy()[slots], ref["scale_tb"][slots]), (name, "scale_tb")
    # the attention forward over the epilogue's forms needs no quantisation of its own
    o1, l1 = fapk.attn_fwd_quantized_kv(P, q, kf, vf)
    o2, l2, _ = fapk.attn_fwd(P, q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("gk", [1.0, 0.4])
def test_projection_nvfp4_mixed(gk):
    """fapk_qkv_proj_nvfp4: the same projection with K's NVFP4 form (decode
    scale gk) in place of its MX forms, bit-exact against the oracle's NVFP4
    quantiser of the kernel's bf16 K; V's MX forms as above; the mixed path's
    forward over those forms bit-identical to its forward over the bf16 K, V."""
    dev = require_gpu()
    Hq, Hkv = 4, 2
    lengths, d_model = [1, 31, 33, 127, 129, 300, 700], 384
    x, w, cu = _inputs(lengths, d_model, Hq, Hkv, seed=91)
    seq = fapk.Seqlens(cu, dev)
    P = fapk.make_problem(seq, Hq, Hkv, 128, 128 ** -0.5, prec=fapk.NVFP4_MIXED, nv_scale_q=0.8, nv_scale_k=gk)
    ws = fapk.workspace(P, fapk.FWD, dev)
    q, k, v, (kc, ks), vf = fapk.qkv_proj_nvfp4(P, x.to(dev), w.to(dev), ws=ws)
    assert fapk.status(ws) == fapk.OK
    ec, es = oracle.quantize_nvfp4(f64(k), gk)
    assert np.array_equal(kc.cpu().numpy(), ec) and np.array_equal(ks.cpu().numpy(), es)
    ref = oracle.quantize_mxfp8(f64(v), cu)
    for key in ("val_tb", "val_pt", "scale_pt"):
        assert np.array_equal(vf[key].cpu().numpy(), ref[key]), key
    o1, l1 = fapk.attn_fwd_quantized_kv_nvfp4(P, q, (kc, ks), vf)
    o2, l2, _ = fapk.attn_fwd(P, q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
