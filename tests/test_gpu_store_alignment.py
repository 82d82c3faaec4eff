"""Output buffers that are 16-byte but not 32-byte aligned: the kernels then
write O, dQ, dK and dV with 16-byte stores instead of 32-byte ones.  Both store
forms carry the same values, so the results must match the aligned call bit for
bit (both paths, both gradient dtypes, d = 64 and 128, ragged documents)."""
import pytest
import torch

from causal_flash_attention_packed_b200 import fapk, workloads as W
from gpu_util import require_gpu, to_dev

pytestmark = pytest.mark.gpu


def _offset_empty(shape, dtype, dev):
    """A tensor of `shape` whose data starts 16 bytes past a 256-byte boundary."""
    n = 1
    for s in shape:
        n *= s
    pad = 16 // torch.empty((), dtype=dtype).element_size()
    flat = torch.full((n + pad,), float("nan"), dtype=dtype, device=dev)
    t = flat[pad:].view(shape)
    assert t.data_ptr() % 32 == 16
    return t


@pytest.mark.parametrize("prec,d,grad_dtype", [(fapk.BF16, 128, fapk.GRAD_F32), (fapk.BF16, 64, fapk.GRAD_BF16),
                                               (fapk.MXFP8, 128, fapk.GRAD_F32)])
def test_unaligned_outputs_match_aligned(prec, d, grad_dtype):
    dev = require_gpu()
    w = W.custom([700, 129, 1000], Hq=4, Hkv=2, d=d, seed=57)
    _, (qd, kd, vd, dod) = to_dev(w, dev)
    seq = fapk.Seqlens(w.cu, dev)
    P = fapk.make_problem(seq, w.Hq, w.Hkv, w.d, w.scale, prec=prec, grad_dtype=grad_dtype)
    gdt = torch.float32 if grad_dtype == fapk.GRAD_F32 else torch.bfloat16

    o, lse, ctx = fapk.attn_fwd(P, qd, kd, vd)
    dq, dk, dv = fapk.attn_bwd(P, qd, kd, vd, o, lse, dod, ctx=ctx)

    o2 = _offset_empty((w.T, w.Hq, d), torch.bfloat16, dev)
    o2, lse2, ctx2 = fapk.attn_fwd(P, qd, kd, vd, o=o2)
    dq2 = _offset_empty((w.T, w.Hq, d), gdt, dev)
    dk2 = _offset_empty((w.T, w.Hkv, d), gdt, dev)
    dv2 = _offset_empty((w.T, w.Hkv, d), gdt, dev)
    fapk.attn_bwd(P, qd, kd, vd, o2, lse2, dod, ctx=ctx2, dq=dq2, dk=dk2, dv=dv2)
    torch.cuda.synchronize()
    for name, a, b in (("O", o, o2), ("LSE", lse, lse2), ("dQ", dq, dq2), ("dK", dk, dk2), ("dV", dv, dv2)):
        assert torch.equal(a.view(torch.int16 if a.element_size() == 2 else torch.int32),
                           b.view(torch.int16 if b.element_size() == 2 else torch.int32)), name
