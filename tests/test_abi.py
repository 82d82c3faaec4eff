"""C-ABI checks that need no GPU: the library loads, exports every entry point
declared in include/fapk.h, and rejects bad arguments on the host before
anything is launched."""
import ctypes
import os
import re

import numpy as np
import pytest

from causal_flash_attention_packed_b200 import build, fapk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return fapk.lib()


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "fapk.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fapk_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    syms = _declared_symbols()
    assert {"fapk_attn_fwd", "fapk_attn_bwd", "fapk_quantize_mxfp8"} <= set(syms)
    for s in syms:
        assert hasattr(L, s), s


def test_strerror_and_version(L):
    for code in range(8):
        assert fapk.strerror(code)
    assert "unknown" in fapk.strerror(99)
    assert L.fapk_version() >= 100


def _problem(**kw):
    seq = type("S", (), {})()
    P = fapk.Problem()
    P.T, P.n_docs, P.max_seqlen, P.Hq, P.Hkv, P.d = 300, 2, 200, 4, 2, 128
    P.scale = 0.088
    P.prec = fapk.BF16
    P.scale_rule = fapk.SCALE_RCEIL
    P.cu_seqlens_dev = 0x1000
    P.cu_seqlens_host = None
    P.grad_dtype = fapk.GRAD_F32
    P.flags = 0
    P.timeout_ms = 0
    for k, v in kw.items():
        setattr(P, k, v)
    return P


def test_workspace_size(L):
    P = _problem()
    fwd = fapk.workspace_size(P, fapk.FWD)
    bwd = fapk.workspace_size(P, fapk.BWD)
    assert fwd > 0 and bwd >= 4 * 300 * 4  # bwd holds D = rowsum(dO*O) in fp32 [Hq][T]
    # ctx: O residual (bf16, T*Hq*d) + fp16 V (T*Hkv*d)
    assert fapk.ctx_size(P) >= 2 * 300 * 128 * (4 + 2)
    assert fwd % 256 == 0 and bwd % 256 == 0
    assert fapk.workspace_size(_problem(d=96), fapk.FWD) == 0
    assert fapk.workspace_size(P, 7) == 0


def _fwd(L, P, ws_bytes=1 << 30, ptrs=(16, 16, 16, 16, 16), ws=256, ctx=4096):
    return L.fapk_attn_fwd(ctypes.byref(P), *ptrs, ctx, ws, ws_bytes, None)


def test_host_validation_codes(L):
    """Every error below is detected on the host, before any CUDA call."""
    assert _fwd(L, _problem(d=96)) == fapk.ERR_UNSUPPORTED
    assert _fwd(L, _problem(Hq=3, Hkv=2)) == fapk.ERR_UNSUPPORTED
    assert _fwd(L, _problem(prec=7)) == fapk.ERR_UNSUPPORTED
    assert _fwd(L, _problem(prec=fapk.MXFP8, scale_rule=fapk.SCALE_OCP)) == fapk.ERR_UNSUPPORTED
    assert _fwd(L, _problem(prec=fapk.MXFP8, scale_rule=7)) == fapk.ERR_UNSUPPORTED
    assert _fwd(L, _problem(Hq=0)) == fapk.ERR_INVALID_ARG
    assert _fwd(L, _problem(T=-1)) == fapk.ERR_INVALID_ARG
    assert _fwd(L, _problem(max_seqlen=0)) == fapk.ERR_INVALID_ARG
    assert _fwd(L, _problem(cu_seqlens_dev=None)) == fapk.ERR_INVALID_ARG
    assert _fwd(L, _problem(), ptrs=(16, None, 16, 16, 16)) == fapk.ERR_INVALID_ARG
    assert _fwd(L, _problem(), ptrs=(16, 24, 16, 16, 16)) == fapk.ERR_INVALID_ARG  # misaligned
    assert _fwd(L, _problem(), ws=512 + 8) == fapk.ERR_INVALID_ARG                  # ws alignment
    assert _fwd(L, _problem(), ctx=None) == fapk.ERR_INVALID_ARG                    # ctx is required
    assert _fwd(L, _problem(), ctx=4096 + 8) == fapk.ERR_INVALID_ARG                # ctx alignment
    assert _fwd(L, _problem(), ws_bytes=16) == fapk.ERR_WORKSPACE_TOO_SMALL
    assert _fwd(L, _problem(scale=float("nan"))) == fapk.ERR_INVALID_ARG
    # T = 0 is a no-op
    assert _fwd(L, _problem(T=0, n_docs=0)) == fapk.OK


@pytest.mark.parametrize("cu,maxlen", [
    ([1, 100, 300], 200),      # does not start at 0
    ([0, 100, 299], 200),      # does not end at T
    ([0, 150, 100, 300], 200), # decreasing
    ([0, 50, 300], 200),       # a document longer than max_seqlen
])
def test_bad_seqlens_detected_on_host(L, cu, maxlen):
    host = np.asarray(cu, dtype=np.int32)
    P = _problem(n_docs=len(cu) - 1, max_seqlen=maxlen, cu_seqlens_host=host.ctypes.data)
    assert _fwd(L, P) == fapk.ERR_BAD_SEQLENS


def test_quantized_kv_forward_validation(L):
    """The forward from pre-quantised K/V takes the MXFP8 path at d = 128 only."""
    f = L.fapk_attn_fwd_quantized_kv
    ptrs = [256] * 11
    assert f(ctypes.byref(_problem(prec=fapk.BF16)), *ptrs, 256, 1 << 30, None) == fapk.ERR_UNSUPPORTED
    assert f(ctypes.byref(_problem(prec=fapk.MXFP8, d=64)), *ptrs, 256, 1 << 30, None) == fapk.ERR_UNSUPPORTED
    bad = list(ptrs)
    bad[2] = 258  # a scale array not 4-byte aligned
    assert f(ctypes.byref(_problem(prec=fapk.MXFP8)), *bad, 256, 1 << 30, None) == fapk.ERR_INVALID_ARG
    assert f(ctypes.byref(_problem(prec=fapk.MXFP8)), *ptrs, 256, 16, None) == fapk.ERR_WORKSPACE_TOO_SMALL


def test_quantize_validation(L):
    q = L.fapk_quantize_mxfp8
    x = 256
    assert q(x, 64, 2, 96, 16, None, 1, 3, 0, 256, 256, 256, 256, None) == fapk.ERR_UNSUPPORTED
    assert q(x, 64, 2, 64, 16, None, 1, 0, 0, 256, 256, 256, 256, None) == fapk.ERR_INVALID_ARG
    assert q(x, 64, 2, 64, 16, None, 1, 3, 5, 256, 256, 256, 256, None) == fapk.ERR_UNSUPPORTED
    assert q(x, 64, 2, 64, 16, None, 1, 1, 0, None, 256, None, None, None) == fapk.ERR_INVALID_ARG
    assert q(x + 8, 64, 2, 64, 16, None, 1, 2, 0, None, None, 256, 256, None) == fapk.ERR_INVALID_ARG
    cu = np.array([0, 10, 60], np.int32)
    assert q(x, 64, 2, 64, 16, cu.ctypes.data, 2, 2, 0, None, None, 256, 256, None) == fapk.ERR_BAD_SEQLENS
    assert q(x, 0, 2, 64, None, None, 0, 3, 0, None, None, None, None, None) == fapk.OK


def test_nvfp4_mixed_validation(L):
    """The mixed NVFP4/FP8 path: RCEIL only, decode scales 0 (=1) or finite
    within [2^-100, 2^100]; its ctx adds Q's and K's NVFP4 forms (64 code bytes
    and 8 scale bytes per token and head, for d = 64 too) to the MXFP8 ctx."""
    nv = dict(prec=fapk.NVFP4_MIXED)
    assert fapk.ctx_size(_problem(d=64, **nv)) >= fapk.ctx_size(_problem(d=64, prec=fapk.MXFP8)) + 300 * 6 * 72
    assert _fwd(L, _problem(scale_rule=fapk.SCALE_OCP, **nv)) == fapk.ERR_UNSUPPORTED
    for bad in (float("nan"), float("inf"), -1.0, 2.0 ** -101, 2.0 ** 101):
        assert _fwd(L, _problem(nv_scale_q=bad, **nv)) == fapk.ERR_INVALID_ARG
        assert _fwd(L, _problem(nv_scale_k=bad, **nv)) == fapk.ERR_INVALID_ARG
    assert _fwd(L, _problem(T=0, n_docs=0, nv_scale_q=0.5, nv_scale_k=4.0, **nv)) == fapk.OK
    P, M = _problem(**nv), _problem(prec=fapk.MXFP8)
    T, Hq, Hkv = P.T, P.Hq, P.Hkv
    assert fapk.ctx_size(P) >= fapk.ctx_size(M) + T * (Hq + Hkv) * 72
    assert fapk.workspace_size(P, fapk.FWD) == fapk.workspace_size(M, fapk.FWD)
    assert fapk.workspace_size(P, fapk.BWD) == fapk.workspace_size(M, fapk.BWD)
    q = L.fapk_quantize_nvfp4
    assert q(256, 64, 2, 64, ctypes.c_float(1.0), 256, 256, None) == fapk.ERR_UNSUPPORTED
    assert q(256, 64, 2, 128, ctypes.c_float(0.0), 256, 256, None) == fapk.ERR_INVALID_ARG
    assert q(256, 64, 2, 128, ctypes.c_float(float("nan")), 256, 256, None) == fapk.ERR_INVALID_ARG
    assert q(264, 64, 2, 128, ctypes.c_float(1.0), 256, 256, None) == fapk.ERR_INVALID_ARG  # x alignment
    assert q(256, 64, 2, 128, ctypes.c_float(1.0), 260, 256, None) == fapk.ERR_INVALID_ARG  # codes alignment
    assert q(256, 0, 2, 128, ctypes.c_float(1.0), None, None, None) == fapk.OK
    # the mixed path's quantised-KV forward and QKV projection
    f = L.fapk_attn_fwd_quantized_kv_nvfp4
    ptrs = [256] * 9
    assert f(ctypes.byref(_problem(prec=fapk.MXFP8)), *ptrs, 256, 1 << 30, None) == fapk.ERR_UNSUPPORTED
    assert f(ctypes.byref(_problem(d=64, **nv)), *ptrs, 256, 1 << 30, None) == fapk.ERR_UNSUPPORTED
    bad = list(ptrs)
    bad[2] = 260  # K's scales not 8-byte aligned
    assert f(ctypes.byref(_problem(**nv)), *bad, 256, 1 << 30, None) == fapk.ERR_INVALID_ARG
    assert f(ctypes.byref(_problem(**nv)), *ptrs, 256, 16, None) == fapk.ERR_WORKSPACE_TOO_SMALL
    g = L.fapk_qkv_proj_nvfp4
    args = [256, 4096, 256, 256, 256, 256, 256, 256, 256, 256, 256, 256, 256]
    assert g(ctypes.byref(_problem(prec=fapk.MXFP8)), *args, 1 << 30, None) == fapk.ERR_UNSUPPORTED
    bad = list(args)
    bad[1] = 4095  # d_model not a multiple of 8
    assert g(ctypes.byref(_problem(**nv)), *bad, 1 << 30, None) == fapk.ERR_INVALID_ARG
    assert g(ctypes.byref(_problem(**nv)), *args, 16, None) == fapk.ERR_WORKSPACE_TOO_SMALL


@pytest.mark.parametrize("prec,rows", [(fapk.BF16, 256), (fapk.MXFP8, 128)])
def test_noalloc_size_limit_matches_its_documented_formula(L, prec, rows):
    """The forward workspace that the no-allocation entry point must fit in its
    1 MiB array is about 17 KiB + 12 B per ceil(max_seqlen/128) + 8 B per
    document (as documented): checked here against the library's own sizing,
    and the limit of about 128 800 documents of one token each."""
    for T, nd, ml in ((32768, 14, 7545), (131072, 30, 65536), (200000, 200000, 1)):
        P = _problem(T=T, n_docs=nd, max_seqlen=ml, prec=prec)
        ws = fapk.workspace_size(P, fapk.FWD)
        levels = -(-ml // rows)
        est = 17 * 1024 + 12 * levels + 8 * nd
        assert abs(ws - est) <= 2048, (T, nd, ml, ws, est)
    limit = 1 << 20
    fits = [n for n in (128000, 128800, 129000)
            if fapk.workspace_size(_problem(T=n, n_docs=n, max_seqlen=1, prec=prec), fapk.FWD) <= limit]
    assert fits == [128000, 128800]
    big = _problem(T=200000, n_docs=200000, max_seqlen=1, prec=prec)
    # rejected on the host, before any CUDA call (dummy aligned pointers)
    assert L.fapk_attn_fwd_noalloc(ctypes.byref(big), 256, 256, 256, 256, 256, 256, None) == \
        fapk.ERR_WORKSPACE_TOO_SMALL
