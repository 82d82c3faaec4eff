"""fp64 CPU oracle for causal packed-document attention (bf16 and MXFP8 paths).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``causal_flash_attention_packed_b200``) never
imports, links or runs anything from here, and this package never imports the
product path: the two share no code.

Everything here is a thin ctypes wrapper around ``oracle.cpp`` (plain fp64 C++
with OpenMP); see that file's header for the pages' definitions it follows and
the readings taken where the pages are silent.  Arrays are numpy float64 in the
layouts of the C-ABI: Q/O/dO ``[T, Hq, d]``, K/V ``[T, Hkv, d]``, LSE
``[Hq, T]``, ``cu_seqlens`` int32 ``[n_docs + 1]``.

The MXFP8 emulation (``mx_attn_fwd`` / ``mx_attn_bwd``) is pinned by its
exact limit on on-grid inputs, its cosine to the exact path, the leak tests run
on it, hand-derived cases of the operand selection (forward and backward) and
of the forward's P~, and element-by-element read-outs of the blocks in which
dS~, P~T and dS~T are quantised (tests/test_oracle_mx*.py).  The mixed
NVFP4/FP8 path (``nvmx_attn_fwd`` / ``nvmx_attn_bwd``: the scores from NVFP4 Q
and K) and its quantiser are pinned by the E2M1 and E4M3 grids, hand-worked
blocks, the exact limit on on-grid inputs and a hand-derived score
(tests/test_oracle_nvfp4.py).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

MX_QUANT_P = 1   # quantise the computed P and dS operands (the method's rule)
MX_RULE_OCP = 2  # use the OCP floor(log2 amax) - 8 scale rule instead of RCEIL
# accuracy-study switches (each takes one quantisation out of the emulation)
MX_KEEP_INPUTS = 4   # Q, K, V, dO unquantised
MX_KEEP_P = 8        # P~ and P~T unquantised
MX_KEEP_DS = 16      # dS~ and dS~T unquantised
MX_SYM_GUARD = 32    # Q and dO per token on the diagonal query block of dK and dV
RULE_RCEIL = 0   # scale exponent X = ceil(log2(amax / 448)): never saturates
RULE_OCP = 1     # scale exponent X = floor(log2 amax) - 8: may saturate to 448


def build(force: bool = False) -> str:
    """Compile oracle.cpp into liboracle.so (g++ -O3 -fopenmp, no fast-math)."""
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    cmd = ["g++", "-O3", "-march=x86-64-v3", "-fopenmp", "-fPIC", "-shared", "-std=c++17",
           "-o", _LIB_PATH + ".tmp", _SRC]
    subprocess.check_call(cmd)
    os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB_PATH)
    P = ctypes.c_void_p
    i = ctypes.c_int
    dbl = ctypes.c_double
    lib.orc_num_threads.restype = i
    lib.orc_set_threads.argtypes = [i]
    head = [i, i, P, i, i, i, dbl]
    lib.orc_attn_fwd.argtypes = head + [P, P, P, P, P]
    lib.orc_attn_bwd.argtypes = head + [P, P, P, P, P, P, P, P, P]
    lib.orc_attn_rows.argtypes = head + [P, P, P, P, i, P, P, P, P, P]
    lib.orc_attn_kv_cols.argtypes = head + [P, P, P, P, i, P, P, P, P]
    lib.orc_attn_kv_cols_from_rows.argtypes = head + [P, P, P, P, P, P, i, P, P, P, P]
    lib.orc_e4m3_encode.argtypes = [dbl]
    lib.orc_e4m3_encode.restype = ctypes.c_uint8
    lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.orc_e4m3_decode.restype = dbl
    lib.orc_block_exponent.argtypes = [dbl, i]
    lib.orc_block_exponent.restype = i
    lib.orc_quant_block.argtypes = [P, i, P, P, i]
    lib.orc_quant_block.restype = ctypes.c_uint8
    lib.orc_quantize_mxfp8.argtypes = [P, i, i, i, P, i, i, i, P, P, P, P]
    lib.orc_mx_attn_fwd.argtypes = head + [P, P, P, i, P, P]
    lib.orc_mx_attn_bwd.argtypes = head + [P, P, P, P, i, P, P, P, P, P]
    f32 = ctypes.c_float
    lib.orc_e2m1_encode.argtypes = [dbl]
    lib.orc_e2m1_encode.restype = ctypes.c_uint8
    lib.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
    lib.orc_e2m1_decode.restype = dbl
    lib.orc_nv_quant_block.argtypes = [P, i, f32, P, P]
    lib.orc_nv_quant_block.restype = ctypes.c_uint8
    lib.orc_quantize_nvfp4.argtypes = [P, i, i, i, f32, P, P]
    lib.orc_nvmx_attn_fwd.argtypes = head + [P, P, P, i, f32, f32, P, P]
    lib.orc_nvmx_attn_bwd.argtypes = head + [P, P, P, P, i, f32, f32, P, P, P, P, P]
    _lib = lib
    return lib


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float64)


def _i32(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.int32)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return _load().orc_num_threads()


def set_threads(n: int) -> None:
    _load().orc_set_threads(int(n))


def _dims(q, k, cu):
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    assert k.shape == (T, Hkv, d) and Hq % Hkv == 0
    assert cu[0] == 0 and cu[-1] == T and np.all(np.diff(cu) >= 0)
    return T, len(cu) - 1, Hq, Hkv, d


def attn_fwd(q, k, v, cu, scale):
    """Exact forward: returns (O [T,Hq,d], LSE [Hq,T]) in fp64."""
    q, k, v, cu = _f64(q), _f64(k), _f64(v), _i32(cu)
    T, nd, Hq, Hkv, d = _dims(q, k, cu)
    o = np.zeros((T, Hq, d))
    lse = np.zeros((Hq, T))
    _load().orc_attn_fwd(T, nd, _ptr(cu), Hq, Hkv, d, float(scale), _ptr(q), _ptr(k), _ptr(v),
                         _ptr(o), _ptr(lse))
    return o, lse


def attn_bwd(q, k, v, do, cu, scale):
    """Exact forward + backward: returns dict o, lse, dq, dk, dv (fp64)."""
    q, k, v, do, cu = _f64(q), _f64(k), _f64(v), _f64(do), _i32(cu)
    T, nd, Hq, Hkv, d = _dims(q, k, cu)
    out = dict(o=np.zeros((T, Hq, d)), lse=np.zeros((Hq, T)), dq=np.zeros((T, Hq, d)),
               dk=np.zeros((T, Hkv, d)), dv=np.zeros((T, Hkv, d)))
    _load().orc_attn_bwd(T, nd, _ptr(cu), Hq, Hkv, d, float(scale), _ptr(q), _ptr(k), _ptr(v),
                         _ptr(do), _ptr(out["o"]), _ptr(out["lse"]), _ptr(out["dq"]),
                         _ptr(out["dk"]), _ptr(out["dv"]))
    return out


def attn_rows(q, k, v, do, cu, scale, tok, head):
    """Exact O, LSE, dQ of selected (token, query-head) rows."""
    q, k, v, do, cu = _f64(q), _f64(k), _f64(v), _f64(do), _i32(cu)
    T, nd, Hq, Hkv, d = _dims(q, k, cu)
    tok, head = _i32(tok), _i32(head)
    n = len(tok)
    o, dq, lse = np.zeros((n, d)), np.zeros((n, d)), np.zeros(n)
    _load().orc_attn_rows(T, nd, _ptr(cu), Hq, Hkv, d, float(scale), _ptr(q), _ptr(k), _ptr(v),
                          _ptr(do), n, _ptr(tok), _ptr(head), _ptr(o), _ptr(lse), _ptr(dq))
    return o, lse, dq


def attn_kv_cols(q, k, v, do, cu, scale, tok, kvhead):
    """Exact dK, dV of selected (token, kv-head) keys."""
    q, k, v, do, cu = _f64(q), _f64(k), _f64(v), _f64(do), _i32(cu)
    T, nd, Hq, Hkv, d = _dims(q, k, cu)
    tok, kvhead = _i32(tok), _i32(kvhead)
    n = len(tok)
    dk, dv = np.zeros((n, d)), np.zeros((n, d))
    _load().orc_attn_kv_cols(T, nd, _ptr(cu), Hq, Hkv, d, float(scale), _ptr(q), _ptr(k),
                             _ptr(v), _ptr(do), n, _ptr(tok), _ptr(kvhead), _ptr(dk), _ptr(dv))
    return dk, dv


def attn_fwd_doc(q, k, v, cu, scale, doc, head, chunk: int = 2048):
    """Exact O [L,d] and LSE [L] of every query of document `doc` for query
    head `head`, for one long document (where the per-(document, head) tasks
    of attn_fwd leave most cores idle).  Plain fp64 torch CPU ops, row by row
    as the definition reads ("GPT Kernel Programlama" page secs. 3-6): the
    score row S_i = scale q_i K^T over the document's keys, the causal mask
    j > i, the stable softmax and O_i = P_i V; rows are handed to the matmul
    `chunk` at a time, each row on its own, so that the library's threads
    share the work."""
    import torch
    cu = _i32(cu)
    T, Hq, d = q.shape
    G = Hq // k.shape[1]
    s, e = int(cu[doc]), int(cu[doc + 1])
    L = e - s
    Q = torch.from_numpy(_f64(q[s:e, head]))
    K = torch.from_numpy(_f64(k[s:e, head // G]))
    V = torch.from_numpy(_f64(v[s:e, head // G]))
    o = torch.empty((L, d), dtype=torch.float64)
    lse = torch.empty(L, dtype=torch.float64)
    for i0 in range(0, L, chunk):
        i1 = min(L, i0 + chunk)
        S = (Q[i0:i1] @ K[:i1].T) * float(scale)
        S.masked_fill_(torch.arange(i1)[None, :] > torch.arange(i0, i1)[:, None], float("-inf"))
        m = S.amax(dim=1, keepdim=True)
        S.sub_(m).exp_()
        ell = S.sum(dim=1, keepdim=True)
        o[i0:i1] = (S @ V[:i1]) / ell
        lse[i0:i1] = (m + torch.log(ell))[:, 0]
    return o.numpy(), lse.numpy()


def attn_kv_cols_from_rows(q, k, v, do, o, lse, cu, scale, tok, kvhead):
    """Exact dK, dV of selected (token, kv-head) keys, given the exact O
    [T,Hq,d] and LSE [Hq,T] of every query that sees them (from attn_fwd or
    attn_fwd_doc); no query row is recomputed."""
    q, k, v, do, o, lse, cu = _f64(q), _f64(k), _f64(v), _f64(do), _f64(o), _f64(lse), _i32(cu)
    T, nd, Hq, Hkv, d = _dims(q, k, cu)
    assert o.shape == q.shape and lse.shape == (Hq, T)
    tok, kvhead = _i32(tok), _i32(kvhead)
    n = len(tok)
    dk, dv = np.zeros((n, d)), np.zeros((n, d))
    _load().orc_attn_kv_cols_from_rows(T, nd, _ptr(cu), Hq, Hkv, d, float(scale), _ptr(q), _ptr(k),
                                       _ptr(v), _ptr(do), _ptr(o), _ptr(lse), n, _ptr(tok), _ptr(kvhead),
                                       _ptr(dk), _ptr(dv))
    return dk, dv


def qkv_proj(x, w, Hq: int, Hkv: int, d: int):
    """Fused QKV projection, exact ("GPT Kernel Programlama" page, sec. 2: the
    three projections of X as one): Y = X W^T in fp64 (a library matmul), its
    columns split into the Q heads, then the K heads, then the V heads.
    x [T, d_model], w [(Hq + 2 Hkv) d, d_model]; returns q [T, Hq, d],
    k, v [T, Hkv, d]."""
    x, w = _f64(x), _f64(w)
    T = x.shape[0]
    assert w.shape == ((Hq + 2 * Hkv) * d, x.shape[1])
    y = x @ w.T
    q = y[:, : Hq * d].reshape(T, Hq, d)
    k = y[:, Hq * d: (Hq + Hkv) * d].reshape(T, Hkv, d)
    v = y[:, (Hq + Hkv) * d:].reshape(T, Hkv, d)
    return q, k, v


# ---- MXFP8 quantiser ----------------------------------------------------

def e4m3_encode(y: float) -> int:
    return int(_load().orc_e4m3_encode(float(y)))


def e4m3_decode(code: int) -> float:
    return float(_load().orc_e4m3_decode(int(code)))


def block_exponent(amax: float, rule: int = RULE_RCEIL) -> int:
    return int(_load().orc_block_exponent(float(amax), int(rule)))


def quant_block(x, rule: int = RULE_RCEIL):
    """Quantise one block: returns (codes uint8[n], dequantised f64[n], scale byte)."""
    x = _f64(x)
    codes = np.zeros(len(x), np.uint8)
    deq = np.zeros(len(x))
    sb = _load().orc_quant_block(_ptr(x), len(x), _ptr(codes), _ptr(deq), int(rule))
    return codes, deq, int(sb)


def tb_slots(T: int, n_docs: int) -> int:
    """Number of token-block scale slots: floor(T/32) + n_docs."""
    return T // 32 + n_docs


def quantize_mxfp8(x, cu, forms: int = 3, rule: int = RULE_RCEIL):
    """quantize_mxfp8 of a [T,H,d] bf16-valued tensor.  Returns a dict with
    val_tb/scale_tb (forms & 1) and val_pt/scale_pt (forms & 2).  Unused
    token-block scale slots hold 0xFF (never a real scale byte here)."""
    x, cu = _f64(x), _i32(cu)
    T, H, d = x.shape
    nd = len(cu) - 1
    out = {}
    vtb = np.zeros((T, H, d), np.uint8)
    stb = np.full((tb_slots(T, nd), H, d // 32), 0xFF, np.uint8)
    vpt = np.zeros((T, H, d), np.uint8)
    spt = np.zeros((T, H, d // 32), np.uint8)
    _load().orc_quantize_mxfp8(_ptr(x), T, H, d, _ptr(cu), nd, forms, int(rule), _ptr(vtb),
                               _ptr(stb), _ptr(vpt), _ptr(spt))
    if forms & 1:
        out["val_tb"], out["scale_tb"] = vtb, stb
    if forms & 2:
        out["val_pt"], out["scale_pt"] = vpt, spt
    return out


def mx_attn_fwd(q, k, v, cu, scale, flags: int = MX_QUANT_P):
    """MXFP8 emulation forward: (O, LSE) in fp64."""
    q, k, v, cu = _f64(q), _f64(k), _f64(v), _i32(cu)
    T, nd, Hq, Hkv, d = _dims(q, k, cu)
    o = np.zeros((T, Hq, d))
    lse = np.zeros((Hq, T))
    _load().orc_mx_attn_fwd(T, nd, _ptr(cu), Hq, Hkv, d, float(scale), _ptr(q), _ptr(k), _ptr(v),
                            int(flags), _ptr(o), _ptr(lse))
    return o, lse


def mx_attn_bwd(q, k, v, do, cu, scale, flags: int = MX_QUANT_P):
    """MXFP8 emulation forward + backward: dict o, lse, dq, dk, dv."""
    q, k, v, do, cu = _f64(q), _f64(k), _f64(v), _f64(do), _i32(cu)
    T, nd, Hq, Hkv, d = _dims(q, k, cu)
    out = dict(o=np.zeros((T, Hq, d)), lse=np.zeros((Hq, T)), dq=np.zeros((T, Hq, d)),
               dk=np.zeros((T, Hkv, d)), dv=np.zeros((T, Hkv, d)))
    _load().orc_mx_attn_bwd(T, nd, _ptr(cu), Hq, Hkv, d, float(scale), _ptr(q), _ptr(k),
                            _ptr(v), _ptr(do), int(flags), _ptr(out["o"]), _ptr(out["lse"]),
                            _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]))
    return out


# ---- mixed NVFP4/FP8 path --------------------------------------------------

def e2m1_encode(y: float) -> int:
    return int(_load().orc_e2m1_encode(float(y)))


def e2m1_decode(code: int) -> float:
    return float(_load().orc_e2m1_decode(int(code)))


def nv_quant_block(x, g: float = 1.0):
    """One NVFP4 block: returns (E2M1 codes uint8[n], dequantised f64[n], E4M3 scale byte)."""
    x = _f64(x)
    codes = np.zeros(len(x), np.uint8)
    deq = np.zeros(len(x))
    sb = _load().orc_nv_quant_block(_ptr(x), len(x), float(g), _ptr(codes), _ptr(deq))
    return codes, deq, int(sb)


def quantize_nvfp4(x, g: float = 1.0):
    """NVFP4 of a [T,H,d] bf16-valued tensor: (codes uint8 [T,H,d/2], channel
    2i in the low nibble; scales uint8 [T,H,d/16])."""
    x = _f64(x)
    T, H, d = x.shape
    codes = np.zeros((T, H, d // 2), np.uint8)
    scales = np.zeros((T, H, d // 16), np.uint8)
    _load().orc_quantize_nvfp4(_ptr(x), T, H, d, float(g), _ptr(codes), _ptr(scales))
    return codes, scales


def nvmx_attn_fwd(q, k, v, cu, scale, flags: int = MX_QUANT_P, gq: float = 1.0, gk: float = 1.0):
    """Mixed NVFP4/FP8 emulation forward: (O, LSE) in fp64."""
    q, k, v, cu = _f64(q), _f64(k), _f64(v), _i32(cu)
    T, nd, Hq, Hkv, d = _dims(q, k, cu)
    o = np.zeros((T, Hq, d))
    lse = np.zeros((Hq, T))
    _load().orc_nvmx_attn_fwd(T, nd, _ptr(cu), Hq, Hkv, d, float(scale), _ptr(q), _ptr(k), _ptr(v),
                              int(flags), float(gq), float(gk), _ptr(o), _ptr(lse))
    return o, lse


def nvmx_attn_bwd(q, k, v, do, cu, scale, flags: int = MX_QUANT_P, gq: float = 1.0, gk: float = 1.0):
    """Mixed NVFP4/FP8 emulation forward + backward: dict o, lse, dq, dk, dv."""
    q, k, v, do, cu = _f64(q), _f64(k), _f64(v), _f64(do), _i32(cu)
    T, nd, Hq, Hkv, d = _dims(q, k, cu)
    out = dict(o=np.zeros((T, Hq, d)), lse=np.zeros((Hq, T)), dq=np.zeros((T, Hq, d)),
               dk=np.zeros((T, Hkv, d)), dv=np.zeros((T, Hkv, d)))
    _load().orc_nvmx_attn_bwd(T, nd, _ptr(cu), Hq, Hkv, d, float(scale), _ptr(q), _ptr(k),
                              _ptr(v), _ptr(do), int(flags), float(gq), float(gk), _ptr(out["o"]),
                              _ptr(out["lse"]), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]))
    return out


def flops_causal(cu, Hq: int, d: int) -> float:
    """Algorithmic causal fwd+bwd FLOPs: 14 d Hq sum_k L_k (L_k + 1) / 2."""
    L = np.diff(np.asarray(cu, dtype=np.int64))
    return 14.0 * d * Hq * float(np.sum(L * (L + 1) // 2))
