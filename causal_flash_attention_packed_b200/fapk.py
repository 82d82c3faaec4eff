"""Python binding of libfapk.so (the C ABI declared in include/fapk.h).

Argument marshalling only: every step of the attention path runs in the
library's CUDA kernels.  torch provides device memory (outputs, workspaces) and
the current stream.  There is no fallback: if ``libfapk.so`` is missing or
cannot be loaded, every call raises ``FapkError``.

Names follow the C ABI without the ``fapk_`` prefix: ``attn_fwd``,
``attn_bwd``, ``quantize_mxfp8``, ``quantize_nvfp4``, ``workspace_size``, ``ctx_size``,
``status``, ``strerror``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfapk.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED = 2
ERR_BAD_SEQLENS = 3
ERR_WORKSPACE_TOO_SMALL = 4
ERR_CUDA = 5
ERR_DEVICE_TIMEOUT = 6
ERR_RANGE = 7
ERR_INTERNAL = 8

BF16 = 0
MXFP8 = 1
NVFP4_MIXED = 2
GRAD_F32 = 0
GRAD_BF16 = 1
SCALE_RCEIL = 0
SCALE_OCP = 1
FWD = 0
BWD = 1
FORM_TB = 1
FORM_PT = 2
FLAG_INJECT_DROP_LOAD = 1
FLAG_CTA_TIMES = 2


class FapkError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {strerror(code) if _lib is not None else code} (status {code})")


class Problem(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int),
        ("n_docs", ctypes.c_int),
        ("max_seqlen", ctypes.c_int),
        ("Hq", ctypes.c_int),
        ("Hkv", ctypes.c_int),
        ("d", ctypes.c_int),
        ("scale", ctypes.c_float),
        ("prec", ctypes.c_int),
        ("scale_rule", ctypes.c_int),
        ("cu_seqlens_dev", ctypes.c_void_p),
        ("cu_seqlens_host", ctypes.c_void_p),
        ("grad_dtype", ctypes.c_int),
        ("flags", ctypes.c_int),
        ("timeout_ms", ctypes.c_int),
        ("timing_events", ctypes.c_void_p),
        ("n_timing_events", ctypes.c_int),
        ("nv_scale_q", ctypes.c_float),
        ("nv_scale_k", ctypes.c_float),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libfapk.so (raises FapkError if it is missing: no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise FapkError(ERR_CUDA, f"{LIB_PATH} is missing; build it with "
                        "`python -m causal_flash_attention_packed_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    PP = ctypes.POINTER(Problem)
    L.fapk_workspace_size.argtypes = [PP, i]
    L.fapk_workspace_size.restype = sz
    L.fapk_ctx_size.argtypes = [PP]
    L.fapk_ctx_size.restype = sz
    L.fapk_attn_fwd.argtypes = [PP, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.fapk_attn_fwd.restype = i
    L.fapk_attn_bwd.argtypes = [PP, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.fapk_attn_bwd.restype = i
    L.fapk_attn_fwd_noalloc.argtypes = [PP, vp, vp, vp, vp, vp, vp, vp]
    L.fapk_attn_fwd_noalloc.restype = i
    L.fapk_attn_fwd_quantized_kv.argtypes = [PP] + [vp] * 12 + [sz, vp]
    L.fapk_attn_fwd_quantized_kv.restype = i
    L.fapk_qkv_proj_mxfp8.argtypes = [PP, vp, i, vp, vp, vp, vp] + [vp] * 8 + [vp, sz, vp]
    L.fapk_qkv_proj_mxfp8.restype = i
    L.fapk_attn_fwd_quantized_kv_nvfp4.argtypes = [PP] + [vp] * 10 + [sz, vp]
    L.fapk_attn_fwd_quantized_kv_nvfp4.restype = i
    L.fapk_qkv_proj_nvfp4.argtypes = [PP, vp, i, vp, vp, vp, vp] + [vp] * 6 + [vp, sz, vp]
    L.fapk_qkv_proj_nvfp4.restype = i
    L.fapk_noalloc_status.argtypes = [vp]
    L.fapk_noalloc_status.restype = i
    L.fapk_quantize_mxfp8.argtypes = [vp, i, i, i, vp, vp, i, i, i, vp, vp, vp, vp, vp]
    L.fapk_quantize_mxfp8.restype = i
    L.fapk_quantize_nvfp4.argtypes = [vp, i, i, i, ctypes.c_float, vp, vp, vp]
    L.fapk_quantize_nvfp4.restype = i
    L.fapk_status.argtypes = [vp, vp]
    L.fapk_status.restype = i
    L.fapk_cta_times.argtypes = [PP, i, i, vp, vp, ctypes.POINTER(ctypes.c_ulonglong), i, ctypes.POINTER(i)]
    L.fapk_cta_times.restype = i
    L.fapk_strerror.argtypes = [i]
    L.fapk_strerror.restype = ctypes.c_char_p
    L.fapk_launch_count.argtypes = []
    L.fapk_launch_count.restype = ctypes.c_uint64
    L.fapk_version.argtypes = []
    L.fapk_version.restype = i
    _lib = L
    return L


def strerror(code: int) -> str:
    return lib().fapk_strerror(int(code)).decode()


def launch_count() -> int:
    return int(lib().fapk_launch_count())


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check(rc: int, what: str) -> None:
    if rc != OK:
        raise FapkError(rc, what)


class Seqlens:
    """cu_seqlens held both on the device (required by the kernels) and on the
    host (validated by the library before launch)."""

    def __init__(self, cu, device="cuda"):
        host = np.ascontiguousarray(np.asarray(cu, dtype=np.int32))
        self.host = host
        self.dev = torch.from_numpy(host.copy()).to(device)
        self.n_docs = len(host) - 1
        self.T = int(host[-1]) if len(host) else 0
        L = np.diff(host.astype(np.int64))
        self.max_seqlen = int(L.max()) if len(L) else 0


def make_problem(seq: Seqlens, Hq: int, Hkv: int, d: int, scale: float, prec: int = BF16,
                 grad_dtype: int = GRAD_F32, scale_rule: int = SCALE_RCEIL, flags: int = 0,
                 timeout_ms: int = 0, validate_host: bool = True, nv_scale_q: float = 0.0,
                 nv_scale_k: float = 0.0) -> Problem:
    P = Problem()
    P.T = seq.T
    P.n_docs = seq.n_docs
    P.max_seqlen = max(1, seq.max_seqlen)
    P.Hq, P.Hkv, P.d = Hq, Hkv, d
    P.scale = float(scale)
    P.prec = prec
    P.scale_rule = scale_rule
    P.cu_seqlens_dev = seq.dev.data_ptr() if seq.T > 0 else None
    P.cu_seqlens_host = seq.host.ctypes.data if validate_host else None
    P.grad_dtype = grad_dtype
    P.flags = flags
    P.timeout_ms = timeout_ms
    P.timing_events = None
    P.n_timing_events = 0
    P.nv_scale_q = float(nv_scale_q)
    P.nv_scale_k = float(nv_scale_k)
    P._seqlens = seq  # the problem points at seq's device array: keep it alive with the problem
    return P


class KernelTimer:
    """CUDA events that a call records between its kernel launches
    (fapk_problem_t.timing_events): ``with_events(P)`` returns a copy of the
    problem that records into this timer's events; ``durations_ms()`` returns
    the time between consecutive events."""

    def __init__(self, n: int):
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in self.events:  # create the underlying cudaEvent_t
            e.record()
        torch.cuda.synchronize()
        self._handles = (ctypes.c_void_p * n)(*[e.cuda_event for e in self.events])

    def with_events(self, P: Problem) -> Problem:
        Q = Problem.from_buffer_copy(P)
        Q._seqlens = getattr(P, "_seqlens", None)
        Q.timing_events = ctypes.cast(self._handles, ctypes.c_void_p)
        Q.n_timing_events = len(self.events)
        return Q

    def durations_ms(self):
        return [a.elapsed_time(b) for a, b in zip(self.events[:-1], self.events[1:])]


def workspace_size(P: Problem, which: int) -> int:
    return int(lib().fapk_workspace_size(ctypes.byref(P), which))


def ctx_size(P: Problem) -> int:
    return int(lib().fapk_ctx_size(ctypes.byref(P)))


def workspace(P: Problem, which: int, device="cuda") -> torch.Tensor:
    n = workspace_size(P, which)
    if n == 0 and P.T > 0:
        raise FapkError(ERR_INVALID_ARG, "workspace_size")
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def attn_fwd(P: Problem, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
             o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
             ctx: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
             stream=None) -> Tuple[torch.Tensor, torch.Tensor, Optional[torch.Tensor]]:
    """fapk_attn_fwd: returns (o [T,Hq,d] bf16, lse [Hq,T] fp32, ctx).  Pass the
    returned ctx to attn_bwd."""
    if o is None:
        o = torch.empty((P.T, P.Hq, P.d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((P.Hq, P.T), dtype=torch.float32, device=q.device)
    if ctx is None:
        ctx = torch.empty(max(ctx_size(P), 256), dtype=torch.uint8, device=q.device)
    if ws is None:
        ws = workspace(P, FWD, q.device)
    rc = lib().fapk_attn_fwd(ctypes.byref(P), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                             _ptr(ctx), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "fapk_attn_fwd")
    return o, lse, ctx


def attn_fwd_noalloc(P: Problem, q, k, v, o, lse, ctx, stream=None):
    """fapk_attn_fwd_noalloc: the forward with the library's fixed scratch array
    instead of a workspace, for callers that cannot allocate device memory.  The
    caller passes every buffer (o, lse, ctx)."""
    rc = lib().fapk_attn_fwd_noalloc(ctypes.byref(P), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                     _ptr(ctx), _stream(stream))
    _check(rc, "fapk_attn_fwd_noalloc")
    return o, lse, ctx


def attn_fwd_quantized_kv(P: Problem, q, k_forms: dict, v_forms: dict, o=None, lse=None, ws=None, stream=None):
    """fapk_attn_fwd_quantized_kv: MXFP8 forward over K and V given in both MX
    forms (dicts with val_tb, scale_tb, val_pt, scale_pt as quantize_mxfp8
    returns them).  Returns (o, lse)."""
    dev = q.device
    if o is None:
        o = torch.empty((P.T, P.Hq, P.d), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((P.Hq, P.T), dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(P, FWD, dev)
    f = [k_forms[n] for n in ("val_tb", "scale_tb", "val_pt", "scale_pt")] + \
        [v_forms[n] for n in ("val_tb", "scale_tb", "val_pt", "scale_pt")]
    rc = lib().fapk_attn_fwd_quantized_kv(ctypes.byref(P), _ptr(q), *[_ptr(t) for t in f], _ptr(o), _ptr(lse),
                                          _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "fapk_attn_fwd_quantized_kv")
    return o, lse


def qkv_proj_mxfp8(P: Problem, x: torch.Tensor, w: torch.Tensor, ws=None, stream=None):
    """fapk_qkv_proj_mxfp8: [Q | K | V] = x w^T with K's and V's MX forms from
    the epilogue.  x [T, d_model] bf16, w [(Hq + 2 Hkv) d, d_model] bf16.
    Returns (q, k, v, k_forms, v_forms); the forms are dicts like
    quantize_mxfp8's, ready for attn_fwd_quantized_kv."""
    dev = x.device
    T, Dm = x.shape
    q = torch.empty((T, P.Hq, P.d), dtype=torch.bfloat16, device=dev)
    k = torch.empty((T, P.Hkv, P.d), dtype=torch.bfloat16, device=dev)
    v = torch.empty((T, P.Hkv, P.d), dtype=torch.bfloat16, device=dev)

    def forms():
        return {"val_tb": torch.empty((T, P.Hkv, P.d), dtype=torch.uint8, device=dev),
                "scale_tb": torch.full((tb_slots(T, P.n_docs), P.Hkv, P.d // 32), 0xFF, dtype=torch.uint8,
                                       device=dev),
                "val_pt": torch.empty((T, P.Hkv, P.d), dtype=torch.uint8, device=dev),
                "scale_pt": torch.empty((T, P.Hkv, P.d // 32), dtype=torch.uint8, device=dev)}

    kf, vf = forms(), forms()
    if ws is None:
        ws = workspace(P, FWD, dev)
    f = [kf[n] for n in ("val_tb", "scale_tb", "val_pt", "scale_pt")] + \
        [vf[n] for n in ("val_tb", "scale_tb", "val_pt", "scale_pt")]
    rc = lib().fapk_qkv_proj_mxfp8(ctypes.byref(P), _ptr(x), Dm, _ptr(w), _ptr(q), _ptr(k), _ptr(v),
                                   *[_ptr(t) for t in f], _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "fapk_qkv_proj_mxfp8")
    return q, k, v, kf, vf


def qkv_proj_nvfp4(P: Problem, x: torch.Tensor, w: torch.Tensor, ws=None, stream=None):
    """fapk_qkv_proj_nvfp4 (mixed path): [Q | K | V] = x w^T with K's NVFP4
    form and V's MX forms from the epilogue.  Returns (q, k, v, (k_codes,
    k_scales), v_forms), ready for attn_fwd_quantized_kv_nvfp4."""
    dev = x.device
    T, Dm = x.shape
    q = torch.empty((T, P.Hq, P.d), dtype=torch.bfloat16, device=dev)
    k = torch.empty((T, P.Hkv, P.d), dtype=torch.bfloat16, device=dev)
    v = torch.empty((T, P.Hkv, P.d), dtype=torch.bfloat16, device=dev)
    kc = torch.empty((T, P.Hkv, P.d // 2), dtype=torch.uint8, device=dev)
    ks = torch.empty((T, P.Hkv, P.d // 16), dtype=torch.uint8, device=dev)
    vf = {"val_tb": torch.empty((T, P.Hkv, P.d), dtype=torch.uint8, device=dev),
          "scale_tb": torch.full((tb_slots(T, P.n_docs), P.Hkv, P.d // 32), 0xFF, dtype=torch.uint8, device=dev),
          "val_pt": torch.empty((T, P.Hkv, P.d), dtype=torch.uint8, device=dev),
          "scale_pt": torch.empty((T, P.Hkv, P.d // 32), dtype=torch.uint8, device=dev)}
    if ws is None:
        ws = workspace(P, FWD, dev)
    f = [vf[n] for n in ("val_tb", "scale_tb", "val_pt", "scale_pt")]
    rc = lib().fapk_qkv_proj_nvfp4(ctypes.byref(P), _ptr(x), Dm, _ptr(w), _ptr(q), _ptr(k), _ptr(v), _ptr(kc),
                                   _ptr(ks), *[_ptr(t) for t in f], _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "fapk_qkv_proj_nvfp4")
    return q, k, v, (kc, ks), vf


def attn_fwd_quantized_kv_nvfp4(P: Problem, q, k_nv, v_forms: dict, o=None, lse=None, ws=None, stream=None):
    """fapk_attn_fwd_quantized_kv_nvfp4 (mixed path): the forward over K in
    NVFP4 (k_nv = (codes, scales) as quantize_nvfp4 returns them) and V in
    both MX forms.  Returns (o, lse)."""
    dev = q.device
    if o is None:
        o = torch.empty((P.T, P.Hq, P.d), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((P.Hq, P.T), dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(P, FWD, dev)
    f = [v_forms[n] for n in ("val_tb", "scale_tb", "val_pt", "scale_pt")]
    rc = lib().fapk_attn_fwd_quantized_kv_nvfp4(ctypes.byref(P), _ptr(q), _ptr(k_nv[0]), _ptr(k_nv[1]),
                                                *[_ptr(t) for t in f], _ptr(o), _ptr(lse), _ptr(ws), ws.numel(),
                                                _stream(stream))
    _check(rc, "fapk_attn_fwd_quantized_kv_nvfp4")
    return o, lse


def attn_bwd(P: Problem, q, k, v, o, lse, dout, ctx=None, dq=None, dk=None, dv=None, ws=None,
             stream=None):
    """fapk_attn_bwd: returns (dq, dk, dv) in the problem's grad dtype."""
    gdt = torch.float32 if P.grad_dtype == GRAD_F32 else torch.bfloat16
    dev = q.device
    if dq is None:
        dq = torch.empty((P.T, P.Hq, P.d), dtype=gdt, device=dev)
    if dk is None:
        dk = torch.empty((P.T, P.Hkv, P.d), dtype=gdt, device=dev)
    if dv is None:
        dv = torch.empty((P.T, P.Hkv, P.d), dtype=gdt, device=dev)
    if ws is None:
        ws = workspace(P, BWD, dev)
    rc = lib().fapk_attn_bwd(ctypes.byref(P), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                             _ptr(dout), _ptr(ctx), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
                             ws.numel(), _stream(stream))
    _check(rc, "fapk_attn_bwd")
    return dq, dk, dv


def tb_slots(T: int, n_docs: int) -> int:
    return T // 32 + n_docs


def quantize_mxfp8(x: torch.Tensor, seq: Seqlens, forms: int = FORM_TB | FORM_PT,
                   scale_rule: int = SCALE_RCEIL, out: Optional[dict] = None, stream=None) -> dict:
    """fapk_quantize_mxfp8 of x [T,H,d] bf16.  Returns a dict of uint8 device
    tensors val_tb/scale_tb (token-block form) and val_pt/scale_pt (per token).
    Token-block scale slots that hold no block are left as allocated (0xFF
    when this function allocates them)."""
    T, H, d = x.shape
    dev = x.device
    out = dict(out or {})
    if forms & FORM_TB:
        out.setdefault("val_tb", torch.empty((T, H, d), dtype=torch.uint8, device=dev))
        out.setdefault("scale_tb", torch.full((tb_slots(T, seq.n_docs), H, d // 32), 0xFF,
                                              dtype=torch.uint8, device=dev))
    if forms & FORM_PT:
        out.setdefault("val_pt", torch.empty((T, H, d), dtype=torch.uint8, device=dev))
        out.setdefault("scale_pt", torch.empty((T, H, d // 32), dtype=torch.uint8, device=dev))
    rc = lib().fapk_quantize_mxfp8(_ptr(x), T, H, d, seq.dev.data_ptr() if T else None,
                                   seq.host.ctypes.data, seq.n_docs, forms, scale_rule,
                                   _ptr(out.get("val_tb")), _ptr(out.get("scale_tb")),
                                   _ptr(out.get("val_pt")), _ptr(out.get("scale_pt")),
                                   _stream(stream))
    _check(rc, "fapk_quantize_mxfp8")
    return out


def quantize_nvfp4(x: torch.Tensor, g: float = 1.0, stream=None):
    """fapk_quantize_nvfp4 of x [T,H,128] bf16 with decode scale g.  Returns
    (codes uint8 [T,H,64], channel 2i in the low nibble of byte i; scales
    uint8 [T,H,8], E4M3)."""
    T, H, d = x.shape
    codes = torch.empty((T, H, d // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty((T, H, d // 16), dtype=torch.uint8, device=x.device)
    _check(lib().fapk_quantize_nvfp4(_ptr(x), T, H, d, float(g), _ptr(codes), _ptr(scales), _stream(stream)),
           "fapk_quantize_nvfp4")
    return codes, scales


def cta_times(P: Problem, which: int, kernel: int, ws: torch.Tensor, stream=None):
    """Per-CTA (start, end) %globaltimer pairs (ns, int64 array [n, 2]) of
    persistent kernel `kernel` of the last call made with FLAG_CTA_TIMES on
    workspace `ws` (forward: 0; backward: 0 = dK/dV, 1 = dQ)."""
    import numpy as np
    out = (ctypes.c_ulonglong * (2 * 1024))()
    n = ctypes.c_int(0)
    _check(lib().fapk_cta_times(ctypes.byref(P), which, kernel, _ptr(ws), _stream(stream), out, 1024,
                                ctypes.byref(n)), "fapk_cta_times")
    return np.array(out[: 2 * n.value], dtype=np.int64).reshape(-1, 2)


def status(ws: torch.Tensor, stream=None) -> int:
    """fapk_status: synchronises the stream and returns the device status word."""
    return int(lib().fapk_status(_ptr(ws), _stream(stream)))


def noalloc_status(stream=None) -> int:
    """fapk_noalloc_status: synchronises the stream and returns the status word
    of the last fapk_attn_fwd_noalloc call on the current device."""
    return int(lib().fapk_noalloc_status(_stream(stream)))
