"""Helpers shared by the GPU parity tests: device setup, oracle inputs and the
tolerance checks.  The oracle sees exactly the bf16 bits the kernels see."""
import numpy as np
import pytest
import torch

from causal_flash_attention_packed_b200 import build, fapk

# bf16 path bars (O, dQ, dK, dV against exact fp64): max |err| <= 2e-2 and
# relative Frobenius error <= 5e-3.  LSE: the kernel's scores are fp32 sums of
# exact bf16 products (relative error ~1e-6) and its log/exp2 are accurate to
# ~1e-6, so 1e-3 absolute is a loose but meaningful bar.
MAX_ABS = 2e-2
REL_FROB = 5e-3
LSE_ABS = 1e-3


def require_gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    build.build()
    fapk.lib()
    return torch.device("cuda:0")


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def rel_frob(a: np.ndarray, b: np.ndarray) -> float:
    n = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / n) if n > 0 else float(np.linalg.norm(a - b))


def check_close(name, got: np.ndarray, ref: np.ndarray, max_abs=MAX_ABS, rel=REL_FROB):
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    ma = float(np.max(np.abs(got - ref))) if got.size else 0.0
    rf = rel_frob(got, ref)
    assert ma <= max_abs and rf <= rel, f"{name}: max_abs={ma:.3e} rel_frob={rf:.3e}"
    return ma, rf


def to_dev(w, dev, with_dout=True):
    q, k, v, do = w.tensors(with_dout)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    dod = do.to(dev) if do is not None else None
    return (q, k, v, do), (qd, kd, vd, dod)
