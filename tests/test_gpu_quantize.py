"""quantize_mxfp8 on the GPU against the oracle: bit-exact codes and scale
bytes (integer/byte work, so the bar is bit-exactness)."""
import numpy as np
import pytest
import torch

import oracle
from causal_flash_attention_packed_b200 import fapk, workloads as W
from gpu_util import require_gpu

pytestmark = pytest.mark.gpu


def _compare(x_bf16: torch.Tensor, cu, rule, forms=3):
    dev = require_gpu()
    seq = fapk.Seqlens(cu, dev)
    got = fapk.quantize_mxfp8(x_bf16.to(dev), seq, forms=forms, scale_rule=rule)
    ref = oracle.quantize_mxfp8(x_bf16.double().numpy(), cu, forms=forms, rule=rule)
    torch.cuda.synchronize()
    for key, val in ref.items():
        g = got[key].cpu().numpy()
        if key == "scale_tb":
            used = val != 0xFF
            assert np.array_equal(g[used], val[used]), key
        else:
            bad = np.count_nonzero(g != val)
            assert bad == 0, f"{key}: {bad} differing bytes"


@pytest.mark.parametrize("rule", [fapk.SCALE_RCEIL, fapk.SCALE_OCP])
def test_every_bf16_value_as_its_own_block(rule):
    """All 65536 bf16 bit patterns (NaN/Inf replaced by 0), two per token in
    separate 32-channel groups so that each is the only non-zero element of its
    per-token block."""
    bits = np.arange(65536, dtype=np.uint32)
    bits[((bits >> 7) & 0xFF) == 0xFF] = 0
    vals = torch.from_numpy((bits << 16).view(np.float32).copy()).to(torch.bfloat16)
    T = 32768
    x = torch.zeros((T, 1, 64), dtype=torch.bfloat16)
    x[:, 0, 0] = vals[:T]
    x[:, 0, 32] = vals[T:]
    _compare(x, np.array([0, T], np.int32), rule, forms=fapk.FORM_PT)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("rule", [fapk.SCALE_RCEIL, fapk.SCALE_OCP])
def test_ragged_documents(d, rule):
    """Document-local token blocks with ragged tails, one-token and empty
    documents, several heads, outlier channels."""
    lengths = [1, 31, 32, 33, 0, 64, 95, 7, 200, 1]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    g = torch.Generator().manual_seed(3)
    x = torch.randn((int(cu[-1]), 3, d), generator=g)
    x[:, 1, 5] *= 20.0
    x[17] *= 1000.0
    _compare(x.to(torch.bfloat16), cu, rule)


def test_full_size_packed_16k():
    """The 16384-token packed workload with outlier channels, K tensor, at full
    size (16384 x 16 x 128), both forms."""
    w = W.config(3, 0)
    _, k, _, _ = w.tensors(with_dout=False)
    _compare(k, w.cu, fapk.SCALE_RCEIL)
