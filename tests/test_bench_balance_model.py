"""The analytic scheduler-balance model of bench.py (reported next to the
measured per-CTA busy times): units in the scheduler's order (documents by tile
count, longest first; head by head; each head's tiles longest work first),
each to the SM that frees up first; the ratio is mean / max of the SMs' tile
work.  Pinned against hand-counted cases and an independent replay."""
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from causal_flash_attention_packed_b200 import workloads as W  # noqa: E402


def _replay(works, num_sms):
    # plain list scheduling: the next unit goes to the least-loaded SM (lowest index on ties)
    loads = [0] * num_sms
    for wk in works:
        i = min(range(num_sms), key=lambda s: (loads[s], s))
        loads[i] += wk
    used = loads[: min(len(works), num_sms)]
    return sum(used) / len(used) / max(used)


def _dq_works(lengths, H):
    nts = [(L + 127) // 128 for L in lengths]
    order = sorted([k for k in range(len(nts)) if nts[k] > 0], key=lambda k: -nts[k])
    return [nts[k] - r for k in order for _ in range(H) for r in range(nts[k])]


def test_one_sm_is_balanced():
    w = W.custom([1000, 300, 129], Hq=4, Hkv=2, d=64)
    for prec in ("bf16", "mxfp8"):
        assert all(v == 1.0 for v in bench.analytic_balance(w, prec, 1).values())


def test_one_unit_per_sm_is_mean_over_max_of_the_units():
    # one document of 8 query tiles, 2 heads, more SMs than units: each SM runs one unit,
    # the dQ units of a head do 8, 7, ..., 1 key tiles -> mean 4.5, max 8
    w = W.custom([1024], Hq=2, Hkv=2, d=128)
    got = bench.analytic_balance(w, "bf16", 148)
    assert got["dq_kernel"] == pytest.approx(4.5 / 8)
    assert got["dkdv_kernel"] == pytest.approx(4.5 / 8)
    # forward, bf16: 256-row units (query tiles 2u, 2u+1) do 4u + 3 key tiles: 15, 11, 7, 3
    assert got["fwd_kernel"] == pytest.approx(np.mean([15, 11, 7, 3]) / 15)


@pytest.mark.parametrize("num_sms", [3, 7, 148])
def test_matches_an_independent_replay(num_sms):
    lengths = [2048, 700, 129, 128, 1, 0, 4000]
    w = W.custom(lengths, Hq=4, Hkv=2, d=64)
    got = bench.analytic_balance(w, "mxfp8", num_sms)
    assert got["dq_kernel"] == pytest.approx(_replay(_dq_works(lengths, 4), num_sms))
    # dK/dV: per KV head, each key tile's unit covers the G = 2 query heads of its group
    kv = [2 * wk for wk in _dq_works(lengths, 2)]
    assert got["dkdv_kernel"] == pytest.approx(_replay(kv, num_sms))
