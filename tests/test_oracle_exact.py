"""Pins of the exact fp64 oracle against closed forms, a library routine and
invariants (CPU only).

Pages: "GPT Kernel Programlama: MatMul, Softmax ve Attention Hesabi" sec. 3-6
(S = QK^T/sqrt(d), causal mask, stable softmax, O = PV); FLAMIA page, sec.
"FLAMIA Mimarisi ve Temel Tasarim Ilkeleri" (packed documents, no repacking).
Each test is chosen so that a plausible mistake in the oracle -- a dropped
term, a wrong sign or index, a transposed operand, a wrong head map -- fails.
"""
import math

import numpy as np
import pytest
import torch


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _cu(lengths):
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)


def test_q_zero_uniform_attention(orc):
    """Q = 0: P_ij = 1/(i-s+1), O_i = prefix mean of V, LSE_i = ln(i-s+1), dK = 0."""
    rng = np.random.default_rng(1)
    lengths = [7, 1, 12, 5]
    cu = _cu(lengths)
    T, Hq, Hkv, d = cu[-1], 4, 2, 8
    q = np.zeros((T, Hq, d))
    k, v, do = _rand(rng, T, Hkv, d), _rand(rng, T, Hkv, d), _rand(rng, T, Hq, d)
    out = orc.attn_bwd(q, k, v, do, cu, 0.37)
    for kd in range(len(lengths)):
        s, e = cu[kd], cu[kd + 1]
        for i in range(s, e):
            n = i - s + 1
            for h in range(Hq):
                g = h // (Hq // Hkv)
                np.testing.assert_allclose(out["o"][i, h], v[s:i + 1, g].mean(0), rtol=0, atol=1e-13)
                assert abs(out["lse"][h, i] - math.log(n)) < 1e-13
    np.testing.assert_allclose(out["dk"], 0.0, atol=1e-13)


def test_one_token_document(orc):
    """A one-token document: O = V, LSE = scale q.k, dQ = dK = 0, dV = dO."""
    rng = np.random.default_rng(2)
    cu = _cu([5, 1, 4])
    T, Hq, Hkv, d, sc = cu[-1], 2, 2, 16, 0.25
    q, k, v, do = (_rand(rng, T, Hq, d), _rand(rng, T, Hkv, d), _rand(rng, T, Hkv, d),
                   _rand(rng, T, Hq, d))
    out = orc.attn_bwd(q, k, v, do, cu, sc)
    i = 5
    for h in range(Hq):
        np.testing.assert_allclose(out["o"][i, h], v[i, h], atol=1e-14)
        assert abs(out["lse"][h, i] - sc * float(q[i, h] @ k[i, h])) < 1e-13
        np.testing.assert_allclose(out["dq"][i, h], 0.0, atol=1e-14)
        np.testing.assert_allclose(out["dk"][i, h], 0.0, atol=1e-14)
        np.testing.assert_allclose(out["dv"][i, h], do[i, h], atol=1e-14)


def test_constant_v(orc):
    """V_j = c for every key: O_i = c and dQ = dK = 0 (dP_ij = D_i)."""
    rng = np.random.default_rng(3)
    cu = _cu([9, 13])
    T, Hq, Hkv, d = cu[-1], 2, 1, 8
    q, k, do = _rand(rng, T, Hq, d), _rand(rng, T, Hkv, d), _rand(rng, T, Hq, d)
    c = rng.standard_normal(d)
    v = np.broadcast_to(c, (T, Hkv, d)).copy()
    out = orc.attn_bwd(q, k, v, do, cu, 0.5)
    np.testing.assert_allclose(out["o"], np.broadcast_to(c, (T, Hq, d)), atol=1e-13)
    np.testing.assert_allclose(out["dq"], 0.0, atol=1e-12)
    np.testing.assert_allclose(out["dk"], 0.0, atol=1e-12)


def test_rows_sum_to_one_and_causal(orc):
    """With V_j = e_(j-s) (one-hot of the key's position), O_i is row i of P:
    it sums to 1 and is exactly zero at j > i and outside the document."""
    rng = np.random.default_rng(4)
    lengths = [11, 6, 16]
    cu = _cu(lengths)
    T, d = cu[-1], 16
    q, k = _rand(rng, T, 1, d) * 2.0, _rand(rng, T, 1, d) * 2.0
    v = np.zeros((T, 1, d))
    for kd in range(len(lengths)):
        for j in range(cu[kd], cu[kd + 1]):
            v[j, 0, j - cu[kd]] = 1.0
    o, _ = orc.attn_fwd(q, k, v, cu, 0.3)
    for kd in range(len(lengths)):
        s, e = cu[kd], cu[kd + 1]
        for i in range(s, e):
            row = o[i, 0]
            assert abs(row.sum() - 1.0) < 1e-14
            assert np.all(row[i - s + 1:] == 0.0)
            assert np.all(row[: i - s + 1] > 0.0)


@pytest.mark.parametrize("G", [1, 2])
def test_single_document_matches_torch_sdpa(orc, G):
    """One document: O, LSE and the gradients equal torch's fp64 CPU causal
    scaled_dot_product_attention (K/V repeated over contiguous head groups)."""
    rng = np.random.default_rng(5 + G)
    T, Hkv, d, sc = 40, 2, 32, 0.21
    Hq = Hkv * G
    q, k, v, do = (_rand(rng, T, Hq, d), _rand(rng, T, Hkv, d), _rand(rng, T, Hkv, d),
                   _rand(rng, T, Hq, d))
    cu = _cu([T])
    out = orc.attn_bwd(q, k, v, do, cu, sc)
    tq = torch.tensor(q).permute(1, 0, 2).requires_grad_(True)
    tk = torch.tensor(k).permute(1, 0, 2).requires_grad_(True)
    tv = torch.tensor(v).permute(1, 0, 2).requires_grad_(True)
    kr = tk.repeat_interleave(G, dim=0)
    vr = tv.repeat_interleave(G, dim=0)
    to = torch.nn.functional.scaled_dot_product_attention(tq, kr, vr, is_causal=True, scale=sc)
    to.backward(torch.tensor(do).permute(1, 0, 2))
    np.testing.assert_allclose(out["o"], to.detach().permute(1, 0, 2).numpy(), atol=1e-12)
    np.testing.assert_allclose(out["dq"], tq.grad.permute(1, 0, 2).numpy(), atol=1e-12)
    np.testing.assert_allclose(out["dk"], tk.grad.permute(1, 0, 2).numpy(), atol=1e-12)
    np.testing.assert_allclose(out["dv"], tv.grad.permute(1, 0, 2).numpy(), atol=1e-12)
    s = torch.einsum("htd,hsd->hts", tq.detach(), kr.detach()) * sc
    s = s.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), 1), float("-inf"))
    np.testing.assert_allclose(out["lse"], torch.logsumexp(s, -1).numpy(), atol=1e-12)


def test_packing_equals_separate_calls_and_permutation(orc):
    """Packed output equals separate per-document calls; permuting the
    documents permutes the outputs (no information crosses documents)."""
    rng = np.random.default_rng(6)
    lengths = [9, 3, 14, 1, 6]
    cu = _cu(lengths)
    T, Hq, Hkv, d, sc = cu[-1], 4, 2, 8, 0.4
    q, k, v, do = (_rand(rng, T, Hq, d), _rand(rng, T, Hkv, d), _rand(rng, T, Hkv, d),
                   _rand(rng, T, Hq, d))
    full = orc.attn_bwd(q, k, v, do, cu, sc)
    for kd in range(len(lengths)):
        s, e = cu[kd], cu[kd + 1]
        one = orc.attn_bwd(q[s:e], k[s:e], v[s:e], do[s:e], _cu([e - s]), sc)
        for key in ("o", "dq", "dk", "dv"):
            np.testing.assert_array_equal(full[key][s:e], one[key])
        np.testing.assert_array_equal(full["lse"][:, s:e], one["lse"])
    perm = [3, 0, 4, 2, 1]
    idx = np.concatenate([np.arange(cu[p], cu[p + 1]) for p in perm])
    cu2 = _cu([lengths[p] for p in perm])
    pout = orc.attn_bwd(q[idx], k[idx], v[idx], do[idx], cu2, sc)
    for key in ("o", "dq", "dk", "dv"):
        np.testing.assert_array_equal(pout[key], full[key][idx])


def test_zero_length_documents(orc):
    """Zero-length documents produce nothing and change nothing."""
    rng = np.random.default_rng(7)
    q, k, v, do = (_rand(rng, 10, 2, 8), _rand(rng, 10, 1, 8), _rand(rng, 10, 1, 8),
                   _rand(rng, 10, 2, 8))
    a = orc.attn_bwd(q, k, v, do, _cu([4, 6]), 0.3)
    b = orc.attn_bwd(q, k, v, do, _cu([0, 4, 0, 0, 6, 0]), 0.3)
    for key in a:
        np.testing.assert_array_equal(a[key], b[key])


def test_finite_difference_gradients(orc):
    """Central differences (h = 1e-6) of L = sum(O * dO) on tiny inputs
    (3 documents, G = 2): relative error <= 1e-6 for dQ, dK, dV."""
    rng = np.random.default_rng(8)
    cu = _cu([6, 1, 9])
    T, Hq, Hkv, d, sc = cu[-1], 4, 2, 4, 0.45
    q, k, v, do = (_rand(rng, T, Hq, d), _rand(rng, T, Hkv, d), _rand(rng, T, Hkv, d),
                   _rand(rng, T, Hq, d))
    out = orc.attn_bwd(q, k, v, do, cu, sc)

    def loss(qq, kk, vv):
        o, _ = orc.attn_fwd(qq, kk, vv, cu, sc)
        return float(np.sum(o * do))

    h = 1e-6
    for name, x, g in (("q", q, out["dq"]), ("k", k, out["dk"]), ("v", v, out["dv"])):
        num = np.zeros_like(x)
        for ix in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[ix] += h
            xm[ix] -= h
            trip_p = [q, k, v]
            trip_m = [q, k, v]
            pos = "qkv".index(name)
            trip_p[pos], trip_m[pos] = xp, xm
            num[ix] = (loss(*trip_p) - loss(*trip_m)) / (2 * h)
        err = np.linalg.norm(num - g) / np.linalg.norm(g)
        assert err <= 1e-6, (name, err)


def test_sampled_rows_and_columns_match_full(orc):
    """The per-row (O, LSE, dQ) and per-key (dK, dV) samplers used for
    full-size parity agree with the full oracle."""
    rng = np.random.default_rng(9)
    cu = _cu([33, 1, 70, 20])
    T, Hq, Hkv, d, sc = cu[-1], 4, 2, 16, 0.25
    q, k, v, do = (_rand(rng, T, Hq, d), _rand(rng, T, Hkv, d), _rand(rng, T, Hkv, d),
                   _rand(rng, T, Hq, d))
    full = orc.attn_bwd(q, k, v, do, cu, sc)
    tok = rng.integers(0, T, 40)
    head = rng.integers(0, Hq, 40)
    o, lse, dq = orc.attn_rows(q, k, v, do, cu, sc, tok, head)
    np.testing.assert_allclose(o, full["o"][tok, head], atol=1e-12)
    np.testing.assert_allclose(lse, full["lse"][head, tok], atol=1e-12)
    np.testing.assert_allclose(dq, full["dq"][tok, head], atol=1e-12)
    kvh = rng.integers(0, Hkv, 40)
    dk, dv = orc.attn_kv_cols(q, k, v, do, cu, sc, tok, kvh)
    np.testing.assert_allclose(dk, full["dk"][tok, kvh], atol=1e-12)
    np.testing.assert_allclose(dv, full["dv"][tok, kvh], atol=1e-12)
    # the forward rows alone, and the keys' gradients from the full oracle's
    # forward rows (P = exp(S - LSE), D = dO . O, no row recomputed)
    for doc in range(len(cu) - 1):
        for h in range(Hq):
            o2, lse2 = orc.attn_fwd_doc(q, k, v, cu, sc, doc, h)
            np.testing.assert_allclose(o2, full["o"][cu[doc]:cu[doc + 1], h], atol=1e-12)
            np.testing.assert_allclose(lse2, full["lse"][h, cu[doc]:cu[doc + 1]], atol=1e-12)
    dk2, dv2 = orc.attn_kv_cols_from_rows(q, k, v, do, full["o"], full["lse"], cu, sc, tok, kvh)
    np.testing.assert_allclose(dk2, full["dk"][tok, kvh], atol=1e-12)
    np.testing.assert_allclose(dv2, full["dv"][tok, kvh], atol=1e-12)
    # a wrong row state moves them: the planted mistake of an LSE off by 0.1
    dk3, _ = orc.attn_kv_cols_from_rows(q, k, v, do, full["o"], full["lse"] + 0.1, cu, sc, tok, kvh)
    assert np.max(np.abs(dk3 - full["dk"][tok, kvh])) > 1e-3


def test_future_perturbation_leaves_past_bit_identical(orc):
    """Causal safety of the oracle itself: randomising every token after t
    (and every later document) leaves O, LSE, dQ at positions <= t unchanged
    bit for bit; with dO_{>t} = 0 in both runs dK, dV at positions <= t are
    unchanged too."""
    rng = np.random.default_rng(10)
    cu = _cu([20, 30, 10])
    T, Hq, Hkv, d, sc = cu[-1], 2, 1, 8, 0.3
    q, k, v, do = (_rand(rng, T, Hq, d), _rand(rng, T, Hkv, d), _rand(rng, T, Hkv, d),
                   _rand(rng, T, Hq, d))
    t = 20 + 13
    q2, k2, v2, do2 = q.copy(), k.copy(), v.copy(), do.copy()
    for x in (q2, k2, v2, do2):
        x[t + 1:] = rng.standard_normal(x[t + 1:].shape)
    a = orc.attn_bwd(q, k, v, do, cu, sc)
    b = orc.attn_bwd(q2, k2, v2, do2, cu, sc)
    for key in ("o", "dq"):
        np.testing.assert_array_equal(a[key][: t + 1], b[key][: t + 1])
    np.testing.assert_array_equal(a["lse"][:, : t + 1], b["lse"][:, : t + 1])
    do[t + 1:] = 0
    do2[t + 1:] = 0
    a = orc.attn_bwd(q, k, v, do, cu, sc)
    b = orc.attn_bwd(q2, k2, v2, do2, cu, sc)
    for key in ("dk", "dv"):
        np.testing.assert_array_equal(a[key][: t + 1], b[key][: t + 1])


def test_qkv_projection_split(orc):
    """The projection's head split: with d_model = (Hq + 2 Hkv) d and W the
    identity, q, k and v are consecutive column slices of x (Q heads first,
    then K, then V); a permutation of W's rows permutes the outputs the same
    way.  Fails a wrong head order or a transposed W."""
    rng = np.random.default_rng(12)
    Hq, Hkv, d, T = 2, 1, 4, 5
    n = (Hq + 2 * Hkv) * d
    x = rng.standard_normal((T, n))
    q, k, v = orc.qkv_proj(x, np.eye(n), Hq, Hkv, d)
    np.testing.assert_array_equal(q.reshape(T, -1), x[:, : Hq * d])
    np.testing.assert_array_equal(k.reshape(T, -1), x[:, Hq * d: (Hq + Hkv) * d])
    np.testing.assert_array_equal(v.reshape(T, -1), x[:, (Hq + Hkv) * d:])
    perm = rng.permutation(n)
    q2, k2, v2 = orc.qkv_proj(x, np.eye(n)[perm], Hq, Hkv, d)
    y2 = np.concatenate([q2.reshape(T, -1), k2.reshape(T, -1), v2.reshape(T, -1)], axis=1)
    np.testing.assert_array_equal(y2, x[:, perm])
    # a non-square W: row r of W gives output column r
    w = rng.standard_normal((n, 3))
    x3 = rng.standard_normal((T, 3))
    q3, _, _ = orc.qkv_proj(x3, w, Hq, Hkv, d)
    assert abs(q3[2, 1, 3] - float(x3[2] @ w[1 * d + 3])) < 1e-13
