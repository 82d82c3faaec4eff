"""Pins of the MXFP8 emulation's computed-operand quantisation and of its
backward operand selection (CPU only).

FLAMIA page, sec. "FLAMIA Mimarisi ve Temel Tasarim Ilkeleri": MXFP8 operands
share one E8M0 scale per 32 elements along the contraction, token-block scales
are document-local, leak guards keep future tokens out of shared scales, and
the backward is consistent with the forward.  The oracle's readings of these
(which it states in its header) are pinned here element by element:

  forward P~ -- quantised per (query row, 32-key block) in the form
                2^(S log2 e - M) with an integer reference M, then divided by
                the row sum taken before quantisation;
  dS~        -- per (query row, 32-key block), the operand of dQ = dS K;
  P~T, dS~T  -- per (key row, 32-query block), document-local, the operands
                of dV = P^T dO and dK = dS^T Q;
  dP         -- uses dO in per-token form; dK and dV use Q and dO in
                token-block form.

Each test names the plausible mistakes it fails.  Values marked "by hand" were
worked out in the docstrings; the blocking tests compute their expectations
from closed forms of P and dS, group them into blocks as the rule says and
quantise each block with the oracle's block quantiser (pinned on its own in
test_oracle_quant.py).
"""
import math

import numpy as np
import pytest


def _cu(lengths):
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)


# ---------------------------------------------------------------------------
# forward P~: a hand-derived row
# ---------------------------------------------------------------------------

# key values k_j of the one query row below; its score to key j is k_j ln2 / 4
_BLK0 = [8, 7, 6, 5, 4, 3, 2, 1, 0, -1, -2, -3, -4, -6, -8, -12, -16, -24, -32, -48, -56, -64, -80] + [0] * 9
_BLK1 = [10, 4, -2, -40, 1, 0, 3, -9]
# by hand: decoded P~ (before division by the row sum) of key block 0 and 1
_PT0 = [0.5, 0.40625, 0.34375, 0.3125, 0.25, 0.203125, 0.171875, 0.15625, 0.125, 0.1015625, 0.0859375,
        0.078125, 0.0625, 0.04296875, 0.03125, 0.015625, 0.0078125, 2.0 ** -9, 2.0 ** -11, 2.0 ** -15,
        2.0 ** -17, 0.0, 0.0] + [0.125] * 9
_PT1 = [0.6875, 0.25, 0.0859375, 2.0 ** -13, 0.15625, 0.125, 0.203125, 13.0 / 512]


def _p_tilde_case(shift=0.0):
    """One 40-token document, d = 64, one head, scale ln2/4.  Query 39 (token
    block 1) is e_0 (+ shift e_1); key j holds k_j in channel 0 and 1 in
    channel 1, so S_39,j = (k_j + shift) ln2 / 4 and S log2 e = (k_j + shift)/4.
    V_j = e_j reads P~_39,j out of O_39[j].  Every input is exact in both MX
    forms (the test checks it), so only the quantisation of P acts."""
    T, d = 40, 64
    q = np.zeros((T, 1, d))
    k = np.zeros((T, 1, d))
    v = np.zeros((T, 1, d))
    q[39, 0, 0] = 1.0
    q[39, 0, 1] = shift
    for j, kj in enumerate(_BLK0 + _BLK1):
        k[j, 0, 0] = kj
        k[j, 0, 1] = 1.0
        v[j, 0, j] = 1.0
    return q, k, v, math.log(2.0) / 4


def _assert_exact_in_mx_forms(orc, x, cu):
    f = orc.quantize_mxfp8(x, cu, forms=3)
    slots = f["scale_tb"]
    dec = np.vectorize(orc.e4m3_decode)
    T, H, d = x.shape
    pt = dec(f["val_pt"]) * np.ldexp(1.0, f["scale_pt"].astype(int) - 127).repeat(32, axis=2)
    np.testing.assert_array_equal(pt, x)
    for kdoc in range(len(cu) - 1):
        s, e = cu[kdoc], cu[kdoc + 1]
        for m in range(0, e - s, 32):
            sl = slice(s + m, min(s + m + 32, e))
            sc = np.ldexp(1.0, slots[s // 32 + kdoc + m // 32].astype(int) - 127).repeat(32, axis=1)
            np.testing.assert_array_equal(dec(f["val_tb"][sl]) * sc[None], x[sl])


def test_forward_p_tilde_by_hand(orc):
    """Row 39 by hand.  M = ceil(max_j k_j / 4) = ceil(10/4) = 3, so
    u_j = 2^(k_j/4 - 3).  Key block 0 (keys 0..31): max u = 2^-1 (k = 8), RCEIL
    X = ceil(log2(2^-1 / 448)) = -9, so u 2^9 = 2^(k/4 + 6) is rounded to E4M3:
      k=8: 256 -> 256 (0x78), decoded 256 * 2^-9 = 0.5
      k=7: 215.27 -> 208 (between 208 and 224) -> 0.40625
      k=6: 181.02 -> 176 -> 0.34375;  k=5: 152.22 -> 160 -> 0.3125
      k=4: 128 -> 0.25;  k=3: 107.63 -> 104 -> 0.203125
      k=2: 90.51 -> 88 -> 0.171875;  k=1: 76.11 -> 80 -> 0.15625
      k=0: 64 -> 0.125;  k=-1: 53.82 -> 52 -> 0.1015625
      k=-2: 45.25 -> 44;  k=-3: 38.05 -> 40;  k=-4: 32;  k=-6: 22.63 -> 22
      k=-8: 16;  k=-12: 8;  k=-16: 4;  k=-24: 1 (2^-9);  k=-32: 2^-2 (2^-11)
      k=-48: 2^-6, the smallest normal (2^-15)
      k=-56: 2^-8, subnormal code 0x02 (2 * 2^-9 * 2^-9 = 2^-17)
      k=-64: 2^-10, half the smallest subnormal: a tie, rounds to even = 0
      k=-80: 2^-14 -> 0
    Key block 1 (keys 32..39, its own scale): max u = 2^(10/4 - 3) = 2^-0.5,
    X = ceil(-0.5 - 8.807) = -9 again:
      k=10: 362.04 -> 352 (0x7B) -> 0.6875;  k=4 -> 0.25;  k=-2 -> 0.0859375
      k=-40: 2^-4 (2^-13);  k=1 -> 0.15625;  k=0 -> 0.125;  k=3 -> 0.203125
      k=-9: 13.45 -> 13 (0x55) -> 13/512
    O_39[j] = P~_j / l with l = sum_j u_j taken before quantisation, and
    LSE_39 = ln sum_j 2^(k_j/4).
    Mistakes this fails: normalising P before quantising it, one scale for
    the whole row, blocks not aligned to 32 keys, the row sum taken after
    quantisation, a floor instead of the RCEIL exponent."""
    q, k, v, sc = _p_tilde_case()
    cu = _cu([40])
    _assert_exact_in_mx_forms(orc, q, cu)
    _assert_exact_in_mx_forms(orc, k, cu)
    _assert_exact_in_mx_forms(orc, v, cu)
    o, lse = orc.mx_attn_fwd(q, k, v, cu, sc)
    ks = np.array(_BLK0 + _BLK1, dtype=float)
    ell = float(np.sum(2.0 ** (ks / 4 - 3)))
    want = np.array(_PT0 + _PT1) / ell
    np.testing.assert_allclose(o[39, 0, :40], want, rtol=1e-14, atol=0)
    assert np.all(o[39, 0, 40:] == 0)
    assert abs(lse[0, 39] - math.log(float(np.sum(2.0 ** (ks / 4))))) < 1e-13
    # the alternative "normalise, then quantise" gives other values
    alt = np.concatenate([orc.quant_block(2.0 ** (ks[:32] / 4 - 3) / ell)[1],
                          orc.quant_block(2.0 ** (ks[32:] / 4 - 3) / ell)[1]])
    assert np.max(np.abs(alt - want) / want.max()) > 1e-2


@pytest.mark.parametrize("shift", [12.0, -12.0])
def test_forward_p_tilde_does_not_depend_on_the_integer_reference(orc, shift):
    """A uniform shift of the row's scores by +-12 ln2/4 moves M by exactly
    +-3 and leaves every code unchanged: O_39 is the same to rounding and LSE
    moves by +-3 ln 2.  MX quantisation is invariant under powers of two, which
    is why any integer running reference of a one-pass kernel gives the
    oracle's codes.  Fails a reference that is not an integer power of two."""
    cu = _cu([40])
    q0, k, v, sc = _p_tilde_case()
    q1, _, _, _ = _p_tilde_case(shift)
    _assert_exact_in_mx_forms(orc, q1, cu)
    o0, lse0 = orc.mx_attn_fwd(q0, k, v, cu, sc)
    o1, lse1 = orc.mx_attn_fwd(q1, k, v, cu, sc)
    np.testing.assert_allclose(o1[39], o0[39], rtol=1e-13, atol=1e-16)
    assert abs(lse1[0, 39] - lse0[0, 39] - shift / 4 * math.log(2.0)) < 1e-12


# ---------------------------------------------------------------------------
# backward blocks: one-hot read-outs of P~T, dS~T and dS~
# ---------------------------------------------------------------------------

_LEAD = 17   # a first document of 17 tokens: the second one starts off the 32-token grid
_L = 40      # the second document: doc-local query blocks [0, 32) and [32, 40)


def _readout_case(seed):
    """Two documents (17 and 40 tokens), one head, d = 128, scale 1.
    In the second document, with doc-local index li of a query and lj of a
    key: Q_i = e_li + a_i e_127, K_j = e_(64+lj) + b_j e_127, dO_i = e_li, so
    S_ij = a_i b_j, dP_ij = V_j[li], D_i = dO_i . O_i = O_i[li], and the
    backward's outputs read the quantised operands out one by one:
      dV_j[li]      = P~T_ji   (dO~tb one-hot)
      dK_j[li]      = dS~T_ji  (Q~tb one-hot in channel li)
      dQ_i[64 + lj] = dS~_ij   (K~ one-hot in channel 64 + lj)
    Range is planted, because MX rounding depends on the blocking only through
    the block scale's range (values far below the block maximum go subnormal
    or to zero): a_i = -4 in query block 0 and +4 in block 1, b_5 = 4 (other
    b_j = 0), so P_(i,5) is about e^-16 / li in block 0 and about 1 in
    block 1; V_j[c] (c < 40) are powers of two in [2^-3, 2^3] or 0, with
    V_2[35] = 2^14 and V_3[35] = -2^14 (so dS_(35,2) = -dS_(35,3) = 2^14/36
    while D_35 stays small).  Every input is exact in both MX forms, so only
    the quantisation of the computed operands acts.  The first document holds
    zeros."""
    rng = np.random.default_rng(seed)
    T, d = _LEAD + _L, 128
    q = np.zeros((T, 1, d))
    k = np.zeros((T, 1, d))
    v = np.zeros((T, 1, d))
    do = np.zeros((T, 1, d))
    for li in range(_L):
        t = _LEAD + li
        q[t, 0, li] = 1.0
        q[t, 0, 127] = -4.0 if li < 32 else 4.0
        k[t, 0, 64 + li] = 1.0
        do[t, 0, li] = 1.0
    k[_LEAD + 5, 0, 127] = 4.0
    vals = rng.choice([-1.0, 1.0], size=(_L, 40)) * 2.0 ** rng.integers(-3, 4, size=(_L, 40))
    vals[rng.random((_L, 40)) < 0.3] = 0.0
    v[_LEAD:, 0, :40] = vals
    v[_LEAD + 2, 0, 35] = 2.0 ** 14
    v[_LEAD + 3, 0, 35] = -(2.0 ** 14)
    return q, k, v, do


def _closed_forms(orc, q, k, v):
    """P and dS of the second document ([query li][key lj]) from the
    definitions: S = Q K^T, P = softmax over j <= i, the forward's P~ quantised
    per (row, 32-key block) as 2^(S log2 e - M) and divided by the row sum,
    O_i[li] = sum_j P~_ij V_j[li] = D_i, dS = P (V_j[li] - D_i)."""
    sl = slice(_LEAD, _LEAD + _L)
    Q, K, V = q[sl, 0], k[sl, 0], v[sl, 0, :40]
    S = Q @ K.T
    P = np.zeros((_L, _L))
    dS = np.zeros((_L, _L))
    log2e = 1.4426950408889634
    for li in range(_L):
        n = li + 1
        s = S[li, :n]
        p = np.exp(s - s.max())
        P[li, :n] = p / p.sum()
        u = np.exp2(s * log2e - math.ceil((s * log2e).max()))
        pf = np.concatenate([orc.quant_block(u[b:b + 32])[1] for b in range(0, n, 32)]) / u.sum()
        D = float(pf @ V[:n, li])
        dS[li, :n] = P[li, :n] * (V[:n, li] - D)
    return P, dS


def _quant_blocks(orc, x, blocks):
    """Quantise each index set in `blocks` as one MX block; returns the
    dequantised array."""
    out = np.zeros_like(x)
    flat = x.reshape(-1)
    res = out.reshape(-1)
    for idx in blocks:
        res[idx] = orc.quant_block(flat[idx])[1]
    return out


def _row_blocks(shape, starts):
    """Index sets (flat) of row r, columns [s, e) for consecutive starts."""
    n, m = shape
    blocks = []
    for r in range(n):
        for a, b in zip(starts[:-1], starts[1:]):
            blocks.append(np.array([r * m + c for c in range(a, min(b, m))], dtype=np.int64))
    return blocks


def _col_blocks(shape, starts):
    n, m = shape
    blocks = []
    for c in range(m):
        for a, b in zip(starts[:-1], starts[1:]):
            blocks.append(np.array([r * m + c for r in range(a, min(b, n))], dtype=np.int64))
    return blocks


LOCAL = [0, 32, 40]                  # document-local 32-blocks
GLOBAL = [0, 32 - _LEAD, 40]         # 32-blocks of the packed token axis (token 32 is li = 15)
WHOLE = [0, 40]                      # one scale for the whole row / column


@pytest.mark.parametrize("seed", [0, 1])
def test_backward_blocks_of_p_t_ds_t_and_ds(orc, seed):
    """P~T and dS~T are quantised per (key, document-local 32-query block), dS~
    per (query, document-local 32-key block); each read out of dV, dK, dQ as
    the readout case describes, and compared with the closed forms quantised
    block by block.  Mistakes this fails (each checked to give other values
    here): quantising P~T or dS~T along keys instead of queries, blocks of the
    packed token axis instead of document-local ones, one scale per column or
    row, dS~ blocked along queries."""
    q, k, v, do = _readout_case(seed)
    cu = _cu([_LEAD, _L])
    for x in (q, k, v, do):
        _assert_exact_in_mx_forms(orc, x, cu)
    out = orc.mx_attn_bwd(q, k, v, do, cu, 1.0)
    P, dS = _closed_forms(orc, q, k, v)
    sl = slice(_LEAD, _LEAD + _L)
    got_pt = out["dv"][sl, 0, :40].T    # [li][lj] = P~T_(lj, li)
    got_dst = out["dk"][sl, 0, :40].T   # [li][lj] = dS~T_(lj, li)
    got_ds = out["dq"][sl, 0, 64:104]   # [li][lj] = dS~_(li, lj)

    want_pt = _quant_blocks(orc, P, _col_blocks(P.shape, LOCAL))
    want_dst = _quant_blocks(orc, dS, _col_blocks(dS.shape, LOCAL))
    want_ds = _quant_blocks(orc, dS, _row_blocks(dS.shape, LOCAL))
    for got, want in ((got_pt, want_pt), (got_dst, want_dst), (got_ds, want_ds)):
        np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-14 * np.max(np.abs(want)))

    def differs(a, b):
        return float(np.max(np.abs(a - b) / (np.abs(b) + 1e-300))) > 0.5

    # every plausible mistake moves some element by more than half its value
    for starts in (GLOBAL, WHOLE):
        assert differs(_quant_blocks(orc, P, _col_blocks(P.shape, starts)), want_pt)
        assert differs(_quant_blocks(orc, dS, _col_blocks(dS.shape, starts)), want_dst)
        assert differs(_quant_blocks(orc, dS, _row_blocks(dS.shape, starts)), want_ds)
    assert differs(_quant_blocks(orc, P, _row_blocks(P.shape, LOCAL)), want_pt)     # P~T along keys
    assert differs(_quant_blocks(orc, dS, _row_blocks(dS.shape, LOCAL)), want_dst)  # dS~T along keys
    assert differs(_quant_blocks(orc, dS, _col_blocks(dS.shape, LOCAL)), want_ds)   # dS~ along queries


def _selection_rows(T, d):
    """Token 2 holds 8192 in channel 1 and token 5 holds 0.2890625 in channel
    0 (both in token block 0 of a one-document, 40-token problem): the
    token-block form of token 5's value is 0.3125, the per-token form
    0.28125 (block scale 2^5 vs 2^-10; see test_oracle_mx)."""
    x = np.zeros((T, 1, d))
    x[2, 0, 1] = 8192.0
    x[5, 0, 0] = 0.2890625
    return x


def test_dp_uses_per_token_do(orc):
    """dP = dO~pt V~^T.  Planted dO (selection rows), V_0 = e_0, Q_5 = e_3,
    K = 0 (so P_5j = 1/6), scale 1, one 40-token document, d = 32.  By hand:
      O_5 = V_0 / 6, D_5 = dO_5 . O_5 = 0.2890625 / 6 (bf16 dO, unquantised);
      dP_(5,0) = dO~pt_5[0] = 0.28125, so dS_(5,0) = (0.28125 - D_5) / 6
        = 0.0388455...;
      dS~T of key 0, query block 0 holds only that value: X = ceil(log2(
        0.0388455 / 448)) = -13, 0.0388455 * 8192 = 318.2 -> 320, i.e. 0.0390625;
      dK_0[3] = dS~T_(0,5) Q~tb_5[3] = 0.0390625.
    With the token-block dO (0.3125) the same steps give 0.044054 * 8192 =
    360.9 -> 352 = 0.04296875.  Fails dO~tb in dP."""
    T, d = 40, 32
    do = _selection_rows(T, d)
    v = np.zeros((T, 1, d))
    v[0, 0, 0] = 1.0
    q = np.zeros((T, 1, d))
    q[5, 0, 3] = 1.0
    k = np.zeros((T, 1, d))
    out = orc.mx_attn_bwd(q, k, v, do, _cu([T]), 1.0)
    assert out["dk"][0, 0, 3] == 0.0390625
    assert out["dk"][0, 0, 3] != 0.04296875


def test_dk_uses_token_block_q_and_dv_token_block_do(orc):
    """dK = scale dS~T Q~tb and dV = P~T dO~tb.  One 40-token document, d = 32,
    scale 1, K = 0 (P_ij = 1/(i+1)).
    dK case: Q = selection rows, V_0 = e_2, dO_5 = e_2.  By hand: O_i[2] =
      1/(i+1), D_5 = 1/6, dP_(5,0) = 1, dS_(5,0) = (1/6)(1 - 1/6) = 5/36; key
      0's query block 0 holds only it: X = -11, 5/36 * 2048 = 284.4 -> 288,
      i.e. 0.140625; dK_0[0] = 0.140625 * Q~tb_5[0] = 0.140625 * 0.3125
      = 0.0439453125 (per-token Q would give 0.140625 * 0.28125).
    dV case: dO = selection rows, V = 0.  P~T of key 0, query block 0 =
      {1/(i+1), i = 0..31}: X = -8, 256/6 = 42.67 -> 44, so P~T_(0,5) =
      44/256 = 0.171875; dV_0[0] = 0.171875 * dO~tb_5[0] = 0.171875 * 0.3125
      = 0.0537109375 (per-token dO would give 0.171875 * 0.28125).
    Fails per-token Q or dO in the query contraction."""
    T, d = 40, 32
    sel = _selection_rows(T, d)
    zeros = np.zeros((T, 1, d))
    v = np.zeros((T, 1, d))
    v[0, 0, 2] = 1.0
    do = np.zeros((T, 1, d))
    do[5, 0, 2] = 1.0
    out = orc.mx_attn_bwd(sel, zeros, v, do, _cu([T]), 1.0)
    assert out["dk"][0, 0, 0] == 0.0439453125
    out = orc.mx_attn_bwd(zeros, zeros, zeros, sel, _cu([T]), 1.0)
    assert out["dv"][0, 0, 0] == 0.0537109375


def test_study_switches_reach_the_exact_oracle(orc):
    """The accuracy-study switches of the emulation (oracle/mx_accuracy_study.py)
    each take one quantisation out; with all three out (inputs, P~/P~T,
    dS~/dS~T) the emulation is the exact oracle on any inputs.  With the
    symmetric guard, dK on the diagonal query block uses the per-token Q: in
    the hand case of test_dk_uses_token_block_q_and_dv_token_block_do that is
    0.140625 * 0.28125."""
    rng = np.random.default_rng(5)
    cu = _cu([45, 1, 70, 33])
    T, Hq, Hkv, d, sc = cu[-1], 4, 2, 64, 0.125
    q, k, v, do = (rng.standard_normal((T, H, d)) for H in (Hq, Hkv, Hkv, Hq))
    ex = orc.attn_bwd(q, k, v, do, cu, sc)
    flags = orc.MX_QUANT_P | orc.MX_KEEP_INPUTS | orc.MX_KEEP_P | orc.MX_KEEP_DS
    mx = orc.mx_attn_bwd(q, k, v, do, cu, sc, flags=flags)
    for key in ex:
        np.testing.assert_allclose(mx[key], ex[key], rtol=0, atol=1e-12, err_msg=key)
    T, d = 40, 32
    sel = _selection_rows(T, d)
    zeros = np.zeros((T, 1, d))
    v = np.zeros((T, 1, d))
    v[0, 0, 2] = 1.0
    do = np.zeros((T, 1, d))
    do[5, 0, 2] = 1.0
    out = orc.mx_attn_bwd(sel, zeros, v, do, _cu([T]), 1.0, flags=orc.MX_QUANT_P | orc.MX_SYM_GUARD)
    assert out["dk"][0, 0, 0] == 0.140625 * 0.28125
