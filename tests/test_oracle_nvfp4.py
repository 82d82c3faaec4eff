"""Pins of the oracle's mixed NVFP4/FP8 path (CPU only).

FLAMIA page, sec. "FLAMIA Mimarisi ve Temel Tasarim Ilkeleri": besides MXFP8,
the kernel family has mixed NVFP4/FP8 training paths, and the forward and
backward stay numerically consistent.  The oracle's reading (stated in its
header): the scores S = Q K^T take Q and K in NVFP4 -- E2M1 codes, one E4M3
scale per 16 channels of one token, a per-tensor fp32 decode scale g -- in the
forward and in the backward's recomputation; every other product is the MXFP8
path's.

Each test names the plausible mistakes it fails.  Values marked "by hand" are
worked out in the docstrings.
"""
import numpy as np
import pytest

# the E2M1 magnitudes of codes 0..7 (1 sign, 2 exponent bits with bias 1, 1 mantissa bit)
_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _cu(lengths):
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)


# ---------------------------------------------------------------------------
# E2M1 element codes
# ---------------------------------------------------------------------------

def _e2m1_brute(y):
    """Nearest E2M1 value by exhaustive search (ties: the even code), sign kept,
    |y| >= 6 saturating; a zero result is code 0."""
    a = abs(y)
    best = min(range(8), key=lambda c: (abs(_E2M1[c] - a), c & 1))
    if best == 0:
        return 0
    return best | (8 if y < 0 else 0)


def test_e2m1_decode_and_round_trip(orc):
    """Codes 0..15 decode to +-{0, .5, 1, 1.5, 2, 3, 4, 6}; every non-zero code
    encodes back to itself.  Fails: a wrong exponent bias, a swapped sign bit,
    a subnormal decoded as normal."""
    for c in range(16):
        v = orc.e2m1_decode(c)
        assert abs(v) == _E2M1[c & 7] and (v < 0) == (c >= 8 and c != 8) or (c == 8 and v == 0.0)
        if c & 7:
            assert orc.e2m1_encode(v) == c


def test_e2m1_rounding_against_brute_force(orc):
    """Every midpoint between neighbours, points just off each midpoint and a
    dense sweep agree with an exhaustive nearest search.  Fails: ties rounded
    away from zero (0.25 -> 0.5, 2.5 -> 3, 5 -> 6), no saturation above 6, a
    negative zero code, the quantum of the wrong binade."""
    mids = [(a + b) / 2 for a, b in zip(_E2M1, _E2M1[1:])]
    ys = []
    for m in mids:
        ys += [m, np.nextafter(m, 0.0), np.nextafter(m, 10.0)]
    ys += list(np.linspace(-7.5, 7.5, 6001)) + [6.0, 6.5, 7.0, 1e9, -1e9, -0.0, 1e-30, -1e-30]
    for y in ys:
        assert orc.e2m1_encode(float(y)) == _e2m1_brute(float(y)), y
    # the ties by hand: 0.25 -> 0, 0.75 -> 1 (code 2), 1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4
    assert [orc.e2m1_encode(y) for y in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)] == [0, 2, 2, 4, 4, 6, 6]


# ---------------------------------------------------------------------------
# NVFP4 blocks
# ---------------------------------------------------------------------------

def test_nv_block_by_hand(orc):
    """x = (2.5, 6, 0 ...), g = 3, by hand: a = 6, a / (6 g) = 1/3, whose
    nearest E4M3 values are 0.3125 and 0.34375 -> s = 0.34375 (byte 0x2B:
    exponent 5, mantissa 3); s g = 1.03125, r = 1/1.03125 = 0.9696...;
    6 r = 5.818 -> 6, 2.5 r = 2.424 -> 2; dequantised 2 * 1.03125 = 2.0625 and
    6 * 1.03125 = 6.1875.  x = (1, 0 ...), g = 1: 1/6 -> s = 0.171875 (0x23),
    r = 5.818, 1 -> 6, dequantised 1.03125.  Fails: the scale taken as a power
    of two, no division by 6, g left out of the scale or of the values,
    truncation instead of rounding."""
    c, dq, sb = orc.nv_quant_block([2.5, 6.0] + [0.0] * 14, 3.0)
    assert sb == 0x2B and list(c[:2]) == [4, 7] and not c[2:].any()
    np.testing.assert_array_equal(dq[:2], [2.0625, 6.1875])
    c, dq, sb = orc.nv_quant_block([1.0] + [0.0] * 15, 1.0)
    assert sb == 0x23 and c[0] == 7 and dq[0] == 1.03125
    # an all-zero block: scale 0, codes 0
    c, dq, sb = orc.nv_quant_block([0.0] * 16, 1.0)
    assert sb == 0 and not c.any() and not dq.any()


@pytest.mark.parametrize("g", [1.0, 0.5, 4.0])
def test_nv_block_exact_on_grid(orc, g):
    """A block whose largest magnitude is 6 c (c a power of two) and whose other
    values are E2M1 magnitudes times c is reproduced exactly, for power-of-two
    g.  Fails: any stray factor in the scale or the dequantisation."""
    rng = np.random.default_rng(1)
    for c in (2.0 ** -3, 1.0, 8.0):
        x = rng.choice(_E2M1, 16) * rng.choice([-1, 1], 16) * c
        x[rng.integers(16)] = -6.0 * c
        _, dq, sb = orc.nv_quant_block(x, g)
        np.testing.assert_array_equal(dq, x)
        assert orc.e4m3_decode(sb) == c / g


def test_nv_block_codes_follow_the_scaled_values(orc):
    """Random blocks: every code is the brute-force E2M1 rounding of x r with
    r = 1/(decode(s) g) in fp32, and no dequantised magnitude exceeds 6 s g.
    Fails: rounding done on x / s in fp64 instead of the stated fp32 steps
    (differs near ties), saturation missing."""
    rng = np.random.default_rng(2)
    for g in (1.0, 0.37):
        for _ in range(200):
            x = (rng.standard_normal(16) * np.exp(rng.uniform(-4, 4))).astype(np.float32).astype(np.float64)
            codes, dq, sb = orc.nv_quant_block(x, g)
            sg = np.float32(orc.e4m3_decode(sb)) * np.float32(g)
            r = np.float32(1.0) / sg if sg > 0 else np.float32(0.0)
            for xi, ci in zip(x, codes):
                assert ci == _e2m1_brute(float(np.float32(xi) * r))
            assert np.all(np.abs(dq) <= 6.0 * float(sg) * (1 + 1e-6))  # sg is rounded to fp32


def test_quantize_nvfp4_layout(orc):
    """The tensor quantiser packs channel 2i into the low nibble of byte i and
    lays the 16-channel scales out as [T][H][d/16], each block quantised alone
    (per token: no block spans two tokens).  Fails: swapped nibbles, blocks of
    32, scales of another token or head."""
    rng = np.random.default_rng(3)
    T, H, d = 5, 3, 64
    x = rng.standard_normal((T, H, d)).astype(np.float32).astype(np.float64)
    x[2, 1, 16:32] *= 1000.0  # one loud block must not touch its neighbours
    codes, scales = orc.quantize_nvfp4(x, 0.5)
    assert codes.shape == (T, H, d // 2) and scales.shape == (T, H, d // 16)
    for t in range(T):
        for h in range(H):
            for b in range(d // 16):
                c, _, sb = orc.nv_quant_block(x[t, h, 16 * b:16 * b + 16], 0.5)
                assert scales[t, h, b] == sb
                packed = codes[t, h, 8 * b:8 * b + 8]
                np.testing.assert_array_equal(packed & 15, c[0::2])
                np.testing.assert_array_equal(packed >> 4, c[1::2])


# ---------------------------------------------------------------------------
# the mixed attention emulation
# ---------------------------------------------------------------------------

def _nv_grid(rng, c, *shape):
    """E2M1 magnitudes times c with one -6 c in every 16-channel block: exact
    in NVFP4 (power-of-two g) and in both MXFP8 forms."""
    x = rng.choice(_E2M1, size=shape) * rng.choice([-1.0, 1.0], size=shape) * c
    x.reshape(-1, 16)[:, 0] = -6.0 * c
    return x


@pytest.mark.parametrize("g", [1.0, 0.5])
def test_mixed_exact_limit_on_grid_inputs(orc, g):
    """With every operand exact in NVFP4 and MXFP8 and P/dS quantisation off,
    the mixed emulation equals the exact oracle.  Fails: a stray term, a g
    applied twice or not at all, a transposed operand."""
    rng = np.random.default_rng(4)
    cu = _cu([45, 1, 70, 33])
    T, Hq, Hkv, d, sc = int(cu[-1]), 4, 2, 64, 0.125
    q, k = _nv_grid(rng, 0.25, T, Hq, d), _nv_grid(rng, 0.5, T, Hkv, d)
    v, do = _nv_grid(rng, 0.25, T, Hkv, d), _nv_grid(rng, 0.125, T, Hq, d)
    ex = orc.attn_bwd(q, k, v, do, cu, sc)
    nv = orc.nvmx_attn_bwd(q, k, v, do, cu, sc, flags=0, gq=g, gk=g)
    for key in ex:
        np.testing.assert_allclose(nv[key], ex[key], rtol=0, atol=1e-11, err_msg=key)


def test_mixed_scores_by_hand(orc):
    """One document, d = 32, Q of token 0 = (2.5, 6, 0 ...), K of token 0 =
    (1, 0 ...) with gq = 3, gk = 1.  By hand (test_nv_block_by_hand):
    Q -> (2.0625, 6.1875), K -> (1.03125, 0), so S_00 = scale * 2.0625 *
    1.03125 and LSE_0 = S_00 (one visible key).  The MXFP8 path keeps both
    exact (S_00 = 2.5 scale).  A second token whose K holds 100 leaves LSE_0
    unchanged: the NVFP4 blocks lie inside one token (no pooling across
    tokens, so no leak guard is needed).  Fails: S from the MXFP8 forms, NVFP4
    on one operand only, g dropped, blocks across tokens."""
    T, d, sc = 2, 32, 0.5
    q = np.zeros((T, 1, d))
    k = np.zeros((T, 1, d))
    v = np.ones((T, 1, d))
    q[0, 0, :2] = [2.5, 6.0]
    k[0, 0, 0] = 1.0
    _, lse = orc.nvmx_attn_fwd(q[:1], k[:1], v[:1], _cu([1]), sc, gq=3.0, gk=1.0)
    assert lse[0, 0] == pytest.approx(sc * 2.0625 * 1.03125, abs=1e-15)
    _, lse_mx = orc.mx_attn_fwd(q[:1], k[:1], v[:1], _cu([1]), sc)
    assert lse_mx[0, 0] == pytest.approx(sc * 2.5, abs=1e-15)
    k[1, 0, 0] = 100.0
    _, lse2 = orc.nvmx_attn_fwd(q, k, v, _cu([2]), sc, gq=3.0, gk=1.0)
    assert lse2[0, 0] == lse[0, 0]


def test_mixed_backward_is_the_straight_through_gradient(orc):
    """P/dS quantisation off, inputs on a k/4 grid that both MXFP8 forms keep
    exactly but NVFP4 does not.  The reading: the scores take their VALUE from
    the NVFP4 Q and K, while the gradient products keep the MXFP8 path's
    operands (dQ = scale dS K~, dK = scale dS^T Q~tb, dV = P^T dO~tb; exact on
    this grid).  torch autograd computes that gradient in fp64 from
    S = scale (Q K^T) with the value of scale Q~nv K~nv^T substituted (the
    oracle's NVFP4 values).  It also checks the backward's recomputed O and
    LSE against the forward's (consistency).  Fails: dK from the NVFP4 Q, dQ
    from the NVFP4 K, backward scores that are not the forward's, a missing D
    term."""
    import torch

    rng = np.random.default_rng(5)
    L, Hq, Hkv, d, sc, gq, gk = 40, 2, 1, 32, 0.3, 0.75, 1.25
    grid = lambda *s: rng.integers(-16, 17, size=s) / 4.0  # noqa: E731
    q, k, v, do = grid(L, Hq, d), grid(L, Hkv, d), grid(L, Hkv, d), grid(L, Hq, d)
    cu = _cu([L])
    mx0 = orc.mx_attn_bwd(q, k, v, do, cu, sc, flags=0)
    ex = orc.attn_bwd(q, k, v, do, cu, sc)
    for key in ex:  # the grid is exact in both MXFP8 forms
        np.testing.assert_allclose(mx0[key], ex[key], atol=1e-11, err_msg=key)

    def deq(x, g):
        codes, scales = orc.quantize_nvfp4(x, g)
        vals = np.empty(x.shape)
        lo, hi = codes & 15, codes >> 4
        vals[..., 0::2] = np.vectorize(orc.e2m1_decode)(lo)
        vals[..., 1::2] = np.vectorize(orc.e2m1_decode)(hi)
        sv = np.vectorize(orc.e4m3_decode)(scales)
        return vals * np.repeat(sv, 16, axis=-1) * g

    qn, kn = deq(q, gq), deq(k, gk)
    assert np.abs(qn - q).max() > 0.1 and np.abs(kn - k).max() > 0.1  # NVFP4 rounding acts
    t = lambda a: torch.tensor(a, dtype=torch.float64, requires_grad=True)  # noqa: E731
    Q, K, V = t(q), t(k), t(v)
    Qn, Kn = torch.tensor(qn), torch.tensor(kn)
    mask = torch.ones(L, L, dtype=torch.bool).tril()
    o = torch.empty(L, Hq, d, dtype=torch.float64)
    outs = []
    for h in range(Hq):
        ex_s = sc * Q[:, h] @ K[:, 0].T  # the gradient's operands
        s = ex_s + (sc * Qn[:, h] @ Kn[:, 0].T - ex_s).detach()  # the value's
        s = s.masked_fill(~mask, float("-inf"))
        outs.append(torch.softmax(s, -1) @ V[:, 0])
    o = torch.stack(outs, 1)
    (o * torch.tensor(do)).sum().backward()
    nv = orc.nvmx_attn_bwd(q, k, v, do, cu, sc, flags=0, gq=gq, gk=gk)
    np.testing.assert_allclose(nv["o"], o.detach().numpy(), atol=1e-11)
    np.testing.assert_allclose(nv["dq"], Q.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(nv["dk"], K.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(nv["dv"], V.grad.numpy(), atol=1e-10)
    o_f, lse_f = orc.nvmx_attn_fwd(q, k, v, cu, sc, flags=0, gq=gq, gk=gk)
    np.testing.assert_array_equal(nv["o"], o_f)
    np.testing.assert_array_equal(nv["lse"], lse_f)
    # with P~ quantised the backward's O, LSE still equal the forward's
    nvq = orc.nvmx_attn_bwd(q, k, v, do, cu, sc, gq=gq, gk=gk)
    o_q, lse_q = orc.nvmx_attn_fwd(q, k, v, cu, sc, gq=gq, gk=gk)
    np.testing.assert_array_equal(nvq["o"], o_q)
    np.testing.assert_array_equal(nvq["lse"], lse_q)
