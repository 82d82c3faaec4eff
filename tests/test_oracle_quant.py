"""Pins of the oracle's MXFP8 quantiser (CPU only).

Formats: E4M3 (bias 7, max finite 448, min normal 2^-6, subnormals down to
2^-9, no infinity) and E8M0 (2^(e-127)), from the OCP Microscaling v1.0
definition; block size 32 and the E4M3/E8M0 choice from the benchmark spec;
the FLAMIA page only names MXFP8 and microscaling.  The checks below compute
the expected codes by an independent route: the exponent from the bf16 bit
pattern and the rounding by nearest-even search on the enumerated E4M3 grid.
"""
import numpy as np
import pytest


def e4m3_grid():
    """All non-negative finite E4M3 values indexed by code 0x00..0x7E, built
    from the format's field definition."""
    vals = []
    for code in range(0x7F):
        e, m = code >> 3, code & 7
        vals.append(m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    return np.array(vals)


GRID = e4m3_grid()


def nearest_even_code(y: float) -> int:
    """Code of |y| rounded to the nearest grid value, ties to the even code,
    saturating at 448 (code 0x7E); sign bit set for negative non-zero."""
    a = abs(y)
    if a >= 448.0:
        c = 0x7E
    else:
        hi = int(np.searchsorted(GRID, a, side="left"))
        if GRID[hi] == a:
            c = hi
        else:
            lo = hi - 1
            dl, dh = a - GRID[lo], GRID[hi] - a
            c = lo if dl < dh else hi if dh < dl else (lo if lo % 2 == 0 else hi)
    if c == 0:
        return 0
    return c | (0x80 if y < 0 else 0)


def test_grid_facts():
    assert GRID[0x78] == 256.0 and GRID[0x7E] == 448.0
    assert GRID[0x08] == 2.0 ** -6 and GRID[0x01] == 2.0 ** -9
    assert np.all(np.diff(GRID) > 0)


@pytest.mark.parametrize("rule", [0, 1])
def test_worked_values(orc, rule):
    """Both rules: a = 1 -> X = -8, code(1.0) = 0x78 (1.0 * 2^8 = 256), scale
    byte 119; a = 448 = 1.75 * 2^8 -> X = 0; an all-zero block -> X = -127.
    OCP rule: a = 500 -> X = 0 and 500 saturates to 448.
    RCEIL rule: a = 500 -> X = 1 (500/2 = 250 <= 448) and 250 rounds to 256
    (quantum 16 in [128, 256)), so 500 -> 512."""
    codes, deq, sb = orc.quant_block(np.array([1.0]), rule)
    assert orc.block_exponent(1.0, rule) == -8 and codes[0] == 0x78 and sb == 119 and deq[0] == 1.0
    assert orc.block_exponent(448.0, rule) == 0
    codes, deq, sb = orc.quant_block(np.array([500.0, -3.0]), rule)
    if rule == 1:
        assert sb == 127 and codes[0] == 0x7E and deq[0] == 448.0
    else:
        assert sb == 128 and codes[0] == 0x78 and deq[0] == 512.0
    assert deq[1] == -3.0
    assert orc.block_exponent(0.0, rule) == -127
    codes, deq, sb = orc.quant_block(np.zeros(32), rule)
    assert sb == 0 and np.all(codes == 0) and np.all(deq == 0)


def test_tie_rounds_to_even(orc):
    """x = 1 + 2^-4 alone: scaled to 272, the midpoint of 256 and 288; ties
    to even give 256, which decodes to 1.0.  1 + 3*2^-4 -> 304, midpoint of
    288 and 320, goes up to 320 (even mantissa)."""
    codes, deq, _ = orc.quant_block(np.array([1.0 + 2.0 ** -4]))
    assert codes[0] == 0x78 and deq[0] == 1.0
    codes, deq, _ = orc.quant_block(np.array([1.0 + 3 * 2.0 ** -4]))
    assert codes[0] == 0x7A and deq[0] == 1.25


def test_e4m3_round_trip(orc):
    """Every finite E4M3 code decodes and re-encodes to itself (negative zero
    is canonicalised to 0x00); the NaN codes are never produced."""
    for c in range(256):
        if c & 0x7F == 0x7F:
            assert np.isnan(orc.e4m3_decode(c))
            continue
        v = orc.e4m3_decode(c)
        assert abs(v) == GRID[c & 0x7F]
        expect = 0 if c == 0x80 else c
        assert orc.e4m3_encode(v) == expect


def _bf16_values():
    bits = np.arange(65536, dtype=np.uint32)
    expo = (bits >> 7) & 0xFF
    bits = bits[expo != 0xFF]
    return bits, (bits << 16).view(np.float32).astype(np.float64)


def _floor_log2_from_bits(b: int) -> int:
    e = (b >> 7) & 0xFF
    if e != 0:
        return e - 127
    m = b & 0x7F
    return -134 + m.bit_length()  # subnormal: value m * 2^-133


def _mantissa_above_175(b: int) -> bool:
    """Is the significand of the bf16 value (in [1, 2)) above 1.75?"""
    e, m = (b >> 7) & 0xFF, b & 0x7F
    if e != 0:
        return m > 96                       # 1 + m/128 > 1.75
    n = m.bit_length()                      # subnormal m * 2^-133
    return 4 * m > 7 * (1 << (n - 1))       # m / 2^(n-1) > 1.75


@pytest.mark.slow
@pytest.mark.parametrize("rule", [0, 1])
def test_brute_force_all_bf16_single_element_blocks(orc, rule):
    """Every finite bf16 value as a one-element block: scale byte and code
    match the independent route (exponent from the bit pattern, nearest-even
    rounding on the E4M3 grid)."""
    bits, vals = _bf16_values()
    bad = 0
    for b, x in zip(bits.tolist(), vals.tolist()):
        codes, deq, sb = orc.quant_block(np.array([x]), rule)
        if x == 0.0:
            exp_sb, exp_code = 0, 0
        else:
            X = _floor_log2_from_bits(b) - 8
            if rule == 0 and _mantissa_above_175(b):
                X += 1
            X = min(127, max(-127, X))
            exp_sb = X + 127
            exp_code = nearest_even_code(x * 2.0 ** -X)
        if sb != exp_sb or codes[0] != exp_code:
            bad += 1
    assert bad == 0


@pytest.mark.parametrize("rule", [0, 1])
def test_random_blocks_error_bound(orc, rule):
    """Random 32-blocks: after scaling, the largest element lands in
    [256, 512) (OCP rule) or (224, 448] (RCEIL rule); codes match the grid
    route."""
    rng = np.random.default_rng(0)
    for trial in range(300):
        x = rng.standard_normal(32) * 10.0 ** rng.uniform(-6, 6)
        x = x.astype(np.float32).astype(np.float64)
        codes, deq, sb = orc.quant_block(x, rule)
        X = sb - 127
        y = x * 2.0 ** -X
        if rule == 1:
            assert 256.0 <= np.max(np.abs(y)) < 512.0
        else:
            assert 224.0 < np.max(np.abs(y)) <= 448.0
        for yi, ci in zip(y, codes):
            assert ci == nearest_even_code(yi)


def _cu(lengths):
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)


def test_quantize_layout_worked_example(orc):
    """Two documents of 40 and 3 tokens, H = 1, d = 32: token blocks are
    document-local ([0,32), [32,40), [40,43)) at slots 0, 1 and
    floor(40/32) + 1 = 2.  Block maxima 1.0, 3.0 and 0.5 give scale bytes
    119, 120 and 118; per-token scales follow each token's own maximum."""
    x = np.zeros((43, 1, 32))
    x[5, 0, 3] = 1.0
    x[7, 0, 9] = -0.75
    x[33, 0, 0] = 3.0
    x[39, 0, 31] = 0.125
    x[41, 0, 2] = -0.5
    out = orc.quantize_mxfp8(x, _cu([40, 3]), forms=3)
    stb = out["scale_tb"][:, 0, 0]
    assert stb.tolist() == [119, 120, 118]
    assert out["val_tb"][5, 0, 3] == 0x78          # 1.0 * 2^8 = 256
    assert out["val_tb"][7, 0, 9] == 0x80 | 0x74   # -0.75 * 2^8 = -192 = -(1.5 * 2^7): e=14, m=4
    assert out["val_tb"][39, 0, 31] == 0x58        # 0.125 * 2^7 = 16 = 2^4
    spt = out["scale_pt"][:, 0, 0]
    assert spt[5] == 119 and spt[7] == 126 - 8 and spt[39] == 124 - 8 + 0
    assert spt[0] == 0                              # all-zero token block
    assert out["val_pt"][39, 0, 31] == 0x78         # its own maximum -> 256


def test_quantize_tb_matches_blockwise(orc):
    """Token-block form: each (document block, head, channel group) tile
    equals quant_block of its gathered values; slots follow floor(s/32)+k+m;
    unused slots stay untouched."""
    rng = np.random.default_rng(1)
    lengths = [70, 1, 0, 33, 31, 64]
    cu = _cu(lengths)
    T, H, d = cu[-1], 3, 64
    x = rng.standard_normal((T, H, d)).astype(np.float32).astype(np.float64)
    x[10, 1, 5] = 300.0
    out = orc.quantize_mxfp8(x, cu, forms=3)
    used = set()
    for k, L in enumerate(lengths):
        s = cu[k]
        for m in range((L + 31) // 32):
            slot = s // 32 + k + m
            assert slot not in used
            used.add(slot)
            t0, t1 = s + 32 * m, min(s + 32 * m + 32, s + L)
            for h in range(H):
                for gi in range(d // 32):
                    blk = x[t0:t1, h, 32 * gi:32 * gi + 32].reshape(-1)
                    codes, _, sb = orc.quant_block(blk)
                    assert out["scale_tb"][slot, h, gi] == sb
                    assert np.array_equal(out["val_tb"][t0:t1, h, 32 * gi:32 * gi + 32].reshape(-1), codes)
    unused = [s for s in range(T // 32 + len(lengths)) if s not in used]
    assert np.all(out["scale_tb"][unused] == 0xFF)


@pytest.mark.parametrize("rule", [0, 1])
def test_power_of_two_invariance(orc, rule):
    """quant(2^k x) = 2^k quant(x) with identical codes (the scale byte moves
    by k), as long as the exponent is not clamped.  The forward's P~ relies on
    this: any integer base-2 row reference gives the same codes."""
    rng = np.random.default_rng(5)
    for _ in range(200):
        x = np.exp(rng.uniform(-12, 0, 32)) * (rng.random(32) < 0.8)
        x = x.astype(np.float32).astype(np.float64)
        if not x.any():
            continue
        c0, d0, s0 = orc.quant_block(x, rule)
        k = int(rng.integers(-20, 21))
        c1, d1, s1 = orc.quant_block(x * 2.0 ** k, rule)
        assert np.array_equal(c0, c1) and s1 == s0 + k
        np.testing.assert_array_equal(d1, d0 * 2.0 ** k)
