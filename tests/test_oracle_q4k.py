"""Pins of the oracle's nested-superblock quantizer (page 2 "量化", the Q4_K
superblock figure: 256 weights = 8 subblocks of 32, 6-bit subblock scale and
minimum quantized against a binary16 super-scale and super-minimum, 4-bit
codes, 4.5 bits per weight).  The page fixes the nesting and the bit counts;
the arithmetic is the reading stated in oracle/oracle.c.  Each pin checks a
step against something other than its own formula: the bit budget, a block
worked out by hand, an independent parse of the 6-bit bitstream, the
round-up characterisation of the super-scales, brute-force nearest choices
(sub-scales, minima, codes) in exact rational arithmetic, and one-hot
products."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

BLOCK = 144


def parse(block):
    """(d, dmin, sc[8], mq[8], codes[256]) from one block's bytes, decoded
    here from the layout alone: little-endian binary16 d and dmin, sixteen
    6-bit fields least-significant-bit first, two codes per byte (low nibble
    first)."""
    block = bytes(block)
    d = float(np.frombuffer(block[0:2], dtype="<f2")[0])
    dmin = float(np.frombuffer(block[2:4], dtype="<f2")[0])
    bits = int.from_bytes(block[4:16], "little")
    fields = [(bits >> (6 * f)) & 63 for f in range(16)]
    codes = [(block[16 + k // 2] >> (4 * (k & 1))) & 15 for k in range(256)]
    return d, dmin, fields[:8], fields[8:], codes


def half_values(W):
    return [Fraction(float(v)) for v in W.float().numpy().ravel()]


def make_case(orc):
    W = synth.weight(6, 1024, seed=11)
    return W, orc.q4k_quantize(synth.half_bits(W))


@pytest.fixture(scope="module")
def case():
    return make_case(oracle.get())


def test_bit_budget(case):
    """144 bytes per 256 weights: 4.5 bits per weight (2 + 2 + 12 + 128)."""
    W, blocks = case
    assert blocks.shape == (6, 1024 // 256 * BLOCK)
    assert BLOCK * 8 / 256 == 4.5 and 2 + 2 + 16 * 6 // 8 + 256 // 2 == BLOCK


def check_block_worked_by_hand(orc):
    """Every subblock holds w_i = -1 + 0.25 (i mod 16).  Then s = 3.75/15 =
    0.25 and m = 1.  d = smallest binary16 >= 0.25/63 = 2^-8 * 1.01587...:
    mantissa 16.25/1024 rounds up to 17, pattern 0x1C11.  dmin = smallest
    binary16 >= 1/63 = 2^-6 * 1.01587...: pattern 0x2411.  Both sub-fields
    round(0.25/d) and round(1/dmin) are round(62.95) = 63, so the 96 field
    bits are all ones.  With S = 63 d and M = 63 dmin, (w + M)/S lies within
    0.011 of i mod 16, so the codes are i mod 16."""
    row = np.array([-1.0 + 0.25 * (i % 16) for i in range(256)], dtype=np.float16)
    blocks = orc.q4k_quantize(row.view(np.uint16).reshape(1, 256))
    expect = [0x11, 0x1C, 0x11, 0x24] + [0xFF] * 12 + [0x10, 0x32, 0x54, 0x76, 0x98, 0xBA,
                                                      0xDC, 0xFE] * 16
    assert blocks[0].tolist() == expect


def check_super_scales_round_up(case):
    """d (dmin) is the smallest binary16 at or above max_j s_j / 63
    (max_j m_j / 63), with s_j = (hi - lo)/15 and m_j = -lo over the
    subblock's range widened to contain 0."""
    W, blocks = case
    w = half_values(W)
    K = 1024
    for n in range(W.shape[0]):
        for b in range(K // 256):
            d, dmin, _, _, _ = parse(blocks[n, b * BLOCK:(b + 1) * BLOCK])
            s, m = [], []
            for j in range(8):
                sub = w[n * K + b * 256 + 32 * j: n * K + b * 256 + 32 * j + 32]
                lo, hi = min([Fraction(0)] + sub), max([Fraction(0)] + sub)
                s.append((hi - lo) / 15)
                m.append(-lo)
            for val, target in ((d, max(s) / 63), (dmin, max(m) / 63)):
                assert Fraction(val) >= target
                below = np.nextafter(np.float16(val), np.float16(0))
                assert Fraction(float(below)) < target


def check_subblock_fields_nearest(case):
    """sc_j is a nearest multiple choice: |s_j - d sc| is minimal over
    sc = 1..63; mq_j likewise for |m_j - dmin mq| over 0..63."""
    W, blocks = case
    w = half_values(W)
    K = 1024
    for n in range(W.shape[0]):
        for b in range(K // 256):
            d, dmin, sc, mq, _ = parse(blocks[n, b * BLOCK:(b + 1) * BLOCK])
            fd, fdm = Fraction(d), Fraction(dmin)
            for j in range(8):
                sub = w[n * K + b * 256 + 32 * j: n * K + b * 256 + 32 * j + 32]
                lo, hi = min([Fraction(0)] + sub), max([Fraction(0)] + sub)
                sj, mj = (hi - lo) / 15, -lo
                assert 1 <= sc[j] <= 63 and 0 <= mq[j] <= 63
                best = min(abs(sj - fd * c) for c in range(1, 64))
                assert abs(sj - fd * sc[j]) == best
                best = min(abs(mj - fdm * c) for c in range(0, 64))
                assert abs(mj - fdm * mq[j]) == best


def check_codes_nearest_given_metadata(case):
    """Every code is a nearest grid point: |w - (S q - M)| is minimal over
    q = 0..15, with S = d sc_j and M = dmin mq_j as stored."""
    W, blocks = case
    w = half_values(W)
    K = 1024
    for n in range(W.shape[0]):
        for b in range(K // 256):
            d, dmin, sc, mq, codes = parse(blocks[n, b * BLOCK:(b + 1) * BLOCK])
            for k in range(256):
                j = k // 32
                S, M = Fraction(d) * sc[j], Fraction(dmin) * mq[j]
                x = w[n * K + b * 256 + k]
                errs = [abs(x - (S * q - M)) for q in range(16)]
                assert errs[codes[k]] == min(errs)


def check_dequantize_from_fields(orc, case):
    """The oracle's dequantization equals S_j q - M_j from the parsed bytes."""
    W, blocks = case
    out = orc.q4k_dequantize(blocks, 6, 1024)
    for n in (0, 5):
        for b in range(4):
            d, dmin, sc, mq, codes = parse(blocks[n, b * BLOCK:(b + 1) * BLOCK])
            ref = [d * sc[k // 32] * codes[k] - dmin * mq[k // 32] for k in range(256)]
            assert np.array_equal(out[n, b * 256:(b + 1) * 256], np.array(ref))


def check_degenerate_blocks(o):
    """An all-zero block stores d = dmin = 0, sub-scales 1, minima 0, codes 0
    and reconstructs exact zeros; a non-negative block has dmin = 0 and
    minima 0."""
    zero = np.zeros((1, 256), dtype=np.uint16)
    blk = o.q4k_quantize(zero)
    d, dmin, sc, mq, codes = parse(blk[0])
    assert (d, dmin) == (0.0, 0.0) and sc == [1] * 8 and mq == [0] * 8 and codes == [0] * 256
    assert np.array_equal(o.q4k_dequantize(blk, 1, 256), np.zeros((1, 256)))
    pos = np.abs(synth.weight(1, 256, seed=4).float().numpy()).astype(np.float16)
    d, dmin, sc, mq, codes = parse(o.q4k_quantize(pos.view(np.uint16))[0])
    assert dmin == 0.0 and mq == [0] * 8 and d > 0.0


def check_matmul_one_hot(o, case):
    """X = e_k gives Y[:, n] = w^[n, k] exactly."""
    W, blocks = case
    Wh = o.q4k_dequantize(blocks, 6, 1024)
    for k in (0, 255, 256, 777, 1023):
        x = np.zeros((1, 1024), dtype=np.float32)
        x[0, k] = 1.0
        xb = (x.view(np.uint32) >> 16).astype(np.uint16)
        y, yabs = o.q4k_matmul(xb, blocks, 6, 1024)
        assert np.array_equal(y[0], Wh[:, k])
        assert np.array_equal(yabs[0], np.abs(Wh[:, k]))


def checks(orc):
    """Every pin as (name, thunk) for one oracle build, cheapest first."""
    c = make_case(orc)
    return [
        ("hand-worked block", lambda: check_block_worked_by_hand(orc)),
        ("degenerate blocks", lambda: check_degenerate_blocks(orc)),
        ("super-scales round up", lambda: check_super_scales_round_up(c)),
        ("sub-block fields nearest", lambda: check_subblock_fields_nearest(c)),
        ("codes nearest", lambda: check_codes_nearest_given_metadata(c)),
        ("dequantize from fields", lambda: check_dequantize_from_fields(orc, c)),
        ("matmul one-hot", lambda: check_matmul_one_hot(orc, c)),
    ]


@pytest.mark.parametrize("index", range(7))
def test_pin(index):
    name, fn = checks(oracle.get())[index]
    fn()


# Plausible mistakes planted in copies of the C oracle (compiled into a
# temporary directory); some pin above must catch each one.
MUTANTS = [
    ("super-scale rounded down",
     "uint16_t d16 = smax > 0.0 ? half_round_up_positive(smax / 63.0) : 0;",
     "uint16_t d16 = smax > 0.0 ? (uint16_t)(half_round_up_positive(smax / 63.0) - 1) : 0;"),
    ("sub-scale truncated", "(int)clampd(nearbyint(s[j] / d), 1.0, 63.0)",
     "(int)clampd(floor(s[j] / d), 1.0, 63.0)"),
    ("minimum from the top of the range", "                m[j] = -lo;",
     "                m[j] = hi;"),
    ("codes truncated", "nearbyint((v + M) / S)", "floor((v + M) / S)"),
    ("6-bit fields most significant bit first",
     "                        int pos = 6 * f + bit;\n                        blk[4 + pos / 8] |=",
     "                        int pos = 6 * f + (5 - bit);\n                        blk[4 + pos / 8] |="),
    ("nibbles swapped", "(k & 1) ? (q << 4) : q", "(k & 1) ? q : (q << 4)"),
    ("dequantize drops the minimum", "d * field[j] * q - dmin * field[8 + j]",
     "d * field[j] * q"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, old, new):
    src = open(oracle.SOURCE).read()
    assert src.count(old) == 1, f"snippet for '{name}' not found exactly once"
    path = tmp_path / "oracle_planted.c"
    path.write_text(src.replace(old, new))
    orc = oracle.Oracle(oracle.build(str(path), str(tmp_path / "liboracle_planted.so"),
                                     force=True))
    caught = []
    for check_name, fn in checks(orc):
        try:
            fn()
        except AssertionError:
            caught.append(check_name)
            break
    assert caught, f"no pin caught the planted mistake '{name}'"
