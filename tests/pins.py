"""Checks that pin the CPU oracle to facts fixed outside itself.

Each ``check_*`` takes an ``oracle.Oracle`` handle and raises AssertionError
on a mismatch, so the same checks run against the real oracle
(``test_oracle_pins.py``) and against copies with a planted mistake
(``test_oracle_mutations.py``), which must fail at least one of them.

What pins what:

* page values -- page 1 section 2 payload bytes (544 B, 2304 B); page 2's
  effective bits (4.5 bpw at group 32, 3.56x, 11.1 % overhead, +2 bpw at
  group 8); page 3's printed step 0.26 and bound 0.13; the meta counts the
  page 1 example asserts (1 per tensor, 2 with groups of 4);
* hand-derived worked values -- the page 1 and page 3 examples worked by hand
  from the section 1 equations (derivations in the comments);
* closed forms and invariants -- |w - w^| <= s/2 on every element (page 3
  "直接答案"), real 0 reconstructed exactly (page 3 "深入原理"), lossless
  round trips on exact grids, ties resolved to even;
* brute force -- every code is the nearest grid point among all 2^b codes;
* decoders -- binary16 and bfloat16 decoding against numpy/torch, the
  binary16 round-up against the sorted binary16 grid;
* matmul -- one-hot and zero activations, exact rational sums, page 2's
  K-major per-group accumulation.
"""
from __future__ import annotations

import bisect
from fractions import Fraction

import numpy as np
import torch

from oracle import paper

# Positive finite binary16 values in increasing order (numpy's decoder).
_HALF_GRID = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)


def half_round_up_exact(x: Fraction) -> float:
    """Smallest binary16 value >= x (x > 0), by bisection on the grid."""
    i = bisect.bisect_left(_HALF_GRID, float(x))
    while i > 0 and Fraction(_HALF_GRID[i - 1]) >= x:
        i -= 1
    while Fraction(_HALF_GRID[i]) < x:
        i += 1
    return float(_HALF_GRID[i])


def to_half_bits(values) -> np.ndarray:
    return np.asarray(values, dtype=np.float16).view(np.uint16)


def half_values(bits_arr) -> np.ndarray:
    return np.asarray(bits_arr, dtype=np.uint16).view(np.float16).astype(np.float64)


def random_half_weights(N: int, K: int, seed: int, std: float = 0.02,
                        outlier_every: int = 0) -> np.ndarray:
    g = torch.Generator().manual_seed(seed)
    W = torch.randn(N, K, generator=g) * std
    if outlier_every:
        W[:, ::outlier_every] *= 20.0
    return W.to(torch.float16).view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------- decoders

def check_half_decoder(orc):
    pats = np.arange(0, 0x10000, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float64)
    got = np.array([orc.half_to_double(int(p)) for p in pats])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(np.isinf(got), np.isinf(ref))


def check_bf16_decoder(orc):
    pats = np.concatenate([np.arange(0, 0x10000, 97, dtype=np.uint32),
                           [0x3F80, 0xBF80, 0x0001, 0x7F7F, 0x8000]]).astype(np.uint16)
    ref = torch.from_numpy(pats.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    got = np.array([orc.bf16_to_double(int(p)) for p in pats])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])


def check_half_round_up(orc):
    rng = np.random.default_rng(5)
    xs = list(np.exp(rng.uniform(np.log(1e-9), np.log(6e4), 3000)))
    xs += list(_HALF_GRID[::97])                      # exact grid points map to themselves
    xs += [float(v) * (1 + 1e-12) for v in _HALF_GRID[:-1:113]]   # just above -> next
    for x in xs:
        want = half_round_up_exact(Fraction(x))
        got = orc.half_to_double(orc.half_round_up(float(x)))
        assert got == want, (x, got, want)


# ------------------------------------------------------- worked examples

def check_p1_example_paper_mode(paper=paper):
    """Page 1 section 1 example in the page's own float semantics.

    Per tensor (group = 8): lo = -8, hi = 7.3, s = 15.3/15 = 1.02,
    z = round(8/1.02 = 7.84) = 8; round(v/1.02) = [-8, 0, 0, 0, 7, 7, 7, 7]
    -> codes [0, 8, 8, 8, 15, 15, 15, 15], x^ = [-8.16, 0, 0, 0, 7.14 x4],
    MAE = 1.16/8 = 0.145.
    Groups of 4: [-8, -0.2, 0.1, 0.3] -> s = 8.3/15, z = round(14.46) = 14,
    codes [0, 14, 14, 15]; [7.0, 7.1, 7.2, 7.3] -> lo widened to 0,
    s = 7.3/15, z = 0, v/s = [14.38, 14.59, 14.79, 15] -> [14, 15, 15, 15];
    MAE = 1.29333/8 = 0.161667 (worse than per tensor, as the page warns).
    """
    x = [-8.0, -0.2, 0.1, 0.3, 7.0, 7.1, 7.2, 7.3]
    q_t, hat_t, meta_t = paper.affine_quantize(x, bits=4)
    q_g, hat_g, meta_g = paper.affine_quantize(x, bits=4, group_size=4)
    assert len(meta_t) == 1 and len(meta_g) == 2            # the page's assert
    assert q_t == [0, 8, 8, 8, 15, 15, 15, 15]
    assert abs(meta_t[0][0] - 1.02) < 1e-12 and meta_t[0][1] == 8
    assert q_g == [0, 14, 14, 15, 14, 15, 15, 15]
    assert [z for _, z in meta_g] == [14, 0]
    mae = lambda a, b: sum(abs(u - v) for u, v in zip(a, b)) / len(a)
    assert abs(mae(x, hat_t) - 0.145) < 1e-12
    assert abs(mae(x, hat_g) - 0.16166666666666667) < 1e-12


def check_p1_example_storage_mode(orc):
    """The same example through the storage-mode oracle (binary16 in,
    binary16 scale rounded up).

    binary16 inputs: -0.2 -> -0.199951171875, 0.1 -> 0.0999755859375,
    0.3 -> 0.300048828125, 7.1 -> 7.1015625, 7.2 -> 7.19921875,
    7.3 -> 7.30078125.
    group 8: (7.30078125 + 8)/15 = 1.020052...; binary16 spacing in [1, 2) is
      2^-10, 1044.53 ulps -> round up to 1045 * 2^-10 = 1.0205078125; z = 8.
    group 4, first: (0.300048828125 + 8)/15 = 0.553336...; spacing 2^-11,
      1133.23 -> 1134 * 2^-11 = 0.5537109375 (nearest would give
      0.55322265625); z = round(8/0.5537 = 14.448) = 14.
    group 4, second: 7.30078125/15 = 0.48671875; spacing 2^-12, 1993.6 ->
      1994 * 2^-12 = 0.48681640625; z = 0.
    Codes equal the paper-mode ones.
    """
    W = to_half_bits([[-8.0, -0.2, 0.1, 0.3, 7.0, 7.1, 7.2, 7.3]])
    q, codes, s, z = orc.quantize(W, 4, 8, False)
    assert half_values(s).ravel().tolist() == [1.0205078125]
    assert half_values(z).ravel().tolist() == [8.0]
    assert q.tolist() == [[0, 8, 8, 8, 15, 15, 15, 15]]
    q, codes, s, z = orc.quantize(W, 4, 4, False)
    assert half_values(s).ravel().tolist() == [0.5537109375, 0.48681640625]
    assert half_values(z).ravel().tolist() == [14.0, 0.0]
    assert q.tolist() == [[0, 14, 14, 15, 14, 15, 15, 15]]
    # packing: byte j = code(2j) | code(2j+1) << 4
    assert codes.tolist() == [[0 | 14 << 4, 14 | 15 << 4, 14 | 15 << 4, 15 | 15 << 4]]


def check_p3_example_paper_mode(golden, paper=paper):
    """Page 3 "代码": INT4 on [-0.9, -0.2, 0.1, 0.5, 3.0] prints step 0.26 and
    bound 0.13.  By hand: s = 3.9/15 = 0.26, z = round(0.9/0.26 = 3.46) = 3,
    round(v/s) = [-3, -1, 0, 2, 12] -> codes [0, 2, 3, 5, 15],
    x^ = [-0.78, -0.26, 0, 0.52, 3.12], max error 0.12 <= 0.13.  Page 1's
    quantizer (range widened to contain 0: the example already straddles 0)
    gives the same codes and zero."""
    xs = [-0.9, -0.2, 0.1, 0.5, 3.0]
    recon, step = paper.quantize_dequantize_p3(xs, 4)
    assert f"{step:.2f}" == golden["printed_step"]
    assert f"{step / 2:.2f}" == golden["printed_bound"]
    assert max(abs(a - b) for a, b in zip(xs, recon)) <= step / 2
    want = [-0.78, -0.26, 0.0, 0.52, 3.12]
    assert all(abs(a - b) < 1e-12 for a, b in zip(recon, want)), recon
    codes_p1, recon_p1, meta = paper.affine_quantize(xs, bits=4)
    assert codes_p1 == [0, 2, 3, 5, 15] and meta[0][1] == 3
    assert all(abs(a - b) < 1e-12 for a, b in zip(recon_p1, want)), recon_p1
    # the clamp of the page's code at work: on [-3.5, 11.5] the scale is 1,
    # z = round(3.5) = 4 and round(11.5) + 4 = 16 -> clamped to 15, x^ = 11
    recon, step = paper.quantize_dequantize_p3([-3.5, 11.5], 4)
    assert step == 1.0 and recon == [-4.0, 11.0]


def check_p3_example(orc, golden):
    """Page 3 "代码" example through the storage-mode oracle: lo =
    -0.89990234375 (binary16 of -0.9), (3 + 0.8999)/15 = 0.2599935; spacing
    2^-12 -> 1064.93 ulps -> 1065 * 2^-12 = 0.260009765625; codes
    [0, 2, 3, 5, 15] as worked by hand in check_p3_example_paper_mode."""
    xs = [-0.9, -0.2, 0.1, 0.5, 3.0]
    W = to_half_bits([xs + [0.0]])                # pad to an even length for packing
    q, _, s, z = orc.quantize(W[:, :5].copy(), 4, 5, False, pack=False)
    assert half_values(s).ravel().tolist() == [0.260009765625]
    assert half_values(z).ravel().tolist() == [3.0]
    assert q.tolist() == [[0, 2, 3, 5, 15]]
    what = 0.260009765625 * (np.array([0, 2, 3, 5, 15]) - 3)
    assert np.max(np.abs(half_values(W[0, :5]) - what)) <= 0.13
    assert f"{0.260009765625:.2f}" == golden["printed_step"]


def check_paper_degenerate_and_zero(paper=paper):
    """Page 1 section 1's example code: a degenerate range gets scale 1.0 and
    zero 0, so an all-zero group comes back as zeros; the widened range keeps
    real 0 exact in every group (page 3 "深入原理")."""
    codes, recon, meta = paper.affine_quantize([0.0] * 4 + [0.5, 1.0, 0.0, 2.0], bits=4,
                                               group_size=4)
    assert meta[0] == (1.0, 0) and codes[:4] == [0, 0, 0, 0] and recon[:4] == [0.0] * 4
    assert meta[1][1] == 0 and abs(meta[1][0] - 2.0 / 15) < 1e-15   # lo widened to 0
    assert recon[6] == 0.0
    codes, recon, _ = paper.affine_quantize([-3.0, 0.0, 1.0, 0.0, 5.0, -0.25], bits=3,
                                            group_size=3)
    assert recon[1] == 0.0 and recon[3] == 0.0


def check_paper_ties_to_even(paper=paper):
    """A 4-bit group on [0, 15/64] has s = 2^-6 and z = 0 exactly in binary64;
    the weights (j + 1/2)/64 sit exactly between codes j and j + 1 and go to
    the even one (Python's round, which the pages' code calls)."""
    vals = [0.0, 15 / 64] + [(j + 0.5) / 64 for j in range(14)]
    codes, _, meta = paper.affine_quantize(vals, bits=4)
    assert meta == [(1 / 64, 0)]
    assert codes == [0, 15] + [j if j % 2 == 0 else j + 1 for j in range(14)]
    neg = [-v for v in vals]                     # z = 15 on the mirrored group
    codes, _, meta = paper.affine_quantize(neg, bits=4)
    assert meta == [(1 / 64, 15)]
    assert codes == [15, 0] + [15 - (j if j % 2 == 0 else j + 1) for j in range(14)]


def check_paper_nearest_and_bound(paper=paper, seed=11):
    """Page 1 section 1's quantizer in binary64 on random groups with an
    outlier: every code is the nearest of the 2^b grid points s (c - z)
    (brute force), and |x - x^| <= s/2 (page 3 "直接答案") up to binary64
    rounding of x/s."""
    rng = np.random.default_rng(seed)
    for bits in (2, 3, 4, 8):
        x = rng.normal(0.0, 0.02, 96)
        x[17] *= 40.0
        codes, recon, meta = paper.affine_quantize(x, bits=bits, group_size=32)
        for i, v in enumerate(x):
            s, z = meta[i // 32]
            grid = [s * (c - z) for c in range(1 << bits)]
            best = min(abs(v - gv) for gv in grid)
            assert abs(v - s * (codes[i] - z)) <= best + 1e-15, (bits, i)
            assert abs(v - recon[i]) <= s / 2 * (1 + 1e-12), (bits, i)


def check_payload(orc, golden):
    """Page 1 section 2: 1024 INT4 @ group 128 with 2-byte scale + 2-byte zero
    = 544 B; 4096 INT4 @ group 64 = 2304 B."""
    for case in golden["payload"]:
        n, g = case["params"], case["group"]
        W = random_half_weights(1, n, seed=n)
        _, codes, s, z = orc.quantize(W, 4, g, False)
        total = codes.nbytes + s.nbytes + z.nbytes
        assert total == case["bytes"], (case, total)


def check_effective_bits(orc, golden):
    """Page 2: group 32 with one binary16 scale -> 4.5 bits/weight, 16/4.5 =
    3.56x compression, 0.5/4.5 = 11.1 % metadata; group 8 adds 2 bits."""
    K = 4096
    W = random_half_weights(1, K, seed=3)
    for case in golden["effective_bits"]:
        _, codes, s, _ = orc.quantize(W, 4, case["group"], True)      # scale only
        bpw = 8.0 * (codes.nbytes + s.nbytes) / K
        assert abs(bpw - case["bits_per_weight"]) < 1e-12
        if "compression" in case:
            assert f"{16 / bpw:.2f}" == case["compression"]
            assert f"{100 * (bpw - 4) / bpw:.1f}" == case["overhead_percent"]


# ------------------------------------------------- invariants, brute force

def _groups(values, group):
    N, K = values.shape
    return values.reshape(N, K // group, group)


def check_error_bound(orc, bits, group, symmetric, W):
    """|w - w^| <= s/2 for every element, with the stored s (page 3)."""
    N, K = W.shape
    q, codes, s, z = orc.quantize(W, bits, group, symmetric)
    what = orc.dequantize(codes, s, z, N, K, bits, group, symmetric)
    w = half_values(W)
    sv = np.repeat(half_values(s), group, axis=1)
    err = np.abs(w - what)                      # exact in binary64
    bad = err > sv / 2
    assert not bad.any(), f"{int(bad.sum())} elements exceed s/2, worst {np.max(err / sv)}"


def check_exact_zero(orc, bits, group, symmetric, W):
    """A weight equal to 0 is reconstructed as exactly 0 (page 3, page 1's
    widened range)."""
    N, K = W.shape
    W = W.copy()
    W[:, ::7] = 0
    W[1::5, 3::11] = 0x8000                     # -0.0
    _, codes, s, z = orc.quantize(W, bits, group, symmetric)
    what = orc.dequantize(codes, s, z, N, K, bits, group, symmetric)
    zero = half_values(W) == 0
    assert np.all(what[zero] == 0.0)


def check_nearest_code_bruteforce(orc, bits, group, symmetric, W):
    """Every code is the grid point nearest to its weight, among all 2^b
    codes; ties go to the even value of (q - z) (round-half-even of w/s,
    then the zero point is added -- page 1's order)."""
    N, K = W.shape
    q, codes, s, z = orc.quantize(W, bits, group, symmetric)
    w = half_values(W)
    sv = half_values(s)
    zv = np.zeros_like(sv) if symmetric else half_values(z)
    if symmetric:
        cand = np.arange(-(1 << (bits - 1)), 1 << (bits - 1))
    else:
        cand = np.arange(0, 1 << bits)
    for n in range(N):
        for k in range(K):
            g = k // group
            sf, zf = Fraction(sv[n, g]), Fraction(zv[n, g])
            wf = Fraction(w[n, k])
            dist = [abs(wf - sf * (c - zf)) for c in cand]
            best = min(dist)
            winners = [int(c) for c, d in zip(cand, dist) if d == best]
            if len(winners) == 1:
                want = winners[0]
            else:
                want = [c for c in winners if (c - int(zf)) % 2 == 0][0]
            assert q[n, k] == want, (n, k, q[n, k], winners)


def check_ties_to_even(orc):
    """Asymmetric 4-bit group on [0, 15/64]: s = 15/64/15 = 2^-6 exactly,
    z = 0; weights (j + 1/2)/64 sit exactly between codes j and j + 1 and must
    go to the even one."""
    vals = [0.0, 15 / 64] + [(j + 0.5) / 64 for j in range(14)]
    W = to_half_bits([vals])
    q, _, s, z = orc.quantize(W, 4, 16, False)
    assert half_values(s).ravel().tolist() == [1 / 64] and half_values(z).ravel().tolist() == [0.0]
    want = [0, 15] + [j if j % 2 == 0 else j + 1 for j in range(14)]
    assert q.tolist() == [want]


def check_lossless_grids(orc):
    """Weights already on a grid come back exactly (a textbook special case):
    symmetric 8-bit w = c/128 for every c in [-127, 127] gives s = 2^-7 and
    codes c; symmetric 4-bit w = c/8 for c in [-7, 7] gives s = 1/8; an
    asymmetric 4-bit group on s*(c - 5) for c in 0..15 gives s and z = 5."""
    c8 = np.arange(-127, 129)                       # 256 values, group 256
    c8[-1] = 0
    q, codes, s, _ = orc.quantize(to_half_bits([c8 / 128.0]), 8, 256, True)
    assert half_values(s).ravel().tolist() == [1 / 128] and q.tolist() == [c8.tolist()]
    assert codes.tolist() == [(c8 + 128).tolist()]   # offset-binary storage
    c4 = np.array(list(range(-7, 8)) + [0])
    q, codes, s, _ = orc.quantize(to_half_bits([c4 / 8.0]), 4, 16, True)
    assert half_values(s).ravel().tolist() == [0.125] and q.tolist() == [c4.tolist()]
    u = c4 + 8
    assert codes.tolist() == [(u[0::2] | (u[1::2] << 4)).tolist()]
    c = np.arange(16)
    q, _, s, z = orc.quantize(to_half_bits([0.375 * (c - 5)]), 4, 16, False)
    assert half_values(s).ravel().tolist() == [0.375] and half_values(z).ravel().tolist() == [5.0]
    assert q.tolist() == [c.tolist()]


def check_degenerate_groups(orc):
    """All-zero groups get scale 1.0 and zero 0 (page 1's degenerate-range
    rule); an all-positive group still has 0 on its grid."""
    W = np.zeros((2, 32), dtype=np.uint16)
    W[1] = to_half_bits(np.linspace(0.5, 2.0, 32))
    for sym in (False, True):
        q, codes, s, z = orc.quantize(W, 4, 32, sym)
        assert half_values(s)[0].tolist() == [1.0]
        assert np.all(q[0] == 0)
        what = orc.dequantize(codes, s, z, 2, 32, 4, 32, sym)
        assert np.all(what[0] == 0.0)
    _, _, s, z = orc.quantize(W, 4, 32, False)
    assert half_values(z)[1].tolist() == [0.0]     # lo widened to 0 -> z = 0
    assert half_values(s)[1].tolist() == [half_round_up_exact(Fraction(2.0) / 15)]


def check_packing_layout(orc, bits, W):
    """Codes are stored row-major; for 4 bits byte j of a row holds k = 2j in
    bits 0-3 and k = 2j + 1 in bits 4-7 (decoded here with numpy)."""
    q, codes, s, z = orc.quantize(W, bits, 32, False)
    if bits == 8:
        assert np.array_equal(codes.astype(np.int32), q)
    else:
        assert np.array_equal(codes & 0x0F, q[:, 0::2])
        assert np.array_equal(codes >> 4, q[:, 1::2])


def check_exact_metadata(orc, bits, group, symmetric, W):
    """Scales, zeros and codes recomputed in exact rational arithmetic (the
    binary16 round-up against the sorted binary16 grid).  This confirms that
    the oracle's binary64 arithmetic decides every rounding exactly."""
    N, K = W.shape
    q, _, s, z = orc.quantize(W, bits, group, symmetric)
    w = half_values(W)
    sv = half_values(s)
    zv = None if symmetric else half_values(z)
    for n in range(N):
        for g in range(K // group):
            vals = [Fraction(v) for v in w[n, g * group:(g + 1) * group]]
            if symmetric:
                qm = (1 << (bits - 1)) - 1
                a = max(abs(v) for v in vals)
                sf = Fraction(1) if a == 0 else Fraction(half_round_up_exact(a / qm))
                zf, lo_c, hi_c = 0, -qm - 1, qm
            else:
                qmax = (1 << bits) - 1
                lo, hi = min(min(vals), 0), max(max(vals), 0)
                if hi == lo:
                    sf, zf = Fraction(1), 0
                else:
                    sf = Fraction(half_round_up_exact((hi - lo) / qmax))
                    zf = min(qmax, max(0, round(-lo / sf)))
                lo_c, hi_c = 0, qmax
            assert Fraction(sv[n, g]) == sf, (n, g)
            if not symmetric:
                assert zv[n, g] == zf, (n, g)
            for i, v in enumerate(vals):
                want = min(hi_c, max(lo_c, round(v / sf) + zf))
                assert q[n, g * group + i] == want, (n, g, i)


# ------------------------------------------------------------------ matmul

def check_matmul_one_hot_and_zero(orc, bits, group, symmetric, W):
    """X = e_k gives Y[0, n] = w^[n, k] exactly (a second row -2 e_k' gives
    -2 w^[n, k']); X = 0 gives Y = 0."""
    N, K = W.shape
    _, codes, s, z = orc.quantize(W, bits, group, symmetric)
    what = orc.dequantize(codes, s, z, N, K, bits, group, symmetric)
    for k in (0, 1, K // 2 + 1, K - 1):
        X = np.zeros((2, K), dtype=np.uint16)
        X[0, k] = 0x3F80                          # bfloat16 1.0
        X[1, K - 1 - k] = 0xC000                  # bfloat16 -2.0
        Y, Yabs = orc.matmul(X, codes, s, z, N, K, bits, group, symmetric)
        assert np.array_equal(Y[0], what[:, k])
        assert np.array_equal(Yabs[0], np.abs(what[:, k]))
        assert np.array_equal(Y[1], -2.0 * what[:, K - 1 - k])
    X = np.zeros((2, K), dtype=np.uint16)
    Y, _ = orc.matmul(X, codes, s, z, N, K, bits, group, symmetric)
    assert np.all(Y == 0)


def check_matmul_exact_sum(orc, bits, group, symmetric, W, seed=7):
    """Small shapes: the sum recomputed with exact rationals."""
    N, K = W.shape
    M = 3
    Xt = torch.randn(M, K, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    X = Xt.view(torch.int16).numpy().view(np.uint16)
    _, codes, s, z = orc.quantize(W, bits, group, symmetric)
    what = orc.dequantize(codes, s, z, N, K, bits, group, symmetric)
    Y, Yabs = orc.matmul(X, codes, s, z, N, K, bits, group, symmetric)
    xv = Xt.double().numpy()
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(a) * Fraction(b) for a, b in zip(xv[m], what[n]))
            assert abs(Fraction(Y[m, n]) - exact) <= Fraction(Yabs[m, n]) * Fraction(1, 10**12)


def check_matmul_kmajor(orc, bits, group, symmetric, W, seed=8, paper=paper):
    """Page 2 "实现": accumulating x[:, group g] @ (q[g] * scale[g]) group by
    group over a [n_groups, group, out] layout gives the same Y (codes here
    already have the zero point subtracted)."""
    N, K = W.shape
    M = 4
    Xt = torch.randn(M, K, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    X = Xt.view(torch.int16).numpy().view(np.uint16)
    q, codes, s, z = orc.quantize(W, bits, group, symmetric)
    Y, Yabs = orc.matmul(X, codes, s, z, N, K, bits, group, symmetric)
    zv = 0.0 if symmetric else np.repeat(half_values(z), group, axis=1)
    qz = (q - zv).astype(np.float64)              # [N, K]
    q_kmajor = qz.T.reshape(K // group, group, N)
    s_kmajor = half_values(s).T.copy()             # [n_groups, N]
    ref = paper.fused_matmul_kmajor(Xt.double().numpy(), q_kmajor, s_kmajor, group)
    assert np.all(np.abs(ref - Y) <= 1e-12 * Yabs + 1e-300)


def check_dense_bf16(orc):
    """Dense reference on exact small integers: Y = X B^T computed by hand."""
    X = torch.tensor([[1, 2, -3, 0], [4, 0, 1, -1]], dtype=torch.bfloat16)
    B = torch.tensor([[1, 0, 0, 0], [0, 1, 1, 0], [2, -1, 0, 3]], dtype=torch.bfloat16)
    xb = X.view(torch.int16).numpy().view(np.uint16)
    bb = B.view(torch.int16).numpy().view(np.uint16)
    Y = orc.matmul_dense_bf16(xb, bb)
    assert Y.tolist() == [[1.0, -1.0, 0.0], [4.0, 1.0, 5.0]]
