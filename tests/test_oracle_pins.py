"""The CPU oracle against what the pages and the mathematics fix (no GPU)."""
import json
import os

import numpy as np
import pytest

import oracle
from tests import pins

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages.json")))

FORMATS = [(b, g, s) for b in (4, 8) for g in (32, 64, 128) for s in (False, True)]


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


def test_half_decoder(orc):
    pins.check_half_decoder(orc)


def test_bf16_decoder(orc):
    pins.check_bf16_decoder(orc)


def test_half_round_up(orc):
    pins.check_half_round_up(orc)


def test_p1_example_paper_mode():
    pins.check_p1_example_paper_mode()


def test_p1_example_storage_mode(orc):
    pins.check_p1_example_storage_mode(orc)


def test_p3_example(orc):
    pins.check_p3_example(orc, GOLDEN["p3_example"])


def test_p3_example_paper_mode():
    pins.check_p3_example_paper_mode(GOLDEN["p3_example"])


def test_paper_degenerate_and_zero():
    pins.check_paper_degenerate_and_zero()


def test_paper_ties_to_even():
    pins.check_paper_ties_to_even()


def test_paper_nearest_and_bound():
    pins.check_paper_nearest_and_bound()


def test_payload_bytes(orc):
    pins.check_payload(orc, GOLDEN)


def test_effective_bits(orc):
    pins.check_effective_bits(orc, GOLDEN)


@pytest.mark.parametrize("bits,group,sym", FORMATS)
def test_error_bound(orc, bits, group, sym):
    # 20k+ groups of N(0, 0.02) with outlier columns: rounding the scale to
    # nearest instead of up breaks the bound on some of them
    W = pins.random_half_weights(160, 128 * 128, seed=bits * 1000 + group, outlier_every=53)
    pins.check_error_bound(orc, bits, group, sym, W)


def test_error_bound_wide_ranges(orc):
    # extremes of binary16: +-65504 next to subnormals, all-negative groups
    W = pins.random_half_weights(64, 256, seed=11, std=1.0)
    W[0, :] = 0x7BFF                        # 65504
    W[1, ::2] = 0xFBFF                      # -65504
    W[2, :] = np.arange(1, 257, dtype=np.uint16)          # subnormals only
    W[3, :] = W[3, :] | 0x8000              # all negative
    W[4, 5] = 0x7BFF
    W[4, 6] = 0x0001
    for bits in (4, 8):
        for sym in (False, True):
            pins.check_error_bound(orc, bits, 32, sym, W)
            pins.check_error_bound(orc, bits, 128, sym, W)


@pytest.mark.parametrize("bits,group,sym", FORMATS)
def test_exact_zero(orc, bits, group, sym):
    W = pins.random_half_weights(16, 512, seed=3)
    pins.check_exact_zero(orc, bits, group, sym, W)


@pytest.mark.parametrize("bits,sym", [(4, False), (4, True), (8, False), (8, True)])
def test_nearest_code_bruteforce(orc, bits, sym):
    W = pins.random_half_weights(3, 64, seed=bits + 10 * sym, outlier_every=17)
    pins.check_nearest_code_bruteforce(orc, bits, 32, sym, W)


def test_ties_to_even(orc):
    pins.check_ties_to_even(orc)


def test_lossless_grids(orc):
    pins.check_lossless_grids(orc)


def test_degenerate_groups(orc):
    pins.check_degenerate_groups(orc)


@pytest.mark.parametrize("bits", [4, 8])
def test_packing_layout(orc, bits):
    pins.check_packing_layout(orc, bits, pins.random_half_weights(8, 256, seed=2))


@pytest.mark.parametrize("bits,group,sym", [(4, 32, False), (4, 128, True), (8, 64, False),
                                            (8, 32, True)])
def test_exact_metadata(orc, bits, group, sym):
    W = pins.random_half_weights(6, 256, seed=21, outlier_every=37)
    pins.check_exact_metadata(orc, bits, group, sym, W)


@pytest.mark.parametrize("bits,group,sym", [(4, 128, False), (4, 32, True), (8, 64, False)])
def test_matmul_one_hot_and_zero(orc, bits, group, sym):
    pins.check_matmul_one_hot_and_zero(orc, bits, group, sym,
                                       pins.random_half_weights(24, 512, seed=4))


@pytest.mark.parametrize("bits,group,sym", [(4, 32, False), (8, 64, True)])
def test_matmul_exact_sum(orc, bits, group, sym):
    pins.check_matmul_exact_sum(orc, bits, group, sym,
                                pins.random_half_weights(5, 128, seed=6, outlier_every=9))


@pytest.mark.parametrize("bits,group,sym", [(4, 128, False), (4, 64, True), (8, 32, False)])
def test_matmul_kmajor(orc, bits, group, sym):
    pins.check_matmul_kmajor(orc, bits, group, sym,
                             pins.random_half_weights(40, 512, seed=9, outlier_every=31))


def test_matmul_at_matches_full(orc):
    W = pins.random_half_weights(33, 256, seed=12)
    X = pins.random_half_weights(3, 256, seed=13)     # any 16-bit pattern source
    X = (X & 0x7F7F) | 0x3000                       # keep them finite bfloat16
    _, codes, s, z = orc.quantize(W, 4, 64, False)
    Y, Yabs = orc.matmul(X, codes, s, z, 33, 256, 4, 64, False)
    ms = np.array([0, 2, 1, 2])
    ns = np.array([0, 32, 7, 5])
    y, yabs = orc.matmul_at(X, codes, s, z, 33, 256, 4, 64, False, ms, ns)
    assert np.array_equal(y, Y[ms, ns]) and np.array_equal(yabs, Yabs[ms, ns])


def test_dense_bf16(orc):
    pins.check_dense_bf16(orc)
