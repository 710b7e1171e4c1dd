"""The information tables of oracle/snr_table.py (values not pinned to any
page): page 3's bound |w - w^| <= scale/2 holds on every group in paper mode,
error falls as bits rise, and the traffic arithmetic agrees with page 1
section 2's payload count (1024 INT4 weights at group 128 = 544 bytes)."""
import numpy as np
import pytest

import synth
from oracle import snr_table


@pytest.fixture(scope="module")
def weights():
    return synth.weight(16, 256, seed=3).float().numpy().astype(np.float64)


@pytest.mark.parametrize("group", [32, 128, 256, None])
def test_error_bound_and_monotone_in_bits(weights, group):
    rows = [snr_table.error_row(weights, b, group) for b in snr_table.BITS]
    for snr, emax, ratio in rows:
        assert np.isfinite(snr) and emax > 0
        assert ratio <= 1.0 + 1e-12          # |w - w^| <= scale/2
    snrs = [r[0] for r in rows]
    assert all(a < b for a, b in zip(snrs, snrs[1:]))


def test_effective_bits_and_payload():
    assert snr_table.effective_bits(4, 128, 1 << 20) == 4.25
    assert snr_table.effective_bits(4, None, 1 << 20) == pytest.approx(4.0, abs=1e-4)
    # fused bytes per weight x 1024 weights = page 1's 544-byte payload
    text = snr_table.tables(16, 256)
    row = [l for l in text.splitlines() if l.startswith("| 4 | 128 | 0.5312")]
    assert row and 0.53125 * 1024 == 544
