"""The synthetic whole-model recipe (no GPU): 32 Llama-8B decoder layers x
7 projections, 6,979,321,856 weights, one distinct seed per matrix
(1000 * layer + projection), and the outlier-column recipe (round(0.005 K)
input channels chosen from the seed + 1)."""
import synth


def test_matrix_list():
    mats = synth.llama8b_matrices()
    assert len(mats) == 32 * 7
    assert sum(n * k for (_, _, _, n, k, _) in mats) == 6_979_321_856
    assert len({m[5] for m in mats}) == len(mats)
    assert mats[7 * 31 + 6] == (31, 6, "down", 4096, 14336, 31006)
    shapes = {(name, n, k) for (_, _, name, n, k, _) in mats}
    assert ("gate", 14336, 4096) in shapes and ("k", 1024, 4096) in shapes


def test_outlier_columns():
    cols = synth.outlier_columns(4096, 5)
    assert len(cols) == round(0.005 * 4096) == 20
    assert len(set(cols.tolist())) == 20 and max(cols.tolist()) < 4096
    assert synth.outlier_columns(4096, 5).tolist() == cols.tolist()  # seeded
