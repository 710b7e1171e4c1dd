"""Plant plausible mistakes in copies of the C oracle and check that the pins
catch every one of them (CPU only; the planted copies are compiled into a
temporary directory and never touch the real oracle)."""
import os

import pytest

import oracle
from tests import pins

SRC = open(oracle.SOURCE).read()

# (name, original snippet, planted replacement)
MUTANTS = [
    ("range not widened to 0",
     "double lo = 0.0, hi = 0.0; /* range must contain real 0 */",
     "double lo = half_bits_to_double(w[0]), hi = lo;"),
    ("scale rounded to nearest",
     "    return lo;\n}",
     "    if (lo > 1 && half_bits_to_double(lo) - x > x - half_bits_to_double((uint16_t)(lo - 1)))\n"
     "        return (uint16_t)(lo - 1);\n    return lo;\n}"),
    ("codes truncated", "nearbyint(v / s) + z", "trunc(v / s) + z"),
    ("codes rounded half away from zero", "nearbyint(v / s) + z", "round(v / s) + z"),
    ("zero point with the wrong sign", "nearbyint(qmin - lo / s)", "nearbyint(qmin + lo / s)"),
    ("nibbles swapped", "if ((k & 1) == 0)\n", "if ((k & 1) == 1)\n"),
    ("dequantize drops the zero point",
     "What[n * K + k] = s * ((double)q - z);", "What[n * K + k] = s * (double)q;"),
    ("dequantize uses the wrong group", "int64_t g = k / group;\n            double s = half_bits_to_double(scales[n * ngroups + g]);\n            double z = symmetric ? 0.0 : half_bits_to_double(zeros[n * ngroups + g]);\n            int q",
     "int64_t g = (k + 1) % ngroups;\n            double s = half_bits_to_double(scales[n * ngroups + g]);\n            double z = symmetric ? 0.0 : half_bits_to_double(zeros[n * ngroups + g]);\n            int q"),
    ("symmetric codes stored without offset",
     "int u = symmetric ? (int)q + (1 << (bits - 1)) : (int)q;",
     "int u = symmetric ? ((int)q & ((1 << bits) - 1)) : (int)q;"),
    ("symmetric qmax off by one",
     "double qm = (double)((1 << (bits - 1)) - 1);", "double qm = (double)(1 << (bits - 1));"),
    ("matmul output transposed",
     "            Y[m * N + n] = acc;\n            Yabs[m * N + n] = accabs;",
     "            Y[n * M + m] = acc;\n            Yabs[n * M + m] = accabs;"),
    ("matmul drops the scale",
     "double w = s * ((double)code_at(codes, K, bits, symmetric, n, k) - z);\n                double p = bf16_bits_to_double(X[m * K + k]) * w;\n                acc += p;",
     "double w = ((double)code_at(codes, K, bits, symmetric, n, k) - z);\n                double p = bf16_bits_to_double(X[m * K + k]) * w;\n                acc += p;"),
    ("half decoder loses the implicit bit",
     "v = ldexp((double)(f + 1024), e - 25);", "v = ldexp((double)f, e - 25);"),
]


def _w(N, K, seed, **kw):
    return pins.random_half_weights(N, K, seed, **kw)


def _checks(orc):
    """Cheap checks first; the first failure already proves detection."""
    return [
        ("p1 storage example", lambda: pins.check_p1_example_storage_mode(orc)),
        ("p3 example", lambda: pins.check_p3_example(
            orc, {"printed_step": "0.26", "printed_bound": "0.13"})),
        ("ties to even", lambda: pins.check_ties_to_even(orc)),
        ("lossless grids", lambda: pins.check_lossless_grids(orc)),
        ("degenerate groups", lambda: pins.check_degenerate_groups(orc)),
        ("packing", lambda: pins.check_packing_layout(orc, 4, _w(4, 128, 2))),
        ("exact zero", lambda: pins.check_exact_zero(orc, 4, 32, False, _w(8, 256, 3))),
        ("error bound 4-bit", lambda: pins.check_error_bound(
            orc, 4, 128, False, _w(160, 16384, 4128, outlier_every=53))),
        ("error bound 8-bit sym", lambda: pins.check_error_bound(
            orc, 8, 128, True, _w(160, 16384, 8128, outlier_every=53))),
        ("matmul one-hot", lambda: pins.check_matmul_one_hot_and_zero(
            orc, 4, 64, False, _w(12, 256, 4))),
        ("matmul exact sum", lambda: pins.check_matmul_exact_sum(
            orc, 4, 32, False, _w(4, 64, 6))),
        ("brute force", lambda: pins.check_nearest_code_bruteforce(
            orc, 4, 32, False, _w(2, 64, 4, outlier_every=17))),
    ]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, old, new):
    assert SRC.count(old) == 1, f"snippet for '{name}' not found exactly once"
    src = tmp_path / "oracle_planted.c"
    src.write_text(SRC.replace(old, new))
    lib = oracle.build(str(src), str(tmp_path / "liboracle_planted.so"), force=True)
    orc = oracle.Oracle(lib)
    caught = []
    for check_name, fn in _checks(orc):
        try:
            fn()
        except AssertionError:
            caught.append(check_name)
            break
    # the planted library is left in place: deleting it would let a later
    # build reuse its inode, and the dynamic loader would hand back this
    # library instead of the new one
    assert caught, f"no pin caught the planted mistake '{name}'"


# ------------------------------------------------------------ paper mode
# The same for the binary64 paper-mode module (oracle/paper.py): each
# mistake is planted in a copy of its source, loaded as a separate module.

PAPER_SRC = open(os.path.join(os.path.dirname(oracle.SOURCE), "paper.py")).read()

PAPER_MUTANTS = [
    ("paper: rounding truncates", "_round = np.rint", "_round = np.trunc"),
    ("paper: rounding half away from zero", "_round = np.rint",
     "_round = lambda t: np.sign(t) * np.floor(np.abs(t) + 0.5)"),
    ("paper: range not widened to 0",
     "x_min = np.minimum(np.minimum.reduceat(v, starts), 0.0)",
     "x_min = np.minimum.reduceat(v, starts)"),
    ("paper: zero point with the wrong sign",
     "z = np.clip(_round(q_min - x_min / s), q_min, q_max)",
     "z = np.clip(_round(q_min + x_min / s), q_min, q_max)"),
    ("paper: reconstruction drops the zero point",
     "x_hat = s[g] * (q - z[g])", "x_hat = s[g] * q"),
    ("paper: degenerate scale not 1", "s = np.where(degenerate, 1.0,", "s = np.where(degenerate, 0.5,"),
    ("paper: group size ignored",
     "size = n if group_size is None else int(group_size)", "size = n"),
    ("paper: page 3 step over 2^b levels",
     "scale = (h - l) / q_max", "scale = (h - l) / (q_max + 1.0)"),
    ("paper: page 3 codes not clamped",
     "q = np.clip(_round(v / scale) + z, 0.0, q_max)", "q = _round(v / scale) + z"),
    ("paper: K-major product drops the scale",
     "blocks = q_kmajor.astype(np.float64) * scales_kmajor.astype(np.float64)[:, None, :]",
     "blocks = q_kmajor.astype(np.float64) + 0.0 * scales_kmajor.astype(np.float64)[:, None, :]"),
    ("paper: K-major groups taken strided",
     "x_groups = x.reshape(x.shape[0], n_groups, group)",
     "x_groups = x.reshape(x.shape[0], group, n_groups).transpose(0, 2, 1)"),
]


def _paper_checks(mod):
    orc = oracle.get()
    golden = {"printed_step": "0.26", "printed_bound": "0.13"}
    return [
        ("p1 paper example", lambda: pins.check_p1_example_paper_mode(mod)),
        ("p3 paper example", lambda: pins.check_p3_example_paper_mode(golden, mod)),
        ("paper degenerate / zero", lambda: pins.check_paper_degenerate_and_zero(mod)),
        ("paper ties to even", lambda: pins.check_paper_ties_to_even(mod)),
        ("paper nearest / bound", lambda: pins.check_paper_nearest_and_bound(mod)),
        ("K-major matmul", lambda: pins.check_matmul_kmajor(
            orc, 4, 32, False, _w(6, 128, 9), paper=mod)),
    ]


@pytest.mark.parametrize("name,old,new", PAPER_MUTANTS, ids=[m[0] for m in PAPER_MUTANTS])
def test_planted_paper_mistake_is_caught(tmp_path, name, old, new):
    import importlib.util
    assert PAPER_SRC.count(old) == 1, f"snippet for '{name}' not found exactly once"
    path = tmp_path / "paper_planted.py"
    path.write_text(PAPER_SRC.replace(old, new))
    spec = importlib.util.spec_from_file_location("paper_planted", str(path))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    caught = []
    for check_name, fn in _paper_checks(mod):
        try:
            fn()
        except (AssertionError, ValueError, IndexError):
            caught.append(check_name)
            break
    assert caught, f"no pin caught the planted mistake '{name}'"
