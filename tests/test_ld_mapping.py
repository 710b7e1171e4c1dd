"""Host replay of the direct-load kernel's index mapping (no GPU).

The formulas below restate those of csrc/gemv_ld.cuh -- the load view of a
lane (tile row r and r + 4, 16-byte chunk c of a 128-byte line holding a
pair of groups), the shared-memory slot of each 8-activation block, the
bfloat16 pair order of the unpack (u_i, u_{i+4}), and which D entries a lane
owns -- and feed them through the documented register layout of
mma.sync.m16n8k16 (A row-major 16x16, B 16x8, D 16x8).  Every owned output
must equal the group's dot product sum_k x_k (128 + u_k) for its tile row,
group and token, and every (row, group, token) must be owned exactly once
(by the lane pair L, L ^ 6 after their shuffle)."""
import numpy as np
import pytest

GROUP = 128


def a_frag(lane):
    g, t = lane >> 2, lane & 3
    # (row, col) of a0..a3, two elements each
    return [[(g, 2 * t), (g, 2 * t + 1)], [(g + 8, 2 * t), (g + 8, 2 * t + 1)],
            [(g, 2 * t + 8), (g, 2 * t + 9)], [(g + 8, 2 * t + 8), (g + 8, 2 * t + 9)]]


def b_frag(lane):
    g, t = lane >> 2, lane & 3
    return [[(2 * t, g), (2 * t + 1, g)], [(2 * t + 8, g), (2 * t + 9, g)]]


def d_frag(lane):
    g, t = lane >> 2, lane & 3
    return [(g, 2 * t), (g, 2 * t + 1), (g + 8, 2 * t), (g + 8, 2 * t + 1)]


def unpack_pairs(codes8):
    """unpack_u4 on one word of eight codes: pairs (u_i, u_{i+4}), i = 0..3,
    as the values 128 + u."""
    return [(128 + codes8[i], 128 + codes8[i + 4]) for i in range(4)]


def stage_x(x, K):
    """The staging of one token's activations: slot ((pair*4 + q)*2 + half)*4
    + t holds the 8-block at k = (2 pair + half)*128 + t*32 + 8q, permuted to
    (x0, x4, x1, x5, x2, x6, x3, x7)."""
    slots = {}
    for e in range(0, K, 8):
        gi, kg = e // GROUP, e % GROUP
        tt, q = kg // 32, (kg % 32) // 8
        slot = (((gi >> 1) * 4 + q) * 2 + (gi & 1)) * 4 + tt
        blk = x[e:e + 8]
        slots[slot] = [(blk[0], blk[4]), (blk[1], blk[5]), (blk[2], blk[6]), (blk[3], blk[7])]
    return slots


@pytest.mark.parametrize("M", [1, 2, 3, 4])
def test_unit_mapping(M):
    rng = np.random.default_rng(M)
    K = 512                                   # two pairs of groups
    rows = 8
    u = rng.integers(0, 16, size=(rows, K))   # codes of one 8-row tile
    x = rng.standard_normal((M, K))
    staged = [stage_x(x[m], K) for m in range(M)]
    for pair in range(K // 256):
        # registers of every lane for this unit
        A = {}
        for lane in range(32):
            r, c = lane >> 3, lane & 7
            k0 = pair * 256 + c * 16 * 2      # byte offset c*16 of the line -> code 32 c
            A[lane] = (u[r, k0:k0 + 32], u[r + 4, k0:k0 + 32])
        D = np.zeros((16, 8))
        for q in range(4):                    # word q of each lane's 16 bytes
            for step in (0, 1):               # even / odd mma of the word
                Am, Bm = np.zeros((16, 16)), np.zeros((16, 8))
                for lane in range(32):
                    g, t = lane >> 2, lane & 3
                    pa = unpack_pairs(A[lane][0][8 * q:8 * q + 8])
                    pb = unpack_pairs(A[lane][1][8 * q:8 * q + 8])
                    regs = ([pa[0], pb[0], pa[1], pb[1]] if step == 0
                            else [pa[2], pb[2], pa[3], pb[3]])
                    for reg, pos in zip(regs, a_frag(lane)):
                        for val, (i, j) in zip(reg, pos):
                            Am[i, j] = val
                    bm, bh = g & 3, g >> 2
                    if bm < M:
                        xv = staged[bm][((pair * 4 + q) * 2 + bh) * 4 + t]
                        bregs = [xv[0], xv[1]] if step == 0 else [xv[2], xv[3]]
                    else:
                        bregs = [(0.0, 0.0), (0.0, 0.0)]
                    for reg, pos in zip(bregs, b_frag(lane)):
                        for val, (i, j) in zip(reg, pos):
                            Bm[i, j] = val
                D += Am @ Bm
        owned = set()
        for lane in range(32):
            g, t = lane >> 2, lane & 3
            hh = g & 1
            if hh != (t >> 1):
                continue
            m0 = (2 * t) & 3
            for idx, (i, j) in enumerate(d_frag(lane)):
                m = m0 + (idx & 1)
                if m >= M:
                    continue
                row = (g >> 1) + (4 if idx >= 2 else 0)
                gi = 2 * pair + hh
                ks = slice(gi * GROUP, (gi + 1) * GROUP)
                want = float(np.dot(x[m, ks], 128 + u[row, ks]))
                assert D[i, j] == pytest.approx(want, rel=1e-12, abs=1e-9)
                key = (row, gi, m)
                assert key not in owned
                owned.add(key)
        assert len(owned) == rows * 2 * M   # every (row, group, token) once
        # the shuffle partner L ^ 6 owns the same row and token, other group
        for lane in range(32):
            g, t = lane >> 2, lane & 3
            p = lane ^ 6
            gp, tp = p >> 2, p & 3
            assert (g >> 1) == (gp >> 1) and ((2 * t) & 3) == ((2 * tp) & 3)
            assert (g & 1) != (gp & 1)
