"""Randomised pin of the oracle's neighbour CSR against a separate brute force.

The brute force below restates the definition from scratch in numpy: every
source j and every lattice image S in a range wide enough for the cutoff
(periodic axes only), the edge vector v = (x_j + S . box) - x_i with each
product and sum rounded separately in the stated order, r^2 = (v_x^2 + v_y^2)
+ v_z^2, kept when r^2 < rcut^2 (strict), (i, i, 0) excluded; rows with more
than nnei_max kept the nnei_max smallest by (r^2, j, S), then put in (j, S)
order.  numpy's elementwise float64 operations round each operation on its
own, so the two must agree bit for bit.  The seeded cases are small systems
with mixed periodic and open axes, cutoffs up to beyond the box length (many
images of one source, self-images included), coordinates outside the box,
and caps that cut through shells.
"""
import numpy as np
import pytest

PBC = [(1, 1, 1)] * 4 + [(1, 1, 0), (1, 0, 1), (0, 1, 1), (1, 0, 0), (0, 0, 0)]


def brute(x, L, pbc, rcut, nnei_max):
    n = x.shape[0]
    box = np.diag(L)
    rc2 = rcut * rcut
    reach = [int(np.ceil((rcut + np.max(np.abs(x[:, k]))) / L[k])) + 2 if pbc[k] else 0
             for k in range(3)]
    grid = np.stack(np.meshgrid(*[np.arange(-r, r + 1) for r in reach], indexing="ij"),
                    axis=-1).reshape(-1, 3)
    S = grid.astype(np.float64)
    rows = []
    for i in range(n):
        cand = []
        for j in range(n):
            v = np.empty((S.shape[0], 3))
            for c in range(3):
                sh = S[:, 0] * box[0, c] + S[:, 1] * box[1, c]
                sh = sh + S[:, 2] * box[2, c]
                v[:, c] = (x[j, c] + sh) - x[i, c]
            r2 = (v[:, 0] * v[:, 0] + v[:, 1] * v[:, 1]) + v[:, 2] * v[:, 2]
            keep = r2 < rc2
            if j == i:
                keep &= np.any(grid != 0, axis=1)
            for m in np.nonzero(keep)[0]:
                cand.append((r2[m], j, *grid[m].tolist(), v[m].copy()))
        raw = len(cand)
        if raw > nnei_max:
            cand = sorted(cand, key=lambda t: t[:5])[:nnei_max]
        cand = sorted(cand, key=lambda t: t[1:5])
        rows.append((raw, cand))
    return rows


@pytest.mark.parametrize("seed", range(40))
def test_csr_matches_independent_brute_force(oracle_mod, seed):
    rng = np.random.default_rng([seed, 77])
    n = int(rng.integers(2, 9))
    L = rng.uniform(1.5, 6.0, 3)
    pbc = PBC[int(rng.integers(len(PBC)))]
    rcut = float(rng.uniform(0.3, 1.3) * np.min(L))      # often beyond L/2
    x = rng.uniform(-0.5, 1.5, size=(n, 3)) * L           # some coordinates outside the box
    want = brute(x, L, pbc, rcut, 10 ** 6)
    raw_max = max(r for r, _ in want)
    nnei_max = max(1, int(rng.integers(1, raw_max + 2))) if raw_max else 1
    if nnei_max < raw_max:
        want = brute(x, L, pbc, rcut, nnei_max)
    csr = oracle_mod.build_csr(x, np.diag(L), list(pbc), rcut, 0.5 * rcut, nnei_max)
    rp = csr["row_ptr"]
    assert np.array_equal(csr["raw"], [r for r, _ in want])
    for i, (raw, cand) in enumerate(want):
        a, b = int(rp[i]), int(rp[i + 1])
        assert b - a == len(cand)
        assert [int(j) for j in csr["src"][a:b]] == [t[1] for t in cand]
        assert csr["shift"][a:b].tolist() == [list(t[2:5]) for t in cand]
        vec = np.array([t[5] for t in cand]).reshape(-1, 3)
        assert np.array_equal(csr["vec"][a:b].view(np.uint8), vec.view(np.uint8))
        r2 = np.array([t[0] for t in cand])
        assert np.array_equal(csr["dist"][a:b], np.sqrt(r2))


def test_random_cases_exercise_the_definition(oracle_mod):
    # the seeded cases above reach what they are meant to: truncated rows,
    # self-images, open axes and sources seen under several shifts
    trunc = self_img = multi = opened = edges = 0
    for seed in range(40):
        rng = np.random.default_rng([seed, 77])
        n = int(rng.integers(2, 9))
        L = rng.uniform(1.5, 6.0, 3)
        pbc = PBC[int(rng.integers(len(PBC)))]
        rcut = float(rng.uniform(0.3, 1.3) * np.min(L))
        x = rng.uniform(-0.5, 1.5, size=(n, 3)) * L
        rows = brute(x, L, pbc, rcut, 10 ** 6)
        raw_max = max(r for r, _ in rows)
        nnei_max = max(1, int(rng.integers(1, raw_max + 2))) if raw_max else 1
        trunc += sum(r > nnei_max for r, _ in rows)
        self_img += sum(1 for i, (_, c) in enumerate(rows) for t in c if t[1] == i)
        multi += sum(len(c) - len({t[1] for t in c}) for _, c in rows)
        opened += not all(pbc)
        edges += sum(len(c) for _, c in rows)
    assert trunc >= 20 and self_img >= 20 and multi >= 50 and opened >= 5 and edges >= 1000
