"""Pins of the oracle's neighbour CSR against lattice geometry, hand-computed
cases, scipy's KD-tree and structural invariants.

What the CSR is: the edge index / edge vector tensors that createEdgeTensors()
builds per neighbour pair (DPA4 LAMMPS issue, Root cause analysis), sorted by
destination into the destination CSR (NeighborGraph issue, Proposed fix), with
the per-centre cap sel / nnei_max (DPA4 issue, Reproduction; NeighborGraph
issue, Measurements).
"""
import json
import os

import numpy as np
import pytest
from scipy.spatial import cKDTree

from neighbour_graph_attention_b200 import configs as C


def _rows(csr):
    rp = csr["row_ptr"]
    return [slice(int(rp[i]), int(rp[i + 1])) for i in range(rp.size - 1)]


# ---------------------------------------------------------------- lattices

# shells of the ideal lattices {d^2 in units of a^2/16 (diamond) or a^2/4 (BCC) : sites},
# from tests/golden/lattice_shells.json
_GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "lattice_shells.json")))
DIAMOND_SHELLS = {int(k): v for k, v in _GOLDEN["diamond"]["shells"].items()}
BCC_SHELLS = {int(k): v for k, v in _GOLDEN["bcc"]["shells"].items()}


def _shell_hist(d, a, unit):
    q = np.rint(d * d / (a * a / unit)).astype(int)
    # every distance must sit on a shell, not between two
    assert np.allclose(d * d / (a * a / unit), q, atol=1e-9)
    vals, cnt = np.unique(q, return_counts=True)
    return dict(zip(vals.tolist(), cnt.tolist()))


@pytest.mark.parametrize("cells,rcut,total", [(2, 6.0, 158), (4, 4.0, 46), (3, 6.0, 158)])
def test_diamond_shells(oracle_mod, cells, rcut, total):
    a = 3.567
    x = C.lattice_sites("diamond", a, cells)
    box = np.diag([a * cells] * 3)
    csr = oracle_mod.build_csr(x, box, [1, 1, 1], rcut, rcut - 0.5, 256)
    counts = np.diff(csr["row_ptr"])
    assert np.all(counts == total)
    expect = {k: v for k, v in DIAMOND_SHELLS.items() if k * a * a / 16 < rcut * rcut}
    for rows in _rows(csr)[:: max(1, len(counts) // 8)]:
        assert _shell_hist(csr["dist"][rows], a, 16) == expect


@pytest.mark.parametrize("cells", [3, 5])
def test_bcc_shells(oracle_mod, cells):
    a, rcut = 2.855, 6.0
    x = C.lattice_sites("bcc", a, cells)
    csr = oracle_mod.build_csr(x, np.diag([a * cells] * 3), [1, 1, 1], rcut, 5.5, 256)
    assert np.all(np.diff(csr["row_ptr"]) == 64)
    expect = {k: v for k, v in BCC_SHELLS.items() if k * a * a / 4 < rcut * rcut}
    assert sum(expect.values()) == 64
    for rows in _rows(csr)[::7]:
        assert _shell_hist(csr["dist"][rows], a, 4) == expect


def test_tiny_cell_self_images(oracle_mod):
    # one atom, simple cubic L = 2, rcut 4.5: the lattice points n != 0 with
    # |n|^2 <= 5 -> 6 + 12 + 8 + 6 + 24 = 56 self-image edges, vec = 2 n exactly
    csr = oracle_mod.build_csr(np.zeros((1, 3)), np.diag([2.0] * 3), [1, 1, 1], 4.5, 4.0, 256)
    assert csr["row_ptr"].tolist() == [0, 56]
    n = [(i, j, k) for i in range(-2, 3) for j in range(-2, 3) for k in range(-2, 3)
         if 0 < i * i + j * j + k * k <= 5]
    assert csr["shift"].tolist() == [list(t) for t in sorted(n)]   # canonical order
    assert np.array_equal(csr["vec"], 2.0 * csr["shift"].astype(np.float64))
    assert np.all(csr["src"] == 0)
    # |vec|^2 is a small integer here, so sqrt is the only rounding
    assert np.array_equal(csr["dist"], np.sqrt(np.sum(csr["vec"] ** 2, axis=1)))


def _sc_integer_lattice(cells):
    # simple cubic, a = 1 A, integer coordinates and box: every edge vector and
    # r^2 is an exact small integer, so equal distances are exact ties
    x = C.lattice_sites("sc", 1.0, cells)
    return x, np.diag([float(cells)] * 3)


def test_cutoff_is_strict_on_an_exact_shell(oracle_mod):
    # the neighbour set is r < rcut: with rcut = 2 A exactly the sites at
    # distance 2 are out (simple cubic shells 6, 12, 8 at r^2 = 1, 2, 3; the 6
    # at r^2 = 4 follow only once rcut passes 2)
    x, box = _sc_integer_lattice(5)
    kept, raw = oracle_mod.counts(x, box, [1, 1, 1], 2.0, 256)
    assert np.all(raw == 6 + 12 + 8)
    kept, raw = oracle_mod.counts(x, box, [1, 1, 1], np.nextafter(2.0, 3.0), 256)
    assert np.all(raw == 6 + 12 + 8 + 6)
    kept, raw = oracle_mod.counts(x, box, [1, 1, 1], 1.0, 256)
    assert np.all(raw == 0)


def test_cap_breaks_exact_ties_by_source_then_shift(oracle_mod):
    # cap 10 on simple cubic with rcut 1.5: the 6 sites at r = 1 are kept and
    # 4 of the 12 exact ties at r = sqrt(2) follow, the smallest by (source,
    # shift); the expected sets come from a direct enumeration in integers
    cells, cap = 5, 10
    x, box = _sc_integer_lattice(cells)
    csr = oracle_mod.build_csr(x, box, [1, 1, 1], 1.5, 1.0, cap)
    xi = np.rint(x).astype(np.int64)
    for i in (0, 7, 62, 124):
        cand = []
        for j in range(xi.shape[0]):
            for S in np.ndindex(3, 3, 3):
                S = np.array(S) - 1
                if j == i and not S.any():
                    continue
                v = xi[j] + S * cells - xi[i]
                r2 = int(v @ v)
                if r2 <= 2:                      # r < 1.5
                    cand.append((r2, j, *S.tolist()))
        assert len(cand) == 18
        want = sorted(sorted(cand)[:cap], key=lambda t: t[1:])   # kept, in canonical order
        rows = _rows(csr)[i]
        got = [(int(j), *map(int, S)) for j, S in zip(csr["src"][rows], csr["shift"][rows])]
        assert got == [t[1:] for t in want]


def test_cap_equal_to_the_count_truncates_nothing(oracle_mod):
    # a row is truncated when its count exceeds nnei_max: simple cubic with
    # rcut 1.5 has exactly 18 neighbours per site
    x, box = _sc_integer_lattice(4)
    full = oracle_mod.build_csr(x, box, [1, 1, 1], 1.5, 1.0, 18)
    assert full["n_truncated"] == 0 and np.all(np.diff(full["row_ptr"]) == 18)
    cut = oracle_mod.build_csr(x, box, [1, 1, 1], 1.5, 1.0, 17)
    assert cut["n_truncated"] == 64 and np.all(np.diff(cut["row_ptr"]) == 17)
    assert np.all(cut["raw"] == 18)


def test_two_atoms_hand_computed(oracle_mod):
    # cubic L = 10, atoms at x = 1 and x = 9: they are 2 A apart through the
    # boundary; 8 A apart directly (outside rcut 3)
    x = np.array([[1.0, 1.0, 1.0], [9.0, 1.0, 1.0]])
    csr = oracle_mod.build_csr(x, np.diag([10.0] * 3), [1, 1, 1], 3.0, 2.5, 8)
    assert csr["row_ptr"].tolist() == [0, 1, 2]
    assert csr["src"].tolist() == [1, 0]
    assert csr["shift"].tolist() == [[-1, 0, 0], [1, 0, 0]]
    assert csr["vec"].tolist() == [[-2.0, 0.0, 0.0], [2.0, 0.0, 0.0]]
    assert csr["dist"].tolist() == [2.0, 2.0]
    assert csr["sw"].tolist() == [1.0, 1.0]
    # open along x: no edge at all
    csr = oracle_mod.build_csr(x, np.diag([10.0] * 3), [0, 1, 1], 3.0, 2.5, 8)
    assert csr["row_ptr"].tolist() == [0, 0, 0]


def test_multi_image_small_box(oracle_mod):
    # rcut > L: source 1 appears under many shifts; compare with a direct
    # enumeration of lattice translations over a generous range
    rng = np.random.default_rng(3)
    L, rcut = 2.5, 4.0
    x = rng.uniform(0, L, size=(3, 3))
    csr = oracle_mod.build_csr(x, np.diag([L] * 3), [1, 1, 1], rcut, 3.5, 1000)
    for i in range(3):
        want = []
        for j in range(3):
            for s in np.ndindex(9, 9, 9):
                S = np.array(s) - 4
                if j == i and not S.any():
                    continue
                v = x[j] + S * L - x[i]
                if v @ v < rcut * rcut:
                    want.append((j, *S.tolist()))
        rows = _rows(csr)[i]
        got = [(int(j), *map(int, S)) for j, S in zip(csr["src"][rows], csr["shift"][rows])]
        assert got == sorted(want)


def test_triclinic_box_same_lattice(oracle_mod):
    # a simple cubic lattice described by a sheared cell has the same shells
    L, rcut = 3.0, 7.0
    x = np.zeros((1, 3))
    cubic = oracle_mod.build_csr(x, np.diag([L] * 3), [1, 1, 1], rcut, 6.5, 2000)
    sheared_box = np.array([[L, 0, 0], [L, L, 0], [0, L, L]], dtype=np.float64)
    sheared = oracle_mod.build_csr(x, sheared_box, [1, 1, 1], rcut, 6.5, 2000)
    assert cubic["row_ptr"][-1] == sheared["row_ptr"][-1]
    assert np.allclose(np.sort(cubic["dist"]), np.sort(sheared["dist"]), rtol=0, atol=1e-12)
    # the shifts map to the same lattice vectors
    t1 = {tuple(np.rint(v / L).astype(int)) for v in cubic["vec"]}
    t2 = {tuple(np.rint(v / L).astype(int)) for v in sheared["vec"]}
    assert t1 == t2


# --------------------------------------------------------------- KD-tree

def _pairs_kdtree(x, boxsize, rcut):
    """Unordered pairs within rcut and their minimum-image distances."""
    tree = cKDTree(x, boxsize=boxsize)
    p = tree.query_pairs(rcut, output_type="ndarray")
    d = x[p[:, 1]] - x[p[:, 0]]
    if boxsize is not None:
        d = d - boxsize * np.rint(d / boxsize)
    return p, np.linalg.norm(d, axis=1)


def test_against_kdtree_periodic(oracle_mod):
    # rcut < L/2: the minimum image is the only image, so scipy's periodic
    # KD-tree (a library routine) gives the same pair set
    x0 = C.lattice_sites("bcc", 2.855, 10)
    L = 2.855 * 10
    rng = np.random.default_rng(11)
    x = np.mod(x0 + rng.normal(0, 0.03, x0.shape), L)
    csr = oracle_mod.build_csr(x, np.diag([L] * 3), [1, 1, 1], 6.0, 5.5, 512)
    p, d = _pairs_kdtree(x, L, 6.0)
    assert csr["row_ptr"][-1] == 2 * len(p)
    dst = np.repeat(np.arange(x.shape[0]), np.diff(csr["row_ptr"]))
    got = {(int(a), int(b)): r for a, b, r in zip(dst, csr["src"], csr["dist"])}
    for (i, j), r in zip(map(tuple, p), d):
        assert abs(got[(i, j)] - r) < 1e-12 and abs(got[(j, i)] - r) < 1e-12


def test_against_kdtree_open_cluster(oracle_mod):
    s = C.system(4, 0)
    x = s["coords"][:1500]
    csr = oracle_mod.build_csr(x, s["box"], s["pbc"], 5.0, 4.5, 1000)
    p, d = _pairs_kdtree(x, None, 5.0)
    assert csr["row_ptr"][-1] == 2 * len(p)
    assert np.all(csr["shift"] == 0)
    dst = np.repeat(np.arange(x.shape[0]), np.diff(csr["row_ptr"]))
    got = {(int(a), int(b)): r for a, b, r in zip(dst, csr["src"], csr["dist"])}
    for (i, j), r in zip(map(tuple, p), d):
        assert abs(got[(i, j)] - r) < 1e-12 and abs(got[(j, i)] - r) < 1e-12


def test_open_equals_huge_periodic_box(oracle_mod):
    s = C.system(4, 1)
    x = s["coords"][:800] + 500.0
    open_ = oracle_mod.build_csr(x, np.zeros((3, 3)), [0, 0, 0], 5.0, 4.5, 96)
    per = oracle_mod.build_csr(x, np.diag([1000.0] * 3), [1, 1, 1], 5.0, 4.5, 96)
    for k in ("row_ptr", "src", "shift", "vec", "dist", "sw"):
        assert np.array_equal(open_[k], per[k]), k


# ---------------------------------------------------------- invariants

def _check_structure(csr, n, nnei_max):
    rp = csr["row_ptr"]
    assert rp[0] == 0 and np.all(np.diff(rp) >= 0)
    assert np.array_equal(np.diff(rp), np.minimum(csr["raw"], nnei_max))
    dst = np.repeat(np.arange(n), np.diff(rp))
    key = np.column_stack([dst, csr["src"], csr["shift"]])
    # strictly increasing (dst, src, Sx, Sy, Sz): canonical and duplicate-free
    diff = np.diff(key, axis=0)
    first = np.argmax(diff != 0, axis=1)
    assert np.all(diff[np.arange(diff.shape[0]), first] > 0)
    assert not np.any((dst == csr["src"]) & ~csr["shift"].any(axis=1))
    assert np.all(csr["dist"] < 0 + np.inf)


@pytest.mark.parametrize("key", [1, 2, 4])
def test_structure_of_workloads(oracle_mod, key):
    w = C.workload(key)
    s = C.system(key, 0)
    csr = oracle_mod.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    _check_structure(csr, w.n_atoms, w.nnei_max)
    # vec is the source image minus the destination; |vec| = dist < rcut
    x = s["coords"]
    dst = np.repeat(np.arange(w.n_atoms), np.diff(csr["row_ptr"]))
    v = x[csr["src"]] + csr["shift"] @ s["box"] - x[dst]
    assert np.allclose(v, csr["vec"], rtol=0, atol=1e-12)
    assert np.allclose(np.linalg.norm(csr["vec"], axis=1), csr["dist"], rtol=1e-15, atol=0)
    assert np.all(csr["dist"] < w.rcut)
    assert np.array_equal(csr["sw"], oracle_mod.switch(csr["dist"], w.rcut, w.r_on))
    if key in (1, 2):
        assert csr["n_truncated"] == w.n_atoms      # 158 > 120 and 46 > 40
    else:
        assert csr["n_truncated"] == 0


def test_truncation_keeps_nearest(oracle_mod):
    # kept edges = the nnei_max smallest of the full list under the total
    # order (r^2, src, shift); selection checked with numpy's lexsort
    w = C.workload(1)
    s = C.system(1, 2)
    full = oracle_mod.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, 10_000)
    cut = oracle_mod.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    for i, (rf, rc) in enumerate(zip(_rows(full), _rows(cut))):
        d2 = full["dist"][rf] ** 2
        sh = full["shift"][rf]
        order = np.lexsort((sh[:, 2], sh[:, 1], sh[:, 0], full["src"][rf], d2))
        keep = np.sort(order[: w.nnei_max])    # back to canonical order
        assert np.array_equal(full["src"][rf][keep], cut["src"][rc])
        assert np.array_equal(full["shift"][rf][keep], cut["shift"][rc])
        assert np.array_equal(full["vec"][rf][keep], cut["vec"][rc])


def test_truncation_on_ideal_shells(oracle_mod):
    # ideal diamond, cap 120: shells up to d^2 = 32 a^2/16 (98 edges) are kept
    # whole, 22 of the 24 at d^2 = 35 a^2/16 follow
    a = 3.567
    x = C.lattice_sites("diamond", a, 2)
    csr = oracle_mod.build_csr(x, np.diag([2 * a] * 3), [1, 1, 1], 6.0, 5.5, 120)
    for rows in _rows(csr):
        h = _shell_hist(csr["dist"][rows], a, 16)
        assert sum(v for k, v in h.items() if k <= 32) == 98
        assert h[35] == 22 and max(h) == 35


def test_symmetric_pairs(oracle_mod):
    # no truncation: (i, j, S) present iff (j, i, -S) present, vec negated
    w = C.workload(2)
    s = C.system(2, 1)
    csr = oracle_mod.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, 256)
    n = w.n_atoms
    dst = np.repeat(np.arange(n), np.diff(csr["row_ptr"]))
    fwd = {(int(i), int(j), *map(int, S)): e
           for e, (i, j, S) in enumerate(zip(dst, csr["src"], csr["shift"]))}
    for (i, j, a, b, c), e in fwd.items():
        r = fwd[(j, i, -a, -b, -c)]
        assert np.allclose(csr["vec"][r], -csr["vec"][e], rtol=0, atol=4e-15)
        assert abs(csr["dist"][r] - csr["dist"][e]) <= 4e-15


def test_unwrapped_coordinates(oracle_mod):
    # moving atoms by whole lattice vectors changes shifts, not geometry
    w = C.workload(2)
    s = C.system(2, 0)
    rng = np.random.default_rng(5)
    lat = rng.integers(-3, 4, size=s["coords"].shape)
    x2 = s["coords"] + lat @ s["box"]
    a = oracle_mod.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    b = oracle_mod.build_csr(x2, s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    assert np.array_equal(a["row_ptr"], b["row_ptr"])
    assert np.array_equal(a["src"], b["src"])
    dst = np.repeat(np.arange(w.n_atoms), np.diff(a["row_ptr"]))
    assert np.array_equal(b["shift"], a["shift"] + lat[dst] - lat[a["src"]])
    assert np.allclose(a["vec"], b["vec"], rtol=0, atol=1e-12)


def test_single_centre_query_matches_full(oracle_mod):
    w = C.workload(4)
    s = C.system(4, 0)
    full = oracle_mod.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    rows = _rows(full)
    for i in (0, 17, 2999, w.n_atoms - 1):
        one = oracle_mod.centre(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max, i)
        for k in ("src", "shift", "vec", "dist", "sw"):
            assert np.array_equal(one[k], full[k][rows[i]]), k
        assert one["raw"] == full["raw"][i]


def test_thread_count_independent(oracle_mod):
    w = C.workload(2)
    s = C.system(2, 2)
    a = oracle_mod.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max,
                             nthreads=1)
    b = oracle_mod.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max,
                             nthreads=4)
    for k in ("row_ptr", "src", "shift", "vec", "dist", "sw"):
        assert np.array_equal(a[k], b[k])


def test_triclinic_brute_force(oracle_mod):
    # a sheared, non-cubic cell (rows are lattice vectors): compare with a
    # fixed, generous range of translations; a transposed box would differ
    rng = np.random.default_rng(9)
    box = np.array([[3.0, 0.0, 0.0], [1.1, 3.2, 0.0], [0.4, -0.7, 4.1]])
    x = rng.uniform(0, 1, size=(4, 3)) @ box
    rcut = 5.0
    csr = oracle_mod.build_csr(x, box, [1, 1, 1], rcut, 4.5, 1000)
    for i in range(4):
        want = []
        for j in range(4):
            for s in np.ndindex(11, 11, 11):
                S = np.array(s) - 5
                if j == i and not S.any():
                    continue
                v = x[j] + S @ box - x[i]
                if v @ v < rcut * rcut:
                    want.append((j, *S.tolist()))
        rows = _rows(csr)[i]
        got = [(int(j), *map(int, S)) for j, S in zip(csr["src"][rows], csr["shift"][rows])]
        assert got == sorted(want)


@pytest.mark.parametrize("lattice", ["diamond", "bcc"])
def test_golden_shells_match_lattice_enumeration(lattice):
    """The stored shell table against a direct count of lattice sites (no
    oracle): every site of an ideal cubic lattice within a few cells of a
    site at the origin, grouped by squared distance in the table's unit."""
    basis = {"diamond": [(0, 0, 0), (0, 2, 2), (2, 0, 2), (2, 2, 0),
                         (1, 1, 1), (1, 3, 3), (3, 1, 3), (3, 3, 1)],   # in units of a/4
             "bcc": [(0, 0, 0), (1, 1, 1)]}[lattice]                    # in units of a/2
    period = {"diamond": 4, "bcc": 2}[lattice]
    r = np.arange(-5, 6)
    cells = np.stack(np.meshgrid(r, r, r, indexing="ij"), axis=-1).reshape(-1, 3) * period
    sites = (cells[:, None, :] + np.array(basis)[None, :, :]).reshape(-1, 3)
    d2 = (sites ** 2).sum(axis=1)          # squared distance in units of (a/4)^2 or (a/2)^2
    table = {int(k): v for k, v in _GOLDEN[lattice]["shells"].items()}
    for k, count in table.items():
        assert k < (5 * period) ** 2       # inside the enumerated cube
        assert int((d2 == k).sum()) == count, (lattice, k)
    # and no shell below the table's largest is missing from it
    for k in np.unique(d2[(d2 > 0) & (d2 <= max(table))]):
        assert int(k) in table, (lattice, int(k))
