"""Pins of the oracle's Verlet-list reuse.

Reuse of the neighbour data across MD steps in which the list is unchanged
(DPA4 LAMMPS issue, Proposed optimizations: cache the device tensors across
steps while the neighbour list is unchanged).  Reading: the list holds every
pair within rcut + skin, uncapped; each step re-evaluates it at the current
coordinates, keeps r < rcut, then caps and orders as the full build does.
While every atom has moved less than skin / 2, each pair within rcut at the
current step was within rcut + skin when the list was built (triangle
inequality), so the result must equal the full brute-force build at the
current coordinates, bit for bit.

The pins: that equality on periodic and open systems with truncated rows,
across several steps of motion; the zero-motion special case; the criterion's
boundary (an atom that moved further does lose pairs); and why the list may
not carry the cap.
"""
import numpy as np
import pytest

from neighbour_graph_attention_b200 import configs as C

KEYS = ("row_ptr", "src", "shift", "vec", "dist", "sw")


def _assert_same(a, b):
    for k in KEYS:
        assert a[k].shape == b[k].shape, k
        assert np.array_equal(a[k].view(np.uint8), b[k].view(np.uint8)), k
    assert np.array_equal(a["raw"], b["raw"])
    assert a["n_truncated"] == b["n_truncated"]


def _moved(rng, x, max_step):
    # every atom moves less than max_step: random direction, length below it
    d = rng.normal(size=x.shape)
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    return x + d * rng.uniform(0.0, max_step, size=(x.shape[0], 1))


@pytest.mark.parametrize("key,skin", [(2, 0.5), (1, 1.0), (4, 0.6)])
def test_reuse_equals_full_build_while_the_criterion_holds(oracle_mod, key, skin):
    w = C.workload(key)
    s = C.system(key, 1)
    x0 = s["coords"]
    if key == 4:            # a slice of the cluster keeps the brute force quick
        x0 = x0[:1500]
    cand = oracle_mod.verlet_candidates(x0, s["box"], s["pbc"], w.rcut, skin)
    rng = np.random.default_rng(key)
    x = x0
    for step in range(3):   # a short trajectory, all within skin / 2 of x0
        x = x0 + (_moved(rng, x0, 0.499 * skin) - x0) * (step + 1) / 3.0
        assert not oracle_mod.needs_rebuild(x, x0, skin)
        got = oracle_mod.verlet_refine(cand, x, s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
        want = oracle_mod.build_csr(x, s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
        _assert_same(got, want)
    if key in (1, 2):       # the cap is exercised: rows are truncated
        assert want["n_truncated"] > 0


def test_zero_motion_is_the_full_build_at_any_skin(oracle_mod):
    w = C.workload(2)
    s = C.system(2, 0)
    want = oracle_mod.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    for skin in (0.0, 0.3, 1.2):
        cand = oracle_mod.verlet_candidates(s["coords"], s["box"], s["pbc"], w.rcut, skin)
        got = oracle_mod.verlet_refine(cand, s["coords"], s["box"], s["pbc"], w.rcut, w.r_on,
                                       w.nnei_max)
        _assert_same(got, want)


def test_exact_shells_at_the_cutoff(oracle_mod):
    # integer simple cubic, every r^2 exact: rcut 2 is strict in the reuse too
    # (6 + 12 + 8 neighbours, not the 6 at r = 2), and a cap of 10 inside the
    # tied shell at r = sqrt(2) picks the same (source, shift) as the full build
    x = C.lattice_sites("sc", 1.0, 5)
    box, pbc = np.diag([5.0] * 3), [1, 1, 1]
    for rcut, cap in ((2.0, 64), (1.5, 10)):
        cand = oracle_mod.verlet_candidates(x, box, pbc, rcut, 0.4)
        got = oracle_mod.verlet_refine(cand, x, box, pbc, rcut, rcut - 0.5, cap)
        _assert_same(got, oracle_mod.build_csr(x, box, pbc, rcut, rcut - 0.5, cap))
        assert np.all(np.diff(got["row_ptr"]) == (26 if rcut == 2.0 else 10))


def test_an_atom_beyond_the_criterion_loses_pairs(oracle_mod):
    # two atoms 5.2 A apart in an open box, rcut 4, skin 1: the list (cutoff
    # 5) does not hold the pair; after the first atom moves 1.5 A toward the
    # second (more than skin / 2) they are 3.7 A apart, within rcut, and only
    # a rebuild finds them
    x0 = np.array([[10.0, 10.0, 10.0], [15.2, 10.0, 10.0]])
    box, pbc = np.zeros((3, 3)), [0, 0, 0]
    cand = oracle_mod.verlet_candidates(x0, box, pbc, 4.0, 1.0)
    assert cand["row_ptr"].tolist() == [0, 0, 0]
    x = x0 + np.array([[1.5, 0.0, 0.0], [0.0, 0.0, 0.0]])
    assert oracle_mod.needs_rebuild(x, x0, 1.0)
    assert oracle_mod.verlet_refine(cand, x, box, pbc, 4.0, 3.5, 8)["row_ptr"].tolist() == \
        [0, 0, 0]
    assert oracle_mod.build_csr(x, box, pbc, 4.0, 3.5, 8)["row_ptr"].tolist() == [0, 1, 2]
    # the criterion itself: a move of exactly skin / 2 already asks for a rebuild
    assert oracle_mod.needs_rebuild(x0 + [[0.5, 0.0, 0.0], [0.0, 0.0, 0.0]], x0, 1.0)
    assert not oracle_mod.needs_rebuild(x0 + [[0.4999, 0.0, 0.0], [0.0, 0.0, 0.0]], x0, 1.0)


def test_the_list_must_not_carry_the_cap(oracle_mod):
    # capping the candidate list at nnei_max (nearest at the old positions)
    # loses pairs that become nearest after motion, so the reading keeps the
    # list uncapped; on diamond-512 (cap 40 < 46 in range) that shows at once
    w = C.workload(2)
    s = C.system(2, 2)
    skin = 0.5
    full = oracle_mod.verlet_candidates(s["coords"], s["box"], s["pbc"], w.rcut, skin)
    capped = oracle_mod.build_csr(s["coords"], s["box"], s["pbc"], w.rcut + skin, w.rcut,
                                  w.nnei_max)
    x = _moved(np.random.default_rng(8), s["coords"], 0.45 * skin)
    want = oracle_mod.build_csr(x, s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    _assert_same(oracle_mod.verlet_refine(full, x, s["box"], s["pbc"], w.rcut, w.r_on,
                                          w.nnei_max), want)
    bad = oracle_mod.verlet_refine(capped, x, s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    assert not np.array_equal(bad["row_ptr"], want["row_ptr"]) or \
        not np.array_equal(bad["src"], want["src"])


def test_rewrapped_atom_triggers_a_rebuild(oracle_mod):
    # shifts in the list refer to the coordinates it was built from: an atom
    # wrapped back into the box jumps by a box length, which the criterion sees
    s = C.system(2, 0)
    x = s["coords"].copy()
    x[7, 0] += s["box"][0][0]
    assert oracle_mod.needs_rebuild(x, s["coords"], 0.5)
    assert oracle_mod.max_displacement(x, s["coords"]) == pytest.approx(s["box"][0][0])
