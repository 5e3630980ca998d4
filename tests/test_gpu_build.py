"""GPU parity of the destination CSR build: bit-exact against the oracle.

The CSR is the on-device replacement of createEdgeTensors() (DPA4 LAMMPS
issue, Root cause analysis) in destination-CSR form (NeighborGraph issue,
Proposed fix). Every array (row_ptr, src, shift, vec, dist, sw) must match
the brute-force oracle byte for byte; at the largest size, sampled centres
are compared one by one and structural properties are checked everywhere.
"""
import functools

import numpy as np
import pytest
import torch

from neighbour_graph_attention_b200 import configs as C

import gpu_util as U

pytestmark = pytest.mark.gpu


@functools.lru_cache(maxsize=None)
def oracle_csr(key, seed):
    import oracle

    w = C.workload(key)
    s = C.system(key, seed)
    return oracle.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("key", [1, 2, 3, 4])
def test_csr_bit_exact(key, seed):
    w = C.workload(key)
    s = C.system(key, seed)
    gpu, _ = U.gpu_build(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max,
                         s["types"], s["n_types"])
    ref = oracle_csr(key, seed)
    assert gpu["status"] == 0
    assert gpu["n_edges"] == ref["row_ptr"][-1]
    assert gpu["n_truncated"] == ref["n_truncated"]
    U.assert_csr_equal(gpu, ref)


def _digests():
    import json
    import os

    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "csr_digests.json")
    with open(path) as f:
        return json.load(f)["graphs"]


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("key", [3, 5])
def test_csr_full_size_digests(key, seed):
    """Every array of the full-size Fe BCC graphs (65,536 and 524,288 atoms),
    edge for edge: SHA-256 of the device CSR against digests of the oracle's
    brute-force CSR, written by tests/golden/make_csr_digests.py (which calls
    only the oracle)."""
    import hashlib

    rec = _digests()[f"{key}:{seed}"]
    w = C.workload(key)
    s = C.system(key, seed)
    assert (rec["n_atoms"], rec["rcut"], rec["nnei_max"]) == (w.n_atoms, w.rcut, w.nnei_max)
    gpu, _ = U.gpu_build(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max,
                         s["types"], s["n_types"])
    assert gpu["status"] == 0
    assert gpu["n_edges"] == rec["n_edges"] and gpu["n_truncated"] == rec["n_truncated"]
    for k, dt in (("row_ptr", np.int64), ("src", np.int32), ("shift", np.int32),
                  ("vec", np.float64), ("dist", np.float64), ("sw", np.float64)):
        a = np.ascontiguousarray(gpu[k], dtype=dt)
        assert hashlib.sha256(a.tobytes()).hexdigest() == rec["sha256"][k], k


def test_largest_system_sampled_and_properties():
    import oracle

    key = 5
    w = C.workload(key)
    s = C.system(key, 0)
    gpu, _ = U.gpu_build(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max,
                         s["types"], s["n_types"])
    n = w.n_atoms
    rp = gpu["row_ptr"]
    assert gpu["status"] == 0 and gpu["n_truncated"] == 0
    # ideal BCC has 64 neighbours within 6 A (next shell 6.22 A); with 0.03 A
    # jitter a handful of 7th-shell pairs cross the cutoff in a box this large
    counts = np.diff(rp)
    assert gpu["n_edges"] == rp[-1] and abs(int(rp[-1]) - 64 * n) < 64
    assert counts.min() >= 62 and counts.max() <= 66 and np.sum(counts != 64) < 32
    rng = np.random.default_rng(123)
    sample = np.concatenate([[0, 1, n - 1], rng.choice(n, 96, replace=False)])
    for i in sample:
        ref = oracle.centre(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max, int(i))
        a, b = int(rp[i]), int(rp[i + 1])
        for k in ("src", "shift", "vec", "dist", "sw"):
            assert np.array_equal(gpu[k][a:b].view(np.uint8), ref[k].view(np.uint8)), (i, k)
    # canonical order and no duplicates everywhere: strictly increasing keys
    dst = np.repeat(np.arange(n), np.diff(rp))
    key_ = (dst.astype(np.int64) << 40) + (gpu["src"].astype(np.int64) << 12) + \
        ((gpu["shift"][:, 0] + 2) << 8) + ((gpu["shift"][:, 1] + 2) << 4) + (gpu["shift"][:, 2] + 2)
    assert np.all(np.abs(gpu["shift"]) <= 1)
    assert np.all(np.diff(key_) > 0)
    assert np.all(gpu["dist"] < w.rcut) and np.all(gpu["dist"] > 0)
    # symmetric pairs: (i, j, S) <-> (j, i, -S), vec negated up to rounding
    fwd = (dst.astype(np.int64) * n + gpu["src"]) * 27 + \
        ((gpu["shift"][:, 0] + 1) * 9 + (gpu["shift"][:, 1] + 1) * 3 + gpu["shift"][:, 2] + 1)
    rev = (gpu["src"].astype(np.int64) * n + dst) * 27 + \
        ((1 - gpu["shift"][:, 0]) * 9 + (1 - gpu["shift"][:, 1]) * 3 + 1 - gpu["shift"][:, 2])
    order = np.argsort(fwd)
    pos = np.searchsorted(fwd[order], rev)
    assert np.array_equal(fwd[order][pos], rev)
    assert np.max(np.abs(gpu["vec"][order][pos] + gpu["vec"])) <= 1e-13


def test_deterministic_and_side_stream():
    w = C.workload(3)
    s = C.system(3, 1)
    a, _ = U.gpu_build(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    side = torch.cuda.Stream()
    noise = torch.randn(4096, 4096, device="cuda")
    with torch.cuda.stream(side):
        for _ in range(3):
            noise = noise @ noise.T * 1e-4                 # concurrent work on the side stream
        b, _ = U.gpu_build(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max,
                           stream=side)
    U.assert_csr_equal(b, a)
    for _ in range(3):
        c, _ = U.gpu_build(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
        U.assert_csr_equal(c, a)


def test_rebuild_reuses_workspace_without_stale_state():
    import oracle

    m = U.mlg()
    w = C.workload(2)
    s0, s1 = C.system(2, 0), C.system(2, 1)
    need = m.mlg_build_csr_workspace_bytes(w.n_atoms, w.rcut, s0["box"], s0["pbc"])
    ws = m.workspace(need)
    ws.fill_(0xAB)                                          # garbage in the workspace
    for s in (s0, s1, s0):
        gpu, _ = U.gpu_build(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max, ws=ws)
        ref = oracle.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
        U.assert_csr_equal(gpu, ref)


def _oracle_vs_gpu(x, box, pbc, rcut, r_on, nnei):
    import oracle

    gpu, _ = U.gpu_build(x, box, pbc, rcut, r_on, nnei)
    ref = oracle.build_csr(x, box, pbc, rcut, r_on, nnei)
    assert gpu["n_truncated"] == ref["n_truncated"]
    U.assert_csr_equal(gpu, ref)
    return gpu


@pytest.mark.parametrize("jitter", [0.0, 0.02])
def test_overflow_rows_beyond_shared_memory(jitter):
    # simple cubic, spacing 1 A, rcut 6: about 900 in-cutoff neighbours, more
    # than the 512 candidates a warp holds in shared memory -> threshold path
    x = C.lattice_sites("sc", 1.0, 12)
    x = np.mod(x + np.random.default_rng(4).normal(0, jitter, x.shape), 12.0)
    g = _oracle_vs_gpu(x, np.diag([12.0] * 3), [1, 1, 1], 6.0, 5.5, 100)
    assert np.all(np.diff(g["row_ptr"]) == 100)


def test_truncation_with_exact_ties():
    # ideal diamond (no jitter): many equal distances at the cap
    a = 3.567
    x = C.lattice_sites("diamond", a, 2)
    _oracle_vs_gpu(x, np.diag([2 * a] * 3), [1, 1, 1], 6.0, 5.5, 120)
    x3 = C.lattice_sites("diamond", a, 3)
    _oracle_vs_gpu(x3, np.diag([3 * a] * 3), [1, 1, 1], 6.0, 5.5, 100)


@pytest.mark.parametrize("case", ["tiny", "three", "mixed_xy", "mixed_x", "unwrapped", "open"])
def test_geometry_cases(case):
    rng = np.random.default_rng(21)
    if case == "tiny":
        g = _oracle_vs_gpu(np.zeros((1, 3)), np.diag([2.0] * 3), [1, 1, 1], 4.5, 4.0, 256)
        assert g["n_edges"] == 56
    elif case == "three":
        x = rng.uniform(0, 2.5, size=(3, 3))
        _oracle_vs_gpu(x, np.diag([2.5] * 3), [1, 1, 1], 4.0, 3.5, 256)
    elif case in ("mixed_xy", "mixed_x"):
        s = C.system(2, 0)
        pbc = [1, 1, 0] if case == "mixed_xy" else [1, 0, 0]
        _oracle_vs_gpu(s["coords"], s["box"], pbc, 4.0, 3.5, 40)
    elif case == "unwrapped":
        s = C.system(2, 2)
        lat = rng.integers(-3, 4, size=s["coords"].shape)
        _oracle_vs_gpu(s["coords"] + lat @ s["box"], s["box"], s["pbc"], 4.0, 3.5, 40)
    elif case == "open":
        s = C.system(4, 2)
        _oracle_vs_gpu(s["coords"][:3000] * 1.3 + 50.0, np.zeros((3, 3)), [0, 0, 0], 5.0, 4.5, 96)


def test_degenerate_sizes():
    # one isolated atom; two atoms out of range; all atoms at one point (open)
    g = _oracle_vs_gpu(np.array([[1.0, 2.0, 3.0]]), np.zeros((3, 3)), [0, 0, 0], 5.0, 4.5, 8)
    assert g["n_edges"] == 0
    _oracle_vs_gpu(np.array([[0.0, 0, 0], [10.0, 0, 0]]), np.zeros((3, 3)), [0, 0, 0], 5.0, 4.5, 8)
    g = _oracle_vs_gpu(np.ones((40, 3)), np.zeros((3, 3)), [0, 0, 0], 5.0, 4.5, 16)
    assert g["n_edges"] == 40 * 16 and np.all(g["dist"] == 0.0)


def test_nonfinite_and_type_status():
    import oracle

    w = C.workload(2)
    s = C.system(2, 0)
    x = s["coords"].copy()
    x[7, 1] = np.nan
    x[300, 0] = np.inf
    types = np.zeros(w.n_atoms, dtype=np.int32)
    types[11] = 5
    gpu, _ = U.gpu_build(x, s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max, types, 2)
    m = U.mlg()
    assert gpu["status"] & m.MLG_STATUS_NONFINITE_COORD
    assert gpu["status"] & m.MLG_STATUS_TYPE_RANGE
    # the other atoms get exactly the oracle's graph (non-finite atoms never pair)
    ref = oracle.build_csr(x, s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    U.assert_csr_equal(gpu, ref)
    assert gpu["row_ptr"][8] == gpu["row_ptr"][7]


def test_capacity_overflow_reported():
    w = C.workload(2)
    s = C.system(2, 0)
    ref = oracle_csr(2, 0)
    e = int(ref["row_ptr"][-1])
    gpu, _ = U.gpu_build(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max,
                         capacity=e - 100)
    m = U.mlg()
    assert gpu["status"] & m.MLG_STATUS_CAPACITY
    assert gpu["n_edges"] == e
    U.assert_csr_equal(gpu, ref, rows=e - 100)
