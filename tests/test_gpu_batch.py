"""GPU parity of the batched build (several systems, one CSR) against the
oracle's per-system graphs joined with atom and edge offsets -- bit for bit.

The source pages batch many structures per GPU call (NValchemi batching) and
report neighbour-cache defects after same-size refills, gradual cell
changes and partition changes.  The library keeps no cache, so each of those
cases must give the fresh graph; the tests run them in sequence on one
workspace and one CSR.
"""
import numpy as np
import pytest
import torch

from neighbour_graph_attention_b200 import configs as C

import gpu_util as U

pytestmark = pytest.mark.gpu

RCUT, R_ON, NNEI = 4.0, 3.5, 48


def _systems(seed):
    rng = np.random.default_rng(seed)
    s2 = C.system(2, seed % 3)
    s1 = C.system(1, seed % 3)
    s4 = C.system(4, seed % 3)
    L = 11.0
    rnd = rng.uniform(0.0, L, size=(200, 3))
    return [
        (s2["coords"], s2["box"], s2["pbc"]),                      # periodic diamond, 512 atoms
        (np.zeros((0, 3)), np.diag([5.0] * 3), [1, 1, 1]),          # empty system
        (s1["coords"], s1["box"], s1["pbc"]),                      # small periodic cell (64)
        (s4["coords"][:300], np.zeros((3, 3)), [0, 0, 0]),          # open cluster (300)
        (rnd, np.diag([L] * 3), [1, 1, 1]),                        # random periodic box (200)
    ]


def oracle_batch(systems):
    import oracle

    rp, src, shift, vec, dist, sw = [np.zeros(1, dtype=np.int64)], [], [], [], [], []
    ntr, aoff, eoff = 0, 0, 0
    for x, box, pbc in systems:
        if len(x) == 0:
            continue
        g = oracle.build_csr(x, box, pbc, RCUT, R_ON, NNEI)
        rp.append(g["row_ptr"][1:] + eoff)
        src.append(g["src"] + aoff)
        shift.append(g["shift"]); vec.append(g["vec"]); dist.append(g["dist"]); sw.append(g["sw"])
        ntr += g["n_truncated"]
        aoff += len(x)
        eoff += int(g["row_ptr"][-1])
    cat = lambda v, dt, shape: np.concatenate(v) if v else np.zeros(shape, dtype=dt)
    return {"row_ptr": np.concatenate(rp), "src": cat(src, np.int32, (0,)),
            "shift": cat(shift, np.int32, (0, 3)), "vec": cat(vec, np.float64, (0, 3)),
            "dist": cat(dist, np.float64, (0,)), "sw": cat(sw, np.float64, (0,)),
            "n_truncated": ntr}


class Batch:
    """One CSR and one workspace, reused across builds (as a cache would be)."""

    def __init__(self, capacity, ws_bytes):
        m = U.mlg()
        self.m = m
        self.n_max = capacity // NNEI
        self.csr = m.Csr.empty(self.n_max, capacity, device="cuda")
        self.ws = m.workspace(ws_bytes, device="cuda")
        self.ws.fill_(0xAB)

    def build(self, systems, capacity=None):
        m = self.m
        keep = []
        descs = []
        for x, box, pbc in systems:
            xd = torch.as_tensor(np.ascontiguousarray(x, dtype=np.float64).reshape(-1, 3),
                                 device="cuda")
            keep.append(xd)
            descs.append(m.make_system(xd, box, pbc))
        need = m.mlg_build_csr_batch_workspace_bytes(descs, RCUT)
        assert 0 < need <= self.ws.numel()
        n = sum(len(x) for x, _, _ in systems)
        csr = self.csr
        if capacity is not None:
            csr = m.Csr(capacity, *[getattr(self.csr, f) for f in
                                    ("row_ptr", "src", "shift", "vec", "dist", "sw", "n_edges",
                                     "n_truncated", "status")])
        m.mlg_build_csr_batch(descs, RCUT, R_ON, NNEI, csr, self.ws)
        torch.cuda.synchronize()
        out = U.csr_to_numpy(csr)
        out["row_ptr"] = out["row_ptr"][: n + 1]
        return out


def test_batch_matches_joined_oracle_graphs():
    systems = _systems(0)
    b = Batch(sum(len(x) for x, _, _ in systems) * NNEI, 64 << 20)
    gpu = b.build(systems)
    ref = oracle_batch(systems)
    assert gpu["status"] == 0
    assert gpu["n_truncated"] == ref["n_truncated"]
    assert gpu["n_edges"] == int(ref["row_ptr"][-1])
    U.assert_csr_equal(gpu, ref)


def test_batch_cache_defect_classes():
    """Same-size refill, gradual cell change, pbc change and a new atom
    partition, one after another on the same buffers: each gives the fresh
    graph."""
    systems = _systems(0)
    b = Batch(2000 * NNEI, 64 << 20)
    steps = []
    refill = list(systems)
    refill[0] = _systems(1)[0]                     # another diamond of the same size
    refill[2] = _systems(2)[2]
    steps.append(refill)
    for t in (1, 2, 3):                            # the box (and atoms) grow by 0.2% a step
        f = 1.0 + 0.002 * t
        grown = list(refill)
        x, box, pbc = refill[0]
        grown[0] = (x * f, np.asarray(box) * f, pbc)
        steps.append(grown)
    flipped = list(steps[-1])
    x, box, _ = flipped[4]
    flipped[4] = (x, box, [1, 1, 0])               # one axis of one system becomes open
    steps.append(flipped)
    x0 = np.concatenate([flipped[3][0], flipped[4][0][:100]])
    steps.append([flipped[0], (x0, np.zeros((3, 3)), [0, 0, 0]),
                  (flipped[4][0][100:], flipped[4][1], [1, 1, 1])])   # a new partition
    for st in steps:
        gpu = b.build(st)
        ref = oracle_batch(st)
        assert gpu["status"] == 0
        assert gpu["n_truncated"] == ref["n_truncated"]
        U.assert_csr_equal(gpu, ref)


def test_batch_capacity_overflow_and_empty():
    systems = _systems(0)
    ref = oracle_batch(systems)
    e = int(ref["row_ptr"][-1])
    b = Batch(sum(len(x) for x, _, _ in systems) * NNEI, 64 << 20)
    gpu = b.build(systems, capacity=e - 333)
    m = U.mlg()
    assert gpu["status"] & m.MLG_STATUS_CAPACITY
    assert gpu["n_edges"] == e
    U.assert_csr_equal(gpu, ref, rows=e - 333)
    empty = b.build([(np.zeros((0, 3)), np.diag([5.0] * 3), [1, 1, 1])])
    assert empty["n_edges"] == 0 and empty["status"] == 0
    assert np.array_equal(empty["row_ptr"], np.zeros(1, dtype=np.int64))
