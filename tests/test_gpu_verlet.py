"""GPU parity of Verlet-skin reuse (mlg_verlet_step).

DPA4 LAMMPS issue, Proposed optimizations: keep the device tensors of the
edge construction while the neighbour list is unchanged, and rebuild at the
MD engine's skin criterion.  The list holds every (source, shift) within
rcut + skin; each step re-evaluates it at the current coordinates, keeps
r < rcut, caps and orders as the full build does.  While no atom has moved
skin / 2, the result must be the oracle's brute-force build at the current
coordinates bit for bit, and also the oracle's own refine of its candidate
list.  The rebuild decision is taken on the device: the list's build counter
shows when it tripped.
"""
import numpy as np
import pytest
import torch

from neighbour_graph_attention_b200 import configs as C

import gpu_util as U

pytestmark = pytest.mark.gpu


def _moved(rng, x, max_step):
    d = rng.normal(size=x.shape)
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    return x + d * rng.uniform(0.0, max_step, size=(x.shape[0], 1))


class Stepper:
    """The device buffers of one system's Verlet stepping."""

    def __init__(self, key, n_atoms, box, pbc, skin, out_cap=None):
        self.m = m = U.mlg()
        self.w = w = C.workload(key)
        self.box, self.pbc, self.skin = box, pbc, skin
        self.x = torch.zeros((n_atoms, 3), dtype=torch.float64, device="cuda")
        self.vl = m.VerletList.empty(n_atoms, n_atoms * 256)
        self.out = m.Csr.empty(n_atoms, n_atoms * w.nnei_max if out_cap is None else out_cap)
        self.ws = m.workspace(m.mlg_verlet_workspace_bytes(n_atoms, w.rcut, skin, box, pbc))
        self.sysd = m.make_system(self.x, box, pbc)

    def step(self, coords):
        self.x.copy_(torch.as_tensor(coords, device="cuda"))
        w = self.w
        self.m.mlg_verlet_step(self.sysd, w.rcut, w.r_on, self.skin, w.nnei_max, self.vl,
                               self.out, self.ws)
        torch.cuda.synchronize()
        got = U.csr_to_numpy(self.out)
        return got, int(self.vl.n_builds.item())


@pytest.mark.parametrize("key,skin,seed", [(2, 0.5, 1), (1, 0.8, 1), (4, 0.6, 1), (2, 0.3, 2)])
def test_steps_match_the_oracle_and_rebuild_past_half_skin(key, skin, seed):
    import oracle

    w = C.workload(key)
    s = C.system(key, seed)
    x0 = s["coords"]
    st = Stepper(key, x0.shape[0], s["box"], s["pbc"], skin)
    got, builds = st.step(x0)
    assert builds == 1 and got["status"] == 0
    U.assert_csr_equal(got, oracle.build_csr(x0, s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max))
    # the device list equals the oracle's candidate list (no row reaches the list's cap)
    cand = oracle.verlet_candidates(x0, s["box"], s["pbc"], w.rcut, skin)
    assert int(st.vl.cand.n_truncated.item()) == 0
    assert np.array_equal(st.vl.cand.row_ptr.cpu().numpy(), cand["row_ptr"])
    e = int(cand["row_ptr"][-1])
    assert np.array_equal(st.vl.cand.src[:e].cpu().numpy(), cand["src"])
    assert np.array_equal(st.vl.cand.shift[:e].cpu().numpy(), cand["shift"])
    rng = np.random.default_rng(100 + key)
    target = _moved(rng, x0, 0.499 * skin)
    for k in range(1, 4):   # a short trajectory, every atom within skin / 2 of x0
        x = x0 + (target - x0) * k / 3.0
        assert not oracle.needs_rebuild(x, x0, skin)
        got, builds = st.step(x)
        assert builds == 1, "rebuilt although no atom moved skin / 2"
        want = oracle.build_csr(x, s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
        U.assert_csr_equal(got, want)
        assert got["n_truncated"] == want["n_truncated"]
        assert got["status"] == 0
        ref = oracle.verlet_refine(cand, x, s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
        U.assert_csr_equal(got, ref)
    if key in (1, 2):
        assert want["n_truncated"] > 0  # the cap is exercised
    # one atom moves past skin / 2: the device asks for a rebuild, and the
    # result is the full build at the new coordinates
    x = target.copy()
    x[7] += np.array([0.6 * skin, 0.0, 0.0])
    assert oracle.needs_rebuild(x, x0, skin)
    got, builds = st.step(x)
    assert builds == 2
    U.assert_csr_equal(got, oracle.build_csr(x, s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max))
    # the next step measures from the new list's coordinates: no rebuild
    got, builds = st.step(x)
    assert builds == 2


def test_zero_skin_rebuilds_every_step():
    import oracle

    key = 2
    w = C.workload(key)
    s = C.system(key, 0)
    st = Stepper(key, w.n_atoms, s["box"], s["pbc"], 0.0)
    for k in range(3):
        got, builds = st.step(s["coords"])
        assert builds == k + 1
    U.assert_csr_equal(got, oracle.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on,
                                             w.nnei_max))


def test_nonfinite_coordinate_forces_a_rebuild_and_is_flagged():
    import oracle

    m = U.mlg()
    key = 2
    w = C.workload(key)
    s = C.system(key, 0)
    st = Stepper(key, w.n_atoms, s["box"], s["pbc"], 0.5)
    st.step(s["coords"])
    x = s["coords"].copy()
    x[3, 1] = np.nan
    got, builds = st.step(x)
    assert builds == 2
    assert got["status"] & m.MLG_STATUS_NONFINITE_COORD
    want = oracle.build_csr(x, s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    U.assert_csr_equal(got, want)


@pytest.mark.parametrize("key", [3, 5])
def test_large_periodic_systems_equal_the_full_gpu_build(key):
    # Fe BCC 65,536 and 524,288 atoms: after a move within skin / 2 the
    # refined CSR equals the library's own full build (itself bit-exact
    # against the oracle) at the moved coordinates
    w = C.workload(key)
    s = C.system(key, 0)
    skin = 1.0
    st = Stepper(key, w.n_atoms, s["box"], s["pbc"], skin)
    st.step(s["coords"])
    rng = np.random.default_rng(7)
    x = _moved(rng, s["coords"], 0.45 * skin)
    got, builds = st.step(x)
    assert builds == 1 and got["status"] == 0
    full, _ = U.gpu_build(x, s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    U.assert_csr_equal(got, full)


def test_list_overflow_is_flagged():
    # diamond-64 at rcut 6 + skin 1: 270-274 candidates per destination, more
    # than the list keeps (256), so the list is incomplete and says so
    m = U.mlg()
    key = 1
    w = C.workload(key)
    s = C.system(key, 1)
    st = Stepper(key, w.n_atoms, s["box"], s["pbc"], 1.0)
    got, builds = st.step(s["coords"])
    assert builds == 1
    assert got["status"] & m.MLG_STATUS_LIST_INCOMPLETE
