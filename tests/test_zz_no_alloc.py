"""The allocation-free CSR build against the workspace build.

mlg_build_csr_noalloc serves callers that cannot allocate device memory (an
MD engine's force callback that owns every allocation, a host plugin without
an allocator): it takes its scratch from a fixed array inside the library.
Its output must be bit-identical to mlg_build_csr's, call after call, since
the array keeps the previous call's contents.

This file sorts last so that a run stopping at the first failure has already
run every other test; it needs nothing from them and passes alone too.
"""
import ctypes

import numpy as np
import pytest
import torch

from neighbour_graph_attention_b200 import configs as C

import gpu_util as U

pytestmark = pytest.mark.gpu


def _noalloc(key, seed):
    m = U.mlg()
    w = C.workload(key)
    s = C.system(key, seed)
    x = torch.as_tensor(s["coords"], device="cuda")
    t = torch.as_tensor(s["types"], device="cuda")
    csr = m.Csr.empty(w.n_atoms, w.n_atoms * w.nnei_max)
    sysd = m.make_system(x, s["box"], s["pbc"], t, s["n_types"])
    m.mlg_build_csr_noalloc(sysd, w.rcut, w.r_on, w.nnei_max, csr)
    torch.cuda.synchronize()
    return U.csr_to_numpy(csr)


def _with_workspace(key, seed):
    w = C.workload(key)
    s = C.system(key, seed)
    gpu, _ = U.gpu_build(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max,
                         s["types"], s["n_types"])
    return gpu


def test_noalloc_matches_workspace_build_on_consecutive_calls():
    # two calls in a row on different systems, then the first one again: the
    # shared array's leftovers from the previous call must not leak
    for key, seed in [(4, 0), (2, 1), (4, 0), (3, 2)]:
        got = _noalloc(key, seed)
        ref = _with_workspace(key, seed)
        assert got["status"] == ref["status"] == 0
        assert got["n_edges"] == ref["n_edges"]
        assert got["n_truncated"] == ref["n_truncated"]
        U.assert_csr_equal(got, ref)


def test_noalloc_allocates_nothing_after_setup():
    m = U.mlg()
    w = C.workload(2)
    s = C.system(2, 0)
    x = torch.as_tensor(s["coords"], device="cuda")
    csr = m.Csr.empty(w.n_atoms, w.n_atoms * w.nnei_max)
    sysd = m.make_system(x, s["box"], s["pbc"])
    m.mlg_build_csr_noalloc(sysd, w.rcut, w.r_on, w.nnei_max, csr)   # set-up call
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(5):
        m.mlg_build_csr_noalloc(sysd, w.rcut, w.r_on, w.nnei_max, csr)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_rejects_systems_beyond_the_array():
    m = U.mlg()
    w = C.workload(5)                       # 524,288 atoms: about 27 MB without the key stash
    s = C.system(5, 0)
    need = m.mlg_build_csr_workspace_bytes(w.n_atoms, w.rcut, s["box"], s["pbc"])
    assert need > m.MLG_NOALLOC_SCRATCH_BYTES
    x = torch.as_tensor(s["coords"], device="cuda")
    csr = m.Csr.empty(w.n_atoms, 1)
    sysd = m.make_system(x, s["box"], s["pbc"])
    csr.row_ptr.fill_(-7)
    code = m.mlg_build_csr_noalloc(sysd, w.rcut, w.r_on, w.nnei_max, csr, check=False)
    torch.cuda.synchronize()
    assert code == m.MLG_ERR_WORKSPACE
    assert bool((csr.row_ptr == -7).all())          # nothing was launched
    assert "workspace" in m.mlg_status_string(code).lower()
