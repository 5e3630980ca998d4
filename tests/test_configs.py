"""The seeded synthetic workloads: determinism, shapes and stated structure."""
import numpy as np
import pytest

from neighbour_graph_attention_b200 import configs as C


@pytest.mark.parametrize("key", [1, 2, 3, 4, 5])
def test_system_shapes_and_determinism(key):
    w = C.workload(key)
    a, b = C.system(key, 0), C.system(key, 0)
    assert a["coords"].shape == (w.n_atoms, 3) and a["coords"].dtype == np.float64
    assert np.array_equal(a["coords"], b["coords"])
    assert not np.array_equal(a["coords"], C.system(key, 1)["coords"])
    assert a["types"].shape == (w.n_atoms,) and a["types"].dtype == np.int32
    if w.periodic:
        L = w.a * w.cells
        assert np.array_equal(a["box"], np.diag([L] * 3))
        assert np.all(a["coords"] >= 0) and np.all(a["coords"] <= L)
        assert a["pbc"].tolist() == [1, 1, 1]
    else:
        assert a["pbc"].tolist() == [0, 0, 0]


def test_protein_cluster_structure():
    s = C.system(4, 0)
    x = s["coords"]
    assert np.bincount(s["types"]).tolist() == [2982, 1908, 537, 537]
    radius = (3 * 5964 / (4 * np.pi * 0.1)) ** (1 / 3)
    assert abs(radius - 24.24) < 0.01
    assert np.all(np.linalg.norm(x, axis=1) <= radius)
    from scipy.spatial import cKDTree
    assert len(cKDTree(x).query_pairs(1.0 - 1e-12)) == 0      # minimum separation


@pytest.mark.parametrize("key", [1, 3])
def test_weights_and_features(key):
    w = C.workload(key)
    W = C.weights(key, 0)
    assert W.shape == (w.n_layers, 3, w.channels, w.channels) and W.dtype == w.np_dtype
    assert abs(W.astype(np.float64).std() * np.sqrt(w.channels) - 1.0) < 0.05
    G = C.features(key, 0, 1000)
    assert G.shape == (1000, w.channels) and G.dtype == w.np_dtype
    assert np.array_equal(G, C.features(key, 0, 1000))
