"""GPU parity of local attention (one query per centre) against the oracle.

LocalAtten of the NeighborGraph issue ("Graph-native alternatives", item 2):
queries from the centres' own feature rows, keys and values from their edges
in the destination CSR.  Tolerances as for the block-dense attention: FP64
max-abs 1e-10; FP32 max-abs 2e-5 * max|oracle| (the oracle computes in fp64
from the fp32 inputs).
"""
import numpy as np
import pytest
import torch

from neighbour_graph_attention_b200 import configs as C

import gpu_util as U

pytestmark = pytest.mark.gpu


def _run(csr_t, n, w, Hn, G, W):
    m = U.mlg()
    dt = U.torch_dtype(w)
    h = torch.as_tensor(Hn, dtype=dt, device="cuda")
    g = torch.zeros((max(csr_t.capacity, 1), w.channels), dtype=dt, device="cuda")
    g[: G.shape[0]] = torch.as_tensor(G, dtype=dt, device="cuda")
    out = torch.full((n, w.channels), float("nan"), dtype=dt, device="cuda")  # every row is written
    wq, wk, wv = (torch.as_tensor(np.ascontiguousarray(x), dtype=dt, device="cuda") for x in W)
    m.mlg_local_attention(csr_t, n, w.nnei_max, w.channels, w.heads, U.mlg_dtype(w), h, g, out,
                          wq, wk, wv)
    torch.cuda.synchronize()
    assert int(csr_t.status.item()) == 0
    return out.cpu().numpy()


def _sw(gpu, w):
    return gpu["sw"] if w.dtype == "f64" else gpu["sw"].astype(np.float32).astype(np.float64)


@pytest.mark.parametrize("key", [1, 2, 4])
def test_local_matches_oracle(key):
    import oracle

    w = C.workload(key)
    s = C.system(key, 0)
    gpu, csr_t = U.gpu_build(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    e, n = gpu["n_edges"], w.n_atoms
    Hn = np.random.default_rng(11).normal(size=(n, w.channels)).astype(w.np_dtype)
    G = C.features(key, 0, e)
    W = C.weights(key, 0)[0]
    out = _run(csr_t, n, w, Hn, G, W)
    ref = oracle.local_attention(gpu["row_ptr"], _sw(gpu, w), Hn, G, W[0], W[1], W[2], w.heads)
    ok, err = U.attn_tolerance_ok(w, out, ref)
    assert ok, err


def test_local_largest_system_sampled_centres():
    import oracle

    key = 5
    w = C.workload(key)
    s = C.system(key, 0)
    gpu, csr_t = U.gpu_build(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    e, n = gpu["n_edges"], w.n_atoms
    rng = np.random.default_rng(12)
    Hn = rng.normal(size=(n, w.channels)).astype(w.np_dtype)
    G = C.features(key, 0, e)
    W = C.weights(key, 0)[0]
    out = _run(csr_t, n, w, Hn, G, W)
    rp, sw = gpu["row_ptr"], _sw(gpu, w)
    sample = np.sort(np.concatenate([[0, n - 1], rng.choice(n, 510, False)]))
    rows = np.concatenate([np.arange(rp[i], rp[i + 1]) for i in sample])
    sub_rp = np.concatenate([[0], np.cumsum(rp[sample + 1] - rp[sample])])
    ref = oracle.local_attention(sub_rp, sw[rows], Hn[sample], G[rows], W[0], W[1], W[2],
                                 w.heads)
    ok, err = U.attn_tolerance_ok(w, out[sample], ref)
    assert ok, err


@pytest.mark.parametrize("dtype,channels,heads", [
    ("f64", 32, 4), ("f32", 128, 8),
    # the warp-per-centre kernel of 32 channels at every head count it takes
    ("f32", 32, 1), ("f64", 32, 2), ("f32", 32, 8),
])
def test_local_empty_rows_and_ones(dtype, channels, heads):
    """A dilute random graph (many centres without edges: zero rows) and all
    value vectors equal to ones (every other row exactly a weighted mean of
    ones)."""
    import oracle
    from neighbour_graph_attention_b200.configs import Workload

    rng = np.random.default_rng(13)
    n_atoms, L = 3000, (3000 / 0.004) ** (1.0 / 3.0)
    x = rng.uniform(0.0, L, size=(n_atoms, 3))
    gpu, csr_t = U.gpu_build(x, np.diag([L] * 3), [1, 1, 1], 4.2, 3.7, 128)
    counts = np.diff(gpu["row_ptr"])
    assert (counts == 0).sum() > 100 and counts.max() > 0
    w = Workload(0, "random", "random", 0, 0, 0, n_atoms, 4.2, 3.7, 128, channels, heads, 1,
                 dtype)
    Hn = rng.normal(size=(n_atoms, channels)).astype(w.np_dtype)
    G = rng.normal(size=(gpu["n_edges"], channels)).astype(w.np_dtype)
    W = [rng.normal(0, 1 / np.sqrt(channels), (channels, channels)).astype(w.np_dtype)
         for _ in range(3)]
    out = _run(csr_t, n_atoms, w, Hn, G, W)
    assert np.array_equal(out[counts == 0], np.zeros(((counts == 0).sum(), channels)))
    ref = oracle.local_attention(gpu["row_ptr"], _sw(gpu, w), Hn, G, W[0], W[1], W[2], heads)
    ok, err = U.attn_tolerance_ok(w, out, ref)
    assert ok, err
    G1 = G.copy()
    G1[:, 0] = 1.0
    Wv = np.zeros_like(W[2])
    Wv[0, :] = 1.0
    out1 = _run(csr_t, n_atoms, w, Hn, G1, [W[0], W[1], Wv])
    tol = 1e-13 if dtype == "f64" else 4e-6
    assert np.max(np.abs(out1[counts > 0].astype(np.float64) - 1.0)) <= tol
