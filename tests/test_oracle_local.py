"""Pins of the oracle's local attention (one query per centre).

Definition (NeighborGraph issue, "Graph-native alternatives", item 2:
LocalAtten maps onto the per-centre CSR segment, queries = centres, keys =
edges): q_i = H_i Wq from the centre's own feature row, K = G_i Wk and
V = G_i Wv from its edges; per head l_b = s_b (q_i . k_b) / sqrt(d); softmax
over the centre's edges; out_i = sum_b P_b V_b; heads concatenated; a centre
without edges has a zero row.

The pins: closed forms (one edge, zero query weights, zero switch, two edges
via the logistic function), invariants (rows sum to one, permutation,
masking) and an independent second formulation (padded tensors with a -inf
mask and torch.softmax).
"""
import math

import numpy as np
import pytest
import torch

from neighbour_graph_attention_b200 import configs as C


def _csr(rng, counts):
    row_ptr = np.zeros(len(counts) + 1, dtype=np.int64)
    np.cumsum(counts, out=row_ptr[1:])
    e = int(row_ptr[-1])
    sw = rng.uniform(0.0, 1.0, e)
    sw[rng.uniform(size=e) < 0.5] = 1.0
    return row_ptr, sw


def _weights(rng, c):
    return [rng.normal(0, 1 / math.sqrt(c), (c, c)) for _ in range(3)]


def dense_local(row_ptr, sw, H, G, Wq, Wk, Wv, heads, pad):
    """Padded (n, pad, c) key blocks, -inf mask, torch.softmax (fp64)."""
    n = row_ptr.size - 1
    c = H.shape[1]
    d = c // heads
    blk = torch.zeros(n, pad, c, dtype=torch.float64)
    s = torch.zeros(n, pad, dtype=torch.float64)
    mask = torch.zeros(n, pad, dtype=torch.bool)
    for i in range(n):
        a, b = int(row_ptr[i]), int(row_ptr[i + 1])
        blk[i, : b - a] = torch.from_numpy(G[a:b])
        s[i, : b - a] = torch.from_numpy(sw[a:b])
        mask[i, : b - a] = True
    q = (torch.from_numpy(H) @ torch.from_numpy(Wq)).view(n, heads, 1, d)
    k = (blk @ torch.from_numpy(Wk)).view(n, pad, heads, d).transpose(1, 2)
    v = (blk @ torch.from_numpy(Wv)).view(n, pad, heads, d).transpose(1, 2)
    logits = (q @ k.transpose(-1, -2)) / math.sqrt(d) * s[:, None, None, :]
    logits = logits.masked_fill(~mask[:, None, None, :], float("-inf"))
    p = torch.softmax(logits, dim=-1)
    o = (p @ v).reshape(n, c)
    o[~mask.any(dim=1)] = 0.0        # no edges: zero row
    return o.numpy()


def test_single_edge_is_value_projection(oracle_mod):
    rng = np.random.default_rng(1)
    row_ptr, sw = _csr(rng, [1, 1, 1])
    H = rng.normal(size=(3, 8))
    G = rng.normal(size=(3, 8))
    Wq, Wk, Wv = _weights(rng, 8)
    out = oracle_mod.local_attention(row_ptr, sw, H, G, Wq, Wk, Wv, 2)
    assert np.allclose(out, G @ Wv, rtol=0, atol=1e-14)


def test_zero_query_is_mean_of_values(oracle_mod):
    rng = np.random.default_rng(2)
    row_ptr, sw = _csr(rng, [5, 9])
    H = rng.normal(size=(2, 16))
    G = rng.normal(size=(14, 16))
    _, Wk, Wv = _weights(rng, 16)
    out = oracle_mod.local_attention(row_ptr, sw, H, G, np.zeros((16, 16)), Wk, Wv, 4)
    V = G @ Wv
    assert np.allclose(out[0], V[:5].mean(axis=0), rtol=0, atol=1e-14)
    assert np.allclose(out[1], V[5:].mean(axis=0), rtol=0, atol=1e-14)


def test_zero_switch_is_uniform(oracle_mod):
    rng = np.random.default_rng(3)
    row_ptr, _ = _csr(rng, [7])
    H = rng.normal(size=(1, 8))
    G = rng.normal(size=(7, 8))
    Wq, Wk, Wv = _weights(rng, 8)
    out = oracle_mod.local_attention(row_ptr, np.zeros(7), H, G, Wq, Wk, Wv, 1)
    assert np.allclose(out[0], (G @ Wv).mean(axis=0), rtol=0, atol=1e-14)


def test_two_edges_logistic_closed_form(oracle_mod):
    # one head, c = d = 4: out = sig(l_0 - l_1) V_0 + sig(l_1 - l_0) V_1 with
    # l_b = s_b (q . k_b) / 2, q = H Wq from the centre row (not an edge row)
    H = np.array([[0.0, 0.0, 1.0, 0.0]])
    G = np.array([[1.0, 0.0, 0.0, 0.0], [0.0, 1.0, 0.0, 0.0]])
    Wq = np.zeros((4, 4)); Wq[2, 1] = 2.0          # q = (0, 2, 0, 0)
    Wk = np.zeros((4, 4)); Wk[0, 1] = 1.0; Wk[1, 1] = 3.0   # k_0 = (0,1,0,0), k_1 = (0,3,0,0)
    Wv = np.zeros((4, 4)); Wv[0, 3] = 1.0; Wv[1, 2] = 1.0   # v_0 = e_3, v_1 = e_2
    s = np.array([1.0, 0.5])
    out = oracle_mod.local_attention(np.array([0, 2]), s, H, G, Wq, Wk, Wv, 1)
    l0, l1 = 1.0 * 2.0 / 2.0, 0.5 * 6.0 / 2.0
    sig = lambda z: 1.0 / (1.0 + math.exp(-z))
    assert np.allclose(out[0], [0.0, 0.0, sig(l1 - l0), sig(l0 - l1)], rtol=0, atol=1e-15)


def test_no_edges_zero_row_and_rows_sum_to_one(oracle_mod):
    rng = np.random.default_rng(4)
    row_ptr, sw = _csr(rng, [3, 0, 6, 0])
    H = rng.normal(size=(4, 8))
    G = rng.normal(size=(9, 8))
    G[:, 0] = 1.0
    Wq, Wk, _ = _weights(rng, 8)
    Wv = np.zeros((8, 8)); Wv[0, :] = 1.0        # every value vector is all ones
    out = oracle_mod.local_attention(row_ptr, sw, H, G, Wq, Wk, Wv, 2)
    assert np.array_equal(out[1], np.zeros(8)) and np.array_equal(out[3], np.zeros(8))
    assert np.allclose(out[[0, 2]], 1.0, rtol=0, atol=1e-15)


def test_permutation_invariance_and_no_leak(oracle_mod):
    rng = np.random.default_rng(5)
    row_ptr, sw = _csr(rng, [11, 17, 6])
    H = rng.normal(size=(3, 16))
    G = rng.normal(size=(34, 16))
    Wq, Wk, Wv = _weights(rng, 16)
    a = oracle_mod.local_attention(row_ptr, sw, H, G, Wq, Wk, Wv, 4)
    perm = np.concatenate([np.arange(11), 11 + rng.permutation(17), np.arange(28, 34)])
    b = oracle_mod.local_attention(row_ptr, sw[perm], H, G[perm], Wq, Wk, Wv, 4)
    assert np.allclose(a, b, rtol=0, atol=1e-14)
    G2 = G.copy(); G2[:11] = 1e3; G2[28:] = -5.0
    c = oracle_mod.local_attention(row_ptr, sw, H, G2, Wq, Wk, Wv, 4)
    assert np.array_equal(a[1], c[1])


@pytest.mark.parametrize("key", [2, 4])
def test_dense_route_agrees(oracle_mod, key):
    w = C.workload(key)
    s = C.system(key, 0)
    csr = oracle_mod.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    rp = csr["row_ptr"]
    if key == 4:
        rp = rp[:801]
    n = rp.size - 1
    rng = np.random.default_rng(6)
    W = C.weights(key, 0).astype(np.float64)
    G = C.features(key, 0, csr["row_ptr"][-1]).astype(np.float64)
    H = rng.normal(size=(n, w.channels))
    out = oracle_mod.local_attention(rp, csr["sw"], H, G, W[0][0], W[0][1], W[0][2], w.heads)
    for pad in (w.nnei_max, 256):
        ref = dense_local(rp, csr["sw"], H, G, W[0][0], W[0][1], W[0][2], w.heads, pad)
        assert np.max(np.abs(out - ref)) <= 1e-12
