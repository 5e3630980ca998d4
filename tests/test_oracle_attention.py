"""Pins of the oracle's block-dense per-centre attention.

Definition (NeighborGraph issue, Proposed fix and Root cause): per centre i
with n real edges, Q = G Wq, K = G Wk, V = G Wv; per head
l_ab = s_a s_b (q_a . k_b) / sqrt(d), softmax over the centre's real edges,
O_a = sum_b P_ab V_b; heads concatenated; padded slots never contribute.

The pins: closed forms (one edge, zero query weights, zero switch, two edges
via the logistic function), invariants (rows sum to one, masking,
permutation) and an independent second formulation -- the dense route's
padded (nloc, nnei_max, c) tensors with a -inf mask and torch.softmax.
"""
import math

import numpy as np
import pytest
import torch

from neighbour_graph_attention_b200 import configs as C


def _random_csr(rng, counts):
    row_ptr = np.zeros(len(counts) + 1, dtype=np.int64)
    np.cumsum(counts, out=row_ptr[1:])
    e = int(row_ptr[-1])
    sw = rng.uniform(0.0, 1.0, e)
    sw[rng.uniform(size=e) < 0.5] = 1.0
    return row_ptr, sw


def _weights(rng, c):
    return [rng.normal(0, 1 / math.sqrt(c), (c, c)) for _ in range(3)]


def dense_route(row_ptr, sw, G, Wq, Wk, Wv, heads, pad):
    """Padded (nloc, pad, c) blocks, -inf key mask, torch.softmax (fp64)."""
    n_loc = row_ptr.size - 1
    c = G.shape[1]
    d = c // heads
    blk = torch.zeros(n_loc, pad, c, dtype=torch.float64)
    s = torch.zeros(n_loc, pad, dtype=torch.float64)
    mask = torch.zeros(n_loc, pad, dtype=torch.bool)
    for i in range(n_loc):
        a, b = int(row_ptr[i]), int(row_ptr[i + 1])
        blk[i, : b - a] = torch.from_numpy(G[a:b])
        s[i, : b - a] = torch.from_numpy(sw[a:b])
        mask[i, : b - a] = True
    q = (blk @ torch.from_numpy(Wq)).view(n_loc, pad, heads, d).transpose(1, 2)
    k = (blk @ torch.from_numpy(Wk)).view(n_loc, pad, heads, d).transpose(1, 2)
    v = (blk @ torch.from_numpy(Wv)).view(n_loc, pad, heads, d).transpose(1, 2)
    logits = q @ k.transpose(-1, -2) / math.sqrt(d)
    logits = logits * s[:, None, :, None] * s[:, None, None, :]
    logits = logits.masked_fill(~mask[:, None, None, :], float("-inf"))
    p = torch.softmax(logits, dim=-1)
    o = (p @ v).transpose(1, 2).reshape(n_loc, pad, c)
    out = np.zeros_like(G)
    for i in range(n_loc):
        a, b = int(row_ptr[i]), int(row_ptr[i + 1])
        out[a:b] = o[i, : b - a].numpy()
    return out


def test_rows_sum_to_one(oracle_mod):
    rng = np.random.default_rng(0)
    row_ptr, sw = _random_csr(rng, [1, 7, 40, 33])
    G = rng.normal(size=(int(row_ptr[-1]), 32))
    Wq, Wk, _ = _weights(rng, 32)
    for i in range(4):
        for h in range(4):
            P = oracle_mod.attention_map(row_ptr, sw, G, Wq, Wk, 4, i, h)
            n = int(row_ptr[i + 1] - row_ptr[i])
            assert P.shape == (n, n)
            assert np.all(P >= 0)
            assert np.max(np.abs(P.sum(axis=1) - 1.0)) <= 1e-15 * max(n, 4)


def test_single_edge_is_value_projection(oracle_mod):
    rng = np.random.default_rng(1)
    row_ptr, sw = _random_csr(rng, [1, 1, 1])
    G = rng.normal(size=(3, 16))
    Wq, Wk, Wv = _weights(rng, 16)
    out = oracle_mod.attention(row_ptr, sw, G, Wq, Wk, Wv, 2)
    assert np.allclose(out, G @ Wv, rtol=0, atol=1e-14)


def test_zero_query_is_mean_of_values(oracle_mod):
    rng = np.random.default_rng(2)
    row_ptr, sw = _random_csr(rng, [5, 12, 3])
    G = rng.normal(size=(20, 24))
    _, Wk, Wv = _weights(rng, 24)
    out = oracle_mod.attention(row_ptr, sw, G, np.zeros((24, 24)), Wk, Wv, 3)
    V = G @ Wv
    for i in range(3):
        a, b = row_ptr[i], row_ptr[i + 1]
        assert np.allclose(out[a:b], V[a:b].mean(axis=0), rtol=0, atol=1e-14)


def test_zero_switch_is_uniform(oracle_mod):
    # s multiplies the logits before the softmax: s = 0 everywhere -> uniform
    rng = np.random.default_rng(3)
    row_ptr, _ = _random_csr(rng, [6, 9])
    G = rng.normal(size=(15, 16))
    Wq, Wk, Wv = _weights(rng, 16)
    out = oracle_mod.attention(row_ptr, np.zeros(15), G, Wq, Wk, Wv, 4)
    V = G @ Wv
    assert np.allclose(out[:6], V[:6].mean(axis=0), rtol=0, atol=1e-14)
    assert np.allclose(out[6:], V[6:].mean(axis=0), rtol=0, atol=1e-14)


def test_two_edges_logistic_closed_form(oracle_mod):
    # n = 2, one head: O_0 = sig(l_00 - l_01) V_0 + sig(l_01 - l_00) V_1, with
    # l_ab = s_a s_b (q_a . k_b) / sqrt(c); q_a = G_a Wq (not k_a . q_b)
    G = np.array([[1.0, 0.0, 0.0, 0.0], [0.0, 1.0, 0.0, 0.0]])
    Wq = np.zeros((4, 4)); Wq[0, 2] = 2.0; Wq[1, 3] = 1.0
    Wk = np.zeros((4, 4)); Wk[0, 2] = 1.0; Wk[1, 2] = 3.0
    Wv = np.eye(4)
    s = np.array([1.0, 0.5])
    out = oracle_mod.attention(np.array([0, 2]), s, G, Wq, Wk, Wv, 1)
    # q_0 = (0,0,2,0), q_1 = (0,0,0,1); k_0 = (0,0,1,0), k_1 = (0,0,3,0)
    l00, l01 = 1 * 1 * 2 / 2.0, 1 * 0.5 * 6 / 2.0
    l10, l11 = 0.0, 0.0
    sig = lambda z: 1.0 / (1.0 + math.exp(-z))
    assert np.allclose(out[0], [sig(l00 - l01), sig(l01 - l00), 0, 0], rtol=0, atol=1e-15)
    assert np.allclose(out[1], [sig(l10 - l11), sig(l11 - l10), 0, 0], rtol=0, atol=1e-15)


def test_two_edges_large_logits(oracle_mod):
    # the same closed form with logits of 1000 and 1500: e^l alone would
    # overflow, the softmax itself does not (its value is shift-invariant)
    G = np.array([[1.0, 0.0, 0.0, 0.0], [0.0, 1.0, 0.0, 0.0]])
    Wq = np.zeros((4, 4)); Wq[0, 2] = 2000.0; Wq[1, 3] = 1.0
    Wk = np.zeros((4, 4)); Wk[0, 2] = 1.0; Wk[1, 2] = 3.0
    Wv = np.eye(4)
    s = np.array([1.0, 0.5])
    out = oracle_mod.attention(np.array([0, 2]), s, G, Wq, Wk, Wv, 1)
    l00, l01 = 2000.0 / 2.0, 0.5 * 6000.0 / 2.0
    assert np.all(np.isfinite(out))
    assert out[0, 1] == 1.0 and 0.0 < out[0, 0] <= 1e-200
    assert abs(out[0, 0] - 1.0 / (1.0 + math.exp(l01 - l00))) <= 1e-15 * out[0, 0]


def test_other_centres_do_not_leak(oracle_mod):
    # masked slots contribute zero: rows outside a centre never enter it
    rng = np.random.default_rng(4)
    row_ptr, sw = _random_csr(rng, [10, 20, 15])
    G = rng.normal(size=(45, 32))
    Wq, Wk, Wv = _weights(rng, 32)
    a = oracle_mod.attention(row_ptr, sw, G, Wq, Wk, Wv, 4)
    G2 = G.copy(); G2[:10] = 1e3 * rng.normal(size=(10, 32)); G2[30:] = -7.0
    sw2 = sw.copy(); sw2[:10] = 0.123
    b = oracle_mod.attention(row_ptr, sw2, G2, Wq, Wk, Wv, 4)
    assert np.array_equal(a[10:30], b[10:30])


def test_permutation_equivariance(oracle_mod):
    rng = np.random.default_rng(5)
    row_ptr, sw = _random_csr(rng, [17])
    G = rng.normal(size=(17, 16))
    Wq, Wk, Wv = _weights(rng, 16)
    perm = rng.permutation(17)
    a = oracle_mod.attention(row_ptr, sw, G, Wq, Wk, Wv, 2)
    b = oracle_mod.attention(row_ptr, sw[perm], G[perm], Wq, Wk, Wv, 2)
    assert np.allclose(a[perm], b, rtol=0, atol=1e-14)


@pytest.mark.parametrize("key", [1, 2, 4])
def test_dense_route_agrees(oracle_mod, key):
    w = C.workload(key)
    s = C.system(key, 0)
    csr = oracle_mod.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    W = C.weights(key, 0).astype(np.float64)
    G = C.features(key, 0, csr["row_ptr"][-1]).astype(np.float64)
    rp = csr["row_ptr"]
    if key == 4:      # a slice of centres keeps the padded tensors small
        rp = rp[:801]
    out = oracle_mod.attention(rp, csr["sw"], G, W[0][0], W[0][1], W[0][2], w.heads)
    for pad in (w.nnei_max, 256):   # padding width must not matter
        ref = dense_route(rp, csr["sw"], G, W[0][0], W[0][1], W[0][2], w.heads, pad)
        e = int(rp[-1])
        assert np.max(np.abs(out[:e] - ref[:e])) <= 1e-12


def test_forward_layers_chain(oracle_mod):
    w = C.workload(2)
    s = C.system(2, 0)
    csr = oracle_mod.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    W = C.weights(2, 0)
    G = C.features(2, 0, csr["row_ptr"][-1])
    outs = oracle_mod.forward(csr["row_ptr"], csr["sw"], G, W, w.heads)
    assert len(outs) == 6
    g = G
    for layer in range(6):
        g = oracle_mod.attention(csr["row_ptr"], csr["sw"], g, *W[layer], w.heads)
        assert np.array_equal(outs[layer], g)


def test_forward_fp32_sees_only_fp32_values(oracle_mod):
    # the fp32 path stores every layer in fp32 and reads s(r) as fp32: each
    # layer's output is an fp32 array, and switch values that round to the
    # same fp32 number give the same result
    w = C.workload(2)
    s = C.system(2, 1)
    csr = oracle_mod.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    W = C.weights(2, 1)[:2].astype(np.float32)
    G = C.features(2, 1, csr["row_ptr"][-1]).astype(np.float32)
    sw = csr["sw"]
    assert np.any(sw.astype(np.float32).astype(np.float64) != sw)
    outs = oracle_mod.forward(csr["row_ptr"], sw, G, W, w.heads, "f32")
    assert [o.dtype for o in outs] == [np.float32, np.float32]
    outs32 = oracle_mod.forward(csr["row_ptr"], sw.astype(np.float32), G, W, w.heads, "f32")
    assert all(np.array_equal(a, b) for a, b in zip(outs, outs32))
    # the second layer reads the first layer's fp32 output
    again = oracle_mod.forward(csr["row_ptr"], sw, outs[0], W[1:], w.heads, "f32")
    assert np.array_equal(again[0], outs[1])
