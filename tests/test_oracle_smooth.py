"""Pins of the oracle's slot-occupancy ("smooth") attention.

The NeighborGraph issue (Numerics note) names only the ingredients: a count
of phantom slots, which can be signed, and a denominator that depends on how
many slots are occupied; the weights factor as
w_b = softmax_b * (sum_b e_b / D~).  The reading: the dense route pads every
centre to nnei_max slots with zero features and zero switch, so a padded
slot's logit is exactly 0, and left unmasked it enters the softmax
denominator (its value row is 0).  The pins: that dense route itself (torch,
padded, no mask), the stated factorization, the vanilla attention when no
slot is padded, and a closed form when every logit is 0.
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


def dense_unmasked(row_ptr, sw, G, Wq, Wk, Wv, heads, nnei_max):
    """The dense route: (nloc, nnei_max, c) blocks, zero features and zero
    switch in padded slots, no mask, torch.softmax over all slots (fp64)."""
    n_loc = row_ptr.size - 1
    c = G.shape[1]
    d = c // heads
    blk = torch.zeros(n_loc, nnei_max, c, dtype=torch.float64)
    s = torch.zeros(n_loc, nnei_max, dtype=torch.float64)
    for i in range(n_loc):
        a, b = int(row_ptr[i]), int(row_ptr[i + 1])
        blk[i, : b - a] = torch.from_numpy(G[a:b])
        s[i, : b - a] = torch.from_numpy(sw[a:b])
    q = (blk @ torch.from_numpy(Wq)).view(n_loc, nnei_max, heads, d).transpose(1, 2)
    k = (blk @ torch.from_numpy(Wk)).view(n_loc, nnei_max, heads, d).transpose(1, 2)
    v = (blk @ torch.from_numpy(Wv)).view(n_loc, nnei_max, heads, d).transpose(1, 2)
    logits = q @ k.transpose(-1, -2) / math.sqrt(d) * s[:, None, :, None] * s[:, None, None, :]
    o = (torch.softmax(logits, dim=-1) @ v).transpose(1, 2).reshape(n_loc, nnei_max, c)
    out = np.zeros_like(G)
    for i in range(n_loc):
        a, b = int(row_ptr[i]), int(row_ptr[i + 1])
        out[a:b] = o[i, : b - a].numpy()
    return out


@pytest.mark.parametrize("key", [2, 4])
def test_dense_padded_route_without_mask(oracle_mod, key):
    w = C.workload(key)
    s = C.system(key, 0)
    csr = oracle_mod.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    rp = csr["row_ptr"]
    if key == 4:
        rp = rp[:401]
    W = C.weights(key, 0).astype(np.float64)
    G = C.features(key, 0, csr["row_ptr"][-1]).astype(np.float64)
    out = oracle_mod.attention_smooth(rp, csr["sw"], G, W[0][0], W[0][1], W[0][2], w.heads,
                                      w.nnei_max)
    ref = dense_unmasked(rp, csr["sw"], G, W[0][0], W[0][1], W[0][2], w.heads, w.nnei_max)
    e = int(rp[-1])
    assert np.max(np.abs(out[:e] - ref[:e])) <= 1e-12
    if key == 4:      # ragged rows: the phantoms change the result
        plain = oracle_mod.attention(rp, csr["sw"], G, W[0][0], W[0][1], W[0][2], w.heads)
        assert np.max(np.abs(out[:e] - plain[:e])) > 1e-3


def test_factorizes_as_rescaled_softmax(oracle_mod):
    """w_b = softmax_b * (sum_b e_b / D~): the smooth output is the plain one
    times the row's occupancy factor, computed here from the logits."""
    rng = np.random.default_rng(3)
    counts = [5, 12, 1, 9]
    nnei = 16
    row_ptr, sw = _csr(rng, counts)
    c, heads = 8, 2
    d = c // heads
    G = rng.normal(size=(int(row_ptr[-1]), c))
    Wq, Wk, Wv = (rng.normal(0, 1 / math.sqrt(c), (c, c)) for _ in range(3))
    smooth = oracle_mod.attention_smooth(row_ptr, sw, G, Wq, Wk, Wv, heads, nnei)
    plain = oracle_mod.attention(row_ptr, sw, G, Wq, Wk, Wv, heads)
    for i in range(len(counts)):
        a, b = int(row_ptr[i]), int(row_ptr[i + 1])
        q, k = G[a:b] @ Wq, G[a:b] @ Wk
        for h in range(heads):
            lg = (q[:, h * d:(h + 1) * d] @ k[:, h * d:(h + 1) * d].T) / math.sqrt(d)
            lg = lg * sw[a:b, None] * sw[None, a:b]
            m = np.maximum(lg.max(axis=1), 0.0)
            e = np.exp(lg - m[:, None]).sum(axis=1)
            factor = e / (e + (nnei - (b - a)) * np.exp(-m))
            assert np.allclose(smooth[a:b, h * d:(h + 1) * d],
                               plain[a:b, h * d:(h + 1) * d] * factor[:, None],
                               rtol=1e-12, atol=1e-14)


def test_full_rows_are_plain_attention(oracle_mod):
    rng = np.random.default_rng(4)
    row_ptr, sw = _csr(rng, [7, 7, 7])
    G = rng.normal(size=(21, 16))
    Wq, Wk, Wv = (rng.normal(0, 0.25, (16, 16)) for _ in range(3))
    smooth = oracle_mod.attention_smooth(row_ptr, sw, G, Wq, Wk, Wv, 4, 7)
    plain = oracle_mod.attention(row_ptr, sw, G, Wq, Wk, Wv, 4)
    assert np.array_equal(smooth, plain)


def test_zero_switch_spreads_over_all_slots(oracle_mod):
    """Every logit 0: each of the nnei_max slots weighs 1 / nnei_max, the
    phantoms carrying zero values, so O_a = sum_b V_b / nnei_max."""
    rng = np.random.default_rng(5)
    row_ptr, _ = _csr(rng, [6, 3])
    G = rng.normal(size=(9, 8))
    Wq, Wk, Wv = (rng.normal(size=(8, 8)) for _ in range(3))
    out = oracle_mod.attention_smooth(row_ptr, np.zeros(9), G, Wq, Wk, Wv, 2, 10)
    V = G @ Wv
    assert np.allclose(out[:6], V[:6].sum(axis=0) / 10, rtol=0, atol=1e-14)
    assert np.allclose(out[6:], V[6:].sum(axis=0) / 10, rtol=0, atol=1e-14)


def test_rows_longer_than_the_cap_are_rejected(oracle_mod):
    rng = np.random.default_rng(6)
    row_ptr, sw = _csr(rng, [5])
    G = rng.normal(size=(5, 4))
    W = np.eye(4)
    with pytest.raises(ValueError):
        oracle_mod.attention_smooth(row_ptr, sw, G, W, W, W, 1, 4)
