"""Randomised pins of the oracle's attention variants against independent
dense formulations (torch, fp64), over seeded shapes: channels and head
counts, ragged and empty rows, switch values including 0 and 1, and feature
scales up to logits in the hundreds.

Each dense formulation is the dense route of the NeighborGraph issue
(Root cause: per-centre (nloc, nnei, nnei) batched products): padded
(nloc, pad, c) blocks with a -inf key mask and torch.softmax for the block
attention; the same blocks without the mask, zero features and zero switch in
the padded slots, for the slot-occupancy attention; one query row per centre
for the local attention.  They share no code with the oracle.
"""
import numpy as np
import pytest

from test_oracle_attention import dense_route
from test_oracle_local import dense_local
from test_oracle_smooth import dense_unmasked

SHAPES = [(4, 1), (8, 2), (16, 4), (24, 3), (32, 4), (48, 6), (64, 8)]


def _case(seed):
    rng = np.random.default_rng([seed, 91])
    c, heads = SHAPES[seed % len(SHAPES)]
    n_loc = int(rng.integers(1, 9))
    counts = rng.integers(0, 31, n_loc)
    counts[rng.integers(n_loc)] = rng.integers(1, 31)        # at least one edge
    row_ptr = np.zeros(n_loc + 1, dtype=np.int64)
    np.cumsum(counts, out=row_ptr[1:])
    e = int(row_ptr[-1])
    sw = rng.uniform(0.0, 1.0, e)
    pick = rng.uniform(size=e)
    sw[pick < 0.3] = 1.0
    sw[pick > 0.9] = 0.0
    scale = float(rng.choice([0.1, 1.0, 4.0, 12.0]))       # 12: logits in the hundreds
    G = rng.normal(0.0, scale, (e, c))
    W = [rng.normal(0.0, 1.0 / np.sqrt(c), (c, c)) for _ in range(3)]
    return row_ptr, sw, G, W, heads, int(counts.max())


def _close(out, ref):
    tol = 1e-12 * max(1.0, float(np.max(np.abs(ref))))
    return float(np.max(np.abs(out - ref))) <= tol if out.size else True


@pytest.mark.parametrize("seed", range(28))
def test_block_attention_random_shapes(oracle_mod, seed):
    row_ptr, sw, G, W, heads, nmax = _case(seed)
    out = oracle_mod.attention(row_ptr, sw, G, *W, heads)
    for pad in (nmax, nmax + 7):
        assert _close(out, dense_route(row_ptr, sw, G, *W, heads, pad))


@pytest.mark.parametrize("seed", range(28))
def test_smooth_attention_random_shapes(oracle_mod, seed):
    row_ptr, sw, G, W, heads, nmax = _case(seed)
    for nnei_max in (nmax, nmax + 9):
        out = oracle_mod.attention_smooth(row_ptr, sw, G, *W, heads, nnei_max)
        assert _close(out, dense_unmasked(row_ptr, sw, G, *W, heads, nnei_max))


@pytest.mark.parametrize("seed", range(28))
def test_local_attention_random_shapes(oracle_mod, seed):
    row_ptr, sw, G, W, heads, nmax = _case(seed)
    rng = np.random.default_rng([seed, 92])
    H = rng.normal(0.0, 1.0, (row_ptr.size - 1, G.shape[1]))
    out = oracle_mod.local_attention(row_ptr, sw, H, G, *W, heads)
    assert _close(out, dense_local(row_ptr, sw, H, G, *W, heads, max(nmax, 1)))
