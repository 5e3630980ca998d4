"""B200-native neighbour-graph construction and block-dense neighbour attention.

The compute path is the C-ABI library ``libmlg.so`` (hand-written CUDA for
sm_100a); :mod:`neighbour_graph_attention_b200.mlg` is its thin ctypes
binding. :mod:`neighbour_graph_attention_b200.configs` draws the seeded
synthetic workloads.
"""

__all__ = ["configs", "mlg"]
