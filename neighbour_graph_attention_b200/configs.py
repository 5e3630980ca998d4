"""Seeded synthetic workloads for the neighbour-graph hot path.

This module only draws inputs: atom positions, box, periodicity, atom types,
attention weights and edge features. It contains none of the method's
arithmetic (no neighbour search, no switch, no attention), so both the CUDA
path and the CPU oracle can take their inputs from here without sharing any
computation.

The five workloads restate the five benchmark systems of the neighbour-graph
attention issue ("NeighborGraph attention is 4-9x slower than dense and
OOM-prone", Measurements table: diamond a = 3.567 A, repinit nsel 120 / rcut 6,
repformer nsel 40 / rcut 4, g1 = 128, g2 = 32, 4 heads), of the DPA4 LAMMPS
issue (Fe BCC, sel = 181, 65,536 atoms) and of the mlipaudit "Inference Speed"
page (protein chains up to 5,964 atoms, Dataset section).

Recipe (all draws from ``numpy.random.default_rng``; independent streams so
that the draw order of one input never shifts another):

* positions: ideal lattice sites in C order of (cell x, cell y, cell z, basis),
  plus N(0, jitter^2) per component from stream ``[seed, 0]``, then wrapped
  into [0, L) on periodic axes. The protein-like cluster instead uses random
  sequential placement in a ball (see :func:`_protein_cluster`).
* weights: per layer Wq, Wk, Wv ~ N(0, 1/c), shape [c][c] (y = x W), drawn in
  that order from stream ``[seed, 1]``.
* edge features: G ~ N(0, 1), shape [E][c] in canonical CSR order, from stream
  ``[seed, 2]``; E is the edge count of the built graph.
* fp32 workloads draw in fp64 and round once to fp32.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

__all__ = ["Workload", "WORKLOADS", "workload", "system", "weights", "features"]


@dataclass(frozen=True)
class Workload:
    """One synthetic system plus its attention shape."""

    key: int            # 1-based index, as numbered in the benchmark list
    name: str
    lattice: str        # "diamond", "bcc" or "cluster"
    a: float            # lattice constant (A); unused for the cluster
    cells: int          # conventional cells per axis (periodic lattices)
    jitter: float       # std of the Gaussian position jitter (A)
    n_atoms: int
    rcut: float
    r_on: float
    nnei_max: int
    channels: int
    heads: int
    n_layers: int
    dtype: str          # "f64" or "f32"

    @property
    def periodic(self) -> bool:
        return self.lattice != "cluster"

    @property
    def head_dim(self) -> int:
        return self.channels // self.heads

    @property
    def np_dtype(self):
        return np.float64 if self.dtype == "f64" else np.float32


# r_on: the first system states a cosine switch from 5.5 to 6 A; the others
# state no onset, so all use r_on = rcut - 0.5 A.
WORKLOADS = {
    1: Workload(1, "diamond-64", "diamond", 3.567, 2, 0.05, 64, 6.0, 5.5, 120, 128, 4, 1, "f64"),
    2: Workload(2, "diamond-512", "diamond", 3.567, 4, 0.05, 512, 4.0, 3.5, 40, 32, 4, 6, "f64"),
    3: Workload(3, "fe-bcc-65536", "bcc", 2.855, 32, 0.03, 65536, 6.0, 5.5, 181, 64, 4, 1, "f32"),
    4: Workload(4, "protein-cluster-5964", "cluster", 0.0, 0, 0.0, 5964, 5.0, 4.5, 96, 128, 8, 2, "f32"),
    5: Workload(5, "fe-bcc-524288", "bcc", 2.855, 64, 0.03, 524288, 6.0, 5.5, 128, 32, 4, 1, "f32"),
}


def workload(key: int) -> Workload:
    return WORKLOADS[int(key)]


_BASIS = {
    # fractional sites of the conventional cubic cell
    "diamond": np.array(
        [[0.0, 0.0, 0.0], [0.0, 0.5, 0.5], [0.5, 0.0, 0.5], [0.5, 0.5, 0.0],
         [0.25, 0.25, 0.25], [0.25, 0.75, 0.75], [0.75, 0.25, 0.75], [0.75, 0.75, 0.25]]),
    "bcc": np.array([[0.0, 0.0, 0.0], [0.5, 0.5, 0.5]]),
    "sc": np.array([[0.0, 0.0, 0.0]]),
    "fcc": np.array([[0.0, 0.0, 0.0], [0.0, 0.5, 0.5], [0.5, 0.0, 0.5], [0.5, 0.5, 0.0]]),
}


def lattice_sites(kind: str, a: float, cells) -> np.ndarray:
    """Ideal sites of a cubic lattice, C order over (cx, cy, cz, basis)."""
    if np.isscalar(cells):
        cells = (int(cells),) * 3
    basis = _BASIS[kind]
    grid = np.stack(np.meshgrid(np.arange(cells[0]), np.arange(cells[1]),
                                np.arange(cells[2]), indexing="ij"), axis=-1).reshape(-1, 3)
    sites = (grid[:, None, :].astype(np.float64) + basis[None, :, :]) * a
    return sites.reshape(-1, 3)


def _protein_cluster(n: int, rng: np.random.Generator, density: float = 0.1,
                     min_sep: float = 1.0) -> np.ndarray:
    """Random sequential placement of ``n`` points in a ball.

    The ball radius R = (3n / (4 pi density))^(1/3) gives the stated number
    density (24.24 A for 5,964 atoms at 0.1 / A^3). Candidates are uniform in
    the ball; one is rejected if an accepted point lies within ``min_sep``.
    """
    radius = (3.0 * n / (4.0 * np.pi * density)) ** (1.0 / 3.0)
    cell = min_sep
    grid: dict = {}
    out = np.empty((n, 3))
    count = 0
    sep2 = min_sep * min_sep
    while count < n:
        batch = rng.uniform(-radius, radius, size=(4096, 3))
        batch = batch[np.einsum("ij,ij->i", batch, batch) <= radius * radius]
        for p in batch:
            key = tuple(np.floor(p / cell).astype(np.int64))
            ok = True
            for dx in (-1, 0, 1):
                for dy in (-1, 0, 1):
                    for dz in (-1, 0, 1):
                        for q in grid.get((key[0] + dx, key[1] + dy, key[2] + dz), ()):
                            d = p - q
                            if d[0] * d[0] + d[1] * d[1] + d[2] * d[2] < sep2:
                                ok = False
                                break
                        if not ok:
                            break
                    if not ok:
                        break
                if not ok:
                    break
            if ok:
                grid.setdefault(key, []).append(p)
                out[count] = p
                count += 1
                if count == n:
                    break
    return out


def system(key: int, seed: int = 0) -> dict:
    """Atom positions, box, periodicity and types of workload ``key``.

    Returns ``coords`` float64 [N][3], ``box`` float64 [3][3] (rows a1, a2,
    a3), ``pbc`` uint8 [3], ``types`` int32 [N], ``n_types``.
    """
    w = workload(key)
    rng = np.random.default_rng([seed, 0])
    if w.periodic:
        sites = lattice_sites(w.lattice, w.a, w.cells)
        assert sites.shape[0] == w.n_atoms
        length = w.a * w.cells
        coords = sites + rng.normal(0.0, w.jitter, size=sites.shape)
        coords = np.mod(coords, length)
        box = np.diag([length] * 3).astype(np.float64)
        pbc = np.ones(3, dtype=np.uint8)
        types = np.zeros(w.n_atoms, dtype=np.int32)
        n_types = 1
    else:
        coords = _protein_cluster(w.n_atoms, rng)
        box = np.zeros((3, 3), dtype=np.float64)
        pbc = np.zeros(3, dtype=np.uint8)
        # H / C / N / O at fractions 0.50 / 0.32 / 0.09 / 0.09, exact counts
        counts = [int(round(0.50 * w.n_atoms)), int(round(0.32 * w.n_atoms)),
                  int(round(0.09 * w.n_atoms))]
        counts.append(w.n_atoms - sum(counts))
        types = np.repeat(np.arange(4, dtype=np.int32), counts)
        types = types[rng.permutation(w.n_atoms)].astype(np.int32)
        n_types = 4
    return {"coords": np.ascontiguousarray(coords, dtype=np.float64), "box": box,
            "pbc": pbc, "types": types, "n_types": n_types}


def weights(key: int, seed: int = 0) -> np.ndarray:
    """Per-layer projection weights, shape [n_layers][3][c][c] (q, k, v)."""
    w = workload(key)
    rng = np.random.default_rng([seed, 1])
    c = w.channels
    out = np.empty((w.n_layers, 3, c, c), dtype=np.float64)
    for layer in range(w.n_layers):
        for m in range(3):
            out[layer, m] = rng.normal(0.0, 1.0 / np.sqrt(c), size=(c, c))
    return out.astype(w.np_dtype)


def features(key: int, seed: int, n_edges: int) -> np.ndarray:
    """Edge features G0 ~ N(0, 1), shape [E][c], in canonical CSR order."""
    w = workload(key)
    rng = np.random.default_rng([seed, 2])
    return rng.normal(0.0, 1.0, size=(int(n_edges), w.channels)).astype(w.np_dtype)
