"""CPU oracle of the neighbour-graph hot path (TEST INFRASTRUCTURE).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library and
its binding) never imports, links or runs anything here, and this package
never imports the product.

The arithmetic lives in ``mlg_oracle.c`` (plain C, fp64, no contraction),
compiled to ``liboracle.so`` beside it. This module only marshals numpy
arrays. Each function names the passage it follows; the C file's header
states the definitions in full:

* neighbour CSR -- deepmd-kit issue "DPA4 .pt2 LAMMPS (C++ AOTI) inference
  3-6x slower than Python (ASE)", Root cause analysis (createEdgeTensors():
  edge index and edge vector per neighbour pair), and issue "NeighborGraph
  attention is 4-9x slower than dense", Proposed fix (destination CSR);
* per-centre cap -- the same issues, Reproduction (sel=181) and Measurements
  (nsel 120 / rcut 6, nsel 40 / rcut 4);
* attention -- NeighborGraph issue, Proposed fix (dense per-centre attention
  with per-row masks) and Root cause (the dense route's per-centre
  (nloc, nnei, nnei) batched products);
* Verlet-list reuse -- DPA4 issue, Proposed optimizations (device tensors
  reused while the neighbour list is unchanged): an uncapped list at
  rcut + skin, re-evaluated at the current coordinates, then capped and
  ordered as the full build.

Parity of the switch cosine, the neighbour set and the attention is pinned by
the ``-m "not gpu"`` tests in ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mlg_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
          "-shared", "-fPIC", "-Wall"]


def build(force: bool = False) -> str:
    """Compile ``mlg_oracle.c`` into ``liboracle.so`` (gcc); with a stand-in
    library named in ``MLG_ORACLE_LIB`` (the mutation tests), return that."""
    alt = os.environ.get("MLG_ORACLE_LIB")
    if alt:
        return alt
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # a deliberately broken copy of this library, compiled by the
            # mutation tests, replaces it when named here (tests only)
            lib = ctypes.CDLL(build())
            i64, i32, dbl = ctypes.c_int64, ctypes.c_int32, ctypes.c_double
            p = ctypes.c_void_p
            lib.oracle_cos_pi.restype = dbl
            lib.oracle_cos_pi.argtypes = [dbl]
            lib.oracle_switch.restype = None
            lib.oracle_switch.argtypes = [i64, p, dbl, dbl, p]
            lib.oracle_count.restype = ctypes.c_int
            lib.oracle_count.argtypes = [i64, p, p, p, dbl, i32, p, p, ctypes.c_int]
            lib.oracle_fill.restype = ctypes.c_int
            lib.oracle_fill.argtypes = [i64, p, p, p, dbl, dbl, i32, p, p, p, p, p, p,
                                        ctypes.c_int]
            lib.oracle_centre.restype = i64
            lib.oracle_centre.argtypes = [i64, p, p, p, dbl, dbl, i32, i64, i64, p, p, p, p,
                                          p, p]
            lib.oracle_attention.restype = ctypes.c_int
            lib.oracle_attention.argtypes = [i64, p, p, i32, i32, p, p, p, p, p, ctypes.c_int]
            lib.oracle_attention_map.restype = ctypes.c_int
            lib.oracle_attention_map.argtypes = [p, p, i32, i32, p, p, p, i64, i32, p]
            lib.oracle_attention_smooth.restype = ctypes.c_int
            lib.oracle_attention_smooth.argtypes = [i64, p, p, i32, i32, i32, p, p, p, p, p,
                                                    ctypes.c_int]
            lib.oracle_refine_count.restype = ctypes.c_int
            lib.oracle_refine_count.argtypes = [i64, p, p, p, dbl, i32, p, p, p, p, p]
            lib.oracle_refine_fill.restype = ctypes.c_int
            lib.oracle_refine_fill.argtypes = [i64, p, p, p, dbl, dbl, i32, p, p, p, p, p, p,
                                               p, p, p]
            lib.oracle_local_attention.restype = ctypes.c_int
            lib.oracle_local_attention.argtypes = [i64, p, p, i32, i32, p, p, p, p, p, p,
                                                   ctypes.c_int]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _geom_args(coords, box, pbc):
    coords = np.ascontiguousarray(coords, dtype=np.float64).reshape(-1, 3)
    box = np.ascontiguousarray(box, dtype=np.float64).reshape(3, 3)
    pbc = np.ascontiguousarray(pbc, dtype=np.uint8).reshape(3)
    return coords, box, pbc


def cos_pi(u: float) -> float:
    """This project's reproducible cos(pi u) (Taylor series of sin)."""
    return _load().oracle_cos_pi(float(u))


def switch(r, rcut: float, r_on: float) -> np.ndarray:
    """Smooth cosine switch s(r): 1 below r_on, 0 at rcut and beyond.

    NeighborGraph issue, Measurements ("graph smooth" / "dense smooth"); the
    onset r_on and the cosine shape follow the benchmark system definitions.
    """
    r = np.ascontiguousarray(r, dtype=np.float64).ravel()
    s = np.empty_like(r)
    _load().oracle_switch(r.size, _ptr(r), float(rcut), float(r_on), _ptr(s))
    return s


def counts(coords, box, pbc, rcut: float, nnei_max: int, nthreads: int = 0):
    """Per-centre kept count min(raw, nnei_max) and raw in-cutoff count."""
    coords, box, pbc = _geom_args(coords, box, pbc)
    n = coords.shape[0]
    kept = np.zeros(n, dtype=np.int32)
    raw = np.zeros(n, dtype=np.int64)
    rc = _load().oracle_count(n, _ptr(coords), _ptr(box), _ptr(pbc), float(rcut),
                              int(nnei_max), _ptr(kept), _ptr(raw), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_count failed ({rc})")
    return kept, raw


def build_csr(coords, box, pbc, rcut: float, r_on: float, nnei_max: int,
              nthreads: int = 0) -> dict:
    """The whole destination-sorted CSR by brute force.

    Returns row_ptr int64 [N+1], src int32 [E], shift int32 [E][3], vec
    float64 [E][3] (source image minus destination), dist float64 [E],
    sw float64 [E], raw int64 [N], n_truncated.
    """
    coords, box, pbc = _geom_args(coords, box, pbc)
    n = coords.shape[0]
    kept, raw = counts(coords, box, pbc, rcut, nnei_max, nthreads)
    row_ptr = np.zeros(n + 1, dtype=np.int64)
    np.cumsum(kept, out=row_ptr[1:])
    e = int(row_ptr[-1])
    src = np.zeros(e, dtype=np.int32)
    shift = np.zeros((e, 3), dtype=np.int32)
    vec = np.zeros((e, 3), dtype=np.float64)
    dist = np.zeros(e, dtype=np.float64)
    sw = np.zeros(e, dtype=np.float64)
    rc = _load().oracle_fill(n, _ptr(coords), _ptr(box), _ptr(pbc), float(rcut), float(r_on),
                             int(nnei_max), _ptr(row_ptr), _ptr(src), _ptr(shift), _ptr(vec),
                             _ptr(dist), _ptr(sw), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_fill failed ({rc})")
    return {"row_ptr": row_ptr, "src": src, "shift": shift, "vec": vec, "dist": dist,
            "sw": sw, "raw": raw, "n_truncated": int(np.count_nonzero(raw > nnei_max))}


def verlet_candidates(coords, box, pbc, rcut: float, skin: float, nthreads: int = 0) -> dict:
    """The candidate list of Verlet reuse: every pair within rcut + skin, with
    no cap (the cap is applied when the list is used).  The CSR dict of
    ``build_csr`` at the larger cutoff."""
    r = float(rcut) + float(skin)
    return build_csr(coords, box, pbc, r, min(float(rcut), r), 1 << 30, nthreads)


def max_displacement(coords, coords_ref) -> float:
    """The largest distance any atom has moved, on the raw (unwrapped)
    coordinates: an atom re-wrapped into the box counts as having moved by a
    box length."""
    d = np.asarray(coords, dtype=np.float64) - np.asarray(coords_ref, dtype=np.float64)
    return float(np.sqrt(np.max(np.sum(d * d, axis=1)))) if d.size else 0.0


def needs_rebuild(coords, coords_ref, skin: float) -> bool:
    """Verlet criterion: the list built at ``coords_ref`` stays complete while
    every atom has moved less than skin / 2."""
    return 2.0 * max_displacement(coords, coords_ref) >= float(skin)


def verlet_refine(cand: dict, coords, box, pbc, rcut: float, r_on: float,
                  nnei_max: int) -> dict:
    """The CSR from a candidate list: every candidate (source, shift)
    re-evaluated at the current coordinates, kept if r < rcut, the cap and
    the canonical order applied as in ``build_csr``.  Equal to ``build_csr``
    at the current coordinates while the Verlet criterion holds."""
    coords, box, pbc = _geom_args(coords, box, pbc)
    n = coords.shape[0]
    cp = np.ascontiguousarray(cand["row_ptr"], dtype=np.int64)
    cs = np.ascontiguousarray(cand["src"], dtype=np.int32)
    ch = np.ascontiguousarray(cand["shift"], dtype=np.int32).reshape(-1, 3)
    if cp.size != n + 1:
        raise ValueError("candidate list and coordinates disagree on the atom count")
    kept = np.zeros(n, dtype=np.int32)
    raw = np.zeros(n, dtype=np.int64)
    lib = _load()
    rc = lib.oracle_refine_count(n, _ptr(coords), _ptr(box), _ptr(pbc), float(rcut),
                                 int(nnei_max), _ptr(cp), _ptr(cs), _ptr(ch), _ptr(kept),
                                 _ptr(raw))
    if rc != 0:
        raise ValueError(f"oracle_refine_count failed ({rc})")
    row_ptr = np.zeros(n + 1, dtype=np.int64)
    np.cumsum(kept, out=row_ptr[1:])
    e = int(row_ptr[-1])
    src = np.zeros(e, dtype=np.int32)
    shift = np.zeros((e, 3), dtype=np.int32)
    vec = np.zeros((e, 3), dtype=np.float64)
    dist = np.zeros(e, dtype=np.float64)
    sw = np.zeros(e, dtype=np.float64)
    rc = lib.oracle_refine_fill(n, _ptr(coords), _ptr(box), _ptr(pbc), float(rcut),
                                float(r_on), int(nnei_max), _ptr(cp), _ptr(cs), _ptr(ch),
                                _ptr(row_ptr), _ptr(src), _ptr(shift), _ptr(vec), _ptr(dist),
                                _ptr(sw))
    if rc != 0:
        raise ValueError(f"oracle_refine_fill failed ({rc})")
    return {"row_ptr": row_ptr, "src": src, "shift": shift, "vec": vec, "dist": dist,
            "sw": sw, "raw": raw, "n_truncated": int(np.count_nonzero(raw > nnei_max))}


def centre(coords, box, pbc, rcut: float, r_on: float, nnei_max: int, i: int) -> dict:
    """The kept edges of one destination ``i`` (brute force over all sources)."""
    coords, box, pbc = _geom_args(coords, box, pbc)
    n = coords.shape[0]
    cap = int(nnei_max)
    src = np.zeros(cap, dtype=np.int32)
    shift = np.zeros((cap, 3), dtype=np.int32)
    vec = np.zeros((cap, 3), dtype=np.float64)
    dist = np.zeros(cap, dtype=np.float64)
    sw = np.zeros(cap, dtype=np.float64)
    raw = np.zeros(1, dtype=np.int64)
    k = _load().oracle_centre(n, _ptr(coords), _ptr(box), _ptr(pbc), float(rcut), float(r_on),
                              int(nnei_max), int(i), cap, _ptr(src), _ptr(shift), _ptr(vec),
                              _ptr(dist), _ptr(sw), _ptr(raw))
    if k < 0:
        raise ValueError(f"oracle_centre failed ({k})")
    return {"src": src[:k], "shift": shift[:k], "vec": vec[:k], "dist": dist[:k],
            "sw": sw[:k], "raw": int(raw[0])}


def _as_f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def attention(row_ptr, sw, G, Wq, Wk, Wv, heads: int, nthreads: int = 0) -> np.ndarray:
    """One block-dense attention layer over every centre of the CSR.

    NeighborGraph issue, Proposed fix: per centre, Q = G Wq, K = G Wk,
    V = G Wv; per head l_ab = s_a s_b (q_a . k_b) / sqrt(d), softmax over the
    centre's real edges, O_a = sum_b P_ab V_b, heads concatenated. Computed in
    fp64 from whatever precision the inputs hold.
    """
    row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int64)
    sw, G = _as_f64(sw), _as_f64(G)
    Wq, Wk, Wv = _as_f64(Wq), _as_f64(Wk), _as_f64(Wv)
    c = G.shape[1]
    out = np.zeros_like(G)
    rc = _load().oracle_attention(row_ptr.size - 1, _ptr(row_ptr), _ptr(sw), c, int(heads),
                                  _ptr(G), _ptr(Wq), _ptr(Wk), _ptr(Wv), _ptr(out),
                                  int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_attention failed ({rc})")
    return out


def attention_smooth(row_ptr, sw, G, Wq, Wk, Wv, heads: int, nnei_max: int,
                     nthreads: int = 0) -> np.ndarray:
    """Slot-occupancy ("smooth") attention (NeighborGraph issue, Numerics note:
    phantom slots counted in an occupancy-dependent denominator; the weights
    factor as w_b = softmax_b * sum_b e_b / D~).

    As ``attention``, plus phi = nnei_max - n phantom slots per centre with
    logit exactly 0 and value 0 -- the dense route's zero-padded slots, left
    unmasked: m = max(max_b l_ab, 0 if phi > 0),
    D~ = sum_b e^(l_ab - m) + phi e^(-m), O_a = sum_b e^(l_ab - m) V_b / D~.
    """
    row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int64)
    sw, G = _as_f64(sw), _as_f64(G)
    Wq, Wk, Wv = _as_f64(Wq), _as_f64(Wk), _as_f64(Wv)
    c = G.shape[1]
    out = np.zeros_like(G)
    rc = _load().oracle_attention_smooth(row_ptr.size - 1, _ptr(row_ptr), _ptr(sw), c,
                                         int(heads), int(nnei_max), _ptr(G), _ptr(Wq), _ptr(Wk),
                                         _ptr(Wv), _ptr(out), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_attention_smooth failed ({rc})")
    return out


def local_attention(row_ptr, sw, H, G, Wq, Wk, Wv, heads: int, nthreads: int = 0) -> np.ndarray:
    """Local attention, one query per centre (NeighborGraph issue, "Graph-native
    alternatives", item 2: LocalAtten with queries = centres, keys = edges).

    q_i = H_i Wq from the centre's own feature row, K = G_i Wk and V = G_i Wv
    from its edges; per head l_b = s_b (q_i . k_b) / sqrt(d), softmax over the
    centre's edges, out_i = sum_b P_b V_b, heads concatenated; a centre
    without edges gets a zero row.  Returns [n_centres][c], computed in fp64.
    """
    row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int64)
    sw, H, G = _as_f64(sw), _as_f64(H), _as_f64(G)
    Wq, Wk, Wv = _as_f64(Wq), _as_f64(Wk), _as_f64(Wv)
    c = H.shape[1]
    n = row_ptr.size - 1
    if H.shape[0] != n:
        raise ValueError("H needs one row per centre")
    out = np.full((n, c), np.nan)   # every row, empty centres too, is the C code's to write
    rc = _load().oracle_local_attention(n, _ptr(row_ptr), _ptr(sw), c, int(heads), _ptr(H),
                                        _ptr(G), _ptr(Wq), _ptr(Wk), _ptr(Wv), _ptr(out),
                                        int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_local_attention failed ({rc})")
    return out


def attention_map(row_ptr, sw, G, Wq, Wk, heads: int, i: int, h: int) -> np.ndarray:
    """Softmax map P[a][b] of centre ``i``, head ``h``."""
    row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int64)
    sw, G, Wq, Wk = _as_f64(sw), _as_f64(G), _as_f64(Wq), _as_f64(Wk)
    n = int(row_ptr[i + 1] - row_ptr[i])
    P = np.zeros((max(n, 0), max(n, 0)), dtype=np.float64)
    rc = _load().oracle_attention_map(_ptr(row_ptr), _ptr(sw), G.shape[1], int(heads), _ptr(G),
                                      _ptr(Wq), _ptr(Wk), int(i), int(h), _ptr(P))
    if rc != 0:
        raise ValueError(f"oracle_attention_map failed ({rc})")
    return P


def forward(row_ptr, sw, G0, W, heads: int, dtype: str = "f64", nthreads: int = 0):
    """Stacked attention layers G^{l+1} = attention(G^l); returns every layer.

    ``W`` is [n_layers][3][c][c]. For fp32 workloads (``dtype == "f32"``) the
    inputs are the fp32-rounded values, s(r) is rounded to fp32 as the fp32
    kernels read it, each layer is computed in fp64 and its output rounded to
    fp32 before it feeds the next layer (the fp32 path stores every layer in
    fp32).
    """
    sw = np.asarray(sw, dtype=np.float64)
    if dtype == "f32":
        sw = sw.astype(np.float32).astype(np.float64)
    outs = []
    g = np.asarray(G0)
    for layer in range(np.asarray(W).shape[0]):
        o = attention(row_ptr, sw, g, W[layer][0], W[layer][1], W[layer][2], heads, nthreads)
        if dtype == "f32":
            o = o.astype(np.float32)
        outs.append(o)
        g = o
    return outs
