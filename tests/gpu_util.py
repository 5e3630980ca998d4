"""Helpers of the GPU parity tests: run the C ABI on torch CUDA tensors."""
from __future__ import annotations

import numpy as np
import torch

from neighbour_graph_attention_b200 import configs as C


def mlg():
    from neighbour_graph_attention_b200 import build

    build.build()
    from neighbour_graph_attention_b200 import mlg as m

    return m


def gpu_build(coords, box, pbc, rcut, r_on, nnei_max, types=None, n_types=0, capacity=None,
              stream=None, ws=None, device="cuda"):
    """Build the CSR on the GPU; returns numpy arrays trimmed to E rows."""
    m = mlg()
    x = torch.as_tensor(np.ascontiguousarray(coords, dtype=np.float64), device=device)
    t = None if types is None else torch.as_tensor(np.asarray(types, dtype=np.int32),
                                                   device=device)
    n = x.shape[0]
    cap = n * nnei_max if capacity is None else capacity
    csr = m.Csr.empty(n, cap, device=device)
    need = m.mlg_build_csr_workspace_bytes(n, rcut, box, pbc)
    if ws is None:
        ws = m.workspace(need, device=device)
    sysd = m.make_system(x, box, pbc, t, n_types)
    m.mlg_build_csr(sysd, rcut, r_on, nnei_max, csr, ws, stream=stream)
    torch.cuda.synchronize()
    return csr_to_numpy(csr), csr


def csr_to_numpy(csr):
    e = int(csr.n_edges.item())
    k = min(e, csr.capacity)
    return {"row_ptr": csr.row_ptr.cpu().numpy(), "src": csr.src[:k].cpu().numpy(),
            "shift": csr.shift[:k].cpu().numpy(), "vec": csr.vec[:k].cpu().numpy(),
            "dist": csr.dist[:k].cpu().numpy(), "sw": csr.sw[:k].cpu().numpy(),
            "n_edges": e, "n_truncated": int(csr.n_truncated.item()),
            "status": int(csr.status.item())}


def assert_csr_equal(gpu, ref, rows=None):
    """Bit-exact comparison of every CSR array (optionally a prefix of rows)."""
    assert np.array_equal(gpu["row_ptr"], ref["row_ptr"]), "row_ptr"
    for k in ("src", "shift", "vec", "dist", "sw"):
        a, b = gpu[k], ref[k]
        if rows is not None:
            a, b = a[:rows], b[:rows]
        assert a.shape == b.shape, k
        # compare bit patterns, so that -0.0 != 0.0 and NaNs are caught too
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8)), k


def torch_dtype(w):
    return torch.float64 if w.dtype == "f64" else torch.float32


def mlg_dtype(w):
    m = mlg()
    return m.MLG_F64 if w.dtype == "f64" else m.MLG_F32


def attn_tolerance_ok(w, out, ref):
    """FP64: max-abs <= 1e-10. FP32: max-abs <= 2e-5 * max|ref| (per layer), and
    also row by row: each output row's max-abs error <= 2e-5 * max|that row of
    ref| (rows whose own scale is below 1e-6 of the global one are held to
    1e-6 of it), so that a row much smaller than the largest cannot hide a
    large relative error. Returns (ok, worst relative error)."""
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = float(np.max(np.abs(out - ref))) if out.size else 0.0
    if w.dtype == "f64":
        return err <= 1e-10, err
    scale = float(np.max(np.abs(ref))) if ref.size else 1.0
    ok = err <= 2e-5 * scale
    worst = err / max(scale, 1e-300)
    if out.size and out.ndim == 2:
        row_scale = np.maximum(np.max(np.abs(ref), axis=1), 1e-6 * scale)
        row_rel = np.max(np.abs(out - ref), axis=1) / np.maximum(row_scale, 1e-300)
        worst_row = float(np.max(row_rel))
        ok = ok and worst_row <= 2e-5
        worst = max(worst, worst_row)
    return ok, worst


def gpu_attention(csr_t, n_centres, w, G, Wq, Wk, Wv, stream=None):
    m = mlg()
    dt = torch_dtype(w)
    dev = csr_t.row_ptr.device
    gin = torch.zeros((max(csr_t.capacity, 1), w.channels), dtype=dt, device=dev)
    gin[: G.shape[0]] = torch.as_tensor(G, dtype=dt, device=dev)
    gout = torch.zeros_like(gin)
    wq, wk, wv = (torch.as_tensor(np.ascontiguousarray(x), dtype=dt, device=dev)
                  for x in (Wq, Wk, Wv))
    m.mlg_block_attention(csr_t, n_centres, w.nnei_max, w.channels, w.heads, mlg_dtype(w), gin,
                          gout, wq, wk, wv, stream=stream)
    torch.cuda.synchronize()
    return gout[: G.shape[0]].cpu().numpy()


def workload_inputs(key, seed):
    w = C.workload(key)
    return w, C.system(key, seed)
