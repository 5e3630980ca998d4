"""GPU tests of the device status word: rows longer than an attention call's
nnei_max, and a bounded wait of the one-launch build made to run out.

A destination with more edges than the nnei_max an attention call is given
is skipped by every kernel path (fused tiles, head-group kernel, generic
kernel, slot-occupancy and local attention): its output rows keep their old
contents and MLG_STATUS_ROW_TOO_LONG is raised.  Every other destination is
computed as usual and must match the oracle.
"""
import dataclasses
import functools

import numpy as np
import pytest
import torch

from neighbour_graph_attention_b200 import configs as C

import gpu_util as U

pytestmark = pytest.mark.gpu

KEY = 4          # open protein-like cluster: ragged rows (about 30 to 70 edges)
CALL_NNEI = 50   # the cap given to the attention calls; the CSR is built with 96


@functools.lru_cache(maxsize=None)
def cluster_graph():
    w = C.workload(KEY)
    s = C.system(KEY, 0)
    return U.gpu_build(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)


def _inputs(channels, heads, dtype, seed):
    rng = np.random.default_rng(seed)
    gpu, csr_t = cluster_graph()
    e = gpu["n_edges"]
    G = rng.standard_normal((e, channels))
    W = [rng.standard_normal((channels, channels)) / np.sqrt(channels) for _ in range(3)]
    if dtype == "f32":
        G = G.astype(np.float32).astype(np.float64)
        W = [x.astype(np.float32).astype(np.float64) for x in W]
    return gpu, csr_t, G, W


def _run(fn, csr_t, gpu, channels, dtype, G, W, heads, nnei):
    m = U.mlg()
    dt = torch.float64 if dtype == "f64" else torch.float32
    e = gpu["n_edges"]
    gin = torch.as_tensor(G, dtype=dt, device="cuda")
    gout = torch.full((e, channels), float("nan"), dtype=dt, device="cuda")
    wq, wk, wv = (torch.as_tensor(x, dtype=dt, device="cuda") for x in W)
    csr_t.status.zero_()
    mdt = m.MLG_F64 if dtype == "f64" else m.MLG_F32
    fn(csr_t, gpu["row_ptr"].size - 1, nnei, channels, heads, mdt, gin, gout, wq, wk, wv)
    torch.cuda.synchronize()
    return gout.cpu().numpy().astype(np.float64), int(csr_t.status.item())


# (dtype, channels, heads): the FP64 tensor-core tile, the tcgen05 tiles (c = 32, 64), the
# head-group kernel (c = 128, fp32 and fp64) and the generic kernel (c = 16)
PATHS = [("f64", 32, 4), ("f32", 32, 4), ("f32", 64, 4), ("f32", 128, 8), ("f64", 128, 4),
         ("f64", 16, 2), ("f32", 48, 3)]


@pytest.mark.parametrize("dtype,channels,heads", PATHS)
@pytest.mark.parametrize("smooth", [False, True])
def test_rows_longer_than_nnei_max_are_skipped_and_flagged(dtype, channels, heads, smooth):
    import oracle

    m = U.mlg()
    gpu, csr_t, G, W = _inputs(channels, heads, dtype, 11)
    rp = gpu["row_ptr"]
    n = np.diff(rp)
    assert (n > CALL_NNEI).any() and (n <= CALL_NNEI).any()
    fn = m.mlg_block_attention_smooth if smooth else m.mlg_block_attention
    out, status = _run(fn, csr_t, gpu, channels, dtype, G, W, heads, CALL_NNEI)
    assert status == m.MLG_STATUS_ROW_TOO_LONG
    sw = gpu["sw"] if dtype == "f64" else gpu["sw"].astype(np.float32).astype(np.float64)
    short = np.flatnonzero(n <= CALL_NNEI)
    long_ = np.flatnonzero(n > CALL_NNEI)
    rows_s = np.concatenate([np.arange(rp[i], rp[i + 1]) for i in short])
    rows_l = np.concatenate([np.arange(rp[i], rp[i + 1]) for i in long_])
    assert np.isnan(out[rows_l]).all(), "an over-long row was written"
    sub_rp = np.concatenate([[0], np.cumsum(n[short])])
    if smooth:
        ref = oracle.attention_smooth(sub_rp, sw[rows_s], G[rows_s], *W, heads, CALL_NNEI)
    else:
        ref = oracle.attention(sub_rp, sw[rows_s], G[rows_s], *W, heads)
    w = C.workload(KEY)
    w = dataclasses.replace(w, dtype=dtype)
    ok, err = U.attn_tolerance_ok(w, out[rows_s], ref)
    assert ok, err


@pytest.mark.parametrize("dtype", ["f64", "f32"])
def test_local_attention_row_longer_than_nnei_max(dtype):
    import oracle

    m = U.mlg()
    channels, heads = 32, 4
    gpu, csr_t, G, W = _inputs(channels, heads, dtype, 12)
    rp = gpu["row_ptr"]
    n = np.diff(rp)
    nc = n.size
    rng = np.random.default_rng(13)
    Hc = rng.standard_normal((nc, channels))
    if dtype == "f32":
        Hc = Hc.astype(np.float32).astype(np.float64)
    dt = torch.float64 if dtype == "f64" else torch.float32
    h_t = torch.as_tensor(Hc, dtype=dt, device="cuda")
    g_t = torch.as_tensor(G, dtype=dt, device="cuda")
    out = torch.full((nc, channels), float("nan"), dtype=dt, device="cuda")
    wq, wk, wv = (torch.as_tensor(x, dtype=dt, device="cuda") for x in W)
    csr_t.status.zero_()
    mdt = m.MLG_F64 if dtype == "f64" else m.MLG_F32
    m.mlg_local_attention(csr_t, nc, CALL_NNEI, channels, heads, mdt, h_t, g_t, out, wq, wk, wv)
    torch.cuda.synchronize()
    assert int(csr_t.status.item()) == m.MLG_STATUS_ROW_TOO_LONG
    o = out.cpu().numpy().astype(np.float64)
    long_ = n > CALL_NNEI
    assert np.all(o[long_] == 0.0), "an over-long centre must get a zero row"
    sw = gpu["sw"] if dtype == "f64" else gpu["sw"].astype(np.float32).astype(np.float64)
    ref = oracle.local_attention(rp, sw, Hc, G, *W, heads)
    w = C.workload(KEY)
    w = dataclasses.replace(w, dtype=dtype)
    ok, err = U.attn_tolerance_ok(w, o[~long_], ref[~long_])
    assert ok, err


def test_one_launch_build_wait_runs_out_cleanly():
    """The bounded waits of the one-launch build: with CTA 0 withholding its
    release flag and each wait cut to a few polls, the other CTAs give up,
    the status word carries MLG_STATUS_TIMEOUT, the call returns, and the
    context stays usable (the next build is exact again)."""
    import oracle

    m = U.mlg()
    key = 2  # diamond-512: the one-launch build
    w = C.workload(key)
    s = C.system(key, 0)
    x = torch.as_tensor(s["coords"], device="cuda")
    csr = m.Csr.empty(w.n_atoms, w.n_atoms * w.nnei_max)
    ws = m.workspace(m.mlg_build_csr_workspace_bytes(w.n_atoms, w.rcut, s["box"], s["pbc"]))
    sysd = m.make_system(x, s["box"], s["pbc"])
    for polls in (4, 64):
        m.mlg_build_csr_wait_test(sysd, w.rcut, w.r_on, w.nnei_max, csr, ws, polls)
        torch.cuda.synchronize()
        assert int(csr.status.item()) & m.MLG_STATUS_TIMEOUT
    # the same workspace and context, a normal build: bit-exact again
    m.mlg_build_csr(sysd, w.rcut, w.r_on, w.nnei_max, csr, ws)
    torch.cuda.synchronize()
    got = U.csr_to_numpy(csr)
    assert got["status"] == 0
    ref = oracle.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
    U.assert_csr_equal(got, ref)
