"""Precision of the split products of the fp32 attention for 32 channels,
modelled in numpy (no GPU): the tcgen05 logits in 3xTF32 and P.V on fp16
m16n8k16 MMAs with P and v split into hi + lo.

The model rounds exactly as the kernel does:
  - TF32 hi = round-to-nearest (ties away) to 10 explicit mantissa bits, lo =
    x - hi; the tensor core reads lo's leading 19 bits; products summed in
    fp32, lo.lo dropped;
  - P = 2^(S - max) in [0, 1]; P_hi = (P + 2^12) - 2^12 in fp32 (a multiple of
    2^-11, exact in fp16), P_lo = fp16(P - P_hi);
  - v scaled by 2^-e (its largest |v| below 2^14), v_hi = fp16(v), v_lo =
    fp16(v - v_hi); O = P_hi v_hi + P_hi v_lo + P_lo v_hi in fp32, unscaled.
Against the exact fp64 result, the error must stay an order of magnitude
inside the 2e-5 relative bar of the fp32 parity tests.
"""
import numpy as np


def _tf32_rna(x):
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = ((b + 0x1000) & 0xFFFFE000).astype(np.uint32)
    return b.view(np.float32)


def _tf32_trunc(x):
    b = np.asarray(x, dtype=np.float32).view(np.uint32) & np.uint32(0xFFFFE000)
    return b.view(np.float32)


def _logits_3xtf32(q, k):
    """S = q . k^T from TF32 hi / lo operands (lo.hi + hi.lo + hi.hi)."""
    q = q.astype(np.float32)
    k = k.astype(np.float32)
    qh, kh = _tf32_rna(q), _tf32_rna(k)
    ql, kl = _tf32_trunc(q - qh), _tf32_trunc(k - kh)
    f = lambda a, b: a.astype(np.float64) @ b.astype(np.float64).T  # exact products
    return (f(ql, kh).astype(np.float32) + f(qh, kl).astype(np.float32)
            + f(qh, kh).astype(np.float32))


def _pv_fp16_split(p, v):
    """O = P.V from fp16 hi / lo of P (the 2^12 trick) and of v (scaled)."""
    p = p.astype(np.float32)
    c = np.float32(4096.0)
    ph = ((p + c) - c).astype(np.float32)
    pl = (p - ph).astype(np.float16).astype(np.float32)
    assert np.array_equal(ph.astype(np.float16).astype(np.float32), ph)  # exact in fp16
    vmax = np.abs(v).max()
    # the largest |v| brought into [2^13, 2^14): small values are scaled up too,
    # so that their lo halves stay normal in fp16
    e = max(int(np.floor(np.log2(vmax))) - 13, -110) if vmax > 0 else 0
    vs = (v * 2.0 ** -e).astype(np.float32)
    vh = vs.astype(np.float16).astype(np.float32)
    vl = (vs - vh).astype(np.float16).astype(np.float32)
    f = lambda a, b: (a.astype(np.float64) @ b.astype(np.float64)).astype(np.float32)
    return (f(ph, vh) + f(ph, vl) + f(pl, vh)).astype(np.float64) * 2.0 ** e


def test_split_products_stay_inside_the_fp32_bar():
    rng = np.random.default_rng(7)
    worst = 0.0
    for scale in (1e-6, 1e-3, 1.0, 3.0):
        for _ in range(20):
            n, d = 64, 8
            g = rng.normal(size=(n, 32)) * scale
            w = rng.normal(0, 1 / np.sqrt(32), size=(3, 32, d))
            sw = rng.uniform(0.2, 1.0, size=n)
            q = (g @ w[0]) * sw[:, None] * (np.log2(np.e) / np.sqrt(d))
            k = (g @ w[1]) * sw[:, None]
            v = g @ w[2]
            s = _logits_3xtf32(q, k).astype(np.float64)
            s_ref = q @ k.T
            p = np.exp2(s - s.max(axis=1, keepdims=True))
            o = _pv_fp16_split(p, v) / p.sum(axis=1, keepdims=True)
            p_ref = np.exp2(s_ref - s_ref.max(axis=1, keepdims=True))
            o_ref = (p_ref @ v) / p_ref.sum(axis=1, keepdims=True)
            rel = np.abs(o - o_ref).max() / np.abs(o_ref).max()
            worst = max(worst, rel)
    assert worst < 2e-6, worst


def test_p_split_is_exact_in_fp16_and_sums_back():
    """P_hi is a multiple of 2^-11 (exact in fp16) and P_hi + P_lo is within
    2^-24 of P over [0, 1] (|P_lo| <= 2^-12, where fp16 steps are at most
    2^-23), including the subnormal range of fp16."""
    p = np.concatenate([np.linspace(0, 1, 20001), 2.0 ** -np.arange(0, 40, 0.25)])
    p = p.astype(np.float32)
    c = np.float32(4096.0)
    ph = ((p + c) - c).astype(np.float32)
    assert np.all(ph * 2048 == np.round(ph * 2048))
    assert np.array_equal(ph.astype(np.float16).astype(np.float32), ph)
    pl = (p - ph).astype(np.float16).astype(np.float64)
    assert np.abs(ph.astype(np.float64) + pl - p.astype(np.float64)).max() <= 2.0 ** -24
