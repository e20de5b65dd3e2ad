"""Shared plumbing for the GPU parity tests (no HCA arithmetic here)."""

import math

import numpy as np
import torch

from compressed_long_context_hca_b200 import binding as B
from compressed_long_context_hca_b200 import build as build_mod
from compressed_long_context_hca_b200 import inputs, ops

# Tolerances: bf16 inputs -> max |err| <= 1e-2 and mean |err| <= 1e-3; f32 inputs ->
# max |err| <= 1e-5 (both against the float64 oracle).
BF16_MAX, BF16_MEAN, F32_MAX = 1e-2, 1e-3, 1e-5


def ensure_built():
    build_mod.build()
    B.lib()


def to64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def run_prefill(x, block=128, window=128, dtype="bf16", page_entries=128, shuffle_pages=True,
                want_lse=False, want_mask=False, scale=None):
    """Compress + prefill on the GPU for PrefillInputs x (CPU tensors). Returns dict."""
    ensure_built()
    dev = torch.device("cuda")
    Q, K, V = (t.to(dev) for t in (x.Q, x.K, x.V))
    G = x.G.to(dev) if x.G is not None else None
    b, T, hq, D = Q.shape
    desc = ops.desc_for_prefill(Q, K, block, window, scale)
    ops.attach_gate(desc, G)
    n_ent = -(-T // block)
    max_pages = max(1, -(-n_ent // page_entries))
    pt = (inputs.page_table(b, max_pages) if shuffle_pages else
          torch.arange(b * max_pages, dtype=torch.int32).view(b, max_pages))
    cache = B.PagedCache(b, n_ent, K.shape[2], D, Q.dtype, page_entries, page_table=pt,
                         device=dev)
    ops.compress(desc, K, V, cache)
    O, lse, dbg = ops.prefill(desc, Q, K, V, cache, want_lse=want_lse, want_mask=want_mask)
    torch.cuda.synchronize()
    return dict(O=O, lse=lse, dbg=dbg, cache=cache, desc=desc)


def bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


def compare(got, ref, max_tol, mean_tol=None, what="", out_bf16=None):
    """Element-wise comparison against the oracle.

    For bf16 outputs (``mean_tol`` given, i.e. the bf16 tolerance) the bound on each
    element is max(max_tol, one bf16 ulp of the reference): a result stored in bf16
    cannot be closer than half an ulp, and past |x| = 2 one ulp exceeds 1e-2. The mean
    bound adds the expected size of one round-to-nearest step (ulp / 4). For |x| < 2
    (all N(0,1) workloads) both reduce to the plain max_tol / mean_tol."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bf16 = mean_tol is not None if out_bf16 is None else out_bf16
    if bf16:
        ulp = bf16_ulp(ref)
        bound = np.maximum(max_tol, ulp)
        mean_bound = (None if mean_tol is None else
                      mean_tol + float((ulp * (np.abs(ref) >= 2.0)).mean()) / 4)
    else:
        bound = np.full_like(err, max_tol)
        mean_bound = mean_tol
    worst = int(np.argmax(err / bound))
    mx, mn = float(err.max()), float(err.mean())
    assert err.flat[worst] <= bound.flat[worst], (
        f"{what}: |err| {err.flat[worst]:.3e} > bound {bound.flat[worst]:.1e} at ref "
        f"{ref.flat[worst]:.4f} (max |err| {mx:.3e}, mean {mn:.3e})")
    if mean_bound is not None:
        assert mn <= mean_bound, f"{what}: mean |err| {mn:.3e} > {mean_bound:.1e}"
    return mx, mn


def p_rounding_bound(x, bi, positions, block=128, window=128):
    """Per-element error bound for bf16 outputs when the softmax is very peaked.

    P is rounded to bf16 before P.V (relative error <= 2^-9 per weight). With weights
    w_i summing to 1 this moves o by sum_i w_i d_i (v_i - o), so
    |err| <= 2^-9 * max_i |v_i - o| <= 2^-9 * (max_i v_i - min_i v_i) over the visible
    values, plus the output rounding (one ulp covers it). Returns the spread
    (max - min of the visible values) per [position, head, dim]; the gate (<= 1) can
    only shrink the error. Built from the set-based visibility, not from the oracle."""
    V = to64(x.V[bi])            # [T, hkv, D]
    T = V.shape[0]
    nb = -(-T // block)
    means = np.stack([V[j * block:min((j + 1) * block, T)].mean(0) for j in range(nb)])
    hq = x.Q.shape[2]
    out = np.empty((len(positions), hq, V.shape[-1]))
    for i, t in enumerate(positions):
        nc = max(0, (t + 1 - window) // block)
        lo = max(0, t - window + 1)
        vals = np.concatenate([means[:nc, 0], V[lo:t + 1, 0]], axis=0)
        out[i] = (vals.max(0) - vals.min(0))[None, :]
    return out


def compare_peaked(got, ref, spread, what=""):
    """bf16 comparison for workloads whose softmax can be dominated by a few keys (the
    every-4th-block x4 inputs): bound = max(1e-2, 2^-9 * spread + ulp(ref)) per element,
    mean bound 1e-3 + 2^-9 * mean(spread) / 4."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bound = np.maximum(BF16_MAX, 2.0 ** -9 * spread + bf16_ulp(ref))
    worst = int(np.argmax(err / bound))
    assert err.flat[worst] <= bound.flat[worst], (
        f"{what}: |err| {err.flat[worst]:.3e} > bound {bound.flat[worst]:.2e} "
        f"(spread {spread.flat[worst]:.2f}, ref {ref.flat[worst]:.3f})")
    mean_bound = BF16_MEAN + 2.0 ** -9 * float(spread.mean()) / 4
    assert err.mean() <= mean_bound, f"{what}: mean |err| {err.mean():.3e} > {mean_bound:.2e}"
    return float(err.max()), float(err.mean())


def default_scale(D):
    return 1.0 / math.sqrt(D)
