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


def compare(got, ref, max_tol, mean_tol=None, what=""):
    err = np.abs(np.asarray(got, dtype=np.float64) - np.asarray(ref, dtype=np.float64))
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    mx, mn = float(err.max()), float(err.mean())
    assert mx <= max_tol, f"{what}: max |err| {mx:.3e} > {max_tol:.1e}"
    if mean_tol is not None:
        assert mn <= mean_tol, f"{what}: mean |err| {mn:.3e} > {mean_tol:.1e}"
    return mx, mn


def default_scale(D):
    return 1.0 / math.sqrt(D)
