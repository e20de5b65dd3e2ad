"""Float64 CPU oracle for Heavily Compressed Attention (HCA).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, links or runs
this module; only the test suite, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may call it.  It shares no
code, table or helper with the CUDA path.

What it restates (each function cites its passage):

* "280B总参数、14B激活！百度开源文心5.5 Flash Base" (aitest123.com news),
  section 二.1 "Latent-Gated Sparse Attention" -- cited below as [news 二.1]:
  an HCA layer turns every 128 tokens into one cache entry, and attention
  runs only over the compressed entries plus a window made of the most
  recent, still uncompressed tokens.
* "百度 ERNIE 5.5 Flash Base 完整解析" (communeify.com), section "六大核心架構
  創新" item 1 "Hybrid MLA-DSA + HCA 與 VHA" -- cited below as [analysis 1]:
  128 consecutive tokens become a single entry (128x compression); the layer
  attends to all compressed history entries together with a short window of
  recent raw tokens; head dimension 512.
* Both pages, "Low-Rank Gated Attention" paragraph: the attention output is
  multiplied by a learned gate.
* The same communeify.com page, section "33.5T 預訓練資料工程與分散式訓練基礎設施"
  item 3 (the FlashMask-4 attention kernel for the 512-wide HCA heads) -- cited below
  as [analysis infra 3]: the operator has a training backward pass (the page quotes
  its speed-up, not its formulas).

Readings taken where the pages are silent:

* pooling rule = arithmetic mean over the valid tokens of the block;
* window = the last W raw tokens, inclusive of the query itself, causal;
* visible compressed entries = blocks that END before the window starts
  (no overlap with the window; a gap of up to block-1 tokens is allowed);
* the partially filled last block is compressed but never visible;
* one softmax over the union of the two key sets, scale supplied (1/sqrt(512));
* the gate is supplied already passed through the sigmoid; it multiplies O.

Everything is float64 NumPy.  The per-position loop is the definition written
out: for each query position, gather its visible keys, one softmax, one
weighted sum.  All heads of a position are handled by one matmul (a library
primitive); there is no tiling across positions.

``hca_prefill_backward`` restates the gradients of the prefill output (dQ, dK, dV
through both the window and the mean pooling, dG); it is pinned by central finite
differences of the forward, torch autograd of an independent dense formulation and
two reductions to causal attention in ``tests/test_oracle_backward.py``.

Parity status: exact values for random inputs are not printed by the pages
("parity unpinned" in that narrow sense); every function below is pinned by
the invariants, reductions to library routines and brute-force checks in
``tests/test_oracle.py``.
"""

from __future__ import annotations

from typing import Iterable, Optional, Tuple

import numpy as np


# ---------------------------------------------------------------------------
# Visibility (integer, exact)
# ---------------------------------------------------------------------------

def window_bounds(t: int, window: int) -> Tuple[int, int]:
    """Raw window of query position ``t``: tokens [lo, hi], inclusive.

    [news 二.1] / [analysis 1]: the window holds the most
    recent uncompressed tokens.  Reading: the last ``window`` tokens up to and
    including ``t`` (causal), clipped at token 0.
    """
    return max(0, t - window + 1), t


def visible_compressed_count(t: int, block: int, window: int) -> int:
    """Number of compressed entries query position ``t`` may attend to.

    Reading of the same passages: entry j (tokens [j*block, (j+1)*block)) is
    visible iff the whole block ends before the raw window starts, i.e.
    (j+1)*block <= t - window + 1.  Entries are a prefix 0..n-1.
    """
    return max(0, (t + 1 - window) // block)


def compressed_entry_count(T: int, block: int) -> int:
    """Entries a sequence of T tokens produces: one per started block.

    [news 二.1]: every 128 tokens become one cache entry; the
    partial last block also gets an entry (reading), hence ceil(T / block).
    """
    return -(-T // block)


def mask_table(T: int, block: int, window: int) -> np.ndarray:
    """int64 [T, 3] rows (n_c, win_lo, win_hi) for every query position."""
    out = np.zeros((T, 3), dtype=np.int64)
    for t in range(T):
        lo, hi = window_bounds(t, window)
        out[t] = (visible_compressed_count(t, block, window), lo, hi)
    return out


# ---------------------------------------------------------------------------
# Compression (mean pooling of each block)
# ---------------------------------------------------------------------------

def compress_blocks(X: np.ndarray, block: int) -> np.ndarray:
    """Mean-pool each run of ``block`` consecutive tokens into one entry.

    X: [T, H, D] (any float dtype, promoted to float64).  Returns
    [ceil(T/block), H, D] float64.  [news 二.1] / [analysis 1]
    (128 tokens -> one entry); pooling = mean (reading), over the
    tokens actually present in the block.
    """
    X = np.asarray(X, dtype=np.float64)
    T = X.shape[0]
    n = compressed_entry_count(T, block)
    out = np.empty((n,) + X.shape[1:], dtype=np.float64)
    for j in range(n):
        seg = X[j * block: min((j + 1) * block, T)]
        out[j] = seg.sum(axis=0) / seg.shape[0]
    return out


# ---------------------------------------------------------------------------
# Attention for one query position
# ---------------------------------------------------------------------------

def _softmax_weighted(scores: np.ndarray, values: np.ndarray):
    """Row softmax of ``scores`` [H, n] and the weighted sum of ``values`` [n, D].

    Returns (out [H, D], lse [H], weights [H, n]); the max is subtracted
    before exponentiation.
    """
    m = scores.max(axis=1, keepdims=True)
    e = np.exp(scores - m)
    s = e.sum(axis=1, keepdims=True)
    w = e / s
    return w @ values, (m + np.log(s))[:, 0], w


def attend_position(q: np.ndarray, Kc: np.ndarray, Vc: np.ndarray,
                    K: np.ndarray, V: np.ndarray, t: int, block: int,
                    window: int, scale: float, return_weights: bool = False):
    """HCA output of all query heads at position ``t``.

    q: [Hq, D]; Kc, Vc: [n_entries, Hkv, D]; K, V: [>= t+1, Hkv, D] raw tokens
    indexed by absolute position.  Query head h reads KV head
    h * Hkv // Hq.  The key set is the visible compressed entries followed by
    the raw window; one softmax runs over both ([news 二.1],
    [analysis 1]).  Returns (o [Hq, D], lse [Hq]) and optionally the
    softmax weights [Hq, n_keys].
    """
    q = np.asarray(q, dtype=np.float64)
    Hq, D = q.shape
    Hkv = K.shape[1]
    nc = visible_compressed_count(t, block, window)
    lo, hi = window_bounds(t, window)
    if nc > Kc.shape[0]:
        raise ValueError("compressed cache holds fewer entries than visible")
    o = np.empty((Hq, V.shape[2]), dtype=np.float64)
    lse = np.empty((Hq,), dtype=np.float64)
    weights = []
    for g in range(Hkv):
        heads = [h for h in range(Hq) if h * Hkv // Hq == g]
        keys = np.concatenate([np.asarray(Kc[:nc, g], np.float64),
                               np.asarray(K[lo:hi + 1, g], np.float64)], axis=0)
        vals = np.concatenate([np.asarray(Vc[:nc, g], np.float64),
                               np.asarray(V[lo:hi + 1, g], np.float64)], axis=0)
        scores = (q[heads] @ keys.T) * scale
        og, lg, wg = _softmax_weighted(scores, vals)
        o[heads] = og
        lse[heads] = lg
        weights.append((heads, wg))
    if return_weights:
        w = np.empty((Hq, nc + hi - lo + 1), dtype=np.float64)
        for heads, wg in weights:
            w[heads] = wg
        return o, lse, w
    return o, lse


# ---------------------------------------------------------------------------
# Prefill and decode front ends
# ---------------------------------------------------------------------------

def hca_prefill(Q: np.ndarray, K: np.ndarray, V: np.ndarray, block: int,
                window: int, scale: float, gate: Optional[np.ndarray] = None,
                positions: Optional[Iterable[int]] = None):
    """HCA attention of one sequence.

    Q: [T, Hq, D]; K, V: [T, Hkv, D]; gate: [T, Hq, D] already sigmoided
    (low-rank gated attention paragraph of [news 二.1] and [analysis 1]: the
    output is multiplied by a gate) or None.  ``positions`` selects the
    query positions to evaluate (default: all).  Returns (O [P, Hq, D],
    LSE [P, Hq]) in float64 for the selected positions, in order.
    """
    Kc = compress_blocks(K, block)
    Vc = compress_blocks(V, block)
    T = Q.shape[0]
    pos = list(range(T)) if positions is None else [int(p) for p in positions]
    O = np.empty((len(pos), Q.shape[1], V.shape[2]), dtype=np.float64)
    L = np.empty((len(pos), Q.shape[1]), dtype=np.float64)
    for i, t in enumerate(pos):
        o, lse = attend_position(Q[t], Kc, Vc, K, V, t, block, window, scale)
        if gate is not None:
            o = o * np.asarray(gate[t], dtype=np.float64)
        O[i] = o
        L[i] = lse
    return O, L


def hca_decode(q: np.ndarray, Kc: np.ndarray, Vc: np.ndarray,
               ring_k: np.ndarray, ring_v: np.ndarray, ctx_len: int,
               block: int, window: int, scale: float,
               gate: Optional[np.ndarray] = None):
    """One decode step: the new token is position t = ctx_len - 1.

    q: [Hq, D]; Kc, Vc: [>= n_c, Hkv, D] cached entries; ring_k, ring_v:
    [window, Hkv, D] where raw token u sits in slot u % window.  The key set
    is exactly the prefill key set of position t ([news 二.1]).
    Returns (o [Hq, D], lse [Hq]).
    """
    t = ctx_len - 1
    lo, hi = window_bounds(t, window)
    Hkv = ring_k.shape[1]
    D = ring_k.shape[2]
    # Lay the window tokens out at their absolute positions.
    Kw = np.zeros((hi + 1, Hkv, D), dtype=np.float64)
    Vw = np.zeros((hi + 1, Hkv, ring_v.shape[2]), dtype=np.float64)
    for u in range(lo, hi + 1):
        Kw[u] = ring_k[u % window]
        Vw[u] = ring_v[u % window]
    o, lse = attend_position(q, Kc, Vc, Kw, Vw, t, block, window, scale)
    if gate is not None:
        o = o * np.asarray(gate, dtype=np.float64)
    return o, lse


# ---------------------------------------------------------------------------
# Softmax over a key set cut into parts (the split of one sequence's keys over GPUs)
# ---------------------------------------------------------------------------
#
# One softmax over a union of disjoint key sets equals a combination of per-part sums
# taken relative to each part's own maximum: with s_i the scores of part k,
# m_k = max_i s_i, l_k = sum_i exp(s_i - m_k) and o_k = sum_i exp(s_i - m_k) v_i, the
# output over all parts is sum_k exp(m_k - M) o_k / sum_k exp(m_k - M) l_k for any M
# (M = max_k m_k keeps every factor <= 1), and the log-sum-exp is M + log of the
# denominator.  This is the algebra behind splitting a decode's keys ([news 二.1]: the
# keys are the compressed entries plus the window) over several devices.

def attend_part(q: np.ndarray, keys: np.ndarray, vals: np.ndarray, scale: float):
    """Unnormalised softmax sums of all query heads over one part of the keys.

    q: [Hq, D]; keys, vals: [n, D] (one KV head).  Returns (m [Hq], l [Hq], o [Hq, Dv])
    with natural-log m; a part with no keys gives m = -inf, l = 0, o = 0.
    """
    q = np.asarray(q, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    vals = np.asarray(vals, dtype=np.float64)
    Hq = q.shape[0]
    if keys.shape[0] == 0:
        return (np.full(Hq, -np.inf), np.zeros(Hq), np.zeros((Hq, vals.shape[-1])))
    s = (q @ keys.T) * scale
    m = s.max(axis=1)
    e = np.exp(s - m[:, None])
    return m, e.sum(axis=1), e @ vals


def merge_parts(ms, ls, os_):
    """Combine the per-part sums of ``attend_part`` (lists over parts) into the softmax
    output [Hq, Dv] and its log-sum-exp [Hq]; parts with l = 0 hold no key."""
    ms = np.stack([np.asarray(m, np.float64) for m in ms])   # [P, Hq]
    ls = np.stack([np.asarray(x, np.float64) for x in ls])
    os_ = np.stack([np.asarray(o, np.float64) for o in os_])  # [P, Hq, Dv]
    live = ls > 0
    M = np.where(live, ms, -np.inf).max(axis=0)
    w = np.where(live, np.exp(np.where(live, ms, 0.0) - M[None, :]), 0.0)
    L = (w * ls).sum(axis=0)
    O = (w[:, :, None] * os_).sum(axis=0) / L[:, None]
    return O, M + np.log(L)


# ---------------------------------------------------------------------------
# Backward (gradients of the prefill output)
# ---------------------------------------------------------------------------
#
# The pages give the operator and note that it is trained: the attention kernel has a
# backward pass whose speed-up they quote ([analysis infra 3]); they print no backward
# formulas.  The backward here is the derivative of the forward
# definition above, taken step by step: gate, weighted sum, softmax, scores, and the
# mean pooling that made the compressed entries.

def pool_backward(dXc: np.ndarray, T: int, block: int) -> np.ndarray:
    """Gradient of ``compress_blocks`` with respect to its input.

    dXc: [n_entries, H, D] gradient of the entries.  Entry j is the mean of the
    tokens of block j, so each of those tokens receives dXc[j] / count_j.
    Returns [T, H, D].
    """
    dXc = np.asarray(dXc, dtype=np.float64)
    out = np.zeros((T,) + dXc.shape[1:], dtype=np.float64)
    for j in range(dXc.shape[0]):
        a, b = j * block, min((j + 1) * block, T)
        if a < b:
            out[a:b] += dXc[j] / (b - a)
    return out


def _softmax_backward(w: np.ndarray, dw: np.ndarray) -> np.ndarray:
    """Gradient of the scores through a row softmax: w (dw - sum_k w dw)."""
    return w * (dw - (w * dw).sum(axis=1, keepdims=True))


def attend_position_backward(q: np.ndarray, do: np.ndarray, Kc: np.ndarray,
                             Vc: np.ndarray, K: np.ndarray, V: np.ndarray, t: int,
                             block: int, window: int, scale: float):
    """Gradients of the (ungated) output of ``attend_position`` at position ``t``.

    do: [Hq, D] gradient of that output.  Returns (dq [Hq, D], dkey, dval) where
    dkey / dval are lists over KV heads g of arrays [n_c + window length, D]: the
    gradient of every key / value row of that head, visible compressed entries first,
    then the raw window in token order -- the key order of the forward.
    """
    q = np.asarray(q, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    Hq = q.shape[0]
    Hkv = K.shape[1]
    nc = visible_compressed_count(t, block, window)
    lo, hi = window_bounds(t, window)
    dq = np.zeros_like(q)
    dkey, dval = [], []
    for g in range(Hkv):
        heads = [h for h in range(Hq) if h * Hkv // Hq == g]
        keys = np.concatenate([np.asarray(Kc[:nc, g], np.float64),
                               np.asarray(K[lo:hi + 1, g], np.float64)], axis=0)
        vals = np.concatenate([np.asarray(Vc[:nc, g], np.float64),
                               np.asarray(V[lo:hi + 1, g], np.float64)], axis=0)
        scores = (q[heads] @ keys.T) * scale
        _, _, w = _softmax_weighted(scores, vals)
        dw = do[heads] @ vals.T                    # d(out)/d(weights)
        ds = _softmax_backward(w, dw) * scale      # d/d(q.k), scale folded in
        dq[heads] = ds @ keys
        dkey.append(ds.T @ q[heads])               # summed over the heads of group g
        dval.append(w.T @ do[heads])
    return dq, dkey, dval


def hca_prefill_backward(Q: np.ndarray, K: np.ndarray, V: np.ndarray, dO: np.ndarray,
                         block: int, window: int, scale: float,
                         gate: Optional[np.ndarray] = None):
    """Gradients of ``hca_prefill`` (all positions) for an output gradient dO.

    Q, dO: [T, Hq, D]; K, V: [T, Hkv, D]; gate: [T, Hq, D] (already sigmoided) or None.
    Returns (dQ [T, Hq, D], dK [T, Hkv, D], dV [T, Hkv, D], dG [T, Hq, D] or None) in
    float64.  Raw keys and values receive their window gradients directly and, through
    the mean pooling, 1/count of the gradient of the compressed entry of their block.
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    dO = np.asarray(dO, dtype=np.float64)
    T, Hq, _ = Q.shape
    Hkv = K.shape[1]
    Kc = compress_blocks(K, block)
    Vc = compress_blocks(V, block)
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    dKc = np.zeros_like(Kc)
    dVc = np.zeros_like(Vc)
    dG = None if gate is None else np.zeros_like(Q)
    for t in range(T):
        do = dO[t]
        if gate is not None:
            g_t = np.asarray(gate[t], dtype=np.float64)
            o, _ = attend_position(Q[t], Kc, Vc, K, V, t, block, window, scale)
            dG[t] = dO[t] * o                      # O = o * G
            do = dO[t] * g_t
        dq, dkey, dval = attend_position_backward(Q[t], do, Kc, Vc, K, V, t, block,
                                                  window, scale)
        dQ[t] = dq
        nc = visible_compressed_count(t, block, window)
        lo, hi = window_bounds(t, window)
        for g in range(Hkv):
            dKc[:nc, g] += dkey[g][:nc]
            dVc[:nc, g] += dval[g][:nc]
            dK[lo:hi + 1, g] += dkey[g][nc:]
            dV[lo:hi + 1, g] += dval[g][nc:]
    dK += pool_backward(dKc, T, block)
    dV += pool_backward(dVc, T, block)
    return dQ, dK, dV, dG


# ---------------------------------------------------------------------------
# Gate from the low-rank query latent, and the cross-head mixing (VHA)
# ---------------------------------------------------------------------------
#
# [news 二.1], "Low-Rank Gated Attention" paragraph, and [analysis 1], its second bullet:
# the output gate is computed from the attention layer's own low-rank query latent, a
# quarter of the hidden width (4096 / 4 = 1024), instead of from the hidden state; the
# attention output is multiplied by it.  Reading: G = sigmoid(q_lat . W_g), one gate value
# per output element, W_g of shape [latent, heads * head_dim].
# Same paragraphs, "Virtual Head Attention": after the attention computation a light
# cross-head low-rank mixing with an identity skip lets the heads exchange information.
# Reading: per position and output column d, the vector of the heads' outputs o_.d becomes
# o_.d + A (B^T o_.d), A and B of shape [heads, rank]; then the gate multiplies.

def sigmoid(x: np.ndarray) -> np.ndarray:
    """1 / (1 + exp(-x)), float64 (the branch keeps exp from overflowing)."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    e = np.exp(x[~pos])
    out[~pos] = e / (1.0 + e)
    return out


def gate_from_latent(q_lat: np.ndarray, W_g: np.ndarray, hq: int, D: int) -> np.ndarray:
    """G = sigmoid(q_lat . W_g) as [T, hq, D]; q_lat [T, L], W_g [L, hq * D]."""
    z = np.asarray(q_lat, np.float64) @ np.asarray(W_g, np.float64)
    return sigmoid(z).reshape(z.shape[0], hq, D)


def vha_mix(O: np.ndarray, A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """Cross-head low-rank mixing with an identity skip: O [T, hq, D], A and B [hq, r];
    out[t, h] = O[t, h] + sum_r A[h, r] sum_g B[g, r] O[t, g]."""
    O = np.asarray(O, np.float64)
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    Z = np.einsum("gr,tgd->trd", B, O)          # the rank-r "virtual heads"
    return O + np.einsum("hr,trd->thd", A, Z)


def attention_output(O_attn: np.ndarray, G: Optional[np.ndarray] = None,
                     A: Optional[np.ndarray] = None, B: Optional[np.ndarray] = None):
    """The layer's attention output from the heads' attention outputs O_attn [T, hq, D]:
    the VHA mixing (if A, B are given), then the gate (if G is given)."""
    out = np.asarray(O_attn, np.float64)
    if A is not None:
        out = vha_mix(out, A, B)
    if G is not None:
        out = out * np.asarray(G, np.float64)
    return out


def visible_pairs(T: int, block: int, window: int) -> Tuple[int, int]:
    """(compressed, raw) query-key pairs per head for a sequence of T tokens."""
    c = 0
    w = 0
    for t in range(T):
        c += visible_compressed_count(t, block, window)
        lo, hi = window_bounds(t, window)
        w += hi - lo + 1
    return c, w


# ---------------------------------------------------------------------------
# 8-bit compressed cache
# ---------------------------------------------------------------------------
#
# The communeify.com page, section "本地部署與推論實戰指南", item 3, serves the model through
# vLLM with an 8-bit KV cache (`--kv-cache-dtype fp8`) -- cited below as [serve fp8].  The
# pages give no format details.  Readings:
#   * element format: e4m3 as in the OCP 8-bit floating-point specification (the default
#     8-bit cache format of that engine): 1 sign bit, 4 exponent bits with bias 7, 3
#     fraction bits, subnormals when the exponent field is 0, no infinities, and the one
#     pattern with all exponent and fraction bits set is NaN, so the largest finite
#     magnitude is 448;
#   * what is stored in 8 bits: the compressed pools Kc and Vc (the cache that grows with
#     the context); the raw window stays in the model's dtype;
#   * scale granularity: one float32 scale per pool (per tensor), stored value =
#     e4m3(entry / scale), read back as value(code) * scale;
#   * quantisation: the block mean as a float32 (the value the 16-bit cache would round
#     from), divided by the scale in float32, rounded to the nearest e4m3 value with ties
#     to the even code, magnitudes of 448 and above stored as 448 (saturation).

_E4M3_MAX = 448.0


def e4m3_value(codes) -> np.ndarray:
    """Value of each 8-bit e4m3 code (uint8 array), float64; NaN for the NaN codes.

    Field layout from the format definition: bit 7 sign, bits 3-6 exponent e (bias 7),
    bits 0-2 fraction m.  e = 0: m/8 * 2^-6 (subnormal, or zero); e = 15 with m = 7: NaN;
    otherwise (1 + m/8) * 2^(e - 7).
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def _e4m3_positive_table() -> np.ndarray:
    """Values of the non-negative finite codes 0..126, ascending with the code."""
    return e4m3_value(np.arange(127, dtype=np.uint8))


def e4m3_quantize(x) -> np.ndarray:
    """Nearest e4m3 code of each float32 value (ties to the even code), saturating
    magnitudes >= 448 to 448; NaN inputs give the NaN code.  Returns uint8."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    table = _e4m3_positive_table()
    a = np.abs(x)
    neg = np.signbit(x)
    hi = np.clip(np.searchsorted(table, a, side="left"), 1, 126)   # table[hi-1] < a <= table[hi]
    lo = hi - 1
    d_lo = a - table[lo]
    d_hi = table[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a == 0.0, 0, code)
    code = np.where(a >= _E4M3_MAX, 126, code)
    code = code | np.where(neg, 0x80, 0)
    code = np.where(np.isnan(x), 0x7F, code)
    return code.astype(np.uint8)


def e4m3_dequantize(codes, scale: float) -> np.ndarray:
    """Stored value of each code of a pool with per-tensor ``scale``: value(code) * scale,
    float64 ([serve fp8], readings above)."""
    return e4m3_value(codes) * np.float64(np.float32(scale))


def compress_blocks_e4m3(X: np.ndarray, block: int, scale: float) -> np.ndarray:
    """Compressed entries of ``compress_blocks`` stored in 8 bits ([serve fp8]).

    The mean of each block, taken as the float32 nearest to its float64 value, divided
    by ``scale`` in float32, rounded to e4m3 (readings above).  Returns uint8 codes of
    shape [ceil(T/block), H, D].
    """
    mean32 = compress_blocks(X, block).astype(np.float32)
    y = (mean32 / np.float32(scale)).astype(np.float32)
    return e4m3_quantize(y)
