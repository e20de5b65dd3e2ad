"""Pins for the float64 oracle (CPU only).

Each pin checks the oracle against something other than itself: a table
worked out by hand, a set-based brute force, a closed form, or a reduction to
a library routine (torch scaled_dot_product_attention in float64, numpy mean,
scipy logsumexp).  ``test_planted_mistakes_are_caught`` plants plausible
mistakes in the oracle and checks that every one of them fails some pin.
"""

import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from scipy.special import logsumexp

from oracle import hca_oracle as ORC

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# helpers that do not use the oracle
# ---------------------------------------------------------------------------

def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(q, k, v, scale, mask=None, causal=False):
    """torch SDPA in float64. q [L, H, D]; k, v [S, H, D]; mask [L, S] bool."""
    tq = torch.from_numpy(np.ascontiguousarray(q.transpose(1, 0, 2)))[None]
    tk = torch.from_numpy(np.ascontiguousarray(k.transpose(1, 0, 2)))[None]
    tv = torch.from_numpy(np.ascontiguousarray(v.transpose(1, 0, 2)))[None]
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    o = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=m, is_causal=causal,
                                       scale=scale)
    return o[0].numpy().transpose(1, 0, 2)


def _expand_kv(x, hq):
    """[S, Hkv, D] -> [S, Hq, D]; query head h reads KV head h*Hkv//Hq."""
    hkv = x.shape[1]
    idx = [h * hkv // hq for h in range(hq)]
    return x[:, idx]


def _brute_visibility(T, B, W):
    """Set-based visibility: (compressed set, window set) for every t."""
    out = []
    for t in range(T):
        win = {u for u in range(T) if t - W + 1 <= u <= t}
        comp = set()
        for j in range((T + B - 1) // B):
            toks = set(range(j * B, min((j + 1) * B, T)))
            if len(toks) == B and max(toks) < t - W + 1:
                comp.add(j)
        out.append((comp, win))
    return out


# ---------------------------------------------------------------------------
# pins, written as plain functions of the oracle module so that the planted
# mistake test can run them against a patched copy
# ---------------------------------------------------------------------------

def pin_golden_mask(orc):
    rows = []
    with open(os.path.join(GOLDEN, "mask_T10_B4_W3.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            t, nc, lo, hi, _gap = line.split()
            rows.append((int(t), int(nc), int(lo), int(hi)))
    got = orc.mask_table(10, 4, 3)
    for t, nc, lo, hi in rows:
        assert tuple(got[t]) == (nc, lo, hi), (t, tuple(got[t]), (nc, lo, hi))
    assert orc.compressed_entry_count(10, 4) == 3


def pin_brute_visibility(orc):
    for T, B, W in [(10, 4, 3), (37, 5, 7), (64, 8, 8), (50, 16, 3), (20, 1, 4),
                    (30, 4, 40), (300, 128, 128)]:
        brute = _brute_visibility(T, B, W)
        for t in range(T):
            comp, win = brute[t]
            nc = orc.visible_compressed_count(t, B, W)
            lo, hi = orc.window_bounds(t, W)
            assert set(range(nc)) == comp, (T, B, W, t)
            assert set(range(lo, hi + 1)) == win, (T, B, W, t)
            # partition of [0, t]: compressed tokens, gap, window are disjoint
            ctoks = set(range(nc * B))
            assert not (ctoks & win)
            gap = set(range(t + 1)) - ctoks - win
            assert len(gap) < B or nc == 0 and len(gap) < B + W
            if t + 1 >= W + B:
                assert len(gap) < B


def pin_entry_count(orc):
    for T, B in [(1, 128), (127, 128), (128, 128), (129, 128), (1024, 128),
                 (131072, 128), (10, 4), (7, 1)]:
        X = np.zeros((T, 1, 1))
        assert orc.compressed_entry_count(T, B) == math.ceil(T / B)
        if T <= 2000:
            assert orc.compress_blocks(X, B).shape[0] == math.ceil(T / B)


def pin_compress_mean(orc):
    X = _rand((512, 2, 16), 1)
    got = orc.compress_blocks(X, 128)
    ref = X.reshape(4, 128, 2, 16).mean(axis=1)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-13)
    # partial last block: mean over the tokens present
    Y = _rand((300, 1, 8), 2)
    got = orc.compress_blocks(Y, 128)
    np.testing.assert_allclose(got[2], np.mean(Y[256:300], axis=0), rtol=0,
                               atol=1e-13)


def pin_full_window_is_causal(orc):
    # W >= T: no block is ever visible, every query sees tokens 0..t
    for D in (8, 512):
        T, hq = 40, 3
        Q, K, V = _rand((T, hq, D), 3), _rand((T, 1, D), 4), _rand((T, 1, D), 5)
        s = 1.0 / math.sqrt(D)
        O, L = orc.hca_prefill(Q, K, V, block=4, window=T, scale=s)
        ref = _sdpa(Q, _expand_kv(K, hq), _expand_kv(V, hq), s, causal=True)
        np.testing.assert_allclose(O, ref, rtol=1e-10, atol=1e-12)
        # log-sum-exp of the causal scores, by scipy
        for t in (0, 7, T - 1):
            sc = (Q[t] @ K[:t + 1, 0].T) * s
            np.testing.assert_allclose(L[t], logsumexp(sc, axis=1), rtol=1e-12)


def pin_block1_is_full(orc):
    # block = 1: every compressed entry is one raw token, so the union is 0..t
    for D, W in ((8, 3), (512, 5)):
        T, hq = 33, 2
        Q, K, V = _rand((T, hq, D), 6), _rand((T, 1, D), 7), _rand((T, 1, D), 8)
        s = 1.0 / math.sqrt(D)
        O, _ = orc.hca_prefill(Q, K, V, block=1, window=W, scale=s)
        ref = _sdpa(Q, _expand_kv(K, hq), _expand_kv(V, hq), s, causal=True)
        np.testing.assert_allclose(O, ref, rtol=1e-10, atol=1e-12)


def pin_augmented_sdpa(orc):
    # HCA == SDPA over [block means ; raw tokens] with a set-built mask
    for (T, B, W, hq, hkv, D) in [(50, 4, 3, 4, 2, 16), (70, 8, 5, 3, 1, 8),
                                  (300, 128, 128, 2, 1, 32)]:
        Q = _rand((T, hq, D), 9)
        K = _rand((T, hkv, D), 10)
        V = _rand((T, hkv, D), 11)
        nb = (T + B - 1) // B
        means_k = np.stack([K[j * B:min((j + 1) * B, T)].mean(0) for j in range(nb)])
        means_v = np.stack([V[j * B:min((j + 1) * B, T)].mean(0) for j in range(nb)])
        Ka = np.concatenate([means_k, K])
        Va = np.concatenate([means_v, V])
        mask = np.zeros((T, nb + T), dtype=bool)
        for t, (comp, win) in enumerate(_brute_visibility(T, B, W)):
            for j in comp:
                mask[t, j] = True
            for u in win:
                mask[t, nb + u] = True
        s = 1.0 / math.sqrt(D)
        ref = _sdpa(Q, _expand_kv(Ka, hq), _expand_kv(Va, hq), s, mask=mask)
        O, _ = orc.hca_prefill(Q, K, V, block=B, window=W, scale=s)
        np.testing.assert_allclose(O, ref, rtol=1e-10, atol=1e-12)


def pin_constant_v(orc):
    T, hq, D = 60, 2, 16
    Q, K = _rand((T, hq, D), 12) * 3, _rand((T, 1, D), 13) * 3
    c = _rand((1, 1, D), 14)
    V = np.repeat(c, T, axis=0)
    O, _ = orc.hca_prefill(Q, K, V, block=4, window=5, scale=0.25)
    np.testing.assert_allclose(O, np.broadcast_to(c, O.shape), rtol=0, atol=1e-12)
    G = 1.0 / (1.0 + np.exp(-_rand((T, hq, D), 15)))
    Og, _ = orc.hca_prefill(Q, K, V, block=4, window=5, scale=0.25, gate=G)
    np.testing.assert_allclose(Og, c * G, rtol=0, atol=1e-12)


def pin_weights_sum_to_one(orc):
    T, hq, D, B, W = 40, 3, 8, 4, 3
    Q, K, V = _rand((T, hq, D), 16), _rand((T, 1, D), 17), _rand((T, 1, D), 18)
    Kc, Vc = orc.compress_blocks(K, B), orc.compress_blocks(V, B)
    for t in range(T):
        o, lse, w = orc.attend_position(Q[t], Kc, Vc, K, V, t, B, W, 0.3,
                                        return_weights=True)
        np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-13)
        nc = orc.visible_compressed_count(t, B, W)
        lo, hi = orc.window_bounds(t, W)
        assert w.shape[1] == nc + hi - lo + 1


def pin_single_key(orc):
    T, hq, D = 9, 4, 8
    Q, K, V = _rand((T, hq, D), 19), _rand((T, 1, D), 20), _rand((T, 1, D), 21)
    O, L = orc.hca_prefill(Q, K, V, block=4, window=3, scale=0.5, positions=[0])
    np.testing.assert_allclose(O[0], np.broadcast_to(V[0, 0], (hq, D)), rtol=0,
                               atol=1e-14)
    np.testing.assert_allclose(L[0], 0.5 * (Q[0] @ K[0, 0]), rtol=1e-13)


def pin_decode_matches_prefill_row(orc):
    T, hq, D, B, W = 77, 4, 16, 8, 6
    Q, K, V = _rand((T, hq, D), 22), _rand((T, 1, D), 23), _rand((T, 1, D), 24)
    G = 1.0 / (1.0 + np.exp(-_rand((T, hq, D), 25)))
    Kc, Vc = orc.compress_blocks(K, B), orc.compress_blocks(V, B)
    O, L = orc.hca_prefill(Q, K, V, B, W, 0.2, gate=G)
    for t in (0, 3, W - 1, W, 40, T - 1):
        rk = np.zeros((W, 1, D))
        rv = np.zeros((W, 1, D))
        for u in range(max(0, t - W + 1), t + 1):
            rk[u % W] = K[u]
            rv[u % W] = V[u]
        o, lse = orc.hca_decode(Q[t], Kc, Vc, rk, rv, t + 1, B, W, 0.2, gate=G[t])
        np.testing.assert_allclose(o, O[t], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse, L[t], rtol=1e-12)


PINS = [pin_golden_mask, pin_brute_visibility, pin_entry_count, pin_compress_mean,
        pin_full_window_is_causal, pin_block1_is_full, pin_augmented_sdpa,
        pin_constant_v, pin_weights_sum_to_one, pin_single_key,
        pin_decode_matches_prefill_row]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin(ORC)


# ---------------------------------------------------------------------------
# planted mistakes: each must fail at least one pin
# ---------------------------------------------------------------------------

def _mut_nc_plus_one(t, block, window):
    return max(0, (t + 2 - window) // block)


def _mut_nc_overlap(t, block, window):
    return max(0, (t + 1) // block)


def _mut_window_wide(t, window):
    return max(0, t - window), t


def _mut_compress_sum(X, block):
    X = np.asarray(X, dtype=np.float64)
    n = -(-X.shape[0] // block)
    return np.stack([X[j * block:(j + 1) * block].sum(0) for j in range(n)])


def _mut_compress_first(X, block):
    X = np.asarray(X, dtype=np.float64)
    n = -(-X.shape[0] // block)
    return np.stack([X[j * block] for j in range(n)])


def _mut_compress_divide_by_block(X, block):
    X = np.asarray(X, dtype=np.float64)
    n = -(-X.shape[0] // block)
    return np.stack([X[j * block:(j + 1) * block].sum(0) / block for j in range(n)])


MUTANTS = {
    "nc_plus_one": ("visible_compressed_count", _mut_nc_plus_one),
    "nc_overlap": ("visible_compressed_count", _mut_nc_overlap),
    "window_wide": ("window_bounds", _mut_window_wide),
    "compress_sum": ("compress_blocks", _mut_compress_sum),
    "compress_first": ("compress_blocks", _mut_compress_first),
    "compress_div_block": ("compress_blocks", _mut_compress_divide_by_block),
}


def _mutant_attend(kind):
    real = ORC.attend_position

    def attend(q, Kc, Vc, K, V, t, block, window, scale, return_weights=False):
        if kind == "no_scale":
            scale = 1.0
        if kind == "kv_head_mod":
            # wrong GQA mapping: query head h reads KV head h % Hkv
            Hq, Hkv = q.shape[0], K.shape[1]
            perm = [h * Hkv // Hq for h in range(Hq)]
            wrong = [h % Hkv for h in range(Hq)]
            if perm != wrong:
                order = np.argsort(np.array(wrong), kind="stable")
                inv = np.argsort(order)
                q = q[order]
                res = real(q, Kc, Vc, K, V, t, block, window, scale, return_weights)
                return tuple(r[inv] for r in res)
        if kind == "transposed_values":
            Kc, Vc, K, V = Kc, Kc, K, K
        return real(q, Kc, Vc, K, V, t, block, window, scale, return_weights)
    return attend


def _mutant_prefill_no_gate():
    real = ORC.hca_prefill

    def prefill(Q, K, V, block, window, scale, gate=None, positions=None):
        return real(Q, K, V, block, window, scale, None, positions)
    return prefill


ALL_MUTANTS = sorted(MUTANTS) + ["no_scale", "kv_head_mod", "transposed_values",
                                 "no_gate"]


@pytest.mark.parametrize("name", ALL_MUTANTS)
def test_planted_mistakes_are_caught(name, monkeypatch):
    if name in MUTANTS:
        attr, fn = MUTANTS[name]
        monkeypatch.setattr(ORC, attr, fn)
    elif name == "no_gate":
        monkeypatch.setattr(ORC, "hca_prefill", _mutant_prefill_no_gate())
    else:
        monkeypatch.setattr(ORC, "attend_position", _mutant_attend(name))
    failed = []
    for pin in PINS:
        try:
            pin(ORC)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"planted mistake {name!r} passed every pin"


# ------------------------------------------------------------------ visible pair counts
def _pairs_by_enumeration(T, block, window):
    """Count (t, key) pairs straight from the visibility rule, with no helper of the
    oracle: entry j is visible to t iff (j + 1) * block <= t + 1 - window; raw token u
    iff t - window < u <= t."""
    c = sum(1 for t in range(T) for j in range(T) if (j + 1) * block <= t + 1 - window)
    w = sum(1 for t in range(T) for u in range(T) if t - window < u <= t)
    return c, w


@pytest.mark.parametrize("T,block,window", [(10, 4, 3), (1, 4, 3), (37, 5, 7), (64, 1, 5),
                                            (50, 8, 64), (200, 16, 40)])
def test_visible_pairs_by_enumeration(T, block, window):
    assert ORC.visible_pairs(T, block, window) == _pairs_by_enumeration(T, block, window)


def test_visible_pairs_hand_table():
    # the T=10, block=4, window=3 table: n_c = 1 at t = 6..9, windows of 1, 2, then 3 keys
    assert ORC.visible_pairs(10, 4, 3) == (4, 1 + 2 + 3 * 8)


def test_bench_pair_count_matches_oracle():
    """bench.py reports FLOPs from its own closed-form pair count; it must agree with the
    oracle's count (pinned above) at the workload shapes' block and window."""
    import bench
    for T in (1, 127, 128, 129, 255, 256, 1000, 4097):
        assert bench.visible_pairs(T) == ORC.visible_pairs(T, 128, 128)


# ------------------------------------------------------------------ softmax over key parts
@pytest.mark.parametrize("cuts", [[0, 40], [0, 13, 40], [0, 1, 2, 39, 40], [0, 0, 20, 20, 40]])
def test_merge_of_parts_is_one_softmax(cuts):
    """Cutting the keys into parts (empty parts included) and merging the per-part sums
    gives scipy's softmax over all keys applied to the values, and scipy's logsumexp."""
    from scipy.special import softmax
    rng = np.random.default_rng(5)
    q = rng.standard_normal((6, 16))
    keys = 3.0 * rng.standard_normal((40, 16))
    vals = rng.standard_normal((40, 9))
    scale = 0.25
    parts = [ORC.attend_part(q, keys[a:b], vals[a:b], scale) for a, b in zip(cuts, cuts[1:])]
    O, lse = ORC.merge_parts(*zip(*parts))
    s = (q @ keys.T) * scale
    assert np.allclose(O, softmax(s, axis=1) @ vals, rtol=0, atol=1e-12)
    assert np.allclose(lse, logsumexp(s, axis=1), rtol=0, atol=1e-12)


def test_single_part_matches_attend_position():
    """One part holding a position's whole key set reproduces attend_position."""
    rng = np.random.default_rng(6)
    T, B, W, D = 300, 16, 40, 8
    K = rng.standard_normal((T, 1, D))
    V = rng.standard_normal((T, 1, D))
    q = rng.standard_normal((3, D))
    Kc, Vc = ORC.compress_blocks(K, B), ORC.compress_blocks(V, B)
    t = 250
    nc = ORC.visible_compressed_count(t, B, W)
    keys = np.concatenate([Kc[:nc, 0], K[t - W + 1:t + 1, 0]])
    vals = np.concatenate([Vc[:nc, 0], V[t - W + 1:t + 1, 0]])
    O, lse = ORC.merge_parts(*zip(ORC.attend_part(q, keys, vals, 0.3)))
    ref, rl = ORC.attend_position(q, Kc, Vc, K, V, t, B, W, 0.3)
    assert np.allclose(O, ref, atol=1e-12) and np.allclose(lse, rl, atol=1e-12)


# ------------------------------------------------------------------ gate from latent, VHA
def test_sigmoid_values_and_symmetry():
    x = np.array([-800.0, -3.0, 0.0, 2.5, 800.0])
    s = ORC.sigmoid(x)
    assert s[2] == 0.5 and s[0] == 0.0 and s[-1] == 1.0
    assert abs(s[1] - 1.0 / (1.0 + math.e ** 3.0)) < 1e-15
    y = np.linspace(-30, 30, 121)
    assert np.allclose(ORC.sigmoid(y) + ORC.sigmoid(-y), 1.0, atol=1e-15)


def test_gate_from_latent_by_loops():
    """Each gate value is sigmoid of one dot product of the latent with a column of W_g,
    laid out head-major: G[t, h, d] uses column h * D + d."""
    rng = np.random.default_rng(11)
    T, L, hq, D = 3, 5, 2, 4
    q = rng.standard_normal((T, L))
    W = rng.standard_normal((L, hq * D))
    G = ORC.gate_from_latent(q, W, hq, D)
    for t in range(T):
        for h in range(hq):
            for d in range(D):
                z = sum(q[t, i] * W[i, h * D + d] for i in range(L))
                assert abs(G[t, h, d] - 1.0 / (1.0 + math.exp(-z))) < 1e-14
    assert np.all(ORC.gate_from_latent(q, np.zeros_like(W), hq, D) == 0.5)


def test_vha_mix_special_cases():
    rng = np.random.default_rng(12)
    T, hq, D, r = 4, 5, 3, 2
    O = rng.standard_normal((T, hq, D))
    # no mixing: the identity skip alone
    assert np.array_equal(ORC.vha_mix(O, np.zeros((hq, r)), rng.standard_normal((hq, r))), O)
    # rank one, A = e_i, B = e_j: head i gains head j's output, the others are unchanged
    A = np.zeros((hq, 1)); A[1, 0] = 1.0
    B = np.zeros((hq, 1)); B[3, 0] = 1.0
    out = ORC.vha_mix(O, A, B)
    want = O.copy(); want[:, 1] += O[:, 3]
    assert np.allclose(out, want, atol=1e-15)
    # equals the explicit [hq, hq] matrix I + A B^T applied across heads, by loops
    A, B = rng.standard_normal((hq, r)), rng.standard_normal((hq, r))
    out = ORC.vha_mix(O, A, B)
    M = [[(1.0 if h == g else 0.0) + sum(A[h, k] * B[g, k] for k in range(r))
          for g in range(hq)] for h in range(hq)]
    for t in range(T):
        for h in range(hq):
            for d in range(D):
                assert abs(out[t, h, d] - sum(M[h][g] * O[t, g, d] for g in range(hq))) < 1e-12


def test_attention_output_order():
    """The mixing runs on the ungated outputs and the gate multiplies after it."""
    rng = np.random.default_rng(13)
    O = rng.standard_normal((2, 3, 4))
    G = rng.uniform(0.1, 0.9, (2, 3, 4))
    A, B = rng.standard_normal((3, 2)), rng.standard_normal((3, 2))
    out = ORC.attention_output(O, G, A, B)
    assert np.allclose(out, ORC.vha_mix(O, A, B) * G, atol=1e-15)
    assert not np.allclose(out, ORC.vha_mix(O * G, A, B))
