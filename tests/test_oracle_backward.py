"""Pins for the oracle's backward, ``hca_prefill_backward`` (CPU only).

Each pin checks the gradients against something other than the backward's own
formulas: central finite differences of the forward oracle (pinned on its own in
test_oracle.py), torch autograd of an independent dense formulation (block means
by a padded reshape, a set-built visibility mask, one masked softmax), and two
reductions to causal attention whose gradients torch computes.
``test_planted_backward_mistakes`` plants plausible mistakes in the oracle and
checks that each one fails some pin.
"""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import hca_oracle as ORC
from tests.test_oracle import _brute_visibility


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _case(T, Hq, Hkv, D, seed, gate=True):
    Q = _rand((T, Hq, D), seed)
    K = _rand((T, Hkv, D), seed + 1)
    V = _rand((T, Hkv, D), seed + 2)
    dO = _rand((T, Hq, D), seed + 3)
    G = 1.0 / (1.0 + np.exp(-_rand((T, Hq, D), seed + 4))) if gate else None
    return Q, K, V, dO, G


def _torch_grads(fn, Q, K, V, G, dO):
    """Gradients of sum(fn(Q, K, V, G) * dO) by torch autograd, float64."""
    tQ, tK, tV = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (Q, K, V))
    tG = None if G is None else torch.tensor(G, dtype=torch.float64, requires_grad=True)
    O = fn(tQ, tK, tV, tG)
    (O * torch.tensor(dO, dtype=torch.float64)).sum().backward()
    return (tQ.grad.numpy(), tK.grad.numpy(), tV.grad.numpy(),
            None if tG is None else tG.grad.numpy())


def _dense_hca(tQ, tK, tV, tG, block, window, scale):
    """HCA as one masked softmax over [block means ; raw tokens], all in torch.

    Block means by a zero-padded reshape divided by the token count of each block;
    the mask from the set-based visibility of test_oracle; query head h reads KV head
    h * Hkv // Hq."""
    T, Hq, D = tQ.shape
    Hkv = tK.shape[1]
    n = -(-T // block)
    pad = n * block - T
    counts = torch.tensor([min(block, T - j * block) for j in range(n)], dtype=torch.float64)

    def means(X):
        Xp = torch.cat([X, X.new_zeros((pad, Hkv, X.shape[2]))], dim=0)
        return Xp.view(n, block, Hkv, X.shape[2]).sum(1) / counts[:, None, None]

    Kc, Vc = means(tK), means(tV)
    mask = torch.zeros((T, n + T), dtype=torch.bool)
    for t, (comp, win) in enumerate(_brute_visibility(T, block, window)):
        for j in comp:
            mask[t, j] = True
        for u in win:
            mask[t, n + u] = True
    outs = []
    for h in range(Hq):
        g = h * Hkv // Hq
        keys = torch.cat([Kc[:, g], tK[:, g]], dim=0)
        vals = torch.cat([Vc[:, g], tV[:, g]], dim=0)
        s = (tQ[:, h] @ keys.T) * scale
        p = torch.softmax(s.masked_fill(~mask, float("-inf")), dim=1)
        outs.append(p @ vals)
    O = torch.stack(outs, dim=1)
    return O if tG is None else O * tG


def _causal_sdpa(tQ, tK, tV, tG, scale):
    """Plain causal attention by torch SDPA; KV heads expanded by indexing."""
    Hq, Hkv = tQ.shape[1], tK.shape[1]
    idx = [h * Hkv // Hq for h in range(Hq)]
    q = tQ.permute(1, 0, 2)[None]
    k = tK[:, idx].permute(1, 0, 2)[None]
    v = tV[:, idx].permute(1, 0, 2)[None]
    o = F.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale)[0].permute(1, 0, 2)
    return o if tG is None else o * tG


def _close(got, want, tol, what):
    if want is None:
        assert got is None, what
        return
    err = float(np.abs(np.asarray(got) - np.asarray(want)).max())
    assert err <= tol, f"{what}: max |err| {err:.3e} > {tol:.1e}"


# ---------------------------------------------------------------------------
# pins (plain functions of the oracle module, so the mutant test can rerun them)
# ---------------------------------------------------------------------------

def pin_finite_differences(orc):
    """Central differences of sum(O * dO) through the forward oracle, every element
    of Q, K, V and G, including compressed entries fed by full blocks."""
    T, B, W, Hq, Hkv, D, scale = 13, 3, 4, 4, 2, 3, 0.7
    Q, K, V, dO, G = _case(T, Hq, Hkv, D, seed=21)
    dQ, dK, dV, dG = orc.hca_prefill_backward(Q, K, V, dO, B, W, scale, gate=G)

    def loss():
        O, _ = orc.hca_prefill(Q, K, V, B, W, scale, gate=G)
        return float((O * dO).sum())

    eps = 1e-6
    for name, X, dX in (("Q", Q, dQ), ("K", K, dK), ("V", V, dV), ("G", G, dG)):
        num = np.empty_like(X)
        for idx in np.ndindex(X.shape):
            x0 = X[idx]
            X[idx] = x0 + eps
            lp = loss()
            X[idx] = x0 - eps
            lm = loss()
            X[idx] = x0
            num[idx] = (lp - lm) / (2 * eps)
        _close(dX, num, 1e-6, f"d{name} vs finite differences")


def pin_dense_autograd(orc):
    """torch autograd of the dense masked-softmax formulation, grouped heads, gate on,
    a ragged last block, several compressed entries per query."""
    T, B, W, Hq, Hkv, D, scale = 150, 8, 12, 4, 2, 16, 0.25
    Q, K, V, dO, G = _case(T, Hq, Hkv, D, seed=31)
    want = _torch_grads(lambda q, k, v, g: _dense_hca(q, k, v, g, B, W, scale), Q, K, V, G, dO)
    got = orc.hca_prefill_backward(Q, K, V, dO, B, W, scale, gate=G)
    for name, a, b in zip("QKVG", got, want):
        _close(a, b, 1e-10, f"d{name} vs dense autograd")


def pin_dense_autograd_64_heads(orc):
    """The operator's head layout: 64 query heads share one KV head, so dK and dV sum the
    contributions of all 64 (torch autograd of the dense formulation, gate on)."""
    T, B, W, Hq, Hkv, D, scale = 160, 16, 24, 64, 1, 16, 0.25
    Q, K, V, dO, G = _case(T, Hq, Hkv, D, seed=61)
    want = _torch_grads(lambda q, k, v, g: _dense_hca(q, k, v, g, B, W, scale), Q, K, V, G, dO)
    got = orc.hca_prefill_backward(Q, K, V, dO, B, W, scale, gate=G)
    for name, a, b in zip("QKVG", got, want):
        _close(a, b, 1e-9, f"d{name} vs dense autograd (64 heads on one KV head)")


def pin_full_window_is_causal(orc):
    """window >= T: no compressed entry is visible, gradients of causal attention."""
    T, B, W, Hq, Hkv, D, scale = 40, 4, 64, 2, 1, 8, 0.3
    Q, K, V, dO, G = _case(T, Hq, Hkv, D, seed=41, gate=False)
    want = _torch_grads(lambda q, k, v, g: _causal_sdpa(q, k, v, g, scale), Q, K, V, G, dO)
    got = orc.hca_prefill_backward(Q, K, V, dO, B, W, scale, gate=None)
    for name, a, b in zip("QKVG", got, want):
        _close(a, b, 1e-10, f"d{name} vs causal SDPA (window >= T)")


def pin_block1_is_causal(orc):
    """block 1: every earlier token is visible exactly once (as its own entry or in the
    window), so the gradients are those of causal attention, through the pooling."""
    T, B, W, Hq, Hkv, D, scale = 40, 1, 5, 4, 2, 8, 0.3
    Q, K, V, dO, G = _case(T, Hq, Hkv, D, seed=51, gate=True)
    want = _torch_grads(lambda q, k, v, g: _causal_sdpa(q, k, v, g, scale), Q, K, V, G, dO)
    got = orc.hca_prefill_backward(Q, K, V, dO, B, W, scale, gate=G)
    for name, a, b in zip("QKVG", got, want):
        _close(a, b, 1e-10, f"d{name} vs causal SDPA (block 1)")


PINS = [pin_finite_differences, pin_dense_autograd, pin_dense_autograd_64_heads,
        pin_full_window_is_causal, pin_block1_is_causal]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_backward_pin(pin):
    pin(ORC)


# ---------------------------------------------------------------------------
# planted mistakes: each must fail at least one pin
# ---------------------------------------------------------------------------

def _mut_pool_no_count(dXc, T, block):
    out = np.zeros((T,) + dXc.shape[1:])
    for j in range(dXc.shape[0]):
        out[j * block:min((j + 1) * block, T)] += dXc[j]
    return out


def _mut_pool_to_first(dXc, T, block):
    out = np.zeros((T,) + dXc.shape[1:])
    for j in range(dXc.shape[0]):
        out[j * block] += dXc[j]
    return out


def _mut_softmax_no_delta(w, dw):
    return w * dw


def _wrap_attend_backward(kind):
    real = ORC.attend_position_backward

    def attend_backward(q, do, Kc, Vc, K, V, t, block, window, scale):
        dq, dkey, dval = real(q, do, Kc, Vc, K, V, t, block, window, scale)
        if kind == "ds_no_scale":
            return dq / scale, [d / scale for d in dkey], dval
        if kind == "swap_dkey_dval":
            return dq, dval, dkey
        if kind == "dkey_first_group_only":
            return dq, [dkey[0]] + [np.zeros_like(d) for d in dkey[1:]], dval
        return dq, dkey, dval
    return attend_backward


def _wrap_prefill_backward_no_gate():
    real = ORC.hca_prefill_backward

    def backward(Q, K, V, dO, block, window, scale, gate=None):
        dQ, dK, dV, _ = real(Q, K, V, dO, block, window, scale, gate=None)
        return dQ, dK, dV, None if gate is None else np.zeros_like(np.asarray(Q, np.float64))
    return backward


def _mut_window_wide(t, window):
    return max(0, t - window), t


MUTANTS = {
    "pool_no_count": ("pool_backward", _mut_pool_no_count),
    "pool_to_first": ("pool_backward", _mut_pool_to_first),
    "softmax_no_delta": ("_softmax_backward", _mut_softmax_no_delta),
    # shared with the forward: the finite differences follow it, the torch pins do not
    "window_wide": ("window_bounds", _mut_window_wide),
}
WRAPPED = ["ds_no_scale", "swap_dkey_dval", "dkey_first_group_only"]


@pytest.mark.parametrize("name", sorted(MUTANTS) + WRAPPED + ["gate_ignored"])
def test_planted_backward_mistakes(name, monkeypatch):
    if name in MUTANTS:
        attr, fn = MUTANTS[name]
        monkeypatch.setattr(ORC, attr, fn)
    elif name == "gate_ignored":
        monkeypatch.setattr(ORC, "hca_prefill_backward", _wrap_prefill_backward_no_gate())
    else:
        monkeypatch.setattr(ORC, "attend_position_backward", _wrap_attend_backward(name))
    failed = []
    for pin in PINS:
        try:
            pin(ORC)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"planted mistake {name!r} passed every pin"
