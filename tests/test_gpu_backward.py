"""GPU prefill backward (hca_attn_prefill_backward) against the float64 oracle's
hca_prefill_backward: dQ, dK, dV and dG element by element."""

import numpy as np
import pytest
import torch

from compressed_long_context_hca_b200 import inputs, ops
from oracle import hca_oracle as orc
from tests.gpu_helpers import (BF16_MAX, BF16_MEAN, F32_MAX, GRAD_REL, compare,
                               default_scale, run_prefill, to64)

pytestmark = pytest.mark.gpu


def _grad_out(x, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(x.Q.shape, generator=g).to(x.Q.dtype)


def _run(x, dO, block, window, dtype, page_entries):
    """Forward (compress + prefill with lse) then backward, all through the C ABI."""
    r = run_prefill(x, block=block, window=window, dtype=dtype, page_entries=page_entries,
                    want_lse=True)
    dev = torch.device("cuda")
    Q, K, V = x.Q.to(dev), x.K.to(dev), x.V.to(dev)
    grads = ops.prefill_backward(r["desc"], Q, K, V, r["cache"], r["lse"], dO.to(dev))
    torch.cuda.synchronize()
    assert int(r["cache"].err.item()) == 0
    return grads


@pytest.mark.parametrize("T,hq,hkv,D,block,window,gate", [
    (37, 2, 1, 32, 4, 3, False),       # tiny ragged, window < block
    (300, 6, 2, 64, 16, 40, True),     # grouped heads, gate, ragged last block
    (513, 3, 1, 128, 128, 128, True),  # block 128, window 128
    (64, 1, 1, 32, 1, 5, False),       # block 1 = full causal attention
    (50, 2, 1, 32, 8, 64, False),      # window >= T = plain causal attention
])
def test_backward_fp32_matches_oracle(T, hq, hkv, D, block, window, gate):
    x = inputs.prefill_inputs(2, T, hq, hkv, D, "f32", seed=61, gate=gate, block=block)
    dO = _grad_out(x, 62)
    dQ, dK, dV, dG = _run(x, dO, block, window, "f32", page_entries=4)
    s = default_scale(D)
    for bi in range(2):
        ref = orc.hca_prefill_backward(to64(x.Q[bi]), to64(x.K[bi]), to64(x.V[bi]),
                                       to64(dO[bi]), block, window, s,
                                       gate=None if x.G is None else to64(x.G[bi]))
        for name, got, want in zip("QKV", (dQ, dK, dV), ref[:3]):
            compare(to64(got[bi]), want, F32_MAX, what=f"d{name}[{bi}]")
        if gate:
            compare(to64(dG[bi]), ref[3], F32_MAX, what=f"dG[{bi}]")
        else:
            assert dG is None


@pytest.mark.parametrize("T,hq,gate,hetero", [
    (700, 64, True, True),      # the training workload's features: x4 blocks, fused gate
    (1000, 16, False, False),
    (129, 8, True, False),      # one compressed... none visible yet: window only
])
def test_backward_bf16_matches_oracle(T, hq, gate, hetero):
    x = inputs.prefill_inputs(1, T, hq, 1, 512, "bf16", seed=63, gate=gate,
                              hetero_blocks=hetero)
    dO = _grad_out(x, 64)
    dQ, dK, dV, dG = _run(x, dO, 128, 128, "bf16", page_entries=128)
    ref = orc.hca_prefill_backward(to64(x.Q[0]), to64(x.K[0]), to64(x.V[0]), to64(dO[0]), 128,
                                   128, default_scale(512),
                                   gate=None if x.G is None else to64(x.G[0]))
    for name, got, want in zip("QKV", (dQ, dK, dV), ref[:3]):
        compare(to64(got[0]), want, BF16_MAX, BF16_MEAN, what=f"d{name}", rel=GRAD_REL)
    if gate:
        compare(to64(dG[0]), ref[3], BF16_MAX, BF16_MEAN, what="dG", rel=GRAD_REL)


def test_backward_bf16_cuda_core_path():
    """bf16 shapes outside the tensor-core path (2 KV heads, head_dim 64) run on the CUDA-core
    kernels in float32 arithmetic."""
    from compressed_long_context_hca_b200 import binding as B
    x = inputs.prefill_inputs(1, 300, 4, 2, 64, "bf16", seed=67, gate=True, block=16)
    dO = _grad_out(x, 68)
    dev = torch.device("cuda")
    Q, K, V, G = (t.to(dev) for t in (x.Q, x.K, x.V, x.G))
    desc = ops.desc_for_prefill(Q, K, 16, 40)
    ops.attach_gate(desc, G)
    cache = B.PagedCache(1, 300 // 16 + 1, 2, 64, torch.bfloat16, 4, device=dev)
    ops.compress(desc, K, V, cache)
    # this shape has no bf16 forward kernel: the lse comes from the oracle
    _, lse = orc.hca_prefill(to64(x.Q[0]), to64(x.K[0]), to64(x.V[0]), 16, 40, default_scale(64))
    lse_t = torch.from_numpy(lse).to(torch.float32)[None].to(dev)
    dQ, dK, dV, dG = ops.prefill_backward(desc, Q, K, V, cache, lse_t, dO.to(dev))
    torch.cuda.synchronize()
    assert int(cache.err.item()) == 0
    ref = orc.hca_prefill_backward(to64(x.Q[0]), to64(x.K[0]), to64(x.V[0]), to64(dO[0]), 16,
                                   40, default_scale(64), gate=to64(x.G[0]))
    for name, got, want in zip("QKVG", (dQ, dK, dV, dG), ref):
        compare(to64(got[0]), want, BF16_MAX, BF16_MEAN, what=f"d{name}", rel=GRAD_REL)


def test_backward_bf16_32k_sampled():
    """The 32K workload (1 x 32768, 64 heads, head_dim 512): dQ at sampled positions, and
    dK / dV of tokens of the last blocks (whose entries no query sees, so the window rows
    alone make their gradient) against the oracle's per-position backward."""
    T, W, blk = 32768, 128, 128
    x = inputs.prefill_inputs(1, T, 64, 1, 512, "bf16", seed=65)
    dO = _grad_out(x, 66)
    dQ, dK, dV, _ = _run(x, dO, blk, W, "bf16", page_entries=128)
    Q, K, V, dO64 = to64(x.Q[0]), to64(x.K[0]), to64(x.V[0]), to64(dO[0])
    Kc, Vc = orc.compress_blocks(K, blk), orc.compress_blocks(V, blk)
    s = default_scale(512)
    rng = np.random.default_rng(7)
    pos = sorted(set([0, 127, 128, 255, 16511, T - 1] + rng.integers(0, T, 10).tolist()))
    for t in pos:
        dq, _, _ = orc.attend_position_backward(Q[t], dO64[t], Kc, Vc, K, V, t, blk, W, s)
        compare(to64(dQ[0, t]), dq, BF16_MAX, BF16_MEAN, what=f"dQ[{t}]", rel=GRAD_REL)
    # tokens of the last block: its entry becomes visible only from position T + 127 on,
    # so dK[u] sums the window rows t in [u, T) alone
    us = [T - 128, T - 100, T - 64, T - 1]
    dk = {u: np.zeros(512) for u in us}
    dv = {u: np.zeros(512) for u in us}
    for t in range(min(us), T):
        _, dkey, dval = orc.attend_position_backward(Q[t], dO64[t], Kc, Vc, K, V, t, blk, W, s)
        nc = orc.visible_compressed_count(t, blk, W)
        lo, _ = orc.window_bounds(t, W)
        for u in us:
            if lo <= u <= t:
                dk[u] += dkey[0][nc + u - lo]
                dv[u] += dval[0][nc + u - lo]
    for u in us:
        compare(to64(dK[0, u, 0]), dk[u], BF16_MAX, BF16_MEAN, what=f"dK[{u}]", rel=GRAD_REL)
        compare(to64(dV[0, u, 0]), dv[u], BF16_MAX, BF16_MEAN, what=f"dV[{u}]", rel=GRAD_REL)
