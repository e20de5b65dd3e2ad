"""GPU: the gate from the low-rank query latent (hca_gate_from_latent, one tcgen05 GEMM with
the sigmoid in its epilogue) and the cross-head mixing with the gate (hca_vha_gate), against
the float64 oracle; and the whole layer output (prefill without a gate, then VHA + gate)."""

import numpy as np
import pytest
import torch

from compressed_long_context_hca_b200 import inputs, ops
from oracle import hca_oracle as orc
from tests.gpu_helpers import (BF16_MAX, BF16_MEAN, F32_MAX, compare, default_scale,
                               ensure_built, run_prefill, to64)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,latent,hq,D", [
    (1000, 1024, 64, 512),   # the pages' shapes: latent = hidden / 4 = 1024, 64 x 512 gates
    (37, 64, 4, 32),         # ragged rows, small latent
    (300, 200, 3, 96),       # latent and width not multiples of the GEMM tiles
])
def test_gate_from_latent(rows, latent, hq, D):
    ensure_built()
    g = torch.Generator().manual_seed(rows)
    q = torch.randn((rows, latent), generator=g).to(torch.bfloat16)
    W = (torch.randn((latent, hq * D), generator=g) / np.sqrt(latent)).to(torch.bfloat16)
    G = ops.gate_from_latent(q.cuda(), W.cuda(), hq, D)
    torch.cuda.synchronize()
    ref = orc.gate_from_latent(to64(q), to64(W), hq, D)
    compare(to64(G), ref, BF16_MAX, BF16_MEAN, what="G")


@pytest.mark.parametrize("dtype,shape,rank,gate", [
    ("bf16", (2, 100, 64, 512), 8, True),
    ("bf16", (1, 33, 16, 512), 16, False),
    ("f32", (2, 50, 6, 64), 3, True),
    ("bf16", (1, 20, 64, 512), 0, True),     # rank 0: the gate alone
])
def test_vha_gate(dtype, shape, rank, gate):
    ensure_built()
    g = torch.Generator().manual_seed(sum(shape) + rank)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    O = torch.randn(shape, generator=g).to(dt)
    b, T, hq, D = shape
    A = torch.randn((hq, rank), generator=g) / 4 if rank else None
    Bm = torch.randn((hq, rank), generator=g) / 4 if rank else None
    G = torch.sigmoid(torch.randn(shape, generator=g)).to(dt) if gate else None
    out = ops.vha_gate(O.cuda(), None if A is None else A.cuda(),
                       None if Bm is None else Bm.cuda(), None if G is None else G.cuda())
    torch.cuda.synchronize()
    tol = (F32_MAX, None) if dtype == "f32" else (BF16_MAX, BF16_MEAN)
    for bi in range(b):
        ref = orc.attention_output(to64(O[bi]), None if G is None else to64(G[bi]),
                                   None if A is None else to64(A), None if Bm is None else to64(Bm))
        compare(to64(out[bi]), ref, tol[0], tol[1], what=f"out[{bi}]")


def test_layer_output_prefill_vha_gate_from_latent():
    """The attention output of an HCA layer end to end on the GPU: the gate from the query
    latent, the prefill without the gate, then the VHA mixing and the gate. The stages hand
    each other bf16 tensors (the gate, the heads' outputs), so each stage is compared with the
    oracle on the input it actually received: the gate and the heads' outputs against the
    oracle's, and the mixed, gated output against the oracle's mixing and gate of those."""
    ensure_built()
    b, T, hq, D, L, r = 2, 600, 64, 512, 1024, 8
    x = inputs.prefill_inputs(b, T, hq, 1, D, "bf16", seed=71)
    g = torch.Generator().manual_seed(72)
    q_lat = torch.randn((b * T, L), generator=g).to(torch.bfloat16)
    W = (torch.randn((L, hq * D), generator=g) / np.sqrt(L)).to(torch.bfloat16)
    A = torch.randn((hq, r), generator=g) / 8
    Bm = torch.randn((hq, r), generator=g) / 8
    G = ops.gate_from_latent(q_lat.cuda(), W.cuda(), hq, D).view(b, T, hq, D)
    res = run_prefill(x)                 # no gate attached: the heads' attention outputs
    out = ops.vha_gate(res["O"], A.cuda(), Bm.cuda(), G)
    torch.cuda.synchronize()
    Gref = orc.gate_from_latent(to64(q_lat), to64(W), hq, D).reshape(b, T, hq, D)
    pos = [0, 1, 127, 128, 255, 256, 300, 599]
    for bi in range(b):
        O_attn, _ = orc.hca_prefill(to64(x.Q[bi]), to64(x.K[bi]), to64(x.V[bi]), 128, 128,
                                    default_scale(D), positions=pos)
        compare(to64(res["O"][bi, pos]), O_attn, BF16_MAX, BF16_MEAN, what=f"O_attn[{bi}]")
        compare(to64(G[bi]), Gref[bi], BF16_MAX, BF16_MEAN, what=f"G[{bi}]")
        ref = orc.attention_output(to64(res["O"][bi, pos]), to64(G[bi, pos]), to64(A),
                                   to64(Bm))
        compare(to64(out[bi, pos]), ref, BF16_MAX, BF16_MEAN, what=f"out[{bi}]")
