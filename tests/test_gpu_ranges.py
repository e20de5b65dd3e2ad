"""GPU: prefill over query-position ranges (hca_attn_prefill_range) and decode over key
parts (hca_attn_decode_partial + hca_decode_merge), the compute steps of splitting one
sequence over several GPUs, run here rank after rank on one GPU, against the oracle."""

import numpy as np
import pytest
import torch

from compressed_long_context_hca_b200 import binding as B
from compressed_long_context_hca_b200 import inputs, ops
from oracle import hca_oracle as orc
from tests.gpu_helpers import (BF16_MAX, BF16_MEAN, F32_MAX, LSE_MAX, LSE_MEAN, compare,
                               default_scale, ensure_built, run_prefill, to64)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,hq,cuts,gate", [
    ("bf16", 64, [0, 384, 640, 1000], True),   # block-aligned ranges (the row partition)
    ("bf16", 64, [0, 300, 555, 1000], False),  # any offsets (chunked prefill)
    ("bf16", 8, [0, 256, 1000], False),        # one-CTA kernel (8 heads)
    ("bf16", 32, [0, 128, 129, 1000], True),   # a one-position range
    ("f32", 4, [0, 200, 1000], True),          # CUDA-core kernel
])
def test_prefill_ranges_match_oracle(dtype, hq, cuts, gate):
    """Each range [q0, q1) runs with only its K/V rows plus the window-1 rows before it
    (the halo) and the full compressed cache; every position against the oracle, and the
    lse and debug mask (absolute positions) too."""
    ensure_built()
    dev = torch.device("cuda")
    T, b, W = 1000, 2, 128
    x = inputs.prefill_inputs(b, T, hq, 1, 512, dtype, seed=31, gate=gate,
                              hetero_blocks=(dtype == "bf16"))
    full = run_prefill(x, dtype=dtype)  # compresses every block into full["cache"]
    cache = full["cache"]
    Q, K, V = x.Q.to(dev), x.K.to(dev), x.V.to(dev)
    G = None if x.G is None else x.G.to(dev)
    tol = (F32_MAX, None) if dtype == "f32" else (BF16_MAX, BF16_MEAN)
    ltol = (1e-5, None) if dtype == "f32" else (LSE_MAX, LSE_MEAN)
    refs = [orc.hca_prefill(to64(x.Q[bi]), to64(x.K[bi]), to64(x.V[bi]), 128, W,
                            default_scale(512), gate=None if x.G is None else to64(x.G[bi]))
            for bi in range(b)]
    for q0, q1 in zip(cuts, cuts[1:]):
        kv0 = max(0, q0 - W + 1)
        desc = ops.desc_for_prefill(Q[:, q0:q1], K)
        ops.attach_gate(desc, None if G is None else G[:, q0:q1].contiguous())
        O, lse, dbg = ops.prefill_range(desc, q0, kv0, Q[:, q0:q1].contiguous(),
                                        K[:, kv0:q1].contiguous(), V[:, kv0:q1].contiguous(),
                                        cache, want_lse=True, want_mask=True)
        torch.cuda.synchronize()
        assert int(cache.err.item()) == 0
        for bi in range(b):
            ref, rl = refs[bi]
            compare(to64(O[bi]), ref[q0:q1], tol[0], tol[1], what=f"[{q0},{q1}) O[{bi}]")
            compare(to64(lse[bi]), rl[q0:q1], ltol[0], ltol[1], what=f"[{q0},{q1}) lse",
                    out_bf16=False)
            want = orc.mask_table(T, 128, W)[q0:q1]
            assert np.array_equal(dbg[bi].cpu().numpy(), want)


def _decode_case(nseq, lo, hi, seed, gate):
    dev = torch.device("cuda")
    W, blk, D, hq = 128, 128, 512, 64
    max_ent = (hi - W) // blk + 1
    x = inputs.decode_inputs(nseq, hq, 1, D, W, blk, lo, hi, max_ent, "bf16", seed, gate)
    cache = B.PagedCache(nseq, max_ent, 1, D, torch.bfloat16, 128,
                         page_table=inputs.page_table(nseq, -(-max_ent // 128), seed),
                         device=dev)
    for b in range(nseq):
        cache.fill(b, x.entries_k[b].to(dev), x.entries_v[b].to(dev))
    desc = B.make_desc(nseq, hi, hq, 1, D)
    ops.attach_gate(desc, None if x.G is None else x.G.to(dev))
    t = dict(q=x.q.to(dev), ctx=x.ctx_len.to(dev), rk=x.ring_k.to(dev), rv=x.ring_v.to(dev))
    return x, desc, cache, t


@pytest.mark.parametrize("parts", [
    [(0, 1 << 30, True)],                               # one part = the whole key set
    [(0, 128, False), (128, 1 << 30, True)],
    [(0, 256, False), (256, 384, False), (384, 1 << 30, False), (0, 0, True)],  # window alone
    [(0, 128 * 100, False), (128 * 100, 128 * 400, True), (128 * 400, 1 << 30, False)],
])
def test_decode_parts_merge_to_the_decode(parts):
    """Disjoint key parts of every sequence (entry ranges of whole tiles, the window in one
    of them; some parts hold no key of the short sequences) merged into the decode output:
    against the oracle, and against hca_attn_decode."""
    ensure_built()
    x, desc, cache, t = _decode_case(6, 300, 60000, seed=41, gate=True)
    buf = ops.decode_partial_buffer(desc, len(parts))
    for k, (e0, e1, win) in enumerate(parts):
        ops.decode_partial(desc, t["q"], t["ctx"], cache, t["rk"], t["rv"], e0, e1, win,
                           buf[k])
    O = torch.empty_like(t["q"])
    lse = torch.empty(t["q"].shape[:2], dtype=torch.float32, device=O.device)
    ops.decode_merge(desc, buf, O, lse)
    O_ref, lse_ref = ops.decode(desc, t["q"], t["ctx"], cache, t["rk"], t["rv"], want_lse=True)
    torch.cuda.synchronize()
    assert int(cache.err.item()) == 0
    for b in range(6):
        ref, rl = orc.hca_decode(to64(x.q[b]), to64(x.entries_k[b]), to64(x.entries_v[b]),
                                 to64(x.ring_k[b]), to64(x.ring_v[b]), int(x.ctx_len[b]), 128,
                                 128, default_scale(512), gate=to64(x.G[b]))
        compare(to64(O[b]), ref, BF16_MAX, BF16_MEAN, what=f"O[{b}]")
        compare(to64(lse[b]), rl, LSE_MAX, LSE_MEAN, what=f"lse[{b}]", out_bf16=False)
        compare(to64(O[b]), to64(O_ref[b]), 1.6e-2, 1e-3, what=f"vs decode O[{b}]")


def test_decode_partial_with_forced_splits():
    """A part long enough to be cut into several splits inside the call (merged into one
    partial by the merge kernel) and a part of one split (written by the decode CTAs):
    merged, both equal the decode."""
    ensure_built()
    x, desc, cache, t = _decode_case(4, 90000, 130000, seed=43, gate=False)
    desc.decode_splits = 5
    buf = ops.decode_partial_buffer(desc, 2)
    ops.decode_partial(desc, t["q"], t["ctx"], cache, t["rk"], t["rv"], 0, 128 * 600, False,
                       buf[0])
    ops.decode_partial(desc, t["q"], t["ctx"], cache, t["rk"], t["rv"], 128 * 600, 1 << 30,
                       True, buf[1])
    O = torch.empty_like(t["q"])
    ops.decode_merge(desc, buf, O)
    torch.cuda.synchronize()
    for b in range(4):
        ref, _ = orc.hca_decode(to64(x.q[b]), to64(x.entries_k[b]), to64(x.entries_v[b]),
                                to64(x.ring_k[b]), to64(x.ring_v[b]), int(x.ctx_len[b]), 128,
                                128, default_scale(512))
        compare(to64(O[b]), ref, BF16_MAX, BF16_MEAN, what=f"O[{b}]")


def test_parallel_paths_in_a_world_of_one():
    """parallel.prefill_rows and parallel.decode_split_entries with the libhca backend and
    no process group (one rank holds everything): the same results as the plain calls,
    within the bf16 tolerance of the oracle."""
    from compressed_long_context_hca_b200 import parallel as P
    ensure_built()
    dev = torch.device("cuda")
    T = 900
    x = inputs.prefill_inputs(1, T, 64, 1, 512, "bf16", seed=51, gate=True)
    be = P.GpuBackend()
    for _ in range(2):  # the second call reuses the backend's buffers
        O = P.prefill_rows(be, None, x.Q.to(dev), x.K.to(dev), x.V.to(dev), T, 128, 128,
                           G=x.G.to(dev))
        torch.cuda.synchronize()
    ref, _ = orc.hca_prefill(to64(x.Q[0]), to64(x.K[0]), to64(x.V[0]), 128, 128,
                             default_scale(512), gate=to64(x.G[0]))
    compare(to64(O[0]), ref, BF16_MAX, BF16_MEAN, what="prefill_rows O")
    xd, desc, cache, t = _decode_case(4, 5000, 40000, seed=52, gate=True)
    n_vis = (int(xd.ctx_len.max()) - 128) // 128
    Od = P.decode_split_entries(be, None, t["q"], t["ctx"], cache, t["rk"], t["rv"], n_vis,
                                desc)
    torch.cuda.synchronize()
    for b in range(4):
        ref, _ = orc.hca_decode(to64(xd.q[b]), to64(xd.entries_k[b]), to64(xd.entries_v[b]),
                                to64(xd.ring_k[b]), to64(xd.ring_v[b]), int(xd.ctx_len[b]),
                                128, 128, default_scale(512), gate=to64(xd.G[b]))
        compare(to64(Od[b]), ref, BF16_MAX, BF16_MEAN, what=f"decode_split_entries O[{b}]")
