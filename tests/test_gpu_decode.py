"""GPU decode (hca_attn_decode) against the float64 oracle, plus cross-path checks."""

import numpy as np
import pytest
import torch

from compressed_long_context_hca_b200 import binding as B
from compressed_long_context_hca_b200 import inputs, ops
from oracle import hca_oracle as orc
from tests.gpu_helpers import (BF16_MAX, BF16_MEAN, F32_MAX, LSE_MAX, LSE_MEAN, bf16_ulp,
                               compare, default_scale, ensure_built, run_prefill, to64)

pytestmark = pytest.mark.gpu


def _setup(nseq, ctx_lo, ctx_hi, dtype="bf16", gate=False, seed=0, hq=64, D=512, W=128,
           block=128, splits=0, pe=128, k_ramp=None):
    ensure_built()
    dev = torch.device("cuda")
    max_ent = max(1, (ctx_hi - W) // block + 1)
    x = inputs.decode_inputs(nseq, hq, 1, D, W, block, ctx_lo, ctx_hi, max_ent, dtype, seed,
                             gate)
    if k_ramp is not None:
        # compressed keys of 128-entry tile j scaled by k_ramp**j (then rounded again), so
        # the running row max grows from one 256-key chunk to the next
        for b in range(nseq):
            ek = x.entries_k[b]
            f = k_ramp ** (torch.arange(ek.shape[0], dtype=torch.float64) // 128)
            x.entries_k[b] = (ek.double() * f[:, None, None]).to(ek.dtype)
    mp = -(-max_ent // pe)
    cache = B.PagedCache(nseq, max_ent, 1, D, x.q.dtype, pe,
                         page_table=inputs.page_table(nseq, mp), device=dev)
    for b in range(nseq):
        cache.fill(b, x.entries_k[b].to(dev), x.entries_v[b].to(dev))
    desc = B.make_desc(nseq, ctx_hi, hq, 1, D, block, W, None,
                       B.HCA_BF16 if dtype == "bf16" else B.HCA_F32, splits)
    G = None if x.G is None else x.G.to(dev)
    ops.attach_gate(desc, G)
    return x, cache, desc


def _run(x, cache, desc):
    dev = torch.device("cuda")
    O, lse = ops.decode(desc, x.q.to(dev), x.ctx_len.to(dev), cache, x.ring_k.to(dev),
                        x.ring_v.to(dev), want_lse=True)
    torch.cuda.synchronize()
    return O, lse


def _oracle(x, b, block=128, W=128):
    D = x.q.shape[-1]
    G = None if x.G is None else to64(x.G[b])
    return orc.hca_decode(to64(x.q[b]), to64(x.entries_k[b]), to64(x.entries_v[b]),
                          to64(x.ring_k[b]), to64(x.ring_v[b]), int(x.ctx_len[b]), block, W,
                          default_scale(D), gate=G)


@pytest.mark.parametrize("nseq,lo,hi,gate", [
    (4, 1, 127, False),            # window only, partly filled ring
    (6, 128, 700, True),           # 0..4 entries
    (8, 8192, 40000, False),       # many tiles, several splits
    (3, 70000, 70000, True),       # equal lengths
])
def test_decode_bf16(nseq, lo, hi, gate):
    x, cache, desc = _setup(nseq, lo, hi, gate=gate)
    O, lse = _run(x, cache, desc)
    for b in range(nseq):
        ref, rl = _oracle(x, b)
        compare(to64(O[b]), ref, BF16_MAX, BF16_MEAN, what=f"O[{b}]")
        compare(to64(lse[b]), rl, LSE_MAX, LSE_MEAN, what=f"lse[{b}]", out_bf16=False)
    assert int(cache.err.item()) == 0


@pytest.mark.parametrize("dtype,hkv,D", [("bf16", 1, 512), ("f32", 2, 64)])
def test_ring_append(dtype, hkv, D):
    """hca_ring_append writes each sequence's new rows to slot (ctx_len - 1) % W, ctx_len
    clamped into [1, seqlen] as decode clamps it: compared byte for byte with plain indexing
    of the same tensors (slots 0 and W - 1, a wrap, a clamp at each end)."""
    ensure_built()
    dev = torch.device("cuda")
    W, seqlen = 128, 5000
    ctx = [1, 128, 129, 4999, 0, 7000]
    nseq = len(ctx)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    g = torch.Generator().manual_seed(31)
    ring_k = torch.randn((nseq, W, hkv, D), generator=g).to(tdt)
    ring_v = torch.randn((nseq, W, hkv, D), generator=g).to(tdt)
    new_k = torch.randn((nseq, hkv, D), generator=g).to(tdt)
    new_v = torch.randn((nseq, hkv, D), generator=g).to(tdt)
    want_k, want_v = ring_k.clone(), ring_v.clone()
    for b, c in enumerate(ctx):
        slot = (min(max(c, 1), seqlen) - 1) % W
        want_k[b, slot] = new_k[b]
        want_v[b, slot] = new_v[b]
    rk, rv = ring_k.to(dev), ring_v.to(dev)
    desc = B.make_desc(nseq, seqlen, 4 * hkv, hkv, D, 128, W, None,
                       B.HCA_BF16 if dtype == "bf16" else B.HCA_F32)
    ops.ring_append(desc, new_k.to(dev), new_v.to(dev),
                    torch.tensor(ctx, dtype=torch.int32, device=dev), rk, rv)
    torch.cuda.synchronize()
    assert torch.equal(rk.cpu(), want_k) and torch.equal(rv.cpu(), want_v)


@pytest.mark.parametrize("nseq,lo,hi,splits", [
    (6, 1, 127, 0),            # window only, partly filled ring
    (8, 8192, 40000, 0),       # several splits: only the last one reads the ring
    (3, 20000, 30000, 1),      # one split
])
def test_decode_append_equals_append_then_decode(nseq, lo, hi, splits):
    """hca_attn_decode_append (the new rows written by the CTA that reads the window)
    gives byte-identical rings and outputs to hca_ring_append followed by hca_attn_decode."""
    x, cache, desc = _setup(nseq, lo, hi, seed=80 + nseq, gate=True, splits=splits)
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(81)
    nk = torch.randn((nseq, 1, 512), generator=g).to(torch.bfloat16).to(dev)
    nv = torch.randn((nseq, 1, 512), generator=g).to(torch.bfloat16).to(dev)
    q, ctx = x.q.to(dev), x.ctx_len.to(dev)
    rk_a, rv_a = x.ring_k.to(dev), x.ring_v.to(dev)
    rk_b, rv_b = rk_a.clone(), rv_a.clone()
    ops.ring_append(desc, nk, nv, ctx, rk_a, rv_a)
    O_a, l_a = ops.decode(desc, q, ctx, cache, rk_a, rv_a, want_lse=True)
    O_b, l_b = ops.decode_append(desc, q, ctx, cache, nk, nv, rk_b, rv_b, want_lse=True)
    torch.cuda.synchronize()
    assert torch.equal(rk_a, rk_b) and torch.equal(rv_a, rv_b)
    assert torch.equal(O_a, O_b) and torch.equal(l_a, l_b)
    assert int(cache.err.item()) == 0


# the last compressed tile holds 16 * odd entries, all visible: its last 32-column score
# piece runs 16 columns past the tile, and those columns (stale tensor memory, scores of an
# earlier tile) must enter neither P nor the row sum
MID_PIECE_CASES = [
    (128 * 80 + 5, 0),            # one compressed tile of 80 entries
    (128 * (256 + 48) + 100, 0),  # last tile of 48 entries
    (128 * (384 + 16) + 127, 2),  # last tile of 16, two splits
    (128 * (128 + 112) + 64, 1),  # last tile of 112, one split
]


@pytest.mark.parametrize("ctx,splits", MID_PIECE_CASES)
def test_decode_tile_ends_mid_piece(ctx, splits):
    x, cache, desc = _setup(2, ctx, ctx, seed=60 + splits, splits=splits)
    O, lse = _run(x, cache, desc)
    for b in range(2):
        ref, rl = _oracle(x, b)
        compare(to64(O[b]), ref, BF16_MAX, BF16_MEAN, what=f"ctx={ctx} O[{b}]")
        compare(to64(lse[b]), rl, LSE_MAX, LSE_MEAN, what=f"ctx={ctx} lse[{b}]", out_bf16=False)
    assert int(cache.err.item()) == 0


def _sample_sequences(ctx_len, n, seed):
    """n sequences drawn by a seeded generator, always with the longest and the shortest
    context among them."""
    lens = ctx_len.numpy()
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(len(lens), size=n, replace=False).tolist())
    pick |= {int(np.argmax(lens)), int(np.argmin(lens))}
    return sorted(pick)


def test_decode_batched_config_sampled():
    """128 sequences with context lengths uniform in [8192, 131072], one query each,
    64 heads, head_dim 512, paged cache + last 128 raw tokens, N(0,1). 24 seeded-random
    sequences plus the longest and the shortest against the oracle."""
    x, cache, desc = _setup(128, 8192, 131072, seed=0)
    O, lse = _run(x, cache, desc)
    for b in _sample_sequences(x.ctx_len, 24, seed=5):
        ref, rl = _oracle(x, b)
        compare(to64(O[b]), ref, BF16_MAX, BF16_MEAN, what=f"O[{b}]")
        compare(to64(lse[b]), rl, LSE_MAX, LSE_MEAN, what=f"lse[{b}]", out_bf16=False)


@pytest.mark.parametrize("splits", [1, 2, 3, 7, 40, 0])
def test_decode_split_invariance(splits):
    """Each key list cut into `splits` splits (40: more than the tiles, capped at one tile
    per split) and merged."""
    x, cache, desc = _setup(5, 20000, 60000, seed=3, splits=splits)
    O, _ = _run(x, cache, desc)
    for b in range(5):
        ref, _ = _oracle(x, b)
        compare(to64(O[b]), ref, BF16_MAX, BF16_MEAN, what=f"splits={splits} O[{b}]")


def test_decode_fp32():
    x, cache, desc = _setup(3, 1, 5000, dtype="f32", gate=True, seed=4, hq=4)
    O, lse = _run(x, cache, desc)
    for b in range(3):
        ref, rl = _oracle(x, b)
        compare(to64(O[b]), ref, F32_MAX, what=f"O[{b}]")
        compare(to64(lse[b]), rl, 1e-5, what=f"lse[{b}]")


def test_decode_equals_prefill_row():
    """The decode step at position t sees exactly the prefill key set of t."""
    T, D, W = 1200, 512, 128
    x = inputs.prefill_inputs(1, T, 64, 1, D, "bf16", seed=9)
    r = run_prefill(x)
    dev = torch.device("cuda")
    K, V, Q = x.K.to(dev), x.V.to(dev), x.Q.to(dev)
    for t in (0, 100, 127, 128, 255, 256, 1000, T - 1):
        rk = torch.zeros((1, W, 1, D), dtype=torch.bfloat16, device=dev)
        rv = torch.zeros_like(rk)
        for u in range(max(0, t - W + 1), t + 1):
            rk[0, u % W] = K[0, u]
            rv[0, u % W] = V[0, u]
        desc = B.make_desc(1, T, 64, 1, D)
        ctx = torch.tensor([t + 1], dtype=torch.int32, device=dev)
        Od, _ = ops.decode(desc, Q[:, t].contiguous(), ctx, r["cache"], rk, rv)
        torch.cuda.synchronize()
        # two bf16-rounded results of the same float32 value may land one bf16 ulp apart
        # (1.6e-2 for |O| in [2, 4))
        compare(to64(Od[0]), to64(r["O"][0, t]), 1.6e-2, 1e-3, what=f"t={t}")


@pytest.mark.parametrize("dtype,hq", [("bf16", 64), ("f32", 4)])
def test_decode_ctx_len_out_of_range_is_clamped_and_flagged(dtype, hq):
    """ctx_len outside [1, seqlen] is clamped into that range and raises HCA_ERR_CTX_RANGE;
    the result then equals a call with the clamped lengths."""
    x, cache, desc = _setup(3, 300, 9000, dtype=dtype, seed=6, hq=hq)
    dev = torch.device("cuda")
    args = (x.q.to(dev), cache, x.ring_k.to(dev), x.ring_v.to(dev))
    bad = torch.tensor([0, int(x.ctx_len[1]), desc.seqlen + 777], dtype=torch.int32)
    good = torch.tensor([1, int(x.ctx_len[1]), desc.seqlen], dtype=torch.int32)
    O_bad, _ = ops.decode(desc, args[0], bad.to(dev), *args[1:])
    torch.cuda.synchronize()
    assert int(cache.err.item()) & B.HCA_ERR_CTX_RANGE
    cache.err.zero_()
    O_good, _ = ops.decode(desc, args[0], good.to(dev), *args[1:])
    torch.cuda.synchronize()
    assert int(cache.err.item()) == 0
    assert torch.equal(O_bad, O_good)


def test_decode_running_max_grows_across_chunks():
    """Keys whose scale grows tile by tile: the row max rises by far more than the lazy
    rescale threshold at every 256-key chunk of a split, so O is rescaled in tensor memory
    between chunks. The softmax is nearly one-hot: the bf16 tolerance holds because P
    enters P.V as a bf16 pair (hi + lo), not as one bf16 value."""
    x, cache, desc = _setup(2, 100000, 110000, seed=8, splits=1, k_ramp=1.8)
    O, lse = _run(x, cache, desc)
    for b in range(2):
        ref, rl = _oracle(x, b)
        compare(to64(O[b]), ref, BF16_MAX, BF16_MEAN, what=f"O[{b}]")
        compare(to64(lse[b]), rl, LSE_MAX, LSE_MEAN, what=f"lse[{b}]", out_bf16=False)
    assert int(cache.err.item()) == 0


@pytest.mark.parametrize("nseq,hq,gate", [(1, 5, True), (3, 33, False), (2, 1, True)])
def test_decode_bf16_odd_head_counts(nseq, hq, gate):
    """hq below 64 and odd: the M = 64 UMMA rows past hq are padding, and the split
    partials of an odd number of heads still start 16-byte aligned in the workspace."""
    x, cache, desc = _setup(nseq, 9000, 40000, seed=10 + hq, hq=hq, gate=gate)
    O, lse = _run(x, cache, desc)
    for b in range(nseq):
        ref, rl = _oracle(x, b)
        compare(to64(O[b]), ref, BF16_MAX, BF16_MEAN, what=f"O[{b}]")
        compare(to64(lse[b]), rl, LSE_MAX, LSE_MEAN, what=f"lse[{b}]", out_bf16=False)
    assert int(cache.err.item()) == 0


def test_decode_more_splits_than_tiles():
    """Short contexts (1 or 2 tiles each) with 50 splits requested: the splits are capped
    at the tiles of the longest context and the empty ones are skipped by the merge."""
    x, cache, desc = _setup(3, 100, 300, seed=12, gate=True, splits=50)
    O, lse = _run(x, cache, desc)
    for b in range(3):
        ref, rl = _oracle(x, b)
        compare(to64(O[b]), ref, BF16_MAX, BF16_MEAN, what=f"O[{b}]")
        compare(to64(lse[b]), rl, LSE_MAX, LSE_MEAN, what=f"lse[{b}]", out_bf16=False)


def test_decode_1m_config_four_steps_sampled():
    """Long-context decode: 16 sequences at context 1,048,576 (8191 entries + 128 raw
    tokens), 64 heads, head_dim 512, gate on, 4 decode steps; the first step's token
    completes block 8191, whose entry hca_compress writes from the ring. The entry is
    checked against the block mean, and 5 seeded-random sequences (a new draw per step)
    against the oracle at every step (the new entry stays invisible to these queries: it is
    visible from position 1,048,703 on)."""
    dev = torch.device("cuda")
    nseq, ctx0, W, blk, steps = 16, 1048576, 128, 128, 4
    n_ent = (ctx0 - W) // blk  # 8191 visible entries
    x = inputs.decode_inputs(nseq, 64, 1, 512, W, blk, ctx0, ctx0, n_ent + 1, "bf16", seed=21)
    tok = inputs.decode_step_tokens(nseq, 64, 1, 512, steps, "bf16", seed=22, gate=True)
    cache = B.PagedCache(nseq, n_ent + 1, 1, 512, torch.bfloat16, 128,
                         page_table=inputs.page_table(nseq, -(-(n_ent + 1) // 128), 23),
                         device=dev)
    for b in range(nseq):
        cache.fill(b, x.entries_k[b, :n_ent].to(dev), x.entries_v[b, :n_ent].to(dev))
    rk, rv = x.ring_k.to(dev), x.ring_v.to(dev)
    rk_h, rv_h = x.ring_k.clone(), x.ring_v.clone()
    cdesc = B.make_desc(nseq, ctx0, 64, 1, 512)
    O = torch.empty((nseq, 64, 512), dtype=torch.bfloat16, device=dev)
    for s in range(steps):
        p = ctx0 - 1 + s
        q = x.q if s == 0 else tok.q[s]
        desc = B.make_desc(nseq, ctx0 + steps, 64, 1, 512)
        ctx = torch.full((nseq,), p + 1, dtype=torch.int32, device=dev)
        ops.attach_gate(desc, tok.G[s].to(dev))
        if s > 0:
            # step 2: the library's ring update as its own launch; steps 3, 4: inside the
            # decode call; plain indexing for the oracle's copy
            nk, nv = tok.k[s].to(dev).contiguous(), tok.v[s].to(dev).contiguous()
            if s == 1:
                ops.ring_append(desc, nk, nv, ctx, rk, rv)
                ops.decode(desc, q.to(dev), ctx, cache, rk, rv, O=O)
            else:
                ops.decode_append(desc, q.to(dev), ctx, cache, nk, nv, rk, rv, O=O)
            rk_h[:, p % W] = tok.k[s]
            rv_h[:, p % W] = tok.v[s]
        else:
            ops.decode(desc, q.to(dev), ctx, cache, rk, rv, O=O)
        if (p + 1) % blk == 0:
            # the block the token completes: compressed after the step (its entry is not
            # visible to the token's own query)
            B.check(B.hca_compress(cdesc, rk.data_ptr(), rv.data_ptr(), W, p // blk, 1, cache.c,
                                   torch.cuda.current_stream().cuda_stream), "hca_compress")
        torch.cuda.synchronize()
        assert int(cache.err.item()) == 0
        for b in sorted(np.random.default_rng(100 + s).choice(nseq, 5, replace=False)):
            ref, _ = orc.hca_decode(to64(q[b]), to64(x.entries_k[b, :n_ent]),
                                    to64(x.entries_v[b, :n_ent]), to64(rk_h[b]), to64(rv_h[b]),
                                    p + 1, blk, W, default_scale(512), gate=to64(tok.G[s][b]))
            compare(to64(O[b]), ref, BF16_MAX, BF16_MEAN, what=f"step {s} O[{b}]")
        if s == 0:
            # entry 8191 = mean of the ring (tokens 8191*128 .. 1048575), in bf16
            assert int(cache.n_entries[0].item()) == n_ent + 1
            row = cache.entry_rows(0, n_ent + 1)[n_ent]
            got = to64(cache.kc.view(-1, 1, 512)[row])
            want = orc.compress_blocks(to64(rk_h[0]), blk)[0]
            # one bf16 rounding of a float32 mean (sum of 128 bf16 values / 128): <= 1 ulp
            assert (np.abs(got - want) <= bf16_ulp(want)).all(), "entry 8191 (K)"
