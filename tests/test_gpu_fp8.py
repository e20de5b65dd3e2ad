"""GPU 8-bit (e4m3) compressed cache against the float64 oracle.

* hca_compress into an e4m3 cache: the stored codes equal the oracle's codes of the block
  means, bit for bit, except where the exact mean lies so close to the midpoint between
  two codes that the float32 summation order decides (then either neighbour is accepted,
  and such elements must be rare).
* hca_attn_decode over an e4m3 cache: output and lse against the oracle's decode over
  the dequantised entries value(code) * scale, at the bf16 tolerance, on the batched and
  1M decode configurations and on ragged shapes (window only, few entries, odd head
  counts, short windows, many splits, a gate, a running max that grows at every tile).
* hca_attn_decode_partial / hca_decode_merge and hca_attn_decode_noalloc on the same
  cache against the workspace path.
"""

import numpy as np
import pytest
import torch

from compressed_long_context_hca_b200 import binding as B
from compressed_long_context_hca_b200 import inputs, ops
from oracle import hca_oracle as orc
from tests.gpu_helpers import (BF16_MAX, BF16_MEAN, LSE_MAX, LSE_MEAN, compare, default_scale,
                               ensure_built, to64)

pytestmark = pytest.mark.gpu

K_SCALE, V_SCALE = 0.0625, 0.0625


def _ramp_codes(codes, step_per_tile):
    """Exponent field of tile j's codes raised by j * step (capped at 14, zero and
    subnormal codes kept): the keys double per tile, so the running max grows."""
    c = codes.to(torch.int32)
    sign, mag = c & 0x80, c & 0x7F
    e, m = mag >> 3, mag & 7
    j = (torch.arange(c.shape[0], dtype=torch.int32) // 128).view(-1, *([1] * (c.dim() - 1)))
    e2 = torch.where(e > 0, torch.clamp(e + step_per_tile * j, max=14), e)
    return (sign | (e2 << 3) | m).to(torch.uint8)


def _setup8(nseq, ctx_lo, ctx_hi, gate=False, seed=0, hq=64, W=128, block=128, splits=0,
            pe=128, ramp=False):
    ensure_built()
    dev = torch.device("cuda")
    D = 512
    max_ent = max(1, (ctx_hi - W) // block + 1)
    x = inputs.decode_inputs_e4m3(nseq, hq, 1, D, W, block, ctx_lo, ctx_hi, max_ent, seed, gate)
    if ramp:
        for b in range(nseq):
            x.entries_k[b] = _ramp_codes(x.entries_k[b] & 0xBF, 1)  # base values <= 1.875
    mp = -(-max_ent // pe)
    cache = B.PagedCache(nseq, max_ent, 1, D, torch.bfloat16, pe,
                         page_table=inputs.page_table(nseq, mp), device=dev,
                         e4m3_scales=(K_SCALE, V_SCALE))
    for b in range(nseq):
        cache.fill(b, x.entries_k[b].to(dev), x.entries_v[b].to(dev))
    desc = B.make_desc(nseq, ctx_hi, hq, 1, D, block, W, None, B.HCA_BF16, splits)
    ops.attach_gate(desc, None if x.G is None else x.G.to(dev))
    return x, cache, desc


def _run(x, cache, desc):
    dev = torch.device("cuda")
    O, lse = ops.decode(desc, x.q.to(dev), x.ctx_len.to(dev), cache, x.ring_k.to(dev),
                        x.ring_v.to(dev), want_lse=True)
    torch.cuda.synchronize()
    return O, lse


def _oracle(x, b, block=128, W=128):
    G = None if x.G is None else to64(x.G[b])
    Kc = orc.e4m3_dequantize(x.entries_k[b].numpy(), K_SCALE)
    Vc = orc.e4m3_dequantize(x.entries_v[b].numpy(), V_SCALE)
    return orc.hca_decode(to64(x.q[b]), Kc, Vc, to64(x.ring_k[b]), to64(x.ring_v[b]),
                          int(x.ctx_len[b]), block, W, default_scale(512), gate=G)


def _check(x, O, lse, seqs, W=128, what=""):
    for b in seqs:
        ref, rl = _oracle(x, b, W=W)
        compare(to64(O[b]), ref, BF16_MAX, BF16_MEAN, what=f"{what} O[{b}]")
        compare(to64(lse[b]), rl, LSE_MAX, LSE_MEAN, what=f"{what} lse[{b}]", out_bf16=False)


# ------------------------------------------------------------------------- compress
def _midpoint_slack(tokens, block, scale):
    """Per entry element: how far the float32 mean may sit from the exact mean, in stored
    units (float32 summation of n terms: n * 2^-24 * sum|x| / n, plus the division)."""
    T = tokens.shape[0]
    n = -(-T // block)
    out = []
    for j in range(n):
        seg = tokens[j * block:min((j + 1) * block, T)]
        out.append((seg.shape[0] + 2) * 2.0 ** -24 * np.abs(seg).sum(0) / seg.shape[0])
    return np.stack(out) / np.float32(scale)


def _assert_codes(got, want, tokens, block, scale, what):
    got = np.asarray(got, np.uint8)
    want = np.asarray(want, np.uint8)
    diff = got != want
    if diff.any():
        # allowed only next to a rounding midpoint of the exact mean
        y = orc.compress_blocks(tokens, block) / np.float64(np.float32(scale))
        gv = orc.e4m3_value(got)
        wv = orc.e4m3_value(want)
        mid = (gv + wv) / 2.0
        slack = _midpoint_slack(tokens, block, scale)
        adjacent = np.abs(got.astype(int) - want.astype(int)) == 1
        near = np.abs(y - mid) <= slack + 2.0 ** -24 * np.abs(y)
        bad = diff & ~(adjacent & near)
        assert not bad.any(), f"{what}: {int(bad.sum())} codes differ away from a midpoint"
        assert diff.mean() < 1e-4, f"{what}: too many midpoint cases ({int(diff.sum())})"


@pytest.mark.parametrize("dtype,T,nseq", [("bf16", 1000, 3), ("bf16", 128 * 40, 2),
                                          ("f32", 777, 2)])
def test_compress_e4m3_codes(dtype, T, nseq):
    """Block means of N(0,1) tokens (partial last block, shuffled pages) stored as e4m3 codes
    with scales 1/64 (K) and 0.0137 (V, not a power of two)."""
    ensure_built()
    dev = torch.device("cuda")
    x = inputs.prefill_inputs(nseq, T, 8, 1, 512, dtype, seed=31)
    K, V = x.K.to(dev), x.V.to(dev)
    n_ent = -(-T // 128)
    ks, vs = 1.0 / 64, 0.0137
    cache = B.PagedCache(nseq, n_ent, 1, 512, K.dtype, 128,
                         page_table=inputs.page_table(nseq, -(-n_ent // 128), 32), device=dev,
                         e4m3_scales=(ks, vs))
    desc = B.make_desc(nseq, T, 8, 1, 512, 128, 128, None,
                       B.HCA_BF16 if dtype == "bf16" else B.HCA_F32)
    ops.compress(desc, K, V, cache)
    torch.cuda.synchronize()
    assert int(cache.err.item()) == 0
    for b in range(nseq):
        assert int(cache.n_entries[b].item()) == n_ent
        rows = torch.tensor(cache.entry_rows(b, n_ent), device=dev)
        for pool, src, sc, name in ((cache.kc, x.K, ks, "K"), (cache.vc, x.V, vs, "V")):
            got = pool.view(-1, 1, 512)[rows].cpu().numpy()
            tok = to64(src[b])
            want = orc.compress_blocks_e4m3(tok, 128, sc)
            _assert_codes(got, want, tok, 128, sc, f"{dtype} T={T} b={b} {name}")


def test_compress_e4m3_saturates_and_keeps_sign():
    """Means beyond 448 * scale store the largest code (0x7e / 0xfe); tiny means round to
    zero or subnormal codes, with their sign."""
    ensure_built()
    dev = torch.device("cuda")
    T = 256
    K = torch.zeros((1, T, 1, 512), dtype=torch.float32)
    K[0, :128, 0, 0] = 1e4          # block 0 column 0: mean 1e4 -> saturates
    K[0, :128, 0, 1] = -1e4
    K[0, 128:, 0, 2] = 2.0 ** -10   # block 1 column 2: mean 2^-10, a tie between 0 and
    #                                 the smallest subnormal 2^-9: the even code 0
    K[0, 128:, 0, 3] = -3 * 2.0 ** -10  # -3 * 2^-10: a tie between codes 1 and 2 -> 2
    V = K.clone()
    cache = B.PagedCache(1, 2, 1, 512, torch.float32, 128, device=dev, e4m3_scales=(1.0, 1.0))
    desc = B.make_desc(1, T, 8, 1, 512, 128, 128, None, B.HCA_F32)
    ops.compress(desc, K.to(dev), V.to(dev), cache)
    torch.cuda.synchronize()
    got = cache.kc.view(-1, 512)[:2].cpu().numpy()
    want = orc.compress_blocks_e4m3(K[0].numpy(), 128, 1.0)[:, 0]
    assert np.array_equal(got, want)
    assert got[0, 0] == 0x7E and got[0, 1] == 0xFE and got[1, 2] == 0 and got[1, 3] == 0x82


# --------------------------------------------------------------------------- decode
@pytest.mark.parametrize("nseq,lo,hi,gate,hq,W", [
    (4, 1, 127, False, 64, 128),         # window only (no compressed entry)
    (6, 128, 700, True, 64, 128),        # 0..4 entries, partial tiles
    (8, 8192, 40000, False, 64, 128),    # many tiles, several splits
    (3, 9000, 40000, True, 33, 128),     # odd head count
    (3, 5000, 30000, False, 5, 64),      # short window (ring tile of 64 keys)
    (2, 3000, 12000, True, 1, 100),      # one head, window not a multiple of 16
])
def test_decode_e4m3(nseq, lo, hi, gate, hq, W):
    x, cache, desc = _setup8(nseq, lo, hi, gate=gate, hq=hq, W=W, seed=40 + nseq + hq)
    O, lse = _run(x, cache, desc)
    _check(x, O, lse, range(nseq), W=W)
    assert int(cache.err.item()) == 0


@pytest.mark.parametrize("ctx,splits", [
    (128 * 80 + 5, 0),            # one compressed tile of 80 entries
    (128 * (256 + 48) + 100, 0),  # last tile of 48 entries
    (128 * (384 + 16) + 127, 2),  # last tile of 16, two splits
    (128 * (128 + 112) + 64, 1),  # last tile of 112, one split
])
def test_decode_e4m3_tile_ends_mid_piece(ctx, splits):
    """The last compressed tile holds 16 * odd entries, all visible: the columns of its
    last 32-column score piece past the tile must enter neither P nor the row sum."""
    x, cache, desc = _setup8(2, ctx, ctx, seed=70 + splits, splits=splits)
    O, lse = _run(x, cache, desc)
    _check(x, O, lse, range(2), what=f"ctx={ctx}")
    assert int(cache.err.item()) == 0


@pytest.mark.parametrize("nseq,lo,hi", [(6, 1, 127), (8, 8192, 40000)])
def test_decode_e4m3_append_equals_append_then_decode(nseq, lo, hi):
    """On the 8-bit cache too, the in-kernel ring update matches hca_ring_append followed by
    hca_attn_decode byte for byte."""
    x, cache, desc = _setup8(nseq, lo, hi, seed=90 + nseq, gate=True)
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(91)
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


def _sample_sequences(ctx_len, n, seed):
    lens = ctx_len.numpy()
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(len(lens), size=n, replace=False).tolist())
    pick |= {int(np.argmax(lens)), int(np.argmin(lens))}
    return sorted(pick)


def test_decode_e4m3_batched_config_sampled():
    """128 sequences with context lengths uniform in [8192, 131072], 64 heads, head_dim 512,
    e4m3 cache + last 128 raw tokens; 24 seeded-random sequences plus the longest and the
    shortest against the oracle."""
    x, cache, desc = _setup8(128, 8192, 131072, seed=50)
    O, lse = _run(x, cache, desc)
    _check(x, O, lse, _sample_sequences(x.ctx_len, 24, seed=51))
    assert int(cache.err.item()) == 0


@pytest.mark.parametrize("splits", [1, 2, 3, 7, 40, 0])
def test_decode_e4m3_split_invariance(splits):
    x, cache, desc = _setup8(5, 20000, 60000, seed=52, splits=splits, gate=True)
    O, lse = _run(x, cache, desc)
    _check(x, O, lse, range(5), what=f"splits={splits}")


def test_decode_e4m3_running_max_grows():
    """Keys that double tile by tile: the row max moves past the lazy rescale threshold
    again and again, and O is rescaled in tensor memory between tiles; nearly one-hot
    softmax (P enters P.V as an f16 pair)."""
    x, cache, desc = _setup8(2, 100000, 110000, seed=53, splits=1, ramp=True)
    O, lse = _run(x, cache, desc)
    _check(x, O, lse, range(2))


def test_decode_e4m3_partial_merge_and_noalloc():
    """The entry range split over two partials (entries [0, 256) and [256, end) with the
    window) merged, and the no-allocation entry point, against the workspace path."""
    x, cache, desc = _setup8(4, 30000, 90000, seed=54, gate=True)
    dev = torch.device("cuda")
    q, ctx = x.q.to(dev), x.ctx_len.to(dev)
    rk, rv = x.ring_k.to(dev), x.ring_v.to(dev)
    O_ws, _ = ops.decode(desc, q, ctx, cache, rk, rv)
    parts = ops.decode_partial_buffer(desc, 2)
    stride = ops.partial_stride(desc)
    ops.decode_partial(desc, q, ctx, cache, rk, rv, 0, 256, False, parts[0])
    ops.decode_partial(desc, q, ctx, cache, rk, rv, 256, 1 << 30, True, parts[1])
    O_m = torch.empty_like(O_ws)
    ops.decode_merge(desc, parts, O_m)
    O_na = torch.empty_like(O_ws)
    B.check(B.hca_attn_decode_noalloc(desc, q.data_ptr(), ctx.data_ptr(), cache.c,
                                      rk.data_ptr(), rv.data_ptr(), O_na.data_ptr(), 0,
                                      torch.cuda.current_stream().cuda_stream), "noalloc")
    torch.cuda.synchronize()
    assert torch.equal(O_na, O_ws)
    for b in range(4):
        ref, _ = _oracle(x, b)
        compare(to64(O_m[b]), ref, BF16_MAX, BF16_MEAN, what=f"merged O[{b}]")
        compare(to64(O_ws[b]), ref, BF16_MAX, BF16_MEAN, what=f"O[{b}]")
    assert int(cache.err.item()) == 0


def test_decode_e4m3_1m_config_sampled():
    """Long-context decode over an e4m3 cache: 16 sequences at context 1,048,576 (8191
    entries + 128 raw tokens), 64 heads, gate on; 5 seeded-random sequences against the
    oracle."""
    x, cache, desc = _setup8(16, 1048576, 1048576, gate=True, seed=55)
    O, lse = _run(x, cache, desc)
    rng = np.random.default_rng(56)
    _check(x, O, lse, sorted(rng.choice(16, 5, replace=False)))
    assert int(cache.err.item()) == 0


def test_decode_e4m3_subnormal_values():
    """Values whose codes are all e4m3 subnormals (exponent field 0) with a large scale:
    the widened values are f16 subnormals on their way through P.V, and must count. Keys
    all zero, so every visible key gets the same weight and O is the mean value."""
    ensure_built()
    dev = torch.device("cuda")
    nseq, ctx, W, D = 3, 20000, 128, 512
    n_ent = (ctx - W) // 128
    g = torch.Generator()
    g.manual_seed(57)
    ek = torch.zeros((nseq, n_ent, 1, D), dtype=torch.uint8)
    ev = torch.randint(1, 8, (nseq, n_ent, 1, D), generator=g).to(torch.uint8)
    q = torch.randn((nseq, 64, D), generator=g).to(torch.bfloat16)
    rk = torch.zeros((nseq, W, 1, D), dtype=torch.bfloat16)
    rv = torch.zeros((nseq, W, 1, D), dtype=torch.bfloat16)
    vs = 64.0  # values m / 8 (m = 1..7): outputs near 0.5, where bf16 rounds finely
    cache = B.PagedCache(nseq, n_ent, 1, D, torch.bfloat16, 128,
                         page_table=inputs.page_table(nseq, -(-n_ent // 128)), device=dev,
                         e4m3_scales=(1.0, vs))
    for b in range(nseq):
        cache.fill(b, ek[b].to(dev), ev[b].to(dev))
    desc = B.make_desc(nseq, ctx, 64, 1, D, 128, W, None, B.HCA_BF16, 0)
    ctxl = torch.full((nseq,), ctx, dtype=torch.int32)
    O, _ = ops.decode(desc, q.to(dev), ctxl.to(dev), cache, rk.to(dev), rv.to(dev))
    torch.cuda.synchronize()
    for b in range(nseq):
        ref, _ = orc.hca_decode(to64(q[b]), orc.e4m3_dequantize(ek[b].numpy(), 1.0),
                                orc.e4m3_dequantize(ev[b].numpy(), vs), to64(rk[b]),
                                to64(rv[b]), ctx, 128, W, default_scale(D))
        assert ref.mean() > 0.25  # the subnormal values carry the output (0 if flushed)
        compare(to64(O[b]), ref, BF16_MAX, BF16_MEAN, what=f"O[{b}]")
