"""GPU compression (hca_compress) against the oracle's block means."""

import numpy as np
import pytest
import torch

from compressed_long_context_hca_b200 import binding as B
from compressed_long_context_hca_b200 import inputs, ops
from oracle import hca_oracle as orc
from tests.gpu_helpers import ensure_built, to64

pytestmark = pytest.mark.gpu


def _bf16_ulp(x):
    # spacing of bf16 numbers at |x| (8 significant bits)
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


@pytest.mark.parametrize("dtype,T,b,hkv,D,block,pe", [
    ("bf16", 1024, 1, 1, 512, 128, 128),
    ("bf16", 1000, 2, 1, 512, 128, 256),     # partial last block, 2 sequences
    ("bf16", 300, 3, 2, 64, 16, 8),          # small head_dim, hkv 2, many pages
    ("f32", 1024, 1, 1, 512, 128, 128),
    ("f32", 77, 2, 1, 32, 5, 4),
])
def test_compress_matches_block_means(dtype, T, b, hkv, D, block, pe):
    ensure_built()
    x = inputs.prefill_inputs(b, T, 1, hkv, D, dtype, seed=3, hetero_blocks=True, block=block)
    dev = torch.device("cuda")
    K, V = x.K.to(dev), x.V.to(dev)
    desc = B.make_desc(b, T, hkv, hkv, D, block, 128, None, B.dtype_code(K))
    n = -(-T // block)
    mp = -(-n // pe)
    cache = B.PagedCache(b, n, hkv, D, K.dtype, pe, page_table=inputs.page_table(b, mp),
                         device=dev)
    ops.compress(desc, K, V, cache)
    torch.cuda.synchronize()
    assert cache.n_entries.cpu().tolist() == [n] * b           # ceil(T / block), exact
    assert int(cache.err.item()) == 0
    for bi in range(b):
        rows = cache.entry_rows(bi, n)
        for src, pool in ((x.K, cache.kc), (x.V, cache.vc)):
            ref = orc.compress_blocks(to64(src[bi]), block)
            got = to64(pool.view(-1, hkv, D)[rows])
            if dtype == "bf16":
                # one rounding of an (almost exact) float32 mean: within one bf16 step
                assert np.all(np.abs(got - ref) <= _bf16_ulp(ref) + 1e-30)
            else:
                # float32 summation of up to `block` terms: |error| <= n * 2^-24 * sum|x|
                # (standard bound), divided by n, plus the final division's rounding
                nb = ref.shape[0]
                absx = np.abs(to64(src[bi]))
                sums = np.stack([absx[j * block:(j + 1) * block].sum(0) for j in range(nb)])
                cnt = np.array([min(block, T - j * block) for j in range(nb)], dtype=np.float64)
                bound = (cnt[:, None, None] * 2.0 ** -24 * sums / cnt[:, None, None]
                         + 2.0 ** -23 * np.abs(ref))
                assert np.all(np.abs(got - ref) <= bound)


def test_compress_ranges_and_ring_stride():
    """Block ranges and a batch stride: compressing blocks one by one from a ring of
    `block` slots gives the same entries as one call over the whole sequence."""
    ensure_built()
    T, D, block = 512, 512, 128
    x = inputs.prefill_inputs(2, T, 1, 1, D, "bf16", seed=5)
    dev = torch.device("cuda")
    K, V = x.K.to(dev), x.V.to(dev)
    desc = B.make_desc(2, T, 1, 1, D, block, block)
    full = B.PagedCache(2, 4, 1, D, K.dtype, 128, device=dev)
    ops.compress(desc, K, V, full)
    part = B.PagedCache(2, 4, 1, D, K.dtype, 128, device=dev)
    for j in range(4):
        ring_k = K[:, j * block:(j + 1) * block].contiguous()   # [2, block, 1, D]
        ring_v = V[:, j * block:(j + 1) * block].contiguous()
        st = B.hca_compress(desc, ring_k.data_ptr(), ring_v.data_ptr(), block, j, 1, part.c,
                            torch.cuda.current_stream().cuda_stream)
        assert st == B.HCA_OK
        torch.cuda.synchronize()
        assert part.n_entries.cpu().tolist() == [j + 1, j + 1]
    assert torch.equal(full.kc, part.kc) and torch.equal(full.vc, part.vc)


def test_compress_bad_page_sets_error_bit():
    ensure_built()
    T, D = 256, 512
    x = inputs.prefill_inputs(1, T, 1, 1, D, "bf16", seed=6)
    dev = torch.device("cuda")
    K, V = x.K.to(dev), x.V.to(dev)
    desc = B.make_desc(1, T, 1, 1, D)
    pt = torch.tensor([[0, 99]], dtype=torch.int32)  # page 99 does not exist
    cache = B.PagedCache(1, 256, 1, D, K.dtype, 128, page_table=pt, device=dev)
    cache.c.num_pages = 2
    ops.compress(desc, K, V, cache)
    torch.cuda.synchronize()
    assert int(cache.err.item()) & B.HCA_ERR_PAGE_RANGE == 0  # 2 entries live in page 0
    big = B.make_desc(1, 129 * 128, 1, 1, D)
    Kb = torch.zeros((1, 129 * 128, 1, D), dtype=torch.bfloat16, device=dev)
    ops.compress(big, Kb, Kb, cache, first_block=128, n_blocks=1)
    torch.cuda.synchronize()
    assert int(cache.err.item()) & B.HCA_ERR_PAGE_RANGE
