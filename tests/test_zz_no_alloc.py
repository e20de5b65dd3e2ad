"""hca_attn_decode_noalloc: the decode entry point for callers that cannot lend the library
device memory (their HBM belongs to another allocator, or their decode loop must not call
cudaMalloc/cudaFree, which can synchronise the device). Its split partials live in a fixed
array inside libhca instead of a caller workspace.

Checked through the C ABI against hca_attn_decode (same kernels, caller workspace: the
results must be bit-identical) and against the float64 oracle, on two calls in a row with
different inputs that both use several splits, so both go through the shared array and a
call can't pass by reading the partials the previous call left there. This file is
collected last on purpose.
"""

import pytest
import torch

from compressed_long_context_hca_b200 import binding as B
from compressed_long_context_hca_b200 import inputs, ops
from oracle import hca_oracle as orc
from tests.gpu_helpers import BF16_MAX, BF16_MEAN, compare, default_scale, ensure_built, to64

pytestmark = pytest.mark.gpu


def _case(seed, nseq, lo, hi, gate, splits):
    dev = torch.device("cuda")
    W, block, D, hq = 128, 128, 512, 64
    max_ent = (hi - W) // block + 1
    x = inputs.decode_inputs(nseq, hq, 1, D, W, block, lo, hi, max_ent, "bf16", seed, gate)
    cache = B.PagedCache(nseq, max_ent, 1, D, torch.bfloat16, 128,
                         page_table=inputs.page_table(nseq, -(-max_ent // 128), seed),
                         device=dev)
    for b in range(nseq):
        cache.fill(b, x.entries_k[b].to(dev), x.entries_v[b].to(dev))
    desc = B.make_desc(nseq, hi, hq, 1, D, decode_splits=splits)
    G = None if x.G is None else x.G.to(dev)
    ops.attach_gate(desc, G)
    t = dict(q=x.q.to(dev), ctx=x.ctx_len.to(dev), rk=x.ring_k.to(dev), rv=x.ring_v.to(dev))
    return x, desc, cache, t


def _with_workspace(desc, cache, t):
    O, lse = ops.decode(desc, t["q"], t["ctx"], cache, t["rk"], t["rv"], want_lse=True)
    torch.cuda.synchronize()
    return O, lse


def _no_alloc(desc, cache, t):
    O = torch.empty_like(t["q"])
    lse = torch.empty(t["q"].shape[:2], dtype=torch.float32, device=O.device)
    st = B.hca_attn_decode_noalloc(desc, t["q"].data_ptr(), t["ctx"].data_ptr(), cache.c,
                                   t["rk"].data_ptr(), t["rv"].data_ptr(), O.data_ptr(),
                                   lse.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == B.HCA_OK, B.hca_status_string(st)
    torch.cuda.synchronize()
    return O, lse


def test_no_alloc_decode_matches_workspace_decode_twice():
    ensure_built()
    # Two different workloads back to back, both cut into several splits so that both go
    # through the library's array (with one split a CTA writes O itself and the array is
    # not used): 16 sequences x 6 splits, then 40 sequences x 3 splits.
    cases = [_case(11, 16, 60000, 90000, gate=True, splits=6),
             _case(12, 40, 300, 20000, gate=False, splits=3)]
    for k, (x, desc, cache, t) in enumerate(cases):
        assert B.hca_decode_workspace_bytes(desc) > 0
        O_ref, lse_ref = _with_workspace(desc, cache, t)
        O, lse = _no_alloc(desc, cache, t)
        # the same kernels on the same inputs: bit-identical to the caller-workspace path
        assert torch.equal(O, O_ref), f"call {k}: O differs from the workspace path"
        assert torch.equal(lse, lse_ref), f"call {k}: lse differs from the workspace path"
        assert int(cache.err.item()) == 0
        # and within the bf16 tolerance of the float64 oracle on a few sequences
        for b in (0, len(x.ctx_len) // 2, len(x.ctx_len) - 1):
            G = None if x.G is None else to64(x.G[b])
            ref, _ = orc.hca_decode(to64(x.q[b]), to64(x.entries_k[b]), to64(x.entries_v[b]),
                                    to64(x.ring_k[b]), to64(x.ring_v[b]), int(x.ctx_len[b]),
                                    128, 128, default_scale(512), gate=G)
            compare(to64(O[b]), ref, BF16_MAX, BF16_MEAN, what=f"call {k} O[{b}]")


def test_no_alloc_rejects_oversized_requests():
    ensure_built()
    # 4096 sequences x 8 splits x 64 heads of float32 partials is far past the fixed array
    desc = B.make_desc(4096, 1 << 20, 64, 1, 512, decode_splits=8)
    assert B.hca_decode_workspace_bytes(desc) > B.HCA_DECODE_NOALLOC_SCRATCH_BYTES
    c = B.HcaCache()
    c.kc_pool = c.vc_pool = c.page_table = c.n_entries = 0x1000
    c.page_entries, c.max_pages, c.num_pages = 128, 8192, 8192
    st = B.hca_attn_decode_noalloc(desc, 16, 16, c, 16, 16, 16, 0, 0)
    assert st == B.HCA_ENOSPACE
    # float32 has no workspace-using kernel to stand in for
    d32 = B.make_desc(1, 100, 4, 1, 512, dtype=B.HCA_F32)
    assert B.hca_attn_decode_noalloc(d32, 16, 16, c, 16, 16, 16, 0, 0) == B.HCA_EUNSUPPORTED
