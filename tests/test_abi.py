"""Host-side checks of the C ABI (CPU only: no kernel is launched).

The library must load, export every symbol include/hca.h declares, agree with the
binding on struct layouts, and reject bad arguments before touching the GPU.
"""

import ctypes
import os
import re

import pytest

from compressed_long_context_hca_b200 import binding as B
from compressed_long_context_hca_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hca.h")


@pytest.fixture(scope="module")
def L():
    build_mod.build()
    return B.lib()


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\**\s+\**(hca_[a-z_0-9]+)\s*\(", src, re.M)
    return sorted(set(names))


def test_header_declares_binding_names():
    assert _declared_functions() == sorted(B.EXPORTED)


def test_library_exports_every_declared_symbol(L):
    for name in _declared_functions():
        assert hasattr(L, name), name
    out = os.popen(f"nm -D --defined-only {B.LIB_PATH}").read()
    for name in _declared_functions():
        assert re.search(rf"\bT {name}\b", out), name


def test_abi_version_and_strings(L):
    assert B.hca_abi_version() == B.ABI_VERSION
    for code in (0, -1, -2, -3, -4):
        assert B.hca_status_string(code).startswith("HCA_")
    assert "unknown" in B.hca_status_string(7)


def test_struct_layouts_match_header():
    # offsets follow the C rules for the field order in hca.h
    assert ctypes.sizeof(B.HcaDesc) == 72
    assert B.HcaDesc.gate.offset == 40
    assert B.HcaDesc.gate_strides.offset == 48
    assert ctypes.sizeof(B.HcaCache) == 72
    assert B.HcaCache.err_word.offset == 48
    assert B.HcaCache.pool_format.offset == 56
    assert B.HcaCache.k_scale.offset == 60 and B.HcaCache.v_scale.offset == 64


def test_struct_layouts_match_c_compiler(tmp_path):
    # the C compiler's own offsets for the header, against the ctypes mirror
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stddef.h>\n#include <stdio.h>\n#include "hca.h"\n'
        "int main(void) {\n"
        '  printf("%zu %zu %zu %zu\\n", sizeof(hca_desc), offsetof(hca_desc, gate),\n'
        "         offsetof(hca_desc, gate_strides), offsetof(hca_desc, decode_splits));\n"
        '  printf("%zu %zu %zu %zu %zu\\n", sizeof(hca_cache), offsetof(hca_cache, err_word),\n'
        "         offsetof(hca_cache, pool_format), offsetof(hca_cache, k_scale),\n"
        "         offsetof(hca_cache, v_scale));\n"
        "  return 0;\n}\n")
    exe = tmp_path / "layout"
    rc = os.system(f"gcc -I {os.path.join(ROOT, 'include')} -o {exe} {src}")
    assert rc == 0
    lines = os.popen(str(exe)).read().split("\n")
    d = [int(x) for x in lines[0].split()]
    c = [int(x) for x in lines[1].split()]
    assert d == [ctypes.sizeof(B.HcaDesc), B.HcaDesc.gate.offset, B.HcaDesc.gate_strides.offset,
                 B.HcaDesc.decode_splits.offset]
    assert c == [ctypes.sizeof(B.HcaCache), B.HcaCache.err_word.offset,
                 B.HcaCache.pool_format.offset, B.HcaCache.k_scale.offset,
                 B.HcaCache.v_scale.offset]


def _cache():
    c = B.HcaCache()
    c.kc_pool = c.vc_pool = c.page_table = c.n_entries = 0x1000
    c.page_entries, c.max_pages, c.num_pages = 128, 4, 4
    return c


def test_validation_rejects_before_launch(L):
    d = B.make_desc(1, 256, 64, 1, 512)
    c = _cache()
    # NULL descriptor / cache / tensors
    assert L.hca_compress(None, 1, 1, 0, 0, 1, ctypes.byref(c), None) == B.HCA_EINVAL
    assert B.hca_compress(d, 0, 0, 256, 0, 1, c) == B.HCA_EINVAL
    assert B.hca_attn_prefill(d, 0, 0, 0, c, 0) == B.HCA_EINVAL
    # hq not a multiple of hkv
    bad = B.make_desc(1, 256, 6, 4, 512)
    assert B.hca_attn_prefill(bad, 16, 16, 16, c, 16) == B.HCA_EINVAL
    # negative sizes
    neg = B.make_desc(1, -1, 64, 1, 512)
    assert B.hca_attn_prefill(neg, 16, 16, 16, c, 16) == B.HCA_EINVAL
    # unsupported dtype code
    d2 = B.make_desc(1, 256, 64, 1, 512, dtype=7)
    assert B.hca_attn_prefill(d2, 16, 16, 16, c, 16) == B.HCA_EUNSUPPORTED
    # bf16 tensor path needs head_dim 512 and hkv 1
    d3 = B.make_desc(1, 256, 64, 1, 256)
    assert B.hca_attn_prefill(d3, 16, 16, 16, c, 16) == B.HCA_EUNSUPPORTED
    d4 = B.make_desc(1, 256, 64, 2, 512)
    assert B.hca_attn_prefill(d4, 16, 16, 16, c, 16) == B.HCA_EUNSUPPORTED
    # window above what the tensor-core tiles cover
    d5 = B.make_desc(1, 256, 64, 1, 512, window=200)
    assert B.hca_attn_prefill(d5, 16, 16, 16, c, 16) == B.HCA_EUNSUPPORTED
    # page size not a multiple of 128 for the bf16 kernels
    c2 = _cache()
    c2.page_entries = 64
    assert B.hca_attn_prefill(d, 16, 16, 16, c2, 16) == B.HCA_EUNSUPPORTED
    # f32 path: head_dim must be a multiple of 32, <= 512
    d6 = B.make_desc(1, 256, 4, 1, 520, dtype=B.HCA_F32)
    assert B.hca_attn_prefill(d6, 16, 16, 16, c, 16) == B.HCA_EUNSUPPORTED
    # misaligned pointer
    assert B.hca_attn_prefill(d, 16 + 2, 16, 16, c, 16) == B.HCA_EINVAL
    # 32-bit row coordinates of the tensor-core kernels: batch * seqlen * hq and the pool's
    # rows must stay below 2^31
    big = B.make_desc(64, 1 << 20, 64, 1, 512)
    assert B.hca_attn_prefill(big, 16, 16, 16, c, 16) == B.HCA_EUNSUPPORTED
    c3 = _cache()
    c3.page_entries, c3.num_pages = 1 << 16, 1 << 15
    assert B.hca_attn_prefill(d, 16, 16, 16, c3, 16) == B.HCA_EUNSUPPORTED
    dd = B.make_desc(1, 1000, 64, 1, 512)
    assert B.hca_attn_decode(dd, 16, 16, c3, 16, 16, 16, 0, 16, 1 << 30) == B.HCA_EUNSUPPORTED


def test_compress_space_and_range_checks(L):
    d = B.make_desc(2, 1000, 64, 1, 512)
    c = _cache()  # 4 pages x 128 entries
    # blocks past the sequence
    assert B.hca_compress(d, 16, 16, 1000, 7, 2, c) == B.HCA_EINVAL
    # more entries than the page table can address
    c.max_pages = 0
    assert B.hca_compress(d, 16, 16, 1000, 0, 1, c) == B.HCA_EINVAL
    c.max_pages = 1
    c.page_entries = 4
    assert B.hca_compress(d, 16, 16, 1000, 0, 7, c) == B.HCA_ENOSPACE
    # zero blocks / empty batch: nothing to do
    assert B.hca_compress(d, 16, 16, 1000, 0, 0, c) == B.HCA_OK
    assert B.hca_compress(B.make_desc(0, 1000, 64, 1, 512), 16, 16, 1000, 0, 1, c) == B.HCA_OK


def test_decode_workspace_and_space(L):
    d = B.make_desc(16, 1 << 20, 64, 1, 512, decode_splits=9)
    n = B.hca_decode_workspace_bytes(d)
    assert n == 16 * 9 * 64 * (512 + 2) * 4
    # 1M context: 8191 entries -> 64 tiles of 128 + the ring tile = 65 tiles; more splits
    # than tiles are capped at one tile each
    d.decode_splits = 100
    assert B.hca_decode_workspace_bytes(d) == 16 * 65 * 64 * (512 + 2) * 4
    d.decode_splits = 9
    assert B.hca_decode_workspace_bytes(B.make_desc(1, 1, 64, 1, 512, dtype=B.HCA_F32)) == 0
    # one split of 3 heads: 6 floats of (max, sum) padded to 8 so the float4 partials of O
    # start 16-byte aligned
    assert B.hca_decode_workspace_bytes(B.make_desc(1, 100, 3, 1, 512)) == (8 + 3 * 512) * 4
    c = _cache()
    st = B.hca_attn_decode(d, 16, 16, c, 16, 16, 16, 0, 16, n - 1)
    assert st == B.HCA_ENOSPACE


def test_e4m3_cache_validation(L):
    d = B.make_desc(1, 1000, 64, 1, 512)
    c = _cache()
    c.pool_format = B.HCA_POOL_E4M3
    # scales must be finite and positive
    for ks, vs in ((0.0, 1.0), (1.0, -1.0), (float("inf"), 1.0), (1.0, float("nan"))):
        c.k_scale, c.v_scale = ks, vs
        assert B.hca_compress(d, 16, 16, 1000, 0, 1, c) == B.HCA_EINVAL
        assert B.hca_attn_decode(d, 16, 16, c, 16, 16, 16, 0, 16, 1 << 30) == B.HCA_EINVAL
    c.k_scale, c.v_scale = 0.01, 0.02
    # the 8-bit cache serves decode: prefill and its backward have no kernel for it
    assert B.hca_attn_prefill(d, 16, 16, 16, c, 16) == B.HCA_EUNSUPPORTED
    assert B.hca_attn_prefill_backward(d, 16, 16, 16, c, 16, 16, 16, 16, 16, 0, 16,
                                  1 << 30) == B.HCA_EUNSUPPORTED
    # nor does the float32 decode
    df = B.make_desc(1, 1000, 4, 1, 512, dtype=B.HCA_F32)
    assert B.hca_attn_decode(df, 16, 16, c, 16, 16, 16, 0, 16, 1 << 30) == B.HCA_EUNSUPPORTED
    # an unknown pool format
    c.pool_format = 5
    assert B.hca_attn_decode(d, 16, 16, c, 16, 16, 16, 0, 16, 1 << 30) == B.HCA_EINVAL


def test_ring_append_validation(L):
    """hca_ring_append rejects what it cannot launch, before any device work."""
    d = B.make_desc(2, 1000, 64, 1, 512)
    # NULL pointers
    assert B.hca_ring_append(d, 0, 16, 16, 16, 16) == B.HCA_EINVAL
    assert B.hca_ring_append(d, 16, 16, 0, 16, 16) == B.HCA_EINVAL
    # every row pointer 16-byte aligned
    assert B.hca_ring_append(d, 16, 16, 16, 24, 16) == B.HCA_EINVAL
    assert B.hca_ring_append(d, 16, 18, 16, 16, 16) == B.HCA_EINVAL
    # rows of hkv * head_dim elements whose size is not a multiple of 16 bytes
    odd = B.make_desc(2, 1000, 4, 1, 12)
    assert B.hca_ring_append(odd, 16, 16, 16, 16, 16) == B.HCA_EUNSUPPORTED
    # an empty batch is a no-op
    assert B.hca_ring_append(B.make_desc(0, 1000, 64, 1, 512), 0, 0, 0, 0, 0) == B.HCA_OK
    # the decode call with the ring update: the new rows are required and 16-byte aligned
    c = _cache()
    args = (16, 16, c)
    assert B.hca_attn_decode_append(d, *args, 0, 16, 16, 16, 16, 0, 16, 1 << 30) == B.HCA_EINVAL
    assert B.hca_attn_decode_append(d, *args, 16, 8, 16, 16, 16, 0, 16, 1 << 30) == B.HCA_EINVAL


def test_set_gate(L):
    d = B.make_desc(1, 8, 64, 1, 512)
    assert B.hca_set_gate(d, 0x2000, (1, 2, 3)) == B.HCA_OK
    assert d.gate == 0x2000 and list(d.gate_strides) == [1, 2, 3]
    assert B.hca_set_gate(d, 0x2000, None) == B.HCA_EINVAL
    assert B.hca_set_gate(d, 0, None) == B.HCA_OK
    assert not d.gate and list(d.gate_strides) == [0, 0, 0]


def test_product_path_has_no_oracle_import():
    # the package must never import the oracle (test infrastructure only)
    pkg = os.path.join(ROOT, "compressed_long_context_hca_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                txt = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", txt, re.M), f
                assert "hca_oracle" not in txt, f


def test_range_partial_and_merge_validation(L):
    """The query/key range of hca_attn_prefill_range, the key part of
    hca_attn_decode_partial and the part list of hca_decode_merge are checked before any
    launch."""
    d = B.make_desc(1, 256, 64, 1, 512)
    c = _cache()
    # K/V rows must cover every window: kv_pos0 <= max(0, q_pos0 - W + 1) ...
    assert B.hca_attn_prefill_range(d, 1000, 1000 - 126, 500, 16, 16, 16, c, 16) == B.HCA_EINVAL
    # ... and kv_pos0 + kv_len >= q_pos0 + seqlen
    assert B.hca_attn_prefill_range(d, 1000, 873, 382, 16, 16, 16, c, 16) == B.HCA_EINVAL
    assert B.hca_attn_prefill_range(d, -1, 0, 256, 16, 16, 16, c, 16) == B.HCA_EINVAL
    # decode part: entry_begin a multiple of 128, entry_end >= entry_begin
    dd = B.make_desc(2, 5000, 64, 1, 512)
    assert B.hca_attn_decode_partial(dd, 16, 16, c, 16, 16, 64, 256, 1, 16, 16,
                                     1 << 20) == B.HCA_EINVAL
    assert B.hca_attn_decode_partial(dd, 16, 16, c, 16, 16, 256, 128, 1, 16, 16,
                                     1 << 20) == B.HCA_EINVAL
    assert B.hca_attn_decode_partial(dd, 16, 16, c, 16, 16, 0, 128, 1, 0, 16,
                                     1 << 20) == B.HCA_EINVAL
    d32 = B.make_desc(2, 5000, 4, 1, 512, dtype=B.HCA_F32)
    assert B.hca_attn_decode_partial(d32, 16, 16, c, 16, 16, 0, 128, 1, 16, 16,
                                     1 << 20) == B.HCA_EUNSUPPORTED
    assert B.hca_decode_partial_bytes(d32) == 0
    # partial size: (m, l) padded to 4 floats, then the float32 rows
    pb = B.hca_decode_partial_bytes(dd)
    assert pb == (((2 * 64 * 2 + 3) // 4 * 4) + 2 * 64 * 512) * 4
    # merge: at least one part, stride >= the partial size and a multiple of 16
    assert B.hca_decode_merge(dd, 16, 0, pb, 16) == B.HCA_EINVAL
    assert B.hca_decode_merge(dd, 16, 2, pb - 16, 16) == B.HCA_EINVAL
    assert B.hca_decode_merge(dd, 16, 2, pb + 8, 16) == B.HCA_EINVAL
    assert B.hca_decode_merge(dd, 0, 2, pb, 16) == B.HCA_EINVAL
    assert B.hca_decode_merge(d32, 16, 2, pb, 16) == B.HCA_EUNSUPPORTED


def test_backward_validation(L):
    d32 = B.make_desc(1, 256, 4, 1, 512, dtype=B.HCA_F32)
    # CUDA-core path: Delta (padded to 4 floats) + dKc and dVc of 2 entries
    assert B.hca_prefill_backward_workspace_bytes(d32) == ((256 * 4 + 3) // 4 * 4 +
                                                           2 * 2 * 512) * 4
    d = B.make_desc(1, 256, 64, 1, 512)
    c = _cache()
    ws = B.hca_prefill_backward_workspace_bytes(d)
    # tensor-core path: at least the float32 window rows of dK, dV and the group's dQ rows
    assert ws >= (2 * 256 * 512 + 256 * 64 * 512) * 4
    q, k, v, lse, do, dq, dk, dv = [16] * 8
    call = lambda desc, dg, w, wb: B.hca_attn_prefill_backward(  # noqa: E731
        desc, q, k, v, c, lse, do, dq, dk, dv, dg, w, wb)
    assert B.hca_attn_prefill_backward(d, q, k, v, c, 0, do, dq, dk, dv, 0, 16,
                                       ws) == B.HCA_EINVAL          # no lse
    assert call(d, 16, 16, ws) == B.HCA_EINVAL                      # dG without a gate
    assert call(d, 0, 16, ws - 16) == B.HCA_ENOSPACE
    assert call(d, 0, 8, ws) == B.HCA_EINVAL                        # misaligned workspace
    assert call(B.make_desc(1, 256, 64, 1, 520), 0, 16, 1 << 30) == B.HCA_EUNSUPPORTED
