"""ctypes binding of libhca (include/hca.h): argument marshalling only.

Every entry point of the C ABI appears here under the same name and takes the same
arguments, with device pointers passed as Python ints (0 = NULL) and streams as ints
(``torch.cuda.current_stream().cuda_stream``). The helpers at the bottom build the
structs from torch tensors; torch provides device memory and streams, nothing else.
If libhca.so cannot be loaded, every call raises: there is no fallback path.
"""

from __future__ import annotations

import ctypes
import math
import os
from ctypes import POINTER, c_char_p, c_float, c_int32, c_int64, c_size_t, c_void_p
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhca.so")

HCA_OK = 0
HCA_EINVAL = -1
HCA_EUNSUPPORTED = -2
HCA_ENOSPACE = -3
HCA_ECUDA = -4
HCA_BF16 = 0
HCA_F32 = 1
HCA_POOL_NATIVE = 0
HCA_POOL_E4M3 = 1
HCA_ERR_PAGE_RANGE = 1
HCA_ERR_CACHE_SHORT = 2
HCA_ERR_TIMEOUT = 4
HCA_ERR_CTX_RANGE = 8
ABI_VERSION = 2

EXPORTED = ("hca_abi_version", "hca_status_string", "hca_set_gate", "hca_compress",
            "hca_attn_prefill", "hca_attn_prefill_range", "hca_decode_workspace_bytes",
            "hca_attn_decode", "hca_decode_partial_bytes", "hca_attn_decode_partial",
            "hca_decode_merge", "hca_prefill_backward_workspace_bytes",
            "hca_attn_prefill_backward", "hca_gate_from_latent", "hca_vha_gate",
            "hca_attn_decode_noalloc", "hca_ring_append", "hca_attn_decode_append")
HCA_DECODE_NOALLOC_SCRATCH_BYTES = 64 << 20


class HcaDesc(ctypes.Structure):
    _fields_ = [("batch", c_int32), ("seqlen", c_int32), ("hq", c_int32), ("hkv", c_int32),
                ("head_dim", c_int32), ("block", c_int32), ("window", c_int32),
                ("scale", c_float), ("dtype", c_int32), ("decode_splits", c_int32),
                ("gate", c_void_p), ("gate_strides", c_int64 * 3)]


class HcaCache(ctypes.Structure):
    _fields_ = [("kc_pool", c_void_p), ("vc_pool", c_void_p), ("page_table", c_void_p),
                ("n_entries", c_void_p), ("page_entries", c_int32), ("max_pages", c_int32),
                ("num_pages", c_int32), ("err_word", c_void_p), ("pool_format", c_int32),
                ("k_scale", c_float), ("v_scale", c_float)]


class HcaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load libhca.so (built by ``build.py``); raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libhca.so not built ({LIB_PATH}); run "
                           "`python -m compressed_long_context_hca_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    L.hca_abi_version.restype = c_int32
    L.hca_abi_version.argtypes = []
    L.hca_status_string.restype = c_char_p
    L.hca_status_string.argtypes = [c_int32]
    L.hca_set_gate.restype = c_int32
    L.hca_set_gate.argtypes = [POINTER(HcaDesc), c_void_p, c_void_p]
    L.hca_compress.restype = c_int32
    L.hca_compress.argtypes = [POINTER(HcaDesc), c_void_p, c_void_p, c_int64, c_int32, c_int32,
                               POINTER(HcaCache), c_void_p]
    L.hca_attn_decode_append.restype = c_int32
    L.hca_attn_decode_append.argtypes = [POINTER(HcaDesc), c_void_p, c_void_p, POINTER(HcaCache),
                                         c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                         c_void_p, c_void_p, c_size_t, c_void_p]
    L.hca_ring_append.restype = c_int32
    L.hca_ring_append.argtypes = [POINTER(HcaDesc), c_void_p, c_void_p, c_void_p, c_void_p,
                                  c_void_p, c_void_p]
    L.hca_attn_prefill.restype = c_int32
    L.hca_attn_prefill.argtypes = [POINTER(HcaDesc), c_void_p, c_void_p, c_void_p,
                                   POINTER(HcaCache), c_void_p, c_void_p, c_void_p, c_void_p]
    L.hca_attn_prefill_range.restype = c_int32
    L.hca_attn_prefill_range.argtypes = [POINTER(HcaDesc), c_int32, c_int32, c_int32, c_void_p,
                                         c_void_p, c_void_p, POINTER(HcaCache), c_void_p,
                                         c_void_p, c_void_p, c_void_p]
    L.hca_decode_partial_bytes.restype = c_size_t
    L.hca_decode_partial_bytes.argtypes = [POINTER(HcaDesc)]
    L.hca_attn_decode_partial.restype = c_int32
    L.hca_attn_decode_partial.argtypes = [POINTER(HcaDesc), c_void_p, c_void_p,
                                          POINTER(HcaCache), c_void_p, c_void_p, c_int32,
                                          c_int32, c_int32, c_void_p, c_void_p, c_size_t,
                                          c_void_p]
    L.hca_decode_merge.restype = c_int32
    L.hca_decode_merge.argtypes = [POINTER(HcaDesc), c_void_p, c_int32, c_int64, c_void_p,
                                   c_void_p, c_void_p]
    L.hca_prefill_backward_workspace_bytes.restype = c_size_t
    L.hca_prefill_backward_workspace_bytes.argtypes = [POINTER(HcaDesc)]
    L.hca_attn_prefill_backward.restype = c_int32
    L.hca_attn_prefill_backward.argtypes = [POINTER(HcaDesc), c_void_p, c_void_p, c_void_p,
                                            POINTER(HcaCache), c_void_p, c_void_p, c_void_p,
                                            c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                            c_void_p]
    L.hca_gate_from_latent.restype = c_int32
    L.hca_gate_from_latent.argtypes = [POINTER(HcaDesc), c_void_p, c_void_p, c_int32, c_void_p,
                                       c_void_p]
    L.hca_vha_gate.restype = c_int32
    L.hca_vha_gate.argtypes = [POINTER(HcaDesc), c_void_p, c_void_p, c_void_p, c_int32,
                               c_void_p, c_void_p]
    L.hca_decode_workspace_bytes.restype = c_size_t
    L.hca_decode_workspace_bytes.argtypes = [POINTER(HcaDesc)]
    L.hca_attn_decode.restype = c_int32
    L.hca_attn_decode.argtypes = [POINTER(HcaDesc), c_void_p, c_void_p, POINTER(HcaCache),
                                  c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                  c_void_p]
    L.hca_attn_decode_noalloc.restype = c_int32
    L.hca_attn_decode_noalloc.argtypes = [POINTER(HcaDesc), c_void_p, c_void_p,
                                          POINTER(HcaCache), c_void_p, c_void_p, c_void_p,
                                          c_void_p, c_void_p]
    if L.hca_abi_version() != ABI_VERSION:
        raise RuntimeError("libhca.so ABI version does not match this binding")
    _lib = L
    return L


# ---------------------------------------------------------------------------
# the C entry points, same names and arguments
# ---------------------------------------------------------------------------

def hca_abi_version() -> int:
    return lib().hca_abi_version()


def hca_status_string(status: int) -> str:
    return lib().hca_status_string(status).decode()


def status_string(status: int) -> str:
    try:
        return hca_status_string(status)
    except Exception:  # library missing: still describe the code
        return str(status)


def hca_set_gate(desc: HcaDesc, gate: int, strides) -> int:
    arr = None if strides is None else (c_int64 * 3)(*strides)
    return lib().hca_set_gate(ctypes.byref(desc), gate or None,
                              None if arr is None else ctypes.cast(arr, c_void_p))


def hca_compress(desc: HcaDesc, K: int, V: int, batch_stride_tokens: int, first_block: int,
                 n_blocks: int, cache: HcaCache, stream: int = 0) -> int:
    return lib().hca_compress(ctypes.byref(desc), K or None, V or None, batch_stride_tokens,
                              first_block, n_blocks, ctypes.byref(cache), stream or None)


def hca_attn_decode_append(desc: HcaDesc, Q: int, ctx_len: int, cache: HcaCache, new_k: int,
                           new_v: int, ring_k: int, ring_v: int, O: int, lse: int,
                           workspace: int, workspace_bytes: int, stream: int = 0) -> int:
    return lib().hca_attn_decode_append(ctypes.byref(desc), Q or None, ctx_len or None,
                                        ctypes.byref(cache), new_k or None, new_v or None,
                                        ring_k or None, ring_v or None, O or None, lse or None,
                                        workspace or None, workspace_bytes, stream or None)


def hca_ring_append(desc: HcaDesc, new_k: int, new_v: int, ctx_len: int, ring_k: int,
                    ring_v: int, stream: int = 0) -> int:
    return lib().hca_ring_append(ctypes.byref(desc), new_k or None, new_v or None,
                                 ctx_len or None, ring_k or None, ring_v or None,
                                 stream or None)


def hca_attn_prefill(desc: HcaDesc, Q: int, K: int, V: int, cache: HcaCache, O: int,
                     lse: int = 0, dbg_mask: int = 0, stream: int = 0) -> int:
    return lib().hca_attn_prefill(ctypes.byref(desc), Q or None, K or None, V or None,
                                  ctypes.byref(cache), O or None, lse or None,
                                  dbg_mask or None, stream or None)


def hca_attn_prefill_range(desc: HcaDesc, q_pos0: int, kv_pos0: int, kv_len: int, Q: int,
                           K: int, V: int, cache: HcaCache, O: int, lse: int = 0,
                           dbg_mask: int = 0, stream: int = 0) -> int:
    return lib().hca_attn_prefill_range(ctypes.byref(desc), q_pos0, kv_pos0, kv_len, Q or None,
                                        K or None, V or None, ctypes.byref(cache), O or None,
                                        lse or None, dbg_mask or None, stream or None)


def hca_decode_partial_bytes(desc: HcaDesc) -> int:
    return lib().hca_decode_partial_bytes(ctypes.byref(desc))


def hca_attn_decode_partial(desc: HcaDesc, Q: int, ctx_len: int, cache: HcaCache, ring_k: int,
                            ring_v: int, entry_begin: int, entry_end: int, with_window: int,
                            partial: int, workspace: int, workspace_bytes: int,
                            stream: int = 0) -> int:
    return lib().hca_attn_decode_partial(ctypes.byref(desc), Q or None, ctx_len or None,
                                         ctypes.byref(cache), ring_k or None, ring_v or None,
                                         entry_begin, entry_end, with_window, partial or None,
                                         workspace or None, workspace_bytes, stream or None)


def hca_decode_merge(desc: HcaDesc, parts: int, n_parts: int, part_stride: int, O: int,
                     lse: int = 0, stream: int = 0) -> int:
    return lib().hca_decode_merge(ctypes.byref(desc), parts or None, n_parts, part_stride,
                                  O or None, lse or None, stream or None)


def hca_prefill_backward_workspace_bytes(desc: HcaDesc) -> int:
    return lib().hca_prefill_backward_workspace_bytes(ctypes.byref(desc))


def hca_attn_prefill_backward(desc: HcaDesc, Q: int, K: int, V: int, cache: HcaCache,
                              lse: int, dO: int, dQ: int, dK: int, dV: int, dG: int,
                              workspace: int, workspace_bytes: int, stream: int = 0) -> int:
    return lib().hca_attn_prefill_backward(ctypes.byref(desc), Q or None, K or None, V or None,
                                           ctypes.byref(cache), lse or None,
                                           dO or None, dQ or None, dK or None, dV or None,
                                           dG or None, workspace or None, workspace_bytes,
                                           stream or None)


def hca_gate_from_latent(desc: HcaDesc, q_lat: int, W_g: int, latent: int, G: int,
                         stream: int = 0) -> int:
    return lib().hca_gate_from_latent(ctypes.byref(desc), q_lat or None, W_g or None, latent,
                                      G or None, stream or None)


def hca_vha_gate(desc: HcaDesc, O: int, A: int, B: int, rank: int, out: int,
                 stream: int = 0) -> int:
    return lib().hca_vha_gate(ctypes.byref(desc), O or None, A or None, B or None, rank,
                              out or None, stream or None)


def hca_decode_workspace_bytes(desc: HcaDesc) -> int:
    return lib().hca_decode_workspace_bytes(ctypes.byref(desc))


def hca_attn_decode(desc: HcaDesc, Q: int, ctx_len: int, cache: HcaCache, ring_k: int,
                    ring_v: int, O: int, lse: int, workspace: int, workspace_bytes: int,
                    stream: int = 0) -> int:
    return lib().hca_attn_decode(ctypes.byref(desc), Q or None, ctx_len or None,
                                 ctypes.byref(cache), ring_k or None, ring_v or None,
                                 O or None, lse or None, workspace or None, workspace_bytes,
                                 stream or None)


def hca_attn_decode_noalloc(desc: HcaDesc, Q: int, ctx_len: int, cache: HcaCache,
                            ring_k: int, ring_v: int, O: int, lse: int = 0,
                            stream: int = 0) -> int:
    """Decode step whose split partials live in the library's own fixed device array, for
    callers that cannot lend it device memory (see include/hca.h)."""
    return lib().hca_attn_decode_noalloc(ctypes.byref(desc), Q or None, ctx_len or None,
                                         ctypes.byref(cache), ring_k or None, ring_v or None,
                                         O or None, lse or None, stream or None)


def check(status: int, what: str) -> None:
    if status != HCA_OK:
        raise HcaError(status, what)


# ---------------------------------------------------------------------------
# struct builders from torch tensors (plumbing: shapes and pointers only)
# ---------------------------------------------------------------------------

def make_desc(batch: int, seqlen: int, hq: int, hkv: int, head_dim: int, block: int = 128,
              window: int = 128, scale: Optional[float] = None, dtype: int = HCA_BF16,
              decode_splits: int = 0) -> HcaDesc:
    d = HcaDesc()
    d.batch, d.seqlen, d.hq, d.hkv = batch, seqlen, hq, hkv
    d.head_dim, d.block, d.window = head_dim, block, window
    d.scale = (1.0 / math.sqrt(head_dim)) if scale is None else scale
    d.dtype = dtype
    d.decode_splits = decode_splits
    d.gate = None
    return d


def dtype_code(t) -> int:
    import torch
    return {torch.bfloat16: HCA_BF16, torch.float32: HCA_F32}[t.dtype]


class PagedCache:
    """Device memory for a paged compressed cache, allocated through torch.

    ``page_table`` is a [batch, max_pages] int32 tensor of page ids (any order).
    ``e4m3_scales=(k_scale, v_scale)`` makes the pools 8-bit (uint8 tensors of e4m3 codes,
    HCA_POOL_E4M3) with those per-pool scales.
    """

    def __init__(self, batch: int, max_entries: int, hkv: int, head_dim: int, dtype,
                 page_entries: int = 128, page_table=None, device="cuda", e4m3_scales=None):
        import torch
        self.page_entries = page_entries
        self.max_pages = max(1, -(-max_entries // page_entries))
        self.num_pages = batch * self.max_pages
        shape = (self.num_pages, page_entries, hkv, head_dim)
        pool_dtype = torch.uint8 if e4m3_scales is not None else dtype
        self.kc = torch.zeros(shape, dtype=pool_dtype, device=device)
        self.vc = torch.zeros(shape, dtype=pool_dtype, device=device)
        if page_table is None:
            page_table = torch.arange(self.num_pages, dtype=torch.int32).view(batch, -1)
        self.page_table = page_table.to(device=device, dtype=torch.int32).contiguous()
        self.n_entries = torch.zeros(batch, dtype=torch.int32, device=device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        c = HcaCache()
        c.kc_pool = self.kc.data_ptr()
        c.vc_pool = self.vc.data_ptr()
        c.page_table = self.page_table.data_ptr()
        c.n_entries = self.n_entries.data_ptr()
        c.page_entries = page_entries
        c.max_pages = self.max_pages
        c.num_pages = self.num_pages
        c.err_word = self.err.data_ptr()
        if e4m3_scales is not None:
            c.pool_format = HCA_POOL_E4M3
            c.k_scale, c.v_scale = float(e4m3_scales[0]), float(e4m3_scales[1])
        self.e4m3_scales = e4m3_scales
        self.c = c

    def entry_rows(self, b: int, n: int):
        """Pool row indices of entries 0..n-1 of sequence b (host-side, for tests)."""
        pt = self.page_table[b].cpu()
        return [int(pt[j // self.page_entries]) * self.page_entries + j % self.page_entries
                for j in range(n)]

    def fill(self, b: int, keys, vals) -> None:
        """Write entries 0..n-1 of sequence b directly (decode workloads state the cache)."""
        import torch
        n = keys.shape[0]
        rows = torch.tensor(self.entry_rows(b, n), device=self.kc.device, dtype=torch.long)
        flat_k = self.kc.view(-1, *self.kc.shape[2:])
        flat_v = self.vc.view(-1, *self.vc.shape[2:])
        flat_k[rows] = keys.to(self.kc.dtype)
        flat_v[rows] = vals.to(self.vc.dtype)
        self.n_entries[b] = n
