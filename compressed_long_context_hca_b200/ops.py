"""torch-tensor front end over the C ABI (shapes, pointers, streams; no arithmetic).

Every function here calls straight into libhca through ``binding`` and raises
``binding.HcaError`` on a non-zero status. Tensors must live on the current CUDA
device and be contiguous.
"""

from __future__ import annotations

from typing import Optional

import torch

from . import binding as B


def _ptr(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.data_ptr()


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def desc_for_prefill(Q: torch.Tensor, K: torch.Tensor, block: int = 128, window: int = 128,
                     scale: Optional[float] = None) -> B.HcaDesc:
    b, T, hq, D = Q.shape
    return B.make_desc(b, T, hq, K.shape[2], D, block, window, scale, B.dtype_code(Q))


def attach_gate(desc: B.HcaDesc, G: Optional[torch.Tensor]) -> None:
    """G: [b, T, hq, D] (prefill) or [nseq, hq, D] (decode), head_dim contiguous."""
    if G is None:
        B.check(B.hca_set_gate(desc, 0, None), "hca_set_gate")
        desc._gate_ref = None
        return
    st = G.stride()
    strides = (st[0], st[1], st[2]) if G.dim() == 4 else (st[0], 0, st[1])
    B.check(B.hca_set_gate(desc, G.data_ptr(), strides), "hca_set_gate")
    desc._gate_ref = G  # the descriptor holds a raw pointer: keep the tensor alive


def compress(desc: B.HcaDesc, K: torch.Tensor, V: torch.Tensor, cache: B.PagedCache,
             first_block: int = 0, n_blocks: Optional[int] = None,
             batch_stride_tokens: Optional[int] = None, stream=None) -> None:
    """Compress blocks [first_block, first_block + n_blocks) of K/V [b, T, hkv, D]."""
    T = desc.seqlen
    if n_blocks is None:
        n_blocks = -(-T // desc.block) - first_block
    if batch_stride_tokens is None:
        batch_stride_tokens = K.shape[1]
    off = first_block * desc.block * K.shape[2] * K.shape[3] * K.element_size()
    st = B.hca_compress(desc, K.data_ptr() + off, V.data_ptr() + off, batch_stride_tokens,
                        first_block, n_blocks, cache.c, _stream(stream))
    B.check(st, "hca_compress")


def ring_append(desc: B.HcaDesc, new_k: torch.Tensor, new_v: torch.Tensor,
                ctx_len: torch.Tensor, ring_k: torch.Tensor, ring_v: torch.Tensor,
                stream=None) -> None:
    """Write the new token's rows new_k/new_v [nseq, hkv, D] into slot (ctx_len - 1) % W of
    the rings ring_k/ring_v [nseq, W, hkv, D] (one launch)."""
    for t in (new_k, new_v, ring_k, ring_v):
        assert t.is_contiguous()
    st = B.hca_ring_append(desc, new_k.data_ptr(), new_v.data_ptr(), ctx_len.data_ptr(),
                           ring_k.data_ptr(), ring_v.data_ptr(), _stream(stream))
    B.check(st, "hca_ring_append")


def prefill(desc: B.HcaDesc, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
            cache: B.PagedCache, O: Optional[torch.Tensor] = None, want_lse: bool = False,
            want_mask: bool = False, stream=None):
    """HCA prefill; returns (O, lse or None, dbg_mask or None)."""
    if O is None:
        O = torch.empty_like(Q)
    b, T, hq, _ = Q.shape
    lse = torch.empty((b, T, hq), dtype=torch.float32, device=Q.device) if want_lse else None
    dbg = torch.full((b, T, 3), -1, dtype=torch.int32, device=Q.device) if want_mask else None
    st = B.hca_attn_prefill(desc, Q.data_ptr(), K.data_ptr(), V.data_ptr(), cache.c,
                            O.data_ptr(), _ptr(lse), _ptr(dbg), _stream(stream))
    B.check(st, "hca_attn_prefill")
    return O, lse, dbg


def decode_workspace(desc: B.HcaDesc, device="cuda") -> torch.Tensor:
    n = B.hca_decode_workspace_bytes(desc)
    return torch.empty(max(16, n), dtype=torch.uint8, device=device)


def decode(desc: B.HcaDesc, q: torch.Tensor, ctx_len: torch.Tensor, cache: B.PagedCache,
           ring_k: torch.Tensor, ring_v: torch.Tensor, O: Optional[torch.Tensor] = None,
           workspace: Optional[torch.Tensor] = None, want_lse: bool = False, stream=None):
    """One decode step; q [nseq, hq, D], ring [nseq, W, hkv, D]. Returns (O, lse or None)."""
    if O is None:
        O = torch.empty_like(q)
    if workspace is None:
        workspace = decode_workspace(desc, q.device)
    lse = (torch.empty(q.shape[:2], dtype=torch.float32, device=q.device) if want_lse
           else None)
    st = B.hca_attn_decode(desc, q.data_ptr(), ctx_len.data_ptr(), cache.c, ring_k.data_ptr(),
                           ring_v.data_ptr(), O.data_ptr(), _ptr(lse), workspace.data_ptr(),
                           workspace.numel(), _stream(stream))
    B.check(st, "hca_attn_decode")
    return O, lse


def decode_append(desc: B.HcaDesc, q: torch.Tensor, ctx_len: torch.Tensor,
                  cache: B.PagedCache, new_k: torch.Tensor, new_v: torch.Tensor,
                  ring_k: torch.Tensor, ring_v: torch.Tensor, O: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, want_lse: bool = False,
                  stream=None):
    """One decode step that first writes the new token's rows new_k/new_v [nseq, hkv, D]
    into ring slot (ctx_len - 1) % W. Returns (O, lse or None)."""
    for t in (new_k, new_v, ring_k, ring_v):
        assert t.is_contiguous()
    if O is None:
        O = torch.empty_like(q)
    if workspace is None:
        workspace = decode_workspace(desc, q.device)
    lse = (torch.empty(q.shape[:2], dtype=torch.float32, device=q.device) if want_lse
           else None)
    st = B.hca_attn_decode_append(desc, q.data_ptr(), ctx_len.data_ptr(), cache.c,
                                  new_k.data_ptr(), new_v.data_ptr(), ring_k.data_ptr(),
                                  ring_v.data_ptr(), O.data_ptr(), _ptr(lse), workspace.data_ptr(),
                                  workspace.numel(), _stream(stream))
    B.check(st, "hca_attn_decode_append")
    return O, lse


def prefill_range(desc: B.HcaDesc, q_pos0: int, kv_pos0: int, Q: torch.Tensor,
                  K: torch.Tensor, V: torch.Tensor, cache: B.PagedCache,
                  O: Optional[torch.Tensor] = None, want_lse: bool = False,
                  want_mask: bool = False, stream=None):
    """Prefill of query positions q_pos0 .. q_pos0 + Q.shape[1] - 1 with K/V rows of
    positions kv_pos0 .. kv_pos0 + K.shape[1] - 1 (desc.seqlen = Q.shape[1])."""
    if O is None:
        O = torch.empty_like(Q)
    b, T, hq, _ = Q.shape
    lse = torch.empty((b, T, hq), dtype=torch.float32, device=Q.device) if want_lse else None
    dbg = torch.full((b, T, 3), -1, dtype=torch.int32, device=Q.device) if want_mask else None
    st = B.hca_attn_prefill_range(desc, q_pos0, kv_pos0, K.shape[1], Q.data_ptr(),
                                  K.data_ptr(), V.data_ptr(), cache.c, O.data_ptr(), _ptr(lse),
                                  _ptr(dbg), _stream(stream))
    B.check(st, "hca_attn_prefill_range")
    return O, lse, dbg


def decode_partial_buffer(desc: B.HcaDesc, n_parts: int = 1, device="cuda") -> torch.Tensor:
    """Device memory for n_parts partial results, part k at byte k * partial_stride(desc)."""
    return torch.empty((n_parts, partial_stride(desc)), dtype=torch.uint8, device=device)


def partial_stride(desc: B.HcaDesc) -> int:
    n = B.hca_decode_partial_bytes(desc)
    return (n + 255) // 256 * 256


def decode_partial(desc: B.HcaDesc, q: torch.Tensor, ctx_len: torch.Tensor,
                   cache: B.PagedCache, ring_k: torch.Tensor, ring_v: torch.Tensor,
                   entry_begin: int, entry_end: int, with_window: bool,
                   out: torch.Tensor, workspace: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """Partial result of a decode step over entries [entry_begin, entry_end) (+ window)
    into `out` (a row of decode_partial_buffer)."""
    if workspace is None:
        workspace = decode_workspace(desc, q.device)
    st = B.hca_attn_decode_partial(desc, q.data_ptr(), ctx_len.data_ptr(), cache.c,
                                   ring_k.data_ptr(), ring_v.data_ptr(), entry_begin,
                                   entry_end, 1 if with_window else 0, out.data_ptr(),
                                   workspace.data_ptr(), workspace.numel(), _stream(stream))
    B.check(st, "hca_attn_decode_partial")
    return out


def decode_merge(desc: B.HcaDesc, parts: torch.Tensor, O: torch.Tensor,
                 lse: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Decode output from the partial results in the rows of `parts` [n_parts, stride]."""
    st = B.hca_decode_merge(desc, parts.data_ptr(), parts.shape[0], parts.stride(0),
                            O.data_ptr(), _ptr(lse), _stream(stream))
    B.check(st, "hca_decode_merge")
    return O


def prefill_backward(desc: B.HcaDesc, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                     cache: B.PagedCache, lse: torch.Tensor, dO: torch.Tensor,
                     workspace: Optional[torch.Tensor] = None, stream=None):
    """Gradients (dQ, dK, dV, dG or None) of hca_attn_prefill for the output gradient dO."""
    dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
    dG = torch.empty_like(Q) if desc.gate else None
    if workspace is None:
        n = B.hca_prefill_backward_workspace_bytes(desc)
        workspace = torch.empty(max(16, n), dtype=torch.uint8, device=Q.device)
    st = B.hca_attn_prefill_backward(desc, Q.data_ptr(), K.data_ptr(), V.data_ptr(), cache.c,
                                     lse.data_ptr(), dO.data_ptr(), dQ.data_ptr(),
                                     dK.data_ptr(), dV.data_ptr(), _ptr(dG),
                                     workspace.data_ptr(), workspace.numel(), _stream(stream))
    B.check(st, "hca_attn_prefill_backward")
    return dQ, dK, dV, dG


def gate_from_latent(q_lat: torch.Tensor, W_g: torch.Tensor, hq: int, head_dim: int,
                     G: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """G [rows, hq, head_dim] = sigmoid(q_lat [rows, latent] . W_g [latent, hq * head_dim])."""
    rows, latent = q_lat.shape
    if G is None:
        G = torch.empty((rows, hq, head_dim), dtype=q_lat.dtype, device=q_lat.device)
    desc = B.make_desc(1, rows, hq, 1, head_dim, dtype=B.dtype_code(q_lat))
    st = B.hca_gate_from_latent(desc, q_lat.data_ptr(), W_g.data_ptr(), latent, G.data_ptr(),
                                _stream(stream))
    B.check(st, "hca_gate_from_latent")
    return G


def vha_gate(O: torch.Tensor, A: Optional[torch.Tensor], Bm: Optional[torch.Tensor],
             G: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
             stream=None) -> torch.Tensor:
    """(O + A (B^T O) across heads) * G for O [b, T, hq, D] (or [nseq, hq, D])."""
    O4 = O if O.dim() == 4 else O.unsqueeze(1)
    b, T, hq, D = O4.shape
    desc = B.make_desc(b, T, hq, 1, D, dtype=B.dtype_code(O))
    if G is not None:
        G4 = G if G.dim() == 4 else G.unsqueeze(1)
        st = G4.stride()
        B.check(B.hca_set_gate(desc, G4.data_ptr(), (st[0], st[1], st[2])), "hca_set_gate")
    if out is None:
        out = torch.empty_like(O)
    rank = 0 if A is None else A.shape[1]
    st = B.hca_vha_gate(desc, O.data_ptr(), _ptr(A), _ptr(Bm), rank, out.data_ptr(),
                        _stream(stream))
    B.check(st, "hca_vha_gate")
    return out
