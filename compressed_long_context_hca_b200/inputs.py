"""Seeded synthetic inputs shared by the tests, the bench and the oracle legs.

This module holds no HCA arithmetic: it only draws random numbers and lays
them out.  Both the CUDA path and the float64 oracle consume the arrays it
returns, so parity never depends on two random streams matching.

Recipe (the workload shapes of the ERNIE-5.5-Flash-Base pages: 64 query
heads, head_dim 512, 128K training and 1M inference context):

* one ``torch.Generator`` seeded with ``seed``; Q, K, V, then the gate logits,
  each drawn as float32 N(0, 1) in that order, then cast to the compute dtype;
* optional "heterogeneous blocks": every block j with j % 4 == 3 (0-based, 128
  tokens) is multiplied by 4 in Q, K and V -- exact in bf16;
* optional gate G = sigmoid(N(0, 1)) of shape [b, T, Hq, D];
* decode: context lengths are uniform integers in [lo, hi] from the same
  generator; cache entries and ring tokens are N(0, 1);
* pages of the compressed cache are handed out in a seeded random order so
  that no test relies on pages being contiguous;
* 8-bit decode workloads: the cache entries are e4m3 codes, a random sign bit over a
  magnitude code uniform in 0..0x5F (drawn as bytes, not computed from values).
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch


def _dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


@dataclass
class PrefillInputs:
    Q: torch.Tensor          # [b, T, hq, D]
    K: torch.Tensor          # [b, T, hkv, D]
    V: torch.Tensor          # [b, T, hkv, D]
    G: Optional[torch.Tensor]  # [b, T, hq, D] or None


def prefill_inputs(batch: int, T: int, hq: int, hkv: int, D: int,
                   dtype: str = "bf16", seed: int = 0,
                   hetero_blocks: bool = False, gate: bool = False,
                   block: int = 128, device: str = "cpu") -> PrefillInputs:
    """Q, K, V (and gate) for one prefill workload, drawn on ``device``."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    dt = _dtype(dtype)

    def draw(h):
        x = torch.randn((batch, T, h, D), generator=g, device=device,
                        dtype=torch.float32)
        if hetero_blocks:
            blk = (torch.arange(T, device=device) // block) % 4 == 3
            x[:, blk] *= 4.0
        return x.to(dt)

    Q = draw(hq)
    K = draw(hkv)
    V = draw(hkv)
    G = None
    if gate:
        G = torch.sigmoid(torch.randn((batch, T, hq, D), generator=g,
                                      device=device, dtype=torch.float32)).to(dt)
    return PrefillInputs(Q, K, V, G)


def page_order(num_pages: int, seed: int = 1234) -> torch.Tensor:
    """A seeded permutation of page ids (int32, CPU)."""
    g = torch.Generator()
    g.manual_seed(seed)
    return torch.randperm(num_pages, generator=g).to(torch.int32)


def page_table(batch: int, max_pages: int, seed: int = 1234) -> torch.Tensor:
    """[batch, max_pages] int32 table over a pool of batch*max_pages pages."""
    return page_order(batch * max_pages, seed).view(batch, max_pages).contiguous()


@dataclass
class DecodeInputs:
    q: torch.Tensor          # [nseq, hq, D]
    ctx_len: torch.Tensor    # [nseq] int32, includes the new token
    entries_k: torch.Tensor  # [nseq, max_entries, hkv, D] compressed K entries
    entries_v: torch.Tensor
    ring_k: torch.Tensor     # [nseq, W, hkv, D]; raw token u sits in slot u % W
    ring_v: torch.Tensor
    G: Optional[torch.Tensor]  # [nseq, hq, D] or None


def decode_inputs(nseq: int, hq: int, hkv: int, D: int, W: int, block: int,
                  ctx_lo: int, ctx_hi: int, max_entries: int,
                  dtype: str = "bf16", seed: int = 0, gate: bool = False,
                  device: str = "cpu") -> DecodeInputs:
    """One decode step: a query per sequence over a synthetic cache.

    Cache entries are drawn N(0, 1) directly (the workload states the cache
    contents, not the history that produced them).
    """
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    dt = _dtype(dtype)
    ctx = torch.randint(ctx_lo, ctx_hi + 1, (nseq,), generator=g, device=device,
                        dtype=torch.int64).to(torch.int32)
    q = torch.randn((nseq, hq, D), generator=g, device=device).to(dt)
    ek = torch.randn((nseq, max_entries, hkv, D), generator=g, device=device).to(dt)
    ev = torch.randn((nseq, max_entries, hkv, D), generator=g, device=device).to(dt)
    rk = torch.randn((nseq, W, hkv, D), generator=g, device=device).to(dt)
    rv = torch.randn((nseq, W, hkv, D), generator=g, device=device).to(dt)
    G = None
    if gate:
        G = torch.sigmoid(torch.randn((nseq, hq, D), generator=g,
                                      device=device)).to(dt)
    return DecodeInputs(q, ctx, ek, ev, rk, rv, G)


def e4m3_codes(shape, generator: torch.Generator, max_magnitude_code: int = 0x5F,
               device: str = "cpu") -> torch.Tensor:
    """Random 8-bit e4m3 codes (uint8): a random sign bit over a magnitude code drawn
    uniformly from 0 .. max_magnitude_code (0x5F: exponent fields 0..11, values up to 30,
    spread evenly over the binades). No NaN code is drawn."""
    mag = torch.randint(0, max_magnitude_code + 1, shape, generator=generator, device=device,
                        dtype=torch.int32)
    sign = torch.randint(0, 2, shape, generator=generator, device=device, dtype=torch.int32)
    return (mag | (sign << 7)).to(torch.uint8)


def decode_inputs_e4m3(nseq: int, hq: int, hkv: int, D: int, W: int, block: int,
                       ctx_lo: int, ctx_hi: int, max_entries: int, seed: int = 0,
                       gate: bool = False, device: str = "cpu") -> DecodeInputs:
    """One decode step over an 8-bit compressed cache: as decode_inputs (bf16 query, ring
    and gate from the same generator order), but the cache entries are e4m3 codes drawn by
    e4m3_codes (the workload states the stored bytes; with a pool scale of 1/16 their
    values lie within +-1.875)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    dt = torch.bfloat16
    ctx = torch.randint(ctx_lo, ctx_hi + 1, (nseq,), generator=g, device=device,
                        dtype=torch.int64).to(torch.int32)
    q = torch.randn((nseq, hq, D), generator=g, device=device).to(dt)
    ek = e4m3_codes((nseq, max_entries, hkv, D), g, device=device)
    ev = e4m3_codes((nseq, max_entries, hkv, D), g, device=device)
    rk = torch.randn((nseq, W, hkv, D), generator=g, device=device).to(dt)
    rv = torch.randn((nseq, W, hkv, D), generator=g, device=device).to(dt)
    G = None
    if gate:
        G = torch.sigmoid(torch.randn((nseq, hq, D), generator=g, device=device)).to(dt)
    return DecodeInputs(q, ctx, ek, ev, rk, rv, G)


@dataclass
class DecodeStepTokens:
    q: torch.Tensor          # [steps, nseq, hq, D] query of each step's new token
    k: torch.Tensor          # [steps, nseq, hkv, D] its key / value (step 0 is unused: the
    v: torch.Tensor          #   first step's token is already in the ring)
    G: Optional[torch.Tensor]  # [steps, nseq, hq, D] or None


def decode_step_tokens(nseq: int, hq: int, hkv: int, D: int, steps: int,
                       dtype: str = "bf16", seed: int = 0, gate: bool = False,
                       device: str = "cpu") -> DecodeStepTokens:
    """New tokens of consecutive decode steps (query, key, value, gate), N(0, 1)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    dt = _dtype(dtype)
    q = torch.randn((steps, nseq, hq, D), generator=g, device=device).to(dt)
    k = torch.randn((steps, nseq, hkv, D), generator=g, device=device).to(dt)
    v = torch.randn((steps, nseq, hkv, D), generator=g, device=device).to(dt)
    G = None
    if gate:
        G = torch.sigmoid(torch.randn((steps, nseq, hq, D), generator=g,
                                      device=device)).to(dt)
    return DecodeStepTokens(q, k, v, G)
