"""Paged KV cache for the oracle -- TEST INFRASTRUCTURE ONLY (part of the oracle).

The pages compare ART with serving stacks that keep the KV cache in fixed-size pages
addressed through a per-sequence block table (vLLM, named on the intelligenzai.it page
and in the summary's experiments).  What a paged cache computes is plain attention over
the sequence's positions; only the address of a position changes: position j of
sequence b lives in page block_table[b, j // page_size], row j % page_size, of a pool
laid out [num_pages, Hkv, page_size, ...].  The oracle therefore gathers the pages back
into a contiguous [B, Hkv, L_max, ...] cache and runs the ordinary decode on it.
Pinned by tests/test_oracle_paged.py (hand example, equality with the contiguous
layout, shared prefixes).
"""
from __future__ import annotations

import numpy as np

from . import decode


def gather(pool: np.ndarray, block_table: np.ndarray, seq_lens, L_max: int) -> np.ndarray:
    """Contiguous [B, Hkv, L_max, ...] from a page pool; positions >= L_b are zero."""
    if pool is None:
        return None
    B = block_table.shape[0]
    _, Hkv, page_size = pool.shape[:3]
    out = np.zeros((B, Hkv, L_max) + pool.shape[3:], dtype=pool.dtype)
    for b in range(B):
        L = int(seq_lens[b])
        for j0 in range(0, L, page_size):
            page = int(block_table[b, j0 // page_size])
            if not 0 <= page < pool.shape[0]:
                raise ValueError(f"block table entry {page} of sequence {b} is not a page")
            j1 = min(j0 + page_size, L)
            out[b, :, j0:j1] = pool[page, :, :j1 - j0]
    return out


def decode_paged(*, kind, q, k_pages, v_pages, block_table, seq_lens, L_max, tile, k_scale_pages=None,
                 v_scale_pages=None, **kw):
    """oracle.decode over the sequences a block table describes (same keyword arguments otherwise)."""
    return decode(kind=kind, q=q, k=gather(k_pages, block_table, seq_lens, L_max),
                  v=gather(v_pages, block_table, seq_lens, L_max),
                  k_scale=gather(k_scale_pages, block_table, seq_lens, L_max),
                  v_scale=gather(v_scale_pages, block_table, seq_lens, L_max),
                  seq_lens=seq_lens, tile=tile, **kw)
