"""Random KV-cache eviction for the oracle -- TEST INFRASTRUCTURE ONLY (part of the oracle).

intelligenzai.it, "La sorprendente sencillez de comprimir la memoria de la IA" (on arXiv
2609.03430, Random Attention): the eviction keeps the tokens of the initial prompt and of
the most recent window and drops the others uniformly at random inside each attention
head, with budgets of about 4x compression; "Resumen Tecnico: ART" S2.4: ART is
orthogonal to such cache policies and runs on what they keep.

Readings (the page gives no formula):
  * eviction acts per (batch, kv head): the cache holds one K/V row per kv head;
  * kept set of a sequence of length L with budget M >= n_sink + n_recent:
      all positions when L <= M; otherwise [0, n_sink), [L - n_recent, L), and the
      m = M - n_sink - n_recent middle positions j (n_sink <= j < L - n_recent) whose
      (key_j, j) pairs are the m smallest, key_j a caller-given uniform uint32 -- a
      uniform draw without replacement;
  * the kept rows are packed into a contiguous cache in increasing position order
    (keys and values are cached after their positional encoding, so the order of the
    packed rows only fixes the tile structure), and the decode runs on min(L, M) rows.
Plain numpy; pinned by tests/test_oracle_evict.py.
"""
from __future__ import annotations

import numpy as np

from . import decode


def kept_positions(L: int, keys: np.ndarray, n_sink: int, n_recent: int, budget: int) -> np.ndarray:
    """Sorted kept positions of one (batch, kv head); keys: uint32 [>= L]."""
    if L <= budget:
        return np.arange(L, dtype=np.int32)
    lo, hi = n_sink, L - n_recent
    m = budget - n_sink - n_recent
    mid = np.arange(lo, hi)
    pick = mid[np.lexsort((mid, keys[lo:hi].astype(np.uint64)))[:m]]
    return np.sort(np.concatenate([np.arange(0, lo), pick, np.arange(hi, L)])).astype(np.int32)


def select(seq_lens, keys: np.ndarray, n_sink: int, n_recent: int, budget: int) -> np.ndarray:
    """kept[B, Hkv, budget] int32 (sorted positions, -1 past min(L_b, budget)); keys [B, Hkv, L_max] uint32."""
    B, Hkv, _ = keys.shape
    out = np.full((B, Hkv, budget), -1, np.int32)
    for b in range(B):
        for h in range(Hkv):
            kp = kept_positions(int(seq_lens[b]), keys[b, h], n_sink, n_recent, budget)
            out[b, h, :len(kp)] = kp
    return out


def compact(x: np.ndarray, kept: np.ndarray) -> np.ndarray:
    """Packed [B, Hkv, budget, ...] rows of x [B, Hkv, L_max, ...] at the kept positions (zero rows past them)."""
    if x is None:
        return None
    B, Hkv, budget = kept.shape
    out = np.zeros((B, Hkv, budget) + x.shape[3:], dtype=x.dtype)
    for b in range(B):
        for h in range(Hkv):
            idx = kept[b, h][kept[b, h] >= 0]
            out[b, h, :len(idx)] = x[b, h, idx]
    return out


def decode_evicted(*, kind, q, k, v, seq_lens, keys, n_sink, n_recent, budget, tile, k_scale=None, v_scale=None,
                   **kw):
    """oracle.decode on the cache that random eviction leaves (same keyword arguments otherwise)."""
    kept = select(seq_lens, keys, n_sink, n_recent, budget)
    lens = np.minimum(np.asarray(seq_lens), budget).astype(np.int32)
    return decode(kind=kind, q=q, k=compact(k, kept), v=compact(v, kept), k_scale=compact(k_scale, kept),
                  v_scale=compact(v_scale, kept), seq_lens=lens, tile=tile, **kw), kept
