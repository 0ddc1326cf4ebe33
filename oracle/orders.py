"""Tile traversal orders for ART -- TEST INFRASTRUCTURE ONLY (part of the oracle).

"Resumen Tecnico: ART" (gist.science, arXiv 2606.00024), S2.4 "Integracion y
Correccion": ART can be combined with other KV-cache policies by reordering the
traversal sequence of the KV blocks, "recency first" or "importance first";
reordering does not change full attention (permutation invariance of attention
under the online softmax); block 0 is always evaluated first.

The page names the two orders without defining them.  Readings implemented here
(the plainest ones, listed with the other readings in the design notes):
  * The split structure applies to positions in the sequence: split s of a
    sequence of n tiles walks positions [floor(s*n/S), floor((s+1)*n/S)), and
    that segment is a permutation of split s's own tiles.  Each split starts
    with its own first tile (the split's "block 0"; tile 0 for split 0).
  * recency first: the split's first tile, then its other tiles from the most
    recent (highest index) back to the oldest.
  * importance first: the split's first tile, then its other tiles by a cheap
    per-tile key summary -- the mean key of the tile's positions, mu_t -- scored
    for the GQA group as max over its query heads of q_h . mu_t, highest first,
    ties to the lower tile index.
All arrays are [B, Hkv, ceil(L_max/T)] int32 with -1 at positions >= ceil(L_b/T).
Plain numpy in float64; pinned by tests/test_oracle_pins.py.
"""
from __future__ import annotations

import numpy as np


def _bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def decode_rows(kind: int, x: np.ndarray, scale: np.ndarray | None = None) -> np.ndarray:
    """Stored K (or V, Q) values as float64: fp32, bf16 bits, or q8 codes x fp16 block scales."""
    if kind == 0:
        return np.asarray(x, dtype=np.float64)
    if kind == 1:
        return _bf16_bits_to_f64(x)
    codes = np.asarray(x, dtype=np.float64)
    sc = np.asarray(scale, dtype=np.uint16).view(np.float16).astype(np.float64)
    return codes * np.repeat(sc, 32, axis=-1)


def split_segments(n: int, S: int):
    return [((s * n) // S, ((s + 1) * n) // S) for s in range(S)]


def tile_order_recency(seq_lens, Hkv: int, L_max: int, T: int, S: int) -> np.ndarray:
    B = len(seq_lens)
    n_max = -(-L_max // T)
    out = np.full((B, Hkv, n_max), -1, np.int32)
    for b in range(B):
        n = -(-int(seq_lens[b]) // T)
        for ta, tb in split_segments(n, S):
            if tb > ta:
                out[b, :, ta:tb] = [ta] + list(range(tb - 1, ta, -1))
    return out


def tile_key_summary(k: np.ndarray, seq_lens, T: int) -> np.ndarray:
    """mu[b, h, t] = mean of the keys at positions [tT, min((t+1)T, L_b)); 0 for t >= n_b.
    k: float64 [B, Hkv, L_max, d] (decoded)."""
    B, Hkv, L_max, d = k.shape
    n_max = -(-L_max // T)
    mu = np.zeros((B, Hkv, n_max, d), np.float64)
    for b in range(B):
        L = int(seq_lens[b])
        for t in range(-(-L // T)):
            j0, j1 = t * T, min((t + 1) * T, L)
            mu[b, :, t] = k[b, :, j0:j1].sum(axis=1) / (j1 - j0)
    return mu


def tile_importance(q: np.ndarray, mu: np.ndarray, seq_lens, T: int) -> np.ndarray:
    """score[b, h, t] = max over the group's query heads g of q[b, h*G+g] . mu[b, h, t]; -inf past n_b.
    q: float64 [B, Hq, d] (decoded)."""
    B, Hq, d = q.shape
    Hkv, n_max = mu.shape[1], mu.shape[2]
    G = Hq // Hkv
    sc = np.full((B, Hkv, n_max), -np.inf)
    for b in range(B):
        n = -(-int(seq_lens[b]) // T)
        for h in range(Hkv):
            dots = q[b, h * G:(h + 1) * G] @ mu[b, h, :n].T  # [G, n]
            sc[b, h, :n] = dots.max(axis=0)
    return sc


def tile_order_importance(scores: np.ndarray, seq_lens, T: int, S: int) -> np.ndarray:
    B, Hkv, n_max = scores.shape
    out = np.full((B, Hkv, n_max), -1, np.int32)
    for b in range(B):
        n = -(-int(seq_lens[b]) // T)
        for h in range(Hkv):
            for ta, tb in split_segments(n, S):
                if tb > ta:
                    rest = sorted(range(ta + 1, tb), key=lambda t: (-scores[b, h, t], t))
                    out[b, h, ta:tb] = [ta] + rest
    return out
