"""The two-pass restatement of the q8 V-skip rule equals the oracle's sequential rule.

The skip rule (puntofijo.es, "La Elegancia de la Omision") drops row j of tile t from the
numerator when exp(s_j - m'_t) < tau, m'_t the running maximum of the split after tile t.  The
GPU runs full attention in two passes: scores with tile and chunk maxima first, then, per chunk
of CT tiles, m'_t = max(maxima of earlier chunks, prefix of the chunk's tile maxima), weights
relative to the chunk's own reference (m' at its last tile), and a combine of all chunk states.
A tile whose maximum already fails the test for every head is not read at all.

Here that decomposition is written out in float64 numpy (no GPU code) and compared with the
oracle, which walks the tiles one by one; the dead-tile claim is checked row by row.
"""
import numpy as np
import pytest

from kv_cache_early_split_b200 import inputs as I
from helpers import oracle_run

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def dequant(w):
    """float64 q [B, Hq, d], K, V [B, Hkv, L_max, d] of a q8 workload."""
    q = (w.q.astype(np.uint32) << 16).view(np.float32).astype(np.float64)

    def one(codes, scale):
        s = scale.view(np.float16).astype(np.float64)
        return codes.astype(np.float64) * np.repeat(s, 32, axis=-1)

    return q, one(w.k, w.k_scale), one(w.v, w.v_scale)


def two_pass(w, tau, CT, S):
    q, K, V = dequant(w)
    B, Hq, d = q.shape
    G = Hq // w.Hkv
    T = w.tile
    out = np.zeros((B, Hq, d))
    dead_tiles = 0
    for b in range(B):
        L = int(w.seq_lens[b])
        n = -(-L // T)
        for hq in range(Hq):
            kvh = hq // G
            s = K[b, kvh, :L] @ q[b, hq] / np.sqrt(d)  # pass 1: every score
            tmax = np.array([s[t * T:min(t * T + T, L)].max() for t in range(n)])
            states = []
            for sp in range(S):
                t0, t1 = (sp * n) // S, ((sp + 1) * n) // S
                chunks = [(c, min(c + CT, t1)) for c in range(t0, t1, CT)]
                cmax = [tmax[a:e].max() for a, e in chunks]
                for ci, (a, e) in enumerate(chunks):  # pass 2: one chunk
                    mb = max(cmax[:ci]) if ci else -np.inf
                    mp = np.maximum(mb, np.maximum.accumulate(tmax[a:e]))  # m'_t of the chunk's tiles
                    ref = mp[-1]
                    lsum, acc = 0.0, np.zeros(d)
                    for t in range(a, e):
                        rows = slice(t * T, min(t * T + T, L))
                        p = np.exp(s[rows] - mp[t - a])
                        wgt = p * np.exp(mp[t - a] - ref)
                        lsum += wgt.sum()
                        keep = ~(p < tau)
                        if np.exp(tmax[t] - mp[t - a]) < tau:  # dead tile: no row may be kept
                            assert not keep.any()
                            dead_tiles += 1
                            continue
                        acc += (wgt * keep) @ V[b, kvh, rows]
                    states.append((ref, lsum, acc))
            M = max(m for m, _, _ in states)  # combine
            den = sum(np.exp(m - M) * l for m, l, _ in states)
            num = sum(np.exp(m - M) * a for m, _, a in states)
            out[b, hq] = num / den
    return out, dead_tiles


CASES = [
    # B, Hq, Hkv, d, L_max, lens, tile, S, CT, kw
    (2, 8, 2, 128, 2048, [2048, 1001], 64, 1, 8, dict(gumbel_scale=6.0, q_scale=2.0)),
    (1, 4, 1, 64, 1500, [1499], 32, 2, 16, dict(gumbel_scale=3.0)),
    (2, 6, 2, 128, 3000, [3000, 17], 16, 3, 32, dict(sink=30.0)),
    (1, 8, 8, 64, 1024, [1000], 64, 1, 29, dict(sink=40.0)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"d{c[3]}-g{c[1] // c[2]}-T{c[6]}-S{c[7]}-CT{c[8]}")
@pytest.mark.parametrize("tau", [0.0, 1e-6, 1e-3])
def test_two_pass_equals_sequential_rule(case, tau):
    B, Hq, Hkv, d, L_max, lens, tile, S, CT, kw = case
    w = I.make_workload(kind="q8", B=B, Hq=Hq, Hkv=Hkv, d=d, L_max=L_max, tile=tile, num_splits=S,
                        seq_lens=lens, seed=31 + tile, **kw)
    o2, dead = two_pass(w, tau, CT, S)
    ref = oracle_run(w, "q8", tau=tau).o
    assert np.max(np.abs(o2 - ref)) <= 1e-12
    if tau > 0 and kw.get("sink"):
        assert dead > 0  # the sink leaves whole tiles below tau


def test_chunking_does_not_matter_without_skip():
    """With tau = 0 every chunk size gives full attention (the combine is exact)."""
    w = I.make_workload(kind="q8", B=1, Hq=4, Hkv=2, d=64, L_max=1200, tile=16, seq_lens=[1187], seed=5)
    outs = [two_pass(w, 0.0, ct, 2)[0] for ct in (8, 13, 32)]
    for o in outs[1:]:
        assert np.max(np.abs(o - outs[0])) <= 1e-12
