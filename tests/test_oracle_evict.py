"""Pins of the oracle's random eviction (oracle/evict.py)."""
import numpy as np
import pytest

import oracle
from oracle import evict
from kv_cache_early_split_b200 import inputs as I
from test_oracle_pins import KIND, _decode_kv, brute


def test_hand_example():
    # L = 10, sink 2, recent 3, budget 7 -> 2 middle picks among positions 2..6 by smallest key
    keys = np.array([9, 9, 50, 7, 50, 3, 99, 9, 9, 9], np.uint32)
    assert evict.kept_positions(10, keys, 2, 3, 7).tolist() == [0, 1, 3, 5, 7, 8, 9]
    # a tie on the key goes to the lower position
    keys2 = np.array([0, 0, 5, 5, 5, 1, 1, 0, 0, 0], np.uint32)
    assert evict.kept_positions(10, keys2, 2, 3, 8).tolist() == [0, 1, 2, 5, 6, 7, 8, 9]
    # short sequences keep everything; a budget equal to sink + recent keeps only those
    assert evict.kept_positions(6, keys, 2, 3, 7).tolist() == list(range(6))
    assert evict.kept_positions(10, keys, 2, 3, 5).tolist() == [0, 1, 7, 8, 9]


def test_selection_is_uniform():
    """Each middle position is kept with probability m / (L - sink - recent): over many key draws
    the counts stay within 5 standard deviations of that rate."""
    L, sink, recent, budget, trials = 60, 4, 6, 20, 4000
    rng = np.random.default_rng(0)
    hits = np.zeros(L)
    for _ in range(trials):
        kp = evict.kept_positions(L, rng.integers(0, 2**32, L, dtype=np.uint64).astype(np.uint32), sink, recent,
                                  budget)
        assert len(kp) == budget and kp[:sink].tolist() == list(range(sink))
        assert kp[-recent:].tolist() == list(range(L - recent, L))
        hits[kp] += 1
    p = (budget - sink - recent) / (L - sink - recent)
    mid = hits[sink:L - recent] / trials
    sd = np.sqrt(p * (1 - p) / trials)
    assert np.all(np.abs(mid - p) <= 5 * sd), (mid.min(), mid.max(), p)


@pytest.mark.parametrize("kind", ["f32", "bf16", "q8"])
def test_evicted_decode_is_attention_over_the_kept_rows(kind):
    """Full attention on the packed cache equals brute-force softmax attention over exactly the kept
    positions of the original cache, per kv head."""
    d = 64 if kind == "q8" else 16
    w = I.make_workload(kind=kind, B=2, Hq=4, Hkv=2, d=d, L_max=300, tile=16, seq_lens=[300, 90], seed=8)
    keys = np.random.default_rng(3).integers(0, 2**32, (2, 2, 300), dtype=np.uint64).astype(np.uint32)
    r, kept = evict.decode_evicted(kind=KIND[kind], q=w.q, k=w.k, v=w.v, k_scale=w.k_scale, v_scale=w.v_scale,
                                   seq_lens=w.seq_lens, keys=keys, n_sink=8, n_recent=32, budget=100, tile=16)
    qd, kd, vd = _decode_kv(w)
    for b in range(2):
        assert r.tiles[b, 0] == -(-min(int(w.seq_lens[b]), 100) // 16)
        for hq in range(4):
            idx = kept[b, hq // 2][kept[b, hq // 2] >= 0]
            ref = brute(qd[b, hq], kd[b, hq // 2], vd[b, hq // 2], idx)
            assert np.max(np.abs(r.o[b, hq] - ref)) <= 1e-12
    assert (kept[1] >= 0).sum(axis=-1).tolist() == [90, 90]  # L = 90 <= budget: nothing evicted
    assert np.array_equal(kept[1, 0, :90], np.arange(90))
