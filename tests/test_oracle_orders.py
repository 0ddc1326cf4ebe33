"""Pins of the oracle's tile traversal orders ("Resumen Tecnico: ART", S2.4).

The page names the orders (recency first, importance first) and states two facts
that pin them: reordering the KV blocks does not change full attention, and block 0
is evaluated first.  The definitions of the two orders are this build's readings
(oracle/orders.py); the pins below fix them by hand-derived sequences, closed forms
and brute force, independently of the oracle's C code where the arithmetic matters.
"""
import numpy as np
import pytest

import oracle
from oracle import orders
from kv_cache_early_split_b200 import inputs as I
from test_oracle_pins import KIND, _decode_kv, brute, run, small


def test_recency_order_hand_example():
    # n = 10 tiles, one split: tile 0, then 9, 8, ..., 1
    o = orders.tile_order_recency([640], 1, 640, 64, 1)
    assert o[0, 0].tolist() == [0, 9, 8, 7, 6, 5, 4, 3, 2, 1]
    # n = 5 tiles (L = 300, ragged), two splits [0, 2) and [2, 5): 0 1 | 2 4 3; positions past n are -1
    o = orders.tile_order_recency([640, 300], 2, 640, 64, 2)
    assert o[1, 0].tolist() == [0, 1, 2, 4, 3, -1, -1, -1, -1, -1]
    assert o[1, 1].tolist() == o[1, 0].tolist()
    assert o[0, 0].tolist() == [0, 4, 3, 2, 1, 5, 9, 8, 7, 6]
    # one tile
    assert orders.tile_order_recency([1], 1, 64, 64, 1)[0, 0].tolist() == [0]


def _random_split_perms(w, S, seed):
    """Any per-split permutation (first tile free): full attention must not see it."""
    rng = np.random.default_rng(seed)
    n_max = -(-w.L_max // w.tile)
    out = np.full((w.B, w.Hkv, n_max), -1, np.int32)
    for b in range(w.B):
        n = -(-int(w.seq_lens[b]) // w.tile)
        for h in range(w.Hkv):
            for ta, tb in orders.split_segments(n, S):
                out[b, h, ta:tb] = ta + rng.permutation(tb - ta)
    return out


@pytest.mark.parametrize("S", [1, 3])
@pytest.mark.parametrize("kind", ["f32", "bf16", "q8"])
def test_ordered_full_attention_is_order_invariant(kind, S):
    d = 64 if kind == "q8" else 16
    w = small(kind, d=d, L_max=200, tile=16, seq_lens=[200, 77])
    ref = run(w, num_splits=S)
    for seed in range(3):
        r = run(w, num_splits=S, tile_order=_random_split_perms(w, S, seed))
        assert np.max(np.abs(r.o - ref.o)) <= 1e-12
        assert np.array_equal(r.tiles, ref.tiles)
    # with the V skip on, each split's skipped set depends on the running max along the order,
    # so only tau = 0 is order-free there
    if kind == "q8":
        a = run(w, num_splits=S, tau=0.0)
        b = run(w, num_splits=S, tau=0.0, tile_order=_random_split_perms(w, S, 9))
        assert np.max(np.abs(a.o - b.o)) <= 1e-12


@pytest.mark.parametrize("S", [1, 2])
@pytest.mark.parametrize("p", [1, 2, 3, 50])
def test_recency_with_inf_thresholds_reads_first_and_newest_tiles(S, p):
    """+inf thresholds hold on every tile, so a split stops after min(p, len) positions of its
    sequence: its first tile and its p-1 most recent tiles -- brute force over exactly those rows."""
    w = small("bf16", d=32, L_max=300, tile=16, seq_lens=[300, 47])
    order = orders.tile_order_recency(w.seq_lens, w.Hkv, w.L_max, w.tile, S)
    art = dict(eps_scale=np.inf, eps_dir=np.inf, patience=p, lanes=[0, 3, 7])
    r = run(w, art=art, num_splits=S, tile_order=order)
    qd, kd, vd = _decode_kv(w)
    for b in range(w.B):
        L = int(w.seq_lens[b])
        n = -(-L // w.tile)
        tiles = []
        for ta, tb in orders.split_segments(n, S):
            ln = tb - ta
            if ln == 0:
                continue
            newest = list(range(tb - 1, ta, -1))[: max(0, min(p, ln) - 1)]
            tiles += [ta] + newest
        rows = np.concatenate([np.arange(t * w.tile, min((t + 1) * w.tile, L)) for t in tiles])
        for hq in range(w.Hq):
            ref = brute(qd[b, hq], kd[b, hq // w.G], vd[b, hq // w.G], rows)
            assert np.max(np.abs(r.o[b, hq] - ref)) <= 1e-12
        exp_used = [min(p, tb - ta) for ta, tb in orders.split_segments(n, S)]
        assert np.all(r.used[b] == np.array(exp_used)[None, :])


def test_ordered_sequence_must_stay_inside_its_split():
    w = small("f32", d=8, L_max=96, tile=16, seq_lens=[96, 96])
    order = orders.tile_order_recency(w.seq_lens, w.Hkv, w.L_max, w.tile, 2)  # splits [0,3) [3,6)
    order[0, 1, 1] = 4  # a tile of split 1 inside split 0's segment
    with pytest.raises(ValueError):
        run(w, num_splits=2, tile_order=order)


def test_key_summary_closed_forms():
    """A tile whose keys are all equal to c has summary c; a ragged last tile averages only the rows
    that exist (rows past L_b hold 1e6 and must not count)."""
    B, Hkv, L_max, d, T = 1, 2, 80, 4, 32
    k = np.zeros((B, Hkv, L_max, d))
    for t in range(3):
        k[0, :, t * T:(t + 1) * T] = np.array([t + 1.0, -t, 0.5 * t, 2.0])
    L = 70  # tile 2 holds rows 64..69 (6 of them)
    k[0, 0, 64:67] = [3.0, 3.0, 3.0, 3.0]
    k[0, 0, 67:70] = [5.0, 1.0, 1.0, -1.0]
    k[0, :, L:] = 1e6
    mu = orders.tile_key_summary(k, [L], T)
    assert mu.shape == (1, 2, 3, 4)
    assert mu[0, 0, 0].tolist() == [1.0, 0.0, 0.0, 2.0]
    assert mu[0, 1, 1].tolist() == [2.0, -1.0, 0.5, 2.0]
    assert mu[0, 0, 2].tolist() == [4.0, 2.0, 2.0, 1.0]  # (3+5)/2, (3+1)/2, (3+1)/2, (3-1)/2
    assert mu[0, 1, 2].tolist() == [3.0, -2.0, 1.0, 2.0]


def test_importance_order_known_ranking():
    """Keys of tile t are c_t * u; the group's two queries are +q and -q with q = 2u, so the score is
    max(2 c_t, -2 c_t) = 2 |c_t|: the order is tile 0, then tiles by |c_t| descending, ties low-first."""
    d, T = 4, 8
    u = np.array([0.5, 0.5, 0.5, 0.5])
    c = [0.1, -3.0, 2.0, 0.5, 3.0, -0.5, 7.0, 0.0]  # |c|: .1 3 2 .5 3 .5 7 0
    n = len(c)
    k = np.zeros((1, 1, n * T, d))
    for t, ct in enumerate(c):
        k[0, 0, t * T:(t + 1) * T] = ct * u
    q = np.stack([2 * u, -2 * u])[None]  # [1, 2, d]
    mu = orders.tile_key_summary(k, [n * T], T)
    sc = orders.tile_importance(q, mu, [n * T], T)
    assert np.allclose(sc[0, 0], [2 * abs(x) for x in c], rtol=0, atol=1e-15)
    o = orders.tile_order_importance(sc, [n * T], T, 1)
    assert o[0, 0].tolist() == [0, 6, 1, 4, 2, 3, 5, 7]
    # two splits [0,4) and [4,8): each keeps its first tile first
    o2 = orders.tile_order_importance(sc, [n * T], T, 2)
    assert o2[0, 0].tolist() == [0, 1, 2, 3, 4, 6, 5, 7]


def test_importance_order_on_a_workload_is_a_valid_sequence():
    w = I.make_workload(kind="bf16", B=2, Hq=8, Hkv=2, d=64, L_max=1000, tile=32, num_splits=3,
                        seq_lens=[1000, 333], seed=3, sink=6.0)
    qd, kd, _ = _decode_kv(w)
    mu = orders.tile_key_summary(kd, w.seq_lens, w.tile)
    sc = orders.tile_importance(qd, mu, w.seq_lens, w.tile)
    o = orders.tile_order_importance(sc, w.seq_lens, w.tile, 3)
    for b in range(w.B):
        n = -(-int(w.seq_lens[b]) // w.tile)
        for h in range(w.Hkv):
            assert np.all(o[b, h, n:] == -1)
            for ta, tb in orders.split_segments(n, 3):
                seg = o[b, h, ta:tb]
                assert sorted(seg.tolist()) == list(range(ta, tb)) and seg[0] == ta
                s = sc[b, h, seg[1:]]
                assert np.all(np.diff(s) <= 0)
    # the ART decode accepts it, and with eps = 0 it is full attention
    r = run(w, art=dict(eps_scale=0.0, eps_dir=0.0, patience=1, lanes=[0, 9]), tile_order=o)
    assert np.max(np.abs(r.o - run(w).o)) <= 1e-12


@pytest.mark.parametrize("kind,tau", [("bf16", 0.0), ("q8", 1e-3)])
def test_ordered_run_equals_natural_run_on_physically_reordered_tiles(kind, tau):
    """Walking a sequence is walking the tiles moved into that order (L a multiple of T): same stop
    tiles, same outputs, and the rule metrics recorded by position in the sequence.  With q8 and
    tau > 0 this also fixes the V-skip running max to be taken along the sequence."""
    d = 64 if kind == "q8" else 16
    w = I.make_workload(kind=kind, B=1, Hq=4, Hkv=2, d=d, L_max=256, tile=16, seq_lens=[256], seed=11,
                        sink=6.0, gumbel_scale=2.0)
    S = 2
    order = orders.tile_order_recency(w.seq_lens, w.Hkv, w.L_max, w.tile, S)
    order[0, 1, 8:] = [8, 12, 9, 15, 10, 14, 11, 13]  # kv head 1, split 1: another permutation
    art = dict(eps_scale=2e-2, eps_dir=5e-3, patience=2, lanes=[0, 3, 5, 8])
    r = run(w, art=art, num_splits=S, tile_order=order, tau=tau, want_metrics=True, no_break=True)
    for h in range(w.Hkv):
        rows = (order[0, h][:, None] * w.tile + np.arange(w.tile)[None, :]).reshape(-1)
        wp = I.make_workload(kind=kind, B=1, Hq=4, Hkv=2, d=d, L_max=256, tile=16, seq_lens=[256], seed=11,
                             sink=6.0, gumbel_scale=2.0)
        for name in ("k", "v", "k_scale", "v_scale"):
            x = getattr(wp, name)
            if x is not None:
                x[:, h] = x[:, h][:, rows]
        rn = run(wp, art=art, num_splits=S, tau=tau, want_metrics=True, no_break=True)
        hs = slice(h * w.G, (h + 1) * w.G)
        assert np.array_equal(r.used[:, hs], rn.used[:, hs])
        assert np.max(np.abs(r.o[:, hs] - rn.o[:, hs])) <= 1e-12
        assert np.allclose(r.metrics[:, hs], rn.metrics[:, hs], rtol=0, atol=1e-12, equal_nan=True)
