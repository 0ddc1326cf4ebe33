"""Pins of the oracle's paged-KV view (oracle/paged.py)."""
import numpy as np
import pytest

import oracle
from oracle import orders, paged
from kv_cache_early_split_b200 import inputs as I
from test_oracle_pins import KIND, run


def test_gather_hand_example():
    # 3 pages of 2 rows, 1 kv head, d = 2; sequence of 3 positions in pages 2 then 0
    pool = np.array([[[[1, 2], [3, 4]]], [[[5, 6], [7, 8]]], [[[9, 10], [11, 12]]]], np.float32)
    table = np.array([[2, 0, -1]], np.int32)
    g = paged.gather(pool, table, [3], 6)
    assert g.shape == (1, 1, 6, 2)
    assert g[0, 0].tolist() == [[9, 10], [11, 12], [1, 2], [0, 0], [0, 0], [0, 0]]
    with pytest.raises(ValueError):
        paged.gather(pool, np.array([[2, 5]], np.int32), [3], 4)


def _paged_run(w, p, **kw):
    return paged.decode_paged(kind=KIND[w.kind], q=w.q, k_pages=p.k, v_pages=p.v, k_scale_pages=p.k_scale,
                              v_scale_pages=p.v_scale, block_table=p.block_table, seq_lens=w.seq_lens,
                              L_max=w.L_max, tile=w.tile, num_splits=w.num_splits, **kw)


@pytest.mark.parametrize("kind", ["f32", "bf16", "q8"])
@pytest.mark.parametrize("page_size", [32, 64, 128])
def test_paged_equals_contiguous(kind, page_size):
    """Pages never referenced hold NaN: any wrong address would show.  Same results as the
    contiguous layout, with and without ART, V skip and a traversal order."""
    d = 64
    w = I.make_workload(kind=kind, B=2, Hq=4, Hkv=2, d=d, L_max=400, tile=32, num_splits=2,
                        seq_lens=[400, 150], seed=4, sink=5.0)
    p = I.paginate(w, page_size, seed=9)
    art = dict(eps_scale=2e-2, eps_dir=5e-3, patience=2, lanes=[0, 5, 9, 33])
    tau = 1e-3 if kind == "q8" else 0.0
    for a in (None, art):
        ref = run(w, art=a, tau=tau)
        got = _paged_run(w, p, art=a, tau=tau)
        assert np.isfinite(got.o).all()
        assert np.array_equal(got.used, ref.used)
        assert np.max(np.abs(got.o - ref.o)) == 0.0
    order = orders.tile_order_recency(w.seq_lens, w.Hkv, w.L_max, w.tile, 2)
    ref = run(w, art=art, tau=tau, tile_order=order)
    got = _paged_run(w, p, art=art, tau=tau, tile_order=order)
    assert np.array_equal(got.used, ref.used) and np.max(np.abs(got.o - ref.o)) == 0.0


def test_shared_prefix_pages():
    """Two sequences whose block tables point at the same pages (a shared prompt) and carry the
    same queries give the same outputs; changing one shared page changes both."""
    w = I.make_workload(kind="bf16", B=2, Hq=2, Hkv=1, d=32, L_max=128, tile=16, seq_lens=[128, 128], seed=2)
    w.q[1] = w.q[0]
    p = I.paginate(w, 32, seed=1)
    p.block_table[1] = p.block_table[0]
    r = _paged_run(w, p)
    assert np.array_equal(r.o[0], r.o[1])
    p.v[p.block_table[0, 2]] = I.bf16_bits(np.ones((1, 32, 32), np.float32))
    r2 = _paged_run(w, p)
    assert np.array_equal(r2.o[0], r2.o[1]) and np.max(np.abs(r2.o - r.o)) > 1e-3
