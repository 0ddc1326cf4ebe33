"""GPU parity of the paged-KV entry points against the oracle's paged view.

Pools carry NaN in every page no sequence uses, so a wrong address shows as NaN.
Bars as in the other parity tests: outputs within TOL of the oracle run to the GPU's
own stop tiles, tile counts within the acceptance rule.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import kv_cache_early_split_b200 as K  # noqa: E402
from kv_cache_early_split_b200 import capi  # noqa: E402
from kv_cache_early_split_b200 import inputs as I  # noqa: E402
from oracle import orders, paged  # noqa: E402
from helpers import KIND, TOL, check_tiles  # noqa: E402

pytestmark = pytest.mark.gpu

CASES = [
    # kind, d, Hq, Hkv, B, L_max, lens, tile, S, page_size   (the first three take the tensor-core kernel)
    ("bf16", 128, 8, 2, 2, 3000, [3000, 1290], 64, 1, 64),
    ("bf16", 128, 4, 2, 2, 4096, [4096, 1000], 128, 2, 256),
    ("bf16", 128, 8, 1, 1, 5000, [4999], 64, 3, 128),
    ("bf16", 128, 8, 2, 2, 2000, [2000, 777], 32, 1, 32),
    ("f32", 64, 4, 2, 2, 1500, [1500, 333], 16, 2, 48),
    ("q8", 128, 8, 2, 2, 2048, [2048, 1001], 64, 1, 128),
    ("q8", 64, 4, 1, 1, 1500, [1499], 32, 2, 64),
]
IDS = [f"{c[0]}-d{c[1]}-g{c[2] // c[3]}-T{c[7]}-S{c[8]}-P{c[9]}" for c in CASES]


def make(kind, d, Hq, Hkv, B, L_max, lens, tile, S, page, seed=0):
    w = I.make_workload(kind=kind, B=B, Hq=Hq, Hkv=Hkv, d=d, L_max=L_max, tile=tile, num_splits=S, seq_lens=lens,
                        seed=3000 + seed, sink=6.0)
    return w, I.paginate(w, page, seed=seed + 5)


def oracle_paged(w, pg, mode, *, art=None, tau=None, forced_used=None, metrics=False, tile_order=None):
    a = art if mode in ("art", "q8_art") else None
    return paged.decode_paged(
        kind=KIND[w.kind], q=w.q, k_pages=pg.k, v_pages=pg.v, k_scale_pages=pg.k_scale, v_scale_pages=pg.v_scale,
        block_table=pg.block_table, seq_lens=w.seq_lens, L_max=w.L_max, tile=w.tile, num_splits=w.num_splits,
        art=a, tau=(tau if mode in ("q8", "q8_art") else 0.0), forced_used=forced_used,
        no_break=metrics and a is not None, want_metrics=metrics and a is not None, n_threads=8, tile_order=tile_order)


def gpu(w, pg, mode, art=None, tau=None, order=None):
    dp = K.upload(w, paged=pg)
    od = None if order is None else torch.from_numpy(np.ascontiguousarray(order)).to(dp.k.device)
    K.decode(dp, mode, art=art, tau=tau, order=od)
    st = K.device_status(dp)
    return dict(o=dp.o.cpu().numpy(), tiles=dp.tiles.cpu().numpy(), used=dp.split_tiles().cpu().numpy(), status=st)


ART = dict(eps_scale=2e-2, eps_dir=5e-3, patience=2)


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_paged_matches_oracle(case):
    w, pg = make(*case)
    lanes = I.probe_lanes_strided(w.d, 16 if w.d == 128 else 8)
    art = dict(ART, lanes=lanes)
    q8 = w.kind == "q8"
    modes = [("q8", None), ("q8_art", art)] if q8 else [("full", None), ("art", art)]
    tau = 1e-3 if q8 else None
    for mode, a in modes:
        g = gpu(w, pg, mode, art=a, tau=tau)
        assert g["status"] == capi.ART_OK
        assert np.isfinite(g["o"]).all()
        if a is None:
            ref = oracle_paged(w, pg, mode, tau=tau)
            assert np.array_equal(g["used"], ref.used)
            err = np.max(np.abs(g["o"] - ref.o))
        else:
            ref = oracle_paged(w, pg, mode, art=a, tau=tau, metrics=True)
            check_tiles(w, ref.metrics, g["used"], a, w.tile, w.num_splits)
            forced = oracle_paged(w, pg, "q8" if q8 else "full", tau=tau, forced_used=g["used"])
            err = np.max(np.abs(g["o"] - forced.o))
        assert err <= TOL[w.kind], (mode, err)


@pytest.mark.parametrize("case", [c for c in CASES if c[0] != "q8"], ids=[i for c, i in zip(CASES, IDS) if c[0] != "q8"])
def test_paged_ordered_art_matches_oracle(case):
    w, pg = make(*case, seed=1)
    art = dict(ART, lanes=I.probe_lanes_strided(w.d, 16 if w.d == 128 else 8))
    order = orders.tile_order_recency(w.seq_lens, w.Hkv, w.L_max, w.tile, w.num_splits)
    g = gpu(w, pg, "art", art=art, order=order)
    assert g["status"] == capi.ART_OK and np.isfinite(g["o"]).all()
    ref = oracle_paged(w, pg, "art", art=art, metrics=True, tile_order=order)
    check_tiles(w, ref.metrics, g["used"], art, w.tile, w.num_splits)
    forced = oracle_paged(w, pg, "full", forced_used=g["used"], tile_order=order)
    assert np.max(np.abs(g["o"] - forced.o)) <= TOL[w.kind]


def test_paged_equals_contiguous_on_the_gpu():
    """The same kernel over the same bytes in two layouts."""
    for case in (CASES[0], CASES[3]):
        w, pg = make(*case, seed=2)
        for mode in ("full", "art"):
            a = dict(ART, lanes=[0, 8, 16]) if mode == "art" else None
            g = gpu(w, pg, mode, art=a)
            dp = K.upload(w)
            K.decode(dp, mode, art=a)
            assert np.max(np.abs(g["o"] - dp.o.cpu().numpy())) <= 1e-6
            assert np.array_equal(g["tiles"], dp.tiles.cpu().numpy())


def test_shared_prefix_pages_on_the_gpu():
    w, pg = make("bf16", 128, 4, 1, 2, 1024, [1024, 1024], 64, 1, 128, seed=3)
    w.q[1] = w.q[0]
    pg.block_table[1] = pg.block_table[0]
    g = gpu(w, pg, "full")
    assert np.array_equal(g["o"][0], g["o"][1])


def test_bad_block_table_entry_is_flagged():
    for case in (CASES[0], CASES[4]):
        w, pg = make(*case)
        pg.block_table[0, 1] = pg.num_pages + 7
        g = gpu(w, pg, "full")
        assert g["status"] == capi.ART_ERR_PAGE
