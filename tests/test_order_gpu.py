"""GPU parity of the tile traversal orders ("Resumen Tecnico: ART", S2.4) through the C ABI.

* Recency sequences: bit-exact against the oracle's builder.
* Key summaries: within fp32 rounding of the oracle's float64 means.
* Importance sequences (scores in fp32 on the GPU, float64 in the oracle): every
  split segment is a permutation of the split's tiles with its first tile first, the
  oracle's scores along it never rise by more than a rounding window, and nearly all
  positions agree with the oracle's sequence.
* Ordered ART decode: GPU and oracle walk the SAME sequences (built by the oracle), with
  the tile acceptance rule and output bars of the other parity tests.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import kv_cache_early_split_b200 as K  # noqa: E402
from kv_cache_early_split_b200 import capi  # noqa: E402
from kv_cache_early_split_b200 import inputs as I  # noqa: E402
from oracle import orders  # noqa: E402
from helpers import TOL, check_tiles, oracle_run  # noqa: E402

pytestmark = pytest.mark.gpu

CASES = [
    # kind, d, Hq, Hkv, B, L_max, lens, tile, S   (the first three take the tensor-core kernel)
    ("bf16", 128, 8, 2, 2, 3000, [3000, 1290], 64, 1),
    ("bf16", 128, 4, 2, 2, 4096, [4096, 1000], 128, 2),
    ("bf16", 128, 8, 1, 1, 5000, [4999], 64, 3),
    ("bf16", 64, 8, 2, 2, 2000, [2000, 777], 32, 1),
    ("f32", 128, 4, 2, 2, 1500, [1500, 333], 64, 2),
    ("f32", 64, 2, 2, 1, 1000, [1000], 16, 1),
]
IDS = [f"{c[0]}-d{c[1]}-g{c[2] // c[3]}-T{c[7]}-S{c[8]}" for c in CASES]


def make(kind, d, Hq, Hkv, B, L_max, lens, tile, S, seed=0):
    return I.make_workload(kind=kind, B=B, Hq=Hq, Hkv=Hkv, d=d, L_max=L_max, tile=tile, num_splits=S,
                           seq_lens=lens, seed=2000 + seed, sink=6.0, gumbel_scale=1.5)


def decoded(w):
    kind = {"f32": 0, "bf16": 1}[w.kind]
    return orders.decode_rows(kind, w.q), orders.decode_rows(kind, w.k)


def oracle_orders(w):
    qd, kd = decoded(w)
    rec = orders.tile_order_recency(w.seq_lens, w.Hkv, w.L_max, w.tile, w.num_splits)
    mu = orders.tile_key_summary(kd, w.seq_lens, w.tile)
    sc = orders.tile_importance(qd, mu, w.seq_lens, w.tile)
    imp = orders.tile_order_importance(sc, w.seq_lens, w.tile, w.num_splits)
    return rec, mu, sc, imp


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_recency_and_summary_match_oracle(case):
    w = make(*case)
    dp = K.upload(w)
    rec, mu, _, _ = oracle_orders(w)
    g_rec = K.tile_order(dp, "recency").cpu().numpy()
    assert np.array_equal(g_rec, rec)
    g_mu = K.key_summary(dp).cpu().numpy()
    assert np.max(np.abs(g_mu - mu)) <= 1e-5 * max(1.0, np.abs(mu).max())


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_importance_order_is_valid_and_agrees(case):
    w = make(*case)
    dp = K.upload(w)
    _, _, sc, imp = oracle_orders(w)
    g = K.tile_order(dp, "importance").cpu().numpy()
    window = 1e-4 * max(1.0, np.abs(sc[np.isfinite(sc)]).max())
    agree = total = 0
    for b in range(w.B):
        n = -(-int(w.seq_lens[b]) // w.tile)
        for h in range(w.Hkv):
            assert np.all(g[b, h, n:] == -1)
            for ta, tb in orders.split_segments(n, w.num_splits):
                seg = g[b, h, ta:tb]
                assert sorted(seg.tolist()) == list(range(ta, tb)) and (tb == ta or seg[0] == ta)
                s = sc[b, h, seg[1:]]
                assert np.all(np.diff(s) <= window)
            agree += int(np.sum(g[b, h, :n] == imp[b, h, :n]))
            total += n
    assert agree >= 0.9 * total, (agree, total)


def run_ordered(w, order, art):
    dp = K.upload(w)
    order_d = torch.from_numpy(np.ascontiguousarray(order, dtype=np.int32)).to(dp.k.device)
    K.decode(dp, "art", art=art, order=order_d)
    st = K.device_status(dp)
    return dict(o=dp.o.cpu().numpy(), tiles=dp.tiles.cpu().numpy(), used=dp.split_tiles().cpu().numpy(),
                read=dp.tiles_read().cpu().numpy(), status=st)


ART_SETTINGS = [
    dict(eps_scale=2e-2, eps_dir=5e-3, patience=1),
    dict(eps_scale=5e-2, eps_dir=2e-2, patience=2),
    dict(eps_scale=0.0, eps_dir=0.0, patience=1),
]


@pytest.mark.parametrize("which", ["recency", "importance"])
@pytest.mark.parametrize("setting", range(len(ART_SETTINGS)))
@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_ordered_art_matches_oracle(case, setting, which):
    w = make(*case, seed=setting)
    rec, _, _, imp = oracle_orders(w)
    order = rec if which == "recency" else imp
    a = dict(ART_SETTINGS[setting], lanes=I.probe_lanes_strided(w.d, 16 if w.d == 128 else 8))
    g = run_ordered(w, order, a)
    assert g["status"] == capi.ART_OK
    ref = oracle_run(w, "art", art=a, metrics=True, tile_order=order)
    check_tiles(w, ref.metrics, g["used"], a, w.tile, w.num_splits)
    forced = oracle_run(w, "full", forced_used=g["used"], tile_order=order)
    err = np.max(np.abs(g["o"] - forced.o))
    assert err <= TOL[w.kind], f"max abs err {err}"
    if a["eps_scale"] == 0.0:  # never stops: full attention, whatever the order
        full = oracle_run(w, "full")
        assert np.max(np.abs(g["o"] - full.o)) <= TOL[w.kind]
        n = -(-w.seq_lens.astype(np.int64) // w.tile)
        assert np.array_equal(g["tiles"], np.repeat(n[:, None], w.Hq, axis=1))


@pytest.mark.parametrize("case", CASES[:3] + CASES[4:5], ids=IDS[:3] + IDS[4:5])
def test_recency_with_inf_thresholds_reads_first_and_newest(case):
    w = make(*case)
    rec = orders.tile_order_recency(w.seq_lens, w.Hkv, w.L_max, w.tile, w.num_splits)
    for p in (1, 3):
        a = dict(eps_scale=float("inf"), eps_dir=float("inf"), patience=p, lanes=[0, 7, 33])
        g = run_ordered(w, rec, a)
        assert g["status"] == capi.ART_OK
        ref = oracle_run(w, "art", art=a, tile_order=rec)
        assert np.array_equal(g["used"], ref.used)
        assert np.max(np.abs(g["o"] - ref.o)) <= TOL[w.kind]


def test_entry_outside_its_split_is_flagged():
    w = make("bf16", 128, 8, 2, 2, 3000, [3000, 1290], 64, 2)
    rec = orders.tile_order_recency(w.seq_lens, w.Hkv, w.L_max, w.tile, 2)
    bad = rec.copy()
    bad[0, 1, 1] = 40  # split 0 covers tiles [0, 23); 40 belongs to split 1
    g = run_ordered(w, bad, dict(eps_scale=0.0, eps_dir=0.0, patience=1, lanes=[0, 1]))
    assert g["status"] == capi.ART_ERR_ORDER
    w2 = make("f32", 64, 2, 2, 1, 1000, [1000], 16, 1)
    rec2 = orders.tile_order_recency(w2.seq_lens, w2.Hkv, w2.L_max, w2.tile, 1)
    rec2[0, 0, 5] = 10_000
    g2 = run_ordered(w2, rec2, dict(eps_scale=0.0, eps_dir=0.0, patience=1, lanes=[0, 1]))
    assert g2["status"] == capi.ART_ERR_ORDER
