"""The five synthetic workloads at their full sizes, in the launch configuration
the benchmark times.  The GPU runs the whole problem; outputs of sampled
(batch, kv head) slabs are checked element by element against the oracle on
the same slab (built bit-identically by the seeded generator), and properties
that hold at any size are checked on every head.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import kv_cache_early_split_b200 as K  # noqa: E402
from kv_cache_early_split_b200 import capi  # noqa: E402
from kv_cache_early_split_b200 import inputs as I  # noqa: E402
from helpers import TOL, check_tiles, oracle_run  # noqa: E402

pytestmark = pytest.mark.gpu

# (workload, modes, sampled (b, kvh) slabs)
CASES = [
    ("fp32_b1_h1_d64_L4k", ("full", "art"), [(0, 0)]),
    ("gqa_b4_h32x8_d128_L32k", ("full", "art"), [(0, 0), (3, 5)]),
    ("gqa_b1_h32x8_d128_L128k", ("full", "art"), [(0, 2)]),
    ("split_b16_h32x8_d128_Lvar", ("full", "art"), [(2, 1), (11, 7)]),
    ("q8_b2_h32x8_d128_L32k", ("q8", "q8_art"), [(1, 3)]),
]

_cache = {}


def full_workload(name):
    if name not in _cache:
        _cache.clear()
        _cache[name] = I.workload(name)
    return _cache[name]


@pytest.mark.parametrize("name,modes,slabs", CASES, ids=[c[0] for c in CASES])
def test_workload(name, modes, slabs):
    w = full_workload(name)
    dp = K.upload(w)
    n = -(-w.seq_lens.astype(np.int64) // w.tile)
    S, G = w.num_splits, w.G
    for mode in modes:
        K.decode(dp, mode)
        assert K.device_status(dp) == capi.ART_OK
        o = dp.o.cpu().numpy()
        tiles = dp.tiles.cpu().numpy()
        used = dp.split_tiles().cpu().numpy()
        read = dp.tiles_read().cpu().numpy()
        assert np.all(np.isfinite(o))
        assert np.array_equal(used.sum(axis=2), tiles)
        assert np.all(tiles >= 1) and np.all(tiles <= n[:, None])
        art_mode = mode in ("art", "q8_art")
        if not art_mode:
            assert np.array_equal(tiles, np.repeat(n[:, None], w.Hq, axis=1))
        for b in range(w.B):
            for h in range(w.Hkv):
                need = used[b, h * G:(h + 1) * G].max(axis=0)
                assert np.all(read[b, h] >= need)
        for (b, h) in slabs:
            ws = I.workload(name, keys_b=[b], keys_h=[h])
            assert np.array_equal(ws.k[0, 0], w.k[b, h]) and np.array_equal(ws.q[0], w.q[b, h * G:(h + 1) * G])
            sl = slice(h * G, (h + 1) * G)
            if art_mode:
                ref = oracle_run(ws, mode, metrics=True)
                exact, amb = check_tiles(ws, ref.metrics, used[b:b + 1, sl], ws.art, ws.tile, S)
                forced = oracle_run(ws, "q8" if mode == "q8_art" else "full", forced_used=used[b:b + 1, sl])
                err = np.max(np.abs(o[b, sl] - forced.o[0]))
                print(f"{name} {mode} slab ({b},{h}): tiles {tiles[b, sl]} of {n[b]} exact={exact} amb={amb} err={err:.2e}")
            else:
                ref = oracle_run(ws, mode)
                err = np.max(np.abs(o[b, sl] - ref.o[0]))
                print(f"{name} {mode} slab ({b},{h}): err={err:.2e}")
            assert err <= TOL[w.kind]
