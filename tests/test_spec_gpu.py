"""The bound on speculative reads (art_params.max_spec_tiles) on the tensor-core kernel.

A call with a bound must give exactly the results of the same call without one (the bound
only changes which K/V tiles are fetched), and per (batch, kv head, split) unit it may fetch no
tile that starts a round at or past (tiles the unit consumed) + bound: at most
consumed + bound + (tiles per round - 1) tiles.  A round holds C * 128 / tile tiles for a
cluster of C CTAs, at most 32.  Each case is also checked against the oracle.

Cases: cluster kernels where every tile holds (every head stops at exactly `patience` tiles; in
one the first wait comes after more rounds than the decision barriers have slots), a
single-CTA-cluster kernel (four splits per sequence, 256 units) with the pages' rule on a
sink-heavy workload, and the q8 tensor-core kernel.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import kv_cache_early_split_b200 as K  # noqa: E402
from kv_cache_early_split_b200 import capi  # noqa: E402
from kv_cache_early_split_b200 import inputs as I  # noqa: E402
from helpers import TOL, oracle_run  # noqa: E402

pytestmark = pytest.mark.gpu

LANES = I.probe_lanes_strided(128, 16)
ALL_HOLD = dict(eps_scale=1e9, eps_dir=1e9, patience=40, lanes=LANES)

CASES = [
    # name, workload, mode, caps, largest tiles-per-round of its launch
    ("bf16-cluster-all-hold",
     dict(kind="bf16", B=2, Hq=8, Hkv=2, L_max=16384, seq_lens=[16384, 11000], art=ALL_HOLD), "art", (1, 20), 32),
    # 128 tiles per unit, 4-CTA clusters (8 tiles a round): the safe point starts 12 rounds ahead,
    # more rounds than the decision barriers have slots, before the first wait
    ("bf16-cluster-late-first-wait",
     dict(kind="bf16", B=4, Hq=32, Hkv=8, L_max=8192, art=dict(ALL_HOLD, patience=96)), "art", (1, 5), 32),
    ("bf16-single-cta",
     dict(kind="bf16", B=16, Hq=32, Hkv=8, L_max=8192, num_splits=4, seq_lens=("uniform", 3000, 8192), sink=8.0,
          art=dict(eps_scale=5e-2, eps_dir=1e-2, patience=2, lanes=LANES)), "art", (1, 4), 2),
    ("q8-cluster",
     dict(kind="q8", B=1, Hq=4, Hkv=1, L_max=8192, tau=1e-6, art=dict(ALL_HOLD, patience=24)), "q8_art", (1, 8), 32),
]


def run(dp, mode, art, cap):
    dp.o.fill_(float("nan"))
    dp.tiles.fill_(-1)
    q8 = {"q8_path": "tensor_core"} if mode == "q8_art" else {}
    K.decode(dp, mode, art=dict(art, max_spec_tiles=cap), **q8)
    assert K.device_status(dp) == capi.ART_OK
    torch.cuda.synchronize()
    return dp.o.cpu().numpy(), dp.tiles.cpu().numpy(), dp.tiles_read().cpu().numpy(), dp.split_tiles().cpu().numpy()


@pytest.mark.parametrize("name,kw,mode,caps,tq_max", CASES, ids=[c[0] for c in CASES])
def test_bounded_speculation_same_results_fewer_reads(name, kw, mode, caps, tq_max):
    w = I.make_workload(d=128, tile=64, seed=47, **kw)
    dp = K.upload(w)
    # (q8: the decode kernel is pinned by path; the query names the default, the two-pass rule)
    assert K.kernel_name(dp, mode) == ("q8_pv_mma_kernel" if mode == "q8_art" else "art_decode_tc_kernel"), name
    o0, t0, r0, s0 = run(dp, mode, w.art, 0)
    # the oracle, run to the GPU's own stop tiles
    ref = oracle_run(w, "q8" if mode == "q8_art" else "full", forced_used=s0)
    assert float(np.max(np.abs(o0 - ref.o))) <= TOL[w.kind]
    G = w.Hq // w.Hkv
    used_unit = s0.reshape(w.B, w.Hkv, G, -1).max(axis=2)  # [B, Hkv, S]: tiles the unit consumed
    for cap in caps:
        o, t, r, s = run(dp, mode, w.art, cap)
        assert np.array_equal(t, t0) and np.array_equal(s, s0), (name, cap)
        assert np.array_equal(o, o0), (name, cap)
        assert K.device_status(dp) == capi.ART_OK
        bound = used_unit + cap + tq_max - 1
        assert np.all(r <= bound), (name, cap, int(np.max(r - bound)))
        print(name, "cap", cap, "read/consumed", float(r.sum()) / float(used_unit.sum()),
              "uncapped", float(r0.sum()) / float(used_unit.sum()))
