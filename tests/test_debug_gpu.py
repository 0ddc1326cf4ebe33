"""The debug build (libart_decode_debug.so, compiled with -DART_DEBUG): device index checks in
front of the kernels' copies and writes that set the status word's index bit -- ART_ERR_INDEX --
instead of trapping (the stand-in for the sanitizer this pool does not offer).

Every kernel family runs through the debug library on small shapes chosen for their edges (a
tile that does not divide the length, a sequence shorter than one tile, length 1, splits,
3 heads per kv head padded to 4, clusters): each call must report ART_OK -- no check fired --
and match the oracle with the parity tests' tolerances (re-run to the GPU's own stop tiles for
ART).  The library swap is local to this module.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import kv_cache_early_split_b200 as K  # noqa: E402
from kv_cache_early_split_b200 import build, capi  # noqa: E402
from kv_cache_early_split_b200 import inputs as I  # noqa: E402
from helpers import TOL, oracle_run  # noqa: E402

pytestmark = pytest.mark.gpu

LANES = I.probe_lanes_strided(128, 16)


@pytest.fixture(scope="module", autouse=True)
def debug_library():
    saved = capi._lib
    capi._lib = capi.load_variant(build.build_debug())
    yield
    capi._lib = saved


def run(w, mode, art=None, q8_path="auto", order=None):
    dp = K.upload(w)
    K.decode(dp, mode, art=art, q8_path=q8_path, order=order)
    assert K.device_status(dp) == capi.ART_OK, capi.art_status_string(K.device_status(dp))
    return dp.o.cpu().numpy(), dp.split_tiles().cpu().numpy()


def check(w, mode, art=None, q8_path="auto"):
    o, used = run(w, mode, art=art, q8_path=q8_path)
    base = {"art": "full", "full": "full", "q8": "q8", "q8_art": "q8"}[mode]
    ref = oracle_run(w, base, forced_used=used if mode in ("art", "q8_art") else None)
    assert float(np.max(np.abs(o - ref.o))) <= TOL[w.kind], mode


CASES = [
    # bf16, tensor cores: T does not divide the lengths, a sequence shorter than a tile, length 1, splits
    ("bf16-tc", dict(kind="bf16", B=4, Hq=16, Hkv=4, d=128, L_max=3000, tile=64, num_splits=3,
                     seq_lens=[3000, 1000, 37, 1], sink=6.0), ("full", "art")),
    # bf16, tensor cores, clusters (one unit: the cluster takes the SMs), tile 128, 3 heads per kv head
    ("bf16-tc-cluster", dict(kind="bf16", B=1, Hq=6, Hkv=2, d=128, L_max=8000, tile=128, seq_lens=[7777],
                             sink=6.0), ("full", "art")),
    # fp32, CUDA cores, d = 64
    ("f32-cuda-core", dict(kind="f32", B=2, Hq=4, Hkv=1, d=64, L_max=777, tile=32, num_splits=2,
                           seq_lens=[777, 100]), ("full", "art")),
    # q8: two passes on the tensor cores (full) and the tensor-core kernel (ART)
    ("q8-tc", dict(kind="q8", B=2, Hq=8, Hkv=2, d=128, L_max=2000, tile=64, num_splits=2, seq_lens=[2000, 333],
                   tau=1e-3, sink=6.0, gumbel_scale=2.0), ("q8", "q8_art")),
    # q8, d = 64: two passes and the one-pass kernel on the CUDA cores
    ("q8-cuda-core", dict(kind="q8", B=1, Hq=4, Hkv=2, d=64, L_max=1500, tile=32, seq_lens=[1499], tau=1e-3),
     ("q8", "q8_art")),
]


@pytest.mark.parametrize("name,kw,modes", CASES, ids=[c[0] for c in CASES])
def test_debug_build_no_index_check_fires(name, kw, modes):
    art = dict(eps_scale=2e-2, eps_dir=5e-3, patience=2, lanes=LANES if kw["d"] == 128 else list(range(8)))
    w = I.make_workload(seed=73, art=art, **kw)
    for mode in modes:
        check(w, mode, art=art if mode in ("art", "q8_art") else None)


def test_debug_build_ordered_and_bounded_speculation():
    """Recency-ordered ART and ART with a speculation bound on the tensor-core kernel."""
    art = dict(eps_scale=1e9, eps_dir=1e9, patience=24, lanes=LANES)
    w = I.make_workload(kind="bf16", B=2, Hq=8, Hkv=2, d=128, L_max=6000, tile=64, num_splits=2,
                        seq_lens=[6000, 2500], seed=74, art=art)
    dp = K.upload(w)
    order = K.tile_order(dp, "recency")
    o, used = run(w, "art", art=art, order=order)
    ref = oracle_run(w, "full", forced_used=used, tile_order=order.cpu().numpy())
    assert float(np.max(np.abs(o - ref.o))) <= TOL["bf16"]
    check(w, "art", art=dict(art, max_spec_tiles=1))
