"""GPU parity of random eviction ahead of ART: selection and packing bit-exact against
the oracle (integer and byte work), the decode on the packed cache within the usual bars."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import kv_cache_early_split_b200 as K  # noqa: E402
from kv_cache_early_split_b200 import capi  # noqa: E402
from kv_cache_early_split_b200 import inputs as I  # noqa: E402
from oracle import evict  # noqa: E402
from helpers import KIND, TOL, check_tiles  # noqa: E402

pytestmark = pytest.mark.gpu


def keys_for(w, seed, hi=2**32):
    rng = np.random.default_rng(seed)
    return rng.integers(0, hi, (w.B, w.Hkv, w.L_max), dtype=np.uint64).astype(np.uint32)


def dev_keys(keys):
    return torch.from_numpy(keys.view(np.int32)).cuda()


SEL = [
    # L_max, lens, sink, recent, budget, key range
    (4096, [4096, 3000, 100], 16, 256, 1024, 2**32),
    (4096, [4096, 2500], 16, 256, 1024, 4),          # heavy ties
    (1000, [1000, 999], 0, 0, 37, 2**32),            # no sink, no recent window
    (1000, [1000, 10], 20, 30, 50, 2**32),           # m = 0: sink and recent only
    (32768, [32768], 64, 1024, 8192, 2**32),         # the 4x budget on a 32K sequence
    (300, [300, 300], 1, 1, 299, 7),
]


@pytest.mark.parametrize("case", SEL)
def test_selection_matches_oracle(case):
    L_max, lens, sink, recent, budget, hi = case
    w = I.make_workload(kind="bf16", B=len(lens), Hq=4, Hkv=2, d=64, L_max=L_max, tile=64, seq_lens=lens, seed=1)
    keys = keys_for(w, 5, hi)
    dp = K.upload(w)
    dp2, kept = K.evict_random(dp, dev_keys(keys), sink, recent, budget)
    ref = evict.select(w.seq_lens, keys, sink, recent, budget)
    assert np.array_equal(kept.cpu().numpy(), ref)
    assert np.array_equal(dp2.seq_lens.cpu().numpy(), np.minimum(w.seq_lens, budget))


def test_bad_seq_len_keeps_nothing():
    w = I.make_workload(kind="bf16", B=2, Hq=2, Hkv=1, d=64, L_max=256, tile=64, seq_lens=[256, 200], seed=1)
    w.seq_lens[1] = 999
    dp = K.upload(w)
    dp2, kept = K.evict_random(dp, dev_keys(keys_for(w, 1)), 4, 8, 64)
    assert np.all(kept.cpu().numpy()[1] == -1) and dp2.seq_lens.cpu().numpy().tolist() == [64, 0]


PACK = [
    ("f32", 64, [500, 120], 128),
    ("bf16", 128, [2048, 1500], 512),
    ("q8", 128, [2048, 700], 512),
    ("q8", 64, [1000, 999], 256),
]


@pytest.mark.parametrize("case", PACK, ids=lambda c: f"{c[0]}-d{c[1]}")
def test_packed_cache_and_decode_match_oracle(case):
    kind, d, lens, budget = case
    w = I.make_workload(kind=kind, B=2, Hq=8, Hkv=2, d=d, L_max=max(lens), tile=64, seq_lens=lens, seed=4, sink=6.0)
    keys = keys_for(w, 9)
    dp = K.upload(w)
    dp2, kept = K.evict_random(dp, dev_keys(keys), 16, 64, budget)
    ref_kept = evict.select(w.seq_lens, keys, 16, 64, budget)
    assert np.array_equal(kept.cpu().numpy(), ref_kept)
    for name in ("k", "v", "k_scale", "v_scale"):
        x = getattr(w, name)
        if x is None:
            continue
        got = getattr(dp2, name).cpu().numpy().view(x.dtype)
        assert np.array_equal(got, evict.compact(x, ref_kept)), name
    lanes = I.probe_lanes_strided(d, 16 if d == 128 else 8)
    art = dict(eps_scale=2e-2, eps_dir=5e-3, patience=2, lanes=lanes)
    modes = [("q8", None, 1e-3), ("q8_art", art, 1e-3)] if kind == "q8" else [("full", None, None), ("art", art, None)]
    for mode, a, tau in modes:
        K.decode(dp2, mode, art=a, tau=tau)
        assert K.device_status(dp2) == capi.ART_OK
        o, used = dp2.o.cpu().numpy(), dp2.split_tiles().cpu().numpy()
        wp = I.make_workload(kind=kind, B=2, Hq=8, Hkv=2, d=d, L_max=budget, tile=64,
                             seq_lens=np.minimum(w.seq_lens, budget), seed=4)
        base = dict(kind=KIND[kind], q=w.q, k=w.k, v=w.v, k_scale=w.k_scale, v_scale=w.v_scale, seq_lens=w.seq_lens,
                    keys=keys, n_sink=16, n_recent=64, budget=budget, tile=64, n_threads=8,
                    tau=(tau if kind == "q8" else 0.0))
        if a is None:
            ref, _ = evict.decode_evicted(**base)
            assert np.array_equal(used, ref.used)
        else:
            ref, _ = evict.decode_evicted(**base, art=a, want_metrics=True, no_break=True)
            check_tiles(wp, ref.metrics, used, a, 64, 1)
            ref, _ = evict.decode_evicted(**base, forced_used=used)
        assert np.max(np.abs(o - ref.o)) <= TOL[kind], mode
