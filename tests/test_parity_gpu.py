"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, element
by element, on seeded synthetic inputs that span several tiles and a ragged
tail, for every entry point and mode, plus edge cases.

Bars: outputs within 1e-5 (fp32 inputs) or 2e-3 (bf16 / q8 inputs) max-abs of
the oracle run to the GPU's own per-split stop tiles; tiles consumed equal to
the oracle's unless an oracle metric lies within 1e-4 of its threshold (see
tests/helpers.py).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import kv_cache_early_split_b200 as K  # noqa: E402
from kv_cache_early_split_b200 import capi  # noqa: E402
from kv_cache_early_split_b200 import inputs as I  # noqa: E402
from helpers import TOL, check_tiles, oracle_run  # noqa: E402

pytestmark = pytest.mark.gpu


def q8_paths(w, mode, tile=None):
    """The q8 implementations that take this shape and mode (art_decode_attn_q8_skipv_path)."""
    T = tile or w.tile
    paths = ["cluster"]
    if mode == "q8" or (w.d == 128 and w.G in (3, 4) and T >= 32):
        paths.append("two_pass")  # (ART: the rule over probe records, on the tensor-core passes)
    if w.d == 128 and w.G in (3, 4) and T in (64, 128) and w.L_max % 2 == 0:
        paths.append("tensor_core")
    return paths


def gpu(w, mode, *, tile=None, S=None, art=None, tau=None, stream=None, q8_path="auto"):
    dp = K.upload(w, num_splits=S, tile=tile)
    K.decode(dp, mode, art=art, tau=tau, stream=stream, q8_path=q8_path)
    st = K.device_status(dp, stream=stream)
    return dict(
        o=dp.o.cpu().numpy(), tiles=dp.tiles.cpu().numpy(), used=dp.split_tiles().cpu().numpy(),
        read=dp.tiles_read().cpu().numpy(), status=st, dp=dp,
    )


def n_tiles(w, tile):
    return -(-w.seq_lens.astype(np.int64) // tile)


def check_full(w, mode="full", tile=None, S=None, tau=None, q8_path="auto"):
    tile = tile or w.tile
    S = S or w.num_splits
    g = gpu(w, mode, tile=tile, S=S, tau=tau, q8_path=q8_path)
    assert g["status"] == capi.ART_OK
    r = oracle_run(w, mode, tile=tile, num_splits=S, tau=tau)
    err = np.max(np.abs(g["o"] - r.o))
    assert err <= TOL[w.kind], f"max abs err {err}"
    n = n_tiles(w, tile)
    assert np.array_equal(g["tiles"], np.repeat(n[:, None], w.Hq, axis=1))
    assert np.array_equal(g["used"], r.used)
    assert np.array_equal(g["read"].sum(axis=2), np.repeat(n[:, None], w.Hkv, axis=1))
    return g


def check_art(w, mode="art", tile=None, S=None, art=None, tau=None, q8_path="auto"):
    tile = tile or w.tile
    S = S or w.num_splits
    a = art or w.art
    g = gpu(w, mode, tile=tile, S=S, art=a, tau=tau, q8_path=q8_path)
    assert g["status"] == capi.ART_OK
    ref = oracle_run(w, mode, tile=tile, num_splits=S, art=a, tau=tau, metrics=True)
    exact, amb = check_tiles(w, ref.metrics, g["used"], a, tile, S)
    assert np.array_equal(g["used"].sum(axis=2), g["tiles"])
    forced = oracle_run(w, "q8" if mode == "q8_art" else "full", tile=tile, num_splits=S, tau=tau,
                        forced_used=g["used"])
    err = np.max(np.abs(g["o"] - forced.o))
    assert err <= TOL[w.kind], f"max abs err {err}"
    # KV tiles read per (b, kvh, split): at least what the slowest head consumed, at most the split
    n = n_tiles(w, tile)
    G = w.G
    for b in range(w.B):
        for s in range(S):
            ln = ((s + 1) * n[b]) // S - (s * n[b]) // S
            for h in range(w.Hkv):
                need = g["used"][b, h * G:(h + 1) * G, s].max()
                assert need <= g["read"][b, h, s] <= ln
    return g, exact, amb


SMALL = [
    # kind, d, Hq, Hkv, B, L_max, lens, tile, S
    ("f32", 64, 1, 1, 1, 1000, [1000], 64, 1),
    ("f32", 128, 8, 2, 2, 700, [700, 333], 32, 2),
    ("bf16", 128, 8, 2, 2, 2000, [2000, 777], 64, 1),
    ("bf16", 64, 8, 1, 3, 500, [500, 17, 250], 16, 1),
    ("bf16", 128, 4, 2, 2, 3000, [2999, 1290], 128, 3),
    ("bf16", 128, 6, 2, 2, 900, [900, 45], 32, 1),
    ("bf16", 128, 2, 1, 1, 5000, [4999], 64, 1),
    ("bf16", 64, 16, 2, 2, 1200, [1200, 1], 64, 2),
    ("bf16", 64, 4, 4, 1, 2048, [2048], 256, 1),
    ("q8", 128, 8, 2, 2, 2048, [2048, 1001], 64, 1),
    ("q8", 64, 4, 1, 1, 1500, [1499], 32, 2),
]


def make_small(kind, d, Hq, Hkv, B, L_max, lens, tile, S, seed=0, **kw):
    return I.make_workload(kind=kind, B=B, Hq=Hq, Hkv=Hkv, d=d, L_max=L_max, tile=tile, num_splits=S,
                           seq_lens=lens, seed=1000 + seed, **kw)


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"{c[0]}-d{c[1]}-g{c[2] // c[3]}-T{c[7]}-S{c[8]}")
def test_full_small(case):
    w = make_small(*case)
    if w.kind == "q8":
        for path in q8_paths(w, "q8"):  # tensor cores / two streaming passes / one pass over a cluster
            check_full(w, "q8", tau=0.0, q8_path=path)
            check_full(w, "q8", tau=1e-6, q8_path=path)
    else:
        check_full(w)


ART_SETTINGS = [
    dict(eps_scale=2e-2, eps_dir=5e-3, patience=1),
    dict(eps_scale=5e-2, eps_dir=2e-2, patience=3),
    dict(eps_scale=float("inf"), eps_dir=float("inf"), patience=2),
    dict(eps_scale=0.0, eps_dir=0.0, patience=1),
    dict(eps_scale=2e-2, eps_dir=float("inf"), patience=2),  # magnitude criterion only
    dict(eps_scale=float("inf"), eps_dir=5e-3, patience=4),  # direction criterion only
]


@pytest.mark.parametrize("setting", range(len(ART_SETTINGS)))
@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"{c[0]}-d{c[1]}-g{c[2] // c[3]}-T{c[7]}-S{c[8]}")
def test_art_small(case, setting):
    w = make_small(*case, seed=setting, sink=6.0)
    a = dict(ART_SETTINGS[setting], lanes=I.probe_lanes_strided(w.d, 16 if w.d == 128 else 8))
    mode = "q8_art" if w.kind == "q8" else "art"
    for path in (q8_paths(w, mode) if w.kind == "q8" else ["auto"]):
        g, exact, amb = check_art(w, mode, art=a, tau=(1e-6 if w.kind == "q8" else None), q8_path=path)
        n = n_tiles(w, w.tile)
        S = w.num_splits
        if a["eps_scale"] == float("inf") and a["eps_dir"] == float("inf"):
            for b in range(w.B):
                lens = [((s + 1) * n[b]) // S - (s * n[b]) // S for s in range(S)]
                assert np.array_equal(g["used"][b], np.tile([min(a["patience"], x) for x in lens], (w.Hq, 1)))
        if a["eps_scale"] == 0.0:
            assert np.array_equal(g["tiles"], np.repeat(n[:, None], w.Hq, axis=1))


def test_art_stops_somewhere_midway():
    """A case where the rule fires inside the sequence for most heads (not at the ends)."""
    w = make_small("bf16", 128, 8, 2, 2, 4096, [4096, 3000], 64, 1, sink=8.0)
    a = dict(eps_scale=5e-2, eps_dir=1e-2, patience=2, lanes=I.probe_lanes_strided(128, 16))
    g, exact, amb = check_art(w, art=a)
    n = n_tiles(w, 64)
    mid = (g["tiles"] > 2) & (g["tiles"] < n[:, None])
    assert mid.mean() > 0.5, g["tiles"]


def test_vskip_actually_skips_and_matches():
    """Skewed logits so that many rows fall below tau; GPU matches the oracle's skip rule."""
    w = I.make_workload(kind="q8", B=1, Hq=4, Hkv=1, d=128, L_max=2048, tile=64, seed=5, gumbel_scale=6.0,
                        q_scale=2.0)
    for tau in (1e-3, 1e-6, 0.0, 2.0):
        for path in q8_paths(w, "q8"):
            check_full(w, "q8", tau=tau, q8_path=path)
        for path in q8_paths(w, "q8_art"):
            check_art(w, "q8_art", tau=tau, q8_path=path,
                      art=dict(eps_scale=2e-2, eps_dir=5e-3, patience=2, lanes=I.probe_lanes_strided(128, 16)))
    full = oracle_run(w, "q8", tau=0.0)
    skip = oracle_run(w, "q8", tau=1e-3)
    assert np.max(np.abs(full.o - skip.o)) > 1e-6  # the skip changed something measurable


Q8_TWO_PASS = [
    # d, Hq, Hkv, B, L_max, lens, tile, S: every head-group width (1, 2, 3 -> 4, 4, 8), d = 64 / 128,
    # chunks of 32 / 16 / 8 tiles (several per split), ragged tails, length 1, empty splits
    (128, 8, 8, 2, 4096, [4096, 1], 16, 1),
    (64, 8, 4, 2, 3000, [2999, 1500], 32, 3),
    (128, 6, 2, 1, 5000, [4937], 64, 2),
    (128, 8, 2, 2, 4500, [4500, 2047], 64, 1),
    (64, 16, 2, 3, 2500, [2500, 777, 3], 128, 4),
    (128, 8, 1, 1, 4096, [4096], 256, 1),
    (128, 32, 8, 1, 2048, [2000], 64, 8),
    # the tensor-core passes (d = 128, 3 or 4 heads, tile >= 32): 32-row steps at tile 32 with a
    # length that ends inside a step and a tensor end inside a box (L_max = 3002), tiles of 128 and
    # 256, a sequence shorter than one step
    (128, 8, 2, 2, 3002, [2999, 20], 32, 3),
    (128, 12, 3, 1, 6000, [5999], 128, 2),
    (128, 4, 1, 2, 4096, [4096, 300], 256, 1),
]


@pytest.mark.parametrize("case", Q8_TWO_PASS, ids=lambda c: f"d{c[0]}-g{c[1] // c[2]}-T{c[6]}-S{c[7]}")
def test_q8_two_pass_shapes(case):
    d, Hq, Hkv, B, L_max, lens, tile, S = case
    w = I.make_workload(kind="q8", B=B, Hq=Hq, Hkv=Hkv, d=d, L_max=L_max, tile=tile, num_splits=S,
                        seq_lens=lens, seed=77 + tile, gumbel_scale=3.0, q_scale=1.5)
    for tau in (0.0, 1e-4):
        for path in q8_paths(w, "q8"):
            check_full(w, "q8", tau=tau, q8_path=path)


def test_q8_two_pass_skips_whole_tiles():
    """A sink key far above every other score: after its tile almost every row of every head
    falls below tau, so the two-pass path leaves whole V tiles unread; outputs still match the
    oracle's row rule, and the same call over a one-pass workspace agrees."""
    w = I.make_workload(kind="q8", B=2, Hq=8, Hkv=2, d=128, L_max=4096, tile=64, seq_lens=[4096, 3001],
                        seed=11, sink=40.0)
    for tau in (1e-6, 1e-3):
        g2 = check_full(w, "q8", tau=tau, q8_path="two_pass")
        for path in ("cluster", "tensor_core"):
            g1 = check_full(w, "q8", tau=tau, q8_path=path)
            assert np.max(np.abs(g1["o"] - g2["o"])) <= TOL["q8"]
    r = oracle_run(w, "q8", tau=1e-6)
    r0 = oracle_run(w, "q8", tau=0.0)
    assert np.max(np.abs(r.o - r0.o)) > 0.0  # rows were skipped


Q8_TC = [
    # d, Hq, Hkv, B, L_max, lens, tile, S: clusters of up to 8 / 16 CTAs (the running-maximum exchange),
    # 3 heads per kv head (padded to 4), several splits, ragged tails, length 1
    (128, 4, 1, 1, 8192, [8192], 64, 1),
    (128, 8, 2, 2, 6000, [6000, 1234], 128, 1),
    (128, 12, 4, 2, 4096, [4096, 4000], 64, 3),
    (128, 4, 1, 3, 3000, [3000, 129, 1], 64, 2),
]


@pytest.mark.parametrize("case", Q8_TC, ids=lambda c: f"g{c[1] // c[2]}-B{c[3]}-L{c[4]}-T{c[6]}-S{c[7]}")
def test_q8_tensor_core_shapes(case):
    d, Hq, Hkv, B, L_max, lens, tile, S = case
    w = I.make_workload(kind="q8", B=B, Hq=Hq, Hkv=Hkv, d=d, L_max=L_max, tile=tile, num_splits=S,
                        seq_lens=lens, seed=91 + tile, gumbel_scale=4.0, sink=6.0)
    a = dict(eps_scale=2e-2, eps_dir=5e-3, patience=2, lanes=I.probe_lanes_strided(128, 16))
    for tau in (0.0, 1e-6, 1e-3):
        check_full(w, "q8", tau=tau, q8_path="tensor_core")
        check_art(w, "q8_art", tau=tau, art=a, q8_path="tensor_core")


def test_empty_splits_and_tiny_lengths():
    w = make_small("bf16", 128, 8, 2, 3, 300, [1, 63, 300], 64, 8)
    check_full(w)
    check_art(w, art=dict(eps_scale=1e-2, eps_dir=1e-3, patience=1, lanes=[0, 5, 77]))


def test_invalid_seq_len_sets_status_and_nan():
    w = make_small("bf16", 128, 8, 2, 2, 256, [256, 100], 64, 1)
    w.seq_lens[1] = 300  # > L_max
    dp = K.upload(w)
    K.decode(dp, "full")
    assert K.device_status(dp) == capi.ART_ERR_SEQLEN
    assert K.device_status(dp) == capi.ART_OK  # cleared on read
    o = dp.o.cpu().numpy()
    assert np.all(np.isnan(o[1])) and not np.any(np.isnan(o[0]))
    assert np.all(dp.tiles.cpu().numpy()[1] == 0)
    w.seq_lens[1] = 0
    dp = K.upload(w)
    K.decode(dp, "art")
    assert K.device_status(dp) == capi.ART_ERR_SEQLEN


def test_deterministic_and_stream():
    w = make_small("bf16", 128, 8, 2, 2, 3000, [3000, 1234], 64, 2, sink=6.0)
    dp = K.upload(w)
    s = torch.cuda.Stream()
    outs = []
    for mode in ("full", "art", "full", "art"):
        with torch.cuda.stream(s):
            K.decode(dp, mode, stream=s.cuda_stream)
        s.synchronize()
        outs.append((dp.o.cpu().numpy().copy(), dp.tiles.cpu().numpy().copy()))
    assert np.array_equal(outs[0][0], outs[2][0]) and np.array_equal(outs[1][0], outs[3][0])
    assert np.array_equal(outs[1][1], outs[3][1])


def test_unsupported_tile_returns_error():
    w = make_small("bf16", 128, 4, 1, 1, 1024, [1024], 256, 1)
    dp = K.upload(w)
    rc = K.decode(dp, "full", check=False)
    assert rc == capi.ART_ERR_UNSUPPORTED


Q8_ART_TWO_PASS = [
    # d, Hq, Hkv, B, L_max, lens, tile, S, n_probe, patience: the rule over per-tile records with more
    # than one round of its CTA (over 512 tiles in a split), 32 probe lanes (one lane per probe lane in
    # the probe pass, the wider rule kernel), 20 lanes, 3 heads per kv head, tile 32, splits
    (128, 4, 1, 1, 40960, [40960], 64, 1, 16, 1),
    (128, 8, 2, 2, 12288, [12288, 5001], 32, 2, 32, 2),
    (128, 6, 2, 1, 9000, [8999], 64, 3, 20, 3),
]


@pytest.mark.parametrize("case", Q8_ART_TWO_PASS, ids=lambda c: f"L{c[4]}-T{c[6]}-S{c[7]}-P{c[8]}-p{c[9]}")
def test_q8_art_two_pass_rounds_and_probe_widths(case):
    d, Hq, Hkv, B, L_max, lens, tile, S, n_probe, patience = case
    lanes = I.probe_lanes_strided(d, n_probe) if 128 % n_probe == 0 else [(7 * i) % d for i in range(n_probe)]
    w = I.make_workload(kind="q8", B=B, Hq=Hq, Hkv=Hkv, d=d, L_max=L_max, tile=tile, num_splits=S,
                        seq_lens=lens, seed=91 + n_probe, sink=6.0, gumbel_scale=2.0)
    # the workloads' thresholds (late stops), and thresholds that always hold with a patience of 600
    # (a split of more than 600 tiles stops at its 600th, in the rule kernel's second round)
    for art in (dict(eps_scale=1e-3, eps_dir=1e-4, patience=patience, lanes=lanes),
                dict(eps_scale=1e9, eps_dir=1e9, patience=600, lanes=lanes)):
        for tau in (1e-6, 1e-3):
            check_art(w, "q8_art", art=art, tau=tau, q8_path="two_pass")
