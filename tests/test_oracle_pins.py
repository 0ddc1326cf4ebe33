"""Pins for the CPU oracle (no GPU): the oracle is checked against things other
than itself -- brute-force softmax attention in extended precision, closed
forms, hand-worked probe values, invariants of attention, and numpy's own
bf16/fp16 decoders.

Method sources (web pages, cited by title and section):
  "Resumen Tecnico: ART" (gist.science, arXiv 2606.00024) S2.1-S2.4;
  "La paradoja de la eficiencia: como omitir redefine la velocidad de los LLM"
  (puntofijo.es), "La Elegancia de la Omision".
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from kv_cache_early_split_b200 import inputs as I

GOLD = os.path.join(os.path.dirname(__file__), "golden")
KIND = {"f32": oracle.KV_F32, "bf16": oracle.KV_BF16, "q8": oracle.KV_Q8}


# ---------------------------------------------------------------- helpers
def _decode_kv(w):
    """K, V, Q as float64 via numpy's own decoders (independent of the oracle's C code)."""
    if w.kind == "f32":
        return w.q.astype(np.float64), w.k.astype(np.float64), w.v.astype(np.float64)
    q = I.bf16_to_f32(w.q).astype(np.float64)
    if w.kind == "bf16":
        return q, I.bf16_to_f32(w.k).astype(np.float64), I.bf16_to_f32(w.v).astype(np.float64)
    ks = w.k_scale.view(np.float16).astype(np.float64)
    vs = w.v_scale.view(np.float16).astype(np.float64)
    k = w.k.astype(np.float64) * np.repeat(ks, 32, axis=-1)
    v = w.v.astype(np.float64) * np.repeat(vs, 32, axis=-1)
    return q, k, v


def brute(qv, K, V, idx):
    """softmax(q K[idx]^T / sqrt(d)) V[idx] in long double, global max, no tiling."""
    d = qv.shape[0]
    q = qv.astype(np.longdouble)
    Ks = K[idx].astype(np.longdouble)
    Vs = V[idx].astype(np.longdouble)
    s = Ks @ q / np.sqrt(np.longdouble(d))
    w = np.exp(s - s.max())
    return (w[:, None] * Vs).sum(axis=0) / w.sum()


def brute_all(w, tiles_per_split=None):
    """Brute force for every (b, hq); tiles_per_split[b,hq,s] limits split s to its first tiles
    (the number of splits is taken from its last axis)."""
    qd, kd, vd = _decode_kv(w)
    S = w.num_splits if tiles_per_split is None else tiles_per_split.shape[-1]
    G = w.G
    out = np.zeros((w.B, w.Hq, w.d), np.float64)
    for b in range(w.B):
        L = int(w.seq_lens[b])
        n = -(-L // w.tile)
        for hq in range(w.Hq):
            idx = []
            for s in range(S):
                ta, tb = (s * n) // S, ((s + 1) * n) // S
                if tiles_per_split is not None:
                    tb = min(tb, ta + int(tiles_per_split[b, hq, s]))
                idx.extend(range(ta * w.tile, min(tb * w.tile, L)))
            out[b, hq] = brute(qd[b, hq], kd[b, hq // G], vd[b, hq // G], np.array(idx))
    return out


def run(w, art=None, **kw):
    return oracle.decode(
        kind=KIND[w.kind], q=w.q, k=w.k, v=w.v, seq_lens=w.seq_lens, tile=w.tile,
        num_splits=kw.pop("num_splits", w.num_splits), k_scale=w.k_scale, v_scale=w.v_scale, art=art, **kw,
    )


def small(kind="bf16", **kw):
    base = dict(kind=kind, B=2, Hq=4, Hkv=2, d=8, L_max=100, tile=16, seed=7, seq_lens=[100, 37])
    base.update(kw)
    return I.make_workload(**base)


def _ev(expr):
    return float(eval(expr, {"sqrt": math.sqrt, "exp": math.exp}))


# ---------------------------------------------------------------- storage decoders
def test_bf16_decoder_matches_numpy_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        ref = I.bf16_to_f32(bits).astype(np.float64)
    got = np.array([oracle.bf16_to_double(b) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_f16_decoder_matches_numpy_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_double(b) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])  # includes subnormals, signed zeros, infinities


def test_q8_roundtrip_bound():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((64, 128)).astype(np.float32) * rng.lognormal(0, 2, (64, 1)).astype(np.float32)
    qi, sb = I.quantize_q8(x)
    s = np.repeat(sb.view(np.float16).astype(np.float64), 32, axis=-1)
    deq = qi.astype(np.float64) * s
    amax = np.repeat(np.abs(x.reshape(64, 4, 32)).max(-1), 32, axis=-1).astype(np.float64)
    # rounding to the code: s/2; fp16 rounding of the scale moves amax by <= 127*|s - amax/127|
    bound = s / 2 + 127 * np.abs(s - amax / 127) + 1e-12
    assert np.all(np.abs(x - deq) <= bound)
    assert np.all(np.abs(qi.astype(int)) <= 127)


# ---------------------------------------------------------------- full attention
@pytest.mark.parametrize("kind", ["f32", "bf16"])
@pytest.mark.parametrize("d,T", [(2, 1), (8, 7), (8, 16), (64, 64), (64, 7)])
def test_full_matches_bruteforce(kind, d, T):
    w = small(kind, d=d, tile=T, L_max=300, seq_lens=[300, 131], seed=11 + d + T)
    r = run(w)
    ref = brute_all(w)
    assert np.max(np.abs(r.o - ref)) <= 1e-12
    n = -(-w.seq_lens // T)
    assert np.array_equal(r.tiles, np.repeat(n[:, None], w.Hq, axis=1))


def test_full_matches_bruteforce_q8():
    w = small("q8", d=64, tile=16, L_max=120, seq_lens=[120, 57], seed=5)
    r = run(w)
    assert np.max(np.abs(r.o - brute_all(w))) <= 1e-12


def test_scaled_scores_golden():
    g = json.load(open(os.path.join(GOLD, "scaled_scores_two_positions.json")))
    q = np.array([[g["q"]]], np.float32)
    k = np.array([[g["k"]]], np.float32)
    v = np.array([[g["v"]]], np.float32)
    exp = np.array([_ev(e) for e in g["o"]])
    for T in (1, 2, 5):
        r = oracle.decode(kind=oracle.KV_F32, q=q, k=k, v=v, seq_lens=np.array([2]), tile=T)
        assert np.max(np.abs(r.o[0, 0] - exp)) <= 1e-15


def test_weights_sum_to_one():
    """V = 1 everywhere => O = 1 exactly up to rounding, for full, split and ART runs."""
    w = small("f32", d=8, seq_lens=[100, 61])
    w.v[:] = 1.0
    for kw in (dict(), dict(num_splits=3), dict(art=dict(eps_scale=np.inf, eps_dir=np.inf, patience=2, lanes=[0, 3]))):
        r = run(w, **kw)
        assert np.max(np.abs(r.o - 1.0)) <= 1e-14


def test_closed_forms():
    # L = 1 -> O = v0
    w = small("f32", seq_lens=[1, 1])
    r = run(w)
    assert np.max(np.abs(r.o - np.repeat(w.v[:, :, 0, :].astype(np.float64), 2, axis=1))) <= 1e-15
    # q = 0 -> mean of V
    w = small("f32", seq_lens=[100, 37])
    w.q[:] = 0
    r = run(w)
    for b, L in enumerate(w.seq_lens):
        mean = w.v[b, :, :L].astype(np.float64).mean(axis=1)
        assert np.max(np.abs(r.o[b] - np.repeat(mean, 2, axis=0))) <= 1e-13
    # identical keys -> mean of V
    w = small("f32", seq_lens=[100, 37])
    w.k[:] = w.k[:, :, :1, :]
    r = run(w)
    for b, L in enumerate(w.seq_lens):
        mean = w.v[b, :, :L].astype(np.float64).mean(axis=1)
        assert np.max(np.abs(r.o[b] - np.repeat(mean, 2, axis=0))) <= 1e-12
    # one key with a +50 logit dominates: O = its value row
    w = small("f32", d=8, seq_lens=[100, 37])
    w.q[:] = 0
    w.q[:, :, 0] = 1.0
    w.k[:] = 0
    w.k[:, :, 13, 0] = 50.0 * math.sqrt(8)
    r = run(w)
    assert np.max(np.abs(r.o - np.repeat(w.v[:, :, 13, :].astype(np.float64), 2, axis=1))) <= 1e-12


def test_split_invariance_full():
    w = small("bf16", d=64, L_max=300, tile=16, seq_lens=[300, 45])
    ref = run(w, num_splits=1)
    for S in range(2, 9):
        r = run(w, num_splits=S)
        assert np.max(np.abs(r.o - ref.o)) <= 1e-12
        assert np.array_equal(r.tiles, ref.tiles)
    # more splits than tiles: empty splits contribute nothing
    w1 = small("bf16", d=8, L_max=16, tile=16, seq_lens=[16, 3])
    r = run(w1, num_splits=5)
    assert np.max(np.abs(r.o - brute_all(w1))) <= 1e-12
    assert np.array_equal(r.tiles, np.ones((2, 4), np.int32))


def test_gqa_equals_mha_with_repeated_heads():
    w = small("bf16", d=64, Hq=8, Hkv=2, L_max=90, seq_lens=[90, 33])
    r = run(w)
    G = w.G
    wm = small("bf16", d=64, Hq=8, Hkv=2, L_max=90, seq_lens=[90, 33])
    wm.Hkv = 8
    wm.k = np.repeat(w.k, G, axis=1)
    wm.v = np.repeat(w.v, G, axis=1)
    rm = run(wm)
    assert np.max(np.abs(r.o - rm.o)) <= 1e-15


def test_tile_permutation_invariance_full():
    """S2.4: reordering KV tiles does not change full attention."""
    w = small("f32", d=8, L_max=96, tile=16, seq_lens=[96, 96])
    ref = run(w)
    perm = np.random.default_rng(1).permutation(6)
    idx = (perm[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)
    w.k = np.ascontiguousarray(w.k[:, :, idx])
    w.v = np.ascontiguousarray(w.v[:, :, idx])
    r = run(w)
    assert np.max(np.abs(r.o - ref.o)) <= 1e-13


# ---------------------------------------------------------------- ART rule
def test_art_hand_example_golden():
    g = json.load(open(os.path.join(GOLD, "art_probe_hand_example.json")))
    q = np.array([[g["q"]]], np.float32)
    k = np.array([[g["k"]]], np.float32)
    v = np.array([[g["v"]]], np.float32)
    L = len(g["v"])
    base = dict(kind=oracle.KV_F32, q=q, k=k, v=v, seq_lens=np.array([L]), tile=1)
    art = dict(eps_scale=0.0, eps_dir=0.0, patience=1, lanes=g["lanes"])
    r = oracle.decode(**base, art=art, want_metrics=True)
    assert np.max(np.abs(r.metrics[0, 0, :, 0] - [_ev(e) for e in g["d_scale"]])) <= 1e-14
    assert np.max(np.abs(r.metrics[0, 0, :, 1] - [_ev(e) for e in g["d_dir"]])) <= 1e-14
    r1 = oracle.decode(**base, art=dict(art, lanes=[1]), want_metrics=True)
    assert np.max(np.abs(r1.metrics[0, 0, :, 0] - [_ev(e) for e in g["lane1_d_scale"]])) <= 1e-14
    assert np.max(np.abs(r1.metrics[0, 0, :, 1] - [_ev(e) for e in g["lane1_d_dir"]])) <= 1e-14
    # lane order does not matter
    r2 = oracle.decode(**base, art=dict(art, lanes=g["lanes"][::-1]), want_metrics=True)
    assert np.allclose(r2.metrics, r.metrics, rtol=0, atol=1e-15)
    for c in g["cases"]:
        a = dict(eps_scale=float(c["eps_scale"]), eps_dir=float(c["eps_dir"]), patience=c["patience"], lanes=c["lanes"])
        rc = oracle.decode(**base, art=a)
        assert rc.tiles[0, 0] == c["tiles"], c
        assert np.max(np.abs(rc.o[0, 0] - [_ev(e) for e in c["o"]])) <= 1e-14, c


def test_art_eps_zero_is_full_attention():
    w = small("bf16", d=64, L_max=300, tile=16, seq_lens=[300, 47])
    full = run(w)
    for S in (1, 3):
        r = run(w, art=dict(eps_scale=0.0, eps_dir=0.0, patience=1, lanes=[0, 5, 9]), num_splits=S)
        assert np.array_equal(r.tiles, full.tiles)
        assert np.max(np.abs(r.o - full.o)) <= 1e-12


@pytest.mark.parametrize("S", [1, 2, 4])
@pytest.mark.parametrize("p", [1, 2, 5, 100])
def test_art_eps_inf_stops_after_patience_tiles(S, p):
    """+inf thresholds hold on every tile; tile 0 is processed first (S2.4), so each split stops after min(p, len)."""
    w = small("bf16", d=64, L_max=300, tile=16, seq_lens=[300, 47])
    r = run(w, art=dict(eps_scale=np.inf, eps_dir=np.inf, patience=p, lanes=[1, 2]), num_splits=S)
    for b, L in enumerate(w.seq_lens):
        n = -(-int(L) // 16)
        lens = [((s + 1) * n) // S - (s * n) // S for s in range(S)]
        assert np.all(r.used[b] == np.array([min(p, ln) for ln in lens])[None, :])
        assert np.all(r.tiles[b] == sum(min(p, ln) for ln in lens))
    assert np.max(np.abs(r.o - brute_all(w, r.used))) <= 1e-12


def test_art_nan_threshold_never_holds():
    w = small("f32", d=8, seq_lens=[100, 37])
    r = run(w, art=dict(eps_scale=np.nan, eps_dir=np.inf, patience=1, lanes=[0]))
    assert np.array_equal(r.tiles, run(w).tiles)


def test_art_v_scale_invariance():
    """Scaling V by c scales every d_scale by |c| and leaves d_direction unchanged."""
    w = small("f32", d=8, L_max=200, tile=8, seq_lens=[200, 77], seed=21)
    art = dict(eps_scale=0.05, eps_dir=2e-3, patience=2, lanes=[0, 2, 4, 7])
    r = run(w, art=art, want_metrics=True, no_break=True)
    c = -4.0
    w.v = w.v * np.float32(c)
    r2 = run(w, art=dict(art, eps_scale=art["eps_scale"] * abs(c)), want_metrics=True, no_break=True)
    m1, m2 = r.metrics, r2.metrics
    ok = ~np.isnan(m1[..., 0])
    assert np.allclose(m2[..., 0][ok], abs(c) * m1[..., 0][ok], rtol=1e-12, atol=1e-14)
    assert np.allclose(m2[..., 1][ok], m1[..., 1][ok], rtol=1e-9, atol=1e-13)
    assert np.array_equal(r.tiles, r2.tiles)
    assert np.max(np.abs(r2.o - c * r.o)) <= 1e-12


def test_art_forced_and_no_break_consistency():
    w = small("bf16", d=64, L_max=400, tile=8, seq_lens=[400, 150], seed=9)
    art = dict(eps_scale=0.02, eps_dir=5e-3, patience=1, lanes=list(range(0, 64, 8)))
    r = run(w, art=art, num_splits=2)
    assert np.any(r.tiles < -(-w.seq_lens[:, None] // 8)), "case should stop early somewhere"
    rf = run(w, forced_used=r.used, num_splits=2)
    assert np.max(np.abs(rf.o - r.o)) <= 1e-15
    assert np.array_equal(rf.used, r.used)
    rn = run(w, art=art, num_splits=2, no_break=True, want_metrics=True)
    assert np.array_equal(rn.used, r.used)
    assert np.max(np.abs(rn.o - r.o)) <= 1e-15
    n = -(-w.seq_lens // 8)
    for b in range(w.B):  # metrics cover every tile of the sequence
        assert not np.any(np.isnan(rn.metrics[b, :, : n[b]]))
    assert np.max(np.abs(r.o - brute_all(w, r.used))) <= 1e-12
    # the rule itself, replayed from the recorded metrics (patience 1: first hold)
    for b in range(w.B):
        nb = int(n[b])
        for hq in range(w.Hq):
            for s in range(2):
                ta, tb = (s * nb) // 2, ((s + 1) * nb) // 2
                m = rn.metrics[b, hq, ta:tb]
                hold = (m[:, 0] < art["eps_scale"]) & (m[:, 1] < art["eps_dir"])
                exp_used = int(np.argmax(hold)) + 1 if hold.any() else tb - ta
                assert r.used[b, hq, s] == exp_used


# ---------------------------------------------------------------- V skip (q8)
def _skip_case(tau):
    w = I.make_workload(kind="q8", B=1, Hq=4, Hkv=1, d=64, L_max=512, tile=32, seed=4, gumbel_scale=6.0, q_scale=2.0)
    r = oracle.decode(kind=oracle.KV_Q8, q=w.q, k=w.k, v=w.v, k_scale=w.k_scale, v_scale=w.v_scale,
                      seq_lens=w.seq_lens, tile=w.tile, tau=tau)
    return w, r


def test_vskip_tau_zero_is_full():
    w, r = _skip_case(0.0)
    assert np.max(np.abs(r.o - brute_all(w))) <= 1e-12


def test_vskip_tau_above_one_skips_everything():
    _, r = _skip_case(2.0)
    assert np.max(np.abs(r.o)) == 0.0


def test_vskip_error_bound():
    """|O_skip - O| <= sum over skipped rows of p_j |v_j| / l (elementwise), with the skip set
    rebuilt here from the definition: p_j = exp(s_j - m'), m' the running max after j's tile."""
    tau = 1e-3
    w, r = _skip_case(tau)
    q, K, V = _decode_kv(w)
    T, L, d = w.tile, int(w.seq_lens[0]), w.d
    nskipped = 0
    for hq in range(w.Hq):
        s = (K[0, 0, :L] @ q[0, hq]) / math.sqrt(d)
        tile_max = np.array([s[t:t + T].max() for t in range(0, L, T)])
        run_max = np.maximum.accumulate(tile_max)
        mprime = np.repeat(run_max, T)[:L]
        p_run = np.exp(s - mprime)
        skipped = p_run < tau
        nskipped += int(skipped.sum())
        pw = np.exp(s - s.max())
        bound = (pw[skipped, None] * np.abs(V[0, 0, :L][skipped])).sum(axis=0) / pw.sum()
        full = brute(q[0, hq], K[0, 0], V[0, 0], np.arange(L))
        assert np.all(np.abs(r.o[0, hq] - full) <= bound + 1e-12)
        # and the skipped part is exactly what is missing
        kept = ~skipped
        exp_o = (pw[kept, None] * V[0, 0, :L][kept]).sum(axis=0) / pw.sum()
        assert np.max(np.abs(r.o[0, hq] - exp_o)) <= 1e-12
    assert nskipped > 0, "the case must actually skip rows"


def test_vskip_record_matches_definition():
    """The oracle's per-row record p / tau (the numerator test of the V skip) against p_j rebuilt
    from the definition as above; rows past the sequence are NaN."""
    tau = 1e-3
    w = I.make_workload(kind="q8", B=1, Hq=4, Hkv=1, d=64, L_max=512, tile=32, seed=4, gumbel_scale=6.0, q_scale=2.0,
                        seq_lens=[449])
    r = oracle.decode(kind=oracle.KV_Q8, q=w.q, k=w.k, v=w.v, k_scale=w.k_scale, v_scale=w.v_scale,
                      seq_lens=w.seq_lens, tile=w.tile, tau=tau, want_vskip=True)
    q, K, V = _decode_kv(w)
    T, L, d = w.tile, int(w.seq_lens[0]), w.d
    for hq in range(w.Hq):
        s = (K[0, 0, :L] @ q[0, hq]) / math.sqrt(d)
        run_max = np.maximum.accumulate(np.array([s[t:t + T].max() for t in range(0, L, T)]))
        p_run = np.exp(s - np.repeat(run_max, T)[:L])
        assert np.allclose(r.vskip[0, hq, :L], p_run / tau, rtol=1e-9, atol=0.0)
        assert np.all(np.isnan(r.vskip[0, hq, L:]))
    assert np.any(r.vskip[0, :, :L] < 1.0) and np.any(r.vskip[0, :, :L] >= 1.0)


def test_vskip_record_is_the_skip_set():
    """With one query head per kv head, leaving a row out of the numerator is the same as zeroing
    its V row: the output with the skip equals the output without it on V with the recorded rows
    (p / tau < 1) zeroed, exactly."""
    tau = 3e-3
    w = I.make_workload(kind="q8", B=2, Hq=3, Hkv=3, d=64, L_max=384, tile=32, seed=9, gumbel_scale=5.0, q_scale=2.0,
                        seq_lens=[384, 301], num_splits=2)
    r = oracle.decode(kind=oracle.KV_Q8, q=w.q, k=w.k, v=w.v, k_scale=w.k_scale, v_scale=w.v_scale,
                      seq_lens=w.seq_lens, tile=w.tile, num_splits=2, tau=tau, want_vskip=True)
    v0 = w.v.copy()
    mask = r.vskip < 1.0  # [B, Hq = Hkv, L_max]; NaN compares False
    assert mask.sum() > 0
    v0[mask] = 0
    r0 = oracle.decode(kind=oracle.KV_Q8, q=w.q, k=w.k, v=v0, k_scale=w.k_scale, v_scale=w.v_scale,
                       seq_lens=w.seq_lens, tile=w.tile, num_splits=2, tau=0.0)
    assert np.array_equal(r.o, r0.o)


def test_named_workloads_shapes():
    for name in I.WORKLOADS:
        w = I.workload(name, keys_b=[0], keys_h=[0])
        assert w.Hq == w.G and w.k.shape[:2] == (1, 1)
    w = I.workload("split_b16_h32x8_d128_Lvar", keys_b=[0, 5], keys_h=[3])
    assert np.all((w.seq_lens >= 8192) & (w.seq_lens <= 65536))
