"""Shared test helpers: oracle runs, GPU runs through the C ABI, and the tile
acceptance rule for ART.

Acceptance (from the task's parity bar): tiles consumed must equal the
oracle's exactly, except that a tile whose oracle d_scale or d_direction lies
within WINDOW of its threshold may count as holding or not; the GPU's stop
tile is accepted if some such assignment, run through the patience rule,
yields it.  Outputs are then compared with the oracle re-run to the GPU's own
per-split stop tiles.
"""
import numpy as np

import oracle

WINDOW = 1e-4
# Lines the GPU tests want shown at the end of the pytest run (see conftest.py).
REPORT = []
TOL = {"f32": 1e-5, "bf16": 2e-3, "q8": 2e-3}
KIND = {"f32": oracle.KV_F32, "bf16": oracle.KV_BF16, "q8": oracle.KV_Q8}


def oracle_run(w, mode, *, num_splits=None, tile=None, forced_used=None, metrics=False, art=None, tau=None,
               n_threads=8, tile_order=None):
    a = (art or w.art) if mode in ("art", "q8_art") else None
    t = w.tau if tau is None else tau
    return oracle.decode(
        kind=KIND[w.kind], q=w.q, k=w.k, v=w.v, k_scale=w.k_scale, v_scale=w.v_scale, seq_lens=w.seq_lens,
        tile=w.tile if tile is None else tile, num_splits=w.num_splits if num_splits is None else num_splits,
        art=a, tau=(t if mode in ("q8", "q8_art") else 0.0), forced_used=forced_used,
        no_break=metrics and a is not None, want_metrics=metrics and a is not None, n_threads=n_threads,
        tile_order=tile_order,
    )


def _status(x, eps):
    if np.isnan(eps):
        return "above"
    if abs(x - eps) <= WINDOW:
        return "amb"
    return "below" if x < eps else "above"


def acceptable_used(metrics, eps_s, eps_d, patience):
    """Set of acceptable tile counts for one split, given oracle metrics [n_s, 2]."""
    accepted = set()
    reach = {0}
    n_s = metrics.shape[0]
    for t in range(n_s):
        s1 = _status(metrics[t, 0], eps_s)
        s2 = _status(metrics[t, 1], eps_d)
        can_hold = s1 != "above" and s2 != "above"
        can_fail = s1 != "below" or s2 != "below"
        nxt = set()
        for run in reach:
            if can_hold:
                if run + 1 >= patience:
                    accepted.add(t + 1)
                else:
                    nxt.add(run + 1)
            if can_fail:
                nxt.add(0)
        reach = nxt
        if not reach:
            break
    if reach:
        accepted.add(n_s)
    return accepted


def check_tiles(w, ref_metrics, gpu_used, art, tile, S):
    """Assert every (b, hq, split) GPU tile count is acceptable; return (#exact, #ambiguous-accepted)."""
    exact = amb = 0
    for b in range(w.B):
        L = int(w.seq_lens[b])
        n = -(-L // tile)
        for hq in range(w.Hq):
            for s in range(S):
                ta, tb = (s * n) // S, ((s + 1) * n) // S
                ok = acceptable_used(ref_metrics[b, hq, ta:tb], art["eps_scale"], art["eps_dir"], art["patience"])
                g = int(gpu_used[b, hq, s])
                assert g in ok, f"b={b} hq={hq} split={s}: gpu used {g} not in acceptable {sorted(ok)}"
                if len(ok) == 1:
                    exact += 1
                else:
                    amb += 1
    return exact, amb
